// Gated-delta-rule decode step: one token per sequence, the fp32 state read
// and written once, in place.  This is the per-layer recurrence that the
// Megakernel of the Lucebox contribution guide (discosf.com/news/5165879,
// section 4) runs inside its fused decode; here it is one memory-bound kernel.
//
// Per state row i (the Dv index) of head (b, h), with alpha = exp(g), beta:
//   sk   = S_i . k,   sq = S_i . q                 (two dot products over Dk)
//   d_i  = beta (v_i - alpha sk)                    (delta-rule residual)
//   S_i <- alpha S_i + d_i k                        (= alpha S_i (I - beta k k^T) + beta v_i k^T)
//   o_i  = S_i . q = alpha sq + d_i (k . q)
// Each warp owns ROWS_PER_WARP = 8 consecutive rows.  Eight lanes share a row:
// lane l holds columns 16 (l % 8) .. +15 of rows 4 i + l / 8 (i = 0, 1), so a
// warp load covers four 128-byte row segments, and a dot product over a row
// reduces over 8 lanes (3 shuffle steps; 15 shuffles per token and lane).  All
// row loads are issued before any reduction, with the streaming cache hint:
// the state is touched once per call.  A call may carry T >= 1 tokens per
// sequence (a short burst, e.g. verifying a few speculated tokens): the rows
// stay in registers across the tokens and the next token's inputs are loaded
// while the current one is applied, so the state crosses HBM once per burst.
#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int D = 128;
constexpr int ROWS_PER_WARP = 8;
constexpr int WARPS = 4;
constexpr int ROWS_PER_CTA = ROWS_PER_WARP * WARPS;  // 32
constexpr int CTAS_PER_HEAD = D / ROWS_PER_CTA;      // 4
constexpr int RG = ROWS_PER_WARP / 4;                // row groups per lane (2)

__device__ __forceinline__ void bf16x8_to_float(uint4 raw, float (&f)[8]) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[e]));
    f[2 * e] = x.x;
    f[2 * e + 1] = x.y;
  }
}

__device__ __forceinline__ float dot4(const float4& a, const float* b) {
  return fmaf(a.x, b[0], fmaf(a.y, b[1], fmaf(a.z, b[2], a.w * b[3])));
}

// Inputs of one token for this lane: 16 columns of k and q, the 8 v entries
// of the warp's rows, and the gate.
struct Tok {
  uint4 k0, k1, q0, q1, v;
  float g, beta;
};
__device__ __forceinline__ Tok load_tok(const DecodeArgs& a, size_t tok, int c0, int row0) {
  Tok t;
  const uint4* kp = reinterpret_cast<const uint4*>(a.k + tok * D + c0);
  const uint4* qp = reinterpret_cast<const uint4*>(a.q + tok * D + c0);
  t.k0 = kp[0];
  t.k1 = kp[1];
  t.q0 = qp[0];
  t.q1 = qp[1];
  t.v = *reinterpret_cast<const uint4*>(a.v + tok * D + row0);
  t.g = a.g[tok];
  t.beta = a.beta[tok];
  return t;
}

// Burst kernel (T > 1): eight lanes per row.  PRE: q / k normalisation or a q
// scale is requested (a separate instantiation keeps the plain one lean).
template <bool PRE>
__global__ void __launch_bounds__(WARPS * 32) decode_burst_kernel(const DecodeArgs a) {
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int head = blockIdx.x / CTAS_PER_HEAD;  // b * H + h
  const int b = head / a.H, h = head - b * a.H;
  const int row0 = (blockIdx.x % CTAS_PER_HEAD) * ROWS_PER_CTA + warp * ROWS_PER_WARP;
  const int sub = lane >> 3;        // row within a group of 4
  const int c0 = 16 * (lane & 7);   // first column of this lane

  // rows row0 + 4 i + sub, columns c0 .. c0+15
  float4* srow = reinterpret_cast<float4*>(a.S + (size_t(head) * D + row0 + sub) * D + c0);
  float4 s[RG][4];
#pragma unroll
  for (int i = 0; i < RG; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) s[i][e] = __ldcs(srow + i * D + e);  // + 4 rows = i * 4 * D / 4

  Tok cur = load_tok(a, size_t(b) * a.T * a.H + h, c0, row0);
#pragma unroll 1
  for (int t = 0; t < a.T; ++t) {
    const size_t tok = (size_t(b) * a.T + t) * a.H + h;  // [B][T][H] index of (b, t, h)
    Tok nxt = cur;
    if (t + 1 < a.T) nxt = load_tok(a, tok + a.H, c0, row0);
    float k[16], q[16], v[8];
    bf16x8_to_float(cur.k0, *reinterpret_cast<float(*)[8]>(k));
    bf16x8_to_float(cur.k1, *reinterpret_cast<float(*)[8]>(k + 8));
    bf16x8_to_float(cur.q0, *reinterpret_cast<float(*)[8]>(q));
    bf16x8_to_float(cur.q1, *reinterpret_cast<float(*)[8]>(q + 8));
    bf16x8_to_float(cur.v, v);
    const float alpha = expf(cur.g);
    const float beta = cur.beta;
    if (PRE && a.qk_norm) {  // x^ = x / sqrt(sum x^2 + 1e-6) over Dk (8 lanes of the row)
      float kk = 0.f, qq = 0.f;
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        kk = fmaf(k[e], k[e], kk);
        qq = fmaf(q[e], q[e], qq);
      }
#pragma unroll
      for (int off = 1; off < 8; off <<= 1) {
        kk += __shfl_xor_sync(0xffffffffu, kk, off);
        qq += __shfl_xor_sync(0xffffffffu, qq, off);
      }
      const float kn = rsqrtf(kk + 1e-6f), qn = rsqrtf(qq + 1e-6f) * a.q_scale;
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        k[e] *= kn;
        q[e] *= qn;
      }
    } else if (PRE) {
#pragma unroll
      for (int e = 0; e < 16; ++e) q[e] *= a.q_scale;
    }

    float kq = 0.f, sk[RG], sq[RG];
#pragma unroll
    for (int e = 0; e < 16; ++e) kq = fmaf(k[e], q[e], kq);
#pragma unroll
    for (int i = 0; i < RG; ++i) {
      sk[i] = dot4(s[i][0], k) + dot4(s[i][1], k + 4) + dot4(s[i][2], k + 8) + dot4(s[i][3], k + 12);
      sq[i] = dot4(s[i][0], q) + dot4(s[i][1], q + 4) + dot4(s[i][2], q + 8) + dot4(s[i][3], q + 12);
    }
#pragma unroll
    for (int off = 1; off < 8; off <<= 1) {
      kq += __shfl_xor_sync(0xffffffffu, kq, off);
#pragma unroll
      for (int i = 0; i < RG; ++i) {
        sk[i] += __shfl_xor_sync(0xffffffffu, sk[i], off);
        sq[i] += __shfl_xor_sync(0xffffffffu, sq[i], off);
      }
    }
#pragma unroll
    for (int i = 0; i < RG; ++i) {
      const float d = beta * (v[4 * i + sub] - alpha * sk[i]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        s[i][e].x = fmaf(alpha, s[i][e].x, d * k[4 * e]);
        s[i][e].y = fmaf(alpha, s[i][e].y, d * k[4 * e + 1]);
        s[i][e].z = fmaf(alpha, s[i][e].z, d * k[4 * e + 2]);
        s[i][e].w = fmaf(alpha, s[i][e].w, d * k[4 * e + 3]);
      }
      if ((lane & 7) == 0) {
        const float ov = fmaf(alpha, sq[i], d * kq);
        const size_t oi = tok * D + row0 + 4 * i + sub;
        if (a.o_bf16)
          reinterpret_cast<__nv_bfloat16*>(a.o)[oi] = __float2bfloat16_rn(ov);
        else
          a.o[oi] = ov;
      }
    }
    cur = nxt;
  }
#pragma unroll
  for (int i = 0; i < RG; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) __stcs(srow + i * D + e, s[i][e]);
}

// Step kernel (used for T = 1, correct for any T): a whole warp per row, lane
// l holding columns 4l .. 4l+3 (one 512-byte access per row), the rows updated
// in registers and stored after the last token.  Measured on B200 against the
// burst layout and against storing each row as soon as it is updated, this
// form streams a 64 MiB state fastest for a single token.
__device__ __forceinline__ float4 bf16x4_to_float4(uint2 raw) {
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
  return make_float4(a.x, a.y, b.x, b.y);
}
__device__ __forceinline__ float dot44(const float4& a, const float4& b) {
  return fmaf(a.x, b.x, fmaf(a.y, b.y, fmaf(a.z, b.z, a.w * b.w)));
}

template <bool PRE>
__global__ void __launch_bounds__(WARPS * 32) decode_step_kernel(const DecodeArgs a) {
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int head = blockIdx.x / CTAS_PER_HEAD;  // b * H + h
  const int b = head / a.H, h = head - b * a.H;
  const int row0 = (blockIdx.x % CTAS_PER_HEAD) * ROWS_PER_CTA + warp * ROWS_PER_WARP;

  float4* srow = reinterpret_cast<float4*>(a.S + (size_t(head) * D + row0) * D) + lane;
  float4 s[ROWS_PER_WARP];
#pragma unroll
  for (int r = 0; r < ROWS_PER_WARP; ++r) s[r] = __ldcs(srow + r * (D / 4));

#pragma unroll 1
  for (int t = 0; t < a.T; ++t) {
    const size_t tok = (size_t(b) * a.T + t) * a.H + h;  // [B][T][H] index of (b, t, h)
    float4 k4 = bf16x4_to_float4(*reinterpret_cast<const uint2*>(a.k + tok * D + 4 * lane));
    float4 q4 = bf16x4_to_float4(*reinterpret_cast<const uint2*>(a.q + tok * D + 4 * lane));
    const uint4 vraw = *reinterpret_cast<const uint4*>(a.v + tok * D + row0);
    const float alpha = expf(a.g[tok]);
    const float beta = a.beta[tok];
    if (PRE && a.qk_norm) {  // x^ = x / sqrt(sum x^2 + 1e-6) over Dk (the whole warp)
      float kk = dot44(k4, k4), qq = dot44(q4, q4);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        kk += __shfl_xor_sync(0xffffffffu, kk, off);
        qq += __shfl_xor_sync(0xffffffffu, qq, off);
      }
      const float kn = rsqrtf(kk + 1e-6f), qn = rsqrtf(qq + 1e-6f) * a.q_scale;
      k4 = make_float4(k4.x * kn, k4.y * kn, k4.z * kn, k4.w * kn);
      q4 = make_float4(q4.x * qn, q4.y * qn, q4.z * qn, q4.w * qn);
    } else if (PRE) {
      q4 = make_float4(q4.x * a.q_scale, q4.y * a.q_scale, q4.z * a.q_scale, q4.w * a.q_scale);
    }

    float kq = dot44(k4, q4);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);
    float sk[ROWS_PER_WARP], sq[ROWS_PER_WARP];
#pragma unroll
    for (int r = 0; r < ROWS_PER_WARP; ++r) {
      sk[r] = dot44(s[r], k4);
      sq[r] = dot44(s[r], q4);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
#pragma unroll
      for (int r = 0; r < ROWS_PER_WARP; ++r) {
        sk[r] += __shfl_xor_sync(0xffffffffu, sk[r], off);
        sq[r] += __shfl_xor_sync(0xffffffffu, sq[r], off);
      }
    }
    const __nv_bfloat16* vv = reinterpret_cast<const __nv_bfloat16*>(&vraw);
    float o_mine = 0.f;
#pragma unroll
    for (int r = 0; r < ROWS_PER_WARP; ++r) {
      const float d = beta * (__bfloat162float(vv[r]) - alpha * sk[r]);
      s[r].x = fmaf(alpha, s[r].x, d * k4.x);
      s[r].y = fmaf(alpha, s[r].y, d * k4.y);
      s[r].z = fmaf(alpha, s[r].z, d * k4.z);
      s[r].w = fmaf(alpha, s[r].w, d * k4.w);
      const float o = fmaf(alpha, sq[r], d * kq);
      if (lane == r) o_mine = o;
    }
    if (lane < ROWS_PER_WARP) {
      if (a.o_bf16)
        reinterpret_cast<__nv_bfloat16*>(a.o)[tok * D + row0 + lane] = __float2bfloat16_rn(o_mine);
      else
        a.o[tok * D + row0 + lane] = o_mine;
    }
  }
#pragma unroll
  for (int r = 0; r < ROWS_PER_WARP; ++r) __stcs(srow + r * (D / 4), s[r]);
}

}  // namespace

int launch_decode(const DecodeArgs& a, cudaStream_t stream) {
  const long long heads = (long long)a.B * a.H;
  if (heads == 0) return 0;
  const unsigned grid = unsigned(heads * CTAS_PER_HEAD);
  const bool pre = a.qk_norm || a.q_scale != 1.f;
  if (a.T == 1) {
    if (pre)
      decode_step_kernel<true><<<grid, WARPS * 32, 0, stream>>>(a);
    else
      decode_step_kernel<false><<<grid, WARPS * 32, 0, stream>>>(a);
  } else {
    if (pre)
      decode_burst_kernel<true><<<grid, WARPS * 32, 0, stream>>>(a);
    else
      decode_burst_kernel<false><<<grid, WARPS * 32, 0, stream>>>(a);
  }
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace gdn
