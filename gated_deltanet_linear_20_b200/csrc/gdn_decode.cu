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
// of the warp's rows, and the gate (VG: the per-column log decays of the
// lane's 16 columns; else the one log decay of the head).
template <bool VG>
struct Tok {
  uint4 k0, k1, q0, q1, v;
  float4 gv[VG ? 4 : 1];
  float g, beta;
};
template <bool VG>
__device__ __forceinline__ Tok<VG> load_tok(const DecodeArgs& a, size_t tok, int c0, int row0) {
  Tok<VG> t;
  const uint4* kp = reinterpret_cast<const uint4*>(a.k + tok * D + c0);
  const uint4* qp = reinterpret_cast<const uint4*>(a.q + tok * D + c0);
  t.k0 = kp[0];
  t.k1 = kp[1];
  t.q0 = qp[0];
  t.q1 = qp[1];
  t.v = *reinterpret_cast<const uint4*>(a.v + tok * D + row0);
  if constexpr (VG) {
    const float4* gp = reinterpret_cast<const float4*>(a.g + tok * D + c0);
#pragma unroll
    for (int e = 0; e < 4; ++e) t.gv[e] = gp[e];
    t.g = 0.f;
  } else {
    t.g = a.g[tok];
  }
  t.beta = a.beta[tok];
  return t;
}

// Burst kernel (T > 1): eight lanes per row.  PRE: q / k normalisation or a q
// scale is requested (a separate instantiation keeps the plain one lean).
// VG: per-channel gate (alpha_j = exp(g_j) per key column j): the decay is
// applied column by column, S_i <- S_i diag(alpha) + d_i k with
// d_i = beta (v_i - (S_i diag(alpha)) . k), so the row dot products take the
// decayed k and q, and o_i = (S_i diag(alpha)) . q + d_i (k . q).
template <bool PRE, bool VG>
__global__ void __launch_bounds__(WARPS * 32, VG ? 4 : 5) decode_burst_kernel(const DecodeArgs a) {
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

  Tok<VG> cur = load_tok<VG>(a, size_t(b) * a.T * a.H + h, c0, row0);
#pragma unroll 1
  for (int t = 0; t < a.T; ++t) {
    const size_t tok = (size_t(b) * a.T + t) * a.H + h;  // [B][T][H] index of (b, t, h)
    Tok<VG> nxt = cur;
    if (t + 1 < a.T) nxt = load_tok<VG>(a, tok + a.H, c0, row0);
    float k[16], q[16], v[8];
    bf16x8_to_float(cur.k0, *reinterpret_cast<float(*)[8]>(k));
    bf16x8_to_float(cur.k1, *reinterpret_cast<float(*)[8]>(k + 8));
    bf16x8_to_float(cur.q0, *reinterpret_cast<float(*)[8]>(q));
    bf16x8_to_float(cur.q1, *reinterpret_cast<float(*)[8]>(q + 8));
    bf16x8_to_float(cur.v, v);
    const float alpha = VG ? 1.f : expf(cur.g);
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

    // VG: the state is decayed in place, column by column (S <- S diag(alpha)),
    // before the row dot products; the scalar decay is applied to the dot
    // products and folded into the update instead
    if constexpr (VG) {
#pragma unroll
      for (int e4 = 0; e4 < 4; ++e4) {
        const float4 gv = cur.gv[e4];
        const float c0 = expf(gv.x), c1 = expf(gv.y), c2 = expf(gv.z), c3 = expf(gv.w);
#pragma unroll
        for (int i = 0; i < RG; ++i) {
          s[i][e4].x *= c0;
          s[i][e4].y *= c1;
          s[i][e4].z *= c2;
          s[i][e4].w *= c3;
        }
      }
    }
    const float a_row = VG ? 1.f : alpha;

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
      const float d = beta * (v[4 * i + sub] - a_row * sk[i]);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if constexpr (VG) {  // already decayed
          s[i][e].x = fmaf(d, k[4 * e], s[i][e].x);
          s[i][e].y = fmaf(d, k[4 * e + 1], s[i][e].y);
          s[i][e].z = fmaf(d, k[4 * e + 2], s[i][e].z);
          s[i][e].w = fmaf(d, k[4 * e + 3], s[i][e].w);
        } else {
          s[i][e].x = fmaf(alpha, s[i][e].x, d * k[4 * e]);
          s[i][e].y = fmaf(alpha, s[i][e].y, d * k[4 * e + 1]);
          s[i][e].z = fmaf(alpha, s[i][e].z, d * k[4 * e + 2]);
          s[i][e].w = fmaf(alpha, s[i][e].w, d * k[4 * e + 3]);
        }
      }
      if ((lane & 7) == 0) {
        const float ov = fmaf(a_row, sq[i], d * kq);
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

// Step kernel (used for T = 1, correct for any T): the state rows of a head
// of dim DH (Dk = Dv = DH) are split into groups of DH / 4 lanes, lane l holding
// columns 4 (l % (DH/4)) .. +3 of one row, so one warp-wide load covers whole
// rows contiguously (one row of 512 bytes at DH = 128, two rows of 256 bytes
// at DH = 64).  Each lane issues LOADS state loads before any arithmetic; the
// rows are updated in registers and stored after the last token.  Measured on
// B200 against the burst layout and against storing each row as soon as it is
// updated, this form streams a 64 MiB state fastest for a single token.  At
// DH = 64 a CTA covers a whole head (64 rows).
__device__ __forceinline__ float4 bf16x4_to_float4(uint2 raw) {
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
  return make_float4(a.x, a.y, b.x, b.y);
}
__device__ __forceinline__ float dot44(const float4& a, const float4& b) {
  return fmaf(a.x, b.x, fmaf(a.y, b.y, fmaf(a.z, b.z, a.w * b.w)));
}

template <int DH>
struct StepGeom {
  static constexpr int LPR = DH / 4;                    // lanes per row (32 or 16)
  static constexpr int RPI = 32 / LPR;                  // rows per warp-wide load (1 or 2)
  static constexpr int LOADS = 8;                       // state loads per lane
  static constexpr int ROWS_PER_WARP = LOADS * RPI;     // 8 or 16
  static constexpr int ROWS_PER_CTA = ROWS_PER_WARP * WARPS;
  static constexpr int CTAS_PER_HEAD = DH / ROWS_PER_CTA;  // 4 or 1
  static_assert(CTAS_PER_HEAD * ROWS_PER_CTA == DH, "rows must tile the head");
};

template <int DH, bool PRE, bool VG>
__global__ void __launch_bounds__(WARPS * 32, 7) decode_step_kernel(const DecodeArgs a) {
  using G = StepGeom<DH>;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int sub = lane / G::LPR;  // row within a warp-wide load
  const int cl = lane % G::LPR;   // columns 4 cl .. 4 cl + 3
  const int head = blockIdx.x / G::CTAS_PER_HEAD;  // b * H + h
  const int b = head / a.H, h = head - b * a.H;
  const int row0 = (blockIdx.x % G::CTAS_PER_HEAD) * G::ROWS_PER_CTA + warp * G::ROWS_PER_WARP;

  // s[i]: row row0 + i RPI + sub
  float4* srow = reinterpret_cast<float4*>(a.S + (size_t(head) * DH + row0 + sub) * DH) + cl;
  float4 s[G::LOADS];
#pragma unroll
  for (int i = 0; i < G::LOADS; ++i) s[i] = __ldcs(srow + i * G::RPI * (DH / 4));

#pragma unroll 1
  for (int t = 0; t < a.T; ++t) {
    const size_t tok = (size_t(b) * a.T + t) * a.H + h;  // [B][T][H] index of (b, t, h)
    float4 k4 = bf16x4_to_float4(*reinterpret_cast<const uint2*>(a.k + tok * DH + 4 * cl));
    float4 q4 = bf16x4_to_float4(*reinterpret_cast<const uint2*>(a.q + tok * DH + 4 * cl));
    // v of the warp's rows: 8 (DH = 128) or 16 (DH = 64) bf16
    uint32_t vw[G::ROWS_PER_WARP / 2];
#pragma unroll
    for (int j = 0; j < G::ROWS_PER_WARP / 8; ++j) {
      const uint4 raw = *reinterpret_cast<const uint4*>(a.v + tok * DH + row0 + 8 * j);
      vw[4 * j] = raw.x;
      vw[4 * j + 1] = raw.y;
      vw[4 * j + 2] = raw.z;
      vw[4 * j + 3] = raw.w;
    }
    float4 g4 = make_float4(0.f, 0.f, 0.f, 0.f);
    if constexpr (VG) g4 = *reinterpret_cast<const float4*>(a.g + tok * DH + 4 * cl);
    const float alpha = VG ? 1.f : expf(a.g[tok]);
    const float beta = a.beta[tok];
    if (PRE && a.qk_norm) {  // x^ = x / sqrt(sum x^2 + 1e-6) over Dk (the lanes of a row)
      float kk = dot44(k4, k4), qq = dot44(q4, q4);
#pragma unroll
      for (int off = G::LPR / 2; off > 0; off >>= 1) {
        kk += __shfl_xor_sync(0xffffffffu, kk, off);
        qq += __shfl_xor_sync(0xffffffffu, qq, off);
      }
      const float kn = rsqrtf(kk + 1e-6f), qn = rsqrtf(qq + 1e-6f) * a.q_scale;
      k4 = make_float4(k4.x * kn, k4.y * kn, k4.z * kn, k4.w * kn);
      q4 = make_float4(q4.x * qn, q4.y * qn, q4.z * qn, q4.w * qn);
    } else if (PRE) {
      q4 = make_float4(q4.x * a.q_scale, q4.y * a.q_scale, q4.z * a.q_scale, q4.w * a.q_scale);
    }

    // the decay of the lane's 4 columns, and k, q as the row dot products take
    // them (decayed per column with VG; the scalar decay goes on the products)
    float4 sc = make_float4(alpha, alpha, alpha, alpha), kd = k4, qd = q4;
    if constexpr (VG) {
      sc = make_float4(expf(g4.x), expf(g4.y), expf(g4.z), expf(g4.w));
      kd = make_float4(sc.x * k4.x, sc.y * k4.y, sc.z * k4.z, sc.w * k4.w);
      qd = make_float4(sc.x * q4.x, sc.y * q4.y, sc.z * q4.z, sc.w * q4.w);
    }
    const float a_row = VG ? 1.f : alpha;

    float kq = dot44(k4, q4);
#pragma unroll
    for (int off = G::LPR / 2; off > 0; off >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);
    float sk[G::LOADS], sq[G::LOADS];
#pragma unroll
    for (int i = 0; i < G::LOADS; ++i) {
      sk[i] = dot44(s[i], kd);
      sq[i] = dot44(s[i], qd);
    }
#pragma unroll
    for (int off = G::LPR / 2; off > 0; off >>= 1) {
#pragma unroll
      for (int i = 0; i < G::LOADS; ++i) {
        sk[i] += __shfl_xor_sync(0xffffffffu, sk[i], off);
        sq[i] += __shfl_xor_sync(0xffffffffu, sq[i], off);
      }
    }
    float o_mine = 0.f;
#pragma unroll
    for (int i = 0; i < G::LOADS; ++i) {
      // v of row i RPI + sub: bf16 number i (RPI = 1), or half `sub` of word i
      const uint32_t w = vw[(i * G::RPI) / 2];
      const uint32_t bits = G::RPI == 1 ? ((i & 1) ? (w >> 16) : (w & 0xffffu))
                                        : (sub ? (w >> 16) : (w & 0xffffu));
      const float vi = __uint_as_float(bits << 16);  // bf16 -> fp32 is exact
      const float d = beta * (vi - a_row * sk[i]);
      s[i].x = fmaf(sc.x, s[i].x, d * k4.x);
      s[i].y = fmaf(sc.y, s[i].y, d * k4.y);
      s[i].z = fmaf(sc.z, s[i].z, d * k4.z);
      s[i].w = fmaf(sc.w, s[i].w, d * k4.w);
      const float o = fmaf(a_row, sq[i], d * kq);
      if (cl == i) o_mine = o;
    }
    if (cl < G::LOADS) {  // lane (sub, cl) holds o of row cl RPI + sub
      const size_t oi = tok * DH + row0 + cl * G::RPI + sub;
      if (a.o_bf16)
        reinterpret_cast<__nv_bfloat16*>(a.o)[oi] = __float2bfloat16_rn(o_mine);
      else
        a.o[oi] = o_mine;
    }
  }
#pragma unroll
  for (int i = 0; i < G::LOADS; ++i) __stcs(srow + i * G::RPI * (DH / 4), s[i]);
}

}  // namespace

int launch_decode(const DecodeArgs& a, cudaStream_t stream) {
  const long long heads = (long long)a.B * a.H;
  if (heads == 0) return 0;
  const bool pre = a.qk_norm || a.q_scale != 1.f;
  if (a.head_dim == 64) {  // the step kernel at any T
    const unsigned grid = unsigned(heads * StepGeom<64>::CTAS_PER_HEAD);
    if (a.vector_gate) {
      if (pre)
        decode_step_kernel<64, true, true><<<grid, WARPS * 32, 0, stream>>>(a);
      else
        decode_step_kernel<64, false, true><<<grid, WARPS * 32, 0, stream>>>(a);
    } else {
      if (pre)
        decode_step_kernel<64, true, false><<<grid, WARPS * 32, 0, stream>>>(a);
      else
        decode_step_kernel<64, false, false><<<grid, WARPS * 32, 0, stream>>>(a);
    }
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
  }
  if (a.head_dim != D) return -1;
  const unsigned grid_step = unsigned(heads * StepGeom<D>::CTAS_PER_HEAD);
  const unsigned grid_burst = unsigned(heads * CTAS_PER_HEAD);
  if (a.vector_gate) {
    if (a.T == 1) {
      if (pre)
        decode_step_kernel<D, true, true><<<grid_step, WARPS * 32, 0, stream>>>(a);
      else
        decode_step_kernel<D, false, true><<<grid_step, WARPS * 32, 0, stream>>>(a);
    } else {
      if (pre)
        decode_burst_kernel<true, true><<<grid_burst, WARPS * 32, 0, stream>>>(a);
      else
        decode_burst_kernel<false, true><<<grid_burst, WARPS * 32, 0, stream>>>(a);
    }
  } else if (a.T == 1) {
    if (pre)
      decode_step_kernel<D, true, false><<<grid_step, WARPS * 32, 0, stream>>>(a);
    else
      decode_step_kernel<D, false, false><<<grid_step, WARPS * 32, 0, stream>>>(a);
  } else {
    if (pre)
      decode_burst_kernel<true, false><<<grid_burst, WARPS * 32, 0, stream>>>(a);
    else
      decode_burst_kernel<false, false><<<grid_burst, WARPS * 32, 0, stream>>>(a);
  }
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace gdn
