// Delta rule with a per-channel gate (KDA): the decay alpha_t = exp(g_t) is a
// vector over the key channels instead of a scalar, applied where the scalar
// gate of the gated delta rule is (the variant that the ROCmFPX gated-delta-net
// prefill note, bittide.aicompass.dev article d2880479, lists among the cases
// its fused kernel left to the old path):
//
//   S_t = S_{t-1} diag(alpha_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,  o_t = S_t q_t,
//
// S in R^{Dv x Dk} stored [Dv][Dk].  Row i of S (a value channel) evolves on its
// own given the token's k, q, alpha and beta:
//   s'  = s o alpha                  (the decay, column by column)
//   d   = beta (v_i - s' . k)        (delta-rule residual)
//   s  <- s' + d k
//   o_i = s . q = s' . q + d (k . q)
// so the rows are split over warps and CTAs and each row walks the tokens in
// fp32 registers: one kernel for prefill (S0 -> S_T) and for decode (S in place),
// exact in the order of the recurrence.  The per-channel decay breaks the
// scalar-gate factorisation that lets the chunked tensor-core kernel apply
// decays as per-token diagonal factors; a chunked form needs Q o Lambda,
// K o Lambda and K / Lambda as rescaled MMA operands.
//
// Layout of a CTA: 4 warps; a warp holds RG groups of 4 rows; the 8 lanes of a
// row hold float4 column blocks j, j+8, j+16, j+24 (j = lane % 8), so the lanes
// of a row read 128 contiguous bytes per access, from global memory and from
// shared memory alike.  Tokens are staged 16 at a time with cp.async into a
// double buffer (k, q, g, v of this CTA's rows, beta); one cooperative pass per
// chunk turns them into fp32 k, q, alpha = exp(g) and k . q in shared memory,
// so each exp is taken once per CTA and not once per row.
#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int D = 128;
constexpr int NT = 16;        // tokens per staged chunk
constexpr int WARPS = 4;
constexpr int THREADS = WARPS * 32;

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ float dot44(const float4& a, const float4& b) {
  return fmaf(a.x, b.x, fmaf(a.y, b.y, fmaf(a.z, b.z, a.w * b.w)));
}

template <int RG>
struct Shape {
  static constexpr int ROWS_PER_WARP = 4 * RG;
  static constexpr int ROWS_PER_CTA = WARPS * ROWS_PER_WARP;  // 16 or 32
  static constexpr int CTAS_PER_HEAD = D / ROWS_PER_CTA;      // 8 or 4
  // staging buffer (cp.async target), bytes
  static constexpr int R_K = 0;
  static constexpr int R_Q = R_K + NT * D * 2;
  static constexpr int R_G = R_Q + NT * D * 2;
  static constexpr int R_V = R_G + NT * D * 4;
  static constexpr int R_B = R_V + NT * ROWS_PER_CTA * 2;
  static constexpr int R_BYTES = R_B + NT * 4;
  // converted chunk, bytes
  static constexpr int C_K = 2 * R_BYTES;
  static constexpr int C_Q = C_K + NT * D * 4;
  static constexpr int C_A = C_Q + NT * D * 4;
  static constexpr int C_KQ = C_A + NT * D * 4;
  static constexpr int SMEM = C_KQ + NT * 4;
  static_assert(R_BYTES % 16 == 0 && C_K % 16 == 0, "16-byte staging pieces");
};

// Issue the copies of tokens t0 .. t0+n-1 of chain (b, h) into one staging buffer.
template <int RG>
__device__ __forceinline__ void stage_chunk(const KdaArgs& a, uint8_t* buf, int b, int h, int t0,
                                            int n, int vrow0) {
  using S = Shape<RG>;
  const int tid = threadIdx.x;
  const uint32_t base = smem_addr(buf);
  auto tok = [&](int j) { return (size_t(b) * a.T + t0 + j) * a.H + h; };  // [B][T][H] index
  for (int p = tid; p < n * 16; p += THREADS) {  // k, q: 16 pieces of 16 B per token
    const int j = p >> 4, c = p & 15;
    const size_t e = tok(j) * D + c * 8;
    cp16(base + S::R_K + j * 256 + c * 16, a.k + e);
    cp16(base + S::R_Q + j * 256 + c * 16, a.q + e);
  }
  for (int p = tid; p < n * 32; p += THREADS) {  // g: 32 pieces per token
    const int j = p >> 5, c = p & 31;
    cp16(base + S::R_G + j * 512 + c * 16, a.g + tok(j) * D + c * 4);
  }
  constexpr int VP = S::ROWS_PER_CTA / 8;  // v of this CTA's rows: 2 or 4 pieces per token
  for (int p = tid; p < n * VP; p += THREADS) {
    const int j = p / VP, c = p % VP;
    cp16(base + S::R_V + j * S::ROWS_PER_CTA * 2 + c * 16, a.v + tok(j) * D + vrow0 + c * 8);
  }
  for (int p = tid; p < n; p += THREADS) cp4(base + S::R_B + p * 4, a.beta + tok(p));
  cp_commit();
}

template <int RG>
__global__ void __launch_bounds__(THREADS) kda_kernel(const KdaArgs a) {
  using S = Shape<RG>;
  extern __shared__ __align__(16) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int head = blockIdx.x / S::CTAS_PER_HEAD;  // b * H + h
  const int b = head / a.H, h = head - b * a.H;
  const int vrow0 = (blockIdx.x % S::CTAS_PER_HEAD) * S::ROWS_PER_CTA;
  const int j8 = lane & 7, sub = lane >> 3;
  const int wrow = warp * S::ROWS_PER_WARP + sub;  // this lane's first row within the CTA

  // rows vrow0 + wrow + 4 i, column blocks j8 + 8 m
  float4 s[RG][4];
  const size_t srow = (size_t(head) * D + vrow0 + wrow) * D;
  if (a.S_in) {
    const float4* src = reinterpret_cast<const float4*>(a.S_in + srow);
#pragma unroll
    for (int i = 0; i < RG; ++i)
#pragma unroll
      for (int m = 0; m < 4; ++m) s[i][m] = __ldcs(src + i * D + j8 + 8 * m);  // +4 rows = i*4*D/4
  } else {
#pragma unroll
    for (int i = 0; i < RG; ++i)
#pragma unroll
      for (int m = 0; m < 4; ++m) s[i][m] = make_float4(0.f, 0.f, 0.f, 0.f);
  }

  const int nch = (a.T + NT - 1) / NT;
  if (nch > 0) stage_chunk<RG>(a, smem, b, h, 0, min(NT, a.T), vrow0);
  const float4* ck = reinterpret_cast<const float4*>(smem + S::C_K);
  const float4* cq = reinterpret_cast<const float4*>(smem + S::C_Q);
  const float4* ca = reinterpret_cast<const float4*>(smem + S::C_A);
  const float* ckq = reinterpret_cast<const float*>(smem + S::C_KQ);

#pragma unroll 1
  for (int c = 0; c < nch; ++c) {
    const int t0 = c * NT, n = min(NT, a.T - t0);
    uint8_t* raw = smem + (c & 1) * S::R_BYTES;
    if (c + 1 < nch) {
      stage_chunk<RG>(a, smem + ((c + 1) & 1) * S::R_BYTES, b, h, t0 + NT, min(NT, a.T - t0 - NT),
                      vrow0);
      cp_wait<1>();
    } else {
      cp_wait<0>();
    }
    __syncthreads();
    // convert: warp w takes tokens w, w+4, ..; lane l columns 4l .. 4l+3
    for (int j = warp; j < n; j += WARPS) {
      const uint2 kr = reinterpret_cast<const uint2*>(raw + S::R_K + j * 256)[lane];
      const uint2 qr = reinterpret_cast<const uint2*>(raw + S::R_Q + j * 256)[lane];
      const float4 gv = reinterpret_cast<const float4*>(raw + S::R_G + j * 512)[lane];
      const float2 k01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&kr.x));
      const float2 k23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&kr.y));
      const float2 q01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&qr.x));
      const float2 q23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&qr.y));
      const float4 kf = make_float4(k01.x, k01.y, k23.x, k23.y);
      const float4 qf = make_float4(q01.x, q01.y, q23.x, q23.y);
      reinterpret_cast<float4*>(smem + S::C_K)[j * 32 + lane] = kf;
      reinterpret_cast<float4*>(smem + S::C_Q)[j * 32 + lane] = qf;
      reinterpret_cast<float4*>(smem + S::C_A)[j * 32 + lane] =
          make_float4(expf(gv.x), expf(gv.y), expf(gv.z), expf(gv.w));
      float kq = dot44(kf, qf);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);
      if (lane == 0) reinterpret_cast<float*>(smem + S::C_KQ)[j] = kq;
    }
    __syncthreads();

    const __nv_bfloat16* rv = reinterpret_cast<const __nv_bfloat16*>(raw + S::R_V);
    const float* rb = reinterpret_cast<const float*>(raw + S::R_B);
#pragma unroll 2
    for (int j = 0; j < n; ++j) {
      float4 kk[4], qq[4], aa[4];
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        kk[m] = ck[j * 32 + j8 + 8 * m];
        qq[m] = cq[j * 32 + j8 + 8 * m];
        aa[m] = ca[j * 32 + j8 + 8 * m];
      }
      const float kq = ckq[j], beta = rb[j];
      float sk[RG], sq[RG];
#pragma unroll
      for (int i = 0; i < RG; ++i) {
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          s[i][m].x *= aa[m].x;
          s[i][m].y *= aa[m].y;
          s[i][m].z *= aa[m].z;
          s[i][m].w *= aa[m].w;
        }
        sk[i] = (dot44(s[i][0], kk[0]) + dot44(s[i][1], kk[1])) +
                (dot44(s[i][2], kk[2]) + dot44(s[i][3], kk[3]));
        sq[i] = (dot44(s[i][0], qq[0]) + dot44(s[i][1], qq[1])) +
                (dot44(s[i][2], qq[2]) + dot44(s[i][3], qq[3]));
      }
#pragma unroll
      for (int off = 1; off < 8; off <<= 1)
#pragma unroll
        for (int i = 0; i < RG; ++i) {
          sk[i] += __shfl_xor_sync(0xffffffffu, sk[i], off);
          sq[i] += __shfl_xor_sync(0xffffffffu, sq[i], off);
        }
      const size_t orow = ((size_t(b) * a.T + t0 + j) * a.H + h) * D + vrow0 + wrow;
#pragma unroll
      for (int i = 0; i < RG; ++i) {
        const float d = beta * (__bfloat162float(rv[j * S::ROWS_PER_CTA + wrow + 4 * i]) - sk[i]);
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          s[i][m].x = fmaf(d, kk[m].x, s[i][m].x);
          s[i][m].y = fmaf(d, kk[m].y, s[i][m].y);
          s[i][m].z = fmaf(d, kk[m].z, s[i][m].z);
          s[i][m].w = fmaf(d, kk[m].w, s[i][m].w);
        }
        if (j8 == 0) a.o[orow + 4 * i] = fmaf(d, kq, sq[i]);
      }
    }
    __syncthreads();  // the converted chunk and this staging buffer are reused
  }

  float4* dst = reinterpret_cast<float4*>(a.S_out + srow);
#pragma unroll
  for (int i = 0; i < RG; ++i)
#pragma unroll
    for (int m = 0; m < 4; ++m) __stcs(dst + i * D + j8 + 8 * m, s[i][m]);
}

}  // namespace

int kda_rows_per_cta(long long heads, int num_sms) {
  // one CTA per SM at most when the chains are few (16 rows per CTA spreads
  // them over more SMs); 32 rows per CTA otherwise, which halves the staging
  // and conversion work per row
  return heads * Shape<1>::CTAS_PER_HEAD <= num_sms ? Shape<1>::ROWS_PER_CTA : Shape<2>::ROWS_PER_CTA;
}

int launch_kda(const KdaArgs& a, int num_sms, cudaStream_t stream) {
  const long long heads = (long long)a.B * a.H;
  if (heads == 0) return 0;
  if (kda_rows_per_cta(heads, num_sms) == Shape<1>::ROWS_PER_CTA) {
    if (!ensure_smem_attr(reinterpret_cast<const void*>(&kda_kernel<1>), 9, Shape<1>::SMEM)) return -1;
    kda_kernel<1><<<unsigned(heads * Shape<1>::CTAS_PER_HEAD), THREADS, Shape<1>::SMEM, stream>>>(a);
  } else {
    if (!ensure_smem_attr(reinterpret_cast<const void*>(&kda_kernel<2>), 10, Shape<2>::SMEM)) return -1;
    kda_kernel<2><<<unsigned(heads * Shape<2>::CTAS_PER_HEAD), THREADS, Shape<2>::SMEM, stream>>>(a);
  }
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace gdn
