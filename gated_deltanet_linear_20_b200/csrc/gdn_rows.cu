// Row-parallel fp32 recurrence: every head dim the chunked tensor-core kernel
// does not cover (Dk, Dv in {64, 128, 256}, Dk != Dv included; the ROCmFPX
// gated-delta-net prefill note, bittide.aicompass.dev article d2880479, lists
// other head dims among the cases its fused kernel left to the old path), and
// the per-channel gate (KDA, listed there too) at every head dim.
//
//   S_t = S_{t-1} diag(alpha_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,  o_t = S_t q_t,
//
// with alpha_t = exp(g_t) a vector over the Dk key channels (per-channel gate)
// or the same scalar on every channel (the gated delta rule).  S in R^{Dv x Dk}
// is stored [Dv][Dk].  Row i of S (a value channel) evolves on its own given
// the token's k, q, alpha and beta:
//   s'  = s o alpha                  (the decay, column by column)
//   d   = beta (v_i - s' . k)        (delta-rule residual)
//   s  <- s' + d k
//   o_i = s . q = s' . q + d (k . q)
// so the rows are split over warps and CTAs and each row walks the tokens in
// fp32 registers, in the order of the recurrence: one kernel for prefill
// (S0 -> S_T) and decode (S in place).
//
// Layout of a CTA: 4 warps; LPR lanes share a row (the launches use LPR = 8:
// a row's dot products take 3 shuffle steps), so a warp holds 32/LPR rows per
// group and RG groups; the lanes of a row hold the float4 column blocks j,
// j+LPR, j+2 LPR, .. (j = lane % LPR, Dk/(4 LPR) blocks), so they touch 128
// contiguous bytes per access, in global and in shared memory alike.  Many
// chains take two row groups per warp (fewer instructions per row), few take
// one (more SMs busy).
// Tokens are staged NT at a time with cp.async into a double buffer (k, q, g,
// this CTA's v rows, beta); one cooperative pass per chunk turns them into
// fp32 k, q, alpha = exp(g) and the token-only scalars below in shared memory,
// so each exp is taken once per CTA and not once per row.  A single token
// (decode) skips the staging: each lane reads its blocks straight from global
// memory.
//
// With the scalar gate the tokens are applied in pairs (t, t+1), so that one
// reduction serves both: with s' = alpha_t s and u = alpha_{t+1} s',
//   d_t     = beta_t (v_t - s'.k_t),                   o_t = s'.q_t + d_t (k_t.q_t)
//   d_{t+1} = beta_{t+1} (v_{t+1} - u.k_{t+1} - d_t c),
//   o_{t+1} = u.q_{t+1} + d_t e + d_{t+1} (k_{t+1}.q_{t+1}),
//   s      <- u + d_t alpha_{t+1} k_t + d_{t+1} k_{t+1}
// where c = alpha_{t+1} k_t.k_{t+1} and e = alpha_{t+1} k_t.q_{t+1} depend on
// the tokens only.  The four dot products s'.k_t, s'.q_t, u.k_{t+1},
// u.q_{t+1} reduce together, so the dependency chain through the lanes'
// shuffles is taken once per two tokens (measured 15-25% faster on few
// chains).  With the per-channel gate the same form needs the vector
// k_t o alpha_{t+1} as a seventh operand and measured no faster, so those
// tokens are applied one at a time.
#include "gdn_internal.h"

namespace gdn {
namespace {

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
__device__ __forceinline__ float4 bf16x4(uint2 raw) {
  const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
  const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
  return make_float4(a.x, a.y, b.x, b.y);
}
__device__ __forceinline__ float4 mul4(const float4& s, const float4& a) {
  return make_float4(s.x * a.x, s.y * a.y, s.z * a.z, s.w * a.w);
}
__device__ __forceinline__ float4 mul4(const float4& s, float a) {
  return make_float4(s.x * a, s.y * a, s.z * a, s.w * a);
}
__device__ __forceinline__ float4 fma4(float d, const float4& k, const float4& s) {
  return make_float4(fmaf(d, k.x, s.x), fmaf(d, k.y, s.y), fmaf(d, k.z, s.z), fmaf(d, k.w, s.w));
}
constexpr int round16(int x) { return (x + 15) / 16 * 16; }

// Sum of v[0..N) by pairs (a tree, so that the partial dot products do not
// form one long dependency chain).
template <int N>
__device__ __forceinline__ float tree_sum(const float (&v)[N]) {
  if constexpr (N == 1) {
    return v[0];
  } else {
    float h[(N + 1) / 2];
#pragma unroll
    for (int i = 0; i < N / 2; ++i) h[i] = v[2 * i] + v[2 * i + 1];
    if constexpr (N % 2) h[N / 2] = v[N - 1];
    return tree_sum<(N + 1) / 2>(h);
  }
}

template <int DK, bool VG, int LPR, int RG>
struct Shape {
  static constexpr int MB = DK / (4 * LPR);           // float4 column blocks per lane
  static constexpr int RSTEP = 32 / LPR;              // rows per group in a warp
  static constexpr int NT = (VG ? 1536 : 2048) / DK;  // tokens per staged chunk
  static constexpr int ROWS_PER_WARP = RSTEP * RG;
  static constexpr int ROWS_PER_CTA = WARPS * ROWS_PER_WARP;  // 8, 16 or 32
  // staging buffer (cp.async target), bytes
  static constexpr int R_K = 0;
  static constexpr int R_Q = R_K + NT * DK * 2;
  static constexpr int R_G = R_Q + NT * DK * 2;
  static constexpr int R_V = R_G + round16(VG ? NT * DK * 4 : NT * 4);
  static constexpr int R_B = R_V + NT * ROWS_PER_CTA * 2;
  static constexpr int R_BYTES = round16(R_B + NT * 4);
  // converted chunk, bytes
  static constexpr int C_K = 2 * R_BYTES;
  static constexpr int C_Q = C_K + NT * DK * 4;
  static constexpr int C_A = C_Q + NT * DK * 4;
  static constexpr int C_KQ = C_A + round16(VG ? NT * DK * 4 : NT * 4);
  static constexpr int NP = NT / 2;                   // token pairs per chunk
  static constexpr int C_C = C_KQ + round16(NT * 4);  // c per pair (scalar gate)
  static constexpr int C_E = C_C + round16(NP * 4);   // e per pair (scalar gate)
  static constexpr int SMEM = C_E + round16(NP * 4);
  static_assert(MB >= 1 && (NT * DK * 2) % 16 == 0 && NT % 2 == 0, "16-byte pieces, whole pairs");
};

template <typename S, int DK, bool VG>
__device__ __forceinline__ void stage_chunk(const RowArgs& a, uint8_t* buf, int b, int h, int t0,
                                            int n, int vrow0) {
  const int tid = threadIdx.x;
  const uint32_t base = smem_addr(buf);
  auto tok = [&](int j) { return (size_t(b) * a.T + t0 + j) * a.H + h; };  // [B][T][H] index
  constexpr int KP = DK / 8;  // 16-byte pieces of a bf16 row of k or q
  for (int p = tid; p < n * KP; p += THREADS) {
    const int j = p / KP, c = p % KP;
    const size_t e = tok(j) * DK + c * 8;
    cp16(base + S::R_K + j * DK * 2 + c * 16, a.k + e);
    cp16(base + S::R_Q + j * DK * 2 + c * 16, a.q + e);
  }
  if constexpr (VG) {
    constexpr int GP = DK / 4;  // 16-byte pieces of an fp32 gate row
    for (int p = tid; p < n * GP; p += THREADS) {
      const int j = p / GP, c = p % GP;
      cp16(base + S::R_G + j * DK * 4 + c * 16, a.g + tok(j) * DK + c * 4);
    }
  } else {
    for (int p = tid; p < n; p += THREADS) cp4(base + S::R_G + p * 4, a.g + tok(p));
  }
  constexpr int VP = S::ROWS_PER_CTA / 8;  // this CTA's v rows: 1, 2 or 4 pieces per token
  for (int p = tid; p < n * VP; p += THREADS) {
    const int j = p / VP, c = p % VP;
    cp16(base + S::R_V + j * S::ROWS_PER_CTA * 2 + c * 16, a.v + tok(j) * a.Dv + vrow0 + c * 8);
  }
  for (int p = tid; p < n; p += THREADS) cp4(base + S::R_B + p * 4, a.beta + tok(p));
  cp_commit();
}

// One token on this lane's rows.  kk, qq: k and q blocks; aa: the decay
// blocks (per-channel gate) or aa[0].x the decay (scalar gate); kq: k . q, or
// a lane's partial of it when KQ_PARTIAL (reduced here with sk and sq).
template <int MB, bool VG, int LPR, int RG, bool KQ_PARTIAL>
__device__ __forceinline__ void apply_token(float4 (&s)[RG][MB], const float4 (&kk)[MB],
                                            const float4 (&qq)[MB], const float4 (&aa)[VG ? MB : 1],
                                            float kq, float beta, const float (&v)[RG],
                                            float (&o)[RG]) {
  float sk[RG], sq[RG];
#pragma unroll
  for (int i = 0; i < RG; ++i) {
    float pk[MB], pq[MB];
#pragma unroll
    for (int m = 0; m < MB; ++m) {
      s[i][m] = VG ? mul4(s[i][m], aa[m]) : mul4(s[i][m], aa[0].x);
      pk[m] = dot44(s[i][m], kk[m]);
      pq[m] = dot44(s[i][m], qq[m]);
    }
    sk[i] = tree_sum(pk);
    sq[i] = tree_sum(pq);
  }
#pragma unroll
  for (int off = 1; off < LPR; off <<= 1) {
#pragma unroll
    for (int i = 0; i < RG; ++i) {
      sk[i] += __shfl_xor_sync(0xffffffffu, sk[i], off);
      sq[i] += __shfl_xor_sync(0xffffffffu, sq[i], off);
    }
    if constexpr (KQ_PARTIAL) kq += __shfl_xor_sync(0xffffffffu, kq, off);
  }
#pragma unroll
  for (int i = 0; i < RG; ++i) {
    const float d = beta * (v[i] - sk[i]);
#pragma unroll
    for (int m = 0; m < MB; ++m) s[i][m] = fma4(d, kk[m], s[i][m]);
    o[i] = fmaf(d, kq, sq[i]);
  }
}

// DIRECT: a single token per chain (decode), read straight from global memory.
template <int DK, bool VG, int LPR, int RG, bool DIRECT>
__global__ void __launch_bounds__(THREADS) rows_kernel(const RowArgs a) {
  using S = Shape<DK, VG, LPR, RG>;
  constexpr int MB = S::MB, RS = S::RSTEP;
  extern __shared__ __align__(16) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ctas_per_head = a.Dv / S::ROWS_PER_CTA;
  const int head = blockIdx.x / ctas_per_head;  // b * H + h
  const int b = head / a.H, h = head - b * a.H;
  const int vrow0 = (blockIdx.x % ctas_per_head) * S::ROWS_PER_CTA;
  const int j8 = lane % LPR, sub = lane / LPR;
  const int wrow = warp * S::ROWS_PER_WARP + sub;  // this lane's first row within the CTA

  // rows vrow0 + wrow + RS i, column blocks j8 + LPR m
  float4 s[RG][MB];
  const size_t srow = (size_t(head) * a.Dv + vrow0 + wrow) * DK;
  if (a.S_in) {
    const float4* src = reinterpret_cast<const float4*>(a.S_in + srow);
#pragma unroll
    for (int i = 0; i < RG; ++i)
#pragma unroll
      for (int m = 0; m < MB; ++m) s[i][m] = __ldcs(src + i * RS * DK / 4 + j8 + LPR * m);
  } else {
#pragma unroll
    for (int i = 0; i < RG; ++i)
#pragma unroll
      for (int m = 0; m < MB; ++m) s[i][m] = make_float4(0.f, 0.f, 0.f, 0.f);
  }

  if constexpr (DIRECT) {
#pragma unroll 1
    for (int t = 0; t < a.T; ++t) {
      const size_t tok = (size_t(b) * a.T + t) * a.H + h;
      float4 kk[MB], qq[MB], aa[VG ? MB : 1];
      float kq = 0.f;
#pragma unroll
      for (int m = 0; m < MB; ++m) {
        kk[m] = bf16x4(*reinterpret_cast<const uint2*>(a.k + tok * DK + 4 * (j8 + LPR * m)));
        qq[m] = bf16x4(*reinterpret_cast<const uint2*>(a.q + tok * DK + 4 * (j8 + LPR * m)));
        kq += dot44(kk[m], qq[m]);
        if constexpr (VG) {
          const float4 gv = *reinterpret_cast<const float4*>(a.g + tok * DK + 4 * (j8 + LPR * m));
          aa[m] = make_float4(expf(gv.x), expf(gv.y), expf(gv.z), expf(gv.w));
        }
      }
      if constexpr (!VG) aa[0].x = expf(a.g[tok]);
      float v[RG], o[RG];
#pragma unroll
      for (int i = 0; i < RG; ++i) v[i] = __bfloat162float(a.v[tok * a.Dv + vrow0 + wrow + RS * i]);
      apply_token<MB, VG, LPR, RG, true>(s, kk, qq, aa, kq, a.beta[tok], v, o);
      if (j8 == 0) {
#pragma unroll
        for (int i = 0; i < RG; ++i) a.o[tok * a.Dv + vrow0 + wrow + RS * i] = o[i];
      }
    }
  } else {
    const int nch = (a.T + S::NT - 1) / S::NT;
    if (nch > 0) stage_chunk<S, DK, VG>(a, smem, b, h, 0, min(S::NT, a.T), vrow0);
    const float4* ck = reinterpret_cast<const float4*>(smem + S::C_K);
    const float4* cq = reinterpret_cast<const float4*>(smem + S::C_Q);
    const float* caf = reinterpret_cast<const float*>(smem + S::C_A);
    const float* ckq = reinterpret_cast<const float*>(smem + S::C_KQ);
#pragma unroll 1
    for (int c = 0; c < nch; ++c) {
      const int t0 = c * S::NT, n = min(S::NT, a.T - t0);
      uint8_t* raw = smem + (c & 1) * S::R_BYTES;
      if (c + 1 < nch) {
        stage_chunk<S, DK, VG>(a, smem + ((c + 1) & 1) * S::R_BYTES, b, h, t0 + S::NT,
                               min(S::NT, a.T - t0 - S::NT), vrow0);
        cp_wait<1>();
      } else {
        cp_wait<0>();
      }
      __syncthreads();
      // convert: warp w takes the token pairs w, w+4, .. (several at once, so
      // that their loads, exps and reductions overlap; Dk = 256 one at a time,
      // its wider rows would spill); lane l holds columns CPL l .. CPL l + CPL - 1.
      // A last odd token is a pair without its second token.
      constexpr int CPL = DK / 32, PAIRS = CPL / 2;
      constexpr int PPW = DK == 256 ? 1 : (S::NP + WARPS - 1) / WARPS;
      const int npairs = (n + 1) / 2;
      for (int p0 = warp; p0 < npairs; p0 += WARPS * PPW) {
        constexpr int NR = VG ? 2 : 4;
        float r[PPW][4];  // k0.q0, k1.q1 and (scalar gate) k0.k1, k0.q1 partials
#pragma unroll
        for (int u = 0; u < PPW; ++u) {
          const int pp = p0 + WARPS * u;
          r[u][0] = r[u][1] = r[u][2] = r[u][3] = 0.f;
          if (pp < npairs) {
            const int t0 = 2 * pp, t1 = t0 + 1;
            const bool two = t1 < n;
            const __nv_bfloat162* k0r = reinterpret_cast<const __nv_bfloat162*>(raw + S::R_K + t0 * DK * 2);
            const __nv_bfloat162* q0r = reinterpret_cast<const __nv_bfloat162*>(raw + S::R_Q + t0 * DK * 2);
#pragma unroll
            for (int e = 0; e < PAIRS; ++e) {
              const int c2 = lane * PAIRS + e;  // float2 index within a token row
              const float2 k0 = __bfloat1622float2(k0r[c2]);
              const float2 q0 = __bfloat1622float2(q0r[c2]);
              reinterpret_cast<float2*>(smem + S::C_K)[t0 * DK / 2 + c2] = k0;
              reinterpret_cast<float2*>(smem + S::C_Q)[t0 * DK / 2 + c2] = q0;
              r[u][0] = fmaf(k0.x, q0.x, fmaf(k0.y, q0.y, r[u][0]));
              if constexpr (VG) {
                const float2 g0 = reinterpret_cast<const float2*>(raw + S::R_G + t0 * DK * 4)[c2];
                reinterpret_cast<float2*>(smem + S::C_A)[t0 * DK / 2 + c2] =
                    make_float2(expf(g0.x), expf(g0.y));
              }
              if (two) {
                const float2 k1 = __bfloat1622float2(
                    reinterpret_cast<const __nv_bfloat162*>(raw + S::R_K + t1 * DK * 2)[c2]);
                const float2 q1 = __bfloat1622float2(
                    reinterpret_cast<const __nv_bfloat162*>(raw + S::R_Q + t1 * DK * 2)[c2]);
                reinterpret_cast<float2*>(smem + S::C_K)[t1 * DK / 2 + c2] = k1;
                reinterpret_cast<float2*>(smem + S::C_Q)[t1 * DK / 2 + c2] = q1;
                r[u][1] = fmaf(k1.x, q1.x, fmaf(k1.y, q1.y, r[u][1]));
                if constexpr (VG) {
                  const float2 g1 = reinterpret_cast<const float2*>(raw + S::R_G + t1 * DK * 4)[c2];
                  reinterpret_cast<float2*>(smem + S::C_A)[t1 * DK / 2 + c2] =
                      make_float2(expf(g1.x), expf(g1.y));
                } else {
                  r[u][2] = fmaf(k0.x, k1.x, fmaf(k0.y, k1.y, r[u][2]));
                  r[u][3] = fmaf(k0.x, q1.x, fmaf(k0.y, q1.y, r[u][3]));
                }
              }
            }
          }
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
#pragma unroll
          for (int u = 0; u < PPW; ++u)
#pragma unroll
            for (int x = 0; x < NR; ++x) r[u][x] += __shfl_xor_sync(0xffffffffu, r[u][x], off);
        if (lane == 0) {
#pragma unroll
          for (int u = 0; u < PPW; ++u) {
            const int pp = p0 + WARPS * u;
            if (pp < npairs) {
              const int t0 = 2 * pp, t1 = t0 + 1;
              float* fk = reinterpret_cast<float*>(smem + S::C_KQ);
              fk[t0] = r[u][0];
              float a1 = 1.f;
              if constexpr (!VG) {
                float* fa = reinterpret_cast<float*>(smem + S::C_A);
                fa[t0] = expf(reinterpret_cast<const float*>(raw + S::R_G)[t0]);
                if (t1 < n) fa[t1] = a1 = expf(reinterpret_cast<const float*>(raw + S::R_G)[t1]);
              }
              if (t1 < n) {
                fk[t1] = r[u][1];
                if constexpr (!VG) {
                  reinterpret_cast<float*>(smem + S::C_C)[pp] = a1 * r[u][2];
                  reinterpret_cast<float*>(smem + S::C_E)[pp] = a1 * r[u][3];
                }
              }
            }
          }
        }
      }
      __syncthreads();

      const __nv_bfloat16* rv = reinterpret_cast<const __nv_bfloat16*>(raw + S::R_V);
      const float* rb = reinterpret_cast<const float*>(raw + S::R_B);
      const float4* ca = reinterpret_cast<const float4*>(smem + S::C_A);
      const float* cc = reinterpret_cast<const float*>(smem + S::C_C);
      const float* ce = reinterpret_cast<const float*>(smem + S::C_E);
      int j = 0;
#pragma unroll 1
      for (; !VG && j + 1 < n; j += 2) {  // scalar gate: token pairs
        const int b0 = j * DK / 4 + j8, b1 = b0 + DK / 4;
        const float a0s = caf[j], a1s = caf[j + 1];
        float px0[RG][MB], py0[RG][MB], px1[RG][MB], py1[RG][MB];
        float4 k0[MB], k1[MB];
#pragma unroll
        for (int m = 0; m < MB; ++m) {
          const float4 q0 = cq[b0 + LPR * m], q1 = cq[b1 + LPR * m];
          k0[m] = ck[b0 + LPR * m];
          k1[m] = ck[b1 + LPR * m];
#pragma unroll
          for (int i = 0; i < RG; ++i) {
            const float4 sp = mul4(s[i][m], a0s);
            px0[i][m] = dot44(sp, k0[m]);
            py0[i][m] = dot44(sp, q0);
            s[i][m] = mul4(sp, a1s);  // u
            px1[i][m] = dot44(s[i][m], k1[m]);
            py1[i][m] = dot44(s[i][m], q1);
          }
        }
        float x0[RG], y0[RG], x1[RG], y1[RG];
#pragma unroll
        for (int i = 0; i < RG; ++i) {
          x0[i] = tree_sum(px0[i]);
          y0[i] = tree_sum(py0[i]);
          x1[i] = tree_sum(px1[i]);
          y1[i] = tree_sum(py1[i]);
        }
#pragma unroll
        for (int off = 1; off < LPR; off <<= 1)
#pragma unroll
          for (int i = 0; i < RG; ++i) {
            x0[i] += __shfl_xor_sync(0xffffffffu, x0[i], off);
            y0[i] += __shfl_xor_sync(0xffffffffu, y0[i], off);
            x1[i] += __shfl_xor_sync(0xffffffffu, x1[i], off);
            y1[i] += __shfl_xor_sync(0xffffffffu, y1[i], off);
          }
        const float beta0 = rb[j], beta1 = rb[j + 1], kq0 = ckq[j], kq1 = ckq[j + 1];
        const float c = cc[j / 2], e = ce[j / 2];
        float o0[RG], o1[RG];
#pragma unroll
        for (int i = 0; i < RG; ++i) {
          const float v0 = __bfloat162float(rv[j * S::ROWS_PER_CTA + wrow + RS * i]);
          const float v1 = __bfloat162float(rv[(j + 1) * S::ROWS_PER_CTA + wrow + RS * i]);
          const float d0 = beta0 * (v0 - x0[i]);
          const float d1 = beta1 * (v1 - fmaf(d0, c, x1[i]));
          o0[i] = fmaf(d0, kq0, y0[i]);
          o1[i] = fmaf(d1, kq1, fmaf(d0, e, y1[i]));
#pragma unroll
          for (int m = 0; m < MB; ++m) s[i][m] = fma4(d1, k1[m], fma4(d0 * a1s, k0[m], s[i][m]));
        }
        if (j8 == 0) {
          const size_t orow = ((size_t(b) * a.T + t0 + j) * a.H + h) * a.Dv + vrow0 + wrow;
          const size_t ostep = size_t(a.H) * a.Dv;  // one token later
#pragma unroll
          for (int i = 0; i < RG; ++i) {
            a.o[orow + RS * i] = o0[i];
            a.o[orow + ostep + RS * i] = o1[i];
          }
        }
      }
#pragma unroll 1
      for (; j < n; ++j) {  // per-channel gate: every token; scalar gate: a last odd one
        float4 kk[MB], qq[MB], aa[VG ? MB : 1];
#pragma unroll
        for (int m = 0; m < MB; ++m) {
          kk[m] = ck[j * DK / 4 + j8 + LPR * m];
          qq[m] = cq[j * DK / 4 + j8 + LPR * m];
          if constexpr (VG) aa[m] = ca[j * DK / 4 + j8 + LPR * m];
        }
        if constexpr (!VG) aa[0].x = caf[j];
        float v[RG], o[RG];
#pragma unroll
        for (int i = 0; i < RG; ++i) v[i] = __bfloat162float(rv[j * S::ROWS_PER_CTA + wrow + RS * i]);
        apply_token<MB, VG, LPR, RG, false>(s, kk, qq, aa, ckq[j], rb[j], v, o);
        if (j8 == 0) {
          const size_t orow = ((size_t(b) * a.T + t0 + j) * a.H + h) * a.Dv + vrow0 + wrow;
#pragma unroll
          for (int i = 0; i < RG; ++i) a.o[orow + RS * i] = o[i];
        }
      }
      __syncthreads();  // the converted chunk and this staging buffer are reused
    }
  }

  float4* dst = reinterpret_cast<float4*>(a.S_out + srow);
#pragma unroll
  for (int i = 0; i < RG; ++i)
#pragma unroll
    for (int m = 0; m < MB; ++m) __stcs(dst + i * RS * DK / 4 + j8 + LPR * m, s[i][m]);
}

template <int DK, bool VG, int LPR, int RG, bool DIRECT>
bool launch_one(const RowArgs& a, long long heads, cudaStream_t stream) {
  using S = Shape<DK, VG, LPR, RG>;
  const int smem = DIRECT ? 0 : S::SMEM;
  static_assert(S::SMEM <= 48 * 1024, "within the default dynamic shared memory");
  const int slot = 16 + (DK == 64 ? 0 : DK == 128 ? 8 : 16) + (VG ? 4 : 0) + (RG - 1) * 2 + DIRECT;
  if (smem > 48 * 1024 &&
      !ensure_smem_attr(reinterpret_cast<const void*>(&rows_kernel<DK, VG, LPR, RG, DIRECT>), slot, smem))
    return false;
  rows_kernel<DK, VG, LPR, RG, DIRECT>
      <<<unsigned(heads * (a.Dv / S::ROWS_PER_CTA)), THREADS, smem, stream>>>(a);
  return cudaGetLastError() == cudaSuccess;
}

template <int DK, bool VG, int LPR, int RG>
bool launch_shape(const RowArgs& a, long long heads, cudaStream_t stream) {
  return a.T == 1 ? launch_one<DK, VG, LPR, RG, true>(a, heads, stream)
                  : launch_one<DK, VG, LPR, RG, false>(a, heads, stream);
}

template <int DK, bool VG>
bool launch_dk(const RowArgs& a, long long heads, int rows, cudaStream_t stream) {
  if (rows == 16) return launch_shape<DK, VG, 8, 1>(a, heads, stream);
  return launch_shape<DK, VG, 8, 2>(a, heads, stream);
}

}  // namespace

int rows_per_cta(long long heads, int Dv, int num_sms) {
  // 32 rows per CTA (two row groups per warp: the fewest instructions per
  // row) when that still gives every SM two CTAs; else 16 rows, which spreads
  // few chains over more SMs.  (16 lanes a row, for twice the warps, measured
  // no faster on few chains: each warp is bound by its own per-token latency.)
  return heads * (Dv / 32) >= 2LL * num_sms ? 32 : 16;
}

bool rows_head_dims_ok(int Dk, int Dv) {
  auto ok = [](int d) { return d == 64 || d == 128 || d == 256; };
  return ok(Dk) && ok(Dv);
}

int launch_rows(const RowArgs& a, int Dk, bool vector_gate, int num_sms, cudaStream_t stream) {
  const long long heads = (long long)a.B * a.H;
  if (heads == 0) return 0;
  if (!rows_head_dims_ok(Dk, a.Dv)) return -1;
  const int rows = rows_per_cta(heads, a.Dv, num_sms);
  bool ok;
  if (Dk == 64)
    ok = vector_gate ? launch_dk<64, true>(a, heads, rows, stream) : launch_dk<64, false>(a, heads, rows, stream);
  else if (Dk == 128)
    ok = vector_gate ? launch_dk<128, true>(a, heads, rows, stream) : launch_dk<128, false>(a, heads, rows, stream);
  else
    ok = vector_gate ? launch_dk<256, true>(a, heads, rows, stream) : launch_dk<256, false>(a, heads, rows, stream);
  return ok ? 0 : -1;
}

}  // namespace gdn
