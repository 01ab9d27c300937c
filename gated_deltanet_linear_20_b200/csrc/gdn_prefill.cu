// Chunked gated-delta-rule prefill for sm_100a: TMA-staged bf16 tiles,
// tcgen05 MMAs accumulating in tensor memory, fp32 state carried across
// chunks in tensor memory.
//
// Recurrence (per sequence b, head h; S in R^{Dv x Dk}):
//   S_t = exp(g_t) S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,  o_t = S_t q_t.
// The ROCmFPX gated-delta-net prefill note (bittide.aicompass.dev article
// d2880479, opening post) moves this prefill from one token at a time to
// 16-token chunks with the state in F32 accumulators, scalar gate, head dim
// 128; here chunks of 16 or 64 tokens run on the 5th-generation tensor cores.
//
// Chunked form used (derived from the recurrence; tokens i, j of one chunk,
// S_c the state entering it, gamma = inclusive cumulative sum of g inside the
// chunk, Gamma = exp(gamma), Dec_ij = exp(gamma_i - gamma_j)):
//   A     = strict_tril(diag(beta) K K^T .* Dec)          (chunk x chunk)
//   T     = (I + A)^{-1}                                  (unit lower triangular)
//   X^T   = V^T diag(beta) - diag-cols(beta Gamma) (S_c K^T)        (Dv x chunk)
//   Dl^T  = X^T T^T                                       (the delta-rule residuals)
//   O^T   = diag-cols(Gamma) (S_c Q^T) + Dl^T Mq^T,  Mq = tril(Q K^T .* Dec)
//   S_out = Gamma_last S_c + Dl^T diag(exp(gamma_last - gamma)) K
//
// One CTA of 512 threads owns one (b, h) chain and walks its tokens in tiles
// of 64 (one TMA tile); with chunk = 16 each tile holds four chunks, processed
// in order.  Warp w reads TMEM lane quarter (w % 4) -- state rows, i.e. the Dv
// index, 32 (w % 4) .. +31 -- and column quarter (w / 4) of every tile it
// touches, so each epilogue is spread over 16 warps.  The fp32 state lives in tensor
// memory, pre-multiplied by the decay of the chunk about to update it, so the
// state-update MMA accumulates straight into it; the tensor core reads the
// state as a bf16 hi/lo pair, also in tensor memory.  Every operand derived
// inside the kernel (S, X, T, the residuals, Mq) is fed to the MMA as hi + lo
// bf16 parts (hi = bf16(x), lo = bf16(x - hi)) so the products keep ~16 bits
// of mantissa; q, k and v are exact bf16 inputs.
//
// Tensor memory (512 columns, fp32 unless noted):
//   [  0,128) S   : state, scaled by the next chunk's total decay  (lane dv, col dk)
//   [128,192) SHI : S hi as bf16 pairs (A operand)                 (lane dv, col dk/2)
//   [192,256) SLO : S lo
//   [256,384) ZQ  : [S K^T | S Q^T]                                (lane dv, col token)
//   [384,448) PD  : [K;Q] K^T (lanes 0..127 = rows of [K;Q]), later Dl^T
//   [448,512) OI  : Dl^T Mq^T                                      (lane dv, col token)
#include "gdn_internal.h"
#include "sm100.cuh"

namespace gdn {
namespace {

using namespace sm100;

constexpr int D = 128;
constexpr int NT = 64;  // tokens per TMA tile
constexpr int NTHREADS = 512;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TM_S = 0, TM_SHI = 128, TM_SLO = 192, TM_ZQ = 256, TM_PD = 384, TM_OI = 448;

// Shared memory map (offsets from a 1024-byte aligned base).
constexpr uint32_t SM_KQ0 = 0;        // 32 KB: [K dk0-63 | Q dk0-63 | K dk64-127 | Q dk64-127]
constexpr uint32_t SM_KQ1 = 32768;    //        each a 64-row x 128-byte SW128 box
constexpr uint32_t SM_V0 = 65536;     // 16 KB: V tile [64 tokens][128] bf16, unswizzled
constexpr uint32_t SM_V1 = 81920;
constexpr uint32_t SM_MQH = 98304;    // 8 KB: Mq rows i, K-major SW128 (64 x 64 bf16)
constexpr uint32_t SM_MQL = 106496;
constexpr uint32_t SM_TH = 114688;    // 8 KB: T rows i (64 x 64)
constexpr uint32_t SM_TL = 122880;
constexpr uint32_t SM_XH = 131072;    // 16 KB: X^T rows dv (128 x 64); then the decay-scaled
constexpr uint32_t SM_XL = 147456;    //        residuals; at the end of a tile, the o tile
constexpr uint32_t SM_DH = 163840;    // 16 KB: Dl^T rows dv (128 x 64)
constexpr uint32_t SM_DL = 180224;
// The triangular solve runs while the X / Dl regions are idle and borrows them:
constexpr int APAD = 68;                      // row pitch (floats): conflict-free float4 rows
constexpr uint32_t SOLVE_MAT = 64 * APAD * 4; // 17408 B
constexpr uint32_t SM_A = SM_XH;              // A   fp32 [64][APAD]
constexpr uint32_t SM_TF = SM_A + SOLVE_MAT;  // T   fp32 [64][APAD]
constexpr uint32_t SM_E = SM_TF + SOLVE_MAT;  // block products fp32 [3][16][16]
constexpr uint32_t SM_O = SM_XH;              // o tile fp32 [64 tokens][128] (32 KB)
constexpr uint32_t SM_MISC = 196608;  // gates, barriers, TMEM slot
constexpr uint32_t MISC_G = 0, MISC_B = 256, MISC_GAM2 = 512, MISC_GAM = 768, MISC_BG = 1024,
                   MISC_DF = 1280, MISC_GC = 1536, MISC_GCN = 1552, MISC_PART = 1560,
                   MISC_BAR = 1600, MISC_TMEM = 1632, MISC_ABORT = 1636;
constexpr uint32_t SMEM_USED = SM_MISC + 2048;
static_assert(SM_E + 3 * 256 * 4 <= SM_DL + 16384, "solve scratch must stay inside the X/Dl regions");
static_assert(SM_O + 64 * 128 * 4 <= SM_DH, "o tile must stay inside the X region");
static_assert(SM_DL + 16384 <= SM_MISC, "tiles overlap the misc area");
constexpr uint32_t TILE_TX_BYTES = 4 * 8192 + 16384;
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;  // 2 s: far beyond any legitimate wait

constexpr float LOG2E = 1.4426950408889634f;

// Byte offset of 16-byte chunk `c` (8 bf16 along K) of row `r` in a K-major
// SW128 tile whose rows are 128 bytes and whose 8-row groups are 1024 B apart.
__device__ __forceinline__ uint32_t sw128_off(int r, int c) {
  return uint32_t((r >> 3) * 1024 + (r & 7) * 128 + (((c ^ r) & 7) << 4));
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c,
                                             uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c),
               "r"(d)
               : "memory");
}
// Splits 8 floats into hi/lo bf16 and stores them as chunk `c` of row `r` in two tiles.
__device__ __forceinline__ void store_split8(uint32_t hi_tile, uint32_t lo_tile, int r, int c,
                                             const float* x) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    __nv_bfloat16 h0, l0, h1, l1;
    split_bf16(x[2 * e], h0, l0);
    split_bf16(x[2 * e + 1], h1, l1);
    h[e] = pack_bf16x2(h0, h1);
    l[e] = pack_bf16x2(l0, l1);
  }
  const uint32_t off = sw128_off(r, c);
  st_shared_v4(hi_tile + off, h[0], h[1], h[2], h[3]);
  st_shared_v4(lo_tile + off, l[0], l[1], l[2], l[3]);
}

// Splits 4 floats into hi/lo bf16 and stores them as the 8-byte half `hf` of
// chunk `c` of row `r` in two tiles.
__device__ __forceinline__ void store_split4(uint32_t hi_tile, uint32_t lo_tile, int r, int c,
                                             int hf, const float* x) {
  __nv_bfloat16 h0, l0, h1, l1, h2, l2, h3, l3;
  split_bf16(x[0], h0, l0);
  split_bf16(x[1], h1, l1);
  split_bf16(x[2], h2, l2);
  split_bf16(x[3], h3, l3);
  const uint32_t off = sw128_off(r, c) + 8u * hf;
  asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(hi_tile + off), "r"(pack_bf16x2(h0, h1)),
               "r"(pack_bf16x2(h2, h3))
               : "memory");
  asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(lo_tile + off), "r"(pack_bf16x2(l0, l1)),
               "r"(pack_bf16x2(l2, l3))
               : "memory");
}

// Splits 32 consecutive state values (columns 32q..32q+31 of this lane's row)
// into bf16 hi/lo pairs and stores them to SHI / SLO.
__device__ __forceinline__ void store_state_split32(uint32_t tlane, int q, const float (&v)[32]) {
  uint32_t hi[16], lo[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) {
    __nv_bfloat16 h0, l0, h1, l1;
    split_bf16(v[2 * e], h0, l0);
    split_bf16(v[2 * e + 1], h1, l1);
    hi[e] = pack_bf16x2(h0, h1);
    lo[e] = pack_bf16x2(l0, l1);
  }
  tmem_st16x2(tlane + TM_SHI + 16 * q, hi, tlane + TM_SLO + 16 * q, lo);
}

struct Flow {
  uint32_t mma_bar;
  uint32_t mma_phase;
  volatile int* abort_flag;
  int* status;
  // All threads wait for the last commit; a wait that gives up flags the CTA.
  __device__ __forceinline__ void wait_mma() {
    if (!mbar_wait_bounded(mma_bar, mma_phase, WAIT_LIMIT_NS)) fail();
    mma_phase ^= 1u;
    tc_fence_after();
  }
  __device__ __forceinline__ void fail() {
    *abort_flag = 1;
    if (status) atomicExch(status, GDN_ERR_DEVICE_TIMEOUT);
  }
};

// Sum of g over the first chunk of a tile held by threads 0..63 (one value
// each, zero past T), i.e. the log-decay of that chunk.  Threads 0..63 call it;
// the result lands in *out.  C == 64 uses `part` as a two-warp scratch slot.
template <int C>
__device__ __forceinline__ void first_chunk_logdecay(int tid, float g, float* part, float* out) {
  float x = (tid < C) ? g : 0.f;
  constexpr int W = C < 32 ? C : 32;
#pragma unroll
  for (int off = W / 2; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off, W);
  if constexpr (C == 64) {
    if (tid == 32) *part = x;
    asm volatile("bar.sync 1, 64;" ::: "memory");  // warps 0 and 1 only
    if (tid == 0) *out = x + *part;
  } else {
    if (tid == 0) *out = x;
  }
}

// One distance-d sweep of the blocked inverse of (I + A), 64 x 64 in 16 x 16
// blocks (diagonal blocks already inverted in Tf):
//   E_p     = sum_{K=J}^{I-1} A_{I,K} T_{K,J}        (I = J + d, p = J)
//   T_{I,J} = -T_{I,I} E_p
// Each thread owns a 1 x 4 strip of outputs so one A load and one float4 T
// load feed four FMAs; all loop bounds are compile-time.
template <int d>
__device__ __forceinline__ void solve_offdiag(int tid, const float* sA, float* sTf, float* sE) {
  constexpr int NSTRIP = (4 - d) * 64;  // (4-d) block pairs x 16 rows x 4 strips
  if (tid < NSTRIP) {
    const int pp = tid >> 6, r = (tid >> 2) & 15, c4 = tid & 3;
    const float* arow = sA + ((pp + d) * 16 + r) * APAD + pp * 16;
    const float* tcol = sTf + (pp * 16) * APAD + pp * 16 + 4 * c4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int k = 0; k < 16 * d; ++k) {
      const float a = arow[k];
      const float4 t = *reinterpret_cast<const float4*>(tcol + k * APAD);
      acc.x = fmaf(a, t.x, acc.x);
      acc.y = fmaf(a, t.y, acc.y);
      acc.z = fmaf(a, t.z, acc.z);
      acc.w = fmaf(a, t.w, acc.w);
    }
    *reinterpret_cast<float4*>(sE + pp * 256 + r * 16 + 4 * c4) = acc;
  }
  __syncthreads();
  if (tid < NSTRIP) {
    const int pp = tid >> 6, r = (tid >> 2) & 15, c4 = tid & 3;
    const int I = pp + d;
    const float* trow = sTf + (I * 16 + r) * APAD + I * 16;
    const float* e = sE + pp * 256 + 4 * c4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const float a = trow[k];
      const float4 t = *reinterpret_cast<const float4*>(e + k * 16);
      acc.x = fmaf(a, t.x, acc.x);
      acc.y = fmaf(a, t.y, acc.y);
      acc.z = fmaf(a, t.z, acc.z);
      acc.w = fmaf(a, t.w, acc.w);
    }
    *reinterpret_cast<float4*>(sTf + (I * 16 + r) * APAD + pp * 16 + 4 * c4) =
        make_float4(-acc.x, -acc.y, -acc.z, -acc.w);
  }
  __syncthreads();
}

template <int C>
__global__ void __launch_bounds__(NTHREADS, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                   const PrefillArgs p) {
  static_assert(C == 16 || C == 64, "chunk must be 16 or 64");
  constexpr int NSUB = NT / C;  // chunks per TMA tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  const uint32_t sb = smem_u32(sm);
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lq = warp & 3;                  // TMEM lane quarter
  const int cg = warp >> 2;                 // column quarter
  const int row = lq * 32 + (tid & 31);     // TMEM lane: Dv row, or row of [K;Q]
  const int chain = blockIdx.x;
  const int b = chain / p.H;
  const int h = chain - b * p.H;
  const int T = p.T, H = p.H;

  float* s_g = reinterpret_cast<float*>(sm + SM_MISC + MISC_G);
  float* s_b = reinterpret_cast<float*>(sm + SM_MISC + MISC_B);
  float* s_gam2 = reinterpret_cast<float*>(sm + SM_MISC + MISC_GAM2);
  float* s_Gam = reinterpret_cast<float*>(sm + SM_MISC + MISC_GAM);
  float* s_bG = reinterpret_cast<float*>(sm + SM_MISC + MISC_BG);
  float* s_df = reinterpret_cast<float*>(sm + SM_MISC + MISC_DF);
  float* s_GC = reinterpret_cast<float*>(sm + SM_MISC + MISC_GC);    // per chunk of this tile
  float* s_GCn = reinterpret_cast<float*>(sm + SM_MISC + MISC_GCN);  // first chunk, next tile
  float* s_part = reinterpret_cast<float*>(sm + SM_MISC + MISC_PART);
  const uint32_t bar_tma0 = sb + SM_MISC + MISC_BAR;
  const uint32_t bar_mma = bar_tma0 + 16;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(sm + SM_MISC + MISC_TMEM);
  volatile int* s_abort = reinterpret_cast<volatile int*>(sm + SM_MISC + MISC_ABORT);
  float* sA = reinterpret_cast<float*>(sm + SM_A);
  float* sTf = reinterpret_cast<float*>(sm + SM_TF);
  float* sE = reinterpret_cast<float*>(sm + SM_E);
  float* sO = reinterpret_cast<float*>(sm + SM_O);

  if (tid == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_o);
    mbar_init(bar_tma0, 1);
    mbar_init(bar_tma0 + 8, 1);
    mbar_init(bar_mma, 1);
    fence_mbar_init();
    *s_abort = 0;
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(s_tmem), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;
  const uint32_t tlane = tmem + (uint32_t(lq * 32) << 16);  // this warp's lane quarter

  Flow flow{bar_mma, 0u, s_abort, p.status};
  const int ntiles = (T + NT - 1) / NT;
  int tma_issued = 0;  // tiles whose TMA was issued (thread 0's view)
  int tma_done = 0;    // tiles whose TMA completion was observed
  const int dv = row;

  auto issue_tile = [&](int c) {
    const int st = c & 1;
    const uint32_t kq = sb + (st ? SM_KQ1 : SM_KQ0);
    const uint32_t vt = sb + (st ? SM_V1 : SM_V0);
    const uint32_t bar = bar_tma0 + 8 * st;
    mbar_arrive_expect_tx(bar, TILE_TX_BYTES);
    tma_load_4d(kq + 0, &tm_k, bar, 0, h, c * NT, b);
    tma_load_4d(kq + 8192, &tm_q, bar, 0, h, c * NT, b);
    tma_load_4d(kq + 16384, &tm_k, bar, 64, h, c * NT, b);
    tma_load_4d(kq + 24576, &tm_q, bar, 64, h, c * NT, b);
    tma_load_4d(vt, &tm_v, bar, 0, h, c * NT, b);
  };

  // ---- gates of tile 0; the first TMA tile
  float g_next = 0.f, b_next = 0.f;
  if (tid < NT && tid < T) {
    const size_t gi = (size_t(b) * T + tid) * H + h;
    g_next = __ldg(p.g + gi);
    b_next = __ldg(p.beta + gi);
  }
  if (tid == 0) {
    issue_tile(0);
    tma_issued = 1;
  }

  // ---- initial state (row dv = tid of S0, or zeros): hi/lo copy, and the
  //      fp32 copy pre-scaled by the decay of the first chunk
  if (tid < NT) first_chunk_logdecay<C>(tid, g_next, s_part, s_GCn);
  __syncthreads();
  {
    const float gc0 = exp2f(*s_GCn * LOG2E);
    const float4* src = p.S0 ? reinterpret_cast<const float4*>(p.S0 + (size_t(chain) * D + dv) * D)
                             : nullptr;
    float v[32];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      float4 x = src ? __ldg(src + 8 * cg + e) : make_float4(0.f, 0.f, 0.f, 0.f);
      v[4 * e] = x.x;
      v[4 * e + 1] = x.y;
      v[4 * e + 2] = x.z;
      v[4 * e + 3] = x.w;
    }
    store_state_split32(tlane, cg, v);
    uint32_t u[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) u[e] = __float_as_uint(gc0 * v[e]);
    tmem_st32(tlane + TM_S + 32 * cg, u);
  }
  tc_fence_before();

  for (int c = 0; c < ntiles; ++c) {
    const int st = c & 1;
    const int t0 = c * NT;
    const uint32_t kq = sb + (st ? SM_KQ1 : SM_KQ0);
    const uint8_t* vtile = sm + (st ? SM_V1 : SM_V0);
    const bool last_tile = (c + 1 == ntiles);

    // ---- gates of this tile (inclusive in-chunk scan); prefetch the next tile
    float g_cur = 0.f;
    if (tid < NT) {
      g_cur = g_next;
      s_g[tid] = g_next;
      s_b[tid] = b_next;
      g_next = 0.f;
      b_next = 0.f;
      const int t = t0 + NT + tid;
      if (t < T) {
        const size_t gi = (size_t(b) * T + t) * H + h;
        g_next = __ldg(p.g + gi);
        b_next = __ldg(p.beta + gi);
      }
      constexpr int W = C < 32 ? C : 32;
      const int ln = tid & 31;
#pragma unroll
      for (int off = 1; off < W; off <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, g_cur, off, W);
        if ((ln & (W - 1)) >= off) g_cur += y;
      }
      if constexpr (C == 64) {
        if (tid == 31) *s_part = g_cur;
      }
    }
    if (tid == 0 && c + 1 < ntiles) {
      issue_tile(c + 1);
      tma_issued = c + 2;
    }
    __syncthreads();
    if (tid < NT) {
      if constexpr (C == 64) {
        if (tid >= 32) g_cur += *s_part;
      }
      s_gam2[tid] = g_cur * LOG2E;
    }
    __syncthreads();
    if (tid < NT) {
      const int last = (tid / C) * C + C - 1;
      const float gi = s_gam2[tid], gl = s_gam2[last];
      const float G = exp2f(gi);
      s_Gam[tid] = G;
      s_bG[tid] = s_b[tid] * G;
      s_df[tid] = exp2f(gl - gi);
      if (tid == last) s_GC[tid / C] = exp2f(gl);
    }
    if (mbar_wait_bounded(bar_tma0 + 8 * st, (c >> 1) & 1, WAIT_LIMIT_NS))
      tma_done = c + 1;
    else
      flow.fail();
    __syncthreads();
    if (*s_abort) goto teardown;

    // ---- P = [K; Q] K^T : M=128 (rows of [K;Q]), N=64 (tokens j), K=128 (dk)
    if (tid == 0) {
      tc_fence_after();
      const uint32_t id = idesc_bf16(128, 64, 0, 0, 0);
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
        mma_ss(tmem + TM_PD, sdesc_sw128(kq + off, 16, 1024), sdesc_sw128(kq + off, 16, 1024), id,
               kk > 0);
      }
      mma_commit(bar_mma);
    }
    flow.wait_mma();

    // ---- masks and decays: rows 0..63 -> A (fp32, for the solve); rows 64..127 -> Mq
    {
      const int i = row & (NT - 1);
      const int cs = (i / C) * C;
      const float gi = s_gam2[i];
      const float bi = s_b[i];
      float P[16];
      tmem_ld16(tlane + TM_PD + 16 * cg, P);
      float m[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int j = 16 * cg + e;
        const bool keep = (j >= cs) && (row < NT ? (j < i) : (j <= i));
        const float x = exp2f(gi - s_gam2[j]) * P[e];
        m[e] = keep ? (row < NT ? bi * x : x) : 0.f;
      }
      if (row < NT) {
        float4* dst = reinterpret_cast<float4*>(sA + i * APAD + 16 * cg);
#pragma unroll
        for (int e = 0; e < 4; ++e) dst[e] = make_float4(m[4 * e], m[4 * e + 1], m[4 * e + 2], m[4 * e + 3]);
      } else {
        store_split8(sb + SM_MQH, sb + SM_MQL, i, 2 * cg, m);
        store_split8(sb + SM_MQH, sb + SM_MQL, i, 2 * cg + 1, m + 8);
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---- T = (I + A)^{-1}, blocked in 16 x 16 blocks.
    //  (1) diagonal blocks: thread r < 64 forms row r of its block's inverse,
    //      x (I + A_bb) = e_r, right-looking: x_i is final once every row
    //      below it has been subtracted, then x_i A_i,j leaves each acc_j (j < i);
    //  (2) with chunk 64, the off-diagonal blocks by distance d = 1..3:
    //      T_{I,J} = -T_{I,I} sum_{K=J}^{I-1} A_{I,K} T_{K,J}.
    if (tid < NT) {
      const int r = tid, bb = r >> 4, rr = r & 15, base = bb * 16;
      float acc[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) acc[j] = (j == rr) ? 1.f : 0.f;
#pragma unroll
      for (int i = 15; i > 0; --i) {
        const float xi = acc[i];
        const float4* arow = reinterpret_cast<const float4*>(sA + (base + i) * APAD + base);
#pragma unroll
        for (int j4 = 0; j4 < 4; ++j4) {
          if (4 * j4 < i) {
            const float4 a = arow[j4];
            if (4 * j4 + 0 < i) acc[4 * j4 + 0] = fmaf(-xi, a.x, acc[4 * j4 + 0]);
            if (4 * j4 + 1 < i) acc[4 * j4 + 1] = fmaf(-xi, a.y, acc[4 * j4 + 1]);
            if (4 * j4 + 2 < i) acc[4 * j4 + 2] = fmaf(-xi, a.z, acc[4 * j4 + 2]);
            if (4 * j4 + 3 < i) acc[4 * j4 + 3] = fmaf(-xi, a.w, acc[4 * j4 + 3]);
          }
        }
      }
      float4* trow = reinterpret_cast<float4*>(sTf + r * APAD);
#pragma unroll
      for (int q4 = 0; q4 < 16; ++q4) {
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if ((q4 >> 2) == bb)
          v = make_float4(acc[4 * (q4 & 3)], acc[4 * (q4 & 3) + 1], acc[4 * (q4 & 3) + 2],
                          acc[4 * (q4 & 3) + 3]);
        trow[q4] = v;
      }
    }
    __syncthreads();
    if constexpr (C == 64) {
      solve_offdiag<1>(tid, sA, sTf, sE);
      solve_offdiag<2>(tid, sA, sTf, sE);
      solve_offdiag<3>(tid, sA, sTf, sE);
    }
    // T (fp32) -> hi/lo bf16 K-major tiles; eight threads per row, one chunk each
    store_split8(sb + SM_TH, sb + SM_TL, tid >> 3, tid & 7, sTf + (tid >> 3) * APAD + 8 * (tid & 7));
    fence_proxy_async_smem();
    __syncthreads();

#pragma unroll 1
    for (int s = 0; s < NSUB; ++s) {
      // ---- [Z | Y] = S_c [K | Q]^T : M=128 (dv), N=2C, K=128 (dk); A = S hi, then S lo
      if (tid == 0) {
        tc_fence_after();
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          const uint32_t a0 = tmem + (part ? TM_SLO : TM_SHI);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
            const uint32_t acc = (part | kk) ? 1u : 0u;
            if constexpr (C == 64) {
              mma_ts(tmem + TM_ZQ, a0 + kk * 8, sdesc_sw128(kq + off, 16, 1024),
                     idesc_bf16(128, 128, 0, 0, 0), acc);
            } else {
              const uint32_t rows = 2048u * s;
              mma_ts(tmem + TM_ZQ + 16 * s, a0 + kk * 8, sdesc_sw128(kq + off + rows, 16, 1024),
                     idesc_bf16(128, 16, 0, 0, 0), acc);
              mma_ts(tmem + TM_ZQ + 64 + 16 * s, a0 + kk * 8,
                     sdesc_sw128(kq + 8192 + off + rows, 16, 1024), idesc_bf16(128, 16, 0, 0, 0),
                     acc);
            }
          }
        }
        mma_commit(bar_mma);
      }
      flow.wait_mma();

      // ---- X^T[dv][n] = beta_n V[n][dv] - beta_n Gamma_n Z[dv][n]  (hi/lo -> SMEM)
      {
        const __nv_bfloat16* V = reinterpret_cast<const __nv_bfloat16*>(vtile);
        if constexpr (C == 64) {
          const int n0 = 16 * cg;
          float Z[16];
          tmem_ld16(tlane + TM_ZQ + n0, Z);
          float x[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int n = n0 + e;
            x[e] = fmaf(s_b[n], __bfloat162float(V[n * D + dv]), -s_bG[n] * Z[e]);
          }
          store_split8(sb + SM_XH, sb + SM_XL, dv, n0 / 8, x);
          store_split8(sb + SM_XH, sb + SM_XL, dv, n0 / 8 + 1, x + 8);
        } else {
          const int n0 = 16 * s + 4 * cg;
          float Z[4];
          tmem_ld4(tlane + TM_ZQ + n0, Z);
          float x[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int n = n0 + e;
            x[e] = fmaf(s_b[n], __bfloat162float(V[n * D + dv]), -s_bG[n] * Z[e]);
          }
          store_split4(sb + SM_XH, sb + SM_XL, dv, n0 / 8, (n0 / 4) & 1, x);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncthreads();

      // ---- Dl^T = X^T T^T : M=128 (dv), N=C (i), K=C (n); 3 hi/lo products
      if (tid == 0) {
        tc_fence_after();
        const uint32_t id = idesc_bf16(128, C, 0, 0, 0);
        const uint32_t trow = uint32_t(C * s / 8) * 1024u;
#pragma unroll
        for (int part = 0; part < 3; ++part) {
          const uint32_t xa = sb + (part == 2 ? SM_XL : SM_XH);
          const uint32_t tb = sb + (part == 1 ? SM_TL : SM_TH) + trow;
#pragma unroll
          for (int ks = 0; ks < C / 16; ++ks) {
            const uint32_t kb = uint32_t(C * s + 16 * ks) * 2u;
            mma_ss(tmem + TM_PD + C * s, sdesc_sw128(xa + kb, 16, 1024),
                   sdesc_sw128(tb + kb, 16, 1024), id, (part | ks) ? 1u : 0u);
          }
        }
        mma_commit(bar_mma);
      }
      flow.wait_mma();

      // ---- residuals: Dl (for the output) and Dl * exp(gamma_last - gamma) (for the state)
      {
        if constexpr (C == 64) {
          const int n0 = 16 * cg;
          float d[16];
          tmem_ld16(tlane + TM_PD + n0, d);
          float dt[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) dt[e] = d[e] * s_df[n0 + e];
          store_split8(sb + SM_DH, sb + SM_DL, dv, n0 / 8, d);
          store_split8(sb + SM_DH, sb + SM_DL, dv, n0 / 8 + 1, d + 8);
          store_split8(sb + SM_XH, sb + SM_XL, dv, n0 / 8, dt);
          store_split8(sb + SM_XH, sb + SM_XL, dv, n0 / 8 + 1, dt + 8);
        } else {
          const int n0 = 16 * s + 4 * cg;
          float d[4];
          tmem_ld4(tlane + TM_PD + n0, d);
          float dt[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) dt[e] = d[e] * s_df[n0 + e];
          store_split4(sb + SM_DH, sb + SM_DL, dv, n0 / 8, (n0 / 4) & 1, d);
          store_split4(sb + SM_XH, sb + SM_XL, dv, n0 / 8, (n0 / 4) & 1, dt);
        }
        // log-decay of the next tile's first chunk (its gates arrived long ago)
        if (s == NSUB - 1 && !last_tile && tid < NT) first_chunk_logdecay<C>(tid, g_next, s_part, s_GCn);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncthreads();

      // ---- O_intra = Dl^T Mq^T (N=C) and S += Dl~^T K (N=128, B = K tile MN-major)
      if (tid == 0) {
        tc_fence_after();
        const uint32_t id = idesc_bf16(128, C, 0, 0, 0);
        const uint32_t mrow = uint32_t(C * s / 8) * 1024u;
#pragma unroll
        for (int part = 0; part < 3; ++part) {
          const uint32_t da = sb + (part == 2 ? SM_DL : SM_DH);
          const uint32_t mb = sb + (part == 1 ? SM_MQL : SM_MQH) + mrow;
#pragma unroll
          for (int ks = 0; ks < C / 16; ++ks) {
            const uint32_t kb = uint32_t(C * s + 16 * ks) * 2u;
            mma_ss(tmem + TM_OI + C * s, sdesc_sw128(da + kb, 16, 1024),
                   sdesc_sw128(mb + kb, 16, 1024), id, (part | ks) ? 1u : 0u);
          }
        }
        const uint32_t idu = idesc_bf16(128, 128, 0, 1, 0);
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          const uint32_t da = sb + (part ? SM_XL : SM_XH);
#pragma unroll
          for (int ks = 0; ks < C / 16; ++ks) {
            const int tok = C * s + 16 * ks;
            mma_ss(tmem + TM_S, sdesc_sw128(da + uint32_t(tok) * 2u, 16, 1024),
                   sdesc_sw128(kq + uint32_t(tok) * 128u, 16384, 1024), idu, 1u);
          }
        }
        mma_commit(bar_mma);
      }
      flow.wait_mma();

      // ---- S_out now sits in TMEM: refresh its hi/lo copy, and pre-scale it by
      //      the next chunk's decay (or store it as S_T after the last chunk)
      {
        const bool final_chunk = last_tile && (s == NSUB - 1);
        const float gnext = (s + 1 < NSUB) ? s_GC[s + 1] : exp2f(*s_GCn * LOG2E);
        float v[32];
        tmem_ld32(tlane + TM_S + 32 * cg, v);
        store_state_split32(tlane, cg, v);
        if (final_chunk) {
          float4* dst = reinterpret_cast<float4*>(p.S_T + (size_t(chain) * D + dv) * D + 32 * cg);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dst[e] = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
        } else {
          uint32_t u[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) u[e] = __float_as_uint(gnext * v[e]);
          tmem_st32(tlane + TM_S + 32 * cg, u);
        }
      }
      tc_fence_before();
      __syncthreads();
      if (*s_abort) goto teardown;
    }

    // ---- o[t][dv] = Gamma_t Y[dv][t] + O_intra[dv][t]: staged in SMEM, one TMA store
    {
      const int n0 = 16 * cg;
      float y[16], oi[16];
      tmem_ld16x2(tlane + TM_ZQ + 64 + n0, y, tlane + TM_OI + n0, oi);
#pragma unroll
      for (int e = 0; e < 16; ++e) sO[(n0 + e) * D + dv] = fmaf(s_Gam[n0 + e], y[e], oi[e]);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tma_store_4d(&tm_o, sb + SM_O, 0, h, t0, b);  // rows past T are clipped by the TMA unit
      bulk_commit();
      bulk_wait_read0();  // the o tile region is rewritten by the next tile's solve
    }
    __syncthreads();
  }

teardown:
  // An aborted CTA may still have a TMA tile in flight: wait for it (bounded)
  // before the shared memory goes away.
  if (tid == 0) {
    bulk_wait0();
    if (*s_abort) {
      for (int c = tma_done; c < tma_issued; ++c)
        mbar_wait_bounded(bar_tma0 + 8 * (c & 1), (c >> 1) & 1, WAIT_LIMIT_NS / 4);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, TMEM_COLS);
}

// T == 0: S_T = S0 (or zeros); nothing else to do.
__global__ void copy_state_kernel(const float* __restrict__ S0, float* __restrict__ S_T,
                                  size_t n4) {
  const size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n4) return;
  float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
  if (S0) v = reinterpret_cast<const float4*>(S0)[i];
  reinterpret_cast<float4*>(S_T)[i] = v;
}

}  // namespace

int launch_prefill(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                   const CUtensorMap& to, const PrefillArgs& a, int chunk, cudaStream_t stream) {
  const int chains = a.B * a.H;
  if (chains == 0) return 0;
  if (a.T == 0) {
    const size_t n4 = size_t(chains) * D * D / 4;
    if (a.S0 == a.S_T) return 0;
    copy_state_kernel<<<unsigned((n4 + 255) / 256), 256, 0, stream>>>(a.S0, a.S_T, n4);
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
  }
  const uint32_t smem = SMEM_USED + 1024;
  cudaError_t err;
  if (chunk == 64) {
    err = cudaFuncSetAttribute(prefill_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               int(smem));
    if (err != cudaSuccess) return -1;
    prefill_kernel<64><<<chains, NTHREADS, smem, stream>>>(tq, tk, tv, to, a);
  } else {
    err = cudaFuncSetAttribute(prefill_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               int(smem));
    if (err != cudaSuccess) return -1;
    prefill_kernel<16><<<chains, NTHREADS, smem, stream>>>(tq, tk, tv, to, a);
  }
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace gdn
