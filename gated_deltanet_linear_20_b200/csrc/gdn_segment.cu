// Second pass of the segmented prefill (sm_100a, tcgen05).
//
// Inside one segment k of a chain the recurrence is affine in the state the
// segment starts from: with S_k the true state before the segment,
//   S_t = S_k F_{k,t} + R_{k,t},   o_t = S_t q_t = S_k f_t + o^R_t,
// where F_{k,t} is the product of the per-token factors exp(g_s)(I - beta_s k_s k_s^T)
// over the segment's tokens up to t (the state reached from the identity with
// v = 0), f_t = F_{k,t} q_t, and R_{k,t}, o^R_t are the state and output reached
// from a zero start (from S0 for k = 0).  The first pass wrote o^R into o, f_t
// into ws_f, and the segment-end R_k, F_k into ws_R, ws_F.  This pass, one CTA
// per (chain, k >= 1):
//   S_1 = R_0;  S_{j+1} = S_j F_j + R_j  (j = 1 .. k-1)        -> S_k
//   o_t += S_k f_t for the tokens t of segment k
//   k = last: S_T = S_k F_k + R_k
// Products run on the tensor cores with every operand as a bf16 hi/lo pair
// (3 MMAs: hi*hi + hi*lo + lo*hi) and fp32 accumulation in tensor memory.
#include "gdn_internal.h"
#include "sm100.cuh"

namespace gdn {
namespace {

using namespace sm100;

constexpr int D = 128;
constexpr int NT = 64;
constexpr int NTHREADS = 256;
// Shared memory (offsets from a 1024-byte aligned base).  Each 128 x 128 bf16
// operand is two 16 KB SW128 blocks of 128 rows x 64 columns (block h holds
// columns 64h .. 64h+63): rows are M for the state (K-major A) and K for the
// transfer matrix (MN-major B).  The f tile is two 8 KB blocks of 64 token rows.
constexpr uint32_t SS_HI = 0, SS_LO = 32768;
constexpr uint32_t SF_HI = 65536, SF_LO = 98304;
constexpr uint32_t SQ_HI = 131072, SQ_LO = 147456;
constexpr uint32_t SM_BAR = 163840;  // one mbarrier (MMA completion) + verdict slot
constexpr uint32_t SMEM_USED = SM_BAR + 64;
constexpr uint32_t TMEM_COLS = 256;
constexpr uint32_t TM_ACC = 0, TM_O = 128;  // 128-column state product, 64-column o tile
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;

// Thread t of the CTA converts row t/2, columns 64 (t%2) .. +63 of a row-major
// 128 x 128 fp32 matrix into the hi/lo bf16 pair of SW128 blocks.  All loads
// are issued before the first shared store (the stores are ordered asm, which
// would otherwise serialise one global latency per chunk).
__device__ __forceinline__ void load_split_matrix(const float* __restrict__ src, uint32_t hi,
                                                  uint32_t lo) {
  const int r = threadIdx.x >> 1, hf = threadIdx.x & 1;
  const float4* row = reinterpret_cast<const float4*>(src + size_t(r) * D + 64 * hf);
  float4 a[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) a[i] = __ldg(row + i);
#pragma unroll
  for (int c8 = 0; c8 < 8; ++c8) {
    const float x[8] = {a[2 * c8].x, a[2 * c8].y, a[2 * c8].z, a[2 * c8].w,
                        a[2 * c8 + 1].x, a[2 * c8 + 1].y, a[2 * c8 + 1].z, a[2 * c8 + 1].w};
    store_split8(hi + 16384u * hf, lo + 16384u * hf, r, c8, x);
  }
}

// 32 consecutive floats of row `row`, columns 64 hf + 32 q .., as registers.
__device__ __forceinline__ void load_row32(const float* __restrict__ p, float (&v)[32]) {
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p) + e);
    v[4 * e] = a.x;
    v[4 * e + 1] = a.y;
    v[4 * e + 2] = a.z;
    v[4 * e + 3] = a.w;
  }
}

struct Fix {
  uint32_t sb, tmem, bar;
  volatile int* verdict;
  int* status;
  uint32_t phase;
  // The leader issued MMAs and committed them to `bar`; every thread waits for
  // them (bounded, decided by the leader) and the CTA agrees on the outcome.
  __device__ __forceinline__ bool wait_mma() {
    if (threadIdx.x == 0) {
      const bool ok = mbar_wait_bounded(bar, phase, WAIT_LIMIT_NS);
      *verdict = ok ? 0 : 1;
      if (!ok && status) atomicExch(status, GDN_ERR_DEVICE_TIMEOUT);
    }
    phase ^= 1u;
    __syncthreads();
    tc_fence_after();
    return *verdict == 0;
  }
};

// acc (TMEM, lane = row of S, column = column of F) = S F.  A = S (K-major),
// B = F (MN-major: K rows of 128 B, N blocks 16 KB apart).
__device__ __forceinline__ void issue_state_product(const Fix& f, uint32_t acc) {
  const uint32_t id = idesc_bf16(128, 128, 0, 1, 0);
#pragma unroll
  for (int part = 0; part < 3; ++part) {
    const uint32_t a = f.sb + (part == 2 ? SS_LO : SS_HI);
    const uint32_t bm = f.sb + (part == 1 ? SF_LO : SF_HI);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      mma_ss(acc, sdesc_sw128(a + (kk >> 2) * 16384u + (kk & 3) * 32u, 16, 1024),
             sdesc_sw128(bm + kk * 2048u, 16384, 1024), id, (part | kk) ? 1u : 0u);
    }
  }
}

// acc (TMEM, lane = dv, column = token of the tile) = S f^T.  B = f tile (K-major).
__device__ __forceinline__ void issue_output_product(const Fix& f, uint32_t acc) {
  const uint32_t id = idesc_bf16(128, 64, 0, 0, 0);
#pragma unroll
  for (int part = 0; part < 3; ++part) {
    const uint32_t a = f.sb + (part == 2 ? SS_LO : SS_HI);
    const uint32_t bm = f.sb + (part == 1 ? SQ_LO : SQ_HI);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const uint32_t ko = (kk & 3) * 32u;
      mma_ss(acc, sdesc_sw128(a + (kk >> 2) * 16384u + ko, 16, 1024),
             sdesc_sw128(bm + (kk >> 2) * 8192u + ko, 16, 1024), id, (part | kk) ? 1u : 0u);
    }
  }
}

__global__ void __launch_bounds__(NTHREADS, 1) segment_fix_kernel(const PrefillArgs p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nk = p.nseg - 1;
  const int chain = blockIdx.x / nk;
  const int k = blockIdx.x - chain * nk + 1;  // segment 1 .. nseg-1
  const int b = chain / p.H, h = chain - b * p.H;
  const size_t mat = size_t(D) * D;
  const float* R = p.ws_R + size_t(chain) * p.nseg * mat;
  const float* F = p.ws_F + size_t(chain) * p.nseg * mat;

  Fix f;
  f.sb = smem_u32(sm);
  f.bar = f.sb + SM_BAR;
  f.verdict = reinterpret_cast<volatile int*>(sm + SM_BAR + 8);
  f.status = p.status;
  f.phase = 0;
  if (tid == 0) {
    mbar_init(f.bar, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(sm + SM_BAR + 16), TMEM_COLS);
    tmem_relinquish();
  }
  // S_1 = R_0
  load_split_matrix(R, f.sb + SS_HI, f.sb + SS_LO);
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  f.tmem = *reinterpret_cast<volatile uint32_t*>(sm + SM_BAR + 16);

  // Warp w reads TMEM lanes 32 (w % 4) ..: its thread owns row `row` of the
  // accumulators, and the column half `hf`.
  const int row = (warp & 3) * 32 + lane, hf = warp >> 2;
  const uint32_t tlane = f.tmem + (uint32_t((warp & 3) * 32) << 16);
  bool ok = true;

  // S_{j+1} = S_j F_j + R_j for j = 1 .. k-1 (and j = k into S_T when k is last)
  const bool last = (k == p.nseg - 1);
  for (int j = 1; ok && j <= (last ? k : k - 1); ++j) {
    load_split_matrix(F + j * mat, f.sb + SF_HI, f.sb + SF_LO);
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      issue_state_product(f, f.tmem + TM_ACC);
      mma_commit(f.bar);
    }
    ok = f.wait_mma();
    if (!ok) break;
    if (j == k) break;  // the S_T product stays in TMEM until the o tiles are done
    const float* rrow = R + j * mat + size_t(row) * D + 64 * hf;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      float v[32], r[32];
      load_row32(rrow + 32 * q, r);
      tmem_ld32(tlane + TM_ACC + 64 * hf + 32 * q, v);
#pragma unroll
      for (int e = 0; e < 32; ++e) v[e] += r[e];
#pragma unroll
      for (int c8 = 0; c8 < 4; ++c8)
        store_split8(f.sb + SS_HI + 16384u * hf, f.sb + SS_LO + 16384u * hf, row, 4 * q + c8,
                     v + 8 * c8);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
  }

  // o_t += S_k f_t over the tokens of segment k, 64 at a time
  const int total_tiles = (p.T + NT - 1) / NT;
  const int tb = k * p.seg_tiles;
  const int te = min(total_tiles, tb + p.seg_tiles);
  for (int c = tb; ok && c < te; ++c) {
    {
      // thread -> token r = tid / 4, 32 features 32 (tid % 4) ..
      const int r = tid >> 2, qd = tid & 3;
      const int t = c * NT + r;
      const float4* src =
          reinterpret_cast<const float4*>(p.ws_f + ((size_t(b) * p.T + t) * p.H + h) * D + 32 * qd);
      const uint32_t blk = 8192u * uint32_t(qd >> 1);
      float x[32];
      if (t < p.T) {
        load_row32(reinterpret_cast<const float*>(src), x);
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) x[e] = 0.f;
      }
#pragma unroll
      for (int c8 = 0; c8 < 4; ++c8)
        store_split8(f.sb + SQ_HI + blk, f.sb + SQ_LO + blk, r, 4 * (qd & 1) + c8, x + 8 * c8);
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      issue_output_product(f, f.tmem + TM_O);
      mma_commit(f.bar);
    }
    ok = f.wait_mma();
    if (!ok) break;
    {
      // this thread: lane dv = row, tokens 32 hf .. 32 hf + 31 of the tile
      // all 32 loads of o first, then the stores (one global latency, not 32)
      const int t0 = c * NT + 32 * hf;
      const int nvalid = min(32, p.T - t0);
      float* orow = p.o + ((size_t(b) * p.T + t0) * p.H + h) * D + row;
      const size_t ts = size_t(p.H) * D;
      float cur[32];
#pragma unroll
      for (int n = 0; n < 32; ++n) cur[n] = (n < nvalid) ? orow[n * ts] : 0.f;
      float v[32];
      tmem_ld32(tlane + TM_O + 32 * hf, v);
#pragma unroll
      for (int n = 0; n < 32; ++n)
        if (n < nvalid) orow[n * ts] = cur[n] + v[n];
    }
    tc_fence_before();
    __syncthreads();
  }

  // S_T = S_k F_k + R_k (the product is already in TMEM)
  if (ok && last) {
    const float* rrow = R + k * mat + size_t(row) * D + 64 * hf;
    float* dst = p.S_T + size_t(chain) * mat + size_t(row) * D + 64 * hf;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      float v[32], r[32];
      load_row32(rrow + 32 * q, r);
      tmem_ld32(tlane + TM_ACC + 64 * hf + 32 * q, v);
#pragma unroll
      for (int e = 0; e < 8; ++e)
        reinterpret_cast<float4*>(dst + 32 * q)[e] =
            make_float4(v[4 * e] + r[4 * e], v[4 * e + 1] + r[4 * e + 1],
                        v[4 * e + 2] + r[4 * e + 2], v[4 * e + 3] + r[4 * e + 3]);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(f.tmem, TMEM_COLS);
}

}  // namespace

int launch_segment_fix(const PrefillArgs& a, cudaStream_t stream) {
  if (a.nseg <= 1) return 0;
  const int ctas = a.B * a.H * (a.nseg - 1);
  const uint32_t smem = SMEM_USED + 1024;
  if (!ensure_smem_attr(reinterpret_cast<const void*>(segment_fix_kernel), 2, int(smem))) return -1;
  segment_fix_kernel<<<ctas, NTHREADS, smem, stream>>>(a);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace gdn
