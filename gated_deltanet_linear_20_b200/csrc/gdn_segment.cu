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
// The chained state S lives in tensor memory as a bf16 hi/lo pair (the A
// operand of every product, lane = row).  Shared memory (offsets from a
// 1024-byte aligned base):
//   F hi/lo: the transfer matrix as the MN-major B operand, two 16 KB SW128
//     blocks each (block h: columns 64h .. 64h+63, rows = K); the f tile (two
//     8 KB blocks of 64 token rows, K-major B) reuses it once the products are done;
//   two fp32 staging buffers filled by cp.async (row pitch 528 B, so that eight
//   consecutive rows read as float4 hit distinct banks): one for the next
//   transfer matrix (or two f tiles), one for R_j and finally S_T.
constexpr uint32_t SF_HI = 0, SF_LO = 32768;
constexpr uint32_t SQ_HI = SF_HI, SQ_LO = SF_HI + 16384;
constexpr uint32_t PITCH = 528;                  // bytes per staged fp32 row
constexpr uint32_t STAGE_BYTES = 128 * PITCH;
constexpr uint32_t SSTAGE = 65536;               // F_{j+1}, then f tiles
constexpr uint32_t STAGE_TILE = 64 * PITCH;      // one staged f tile
constexpr uint32_t RSTAGE = SSTAGE + STAGE_BYTES;  // R_j, then S_T
constexpr uint32_t SM_BAR = RSTAGE + STAGE_BYTES;  // mbarrier, verdict, TMEM slot
constexpr uint32_t SMEM_USED = SM_BAR + 64;
static_assert(SMEM_USED + 1024 <= 232448, "shared memory budget");
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TM_ACC = 0, TM_SHI = 128, TM_SLO = 192, TM_O = 256;
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all_but_one() {
  asm volatile("cp.async.wait_group 1;" ::: "memory");
}

// Row-major 128 x 128 fp32 matrix -> staging buffer (asynchronous; 16 chunks
// of 16 B per thread, consecutive threads on consecutive chunks).
__device__ __forceinline__ void stage_matrix(uint32_t stage, const float* __restrict__ src) {
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const int c = threadIdx.x + NTHREADS * i;  // chunk: row c / 32, 16-byte column c % 32
    cp_async16(stage + uint32_t(c >> 5) * PITCH + uint32_t(c & 31) * 16u, src + 4 * c);
  }
  cp_async_commit();
}

// f_t rows of the tokens t0 .. t0+63 of chain (b, h) -> one staged tile
// (tokens at or past T are skipped; the split zeroes them).
__device__ __forceinline__ void stage_f_tile(uint32_t stage, const PrefillArgs& p, int b, int h,
                                             int t0) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int c = threadIdx.x + NTHREADS * i;  // chunk: token row c / 32, column c % 32
    const int t = t0 + (c >> 5);
    if (t < p.T)
      cp_async16(stage + uint32_t(c >> 5) * PITCH + uint32_t(c & 31) * 16u,
                 p.ws_f + ((size_t(b) * p.T + t) * p.H + h) * D + 4 * (c & 31));
  }
  cp_async_commit();
}

__device__ __forceinline__ float4 lds4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}
__device__ __forceinline__ void sts4(uint32_t addr, float4 v) {
  st_shared_v4(addr, __float_as_uint(v.x), __float_as_uint(v.y), __float_as_uint(v.z),
               __float_as_uint(v.w));
}

// Staged 128 x 128 matrix -> hi/lo SW128 blocks (the MN-major B operand).
// Thread t: row t % 128, columns 64 (t / 128) ..; eight consecutive threads
// read eight rows.
__device__ __forceinline__ void split_staged_matrix(uint32_t stage, uint32_t hi, uint32_t lo) {
  const int r = threadIdx.x & 127, hf = threadIdx.x >> 7;
  const uint32_t row = stage + uint32_t(r) * PITCH + uint32_t(hf) * 256u;
#pragma unroll
  for (int c8 = 0; c8 < 8; ++c8) {
    const float4 a = lds4(row + 32u * c8), b = lds4(row + 32u * c8 + 16u);
    const float x[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    store_split8(hi + 16384u * hf, lo + 16384u * hf, r, c8, x);
  }
}

// Staged f tile -> hi/lo K-major blocks (rows = tokens).  Thread t: token row
// t % 64, features 32 (t / 64) ..; rows at or past T become zeros.
__device__ __forceinline__ void split_staged_f(uint32_t stage, uint32_t hi, uint32_t lo, int nrows) {
  const int r = threadIdx.x & 63, qd = threadIdx.x >> 6;
  const uint32_t row = stage + uint32_t(r) * PITCH + uint32_t(qd) * 128u;
  const uint32_t blk = 8192u * uint32_t(qd >> 1);
#pragma unroll
  for (int c8 = 0; c8 < 4; ++c8) {
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
    if (r < nrows) {
      a = lds4(row + 32u * c8);
      b = lds4(row + 32u * c8 + 16u);
    }
    const float x[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    store_split8(hi + blk, lo + blk, r, 4 * (qd & 1) + c8, x);
  }
}

// 32 staged floats of row `row` starting at column `col` (epilogue mapping:
// lane = row, so eight consecutive lanes read eight rows).
__device__ __forceinline__ void lds_row32(uint32_t stage, int row, int col, float (&v)[32]) {
  const uint32_t a = stage + uint32_t(row) * PITCH + uint32_t(col) * 4u;
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float4 x = lds4(a + 16u * e);
    v[4 * e] = x.x;
    v[4 * e + 1] = x.y;
    v[4 * e + 2] = x.z;
    v[4 * e + 3] = x.w;
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

// acc (TMEM, lane = row of S, column = column of F) = S F.  A = S hi / lo in
// TMEM, B = F (MN-major: K rows of 128 B, N blocks 16 KB apart).
__device__ __forceinline__ void issue_state_product(const Fix& f, uint32_t acc) {
  const uint32_t id = idesc_bf16(128, 128, 0, 1, 0);
  const uint64_t d0 = sdesc_sw128(f.sb, 16384, 1024);
#pragma unroll
  for (int part = 0; part < 3; ++part) {
    const uint32_t a = f.tmem + (part == 2 ? TM_SLO : TM_SHI);
    const uint32_t bm = part == 1 ? SF_LO : SF_HI;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
      mma_ts(acc, a + 8u * kk, sdesc_add(d0, bm + kk * 2048u), id, (part | kk) ? 1u : 0u);
  }
}

// acc (TMEM, lane = dv, column = token of the tile) = S f^T.  B = f tile (K-major).
__device__ __forceinline__ void issue_output_product(const Fix& f, uint32_t acc) {
  const uint32_t id = idesc_bf16(128, 64, 0, 0, 0);
  const uint64_t d0 = sdesc_sw128(f.sb, 16, 1024);
#pragma unroll
  for (int part = 0; part < 3; ++part) {
    const uint32_t a = f.tmem + (part == 2 ? TM_SLO : TM_SHI);
    const uint32_t bm = part == 1 ? SQ_LO : SQ_HI;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
      mma_ts(acc, a + 8u * kk, sdesc_add(d0, bm + (kk >> 2) * 8192u + (kk & 3) * 32u), id,
             (part | kk) ? 1u : 0u);
  }
}

// Writes 32 consecutive state values (columns col .. col+31 of this lane's row)
// as bf16 hi/lo pairs into the state's TMEM columns.
__device__ __forceinline__ void store_state32(uint32_t tlane, int col, const float (&v)[32]) {
  uint32_t hi[16], lo[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) split2_bf16(v[2 * e], v[2 * e + 1], hi[e], lo[e]);
  tmem_st16x2(tlane + TM_SHI + col / 2, hi, tlane + TM_SLO + col / 2, lo);
}

__global__ void __launch_bounds__(NTHREADS, 1) segment_fix_kernel(const PrefillArgs p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // CTA -> (chain, segment k >= 1, part of the segment's o correction)
  const int per = (p.nseg - 1) * p.fix_parts;
  const int chain = blockIdx.x / per;
  const int rem = blockIdx.x - chain * per;
  const int k = rem / p.fix_parts + 1;  // segment 1 .. nseg-1
  const int part = rem - (k - 1) * p.fix_parts;
  const int b = chain / p.H, h = chain - b * p.H;
  const size_t mat = size_t(D) * D;
  const float* R = p.ws_R + size_t(chain) * p.nseg * mat;
  const float* F = p.ws_F + size_t(chain) * p.nseg * mat;
  const bool last = (k == p.nseg - 1) && part == 0;  // this CTA also forms S_T
  const int nprod = last ? k : k - 1;  // chained products S_j F_j, j = 1 .. nprod
  // R_j is added after product j for j < k, and after the last product (j = k)
  // of the last segment, where it completes S_T
  auto need_r = [&](int j) { return j < k || (last && j == k); };

  Fix f;
  f.sb = smem_u32(sm);
  f.bar = f.sb + SM_BAR;
  f.verdict = reinterpret_cast<volatile int*>(sm + SM_BAR + 8);
  f.status = p.status;
  f.phase = 0;
  const uint32_t stage = f.sb + SSTAGE, rstage = f.sb + RSTAGE;

  // Prologue: set-up first (this grid may be launched before the first pass
  // has finished), then wait for the first pass and stream R_0 (= S_1) and F_1
  // into the two staging buffers.
  if (tid == 0) {
    mbar_init(f.bar, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(sm + SM_BAR + 16), TMEM_COLS);
    tmem_relinquish();
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");
  stage_matrix(rstage, R);
  if (nprod >= 1) stage_matrix(stage, F + mat);
  if (nprod >= 1) cp_async_wait_all_but_one(); else cp_async_wait_all();
  tc_fence_before();
  __syncthreads();  // R_0 staged, TMEM allocated
  tc_fence_after();
  f.tmem = *reinterpret_cast<volatile uint32_t*>(sm + SM_BAR + 16);

  // Warp w reads TMEM lanes 32 (w % 4) ..: its thread owns row `row` of the
  // accumulators, and the column half `hf`.
  const int row = (warp & 3) * 32 + lane, hf = warp >> 2;
  const uint32_t tlane = f.tmem + (uint32_t((warp & 3) * 32) << 16);
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    float v[32];
    lds_row32(rstage, row, 64 * hf + 32 * q, v);
    store_state32(tlane, 64 * hf + 32 * q, v);
  }
  tc_fence_before();
  __syncthreads();  // S_1 in TMEM; the R staging buffer is free
  if (need_r(1)) stage_matrix(rstage, R + mat);
  bool ok = true;

  // S_{j+1} = S_j F_j + R_j for j = 1 .. k-1; for the last segment also
  // S_k F_k, kept in TMEM for S_T.  F_{j+1} streams in during product j, and
  // R_{j+1} during the epilogue of product j + 1's predecessor.
  // cp.async groups complete in commit order: F_j was committed before R_j,
  // and R_j before F_{j+1}.
  for (int j = 1; ok && j <= nprod; ++j) {
    if (need_r(j)) cp_async_wait_all_but_one(); else cp_async_wait_all();
    __syncthreads();                                   // F_j staged (R_j may be in flight)
    split_staged_matrix(stage, f.sb + SF_HI, f.sb + SF_LO);
    fence_proxy_async_smem();
    __syncthreads();                                   // staging free, SF ready
    if (tid == 0) {
      tc_fence_after();
      issue_state_product(f, f.tmem + TM_ACC);
      mma_commit(f.bar);
    }
    if (j < nprod) stage_matrix(stage, F + (j + 1) * mat);
    if (j < k) {                                       // R_j staged (F_{j+1} may be in flight)
      if (j < nprod) cp_async_wait_all_but_one(); else cp_async_wait_all();
    }
    ok = f.wait_mma();                                 // (its barrier publishes R_j)
    if (!ok || j == k) break;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      float v[32], r[32];
      lds_row32(rstage, row, 64 * hf + 32 * q, r);
      tmem_ld32(tlane + TM_ACC + 64 * hf + 32 * q, v);
#pragma unroll
      for (int e = 0; e < 32; ++e) v[e] += r[e];
      store_state32(tlane, 64 * hf + 32 * q, v);
    }
    tc_fence_before();
    __syncthreads();                                   // S_{j+1} in TMEM; R staging free
    if (need_r(j + 1)) stage_matrix(rstage, R + (j + 1) * mat);
  }

  // o_t += S_k f_t over the tokens of segment k, 64 at a time; tile i + 1
  // streams into the other staging half while tile i is multiplied.
  const int total_tiles = (p.T + NT - 1) / NT;
  const int sb0 = k * p.seg_tiles, se0 = min(total_tiles, sb0 + p.seg_tiles);
  const int per_part = (se0 - sb0 + p.fix_parts - 1) / p.fix_parts;
  const int tb = min(se0, sb0 + part * per_part);
  const int te = min(se0, tb + per_part);
  if (ok && tb < te) stage_f_tile(stage, p, b, h, tb * NT);
  for (int c = tb; ok && c < te; ++c) {
    const uint32_t st = stage + uint32_t((c - tb) & 1) * STAGE_TILE;
    cp_async_wait_all();
    __syncthreads();                                   // tile c staged
    split_staged_f(st, f.sb + SQ_HI, f.sb + SQ_LO, min(NT, p.T - c * NT));
    fence_proxy_async_smem();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      issue_output_product(f, f.tmem + TM_O);
      mma_commit(f.bar);
    }
    if (c + 1 < te) stage_f_tile(stage + uint32_t((c + 1 - tb) & 1) * STAGE_TILE, p, b, h, (c + 1) * NT);
    // this thread: lane dv = row, tokens 32 hf .. 32 hf + 31 of the tile; the
    // loads of o go out before the wait
    const int t0 = c * NT + 32 * hf;
    const int nvalid = min(32, p.T - t0);
    float* orow = p.o + ((size_t(b) * p.T + t0) * p.H + h) * D + row;
    const size_t ts = size_t(p.H) * D;
    float cur[32];
#pragma unroll
    for (int n = 0; n < 32; ++n) cur[n] = (n < nvalid) ? orow[n * ts] : 0.f;
    ok = f.wait_mma();
    if (!ok) break;
    float v[32];
    tmem_ld32(tlane + TM_O + 32 * hf, v);
#pragma unroll
    for (int n = 0; n < 32; ++n)
      if (n < nvalid) orow[n * ts] = cur[n] + v[n];
    tc_fence_before();
    __syncthreads();
  }
  cp_async_wait_all();
  __syncthreads();  // R_k staged (last segment)

  // S_T = S_k F_k + R_k (the product is in TMEM): each thread adds its part in
  // the R staging buffer, then the CTA copies the buffer out row by row.
  if (ok && last) {
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int col = 64 * hf + 32 * q;
      float v[32], r[32];
      lds_row32(rstage, row, col, r);
      tmem_ld32(tlane + TM_ACC + col, v);
      const uint32_t a = rstage + uint32_t(row) * PITCH + uint32_t(col) * 4u;
#pragma unroll
      for (int e = 0; e < 8; ++e)
        sts4(a + 16u * e, make_float4(v[4 * e] + r[4 * e], v[4 * e + 1] + r[4 * e + 1],
                                      v[4 * e + 2] + r[4 * e + 2], v[4 * e + 3] + r[4 * e + 3]));
    }
    __syncthreads();
    float4* dst = reinterpret_cast<float4*>(p.S_T + size_t(chain) * mat);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int c = tid + NTHREADS * i;  // chunk: row c / 32, 16-byte column c % 32
      dst[c] = lds4(rstage + uint32_t(c >> 5) * PITCH + uint32_t(c & 31) * 16u);
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
  const int ctas = a.B * a.H * (a.nseg - 1) * a.fix_parts;
  const uint32_t smem = SMEM_USED + 1024;
  if (!ensure_smem_attr(reinterpret_cast<const void*>(segment_fix_kernel), 2, int(smem))) return -1;
  // programmatic dependent launch: the kernel's set-up overlaps the end of the
  // first pass; griddepcontrol.wait inside orders every access to its outputs
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(ctas));
  cfg.blockDim = dim3(NTHREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, segment_fix_kernel, a) == cudaSuccess ? 0 : -1;
}

}  // namespace gdn
