// Test-only kernel: runs one tcgen05.mma configuration of the kinds the
// prefill kernel uses on a single 128x128 tile and writes the fp32 result, so
// that descriptor encodings, operand majors, A-from-tensor-memory, sub-block
// offsets and operand negation can each be checked against a host matmul.
//
// Modes (A is [128 m][128 k] bf16 row-major; D is [128 m][128 n] fp32):
//   0: D = A B^T, B [128 n][128 k] K-major (SW128), N = 128
//   1: D = A B,   B [128 k][128 n] MN-major (SW128, two 64-column blocks), N = 128
//   2: D = A B^T with A read from tensor memory (bf16 pairs per column), N = 128
//   3: D[:, 0:16] = A[:, 16:32] B[32:48, 16:32]^T (one K=16 step, N=16, offsets in both)
//   4: D = 1 - A B^T (D preset to 1 by tcgen05.st, A negated in the instruction)
//   5: D[:, 0:64] = A B[0:64]^T, N = 64
//   6: D[:, 0:64] = A^T B[0:64]^T with A read MN-major: the tile holds A's rows
//      (index k) with m contiguous in two 64-m blocks 16 KB apart, N = 64
//   7: D[:, 0:64] = A[0:64]^T B[0:64, 0:64]^T, A MN-major over 64 k rows in two
//      64-m blocks 8 KB apart (K = 64: four K=16 steps), N = 64
//   8: D[:, 0:64] = A B'^T with B' MN-major: the tile holds B's rows (index k)
//      with n contiguous, N = 64 (one 64-n block), K = 128
#include <cstdint>

#include "sm100.cuh"

using namespace gdn::sm100;

namespace {

__device__ __forceinline__ uint32_t sw_off(int r, int c) {
  return uint32_t((r >> 3) * 1024 + (r & 7) * 128 + (((c ^ r) & 7) << 4));
}

__global__ void __launch_bounds__(128, 1)
    umma_selftest_kernel(const __nv_bfloat16* __restrict__ A, const __nv_bfloat16* __restrict__ B,
                         float* __restrict__ Dout, int mode, int* status) {
  extern __shared__ uint8_t raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(sm);
  const uint32_t sa = sb, sbB = sb + 32768;  // A: 2 boxes x 16 KB; B: 2 boxes x 16 KB
  const uint32_t bar = sb + 65536;
  uint32_t* slot = reinterpret_cast<uint32_t*>(sm + 65536 + 16);
  const int tid = threadIdx.x, warp = tid >> 5;

  // A row tid -> K-major SW128, two boxes of 64 k
  for (int c = 0; c < 16; ++c) {
    const uint4 v = *reinterpret_cast<const uint4*>(A + tid * 128 + c * 8);
    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(sa + (c >> 3) * 16384 + sw_off(tid, c & 7)),
                 "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w));
  }
  // B row tid: K-major ([n][k]) or MN-major ([k][n], rows are k, two 64-n blocks)
  for (int c = 0; c < 16; ++c) {
    const uint4 v = *reinterpret_cast<const uint4*>(B + tid * 128 + c * 8);
    asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(sbB + (c >> 3) * 16384 + sw_off(tid, c & 7)),
                 "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w));
  }
  if (mode == 7) {
    // rows k < 64 only: A[k][0:64] in block 0, A[k][64:128] in block 1 (8 KB apart)
    __syncthreads();
    if (tid < 64) {
      for (int c = 0; c < 16; ++c) {
        const uint4 v = *reinterpret_cast<const uint4*>(A + tid * 128 + c * 8);
        asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(sa + (c >> 3) * 8192 + sw_off(tid, c & 7)),
                     "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w));
      }
    }
  }
  fence_proxy_async_smem();
  if (tid == 0) {
    mbar_init(bar, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;
  const uint32_t tlane = tmem + (uint32_t(warp * 32) << 16);
  const uint32_t TD = 0, TA = 256;

  if (mode == 2) {  // A row tid -> TMEM columns TA.. as bf16 pairs
    for (int g = 0; g < 4; ++g) {
      uint32_t u[16];
      for (int e = 0; e < 16; ++e)
        u[e] = *reinterpret_cast<const uint32_t*>(A + tid * 128 + 32 * g + 2 * e);
      tmem_st16(tlane + TA + 16 * g, u);
    }
  }
  if (mode == 4) {
    uint32_t one[16];
    for (int e = 0; e < 16; ++e) one[e] = __float_as_uint(1.f);
    for (int g = 0; g < 8; ++g) tmem_st16(tlane + TD + 16 * g, one);
  }
  tc_fence_before();
  __syncthreads();

  if (tid == 0) {
    tc_fence_after();
    for (int kk = 0; kk < 8; ++kk) {
      const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
      const uint64_t ad = sdesc_sw128(sa + off, 16, 1024);
      if (mode == 0) {
        mma_ss(tmem + TD, ad, sdesc_sw128(sbB + off, 16, 1024), idesc_bf16(128, 128, 0, 0, 0), kk > 0);
      } else if (mode == 1) {
        // B rows are k: 16 k per step = 2 row groups of 1024 B; k >= 64 lives in rows 64.. of
        // the same 64-n block (rows 0..127 of each block), blocks 16 KB apart.
        mma_ss(tmem + TD, ad, sdesc_sw128(sbB + kk * 2048, 16384, 1024), idesc_bf16(128, 128, 0, 1, 0), kk > 0);
      } else if (mode == 2) {
        mma_ts(tmem + TD, tmem + TA + kk * 8, sdesc_sw128(sbB + off, 16, 1024), idesc_bf16(128, 128, 0, 0, 0), kk > 0);
      } else if (mode == 3) {
        if (kk == 1)
          mma_ss(tmem + TD, sdesc_sw128(sa + 32, 16, 1024), sdesc_sw128(sbB + 4096 + 32, 16, 1024),
                 idesc_bf16(128, 16, 0, 0, 0), 0);
      } else if (mode == 4) {
        mma_ss(tmem + TD, ad, sdesc_sw128(sbB + off, 16, 1024), idesc_bf16(128, 128, 0, 0, 1), 1);
      } else if (mode == 5) {
        mma_ss(tmem + TD, ad, sdesc_sw128(sbB + off, 16, 1024), idesc_bf16(128, 64, 0, 0, 0), kk > 0);
      } else if (mode == 6) {
        mma_ss(tmem + TD, sdesc_sw128(sa + kk * 2048, 16384, 1024), sdesc_sw128(sbB + off, 16, 1024),
               idesc_bf16(128, 64, 1, 0, 0), kk > 0);
      } else if (mode == 7) {
        if (kk < 4)
          mma_ss(tmem + TD, sdesc_sw128(sa + kk * 2048, 8192, 1024), sdesc_sw128(sbB + kk * 32, 16, 1024),
                 idesc_bf16(128, 64, 1, 0, 0), kk > 0);
      } else if (mode == 8) {
        mma_ss(tmem + TD, ad, sdesc_sw128(sbB + kk * 2048, 16384, 1024), idesc_bf16(128, 64, 0, 1, 0), kk > 0);
      }
    }
    mma_commit(bar);
  }
  if (!mbar_wait_bounded(bar, 0, 1000000000ull)) {
    if (tid == 0) atomicExch(status, -7);
  }
  tc_fence_after();
  for (int g = 0; g < 8; ++g) {
    float r[16];
    tmem_ld16(tlane + TD + 16 * g, r);
    for (int e = 0; e < 16; ++e) Dout[tid * 128 + 16 * g + e] = r[e];
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
}


// Issue-rate probe: tcgen05.mma (kind::f16, M = 128, N = 32/64/128/256 by
// mode & 3) on zeroed operands; records, per CTA, the wall time of the issue
// loop and the time until the products have completed (ns).
//   mode & 4 : A from tensor memory (else shared memory)
//   mode & 8 : consecutive MMAs rotate over 4 accumulators (N <= 128, A from
//              shared memory) instead of all accumulating into one
//   mode & 16: two threads (warps 0 and 1) each issue half of the MMAs, into
//              accumulators 256 columns apart (N <= 128, A from shared memory)
__global__ void __launch_bounds__(128, 1) umma_issue_kernel(int mode, int n_mma,
                                                             unsigned long long* out, int* status) {
  extern __shared__ uint8_t raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sb = smem_u32(sm);
  const uint32_t bar = sb + 65536;
  uint32_t* slot = reinterpret_cast<uint32_t*>(sm + 65536 + 16);
  const int tid = threadIdx.x, warp = tid >> 5;
  for (int i = tid; i < 65536 / 16; i += 128) reinterpret_cast<uint4*>(sm)[i] = make_uint4(0, 0, 0, 0);
  fence_proxy_async_smem();
  if (tid == 0) {
    mbar_init(bar, 1);
    mbar_init(bar + 8, 1);  // the second issuer's completion
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *slot;
  const bool two = (mode & 16) != 0;
  if (tid == 0 || (two && tid == 32)) {
    // A: 128 rows x 128 B at sb (K-major); B: up to 256 rows x 128 B at sb + 32 KB;
    // D: TMEM columns from 0 (rotating: 0, 128, 256, 384; second issuer: 256 ..);
    // A from TMEM: columns 256 .. 319
    const uint64_t a = sdesc_sw128(sb, 16, 1024), b = sdesc_sw128(sb + 32768, 16, 1024);
    const int N = (mode & 3) == 0 ? 64 : (mode & 3) == 1 ? 128 : (mode & 3) == 2 ? 256 : 32;
    const uint32_t id = idesc_bf16(128, N, 0, 0, 0);
    const uint32_t dbase = tmem + (tid == 32 ? 256u : 0u);
    const int n = two ? n_mma / 2 : n_mma;
    const unsigned long long t0 = globaltimer_ns();
    for (int i = 0; i < n; ++i) {
      const uint32_t kk = i & 3;
      if (mode & 4)
        mma_ts(dbase, tmem + 256 + kk * 8, sdesc_add(b, kk * 32), id, 1u);
      else if (mode & 8)
        mma_ss(dbase + 128u * (i & 3), sdesc_add(a, kk * 32), sdesc_add(b, kk * 32), id, 1u);
      else
        mma_ss(dbase, sdesc_add(a, kk * 32), sdesc_add(b, kk * 32), id, 1u);
    }
    const unsigned long long t1 = globaltimer_ns();
    mma_commit(bar + (tid == 32 ? 8u : 0u));
    if (!mbar_wait_bounded(bar + (tid == 32 ? 8u : 0u), 0, 1000000000ull)) atomicExch(status, -7);
    const unsigned long long t2 = globaltimer_ns();
    if (tid == 0) {
      out[2 * blockIdx.x] = t1 - t0;
      out[2 * blockIdx.x + 1] = t2 - t0;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace

extern "C" int umma_selftest(const void* A, const void* B, float* D, int mode, int* status,
                             void* stream) {
  const int smem = 65536 + 1024 + 64;
  if (cudaFuncSetAttribute(umma_selftest_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
      cudaSuccess)
    return -1;
  umma_selftest_kernel<<<1, 128, smem, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const __nv_bfloat16*>(A), static_cast<const __nv_bfloat16*>(B), D, mode, status);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

extern "C" int umma_issue_probe(int mode, int n_mma, int ctas, unsigned long long* out, int* status,
                                void* stream) {
  const int smem = 65536 + 1024 + 64;
  if (mode < 0 || mode > 31 || ((mode & 24) && ((mode & 4) || (mode & 3) == 2)) || n_mma < 2 ||
      ctas < 1 ||
      cudaFuncSetAttribute(umma_issue_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
          cudaSuccess)
    return -1;
  umma_issue_kernel<<<ctas, 128, smem, static_cast<cudaStream_t>(stream)>>>(mode, n_mma, out, status);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}
