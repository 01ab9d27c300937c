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
// Each warp owns ROWS_PER_WARP consecutive rows; lane l holds columns
// 4l..4l+3 of every row, so a row is one fully coalesced 512-byte access.
// All row loads of a warp are issued before any reduction (bytes in flight),
// and the loads/stores use the streaming cache hint: the state is touched
// once per step.
#include "gdn_internal.h"

namespace gdn {
namespace {

constexpr int D = 128;
constexpr int ROWS_PER_WARP = 8;
constexpr int WARPS = 4;
constexpr int ROWS_PER_CTA = ROWS_PER_WARP * WARPS;  // 32
constexpr int CTAS_PER_HEAD = D / ROWS_PER_CTA;      // 4

__device__ __forceinline__ float4 bf16x4_to_float4(uint2 raw) {
  const __nv_bfloat162 lo = *reinterpret_cast<const __nv_bfloat162*>(&raw.x);
  const __nv_bfloat162 hi = *reinterpret_cast<const __nv_bfloat162*>(&raw.y);
  const float2 a = __bfloat1622float2(lo);
  const float2 b = __bfloat1622float2(hi);
  return make_float4(a.x, a.y, b.x, b.y);
}

__device__ __forceinline__ float dot4(const float4& a, const float4& b) {
  return fmaf(a.x, b.x, fmaf(a.y, b.y, fmaf(a.z, b.z, a.w * b.w)));
}

__global__ void __launch_bounds__(WARPS * 32) decode_kernel(const DecodeArgs a) {
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int head = blockIdx.x / CTAS_PER_HEAD;  // b * H + h
  const int row0 = (blockIdx.x % CTAS_PER_HEAD) * ROWS_PER_CTA + warp * ROWS_PER_WARP;

  float4* srow = reinterpret_cast<float4*>(a.S + (size_t(head) * D + row0) * D) + lane;
  float4 s[ROWS_PER_WARP];
#pragma unroll
  for (int r = 0; r < ROWS_PER_WARP; ++r) s[r] = __ldcs(srow + r * (D / 4));

  const float4 k4 = bf16x4_to_float4(*reinterpret_cast<const uint2*>(a.k + size_t(head) * D + 4 * lane));
  const float4 q4 = bf16x4_to_float4(*reinterpret_cast<const uint2*>(a.q + size_t(head) * D + 4 * lane));
  const uint4 vraw = *reinterpret_cast<const uint4*>(a.v + size_t(head) * D + row0);
  const float alpha = expf(a.g[head]);
  const float beta = a.beta[head];

  float kq = dot4(k4, q4);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) kq += __shfl_xor_sync(0xffffffffu, kq, off);

  float sk[ROWS_PER_WARP], sq[ROWS_PER_WARP];
#pragma unroll
  for (int r = 0; r < ROWS_PER_WARP; ++r) {
    sk[r] = dot4(s[r], k4);
    sq[r] = dot4(s[r], q4);
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
    float4 x = s[r];
    x.x = fmaf(alpha, x.x, d * k4.x);
    x.y = fmaf(alpha, x.y, d * k4.y);
    x.z = fmaf(alpha, x.z, d * k4.z);
    x.w = fmaf(alpha, x.w, d * k4.w);
    __stcs(srow + r * (D / 4), x);
    const float o = fmaf(alpha, sq[r], d * kq);
    if (lane == r) o_mine = o;
  }
  if (lane < ROWS_PER_WARP) a.o[size_t(head) * D + row0 + lane] = o_mine;
}

}  // namespace

int launch_decode(const DecodeArgs& a, cudaStream_t stream) {
  const long long heads = (long long)a.B * a.H;
  if (heads == 0) return 0;
  decode_kernel<<<unsigned(heads * CTAS_PER_HEAD), WARPS * 32, 0, stream>>>(a);
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace gdn
