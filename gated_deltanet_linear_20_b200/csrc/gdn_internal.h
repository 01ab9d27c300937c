// Internal declarations shared by the C-ABI layer and the kernel files.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "../../include/gdn.h"

namespace gdn {

struct PrefillArgs {
  const float* g;
  const float* beta;
  const float* S0;  // may be null (zeros)
  float* o;
  float* S_T;
  int B, T, H;
  int* status;      // may be null
};

struct DecodeArgs {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const float* g;
  const float* beta;
  float* S;
  float* o;
  int B, H;
};

// Both return 0 on success, -1 when the launch failed.
int launch_prefill(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                   const PrefillArgs& a, int chunk, cudaStream_t stream);
int launch_decode(const DecodeArgs& a, cudaStream_t stream);

}  // namespace gdn
