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
  // Segmented schedule.  nseg == 1: one CTA walks each chain from S0 to S_T.
  // nseg > 1: the tiles of a chain are cut into nseg segments of seg_tiles
  // tiles (the last may be shorter); the first pass runs, per segment k, an
  // "R" CTA (start from S0 for k = 0, else from zero; writes o and the end
  // state R_k) and, for k >= 1, an "F" CTA (start from the identity with
  // v = 0; writes f_t = F q_t like o and the transfer matrix F_k); the second
  // pass chains S_k+1 = S_k F_k + R_k and adds S_k f_t to o.
  int nseg, seg_tiles;
  int fix_parts;    // CTAs sharing the o correction of one segment in the second pass
  float* ws_f;      // f_t of the F CTAs, laid out like o            [B][T][H][128]
  float* ws_R;      // end state of each R CTA                         [B*H][nseg][128][128]
  float* ws_F;      // transfer matrix of each F CTA (slot 0 unused)   [B*H][nseg][128][128]
  // Packed sequences (or null): B sequences of lengths cu[n+1] - cu[n] packed
  // along T (the views then have one batch entry); chain n H + h walks
  // tokens [cu[n], cu[n+1]).
  const int* cu_seqlens;
  // State snapshots (packed sequences only; snaps == null: none): the state
  // after every snap_every tokens (a multiple of 64) of each sequence, at
  // snaps[(k_n + j) H + h] with k_n = sum over earlier sequences m of
  // len_m / snap_every; n_snaps slots in all.
  float* snaps;
  int snap_every, n_snaps;
  // q and k L2-normalised per token and head inside the kernel (nonzero), q
  // multiplied by q_scale afterwards (1: unchanged).  Set explicitly.
  int qk_norm;
  float q_scale;
  int o_bf16;  // o is bf16 (same layout); single-pass schedule only
  // Head dims: Dk (64 or 128) is the kernel's template parameter; Dv is 64,
  // 128 or 256.  dv_ctas CTAs share a chain, each owning dv_box = min(Dv, 128)
  // consecutive rows of its state (Dv = 256: two CTAs of 128 rows; Dv = 64:
  // one CTA whose rows 64..127 stay zero).
  int Dk, Dv, dv_ctas, dv_box;
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
  int T;  // tokens per sequence in this call (q, k, v, g, beta, o laid out [B][T][H])
  int qk_norm;    // as in PrefillArgs
  float q_scale;
  int o_bf16;     // o is bf16 (same layout)
  int vector_gate;  // g is [B][T][H][Dk], one log decay per key channel (no fused options)
  int head_dim;     // Dk = Dv: 128, or 64 (no fused options)
};

// Row-parallel fp32 kernel (any supported head dims; scalar or per-channel gate).
struct RowArgs {
  const __nv_bfloat16* q;  // [B][T][H][Dk]
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;  // [B][T][H][Dv]
  const float* g;          // [B][T][H][Dk] (per-channel gate) or [B][T][H]
  const float* beta;       // [B][T][H]
  const float* S_in;       // [B][H][Dv][Dk] or null (zeros)
  float* S_out;            // may equal S_in
  float* o;                // [B][T][H][Dv]
  int B, H, T, Dv;
};

// Chunked per-channel-gate (KDA) prefill on the tensor cores, Dk = Dv = 128.
struct KdaArgs {
  const float* g;     // [B][T][H][128] natural-log decays per key channel
  const float* beta;  // [B][T][H]
  const float* S0;    // [B][H][Dv][128] or null (zeros)
  float* S_T;         // may equal S0
  int B, T, H;
  int* status;        // may be null
  int qk_norm;        // q, k L2-normalised per token and head in the kernel
  float q_scale;      // q multiplied by this after the normalisation
  int Dv;             // 64, 128 or 256 (Dk is 128)
  int o_bf16;         // o written as bf16
  const int* cu_seqlens = nullptr;  // packed sequences: [B + 1] token offsets (views with B = 1)
  float* o = nullptr;               // o (fp32, or bf16 with o_bf16): the packed last tile's row copy
  float* snaps = nullptr;           // packed sequences: state snapshots, or null
  int snap_every = 0;               // tokens between snapshots (a multiple of 32)
  int n_snaps = 0;                  // slots in snaps
};

// Sets the dynamic shared-memory limit of `func` to `bytes` once per device
// (slot: a small per-kernel index); returns false if the attribute call failed.
bool ensure_smem_attr(const void* func, int slot, int bytes);

// Both return 0 on success, -1 when the launch failed.
// tq, tk, tv: bf16 inputs; to: o, tf: the f output of the transfer-matrix
// CTAs (ws_f; equal to `to` without segments) -- fp32, box 64 tokens x 128.
int launch_prefill(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                   const CUtensorMap& to, const CUtensorMap& tf, const PrefillArgs& a, int chunk,
                   cudaStream_t stream);
// tq, tk: bf16 q, k boxes of 64 features x 32 tokens (SW128); tv: bf16 v, and
// to: fp32 o, boxes of min(Dv, 128) features x 32 tokens, unswizzled; tg: fp32
// g, 128 x 32.  T > 0 and B*H > 0; Dk = 128, a.Dv 64, 128 or 256.
int launch_kda_prefill(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& to, const CUtensorMap& tg, const KdaArgs& a,
                       cudaStream_t stream);
int launch_decode(const DecodeArgs& a, cudaStream_t stream);
// Second pass of the segmented schedule (a.nseg > 1).
int launch_segment_fix(const PrefillArgs& a, cudaStream_t stream);
// Row-parallel recurrence (Dk, Dv in {64, 128, 256}); num_sms picks the rows
// per CTA.  Returns 0, or -1 when the dims are unsupported or the launch failed.
int launch_rows(const RowArgs& a, int Dk, bool vector_gate, int num_sms, cudaStream_t stream);
int rows_per_cta(long long heads, int Dv, int num_sms);
bool rows_head_dims_ok(int Dk, int Dv);

}  // namespace gdn
