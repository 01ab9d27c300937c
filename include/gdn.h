/*
 * gdn.h -- C ABI of libgdn_b200.so: the gated delta rule (gated DeltaNet
 * linear attention) on NVIDIA B200 (sm_100a).
 *
 * The operation.  For every sequence b and head h independently, with the
 * state S in R^{Dv x Dk}:
 *
 *     alpha_t = exp(g_t)
 *     S_t     = alpha_t * S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *     o_t     = S_t q_t
 *
 * This is the recurrence of the linear-attention layers of the hybrid
 * Qwen 3.5 models.  The ROCmFPX gated-delta-net prefill note
 * (bittide.aicompass.dev article d2880479, opening post) describes its prefill
 * in this setting: a scalar gate per token and head, head dim 128, one
 * sequence per call, 16-token chunks, and the state held in F32 accumulators.
 * Its decode step is the per-layer recurrence fused into the Megakernel of the
 * Lucebox contribution guide (discosf.com/news/5165879, section 4, "CUDA/HIP
 * kernel optimisation: the Megakernel example").
 *
 * Layouts.  Every array is dense and row-major (last index fastest):
 *     q, k      [B][T][H][Dk]   bf16
 *     v         [B][T][H][Dv]   bf16
 *     g, beta   [B][T][H]       fp32   (g is the natural log of alpha)
 *     S0, S_T   [B][H][Dv][Dk]  fp32   (row i of S is contiguous in Dk)
 *     o         [B][T][H][Dv]   fp32
 * The decode step drops the T index.  q and k are used as given: callers
 * normalise or scale them beforehand if their model does so.
 *
 * Ownership and execution.  All pointers are DEVICE pointers owned by the
 * caller.  The library allocates no device memory and is safe to call from
 * several host threads; between calls it keeps only host-side caches (per
 * device: compute capability, SM count, kernel attributes already set).  Work is enqueued on
 * `stream` (a cudaStream_t; NULL means the legacy default stream) and the call
 * returns before it completes.  S_T may be the same buffer as S0 (each chain
 * reads its S0 before writing its S_T); neither o nor S_T may overlap q, k, v,
 * g or beta, and o may not overlap the state.
 *
 * Errors.  A negative return value means nothing was launched:
 *     GDN_ERR_NULL         a required pointer is NULL
 *     GDN_ERR_ALIGN        q/k/v/o/S pointers must be 16-byte aligned, g/beta 4-byte
 *     GDN_ERR_SHAPE        a size is negative or the problem exceeds 2^31-1 elements
 *     GDN_ERR_UNSUPPORTED  a head dim not in {64, 128, 256}; fused options where
 *                          the kernel serving the head dims has none (prefill
 *                          with Dk = 256; decode outside 64 x 64 and 128 x 128;
 *                          the per-channel-gate prefill with Dk other than 128);
 *                          packed sequences with Dk = 256;
 *                          chunk not in {16, 64}; or the current device is not
 *                          compute capability 10.0
 *     GDN_ERR_ALIAS        o or S_T overlaps an input, or o overlaps the state
 *     GDN_ERR_LAUNCH       the CUDA launch (or a CUDA runtime query) failed
 *     GDN_ERR_WORKSPACE    gdn_prefill_ws: workspace NULL, misaligned (256 B) or
 *                          smaller than gdn_prefill_workspace_bytes asked for
 *     GDN_ERR_STATIC_WORKSPACE_LIMIT  gdn_prefill_static_ws: the problem needs more
 *                          scratch than GDN_STATIC_WORKSPACE_BYTES
 * Device-side waits are bounded: if one gives up, the kernel writes
 * GDN_ERR_DEVICE_TIMEOUT to *status (when status is non-NULL), releases its
 * tensor memory and returns; read it with gdn_query_status.  The kernels never
 * trap and never print.
 */
#ifndef GDN_B200_H_
#define GDN_B200_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

#define GDN_ABI_VERSION 8

enum gdn_status_code {
  GDN_OK = 0,
  GDN_ERR_NULL = -1,
  GDN_ERR_ALIGN = -2,
  GDN_ERR_SHAPE = -3,
  GDN_ERR_UNSUPPORTED = -4,
  GDN_ERR_ALIAS = -5,
  GDN_ERR_LAUNCH = -6,
  GDN_ERR_DEVICE_TIMEOUT = -7,
  GDN_ERR_WORKSPACE = -8,
  GDN_ERR_STATIC_WORKSPACE_LIMIT = -9
};

/* Size of the library's built-in device scratch used by gdn_prefill_static_ws. */
#define GDN_STATIC_WORKSPACE_BYTES (16u << 20)

/* Optional pre-steps fused into the kernels (gdn_prefill_ex, gdn_decode_ex,
 * gdn_kda_prefill_ex, gdn_kda_decode_ex).
 *   size      : sizeof(gdn_options) (a smaller value is rejected)
 *   qk_l2norm : nonzero: q and k are L2-normalised per token and head before
 *               use, x^ = x / sqrt(sum_d x_d^2 + 1e-6), in fp32 from the bf16
 *               inputs.  The hybrid models normalise q and k before this layer;
 *               fusing it saves a pass over q and k (the inputs are read once).
 *   q_scale   : q is multiplied by this after the normalisation (1: unchanged;
 *               e.g. Dk^-1/2).
 *   o_bf16    : nonzero: o is written as bf16 (same layout; the fp32 value
 *               rounded to nearest even), halving its bytes.  A prefill with
 *               it runs the single-pass schedule (no workspace is used).
 * NULL options mean qk_l2norm = 0, q_scale = 1, o_bf16 = 0.  `size` is
 * sizeof(gdn_options) as the caller compiled it: 12 (a struct without o_bf16)
 * reads as o_bf16 = 0; anything below 12 is GDN_ERR_UNSUPPORTED. */
typedef struct gdn_options {
  int size;
  int qk_l2norm;
  float q_scale;
  int o_bf16;
} gdn_options;

/* Returns GDN_ABI_VERSION of the built library; callers compare it with the
 * header they compiled against and refuse to proceed on a mismatch. */
int gdn_abi_version(void);

/* Static, NUL-terminated description of a status code (never NULL). */
const char* gdn_status_str(int code);

/* Chunked prefill over T tokens (the chunked form of the recurrence above; the
 * ROCmFPX gated-delta-net prefill note, opening post, motivates chunking).
 *   q, k, v, g, beta : inputs as laid out above (device)
 *   S0   : initial state, or NULL for zeros (device)
 *   o    : output, written for every t < T (device)
 *   S_T  : final state, written (device; may equal S0)
 *   B, T, H : batch, tokens per sequence, heads; B*H == 0 or T == 0 are valid
 *             (T == 0 only writes S_T = S0, or zeros)
 *   Dk, Dv  : head dims, each 64, 128 or 256.  Dk = 64 or 128 runs the
 *             chunked tensor-core kernel (Dv = 256 on two CTAs per chain; the
 *             segmented schedule only at 128 x 128); Dk = 256 runs the
 *             row-parallel fp32 kernel (token by token, exact in the
 *             recurrence's order; chunk, workspace and schedule do not apply
 *             to it).  Other values: GDN_ERR_UNSUPPORTED
 *   chunk   : 16 or 64 -- tokens per chunk of the chunked form; the result is
 *             the same recurrence either way (up to rounding)
 *   status  : optional device int; a bounded device wait that gives up stores
 *             GDN_ERR_DEVICE_TIMEOUT there (it is never cleared by the library)
 *   stream  : cudaStream_t to launch on
 * Returns GDN_OK after enqueueing, or a negative gdn_status_code. */
int gdn_prefill(const void* q, const void* k, const void* v, const float* g, const float* beta,
                const float* S0, float* o, float* S_T, int B, int T, int H, int Dk, int Dv,
                int chunk, int* status, void* stream);

/* Workspace, in bytes, that gdn_prefill_ws needs for this problem on the
 * current device (the schedule depends on its multiprocessor count), or 0 when
 * it would run the single-pass schedule of gdn_prefill.  Invalid arguments
 * give 0 too; gdn_prefill_ws then reports them. */
size_t gdn_prefill_workspace_bytes(int B, int T, int H, int Dk, int Dv, int chunk);

/* Prefill of N sequences of different lengths packed along the token axis
 * (no padding between them): sequence n is tokens cu_seqlens[n] ..
 * cu_seqlens[n+1]-1 of the packed arrays.  The recurrence and its chunked form
 * are those of gdn_prefill, per sequence and head; the pages' prefill note
 * works on one sequence at a time, and packing is how a serving batch arrives.
 *   q, k [total_T][H][Dk] bf16; v [total_T][H][Dv] bf16; g, beta [total_T][H]
 *   fp32; o [total_T][H][Dv] fp32 (device)
 *   S0, S_T [N][H][Dv][Dk] fp32 (S0 may be NULL; S_T may equal S0) (device)
 *   cu_seqlens : device int[N+1], cu_seqlens[0] = 0, non-decreasing,
 *                cu_seqlens[N] = total_T.  A sequence whose offsets are out of
 *                order or past total_T is detected on the device: GDN_ERR_SHAPE
 *                goes to *status and that sequence's outputs are not written.
 *                Empty sequences are allowed (S_T = S0, or zeros).
 *   N, total_T, H : sequences, packed tokens, heads.  One pass per (sequence,
 *                head); the segmented schedule of gdn_prefill_ws is not used.
 *   snaps      : optional device fp32 output (NULL: none) of state snapshots,
 *                for prefix caching and for rolling back speculated tokens:
 *                the state after tokens j*snap_every of sequence n (j = 1 ..
 *                len_n / snap_every; the last one equals S_T when len_n is a
 *                multiple) goes to snaps[(k_n + j - 1) H + h][Dv][Dk], where k_n
 *                = sum over m < n of len_m / snap_every.
 *   snap_every : a positive multiple of 64 when snaps is given, else ignored
 *   n_snaps    : slots in snaps (sum over all n of len_n / snap_every); a
 *                sequence whose slots would pass it, or that follows a
 *                sequence with invalid offsets, gets none, and GDN_ERR_SHAPE
 *                goes to *status.
 * Dk must be 64 or 128 and Dv 64, 128 or 256: packed sequences run on the
 * chunked tensor-core kernel only (not on the Dk = 256 row kernel).  chunk,
 * status, stream and the other rules as for gdn_prefill. */
int gdn_prefill_varlen(const void* q, const void* k, const void* v, const float* g,
                       const float* beta, const float* S0, float* o, float* S_T,
                       const int* cu_seqlens, int N, int total_T, int H, int Dk, int Dv,
                       int chunk, float* snaps, int snap_every, int n_snaps, int* status,
                       void* stream);

/* gdn_prefill_varlen with options (gdn_options; NULL = none): qk_l2norm
 * and q_scale as in gdn_prefill_ex, applied to every token of every packed
 * sequence, and o_bf16 writes o as bf16 (the fp32 value rounded to nearest
 * even; o then needs total_T*H*Dv*2 bytes).  Everything else as for
 * gdn_prefill_varlen. */
int gdn_prefill_varlen_ex(const void* q, const void* k, const void* v, const float* g,
                          const float* beta, const float* S0, float* o, float* S_T,
                          const int* cu_seqlens, int N, int total_T, int H, int Dk, int Dv,
                          int chunk, float* snaps, int snap_every, int n_snaps,
                          const gdn_options* opts, int* status, void* stream);

/* gdn_prefill_ws with options (gdn_options above; NULL = none); with a NULL
 * workspace it runs the single pass of gdn_prefill.  Invalid options (size
 * too small, q_scale NaN) return GDN_ERR_UNSUPPORTED, and so do non-default
 * options with Dk = 256 (the row kernel; every head-dim pair with Dk = 64 or
 * 128 runs the chunked tensor-core kernel, which has them). */
int gdn_prefill_ex(const void* q, const void* k, const void* v, const float* g,
                   const float* beta, const float* S0, float* o, float* S_T, int B, int T, int H,
                   int Dk, int Dv, int chunk, void* workspace, size_t workspace_bytes,
                   const gdn_options* opts, int* status, void* stream);

/* The schedule gdn_prefill_ws picks for B*H chains of T tokens on a device
 * with num_sms multiprocessors (no device is touched): *nseg segments per chain
 * (1: the single pass of gdn_prefill) of *seg_tiles 64-token tiles each (the
 * last may be shorter), needing *ws_bytes of workspace.  Returns GDN_OK, or
 * GDN_ERR_SHAPE for negative sizes, GDN_ERR_NULL for a NULL output pointer. */
int gdn_prefill_schedule(int B, int T, int H, int num_sms, int* nseg, int* seg_tiles,
                         size_t* ws_bytes);

/* gdn_prefill with a caller-provided device workspace, which lets chains that
 * are too few to fill the GPU be cut into segments walked in parallel.  The
 * pages have no such schedule; it follows from the recurrence itself: over a
 * stretch of tokens the state is affine in the state the stretch starts from,
 *     S_t = S_start F_t + R_t,   o_t = S_start (F_t q_t) + o_t^R,
 * with F_t the ordered product of the factors alpha_s (I - beta_s k_s k_s^T)
 * and R_t, o_t^R the state and output from a zero start.  A first launch
 * walks every segment from zero (and, for each segment after the first, from
 * the identity with v = 0, which yields F and F q_t); a second launch chains
 * the segment-end states and adds S_start F_t q_t to o.  The result is the
 * same recurrence up to rounding.
 *   workspace       : device memory of at least gdn_prefill_workspace_bytes
 *                     (same sizes, same current device), 256-byte aligned,
 *                     overlapping no argument; may be NULL when that is 0.
 *                     Its contents on entry do not matter and are left
 *                     unspecified; two calls in flight must not share it.
 *   workspace_bytes : its size
 * Every other argument, and the results, as for gdn_prefill.  Returns GDN_OK,
 * GDN_ERR_WORKSPACE, or another negative code as for gdn_prefill. */
int gdn_prefill_ws(const void* q, const void* k, const void* v, const float* g,
                   const float* beta, const float* S0, float* o, float* S_T, int B, int T, int H,
                   int Dk, int Dv, int chunk, void* workspace, size_t workspace_bytes,
                   int* status, void* stream);

/* gdn_prefill_ws without any caller workspace and without any device
 * allocation: the scratch is a file-scope device array of the library of
 * GDN_STATIC_WORKSPACE_BYTES (16 MiB).  The pages have no counterpart; it
 * exists for callers that may not allocate.
 *   Problems whose schedule needs more scratch than that (see
 *   gdn_prefill_workspace_bytes; the single-pass schedule needs none) are
 *   rejected with GDN_ERR_STATIC_WORKSPACE_LIMIT before anything is launched.
 *   The scratch needs no zeroing: every byte read is written earlier in the
 *   same call.
 *   Every call looks up the array's device address on the current device
 *   (cudaGetSymbolAddress; cheap once the library's module is loaded there).
 *   The first call on a device may load that module, so make it before any
 *   stream capture.
 *   All calls on a device share the one array: calls whose executions
 *   overlap (other streams, other host threads) race on it and must be
 *   serialised by the caller.
 * Arguments, results and other errors as for gdn_prefill. */
int gdn_prefill_static_ws(const void* q, const void* k, const void* v, const float* g,
                          const float* beta, const float* S0, float* o, float* S_T, int B,
                          int T, int H, int Dk, int Dv, int chunk, int* status, void* stream);

/* One decode step for B sequences (the recurrence above with T = 1), the state
 * read and written in place (the Megakernel decode of the Lucebox contribution
 * guide, section 4, is where this step runs once per layer and token).
 *   q, k [B][H][Dk] bf16; v [B][H][Dv] bf16; g, beta [B][H] fp32 (device)
 *   S    [B][H][Dv][Dk] fp32, updated in place (device)
 *   o    [B][H][Dv] fp32, written (device)
 *   Dk, Dv each 64, 128 or 256 (128 x 128 and 64 x 64: the streaming decode
 *   kernel; other pairs: the row-parallel kernel); B*H == 0 is a no-op.
 * status and stream as for gdn_prefill.  Returns GDN_OK or a negative code. */
int gdn_decode_step(const void* q, const void* k, const void* v, const float* g,
                    const float* beta, float* S, float* o, int B, int H, int Dk, int Dv,
                    int* status, void* stream);

/* T decode tokens per sequence in one call (T = 1 is gdn_decode_step): the
 * recurrence above applied to tokens 1..T in order, starting from S and
 * leaving S_T in S.  The state is read once and written once, so a short burst
 * costs one state round trip instead of T: e.g. the block of drafted tokens
 * that speculative decoding verifies at once (the DFlash contribution guide,
 * discosf.com/news/4742660, opening section: block drafts for speculative
 * decoding).  For long T, gdn_prefill is faster.
 *   q, k [B][T][H][Dk] bf16; v [B][T][H][Dv] bf16; g, beta [B][T][H] fp32 (device)
 *   S    [B][H][Dv][Dk] fp32, updated in place (device)
 *   o    [B][T][H][Dv] fp32, written (device)
 *   Dk, Dv each 64, 128 or 256 (128 x 128 and 64 x 64: the streaming decode
 *   kernels; other pairs: the row-parallel kernel); B*H == 0 or T == 0 is a
 *   no-op.
 * status and stream as for gdn_prefill.  Returns GDN_OK or a negative code. */
int gdn_decode_tokens(const void* q, const void* k, const void* v, const float* g,
                      const float* beta, float* S, float* o, int B, int T, int H, int Dk, int Dv,
                      int* status, void* stream);

/* gdn_decode_tokens with options (gdn_options; NULL = none).  Non-default
 * options need Dk = Dv = 128 or Dk = Dv = 64, the dims the streaming decode
 * kernels serve (else GDN_ERR_UNSUPPORTED). */
int gdn_decode_ex(const void* q, const void* k, const void* v, const float* g,
                  const float* beta, float* S, float* o, int B, int T, int H, int Dk, int Dv,
                  const gdn_options* opts, int* status, void* stream);

/* Delta rule with a per-channel gate (KDA): alpha_t = exp(g_t) is a vector
 * over the key channels, applied where the scalar gate is (the variant that the
 * ROCmFPX gated-delta-net prefill note, bittide.aicompass.dev article
 * d2880479, lists among the cases its fused kernel left to the old path):
 *     S_t = S_{t-1} diag(alpha_t) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T
 *     o_t = S_t q_t
 * for t = 1..T of each of the B*H chains.  With Dk = 128 (Dv 64, 128 or 256)
 * it runs chunked on the tensor cores (32-token chunks; every derived operand
 * as a bf16 hi/lo pair; exact up to rounding while a key channel's decay over
 * 16 tokens stays above e^-87, the fp32 range; Dv = 256 on two CTAs per
 * chain); Dk = 64 or 256 run token by token in fp32.
 *   q, k [B][T][H][Dk] bf16; v [B][T][H][Dv] bf16 (device, 16-byte aligned)
 *   g    [B][T][H][Dk] fp32, natural-log decays (device, 16-byte aligned;
 *        g > 0 is accepted and grows the state)
 *   beta [B][T][H] fp32 (device)
 *   S0   [B][H][Dv][Dk] fp32 or NULL (zeros); S_T written, same layout; S_T
 *        may be S0 (in place) but may not partly overlap it (16-byte aligned)
 *   o    [B][T][H][Dv] fp32, written (device); may not overlap any other array
 *   Dk, Dv each 64, 128 or 256.  B*H == 0 is a no-op; T == 0 copies S0 (or
 *   zeros) to S_T.
 * status: optional device int; the tensor-core path's bounded waits store
 * GDN_ERR_DEVICE_TIMEOUT there if one gives up (the row kernel never writes it).
 * stream is a cudaStream_t.  Returns GDN_OK or a negative code; nothing is
 * launched on an error. */
int gdn_kda_prefill(const void* q, const void* k, const void* v, const float* g,
                    const float* beta, const float* S0, float* o, float* S_T, int B, int T,
                    int H, int Dk, int Dv, int* status, void* stream);

/* The per-channel-gate recurrence with the state updated in place: T tokens
 * per sequence starting from S and leaving S_T in S (T = 1: one decode step).
 * At 128 x 128 and 64 x 64 it runs the streaming decode kernel (the decay
 * applied per key column of each state row in registers); other head dims run
 * the row kernel.  Either reads and writes the state once per call.  Arguments
 * as for gdn_kda_prefill with S0 = S_T = S, except that o needs only 4-byte
 * alignment; status is never written. */
int gdn_kda_decode(const void* q, const void* k, const void* v, const float* g,
                   const float* beta, float* S, float* o, int B, int T, int H, int Dk, int Dv,
                   int* status, void* stream);

/* gdn_kda_prefill / gdn_kda_decode with options (gdn_options; NULL = none).
 * qk_l2norm and q_scale are applied to each token's q and k before any decay,
 * as in gdn_prefill_ex, and o_bf16 writes o as bf16 (the fp32 value rounded
 * to nearest even; o then needs B*T*H*Dv*2 bytes); they need Dk = 128 in the
 * prefill (any Dv), and 128 x 128 or 64 x 64 in decode (else
 * GDN_ERR_UNSUPPORTED, as for an invalid struct).  Everything else as for the
 * calls without options. */
int gdn_kda_prefill_ex(const void* q, const void* k, const void* v, const float* g,
                       const float* beta, const float* S0, float* o, float* S_T, int B, int T,
                       int H, int Dk, int Dv, const gdn_options* opts, int* status, void* stream);
int gdn_kda_decode_ex(const void* q, const void* k, const void* v, const float* g,
                      const float* beta, float* S, float* o, int B, int T, int H, int Dk, int Dv,
                      const gdn_options* opts, int* status, void* stream);

/* gdn_kda_prefill for N sequences of different lengths packed along the token
 * axis, as in gdn_prefill_varlen: sequence n is tokens cu_seqlens[n] ..
 * cu_seqlens[n+1]-1 of the packed arrays, each (sequence, head) one chain of
 * the per-channel-gate recurrence.
 *   q, k, g [total_T][H][128]; v, o [total_T][H][Dv]; beta [total_T][H]
 *   (types and alignment as for gdn_kda_prefill; o fp32)
 *   S0, S_T [N][H][Dv][128] fp32 (S0 may be NULL; S_T may equal S0)
 *   cu_seqlens : device int[N+1], 0 = cu_seqlens[0] <= ... <= cu_seqlens[N] =
 *                total_T.  Offsets out of order or past total_T are detected
 *                on the device: GDN_ERR_SHAPE goes to *status and that
 *                sequence's outputs are not written.  Empty sequences are
 *                allowed (S_T = S0, or zeros).
 *   snaps, snap_every, n_snaps : optional state snapshots, laid out and
 *                bounded as in gdn_prefill_varlen ([Dv][128] per slot), except
 *                that snap_every is a positive multiple of 32 (the kernel's
 *                chunk); NULL snaps: none.
 * Dk must be 128 and Dv 64, 128 or 256 (the chunked tensor-core kernel, one
 * CTA per chain, two with Dv = 256); options through the _ex call below.
 * N*H == 0 is a no-op.
 * status: optional device int; GDN_ERR_SHAPE (offsets, snapshot slots) or
 * GDN_ERR_DEVICE_TIMEOUT (a bounded wait gave up) is stored there.  Returns
 * GDN_OK, or a negative code for invalid arguments (nothing is launched). */
int gdn_kda_prefill_varlen(const void* q, const void* k, const void* v, const float* g,
                           const float* beta, const float* S0, float* o, float* S_T,
                           const int* cu_seqlens, int N, int total_T, int H, int Dk, int Dv,
                           float* snaps, int snap_every, int n_snaps, int* status, void* stream);

/* gdn_kda_prefill_varlen with options: qk_l2norm, q_scale and o_bf16 as in
 * gdn_kda_prefill_ex.  Everything else as for gdn_kda_prefill_varlen. */
int gdn_kda_prefill_varlen_ex(const void* q, const void* k, const void* v, const float* g,
                              const float* beta, const float* S0, float* o, float* S_T,
                              const int* cu_seqlens, int N, int total_T, int H, int Dk, int Dv,
                              float* snaps, int snap_every, int n_snaps,
                              const gdn_options* opts, int* status, void* stream);

/* Synchronises `stream`, then reads the device status word written by the
 * kernels.  Returns the word (GDN_OK, GDN_ERR_DEVICE_TIMEOUT, or GDN_ERR_SHAPE
 * from the packed-sequence calls), GDN_ERR_NULL (status_dev is NULL) or
 * GDN_ERR_LAUNCH (the synchronisation or copy failed). */
int gdn_query_status(const int* status_dev, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* GDN_B200_H_ */
