// Chunked gated-delta-rule prefill for sm_100a: TMA-staged bf16 tiles,
// tcgen05 MMAs accumulating in tensor memory, fp32 state carried across
// chunks in tensor memory, warp-specialised so that the work of consecutive
// tiles overlaps.
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
// One CTA of 512 threads owns one (b, h) chain (with Dv = 256, two CTAs own
// 128 rows of its state each) and walks its tokens in tiles of 64 (one TMA
// tile); with chunk = 16 each tile holds four chunks.  The key dimension Dk is
// 64 or 128 (a template parameter: the K-dimension of the S products, the
// state's TMEM columns and the K/Q boxes); the rows of the state a CTA owns are
// the MMAs' M = 128 lanes (Dv = 64 keeps lanes 64..127 at zero).  The
// warps split into three roles that run concurrently and hand off through
// mbarriers:
//   * chain  (warps 0-3 and 12-15, 256 threads): everything that depends on
//     the state -- S_c [K;Q]^T, X, Dl = X T^T, the output and state-update
//     products and their epilogues -- for tile c;
//   * side (warps 4-11, 256 threads): the state-independent work of tile c+1
//     -- gates, [K;Q] K^T, the masks and decays, the triangular solve --
//     handing T and Mq to the chain once the chain has finished with tile
//     c's, and draining o of tile c from tensor memory to HBM as soon as the
//     chain has produced it.
// Warp w reads TMEM lane quarter (w % 4); the two warpgroups of each role
// split the columns of each tile in halves.  The fp32 state lives in tensor memory,
// pre-multiplied by the decay of the chunk about to update it, so the
// state-update MMA accumulates straight into it; the tensor core reads the
// state as a bf16 hi/lo pair, also in tensor memory.  Every operand derived
// inside the kernel (S, X, T, the residuals, Mq) is fed to the MMA as hi + lo
// bf16 parts (hi = bf16(x), lo = bf16(x - hi)) so the products keep ~16 bits
// of mantissa; q, k and v are exact bf16 inputs.
//
// Tensor memory (512 columns, fp32 unless noted; with Dk = 64 the state uses
// the first half of its ranges):
//   [  0,128) S   : state, scaled by the next chunk's total decay  (lane dv, col dk)
//   [128,192) SHI : S hi as bf16 pairs (A operand)                 (lane dv, col dk/2)
//   [192,256) SLO : S lo
//   [256,320) Z   : S K^T, then X^T as a bf16 hi/lo pair (the A operand of the
//                   residual product), then Dl~^T as a hi/lo pair (the A
//                   operand of the state update)              (lane dv, col token)
//   [320,384) Y   : S Q^T                                          (lane dv, col token)
//   [384,448) P   : [K;Q] K^T (lanes = rows of [K;Q]; K side only)
//   [448,512) OI  : Dl^T, then Dl^T Mq^T                           (lane dv, col token)
// Reading the residual product's and the state update's A operands from tensor
// memory halves their MMA issue cost against shared-memory operands.
#include "gdn_internal.h"
#include "sm100.cuh"

namespace gdn {
namespace {

using namespace sm100;

constexpr int D = 128;
constexpr int NT = 64;  // tokens per TMA tile
constexpr int NTHREADS = 512;
constexpr int CHAIN_THREADS = 256, SIDE_THREADS = 256;
constexpr int BAR_CHAIN = 1, BAR_SIDE = 2, BAR_SCAN = 3;  // named barriers
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TM_S = 0, TM_SHI = 128, TM_SLO = 192, TM_Z = 256, TM_Y = 320, TM_P = 384,
                   TM_OI = 448;

// Shared memory map (offsets from a 1024-byte aligned base).
constexpr uint32_t SM_KQ0 = 0;        // 32 KB: [K dk0-63 | Q dk0-63 | K dk64-127 | Q dk64-127]
constexpr uint32_t SM_KQ1 = 32768;    //        each a 64-row x 128-byte SW128 box
constexpr uint32_t SM_V = 65536;      // 16 KB: V tile [64 tokens][128] bf16, unswizzled
constexpr uint32_t SM_MQH = 81920;    // 8 KB: Mq rows i, K-major SW128 (64 x 64 bf16)
constexpr uint32_t SM_MQL = 90112;
constexpr uint32_t SM_TH = 98304;     // 8 KB: T rows i (64 x 64)
constexpr uint32_t SM_TL = 106496;
constexpr uint32_t SM_XH = 114688;    // 32 KB staging: the fp32 o tile [64 tokens][128]
constexpr uint32_t SM_XL = 131072;    //   (and, with the Dl^T tiles after them, the 64 KB end state)
constexpr uint32_t SM_DH = 147456;    // 16 KB: Dl^T rows dv (128 x 64)
constexpr uint32_t SM_DL = 163840;
constexpr int APAD = 68;                      // row pitch (floats): conflict-free float4 rows
constexpr uint32_t SOLVE_MAT = 64 * APAD * 4; // 17408 B
constexpr uint32_t SM_A = 180224;             // A  fp32 [64][APAD] (K side)
constexpr uint32_t SM_TF = SM_A + SOLVE_MAT;  // T  fp32 [64][APAD] (K side)
// T_II A_IK blocks fp32 [6][16][AT_PITCH] (K side); the 20-float row pitch puts the
// eight rows a warp reads at once in eight distinct banks
constexpr int AT_PITCH = 20, AT_BLOCK = 16 * AT_PITCH;
constexpr uint32_t SM_AT = SM_TF + SOLVE_MAT;
constexpr uint32_t SM_GATES = SM_AT + 6 * AT_BLOCK * 4;  // gate buffers (tile c uses c % GATE_BUFS)
constexpr uint32_t GATE_BYTES = 1808;
// The side role writes tile c's gates after the chain released tile c-3
// (tm_free); the chain's last reader of tile c-4's buffer (the o drain) runs
// before it starts tile c-3's MMAs, so four buffers never overlap a reader.
constexpr int GATE_BUFS = 4;
// per-token arrays of a gate buffer (64 floats each; G_GC: one float per chunk):
//   gamma (log2), beta, beta Gamma |k|^-1, exp(gamma_last - gamma) |k|^-1,
//   Gamma q_scale |q|^-1, |k|^-1, q_scale |q|^-1, Gamma_last per chunk
// (the |.|^-1 factors are 1 without in-kernel normalisation)
constexpr uint32_t G_GAM2 = 0, G_B = 256, G_BG = 512, G_DF = 768, G_GAM = 1024, G_KN = 1280,
                   G_QN = 1536, G_GC = 1792;
static_assert(GATE_BYTES % 16 == 0 && G_GC + 16 <= GATE_BYTES, "gate buffer layout");
constexpr uint32_t SM_BAR = SM_GATES + GATE_BUFS * GATE_BYTES;
constexpr uint32_t SM_MISC = SM_BAR + 256;    // TMEM slot, abort flags, scan scratch, counters
constexpr uint32_t SMEM_USED = SM_MISC + 256;
static_assert(SM_A >= SM_DL + 16384, "K-side scratch overlaps the residual tiles");
static_assert(SM_DL + 16384 - SM_XH == 65536, "o staging and Dl^T tiles form the 64 KB end-state staging area");
static_assert(SMEM_USED + 1024 <= 232448, "shared memory budget");

// mbarriers (8 bytes each, offsets inside SM_BAR)
// The gates of tile c are signalled on B_GFULL + 8 (c % 4): the side role can
// finish the gates of tile c + 2 before the chain has waited for tile c's, so
// two barriers with parity waits could alias; four cannot (tile c + 4 needs
// the chain to have finished tile c + 2).
constexpr uint32_t B_FULL0 = 0, B_FULL1 = 8, B_VFULL = 16, B_PFULL = 24, B_TMFULL = 32,
                   B_TMFREE = 40, B_ZQ = 48, B_DL = 56, B_SU = 64, B_GFULL = 72, B_OI = 104,
                   B_CLEAN0 = 112, B_CLEAN1 = 120, B_CLEAN2 = 128, B_CLEAN3 = 136;
constexpr int NUM_BARS = 18;
// MMA issuers: tcgen05.mma costs ~40-100 ns to issue from one thread, and
// issuers in different warps proceed in parallel, so independent products are
// issued by different threads: the chain leader (thread 0: [Z|Y], Dl, the
// state update), a second chain thread (the output product) and, on the side,
// a thread outside the solve's first phase ([K;Q] K^T).
constexpr int OI_ISSUER = 384;   // warp 12, lane 0
constexpr int P_ISSUER = 192;    // warp 6, lane 0 (side thread kt = 64)
__device__ __forceinline__ uint32_t gfull_off(int c) { return B_GFULL + 8u * uint32_t(c & 3); }
__device__ __forceinline__ uint32_t gfull_parity(int c) { return uint32_t(c >> 2) & 1u; }
// misc slots (offsets inside SM_MISC)
constexpr uint32_t M_TMEM = 0, M_ABORT = 4, M_PART = 8, M_KQ_ISSUED = 12, M_KQ_SEEN = 16,
                   M_V_ISSUED = 20, M_V_SEEN = 24, M_FLAG_CHAIN = 32,
                   M_FLAG_SIDE = 40,  // two verdict slots per role
                   M_SNAP_TILES = 48,  // tiles between state snapshots (0: none)
                   M_SNAP_PTR = 56,    // this chain's first snapshot slot (8 bytes)
                   M_OROW = 64;        // o's row width (Dv), set at start
static_assert(M_SNAP_PTR + 8 <= 64, "misc slots (the first 64 bytes are cleared at start)");
static_assert(8 * NUM_BARS <= 256, "barrier slots");

// K and Q of a tile: Dk / 64 boxes each of 64 tokens x 128 bytes
template <int DK>
constexpr uint32_t kq_tx_bytes() { return uint32_t(DK / 64) * 2u * 8192u; }
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;  // 2 s: far beyond any legitimate wait
constexpr float LOG2E = 1.4426950408889634f;

// Splits 32 consecutive state values (columns 32q..32q+31 of this lane's row)
// into bf16 hi/lo pairs and stores them to SHI / SLO.
__device__ __forceinline__ void store_state_split32(uint32_t tlane, int q, const float (&v)[32]) {
  uint32_t hi[16], lo[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) split2_bf16(v[2 * e], v[2 * e + 1], hi[e], lo[e]);
  tmem_st16x2(tlane + TM_SHI + 16 * q, hi, tlane + TM_SLO + 16 * q, lo);
}
__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }

// N consecutive values of this thread's TMEM lane (a chunk's tokens) as bf16
// hi/lo pairs: N/2 columns of hi at t_hi, N/2 of lo at t_lo (the layout an MMA
// A operand read from tensor memory takes: lane = row, K packed 2 per column).
template <int N>
__device__ __forceinline__ void store_pairs_split(uint32_t t_hi, uint32_t t_lo, const float (&v)[N]) {
  static_assert(N == 32 || N == 8, "a chunk half of 64 or 16 tokens");
  if constexpr (N == 32) {
    uint32_t hi[16], lo[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) split2_bf16(v[2 * e], v[2 * e + 1], hi[e], lo[e]);
    tmem_st16x2(t_hi, hi, t_lo, lo);
  } else {
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) split2_bf16(v[2 * e], v[2 * e + 1], hi[e], lo[e]);
    tmem_st4x2(t_hi, hi, t_lo, lo);
  }
}

// Shared state of one CTA.
struct Ctx {
  uint8_t* sm;
  uint32_t sb;        // shared-window address of sm
  uint32_t tmem;      // TMEM base (lane 0, column 0)
  int* status;
  int H;
  volatile int* abort_flag;
  int tok0;            // token coordinate (in the TMA views) of this CTA's first tile
  int tend;            // first token coordinate past this CTA's sequence: padding from there on
  int tmap;            // token extent of the TMA views (T, or the packed total)
  bool vzero;          // v taken as zero (transfer-matrix CTA of the segmented schedule)
  bool s0_identity;    // start from the identity instead of s0src / zeros
  const float* s0src;  // start state of this chain [128][128], or null
  float* odst;         // destination of o-like outputs, laid out like o
  const CUtensorMap* tmo;  // TMA view of odst: [B][T][H][128] fp32, box 64 tokens x 128
  float* sdst;         // destination of the end state rows owned by this CTA
  int dv0;             // first state row (value channel) owned by this CTA
  __device__ __forceinline__ uint32_t bar(uint32_t off) const { return sb + SM_BAR + off; }
  __device__ __forceinline__ float* gates(int c) const {
    return reinterpret_cast<float*>(sm + SM_GATES + (c % GATE_BUFS) * GATE_BYTES);
  }
  __device__ __forceinline__ volatile int* misc(uint32_t off) const {
    return reinterpret_cast<volatile int*>(sm + SM_MISC + off);
  }
  __device__ __forceinline__ void fail() const {
    *abort_flag = 1;
    if (status) atomicExch(status, GDN_ERR_DEVICE_TIMEOUT);
  }
};

// Role-wide agreement on whether to go on.  The role leader decides (after a
// bounded wait on an mbarrier phase, in wait()), writes the verdict to one of
// two slots, and the role meets at its named barrier; every thread then reads
// the same verdict, so the whole role takes the same path.  The slots
// alternate: a slot is rewritten only two agreements later, after every
// thread has passed the barrier of the agreement in between.
struct RoleSync {
  int bar_id, nthreads;
  uint32_t flag_off;
  bool leader;
  int n;  // agreements so far (identical in every thread of the role)
  __device__ __forceinline__ bool agree(const Ctx& x, bool leader_ok) {
    volatile int* slot = x.misc(flag_off + 4u * (n & 1));
    ++n;
    if (leader) *slot = leader_ok ? 0 : 1;
    named_bar(bar_id, nthreads);
    const bool ok = (*slot == 0);
    tc_fence_after();
    return ok;
  }
  // Leader waits (bounded) for the given phase parity of `bar`.
  __device__ __forceinline__ bool wait(const Ctx& x, uint32_t bar, uint32_t parity) {
    bool ok = true;
    if (leader) {
      ok = (*x.abort_flag == 0) && mbar_wait_bounded(bar, parity, WAIT_LIMIT_NS);
      if (!ok) x.fail();
    }
    return agree(x, ok);
  }
  __device__ __forceinline__ bool check(const Ctx& x) {
    return agree(x, !leader || *x.abort_flag == 0);
  }
};

template <int DK>
__device__ __forceinline__ void issue_kq(const Ctx& x, const CUtensorMap* tq, const CUtensorMap* tk,
                                         int c, int h, int b) {
  const uint32_t kq = x.sb + ((c & 1) ? SM_KQ1 : SM_KQ0);
  const uint32_t bar = x.bar((c & 1) ? B_FULL1 : B_FULL0);
  mbar_arrive_expect_tx(bar, kq_tx_bytes<DK>());
  const int t0 = x.tok0 + c * NT;
  tma_load_4d(kq + 0, tk, bar, 0, h, t0, b);
  tma_load_4d(kq + 8192, tq, bar, 0, h, t0, b);
  if constexpr (DK == 128) {
    tma_load_4d(kq + 16384, tk, bar, 64, h, t0, b);
    tma_load_4d(kq + 24576, tq, bar, 64, h, t0, b);
  }
  *x.misc(M_KQ_ISSUED) = c + 1;
}
// V rows dv0 .. dv0 + DVB - 1 of the tile's 64 tokens ([64][DVB] bf16)
template <int DVB>
__device__ __forceinline__ void issue_v(const Ctx& x, const CUtensorMap* tv, int c, int h, int b) {
  const uint32_t bar = x.bar(B_VFULL);
  mbar_arrive_expect_tx(bar, uint32_t(NT * DVB * 2));
  tma_load_4d(x.sb + SM_V, tv, bar, x.dv0, h, x.tok0 + c * NT, b);
  *x.misc(M_V_ISSUED) = c + 1;
}

// Off-diagonal blocks of T = (I + A)^{-1}, 64 x 64 in 16 x 16 blocks, once the
// diagonal blocks T_II are in Tf.  With At_IK = T_II A_IK (K < I), block row I
// of (I + A) T = I gives
//   T_IJ = -sum_{K=J}^{I-1} At_IK T_KJ            (I > J),
// computed by distance d = I - J = 1, 2, 3 after one pass that forms all six
// At blocks.  A thread owns 1 x 4 strips of outputs; each dot product is split
// over two accumulators; all loop bounds are compile-time.  The strip and block
// loops stay rolled (only the 16-term dot products are unrolled): the per-tile
// code path is long enough for instruction fetch to show, and on B200 this form
// ran the 128-chain prefill ~4% faster than the fully unrolled one.
__device__ __forceinline__ int at_index(int I, int K) { return (I * (I - 1)) / 2 + K; }  // 0..5

__device__ __forceinline__ void solve_at_blocks(int kt, const float* sA, const float* sTf, float* sAt) {
  // 6 blocks x 16 rows x 4 strips = 384 strips
#pragma unroll 1
  for (int st = kt; st < 384; st += SIDE_THREADS) {
    const int blk = st >> 6, r = (st >> 2) & 15, c4 = st & 3;
    const int I = blk < 1 ? 1 : (blk < 3 ? 2 : 3);
    const int K = blk - at_index(I, 0);
    const float* trow = sTf + (I * 16 + r) * APAD + I * 16;        // T_II row r
    const float* acol = sA + (I * 16) * APAD + K * 16 + 4 * c4;     // A_IK rows m, cols 4c4..
    float4 a0 = make_float4(0.f, 0.f, 0.f, 0.f), a1 = a0;
#pragma unroll
    for (int m = 0; m < 16; m += 2) {
      const float t0 = trow[m], t1 = trow[m + 1];
      const float4 x0 = ld4(acol + m * APAD), x1 = ld4(acol + (m + 1) * APAD);
      a0.x = fmaf(t0, x0.x, a0.x); a0.y = fmaf(t0, x0.y, a0.y);
      a0.z = fmaf(t0, x0.z, a0.z); a0.w = fmaf(t0, x0.w, a0.w);
      a1.x = fmaf(t1, x1.x, a1.x); a1.y = fmaf(t1, x1.y, a1.y);
      a1.z = fmaf(t1, x1.z, a1.z); a1.w = fmaf(t1, x1.w, a1.w);
    }
    *reinterpret_cast<float4*>(sAt + blk * AT_BLOCK + r * AT_PITCH + 4 * c4) =
        make_float4(a0.x + a1.x, a0.y + a1.y, a0.z + a1.z, a0.w + a1.w);
  }
}

template <int d>
__device__ __forceinline__ void solve_distance(int kt, const float* sAt, float* sTf) {
  constexpr int NSTRIP = (4 - d) * 64;
#pragma unroll 1
  for (int st = kt; st < NSTRIP; st += SIDE_THREADS) {
    const int J = st >> 6, r = (st >> 2) & 15, c4 = st & 3;
    const int I = J + d;
    float4 a0 = make_float4(0.f, 0.f, 0.f, 0.f), a1 = a0;
#pragma unroll 1
    for (int K = J; K < I; ++K) {
      const float* atrow = sAt + at_index(I, K) * AT_BLOCK + r * AT_PITCH;  // At_IK row r
      const float* tcol = sTf + (K * 16) * APAD + J * 16 + 4 * c4;    // T_KJ rows, cols 4c4..
#pragma unroll
      for (int m = 0; m < 16; m += 2) {
        const float t0 = atrow[m], t1 = atrow[m + 1];
        const float4 x0 = ld4(tcol + m * APAD), x1 = ld4(tcol + (m + 1) * APAD);
        a0.x = fmaf(t0, x0.x, a0.x); a0.y = fmaf(t0, x0.y, a0.y);
        a0.z = fmaf(t0, x0.z, a0.z); a0.w = fmaf(t0, x0.w, a0.w);
        a1.x = fmaf(t1, x1.x, a1.x); a1.y = fmaf(t1, x1.y, a1.y);
        a1.z = fmaf(t1, x1.z, a1.z); a1.w = fmaf(t1, x1.w, a1.w);
      }
    }
    *reinterpret_cast<float4*>(sTf + (I * 16 + r) * APAD + J * 16 + 4 * c4) =
        make_float4(-(a0.x + a1.x), -(a0.y + a1.y), -(a0.z + a1.z), -(a0.w + a1.w));
  }
}

// ============================================================== K side
// Per tile c: [K;Q] K^T -> masks / decays -> T = (I + A)^{-1}; the next
// tile's [K;Q] K^T is issued as soon as this tile's P has been read, and the
// next tile's gates are formed before waiting for the chain; then, once the
// chain has released tile c-1's T and Mq, writes T(c), Mq(c).
// |k_j|^-1 and q_scale |q_i|^-1 of tile c into its gate buffer (all side
// threads; with normalisation off, just 1 and q_scale).  Thread t sums the
// squares of half a row of [K; Q] (Dk = 128: the 64 bf16 of one 128-byte SW128
// row; Dk = 64: half of the row's one 128-byte line; the chunk order of the
// swizzle does not matter for a sum) and the two halves meet by a shuffle.
// x^ = x / sqrt(sum x^2 + 1e-6).
template <int DK>
__device__ __forceinline__ void side_norms(const Ctx& x, int kt, int c, const PrefillArgs& p) {
  float* G = x.gates(c);
  if (!p.qk_norm) {
    if (kt < NT) {
      G[G_KN / 4 + kt] = 1.f;
      G[G_QN / 4 + kt] = p.q_scale;
    }
    return;
  }
  const int r = kt >> 1, hf = kt & 1;  // row of [K; Q] (0..63 K, 64..127 Q), dk half
  const int rr = r & (NT - 1);
  // Dk = 128: half hf is the box of dk 64 hf ..; Dk = 64: the 16-byte chunks
  // 4 hf .. 4 hf + 3 of the row's line
  const uint32_t row = x.sb + ((c & 1) ? SM_KQ1 : SM_KQ0) + (r < NT ? 0u : 8192u) +
                       (DK == 128 ? (hf ? 16384u : 0u) : 64u * uint32_t(hf)) +
                       uint32_t(rr >> 3) * 1024u + uint32_t(rr & 7) * 128u;
  float ss = 0.f;
#pragma unroll
  for (int ch = 0; ch < DK / 16; ++ch) {
    uint32_t w[4];
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3])
                 : "r"(row + 16u * ch));
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[e]));
      ss = fmaf(f.x, f.x, fmaf(f.y, f.y, ss));
    }
  }
  ss += __shfl_xor_sync(0xffffffffu, ss, 1);
  if (hf == 0) {
    const float inv = rsqrtf(ss + 1e-6f);
    if (r < NT)
      G[G_KN / 4 + rr] = inv;
    else
      G[G_QN / 4 + rr] = inv * p.q_scale;
  }
}

// CLOSE: end with a role-wide barrier and signal the gates' barrier; without
// it the caller does both (in its next agreement).
template <int C, bool PRE, bool CLOSE = true>
__device__ __forceinline__ void side_gates(const Ctx& x, int kt, int c, int T, float& g_next,
                                           float& b_next, const PrefillArgs& p, int b, int h,
                                           volatile float* s_part) {
  // inclusive in-chunk scan of g over tile c (threads kt < 64), decays
  float* G = x.gates(c);
  const int H = p.H;
  if (kt < NT) {
    float gc = g_next;
    const float bc = b_next;
    g_next = 0.f;
    b_next = 0.f;
    const int t = x.tok0 + (c + 1) * NT + kt;
    if (t < x.tend) {  // tokens past the sequence are padding: g = beta = 0, an exact identity
      const size_t gi = (size_t(b) * T + t) * H + h;
      g_next = __ldg(p.g + gi);
      b_next = __ldg(p.beta + gi);
    }
    constexpr int W = C < 32 ? C : 32;
    const int ln = kt & 31;
#pragma unroll
    for (int off = 1; off < W; off <<= 1) {
      const float y = __shfl_up_sync(0xffffffffu, gc, off, W);
      if ((ln & (W - 1)) >= off) gc += y;
    }
    if constexpr (C == 64) {
      if (kt == 31) *s_part = gc;
      named_bar(BAR_SCAN, 64);
      if (kt >= 32) gc += *s_part;
    }
    G[G_GAM2 / 4 + kt] = gc * LOG2E;
    G[G_B / 4 + kt] = bc;
  }
  named_bar(BAR_SIDE, SIDE_THREADS);
  if (kt < NT) {
    const int last = (kt / C) * C + C - 1;
    const float gi = G[G_GAM2 / 4 + kt], gl = G[G_GAM2 / 4 + last];
    const float Gm = fast_exp2(gi);
    if constexpr (PRE) {  // fold |k|^-1 and q_scale |q|^-1
      const float kn = G[G_KN / 4 + kt];
      G[G_GAM / 4 + kt] = Gm * G[G_QN / 4 + kt];
      G[G_BG / 4 + kt] = G[G_B / 4 + kt] * Gm * kn;
      G[G_DF / 4 + kt] = fast_exp2(gl - gi) * kn;
    } else {
      G[G_GAM / 4 + kt] = Gm;
      G[G_BG / 4 + kt] = G[G_B / 4 + kt] * Gm;
      G[G_DF / 4 + kt] = fast_exp2(gl - gi);
    }
    if (kt == last) G[G_GC / 4 + kt / C] = fast_exp2(gl);
  }
  if constexpr (CLOSE) {
    named_bar(BAR_SIDE, SIDE_THREADS);
    if (kt == 0) mbar_arrive(x.bar(gfull_off(c)));
  }
}

template <int DK>
__device__ __forceinline__ void issue_p(const Ctx& x, int c) {
  const uint64_t d0 = sdesc_sw128(x.sb + ((c & 1) ? SM_KQ1 : SM_KQ0), 16, 1024);
  const uint32_t id = idesc_bf16(128, 64, 0, 0, 0);
#pragma unroll
  for (int kk = 0; kk < DK / 16; ++kk) {
    const uint64_t d = sdesc_add(d0, (kk >> 2) * 16384 + (kk & 3) * 32);
    mma_ss(x.tmem + TM_P, d, d, id, kk > 0);
  }
  mma_commit(x.bar(B_PFULL));
}

// Copies rows 0 .. nvalid-1 of the staged fp32 o tile (rows of DVB floats) to
// dst (row r at dst + r rowstride), thread ct of the chain role taking every
// CHAIN_THREADS-th 16-byte chunk.  Kept out of line: it runs only for the last
// tile of a packed sequence.
template <int DVB>
__device__ __noinline__ void store_partial_tile(const float4* src, float* dst, size_t rowstride,
                                                int nvalid, int ct) {
  for (int i = ct; i < nvalid * (DVB / 4); i += CHAIN_THREADS) {
    const int r = i / (DVB / 4), j = i % (DVB / 4);
    reinterpret_cast<float4*>(dst + size_t(r) * rowstride)[j] = src[i];
  }
}

// The same for a bf16 staging tile (rows of DVB bf16, DVB / 8 chunks of 16 bytes).
template <int DVB>
__device__ __noinline__ void store_partial_tile_bf16(const uint4* src, __nv_bfloat16* dst,
                                                     size_t rowstride, int nvalid, int ct) {
  for (int i = ct; i < nvalid * (DVB / 8); i += CHAIN_THREADS) {
    const int r = i / (DVB / 8), j = i % (DVB / 8);
    reinterpret_cast<uint4*>(dst + size_t(r) * rowstride)[j] = src[i];
  }
}

// o[t][dv] = Gamma_t Y[dv][t] + O_intra[dv][t] of tile c.  This thread's 32
// tokens (32 hf ..) of lane dv go into the fp32 [64 tokens][128] o staging
// tile; the leader then stores the tile with TMA (tokens at or past T are
// dropped by the copy).  Before the next tile's staging is written the leader
// waits for the copy to have read it (at the next tile's first agreement).
// OBF: o is bf16 (tile rows of 2 DVB bytes, stored through a bf16 view).
template <bool OBF, int DVB, bool PK>
__device__ __forceinline__ void output_drain(const Ctx& x, uint32_t tlane, int b, int h, int dv,
                                             int hf, int c, bool leader) {
  const float* G = x.gates(c);
  // staging tile [64 tokens][DVB]; with DVB = 64 lanes 64..127 hold zero rows
  const bool own = DVB == D || dv < DVB;
  float* so = reinterpret_cast<float*>(x.sm + SM_XH) + dv;
  __nv_bfloat16* so16 = reinterpret_cast<__nv_bfloat16*>(x.sm + SM_XH) + dv;
#pragma unroll
  for (int q = 0; q < 2; ++q) {
    float y[16], oi[16];
    tmem_ld16x2(tlane + TM_Y + 32 * hf + 16 * q, y, tlane + TM_OI + 32 * hf + 16 * q, oi);
#pragma unroll
    for (int e4 = 0; e4 < 4; ++e4) {
      const float4 gm = ld4(G + G_GAM / 4 + 32 * hf + 16 * q + 4 * e4);
      const float gv[4] = {gm.x, gm.y, gm.z, gm.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int n = 32 * hf + 16 * q + 4 * e4 + e;  // token within the tile
        const float ov = fmaf(gv[e], y[4 * e4 + e], oi[4 * e4 + e]);
        if (!own) continue;
        if constexpr (OBF)
          so16[n * DVB] = __float2bfloat16_rn(ov);
        else
          so[n * DVB] = ov;
      }
    }
  }
  fence_proxy_async_smem();
  named_bar(BAR_CHAIN, CHAIN_THREADS);
  const int ts = x.tok0 + c * NT;
  if (ts + NT <= x.tend || x.tend == x.tmap) {
    // whole tile, or the view's own end clips it
    if (leader) {
      tma_store_4d(x.tmo, x.sb + SM_XH, x.dv0, h, ts, b);
      bulk_commit();
    }
  } else if constexpr (!OBF && PK) {
    // last tile of a packed sequence: the rows past it belong to the next
    // sequence, so only the valid rows are copied out
    store_partial_tile<DVB>(reinterpret_cast<const float4*>(x.sm + SM_XH),
                            x.odst + ((size_t(b) * x.tmap + ts) * x.H + h) * *x.misc(M_OROW) + x.dv0,
                            size_t(x.H) * *x.misc(M_OROW), x.tend - ts, hf * 128 + dv);
  } else if constexpr (OBF && PK) {
    store_partial_tile_bf16<DVB>(
        reinterpret_cast<const uint4*>(x.sm + SM_XH),
        reinterpret_cast<__nv_bfloat16*>(x.odst) + ((size_t(b) * x.tmap + ts) * x.H + h) * *x.misc(M_OROW) + x.dv0,
        size_t(x.H) * *x.misc(M_OROW), x.tend - ts, hf * 128 + dv);
  }
}

template <int C, bool PRE, int DK, int DVB>
__device__ void kside_role(const Ctx& x, const CUtensorMap* tq, const CUtensorMap* tk,
                           const CUtensorMap* tv, const PrefillArgs& p, int b, int h, int ntiles) {
  const int kt = threadIdx.x - 128;        // 0..255
  const int warp = threadIdx.x >> 5;
  const int lq = warp & 3;
  const int hf = (warp >= 8) ? 1 : 0;      // column half
  const int row = lq * 32 + (threadIdx.x & 31);  // TMEM lane: row of [K;Q], or Dv row
  const bool leader = (kt == 0);
  const uint32_t tlane = x.tmem + (uint32_t(lq * 32) << 16);
  const int T = p.T;
  float* sA = reinterpret_cast<float*>(x.sm + SM_A);
  float* sTf = reinterpret_cast<float*>(x.sm + SM_TF);
  float* sAt = reinterpret_cast<float*>(x.sm + SM_AT);
  volatile float* s_part = reinterpret_cast<volatile float*>(x.misc(M_PART));
  RoleSync rs{BAR_SIDE, SIDE_THREADS, M_FLAG_SIDE, leader, 0};

  if (leader) {
    issue_kq<DK>(x, tq, tk, 0, h, b);
    if (ntiles > 1) issue_kq<DK>(x, tq, tk, 1, h, b);
    if (!x.vzero) issue_v<DVB>(x, tv, 0, h, b);
  }
  float g_next = 0.f, b_next = 0.f;
  if (kt < NT && x.tok0 + kt < x.tend) {
    const size_t gi = (size_t(b) * T + x.tok0 + kt) * p.H + h;
    g_next = __ldg(p.g + gi);
    b_next = __ldg(p.beta + gi);
  }
  if constexpr (PRE) {
    if (p.qk_norm && !rs.wait(x, x.bar(B_FULL0), 0)) return;  // the norms read tile 0
    side_norms<DK>(x, kt, 0, p);
    named_bar(BAR_SIDE, SIDE_THREADS);
  }
  side_gates<C, PRE>(x, kt, 0, T, g_next, b_next, p, b, h, s_part);
  if (!rs.wait(x, x.bar(B_FULL0), 0)) return;
  const bool p_iss = (threadIdx.x == P_ISSUER);
  if (p_iss) {
    *x.misc(M_KQ_SEEN) = 1;
    issue_p<DK>(x, 0);
  }
  int p_issued = 1;  // tiles whose P MMA was issued (the issuer's view)
  float mq[32];      // this thread's half row of Mq (lanes 64..127)

  for (int c = 0; c < ntiles; ++c) {
    const float* G = x.gates(c);
    if (!rs.wait(x, x.bar(B_PFULL), c & 1)) return;

    // ---- masks and decays of P(c), columns 32 hf ..: rows 0..63 -> A =
    //      strict_tril(beta_i Dec_ij k_i.k_j) (fp32, for the solve); rows 64..127
    //      -> Mq = tril(Dec_ij q_i.k_j) (registers)
    {
      const int i = row & (NT - 1);
      const int cs = (i / C) * C;
      const float gi = G[G_GAM2 / 4 + i];
      // row factor: beta_i (|k_i|^-1) for A, 1 (q_scale |q_i|^-1) for Mq
      float bi = (row < NT) ? G[G_B / 4 + i] : 1.f;
      if constexpr (PRE) bi = (row < NT) ? bi * G[G_KN / 4 + i] : G[G_QN / 4 + i];
      float P[32];
      tmem_ld32(tlane + TM_P + 32 * hf, P);
#pragma unroll
      for (int e4 = 0; e4 < 8; ++e4) {
        const float4 gj = ld4(G + G_GAM2 / 4 + 32 * hf + 4 * e4);
        const float gjv[4] = {gj.x, gj.y, gj.z, gj.w};
        float knv[4] = {1.f, 1.f, 1.f, 1.f};
        if constexpr (PRE) {
          const float4 kj = ld4(G + G_KN / 4 + 32 * hf + 4 * e4);
          knv[0] = kj.x; knv[1] = kj.y; knv[2] = kj.z; knv[3] = kj.w;
        }
        float m[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = 32 * hf + 4 * e4 + e;
          float v = bi * fast_exp2(gi - gjv[e]) * P[4 * e4 + e];
          if constexpr (PRE) v *= knv[e];
          m[e] = (j >= cs && (row < NT ? j < i : j <= i)) ? v : 0.f;
          mq[4 * e4 + e] = m[e];
        }
        if (row < NT)
          *reinterpret_cast<float4*>(sA + i * APAD + 32 * hf + 4 * e4) =
              make_float4(m[0], m[1], m[2], m[3]);
      }
    }
    tc_fence_before();
    named_bar(BAR_SIDE, SIDE_THREADS);
    // P(c) has been read: start P(c+1) now if its tile has landed
    if (p_iss && c + 1 < ntiles && p_issued == c + 1 &&
        mbar_try_wait(x.bar(((c + 1) & 1) ? B_FULL1 : B_FULL0), ((c + 1) >> 1) & 1)) {
      tc_fence_after();
      *x.misc(M_KQ_SEEN) = c + 2;
      issue_p<DK>(x, c + 1);
      p_issued = c + 2;
    }

    // ---- T = (I + A)^{-1}, blocked in 16 x 16 blocks.
    //  (1) diagonal blocks: thread r < 64 forms row r of its block's inverse,
    //      x (I + A_bb) = e_r, right-looking: x_i is final once every row
    //      below it has been subtracted, then x_i A_i,j leaves each acc_j (j < i);
    //  (2) with chunk 64: At_IK = T_II A_IK, then T_IJ = -sum_K At_IK T_KJ by distance.
    if (kt < NT) {
      const int r = kt, bb = r >> 4, rr = r & 15, base = bb * 16;
      float acc[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) acc[j] = (j == rr) ? 1.f : 0.f;
#pragma unroll
      for (int i = 15; i > 0; --i) {
        const float xi = acc[i];
        const float* arow = sA + (base + i) * APAD + base;
#pragma unroll
        for (int j4 = 0; j4 < 4; ++j4) {
          if (4 * j4 < i) {
            const float4 a = ld4(arow + 4 * j4);
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
    named_bar(BAR_SIDE, SIDE_THREADS);
    if constexpr (C == 64) {
      solve_at_blocks(kt, sA, sTf, sAt);
      named_bar(BAR_SIDE, SIDE_THREADS);
      solve_distance<1>(kt, sAt, sTf);
      named_bar(BAR_SIDE, SIDE_THREADS);
      solve_distance<2>(kt, sAt, sTf);
      named_bar(BAR_SIDE, SIDE_THREADS);
      solve_distance<3>(kt, sAt, sTf);
      // (the role-wide barriers of the next tile's gates, or the hand-over's
      // agreement, order these rows of T before the hand-over reads them)
    }

    // ---- gates of the next tile, while the chain is still on tile c-1 / c (with
    //      normalisation they need the tile's norms, hence the tile itself)
    if (c + 1 < ntiles) {
      if constexpr (PRE) {
        if (p.qk_norm && !rs.wait(x, x.bar(((c + 1) & 1) ? B_FULL1 : B_FULL0), ((c + 1) >> 1) & 1))
          return;
        side_norms<DK>(x, kt, c + 1, p);
        named_bar(BAR_SIDE, SIDE_THREADS);
      }
      side_gates<C, PRE, false>(x, kt, c + 1, T, g_next, b_next, p, b, h, s_part);
    }

    // ---- hand T(c), Mq(c) to the chain once it is done with tile c-1's; the
    //      same agreement closes the next tile's gates
    {
      bool ok = true;
      if (leader) {
        if (c > 0) ok = (*x.abort_flag == 0) && mbar_wait_bounded(x.bar(B_TMFREE), (c - 1) & 1, WAIT_LIMIT_NS);
        if (!ok) x.fail();
      }
      if (!rs.agree(x, ok)) return;
      if (leader && c + 1 < ntiles) mbar_arrive(x.bar(gfull_off(c + 1)));
    }
    if (row < NT) {
#pragma unroll
      for (int c8 = 0; c8 < 4; ++c8)
        store_split8(x.sb + SM_TH, x.sb + SM_TL, row, 4 * hf + c8, sTf + row * APAD + 32 * hf + 8 * c8);
    } else {
#pragma unroll
      for (int c8 = 0; c8 < 4; ++c8)
        store_split8(x.sb + SM_MQH, x.sb + SM_MQL, row - NT, 4 * hf + c8, mq + 8 * c8);
    }
    fence_proxy_async_smem();
    named_bar(BAR_SIDE, SIDE_THREADS);
    if (leader) mbar_arrive(x.bar(B_TMFULL));

    // ---- P(c+1), if it could not be started early: its issuer waits for the
    //      tile alone (a failed wait aborts the CTA; the next agreement sees it)
    if (c + 1 < ntiles && p_iss && p_issued == c + 1) {
      if (*x.abort_flag == 0 &&
          mbar_wait_bounded(x.bar(((c + 1) & 1) ? B_FULL1 : B_FULL0), ((c + 1) >> 1) & 1, WAIT_LIMIT_NS)) {
        tc_fence_after();
        *x.misc(M_KQ_SEEN) = c + 2;
        issue_p<DK>(x, c + 1);
        p_issued = c + 2;
      } else {
        x.fail();
      }
    }
  }
}

// Copies columns col0 .. col0+63 of this lane's state row (fp32, TMEM) to
// dst_row + col0.  Out of line: it runs only at snapshot tile ends.
__device__ __noinline__ void snapshot_row(uint32_t tlane, int col0, float* dst_row) {
#pragma unroll 1
  for (int q = 0; q < 2; ++q) {
    float v[32];
    tmem_ld32(tlane + TM_S + col0 + 32 * q, v);
#pragma unroll
    for (int e = 0; e < 8; ++e)
      reinterpret_cast<float4*>(dst_row + col0 + 32 * q)[e] =
          make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
  }
}
// The same for the other head dims: NQ groups of 32 columns (own: the lane
// holds one of the CTA's rows; the loads are warp-wide either way).
template <int NQ>
__device__ __noinline__ void snapshot_row_n(uint32_t tlane, int col0, float* dst_row, bool own) {
#pragma unroll 1
  for (int q = 0; q < NQ; ++q) {
    float v[32];
    tmem_ld32(tlane + TM_S + col0 + 32 * q, v);
    if (!own) continue;
#pragma unroll
    for (int e = 0; e < 8; ++e)
      reinterpret_cast<float4*>(dst_row + col0 + 32 * q)[e] =
          make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
  }
}

// Copies the staged 128 x 128 fp32 state (rows of 512 B, 16-byte chunks
// XOR-swizzled by the row) to dst, row by row: chain thread ct takes every
// CHAIN_THREADS-th chunk.
__device__ __noinline__ void copy_staged_state(const uint8_t* stg, float* dst, int ct) {
  float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll 4
  for (int i = 0; i < 16; ++i) {
    const int cidx = ct + CHAIN_THREADS * i;  // 16-byte chunk: row cidx / 32, column cidx % 32
    const int r = cidx >> 5, j = cidx & 31;
    d4[cidx] = *reinterpret_cast<const float4*>(stg + r * 512 + ((j ^ (r & 7)) * 16));
  }
}

// Z = S_c K^T (into TM_Z) and Y = S_c Q^T (into TM_Y) for chunk s of the tile
// in `kq`: A = the bf16 hi / lo state pair in TMEM, B = K and Q rows.  With
// chunk 64 the K and Q rows of the tile are adjacent (64 + 64 rows) and Y sits
// right after Z in TMEM, so one N = 128 MMA per step computes both.
template <int C, int DK>
__device__ __forceinline__ void issue_zq(const Ctx& x, uint32_t kq, int s) {
  // C rows of 128 B per chunk (C = 16)
  const uint64_t d0 = sdesc_sw128(kq + 2048u * uint32_t(s), 16, 1024);
#pragma unroll
  for (int part = 0; part < 2; ++part) {
    const uint32_t a0 = x.tmem + (part ? TM_SLO : TM_SHI);
#pragma unroll
    for (int kk = 0; kk < DK / 16; ++kk) {
      const uint32_t off = (kk >> 2) * 16384 + (kk & 3) * 32;
      const uint32_t acc = (part | kk) ? 1u : 0u;
      if constexpr (C == 64) {
        static_assert(TM_Y == TM_Z + 64, "Y follows Z");
        mma_ts(x.tmem + TM_Z, a0 + kk * 8, sdesc_add(d0, off), idesc_bf16(128, 128, 0, 0, 0), acc);
      } else {
        const uint32_t id = idesc_bf16(128, C, 0, 0, 0);
        mma_ts(x.tmem + TM_Z + C * s, a0 + kk * 8, sdesc_add(d0, off), id, acc);
        mma_ts(x.tmem + TM_Y + C * s, a0 + kk * 8, sdesc_add(d0, off + 8192), id, acc);
      }
    }
  }
}

// ============================================================== chain
template <int C, bool OBF, int DK, int DVB, bool PK>
__device__ void chain_role(const Ctx& x, const CUtensorMap* tq, const CUtensorMap* tk,
                           const CUtensorMap* tv, const PrefillArgs& p, int chain, int b, int h,
                           int ntiles) {
  constexpr int NSUB = NT / C;
  constexpr int NC = C / 2;      // columns of a chunk per chain thread
  constexpr int NQ = DK / 64;    // 32-column groups of the state per chain thread
  constexpr int SCOLS = DK / 2;  // state columns per chain thread
  const int warp = threadIdx.x >> 5;
  const int lq = warp & 3;
  const int ch = (warp >= 12) ? 1 : 0;      // column half
  const int dv = lq * 32 + (threadIdx.x & 31);
  const bool leader = (threadIdx.x == 0);
  const uint32_t tlane = x.tmem + (uint32_t(lq * 32) << 16);
  const uint32_t sb = x.sb;
  RoleSync rs{BAR_CHAIN, CHAIN_THREADS, M_FLAG_CHAIN, leader, 0};

  // ---- initial state (row dv of S0, or zeros; rows past the CTA's own stay
  //      zero): hi/lo copy, and the fp32 copy pre-scaled by the decay of the
  //      first chunk
  if (!rs.wait(x, x.bar(gfull_off(0)), gfull_parity(0))) return;
  {
    const float gc0 = x.gates(0)[G_GC / 4];
    const float4* src = (x.s0src && (DVB == D || dv < DVB))
                            ? reinterpret_cast<const float4*>(x.s0src + size_t(dv) * DK)
                            : nullptr;
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
      const int qq = NQ * ch + q;  // 32-column group
      float v[32];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float4 a = src ? __ldg(src + 8 * qq + e) : make_float4(0.f, 0.f, 0.f, 0.f);
        v[4 * e] = a.x;
        v[4 * e + 1] = a.y;
        v[4 * e + 2] = a.z;
        v[4 * e + 3] = a.w;
      }
      if (x.s0_identity) {
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = (32 * qq + e == dv) ? 1.f : 0.f;
      }
      store_state_split32(tlane, qq, v);
      uint32_t u[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) u[e] = __float_as_uint(gc0 * v[e]);
      tmem_st32(tlane + TM_S + 32 * qq, u);
    }
  }
  tc_fence_before();
  named_bar(BAR_CHAIN, CHAIN_THREADS);

  uint32_t sc = 0;  // chunks processed (phase of the per-chunk MMA barriers)
  for (int c = 0; c < ntiles; ++c) {
    const uint32_t kq = sb + ((c & 1) ? SM_KQ1 : SM_KQ0);
    const float* G = x.gates(c);
    const bool last_tile = (c + 1 == ntiles);
#pragma unroll 1
    for (int s = 0; s < NSUB; ++s, ++sc) {
      // ---- Z = S_c K^T and Y = S_c Q^T : M=128 (dv), N=C each, K=128 (dk); A = S hi,
      //      then S lo
      if (leader) {
        bool ok = true;
        if (s == 0) {
          ok = mbar_wait_bounded(x.bar((c & 1) ? B_FULL1 : B_FULL0), (c >> 1) & 1, WAIT_LIMIT_NS);
        }
        if (!ok) x.fail();
        if (ok && !*x.abort_flag) {
          tc_fence_after();
          issue_zq<C, DK>(x, kq, s);
          mma_commit(x.bar(B_ZQ));
        }
      }
      // one agreement: Z is in TMEM and, at a tile's first chunk, its gates and V are in
      {
        bool ok = true;
        if (leader) {
          bulk_wait_read0();  // the previous tile's o store has read its staging tile
          ok = (*x.abort_flag == 0) && mbar_wait_bounded(x.bar(B_ZQ), sc & 1, WAIT_LIMIT_NS);
          if (ok && s == 0)
            ok = mbar_wait_bounded(x.bar(gfull_off(c)), gfull_parity(c), WAIT_LIMIT_NS);
          if (ok && s == 0 && !x.vzero) {
            ok = mbar_wait_bounded(x.bar(B_VFULL), c & 1, WAIT_LIMIT_NS);
            if (ok) *x.misc(M_V_SEEN) = c + 1;
          }
          if (!ok) x.fail();
        }
        if (!rs.agree(x, ok)) return;
      }

      // ---- X^T[dv][n] = beta_n V[n][dv] - beta_n Gamma_n Z[dv][n], as a hi/lo
      //      pair into the chunk's Z columns once every thread has read its Z
      //      (the A operand of the residual product, read from tensor memory)
      {
        const __nv_bfloat16* V = reinterpret_cast<const __nv_bfloat16*>(x.sm + SM_V);
        const int n0 = C * s + NC * ch;
        float z[NC];
        if constexpr (NC == 32) {
          tmem_ld32(tlane + TM_Z + n0, z);
        } else {
          float za[4], zb[4];
          tmem_ld4(tlane + TM_Z + n0, za);
          tmem_ld4(tlane + TM_Z + n0 + 4, zb);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            z[e] = za[e];
            z[4 + e] = zb[e];
          }
        }
        float xv[NC];
#pragma unroll
        for (int e4 = 0; e4 < NC / 4; ++e4) {
          const float4 bb = ld4(G + G_B / 4 + n0 + 4 * e4);
          const float4 bg = ld4(G + G_BG / 4 + n0 + 4 * e4);
          const float bv[4] = {bb.x, bb.y, bb.z, bb.w};
          const float gv[4] = {bg.x, bg.y, bg.z, bg.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int n = n0 + 4 * e4 + e;
            const float vn = (x.vzero || (DVB != D && dv >= DVB)) ? 0.f : __bfloat162float(V[n * DVB + dv]);
            xv[4 * e4 + e] = fmaf(bv[e], vn, -gv[e] * z[4 * e4 + e]);
          }
        }
        named_bar(BAR_CHAIN, CHAIN_THREADS);  // every thread's Z columns have been read
        store_pairs_split<NC>(tlane + TM_Z + C * s + NC * ch / 2, tlane + TM_Z + C * s + C / 2 + NC * ch / 2,
                              xv);
      }
      tc_fence_before();
      named_bar(BAR_CHAIN, CHAIN_THREADS);
      if (leader && s == NSUB - 1 && !last_tile && !x.vzero) issue_v<DVB>(x, tv, c + 1, h, b);  // V(c) read

      // ---- Dl^T = X^T T^T : M=128 (dv), N=C (i), K=C (n); 3 hi/lo products, A (X)
      //      from tensor memory, into the chunk's O_intra columns (free until its
      //      output product)
      if (leader) {
        bool ok = true;
        if (s == 0) ok = mbar_wait_bounded(x.bar(B_TMFULL), c & 1, WAIT_LIMIT_NS);
        if (!ok) x.fail();
        if (ok && !*x.abort_flag) {
          tc_fence_after();
          const uint32_t id = idesc_bf16(128, C, 0, 0, 0);
          const uint64_t d0 = sdesc_sw128(sb + uint32_t(C * s) * 2u, 16, 1024);  // chunk's K offset
          const uint32_t trow = uint32_t(C * s / 8) * 1024u;
#pragma unroll
          for (int part = 0; part < 3; ++part) {
            const uint32_t xa = x.tmem + TM_Z + C * s + (part == 2 ? C / 2 : 0);
            const uint32_t tb = (part == 1 ? SM_TL : SM_TH) + trow;
#pragma unroll
            for (int ks = 0; ks < C / 16; ++ks) {
              const uint32_t kb = uint32_t(16 * ks) * 2u;
              mma_ts(x.tmem + TM_OI + C * s, xa + 8 * ks, sdesc_add(d0, tb + kb), id,
                     (part | ks) ? 1u : 0u);
            }
          }
          mma_commit(x.bar(B_DL));
        }
      }
      {
        // the previous chunk's output product (another issuer) must have read the
        // Dl tiles before they are rewritten
        bool ok = true;
        if (leader) {
          ok = (*x.abort_flag == 0) && mbar_wait_bounded(x.bar(B_DL), sc & 1, WAIT_LIMIT_NS);
          if (ok && s > 0) ok = mbar_wait_bounded(x.bar(B_OI), (sc - 1) & 1, WAIT_LIMIT_NS);
          if (!ok) x.fail();
        }
        if (!rs.agree(x, ok)) return;
      }

      // ---- residuals: Dl (for the output product: hi/lo into shared memory) and
      //      Dl~ = Dl * exp(gamma_last - gamma) (for the state update: hi/lo into the
      //      chunk's Z columns, whose X has been consumed)
      {
        const int n0 = C * s + NC * ch;
        float d[NC];
        if constexpr (NC == 32) {
          tmem_ld32(tlane + TM_OI + n0, d);
        } else {
          float da[4], db[4];
          tmem_ld4(tlane + TM_OI + n0, da);
          tmem_ld4(tlane + TM_OI + n0 + 4, db);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            d[e] = da[e];
            d[4 + e] = db[e];
          }
        }
        float dt[NC];
#pragma unroll
        for (int e4 = 0; e4 < NC / 4; ++e4) {
          const float4 f = ld4(G + G_DF / 4 + n0 + 4 * e4);
          dt[4 * e4 + 0] = d[4 * e4 + 0] * f.x;
          dt[4 * e4 + 1] = d[4 * e4 + 1] * f.y;
          dt[4 * e4 + 2] = d[4 * e4 + 2] * f.z;
          dt[4 * e4 + 3] = d[4 * e4 + 3] * f.w;
        }
#pragma unroll
        for (int e = 0; e < NC / 8; ++e) store_split8(sb + SM_DH, sb + SM_DL, dv, n0 / 8 + e, d + 8 * e);
        store_pairs_split<NC>(tlane + TM_Z + C * s + NC * ch / 2, tlane + TM_Z + C * s + C / 2 + NC * ch / 2,
                              dt);
      }
      fence_proxy_async_smem();
      tc_fence_before();
      named_bar(BAR_CHAIN, CHAIN_THREADS);

      // ---- S += Dl~^T K (N = Dk, B = K tile MN-major; the chain leader) and
      //      O_intra = Dl^T Mq^T (N = C; a second issuer), committed separately:
      //      the state epilogue waits for the update only
      if (leader && !*x.abort_flag) {
        tc_fence_after();
        const uint32_t idu = idesc_bf16(128, DK, 0, 1, 0);
        const uint64_t dk = sdesc_sw128(kq + uint32_t(C * s) * 128u, 16384, 1024);  // K rows, MN-major
#pragma unroll
        for (int part = 0; part < 2; ++part) {
          const uint32_t da = x.tmem + TM_Z + C * s + (part ? C / 2 : 0);  // Dl~ hi / lo (TMEM)
#pragma unroll
          for (int ks = 0; ks < C / 16; ++ks) {
            mma_ts(x.tmem + TM_S, da + 8 * ks, sdesc_add(dk, uint32_t(16 * ks) * 128u), idu, 1u);
          }
        }
        mma_commit(x.bar(B_SU));
      }
      if (threadIdx.x == OI_ISSUER && !*x.abort_flag) {
        tc_fence_after();
        const uint32_t id = idesc_bf16(128, C, 0, 0, 0);
        const uint64_t d0 = sdesc_sw128(sb + uint32_t(C * s) * 2u, 16, 1024);  // chunk's K offset
        const uint32_t mrow = uint32_t(C * s / 8) * 1024u;
#pragma unroll
        for (int part = 0; part < 3; ++part) {
          const uint32_t da = part == 2 ? SM_DL : SM_DH;
          const uint32_t mb = (part == 1 ? SM_MQL : SM_MQH) + mrow;
#pragma unroll
          for (int ks = 0; ks < C / 16; ++ks) {
            const uint32_t kb = uint32_t(16 * ks) * 2u;
            mma_ss(x.tmem + TM_OI + C * s, sdesc_add(d0, da + kb), sdesc_add(d0, mb + kb), id,
                   (part | ks) ? 1u : 0u);
          }
        }
        mma_commit(x.bar(B_OI));
        if (s == NSUB - 1) mma_commit(x.bar(B_TMFREE));  // T(c), Mq(c) consumed (Dl(c) waited)
      }
      if (!rs.wait(x, x.bar(B_SU), sc & 1)) return;
      if (leader && s == NSUB - 1 && c + 2 < ntiles) issue_kq<DK>(x, tq, tk, c + 2, h, b);  // KQ(c) read

      // ---- the last tile: o first (its staging area then holds the end state)
      if (last_tile && s == NSUB - 1) {
        if (!rs.wait(x, x.bar(B_OI), sc & 1)) return;
        output_drain<OBF, DVB, PK>(x, tlane, b, h, dv, ch, c, leader);
      }

      // ---- S_out now sits in TMEM: refresh its hi/lo copy, and pre-scale it by
      //      the next chunk's decay (or store it as S_T after the last chunk)
      {
        const bool final_chunk = last_tile && (s == NSUB - 1);
        float gnext = 0.f;
        if (s + 1 < NSUB) {
          gnext = G[G_GC / 4 + s + 1];
        } else if (!last_tile) {
          if (!rs.wait(x, x.bar(gfull_off(c + 1)), gfull_parity(c + 1))) return;
          gnext = x.gates(c + 1)[G_GC / 4];
        }
        if (final_chunk && (DK != D || DVB != D)) {
          // other head dims: this thread's columns of its own row, straight to HBM,
          // and into the last snapshot slot when the packed sequence ends on one
          // (the loads are warp-wide; lanes past the CTA's rows store nothing)
          const bool own = DVB == D || dv < DVB;
          float4* dst = reinterpret_cast<float4*>(x.sdst + size_t(dv) * DK + SCOLS * ch);
          float4* sdst = nullptr;
          if constexpr (PK) {
            const int stiles = *x.misc(M_SNAP_TILES);
            if (stiles && (x.tend - x.tok0) % (stiles * NT) == 0)
              sdst = reinterpret_cast<float4*>(
                  *reinterpret_cast<float* volatile*>(x.sm + SM_MISC + M_SNAP_PTR) +
                  size_t((x.tend - x.tok0) / (stiles * NT) - 1) * x.H * p.Dv * DK + size_t(dv) * DK +
                  SCOLS * ch);
          }
#pragma unroll
          for (int q = 0; q < NQ; ++q) {
            float v[32];
            tmem_ld32(tlane + TM_S + SCOLS * ch + 32 * q, v);
            if (!own) continue;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float4 w = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
              dst[8 * q + e] = w;
              if (sdst) sdst[8 * q + e] = w;
            }
          }
        } else if (final_chunk) {
          // the end state goes out through the o staging / Dl^T region (64 KB, free once
          // the o store has read it): rows of 512 B whose 16-byte chunks are
          // XOR-swizzled by the row, then copied out row by row
          if (leader) bulk_wait_read0();
          named_bar(BAR_CHAIN, CHAIN_THREADS);
          const uint32_t stg = sb + SM_XH;
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            const int col = 64 * ch + 32 * q;
            float v[32];
            tmem_ld32(tlane + TM_S + col, v);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              st_shared_v4(stg + uint32_t(dv) * 512u + uint32_t(((col / 4 + e) ^ (dv & 7)) * 16),
                           __float_as_uint(v[4 * e]), __float_as_uint(v[4 * e + 1]),
                           __float_as_uint(v[4 * e + 2]), __float_as_uint(v[4 * e + 3]));
          }
          named_bar(BAR_CHAIN, CHAIN_THREADS);
          copy_staged_state(x.sm + SM_XH, x.sdst, ch * 128 + dv);
          if constexpr (PK) {
            const int stiles = *x.misc(M_SNAP_TILES);
            if (stiles && (x.tend - x.tok0) % (stiles * NT) == 0) {
              // the sequence ends on a snapshot boundary: its last snapshot is S_T
              float* snap = *reinterpret_cast<float* volatile*>(x.sm + SM_MISC + M_SNAP_PTR);
              copy_staged_state(x.sm + SM_XH,
                                snap + size_t((x.tend - x.tok0) / (stiles * NT) - 1) * x.H * p.Dv * D,
                                ch * 128 + dv);
            }
          }
        } else {
          // at a snapshot tile end, the state itself first goes to its slot
          if (PK && s == NSUB - 1) {
            const int stiles = *x.misc(M_SNAP_TILES);
            if (stiles && (c + 1) % stiles == 0) {
              float* snap = *reinterpret_cast<float* volatile*>(x.sm + SM_MISC + M_SNAP_PTR);
              if constexpr (DK == D && DVB == D)
                snapshot_row(tlane, 64 * ch, snap + (size_t((c + 1) / stiles - 1) * x.H * p.Dv + dv) * D);
              else
                snapshot_row_n<NQ>(tlane, SCOLS * ch,
                                   snap + size_t((c + 1) / stiles - 1) * x.H * p.Dv * DK + size_t(dv) * DK,
                                   DVB == D || dv < DVB);
            }
          }
          // this thread's DK / 2 columns, 32 at a time: load, split, store hi / lo /
          // pre-scaled fp32 in one waited group
#pragma unroll
          for (int q = 0; q < NQ; ++q) {
            const int col = SCOLS * ch + 32 * q;
            float v[32];
            tmem_ld32(tlane + TM_S + col, v);
            uint32_t hi[16], lo[16], u[32];
#pragma unroll
            for (int e = 0; e < 16; ++e) split2_bf16(v[2 * e], v[2 * e + 1], hi[e], lo[e]);
#pragma unroll
            for (int e = 0; e < 32; ++e) u[e] = __float_as_uint(gnext * v[e]);
            tmem_st_state(tlane + TM_SHI + col / 2, hi, tlane + TM_SLO + col / 2, lo,
                          tlane + TM_S + col, u);
          }
        }
      }
      // ---- o of the whole tile is complete after its last chunk's output
      //      product: o[t][dv] = Gamma_t Y[dv][t] + O_intra[dv][t], to HBM (before
      //      the next tile's [Z|Y] product rewrites Y)
      if (s == NSUB - 1 && !last_tile) {
        tc_fence_before();
        if (!rs.wait(x, x.bar(B_OI), sc & 1)) return;
        output_drain<OBF, DVB, PK>(x, tlane, b, h, dv, ch, c, leader);
      }
      tc_fence_before();
      if (!rs.check(x)) return;
    }
  }
}

template <int C, bool PRE, bool OBF, int DK, int DVB, bool PK = false>
__global__ void __launch_bounds__(NTHREADS, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                   const __grid_constant__ CUtensorMap tm_f, const PrefillArgs p) {
  static_assert(C == 16 || C == 64, "chunk must be 16 or 64");
  static_assert(DK == 64 || DK == 128, "key dimension must be 64 or 128");
  static_assert(DVB == 64 || DVB == 128, "a CTA owns 64 or 128 rows of the state");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int total_tiles = (p.T + NT - 1) / NT;
  // CTA -> (chain, segment, kind, rows of the state); see PrefillArgs
  const int dvpart = int(blockIdx.x) % p.dv_ctas;
  const int cta = int(blockIdx.x) / p.dv_ctas;
  int chain = cta, seg = 0;
  bool frun = false;
  if (p.nseg > 1) {
    const int per = 2 * p.nseg - 1;
    chain = cta / per;
    const int j = cta - chain * per;
    frun = j >= p.nseg;
    seg = frun ? j - p.nseg + 1 : j;
  }
  if constexpr (PK) {
    // longest sequences first: CTAs start in index order, so slot n H + h of the
    // grid takes the sequence of rank n by (length descending, index), a
    // bijection whatever the offsets hold; the shorter chains then fill the SMs
    // the long ones leave.  Up to one sequence per thread (else index order).
    if (p.B <= NTHREADS) {
      int* lens = reinterpret_cast<int*>(sm + SM_A);  // scratch: the solve has not started
      for (int i = tid; i < p.B; i += NTHREADS)
        lens[i] = __ldg(p.cu_seqlens + i + 1) - __ldg(p.cu_seqlens + i);
      __syncthreads();
      const int r = chain / p.H;
      if (tid < p.B) {
        const int L = lens[tid];
        int rank = 0;
        for (int m = 0; m < p.B; ++m) {
          const int Lm = lens[m];
          rank += (Lm > L || (Lm == L && m < tid)) ? 1 : 0;
        }
        if (rank == r) lens[NTHREADS] = tid;
      }
      __syncthreads();
      chain = lens[NTHREADS] * p.H + (chain - r * p.H);
    }
  }
  int b = chain / p.H;
  const int h = chain - b * p.H;
  const size_t cstate = size_t(chain) * p.Dv * DK;  // this chain's state
  const int dv0 = dvpart * 128;                       // first row owned by this CTA

  Ctx x;
  x.sm = sm;
  x.sb = smem_u32(sm);
  x.status = p.status;
  x.H = p.H;
  x.abort_flag = reinterpret_cast<volatile int*>(sm + SM_MISC + M_ABORT);
  x.tok0 = 0;
  x.tend = p.T;
  x.tmap = p.T;
  x.dv0 = dv0;
  int ntiles = total_tiles;
  if (PK) {
    // packed sequences: chain = n H + h walks tokens [cu[n], cu[n+1]) of views with B = 1
    const int start = __ldg(p.cu_seqlens + b), end = __ldg(p.cu_seqlens + b + 1);
    if (start < 0 || end < start || end > p.T) {
      if (tid == 0 && p.status) atomicExch(p.status, GDN_ERR_SHAPE);
      return;
    }
    x.tok0 = start;
    x.tend = end;
    b = 0;
    ntiles = (end - start + NT - 1) / NT;
    if (ntiles == 0) {  // empty sequence: S_T = S0 (or zeros), this CTA's rows
      const size_t off = cstate + size_t(dv0) * DK;
      const float4* src = p.S0 ? reinterpret_cast<const float4*>(p.S0 + off) : nullptr;
      float4* dst = reinterpret_cast<float4*>(p.S_T + off);
      for (int i = tid; i < p.dv_box * DK / 4; i += NTHREADS)
        dst[i] = src ? src[i] : make_float4(0.f, 0.f, 0.f, 0.f);
      return;
    }
  }
  x.vzero = frun;
  x.s0_identity = frun;
  x.s0src = (seg == 0 && p.S0) ? p.S0 + cstate + size_t(dv0) * DK : nullptr;
  x.odst = frun ? p.ws_f : p.o;
  x.tmo = frun ? &tm_f : &tm_o;
  if (p.nseg > 1) {
    const int tb = seg * p.seg_tiles;
    x.tok0 = tb * NT;
    ntiles = min(p.seg_tiles, total_tiles - tb);
    x.sdst = (frun ? p.ws_F : p.ws_R) + (size_t(chain) * p.nseg + seg) * D * D;
  } else {
    x.sdst = p.S_T + cstate + size_t(dv0) * DK;
  }
  if (tid == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(x.tmo);
    for (int i = 0; i < NUM_BARS; ++i) mbar_init(x.sb + SM_BAR + 8 * i, 1);
    fence_mbar_init();
    for (int i = 0; i < 16; ++i) reinterpret_cast<volatile int*>(sm + SM_MISC)[i] = 0;
    if (PK) *reinterpret_cast<volatile int*>(sm + SM_MISC + M_OROW) = p.Dv;
    if (PK && p.snaps) {
      // first snapshot slot of this sequence: one per snap_every tokens of
      // every earlier sequence; an invalid earlier entry (its own CTAs report
      // it) leaves this sequence without snapshots rather than with a slot
      // index computed from garbage
      const int n = chain / p.H;
      int base = 0;
      bool offsets_ok = true;
      for (int m = 0; m < n; ++m) {
        const int s0 = __ldg(p.cu_seqlens + m), s1 = __ldg(p.cu_seqlens + m + 1);
        if (s0 < 0 || s1 < s0 || s1 > p.T) {
          offsets_ok = false;
          break;
        }
        base += (s1 - s0) / p.snap_every;
      }
      if (!offsets_ok || base < 0 || base + (x.tend - x.tok0) / p.snap_every > p.n_snaps) {
        if (p.status) atomicExch(p.status, GDN_ERR_SHAPE);
      } else {
        *reinterpret_cast<float* volatile*>(sm + SM_MISC + M_SNAP_PTR) =
            p.snaps + (size_t(base) * p.H + h) * p.Dv * DK + size_t(dv0) * DK;
        *x.misc(M_SNAP_TILES) = p.snap_every / NT;
      }
    }
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(sm + SM_MISC + M_TMEM), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  x.tmem = *reinterpret_cast<volatile uint32_t*>(sm + SM_MISC + M_TMEM);

  // a dependent launch (the segment fix) may begin its set-up now; it waits
  // for this grid to complete before it reads anything this grid writes
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (warp < 4 || warp >= 12)
    chain_role<C, OBF, DK, DVB, PK>(x, &tm_q, &tm_k, &tm_v, p, chain, b, h, ntiles);
  else
    kside_role<C, PRE, DK, DVB>(x, &tm_q, &tm_k, &tm_v, p, b, h, ntiles);

  // every MMA issuer waits (bounded) for its own products in flight
  if (tid == 0 || tid == 128 || tid == OI_ISSUER || tid == P_ISSUER) {
    const uint32_t bc = x.bar(tid == 0 ? B_CLEAN0 : tid == 128 ? B_CLEAN1 : tid == OI_ISSUER ? B_CLEAN2 : B_CLEAN3);
    mma_commit(bc);
    mbar_wait_bounded(bc, 0, WAIT_LIMIT_NS / 4);
  }
  if (tid == 0) bulk_wait0();  // the chain leader's o stores have completed
  tc_fence_before();
  __syncthreads();
  // An aborted CTA may still have TMA loads in flight: wait for them (bounded)
  // before the shared memory is released.
  if (tid == 0 && *x.abort_flag) {
    const int kq_issued = *x.misc(M_KQ_ISSUED), kq_seen = *x.misc(M_KQ_SEEN);
    for (int c = kq_seen; c < kq_issued; ++c)
      mbar_wait_bounded(x.bar((c & 1) ? B_FULL1 : B_FULL0), (c >> 1) & 1, WAIT_LIMIT_NS / 4);
    const int v_issued = *x.misc(M_V_ISSUED), v_seen = *x.misc(M_V_SEEN);
    if (v_issued > v_seen) mbar_wait_bounded(x.bar(B_VFULL), (v_issued - 1) & 1, WAIT_LIMIT_NS / 4);
  }
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(x.tmem, TMEM_COLS);
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
                   const CUtensorMap& to, const CUtensorMap& tf, const PrefillArgs& a, int chunk,
                   cudaStream_t stream) {
  const int chains = a.B * a.H;
  if (chains == 0) return 0;
  if (a.T == 0) {
    const size_t n4 = size_t(chains) * a.Dv * a.Dk / 4;
    if (a.S0 == a.S_T) return 0;
    copy_state_kernel<<<unsigned((n4 + 255) / 256), 256, 0, stream>>>(a.S0, a.S_T, n4);
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
  }
  const uint32_t smem = SMEM_USED + 1024;
  const int ctas = (a.nseg > 1 ? chains * (2 * a.nseg - 1) : chains) * a.dv_ctas;
  const bool pre = a.qk_norm || a.q_scale != 1.f;  // fused q / k pre-steps requested
  auto go = [&](auto kernel, int slot) {
    if (!ensure_smem_attr(reinterpret_cast<const void*>(kernel), slot, int(smem))) return false;
    kernel<<<ctas, NTHREADS, smem, stream>>>(tq, tk, tv, to, tf, a);
    return true;
  };
  const bool obf = a.o_bf16 != 0;
  bool ok;
  if (a.cu_seqlens) {
    // packed sequences (the pre-steps and bf16 o on request): their own
    // instantiations, so that the dense kernels carry none of the per-sequence paths
    const bool c64 = chunk == 64;
    if (!pre && !obf) {
      if (a.Dk == D)
        ok = a.dv_box == D ? (c64 ? go(prefill_kernel<64, false, false, 128, 128, true>, 55)
                                  : go(prefill_kernel<16, false, false, 128, 128, true>, 56))
                           : (c64 ? go(prefill_kernel<64, false, false, 128, 64, true>, 57)
                                  : go(prefill_kernel<16, false, false, 128, 64, true>, 58));
      else
        ok = a.dv_box == D ? (c64 ? go(prefill_kernel<64, false, false, 64, 128, true>, 59)
                                  : go(prefill_kernel<16, false, false, 64, 128, true>, 60))
                           : (c64 ? go(prefill_kernel<64, false, false, 64, 64, true>, 61)
                                  : go(prefill_kernel<16, false, false, 64, 64, true>, 62));
    } else if (obf) {
      // bf16 o: the pre-step instantiations (with no pre-step requested their
      // factors are exactly 1)
      if (a.Dk == D)
        ok = a.dv_box == D ? (c64 ? go(prefill_kernel<64, true, true, 128, 128, true>, 78)
                                  : go(prefill_kernel<16, true, true, 128, 128, true>, 79))
                           : (c64 ? go(prefill_kernel<64, true, true, 128, 64, true>, 80)
                                  : go(prefill_kernel<16, true, true, 128, 64, true>, 81));
      else
        ok = a.dv_box == D ? (c64 ? go(prefill_kernel<64, true, true, 64, 128, true>, 82)
                                  : go(prefill_kernel<16, true, true, 64, 128, true>, 83))
                           : (c64 ? go(prefill_kernel<64, true, true, 64, 64, true>, 84)
                                  : go(prefill_kernel<16, true, true, 64, 64, true>, 85));
    } else {
      if (a.Dk == D)
        ok = a.dv_box == D ? (c64 ? go(prefill_kernel<64, true, false, 128, 128, true>, 67)
                                  : go(prefill_kernel<16, true, false, 128, 128, true>, 68))
                           : (c64 ? go(prefill_kernel<64, true, false, 128, 64, true>, 69)
                                  : go(prefill_kernel<16, true, false, 128, 64, true>, 70));
      else
        ok = a.dv_box == D ? (c64 ? go(prefill_kernel<64, true, false, 64, 128, true>, 71)
                                  : go(prefill_kernel<16, true, false, 64, 128, true>, 72))
                           : (c64 ? go(prefill_kernel<64, true, false, 64, 64, true>, 73)
                                  : go(prefill_kernel<16, true, false, 64, 64, true>, 74));
    }
  } else if (a.Dk == D && a.dv_box == D && a.Dv != D) {
    // Dv = 256: the 128 x 128 kernels on two CTAs per chain (rows dv0 .. dv0 + 127)
    if (chunk == 64)
      ok = obf ? (pre ? go(prefill_kernel<64, true, true, 128, 128>, 5) : go(prefill_kernel<64, false, true, 128, 128>, 6))
               : (pre ? go(prefill_kernel<64, true, false, 128, 128>, 3) : go(prefill_kernel<64, false, false, 128, 128>, 0));
    else
      ok = obf ? (pre ? go(prefill_kernel<16, true, true, 128, 128>, 7) : go(prefill_kernel<16, false, true, 128, 128>, 8))
               : (pre ? go(prefill_kernel<16, true, false, 128, 128>, 4) : go(prefill_kernel<16, false, false, 128, 128>, 1));
  } else if (a.Dk != D || a.Dv != D) {
    // Dk = 64 or Dv = 64: the pre-steps are always compiled in (with none
    // requested their factors are exactly 1, so the result is the plain one);
    // bf16 o is a separate instantiation
    const bool c64 = chunk == 64;
    if (a.Dk == D)  // Dv = 64
      ok = obf ? (c64 ? go(prefill_kernel<64, true, true, 128, 64>, 49)
                      : go(prefill_kernel<16, true, true, 128, 64>, 50))
               : (c64 ? go(prefill_kernel<64, true, false, 128, 64>, 9)
                      : go(prefill_kernel<16, true, false, 128, 64>, 10));
    else if (a.dv_box == D)  // Dk = 64, Dv = 128
      ok = obf ? (c64 ? go(prefill_kernel<64, true, true, 64, 128>, 51)
                      : go(prefill_kernel<16, true, true, 64, 128>, 52))
               : (c64 ? go(prefill_kernel<64, true, false, 64, 128>, 11)
                      : go(prefill_kernel<16, true, false, 64, 128>, 12));
    else  // Dk = Dv = 64
      ok = obf ? (c64 ? go(prefill_kernel<64, true, true, 64, 64>, 53)
                      : go(prefill_kernel<16, true, true, 64, 64>, 54))
               : (c64 ? go(prefill_kernel<64, true, false, 64, 64>, 13)
                      : go(prefill_kernel<16, true, false, 64, 64>, 14));
  } else if (chunk == 64) {
    if (obf)
      ok = pre ? go(prefill_kernel<64, true, true, 128, 128>, 5) : go(prefill_kernel<64, false, true, 128, 128>, 6);
    else
      ok = pre ? go(prefill_kernel<64, true, false, 128, 128>, 3) : go(prefill_kernel<64, false, false, 128, 128>, 0);
  } else {
    if (obf)
      ok = pre ? go(prefill_kernel<16, true, true, 128, 128>, 7) : go(prefill_kernel<16, false, true, 128, 128>, 8);
    else
      ok = pre ? go(prefill_kernel<16, true, false, 128, 128>, 4) : go(prefill_kernel<16, false, false, 128, 128>, 1);
  }
  if (!ok) return -1;
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace gdn
