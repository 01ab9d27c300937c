// Chunked delta rule with a per-channel gate (KDA) on the 5th-generation tensor
// cores (sm_100a): 32-token TMA tiles, tcgen05 MMAs accumulating in tensor
// memory, the fp32 state carried from chunk to chunk in tensor memory.
//
// Recurrence (per sequence b, head h; S in R^{Dv x Dk}, Dk = 128, Dv = 64, 128
// or 256; g_t a vector of natural-log decays over the key channels):
//   S_t = S_{t-1} diag(exp(g_t)) (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,  o_t = S_t q_t.
// The ROCmFPX gated-delta-net prefill note (bittide.aicompass.dev article
// d2880479, opening post) names KDA among the cases its chunked kernel left to
// the per-token path; this kernel chunks it.
//
// Chunked form (tokens i, j of one chunk; S_c the state entering it;
// gamma_i = inclusive cumulative sum of g inside the chunk, per channel, and
// Lambda_i = exp(gamma_i); r = the chunk's middle token):
//   K+ = K o Lambda,  Q+ = Q o Lambda                 (decayed from the chunk start)
//   K' = K o Lambda / Lambda_r,  Q' = Q o Lambda / Lambda_r,  K'' = K o Lambda_r / Lambda
//   A  = strict_tril(diag(beta) K' K''^T),   Mq = tril(Q' K''^T)   (r cancels)
//   T  = (I + A)^{-1}
//   X^T  = V^T diag(beta) - (S_c K+^T) diag(beta),   Dl^T = X^T T^T
//   O^T  = S_c Q+^T + Dl^T Mq^T
//   S'   = S_c diag(Lambda_last) + Dl^T (K o Lambda_last / Lambda)
// The reference r keeps every factor of K', Q', K'' within exp(+-16 |g|) for a
// 32-token chunk: exact while a channel's decay over 16 tokens stays above
// e^-87 (the fp32 range); beyond that the exponents are clamped (no inf/NaN).
//
// One CTA of 512 threads owns one (b, h) chain (with Dv = 256, two CTAs own
// 128 rows of its state each; with Dv = 64, lanes 64..127 of the state stay
// zero); two roles hand off through mbarriers:
//   * chain (warps 0-3, 12-15): S_c [K+;Q+]^T, X, Dl = X T^T, the state update
//     and the output product, their epilogues, and the o store;
//   * side (warps 4-11), one chunk ahead: the gates (per-channel cumulative
//     decays), the decayed operand tiles, [K';Q'] K''^T, masks, the triangular
//     solve, and the hand-over of T, Mq and the chain's operand tiles.
// Every operand derived in the kernel is fed to the tensor core as a bf16
// hi/lo pair (hi = bf16(x), lo = bf16(x - hi)); products of two derived
// operands take hi*hi + hi*lo + lo*hi.  Where a product has an exact A
// operand or a free N dimension, the hi and lo of one operand are stacked
// along N and the halves summed in the epilogue (fewer MMA instructions).
//
// Tensor memory (512 columns, fp32):
//   [  0,128) S   : state, pre-scaled by the next chunk's decay (per column)
//   [128,192) SHI : S hi (bf16 pairs)      [192,256) SLO : S lo
//   [256,384) ZQ  : [Z | Y] of S hi x [K+;Q+] hi, then [Z | Y] of S hi x lo    (32 cols each)
//   [384,448) P   : [K';Q'] x [K'' hi | K'' lo]   (lanes 0..63 used)
//   [448,512) DO  : [Dl | Dl'] of X x [T hi | T lo], then [O | O'] of Dl x [Mq hi | Mq lo]
// Once a thread has read its Z columns, the same 16 columns take its tokens'
// X^T as a bf16 hi/lo pair (8 + 8 columns: the A operand of Dl = X T^T, read
// from tensor memory), and once Dl is in, its tokens' Dl^T likewise (the A
// operand of the state update and of the output product).  An MMA reads A from
// tensor memory at about a third of the issue cost of a shared-memory A.
#include "gdn_internal.h"
#include "sm100.cuh"

namespace gdn {
namespace {

using namespace sm100;

constexpr int D = 128;
constexpr int NT = 32;  // tokens per tile (= chunk)
constexpr int NTHREADS = 512;
constexpr int CHAIN_THREADS = 256, SIDE_THREADS = 256;
constexpr int BAR_CHAIN = 1, BAR_SIDE = 2;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t TM_S = 0, TM_SHI = 128, TM_SLO = 192, TM_ZQ = 256, TM_P = 384, TM_DO = 448;
// X^T, then Dl^T, as hi/lo pairs in the Z columns: chain thread half ch (tokens
// 16 ch .. 16 ch + 15) at TM_X + 16 ch (hi) and TM_X + 16 ch + 8 (lo)
constexpr uint32_t TM_X = TM_ZQ;
// The output product is issued by a second chain thread (warp 12), in parallel
// with the state update from the chain leader.
constexpr int OI_ISSUER = 384;

// Shared memory (offsets from a 1024-byte aligned base).  K-major SW128 tiles
// have 128-byte rows (64 bf16 along K) in 8-row groups 1024 B apart.
constexpr uint32_t SM_KQ = 0;          // raw [K dk0-63 | Q dk0-63 | K dk64-127 | Q dk64-127], 4 KB boxes
constexpr uint32_t SM_V = 16384;       // raw V [32 tokens][DVB] bf16 (the CTA's rows)
// The chain's operand tiles (ZQB: [K+;Q+], KT: K~) are double-buffered (tile c
// in buffer c & 1), so the side writes them as soon as it derives them; the
// solve's scratch (A, T, the exchange area) lives in the P operand region,
// which is dead from P's completion to the next tile's operands.
constexpr uint32_t SM_ZQB0 = 24576;    // [K+ hi; Q+ hi; K+ lo; Q+ lo] 128 rows, boxes dk0-63 / dk64-127 16 KB apart
constexpr uint32_t SM_PA = 57344;      // [K' hi; Q' hi; K' lo; Q' lo] 128 rows, boxes 16 KB apart
constexpr uint32_t SM_PB = 90112;      // [K'' hi; K'' lo] 64 rows, boxes 8 KB apart
constexpr uint32_t SM_KT0 = 106496;    // K~ = K o Lambda_last / Lambda, rows j, MN-major: hi (2 x 4 KB), lo at +8 KB
constexpr uint32_t SM_XH = 122880;     // the [32][DVB] o staging tile, fp32 or bf16 (up to 16 KB)
constexpr uint32_t SM_G = 139264;      // g tile [32 tokens][128] fp32
constexpr uint32_t SM_ZQB1 = 155648;
constexpr uint32_t SM_KT1 = 188416;
constexpr uint32_t SM_TM = 204800;     // [T hi; T lo] rows i (32 + 32), K = 32 tokens
constexpr uint32_t SM_MQ = 212992;     // [Mq hi; Mq lo]
constexpr int APAD = 36;               // solve row pitch (floats)
constexpr uint32_t SM_A = SM_PA;                   // A fp32 [32][APAD]
constexpr uint32_t SM_TF = SM_A + 32 * APAD * 4;   // T fp32 [32][APAD]
constexpr uint32_t SM_X = SM_TF + 32 * APAD * 4;   // exchange: per-quarter channel sums [4][128],
                                                   // then the solve's [16][16] product
constexpr uint32_t SM_GATES = SM_MQ + 8192;
constexpr uint32_t GATE_BYTES = 640;   // beta [32], Lambda_last [128]
constexpr uint32_t G_B = 0, G_LC = 128;
constexpr int GATE_BUFS = 4;
constexpr uint32_t SM_BAR = SM_GATES + GATE_BUFS * GATE_BYTES;
constexpr uint32_t SM_MISC = SM_BAR + 256;
constexpr uint32_t SMEM_USED = SM_MISC + 256;
static_assert(SM_ZQB0 % 1024 == 0 && SM_ZQB1 % 1024 == 0 && SM_PA % 1024 == 0 && SM_PB % 1024 == 0 &&
                  SM_KT0 % 1024 == 0 && SM_KT1 % 1024 == 0 && SM_XH % 1024 == 0 && SM_TM % 1024 == 0 &&
                  SM_MQ % 1024 == 0 && SM_G % 1024 == 0,
              "SW128 tiles need 1024-byte alignment");
static_assert(SM_ZQB0 + 32768 <= SM_PA && SM_PA + 32768 <= SM_PB && SM_PB + 16384 <= SM_KT0 &&
                  SM_KT0 + 16384 <= SM_XH && SM_XH + 16384 <= SM_G && SM_G + 16384 <= SM_ZQB1 &&
                  SM_ZQB1 + 32768 <= SM_KT1 && SM_KT1 + 16384 <= SM_TM && SM_TM + 8192 <= SM_MQ,
              "operand regions");
static_assert(SM_X + 4 * 128 * 4 <= SM_PA + 32768, "solve scratch inside the P operand region");
static_assert(SMEM_USED + 1024 <= 232448, "shared memory budget");
__device__ __forceinline__ uint32_t zqb_buf(int c) { return (c & 1) ? SM_ZQB1 : SM_ZQB0; }
__device__ __forceinline__ uint32_t kt_buf(int c) { return (c & 1) ? SM_KT1 : SM_KT0; }

// mbarriers (8 bytes each, offsets inside SM_BAR)
// B_OPFULL, B_OPFREE: one per operand buffer (tile c: + 8 (c & 1), parity (c >> 1) & 1)
constexpr uint32_t B_KQFULL = 0, B_VFULL = 8, B_P = 16, B_TMFULL = 24, B_TMFREE = 32,
                   B_OPFULL = 40, B_OPFREE = 56, B_ZQ = 72, B_DL = 80, B_SU = 88, B_OI = 96,
                   B_CLEAN0 = 104, B_CLEAN1 = 112, B_CLEAN2 = 120, B_GLD = 128,
                   B_GFULL = 136;  // B_GFULL: 4 barriers
constexpr int NUM_BARS = 21;
static_assert(8 * NUM_BARS <= 256, "barrier slots");
__device__ __forceinline__ uint32_t gfull_off(int c) { return B_GFULL + 8u * uint32_t(c & 3); }
__device__ __forceinline__ uint32_t gfull_parity(int c) { return uint32_t(c >> 2) & 1u; }
constexpr uint32_t M_TMEM = 0, M_ABORT = 4, M_KQ_ISSUED = 12, M_KQ_SEEN = 16, M_V_ISSUED = 20,
                   M_V_SEEN = 24, M_FLAG_CHAIN = 32, M_FLAG_SIDE = 40, M_G_ISSUED = 48,
                   M_G_SEEN = 52;

constexpr uint32_t KQ_TX_BYTES = 4 * 4096;
constexpr uint32_t G_TX_BYTES = NT * D * 4;
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;  // 2 s: far beyond any legitimate wait
constexpr float LOG2E = 1.4426950408889634f;
constexpr float EXP2_CLAMP = 126.f;

__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }
// Two 8-column tensor-memory stores (a hi / lo pair), one wait.
__device__ __forceinline__ void tmem_st8x2(uint32_t ta, const uint32_t (&a)[8], uint32_t tb,
                                           const uint32_t (&b)[8]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%2,%3,%4,%5,%6,%7,%8,%9};\n\t"
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%1], {%10,%11,%12,%13,%14,%15,%16,%17};\n\t"
      "tcgen05.wait::st.sync.aligned;" ::"r"(ta), "r"(tb),
      "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(a[4]), "r"(a[5]), "r"(a[6]), "r"(a[7]),
      "r"(b[0]), "r"(b[1]), "r"(b[2]), "r"(b[3]), "r"(b[4]), "r"(b[5]), "r"(b[6]), "r"(b[7])
      : "memory");
}
__device__ __forceinline__ float exp2c(float x) {
  return fast_exp2(fminf(fmaxf(x, -EXP2_CLAMP), EXP2_CLAMP));
}
// 32-bit shared-memory store / load at a register address plus a constant offset.
template <uint32_t OFF>
__device__ __forceinline__ void sts32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.b32 [%0+%2], %1;" ::"r"(addr), "r"(v), "n"(OFF) : "memory");
}
template <uint32_t OFF>
__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1+%2];" : "=r"(v) : "r"(addr), "n"(OFF) : "memory");
  return v;
}

struct Ctx {
  uint8_t* sm;
  uint32_t sb;
  uint32_t tmem;
  int* status;
  volatile int* abort_flag;
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

// Role-wide agreement: the leader decides (after a bounded wait), every thread
// of the role reads the verdict after the role's named barrier.  Called from
// one site per agreement, so that the whole warp reaches the barrier together.
struct RoleSync {
  int bar_id, nthreads;
  uint32_t flag_off;
  bool leader;
  int n;
  __device__ __forceinline__ bool agree(const Ctx& x, bool leader_ok) {
    volatile int* slot = x.misc(flag_off + 4u * (n & 1));
    ++n;
    if (leader) *slot = leader_ok ? 0 : 1;
    named_bar(bar_id, nthreads);
    const bool ok = (*slot == 0);
    tc_fence_after();
    return ok;
  }
  __device__ __forceinline__ bool wait(const Ctx& x, uint32_t bar, uint32_t parity) {
    bool ok = true;
    if (leader) {
      ok = (*x.abort_flag == 0) && mbar_wait_bounded(bar, parity, WAIT_LIMIT_NS);
      if (!ok) x.fail();
    }
    return agree(x, ok);
  }
};
__device__ __forceinline__ bool lead_wait(const Ctx& x, uint32_t bar, uint32_t parity) {
  if (*x.abort_flag) return false;
  if (mbar_wait_bounded(bar, parity, WAIT_LIMIT_NS)) return true;
  x.fail();
  return false;
}

// tb: the token coordinate of tile 0 (a packed sequence's first token, else 0)
__device__ __forceinline__ void issue_kq(const Ctx& x, const CUtensorMap* tq, const CUtensorMap* tk,
                                         int c, int h, int b, int tb) {
  const uint32_t bar = x.bar(B_KQFULL);
  mbar_arrive_expect_tx(bar, KQ_TX_BYTES);
  const int t0 = tb + c * NT;
  tma_load_4d(x.sb + SM_KQ + 0, tk, bar, 0, h, t0, b);
  tma_load_4d(x.sb + SM_KQ + 4096, tq, bar, 0, h, t0, b);
  tma_load_4d(x.sb + SM_KQ + 8192, tk, bar, 64, h, t0, b);
  tma_load_4d(x.sb + SM_KQ + 12288, tq, bar, 64, h, t0, b);
  *x.misc(M_KQ_ISSUED) = c + 1;
}
// V rows dv0 .. dv0 + DVB - 1 of tile c ([32 tokens][DVB] bf16)
template <int DVB>
__device__ __forceinline__ void issue_v(const Ctx& x, const CUtensorMap* tv, int c, int h, int b, int dv0,
                                        int tb) {
  const uint32_t bar = x.bar(B_VFULL);
  mbar_arrive_expect_tx(bar, uint32_t(NT * DVB * 2));
  tma_load_4d(x.sb + SM_V, tv, bar, dv0, h, tb + c * NT, b);
  *x.misc(M_V_ISSUED) = c + 1;
}

// g of tile c ([32 tokens][128] fp32; tokens past T read as 0), issued once
// every side thread has read tile c - 1's
__device__ __forceinline__ void issue_g(const Ctx& x, const CUtensorMap* tg, int c, int h, int b, int tb) {
  const uint32_t bar = x.bar(B_GLD);
  mbar_arrive_expect_tx(bar, G_TX_BYTES);
  tma_load_4d(x.sb + SM_G, tg, bar, 0, h, tb + c * NT, b);
  *x.misc(M_G_ISSUED) = c + 1;
}

// ============================================================== side role
// Thread kt: channel pair cp = kt % 64 (channels 2cp, 2cp+1) and token quarter
// qt = kt / 64 (tokens 8qt .. 8qt+7 of the tile) for the gates and operands;
// TMEM lane quarter (warp % 4) and column half for the masks.
// PRE: q and k are L2-normalised per token and head (and q scaled) on the way
// in, before any decay is applied.  PK: a packed sequence (tokens tb .. tend - 1
// of the views): tokens of the next sequence in its last tile are made padding
// (g = beta = 0, an exact identity).
template <bool PRE, bool PK>
__device__ void side_role(const Ctx& x, const CUtensorMap* tq, const CUtensorMap* tk,
                          const CUtensorMap* tg, const KdaArgs& p, int b, int h, int ntiles, int tb,
                          int tend) {
  const int kt = threadIdx.x - 128;
  const int warp = threadIdx.x >> 5;
  const int lq = warp & 3;
  const int hf = (warp >= 8) ? 1 : 0;
  const bool leader = (kt == 0);
  const uint32_t tlane = x.tmem + (uint32_t(lq * 32) << 16);
  const uint32_t sb = x.sb;
  const int cp = kt & 63, qt = kt >> 6;
  const int d0 = 2 * cp;
  // This thread's element (row 8 qt + t, columns d0, d0 + 1) of a K-major SW128
  // tile whose 64-column boxes are `bx` bytes apart sits at tile_off(bx) +
  // row_off(t): rows 8 qt .. 8 qt + 7 form one 8-row group, so the swizzle
  // involves only t and d0's 16-byte chunk; row r + 32 m lies 4096 m bytes on.
  const uint32_t cix = uint32_t((d0 & 63) >> 3);
  const auto tile_off = [&](uint32_t bx) {
    return uint32_t(d0 >> 6) * bx + uint32_t(qt) * 1024u + uint32_t(d0 & 7) * 2u;
  };
  const auto row_off = [&](int t) { return uint32_t(t) * 128u + ((cix ^ uint32_t(t)) << 4); };
  float* sA = reinterpret_cast<float*>(x.sm + SM_A);
  float* sT = reinterpret_cast<float*>(x.sm + SM_TF);
  float* sX = reinterpret_cast<float*>(x.sm + SM_X);
  RoleSync rs{BAR_SIDE, SIDE_THREADS, M_FLAG_SIDE, leader, 0};
  // beta of token kt of the next tile, loaded one tile ahead (kt < 32)
  float beta_next = 0.f;
  if (kt < NT && tb + kt < tend) beta_next = __ldg(p.beta + (size_t(b) * p.T + tb + kt) * p.H + h);

  for (int c = 0; c < ntiles; ++c) {
    // ---- 1. gates: g of this thread's 8 tokens x 2 channels (from the tile's
    //      TMA buffer), cumulative sums (log2 units) across the tile, beta, and
    //      Lambda_last per channel
    float gm[8][2];
    {
      // tile 0's g is waited for here, every later tile's in the agreement that
      // ends the previous tile
      if (c == 0) {
        if (!rs.wait(x, x.bar(B_GLD), 0)) return;
        if (leader) *x.misc(M_G_SEEN) = 1;
      }
      const float* sg = reinterpret_cast<const float*>(x.sm + SM_G);
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        float2 g2 = *reinterpret_cast<const float2*>(sg + (8 * qt + t) * D + d0);
        if constexpr (PK) {
          if (tb + c * NT + 8 * qt + t >= tend) g2 = make_float2(0.f, 0.f);
        }
        // rounded products (never contracted into the sums below): the packed
        // instantiation, which selects g first, then rounds exactly as this one
        gm[t][0] = __fmul_rn(g2.x, LOG2E);
        gm[t][1] = __fmul_rn(g2.y, LOG2E);
      }
#pragma unroll
      for (int t = 1; t < 8; ++t) {
        gm[t][0] += gm[t - 1][0];
        gm[t][1] += gm[t - 1][1];
      }
      *reinterpret_cast<float2*>(sX + qt * 128 + d0) = make_float2(gm[7][0], gm[7][1]);
      if (kt < NT) {
        x.gates(c)[G_B / 4 + kt] = beta_next;
        const int tok = tb + (c + 1) * NT + kt;
        beta_next = tok < tend ? __ldg(p.beta + (size_t(b) * p.T + tok) * p.H + h) : 0.f;
      }
    }
    named_bar(BAR_SIDE, SIDE_THREADS);
    // every thread has read g(c): the buffer takes g(c + 1)
    if (leader && c + 1 < ntiles) issue_g(x, tg, c + 1, h, b, tb);
    float gref[2], glast[2];
    {
      float pre[2] = {0.f, 0.f}, tot[2] = {0.f, 0.f}, half[2] = {0.f, 0.f};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 s2 = *reinterpret_cast<const float2*>(sX + q * 128 + d0);
        if (q < qt) { pre[0] += s2.x; pre[1] += s2.y; }
        if (q < 2) { half[0] += s2.x; half[1] += s2.y; }
        tot[0] += s2.x;
        tot[1] += s2.y;
      }
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        gm[t][0] += pre[0];
        gm[t][1] += pre[1];
      }
      // reference: after token 15; last: after token 31
      gref[0] = half[0]; gref[1] = half[1];
      glast[0] = tot[0]; glast[1] = tot[1];
      if (qt == 0) {
        float* G = x.gates(c);
        *reinterpret_cast<float2*>(G + G_LC / 4 + d0) = make_float2(exp2c(tot[0]), exp2c(tot[1]));
      }
    }

    // ---- 2. the decayed operands of this thread's 8 tokens x 2 channels, to
    //      shared memory: the P operands, and the chain's [K+;Q+] and K~ into
    //      buffer c & 1 once the chain's state update of tile c - 2 (their last
    //      reader) has completed
    {
      bool ok = true;
      if (leader) {
        ok = lead_wait(x, x.bar(B_KQFULL), c & 1) &&
             (c < 2 || lead_wait(x, x.bar(B_OPFREE + 8u * uint32_t(c & 1)), ((c - 2) >> 1) & 1));
        if (ok) *x.misc(M_KQ_SEEN) = c + 1;
      }
      // (this agreement also closes the gates: every thread has written its
      // gate entries and read the exchange area, which the operands overwrite)
      if (!rs.agree(x, ok)) return;
      if (leader) mbar_arrive(x.bar(gfull_off(c)));
      // with PRE, the per-token factors |k|^-1 and q_scale |q|^-1 of this
      // thread's 8 tokens: sums of squares over the 64 threads of the token
      // quarter (two warps: a shuffle reduction each, then the exchange area)
      float kn[8], qn[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) kn[t] = qn[t] = 1.f;
      if constexpr (PRE) {
        if (p.qk_norm) {
          const int half = (kt >> 5) & 1;
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            const uint32_t ro = row_off(t);
            const uint32_t kw = lds32<0>(sb + SM_KQ + tile_off(8192u) + ro);
            const uint32_t qw = lds32<4096>(sb + SM_KQ + tile_off(8192u) + ro);
            const float2 kf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&kw));
            const float2 qf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&qw));
            float sk = fmaf(kf.x, kf.x, kf.y * kf.y), sq = fmaf(qf.x, qf.x, qf.y * qf.y);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
              sk += __shfl_xor_sync(0xffffffffu, sk, off);
              sq += __shfl_xor_sync(0xffffffffu, sq, off);
            }
            if ((kt & 31) == 0) {
              sX[(qt * 2 + half) * 16 + 2 * t] = sk;
              sX[(qt * 2 + half) * 16 + 2 * t + 1] = sq;
            }
          }
          named_bar(BAR_SIDE, SIDE_THREADS);
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            const float sk = sX[(qt * 2) * 16 + 2 * t] + sX[(qt * 2 + 1) * 16 + 2 * t];
            const float sq = sX[(qt * 2) * 16 + 2 * t + 1] + sX[(qt * 2 + 1) * 16 + 2 * t + 1];
            kn[t] = rsqrtf(sk + 1e-6f);
            qn[t] = rsqrtf(sq + 1e-6f) * p.q_scale;
          }
        } else {
#pragma unroll
          for (int t = 0; t < 8; ++t) qn[t] = p.q_scale;
        }
      }
      // per channel: Lambda_r (from the tile start) and Lambda_last / Lambda_r,
      // so that K+ = K' Lambda_r, Q+ = Q' Lambda_r and K~ = K'' Lambda_last / Lambda_r
      // take two exponentials per token and channel instead of four (products
      // capped at 2^126 like the exponents: no inf where g > 0 grows the state)
      float lr[2], llr[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        lr[e] = exp2c(gref[e]);
        llr[e] = exp2c(glast[e] - gref[e]);
      }
      constexpr float CAP = 8.5070592e37f;  // 2^126
      const uint32_t kq_t = sb + SM_KQ + tile_off(8192u);  // K rows r; Q rows r at +4096
      const uint32_t pa_t = sb + SM_PA + tile_off(16384u);  // rows r, 32 + r, 64 + r, 96 + r
      const uint32_t pb_t = sb + SM_PB + tile_off(8192u);   // rows r, 32 + r
      const uint32_t zq_t = sb + zqb_buf(c) + tile_off(16384u);  // rows r, 32 + r, 64 + r, 96 + r
      const uint32_t kt_t = sb + kt_buf(c) + tile_off(4096u);    // rows j, 64-column blocks 4 KB apart
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        const uint32_t ro = row_off(t);
        const uint32_t kw = lds32<0>(kq_t + ro), qw = lds32<4096>(kq_t + ro);
        const float2 kf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&kw));
        const float2 qf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&qw));
        const float kv[2] = {kf.x * kn[t], kf.y * kn[t]}, qv[2] = {qf.x * qn[t], qf.y * qn[t]};
        float k1[2], q1[2], k2[2], kp[2], qp[2], kt2[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const float ep = exp2c(gm[t][e] - gref[e]);   // Lambda_t / Lambda_r
          const float em = exp2c(gref[e] - gm[t][e]);   // Lambda_r / Lambda_t
          const float eplus = fminf(ep * lr[e], CAP);   // Lambda_t (from the tile start)
          const float etil = fminf(em * llr[e], CAP);   // Lambda_last / Lambda_t
          k1[e] = kv[e] * ep;
          q1[e] = qv[e] * ep;
          k2[e] = kv[e] * em;
          kp[e] = kv[e] * eplus;
          qp[e] = qv[e] * eplus;
          kt2[e] = kv[e] * etil;
        }
        uint32_t hi, lo;
        split2_bf16(k1[0], k1[1], hi, lo);  // K' hi row r, lo row 64 + r
        sts32<0>(pa_t + ro, hi);
        sts32<8192>(pa_t + ro, lo);
        split2_bf16(q1[0], q1[1], hi, lo);  // Q' hi row 32 + r, lo row 96 + r
        sts32<4096>(pa_t + ro, hi);
        sts32<12288>(pa_t + ro, lo);
        split2_bf16(k2[0], k2[1], hi, lo);  // K'' hi row r, lo row 32 + r
        sts32<0>(pb_t + ro, hi);
        sts32<4096>(pb_t + ro, lo);
        split2_bf16(kp[0], kp[1], hi, lo);  // K+ hi row r, lo row 64 + r
        sts32<0>(zq_t + ro, hi);
        sts32<8192>(zq_t + ro, lo);
        split2_bf16(qp[0], qp[1], hi, lo);  // Q+ hi row 32 + r, lo row 96 + r
        sts32<4096>(zq_t + ro, hi);
        sts32<12288>(zq_t + ro, lo);
        split2_bf16(kt2[0], kt2[1], hi, lo);  // K~ rows j: hi, lo 8 KB on
        sts32<0>(kt_t + ro, hi);
        sts32<8192>(kt_t + ro, lo);
      }
    }
    fence_proxy_async_smem();
    named_bar(BAR_SIDE, SIDE_THREADS);  // the raw tile is read; every operand is in place
    if (leader) mbar_arrive(x.bar(B_OPFULL + 8u * uint32_t(c & 1)));
    // ---- 3. P = [K' hi; Q' hi; K' lo; Q' lo] [K'' hi | K'' lo]^T  (M=128, N=64):
    //      lanes 0..63 hold hi x hi | hi x lo, lanes 64..127 lo x hi | (unused lo x lo)
    {
      bool ok = true;
      if (leader) {
        if (c + 1 < ntiles) issue_kq(x, tq, tk, c + 1, h, b, tb);
        tc_fence_after();
        const uint32_t id64 = idesc_bf16(128, 64, 0, 0, 0);
        const uint64_t da = sdesc_sw128(sb + SM_PA, 16, 1024), db = sdesc_sw128(sb + SM_PB, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(x.tmem + TM_P, sdesc_add(da, (kk >> 2) * 16384 + (kk & 3) * 32),
                 sdesc_add(db, (kk >> 2) * 8192 + (kk & 3) * 32), id64, kk > 0);
        mma_commit(x.bar(B_P));
        ok = lead_wait(x, x.bar(B_P), c & 1);
      }
      if (!rs.agree(x, ok)) return;
    }
    // ---- 4. masks: rows 0..31 (K') -> A = strict_tril(beta_i P_ij) (fp32, for the
    //      solve); rows 32..63 (Q') -> Mq = tril(P_ij) (registers).  The lo x hi
    //      terms of row i sit in lane 64 + i (K') or 96 + i (Q'): those warps pass
    //      them through shared memory (the A and T scratch, rewritten only after)
    float mq[16];
    {
      const float* G = x.gates(c);
      const int i = threadIdx.x & 31;
      float* xch = (lq & 1) ? sT : sA;
      if (lq >= 2) {
        float pl[16];
        tmem_ld16(tlane + TM_P + 16 * hf, pl);
#pragma unroll
        for (int e4 = 0; e4 < 4; ++e4)
          *reinterpret_cast<float4*>(xch + i * APAD + 16 * hf + 4 * e4) =
              make_float4(pl[4 * e4], pl[4 * e4 + 1], pl[4 * e4 + 2], pl[4 * e4 + 3]);
      }
      named_bar(BAR_SIDE, SIDE_THREADS);
      if (lq < 2) {
        float pa[16], pb[16];
        tmem_ld16x2(tlane + TM_P + 16 * hf, pa, tlane + TM_P + 32 + 16 * hf, pb);
        const float bi = (lq == 0) ? G[G_B / 4 + i] : 1.f;
#pragma unroll
        for (int e4 = 0; e4 < 4; ++e4) {
          const float4 l = ld4(xch + i * APAD + 16 * hf + 4 * e4);
          const float lv[4] = {l.x, l.y, l.z, l.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int j = 16 * hf + 4 * e4 + e;
            const float v = bi * ((pa[4 * e4 + e] + lv[e]) + pb[4 * e4 + e]);
            mq[4 * e4 + e] = (lq == 0 ? j < i : j <= i) ? v : 0.f;
          }
        }
        if (lq == 0) {
#pragma unroll
          for (int e4 = 0; e4 < 4; ++e4)
            *reinterpret_cast<float4*>(sA + i * APAD + 16 * hf + 4 * e4) =
                make_float4(mq[4 * e4], mq[4 * e4 + 1], mq[4 * e4 + 2], mq[4 * e4 + 3]);
        }
      }
    }
    tc_fence_before();
    named_bar(BAR_SIDE, SIDE_THREADS);
    // ---- 5. T = (I + A)^{-1}: 16 x 16 diagonal blocks by substitution, then
    //      T_10 = -T_11 (A_10 T_00)
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
#pragma unroll
      for (int q4 = 0; q4 < 8; ++q4) {
        float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
        if ((q4 >> 2) == bb)
          v = make_float4(acc[4 * (q4 & 3)], acc[4 * (q4 & 3) + 1], acc[4 * (q4 & 3) + 2],
                          acc[4 * (q4 & 3) + 3]);
        *reinterpret_cast<float4*>(sT + r * APAD + 4 * q4) = v;
      }
    }
    named_bar(BAR_SIDE, SIDE_THREADS);
    {
      const int r = kt >> 4, cc = kt & 15;  // X[r][cc] = sum_k A[16 + r][k] T[k][cc]
      float a0 = 0.f, a1 = 0.f;
#pragma unroll
      for (int k = 0; k < 16; k += 2) {
        a0 = fmaf(sA[(16 + r) * APAD + k], sT[k * APAD + cc], a0);
        a1 = fmaf(sA[(16 + r) * APAD + k + 1], sT[(k + 1) * APAD + cc], a1);
      }
      sX[r * 16 + cc] = a0 + a1;
    }
    named_bar(BAR_SIDE, SIDE_THREADS);
    {
      const int r = kt >> 4, cc = kt & 15;  // T[16 + r][cc] = -sum_k T[16 + r][16 + k] X[k][cc]
      float a0 = 0.f, a1 = 0.f;
#pragma unroll
      for (int k = 0; k < 16; k += 2) {
        a0 = fmaf(sT[(16 + r) * APAD + 16 + k], sX[k * 16 + cc], a0);
        a1 = fmaf(sT[(16 + r) * APAD + 17 + k], sX[(k + 1) * 16 + cc], a1);
      }
      sT[(16 + r) * APAD + cc] = -(a0 + a1);
    }
    // ---- 6. hand T and Mq to the chain once T is complete and the chain is done
    //      with the previous tile's (its output product, the last reader, has
    //      completed): one agreement
    {
      bool ok = true;
      if (leader && c > 0) ok = lead_wait(x, x.bar(B_TMFREE), (c - 1) & 1);
      if (!rs.agree(x, ok)) return;
    }
    if (kt < 4 * NT) {  // T: row i = kt / 4, 8 columns each
      const int i = kt >> 2, cc = kt & 3;
      store_split8(sb + SM_TM, sb + SM_TM + 4096, i, cc, sT + i * APAD + 8 * cc);
    }
    if (lq == 1) {  // Mq row threadIdx % 32, columns 16 hf ..
      const int i = threadIdx.x & 31;
#pragma unroll
      for (int e = 0; e < 2; ++e) store_split8(sb + SM_MQ, sb + SM_MQ + 4096, i, 2 * hf + e, mq + 8 * e);
    }
    fence_proxy_async_smem();
    {
      // T and Mq are in place, and the next tile's g has landed: one agreement
      bool ok = true;
      if (leader && c + 1 < ntiles) {
        ok = lead_wait(x, x.bar(B_GLD), (c + 1) & 1);
        if (ok) *x.misc(M_G_SEEN) = c + 2;
      }
      if (!rs.agree(x, ok)) return;
    }
    if (leader) mbar_arrive(x.bar(B_TMFULL));
  }
}

// ============================================================== chain role
// DVB: rows of the state this CTA owns (64 or 128); DV2: two CTAs per chain
// (Dv = 256), this one owning rows dv0 = 128 (blockIdx & 1) ..; OBF: o is
// bf16 (the fp32 value rounded to nearest even, through a bf16 TMA view)
// snap (PK only; null: none): this CTA's first snapshot row, slot j (j = 1, 2, ..)
// taking the state after j * stiles tiles
template <int DVB, bool DV2, bool OBF, bool PK>
__device__ void chain_role(const Ctx& x, const CUtensorMap* tv, const CUtensorMap* tmo,
                           const KdaArgs& p, int chain, int b, int h, int ntiles, int tb, int tend,
                           float* snap, int stiles) {
  constexpr int DVW = DV2 ? 2 * D : DVB;  // Dv: rows of the chain's state
  const int dv0 = DV2 ? D * (int(blockIdx.x) & 1) : 0;
  const int warp = threadIdx.x >> 5;
  const int lq = warp & 3;
  const int ch = (warp >= 12) ? 1 : 0;  // column half
  const int dv = lq * 32 + (threadIdx.x & 31);
  const bool leader = (threadIdx.x == 0);
  const uint32_t tlane = x.tmem + (uint32_t(lq * 32) << 16);
  const uint32_t sb = x.sb;
  RoleSync rs{BAR_CHAIN, CHAIN_THREADS, M_FLAG_CHAIN, leader, 0};
  const size_t cstate = size_t(chain) * DVW * D + size_t(dv0) * D;  // this CTA's first row
  const bool own = DVB == D || dv < DVB;  // the lane holds one of the CTA's rows

  // ---- initial state (row dv of S0, or zeros): hi/lo copy, and the fp32 copy
  //      pre-scaled, column by column, by the decay of the first tile
  if (!rs.wait(x, x.bar(gfull_off(0)), gfull_parity(0))) return;
  {
    const float* LC = x.gates(0) + G_LC / 4;
    const float4* src =
        (p.S0 && own) ? reinterpret_cast<const float4*>(p.S0 + cstate + size_t(dv) * D) : nullptr;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int col = 64 * ch + 32 * q;
      float v[32];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float4 a = src ? __ldg(src + col / 4 + e) : make_float4(0.f, 0.f, 0.f, 0.f);
        v[4 * e] = a.x; v[4 * e + 1] = a.y; v[4 * e + 2] = a.z; v[4 * e + 3] = a.w;
      }
      uint32_t hi[16], lo[16], u[32];
#pragma unroll
      for (int e = 0; e < 16; ++e) split2_bf16(v[2 * e], v[2 * e + 1], hi[e], lo[e]);
#pragma unroll
      for (int e = 0; e < 32; ++e) u[e] = __float_as_uint(LC[col + e] * v[e]);
      tmem_st_state(tlane + TM_SHI + col / 2, hi, tlane + TM_SLO + col / 2, lo, tlane + TM_S + col, u);
    }
  }
  tc_fence_before();
  named_bar(BAR_CHAIN, CHAIN_THREADS);

  for (int c = 0; c < ntiles; ++c) {
    const float* G = x.gates(c);
    const bool last = (c + 1 == ntiles);
    const int n0 = 16 * ch;  // this thread's tokens of the tile
    // ---- [Z|Y] = S_c [K+;Q+]^T: S hi x [hi rows; lo rows] (N=128), S lo x hi rows (N=64)
    if (leader) {
      if (lead_wait(x, x.bar(B_OPFULL + 8u * uint32_t(c & 1)), (c >> 1) & 1)) {
        tc_fence_after();
        const uint64_t db = sdesc_sw128(sb + zqb_buf(c), 16, 1024);
        const uint32_t id128 = idesc_bf16(128, 128, 0, 0, 0), id64 = idesc_bf16(128, 64, 0, 0, 0);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(x.tmem + TM_ZQ, x.tmem + TM_SHI + kk * 8,
                 sdesc_add(db, (kk >> 2) * 16384 + (kk & 3) * 32), id128, kk > 0);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(x.tmem + TM_ZQ, x.tmem + TM_SLO + kk * 8,
                 sdesc_add(db, (kk >> 2) * 16384 + (kk & 3) * 32), id64, 1u);
        mma_commit(x.bar(B_ZQ));
      }
    }
    // ---- X^T[dv][n] = beta_n (V[n][dv] - Z[dv][n]) (hi/lo -> this thread's Z columns)
    {
      bool ok = true;
      if (leader) {
        bulk_wait_read0();  // the previous tile's o store has read the staging tile
        ok = lead_wait(x, x.bar(B_ZQ), c & 1) && lead_wait(x, x.bar(gfull_off(c)), gfull_parity(c)) &&
             lead_wait(x, x.bar(B_VFULL), c & 1);
        if (ok) *x.misc(M_V_SEEN) = c + 1;
      }
      if (!rs.agree(x, ok)) return;
    }
    {
      float za[16], zb[16];
      tmem_ld16x2(tlane + TM_ZQ + n0, za, tlane + TM_ZQ + 64 + n0, zb);
      const __nv_bfloat16* V = reinterpret_cast<const __nv_bfloat16*>(x.sm + SM_V);
      float xv[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int n = n0 + e;
        const float vn = own ? __bfloat162float(V[n * DVB + dv]) : 0.f;
        xv[e] = G[G_B / 4 + n] * (vn - (za[e] + zb[e]));
      }
      uint32_t xh[8], xl[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) split2_bf16(xv[2 * e], xv[2 * e + 1], xh[e], xl[e]);
      tmem_st8x2(tlane + TM_X + 16 * ch, xh, tlane + TM_X + 16 * ch + 8, xl);
    }
    tc_fence_before();
    named_bar(BAR_CHAIN, CHAIN_THREADS);
    // ---- Dl^T = X^T T^T: X hi x [T hi; T lo] (N=64), X lo x T hi (N=32); K = 32,
    //      A from tensor memory (K step ks = the tokens of chain half ks)
    if (leader) {
      if (!last) issue_v<DVB>(x, tv, c + 1, h, b, dv0, tb);  // V(c) has been read
      if (lead_wait(x, x.bar(B_TMFULL), c & 1)) {
        tc_fence_after();
        const uint32_t id64 = idesc_bf16(128, 64, 0, 0, 0), id32 = idesc_bf16(128, 32, 0, 0, 0);
        const uint64_t dt = sdesc_sw128(sb + SM_TM, 16, 1024);
#pragma unroll
        for (int ks = 0; ks < 2; ++ks)
          mma_ts(x.tmem + TM_DO, x.tmem + TM_X + 16 * ks, sdesc_add(dt, 32 * ks), id64, ks > 0);
#pragma unroll
        for (int ks = 0; ks < 2; ++ks)
          mma_ts(x.tmem + TM_DO, x.tmem + TM_X + 16 * ks + 8, sdesc_add(dt, 32 * ks), id32, 1u);
        mma_commit(x.bar(B_DL));
      }
    }
    if (!rs.wait(x, x.bar(B_DL), c & 1)) return;
    {
      float da[16], db2[16];
      tmem_ld16x2(tlane + TM_DO + n0, da, tlane + TM_DO + 32 + n0, db2);
#pragma unroll
      for (int e = 0; e < 16; ++e) da[e] += db2[e];
      // X^T has been consumed (Dl is complete): Dl^T takes its columns
      uint32_t dh[8], dl[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) split2_bf16(da[2 * e], da[2 * e + 1], dh[e], dl[e]);
      tmem_st8x2(tlane + TM_X + 16 * ch, dh, tlane + TM_X + 16 * ch + 8, dl);
    }
    tc_fence_before();
    named_bar(BAR_CHAIN, CHAIN_THREADS);
    // ---- S += Dl^T K~ (3 hi/lo products, N=128, B MN-major; the chain leader)
    //      and O_intra = Dl^T Mq^T: Dl hi x [Mq hi; Mq lo] (N=64), Dl lo x Mq hi
    //      (N=32; a second issuer), A from tensor memory, committed separately
    if (leader && !*x.abort_flag) {
      tc_fence_after();
      const uint32_t idu = idesc_bf16(128, 128, 0, 1, 0);
#pragma unroll
      for (int part = 0; part < 3; ++part) {
        const uint32_t a = x.tmem + TM_X + (part == 2 ? 8 : 0);
        const uint32_t kb = kt_buf(c) + (part == 1 ? 8192u : 0u);
#pragma unroll
        for (int ks = 0; ks < 2; ++ks)
          mma_ts(x.tmem + TM_S, a + 16 * ks, sdesc_sw128(sb + kb + 2048 * ks, 4096, 1024), idu, 1u);
      }
      mma_commit(x.bar(B_SU));
      mma_commit(x.bar(B_OPFREE + 8u * uint32_t(c & 1)));  // [K+;Q+] (read by [Z|Y]) and K~ consumed
    }
    if (threadIdx.x == OI_ISSUER && !*x.abort_flag) {
      tc_fence_after();
      const uint32_t id64 = idesc_bf16(128, 64, 0, 0, 0), id32 = idesc_bf16(128, 32, 0, 0, 0);
      const uint64_t dm = sdesc_sw128(sb + SM_MQ, 16, 1024);
#pragma unroll
      for (int ks = 0; ks < 2; ++ks)
        mma_ts(x.tmem + TM_DO, x.tmem + TM_X + 16 * ks, sdesc_add(dm, 32 * ks), id64, ks > 0);
#pragma unroll
      for (int ks = 0; ks < 2; ++ks)
        mma_ts(x.tmem + TM_DO, x.tmem + TM_X + 16 * ks + 8, sdesc_add(dm, 32 * ks), id32, 1u);
      mma_commit(x.bar(B_OI));
      mma_commit(x.bar(B_TMFREE));  // T and Mq consumed (T by Dl, which has completed)
    }
    // ---- o[t][dv] = Y[dv][t] + O_intra[dv][t] (both halves), staged fp32 in
    //      shared memory (the previous tile's store has read it: the leader
    //      waited before this tile's X agreement), one TMA store
    if (!rs.wait(x, x.bar(B_OI), c & 1)) return;
    {
      float ya[16], yb[16], oa[16], ob[16];
      tmem_ld16x2(tlane + TM_ZQ + 32 + n0, ya, tlane + TM_ZQ + 96 + n0, yb);
      tmem_ld16x2(tlane + TM_DO + n0, oa, tlane + TM_DO + 32 + n0, ob);
      if (own) {
        if constexpr (OBF) {
          __nv_bfloat16* so = reinterpret_cast<__nv_bfloat16*>(x.sm + SM_XH) + dv;
#pragma unroll
          for (int e = 0; e < 16; ++e)
            so[(n0 + e) * DVB] = __float2bfloat16_rn((ya[e] + yb[e]) + (oa[e] + ob[e]));
        } else {
          float* so = reinterpret_cast<float*>(x.sm + SM_XH) + dv;
#pragma unroll
          for (int e = 0; e < 16; ++e) so[(n0 + e) * DVB] = (ya[e] + yb[e]) + (oa[e] + ob[e]);
        }
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    named_bar(BAR_CHAIN, CHAIN_THREADS);
    if (!PK || tb + (c + 1) * NT <= tend || tend == p.T) {
      // a whole tile, or the view's own end clips it
      if (leader) {
        tma_store_4d(tmo, sb + SM_XH, dv0, h, tb + c * NT, b);
        bulk_commit();
      }
    } else if constexpr (PK && !OBF) {
      // the last tile of a packed sequence: the rows past it are the next
      // sequence's, so only the valid rows are copied out, 16 bytes at a time
      const int nvalid = tend - (tb + c * NT);
      const float4* src = reinterpret_cast<const float4*>(x.sm + SM_XH);
      float* dst = p.o + (size_t(tb + c * NT) * p.H + h) * DVW + dv0;
      const int ct = (warp >= 12 ? 128 : 0) + lq * 32 + (threadIdx.x & 31);  // 0 .. 255
      for (int i = ct; i < nvalid * (DVB / 4); i += CHAIN_THREADS) {
        const int r = i / (DVB / 4), j = i % (DVB / 4);
        reinterpret_cast<float4*>(dst + size_t(r) * p.H * DVW)[j] = src[i];
      }
    } else if constexpr (PK && OBF) {
      // the same for bf16 o (rows of DVB bf16: DVB / 8 chunks of 16 bytes)
      const int nvalid = tend - (tb + c * NT);
      const uint4* src = reinterpret_cast<const uint4*>(x.sm + SM_XH);
      __nv_bfloat16* dst =
          reinterpret_cast<__nv_bfloat16*>(p.o) + (size_t(tb + c * NT) * p.H + h) * DVW + dv0;
      const int ct = (warp >= 12 ? 128 : 0) + lq * 32 + (threadIdx.x & 31);
      for (int i = ct; i < nvalid * (DVB / 8); i += CHAIN_THREADS) {
        const int r = i / (DVB / 8), j = i % (DVB / 8);
        reinterpret_cast<uint4*>(dst + size_t(r) * p.H * DVW)[j] = src[i];
      }
    }
    // ---- state epilogue: the update has completed (its commit preceded the
    //      output product's); refresh hi/lo and pre-scale by the next tile's
    //      decay per column, or store S_T
    if (!rs.wait(x, x.bar(B_SU), c & 1)) return;
    // the state after this tile goes to a snapshot slot every stiles tiles (a
    // last tile that the sequence ends inside is no boundary)
    float* snap_row = nullptr;
    if constexpr (PK) {
      if (snap && own && (c + 1) % stiles == 0 && (c + 1) * NT <= tend - tb)
        snap_row = snap + (size_t((c + 1) / stiles - 1) * p.H * DVW + dv) * D;
    }
    if (!last) {
      if (!rs.wait(x, x.bar(gfull_off(c + 1)), gfull_parity(c + 1))) return;
      const float* LC = x.gates(c + 1) + G_LC / 4;
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int col = 64 * ch + 32 * q;
        float v[32];
        tmem_ld32(tlane + TM_S + col, v);
        if constexpr (PK) {
          if (snap_row) {
            float4* sd = reinterpret_cast<float4*>(snap_row + col);
#pragma unroll
            for (int e = 0; e < 8; ++e) sd[e] = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
          }
        }
        uint32_t hi[16], lo[16], u[32];
#pragma unroll
        for (int e = 0; e < 16; ++e) split2_bf16(v[2 * e], v[2 * e + 1], hi[e], lo[e]);
#pragma unroll
        for (int e4 = 0; e4 < 8; ++e4) {
          const float4 l = ld4(LC + col + 4 * e4);
          u[4 * e4 + 0] = __float_as_uint(l.x * v[4 * e4 + 0]);
          u[4 * e4 + 1] = __float_as_uint(l.y * v[4 * e4 + 1]);
          u[4 * e4 + 2] = __float_as_uint(l.z * v[4 * e4 + 2]);
          u[4 * e4 + 3] = __float_as_uint(l.w * v[4 * e4 + 3]);
        }
        tmem_st_state(tlane + TM_SHI + col / 2, hi, tlane + TM_SLO + col / 2, lo, tlane + TM_S + col, u);
      }
      tc_fence_before();
      named_bar(BAR_CHAIN, CHAIN_THREADS);
    } else {
      float4* dst = reinterpret_cast<float4*>(p.S_T + cstate + size_t(dv) * D + 64 * ch);
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        float v[32];
        tmem_ld32(tlane + TM_S + 64 * ch + 32 * q, v);
        if (!own) continue;
#pragma unroll
        for (int e = 0; e < 8; ++e) dst[8 * q + e] = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
        if constexpr (PK) {
          if (snap_row) {  // the sequence ends on a snapshot boundary: that slot is S_T
            float4* sd = reinterpret_cast<float4*>(snap_row + 64 * ch + 32 * q);
#pragma unroll
            for (int e = 0; e < 8; ++e) sd[e] = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
          }
        }
      }
    }
  }
}

template <bool PRE, int DVB, bool DV2, bool OBF = false, bool PK = false>
__global__ void __launch_bounds__(NTHREADS, 1)
    kda_prefill_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                       const __grid_constant__ CUtensorMap tm_g, const KdaArgs p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  int chain = DV2 ? int(blockIdx.x) >> 1 : int(blockIdx.x);
  int b = chain / p.H;
  const int h = chain - (chain / p.H) * p.H;
  int ntiles = (p.T + NT - 1) / NT;
  int tb = 0, tend = p.T;  // this chain's tokens in the views
  float* snap = nullptr;   // this CTA's first snapshot row (packed sequences)
  int stiles = 1;
  if constexpr (PK) {
    // longest sequences first: CTAs start in index order, so slot r of the
    // grid takes the sequence of rank r by (length descending, index), a
    // bijection whatever the offsets hold; the shorter chains then fill the
    // SMs the long ones leave.  Up to one sequence per thread (else index order).
    if (p.B <= NTHREADS) {
      int* lens = reinterpret_cast<int*>(sm + SM_G);  // scratch: g(0) is not issued yet
      for (int i = tid; i < p.B; i += NTHREADS)
        lens[i] = __ldg(p.cu_seqlens + i + 1) - __ldg(p.cu_seqlens + i);
      __syncthreads();
      if (tid < p.B) {
        const int L = lens[tid];
        int rank = 0;
        for (int m = 0; m < p.B; ++m) {
          const int Lm = lens[m];
          rank += (Lm > L || (Lm == L && m < tid)) ? 1 : 0;
        }
        if (rank == b) lens[NTHREADS] = tid;
      }
      __syncthreads();
      b = lens[NTHREADS];
      chain = b * p.H + h;
    }
    // packed sequences: chain n H + h walks tokens [cu[n], cu[n+1]) of views with B = 1
    tb = __ldg(p.cu_seqlens + b);
    tend = __ldg(p.cu_seqlens + b + 1);
    if (tb < 0 || tend < tb || tend > p.T) {
      if (tid == 0 && p.status) atomicExch(p.status, GDN_ERR_SHAPE);
      return;
    }
    b = 0;
    ntiles = (tend - tb + NT - 1) / NT;
    if (p.snaps) {
      // first snapshot slot of this sequence: one per snap_every tokens of every
      // earlier sequence; an invalid earlier entry (its own CTAs report it)
      // leaves this sequence without snapshots
      int base = 0;
      bool offsets_ok = true;
      for (int m = 0; m < chain / p.H; ++m) {
        const int s0 = __ldg(p.cu_seqlens + m), s1 = __ldg(p.cu_seqlens + m + 1);
        if (s0 < 0 || s1 < s0 || s1 > p.T) {
          offsets_ok = false;
          break;
        }
        base += (s1 - s0) / p.snap_every;
      }
      if (!offsets_ok || base + (tend - tb) / p.snap_every > p.n_snaps) {
        if (tid == 0 && p.status) atomicExch(p.status, GDN_ERR_SHAPE);
      } else {
        snap = p.snaps + (size_t(base) * p.H + h) * (DV2 ? 2 * D : DVB) * D +
               size_t(DV2 ? D * (int(blockIdx.x) & 1) : 0) * D;
        stiles = p.snap_every / NT;
      }
    }
    if (ntiles == 0) {  // an empty sequence: S_T = S0 (or zeros), this CTA's rows
      const int rows = DVB;
      const size_t off = size_t(chain) * (DV2 ? 2 * D : DVB) * D +
                         size_t(DV2 ? D * (int(blockIdx.x) & 1) : 0) * D;
      const float4* src = p.S0 ? reinterpret_cast<const float4*>(p.S0 + off) : nullptr;
      float4* dst = reinterpret_cast<float4*>(p.S_T + off);
      for (int i = tid; i < rows * D / 4; i += NTHREADS)
        dst[i] = src ? src[i] : make_float4(0.f, 0.f, 0.f, 0.f);
      return;
    }
  }

  Ctx x;
  x.sm = sm;
  x.sb = smem_u32(sm);
  x.status = p.status;
  x.abort_flag = reinterpret_cast<volatile int*>(sm + SM_MISC + M_ABORT);
  if (tid == 0) {
    prefetch_tmap(&tm_q);
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_v);
    prefetch_tmap(&tm_o);
    prefetch_tmap(&tm_g);
    for (int i = 0; i < NUM_BARS; ++i) mbar_init(x.sb + SM_BAR + 8 * i, 1);
    fence_mbar_init();
    for (int i = 0; i < 16; ++i) reinterpret_cast<volatile int*>(sm + SM_MISC)[i] = 0;
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(sm + SM_MISC + M_TMEM), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  x.tmem = *reinterpret_cast<volatile uint32_t*>(sm + SM_MISC + M_TMEM);
  if (tid == 0) {
    issue_kq(x, &tm_q, &tm_k, 0, h, b, tb);
    issue_v<DVB>(x, &tm_v, 0, h, b, DV2 ? D * (int(blockIdx.x) & 1) : 0, tb);
    issue_g(x, &tm_g, 0, h, b, tb);
  }
  if (warp < 4 || warp >= 12)
    chain_role<DVB, DV2, OBF, PK>(x, &tm_v, &tm_o, p, chain, b, h, ntiles, tb, tend, snap, stiles);
  else
    side_role<PRE, PK>(x, &tm_q, &tm_k, &tm_g, p, b, h, ntiles, tb, tend);

  // each MMA-issuing thread waits (bounded) for its own products in flight
  if (tid == 0 || tid == 128 || tid == OI_ISSUER) {
    const uint32_t bc = x.bar(tid == 0 ? B_CLEAN0 : (tid == 128 ? B_CLEAN1 : B_CLEAN2));
    mma_commit(bc);
    mbar_wait_bounded(bc, 0, WAIT_LIMIT_NS / 4);
  }
  if (tid == 0) bulk_wait0();  // the o stores have completed
  tc_fence_before();
  __syncthreads();
  // An aborted CTA may still have TMA loads in flight: wait for them (bounded)
  // before the shared memory is released.
  if (tid == 0 && *x.abort_flag) {
    const int kq_issued = *x.misc(M_KQ_ISSUED), kq_seen = *x.misc(M_KQ_SEEN);
    if (kq_issued > kq_seen) mbar_wait_bounded(x.bar(B_KQFULL), (kq_issued - 1) & 1, WAIT_LIMIT_NS / 4);
    const int v_issued = *x.misc(M_V_ISSUED), v_seen = *x.misc(M_V_SEEN);
    if (v_issued > v_seen) mbar_wait_bounded(x.bar(B_VFULL), (v_issued - 1) & 1, WAIT_LIMIT_NS / 4);
    const int g_issued = *x.misc(M_G_ISSUED), g_seen = *x.misc(M_G_SEEN);
    if (g_issued > g_seen) mbar_wait_bounded(x.bar(B_GLD), (g_issued - 1) & 1, WAIT_LIMIT_NS / 4);
  }
  __syncthreads();
  tc_fence_after();
  if (warp == 0) tmem_dealloc(x.tmem, TMEM_COLS);
}

}  // namespace

int launch_kda_prefill(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& to, const CUtensorMap& tg, const KdaArgs& a,
                       cudaStream_t stream) {
  const int chains = a.B * a.H;
  if (chains == 0 || (a.T == 0 && !a.cu_seqlens)) return -1;
  const uint32_t smem = SMEM_USED + 1024;
  const bool pre = a.qk_norm || a.q_scale != 1.f;
  auto go = [&](auto kernel, int slot, int ctas) {
    if (!ensure_smem_attr(reinterpret_cast<const void*>(kernel), slot, int(smem))) return false;
    kernel<<<ctas, NTHREADS, smem, stream>>>(tq, tk, tv, to, tg, a);
    return true;
  };
  bool ok;
  if (a.cu_seqlens && a.o_bf16) {  // packed sequences, bf16 o (pre-step instantiations)
    if (a.Dv == D)
      ok = go(kda_prefill_kernel<true, 128, false, true, true>, 86, chains);
    else if (a.Dv == 2 * D)
      ok = go(kda_prefill_kernel<true, 128, true, true, true>, 87, 2 * chains);
    else if (a.Dv == 64)
      ok = go(kda_prefill_kernel<true, 64, false, true, true>, 88, chains);
    else
      return -1;
  } else if (a.cu_seqlens) {  // packed sequences (fp32 o; the pre-steps on request)
    if (a.Dv == D)
      ok = pre ? go(kda_prefill_kernel<true, 128, false, false, true>, 75, chains)
               : go(kda_prefill_kernel<false, 128, false, false, true>, 64, chains);
    else if (a.Dv == 2 * D)
      ok = pre ? go(kda_prefill_kernel<true, 128, true, false, true>, 76, 2 * chains)
               : go(kda_prefill_kernel<false, 128, true, false, true>, 65, 2 * chains);
    else if (a.Dv == 64)
      ok = pre ? go(kda_prefill_kernel<true, 64, false, false, true>, 77, chains)
               : go(kda_prefill_kernel<false, 64, false, false, true>, 66, chains);
    else
      return -1;
  } else if (a.o_bf16) {
    // bf16 o: the pre-step instantiations (with none requested their factors are
    // exactly 1, so o is the fp32 call's o rounded)
    if (a.Dv == D)
      ok = go(kda_prefill_kernel<true, 128, false, true>, 43, chains);
    else if (a.Dv == 2 * D)
      ok = go(kda_prefill_kernel<true, 128, true, true>, 44, 2 * chains);
    else if (a.Dv == 64)
      ok = go(kda_prefill_kernel<true, 64, false, true>, 45, chains);
    else
      return -1;
  } else if (a.Dv == D)
    ok = pre ? go(kda_prefill_kernel<true, 128, false>, 48, chains)
             : go(kda_prefill_kernel<false, 128, false>, 15, chains);
  else if (a.Dv == 2 * D)  // two CTAs per chain
    ok = pre ? go(kda_prefill_kernel<true, 128, true>, 63, 2 * chains)
             : go(kda_prefill_kernel<false, 128, true>, 40, 2 * chains);
  else if (a.Dv == 64)
    ok = pre ? go(kda_prefill_kernel<true, 64, false>, 41, chains)
             : go(kda_prefill_kernel<false, 64, false>, 42, chains);
  else
    return -1;
  if (!ok) return -1;
  return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

}  // namespace gdn
