// C-ABI entry points of libgdn_b200.so (declared in include/gdn.h): argument
// validation, TMA descriptor encoding on the host, launches on the caller's
// stream.  No device memory is allocated here.  Between calls the library
// keeps only host-side caches: the driver entry point of
// cuTensorMapEncodeTiled, per-device facts (compute capability, SM count) and
// which kernels already had their shared-memory limit raised on a device.
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cstddef>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "gdn_internal.h"

// Built-in scratch of gdn_prefill_static_ws (no allocation anywhere).
static __device__ __align__(256) unsigned char g_static_ws[GDN_STATIC_WORKSPACE_BYTES];

namespace {

constexpr int kHeadDim = 128;

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  if (!a || !b || na == 0 || nb == 0) return false;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + nb && b0 < a0 + na;
}

// Per-device facts queried once: compute capability and multiprocessor count.
constexpr int kMaxDevices = 64;
struct DeviceInfo {
  std::atomic<int> state{0};  // 0 unknown, 1 known
  int cc_major = 0, cc_minor = 0, sms = 0;
};
DeviceInfo g_devices[kMaxDevices];
std::mutex g_device_mutex;

int device_info(const DeviceInfo** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return GDN_ERR_LAUNCH;
  if (dev >= kMaxDevices) return GDN_ERR_UNSUPPORTED;
  DeviceInfo& d = g_devices[dev];
  if (d.state.load(std::memory_order_acquire) == 0) {
    std::lock_guard<std::mutex> lock(g_device_mutex);
    if (d.state.load(std::memory_order_relaxed) == 0) {
      if (cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
          cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return GDN_ERR_LAUNCH;
      d.state.store(1, std::memory_order_release);
    }
  }
  *out = &d;
  return GDN_OK;
}

// The current device must be an sm_100 part (the only architecture built).
int check_device() {
  const DeviceInfo* d = nullptr;
  const int rc = device_info(&d);
  if (rc != GDN_OK) return rc;
  if (d->cc_major != 10 || d->cc_minor != 0) return GDN_ERR_UNSUPPORTED;
  return GDN_OK;
}

// 4-D view [B][T][H][F] of an activation (bf16 input or fp32 output, F its
// feature dim); box = `box_inner` features x `box_tokens` tokens of one head.
// Loads of tokens past T read zeros; stores past T are dropped.
bool encode_act(CUtensorMap* map, const void* base, int B, int T, int H, int box_inner,
                CUtensorMapSwizzle swz, CUtensorMapDataType dtype, int esize, int F = kHeadDim,
                int box_tokens = 64) {
  auto enc = get_encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[4] = {cuuint64_t(F), cuuint64_t(H), cuuint64_t(T), cuuint64_t(B)};
  const cuuint64_t strides[3] = {cuuint64_t(F) * esize, cuuint64_t(H) * F * esize,
                                 cuuint64_t(T) * H * F * esize};
  const cuuint32_t box[4] = {cuuint32_t(box_inner), 1, cuuint32_t(box_tokens), 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(map, dtype, 4, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int num_sms(int* sms) {
  const DeviceInfo* d = nullptr;
  const int rc = device_info(&d);
  if (rc != GDN_OK) return rc;
  *sms = d->sms;
  return GDN_OK;
}

// Segmented schedule for B*H chains of T tokens on `sms` multiprocessors (one
// prefill CTA per SM).  A chain cut into n segments of L tiles costs 2n - 1 CTAs
// in the first launch, which must fit in one wave; its time is modelled, in
// units of one tile of the single-pass kernel (about 8 us), as
//     single pass:  tiles
//     n segments :  1.2 L + 0.4 (n - 1) + 0.6
// (a segment tile also pays its share of the second launch; each chained
// segment end costs one 128 x 128 x 128 product there; plus one launch), and
// the cheapest n is taken.
struct SegPlan {
  int nseg, seg_tiles;
  size_t ws_bytes, off_R, off_F;
  int fix_parts;  // CTAs per segment in the second launch (splitting its o correction)
};
SegPlan plan_segments(int B, int T, int H, int sms) {
  const long long chains = (long long)B * H;
  const int tiles = (T + 63) / 64;
  SegPlan best{1, tiles, 0, 0, 0, 1};
  if (chains <= 0 || tiles < 2 || sms <= 0) return best;
  const long long nmax = (sms / chains + 1) / 2;
  double best_cost = tiles;
  for (long long n = 2; n <= nmax && n <= tiles; ++n) {
    const int L = int((tiles + n - 1) / n);
    const int nn = (tiles + L - 1) / L;  // segments actually used
    const double cost = 1.2 * L + 0.4 * (nn - 1) + 0.6;
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best.nseg = nn;
      best.seg_tiles = L;
    }
  }
  if (best.nseg > 1) {
    // the second launch may split each segment's o correction over a few CTAs
    // as long as it stays within one wave
    const long long fix_ctas = chains * (best.nseg - 1);
    best.fix_parts = int(std::max<long long>(1, std::min<long long>(best.seg_tiles, sms / fix_ctas)));
    best.fix_parts = std::min(best.fix_parts, 4);
    const size_t f_bytes = size_t(chains) * T * kHeadDim * 4;
    const size_t mats = size_t(chains) * best.nseg * kHeadDim * kHeadDim * 4;
    best.off_R = (f_bytes + 255) & ~size_t(255);
    best.off_F = best.off_R + mats;
    best.ws_bytes = best.off_F + mats;
  }
  return best;
}

// Reads the options (NULL: defaults); false if they are invalid.
bool read_options(const gdn_options* opts, int* qk_norm, float* q_scale, int* o_bf16) {
  *qk_norm = 0;
  *q_scale = 1.f;
  *o_bf16 = 0;
  if (!opts) return true;
  // a struct from before o_bf16 existed ends at it: o stays fp32
  if (opts->size < int(offsetof(gdn_options, o_bf16))) return false;
  *qk_norm = opts->qk_l2norm ? 1 : 0;
  *q_scale = opts->q_scale;
  if (opts->size >= int(sizeof(gdn_options))) *o_bf16 = opts->o_bf16 ? 1 : 0;
  return opts->q_scale == opts->q_scale;  // not NaN
}

// The row-parallel fp32 kernel: the per-channel gate at every supported head
// dim, and the scalar gate at head dims other than 128 x 128.  g is [B][T][H][Dk]
// with vector_gate, else [B][T][H].  S_T may be S0 (in place).
int rows_impl(const void* q, const void* k, const void* v, const float* g, const float* beta,
              const float* S0, float* o, float* S_T, int B, int T, int H, int Dk, int Dv,
              bool vector_gate, void* stream) {
  if (B < 0 || T < 0 || H < 0) return GDN_ERR_SHAPE;
  if (!gdn::rows_head_dims_ok(Dk, Dv)) return GDN_ERR_UNSUPPORTED;
  const long long heads = (long long)B * H;
  if (heads * Dk * Dv > 0x7fffffffLL || heads * T * (Dk > Dv ? Dk : Dv) > 0x7fffffffLL)
    return GDN_ERR_SHAPE;
  if (heads == 0) return GDN_OK;
  if (!S_T) return GDN_ERR_NULL;
  if (T > 0 && (!q || !k || !v || !g || !beta || !o)) return GDN_ERR_NULL;
  if (!aligned(S_T, 16) || (S0 && !aligned(S0, 16))) return GDN_ERR_ALIGN;
  if (T > 0 && (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) ||
                !aligned(g, vector_gate ? 16 : 4) || !aligned(o, 4) || !aligned(beta, 4)))
    return GDN_ERR_ALIGN;
  const size_t toks = size_t(heads) * T;
  const size_t qk_bytes = toks * Dk * 2, v_bytes = toks * Dv * 2, o_bytes = toks * Dv * 4;
  const size_t g_bytes = toks * (vector_gate ? Dk : 1) * 4, beta_bytes = toks * 4;
  const size_t state_bytes = size_t(heads) * Dk * Dv * 4;
  if (S0 && S0 != S_T && overlaps(S0, state_bytes, S_T, state_bytes)) return GDN_ERR_ALIAS;
  if (T > 0) {
    const void* ins[5] = {q, k, v, g, beta};
    const size_t in_bytes[5] = {qk_bytes, qk_bytes, v_bytes, g_bytes, beta_bytes};
    for (int i = 0; i < 5; ++i)
      if (overlaps(o, o_bytes, ins[i], in_bytes[i]) || overlaps(S_T, state_bytes, ins[i], in_bytes[i]))
        return GDN_ERR_ALIAS;
    if (overlaps(o, o_bytes, S_T, state_bytes) || overlaps(o, o_bytes, S0, state_bytes))
      return GDN_ERR_ALIAS;
  } else if (S0 == S_T) {
    return GDN_OK;
  }
  const int dev_ok = check_device();
  if (dev_ok != GDN_OK) return dev_ok;
  int sms = 0;
  const int rc = num_sms(&sms);
  if (rc != GDN_OK) return rc;
  gdn::RowArgs a{static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
                 static_cast<const __nv_bfloat16*>(v), g, beta, S0, S_T, o, B, H, T, Dv};
  return gdn::launch_rows(a, Dk, vector_gate, sms, static_cast<cudaStream_t>(stream)) == 0
             ? GDN_OK
             : GDN_ERR_LAUNCH;
}

// The streaming decode kernel (Dk = Dv = DH, 128 or 64), the state updated in
// place.  vector_gate: g is [B][T][H][DH], else [B][T][H].  o_align: the
// alignment the entry point documents for o.
int decode_impl(const void* q, const void* k, const void* v, const float* g, const float* beta,
                float* S, float* o, int B, int T, int H, int DH, int qk_norm, float q_scale,
                int o_bf16, bool vector_gate, size_t o_align, void* stream) {
  const long long heads = (long long)B * H;
  if (heads * DH * DH > 0x7fffffffLL || heads * T * DH > 0x7fffffffLL) return GDN_ERR_SHAPE;
  if (heads == 0 || T == 0) return GDN_OK;
  if (!q || !k || !v || !g || !beta || !S || !o) return GDN_ERR_NULL;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(S, 16) ||
      !aligned(o, o_align) || !aligned(g, vector_gate ? 16 : 4) || !aligned(beta, 4))
    return GDN_ERR_ALIGN;
  const size_t toks = size_t(heads) * T;
  const size_t vec_bf16 = toks * DH * 2, o_bytes = toks * DH * (o_bf16 ? 2 : 4);
  const size_t state_bytes = size_t(heads) * DH * DH * 4;
  const size_t g_bytes = toks * (vector_gate ? DH : 1) * 4, beta_bytes = toks * 4;
  const void* ins[5] = {q, k, v, g, beta};
  const size_t in_bytes[5] = {vec_bf16, vec_bf16, vec_bf16, g_bytes, beta_bytes};
  for (int i = 0; i < 5; ++i)
    if (overlaps(o, o_bytes, ins[i], in_bytes[i]) || overlaps(S, state_bytes, ins[i], in_bytes[i]))
      return GDN_ERR_ALIAS;
  if (overlaps(o, o_bytes, S, state_bytes)) return GDN_ERR_ALIAS;
  const int dev_ok = check_device();
  if (dev_ok != GDN_OK) return dev_ok;
  gdn::DecodeArgs a{static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
                    static_cast<const __nv_bfloat16*>(v), g, beta, S, o, B, H, T, qk_norm, q_scale,
                    o_bf16, vector_gate ? 1 : 0, DH};
  return gdn::launch_decode(a, static_cast<cudaStream_t>(stream)) == 0 ? GDN_OK : GDN_ERR_LAUNCH;
}

int prefill_impl(const void* q, const void* k, const void* v, const float* g, const float* beta,
                 const float* S0, float* o, float* S_T, int B, int T, int H, int Dk, int Dv,
                 int chunk, void* ws, size_t ws_bytes, bool allow_segments, int* status,
                 void* stream, const gdn_options* opts = nullptr) {
  int qk_norm = 0, o_bf16 = 0;
  float q_scale = 1.f;
  if (!read_options(opts, &qk_norm, &q_scale, &o_bf16)) return GDN_ERR_UNSUPPORTED;
  if (o_bf16) allow_segments = false;  // the segment fix accumulates o in fp32
  if (B < 0 || T < 0 || H < 0) return GDN_ERR_SHAPE;
  if (chunk != 16 && chunk != 64) return GDN_ERR_UNSUPPORTED;
  if (Dk != kHeadDim || Dv != kHeadDim) {
    // other head dims: Dk = 64 or 128 run the chunked tensor-core kernel, with the
    // fused options; Dk = 256 takes the row kernel (its fp32 state and bf16 hi/lo
    // copy alone would fill the 512 TMEM columns), which has none
    if (!gdn::rows_head_dims_ok(Dk, Dv)) return GDN_ERR_UNSUPPORTED;
    if (Dk == 256) {
      if (qk_norm || q_scale != 1.f || o_bf16) return GDN_ERR_UNSUPPORTED;
      return rows_impl(q, k, v, g, beta, S0, o, S_T, B, T, H, Dk, Dv, false, stream);
    }
    allow_segments = false;  // the segmented schedule is built for 128 x 128 states
  }
  const long long chains = (long long)B * H;
  const long long act = chains * T * (Dk > Dv ? Dk : Dv);
  if (act > 0x7fffffffLL || chains * Dk * Dv > 0x7fffffffLL) return GDN_ERR_SHAPE;
  if (chains == 0) return GDN_OK;
  if (!S_T) return GDN_ERR_NULL;
  if (T > 0 && (!q || !k || !v || !g || !beta || !o)) return GDN_ERR_NULL;
  if (!aligned(S_T, 16) || (S0 && !aligned(S0, 16))) return GDN_ERR_ALIGN;
  if (T > 0 && (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
                !aligned(g, 4) || !aligned(beta, 4)))
    return GDN_ERR_ALIGN;
  const size_t toks = size_t(chains) * T;
  const size_t qk_bytes = toks * Dk * 2, v_bytes = toks * Dv * 2;
  const size_t act_f32 = toks * Dv * (o_bf16 ? 2 : 4);  // o bytes
  const size_t gate_bytes = toks * 4, state_bytes = size_t(chains) * Dk * Dv * 4;
  if (T > 0 && (overlaps(o, act_f32, q, qk_bytes) || overlaps(o, act_f32, k, qk_bytes) ||
                overlaps(o, act_f32, v, v_bytes) || overlaps(o, act_f32, g, gate_bytes) ||
                overlaps(o, act_f32, beta, gate_bytes) || overlaps(o, act_f32, S0, state_bytes) ||
                overlaps(o, act_f32, S_T, state_bytes)))
    return GDN_ERR_ALIAS;
  if (S0 && S0 != S_T && overlaps(S0, state_bytes, S_T, state_bytes)) return GDN_ERR_ALIAS;
  // one chain may write its S_T while another still reads its inputs
  if (T > 0 && (overlaps(S_T, state_bytes, q, qk_bytes) || overlaps(S_T, state_bytes, k, qk_bytes) ||
                overlaps(S_T, state_bytes, v, v_bytes) || overlaps(S_T, state_bytes, g, gate_bytes) ||
                overlaps(S_T, state_bytes, beta, gate_bytes)))
    return GDN_ERR_ALIAS;
  const int dev_ok = check_device();
  if (dev_ok != GDN_OK) return dev_ok;

  const int dv_box = Dv < kHeadDim ? Dv : kHeadDim;
  gdn::PrefillArgs a{g,      beta, S0,      o,       S_T,     B,      T,
                     H,      status, 1,      (T + 63) / 64, 1, nullptr, nullptr, nullptr,
                     nullptr, nullptr, 0,      0, qk_norm, q_scale, o_bf16,
                     Dk,     Dv,   Dv / dv_box, dv_box};
  if (allow_segments && T > 0) {
    int sms = 0;
    if (num_sms(&sms) != GDN_OK) return GDN_ERR_LAUNCH;
    const SegPlan plan = plan_segments(B, T, H, sms);
    if (plan.nseg > 1) {
      if (!ws || !aligned(ws, 256) || ws_bytes < plan.ws_bytes) return GDN_ERR_WORKSPACE;
      const void* args[] = {q, k, v, g, beta, S0, o, S_T};
      const size_t sizes[] = {qk_bytes, qk_bytes, v_bytes, gate_bytes, gate_bytes, state_bytes,
                              act_f32, state_bytes};
      for (int i = 0; i < 8; ++i)
        if (overlaps(ws, plan.ws_bytes, args[i], sizes[i])) return GDN_ERR_ALIAS;
      uint8_t* base = static_cast<uint8_t*>(ws);
      a.nseg = plan.nseg;
      a.seg_tiles = plan.seg_tiles;
      a.fix_parts = plan.fix_parts;
      a.ws_f = reinterpret_cast<float*>(base);
      a.ws_R = reinterpret_cast<float*>(base + plan.off_R);
      a.ws_F = reinterpret_cast<float*>(base + plan.off_F);
    }
  }
  CUtensorMap tq{}, tk{}, tv{}, to{}, tf{};
  if (T > 0) {
    const auto bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, f32 = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    if (!encode_act(&tq, q, B, T, H, 64, CU_TENSOR_MAP_SWIZZLE_128B, bf, 2, Dk) ||
        !encode_act(&tk, k, B, T, H, 64, CU_TENSOR_MAP_SWIZZLE_128B, bf, 2, Dk) ||
        !encode_act(&tv, v, B, T, H, dv_box, CU_TENSOR_MAP_SWIZZLE_NONE, bf, 2, Dv) ||
        !encode_act(&to, o, B, T, H, dv_box, CU_TENSOR_MAP_SWIZZLE_NONE, o_bf16 ? bf : f32,
                    o_bf16 ? 2 : 4, Dv))
      return GDN_ERR_LAUNCH;
    tf = to;
    if (a.nseg > 1 && !encode_act(&tf, a.ws_f, B, T, H, 128, CU_TENSOR_MAP_SWIZZLE_NONE, f32, 4))
      return GDN_ERR_LAUNCH;
  }
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (gdn::launch_prefill(tq, tk, tv, to, tf, a, chunk, st) != 0) return GDN_ERR_LAUNCH;
  if (a.nseg > 1 && gdn::launch_segment_fix(a, st) != 0) return GDN_ERR_LAUNCH;
  return GDN_OK;
}

// Device address of the built-in scratch on the current device.  Looked up
// on every call (a cheap table lookup once the module is loaded), so that the
// address stays right after a device reset or in another context of the same
// device.  The first lookup on a device may load the module there, which is
// why the first call on a device should come before any stream capture.
int static_workspace(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_static_ws) != cudaSuccess || !p) return GDN_ERR_LAUNCH;
  *out = p;
  return GDN_OK;
}

}  // namespace

namespace gdn {
bool ensure_smem_attr(const void* func, int slot, int bytes) {
  static std::atomic<uint64_t> done[96];  // bit d: device d, per kernel slot
  int dev = 0;
  if (slot < 0 || slot >= 96 || cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
    return false;
  const uint64_t bit = uint64_t(1) << dev;
  if (done[slot].load(std::memory_order_acquire) & bit) return true;
  if (cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess)
    return false;
  done[slot].fetch_or(bit, std::memory_order_acq_rel);
  return true;
}
}  // namespace gdn

extern "C" {

int gdn_abi_version(void) { return GDN_ABI_VERSION; }

const char* gdn_status_str(int code) {
  switch (code) {
    case GDN_OK: return "ok";
    case GDN_ERR_NULL: return "a required pointer is NULL";
    case GDN_ERR_ALIGN: return "misaligned pointer (q/k/v/o/S need 16 bytes, g/beta 4 bytes)";
    case GDN_ERR_SHAPE: return "negative size or problem larger than 2^31-1 elements";
    case GDN_ERR_UNSUPPORTED: return "unsupported configuration (head dims in {64, 128, 256}; fused options not with Dk = 256, nor in decode outside 64 x 64 and 128 x 128, nor in the per-channel-gate prefill with Dk other than 128; packed sequences not with Dk = 256; chunk 16 or 64; device sm_100)";
    case GDN_ERR_ALIAS: return "output overlaps an input";
    case GDN_ERR_LAUNCH: return "CUDA launch or runtime query failed";
    case GDN_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait gave up";
    case GDN_ERR_WORKSPACE: return "workspace NULL, not 256-byte aligned, or smaller than gdn_prefill_workspace_bytes";
    case GDN_ERR_STATIC_WORKSPACE_LIMIT: return "problem needs more scratch than the built-in GDN_STATIC_WORKSPACE_BYTES (16 MiB); use gdn_prefill_ws";
    default: return "unknown status code";
  }
}

int gdn_prefill(const void* q, const void* k, const void* v, const float* g, const float* beta,
                const float* S0, float* o, float* S_T, int B, int T, int H, int Dk, int Dv,
                int chunk, int* status, void* stream) {
  return prefill_impl(q, k, v, g, beta, S0, o, S_T, B, T, H, Dk, Dv, chunk, nullptr, 0, false,
                      status, stream);
}

size_t gdn_prefill_workspace_bytes(int B, int T, int H, int Dk, int Dv, int chunk) {
  if (B < 0 || T < 0 || H < 0 || Dk != kHeadDim || Dv != kHeadDim || (chunk != 16 && chunk != 64))
    return 0;
  const long long chains = (long long)B * H;
  if (chains == 0 || chains * T * kHeadDim > 0x7fffffffLL) return 0;
  int sms = 0;
  if (num_sms(&sms) != GDN_OK) return 0;
  return plan_segments(B, T, H, sms).ws_bytes;
}

int gdn_prefill_ex(const void* q, const void* k, const void* v, const float* g,
                   const float* beta, const float* S0, float* o, float* S_T, int B, int T, int H,
                   int Dk, int Dv, int chunk, void* workspace, size_t workspace_bytes,
                   const gdn_options* opts, int* status, void* stream) {
  // without a workspace: the single pass of gdn_prefill
  return prefill_impl(q, k, v, g, beta, S0, o, S_T, B, T, H, Dk, Dv, chunk, workspace,
                      workspace_bytes, workspace != nullptr, status, stream, opts);
}

int gdn_prefill_schedule(int B, int T, int H, int num_sms, int* nseg, int* seg_tiles,
                         size_t* ws_bytes) {
  if (!nseg || !seg_tiles || !ws_bytes) return GDN_ERR_NULL;
  if (B < 0 || T < 0 || H < 0 || num_sms < 0) return GDN_ERR_SHAPE;
  const SegPlan plan = plan_segments(B, T, H, num_sms);
  *nseg = plan.nseg;
  *seg_tiles = plan.seg_tiles;
  *ws_bytes = plan.ws_bytes;
  return GDN_OK;
}

int gdn_prefill_ws(const void* q, const void* k, const void* v, const float* g,
                   const float* beta, const float* S0, float* o, float* S_T, int B, int T, int H,
                   int Dk, int Dv, int chunk, void* workspace, size_t workspace_bytes,
                   int* status, void* stream) {
  return prefill_impl(q, k, v, g, beta, S0, o, S_T, B, T, H, Dk, Dv, chunk, workspace,
                      workspace_bytes, true, status, stream);
}

int gdn_prefill_varlen(const void* q, const void* k, const void* v, const float* g,
                       const float* beta, const float* S0, float* o, float* S_T,
                       const int* cu_seqlens, int N, int total_T, int H, int Dk, int Dv,
                       int chunk, float* snaps, int snap_every, int n_snaps, int* status,
                       void* stream) {
  return gdn_prefill_varlen_ex(q, k, v, g, beta, S0, o, S_T, cu_seqlens, N, total_T, H, Dk, Dv,
                               chunk, snaps, snap_every, n_snaps, nullptr, status, stream);
}

int gdn_prefill_varlen_ex(const void* q, const void* k, const void* v, const float* g,
                          const float* beta, const float* S0, float* o, float* S_T,
                          const int* cu_seqlens, int N, int total_T, int H, int Dk, int Dv,
                          int chunk, float* snaps, int snap_every, int n_snaps,
                          const gdn_options* opts, int* status, void* stream) {
  int qk_norm = 0, o_bf16 = 0;
  float q_scale = 1.f;
  if (!read_options(opts, &qk_norm, &q_scale, &o_bf16)) return GDN_ERR_UNSUPPORTED;
  if (N < 0 || total_T < 0 || H < 0 || n_snaps < 0) return GDN_ERR_SHAPE;
  // the chunked tensor-core kernel's head dims: Dk 64 or 128, Dv 64, 128 or 256
  if ((Dk != 64 && Dk != kHeadDim) || !gdn::rows_head_dims_ok(Dk, Dv) ||
      (chunk != 16 && chunk != 64))
    return GDN_ERR_UNSUPPORTED;
  if (snaps && (snap_every <= 0 || snap_every % 64 != 0)) return GDN_ERR_UNSUPPORTED;
  const long long chains = (long long)N * H;
  const long long act_k = (long long)total_T * H * Dk, act_v = (long long)total_T * H * Dv;
  if (act_k > 0x7fffffffLL || act_v > 0x7fffffffLL || chains * Dk * Dv > 0x7fffffffLL)
    return GDN_ERR_SHAPE;
  if (chains == 0) return GDN_OK;
  if (!S_T || !cu_seqlens) return GDN_ERR_NULL;
  if (total_T > 0 && (!q || !k || !v || !g || !beta || !o)) return GDN_ERR_NULL;
  if (!aligned(S_T, 16) || (S0 && !aligned(S0, 16)) || !aligned(cu_seqlens, 4)) return GDN_ERR_ALIGN;
  if (total_T > 0 && (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
                      !aligned(g, 4) || !aligned(beta, 4)))
    return GDN_ERR_ALIGN;
  const size_t act_bf16 = size_t(act_k) * 2, v_bf16 = size_t(act_v) * 2;
  const size_t o_bytes = size_t(act_v) * (o_bf16 ? 2 : 4);
  const size_t gate_bytes = size_t(total_T) * H * 4;
  const size_t state_bytes = size_t(chains) * Dk * Dv * 4, cu_bytes = size_t(N + 1) * 4;
  if (total_T > 0 && (overlaps(o, o_bytes, q, act_bf16) || overlaps(o, o_bytes, k, act_bf16) ||
                      overlaps(o, o_bytes, v, v_bf16) || overlaps(o, o_bytes, g, gate_bytes) ||
                      overlaps(o, o_bytes, beta, gate_bytes) || overlaps(o, o_bytes, S0, state_bytes) ||
                      overlaps(o, o_bytes, S_T, state_bytes) || overlaps(o, o_bytes, cu_seqlens, cu_bytes)))
    return GDN_ERR_ALIAS;
  if (S0 && S0 != S_T && overlaps(S0, state_bytes, S_T, state_bytes)) return GDN_ERR_ALIAS;
  if (overlaps(S_T, state_bytes, cu_seqlens, cu_bytes)) return GDN_ERR_ALIAS;
  if (total_T > 0 && (overlaps(S_T, state_bytes, q, act_bf16) || overlaps(S_T, state_bytes, k, act_bf16) ||
                      overlaps(S_T, state_bytes, v, v_bf16) || overlaps(S_T, state_bytes, g, gate_bytes) ||
                      overlaps(S_T, state_bytes, beta, gate_bytes)))
    return GDN_ERR_ALIAS;
  if (snaps) {
    const size_t snap_bytes = size_t(n_snaps) * H * Dk * Dv * 4;
    if (!aligned(snaps, 16)) return GDN_ERR_ALIGN;
    if ((total_T > 0 && overlaps(snaps, snap_bytes, o, o_bytes)) ||
        overlaps(snaps, snap_bytes, S_T, state_bytes) || overlaps(snaps, snap_bytes, S0, state_bytes) ||
        overlaps(snaps, snap_bytes, cu_seqlens, cu_bytes) ||
        (total_T > 0 && (overlaps(snaps, snap_bytes, q, act_bf16) || overlaps(snaps, snap_bytes, k, act_bf16) ||
                         overlaps(snaps, snap_bytes, v, v_bf16) || overlaps(snaps, snap_bytes, g, gate_bytes) ||
                         overlaps(snaps, snap_bytes, beta, gate_bytes))))
      return GDN_ERR_ALIAS;
  }
  const int dev_ok = check_device();
  if (dev_ok != GDN_OK) return dev_ok;

  // B = N chains of sequences, T = total_T: the views are [1][total_T][H][Dk or Dv]
  const int dv_box = Dv < kHeadDim ? Dv : kHeadDim;
  gdn::PrefillArgs a{g,      beta, S0,      o,       S_T,     N,      total_T,
                     H,      status, 1,      (total_T + 63) / 64, 1, nullptr, nullptr, nullptr,
                     cu_seqlens, snaps, snaps ? snap_every : 0, snaps ? n_snaps : 0, qk_norm, q_scale, o_bf16,
                     Dk,     Dv,   Dv / dv_box, dv_box};
  CUtensorMap tq{}, tk{}, tv{}, to{};
  // a valid (never read) view when every sequence is empty: S_T holds at least
  // one token's worth of any of these rows (Dk Dv >= Dk, Dv)
  const int Tv = total_T > 0 ? total_T : 1;
  const void* qv = total_T > 0 ? q : S_T;
  const auto bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, f32 = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  if (!encode_act(&tq, qv, 1, Tv, H, 64, CU_TENSOR_MAP_SWIZZLE_128B, bf, 2, Dk) ||
      !encode_act(&tk, total_T > 0 ? k : S_T, 1, Tv, H, 64, CU_TENSOR_MAP_SWIZZLE_128B, bf, 2, Dk) ||
      !encode_act(&tv, total_T > 0 ? v : S_T, 1, Tv, H, dv_box, CU_TENSOR_MAP_SWIZZLE_NONE, bf, 2, Dv) ||
      !encode_act(&to, total_T > 0 ? static_cast<const void*>(o) : S_T, 1, Tv, H, dv_box,
                  CU_TENSOR_MAP_SWIZZLE_NONE, o_bf16 ? bf : f32, o_bf16 ? 2 : 4, Dv))
    return GDN_ERR_LAUNCH;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  return gdn::launch_prefill(tq, tk, tv, to, to, a, chunk, st) == 0 ? GDN_OK : GDN_ERR_LAUNCH;
}

int gdn_prefill_static_ws(const void* q, const void* k, const void* v, const float* g,
                          const float* beta, const float* S0, float* o, float* S_T, int B,
                          int T, int H, int Dk, int Dv, int chunk, int* status, void* stream) {
  // the shape checks of prefill_impl come first, so that bad arguments get
  // their own codes rather than the limit
  if (B < 0 || T < 0 || H < 0) return GDN_ERR_SHAPE;
  if (chunk != 16 && chunk != 64) return GDN_ERR_UNSUPPORTED;
  if (Dk != kHeadDim || Dv != kHeadDim)  // other head dims run one pass, which needs no scratch
    return prefill_impl(q, k, v, g, beta, S0, o, S_T, B, T, H, Dk, Dv, chunk, nullptr, 0, false,
                        status, stream);
  const long long chains = (long long)B * H;
  if (chains * T * kHeadDim > 0x7fffffffLL || chains * kHeadDim * kHeadDim > 0x7fffffffLL)
    return GDN_ERR_SHAPE;
  if (chains == 0 || T == 0)
    return prefill_impl(q, k, v, g, beta, S0, o, S_T, B, T, H, Dk, Dv, chunk, nullptr, 0, false,
                        status, stream);
  const int dev_ok = check_device();
  if (dev_ok != GDN_OK) return dev_ok;
  int sms = 0;
  if (num_sms(&sms) != GDN_OK) return GDN_ERR_LAUNCH;
  const SegPlan plan = plan_segments(B, T, H, sms);
  if (plan.ws_bytes > GDN_STATIC_WORKSPACE_BYTES) return GDN_ERR_STATIC_WORKSPACE_LIMIT;
  void* ws = nullptr;
  if (plan.ws_bytes > 0) {
    const int rc = static_workspace(&ws);
    if (rc != GDN_OK) return rc;
  }
  return prefill_impl(q, k, v, g, beta, S0, o, S_T, B, T, H, Dk, Dv, chunk, ws,
                      ws ? size_t(GDN_STATIC_WORKSPACE_BYTES) : 0, true, status, stream);
}

int gdn_decode_step(const void* q, const void* k, const void* v, const float* g,
                    const float* beta, float* S, float* o, int B, int H, int Dk, int Dv,
                    int* status, void* stream) {
  return gdn_decode_tokens(q, k, v, g, beta, S, o, B, 1, H, Dk, Dv, status, stream);
}

int gdn_decode_tokens(const void* q, const void* k, const void* v, const float* g,
                      const float* beta, float* S, float* o, int B, int T, int H, int Dk, int Dv,
                      int* status, void* stream) {
  return gdn_decode_ex(q, k, v, g, beta, S, o, B, T, H, Dk, Dv, nullptr, status, stream);
}

int gdn_decode_ex(const void* q, const void* k, const void* v, const float* g,
                  const float* beta, float* S, float* o, int B, int T, int H, int Dk, int Dv,
                  const gdn_options* opts, int* status, void* stream) {
  (void)status;  // the decode kernels have no device-side waits
  int qk_norm = 0, o_bf16 = 0;
  float q_scale = 1.f;
  if (!read_options(opts, &qk_norm, &q_scale, &o_bf16)) return GDN_ERR_UNSUPPORTED;
  if (B < 0 || H < 0 || T < 0) return GDN_ERR_SHAPE;
  if (Dk != kHeadDim || Dv != kHeadDim) {
    // other head dims: 64 x 64 streams through the decode kernel (with the fused
    // options), the rest through the row kernel (without), the state in place
    if (!gdn::rows_head_dims_ok(Dk, Dv)) return GDN_ERR_UNSUPPORTED;
    if ((long long)B * H > 0 && !S) return GDN_ERR_NULL;
    if (Dk == 64 && Dv == 64)
      return decode_impl(q, k, v, g, beta, S, o, B, T, H, 64, qk_norm, q_scale, o_bf16, false, 4,
                         stream);
    if (qk_norm || q_scale != 1.f || o_bf16) return GDN_ERR_UNSUPPORTED;
    return rows_impl(q, k, v, g, beta, S, o, S, B, T, H, Dk, Dv, false, stream);
  }
  return decode_impl(q, k, v, g, beta, S, o, B, T, H, kHeadDim, qk_norm, q_scale, o_bf16, false,
                     16, stream);
}

int gdn_kda_prefill(const void* q, const void* k, const void* v, const float* g,
                    const float* beta, const float* S0, float* o, float* S_T, int B, int T,
                    int H, int Dk, int Dv, int* status, void* stream) {
  return gdn_kda_prefill_ex(q, k, v, g, beta, S0, o, S_T, B, T, H, Dk, Dv, nullptr, status, stream);
}

int gdn_kda_prefill_ex(const void* q, const void* k, const void* v, const float* g,
                       const float* beta, const float* S0, float* o, float* S_T, int B, int T,
                       int H, int Dk, int Dv, const gdn_options* opts, int* status, void* stream) {
  int qk_norm = 0, o_bf16 = 0;
  float q_scale = 1.f;
  if (!read_options(opts, &qk_norm, &q_scale, &o_bf16)) return GDN_ERR_UNSUPPORTED;
  const bool fused = qk_norm || q_scale != 1.f || o_bf16;
  // the row kernel validates every argument; with Dk = 128 (Dv = 64, 128 or 256)
  // and tokens to process the chunked tensor-core kernel runs instead (same
  // validation first); the fused options exist on the tensor-core kernel only
  if (B < 0 || T < 0 || H < 0) return GDN_ERR_SHAPE;
  const bool tc = Dk == kHeadDim && (Dv == 64 || Dv == kHeadDim || Dv == 2 * kHeadDim);
  if (fused && !tc) return GDN_ERR_UNSUPPORTED;
  if (o_bf16 && T == 0) o_bf16 = 0;  // no o is written
  if (!tc || T == 0 || (long long)B * H == 0)
    return rows_impl(q, k, v, g, beta, S0, o, S_T, B, T, H, Dk, Dv, true, stream);
  const long long chains = (long long)B * H;
  if (chains * T * Dv > 0x7fffffffLL || chains * kHeadDim * Dv > 0x7fffffffLL) return GDN_ERR_SHAPE;
  if (!S_T || !q || !k || !v || !g || !beta || !o) return GDN_ERR_NULL;
  if (!aligned(S_T, 16) || (S0 && !aligned(S0, 16)) || !aligned(q, 16) || !aligned(k, 16) ||
      !aligned(v, 16) || !aligned(g, 16) || !aligned(o, 16) || !aligned(beta, 4))
    return GDN_ERR_ALIGN;
  const size_t toks = size_t(chains) * T;
  const size_t act_bf16 = toks * kHeadDim * 2, v_bf16 = toks * Dv * 2,
               o_bytes = toks * Dv * (o_bf16 ? 2 : 4);
  const size_t g_bytes = toks * kHeadDim * 4, beta_bytes = toks * 4;
  const size_t state_bytes = size_t(chains) * kHeadDim * Dv * 4;
  if (S0 && S0 != S_T && overlaps(S0, state_bytes, S_T, state_bytes)) return GDN_ERR_ALIAS;
  const void* ins[5] = {q, k, v, g, beta};
  const size_t in_bytes[5] = {act_bf16, act_bf16, v_bf16, g_bytes, beta_bytes};
  for (int i = 0; i < 5; ++i)
    if (overlaps(o, o_bytes, ins[i], in_bytes[i]) || overlaps(S_T, state_bytes, ins[i], in_bytes[i]))
      return GDN_ERR_ALIAS;
  if (overlaps(o, o_bytes, S_T, state_bytes) || overlaps(o, o_bytes, S0, state_bytes))
    return GDN_ERR_ALIAS;
  const int dev_ok = check_device();
  if (dev_ok != GDN_OK) return dev_ok;
  CUtensorMap tq{}, tk{}, tv{}, to{}, tg{};
  const int dv_box = Dv < kHeadDim ? Dv : kHeadDim;  // the rows one CTA owns
  const auto bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, f32 = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  if (!encode_act(&tg, g, B, T, H, 128, CU_TENSOR_MAP_SWIZZLE_NONE, f32, 4, kHeadDim, 32) ||
      !encode_act(&tq, q, B, T, H, 64, CU_TENSOR_MAP_SWIZZLE_128B, bf, 2, kHeadDim, 32) ||
      !encode_act(&tk, k, B, T, H, 64, CU_TENSOR_MAP_SWIZZLE_128B, bf, 2, kHeadDim, 32) ||
      !encode_act(&tv, v, B, T, H, dv_box, CU_TENSOR_MAP_SWIZZLE_NONE, bf, 2, Dv, 32) ||
      !encode_act(&to, o, B, T, H, dv_box, CU_TENSOR_MAP_SWIZZLE_NONE, o_bf16 ? bf : f32,
                  o_bf16 ? 2 : 4, Dv, 32))
    return GDN_ERR_LAUNCH;
  gdn::KdaArgs a{g, beta, S0, S_T, B, T, H, status, qk_norm, q_scale, Dv, o_bf16};
  return gdn::launch_kda_prefill(tq, tk, tv, to, tg, a, static_cast<cudaStream_t>(stream)) == 0
             ? GDN_OK
             : GDN_ERR_LAUNCH;
}

int gdn_kda_prefill_varlen(const void* q, const void* k, const void* v, const float* g,
                           const float* beta, const float* S0, float* o, float* S_T,
                           const int* cu_seqlens, int N, int total_T, int H, int Dk, int Dv,
                           float* snaps, int snap_every, int n_snaps, int* status, void* stream) {
  return gdn_kda_prefill_varlen_ex(q, k, v, g, beta, S0, o, S_T, cu_seqlens, N, total_T, H, Dk, Dv,
                                   snaps, snap_every, n_snaps, nullptr, status, stream);
}

int gdn_kda_prefill_varlen_ex(const void* q, const void* k, const void* v, const float* g,
                              const float* beta, const float* S0, float* o, float* S_T,
                              const int* cu_seqlens, int N, int total_T, int H, int Dk, int Dv,
                              float* snaps, int snap_every, int n_snaps, const gdn_options* opts,
                              int* status, void* stream) {
  int qk_norm = 0, o_bf16 = 0;
  float q_scale = 1.f;
  if (!read_options(opts, &qk_norm, &q_scale, &o_bf16)) return GDN_ERR_UNSUPPORTED;
  if (N < 0 || total_T < 0 || H < 0 || n_snaps < 0) return GDN_ERR_SHAPE;
  if (Dk != kHeadDim || (Dv != 64 && Dv != kHeadDim && Dv != 2 * kHeadDim)) return GDN_ERR_UNSUPPORTED;
  if (snaps && (snap_every <= 0 || snap_every % 32 != 0)) return GDN_ERR_UNSUPPORTED;
  const long long chains = (long long)N * H;
  if ((long long)total_T * H * Dv > 0x7fffffffLL || (long long)total_T * H * kHeadDim > 0x7fffffffLL ||
      chains * kHeadDim * Dv > 0x7fffffffLL)
    return GDN_ERR_SHAPE;
  if (chains == 0) return GDN_OK;
  if (!S_T || !cu_seqlens) return GDN_ERR_NULL;
  if (total_T > 0 && (!q || !k || !v || !g || !beta || !o)) return GDN_ERR_NULL;
  if (!aligned(S_T, 16) || (S0 && !aligned(S0, 16)) || !aligned(cu_seqlens, 4)) return GDN_ERR_ALIGN;
  if (total_T > 0 && (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(g, 16) ||
                      !aligned(o, 16) || !aligned(beta, 4)))
    return GDN_ERR_ALIGN;
  const size_t toks = size_t(total_T) * H;
  const size_t act_bf16 = toks * kHeadDim * 2, v_bf16 = toks * Dv * 2, o_bytes = toks * Dv * (o_bf16 ? 2 : 4);
  const size_t g_bytes = toks * kHeadDim * 4, beta_bytes = toks * 4;
  const size_t state_bytes = size_t(chains) * kHeadDim * Dv * 4, cu_bytes = size_t(N + 1) * 4;
  if (S0 && S0 != S_T && overlaps(S0, state_bytes, S_T, state_bytes)) return GDN_ERR_ALIAS;
  if (overlaps(S_T, state_bytes, cu_seqlens, cu_bytes)) return GDN_ERR_ALIAS;
  if (total_T > 0) {
    const void* ins[6] = {q, k, v, g, beta, cu_seqlens};
    const size_t in_bytes[6] = {act_bf16, act_bf16, v_bf16, g_bytes, beta_bytes, cu_bytes};
    for (int i = 0; i < 6; ++i)
      if (overlaps(o, o_bytes, ins[i], in_bytes[i]) ||
          (i < 5 && overlaps(S_T, state_bytes, ins[i], in_bytes[i])))
        return GDN_ERR_ALIAS;
    if (overlaps(o, o_bytes, S_T, state_bytes) || overlaps(o, o_bytes, S0, state_bytes))
      return GDN_ERR_ALIAS;
  }
  if (snaps) {
    const size_t snap_bytes = size_t(n_snaps) * H * kHeadDim * Dv * 4;
    if (!aligned(snaps, 16)) return GDN_ERR_ALIGN;
    const void* others[8] = {q, k, v, g, beta, o, S_T, S0};
    const size_t other_bytes[8] = {act_bf16, act_bf16, v_bf16, g_bytes, beta_bytes, o_bytes,
                                   state_bytes, state_bytes};
    for (int i = 0; i < 8; ++i)
      if ((i >= 6 || total_T > 0) && overlaps(snaps, snap_bytes, others[i], other_bytes[i]))
        return GDN_ERR_ALIAS;
    if (overlaps(snaps, snap_bytes, cu_seqlens, cu_bytes)) return GDN_ERR_ALIAS;
  }
  const int dev_ok = check_device();
  if (dev_ok != GDN_OK) return dev_ok;
  // the views are [1][total_T][H][..]; with every sequence empty they are one
  // never-read token of S_T (which holds at least Dk Dv >= Dk, Dv floats)
  const int Tv = total_T > 0 ? total_T : 1;
  const auto pick = [&](const void* a) { return total_T > 0 ? a : static_cast<const void*>(S_T); };
  CUtensorMap tq{}, tk{}, tv{}, to{}, tg{};
  const int dv_box = Dv < kHeadDim ? Dv : kHeadDim;
  const auto bf = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, f32 = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  if (!encode_act(&tg, pick(g), 1, Tv, H, 128, CU_TENSOR_MAP_SWIZZLE_NONE, f32, 4, kHeadDim, 32) ||
      !encode_act(&tq, pick(q), 1, Tv, H, 64, CU_TENSOR_MAP_SWIZZLE_128B, bf, 2, kHeadDim, 32) ||
      !encode_act(&tk, pick(k), 1, Tv, H, 64, CU_TENSOR_MAP_SWIZZLE_128B, bf, 2, kHeadDim, 32) ||
      !encode_act(&tv, pick(v), 1, Tv, H, dv_box, CU_TENSOR_MAP_SWIZZLE_NONE, bf, 2, Dv, 32) ||
      !encode_act(&to, pick(o), 1, Tv, H, dv_box, CU_TENSOR_MAP_SWIZZLE_NONE, o_bf16 ? bf : f32,
                  o_bf16 ? 2 : 4, Dv, 32))
    return GDN_ERR_LAUNCH;
  gdn::KdaArgs a{g,  beta, S0, S_T,        N, total_T, H,     status, qk_norm, q_scale, Dv, o_bf16, cu_seqlens,
                 o,  snaps, snaps ? snap_every : 0, snaps ? n_snaps : 0};
  return gdn::launch_kda_prefill(tq, tk, tv, to, tg, a, static_cast<cudaStream_t>(stream)) == 0
             ? GDN_OK
             : GDN_ERR_LAUNCH;
}

int gdn_kda_decode(const void* q, const void* k, const void* v, const float* g,
                   const float* beta, float* S, float* o, int B, int T, int H, int Dk, int Dv,
                   int* status, void* stream) {
  return gdn_kda_decode_ex(q, k, v, g, beta, S, o, B, T, H, Dk, Dv, nullptr, status, stream);
}

int gdn_kda_decode_ex(const void* q, const void* k, const void* v, const float* g,
                      const float* beta, float* S, float* o, int B, int T, int H, int Dk, int Dv,
                      const gdn_options* opts, int* status, void* stream) {
  (void)status;  // the decode kernels have no device-side waits
  int qk_norm = 0, o_bf16 = 0;
  float q_scale = 1.f;
  if (!read_options(opts, &qk_norm, &q_scale, &o_bf16)) return GDN_ERR_UNSUPPORTED;
  const bool fused = qk_norm || q_scale != 1.f || o_bf16;
  if (B < 0 || T < 0 || H < 0) return GDN_ERR_SHAPE;
  if (fused && !(Dk == Dv && (Dk == kHeadDim || Dk == 64))) return GDN_ERR_UNSUPPORTED;
  if ((long long)B * H > 0 && !S) return GDN_ERR_NULL;
  // Dk = Dv = 128 or 64: the streaming decode kernel; other head dims: the row
  // kernel (both read and write the state once per call)
  if (Dk == Dv && (Dk == kHeadDim || Dk == 64))
    return decode_impl(q, k, v, g, beta, S, o, B, T, H, Dk, qk_norm, q_scale, o_bf16, true, 4,
                       stream);
  return rows_impl(q, k, v, g, beta, S, o, S, B, T, H, Dk, Dv, true, stream);
}

int gdn_query_status(const int* status_dev, void* stream) {
  if (!status_dev) return GDN_ERR_NULL;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return GDN_ERR_LAUNCH;
  int v = 0;
  if (cudaMemcpy(&v, status_dev, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return GDN_ERR_LAUNCH;
  return v;
}

}  // extern "C"
