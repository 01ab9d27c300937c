/* A plain C99 client of libgdn_b200.so: it includes include/gdn.h as C (no
 * C++, no torch) and calls the entry points that need no device -- the ABI
 * version, the status strings, the schedule query -- and the validation paths
 * of the compute entry points, each of which must return its documented code
 * before touching a device.  Prints one line per check and exits 0 only if all
 * pass; tests/test_abi.py builds it with gcc and runs it on the CPU. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "gdn.h"

static int failures = 0;

static void check(int cond, const char* what) {
  printf("%s %s\n", cond ? "ok  " : "FAIL", what);
  if (!cond) ++failures;
}

int main(void) {
  /* an address that is 16-byte aligned and never dereferenced: every call
   * below fails validation first */
  char* const P = (char*)(uintptr_t)0x7f0000000000ull;
  const void* q = P;
  const void* k = P + 0x1000000;
  const void* v = P + 0x2000000;
  const float* g = (const float*)(P + 0x3000000);
  const float* beta = (const float*)(P + 0x3100000);
  float* S = (float*)(P + 0x4000000);
  float* o = (float*)(P + 0x5000000);
  int nseg = 0, seg_tiles = 0;
  size_t ws = 0;
  gdn_options opts;

  check(gdn_abi_version() == GDN_ABI_VERSION, "gdn_abi_version matches the header");
  check(strcmp(gdn_status_str(GDN_OK), "") != 0, "gdn_status_str(GDN_OK) is a message");
  check(gdn_status_str(-12345) != NULL, "gdn_status_str of an unknown code is not NULL");

  check(gdn_prefill_schedule(4, 32768, 32, 148, &nseg, &seg_tiles, &ws) == GDN_OK && nseg == 1 &&
            ws == 0,
        "schedule: 128 chains run the single pass without workspace");
  check(gdn_prefill_schedule(1, 512, 16, 148, &nseg, &seg_tiles, &ws) == GDN_OK && nseg > 1 &&
            seg_tiles * nseg >= 8 && ws > 0,
        "schedule: 16 chains of 8 tiles are segmented and need a workspace");
  check(gdn_prefill_schedule(-1, 512, 16, 148, &nseg, &seg_tiles, &ws) == GDN_ERR_SHAPE,
        "schedule: negative B is GDN_ERR_SHAPE");
  check(gdn_prefill_schedule(1, 512, 16, 148, NULL, &seg_tiles, &ws) == GDN_ERR_NULL,
        "schedule: NULL output is GDN_ERR_NULL");

  check(gdn_prefill(q, k, v, g, beta, NULL, o, NULL, 1, 64, 2, 128, 128, 64, NULL, NULL) ==
            GDN_ERR_NULL,
        "prefill: NULL S_T is GDN_ERR_NULL");
  check(gdn_prefill(q, k, v, g, beta, NULL, o, S, 1, 64, 2, 128, 128, 32, NULL, NULL) ==
            GDN_ERR_UNSUPPORTED,
        "prefill: chunk 32 is GDN_ERR_UNSUPPORTED");
  check(gdn_prefill(q, k, v, g, beta, NULL, o, S, 1, 64, 2, 96, 128, 64, NULL, NULL) ==
            GDN_ERR_UNSUPPORTED,
        "prefill: Dk = 96 is GDN_ERR_UNSUPPORTED");
  check(gdn_prefill(q, k, v, g, beta, NULL, o, S, -1, 64, 2, 128, 128, 64, NULL, NULL) ==
            GDN_ERR_SHAPE,
        "prefill: negative B is GDN_ERR_SHAPE");
  check(gdn_prefill((const char*)q + 8, k, v, g, beta, NULL, o, S, 1, 64, 2, 128, 128, 64, NULL,
                    NULL) == GDN_ERR_ALIGN,
        "prefill: misaligned q is GDN_ERR_ALIGN");
  check(gdn_prefill(q, k, v, g, beta, NULL, (float*)k, S, 1, 64, 2, 128, 128, 64, NULL, NULL) ==
            GDN_ERR_ALIAS,
        "prefill: o on top of k is GDN_ERR_ALIAS");

  check(gdn_decode_step(q, k, v, g, beta, NULL, o, 4, 2, 128, 128, NULL, NULL) == GDN_ERR_NULL,
        "decode: NULL S is GDN_ERR_NULL");
  check(gdn_decode_step(q, k, v, g, beta, S, (float*)((char*)S + 64), 4, 2, 128, 128, NULL, NULL) ==
            GDN_ERR_ALIAS,
        "decode: o inside the state is GDN_ERR_ALIAS");
  check(gdn_decode_step(q, k, v, g, beta, S, o, 0, 2, 128, 128, NULL, NULL) == GDN_OK,
        "decode: B = 0 is a no-op");

  opts.size = (int)sizeof(gdn_options);
  opts.qk_l2norm = 1;
  opts.q_scale = 1.f;
  opts.o_bf16 = 0;
  check(gdn_decode_ex(q, k, v, g, beta, S, o, 4, 1, 2, 64, 128, &opts, NULL, NULL) ==
            GDN_ERR_UNSUPPORTED,
        "decode_ex: fused options at 64 x 128 (row kernel) are GDN_ERR_UNSUPPORTED");
  check(gdn_prefill_ex(q, k, v, g, beta, NULL, o, S, 1, 64, 2, 256, 256, 64, NULL, 0, &opts, NULL,
                       NULL) == GDN_ERR_UNSUPPORTED,
        "prefill_ex: fused options with Dk = 256 (row kernel) are GDN_ERR_UNSUPPORTED");
  opts.size = 4;
  check(gdn_decode_ex(q, k, v, g, beta, S, o, 4, 1, 2, 128, 128, &opts, NULL, NULL) ==
            GDN_ERR_UNSUPPORTED,
        "decode_ex: an options struct of 4 bytes is GDN_ERR_UNSUPPORTED");

  check(gdn_kda_decode(q, k, v, g, beta, NULL, o, 4, 1, 2, 128, 128, NULL, NULL) == GDN_ERR_NULL,
        "kda_decode: NULL S is GDN_ERR_NULL");
  check(gdn_kda_prefill(q, k, v, g, beta, NULL, o, S, 1, 64, 2, 100, 128, NULL, NULL) ==
            GDN_ERR_UNSUPPORTED,
        "kda_prefill: Dk = 100 is GDN_ERR_UNSUPPORTED");
  check(gdn_kda_prefill_varlen(q, k, v, g, beta, NULL, o, S, (const int*)beta, 1, 64, 2, 64, 64,
                               NULL, 0, 0, NULL, NULL) == GDN_ERR_UNSUPPORTED,
        "kda_prefill_varlen: Dk = 64 is GDN_ERR_UNSUPPORTED");
  check(gdn_kda_prefill_varlen(q, k, v, g, beta, NULL, o, S, NULL, 1, 64, 2, 128, 128, NULL, 0, 0,
                               NULL, NULL) == GDN_ERR_NULL,
        "kda_prefill_varlen: NULL cu_seqlens is GDN_ERR_NULL");
  check(gdn_kda_prefill_varlen(q, k, v, g, beta, NULL, o, S, (const int*)beta, 1, 64, 2, 128, 128,
                               S, 48, 1, NULL, NULL) == GDN_ERR_UNSUPPORTED,
        "kda_prefill_varlen: snapshots every 48 tokens are GDN_ERR_UNSUPPORTED");

  check(gdn_query_status(NULL, NULL) == GDN_ERR_NULL, "query_status: NULL word is GDN_ERR_NULL");

  printf("%d failure(s)\n", failures);
  return failures ? 1 : 0;
}
