/* A plain C client of libgs_b200.so: it includes nothing but include/gs.h and
 * the C standard library, links the shared library, and exercises the calls
 * that need no GPU -- version, status strings, workspace sizes and argument
 * checks, which return before any CUDA call. Built and run by
 * tests/test_c_abi.py. */
#include <stdio.h>
#include <string.h>

#include "gs.h"

static int fails = 0;
#define CHECK(c)                                                    \
  do {                                                              \
    if (!(c)) {                                                     \
      printf("FAIL %s:%d %s\n", __FILE__, __LINE__, #c);            \
      ++fails;                                                      \
    }                                                               \
  } while (0)

int main(void) {
  CHECK(gs_abi_version() == GS_ABI_VERSION);
  for (int s = GS_OK; s <= GS_ERR_CUDA; ++s) {
    const char* msg = gs_status_string((gs_status)s);
    CHECK(msg != NULL && strlen(msg) > 0);
  }

  gs_camera cam;
  memset(&cam, 0, sizeof cam);
  cam.viewmat[0] = cam.viewmat[5] = cam.viewmat[10] = 1.f;
  cam.viewmat[11] = 8.f;
  cam.fx = cam.fy = 100.f;
  cam.cx = cam.cy = 64.f;
  cam.width = cam.height = 128;
  const size_t small = gs_workspace_size(1000, 1, &cam, 10000, GS_SORT_FULL64);
  const size_t large = gs_workspace_size(1000, 1, &cam, 1000000, GS_SORT_FULL64);
  CHECK(small > 0 && large > small);
  CHECK(gs_workspace_size(-1, 1, &cam, 10, GS_SORT_FULL64) == 0);
  CHECK(gs_workspace_size(10, 0, &cam, 10, GS_SORT_FULL64) == 0);

  /* the sort plan of a 3840 x 2160 view: pairs by tile column, ranges from
   * the tile counts, the 135 rows as one-byte keys */
  {
    gs_camera c4 = cam;
    c4.width = 3840;
    c4.height = 2160;
    gs_sort_plan pl;
    memset(&pl, 0xff, sizeof pl);
    CHECK(sizeof(gs_sort_plan) == 40);
    CHECK(gs_bin_sort_plan(1000, 1, &c4, GS_SORT_PRESORT, &pl) == GS_OK);
    CHECK(pl.path == GS_PATH_COLUMNS && pl.ranges_from_counts == 1 && pl.pair_key_bytes == 1);
    CHECK(pl.pair_passes == 1 && pl.reserved == 0);
    CHECK(gs_bin_sort_plan(1000, 1, &c4, GS_SORT_FULL64, &pl) == GS_OK);
    CHECK(pl.pair_key_bytes == 8 && pl.ranges_from_counts == 1);
  }

  gs_params p;
  memset(&p, 0, sizeof p);
  p.n = 10;
  p.sh_degree = 4; /* degrees stop at 3 */
  gs_projected out;
  memset(&out, 0, sizeof out);
  /* an aligned address that is never dereferenced: every call below returns
   * before anything is enqueued */
  void* ws = (void*)(uintptr_t)4096;
  CHECK(gs_project(&p, &cam, 1, &out, ws, NULL) == GS_ERR_INVALID_ARG);
  p.sh_degree = 0;
  p.n = (int64_t)1 << 31;
  CHECK(gs_project(&p, &cam, 1, &out, ws, NULL) == GS_ERR_OVERFLOW);
  CHECK(gs_project(&p, &cam, 1, &out, NULL, NULL) == GS_ERR_INVALID_ARG); /* no status word */

  CHECK(gs_debug_stall(GS_STALL_RASTER_FWD, -1, 0.0) == GS_ERR_INVALID_ARG);
  CHECK(gs_debug_stall(7, 0, 0.0) == GS_ERR_INVALID_ARG);
  CHECK(gs_debug_stall(GS_STALL_NONE, 0, -1.0) == GS_ERR_INVALID_ARG);
  CHECK(gs_debug_stall(GS_STALL_NONE, 0, 0.0) == GS_OK);
  CHECK((GS_STATUS_BIT_CAPACITY | GS_STATUS_BIT_TIMEOUT | GS_STATUS_BIT_BOUNDS |
         GS_STATUS_BIT_NONFINITE) == 15u);

  CHECK(gs_l1_dssim_workspace_size(2) == 2 * 16 + 16);
  CHECK(gs_l1_dssim(NULL, NULL, 0, 8, 8, 0.2f, NULL, NULL, NULL, 0, NULL) == GS_OK);
  CHECK(gs_l1_dssim(NULL, NULL, 1, 8, 8, 0.2f, NULL, NULL, NULL, 0, NULL) ==
        GS_ERR_INVALID_ARG);

  gs_sh_quant q;
  memset(&q, 0, sizeof q);
  q.k3 = 12;
  q.bits = 8;
  CHECK(gs_sh_quantize(NULL, &q, NULL) == GS_OK); /* no Gaussians: nothing to do */
  q.bits = 12;
  CHECK(gs_sh_quantize(NULL, &q, NULL) == GS_ERR_INVALID_ARG);
  q.bits = 16;
  q.layout = 2; /* neither planar nor packed */
  CHECK(gs_sh_quantize(NULL, &q, NULL) == GS_ERR_INVALID_ARG);
  q.layout = GS_QUANT_PACKED;
  CHECK(gs_sh_quantize(NULL, &q, NULL) == GS_OK);
  CHECK(gs_densify_sh_quant_workspace_size(1000, 1500) > 0);
  CHECK(gs_densify_sh_quant_workspace_size(-1, 0) == 0);
  /* quantised SH and float SH together are refused */
  p.n = 10;
  p.sh = (const float*)(uintptr_t)4096;
  p.sh_quant = &q;
  CHECK(gs_project(&p, &cam, 1, &out, ws, NULL) == GS_ERR_INVALID_ARG);

  CHECK(gs_adam_step(NULL, 1, 0.9f, 0.999f, 1e-15f, 1, NULL) == GS_ERR_INVALID_ARG);
  CHECK(gs_densify_workspace_size(1000) > 0 && gs_densify_workspace_size(-1) == 0);

  if (fails) {
    printf("c abi check: %d failure(s)\n", fails);
    return 1;
  }
  printf("c abi check ok\n");
  return 0;
}
