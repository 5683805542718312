// capi.cu -- the extern "C" entry points declared in include/gs.h.
//
// Host-side argument checks, workspace carving and kernel launches. Nothing
// here allocates device memory or keeps state between calls (the only
// process-wide setting is the test hook of gs_debug_stall).

#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <cuda_runtime.h>

#include "gs_internal.h"

using namespace gsb;

namespace {

constexpr size_t kAlign = 256;
constexpr size_t kControlBytes = 4096;  // status word, counters, device scalars
constexpr size_t kStatusOffset = 0;
constexpr size_t kCountersOffset = 64;   // 16 x uint32
constexpr size_t kNItemsOffset = 256;    // int64
constexpr size_t kPairTotalOffset = 264; // uint64
constexpr size_t kNVisibleOffset = 512;  // uint32 [GS_MAX_VIEWS]
constexpr size_t kScanNOffset = 640;     // int64
constexpr size_t kHistBytes = 256 * sizeof(uint32_t);  // digit totals of the current pass
constexpr int64_t kMaxPairCapacity = GS_MAX_PAIR_CAPACITY;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

int bits_for(uint64_t max_value) {
  int b = 0;
  while (max_value) { ++b; max_value >>= 1; }
  return b;
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

struct Layout {
  RadixPlan pairs, presort;
  bool tile_emit = false;
  int gsize = 0, tile_bpv = 0;
  bool column_emit = false;
  bool count_ranges = false;
  int row_key_bytes = 4;
  int cbits = 0;
  int key_bytes = 8;
  int64_t counts_stride = 0;
  size_t off_hist = 0, off_emit_lb = 0, off_counts = 0, off_keys0 = 0, off_keys1 = 0,
         off_vals1 = 0, off_pkeys0 = 0, off_pkeys1 = 0, off_pvals0 = 0, off_pvals1 = 0,
         off_crect = 0, off_tile_totals = 0, off_tile_base = 0, off_digit_hist = 0,
         off_sweep_lb = 0, off_tdiff = 0, off_view_pairs = 0;
  size_t sweep_lb_bytes = 0, tdiff_bytes = 0;
  size_t total = 0;
};

bool check_cams(const gs_camera* cams, int32_t n_views) {
  if (!cams || n_views < 1 || n_views > GS_MAX_VIEWS) return false;
  for (int v = 0; v < n_views; ++v) {
    if (cams[v].width <= 0 || cams[v].height <= 0) return false;
    if (cams[v].width != cams[0].width || cams[v].height != cams[0].height) return false;
  }
  const Grid g = grid_of(cams[0]);
  if (g.tiles_x > 65535 || g.tiles_y > 65535) return false;
  return true;
}

bool make_layout(int64_t n, int32_t n_views, const gs_camera* cams, int64_t capacity, int32_t mode,
                 Layout& L) {
  // pair positions are 32-bit inside the sort
  if (n < 0 || n >= (1ll << 31) || capacity < 0 || capacity > kMaxPairCapacity) return false;
  if (mode != GS_SORT_FULL64 && mode != GS_SORT_PRESORT) return false;
  if (!check_cams(cams, n_views)) return false;
  const Grid g = grid_of(cams[0]);
  const uint64_t tiles = (uint64_t)g.tiles_per_view * (uint64_t)n_views;
  if (tiles >= (1ull << 32)) return false;
  const int tile_bits = bits_for(tiles - 1);
  const int64_t items = n * n_views;
  if (mode == GS_SORT_FULL64) {
    L.key_bytes = 8;
    L.pairs = make_radix_plan(32 + tile_bits, false);
    L.count_ranges = count_ranges_fit(g);
  } else {
    L.key_bytes = 4;
    L.presort = make_radix_plan(32 + bits_for((uint64_t)n_views - 1), false);
    L.tile_emit = tile_emission(g);
    L.column_emit = !L.tile_emit && column_emission(g);
    if (L.tile_emit) {
      L.gsize = tile_gsize(n);
      L.tile_bpv = (int)((n + L.gsize - 1) / L.gsize);
    } else if (L.column_emit) {
      // keys row << cbits | column; the radix passes sort the row bits
      L.cbits = bits_for((uint64_t)g.tiles_x - 1);
      if (L.cbits == 0) L.cbits = 1;
      L.count_ranges = count_ranges_fit(g);
      const uint64_t rows = (uint64_t)g.tiles_y * n_views;
      L.pairs = make_radix_plan(bits_for(rows - 1), true);
      if (L.count_ranges && rows <= 65536) {
        // the ranges come from the tile counts: the keys are the rows alone
        L.row_key_bytes = rows <= 256 ? 1 : 2;
        L.key_bytes = L.row_key_bytes;
      } else {
        for (int i = 0; i < L.pairs.passes; ++i) L.pairs.shift[i] += L.cbits;
      }
    } else {
      L.pairs = make_radix_plan(tile_bits, true);
    }
  }
  int64_t parts = pair_partitions(capacity);
  if (mode == GS_SORT_PRESORT) {
    const int64_t p2 = presort_partitions(items);
    if (p2 > parts) parts = p2;
    const int64_t p3 = L.tile_emit ? L.tile_bpv : column_blocks(items);
    if (p3 > parts) parts = p3;
  }
  L.counts_stride = parts > 0 ? (parts + 3) / 4 * 4 : 4;
  // counts rows: radix digits, tile columns, or every tile of every view
  // (rounded up to whole groups of 8 tiles)
  const int64_t trows = ((int64_t)tiles + 7) / 8 * 8;
  const int64_t rows = L.tile_emit && trows > 256 ? trows : 256;
  size_t off = kControlBytes;
  L.off_hist = off; off = align_up(off + kHistBytes);
  L.off_emit_lb = off; off = align_up(off + (size_t)emit_blocks(items) * 8);
  L.off_counts = off; off = align_up(off + (size_t)rows * L.counts_stride * 4);
  // pair keys and the second id buffer: not needed when pairs are placed
  // straight at their positions
  const int64_t kcap = L.tile_emit ? 0 : capacity;
  L.off_keys0 = off; off = align_up(off + (size_t)kcap * L.key_bytes);
  L.off_keys1 = off; off = align_up(off + (size_t)kcap * L.key_bytes);
  L.off_vals1 = off; off = align_up(off + (size_t)kcap * 4);
  // single-sweep passes (the pair keys in full-64 mode, the depth keys in
  // presort mode): every pass's digit counts, one look-back word per
  // (partition, digit)
  L.off_digit_hist = off; off = align_up(off + 8 * 256 * sizeof(uint32_t));
  L.sweep_lb_bytes = (size_t)(mode == GS_SORT_FULL64 ? pair_partitions(capacity)
                                                     : presort_partitions(items)) *
                     256 * sizeof(uint64_t);
  L.off_sweep_lb = off; off = align_up(off + L.sweep_lb_bytes);
  if (mode == GS_SORT_PRESORT) {
    L.off_pkeys0 = off; off = align_up(off + (size_t)items * 8);
    L.off_pkeys1 = off; off = align_up(off + (size_t)items * 8);
    L.off_pvals0 = off; off = align_up(off + (size_t)items * 4);
    L.off_pvals1 = off; off = align_up(off + (size_t)items * 4);
    if (L.column_emit || L.tile_emit) {
      L.off_crect = off; off = align_up(off + (size_t)items * 16);
    }
    if (L.tile_emit) {
      L.off_tile_totals = off; off = align_up(off + (size_t)tiles * 4);
      L.off_tile_base = off; off = align_up(off + (size_t)tiles * 4);
    }
  }
  if (L.count_ranges) {
    // per view: the tile-count difference array, and the view's pair total
    L.tdiff_bytes = (size_t)n_views * (g.tiles_x + 1) * (g.tiles_y + 1) * sizeof(int);
    L.off_tdiff = off; off = align_up(off + L.tdiff_bytes);
    L.off_view_pairs = off; off = align_up(off + GS_MAX_VIEWS * sizeof(uint64_t));
  }
  L.total = off;
  return true;
}

CamSet pack_cams(const gs_camera* cams, int32_t n_views) {
  CamSet s;
  std::memset(&s, 0, sizeof(s));
  for (int v = 0; v < n_views; ++v) s.c[v] = cams[v];
  return s;
}

inline gs_status cuda_status(cudaError_t e) { return e == cudaSuccess ? GS_OK : GS_ERR_CUDA; }

// gs_debug_stall's setting: which wait site stalls which block, and the wait
// limit while it holds.
std::atomic<int32_t> g_stall_site{GS_STALL_NONE};
std::atomic<int64_t> g_stall_index{-1};
std::atomic<uint64_t> g_wait_ns{0};

WaitCfg wait_cfg(int32_t site) {
  WaitCfg w;
  const uint64_t ns = g_wait_ns.load();
  w.limit_ns = ns ? ns : kWaitLimitNs;
  w.stall = g_stall_site.load() == site ? g_stall_index.load() : -1;
  return w;
}

bool status_ws_ok(const void* ws) { return ws && aligned(ws, kAlign); }

uint32_t* status_word(void* ws) {
  return reinterpret_cast<uint32_t*>(static_cast<unsigned char*>(ws) + kStatusOffset);
}

bool quant_ok(const gs_sh_quant* q) {
  if (!q || q->n < 0 || q->n >= (1ll << 31)) return false;
  if (q->bits != 8 && q->bits != 16) return false;
  if (q->k3 != 3 && q->k3 != 12 && q->k3 != 27 && q->k3 != 48) return false;
  if (q->layout != GS_QUANT_PLANAR && q->layout != GS_QUANT_PACKED) return false;
  if (q->n == 0) return true;
  // codes (and packed moments) move four at a time
  const size_t a = q->layout == GS_QUANT_PACKED ? 8 : (size_t)(q->bits / 2);
  return q->codes && q->bounds && aligned(q->codes, a) && aligned(q->bounds, 8);
}

// The SH source of a parameter set: exactly one of sh and sh_quant, the
// codes matching n and the degree.
bool params_sh_ok(const gs_params& p) {
  if (!p.sh_quant) return p.sh != nullptr;
  if (p.sh || !quant_ok(p.sh_quant)) return false;
  return p.sh_quant->n == p.n && p.sh_quant->k3 == 3 * (p.sh_degree + 1) * (p.sh_degree + 1);
}

}  // namespace

extern "C" {

int32_t gs_abi_version(void) { return GS_ABI_VERSION; }

const char* gs_status_string(gs_status s) {
  switch (s) {
    case GS_OK: return "ok";
    case GS_ERR_INVALID_ARG: return "invalid argument";
    case GS_ERR_CAPACITY: return "pair capacity exceeded";
    case GS_ERR_OVERFLOW: return "size exceeds a 32-bit field";
    case GS_ERR_DEVICE_TIMEOUT: return "a bounded device-side wait gave up";
    case GS_ERR_NONFINITE: return "non-finite input";
    case GS_ERR_CUDA: return "CUDA runtime error";
  }
  return "unknown status";
}

size_t gs_workspace_size(int64_t n, int32_t n_views, const gs_camera* cams, int64_t pair_capacity,
                         int32_t sort_mode) {
  Layout L;
  if (!make_layout(n, n_views, cams, pair_capacity, sort_mode, L)) return 0;
  return L.total;
}

gs_status gs_project(const gs_params* params, const gs_camera* cams, int32_t n_views,
                     gs_projected* out, void* ws, void* stream) {
  if (!params || !out || !check_cams(cams, n_views) || !status_ws_ok(ws))
    return GS_ERR_INVALID_ARG;
  const gs_params& p = *params;
  if (p.n < 0) return GS_ERR_INVALID_ARG;
  if (p.n >= (1ll << 31) || p.n * n_views >= (1ll << 40)) return GS_ERR_OVERFLOW;
  if (p.sh_degree < 0 || p.sh_degree > 3) return GS_ERR_INVALID_ARG;
  if (p.n == 0) return GS_OK;
  if (!p.means || !p.log_scales || !p.quats || !p.opacity_logit || !params_sh_ok(p) ||
      !out->records || !out->bins || !out->radii)
    return GS_ERR_INVALID_ARG;
  if (!aligned(p.means, 16) || !aligned(p.log_scales, 16) || !aligned(p.quats, 16) ||
      !aligned(out->records, 16) || !aligned(out->bins, 16))
    return GS_ERR_INVALID_ARG;
  const CamSet cs = pack_cams(cams, n_views);
  return cuda_status(launch_project(p, cs, n_views, out->records, out->bins, out->radii,
                                    status_word(ws), wait_cfg(GS_STALL_NONE),
                                    static_cast<cudaStream_t>(stream)));
}

gs_status gs_bin_sort(const gs_projected* proj, const gs_camera* cams, int32_t n_views, int64_t n,
                      int32_t sort_mode, gs_binned* out, void* ws, size_t ws_bytes,
                      void* stream) {
  if (!proj || !out || !ws) return GS_ERR_INVALID_ARG;
  if (n >= (1ll << 31)) return GS_ERR_OVERFLOW;
  Layout L;
  if (!make_layout(n, n_views, cams, out->pair_capacity, sort_mode, L)) return GS_ERR_INVALID_ARG;
  if (ws_bytes < L.total || !aligned(ws, kAlign)) return GS_ERR_INVALID_ARG;
  if (!out->ids || !out->ranges || !out->n_pairs) return GS_ERR_INVALID_ARG;
  if (n > 0 && (!proj->bins || !aligned(proj->bins, 16))) return GS_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned char* w = static_cast<unsigned char*>(ws);
  const Grid g = grid_of(cams[0]);
  const int64_t tiles = (int64_t)g.tiles_per_view * n_views;
  const int64_t items = n * n_views;

  if (cudaMemsetAsync(w + kCountersOffset, 0, 16 * sizeof(uint32_t), st) != cudaSuccess ||
      cudaMemsetAsync(w + kPairTotalOffset, 0, sizeof(uint64_t), st) != cudaSuccess ||
      cudaMemsetAsync(w + kNVisibleOffset, 0, GS_MAX_VIEWS * sizeof(uint32_t), st) != cudaSuccess ||
      cudaMemsetAsync(w + L.off_emit_lb, 0, (size_t)emit_blocks(items) * 8, st) != cudaSuccess ||
      cudaMemsetAsync(out->ranges, 0, (size_t)tiles * 2 * sizeof(int64_t), st) != cudaSuccess)
    return GS_ERR_CUDA;
  if (cudaMemsetAsync(w + L.off_digit_hist, 0, 8 * 256 * sizeof(uint32_t), st) != cudaSuccess ||
      (L.sweep_lb_bytes &&
       cudaMemsetAsync(w + L.off_sweep_lb, 0, L.sweep_lb_bytes, st) != cudaSuccess))
    return GS_ERR_CUDA;
  if (L.count_ranges &&
      (cudaMemsetAsync(w + L.off_tdiff, 0, L.tdiff_bytes, st) != cudaSuccess ||
       cudaMemsetAsync(w + L.off_view_pairs, 0, GS_MAX_VIEWS * sizeof(uint64_t), st) !=
           cudaSuccess))
    return GS_ERR_CUDA;

  BinSortArgs a{};
  a.bins = proj->bins;
  a.n = (int)n;
  a.n_views = n_views;
  a.mode = sort_mode;
  a.grid = g;
  a.capacity = out->pair_capacity;
  a.tile_emit = L.tile_emit;
  a.gsize = L.gsize;
  a.tile_bpv = L.tile_bpv;
  a.column_emit = L.column_emit;
  a.cbits = L.cbits;
  a.count_ranges = L.count_ranges;
  a.row_key_bytes = L.row_key_bytes;
  if (L.count_ranges) {
    a.tile_diff = reinterpret_cast<int*>(w + L.off_tdiff);
    a.view_pairs = reinterpret_cast<unsigned long long*>(w + L.off_view_pairs);
  }
  a.pairs = L.pairs;
  a.presort = L.presort;
  a.emit_buf = L.pairs.passes & 1;
  a.keys[0] = reinterpret_cast<uint64_t*>(w + L.off_keys0);
  a.keys[1] = reinterpret_cast<uint64_t*>(w + L.off_keys1);
  a.vals[0] = out->ids;
  a.vals[1] = reinterpret_cast<uint32_t*>(w + L.off_vals1);
  if (sort_mode == GS_SORT_PRESORT) {
    a.pkeys[0] = reinterpret_cast<uint64_t*>(w + L.off_pkeys0);
    a.pkeys[1] = reinterpret_cast<uint64_t*>(w + L.off_pkeys1);
    a.pvals[0] = reinterpret_cast<uint32_t*>(w + L.off_pvals0);
    a.pvals[1] = reinterpret_cast<uint32_t*>(w + L.off_pvals1);
  }
  a.totals = reinterpret_cast<uint32_t*>(w + L.off_hist);
  a.counts = reinterpret_cast<uint32_t*>(w + L.off_counts);
  a.counts_stride = L.counts_stride;
  a.emit_lookback = reinterpret_cast<uint64_t*>(w + L.off_emit_lb);
  a.digit_hist = reinterpret_cast<uint32_t*>(w + L.off_digit_hist);
  a.sweep_lookback = reinterpret_cast<uint64_t*>(w + L.off_sweep_lb);
  a.counters = reinterpret_cast<uint32_t*>(w + kCountersOffset);
  a.status = reinterpret_cast<uint32_t*>(w + kStatusOffset);
  a.wait = wait_cfg(GS_STALL_EMIT_LOOKBACK);
  a.sort_wait = wait_cfg(GS_STALL_SORT_LOOKBACK);
  a.n_pairs = out->n_pairs;
  a.n_items_dev = reinterpret_cast<int64_t*>(w + kNItemsOffset);
  a.pair_total = reinterpret_cast<unsigned long long*>(w + kPairTotalOffset);
  if (L.column_emit || L.tile_emit) a.crect = reinterpret_cast<uint4*>(w + L.off_crect);
  a.n_visible = reinterpret_cast<uint32_t*>(w + kNVisibleOffset);
  a.scan_n = reinterpret_cast<int64_t*>(w + kScanNOffset);
  if (L.tile_emit) {
    a.tile_totals = reinterpret_cast<uint32_t*>(w + L.off_tile_totals);
    a.tile_base = reinterpret_cast<uint32_t*>(w + L.off_tile_base);
  }
  a.ranges = out->ranges;
  a.n_tiles = tiles;
  return cuda_status(launch_bin_sort(a, st));
}

gs_status gs_rasterize_fwd(const gs_projected* proj, const gs_binned* bins, const gs_camera* cams,
                           int32_t n_views, int64_t n, const float* bg, float* image,
                           float* final_T, uint32_t* n_contrib, uint8_t* warp_masks, void* ws,
                           void* stream) {
  if (!proj || !bins || !bg || !check_cams(cams, n_views) || !status_ws_ok(ws))
    return GS_ERR_INVALID_ARG;
  if (n < 0) return GS_ERR_INVALID_ARG;
  if (n >= (1ll << 31)) return GS_ERR_OVERFLOW;
  if (!image || !final_T || !n_contrib || !bins->ranges || !bins->ids) return GS_ERR_INVALID_ARG;
  if (n > 0 && (!proj->records || !aligned(proj->records, 16))) return GS_ERR_INVALID_ARG;
  const Grid g = grid_of(cams[0]);
  return cuda_status(launch_raster_fwd(proj->records, bins->ids, bins->ranges, bins->pair_capacity,
                                       g, n_views, (int)n, bg, image, final_T, n_contrib,
                                       warp_masks, status_word(ws),
                                       wait_cfg(GS_STALL_RASTER_FWD),
                                       static_cast<cudaStream_t>(stream)));
}

namespace {

gs_status check_grads_args(const gs_params& p, const gs_grads* grads, bool need) {
  if (!grads) return need ? GS_ERR_INVALID_ARG : GS_OK;
  if (p.n > 0 && (!p.means || !p.log_scales || !p.quats || !p.opacity_logit ||
                  !params_sh_ok(p) || !grads->means || !grads->log_scales || !grads->quats ||
                  !grads->opacity_logit || !grads->sh))
    return GS_ERR_INVALID_ARG;
  if (!aligned(p.means, 16) || !aligned(p.log_scales, 16) || !aligned(p.quats, 16) ||
      !aligned(grads->means, 16) || !aligned(grads->log_scales, 16) ||
      !aligned(grads->quats, 16))
    return GS_ERR_INVALID_ARG;
  return GS_OK;
}

}  // namespace

gs_status gs_project_bwd(const gs_params* params, const gs_camera* cams, int32_t n_views,
                         const int32_t* radii, const float* grad2d, gs_grads* grads,
                         void* stream) {
  if (!params || !check_cams(cams, n_views)) return GS_ERR_INVALID_ARG;
  const gs_params& p = *params;
  if (p.n < 0 || p.sh_degree < 0 || p.sh_degree > 3) return GS_ERR_INVALID_ARG;
  if (p.n >= (1ll << 31)) return GS_ERR_OVERFLOW;
  const gs_status s = check_grads_args(p, grads, true);
  if (s != GS_OK) return s;
  if (p.n == 0) return GS_OK;
  if (!radii || !grad2d || !aligned(grad2d, 16)) return GS_ERR_INVALID_ARG;
  const CamSet cs = pack_cams(cams, n_views);
  return cuda_status(launch_project_bwd(p, cs, n_views, grad2d, radii, *grads,
                                        static_cast<cudaStream_t>(stream)));
}

gs_status gs_project_bwd_adam(const gs_params* params, const gs_camera* cams, int32_t n_views,
                              const int32_t* radii, const float* grad2d, gs_grads* exp_avg,
                              gs_grads* exp_avg_sq, const float* lr, float beta1, float beta2,
                              float eps, int64_t step, float* accum_plain, float* accum_abs,
                              int32_t* denom, void* stream) {
  if (!params || !check_cams(cams, n_views) || !exp_avg || !exp_avg_sq || !lr)
    return GS_ERR_INVALID_ARG;
  const gs_params& p = *params;
  if (p.n < 0 || p.sh_degree < 0 || p.sh_degree > 3 || p.sh_quant) return GS_ERR_INVALID_ARG;
  if (p.n >= (1ll << 31)) return GS_ERR_OVERFLOW;
  if (step < 1 || !(beta1 >= 0.f && beta1 < 1.f) || !(beta2 >= 0.f && beta2 < 1.f) ||
      !(eps >= 0.f))
    return GS_ERR_INVALID_ARG;
  const bool stats = accum_plain || accum_abs || denom;
  if (stats && !(accum_plain && accum_abs && denom)) return GS_ERR_INVALID_ARG;
  // the moments take the gradients' place: same layouts and alignment checks
  if (check_grads_args(p, exp_avg, true) != GS_OK || check_grads_args(p, exp_avg_sq, true) != GS_OK)
    return GS_ERR_INVALID_ARG;
  if (p.n == 0) return GS_OK;
  if (!radii || !grad2d || !aligned(grad2d, 16)) return GS_ERR_INVALID_ARG;
  // the SH blocks move as float4
  if (!aligned(p.sh, 16) || !aligned(exp_avg->sh, 16) || !aligned(exp_avg_sq->sh, 16))
    return GS_ERR_INVALID_ARG;
  AdamTail t{};
  t.p_means = reinterpret_cast<float4*>(const_cast<float*>(p.means));
  t.p_log_scales = reinterpret_cast<float4*>(const_cast<float*>(p.log_scales));
  t.p_quats = reinterpret_cast<float4*>(const_cast<float*>(p.quats));
  t.p_logit = const_cast<float*>(p.opacity_logit);
  t.p_sh = const_cast<float*>(p.sh);
  t.m_means = reinterpret_cast<float4*>(exp_avg->means);
  t.m_log_scales = reinterpret_cast<float4*>(exp_avg->log_scales);
  t.m_quats = reinterpret_cast<float4*>(exp_avg->quats);
  t.m_logit = exp_avg->opacity_logit;
  t.m_sh = exp_avg->sh;
  t.v_means = reinterpret_cast<float4*>(exp_avg_sq->means);
  t.v_log_scales = reinterpret_cast<float4*>(exp_avg_sq->log_scales);
  t.v_quats = reinterpret_cast<float4*>(exp_avg_sq->quats);
  t.v_logit = exp_avg_sq->opacity_logit;
  t.v_sh = exp_avg_sq->sh;
  for (int k = 0; k < 5; ++k) t.lr[k] = lr[k];
  t.b1 = beta1;
  t.b2 = beta2;
  t.eps = eps;
  // the bias corrections exactly as gs_adam_step takes them
  t.ibc1 = (float)(1.0 / (1.0 - pow((double)beta1, (double)step)));
  t.ibc2 = (float)(1.0 / (1.0 - pow((double)beta2, (double)step)));
  t.accum_plain = accum_plain;
  t.accum_abs = accum_abs;
  t.denom = denom;
  const CamSet cs = pack_cams(cams, n_views);
  return cuda_status(launch_project_bwd_adam(p, cs, n_views, grad2d, radii, t,
                                             static_cast<cudaStream_t>(stream)));
}

gs_status gs_rasterize_bwd(const gs_params* params, const gs_projected* proj,
                           const gs_binned* bins, const gs_camera* cams, int32_t n_views,
                           const float* bg, const float* dL_dimage, const float* final_T,
                           const uint32_t* n_contrib, const uint8_t* warp_masks,
                           float* grad2d, gs_grads* grads, void* ws, void* stream) {
  if (!params || !proj || !bins || !bg || !check_cams(cams, n_views) || !status_ws_ok(ws))
    return GS_ERR_INVALID_ARG;
  const gs_params& p = *params;
  if (p.n < 0 || p.sh_degree < 0 || p.sh_degree > 3) return GS_ERR_INVALID_ARG;
  if (p.n >= (1ll << 31)) return GS_ERR_OVERFLOW;
  if (!dL_dimage || !final_T || !n_contrib || !bins->ranges || !bins->ids)
    return GS_ERR_INVALID_ARG;
  if (p.n > 0 && (!proj->records || !proj->radii || !grad2d)) return GS_ERR_INVALID_ARG;
  if (!aligned(grad2d, 16)) return GS_ERR_INVALID_ARG;
  const gs_status s = check_grads_args(p, grads, false);
  if (s != GS_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const Grid g = grid_of(cams[0]);
  if (cudaMemsetAsync(grad2d, 0, (size_t)p.n * n_views * GS_GRAD2D_FLOATS * sizeof(float), st) !=
      cudaSuccess)
    return GS_ERR_CUDA;
  cudaError_t e = launch_raster_bwd(proj->records, bins->ids, bins->ranges, bins->pair_capacity, g,
                                    n_views, (int)p.n, bg, dL_dimage, final_T, n_contrib,
                                    warp_masks, grad2d,
                                    status_word(ws),
                                    wait_cfg(GS_STALL_RASTER_BWD), st);
  if (e != cudaSuccess) return GS_ERR_CUDA;
  if (!grads) return GS_OK;
  const CamSet cs = pack_cams(cams, n_views);
  return cuda_status(launch_project_bwd(p, cs, n_views, grad2d, proj->radii, *grads, st));
}

gs_status gs_densify_stats(const float* grad2d, const int32_t* radii, int32_t n_views, int64_t n,
                           float* accum_plain, float* accum_abs, int32_t* denom, void* stream) {
  if (n < 0 || n_views < 1 || n_views > GS_MAX_VIEWS) return GS_ERR_INVALID_ARG;
  if (n >= (1ll << 31)) return GS_ERR_OVERFLOW;
  if (n == 0) return GS_OK;
  if (!grad2d || !radii || !accum_plain || !accum_abs || !denom || !aligned(grad2d, 16))
    return GS_ERR_INVALID_ARG;
  return cuda_status(launch_densify(grad2d, radii, n_views, (int)n, accum_plain, accum_abs, denom,
                                    static_cast<cudaStream_t>(stream)));
}

gs_status gs_adam_step(const gs_adam_group* groups, int32_t n_groups, float beta1, float beta2,
                       float eps, int64_t step, void* stream) {
  if (!groups || n_groups < 1 || n_groups > 8 || step < 1) return GS_ERR_INVALID_ARG;
  if (!(beta1 >= 0.f && beta1 < 1.f) || !(beta2 >= 0.f && beta2 < 1.f) || !(eps >= 0.f))
    return GS_ERR_INVALID_ARG;
  for (int k = 0; k < n_groups; ++k) {
    const gs_adam_group& gr = groups[k];
    if (gr.count < 0) return GS_ERR_INVALID_ARG;
    if (gr.count == 0) continue;
    if (!gr.param || !gr.grad || !gr.exp_avg || !gr.exp_avg_sq) return GS_ERR_INVALID_ARG;
    if (!aligned(gr.param, 16) || !aligned(gr.grad, 16) || !aligned(gr.exp_avg, 16) ||
        !aligned(gr.exp_avg_sq, 16))
      return GS_ERR_INVALID_ARG;
  }
  return cuda_status(
      launch_adam(groups, n_groups, beta1, beta2, eps, step, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

// ---------------------------------------------------------------------------
// gs_bin_sort_noalloc: gs_bin_sort with its workspace in a fixed device array,
// for callers that cannot allocate device memory themselves.
namespace {

// The scratch. In host code this name is a host-side stand-in, not a device
// address: the address is looked up once per device with
// cudaGetSymbolAddress and passed to the kernels.
static __device__ __align__(256) unsigned char g_noalloc_scratch[GS_NOALLOC_SCRATCH_BYTES];

// Device address of the scratch on the current device, looked up on every
// call (a host-side query, cheap after the first one on a device): a cached
// address would go stale when a cudaDeviceReset rebuilds the context.
gs_status noalloc_scratch(void** addr) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return GS_ERR_CUDA;
  *addr = p;
  return GS_OK;
}

}  // namespace

extern "C" {

gs_status gs_bin_sort_noalloc(const gs_projected* proj, const gs_camera* cams, int32_t n_views,
                              int64_t n, int32_t sort_mode, gs_binned* out,
                              int32_t* device_status, void* stream) {
  if (!proj || !out) return GS_ERR_INVALID_ARG;
  const size_t need = gs_workspace_size(n, n_views, cams, out->pair_capacity, sort_mode);
  if (need == 0 || need > (size_t)GS_NOALLOC_SCRATCH_BYTES) return GS_ERR_INVALID_ARG;
  void* ws = nullptr;
  gs_status s = noalloc_scratch(&ws);
  if (s != GS_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the array keeps the previous call's contents: start from a clear status
  // word (gs_bin_sort clears the counters, histograms and look-back state it
  // relies on)
  if (cudaMemsetAsync(ws, 0, sizeof(uint32_t), st) != cudaSuccess) return GS_ERR_CUDA;
  s = gs_bin_sort(proj, cams, n_views, n, sort_mode, out, ws, GS_NOALLOC_SCRATCH_BYTES, stream);
  if (s != GS_OK) return s;
  if (device_status &&
      cudaMemcpyAsync(device_status, ws, sizeof(int32_t), cudaMemcpyDeviceToDevice, st) !=
          cudaSuccess)
    return GS_ERR_CUDA;
  return GS_OK;
}

gs_status gs_densify_params_from_cutoffs(double grad_threshold, double scale_split,
                                         double min_opacity, double max_scale,
                                         double split_shrink, gs_densify_params* out) {
  if (!out || !(scale_split > 0.0) || !(max_scale > 0.0) || !(split_shrink > 0.0) ||
      !(min_opacity > 0.0 && min_opacity < 1.0))
    return GS_ERR_INVALID_ARG;
  out->grad_threshold = (float)grad_threshold;
  out->log_scale_split = (float)std::log(scale_split);
  out->logit_min_opacity = (float)std::log(min_opacity / (1.0 - min_opacity));
  out->log_max_scale = (float)std::log(max_scale);
  out->log_split_shrink = (float)std::log(split_shrink);
  out->reserved = 0;
  return GS_OK;
}

size_t gs_densify_workspace_size(int64_t n) {
  if (n < 0 || n >= (1ll << 31)) return 0;
  size_t off = kControlBytes;
  off = align_up(off + (size_t)densify_blocks(n) * sizeof(uint32_t));
  off = align_up(off + (size_t)n);  // codes, when the caller passes none
  return off;
}

namespace {
// with_sh false: the SH block is not touched (quantised SH), its pointer is
// not needed
bool dp_tensors(const gs_grads* g, bool need, bool with_sh, gsb::DpTensorPtrs& t) {
  if (!g) return !need;
  t = gsb::DpTensorPtrs{g->means, g->log_scales, g->quats, g->opacity_logit,
                        with_sh ? g->sh : nullptr};
  return t.means && t.log_scales && t.quats && t.logit && (!with_sh || t.sh) &&
         aligned(t.means, 16) && aligned(t.log_scales, 16) && aligned(t.quats, 16) &&
         aligned(t.sh, 16);
}
}  // namespace

gs_status gs_densify_and_prune(const gs_params* in, const gs_grads* m_in, const gs_grads* v_in,
                               const float* accum, const int32_t* denom, const float* z,
                               const gs_densify_params* dp, gs_grads* out, gs_grads* m_out,
                               gs_grads* v_out, int64_t out_capacity, int64_t* n_out,
                               int8_t* codes, void* ws, size_t ws_bytes, void* stream) {
  if (!in || !dp || !n_out || !ws || !m_in || !v_in || !out || !m_out || !v_out)
    return GS_ERR_INVALID_ARG;
  if (in->n < 0 || in->sh_degree < 0 || in->sh_degree > 3 || out_capacity < 0)
    return GS_ERR_INVALID_ARG;
  if (in->n >= (1ll << 31) || out_capacity >= (1ll << 31)) return GS_ERR_OVERFLOW;
  const size_t need = gs_densify_workspace_size(in->n);
  if (ws_bytes < need || !aligned(ws, kAlign)) return GS_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int n = (int)in->n;
  if (n == 0) return cuda_status(cudaMemsetAsync(n_out, 0, sizeof(int64_t), st));
  gs_grads pin{const_cast<float*>(in->means), const_cast<float*>(in->log_scales),
               const_cast<float*>(in->quats), const_cast<float*>(in->opacity_logit),
               const_cast<float*>(in->sh)};
  // quantised SH: the SH blocks are gs_densify_sh_quant's, which needs the codes
  const bool with_sh = in->sh_quant == nullptr;
  if (!params_sh_ok(*in) || (!with_sh && !codes)) return GS_ERR_INVALID_ARG;
  gsb::DpTensorPtrs tp, tm, tv, op, om, ov;
  if (!dp_tensors(&pin, true, with_sh, tp) || !dp_tensors(m_in, true, with_sh, tm) ||
      !dp_tensors(v_in, true, with_sh, tv) || !dp_tensors(out, true, with_sh, op) ||
      !dp_tensors(m_out, true, with_sh, om) || !dp_tensors(v_out, true, with_sh, ov))
    return GS_ERR_INVALID_ARG;
  if (!accum || !denom || !z) return GS_ERR_INVALID_ARG;
  unsigned char* w = static_cast<unsigned char*>(ws);
  uint32_t* block_counts = reinterpret_cast<uint32_t*>(w + kControlBytes);
  int8_t* code_buf = codes ? codes
                           : reinterpret_cast<int8_t*>(
                                 w + align_up(kControlBytes + (size_t)densify_blocks(n) * 4));
  gsb::DensifyArgs a{dp->grad_threshold, dp->log_scale_split, dp->logit_min_opacity,
                     dp->log_max_scale, dp->log_split_shrink};
  const int k3 = with_sh ? 3 * (in->sh_degree + 1) * (in->sh_degree + 1) : 0;
  return cuda_status(gsb::launch_densify_and_prune(
      tp, tm, tv, accum, denom, z, n, k3, a, code_buf, block_counts, out_capacity, n_out,
      reinterpret_cast<uint32_t*>(w + kStatusOffset), op, om, ov, st));
}

size_t gs_l1_dssim_workspace_size(int32_t n_views) {
  if (n_views < 0) return 0;
  return (size_t)n_views * 2 * sizeof(double) + 16;
}

gs_status gs_l1_dssim(const float* image, const float* target, int32_t n_views, int32_t height,
                      int32_t width, float lambda, double* terms, float* dL_dimage, void* ws,
                      size_t ws_bytes, void* stream) {
  if (n_views < 0 || n_views > 21845) return GS_ERR_INVALID_ARG;
  if (n_views == 0) return GS_OK;
  if (height < 1 || width < 1 || height > 2097120) return GS_ERR_INVALID_ARG;
  if (!(lambda >= 0.f && lambda <= 1.f)) return GS_ERR_INVALID_ARG;
  if (!image || !target || !terms || !ws || !aligned(ws, 8) || !aligned(terms, 8))
    return GS_ERR_INVALID_ARG;
  if (!aligned(image, 4) || !aligned(target, 4) || (dL_dimage && !aligned(dL_dimage, 4)))
    return GS_ERR_INVALID_ARG;
  if (ws_bytes < gs_l1_dssim_workspace_size(n_views)) return GS_ERR_INVALID_ARG;
  double* sums = static_cast<double*>(ws);
  unsigned* done = reinterpret_cast<unsigned*>(sums + 2 * (size_t)n_views);
  return cuda_status(gsb::launch_l1_dssim(image, target, n_views, height, width, lambda, terms,
                                          dL_dimage, sums, done,
                                          static_cast<cudaStream_t>(stream)));
}

gs_status gs_sh_quantize(const float* sh, const gs_sh_quant* q, void* stream) {
  if (!quant_ok(q)) return GS_ERR_INVALID_ARG;
  if (q->n == 0) return GS_OK;
  if (!sh || !aligned(sh, 4)) return GS_ERR_INVALID_ARG;
  return cuda_status(gsb::launch_sh_quantize(sh, *q, static_cast<cudaStream_t>(stream)));
}

gs_status gs_sh_dequantize(const gs_sh_quant* q, float* sh, void* stream) {
  if (!quant_ok(q)) return GS_ERR_INVALID_ARG;
  if (q->n == 0) return GS_OK;
  if (!sh || !aligned(sh, 4)) return GS_ERR_INVALID_ARG;
  return cuda_status(gsb::launch_sh_dequantize(*q, sh, static_cast<cudaStream_t>(stream)));
}

gs_status gs_adam_step_sh_quant(const gs_sh_quant* q, const float* grad_sh, uint16_t* exp_avg,
                                uint16_t* exp_avg_sq, float lr, float beta1, float beta2,
                                float eps, int64_t step, int32_t rounding, uint64_t seed,
                                void* stream) {
  if (!quant_ok(q) || step < 1 || (rounding != 0 && rounding != 1)) return GS_ERR_INVALID_ARG;
  if (!(beta1 >= 0.f && beta1 < 1.f) || !(beta2 >= 0.f && beta2 < 1.f) || !(eps >= 0.f))
    return GS_ERR_INVALID_ARG;
  // packed blocks carry their moments; planar moments come beside the state
  const bool packed = q->layout == GS_QUANT_PACKED;
  if (packed ? (exp_avg || exp_avg_sq) : (q->n > 0 && (!exp_avg || !exp_avg_sq)))
    return GS_ERR_INVALID_ARG;
  if (q->n == 0) return GS_OK;
  if (!grad_sh || !aligned(grad_sh, 4) || !aligned(exp_avg, 8) || !aligned(exp_avg_sq, 8))
    return GS_ERR_INVALID_ARG;
  return cuda_status(gsb::launch_adam_sh_quant(*q, grad_sh, exp_avg, exp_avg_sq, lr, beta1, beta2,
                                               eps, step, rounding, seed,
                                               static_cast<cudaStream_t>(stream)));
}

size_t gs_densify_sh_quant_workspace_size(int64_t n_in, int64_t n_out) {
  if (n_in < 0 || n_in >= (1ll << 31) || n_out < 0 || n_out >= (1ll << 31)) return 0;
  size_t off = kControlBytes;
  off = align_up(off + (size_t)densify_blocks(n_in) * sizeof(uint32_t));  // block counts
  off = align_up(off + sizeof(int64_t));                                  // the map's count
  off = align_up(off + (size_t)n_out * sizeof(uint32_t));                 // output -> input
  return off;
}

gs_status gs_densify_sh_quant(const gs_sh_quant* in, const uint16_t* m_in, const uint16_t* v_in,
                              const int8_t* decisions, const gs_sh_quant* out, uint16_t* m_out,
                              uint16_t* v_out, void* ws, size_t ws_bytes, void* stream) {
  if (!quant_ok(in) || !quant_ok(out) || !ws || !aligned(ws, kAlign)) return GS_ERR_INVALID_ARG;
  if (in->k3 != out->k3 || in->bits != out->bits || in->layout != out->layout)
    return GS_ERR_INVALID_ARG;
  if (out->n > 2 * in->n) return GS_ERR_INVALID_ARG;
  const bool packed = in->layout == GS_QUANT_PACKED;
  if (packed ? (m_in || v_in || m_out || v_out)
             : (!m_in || !v_in || !m_out || !v_out || !aligned(m_in, 8) || !aligned(v_in, 8) ||
                !aligned(m_out, 8) || !aligned(v_out, 8)))
    return GS_ERR_INVALID_ARG;
  if (in->n > 0 && !decisions) return GS_ERR_INVALID_ARG;
  if (ws_bytes < gs_densify_sh_quant_workspace_size(in->n, out->n)) return GS_ERR_INVALID_ARG;
  if (in->n == 0) return out->n == 0 ? GS_OK : GS_ERR_INVALID_ARG;
  unsigned char* w = static_cast<unsigned char*>(ws);
  size_t off = kControlBytes;
  uint32_t* block_counts = reinterpret_cast<uint32_t*>(w + off);
  off = align_up(off + (size_t)densify_blocks(in->n) * sizeof(uint32_t));
  int64_t* n_out_dev = reinterpret_cast<int64_t*>(w + off);
  off = align_up(off + sizeof(int64_t));
  uint32_t* src = reinterpret_cast<uint32_t*>(w + off);
  return cuda_status(gsb::launch_densify_sh_quant(*in, m_in, v_in, decisions, *out, m_out, v_out,
                                                  block_counts, n_out_dev, src,
                                                  reinterpret_cast<uint32_t*>(w + kStatusOffset),
                                                  static_cast<cudaStream_t>(stream)));
}

gs_status gs_bin_sort_plan(int64_t n, int32_t n_views, const gs_camera* cams,
                           int32_t sort_mode, gs_sort_plan* plan) {
  Layout L;
  if (!plan || !make_layout(n, n_views, cams, 0, sort_mode, L)) return GS_ERR_INVALID_ARG;
  plan->path = L.tile_emit ? GS_PATH_TILES : (L.column_emit ? GS_PATH_COLUMNS : GS_PATH_TILE_ID);
  plan->presort_passes = sort_mode == GS_SORT_PRESORT ? L.presort.passes : 0;
  plan->pair_passes = L.tile_emit ? 0 : L.pairs.passes;
  plan->gaussians_per_block = L.tile_emit ? L.gsize : 0;
  plan->pair_single_sweep = pair_passes_single_sweep(L.pairs, sort_mode) ? 1 : 0;
  plan->ranges_from_counts = L.count_ranges ? 1 : 0;
  plan->pair_key_bytes = L.tile_emit ? 0 : L.key_bytes;
  plan->reserved = 0;
  plan->blocks_per_view = L.tile_emit ? L.tile_bpv : 0;
  return GS_OK;
}

gs_status gs_debug_stall(int32_t site, int64_t index, double wait_limit_s) {
  if (site < GS_STALL_NONE || site > GS_STALL_SORT_LOOKBACK) return GS_ERR_INVALID_ARG;
  if (!(wait_limit_s >= 0.0) || wait_limit_s > 60.0) return GS_ERR_INVALID_ARG;
  if (site != GS_STALL_NONE && index < 0) return GS_ERR_INVALID_ARG;
  g_stall_site.store(GS_STALL_NONE);
  g_stall_index.store(site == GS_STALL_NONE ? -1 : index);
  g_wait_ns.store((uint64_t)std::llround(wait_limit_s * 1e9));
  g_stall_site.store(site);
  return GS_OK;
}

gs_status gs_get_status(void* ws, void* stream) {
  if (!ws) return GS_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return GS_ERR_CUDA;
  uint32_t word = 0;
  unsigned char* w = static_cast<unsigned char*>(ws);
  if (cudaMemcpy(&word, w + kStatusOffset, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
    return GS_ERR_CUDA;
  if (cudaMemset(w + kStatusOffset, 0, sizeof(uint32_t)) != cudaSuccess) return GS_ERR_CUDA;
  if (word & kStatusTimeout) return GS_ERR_DEVICE_TIMEOUT;
  if (word & kStatusBounds) return GS_ERR_OVERFLOW;
  if (word & kStatusCapacity) return GS_ERR_CAPACITY;
  if (word & kStatusNonfinite) return GS_ERR_NONFINITE;
  return GS_OK;
}

}  // extern "C"
