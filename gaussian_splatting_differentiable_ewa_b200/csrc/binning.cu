// binning.cu -- tile binning with depth sort, sm_100a.
//
// Assign every projected Gaussian to the 16x16 tiles its 3-sigma rectangle
// touches and order each tile's list by depth ("Better Gaussian Splatting in
// Julia", pwwt.cn sec. 3.3 steps 1-2 and 4.3; lshu.cn sec. 3.2
// assign_to_tiles / sort_by_depth!), ties broken by Gaussian index.
//
//  k_depth_keys    (presort mode) per-Gaussian (view, depth) keys.
//  k_emit          one pass over the Gaussians: pair counts, a single-pass
//                  scan across blocks (decoupled look-back, one warp reading
//                  32 predecessors per round trip) and emission of the
//                  (key, id) pairs through shared-memory staging.
//  k_tile_count / k_tile_base / k_emit_tiles
//                  (presort mode, tile grids up to ~40k tiles) every pair
//                  straight to its final position: per (Gaussian block,
//                  tile) counts from a 2-D difference array, their scans over
//                  blocks and over tiles (which are also the ranges), then
//                  one warp per (block, 32 x 16 tile region) streams the
//                  block's rectangles in depth order and writes each pair at
//                  its tile's next position.
//  k_col_count / k_emit_cols
//                  (presort mode, up to 256 tile columns) emission already
//                  ordered by tile column: per-block column counts from a
//                  difference array, their scan, then lanes owning columns
//                  append their pairs in depth order through shared-memory
//                  buffers written out warp-wide. The radix passes then sort
//                  by row alone; the keys are the row in one or two bytes
//                  when the ranges come from the tile counts, else
//                  row << cbits | column.
//  k_tile_hist / k_tile_ranges
//                  (column path and full-64 mode, grids whose per-view tile
//                  counters fit a block) every tile's pair count from a
//                  per-view 2-D difference array of the rectangles' corners,
//                  and a scan of the counts per view: the ranges before the
//                  pairs exist, so nothing reads the sorted keys.
//  k_digit_hist / k_onesweep
//                  the 64-bit sorts (depth presort; full-64 pair keys): a
//                  stable least-significant-digit radix sort with 8-bit
//                  digits, single-sweep. One read of the keys counts the
//                  digits of every pass; each pass is then one kernel whose
//                  partitions (taken in launch order by a ticket) rank their
//                  keys stably in shared memory and find their global
//                  offsets by decoupled look-back over the partitions before
//                  them, one thread per digit.
//  k_radix_count / k_radix_scan / k_radix_scatter
//                  the 8-, 16- and 32-bit sorts (row or tile bits after
//                  column or tile-id emission), reduce-then-scan: per-partition digit
//                  counts, a per-digit scan over partitions (with the digit
//                  totals), then a scatter that ranks each partition's keys
//                  stably (ballots over warp-striped steps), stages them in
//                  shared memory and writes runs of equal digits. The bits
//                  are split evenly over the fewest passes (13 bits: 7 + 6),
//                  so each key costs one ballot per bit of its pass.
//  k_ranges        [start, end) of each tile in the sorted pairs (where the
//                  tile counts do not give them).
// Look-back waits (emission and single-sweep passes) are bounded in time
// (WaitCfg) and report through the status word instead of hanging; the
// reduce-then-scan passes never wait on other blocks.

#include <cuda_runtime.h>

#include "gs_internal.h"

namespace gsb {
namespace {

constexpr int kEmitThreads = 256;
constexpr int kEmitItemsPerThread = 4;
constexpr int kEmitItems = kEmitThreads * kEmitItemsPerThread;

constexpr int kSortThreads = 256;
constexpr int kSortWarps = kSortThreads / 32;
constexpr int kSortItems = 16;                        // pair passes
constexpr int kSortTile = kSortThreads * kSortItems;  // keys per partition
constexpr int kPresortItems = 16;                     // per-Gaussian depth passes
constexpr int kColItems = 256;     // Gaussians per column-emission block
constexpr int kColBuf = 32;        // pairs a column stages before a warp-wide write
constexpr int kColStage = 128;     // rectangles a column-emission warp compacts at a time
constexpr int kMaxColumns = 256;   // widest tile grid the column emission takes
constexpr int kColPitch = 33;      // buffer row: conflict-free along and across columns
constexpr int kRegionCols = 32;    // tile-emission region: kRegionCols x kRegionRows tiles
constexpr int kRegionRows = 16;
constexpr int kEmitWarps = 2;      // tile-emission regions (one per warp) per block
// tile emission: rectangle batches loaded ahead of the one being placed. A
// batch without a hit takes far less than a load's latency; small scenes'
// rectangles stay in L2 (2 ahead suffice), large ones come from DRAM: 12
// ahead measured 17.6 against 20.0 ms for the 6M x 8-view binning (16 ahead
// lowers occupancy and is slower again).
constexpr int kEmitAheadL2 = 2, kEmitAheadDram = 12;
constexpr int kTileDiffBytes = 160 * 1024;  // largest tile-count difference array

__device__ __forceinline__ uint32_t get_block_index(uint32_t* counter) {
  __shared__ uint32_t s_idx;
  if (threadIdx.x == 0) s_idx = atomicAdd(counter, 1u);
  __syncthreads();
  return s_idx;
}

// Exclusive block-wide scan of one uint32 per thread (256 threads).
__device__ __forceinline__ uint32_t block_exclusive_scan_256(uint32_t x, uint32_t* s_warp,
                                                             uint32_t& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = lane < 8 ? s_warp[lane] : 0u;
    uint32_t wi = w;
#pragma unroll
    for (int o = 1; o < 8; o <<= 1) {
      uint32_t y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += y;
    }
    if (lane < 8) s_warp[lane] = wi - w;  // exclusive warp offsets
    if (lane == 7) s_warp[8] = wi;        // block total
  }
  __syncthreads();
  total = s_warp[8];
  uint32_t r = s_warp[warp] + incl - x;
  __syncthreads();
  return r;
}

// Decoupled look-back for one value per block, run by warp 0 of the block.
// Publishes the block aggregate, then the warp reads 32 predecessors per
// round trip and sums them back to the nearest inclusive prefix; publishes
// the block's inclusive prefix and returns the exclusive prefix (to all lanes
// of warp 0).
// A block whose index is wc.stall (a test hook) publishes nothing, so the
// waits of its successors run out.
__device__ uint64_t warp_block_lookback(uint64_t* lb, uint32_t idx, uint64_t aggregate,
                                        uint32_t* status, const WaitCfg& wc) {
  const int lane = threadIdx.x & 31;
  const bool publish = (int64_t)idx != wc.stall;
  if (idx == 0) {
    if (lane == 0 && publish) st_relaxed_u64(&lb[0], kLbPrefix | aggregate);
    return 0;
  }
  if (lane == 0 && publish) st_relaxed_u64(&lb[idx], kLbAggregate | aggregate);
  uint64_t excl = 0;
  int64_t base = (int64_t)idx - 1;
  while (true) {
    const int64_t j = base - lane;
    uint64_t w = j >= 0 ? ld_relaxed_u64(&lb[j]) : kLbPrefix;
    if ((w >> 62) == 0) w = lookback_wait(&lb[j], wc.limit_ns, status);
    const uint32_t pre = __ballot_sync(0xffffffffu, (w >> 62) == 2);
    const int first = pre ? __ffs(pre) - 1 : 32;  // nearest inclusive prefix
    uint64_t val = lane <= first ? (w & kLbValueMask) : 0ull;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) val += __shfl_xor_sync(0xffffffffu, val, o);
    excl += val;
    if (pre) break;
    base -= 32;
  }
  if (lane == 0 && publish) st_relaxed_u64(&lb[idx], kLbPrefix | (excl + aggregate));
  return excl;
}

template <typename K>
struct KeyTraits;
template <>
struct KeyTraits<uint64_t> {
  static constexpr int kBits = 64;
};
template <>
struct KeyTraits<uint32_t> {
  static constexpr int kBits = 32;
};

// ---------------------------------------------------------------------------
// Presort keys: (view << 32 | depth bits) for visible Gaussians, all ones for
// culled ones, value = Gaussian index within its view.
__global__ void __launch_bounds__(256) k_depth_keys(const float4* __restrict__ bins, int n,
                                                   int n_views, uint64_t* __restrict__ keys,
                                                   uint32_t* __restrict__ vals,
                                                   int64_t* __restrict__ n_items_out,
                                                   uint32_t* __restrict__ n_visible,
                                                   uint32_t* __restrict__ status) {
  __shared__ uint32_t s_vis[GS_MAX_VIEWS];
  if (threadIdx.x < GS_MAX_VIEWS) s_vis[threadIdx.x] = 0u;
  __syncthreads();
  if (blockIdx.x == 0 && threadIdx.x == 0) *n_items_out = (int64_t)n * n_views;
  const int64_t total = (int64_t)n * n_views;
  for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < total;
       j += (int64_t)gridDim.x * blockDim.x) {
    const float4 r2 = __ldg(&bins[j]);  // depth key, tile_x, tile_y
    if (__float_as_uint(r2.x) == kNonfiniteKeyBits) atomicOr(status, kStatusNonfinite);
    const uint32_t txw = __float_as_uint(r2.y), tyw = __float_as_uint(r2.z);
    const bool vis = (txw & 0xffffu) <= (txw >> 16) && (tyw & 0xffffu) <= (tyw >> 16);
    const int view = (int)(j / n);
    keys[j] = vis ? (((uint64_t)view << 32) | (uint64_t)__float_as_uint(r2.x)) : ~0ull;
    vals[j] = (uint32_t)(j - (int64_t)view * n);
    if (vis) atomicAdd(&s_vis[view], 1u);
  }
  __syncthreads();
  if (threadIdx.x < n_views && s_vis[threadIdx.x]) atomicAdd(&n_visible[threadIdx.x], s_vis[threadIdx.x]);
}

// ---------------------------------------------------------------------------
// Tile emission (presort mode, tile grids whose difference array fits in
// shared memory). Every pair goes straight to its final position:
// view v's presorted Gaussians are cut into blocks of `gsize`; for block b and
// tile t, cnt(t, b) = number of the block's rectangles covering t. A scan
// over b (per tile) and one over t give pair (t, Gaussian g of block b) the
// position base(t) + sum_{b' < b} cnt(t, b') + (rank of g among the block's
// Gaussians covering t), which is depth order within the tile -- the order
// of the stable (tile, depth) sort -- and the ranges are the scans
// themselves. No pair keys, no sort of the pairs.

// Rectangle of presorted item `item`; false for a culled or empty one.
__device__ __forceinline__ bool presorted_rect(const float4* __restrict__ bins,
                                               const uint64_t* __restrict__ pkeys,
                                               const uint32_t* __restrict__ pvals, int n,
                                               int64_t item, uint32_t& rx, uint32_t& ry,
                                               uint32_t& view, uint32_t& id) {
  const uint64_t pk = pkeys[item];
  if (pk == ~0ull) return false;
  view = (uint32_t)(pk >> 32);
  id = pvals[item];
  const float4 r2 = __ldg(&bins[(int64_t)view * n + id]);
  rx = __float_as_uint(r2.y);  // x0 | x1 << 16
  ry = __float_as_uint(r2.z);  // y0 | y1 << 16
  return (rx & 0xffffu) <= (rx >> 16) && (ry & 0xffffu) <= (ry >> 16);
}

// Count table entry of (global tile t, Gaussian block b): groups of 8 tiles,
// block-major inside a group, so a block writes 8 neighbouring tiles' counts
// as one 32-byte run and a group's entries over all blocks are contiguous.
__device__ __forceinline__ int64_t tcount_index(int64_t t, int64_t b, int64_t stride) {
  return ((t >> 3) * stride + b) * 8 + (t & 7);
}

// Start of view v's visible Gaussians in the presorted order (sorted by
// (view, depth) with culled ones last) and their number.
__device__ __forceinline__ void view_span(const uint32_t* __restrict__ n_visible, int v,
                                          int64_t& start, int64_t& count) {
  int64_t s0 = 0;
  for (int u = 0; u < v; ++u) s0 += n_visible[u];
  start = s0;
  count = n_visible[v];
}

// (1) cnt(t, b) for block (b, v): a 2-D difference array over the view's
// tile grid (+1 / -1 at the rectangle's four corners), summed along rows then
// columns. Also the packed rectangles (x0 | x1 << 16, y0 | y1 << 16, 0, id)
// for the emission and the exact pair total. Grid (blocks per view, views).
__global__ void __launch_bounds__(256) k_tile_count(
    const float4* __restrict__ bins, const uint64_t* __restrict__ pkeys,
    const uint32_t* __restrict__ pvals, int n, Grid g, int gsize,
    const uint32_t* __restrict__ n_visible, uint32_t* __restrict__ counts, int64_t stride,
    unsigned long long* __restrict__ pair_total, uint4* __restrict__ crect,
    int64_t* __restrict__ scan_n) {
  extern __shared__ int s_d[];  // [tiles_y + 1][tiles_x + 1]
  __shared__ unsigned long long s_tot[8];
  const int v = blockIdx.y, b = blockIdx.x;
  if (b == 0 && v == 0 && threadIdx.x == 0) *scan_n = gridDim.x;
  int64_t vs, nv;
  view_span(n_visible, v, vs, nv);
  const int64_t first = vs + (int64_t)b * gsize;
  const int64_t last = min(vs + nv, first + gsize);
  const int W = g.tiles_x + 1, H = g.tiles_y + 1;
  for (int k = threadIdx.x; k < W * H; k += 256) s_d[k] = 0;
  __syncthreads();
  uint64_t mine = 0;
  // four items per thread at a time: all their loads issue before any use
  for (int64_t base = first + threadIdx.x; base < last; base += 4 * 256) {
    uint64_t pk[4];
    uint32_t id[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t item = base + u * 256;
      pk[u] = item < last ? pkeys[item] : ~0ull;
      id[u] = item < last ? pvals[item] : 0u;
    }
    float4 r2[4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      r2[u] = pk[u] != ~0ull ? __ldg(&bins[(int64_t)(pk[u] >> 32) * n + id[u]])
                             : make_float4(0.f, __uint_as_float(1u), 0.f, 0.f);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t item = base + u * 256;
      if (item >= last) break;
      const uint32_t rx = __float_as_uint(r2[u].y), ry = __float_as_uint(r2[u].z);
      const int x0 = rx & 0xffffu, x1 = rx >> 16, y0 = ry & 0xffffu, y1 = ry >> 16;
      if (x0 <= x1 && y0 <= y1) {
        atomicAdd(&s_d[y0 * W + x0], 1);
        atomicAdd(&s_d[y0 * W + x1 + 1], -1);
        atomicAdd(&s_d[(y1 + 1) * W + x0], -1);
        atomicAdd(&s_d[(y1 + 1) * W + x1 + 1], 1);
        mine += (uint64_t)(x1 - x0 + 1) * (uint64_t)(y1 - y0 + 1);
        crect[item] = make_uint4(rx, ry, 0u, id[u]);
      } else {
        crect[item] = make_uint4(1u, 0u, 0u, 0u);  // empty: x0 > x1
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mine += __shfl_xor_sync(0xffffffffu, mine, o);
  if ((threadIdx.x & 31) == 0) s_tot[threadIdx.x >> 5] = mine;
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned long long t = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) t += s_tot[w];
    if (t) atomicAdd(pair_total, t);
  }
  // running sums along each row, then down each column
  for (int r = threadIdx.x; r < H - 1; r += 256) {
    int acc = 0;
    for (int c = 0; c < W - 1; ++c) {
      acc += s_d[r * W + c];
      s_d[r * W + c] = acc;
    }
  }
  __syncthreads();
  for (int c = threadIdx.x; c < W - 1; c += 256) {
    int acc = 0;
    for (int r = 0; r < H - 1; ++r) {
      acc += s_d[r * W + c];
      s_d[r * W + c] = acc;
    }
  }
  __syncthreads();
  const int tpv = g.tiles_per_view;
  for (int t = threadIdx.x; t < tpv; t += 256) {
    const int r = t / g.tiles_x, c = t - r * g.tiles_x;
    counts[tcount_index((int64_t)v * tpv + t, b, stride)] = (uint32_t)s_d[r * W + c];
  }
}

// (2a) per tile: exclusive scan of cnt(t, b) over the blocks b, in place, and
// the tile's total. One block per group of 8 tiles; thread i takes blocks
// i, i + 256, ... with the group's 8 counts of a block in two 16-byte loads,
// scanning the 8 tiles side by side.
__global__ void __launch_bounds__(256) k_tile_scan(uint32_t* __restrict__ counts, int64_t stride,
                                                  int bpv, int64_t n_tiles,
                                                  uint32_t* __restrict__ totals) {
  __shared__ uint32_t s_w[8][9];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t g = blockIdx.x;
  uint4* grp = reinterpret_cast<uint4*>(counts + g * stride * 8);
  uint32_t carry[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  for (int b0 = 0; b0 < bpv; b0 += 256) {
    const int b = b0 + (int)threadIdx.x;
    uint32_t x[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (b < bpv) {
      const uint4 lo = grp[2 * b], hi = grp[2 * b + 1];
      x[0] = lo.x; x[1] = lo.y; x[2] = lo.z; x[3] = lo.w;
      x[4] = hi.x; x[5] = hi.y; x[6] = hi.z; x[7] = hi.w;
    }
    uint32_t inc[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) inc[k] = x[k];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, inc[k], o);
        if (lane >= o) inc[k] += y;
      }
    }
    if (lane == 31) {
#pragma unroll
      for (int k = 0; k < 8; ++k) s_w[warp][k] = inc[k];
    }
    __syncthreads();
    uint32_t before[8], chunk[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      uint32_t pre = 0, all = 0;
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        const uint32_t s = s_w[w][k];
        pre += w < warp ? s : 0u;
        all += s;
      }
      before[k] = pre;
      chunk[k] = all;
    }
    if (b < bpv) {
      uint32_t o[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) o[k] = carry[k] + before[k] + inc[k] - x[k];
      grp[2 * b] = make_uint4(o[0], o[1], o[2], o[3]);
      grp[2 * b + 1] = make_uint4(o[4], o[5], o[6], o[7]);
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) carry[k] += chunk[k];
    __syncthreads();
  }
  if (threadIdx.x < 8) {
    const int64_t t = g * 8 + threadIdx.x;
    uint32_t c = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) c = k == (int)threadIdx.x ? carry[k] : c;
    if (t < n_tiles) totals[t] = c;
  }
}

// (2b) base(t): exclusive scan of the tile totals over all tiles (one block),
// the ranges, the pair count and the capacity check.
__global__ void __launch_bounds__(1024) k_tile_base(
    const uint32_t* __restrict__ tile_totals, int64_t n_tiles,
    const unsigned long long* __restrict__ pair_total, int64_t capacity,
    uint32_t* __restrict__ tile_base, int64_t* __restrict__ ranges, int64_t* __restrict__ n_pairs,
    uint32_t* __restrict__ status) {
  __shared__ uint32_t s_w[32];
  const unsigned long long total = *pair_total;
  if (threadIdx.x == 0) {
    *n_pairs = (int64_t)total;
    if ((int64_t)total > capacity) atomicOr(status, kStatusCapacity);
  }
  if ((int64_t)total > capacity) return;  // every range stays empty
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t carry = 0;
  for (int64_t base = 0; base < n_tiles; base += 1024) {
    const int64_t t = base + threadIdx.x;
    const uint32_t x = t < n_tiles ? tile_totals[t] : 0u;
    uint32_t incl = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) s_w[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const uint32_t w = s_w[lane];
      uint32_t wi = w;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, wi, o);
        if (lane >= o) wi += y;
      }
      s_w[lane] = wi - w;
    }
    __syncthreads();
    const uint32_t start = carry + s_w[warp] + incl - x;
    if (t < n_tiles) {
      tile_base[t] = start;
      ranges[2 * t] = start;
      ranges[2 * t + 1] = (int64_t)start + x;
    }
    __syncthreads();
    if (threadIdx.x == 1023) s_w[0] = start + x;  // carry into the next chunk
    __syncthreads();
    carry = s_w[0];
    __syncthreads();
  }
}

// (3) emission. Each warp of block (b, ., v) places Gaussian block b's pairs
// in one region of kRegionCols x kRegionRows tiles. Every tile of the
// region keeps the position of its next pair in shared memory (base(t) plus
// the pairs earlier blocks put there); the warp streams the block's
// rectangles in depth order, 32 per coalesced load, and for each one that
// reaches the region writes its pairs at once, one lane per tile (a rectangle
// has one pair per tile, so no two lanes share a counter), straight to their
// final positions. The counters' rows are padded by one word so that the
// tiles of a rectangle's column sit in different banks.
constexpr int kNextPitch = kRegionCols + 1;
template <int kEmitAhead>
__global__ void __launch_bounds__(32 * kEmitWarps) k_emit_tiles(
    const uint4* __restrict__ crect, int gsize, const uint32_t* __restrict__ n_visible, Grid g,
    int n_regions, const uint32_t* __restrict__ offsets, int64_t stride,
    const uint32_t* __restrict__ tile_base, const unsigned long long* __restrict__ pair_total,
    uint32_t* __restrict__ ids_out, int64_t capacity, uint32_t* __restrict__ status) {
  constexpr int kTiles = kRegionCols * kRegionRows;
  __shared__ uint32_t s_next_all[kEmitWarps][kRegionRows * kNextPitch];
  if ((int64_t)*pair_total > capacity) return;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int region = blockIdx.y * kEmitWarps + warp;  // warps of a block: regions side by side
  if (region >= n_regions) return;
  uint32_t* s_next = s_next_all[warp];
  const int v = blockIdx.z, b = blockIdx.x;
  const int ncg = (g.tiles_x + kRegionCols - 1) / kRegionCols;
  const int c0 = kRegionCols * (region % ncg), r0 = kRegionRows * (region / ncg);
  const int c1 = min(c0 + kRegionCols, g.tiles_x) - 1, r1 = min(r0 + kRegionRows, g.tiles_y) - 1;
  int64_t vs, nv;
  view_span(n_visible, v, vs, nv);
  const int64_t first = vs + (int64_t)b * gsize;
  const int64_t last = min(vs + nv, first + gsize);
  if (first >= last) return;
  const int tpv = g.tiles_per_view;
  for (int li = lane; li < kTiles; li += 32) {
    const int rr = li / kRegionCols, cc = li % kRegionCols;
    const int r = r0 + rr, c = c0 + cc;
    uint32_t next = 0;
    if (r <= r1 && c <= c1) {
      const int64_t t = (int64_t)v * tpv + (int64_t)r * g.tiles_x + c;
      next = tile_base[t] + offsets[tcount_index(t, b, stride)];
    }
    s_next[rr * kNextPitch + cc] = next;
  }
  __syncwarp();
  // a ring of kEmitAhead batches of rectangles in flight while one is placed
  uint4 q[kEmitAhead];
#pragma unroll
  for (int k = 0; k < kEmitAhead; ++k) {
    q[k] = make_uint4(1u, 0u, 0u, 0u);
    if (first + 32 * k + lane < last) q[k] = crect[first + 32 * k + lane];
  }
  for (int64_t i0 = first; i0 < last; i0 += 32) {
    const uint4 cur = q[0];
#pragma unroll
    for (int k = 0; k + 1 < kEmitAhead; ++k) q[k] = q[k + 1];
    q[kEmitAhead - 1] = make_uint4(1u, 0u, 0u, 0u);
    if (i0 + 32 * kEmitAhead + lane < last) q[kEmitAhead - 1] = crect[i0 + 32 * kEmitAhead + lane];
    const int x0 = cur.x & 0xffffu, x1 = cur.x >> 16, y0 = cur.y & 0xffffu, y1 = cur.y >> 16;
    uint32_t hits = __ballot_sync(0xffffffffu,
                                  x0 <= x1 && x1 >= c0 && x0 <= c1 && y1 >= r0 && y0 <= r1);
    while (hits) {
      const int L = __ffs(hits) - 1;
      hits &= hits - 1;
      const uint32_t rx = __shfl_sync(0xffffffffu, cur.x, L);
      const uint32_t ry = __shfl_sync(0xffffffffu, cur.y, L);
      const uint32_t id = __shfl_sync(0xffffffffu, cur.w, L);
      const int cx0 = max((int)(rx & 0xffffu), c0), cx1 = min((int)(rx >> 16), c1);
      const int ry0 = max((int)(ry & 0xffffu), r0), ry1 = min((int)(ry >> 16), r1);
      const int wp = cx1 - cx0 + 1;
      const int np = wp * (ry1 - ry0 + 1);
      const float inv_wp = 1.f / (float)wp;
      for (int p0 = 0; p0 < np; p0 += 32) {
        const int p = p0 + lane;
        if (p < np) {
          const int rr = min((int)(((float)p + 0.5f) * inv_wp), ry1 - ry0);
          const int cc = p - rr * wp;
          const int li = (ry0 - r0 + rr) * kNextPitch + (cx0 - c0 + cc);
          const uint32_t pos = s_next[li];
          s_next[li] = pos + 1;
          if ((int64_t)pos < capacity) ids_out[pos] = id;
          else atomicOr(status, kStatusBounds);
        }
      }
      __syncwarp();
    }
  }
}

// ---------------------------------------------------------------------------
// Column emission (presort mode, images up to kMaxColumns tiles wide).
// A pair's key is row << cbits | column, row = view * tiles_y + tile row:
// ordering by it is ordering by global tile. The emission hands out pairs
// already ordered by column (stable in depth order), which is the first
// least-significant-digit pass of that order; the radix passes that follow
// sort by row only.

// (1) pairs per tile column of each block of kColItems presorted Gaussians:
// a difference array over columns weighted by the rectangle's height, then a
// prefix over the columns. Also adds the block's pairs to the 64-bit total.
__global__ void __launch_bounds__(kColItems) k_col_count(
    const float4* __restrict__ bins, const uint64_t* __restrict__ pkeys,
    const uint32_t* __restrict__ pvals, int n, int n_views, Grid g, uint32_t* __restrict__ counts,
    int64_t stride, unsigned long long* __restrict__ pair_total, uint4* __restrict__ crect) {
  __shared__ int s_diff[kMaxColumns + 1];
  __shared__ uint32_t s_warp[9];
  const int64_t items = (int64_t)n * n_views;
  for (int c = threadIdx.x; c <= kMaxColumns; c += kColItems) s_diff[c] = 0;
  __syncthreads();
  const int64_t item = (int64_t)blockIdx.x * kColItems + threadIdx.x;
  uint32_t rx, ry, view, id;
  uint64_t mine = 0;
  if (item < items) {
    if (presorted_rect(bins, pkeys, pvals, n, item, rx, ry, view, id)) {
      const int h = (int)((ry >> 16) - (ry & 0xffffu) + 1);
      atomicAdd(&s_diff[rx & 0xffffu], h);
      atomicAdd(&s_diff[(rx >> 16) + 1], -h);
      mine = (uint64_t)h * ((rx >> 16) - (rx & 0xffffu) + 1);
      crect[item] = make_uint4(rx, ry, view * (uint32_t)g.tiles_y, id);
    } else {
      crect[item] = make_uint4(1u, 0u, 0u, 0u);  // empty: x0 > x1
    }
  }
  // the block's pair total: warp sums, then one 64-bit atomic per block
  __shared__ unsigned long long s_tot[kColItems / 32];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mine += __shfl_xor_sync(0xffffffffu, mine, o);
  if ((threadIdx.x & 31) == 0) s_tot[threadIdx.x >> 5] = mine;
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned long long b = 0;
#pragma unroll
    for (int w = 0; w < kColItems / 32; ++w) b += s_tot[w];
    if (b) atomicAdd(pair_total, b);
  }
  const int t = threadIdx.x;
  const int d = t < g.tiles_x ? s_diff[t] : 0;
  uint32_t tot;
  const uint32_t excl = block_exclusive_scan_256((uint32_t)d, s_warp, tot);
  if (t < g.tiles_x) counts[(int64_t)t * stride + blockIdx.x] = excl + (uint32_t)d;
}

// (3) emission. Block (b, w) -- one warp -- takes Gaussian block b's pairs in
// tile columns 32w .. 32w + 31; lane l owns column 32w + l (its buffer and
// its next global position). The warp compacts the block's Gaussians to those
// whose rectangle reaches its columns (depth order kept) and walks them,
// writing a rectangle's pairs at once, one lane per (row, column) pair, each
// into its column's buffer in shared memory after the pairs already there. A
// column whose buffer cannot take the rectangle's rows is first written out
// by the whole warp to the column's next global positions (coalesced), so a
// column's pairs leave in depth order. One warp per block lets the scheduler
// balance column groups of very different load (the image centre against its
// edges). offsets: [column][block] exclusive scans over blocks; totals: pairs
// per column; crect: the presorted rectangles (x0 | x1 << 16, y0 | y1 << 16,
// first row of the view, Gaussian index).

// Warp-wide write of the first `count` (<= 32) pairs of buffer column `bc`
// to global positions base, base + 1, ...
template <typename KT>
__device__ __forceinline__ void flush_column(KT* __restrict__ keys_out,
                                             uint32_t* __restrict__ ids_out, int64_t capacity,
                                             const KT* s_bk, const uint32_t* s_bi, int bc,
                                             uint32_t base, uint32_t count,
                                             uint32_t* __restrict__ status) {
  const uint32_t lane = threadIdx.x & 31;
  if (lane < count) {
    const uint32_t pos = base + lane;
    if ((int64_t)pos < capacity) {
      keys_out[pos] = s_bk[lane * kColPitch + bc];
      ids_out[pos] = s_bi[lane * kColPitch + bc];
    } else {
      atomicOr(status, kStatusBounds);
    }
  }
}

// KT: the key type. 32 bits: row << cbits | column (the ranges are then read
// off the sorted keys); 8 or 16 bits: the row alone, when the ranges come
// from the tile counts and only the rows pass reads the keys.
template <typename KT>
__global__ void __launch_bounds__(32) k_emit_cols(
    const uint4* __restrict__ crect, int64_t items, Grid g, int cbits,
    const uint32_t* __restrict__ offsets, int64_t stride, const uint32_t* __restrict__ totals,
    const unsigned long long* __restrict__ pair_total, KT* __restrict__ keys_out,
    uint32_t* __restrict__ ids_out, int64_t capacity, int64_t* __restrict__ n_pairs,
    uint32_t* __restrict__ status) {
  // keys buffered at their own width: narrow keys leave room for more blocks
  // per SM (one-byte keys: 9.4 KB a block against 12.5 KB)
  __shared__ KT s_bk[kColBuf * kColPitch];
  __shared__ uint32_t s_bi[kColBuf * kColPitch];
  __shared__ uint4 s_rect[kColStage];  // this warp's rectangles, compacted
  const int lane = threadIdx.x;
  const unsigned long long total = *pair_total;
  if (blockIdx.x == 0 && blockIdx.y == 0 && lane == 0) {
    *n_pairs = (int64_t)total;
    if ((int64_t)total > capacity) atomicOr(status, kStatusCapacity);
  }
  if ((int64_t)total > capacity) return;  // nothing is emitted
  const uint32_t wlo = 32u * blockIdx.y, col = wlo + (uint32_t)lane;
  // first position of this block's pairs in column col: pairs of lower
  // columns plus column col's pairs from earlier blocks
  uint32_t below = 0;
  for (uint32_t c = (uint32_t)lane; c < wlo; c += 32) below += totals[c];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) below += __shfl_xor_sync(0xffffffffu, below, o);
  uint32_t tot_c = col < (uint32_t)g.tiles_x ? totals[col] : 0u;
  uint32_t incl = tot_c;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  uint32_t gofs = below + incl - tot_c;
  if (col < (uint32_t)g.tiles_x) gofs += offsets[(int64_t)col * stride + blockIdx.x];
  const uint32_t lt = lanemask_lt();
  const int64_t first = (int64_t)blockIdx.x * kColItems;
  uint32_t fill = 0;
  // the block's rectangles kColStage at a time (a smaller staging buffer, more
  // blocks per SM): compact those that reach columns wlo .. wlo + 31, in
  // depth order, then place their pairs
  for (int stage = 0; stage < kColItems; stage += kColStage) {
    int cnt = 0;
    __syncwarp();  // the previous stage's rectangles are read
#pragma unroll 2
    for (int c = 0; c < kColStage / 32; ++c) {
      const int64_t item = first + stage + c * 32 + lane;
      uint4 r = make_uint4(1u, 0u, 0u, 0u);
      if (item < items) r = crect[item];
      const uint32_t x0 = r.x & 0xffffu, x1 = r.x >> 16;
      const bool hit = x0 <= x1 && x1 >= wlo && x0 <= wlo + 31u;
      const uint32_t bal = __ballot_sync(0xffffffffu, hit);
      if (hit) s_rect[cnt + __popc(bal & lt)] = r;
      cnt += __popc(bal);
    }
    __syncwarp();
    for (int k = 0; k < cnt; ++k) {
      const uint4 r = s_rect[k];
      // this warp's columns of the rectangle
      const uint32_t cx0 = max(r.x & 0xffffu, wlo);
      const uint32_t cx1 = min(r.x >> 16, wlo + 31u);
      const uint32_t wp = cx1 - cx0 + 1;
      const float inv_wp = 1.f / (float)wp;
      const bool owner = col >= cx0 && col <= cx1;
      const uint32_t y0 = r.y & 0xffffu, h = (r.y >> 16) - y0 + 1;
      const uint32_t row0 = r.z + y0;
      for (uint32_t r0 = 0; r0 < h; r0 += kColBuf) {  // row chunks, uniform across the warp
        const uint32_t hc = min(h - r0, (uint32_t)kColBuf);
        // make room: columns that cannot take hc more pairs are written out
        uint32_t need = __ballot_sync(0xffffffffu, owner && fill + hc > kColBuf);
        if (need) {
          __syncwarp();
          do {
            const int L = __ffs(need) - 1;
            need &= need - 1;
            flush_column(keys_out, ids_out, capacity, s_bk, s_bi, L,
                         __shfl_sync(0xffffffffu, gofs, L), __shfl_sync(0xffffffffu, fill, L),
                         status);
            if (lane == L) {
              gofs += fill;
              fill = 0;
            }
          } while (need);
          __syncwarp();
        }
        // the chunk's wp * hc pairs, 32 at a time: pair p is row p / wp, column
        // cx0 + p % wp, written after that column's fill pairs
        const uint32_t np = wp * hc;
        for (uint32_t p0 = 0; p0 < np; p0 += 32) {
          const uint32_t p = p0 + (uint32_t)lane;
          const uint32_t rr = min((uint32_t)(((float)p + 0.5f) * inv_wp), hc - 1);
          const uint32_t cc = min(p - rr * wp, wp - 1);
          const uint32_t bc = cx0 + cc - wlo;  // buffer column = owning lane
          const uint32_t f = __shfl_sync(0xffffffffu, fill, (int)bc);
          if (p < np) {
            const int at = (int)(f + rr) * kColPitch + (int)bc;
            if constexpr (sizeof(KT) == 4)
              s_bk[at] = ((row0 + r0 + rr) << cbits) | (wlo + bc);
            else
              s_bk[at] = (KT)(row0 + r0 + rr);
            s_bi[at] = r.w;
          }
        }
        if (owner) fill += hc;
      }
    }
  }
  // what is left in each column's buffer
  __syncwarp();
  uint32_t left = __ballot_sync(0xffffffffu, fill > 0);
  while (left) {
    const int L = __ffs(left) - 1;
    left &= left - 1;
    flush_column(keys_out, ids_out, capacity, s_bk, s_bi, L, __shfl_sync(0xffffffffu, gofs, L),
                 __shfl_sync(0xffffffffu, fill, L), status);
  }
}
// (4) the ranges, from the tile counts instead of the sorted keys (grids
// whose difference array fits a block's shared memory). The pairs end up
// ordered by global tile, view-major and row-major within a view, so tile
// t's slice starts after every pair of the views before it and of the tiles
// before it in its view; a tile's pair count is the number of rectangles
// covering it. The rows pass then needs no keys written: nothing reads them.

// (4a) per view: a 2-D difference array of the rectangles' corners (+1 at
// (y0, x0) and (y1 + 1, x1 + 1), -1 at (y0, x1 + 1) and (y1 + 1, x0)),
// summed per block in shared memory and added into the view's array in
// global memory, and the view's pair total. Grid (blocks per view, views):
// block b takes a contiguous share of the view's rectangles -- its presorted
// visible ones (kBins false, from the packed rectangles of the column
// emission), or all n of its binning records (kBins true, full-64 mode).
template <bool kBins>
__global__ void __launch_bounds__(1024) k_tile_hist(const uint4* __restrict__ crect,
                                                    const float4* __restrict__ bins, int n,
                                                    const uint32_t* __restrict__ n_visible,
                                                    Grid g, int* __restrict__ diff,
                                                    unsigned long long* __restrict__ view_pairs) {
  extern __shared__ int s_d[];  // [tiles_y + 1][tiles_x + 1]
  __shared__ unsigned long long s_tot[32];
  const int v = blockIdx.y;
  const int W = g.tiles_x + 1, H = g.tiles_y + 1;
  for (int k = threadIdx.x; k < W * H; k += blockDim.x) s_d[k] = 0;
  __syncthreads();
  int64_t vs, nv;
  if (kBins) {
    vs = (int64_t)v * n;
    nv = n;
  } else {
    view_span(n_visible, v, vs, nv);
  }
  const int64_t share = (nv + gridDim.x - 1) / gridDim.x;
  const int64_t first = vs + (int64_t)blockIdx.x * share;
  const int64_t last = min(vs + nv, first + share);
  uint64_t mine = 0;
  for (int64_t i = first + threadIdx.x; i < last; i += blockDim.x) {
    uint32_t rx, ry;
    if (kBins) {
      const float4 b = __ldg(&bins[i]);
      rx = __float_as_uint(b.y);
      ry = __float_as_uint(b.z);
    } else {
      const uint4 r = crect[i];
      rx = r.x;
      ry = r.y;
    }
    const int x0 = rx & 0xffffu, x1 = rx >> 16, y0 = ry & 0xffffu, y1 = ry >> 16;
    if (x0 <= x1 && y0 <= y1) {
      atomicAdd(&s_d[y0 * W + x0], 1);
      atomicAdd(&s_d[y0 * W + x1 + 1], -1);
      atomicAdd(&s_d[(y1 + 1) * W + x0], -1);
      atomicAdd(&s_d[(y1 + 1) * W + x1 + 1], 1);
      mine += (uint64_t)(x1 - x0 + 1) * (uint64_t)(y1 - y0 + 1);
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mine += __shfl_xor_sync(0xffffffffu, mine, o);
  if ((threadIdx.x & 31) == 0) s_tot[threadIdx.x >> 5] = mine;
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned long long t = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) t += s_tot[w];
    if (t) atomicAdd(&view_pairs[v], t);
  }
  int* gd = diff + (int64_t)v * W * H;
  for (int k = threadIdx.x; k < W * H; k += blockDim.x) {
    const int x = s_d[k];
    if (x) atomicAdd(&gd[k], x);
  }
}

// (4b) per view (one block of 1024 threads each): the difference array summed
// along rows then columns gives each tile's count; thread i takes a run of
// consecutive tiles, a block scan of the runs' sums gives every tile's start
// within the view, after the pairs of the views before it. Nothing is written
// when the pairs of all views exceed the capacity (every range stays empty,
// as zeroed).
__global__ void __launch_bounds__(1024) k_tile_ranges(
    const int* __restrict__ diff, const unsigned long long* __restrict__ view_pairs,
    int n_views, Grid g, int64_t capacity, int64_t* __restrict__ ranges) {
  extern __shared__ int s_d[];  // [tiles_y + 1][tiles_x + 1]
  __shared__ uint32_t s_warp[33];
  unsigned long long total = 0;
  for (int u = 0; u < n_views; ++u) total += view_pairs[u];
  if ((int64_t)total > capacity) return;
  const int v = blockIdx.x;
  const int W = g.tiles_x + 1, H = g.tiles_y + 1;
  const int* gd = diff + (int64_t)v * W * H;
  for (int k = threadIdx.x; k < W * H; k += blockDim.x) s_d[k] = gd[k];
  __syncthreads();
  for (int r = threadIdx.x; r < H - 1; r += blockDim.x) {
    int acc = 0;
    for (int c = 0; c < W - 1; ++c) {
      acc += s_d[r * W + c];
      s_d[r * W + c] = acc;
    }
  }
  __syncthreads();
  for (int c = threadIdx.x; c < W - 1; c += blockDim.x) {
    int acc = 0;
    for (int r = 0; r < H - 1; ++r) {
      acc += s_d[r * W + c];
      s_d[r * W + c] = acc;
    }
  }
  __syncthreads();
  int64_t base = 0;
  for (int u = 0; u < v; ++u) base += (int64_t)view_pairs[u];
  const int tpv = g.tiles_per_view;
  const int run = (tpv + (int)blockDim.x - 1) / (int)blockDim.x;
  const int t0 = (int)threadIdx.x * run;
  // a view's pairs are at most the capacity (checked above): 32 bits hold them
  uint32_t sum = 0;
  for (int t = t0; t < min(t0 + run, tpv); ++t) {
    const int r = t / g.tiles_x;
    sum += (uint32_t)s_d[r * W + (t - r * g.tiles_x)];
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const uint32_t w = lane < (int)(blockDim.x >> 5) ? s_warp[lane] : 0u;
    uint32_t wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += y;
    }
    s_warp[lane] = wi - w;
  }
  __syncthreads();
  int64_t pos = base + (int64_t)(s_warp[warp] + incl - sum);
  int64_t* rv = ranges + 2 * (int64_t)v * tpv;
  for (int t = t0; t < min(t0 + run, tpv); ++t) {
    const int r = t / g.tiles_x;
    const int64_t c = s_d[r * W + (t - r * g.tiles_x)];
    rv[2 * (int64_t)t] = pos;
    rv[2 * (int64_t)t + 1] = pos + c;
    pos += c;
  }
}

// Fused pair count + scan + emission.
// MODE 0 (full 64-bit keys): items are the n_views * n Gaussians in index
//   order; key = (global tile << 32) | depth bits.
// MODE 1 (presorted): items are the presorted (key, index) list; key = global
//   tile (32-bit).
// An item's pairs are its rectangle's tiles in row-major order.
// Counting: each thread takes 4 consecutive items; block scan; decoupled
// look-back for the block's global offset.
// Emission, window by window of the block's pairs: thread t takes pairs
// 8t .. 8t+7 of the window (4 in MODE 0) -- one binary search over the item
// offsets, then row / column stepping -- and stages them in shared memory
// (one pad word per 32 so the strided writes hit distinct banks); the block
// then writes the window out with coalesced stores.
template <int MODE, typename K>
__global__ void __launch_bounds__(kEmitThreads) k_emit(
    const float4* __restrict__ bins, const uint64_t* __restrict__ pkeys,
    const uint32_t* __restrict__ pvals, int n, int n_views, Grid g,
    K* __restrict__ keys_out, uint32_t* __restrict__ ids_out, int64_t capacity,
    int64_t* __restrict__ n_pairs, uint64_t* __restrict__ lookback, uint32_t* __restrict__ block_counter,
    uint32_t* __restrict__ status, WaitCfg wc) {
  constexpr int kPer = MODE == 0 ? 4 : 8;           // pairs per thread per window
  constexpr int kWin = kPer * kEmitThreads;         // pairs per window
  constexpr int kWinPad = kWin + kWin / 32;
  __shared__ uint32_t s_off[kEmitItems + 1];
  __shared__ uint32_t s_rx[kEmitItems];   // x0 | width << 16
  __shared__ uint32_t s_ry[kEmitItems];   // y0 | view << 16
  __shared__ uint32_t s_id[kEmitItems];
  __shared__ uint32_t s_depth[MODE == 0 ? kEmitItems : 1];
  __shared__ K s_key[kWinPad];
  __shared__ uint32_t s_sid[kWinPad];
  __shared__ uint32_t s_warp[9];
  __shared__ uint64_t s_base;

  const uint32_t bidx = get_block_index(block_counter);
  const int64_t n_items = (int64_t)n * n_views;
  const int64_t first = (int64_t)bidx * kEmitItems;

  uint32_t cnt[kEmitItemsPerThread];
  uint32_t tsum = 0;
#pragma unroll
  for (int k = 0; k < kEmitItemsPerThread; ++k) {
    const int li = threadIdx.x * kEmitItemsPerThread + k;
    const int64_t item = first + li;
    uint32_t c = 0, rx = 0, ry = 0, id = 0, depth = 0;
    if (item < n_items) {
      int64_t rec_index;
      int vw;
      if (MODE == 0) {
        vw = (int)(item / n);
        id = (uint32_t)(item - (int64_t)vw * n);
        rec_index = item;
      } else {
        const uint64_t pk = pkeys[item];
        vw = pk == ~0ull ? -1 : (int)(pk >> 32);
        id = pvals[item];
        rec_index = (int64_t)(vw < 0 ? 0 : vw) * n + id;
      }
      if (vw >= 0) {
        const float4 r2 = __ldg(&bins[rec_index]);
        if (MODE == 0 && __float_as_uint(r2.x) == kNonfiniteKeyBits)
          atomicOr(status, kStatusNonfinite);
        const uint32_t txw = __float_as_uint(r2.y), tyw = __float_as_uint(r2.z);
        const uint32_t x0 = txw & 0xffffu, x1 = txw >> 16, y0 = tyw & 0xffffu, y1 = tyw >> 16;
        if (x0 <= x1 && y0 <= y1) {
          const uint32_t w = x1 - x0 + 1;
          c = w * (y1 - y0 + 1);
          rx = x0 | (w << 16);
          ry = y0 | ((uint32_t)vw << 16);
          depth = __float_as_uint(r2.x);
        }
      }
    }
    cnt[k] = c;
    s_rx[li] = rx;
    s_ry[li] = ry;
    s_id[li] = id;
    if (MODE == 0) s_depth[li] = depth;
    tsum += c;
  }
  uint32_t block_total;
  uint32_t toff = block_exclusive_scan_256(tsum, s_warp, block_total);
#pragma unroll
  for (int k = 0; k < kEmitItemsPerThread; ++k) {
    s_off[threadIdx.x * kEmitItemsPerThread + k] = toff;
    toff += cnt[k];
  }
  if (threadIdx.x < 32) {
    const uint64_t base = warp_block_lookback(lookback, bidx, block_total, status, wc);
    if (threadIdx.x == 0) {
      s_off[kEmitItems] = block_total;
      s_base = base;
      const uint32_t n_blocks = (uint32_t)((n_items + kEmitItems - 1) / kEmitItems);
      if (bidx == n_blocks - 1) *n_pairs = (int64_t)(base + block_total);
      if ((int64_t)(base + block_total) > capacity) atomicOr(status, kStatusCapacity);
    }
  }
  __syncthreads();
  const uint64_t base = s_base;
  if ((int64_t)(base + block_total) > capacity) return;  // nothing is emitted

  const uint32_t tiles_x = (uint32_t)g.tiles_x, tpv = (uint32_t)g.tiles_per_view;
  for (uint32_t w0 = 0; w0 < block_total; w0 += kWin) {
    const uint32_t p0 = w0 + threadIdx.x * kPer;
    if (p0 < block_total) {
      // item owning pair p0: largest k with s_off[k] <= p0 (skips empty items)
      int lo = 0, hi = kEmitItems - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_off[mid] <= p0) lo = mid; else hi = mid - 1;
      }
      int k = lo;
      uint32_t end_k = s_off[k + 1];
      uint32_t rx = s_rx[k], ry = s_ry[k];
      uint32_t w = rx >> 16;
      const uint32_t local = p0 - s_off[k];
      uint32_t row = local / w, col = local - row * w;
      uint32_t id = s_id[k];
      uint32_t depth = MODE == 0 ? s_depth[k] : 0u;
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        const uint32_t p = p0 + i;
        if (p >= block_total) break;
        if (p >= end_k) {  // next item that has pairs
          do {
            ++k;
            end_k = s_off[k + 1];
          } while (p >= end_k);
          rx = s_rx[k];
          ry = s_ry[k];
          w = rx >> 16;
          row = 0;
          col = 0;
          id = s_id[k];
          if (MODE == 0) depth = s_depth[k];
        }
        const uint32_t tile = (ry >> 16) * tpv + ((ry & 0xffffu) + row) * tiles_x + (rx & 0xffffu) + col;
        const uint32_t q = p - w0;
        const uint32_t si = q + (q >> 5);
        s_key[si] = MODE == 0 ? (K)(((uint64_t)tile << 32) | depth) : (K)tile;
        s_sid[si] = id;
        if (++col == w) {
          col = 0;
          ++row;
        }
      }
    }
    __syncthreads();
    const uint32_t m = min((uint32_t)kWin, block_total - w0);
    for (uint32_t q = threadIdx.x; q < m; q += kEmitThreads) {
      const uint32_t si = q + (q >> 5);
      keys_out[base + w0 + q] = s_key[si];
      ids_out[base + w0 + q] = s_sid[si];
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// Radix pass, reduce-then-scan, on a BITS-wide digit (key >> shift) & (2^BITS
// - 1). Partition p holds keys [p * TILE, (p + 1) * TILE), TILE = 256 * ITEMS.
// counts: uint32 [2^BITS][stride], digit-major. Positions are 32-bit (the
// caller keeps every key count below 2^31).

template <int ITEMS>
struct SortTile {
  static constexpr int kItems = kSortThreads * ITEMS;
};

// (1) digit counts of one partition (per-warp shared histograms).
template <typename K, int BITS, int ITEMS>
__global__ void __launch_bounds__(kSortThreads) k_radix_count(
    const K* __restrict__ keys, const int64_t* __restrict__ n_ptr, int64_t capacity, int shift,
    uint32_t* __restrict__ counts, int64_t stride) {
  constexpr int R = 1 << BITS;
  constexpr uint32_t M = R - 1;
  constexpr int TILE = SortTile<ITEMS>::kItems;
  __shared__ uint32_t s_h[kSortWarps][R];
  const int64_t n64 = *n_ptr;
  if (n64 > capacity || n64 <= 0) return;
  const uint32_t n = (uint32_t)n64;
  const uint32_t p = blockIdx.x;
  if (p * (uint32_t)TILE >= n) return;
  const int tid = threadIdx.x, warp = tid >> 5;
  for (int k = tid; k < kSortWarps * R; k += kSortThreads) (&s_h[0][0])[k] = 0u;
  // a histogram needs no order: each thread takes ITEMS consecutive keys,
  // with 16-byte loads when they are all there
  static_assert((ITEMS * sizeof(K)) % 16 == 0, "whole 16-byte loads");
  constexpr int kVec = (int)(ITEMS * sizeof(K) / 16);
  const uint32_t first = p * (uint32_t)TILE + (uint32_t)tid * ITEMS;
  K key[ITEMS];
  if (first + ITEMS <= n) {
    uint4 v[kVec];
    const uint4* src = reinterpret_cast<const uint4*>(keys + first);
#pragma unroll
    for (int q = 0; q < kVec; ++q) v[q] = src[q];
    memcpy(key, v, sizeof(key));
  } else {
#pragma unroll
    for (int it = 0; it < ITEMS; ++it) key[it] = first + it < n ? keys[first + it] : (K)0;
  }
  __syncthreads();
#pragma unroll
  for (int it = 0; it < ITEMS; ++it) {
    if (first + it < n) atomicAdd(&s_h[warp][(uint32_t)(key[it] >> shift) & M], 1u);
  }
  __syncthreads();
  for (int d = tid; d < R; d += kSortThreads) {
    uint32_t c = 0;
#pragma unroll
    for (int w = 0; w < kSortWarps; ++w) c += s_h[w][d];
    counts[(int64_t)d * stride + p] = c;
  }
}

// (2) per digit (one block each): exclusive scan of its counts over the
// partitions, in place (coalesced 4-wide loads), and the digit's total.
__global__ void __launch_bounds__(256) k_radix_scan(uint32_t* __restrict__ counts, int64_t stride,
                                                   const int64_t* __restrict__ n_ptr,
                                                   int64_t capacity, int tile,
                                                   uint32_t* __restrict__ totals) {
  __shared__ uint32_t s_warp[9];
  const int64_t n = *n_ptr;
  if (n > capacity || n <= 0) return;
  const int64_t parts = (n + tile - 1) / tile;
  uint32_t* row = counts + (int64_t)blockIdx.x * stride;
  uint32_t carry = 0;
  for (int64_t base = 0; base < parts; base += 4 * 256) {
    const int64_t i0 = base + 4 * (int64_t)threadIdx.x;
    const bool full = i0 + 4 <= parts;
    uint32_t v[4];
    if (full) {
      const uint4 q = *reinterpret_cast<const uint4*>(row + i0);
      v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
    } else {
#pragma unroll
      for (int k = 0; k < 4; ++k) v[k] = i0 + k < parts ? row[i0 + k] : 0u;
    }
    uint32_t tot;
    uint32_t run = carry + block_exclusive_scan_256(v[0] + v[1] + v[2] + v[3], s_warp, tot);
    uint32_t o[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      o[k] = run;
      run += v[k];
    }
    if (full) {
      *reinterpret_cast<uint4*>(row + i0) = make_uint4(o[0], o[1], o[2], o[3]);
    } else {
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (i0 + k < parts) row[i0 + k] = o[k];
    }
    carry += tot;
  }
  if (threadIdx.x == 0) totals[blockIdx.x] = carry;
}

// Lanes of the warp holding the same BITS-bit value d: the intersection over
// the bits of d of the ballot of lanes agreeing on that bit. Costs the same
// whatever the values (unlike match.any, whose cost grows with the number of
// distinct values).
template <int BITS>
__device__ __forceinline__ uint32_t warp_peers(uint32_t d) {
  uint32_t peers = 0xffffffffu;
#pragma unroll
  for (int b = 0; b < BITS; ++b) {
    const uint32_t bal = __ballot_sync(0xffffffffu, (d >> b) & 1u);
    peers &= ((d >> b) & 1u) ? bal : ~bal;
  }
  return peers;
}

// Scatter blocks per SM (reduce-then-scan scatter and single-sweep pass). The
// passes are bound by latency at low occupancy (their DRAM traffic is the
// keys' and values' bytes, read and written once): with 64-bit keys and 16
// keys per thread, three blocks (80 registers, a few spilled) measured 6 %
// faster than two on a 985M-key sort.
template <typename K, int ITEMS>
struct ScatterOcc {
  static constexpr int kBlocks = 3;
};
// Narrow keys (the rows of the column path) hold few registers: four blocks.
template <int ITEMS>
struct ScatterOcc<uint8_t, ITEMS> {
  static constexpr int kBlocks = 4;
};
template <int ITEMS>
struct ScatterOcc<uint16_t, ITEMS> {
  static constexpr int kBlocks = 4;
};

template <typename K, int BITS, int ITEMS>
size_t scatter_smem_bytes() {
  constexpr int R = 1 << BITS;
  return (size_t)SortTile<ITEMS>::kItems * (sizeof(K) + 4) + (size_t)(kSortWarps + 1) * R * 4;
}

// (3) stable scatter of one partition: loads (warp-striped), per-warp digit
// counts, block-local digit starts, ranking by ballots, staging in shared
// memory in sorted order, then runs of equal digits written at their global
// offsets. Keys past the end take the largest digit: they rank after every
// real key of the partition and are never written. keys_out may be null (a
// last pass whose keys nothing reads): then only the values are written.
template <typename K, int BITS, int ITEMS>
__global__ void __launch_bounds__(kSortThreads, (ScatterOcc<K, ITEMS>::kBlocks)) k_radix_scatter(
    const K* __restrict__ keys_in, const uint32_t* __restrict__ vals_in,
    K* __restrict__ keys_out, uint32_t* __restrict__ vals_out,
    const int64_t* __restrict__ n_ptr, int64_t capacity, int shift,
    const uint32_t* __restrict__ offsets, int64_t stride, const uint32_t* __restrict__ totals,
    uint32_t* __restrict__ status) {
  constexpr int R = 1 << BITS;
  constexpr uint32_t M = R - 1;
  constexpr int TILE = SortTile<ITEMS>::kItems;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  K* s_keys = reinterpret_cast<K*>(smem_raw);                          // [TILE]
  uint32_t* s_vals = reinterpret_cast<uint32_t*>(s_keys + TILE);       // [TILE]
  uint32_t* s_whist = s_vals + TILE;                                   // [warps][R]
  uint32_t* s_delta = s_whist + kSortWarps * R;                        // [R]
  __shared__ uint32_t s_scan[9];

  const int64_t n64 = *n_ptr;
  if (n64 > capacity || n64 <= 0) return;
  const uint32_t n = (uint32_t)n64;
  const uint32_t p = blockIdx.x;
  if (p * (uint32_t)TILE >= n) return;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int k = tid; k < kSortWarps * R; k += kSortThreads) s_whist[k] = 0u;
  const uint32_t first = p * (uint32_t)TILE + (uint32_t)warp * (ITEMS * 32) + lane;
  K key[ITEMS];
  uint32_t val[ITEMS];
#pragma unroll
  for (int it = 0; it < ITEMS; ++it) {
    const uint32_t idx = first + it * 32;
    key[it] = idx < n ? keys_in[idx] : (K)0;
    val[it] = idx < n ? vals_in[idx] : 0u;
  }
  // digit d's keys of this partition start at totals(< d) + offsets[d][p]
  const uint32_t gbase = tid < R ? offsets[(int64_t)tid * stride + p] : 0u;
  const uint32_t dtotal = tid < R ? totals[tid] : 0u;
  __syncthreads();
  uint32_t* wh = s_whist + warp * R;
#pragma unroll
  for (int it = 0; it < ITEMS; ++it) {
    const uint32_t idx = first + it * 32;
    const uint32_t d = idx < n ? ((uint32_t)(key[it] >> shift) & M) : M;
    atomicAdd(&wh[d], 1u);
  }
  uint32_t all;
  const uint32_t dbase = block_exclusive_scan_256(dtotal, s_scan, all);  // syncs the block
  // per digit: warp offsets, block count, block-local start
  uint32_t count = 0;
  if (tid < R) {
#pragma unroll
    for (int w = 0; w < kSortWarps; ++w) {
      const uint32_t c = s_whist[w * R + tid];
      s_whist[w * R + tid] = count;
      count += c;
    }
  }
  uint32_t tot;
  const uint32_t lstart = block_exclusive_scan_256(count, s_scan, tot);
  if (tid < R) {
    s_delta[tid] = dbase + gbase - lstart;  // local slot j -> global position j + delta
#pragma unroll
    for (int w = 0; w < kSortWarps; ++w) s_whist[w * R + tid] += lstart;
  }
  __syncthreads();
  // stable rank within the warp -> position within the partition
  const uint32_t lt = lanemask_lt();
#pragma unroll
  for (int it = 0; it < ITEMS; ++it) {
    const uint32_t idx = first + it * 32;
    const uint32_t d = idx < n ? ((uint32_t)(key[it] >> shift) & M) : M;
    const uint32_t peers = warp_peers<BITS>(d);
    const uint32_t before = wh[d];
    __syncwarp();
    if ((peers & lt) == 0) wh[d] = before + __popc(peers);
    __syncwarp();
    const uint32_t pos = before + __popc(peers & lt);
    s_keys[pos] = key[it];
    s_vals[pos] = val[it];
  }
  __syncthreads();
  const uint32_t remain = n - p * (uint32_t)TILE;
  const uint32_t valid = remain < (uint32_t)TILE ? remain : (uint32_t)TILE;
  for (uint32_t j = tid; j < valid; j += kSortThreads) {
    const K k = s_keys[j];
    const uint32_t gpos = j + s_delta[(uint32_t)(k >> shift) & M];
    if (gpos < n) {
      if (keys_out) keys_out[gpos] = k;
      vals_out[gpos] = s_vals[j];
    } else {
      atomicOr(status, kStatusBounds);
    }
  }
}

// ---------------------------------------------------------------------------
// Single-sweep radix passes (the full 64-bit key sort). One kernel counts
// the digits of every pass over all keys at once; then each pass is one
// kernel. A pass's partitions take their indices in launch order (an atomic
// ticket), publish their digit counts, and find each digit's global offset
// by decoupled look-back over the partitions before them: a partition
// publishes its counts (an aggregate) before it waits on anything, and after
// its look-back its inclusive prefix, so a waiting partition walks back only
// to the nearest prefix, and every partition it waits on is already running.
// Look-back words: [63:34] pass tag, [33:32] flag (1 aggregate, 2 inclusive
// prefix), [31:0] count; the array is zeroed per call and each pass has its
// own tag. A wait that runs out of time takes a zero prefix and reports.
constexpr uint64_t kSwAgg = 1ull << 32;
constexpr uint64_t kSwPre = 2ull << 32;
constexpr uint64_t kSwFlags = 3ull << 32;
constexpr int kSwBatch = 4;

// Digit counts of every pass in one read of the keys. A thread takes 8
// consecutive keys (vector loads) and adds each run of equal digits with one
// shared atomic: a Gaussian's pairs are emitted together and share their
// depth, so runs are long and the atomics few.
template <typename K>
__global__ void __launch_bounds__(256) k_digit_hist(const K* __restrict__ keys,
                                                    const int64_t* __restrict__ n_ptr,
                                                    int64_t capacity, RadixPlan plan,
                                                    uint32_t* __restrict__ hist) {
  __shared__ uint32_t s_h[8][256];
  const int64_t n = *n_ptr;
  if (n > capacity || n <= 0) return;
  for (int k = threadIdx.x; k < 8 * 256; k += 256) (&s_h[0][0])[k] = 0u;
  __syncthreads();
  const int64_t chunks = (n + 7) / 8;
  for (int64_t c = (int64_t)blockIdx.x * 256 + threadIdx.x; c < chunks;
       c += (int64_t)gridDim.x * 256) {
    const int64_t base = c * 8;
    const int cnt = n - base < 8 ? (int)(n - base) : 8;
    K k[8];
    if (cnt == 8) {
      uint4 raw[sizeof(K) / 2];
      const uint4* src = reinterpret_cast<const uint4*>(keys + base);
#pragma unroll
      for (int r = 0; r < (int)(sizeof(K) / 2); ++r) raw[r] = src[r];
      memcpy(k, raw, sizeof(k));
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) k[j] = j < cnt ? keys[base + j] : (K)0;
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      if (q >= plan.passes) break;
      const int sh = plan.shift[q];
      uint32_t prev = (uint32_t)(k[0] >> sh) & 255u, run = 1;
#pragma unroll
      for (int j = 1; j < 8; ++j) {
        if (j >= cnt) break;
        const uint32_t d = (uint32_t)(k[j] >> sh) & 255u;
        if (d == prev) {
          ++run;
        } else {
          atomicAdd(&s_h[q][prev], run);
          prev = d;
          run = 1;
        }
      }
      atomicAdd(&s_h[q][prev], run);
    }
  }
  __syncthreads();
  for (int k = threadIdx.x; k < plan.passes * 256; k += 256) {
    const uint32_t c = (&s_h[0][0])[k];
    if (c) atomicAdd(&hist[k], c);
  }
}

template <typename K, int ITEMS>
__global__ void __launch_bounds__(kSortThreads, (ScatterOcc<K, ITEMS>::kBlocks)) k_onesweep(
    const K* __restrict__ keys_in, const uint32_t* __restrict__ vals_in,
    K* __restrict__ keys_out, uint32_t* __restrict__ vals_out,
    const int64_t* __restrict__ n_ptr, int64_t capacity, int shift, int pass,
    const uint32_t* __restrict__ hist, uint64_t* __restrict__ lookback,
    uint32_t* __restrict__ ticket, WaitCfg wc, uint32_t* __restrict__ status) {
  constexpr int R = 256;
  constexpr uint32_t M = R - 1;
  constexpr int TILE = SortTile<ITEMS>::kItems;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  K* s_keys = reinterpret_cast<K*>(smem_raw);                          // [TILE]
  uint32_t* s_vals = reinterpret_cast<uint32_t*>(s_keys + TILE);       // [TILE]
  uint32_t* s_whist = s_vals + TILE;                                   // [warps][R]
  uint32_t* s_delta = s_whist + kSortWarps * R;                        // [R]
  __shared__ uint32_t s_scan[9];
  __shared__ uint32_t s_p;

  const int64_t n64 = *n_ptr;
  if (n64 > capacity || n64 <= 0) return;
  const uint32_t n = (uint32_t)n64;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) s_p = atomicAdd(ticket, 1u);
  for (int k = tid; k < kSortWarps * R; k += kSortThreads) s_whist[k] = 0u;
  __syncthreads();
  const uint32_t p = s_p;
  if ((uint64_t)p * TILE >= n) return;  // the whole block: no partition left
  const uint32_t first = p * (uint32_t)TILE + (uint32_t)warp * (ITEMS * 32) + lane;
  K key[ITEMS];
  uint32_t val[ITEMS];
#pragma unroll
  for (int it = 0; it < ITEMS; ++it) {
    const uint32_t idx = first + it * 32;
    key[it] = idx < n ? keys_in[idx] : (K)0;
    val[it] = idx < n ? vals_in[idx] : 0u;
  }
  const uint32_t hcount = hist[tid];
  uint32_t* wh = s_whist + warp * R;
#pragma unroll
  for (int it = 0; it < ITEMS; ++it) {
    const uint32_t idx = first + it * 32;
    const uint32_t d = idx < n ? ((uint32_t)(key[it] >> shift) & M) : M;
    atomicAdd(&wh[d], 1u);
  }
  __syncthreads();
  // per digit: warp offsets and the partition's count (keys past the end sit
  // in the largest digit and are not counted)
  uint32_t count = 0;
  {
#pragma unroll
    for (int w = 0; w < kSortWarps; ++w) {
      const uint32_t c = s_whist[w * R + tid];
      s_whist[w * R + tid] = count;
      count += c;
    }
  }
  const uint32_t remain = n - p * (uint32_t)TILE;
  const uint32_t valid = remain < (uint32_t)TILE ? remain : (uint32_t)TILE;
  const uint32_t real = tid == (int)M ? count - ((uint32_t)TILE - valid) : count;
  const uint64_t tag = (uint64_t)(pass + 1) << 34;
  uint64_t* row = lookback + (uint64_t)p * R;
  const bool publish = (int64_t)p != wc.stall;  // test hook: a silent partition
  if (publish) st_relaxed_u64(row + tid, tag | (p == 0 ? kSwPre : kSwAgg) | real);
  uint32_t tot;
  const uint32_t lstart = block_exclusive_scan_256(count, s_scan, tot);  // syncs the block
#pragma unroll
  for (int w = 0; w < kSortWarps; ++w) s_whist[w * R + tid] += lstart;
  __syncthreads();
  // stable rank within the warp -> position within the partition
  const uint32_t lt = lanemask_lt();
#pragma unroll
  for (int it = 0; it < ITEMS; ++it) {
    const uint32_t idx = first + it * 32;
    const uint32_t d = idx < n ? ((uint32_t)(key[it] >> shift) & M) : M;
    const uint32_t peers = warp_peers<8>(d);
    const uint32_t before = wh[d];
    __syncwarp();
    if ((peers & lt) == 0) wh[d] = before + __popc(peers);
    __syncwarp();
    const uint32_t pos = before + __popc(peers & lt);
    s_keys[pos] = key[it];
    s_vals[pos] = val[it];
  }
  // the pass's digit starts, then this partition's global offsets; ranking
  // first gives the partitions before this one time to publish prefixes
  uint32_t all;
  const uint32_t dbase = block_exclusive_scan_256(hcount, s_scan, all);  // syncs the block
  // decoupled look-back for this thread's digit
  // (kSwBatch predecessors' words are loaded at once, so a long walk costs
  // one load latency per batch rather than per partition)
  uint32_t excl = 0;
  if (p > 0) {
    int64_t j = (int64_t)p - 1;
    bool done = false;
    while (!done && j >= 0) {
      uint64_t w[kSwBatch];
#pragma unroll
      for (int b = 0; b < kSwBatch; ++b)
        w[b] = j - b >= 0 ? ld_relaxed_u64(lookback + (uint64_t)(j - b) * R + tid) : 0ull;
#pragma unroll
      for (int b = 0; b < kSwBatch; ++b) {
        if (done || j - b < 0) break;
        uint64_t v = w[b];
        if ((v & ~((1ull << 34) - 1)) != tag || (v & kSwFlags) == 0) {
          const uint64_t* src = lookback + (uint64_t)(j - b) * R + tid;
          const uint64_t t0 = globaltimer_ns();
          while (true) {
            __nanosleep(32);
            v = ld_relaxed_u64(src);
            if ((v & ~((1ull << 34) - 1)) == tag && (v & kSwFlags) != 0) break;
            if (globaltimer_ns() - t0 > wc.limit_ns) {
              atomicOr(status, kStatusTimeout);
              v = tag | kSwPre;  // give up: a zero prefix ends the walk
              break;
            }
          }
        }
        excl += (uint32_t)v;
        if ((v & kSwFlags) == kSwPre) done = true;
      }
      j -= kSwBatch;
    }
    if (publish) st_relaxed_u64(row + tid, tag | kSwPre | (excl + real));
  }
  s_delta[tid] = dbase + excl - lstart;  // local slot -> global position
  __syncthreads();
  for (uint32_t j = tid; j < valid; j += kSortThreads) {
    const K k = s_keys[j];
    const uint32_t gpos = j + s_delta[(uint32_t)(k >> shift) & M];
    if (gpos < n) {
      if (keys_out) keys_out[gpos] = k;
      vals_out[gpos] = s_vals[j];
    } else {
      atomicOr(status, kStatusBounds);
    }
  }
}

// Tile id of a sorted key.
template <typename K>
__device__ __forceinline__ uint32_t tile_of(K k) {
  return (uint32_t)(((uint64_t)k) >> (KeyTraits<K>::kBits == 64 ? 32 : 0));
}

// [start, end) of every tile present in the sorted keys. Each thread takes 8
// consecutive keys with vector loads (a full chunk) and compares neighbours.
// cbits > 0: 32-bit keys are row << cbits | column (column emission), decoded
// to row * tiles_x + column; the decoding is monotone, so runs stay runs.
template <typename K>
__global__ void k_ranges(const K* __restrict__ keys, const int64_t* __restrict__ n_ptr,
                         int64_t capacity, int64_t n_tiles, int cbits, uint32_t tiles_x,
                         int64_t* __restrict__ ranges, uint32_t* __restrict__ status) {
  const int64_t n = *n_ptr;
  if (n > capacity) return;
  constexpr int C = 8;
  const int64_t chunks = (n + C - 1) / C;
  for (int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; c < chunks;
       c += (int64_t)gridDim.x * blockDim.x) {
    const int64_t i0 = c * C;
    uint32_t t[C];
    if (i0 + C <= n) {
      if (KeyTraits<K>::kBits == 32) {
        const uint4* p4 = reinterpret_cast<const uint4*>(keys + i0);
        const uint4 a = p4[0], b = p4[1];
        t[0] = a.x; t[1] = a.y; t[2] = a.z; t[3] = a.w;
        t[4] = b.x; t[5] = b.y; t[6] = b.z; t[7] = b.w;
      } else {
        const ulonglong2* p2 = reinterpret_cast<const ulonglong2*>(keys + i0);
#pragma unroll
        for (int q = 0; q < C / 2; ++q) {
          const ulonglong2 v = p2[q];
          t[2 * q] = (uint32_t)(v.x >> 32);
          t[2 * q + 1] = (uint32_t)(v.y >> 32);
        }
      }
    } else {
#pragma unroll
      for (int k = 0; k < C; ++k) t[k] = i0 + k < n ? tile_of(keys[i0 + k]) : 0u;
    }
    uint32_t prev = i0 > 0 ? tile_of(keys[i0 - 1]) : 0xffffffffu;
    if (cbits > 0) {
      const uint32_t cm = (1u << cbits) - 1u;
#pragma unroll
      for (int k = 0; k < C; ++k) t[k] = (t[k] >> cbits) * tiles_x + (t[k] & cm);
      if (i0 > 0) prev = (prev >> cbits) * tiles_x + (prev & cm);
    }
#pragma unroll
    for (int k = 0; k < C; ++k) {
      const int64_t i = i0 + k;
      if (i >= n) break;
      const uint32_t cur = t[k];
      if ((int64_t)cur >= n_tiles) {
        atomicOr(status, kStatusBounds);
        prev = cur;
        continue;
      }
      if (i == 0) {
        ranges[2 * (int64_t)cur] = 0;
      } else if (cur != prev) {
        ranges[2 * (int64_t)cur] = i;
        if ((int64_t)prev < n_tiles) ranges[2 * (int64_t)prev + 1] = i;
      }
      if (i == n - 1) ranges[2 * (int64_t)cur + 1] = n;
      prev = cur;
    }
  }
}


template <typename K, int BITS, int ITEMS>
cudaError_t radix_pass(const K* kin, const uint32_t* vin, K* kout, uint32_t* vout,
                       const int64_t* n_ptr, int64_t capacity, int64_t parts, int shift,
                       uint32_t* counts, int64_t stride, uint32_t* totals, uint32_t* status,
                       cudaStream_t stream) {
  const size_t smem = scatter_smem_bytes<K, BITS, ITEMS>();
  cudaError_t e = cudaFuncSetAttribute(k_radix_scatter<K, BITS, ITEMS>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k_radix_count<K, BITS, ITEMS><<<(unsigned)parts, kSortThreads, 0, stream>>>(
      kin, n_ptr, capacity, shift, counts, stride);
  k_radix_scan<<<1u << BITS, 256, 0, stream>>>(counts, stride, n_ptr, capacity,
                                               SortTile<ITEMS>::kItems, totals);
  k_radix_scatter<K, BITS, ITEMS><<<(unsigned)parts, kSortThreads, smem, stream>>>(
      kin, vin, kout, vout, n_ptr, capacity, shift, counts, stride, totals, status);
  return cudaGetLastError();
}

// The plan's passes, ping-ponging between (keys_a, vals_a) and (keys_b,
// vals_b); grids sized for `max_items`, the device count read from n_ptr.
// last_keys false: the last pass writes the values only.
template <typename K, int ITEMS>
cudaError_t run_radix_passes(K* keys_a, uint32_t* vals_a, K* keys_b, uint32_t* vals_b,
                             const int64_t* n_ptr, int64_t capacity, int64_t max_items,
                             const RadixPlan& plan, uint32_t* counts, int64_t stride,
                             uint32_t* totals, uint32_t* status, cudaStream_t stream,
                             bool last_keys = true) {
  const int64_t parts = (max_items + SortTile<ITEMS>::kItems - 1) / SortTile<ITEMS>::kItems;
  if (parts == 0) return cudaSuccess;
  K* kin = keys_a;
  uint32_t* vin = vals_a;
  K* kout = keys_b;
  uint32_t* vout = vals_b;
  for (int p = 0; p < plan.passes; ++p) {
    const int sh = plan.shift[p];
    K* kout_p = (p + 1 == plan.passes && !last_keys) ? nullptr : kout;
    cudaError_t e = cudaErrorInvalidValue;
    if constexpr (sizeof(K) <= 4) {
      switch (plan.bits[p]) {
        case 4: e = radix_pass<K, 4, ITEMS>(kin, vin, kout_p, vout, n_ptr, capacity, parts, sh, counts, stride, totals, status, stream); break;
        case 5: e = radix_pass<K, 5, ITEMS>(kin, vin, kout_p, vout, n_ptr, capacity, parts, sh, counts, stride, totals, status, stream); break;
        case 6: e = radix_pass<K, 6, ITEMS>(kin, vin, kout_p, vout, n_ptr, capacity, parts, sh, counts, stride, totals, status, stream); break;
        case 7: e = radix_pass<K, 7, ITEMS>(kin, vin, kout_p, vout, n_ptr, capacity, parts, sh, counts, stride, totals, status, stream); break;
        case 8: e = radix_pass<K, 8, ITEMS>(kin, vin, kout_p, vout, n_ptr, capacity, parts, sh, counts, stride, totals, status, stream); break;
        default: break;
      }
    } else {
      if (plan.bits[p] == 8)
        e = radix_pass<K, 8, ITEMS>(kin, vin, kout_p, vout, n_ptr, capacity, parts, sh, counts, stride, totals, status, stream);
    }
    if (e != cudaSuccess) return e;
    K* tk = kin; kin = kout; kout = tk;
    uint32_t* tv = vin; vin = vout; vout = tv;
  }
  return cudaSuccess;
}

// The plan's passes (8-bit digits) as single-sweep passes, ping-ponging like
// run_radix_passes. hist: [8][256] digit counts, zeroed by the caller;
// lookback: [parts][256] words, zeroed by the caller; tickets: one zeroed
// counter per pass.
template <typename K, int ITEMS>
cudaError_t run_onesweep_passes(K* keys_a, uint32_t* vals_a, K* keys_b, uint32_t* vals_b,
                                const int64_t* n_ptr, int64_t capacity, int64_t max_items,
                                const RadixPlan& plan, uint32_t* hist, uint64_t* lookback,
                                uint32_t* tickets, const WaitCfg& wc, uint32_t* status,
                                int sms, cudaStream_t stream, bool last_keys = true) {
  const int64_t parts = (max_items + SortTile<ITEMS>::kItems - 1) / SortTile<ITEMS>::kItems;
  if (parts == 0) return cudaSuccess;
  for (int q = 0; q < plan.passes; ++q)
    if (plan.bits[q] != 8) return cudaErrorInvalidValue;
  k_digit_hist<K><<<sms * 4, 256, 0, stream>>>(keys_a, n_ptr, capacity, plan, hist);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t smem = scatter_smem_bytes<K, 8, ITEMS>();
  e = cudaFuncSetAttribute(k_onesweep<K, ITEMS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem);
  if (e != cudaSuccess) return e;
  K* kin = keys_a;
  uint32_t* vin = vals_a;
  K* kout = keys_b;
  uint32_t* vout = vals_b;
  for (int q = 0; q < plan.passes; ++q) {
    k_onesweep<K, ITEMS><<<(unsigned)parts, kSortThreads, smem, stream>>>(
        kin, vin, (q + 1 == plan.passes && !last_keys) ? nullptr : kout, vout, n_ptr, capacity,
        plan.shift[q], q, hist + 256 * q, lookback, tickets + q, wc, status);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    K* tk = kin; kin = kout; kout = tk;
    uint32_t* tv = vin; vin = vout; vout = tv;
  }
  return cudaSuccess;
}

int num_sms() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

}  // namespace

bool pair_passes_single_sweep(const RadixPlan& pairs, int sort_mode) {
  return sort_mode == GS_SORT_FULL64 && pairs.passes > 0;
}

RadixPlan make_radix_plan(int key_bits, bool balanced) {
  RadixPlan pl;
  pl.passes = (key_bits + 7) / 8;
  int shift = 0;
  for (int i = 0; i < pl.passes; ++i) {
    int w = 8;
    if (balanced) w = key_bits / pl.passes + (i < key_bits % pl.passes ? 1 : 0);
    pl.shift[i] = shift;
    // a digit wider than its share also covers bits of the next pass (or
    // zero bits above the key), which keeps the final order unchanged
    pl.bits[i] = w < 4 ? 4 : w;
    shift += w;
  }
  return pl;
}

int64_t pair_partitions(int64_t items) { return (items + kSortTile - 1) / kSortTile; }
int64_t presort_partitions(int64_t items) {
  return (items + SortTile<kPresortItems>::kItems - 1) / SortTile<kPresortItems>::kItems;
}
int64_t emit_blocks(int64_t items) { return (items + kEmitItems - 1) / kEmitItems; }
int64_t column_blocks(int64_t items) { return (items + kColItems - 1) / kColItems; }
bool column_emission(const Grid& g) { return g.tiles_x <= kMaxColumns; }
// Pairs placed straight at their positions on grids of up to 16384 tiles per
// view (a 1080p view has 8160): there one warp per (Gaussian block, region)
// keeps enough regions busy. A 4K view (32400 tiles) gives each Gaussian
// block 72 regions to scan, and the emission by column (then one radix pass
// over the rows) measured 1.7x faster there (12.0 against 20.5 ms for 849M
// pairs).
bool count_ranges_fit(const Grid& g) {
  return (int64_t)(g.tiles_x + 1) * (g.tiles_y + 1) * (int64_t)sizeof(int) <= kTileDiffBytes;
}
bool tile_emission(const Grid& g) {
  return g.tiles_per_view <= 16384 &&
         (int64_t)(g.tiles_x + 1) * (g.tiles_y + 1) * (int64_t)sizeof(int) <= kTileDiffBytes;
}
// Gaussians per block of the tile placement: 768 at a million Gaussians;
// fewer for small scenes, so that there are about four blocks per SM (one
// warp works through a block's rectangles in order, ~0.2 us each, so a
// 1000-Gaussian scene in two blocks of 768 took 0.15 ms); 4096 beyond two
// million, which keeps the (tile, block) count table small.
int tile_gsize(int64_t n) {
  if (n > (2 << 20)) return 4096;
  const int64_t g = n / (148 * 4) / 32 * 32;
  return g < 32 ? 32 : (g > 768 ? 768 : (int)g);
}

// The 32-bit pair keys of the column and tile-id paths, reduce-then-scan
// passes over their evenly split digits. (Single-sweep passes were measured
// slower on these keys: a 4K view's one 8-bit row pass over 849M pairs took
// the whole binning from 11.9 to 13.0 ms.)
template <typename KT>
cudaError_t sort_pairs(const BinSortArgs& a, cudaStream_t stream) {
  return run_radix_passes<KT, kSortItems>(
      reinterpret_cast<KT*>(a.keys[a.emit_buf]), a.vals[a.emit_buf],
      reinterpret_cast<KT*>(a.keys[a.emit_buf ^ 1]), a.vals[a.emit_buf ^ 1], a.n_pairs,
      a.capacity, a.capacity, a.pairs, a.counts, a.counts_stride, a.totals, a.status, stream,
      !a.count_ranges);
}

// The column path from the emission on, with KT keys: emission, the rows
// passes, the ranges off the keys unless they came from the counts.
template <typename KT>
cudaError_t emit_and_sort_columns(const BinSortArgs& a, int64_t n_items, int64_t cb, int sms,
                                  cudaStream_t stream) {
  const dim3 grid((unsigned)cb, (unsigned)((a.grid.tiles_x + 31) / 32));
  k_emit_cols<KT><<<grid, 32, 0, stream>>>(
      a.crect, n_items, a.grid, a.cbits, a.counts, a.counts_stride, a.totals, a.pair_total,
      reinterpret_cast<KT*>(a.keys[a.emit_buf]), a.vals[a.emit_buf], a.capacity, a.n_pairs,
      a.status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // 3) stable sort by row
  if ((e = sort_pairs<KT>(a, stream)) != cudaSuccess) return e;
  if (a.count_ranges) return cudaSuccess;
  if constexpr (sizeof(KT) == 4) {
    const int out = a.emit_buf ^ (a.pairs.passes & 1);
    k_ranges<uint32_t><<<sms * 4, 256, 0, stream>>>(
        reinterpret_cast<uint32_t*>(a.keys[out]), a.n_pairs, a.capacity, a.n_tiles, a.cbits,
        (uint32_t)a.grid.tiles_x, a.ranges, a.status);
    return cudaGetLastError();
  }
  return cudaErrorInvalidValue;  // narrow keys carry no column: ranges come from the counts
}

cudaError_t launch_bin_sort(const BinSortArgs& a, cudaStream_t stream) {
  cudaError_t e;
  const int64_t n_items = (int64_t)a.n * a.n_views;
  const auto bins4 = reinterpret_cast<const float4*>(a.bins);
  if (n_items == 0) {
    return cudaMemsetAsync(a.n_pairs, 0, sizeof(int64_t), stream);
  }
  const int sms = num_sms();
  const int64_t eb = emit_blocks(n_items);
  if (a.mode == GS_SORT_PRESORT) {
    // 1) keys (view << 32 | depth) over all Gaussians of all views, sorted
    int64_t blocks = (n_items + 255) / 256;
    if (blocks > (int64_t)sms * 8) blocks = (int64_t)sms * 8;
    k_depth_keys<<<(int)blocks, 256, 0, stream>>>(bins4, a.n, a.n_views, a.pkeys[0], a.pvals[0],
                                                  a.n_items_dev, a.n_visible, a.status);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    e = run_onesweep_passes<uint64_t, kPresortItems>(
        a.pkeys[0], a.pvals[0], a.pkeys[1], a.pvals[1], a.n_items_dev, n_items, n_items,
        a.presort, a.digit_hist, a.sweep_lookback, a.counters + 1, a.sort_wait, a.status, sms,
        stream);
    if (e != cudaSuccess) return e;
    const int fin = a.presort.passes & 1;
    if (a.tile_emit) {
      // 2) pairs per (tile, Gaussian block), their scans, placement
      const Grid& g = a.grid;
      const size_t dsmem = (size_t)(g.tiles_x + 1) * (g.tiles_y + 1) * sizeof(int);
      if ((e = cudaFuncSetAttribute(k_tile_count, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)dsmem)) != cudaSuccess)
        return e;
      k_tile_count<<<dim3((unsigned)a.tile_bpv, (unsigned)a.n_views), 256, dsmem, stream>>>(
          bins4, a.pkeys[fin], a.pvals[fin], a.n, g, a.gsize, a.n_visible, a.counts,
          a.counts_stride, a.pair_total, a.crect, a.scan_n);
      k_tile_scan<<<(unsigned)((a.n_tiles + 7) / 8), 256, 0, stream>>>(
          a.counts, a.counts_stride, a.tile_bpv, a.n_tiles, a.tile_totals);
      k_tile_base<<<1, 1024, 0, stream>>>(a.tile_totals, a.n_tiles, a.pair_total, a.capacity,
                                          a.tile_base, a.ranges, a.n_pairs, a.status);
      const int regions = ((g.tiles_x + kRegionCols - 1) / kRegionCols) *
                          ((g.tiles_y + kRegionRows - 1) / kRegionRows);
      const unsigned rblocks = (unsigned)((regions + kEmitWarps - 1) / kEmitWarps);
      // the packed rectangles (16 B per item) fit in L2 up to ~3M items
      const dim3 grid((unsigned)a.tile_bpv, rblocks, (unsigned)a.n_views);
      if (n_items * 16 <= (int64_t)(48 << 20))
        k_emit_tiles<kEmitAheadL2><<<grid, 32 * kEmitWarps, 0, stream>>>(
            a.crect, a.gsize, a.n_visible, g, regions, a.counts, a.counts_stride, a.tile_base,
            a.pair_total, a.vals[0], a.capacity, a.status);
      else
        k_emit_tiles<kEmitAheadDram><<<grid, 32 * kEmitWarps, 0, stream>>>(
            a.crect, a.gsize, a.n_visible, g, regions, a.counts, a.counts_stride, a.tile_base,
            a.pair_total, a.vals[0], a.capacity, a.status);
      return cudaGetLastError();
    }
    if (a.column_emit) {
      // 2) pairs per column and block, their scan, emission by column
      const int64_t cb = column_blocks(n_items);
      k_col_count<<<(unsigned)cb, kColItems, 0, stream>>>(bins4, a.pkeys[fin], a.pvals[fin], a.n,
                                                          a.n_views, a.grid, a.counts,
                                                          a.counts_stride, a.pair_total, a.crect);
      if (a.count_ranges) {
        // the ranges from the tile counts, before the pairs exist
        const Grid& g = a.grid;
        const size_t dsmem = (size_t)(g.tiles_x + 1) * (g.tiles_y + 1) * sizeof(int);
        if ((e = cudaFuncSetAttribute(k_tile_hist<false>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dsmem)) !=
                cudaSuccess ||
            (e = cudaFuncSetAttribute(k_tile_ranges, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)dsmem)) != cudaSuccess)
          return e;
        // about one 1024-thread block per SM over all views
        const int bpv = sms / a.n_views > 0 ? sms / a.n_views : 1;
        k_tile_hist<false><<<dim3((unsigned)bpv, (unsigned)a.n_views), 1024, dsmem, stream>>>(
            a.crect, nullptr, a.n, a.n_visible, g, a.tile_diff, a.view_pairs);
        k_tile_ranges<<<(unsigned)a.n_views, 1024, dsmem, stream>>>(
            a.tile_diff, a.view_pairs, a.n_views, g, a.capacity, a.ranges);
      }
      k_radix_scan<<<(unsigned)a.grid.tiles_x, 256, 0, stream>>>(
          a.counts, a.counts_stride, a.n_items_dev, n_items, kColItems, a.totals);
      if (a.row_key_bytes == 1) return emit_and_sort_columns<uint8_t>(a, n_items, cb, sms, stream);
      if (a.row_key_bytes == 2)
        return emit_and_sort_columns<uint16_t>(a, n_items, cb, sms, stream);
      return emit_and_sort_columns<uint32_t>(a, n_items, cb, sms, stream);
    }
    // 2) emission in depth order, 32-bit tile keys
    k_emit<1, uint32_t><<<(unsigned)eb, kEmitThreads, 0, stream>>>(
        bins4, a.pkeys[fin], a.pvals[fin], a.n, a.n_views, a.grid,
        reinterpret_cast<uint32_t*>(a.keys[a.emit_buf]), a.vals[a.emit_buf], a.capacity,
        a.n_pairs, a.emit_lookback, a.counters + 0, a.status, a.wait);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // 3) stable sort by tile
    e = sort_pairs<uint32_t>(a, stream);
    if (e != cudaSuccess) return e;
    const int out = a.emit_buf ^ (a.pairs.passes & 1);
    k_ranges<uint32_t><<<sms * 4, 256, 0, stream>>>(reinterpret_cast<uint32_t*>(a.keys[out]),
                                                   a.n_pairs, a.capacity, a.n_tiles, 0, 0u,
                                                   a.ranges, a.status);
    return cudaGetLastError();
  }
  // full 64-bit keys
  k_emit<0, uint64_t><<<(unsigned)eb, kEmitThreads, 0, stream>>>(
      bins4, nullptr, nullptr, a.n, a.n_views, a.grid, a.keys[a.emit_buf], a.vals[a.emit_buf],
      a.capacity, a.n_pairs, a.emit_lookback, a.counters + 0, a.status, a.wait);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if (a.count_ranges) {
    // the ranges from the tile counts of the binning records; the last pass
    // then writes no keys
    const Grid& g = a.grid;
    const size_t dsmem = (size_t)(g.tiles_x + 1) * (g.tiles_y + 1) * sizeof(int);
    if ((e = cudaFuncSetAttribute(k_tile_hist<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)dsmem)) != cudaSuccess ||
        (e = cudaFuncSetAttribute(k_tile_ranges, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  (int)dsmem)) != cudaSuccess)
      return e;
    const int bpv = sms / a.n_views > 0 ? sms / a.n_views : 1;
    k_tile_hist<true><<<dim3((unsigned)bpv, (unsigned)a.n_views), 1024, dsmem, stream>>>(
        nullptr, bins4, a.n, nullptr, g, a.tile_diff, a.view_pairs);
    k_tile_ranges<<<(unsigned)a.n_views, 1024, dsmem, stream>>>(
        a.tile_diff, a.view_pairs, a.n_views, g, a.capacity, a.ranges);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  e = run_onesweep_passes<uint64_t, kSortItems>(a.keys[a.emit_buf], a.vals[a.emit_buf],
                                                a.keys[a.emit_buf ^ 1], a.vals[a.emit_buf ^ 1],
                                                a.n_pairs, a.capacity, a.capacity, a.pairs,
                                                a.digit_hist, a.sweep_lookback, a.counters + 1,
                                                a.sort_wait, a.status, sms, stream,
                                                !a.count_ranges);
  if (e != cudaSuccess) return e;
  if (a.count_ranges) return cudaSuccess;
  const int out = a.emit_buf ^ (a.pairs.passes & 1);
  k_ranges<uint64_t><<<sms * 4, 256, 0, stream>>>(a.keys[out], a.n_pairs, a.capacity, a.n_tiles,
                                                  0, 0u, a.ranges, a.status);
  return cudaGetLastError();
}

}  // namespace gsb
