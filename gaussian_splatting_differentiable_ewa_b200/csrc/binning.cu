// binning.cu -- tile binning with depth sort, sm_100a.
//
// Assign every projected Gaussian to the 16x16 tiles its 3-sigma rectangle
// touches and order each tile's list by depth ("Better Gaussian Splatting in
// Julia", pwwt.cn sec. 3.3 steps 1-2 and 4.3; lshu.cn sec. 3.2
// assign_to_tiles / sort_by_depth!), ties broken by Gaussian index.
//
//  k_emit      one pass over the Gaussians: per-Gaussian pair counts, a
//              single-pass scan (decoupled look-back between blocks), and
//              load-balanced emission of (key, id) pairs by the whole block;
//              the digit histograms of the following radix passes are
//              accumulated on the way, so the sort needs no upsweep pass.
//  k_onesweep  one least-significant-digit pass of a stable radix sort with
//              8-bit digits: warp-level ranking with match.any, per-digit
//              decoupled look-back across partitions, scatter through shared
//              memory so global writes are runs of equal digits.
//  k_ranges    [start, end) of each tile in the sorted pairs.
// Every device-side wait is bounded (kSpinLimit) and reports through the
// status word instead of hanging.

#include <cuda_runtime.h>

#include "gs_internal.h"

namespace gsb {
namespace {

constexpr int kEmitThreads = 256;
constexpr int kEmitItemsPerThread = 4;
constexpr int kEmitItems = kEmitThreads * kEmitItemsPerThread;

constexpr int kSortThreads = 256;
constexpr int kSortWarps = kSortThreads / 32;
constexpr int kSortItems = 16;
constexpr int kSortTile = kSortThreads * kSortItems;  // keys per partition
constexpr int kRadix = 256;

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

// Exclusive prefix of partition p from the look-back words of partitions
// p-1, p-2, ... (word of partition j at base[j * stride]): one thread walks
// back kWin partitions per round trip (kWin independent loads), waiting only
// on words still empty, until it reaches an inclusive prefix. The window
// matters for throughput: with B partitions in flight a partition sums about
// B aggregates, i.e. B / kWin round trips.
template <int kWin>
__device__ __forceinline__ uint64_t windowed_lookback(const uint64_t* base, int64_t stride,
                                                      int64_t p, uint32_t* status) {
  uint64_t excl = 0;
  int64_t j = p - 1;
  while (j >= 0) {
    uint64_t w[kWin];
#pragma unroll
    for (int k = 0; k < kWin; ++k) w[k] = (j - k >= 0) ? ld_relaxed_u64(base + (j - k) * stride) : 0ull;
    bool found = false;
#pragma unroll
    for (int k = 0; k < kWin; ++k) {
      if (found || j - k < 0) continue;
      uint64_t v = w[k];
      if ((v >> 62) == 0) v = lookback_wait(base + (j - k) * stride, status);
      excl += v & kLbValueMask;
      if ((v >> 62) == 2) found = true;
    }
    if (found) break;
    j -= kWin;
  }
  return excl;
}

// Decoupled look-back for one value per block, run by warp 0 of the block.
// Publishes the block aggregate, then the warp reads 32 predecessors per
// round trip and sums them back to the nearest inclusive prefix; publishes
// the block's inclusive prefix and returns the exclusive prefix (to all lanes
// of warp 0).
__device__ uint64_t warp_block_lookback(uint64_t* lb, uint32_t idx, uint64_t aggregate,
                                        uint32_t* status) {
  const int lane = threadIdx.x & 31;
  if (idx == 0) {
    if (lane == 0) st_relaxed_u64(&lb[0], kLbPrefix | aggregate);
    return 0;
  }
  if (lane == 0) st_relaxed_u64(&lb[idx], kLbAggregate | aggregate);
  uint64_t excl = 0;
  int64_t base = (int64_t)idx - 1;
  while (true) {
    const int64_t j = base - lane;
    uint64_t w = j >= 0 ? ld_relaxed_u64(&lb[j]) : kLbPrefix;
    if ((w >> 62) == 0) w = lookback_wait(&lb[j], status);
    const uint32_t pre = __ballot_sync(0xffffffffu, (w >> 62) == 2);
    const int first = pre ? __ffs(pre) - 1 : 32;  // nearest inclusive prefix
    uint64_t val = lane <= first ? (w & kLbValueMask) : 0ull;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) val += __shfl_xor_sync(0xffffffffu, val, o);
    excl += val;
    if (pre) break;
    base -= 32;
  }
  if (lane == 0) st_relaxed_u64(&lb[idx], kLbPrefix | (excl + aggregate));
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
// culled ones, value = Gaussian index within its view. Also histograms the
// key digits of the presort passes.
__global__ void __launch_bounds__(256) k_depth_keys(const float4* __restrict__ bins, int n,
                                                   int n_views, int passes,
                                                   uint64_t* __restrict__ keys,
                                                   uint32_t* __restrict__ vals,
                                                   unsigned long long* __restrict__ hist,
                                                   int64_t* __restrict__ n_items_out) {
  if (blockIdx.x == 0 && threadIdx.x == 0) *n_items_out = (int64_t)n * n_views;
  __shared__ uint32_t s_hist[8][kRadix];
  for (int k = threadIdx.x; k < 8 * kRadix; k += blockDim.x) (&s_hist[0][0])[k] = 0u;
  __syncthreads();
  const int64_t total = (int64_t)n * n_views;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const uint32_t lt = lanemask_lt();
  // uniform trip count per warp so the match.any below sees every lane
  for (int64_t j0 = (int64_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31); j0 < total;
       j0 += stride) {
    const int64_t j = j0 + (threadIdx.x & 31);
    const bool in = j < total;
    uint64_t key = ~0ull;
    if (in) {
      const float4 r2 = __ldg(&bins[j]);  // depth key, tile_x, tile_y
      const uint32_t txw = __float_as_uint(r2.y), tyw = __float_as_uint(r2.z);
      const bool vis = (txw & 0xffffu) <= (txw >> 16) && (tyw & 0xffffu) <= (tyw >> 16);
      const int view = (int)(j / n);
      key = vis ? (((uint64_t)view << 32) | (uint64_t)__float_as_uint(r2.x)) : ~0ull;
      keys[j] = key;
      vals[j] = (uint32_t)(j - (int64_t)view * n);
    }
    // warp-aggregated histogram: one shared atomic per distinct digit
    for (int d = 0; d < passes; ++d) {
      const uint32_t dv = in ? (uint32_t)((key >> (8 * d)) & 0xff) : 256u;
      const uint32_t peers = __match_any_sync(0xffffffffu, dv);
      if (in && (peers & lt) == 0) atomicAdd(&s_hist[d][dv], (uint32_t)__popc(peers));
    }
  }
  __syncthreads();
  for (int k = threadIdx.x; k < passes * kRadix; k += blockDim.x) {
    const uint32_t c = (&s_hist[0][0])[k];
    if (c) atomicAdd(&hist[k], (unsigned long long)c);
  }
}

// ---------------------------------------------------------------------------
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
// Histograms of the following radix passes (digit d into hist[d][256] for
// d < passes): depth digits once per item weighted by its pair count, tile
// byte 0 per pair, higher tile bytes as per-thread runs.
template <int MODE, typename K>
__global__ void __launch_bounds__(kEmitThreads) k_emit(
    const float4* __restrict__ bins, const uint64_t* __restrict__ pkeys,
    const uint32_t* __restrict__ pvals, int n, int n_views, Grid g, int passes,
    K* __restrict__ keys_out, uint32_t* __restrict__ ids_out, int64_t capacity,
    int64_t* __restrict__ n_pairs, unsigned long long* __restrict__ hist,
    uint64_t* __restrict__ lookback, uint32_t* __restrict__ block_counter,
    uint32_t* __restrict__ status) {
  constexpr int kPer = MODE == 0 ? 4 : 8;           // pairs per thread per window
  constexpr int kWin = kPer * kEmitThreads;         // pairs per window
  constexpr int kWinPad = kWin + kWin / 32;
  constexpr int kTileDigit0 = MODE == 0 ? 4 : 0;    // digit index of tile byte 0
  __shared__ uint32_t s_off[kEmitItems + 1];
  __shared__ uint32_t s_rx[kEmitItems];   // x0 | width << 16
  __shared__ uint32_t s_ry[kEmitItems];   // y0 | view << 16
  __shared__ uint32_t s_id[kEmitItems];
  __shared__ uint32_t s_depth[MODE == 0 ? kEmitItems : 1];
  __shared__ uint32_t s_hist[8][kRadix];
  __shared__ K s_key[kWinPad];
  __shared__ uint32_t s_sid[kWinPad];
  __shared__ uint32_t s_warp[9];
  __shared__ uint64_t s_base;

  const uint32_t bidx = get_block_index(block_counter);
  const int64_t n_items = (int64_t)n * n_views;
  const int64_t first = (int64_t)bidx * kEmitItems;
  for (int k = threadIdx.x; k < 8 * kRadix; k += kEmitThreads) (&s_hist[0][0])[k] = 0u;

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
    const uint64_t base = warp_block_lookback(lookback, bidx, block_total, status);
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

  // depth digits are shared by all pairs of a Gaussian: count them per item
  if (MODE == 0) {
#pragma unroll
    for (int k = 0; k < kEmitItemsPerThread; ++k) {
      if (!cnt[k]) continue;
      const uint32_t dbits = s_depth[threadIdx.x * kEmitItemsPerThread + k];
#pragma unroll
      for (int d = 0; d < 4; ++d) atomicAdd(&s_hist[d][(dbits >> (8 * d)) & 0xff], cnt[k]);
    }
  }

  const uint32_t tiles_x = (uint32_t)g.tiles_x, tpv = (uint32_t)g.tiles_per_view;
  const int n_tile_digits = passes - kTileDigit0;
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
      uint32_t run_v[3] = {0u, 0u, 0u}, run_n[3] = {0u, 0u, 0u};
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
        atomicAdd(&s_hist[kTileDigit0][tile & 255u], 1u);
#pragma unroll
        for (int dd = 1; dd < 4; ++dd) {
          if (dd >= n_tile_digits) break;
          const uint32_t dv = (tile >> (8 * dd)) & 255u;
          if (run_n[dd - 1] && dv != run_v[dd - 1]) {
            atomicAdd(&s_hist[kTileDigit0 + dd][run_v[dd - 1]], run_n[dd - 1]);
            run_n[dd - 1] = 0;
          }
          run_v[dd - 1] = dv;
          ++run_n[dd - 1];
        }
        if (++col == w) {
          col = 0;
          ++row;
        }
      }
#pragma unroll
      for (int dd = 1; dd < 4; ++dd)
        if (run_n[dd - 1]) atomicAdd(&s_hist[kTileDigit0 + dd][run_v[dd - 1]], run_n[dd - 1]);
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
  for (int k = threadIdx.x; k < passes * kRadix; k += kEmitThreads) {
    const uint32_t c = (&s_hist[0][0])[k];
    if (c) atomicAdd(&hist[k], (unsigned long long)c);
  }
}

// Clear the look-back words of `passes` regions for the pair count now in
// *n_items (device), partitions of kSortTile keys.
__global__ void k_clear_lookback(uint64_t* __restrict__ lb, const int64_t* __restrict__ n_items,
                                 int64_t capacity, int passes, int64_t region_words) {
  const int64_t n = *n_items;
  if (n > capacity) return;
  const int64_t words = ((n + kSortTile - 1) / kSortTile) * kRadix;
  for (int p = 0; p < passes; ++p) {
    uint64_t* base = lb + p * region_words;
    for (int64_t w = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; w < words;
         w += (int64_t)gridDim.x * blockDim.x)
      base[w] = 0ull;
  }
}

// Blocks per SM of the radix pass, by key width (register budget).
template <typename K>
struct SortOcc;
template <>
struct SortOcc<uint32_t> {
  static constexpr int kBlocks = 3;
};
template <>
struct SortOcc<uint64_t> {
  static constexpr int kBlocks = 2;
};

// One stable LSD radix pass over digit (key >> shift) & 0xff.
// Per partition of kSortTile keys: (1) all keys and values are loaded first
// (independent loads in flight together); (2) per-warp digit counts with
// shared-memory atomics; (3) per digit, the counts over warps give each
// warp's offset and the block's count, which is published to the look-back
// array at once, before ranking; (4) each warp ranks its keys stably with
// match.any over warp-striped steps; (5) scatter into shared memory in
// sorted order; (6) look-back for the global offset of every digit (32
// predecessors per round trip); (7) write runs of equal digits to global
// memory.
template <typename K>
__global__ void __launch_bounds__(kSortThreads, SortOcc<K>::kBlocks) k_onesweep(
    const K* __restrict__ keys_in, const uint32_t* __restrict__ vals_in,
    K* __restrict__ keys_out, uint32_t* __restrict__ vals_out,
    const int64_t* __restrict__ n_ptr, int64_t capacity, int shift,
    const unsigned long long* __restrict__ hist, uint64_t* __restrict__ lookback,
    uint32_t* __restrict__ part_counter, uint32_t* __restrict__ status) {
  // layout: 64-bit arrays first so every carve-out is naturally aligned
  extern __shared__ __align__(16) unsigned char smem_raw[];
  uint64_t* s_gexcl = reinterpret_cast<uint64_t*>(smem_raw);            // [256]
  uint64_t* s_gbase = s_gexcl + kRadix;                                 // [256]
  K* s_keys = reinterpret_cast<K*>(s_gbase + kRadix);                   // [tile]
  uint32_t* s_vals = reinterpret_cast<uint32_t*>(s_keys + kSortTile);   // [tile]
  uint32_t* s_whist = s_vals + kSortTile;                               // [warps][257]
  uint32_t* s_lstart = s_whist + kSortWarps * (kRadix + 1);             // [256]
  uint32_t* s_scan = s_lstart + kRadix;                                 // [16]
  __shared__ uint32_t s_part;

  const int64_t n = *n_ptr;
  if (n > capacity || n <= 0) return;
  const int64_t parts = (n + kSortTile - 1) / kSortTile;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  // global exclusive prefix of this digit's histogram (same for every block)
  {
    const unsigned long long c = hist[tid];
    unsigned long long incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      unsigned long long y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    __shared__ unsigned long long s_w[8];
    if (lane == 31) s_w[warp] = incl;
    __syncthreads();
    unsigned long long wo = 0;
    for (int w = 0; w < warp; ++w) wo += s_w[w];
    s_gexcl[tid] = wo + incl - c;
    __syncthreads();
  }

  uint32_t* wh = s_whist + warp * (kRadix + 1);
  const uint32_t lt = lanemask_lt();
  while (true) {
    if (tid == 0) s_part = atomicAdd(part_counter, 1u);
    for (int k = tid; k < kSortWarps * (kRadix + 1); k += kSortThreads) s_whist[k] = 0u;
    __syncthreads();
    const int64_t p = s_part;
    if (p >= parts) break;
    const int64_t first = p * kSortTile + warp * (kSortItems * 32);

    // (1) loads, warp-striped: step `it` of this warp covers 32 consecutive keys
    K key[kSortItems];
    uint32_t val[kSortItems];
#pragma unroll
    for (int it = 0; it < kSortItems; ++it) {
      const int64_t idx = first + it * 32 + lane;
      key[it] = idx < n ? keys_in[idx] : (K)0;
      val[it] = idx < n ? vals_in[idx] : 0u;
    }
    // (2) per-warp digit counts (digit 256 marks an empty slot)
#pragma unroll
    for (int it = 0; it < kSortItems; ++it) {
      const int64_t idx = first + it * 32 + lane;
      const uint32_t d = idx < n ? (uint32_t)((key[it] >> shift) & 0xff) : (uint32_t)kRadix;
      atomicAdd(&wh[d], 1u);
    }
    __syncthreads();
    // (3) per digit: warp offsets, block count, early aggregate
    const int b = tid;  // 256 threads == 256 digits
    uint32_t count = 0;
#pragma unroll
    for (int w = 0; w < kSortWarps; ++w) {
      const uint32_t c = s_whist[w * (kRadix + 1) + b];
      s_whist[w * (kRadix + 1) + b] = count;
      count += c;
    }
    uint64_t* lb = lookback + p * kRadix + b;
    st_relaxed_u64(lb, (p == 0 ? kLbPrefix : kLbAggregate) | (uint64_t)count);
    uint32_t tot;
    const uint32_t lstart = block_exclusive_scan_256(count, s_scan, tot);
    s_lstart[b] = lstart;
    // running position of each digit for this warp = local start + warp offset
#pragma unroll
    for (int w = 0; w < kSortWarps; ++w) s_whist[w * (kRadix + 1) + b] += lstart;
    __syncthreads();
    // (4) stable rank within the warp -> final position within the partition
    uint32_t pos[kSortItems];
#pragma unroll
    for (int it = 0; it < kSortItems; ++it) {
      const int64_t idx = first + it * 32 + lane;
      const uint32_t d = idx < n ? (uint32_t)((key[it] >> shift) & 0xff) : (uint32_t)kRadix;
      const uint32_t peers = __match_any_sync(0xffffffffu, d);
      const uint32_t before = wh[d];
      __syncwarp();
      if ((peers & lt) == 0) wh[d] = before + __popc(peers);
      __syncwarp();
      pos[it] = before + __popc(peers & lt);
    }
    // (5) scatter into shared memory in sorted order (frees the registers)
#pragma unroll
    for (int it = 0; it < kSortItems; ++it) {
      const int64_t idx = first + it * 32 + lane;
      if (idx < n) {
        s_keys[pos[it]] = key[it];
        s_vals[pos[it]] = val[it];
      }
    }
    // (6) look-back: global start of each digit's run from this partition
    uint64_t excl = 0;
    if (p > 0) {
      excl = windowed_lookback<32>(lookback + b, kRadix, p, status);
      st_relaxed_u64(lb, kLbPrefix | (excl + count));
    }
    s_gbase[b] = s_gexcl[b] + excl;
    __syncthreads();
    // (7) write runs of equal digits out
    const int64_t remain = n - p * kSortTile;
    const int valid_count = remain < kSortTile ? (int)remain : kSortTile;
    for (int j = tid; j < valid_count; j += kSortThreads) {
      const K k = s_keys[j];
      const uint32_t d = (uint32_t)((k >> shift) & 0xff);
      const uint64_t gpos = s_gbase[d] + (uint64_t)(j - (int)s_lstart[d]);
      if (gpos < (uint64_t)n) {
        keys_out[gpos] = k;
        vals_out[gpos] = s_vals[j];
      } else {
        atomicOr(status, kStatusBounds);
      }
    }
    __syncthreads();
  }
}

// Tile id of a sorted key.
template <typename K>
__device__ __forceinline__ uint32_t tile_of(K k) {
  return (uint32_t)(((uint64_t)k) >> (KeyTraits<K>::kBits == 64 ? 32 : 0));
}

// [start, end) of every tile present in the sorted keys. Each thread takes 8
// consecutive keys with vector loads (a full chunk) and compares neighbours.
template <typename K>
__global__ void k_ranges(const K* __restrict__ keys, const int64_t* __restrict__ n_ptr,
                         int64_t capacity, int64_t n_tiles, int64_t* __restrict__ ranges,
                         uint32_t* __restrict__ status) {
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

size_t sort_smem_bytes(int key_bytes) {
  return (size_t)kRadix * 8 * 2 + (size_t)kSortTile * key_bytes + (size_t)kSortTile * 4 +
         (size_t)kSortWarps * (kRadix + 1) * 4 + (size_t)kRadix * 4 + 16 * 4;
}

template <typename K>
cudaError_t run_onesweep_passes(K* keys_a, uint32_t* vals_a, K* keys_b, uint32_t* vals_b,
                                const int64_t* n_ptr, int64_t capacity, int first_digit,
                                int passes, const unsigned long long* hist,
                                uint64_t* lookback, int64_t region_words, uint32_t* counters,
                                uint32_t* status, int grid, cudaStream_t stream) {
  const size_t smem = sort_smem_bytes(sizeof(K));
  cudaError_t e = cudaFuncSetAttribute(k_onesweep<K>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  K* kin = keys_a;
  uint32_t* vin = vals_a;
  K* kout = keys_b;
  uint32_t* vout = vals_b;
  for (int p = 0; p < passes; ++p) {
    const int d = first_digit + p;
    k_onesweep<K><<<grid, kSortThreads, smem, stream>>>(
        kin, vin, kout, vout, n_ptr, capacity, 8 * d, hist + (size_t)d * kRadix,
        lookback + (size_t)p * region_words, counters + p, status);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    K* tk = kin; kin = kout; kout = tk;
    uint32_t* tv = vin; vin = vout; vout = tv;
  }
  return cudaSuccess;
}

int sort_grid(int key_bytes, int64_t max_items) {
  int dev = 0, sms = 148, per_sm = 2;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const size_t smem = sort_smem_bytes(key_bytes);
  if (key_bytes == 8) {
    cudaFuncSetAttribute(k_onesweep<uint64_t>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_onesweep<uint64_t>, kSortThreads, smem);
  } else {
    cudaFuncSetAttribute(k_onesweep<uint32_t>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_onesweep<uint32_t>, kSortThreads, smem);
  }
  if (per_sm < 1) per_sm = 1;
  const int64_t parts = (max_items + kSortTile - 1) / kSortTile;
  int64_t grid = (int64_t)sms * per_sm;
  if (parts < grid) grid = parts;
  return grid < 1 ? 1 : (int)grid;
}

}  // namespace

int64_t sort_partitions(int64_t items) { return (items + kSortTile - 1) / kSortTile; }
int64_t emit_blocks(int64_t items) { return (items + kEmitItems - 1) / kEmitItems; }

cudaError_t launch_bin_sort(const BinSortArgs& a, cudaStream_t stream) {
  cudaError_t e;
  const int64_t n_items = (int64_t)a.n * a.n_views;
  const auto rec4 = reinterpret_cast<const float4*>(a.bins);
  if (n_items == 0) {
    return cudaMemsetAsync(a.n_pairs, 0, sizeof(int64_t), stream);
  }
  const int64_t lb_region = a.lookback_region_words;
  if (a.mode == GS_SORT_PRESORT) {
    // 1) keys (view << 32 | depth) over all Gaussians of all views
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    int64_t blocks = (n_items + 255) / 256;
    if (blocks > (int64_t)sms * 8) blocks = (int64_t)sms * 8;
    k_depth_keys<<<(int)blocks, 256, 0, stream>>>(rec4, a.n, a.n_views, a.presort_passes,
                                                 a.pkeys[0], a.pvals[0], a.presort_hist,
                                                 a.n_items_dev);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // the presort look-back regions are sized for n_items (host-known)
    e = cudaMemsetAsync(a.lookback, 0,
                        (size_t)a.presort_passes * lb_region * sizeof(uint64_t), stream);
    if (e != cudaSuccess) return e;
    e = run_onesweep_passes<uint64_t>(a.pkeys[0], a.pvals[0], a.pkeys[1], a.pvals[1],
                                      a.n_items_dev, n_items, 0, a.presort_passes,
                                      a.presort_hist, a.lookback, lb_region, a.counters + 8,
                                      a.status, sort_grid(8, n_items), stream);
    if (e != cudaSuccess) return e;
    const int fin = a.presort_passes & 1;
    // 2) emission in depth order, 32-bit tile keys
    const int64_t eb = emit_blocks(n_items);
    k_emit<1, uint32_t><<<(unsigned)eb, kEmitThreads, 0, stream>>>(
        rec4, a.pkeys[fin], a.pvals[fin], a.n, a.n_views, a.grid, a.pair_passes,
        reinterpret_cast<uint32_t*>(a.keys[a.emit_buf]), a.vals[a.emit_buf], a.capacity,
        a.n_pairs, a.hist, a.emit_lookback, a.counters + 0, a.status);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    k_clear_lookback<<<sms * 4, 256, 0, stream>>>(a.lookback, a.n_pairs, a.capacity,
                                                  a.pair_passes, lb_region);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    e = run_onesweep_passes<uint32_t>(
        reinterpret_cast<uint32_t*>(a.keys[a.emit_buf]), a.vals[a.emit_buf],
        reinterpret_cast<uint32_t*>(a.keys[a.emit_buf ^ 1]), a.vals[a.emit_buf ^ 1], a.n_pairs,
        a.capacity, 0, a.pair_passes, a.hist, a.lookback, lb_region, a.counters + 1, a.status,
        sort_grid(4, a.capacity), stream);
    if (e != cudaSuccess) return e;
    const int out = a.emit_buf ^ (a.pair_passes & 1);
    k_ranges<uint32_t><<<sms * 4, 256, 0, stream>>>(reinterpret_cast<uint32_t*>(a.keys[out]),
                                                   a.n_pairs, a.capacity, a.n_tiles, a.ranges, a.status);
    return cudaGetLastError();
  }
  // full 64-bit keys
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t eb = emit_blocks(n_items);
  k_emit<0, uint64_t><<<(unsigned)eb, kEmitThreads, 0, stream>>>(
      rec4, nullptr, nullptr, a.n, a.n_views, a.grid, a.pair_passes, a.keys[a.emit_buf],
      a.vals[a.emit_buf], a.capacity, a.n_pairs, a.hist, a.emit_lookback, a.counters + 0,
      a.status);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  k_clear_lookback<<<sms * 4, 256, 0, stream>>>(a.lookback, a.n_pairs, a.capacity, a.pair_passes,
                                                lb_region);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  e = run_onesweep_passes<uint64_t>(a.keys[a.emit_buf], a.vals[a.emit_buf], a.keys[a.emit_buf ^ 1],
                                    a.vals[a.emit_buf ^ 1], a.n_pairs, a.capacity, 0,
                                    a.pair_passes, a.hist, a.lookback, lb_region, a.counters + 1,
                                    a.status, sort_grid(8, a.capacity), stream);
  if (e != cudaSuccess) return e;
  const int out = a.emit_buf ^ (a.pair_passes & 1);
  k_ranges<uint64_t><<<sms * 4, 256, 0, stream>>>(a.keys[out], a.n_pairs, a.capacity, a.n_tiles,
                                                 a.ranges, a.status);
  return cudaGetLastError();
}

}  // namespace gsb
