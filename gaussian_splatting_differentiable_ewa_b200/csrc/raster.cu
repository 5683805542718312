// raster.cu -- tile rasteriser, forward and backward, sm_100a.
//
// One 16x16 tile per 256-thread block, one thread per pixel ("Better Gaussian
// Splatting in Julia", pwwt.cn sec. 5.4: a pixel block per thread group, each
// group compositing serially, groups in parallel -- no atomics on pixels).
// The tile's depth-sorted list is consumed in batches of 256 records; each
// thread stages one 48-byte record into shared memory with a TMA bulk copy
// (cp.async.bulk, completing on an mbarrier), double-buffered so the next
// batch is in flight while the current one is blended.
//
// Forward (pwwt.cn sec. 3.3 `composite`, front to back; lshu.cn sec. 3.2
// `blend`): alpha = min(0.99, o exp(-q/2)); skip alpha < 1/255; stop before a
// Gaussian that would take T below 1e-4; a block leaves its list once every
// thread is done (block-wide vote at batch boundaries, warps leave the inner
// loop as soon as all their lanes are done).
//
// Backward: each pixel replays its contributors back to front, recovering
// T_k = T_{k+1} / (1 - alpha_k) and the colour behind,
//   dC/dc_k = alpha_k T_k,
//   dC/dalpha_k = T_k (c_k - B_k) - T_final bg / (1 - alpha_k),
// B_k = alpha_{k+1} c_{k+1} + (1 - alpha_{k+1}) B_{k+1}. Per Gaussian the
// warp sums its pixels' terms with shuffles, the block sums its warps in
// shared memory, and one vector atomic per 4 floats goes to global memory.

#include <cuda_runtime.h>

#include "gs_internal.h"

namespace gsb {
namespace {

constexpr int kBatch = kTilePixels;          // records per batch
constexpr int kRecBytes = GS_RECORD_FLOATS * 4;  // 48

struct RasterGeom {
  Grid g;
  int n;
  int64_t capacity;  // length of ids
};

// A tile's [start, end) slice, clipped to the ids buffer (a malformed range
// renders as empty instead of reading outside the buffer).
__device__ __forceinline__ void tile_range(const int64_t* ranges, int tile, int64_t capacity,
                                           int64_t& start, int64_t& end) {
  start = ranges[2 * (int64_t)tile];
  end = ranges[2 * (int64_t)tile + 1];
  if (start < 0 || end > capacity || end < start) start = end = 0;
}

__device__ __forceinline__ void tile_coords(const Grid& g, int tile, int& view, int& px, int& py) {
  view = tile / g.tiles_per_view;
  const int t = tile - view * g.tiles_per_view;
  const int ty = t / g.tiles_x;
  const int tx = t - ty * g.tiles_x;
  px = tx * kTile + (threadIdx.x & (kTile - 1));
  py = ty * kTile + (threadIdx.x >> 4);
}

__global__ void __launch_bounds__(kTilePixels) k_raster_fwd(
    const float* __restrict__ records, const uint32_t* __restrict__ ids,
    const int64_t* __restrict__ ranges, RasterGeom geo, float bg0, float bg1, float bg2,
    float* __restrict__ image, float* __restrict__ final_T, uint32_t* __restrict__ n_contrib,
    uint32_t* __restrict__ status) {
  __shared__ __align__(128) float s_rec[2][kBatch][GS_RECORD_FLOATS];
  __shared__ __align__(8) uint64_t s_bar[2];

  const int tile = blockIdx.x;
  int view, px, py;
  tile_coords(geo.g, tile, view, px, py);
  const bool inside = px < geo.g.width && py < geo.g.height;
  int64_t start, end;
  tile_range(ranges, tile, geo.capacity, start, end);
  const int64_t cnt = end - start;
  const int nb = (int)((cnt + kBatch - 1) / kBatch);
  const float* rec_view = records + (size_t)view * geo.n * GS_RECORD_FLOATS;

  if (threadIdx.x == 0) {
    mbar_init(&s_bar[0], 1);
    mbar_init(&s_bar[1], 1);
    fence_mbar_init();
  }
  __syncthreads();

  auto issue = [&](int b) {
    const int buf = b & 1;
    const int64_t first = start + (int64_t)b * kBatch;
    const int64_t rem = end - first;
    const int m = rem < kBatch ? (int)rem : kBatch;
    if (threadIdx.x == 0) mbar_arrive_expect_tx(&s_bar[buf], (uint32_t)(m * kRecBytes));
    if ((int)threadIdx.x < m) {
      uint32_t id = __ldg(&ids[first + threadIdx.x]);
      if (id >= (uint32_t)geo.n) id = 0;  // never read outside the records
      bulk_copy_g2s(&s_rec[buf][threadIdx.x][0], rec_view + (size_t)id * GS_RECORD_FLOATS,
                    kRecBytes, &s_bar[buf]);
    }
  };

  const float pxc = (float)px + 0.5f, pyc = (float)py + 0.5f;
  float T = 1.f, c0 = 0.f, c1 = 0.f, c2 = 0.f;
  uint32_t last = 0;
  bool done = !inside;
  if (nb > 0) issue(0);
  int b = 0;
  for (; b < nb; ++b) {
    if (!__syncthreads_or(!done)) break;
    if (b + 1 < nb) issue(b + 1);
    if (!mbar_wait_bounded(&s_bar[b & 1], (uint32_t)((b >> 1) & 1), status)) {
      done = true;
      b = nb;  // a copy never landed: give up on the tile
      break;
    }
    const int64_t rem = cnt - (int64_t)b * kBatch;
    const int m = rem < kBatch ? (int)rem : kBatch;
    const float(*batch)[GS_RECORD_FLOATS] = s_rec[b & 1];
    for (int j = 0; j < m && !done; ++j) {
      const float4 r0 = *reinterpret_cast<const float4*>(&batch[j][0]);
      const float4 r1 = *reinterpret_cast<const float4*>(&batch[j][4]);
      const float rb = batch[j][R_B];
      const SplatEval e = splat_eval(pxc, pyc, r0.x, r0.y, r0.z, r0.w, r1.x, r1.y);
      if (e.alpha < kAlphaMin) continue;
      const float Tn = T * (1.f - e.alpha);
      if (Tn < kTMin) {
        done = true;
        break;
      }
      const float w = e.alpha * T;
      c0 = fmaf(r1.z, w, c0);
      c1 = fmaf(r1.w, w, c1);
      c2 = fmaf(rb, w, c2);
      T = Tn;
      last = (uint32_t)(b * kBatch + j + 1);
    }
  }
  // a batch issued but not consumed must land before the block exits
  if (b < nb) mbar_wait_bounded(&s_bar[b & 1], (uint32_t)((b >> 1) & 1), status);

  if (inside) {
    const size_t hw = (size_t)geo.g.width * geo.g.height;
    const size_t pix = (size_t)py * geo.g.width + px;
    float* img = image + (size_t)view * 3 * hw;
    img[pix] = c0 + T * bg0;
    img[hw + pix] = c1 + T * bg1;
    img[2 * hw + pix] = c2 + T * bg2;
    final_T[(size_t)view * hw + pix] = T;
    n_contrib[(size_t)view * hw + pix] = last;
  }
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__global__ void __launch_bounds__(kTilePixels) k_raster_bwd(
    const float* __restrict__ records, const uint32_t* __restrict__ ids,
    const int64_t* __restrict__ ranges, RasterGeom geo, float bg0, float bg1, float bg2,
    const float* __restrict__ dL_dimage, const float* __restrict__ final_T,
    const uint32_t* __restrict__ n_contrib, float* __restrict__ grad2d,
    uint32_t* __restrict__ status) {
  __shared__ __align__(128) float s_rec[2][kBatch][GS_RECORD_FLOATS];
  __shared__ __align__(16) float s_acc[kBatch][GS_GRAD2D_FLOATS];
  __shared__ uint32_t s_id[2][kBatch];
  __shared__ __align__(8) uint64_t s_bar[2];
  __shared__ uint32_t s_wmax[kTilePixels / 32];

  const int tile = blockIdx.x;
  int view, px, py;
  tile_coords(geo.g, tile, view, px, py);
  const bool inside = px < geo.g.width && py < geo.g.height;
  const size_t hw = (size_t)geo.g.width * geo.g.height;
  const size_t pix = (size_t)py * geo.g.width + px;
  int64_t start, end;
  tile_range(ranges, tile, geo.capacity, start, end);
  const float* rec_view = records + (size_t)view * geo.n * GS_RECORD_FLOATS;
  float* g2_view = grad2d + (size_t)view * geo.n * GS_GRAD2D_FLOATS;

  // per-pixel state
  float T = 1.f, Tfin = 1.f, g0 = 0.f, g1 = 0.f, g2 = 0.f;
  uint32_t my_nc = 0;
  if (inside) {
    Tfin = final_T[(size_t)view * hw + pix];
    T = Tfin;
    my_nc = n_contrib[(size_t)view * hw + pix];
    const float* gi = dL_dimage + (size_t)view * 3 * hw;
    g0 = gi[pix];
    g1 = gi[hw + pix];
    g2 = gi[2 * hw + pix];
  }
  const float bgg = bg0 * g0 + bg1 * g1 + bg2 * g2;
  float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f;  // colour behind, seen from just behind
  float last_a = 0.f, last_r = 0.f, last_g = 0.f, last_b = 0.f;

  // the longest prefix any pixel of the tile used
  uint32_t wm = __reduce_max_sync(0xffffffffu, my_nc);
  if ((threadIdx.x & 31) == 0) s_wmax[threadIdx.x >> 5] = wm;
  if (threadIdx.x == 0) {
    mbar_init(&s_bar[0], 1);
    mbar_init(&s_bar[1], 1);
    fence_mbar_init();
  }
  __syncthreads();
  uint32_t maxc = 0;
#pragma unroll
  for (int w = 0; w < kTilePixels / 32; ++w) maxc = max(maxc, s_wmax[w]);
  int64_t used = end - start;
  if ((int64_t)maxc < used) used = maxc;
  const int nb = (int)((used + kBatch - 1) / kBatch);

  // batches are consumed from the last (deepest) to the first
  auto issue = [&](int it) {
    const int b = nb - 1 - it;
    const int buf = it & 1;
    const int64_t first = start + (int64_t)b * kBatch;
    const int64_t rem = used - (int64_t)b * kBatch;
    const int m = rem < kBatch ? (int)rem : kBatch;
    if (threadIdx.x == 0) mbar_arrive_expect_tx(&s_bar[buf], (uint32_t)(m * kRecBytes));
    if ((int)threadIdx.x < m) {
      uint32_t id = __ldg(&ids[first + threadIdx.x]);
      if (id >= (uint32_t)geo.n) id = 0;  // never read outside the records
      s_id[buf][threadIdx.x] = id;
      bulk_copy_g2s(&s_rec[buf][threadIdx.x][0], rec_view + (size_t)id * GS_RECORD_FLOATS,
                    kRecBytes, &s_bar[buf]);
    }
  };

  const float pxc = (float)px + 0.5f, pyc = (float)py + 0.5f;
  const int lane = threadIdx.x & 31;
  if (nb > 0) issue(0);
  for (int it = 0; it < nb; ++it) {
    const int b = nb - 1 - it;
    const int buf = it & 1;
    __syncthreads();  // previous batch fully consumed and flushed
    if (it + 1 < nb) issue(it + 1);
#pragma unroll
    for (int k = 0; k < GS_GRAD2D_FLOATS; ++k) s_acc[threadIdx.x][k] = 0.f;
    // barrier: the accumulators are zeroed and this batch's ids are visible
    const bool ok =
        __syncthreads_and(mbar_wait_bounded(&s_bar[buf], (uint32_t)((it >> 1) & 1), status));
    if (!ok) break;
    const int64_t rem = used - (int64_t)b * kBatch;
    const int m = rem < kBatch ? (int)rem : kBatch;
    const float(*batch)[GS_RECORD_FLOATS] = s_rec[buf];
    for (int j = m - 1; j >= 0; --j) {
      const uint32_t pos = (uint32_t)(b * kBatch + j);
      bool contrib = inside && pos < my_nc;
      float v[10];
#pragma unroll
      for (int k = 0; k < 10; ++k) v[k] = 0.f;
      if (contrib) {
        const float4 r0 = *reinterpret_cast<const float4*>(&batch[j][0]);
        const float4 r1 = *reinterpret_cast<const float4*>(&batch[j][4]);
        const float rb = batch[j][R_B];
        const SplatEval e = splat_eval(pxc, pyc, r0.x, r0.y, r0.z, r0.w, r1.x, r1.y);
        if (e.alpha < kAlphaMin) {
          contrib = false;
        } else {
          const float one_m = 1.f - e.alpha;
          T = T / one_m;  // transmittance in front of this Gaussian
          const float w = e.alpha * T;
          v[6] = w * g0;
          v[7] = w * g1;
          v[8] = w * g2;
          acc0 = last_a * last_r + (1.f - last_a) * acc0;
          acc1 = last_a * last_g + (1.f - last_a) * acc1;
          acc2 = last_a * last_b + (1.f - last_a) * acc2;
          const float dLda = T * ((r1.z - acc0) * g0 + (r1.w - acc1) * g1 + (rb - acc2) * g2) -
                             Tfin * bgg / one_m;
          last_a = e.alpha;
          last_r = r1.z;
          last_g = r1.w;
          last_b = rb;
          if (e.alpha_raw < kAlphaMax) {
            const float dpow = e.alpha * dLda;  // d alpha / d power = alpha
            v[5] = e.G * dLda;                  // d alpha / d opacity = G
            const float du = dpow * (r0.z * e.dx + r0.w * e.dy);
            const float dv = dpow * (r0.w * e.dx + r1.x * e.dy);
            v[0] = du;
            v[1] = dv;
            v[2] = -0.5f * e.dx * e.dx * dpow;
            v[3] = -e.dx * e.dy * dpow;
            v[4] = -0.5f * e.dy * e.dy * dpow;
            v[9] = sqrtf(du * du + dv * dv);
          }
        }
      }
      if (__any_sync(0xffffffffu, contrib)) {
#pragma unroll
        for (int k = 0; k < 10; ++k) v[k] = warp_sum(v[k]);
        if (lane == 0) {
#pragma unroll
          for (int k = 0; k < 10; ++k) atomicAdd(&s_acc[j][k], v[k]);
        }
      }
    }
    __syncthreads();
    if ((int)threadIdx.x < m) {
      const float4 a = *reinterpret_cast<const float4*>(&s_acc[threadIdx.x][0]);
      const float4 bq = *reinterpret_cast<const float4*>(&s_acc[threadIdx.x][4]);
      const float4 c = *reinterpret_cast<const float4*>(&s_acc[threadIdx.x][8]);
      const bool nz = a.x != 0.f || a.y != 0.f || a.z != 0.f || a.w != 0.f || bq.x != 0.f ||
                      bq.y != 0.f || bq.z != 0.f || bq.w != 0.f || c.x != 0.f || c.y != 0.f;
      if (nz) {
        float* dst = g2_view + (size_t)s_id[buf][threadIdx.x] * GS_GRAD2D_FLOATS;
        red_add_v4(dst, a.x, a.y, a.z, a.w);
        red_add_v4(dst + 4, bq.x, bq.y, bq.z, bq.w);
        red_add_v4(dst + 8, c.x, c.y, 0.f, 0.f);
      }
    }
  }
}

}  // namespace

cudaError_t launch_raster_fwd(const float* records, const uint32_t* ids, const int64_t* ranges,
                              int64_t capacity, const Grid& g, int n_views, int n,
                              const float bg[3], float* image, float* final_T,
                              uint32_t* n_contrib, uint32_t* status, cudaStream_t stream) {
  const int64_t tiles = (int64_t)g.tiles_per_view * n_views;
  if (tiles == 0) return cudaSuccess;
  RasterGeom geo{g, n, n > 0 ? capacity : 0};
  k_raster_fwd<<<(unsigned)tiles, kTilePixels, 0, stream>>>(records, ids, ranges, geo, bg[0], bg[1],
                                                            bg[2], image, final_T, n_contrib, status);
  return cudaGetLastError();
}

cudaError_t launch_raster_bwd(const float* records, const uint32_t* ids, const int64_t* ranges,
                              int64_t capacity, const Grid& g, int n_views, int n,
                              const float bg[3], const float* dL_dimage, const float* final_T,
                              const uint32_t* n_contrib, float* grad2d, uint32_t* status,
                              cudaStream_t stream) {
  const int64_t tiles = (int64_t)g.tiles_per_view * n_views;
  if (tiles == 0) return cudaSuccess;
  RasterGeom geo{g, n, n > 0 ? capacity : 0};
  k_raster_bwd<<<(unsigned)tiles, kTilePixels, 0, stream>>>(records, ids, ranges, geo, bg[0], bg[1],
                                                            bg[2], dL_dimage, final_T, n_contrib,
                                                            grad2d, status);
  return cudaGetLastError();
}

}  // namespace gsb
