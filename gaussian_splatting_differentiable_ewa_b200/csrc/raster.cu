// raster.cu -- tile rasteriser, forward and backward, sm_100a.
//
// One 16x16 tile per 256-thread block, one thread per pixel ("Better Gaussian
// Splatting in Julia", pwwt.cn sec. 5.4: a pixel block per thread group, each
// group compositing serially, groups in parallel -- no atomics on pixels).
// Each warp owns an 8x4 pixel block of the tile.
//
// The tile's depth-sorted list is consumed in batches of 256 records; each
// thread stages one 48-byte record into shared memory with a TMA bulk copy
// (cp.async.bulk completing on an mbarrier), double-buffered so the next batch
// is in flight while the current one is blended. When a batch lands, thread j
// rewrites record j into evaluation form (log2-scaled conic, log2 opacity) and
// marks which warps' pixel blocks its alpha >= 1/255 box reaches; every warp
// then compacts the batch to the records that can touch its pixels (ballot +
// popc, order kept) and walks only those. The box is conservative, so the
// skipped records are exactly ones every pixel of the block would skip.
//
// Forward (pwwt.cn sec. 3.3 `composite`, front to back; lshu.cn sec. 3.2
// `blend`): alpha = min(0.99, o exp(-q/2)); skip alpha < 1/255; stop before a
// Gaussian that would take T below 1e-4; a warp stops once all its lanes are
// done and a block once all its warps are (votes).
//
// Backward: each pixel replays its contributors back to front, recovering
// T_k = T_{k+1} / (1 - alpha_k) and the colour behind,
//   dC/dc_k = alpha_k T_k,
//   dC/dalpha_k = T_k (c_k - B_k) - T_final bg / (1 - alpha_k),
// B_k = alpha_{k+1} c_{k+1} + (1 - alpha_{k+1}) B_{k+1}. Per Gaussian the warp
// sums its lanes' ten terms with a transposing butterfly (16 shuffles, each
// lane ends with one total), the block sums its warps in shared memory, and
// three 4-float vector atomics go to global memory.

#include <cuda_runtime.h>

#include "gs_internal.h"

namespace gsb {
namespace {

constexpr int kBatch = kTilePixels;              // records per batch
constexpr int kRecBytes = GS_RECORD_FLOATS * 4;  // 48
constexpr int kWarps = kTilePixels / 32;         // 8 warps, 8x4 pixels each
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kLog2AlphaMin = -7.994353436858858f;  // log2(1/255)

// Evaluation-form record slots (after the per-batch rewrite in shared memory):
// 0 u, 1 v, 2 A = -log2(e)/2 conic_a, 3 B = -log2(e) conic_b,
// 4 C = -log2(e)/2 conic_c, 5 log2(opacity), 6..8 colour, 9 1/opacity.
enum EvalSlot { E_U = 0, E_V = 1, E_A = 2, E_B = 3, E_C = 4, E_LO = 5, E_R = 6, E_G = 7,
                E_BL = 8, E_IO = 9 };

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

struct TilePix {
  int view, x0, y0, px, py;
};

__device__ __forceinline__ TilePix tile_pixel(const Grid& g, int tile) {
  TilePix t;
  t.view = tile / g.tiles_per_view;
  const int tt = tile - t.view * g.tiles_per_view;
  const int ty = tt / g.tiles_x;
  t.x0 = (tt - ty * g.tiles_x) * kTile;
  t.y0 = ty * kTile;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  t.px = t.x0 + 8 * (warp & 1) + (lane & 7);
  t.py = t.y0 + 4 * (warp >> 1) + (lane >> 3);
  return t;
}

// log2 of the unclamped alpha at pixel centre (pxc, pyc): the one
// expression both directions use, so their skip / stop decisions agree.
__device__ __forceinline__ float eval_log2_alpha(const float* r, float pxc, float pyc, float& dx,
                                                 float& dy) {
  dx = pxc - r[E_U];
  dy = pyc - r[E_V];
  return fmaf(r[E_A] * dx, dx, fmaf(r[E_B] * dx, dy, fmaf(r[E_C] * dy, dy, r[E_LO])));
}

// Rewrite record j of a landed batch into evaluation form and return the
// 8-bit mask of warps whose pixel block its alpha >= 1/255 box overlaps.
__device__ __forceinline__ uint32_t prepare_record(float* r, int x0, int y0) {
  const float u = r[R_U], v = r[R_V], hx = r[R_HX], hy = r[R_HY];
  const float o = r[R_OPAC];
  const float ca = r[R_CA], cb = r[R_CB], cc = r[R_CC];
  r[E_A] = -0.5f * kLog2e * ca;
  r[E_B] = -kLog2e * cb;
  r[E_C] = -0.5f * kLog2e * cc;
  r[E_LO] = __log2f(o);
  r[E_IO] = 1.f / o;
  if (!(hx >= 0.f)) return 0u;
  // pixel-centre extents of the warp blocks: x blocks of 8, y blocks of 4
  uint32_t xm = 0, ym = 0;
#pragma unroll
  for (int bx = 0; bx < 2; ++bx) {
    const float lo = (float)(x0 + 8 * bx) + 0.5f, hi = lo + 7.f;
    if (u + hx >= lo && u - hx <= hi) xm |= 1u << bx;
  }
#pragma unroll
  for (int by = 0; by < 4; ++by) {
    const float lo = (float)(y0 + 4 * by) + 0.5f, hi = lo + 3.f;
    if (v + hy >= lo && v - hy <= hi) ym |= 1u << by;
  }
  uint32_t mask = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w)
    if (((xm >> (w & 1)) & 1u) && ((ym >> (w >> 1)) & 1u)) mask |= 1u << w;
  return mask;
}

// Warp-wide compaction of the batch entries whose mask has this warp's bit,
// in batch order. Returns the count.
__device__ __forceinline__ int warp_list(const uint8_t* s_mask, uint8_t* list, int m) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t lt = lanemask_lt();
  int cnt = 0;
#pragma unroll
  for (int c = 0; c < kBatch / 32; ++c) {
    const int j = c * 32 + lane;
    const bool bit = j < m && ((s_mask[j] >> warp) & 1u);
    const uint32_t bal = __ballot_sync(0xffffffffu, bit);
    if (bit) list[cnt + __popc(bal & lt)] = (uint8_t)j;
    cnt += __popc(bal);
  }
  __syncwarp();
  return cnt;
}

__global__ void __launch_bounds__(kTilePixels) k_raster_fwd(
    const float* __restrict__ records, const uint32_t* __restrict__ ids,
    const int64_t* __restrict__ ranges, RasterGeom geo, float bg0, float bg1, float bg2,
    float* __restrict__ image, float* __restrict__ final_T, uint32_t* __restrict__ n_contrib,
    uint32_t* __restrict__ status) {
  __shared__ __align__(128) float s_rec[2][kBatch][GS_RECORD_FLOATS];
  __shared__ __align__(8) uint64_t s_bar[2];
  __shared__ uint8_t s_mask[kBatch];
  __shared__ uint8_t s_list[kWarps][kBatch];

  const int tile = blockIdx.x;
  const TilePix tp = tile_pixel(geo.g, tile);
  const bool inside = tp.px < geo.g.width && tp.py < geo.g.height;
  int64_t start, end;
  tile_range(ranges, tile, geo.capacity, start, end);
  const int64_t cnt = end - start;
  const int nb = (int)((cnt + kBatch - 1) / kBatch);
  const float* rec_view = records + (size_t)tp.view * geo.n * GS_RECORD_FLOATS;
  const int warp = threadIdx.x >> 5;

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

  const float pxc = (float)tp.px + 0.5f, pyc = (float)tp.py + 0.5f;
  float T = 1.f, c0 = 0.f, c1 = 0.f, c2 = 0.f;
  uint32_t last = 0;
  bool done = !inside;
  if (nb > 0) issue(0);
  int b = 0;
  for (; b < nb; ++b) {
    if (!__syncthreads_or(!done)) break;  // block vote; also frees buffer (b+1)&1
    if (b + 1 < nb) issue(b + 1);
    const int buf = b & 1;
    if (!__syncthreads_and(mbar_wait_bounded(&s_bar[buf], (uint32_t)((b >> 1) & 1), status))) {
      b = nb;  // a copy never landed: give up on the tile
      break;
    }
    const int64_t rem = cnt - (int64_t)b * kBatch;
    const int m = rem < kBatch ? (int)rem : kBatch;
    if ((int)threadIdx.x < m) s_mask[threadIdx.x] = (uint8_t)prepare_record(&s_rec[buf][threadIdx.x][0], tp.x0, tp.y0);
    __syncthreads();
    const int wc = warp_list(s_mask, s_list[warp], m);
    for (int k = 0; k < wc; ++k) {
      if ((k & 3) == 0 && __all_sync(0xffffffffu, done)) break;  // warp vote
      if (done) continue;
      const int j = s_list[warp][k];
      const float* r = &s_rec[buf][j][0];
      float dx, dy;
      const float p = eval_log2_alpha(r, pxc, pyc, dx, dy);
      if (p < kLog2AlphaMin) continue;  // alpha < 1/255
      const float a = fminf(kAlphaMax, exp2f(p));
      const float Tn = T * (1.f - a);
      if (Tn < kTMin) {
        done = true;
        continue;
      }
      const float w = a * T;
      c0 = fmaf(r[E_R], w, c0);
      c1 = fmaf(r[E_G], w, c1);
      c2 = fmaf(r[E_BL], w, c2);
      T = Tn;
      last = (uint32_t)(b * kBatch + j + 1);
    }
  }
  // a batch issued but not consumed must land before the block exits
  if (b < nb) mbar_wait_bounded(&s_bar[b & 1], (uint32_t)((b >> 1) & 1), status);

  if (inside) {
    const size_t hw = (size_t)geo.g.width * geo.g.height;
    const size_t pix = (size_t)tp.py * geo.g.width + tp.px;
    float* img = image + (size_t)tp.view * 3 * hw;
    img[pix] = c0 + T * bg0;
    img[hw + pix] = c1 + T * bg1;
    img[2 * hw + pix] = c2 + T * bg2;
    final_T[(size_t)tp.view * hw + pix] = T;
    n_contrib[(size_t)tp.view * hw + pix] = last;
  }
}

// Transposing butterfly: v[0..15] per lane in, the warp total of value
// (lane >> 1) & 15 out (lanes 2k and 2k+1 both hold total k). 16 shuffles.
__device__ __forceinline__ float warp_sum16(const float (&v)[16]) {
  const int lane = threadIdx.x & 31;
  float a[8];
  const bool h16 = lane & 16;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const float send = h16 ? v[k] : v[k + 8];
    const float keep = h16 ? v[k + 8] : v[k];
    a[k] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
  }
  float b[4];
  const bool h8 = lane & 8;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float send = h8 ? a[k] : a[k + 4];
    const float keep = h8 ? a[k + 4] : a[k];
    b[k] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
  }
  float c[2];
  const bool h4 = lane & 4;
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const float send = h4 ? b[k] : b[k + 2];
    const float keep = h4 ? b[k + 2] : b[k];
    c[k] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
  }
  const bool h2 = lane & 2;
  float d = (h2 ? c[1] : c[0]) + __shfl_xor_sync(0xffffffffu, h2 ? c[0] : c[1], 2);
  d += __shfl_xor_sync(0xffffffffu, d, 1);
  return d;
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
  __shared__ uint32_t s_wmax[kWarps];
  __shared__ uint8_t s_mask[kBatch];
  __shared__ uint8_t s_list[kWarps][kBatch];

  const int tile = blockIdx.x;
  const TilePix tp = tile_pixel(geo.g, tile);
  const bool inside = tp.px < geo.g.width && tp.py < geo.g.height;
  const size_t hw = (size_t)geo.g.width * geo.g.height;
  const size_t pix = (size_t)tp.py * geo.g.width + tp.px;
  int64_t start, end;
  tile_range(ranges, tile, geo.capacity, start, end);
  const float* rec_view = records + (size_t)tp.view * geo.n * GS_RECORD_FLOATS;
  float* g2_view = grad2d + (size_t)tp.view * geo.n * GS_GRAD2D_FLOATS;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // per-pixel state
  float T = 1.f, Tfin = 1.f, g0 = 0.f, g1 = 0.f, g2 = 0.f;
  uint32_t my_nc = 0;
  if (inside) {
    Tfin = final_T[(size_t)tp.view * hw + pix];
    T = Tfin;
    my_nc = n_contrib[(size_t)tp.view * hw + pix];
    const float* gi = dL_dimage + (size_t)tp.view * 3 * hw;
    g0 = gi[pix];
    g1 = gi[hw + pix];
    g2 = gi[2 * hw + pix];
  }
  const float bgg = bg0 * g0 + bg1 * g1 + bg2 * g2;
  float acc0 = 0.f, acc1 = 0.f, acc2 = 0.f;  // colour behind, seen from just behind
  float last_a = 0.f, last_r = 0.f, last_g = 0.f, last_b = 0.f;

  // the longest prefix any pixel of the tile used
  const uint32_t wm = __reduce_max_sync(0xffffffffu, my_nc);
  if (lane == 0) s_wmax[warp] = wm;
  if (threadIdx.x == 0) {
    mbar_init(&s_bar[0], 1);
    mbar_init(&s_bar[1], 1);
    fence_mbar_init();
  }
  __syncthreads();
  uint32_t maxc = 0;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) maxc = max(maxc, s_wmax[w]);
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

  const float pxc = (float)tp.px + 0.5f, pyc = (float)tp.py + 0.5f;
  if (nb > 0) issue(0);
  for (int it = 0; it < nb; ++it) {
    const int b = nb - 1 - it;
    const int buf = it & 1;
    __syncthreads();  // previous batch fully consumed and flushed
    if (it + 1 < nb) issue(it + 1);
    const int64_t rem = used - (int64_t)b * kBatch;
    const int m = rem < kBatch ? (int)rem : kBatch;
    if (!__syncthreads_and(mbar_wait_bounded(&s_bar[buf], (uint32_t)((it >> 1) & 1), status)))
      break;
    if ((int)threadIdx.x < m)
      s_mask[threadIdx.x] = (uint8_t)prepare_record(&s_rec[buf][threadIdx.x][0], tp.x0, tp.y0);
#pragma unroll
    for (int k = 0; k < GS_GRAD2D_FLOATS; ++k) s_acc[threadIdx.x][k] = 0.f;
    __syncthreads();
    const int wc = warp_list(s_mask, s_list[warp], m);
    for (int k = wc - 1; k >= 0; --k) {
      const int j = s_list[warp][k];
      const uint32_t pos = (uint32_t)(b * kBatch + j);
      bool contrib = inside && pos < my_nc;
      float v[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) v[e] = 0.f;
      if (contrib) {
        const float* r = &s_rec[buf][j][0];
        float dx, dy;
        const float p = eval_log2_alpha(r, pxc, pyc, dx, dy);
        if (p < kLog2AlphaMin) {
          contrib = false;
        } else {
          const float a_raw = exp2f(p);
          const float a = fminf(kAlphaMax, a_raw);
          const float one_m = 1.f - a;
          T = T / one_m;  // transmittance in front of this Gaussian
          const float w = a * T;
          const float cr = r[E_R], cg = r[E_G], cbl = r[E_BL];
          v[6] = w * g0;
          v[7] = w * g1;
          v[8] = w * g2;
          acc0 = last_a * last_r + (1.f - last_a) * acc0;
          acc1 = last_a * last_g + (1.f - last_a) * acc1;
          acc2 = last_a * last_b + (1.f - last_a) * acc2;
          const float dLda = T * ((cr - acc0) * g0 + (cg - acc1) * g1 + (cbl - acc2) * g2) -
                             Tfin * bgg / one_m;
          last_a = a;
          last_r = cr;
          last_g = cg;
          last_b = cbl;
          if (a_raw < kAlphaMax) {
            const float dpow = a * dLda;       // d alpha / d (-q/2) = alpha
            v[5] = a * r[E_IO] * dLda;         // d alpha / d opacity = alpha / o
            // -q/2 = ln2 (A dx^2 + B dx dy + C dy^2) with dx = px - u
            const float du = -dpow * kLn2 * (2.f * r[E_A] * dx + r[E_B] * dy);
            const float dv = -dpow * kLn2 * (r[E_B] * dx + 2.f * r[E_C] * dy);
            v[0] = du;
            v[1] = dv;
            v[2] = -0.5f * dx * dx * dpow;
            v[3] = -dx * dy * dpow;
            v[4] = -0.5f * dy * dy * dpow;
            v[9] = sqrtf(du * du + dv * dv);
          }
        }
      }
      const uint32_t bal = __ballot_sync(0xffffffffu, contrib);
      if (bal == 0u) continue;
      if (__popc(bal) == 1) {
        if (contrib) {
#pragma unroll
          for (int e = 0; e < 10; ++e) atomicAdd(&s_acc[j][e], v[e]);
        }
      } else {
        const float tot = warp_sum16(v);
        const int idx = (lane >> 1) & 15;
        if ((lane & 1) == 0 && idx < 10) atomicAdd(&s_acc[j][idx], tot);
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
