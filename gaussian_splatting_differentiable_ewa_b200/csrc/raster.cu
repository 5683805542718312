// raster.cu -- tile rasteriser, forward and backward, sm_100a.
//
// One 16x16 tile per thread block ("Better Gaussian Splatting in Julia",
// pwwt.cn sec. 5.4: a pixel block per thread group, each group compositing
// serially, groups in parallel -- no atomics on pixels). Each thread takes
// 2 NP pixels of one column, four rows apart -- (x, y), (x, y + 4), ...,
// (x, y + 4 (2 NP - 1)) -- so a warp owns an 8-column block of 8 NP rows and
// a tile has 4 / NP warps. A thread's pixels share their x offset from every
// Gaussian centre (and with it half of the evaluation), and the per-pixel
// arithmetic runs two-wide on the FP32x2 pipe (__ffma2_rn / __fadd2_rn /
// __fmul2_rn: each half rounds exactly like the scalar operation, so pixel
// results do not depend on the grouping).
//
// The tile's depth-sorted list is consumed in batches of one record per
// thread; each thread stages one 64-byte record into shared memory with a TMA
// bulk copy (cp.async.bulk completing on an mbarrier). When a batch lands,
// thread j marks which warps' pixel blocks record j's alpha >= 1/255 ellipse
// reaches (its bounding box, then the ellipse itself against the block's
// rectangle); every warp then compacts the batch to the records that can
// touch its pixels (ballot + popc, order kept) and walks only those. The test
// is conservative, so the skipped records are exactly ones every pixel of the
// block would skip. The forward copies each landed record into a separate
// array of (x, x) pairs, so the landing buffer is free for the next batch's
// copy at once; the backward reads records in place and double-buffers.
//
// Per (pixel, splat) the record's evaluation form (see gs.h) gives
//   d = P - (uh, vh), p_i = w_i . d + c_i, zq = p1^2 + p2^2 + nlo
// with zq = -log2(255 alpha_raw): the splat counts iff zq <= 0, and
// alpha_raw = 2^-zq / 255. Sums of squares of well-scaled terms: the float
// result stays within a few units of float rounding of zq's magnitude also
// for elongated splats and for means far from the origin (the mean's float
// remainder is carried in c_i), with no cancellation as in the conic form.
//
// Forward (pwwt.cn sec. 3.3 `composite`, front to back; lshu.cn sec. 3.2
// `blend`): alpha = min(0.99, o exp(-q/2)); skip alpha < 1/255; stop before a
// Gaussian that would take T below 1e-4; a warp stops once all its pixels are
// done and a block once all its warps are (votes).
//
// Device-side conditions go to the status word: a list entry naming a
// Gaussian >= n is clipped to record 0 and masked out (it reaches no pixel),
// a range outside the ids buffer renders as empty (both kStatusBounds); a
// batch whose copy does not land within the wait limit ends the tile
// (kStatusTimeout), after waiting once more for any copy still in flight.
//
// Backward: each pixel replays its contributors back to front, recovering
// T_k = T_{k+1} / (1 - alpha_k), with B_k the colour composited behind k,
//   dC/dc_k = alpha_k T_k,
//   dC/dalpha_k = T_k (c_k - B_k) - T_final bg / (1 - alpha_k),
//   B_{k-1} = B_k + alpha_k (c_k - B_k).
// Per Gaussian a thread adds its pixels' ten terms, the warp sums its lanes
// with a transposing butterfly (14 shuffles), the block sums its warps in
// shared memory, and three 4-float vector atomics go to global memory.

#include <cuda_runtime.h>

#include "gs_internal.h"

namespace gsb {
namespace {

// Pixel pairs per thread of the kernels launched: 1 (two pixels per thread,
// 128-thread blocks of four warps, each warp an 8 x 8 pixel block). Two pairs
// (64-thread blocks, 8 x 16 blocks per warp) measured slower on the 1M-splat
// 1080p frame: forward 0.308 against 0.303 ms, backward 0.613 against 0.584
// ms -- fewer resident warps (80 and 111 registers) and longer warp lists
// outweigh the evaluation and reduction shared by four pixels.
constexpr int kPairs = 1;

template <int NP>
struct Shape {
  static constexpr int kThreads = 128 / NP;      // 2 NP pixels per thread, 256 per tile
  static constexpr int kWarps = kThreads / 32;   // 4 / NP
  static constexpr int kBatch = kThreads;        // records per batch: one per thread
  static constexpr int kBlockRows = 8 * NP;      // a warp's block: 8 columns x kBlockRows rows
};

constexpr int kRecBytes = GS_RECORD_FLOATS * 4;  // 64
constexpr float kInv255 = 1.0f / 255.0f;
constexpr float kTwoLn2 = 1.3862943611198906f;   // 1 / (log2(e) / 2)

static_assert(kRecBytes % 16 == 0, "bulk copies move multiples of 16 bytes");

// Forward evaluation form of a record, one (x, x) pair per field, so the
// multi-pixel arithmetic takes every operand straight from shared memory:
// -uh, -vh, w1x, w1y, c1, w2x, w2y, c2, nlo, colour r g b. 96 bytes.
enum EvPair { V_NU = 0, V_NV, V_W1X, V_W1Y, V_C1, V_W2X, V_W2Y, V_C2, V_NLO, V_R, V_G, V_BL,
              kEvPairs };

struct RasterGeom {
  Grid g;
  int n;
  int64_t capacity;  // length of ids
};

__device__ __forceinline__ float2 f2(float x) { return make_float2(x, x); }

// alpha_raw = 2^-zq / 255 (zq = -log2(255 alpha_raw)); both directions call
// this, so their alphas are bit-identical.
__device__ __forceinline__ float alpha_raw_of(float zq) { return exp2f(-zq) * kInv255; }

// A tile's [start, end) slice, clipped to the ids buffer (a malformed range
// renders as empty instead of reading outside the buffer, and is reported).
__device__ __forceinline__ void tile_range(const int64_t* ranges, int tile, int64_t capacity,
                                           int64_t& start, int64_t& end, uint32_t* status) {
  start = ranges[2 * (int64_t)tile];
  end = ranges[2 * (int64_t)tile + 1];
  if (start < 0 || end > capacity || end < start) {
    if (threadIdx.x == 0 && status) atomicOr(status, kStatusBounds);
    start = end = 0;
  }
}

// The thread's pixels: column px, rows py + 4 i for i < 2 NP; pair k holds
// rows py + 8k and py + 8k + 4.
template <int NP>
struct TilePix {
  int view, x0, y0, px, py;
  bool in[2 * NP];
};

template <int NP>
__device__ __forceinline__ TilePix<NP> tile_pixel(const Grid& g, int tile) {
  TilePix<NP> t;
  t.view = tile / g.tiles_per_view;
  const int tt = tile - t.view * g.tiles_per_view;
  const int ty = tt / g.tiles_x;
  t.x0 = (tt - ty * g.tiles_x) * kTile;
  t.y0 = ty * kTile;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  t.px = t.x0 + 8 * (warp & 1) + (lane & 7);
  t.py = t.y0 + Shape<NP>::kBlockRows * (warp >> 1) + (lane >> 3);
#pragma unroll
  for (int i = 0; i < 2 * NP; ++i) t.in[i] = t.px < g.width && t.py + 4 * i < g.height;
  return t;
}

// Mask of the warps whose pixel block (8 columns x kBlockRows rows) the
// alpha >= 1/255 box [u - hx, u + hx] x [v - hy, v + hy] overlaps, on
// pixel-centre extents (a record without a box, hx < 0 or NaN, reaches none).
template <int NP>
__device__ __forceinline__ uint32_t warp_block_mask(float u, float v, float hx, float hy, int x0,
                                                    int y0) {
  constexpr int R = Shape<NP>::kBlockRows;
  if (!(hx >= 0.f)) return 0u;
  uint32_t xm = 0, ym = 0;
#pragma unroll
  for (int bi = 0; bi < 2; ++bi) {
    const float xlo = (float)(x0 + 8 * bi) + 0.5f, xhi = xlo + 7.f;
    if (u + hx >= xlo && u - hx <= xhi) xm |= 1u << bi;
  }
#pragma unroll
  for (int bi = 0; bi < kTile / R; ++bi) {
    const float ylo = (float)(y0 + R * bi) + 0.5f, yhi = ylo + (float)(R - 1);
    if (v + hy >= ylo && v - hy <= yhi) ym |= 1u << bi;
  }
  uint32_t mask = 0;
#pragma unroll
  for (int w = 0; w < Shape<NP>::kWarps; ++w)
    if (((xm >> (w & 1)) & 1u) && ((ym >> (w >> 1)) & 1u)) mask |= 1u << w;
  return mask;
}

// Refines warp_block_mask with the ellipse itself: a warp's block of pixel
// centres [xlo, xlo + 7] x [ylo, ylo + kBlockRows - 1] keeps the splat only
// if the quadratic q'(d) = (w1 . d)^2 + (w2 . d)^2 (d from the float mean)
// reaches at most Q' = -nlo somewhere on that rectangle: 0 when the mean is
// inside, else the least value over the four edges (on an edge q' is a
// parabola in the free coordinate, minimised at its vertex clamped to the
// edge). Q' is padded (0.2 % + 0.01) well beyond the float rounding of the
// rasteriser's zq and the mean's float remainder, so no pixel the per-pixel
// test takes is dropped; the axis-aligned box alone keeps ~40 % more (warp,
// splat) pairs, whose ellipse misses the block.
template <int NP>
__device__ __forceinline__ uint32_t warp_block_mask_ellipse(const float* r, uint32_t box, int x0,
                                                            int y0) {
  constexpr int R = Shape<NP>::kBlockRows;
  if (box == 0u) return 0u;
  const float w1x = r[R_W1X], w1y = r[R_W1Y], w2x = r[R_W2X], w2y = r[R_W2Y];
  const float a = fmaf(w1x, w1x, w2x * w2x), b = fmaf(w1x, w1y, w2x * w2y);
  const float c = fmaf(w1y, w1y, w2y * w2y);
  const float ia = 1.f / a, ic = 1.f / c;
  const float qm = fmaf(-r[R_NLO], 1.002f, 0.01f);
  const float u = r[R_U], v = r[R_V];
  uint32_t mask = 0;
#pragma unroll
  for (int w = 0; w < Shape<NP>::kWarps; ++w) {
    if (!((box >> w) & 1u)) continue;
    const float ex0 = (float)(x0 + 8 * (w & 1)) + 0.5f - u, ex1 = ex0 + 7.f;
    const float ey0 = (float)(y0 + R * (w >> 1)) + 0.5f - v, ey1 = ey0 + (float)(R - 1);
    bool hit = ex0 <= 0.f && ex1 >= 0.f && ey0 <= 0.f && ey1 >= 0.f;
    float best = __int_as_float(0x7f800000);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float ex = e ? ex1 : ex0;  // vertical edges
      const float dy = fminf(fmaxf(-b * ex * ic, ey0), ey1);
      best = fminf(best, fmaf(a * ex, ex, fmaf(2.f * b * ex, dy, c * dy * dy)));
      const float ey = e ? ey1 : ey0;  // horizontal edges
      const float dx = fminf(fmaxf(-b * ey * ia, ex0), ex1);
      best = fminf(best, fmaf(c * ey, ey, fmaf(2.f * b * ey, dx, a * dx * dx)));
    }
    hit = hit || best <= qm;
    mask |= hit ? 1u << w : 0u;
  }
  return mask;
}

// Both tests on a record in its stored form, out of line: the backward runs
// it only when no forward masks are given, and inlined there its registers
// counted against the whole walk (70 registers, 7 blocks per SM, against 64
// and 8 out of line: 0.550 against 0.573 ms on the 1M-splat 1080p frame).
template <int NP>
__device__ __noinline__ uint32_t record_block_mask(const float* r, int x0, int y0) {
  return warp_block_mask_ellipse<NP>(
      r, warp_block_mask<NP>(r[R_U], r[R_V], r[R_HX], r[R_HY], x0, y0), x0, y0);
}

// The pixel-independent part of the evaluation at column pxc: dx = pxc - uh
// and a_i = fma(w_ix, dx, c_i), as (x, x) pairs.
struct EvCol {
  float2 a1, a2;
};

__device__ __forceinline__ EvCol eval_col(const float2* e, float2 pxc) {
  const float2 dx = __fadd2_rn(pxc, e[V_NU]);
  return EvCol{__ffma2_rn(e[V_W1X], dx, e[V_C1]), __ffma2_rn(e[V_W2X], dx, e[V_C2])};
}

// zq of a pixel pair of that column at rows pyc.x, pyc.y:
//   dy = pyc - vh, p_i = fma(w_iy, dy, a_i), zq = fma(p1, p1, fma(p2, p2, nlo)).
// The backward evaluates the same IEEE operations in the same order
// (eval_zq_s), so the skip / stop decisions of the two directions agree bit
// for bit.
__device__ __forceinline__ float2 eval_zq(const float2* e, const EvCol& col, float2 pyc) {
  const float2 dy = __fadd2_rn(pyc, e[V_NV]);
  const float2 p1 = __ffma2_rn(e[V_W1Y], dy, col.a1);
  const float2 p2 = __ffma2_rn(e[V_W2Y], dy, col.a2);
  return __ffma2_rn(p1, p1, __ffma2_rn(p2, p2, e[V_NLO]));
}

// Write the forward evaluation form of landed record r and return the mask
// of warps whose pixel block its alpha >= 1/255 ellipse reaches.
template <int NP>
__device__ __forceinline__ uint32_t prepare_record(const float* r, float2* e, int x0, int y0) {
  const float u = r[R_U], v = r[R_V];
  float4* e4 = reinterpret_cast<float4*>(e);
  e4[0] = make_float4(-u, -u, -v, -v);
  e4[1] = make_float4(r[R_W1X], r[R_W1X], r[R_W1Y], r[R_W1Y]);
  e4[2] = make_float4(r[R_C1], r[R_C1], r[R_W2X], r[R_W2X]);
  e4[3] = make_float4(r[R_W2Y], r[R_W2Y], r[R_C2], r[R_C2]);
  e4[4] = make_float4(r[R_NLO], r[R_NLO], r[R_R], r[R_R]);
  e4[5] = make_float4(r[R_G], r[R_G], r[R_B], r[R_B]);
  return warp_block_mask_ellipse<NP>(r, warp_block_mask<NP>(u, v, r[R_HX], r[R_HY], x0, y0), x0,
                                     y0);
}

// eval_col / eval_zq on a record in its stored (scalar) form, the same IEEE
// operations in the same order (the column part shared by the thread's
// pixels); also returns dx, dy and p1, p2 for the gradients.
__device__ __forceinline__ void eval_col_s(const float* r, float pxc, float& dx, float& a1,
                                           float& a2) {
  dx = __fsub_rn(pxc, r[R_U]);
  a1 = __fmaf_rn(r[R_W1X], dx, r[R_C1]);
  a2 = __fmaf_rn(r[R_W2X], dx, r[R_C2]);
}

__device__ __forceinline__ float2 eval_zq_s(const float* r, float a1, float a2, float2 pyc,
                                            float2& dy, float2& p1, float2& p2) {
  dy = __fadd2_rn(pyc, f2(-r[R_V]));
  p1 = __ffma2_rn(f2(r[R_W1Y]), dy, f2(a1));
  p2 = __ffma2_rn(f2(r[R_W2Y]), dy, f2(a2));
  return __ffma2_rn(p1, p1, __ffma2_rn(p2, p2, f2(r[R_NLO])));
}

// Warp-wide compaction of the batch entries j < m whose mask has this warp's
// bit, in batch order. Returns the count.
template <int NP>
__device__ __forceinline__ int warp_list(const uint8_t* s_mask, uint8_t* list, int m) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t lt = lanemask_lt();
  int cnt = 0;
#pragma unroll
  for (int c = 0; c < Shape<NP>::kBatch / 32; ++c) {
    const int j = c * 32 + lane;
    const bool bit = j < m && ((s_mask[j] >> warp) & 1u);
    const uint32_t bal = __ballot_sync(0xffffffffu, bit);
    if (bit) list[cnt + __popc(bal & lt)] = (uint8_t)j;
    cnt += __popc(bal);
  }
  __syncwarp();
  return cnt;
}

template <int NP>
__global__ void __launch_bounds__(Shape<NP>::kThreads) k_raster_fwd(
    const float* __restrict__ records, const uint32_t* __restrict__ ids,
    const int64_t* __restrict__ ranges, RasterGeom geo, float bg0, float bg1, float bg2,
    float* __restrict__ image, float* __restrict__ final_T, uint32_t* __restrict__ n_contrib,
    uint8_t* __restrict__ wmask_out, uint32_t* __restrict__ status, WaitCfg wc) {
  using Sh = Shape<NP>;
  constexpr int kBatch = Sh::kBatch;
  __shared__ __align__(128) float s_rec[kBatch][GS_RECORD_FLOATS];
  __shared__ __align__(16) float2 s_ev[kBatch][kEvPairs];
  __shared__ __align__(8) uint64_t s_bar;
  __shared__ uint8_t s_mask[kBatch];
  __shared__ uint8_t s_list[Sh::kWarps][kBatch];

  const int tile = blockIdx.x;
  const TilePix<NP> tp = tile_pixel<NP>(geo.g, tile);
  int64_t start, end;
  tile_range(ranges, tile, geo.capacity, start, end, status);
  const int64_t cnt = end - start;
  const int nb = (int)((cnt + kBatch - 1) / kBatch);
  const float* rec_view = records + (size_t)tp.view * geo.n * GS_RECORD_FLOATS;
  const int warp = threadIdx.x >> 5;
  // test hook: this tile issues no copies and waits in vain
  const bool stalled = (int64_t)tile == wc.stall;

  if (threadIdx.x == 0) {
    mbar_init(&s_bar, 1);
    fence_mbar_init();
  }
  __syncthreads();

  // batch b's records land in s_rec (one copy in flight at a time: a batch
  // is converted into s_ev as soon as it lands, which frees s_rec for the
  // next one while the current batch is blended)
  bool clipped = false;  // this thread's entry of the batch in flight named no Gaussian
  auto issue = [&](int b) {
    if (stalled) return;
    const int64_t first = start + (int64_t)b * kBatch;
    const int64_t rem = end - first;
    const int m = rem < kBatch ? (int)rem : kBatch;
    if (threadIdx.x == 0) mbar_arrive_expect_tx(&s_bar, (uint32_t)(m * kRecBytes));
    if ((int)threadIdx.x < m) {
      uint32_t id = __ldg(&ids[first + threadIdx.x]);
      clipped = id >= (uint32_t)geo.n;
      if (clipped) {  // never read outside the records
        id = 0;
        atomicOr(status, kStatusBounds);
      }
      bulk_copy_g2s(&s_rec[threadIdx.x][0], rec_view + (size_t)id * GS_RECORD_FLOATS, kRecBytes,
                    &s_bar);
    }
  };

  const float kInf = __int_as_float(0x7f800000);
  const float2 pxc = f2((float)tp.px + 0.5f);
  float2 pyc[NP];
  float2 T[NP], c0[NP], c1[NP], c2[NP];
  uint32_t last[2 * NP];
  // a pixel takes a splat when zq <= its threshold: 0 while it composites,
  // -inf once it is done (or outside the image)
  float thr[2 * NP];
  bool done = true;
#pragma unroll
  for (int k = 0; k < NP; ++k) {
    pyc[k] = make_float2((float)(tp.py + 8 * k) + 0.5f, (float)(tp.py + 8 * k) + 4.5f);
    T[k] = f2(1.f);
    c0[k] = c1[k] = c2[k] = f2(0.f);
  }
#pragma unroll
  for (int i = 0; i < 2 * NP; ++i) {
    last[i] = 0;
    thr[i] = tp.in[i] ? 0.f : -kInf;
    done = done && !tp.in[i];
  }
  const float2 one = f2(1.f), mone = f2(-1.f);
  bool pending = false;  // batch b's copy is in flight
  if (nb > 0) {
    issue(0);
    pending = !stalled;
  }
  int b = 0;
  for (; b < nb; ++b) {
    if (!__syncthreads_or(!done)) break;  // block vote; the previous batch is finished
    if (!__syncthreads_and(mbar_wait_bounded(&s_bar, (uint32_t)(b & 1), wc.limit_ns, status)))
      break;  // a copy did not land in time: give up on the tile
    pending = false;
    const int64_t rem = cnt - (int64_t)b * kBatch;
    const int m = rem < kBatch ? (int)rem : kBatch;
    if ((int)threadIdx.x < m) {
      const uint32_t mask = prepare_record<NP>(&s_rec[threadIdx.x][0], &s_ev[threadIdx.x][0],
                                               tp.x0, tp.y0);
      const uint8_t mk = clipped ? 0u : (uint8_t)mask;
      s_mask[threadIdx.x] = mk;
      if (wmask_out) wmask_out[start + (int64_t)b * kBatch + threadIdx.x] = mk;
    }
    __syncthreads();  // s_rec is free again
    if (b + 1 < nb) {
      issue(b + 1);
      pending = !stalled;
    }
    const int wc_n = warp_list<NP>(s_mask, s_list[warp], m);
    const uint32_t pos0 = (uint32_t)(b * kBatch + 1);
    for (int k = 0; k < wc_n; ++k) {
      if ((k & 3) == 0 && __all_sync(0xffffffffu, done)) break;  // warp vote
      const int j = s_list[warp][k];
      const float2* e = &s_ev[j][0];
      const EvCol col = eval_col(e, pxc);
      float2 zq[NP];
      bool ok[2 * NP];
      bool any = false;
#pragma unroll
      for (int q = 0; q < NP; ++q) {
        zq[q] = eval_zq(e, col, pyc[q]);
        ok[2 * q] = zq[q].x <= thr[2 * q];
        ok[2 * q + 1] = zq[q].y <= thr[2 * q + 1];
        any = any || ok[2 * q] || ok[2 * q + 1];
      }
      if (!any) continue;
      const uint32_t pos1 = pos0 + (uint32_t)j;
      bool stop = false;
#pragma unroll
      for (int q = 0; q < NP; ++q) {
        bool o0 = ok[2 * q], o1 = ok[2 * q + 1];
        float2 a = make_float2(o0 ? fminf(kAlphaMax, alpha_raw_of(zq[q].x)) : 0.f,
                               o1 ? fminf(kAlphaMax, alpha_raw_of(zq[q].y)) : 0.f);
        float2 Tn = __fmul2_rn(T[q], __ffma2_rn(a, mone, one));  // T (1 - alpha)
        if (Tn.x < kTMin || Tn.y < kTMin) {
          // the pixel stops before this Gaussian: it takes no part in it
          if (Tn.x < kTMin) {
            a.x = 0.f;
            Tn.x = T[q].x;
            thr[2 * q] = -kInf;
            o0 = false;
          }
          if (Tn.y < kTMin) {
            a.y = 0.f;
            Tn.y = T[q].y;
            thr[2 * q + 1] = -kInf;
            o1 = false;
          }
          stop = true;
        }
        const float2 w = __fmul2_rn(a, T[q]);
        c0[q] = __ffma2_rn(e[V_R], w, c0[q]);
        c1[q] = __ffma2_rn(e[V_G], w, c1[q]);
        c2[q] = __ffma2_rn(e[V_BL], w, c2[q]);
        T[q] = Tn;
        last[2 * q] = o0 ? pos1 : last[2 * q];
        last[2 * q + 1] = o1 ? pos1 : last[2 * q + 1];
      }
      if (stop) {
        bool d = true;
#pragma unroll
        for (int i = 0; i < 2 * NP; ++i) d = d && thr[i] == -kInf;
        done = d;
      }
    }
  }
  // a batch issued but not consumed must land before the block exits
  if (pending) mbar_wait_bounded(&s_bar, (uint32_t)(b & 1), wc.limit_ns, status);

  const size_t hw = (size_t)geo.g.width * geo.g.height;
  float* img = image + (size_t)tp.view * 3 * hw;
  float* tf = final_T + (size_t)tp.view * hw;
  uint32_t* nc = n_contrib + (size_t)tp.view * hw;
#pragma unroll
  for (int i = 0; i < 2 * NP; ++i) {
    if (!tp.in[i]) continue;
    const int q = i >> 1;
    const float Ti = (i & 1) ? T[q].y : T[q].x;
    const size_t pix = (size_t)(tp.py + 4 * i) * geo.g.width + tp.px;
    img[pix] = fmaf(Ti, bg0, (i & 1) ? c0[q].y : c0[q].x);
    img[hw + pix] = fmaf(Ti, bg1, (i & 1) ? c1[q].y : c1[q].x);
    img[2 * hw + pix] = fmaf(Ti, bg2, (i & 1) ? c2[q].y : c2[q].x);
    tf[pix] = Ti;
    nc[pix] = last[i];
  }
}

// Warp sum of ten per-lane values by a transposing butterfly: each exchange
// sends the half of the live values the partner keeps, so the live set halves
// per step (5, 3, 2, 2, 2 shuffles). On return lane l holds in `t0` the total
// of value ((l>>2)&1) + 3((l>>3)&1) + 5((l>>4)&1) -- one of 0,1,3,4,5,6,8,9 --
// and in `t1` the total of value 2 + 5((l>>4)&1), i.e. 2 or 7.
__device__ __forceinline__ void warp_sum10(const float (&v)[10], float& t0, float& t1) {
  const int lane = threadIdx.x & 31;
  const bool h16 = lane & 16, h8 = lane & 8, h4 = lane & 4;
  float a[5];
#pragma unroll
  for (int k = 0; k < 5; ++k) {
    const float send = h16 ? v[k] : v[k + 5];
    const float keep = h16 ? v[k + 5] : v[k];
    a[k] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
  }
  const float b0 = (h8 ? a[3] : a[0]) + __shfl_xor_sync(0xffffffffu, h8 ? a[0] : a[3], 8);
  const float b1 = (h8 ? a[4] : a[1]) + __shfl_xor_sync(0xffffffffu, h8 ? a[1] : a[4], 8);
  const float b2 = a[2] + __shfl_xor_sync(0xffffffffu, a[2], 8);
  float c0 = (h4 ? b1 : b0) + __shfl_xor_sync(0xffffffffu, h4 ? b0 : b1, 4);
  float c1 = b2 + __shfl_xor_sync(0xffffffffu, b2, 4);
  c0 += __shfl_xor_sync(0xffffffffu, c0, 2);
  c1 += __shfl_xor_sync(0xffffffffu, c1, 2);
  c0 += __shfl_xor_sync(0xffffffffu, c0, 1);
  c1 += __shfl_xor_sync(0xffffffffu, c1, 1);
  t0 = c0;
  t1 = c1;
}

template <int NP>
__global__ void __launch_bounds__(Shape<NP>::kThreads) k_raster_bwd(
    const float* __restrict__ records, const uint32_t* __restrict__ ids,
    const int64_t* __restrict__ ranges, RasterGeom geo, float bg0, float bg1, float bg2,
    const float* __restrict__ dL_dimage, const float* __restrict__ final_T,
    const uint32_t* __restrict__ n_contrib, const uint8_t* __restrict__ wmask_in,
    float* __restrict__ grad2d, uint32_t* __restrict__ status, WaitCfg wc) {
  using Sh = Shape<NP>;
  constexpr int kBatch = Sh::kBatch;
  constexpr int kWarps = Sh::kWarps;
  __shared__ __align__(128) float s_rec[2][kBatch][GS_RECORD_FLOATS];
  __shared__ __align__(16) float s_acc[kBatch][GS_GRAD2D_FLOATS];
  __shared__ uint32_t s_id[2][kBatch];
  __shared__ __align__(8) uint64_t s_bar[2];
  __shared__ uint32_t s_wmax[kWarps];
  __shared__ uint8_t s_mask[kBatch];
  __shared__ uint8_t s_list[kWarps][kBatch];

  const int tile = blockIdx.x;
  const TilePix<NP> tp = tile_pixel<NP>(geo.g, tile);
  const size_t hw = (size_t)geo.g.width * geo.g.height;
  int64_t start, end;
  tile_range(ranges, tile, geo.capacity, start, end, status);
  const float* rec_view = records + (size_t)tp.view * geo.n * GS_RECORD_FLOATS;
  float* g2_view = grad2d + (size_t)tp.view * geo.n * GS_GRAD2D_FLOATS;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool stalled = (int64_t)tile == wc.stall;  // test hook, see k_raster_fwd

  // per-pixel state, by pixel pairs; an outside pixel has no contributors and
  // zero upstream gradient
  float2 Tfin[NP], g0[NP], g1[NP], g2[NP];
  uint32_t nc[2 * NP];
  {
    const float* tf = final_T + (size_t)tp.view * hw;
    const uint32_t* ncv = n_contrib + (size_t)tp.view * hw;
    const float* gi = dL_dimage + (size_t)tp.view * 3 * hw;
#pragma unroll
    for (int q = 0; q < NP; ++q) {
      Tfin[q] = f2(1.f);
      g0[q] = g1[q] = g2[q] = f2(0.f);
    }
#pragma unroll
    for (int i = 0; i < 2 * NP; ++i) {
      nc[i] = 0;
      if (!tp.in[i]) continue;
      const size_t pix = (size_t)(tp.py + 4 * i) * geo.g.width + tp.px;
      const int q = i >> 1;
      float* tq = (i & 1) ? &Tfin[q].y : &Tfin[q].x;
      *tq = tf[pix];
      nc[i] = ncv[pix];
      ((i & 1) ? g0[q].y : g0[q].x) = gi[pix];
      ((i & 1) ? g1[q].y : g1[q].x) = gi[hw + pix];
      ((i & 1) ? g2[q].y : g2[q].x) = gi[2 * hw + pix];
    }
  }
  // T_final (bg . dL/dC): the background's share of dC/dalpha, before 1/(1-alpha)
  float2 tfbg[NP], T[NP], acc0[NP], acc1[NP], acc2[NP];  // acc: colour behind
#pragma unroll
  for (int q = 0; q < NP; ++q) {
    tfbg[q] = __fmul2_rn(Tfin[q], __ffma2_rn(f2(bg2), g2[q],
                                             __ffma2_rn(f2(bg1), g1[q], __fmul2_rn(f2(bg0), g0[q]))));
    T[q] = Tfin[q];
    acc0[q] = acc1[q] = acc2[q] = f2(0.f);
  }

  // the longest prefix any pixel of the warp, and of the tile, used
  uint32_t mine = 0;
#pragma unroll
  for (int i = 0; i < 2 * NP; ++i) mine = max(mine, nc[i]);
  const uint32_t wm = __reduce_max_sync(0xffffffffu, mine);
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

  // batches are consumed from the last (deepest) to the first; iteration it
  // uses buffer it & 1 and phase (it >> 1) & 1 of that buffer's barrier
  int pend[2] = {-1, -1};  // iteration whose copy into the buffer is in flight
  bool clipped[2] = {false, false};
  auto issue = [&](int it) {
    if (stalled) return;
    const int b = nb - 1 - it;
    const int buf = it & 1;
    const int64_t first = start + (int64_t)b * kBatch;
    const int64_t rem = used - (int64_t)b * kBatch;
    const int m = rem < kBatch ? (int)rem : kBatch;
    if (threadIdx.x == 0) mbar_arrive_expect_tx(&s_bar[buf], (uint32_t)(m * kRecBytes));
    if ((int)threadIdx.x < m) {
      uint32_t id = __ldg(&ids[first + threadIdx.x]);
      clipped[buf] = id >= (uint32_t)geo.n;
      if (clipped[buf]) {  // never read outside the records
        id = 0;
        atomicOr(status, kStatusBounds);
      }
      s_id[buf][threadIdx.x] = id;
      bulk_copy_g2s(&s_rec[buf][threadIdx.x][0], rec_view + (size_t)id * GS_RECORD_FLOATS,
                    kRecBytes, &s_bar[buf]);
    }
    pend[buf] = it;
  };

  const float pxc = (float)tp.px + 0.5f;
  float2 pyc[NP];
#pragma unroll
  for (int q = 0; q < NP; ++q)
    pyc[q] = make_float2((float)(tp.py + 8 * q) + 0.5f, (float)(tp.py + 8 * q) + 4.5f);
  if (nb > 0) issue(0);
  for (int it = 0; it < nb; ++it) {
    const int b = nb - 1 - it;
    const int buf = it & 1;
    __syncthreads();  // previous batch fully consumed and flushed
    if (it + 1 < nb) issue(it + 1);
    const int64_t rem = used - (int64_t)b * kBatch;
    const int m = rem < kBatch ? (int)rem : kBatch;
    if (!__syncthreads_and(
            mbar_wait_bounded(&s_bar[buf], (uint32_t)((it >> 1) & 1), wc.limit_ns, status)))
      break;  // a copy did not land in time: give up on the tile
    pend[buf] = -1;
    if ((int)threadIdx.x < m) {
      float* r = &s_rec[buf][threadIdx.x][0];
      // the forward's mask of this entry, or the same test again
      const uint32_t mask =
          wmask_in ? (uint32_t)wmask_in[start + (int64_t)b * kBatch + threadIdx.x]
                   : record_block_mask<NP>(r, tp.x0, tp.y0);
      s_mask[threadIdx.x] = clipped[buf] ? 0u : (uint8_t)mask;
      r[R_OPAC] = 1.f / r[R_OPAC];  // d alpha / d opacity = alpha / o
    }
    {
      float4* z = reinterpret_cast<float4*>(&s_acc[threadIdx.x][0]);
      z[0] = z[1] = z[2] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    __syncthreads();
    // this warp's pixels use no entry at or past the longest prefix among them
    const int64_t wlim = (int64_t)wm - (int64_t)b * kBatch;
    const int wc_n =
        warp_list<NP>(s_mask, s_list[warp], wlim < m ? (wlim > 0 ? (int)wlim : 0) : m);
    for (int k = wc_n - 1; k >= 0; --k) {
      const int j = s_list[warp][k];
      const uint32_t pos = (uint32_t)(b * kBatch + j);
      const float* r = &s_rec[buf][j][0];
      float dx, a1, a2;
      eval_col_s(r, pxc, dx, a1, a2);
      float2 dy[NP], p1[NP], p2[NP], zq[NP];
      bool ok[2 * NP];
      bool any = false;
#pragma unroll
      for (int q = 0; q < NP; ++q) {
        zq[q] = eval_zq_s(r, a1, a2, pyc[q], dy[q], p1[q], p2[q]);
        ok[2 * q] = pos < nc[2 * q] && zq[q].x <= 0.f;
        ok[2 * q + 1] = pos < nc[2 * q + 1] && zq[q].y <= 0.f;
        any = any || ok[2 * q] || ok[2 * q + 1];
      }
      const uint32_t bal = __ballot_sync(0xffffffffu, any);
      if (bal == 0u) continue;
      float v[10];
#pragma unroll
      for (int e = 0; e < 10; ++e) v[e] = 0.f;
#pragma unroll
      for (int q = 0; q < NP; ++q) {
        const bool o0 = ok[2 * q], o1 = ok[2 * q + 1];
        // a pixel that does not blend this Gaussian takes alpha = 0, which
        // leaves its T and colour-behind unchanged and adds nothing below
        const float2 araw = make_float2(alpha_raw_of(zq[q].x), alpha_raw_of(zq[q].y));
        const float2 a = make_float2(o0 ? fminf(kAlphaMax, araw.x) : 0.f,
                                     o1 ? fminf(kAlphaMax, araw.y) : 0.f);
        const float2 one_m = __fadd2_rn(f2(1.f), make_float2(-a.x, -a.y));
        const float2 inv = make_float2(o0 ? 1.f / one_m.x : 1.f, o1 ? 1.f / one_m.y : 1.f);
        T[q] = __fmul2_rn(T[q], inv);  // transmittance in front of this Gaussian
        const float2 w = __fmul2_rn(a, T[q]);
        const float2 d0 = __fadd2_rn(f2(r[R_R]), make_float2(-acc0[q].x, -acc0[q].y));
        const float2 d1 = __fadd2_rn(f2(r[R_G]), make_float2(-acc1[q].x, -acc1[q].y));
        const float2 d2 = __fadd2_rn(f2(r[R_B]), make_float2(-acc2[q].x, -acc2[q].y));
        float2 s = __fmul2_rn(d0, g0[q]);
        s = __ffma2_rn(d1, g1[q], s);
        s = __ffma2_rn(d2, g2[q], s);
        const float2 bgt = __fmul2_rn(tfbg[q], inv);
        const float2 dLda = __ffma2_rn(T[q], s, make_float2(-bgt.x, -bgt.y));
        acc0[q] = __ffma2_rn(a, d0, acc0[q]);
        acc1[q] = __ffma2_rn(a, d1, acc1[q]);
        acc2[q] = __ffma2_rn(a, d2, acc2[q]);
        // d alpha / d(-q/2) = alpha below the clamp, 0 on it
        float2 dpow = __fmul2_rn(a, dLda);
        dpow.x = araw.x < kAlphaMax ? dpow.x : 0.f;
        dpow.y = araw.y < kAlphaMax ? dpow.y : 0.f;
        // d alpha / d mean = alpha conic d = alpha 2 ln2 W^T (p1, p2)
        const float2 dpl = __fmul2_rn(dpow, f2(kTwoLn2));
        const float2 du = __fmul2_rn(
            dpl, __ffma2_rn(f2(r[R_W1X]), p1[q], __fmul2_rn(f2(r[R_W2X]), p2[q])));
        const float2 dv = __fmul2_rn(
            dpl, __ffma2_rn(f2(r[R_W1Y]), p1[q], __fmul2_rn(f2(r[R_W2Y]), p2[q])));
        const float2 dyd = __fmul2_rn(dy[q], dpow);
        const float2 dy2d = __fmul2_rn(dy[q], dyd);
        const float2 wg0 = __fmul2_rn(w, g0[q]), wg1 = __fmul2_rn(w, g1[q]);
        const float2 wg2 = __fmul2_rn(w, g2[q]);
        const float2 n2 = __ffma2_rn(dv, dv, __fmul2_rn(du, du));
        const float sd = dpow.x + dpow.y;
        v[0] += du.x + du.y;
        v[1] += dv.x + dv.y;
        // d alpha / d conic = -alpha/2 (dx^2, 2 dx dy, dy^2)
        v[2] += -0.5f * dx * dx * sd;
        v[3] += -dx * (dyd.x + dyd.y);
        v[4] += -0.5f * (dy2d.x + dy2d.y);
        v[5] += r[R_OPAC] * sd;  // d alpha / d opacity = alpha / o (slot holds 1/o)
        v[6] += wg0.x + wg0.y;
        v[7] += wg1.x + wg1.y;
        v[8] += wg2.x + wg2.y;
        v[9] += sqrtf(n2.x) + sqrtf(n2.y);
      }
      if (__popc(bal) == 1) {
        if (any) {
#pragma unroll
          for (int e = 0; e < 10; ++e) atomicAdd(&s_acc[j][e], v[e]);
        }
      } else {
        float t0, t1;
        warp_sum10(v, t0, t1);
        const bool first = (lane & 3) == 0;
        const int e = first ? ((lane >> 2) & 1) + 3 * ((lane >> 3) & 1) + 5 * ((lane >> 4) & 1)
                            : 2 + 5 * ((lane >> 4) & 1);
        if (first || (lane & 15) == 2) atomicAdd(&s_acc[j][e], first ? t0 : t1);
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
  // after a wait that gave up: copies still in flight land before the block
  // exits
#pragma unroll
  for (int bf = 0; bf < 2; ++bf)
    if (pend[bf] >= 0)
      mbar_wait_bounded(&s_bar[bf], (uint32_t)((pend[bf] >> 1) & 1), wc.limit_ns, status);
}

}  // namespace

cudaError_t launch_raster_fwd(const float* records, const uint32_t* ids, const int64_t* ranges,
                              int64_t capacity, const Grid& g, int n_views, int n,
                              const float bg[3], float* image, float* final_T,
                              uint32_t* n_contrib, uint8_t* warp_masks, uint32_t* status,
                              const WaitCfg& wc,
                              cudaStream_t stream) {
  const int64_t tiles = (int64_t)g.tiles_per_view * n_views;
  if (tiles == 0) return cudaSuccess;
  RasterGeom geo{g, n, n > 0 ? capacity : 0};
  k_raster_fwd<kPairs><<<(unsigned)tiles, Shape<kPairs>::kThreads, 0, stream>>>(
      records, ids, ranges, geo, bg[0], bg[1], bg[2], image, final_T, n_contrib, warp_masks, status,
      wc);
  return cudaGetLastError();
}

cudaError_t launch_raster_bwd(const float* records, const uint32_t* ids, const int64_t* ranges,
                              int64_t capacity, const Grid& g, int n_views, int n,
                              const float bg[3], const float* dL_dimage, const float* final_T,
                              const uint32_t* n_contrib, const uint8_t* warp_masks,
                              float* grad2d, uint32_t* status,
                              const WaitCfg& wc, cudaStream_t stream) {
  const int64_t tiles = (int64_t)g.tiles_per_view * n_views;
  if (tiles == 0) return cudaSuccess;
  RasterGeom geo{g, n, n > 0 ? capacity : 0};
  k_raster_bwd<kPairs><<<(unsigned)tiles, Shape<kPairs>::kThreads, 0, stream>>>(
      records, ids, ranges, geo, bg[0], bg[1], bg[2], dL_dimage, final_T, n_contrib, warp_masks,
      grad2d,
      status, wc);
  return cudaGetLastError();
}

}  // namespace gsb
