// gs_device.cuh -- device-side helpers shared by the sm_100a kernels.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/gs.h"

namespace gsb {

// Method constants (the task's stated values; the pages print none of them).
constexpr int kTile = GS_TILE;                 // 16x16 pixel tiles
constexpr int kTilePixels = kTile * kTile;     // 256 threads per raster block
constexpr double kNear = 0.2;                  // near-plane cull
constexpr double kLowPass = 0.3;               // + 0.3 I on the 2D covariance
constexpr float kAlphaMax = 0.99f;             // alpha clamp
constexpr float kAlphaMin = 1.0f / 255.0f;     // alpha skip threshold
constexpr float kTMin = 1e-4f;                 // transmittance stop
constexpr int kMaxRadius = 1 << 30;            // radius saturation

// Status bits OR-ed into the workspace status word.
constexpr uint32_t kStatusCapacity = 1u << 0;
constexpr uint32_t kStatusTimeout = 1u << 1;
constexpr uint32_t kStatusBounds = 1u << 2;
constexpr uint32_t kStatusNonfinite = 1u << 3;

// Depth key that marks a Gaussian culled for a non-finite parameter or
// colour (a quiet NaN no depth computation produces); the binning raises
// kStatusNonfinite when it meets one.
constexpr uint32_t kNonfiniteKeyBits = 0x7FC0BAD0u;

// Every device-side wait (an mbarrier phase, a look-back flag) gives up after
// a time limit on the global nanosecond timer, sets kStatusTimeout and
// returns. `stall` names one block (a raster tile, an emission block) that
// is made to wait for something that never comes -- a test hook that
// exercises the timeout path; -1 (the default) stalls nothing.
struct WaitCfg {
  uint64_t limit_ns;
  int64_t stall;
};
constexpr uint64_t kWaitLimitNs = 2000ull * 1000ull * 1000ull;  // 2 s

// Cameras travel in the kernel parameter block.
struct CamSet {
  gs_camera c[GS_MAX_VIEWS];
};

struct Grid {
  int width, height, tiles_x, tiles_y, tiles_per_view;
};

__host__ __device__ inline Grid grid_of(const gs_camera& c) {
  Grid g;
  g.width = c.width;
  g.height = c.height;
  g.tiles_x = (c.width + kTile - 1) / kTile;
  g.tiles_y = (c.height + kTile - 1) / kTile;
  g.tiles_per_view = g.tiles_x * g.tiles_y;
  return g;
}

// Raster record field offsets (floats), see gs.h. The 2D Gaussian is kept in
// the form the rasteriser evaluates: the mean split into a float and the
// float of its remainder (carried in c1, c2), the rows w1, w2 of W with
// W^T W = (log2(e) / 2) conic, and nlo = -log2(255 opacity), so that
//   zq = (w1 . d)^2 + (w2 . d)^2 - log2(255 o) = -log2(255 alpha_raw)
// and a pixel takes the splat iff zq <= 0.
enum RecField {
  R_U = 0, R_V = 1, R_W1X = 2, R_W1Y = 3, R_C1 = 4, R_W2X = 5, R_W2Y = 6, R_C2 = 7,
  R_NLO = 8, R_R = 9, R_G = 10, R_B = 11, R_HX = 12, R_HY = 13, R_OPAC = 14, R_SPARE = 15
};
// Binning record (one float4): depth key, tile_x word, tile_y word, 0.
// Screen-space gradient fields (floats), see gs.h.
enum G2Field {
  G_U = 0, G_V = 1, G_CA = 2, G_CB = 3, G_CC = 4, G_OPAC = 5,
  G_R = 6, G_G = 7, G_B = 8, G_ABS = 9
};

// ---------------------------------------------------------------- PTX wrappers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

// One TMA bulk copy global -> shared, completing `bytes` on `bar`.
// dst and src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_copy_g2s(void* dst, const void* src, uint32_t bytes,
                                              uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait on an mbarrier phase: gives up after limit_ns, flags the
// status (when given) and returns false. After a false return the caller
// must not read the buffer, and must wait again before exiting if a copy
// into it may still be in flight.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity,
                                                  uint64_t limit_ns, uint32_t* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer_ns() - t0 > limit_ns) break;
    __nanosleep(64);
  }
  if (status) atomicOr(status, kStatusTimeout);
  return false;
}

// Vector float reduction into global memory (sm_90+), 16-byte aligned.
__device__ __forceinline__ void red_add_v4(float* addr, float a, float b, float c, float d) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(addr), "f"(a), "f"(b),
               "f"(c), "f"(d)
               : "memory");
}

// 64-bit relaxed device-scope load / store for decoupled look-back words.
__device__ __forceinline__ uint64_t ld_relaxed_u64(const uint64_t* p) {
  uint64_t v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_relaxed_u64(uint64_t* p, uint64_t v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// Look-back word: [63:62] flag (0 empty, 1 aggregate, 2 inclusive prefix),
// [61:0] count.
constexpr uint64_t kLbAggregate = 1ull << 62;
constexpr uint64_t kLbPrefix = 2ull << 62;
constexpr uint64_t kLbValueMask = (1ull << 62) - 1;

// Wait (bounded by limit_ns) until a look-back word is non-empty; returns it.
// On timeout flags the status and returns an inclusive-prefix word of 0 so
// that the caller terminates.
__device__ __forceinline__ uint64_t lookback_wait(const uint64_t* p, uint64_t limit_ns,
                                                  uint32_t* status) {
  uint64_t w = ld_relaxed_u64(p);
  if ((w >> 62) != 0) return w;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    __nanosleep(100);
    w = ld_relaxed_u64(p);
    if ((w >> 62) != 0) return w;
    if (globaltimer_ns() - t0 > limit_ns) break;
  }
  atomicOr(status, kStatusTimeout);
  return kLbPrefix;
}

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// One Adam update (lshu.cn sec. 3.3; Kingma and Ba with bias correction,
// eps outside the square root); ibc1 = 1 / (1 - b1^t), ibc2 = 1 / (1 - b2^t).
// The square root and the division use the SFU (a few ulp on the step, far
// inside the update's own scale), which keeps the callers on HBM rather than
// on the multi-instruction IEEE sequences. Shared by the Adam kernel and the
// fused projection backward, so the two give identical parameters.
__device__ __forceinline__ void adam_one(float& p, float g, float& m, float& v, float lr, float b1,
                                         float b2, float eps, float ibc1, float ibc2) {
  m = fmaf(b1, m, (1.f - b1) * g);
  v = fmaf(b2, v, (1.f - b2) * g * g);
  const float denom = sqrtf(v * ibc2) + eps;
  p -= __fdividef(lr * (m * ibc1), denom);
}

// Start moving the 128-byte line holding p towards L2 (no register result).
__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

__device__ __forceinline__ int lane_of_thread() { return (int)(threadIdx.x & 31); }

// ||(gx, gy)|| of a view's screen-space mean gradient (the plain
// densification statistic), one fixed operation sequence for every caller.
__device__ __forceinline__ float densify_norm(float gx, float gy) {
  return sqrtf(fmaf(gx, gx, gy * gy));
}

}  // namespace gsb
