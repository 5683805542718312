// loss.cu -- the photometric training loss and its gradient in one kernel.
//
// Second Julia page (lshu.cn, sec. 3.3): the rendered image x is compared to
// the target y by L = (1 - lambda) * mean|x - y| + lambda * (1 - mean SSIM)
// with lambda about 0.2. SSIM takes the constants of its own definition
// (Wang et al. 2004): an 11 x 11 Gaussian window, sigma 1.5, normalised to 1;
// C1 = 0.01^2, C2 = 0.03^2; the map is taken at every pixel with the image
// zero outside its border; both means run over a view's pixels and channels.
//
// One block owns a 32 x 32 output tile of one colour plane and does, in
// shared memory:
//   load   x, y over the tile grown by 10 pixels (zero outside the image);
//   H1     the window moments filtered along rows over the tile grown by 5
//          columns (the window is separable); SSIM needs Exx and Eyy only
//          through var x + var y, so four moments suffice: x, y, xx + yy, xy,
//          carried as the pairs (x, y) and (xx + yy, xy);
//   V1     the same along columns -> mx, my, Ess, Exy over the tile grown by
//          5, then SSIM and its partial derivatives with respect to mx, Ess
//          and Exy at every one of those pixels inside the image;
//   H2/V2  the three partial maps filtered back (the window is symmetric,
//          so the adjoint filter is the same one) over the tile;
//   grad   dL/dx = (1-l)/N sign(x-y) - l/N (Pmx + 2 x Pss + y Pxy).
// Every thread runs a few outputs of a pass at once, sliding along the
// filter direction, so each shared-memory value it reads serves several taps.
// The moment pairs go through packed FP32x2 instructions. The partial maps
// reuse the shared memory of the row-filtered moments, so three blocks fit
// on an SM.
// Loss sums are block-reduced and added into double accumulators; the last
// block to finish writes each view's loss terms.

#include <cuda_runtime.h>

#include <cstdint>

#include "gs.h"
#include "gs_internal.h"

namespace gsb {
namespace {

constexpr int kT = 32;               // output tile edge
constexpr int kR = 5;                // window radius
constexpr int kIn = kT + 4 * kR;     // 52: loaded region edge
constexpr int kMid = kT + 2 * kR;    // 42: moment region edge
constexpr int kInPitch = 53;         // float2 pitch of the loaded region
constexpr int kMidPitch = 43;        // pitch of the moment and partial maps
constexpr int kOutPitch = 33;        // pitch of the row-filtered partial maps
constexpr int kLossThreads = 384;
constexpr int kLossBlocksPerSm = 3;

// Outputs per thread in each pass; 42 = 7 x 6 and 32 = 8 x 4.
constexpr int kK1 = 6;
constexpr int kK2 = 4;
constexpr int kSeg1 = kMid / kK1;    // 7
constexpr int kSeg2 = kT / kK2;      // 8
static_assert(kSeg1 * kK1 == kMid && kSeg2 * kK2 == kT, "segments tile the rows");
static_assert(kMid * kSeg1 <= kLossThreads, "one column item per thread in V1");

// The 11 taps of the normalised 1-D Gaussian of sigma 1.5 (the 2-D window
// is their outer product), computed at compile time: exp by its Taylor
// series in double, which converges to double precision for |x| <= 6.
constexpr double taylor_exp(double x) {
  double term = 1.0, sum = 1.0;
  for (int k = 1; k < 60; ++k) {
    term *= x / k;
    sum += term;
  }
  return sum;
}
constexpr double tap_raw(int d) { return taylor_exp(-(double)(d * d) / (2.0 * 1.5 * 1.5)); }
constexpr double tap_sum() {
  double t = 0.0;
  for (int d = -kR; d <= kR; ++d) t += tap_raw(d);
  return t;
}
constexpr float tap(int d) { return (float)(tap_raw(d - kR) / tap_sum()); }

struct LossSmem {
  float2 xy[kIn][kInPitch];          // (x, y) over the loaded region
  union {
    struct {
      float2 m[kIn][kMidPitch];      // row-filtered (x, y)
      float2 e[kIn][kMidPitch];      // row-filtered (xx + yy, xy)
    } h;
    struct {
      float2 pab[kMid][kMidPitch];   // (dS/dmx, dS/dEss) per moment pixel
      float pc[kMid][kMidPitch];     // dS/dExy per moment pixel
      float2 qab[kMid][kOutPitch];   // the same two filtered along rows
      float qc[kMid][kOutPitch];     // dS/dExy filtered along rows
    } p;
  } u;
  float red[2][kLossThreads / 32];
  unsigned last;
};

__device__ __forceinline__ float2 f2(float a) { return make_float2(a, a); }

// Sum over the block, valid in thread 0; every thread must call it.
__device__ __forceinline__ float block_sum(float v, float* red) {
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float s = 0.f;
  if (threadIdx.x == 0)
    for (int w = 0; w < kLossThreads / 32; ++w) s += red[w];
  return s;
}

template <bool kGrad>
__global__ void __launch_bounds__(kLossThreads, kLossBlocksPerSm)
k_l1_dssim(const float* __restrict__ image, const float* __restrict__ target, int H, int W,
           float lambda, float inv_n, double* __restrict__ sums,
           unsigned* __restrict__ done, double* __restrict__ terms, int n_views,
           float* __restrict__ grad) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  LossSmem& s = *reinterpret_cast<LossSmem*>(smem_raw);
  const int tid = threadIdx.x;
  const int X0 = blockIdx.x * kT, Y0 = blockIdx.y * kT;
  const int plane = blockIdx.z;
  const size_t base = (size_t)plane * H * W;
  const float* xp = image + base;
  const float* yp = target + base;

  // load: (x, y) over the tile grown by 10, zero outside; L1 over the tile
  float l1 = 0.f;
  constexpr int kLoadRounds = (kIn * kIn + kLossThreads - 1) / kLossThreads;
#pragma unroll
  for (int k = 0; k < kLoadRounds; ++k) {
    const int i = tid + k * kLossThreads;
    if (i >= kIn * kIn) break;
    const int r = i / kIn, c = i - r * kIn;
    const int gy = Y0 - 2 * kR + r, gx = X0 - 2 * kR + c;
    float2 v = make_float2(0.f, 0.f);
    if (gy >= 0 && gy < H && gx >= 0 && gx < W) {
      const size_t o = (size_t)gy * W + gx;
      v = make_float2(__ldg(xp + o), __ldg(yp + o));
      if (r >= 2 * kR && r < 2 * kR + kT && c >= 2 * kR && c < 2 * kR + kT)
        l1 += fabsf(v.x - v.y);
    }
    s.xy[r][c] = v;
  }
  __syncthreads();

  constexpr float g[2 * kR + 1] = {tap(0), tap(1), tap(2), tap(3), tap(4), tap(5),
                                   tap(6), tap(7), tap(8), tap(9), tap(10)};

  // H1: along rows, moment column c of loaded row r reads loaded columns c..c+10
  for (int it = tid; it < kIn * kSeg1; it += kLossThreads) {
    const int r = it % kIn, c0 = (it / kIn) * kK1;
    float2 am[kK1], ae[kK1];
#pragma unroll
    for (int o = 0; o < kK1; ++o) {
      am[o] = make_float2(0.f, 0.f);
      ae[o] = make_float2(0.f, 0.f);
    }
#pragma unroll
    for (int j = 0; j < kK1 + 2 * kR; ++j) {
      const float2 v = s.xy[r][c0 + j];
      const float2 sp = make_float2(fmaf(v.x, v.x, v.y * v.y), v.x * v.y);
#pragma unroll
      for (int o = 0; o < kK1; ++o) {
        const int d = j - o;
        if (d >= 0 && d <= 2 * kR) {
          am[o] = __ffma2_rn(f2(g[d]), v, am[o]);
          ae[o] = __ffma2_rn(f2(g[d]), sp, ae[o]);
        }
      }
    }
#pragma unroll
    for (int o = 0; o < kK1; ++o) {
      s.u.h.m[r][c0 + o] = am[o];
      s.u.h.e[r][c0 + o] = ae[o];
    }
  }
  __syncthreads();

  // V1: along columns, then SSIM and its partials at moment pixel (r, c),
  // image pixel (Y0 - 5 + r, X0 - 5 + c); the partials wait in registers
  // until every thread has read the row-filtered moments they overwrite
  const float C1 = 1e-4f, C2 = 9e-4f;
  float ssim = 0.f;
  float2 pab[kK1];
  float pc[kK1];
  const int v1_c = tid % kMid, v1_r0 = (tid / kMid) * kK1;
  if (tid < kMid * kSeg1) {
    const int c = v1_c, r0 = v1_r0;
    float2 am[kK1], ae[kK1];
#pragma unroll
    for (int o = 0; o < kK1; ++o) {
      am[o] = make_float2(0.f, 0.f);
      ae[o] = make_float2(0.f, 0.f);
    }
#pragma unroll
    for (int j = 0; j < kK1 + 2 * kR; ++j) {
      const float2 m = s.u.h.m[r0 + j][c];
      const float2 e = s.u.h.e[r0 + j][c];
#pragma unroll
      for (int o = 0; o < kK1; ++o) {
        const int d = j - o;
        if (d >= 0 && d <= 2 * kR) {
          am[o] = __ffma2_rn(f2(g[d]), m, am[o]);
          ae[o] = __ffma2_rn(f2(g[d]), e, ae[o]);
        }
      }
    }
    const int gx = X0 - kR + c;
    const bool col_in = gx >= 0 && gx < W;
    const bool col_tile = c >= kR && c < kR + kT;
#pragma unroll
    for (int o = 0; o < kK1; ++o) {
      const int r = r0 + o;
      const int gy = Y0 - kR + r;
      pab[o] = make_float2(0.f, 0.f);
      pc[o] = 0.f;
      if (col_in && gy >= 0 && gy < H) {
        const float mx = am[o].x, my = am[o].y;
        const float mxy = mx * my, mm = fmaf(mx, mx, my * my);
        const float a1 = 2.f * mxy + C1, a2 = 2.f * (ae[o].y - mxy) + C2;
        const float b1 = mm + C1, b2 = (ae[o].x - mm) + C2;
        const float inv_den = 1.f / (b1 * b2);
        const float S = a1 * a2 * inv_den;
        if (col_tile && r >= kR && r < kR + kT) ssim += S;
        if (kGrad) {
          // S = a1 a2 / (b1 b2): d/dmx through a1, a2, b1, b2; d/dEss only
          // through b2; d/dExy only through a2
          pab[o].x = (2.f * my * (a2 - a1) - S * 2.f * mx * (b2 - b1)) * inv_den;
          pab[o].y = -S * b1 * inv_den;
          pc[o] = 2.f * a1 * inv_den;
        }
      }
    }
  }

  if (kGrad) {
    __syncthreads();
    if (tid < kMid * kSeg1) {
#pragma unroll
      for (int o = 0; o < kK1; ++o) {
        s.u.p.pab[v1_r0 + o][v1_c] = pab[o];
        s.u.p.pc[v1_r0 + o][v1_c] = pc[o];
      }
    }
    __syncthreads();
    // H2: along rows of the partial maps, tile column u reads moment columns u..u+10
    for (int it = tid; it < kMid * kSeg2; it += kLossThreads) {
      const int r = it % kMid, u0 = (it / kMid) * kK2;
      float2 qab[kK2];
      float qc[kK2];
#pragma unroll
      for (int o = 0; o < kK2; ++o) {
        qab[o] = make_float2(0.f, 0.f);
        qc[o] = 0.f;
      }
#pragma unroll
      for (int j = 0; j < kK2 + 2 * kR; ++j) {
        const float2 p = s.u.p.pab[r][u0 + j];
        const float pc = s.u.p.pc[r][u0 + j];
#pragma unroll
        for (int o = 0; o < kK2; ++o) {
          const int d = j - o;
          if (d >= 0 && d <= 2 * kR) {
            qab[o] = __ffma2_rn(f2(g[d]), p, qab[o]);
            qc[o] = fmaf(g[d], pc, qc[o]);
          }
        }
      }
#pragma unroll
      for (int o = 0; o < kK2; ++o) {
        s.u.p.qab[r][u0 + o] = qab[o];
        s.u.p.qc[r][u0 + o] = qc[o];
      }
    }
    __syncthreads();
    // V2 and the gradient at tile pixel (t, u)
    const float k1 = (1.f - lambda) * inv_n, k2 = lambda * inv_n;
    for (int it = tid; it < kT * kSeg2; it += kLossThreads) {
      const int u = it % kT, t0 = (it / kT) * kK2;
      float2 qab[kK2];
      float qc[kK2];
#pragma unroll
      for (int o = 0; o < kK2; ++o) {
        qab[o] = make_float2(0.f, 0.f);
        qc[o] = 0.f;
      }
#pragma unroll
      for (int j = 0; j < kK2 + 2 * kR; ++j) {
        const float2 p = s.u.p.qab[t0 + j][u];
        const float pc = s.u.p.qc[t0 + j][u];
#pragma unroll
        for (int o = 0; o < kK2; ++o) {
          const int d = j - o;
          if (d >= 0 && d <= 2 * kR) {
            qab[o] = __ffma2_rn(f2(g[d]), p, qab[o]);
            qc[o] = fmaf(g[d], pc, qc[o]);
          }
        }
      }
      const int gx = X0 + u;
      if (gx < W) {
#pragma unroll
        for (int o = 0; o < kK2; ++o) {
          const int gy = Y0 + t0 + o;
          if (gy < H) {
            const float2 v = s.xy[2 * kR + t0 + o][2 * kR + u];
            const float dx = v.x - v.y;
            const float sgn = dx > 0.f ? 1.f : (dx < 0.f ? -1.f : 0.f);
            const float gs = qab[o].x + 2.f * v.x * qab[o].y + v.y * qc[o];
            grad[base + (size_t)gy * W + gx] = k1 * sgn - k2 * gs;
          }
        }
      }
    }
  }

  // loss sums of the tile into the view's double accumulators
  const float bl1 = block_sum(l1, s.red[0]);
  __syncthreads();
  const float bss = block_sum(ssim, s.red[1]);
  if (tid == 0) {
    const int view = plane / 3;
    atomicAdd(sums + 2 * view, (double)bl1);
    atomicAdd(sums + 2 * view + 1, (double)bss);
    __threadfence();
    const unsigned n_blocks = gridDim.x * gridDim.y * gridDim.z;
    s.last = atomicAdd(done, 1u) == n_blocks - 1 ? 1u : 0u;
  }
  __syncthreads();
  if (s.last) {
    __threadfence();
    const double inv_nd = 1.0 / (3.0 * (double)H * (double)W);
    for (int v = tid; v < n_views; v += kLossThreads) {
      const double ml1 = __ldcg(sums + 2 * v) * inv_nd;
      const double mss = __ldcg(sums + 2 * v + 1) * inv_nd;
      terms[3 * v + 0] = (1.0 - (double)lambda) * ml1 + (double)lambda * (1.0 - mss);
      terms[3 * v + 1] = ml1;
      terms[3 * v + 2] = mss;
    }
  }
}

}  // namespace

size_t loss_smem_bytes() { return sizeof(LossSmem); }

cudaError_t launch_l1_dssim(const float* image, const float* target, int n_views, int H, int W,
                            float lambda, double* terms, float* grad, double* sums,
                            unsigned* done, cudaStream_t stream) {
  cudaError_t e = cudaMemsetAsync(sums, 0, sizeof(double) * 2 * n_views + 16, stream);
  if (e != cudaSuccess) return e;
  const dim3 grid((W + kT - 1) / kT, (H + kT - 1) / kT, 3 * n_views);
  const size_t smem = sizeof(LossSmem);
  const float inv_n = (float)(1.0 / (3.0 * (double)H * (double)W));
  if (grad) {
    e = cudaFuncSetAttribute(k_l1_dssim<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    k_l1_dssim<true><<<grid, kLossThreads, smem, stream>>>(image, target, H, W, lambda,
                                                            inv_n, sums, done, terms, n_views,
                                                            grad);
  } else {
    e = cudaFuncSetAttribute(k_l1_dssim<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    k_l1_dssim<false><<<grid, kLossThreads, smem, stream>>>(image, target, H, W, lambda,
                                                             inv_n, sums, done, terms, n_views,
                                                             nullptr);
  }
  return cudaGetLastError();
}

}  // namespace gsb
