// optim.cu -- densification statistics and the fused Adam step, sm_100a.
//
// Densification statistics (the absolute-gradient densification tutorial,
// jsqmd.com sec. 2 table and sec. 3.1 add_densification_stats): per view and
// visible Gaussian, the plain view-space gradient ||sum_p g_p|| and the
// absolute one sum_p ||g_p|| (the latter already summed by the rasteriser's
// backward), plus a visibility count.
//
// Adam (lshu.cn sec. 3.3 / 5.3, per-group learning rates): one launch over
// every group, float4-vectorised, streaming loads and stores (each float is
// touched once per step), square root and division on the SFU.

#include <cuda_runtime.h>

#include "gs_internal.h"

namespace gsb {
namespace {

__global__ void __launch_bounds__(256) k_densify(const float4* __restrict__ grad2d,
                                                 const int* __restrict__ radii, int n,
                                                 int n_views, float* __restrict__ accum_plain,
                                                 float* __restrict__ accum_abs,
                                                 int* __restrict__ denom) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  float pl = 0.f, ab = 0.f;
  int cnt = 0;
  for (int v = 0; v < n_views; ++v) {
    const size_t r = (size_t)v * n + i;
    if (radii[r] <= 0) continue;
    const float4 a = grad2d[r * 3 + 0];
    const float4 c = grad2d[r * 3 + 2];
    pl += densify_norm(a.x, a.y);
    ab += c.y;
    ++cnt;
  }
  if (cnt) {
    accum_plain[i] += pl;
    accum_abs[i] += ab;
    denom[i] += cnt;
  }
}

struct AdamTable {
  float* p[8];
  const float* g[8];
  float* m[8];
  float* v[8];
  int64_t count[8];
  float lr[8];
  int64_t block_start[9];
  int n_groups;
};

constexpr int kAdamThreads = 256;
constexpr int kAdamVecPerThread = 4;
constexpr int64_t kAdamFloatsPerBlock = (int64_t)kAdamThreads * kAdamVecPerThread * 4;

__global__ void __launch_bounds__(kAdamThreads) k_adam(AdamTable t, float b1, float b2, float eps,
                                                       float ibc1, float ibc2) {
  int gi = 0;
  while (gi + 1 < t.n_groups && (int64_t)blockIdx.x >= t.block_start[gi + 1]) ++gi;
  const int64_t count = t.count[gi];
  const int64_t base = ((int64_t)blockIdx.x - t.block_start[gi]) * kAdamFloatsPerBlock;
  float* __restrict__ P = t.p[gi];
  const float* __restrict__ G = t.g[gi];
  float* __restrict__ M = t.m[gi];
  float* __restrict__ V = t.v[gi];
  const float lr = t.lr[gi];
#pragma unroll
  for (int k = 0; k < kAdamVecPerThread; ++k) {
    const int64_t e = base + ((int64_t)k * kAdamThreads + threadIdx.x) * 4;
    if (e + 4 <= count) {
      // every float is read and written once per step: stream past L2
      float4 p = __ldcs(reinterpret_cast<const float4*>(P + e));
      const float4 g = __ldcs(reinterpret_cast<const float4*>(G + e));
      float4 m = __ldcs(reinterpret_cast<const float4*>(M + e));
      float4 v = __ldcs(reinterpret_cast<const float4*>(V + e));
      adam_one(p.x, g.x, m.x, v.x, lr, b1, b2, eps, ibc1, ibc2);
      adam_one(p.y, g.y, m.y, v.y, lr, b1, b2, eps, ibc1, ibc2);
      adam_one(p.z, g.z, m.z, v.z, lr, b1, b2, eps, ibc1, ibc2);
      adam_one(p.w, g.w, m.w, v.w, lr, b1, b2, eps, ibc1, ibc2);
      __stcs(reinterpret_cast<float4*>(P + e), p);
      __stcs(reinterpret_cast<float4*>(M + e), m);
      __stcs(reinterpret_cast<float4*>(V + e), v);
    } else {
      for (int64_t f = e; f < count && f < e + 4; ++f) {
        float p = P[f], m = M[f], v = V[f];
        adam_one(p, G[f], m, v, lr, b1, b2, eps, ibc1, ibc2);
        P[f] = p;
        M[f] = m;
        V[f] = v;
      }
    }
  }
}

}  // namespace

cudaError_t launch_densify(const float* grad2d, const int* radii, int n_views, int n,
                           float* accum_plain, float* accum_abs, int* denom, cudaStream_t stream) {
  if (n == 0) return cudaSuccess;
  k_densify<<<(n + 255) / 256, 256, 0, stream>>>(reinterpret_cast<const float4*>(grad2d), radii,
                                                 n, n_views, accum_plain, accum_abs, denom);
  return cudaGetLastError();
}

cudaError_t launch_adam(const gs_adam_group* groups, int n_groups, float b1, float b2, float eps,
                        int64_t step, cudaStream_t stream) {
  AdamTable t;
  t.n_groups = n_groups;
  int64_t blocks = 0;
  for (int k = 0; k < n_groups; ++k) {
    t.p[k] = groups[k].param;
    t.g[k] = groups[k].grad;
    t.m[k] = groups[k].exp_avg;
    t.v[k] = groups[k].exp_avg_sq;
    t.count[k] = groups[k].count;
    t.lr[k] = groups[k].lr;
    t.block_start[k] = blocks;
    blocks += (groups[k].count + kAdamFloatsPerBlock - 1) / kAdamFloatsPerBlock;
  }
  t.block_start[n_groups] = blocks;
  if (blocks == 0) return cudaSuccess;
  const double bc1 = 1.0 - pow((double)b1, (double)step);
  const double bc2 = 1.0 - pow((double)b2, (double)step);
  k_adam<<<(unsigned)blocks, kAdamThreads, 0, stream>>>(t, b1, b2, eps, (float)(1.0 / bc1),
                                                        (float)(1.0 / bc2));
  return cudaGetLastError();
}

}  // namespace gsb
