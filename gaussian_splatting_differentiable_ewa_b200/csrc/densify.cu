// densify.cu -- densify_and_prune: clone, split and prune with stream
// compaction, sm_100a.
//
// The absolute-gradient densification tutorial (jsqmd.com sec. 1 and 3.3):
// a Gaussian's average view-space gradient accum / denom above a threshold
// makes it densify -- a small one is cloned, a large one is split -- and faint
// or oversized Gaussians are pruned. Each Gaussian, in index order, becomes
// zero (pruned), one (kept), or two (clone: itself then a copy; split: two
// children) output Gaussians; the output is compacted in that order.
//
//  k_dp_decide  decision per Gaussian (float32, on the raw log-scales and
//               logit against thresholds the host converts) and output
//               count per block.
//  k_dp_scan    exclusive scan of the block counts (one block), the output
//               count and the capacity check.
//  k_dp_emit    every output Gaussian at its position: parameters and Adam
//               moments copied for the kept ones, moments zero for the new
//               ones; a split child's mean is mean + R (s * z) with the
//               caller's normal draws z, its log-scales shrink by
//               log_split_shrink. Each thread writes its Gaussian's small
//               fields; the SH blocks (most of the bytes) are moved by the
//               whole warp in contiguous runs; six blocks per SM (40
//               registers) keep more of those runs in flight.
//  k_dsq_count / k_dsq_map  the same positions from given decisions, as an
//               output -> input map for quantised SH (quant.cu re-encodes
//               the output groups from it).

#include <cuda_runtime.h>

#include "gs_internal.h"

namespace gsb {
namespace {

constexpr int kDpThreads = 256;
constexpr int8_t kPrune = 0, kKeep = 1, kClone = 2, kSplit = 3;

__device__ __forceinline__ int dp_count(int8_t c) { return c == kPrune ? 0 : (c == kKeep ? 1 : 2); }

__global__ void __launch_bounds__(kDpThreads) k_dp_decide(
    const float4* __restrict__ log_scales, const float* __restrict__ logit,
    const float* __restrict__ accum, const int32_t* __restrict__ denom, int n, DensifyArgs p,
    int8_t* __restrict__ codes, uint32_t* __restrict__ block_counts) {
  __shared__ uint32_t s_w[kDpThreads / 32];
  const int i = blockIdx.x * kDpThreads + threadIdx.x;
  int cnt = 0;
  if (i < n) {
    const float4 ls = __ldg(&log_scales[i]);
    const float max_ls = fmaxf(ls.x, fmaxf(ls.y, ls.z));
    const int32_t d = __ldg(&denom[i]);
    // the average gradient above the threshold, as accum > threshold * denom
    const bool hot = d > 0 && __ldg(&accum[i]) > __fmul_rn(p.grad_threshold, (float)d);
    const bool prune = __ldg(&logit[i]) < p.logit_min_opacity || max_ls > p.log_max_scale;
    int8_t c = kKeep;
    if (hot) c = max_ls > p.log_scale_split ? kSplit : kClone;
    if (prune) c = kPrune;
    codes[i] = c;
    cnt = dp_count(c);
  }
  uint32_t s = (uint32_t)cnt;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) s_w[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t t = 0;
#pragma unroll
    for (int w = 0; w < kDpThreads / 32; ++w) t += s_w[w];
    block_counts[blockIdx.x] = t;
  }
}

// One block of 1024 threads: exclusive scan of the block counts in place.
__global__ void __launch_bounds__(1024) k_dp_scan(uint32_t* __restrict__ block_counts, int nb,
                                                 int64_t capacity, int64_t* __restrict__ n_out,
                                                 uint32_t* __restrict__ status) {
  __shared__ uint32_t s_w[32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t carry = 0;
  for (int base = 0; base < nb; base += 1024) {
    const int b = base + (int)threadIdx.x;
    const uint32_t x = b < nb ? block_counts[b] : 0u;
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
    if (b < nb) block_counts[b] = start;
    __syncthreads();
    if (threadIdx.x == 1023) s_w[0] = start + x;
    __syncthreads();
    carry = s_w[0];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    *n_out = (int64_t)carry;
    if ((int64_t)carry > capacity) atomicOr(status, kStatusCapacity);
  }
}

// Rotation of the unit quaternion (w, x, y, z) applied to u.
__device__ __forceinline__ float3 rotate(float4 q, float3 u) {
  const float w = q.x, x = q.y, y = q.z, z = q.w;
  const float r00 = 1.f - 2.f * (y * y + z * z), r01 = 2.f * (x * y - w * z),
              r02 = 2.f * (x * z + w * y);
  const float r10 = 2.f * (x * y + w * z), r11 = 1.f - 2.f * (x * x + z * z),
              r12 = 2.f * (y * z - w * x);
  const float r20 = 2.f * (x * z - w * y), r21 = 2.f * (y * z + w * x),
              r22 = 1.f - 2.f * (x * x + y * y);
  return make_float3(r00 * u.x + r01 * u.y + r02 * u.z, r10 * u.x + r11 * u.y + r12 * u.z,
                     r20 * u.x + r21 * u.y + r22 * u.z);
}

struct DpTensors {
  float4* means;
  float4* log_scales;
  float4* quats;
  float* logit;
  float* sh;
};
struct DpConst {
  const float4* means;
  const float4* log_scales;
  const float4* quats;
  const float* logit;
  const float* sh;
};

// Moments of Gaussian i copied to slot o, or zeroed (all but the SH block,
// which the warp moves together: copy_sh_warp).
__device__ __forceinline__ void put_moments(const DpConst& in, const DpTensors& out, int64_t i,
                                            int64_t o, bool zero) {
  const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
  out.means[o] = zero ? z4 : __ldg(&in.means[i]);
  out.log_scales[o] = zero ? z4 : __ldg(&in.log_scales[i]);
  out.quats[o] = zero ? z4 : __ldg(&in.quats[i]);
  out.logit[o] = zero ? 0.f : __ldg(&in.logit[i]);
}

// The SH blocks (parameters and both moments) of the warp's 32 Gaussians,
// moved by the whole warp so that every access is part of a contiguous run:
// the warp walks the (Gaussian, element) items of its Gaussians' three
// blocks 32 at a time (float4 elements when k3 is a multiple of 4), four
// rounds of loads in flight. A kept Gaussian keeps its moments; a clone's
// second copy and both split children get zeros.
template <typename E>
__device__ __forceinline__ void copy_sh_warp(const DpConst& p_in, const DpConst& m_in,
                                             const DpConst& v_in, const DpTensors& p_out,
                                             const DpTensors& m_out, const DpTensors& v_out,
                                             int k3, int8_t c_lane, int64_t pos_lane,
                                             int64_t i_warp) {
  constexpr int kW = (int)(sizeof(E) / sizeof(float));
  const int per = k3 / kW;           // elements per block
  const int items = 3 * per;         // per Gaussian
  const int total = 32 * items;      // a multiple of 32: every lane runs every round
  const int lane = threadIdx.x & 31;
#pragma unroll 4
  for (int f = lane; f < total; f += 32) {
    const int j = f / items, r = f - j * items;
    const int c = __shfl_sync(0xffffffffu, (int)c_lane, j);
    const int64_t pos = __shfl_sync(0xffffffffu, pos_lane, j);
    if (c == 0) continue;            // pruned
    const int arr = r / per, q = r - arr * per;
    const float* src = arr == 0 ? p_in.sh : (arr == 1 ? m_in.sh : v_in.sh);
    float* dst = arr == 0 ? p_out.sh : (arr == 1 ? m_out.sh : v_out.sh);
    const E v = __ldg(reinterpret_cast<const E*>(src + (i_warp + j) * k3) + q);
    const int nout = c == 1 ? 1 : 2;  // kKeep: one output, clone / split: two
    for (int copy = 0; copy < nout; ++copy) {
      const bool zero = arr > 0 && (c == 3 || copy == 1);
      E* d = reinterpret_cast<E*>(dst + (pos + copy) * k3) + q;
      *d = zero ? E{} : v;
    }
  }
}

// Every field but the SH blocks of Gaussian i's outputs at pos (and pos + 1).
__device__ __forceinline__ void emit_fields(const DpConst& p_in, const DpConst& m_in,
                                            const DpConst& v_in, const float* __restrict__ z,
                                            int64_t i, int64_t pos, int8_t c,
                                            float log_split_shrink, const DpTensors& p_out,
                                            const DpTensors& m_out, const DpTensors& v_out) {
  const float4 mu = __ldg(&p_in.means[i]);
  const float4 ls = __ldg(&p_in.log_scales[i]);
  const float4 q = __ldg(&p_in.quats[i]);
  const float lg = __ldg(&p_in.logit[i]);
  if (c == kKeep || c == kClone) {
    for (int copy = 0; copy < (c == kClone ? 2 : 1); ++copy) {
      const int64_t o = pos + copy;
      p_out.means[o] = mu;
      p_out.log_scales[o] = ls;
      p_out.quats[o] = q;
      p_out.logit[o] = lg;
      put_moments(m_in, m_out, i, o, copy == 1);
      put_moments(v_in, v_out, i, o, copy == 1);
    }
    return;
  }
  // split: two children
  const float qn = rsqrtf(q.x * q.x + q.y * q.y + q.z * q.z + q.w * q.w);
  const float4 qu = make_float4(q.x * qn, q.y * qn, q.z * qn, q.w * qn);
  const float3 s = make_float3(__expf(ls.x), __expf(ls.y), __expf(ls.z));
  const float4 lsc = make_float4(ls.x - log_split_shrink, ls.y - log_split_shrink,
                                 ls.z - log_split_shrink, ls.w);
  for (int ch = 0; ch < 2; ++ch) {
    const int64_t o = pos + ch;
    const float* zc = z + (i * 2 + ch) * 3;
    const float3 d = rotate(qu, make_float3(s.x * __ldg(&zc[0]), s.y * __ldg(&zc[1]),
                                            s.z * __ldg(&zc[2])));
    p_out.means[o] = make_float4(mu.x + d.x, mu.y + d.y, mu.z + d.z, mu.w);
    p_out.log_scales[o] = lsc;
    p_out.quats[o] = q;
    p_out.logit[o] = lg;
    put_moments(m_in, m_out, i, o, true);
    put_moments(v_in, v_out, i, o, true);
  }
}

__global__ void __launch_bounds__(kDpThreads, 6) k_dp_emit(
    DpConst p_in, DpConst m_in, DpConst v_in, const float* __restrict__ z, int n, int k3,
    float log_split_shrink, const int8_t* __restrict__ codes,
    const uint32_t* __restrict__ block_offsets, const int64_t* __restrict__ n_out,
    int64_t capacity, DpTensors p_out, DpTensors m_out, DpTensors v_out) {
  __shared__ uint32_t s_w[kDpThreads / 32];
  if (*n_out > capacity) return;  // nothing is written
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t i = (int64_t)blockIdx.x * kDpThreads + threadIdx.x;
  const int8_t c = i < n ? codes[i] : kPrune;
  const uint32_t cnt = (uint32_t)dp_count(c);
  uint32_t incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) s_w[warp] = incl;
  __syncthreads();
  uint32_t before = 0;
#pragma unroll
  for (int w = 0; w < kDpThreads / 32; ++w) before += w < warp ? s_w[w] : 0u;
  const int64_t pos = (int64_t)block_offsets[blockIdx.x] + before + incl - cnt;
  if (c != kPrune) emit_fields(p_in, m_in, v_in, z, i, pos, c, log_split_shrink, p_out, m_out,
                               v_out);
  // the SH blocks, the warp together
  if ((k3 & 3) == 0)
    copy_sh_warp<float4>(p_in, m_in, v_in, p_out, m_out, v_out, k3, c, pos, i - lane);
  else
    copy_sh_warp<float>(p_in, m_in, v_in, p_out, m_out, v_out, k3, c, pos, i - lane);
}

// Output counts of each block of decisions (the quantised-SH map).
__global__ void __launch_bounds__(kDpThreads) k_dsq_count(const int8_t* __restrict__ codes, int n,
                                                          uint32_t* __restrict__ block_counts) {
  __shared__ uint32_t s_w[kDpThreads / 32];
  const int i = blockIdx.x * kDpThreads + threadIdx.x;
  uint32_t s = i < n ? (uint32_t)dp_count(codes[i]) : 0u;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) s_w[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t t = 0;
#pragma unroll
    for (int w = 0; w < kDpThreads / 32; ++w) t += s_w[w];
    block_counts[blockIdx.x] = t;
  }
}

// src[o] for every output o of input i (positions as k_dp_emit takes them):
// i, with bit 31 set for a clone's copy and both split children (their
// moments start at zero).
__global__ void __launch_bounds__(kDpThreads) k_dsq_map(const int8_t* __restrict__ codes, int n,
                                                        const uint32_t* __restrict__ block_offsets,
                                                        const int64_t* __restrict__ n_out,
                                                        int64_t capacity,
                                                        uint32_t* __restrict__ src) {
  __shared__ uint32_t s_w[kDpThreads / 32];
  if (*n_out > capacity) return;  // nothing is written
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t i = (int64_t)blockIdx.x * kDpThreads + threadIdx.x;
  const int8_t c = i < n ? codes[i] : kPrune;
  const uint32_t cnt = (uint32_t)dp_count(c);
  uint32_t incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) s_w[warp] = incl;
  __syncthreads();
  uint32_t before = 0;
#pragma unroll
  for (int w = 0; w < kDpThreads / 32; ++w) before += w < warp ? s_w[w] : 0u;
  const int64_t pos = (int64_t)block_offsets[blockIdx.x] + before + incl - cnt;
  const uint32_t id = (uint32_t)i, zero = 0x80000000u;
  if (c == kKeep) {
    src[pos] = id;
  } else if (c == kClone) {
    src[pos] = id;
    src[pos + 1] = id | zero;
  } else if (c == kSplit) {
    src[pos] = id | zero;
    src[pos + 1] = id | zero;
  }
}


DpConst to_const(const DpTensorPtrs& t) {
  return DpConst{reinterpret_cast<const float4*>(t.means), reinterpret_cast<const float4*>(t.log_scales),
                 reinterpret_cast<const float4*>(t.quats), t.logit, t.sh};
}
DpTensors to_mut(const DpTensorPtrs& t) {
  return DpTensors{reinterpret_cast<float4*>(t.means), reinterpret_cast<float4*>(t.log_scales),
                   reinterpret_cast<float4*>(t.quats), t.logit, t.sh};
}

}  // namespace

int64_t densify_blocks(int64_t n) { return (n + kDpThreads - 1) / kDpThreads; }

cudaError_t launch_densify_and_prune(const DpTensorPtrs& p_in, const DpTensorPtrs& m_in,
                                     const DpTensorPtrs& v_in, const float* accum,
                                     const int32_t* denom, const float* z, int n, int k3,
                                     const DensifyArgs& args, int8_t* codes,
                                     uint32_t* block_counts, int64_t capacity, int64_t* n_out,
                                     uint32_t* status, const DpTensorPtrs& p_out,
                                     const DpTensorPtrs& m_out, const DpTensorPtrs& v_out,
                                     cudaStream_t stream) {
  const int nb = (int)densify_blocks(n);
  if (nb == 0) return cudaMemsetAsync(n_out, 0, sizeof(int64_t), stream);
  k_dp_decide<<<nb, kDpThreads, 0, stream>>>(reinterpret_cast<const float4*>(p_in.log_scales),
                                             p_in.logit, accum, denom, n, args, codes,
                                             block_counts);
  k_dp_scan<<<1, 1024, 0, stream>>>(block_counts, nb, capacity, n_out, status);
  k_dp_emit<<<nb, kDpThreads, 0, stream>>>(to_const(p_in), to_const(m_in), to_const(v_in), z, n,
                                           k3, args.log_split_shrink, codes, block_counts, n_out,
                                           capacity, to_mut(p_out), to_mut(m_out), to_mut(v_out));
  return cudaGetLastError();
}

cudaError_t launch_densify_map(const int8_t* decisions, int n, uint32_t* block_counts,
                               int64_t capacity, int64_t* n_out, uint32_t* src,
                               uint32_t* status, cudaStream_t stream) {
  const int nb = (int)densify_blocks(n);
  if (nb == 0) return cudaMemsetAsync(n_out, 0, sizeof(int64_t), stream);
  k_dsq_count<<<nb, kDpThreads, 0, stream>>>(decisions, n, block_counts);
  k_dp_scan<<<1, 1024, 0, stream>>>(block_counts, nb, capacity, n_out, status);
  k_dsq_map<<<nb, kDpThreads, 0, stream>>>(decisions, n, block_counts, n_out, capacity, src);
  return cudaGetLastError();
}

}  // namespace gsb
