// quant.cu -- quantised SH state: encode, decode, and Adam on the codes.
//
// The Spirula VRAM page (sec. 魔法一, quantised training) keeps the SH
// coefficients as 8- or 16-bit fixed point, every 256 units sharing one
// (min, max) pair, gradients in float32 and the Adam moments in 16-bit words
// in a transposed layout. Here a unit is one SH value and the layout is
// coefficient-major: codes [3K][n_pad], one group = one coefficient of 256
// consecutive Gaussians, bounds float2 [3K][n_pad / 256]; the moments are
// bfloat16 [3K][n_pad] beside them. A code q decodes to
// min + q (max - min) / (2^b - 1).
//
// One 256-thread block owns one group of Gaussians for every coefficient.
// The float32 SH (or its gradient) of those Gaussians, [256][3K] in the
// parameter layout, is staged through shared memory transposed, so that a
// warp then works on whole coefficients: lane l holds the four consecutive
// Gaussians 4 l .. 4 l + 3 of each half of the group, moves their codes and
// moments with one vector access per array and half, and takes the group's
// min and max with warp shuffles. Loads are issued for both halves before
// any arithmetic, so each warp keeps six vector loads in flight.

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <type_traits>

#include "gs.h"
#include "gs_internal.h"

namespace gsb {
namespace {

constexpr int kQG = GS_QUANT_GROUP;   // Gaussians per group = threads per block
constexpr int kQPitch = kQG + 4;      // shared row of one coefficient (16-byte rows)
constexpr int kPerLane = 8;           // values per lane and coefficient: 2 halves x 4

template <int BITS>
struct CodeT;
template <>
struct CodeT<8> {
  using T = uint8_t;
  using Vec = uint32_t;   // four codes
  __device__ static void unpack(Vec w, float (&c)[4]) {
#pragma unroll
    for (int k = 0; k < 4; ++k) c[k] = (float)((w >> (8 * k)) & 0xffu);
  }
  __device__ static Vec pack(const int (&c)[4]) {
    return (uint32_t)c[0] | ((uint32_t)c[1] << 8) | ((uint32_t)c[2] << 16) |
           ((uint32_t)c[3] << 24);
  }
};
template <>
struct CodeT<16> {
  using T = uint16_t;
  using Vec = uint2;      // four codes
  __device__ static void unpack(Vec w, float (&c)[4]) {
    c[0] = (float)(w.x & 0xffffu);
    c[1] = (float)(w.x >> 16);
    c[2] = (float)(w.y & 0xffffu);
    c[3] = (float)(w.y >> 16);
  }
  __device__ static Vec pack(const int (&c)[4]) {
    return make_uint2((uint32_t)c[0] | ((uint32_t)c[1] << 16),
                      (uint32_t)c[2] | ((uint32_t)c[3] << 16));
  }
};

// four bfloat16 in a uint2 <-> float
__device__ __forceinline__ void unpack_bf16(uint2 w, float (&f)[4]) {
  f[0] = __uint_as_float(w.x << 16);
  f[1] = __uint_as_float(w.x & 0xffff0000u);
  f[2] = __uint_as_float(w.y << 16);
  f[3] = __uint_as_float(w.y & 0xffff0000u);
}
__device__ __forceinline__ uint16_t bf16_bits(float f) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

// SplitMix64 (Steele, Lea and Flood 2014): output number counter + 1 from
// `seed`, i.e. the variant-13 mix of seed + (counter + 1) * gamma.
__device__ __forceinline__ uint64_t splitmix64(uint64_t seed, uint64_t counter) {
  uint64_t z = seed + (counter + 1ull) * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__device__ __forceinline__ float warp_min(float v) {
  for (int o = 16; o; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Position in the group of the lane's value e (half e / 4, element e % 4).
__device__ __forceinline__ int lane_pos(int e) {
  return 128 * (e >> 2) + 4 * (int)(threadIdx.x & 31) + (e & 3);
}

// [cnt][K3] floats at src -> s[j][t] (t < cnt), coalesced reads: 16-byte
// loads when K3 is a multiple of 4 (the group's rows start 16-byte aligned
// when src is), else 4-byte loads.
template <int K3>
__device__ __forceinline__ void stage_transposed(const float* __restrict__ src, int cnt,
                                                 float* s, bool vec_ok) {
  if constexpr (K3 % 4 == 0) {
    if (vec_ok) {
      constexpr int kQuads = K3 / 4;
      const int total = cnt * kQuads;
      const float4* src4 = reinterpret_cast<const float4*>(src);
#pragma unroll 4
      for (int e = threadIdx.x; e < total; e += kQG) {
        const int t = e / kQuads;
        const int j = 4 * (e - t * kQuads);
        const float4 v = __ldg(src4 + e);
        s[j * kQPitch + t] = v.x;
        s[(j + 1) * kQPitch + t] = v.y;
        s[(j + 2) * kQPitch + t] = v.z;
        s[(j + 3) * kQPitch + t] = v.w;
      }
      return;
    }
  }
  const int total = cnt * K3;
#pragma unroll 4
  for (int e = threadIdx.x; e < total; e += kQG) {
    const int t = e / K3;
    s[(e - t * K3) * kQPitch + t] = __ldg(src + e);
  }
}

// Store four consecutive values at row[base ..]: one vector store when all
// four are real Gaussians, element stores for the ragged end of the last group.
template <typename T, typename Vec>
__device__ __forceinline__ void store4(T* row, int base, int cnt, Vec packed,
                                       const T (&each)[4]) {
  if (base + 4 <= cnt) {
    *reinterpret_cast<Vec*>(row + base) = packed;
  } else {
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (base + k < cnt) row[base + k] = each[k];
  }
}

// Encode the lane's values x[e] (group positions lane_pos(e) of coefficient
// j) with the group's min and max, in float32 exactly as stated above:
// t = (x - min) * ((2^b - 1) / (max - min)), then rint(t) or floor(t + u).
template <int BITS>
__device__ __forceinline__ void encode_group(const float (&x)[kPerLane], int cnt, int j, int g,
                                             int64_t i0, int64_t n_pad, int n_groups,
                                             typename CodeT<BITS>::T* __restrict__ codes,
                                             float2* __restrict__ bounds, int rounding,
                                             uint64_t seed, uint64_t ctr_base) {
  using C = CodeT<BITS>;
  float lo = INFINITY, hi = -INFINITY;
#pragma unroll
  for (int e = 0; e < kPerLane; ++e)
    if (lane_pos(e) < cnt) {
      lo = fminf(lo, x[e]);
      hi = fmaxf(hi, x[e]);
    }
  lo = warp_min(lo);
  hi = warp_max(hi);
  if ((threadIdx.x & 31) == 0) bounds[(int64_t)j * n_groups + g] = make_float2(lo, hi);
  constexpr int qmax = (1 << BITS) - 1;
  const float range = __fsub_rn(hi, lo);
  const float inv = range > 0.f ? __fdiv_rn((float)qmax, range) : 0.f;
  typename C::T* row = codes + (int64_t)j * n_pad + i0;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    int c[4];
    typename C::T each[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int e = 4 * h + k;
      const float t = __fmul_rn(__fsub_rn(x[e], lo), inv);
      int q;
      if (rounding == 0) {
        q = __float2int_rn(t);
      } else {
        const uint64_t ctr = ctr_base + ((uint64_t)j << 31) + (uint64_t)(i0 + lane_pos(e));
        const float u = __uint2float_rn((unsigned)(splitmix64(seed, ctr) >> 40)) * 0x1p-24f;
        q = __float2int_rd(__fadd_rn(t, u));
      }
      c[k] = min(max(q, 0), qmax);
      each[k] = (typename C::T)c[k];
    }
    const int base = lane_pos(4 * h);
    if (base < cnt) store4(row, base, cnt, C::pack(c), each);
  }
}

template <int BITS, int K3>
__global__ void __launch_bounds__(kQG) k_sh_quantize(const float* __restrict__ sh, int64_t n,
                                                     int64_t n_pad,
                                                     typename CodeT<BITS>::T* __restrict__ codes,
                                                     float2* __restrict__ bounds) {
  extern __shared__ float4 s_q4[];
  float* s_q = reinterpret_cast<float*>(s_q4);
  const int g = blockIdx.x;
  const int64_t i0 = (int64_t)g * kQG;
  const int cnt = (int)(n - i0 < kQG ? n - i0 : kQG);
  const int n_groups = (int)(n_pad / kQG);
  stage_transposed<K3>(sh + i0 * K3, cnt, s_q,
                       (reinterpret_cast<uintptr_t>(sh) & 15) == 0);
  __syncthreads();
  const int warp = threadIdx.x >> 5;
  for (int j = warp; j < K3; j += kQG / 32) {
    float x[kPerLane];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const float4 v = *reinterpret_cast<const float4*>(s_q + j * kQPitch + lane_pos(4 * h));
      x[4 * h] = v.x;
      x[4 * h + 1] = v.y;
      x[4 * h + 2] = v.z;
      x[4 * h + 3] = v.w;
    }
    encode_group<BITS>(x, cnt, j, g, i0, n_pad, n_groups, codes, bounds, 0, 0, 0);
  }
}

template <int BITS, int K3>
__global__ void __launch_bounds__(kQG)
    k_sh_dequantize(const typename CodeT<BITS>::T* __restrict__ codes,
                    const float2* __restrict__ bounds, int64_t n, int64_t n_pad,
                    float* __restrict__ sh) {
  using C = CodeT<BITS>;
  extern __shared__ float4 s_q4[];
  float* s_q = reinterpret_cast<float*>(s_q4);
  const int g = blockIdx.x;
  const int64_t i0 = (int64_t)g * kQG;
  const int cnt = (int)(n - i0 < kQG ? n - i0 : kQG);
  const int n_groups = (int)(n_pad / kQG);
  const int warp = threadIdx.x >> 5;
  constexpr float qmax = (float)((1 << BITS) - 1);
  for (int j = warp; j < K3; j += kQG / 32) {
    const float2 b = __ldg(bounds + (int64_t)j * n_groups + g);
    const float step = __fdiv_rn(__fsub_rn(b.y, b.x), qmax);
    const typename C::T* row = codes + (int64_t)j * n_pad + i0;
    typename C::Vec w[2];
#pragma unroll
    for (int h = 0; h < 2; ++h)
      w[h] = __ldg(reinterpret_cast<const typename C::Vec*>(row + lane_pos(4 * h)));
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float c[4];
      C::unpack(w[h], c);
      float4 o;
      o.x = __fmaf_rn(c[0], step, b.x);
      o.y = __fmaf_rn(c[1], step, b.x);
      o.z = __fmaf_rn(c[2], step, b.x);
      o.w = __fmaf_rn(c[3], step, b.x);
      *reinterpret_cast<float4*>(s_q + j * kQPitch + lane_pos(4 * h)) = o;
    }
  }
  __syncthreads();
  float* dst = sh + i0 * K3;
  const int total = cnt * K3;
  for (int e = threadIdx.x; e < total; e += kQG) {
    const int t = e / K3;
    dst[e] = s_q[(e - t * K3) * kQPitch + t];
  }
}

template <int BITS, int K3>
__global__ void __launch_bounds__(kQG)
    k_adam_sh_quant(typename CodeT<BITS>::T* __restrict__ codes, float2* __restrict__ bounds,
                    const float* __restrict__ grad, uint16_t* __restrict__ m_buf,
                    uint16_t* __restrict__ v_buf, int64_t n, int64_t n_pad, float lr,
                    float beta1, float beta2, float eps, float ibc1, float ibc2, int rounding,
                    uint64_t seed, uint64_t ctr_base) {
  using C = CodeT<BITS>;
  extern __shared__ float4 s_q4[];
  float* s_q = reinterpret_cast<float*>(s_q4);
  const int g = blockIdx.x;
  const int64_t i0 = (int64_t)g * kQG;
  const int cnt = (int)(n - i0 < kQG ? n - i0 : kQG);
  const int n_groups = (int)(n_pad / kQG);
  const int warp = threadIdx.x >> 5;
  constexpr float qmax = (float)((1 << BITS) - 1);
  // the codes and moments of the warp's first coefficient are requested
  // before the gradient staging, so both streams are in flight together
  typename C::Vec w[2];
  uint2 mw[2], vw[2];
  auto load_coef = [&](int j) {
    const int64_t off = (int64_t)j * n_pad + i0;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int base = lane_pos(4 * h);
      w[h] = *reinterpret_cast<const typename C::Vec*>(codes + off + base);
      mw[h] = *reinterpret_cast<const uint2*>(m_buf + off + base);
      vw[h] = *reinterpret_cast<const uint2*>(v_buf + off + base);
    }
  };
  if (warp < K3) load_coef(warp);
  stage_transposed<K3>(grad + i0 * K3, cnt, s_q, (reinterpret_cast<uintptr_t>(grad) & 15) == 0);
  __syncthreads();
  for (int j = warp; j < K3; j += kQG / 32) {
    const int64_t off = (int64_t)j * n_pad + i0;
    const float2 b = bounds[(int64_t)j * n_groups + g];
    if (j != warp) load_coef(j);   // the padding past n is in bounds
    const float step = __fdiv_rn(__fsub_rn(b.y, b.x), qmax);
    float x[kPerLane];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int base = lane_pos(4 * h);
      const float4 gv = *reinterpret_cast<const float4*>(s_q + j * kQPitch + base);
      const float gr[4] = {gv.x, gv.y, gv.z, gv.w};
      float c[4], m[4], v[4];
      C::unpack(w[h], c);
      unpack_bf16(mw[h], m);
      unpack_bf16(vw[h], v);
      uint16_t mb[4], vb[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const float p = __fmaf_rn(c[k], step, b.x);
        m[k] = beta1 * m[k] + (1.f - beta1) * gr[k];
        v[k] = beta2 * v[k] + (1.f - beta2) * gr[k] * gr[k];
        x[4 * h + k] = p - lr * (m[k] * ibc1) / (sqrtf(v[k] * ibc2) + eps);
        mb[k] = bf16_bits(m[k]);
        vb[k] = bf16_bits(v[k]);
      }
      if (base < cnt) {
        store4(m_buf + off, base, cnt,
               make_uint2(mb[0] | ((uint32_t)mb[1] << 16), mb[2] | ((uint32_t)mb[3] << 16)),
               mb);
        store4(v_buf + off, base, cnt,
               make_uint2(vb[0] | ((uint32_t)vb[1] << 16), vb[2] | ((uint32_t)vb[3] << 16)),
               vb);
      }
    }
    // every lane has read the group's old bounds before lane 0 rewrites them
    __syncwarp();
    encode_group<BITS>(x, cnt, j, g, i0, n_pad, n_groups, codes, bounds, rounding, seed,
                       ctr_base);
  }
}

template <typename K>
cudaError_t set_smem(K kernel, size_t bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
}

// Calls f(integral_constant K3) for the four SH sizes.
template <typename F>
cudaError_t with_k3(int k3, F&& f) {
  switch (k3) {
    case 3: return f(std::integral_constant<int, 3>());
    case 12: return f(std::integral_constant<int, 12>());
    case 27: return f(std::integral_constant<int, 27>());
    case 48: return f(std::integral_constant<int, 48>());
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

cudaError_t launch_sh_quantize(const float* sh, int64_t n, int k3, int bits, void* codes,
                               float2* bounds, cudaStream_t stream) {
  const int64_t n_pad = (n + kQG - 1) / kQG * kQG;
  const unsigned grid = (unsigned)(n_pad / kQG);
  const size_t smem = sizeof(float) * k3 * kQPitch;
  return with_k3(k3, [&](auto K) -> cudaError_t {
    constexpr int K3 = decltype(K)::value;
    cudaError_t e;
    if (bits == 8) {
      if ((e = set_smem(k_sh_quantize<8, K3>, smem)) != cudaSuccess) return e;
      k_sh_quantize<8, K3><<<grid, kQG, smem, stream>>>(sh, n, n_pad,
                                                         static_cast<uint8_t*>(codes), bounds);
    } else {
      if ((e = set_smem(k_sh_quantize<16, K3>, smem)) != cudaSuccess) return e;
      k_sh_quantize<16, K3><<<grid, kQG, smem, stream>>>(sh, n, n_pad,
                                                          static_cast<uint16_t*>(codes), bounds);
    }
    return cudaGetLastError();
  });
}

cudaError_t launch_sh_dequantize(const void* codes, const float2* bounds, int64_t n, int k3,
                                 int bits, float* sh, cudaStream_t stream) {
  const int64_t n_pad = (n + kQG - 1) / kQG * kQG;
  const unsigned grid = (unsigned)(n_pad / kQG);
  const size_t smem = sizeof(float) * k3 * kQPitch;
  return with_k3(k3, [&](auto K) -> cudaError_t {
    constexpr int K3 = decltype(K)::value;
    cudaError_t e;
    if (bits == 8) {
      if ((e = set_smem(k_sh_dequantize<8, K3>, smem)) != cudaSuccess) return e;
      k_sh_dequantize<8, K3><<<grid, kQG, smem, stream>>>(static_cast<const uint8_t*>(codes),
                                                           bounds, n, n_pad, sh);
    } else {
      if ((e = set_smem(k_sh_dequantize<16, K3>, smem)) != cudaSuccess) return e;
      k_sh_dequantize<16, K3><<<grid, kQG, smem, stream>>>(static_cast<const uint16_t*>(codes),
                                                            bounds, n, n_pad, sh);
    }
    return cudaGetLastError();
  });
}

cudaError_t launch_adam_sh_quant(void* codes, float2* bounds, const float* grad, uint16_t* m,
                                 uint16_t* v, int64_t n, int k3, int bits, float lr, float beta1,
                                 float beta2, float eps, int64_t step, int rounding,
                                 uint64_t seed, cudaStream_t stream) {
  const int64_t n_pad = (n + kQG - 1) / kQG * kQG;
  const unsigned grid = (unsigned)(n_pad / kQG);
  const size_t smem = sizeof(float) * k3 * kQPitch;
  const float ibc1 = (float)(1.0 / (1.0 - pow((double)beta1, (double)step)));
  const float ibc2 = (float)(1.0 / (1.0 - pow((double)beta2, (double)step)));
  const uint64_t ctr_base = (uint64_t)step << 37;
  return with_k3(k3, [&](auto K) -> cudaError_t {
    constexpr int K3 = decltype(K)::value;
    cudaError_t e;
    if (bits == 8) {
      if ((e = set_smem(k_adam_sh_quant<8, K3>, smem)) != cudaSuccess) return e;
      k_adam_sh_quant<8, K3><<<grid, kQG, smem, stream>>>(
          static_cast<uint8_t*>(codes), bounds, grad, m, v, n, n_pad, lr, beta1, beta2, eps,
          ibc1, ibc2, rounding, seed, ctr_base);
    } else {
      if ((e = set_smem(k_adam_sh_quant<16, K3>, smem)) != cudaSuccess) return e;
      k_adam_sh_quant<16, K3><<<grid, kQG, smem, stream>>>(
          static_cast<uint16_t*>(codes), bounds, grad, m, v, n, n_pad, lr, beta1, beta2, eps,
          ibc1, ibc2, rounding, seed, ctr_base);
    }
    return cudaGetLastError();
  });
}

}  // namespace gsb
