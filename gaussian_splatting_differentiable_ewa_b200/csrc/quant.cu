// quant.cu -- quantised SH state: encode, decode, Adam on the codes, and
// densify_and_prune of the codes.
//
// The Spirula VRAM page (sec. 魔法一, quantised training) keeps the SH
// coefficients as 8- or 16-bit fixed point, every 256 units sharing one
// (min, max) pair, gradients in float32 and the Adam state in 16-bit words,
// parameter and moments transposed and packed together. Here a unit is one SH
// value and both layouts are coefficient-major, one group = one coefficient of
// 256 consecutive Gaussians, bounds float2 [3K][n_pad / 256]:
//   planar  codes [3K][n_pad] (8 or 16 bits), bfloat16 moments [3K][n_pad]
//           in two arrays beside them;
//   packed  uint16 blocks [3K][n_pad / 32][3][32]: the codes of 32
//           consecutive Gaussians, then their two moments, 192 bytes.
// A code q decodes to min + q (max - min) / (2^b - 1).
//
// One 256-thread block owns one group of Gaussians for every coefficient.
// The float32 SH (or its gradient) of those Gaussians, [256][3K] in the
// parameter layout, is staged through shared memory transposed, so that a
// warp then works on whole coefficients: lane l holds the four consecutive
// Gaussians 4 l .. 4 l + 3 of each half of the group (always inside one
// packed block), moves their codes and moments with one vector access per
// array and half, and takes the group's min and max with warp shuffles.
// Loads are issued for both halves before any arithmetic, so each warp keeps
// six vector loads in flight.

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

// Where the four values (j, i .. i + 3) of a layout live (i a multiple of 4).
// S is the stored code type (packed blocks hold 16-bit words for 8-bit codes
// too); the moments follow the codes of a packed block at +32 and +64 words.
template <int BITS, int LAYOUT>
struct QL;
template <int BITS>
struct QL<BITS, GS_QUANT_PLANAR> {
  using S = CodeT<BITS>;
  __device__ static typename S::T* code(void* codes, int j, int64_t i, int64_t n_pad) {
    return static_cast<typename S::T*>(codes) + (int64_t)j * n_pad + i;
  }
  __device__ static uint16_t* mom(void*, uint16_t* arr, int, int j, int64_t i, int64_t n_pad) {
    return arr + (int64_t)j * n_pad + i;
  }
};
template <int BITS>
struct QL<BITS, GS_QUANT_PACKED> {
  using S = CodeT<16>;
  __device__ static uint16_t* code(void* codes, int j, int64_t i, int64_t n_pad) {
    return static_cast<uint16_t*>(codes) + (((int64_t)j * (n_pad >> 5) + (i >> 5)) * 96 + (i & 31));
  }
  __device__ static uint16_t* mom(void* codes, uint16_t*, int which, int j, int64_t i,
                                  int64_t n_pad) {
    return code(codes, j, i, n_pad) + 32 * which;
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

// Store four consecutive values at p: one vector store when all four are
// real Gaussians (avail >= 4), element stores for the ragged end of the last
// group.
template <typename T, typename Vec>
__device__ __forceinline__ void store4(T* p, int avail, Vec packed, const T (&each)[4]) {
  if (avail >= 4) {
    *reinterpret_cast<Vec*>(p) = packed;
  } else {
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (k < avail) p[k] = each[k];
  }
}

__device__ __forceinline__ uint2 pack_bf16x4(const uint16_t (&b)[4]) {
  return make_uint2(b[0] | ((uint32_t)b[1] << 16), b[2] | ((uint32_t)b[3] << 16));
}

// Encode the lane's values x[e] (group positions lane_pos(e) of coefficient
// j) with the group's min and max, in float32 exactly as stated above:
// t = (x - min) * ((2^b - 1) / (max - min)), then rint(t) or floor(t + u).
template <int BITS, int LAYOUT>
__device__ __forceinline__ void encode_group(const float (&x)[kPerLane], int cnt, int j, int g,
                                             int64_t i0, int64_t n_pad, int n_groups,
                                             void* __restrict__ codes,
                                             float2* __restrict__ bounds, int rounding,
                                             uint64_t seed, uint64_t ctr_base) {
  using L = QL<BITS, LAYOUT>;
  using C = typename L::S;
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
    if (base < cnt) store4(L::code(codes, j, i0 + base, n_pad), cnt - base, C::pack(c), each);
  }
}

template <int BITS, int K3, int LAYOUT>
__global__ void __launch_bounds__(kQG) k_sh_quantize(const float* __restrict__ sh, int64_t n,
                                                     int64_t n_pad, void* __restrict__ codes,
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
    encode_group<BITS, LAYOUT>(x, cnt, j, g, i0, n_pad, n_groups, codes, bounds, 0, 0, 0);
  }
}

template <int BITS, int K3, int LAYOUT>
__global__ void __launch_bounds__(kQG)
    k_sh_dequantize(const void* __restrict__ codes, const float2* __restrict__ bounds, int64_t n,
                    int64_t n_pad, float* __restrict__ sh) {
  using L = QL<BITS, LAYOUT>;
  using C = typename L::S;
  extern __shared__ float4 s_q4[];
  float* s_q = reinterpret_cast<float*>(s_q4);
  const int g = blockIdx.x;
  const int64_t i0 = (int64_t)g * kQG;
  const int cnt = (int)(n - i0 < kQG ? n - i0 : kQG);
  const int n_groups = (int)(n_pad / kQG);
  const int warp = threadIdx.x >> 5;
  constexpr float qmax = (float)((1 << BITS) - 1);
  void* cw = const_cast<void*>(codes);
  for (int j = warp; j < K3; j += kQG / 32) {
    const float2 b = __ldg(bounds + (int64_t)j * n_groups + g);
    const float step = __fdiv_rn(__fsub_rn(b.y, b.x), qmax);
    typename C::Vec w[2];
#pragma unroll
    for (int h = 0; h < 2; ++h)
      w[h] = __ldg(reinterpret_cast<const typename C::Vec*>(
          L::code(cw, j, i0 + lane_pos(4 * h), n_pad)));
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

template <int BITS, int K3, int LAYOUT>
__global__ void __launch_bounds__(kQG)
    k_adam_sh_quant(void* __restrict__ codes, float2* __restrict__ bounds,
                    const float* __restrict__ grad, uint16_t* __restrict__ m_buf,
                    uint16_t* __restrict__ v_buf, int64_t n, int64_t n_pad, float lr,
                    float beta1, float beta2, float eps, float ibc1, float ibc2, int rounding,
                    uint64_t seed, uint64_t ctr_base) {
  using L = QL<BITS, LAYOUT>;
  using C = typename L::S;
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
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int64_t i = i0 + lane_pos(4 * h);
      w[h] = *reinterpret_cast<const typename C::Vec*>(L::code(codes, j, i, n_pad));
      mw[h] = *reinterpret_cast<const uint2*>(L::mom(codes, m_buf, 1, j, i, n_pad));
      vw[h] = *reinterpret_cast<const uint2*>(L::mom(codes, v_buf, 2, j, i, n_pad));
    }
  };
  if (warp < K3) load_coef(warp);
  stage_transposed<K3>(grad + i0 * K3, cnt, s_q, (reinterpret_cast<uintptr_t>(grad) & 15) == 0);
  __syncthreads();
  for (int j = warp; j < K3; j += kQG / 32) {
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
        const int64_t i = i0 + base;
        store4(L::mom(codes, m_buf, 1, j, i, n_pad), cnt - base, pack_bf16x4(mb), mb);
        store4(L::mom(codes, v_buf, 2, j, i, n_pad), cnt - base, pack_bf16x4(vb), vb);
      }
    }
    // every lane has read the group's old bounds before lane 0 rewrites them
    __syncwarp();
    encode_group<BITS, LAYOUT>(x, cnt, j, g, i0, n_pad, n_groups, codes, bounds, rounding, seed,
                               ctr_base);
  }
}

// densify_and_prune of the codes: output group g (256 outputs) takes, for
// every coefficient, the decoded values of the inputs src[o] & 0x7fffffff
// it comes from, writes their moments (zero where bit 31 of src[o] is set)
// and encodes the group anew with nearest rounding. A count that differs
// from the map's (*n_out_dev) writes nothing and reports.
template <int BITS, int K3, int LAYOUT>
__global__ void __launch_bounds__(kQG)
    k_dsq_emit(const void* __restrict__ in_codes, const float2* __restrict__ in_bounds,
               const uint16_t* __restrict__ m_in, const uint16_t* __restrict__ v_in,
               int64_t n_pad_in, const uint32_t* __restrict__ src,
               const int64_t* __restrict__ n_out_dev, int64_t n_out, int64_t n_pad_out,
               void* __restrict__ out_codes, float2* __restrict__ out_bounds,
               uint16_t* __restrict__ m_out, uint16_t* __restrict__ v_out,
               uint32_t* __restrict__ status) {
  using L = QL<BITS, LAYOUT>;
  using C = typename L::S;
  if (*n_out_dev != n_out) {
    if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(status, kStatusCapacity);
    return;
  }
  const int g = blockIdx.x;
  const int64_t i0 = (int64_t)g * kQG;
  const int cnt = (int)(n_out - i0 < kQG ? n_out - i0 : kQG);
  const int n_groups_in = (int)(n_pad_in / kQG), n_groups_out = (int)(n_pad_out / kQG);
  const int warp = threadIdx.x >> 5;
  constexpr float qmax = (float)((1 << BITS) - 1);
  void* icw = const_cast<void*>(in_codes);
  uint16_t* mi = const_cast<uint16_t*>(m_in);
  uint16_t* vi = const_cast<uint16_t*>(v_in);
  uint32_t sv[kPerLane];
#pragma unroll
  for (int e = 0; e < kPerLane; ++e) sv[e] = lane_pos(e) < cnt ? __ldg(&src[i0 + lane_pos(e)]) : 0u;
  for (int j = warp; j < K3; j += kQG / 32) {
    float x[kPerLane];
    uint16_t mb[kPerLane], vb[kPerLane];
#pragma unroll
    for (int e = 0; e < kPerLane; ++e) {
      const int64_t i = sv[e] & 0x7fffffffu;
      const bool zero = (sv[e] >> 31) != 0u;
      const float2 b = __ldg(in_bounds + (int64_t)j * n_groups_in + (i >> 8));
      const float step = __fdiv_rn(__fsub_rn(b.y, b.x), qmax);
      const float q = (float)*L::code(icw, j, i, n_pad_in);
      x[e] = __fmaf_rn(q, step, b.x);
      mb[e] = zero ? (uint16_t)0 : *L::mom(icw, mi, 1, j, i, n_pad_in);
      vb[e] = zero ? (uint16_t)0 : *L::mom(icw, vi, 2, j, i, n_pad_in);
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int base = lane_pos(4 * h);
      if (base < cnt) {
        const uint16_t m4[4] = {mb[4 * h], mb[4 * h + 1], mb[4 * h + 2], mb[4 * h + 3]};
        const uint16_t v4[4] = {vb[4 * h], vb[4 * h + 1], vb[4 * h + 2], vb[4 * h + 3]};
        store4(L::mom(out_codes, m_out, 1, j, i0 + base, n_pad_out), cnt - base, pack_bf16x4(m4),
               m4);
        store4(L::mom(out_codes, v_out, 2, j, i0 + base, n_pad_out), cnt - base, pack_bf16x4(v4),
               v4);
      }
    }
    encode_group<BITS, LAYOUT>(x, cnt, j, g, i0, n_pad_out, n_groups_out, out_codes, out_bounds,
                               0, 0, 0);
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

// Calls f(integral_constant BITS, integral_constant LAYOUT) for the state's
// code width and layout.
template <typename F>
cudaError_t with_bits_layout(const gs_sh_quant& q, F&& f) {
  const bool packed = q.layout == GS_QUANT_PACKED;
  if (q.bits == 8)
    return packed ? f(std::integral_constant<int, 8>(), std::integral_constant<int, 1>())
                  : f(std::integral_constant<int, 8>(), std::integral_constant<int, 0>());
  return packed ? f(std::integral_constant<int, 16>(), std::integral_constant<int, 1>())
                : f(std::integral_constant<int, 16>(), std::integral_constant<int, 0>());
}

int64_t padded(int64_t n) { return (n + kQG - 1) / kQG * kQG; }

}  // namespace

cudaError_t launch_sh_quantize(const float* sh, const gs_sh_quant& q, cudaStream_t stream) {
  const int64_t n_pad = padded(q.n);
  const unsigned grid = (unsigned)(n_pad / kQG);
  const size_t smem = sizeof(float) * q.k3 * kQPitch;
  auto bounds = reinterpret_cast<float2*>(q.bounds);
  return with_k3(q.k3, [&](auto K) -> cudaError_t {
    return with_bits_layout(q, [&](auto B, auto LY) -> cudaError_t {
      constexpr int K3 = decltype(K)::value, BITS = decltype(B)::value, LAY = decltype(LY)::value;
      cudaError_t e = set_smem(k_sh_quantize<BITS, K3, LAY>, smem);
      if (e != cudaSuccess) return e;
      k_sh_quantize<BITS, K3, LAY><<<grid, kQG, smem, stream>>>(sh, q.n, n_pad, q.codes, bounds);
      return cudaGetLastError();
    });
  });
}

cudaError_t launch_sh_dequantize(const gs_sh_quant& q, float* sh, cudaStream_t stream) {
  const int64_t n_pad = padded(q.n);
  const unsigned grid = (unsigned)(n_pad / kQG);
  const size_t smem = sizeof(float) * q.k3 * kQPitch;
  auto bounds = reinterpret_cast<const float2*>(q.bounds);
  return with_k3(q.k3, [&](auto K) -> cudaError_t {
    return with_bits_layout(q, [&](auto B, auto LY) -> cudaError_t {
      constexpr int K3 = decltype(K)::value, BITS = decltype(B)::value, LAY = decltype(LY)::value;
      cudaError_t e = set_smem(k_sh_dequantize<BITS, K3, LAY>, smem);
      if (e != cudaSuccess) return e;
      k_sh_dequantize<BITS, K3, LAY><<<grid, kQG, smem, stream>>>(q.codes, bounds, q.n, n_pad,
                                                                  sh);
      return cudaGetLastError();
    });
  });
}

cudaError_t launch_adam_sh_quant(const gs_sh_quant& q, const float* grad, uint16_t* m,
                                 uint16_t* v, float lr, float beta1, float beta2, float eps,
                                 int64_t step, int rounding, uint64_t seed, cudaStream_t stream) {
  const int64_t n_pad = padded(q.n);
  const unsigned grid = (unsigned)(n_pad / kQG);
  const size_t smem = sizeof(float) * q.k3 * kQPitch;
  const float ibc1 = (float)(1.0 / (1.0 - pow((double)beta1, (double)step)));
  const float ibc2 = (float)(1.0 / (1.0 - pow((double)beta2, (double)step)));
  const uint64_t ctr_base = (uint64_t)step << 37;
  auto bounds = reinterpret_cast<float2*>(q.bounds);
  return with_k3(q.k3, [&](auto K) -> cudaError_t {
    return with_bits_layout(q, [&](auto B, auto LY) -> cudaError_t {
      constexpr int K3 = decltype(K)::value, BITS = decltype(B)::value, LAY = decltype(LY)::value;
      cudaError_t e = set_smem(k_adam_sh_quant<BITS, K3, LAY>, smem);
      if (e != cudaSuccess) return e;
      k_adam_sh_quant<BITS, K3, LAY><<<grid, kQG, smem, stream>>>(
          q.codes, bounds, grad, m, v, q.n, n_pad, lr, beta1, beta2, eps, ibc1, ibc2, rounding,
          seed, ctr_base);
      return cudaGetLastError();
    });
  });
}

cudaError_t launch_densify_sh_quant(const gs_sh_quant& in, const uint16_t* m_in,
                                    const uint16_t* v_in, const int8_t* decisions,
                                    const gs_sh_quant& out, uint16_t* m_out, uint16_t* v_out,
                                    uint32_t* block_counts, int64_t* n_out_dev, uint32_t* src,
                                    uint32_t* status, cudaStream_t stream) {
  cudaError_t e = launch_densify_map(decisions, (int)in.n, block_counts, out.n, n_out_dev, src,
                                     status, stream);
  if (e != cudaSuccess || out.n == 0) return e;
  const int64_t n_pad_in = padded(in.n), n_pad_out = padded(out.n);
  const unsigned grid = (unsigned)(n_pad_out / kQG);
  auto ib = reinterpret_cast<const float2*>(in.bounds);
  auto ob = reinterpret_cast<float2*>(out.bounds);
  return with_k3(in.k3, [&](auto K) -> cudaError_t {
    return with_bits_layout(in, [&](auto B, auto LY) -> cudaError_t {
      constexpr int K3 = decltype(K)::value, BITS = decltype(B)::value, LAY = decltype(LY)::value;
      k_dsq_emit<BITS, K3, LAY><<<grid, kQG, 0, stream>>>(in.codes, ib, m_in, v_in, n_pad_in,
                                                          src, n_out_dev, out.n, n_pad_out,
                                                          out.codes, ob, m_out, v_out, status);
      return cudaGetLastError();
    });
  });
}

}  // namespace gsb
