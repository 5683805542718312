// project.cu -- EWA projection of 3D Gaussians and its backward, sm_100a.
//
// Forward ("Better Gaussian Splatting in Julia", pwwt.cn sec. 3.2
// project_gaussian; lshu.cn sec. 3.2: world -> camera -> pixel with division
// by depth, 3D covariance through the Jacobian of that map): one thread per
// Gaussian, looping over the views so the parameters are read once; a block's
// SH coefficients arrive in shared memory by one TMA bulk copy issued at the
// start, overlapping the geometry. The
// geometry that ends in a discrete decision (depth key, radius, tile
// rectangle) is evaluated in double, so that the decision is the exact one up
// to double rounding; colour is evaluated in float.
//
// Backward: chain rule of the same map, float, one thread per Gaussian,
// summing the views in registers before one write of every gradient; the
// block's SH coefficients stream into shared memory (cp.async) while the
// parameters load and the view-independent part is computed.
//
// Quantised SH (the Spirula page's codes with per-256 bounds): both kernels
// read the codes where they use them and decode each one as the decoder
// does, fma(q, (max - min) / (2^b - 1), min), so colour and gradients equal
// those of the float path on the decoded coefficients bit for bit. A forward
// block of 256 Gaussians is one group of the codes.

#include <cuda_runtime.h>

#include <type_traits>

#include "gs_internal.h"

namespace gsb {
namespace {

// Real spherical harmonics on the unit sphere, index l*l + l + m, l <= 3,
// with the Condon-Shortley phase carried into the real form:
//   Y_l0 = K_l0 P_l(z);  Y_lm = sqrt2 K_l|m| P_l^|m|(z) {cos m phi, sin |m| phi}.
// Normalisation constants:
constexpr float kY0 = 0.28209479177387814f;   // 1 / (2 sqrt(pi))
constexpr float kY1 = 0.48860251190291992f;   // sqrt(3 / (4 pi))
constexpr float kY2a = 1.0925484305920792f;   // sqrt(15 / pi) / 2
constexpr float kY2b = 0.31539156525252005f;  // sqrt(5 / pi) / 4
constexpr float kY2c = 0.54627421529603959f;  // sqrt(15 / pi) / 4
constexpr float kY3a = 0.59004358992664352f;  // sqrt(35 / (2 pi)) / 4
constexpr float kY3b = 2.8906114426405538f;   // sqrt(105 / pi) / 2
constexpr float kY3c = 0.45704579946446572f;  // sqrt(21 / (2 pi)) / 4
constexpr float kY3d = 0.37317633259011546f;  // sqrt(7 / pi) / 4
constexpr float kY3e = 1.4453057213202769f;   // sqrt(105 / pi) / 4

template <int DEG>
__device__ __forceinline__ void sh_basis(float x, float y, float z, float* Y) {
  Y[0] = kY0;
  if (DEG >= 1) {
    Y[1] = -kY1 * y;
    Y[2] = kY1 * z;
    Y[3] = -kY1 * x;
  }
  if (DEG >= 2) {
    float xx = x * x, yy = y * y, zz = z * z;
    Y[4] = kY2a * x * y;
    Y[5] = -kY2a * y * z;
    Y[6] = kY2b * (3.f * zz - 1.f);
    Y[7] = -kY2a * x * z;
    Y[8] = kY2c * (xx - yy);
    if (DEG >= 3) {
      Y[9] = -kY3a * y * (3.f * xx - yy);
      Y[10] = kY3b * x * y * z;
      Y[11] = -kY3c * y * (5.f * zz - 1.f);
      Y[12] = kY3d * z * (5.f * zz - 3.f);
      Y[13] = -kY3c * x * (5.f * zz - 1.f);
      Y[14] = kY3e * z * (xx - yy);
      Y[15] = -kY3a * x * (xx - 3.f * yy);
    }
  }
}

// sum_k w_k grad Y_k: the gradient of the polynomials above with respect to
// x, y, z taken as independent variables, weighted by w (the caller projects
// onto the sphere's tangent plane, which removes the difference between
// equivalent forms on the sphere). Accumulates into (gx, gy, gz).
template <int DEG>
__device__ __forceinline__ void sh_dir_grad(float x, float y, float z, const float* w, float& gx,
                                            float& gy, float& gz) {
  if (DEG >= 1) {
    gy -= kY1 * w[1];
    gz += kY1 * w[2];
    gx -= kY1 * w[3];
  }
  if (DEG >= 2) {
    gx += kY2a * (y * w[4] - z * w[7]) + 2.f * kY2c * x * w[8];
    gy += kY2a * (x * w[4] - z * w[5]) - 2.f * kY2c * y * w[8];
    gz += 6.f * kY2b * z * w[6] - kY2a * (y * w[5] + x * w[7]);
  }
  if (DEG >= 3) {
    const float xx = x * x, yy = y * y, zz = z * z;
    const float p5 = 5.f * zz - 1.f;
    gx += -6.f * kY3a * x * y * w[9] + kY3b * y * z * w[10] - kY3c * p5 * w[13] +
          2.f * kY3e * x * z * w[14] - 3.f * kY3a * (xx - yy) * w[15];
    gy += -3.f * kY3a * (xx - yy) * w[9] + kY3b * x * z * w[10] - kY3c * p5 * w[11] -
          2.f * kY3e * y * z * w[14] + 6.f * kY3a * x * y * w[15];
    gz += kY3b * x * y * w[10] - 10.f * kY3c * y * z * w[11] + kY3d * (15.f * zz - 3.f) * w[12] -
          10.f * kY3c * x * z * w[13] + kY3e * (xx - yy) * w[14];
  }
}

// Rotation matrix of the normalised quaternion (w, x, y, z).
template <typename T>
__device__ __forceinline__ void quat_to_rot(T w, T x, T y, T z, T R[3][3]) {
  R[0][0] = T(1) - T(2) * (y * y + z * z);
  R[0][1] = T(2) * (x * y - w * z);
  R[0][2] = T(2) * (x * z + w * y);
  R[1][0] = T(2) * (x * y + w * z);
  R[1][1] = T(1) - T(2) * (x * x + z * z);
  R[1][2] = T(2) * (y * z - w * x);
  R[2][0] = T(2) * (x * z - w * y);
  R[2][1] = T(2) * (y * z + w * x);
  R[2][2] = T(1) - T(2) * (x * x + y * y);
}

__device__ __forceinline__ long long floor_tile(double a) {
  return static_cast<long long>(floor(a * (1.0 / kTile)));
}

constexpr double kHalfLog2e = 0.72134752044448170;  // log2(e) / 2
constexpr double kInvLn2 = 1.4426950408889634;      // 1 / ln 2
constexpr double kLog2_255 = 7.9943534368588578;    // log2(255)

constexpr int kProjThreads = 128;     // projection backward block
constexpr int kProjFwdThreads = 256;  // projection forward block
constexpr int kShStride = kProjThreads + 1;  // padded row: conflict-free banks
constexpr int kFwdQStride = kProjFwdThreads + 1;  // forward, decoded codes

// Stage the SH coefficients of Gaussians [i0, i0 + cnt) in shared memory,
// coefficient-major with a padded row (s[c * kShStride + local i]), by
// asynchronous 4-byte copies (cp.async) of the contiguous global block: the
// caller keeps working and calls cp_async_wait_all() + __syncthreads() before
// the reads.
template <int K3>
__device__ __forceinline__ void stage_sh_async(const float* __restrict__ sh, int64_t i0, int cnt,
                                               float* __restrict__ s) {
  const float* src = sh + i0 * K3;
  const int total = cnt * K3;
  for (int e = threadIdx.x; e < total; e += kProjThreads) {
    const int i = e / K3, c = e - i * K3;
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(&s[c * kShStride + i])),
                 "l"(src + e)
                 : "memory");
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
}

__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_group 0;" ::: "memory");
}

// Write staged values back to the contiguous global block (coalesced).
template <int K3>
__device__ __forceinline__ void unstage_sh(float* __restrict__ dst, int64_t i0, int cnt,
                                           const float* __restrict__ s) {
  float* d = dst + i0 * K3;
  const int total = cnt * K3;
  for (int e = threadIdx.x; e < total; e += kProjThreads) {
    const int i = e / K3, c = e - i * K3;
    d[e] = s[c * kShStride + i];
  }
}

// Colour from the SH coefficients of one Gaussian read straight from global
// memory (16-byte loads when the per-Gaussian block allows) at unit direction
// (x, y, z): rgb_c = max(0, sum_k Y_k sh_kc + 0.5).
template <int DEG>
__device__ __forceinline__ bool sh_colour_global(const float* __restrict__ shi, float x, float y,
                                                 float z, float rgb[3]) {
  constexpr int K = (DEG + 1) * (DEG + 1);
  float Y[16];
  sh_basis<DEG>(x, y, z, Y);
  float acc[3] = {0.5f, 0.5f, 0.5f};
  if ((K * 3) % 4 == 0) {
    const float4* s4 = reinterpret_cast<const float4*>(shi);
#pragma unroll
    for (int q = 0; q < K * 3 / 4; ++q) {
      const float4 c = __ldg(&s4[q]);
      const float cv[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int idx = 4 * q + e;
        acc[idx % 3] = fmaf(Y[idx / 3], cv[e], acc[idx % 3]);
      }
    }
  } else {
#pragma unroll
    for (int idx = 0; idx < K * 3; ++idx) acc[idx % 3] = fmaf(Y[idx / 3], __ldg(&shi[idx]), acc[idx % 3]);
  }
#pragma unroll
  for (int ch = 0; ch < 3; ++ch) rgb[ch] = fmaxf(acc[ch], 0.f);
  return isfinite(acc[0] + acc[1] + acc[2]);  // before the clamp, which drops a NaN
}

// Colour from the SH coefficients of one Gaussian staged in shared memory
// (16-byte loads), same arithmetic as sh_colour_global.
template <int DEG>
__device__ __forceinline__ bool sh_colour_smem(const float* __restrict__ shi, float x, float y,
                                               float z, float rgb[3]) {
  constexpr int K = (DEG + 1) * (DEG + 1);
  float Y[16];
  sh_basis<DEG>(x, y, z, Y);
  float acc[3] = {0.5f, 0.5f, 0.5f};
  if ((K * 3) % 4 == 0) {
    const float4* s4 = reinterpret_cast<const float4*>(shi);
#pragma unroll
    for (int q = 0; q < K * 3 / 4; ++q) {
      const float4 c = s4[q];
      const float cv[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int idx = 4 * q + e;
        acc[idx % 3] = fmaf(Y[idx / 3], cv[e], acc[idx % 3]);
      }
    }
  } else {
#pragma unroll
    for (int idx = 0; idx < K * 3; ++idx) acc[idx % 3] = fmaf(Y[idx / 3], shi[idx], acc[idx % 3]);
  }
#pragma unroll
  for (int ch = 0; ch < 3; ++ch) rgb[ch] = fmaxf(acc[ch], 0.f);
  return isfinite(acc[0] + acc[1] + acc[2]);  // before the clamp, which drops a NaN
}

// (min, step) of value j in group g, the step rounded as the decoder rounds it.
__device__ __forceinline__ float2 shq_scale(const ShQuant& q, int j, int64_t g) {
  const float2 b = __ldg(q.bounds + (int64_t)j * q.n_groups + g);
  return make_float2(b.x, __fdiv_rn(__fsub_rn(b.y, b.x), q.qmax));
}

// Colour from coefficients staged coefficient-major in shared memory
// (shi[idx * STRIDE]), same arithmetic as sh_colour_smem.
template <int DEG, int STRIDE>
__device__ __forceinline__ bool sh_colour_strided(const float* __restrict__ shi, float x, float y,
                                                  float z, float rgb[3]) {
  constexpr int K = (DEG + 1) * (DEG + 1);
  float Y[16];
  sh_basis<DEG>(x, y, z, Y);
  float acc[3] = {0.5f, 0.5f, 0.5f};
#pragma unroll
  for (int idx = 0; idx < K * 3; ++idx)
    acc[idx % 3] = fmaf(Y[idx / 3], shi[idx * STRIDE], acc[idx % 3]);
#pragma unroll
  for (int ch = 0; ch < 3; ++ch) rgb[ch] = fmaxf(acc[ch], 0.f);
  return isfinite(acc[0] + acc[1] + acc[2]);  // before the clamp, which drops a NaN
}

// The K3 decoded coefficients of Gaussian i into dst[c * STRIDE]: each
// thread its own Gaussian, so a warp's loads of one coefficient are
// consecutive codes, twelve loads in flight at a time.
template <int K3, int KIND, int STRIDE>
__device__ __forceinline__ void decode_codes(const ShQuant& q, const float2* s_qs, int64_t i,
                                             float* dst) {
  using T = typename std::conditional<KIND == kShqPlanar8, uint8_t, unsigned short>::type;
  const int64_t base = KIND == kShqPacked ? (i >> 5) * 96 + (i & 31) : i;
  const int64_t stride = KIND == kShqPacked ? (q.n_pad >> 5) * 96 : q.n_pad;
  const T* p = static_cast<const T*>(q.codes) + base;
  constexpr int kChunk = K3 < 12 ? K3 : 12;
#pragma unroll
  for (int c0 = 0; c0 < K3; c0 += kChunk) {
    float cv[kChunk];
#pragma unroll
    for (int k = 0; k < kChunk; ++k) {
      if (c0 + k < K3) cv[k] = (float)__ldg(p);
      p += stride;
    }
#pragma unroll
    for (int k = 0; k < kChunk; ++k) {
      const int c = c0 + k;
      if (c >= K3) break;
      const float2 sc = s_qs[c];
      dst[c * STRIDE] = __fmaf_rn(cv[k], sc.y, sc.x);
    }
  }
}

static_assert(kProjFwdThreads == GS_QUANT_GROUP, "a forward block is one group of the codes");

// QK: -1 float SH, else the kind of quantised codes (compile-time, so the
// decode carries no layout branches).
template <int DEG, int QK>
__global__ void __launch_bounds__(kProjFwdThreads, 3) k_project(const float4* __restrict__ means,
                                                          const float4* __restrict__ log_scales,
                                                          const float4* __restrict__ quats,
                                                          const float* __restrict__ logit,
                                                          const float* __restrict__ sh, int n,
                                                          int n_views, CamSet cams,
                                                          float4* __restrict__ records,
                                                          float4* __restrict__ bins,
                                                          int* __restrict__ radii,
                                                          uint32_t* __restrict__ status,
                                                          uint64_t wait_ns, ShQuant shq) {
  constexpr int K = (DEG + 1) * (DEG + 1);
  constexpr bool QUANT = QK >= 0;
  // the block's SH coefficients are one contiguous range: a full block with a
  // 16-byte-aligned array fetches them with one bulk copy that lands while
  // the geometry is computed
  extern __shared__ __align__(16) float s_sh[];  // [kProjFwdThreads][K * 3] (codes: [K * 3][257])
  __shared__ __align__(8) uint64_t s_bar;
  __shared__ float2 s_qs[QUANT ? 48 : 1];       // quantised: (min, step) per value
  const int64_t i0 = (int64_t)blockIdx.x * kProjFwdThreads;
  if constexpr (QUANT) {
    // the block's codes decoded at once into s_sh [K * 3][kFwdQStride], each
    // thread its own Gaussian's column (read back only by that thread)
    if (threadIdx.x < K * 3) s_qs[threadIdx.x] = shq_scale(shq, threadIdx.x, blockIdx.x);
    __syncthreads();
    if (i0 + threadIdx.x < (int64_t)n)
      decode_codes<K * 3, (QK < 0 ? 0 : QK), kFwdQStride>(shq, s_qs, i0 + threadIdx.x,
                                                         s_sh + threadIdx.x);
  }
  const bool staged = !QUANT && ((reinterpret_cast<uintptr_t>(sh) & 15) == 0) &&
                      i0 + kProjFwdThreads <= (int64_t)n;
  if (staged) {
    if (threadIdx.x == 0) {
      constexpr uint32_t bytes = kProjFwdThreads * K * 3 * sizeof(float);
      mbar_init(&s_bar, 1);
      fence_mbar_init();
      mbar_arrive_expect_tx(&s_bar, bytes);
      bulk_copy_g2s(s_sh, sh + i0 * K * 3, bytes, &s_bar);
    }
    __syncthreads();
  }
  bool sh_ready = !staged;
  const int i = blockIdx.x * kProjFwdThreads + threadIdx.x;
  if (i >= n) return;  // only in a partial block, which is not staged
  const float4 m = __ldg(&means[i]);
  const float4 ls = __ldg(&log_scales[i]);
  const float4 q = __ldg(&quats[i]);
  const float lg = __ldg(&logit[i]);
  // a non-finite parameter or a zero quaternion culls the Gaussian in every
  // view and marks its depth key
  const bool finite_in = isfinite(m.x) && isfinite(m.y) && isfinite(m.z) && isfinite(ls.x) &&
                         isfinite(ls.y) && isfinite(ls.z) && isfinite(q.x) && isfinite(q.y) &&
                         isfinite(q.z) && isfinite(q.w) && isfinite(lg) &&
                         (q.x != 0.f || q.y != 0.f || q.z != 0.f || q.w != 0.f);

  // view-independent: M = R diag(exp(s)) in double
  double qw = q.x, qx = q.y, qy = q.z, qz = q.w;
  double qinv = 1.0 / sqrt(qw * qw + qx * qx + qy * qy + qz * qz);
  qw *= qinv; qx *= qinv; qy *= qinv; qz *= qinv;
  double R[3][3];
  quat_to_rot<double>(qw, qx, qy, qz, R);
  const double s[3] = {exp((double)ls.x), exp((double)ls.y), exp((double)ls.z)};
  double M[3][3];
#pragma unroll
  for (int a = 0; a < 3; ++a)
#pragma unroll
    for (int b = 0; b < 3; ++b) M[a][b] = R[a][b] * s[b];
  const double opac_d = 1.0 / (1.0 + exp(-(double)lg));
  // alpha >= 1/255 needs q <= Q = 2 ln(255 o); Q <= 0: the splat never counts
  const double Qa = 2.0 * log(255.0 * opac_d);
  const float* shi = QUANT ? nullptr : sh + (size_t)i * K * 3;

  const Grid g = grid_of(cams.c[0]);
  for (int v = 0; v < n_views; ++v) {
    const gs_camera& c = cams.c[v];
    const double mx = m.x, my = m.y, mz = m.z;
    const double W[3][3] = {{c.viewmat[0], c.viewmat[1], c.viewmat[2]},
                            {c.viewmat[4], c.viewmat[5], c.viewmat[6]},
                            {c.viewmat[8], c.viewmat[9], c.viewmat[10]}};
    const double tx = fma(W[0][0], mx, fma(W[0][1], my, fma(W[0][2], mz, (double)c.viewmat[3])));
    const double ty = fma(W[1][0], mx, fma(W[1][1], my, fma(W[1][2], mz, (double)c.viewmat[7])));
    const double tz = fma(W[2][0], mx, fma(W[2][1], my, fma(W[2][2], mz, (double)c.viewmat[11])));
    // sort key: float32 depth as a fixed chain of correctly rounded fmas of
    // the float inputs, so it is one well-defined float; it also decides the
    // near-plane cull
    const float key = __fmaf_rn(c.viewmat[8], m.x,
                                __fmaf_rn(c.viewmat[9], m.y, __fmaf_rn(c.viewmat[10], m.z, c.viewmat[11])));
    float rec[GS_RECORD_FLOATS];
#pragma unroll
    for (int k = 0; k < GS_RECORD_FLOATS; ++k) rec[k] = 0.f;
    int radius = 0;
    bool nonfinite = !finite_in;
    bool ok = finite_in && key >= (float)kNear;
    long long x0 = 1, x1 = 0, y0 = 1, y1 = 0;
    if (ok) {
      const double iz = 1.0 / tz;
      const double fx = c.fx, fy = c.fy;
      const double a0 = fx * iz, a2 = -fx * tx * iz * iz;
      const double b1 = fy * iz, b2 = -fy * ty * iz * iz;
      // rows of T = J W
      double T0[3], T1[3];
#pragma unroll
      for (int j = 0; j < 3; ++j) {
        T0[j] = a0 * W[0][j] + a2 * W[2][j];
        T1[j] = b1 * W[1][j] + b2 * W[2][j];
      }
      // V = T M, cov2d = V V^T + 0.3 I
      double V0[3], V1[3];
#pragma unroll
      for (int k = 0; k < 3; ++k) {
        V0[k] = T0[0] * M[0][k] + T0[1] * M[1][k] + T0[2] * M[2][k];
        V1[k] = T1[0] * M[0][k] + T1[1] * M[1][k] + T1[2] * M[2][k];
      }
      const double A = V0[0] * V0[0] + V0[1] * V0[1] + V0[2] * V0[2] + kLowPass;
      const double B = V0[0] * V1[0] + V0[1] * V1[1] + V0[2] * V1[2];
      const double C = V1[0] * V1[0] + V1[1] * V1[1] + V1[2] * V1[2] + kLowPass;
      const double det = A * C - B * B;
      ok = det > 0.0;
      if (ok) {
        const double idet = 1.0 / det;
        const double mid = 0.5 * (A + C);
        const double rr = sqrt(0.25 * (A - C) * (A - C) + B * B);
        const double lam = mid + rr;
        double rd = ceil(3.0 * sqrt(lam));
        if (!(rd <= (double)kMaxRadius)) rd = (double)kMaxRadius;
        radius = (int)rd;
        const double u = fx * tx * iz + (double)c.cx;
        const double vv = fy * ty * iz + (double)c.cy;
        const long long fx0 = floor_tile(u - radius), fx1 = floor_tile(u + radius);
        const long long fy0 = floor_tile(vv - radius), fy1 = floor_tile(vv + radius);
        x0 = fx0 < 0 ? 0 : fx0;
        x1 = fx1 > g.tiles_x - 1 ? g.tiles_x - 1 : fx1;
        y0 = fy0 < 0 ? 0 : fy0;
        y1 = fy1 > g.tiles_y - 1 ? g.tiles_y - 1 : fy1;
        ok = (x0 <= x1) && (y0 <= y1);
        if (ok) {
          // evaluation form: q' = (log2(e)/2) d^T cov^-1 d = (w1 . d)^2 + (w2 . d)^2
          // with w_i = sqrt(log2(e) / (2 lambda_i)) e_i over the unit eigenvectors
          // e_i of cov2d (lambda_2 = det / lambda_1 without cancellation; e_1 from
          // the row of cov2d - lambda_1 I that has no cancellation)
          const double h = 0.5 * (A - C);
          double e1x = h >= 0.0 ? h + rr : B, e1y = h >= 0.0 ? B : rr - h;
          const double en = sqrt(e1x * e1x + e1y * e1y);
          if (en > 0.0) {
            e1x /= en;
            e1y /= en;
          } else {  // isotropic: any orthonormal pair
            e1x = 1.0;
            e1y = 0.0;
          }
          const double k1 = sqrt(kHalfLog2e / lam), k2 = sqrt(kHalfLog2e * lam * idet);
          const float w1x = (float)(k1 * e1x), w1y = (float)(k1 * e1y);
          const float w2x = (float)(-k2 * e1y), w2y = (float)(k2 * e1x);
          // the mean as a float plus the float rows applied to its remainder
          const float uh = (float)u, vh = (float)vv;
          const double ulo = u - (double)uh, vlo = vv - (double)vh;
          rec[R_U] = uh;
          rec[R_V] = vh;
          rec[R_W1X] = w1x;
          rec[R_W1Y] = w1y;
          rec[R_C1] = (float)(-((double)w1x * ulo + (double)w1y * vlo));
          rec[R_W2X] = w2x;
          rec[R_W2Y] = w2y;
          rec[R_C2] = (float)(-((double)w2x * ulo + (double)w2y * vlo));
          // -log2(255 o), o = 1 / (1 + e^-logit): log2(255) - log2(1 + e^-logit)
          rec[R_NLO] = (float)(log1p(exp(-(double)lg)) * kInvLn2 - kLog2_255);
          rec[R_OPAC] = (float)opac_d;
          // half-widths of the box around {q <= Q}, with Q padded (0.2 % +
          // 1e-4) well beyond the float rounding of the rasteriser's alpha
          // test, so the box holds every pixel that test can accept
          const double Qp = Qa + 2e-3 * fabs(Qa) + 1e-4;
          if (Qp > 0.0) {
            rec[R_HX] = (float)(sqrt(Qp * A) + 1e-2);
            rec[R_HY] = (float)(sqrt(Qp * C) + 1e-2);
          } else {
            rec[R_HX] = -1.f;
            rec[R_HY] = -1.f;
          }
          // colour: SH at the direction from the camera centre to the mean
          float dxv = m.x - c.campos[0], dyv = m.y - c.campos[1], dzv = m.z - c.campos[2];
          float inv = rsqrtf(dxv * dxv + dyv * dyv + dzv * dzv);
          float rgb[3];
          bool colour_finite;
          if (staged && !sh_ready) sh_ready = mbar_wait_bounded(&s_bar, 0u, wait_ns, status);
          if constexpr (QUANT) {
            colour_finite = sh_colour_strided<DEG, kFwdQStride>(s_sh + threadIdx.x, dxv * inv,
                                                                 dyv * inv, dzv * inv, rgb);
          } else if (sh_ready && staged) {
            colour_finite = sh_colour_smem<DEG>(s_sh + (size_t)threadIdx.x * K * 3, dxv * inv,
                                                dyv * inv, dzv * inv, rgb);
          } else {  // not staged, or the staging copy did not land in time
            colour_finite = sh_colour_global<DEG>(shi, dxv * inv, dyv * inv, dzv * inv, rgb);
          }
          rec[R_R] = rgb[0];
          rec[R_G] = rgb[1];
          rec[R_B] = rgb[2];
          // a non-finite SH coefficient shows in the colour
          if (!colour_finite) {
            ok = false;
            nonfinite = true;
          }
        }
      }
    }
    if (!ok) {
      radius = 0;
      x0 = 1; x1 = 0; y0 = 1; y1 = 0;
#pragma unroll
      for (int k = 0; k < GS_RECORD_FLOATS; ++k) rec[k] = 0.f;
      rec[R_HX] = -1.f;
      rec[R_HY] = -1.f;
    }
    const size_t r = (size_t)v * n + i;
    float4* out = records + r * (GS_RECORD_FLOATS / 4);
#pragma unroll
    for (int k = 0; k < GS_RECORD_FLOATS / 4; ++k)
      out[k] = make_float4(rec[4 * k], rec[4 * k + 1], rec[4 * k + 2], rec[4 * k + 3]);
    bins[r] = make_float4(nonfinite ? __uint_as_float(kNonfiniteKeyBits) : key,
                          __uint_as_float((uint32_t)x0 | ((uint32_t)x1 << 16)),
                          __uint_as_float((uint32_t)y0 | ((uint32_t)y1 << 16)), 0.f);
    radii[r] = radius;
  }
  // a staged copy lands before the block exits, even if no view needed it
  // (after a wait that gave up, this waits once more for it)
  if (staged && !sh_ready) mbar_wait_bounded(&s_bar, 0u, wait_ns, status);
}

// Backward of k_project for the raw parameters, summing every view in which
// the Gaussian was visible (radius > 0).
// SH coefficients come in, and SH gradients go out, through shared memory
// (coefficient-major, coalesced global traffic); the SH gradients are summed
// over views in shared memory rather than in registers. With ALIAS (one view)
// the gradients overwrite the staged coefficients slot by slot.
// With FUSE the gradients are not written: the Adam step (adam_one, the
// update of the Adam kernel) is applied to the parameters in place and the
// densification statistics are accumulated from the same screen-space
// gradients (densify_norm, as the statistics kernel), so the fused tail gives
// what the three separate calls give, bit for bit.
template <int DEG, bool ALIAS, bool QUANT, bool FUSE>
__global__ void __launch_bounds__(kProjThreads, 6) k_project_bwd(
    const float4* __restrict__ means, const float4* __restrict__ log_scales,
    const float4* __restrict__ quats, const float* __restrict__ logit,
    const float* __restrict__ sh, const float4* __restrict__ grad2d,
    const int* __restrict__ radii, int n, int n_views, CamSet cams, float4* __restrict__ g_means,
    float4* __restrict__ g_log_scales, float4* __restrict__ g_quats, float* __restrict__ g_logit,
    float* __restrict__ g_sh, ShQuant shq, AdamTail tail) {
  constexpr int K = (DEG + 1) * (DEG + 1);
  constexpr int K3 = K * 3;
  extern __shared__ float s_pb[];
  float* s_coef = s_pb;                                 // [K3][kShStride]
  float* s_dsh = ALIAS ? s_pb : s_pb + K3 * kShStride;  // [K3][kShStride]
  const int64_t i0 = (int64_t)blockIdx.x * kProjThreads;
  const int cnt = (int)min((int64_t)kProjThreads, (int64_t)n - i0);
  if constexpr (QUANT) {
    // decoded into the same coefficient-major slots (coalesced code reads)
    __shared__ float2 s_qs[K3];
    if (threadIdx.x < K3) s_qs[threadIdx.x] = shq_scale(shq, threadIdx.x, i0 / GS_QUANT_GROUP);
    __syncthreads();
    if ((int)threadIdx.x < cnt) {
      const int64_t i = i0 + threadIdx.x;
      float* dst = s_coef + threadIdx.x;
      if (shq.kind == kShqPlanar8)
        decode_codes<K3, kShqPlanar8, kShStride>(shq, s_qs, i, dst);
      else if (shq.kind == kShqPlanar16)
        decode_codes<K3, kShqPlanar16, kShStride>(shq, s_qs, i, dst);
      else
        decode_codes<K3, kShqPacked, kShStride>(shq, s_qs, i, dst);
    }
  } else {
    // the coefficients stream into shared memory while the parameters load
    // and the view-independent part is computed
    stage_sh_async<K3>(sh, i0, cnt, s_coef);
  }
  if (!ALIAS) {
#pragma unroll
    for (int c = 0; c < K3; ++c) s_dsh[c * kShStride + threadIdx.x] = 0.f;
  }
  const int i = (int)i0 + threadIdx.x;
  const bool live = i < n;
  const int il = live ? i : (int)i0;  // a dead thread computes on a valid index, writes nothing
  // fused: the parameters are read where this thread later writes them
  const float4 m = FUSE ? tail.p_means[il] : __ldg(&means[il]);
  const float4 ls = FUSE ? tail.p_log_scales[il] : __ldg(&log_scales[il]);
  const float4 q = FUSE ? tail.p_quats[il] : __ldg(&quats[il]);
  const float lg = FUSE ? tail.p_logit[il] : __ldg(&logit[il]);

  const float qn2 = q.x * q.x + q.y * q.y + q.z * q.z + q.w * q.w;
  const float qinv = rsqrtf(qn2);
  const float qw = q.x * qinv, qx = q.y * qinv, qy = q.z * qinv, qz = q.w * qinv;
  float R[3][3];
  quat_to_rot<float>(qw, qx, qy, qz, R);
  const float s[3] = {__expf(ls.x), __expf(ls.y), __expf(ls.z)};
  float M[3][3];
#pragma unroll
  for (int a = 0; a < 3; ++a)
#pragma unroll
    for (int b = 0; b < 3; ++b) M[a][b] = R[a][b] * s[b];
  const float opac = 1.f / (1.f + __expf(-lg));

  float dM[3][3] = {{0.f, 0.f, 0.f}, {0.f, 0.f, 0.f}, {0.f, 0.f, 0.f}};
  float dmu[3] = {0.f, 0.f, 0.f};
  float dopac = 0.f;
  const float* cf_t = s_coef + threadIdx.x;
  float* dsh_t = s_dsh + threadIdx.x;
  cp_async_wait_all();
  __syncthreads();
  float st_plain = 0.f, st_abs = 0.f;  // fused densification statistics
  int st_cnt = 0;
  if constexpr (FUSE) {
    // the moments this block updates at the end start towards L2 now, so
    // their loads there overlap the chain rule below
    // (one request per 128-byte line: every 8th lane for the float4 arrays,
    // the first lane for the float ones)
    if (live && (lane_of_thread() & 7) == 0) {
      prefetch_l2(tail.m_means + i);
      prefetch_l2(tail.v_means + i);
      prefetch_l2(tail.m_log_scales + i);
      prefetch_l2(tail.v_log_scales + i);
      prefetch_l2(tail.m_quats + i);
      prefetch_l2(tail.v_quats + i);
      if (lane_of_thread() == 0) {
        prefetch_l2(tail.m_logit + i);
        prefetch_l2(tail.v_logit + i);
      }
    }
    const int64_t sb = i0 * K3;
    const int lines = (cnt * K3 + 31) / 32;  // 128-byte lines of the block's SH range
    for (int l = threadIdx.x; l < lines; l += kProjThreads) {
      prefetch_l2(tail.m_sh + sb + 32 * l);
      prefetch_l2(tail.v_sh + sb + 32 * l);
      prefetch_l2(tail.p_sh + sb + 32 * l);
    }
  }
  if (live) {
  bool touched = false;
  for (int v = 0; v < n_views; ++v) {
    if (radii[(size_t)v * n + i] <= 0) continue;
    touched = true;
    const float4* G4 = grad2d + ((size_t)v * n + i) * 3;
    const float4 ga = G4[0], gb = G4[1], gc = G4[2];
    const float G[9] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w, gc.x};
    if (FUSE) {
      st_plain += densify_norm(ga.x, ga.y);
      st_abs += gc.y;
      ++st_cnt;
    }
    const gs_camera& c = cams.c[v];
    const float W[3][3] = {{c.viewmat[0], c.viewmat[1], c.viewmat[2]},
                           {c.viewmat[4], c.viewmat[5], c.viewmat[6]},
                           {c.viewmat[8], c.viewmat[9], c.viewmat[10]}};
    const float tx = W[0][0] * m.x + W[0][1] * m.y + W[0][2] * m.z + c.viewmat[3];
    const float ty = W[1][0] * m.x + W[1][1] * m.y + W[1][2] * m.z + c.viewmat[7];
    const float tz = W[2][0] * m.x + W[2][1] * m.y + W[2][2] * m.z + c.viewmat[11];
    const float iz = 1.f / tz, iz2 = iz * iz;
    const float fx = c.fx, fy = c.fy;
    const float a0 = fx * iz, a2 = -fx * tx * iz2, b1 = fy * iz, b2 = -fy * ty * iz2;
    float T0[3], T1[3];
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      T0[j] = a0 * W[0][j] + a2 * W[2][j];
      T1[j] = b1 * W[1][j] + b2 * W[2][j];
    }
    float V0[3], V1[3];
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      V0[k] = T0[0] * M[0][k] + T0[1] * M[1][k] + T0[2] * M[2][k];
      V1[k] = T1[0] * M[0][k] + T1[1] * M[1][k] + T1[2] * M[2][k];
    }
    const float n0 = V0[0] * V0[0] + V0[1] * V0[1] + V0[2] * V0[2];
    const float n1 = V1[0] * V1[0] + V1[1] * V1[1] + V1[2] * V1[2];
    const float A = n0 + 0.3f;
    const float B = V0[0] * V1[0] + V0[1] * V1[1] + V0[2] * V1[2];
    const float C = n1 + 0.3f;
    // det = (A-0.3)(C-0.3) - B^2 + 0.3 (A + C - 0.6) + 0.09, with the first
    // part written as |V0 x V1|^2 (Lagrange's identity) to avoid cancellation
    const float cx_ = V0[1] * V1[2] - V0[2] * V1[1];
    const float cy_ = V0[2] * V1[0] - V0[0] * V1[2];
    const float cz_ = V0[0] * V1[1] - V0[1] * V1[0];
    const float det = cx_ * cx_ + cy_ * cy_ + cz_ * cz_ + 0.3f * (n0 + n1) + 0.09f;
    const float id2 = 1.f / (det * det);
    // conic (a, b, c) = (C, -B, A) / det
    const float dA = (-C * C * G[G_CA] + B * C * G[G_CB] - B * B * G[G_CC]) * id2;
    const float dB = (2.f * B * C * G[G_CA] - (A * C + B * B) * G[G_CB] + 2.f * A * B * G[G_CC]) * id2;
    const float dC = (-B * B * G[G_CA] + A * B * G[G_CB] - A * A * G[G_CC]) * id2;
    float dV0[3], dV1[3];
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      dV0[k] = 2.f * dA * V0[k] + dB * V1[k];
      dV1[k] = dB * V0[k] + 2.f * dC * V1[k];
    }
    float dT0[3], dT1[3];
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      dT0[j] = dV0[0] * M[j][0] + dV0[1] * M[j][1] + dV0[2] * M[j][2];
      dT1[j] = dV1[0] * M[j][0] + dV1[1] * M[j][1] + dV1[2] * M[j][2];
#pragma unroll
      for (int k = 0; k < 3; ++k) dM[j][k] += T0[j] * dV0[k] + T1[j] * dV1[k];
    }
    const float da0 = dT0[0] * W[0][0] + dT0[1] * W[0][1] + dT0[2] * W[0][2];
    const float da2 = dT0[0] * W[2][0] + dT0[1] * W[2][1] + dT0[2] * W[2][2];
    const float db1 = dT1[0] * W[1][0] + dT1[1] * W[1][1] + dT1[2] * W[1][2];
    const float db2 = dT1[0] * W[2][0] + dT1[1] * W[2][1] + dT1[2] * W[2][2];
    const float gu = G[G_U], gv = G[G_V];
    const float dtx = gu * fx * iz - da2 * fx * iz2;
    const float dty = gv * fy * iz - db2 * fy * iz2;
    const float dtz = -gu * fx * tx * iz2 - gv * fy * ty * iz2 - da0 * fx * iz2 - db1 * fy * iz2 +
                      2.f * da2 * fx * tx * iz2 * iz + 2.f * db2 * fy * ty * iz2 * iz;
#pragma unroll
    for (int j = 0; j < 3; ++j) dmu[j] += W[0][j] * dtx + W[1][j] * dty + W[2][j] * dtz;
    dopac += G[G_OPAC];

    // colour: rgb_c = max(0, sum_k Y_k(d) sh_kc + 0.5), d = normalize(mu - campos)
    const float wx = m.x - c.campos[0], wy = m.y - c.campos[1], wz = m.z - c.campos[2];
    const float winv = rsqrtf(wx * wx + wy * wy + wz * wz);
    const float dx = wx * winv, dy = wy * winv, dz = wz * winv;
    float Y[16], wk[16];
    sh_basis<DEG>(dx, dy, dz, Y);
#pragma unroll
    for (int k = 0; k < K; ++k) wk[k] = 0.f;
#pragma unroll
    for (int ch = 0; ch < 3; ++ch) {
      float raw = 0.5f;
#pragma unroll
      for (int k = 0; k < K; ++k) raw = fmaf(Y[k], cf_t[(k * 3 + ch) * kShStride], raw);
      // a clamped channel passes no gradient; with one view the gradient slot
      // is the coefficient's own (read above), written once
      const float gcol = raw > 0.f ? G[G_R + ch] : 0.f;
#pragma unroll
      for (int k = 0; k < K; ++k) {
        const float cf = cf_t[(k * 3 + ch) * kShStride];
        if (ALIAS)
          dsh_t[(k * 3 + ch) * kShStride] = Y[k] * gcol;
        else
          dsh_t[(k * 3 + ch) * kShStride] += Y[k] * gcol;
        wk[k] = fmaf(gcol, cf, wk[k]);
      }
    }
    float gdx = 0.f, gdy = 0.f, gdz = 0.f;
    sh_dir_grad<DEG>(dx, dy, dz, wk, gdx, gdy, gdz);
    // through d = w / |w|: (I - d d^T) / |w|
    const float dd = gdx * dx + gdy * dy + gdz * dz;
    dmu[0] += (gdx - dx * dd) * winv;
    dmu[1] += (gdy - dy * dd) * winv;
    dmu[2] += (gdz - dz * dd) * winv;
  }

  if (ALIAS && !touched) {  // no view wrote this Gaussian's slots
#pragma unroll
    for (int c = 0; c < K3; ++c) dsh_t[c * kShStride] = 0.f;
  }

  // M = R diag(s): dL/ds_k = sum_j dM_jk R_jk, dL/dR_jk = dM_jk s_k
  float dls[3];
#pragma unroll
  for (int k = 0; k < 3; ++k)
    dls[k] = (dM[0][k] * R[0][k] + dM[1][k] * R[1][k] + dM[2][k] * R[2][k]) * s[k];
  float dR[3][3];
#pragma unroll
  for (int j = 0; j < 3; ++j)
#pragma unroll
    for (int k = 0; k < 3; ++k) dR[j][k] = dM[j][k] * s[k];
  // rotation matrix entries as functions of the unit quaternion (w, x, y, z)
  float dqw = 2.f * (-qz * dR[0][1] + qy * dR[0][2] + qz * dR[1][0] - qx * dR[1][2] -
                     qy * dR[2][0] + qx * dR[2][1]);
  float dqx = 2.f * (qy * dR[0][1] + qz * dR[0][2] + qy * dR[1][0] - qw * dR[1][2] +
                     qz * dR[2][0] + qw * dR[2][1]) -
              4.f * qx * (dR[1][1] + dR[2][2]);
  float dqy = 2.f * (qx * dR[0][1] + qw * dR[0][2] + qx * dR[1][0] + qz * dR[1][2] -
                     qw * dR[2][0] + qz * dR[2][1]) -
              4.f * qy * (dR[0][0] + dR[2][2]);
  float dqz = 2.f * (-qw * dR[0][1] + qx * dR[0][2] + qw * dR[1][0] + qy * dR[1][2] +
                     qx * dR[2][0] + qy * dR[2][1]) -
              4.f * qz * (dR[0][0] + dR[1][1]);
  // through the normalisation q_hat = q / |q|
  const float proj = dqw * qw + dqx * qx + dqy * qy + dqz * qz;
  dqw = (dqw - qw * proj) * qinv;
  dqx = (dqx - qx * proj) * qinv;
  dqy = (dqy - qy * proj) * qinv;
  dqz = (dqz - qz * proj) * qinv;

  if constexpr (FUSE) {
    const float b1 = tail.b1, b2 = tail.b2, eps = tail.eps, c1 = tail.ibc1, c2 = tail.ibc2;
    auto step4 = [&](float4 p, float4 g, float4* P, float4* Mv, float4* Vv, float lr) {
      float4 mm = __ldcs(Mv + i), vv = __ldcs(Vv + i);
      adam_one(p.x, g.x, mm.x, vv.x, lr, b1, b2, eps, c1, c2);
      adam_one(p.y, g.y, mm.y, vv.y, lr, b1, b2, eps, c1, c2);
      adam_one(p.z, g.z, mm.z, vv.z, lr, b1, b2, eps, c1, c2);
      adam_one(p.w, g.w, mm.w, vv.w, lr, b1, b2, eps, c1, c2);
      __stcs(P + i, p);
      __stcs(Mv + i, mm);
      __stcs(Vv + i, vv);
    };
    step4(m, make_float4(dmu[0], dmu[1], dmu[2], 0.f), tail.p_means, tail.m_means, tail.v_means,
          tail.lr[0]);
    step4(ls, make_float4(dls[0], dls[1], dls[2], 0.f), tail.p_log_scales, tail.m_log_scales,
          tail.v_log_scales, tail.lr[1]);
    step4(q, make_float4(dqw, dqx, dqy, dqz), tail.p_quats, tail.m_quats, tail.v_quats,
          tail.lr[2]);
    float pl = lg, ml = tail.m_logit[i], vl = tail.v_logit[i];
    adam_one(pl, dopac * opac * (1.f - opac), ml, vl, tail.lr[3], b1, b2, eps, c1, c2);
    tail.p_logit[i] = pl;
    tail.m_logit[i] = ml;
    tail.v_logit[i] = vl;
    if (tail.accum_plain && st_cnt) {
      tail.accum_plain[i] += st_plain;
      tail.accum_abs[i] += st_abs;
      tail.denom[i] += st_cnt;
    }
  } else {
    g_means[i] = make_float4(dmu[0], dmu[1], dmu[2], 0.f);
    g_log_scales[i] = make_float4(dls[0], dls[1], dls[2], 0.f);
    g_quats[i] = make_float4(dqw, dqx, dqy, dqz);
    g_logit[i] = dopac * opac * (1.f - opac);
  }
  }
  __syncthreads();
  if constexpr (FUSE) {
    // the block's SH coefficients and their moments: one contiguous range,
    // moved as float4 (16-byte aligned: the block starts at a multiple of
    // 128 Gaussians) with four vectors of each array in flight per thread;
    // every float is read and written once, so the accesses stream past L2
    const int64_t base = i0 * K3;
    const int total = cnt * K3;
    const int total4 = total >> 2;
    const float lr = tail.lr[4];
    float4* P4 = reinterpret_cast<float4*>(tail.p_sh + base);
    float4* M4 = reinterpret_cast<float4*>(tail.m_sh + base);
    float4* V4 = reinterpret_cast<float4*>(tail.v_sh + base);
    auto grad_at = [&](int e) {
      const int t = e / K3, c = e - t * K3;
      return s_dsh[c * kShStride + t];
    };
#pragma unroll 4
    for (int e4 = threadIdx.x; e4 < total4; e4 += kProjThreads) {
      float4 p = __ldcs(P4 + e4), mm = __ldcs(M4 + e4), vv = __ldcs(V4 + e4);
      const int e = 4 * e4;
      adam_one(p.x, grad_at(e), mm.x, vv.x, lr, tail.b1, tail.b2, tail.eps, tail.ibc1, tail.ibc2);
      adam_one(p.y, grad_at(e + 1), mm.y, vv.y, lr, tail.b1, tail.b2, tail.eps, tail.ibc1,
               tail.ibc2);
      adam_one(p.z, grad_at(e + 2), mm.z, vv.z, lr, tail.b1, tail.b2, tail.eps, tail.ibc1,
               tail.ibc2);
      adam_one(p.w, grad_at(e + 3), mm.w, vv.w, lr, tail.b1, tail.b2, tail.eps, tail.ibc1,
               tail.ibc2);
      __stcs(P4 + e4, p);
      __stcs(M4 + e4, mm);
      __stcs(V4 + e4, vv);
    }
    for (int e = 4 * total4 + threadIdx.x; e < total; e += kProjThreads) {  // ragged end
      float p = tail.p_sh[base + e], mm = tail.m_sh[base + e], vv = tail.v_sh[base + e];
      adam_one(p, grad_at(e), mm, vv, lr, tail.b1, tail.b2, tail.eps, tail.ibc1, tail.ibc2);
      tail.p_sh[base + e] = p;
      tail.m_sh[base + e] = mm;
      tail.v_sh[base + e] = vv;
    }
  } else {
    unstage_sh<K3>(g_sh, i0, cnt, s_dsh);
  }
}

}  // namespace

cudaError_t launch_project(const gs_params& p, const CamSet& cams, int n_views, float* records,
                           float* bins, int* radii, uint32_t* status, const WaitCfg& wc,
                           cudaStream_t stream) {
  const int n = (int)p.n;
  if (n == 0) return cudaSuccess;
  const int threads = kProjFwdThreads;
  const int blocks = (n + threads - 1) / threads;
  auto m = reinterpret_cast<const float4*>(p.means);
  auto s = reinterpret_cast<const float4*>(p.log_scales);
  auto q = reinterpret_cast<const float4*>(p.quats);
  auto r = reinterpret_cast<float4*>(records);
  auto b = reinterpret_cast<float4*>(bins);
  const ShQuant shq = shq_of(p.sh_quant);
#define GS_PFWD1(D, Q)                                                                       \
  {                                                                                          \
    const int smem = (Q >= 0 ? kFwdQStride : threads) * 3 * (D + 1) * (D + 1) * (int)sizeof(float); \
    cudaFuncSetAttribute(k_project<D, Q>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem); \
    k_project<D, Q><<<blocks, threads, smem, stream>>>(m, s, q, p.opacity_logit, p.sh, n,     \
                                                       n_views, cams, r, b, radii, status,    \
                                                       wc.limit_ns, shq);                     \
  }
#define GS_PFWD(D)                                 \
  if (!p.sh_quant) {                               \
    GS_PFWD1(D, -1);                               \
  } else if (shq.kind == kShqPlanar8) {            \
    GS_PFWD1(D, kShqPlanar8);                      \
  } else if (shq.kind == kShqPlanar16) {           \
    GS_PFWD1(D, kShqPlanar16);                     \
  } else {                                         \
    GS_PFWD1(D, kShqPacked);                       \
  }
  switch (p.sh_degree) {
    case 0: GS_PFWD(0); break;
    case 1: GS_PFWD(1); break;
    case 2: GS_PFWD(2); break;
    default: GS_PFWD(3); break;
  }
#undef GS_PFWD
#undef GS_PFWD1
  return cudaGetLastError();
}

cudaError_t launch_project_bwd(const gs_params& p, const CamSet& cams, int n_views,
                               const float* grad2d, const int* radii, const gs_grads& g,
                               cudaStream_t stream) {
  const int n = (int)p.n;
  if (n == 0) return cudaSuccess;
  const int threads = kProjThreads;
  const int blocks = (n + threads - 1) / threads;
  const int K3 = 3 * (p.sh_degree + 1) * (p.sh_degree + 1);
  const bool alias = n_views == 1;
  const size_t smem = (size_t)(alias ? 1 : 2) * K3 * kShStride * sizeof(float);
  const ShQuant shq = shq_of(p.sh_quant);
  auto m = reinterpret_cast<const float4*>(p.means);
  auto s = reinterpret_cast<const float4*>(p.log_scales);
  auto q = reinterpret_cast<const float4*>(p.quats);
  auto g2 = reinterpret_cast<const float4*>(grad2d);
  auto gm = reinterpret_cast<float4*>(g.means);
  auto gs = reinterpret_cast<float4*>(g.log_scales);
  auto gq = reinterpret_cast<float4*>(g.quats);
#define GS_PBWD2(D, AL, Q)                                                                    \
  cudaFuncSetAttribute(k_project_bwd<D, AL, Q, false>,                                           \
                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);                  \
  k_project_bwd<D, AL, Q, false><<<blocks, threads, smem, stream>>>(                             \
      m, s, q, p.opacity_logit, p.sh, g2, radii, n, n_views, cams, gm, gs, gq, g.opacity_logit,  \
      g.sh, shq, AdamTail{})
#define GS_PBWD1(D, AL)       \
  if (p.sh_quant) {           \
    GS_PBWD2(D, AL, true);    \
  } else {                    \
    GS_PBWD2(D, AL, false);   \
  }
#define GS_PBWD(D)            \
  if (alias) {                \
    GS_PBWD1(D, true);        \
  } else {                    \
    GS_PBWD1(D, false);       \
  }
  switch (p.sh_degree) {
    case 0: GS_PBWD(0); break;
    case 1: GS_PBWD(1); break;
    case 2: GS_PBWD(2); break;
    default: GS_PBWD(3); break;
  }
#undef GS_PBWD
#undef GS_PBWD1
#undef GS_PBWD2
  return cudaGetLastError();
}

cudaError_t launch_project_bwd_adam(const gs_params& p, const CamSet& cams, int n_views,
                                    const float* grad2d, const int* radii, const AdamTail& t,
                                    cudaStream_t stream) {
  const int n = (int)p.n;
  if (n == 0) return cudaSuccess;
  const int threads = kProjThreads;
  const int blocks = (n + threads - 1) / threads;
  const int K3 = 3 * (p.sh_degree + 1) * (p.sh_degree + 1);
  const bool alias = n_views == 1;
  const size_t smem = (size_t)(alias ? 1 : 2) * K3 * kShStride * sizeof(float);
  auto g2 = reinterpret_cast<const float4*>(grad2d);
  // the parameters are read through the tail's pointers (they are updated in place)
#define GS_PBWDF1(D, AL)                                                                        \
  cudaFuncSetAttribute(k_project_bwd<D, AL, false, true>,                                         \
                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);                   \
  k_project_bwd<D, AL, false, true><<<blocks, threads, smem, stream>>>(                           \
      t.p_means, t.p_log_scales, t.p_quats, t.p_logit, t.p_sh, g2, radii, n, n_views, cams,      \
      nullptr, nullptr, nullptr, nullptr, nullptr, ShQuant{}, t)
#define GS_PBWDF(D)           \
  if (alias) {                \
    GS_PBWDF1(D, true);       \
  } else {                    \
    GS_PBWDF1(D, false);      \
  }
  switch (p.sh_degree) {
    case 0: GS_PBWDF(0); break;
    case 1: GS_PBWDF(1); break;
    case 2: GS_PBWDF(2); break;
    default: GS_PBWDF(3); break;
  }
#undef GS_PBWDF
#undef GS_PBWDF1
  return cudaGetLastError();
}

}  // namespace gsb
