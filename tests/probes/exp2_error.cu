// exp2_error.cu -- exhaustive relative error of the float exp2 the rasteriser
// uses (exp2f under --use_fast_math, the SFU's approximate exp2), over every
// float a in [lo, hi], against exp2 taken in double. Prints the largest
// relative error and the argument where it occurs. A test helper: the parity
// tests hold the kernel's alpha to a bound that includes this error.
#include <cstdio>
#include <cstdint>
#include <cstring>
#include <cuda_runtime.h>

__global__ void k_exp2_error(uint32_t first_bits, uint32_t count, unsigned long long* worst) {
  const uint32_t stride = gridDim.x * blockDim.x;
  double local = 0.0;
  uint32_t arg = 0;
  for (uint32_t i = blockIdx.x * blockDim.x + threadIdx.x; i < count; i += stride) {
    const float a = __uint_as_float(first_bits + i);
    const float f = exp2f(a);
    const double ref = exp2((double)a);
    const double rel = fabs((double)f - ref) / ref;
    if (rel > local) {
      local = rel;
      arg = first_bits + i;
    }
  }
  // pack (error bits, argument) so one atomicMax keeps the worst pair
  const unsigned long long key =
      ((unsigned long long)__float_as_uint((float)local) << 32) | (unsigned long long)arg;
  atomicMax(worst, key);
}

int main(int argc, char** argv) {
  float lo = 0.0f, hi = 8.0f;
  if (argc > 2) {
    lo = (float)atof(argv[1]);
    hi = (float)atof(argv[2]);
  }
  // positive floats are ordered like their bits: walk [bits(lo), bits(hi)]
  uint32_t b0, b1;
  std::memcpy(&b0, &lo, 4);
  std::memcpy(&b1, &hi, 4);
  if (lo < 0.f || hi < lo) {
    std::printf("need 0 <= lo <= hi\n");
    return 2;
  }
  unsigned long long* d = nullptr;
  if (cudaMalloc(&d, sizeof(*d)) != cudaSuccess) return 1;
  cudaMemset(d, 0, sizeof(*d));
  k_exp2_error<<<148 * 8, 256>>>(b0, b1 - b0 + 1, d);
  unsigned long long h = 0;
  if (cudaMemcpy(&h, d, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return 1;
  cudaFree(d);
  const uint32_t eb = (uint32_t)(h >> 32), ab = (uint32_t)h;
  float e, a;
  std::memcpy(&e, &eb, 4);
  std::memcpy(&a, &ab, 4);
  std::printf("max_rel_err %.9e at %.9g over %u floats\n", e, a, b1 - b0 + 1);
  return 0;
}
