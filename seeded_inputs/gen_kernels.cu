// Device twin of seeded_inputs/gen.py: the same counter-based generator, so
// that large synthetic tensors (the 8.94 GB of 70B-shaped head weights) can be
// drawn directly in GPU memory with the exact bits the host version gives.
//
// r_i   = splitmix64-finaliser(key + (i + 1) * 0x9E3779B97F4A7C15)
// c     = sum of the four 16-bit fields of r_i - 131070   (exact integer)
// value = fp32_rne( fp64(c) * scale ), then bf16_rne for bf16 tensors.
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

__device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__device__ __forceinline__ float draw(uint64_t key, uint64_t idx, double scale) {
  const uint64_t r = mix64(key + (idx + 1ull) * 0x9E3779B97F4A7C15ull);
  const int64_t s = int64_t(r & 0xFFFF) + int64_t((r >> 16) & 0xFFFF) + int64_t((r >> 32) & 0xFFFF) + int64_t(r >> 48);
  const double x = __dmul_rn(double(s - 131070), scale);
  return __double2float_rn(x);
}

__global__ void normal_bf16_kernel(uint16_t* out, uint64_t n, uint64_t key, uint64_t start, double scale) {
  for (uint64_t i = blockIdx.x * uint64_t(blockDim.x) + threadIdx.x; i < n; i += uint64_t(gridDim.x) * blockDim.x) {
    uint32_t b = __float_as_uint(draw(key, start + i, scale));
    b += 0x7FFFu + ((b >> 16) & 1u);
    out[i] = uint16_t(b >> 16);
  }
}

__global__ void normal_f32_kernel(float* out, uint64_t n, uint64_t key, uint64_t start, double scale) {
  for (uint64_t i = blockIdx.x * uint64_t(blockDim.x) + threadIdx.x; i < n; i += uint64_t(gridDim.x) * blockDim.x)
    out[i] = draw(key, start + i, scale);
}

int grid_for(uint64_t n) {
  uint64_t g = (n + 255) / 256;
  return int(g > 148ull * 32 ? 148ull * 32 : (g == 0 ? 1 : g));
}

}  // namespace

extern "C" {

__attribute__((visibility("default"))) int sg_normal_bf16(uint16_t* out, uint64_t n, uint64_t key, uint64_t start,
                                                          double scale, void* stream) {
  if (!out) return -1;
  if (n == 0) return 0;
  normal_bf16_kernel<<<grid_for(n), 256, 0, static_cast<cudaStream_t>(stream)>>>(out, n, key, start, scale);
  return cudaGetLastError() == cudaSuccess ? 0 : -3;
}

__attribute__((visibility("default"))) int sg_normal_f32(float* out, uint64_t n, uint64_t key, uint64_t start,
                                                         double scale, void* stream) {
  if (!out) return -1;
  if (n == 0) return 0;
  normal_f32_kernel<<<grid_for(n), 256, 0, static_cast<cudaStream_t>(stream)>>>(out, n, key, start, scale);
  return cudaGetLastError() == cudaSuccess ? 0 : -3;
}

}  // extern "C"
