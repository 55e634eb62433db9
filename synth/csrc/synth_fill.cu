// Device-side filler for the synthetic weight blob.
//
// Produces, for each element index i of a tensor, exactly the value that the
// numpy generator in synth/gen.py produces: splitmix64 on (base + i), the
// Irwin-Hall sum of the four 16-bit lanes, one correctly rounded fp32 multiply,
// and (for bf16 tensors) round-to-nearest-even to bf16. Only integer operations
// and a single IEEE multiply are involved, so the two sides agree bit for bit.
// This is input generation, not part of the denoising path.

#include <cstdint>
#include <cuda_runtime.h>

namespace {

__host__ __device__ inline uint64_t splitmix64(uint64_t z) {
  z += 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__device__ inline float normal_value(uint64_t base, uint64_t i) {
  uint64_t z = splitmix64(base + i);
  int64_t s = (int64_t)(z & 0xFFFF) + (int64_t)((z >> 16) & 0xFFFF) +
              (int64_t)((z >> 32) & 0xFFFF) + (int64_t)(z >> 48);
  int32_t n = (int32_t)(2 * s - 4 * 65535);
  const float scale = __uint_as_float(0x348DE3BDu);
  return __fmul_rn(__int2float_rn(n), scale);
}

__device__ inline uint16_t bf16_rne_bits(float f) {
  uint32_t u = __float_as_uint(f);
  uint32_t r = (u + 0x7FFFu + ((u >> 16) & 1u)) >> 16;
  return (uint16_t)r;
}

__global__ void fill_normal_kernel(void* dst, uint64_t n, uint64_t base, int bf16) {
  uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
  for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
    float w = normal_value(base, i);
    if (bf16) reinterpret_cast<uint16_t*>(dst)[i] = bf16_rne_bits(w);
    else reinterpret_cast<float*>(dst)[i] = w;
  }
}

__global__ void fill_ones_kernel(void* dst, uint64_t n, int bf16) {
  uint64_t stride = (uint64_t)gridDim.x * blockDim.x;
  for (uint64_t i = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
    if (bf16) reinterpret_cast<uint16_t*>(dst)[i] = 0x3F80;
    else reinterpret_cast<float*>(dst)[i] = 1.0f;
  }
}

}  // namespace

extern "C" {

// Fills n elements at dst (device memory) with tensor `tid` of stream `seed`.
// kind: 0 = normal deviates, 1 = ones. bf16: 1 = bf16 elements, 0 = fp32.
// Returns 0, or the cudaError_t of the launch.
int synth_fill(void* dst, uint64_t n, uint64_t seed, uint32_t tid, int kind, int bf16,
               void* stream) {
  if (n == 0) return 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint64_t blocks = (n + 255) / 256;
  if (blocks > 148ull * 32) blocks = 148ull * 32;
  if (kind == 1) {
    fill_ones_kernel<<<(unsigned)blocks, 256, 0, s>>>(dst, n, bf16);
  } else {
    uint64_t base = splitmix64(((seed & 0xFFFFFFFFull) << 32) | (uint64_t)tid);
    fill_normal_kernel<<<(unsigned)blocks, 256, 0, s>>>(dst, n, base, bf16);
  }
  return (int)cudaGetLastError();
}

}  // extern "C"
