// Device twin of tenant_mixed_precision_b200/synth.py's counter-based input stream.
//
// Test and benchmark inputs only: this library draws numbers and holds none of the method's
// arithmetic.  SplitMix64 (Steele, Lea and Flood, OOPSLA 2014): state_i = key + (i+1)*GAMMA,
// output = mix64(state_i), key = mix64(mix64(seed + GAMMA) ^ (stream + 2*GAMMA)).  A value is the
// centred Irwin-Hall(4) sum of the four 16-bit fields, (h0+h1+h2+h3+2-2^17)/2^16 (exact in fp32),
// times an fp32 constant c with one round-to-nearest-even multiply.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define GAMMA 0x9E3779B97F4A7C15ull

__host__ __device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

static uint64_t stream_key(uint64_t seed, uint64_t stream) {
  const uint64_t a = mix64(seed + GAMMA);
  return mix64(a ^ (stream + GAMMA + GAMMA));
}

__device__ __forceinline__ float ih4(uint64_t key, uint64_t i, float c) {
  const uint64_t w = mix64(key + (i + 1) * GAMMA);
  const int64_t s = (int64_t)(w & 0xFFFF) + (int64_t)((w >> 16) & 0xFFFF) + (int64_t)((w >> 32) & 0xFFFF) +
                    (int64_t)(w >> 48);
  const float base = __fmul_rn((float)(s + 2 - (1 << 17)), 1.0f / 65536.0f);
  return __fmul_rn(base, c);
}

__global__ void k_normal_f32(uint64_t key, uint64_t start, uint64_t n, float c, float* out) {
  for (uint64_t i = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; i < n; i += (uint64_t)gridDim.x * blockDim.x)
    out[i] = ih4(key, start + i, c);
}

__global__ void k_normal_bf16(uint64_t key, uint64_t start, uint64_t n, float c, __nv_bfloat16* out) {
  for (uint64_t i = blockIdx.x * (uint64_t)blockDim.x + threadIdx.x; i < n; i += (uint64_t)gridDim.x * blockDim.x)
    out[i] = __float2bfloat16_rn(ih4(key, start + i, c));
}

static unsigned grid_for(uint64_t n) {
  uint64_t b = (n + 255) / 256;
  return (unsigned)(b < 148ull * 32 ? (b ? b : 1) : 148ull * 32);
}

extern "C" int dcs_normal_f32(uint64_t seed, uint64_t stream, uint64_t start, uint64_t n, float c, float* out,
                              void* cuda_stream) {
  if (n == 0) return 0;
  k_normal_f32<<<grid_for(n), 256, 0, (cudaStream_t)cuda_stream>>>(stream_key(seed, stream), start, n, c, out);
  return (int)cudaGetLastError();
}

extern "C" int dcs_normal_bf16(uint64_t seed, uint64_t stream, uint64_t start, uint64_t n, float c, void* out,
                               void* cuda_stream) {
  if (n == 0) return 0;
  k_normal_bf16<<<grid_for(n), 256, 0, (cudaStream_t)cuda_stream>>>(stream_key(seed, stream), start, n, c,
                                                                     (__nv_bfloat16*)out);
  return (int)cudaGetLastError();
}
