// Device fill of the seeded synthetic expert weights (the CUDA side of the
// input generator in synth/__init__.py).  Input generation only: no step of
// the MoE layer is computed here.
//
// SplitMix64 (Steele, Lea and Flood, OOPSLA 2014; finaliser constants as
// published with Vigna's splitmix64): word i of the stream with key K is
// mix64(K + (i + 1) * 0x9E3779B97F4A7C15).
//   codes : byte j = byte (j % 8) of word j / 8 (little-endian)
//   scales: element j = fp16_rn( 0.005f + 0.015f * ((word_j >> 40) * 2^-24) ),
//           multiply and add rounded separately in fp32.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

__device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__device__ __forceinline__ uint64_t word_at(uint64_t key, uint64_t i) {
  return mix64(key + (i + 1ull) * 0x9E3779B97F4A7C15ull);
}

// dst receives bytes [start, start + count) of the stream; start % 8 == 0.
__global__ void fill_codes_kernel(uint64_t key, uint64_t start, uint64_t count, uint8_t* dst) {
  const uint64_t nwords = (count + 7) / 8;
  const uint64_t w0 = start / 8;
  for (uint64_t i = blockIdx.x * static_cast<uint64_t>(blockDim.x) + threadIdx.x; i < nwords;
       i += static_cast<uint64_t>(gridDim.x) * blockDim.x) {
    const uint64_t v = word_at(key, w0 + i);
    if (8 * i + 8 <= count) {
      reinterpret_cast<uint2*>(dst)[i] = make_uint2(static_cast<uint32_t>(v), static_cast<uint32_t>(v >> 32));
    } else {
      for (uint64_t b = 0; 8 * i + b < count; ++b) dst[8 * i + b] = static_cast<uint8_t>(v >> (8 * b));
    }
  }
}

__global__ void fill_scales_kernel(uint64_t key, uint64_t start, uint64_t count, uint16_t* dst) {
  for (uint64_t i = blockIdx.x * static_cast<uint64_t>(blockDim.x) + threadIdx.x; i < count;
       i += static_cast<uint64_t>(gridDim.x) * blockDim.x) {
    const uint64_t v = word_at(key, start + i);
    const float u = static_cast<float>(static_cast<uint32_t>(v >> 40)) * 5.9604644775390625e-08f;  // 2^-24
    const float s = __fadd_rn(__fmul_rn(u, 0.015f), 0.005f);
    dst[i] = __half_as_ushort(__float2half_rn(s));
  }
}

}  // namespace

extern "C" {

// Returns 0 on success, 1 on a bad argument, 2 on a CUDA launch error.
int coli_synth_fill_codes(uint64_t key, uint64_t start, uint64_t count, uint8_t* dst, void* stream) {
  if ((start % 8) != 0 || (!dst && count) || (reinterpret_cast<uintptr_t>(dst) % 8) != 0) return 1;
  if (count == 0) return 0;
  const uint64_t nwords = (count + 7) / 8;
  uint64_t blocks = (nwords + 255) / 256;
  if (blocks > 65536) blocks = 65536;
  fill_codes_kernel<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(key, start, count, dst);
  return cudaPeekAtLastError() == cudaSuccess ? 0 : 2;
}

int coli_synth_fill_scales(uint64_t key, uint64_t start, uint64_t count, uint16_t* dst, void* stream) {
  if (!dst && count) return 1;
  if (count == 0) return 0;
  uint64_t blocks = (count + 255) / 256;
  if (blocks > 65536) blocks = 65536;
  fill_scales_kernel<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(key, start, count, dst);
  return cudaPeekAtLastError() == cudaSuccess ? 0 : 2;
}

}  // extern "C"
