// Device twin of starkv_inputs/gen.py: the same counter-based generator
// (SplitMix64 finaliser of key + (i+1)*golden; Irwin-Hall of four 16-bit
// fields; fp32 scale; fp32 spectrum multiply; fp16 round-to-nearest).  Used by
// tests and the benchmark to fill large device buffers with exactly the bytes
// the host generator defines.  Holds no part of the method's arithmetic.
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <cstdint>

namespace {

__device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z ^= z >> 30;
  z *= 0xBF58476D1CE4E5B9ull;
  z ^= z >> 27;
  z *= 0x94D049BB133111EBull;
  z ^= z >> 31;
  return z;
}

// out[i][j] = fp16( fp32(ih4(key, (row_offset+i)*row_len + j) * IH4_SCALE) * spectrum[j % spec_len] )
__global__ void gen_codes_kernel(uint64_t key, int64_t n_rows, int32_t row_len, int64_t row_offset,
                                 const float* spectrum, int32_t spec_len, float ih4_scale, __half* out) {
  const int64_t n = n_rows * row_len;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t i = e / row_len;
    const int32_t j = static_cast<int32_t>(e - i * row_len);
    const uint64_t idx = static_cast<uint64_t>((row_offset + i) * row_len + j);
    const uint64_t z = mix64(key + (idx + 1ull) * 0x9E3779B97F4A7C15ull);
    const int64_t s = static_cast<int64_t>(z & 0xFFFF) + static_cast<int64_t>((z >> 16) & 0xFFFF) +
                      static_cast<int64_t>((z >> 32) & 0xFFFF) + static_cast<int64_t>(z >> 48) - 131070;
    float x = __fmul_rn(static_cast<float>(s), ih4_scale);
    if (spectrum) x = __fmul_rn(x, spectrum[j % spec_len]);
    out[e] = __float2half_rn(x);
  }
}

}  // namespace

extern "C" int starkv_gen_codes(uint64_t key, int64_t n_rows, int32_t row_len, int64_t row_offset,
                                const float* spectrum, int32_t spec_len, float ih4_scale, void* out,
                                void* stream) {
  if (n_rows < 0 || row_len <= 0 || !out || (spectrum && spec_len <= 0)) return 1;
  if (n_rows == 0) return 0;
  const int64_t n = n_rows * row_len;
  int64_t blocks = (n + 255) / 256;
  if (blocks > 148 * 64) blocks = 148 * 64;
  gen_codes_kernel<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      key, n_rows, row_len, row_offset, spectrum, spec_len, ih4_scale, static_cast<__half*>(out));
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}
