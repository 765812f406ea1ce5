// Device-side twin of the integer part of the seeded input generator in synth/__init__.py.
//
// Test and bench infrastructure only: it draws dense trits and int8 output-head weights on the
// GPU so that multi-gigabyte synthetic weights need not cross PCIe. It holds none of the arithmetic
// of the method. The generator is SplitMix64 (Steele, Lea & Flood, OOPSLA 2014): element
// (row, col) of a tensor is output number row*K+col+1 of the stream whose state starts at `key`.
// Keys and thresholds are computed on the host by synth/__init__.py and passed in, so both sides
// agree bit for bit (integer arithmetic only).
#include <cstdint>
#include <cuda_runtime.h>

namespace {

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;

__device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// Eight consecutive elements per thread, written as two 32-bit words.
__global__ void k_trits(uint64_t key, uint64_t t0, uint64_t t1, int64_t n_elems, int64_t first_counter,
                        int8_t* __restrict__ out) {
  const int64_t n8 = n_elems / 8;
  for (int64_t v = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; v < n8; v += (int64_t)gridDim.x * blockDim.x) {
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const uint64_t c = (uint64_t)(first_counter + v * 8 + e);
      const uint64_t u = mix64(key + (c + 1ull) * kGamma);
      const int8_t tr = u < t0 ? 0 : (u < t1 ? 1 : -1);
      w[e >> 2] |= (uint32_t)(uint8_t)tr << (8 * (e & 3));
    }
    reinterpret_cast<uint2*>(out)[v] = make_uint2(w[0], w[1]);
  }
}

__global__ void k_head(uint64_t key, int64_t n_elems, int64_t first_counter, int8_t* __restrict__ out) {
  const int64_t n8 = n_elems / 8;
  for (int64_t v = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; v < n8; v += (int64_t)gridDim.x * blockDim.x) {
    uint32_t w[2] = {0u, 0u};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const uint64_t c = (uint64_t)(first_counter + v * 8 + e);
      const uint64_t u = mix64(key + (c + 1ull) * kGamma);
      const int8_t q = (int8_t)((int)(u % 255ull) - 127);
      w[e >> 2] |= (uint32_t)(uint8_t)q << (8 * (e & 3));
    }
    reinterpret_cast<uint2*>(out)[v] = make_uint2(w[0], w[1]);
  }
}

int grid_for(int64_t n8) {
  int64_t g = (n8 + 255) / 256;
  if (g > 148 * 16) g = 148 * 16;
  if (g < 1) g = 1;
  return (int)g;
}

}  // namespace

extern "C" {

// Rows [row0, row0 + N) of an (unbounded) N x K trit tensor into out (int8, N*K, 8-byte aligned).
// Returns 0 on success, 1 on bad arguments, 2 on a launch error.
int synth_trits(uint64_t key, uint64_t t0, uint64_t t1, int64_t N, int64_t K, int64_t row0, int8_t* out,
                void* stream) {
  if (!out || N < 0 || K <= 0 || row0 < 0 || (K % 8) != 0 || (reinterpret_cast<uintptr_t>(out) & 7u)) return 1;
  const int64_t n = N * K;
  if (n == 0) return 0;
  k_trits<<<grid_for(n / 8), 256, 0, (cudaStream_t)stream>>>(key, t0, t1, n, row0 * K, out);
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

int synth_head(uint64_t key, int64_t V, int64_t K, int64_t row0, int8_t* out, void* stream) {
  if (!out || V < 0 || K <= 0 || row0 < 0 || (K % 8) != 0 || (reinterpret_cast<uintptr_t>(out) & 7u)) return 1;
  const int64_t n = V * K;
  if (n == 0) return 0;
  k_head<<<grid_for(n / 8), 256, 0, (cudaStream_t)stream>>>(key, n, row0 * K, out);
  return cudaGetLastError() == cudaSuccess ? 0 : 2;
}

}  // extern "C"
