// Internal launch interface between the C ABI (tern_abi.cu) and the kernel files.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace tern {

// Ternary GEMV / small-M GEMM (tern_gemv.cu).
struct GemmParams {
  const uint32_t* planes;
  const uint16_t* scale;
  int32_t N, K;
  const void* x;          // bf16 bits [M][K] (mode 0) or int8 [M][K] (mode 1)
  const float* sx;        // [M], int8 mode only
  float* y;               // [M][N]
  int32_t M;              // 1..16
  int32_t mode;           // 0 = bf16 activations, 1 = int8 activations
  int32_t kr;             // trits of K per CTA (multiple of 128); ksplit * kr == K
  int32_t ksplit;         // CTAs splitting K in one cluster: 1, 2, 4 or 8
};
size_t gemm_smem_bytes(int mode, int M, int kr);
int gemm_rows_per_cta();
cudaError_t launch_tern_gemm(const GemmParams& p, bool pdl, cudaStream_t st);

// int8 output head with argmax (tern_head.cu).
struct HeadParams {
  const int8_t* W;
  const uint16_t* sh;
  int32_t V, K, M;
  int32_t mode;           // 0 = bf16 activations (three exact int8 limbs), 1 = int8 activations
  const void* x;
  const float* sx;
  int32_t* argmax;
  float* maxval;
  float* logits;          // optional [M][V]
  unsigned long long* keys;  // workspace: M packed (value key, index) maxima
  unsigned int* counter;     // workspace: CTAs finished
  int32_t kr, ksplit;
  int32_t nrb;            // row blocks of 128 rows
  int32_t nby;            // CTAs along the row-block axis (persistent loop)
};
size_t head_workspace_bytes(int M);
size_t head_smem_bytes(int mode, int M, int kr);
cudaError_t launch_head(const HeadParams& p, bool pdl, cudaStream_t st);

// Loader kernels (tern_pack.cu).
cudaError_t launch_pack_trits(const int8_t* src, int32_t N, int32_t K, uint32_t* planes, int32_t* flag,
                              cudaStream_t st);
cudaError_t launch_unpack_base3(const uint8_t* src, int32_t N, int32_t K, uint32_t* planes, int32_t* flag,
                                cudaStream_t st);
cudaError_t launch_encode_base3(const int8_t* src, int32_t N, int32_t K, uint8_t* out, int32_t* flag,
                                cudaStream_t st);
cudaError_t launch_occupancy(const uint32_t* planes, int32_t N, int32_t K, int64_t* counts, cudaStream_t st);

// Activation quantiser (tern_act.cu).
cudaError_t launch_quantize(const uint16_t* x, int32_t M, int32_t K, int8_t* q, float* sx, cudaStream_t st);

}  // namespace tern
