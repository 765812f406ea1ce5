// Per-token absmax int8 quantisation of bf16 activations: the int8-activation runtime of the
// PyTorchKR review "Fermion Research, 3진 계열 포맷으로 직접 학습한 Neutrino-1 모델군 3종 공개",
// section "토큰 동일성의 경계: 그리디, float32, 그리고 두 개의 근접 동점". The pages do not give
// the quantiser; this library's reading is s_x = absmax / 127 and q = clamp(rint(x / s_x),
// -127, 127), both divisions IEEE fp32 round-to-nearest, rint rounding half to even.
#include <cstdint>
#include <cuda_runtime.h>

#include "tern_device.cuh"
#include "tern_kernels.h"
#include "tern_prologue.cuh"

namespace tern {
namespace {

// One CTA per activation row.
__global__ void __launch_bounds__(256) k_quantize(const uint16_t* __restrict__ x, int32_t K, int8_t* __restrict__ q,
                                                  float* __restrict__ sx) {
  __shared__ float red[8];
  const int64_t row = blockIdx.x;
  const uint16_t* xr = x + row * K;
  pdl_wait();
  float amax = 0.0f;
  for (int k = threadIdx.x * 8; k < K; k += blockDim.x * 8) {
    const uint4 v = ld_nc(xr + k);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      amax = fmaxf(amax, fabsf(bf16_bits_to_float(w[e] & 0xFFFFu)));
      amax = fmaxf(amax, fabsf(bf16_bits_to_float(w[e] >> 16)));
    }
  }
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) amax = fmaxf(amax, red[i]);
  const float s = __fdiv_rn(amax, 127.0f);
  if (threadIdx.x == 0) sx[row] = s;
  int8_t* qr = q + row * K;
  for (int k = threadIdx.x * 8; k < K; k += blockDim.x * 8) {
    const uint4 v = ld_nc(xr + k);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t out[2] = {0u, 0u};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const uint32_t bits = (e & 1) ? (w[e >> 1] >> 16) : (w[e >> 1] & 0xFFFFu);
      int qi = 0;
      if (s != 0.0f) {
        qi = __float2int_rn(__fdiv_rn(bf16_bits_to_float(bits), s));   // round half to even
        qi = qi > 127 ? 127 : (qi < -127 ? -127 : qi);
      }
      out[e >> 2] |= (uint32_t)(uint8_t)(int8_t)qi << (8 * (e & 3));
    }
    *reinterpret_cast<uint2*>(qr + k) = make_uint2(out[0], out[1]);
  }
  pdl_launch_dependents();
}

// One CTA per row: the prologue's bf16 row (tern_prologue.cuh), as the batched launch computes it
// inside its operand preparation.
constexpr int kProThreads = 256;
__global__ void __launch_bounds__(kProThreads) k_prologue(int32_t kind, const void* src, const uint16_t* gain,
                                                         float eps, int32_t K, uint16_t* out) {
  __shared__ double red[kProThreads / 32];
  const int64_t row = blockIdx.x;
  const int64_t row_elems = (int64_t)K * (kind == kProSwiGLU ? 2 : 1);
  const void* s = kind == kProBF16 ? static_cast<const void*>(static_cast<const uint16_t*>(src) + row * K)
                                   : static_cast<const void*>(static_cast<const float*>(src) + row * row_elems);
  pdl_wait();
  const double r = kind == kProRMSNorm ? rmsnorm_r<kProThreads>(static_cast<const float*>(s), K, eps, red) : 1.0;
  for (int k = threadIdx.x * 8; k < K; k += kProThreads * 8)
    *reinterpret_cast<uint4*>(out + row * K + k) = prologue8(kind, s, gain, K, k, r);
  pdl_launch_dependents();
}

}  // namespace

cudaError_t launch_prologue(int32_t kind, const void* src, const uint16_t* gain, float eps, int32_t M, int32_t K,
                            uint16_t* out, cudaStream_t st) {
  k_prologue<<<M, kProThreads, 0, st>>>(kind, src, gain, eps, K, out);
  return cudaGetLastError();
}

cudaError_t launch_quantize(const uint16_t* x, int32_t M, int32_t K, int8_t* q, float* sx, cudaStream_t st) {
  k_quantize<<<M, 256, 0, st>>>(x, K, q, sx);
  return cudaGetLastError();
}

}  // namespace tern
