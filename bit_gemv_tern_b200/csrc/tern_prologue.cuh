// Activation prologues: the step before a linear layer, computed where its operands are prepared.
//
// In the Qwen3 block of the Neutrino-1 models (PyTorchKR review "Fermion Research, 3진 계열 포맷으로
// 직접 학습한 Neutrino-1 모델군 3종 공개", model table section "세 모델과 하나의 컨테이너") the input
// of q|k|v and of gate|up is an RMSNorm of the residual stream, and the input of down is the SwiGLU
// of the gate|up output. Each prologue turns fp32 rows (or bf16 rows) into the bf16 activation the
// linear consumes, all in fp64 with one round-to-nearest-even step to bf16:
//   kind 1 (bf16):    x_k                               (the activation as given, bf16)
//   kind 2 (cast):    bf16(s_k)                         (an fp32 row)
//   kind 3 (RMSNorm): bf16((s_k * r) * g_k), r = 1 / sqrt(sum_k s_k^2 / K + eps), g a bf16 gain
//   kind 4 (SwiGLU):  bf16(silu(s_k) * s_(K+k)), silu(z) = z / (1 + exp(-z)), gate then up
// The int8-activation mode then quantises that bf16 row per token (tern_device.cuh, quant_i8).
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "tern_device.cuh"

namespace tern {

enum : int32_t { kProNone = 0, kProBF16 = 1, kProCast = 2, kProRMSNorm = 3, kProSwiGLU = 4 };

// Sum of the fp64 values of a CTA in a fixed order (a butterfly inside each warp, then warp
// partials in warp order), so every launch gives the same bits. `red` holds one double per warp.
template <int kThreadsT>
__device__ __forceinline__ double block_sum_fixed(double v, double* red) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  __syncthreads();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  double s = 0.0;
  for (int w = 0; w < kThreadsT / 32; ++w) s += red[w];
  return s;
}

// RMSNorm's reciprocal root mean square of one fp32 row of K elements (every thread gets it).
template <int kThreadsT>
__device__ __forceinline__ double rmsnorm_r(const float* src, int K, float eps, double* red) {
  double ss = 0.0;
  for (int k = threadIdx.x * 4; k < K; k += kThreadsT * 4) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(src + k));
    ss += (double)v.x * v.x + (double)v.y * v.y + (double)v.z * v.z + (double)v.w * v.w;
  }
  ss = block_sum_fixed<kThreadsT>(ss, red);
  return 1.0 / sqrt(ss / (double)K + (double)eps);
}

// The prologue's bf16 values of elements k .. k+7 of a row (k % 8 == 0), packed two per word.
//   src: the row (bf16 bits for kProBF16, fp32 otherwise; SwiGLU rows hold 2K values)
__device__ __forceinline__ uint4 prologue8(int kind, const void* src, const uint16_t* gain, int K, int k, double r) {
  if (kind == kProBF16) return ld_nc(static_cast<const uint16_t*>(src) + k);
  const float* s = static_cast<const float*>(src);
  const float4 a0 = __ldg(reinterpret_cast<const float4*>(s + k)), a1 = __ldg(reinterpret_cast<const float4*>(s + k + 4));
  const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
  uint16_t h[8];
  if (kind == kProSwiGLU) {
    const float4 b0 = __ldg(reinterpret_cast<const float4*>(s + K + k)), b1 = __ldg(reinterpret_cast<const float4*>(s + K + k + 4));
    const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const double z = (double)a[e];
      h[e] = bf16_rn((z / (1.0 + exp(-z))) * (double)b[e]);
    }
  } else if (kind == kProRMSNorm) {
    const uint4 gw = ld_nc(gain + k);
    const uint32_t g[4] = {gw.x, gw.y, gw.z, gw.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const double ge = (double)bf16_bits_to_float((e & 1) ? (g[e >> 1] >> 16) : (g[e >> 1] & 0xFFFFu));
      h[e] = bf16_rn(((double)a[e] * r) * ge);
    }
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) h[e] = bf16_rn((double)a[e]);
  }
  return make_uint4(h[0] | ((uint32_t)h[1] << 16), h[2] | ((uint32_t)h[3] << 16), h[4] | ((uint32_t)h[5] << 16),
                    h[6] | ((uint32_t)h[7] << 16));
}

// Largest magnitude among 8 packed bf16 values (as fp32; NaN-free inputs).
__device__ __forceinline__ float absmax8(uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  float m = 0.0f;
#pragma unroll
  for (int e = 0; e < 4; ++e)
    m = fmaxf(m, fmaxf(fabsf(bf16_bits_to_float(w[e] & 0xFFFFu)), fabsf(bf16_bits_to_float(w[e] >> 16))));
  return m;
}

}  // namespace tern
