// Ternary GEMV (M = 1) and small-M GEMM (M <= 16) over the packed two-plane layout.
//
//   Y[m][n] = scale[n] * sum_k t[n][k] * X[m][k]
//
// The contraction of a linear layer, y_j = sum_i w_ij x_i (PyTorchKR review "Fermion Research,
// 3진 계열 포맷으로 직접 학습한 Neutrino-1 모델군 3종 공개", section "학습 중에 포맷이 있어야 하는
// 이유", displayed equation), with ternary weights decoded inside the kernel (aiatolah.com,
// "Neutrino-1 8B: modelo ternario ...", second paragraph). At decode batch sizes this is bound by
// the bytes of weights streamed per token (same review, section "뉴트리노 엔진": tok/s_max =
// memory bandwidth / bytes per token), so the kernel is built to stream the 2-bit planes at HBM
// speed and to spend well under one instruction per trit on the decode:
//   * each lane streams 128-bit words of both planes of two rows straight into registers, with
//     the next 512-trit chunk in flight while the current one is decoded;
//   * one LOP3 pair + rotate merges a mask/sign word pair into 2-bit fields, and one shift + AND
//     per register turns them into tensor-core operands holding 64*t (int8) or 2.0*t (bf16)
//     (see tern_device.cuh); the warp's 16 rows x 32 trits go through mma.sync, where the +-1
//     products are exact (the add / skip / subtract rule, origotech.dev Figure I);
//   * the activation slice of the CTA is staged once in shared memory (swizzled, conflict-free);
//     for M > 1 every decoded weight register is reused for all M activation rows (n-groups);
//   * CTAs of one row block that split K form a thread-block cluster and add their partial sums
//     through distributed shared memory in rank order: no global scratch, deterministic results.
// int8 mode accumulates exactly in int32 (64 * sum t*q); bf16 mode accumulates 2 * sum t*x in
// fp32 on the tensor cores.
#include <cooperative_groups.h>
#include <cstdint>
#include <cuda_runtime.h>
#include <type_traits>

#include "tern_device.cuh"
#include "tern_kernels.h"

namespace cg = cooperative_groups;

namespace tern {
namespace {

constexpr int kRows = 128;  // rows per CTA: 8 warps x 16 rows

__device__ __forceinline__ uint32_t u4get(const uint4& v, int e) {
  return e == 0 ? v.x : (e == 1 ? v.y : (e == 2 ? v.z : v.w));
}

template <int MODE, int NG>
__global__ void __launch_bounds__(kThreads) k_tern_gemm(const GemmParams p) {
  extern __shared__ __align__(16) uint32_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int ks = blockIdx.x;                       // K slice = cluster rank
  const int k0 = ks * p.kr;
  const int row0 = blockIdx.y * kRows + warp * 16;
  const int KM = p.K >> 5;                         // words per plane per row
  const int nw = p.kr >> 5;                        // words per plane in this slice (multiple of 4)
  const int nchunks = (nw + 15) >> 4;
  const bool warp_live = row0 < p.N;
  const int ra = min(row0 + g, p.N - 1), rb = min(row0 + g + 8, p.N - 1);
  const uint32_t* pa = p.planes + (size_t)ra * (2 * KM) + (k0 >> 5);
  const uint32_t* pb = p.planes + (size_t)rb * (2 * KM) + (k0 >> 5);

  // weight chunk c: words [16c + 4t, 16c + 4t + 4) of both planes of rows ra, rb
  auto load_chunk = [&](int c, uint4 (&w)[4]) {
    const int off = 16 * c + 4 * t;
    if (warp_live && off < nw) {
      w[0] = ld_stream(pa + off);
      w[1] = ld_stream(pb + off);
      w[2] = ld_stream(pa + KM + off);
      w[3] = ld_stream(pb + KM + off);
    } else {
      w[0] = w[1] = w[2] = w[3] = make_uint4(0u, 0u, 0u, 0u);
    }
  };
  // Weights do not depend on the preceding kernel: start streaming them before the dependency wait.
  uint4 cur[4], nxt[4];
  load_chunk(0, cur);
  load_chunk(1, nxt);
  pdl_wait();

  // ---- stage the activation slice X[:, k0 : k0 + kr) in shared memory --------------------------
  const int RS = (MODE == 0 ? p.kr / 2 : p.kr / 4) + 16;   // words per activation row (+16: banks)
  if (MODE == 0) {
    const int per_row = p.kr >> 3;                          // 16-byte chunks of 8 bf16
    const uint16_t* xs = static_cast<const uint16_t*>(p.x);
    for (int i = threadIdx.x; i < p.M * per_row; i += kThreads) {
      const int m = i / per_row, v = i - m * per_row;
      const uint4 val = ld_nc(xs + (size_t)m * p.K + k0 + 8 * v);
      *reinterpret_cast<uint4*>(smem + m * RS + 4 * (v ^ ((v >> 4) & 3))) = val;
    }
  } else {
    const int per_row = p.kr >> 4;                          // 16-byte halves of 32-trit blocks
    const int8_t* xs = static_cast<const int8_t*>(p.x);
    for (int i = threadIdx.x; i < p.M * per_row; i += kThreads) {
      const int m = i / per_row, v = i - m * per_row;
      const uint4 val = permute_i8_half(ld_nc(xs + (size_t)m * p.K + k0 + 16 * v));
      *reinterpret_cast<uint4*>(smem + m * RS + 4 * (v ^ ((v >> 3) & 3))) = val;
    }
  }
  __syncthreads();

  using Acc = typename std::conditional<MODE == 0, float, int>::type;
  Acc acc[NG][4];
#pragma unroll
  for (int n = 0; n < NG; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = Acc(0);

  for (int c = 0; c < nchunks; ++c) {
    const bool live = (16 * c + 4 * t) < nw;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int w = 16 * c + 4 * t + e;                     // local word index of this lane
      uint32_t wa0, wb0, wa1, wb1;
      merge_planes(u4get(cur[0], e), u4get(cur[2], e), wa0, wb0);   // row ra
      merge_planes(u4get(cur[1], e), u4get(cur[3], e), wa1, wb1);   // row rb
      if constexpr (MODE == 0) {
        uint32_t xb[NG][16];
#pragma unroll
        for (int n = 0; n < NG; ++n) {
          const int m = 8 * n + g;
          if (live && m < p.M) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int ch = 4 * w + q;
              const uint4 v = *reinterpret_cast<const uint4*>(smem + m * RS + 4 * (ch ^ ((ch >> 4) & 3)));
              xb[n][4 * q] = v.x; xb[n][4 * q + 1] = v.y; xb[n][4 * q + 2] = v.z; xb[n][4 * q + 3] = v.w;
            }
          } else {
#pragma unroll
            for (int q = 0; q < 16; ++q) xb[n][q] = 0u;
          }
        }
#define TERN_BF16_STEP(A0, A1)                                                                    \
  {                                                                                              \
    const uint32_t a0 = dec_bf16<A0>(wa0, wb0), a1 = dec_bf16<A0>(wa1, wb1);                     \
    const uint32_t a2 = dec_bf16<A1>(wa0, wb0), a3 = dec_bf16<A1>(wa1, wb1);                     \
    _Pragma("unroll") for (int n = 0; n < NG; ++n) mma_bf16(acc[n], a0, a1, a2, a3, xb[n][A0], xb[n][A1]); \
  }
        TERN_BF16_STEP(0, 1) TERN_BF16_STEP(2, 3) TERN_BF16_STEP(4, 5) TERN_BF16_STEP(6, 7)
        TERN_BF16_STEP(8, 9) TERN_BF16_STEP(10, 11) TERN_BF16_STEP(12, 13) TERN_BF16_STEP(14, 15)
#undef TERN_BF16_STEP
      } else {
        uint32_t xb[NG][8];
#pragma unroll
        for (int n = 0; n < NG; ++n) {
          const int m = 8 * n + g;
          if (live && m < p.M) {
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              const int ch = 2 * w + q;
              const uint4 v = *reinterpret_cast<const uint4*>(smem + m * RS + 4 * (ch ^ ((ch >> 3) & 3)));
              xb[n][4 * q] = v.x; xb[n][4 * q + 1] = v.y; xb[n][4 * q + 2] = v.z; xb[n][4 * q + 3] = v.w;
            }
          } else {
#pragma unroll
            for (int q = 0; q < 8; ++q) xb[n][q] = 0u;
          }
        }
#define TERN_I8_STEP(R0, R1)                                                                      \
  {                                                                                              \
    const uint32_t a0 = dec_i8<R0>(wa0, wb0), a1 = dec_i8<R0>(wa1, wb1);                         \
    const uint32_t a2 = dec_i8<R1>(wa0, wb0), a3 = dec_i8<R1>(wa1, wb1);                         \
    _Pragma("unroll") for (int n = 0; n < NG; ++n) mma_s8(acc[n], a0, a1, a2, a3, xb[n][R0], xb[n][R1]); \
  }
        TERN_I8_STEP(0, 1) TERN_I8_STEP(2, 3) TERN_I8_STEP(4, 5) TERN_I8_STEP(6, 7)
#undef TERN_I8_STEP
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) cur[i] = nxt[i];
    load_chunk(c + 2, nxt);
  }
  pdl_launch_dependents();

  // ---- epilogue ----------------------------------------------------------------------------------
  // int8: y = ((float)(acc / 64) * s_x) * scale, two fp32 round-to-nearest multiplies.
  // bf16: y = (acc * 0.5) * scale.
  auto finish = [&](Acc v, int m, int row) -> float {
    const float sc = f16_bits_to_float(p.scale[row]);
    if constexpr (MODE == 0) {
      return __fmul_rn(__fmul_rn(v, 0.5f), sc);
    } else {
      return __fmul_rn(__fmul_rn(__int2float_rn(v >> 6), p.sx[m]), sc);
    }
  };
  if (p.ksplit == 1) {
#pragma unroll
    for (int n = 0; n < NG; ++n)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int m = 8 * n + 2 * t + (i & 1);
        const int row = row0 + g + 8 * (i >> 1);
        if (m < p.M && row < p.N) p.y[(size_t)m * p.N + row] = finish(acc[n][i], m, row);
      }
    return;
  }
  // Split K: partial tile [kRows][8*NG] in this CTA's shared memory, then a cluster-wide sum.
  constexpr int kCols = 8 * NG;
  Acc* part = reinterpret_cast<Acc*>(smem + p.M * RS);
#pragma unroll
  for (int n = 0; n < NG; ++n)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int col = 8 * n + 2 * t + (i & 1);
      const int lrow = warp * 16 + g + 8 * (i >> 1);
      part[lrow * kCols + col] = acc[n][i];
    }
  cg::cluster_group cluster = cg::this_cluster();
  cluster.sync();
  const int rows_per_rank = kRows / p.ksplit;
  for (int i = threadIdx.x; i < rows_per_rank * kCols; i += kThreads) {
    const int lrow = ks * rows_per_rank + i / kCols, col = i % kCols;
    const int row = blockIdx.y * kRows + lrow;
    if (col >= p.M || row >= p.N) continue;
    Acc sum = Acc(0);
    for (int r = 0; r < p.ksplit; ++r) {
      const Acc* rp = cluster.map_shared_rank(part, r);
      sum += rp[lrow * kCols + col];
    }
    p.y[(size_t)col * p.N + row] = finish(sum, col, row);
  }
  cluster.sync();
}

template <int MODE, int NG>
cudaError_t launch_one(const GemmParams& p, size_t smem, bool pdl, cudaStream_t st) {
  auto kern = k_tern_gemm<MODE, NG>;
  // Raise the kernel's dynamic shared-memory limit once per size increase (not on every launch).
  static int smem_set = 0;
  cudaError_t e = cudaSuccess;
  if ((int)smem > smem_set) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    smem_set = (int)smem;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.ksplit, (p.N + kRows - 1) / kRows, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (p.ksplit > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = p.ksplit;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

}  // namespace

// Shared-memory bytes of one CTA: activation slice (+ padding) and the split-K partial tile.
size_t gemm_smem_bytes(int mode, int M, int kr) {
  const int RS = (mode == 0 ? kr / 2 : kr / 4) + 16;
  const int ng = (M + 7) / 8;
  return (size_t)M * RS * 4 + (size_t)kRows * 8 * ng * 4;
}

int gemm_rows_per_cta() { return kRows; }

cudaError_t launch_tern_gemm(const GemmParams& p, bool pdl, cudaStream_t st) {
  const int mode = p.mode;
  const int ng = (p.M + 7) / 8;
  const size_t smem = gemm_smem_bytes(mode, p.M, p.kr);
  if (mode == 0) return ng == 1 ? launch_one<0, 1>(p, smem, pdl, st) : launch_one<0, 2>(p, smem, pdl, st);
  return ng == 1 ? launch_one<1, 1>(p, smem, pdl, st) : launch_one<1, 2>(p, smem, pdl, st);
}

}  // namespace tern
