// Ternary GEMV (M = 1) and small-M GEMM (M <= 16) over the packed two-plane layout.
//
//   Y[m][n] = scale[n] * sum_k t[n][k] * X[m][k]
//
// The contraction of a linear layer, y_j = sum_i w_ij x_i (PyTorchKR review "Fermion Research,
// 3진 계열 포맷으로 직접 학습한 Neutrino-1 모델군 3종 공개", section "학습 중에 포맷이 있어야 하는
// 이유", displayed equation), with ternary weights decoded inside the kernel (aiatolah.com,
// "Neutrino-1 8B: modelo ternario ...", second paragraph). At decode batch sizes this is bound by
// the bytes of weights streamed per token (same review, section "뉴트리노 엔진": tok/s_max =
// memory bandwidth / bytes per token), so the kernel streams the 2-bit planes and spends well under
// one instruction per trit on the decode:
//   * each lane streams 128-bit words of both planes of two rows straight into registers, with
//     the next 512-trit chunk in flight while the current one is decoded;
//   * one LOP3 pair + rotate merges a mask/sign word pair into 2-bit fields, and one shift + AND
//     per register turns them into int8 tensor-core operands holding 64*t (see tern_device.cuh);
//     the warp's 16 rows x 32 trits go through mma.sync s8 x s8, where the +-1 products are exact
//     (the add / skip / subtract rule, origotech.dev Figure I);
//   * the activation slice of the CTA is staged once in shared memory as int8 operand columns:
//     q itself (int8 mode), or four exact int8 limbs per token of a 30-bit fixed-point value
//     relative to 2^E, E from the absmax of the token's slice (bf16 mode; tern_device.cuh gives
//     the error bound); every decoded weight register is reused for all columns (n-groups);
//   * CTAs of one row block that split K form a thread-block cluster and add their partial sums
//     through distributed shared memory in rank order: no global scratch, deterministic results.
// All sums are exact integers: int8 mode ends with y = ((float)acc * s_x) * scale (two fp32
// round-to-nearest multiplies), bf16 mode combines limbs and K slices in fp64 and rounds once.
#include <atomic>
#include <cooperative_groups.h>
#include <cstdint>
#include <cuda_runtime.h>

#include "tern_device.cuh"
#include "tern_kernels.h"

namespace cg = cooperative_groups;

namespace tern {
namespace {

constexpr int kRows = 128;  // rows per CTA: 8 warps x 16 rows

__device__ __forceinline__ uint32_t u4get(const uint4& v, int e) {
  return e == 0 ? v.x : (e == 1 ? v.y : (e == 2 ? v.z : v.w));
}

// Operand columns of the staged slice: q of each token (int8 mode) or four limbs per token, top
// limb first (bf16 mode: column 4m + l).
__host__ __device__ inline int gemm_cols(int mode, int M) { return mode == 0 ? 4 * M : M; }
// Words per staged operand column: the slice's bytes plus 16 words of bank skew.
__host__ __device__ inline int gemm_col_words(int kr) { return kr / 4 + 16; }
// Word offset of 16-byte half v of a column (swizzled so that the quad's loads hit distinct banks).
__device__ __forceinline__ int gemm_half_ofs(int v) { return 4 * (v ^ ((v >> 3) & 3)); }

template <int MODE, int NG>
__global__ void __launch_bounds__(kThreads) k_tern_gemm(const GemmParams p) {
  extern __shared__ __align__(16) uint32_t smem[];
  __shared__ int expo[16];                         // bf16 mode: limb exponent of each token's slice
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
  const int ncols = gemm_cols(MODE, p.M);
  const int RS = gemm_col_words(p.kr);

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

  // ---- stage the activation slice X[:, k0 : k0 + kr) as int8 operand columns ---------------------
  const int per_row = p.kr >> 4;                            // 16-element halves of 32-trit blocks
  if (MODE == 1) {
    const int8_t* xs = static_cast<const int8_t*>(p.x);
    for (int i = threadIdx.x; i < p.M * per_row; i += kThreads) {
      const int m = i / per_row, v = i - m * per_row;
      const uint4 val = permute_i8_half(ld_nc(xs + (size_t)m * p.K + k0 + 16 * v));
      *reinterpret_cast<uint4*>(smem + m * RS + gemm_half_ofs(v)) = val;
    }
  } else {
    const uint16_t* xs = static_cast<const uint16_t*>(p.x);
    for (int m = warp; m < p.M; m += kThreads / 32) {
      float amax = 0.0f;
      for (int k = lane * 8; k < p.kr; k += 256) {
        const uint4 v = ld_nc(xs + (size_t)m * p.K + k0 + k);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e)
          amax = fmaxf(amax, fmaxf(fabsf(bf16_bits_to_float(w[e] & 0xFFFFu)), fabsf(bf16_bits_to_float(w[e] >> 16))));
      }
      for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
      if (lane == 0) expo[m] = limb_exponent(amax);
    }
    __syncthreads();
    for (int i = threadIdx.x; i < p.M * per_row; i += kThreads) {
      const int m = i / per_row, v = i - m * per_row;
      const int E = expo[m];
      const uint16_t* xb = xs + (size_t)m * p.K + k0 + 16 * v;
      const uint4 a = ld_nc(xb), b = ld_nc(xb + 8);
      const uint32_t wv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
      uint32_t l[4][4];
      limbs_of_bf16<4>(wv, E, l);
#pragma unroll
      for (int c = 0; c < 4; ++c)
        *reinterpret_cast<uint4*>(smem + (4 * m + c) * RS + gemm_half_ofs(v)) =
            permute_i8_half(make_uint4(l[c][0], l[c][1], l[c][2], l[c][3]));
    }
  }
  __syncthreads();

  int acc[NG][4];
#pragma unroll
  for (int n = 0; n < NG; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0;

  for (int c = 0; c < nchunks; ++c) {
    const bool live = (16 * c + 4 * t) < nw;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int w = 16 * c + 4 * t + e;                     // local word index of this lane
      uint32_t wa0, wb0, wa1, wb1;
      merge_planes(u4get(cur[0], e), u4get(cur[2], e), wa0, wb0);   // row ra
      merge_planes(u4get(cur[1], e), u4get(cur[3], e), wa1, wb1);   // row rb
      // the word's operand registers of both rows: 64 * t per byte
      const uint32_t A[8][2] = {
          {dec_i8<0>(wa0, wb0), dec_i8<0>(wa1, wb1)}, {dec_i8<1>(wa0, wb0), dec_i8<1>(wa1, wb1)},
          {dec_i8<2>(wa0, wb0), dec_i8<2>(wa1, wb1)}, {dec_i8<3>(wa0, wb0), dec_i8<3>(wa1, wb1)},
          {dec_i8<4>(wa0, wb0), dec_i8<4>(wa1, wb1)}, {dec_i8<5>(wa0, wb0), dec_i8<5>(wa1, wb1)},
          {dec_i8<6>(wa0, wb0), dec_i8<6>(wa1, wb1)}, {dec_i8<7>(wa0, wb0), dec_i8<7>(wa1, wb1)}};
#pragma unroll
      for (int n = 0; n < NG; ++n) {
        const int col = 8 * n + g;
        uint32_t xb[8];
        if (live && col < ncols) {
#pragma unroll
          for (int q = 0; q < 2; ++q) {
            const uint4 v = *reinterpret_cast<const uint4*>(smem + col * RS + gemm_half_ofs(2 * w + q));
            xb[4 * q] = v.x; xb[4 * q + 1] = v.y; xb[4 * q + 2] = v.z; xb[4 * q + 3] = v.w;
          }
        } else {
#pragma unroll
          for (int q = 0; q < 8; ++q) xb[q] = 0u;
        }
#pragma unroll
        for (int r = 0; r < 8; r += 2) mma_s8(acc[n], A[r][0], A[r][1], A[r + 1][0], A[r + 1][1], xb[r], xb[r + 1]);
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) cur[i] = nxt[i];
    load_chunk(c + 2, nxt);
  }
  pdl_launch_dependents();

  // ---- epilogue: exact sums (acc = 64 * sum), one rounding ----------------------------------------
  if (MODE == 1 && p.ksplit == 1) {
#pragma unroll
    for (int n = 0; n < NG; ++n)
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int m = 8 * n + 2 * t + (i & 1);
        const int row = row0 + g + 8 * (i >> 1);
        if (m < p.M && row < p.N) {
          const int sum = acc[n][i] >> 6;
          p.y[(size_t)m * p.N + row] = __fmul_rn(__fmul_rn(__int2float_rn(sum), p.sx[m]), f16_bits_to_float(p.scale[row]));
          if (p.acc) p.acc[(size_t)m * p.N + row] = sum;
        }
      }
    return;
  }
  // partial tile [kRows][8 * NG] in this CTA's shared memory, then (split K) a cluster-wide sum
  constexpr int kCols = 8 * NG;
  int* part = reinterpret_cast<int*>(smem + ncols * RS);
#pragma unroll
  for (int n = 0; n < NG; ++n)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int col = 8 * n + 2 * t + (i & 1);
      const int lrow = warp * 16 + g + 8 * (i >> 1);
      part[lrow * kCols + col] = acc[n][i] >> 6;
    }
  cg::cluster_group cluster = cg::this_cluster();
  if (p.ksplit > 1) cluster.sync(); else __syncthreads();
  const int rows_per_rank = kRows / p.ksplit;
  for (int i = threadIdx.x; i < rows_per_rank * p.M; i += kThreads) {
    const int lrow = ks * rows_per_rank + i / p.M, m = i % p.M;
    const int row = blockIdx.y * kRows + lrow;
    if (row >= p.N) continue;
    const float sc = f16_bits_to_float(p.scale[row]);
    if (MODE == 1) {
      int sum = 0;
      for (int r = 0; r < p.ksplit; ++r) sum += cluster.map_shared_rank(part, r)[lrow * kCols + m];
      p.y[(size_t)m * p.N + row] = __fmul_rn(__fmul_rn(__int2float_rn(sum), p.sx[m]), sc);
      if (p.acc) p.acc[(size_t)m * p.N + row] = sum;
    } else {
      double tot = 0.0;
      for (int r = 0; r < p.ksplit; ++r) {
        const int* rp = (p.ksplit > 1 ? cluster.map_shared_rank(part, r) : part) + lrow * kCols + 4 * m;
        const int E = (p.ksplit > 1 ? cluster.map_shared_rank(expo, r) : expo)[m];
        tot += ldexp((double)limb_combine(rp[0], rp[1], rp[2], rp[3]), E - kLimbFrac);
      }
      p.y[(size_t)m * p.N + row] = (float)(tot * (double)sc);
    }
  }
  if (p.ksplit > 1) cluster.sync();
}

template <int MODE, int NG>
cudaError_t launch_one(const GemmParams& p, size_t smem, bool pdl, cudaStream_t st) {
  auto kern = k_tern_gemm<MODE, NG>;
  static std::atomic<unsigned long long> smem_raised{0};
  cudaError_t e = allow_max_dynamic_smem(kern, smem_raised);
  if (e != cudaSuccess) return e;
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

template <int MODE>
cudaError_t launch_mode(const GemmParams& p, int ng, size_t smem, bool pdl, cudaStream_t st) {
  switch (ng) {
    case 1: return launch_one<MODE, 1>(p, smem, pdl, st);
    case 2: return launch_one<MODE, 2>(p, smem, pdl, st);
    case 3: return launch_one<MODE, 3>(p, smem, pdl, st);
    case 4: return launch_one<MODE, 4>(p, smem, pdl, st);
    case 5: return launch_one<MODE, 5>(p, smem, pdl, st);
    case 6: return launch_one<MODE, 6>(p, smem, pdl, st);
    case 7: return launch_one<MODE, 7>(p, smem, pdl, st);
    default: return launch_one<MODE, 8>(p, smem, pdl, st);
  }
}

}  // namespace

// Shared-memory bytes of one CTA: the operand columns of the activation slice and the partial tile.
size_t gemm_smem_bytes(int mode, int M, int kr) {
  const int ncols = gemm_cols(mode, M);
  const int ng = (ncols + 7) / 8;
  return (size_t)ncols * gemm_col_words(kr) * 4 + (size_t)kRows * 8 * ng * 4;
}

int gemm_rows_per_cta() { return kRows; }

cudaError_t launch_tern_gemm(const GemmParams& p, bool pdl, cudaStream_t st) {
  const int ng = (gemm_cols(p.mode, p.M) + 7) / 8;
  const size_t smem = gemm_smem_bytes(p.mode, p.M, p.kr);
  return p.mode == 0 ? launch_mode<0>(p, ng, smem, pdl, st) : launch_mode<1>(p, ng, smem, pdl, st);
}

}  // namespace tern
