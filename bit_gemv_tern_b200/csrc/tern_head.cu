// int8 output head with fused per-row scale and greedy argmax.
//
//   logits[m][v] = s_h[v] * sum_k W[v][k] * x[m][k],   argmax[m] = argmax_v logits[m][v]
//
// The head stays int8 (PyTorchKR review "Fermion Research, 3진 계열 포맷으로 직접 학습한
// Neutrino-1 모델군 3종 공개", section "3진 계열이라는 이름의 실체"), and the unembedding is the
// single step that runs at the DRAM roofline, 43% of a decode step's DRAM traffic (same review,
// section "뉴트리노 엔진"). Greedy decoding takes the argmax; independent implementations may differ
// on near ties (section "토큰 동일성의 경계"); here an exact tie goes to the lowest index.
//
// Design: int8 W rows feed mma.sync directly as the A operand (no decode at all); the activation
// is the B operand. int8 mode uses q from the per-token quantiser and is bit-exact. bf16 mode
// turns each bf16 x into four int8 limbs of a 30-bit fixed-point value relative to 2^E, E from the
// absmax of this CTA's K slice (exact for every x within 2^-23 of that absmax, rounding by at most
// 2^(E - 31) below it; see tern_device.cuh), so the products and the int32 sums stay exact; limbs
// and K slices are combined in fp64 before the single rounding to fp32. Limbs (and the M rows)
// occupy the eight columns of each tensor-core n-group, which for M = 1 come for free. CTAs splitting K form a
// cluster and add partial sums through distributed shared memory. The running maximum per row is
// kept as a packed (order-preserving value key, inverted index) 64-bit word, reduced with
// shared-memory and then global atomicMax; the last CTA to finish publishes the result and
// zero-fills the workspace again.
#include <atomic>
#include <cooperative_groups.h>
#include <cstdint>
#include <type_traits>
#include <cuda_runtime.h>

#include "tern_device.cuh"
#include "tern_kernels.h"

namespace cg = cooperative_groups;

namespace tern {
namespace {

constexpr int kHeadRows = 128;   // rows per row block: 8 warps x 16 rows

// BS: block-scaled weights (FV5B-style): one fp32 scale per row and 256-weight block instead of the
// fp16 row scale; the exact int32 sums of each block are scaled into fp64 accumulators.
// WE: one token and K whole in the CTA (the launcher checks both); each warp forms its own rows'
// logits (see the epilogue below).
template <int MODE, int NG, bool BS, bool WE = false>
__global__ void __launch_bounds__(kThreads, 2) k_head(const HeadParams p) {
  extern __shared__ __align__(16) uint32_t smem[];
  __shared__ unsigned long long best[16];
  __shared__ int expo[16];
  __shared__ int is_last;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int ks = blockIdx.x;
  const int k0 = ks * p.kr;
  const int ncols = MODE == 0 ? 4 * p.M : p.M;
  const int RS = p.kr / 4 + 4;             // words per staged activation column (+4: banks)
  const int nch = p.kr / 128;              // 128-byte chunks per row in this slice
  if (threadIdx.x < 16) best[threadIdx.x] = 0ull;

  // chunk c of a row block: 32 bytes of rows ra, rb at k0 + 128c + 32t
  const int8_t* pa = nullptr;
  const int8_t* pb = nullptr;
  bool warp_live = false;
  auto set_rows = [&](int rb) {
    const int row0 = rb * kHeadRows + warp * 16;
    warp_live = row0 < p.V;
    const int ra = min(row0 + g, p.V - 1), rbb = min(row0 + g + 8, p.V - 1);
    pa = p.W + (size_t)ra * p.K + k0 + 32 * t;
    pb = p.W + (size_t)rbb * p.K + k0 + 32 * t;
  };
  auto load_chunk = [&](int c, uint4 (&w)[4]) {
    if (warp_live && c < nch) {
      w[0] = ld_stream(pa + 128 * c);
      w[1] = ld_stream(pa + 128 * c + 16);
      w[2] = ld_stream(pb + 128 * c);
      w[3] = ld_stream(pb + 128 * c + 16);
    } else {
      w[0] = w[1] = w[2] = w[3] = make_uint4(0u, 0u, 0u, 0u);
    }
  };

  int rb = blockIdx.y;
  uint4 cur[4], nxt[4], nx2[4];                // three chunks of the warp's rows in flight
  set_rows(rb);
  // The first three chunks' weights: int8 mode issues them before the dependency wait; bf16 mode
  // once its activation staging (two passes over the K slice) has read its inputs, since issued
  // first they fill the memory queues and the staging waits behind them (0.6B head 28.7 -> 27.4
  // us in bf16 mode; int8 mode, with a plain copy to stage, is faster with them first).
  if (MODE == 1) {
    load_chunk(0, cur);
    load_chunk(1, nxt);
    load_chunk(2, nx2);
  }
  pdl_wait();

  // ---- stage activations: column c of the B operand holds K-slice bytes -------------------------
  if (MODE == 1) {
    const int8_t* xq = static_cast<const int8_t*>(p.x);
    const int per_row = p.kr / 16;
    for (int i = threadIdx.x; i < p.M * per_row; i += kThreads) {
      const int m = i / per_row, v = i - m * per_row;
      *reinterpret_cast<uint4*>(smem + m * RS + 4 * v) = ld_nc(xq + (size_t)m * p.K + k0 + 16 * v);
    }
  } else {
    const uint16_t* xb = static_cast<const uint16_t*>(p.x);
    for (int m = warp; m < p.M; m += kThreads / 32) {
      float amax = 0.0f;
      for (int k = lane * 8; k < p.kr; k += 256) {
        const uint4 v = ld_nc(xb + (size_t)m * p.K + k0 + k);
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e)
          amax = fmaxf(amax, fmaxf(fabsf(bf16_bits_to_float(w[e] & 0xFFFFu)), fabsf(bf16_bits_to_float(w[e] >> 16))));
      }
      for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
      if (lane == 0) expo[m] = limb_exponent(amax);
    }
    __syncthreads();
    const int per_row = p.kr / 8;
    for (int i = threadIdx.x; i < p.M * per_row; i += kThreads) {
      const int m = i / per_row, v = i - m * per_row;
      const int E = expo[m];
      const uint4 val = ld_nc(xb + (size_t)m * p.K + k0 + 8 * v);
      const uint32_t w[4] = {val.x, val.y, val.z, val.w};
      uint32_t l[4][2];
      limbs_of_bf16<2>(w, E, l);
#pragma unroll
      for (int c = 0; c < 4; ++c) *reinterpret_cast<uint2*>(smem + (4 * m + c) * RS + 2 * v) = make_uint2(l[c][0], l[c][1]);
    }
  }
  if (MODE == 0) {
    load_chunk(0, cur);
    load_chunk(1, nxt);
    load_chunk(2, nx2);
  }
  __syncthreads();

  // Let the next kernel of the chain get resident and start its own weight prefetch.
  pdl_launch_dependents();
  constexpr int kCols = 8 * NG;
  using PT = typename std::conditional<BS, double, int>::type;
  PT* part = reinterpret_cast<PT*>(smem + ncols * RS + (BS ? ((ncols * RS) & 1) : 0));
  cg::cluster_group cluster = cg::this_cluster();
  const int rows_per_rank = kHeadRows / p.ksplit;
  const int nblk = p.K >> 8;
  for (; rb < p.nrb; rb += p.nby) {
    int acc[NG][4];
#pragma unroll
    for (int n = 0; n < NG; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0;
    double Yb[BS ? NG : 1][4];
#pragma unroll
    for (int n = 0; n < (BS ? NG : 1); ++n) Yb[n][0] = Yb[n][1] = Yb[n][2] = Yb[n][3] = 0.0;
    const int brow0 = min(rb * kHeadRows + warp * 16 + g, p.V - 1), brow1 = min(rb * kHeadRows + warp * 16 + g + 8, p.V - 1);

    for (int c = 0; c < nch; ++c) {
#pragma unroll
      for (int n = 0; n < NG; ++n) {
        const int col = 8 * n + g;
        uint4 b0 = make_uint4(0u, 0u, 0u, 0u), b1 = b0;
        if (col < ncols) {
          const uint32_t* cp = smem + col * RS + 32 * c + 8 * t;
          b0 = *reinterpret_cast<const uint4*>(cp);
          b1 = *reinterpret_cast<const uint4*>(cp + 4);
        }
        // k-slots: lane t owns bytes [32t, 32t + 32) of the 128-byte chunk, four MMAs of 32.
        mma_s8(acc[n], cur[0].x, cur[2].x, cur[0].y, cur[2].y, b0.x, b0.y);
        mma_s8(acc[n], cur[0].z, cur[2].z, cur[0].w, cur[2].w, b0.z, b0.w);
        mma_s8(acc[n], cur[1].x, cur[3].x, cur[1].y, cur[3].y, b1.x, b1.y);
        mma_s8(acc[n], cur[1].z, cur[3].z, cur[1].w, cur[3].w, b1.z, b1.w);
      }
      if (BS && (c & 1)) {
        // a whole 256-weight block: its exact sums times the block's scale, into fp64
        const int blk = ((k0 + 128 * c) >> 8);
        const double s0 = (double)__ldg(p.bscale + (size_t)brow0 * nblk + blk);
        const double s1 = (double)__ldg(p.bscale + (size_t)brow1 * nblk + blk);
#pragma unroll
        for (int n = 0; n < (BS ? NG : 1); ++n)
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            Yb[n][i] += ((i >> 1) ? s1 : s0) * (double)acc[n][i];
            acc[n][i] = 0;
          }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        cur[i] = nxt[i];
        nxt[i] = nx2[i];
      }
      load_chunk(c + 3, nx2);
    }
    // the next row block's first chunks stream in while this block's outputs are formed
    if (rb + p.nby < p.nrb) {
      set_rows(rb + p.nby);
      load_chunk(0, cur);
      load_chunk(1, nxt);
      load_chunk(2, nx2);
    }

    if (WE) {
      // one token, K whole in this CTA: each warp forms its own 16 rows' logits from its
      // accumulators (lane t = 0 holds columns 0 and 1 of rows g and g + 8, lane t = 1 columns 2
      // and 3) and goes on to its next block without waiting for the other warps. The launcher
      // takes this for short rows only: measured, the 0.6B head (K = 1024) is 3-5% faster, while
      // at K = 4096 the block-synchronous epilogue below is faster.
      int w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) w[i] = __shfl_down_sync(0xFFFFFFFFu, acc[0][i], 1);
      if (t == 0) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int row = rb * kHeadRows + warp * 16 + g + 8 * h;
          if (row >= p.V) continue;
          const float shv = f16_bits_to_float(p.sh[row]);
          float logit;
          if (MODE == 1) {
            logit = __fmul_rn(__fmul_rn(__int2float_rn(acc[0][2 * h]), p.sx[0]), shv);
          } else {
            const long long D = limb_combine((long long)acc[0][2 * h], (long long)acc[0][2 * h + 1], (long long)w[2 * h],
                                             (long long)w[2 * h + 1]);
            logit = (float)(ldexp((double)D, expo[0] - kLimbFrac) * (double)shv);
          }
          if (p.logits) p.logits[row] = logit;
          const unsigned long long key =
              ((unsigned long long)float_order_key(logit) << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)row);
          atomicMax(&best[0], key);
        }
      }
      continue;
    }

    // partial sums of this K slice: part[local row][column]
#pragma unroll
    for (int n = 0; n < NG; ++n)
#pragma unroll
      for (int i = 0; i < 4; ++i)
        part[(warp * 16 + g + 8 * (i >> 1)) * kCols + 8 * n + 2 * t + (i & 1)] =
            BS ? (PT)Yb[BS ? n : 0][i] : (PT)acc[n][i];
    if (p.ksplit > 1) cluster.sync(); else __syncthreads();

    for (int i = threadIdx.x; i < rows_per_rank * p.M; i += kThreads) {
      const int lrow = ks * rows_per_rank + i / p.M, m = i % p.M;
      const int row = rb * kHeadRows + lrow;
      if (row >= p.V) continue;
      float logit;
      if (BS) {
        // the fp64 block-scaled sums of every K slice, then one rounding (int8 mode after * s_x)
        double tot = 0.0;
        for (int r = 0; r < p.ksplit; ++r) {
          const PT* rp = (p.ksplit > 1 ? cluster.map_shared_rank(part, r) : part) + lrow * kCols;
          if (MODE == 1) {
            tot += (double)rp[m];
          } else {
            const int E = (p.ksplit > 1 ? cluster.map_shared_rank(expo, r) : expo)[m];
            const PT* l = rp + 4 * m;
            tot += ldexp((((double)l[0] * 256.0 + (double)l[1]) * 256.0 + (double)l[2]) * 256.0 + (double)l[3],
                         E - kLimbFrac);
          }
        }
        logit = MODE == 1 ? (float)((double)p.sx[m] * tot) : (float)tot;
      } else if (MODE == 1) {
        const float shv = f16_bits_to_float(p.sh[row]);
        int a = 0;
        for (int r = 0; r < p.ksplit; ++r)
          a += (int)(p.ksplit > 1 ? cluster.map_shared_rank(part, r) : part)[lrow * kCols + m];
        logit = __fmul_rn(__fmul_rn(__int2float_rn(a), p.sx[m]), shv);
      } else {
        const float shv = f16_bits_to_float(p.sh[row]);
        double tot = 0.0;
        for (int r = 0; r < p.ksplit; ++r) {
          const PT* rp = (p.ksplit > 1 ? cluster.map_shared_rank(part, r) : part) + lrow * kCols + 4 * m;
          const int E = (p.ksplit > 1 ? cluster.map_shared_rank(expo, r) : expo)[m];
          const long long D = limb_combine((long long)rp[0], (long long)rp[1], (long long)rp[2], (long long)rp[3]);
          tot += ldexp((double)D, E - kLimbFrac);
        }
        logit = (float)(tot * (double)shv);
      }
      if (p.logits) p.logits[(size_t)m * p.V + row] = logit;
      const unsigned long long key =
          ((unsigned long long)float_order_key(logit) << 32) | (unsigned long long)(0xFFFFFFFFu - (uint32_t)row);
      atomicMax(&best[m], key);
    }
    if (p.ksplit > 1) cluster.sync(); else __syncthreads();
  }

  // ---- grid-wide argmax: global atomicMax, then the last CTA publishes and resets ----------------
  __syncthreads();
  if (threadIdx.x < p.M && best[threadIdx.x] != 0ull) atomicMax(&p.keys[threadIdx.x], best[threadIdx.x]);
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned int total = gridDim.x * gridDim.y;
    is_last = (atomicAdd(p.counter, 1u) == total - 1u);
  }
  __syncthreads();
  if (is_last) {
    __threadfence();
    if (threadIdx.x < p.M) {
      const unsigned long long key = atomicExch(&p.keys[threadIdx.x], 0ull);
      const int32_t idx = (int32_t)(0xFFFFFFFFu - (uint32_t)(key & 0xFFFFFFFFull));
      p.argmax[threadIdx.x] = idx;
      p.maxval[threadIdx.x] = float_from_order_key((uint32_t)(key >> 32));
      expo[threadIdx.x] = idx;                       // the winners, for the verify round below
    }
    if (threadIdx.x == 0) atomicExch(p.counter, 0u);
    if (p.accept) {
      // verify round: the longest prefix of drafts equal to the greedy tokens, then the target's
      // own next token (PyTorchKR review, section "검증된 추측 디코딩")
      __syncthreads();
      if (threadIdx.x == 0) {
        int n = 0;
        while (n < p.M - 1 && p.draft[n] == expo[n]) ++n;
        p.accept[0] = n;
        p.accept[1] = expo[n];
      }
    }
  }
}

// The acceptance rule alone, on argmax indices already on the device (one thread).
__global__ void k_verify_accept(const int32_t* argmax, const int32_t* draft, int32_t k, int32_t* accept) {
  pdl_wait();
  if (threadIdx.x == 0) {
    int n = 0;
    while (n < k && draft[n] == argmax[n]) ++n;
    accept[0] = n;
    accept[1] = argmax[n];
  }
}

template <int MODE, int NG, bool BS, bool WE = false>
cudaError_t launch_ng(const HeadParams& p, size_t smem, bool pdl, cudaStream_t st) {
  auto kern = k_head<MODE, NG, BS, WE>;
  static std::atomic<unsigned long long> smem_raised{0};
  cudaError_t e = allow_max_dynamic_smem(kern, smem_raised);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.ksplit, p.nby, 1);
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
cudaError_t launch_mode(const HeadParams& p, int ng, size_t smem, bool pdl, cudaStream_t st) {
  if (p.bscale) {
    switch (ng) {
      case 1: return launch_ng<MODE, 1, true>(p, smem, pdl, st);
      case 2: return launch_ng<MODE, 2, true>(p, smem, pdl, st);
      case 3: return launch_ng<MODE, 3, true>(p, smem, pdl, st);
      default: return launch_ng<MODE, 4, true>(p, smem, pdl, st);
    }
  }
  switch (ng) {
    case 1:
      if (p.M == 1 && p.ksplit == 1 && p.K <= 2048) return launch_ng<MODE, 1, false, true>(p, smem, pdl, st);
      return launch_ng<MODE, 1, false>(p, smem, pdl, st);
    case 2: return launch_ng<MODE, 2, false>(p, smem, pdl, st);
    case 3: return launch_ng<MODE, 3, false>(p, smem, pdl, st);
    case 4: return launch_ng<MODE, 4, false>(p, smem, pdl, st);
    case 5: return launch_ng<MODE, 5, false>(p, smem, pdl, st);
    case 6: return launch_ng<MODE, 6, false>(p, smem, pdl, st);
    case 7: return launch_ng<MODE, 7, false>(p, smem, pdl, st);
    default: return launch_ng<MODE, 8, false>(p, smem, pdl, st);
  }
}

}  // namespace

size_t head_workspace_bytes(int M) { return 16 + 8 * (size_t)M; }

cudaError_t launch_verify_accept(const int32_t* argmax, const int32_t* draft, int32_t k, int32_t* accept,
                                 cudaStream_t st) {
  k_verify_accept<<<1, 32, 0, st>>>(argmax, draft, k, accept);
  return cudaGetLastError();
}

size_t head_smem_bytes(int mode, int M, int kr, bool block_scaled) {
  const int ncols = mode == 0 ? 4 * M : M;
  const int ng = (ncols + 7) / 8;
  return (size_t)ncols * (kr / 4 + 4) * 4 + (block_scaled ? 8 : 0) +
         (size_t)kHeadRows * 8 * ng * (block_scaled ? 8 : 4);
}

cudaError_t launch_head(const HeadParams& p, bool pdl, cudaStream_t st) {
  const int ncols = p.mode == 0 ? 4 * p.M : p.M;
  const int ng = (ncols + 7) / 8;
  const size_t smem = head_smem_bytes(p.mode, p.M, p.kr, p.bscale != nullptr);
  return p.mode == 0 ? launch_mode<0>(p, ng, smem, pdl, st) : launch_mode<1>(p, ng, smem, pdl, st);
}

}  // namespace tern
