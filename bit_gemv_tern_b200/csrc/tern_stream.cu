// Persistent, TMA-fed ternary GEMV for M = 1 (decode), both activation modes.
//
//   y[n] = scale[n] * sum_k t[n][k] * x[k]
//
// At decode batch size the linear layers are bound by the bytes streamed per token (PyTorchKR
// review "Fermion Research, 3진 계열 포맷으로 직접 학습한 Neutrino-1 모델군 3종 공개", section
// "뉴트리노 엔진": tok/s_max = bandwidth / bytes per token), and the time above that floor sits in
// the ~120 kernel boundaries of a step and the dependency chains inside small kernels (same
// section). This kernel is built around that: one CTA per SM for the whole matrix, with
//   * a producer warp that streams the CTA's share of the packed planes through a ring of
//     shared-memory stages with cp.async.bulk (TMA) and mbarriers (one copy per row, rows padded
//     so the consumers' reads are bank-conflict free); it starts before the dependency wait, so
//     while the previous kernel of the chain is still running, the ring already fills;
//   * griddepcontrol.launch_dependents at entry, so the next kernel's CTA can become resident
//     next to this one and prefetch its own weights (programmatic dependent launch);
//   * 8 or 16 consumer warps that wait for the previous kernel only when they need the
//     activation, stage it once, then decode the merged 2-bit fields into u8 tensor-core operands
//     (one AND per register, see merge_planes_offset in tern_device.cuh) and run mma.sync u8 x s8
//     with four field accumulators;
//   * int8 mode: x = q (per-token int8), exact int32 sums; bf16 mode: x becomes four int8 limbs of
//     a 30-bit fixed-point value relative to 2^E (E from the absmax of the warp's K part; see
//     tern_device.cuh for the error bound), which sit in four columns of the n = 8 operand for free
//     at M = 1, so the products and sums stay exact integers and only the encoding and the final
//     fp64 -> fp32 conversion round;
//   * every wait on an mbarrier is bounded; on timeout the kernel latches TERN_ETIMEOUT in a
//     device word (read with tern_device_status), stops and returns.
#include <cstdint>
#include <cuda_runtime.h>

#include "tern_device.cuh"
#include "tern_kernels.h"

namespace tern {

__device__ int g_error_latch = 0;

namespace {

constexpr int kConsumerWarps = 8;   // warps per consumer group
constexpr uint32_t kWaitTries = 1u << 13;      // x ~0.5 ms suspend hint: seconds before giving up

// ---- mbarrier / bulk-copy primitives ------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
// Bounded wait for phase `parity` of an mbarrier: false after kWaitTries suspended polls.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
  for (uint32_t i = 0; i < kWaitTries; ++i) {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(done)
        : "r"(bar), "r"(parity), "r"(500000u)
        : "memory");
    if (done) return true;
  }
  return false;
}
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(dst), "l"(src), "r"(bytes), "r"(bar) : "memory");
}
__device__ __forceinline__ void latch_timeout() { atomicExch(&g_error_latch, 5); }

__device__ __forceinline__ uint32_t u4get(const uint4& v, int e) {
  return e == 0 ? v.x : (e == 1 ? v.y : (e == 2 ? v.z : v.w));
}

// ---- the kernel --------------------------------------------------------------------------------
// Stage = TS consecutive tiles of 16 rows x the full K: one contiguous range of the row-major planes,
// moved by a single bulk copy. The CW consumer warps form CW / 8 groups that take the stages in
// turn (several stages decode at once); within a group, warp j handles tile j / WPT of the stage and
// K part j % WPT (WPT = 8 / TS). A warp always has the same K part, so it stages only its own slice
// of x, and its int8 limbs (bf16 mode) take their exponent from that slice. With XREG (each part is
// exactly one 512-trit chunk) the warp's activation operands stay in registers for the whole
// kernel. A tile's WPT partial sums meet in a shared-memory slot; the last warp to add its part
// (shared-memory counter) finishes the tile, so no consumer ever waits for another one.
//
// Decode (see merge_planes_offset): each operand register is one AND of a merged word; field
// position i of every byte carries 4^i * (t + 2), so the four MMA chains are the four positions and
// a part's sum is  sum_i (acc_i >> 2i) - 2 * sum_k x_k  (exact integers).
//
// Activation words of a warp's part are stored so that lane t's eight operand words for word e of
// chunk c sit at ((4c + e) * 4 + t) * 8: the four lanes of a quarter-warp read 16 distinct banks.
template <int MODE, int CW, bool XREG>
__global__ void __launch_bounds__((CW + 1) * 32, 1) k_tern_stream(const StreamParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int NC = MODE == 0 ? 4 : 1;                           // activation columns (limbs or q)
  constexpr int NGRP = CW / 8;                                    // consumer groups
  const int S = p.stages, TS = p.ts, WPT = 8 / TS;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem);          // full[S], empty[S]
  const uint32_t full0 = smem_u32(bars), empty0 = full0 + 8 * S;
  int* expo = reinterpret_cast<int*>(smem + 256);               // [CW] limb exponent of each warp's part
  int* cnt = reinterpret_cast<int*>(smem + 512);                // [S][TS] arrival counters (<= 128)
  uint8_t* ring = smem + 1024;
  int* part = reinterpret_cast<int*>(ring + (size_t)S * p.stage_bytes);   // [S][8][16][NC]
  uint32_t* xs = reinterpret_cast<uint32_t*>(part + S * 8 * 16 * NC);      // [CW][NC][x_words]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int groups = (p.tiles + TS - 1) / TS;
  const int g0 = (int)((long long)groups * blockIdx.x / gridDim.x);
  const int g1 = (int)((long long)groups * (blockIdx.x + 1) / gridDim.x);
  const int n_units = g1 - g0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(full0 + 8 * i, 1);
      mbar_init(empty0 + 8 * i, 8);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  for (int i = threadIdx.x; i < S * TS; i += blockDim.x) cnt[i] = 0;
  __syncthreads();
  pdl_launch_dependents();

  const int KM = p.K >> 5;                 // words per plane per row
  const size_t row_bytes = (size_t)p.K / 4;
  if (warp == CW) {
    // ============================ producer: one bulk copy per stage ============================
    if (lane == 0) {
      bool ok = true;
      for (int u = 0; u < n_units; ++u) {
        const int s = u % S;
        if (u >= S && !(ok = mbar_wait(empty0 + 8 * s, ((u / S) - 1) & 1))) break;
        const int r0 = (g0 + u) * TS * 16;
        const uint32_t bytes = (uint32_t)(min(TS * 16, p.N - r0) * row_bytes);
        mbar_arrive_expect_tx(full0 + 8 * s, bytes);
        bulk_g2s(smem_u32(ring + (size_t)s * p.stage_bytes), p.planes + (size_t)r0 * (2 * KM), bytes, full0 + 8 * s);
      }
      if (!ok) latch_timeout();
      // Do not exit with copies in flight: wait (bounded) for the last stages issued.
      for (int u = n_units > S ? n_units - S : 0; u < n_units; ++u)
        if (!mbar_wait(full0 + 8 * (u % S), (u / S) & 1)) break;
    }
    return;
  }

  // ============================ consumers ============================
  const int g = lane >> 2, t = lane & 3;
  const int grp = warp >> 3, j = warp & 7;         // group, warp within the group
  const int tw = j / WPT, pw = j % WPT;            // tile within the stage, K part
  const int part_words = KM / WPT;                 // words per plane of this warp's K part (% 4 == 0)
  const int w0 = pw * part_words;                  // first word of the part
  const int nchunks = (part_words + 15) >> 4;
  uint32_t* xw = xs + warp * NC * p.x_words;       // this warp's activation columns

  pdl_wait();
  // ---- stage this warp's K part of x (permuted int8 operand words) and its column sums -------
  // 32-trit word w of the part -> slot ((w / 16) * 4 + w % 4) * 4 + (w % 16) / 4, eight words each.
  const int nhalf = part_words * 2;                // 16-byte halves of 32-trit blocks in the part
  auto slot_of = [](int v) {                       // v = 2 * w + half
    const int w = v >> 1;
    return ((((w >> 4) << 2) + (w & 3)) * 4 + ((w & 15) >> 2)) * 8 + 4 * (v & 1);
  };
  auto bsum = [](uint32_t w) {                     // sum of the four signed bytes of a word
    return __dp4a((int)w, 0x01010101, 0);
  };
  int xsum[NC];
#pragma unroll
  for (int c = 0; c < NC; ++c) xsum[c] = 0;
  if (MODE == 1) {
    const int8_t* xq = static_cast<const int8_t*>(p.x) + (size_t)w0 * 32;
    for (int v = lane; v < nhalf; v += 32) {
      const uint4 q = ld_nc(xq + 16 * v);
      xsum[0] += bsum(q.x) + bsum(q.y) + bsum(q.z) + bsum(q.w);
      *reinterpret_cast<uint4*>(xw + slot_of(v)) = permute_i8_half(q);
    }
  } else {
    const uint16_t* xb = static_cast<const uint16_t*>(p.x) + (size_t)w0 * 32;
    uint4 a = make_uint4(0u, 0u, 0u, 0u), b = a;     // this lane's 16 elements (one half), kept in registers
    float amax = 0.0f;
    const bool mine = lane < nhalf;                  // parts of at most 512 trits: one half per lane
    for (int v = lane; v < nhalf; v += 32) {
      const uint4 a2 = ld_nc(xb + 16 * v), b2 = ld_nc(xb + 16 * v + 8);
      if (v == lane) { a = a2; b = b2; }
      const uint32_t wv[8] = {a2.x, a2.y, a2.z, a2.w, b2.x, b2.y, b2.z, b2.w};
#pragma unroll
      for (int e = 0; e < 8; ++e)
        amax = fmaxf(amax, fmaxf(fabsf(bf16_bits_to_float(wv[e] & 0xFFFFu)), fabsf(bf16_bits_to_float(wv[e] >> 16))));
    }
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    const int E = limb_exponent(amax);
    if (lane == 0) expo[warp] = E;
    for (int v = lane; v < nhalf; v += 32) {
      uint4 a2 = a, b2 = b;
      if (!(mine && v == lane)) { a2 = ld_nc(xb + 16 * v); b2 = ld_nc(xb + 16 * v + 8); }
      const uint32_t wv[8] = {a2.x, a2.y, a2.z, a2.w, b2.x, b2.y, b2.z, b2.w};
      uint32_t l[4][4];
      limbs_of_bf16<4>(wv, E, l);
      const int o = slot_of(v);
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        xsum[c] += bsum(l[c][0]) + bsum(l[c][1]) + bsum(l[c][2]) + bsum(l[c][3]);
        *reinterpret_cast<uint4*>(xw + c * p.x_words + o) = permute_i8_half(make_uint4(l[c][0], l[c][1], l[c][2], l[c][3]));
      }
    }
  }
#pragma unroll
  for (int c = 0; c < NC; ++c)
    for (int o = 16; o > 0; o >>= 1) xsum[c] += __shfl_xor_sync(0xFFFFFFFFu, xsum[c], o);
  __syncwarp();
  // offset of this lane's two accumulator columns (2t, 2t + 1): 2 * sum_k x_k of that column
  int corr[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int col = 2 * t + h;
    int v = 0;
#pragma unroll
    for (int c = 0; c < NC; ++c) v = (c == col) ? xsum[c] : v;
    corr[h] = 2 * v;
  }

  // activation operands: registers (one chunk per warp) or the staged shared-memory words
  const bool has_x = g < NC;
  const uint32_t* xl = xw + (has_x ? g : 0) * p.x_words + t * 8;
  uint32_t xr[XREG ? 4 : 1][8];
  if constexpr (XREG) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint4 x0 = *reinterpret_cast<const uint4*>(xl + e * 32);
      const uint4 x1 = *reinterpret_cast<const uint4*>(xl + e * 32 + 4);
      xr[e][0] = x0.x; xr[e][1] = x0.y; xr[e][2] = x0.z; xr[e][3] = x0.w;
      xr[e][4] = x1.x; xr[e][5] = x1.y; xr[e][6] = x1.z; xr[e][7] = x1.w;
    }
  }

  // ---- main loop: this group's stages ----------------------------------------------------------
  bool ok = true;
  const int row_w = 2 * KM;                        // words per staged row
  for (int u = grp; u < n_units && ok; u += NGRP) {
    const int s = u % S;
    if (!(ok = mbar_wait(full0 + 8 * s, (u / S) & 1))) break;
    const uint32_t* st = reinterpret_cast<const uint32_t*>(ring + (size_t)s * p.stage_bytes);
    const uint32_t* ra = st + (tw * 16 + g) * row_w + w0 + 4 * t;
    const uint32_t* rb = ra + 8 * row_w;
    int acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a) acc[a][0] = acc[a][1] = acc[a][2] = acc[a][3] = 0;
    for (int c = 0; c < (XREG ? 1 : nchunks); ++c) {
      const bool live = XREG || (16 * c + 4 * t) < part_words;
      uint4 ma = make_uint4(0u, 0u, 0u, 0u), mb = ma, sa = ma, sb = ma;
      if (live) {
        ma = *reinterpret_cast<const uint4*>(ra + 16 * c);
        mb = *reinterpret_cast<const uint4*>(rb + 16 * c);
        sa = *reinterpret_cast<const uint4*>(ra + KM + 16 * c);
        sb = *reinterpret_cast<const uint4*>(rb + KM + 16 * c);
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        uint32_t xb[8];
        if constexpr (XREG) {
#pragma unroll
          for (int q = 0; q < 8; ++q) xb[q] = xr[e][q];
        } else {
          uint4 x0 = make_uint4(0u, 0u, 0u, 0u), x1 = x0;
          if (live) {
            x0 = *reinterpret_cast<const uint4*>(xl + c * 128 + e * 32);
            x1 = *reinterpret_cast<const uint4*>(xl + c * 128 + e * 32 + 4);
          }
          xb[0] = x0.x; xb[1] = x0.y; xb[2] = x0.z; xb[3] = x0.w;
          xb[4] = x1.x; xb[5] = x1.y; xb[6] = x1.z; xb[7] = x1.w;
        }
        uint32_t wa0, wb0, wa1, wb1;
        merge_planes_offset(u4get(ma, e), u4get(sa, e), wa0, wb0);
        merge_planes_offset(u4get(mb, e), u4get(sb, e), wa1, wb1);
        if (!live) wa0 = wb0 = wa1 = wb1 = 0u;                 // no data: contributes nothing
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint32_t M = 0x03030303u << (2 * i);
          mma_u8s8(acc[i], wa0 & M, wa1 & M, wb0 & M, wb1 & M, xb[i], xb[4 + i]);
        }
      }
    }
    // ---- this warp's partial for the tile; the last of its WPT warps finishes the tile ---------
    int* slot = part + (s * 8 + j) * 16 * NC;
    if (t < (NC + 1) / 2) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int col = 2 * t + (q & 1);
        if (col < NC)
          slot[(g + 8 * (q >> 1)) * NC + col] =
              acc[0][q] + (acc[1][q] >> 2) + (acc[2][q] >> 4) + (acc[3][q] >> 6) - corr[q & 1];
      }
    }
    __syncwarp();
    int last = 0;
    if (lane == 0) {
      __threadfence_block();
      last = atomicAdd(&cnt[s * TS + tw], 1) == WPT - 1;
    }
    last = __shfl_sync(0xFFFFFFFFu, last, 0);
    if (last) {
      __threadfence_block();
      const int row = (g0 + u) * TS * 16 + tw * 16 + lane;
      if (lane < 16 && row < p.N) {
        const int* base = part + (s * 8 + tw * WPT) * 16 * NC + lane * NC;
        const float sc = f16_bits_to_float(p.scale[row]);
        float y;
        if (MODE == 1) {
          int sum = 0;
          for (int q = 0; q < WPT; ++q) sum += base[q * 16 * NC];
          y = __fmul_rn(__fmul_rn(__int2float_rn(sum), p.sx[0]), sc);
          if (p.acc) p.acc[row] = sum;
        } else {
          double tot = 0.0;
          for (int q = 0; q < WPT; ++q) {
            const int* b = base + q * 16 * NC;
            const long long D = limb_combine(b[0], b[1], b[2], b[3]);
            tot += ldexp((double)D, expo[grp * 8 + tw * WPT + q] - kLimbFrac);
          }
          y = (float)(tot * (double)sc);
        }
        p.y[row] = y;
      }
      __syncwarp();
      if (lane == 0) cnt[s * TS + tw] = 0;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty0 + 8 * s);             // stage read; slot and counter reusable
  }
  if (!ok && lane == 0) latch_timeout();
}

}  // namespace

// Stage plan: a stage is TS whole tiles (16 rows x K) in one bulk copy; WPT = 8 / TS consumer
// warps split each tile's K into parts of whole 128-trit groups. Preference: parts of whole
// 512-trit chunks (no idle lanes), then stages of at least 8 KB, then fewer tiles per stage.
bool plan_stream(int N, int K, int mode, StreamParams& p, size_t& smem) {
  const int units = K / 128;
  if (p.cw != 8 && p.cw != 16) p.cw = 16;
  int best_ts = 0, best_score = -1;
  for (int ts = 1; ts <= kConsumerWarps; ts <<= 1) {
    const int wpt = kConsumerWarps / ts;
    if (units % wpt) continue;
    const long long bytes = (long long)ts * 16 * K / 4;
    if (bytes > 56 * 1024) continue;
    const int part_words = units * 4 / wpt;
    const int score = (part_words % 16 == 0 ? 4 : 0) + (bytes >= 8 * 1024 ? 2 : 0);
    if (score > best_score) { best_score = score; best_ts = ts; }
  }
  if (!best_ts) return false;
  p.N = N;
  p.K = K;
  p.ts = best_ts;
  p.stage_bytes = best_ts * 16 * (K / 4);
  p.tiles = (N + 15) / 16;
  const int nc = mode == 0 ? 4 : 1;
  const int wpt = kConsumerWarps / best_ts;
  const int part_words = K / 32 / wpt;
  p.x_words = ((part_words + 15) / 16) * 128 + 4;  // whole chunks of one K part (+4 words: banks)
  const size_t x_bytes = (size_t)p.cw * nc * p.x_words * 4;
  const size_t budget = p.cw == 8 ? 110 * 1024 : 200 * 1024;
  int stages = 0;
  for (int s = 16; s >= 2; --s) {
    const size_t need = 1024 + (size_t)s * p.stage_bytes + (size_t)s * 8 * 16 * nc * 4 + x_bytes;
    if (need <= budget) { stages = s; break; }
  }
  if (!stages) stages = 2;
  p.stages = stages;
  smem = 1024 + (size_t)stages * p.stage_bytes + (size_t)stages * 8 * 16 * nc * 4 + x_bytes;
  p.mode = mode;
  p.ks = K;
  p.pitch = K / 4;
  return smem <= 200 * 1024;
}

template <int MODE, int CW, bool XREG>
cudaError_t launch_cw(const cudaLaunchConfig_t& cfg0, const StreamParams& p, size_t smem) {
  static std::atomic<unsigned long long> smem_raised{0};
  cudaError_t e = allow_max_dynamic_smem(k_tern_stream<MODE, CW, XREG>, smem_raised);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = cfg0;
  cfg.blockDim = dim3((CW + 1) * 32, 1, 1);
  return cudaLaunchKernelEx(&cfg, k_tern_stream<MODE, CW, XREG>, p);
}

template <int MODE, bool XREG>
cudaError_t launch_x(const cudaLaunchConfig_t& cfg, const StreamParams& p, size_t smem) {
  return p.cw == 8 ? launch_cw<MODE, 8, XREG>(cfg, p, smem) : launch_cw<MODE, 16, XREG>(cfg, p, smem);
}

cudaError_t launch_stream(const StreamParams& p, size_t smem, bool pdl, cudaStream_t st) {
  const int groups = (p.tiles + p.ts - 1) / p.ts;
  const int sms = device_sm_count();
  const int grid = groups < sms ? groups : sms;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  int na = 0;
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  const bool xreg = (p.K / 32) / (8 / p.ts) == 16;          // one 512-trit chunk per warp
  if (p.mode == 0) return xreg ? launch_x<0, true>(cfg, p, smem) : launch_x<0, false>(cfg, p, smem);
  return xreg ? launch_x<1, true>(cfg, p, smem) : launch_x<1, false>(cfg, p, smem);
}

cudaError_t read_and_clear_error_latch(int* out, cudaStream_t st) {
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return e;
  e = cudaMemcpyFromSymbol(out, g_error_latch, sizeof(int));
  if (e != cudaSuccess) return e;
  const int zero = 0;
  return cudaMemcpyToSymbol(g_error_latch, &zero, sizeof(int));
}

}  // namespace tern
