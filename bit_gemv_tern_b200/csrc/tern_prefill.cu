// Prefill dense contraction on the 5th-generation tensor cores (tcgen05 + TMEM).
//
//   Y[m][n] = scale[n] * sum_k t[n][k] * X[m][k],   X bf16 [M][K], t packed ternary, Y fp32 [M][N]
//
// Prefill runs the same linear layers at M = prompt length ("batched prefill" of the PyTorchKR
// review "Fermion Research, 3진 계열 포맷으로 직접 학습한 Neutrino-1 모델군 3종 공개", section
// "실행해보기"), which makes the product a genuine dense contraction. The ternary weights stay
// packed in HBM and are expanded only inside the kernel, in shared memory, right before the
// tensor cores read them (weights packed at rest, aiatolah.com "Neutrino-1 8B: modelo ternario
// ...", second paragraph); the products by +-1 / 0 are exact (origotech.dev Figure I).
//
// One persistent CTA per SM walks output tiles of H x 128 tokens x BN = 256 weight rows:
//   warp 0      TMA producer: X tile (H x 128 x 64 bf16, 128-byte swizzle) per K stage;
//   warp 1      allocates 512 TMEM columns and one lane issues tcgen05.mma kind::f16 (A = X,
//               B = expanded weights, both K-major; M = 128 per instruction, one instruction per
//               128-token half); tcgen05.commit frees a stage when the MMAs reading it are done;
//   warps 2..9  expand the tile's 256 weight rows x 64 trits to bf16 (2.0 * t, the field decode
//               of tern_device.cuh) in the same swizzled layout the tensor core reads;
//   warps 10..13 epilogue: tcgen05.ld of the accumulator their TMEM lane quarter owns, times
//               0.5 * scale[n], stored to Y.
// H = 1: two 128 x 256 fp32 accumulators, so the next tile's MMAs run during the epilogue.
// H = 2: both halves of a 256-token tile read every expanded weight stage, which halves the
//        expansion work and cuts shared-memory traffic per flop by a sixth; the two halves' 128 x
//        256 accumulators fill TMEM, so the tensor core waits for each tile's epilogue. The host
//        takes H = 2 when its tiles still fill the GPU.
// Every mbarrier wait is bounded; a kernel that gives up latches TERN_ETIMEOUT, drains what it
// issued (bounded), frees its TMEM and returns.
#include <cstdint>
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "tern_device.cuh"
#include "tern_kernels.h"

namespace tern {

__device__ int g_prefill_latch = 0;

namespace {

constexpr int BM = 128;                          // tokens per MMA (tile half): UMMA M, TMEM lanes
constexpr int BN = 256;                          // weight rows per tile: UMMA N, accumulator columns
constexpr int BK = 64;                           // K per stage: one 128-byte swizzle span of bf16
constexpr int kHalfBytes = BM * BK * 2;          // 16 KB: one 128-token X tile of a stage
constexpr int kBBytes = BN * BK * 2;             // 32 KB
#ifndef TERN_PREFILL_DEC_WARPS
#define TERN_PREFILL_DEC_WARPS 8
#endif
constexpr int kDecWarps = TERN_PREFILL_DEC_WARPS, kEpiWarps = 4;
constexpr int kRowsPerDec = BN / (kDecWarps * 32);   // weight rows expanded per decoder thread
static_assert(kRowsPerDec * kDecWarps * 32 == BN, "decoder rows");
constexpr int kPrefillThreads = (2 + kDecWarps + kEpiWarps) * 32;
constexpr int kTmemCols = 2 * BN;                // two 128 x 256 fp32 accumulators
constexpr int kStageTile = 32 * 32 * 4;          // epilogue staging: 32 rows x 32 fp32 columns per warp
constexpr uint32_t kWaitTries = 1u << 13;
// Shape of the kernel for H 128-token halves per tile.
//   smem: [A stages][B stages][barriers + TMEM address][epilogue scales], stages 1024-byte aligned
template <int H>
struct Shape {
  static constexpr int kTileM = BM * H;                    // tokens per tile
  static constexpr int kStages = H == 1 ? 4 : 3;
  static constexpr int kABytes = H * kHalfBytes;
  static constexpr int kAccBufs = H == 1 ? 2 : 1;          // accumulator buffers (tiles in flight)
  static constexpr int kSmemA = 0;
  static constexpr int kSmemB = kStages * kABytes;
  static constexpr int kSmemBar = kSmemB + kStages * kBBytes;
  // + barriers, epilogue scales, epilogue staging tiles, alignment slack
  static constexpr int kSmemBytes = kSmemBar + 256 + kEpiWarps * BN * 4 + kEpiWarps * kStageTile + 1024;
  static_assert(kAccBufs * H * BN == kTmemCols, "TMEM columns");
};

// Instruction descriptor of tcgen05.mma kind::f16: fp32 accumulator, A and B bf16, both
// K-major, N = 256, M = 128.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                            ((uint32_t)(BM >> 4) << 24);

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
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
// Tiled 2-d tensor load (no multicast): box at (c0 = k, c1 = token).
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int c0, int c1, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void sts128(uint32_t a, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(x), "r"(y), "r"(z), "r"(w) : "memory");
}
__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a) : "memory");
  return v;
}
__device__ __forceinline__ uint4 ldg128(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}
// K-major, 128-byte-swizzled operand descriptor (sm_100 layout): start address, leading byte
// offset 16 (unused for swizzled K-major), stride byte offset 1024 (8 rows x 128 B), version 1,
// swizzle mode 2 (128 B).
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)(16u >> 4) << 16;
  d |= (uint64_t)(1024u >> 4) << 32;
  d |= (uint64_t)1u << 46;
  d |= (uint64_t)2u << 61;
  return d;
}
__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t accum) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n"
      ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum)
      : "memory");
}
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 consecutive fp32 accumulator columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// bf16 register A (0..15) of a merged word pair: trits 2A, 2A+1 of the 32-trit word as 2.0 * t.
template <int A>
__device__ __forceinline__ uint32_t dec2(uint32_t wa, uint32_t wb) {
  return dec_bf16<A>(wa, wb);
}

template <int H>
__global__ void __launch_bounds__(kPrefillThreads, 1) k_prefill(const __grid_constant__ PrefillParams p) {
  using SH = Shape<H>;
  constexpr int kStages = SH::kStages, kABytes = SH::kABytes, kTileM = SH::kTileM, kAccBufs = SH::kAccBufs;
  constexpr int kSmemA = SH::kSmemA, kSmemB = SH::kSmemB, kSmemBar = SH::kSmemBar;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte alignment for the swizzled tiles
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const uint32_t sA = base + kSmemA, sB = base + kSmemB, sBar = base + kSmemBar;
  const uint32_t a_full = sBar, b_full = sBar + 8 * kStages, empty = sBar + 16 * kStages;
  const uint32_t acc_full = sBar + 24 * kStages, acc_empty = acc_full + 16, done_bar = acc_empty + 16;
  const uint32_t tmem_slot = done_bar + 8;
  const uint32_t sScale = sBar + 256;                 // [4 epilogue warps][BN] floats
  const uint32_t sStage = sScale + kEpiWarps * BN * 4;  // [4 epilogue warps][32 rows][128 B]
  uint32_t* tmem_slot_ptr = reinterpret_cast<uint32_t*>(smem_raw + (tmem_slot - raw));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles_n = (p.N + BN - 1) / BN, tiles_m = (p.M + kTileM - 1) / kTileM;
  const int tiles = tiles_m * tiles_n;
  const int KT = p.K / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(a_full + 8 * s, 1);
      mbar_init(b_full + 8 * s, kDecWarps);
      mbar_init(empty + 8 * s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(acc_full + 8 * a, 1);
      mbar_init(acc_empty + 8 * a, kEpiWarps);
    }
    mbar_init(done_bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(tmem_slot), "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot_ptr;
  bool ok = true;

  if (warp == 0) {
    // ---------------- TMA producer: X tiles ----------------
    if (lane == 0) {
      int q = 0;
      for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
        const int mt = tile / tiles_n;
        for (int kt = 0; kt < KT; ++kt, ++q) {
          const int s = q % kStages;
          if (q >= kStages && !(ok = mbar_wait(empty + 8 * s, ((q / kStages) - 1) & 1))) break;
          mbar_arrive_expect_tx(a_full + 8 * s, kABytes);
          tma_load_2d(sA + s * kABytes, &p.xmap, kt * BK, mt * kTileM, a_full + 8 * s);
        }
      }
      // do not leave with copies in flight (bounded, also after a give-up)
      for (int r = q > kStages ? q - kStages : 0; r < q; ++r)
        if (!mbar_wait(a_full + 8 * (r % kStages), (r / kStages) & 1)) { ok = false; break; }
    }
  } else if (warp == 1) {
    // ---------------- MMA issue (one lane) ----------------
    if (lane == 0) {
      int q = 0, tl = 0;
      for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x, ++tl) {
        const int acc = tl % kAccBufs, use = tl / kAccBufs;
        if (use >= 1 && !(ok = mbar_wait(acc_empty + 8 * acc, (use - 1) & 1))) break;
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(acc * H * BN);
        for (int kt = 0; kt < KT; ++kt, ++q) {
          const int s = q % kStages;
          const uint32_t ph = (q / kStages) & 1;
          if (!(ok = mbar_wait(a_full + 8 * s, ph))) break;
          if (!(ok = mbar_wait(b_full + 8 * s, ph))) break;
          tc_fence_after();
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
#pragma unroll
            for (int h = 0; h < H; ++h)                 // every half reads the same weight stage
              umma_bf16(d + (uint32_t)(h * BN), umma_desc(sA + s * kABytes + h * kHalfBytes + 32 * k),
                        umma_desc(sB + s * kBBytes + 32 * k), kIdesc, (kt > 0 || k > 0) ? 1u : 0u);
          umma_commit(empty + 8 * s);                 // the stage is free once these MMAs are done
        }
        if (!ok) break;
        umma_commit(acc_full + 8 * acc);              // the accumulator is complete
      }
      // every MMA this thread issued has completed once done_bar flips
      umma_commit(done_bar);
      if (!mbar_wait(done_bar, 0)) ok = false;
    }
  } else if (warp < 2 + kDecWarps) {
    // ---------------- weight expansion: 256 rows x 64 trits -> bf16, swizzled ----------------
    const int d = threadIdx.x - 64;                   // rows d, d + 32 * kDecWarps, ... of the tile
    const int KW = p.K / 16;                          // words per row (both planes)
    int q = 0;
    for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
      const int nt = tile % tiles_n;
      const uint32_t* rowp[kRowsPerDec];
      bool live[kRowsPerDec];
#pragma unroll
      for (int h = 0; h < kRowsPerDec; ++h) {
        const int n = nt * BN + d + 32 * kDecWarps * h;
        live[h] = n < p.N;
        rowp[h] = p.planes + (size_t)(live[h] ? n : 0) * KW;
      }
      // 16-byte loads of each plane cover two stages (a pair); pairs are loaded two pairs ahead
      //   p0 = the pair being decoded, p1, p2 = the next two
      uint4 pm[3][kRowsPerDec], ps[3][kRowsPerDec];
#pragma unroll
      for (int j = 0; j < 3; ++j)
#pragma unroll
        for (int h = 0; h < kRowsPerDec; ++h) {
          const bool in = live[h] && 2 * j < KT;
          pm[j][h] = in ? ldg128(rowp[h] + 4 * j) : make_uint4(0u, 0u, 0u, 0u);
          ps[j][h] = in ? ldg128(rowp[h] + KW / 2 + 4 * j) : make_uint4(0u, 0u, 0u, 0u);
        }
      for (int kt = 0; kt < KT; ++kt, ++q) {
        const int s = q % kStages;
        uint2 cm[kRowsPerDec], cs[kRowsPerDec];
#pragma unroll
        for (int h = 0; h < kRowsPerDec; ++h) {
          cm[h] = (kt & 1) ? make_uint2(pm[0][h].z, pm[0][h].w) : make_uint2(pm[0][h].x, pm[0][h].y);
          cs[h] = (kt & 1) ? make_uint2(ps[0][h].z, ps[0][h].w) : make_uint2(ps[0][h].x, ps[0][h].y);
        }
        if (kt & 1) {                                    // pair done: shift the queue, fetch pair + 3
          const int j3 = (kt >> 1) + 3;
#pragma unroll
          for (int h = 0; h < kRowsPerDec; ++h) {
            pm[0][h] = pm[1][h]; pm[1][h] = pm[2][h];
            ps[0][h] = ps[1][h]; ps[1][h] = ps[2][h];
            const bool in = live[h] && 2 * j3 < KT;
            pm[2][h] = in ? ldg128(rowp[h] + 4 * j3) : make_uint4(0u, 0u, 0u, 0u);
            ps[2][h] = in ? ldg128(rowp[h] + KW / 2 + 4 * j3) : make_uint4(0u, 0u, 0u, 0u);
          }
        }
        if (q >= kStages && !(ok = mbar_wait(empty + 8 * s, ((q / kStages) - 1) & 1))) break;
        const uint32_t tileB = sB + s * kBBytes;
#pragma unroll
        for (int h = 0; h < kRowsPerDec; ++h) {
          const int r = d + 32 * kDecWarps * h;
          const uint32_t rowa = tileB + r * 128;
          const int sw = r & 7;
#pragma unroll
          for (int w = 0; w < 2; ++w) {
            uint32_t wa, wb;
            merge_planes(w ? cm[h].y : cm[h].x, w ? cs[h].y : cs[h].x, wa, wb);
            // 16-byte chunk c holds trits 8c .. 8c+7 of the stage: word w, registers 4(c%4) ..
            sts128(rowa + (((4 * w + 0) ^ sw) << 4), dec2<0>(wa, wb), dec2<1>(wa, wb), dec2<2>(wa, wb), dec2<3>(wa, wb));
            sts128(rowa + (((4 * w + 1) ^ sw) << 4), dec2<4>(wa, wb), dec2<5>(wa, wb), dec2<6>(wa, wb), dec2<7>(wa, wb));
            sts128(rowa + (((4 * w + 2) ^ sw) << 4), dec2<8>(wa, wb), dec2<9>(wa, wb), dec2<10>(wa, wb), dec2<11>(wa, wb));
            sts128(rowa + (((4 * w + 3) ^ sw) << 4), dec2<12>(wa, wb), dec2<13>(wa, wb), dec2<14>(wa, wb), dec2<15>(wa, wb));
          }
        }
        // generic-proxy writes -> visible to the tensor core (async proxy), then signal
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(b_full + 8 * s);
      }
    }
  } else {
    // ---------------- epilogue: TMEM -> registers -> 0.5 * scale -> Y ----------------
    const int quarter = warp & 3;                     // TMEM lanes 32*quarter .. +31
    // this warp's copy of 0.5 * scale[n] for the tile's columns (no cross-warp barrier)
    float* hs = reinterpret_cast<float*>(smem_raw + (sScale - raw)) + quarter * BN;
    int tl = 0;
    for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x, ++tl) {
      const int mt = tile / tiles_n, nt = tile % tiles_n;
      const int acc = tl % kAccBufs, use = tl / kAccBufs;
      __syncwarp();
#pragma unroll
      for (int i = 0; i < BN / 32; ++i) {
        const int n = nt * BN + lane + 32 * i;
        hs[lane + 32 * i] = n < p.N ? 0.5f * f16_bits_to_float(p.scale[n]) : 0.0f;
      }
      __syncwarp();
      if (!(ok = mbar_wait(acc_full + 8 * acc, use & 1))) break;
      tc_fence_after();
#pragma unroll 1
      for (int h = 0; h < H; ++h) {
        const int m = mt * kTileM + h * BM + quarter * 32 + lane;
        float* yrow = p.Y + (size_t)(m < p.M ? m : 0) * p.N;
#pragma unroll 1
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)((acc * H + h) * BN + 32 * c), r);
          const int n0 = nt * BN + 32 * c;
          const float* sc = hs + 32 * c;
          if (p.vec_store && n0 + 32 <= p.N) {
            // through this warp's staging tile (16-byte chunks swizzled by row, conflict-free both
            // ways), so that every store instruction writes four whole 128-byte rows of Y
            const uint32_t stg = sStage + (uint32_t)(quarter * kStageTile);
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const float4 s4 = *reinterpret_cast<const float4*>(sc + 4 * j);
              sts128(stg + lane * 128 + ((j ^ (lane & 7)) << 4), __float_as_uint(__uint_as_float(r[4 * j + 0]) * s4.x),
                     __float_as_uint(__uint_as_float(r[4 * j + 1]) * s4.y),
                     __float_as_uint(__uint_as_float(r[4 * j + 2]) * s4.z),
                     __float_as_uint(__uint_as_float(r[4 * j + 3]) * s4.w));
            }
            __syncwarp();
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const int rr = 4 * i + (lane >> 3), cj = lane & 7;
              const uint4 v = lds128(stg + rr * 128 + ((cj ^ (rr & 7)) << 4));
              const int mm = m - lane + rr;
              if (mm < p.M) *reinterpret_cast<uint4*>(p.Y + (size_t)mm * p.N + n0 + 4 * cj) = v;
            }
            __syncwarp();
          } else if (m < p.M) {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (n0 + j < p.N) yrow[n0 + j] = __uint_as_float(r[j]) * sc[j];
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty + 8 * acc);
    }
  }

  if (!ok) atomicExch(&g_prefill_latch, 5);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }
  return fn;
}

}  // namespace

bool plan_prefill(PrefillParams& p, const uint16_t* X, int& grid, size_t& smem) {
  if (p.M < 1 || p.N < 1 || p.K < BK || p.K % 128) return false;
  PFN_cuTensorMapEncodeTiled_v12000 encode = encode_fn();
  if (!encode) return false;
  // two 128-token halves per tile while such tiles still give every SM one (they halve the weight
  // expansion per flop); 128-token tiles otherwise
  const int tiles_n = (p.N + BN - 1) / BN;
  const int sms = device_sm_count();
  p.halves = (long long)((p.M + 2 * BM - 1) / (2 * BM)) * tiles_n >= sms ? 2 : 1;
  const int tile_m = BM * p.halves;
  const cuuint64_t dims[2] = {(cuuint64_t)p.K, (cuuint64_t)p.M};
  const cuuint64_t strides[1] = {(cuuint64_t)p.K * 2};
  const cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)tile_m};
  const cuuint32_t estr[2] = {1, 1};
  if (encode(&p.xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(X), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  const long long tiles = (long long)((p.M + tile_m - 1) / tile_m) * tiles_n;
  grid = tiles < sms ? (int)tiles : sms;
  smem = p.halves == 2 ? Shape<2>::kSmemBytes : Shape<1>::kSmemBytes;
  return true;
}

template <int H>
cudaError_t launch_prefill_h(const PrefillParams& p, int grid, size_t smem, cudaStream_t st) {
  static std::atomic<unsigned long long> smem_raised{0};
  cudaError_t e = allow_max_dynamic_smem(k_prefill<H>, smem_raised);
  if (e != cudaSuccess) return e;
  k_prefill<H><<<grid, kPrefillThreads, smem, st>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_prefill(const PrefillParams& p, int grid, size_t smem, cudaStream_t st) {
  return p.halves == 2 ? launch_prefill_h<2>(p, grid, smem, st) : launch_prefill_h<1>(p, grid, smem, st);
}

cudaError_t read_and_clear_prefill_latch(int* out) {
  cudaError_t e = cudaMemcpyFromSymbol(out, g_prefill_latch, sizeof(int));
  if (e != cudaSuccess) return e;
  const int zero = 0;
  return cudaMemcpyToSymbol(g_prefill_latch, &zero, sizeof(int));
}

}  // namespace tern
