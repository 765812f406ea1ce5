// Batched M = 1 ternary GEMV: a whole list of linear layers in two launches.
//
//   for every item i:  y_i[n] = scale_i[n] * sum_k t_i[n][k] * x_i[k]
//
// A decode step streams every weight of the stack once per token (PyTorchKR review "Fermion
// Research, 3진 계열 포맷으로 직접 학습한 Neutrino-1 모델군 3종 공개", section "뉴트리노 엔진":
// tok/s_max = memory bandwidth / bytes per token); the same section measures most of the time above
// that floor at the ~120 kernel boundaries of a step. Here the boundaries are gone: one persistent
// launch walks all items, so the weight stream never pauses between layers.
//
//   1. k_batch_prep (one CTA per item) turns each activation into ready-to-load tensor-core operand
//      blocks: int8 q permuted to the decode's byte order (int8 mode), or three exact int8 limbs of
//      a 22-bit fixed-point value relative to 2^E with E from the item's absmax (bf16 mode), plus
//      the per-part column sums that remove the decode offset.
//   2. k_batch_stream (one CTA per SM) splits the list's tile groups evenly by bytes. Its producer
//      warp streams, in order, each item's operand block into a double buffer and each stage of
//      weights (TS whole tiles of 16 rows x K, one contiguous cp.async.bulk) into a ring of S
//      stages. 12 consumer warps walk the stages in order; each warp handles 2 of the stage's 24
//      (tile, 512-trit K part) pairs: decode (one AND per operand register, see
//      tern_device.cuh), mma.sync u8 x s8, add the part into the tile's shared-memory accumulator
//      with integer atomics; the warp that completes a tile writes its outputs.
// All sums are exact integers; int8 mode ends with y = ((float)acc * s_x) * scale (two fp32
// round-to-nearest multiplies), bf16 mode with one fp64 -> fp32 rounding. Every mbarrier wait is
// bounded and latches TERN_ETIMEOUT on give-up.
#include <cstdint>
#include <cuda_runtime.h>

#include "tern_device.cuh"
#include "tern_kernels.h"

namespace tern {

// Set to TERN_ETIMEOUT (5) when a bounded wait of the batched kernels gives up.
__device__ int g_batch_latch = 0;

namespace {

constexpr int kCW = 12;                               // consumer warps (one group, in unit order)
constexpr int kBatchThreads = (kCW + 1) * 32;
constexpr uint32_t kWaitTries = 1u << 13;
constexpr int kLimbFrac = 22;

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
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(dst), "l"(src), "r"(bytes), "r"(bar) : "memory");
}
__device__ __forceinline__ uint32_t u4get(const uint4& v, int e) {
  return e == 0 ? v.x : (e == 1 ? v.y : (e == 2 ? v.z : v.w));
}
__device__ __forceinline__ int bsum(uint32_t w) { return __dp4a((int)w, 0x01010101, 0); }

// Operand slot of 16-byte half h of word w (0..15) of a 512-trit part: lane t = w / 4 reads the
// eight words of its word e = w % 4 at ((e * 4) + t) * 8, so a quarter-warp's loads hit distinct banks.
__device__ __forceinline__ int part_slot(int w, int h) { return ((w & 3) * 4 + (w >> 2)) * 8 + 4 * h; }

// ---------------------------------------------------------------------------------------------
// prep: one CTA per item
__global__ void __launch_bounds__(256) k_batch_prep(const BatchParams p) {
  const BatchItem& it = p.items[blockIdx.x];
  uint32_t* blk = reinterpret_cast<uint32_t*>(p.xprep + it.xoff);
  const int K = it.K, KP = it.kp, NC = p.nc;
  const int xcw = KP * 128 + 4;                      // words per column
  int* meta = reinterpret_cast<int*>(blk + NC * xcw);  // [KP][NC] sums, then E
  __shared__ float red[8];
  __shared__ int sums[24 * 3];
  __shared__ int Esh;
  pdl_wait();
  for (int i = threadIdx.x; i < NC * xcw; i += blockDim.x) blk[i] = 0u;
  for (int i = threadIdx.x; i < KP * NC; i += blockDim.x) sums[i] = 0;
  float f = 1.0f;
  if (p.mode == 0) {
    const uint16_t* xb = static_cast<const uint16_t*>(it.x);
    float amax = 0.0f;
    for (int k = threadIdx.x * 8; k < K; k += blockDim.x * 8) {
      const uint4 v = ld_nc(xb + k);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e)
        amax = fmaxf(amax, fmaxf(fabsf(bf16_bits_to_float(w[e] & 0xFFFFu)), fabsf(bf16_bits_to_float(w[e] >> 16))));
    }
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
    __syncthreads();
    if (threadIdx.x == 0) {
      float m = red[0];
      for (int i = 1; i < 8; ++i) m = fmaxf(m, red[i]);
      int E = 0;
      if (m > 0.0f) {
        frexpf(m, &E);                               // m < 2^E
        E = max(E, -100);
      }
      Esh = E;
    }
    __syncthreads();
    f = ldexpf(1.0f, kLimbFrac - Esh);
  }
  __syncthreads();
  // one 16-element half of a 32-trit word per thread iteration
  for (int v = threadIdx.x; v < K / 16; v += blockDim.x) {
    const int word = v >> 1, h = v & 1;              // global word index and half
    const int part = word >> 4, w = word & 15;
    const int slot = part * 128 + part_slot(w, h);
    if (p.mode == 1) {
      const uint4 q = ld_nc(static_cast<const int8_t*>(it.x) + 16 * v);
      atomicAdd(&sums[part], bsum(q.x) + bsum(q.y) + bsum(q.z) + bsum(q.w));
      *reinterpret_cast<uint4*>(blk + slot) = permute_i8_half(q);
    } else {
      const uint16_t* xb = static_cast<const uint16_t*>(it.x) + 16 * v;
      const uint4 a = ld_nc(xb), b = ld_nc(xb + 8);
      const uint32_t wv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
      uint32_t l[3][4] = {};
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const uint32_t bits = (e & 1) ? (wv[e >> 1] >> 16) : (wv[e >> 1] & 0xFFFFu);
        const int X = __float2int_rn(bf16_bits_to_float(bits) * f);   // exact power-of-two scaling
        const int L0 = (int)(int8_t)(X & 0xFF);
        const int X1 = (X - L0) >> 8;
        const int L1 = (int)(int8_t)(X1 & 0xFF);
        const int L2 = (X1 - L1) >> 8;                                 // |L2| <= 64
        const int sh = 8 * (e & 3);
        l[0][e >> 2] |= (uint32_t)(uint8_t)L2 << sh;
        l[1][e >> 2] |= (uint32_t)(uint8_t)L1 << sh;
        l[2][e >> 2] |= (uint32_t)(uint8_t)L0 << sh;
      }
#pragma unroll
      for (int c = 0; c < 3; ++c) {
        atomicAdd(&sums[part * 3 + c], bsum(l[c][0]) + bsum(l[c][1]) + bsum(l[c][2]) + bsum(l[c][3]));
        *reinterpret_cast<uint4*>(blk + c * xcw + slot) = permute_i8_half(make_uint4(l[c][0], l[c][1], l[c][2], l[c][3]));
      }
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < KP * NC; i += blockDim.x) meta[i] = sums[i];
  if (threadIdx.x == 0) meta[KP * NC] = p.mode == 0 ? Esh : 0;
  pdl_launch_dependents();
}

// ---------------------------------------------------------------------------------------------
template <int MODE>
__global__ void __launch_bounds__(kBatchThreads, 1) k_batch_stream(const BatchParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int NC = MODE == 0 ? 3 : 1;
  const int S = p.stages;
  // layout: [bars 512 B][tile counters 512 B][ring S x slot][x buffers 2 x xslot][tile acc S x 12 x 16 x NC]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
  const uint32_t full0 = smem_u32(bars);                  // [S]
  const uint32_t empty0 = full0 + 8 * S;                  // [S]
  const uint32_t xfull0 = empty0 + 8 * S;                 // [2]
  const uint32_t xempty0 = xfull0 + 16;                   // [2]
  int* cnt = reinterpret_cast<int*>(smem + 512);          // [S][12]
  uint8_t* ring = smem + 1024;
  uint8_t* xbuf = ring + (size_t)S * p.stage_slot_bytes;
  int* tacc = reinterpret_cast<int*>(xbuf + 2 * (size_t)p.x_slot_bytes);   // [S][12][16][NC]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int u0 = p.cta_unit[blockIdx.x], u1 = p.cta_unit[blockIdx.x + 1];
  const int n = u1 - u0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(full0 + 8 * i, 1);
      mbar_init(empty0 + 8 * i, kCW);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(xfull0 + 8 * b, 1);
      mbar_init(xempty0 + 8 * b, kCW);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  for (int i = threadIdx.x; i < S * 12; i += blockDim.x) cnt[i] = 0;
  for (int i = threadIdx.x; i < S * 12 * 16 * NC; i += blockDim.x) tacc[i] = 0;
  __syncthreads();
  pdl_launch_dependents();
  if (n <= 0) return;

  // item of the first unit
  int first_item = 0;
  while (first_item + 1 < p.count && p.items[first_item + 1].unit0 <= u0) ++first_item;

  if (warp == kCW) {
    // ====================== producer (lane 0) ======================
    if (lane != 0) return;
    bool ok = true;
    auto issue_weights = [&](int lu, int it) -> bool {
      const int s = lu % S;
      if (lu >= S && !mbar_wait(empty0 + 8 * s, ((lu / S) - 1) & 1)) return false;
      const BatchItem& b = p.items[it];
      const int grp = (u0 + lu) - b.unit0;
      const int r0 = grp * b.ts * 16;
      const uint32_t row_bytes = (uint32_t)b.K / 4;
      const uint32_t bytes = (uint32_t)min(b.ts * 16, b.N - r0) * row_bytes;
      mbar_arrive_expect_tx(full0 + 8 * s, bytes);
      bulk_g2s(smem_u32(ring + (size_t)s * p.stage_slot_bytes), b.planes + (size_t)r0 * (b.K / 16), bytes, full0 + 8 * s);
      return true;
    };
    // weights of the first stages do not depend on earlier kernels: start them before the wait
    int it = first_item;
    const int pre = n < S ? n : S;
    for (int lu = 0; lu < pre && ok; ++lu) {
      while (it + 1 < p.count && p.items[it + 1].unit0 <= u0 + lu) ++it;
      ok = issue_weights(lu, it);
    }
    pdl_wait();
    it = first_item;
    int seq = -1;                                         // item sequence number in this CTA
    for (int lu = 0; lu < n && ok; ++lu) {
      int it_new = it;
      while (it_new + 1 < p.count && p.items[it_new + 1].unit0 <= u0 + lu) ++it_new;
      if (lu == 0 || it_new != it) {
        it = it_new;
        ++seq;
        const int b = seq & 1;
        if (seq >= 2 && !(ok = mbar_wait(xempty0 + 8 * b, ((seq >> 1) - 1) & 1))) break;
        const uint32_t bytes = (uint32_t)p.items[it].xbytes;
        mbar_arrive_expect_tx(xfull0 + 8 * b, bytes);
        bulk_g2s(smem_u32(xbuf + (size_t)b * p.x_slot_bytes), p.xprep + p.items[it].xoff, bytes, xfull0 + 8 * b);
      }
      if (lu >= pre) ok = issue_weights(lu, it);
    }
    if (!ok) atomicExch(&g_batch_latch, 5);
    // do not exit with copies in flight
    for (int lu = n > S ? n - S : 0; lu < n; ++lu)
      if (!mbar_wait(full0 + 8 * (lu % S), (lu / S) & 1)) break;
    return;
  }

  // ====================== consumers ======================
  const int g = lane >> 2, t = lane & 3;
  const int j = warp;
  bool ok = true;
  int it = first_item, seq = 0, released = 0, acquired = -1;
  // Release of an item's operand buffer: every warp arrives once per item, in item order (all warps
  // see every unit), so item q's arrivals never mix with item q - 2's on the same barrier.
  for (int lu = 0; lu < n && ok; ++lu) {
    // item of this unit and its sequence number
    while (it + 1 < p.count && p.items[it + 1].unit0 <= u0 + lu) {
      ++it;
      ++seq;
    }
    for (; released < seq; ++released) {                 // items this warp has passed
      __syncwarp();
      if (lane == 0) mbar_arrive(xempty0 + 8 * (released & 1));
    }
    if (acquired != seq) {
      if (!(ok = mbar_wait(xfull0 + 8 * (seq & 1), (seq >> 1) & 1))) break;
      acquired = seq;
    }
    const int s = lu % S;
    if (!(ok = mbar_wait(full0 + 8 * s, (lu / S) & 1))) break;
    const BatchItem& B = p.items[it];
    const int KM = B.K >> 5, KP = B.kp, TS = B.ts;
    const int grp_idx = (u0 + lu) - B.unit0;
    const int xcw = KP * 128 + 4;
    const uint32_t* xb_base = reinterpret_cast<const uint32_t*>(xbuf + (size_t)(seq & 1) * p.x_slot_bytes);
    const int* meta = reinterpret_cast<const int*>(xb_base + NC * xcw);
    const uint32_t* st = reinterpret_cast<const uint32_t*>(ring + (size_t)s * p.stage_slot_bytes);
    const int row_w = 2 * KM;
    const int pairs = TS * KP;
    int* acc_s = tacc + s * 12 * 16 * NC;
    int* cnt_s = cnt + s * 12;
    for (int pr = j; pr < pairs; pr += kCW) {
      const int tile = pr / KP, part = pr - tile * KP;
      const int wbase = part * 16 + 4 * t;                // first word of this lane in the part
      const bool live = wbase < KM;
      const uint32_t* ra = st + (tile * 16 + g) * row_w + wbase;
      const uint32_t* rb = ra + 8 * row_w;
      const uint32_t* xl = xb_base + (g < NC ? g : 0) * xcw + part * 128 + t * 8;
      int acc[4][4];
#pragma unroll
      for (int a = 0; a < 4; ++a) acc[a][0] = acc[a][1] = acc[a][2] = acc[a][3] = 0;
      uint4 ma = make_uint4(0u, 0u, 0u, 0u), mb = ma, sa = ma, sb = ma;
      if (live) {
        ma = *reinterpret_cast<const uint4*>(ra);
        mb = *reinterpret_cast<const uint4*>(rb);
        sa = *reinterpret_cast<const uint4*>(ra + KM);
        sb = *reinterpret_cast<const uint4*>(rb + KM);
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint4 x0 = *reinterpret_cast<const uint4*>(xl + e * 32);
        const uint4 x1 = *reinterpret_cast<const uint4*>(xl + e * 32 + 4);
        uint32_t wa0, wb0, wa1, wb1;
        merge_planes_offset(u4get(ma, e), u4get(sa, e), wa0, wb0);
        merge_planes_offset(u4get(mb, e), u4get(sb, e), wa1, wb1);
        if (!live) wa0 = wb0 = wa1 = wb1 = 0u;
        mma_u8s8(acc[0], wa0 & 0x03030303u, wa1 & 0x03030303u, wb0 & 0x03030303u, wb1 & 0x03030303u, x0.x, x1.x);
        mma_u8s8(acc[1], wa0 & 0x0C0C0C0Cu, wa1 & 0x0C0C0C0Cu, wb0 & 0x0C0C0C0Cu, wb1 & 0x0C0C0C0Cu, x0.y, x1.y);
        mma_u8s8(acc[2], wa0 & 0x30303030u, wa1 & 0x30303030u, wb0 & 0x30303030u, wb1 & 0x30303030u, x0.z, x1.z);
        mma_u8s8(acc[3], wa0 & 0xC0C0C0C0u, wa1 & 0xC0C0C0C0u, wb0 & 0xC0C0C0C0u, wb1 & 0xC0C0C0C0u, x0.w, x1.w);
      }
      // this part's exact sums for the lane's rows and columns (offset 2 * sum x removed)
      if (t < (NC + 1) / 2) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int col = 2 * t + (q & 1);
          if (col < NC) {
            const int v = acc[0][q] + (acc[1][q] >> 2) + (acc[2][q] >> 4) + (acc[3][q] >> 6) - 2 * meta[part * NC + col];
            atomicAdd(&acc_s[(tile * 16 + g + 8 * (q >> 1)) * NC + col], v);
          }
        }
      }
      __syncwarp();
      int done = 0;
      if (lane == 0) {
        __threadfence_block();
        done = atomicAdd(&cnt_s[tile], 1) == KP - 1;
      }
      done = __shfl_sync(0xFFFFFFFFu, done, 0);
      if (done) {                                          // all K parts of the tile are in
        __threadfence_block();
        const int row = (grp_idx * TS + tile) * 16 + lane;
        if (lane < 16) {
          int* ta = acc_s + (tile * 16 + lane) * NC;
          if (row < B.N) {
            const float sc = f16_bits_to_float(B.scale[row]);
            float y;
            if (MODE == 1) {
              y = __fmul_rn(__fmul_rn(__int2float_rn(ta[0]), B.sx[0]), sc);
            } else {
              const long long D = (long long)ta[0] * 65536 + (long long)ta[1] * 256 + (long long)ta[2];
              y = (float)(ldexp((double)D, meta[KP * NC] - kLimbFrac) * (double)sc);
            }
            B.y[row] = y;
          }
#pragma unroll
          for (int c = 0; c < NC; ++c) ta[c] = 0;
        }
        __syncwarp();
        if (lane == 0) cnt_s[tile] = 0;
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty0 + 8 * s);
  }
  // release the last item of this CTA (every earlier one was released on leaving it)
  if (ok) {
    for (; released <= seq; ++released) {
      __syncwarp();
      if (lane == 0) mbar_arrive(xempty0 + 8 * (released & 1));
    }
  } else if (lane == 0) {
    atomicExch(&g_batch_latch, 5);
  }
}

}  // namespace

bool plan_batch(BatchParams& p, size_t& smem, size_t& workspace) {
  const int nc = p.mode == 0 ? 3 : 1;
  p.nc = nc;
  // stage: TS whole tiles, at most 48 KB and 12 tiles; K parts of 512 trits (the last one partial)
  const int kSlot = 48 * 1024;
  long long total_bytes = 0;
  int units = 0, max_x = 0, max_slot = 0;
  size_t xoff = 0;
  for (int i = 0; i < p.count; ++i) {
    BatchItem& it = p.items[i];
    if (it.K % 128 || it.K <= 0 || it.N <= 0) return false;
    const int tile_bytes = 16 * it.K / 4;
    int ts = kSlot / tile_bytes;
    if (ts > 12) ts = 12;
    if (ts < 1) return false;                              // a tile larger than a stage slot
    it.ts = ts;
    it.kp = (it.K + 511) / 512;
    if (it.kp > 24) return false;
    it.unit0 = units;
    const int tiles = (it.N + 15) / 16;
    it.units = (tiles + ts - 1) / ts;
    units += it.units;
    const int xcw = it.kp * 128 + 4;
    int xb = nc * xcw * 4 + (it.kp * nc + 1) * 4;
    xb = (xb + 15) & ~15;
    it.xbytes = xb;
    it.xoff = (uint32_t)xoff;
    xoff += (size_t)xb;
    if (xb > max_x) max_x = xb;
    if (ts * tile_bytes > max_slot) max_slot = ts * tile_bytes;
    total_bytes += (long long)it.N * it.K / 4;
  }
  p.total_units = units;
  p.stage_slot_bytes = max_slot;
  p.x_slot_bytes = max_x;
  workspace = xoff;
  // balanced by weight bytes: CTA c starts at the first unit whose start byte reaches c/G of the total
  const int grid = units < 148 ? units : 148;
  p.grid = grid;
  long long acc = 0;
  int c = 0;
  p.cta_unit[0] = 0;
  for (int i = 0; i < p.count; ++i) {
    const BatchItem& it = p.items[i];
    const long long unit_bytes = (long long)it.ts * 16 * it.K / 4;
    for (int u = 0; u < it.units; ++u) {
      while (c + 1 < grid && acc >= total_bytes * (c + 1) / grid) p.cta_unit[++c] = it.unit0 + u;
      acc += unit_bytes;
    }
  }
  while (c + 1 <= grid) p.cta_unit[++c] = units;
  p.cta_unit[grid] = units;
  const size_t fixed = 1024 + 2 * (size_t)max_x;
  int stages = 0;
  for (int s = 6; s >= 2; --s) {
    const size_t need = fixed + (size_t)s * max_slot + (size_t)s * 12 * 16 * nc * 4;
    if (need <= 226 * 1024) { stages = s; break; }
  }
  if (!stages) return false;
  p.stages = stages;
  smem = fixed + (size_t)stages * max_slot + (size_t)stages * 12 * 16 * nc * 4;
  return true;
}

cudaError_t read_and_clear_batch_latch(int* out) {
  cudaError_t e = cudaMemcpyFromSymbol(out, g_batch_latch, sizeof(int));
  if (e != cudaSuccess) return e;
  const int zero = 0;
  return cudaMemcpyToSymbol(g_batch_latch, &zero, sizeof(int));
}

cudaError_t launch_batch(const BatchParams& p, size_t smem, bool pdl, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  int na = 0;
  if (pdl) {
    attr[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[na].val.programmaticStreamSerializationAllowed = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  cfg.stream = st;
  // 1. operand blocks
  cfg.gridDim = dim3(p.count, 1, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cudaError_t e = cudaLaunchKernelEx(&cfg, k_batch_prep, p);
  if (e != cudaSuccess) return e;
  // 2. the stream (always programmatically dependent on the prep launch)
  cudaLaunchAttribute attr2[1];
  attr2[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr2[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr2;
  cfg.numAttrs = 1;
  cfg.gridDim = dim3(p.grid, 1, 1);
  cfg.blockDim = dim3(kBatchThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  if (p.mode == 0) {
    static int set0 = 0;
    if ((int)smem > set0) {
      e = cudaFuncSetAttribute(k_batch_stream<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      set0 = (int)smem;
    }
    return cudaLaunchKernelEx(&cfg, k_batch_stream<0>, p);
  }
  static int set1 = 0;
  if ((int)smem > set1) {
    e = cudaFuncSetAttribute(k_batch_stream<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    set1 = (int)smem;
  }
  return cudaLaunchKernelEx(&cfg, k_batch_stream<1>, p);
}

}  // namespace tern
