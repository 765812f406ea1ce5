// A decode step whose linear layers depend on one another, in one persistent launch (M = 1).
//
// The pages place the time a decode token spends above its DRAM floor in the dependency chains
// between and inside the ~120 kernels of a step (PyTorchKR review "Fermion Research, 3진 계열
// 포맷으로 직접 학습한 Neutrino-1 모델군 3종 공개", section "뉴트리노 엔진: 토큰 하나의 시간은 어디로
// 가는가"). Here the chain of a step's linears runs as one cooperative kernel, one CTA per SM:
//   * a producer lane streams the weights of every linear, one after the other, through a ring of
//     shared-memory stages (tensor TMA of the row-major planes, no multicast). Weights do not
//     depend on activations, so the ring keeps filling while the consumers wait for the previous
//     linear's outputs: the weight stream does not stop at a linear's boundary;
//   * the consumer warps of every CTA take an even share of each linear's (row block, 512-trit part)
//     units. Before a linear, they wait (bounded) until every CTA has finished the linear it reads,
//     then compute its activation from that output -- RMSNorm, an fp32 cast, or a bf16 row such as
//     the SwiGLU output -- exactly as the batched prologues do (tern_prologue.cuh), encode the parts
//     they need as int8 operands (four exact limbs of the row's 30-bit fixed point, or the int8
//     quantiser's q) and run the signed decode (64 * t bytes) through mma.sync s8 x s8;
//   * a gate|up linear whose rows interleave gate and up in groups of eight writes, besides its
//     fp32 outputs, the SwiGLU activation bf16(silu(gate) * up) of each pair: a lane holds rows r
//     and r + 8 of its tile, i.e. the gate and the up row of one feature (the SwiGLU epilogue);
//   * a row block split between CTAs adds exact partial sums in a workspace slot; its last
//     contributor writes the outputs and clears the slot for the next call; a CTA that has finished
//     its share of a linear bumps that linear's completion counter (release); the last CTA of the
//     launch clears the counters.
// All sums are exact integers and the prologues are the batched path's arithmetic, so every output
// equals tern_gemm_batch_pro's with the same prologue, bit for bit. Every wait is bounded and latches
// TERN_ETIMEOUT on give-up.
#include <atomic>
#include <cstdint>
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <new>

#include "tern_device.cuh"
#include "tern_kernels.h"
#include "tern_prologue.cuh"

namespace tern {

__device__ int g_chain_latch = 0;

namespace {

constexpr int kCW = 12;                          // consumer warps
constexpr int kTPW = 2;                          // tiles of 16 rows per consumer warp
constexpr int kBoxRows = kCW * 16;               // rows of one TMA box
constexpr int kStageRows = kBoxRows * kTPW;      // rows of a row block (384)
constexpr int kPartWords = 16;                   // words per plane and row in a 512-trit part
constexpr int kBoxBytes = 2 * kBoxRows * kPartWords * 4;
constexpr int kStageBytes = kTPW * kBoxBytes;    // 49152
constexpr int kColWords = 132;                   // operand words per column and part (128 + skew)
constexpr int kConsumers = kCW * 32;
constexpr uint32_t kWaitTries = 1u << 13;
constexpr long long kSpinNs = 4000000000LL;      // dependency waits give up after ~4 s

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
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int c0, int c1, int c2, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];"
      ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
      : "memory");
}
__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t u4get(const uint4& v, int e) {
  return e == 0 ? v.x : (e == 1 ? v.y : (e == 2 ? v.z : v.w));
}
__device__ __forceinline__ double exp2_i(int e) { return __longlong_as_double((long long)(e + 1023) << 52); }
// consumer-only barrier (the producer warp never joins it)
__device__ __forceinline__ void consumers_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kConsumers) : "memory"); }
// the same barrier, returning the AND of every consumer thread's predicate (uniform, race-free)
__device__ __forceinline__ bool consumers_all(bool v) {
  int r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.s32 p, %1, 0;\n bar.red.and.pred q, 1, %2, p;\n selp.s32 %0, 1, 0, q;\n}\n"
      : "=r"(r)
      : "r"((int)v), "n"(kConsumers)
      : "memory");
  return r != 0;
}
// L2 loads of data other CTAs wrote during this launch (no stale L1 lines)
__device__ __forceinline__ float4 ldcg4(const float* p) { return __ldcg(reinterpret_cast<const float4*>(p)); }
__device__ __forceinline__ uint4 ldcg16(const uint16_t* p) { return __ldcg(reinterpret_cast<const uint4*>(p)); }

// Operand words of word w (0..15) of a part, as in the batched kernel: lane t = w / 4 reads the eight
// words of its word e = w % 4 at ((e * 4) + t) * 8.
__device__ __forceinline__ int part_slot(int w) { return ((w & 3) * 4 + (w >> 2)) * 8; }

// CTA range of a linear with P units over G CTAs: [P c / G, P (c + 1) / G); the CTA owning unit p.
__device__ __forceinline__ int range_start(int P, int G, int c) { return (int)((long long)P * c / G); }
__device__ __forceinline__ int owner(int P, int G, int p) { return (int)(((long long)(p + 1) * G - 1) / P); }
// Number of CTAs that own units of [b0, b1): owners are nondecreasing in the unit index, but with
// fewer units than CTAs the CTAs between two owners own none, so count the distinct owners.
__device__ __forceinline__ int contributors(int P, int G, int b0, int b1) {
  int n = 1, o = owner(P, G, b0);
  for (int u = b0 + 1; u < b1; ++u) {
    const int v = owner(P, G, u);
    n += v != o;
    o = v;
  }
  return n;
}

// 8 bf16 values (k .. k+7) of the linear's activation row, computed from its source with the
// prologue's arithmetic; sources written during the launch are read through L2.
__device__ __forceinline__ uint4 act8(const ChainItem& it, int k, double r) {
  if (it.kind == kProBF16) return ldcg16(static_cast<const uint16_t*>(it.src) + k);
  const float* s = static_cast<const float*>(it.src);
  const float4 a0 = ldcg4(s + k), a1 = ldcg4(s + k + 4);
  const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
  uint16_t h[8];
  if (it.kind == kProRMSNorm) {
    const uint4 gw = ld_nc(it.gain + k);
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

// Bounded wait until every participating CTA has finished linear `dep` (acquire).
__device__ bool wait_done(const int* done, int dep, int need) {
  const long long t0 = clock64();
  long long spins = 0;
  while (true) {
    int v;
    asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(done + dep) : "memory");
    if (v >= need) return true;
    if (++spins > 64) __nanosleep(200);
    if (clock64() - t0 > kSpinNs * 2) return false;  // ~4 s at 2 GHz
  }
}

template <int MODE>
__global__ void __launch_bounds__((kCW + 1) * 32, 1) k_chain(const ChainParams p) {
  extern __shared__ __align__(1024) uint8_t smem[];
  constexpr int NCOL = MODE == 0 ? 4 : 1;                  // limb columns or q
  const int S = p.stages;
  const uint32_t full0 = smem_u32(smem), empty0 = full0 + 8 * S;
  const uint32_t ring = smem_u32(smem + 1024);
  uint32_t* segbuf = reinterpret_cast<uint32_t*>(smem + 1024 + (size_t)S * kStageBytes);   // [kp][NCOL * kColWords]
  const uint32_t seg0 = smem_u32(segbuf);
  __shared__ double dred[kCW];
  __shared__ float fred[kCW];
  __shared__ int sh_E;
  __shared__ float sh_sx;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = gridDim.x, c = blockIdx.x;
  const ChainItem* items = p.items;

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(full0 + 8 * i, 1);
      mbar_init(empty0 + 8 * i, kCW);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  __syncthreads();
  pdl_wait();

  if (warp == kCW) {
    // ====================== producer (lane 0): the weights of every linear, in order ==============
    if (lane != 0) return;
    int s = 0, q = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int i = 0; i < p.count && ok; ++i) {
      const ChainItem& it = items[i];
      const int P = it.units * it.kp;
      // the tensor map was written to global memory by the host: order it before its TMA use
      asm volatile("fence.proxy.tensormap::generic.acquire.gpu [%0], 128;" ::"l"(&it.tmap) : "memory");
      for (int u = range_start(P, G, c); u < range_start(P, G, c + 1) && ok; ++u) {
        const int rb = u / it.kp, part = u - rb * it.kp;
        if (q >= S && !(ok = mbar_wait(empty0 + 8 * s, ph ^ 1u))) break;
        int boxes = 0;
        for (int b = 0; b < kTPW; ++b) boxes += (rb * kStageRows + b * kBoxRows < it.N) ? 1 : 0;
        const uint32_t bar = full0 + 8 * s, dst = ring + (uint32_t)s * kStageBytes;
        mbar_arrive_expect_tx(bar, (uint32_t)(boxes * kBoxBytes));
        for (int b = 0; b < boxes; ++b)
          tma_load_3d(dst + b * kBoxBytes, &it.tmap, part * kPartWords, rb * kStageRows + b * kBoxRows, 0, bar);
        ++q;
        if (++s == S) { s = 0; ph ^= 1u; }
      }
    }
    if (!ok) atomicExch(&g_chain_latch, 5);
    // do not exit with copies in flight: wait for the stages issued last
    for (int k = q > S ? q - S : 0; k < q; ++k)
      if (!mbar_wait(full0 + 8 * (k % S), (uint32_t)((k / S) & 1))) { atomicExch(&g_chain_latch, 5); break; }
    return;
  }

  // ====================== consumers ======================
  const int g = lane >> 2, t = lane & 3;
  const int tid = threadIdx.x;                                  // 0 .. kConsumers-1
  const bool live0 = MODE == 0 ? g < NCOL : g == 0;             // lanes whose MMA column carries data
  const uint32_t wofs = (uint32_t)((warp * 16 + g) * kPartWords * 4 + t * 16);
  int s = 0;
  uint32_t ph = 0;
  bool ok = true;
  for (int i = 0; i < p.count && ok; ++i) {
    const ChainItem& it = items[i];
    const int K = it.K, kp = it.kp;
    const int P = it.units * kp;
    const int p0 = range_start(P, G, c), p1 = range_start(P, G, c + 1);
    if (p0 >= p1) continue;                                     // no share of this linear
    // ---- 1. the linear's activation: wait for its source, statistics over the whole row ----------
    if (it.dep >= 0) {
      bool got = true;
      if (tid == 0) {
        const ChainItem& d = items[it.dep];
        const int Pd = d.units * d.kp;
        got = wait_done(p.done, it.dep, Pd < G ? Pd : G);
      }
      if (!consumers_all(got)) { ok = false; break; }          // uniform: every consumer breaks
    }
    double r = 1.0;
    if (it.kind == kProRMSNorm) {
      double ss = 0.0;
      const float* src = static_cast<const float*>(it.src);
      for (int k = tid * 4; k < K; k += kConsumers * 4) {
        const float4 v = ldcg4(src + k);
        ss += (double)v.x * v.x + (double)v.y * v.y + (double)v.z * v.z + (double)v.w * v.w;
      }
      for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
      if (lane == 0) dred[warp] = ss;
      consumers_sync();
      double tot = 0.0;
      for (int w = 0; w < kCW; ++w) tot += dred[w];
      r = 1.0 / sqrt(tot / (double)K + (double)it.eps);
    }
    float amax = 0.0f;
    for (int k = tid * 8; k < K; k += kConsumers * 8) amax = fmaxf(amax, absmax8(act8(it, k, r)));
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    if (lane == 0) fred[warp] = amax;
    consumers_sync();
    if (tid == 0) {
      float mx = fred[0];
      for (int w = 1; w < kCW; ++w) mx = fmaxf(mx, fred[w]);
      if (MODE == 0) {
        sh_E = limb_exponent(mx);
      } else {
        sh_sx = __fdiv_rn(mx, 127.0f);
        if (p0 == 0 && it.sx_out) it.sx_out[0] = sh_sx;     // the CTA holding unit 0
      }
    }
    consumers_sync();
    const int E = sh_E;
    const float sxv = sh_sx;
    // ---- 2. operand segments of the parts this CTA streams (all parts when it covers a row block) ---
    {
      const bool all = p1 - p0 >= kp;
      const int first = p0 % kp, cnt = all ? kp : p1 - p0;
      // one 16-element half of a 32-trit word per thread iteration; parts first .. first + cnt - 1 (mod kp)
      for (int v = tid; v < cnt * 32; v += kConsumers) {
        const int part = (first + v / 32) % kp, wh = v % 32, w = wh >> 1, h = wh & 1;
        const int k = part * 512 + 32 * w + 16 * h;
        uint32_t* seg = segbuf + (size_t)part * (NCOL * kColWords) + part_slot(w);
        if (k >= K) {                                           // past the row: zero operands
          for (int col = 0; col < NCOL; ++col) {
            uint32_t* d = seg + col * kColWords;
            d[0 + h] = d[2 + h] = d[4 + h] = d[6 + h] = 0u;
          }
          continue;
        }
        const uint4 a = act8(it, k, r), b = act8(it, k + 8, r);
        const uint32_t wv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        uint32_t l[NCOL][4] = {};
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float xf = bf16_bits_to_float((e & 1) ? (wv[e >> 1] >> 16) : (wv[e >> 1] & 0xFFFFu));
          const int sh = 8 * (e & 3);
          if (MODE == 0) {
            int L[4];
            limbs_of(limb_fixed(xf, E), L);
#pragma unroll
            for (int col = 0; col < NCOL; ++col) l[col][e >> 2] |= (uint32_t)(uint8_t)L[col] << sh;
          } else {
            l[0][e >> 2] |= (uint32_t)(uint8_t)(int8_t)quant_i8(xf, sxv) << sh;
          }
        }
#pragma unroll
        for (int col = 0; col < NCOL; ++col) {
          const uint4 pv = permute_i8_half(make_uint4(l[col][0], l[col][1], l[col][2], l[col][3]));
          uint32_t* d = seg + col * kColWords;
          d[0 + h] = pv.x;
          d[2 + h] = pv.y;
          d[4 + h] = pv.z;
          d[6 + h] = pv.w;
        }
      }
    }
    consumers_sync();
    // ---- 3. stream this CTA's share, row block by row block ----------------------------------------
    for (int u = p0; u < p1 && ok;) {
      const int rb = u / kp;
      const int pend = min(p1, (rb + 1) * kp);                  // this CTA's parts of the block: [u, pend)
      const int need = contributors(P, G, rb * kp, (rb + 1) * kp);
      const int row_base = rb * kStageRows + warp * 16;
      int acc[kTPW][4];
#pragma unroll
      for (int a = 0; a < kTPW; ++a) acc[a][0] = acc[a][1] = acc[a][2] = acc[a][3] = 0;
      uint16_t sc_bits[kTPW][2];
#pragma unroll
      for (int a = 0; a < kTPW; ++a)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int row = row_base + a * kBoxRows + g + 8 * h;
          sc_bits[a][h] = (t == 0 && row < it.N) ? it.scale[row] : (uint16_t)0;
        }
      for (int uu = u; uu < pend; ++uu) {
        if (!(ok = mbar_wait(full0 + 8 * s, ph))) break;
        const int part = uu % kp;
        const uint32_t st = ring + (uint32_t)s * kStageBytes;
        const uint32_t xo = seg0 + (uint32_t)(part * NCOL * kColWords + (live0 ? g : 0) * kColWords + t * 8) * 4;
        uint4 ma[kTPW], mb[kTPW], sa[kTPW], sb[kTPW];
#pragma unroll
        for (int a = 0; a < kTPW; ++a) {
          const uint32_t rr = st + a * kBoxBytes + wofs;
          ma[a] = lds128(rr);
          mb[a] = lds128(rr + 8 * kPartWords * 4);
          sa[a] = lds128(rr + kBoxRows * kPartWords * 4);
          sb[a] = lds128(rr + (kBoxRows + 8) * kPartWords * 4);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
          const uint4 x01 = live0 ? lds128(xo + e * 128) : zero;
          const uint4 x23 = live0 ? lds128(xo + e * 128 + 16) : zero;
#pragma unroll
          for (int a = 0; a < kTPW; ++a) {
            uint32_t wa0, wb0, wa1, wb1;
            merge_planes(u4get(ma[a], e), u4get(sa[a], e), wa0, wb0);
            merge_planes(u4get(mb[a], e), u4get(sb[a], e), wa1, wb1);
#pragma unroll
            for (int f = 0; f < 4; ++f) {
              const uint32_t b0 = f < 2 ? u4get(x01, 2 * f) : u4get(x23, 2 * f - 4);
              const uint32_t b1 = f < 2 ? u4get(x01, 2 * f + 1) : u4get(x23, 2 * f - 3);
              mma_s8(acc[a], (wa0 << (6 - 2 * f)) & 0xC0C0C0C0u, (wa1 << (6 - 2 * f)) & 0xC0C0C0C0u,
                     (wb0 << (6 - 2 * f)) & 0xC0C0C0C0u, (wb1 << (6 - 2 * f)) & 0xC0C0C0C0u, b0, b1);
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty0 + 8 * s);
        if (++s == S) { s = 0; ph ^= 1u; }
      }
      if (!ok) break;                                         // to the CTA-uniform check of step 4
      // exact sums of this CTA's parts (acc = 64 * sum)
      int V[kTPW][4];
#pragma unroll
      for (int a = 0; a < kTPW; ++a)
#pragma unroll
        for (int q = 0; q < 4; ++q) V[a][q] = acc[a][q] >> 6;
      bool emit = true;
      if (need > 1) {
        // the block is split between CTAs: add into its slot; the last contributor (per warp) reads
        // the totals back, writes the outputs and clears the slot and counter for the next call
        int* sums = p.scratch + it.scratch_off + (size_t)rb * kStageRows * 8;
        int* counter = p.scratch + it.counter_off + rb * kCW + warp;
#pragma unroll
        for (int a = 0; a < kTPW; ++a)
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int col = 2 * t + (q & 1);
            if (col < NCOL) atomicAdd(&sums[(a * kBoxRows + warp * 16 + g + 8 * (q >> 1)) * 8 + col], V[a][q]);
          }
        __threadfence();
        __syncwarp();
        int last = 0;
        if (lane == 0) last = atomicAdd(counter, 1) == need - 1;
        last = __shfl_sync(0xFFFFFFFFu, last, 0);
        if (last) {
          __threadfence();
#pragma unroll
          for (int a = 0; a < kTPW; ++a)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int col = 2 * t + (q & 1);
              if (col < NCOL) {
                int* e = &sums[(a * kBoxRows + warp * 16 + g + 8 * (q >> 1)) * 8 + col];
                V[a][q] = __ldcg(e);
                *e = 0;
              }
            }
          if (lane == 0) *counter = 0;
        } else {
          emit = false;
        }
      }
#pragma unroll
      for (int a = 0; a < kTPW && emit; ++a) {
        const int r0 = row_base + a * kBoxRows + g;             // rows r0 (q = 0, 1) and r0 + 8 (q = 2, 3)
        float y[2] = {0.0f, 0.0f};
        if (MODE == 1) {
#pragma unroll
          for (int h = 0; h < 2; ++h)
            y[h] = __fmul_rn(__fmul_rn(__int2float_rn(V[a][2 * h]), sxv), f16_bits_to_float(sc_bits[a][h]));
        } else {
          // lane t = 0 holds columns 0 (L3) and 1 (L2), lane t = 1 columns 2 (L1) and 3 (L0)
          int w[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) w[q] = __shfl_down_sync(0xFFFFFFFFu, V[a][q], 1);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const long long D = limb_combine(V[a][2 * h], V[a][2 * h + 1], w[2 * h], w[2 * h + 1]);
            y[h] = (float)((double)D * exp2_i(E - kLimbFrac) * (double)f16_bits_to_float(sc_bits[a][h]));
          }
        }
        if (t == 0) {
#pragma unroll
          for (int h = 0; h < 2; ++h)
            if (r0 + 8 * h < it.N) it.y[r0 + 8 * h] = y[h];
          if (it.hout && r0 + 8 < it.N) {
            // SwiGLU epilogue: rows r0 (gate) and r0 + 8 (up) of the interleaved tile are one feature
            const double z = (double)y[0];
            it.hout[(r0 - g) / 2 + g] = bf16_rn((z / (1.0 + exp(-z))) * (double)y[1]);
          }
        }
      }
      u = pend;
    }
    // ---- 4. this CTA's share of the linear is written: release it --------------------------------
    // (a warp whose bounded wait gave up still arrives here, so the decision is CTA-uniform)
    ok = consumers_all(ok);
    if (!ok) break;
    if (tid == 0) {
      __threadfence();
      atomicAdd(p.done + i, 1);
    }
  }
  if (!ok && lane == 0) atomicExch(&g_chain_latch, 5);
  // the last CTA of the launch clears the completion counters for the next call
  consumers_sync();
  if (tid == 0) {
    __threadfence();
    if (atomicAdd(p.finished, 1) == G - 1) {
      for (int i = 0; i < p.count; ++i) atomicExch(p.done + i, 0);
      atomicExch(p.finished, 0);
    }
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

// Host plan of a chain: tensor maps, per-linear units and parts, scratch offsets, the stage ring.
bool plan_chain(ChainItem* items, int count, int mode, const uint32_t* const* planes, ChainLayout& L) {
  PFN_cuTensorMapEncodeTiled_v12000 encode = encode_fn();
  if (!encode) return false;
  const int ncol = mode == 0 ? 4 : 1;
  size_t scratch = 0;                                            // int32 words
  int kp_max = 1;
  for (int i = 0; i < count; ++i) {
    ChainItem& it = items[i];
    if (it.K % 128 || it.K <= 0 || it.N <= 0 || it.K > 12288) return false;
    it.kp = (it.K + 511) / 512;
    it.units = (it.N + kStageRows - 1) / kStageRows;
    if (it.kp > kp_max) kp_max = it.kp;
    it.scratch_off = (uint32_t)scratch;
    scratch += (size_t)it.units * kStageRows * 8;
    it.counter_off = (uint32_t)scratch;
    scratch += (size_t)it.units * kCW;
    if (scratch > 0x7FFFFFFF) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)(it.K / 32), (cuuint64_t)it.N, 2};
    const cuuint64_t strides[2] = {(cuuint64_t)it.K / 4, (cuuint64_t)it.K / 8};
    const cuuint32_t box[3] = {(cuuint32_t)kPartWords, (cuuint32_t)kBoxRows, 2};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (encode(&it.tmap, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<uint32_t*>(planes[i]), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  }
  const size_t seg_bytes = (size_t)kp_max * ncol * kColWords * 4;
  const size_t budget = 226 * 1024;                              // dynamic: the opt-in limit less 1 KB static
  if (1024 + seg_bytes + 2 * (size_t)kStageBytes > budget) return false;
  int stages = (int)((budget - 1024 - seg_bytes) / kStageBytes);
  if (stages > 4) stages = 4;
  L.stages = stages;
  L.smem = 1024 + (size_t)stages * kStageBytes + seg_bytes;
  L.scratch_words = scratch;
  return true;
}

cudaError_t launch_chain(const ChainParams& p, size_t smem, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;                  // every CTA resident at once
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.stream = st;
  cfg.gridDim = dim3(p.grid, 1, 1);
  cfg.blockDim = dim3((kCW + 1) * 32, 1, 1);
  cfg.dynamicSmemBytes = smem;
  static std::atomic<unsigned long long> raised0{0}, raised1{0};
  if (p.mode == 0) {
    cudaError_t e = allow_max_dynamic_smem(k_chain<0>, raised0);
    if (e != cudaSuccess) return e;
    return cudaLaunchKernelEx(&cfg, k_chain<0>, p);
  }
  cudaError_t e = allow_max_dynamic_smem(k_chain<1>, raised1);
  if (e != cudaSuccess) return e;
  return cudaLaunchKernelEx(&cfg, k_chain<1>, p);
}

int chain_grid() {
  // one CTA per SM (the kernel's shared memory allows no more), at most the SM count
  return device_sm_count();
}

cudaError_t read_and_clear_chain_latch(int* out) {
  cudaError_t e = cudaMemcpyFromSymbol(out, g_chain_latch, sizeof(int));
  if (e != cudaSuccess) return e;
  const int zero = 0;
  return cudaMemcpyToSymbol(g_chain_latch, &zero, sizeof(int));
}

}  // namespace tern
