// A decode step whose linear layers depend on one another, in one persistent launch (M = 1).
//
// The pages place the time a decode token spends above its DRAM floor in the dependency chains
// between and inside the ~120 kernels of a step (PyTorchKR review "Fermion Research, 3진 계열
// 포맷으로 직접 학습한 Neutrino-1 모델군 3종 공개", section "뉴트리노 엔진: 토큰 하나의 시간은 어디로
// 가는가"). Here the chain of a step's linears runs as one cooperative kernel, one CTA per SM:
//   * every linear's rows are cut into chunks of R rows (R a multiple of 16, about N / CTAs), and
//     CTA c owns chunks c, c + G, ... over the whole of K, so no output needs a sum from another CTA;
//   * a producer lane streams the weights of every linear, one after the other, through a ring of
//     shared-memory stages (tensor TMA of the row-major planes, no multicast): a stage holds the
//     chunk's rows for ps consecutive 512-trit parts. Weights do not depend on activations, so the
//     ring keeps filling while the consumers wait for the previous linear's outputs: the weight
//     stream does not stop at a linear's boundary;
//   * before a linear the consumer warps wait (bounded) until every CTA has finished the linear it
//     reads, then compute its activation from that output -- RMSNorm, an fp32 cast, or a bf16 row
//     such as the SwiGLU output -- exactly as the batched prologues do (tern_prologue.cuh), and
//     encode every 512-trit part as int8 operands (four exact limbs of the row's 30-bit fixed
//     point, or the int8 quantiser's q);
//   * the 12 consumer warps split a chunk's 16-row tiles, and the parts of a stage between the warps
//     of one tile; each runs the signed decode (64 * t bytes) through mma.sync s8 x s8, and the warps
//     of a tile add their exact sums through shared memory before one of them writes the outputs;
//   * a gate|up linear whose rows interleave gate and up in groups of eight writes, besides its
//     fp32 outputs, the SwiGLU activation bf16(silu(gate) * up) of each pair: a lane holds rows r
//     and r + 8 of its tile, i.e. the gate and the up row of one feature (the SwiGLU epilogue);
//   * a CTA that has written its chunks of a linear bumps that linear's completion counter
//     (release); the last CTA of the launch clears the counters for the next call.
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
constexpr int kMaxRows = kCW * 16;               // rows of a chunk at most: one 16-row tile per warp
constexpr int kPartWords = 16;                   // words per plane and row in a 512-trit part
constexpr int kStageBytes = 24576;               // one ring stage: 2 planes x R rows x ps parts x 64 B
constexpr int kColWords = 132;                   // operand words per column and part (128 + skew)
constexpr int kConsumers = kCW * 32;
constexpr int kMaxK = 12288;
constexpr int kJH = kMaxK / (16 * kConsumers);  // 16-element halves of the activation per consumer thread
static_assert(kJH * 16 * kConsumers == kMaxK, "activation row split");
constexpr int kRedBytes = kCW * 32 * 4 * 4;      // cross-warp sums: [warp][lane][4] int32

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

// Operand words of word w (0..15) of a part, as in the batched kernel: lane t = w / 4 reads the eight
// words of its word e = w % 4 at ((e * 4) + t) * 8.
__device__ __forceinline__ int part_slot(int w) { return ((w & 3) * 4 + (w >> 2)) * 8; }

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
  // after the ring: operand segments [seg_parts][NCOL * kColWords] words, the cross-warp sums
  uint32_t* segbuf = reinterpret_cast<uint32_t*>(smem + 1024 + (size_t)S * kStageBytes);
  const uint32_t seg0 = smem_u32(segbuf);
  int* red = reinterpret_cast<int*>(segbuf + (size_t)p.seg_parts * NCOL * kColWords);
  __shared__ double dred[kCW];
  __shared__ float fred[kCW];
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
      // the tensor map was written to global memory by the host: order it before its TMA use
      asm volatile("fence.proxy.tensormap::generic.acquire.gpu [%0], 128;" ::"l"(&it.tmap) : "memory");
      const uint32_t bytes = (uint32_t)(it.rows * it.ps * 128);
      for (int ch = c; ch < it.chunks && ok; ch += G)
        for (int st = 0; st < it.nst; ++st) {
          if (q >= S && !(ok = mbar_wait(empty0 + 8 * s, ph ^ 1u))) break;
          const uint32_t bar = full0 + 8 * s;
          mbar_arrive_expect_tx(bar, bytes);
          tma_load_3d(ring + (uint32_t)s * kStageBytes, &it.tmap, st * it.ps * kPartWords, ch * it.rows, 0, bar);
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
  int s = 0;
  uint32_t ph = 0;
  bool ok = true;
  for (int i = 0; i < p.count && ok; ++i) {
    const ChainItem& it = items[i];
    // the next linear's descriptor into L1 (its gains follow into L2 once this linear is done):
    // neither depends on this linear
    const bool has_next = i + 1 < p.count;
    if (has_next && tid == 0)
      asm volatile("prefetch.global.L1 [%0];" ::"l"(reinterpret_cast<const uint8_t*>(items + i + 1) + 128));
    const uint16_t* next_gain = has_next ? items[i + 1].gain : nullptr;
    const int next_k = has_next ? items[i + 1].K : 0;
    if (c >= it.chunks) continue;                               // no rows of this linear
    // every field this linear needs, into registers now: the descriptor line may have left L1
    const int K = it.K, kp = it.kp, kind = it.kind, N = it.N, rows = it.rows, chunks = it.chunks;
    const int ps = it.ps, nst = it.nst, dep = it.dep, dep_need = it.dep_need;
    const float eps = it.eps;
    const uint16_t* scale = it.scale;
    float* yout = it.y;
    uint16_t* hout = it.hout;
    float* sx_out = it.sx_out;
    const void* src = it.src;
    const uint16_t* gain = it.gain;
    // each thread's 16-element halves of the activation row -- v = tid + j kConsumers, elements
    // 16 v .. 16 v + 15: one unit of the operand layout -- stay in registers from the loads to the
    // operands. The gains do not depend on the source: load them before the wait.
    const int nh = kp * 32;                                     // halves of the row's parts (zeros past K)
    uint4 gw[kJH][2];
#pragma unroll
    for (int j = 0; j < kJH; ++j) {
      const int k = 16 * (tid + j * kConsumers);
      const bool in = k < K && kind == kProRMSNorm;
      gw[j][0] = in ? __ldg(reinterpret_cast<const uint4*>(gain + k)) : make_uint4(0u, 0u, 0u, 0u);
      gw[j][1] = in ? __ldg(reinterpret_cast<const uint4*>(gain + k + 8)) : make_uint4(0u, 0u, 0u, 0u);
    }
    // ---- 1. wait for the source ----------------------------------------------------------------
    if (dep >= 0) {
      bool got = true;
      if (tid == 0) got = wait_done(p.done, dep, dep_need);
      if (!consumers_all(got)) { ok = false; break; }          // uniform: every consumer breaks
    }
    // ---- 2. the activation: sum of squares (RMSNorm), the bf16 values and their absmax ----------
    float4 av[kJH][4];
    double r = 1.0;
    if (kind != kProBF16) {
      double ss = 0.0;
#pragma unroll
      for (int j = 0; j < kJH; ++j) {
        const int k = 16 * (tid + j * kConsumers);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          av[j][u] = k < K ? ldcg4(static_cast<const float*>(src) + k + 4 * u) : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
          ss += (double)av[j][u].x * av[j][u].x + (double)av[j][u].y * av[j][u].y + (double)av[j][u].z * av[j][u].z +
                (double)av[j][u].w * av[j][u].w;
        }
      }
      if (kind == kProRMSNorm) {
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
        if (lane == 0) dred[warp] = ss;
        consumers_sync();
        double tot = 0.0;
        for (int w = 0; w < kCW; ++w) tot += dred[w];
        r = 1.0 / sqrt(tot / (double)K + (double)eps);
      }
    }
    uint32_t hv[kJH][8];                                        // the bf16 values, two per word
    float amax = 0.0f;
#pragma unroll
    for (int j = 0; j < kJH; ++j) {
      const int k = 16 * (tid + j * kConsumers);
#pragma unroll
      for (int e = 0; e < 8; ++e) hv[j][e] = 0u;
      if (k < K) {
        if (kind == kProBF16) {
          const uint4 x0 = __ldcg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(src) + k));
          const uint4 x1 = __ldcg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(src) + k + 8));
          hv[j][0] = x0.x; hv[j][1] = x0.y; hv[j][2] = x0.z; hv[j][3] = x0.w;
          hv[j][4] = x1.x; hv[j][5] = x1.y; hv[j][6] = x1.z; hv[j][7] = x1.w;
        } else {
          const uint32_t gg[8] = {gw[j][0].x, gw[j][0].y, gw[j][0].z, gw[j][0].w, gw[j][1].x, gw[j][1].y, gw[j][1].z, gw[j][1].w};
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float4 q4 = av[j][e >> 2];
            const float a = (e & 3) == 0 ? q4.x : ((e & 3) == 1 ? q4.y : ((e & 3) == 2 ? q4.z : q4.w));
            uint32_t h;
            if (kind == kProRMSNorm) {
              const uint32_t gb = (e & 1) ? (gg[e >> 1] >> 16) : (gg[e >> 1] & 0xFFFFu);
              h = bf16_rn(((double)a * r) * (double)bf16_bits_to_float(gb));
            } else {
              h = bf16_rn((double)a);
            }
            hv[j][e >> 1] |= h << (16 * (e & 1));
          }
        }
#pragma unroll
        for (int e = 0; e < 8; ++e)
          amax = fmaxf(amax, fmaxf(fabsf(bf16_bits_to_float(hv[j][e] & 0xFFFFu)), fabsf(bf16_bits_to_float(hv[j][e] >> 16))));
      }
    }
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    if (lane == 0) fred[warp] = amax;
    consumers_sync();
    // every thread reduces the warp maxima itself (one barrier instead of two); fred is next
    // written after the operand build's barrier
    float mx = fred[0];
#pragma unroll
    for (int w = 1; w < kCW; ++w) mx = fmaxf(mx, fred[w]);
    const int E = MODE == 0 ? limb_exponent(mx) : 0;
    const float sxv = MODE == 1 ? __fdiv_rn(mx, 127.0f) : 0.0f;
    if (MODE == 1 && tid == 0 && c == 0 && sx_out) sx_out[0] = sxv;   // CTA 0 owns chunk 0
    // ---- 3. operand segments of every part, from the registers ------------------------------------
#pragma unroll
    for (int j = 0; j < kJH; ++j) {
      const int v = tid + j * kConsumers;
      if (v >= nh) continue;
      const int part = v >> 5, w = (v & 31) >> 1, h = v & 1;
      uint32_t* seg = segbuf + (size_t)part * (NCOL * kColWords) + part_slot(w);
      uint32_t l[NCOL][4] = {};                                // zeros past K
#pragma unroll
      for (int g4 = 0; g4 < 4; ++g4) {                          // elements 4 g4 .. 4 g4 + 3
        int X[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t w2 = hv[j][2 * g4 + (e >> 1)];
          const float xf = bf16_bits_to_float((e & 1) ? (w2 >> 16) : (w2 & 0xFFFFu));
          X[e] = MODE == 0 ? limb_fixed(xf, E) : quant_i8(xf, sxv);
        }
        if (MODE == 0) {
          uint32_t o[4];
          limbs4_of(X, o);
#pragma unroll
          for (int col = 0; col < NCOL; ++col) l[col][g4] = o[col];
        } else {
          l[0][g4] = (X[0] & 0xFF) | ((X[1] & 0xFF) << 8) | ((X[2] & 0xFF) << 16) | ((uint32_t)X[3] << 24);
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
    consumers_sync();
    // ---- 4. this CTA's chunks: warps split the 16-row tiles, then a stage's parts -----------------
    const int T = rows >> 4;                                 // tiles of a chunk (<= kCW)
    const int wpt = kCW / T;                                    // warps per tile
    const bool active = warp < T * wpt;
    const int tile = warp % T, lg = warp / T;
    const int rstride = 64 * ps;                             // bytes of one row of a plane in a stage
    for (int ch = c; ch < chunks && ok; ch += G) {
      const int r0 = ch * rows + tile * 16 + g;              // rows r0 (q = 0, 1) and r0 + 8 (q = 2, 3)
      uint16_t sc_bits[2];
#pragma unroll
      for (int h = 0; h < 2; ++h)
        sc_bits[h] = (active && lg == 0 && t == 0 && r0 + 8 * h < N) ? scale[r0 + 8 * h] : (uint16_t)0;
      int acc4[4][4] = {};                                      // one chain per decode field f
      for (int st = 0; st < nst; ++st) {
        if (!(ok = mbar_wait(full0 + 8 * s, ph))) break;
        if (active) {
          const uint32_t rowa = ring + (uint32_t)s * kStageBytes + (uint32_t)((tile * 16 + g) * rstride + t * 16);
          const uint32_t planeb = (uint32_t)(rows * rstride);
          for (int pp = lg; pp < ps; pp += wpt) {
            const int part = st * ps + pp;
            if (part >= kp) break;
            const uint32_t ra = rowa + pp * 64;
            const uint4 ma = lds128(ra), mb = lds128(ra + 8 * rstride);
            const uint4 sa = lds128(ra + planeb), sb = lds128(ra + planeb + 8 * rstride);
            const uint32_t xo = seg0 + (uint32_t)(part * NCOL * kColWords + (live0 ? g : 0) * kColWords + t * 8) * 4;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
              const uint4 x01 = live0 ? lds128(xo + e * 128) : zero;
              const uint4 x23 = live0 ? lds128(xo + e * 128 + 16) : zero;
              uint32_t wa0, wb0, wa1, wb1;
              merge_planes(u4get(ma, e), u4get(sa, e), wa0, wb0);
              merge_planes(u4get(mb, e), u4get(sb, e), wa1, wb1);
#pragma unroll
              for (int f = 0; f < 4; ++f) {
                const uint32_t b0 = f < 2 ? u4get(x01, 2 * f) : u4get(x23, 2 * f - 4);
                const uint32_t b1 = f < 2 ? u4get(x01, 2 * f + 1) : u4get(x23, 2 * f - 3);
                mma_s8(acc4[f], (wa0 << (6 - 2 * f)) & 0xC0C0C0C0u, (wa1 << (6 - 2 * f)) & 0xC0C0C0C0u,
                       (wb0 << (6 - 2 * f)) & 0xC0C0C0C0u, (wb1 << (6 - 2 * f)) & 0xC0C0C0C0u, b0, b1);
              }
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty0 + 8 * s);
        if (++s == S) { s = 0; ph ^= 1u; }
      }
      // the tile's exact sums: the warps of a tile add theirs through shared memory (acc = 64 * sum)
      int acc[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[q] = acc4[0][q] + acc4[1][q] + acc4[2][q] + acc4[3][q];
      if (!consumers_all(ok)) { ok = false; break; }
      if (wpt > 1) {
        if (active && lg > 0) {
#pragma unroll
          for (int q = 0; q < 4; ++q) red[(warp * 32 + lane) * 4 + q] = acc[q];
        }
        consumers_sync();
        if (active && lg == 0)
          for (int l = 1; l < wpt; ++l)
#pragma unroll
            for (int q = 0; q < 4; ++q) acc[q] += red[((warp + l * T) * 32 + lane) * 4 + q];
      }
      if (active && lg == 0) {
        int V[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) V[q] = acc[q] >> 6;
        float y[2] = {0.0f, 0.0f};
        if (MODE == 1) {
#pragma unroll
          for (int h = 0; h < 2; ++h) y[h] = __fmul_rn(__fmul_rn(__int2float_rn(V[2 * h]), sxv), f16_bits_to_float(sc_bits[h]));
        } else {
          // lane t = 0 holds columns 0 (L3) and 1 (L2), lane t = 1 columns 2 (L1) and 3 (L0)
          int w[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) w[q] = __shfl_down_sync(0xFFFFFFFFu, V[q], 1);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const long long D = limb_combine(V[2 * h], V[2 * h + 1], w[2 * h], w[2 * h + 1]);
            y[h] = (float)((double)D * exp2_i(E - kLimbFrac) * (double)f16_bits_to_float(sc_bits[h]));
          }
        }
        if (t == 0) {
#pragma unroll
          for (int h = 0; h < 2; ++h)
            if (r0 + 8 * h < N) yout[r0 + 8 * h] = y[h];
          if (hout && r0 + 8 < N) {
            // SwiGLU epilogue: rows r0 (gate) and r0 + 8 (up) of the interleaved tile are one feature
            const double z = (double)y[0];
            hout[(r0 - g) / 2 + g] = bf16_rn((z / (1.0 + exp(-z))) * (double)y[1]);
          }
        }
      }
    }
    if (next_gain && tid * 64 < next_k) asm volatile("prefetch.global.L2 [%0];" ::"l"(next_gain + tid * 64));
    // ---- 5. this CTA's chunks of the linear are written: release them ----------------------------
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

// Host plan of a chain: per linear the chunk rows R (a multiple of 16, at most 192), the parts per
// stage, the tensor map (boxes of 16 ps words x R rows x 2 planes), and the shared-memory layout.
bool plan_chain(ChainItem* items, int count, int mode, int grid, const uint32_t* const* planes, ChainLayout& L) {
  PFN_cuTensorMapEncodeTiled_v12000 encode = encode_fn();
  if (!encode || grid < 1) return false;
  const int ncol = mode == 0 ? 4 : 1;
  int kp_max = 1;
  for (int i = 0; i < count; ++i) {
    ChainItem& it = items[i];
    if (it.K % 128 || it.K <= 0 || it.N <= 0 || it.K > kMaxK) return false;
    it.kp = (it.K + 511) / 512;
    long long R = ((long long)it.N + grid - 1) / grid;
    R = (R + 15) / 16 * 16;
    if (R > kMaxRows) R = kMaxRows;
    it.rows = (int)R;
    it.chunks = (int)(((long long)it.N + R - 1) / R);
    int ps = kStageBytes / (it.rows * 128);
    if (ps > it.kp) ps = it.kp;
    if (ps > 16) ps = 16;
    if (ps < 1) return false;
    it.ps = ps;
    it.nst = (it.kp + ps - 1) / ps;
    if (it.kp > kp_max) kp_max = it.kp;
    it.dep_need = 0;
    if (it.dep >= 0) {
      if (it.dep >= i) return false;
      it.dep_need = items[it.dep].chunks < grid ? items[it.dep].chunks : grid;
    }
    const cuuint64_t dims[3] = {(cuuint64_t)(it.K / 32), (cuuint64_t)it.N, 2};
    const cuuint64_t strides[2] = {(cuuint64_t)it.K / 4, (cuuint64_t)it.K / 8};
    const cuuint32_t box[3] = {(cuuint32_t)(kPartWords * ps), (cuuint32_t)it.rows, 2};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (encode(&it.tmap, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<uint32_t*>(planes[i]), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  }
  // shared memory: barriers (1 KB), the stage ring, the operand segments, the cross-warp sums
  const size_t seg_bytes = (size_t)kp_max * ncol * kColWords * 4;
  const size_t fixed = 1024 + seg_bytes + kRedBytes;
  const size_t budget = 226 * 1024;                              // dynamic: the opt-in limit less 1 KB static
  if (fixed + 2 * (size_t)kStageBytes > budget) return false;
  int stages = (int)((budget - fixed) / kStageBytes);
  if (stages > 8) stages = 8;
  L.stages = stages;
  L.seg_parts = kp_max;
  L.smem = fixed + (size_t)stages * kStageBytes;
  L.scratch_words = 0;
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
