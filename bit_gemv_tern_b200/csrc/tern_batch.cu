// Batched GEMV (M = 1) and small-M GEMM (M = 2..16): a whole list of linear layers in two
// launches.
//
//   for every item i:  y_i[m][n] = scale_i[n] * sum_k t_i[n][k] * x_i[m][k]
//
// A decode step streams every weight of the stack once per token (PyTorchKR review "Fermion
// Research, 3진 계열 포맷으로 직접 학습한 Neutrino-1 모델군 3종 공개", section "뉴트리노 엔진":
// tok/s_max = memory bandwidth / bytes per token); the same section measures most of the time above
// that floor at the ~120 kernel boundaries of a step. Here one persistent launch walks all items, so
// the weight stream never pauses between layers.
//
//   1. k_batch_prep (one CTA per item and token slot) turns each activation into ready-to-load
//      tensor-core operand segments, one per 512-trit K part: int8 q permuted to the decode's byte
//      order (int8 mode), or four exact int8 limbs of a 30-bit fixed-point value relative to 2^E with
//      E from the item's absmax (bf16 mode, see tern_device.cuh), followed by the item's column sums
//      (which remove the decode offset) and E. Tokens occupy the MMA's n-columns (see seg_cols).
//   2. k_batch_stream (one CTA per SM) splits the list's (row block, K part) sequence evenly by
//      bytes, so a row block may be shared by neighbouring CTAs. Its producer lane walks the CTA's
//      row blocks part by part: each stage of the ring receives, by tensor TMA, the mask and sign
//      words of the block's rows for one K part (the packed planes seen as a [plane][row][word]
//      tensor, so the row-major layout is read in place) plus that part's operand segment. The
//      consumer warps walk the stages in order; warp w owns kTPW tiles of 16 rows of the block,
//      decodes them (one AND per operand register, see tern_device.cuh) into mma.sync u8 x s8
//      products, and keeps the sums in registers across all parts of the block, so a tile's
//      outputs are written once, at its end. (bf16 lists of 9..16 rows run on the tensor-core
//      kernels of tern_tc.cu instead.)
// All sums are exact integers; int8 mode ends with y = ((float)acc * s_x) * scale (two fp32
// round-to-nearest multiplies), bf16 mode with one fp64 -> fp32 rounding. Every mbarrier wait is
// bounded and latches TERN_ETIMEOUT on give-up.
#include <atomic>
#include <cstdint>
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "tern_device.cuh"
#include "tern_kernels.h"
#include "tern_prologue.cuh"

namespace tern {

// Set to TERN_ETIMEOUT (5) when a bounded wait of the batched kernels gives up.
__device__ int g_batch_latch = 0;

namespace {

constexpr int kPartWords = 16;                        // words per plane and row in a 512-trit part
// Consumer warps of a kernel shape, and the rows / bytes of one TMA box (tile slot a of every
// consumer warp). A CTA's warps are spread over the SM's four sub-partitions, each with 16K
// registers: 12 consumers + 1 producer put 4 warps on one sub-partition (<= 128 registers per
// thread), 11 + 1 put 3 (<= 168).
__host__ __device__ constexpr int box_rows(int cw) { return cw * 16; }
__host__ __device__ constexpr int box_bytes(int cw) { return 2 * box_rows(cw) * kPartWords * 4; }
constexpr int kColWords = 132;                        // operand words per column and part (128 + bank skew)
constexpr uint32_t kWaitTries = 1u << 13;

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
// Tiled 3-d tensor load (no multicast): the box at coordinates (word c0, row c1, plane c2).
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int c0, int c1, int c2,
                                            uint32_t bar) {
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
__device__ __forceinline__ int bsum(uint32_t w) { return __dp4a((int)w, 0x01010101, 0); }
// 2^e as a double for |e| < 1000 (built from the exponent field: exact).
__device__ __forceinline__ double exp2_i(int e) { return __longlong_as_double((long long)(e + 1023) << 52); }

// Operand words of word w (0..15) of a 512-trit part: lane t = w / 4 reads the eight words of its
// word e = w % 4 at ((e * 4) + t) * 8 (so a quarter-warp's loads hit distinct banks), ordered
// (field 0: b0, b1), (field 1: b0, b1), ...: each tensor-core B register pair is two adjacent
// words of one 128-bit load. b0 / b1 come from 16-byte half h = 0 / 1 of the permuted activation.
__device__ __forceinline__ int part_slot(int w) { return ((w & 3) * 4 + (w >> 2)) * 8; }
__device__ __forceinline__ void store_operand_half(uint32_t* slot, int h, uint4 v) {
  slot[0 + h] = v.x;
  slot[2 + h] = v.y;
  slot[4 + h] = v.z;
  slot[6 + h] = v.w;
}

// ---------------------------------------------------------------------------------------------
// Operand columns of a segment. M = 1 (mp == 1): the nc columns are the limbs L3, L2, L1, L0
// (bf16 mode, top limb first) or q (int8 mode). M >= 2: int8 mode (mp = 8 or 16 token slots)
// column m = token m; bf16 mode column l * mp + m = limb l of token m. With mp = 8 or 16 each MMA
// group of 8 columns holds one limb of eight tokens and a lane ends up with all four limbs of the
// tokens it owns; with mp = 2 or 4 the 8 or 16 columns fill one or two groups and the epilogue
// gathers the limbs.
constexpr int kLimbs = 4;
__host__ __device__ constexpr int seg_cols(int mode, int mp) {
  return mp == 1 ? (mode == 0 ? kLimbs : 1) : (mode == 0 ? kLimbs * mp : mp);
}
// Segment words: columns, then the column sums over all of K, then E per token slot, padded to 16 B.
__host__ __device__ constexpr int seg_words(int mode, int mp) {
  return (seg_cols(mode, mp) * kColWords + seg_cols(mode, mp) + mp + 3) & ~3;
}

// prep: one CTA of NT threads per (item, token slot). Block layout: kp segments of seg_bytes. An
// item with a prologue first computes its bf16 row into shared memory (tern_prologue.cuh), then
// encodes from there; int8 mode quantises that row per token here, so no separate quantiser launch
// runs. Two shapes:
//   PRO: lists with prologue items, 1024 threads (each pass over a row of up to 8192 elements is a
//        single round of loads) and the row buffer in shared memory;
//   !PRO: plain lists, 256 threads with at most 48 registers and no row buffer, so that a CTA fits
//        on an SM next to a stream CTA (128 registers x 416 threads, ~205 KB of shared memory): the
//        stream kernel, released at this kernel's entry, need not wait for the prep CTAs to leave
//        (measured: the 0.6B stack 31.8 -> 31.1 us against 1024-thread CTAs; the 8B unchanged).
constexpr int kPrepThreads = 1024;
constexpr int kPrepThreadsPlain = 256;
constexpr int kPrepMaxK = 12288;
template <int NT, bool PRO>
__global__ void __launch_bounds__(NT, PRO ? 1 : 5) k_batch_prep(const __grid_constant__ PrepParams p) {
  const PrepItem& it = p.items[blockIdx.x];
  const int m = blockIdx.y;                          // token slot (< mp)
  uint32_t* blk = reinterpret_cast<uint32_t*>(p.xprep + it.xoff);
  const int K = it.K, KP = it.kp, mp = p.mp;
  const int ncols = seg_cols(p.mode, mp);
  const int segw = p.seg_bytes / 4;
  const int nl = p.mode == 0 ? kLimbs : 1;           // columns of this token
  const bool pro = PRO && it.kind != kProNone;
  int colof[kLimbs];
  for (int l = 0; l < kLimbs; ++l) colof[l] = mp == 1 ? l : l * mp + m;
  const bool live = m < p.M;
  __shared__ float red[NT / 32];
  __shared__ double dred[NT / 32];
  __shared__ int sums[kLimbs];
  __shared__ int Esh;
  __shared__ float ssh;
  __shared__ __align__(16) uint16_t xs[PRO ? kPrepMaxK : 8];  // a prologue item's prepared bf16 row
  pdl_wait();
  // let the stream kernel get resident now: its producer prefetches weights, which do not depend
  // on this kernel, and its consumers wait for this grid's completion before reading segments
  pdl_launch_dependents();
  {
    // the split-block sums and counters of the stream start at zero
    uint32_t* scr = reinterpret_cast<uint32_t*>(p.xprep + p.scratch_off);
    const int nct = gridDim.x * gridDim.y, ct = blockIdx.y * gridDim.x + blockIdx.x;
    for (int i = ct * blockDim.x + threadIdx.x; i < p.scratch_words; i += nct * blockDim.x) scr[i] = 0u;
  }
  // words of this token's columns that the loop below does not write read as zero: all of them
  // for an empty token slot, else the words of the last part past K (K % 512 != 0)
  {
    const int wl = live ? K / 32 - 16 * (KP - 1) : 0;      // words written in the last part
    const int p0 = live ? KP - 1 : 0;                       // first part with unwritten words
    const int per_part = (16 - wl) * 8;                     // unwritten operand words per column
    for (int i = threadIdx.x; i < (KP - p0) * nl * per_part; i += blockDim.x) {
      const int part = p0 + i / (nl * per_part), r = i % (nl * per_part);
      const int c = r / per_part, j = r % per_part;
      blk[part * segw + colof[c] * kColWords + part_slot(wl + j / 8) + j % 8] = 0u;
    }
  }
  if (threadIdx.x < kLimbs) sums[threadIdx.x] = 0;
  if (threadIdx.x == 0) { Esh = 0; ssh = 0.0f; }
  // the bf16 row of a prologue item, into shared memory (and the optional bf16 copy)
  float amax = 0.0f;
  if (live && pro) {
    const size_t row_elems = (size_t)K * (it.kind == kProSwiGLU ? 2 : 1);
    const void* src = it.kind == kProBF16 ? static_cast<const void*>(static_cast<const uint16_t*>(it.x) + (size_t)m * K)
                                          : static_cast<const void*>(static_cast<const float*>(it.x) + (size_t)m * row_elems);
    const double r = it.kind == kProRMSNorm ? rmsnorm_r<NT>(static_cast<const float*>(src), K, it.eps, dred) : 1.0;
    uint16_t* xo = (p.mode == 0 && it.xout) ? static_cast<uint16_t*>(it.xout) + (size_t)m * K : nullptr;
    for (int k = threadIdx.x * 8; k < K; k += NT * 8) {
      const uint4 v = prologue8(it.kind, src, it.gain, K, k, r);
      *reinterpret_cast<uint4*>(xs + k) = v;
      if (xo) *reinterpret_cast<uint4*>(xo + k) = v;
      amax = fmaxf(amax, absmax8(v));
    }
  } else if (live && p.mode == 0) {
    const uint16_t* xb = static_cast<const uint16_t*>(it.x) + (size_t)m * K;
    for (int k = threadIdx.x * 8; k < K; k += NT * 8) amax = fmaxf(amax, absmax8(ld_nc(xb + k)));
  }
  if (live && (p.mode == 0 || pro)) {
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
    __syncthreads();
    if (threadIdx.x == 0) {
      float mx = red[0];
      for (int i = 1; i < NT / 32; ++i) mx = fmaxf(mx, red[i]);
      if (p.mode == 0) {
        Esh = limb_exponent(mx);
      } else {
        const float sx = __fdiv_rn(mx, 127.0f);     // the per-token quantiser's scale
        ssh = sx;
        it.sx_out[m] = sx;
      }
    }
  }
  __syncthreads();
  const int E = Esh;
  const float sq = ssh;
  int8_t* qo = (p.mode == 1 && pro && it.xout) ? static_cast<int8_t*>(it.xout) + (size_t)m * K : nullptr;
  // one 16-element half of a 32-trit word per thread iteration
  int ls[kLimbs] = {0, 0, 0, 0};
  for (int v = threadIdx.x; live && v < K / 16; v += blockDim.x) {
    const int word = v >> 1, h = v & 1;              // global word index and half
    const int part = word >> 4, w = word & 15;
    uint32_t* seg = blk + part * segw + part_slot(w);
    uint4 a, b;                                      // 16 bf16 values of this half (bf16 sources)
    if (pro) {
      a = *reinterpret_cast<const uint4*>(xs + 16 * v);
      b = *reinterpret_cast<const uint4*>(xs + 16 * v + 8);
    } else if (p.mode == 0) {
      const uint16_t* xb = static_cast<const uint16_t*>(it.x) + (size_t)m * K + 16 * v;
      a = ld_nc(xb);
      b = ld_nc(xb + 8);
    }
    if (p.mode == 1) {
      uint4 q;
      if (pro) {
        const uint32_t wv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        uint32_t qw[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const uint32_t bits = (e & 1) ? (wv[e >> 1] >> 16) : (wv[e >> 1] & 0xFFFFu);
          qw[e >> 2] |= (uint32_t)(uint8_t)(int8_t)quant_i8(bf16_bits_to_float(bits), sq) << (8 * (e & 3));
        }
        q = make_uint4(qw[0], qw[1], qw[2], qw[3]);
        if (qo) *reinterpret_cast<uint4*>(qo + 16 * v) = q;
      } else {
        q = ld_nc(static_cast<const int8_t*>(it.x) + (size_t)m * K + 16 * v);
      }
      ls[0] += bsum(q.x) + bsum(q.y) + bsum(q.z) + bsum(q.w);
      store_operand_half(seg + colof[0] * kColWords, h, permute_i8_half(q));
    } else {
      const uint32_t wv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
      uint32_t l[kLimbs][4];
      limbs_of_bf16<4>(wv, E, l);
#pragma unroll
      for (int c = 0; c < kLimbs; ++c) {
        ls[c] += bsum(l[c][0]) + bsum(l[c][1]) + bsum(l[c][2]) + bsum(l[c][3]);
        store_operand_half(seg + colof[c] * kColWords, h, permute_i8_half(make_uint4(l[c][0], l[c][1], l[c][2], l[c][3])));
      }
    }
  }
  for (int c = 0; c < nl; ++c) {
    int v = ls[c];
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    if ((threadIdx.x & 31) == 0) atomicAdd(&sums[c], v);
  }
  __syncthreads();
  // every segment carries the sums over all of K and E, so the consumer reads them from a stage
  for (int part = threadIdx.x; part < KP; part += blockDim.x) {
    int* meta = reinterpret_cast<int*>(blk + part * segw + ncols * kColWords);
    for (int c = 0; c < nl; ++c) meta[colof[c]] = sums[c];
    meta[ncols + m] = E;
  }
}

// ---------------------------------------------------------------------------------------------
// MODE: 0 bf16 / 1 int8 activations; MP: token slots (1, 2, 4, 8 or 16; 2 and 4 in bf16 mode
// only); TPW: tiles per consumer warp; CW: consumer warps. The decode is the offset decode (bytes
// 4^i * (t + 2), four field accumulators per column group, the offset removed with the column sums).
template <int MODE, int MP, int TPW, int CW>
__global__ void __launch_bounds__((CW + 1) * 32, 1) k_batch_stream(const __grid_constant__ BatchParams p) {
  constexpr int kCW = CW;
  constexpr int kBoxRows = box_rows(CW);
  constexpr int kBoxBytes = box_bytes(CW);
  extern __shared__ __align__(1024) uint8_t smem[];
  // PACK: bf16 mode with 2, 4 or 6 token slots, whose 4 * MP limb columns share one, two or three
  // MMA groups (a lane then holds limbs of several tokens; the epilogue gathers them by shuffles)
  constexpr bool PACK = MP == 2 || MP == 4 || MP == 6;
  static_assert(!PACK || MODE == 0, "packed token slots are a bf16-mode shape");
  constexpr int NCOL = seg_cols(MODE, MP);
  constexpr int G = MP == 1 ? 1 : (NCOL + 7) / 8;           // MMA column groups
  constexpr int JJ = (MP == 1 || PACK) ? 1 : MP / 8;        // groups per limb (token octets)
  constexpr int kStageRowsT = kBoxRows * TPW;
  constexpr int kWStageBytesT = TPW * kBoxBytes;
  const int S = p.stages;
  // layout: [full[S], empty[S] mbarriers; 1 KB][ring: S slots of stage_slot_bytes]
  //   slot: [tile slot 0 box][tile slot 1 box]...[operand segment]
  //   box:  [plane 0: kBoxRows rows x 64 B][plane 1: kBoxRows rows x 64 B]
  const uint32_t full0 = smem_u32(smem);
  const uint32_t empty0 = full0 + 8 * S;
  const uint32_t ring = smem_u32(smem + 1024);
  const uint32_t slot_bytes = (uint32_t)p.stage_slot_bytes;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g0 = p.cta_part[blockIdx.x], g1 = p.cta_part[blockIdx.x + 1];

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(full0 + 8 * i, 1);
      mbar_init(empty0 + 8 * i, kCW);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  __syncthreads();
  pdl_launch_dependents();
  if (g1 <= g0) return;

  // item, row block and part of the first stage
  const int first_item = p.cta_item[blockIdx.x];
  const int first_rb = (g0 - p.items[first_item].part0) / p.items[first_item].kp;
  const int first_part = (g0 - p.items[first_item].part0) - first_rb * p.items[first_item].kp;

  if (warp == kCW) {
    // ====================== producer (lane 0) ======================
    if (lane != 0) return;
    // stages of this CTA in order: (item, row block, part)
    const int n = g1 - g0;
    bool ok = true;
    // 1. weights of the first stages: they do not depend on earlier kernels
    const int pre = n < S ? n : S;
    int it = first_item, rb = first_rb, part = first_part;
    for (int q = 0; q < pre; ++q) {
      const BatchItem& B = p.items[it];
      const uint32_t bar = full0 + 8 * q;
      const uint32_t dst = ring + (uint32_t)q * slot_bytes;
      int boxes = 0;
      for (int b = 0; b < TPW; ++b) boxes += (rb * kStageRowsT + b * kBoxRows < B.N) ? 1 : 0;
      mbar_arrive_expect_tx(bar, (uint32_t)(boxes * kBoxBytes + p.seg_bytes));
      for (int b = 0; b < boxes; ++b)
        tma_load_3d(dst + b * kBoxBytes, &p.tmap[it], part * kPartWords, rb * kStageRowsT + b * kBoxRows, 0, bar);
      if (++part == B.kp) {
        part = 0;
        if (++rb == B.units) { rb = 0; ++it; }
      }
    }
    pdl_wait();
    // 2. every stage: its operand segment and, past the first S, its weights once the slot is free
    it = first_item; rb = first_rb; part = first_part;
    int s = 0, nq = 0;
    uint32_t ph = 0;
    for (int q = 0; q < n && ok; ++q) {
      const BatchItem& B = p.items[it];
      const uint32_t bar = full0 + 8 * s;
      const uint32_t dst = ring + (uint32_t)s * slot_bytes;
      if (q >= S) {
        if (!(ok = mbar_wait(empty0 + 8 * s, ph ^ 1u))) break;
        int boxes = 0;
        for (int b = 0; b < TPW; ++b) boxes += (rb * kStageRowsT + b * kBoxRows < B.N) ? 1 : 0;
        mbar_arrive_expect_tx(bar, (uint32_t)(boxes * kBoxBytes + p.seg_bytes));
        for (int b = 0; b < boxes; ++b)
          tma_load_3d(dst + b * kBoxBytes, &p.tmap[it], part * kPartWords, rb * kStageRowsT + b * kBoxRows, 0, bar);
      }
      bulk_g2s(dst + kWStageBytesT, p.xprep + B.xoff + (size_t)part * p.seg_bytes, (uint32_t)p.seg_bytes, bar);
      ++nq;
      if (++part == B.kp) {
        part = 0;
        if (++rb == B.units) { rb = 0; ++it; }
      }
      if (++s == S) { s = 0; ph ^= 1u; }
    }
    if (!ok) atomicExch(&g_batch_latch, 5);
    // do not exit with copies in flight (on the error path too): wait for the last nq stages to
    // land. A wait gives up only at some q >= S, before that stage's weights are issued, so every
    // copy in flight belongs to one of the stages [0, nq) issued in full.
    for (int q = nq > S ? nq - S : 0; q < nq; ++q) {
      if (!mbar_wait(full0 + 8 * (q % S), (uint32_t)((q / S) & 1))) {
        atomicExch(&g_batch_latch, 5);
        break;
      }
    }
    return;
  }

  // ====================== consumers ======================
  constexpr int NF = 4;                                      // accumulators per column group
  const int g = lane >> 2, t = lane & 3;
  // operand column of group j this lane feeds: M = 1: the lane's limb (rows g >= nc repeat column 0)
  // columns past NCOL (M = 1, PACK) repeat a real column; their sums are never read
  const int col0 = (MP == 1 || PACK) ? (g < NCOL ? g : 0) : g;
  const int col1 = 8 + g < NCOL ? 8 + g : 8;                // PACK, MP >= 4: group 1
  // lanes whose column of group 0 / group 1 exists (M = 1, PACK); the others feed zeros, so the
  // tensor cores multiply no real data into the accumulators that are never read
  const bool live0 = (MP == 1 || PACK) ? g < NCOL : true;
  const bool live1 = PACK ? 8 + g < NCOL : true;
  // byte offsets inside a slot
  const uint32_t wofs = (uint32_t)((warp * 16 + g) * kPartWords * 4 + t * 16);   // plane 0, row g
  const uint32_t xofs = (uint32_t)(kWStageBytesT + (col0 * kColWords + t * 8) * 4);
  const uint32_t xofs1 = (uint32_t)(kWStageBytesT + (col1 * kColWords + t * 8) * 4);
  const uint32_t mofs = (uint32_t)(kWStageBytesT + NCOL * kColWords * 4);
  const int M = p.M;
  constexpr int NCOLP = 8 * G;                              // scratch columns per row
  constexpr int NL = MODE == 0 ? kLimbs : 1;                // columns per token
  const uint32_t split = p.cta_split[blockIdx.x];
  const int slot_first = (int)(split & 0xFFu) - 1, need_first = (int)((split >> 8) & 0xFFu);
  const int slot_last = (int)((split >> 16) & 0xFFu) - 1, need_last = (int)(split >> 24);
  auto lds32 = [](uint32_t a) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
    return (int)v;
  };
  bool ok = true;
  int it = first_item, rb = first_rb, pstart = first_part;
  int s = 0;
  uint32_t ph = 0;
  for (int gq = g0; gq < g1 && ok;) {
    const BatchItem& B = p.items[it];
    const int KP = B.kp;
    const int pend = min(KP, pstart + (g1 - gq));           // this CTA's parts of the block: [pstart, pend)
    int slot = -1, need = 0;                                // block shared with other CTAs
    if (gq == g0) { slot = slot_first; need = need_first; }
    if (gq + (pend - pstart) == g1 && slot_last >= 0) { slot = slot_last; need = need_last; }
    const int row_base = rb * kStageRowsT + warp * 16;         // first row of this warp's tile slot 0
    int acc[TPW][G][NF][4];
#pragma unroll
    for (int a = 0; a < TPW; ++a)
#pragma unroll
      for (int j = 0; j < G; ++j)
#pragma unroll
        for (int i = 0; i < NF; ++i) acc[a][j][i][0] = acc[a][j][i][1] = acc[a][j][i][2] = acc[a][j][i][3] = 0;
    // column sums (over all of K; they remove the decode offset) and exponents of the columns this
    // lane owns.  M = 1: tot[0][c][0] for every column c, E;  M >= 2: [jj][limb][token parity], E
    // per [jj][parity]
    int tot[JJ][kLimbs][2];
    int Etok[JJ][2];
    float sxv[JJ][2];
#pragma unroll
    for (int jj = 0; jj < JJ; ++jj)
#pragma unroll
      for (int b = 0; b < 2; ++b) {
        Etok[jj][b] = 0;
#pragma unroll
        for (int l = 0; l < kLimbs; ++l) tot[jj][l][b] = 0;
      }
    // the epilogue's reads of the row scales (weights: written before any launch of this list),
    // issued now so that they land while the block streams
    uint16_t sc_bits[TPW][2];
#pragma unroll
    for (int a = 0; a < TPW; ++a)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int row = row_base + a * kBoxRows + g + 8 * h;
        sc_bits[a][h] = ((MP > 1 || t == 0) && row < B.N) ? B.scale[row] : (uint16_t)0;
      }
    for (int part = pstart; part < pend; ++part) {
      if (!(ok = mbar_wait(full0 + 8 * s, ph))) break;
      // s_x comes from an earlier kernel: read only after a stage has landed (the producer issues
      // every copy after its grid-dependency wait)
      if (MODE == 1 && part == pstart) {
#pragma unroll
        for (int jj = 0; jj < JJ; ++jj)
#pragma unroll
          for (int b = 0; b < 2; ++b) {
            const int m = MP == 1 ? 0 : 8 * jj + 2 * t + b;
            sxv[jj][b] = m < M ? B.sx[m] : 0.0f;
          }
      }
      const uint32_t st = ring + (uint32_t)s * slot_bytes;
      uint4 ma[TPW], mb[TPW], sa[TPW], sb[TPW];
#pragma unroll
      for (int a = 0; a < TPW; ++a) {
        const uint32_t r = st + a * kBoxBytes + wofs;
        ma[a] = lds128(r);
        mb[a] = lds128(r + 8 * kPartWords * 4);
        sa[a] = lds128(r + kBoxRows * kPartWords * 4);
        sb[a] = lds128(r + (kBoxRows + 8) * kPartWords * 4);
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        // the word's operand registers for every tile (4 fields x 4 registers), then one group of
        // activation columns at a time
        uint32_t A[TPW][4][4];
#pragma unroll
        for (int a = 0; a < TPW; ++a) {
          uint32_t wa0, wb0, wa1, wb1;
          merge_planes_offset(u4get(ma[a], e), u4get(sa[a], e), wa0, wb0);
          merge_planes_offset(u4get(mb[a], e), u4get(sb[a], e), wa1, wb1);
#pragma unroll
          for (int i = 0; i < 4; ++i) {                     // field i in place -> 4^i * (t + 2)
            const uint32_t msk = 0x03030303u << (2 * i);
            A[a][i][0] = wa0 & msk;
            A[a][i][1] = wa1 & msk;
            A[a][i][2] = wb0 & msk;
            A[a][i][3] = wb1 & msk;
          }
        }
#pragma unroll
        for (int j = 0; j < G; ++j) {
          // (b0, b1) of fields 0, 1 and of fields 2, 3
          const uint32_t xo = (PACK && j == 1) ? xofs1 : xofs + (uint32_t)(j * 8 * kColWords) * 4;
          const bool live = (PACK && j == 1) ? live1 : (j == 0 ? live0 : true);
          const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
          const uint4 x01 = live ? lds128(st + xo + e * 128) : zero;
          const uint4 x23 = live ? lds128(st + xo + e * 128 + 16) : zero;
#pragma unroll
          for (int a = 0; a < TPW; ++a)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const uint32_t b0 = i < 2 ? u4get(x01, 2 * i) : u4get(x23, 2 * i - 4);
              const uint32_t b1 = i < 2 ? u4get(x01, 2 * i + 1) : u4get(x23, 2 * i - 3);
              mma_u8s8(acc[a][j][i], A[a][i][0], A[a][i][1], A[a][i][2], A[a][i][3], b0, b1);
            }
        }
      }
      if (part == pend - 1) {                                // sums over all of K and E ride in every segment
        if (MP == 1) {
          const uint4 m4 = lds128(st + mofs);               // the NCOL (<= 4) column sums
          tot[0][0][0] = (int)m4.x;
          tot[0][1][0] = (int)m4.y;
          tot[0][2][0] = (int)m4.z;
          tot[0][3][0] = (int)m4.w;
          if (MODE == 0) Etok[0][0] = lds32(st + mofs + 4u * NCOL);
        } else if (PACK) {
          // lane t reads tokens t and (MP = 6) t + 4: their column sums and E
#pragma unroll
          for (int b = 0; b < (MP > 4 ? 2 : 1); ++b) {
            const int m = t + 4 * b < MP ? t + 4 * b : 0;
#pragma unroll
            for (int l = 0; l < kLimbs; ++l) tot[0][l][b] = lds32(st + mofs + 4u * (uint32_t)(l * MP + m));
            Etok[0][b] = lds32(st + mofs + 4u * (uint32_t)(NCOL + m));
          }
        } else {
#pragma unroll
          for (int jj = 0; jj < JJ; ++jj)
#pragma unroll
            for (int b = 0; b < 2; ++b) {
              const int m = 8 * jj + 2 * t + b;
#pragma unroll
              for (int l = 0; l < NL; ++l) tot[jj][l][b] = lds32(st + mofs + 4u * (uint32_t)(l * MP + m));
              if (MODE == 0) Etok[jj][b] = lds32(st + mofs + 4u * (uint32_t)(NCOL + m));
            }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(empty0 + 8 * s);
      if (++s == S) { s = 0; ph ^= 1u; }
    }
    if (!ok) break;
    // ---- outputs of this warp's tiles: exact integer sums, one rounding ----------------------------
    // the field accumulators of each (row, column) combined exactly (the offset is removed below;
    // the signed decode carries the factor 64)
    int V[TPW][G][4];
#pragma unroll
    for (int a = 0; a < TPW; ++a)
#pragma unroll
      for (int j = 0; j < G; ++j)
#pragma unroll
        for (int q = 0; q < 4; ++q)
          V[a][j][q] = acc[a][j][0][q] + (acc[a][j][1][q] >> 2) + (acc[a][j][2][q] >> 4) + (acc[a][j][3][q] >> 6);
    bool emit = true;
    if (slot >= 0) {
      // a block split between CTAs: add this CTA's part sums; the last contributor (per warp)
      // reads the totals back and writes the outputs
      int* sums = reinterpret_cast<int*>(p.xprep + p.scratch_off) + (size_t)slot * kStageRowsT * NCOLP;
      int* counter = reinterpret_cast<int*>(p.xprep + p.scratch_off) + (size_t)p.nslots * kStageRowsT * NCOLP +
                     slot * kCW + warp;
#pragma unroll
      for (int a = 0; a < TPW; ++a)
#pragma unroll
        for (int j = 0; j < G; ++j)
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int col = 8 * j + 2 * t + (q & 1);
            if (col < NCOL)
              atomicAdd(&sums[(a * kBoxRows + warp * 16 + g + 8 * (q >> 1)) * NCOLP + col], V[a][j][q]);
          }
      __threadfence();
      __syncwarp();
      int last = 0;
      if (lane == 0) last = atomicAdd(counter, 1) == need - 1;
      last = __shfl_sync(0xFFFFFFFFu, last, 0);
      if (last) {
        __threadfence();
#pragma unroll
        for (int a = 0; a < TPW; ++a)
#pragma unroll
          for (int j = 0; j < G; ++j)
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int col = 8 * j + 2 * t + (q & 1);
              if (col < NCOL)
                V[a][j][q] = __ldcg(&sums[(a * kBoxRows + warp * 16 + g + 8 * (q >> 1)) * NCOLP + col]);
            }
      } else {
        emit = false;
      }
    }
#pragma unroll
    for (int a = 0; a < TPW && emit; ++a) {
      const int r0 = row_base + a * kBoxRows + g;            // rows r0 (q = 0, 1) and r0 + 8 (q = 2, 3)
      if (MP == 1) {
        int v[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) v[q] = V[a][0][q];
        if (MODE == 1) {
          if (t == 0) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int row = r0 + 8 * h;
              if (row < B.N) {
                const int S1 = v[2 * h] - 2 * tot[0][0][0];
                B.y[row] = __fmul_rn(__fmul_rn(__int2float_rn(S1), sxv[0][0]), f16_bits_to_float(sc_bits[a][h]));
              }
            }
          }
        } else {
          // lane t = 0 holds columns 0 (L3) and 1 (L2), lane t = 1 columns 2 (L1) and 3 (L0)
          int w[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) w[q] = __shfl_down_sync(0xFFFFFFFFu, v[q], 1);
          if (t == 0) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int row = r0 + 8 * h;
              if (row < B.N) {
                const long long D = limb_combine(v[2 * h] - 2LL * tot[0][0][0], v[2 * h + 1] - 2LL * tot[0][1][0],
                                                 w[2 * h] - 2LL * tot[0][2][0], w[2 * h + 1] - 2LL * tot[0][3][0]);
                B.y[row] = (float)((double)D * exp2_i(Etok[0][0] - kLimbFrac) * (double)f16_bits_to_float(sc_bits[a][h]));
              }
            }
          }
        }
      } else if (PACK) {
        // limb l of token m sits in column c = l * MP + m: group c / 8, held by quad lane
        // (c % 8) / 2 as half c % 2 of its row pair; lane t = m % 4 gathers its token's limbs
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int row = r0 + 8 * h;
#pragma unroll
          for (int m = 0; m < MP; ++m) {
            long long L[kLimbs];
#pragma unroll
            for (int l = 0; l < kLimbs; ++l) {
              const int c = l * MP + m;
              L[l] = __shfl_sync(0xFFFFFFFFu, V[a][c >> 3][2 * h + (c & 1)], (lane & ~3) | ((c & 7) >> 1)) -
                     2LL * tot[0][l][m >> 2];
            }
            if (t == (m & 3) && m < M && row < B.N) {
              const long long D = limb_combine(L[0], L[1], L[2], L[3]);
              B.y[(size_t)m * B.N + row] =
                  (float)((double)D * exp2_i(Etok[0][m >> 2] - kLimbFrac) * (double)f16_bits_to_float(sc_bits[a][h]));
            }
          }
        }
      } else {
        // lane (g, t) holds, for rows r0 and r0 + 8, the columns 2t and 2t + 1 of every group:
        // tokens m = 8 jj + 2t + b, with all of their limbs (groups l * JJ + jj)
#pragma unroll
        for (int jj = 0; jj < JJ; ++jj)
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int b = q & 1, h = q >> 1;
            const int m = 8 * jj + 2 * t + b;
            const int row = r0 + 8 * h;
            if (m < M && row < B.N) {
              const float sc = f16_bits_to_float(sc_bits[a][h]);
              if (MODE == 1) {
                const int S1 = V[a][jj][q] - 2 * tot[jj][0][b];
                B.y[(size_t)m * B.N + row] = __fmul_rn(__fmul_rn(__int2float_rn(S1), sxv[jj][b]), sc);
              } else {
                long long Sl[kLimbs];
#pragma unroll
                for (int l = 0; l < kLimbs; ++l) Sl[l] = (long long)V[a][l * JJ + jj][q] - 2LL * tot[jj][l][b];
                const long long D = limb_combine(Sl[0], Sl[1], Sl[2], Sl[3]);
                B.y[(size_t)m * B.N + row] = (float)((double)D * exp2_i(Etok[jj][b] - kLimbFrac) * (double)sc);
              }
            }
          }
      }
    }
    gq += pend - pstart;
    pstart = 0;
    if (++rb == B.units) { rb = 0; ++it; }
  }
  if (!ok && lane == 0) atomicExch(&g_batch_latch, 5);
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

// Token slots, tiles per warp and consumer warps for M rows: the accumulators (tiles x groups x
// fields x 4 registers) stay at or under 64 registers.
void batch_shape(int mode, int M, int& mp, int& tpw, int& cw) {
  if (M == 1 || (mode == 0 && M == 2)) {       // one MMA group: 1 or 4 columns, or 2 x 4 limbs
    mp = M;
    tpw = 2;
    cw = 12;
    return;
  }
  if (mode == 0 && M <= 4) {                    // 4 x 4 limbs in two groups
    mp = 4;
    tpw = 2;
    cw = 11;
    return;
  }
  if (mode == 0 && M <= 6) {                    // 4 x 6 limbs in three groups
    mp = 6;
    tpw = 1;
    cw = 11;
    return;
  }
  mp = M <= 8 ? 8 : 16;                         // int8: one or two groups; bf16 (5..8 rows): four
  tpw = mode == 0 ? 1 : 2;                      // groups, one per limb, so one tile per warp (bf16
  cw = 11;                                      // lists of 9..16 rows run on tern_tc.cu's kernels)
}

template <int MODE, int MP, int TPW, int CW>
cudaError_t launch_stream_kernel(cudaLaunchConfig_t& cfg, const BatchParams& p) {
  static std::atomic<unsigned long long> smem_raised{0};
  cudaError_t e = allow_max_dynamic_smem(k_batch_stream<MODE, MP, TPW, CW>, smem_raised);
  if (e != cudaSuccess) return e;
  cfg.blockDim = dim3((CW + 1) * 32, 1, 1);
  return cudaLaunchKernelEx(&cfg, k_batch_stream<MODE, MP, TPW, CW>, p);
}

}  // namespace

bool plan_batch(BatchParams& p, const uint32_t* const* planes, size_t& smem, size_t& workspace) {
  if (p.M < 1 || p.M > 16) return false;
  int mp = 1, tpw = 2, cw = 12;
  if (p.tc) {
    // tensor-core path (tern_tc.cu): 8 decoder warps own the 128 rows of a box (one TMEM lane
    // each), two boxes per 256-row block; B segments of tc_cols x 512 bytes per part
    if (p.M < 2) return false;
    mp = tc_token_slots(p.mode, p.M);
    cw = tc_consumer_warps();
    tpw = tc_stage_rows() / box_rows(cw);
  } else {
    if (p.mode == 0 && p.M > 8) return false;           // bf16 lists of 9..16 rows: tensor cores only
    batch_shape(p.mode, p.M, mp, tpw, cw);
  }
  p.mp = mp;
  p.tpw = tpw;
  p.cw = cw;
  const int kBoxRows = box_rows(cw), kBoxBytes = box_bytes(cw);
  p.nc = p.tc ? (p.mode == 0 ? 4 * mp : mp) : seg_cols(p.mode, mp);
  p.seg_bytes = p.tc ? tc_segment_bytes(p.mode, mp) : seg_words(p.mode, mp) * 4;
  const int stage_rows = kBoxRows * tpw;
  const int ncolp = 8 * ((p.nc + 7) / 8);                 // scratch columns: 8 per MMA group
  PFN_cuTensorMapEncodeTiled_v12000 encode = encode_fn();
  if (!encode) return false;
  long long total_cost = 0;
  int units = 0, parts = 0;
  size_t xoff = 0;
  for (int i = 0; i < p.count; ++i) {
    BatchItem& it = p.items[i];
    if (it.K % 128 || it.K <= 0 || it.N <= 0) return false;
    it.kp = (it.K + 511) / 512;
    it.unit0 = units;
    it.units = (it.N + stage_rows - 1) / stage_rows;
    it.part0 = parts;
    units += it.units;
    if ((long long)parts + (long long)it.units * it.kp > 0x3FFFFFFF) return false;
    parts += it.units * it.kp;
    it.xoff = (uint32_t)xoff;
    xoff += (size_t)it.kp * p.seg_bytes;
    // cost of the item's parts: every stage of a block costs the same, a partial last block's too
    // (the consumers run the MMAs of all their tiles, and at M = 1 the MMAs take about as long as
    // a full stage's bytes): measured, counting stages rather than bytes made the 0.6B stack 2.5%
    // and the 8B stack 2.2% faster
    total_cost += (long long)it.units * stage_rows * it.kp * 128;
    // planes of row n: mask words [n * K/16, n * K/16 + K/32), its sign words right after
    const cuuint64_t dims[3] = {(cuuint64_t)(it.K / 32), (cuuint64_t)it.N, 2};
    const cuuint64_t strides[2] = {(cuuint64_t)it.K / 4, (cuuint64_t)it.K / 8};   // bytes: row, plane
    const cuuint32_t box[3] = {(cuuint32_t)kPartWords, (cuuint32_t)kBoxRows, 2};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (encode(&p.tmap[i], CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<uint32_t*>(planes[i]), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               p.tc ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_NONE,   // tc: conflict-free row reads
               CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return false;
  }
  p.total_units = units;
  // CTA c starts at the first part whose cost prefix reaches c/G of the total: the split is
  // balanced to one 512-trit part, and a row block may be shared by neighbouring CTAs. A start
  // within four parts of a block boundary moves to it instead: sharing a block costs its CTAs a
  // round of atomics, a fence and a counter, which weighs most where a CTA streams few parts
  // (measured: the 0.6B stack, ~16 parts per CTA, 40.3 -> 37.4 us; the 8B stack unchanged, where
  // only blocks of K = 12288 (24 parts) still split far from their ends).
  constexpr long long kSnapParts = 4;
  const int grid = persistent_grid(parts);
  p.grid = grid;
  {
    int c = 1;
    long long acc = 0;
    p.cta_part[0] = 0;
    for (int i = 0; i < p.count && c < grid; ++i) {
      const BatchItem& it = p.items[i];
      for (int u = 0; u < it.units && c < grid; ++u) {
        const long long cu = (long long)stage_rows * 128;
        const int ustart = it.part0 + u * it.kp;
        while (c < grid && total_cost * c / grid < acc + cu * it.kp) {
          long long off = (total_cost * c / grid - acc + cu - 1) / cu;   // parts of this block before c
          if (off < 0) off = 0;
          if (off <= kSnapParts) off = 0;
          else if (it.kp - off <= kSnapParts) off = it.kp;
          int start = ustart + (int)off;
          if (start < p.cta_part[c - 1]) start = p.cta_part[c - 1];
          p.cta_part[c++] = start;
        }
        acc += cu * it.kp;
      }
    }
    for (; c <= grid; ++c) p.cta_part[c] = parts;
    p.cta_part[grid] = parts;
  }
  // each CTA's first item: a scan of items[] (kernel parameters, read through the constant cache)
  // at the kernel's entry cost the last CTAs of a 112-item list up to 10 us before their first load
  {
    int i = 0;
    for (int c = 0; c < grid; ++c) {
      while (i + 1 < p.count && p.items[i + 1].part0 <= p.cta_part[c]) ++i;
      p.cta_item[c] = (int16_t)i;
    }
  }
  // blocks shared by several CTAs: one scratch slot each, with its contributor count
  auto unit_of = [&](int gpart, int& ustart, int& uend) {
    int i = 0;
    while (i + 1 < p.count && p.items[i + 1].part0 <= gpart) ++i;
    const BatchItem& it = p.items[i];
    const int u = (gpart - it.part0) / it.kp;
    ustart = it.part0 + u * it.kp;
    uend = ustart + it.kp;
    return it.unit0 + u;
  };
  int nslots = 0;
  int slot_unit[160], slot_need[160];
  for (int c = 0; c < grid; ++c) {
    p.cta_split[c] = 0;
    const int lo = p.cta_part[c], hi = p.cta_part[c + 1];
    if (lo >= hi) continue;
    int ends[2] = {lo, hi - 1};
    uint32_t code = 0;
    for (int e = 0; e < 2; ++e) {
      int us, ue;
      const int u = unit_of(ends[e], us, ue);
      if (us >= lo && ue <= hi) continue;               // the block is this CTA's alone
      int sl = -1;
      for (int k = 0; k < nslots; ++k)
        if (slot_unit[k] == u) sl = k;
      if (sl < 0) {
        if (nslots >= 160 || nslots >= 254) return false;
        sl = nslots++;
        slot_unit[sl] = u;
        int need = 0;                                   // CTAs whose range meets [us, ue)
        for (int d = 0; d < grid; ++d)
          if (p.cta_part[d] < p.cta_part[d + 1] && p.cta_part[d] < ue && p.cta_part[d + 1] > us) ++need;
        if (need > 255) return false;
        slot_need[sl] = need;
      }
      code |= ((uint32_t)(sl + 1) | ((uint32_t)slot_need[sl] << 8)) << (16 * e);
    }
    p.cta_split[c] = code;
  }
  p.nslots = nslots;
  // workspace: operand segments, (tc) the token exponents [count][16], then the split sums
  // [slot][rows][ncolp] and counters [slot][cw]
  xoff = (xoff + 15) & ~(size_t)15;
  p.meta_off = (uint32_t)xoff;
  if (p.tc) xoff += (size_t)p.count * 16 * 4;
  p.scratch_off = (uint32_t)xoff;
  p.scratch_words = nslots * (stage_rows * ncolp + cw);
  workspace = xoff + (size_t)p.scratch_words * 4 + 16;
  if (workspace > 0xFFFFFFFFull) return false;
  p.stage_slot_bytes = (tpw * kBoxBytes + p.seg_bytes + 1023) & ~1023;
  const size_t budget = 227 * 1024;
  const size_t fixed = p.tc ? tc_smem_bytes(0, 0) : 1024;
  int stages = (int)((budget - fixed) / (size_t)p.stage_slot_bytes);
  if (stages > 8) stages = 8;
  if (stages < 2) return false;
  p.stages = stages;
  smem = p.tc ? tc_smem_bytes(stages, p.stage_slot_bytes) : 1024 + (size_t)stages * p.stage_slot_bytes;
  return true;
}

cudaError_t read_and_clear_batch_latch(int* out) {
  cudaError_t e = cudaMemcpyFromSymbol(out, g_batch_latch, sizeof(int));
  if (e != cudaSuccess) return e;
  const int zero = 0;
  return cudaMemcpyToSymbol(g_batch_latch, &zero, sizeof(int));
}

void plan_prep(const BatchParams& b, PrepParams& q) {
  q.count = b.count;
  q.mode = b.mode;
  q.M = b.M;
  q.mp = b.mp;
  q.seg_bytes = b.seg_bytes;
  q.xprep = b.xprep;
  q.scratch_off = b.scratch_off;
  q.scratch_words = b.scratch_words;
  q.meta_off = b.meta_off;
  for (int i = 0; i < b.count; ++i) {
    q.items[i].K = b.items[i].K;
    q.items[i].kp = b.items[i].kp;
    q.items[i].xoff = b.items[i].xoff;
  }
}

cudaError_t launch_batch(const BatchParams& p, const PrepParams& q, size_t smem, bool pdl, cudaStream_t st) {
  if (p.tc) return launch_tc(p, q, smem, pdl, st);
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
  // 1. operand segments: one CTA per (item, token slot)
  bool any_pro = false;
  for (int i = 0; i < q.count; ++i) any_pro = any_pro || q.items[i].kind != kProNone;
  cfg.gridDim = dim3(p.count, p.mp, 1);
  cfg.blockDim = dim3(any_pro ? kPrepThreads : kPrepThreadsPlain, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cudaError_t e = cudaSuccess;
  if (any_pro) {
    e = cudaLaunchKernelEx(&cfg, k_batch_prep<kPrepThreads, true>, q);
  } else {
    static std::atomic<unsigned long long> carveout_set{0};
    e = prefer_max_shared_carveout(k_batch_prep<kPrepThreadsPlain, false>, carveout_set);
    if (e == cudaSuccess) e = cudaLaunchKernelEx(&cfg, k_batch_prep<kPrepThreadsPlain, false>, q);
  }
  if (e != cudaSuccess) return e;
  // 2. the stream (always programmatically dependent on the prep launch)
  cudaLaunchAttribute attr2[1];
  attr2[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr2[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr2;
  cfg.numAttrs = 1;
  cfg.gridDim = dim3(p.grid, 1, 1);
  cfg.dynamicSmemBytes = smem;
  if (p.mode == 0) {
    if (p.mp == 1) return launch_stream_kernel<0, 1, 2, 12>(cfg, p);
    if (p.mp == 2) return launch_stream_kernel<0, 2, 2, 12>(cfg, p);
    if (p.mp == 4) return launch_stream_kernel<0, 4, 2, 11>(cfg, p);
    if (p.mp == 6) return launch_stream_kernel<0, 6, 1, 11>(cfg, p);
    if (p.mp == 8) return launch_stream_kernel<0, 8, 1, 11>(cfg, p);
    return cudaErrorInvalidValue;
  }
  if (p.mp == 1) return launch_stream_kernel<1, 1, 2, 12>(cfg, p);
  if (p.mp == 8) return launch_stream_kernel<1, 8, 2, 11>(cfg, p);
  return launch_stream_kernel<1, 16, 2, 11>(cfg, p);
}

}  // namespace tern
