// Small-M batched GEMM on the 5th-generation tensor cores (tcgen05, weights held in TMEM).
//
//   for every item i:  y_i[m][n] = scale_i[n] * sum_k t_i[n][k] * x_i[m][k],   m < M <= 16
//
// The draft-verify pass of speculative decoding runs every linear of the stack at M = k + 1
// activation rows (PyTorchKR review "Fermion Research, 3진 계열 포맷으로 직접 학습한 Neutrino-1
// 모델군 3종 공개", section "검증된 추측 디코딩": 1-7 drafted tokens checked in one batched pass);
// the weights still stream once, so the pass should cost what M = 1 costs. With bf16 activations
// held as four exact int8 limbs (tern_device.cuh), M rows make 4M operand columns, and the
// warp-level mma.sync path of tern_batch.cu spends more time in the tensor pipe than the weights
// take to arrive once M >= 5. Here the product runs on tcgen05 instead:
//   * the operand preparation (k_tc_prep, one CTA per item and token slot) writes each item's
//     activation columns (four limbs per token, or the int8 q) as the MMA's B operand: per 512-trit
//     part, four 128-trit chunks of N rows x 128 bytes in the 128-byte-swizzled K-major layout the
//     tensor core reads from shared memory, in the decode's k order (permute_i8_half); an item
//     with a prologue (tern_prologue.cuh) computes its activation first;
//   * k_tc_stream (one CTA per SM) walks the same balanced (row block, part) sequence as the
//     mma.sync stream, with row blocks of 256 rows (two groups of 128):
//       warp 0      producer: per stage, the block's mask and sign words (tensor TMA, 64-byte
//                   swizzle, no multicast) and the part's B segment (bulk copy);
//       warp 1      allocates 512 TMEM columns; one lane issues tcgen05.mma kind::i8 with A (the
//                   weights) in TMEM and B in shared memory: M = 128 rows, N = the operand
//                   columns, K = 32 per instruction, int32 accumulators in TMEM;
//       warps 2..17 sixteen decoders, two per (row group, TMEM lane quarter): each thread owns one
//                   weight row (a TMEM lane) and, for alternate 128-trit chunks of a stage,
//                   decodes the row's 32-trit words into signed bytes 64 * t (one shift and one
//                   AND per register, the signed decode of tern_device.cuh) and stores them into
//                   TMEM with tcgen05.st through four A slots; at the end of a row block the
//                   decoders of even chunks read their row's accumulators (tcgen05.ld) and write
//                   the outputs.
// Every sum is an exact integer (|64 t L| <= 2^13 per product, K <= 12288), so the outputs equal
// the mma.sync path's bit for bit: int8 mode y = ((float)acc * s_x) * scale with two fp32
// roundings, bf16 mode one fp64 -> fp32 rounding of the recombined limb sums. Every wait is bounded;
// a kernel that gives up latches TERN_ETIMEOUT, drains what it issued, frees its TMEM and returns.
#include <atomic>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "tern_device.cuh"
#include "tern_kernels.h"
#include "tern_prologue.cuh"

namespace tern {

__device__ int g_tc_latch = 0;

namespace {

constexpr int kRG = 2;                           // row groups of 128 per row block
constexpr int kRows = 128 * kRG;                 // rows of a row block (one stage)
constexpr int kBox = 2 * 128 * 64;               // bytes of one row group's box: 2 planes x 128 rows x 64 B
constexpr int kNA = 4;                           // TMEM A slots (one 128-trit chunk of both row groups)
constexpr int kEpiWarps = 8;                     // one per (row group, TMEM lane quarter): the epilogue
constexpr int kDecWarps = 2 * kEpiWarps;         // decoders: the same, once per chunk parity
constexpr int kTcThreads = (2 + kDecWarps) * 32;
constexpr int kTmemCols = 512;
constexpr int kDCol = 0;                         // accumulators: row group g at columns 64 g ..
constexpr int kACol = 64 * kRG;                  // A slots: slot a, row group g at kACol + 32 (kRG a + g)
static_assert(kACol + 32 * kRG * kNA <= 512, "TMEM columns");
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
// Spin (no suspension) until the phase completes: for the single MMA-issuing thread, whose waits
// are short and on the critical path. Bounded like mbar_wait.
__device__ __forceinline__ bool mbar_spin(uint32_t bar, uint32_t parity) {
  const long long t0 = clock64();
  for (uint32_t i = 0;; ++i) {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    if (done) return true;
    if ((i & 1023u) == 1023u && clock64() - t0 > 8000000000LL) return false;   // ~4 s
  }
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
// Tiled 3-d tensor load (no multicast): the box at (word c0, row c1, plane c2).
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
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// K-major, 128-byte-swizzled shared-memory operand descriptor: start address, leading byte offset
// 16 (unused when swizzled), stride byte offset 1024 (8 rows x 128 B), version 1, swizzle 128 B.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)(16u >> 4) << 16;
  d |= (uint64_t)(1024u >> 4) << 32;
  d |= (uint64_t)1u << 46;
  d |= (uint64_t)2u << 61;
  return d;
}
// Instruction descriptor of tcgen05.mma kind::i8: int32 accumulator, A and B signed 8-bit, both
// K-major, M = 128, N columns.
template <int N>
constexpr uint32_t idesc_i8() {
  return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}
// D[128 x N] (+)= A[128 x 32] (TMEM) * B[N x 32]^T (shared memory)
__device__ __forceinline__ void mma_i8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc, uint32_t accum) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n}\n"
      ::"r"(d_tmem), "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accum)
      : "memory");
}
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
// 32 consecutive columns of this thread's TMEM lane <- r[0..31]
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),
        "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),
        "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
// 8 consecutive columns of this thread's TMEM lane -> r[0..7] (waits for the load)
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, int (&r)[8]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];\n"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ double exp2_i(int e) { return __longlong_as_double((long long)(e + 1023) << 52); }

// Operand columns of the tensor-core path: bf16 mode four limbs per token slot (column 4 m + l,
// limb l top first), int8 mode one (column m).
__host__ __device__ constexpr int tc_cols(int mode, int mp) { return mode == 0 ? 4 * mp : mp; }

// ---------------------------------------------------------------------------------------------
// Operand preparation: one CTA per (item, token slot m). Writes the slot's columns of every part's
// B segment (zeros past K and for slots m >= M), the token's exponent E (bf16 mode) into the
// metadata, and clears the split-block scratch. An item with a prologue first computes its bf16 row
// into shared memory (tern_prologue.cuh, the arithmetic and thread count of tern_act_prologue), then
// encodes from there; int8 mode quantises that row here (tern_quantize_act's quantiser), writing s_x
// and, if asked, the prepared activation.
constexpr int kTcPrepThreads = 256;
constexpr int kTcPrepMaxK = 12288;
__global__ void __launch_bounds__(kTcPrepThreads) k_tc_prep(const __grid_constant__ PrepParams p) {
  const PrepItem& it = p.items[blockIdx.x];
  const int m = blockIdx.y;
  const int K = it.K, KP = it.kp;
  const int nc = tc_cols(p.mode, p.mp);
  const bool live = m < p.M;
  const bool pro = it.kind != kProNone;
  uint8_t* blk = p.xprep + it.xoff;
  __shared__ float red[kTcPrepThreads / 32];
  __shared__ double dred[kTcPrepThreads / 32];
  __shared__ int Esh;
  __shared__ float ssh;
  __shared__ __align__(16) uint16_t xs[kTcPrepMaxK];         // a prologue item's prepared bf16 row
  pdl_wait();
  // the stream kernel may get resident now: its producer prefetches weights, and it waits for this
  // grid's completion before it reads a segment
  pdl_launch_dependents();
  {
    uint32_t* scr = reinterpret_cast<uint32_t*>(p.xprep + p.scratch_off);
    const int nct = gridDim.x * gridDim.y, ct = blockIdx.y * gridDim.x + blockIdx.x;
    for (int i = ct * blockDim.x + threadIdx.x; i < p.scratch_words; i += nct * blockDim.x) scr[i] = 0u;
  }
  float amax = 0.0f;
  if (live && pro) {
    const size_t row_elems = (size_t)K * (it.kind == kProSwiGLU ? 2 : 1);
    const void* src = it.kind == kProBF16 ? static_cast<const void*>(static_cast<const uint16_t*>(it.x) + (size_t)m * K)
                                          : static_cast<const void*>(static_cast<const float*>(it.x) + (size_t)m * row_elems);
    const double r =
        it.kind == kProRMSNorm ? rmsnorm_r<kTcPrepThreads>(static_cast<const float*>(src), K, it.eps, dred) : 1.0;
    uint16_t* xo = (p.mode == 0 && it.xout) ? static_cast<uint16_t*>(it.xout) + (size_t)m * K : nullptr;
    for (int k = threadIdx.x * 8; k < K; k += kTcPrepThreads * 8) {
      const uint4 v = prologue8(it.kind, src, it.gain, K, k, r);
      *reinterpret_cast<uint4*>(xs + k) = v;
      if (xo) *reinterpret_cast<uint4*>(xo + k) = v;
      amax = fmaxf(amax, absmax8(v));
    }
  } else if (live && p.mode == 0) {
    const uint16_t* xb = static_cast<const uint16_t*>(it.x) + (size_t)m * K;
    for (int k = threadIdx.x * 8; k < K; k += kTcPrepThreads * 8) amax = fmaxf(amax, absmax8(ld_nc(xb + k)));
  }
  int E = 0;
  float sq = 0.0f;
  if (p.mode == 0 || pro) {
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
    __syncthreads();
    if (threadIdx.x == 0) {
      float mx = red[0];
      for (int i = 1; i < kTcPrepThreads / 32; ++i) mx = fmaxf(mx, red[i]);
      if (p.mode == 0) {
        Esh = limb_exponent(mx);
        reinterpret_cast<int*>(p.xprep + p.meta_off)[blockIdx.x * 16 + m] = Esh;
      } else {
        ssh = __fdiv_rn(mx, 127.0f);                          // the per-token quantiser's scale
        if (live) it.sx_out[m] = ssh;
      }
    }
    __syncthreads();
    E = Esh;
    sq = ssh;
  }
  int8_t* qo = (p.mode == 1 && pro && live && it.xout) ? static_cast<int8_t*>(it.xout) + (size_t)m * K : nullptr;
  // one 16-element half of a 32-trit word per iteration, over every part (past K: zeros)
  const size_t part_bytes = (size_t)4 * nc * 128;
  for (int v = threadIdx.x; v < KP * 32; v += kTcPrepThreads) {
    const int part = v >> 5, w = (v & 31) >> 1, h = v & 1;
    const int k = part * 512 + 32 * w + 16 * h;
    const int chunk = w >> 2, u = 2 * (w & 3) + h;      // 16-byte unit of the 128-byte row
    uint8_t* base = blk + part * part_bytes + (size_t)chunk * nc * 128;
    const bool have = live && k < K;
    // the 16 bf16 values (prologue row or bf16 input) of this half
    uint32_t wv[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
    if (have && (pro || p.mode == 0)) {
      const uint16_t* xb = pro ? xs + k : static_cast<const uint16_t*>(it.x) + (size_t)m * K + k;
      const uint4 a = pro ? *reinterpret_cast<const uint4*>(xb) : ld_nc(xb);
      const uint4 b = pro ? *reinterpret_cast<const uint4*>(xb + 8) : ld_nc(xb + 8);
      wv[0] = a.x; wv[1] = a.y; wv[2] = a.z; wv[3] = a.w; wv[4] = b.x; wv[5] = b.y; wv[6] = b.z; wv[7] = b.w;
    }
    if (p.mode == 1) {
      uint4 q = make_uint4(0u, 0u, 0u, 0u);
      if (have) {
        if (pro) {
          uint32_t qw[4] = {0u, 0u, 0u, 0u};
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const uint32_t bits = (e & 1) ? (wv[e >> 1] >> 16) : (wv[e >> 1] & 0xFFFFu);
            qw[e >> 2] |= (uint32_t)(uint8_t)(int8_t)quant_i8(bf16_bits_to_float(bits), sq) << (8 * (e & 3));
          }
          q = make_uint4(qw[0], qw[1], qw[2], qw[3]);
          if (qo) *reinterpret_cast<uint4*>(qo + k) = q;
        } else {
          q = ld_nc(static_cast<const int8_t*>(it.x) + (size_t)m * K + k);
        }
        q = permute_i8_half(q);
      }
      const int n = m;
      *reinterpret_cast<uint4*>(base + n * 128 + ((u ^ (n & 7)) << 4)) = q;
    } else {
      uint32_t l[4][4] = {};
      if (have) limbs_of_bf16<4>(wv, E, l);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int n = 4 * m + c;
        const uint4 q = permute_i8_half(make_uint4(l[c][0], l[c][1], l[c][2], l[c][3]));
        *reinterpret_cast<uint4*>(base + n * 128 + ((u ^ (n & 7)) << 4)) = q;
      }
    }
  }
}

// ---------------------------------------------------------------------------------------------
// MODE: 0 bf16 / 1 int8 activations; MP: token slots (4, 8 or 16 in bf16 mode; 8 or 16 in int8).
template <int MODE, int MP>
__global__ void __launch_bounds__(kTcThreads, 1) k_tc_stream(const __grid_constant__ BatchParams p) {
  constexpr int N = tc_cols(MODE, MP);
  static_assert(N % 8 == 0 && N <= 64, "MMA N");
  constexpr uint32_t kIdesc = idesc_i8<N>();
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;           // 1 KB aligned: swizzled boxes and segments
  const int S = p.stages;
  const uint32_t slot_bytes = (uint32_t)p.stage_slot_bytes;
  const uint32_t ring = base;
  const uint32_t bars = base + (uint32_t)S * slot_bytes;  // [full S][empty S][afull 4][aempty 4][dfull][done][tmem]
  const uint32_t full0 = bars, empty0 = bars + 8 * S, afull0 = bars + 16 * S, aempty0 = afull0 + 8 * kNA;
  const uint32_t dfull = aempty0 + 8 * kNA, done_bar = dfull + 8, tmem_slot = done_bar + 8;
  const uint32_t* tmem_slot_ptr = reinterpret_cast<const uint32_t*>(smem_raw + (tmem_slot - raw));

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g0 = p.cta_part[blockIdx.x], g1 = p.cta_part[blockIdx.x + 1];

  if (threadIdx.x == 0) {
    for (int i = 0; i < S; ++i) {
      mbar_init(full0 + 8 * i, 1);
      mbar_init(empty0 + 8 * i, 1);
    }
    for (int a = 0; a < kNA; ++a) {
      mbar_init(afull0 + 8 * a, kEpiWarps);                 // the decoder warps of the chunk it holds
      mbar_init(aempty0 + 8 * a, 1);
    }
    mbar_init(dfull, 1);
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
  pdl_launch_dependents();
  bool ok = true;

  // item, row block and part of the first stage
  const int first_item = g1 > g0 ? p.cta_item[blockIdx.x] : 0;
  const int fkp = p.items[first_item].kp;
  const int first_rb = g1 > g0 ? (g0 - p.items[first_item].part0) / fkp : 0;
  const int first_part = g1 > g0 ? (g0 - p.items[first_item].part0) - first_rb * fkp : 0;
  const int n_stages = g1 > g0 ? g1 - g0 : 0;

  if (warp == 0) {
    // ====================== producer (lane 0) ======================
    if (lane == 0 && n_stages > 0) {
      const int pre = n_stages < S ? n_stages : S;
      int it = first_item, rb = first_rb, part = first_part;
      // 1. the weights of the first stages (they do not depend on earlier kernels)
      for (int q = 0; q < pre; ++q) {
        const BatchItem& B = p.items[it];
        const uint32_t bar = full0 + 8 * q, dst = ring + (uint32_t)q * slot_bytes;
        int boxes = 0;
        for (int b = 0; b < kRG; ++b) boxes += (rb * kRows + b * 128 < B.N) ? 1 : 0;
        mbar_arrive_expect_tx(bar, (uint32_t)(boxes * kBox + p.seg_bytes));
        for (int b = 0; b < boxes; ++b) tma_load_3d(dst + b * kBox, &p.tmap[it], part * 16, rb * kRows + b * 128, 0, bar);
        if (++part == B.kp) {
          part = 0;
          if (++rb == B.units) { rb = 0; ++it; }
        }
      }
      pdl_wait();
      // 2. every stage's operand segment and, past the first S, its weights once the slot is free
      it = first_item; rb = first_rb; part = first_part;
      int s = 0, nq = 0;
      uint32_t ph = 0;
      for (int q = 0; q < n_stages && ok; ++q) {
        const BatchItem& B = p.items[it];
        const uint32_t bar = full0 + 8 * s, dst = ring + (uint32_t)s * slot_bytes;
        if (q >= S) {
          if (!(ok = mbar_wait(empty0 + 8 * s, ph ^ 1u))) break;
          int boxes = 0;
          for (int b = 0; b < kRG; ++b) boxes += (rb * kRows + b * 128 < B.N) ? 1 : 0;
          mbar_arrive_expect_tx(bar, (uint32_t)(boxes * kBox + p.seg_bytes));
          for (int b = 0; b < boxes; ++b) tma_load_3d(dst + b * kBox, &p.tmap[it], part * 16, rb * kRows + b * 128, 0, bar);
        }
        bulk_g2s(dst + kRG * kBox, p.xprep + B.xoff + (size_t)part * p.seg_bytes, (uint32_t)p.seg_bytes, bar);
        ++nq;
        if (++part == B.kp) {
          part = 0;
          if (++rb == B.units) { rb = 0; ++it; }
        }
        if (++s == S) { s = 0; ph ^= 1u; }
      }
      // do not leave with copies in flight (on the error path too): wait for the last stages issued.
      // A wait gives up only at some q >= S, before that stage's weights are issued, so every copy
      // in flight belongs to one of the stages [0, nq), each issued in full.
      for (int q = nq > S ? nq - S : 0; q < nq; ++q)
        if (!mbar_wait(full0 + 8 * (q % S), (uint32_t)((q / S) & 1))) { ok = false; break; }
    }
  } else if (warp == 1) {
    // ====================== MMA issue (lane 0) ======================
    if (lane == 0 && n_stages > 0) {
      int it = first_item, rb = first_rb, part = first_part;
      int s = 0, ac = 0;
      uint32_t ph = 0;
      bool first_of_block = true;
      for (int q = 0; q < n_stages && ok; ++q) {
        const BatchItem& B = p.items[it];
        const bool last_of_block = (part == B.kp - 1) || (q == n_stages - 1);
        if (!(ok = mbar_spin(full0 + 8 * s, ph))) break;
        // the stage's four chunks fill A slots 0..3 in order (kNA == 4), so every slot index, TMEM
        // address and descriptor offset below is a constant of the unrolled code: a straight run of
        // MMAs issues at the tensor core's own pace, a rolled loop around them costs far more
        static_assert(kNA == 4, "one A slot per chunk of a stage");
        const uint32_t aph = (uint32_t)((ac / kNA) & 1);
        const uint64_t b0 = smem_desc_sw128(ring + (uint32_t)s * slot_bytes + kRG * kBox);
        const uint32_t acc0 = first_of_block ? 0u : 1u;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          if (ok) ok = mbar_spin(afull0 + 8 * c, aph);
          if (ok) {
            tc_fence_after();
#pragma unroll
            for (int g = 0; g < kRG; ++g)
#pragma unroll
              for (int ks = 0; ks < 4; ++ks)
                mma_i8_ts(tmem + (uint32_t)(kDCol + 64 * g), tmem + (uint32_t)(kACol + 32 * (kRG * c + g) + 8 * ks),
                          b0 + (uint64_t)((c * N * 128 + 32 * ks) >> 4), kIdesc, (c == 0 && ks == 0) ? acc0 : 1u);
            mma_commit(aempty0 + 8 * c);                  // the A slot is free once these MMAs are done
          }
        }
        ac += 4;
        if (!ok) break;
        mma_commit(empty0 + 8 * s);                       // the stage too (B read, planes decoded)
        if (last_of_block) mma_commit(dfull);             // the block's accumulators are complete
        first_of_block = last_of_block;
        if (++part == B.kp) {
          part = 0;
          if (++rb == B.units) { rb = 0; ++it; }
        }
        if (++s == S) { s = 0; ph ^= 1u; }
      }
      // every MMA issued has completed once done_bar flips
      mma_commit(done_bar);
      if (!mbar_wait(done_bar, 0)) ok = false;
    }
  } else {
    // ====================== decoders / epilogue ======================
    const int d = warp - 2;                                // 0 .. 15
    const int g = (d >> 2) & 1;                            // row group
    const int cp = d >> 3;                                 // chunks cp and cp + 2 of every stage
    const int de = d & 7;                                  // epilogue warp index (cp == 0 warps)
    const int quarter = warp & 3;                          // TMEM lanes 32 quarter .. + 31
    const int r = 32 * quarter + lane;                     // row within the group
    const uint32_t lane_addr = (uint32_t)(32 * quarter) << 16;
    const uint32_t split = p.cta_split[blockIdx.x];
    const int slot_first = (int)(split & 0xFFu) - 1, need_first = (int)((split >> 8) & 0xFFu);
    const int slot_last = (int)((split >> 16) & 0xFFu) - 1, need_last = (int)(split >> 24);
    constexpr int NCOLP = N;
    int it = first_item, rb = first_rb, part = first_part;
    int s = 0, blk = 0;
    uint32_t ph = 0;
    int gq = g0;                                           // global part of the block's first stage
    int pstart = first_part;
    for (int q = 0; q < n_stages && ok; ++q) {
      const BatchItem& B = p.items[it];
      const bool last_of_block = (part == B.kp - 1) || (q == n_stages - 1);
      if (!(ok = mbar_wait(full0 + 8 * s, ph))) break;
      const uint32_t box = ring + (uint32_t)s * slot_bytes + (uint32_t)(g * kBox);
      for (int c = cp; c < 4 && ok; c += 2) {
        const int ac = 4 * q + c, a = ac % kNA, use = ac / kNA;   // chunks fill the A slots in turn
        if (use > 0) {
          if (!(ok = mbar_wait(aempty0 + 8 * a, (uint32_t)((use - 1) & 1)))) break;
          tc_fence_after();                                 // the MMAs that read the slot are done
        }
        // words 4c .. 4c + 3 of this row: 16-byte chunk c of its 64-byte row, 64-byte swizzle
        const uint32_t off = (uint32_t)(r * 64 + ((c ^ ((r >> 1) & 3)) << 4));
        const uint4 mw = lds128(box + off), sw = lds128(box + 128 * 64 + off);
        const uint32_t mwv[4] = {mw.x, mw.y, mw.z, mw.w}, swv[4] = {sw.x, sw.y, sw.z, sw.w};
        uint32_t A[32];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          uint32_t wa, wb;
          merge_planes(mwv[e], swv[e], wa, wb);
          A[8 * e + 0] = dec_i8<0>(wa, wb);
          A[8 * e + 1] = dec_i8<1>(wa, wb);
          A[8 * e + 2] = dec_i8<2>(wa, wb);
          A[8 * e + 3] = dec_i8<3>(wa, wb);
          A[8 * e + 4] = dec_i8<4>(wa, wb);
          A[8 * e + 5] = dec_i8<5>(wa, wb);
          A[8 * e + 6] = dec_i8<6>(wa, wb);
          A[8 * e + 7] = dec_i8<7>(wa, wb);
        }
        tmem_st32(tmem + lane_addr + (uint32_t)(kACol + 32 * (kRG * a + g)), A);
        asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(afull0 + 8 * a);
      }
      if (!ok) break;
      if (last_of_block) {
        const int pend = part + 1;                            // this CTA's parts of the block: [pstart, pend)
        if (cp == 0) {
          // ---- the block's outputs: this thread's row, all N accumulator columns ----
          if (!(ok = mbar_wait(dfull, (uint32_t)(blk & 1)))) break;
          tc_fence_after();
          const int row = rb * kRows + g * 128 + r;
          int slot = -1, need = 0;
          if (gq == g0) { slot = slot_first; need = need_first; }
          if (gq + (pend - pstart) == g1 && slot_last >= 0) { slot = slot_last; need = need_last; }
          int V[N];
#pragma unroll
          for (int c8 = 0; c8 < N / 8; ++c8) {
            int t8[8];
            tmem_ld8(tmem + lane_addr + (uint32_t)(kDCol + 64 * g + 8 * c8), t8);
#pragma unroll
            for (int j = 0; j < 8; ++j) V[8 * c8 + j] = t8[j] >> 6;      // exact: every term is 64 * t * x
          }
          tc_fence_before();
          bool emit = true;
          if (slot >= 0) {
            int* sums = reinterpret_cast<int*>(p.xprep + p.scratch_off) + (size_t)slot * kRows * NCOLP;
            int* counter = reinterpret_cast<int*>(p.xprep + p.scratch_off) + (size_t)p.nslots * kRows * NCOLP +
                           slot * kEpiWarps + de;
            int* mine = sums + (size_t)(g * 128 + r) * NCOLP;
#pragma unroll
            for (int j = 0; j < N; ++j) atomicAdd(mine + j, V[j]);
            __threadfence();
            __syncwarp();
            int last = 0;
            if (lane == 0) last = atomicAdd(counter, 1) == need - 1;
            last = __shfl_sync(0xFFFFFFFFu, last, 0);
            if (last) {
              __threadfence();
#pragma unroll
              for (int j = 0; j < N; ++j) V[j] = __ldcg(mine + j);
            } else {
              emit = false;
            }
          }
          if (emit && row < B.N) {
            const double sc = (double)f16_bits_to_float(B.scale[row]);
            if (MODE == 1) {
#pragma unroll
              for (int m = 0; m < MP; ++m)
                if (m < p.M) B.y[(size_t)m * B.N + row] = __fmul_rn(__fmul_rn(__int2float_rn(V[m]), B.sx[m]), (float)sc);
            } else {
              const int* Em = reinterpret_cast<const int*>(p.xprep + p.meta_off) + it * 16;
#pragma unroll
              for (int m = 0; m < MP; ++m)
                if (m < p.M) {
                  const long long D = limb_combine(V[4 * m], V[4 * m + 1], V[4 * m + 2], V[4 * m + 3]);
                  B.y[(size_t)m * B.N + row] = (float)((double)D * exp2_i(Em[m] - kLimbFrac) * sc);
                }
            }
          }
        }
        ++blk;
        gq += pend - pstart;
        pstart = 0;
      }
      if (++part == B.kp) {
        part = 0;
        if (++rb == B.units) { rb = 0; ++it; }
      }
      if (++s == S) { s = 0; ph ^= 1u; }
    }
  }

  if (!ok) atomicExch(&g_tc_latch, 5);
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

template <int MODE, int MP>
cudaError_t launch_tc_stream(cudaLaunchConfig_t& cfg, const BatchParams& p) {
  static std::atomic<unsigned long long> raised{0};
  cudaError_t e = allow_max_dynamic_smem(k_tc_stream<MODE, MP>, raised);
  if (e != cudaSuccess) return e;
  return cudaLaunchKernelEx(&cfg, k_tc_stream<MODE, MP>, p);
}

}  // namespace

int tc_token_slots(int mode, int M) {
  if (mode == 0) return M <= 4 ? 4 : (M <= 8 ? 8 : 16);
  return M <= 8 ? 8 : 16;
}
int tc_segment_bytes(int mode, int mp) { return tc_cols(mode, mp) * 512; }
int tc_stage_rows() { return kRows; }
// The plan's warps per TMA box (box_rows = 16 per warp: 128 rows) and split counters per slot (the
// kernel uses kEpiWarps of them).
int tc_consumer_warps() { return 8; }   // 8 x 16 = 128 rows per box
// 1 KB of alignment slack, the ring, then the barriers (16 per stage, 16 per A slot, 20 more)
constexpr int kBarBytes = 512;
static_assert(16 * 8 + 16 * kNA + 20 <= kBarBytes, "barrier area");
size_t tc_smem_bytes(int stages, int slot_bytes) { return 1024 + (size_t)stages * slot_bytes + kBarBytes; }

cudaError_t launch_tc(const BatchParams& p, const PrepParams& q, size_t smem, bool pdl, cudaStream_t st) {
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
  cfg.gridDim = dim3(p.count, p.mp, 1);
  cfg.blockDim = dim3(kTcPrepThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cudaError_t e = cudaLaunchKernelEx(&cfg, k_tc_prep, q);
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr2[1];
  attr2[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr2[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t c2 = {};
  c2.attrs = attr2;
  c2.numAttrs = 1;
  c2.stream = st;
  c2.gridDim = dim3(p.grid, 1, 1);
  c2.blockDim = dim3(kTcThreads, 1, 1);
  c2.dynamicSmemBytes = smem;
  if (p.mode == 0) {
    if (p.mp == 4) return launch_tc_stream<0, 4>(c2, p);
    if (p.mp == 8) return launch_tc_stream<0, 8>(c2, p);
    if (p.mp == 16) return launch_tc_stream<0, 16>(c2, p);
  } else {
    if (p.mp == 8) return launch_tc_stream<1, 8>(c2, p);
    if (p.mp == 16) return launch_tc_stream<1, 16>(c2, p);
  }
  return cudaErrorInvalidValue;
}

cudaError_t read_and_clear_tc_latch(int* out) {
  cudaError_t e = cudaMemcpyFromSymbol(out, g_tc_latch, sizeof(int));
  if (e != cudaSuccess) return e;
  const int zero = 0;
  return cudaMemcpyToSymbol(g_tc_latch, &zero, sizeof(int));
}

}  // namespace tern
