// Loader-side kernels: packing trits into the two-plane layout, the base-3 transport in both
// directions, and per-row occupancy counts: streaming integer kernels whose roofline is HBM.
//
// Sources: weights packed at rest and decoded inside the matrix kernels (aiatolah.com,
// "Neutrino-1 8B: modelo ternario de 3,88 GB roda em GPU e laptop", second paragraph); the
// transport form of the ternary lane expands bit-exactly into the container (PyTorchKR review
// "Fermion Research, 3진 계열 포맷으로 직접 학습한 Neutrino-1 모델군 3종 공개", section
// "3진 계열이라는 이름의 실체"); per-tensor zero / +1 / -1 occupancy (same review, section
// "출하된 컨테이너를 직접 읽기: 62.63%의 침묵"). The packed layout is defined in include/tern.h.
#include <cstdint>
#include <cuda_runtime.h>

#include "tern_device.cuh"
#include "tern_kernels.h"

namespace tern {
namespace {

__device__ __forceinline__ void set_flag(int32_t* flag) { atomicExch(flag, 1); }

// Byte -> five trits as (mask5 | sign5 << 16), in natural order; all ones marks an invalid byte
// (> 242), which also sets bit 31 of the OR of a run's entries.
__device__ __forceinline__ void build_base3_lut(uint32_t* lut) {
  for (int b = threadIdx.x; b < 256; b += blockDim.x) {
    uint32_t e = 0xFFFFFFFFu;
    if (b < 243) {
      int v = b;
      uint32_t m = 0, s = 0;
      for (int i = 0; i < 5; ++i) {
        const int d = v % 3;
        v /= 3;
        m |= (uint32_t)(d != 1) << i;
        s |= (uint32_t)(d == 0) << i;
      }
      e = m | (s << 16);
    }
    lut[b] = e;
  }
}

// Natural-order bits -> the layout's order: bit j moves to p(j), which swaps bits 0 and 4 of
// the index j (one delta swap: positions with j0 = 1, j4 = 0 trade places with j + 15).
__device__ __forceinline__ uint32_t to_mask_order(uint32_t x) {
  const uint32_t t = lop3<0x28u>(x >> 15, x, 0x0000AAAAu);    // ((x >> 15) ^ x) & 0xAAAA
  return lop3<0x96u>(x, t, t << 15);                         // x ^ t ^ (t << 15)
}

// int8 trits -> planes: one thread per 32-trit word (32 bytes in, one mask and one sign word
// out). A single tensor puts its rows on the grid's y axis, so no index needs a division; a
// batch of tensors walks work units of 16 rows x 128 words in one persistent launch. In a valid
// trit byte
// (0x00, 0x01 or 0xFF) bit 0 is the mask bit and bit 7 the sign bit; one multiply by
// 1 + 2^7 + 2^14 + 2^21 gathers those bits of a word's four bytes into four adjacent bits (the
// partial products never overlap, so there are no carries): mask bits of bytes 0..3 land at
// bits 21..24, sign bits at 28..31. A byte is valid iff its bits 1..7 are all equal and bit 1
// set implies bit 0 set.
constexpr int kPackThreads = 128;
constexpr int kPackUnitRows = 16;                 // rows of one batched work unit
// One 32-trit word: 32 bytes in, the mask and sign words out (bit order of the layout).
__device__ __forceinline__ void pack_word(const int8_t* __restrict__ src, uint32_t* __restrict__ planes, int row,
                                          int col, int KM, uint32_t& bad) {
  const uint4* q = reinterpret_cast<const uint4*>(src + ((int64_t)row * KM + col) * 32);
  const uint4 v0 = ld_stream(q), v1 = ld_stream(q + 1);
  const uint32_t b[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
  uint32_t m = 0u, s = 0u;
#pragma unroll
  for (int k = 0; k < 8; ++k) {                      // trits 4k .. 4k+3 in natural order
    const uint32_t x = b[k], y = x >> 1;
    // gathered nibble at bits 21..24 (mask) / 28..31 (sign), moved to bits 4k..4k+3; the other
    // partial products land outside the nibble's place and are masked off
    const uint32_t gm = (x & 0x01010101u) * 0x00204081u, gs = (x & 0x80808080u) * 0x00204081u;
    const uint32_t um = 4 * k <= 21 ? gm >> (21 - 4 * k) : gm << (4 * k - 21);
    const uint32_t us = gs >> (28 - 4 * k);
    m = lop3<0xEAu>(um, 0xFu << (4 * k), m);         // m | (um & nibble)
    s = lop3<0xEAu>(us, 0xFu << (4 * k), s);
    bad = lop3<0xFEu>(bad, lop3<0x28u>(x, y, 0x7E7E7E7Eu), lop3<0x20u>(y, x, 0x01010101u));
  }
  const uint32_t sp = to_mask_order(s);
  uint32_t* row_p = planes + (int64_t)row * (2 * (int64_t)KM);
  row_p[col] = to_mask_order(m);
  row_p[KM + col] = (sp << 1) | (sp >> 31);          // the sign bit sits one above its mask bit
}

__global__ void __launch_bounds__(kPackThreads) k_pack_trits(const int8_t* __restrict__ src, int32_t N, int32_t KM,
                                                             uint32_t* __restrict__ planes, int32_t* __restrict__ flag) {
  const int col = blockIdx.x * kPackThreads + threadIdx.x;
  uint32_t bad = 0u;
  if (col < KM)
    for (int row = blockIdx.y; row < N; row += gridDim.y) pack_word(src, planes, row, col, KM, bad);
  if (__any_sync(0xFFFFFFFFu, bad != 0u) && (threadIdx.x & 31) == 0) set_flag(flag);
}

// Several tensors in one persistent launch: unit u of item i covers rows [16r, 16r + 16) and words
// [128c, 128c + 128) of each row, u - unit0[i] = r * (column blocks) + c.
__global__ void __launch_bounds__(kPackThreads) k_pack_trits_batch(const __grid_constant__ PackBatch p,
                                                                   int32_t* __restrict__ flag) {
  uint32_t bad = 0u;
  for (int u = blockIdx.x; u < p.units; u += gridDim.x) {
    int lo = 0, hi = p.count - 1;                   // last item with unit0 <= u
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (p.unit0[mid] <= u) lo = mid; else hi = mid - 1;
    }
    const int KM = p.KM[lo], N = p.N[lo];
    const int gx = (KM + kPackThreads - 1) / kPackThreads;
    const int lu = u - p.unit0[lo];
    const int rg = lu / gx, col = (lu - rg * gx) * kPackThreads + threadIdx.x;
    if (col < KM) {
      const int r1 = min(N, (rg + 1) * kPackUnitRows);
#pragma unroll 4
      for (int row = rg * kPackUnitRows; row < r1; ++row) pack_word(p.src[lo], p.planes[lo], row, col, KM, bad);
    }
  }
  if (__any_sync(0xFFFFFFFFu, bad != 0u) && (threadIdx.x & 31) == 0) set_flag(flag);
}

constexpr int kB3Threads = 256;
constexpr int kB3StageBytes = 16 * 1024;          // transport bytes per block (whole rows)
constexpr int kB3Slot = 48;                       // shared-memory bytes per 32-byte run

// The five words of a copy window that reaches the end of the transport buffer: the words wholly
// inside it as words, the last partial one byte by byte, zeros past the end (n = bytes left).
struct Words5 {
  uint32_t w0, w1, w2, w3, w4;
};
__device__ __noinline__ uint32_t load_tail_word(const uint8_t* p, int n) {
  uint32_t x = 0u;
  if (n >= 4) return __ldg(reinterpret_cast<const uint32_t*>(p));
  for (int t = 0; t < 4; ++t)
    if (t < n) x |= (uint32_t)__ldg(p + t) << (8 * t);
  return x;
}
__device__ __noinline__ Words5 load_tail_words(const uint8_t* p, int n) {
  Words5 r;
  r.w0 = load_tail_word(p, n);
  r.w1 = load_tail_word(p + 4, n - 4);
  r.w2 = load_tail_word(p + 8, n - 8);
  r.w3 = load_tail_word(p + 12, n - 12);
  r.w4 = load_tail_word(p + 16, n - 16);
  return r;
}

// A tensor's constants for the unpack walks, computed once per tensor and thread: run j of a
// block (32 transport bytes = 160 trits) is run i of block row rr, and each walk advances j by a
// fixed step, so (rr, i) advance by (step / rpr, step % rpr) without a division per block.
struct B3Shape {
  const uint8_t* src;
  uint32_t* planes;
  int N, KW, rb, rows, rpr;
  int64_t total;                                   // transport bytes of the tensor
  int c_rr, c_i, c_dq, c_dr;                       // copy walk: j = tid / 2, step blockDim / 2
  int d_rr, d_i, d_dq, d_dr;                       // decode walk: j = tid, step blockDim
};
__device__ __forceinline__ B3Shape b3_shape(const uint8_t* src, uint32_t* planes, int N, int K, int rows) {
  B3Shape s;
  s.src = src;
  s.planes = planes;
  s.N = N;
  s.KW = K / 32;
  s.rb = (K + 4) / 5;
  s.rows = rows;
  s.rpr = (s.KW + 4) / 5;
  s.total = (int64_t)N * s.rb;
  const int jc = threadIdx.x >> 1, sc = blockDim.x >> 1, jd = threadIdx.x, sd = blockDim.x;
  s.c_rr = jc / s.rpr;
  s.c_i = jc - s.c_rr * s.rpr;
  s.c_dq = sc / s.rpr;
  s.c_dr = sc - s.c_dq * s.rpr;
  s.d_rr = jd / s.rpr;
  s.d_i = jd - s.d_rr * s.rpr;
  s.d_dq = sd / s.rpr;
  s.d_dr = sd - s.d_dq * s.rpr;
  return s;
}

// One block of whole transport rows, three phases (the CTA has built the byte table first):
//   1. copy: run j (32 bytes = 160 trits = 5 output words) of the block goes to its own 48-byte
//      slot, so that phase 2's two 16-byte reads per lane hit distinct banks;
//   2. decode: a table turns each byte into its five mask and five sign bits in natural order;
//      the bits are gathered per 32-trit word, moved to the layout's bit order and written to a
//      shared-memory copy of the block's output rows;
//   3. write-out: the block's rows are contiguous in the planes, copied with 16-byte stores.
__device__ __forceinline__ void unpack_base3_block(const B3Shape& S, int32_t block, int32_t* __restrict__ flag,
                                                   uint4* b3_smem) {
  const uint8_t* __restrict__ src = S.src;
  const int N = S.N, KW = S.KW, rb = S.rb, rows_per_cta = S.rows, rpr = S.rpr;
  const int r0 = block * rows_per_cta;
  const int nrow = min(N - r0, rows_per_cta);
  const int nruns = nrow * rpr;
  const uint32_t* lut = reinterpret_cast<const uint32_t*>(b3_smem);
  uint8_t* runs = reinterpret_cast<uint8_t*>(b3_smem) + 1024;
  uint32_t* outw = reinterpret_cast<uint32_t*>(runs + (size_t)rows_per_cta * rpr * kB3Slot);
  const int64_t total = S.total;
  const int step = blockDim.x / 2;                 // copy phase: two half-runs per run
  const int dq = S.c_dq, dr = S.c_dr;
  // 1. copy: half-runs of 16 bytes, each from five aligned words of the transport. Offsets are
  // 32-bit, relative to the aligned word at or below the block's first byte; only a window that
  // reaches the buffer's end takes the byte-wise path.
  {
    const int64_t b0 = (int64_t)r0 * rb;             // the block's first transport byte
    const uint8_t* base = src + (b0 & ~(int64_t)3);
    const int lead = (int)(b0 & 3);
    const int64_t rem64 = total - (b0 & ~(int64_t)3);
    const int remain = rem64 > 0x7FFFFFFF ? 0x7FFFFFFF : (int)rem64;   // bytes from base to the end
    int j = threadIdx.x >> 1, rr = S.c_rr, i = S.c_i;
    const int h = threadIdx.x & 1;
    for (; j < nruns; j += step) {
      const int off = lead + rr * rb + 32 * i + 16 * h; // byte offset of the half-run from base
      const int oa = off & ~3;
      const uint32_t sh = 8u * (uint32_t)(off & 3);
      uint32_t w[5];
      if (oa + 20 <= remain) {
#pragma unroll
        for (int k = 0; k < 5; ++k) w[k] = __ldg(reinterpret_cast<const uint32_t*>(base + oa + 4 * k));
      } else {
        const Words5 t = load_tail_words(base + oa, remain - oa);
        w[0] = t.w0; w[1] = t.w1; w[2] = t.w2; w[3] = t.w3; w[4] = t.w4;
      }
      // bytes past the row's end belong to the next row: they only reach trits past K, never written
      uint4 v;
      v.x = __funnelshift_r(w[0], w[1], sh);
      v.y = __funnelshift_r(w[1], w[2], sh);
      v.z = __funnelshift_r(w[2], w[3], sh);
      v.w = __funnelshift_r(w[3], w[4], sh);
      *reinterpret_cast<uint4*>(runs + (size_t)j * kB3Slot + 16 * h) = v;
      rr += dq;
      i += dr;
      if (i >= rpr) { i -= rpr; ++rr; }
    }
  }
  __syncthreads();
  // 2. decode
  bool bad = false;
  {
    const int step2 = blockDim.x;
    const int eq = S.d_dq, er = S.d_dr;
    int j = threadIdx.x, rr = S.d_rr, i = S.d_i;
    for (; j < nruns; j += step2) {
      const uint4 lo = *reinterpret_cast<const uint4*>(runs + (size_t)j * kB3Slot);
      const uint4 hi = *reinterpret_cast<const uint4*>(runs + (size_t)j * kB3Slot + 16);
      const uint32_t by[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
      // groups of 16 trits: W[k] holds the group's 16 mask bits low and 16 sign bits high, so one
      // shifted table entry (mask5 | sign5 << 16) lands both fields of a byte with one add; the
      // bytes whose five trits cross a group boundary are added in two parts
      // A row's last run also holds bytes past the row: the next row's own bytes, or zeros past
      // the buffer, so an invalid byte among them is an invalid byte of the transport too.
      uint32_t W[10] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
      uint32_t eor = 0u;
#pragma unroll
      for (int b = 0; b < 32; ++b) {
        const uint32_t e = lut[__byte_perm(by[b >> 2], 0u, 0x4440u | (uint32_t)(b & 3))];
        eor |= e;
        const int k = (5 * b) >> 4, o = (5 * b) & 15;
        if (o <= 11) {
          W[k] += e << o;
        } else {
          // low parts stay in group k (mask bits o..15, sign bits 16+o..31), high parts open k+1
          W[k] += (e << o) & (0x0000FFFFu | (0xFFFFFFFFu << (16 + o)));
          W[k + 1] += ((e & 31u) >> (16 - o)) | ((((e >> 16) & 31u) >> (16 - o)) << 16);
        }
      }
      uint32_t m[5], s[5];
#pragma unroll
      for (int u = 0; u < 5; ++u) {
        m[u] = __byte_perm(W[2 * u], W[2 * u + 1], 0x5410);   // low halves: mask bits of trits 32u ..
        s[u] = __byte_perm(W[2 * u], W[2 * u + 1], 0x7632);   // high halves: their sign bits
      }
      bad |= (eor >> 31) != 0u;
      uint32_t* rowo = outw + (size_t)rr * 2 * KW;
#pragma unroll
      for (int u = 0; u < 5; ++u) {
        const int w = 5 * i + u;
        if (w < KW) {
          rowo[w] = to_mask_order(m[u]);
          const uint32_t sp = to_mask_order(s[u]);
          rowo[KW + w] = (sp << 1) | (sp >> 31);     // the sign bit sits one above its mask bit
        }
      }
      rr += eq;
      i += er;
      if (i >= rpr) { i -= rpr; ++rr; }
    }
  }
  if (__any_sync(0xFFFFFFFFu, bad) && (threadIdx.x & 31) == 0) set_flag(flag);
  __syncthreads();
  // 3. write-out: nrow rows x 2*KW words, contiguous in the planes (KW % 4 == 0)
  const int nvec = nrow * 2 * KW / 4;
  uint4* dst = reinterpret_cast<uint4*>(S.planes + (size_t)r0 * 2 * KW);
  const uint4* from = reinterpret_cast<const uint4*>(outw);
  for (int v = threadIdx.x; v < nvec; v += blockDim.x) dst[v] = from[v];
}

// Persistent: each CTA builds the byte table once, then walks blocks of rows grid-strided.
__global__ void __launch_bounds__(kB3Threads, 5) k_unpack_base3(const uint8_t* __restrict__ src, int32_t N, int32_t KW,
                                                              int32_t rb, int32_t rows_per_cta, int32_t nblocks,
                                                              uint32_t* __restrict__ planes, int32_t* __restrict__ flag) {
  extern __shared__ uint4 b3_smem[];
  build_base3_lut(reinterpret_cast<uint32_t*>(b3_smem));
  __syncthreads();
  const B3Shape S = b3_shape(src, planes, N, KW * 32, rows_per_cta);
  for (int block = blockIdx.x; block < nblocks; block += gridDim.x) unpack_base3_block(S, block, flag, b3_smem);
}

// Persistent over the blocks of all items in order; a CTA's item index only moves forward.
__global__ void __launch_bounds__(kB3Threads, 5) k_unpack_base3_batch(const __grid_constant__ Base3Batch p,
                                                                    int32_t nblocks, int32_t* __restrict__ flag) {
  extern __shared__ uint4 b3_smem[];
  build_base3_lut(reinterpret_cast<uint32_t*>(b3_smem));
  __syncthreads();
  int lo = 0, cur = -1;
  B3Shape S;
  for (int block = blockIdx.x; block < nblocks; block += gridDim.x) {
    while (lo + 1 < p.count && p.block0[lo + 1] <= block) ++lo;   // last item with block0 <= block
    if (lo != cur) {
      S = b3_shape(p.src[lo], p.planes[lo], p.N[lo], p.K[lo], p.rows[lo]);
      cur = lo;
    }
    unpack_base3_block(S, block - p.block0[lo], flag, b3_smem);
  }
}

// One thread per transport byte.
__global__ void k_encode_base3(const int8_t* __restrict__ src, int64_t n_bytes, int32_t K, int32_t row_bytes,
                               uint8_t* __restrict__ out, int32_t* __restrict__ flag) {
  bool bad = false;
  for (int64_t o = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; o < n_bytes;
       o += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = o / row_bytes;
    const int j = (int)(o % row_bytes);
    const int8_t* rp = src + row * (int64_t)K;
    int b = 0, p3 = 1;
#pragma unroll
    for (int i = 0; i < 5; ++i) {
      const int k = 5 * j + i;
      int d = 1;
      if (k < K) {
        const int t = rp[k];
        bad |= (t < -1 || t > 1);
        d = t + 1;
      }
      b += d * p3;
      p3 *= 3;
    }
    out[o] = (uint8_t)(b > 242 ? 121 : b);
  }
  if (__any_sync(0xFFFFFFFFu, bad) && (threadIdx.x & 31) == 0) set_flag(flag);
}

// One warp per row: popcounts of the two planes.
__global__ void k_occupancy(const uint32_t* __restrict__ planes, int32_t N, int32_t K, int64_t* __restrict__ counts) {
  const int KM = K / 32;
  const int warps = blockDim.x / 32;
  for (int row = blockIdx.x * warps + threadIdx.x / 32; row < N; row += gridDim.x * warps) {
    const uint32_t* rp = planes + (int64_t)row * 2 * KM;
    int nz = 0, neg = 0;
    for (int c = threadIdx.x & 31; c < KM; c += 32) {
      const uint32_t m = rp[c], s = rp[KM + c];
      nz += __popc(m);
      neg += __popc(s & __funnelshift_l(m, m, 1));
    }
    for (int o = 16; o > 0; o >>= 1) {
      nz += __shfl_xor_sync(0xFFFFFFFFu, nz, o);
      neg += __shfl_xor_sync(0xFFFFFFFFu, neg, o);
    }
    if ((threadIdx.x & 31) == 0) {
      counts[3 * (int64_t)row] = K - nz;
      counts[3 * (int64_t)row + 1] = nz - neg;
      counts[3 * (int64_t)row + 2] = neg;
    }
  }
}

int grid_for(int64_t work, int threads) {
  int64_t g = (work + threads - 1) / threads;
  const int64_t cap = (int64_t)device_sm_count() * 32;
  return (int)(g < 1 ? 1 : (g > cap ? cap : g));
}

}  // namespace

cudaError_t launch_pack_trits(const int8_t* src, int32_t N, int32_t K, uint32_t* planes, int32_t* flag,
                              cudaStream_t st) {
  const int KM = K / 32;
  const int gx = (KM + kPackThreads - 1) / kPackThreads;
  int gy = (device_sm_count() * 16 + gx - 1) / gx;       // ~16 CTAs per SM over all columns
  if (gy > N) gy = N;
  if (gy > 65535) gy = 65535;
  k_pack_trits<<<dim3(gx, gy), kPackThreads, 0, st>>>(src, N, KM, planes, flag);
  return cudaGetLastError();
}

void base3_plan(int32_t K, int& rows, size_t& smem) {
  const int rb = (K + 4) / 5, KW = K / 32, rpr = (KW + 4) / 5;
  rows = kB3StageBytes / rb;
  if (rows < 1) rows = 1;
  smem = 1024 + (size_t)rows * rpr * kB3Slot + (size_t)rows * K / 4;
}

// Resident CTAs of a persistent unpack kernel (at least one), capped by the blocks there are.
int base3_grid(const void* fn, size_t smem, int nblocks) {
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kB3Threads, smem) != cudaSuccess || per_sm < 1)
    per_sm = 1;
  const long long g = (long long)per_sm * device_sm_count();
  return (int)(g < nblocks ? g : (nblocks < 1 ? 1 : nblocks));
}

cudaError_t launch_unpack_base3(const uint8_t* src, int32_t N, int32_t K, uint32_t* planes, int32_t* flag,
                                cudaStream_t st) {
  int rows = 1;
  size_t smem = 0;
  base3_plan(K, rows, smem);
  const int nblocks = (N + rows - 1) / rows;
  static std::atomic<unsigned long long> smem_raised{0};
  cudaError_t e = allow_max_dynamic_smem(k_unpack_base3, smem_raised);
  if (e != cudaSuccess) return e;
  const int grid = base3_grid(reinterpret_cast<const void*>(k_unpack_base3), smem, nblocks);
  k_unpack_base3<<<grid, kB3Threads, smem, st>>>(src, N, K / 32, (K + 4) / 5, rows, nblocks, planes, flag);
  return cudaGetLastError();
}

cudaError_t launch_pack_trits_batch(PackBatch& p, int32_t* flag, cudaStream_t st) {
  int64_t units = 0;
  for (int i = 0; i < p.count; ++i) {
    p.unit0[i] = (int32_t)units;
    units += (int64_t)((p.N[i] + kPackUnitRows - 1) / kPackUnitRows) * ((p.KM[i] + kPackThreads - 1) / kPackThreads);
  }
  if (units > 0x7FFFFFFF) return cudaErrorInvalidValue;
  p.units = (int32_t)units;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_pack_trits_batch, kPackThreads, 0) != cudaSuccess ||
      per_sm < 1)
    per_sm = 1;
  const int64_t g = (int64_t)per_sm * device_sm_count();
  k_pack_trits_batch<<<(unsigned)(g < units ? g : units), kPackThreads, 0, st>>>(p, flag);
  return cudaGetLastError();
}

cudaError_t launch_unpack_base3_batch(Base3Batch& p, int32_t* flag, cudaStream_t st) {
  size_t smem = 0;
  int64_t blocks = 0;
  for (int i = 0; i < p.count; ++i) {
    int rows = 1;
    size_t sm = 0;
    base3_plan(p.K[i], rows, sm);
    p.rows[i] = rows;
    p.block0[i] = (int32_t)blocks;
    blocks += (p.N[i] + rows - 1) / rows;
    if (sm > smem) smem = sm;
  }
  if (blocks > 0x7FFFFFFF) return cudaErrorInvalidValue;
  static std::atomic<unsigned long long> smem_raised{0};
  cudaError_t e = allow_max_dynamic_smem(k_unpack_base3_batch, smem_raised);
  if (e != cudaSuccess) return e;
  const int grid = base3_grid(reinterpret_cast<const void*>(k_unpack_base3_batch), smem, (int)blocks);
  k_unpack_base3_batch<<<grid, kB3Threads, smem, st>>>(p, (int32_t)blocks, flag);
  return cudaGetLastError();
}

cudaError_t launch_encode_base3(const int8_t* src, int32_t N, int32_t K, uint8_t* out, int32_t* flag,
                                cudaStream_t st) {
  const int64_t n_bytes = (int64_t)N * ((K + 4) / 5);
  k_encode_base3<<<grid_for(n_bytes, 256), 256, 0, st>>>(src, n_bytes, K, (K + 4) / 5, out, flag);
  return cudaGetLastError();
}

cudaError_t launch_occupancy(const uint32_t* planes, int32_t N, int32_t K, int64_t* counts, cudaStream_t st) {
  k_occupancy<<<grid_for((int64_t)N * 32, 256), 256, 0, st>>>(planes, N, K, counts);
  return cudaGetLastError();
}

}  // namespace tern
