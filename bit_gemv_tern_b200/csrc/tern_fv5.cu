// Five-valued weights in 256-weight blocks (FV5-style): packing, the GEMV / small-M product of one
// matrix, and a list of matrices at M = 1 in one persistent launch (k_fv5_batch, below).
//
// The pages' shipped linear format (PyTorchKR review "Fermion Research, 3진 계열 포맷으로 직접
// 학습한 Neutrino-1 모델군 3종 공개", section "FV5와 FV5B: llama.cpp 포크가 공개한 블록 구조")
// stores 256 weights per block as three bitplanes and two fp32 scales, s_lo and s_hi: sign and
// zero plus two magnitude steps. This library's reading (include/tern.h): a code c in -2..2 per
// weight, w = sign(c) * (|c| == 2 ? s_hi : s_lo) of its row and block, planes mask / sign / high
// magnitude in the ternary layout's bit order, words transposed inside each 512-trit group so that
// lane t of a quad reads logical words t, 4 + t, 8 + t, 12 + t as one 128-bit load.
//
//   Y[m][n] = sum_b ( s_lo[n][b] * sum_{k in b, |c| = 1} sign * X[m][k]
//                   + s_hi[n][b] * sum_{k in b, |c| = 2} sign * X[m][k] )
//
// Kernel: as the ternary small-M kernel (tern_gemv.cu): 16-row warp tiles, the K slice of the
// activations staged once as int8 operand columns (q, or four exact limbs per token), CTAs splitting
// K form a cluster. Each word is split into its low- and high-magnitude ternary parts (mask & ~g,
// sign & ~g; mask & g, sign & g), each decoded to 64 * t bytes and multiplied exactly by the
// tensor cores into its own int32 accumulators. Step e of a 512-trit chunk covers logical words
// 4e .. 4e + 3 of all four quad lanes, i.e. trits 128e .. 128e + 127, so steps 0-1 and 2-3 are the
// chunk's two blocks: after each block the exact sums are scaled by the block's s_lo and s_hi and
// added into fp64 accumulators, which the epilogue rounds once to fp32 (int8 mode after * s_x).
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
__device__ __forceinline__ int fv5_cols(int mode, int M) { return mode == 0 ? 4 * M : M; }
__device__ __forceinline__ int col_words(int kr) { return kr / 4 + 16; }
__device__ __forceinline__ int half_ofs(int v) { return 4 * (v ^ ((v >> 3) & 3)); }
__device__ __forceinline__ uint32_t smem_u32(const void* p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }

// ---- pack -------------------------------------------------------------------------------------------
// One thread per (row, logical 32-trit word): 32 codes in, the three plane words out at the word's
// stored position.
__global__ void k_fv5_pack(const int8_t* __restrict__ codes, int64_t words, int32_t KW, uint32_t* __restrict__ planes,
                           int32_t* flag) {
  bool bad = false;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < words; i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = i / KW;
    const int w = (int)(i - row * KW);
    const int8_t* c = codes + i * 32;
    const uint4 v0 = ld_stream(c), v1 = ld_stream(c + 16);
    const uint32_t b[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
    uint32_t m = 0u, s = 0u, g = 0u;                        // natural order: bit j = trit j of the word
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const int x = (int8_t)(b[j >> 2] >> (8 * (j & 3)));
      bad |= x < -2 || x > 2;
      m |= (uint32_t)(x != 0) << j;
      s |= (uint32_t)(x < 0) << j;
      g |= (uint32_t)(x == 2 || x == -2) << j;
    }
    // natural order -> the layout's order p(j) (swap bits 0 and 4 of j)
    auto order = [](uint32_t x) {
      const uint32_t t = lop3<0x28u>(x >> 15, x, 0x0000AAAAu);
      return lop3<0x96u>(x, t, t << 15);
    };
    const int grp = w >> 4, li = w & 15;
    const int sw = 16 * grp + 4 * (li & 3) + (li >> 2);     // stored position of logical word w
    uint32_t* rp = planes + row * 3 * (int64_t)KW;
    const uint32_t sp = order(s);
    rp[sw] = order(m);
    rp[KW + sw] = (sp << 1) | (sp >> 31);
    rp[2 * KW + sw] = order(g);
  }
  if (__any_sync(0xFFFFFFFFu, bad) && (threadIdx.x & 31) == 0) atomicExch(flag, 1);
}

// ---- product ----------------------------------------------------------------------------------------
template <int MODE, int NG>
__global__ void __launch_bounds__(kThreads) k_fv5_gemm(const Fv5Params p) {
  extern __shared__ __align__(16) uint32_t smem[];
  __shared__ int expo[16];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int ks = blockIdx.x;
  const int k0 = ks * p.kr;
  const int row0 = blockIdx.y * kRows + warp * 16;
  const int KM = p.K >> 5;
  const int nw = p.kr >> 5;                                // multiple of 16
  const int nchunks = nw >> 4;
  const bool warp_live = row0 < p.N;
  const int ra = min(row0 + g, p.N - 1), rb = min(row0 + g + 8, p.N - 1);
  const uint32_t* pa = p.planes + (size_t)ra * (3 * KM) + (k0 >> 5);
  const uint32_t* pb = p.planes + (size_t)rb * (3 * KM) + (k0 >> 5);
  const int nblk = p.K >> 8;
  const float2* sca = reinterpret_cast<const float2*>(p.scales) + (size_t)ra * nblk + (k0 >> 8);
  const float2* scb = reinterpret_cast<const float2*>(p.scales) + (size_t)rb * nblk + (k0 >> 8);
  const int ncols = fv5_cols(MODE, p.M);
  const int RS = col_words(p.kr);

  // chunk c: stored words [16c + 4t, 16c + 4t + 4) of the three planes of rows ra, rb
  auto load_chunk = [&](int c, uint4 (&w)[6]) {
    const int off = 16 * c + 4 * t;
    if (warp_live && c < nchunks) {
      w[0] = ld_stream(pa + off);
      w[1] = ld_stream(pb + off);
      w[2] = ld_stream(pa + KM + off);
      w[3] = ld_stream(pb + KM + off);
      w[4] = ld_stream(pa + 2 * KM + off);
      w[5] = ld_stream(pb + 2 * KM + off);
    } else {
#pragma unroll
      for (int i = 0; i < 6; ++i) w[i] = make_uint4(0u, 0u, 0u, 0u);
    }
  };
  uint4 cur[6], nxt[6];
  // the first two chunks' weights: int8 mode before the dependency wait, bf16 mode after its
  // two-pass staging of the activations (issued first, they would hold up its reads)
  if (MODE == 1) {
    load_chunk(0, cur);
    load_chunk(1, nxt);
  }
  pdl_wait();

  // ---- stage the activation slice as int8 operand columns (as tern_gemv.cu) ----------------------
  const int per_row = p.kr >> 4;
  if (MODE == 1) {
    const int8_t* xs = static_cast<const int8_t*>(p.x);
    for (int i = threadIdx.x; i < p.M * per_row; i += kThreads) {
      const int m = i / per_row, v = i - m * per_row;
      *reinterpret_cast<uint4*>(smem + m * RS + half_ofs(v)) = permute_i8_half(ld_nc(xs + (size_t)m * p.K + k0 + 16 * v));
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
        *reinterpret_cast<uint4*>(smem + (4 * m + c) * RS + half_ofs(v)) =
            permute_i8_half(make_uint4(l[c][0], l[c][1], l[c][2], l[c][3]));
    }
    load_chunk(0, cur);
    load_chunk(1, nxt);
  }
  __syncthreads();

  double Y[NG][4];
#pragma unroll
  for (int n = 0; n < NG; ++n) Y[n][0] = Y[n][1] = Y[n][2] = Y[n][3] = 0.0;

  for (int c = 0; c < nchunks; ++c) {
#pragma unroll
    for (int half = 0; half < 2; ++half) {                 // the chunk's two 256-weight blocks
      int accL[NG][4], accH[NG][4];
#pragma unroll
      for (int n = 0; n < NG; ++n)
#pragma unroll
        for (int i = 0; i < 4; ++i) accL[n][i] = accH[n][i] = 0;
#pragma unroll
      for (int ee = 0; ee < 2; ++ee) {
        const int e = 2 * half + ee;
        const int w = 16 * c + 4 * e + t;                  // logical word of this lane
        const uint32_t ga = u4get(cur[4], e), gb = u4get(cur[5], e);
        uint32_t la0, lb0, la1, lb1, ha0, hb0, ha1, hb1;
        merge_planes(u4get(cur[0], e) & ~ga, u4get(cur[2], e) & ~(ga << 1 | ga >> 31), la0, lb0);
        merge_planes(u4get(cur[1], e) & ~gb, u4get(cur[3], e) & ~(gb << 1 | gb >> 31), la1, lb1);
        merge_planes(u4get(cur[0], e) & ga, u4get(cur[2], e) & (ga << 1 | ga >> 31), ha0, hb0);
        merge_planes(u4get(cur[1], e) & gb, u4get(cur[3], e) & (gb << 1 | gb >> 31), ha1, hb1);
        const uint32_t AL[8][2] = {
            {dec_i8<0>(la0, lb0), dec_i8<0>(la1, lb1)}, {dec_i8<1>(la0, lb0), dec_i8<1>(la1, lb1)},
            {dec_i8<2>(la0, lb0), dec_i8<2>(la1, lb1)}, {dec_i8<3>(la0, lb0), dec_i8<3>(la1, lb1)},
            {dec_i8<4>(la0, lb0), dec_i8<4>(la1, lb1)}, {dec_i8<5>(la0, lb0), dec_i8<5>(la1, lb1)},
            {dec_i8<6>(la0, lb0), dec_i8<6>(la1, lb1)}, {dec_i8<7>(la0, lb0), dec_i8<7>(la1, lb1)}};
        const uint32_t AH[8][2] = {
            {dec_i8<0>(ha0, hb0), dec_i8<0>(ha1, hb1)}, {dec_i8<1>(ha0, hb0), dec_i8<1>(ha1, hb1)},
            {dec_i8<2>(ha0, hb0), dec_i8<2>(ha1, hb1)}, {dec_i8<3>(ha0, hb0), dec_i8<3>(ha1, hb1)},
            {dec_i8<4>(ha0, hb0), dec_i8<4>(ha1, hb1)}, {dec_i8<5>(ha0, hb0), dec_i8<5>(ha1, hb1)},
            {dec_i8<6>(ha0, hb0), dec_i8<6>(ha1, hb1)}, {dec_i8<7>(ha0, hb0), dec_i8<7>(ha1, hb1)}};
#pragma unroll
        for (int n = 0; n < NG; ++n) {
          const int col = 8 * n + g;
          uint32_t xb[8];
          if (col < ncols) {
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              const uint4 v = *reinterpret_cast<const uint4*>(smem + col * RS + half_ofs(2 * w + q));
              xb[4 * q] = v.x; xb[4 * q + 1] = v.y; xb[4 * q + 2] = v.z; xb[4 * q + 3] = v.w;
            }
          } else {
#pragma unroll
            for (int q = 0; q < 8; ++q) xb[q] = 0u;
          }
#pragma unroll
          for (int r = 0; r < 8; r += 2) {
            mma_s8(accL[n], AL[r][0], AL[r][1], AL[r + 1][0], AL[r + 1][1], xb[r], xb[r + 1]);
            mma_s8(accH[n], AH[r][0], AH[r][1], AH[r + 1][0], AH[r + 1][1], xb[r], xb[r + 1]);
          }
        }
      }
      // the block's exact sums (acc = 64 * sum), scaled by its s_lo and s_hi, into fp64
      const int blk = 2 * c + half;
      const float2 sa = warp_live ? __ldg(sca + blk) : make_float2(0.f, 0.f);
      const float2 sb = warp_live ? __ldg(scb + blk) : make_float2(0.f, 0.f);
#pragma unroll
      for (int n = 0; n < NG; ++n)
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 s2 = (i >> 1) ? sb : sa;
          Y[n][i] += (double)s2.x * (double)(accL[n][i] >> 6) + (double)s2.y * (double)(accH[n][i] >> 6);
        }
    }
#pragma unroll
    for (int i = 0; i < 6; ++i) cur[i] = nxt[i];
    load_chunk(c + 2, nxt);
  }
  pdl_launch_dependents();

  // ---- epilogue: partial tile [kRows][8 * NG] doubles, then (split K) a cluster-wide sum ----------
  constexpr int kCols = 8 * NG;
  double* part = reinterpret_cast<double*>(smem + ncols * RS + (ncols * RS & 1));
#pragma unroll
  for (int n = 0; n < NG; ++n)
#pragma unroll
    for (int i = 0; i < 4; ++i)
      part[(warp * 16 + g + 8 * (i >> 1)) * kCols + 8 * n + 2 * t + (i & 1)] = Y[n][i];
  cg::cluster_group cluster = cg::this_cluster();
  if (p.ksplit > 1) cluster.sync(); else __syncthreads();
  const int rows_per_rank = kRows / p.ksplit;
  for (int i = threadIdx.x; i < rows_per_rank * p.M; i += kThreads) {
    const int lrow = ks * rows_per_rank + i / p.M, m = i % p.M;
    const int row = blockIdx.y * kRows + lrow;
    if (row >= p.N) continue;
    double tot = 0.0;
    for (int r = 0; r < p.ksplit; ++r) {
      const double* rp = (p.ksplit > 1 ? cluster.map_shared_rank(part, r) : part) + lrow * kCols;
      if (MODE == 1) {
        tot += rp[m];
      } else {
        const int E = (p.ksplit > 1 ? cluster.map_shared_rank(expo, r) : expo)[m];
        const double* l = rp + 4 * m;
        tot += ldexp(((l[0] * 256.0 + l[1]) * 256.0 + l[2]) * 256.0 + l[3], E - kLimbFrac);
      }
    }
    p.y[(size_t)m * p.N + row] = MODE == 1 ? (float)((double)p.sx[m] * tot) : (float)tot;
  }
  if (p.ksplit > 1) cluster.sync();
}

// ---- a list of linears at M = 1 in one persistent launch ---------------------------------------------
// Work units are 16-row tiles of one item over the whole of K; the host cuts the list into
// contiguous ranges of tiles with equal numbers of 512-trit chunks, one per CTA, two CTAs per SM
// (a range also closes where its items' staged activations would outgrow the shared-memory budget).
// A CTA stages the activations of all of its range's items at once (all K) as the batched stream's
// operand words (tern_batch.cu: eight words per 32-trit word, in natural word order here since the
// planes' word transposition already gives each quad lane its word) together with each 256-weight
// block's column sums. Its chunks are then cut into eight equal contiguous parts, one per warp, so a
// tile may be split between two warps (or, for a tile longer than a part, several). The blocks of a
// tile must still be added in order, so the fp64 partial sums of a tile's first part are handed to
// the owner of its next part: a warp takes the head of its last tile first (publishing its partial
// sums in shared memory at once), then its whole tiles, and the tail of its first tile last (taking
// the partial sums published by the previous part's owner, long since ready). Each wait is bounded.
// A word's low- and high-magnitude parts take the offset decode of the batched stream (one AND per
// operand register: field i in place reads 4^i (t + 2)) in turn, each into one set of four field
// accumulators; at a block's end the exact sums (the offset removed with the block's column sums)
// are scaled by s_lo and s_hi into fp64, as in k_fv5_gemm, and the owner of a tile's last part
// writes its rows' outputs.
constexpr int kWarps = kThreads / 32;
constexpr long long kHandSpin = 4000000000LL;               // clock64 cycles (~2 s) before a wait gives up
__device__ int g_fv5_latch = 0;

template <int MODE>
__global__ void __launch_bounds__(kThreads, 2) k_fv5_batch(const __grid_constant__ Fv5BatchParams p) {
  extern __shared__ __align__(16) uint32_t smem[];         // the range's items' activations, back to back
  __shared__ double hand[kWarps][4][32];                    // partial sums handed to warp w
  __shared__ int hflag[kWarps];
  __shared__ float fredw[kFv5MaxItemsPerCTA][kWarps];       // per item, per warp absmax (bf16 mode)
  __shared__ int offs[kFv5MaxItemsPerCTA], expo[kFv5MaxItemsPerCTA];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const int u0 = p.cta_unit[blockIdx.x], u1 = p.cta_unit[blockIdx.x + 1];
  if (u0 >= u1) return;
  constexpr int NC = MODE == 0 ? 4 : 1;
  const int i0 = p.cta_item[blockIdx.x];
  int iend = i0 + 1;                                        // items [i0, iend) meet the range
  while (iend < p.count && p.unit0[iend] < u1) ++iend;
  auto tiles_of = [&](int j) { return min(u1, p.unit0[j + 1]) - max(u0, p.unit0[j]); };
  // this warp's chunks [a, b) of the range's Wc
  int Wc = 0;
  for (int j = i0; j < iend; ++j) Wc += tiles_of(j) * (p.items[j].K >> 9);
  const int a = (int)((long long)Wc * warp / kWarps), b = (int)((long long)Wc * (warp + 1) / kWarps);
  // chunk x of the range -> item, tile, chunk of the tile
  auto locate = [&](int x, int& item, int& u, int& c) {
    int j = i0;
    while (true) {
      const int nch = p.items[j].K >> 9, cj = tiles_of(j) * nch;
      if (x < cj || j + 1 >= iend) {
        item = j;
        u = max(u0, p.unit0[j]) + x / nch;
        c = x % nch;
        return;
      }
      x -= cj;
      ++j;
    }
  };
  int iA = 0, uA = 0, cA = 0, iB = 0, uB = 0, cBe = 0, npieces = 0;
  if (a < b) {
    locate(a, iA, uA, cA);
    locate(b - 1, iB, uB, cBe);
    ++cBe;
    npieces = uA == uB ? 1 : uB - uA + 1;
  }
  const bool headB = cBe < (p.items[iB].K >> 9);
  // piece k in the order taken: the head of the last tile (if split), the whole tiles, the first tile
  auto piece = [&](int k, int& item, int& u, int& ca, int& cb) {
    if (uA == uB) { item = iA; u = uA; ca = cA; cb = cBe; return; }
    if (k == uB - uA) { item = iA; u = uA; ca = cA; cb = p.items[iA].K >> 9; return; }
    if (headB && k == 0) { item = iB; u = uB; ca = 0; cb = cBe; return; }
    u = headB ? uA + k : uA + 1 + k;
    int j = iA;
    while (p.unit0[j + 1] <= u) ++j;
    item = j;
    ca = 0;
    cb = p.items[j].K >> 9;
  };
  // the fetch side runs two chunks ahead of the products, across pieces
  int fk = 0, f_u = 0, f_c = 0, f_cb = 0, f_KM = 0;
  const uint32_t *pa = nullptr, *pb = nullptr;
  auto fetch_setup = [&](int k) {
    int item;
    piece(k, item, f_u, f_c, f_cb);
    const Fv5BatchItem& I = p.items[item];
    f_KM = I.K >> 5;
    const int row0 = (f_u - p.unit0[item]) * 16;
    const int ra = min(row0 + g, I.N - 1), rb = min(row0 + g + 8, I.N - 1);
    pa = I.planes + (size_t)ra * (3 * f_KM);
    pb = I.planes + (size_t)rb * (3 * f_KM);
  };
  auto fetch_next = [&](uint4 (&w)[6]) {
    if (fk < npieces) {
      const int off = 16 * f_c + 4 * t;
      w[0] = ld_stream(pa + off);
      w[1] = ld_stream(pb + off);
      w[2] = ld_stream(pa + f_KM + off);
      w[3] = ld_stream(pb + f_KM + off);
      w[4] = ld_stream(pa + 2 * f_KM + off);
      w[5] = ld_stream(pb + 2 * f_KM + off);
      if (++f_c == f_cb && ++fk < npieces) fetch_setup(fk);
    } else {
#pragma unroll
      for (int i = 0; i < 6; ++i) w[i] = make_uint4(0u, 0u, 0u, 0u);
    }
  };
  uint4 cur[6], nxt[6];
  int par = 0;                                              // the buffer of the next chunk to take
  if (npieces > 0) fetch_setup(0);
  pdl_wait();

  // ---- stage the range's activations: operand words and per-block column sums --------------------
  if (threadIdx.x < kWarps) hflag[threadIdx.x] = 0;
  {
    int off = 0;
    for (int j = i0; j < iend; ++j) {
      const Fv5BatchItem& I = p.items[j];
      const int K = I.K, nblk = K >> 8, jj = j - i0;
      int* bsum = reinterpret_cast<int*>(smem + off + NC * (K / 4 + 4));
      for (int i = threadIdx.x; i < NC * nblk; i += kThreads) bsum[i] = 0;
      if (threadIdx.x == 0) offs[jj] = off;
      if (MODE == 0) {
        const uint16_t* xs = static_cast<const uint16_t*>(I.x);
        float amax = 0.0f;
        for (int k = threadIdx.x * 8; k < K; k += kThreads * 8) {
          const uint4 v = ld_nc(xs + k);
          const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int e = 0; e < 4; ++e)
            amax = fmaxf(amax, fmaxf(fabsf(bf16_bits_to_float(w[e] & 0xFFFFu)), fabsf(bf16_bits_to_float(w[e] >> 16))));
        }
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xFFFFFFFFu, amax, o));
        if (lane == 0) fredw[jj][warp] = amax;
      }
      off += fv5_stage_words(NC, K);
    }
  }
  __syncthreads();                                          // absmax partials, zeroed sums, offsets
  for (int j = i0; j < iend; ++j) {
    const Fv5BatchItem& I = p.items[j];
    const int K = I.K, nblk = K >> 8, jj = j - i0, RS = K / 4 + 4;
    uint32_t* xb = smem + offs[jj];
    int* bsum = reinterpret_cast<int*>(xb + NC * RS);
    int E = 0;
    if (MODE == 0) {
      float mx = fredw[jj][0];
#pragma unroll
      for (int i = 1; i < kWarps; ++i) mx = fmaxf(mx, fredw[jj][i]);
      E = limb_exponent(mx);
      if (threadIdx.x == 0) expo[jj] = E;
    }
    for (int v = threadIdx.x; v < (K >> 4); v += kThreads) {  // 16-element halves
      const int w = v >> 1, h = v & 1, blk = v >> 4;
      if (MODE == 1) {
        const uint4 q = ld_nc(static_cast<const int8_t*>(I.x) + 16 * v);
        atomicAdd(&bsum[blk], __dp4a((int)q.x, 0x01010101, 0) + __dp4a((int)q.y, 0x01010101, 0) +
                                  __dp4a((int)q.z, 0x01010101, 0) + __dp4a((int)q.w, 0x01010101, 0));
        const uint4 o = permute_i8_half(q);
        uint32_t* slot = xb + w * 8;
        slot[0 + h] = o.x; slot[2 + h] = o.y; slot[4 + h] = o.z; slot[6 + h] = o.w;
      } else {
        const uint16_t* xe = static_cast<const uint16_t*>(I.x) + 16 * v;
        const uint4 lo = ld_nc(xe), hi = ld_nc(xe + 8);
        const uint32_t wv[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
        uint32_t l[4][4];
        limbs_of_bf16<4>(wv, E, l);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          atomicAdd(&bsum[c * nblk + blk], __dp4a((int)l[c][0], 0x01010101, 0) + __dp4a((int)l[c][1], 0x01010101, 0) +
                                               __dp4a((int)l[c][2], 0x01010101, 0) + __dp4a((int)l[c][3], 0x01010101, 0));
          const uint4 o = permute_i8_half(make_uint4(l[c][0], l[c][1], l[c][2], l[c][3]));
          uint32_t* slot = xb + c * RS + w * 8;
          slot[0 + h] = o.x; slot[2 + h] = o.y; slot[4 + h] = o.z; slot[6 + h] = o.w;
        }
      }
    }
  }
  // the first two chunks' weights, issued once the staging's activation reads are done (issued
  // before them, the whole grid's first chunks fill the memory queues and the staging waits
  // behind them: 3% slower over three 8B layers)
  fetch_next(cur);
  fetch_next(nxt);
  __syncthreads();

  // ---- this warp's pieces ---------------------------------------------------------------------------
  // accumulator register q holds row g + 8 (q >> 1), column 2t + (q & 1)
  const int colq0 = 2 * t, colq1 = 2 * t + 1;
  for (int k = 0; k < npieces; ++k) {
    int item, u, ca, cb;
    piece(k, item, u, ca, cb);
    const Fv5BatchItem& I = p.items[item];
    const int K = I.K, nblk = K >> 8, nch = K >> 9, RS = K / 4 + 4, jj = item - i0;
    const uint32_t* xb = smem + offs[jj];
    const int* bsum = reinterpret_cast<const int*>(xb + NC * RS);
    const int row0 = (u - p.unit0[item]) * 16;
    const int ra = min(row0 + g, I.N - 1), rb = min(row0 + g + 8, I.N - 1);
    const float2* sca = reinterpret_cast<const float2*>(I.scales) + (size_t)ra * nblk;
    const float2* scb = reinterpret_cast<const float2*>(I.scales) + (size_t)rb * nblk;
    double Y[4] = {0.0, 0.0, 0.0, 0.0};
    if (ca > 0) {                                           // the tile's earlier blocks: their sums
      bool ok = true;
      if (lane == 0) {
        const long long t0 = clock64();
        int v = 0, spins = 0;
        while (true) {
          asm volatile("ld.acquire.cta.shared.s32 %0, [%1];" : "=r"(v) : "r"(smem_u32(&hflag[warp])) : "memory");
          if (v) break;
          if (++spins > 32) __nanosleep(100);
          if (clock64() - t0 > kHandSpin) { ok = false; break; }
        }
        if (!ok) atomicExch(&g_fv5_latch, 5);
      }
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (ok) {
        int v;
        asm volatile("ld.acquire.cta.shared.s32 %0, [%1];" : "=r"(v) : "r"(smem_u32(&hflag[warp])) : "memory");
#pragma unroll
        for (int q = 0; q < 4; ++q) Y[q] = hand[warp][q][lane];
      }
    }
    // the chunk at step s of this warp sits in buffer s & 1 and is refilled, once used, with the
    // chunk two steps on: the two buffers alternate without register copies
    auto chunk = [&](const uint4 (&cw)[6], int c) {
  #pragma unroll
        for (int half = 0; half < 2; ++half) {                // the chunk's two 256-weight blocks
          const int blk = 2 * c + half;
          const int cs0 = colq0 < NC ? bsum[colq0 * nblk + blk] : 0;
          const int cs1 = colq1 < NC ? bsum[colq1 * nblk + blk] : 0;
          int R[2][4];                                        // offset sums: all nonzero weights, high magnitudes
  #pragma unroll
          for (int part = 0; part < 2; ++part) {              // all nonzero weights, then the high magnitudes:
            int acc[4][4] = {};                               // one set of field accumulators live at a time
  #pragma unroll
            for (int ee = 0; ee < 2; ++ee) {
              const int e = 2 * half + ee;
              const int w = 16 * c + 4 * e + t;               // logical word of this lane
              uint32_t ma = u4get(cw[0], e), mb = u4get(cw[1], e), sa = u4get(cw[2], e), sb = u4get(cw[3], e);
              if (part) {
                const uint32_t ga = u4get(cw[4], e), gb = u4get(cw[5], e);
                ma &= ga;
                mb &= gb;
                sa &= __funnelshift_l(ga, ga, 1);
                sb &= __funnelshift_l(gb, gb, 1);
              }
              uint32_t a0, b0, a1, b1;
              merge_planes_offset(ma, sa, a0, b0);
              merge_planes_offset(mb, sb, a1, b1);
              uint4 x01 = make_uint4(0u, 0u, 0u, 0u), x23 = x01;
              if (g < NC) {
                const uint32_t* xo = xb + g * RS + w * 8;
                x01 = *reinterpret_cast<const uint4*>(xo);
                x23 = *reinterpret_cast<const uint4*>(xo + 4);
              }
  #pragma unroll
              for (int i = 0; i < 4; ++i) {                   // field i in place -> 4^i * (t + 2)
                const uint32_t msk = 0x03030303u << (2 * i);
                const uint32_t x0 = i < 2 ? u4get(x01, 2 * i) : u4get(x23, 2 * i - 4);
                const uint32_t x1 = i < 2 ? u4get(x01, 2 * i + 1) : u4get(x23, 2 * i - 3);
                mma_u8s8(acc[i], a0 & msk, a1 & msk, b0 & msk, b1 & msk, x0, x1);
              }
            }
  #pragma unroll
            for (int q = 0; q < 4; ++q) R[part][q] = acc[0][q] + (acc[1][q] >> 2) + (acc[2][q] >> 4) + (acc[3][q] >> 6);
          }
          // low magnitudes = all - high (the offsets cancel); the high part's offset 2 per weight
          // removed with the block's column sums
          int vv[2][4];
  #pragma unroll
          for (int q = 0; q < 4; ++q) {
            vv[0][q] = R[0][q] - R[1][q];
            vv[1][q] = R[1][q] - 2 * ((q & 1) ? cs1 : cs0);
          }
          // scaled by the block's s_lo and s_hi, into fp64
          const float2 sa = __ldg(sca + blk), sb = __ldg(scb + blk);
  #pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 s2 = (q >> 1) ? sb : sa;
            Y[q] += (double)s2.x * (double)vv[0][q] + (double)s2.y * (double)vv[1][q];
          }
        }
    };
    for (int c = ca; c < cb; ++c, par ^= 1) {
      if (par == 0) {
        chunk(cur, c);
        fetch_next(cur);
      } else {
        chunk(nxt, c);
        fetch_next(nxt);
      }
    }
    if (cb < nch) {                                         // hand the sums to the next part's owner
      const int dst = (int)((8LL * b + 7) / Wc);
#pragma unroll
      for (int q = 0; q < 4; ++q) hand[dst][q][lane] = Y[q];
      __threadfence_block();
      __syncwarp();
      if (lane == 0)
        asm volatile("st.release.cta.shared.s32 [%0], %1;" :: "r"(smem_u32(&hflag[dst])), "r"(1) : "memory");
      continue;
    }
    // ---- outputs: lane t = 0 holds columns 0, 1 of rows g and g + 8, lane t = 1 columns 2, 3 -----
    double w2[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) w2[i] = __shfl_down_sync(0xFFFFFFFFu, Y[i], 1);
    if (t == 0) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int row = row0 + g + 8 * h;
        if (row >= I.N) continue;
        float yv;
        if (MODE == 1) {
          yv = (float)((double)I.sx[0] * Y[2 * h]);
        } else {
          yv = (float)ldexp(((Y[2 * h] * 256.0 + Y[2 * h + 1]) * 256.0 + w2[2 * h]) * 256.0 + w2[2 * h + 1],
                            expo[jj] - kLimbFrac);
        }
        I.y[row] = yv;
      }
    }
  }
}

template <int MODE, int NG>
cudaError_t launch_fv5_one(const Fv5Params& p, size_t smem, cudaStream_t st) {
  auto kern = k_fv5_gemm<MODE, NG>;
  static std::atomic<unsigned long long> smem_raised{0};
  cudaError_t e = allow_max_dynamic_smem(kern, smem_raised);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.ksplit, (p.N + kRows - 1) / kRows, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  int na = 0;
  if (p.ksplit > 1) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = p.ksplit;
    attr[na].val.clusterDim.y = 1;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, kern, p);
}

}  // namespace

size_t fv5_smem_bytes(int mode, int M, int kr) {
  const int ncols = mode == 0 ? 4 * M : M;
  const int ng = (ncols + 7) / 8;
  return (size_t)ncols * (kr / 4 + 16) * 4 + 8 + (size_t)kRows * 8 * ng * 8;
}

int fv5_rows_per_cta() { return kRows; }

cudaError_t launch_fv5_gemm(const Fv5Params& p, cudaStream_t st) {
  const int ng = ((p.mode == 0 ? 4 * p.M : p.M) + 7) / 8;
  const size_t smem = fv5_smem_bytes(p.mode, p.M, p.kr);
  if (p.mode == 1) return ng == 1 ? launch_fv5_one<1, 1>(p, smem, st) : launch_fv5_one<1, 2>(p, smem, st);
  switch (ng) {
    case 1: return launch_fv5_one<0, 1>(p, smem, st);
    case 2: return launch_fv5_one<0, 2>(p, smem, st);
    case 3: return launch_fv5_one<0, 3>(p, smem, st);
    default: return launch_fv5_one<0, 4>(p, smem, st);
  }
}

cudaError_t launch_fv5_batch(Fv5BatchParams& p, cudaStream_t st) {
  // units (16-row tiles) and their costs (512-trit chunks), then contiguous ranges of equal cost,
  // one per CTA, each closed early where its items' staged activations would outgrow the budget
  const int nc = p.mode == 0 ? 4 : 1;
  int64_t units = 0, total = 0;
  p.kmax = 0;
  for (int i = 0; i < p.count; ++i) {
    p.unit0[i] = (int32_t)units;
    units += (p.items[i].N + 15) / 16;
    total += (int64_t)((p.items[i].N + 15) / 16) * (p.items[i].K / 512);
    if (p.items[i].K > p.kmax) p.kmax = p.items[i].K;
    if (fv5_stage_words(nc, p.items[i].K) > kFv5StageBudgetWords) return cudaErrorInvalidValue;
  }
  if (units > 0x7FFFFFFF || total > 0x7FFFFFFF) return cudaErrorInvalidValue;
  p.unit0[p.count] = (int32_t)units;
  // two CTAs per SM (16 warps: the decode and MMA chains of one CTA's 8 warps leave the SM idle)
  long long G = 2LL * device_sm_count();
  if (G > units) G = units;
  if (G < 1) G = 1;
  int c = 0, it = 0, last = -1, nitems = 0, words = 0, max_words = 0;
  int64_t acc = 0, q = 1;
  p.cta_unit[0] = 0;
  for (int64_t u = 0; u < units; ++u) {
    while (it + 1 < p.count && p.unit0[it + 1] <= u) ++it;
    if (it != last) {                                      // the range meets a new item
      const int need = fv5_stage_words(nc, p.items[it].K);
      if (nitems > 0 && (words + need > kFv5StageBudgetWords || nitems == kFv5MaxItemsPerCTA)) {
        if (c + 1 >= kFv5MaxCTAs) return cudaErrorInvalidValue;
        p.cta_unit[++c] = (int32_t)u;
        words = 0;
        nitems = 0;
      }
      words += need;
      ++nitems;
      last = it;
      if (words > max_words) max_words = words;
    }
    acc += p.items[it].K / 512;
    if (q < G && acc * G >= total * q) {                   // a quantile of the cost: close the range
      while (q < G && acc * G >= total * q) ++q;
      if (u + 1 < units) {
        if (c + 1 >= kFv5MaxCTAs) return cudaErrorInvalidValue;
        p.cta_unit[++c] = (int32_t)(u + 1);
        words = 0;
        nitems = 0;
        last = -1;
      }
    }
  }
  const int grid = c + 1;
  p.cta_unit[grid] = (int32_t)units;
  p.grid = grid;
  for (int k = 0, i = 0; k < grid; ++k) {
    while (i + 1 < p.count && p.unit0[i + 1] <= p.cta_unit[k]) ++i;
    p.cta_item[k] = (int16_t)i;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)max_words * 4;
  cfg.stream = st;
  if (p.mode == 0) {
    static std::atomic<unsigned long long> raised{0};
    cudaError_t e = allow_max_dynamic_smem(k_fv5_batch<0>, raised);
    if (e != cudaSuccess) return e;
    return cudaLaunchKernelEx(&cfg, k_fv5_batch<0>, p);
  }
  static std::atomic<unsigned long long> raised1{0};
  cudaError_t e = allow_max_dynamic_smem(k_fv5_batch<1>, raised1);
  if (e != cudaSuccess) return e;
  return cudaLaunchKernelEx(&cfg, k_fv5_batch<1>, p);
}

cudaError_t read_and_clear_fv5_latch(int* out) {
  cudaError_t e = cudaMemcpyFromSymbol(out, g_fv5_latch, sizeof(int));
  if (e != cudaSuccess) return e;
  const int zero = 0;
  return cudaMemcpyToSymbol(g_fv5_latch, &zero, sizeof(int));
}

cudaError_t launch_fv5_pack(const int8_t* codes, int32_t N, int32_t K, uint32_t* planes, int32_t* flag,
                            cudaStream_t st) {
  const int64_t words = (int64_t)N * (K / 32);
  const int64_t cap = (int64_t)device_sm_count() * 16;
  const int64_t blocks = (words + 255) / 256;
  k_fv5_pack<<<(unsigned)(blocks < cap ? blocks : cap), 256, 0, st>>>(codes, words, K / 32, planes, flag);
  return cudaGetLastError();
}

}  // namespace tern
