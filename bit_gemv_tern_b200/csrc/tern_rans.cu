// Order-0 entropy-coded transport of the ternary lane: rANS encode and decode on the device.
//
// The transport of the Neutrino-1 ternary lane is coded close to its order-0 bound (PyTorchKR
// review "Fermion Research, 3진 계열 포맷으로 직접 학습한 Neutrino-1 모델군 3종 공개", section
// "3진 계열이라는 이름의 실체": the 0.6B container shrinks to within 0.007% of that bound); the
// pages do not name the coder. This library uses byte-wise range asymmetric numeral systems
// (J. Duda, 2013) with one static 12-bit frequency table per tensor and one stream per row, so
// that every row decodes on its own thread:
//   symbols s = 0 (t = 0), 1 (t = +1), 2 (t = -1); frequencies f_s >= 1, sum 4096; state x in
//   [2^23, 2^31). Encoding runs from a row's last trit to its first from x = 2^23: while
//   x >= 2^19 f_s emit the low byte of x and shift it out; x = (x / f_s) 4096 + x % f_s + cum_s.
//   The final x follows low byte first; the row's stream is every emitted byte in reverse order.
//   Decoding reads forward: x = the first four bytes, big-endian; per trit slot = x % 4096, s =
//   the symbol whose [cum_s, cum_s + f_s) holds slot, x = f_s (x / 4096) + slot - cum_s, then
//   while x < 2^23: x = 256 x + next byte. A valid row ends at x = 2^23 with all its bytes read.
//   A tensor's frequencies: f_s = max(1, floor(4096 c_s / total)) of its trit counts c_s, the rest
//   (4096 - sum f) added to the most frequent symbol (the lowest s on ties).
// Decoding writes the packed two-plane layout of include/tern.h directly (bit order as tern_pack).
#include <cstdint>
#include <cuda_runtime.h>

#include "tern_device.cuh"
#include "tern_kernels.h"

namespace tern {
namespace {

constexpr uint32_t kRansL = 1u << 23;
constexpr int kRansThreads = 128;

__device__ __forceinline__ void set_flag(int32_t* flag) { atomicExch(flag, 1); }

// Natural-order bits of a 32-trit word -> the layout's order (see tern_pack.cu): bit j moves to
// p(j), which swaps bits 0 and 4 of the index j.
__device__ __forceinline__ uint32_t to_layout_order(uint32_t x) {
  const uint32_t t = lop3<0x28u>(x >> 15, x, 0x0000AAAAu);    // ((x >> 15) ^ x) & 0xAAAA
  return lop3<0x96u>(x, t, t << 15);                         // x ^ t ^ (t << 15)
}

// ---- encode ---------------------------------------------------------------------------------------
// Trit counts of the tensor (zeros, +1, -1); invalid trit values set the flag.
__global__ void k_rans_count(const int8_t* __restrict__ t, int64_t n16, unsigned long long* counts, int32_t* flag) {
  unsigned long long c0 = 0, c1 = 0, c2 = 0;
  bool bad = false;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n16; i += (int64_t)gridDim.x * blockDim.x) {
    const uint4 v = ld_stream(t + 16 * i);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int8_t x = (int8_t)(w[e] >> (8 * b));
        c0 += x == 0;
        c1 += x == 1;
        c2 += x == -1;
        bad |= x < -1 || x > 1;
      }
    }
  }
  for (int o = 16; o > 0; o >>= 1) {
    c0 += __shfl_xor_sync(0xFFFFFFFFu, c0, o);
    c1 += __shfl_xor_sync(0xFFFFFFFFu, c1, o);
    c2 += __shfl_xor_sync(0xFFFFFFFFu, c2, o);
  }
  if ((threadIdx.x & 31) == 0) {
    atomicAdd(&counts[0], c0);
    atomicAdd(&counts[1], c1);
    atomicAdd(&counts[2], c2);
  }
  if (__any_sync(0xFFFFFFFFu, bad) && (threadIdx.x & 31) == 0) set_flag(flag);
}

// The frequency table from the counts (one thread).
__global__ void k_rans_freq(const unsigned long long* counts, uint16_t* freq) {
  if (threadIdx.x != 0) return;
  const long long n = (long long)(counts[0] + counts[1] + counts[2]);
  long long f[3], sum = 0;
  int best = 0;
  for (int s = 0; s < 3; ++s) {
    f[s] = (long long)counts[s] * 4096 / n;
    if (f[s] < 1) f[s] = 1;
    sum += f[s];
    if (counts[s] > counts[best]) best = s;
  }
  f[best] += 4096 - sum;
  for (int s = 0; s < 3; ++s) freq[s] = (uint16_t)f[s];
}

// One thread per row: the row's stream, written backward from the end of its slot of `cap` bytes
// (so it ends up in reading order); its length goes to len[row].
__global__ void __launch_bounds__(kRansThreads) k_rans_encode_rows(const int8_t* __restrict__ t, int32_t N, int32_t K,
                                                                  const uint16_t* __restrict__ freq, uint8_t* slots,
                                                                  int64_t cap, uint32_t* len) {
  const int row = blockIdx.x * blockDim.x + threadIdx.x;
  if (row >= N) return;
  const uint32_t f[3] = {freq[0], freq[1], freq[2]};
  const uint32_t cum[3] = {0u, f[0], f[0] + f[1]};
  const int8_t* tr = t + (int64_t)row * K;
  uint8_t* end = slots + (int64_t)row * cap + cap;      // bytes go to end[-1], end[-2], ...
  int64_t e = 0;
  uint32_t x = kRansL;
  for (int k0 = K - 16; k0 >= 0; k0 -= 16) {
    const uint4 v = ld_stream(tr + k0);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 15; j >= 0; --j) {
      const int8_t tv = (int8_t)(w[j >> 2] >> (8 * (j & 3)));
      const int s = tv == 0 ? 0 : (tv == 1 ? 1 : 2);
      const uint32_t fs = f[s];
      const uint32_t x_max = (1u << 19) * fs;            // <= 2^31: fits
      while (x >= x_max) {
        end[-1 - e] = (uint8_t)(x & 255u);
        ++e;
        x >>= 8;
      }
      x = (x / fs) * 4096u + x % fs + cum[s];
    }
  }
  for (int b = 0; b < 4; ++b) {
    end[-1 - e] = (uint8_t)(x & 255u);
    ++e;
    x >>= 8;
  }
  len[row] = (uint32_t)e;
}

// Inclusive prefix sums of the row lengths -> row_end (one CTA, rows in chunks of its width).
constexpr int kScanThreads = 1024;
__global__ void __launch_bounds__(kScanThreads) k_rans_scan(const uint32_t* __restrict__ len, int32_t N,
                                                           uint32_t* __restrict__ row_end, int32_t* flag) {
  __shared__ unsigned long long warp_tot[kScanThreads / 32];
  __shared__ unsigned long long carry;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int base = 0; base < N; base += kScanThreads) {
    const int i = base + threadIdx.x;
    unsigned long long v = i < N ? len[i] : 0ull;
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long u = __shfl_up_sync(0xFFFFFFFFu, v, o);
      if (lane >= o) v += u;
    }
    if (lane == 31) warp_tot[warp] = v;
    __syncthreads();
    unsigned long long before = carry;
    for (int w = 0; w < warp; ++w) before += warp_tot[w];
    const unsigned long long inc = before + v;
    if (i < N) {
      if (inc > 0xFFFFFFFFull) set_flag(flag);
      row_end[i] = (uint32_t)inc;
    }
    __syncthreads();
    if (threadIdx.x == kScanThreads - 1) carry = inc;
    __syncthreads();
  }
}

// One warp per row: its stream from the tail of its slot to the payload at row_end[row] - len.
__global__ void k_rans_compact(const uint8_t* __restrict__ slots, int64_t cap, const uint32_t* __restrict__ len,
                               const uint32_t* __restrict__ row_end, int32_t N, uint8_t* __restrict__ payload,
                               uint64_t capacity, int32_t* flag) {
  const int row = (int)((blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= N) return;
  const uint32_t n = len[row], e = row_end[row];
  if ((uint64_t)e > capacity || e < n) {                // the payload buffer is too small
    if (lane == 0) set_flag(flag);
    return;
  }
  const uint8_t* src = slots + (int64_t)row * cap + cap - n;
  uint8_t* dst = payload + (e - n);
  for (uint32_t i = lane; i < n; i += 32) dst[i] = src[i];
}

// ---- decode -----------------------------------------------------------------------------------------
// One thread per row of every item (rows of the items back to back). Reads are bounded by the
// row's [start, end) and the item's payload size; a row that is not a valid stream sets the flag.
__global__ void __launch_bounds__(kRansThreads) k_rans_decode(const __grid_constant__ RansBatch p, int32_t* flag) {
  const int64_t g = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (g >= p.rows_total) return;
  int it = 0;
  {
    int lo = 0, hi = p.count - 1;                      // last item with row0 <= g
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (p.row0[mid] <= g) lo = mid; else hi = mid - 1;
    }
    it = lo;
  }
  const RansItem& I = p.items[it];
  const int row = (int)(g - p.row0[it]);
  const uint32_t f[3] = {I.freq[0], I.freq[1], I.freq[2]};
  if (f[0] < 1 || f[1] < 1 || f[2] < 1 || f[0] + f[1] + f[2] != 4096u) {
    set_flag(flag);
    return;
  }
  const uint32_t c1 = f[0], c2 = f[0] + f[1];
  const uint32_t start = row ? I.row_end[row - 1] : 0u, end = I.row_end[row];
  if (end < start || end - start < 4 || (uint64_t)end > I.payload_bytes) {
    set_flag(flag);
    return;
  }
  const uint8_t* s = I.payload;
  uint32_t p0 = start;
  uint32_t x = ((uint32_t)__ldg(s + p0) << 24) | ((uint32_t)__ldg(s + p0 + 1) << 16) |
               ((uint32_t)__ldg(s + p0 + 2) << 8) | (uint32_t)__ldg(s + p0 + 3);
  p0 += 4;
  // the next four stream bytes, loaded ahead (zeros past the row's end; reading one of those is
  // an error caught by the position check)
  uint32_t ahead = 0u;
#pragma unroll
  for (int b = 0; b < 4; ++b) ahead = (ahead << 8) | (p0 + b < end ? (uint32_t)__ldg(s + p0 + b) : 0u);
  const int KW = I.K / 32;                             // a multiple of 4 (K % 128 == 0)
  uint32_t* rowp = I.planes + (int64_t)row * 2 * KW;
  bool ok = true;
  // four words (128 trits) per plane at a time, written as one 16-byte store each: every thread
  // writes its own row, so word-sized stores would each touch a sector of their own
  for (int w0 = 0; w0 < KW && ok; w0 += 4) {
    uint32_t mw[4], sw[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      uint32_t m = 0u, sg = 0u;
#pragma unroll 8
      for (int j = 0; j < 32; ++j) {
        const uint32_t slot = x & 4095u;
        const uint32_t sym = (slot >= c1) + (slot >= c2);
        const uint32_t fs = sym == 0 ? f[0] : (sym == 1 ? f[1] : f[2]);
        const uint32_t cs = sym == 0 ? 0u : (sym == 1 ? c1 : c2);
        m |= (uint32_t)(sym != 0) << j;
        sg |= (uint32_t)(sym == 2) << j;
        x = fs * (x >> 12) + slot - cs;
#pragma unroll 1
        for (int r = 0; r < 2 && x < kRansL; ++r) {   // at most two bytes per trit (x >= 2^11 here)
          x = (x << 8) | (ahead >> 24);
          const uint32_t q = p0 + 4;
          ahead = (ahead << 8) | (q < end ? (uint32_t)__ldg(s + q) : 0u);
          ++p0;
        }
      }
      mw[u] = to_layout_order(m);
      const uint32_t sp = to_layout_order(sg);
      sw[u] = (sp << 1) | (sp >> 31);                  // the sign bit sits one above its mask bit
    }
    *reinterpret_cast<uint4*>(rowp + w0) = make_uint4(mw[0], mw[1], mw[2], mw[3]);
    *reinterpret_cast<uint4*>(rowp + KW + w0) = make_uint4(sw[0], sw[1], sw[2], sw[3]);
    ok = p0 <= end;
  }
  if (!ok || x != kRansL || p0 != end) set_flag(flag);
}

}  // namespace

size_t rans_slot_bytes(int32_t K) { return ((size_t)2 * K + 8 + 15) & ~(size_t)15; }

size_t rans_workspace_bytes(int32_t N, int32_t K) {
  return 64 + (size_t)N * 4 + (size_t)N * rans_slot_bytes(K);
}

cudaError_t launch_rans_encode(const int8_t* trits, int32_t N, int32_t K, uint16_t* freq, uint32_t* row_end,
                               uint8_t* payload, uint64_t capacity, void* workspace, int32_t* flag, cudaStream_t st) {
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  unsigned long long* counts = reinterpret_cast<unsigned long long*>(ws);
  uint32_t* len = reinterpret_cast<uint32_t*>(ws + 64);
  uint8_t* slots = ws + 64 + (((size_t)N * 4 + 15) & ~(size_t)15);
  const int64_t cap = (int64_t)rans_slot_bytes(K);
  cudaError_t e = cudaMemsetAsync(counts, 0, 3 * sizeof(unsigned long long), st);
  if (e != cudaSuccess) return e;
  const int64_t n16 = (int64_t)N * K / 16;
  const int64_t cap_grid = (int64_t)device_sm_count() * 8;
  const int grid = (int)((n16 + 255) / 256 < cap_grid ? (n16 + 255) / 256 : cap_grid);
  k_rans_count<<<grid < 1 ? 1 : grid, 256, 0, st>>>(trits, n16, counts, flag);
  k_rans_freq<<<1, 32, 0, st>>>(counts, freq);
  k_rans_encode_rows<<<(N + kRansThreads - 1) / kRansThreads, kRansThreads, 0, st>>>(trits, N, K, freq, slots, cap, len);
  k_rans_scan<<<1, kScanThreads, 0, st>>>(len, N, row_end, flag);
  const int64_t threads = (int64_t)N * 32;
  k_rans_compact<<<(unsigned)((threads + 255) / 256), 256, 0, st>>>(slots, cap, len, row_end, N, payload, capacity,
                                                                    flag);
  return cudaGetLastError();
}

cudaError_t launch_rans_decode(RansBatch& p, int32_t* flag, cudaStream_t st) {
  int64_t rows = 0;
  for (int i = 0; i < p.count; ++i) {
    p.row0[i] = rows;
    rows += p.items[i].N;
  }
  p.rows_total = rows;
  if (rows < 1) return cudaSuccess;
  k_rans_decode<<<(unsigned)((rows + kRansThreads - 1) / kRansThreads), kRansThreads, 0, st>>>(p, flag);
  return cudaGetLastError();
}

}  // namespace tern
