// Internal launch interface between the C ABI (tern_abi.cu) and the kernel files.
#pragma once

#include <atomic>
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/tern.h"

namespace tern {

// Persistent kernels launch at most one CTA per SM and at most kMaxGridCTAs of them (the batch
// plan keeps one split record per CTA in the kernel parameters); 148 = the SMs of a B200.
constexpr int kMaxGridCTAs = 148;

// SMs of the current device (148 on a B200; 148 if the query fails, which the launch then reports).
inline int device_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      n <= 0)
    return kMaxGridCTAs;
  return n;
}

// CTAs of a persistent launch over `work` units: one per SM, at most kMaxGridCTAs and `work`.
inline int persistent_grid(long long work) {
  long long g = device_sm_count();
  if (g > kMaxGridCTAs) g = kMaxGridCTAs;
  if (work < g) g = work;
  return g < 1 ? 1 : (int)g;
}

// Allow a kernel the device's whole opt-in dynamic shared memory (less its static shared memory).
// The attribute belongs to one device, so each device is set up on its first launch there; `done`
// holds one bit per device index below 64 (devices past that are set up on every launch). Two host
// threads that race here both set the same value.
template <typename F>
cudaError_t allow_max_dynamic_smem(F* kern, std::atomic<unsigned long long>& done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = (dev >= 0 && dev < 64) ? 1ull << dev : 0ull;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  int optin = 0;
  e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return e;
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, optin - (int)fa.sharedSizeBytes);
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

// Prefer the largest shared-memory carveout for a kernel that runs just before (and overlaps) a
// kernel using nearly all of an SM's shared memory: an SM whose L1/shared split must change waits
// until its resident CTAs have left, so a small kernel at the default carveout would hold the big
// one off its SM. Set up once per device, as above.
template <typename F>
cudaError_t prefer_max_shared_carveout(F* kern, std::atomic<unsigned long long>& done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = (dev >= 0 && dev < 64) ? 1ull << dev : 0ull;
  if (bit && (done.load(std::memory_order_acquire) & bit)) return cudaSuccess;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, (int)cudaSharedmemCarveoutMaxShared);
  if (e == cudaSuccess && bit) done.fetch_or(bit, std::memory_order_acq_rel);
  return e;
}

// Ternary GEMV / small-M GEMM (tern_gemv.cu).
struct GemmParams {
  const uint32_t* planes;
  const uint16_t* scale;
  int32_t N, K;
  const void* x;          // bf16 bits [M][K] (mode 0) or int8 [M][K] (mode 1)
  const float* sx;        // [M], int8 mode only
  float* y;               // [M][N]
  int32_t* acc;           // int8 mode, optional: the exact sums sum_k t*q, [M][N]
  int32_t M;              // 1..16
  int32_t mode;           // 0 = bf16 activations, 1 = int8 activations
  int32_t kr;             // trits of K per CTA (multiple of 128); ksplit * kr == K
  int32_t ksplit;         // CTAs splitting K in one cluster: 1, 2, 4 or 8
};
size_t gemm_smem_bytes(int mode, int M, int kr);
int gemm_rows_per_cta();
cudaError_t launch_tern_gemm(const GemmParams& p, bool pdl, cudaStream_t st);

// Persistent TMA-fed M = 1 GEMV (tern_stream.cu).
struct StreamParams {
  const uint32_t* planes;
  const uint16_t* scale;
  int32_t N, K;
  const void* x;          // bf16 bits [K] (mode 0) or int8 [K] (mode 1)
  const float* sx;        // [1], int8 mode only
  float* y;               // [N]
  int32_t* acc;           // int8 mode, optional: the exact sums sum_k t*q, [N]
  int32_t mode;
  int32_t ks;             // trits of K per stage (divides K)
  int32_t ts;             // tiles of 16 rows per stage (1, 2, 4 or 8)
  int32_t pitch;          // shared-memory bytes per staged row
  int32_t stage_bytes;
  int32_t stages;         // ring depth
  int32_t tiles;          // ceil(N / 16)
  int32_t x_words;        // shared-memory words per staged activation column
  int32_t cw;             // consumer warps: 8 (two CTAs per SM) or 16 (one CTA per SM)
};
bool plan_stream(int N, int K, int mode, StreamParams& p, size_t& smem);
cudaError_t launch_stream(const StreamParams& p, size_t smem, bool pdl, cudaStream_t st);
// Reads and clears the device word that kernels set when a bounded wait gives up.
cudaError_t read_and_clear_error_latch(int* out, cudaStream_t st);

// Batched GEMV / small-M GEMM over a list of matrices (tern_batch.cu).
struct BatchItem {
  const uint16_t* scale;
  float* y;               // [M][N]
  const float* sx;        // int8 mode: s_x [M] (written by the prep launch for prologue items)
  int32_t N, K;
  int32_t kp;             // 512-trit K parts (the last may be partial): stages per row block
  int32_t unit0;          // first global unit (row block) of the item
  int32_t units;          // row blocks of the item
  int32_t part0;          // first global part (unit x 512-trit K part) of the item
  uint32_t xoff;          // byte offset of the item's operand block in the workspace
};
constexpr int kBatchMaxItems = 160;
struct BatchParams {
  CUtensorMap tmap[kBatchMaxItems];  // per item: planes viewed as [2 planes][N rows][K/32 words]
  BatchItem items[kBatchMaxItems];
  int32_t count;
  int32_t mode;           // 0 = bf16 activations (four int8 limbs), 1 = int8
  int32_t nc;             // operand columns of a segment
  int32_t M;              // activation rows (tokens), 1..16
  int32_t mp;             // token slots: 1, 2 / 4 (bf16 mode), 8 or 16
  int32_t tpw;            // tiles of 16 rows per consumer warp
  int32_t cw;             // consumer warps
  int32_t total_units;
  int32_t grid;
  int32_t stages;
  int32_t stage_slot_bytes;
  int32_t seg_bytes;      // operand bytes of one 512-trit part (all columns + sums + exponent)
  uint8_t* xprep;         // workspace: operand blocks
  int32_t cta_part[kMaxGridCTAs + 1];  // CTA c handles global parts [cta_part[c], cta_part[c + 1])
  int16_t cta_item[kMaxGridCTAs];      // the item holding CTA c's first part (no scan of items[] at entry)
  // Row blocks split between CTAs: each contributor adds exact partial sums into a workspace
  // slot; the last one (per warp, by counter) writes the outputs.
  // per CTA, 8 bits each: slot of its first block + 1, that block's contributors, slot of its
  // last block + 1, that block's contributors (slot + 1 = 0: the block is this CTA's alone)
  uint32_t cta_split[kMaxGridCTAs];
  int32_t nslots;
  uint32_t scratch_off;   // workspace byte offset: [nslots][rows][8 * groups] int32, then counters
  int32_t scratch_words;  // words to zero before the stream (sums and counters)
  int32_t tc;             // 1: the tensor-core (tcgen05) small-M kernels of tern_tc.cu
  uint32_t meta_off;      // tc: workspace byte offset of the token exponents E [count][16] int32
};
static_assert(sizeof(BatchParams) <= 32764, "kernel parameter limit");
// The operand preparation of one item (the prep launch): where its activation comes from and the
// prologue that turns it into the linear's bf16 (or int8) activation (tern_prologue.cuh).
struct PrepItem {
  const void* x;          // kProNone: bf16 [M][K] (bf16 mode) or int8 q [M][K]; kProBF16: bf16 [M][K];
                          // kProCast, kProRMSNorm: fp32 [M][K]; kProSwiGLU: fp32 [M][2K] (gate | up)
  const uint16_t* gain;   // kProRMSNorm: bf16 [K]
  void* xout;             // prologue items, optional: the prepared activation (bf16, or int8 q) [M][K]
  float* sx_out;          // prologue items in int8 mode: s_x [M]
  float eps;              // kProRMSNorm
  int32_t kind;           // kProNone .. kProSwiGLU
  int32_t K, kp;
  uint32_t xoff;          // byte offset of the item's operand block in the workspace
};
struct PrepParams {
  PrepItem items[kBatchMaxItems];
  int32_t count, mode, M, mp, seg_bytes;
  uint8_t* xprep;
  uint32_t scratch_off;
  int32_t scratch_words;
  uint32_t meta_off;      // tc: token exponents E [count][16] int32
};
static_assert(sizeof(PrepParams) <= 32764, "kernel parameter limit");
// Host: fills tmap/kp/units/xoff, the stage ring and the CTA split; fails on unsupported shapes.
bool plan_batch(BatchParams& p, const uint32_t* const* planes, size_t& smem, size_t& workspace);
// Copies the plan's per-item fields (K, kp, xoff, mode, workspace layout) into the prep parameters,
// whose activation sources and prologues the caller has filled.
void plan_prep(const BatchParams& b, PrepParams& q);
cudaError_t launch_batch(const BatchParams& p, const PrepParams& q, size_t smem, bool pdl, cudaStream_t st);
cudaError_t read_and_clear_batch_latch(int* out);
// Small-M lists on tcgen05 (tern_tc.cu): the shape of the plan when BatchParams::tc is set, and the
// launch pair (operand preparation, stream) that replaces launch_batch's.
int tc_token_slots(int mode, int M);
int tc_segment_bytes(int mode, int mp);
int tc_stage_rows();
int tc_consumer_warps();
size_t tc_smem_bytes(int stages, int slot_bytes);
cudaError_t launch_tc(const BatchParams& p, const PrepParams& q, size_t smem, bool pdl, cudaStream_t st);
cudaError_t read_and_clear_tc_latch(int* out);

// Prefill dense contraction on tcgen05 (tern_prefill.cu).
struct PrefillParams {
  CUtensorMap xmap;       // X bf16 [M][K], boxes of 64 x (128 * halves), 128-byte swizzle
  const uint32_t* planes;
  const uint16_t* scale;
  float* Y;               // [M][N]
  int32_t M, N, K;
  int32_t vec_store;      // Y rows 16-byte aligned (N % 4 == 0 and Y aligned): 128-bit stores
  int32_t halves;         // 128-token halves per tile (1 or 2), set by plan_prefill
};
bool plan_prefill(PrefillParams& p, const uint16_t* X, int& grid, size_t& smem);
cudaError_t launch_prefill(const PrefillParams& p, int grid, size_t smem, cudaStream_t st);
cudaError_t read_and_clear_prefill_latch(int* out);

// int8 output head with argmax (tern_head.cu).
struct HeadParams {
  const int8_t* W;
  const uint16_t* sh;
  int32_t V, K, M;
  int32_t mode;           // 0 = bf16 activations (three exact int8 limbs), 1 = int8 activations
  const void* x;
  const float* sx;
  int32_t* argmax;
  float* maxval;
  float* logits;          // optional [M][V]
  unsigned long long* keys;  // workspace: M packed (value key, index) maxima
  unsigned int* counter;     // workspace: CTAs finished
  const float* bscale;       // block-scaled head (FV5B-style), optional: fp32 [V][K / 256]
  const int32_t* draft;      // verify round, optional: M - 1 drafted tokens
  int32_t* accept;           // verify round: {accepted drafts n, next token argmax[n]}
  int32_t kr, ksplit;
  int32_t nrb;            // row blocks of 128 rows
  int32_t nby;            // CTAs along the row-block axis (persistent loop)
};
size_t head_workspace_bytes(int M);
size_t head_smem_bytes(int mode, int M, int kr, bool block_scaled);
cudaError_t launch_head(const HeadParams& p, bool pdl, cudaStream_t st);
cudaError_t launch_verify_accept(const int32_t* argmax, const int32_t* draft, int32_t k, int32_t* accept,
                                 cudaStream_t st);
// Every argument check of i8_head_gemv_argmax_ex and its launch plan (tern_abi.cu); enqueues nothing.
tern_status plan_head_call(const int8_t* W_dev, const uint16_t* scale_f16_dev, int32_t V, int32_t K, int32_t M,
                           tern_act act, const void* X_dev, const float* x_scale_dev, int32_t* argmax_dev,
                           float* maxval_dev, float* logits_dev, void* workspace_dev, size_t workspace_bytes,
                           uint32_t flags, HeadParams& p, const float* block_scale_dev);

// Loader kernels (tern_pack.cu).
constexpr int kPackMaxItems = 256;
struct Base3Batch {
  const uint8_t* src[kPackMaxItems];
  uint32_t* planes[kPackMaxItems];
  int32_t N[kPackMaxItems], K[kPackMaxItems];
  int32_t rows[kPackMaxItems];     // rows per CTA (set by the launcher)
  int32_t block0[kPackMaxItems];   // first CTA of each item (set by the launcher)
  int32_t count;
};
cudaError_t launch_unpack_base3_batch(Base3Batch& p, int32_t* flag, cudaStream_t st);
// int8 trits of several tensors packed in one launch: work units of 16 rows x 128 words.
struct PackBatch {
  const int8_t* src[kPackMaxItems];
  uint32_t* planes[kPackMaxItems];
  int32_t N[kPackMaxItems], KM[kPackMaxItems];     // rows, words per row and plane (K / 32)
  int32_t unit0[kPackMaxItems];                    // first work unit of each item (set by the launcher)
  int32_t count, units;
};
cudaError_t launch_pack_trits_batch(PackBatch& p, int32_t* flag, cudaStream_t st);
cudaError_t launch_pack_trits(const int8_t* src, int32_t N, int32_t K, uint32_t* planes, int32_t* flag,
                              cudaStream_t st);
cudaError_t launch_unpack_base3(const uint8_t* src, int32_t N, int32_t K, uint32_t* planes, int32_t* flag,
                                cudaStream_t st);
cudaError_t launch_encode_base3(const int8_t* src, int32_t N, int32_t K, uint8_t* out, int32_t* flag,
                                cudaStream_t st);
cudaError_t launch_occupancy(const uint32_t* planes, int32_t N, int32_t K, int64_t* counts, cudaStream_t st);

// Dependent decode chain in one cooperative launch (tern_chain.cu). The plan (this array) lives in
// device memory; tensor maps need 64-byte alignment there.
struct alignas(64) ChainItem {
  CUtensorMap tmap;           // planes as [plane 2][row N][word K/32]
  const uint16_t* scale;      // fp16 [N]
  float* y;                   // fp32 [N]
  uint16_t* hout;             // SwiGLU output bf16 [N / 2] (rows interleave gate and up by 8), or null
  float* sx_out;              // int8 mode: s_x of this linear's activation, or null
  const void* src;            // the activation's source: bf16 [K] (kProBF16) or fp32 [K]
  const uint16_t* gain;       // kProRMSNorm: bf16 [K]
  float eps;
  int32_t kind;               // kProBF16, kProCast or kProRMSNorm
  int32_t dep;                // linear whose outputs src holds (-1: written before the launch)
  int32_t N, K, kp;
  int32_t rows;               // rows of a chunk (a multiple of 16, <= 192); CTA c owns chunks c, c + grid, ...
  int32_t chunks;             // ceil(N / rows)
  int32_t ps;                 // 512-trit parts per ring stage
  int32_t nst;                // stages per chunk: ceil(kp / ps)
  int32_t dep_need;           // CTAs that release the linear dep: min(its chunks, grid)
};
struct ChainParams {
  const ChainItem* items;     // device
  int32_t count, mode, grid, stages;
  int32_t seg_parts;          // operand segment slots in shared memory (parts a CTA streams per linear)
  int32_t* done;              // device: completion counter of each linear [count]
  int32_t* finished;          // device: CTAs finished with the whole chain
  int32_t* scratch;           // unused (no output needs another CTA's sums)
};
struct ChainLayout {
  int stages;
  int seg_parts;
  size_t smem;
  size_t scratch_words;
};
// grid: the launch's CTAs (chain_grid()), which fixes how many parts a CTA prepares per linear.
bool plan_chain(ChainItem* items, int count, int mode, int grid, const uint32_t* const* planes, ChainLayout& L);
cudaError_t launch_chain(const ChainParams& p, size_t smem, cudaStream_t st);
int chain_grid();
cudaError_t read_and_clear_chain_latch(int* out);

// Five-valued weights (tern_fv5.cu).
struct Fv5Params {
  const uint32_t* planes;     // [N][3 K / 32]: mask, sign, magnitude planes (words transposed per 512 trits)
  const float* scales;        // [N][K / 256][2]: s_lo, s_hi
  int32_t N, K;
  const void* x;              // bf16 [M][K] or int8 [M][K]
  const float* sx;            // int8 mode: [M]
  float* y;                   // [M][N]
  int32_t M, mode, kr, ksplit;
};
// A list of five-valued linears at M = 1 in one persistent launch (tern_fv5.cu): units of 128 rows
// of one item over the whole of K, cut into contiguous, cost-balanced ranges per CTA.
struct Fv5BatchItem {
  const uint32_t* planes;
  const float* scales;
  const void* x;              // bf16 [K] or int8 [K]
  const float* sx;            // int8 mode: [1]
  float* y;                   // [N]
  int32_t N, K;
};
// Two CTAs per SM, plus one extra range per item at most (a range closes early where its items'
// staged activations would outgrow the budget below).
constexpr int kFv5MaxCTAs = 2 * kMaxGridCTAs + kBatchMaxItems;
constexpr int kFv5MaxItemsPerCTA = 32;
constexpr int kFv5StageBudgetWords = 24576;   // 96 KB of staged activations per CTA
// Words one item's staged activation takes: nc operand columns of K / 4 + 4 words, then nc column
// sums per 256-weight block; rounded up to four words (16-byte aligned columns).
__host__ __device__ inline int fv5_stage_words(int nc, int K) { return (nc * (K / 4 + 4) + nc * (K / 256) + 3) & ~3; }
struct Fv5BatchParams {
  Fv5BatchItem items[kBatchMaxItems];
  int32_t unit0[kBatchMaxItems + 1];   // first unit of each item; unit0[count] = all units
  int32_t cta_unit[kFv5MaxCTAs + 1];   // CTA c takes units [cta_unit[c], cta_unit[c + 1])
  int16_t cta_item[kFv5MaxCTAs];       // the item of CTA c's first unit
  int32_t count, mode, grid, kmax;
};
cudaError_t launch_fv5_batch(Fv5BatchParams& p, cudaStream_t st);
cudaError_t read_and_clear_fv5_latch(int* out);
size_t fv5_smem_bytes(int mode, int M, int kr);
int fv5_rows_per_cta();
cudaError_t launch_fv5_gemm(const Fv5Params& p, cudaStream_t st);
cudaError_t launch_fv5_pack(const int8_t* codes, int32_t N, int32_t K, uint32_t* planes, int32_t* flag,
                            cudaStream_t st);

// Order-0 rANS transport (tern_rans.cu).
struct RansItem {
  const uint16_t* freq;       // device: the tensor's three 12-bit frequencies (t = 0, +1, -1)
  const uint32_t* row_end;    // device: end byte of each row's stream in the payload [N]
  const uint8_t* payload;     // device: the rows' streams back to back
  uint64_t payload_bytes;     // bytes of the payload buffer (reads never go past it)
  int32_t N, K;
  uint32_t* planes;           // output: packed planes, N * K / 16 words
};
struct RansBatch {
  RansItem items[kPackMaxItems];
  int64_t row0[kPackMaxItems];  // first global row of each item (set by the launcher)
  int64_t rows_total;
  int32_t count;
};
size_t rans_slot_bytes(int32_t K);
size_t rans_workspace_bytes(int32_t N, int32_t K);
cudaError_t launch_rans_encode(const int8_t* trits, int32_t N, int32_t K, uint16_t* freq, uint32_t* row_end,
                               uint8_t* payload, uint64_t capacity, void* workspace, int32_t* flag, cudaStream_t st);
cudaError_t launch_rans_decode(RansBatch& p, int32_t* flag, cudaStream_t st);

// Activation quantiser and standalone prologue (tern_act.cu).
cudaError_t launch_quantize(const uint16_t* x, int32_t M, int32_t K, int8_t* q, float* sx, cudaStream_t st);
cudaError_t launch_prologue(int32_t kind, const void* src, const uint16_t* gain, float eps, int32_t M, int32_t K,
                            uint16_t* out, cudaStream_t st);

}  // namespace tern
