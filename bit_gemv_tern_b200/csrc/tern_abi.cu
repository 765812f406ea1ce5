// C ABI of libterngemv.so (declared and documented in include/tern.h): argument validation,
// launch planning and kernel launches. No entry point allocates device memory or keeps state.
#include <cstdint>
#include <cuda_runtime.h>
#include <new>

#include "../../include/tern.h"
#include "tern_kernels.h"

namespace {

// Consumer warps of the M = 1 streaming kernel (8: two CTAs per SM; 16: one CTA per SM).
#ifndef TERN_STREAM_CW
#define TERN_STREAM_CW 16
#endif
constexpr size_t kGemmSmemCap = 160 * 1024;
constexpr size_t kHeadSmemCap = 100 * 1024;

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }
inline cudaStream_t cs(tern_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }
inline tern_status from_cuda(cudaError_t e) { return e == cudaSuccess ? TERN_OK : TERN_ECUDA; }

bool valid_shape(int32_t N, int32_t K) { return N > 0 && K > 0 && (K % 128) == 0; }

tern_status check_matrix(const tern_matrix* W) {
  if (!W || !W->planes || !W->scale_f16) return TERN_EINVAL;
  if (!valid_shape(W->N, W->K)) return TERN_ESHAPE;
  if (!aligned(W->planes, 16) || !aligned(W->scale_f16, 2)) return TERN_EINVAL;
  return TERN_OK;
}

// Split K over a cluster of up to 8 CTAs so that small matrices still cover every SM.
bool plan_gemm(int N, int K, int M, int mode, int& ksplit) {
  const int row_blocks = (N + tern::gemm_rows_per_cta() - 1) / tern::gemm_rows_per_cta();
  const int units = K / 128;
  const int sms = tern::device_sm_count();
  int ks = 1;
  while (ks < 8 && row_blocks * ks < 2 * sms && units % (2 * ks) == 0) ks *= 2;
  while (tern::gemm_smem_bytes(mode, M, K / ks) > kGemmSmemCap && ks < 8 && units % (2 * ks) == 0) ks *= 2;
  if (tern::gemm_smem_bytes(mode, M, K / ks) > kGemmSmemCap) return false;
  ksplit = ks;
  return true;
}

}  // namespace

namespace tern {

// Every argument check of i8_head_gemv_argmax_ex and its launch plan, with nothing enqueued.
tern_status plan_head_call(const int8_t* W_dev, const uint16_t* scale_f16_dev, int32_t V, int32_t K, int32_t M,
                           tern_act act, const void* X_dev, const float* x_scale_dev, int32_t* argmax_dev,
                           float* maxval_dev, float* logits_dev, void* workspace_dev, size_t workspace_bytes,
                           uint32_t flags, HeadParams& p, const float* block_scale_dev) {
  const bool bs = block_scale_dev != nullptr;
  if (!W_dev || (!bs && !scale_f16_dev) || !X_dev || !argmax_dev || !maxval_dev || !workspace_dev) return TERN_EINVAL;
  if (act != TERN_ACT_BF16 && act != TERN_ACT_INT8) return TERN_EINVAL;
  if (flags & ~TERN_FLAG_PDL) return TERN_EINVAL;
  if (!valid_shape(V, K) || M < 1 || M > 16) return TERN_ESHAPE;
  if (bs && (K % 256 || (act == TERN_ACT_BF16 && M > 8))) return TERN_ESHAPE;
  if (!aligned(W_dev, 16) || !aligned(X_dev, 16) || !aligned(workspace_dev, 16) ||
      (!bs && !aligned(scale_f16_dev, 2)) || (bs && !aligned(block_scale_dev, 4)))
    return TERN_EINVAL;
  if (!aligned(argmax_dev, 4) || !aligned(maxval_dev, 4) || (logits_dev && !aligned(logits_dev, 4)))
    return TERN_EINVAL;
  if (act == TERN_ACT_INT8 && (!x_scale_dev || !aligned(x_scale_dev, 4))) return TERN_EINVAL;
  if (workspace_bytes < head_workspace_bytes(M)) return TERN_EINVAL;
  p = HeadParams{};
  p.W = W_dev;
  p.sh = scale_f16_dev;
  p.V = V;
  p.K = K;
  p.M = M;
  p.mode = act == TERN_ACT_BF16 ? 0 : 1;
  p.x = X_dev;
  p.sx = x_scale_dev;
  p.argmax = argmax_dev;
  p.maxval = maxval_dev;
  p.logits = logits_dev;
  p.counter = static_cast<unsigned int*>(workspace_dev);
  p.keys = reinterpret_cast<unsigned long long*>(static_cast<char*>(workspace_dev) + 16);
  p.bscale = block_scale_dev;
  const int units = K / (bs ? 256 : 128);            // a K slice holds whole units
  int ks = 1;
  while (head_smem_bytes(p.mode, M, K / ks, bs) > kHeadSmemCap && ks < 8 && units % (2 * ks) == 0) ks *= 2;
  if (head_smem_bytes(p.mode, M, K / ks, bs) > kHeadSmemCap) return TERN_ESHAPE;
  p.ksplit = ks;
  p.kr = K / ks;
  p.nrb = (V + 127) / 128;
  int nby = (2 * device_sm_count()) / ks;
  if (nby > p.nrb) nby = p.nrb;
  if (nby < 1) nby = 1;
  p.nby = nby;
  return TERN_OK;
}

}  // namespace tern

extern "C" {

const char* tern_status_string(tern_status s) {
  switch (s) {
    case TERN_OK: return "TERN_OK";
    case TERN_EINVAL: return "TERN_EINVAL: invalid argument";
    case TERN_ESHAPE: return "TERN_ESHAPE: invalid shape";
    case TERN_EBADCODE: return "TERN_EBADCODE: invalid trit or transport byte in the input";
    case TERN_ECUDA: return "TERN_ECUDA: CUDA error";
    case TERN_ETIMEOUT: return "TERN_ETIMEOUT: bounded device wait gave up";
  }
  return "unknown tern_status";
}

size_t tern_packed_bytes(int32_t N, int32_t K) {
  return valid_shape(N, K) ? (size_t)N * (size_t)K / 4 : 0;
}

size_t tern_base3_bytes(int32_t N, int32_t K) {
  return valid_shape(N, K) ? (size_t)N * (size_t)((K + 4) / 5) : 0;
}

tern_status tern_pack(tern_src src, const void* src_dev, int32_t N, int32_t K, uint32_t* planes_dev,
                      int32_t* err_flag_dev, tern_stream_t stream) {
  if (!src_dev || !planes_dev || !err_flag_dev) return TERN_EINVAL;
  if (src != TERN_SRC_INT8_TRITS && src != TERN_SRC_BASE3) return TERN_EINVAL;
  if (!valid_shape(N, K)) return TERN_ESHAPE;
  if (!aligned(planes_dev, 16) || !aligned(err_flag_dev, 4)) return TERN_EINVAL;
  if (src == TERN_SRC_INT8_TRITS && !aligned(src_dev, 16)) return TERN_EINVAL;
  if (src == TERN_SRC_BASE3 && !aligned(src_dev, 4)) return TERN_EINVAL;
  cudaError_t e = cudaMemsetAsync(err_flag_dev, 0, sizeof(int32_t), cs(stream));
  if (e != cudaSuccess) return TERN_ECUDA;
  if (src == TERN_SRC_INT8_TRITS)
    e = tern::launch_pack_trits(static_cast<const int8_t*>(src_dev), N, K, planes_dev, err_flag_dev, cs(stream));
  else
    e = tern::launch_unpack_base3(static_cast<const uint8_t*>(src_dev), N, K, planes_dev, err_flag_dev, cs(stream));
  return from_cuda(e);
}

tern_status tern_pack_batch(tern_src src, const tern_pack_item* items, int32_t count, int32_t* err_flag_dev,
                            tern_stream_t stream) {
  if (!items || !err_flag_dev) return TERN_EINVAL;
  if (src != TERN_SRC_INT8_TRITS && src != TERN_SRC_BASE3) return TERN_EINVAL;
  if (count < 1 || count > TERN_PACK_MAX_ITEMS) return TERN_ESHAPE;
  if (!aligned(err_flag_dev, 4)) return TERN_EINVAL;
  for (int i = 0; i < count; ++i) {
    const tern_pack_item& it = items[i];
    if (!it.src_dev || !it.planes_dev) return TERN_EINVAL;
    if (!valid_shape(it.N, it.K)) return TERN_ESHAPE;
    if (!aligned(it.planes_dev, 16) || !aligned(it.src_dev, src == TERN_SRC_BASE3 ? 4 : 16)) return TERN_EINVAL;
  }
  cudaError_t e = cudaMemsetAsync(err_flag_dev, 0, sizeof(int32_t), cs(stream));
  if (e != cudaSuccess) return TERN_ECUDA;
  if (src == TERN_SRC_INT8_TRITS) {
    tern::PackBatch* pb = new (std::nothrow) tern::PackBatch();
    if (!pb) return TERN_EINVAL;
    pb->count = count;
    for (int i = 0; i < count; ++i) {
      pb->src[i] = static_cast<const int8_t*>(items[i].src_dev);
      pb->planes[i] = items[i].planes_dev;
      pb->N[i] = items[i].N;
      pb->KM[i] = items[i].K / 32;
    }
    e = tern::launch_pack_trits_batch(*pb, err_flag_dev, cs(stream));
    delete pb;
    return from_cuda(e);
  }
  tern::Base3Batch* b = new (std::nothrow) tern::Base3Batch();
  if (!b) return TERN_EINVAL;
  b->count = count;
  for (int i = 0; i < count; ++i) {
    b->src[i] = static_cast<const uint8_t*>(items[i].src_dev);
    b->planes[i] = items[i].planes_dev;
    b->N[i] = items[i].N;
    b->K[i] = items[i].K;
  }
  e = tern::launch_unpack_base3_batch(*b, err_flag_dev, cs(stream));
  delete b;
  return from_cuda(e);
}

size_t tern_rans_payload_bound(int32_t N, int32_t K) {
  return valid_shape(N, K) ? (size_t)N * (tern::rans_slot_bytes(K)) : 0;
}

size_t tern_rans_workspace_bytes(int32_t N, int32_t K) {
  return valid_shape(N, K) ? tern::rans_workspace_bytes(N, K) : 0;
}

tern_status tern_rans_encode(const int8_t* trits_dev, int32_t N, int32_t K, uint16_t* freq_dev, uint32_t* row_end_dev,
                             uint8_t* payload_dev, size_t payload_capacity, void* workspace_dev, size_t workspace_bytes,
                             int32_t* err_flag_dev, tern_stream_t stream) {
  if (!trits_dev || !freq_dev || !row_end_dev || !payload_dev || !workspace_dev || !err_flag_dev) return TERN_EINVAL;
  if (!valid_shape(N, K)) return TERN_ESHAPE;
  if (!aligned(trits_dev, 16) || !aligned(freq_dev, 2) || !aligned(row_end_dev, 4) || !aligned(workspace_dev, 16) ||
      !aligned(err_flag_dev, 4))
    return TERN_EINVAL;
  if (workspace_bytes < tern::rans_workspace_bytes(N, K)) return TERN_EINVAL;
  if (cudaMemsetAsync(err_flag_dev, 0, sizeof(int32_t), cs(stream)) != cudaSuccess) return TERN_ECUDA;
  return from_cuda(tern::launch_rans_encode(trits_dev, N, K, freq_dev, row_end_dev, payload_dev, payload_capacity,
                                            workspace_dev, err_flag_dev, cs(stream)));
}

tern_status tern_rans_decode(const tern_rans_item* items, int32_t count, int32_t* err_flag_dev, tern_stream_t stream) {
  if (!items || !err_flag_dev || !aligned(err_flag_dev, 4)) return TERN_EINVAL;
  if (count < 1 || count > TERN_PACK_MAX_ITEMS) return TERN_ESHAPE;
  for (int i = 0; i < count; ++i) {
    const tern_rans_item& it = items[i];
    if (!it.freq_dev || !it.row_end_dev || !it.payload_dev || !it.planes_dev) return TERN_EINVAL;
    if (!valid_shape(it.N, it.K)) return TERN_ESHAPE;
    if (!aligned(it.freq_dev, 2) || !aligned(it.row_end_dev, 4) || !aligned(it.planes_dev, 16)) return TERN_EINVAL;
  }
  tern::RansBatch* b = new (std::nothrow) tern::RansBatch();
  if (!b) return TERN_EINVAL;
  b->count = count;
  for (int i = 0; i < count; ++i) {
    b->items[i].freq = items[i].freq_dev;
    b->items[i].row_end = items[i].row_end_dev;
    b->items[i].payload = items[i].payload_dev;
    b->items[i].payload_bytes = items[i].payload_bytes;
    b->items[i].N = items[i].N;
    b->items[i].K = items[i].K;
    b->items[i].planes = items[i].planes_dev;
  }
  tern_status st = TERN_OK;
  if (cudaMemsetAsync(err_flag_dev, 0, sizeof(int32_t), cs(stream)) != cudaSuccess) st = TERN_ECUDA;
  if (st == TERN_OK) st = from_cuda(tern::launch_rans_decode(*b, err_flag_dev, cs(stream)));
  delete b;
  return st;
}

tern_status tern_base3_encode(const int8_t* trits_dev, int32_t N, int32_t K, uint8_t* out_dev,
                              int32_t* err_flag_dev, tern_stream_t stream) {
  if (!trits_dev || !out_dev || !err_flag_dev) return TERN_EINVAL;
  if (!valid_shape(N, K)) return TERN_ESHAPE;
  if (!aligned(err_flag_dev, 4)) return TERN_EINVAL;
  if (cudaMemsetAsync(err_flag_dev, 0, sizeof(int32_t), cs(stream)) != cudaSuccess) return TERN_ECUDA;
  return from_cuda(tern::launch_encode_base3(trits_dev, N, K, out_dev, err_flag_dev, cs(stream)));
}

tern_status tern_occupancy(const tern_matrix* W, int64_t* counts_dev, tern_stream_t stream) {
  if (!W || !W->planes || !counts_dev) return TERN_EINVAL;
  if (!valid_shape(W->N, W->K)) return TERN_ESHAPE;
  if (!aligned(W->planes, 16) || !aligned(counts_dev, 8)) return TERN_EINVAL;
  return from_cuda(tern::launch_occupancy(W->planes, W->N, W->K, counts_dev, cs(stream)));
}

tern_status tern_quantize_act(const uint16_t* x_bf16_dev, int32_t M, int32_t K, int8_t* q_dev, float* s_x_dev,
                              tern_stream_t stream) {
  if (!x_bf16_dev || !q_dev || !s_x_dev) return TERN_EINVAL;
  if (M < 1 || M > 4096 || !valid_shape(1, K)) return TERN_ESHAPE;
  if (!aligned(x_bf16_dev, 16) || !aligned(q_dev, 8) || !aligned(s_x_dev, 4)) return TERN_EINVAL;
  return from_cuda(tern::launch_quantize(x_bf16_dev, M, K, q_dev, s_x_dev, cs(stream)));
}

namespace {

// The single-matrix product behind tern_gemv and tern_gemm_small_m: the persistent stream kernel
// for M = 1 where its plan fits, the cluster split-K kernel otherwise.
tern_status gemm_one(const tern_matrix* W, int32_t M, tern_act act, const void* X_dev, const float* x_scale_dev,
                     float* Y_dev, int32_t* acc_dev, uint32_t flags, tern_stream_t stream) {
  tern_status st = check_matrix(W);
  if (st != TERN_OK) return st;
  if (act != TERN_ACT_BF16 && act != TERN_ACT_INT8) return TERN_EINVAL;
  if (flags & ~TERN_FLAG_PDL) return TERN_EINVAL;
  if (M < 1 || M > 16) return TERN_ESHAPE;
  if (!X_dev || !Y_dev || !aligned(X_dev, 16) || !aligned(Y_dev, 4)) return TERN_EINVAL;
  if (act == TERN_ACT_INT8 && (!x_scale_dev || !aligned(x_scale_dev, 4))) return TERN_EINVAL;
  if (acc_dev && (act != TERN_ACT_INT8 || !aligned(acc_dev, 4))) return TERN_EINVAL;
  if (M == 1) {
    tern::StreamParams sp = {};
    sp.cw = TERN_STREAM_CW;
    size_t smem = 0;
    if (tern::plan_stream(W->N, W->K, act == TERN_ACT_BF16 ? 0 : 1, sp, smem)) {
      sp.planes = W->planes;
      sp.scale = W->scale_f16;
      sp.x = X_dev;
      sp.sx = x_scale_dev;
      sp.y = Y_dev;
      sp.acc = acc_dev;
      return from_cuda(tern::launch_stream(sp, smem, (flags & TERN_FLAG_PDL) != 0, cs(stream)));
    }
  }
  tern::GemmParams p = {};
  p.planes = W->planes;
  p.scale = W->scale_f16;
  p.N = W->N;
  p.K = W->K;
  p.x = X_dev;
  p.sx = x_scale_dev;
  p.y = Y_dev;
  p.acc = acc_dev;
  p.M = M;
  p.mode = act == TERN_ACT_BF16 ? 0 : 1;
  if (!plan_gemm(p.N, p.K, M, p.mode, p.ksplit)) return TERN_ESHAPE;
  p.kr = p.K / p.ksplit;
  return from_cuda(tern::launch_tern_gemm(p, (flags & TERN_FLAG_PDL) != 0, cs(stream)));
}

}  // namespace

tern_status tern_gemm_small_m_ex(const tern_matrix* W, int32_t M, tern_act act, const void* X_dev,
                                 const float* x_scale_dev, float* Y_dev, uint32_t flags, tern_stream_t stream) {
  return gemm_one(W, M, act, X_dev, x_scale_dev, Y_dev, nullptr, flags, stream);
}

tern_status tern_gemm_small_m(const tern_matrix* W, int32_t M, tern_act act, const void* X_dev,
                              const float* x_scale_dev, float* Y_dev, tern_stream_t stream) {
  return gemm_one(W, M, act, X_dev, x_scale_dev, Y_dev, nullptr, 0u, stream);
}

tern_status tern_gemv_ex(const tern_matrix* W, tern_act act, const void* x_dev, const float* x_scale_dev,
                         float* y_dev, int32_t* acc_i32_dev, uint32_t flags, tern_stream_t stream) {
  return gemm_one(W, 1, act, x_dev, x_scale_dev, y_dev, acc_i32_dev, flags, stream);
}

tern_status tern_gemv(const tern_matrix* W, tern_act act, const void* x_dev, const float* x_scale_dev,
                      float* y_dev, int32_t* acc_i32_dev, tern_stream_t stream) {
  return gemm_one(W, 1, act, x_dev, x_scale_dev, y_dev, acc_i32_dev, 0u, stream);
}

namespace {

// Validates a list (and its prologues, if any) and plans both launches. With check_ptrs false
// only the shapes and modes are checked (the workspace query).
// Which small-M kernels run a list: the tensor-core (tcgen05) ones for bf16 lists of 9..16 rows
// (the only kernels there) and wherever the caller asks for them (M >= 2); the mma.sync ones for
// everything else (measured faster wherever both exist).
bool use_tc(int32_t M, tern_act act, uint32_t flags) {
  if (M < 2) return false;
  if (flags & TERN_FLAG_TCGEN05) return true;
  return act == TERN_ACT_BF16 && M >= 9;
}

tern_status fill_batch(const tern_gemv_item* items, const tern_prologue* pro, int32_t count, int32_t M, tern_act act,
                       bool check_ptrs, bool tc, tern::BatchParams& bp, tern::PrepParams& pp, size_t& smem, size_t& ws) {
  if (!items) return TERN_EINVAL;
  if (act != TERN_ACT_BF16 && act != TERN_ACT_INT8) return TERN_EINVAL;
  if (count < 1 || count > TERN_BATCH_MAX_ITEMS || M < 1 || M > 16) return TERN_ESHAPE;
  bp.count = count;
  bp.M = M;
  bp.mode = act == TERN_ACT_BF16 ? 0 : 1;
  bp.tc = tc ? 1 : 0;
  const uint32_t* planes[TERN_BATCH_MAX_ITEMS];
  for (int i = 0; i < count; ++i) {
    const tern_gemv_item& in = items[i];
    const int kind = pro ? pro[i].kind : TERN_PRO_NONE;
    if (kind < TERN_PRO_NONE || kind > TERN_PRO_SWIGLU) return TERN_EINVAL;
    if (check_ptrs) {
      tern_status st = check_matrix(&in.W);
      if (st != TERN_OK) return st;
    } else if (!valid_shape(in.W.N, in.W.K)) {
      return TERN_ESHAPE;
    }
    if (in.W.K > 12288) return TERN_ESHAPE;
    if (check_ptrs) {
      if (!in.y_dev || !aligned(in.y_dev, 4)) return TERN_EINVAL;
      if (kind == TERN_PRO_NONE) {
        if (!in.x_dev || !aligned(in.x_dev, 16)) return TERN_EINVAL;
        if (act == TERN_ACT_INT8 && (!in.x_scale_dev || !aligned(in.x_scale_dev, 4))) return TERN_EINVAL;
      } else {
        const tern_prologue& pr = pro[i];
        if (!pr.src_dev || !aligned(pr.src_dev, 16)) return TERN_EINVAL;
        if (kind == TERN_PRO_RMSNORM && (!pr.gain_dev || !aligned(pr.gain_dev, 16) || !(pr.eps >= 0.0f) ||
                                         pr.eps > 3.0e38f))
          return TERN_EINVAL;
        if (in.x_dev && !aligned(in.x_dev, 16)) return TERN_EINVAL;       // optional copy of the activation
        if (act == TERN_ACT_INT8 && (!in.x_scale_dev || !aligned(in.x_scale_dev, 4))) return TERN_EINVAL;
      }
    }
    tern::BatchItem& it = bp.items[i];
    planes[i] = in.W.planes;
    it.scale = in.W.scale_f16;
    it.y = in.y_dev;
    it.sx = in.x_scale_dev;
    it.N = in.W.N;
    it.K = in.W.K;
    tern::PrepItem& q = pp.items[i];
    q.kind = kind;
    if (kind == TERN_PRO_NONE) {
      q.x = in.x_dev;
      q.gain = nullptr;
      q.xout = nullptr;
      q.sx_out = nullptr;
      q.eps = 0.0f;
    } else {
      q.x = pro[i].src_dev;
      q.gain = pro[i].gain_dev;
      q.xout = const_cast<void*>(in.x_dev);
      q.sx_out = const_cast<float*>(in.x_scale_dev);
      q.eps = pro[i].eps;
    }
  }
  if (!tern::plan_batch(bp, planes, smem, ws)) return TERN_ESHAPE;
  return TERN_OK;
}

tern_status run_batch(const tern_gemv_item* items, const tern_prologue* pro, int32_t count, int32_t M, tern_act act,
                      void* workspace_dev, size_t workspace_bytes, uint32_t flags, tern_stream_t stream) {
  if (flags & ~(TERN_FLAG_PDL | TERN_FLAG_TCGEN05)) return TERN_EINVAL;
  if ((flags & TERN_FLAG_TCGEN05) && M < 2) return TERN_EINVAL;                    // no tcgen05 kernel at M = 1
  if (!workspace_dev || !aligned(workspace_dev, 16)) return TERN_EINVAL;
  tern::BatchParams* bp = new (std::nothrow) tern::BatchParams();
  tern::PrepParams* pp = new (std::nothrow) tern::PrepParams();
  tern_status st = (bp && pp) ? TERN_OK : TERN_EINVAL;
  size_t smem = 0, ws = 0;
  if (st == TERN_OK)
    st = fill_batch(items, pro, count, M, act, true, use_tc(M, act, flags), *bp, *pp, smem, ws);
  if (st == TERN_OK && workspace_bytes < ws) st = TERN_EINVAL;
  if (st == TERN_OK) {
    bp->xprep = static_cast<uint8_t*>(workspace_dev);
    tern::plan_prep(*bp, *pp);
    st = from_cuda(tern::launch_batch(*bp, *pp, smem, (flags & TERN_FLAG_PDL) != 0, cs(stream)));
  }
  delete bp;
  delete pp;
  return st;
}

}  // namespace

size_t tern_gemm_batch_workspace_bytes(const tern_gemv_item* items, int32_t count, int32_t M, tern_act act) {
  tern::BatchParams* bp = new (std::nothrow) tern::BatchParams();
  tern::PrepParams* pp = new (std::nothrow) tern::PrepParams();
  // enough for either kernel family the launch flags can choose
  size_t smem = 0, ws = 0, ws_tc = 0;
  const bool legacy = act != TERN_ACT_BF16 || M <= 8;
  tern_status st = (bp && pp) ? TERN_OK : TERN_EINVAL;
  if (st == TERN_OK && legacy) st = fill_batch(items, nullptr, count, M, act, false, false, *bp, *pp, smem, ws);
  if (st == TERN_OK && M >= 2) {
    *bp = tern::BatchParams();
    st = fill_batch(items, nullptr, count, M, act, false, true, *bp, *pp, smem, ws_tc);
  }
  delete bp;
  delete pp;
  return st == TERN_OK ? (ws > ws_tc ? ws : ws_tc) : 0;
}

size_t tern_gemv_batch_workspace_bytes(const tern_gemv_item* items, int32_t count, tern_act act) {
  return tern_gemm_batch_workspace_bytes(items, count, 1, act);
}

tern_status tern_gemm_batch(const tern_gemv_item* items, int32_t count, int32_t M, tern_act act,
                            void* workspace_dev, size_t workspace_bytes, uint32_t flags, tern_stream_t stream) {
  return run_batch(items, nullptr, count, M, act, workspace_dev, workspace_bytes, flags, stream);
}

tern_status tern_gemm_batch_pro(const tern_gemv_item* items, const tern_prologue* prologues, int32_t count, int32_t M,
                                tern_act act, void* workspace_dev, size_t workspace_bytes, uint32_t flags,
                                tern_stream_t stream) {
  if (!prologues) return TERN_EINVAL;
  return run_batch(items, prologues, count, M, act, workspace_dev, workspace_bytes, flags, stream);
}

tern_status tern_gemv_batch(const tern_gemv_item* items, int32_t count, tern_act act, void* workspace_dev,
                            size_t workspace_bytes, uint32_t flags, tern_stream_t stream) {
  return tern_gemm_batch(items, count, 1, act, workspace_dev, workspace_bytes, flags, stream);
}

tern_status tern_act_prologue(const tern_prologue* pro, int32_t M, int32_t K, uint16_t* x_bf16_dev,
                              tern_stream_t stream) {
  if (!pro || !pro->src_dev || !x_bf16_dev) return TERN_EINVAL;
  if (pro->kind < TERN_PRO_BF16 || pro->kind > TERN_PRO_SWIGLU) return TERN_EINVAL;
  if (M < 1 || M > 65536 || !valid_shape(1, K)) return TERN_ESHAPE;
  if (!aligned(pro->src_dev, 16) || !aligned(x_bf16_dev, 16)) return TERN_EINVAL;
  if (pro->kind == TERN_PRO_RMSNORM &&
      (!pro->gain_dev || !aligned(pro->gain_dev, 16) || !(pro->eps >= 0.0f) || pro->eps > 3.0e38f))
    return TERN_EINVAL;
  return from_cuda(tern::launch_prologue(pro->kind, pro->src_dev, pro->gain_dev, pro->eps, M, K, x_bf16_dev,
                                         cs(stream)));
}

size_t i8_head_workspace_bytes(int32_t V, int32_t M) {
  if (V <= 0 || M < 1 || M > 16) return 0;
  return tern::head_workspace_bytes(M);
}

tern_status i8_head_gemv_argmax_ex(const int8_t* W_dev, const uint16_t* scale_f16_dev, int32_t V, int32_t K,
                                   int32_t M, tern_act act, const void* X_dev, const float* x_scale_dev,
                                   int32_t* argmax_dev, float* maxval_dev, float* logits_dev,
                                   void* workspace_dev, size_t workspace_bytes, uint32_t flags,
                                   tern_stream_t stream) {
  tern::HeadParams p = {};
  const tern_status st = tern::plan_head_call(W_dev, scale_f16_dev, V, K, M, act, X_dev, x_scale_dev, argmax_dev,
                                              maxval_dev, logits_dev, workspace_dev, workspace_bytes, flags, p,
                                              nullptr);
  if (st != TERN_OK) return st;
  return from_cuda(tern::launch_head(p, (flags & TERN_FLAG_PDL) != 0, cs(stream)));
}

tern_status i8_head_verify(const int8_t* W_dev, const uint16_t* scale_f16_dev, int32_t V, int32_t K, int32_t M,
                           tern_act act, const void* X_dev, const float* x_scale_dev, const int32_t* draft_dev,
                           int32_t* argmax_dev, float* maxval_dev, int32_t* accept_dev, void* workspace_dev,
                           size_t workspace_bytes, tern_stream_t stream) {
  if (!accept_dev || !aligned(accept_dev, 4)) return TERN_EINVAL;
  if (M > 1 && (!draft_dev || !aligned(draft_dev, 4))) return TERN_EINVAL;
  tern::HeadParams p = {};
  const tern_status st = tern::plan_head_call(W_dev, scale_f16_dev, V, K, M, act, X_dev, x_scale_dev, argmax_dev,
                                              maxval_dev, nullptr, workspace_dev, workspace_bytes, 0u, p, nullptr);
  if (st != TERN_OK) return st;
  p.draft = draft_dev;
  p.accept = accept_dev;
  return from_cuda(tern::launch_head(p, false, cs(stream)));
}

tern_status tern_verify_accept(const int32_t* argmax_dev, const int32_t* draft_dev, int32_t k, int32_t* accept_dev,
                               tern_stream_t stream) {
  if (!argmax_dev || !accept_dev || (k > 0 && !draft_dev)) return TERN_EINVAL;
  if (!aligned(argmax_dev, 4) || !aligned(accept_dev, 4) || (draft_dev && !aligned(draft_dev, 4))) return TERN_EINVAL;
  if (k < 0 || k > 65535) return TERN_ESHAPE;
  return from_cuda(tern::launch_verify_accept(argmax_dev, draft_dev, k, accept_dev, cs(stream)));
}

tern_status i8_head_gemv_argmax(const int8_t* W_dev, const uint16_t* scale_f16_dev, int32_t V, int32_t K, int32_t M,
                                tern_act act, const void* X_dev, const float* x_scale_dev, int32_t* argmax_dev,
                                float* maxval_dev, float* logits_dev, void* workspace_dev, size_t workspace_bytes,
                                tern_stream_t stream) {
  return i8_head_gemv_argmax_ex(W_dev, scale_f16_dev, V, K, M, act, X_dev, x_scale_dev, argmax_dev, maxval_dev,
                                logits_dev, workspace_dev, workspace_bytes, 0u, stream);
}

size_t tern_fv5_packed_bytes(int32_t N, int32_t K) {
  return (N > 0 && K > 0 && K % 512 == 0) ? (size_t)N * (size_t)K * 3 / 8 : 0;
}

tern_status tern_fv5_pack(const int8_t* codes_dev, int32_t N, int32_t K, uint32_t* planes_dev, int32_t* err_flag_dev,
                          tern_stream_t stream) {
  if (!codes_dev || !planes_dev || !err_flag_dev) return TERN_EINVAL;
  if (N <= 0 || K <= 0 || K % 512) return TERN_ESHAPE;
  if (!aligned(codes_dev, 16) || !aligned(planes_dev, 16) || !aligned(err_flag_dev, 4)) return TERN_EINVAL;
  if (cudaMemsetAsync(err_flag_dev, 0, sizeof(int32_t), cs(stream)) != cudaSuccess) return TERN_ECUDA;
  return from_cuda(tern::launch_fv5_pack(codes_dev, N, K, planes_dev, err_flag_dev, cs(stream)));
}

tern_status tern_fv5_gemm(const tern_fv5_matrix* W, int32_t M, tern_act act, const void* X_dev, const float* x_scale_dev,
                          float* Y_dev, tern_stream_t stream) {
  if (!W || !W->planes || !W->scales) return TERN_EINVAL;
  if (W->N <= 0 || W->K <= 0 || W->K % 512) return TERN_ESHAPE;
  if (act != TERN_ACT_BF16 && act != TERN_ACT_INT8) return TERN_EINVAL;
  if (M < 1 || M > (act == TERN_ACT_BF16 ? 8 : 16)) return TERN_ESHAPE;
  if (!aligned(W->planes, 16) || !aligned(W->scales, 8)) return TERN_EINVAL;
  if (!X_dev || !Y_dev || !aligned(X_dev, 16) || !aligned(Y_dev, 4)) return TERN_EINVAL;
  if (act == TERN_ACT_INT8 && (!x_scale_dev || !aligned(x_scale_dev, 4))) return TERN_EINVAL;
  tern::Fv5Params p = {};
  p.planes = W->planes;
  p.scales = W->scales;
  p.N = W->N;
  p.K = W->K;
  p.x = X_dev;
  p.sx = x_scale_dev;
  p.y = Y_dev;
  p.M = M;
  p.mode = act == TERN_ACT_BF16 ? 0 : 1;
  // split K over a cluster of up to 8 CTAs (whole 512-trit groups per slice) to cover the SMs
  const int row_blocks = (p.N + tern::fv5_rows_per_cta() - 1) / tern::fv5_rows_per_cta();
  const int units = p.K / 512;
  const int sms = tern::device_sm_count();
  int ks = 1;
  while (ks < 8 && row_blocks * ks < 2 * sms && units % (2 * ks) == 0) ks *= 2;
  while (tern::fv5_smem_bytes(p.mode, M, p.K / ks) > kGemmSmemCap && ks < 8 && units % (2 * ks) == 0) ks *= 2;
  if (tern::fv5_smem_bytes(p.mode, M, p.K / ks) > kGemmSmemCap) return TERN_ESHAPE;
  p.ksplit = ks;
  p.kr = p.K / ks;
  return from_cuda(tern::launch_fv5_gemm(p, cs(stream)));
}

tern_status tern_fv5_gemv_batch(const tern_fv5_batch_item* items, int32_t count, tern_act act, tern_stream_t stream) {
  if (!items) return TERN_EINVAL;
  if (act != TERN_ACT_BF16 && act != TERN_ACT_INT8) return TERN_EINVAL;
  if (count < 1 || count > TERN_FV5_BATCH_MAX_ITEMS || count > tern::kBatchMaxItems) return TERN_ESHAPE;
  tern::Fv5BatchParams* p = new (std::nothrow) tern::Fv5BatchParams();
  if (!p) return TERN_EINVAL;
  tern_status st = TERN_OK;
  for (int i = 0; i < count && st == TERN_OK; ++i) {
    const tern_fv5_batch_item& in = items[i];
    if (!in.W.planes || !in.W.scales || !in.x_dev || !in.y_dev) st = TERN_EINVAL;
    else if (in.W.N <= 0 || in.W.K <= 0 || in.W.K % 512 || in.W.K > 12288) st = TERN_ESHAPE;
    else if (!aligned(in.W.planes, 16) || !aligned(in.W.scales, 8) || !aligned(in.x_dev, 16) || !aligned(in.y_dev, 4))
      st = TERN_EINVAL;
    else if (act == TERN_ACT_INT8 && (!in.x_scale_dev || !aligned(in.x_scale_dev, 4))) st = TERN_EINVAL;
    else {
      tern::Fv5BatchItem& it = p->items[i];
      it.planes = in.W.planes;
      it.scales = in.W.scales;
      it.x = in.x_dev;
      it.sx = act == TERN_ACT_INT8 ? in.x_scale_dev : nullptr;
      it.y = in.y_dev;
      it.N = in.W.N;
      it.K = in.W.K;
    }
  }
  if (st == TERN_OK) {
    p->count = count;
    p->mode = act == TERN_ACT_BF16 ? 0 : 1;
    st = from_cuda(tern::launch_fv5_batch(*p, cs(stream)));
  }
  delete p;
  return st;
}

tern_status fv5b_head_gemv_argmax(const int8_t* W_dev, const float* block_scale_dev, int32_t V, int32_t K, int32_t M,
                                  tern_act act, const void* X_dev, const float* x_scale_dev, int32_t* argmax_dev,
                                  float* maxval_dev, float* logits_dev, void* workspace_dev, size_t workspace_bytes,
                                  tern_stream_t stream) {
  if (!block_scale_dev) return TERN_EINVAL;
  tern::HeadParams p = {};
  const tern_status st = tern::plan_head_call(W_dev, nullptr, V, K, M, act, X_dev, x_scale_dev, argmax_dev, maxval_dev,
                                              logits_dev, workspace_dev, workspace_bytes, 0u, p, block_scale_dev);
  if (st != TERN_OK) return st;
  return from_cuda(tern::launch_head(p, false, cs(stream)));
}

namespace {

// Workspace layout of a chain: [items (64-byte aligned)][done counters][finished] (no scratch).
struct ChainWs {
  size_t items, done, finished, scratch, total;
};
ChainWs chain_ws(int count, size_t scratch_words) {
  ChainWs w;
  w.items = 0;
  w.done = ((size_t)count * sizeof(tern::ChainItem) + 63) & ~(size_t)63;
  w.finished = w.done + (((size_t)count * 4 + 63) & ~(size_t)63);
  w.scratch = w.finished + 64;
  w.total = w.scratch + scratch_words * 4;
  return w;
}

// Checks and converts the items (check_ptrs false: shapes and sources only).
tern_status chain_items(const tern_chain_item* items, int32_t count, tern_act act, bool check_ptrs, tern::ChainItem* out,
                        const uint32_t** planes) {
  if (!items) return TERN_EINVAL;
  if (act != TERN_ACT_BF16 && act != TERN_ACT_INT8) return TERN_EINVAL;
  if (count < 1 || count > TERN_CHAIN_MAX_ITEMS) return TERN_ESHAPE;
  for (int i = 0; i < count; ++i) {
    const tern_chain_item& in = items[i];
    if (check_ptrs) {
      tern_status st = check_matrix(&in.W);
      if (st != TERN_OK) return st;
    } else if (!valid_shape(in.W.N, in.W.K)) {
      return TERN_ESHAPE;
    }
    if (in.W.K > 12288) return TERN_ESHAPE;
    if (in.kind != TERN_PRO_BF16 && in.kind != TERN_PRO_CAST && in.kind != TERN_PRO_RMSNORM) return TERN_EINVAL;
    if (in.src_item >= i || in.src_item < -1) return TERN_EINVAL;
    if (in.swiglu_out && in.W.N % 16) return TERN_ESHAPE;
    if (in.src_item >= 0) {
      const tern_chain_item& d = items[in.src_item];
      if (in.src_h) {
        if (!d.swiglu_out || in.kind != TERN_PRO_BF16) return TERN_EINVAL;
        if (d.W.N / 2 < in.W.K) return TERN_ESHAPE;
      } else {
        if (in.kind == TERN_PRO_BF16) return TERN_EINVAL;          // a y source is fp32
        if (d.W.N < in.W.K) return TERN_ESHAPE;
      }
    }
    if (check_ptrs) {
      if (in.src_item < 0 && (!in.src_dev || !aligned(in.src_dev, 16))) return TERN_EINVAL;
      if (in.kind == TERN_PRO_RMSNORM &&
          (!in.gain_dev || !aligned(in.gain_dev, 16) || !(in.eps >= 0.0f) || in.eps > 3.0e38f))
        return TERN_EINVAL;
      if (!in.y_dev || !aligned(in.y_dev, 16)) return TERN_EINVAL;
      if (in.swiglu_out && (!in.h_dev || !aligned(in.h_dev, 16))) return TERN_EINVAL;
      if (in.x_scale_dev && !aligned(in.x_scale_dev, 4)) return TERN_EINVAL;
    }
    if (out) {
      tern::ChainItem& c = out[i];
      c = tern::ChainItem{};
      planes[i] = in.W.planes;
      c.scale = in.W.scale_f16;
      c.y = in.y_dev;
      c.hout = in.swiglu_out ? in.h_dev : nullptr;
      c.sx_out = act == TERN_ACT_INT8 ? in.x_scale_dev : nullptr;
      c.src = in.src_item < 0 ? in.src_dev
                              : (in.src_h ? static_cast<const void*>(items[in.src_item].h_dev)
                                          : static_cast<const void*>(items[in.src_item].y_dev));
      c.gain = in.gain_dev;
      c.eps = in.eps;
      c.kind = in.kind;
      c.dep = in.src_item;
      c.N = in.W.N;
      c.K = in.W.K;
    }
  }
  return TERN_OK;
}

}  // namespace

size_t tern_chain_workspace_bytes(const tern_chain_item* items, int32_t count, tern_act act) {
  if (chain_items(items, count, act, false, nullptr, nullptr) != TERN_OK) return 0;
  return chain_ws(count, 0).total;                              // every output is one CTA's: no scratch
}

tern_status tern_chain_plan(const tern_chain_item* items, int32_t count, tern_act act, void* workspace_dev,
                            size_t workspace_bytes, tern_chain* chain) {
  if (!chain || !workspace_dev || !aligned(workspace_dev, 64)) return TERN_EINVAL;
  tern::ChainItem* host = new (std::nothrow) tern::ChainItem[count > 0 && count <= TERN_CHAIN_MAX_ITEMS ? count : 1];
  const uint32_t** planes = new (std::nothrow) const uint32_t*[count > 0 && count <= TERN_CHAIN_MAX_ITEMS ? count : 1];
  tern_status st = (host && planes) ? chain_items(items, count, act, true, host, planes) : TERN_EINVAL;
  tern::ChainLayout L = {};
  const int grid = tern::chain_grid();
  if (st == TERN_OK && !tern::plan_chain(host, count, act == TERN_ACT_BF16 ? 0 : 1, grid, planes, L)) st = TERN_ESHAPE;
  ChainWs w = chain_ws(count > 0 ? count : 1, L.scratch_words);
  if (st == TERN_OK && workspace_bytes < w.total) st = TERN_EINVAL;
  if (st == TERN_OK) {
    uint8_t* ws = static_cast<uint8_t*>(workspace_dev);
    if (cudaMemcpy(ws + w.items, host, (size_t)count * sizeof(tern::ChainItem), cudaMemcpyHostToDevice) != cudaSuccess ||
        cudaMemset(ws + w.done, 0, w.total - w.done) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess)
      st = TERN_ECUDA;
  }
  if (st == TERN_OK) {
    chain->workspace_dev = workspace_dev;
    chain->count = count;
    chain->mode = act == TERN_ACT_BF16 ? 0 : 1;
    chain->grid = grid;
    chain->stages = L.stages;
    chain->seg_parts = L.seg_parts;
    chain->smem_bytes = L.smem;
  }
  delete[] host;
  delete[] planes;
  return st;
}

tern_status tern_chain_run(const tern_chain* chain, tern_stream_t stream) {
  if (!chain || !chain->workspace_dev || chain->count < 1 || chain->grid < 1 || chain->stages < 2 ||
      chain->seg_parts < 1)
    return TERN_EINVAL;
  const ChainWs w = chain_ws(chain->count, 0);
  uint8_t* ws = static_cast<uint8_t*>(chain->workspace_dev);
  tern::ChainParams p = {};
  p.items = reinterpret_cast<const tern::ChainItem*>(ws + w.items);
  p.count = chain->count;
  p.mode = chain->mode;
  p.grid = chain->grid;
  p.stages = chain->stages;
  p.seg_parts = chain->seg_parts;
  p.done = reinterpret_cast<int32_t*>(ws + w.done);
  p.finished = reinterpret_cast<int32_t*>(ws + w.finished);
  p.scratch = reinterpret_cast<int32_t*>(ws + w.scratch);
  return from_cuda(tern::launch_chain(p, chain->smem_bytes, cs(stream)));
}

tern_status tern_read_flag(const int32_t* err_flag_dev, tern_stream_t stream) {
  if (!err_flag_dev) return TERN_EINVAL;
  if (cudaStreamSynchronize(cs(stream)) != cudaSuccess) return TERN_ECUDA;
  int32_t v = 0;
  if (cudaMemcpy(&v, err_flag_dev, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return TERN_ECUDA;
  return v == 0 ? TERN_OK : TERN_EBADCODE;
}

tern_status tern_device_status(tern_stream_t stream) {
  int v = 0, w = 0, x = 0, c = 0, t = 0, f = 0;
  if (tern::read_and_clear_error_latch(&v, cs(stream)) != cudaSuccess) return TERN_ECUDA;
  if (tern::read_and_clear_batch_latch(&w) != cudaSuccess) return TERN_ECUDA;
  if (tern::read_and_clear_prefill_latch(&x) != cudaSuccess) return TERN_ECUDA;
  if (tern::read_and_clear_chain_latch(&c) != cudaSuccess) return TERN_ECUDA;
  if (tern::read_and_clear_tc_latch(&t) != cudaSuccess) return TERN_ECUDA;
  if (tern::read_and_clear_fv5_latch(&f) != cudaSuccess) return TERN_ECUDA;
  return (v == 0 && w == 0 && x == 0 && c == 0 && t == 0 && f == 0) ? TERN_OK : TERN_ETIMEOUT;
}

tern_status tern_gemm_prefill(const tern_matrix* W, int32_t M, const uint16_t* X_bf16_dev, float* Y_dev,
                              tern_stream_t stream) {
  tern_status st = check_matrix(W);
  if (st != TERN_OK) return st;
  if (!X_bf16_dev || !Y_dev || !aligned(X_bf16_dev, 16) || !aligned(Y_dev, 4)) return TERN_EINVAL;
  if (M < 1 || M > 65536) return TERN_ESHAPE;
  tern::PrefillParams p = {};
  p.planes = W->planes;
  p.scale = W->scale_f16;
  p.Y = Y_dev;
  p.M = M;
  p.N = W->N;
  p.K = W->K;
  p.vec_store = (W->N % 4 == 0 && aligned(Y_dev, 16)) ? 1 : 0;
  int grid = 0;
  size_t smem = 0;
  if (!tern::plan_prefill(p, X_bf16_dev, grid, smem)) return TERN_ESHAPE;
  return from_cuda(tern::launch_prefill(p, grid, smem, cs(stream)));
}

}  // extern "C"
