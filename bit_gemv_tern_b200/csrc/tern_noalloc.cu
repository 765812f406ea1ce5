// No-allocation entry point of the int8 output head: i8_head_gemv_argmax_noalloc (include/tern.h).
//
// i8_head_gemv_argmax takes its scratch (the finished-CTA counter and one packed (value, index)
// maximum per activation row) from the caller. This entry point uses one library-internal device
// array instead, so a caller needs no device buffer beyond the inputs and outputs. The array is
// file-scope and sized for the largest M the head accepts (16 activation rows). Its address is
// looked up once per device with cudaGetSymbolAddress, with that device current. Each call checks
// every argument and plans the launch first (an invalid call enqueues nothing), then clears the
// bytes it uses with cudaMemsetAsync on its own stream and launches the head with that scratch. No
// call allocates or frees device memory. Every call on a device shares the one array, so calls
// that overlap in time race.
#include <cstdint>
#include <mutex>
#include <cuda_runtime.h>

#include "../../include/tern.h"
#include "tern_kernels.h"

namespace {

// 16 bytes of counter + 8 bytes per activation row, M <= 16: 144 bytes used.
constexpr size_t kScratchBytes = TERN_HEAD_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_head_scratch[kScratchBytes];

std::mutex g_mu;
void* g_addr[kMaxDevices] = {};

// Device address of g_head_scratch on the current device (looked up on the first call there).
tern_status scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return TERN_ECUDA;
  if (dev < 0 || dev >= kMaxDevices) return TERN_EINVAL;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_head_scratch) != cudaSuccess || !p) return TERN_ECUDA;
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return TERN_OK;
}

}  // namespace

tern_status i8_head_gemv_argmax_noalloc(const int8_t* W_dev, const uint16_t* scale_f16_dev, int32_t V, int32_t K,
                                        int32_t M, tern_act act, const void* X_dev, const float* x_scale_dev,
                                        int32_t* argmax_dev, float* maxval_dev, float* logits_dev,
                                        tern_stream_t stream) {
  if (M < 1 || M > TERN_HEAD_NOALLOC_MAX_M) return TERN_ESHAPE;
  const size_t need = i8_head_workspace_bytes(V, M);
  if (need == 0 || need > kScratchBytes) return TERN_ESHAPE;
  void* ws = nullptr;
  tern_status st = scratch_address(&ws);
  if (st != TERN_OK) return st;
  tern::HeadParams p = {};
  st = tern::plan_head_call(W_dev, scale_f16_dev, V, K, M, act, X_dev, x_scale_dev, argmax_dev, maxval_dev,
                            logits_dev, ws, kScratchBytes, 0u, p, nullptr);
  if (st != TERN_OK) return st;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(ws, 0, need, s) != cudaSuccess) return TERN_ECUDA;
  return tern::launch_head(p, false, s) == cudaSuccess ? TERN_OK : TERN_ECUDA;
}
