/*
 * tern.h -- C ABI of libterngemv.so: packed-ternary linear layers and the int8 output head on
 * NVIDIA B200 (sm_100a).
 *
 * Sources, cited by page and section heading:
 *   [R] PyTorchKR review "Fermion Research, 3진 계열 포맷으로 직접 학습한 Neutrino-1 모델군 3종 공개"
 *       (discuss.pytorch.kr/t/11456);
 *   [A] aiatolah.com, "Neutrino-1 8B: modelo ternario de 3,88 GB roda em GPU e laptop";
 *   [O] origotech.dev, "더 적은 비트로 계산하기" (lowbit explainer).
 *
 * What the library computes
 *   A linear layer's output feature is a sum of weight x activation terms, y_j = sum_i w_ij x_i
 *   ([R] "학습 중에 포맷이 있어야 하는 이유", displayed equation). Here w_ij = scale_j * t_ij with a
 *   trit t in {-1, 0, +1}, so each term is an add, a skip or a subtract ([O] Figure I). Weights stay
 *   packed at rest and are decoded inside the matrix kernels; no fp16/fp32 weight copy is ever
 *   made ([A] second paragraph and "Formato unico, tres portas"). The transport form of the
 *   ternary lane expands bit-exactly into the packed container ([R] "3진 계열이라는 이름의 실체";
 *   [A] "Formato unico"); embeddings and the output head stay int8 ([R] same section).
 *
 * Conventions (every entry point)
 *   - Every pointer named *_dev is device memory owned by the caller; the library keeps no
 *     reference after the call returns and allocates no device memory.
 *   - Work is enqueued asynchronously on `stream` (NULL = the legacy default stream); nothing
 *     synchronises except tern_read_flag and tern_device_status.
 *   - Argument errors are returned before anything is enqueued. A launch error is returned as
 *     TERN_ECUDA (the CUDA error is left to cudaGetLastError-style inspection by the caller).
 *   - Data errors that only the device can see (a trit outside {-1,0,+1}, a transport byte above
 *     242) set *err_flag_dev to a nonzero value; read it with tern_read_flag. Kernels never trap and
 *     never wait without a bound.
 *   - Outputs are deterministic: the same inputs give the same bits on every run.
 *   - Precision of the bf16 mode: products with the ternary (or int8) weights are exact and sums
 *     are exact integers; the only roundings are the activation encoding (a group of activations
 *     with absmax below 2^E is held on a grid of 2^(E - 30), so an activation moves by at most
 *     2^(E - 31)) and the final conversion to fp32. Every output y of a K-term product is
 *     therefore within scale * K * 2^-30 * sum_k |x_k| (+ half an fp32 ulp of y) of the exact
 *     value, whatever the inputs' dynamic range; for K <= 12288 that is under 1.2e-5 * scale *
 *     sum_k |x_k|. tern_gemm_prefill instead accumulates exact bf16 products in fp32 on the
 *     tensor cores.
 *   - Global state, all of it: one device word per kernel family that latches TERN_ETIMEOUT when
 *     a bounded wait gives up (shared by every stream and caller on a device; tern_device_status
 *     reads and clears them), the scratch array of i8_head_gemv_argmax_noalloc, and host-side
 *     records, per device, of the kernel attributes already set and of that array's address.
 *
 * Deliberate differences from the entry points sketched for this library's boundary
 *   - tern_pack takes no scale argument: the per-row fp16 scales stay a separate caller array
 *     that a tern_matrix points to; packing would only copy it.
 *   - The launch flags of the *_ex entry points, the batched entry points (tern_pack_batch,
 *     tern_gemv_batch, tern_gemm_batch), tern_base3_encode, the rANS transport (tern_rans_*),
 *     tern_occupancy, tern_quantize_act,
 *     the prologues (tern_gemm_batch_pro, tern_act_prologue), the verify round (i8_head_verify,
 *     tern_verify_accept), the five-valued blocks (tern_fv5_*, fv5b_head_gemv_argmax), the dependent chain
 *     (tern_chain_*) and i8_head_gemv_argmax_noalloc are additions.
 *
 * Packed layout (this library's own; the pages' FV5 bit-planes are only partly described)
 *   Matrix N x K, K a multiple of 128. Row n occupies K/16 uint32 words at word offset n*K/16:
 *     words [0, K/32)     nonzero-mask plane, bit = (t != 0)
 *     words [K/32, K/16)  sign plane,         bit = (t == -1)   (0 wherever the mask bit is 0)
 *   Trit k of the row sits in word k/32 of each plane. With j = k % 32:
 *     mask bit position  p(j) = 16*(j % 2) + (j / 16) + 2*((j % 16) / 2)
 *     sign bit position  (p(j) + 1) % 32
 *   i.e. the sign plane is the mask plane's bit order rotated by one. This order lets a kernel
 *   merge one mask word and one sign word into two words of sixteen 2-bit two's-complement
 *   fields (m in the low bit, s in the high bit) and read a field placed in the top two bits of
 *   a byte as the int8 value 64*t, or in the top two bits of a half-word as the bf16 value
 *   2.0*t, with one shift and one AND. Per-row scales are a separate fp16[N] array.
 *   Packed size: N*K/4 bytes of planes + 2*N bytes of scales.
 *
 * Transport layout (base 3, fixed rate)
 *   Row n occupies ceil(K/5) bytes at byte offset n*ceil(K/5). Byte j of a row holds trits
 *   5j..5j+4 as b = d0 + 3*d1 + 9*d2 + 27*d3 + 81*d4 with d_i = t_(5j+i) + 1. Trits past the end of
 *   the row are written as t = 0 (d = 1) and ignored on reading; bytes 243..255 are invalid.
 */
#ifndef TERN_H_
#define TERN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Everything declared below is exported from libterngemv.so, which is otherwise built with
 * hidden symbol visibility. */
#if defined(__GNUC__)
#pragma GCC visibility push(default)
#endif

/* Same object as cudaStream_t; declared here so that this header needs no CUDA header. */
typedef struct CUstream_st* tern_stream_t;

typedef enum {
  TERN_OK = 0,
  TERN_EINVAL = 1,    /* null pointer, unknown enum value, misaligned pointer, bad flags      */
  TERN_ESHAPE = 2,    /* N <= 0, K <= 0, K % 128 != 0, M out of range, size overflow          */
  TERN_EBADCODE = 3,  /* device saw an invalid trit / transport byte (via the error flag)     */
  TERN_ECUDA = 4,     /* a CUDA runtime call or kernel launch failed                          */
  TERN_ETIMEOUT = 5   /* a bounded device-side wait gave up (see tern_device_status)          */
} tern_status;

typedef enum { TERN_ACT_BF16 = 0, TERN_ACT_INT8 = 1 } tern_act;
typedef enum { TERN_SRC_INT8_TRITS = 0, TERN_SRC_BASE3 = 1 } tern_src;

/* Launch flags for the *_ex entry points.
 * TERN_FLAG_PDL: launch with programmatic dependent launch. The kernel may start while the
 *   previous kernel on the stream is still running; it reads weights before waiting for that
 *   kernel, and reads activations / writes outputs only after. Only valid when the weight
 *   buffers are not written by work still in flight on the stream (true in a decode loop). */
#define TERN_FLAG_PDL 1u
/* TERN_FLAG_TCGEN05 (tern_gemm_batch / tern_gemm_batch_pro only, M >= 2): run the list on the
 *   tensor-core (tcgen05) small-M kernels, which otherwise take only bf16 lists of 9..16 rows (the
 *   warp-level mma.sync kernels, bit-identical, run everything else and are faster wherever both
 *   exist). For comparisons. */
#define TERN_FLAG_TCGEN05 2u

/* A packed ternary matrix: views of caller-owned device memory. */
typedef struct {
  int32_t N;                  /* rows (output features), > 0                                */
  int32_t K;                  /* columns (input features), > 0, multiple of 128             */
  const uint32_t* planes;     /* device, N*K/16 words in the packed layout, 16-byte aligned */
  const uint16_t* scale_f16;  /* device, N fp16 bit patterns (per-row scale)                */
} tern_matrix;

/* Human-readable name of a status code (static string). */
const char* tern_status_string(tern_status s);

/* Bytes of packed planes for an N x K matrix (N*K/4); 0 if the shape is invalid. */
size_t tern_packed_bytes(int32_t N, int32_t K);

/* Bytes of the base-3 transport for an N x K matrix (N*ceil(K/5)); 0 if the shape is invalid. */
size_t tern_base3_bytes(int32_t N, int32_t K);

/* Pack a ternary matrix into the planes layout (the loader step: weights packed at rest, [A]).
 *   src = TERN_SRC_INT8_TRITS: src_dev is int8[N][K] row-major with values in {-1, 0, +1}.
 *   src = TERN_SRC_BASE3:      src_dev is the transport, uint8[N][ceil(K/5)] (layout above), 4-byte
 *                              aligned; it is expanded bit-exactly ([R] "3진 계열이라는 이름의 실체").
 *   planes_dev: output, N*K/16 uint32 words, 16-byte aligned.
 *   err_flag_dev: int32 on the device; cleared by this call on the stream, then set nonzero if
 *   any input value is invalid (the planes are then unspecified). Required. */
tern_status tern_pack(tern_src src, const void* src_dev, int32_t N, int32_t K, uint32_t* planes_dev,
                      int32_t* err_flag_dev, tern_stream_t stream);

/* One tensor of a tern_pack_batch call: views of caller-owned device memory. */
typedef struct {
  const void* src_dev;        /* as tern_pack's src_dev for the call's src kind        */
  int32_t N, K;               /* shape, as for tern_pack                               */
  uint32_t* planes_dev;       /* output planes, N*K/16 words, 16-byte aligned          */
} tern_pack_item;

#define TERN_PACK_MAX_ITEMS 256

/* tern_pack over a list of tensors (a whole model's transport at load time): one clear of
 * err_flag_dev, then one launch for all items (for either source kind). Results are
 * bit-identical to tern_pack per item; the flag is set if
 * any item holds an invalid value. items: host array of 1..TERN_PACK_MAX_ITEMS descriptors,
 * read during the call only. No output may overlap another item's input or output. */
tern_status tern_pack_batch(tern_src src, const tern_pack_item* items, int32_t count, int32_t* err_flag_dev,
                            tern_stream_t stream);

/* Encode dense trits int8[N][K] into the base-3 transport uint8[N][ceil(K/5)] (the inverse of
 * tern_pack with TERN_SRC_BASE3). err_flag_dev as for tern_pack. */
tern_status tern_base3_encode(const int8_t* trits_dev, int32_t N, int32_t K, uint8_t* out_dev,
                              int32_t* err_flag_dev, tern_stream_t stream);

/* Order-0 entropy-coded transport of a ternary tensor (rANS). The pages code the transport close
 * to its order-0 coding bound ([R] "3진 계열이라는 이름의 실체": within 0.007% of it for the 0.6B)
 * without naming the coder; this library's coder is byte-wise range asymmetric numeral systems
 * (J. Duda, 2013), one static 12-bit frequency table per tensor and one stream per row:
 *   - symbols s = 0 (t = 0), 1 (t = +1), 2 (t = -1); freq[s] >= 1, freq[0] + freq[1] + freq[2] =
 *     4096; cum = (0, freq[0], freq[0] + freq[1]); the table of a tensor is
 *     f_s = max(1, floor(4096 c_s / (N*K))) of its trit counts c_s, with 4096 - sum f added to the
 *     most frequent symbol (the lowest s on ties);
 *   - a row is encoded from its last trit to its first, from x = 2^23: while x >= 2^19 freq[s],
 *     the low byte of x is emitted and shifted out; x = (x / freq[s]) * 4096 + x % freq[s] +
 *     cum[s]; then the final x, low byte first. The row's stream is every emitted byte in reverse
 *     order (it starts with the final state, most significant byte first);
 *   - row n's stream occupies payload bytes [row_end[n-1], row_end[n]) (row_end[-1] = 0).
 * Size: the order-0 entropy of the tensor plus 24..32 bits per row (about 1.334 bits per trit at
 * the 8B geometry's distribution, against 1.6 for the base-3 transport). */
typedef struct {
  const uint16_t* freq_dev;     /* device, 3 frequencies                                        */
  const uint32_t* row_end_dev;  /* device, N end offsets                                        */
  const uint8_t* payload_dev;   /* device, the streams                                          */
  size_t payload_bytes;         /* size of the payload buffer: no read goes past it            */
  int32_t N, K;                 /* shape, K % 128 == 0                                          */
  uint32_t* planes_dev;         /* output planes, N*K/16 words, 16-byte aligned                 */
} tern_rans_item;

/* Payload bytes to provide to tern_rans_encode (an upper bound of any tensor's stream). */
size_t tern_rans_payload_bound(int32_t N, int32_t K);
/* Scratch bytes tern_rans_encode needs. */
size_t tern_rans_workspace_bytes(int32_t N, int32_t K);

/* Encodes int8 trits [N][K] (16-byte aligned) into the transport: freq_dev (3 x uint16),
 * row_end_dev (N x uint32) and payload_dev (payload_capacity bytes, at least
 * tern_rans_payload_bound; the stream's size is row_end[N-1]). err_flag_dev is cleared, then set if
 * a value is not a trit or the payload does not fit (outputs then unspecified). workspace_dev:
 * tern_rans_workspace_bytes(N, K) bytes, 16-byte aligned, contents need no initialisation. */
tern_status tern_rans_encode(const int8_t* trits_dev, int32_t N, int32_t K, uint16_t* freq_dev, uint32_t* row_end_dev,
                             uint8_t* payload_dev, size_t payload_capacity, void* workspace_dev, size_t workspace_bytes,
                             int32_t* err_flag_dev, tern_stream_t stream);

/* Decodes a list of transports (1..TERN_PACK_MAX_ITEMS, e.g. a whole model at load time) into
 * their packed planes in one launch, bit-exactly (the planes equal tern_pack of the same trits).
 * err_flag_dev is cleared, then set if any row is not a valid stream (frequencies not summing to
 * 4096, a row range outside the payload, a row that does not end in the initial state with all of
 * its bytes read); that row's planes are then unspecified. No read leaves a row's byte range. */
tern_status tern_rans_decode(const tern_rans_item* items, int32_t count, int32_t* err_flag_dev, tern_stream_t stream);

/* Per-row occupancy of a packed matrix ([R] "출하된 컨테이너를 직접 읽기": zero / +1 / -1
 * fractions of each tensor). counts_dev: int64[N][3] = {zeros, plus_ones, minus_ones}. */
tern_status tern_occupancy(const tern_matrix* W, int64_t* counts_dev, tern_stream_t stream);

/* Per-token absmax int8 quantisation of bf16 activations (the int8-activation runtime of
 * [R] "토큰 동일성의 경계"): for each of the M rows of x (bf16 bits, M x K row-major),
 *   s_x = absmax / 127 (fp32 division),  q = clamp(rint(x / s_x), -127, 127)  (fp32 division,
 *   round half to even); an all-zero row gives s_x = 0 and q = 0. Finite inputs.
 * q_dev: int8[M][K]; s_x_dev: float[M]. 1 <= M <= 4096, K % 128 == 0. */
tern_status tern_quantize_act(const uint16_t* x_bf16_dev, int32_t M, int32_t K, int8_t* q_dev,
                              float* s_x_dev, tern_stream_t stream);

/* M = 1 ternary GEMV: y[n] = scale[n] * sum_k t[n][k] * x[k]  ([R] "학습 중에 포맷이 있어야 하는
 * 이유"; [O] Figure I).
 *   act = TERN_ACT_BF16: x_dev = bf16[K] (bit patterns); x_scale_dev ignored (may be NULL).
 *                        Exact integer sums of the encoded activations (see Conventions).
 *   act = TERN_ACT_INT8: x_dev = int8[K] from tern_quantize_act, x_scale_dev = &s_x (device).
 *                        acc = sum t*q in int32 (exact), y = ((float)acc * s_x) * scale with two
 *                        fp32 round-to-nearest multiplies.
 *   y_dev: float[N]. x_dev 16-byte aligned.
 *   acc_i32_dev: optional int32[N] (NULL to skip): int8 mode writes acc itself there; must be NULL
 *                in bf16 mode (TERN_EINVAL otherwise). */
tern_status tern_gemv(const tern_matrix* W, tern_act act, const void* x_dev, const float* x_scale_dev,
                      float* y_dev, int32_t* acc_i32_dev, tern_stream_t stream);
tern_status tern_gemv_ex(const tern_matrix* W, tern_act act, const void* x_dev, const float* x_scale_dev,
                         float* y_dev, int32_t* acc_i32_dev, uint32_t flags, tern_stream_t stream);

/* One M = 1 GEMV of a batch: y[n] = scale[n] * sum_k t[n][k] * x[k] for matrix W. */
typedef struct {
  tern_matrix W;              /* packed matrix, K a multiple of 128 and at most 12288           */
  const void* x_dev;          /* bf16[K] or int8[K] (16-byte aligned)                          */
  const float* x_scale_dev;   /* int8 mode: &s_x from tern_quantize_act; bf16 mode: ignored     */
  float* y_dev;               /* float[N]                                                      */
} tern_gemv_item;

#define TERN_BATCH_MAX_ITEMS 160

/* Workspace bytes tern_gemv_batch needs for these items (0 if the list is invalid). */
size_t tern_gemv_batch_workspace_bytes(const tern_gemv_item* items, int32_t count, tern_act act);

/* A list of independent M = 1 GEMVs -- e.g. every linear layer of a decode step whose inputs are
 * ready -- computed by two launches: one that turns every activation into tensor-core operand
 * blocks in the workspace, and one persistent kernel (one CTA per SM) that streams all the
 * matrices' packed weights back to back through shared memory, so the weight stream never stops
 * at a layer boundary (the pages place the time above a decode step's DRAM floor at its kernel
 * boundaries: [R] "뉴트리노 엔진"). Arithmetic as for tern_gemv; results are deterministic and,
 * in int8 mode, bit-identical to tern_gemv's. Items must not alias: no y_dev may overlap another
 * item's weights, activations or outputs.
 *   items: host array of `count` descriptors (1 <= count <= TERN_BATCH_MAX_ITEMS), read during
 *          the call only.
 *   workspace_dev: device scratch of at least tern_gemv_batch_workspace_bytes(...) bytes,
 *          16-byte aligned; its contents need no initialisation and are overwritten.
 *   flags: TERN_FLAG_PDL as for tern_gemv_ex (the first launch waits for the preceding kernel
 *          before reading activations; weights are read only after that launch started). */
tern_status tern_gemv_batch(const tern_gemv_item* items, int32_t count, tern_act act, void* workspace_dev,
                            size_t workspace_bytes, uint32_t flags, tern_stream_t stream);

/* Workspace bytes tern_gemm_batch needs for these items and M activation rows (0 if invalid). */
size_t tern_gemm_batch_workspace_bytes(const tern_gemv_item* items, int32_t count, int32_t M, tern_act act);
/* (Only the items' shapes are read: activation and output pointers may be NULL in this query.) */

/* tern_gemv_batch for M activation rows per item (the draft-verify pass of speculative decoding
 * over a whole layer list, [R] "검증된 추측 디코딩"): for every item,
 *   Y[m][n] = scale[n] * sum_k t[n][k] * X[m][k],  0 <= m < M, 1 <= M <= 16,
 * with each item's x_dev = X: bf16[M][K] or int8[M][K] row-major, x_scale_dev = float[M] (int8
 * mode), y_dev = Y: float[M][N]. Each decoded weight word feeds all M rows; the weights stream
 * once. Arithmetic, determinism, aliasing rule, workspace and flags as for tern_gemv_batch (whose
 * call equals this one with M = 1), plus TERN_FLAG_TCGEN05. bf16 lists of 9..16 rows run on the
 * 5th-generation tensor cores (tcgen05: the decoded weights are the MMA's A operand in tensor
 * memory, the activation columns (four limbs per row) its B operand in shared memory); every other
 * list on warp-level mma.sync. Results are bit-identical wherever both exist. */
tern_status tern_gemm_batch(const tern_gemv_item* items, int32_t count, int32_t M, tern_act act,
                            void* workspace_dev, size_t workspace_bytes, uint32_t flags, tern_stream_t stream);

/* Activation prologues: the step before a linear in the Qwen3 block of the Neutrino-1 models
 * ([R] "세 모델과 하나의 컨테이너", model table: RMSNorm before q|k|v and gate|up, SwiGLU before
 * down), computed where the linear's operands are prepared, so it costs no launch of its own. Each
 * kind turns source rows into the bf16 activation the linear consumes, in fp64 with one rounding
 * to nearest (ties to even) to bf16:
 *   TERN_PRO_BF16:    x = the bf16 source row as given (int8 mode then quantises it in place of a
 *                     tern_quantize_act launch)
 *   TERN_PRO_CAST:    x_k = bf16(s_k) of an fp32 row
 *   TERN_PRO_RMSNORM: x_k = bf16((s_k * r) * gain_k), r = 1 / sqrt(sum_k s_k^2 / K + eps)
 *   TERN_PRO_SWIGLU:  x_k = bf16(silu(s_k) * s_(K+k)), silu(z) = z / (1 + e^-z), of a gate|up row of
 *                     2K fp32 values (gate first, as tern_gemm_batch writes a fused gate|up output)
 * In int8 mode the bf16 row is then quantised exactly as tern_quantize_act does. */
typedef enum {
  TERN_PRO_NONE = 0, TERN_PRO_BF16 = 1, TERN_PRO_CAST = 2, TERN_PRO_RMSNORM = 3, TERN_PRO_SWIGLU = 4
} tern_prologue_kind;

typedef struct {
  int32_t kind;               /* tern_prologue_kind                                              */
  float eps;                  /* TERN_PRO_RMSNORM: added to the mean square, finite and >= 0     */
  const void* src_dev;        /* source rows, 16-byte aligned: bf16 [M][K] (BF16), fp32 [M][K]
                                 (CAST, RMSNORM) or fp32 [M][2K] (SWIGLU)                         */
  const uint16_t* gain_dev;   /* TERN_PRO_RMSNORM: bf16 [K] gains, 16-byte aligned               */
} tern_prologue;

/* tern_gemm_batch with a prologue per item: prologues[i] (host array of `count`) prepares item i's
 * activation from its source rows inside the batch's operand-preparation launch. For an item with
 * kind TERN_PRO_NONE the item is read as for tern_gemm_batch. For any other kind:
 *   x_dev        optional output (NULL to skip): the prepared activation, bf16 [M][K] (bf16 mode)
 *                or the quantised int8 q [M][K] (int8 mode), 16-byte aligned;
 *   x_scale_dev  int8 mode, required output: s_x [M] of the per-token quantiser.
 * Results are bit-identical to tern_act_prologue, then (int8 mode) tern_quantize_act, then
 * tern_gemm_batch on the prepared rows. Workspace: tern_gemm_batch_workspace_bytes of the items. */
tern_status tern_gemm_batch_pro(const tern_gemv_item* items, const tern_prologue* prologues, int32_t count,
                                int32_t M, tern_act act, void* workspace_dev, size_t workspace_bytes,
                                uint32_t flags, tern_stream_t stream);

/* The prologue alone: M rows of K (K % 128 == 0) bf16 activations into x_bf16_dev [M][K]
 * (16-byte aligned). Kind TERN_PRO_NONE is invalid here. */
tern_status tern_act_prologue(const tern_prologue* pro, int32_t M, int32_t K, uint16_t* x_bf16_dev,
                              tern_stream_t stream);

/* Small-M GEMM for the draft-verify pass of speculative decoding ([R] "검증된 추측 디코딩": the
 * 8B scores up to seven drafted positions in one batched forward pass):
 *   Y[m][n] = scale[n] * sum_k t[n][k] * X[m][k],  0 <= m < M, 1 <= M <= 16.
 * Each decoded weight word is reused for all M rows. X_dev: bf16[M][K] or int8[M][K];
 * x_scale_dev: float[M] (int8 only); Y_dev: float[M][N]. Arithmetic as for tern_gemv. */
tern_status tern_gemm_small_m(const tern_matrix* W, int32_t M, tern_act act, const void* X_dev,
                              const float* x_scale_dev, float* Y_dev, tern_stream_t stream);
tern_status tern_gemm_small_m_ex(const tern_matrix* W, int32_t M, tern_act act, const void* X_dev,
                                 const float* x_scale_dev, float* Y_dev, uint32_t flags,
                                 tern_stream_t stream);

/* Prefill dense contraction ([R] "실행해보기": batched prefill):
 *   Y[m][n] = scale[n] * sum_k t[n][k] * X[m][k] for 1 <= M <= 65536 rows of bf16 activations,
 * computed as a genuine dense matrix product on the 5th-generation tensor cores: trits expanded
 * to bf16 (2.0 * t) in shared memory, tcgen05 MMA with the fp32 accumulator in tensor memory,
 * times 0.5 * scale[n] at the end (one fp32 rounding of the accumulated sum, which the tensor
 * core forms in fp32). X_bf16_dev: bf16[M][K] row-major, 16-byte aligned; Y_dev: float[M][N],
 * 4-byte aligned (16-byte aligned with N % 4 == 0 for the fastest stores). */
tern_status tern_gemm_prefill(const tern_matrix* W, int32_t M, const uint16_t* X_bf16_dev, float* Y_dev,
                              tern_stream_t stream);

/* Scratch bytes i8_head_gemv_argmax needs for V rows and M activation rows. */
size_t i8_head_workspace_bytes(int32_t V, int32_t M);

/* int8 output head with fused per-row scale and greedy argmax ([R] "3진 계열이라는 이름의 실체":
 * the head stays int8; [R] "뉴트리노 엔진": the unembedding streams at the DRAM roofline):
 *   logits[m][v] = s_h[v] * sum_k W[v][k] * x[m][k],   argmax[m] = argmax_v logits[m][v]
 * with the lowest index winning an exact tie, maxval[m] = logits[m][argmax[m]].
 *   W_dev: int8[V][K] row-major, 16-byte aligned; scale_f16_dev: fp16[V]; K % 128 == 0;
 *   1 <= M <= 16; act/X_dev/x_scale_dev as for tern_gemm_small_m (int8 mode: logits =
 *   ((float)acc * s_x) * s_h, bit-exact; bf16 mode: exact products, fp32-rounded logits).
 *   logits_dev: optional float[M][V] (NULL to skip writing the logits).
 *   workspace_dev: at least i8_head_workspace_bytes(V, M) bytes, 16-byte aligned, zero-filled
 *   before its first use; every call leaves it zero-filled again, so one buffer serves any
 *   number of calls in stream order (two calls that overlap in time need two buffers). */
tern_status i8_head_gemv_argmax(const int8_t* W_dev, const uint16_t* scale_f16_dev, int32_t V, int32_t K,
                                int32_t M, tern_act act, const void* X_dev, const float* x_scale_dev,
                                int32_t* argmax_dev, float* maxval_dev, float* logits_dev,
                                void* workspace_dev, size_t workspace_bytes, tern_stream_t stream);
tern_status i8_head_gemv_argmax_ex(const int8_t* W_dev, const uint16_t* scale_f16_dev, int32_t V,
                                   int32_t K, int32_t M, tern_act act, const void* X_dev,
                                   const float* x_scale_dev, int32_t* argmax_dev, float* maxval_dev,
                                   float* logits_dev, void* workspace_dev, size_t workspace_bytes,
                                   uint32_t flags, tern_stream_t stream);

/* The verify round of speculative decoding on the device ([R] "검증된 추측 디코딩: 속도만 바꾸고
 * 답은 바꾸지 않는다": the target scores the drafted positions in one batched pass and keeps the
 * longest prefix of drafts that equal its own greedy tokens). i8_head_gemv_argmax over the
 * M = k + 1 activation rows of the verify pass (row j: the position after which draft[j] was
 * proposed; row k: after the last draft), then, in the same launch, the acceptance count:
 *   n = the largest j <= k with draft[i] == argmax[i] for every i < j,
 *   accept_dev[0] = n, accept_dev[1] = argmax[n]   (the round yields n + 1 tokens)
 * draft_dev: int32 [M - 1] (may be NULL when M = 1); accept_dev: int32 [2]. Other arguments as
 * for i8_head_gemv_argmax (no logits output, no flags). */
tern_status i8_head_verify(const int8_t* W_dev, const uint16_t* scale_f16_dev, int32_t V, int32_t K, int32_t M,
                           tern_act act, const void* X_dev, const float* x_scale_dev, const int32_t* draft_dev,
                           int32_t* argmax_dev, float* maxval_dev, int32_t* accept_dev, void* workspace_dev,
                           size_t workspace_bytes, tern_stream_t stream);

/* The acceptance rule alone on k + 1 argmax indices already on the device (argmax_dev int32
 * [k + 1], draft_dev int32 [k], accept_dev int32 [2] as above; 0 <= k <= 65535). */
tern_status tern_verify_accept(const int32_t* argmax_dev, const int32_t* draft_dev, int32_t k, int32_t* accept_dev,
                               tern_stream_t stream);

/* No-allocation variant of i8_head_gemv_argmax. The source pages describe no counterpart: it is
 * an interface convenience of this library. Same arguments, results and error codes as
 * i8_head_gemv_argmax, minus the workspace: the scratch is one library-internal device array of
 * TERN_HEAD_NOALLOC_SCRATCH_BYTES bytes per device, enough for M <= TERN_HEAD_NOALLOC_MAX_M.
 *   - M outside 1..TERN_HEAD_NOALLOC_MAX_M (scratch need above the array's size): TERN_ESHAPE,
 *     nothing launched.
 *   - The first call on a device looks up the array's address (cudaGetSymbolAddress, with that
 *     device current) and keeps it; that first call must come before any stream capture. The kept
 *     address belongs to the device's context: after cudaDeviceReset on that device, this entry
 *     point must not be called again in the process.
 *   - Every argument is checked before anything is enqueued, exactly as for i8_head_gemv_argmax.
 *   - Each call clears the scratch bytes it uses (cudaMemsetAsync on `stream`) before the launch;
 *     no call allocates or frees device memory.
 *   - All calls on one device share the array: calls that overlap in time (different streams,
 *     host threads) race and may return wrong results. Order them on one stream. */
#define TERN_HEAD_NOALLOC_MAX_M 16
#define TERN_HEAD_NOALLOC_SCRATCH_BYTES 256
tern_status i8_head_gemv_argmax_noalloc(const int8_t* W_dev, const uint16_t* scale_f16_dev, int32_t V,
                                        int32_t K, int32_t M, tern_act act, const void* X_dev,
                                        const float* x_scale_dev, int32_t* argmax_dev, float* maxval_dev,
                                        float* logits_dev, tern_stream_t stream);

/* A decode step's chain of dependent linear layers in one cooperative launch (M = 1). The pages put
 * the time above a decode step's DRAM floor in the dependency chains between its ~120 kernels
 * ([R] "뉴트리노 엔진: 토큰 하나의 시간은 어디로 가는가"); here every linear of the chain runs in one
 * persistent kernel whose weight stream continues across the linears while each linear waits for
 * the one it reads. Item i's activation is its prologue (as for tern_gemm_batch_pro) applied to:
 *   src_item < 0:  src_dev, written before the launch;
 *   src_item = j:  item j's fp32 output y (kinds TERN_PRO_CAST, TERN_PRO_RMSNORM: its first K
 *                  values), or, with src_h = 1 (kind TERN_PRO_BF16), item j's SwiGLU output h.
 * An item with swiglu_out = 1 has its rows interleaved in groups of eight: rows 16j .. 16j + 7 are
 * gate rows 8j .. 8j + 7 and rows 16j + 8 .. 16j + 15 the matching up rows (N % 16 == 0); besides y it
 * writes h[8j + i] = bf16(silu(y[16j + i]) * y[16j + 8 + i]) (silu(z) = z / (1 + e^-z), fp64, one
 * rounding) -- the SwiGLU of the gate|up output, fused into its epilogue.
 * Outputs equal tern_gemm_batch_pro's for the same prologue and source, bit for bit, in both modes. */
typedef struct {
  tern_matrix W;                /* K <= 12288                                                     */
  int32_t kind;                 /* TERN_PRO_BF16, TERN_PRO_CAST or TERN_PRO_RMSNORM              */
  int32_t src_item;             /* an earlier item, or -1                                         */
  int32_t src_h;                /* 1: the source is item src_item's SwiGLU output h               */
  int32_t swiglu_out;           /* 1: interleaved gate|up rows; h_dev receives the SwiGLU        */
  float eps;                    /* TERN_PRO_RMSNORM                                               */
  const void* src_dev;          /* src_item < 0: bf16 [K] (BF16) or fp32 [K], 16-byte aligned     */
  const uint16_t* gain_dev;     /* TERN_PRO_RMSNORM: bf16 [K], 16-byte aligned                   */
  float* y_dev;                 /* fp32 [N], 16-byte aligned                                      */
  uint16_t* h_dev;              /* swiglu_out: bf16 [N / 2], 16-byte aligned                      */
  float* x_scale_dev;           /* int8 mode, optional output: s_x of this item's activation      */
} tern_chain_item;

/* Host handle of a planned chain (filled by tern_chain_plan; owned by the caller). */
typedef struct {
  void* workspace_dev;
  int32_t count, mode, grid, stages;
  int32_t seg_parts;            /* operand segments a CTA prepares per linear (plan detail)       */
  size_t smem_bytes;
} tern_chain;

#define TERN_CHAIN_MAX_ITEMS 4096

/* Workspace bytes of a chain (0 if the list is invalid; pointers are not checked). */
size_t tern_chain_workspace_bytes(const tern_chain_item* items, int32_t count, tern_act act);

/* Checks the items, writes the chain's plan (tensor maps, per-linear shapes and sources) into
 * workspace_dev (64-byte aligned, at least tern_chain_workspace_bytes) and clears its counters and
 * scratch. Synchronous (blocking copies): call it once, before any stream capture. */
tern_status tern_chain_plan(const tern_chain_item* items, int32_t count, tern_act act, void* workspace_dev,
                            size_t workspace_bytes, tern_chain* chain);

/* Runs the planned chain on `stream` (one cooperative launch: one CTA per SM, all resident). The
 * workspace is left ready for the next run; two runs of one workspace must not overlap in time. A
 * wait that gives up latches TERN_ETIMEOUT (tern_device_status) and the outputs are incomplete. */
tern_status tern_chain_run(const tern_chain* chain, tern_stream_t stream);

/* Five-valued weights in 256-weight blocks and the block-scaled int8 head: this library's reading of
 * the pages' shipped FV5 and FV5B types ([R] "FV5와 FV5B: llama.cpp 포크가 공개한 블록 구조":
 * 256 weights per block, three bitplanes plus fp32 s_lo and s_hi, 3.25 bits per weight; FV5B: int8
 * with one fp32 scale per block, used for the embedding and output head).
 *   - A weight is a code c in {-2, -1, 0, +1, +2}: w = 0, sign(c) * s_lo[b] (|c| = 1) or
 *     sign(c) * s_hi[b] (|c| = 2), b = the weight's 256-weight block of its row. K % 512 == 0.
 *   - Planes of a row: mask (c != 0), sign (c < 0), high magnitude (|c| = 2), K/32 words each, in
 *     the ternary layout's bit order (mask and magnitude bit of in-word trit j at p(j), sign bit at
 *     (p(j) + 1) % 32); inside each group of 16 words (512 trits) of a plane, logical word
 *     w = 4e + t is stored at position 4t + e. Row n = [mask | sign | magnitude], 3K/32 words.
 *   - Scales: fp32 [N][K/256][2] = (s_lo, s_hi) of each row and block.
 *   - Products: exact integer sums per block, scaled per block in fp64 and rounded once to fp32
 *     (int8 mode: fp32(s_x * sum_b (s_lo A_lo + s_hi A_hi))). bf16 mode keeps the per-output bound
 *     of the bf16 mode with max(s_lo, s_hi) of the row in place of the row scale. */
typedef struct {
  int32_t N, K;                 /* rows, K % 512 == 0                                           */
  const uint32_t* planes;       /* device, N * 3K/32 words, 16-byte aligned                     */
  const float* scales;          /* device, N * K/256 * 2 fp32 (s_lo, s_hi), 8-byte aligned      */
} tern_fv5_matrix;

/* Bytes of FV5 planes for N x K (3NK/8); 0 if the shape is invalid. */
size_t tern_fv5_packed_bytes(int32_t N, int32_t K);

/* Packs codes int8 [N][K] (values -2..2, 16-byte aligned) into planes_dev (N * 3K/32 words);
 * err_flag_dev is cleared, then set if a code is outside -2..2. */
tern_status tern_fv5_pack(const int8_t* codes_dev, int32_t N, int32_t K, uint32_t* planes_dev, int32_t* err_flag_dev,
                          tern_stream_t stream);

/* Y[m][n] = sum_k w[n][k] X[m][k] for 1 <= M <= 8 (bf16) or 16 (int8) activation rows; X, x_scale
 * and Y as for tern_gemm_small_m. */
tern_status tern_fv5_gemm(const tern_fv5_matrix* W, int32_t M, tern_act act, const void* X_dev, const float* x_scale_dev,
                          float* Y_dev, tern_stream_t stream);

/* A list of five-valued linears at M = 1 in one persistent launch (the batched counterpart of
 * tern_fv5_gemm for a decode step: no launch per linear). Item i: y_i[n] = sum_k w_i[n][k] x_i[k],
 * x_i bf16 [K] or int8 [K] with x_scale_i [1] (int8 mode), y_i fp32 [N]; the same products and
 * rounding as tern_fv5_gemm at M = 1, the block sums added in block order (a 16-row tile split
 * between warps hands its partial sums on in that order, so int8 mode stays bit-identical).
 * 1 <= count <= 160, K % 512 == 0 and K <= 12288 per item; W, x (16-byte aligned), x_scale (int8
 * mode, 4-byte aligned) and y (4-byte aligned) device pointers, caller-owned; no workspace; y
 * must not overlap any item's x. Argument errors return before anything is enqueued. The hand-off
 * between warps is a bounded wait: if it gives up, TERN_ETIMEOUT latches (tern_device_status) and
 * the outputs are incomplete. */
typedef struct {
  tern_fv5_matrix W;
  const void* x_dev;
  const float* x_scale_dev;
  float* y_dev;
} tern_fv5_batch_item;
#define TERN_FV5_BATCH_MAX_ITEMS 160
tern_status tern_fv5_gemv_batch(const tern_fv5_batch_item* items, int32_t count, tern_act act, tern_stream_t stream);

/* The int8 head with one fp32 scale per row and 256-weight block (block_scale_dev: fp32
 * [V][K/256], 4-byte aligned; K % 256 == 0) instead of the fp16 row scale:
 *   logits[m][v] = sum_b block_scale[v][b] * sum_{k in b} W[v][k] x[m][k],
 * argmax with the lowest index on exact ties. bf16 mode M <= 8, int8 mode M <= 16; other
 * arguments and the workspace as for i8_head_gemv_argmax. */
tern_status fv5b_head_gemv_argmax(const int8_t* W_dev, const float* block_scale_dev, int32_t V, int32_t K, int32_t M,
                                  tern_act act, const void* X_dev, const float* x_scale_dev, int32_t* argmax_dev,
                                  float* maxval_dev, float* logits_dev, void* workspace_dev, size_t workspace_bytes,
                                  tern_stream_t stream);

/* Synchronise `stream`, read *err_flag_dev and map it: 0 -> TERN_OK, nonzero -> TERN_EBADCODE. */
tern_status tern_read_flag(const int32_t* err_flag_dev, tern_stream_t stream);

/* Synchronise `stream` and report whether any kernel of this library on the current device gave
 * up a bounded wait (an mbarrier that did not complete within seconds) since the last call:
 * TERN_ETIMEOUT if so, else TERN_OK. Reading clears the device's latches (one device word per
 * kernel family, the library's only device-side state besides the no-allocation head's scratch;
 * they are shared by every stream and caller of the device). Kernels that give up stop early and
 * leave their outputs incomplete; they never hang or trap. */
tern_status tern_device_status(tern_stream_t stream);

#if defined(__GNUC__)
#pragma GCC visibility pop
#endif

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* TERN_H_ */
