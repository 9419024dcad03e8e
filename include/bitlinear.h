/*
 * bitlinear.h - C ABI of the B200 (sm_100a) BitLinear forward library.
 *
 * What it computes: the BitLinear layer of BitNet b1.58 ("The Era of 1-bit LLMs: All
 * Large Language Models are in 1.58 Bits"). Per the dmarx anthology record LIT-380 (Key
 * takeaways, bullet 1), BitLinear takes the place of nn.Linear, an absmean quantization
 * function limits the weights to {-1, 0, +1} and activations are held in 8 bits; bullet 4
 * notes that the matrix product then needs only integer additions. The searcharxiv.com
 * abstract page (Abstract) has every weight ternary. The pages give no formula;
 * the library implements the plainest reading:
 *
 *   gamma    = mean |W|                                    (fp32; exact sum, rounded once)
 *   c[n,k]   = RoundClip(W[n,k] / (gamma + eps), -1, 1)     (fp32 quotient, ties to even)
 *   a_t      = max_k |x[t,k]|,  r_t = 127 / a_t,  s_t = a_t / 127           (fp32)
 *   q[t,k]   = clip(rne(x[t,k] * r_t), -127, 127)           (0 if a_t == 0 or x == 0)
 *   acc[t,n] = sum_k c[n,k] * q[t,k]                         (exact int32)
 *   y[t,n]   = float(acc[t,n]) * (s_t * gamma)               (fp32, or its bf16 RNE)
 *
 * Shapes follow nn.Linear: W [N][K] (out x in), x [M][K], y [M][N], all row-major.
 *
 * Packed weight format (a 1.58-bit weight stored in 2 bits, hackerpaper HN page,
 * thread 17): trit c is stored as the 2-bit code u = c + 1 (0, 1, 2; 3 is never
 * written). Row n occupies K/4 bytes at byte offset n*K/4. The little-endian 32-bit word
 * g of a row holds trits k = 16g .. 16g+15; trit k = 16g + 4j + i (i, j in 0..3) is in
 * bits 8i+2j .. 8i+2j+1 of that word. (Shifting the word right by 2j and masking with
 * 0x03030303 yields trits 16g+4j .. 16g+4j+3 as four consecutive bytes.)
 *
 * Conventions for every entry point:
 *  - Ownership: the caller allocates and frees every buffer. Device pointers must stay
 *    valid until the work queued on `stream` has finished. The library keeps no pointer
 *    after a call returns and never allocates or frees device memory in these calls.
 *  - Execution: work is queued asynchronously on `stream` (a cudaStream_t; NULL is the
 *    legacy default stream) on the current CUDA device. Argument errors are reported
 *    synchronously, before anything is queued. A failed launch returns BL_ERR_CUDA.
 *    Faults found on the device (non-finite input, a wait that timed out) are recorded
 *    in a per-device status word read by bitlinear_get_device_status().
 *  - Shapes: M, N >= 1; K >= 64 and K % 64 == 0; M*K, N*K and M*N below 2^31.
 *    Otherwise BL_ERR_UNSUPPORTED_SHAPE.
 *  - Alignment: every device pointer 16-byte aligned, else BL_ERR_MISALIGNED.
 *  - Thread safety: calls on different streams may run concurrently; they share only the
 *    device status word.
 */
#ifndef BITLINEAR_H_
#define BITLINEAR_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BL_OK = 0,
  BL_ERR_INVALID_ARG = 1,       /* null pointer, bad dtype, eps < 0 or not finite */
  BL_ERR_UNSUPPORTED_SHAPE = 2, /* shape outside the limits above */
  BL_ERR_MISALIGNED = 3,        /* a pointer is not 16-byte aligned */
  BL_ERR_CUDA = 4,              /* a CUDA runtime call or kernel launch failed */
  BL_ERR_TIMEOUT = 5,           /* a device-side wait exceeded its limit (status word) */
  BL_ERR_NONFINITE = 6,         /* Inf or NaN in W or x (status word) */
  BL_ERR_WORKSPACE = 7          /* workspace missing or smaller than required */
} bl_status;

typedef enum { BL_F32 = 0, BL_BF16 = 1, BL_I32 = 2 } bl_dtype;

/* One BitLinear layer of a chain (bitlinear_chain_forward). */
typedef struct {
  const uint8_t* packed; /* device [N][K/4], from bitlinear_quantize_weights */
  const float* gamma;    /* device, one float */
  int N, K;              /* out x in */
  int src;               /* its input: -1 = the chain input x, j = the output of layer j < this */
  void* out;             /* device [M][N] bf16 to receive its output, or NULL (then kept in
                            the workspace); ignored for the last layer, which writes y */
} bl_layer;

/* Device bytes of workspace that bitlinear_quantize_weights (for N x K) and
 * bitlinear_forward / bitlinear_contract_i32 (for M x N x K) need; the largest of the
 * three. Pure host function. Returns 0 for shapes the library rejects. */
size_t bitlinear_workspace_size(int M, int N, int K);

/* Absmean ternary weight quantization (LIT-380 bullet 1; Abstract of the searcharxiv.com
 * page): gamma = mean|W| over all N*K weights, then every weight becomes the code
 * RoundClip(w / (gamma + eps), -1, 1), packed 2 bits per trit.
 *   W       device, [N][K] row-major, fp32 (w_dtype BL_F32) or bf16 (BL_BF16); read only.
 *   eps     >= 0, finite (1e-5 is the usual choice); added to gamma in fp32.
 *   packed  device, N*K/4 bytes, written in the packed format above.
 *   gamma   device, one float, written.
 *   ws      device workspace of at least bitlinear_workspace_size(1, N, K) bytes; its
 *           contents on entry do not matter and are clobbered.
 * gamma is the exact sum of |w| rounded once to double, divided by N*K in double and
 * rounded to float, so it does not depend on launch shape or summation order.
 * Inf/NaN in W sets BL_ERR_NONFINITE in the device status word (outputs undefined). */
bl_status bitlinear_quantize_weights(const void* W, int w_dtype, int N, int K, float eps,
                                     uint8_t* packed, float* gamma, void* ws,
                                     size_t ws_bytes, void* stream);

/* Words of the exact sum of |w| that bitlinear_weight_abssum writes. */
#define BL_ABSSUM_WORDS 14

/* Tensor parallelism, step 1 of 2 of the absmean weight quantization of a matrix split
 * over several GPUs (rows for a column-parallel layer, columns for a row-parallel one):
 * gamma is the mean of |w| over the WHOLE matrix (LIT-380 bullet 1; one scale per weight
 * tensor), so each GPU first forms the exact sum of |w| over its own shard.
 *   W     device, the shard [N][K] row-major (its own contiguous copy), fp32 or bf16.
 *   sums  device, BL_ABSSUM_WORDS uint64, written: the exact sum S of |w| over the shard
 *         as S * 2^149 = sum_j sums[j] * 2^(32 j) (columns not carried, each below 2^57).
 *         The words of several shards add up exactly (plain uint64 addition, e.g. an
 *         NCCL sum all-reduce) to the words of their union.
 *   ws    device workspace of at least bitlinear_workspace_size(1, N, K) bytes.
 * Inf/NaN in W sets BL_ERR_NONFINITE in the device status word. */
bl_status bitlinear_weight_abssum(const void* W, int w_dtype, int N, int K, uint64_t* sums,
                                  void* ws, size_t ws_bytes, void* stream);

/* Tensor parallelism, step 2 of 2: gamma = (S rounded once to double) / n_total rounded to
 * float, from the added words of every shard, then the codes of THIS shard's weights,
 * RoundClip(w / (gamma + eps), -1, 1), 2-bit packed as bitlinear_quantize_weights does.
 * With every shard's words added, gamma and the codes are bit for bit those of
 * bitlinear_quantize_weights on the whole matrix.
 *   W        device, the shard [N][K] (the one given to step 1).
 *   n_total  number of weights of the whole matrix (>= N * K).
 *   sums     device, BL_ABSSUM_WORDS uint64: the words of all shards, added.
 *   packed   device, N*K/4 bytes; gamma device, one float; both written.
 * Non-finite weights are reported by step 1, not here. */
bl_status bitlinear_quantize_weights_from_abssum(const void* W, int w_dtype, int N, int K,
                                                 long long n_total, const uint64_t* sums,
                                                 float eps, uint8_t* packed, float* gamma,
                                                 void* stream);

/* Per-token absmax int8 activation quantization (8-bit activations, LIT-380
 * bullet 1): q = clip(rne(x * (127 / a_t)), -127, 127), scale_t = a_t / 127.
 *   x      device, [M][K], fp32 or bf16 (x_dtype); read only.
 *   xq     device, [M][K] int8, written.
 *   scale  device, [M] fp32, written (0 for an all-zero row).
 * Inf/NaN in x sets BL_ERR_NONFINITE in the device status word. */
bl_status bitlinear_quantize_acts(const void* x, int x_dtype, int M, int K, int8_t* xq,
                                  float* scale, void* stream);

/* Per-token absolute maximum a_t = max_k |x[t,k]| (the first half of the activation
 * quantization). Under tensor parallelism with K split, each GPU holds a K-shard of every
 * token row; the MAX all-reduce of these per-shard values is the row's a_t.
 *   x     device, [M][K] fp32 or bf16.   amax  device, [M] fp32, written.
 * Inf/NaN in x sets BL_ERR_NONFINITE in the device status word. */
bl_status bitlinear_act_absmax(const void* x, int x_dtype, int M, int K, float* amax,
                               void* stream);

/* The activation quantization with a_t given: q = clip(rne(x * fl(127 / a_t)), -127, 127),
 * scale_t = fl(a_t / 127), exactly as bitlinear_quantize_acts computes them when a_t is
 * the row's own absmax. For a K-shard of the rows, pass the absmax of the whole rows.
 *   x      device, [M][K].   amax   device, [M] fp32 (a_t >= 0; values of x above a_t
 *   clip to +-127).   xq     device, [M][K] int8, written.   scale  device, [M], written. */
bl_status bitlinear_quantize_acts_absmax(const void* x, int x_dtype, int M, int K,
                                         const float* amax, int8_t* xq, float* scale,
                                         void* stream);

/* The rescale on its own: y[t,n] = fl(float(acc[t,n]) * fl(scale_t * gamma)) (fp32, or the
 * bf16 RNE of that value), for an int32 product formed elsewhere, e.g. the SUM
 * all-reduce of per-GPU partial products of bitlinear_contract_i32 under a K split (an
 * exact integer sum, so the result equals the single-GPU forward bit for bit).
 *   acc    device, [M][N] int32.   scale  device, [M].   gamma  device, one float.
 *   y      device, [M][N], y_dtype BL_F32 or BL_BF16, written.
 * M, N >= 1 and M*N below 2^31, else BL_ERR_UNSUPPORTED_SHAPE. */
bl_status bitlinear_rescale(const int32_t* acc, const float* scale, const float* gamma,
                            void* y, int y_dtype, int M, int N, void* stream);

/* The BitLinear forward: quantize x per token, contract with the packed ternary weights
 * in exact int32 (additions only, LIT-380 bullet 4) and rescale by s_t * gamma.
 *   x       device, [M][K], fp32 or bf16 (x_dtype).
 *   packed  device, [N][K/4] packed codes from bitlinear_quantize_weights.
 *   gamma   device, one float.
 *   y       device, [M][N], y_dtype BL_F32 or BL_BF16 (RNE of the fp32 value).
 *   ws      device workspace of at least bitlinear_workspace_size(M, N, K) bytes.
 * Small M runs one CUDA-core kernel that quantizes x in its prologue; larger M quantizes
 * x into the workspace and runs the tcgen05 int8 tensor-core GEMM. Both give the same
 * bits. */
bl_status bitlinear_forward(const void* x, int x_dtype, const uint8_t* packed,
                            const float* gamma, void* y, int y_dtype, int M, int N, int K,
                            void* ws, size_t ws_bytes, void* stream);

/* Workspace bytes of bitlinear_chain_forward for these layers and M tokens; 0 if the
 * chain is invalid. Pure host function. */
size_t bitlinear_chain_workspace_size(int M, const bl_layer* layers, int L);

/* A chain of BitLinear layers over one batch of M tokens, every layer as in
 * bitlinear_forward: layer l reads x (src = -1) or the output of an earlier layer, every
 * output but the last is kept in bf16 (the activation type of the model), the last
 * layer writes y. Several layers may read the same input (the gate and up projections of
 * a feed-forward block); the input is then quantized once.
 * Fused across layers: the kernel that writes a layer's output also forms the per-token
 * absmax of it (atomic max in its epilogue), so the next layer's activation quantization
 * is a single pass (or part of the GEMV's prologue); every kernel is launched with
 * programmatic dependent launch, so it sets up, and prefetches its packed weights (TMA
 * into shared memory, or into L2), while the kernel before it still runs. Capture the call
 * in a CUDA graph to take the host out of the loop. The skinny kernel's K splits may
 * exchange int32 sums up to the packed weight bytes here (a quarter in bitlinear_forward):
 * the chain clears its sums once per call and every kernel leaves them cleared. Results
 * equal layer-by-layer bitlinear_forward calls with bf16 intermediates, bit for bit.
 *   x       device [M][K of the layers with src = -1], fp32 or bf16.
 *   layers  host array of L layers; K of a layer with src = j equals N of layer j.
 *   y       device [M][N of the last layer], BL_F32 or BL_BF16.
 *   ws      device, at least bitlinear_chain_workspace_size bytes (contents ignored).
 * Errors as bitlinear_forward; BL_ERR_INVALID_ARG for a bad src, null pointers or L < 1. */
bl_status bitlinear_chain_forward(const void* x, int x_dtype, int M, const bl_layer* layers,
                                  int L, void* y, int y_dtype, void* ws, size_t ws_bytes,
                                  void* stream);

/* Base-3 weight format (hackerpaper HN page, thread 3: five ternary digits fit a byte,
 * 3^5 = 243 <= 256): 1.6 bits per weight, 0.8 of the 2-bit format's bytes, for the
 * bandwidth-bound decode path. Row n occupies bitlinear_base3_row_bytes(K) =
 * ceil(K/80)*16 bytes at n times that; in each 16-byte chunk j of a row, byte i holds the
 * trits k = 80 j + 16 p + i (p = 0..4; past K they are 0) as B = ceil(256 v / 243), where
 * v = sum_p (c_p + 1) 3^(4-p). The digits come back as floor(B 3^(p+1) / 256) mod 3.
 * Pure host function; 0 for K that the library rejects. */
size_t bitlinear_base3_row_bytes(int K);

/* Converts packed weights from the 2-bit format (bitlinear_quantize_weights) to the base-3
 * format: the same codes, bit for bit.
 *   packed   device [N][K/4].   packed3  device [N][bitlinear_base3_row_bytes(K)], written. */
bl_status bitlinear_pack_base3(const uint8_t* packed, int N, int K, uint8_t* packed3,
                               void* stream);

/* bitlinear_forward on base-3 weights, for decode batches of M <= 4 tokens (a CUDA-core
 * GEMV that quantizes x in its prologue and decodes five trits per byte with multiplies
 * by 3). Same arguments and bits as bitlinear_forward; no workspace.
 * BL_ERR_UNSUPPORTED_SHAPE for M > 4 or M * ceil(K/80) * 80 above 200 KB. */
bl_status bitlinear_forward_base3(const void* x, int x_dtype, const uint8_t* packed3,
                                  const float* gamma, void* y, int y_dtype, int M, int N, int K,
                                  void* stream);

/* The transposed 2-bit weights: row k of packedT [K][N/4] holds the trits W[., k] along n,
 * in the packed format above. Input of bitlinear_backward's grad_x (its contraction runs
 * over n). N % 64 == 0, else BL_ERR_UNSUPPORTED_SHAPE.
 *   packed  device [N][K/4].   packedT  device [K][N/4], written. */
bl_status bitlinear_pack_transpose(const uint8_t* packed, int N, int K, uint8_t* packedT,
                                   void* stream);

/* Workspace bytes of bitlinear_backward (0 for shapes it rejects). Pure host function. */
size_t bitlinear_backward_workspace_size(int M, int N, int K);

/* BitLinear backward for quantization-aware training with the straight-through
 * estimator (hackerpaper HN page, thread 21: the quantizers' rounding passes gradients
 * unchanged; LIT-380 bullet 1: b1.58 is trained with the quantizers in place). With the
 * forward y = X~ W~^T, X~ = q s (per-token int8 activations), W~ = gamma c:
 *   grad_x[t,k] = gamma * sum_n G[t,n] c[n,k]          (fp32 [M][K])
 *   grad_w[n,k] = sum_t G[t,n] X~[t,k]                  (fp32 [N][K])
 * where X~ is held in bf16, X~ = bf16(q * s), q and s the forward's quantization of x.
 * Both run on the tcgen05 tensor cores as bf16 x bf16 -> fp32 contractions; products are
 * exact, only the fp32 accumulation order differs from a sequential sum.
 *   x        device [M][K] fp32 or bf16: the forward's input (needed for grad_w).
 *   grad_y   device [M][N] bf16: dL/dy.
 *   packedT  device [K][N/4] from bitlinear_pack_transpose (needed for grad_x).
 *   gamma    device, one float (needed for grad_x).
 *   grad_x   device [M][K] fp32, or NULL to skip.   grad_w  device [N][K] fp32, or NULL.
 *   ws       device, bitlinear_backward_workspace_size(M, N, K) bytes (for grad_w).
 * N % 64 == 0, else BL_ERR_UNSUPPORTED_SHAPE. */
bl_status bitlinear_backward(const void* x, int x_dtype, const void* grad_y,
                             const uint8_t* packedT, const float* gamma, float* grad_x,
                             float* grad_w, int M, int N, int K, void* ws, size_t ws_bytes,
                             void* stream);

/* The integer stage alone (test hook, same kernels as bitlinear_forward):
 * acc[t,n] = sum_k c[n,k] * xq[t,k].
 *   xq      device, [M][K] int8 (values in [-127, 127]).
 *   packed  device, [N][K/4].
 *   acc     device, [M][N] int32, written.
 *   ws      device workspace of at least bitlinear_workspace_size(M, N, K) bytes. */
bl_status bitlinear_contract_i32(const int8_t* xq, const uint8_t* packed, int32_t* acc,
                                 int M, int N, int K, void* ws, size_t ws_bytes,
                                 void* stream);

/* bitlinear_forward without a workspace argument. The paper has no counterpart: this
 * entry point exists for callers that cannot allocate device memory at the point of
 * call, e.g. code running inside another runtime whose memory planner owns the whole
 * device and forbids further cudaMalloc, or latency-critical paths that avoid cudaMalloc
 * and cudaFree because those calls can synchronize the device.
 *   Same arguments, results and errors as bitlinear_forward, minus ws / ws_bytes.
 *   Scratch: a 16 MiB array compiled into the library (held on every GPU that loads it
 *   until the process exits). Small M needs none; otherwise M*K + 8*M bytes (each part
 *   rounded up to 256) must fit in 16 MiB, else BL_ERR_WORKSPACE is returned before
 *   anything is queued.
 *   Kernels: the same CUDA-core GEMV as bitlinear_forward for the smallest M; up to 256
 *   tokens the skinny tensor-core kernel with K never split across CTAs (bitlinear_forward
 *   splits K on shapes with few weight tiles, so those shapes run slower here, e.g. 16
 *   tokens on a 3200 x 8640 matrix); above 256 tokens the prefill GEMM. Same bits either
 *   way.
 *   The first call on a device looks up the array's device address (cudaGetSymbolAddress)
 *   and caches it; make that first call before any stream capture.
 *   Every call on a device shares the one array: calls whose work overlaps on the GPU
 *   race and give undefined results. The library allocates and frees nothing here. */
bl_status bitlinear_forward_noalloc(const void* x, int x_dtype, const uint8_t* packed,
                                    const float* gamma, void* y, int y_dtype, int M, int N,
                                    int K, void* stream);

/* Waits for `stream`, then reads and clears the current device's status word:
 * BL_OK, BL_ERR_NONFINITE or BL_ERR_TIMEOUT (the first recorded wins in that order of
 * severity: TIMEOUT over NONFINITE). BL_ERR_CUDA if the wait or the read fails. */
bl_status bitlinear_get_device_status(void* stream);

/* Test hook for the bounded-wait machinery: runs one block that waits on an mbarrier no
 * thread ever arrives on, giving up after `timeout_ns` nanoseconds (1e3 .. 5e9). The
 * kernel then records BL_ERR_TIMEOUT in the status word and exits normally, so the
 * context stays usable. */
bl_status bitlinear_debug_timeout_probe(uint64_t timeout_ns, void* stream);

/* Introspection of the forward's kernel choice, for tests; pure host code (no device,
 * nothing queued). For an M x N x K forward on a GPU with `sms` multiprocessors:
 *   *path      0 = CUDA-core GEMV (M <= 2, or M <= 4 with at most 2 MB of packed weights),
 *              1 = skinny tcgen05 kernel (other M <= 256), 2 = prefill tcgen05 GEMM.
 *   *k_splits  CTAs sharing each 128-row weight tile along K on path 1: as many as the CTA
 *              slots (two per SM up to 64 tokens, one above) hold in one wave, with at least
 *              8 K blocks of 128 per split and the int32 sums they exchange, M*N*4 bytes per
 *              split, within a quarter of the packed weight bytes; 1 otherwise.
 * BL_ERR_INVALID_ARG for null pointers or sms < 1; BL_ERR_UNSUPPORTED_SHAPE as above. */
bl_status bitlinear_debug_plan(int M, int N, int K, int sms, int* path, int* k_splits);

/* Human-readable name of a status code (static string). */
const char* bitlinear_status_string(bl_status status);

#ifdef __cplusplus
}
#endif

#endif /* BITLINEAR_H_ */
