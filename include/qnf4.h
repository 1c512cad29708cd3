/*
 * qnf4.h -- C ABI of libqnf4.so: a B200 (sm_100a) library for the QLoRA-style
 * NF4-quantized linear layer.
 *
 * Sources (page title, section):
 *   [QLoRA]  "QLoRA: Efficient Finetuning of Quantized LLMs" (Heng's Blog):
 *            opening formula h = dequant(W0^NF4) x + (alpha/r) B A x;
 *            贡献一 4-bit NormalFloat (NF4); 贡献二 Double Quantization.
 *   [AQLoRA] "AQLoRA: a zero-search scheme for fast quantized LoRA fine-tuning",
 *            §3.1 profiling pass (blockwise NF4 reconstruction error).
 *   [LowRA]  "LowRA" article (cloud.tencent.com.cn), §4.1 per-output-channel
 *            quantization, group normalisation, thresholds and mappings (Fig. 3).
 *
 * Conventions shared by every entry point:
 *   - All buffers are allocated and owned by the caller. The library never
 *     allocates or frees device memory and never synchronises the stream, except
 *     qnf4_check(), which synchronises to read the device error flag, and
 *     qnf4_loftq_nf4(), whose first call on a device creates cuBLAS / cuSOLVER handles.
 *   - Pointers are device pointers unless the comment says "host".
 *   - Every device pointer must be 16-byte aligned (QNF4_ERR_ALIGN otherwise).
 *   - Matrices are row-major. W0 is [N, K] (N output features, K input features),
 *     x is [M, K] (M tokens), A is [r, K], B is [N, r], h is [M, N].
 *   - bf16 buffers are passed as void*; fp32 as float*.
 *   - K must be a multiple of 64 (QNF4_ERR_SHAPE otherwise). block1 must be 64 and
 *     block2 256 (the sizes the QLoRA page fixes); other values give QNF4_ERR_ARG.
 *   - Arguments are validated on the host before any launch; a bad argument returns
 *     without touching the GPU. A launch failure returns QNF4_ERR_CUDA. A kernel
 *     whose bounded wait gives up sets a device flag that qnf4_check() reports as
 *     QNF4_ERR_TIMEOUT. qnf4_last_error() gives a message for the calling thread.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL is the legacy default
 *     stream) and is asynchronous to the host.
 *   - Workspace: entry points with (ws, ws_bytes) need at least
 *     qnf4_workspace_size(op, ...) bytes of device scratch (QNF4_ERR_WORKSPACE
 *     otherwise). The contents need not be initialised. Calls that share a
 *     workspace must be ordered on one stream.
 */
#ifndef QNF4_H
#define QNF4_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define QNF4_API __attribute__((visibility("default")))
#else
#define QNF4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  QNF4_OK = 0,
  QNF4_ERR_ARG = 1,
  QNF4_ERR_SHAPE = 2,
  QNF4_ERR_ALIGN = 3,
  QNF4_ERR_CUDA = 4,
  QNF4_ERR_TIMEOUT = 5,
  QNF4_ERR_WORKSPACE = 6,
  QNF4_ERR_BOUNDS = 7   /* checked build (libqnf4_checked.so) only: a kernel index was
                           outside its buffer; the access was skipped (see qnf4_check) */
} qnf4_status;

/* Output dtype selector for qnf4_dequant. */
enum { QNF4_OUT_F32 = 0, QNF4_OUT_BF16 = 1 };

/* Operation selector for qnf4_workspace_size. */
enum {
  QNF4_OP_QUANTIZE = 0,     /* qnf4_nf4_quantize (with sse) and qnf4_nf4_recon_error */
  QNF4_OP_DOUBLE_QUANT = 1, /* qnf4_double_quant                                    */
  QNF4_OP_FWD = 2,          /* qnf4_qlora_linear_fwd, qnf4_dense_linear_fwd          */
  QNF4_OP_BWD = 3,          /* qnf4_qlora_linear_bwd, qnf4_dense_linear_bwd          */
  QNF4_OP_CHANQ_FWD = 4,    /* qnf4_chanq_linear_fwd                                 */
  QNF4_OP_CHANQ_BWD = 5,    /* qnf4_chanq_linear_bwd                                 */
  QNF4_OP_LOFTQ = 6,        /* qnf4_loftq_nf4                                        */
  QNF4_OP_LAYER_STATS = 7,  /* qnf4_nf4_layer_stats                                  */
  QNF4_OP_QUANTIZE_WEIGHT = 8, /* qnf4_quantize_weight                               */
  QNF4_OP_QUANTIZE_WEIGHT_GROUP = 9, /* qnf4_quantize_weight_group (any shapes)       */
  QNF4_OP_LAYER_STATS_GROUP = 10 /* qnf4_nf4_layer_stats_group (any shapes)           */
};

/* A double-quantized NF4 weight [QLoRA 贡献一/贡献二]. All pointers are device
 * pointers owned by the caller.
 *   packed : uint8 [N*K/2]. Row-major flattened codes; element 2j in the high nibble
 *            of byte j, element 2j+1 in the low nibble.
 *   code2  : uint8 [nb1], nb1 = N*K/64. OCP FP8 E4M3 code of each first-level
 *            constant minus the tensor mean, divided by its 256-block scale.
 *   scale2 : fp32 [nb2], nb2 = ceil(nb1/256). absmax of (c - mean) over the block / 448.
 *   mean   : fp32 [1]. The tensor mean of the first-level constants.
 * The first-level constant of block b is restored as fma(e4m3(code2[b]),
 * scale2[b/256], mean); weight i of block b as levels[code_i] * that constant. */
typedef struct {
  int64_t N, K;
  int32_t block1; /* 64  */
  int32_t block2; /* 256 */
  const uint8_t* packed;
  const uint8_t* code2;
  const float* scale2;
  const float* mean;
} qnf4_weight;

/* [QLoRA 贡献一] The 16 NF4 levels (sorted, exact 0 at index 7, -1 and +1 at the
 * ends) and the 15 fp32 decision thresholds: threshold k is the smallest fp32
 * strictly above the exact midpoint of levels k and k+1, so that
 * code = #{k : x >= threshold[k]} is the nearest level with ties to the lower one.
 * Levels come from 9 (positive) and 8 (negative) evenly spaced probabilities
 * between 1 - (1/32 + 1/30)/2 and 1/2, through the inverse normal CDF, the shared
 * zero kept once, normalised by the largest magnitude and rounded once to fp32.
 * Host pointers; either may be NULL. Never fails once the library is loaded. */
QNF4_API qnf4_status qnf4_nf4_codebook(float levels[16], float thresholds[15]);

/* [QLoRA 贡献一] Blockwise NF4 quantization of a bf16 weight W [N, K].
 * For each 64-element block b of the row-major flattened W:
 *   absmax[b] = max |w| (fp32, exact); x = fp32(w / absmax[b]) (IEEE division);
 *   code = #{k : x >= threshold[k]}; an all-zero block gets absmax 0 and code 7.
 * Outputs: packed uint8 [N*K/2] (nibble order as in qnf4_weight), absmax fp32
 * [N*K/64]. If sse is not NULL it receives (device, 1 double) the sum over all
 * elements of (w - fp32(levels[code] * absmax))^2, the single-level round-trip
 * error [AQLoRA §3.1]; then ws must hold qnf4_workspace_size(QNF4_OP_QUANTIZE,...). */
QNF4_API qnf4_status qnf4_nf4_quantize(const void* W_bf16, int64_t N, int64_t K, int32_t block1,
                              uint8_t* packed, float* absmax, double* sse,
                              void* ws, size_t ws_bytes, void* stream);

/* [QLoRA 贡献二] Double quantization of the first-level constants absmax [nb1].
 *   mean = fp32(float64 sum of absmax / nb1), one per tensor, written to mean[0];
 *   for each 256-block j: scale2[j] = fp32(max_b |absmax[b] - mean| / 448);
 *   code2[b] = E4M3 round-to-nearest-even, saturating, of fp32((absmax[b]-mean)/scale2[j]).
 *   A block whose mean-subtracted constants are all zero stores scale2 0, code2 0.
 * Outputs are device buffers: code2 uint8 [nb1], scale2 fp32 [ceil(nb1/256)],
 * mean fp32 [1]. */
QNF4_API qnf4_status qnf4_double_quant(const float* absmax, int64_t nb1, int32_t block2,
                              uint8_t* code2, float* scale2, float* mean,
                              void* ws, size_t ws_bytes, void* stream);

/* [QLoRA 贡献一 + 贡献二; AQLoRA §3.1] The whole quantization of a bf16 weight [N, K] in two
 * launches: packed NF4 codes and fp32 absmax (as qnf4_nf4_quantize), code2 / scale2 / mean
 * (as qnf4_double_quant, bit for bit: the tensor mean's float64 sum is exact) and, when sse
 * is not NULL, the reconstruction SSE (as qnf4_nf4_quantize's, bit for bit). The quantizer
 * hands the constant sums to the encoder, which also folds the SSE. N, K > 0, K a multiple
 * of 64. Workspace: QNF4_OP_QUANTIZE_WEIGHT. */
QNF4_API qnf4_status qnf4_quantize_weight(const void* W_bf16, int64_t N, int64_t K, uint8_t* packed,
                                 float* absmax, uint8_t* code2, float* scale2, float* mean,
                                 double* sse, void* ws, size_t ws_bytes, void* stream);

/* [QLoRA 贡献一 + 贡献二; AQLoRA §3.1] qnf4_quantize_weight for n (1..8) independent weights
 * in two launches, whose work forms one list (so a set of layers streams as one matrix
 * would). Host arrays of n entries: W[l] (bf16 [N[l], K[l]], device), N[l], K[l] (> 0, K[l]
 * a multiple of 64), the device outputs packed[l], absmax[l], code2[l], scale2[l], mean[l]
 * as qnf4_quantize_weight's, and sse (NULL for none, else n device pointers to one double
 * each). Every output but the SSE equals qnf4_quantize_weight's bit for bit; each SSE is the
 * same float64 sum of fp32 block sums, grouped differently (equal up to float64 rounding).
 * Workspace: qnf4_workspace_size(QNF4_OP_QUANTIZE_WEIGHT_GROUP, 0, 0, 0, 0). */
QNF4_API qnf4_status qnf4_quantize_weight_group(int32_t n, const void* const* W, const int64_t* N,
                                       const int64_t* K, uint8_t* const* packed, float* const* absmax,
                                       uint8_t* const* code2, float* const* scale2, float* const* mean,
                                       double* const* sse, void* ws, size_t ws_bytes, void* stream);

/* [QLoRA 贡献二] A matrix quantized as row shards (one per process): the tensor mean needs
 * the float64 sum of all its constants. qnf4_dq_sum writes this shard's sum to *sum (device,
 * 1 double; workspace QNF4_OP_DOUBLE_QUANT); the caller adds the shards' sums (an exact
 * all-reduce: bf16-derived constants sum exactly in float64) and passes the total and the
 * matrix's constant count to qnf4_double_quant_shard, which encodes this shard's nb1
 * constants exactly as qnf4_double_quant encodes them inside the whole matrix, provided the
 * shard starts on a 256-constant boundary (its rows a multiple of 256 / gcd(256, K / 64)).
 * Outputs are the shard's slices of code2 / scale2, and the (global) mean. */
QNF4_API qnf4_status qnf4_dq_sum(const float* absmax, int64_t nb1, double* sum, void* ws,
                        size_t ws_bytes, void* stream);
QNF4_API qnf4_status qnf4_double_quant_shard(const float* absmax, int64_t nb1, int32_t block2,
                                    const double* total_sum, int64_t total_count,
                                    uint8_t* code2, float* scale2, float* mean, void* stream);

/* [QLoRA opening formula, 贡献二] Two-level dequantization of a whole weight to
 * out [N, K] as fp32 (out_dtype QNF4_OUT_F32) or bf16 round-to-nearest-even
 * (QNF4_OUT_BF16). Meant for tests and export: the linear layer never writes the
 * dequantized weight to memory. */
QNF4_API qnf4_status qnf4_dequant(const qnf4_weight* w, void* out, int32_t out_dtype, void* stream);

/* [QLoRA opening formula] h = x * bf16(W_hat)^T + scale * (x A^T) B^T, with W_hat
 * the two-level dequantized NF4 weight, fp32 accumulation, h written as bf16 [M, N].
 * x [M, K], A [r, K], B [N, r] are bf16. scale is alpha/r (or any adapter scale,
 * e.g. rank-stabilised). 1 <= r <= 64. M >= 0 (M = 0 is a no-op). */
QNF4_API qnf4_status qnf4_qlora_linear_fwd(const qnf4_weight* w, const void* x, int64_t M,
                                  const void* A, const void* B, int32_t r, float scale,
                                  void* h, void* ws, size_t ws_bytes, void* stream);

/* [QLoRA opening formula] The forward of n (1..8) independent layers at decode sizes
 * (1 <= M <= 16 tokens) in one launch pair: layer l computes h[l] = x[l] bf16(W_hat_l)^T
 * + scale (x[l] A[l]^T) B[l]^T exactly as qnf4_qlora_linear_fwd does for it (each row's
 * arithmetic is the same, so the results are bit-identical to n separate calls). All
 * layers share M, r and scale; w is an array of n weights, x, A, B and h host arrays of
 * n device pointers with each layer's own shapes (as for the single call). The launch
 * spreads the layers' weight rows over the SMs by bytes, so small layers do not leave
 * SMs idle. ws must hold the sum over the layers of
 * qnf4_workspace_size(QNF4_OP_FWD, N_l, K_l, M, r). Errors: QNF4_ERR_ARG for n outside
 * 1..8 or NULL arrays, QNF4_ERR_SHAPE for M outside 1..16, and each layer's checks of the
 * single call. */
QNF4_API qnf4_status qnf4_qlora_linear_fwd_group(int32_t n, const qnf4_weight* w,
                                                 const void* const* x, int64_t M,
                                                 const void* const* A, const void* const* B,
                                                 int32_t r, float scale, void* const* h,
                                                 void* ws, size_t ws_bytes, void* stream);

/* The forward above without a workspace argument, for callers that cannot allocate
 * device memory: code that runs where cudaMalloc is unavailable or forbidden (an
 * allocator callback, a host hook inside a pre-planned inference engine, a caller
 * that owns no device allocator). The pages have no counterpart; this is a library
 * convenience. The workspace is a file-scope device array of 32 MiB in this library,
 * held by every GPU that loads it until the process exits. Shapes whose workspace
 * (qnf4_workspace_size(QNF4_OP_FWD, N, K, M, r)) exceeds 32 MiB are rejected with
 * QNF4_ERR_WORKSPACE before any launch; on a 148-SM B200 every N, K and r <= 64 fits
 * up to M = 65536 tokens (the split-K partial tiles take at most 19.4 MB, the bf16
 * adapter projection 128 bytes per token). The first call on a device looks up the
 * array's device address (once per device); make that first call before any stream
 * capture. All calls share the one array and it keeps the last call's contents, so
 * calls that overlap on the GPU (concurrent streams, or devices sharing a context)
 * race; calls ordered on one stream are safe. It runs the same kernels with the same
 * tiling as qnf4_qlora_linear_fwd, so its results are bit-identical to that call's. */
QNF4_API qnf4_status qnf4_qlora_linear_fwd_noalloc(const qnf4_weight* w, const void* x, int64_t M,
                                                   const void* A, const void* B, int32_t r,
                                                   float scale, void* h, void* stream);

/* [QLoRA opening formula: gradients reach only A and B through the frozen base]
 * Given dY [M, N] bf16:
 *   v  = dY B                          (fp32, internal)
 *   dX = dY bf16(W_hat) + scale v A    bf16 [M, K]
 *   dA = scale v^T x                   fp32 [r, K]   (written, not accumulated)
 *   dB = scale dY^T (x A^T)            fp32 [N, r]   (written, not accumulated)
 * There is no gradient for the frozen base. */
QNF4_API qnf4_status qnf4_qlora_linear_bwd(const qnf4_weight* w, const void* x, const void* dY,
                                  int64_t M, const void* A, const void* B, int32_t r,
                                  float scale, void* dX, float* dA, float* dB,
                                  void* ws, size_t ws_bytes, void* stream);

/* [AQLoRA §3.1] Per-layer NF4 reconstruction error of a bf16 weight [N, K]:
 * sse (device, 1 double) = sum over 64-blocks b of ||b - absmax-NF4^-1(absmax-NF4(b))||^2,
 * single-level (no double quantization), fp32 dequant values, float64 accumulation.
 * The caller divides by N*K for epsilon and ranks layers (qnf4_rank_topk). */
QNF4_API qnf4_status qnf4_nf4_recon_error(const void* W_bf16, int64_t N, int64_t K, int32_t block1,
                                 double* sse, void* ws, size_t ws_bytes, void* stream);

/* [AQLoRA §3.1] Both statistics of the profiling pass in one read of a bf16 weight [N, K]:
 * sse (device, 1 double) exactly as qnf4_nf4_recon_error, and below (device, 1 double) =
 * #{elements with |w| < tau}, an exact integer; the layer's sparsity is below / (N K).
 * The page's tau is 0.01: pass 0.01f (for bf16 weights the same test as the real 0.01).
 * K a multiple of 64, tau finite and >= 0. Workspace: QNF4_OP_LAYER_STATS. */
QNF4_API qnf4_status qnf4_nf4_layer_stats(const void* W, int64_t N, int64_t K, float tau,
                                 double* sse, double* below, void* ws, size_t ws_bytes,
                                 void* stream);

/* [AQLoRA §3.1] The profiling pass over n (1..8) independent weights in one read of each
 * (one quantizer launch over all of them, then the sums): sse[l] (device, 1 double) as
 * qnf4_nf4_recon_error's for weight l, and, when below is not NULL, below[l] (device, 1
 * double) = #{elements of weight l with |w| < tau} as qnf4_nf4_layer_stats's (tau finite and
 * >= 0; ignored when below is NULL). Host arrays of n entries: W (bf16 [N[l], K[l]],
 * device), N, K (> 0, K[l] a multiple of 64), sse, below. The counts equal the single calls';
 * each SSE equals them up to float64 rounding (its partials are grouped differently).
 * Workspace: qnf4_workspace_size(QNF4_OP_LAYER_STATS_GROUP, 0, 0, 0, 0). */
QNF4_API qnf4_status qnf4_nf4_layer_stats_group(int32_t n, const void* const* W, const int64_t* N,
                                       const int64_t* K, float tau, double* const* sse,
                                       double* const* below, void* ws, size_t ws_bytes,
                                       void* stream);

/* [AQLoRA abstract, §3.1] Host helper: indices of the k layers with the largest
 * epsilon = sse[i] / n_params[i], in descending order, ties to the lower index.
 * Host pointers; out holds k entries. */
QNF4_API qnf4_status qnf4_rank_topk(const double* sse, const int64_t* n_params, int32_t n_layers,
                           int32_t k, int32_t* out);

/* [AQLoRA abstract: protected layers stay 16-bit and skip dequantization] Dense
 * bf16 variants of the linear layer for those layers: W_bf16 [N, K] replaces the
 * NF4 weight; everything else is as in qnf4_qlora_linear_fwd / _bwd. */
QNF4_API qnf4_status qnf4_dense_linear_fwd(const void* W_bf16, int64_t N, int64_t K, const void* x,
                                  int64_t M, const void* A, const void* B, int32_t r,
                                  float scale, void* h, void* ws, size_t ws_bytes,
                                  void* stream);
QNF4_API qnf4_status qnf4_dense_linear_bwd(const void* W_bf16, int64_t N, int64_t K, const void* x,
                                  const void* dY, int64_t M, const void* A, const void* B,
                                  int32_t r, float scale, void* dX, float* dA, float* dB,
                                  void* ws, size_t ws_bytes, void* stream);

/* [LowRA §4.1, Fig. 3] Per-output-channel threshold quantization of W [N, K] bf16.
 * Row i uses bits[i] in {1, 2, 4} and its 2^b - 1 sorted fp32 bin edges
 * thr[thr_off[i] .. thr_off[i+1]). Per 64-element group: absmax[g] = max |w|;
 * x = fp32(w / absmax[g]) (0 for an all-zero group); code = #{k : x > edge_k}.
 * Row i's codes are written MSB-first, b bits each, at packed + row_off[i]
 * (row_off [N+1] int64 byte offsets, row_off[i+1] - row_off[i] = K*b/8).
 * bits, thr, thr_off, row_off are device pointers; absmax is fp32 [N*K/64]. */
QNF4_API qnf4_status qnf4_chanq_quantize(const void* W_bf16, int64_t N, int64_t K, const uint8_t* bits,
                                const float* thr, const int64_t* thr_off, uint8_t* packed,
                                const int64_t* row_off, float* absmax, void* stream);

/* [LowRA §3 (per-channel dequant kernel used in fine-tuning), §4.1] Forward of the
 * linear layer over a per-channel quantized base:
 *   w_hat[i, j] = fp32(map[map_off[i] + code_ij] * absmax[group]), rounded to bf16,
 *   h = x w_hat^T + scale (x A^T) B^T, fp32 accumulation, h bf16 [M, N].
 * map fp32 with 2^bits[i] entries per row at map_off[i] (map_off [N+1] int64). */
QNF4_API qnf4_status qnf4_chanq_linear_fwd(const uint8_t* packed, const int64_t* row_off,
                                  const uint8_t* bits, const float* map, const int64_t* map_off,
                                  const float* absmax, int64_t N, int64_t K, const void* x,
                                  int64_t M, const void* A, const void* B, int32_t r, float scale,
                                  void* h, void* ws, size_t ws_bytes, void* stream);

/* [LowRA §3 (the per-channel dequantization used in fine-tuning), QLoRA's
 * backward through the frozen base] Backward of the linear layer over a per-channel
 * quantized base (the same inputs as qnf4_chanq_linear_fwd, plus dY [M, N] bf16):
 *   v  = dY B,
 *   dX = dY bf16(w_hat) + scale v A        bf16 [M, K]
 *   dA = scale v^T x                       fp32 [r, K]
 *   dB = scale dY^T (x A^T)                fp32 [N, r]
 * with w_hat as in qnf4_chanq_linear_fwd; no gradient for the frozen base. N must be
 * a multiple of 8. The workspace (qnf4_workspace_size with QNF4_OP_CHANQ_BWD) also
 * holds the codes widened to 4 bits and the rows' 16-entry tables, rebuilt each call.
 * dA and dB are written, not accumulated; M = 0 writes them as zeros. */
QNF4_API qnf4_status qnf4_chanq_linear_bwd(const uint8_t* packed, const int64_t* row_off,
                                  const uint8_t* bits, const float* map, const int64_t* map_off,
                                  const float* absmax, int64_t N, int64_t K, const void* x,
                                  const void* dY, int64_t M, const void* A, const void* B,
                                  int32_t r, float scale, void* dX, float* dA, float* dB,
                                  void* ws, size_t ws_bytes, void* stream);

/* [LowRA 第五部分 (the mapping and threshold learner), with the §4.1 group normalisation]
 * Weighted Lloyd-Max learning of every row's mapping and thresholds at one bit width.
 * W_bf16 [N, K] (K a multiple of 64, at most 32768); bits in {1, 2, 4}; thr0 the 2^b - 1
 * initial thresholds shared by all rows (device, fp32, ascending: 0.0 for 1 bit, the
 * NormalFloat midpoints for 2 and 4 bits in the page's scheme); iters >= 1 the cap.
 * Per row, values x = fp32(w / g) weighted by their 64-group absmax g; each iteration
 * assigns x to bin #{k : x > t_k}, sets each centre to its bin's weighted mean (float64
 * sums, rounded to fp32; an empty bin keeps its centre) and each threshold to the fp32
 * midpoint of its neighbours, and the learner stops once the weighted error no longer
 * decreases. Outputs (device): map fp32 [N, 2^b], thr fp32 [N, 2^b - 1] (the last
 * tables), err float64 [N] = mean over the row of (w - fp32(map[c] g))^2 with c from
 * thr (the channel's quantization error, e.g. for a precision allocation), and
 * iters_done int32 [N] (or NULL). Deterministic. */
QNF4_API qnf4_status qnf4_chanq_learn(const void* W_bf16, int64_t N, int64_t K, int32_t bits,
                             const float* thr0, int32_t iters, float* map, float* thr,
                             double* err, int32_t* iters_done, void* stream);

/* [LowRA workflow: quantize, take the quantization error, initialise the low-rank tensors
 * with LoftQ, five alternating steps; QLoRA's NF4 + double quantization as the quantizer]
 * With A = 0, B = 0 at the start, each step: Q = dequant(NF4 + double quant(bf16(W - B A)))
 * into packed / code2 / scale2 / mean (the qnf4_weight layout of qnf4_nf4_quantize and
 * qnf4_double_quant); R = W - Q; B = U S^(1/2), A = S^(1/2) V^T from the rank-r truncated
 * SVD U S V^T of R; errs[t] = ||W - Q - B A||_F^2 (float64, the discarded squared singular
 * values). The SVD goes through the Gram matrix of R in fp32 (cuBLAS sgemm, cuSOLVER syevd,
 * loaded at first use: QNF4_ERR_CUDA if they are absent; the first call on a device creates
 * one handle of each, owned by the library for the process, and sets them to `stream`, so
 * concurrent calls on different streams must not overlap). W_bf16 [N, K], K a multiple of 64,
 * 1 <= r <= min(N, K), min(N, K) <= 16384, steps >= 1. Outputs (device): the last step's
 * quantized base, A fp32 [r, K], B fp32 [N, r], errs [steps]. Workspace: QNF4_OP_LOFTQ. */
QNF4_API qnf4_status qnf4_loftq_nf4(const void* W_bf16, int64_t N, int64_t K, int32_t r,
                           int32_t steps, uint8_t* packed, uint8_t* code2, float* scale2,
                           float* mean, float* A, float* B, double* errs, void* ws,
                           size_t ws_bytes, void* stream);

/* Bytes of device workspace an operation needs for these sizes (0 if none). */
QNF4_API size_t qnf4_workspace_size(int32_t op, int64_t N, int64_t K, int64_t M, int32_t r);

/* Synchronise `stream`, then report and clear the device error flag: QNF4_OK, or
 * QNF4_ERR_TIMEOUT if a bounded wait inside a kernel gave up since the last check,
 * QNF4_ERR_BOUNDS (checked build only) if a kernel index fell outside its buffer,
 * or QNF4_ERR_CUDA if the stream holds a CUDA error or a LoftQ eigensolve reported
 * failure (cuSOLVER info != 0). */
QNF4_API qnf4_status qnf4_check(void* stream);

/* Upper bound, in nanoseconds, on any single wait inside a kernel before it gives
 * up with QNF4_ERR_TIMEOUT (default 1e9). Applies to kernels launched afterwards. */
QNF4_API qnf4_status qnf4_set_wait_timeout_ns(uint64_t ns);

/* Number of kernels this library has launched in this process (all threads, all
 * devices). Memsets are not counted. For benchmarks that report their launches. */
QNF4_API unsigned long long qnf4_launch_count(void);

/* Profiling hook. While set (non-NULL), every linear forward / backward call made
 * from the calling thread records the cudaEvent_t `start` on its stream right before
 * launching its dequant-GEMM kernel (the forward h GEMM, or the backward dX GEMM)
 * and `stop` right after it, so the caller can time that kernel alone. Both or
 * neither (NULL, NULL turns it off). The events are owned by the caller. */
QNF4_API qnf4_status qnf4_set_timing_events(void* start, void* stop);

/* Message describing the last error returned on the calling thread. */
QNF4_API const char* qnf4_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* QNF4_H */
