/*
 * qlora.h -- C ABI of the int8-frozen-kernel LoRA Dense layer library
 * (libqlora.so), sm_100a.
 *
 * The layer: a Dense layer whose kernel is frozen int8 with one fp32 scale
 * per output channel, fine-tuned through a floating-point LoRA adapter
 * ("Introduce QLoRA-like technique", Keras PR 19356, Highlights: training
 * with frozen int8 weights for Dense; "Parameter-efficient fine-tuning of
 * GPT-2 with LoRA", section "LoRA equation": output = W0 x + b0 + B A x,
 * scaled by alpha / rank as in section "Create LoRA layer").
 *
 * Shapes and names (all buffers row-major and contiguous):
 *   M tokens, K in_features, N out_features, r LoRA rank, c = alpha / r
 *   W  [K,N]  fp32 float kernel (input of qlora_quantize_weight only)
 *   Wq [N,K]  int8 frozen kernel, one row per output channel (K-major)
 *   sw [N]    fp32 per-output-channel scale
 *   X  [M,K]  activations in act_dtype          Y  [M,N] act_dtype
 *   dY [M,N]  act_dtype                          dX [M,K] act_dtype
 *   A  [K,r]  fp32    B [r,N] fp32    bias [N] fp32
 *   xA [M,r]  fp32 (x . A of the unquantized input, kept for the backward)
 *   dA [K,r], dB [r,N], dbias [N]  fp32
 *
 * Quantization (the pages give no formula; this is the library's reading):
 * symmetric abs-max, s = amax / 127, q = clamp(rne(v * (127 / amax)), -127,
 * 127), IEEE fp32, one rounding per operation; amax == 0 gives q = 0, s = 0.
 *
 * Memory and ownership: every pointer argument is a DEVICE pointer owned by
 * the caller, except `d` and `dbg`, which are host pointers read during the
 * call.  The library allocates no device memory.  Scratch space is the
 * caller's `workspace` of at least qlora_workspace_bytes(d, M) bytes, 256-byte
 * aligned; its contents on entry do not matter.
 *
 * Streams: `stream` is a cudaStream_t (NULL = the legacy default stream).
 * Every call only enqueues work on `stream` and returns; QLORA_OK means the
 * launches were enqueued.  Device-side failures surface at the caller's next
 * synchronisation (cudaGetLastError) or through qlora_device_status().
 * Calls on the same stream are ordered; calls that share an output or a
 * workspace must not run concurrently on different streams.
 *
 * Errors: every call validates its arguments before launching anything and
 * then returns a negative qlora_status without touching any output.  The
 * checks are: non-NULL required pointers (EINVAL), M, K, N >= 1 and
 * 1 <= r <= 64 (ESHAPE), K a multiple of 16 (EUNSUPPORTED: the int8 rows are
 * moved by the Tensor Memory Accelerator, whose row pitch must be a multiple
 * of 16 bytes), 16-byte aligned pointers for X, Y, dY, dX, Wq, Wq_out and
 * the workspace, and 4-byte aligned fp32 vectors (EALIGN).  A CUDA error while
 * enqueuing returns ECUDA.  qlora_last_error() gives a message for the last
 * non-OK status of the calling thread.
 */
#ifndef QLORA_H
#define QLORA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    QLORA_F32 = 0,
    QLORA_BF16 = 1
} qlora_dtype;

typedef enum {
    QLORA_OK = 0,
    QLORA_EINVAL = -1,
    QLORA_EALIGN = -2,
    QLORA_ESHAPE = -3,
    QLORA_ECUDA = -4,
    QLORA_EUNSUPPORTED = -5,
    QLORA_ETIMEOUT = -6
} qlora_status;

/* One layer: in_features K, out_features N, rank r (1..64), LoRA alpha and
 * the activation dtype of X, Y, dY and dX. */
typedef struct {
    int K;
    int N;
    int r;
    float alpha;
    qlora_dtype act_dtype;
} qlora_layer_desc;

/* Optional debug outputs of qlora_forward (any member may be NULL): the
 * quantized input Xq [M,K] int8, its row scales sx [M] fp32 and the int32
 * accumulator acc [M,N] of the int8 GEMM. */
typedef struct {
    int8_t* xq;
    float* sx;
    int32_t* acc;
} qlora_debug;

/*
 * Frozen-kernel quantization, once per layer ("Introduce QLoRA-like
 * technique", Highlights and the model.quantize("int8") call of its
 * benchmark script): W [K,N] fp32 -> Wq [N,K] int8 (transposed so that
 * each output channel's K values are contiguous) and sw [N] fp32, abs-max
 * per output channel n.  Wq and sw are bit-exact with the reading above.
 */
int qlora_quantize_weight(const float* W, int K, int N, int8_t* Wq, float* sw,
                          void* stream);

/* Bytes of scratch that qlora_forward and qlora_backward need for M tokens
 * (the same workspace serves both).  Returns 0 for an invalid descriptor. */
size_t qlora_workspace_bytes(const qlora_layer_desc* d, int M);

/*
 * Forward: Y = (Xq Wq^T) * sx[m] * sw[n] + bias[n] + c * (X A) B.
 * The int8 GEMM (int32 accumulate) follows "Introduce QLoRA-like technique"
 * (Results table, int8 Dense); the LoRA term follows "Parameter-efficient
 * fine-tuning of GPT-2 with LoRA", section "LoRA equation".  Each input row
 * is quantized by abs-max (Xq, sx); the LoRA branch uses the unquantized X.
 * bias may be NULL.  xA [M,r] receives X . A (needed by qlora_backward).
 * dbg may be NULL; its non-NULL members receive Xq, sx and the int32
 * accumulator.  Y must not alias X.
 */
int qlora_forward(const qlora_layer_desc* d, int M, const void* X, const int8_t* Wq,
                  const float* sw, const float* bias, const float* A, const float* B,
                  void* Y, float* xA, void* workspace, size_t workspace_bytes,
                  const qlora_debug* dbg, void* stream);

/*
 * Backward of L with upstream gradient dY: the frozen int8 kernel receives
 * no gradient ("How to fine-tune the 4-bit model?" thread: the integer
 * weights are not changed during gradient descent), the input quantizer is
 * passed straight through:
 *   G  = dY B^T                                  [M,r]
 *   dX = dY (Wq * sw)^T + c * G A^T              [M,K]  (may be NULL)
 *   dA = c * X^T G                               [K,r]
 *   dB = c * xA^T dY                             [r,N]
 *   dbias = sum over rows of dY                  [N]    (may be NULL)
 * xA must be the one qlora_forward returned for this X.  In bf16 the
 * dequantized kernel Wq * sw is rounded to bf16 before the tensor-core
 * product; accumulation is fp32.  dA, dB and dbias are deterministic
 * (fixed reduction order, no atomics).
 * Streams: all work is ordered after earlier work on `stream`, and later
 * work on `stream` is ordered after all of it.  From 512 tokens, with dX
 * requested, the dA pass runs on a second stream of the library's (one per
 * host thread and device, created on the first such call; make that call
 * outside a global-mode stream capture) beside the dX GEMM, joined back to
 * `stream` by events; stream capture records the two branches.  If the
 * second stream cannot be created everything runs on `stream`.
 */
int qlora_backward(const qlora_layer_desc* d, int M, const void* X, const void* dY,
                   const int8_t* Wq, const float* sw, const float* A, const float* B,
                   const float* xA, void* dX, float* dA, float* dB, float* dbias,
                   void* workspace, size_t workspace_bytes, void* stream);

/* Size of the static scratch behind qlora_backward_noalloc (8 MiB per device). */
#define QLORA_NOALLOC_SCRATCH_BYTES (8 * 1024 * 1024)

/*
 * qlora_backward without a workspace argument (the pages have no counterpart:
 * it is a calling convention, not part of the method).  Same arguments,
 * results and error codes as qlora_backward, minus workspace/workspace_bytes.
 *
 * Who it is for: callers that must not allocate device memory at the point
 * of the call and hold no spare buffer to lend, e.g. code that runs inside
 * an allocator's own callbacks, a host that forbids allocation once its
 * steady state begins, or a runtime whose memory pool is already committed.
 * The scratch it needs (the per-column-block G slices of the rank-r backward)
 * is a file-scope device array of QLORA_NOALLOC_SCRATCH_BYTES reserved when
 * the library's module is loaded on a device; the call itself allocates no
 * device memory.  Nothing in the scratch has to start at zero: each call
 * writes every scratch element it reads before reading it.
 *
 * Limit: the layer needs S * M * r * 4 bytes of scratch for its S slices of
 * G (S = ceil(N/128) for bf16 layers with N a multiple of 8, else
 * ceil(N/64)), plus M * r * 4 bytes for G itself when S > 8, each part
 * rounded up to 256.  A call that needs more than QLORA_NOALLOC_SCRATCH_BYTES
 * returns QLORA_ESHAPE with a message stating both sizes, before any launch.
 * Use qlora_backward with a workspace for such layers.
 *
 * Set-up: the first call on each device (with that device current) looks up
 * the device addresses of the scratch and of the status word with
 * cudaGetSymbolAddress and caches them; a failed lookup returns QLORA_ECUDA.
 * Make the first call on a device before any stream capture begins.  The
 * cached addresses belong to the device's current context: after
 * cudaDeviceReset (or anything else that destroys that context) they are
 * stale, and this entry point must not be called again in the process.
 *
 * Concurrency: all calls on one device share the one scratch.  Calls issued
 * to the same stream are ordered and safe; calls that can overlap on the
 * device (different streams without ordering between them, or several host
 * threads) race on the scratch and give undefined results.
 */
int qlora_backward_noalloc(const qlora_layer_desc* d, int M, const void* X, const void* dY,
                           const int8_t* Wq, const float* sw, const float* A, const float* B,
                           const float* xA, void* dX, float* dA, float* dB, float* dbias,
                           void* stream);

/* ------------------------------------------------------------------------
 * Step-level entry points.  qlora_forward is qlora_quantize_input followed
 * by qlora_gemm_forward; qlora_backward is qlora_lora_grad_dy, then
 * qlora_gemm_dx, then qlora_lora_grad_x.  They are exported so that a caller
 * can schedule, overlap or time the steps one by one.  Same conventions as
 * above; M == 0 is a no-op (the gradient steps then write zeros).
 * ------------------------------------------------------------------------ */

/* a1: per-row abs-max quantization of X into Xq [M,K] int8 and sx [M] fp32
 * (bit-exact with the reading above), and xA = X . A [M,r] fp32 from the
 * same read of X ("LoRA equation": the adapter sees the layer input). */
int qlora_quantize_input(const qlora_layer_desc* d, int M, const void* X, const float* A,
                         int8_t* Xq, float* sx, float* xA, void* stream);

/* a2: Y = (Xq Wq^T) * sx[m] * sw[n] + bias[n] + c * xA B on the int8 tensor
 * cores (int32 accumulate).  bias and acc may be NULL; a non-NULL acc
 * [M,N] int32 receives the raw accumulator. */
int qlora_gemm_forward(const qlora_layer_desc* d, int M, const int8_t* Xq, const float* sx,
                       const int8_t* Wq, const float* sw, const float* bias, const float* xA,
                       const float* B, void* Y, int32_t* acc, void* stream);

/* a2 for a layer followed by a ReLU, as the hidden layers of the MLP in
 * "Introduce QLoRA-like technique" (benchmark script: Dense layers with ReLU
 * between them; the ReLU is not part of the layer): the same Y, then
 * Y = max(Y, 0) in the epilogue, bit-identical to qlora_gemm_forward followed
 * by qlora_relu, without the second pass over Y.  acc, if not NULL, still
 * receives the raw accumulator. */
int qlora_gemm_forward_relu(const qlora_layer_desc* d, int M, const int8_t* Xq, const float* sx,
                            const int8_t* Wq, const float* sw, const float* bias, const float* xA,
                            const float* B, void* Y, int32_t* acc, void* stream);

/* a3: one pass over dY: dB = c * xA^T dY [r,N] and, if dbias is not NULL,
 * dbias = column sums of dY [N]; G = dY B^T is left in the workspace (as
 * per-column-block slices) for the a4 and a5 calls that follow on the same
 * workspace, with no forward call on that workspace in between.  If G is
 * not NULL, the summed G [M,r] is also written there.  Deterministic. */
int qlora_lora_grad_dy(const qlora_layer_desc* d, int M, const void* dY, const float* B,
                       const float* xA, float* dB, float* dbias, float* G, void* workspace,
                       size_t workspace_bytes, void* stream);

/* a3 in two halves, for callers that put G on their critical path and the
 * parameter gradients on another stream:
 *   qlora_lora_g      : G = dY B^T into the workspace, exactly as
 *                       qlora_lora_grad_dy leaves it for a4 and a5;
 *   qlora_lora_grad_b : dB = c * xA^T dY [r,N] and, if dbias is not NULL,
 *                       dbias = column sums of dY [N]; touches no workspace.
 * Together they give the same results as qlora_lora_grad_dy, each with one
 * more read of dY.  Deterministic. */
int qlora_lora_g(const qlora_layer_desc* d, int M, const void* dY, const float* B,
                 void* workspace, size_t workspace_bytes, void* stream);
int qlora_lora_grad_b(const qlora_layer_desc* d, int M, const void* dY, const float* xA,
                      float* dB, float* dbias, void* stream);

/* a4: dX = dY (Wq * sw)^T + c * G A^T [M,K], G from the workspace that a3
 * filled; the int8 kernel is de-quantized tile by tile in shared memory
 * ("How to fine-tune the 4-bit model?": de-quantize in place before the
 * matrix unit). */
int qlora_gemm_dx(const qlora_layer_desc* d, int M, const void* dY, const int8_t* Wq,
                  const float* sw, const float* A, void* dX, const void* workspace,
                  size_t workspace_bytes, void* stream);

/* a4 for a layer whose input X [M,K] (act_dtype, 16-byte aligned) is the
 * output of a ReLU: dX is taken back through that ReLU as well, dX = 0 where
 * X <= 0, in the epilogue; bit-identical to qlora_gemm_dx followed by
 * qlora_relu_backward(dX, X), without the second pass over dX. */
int qlora_gemm_dx_relu(const qlora_layer_desc* d, int M, const void* dY, const int8_t* Wq,
                       const float* sw, const float* A, const void* X, void* dX,
                       const void* workspace, size_t workspace_bytes, void* stream);

/* a5: one pass over X: dA = c * X^T G [K,r], G from the workspace that a3
 * filled.  Deterministic. */
int qlora_lora_grad_x(const qlora_layer_desc* d, int M, const void* X, float* dA,
                      const void* workspace, size_t workspace_bytes, void* stream);

/* Launch policy of the column-sum passes on the tensor cores (bf16 layers):
 * the dB/dbias half of a3 (qlora_lora_grad_dy, qlora_lora_grad_b) and a5
 * (qlora_lora_grad_x).  They sum over the M rows; by default the rows of a
 * 128-column block are spread over a cluster of up to 8 CTAs, which gives
 * the lowest latency for a pass that runs alone.  rows > 0 makes every CTA
 * cover at least that many rows (rounded up to 128), so a pass occupies
 * fewer SMs for longer: the choice for passes that run on a side stream
 * beside a larger kernel that needs the SMs.  rows == 0 restores the
 * default.  Results change only by the fp32 rounding of the different
 * grouping and stay deterministic for a given setting.  Process-wide, for
 * launches made after the call (a captured graph keeps the launch shape it
 * was captured with): one value shared by every caller in the process, so a
 * caller that changes it should restore it around its own launches (the MLP
 * stack does); returns the previous setting, or QLORA_EINVAL for rows
 * outside [0, 2^24].  The pages have no counterpart. */
int qlora_set_rank_pass_rows(int rows);

/* ------------------------------------------------------------------------
 * Packed int4 frozen kernels (keras-llm-light, "Simplified Int4Variable
 * quantization": two int4 values in one int8 byte; "How to fine-tune the
 * 4-bit model?": a frozen 4-bit kernel under an fp32 LoRA, de-quantized in
 * place before the matrix unit).  Reading (the pages give no formula): the
 * int8 quantizer with 7 in place of 127, per output channel n,
 *   sw[n] = amax / 7,  q[n,k] = clamp(rne(W[k,n] * (7 / amax)), -7, 7)
 * in fp32, one rounding per operation; Wp [N, K/2] bytes, byte j of row n
 * holding q[n,2j] in its low nibble and q[n,2j+1] in its high nibble (two's
 * complement).  An int4 layer computes exactly what the int8 layer computes
 * with these codes as its Wq.  K must be a multiple of 32
 * (QLORA_EUNSUPPORTED otherwise); Wp is 16-byte aligned.
 *
 * qlora_gemm_forward_int4 and qlora_gemm_dx_int4 read the packed codes
 * directly and expand them in shared memory.  qlora_unpack_int4 gives the
 * int8 codes for the composite calls (qlora_forward, qlora_backward).
 * ------------------------------------------------------------------------ */

/* a0 for int4: W [K,N] fp32 -> Wp [N, K/2] packed codes, sw [N].  Bit-exact. */
int qlora_quantize_weight_int4(const float* W, int K, int N, uint8_t* Wp, float* sw,
                               void* stream);

/* Wp [N, K/2] -> Wq [N, K] int8 codes in [-8, 7] (Wq 16-byte aligned).  Bit-exact. */
int qlora_unpack_int4(const uint8_t* Wp, int K, int N, int8_t* Wq, void* stream);

/* a2 with packed int4 codes: the int8 GEMM and epilogue of qlora_gemm_forward
 * on the codes, which dedicated warps expand from Wp into each stage's int8
 * tile.  Bit-identical to qlora_gemm_forward given the unpacked codes.  It
 * needs no int8 copy of the kernel, but at K >= 4096 the expansion paces the
 * stages and it runs at about half the speed of qlora_gemm_forward; there,
 * qlora_unpack_int4 once followed by qlora_gemm_forward is faster. */
int qlora_gemm_forward_int4(const qlora_layer_desc* d, int M, const int8_t* Xq, const float* sx,
                            const uint8_t* Wp, const float* sw, const float* bias, const float* xA,
                            const float* B, void* Y, int32_t* acc, void* stream);

/* a4 with packed int4 codes: dX = dY (q * sw)^T + c * G A^T, the nibbles
 * de-quantized in shared memory; G from the workspace as qlora_gemm_dx.
 * Bit-identical to qlora_gemm_dx given the unpacked codes. */
int qlora_gemm_dx_int4(const qlora_layer_desc* d, int M, const void* dY, const uint8_t* Wp,
                       const float* sw, const float* A, void* dX, const void* workspace,
                       size_t workspace_bytes, void* stream);

/* a6 for int4: the merged kernel of qlora_merge (same operations, same
 * order), re-quantized per channel to int4 and packed into Wp_out [N, K/2],
 * sw_out [N].  Bit-exact.  Outputs must not alias the inputs. */
int qlora_merge_int4(const qlora_layer_desc* d, const uint8_t* Wp, const float* sw,
                     const float* A, const float* B, uint8_t* Wp_out, float* sw_out,
                     void* stream);

/* ------------------------------------------------------------------------
 * Outlier-compensated int8 kernels (keras-llm-light, "Weights
 * quantization": the weights are quantized after the outliers beyond a
 * 99.9 percentile cutoff are taken out and kept in fp16; "Simplified
 * Int8Variable quantization": the kernel is rebuilt as bias + code * scale
 * with the outliers written back, and the activations are not quantized).
 *
 * Reading (the pages give no formula): one affine code per tensor.  lo and
 * hi are the 0.1th and 99.9th percentiles of all K*N entries of W (linear
 * interpolation between the order statistics at (K*N - 1) p / 100, in fp64,
 * stored as fp32).  Entries strictly below lo or above hi are outliers,
 * kept as fp16 (round to nearest even) with code 0; scale = fl32((hi - lo) /
 * 255), bias = lo, and every other entry gets
 *   code = clamp(rne(fl32(fl32(w - bias) / scale)), 0, 255)   (0 if scale == 0).
 * The rebuilt kernel is Wr = fl32(bias + fl32(code * scale)), the fp16 value
 * at the outliers; a bf16 layer rounds Wr to bf16 before the tensor cores.
 *
 * Storage (struct qlora_outlier_kernel, all device memory owned by the caller):
 *   codes_nk [N,K] uint8 (16-byte aligned; the dX GEMM's layout)
 *   codes_kn [K,N] uint8 (16-byte aligned; the forward GEMM's layout)
 *   par [4] fp32: lo, hi, scale, bias
 *   start_nk [N * ceil(K/128) + 1] int32, ent_nk [cap] uint32: the outliers of
 *     row n, columns 128b .. 128b+127 of codes_nk are ent_nk[start_nk[n *
 *     ceil(K/128) + b] .. start_nk[n * ceil(K/128) + b + 1]), each entry
 *     (column - 128b) << 16 | fp16 bits; the order inside a bucket is not
 *     specified
 *   start_kn [K * ceil(N/128) + 1], ent_kn [cap]: the same for codes_kn
 *   cap: entries of ent_nk and of ent_kn, at least qlora_outlier_cap(K, N)
 * The layer: Y = X Wr + bias + c (X A) B; its backward as qlora_backward with
 * Wr in place of Wq * sw.  Layer constraints as for int8 layers (K a multiple
 * of 16); bf16 layers run on the tensor cores when N is a multiple of 16.
 * ------------------------------------------------------------------------ */
typedef struct {
    uint8_t* codes_nk;
    uint8_t* codes_kn;
    float* par;
    int* start_nk;
    uint32_t* ent_nk;
    int* start_kn;
    uint32_t* ent_kn;
    int cap;
} qlora_outlier_kernel;

/* Upper bound on the number of outliers of a K x N kernel (the entries
 * strictly outside the two percentiles): (i_lo + 1) + (K*N - 1 - i_hi) with
 * i = floor((K*N - 1) p / 100).  0 for an invalid shape. */
size_t qlora_outlier_cap(int K, int N);

/* Bytes of scratch that qlora_outlier_quantize needs (256-byte aligned). */
size_t qlora_outlier_workspace_bytes(int K, int N);

/* a0 for outlier-compensated kernels: W [K,N] fp32 -> every member of *q.
 * Codes, par and the set of outliers in each bucket are bit-exact with the
 * reading above.  K >= 1, N >= 1, K*N < 2^31; q is a host pointer. */
int qlora_outlier_quantize(const float* W, int K, int N, const qlora_outlier_kernel* q,
                           void* workspace, size_t workspace_bytes, void* stream);

/* Forward of an outlier-compensated layer: xA = X A [M,r], then
 * Y = X Wr + bias + c xA B, the kernel rebuilt tile by tile in shared memory
 * (codes_kn, ent_kn) in front of the tensor cores.  bias may be NULL.
 * workspace: at least qlora_workspace_bytes(d, M). */
int qlora_outlier_forward(const qlora_layer_desc* d, int M, const void* X,
                          const qlora_outlier_kernel* q, const float* bias, const float* A,
                          const float* B, void* Y, float* xA, void* workspace,
                          size_t workspace_bytes, void* stream);

/* Backward of an outlier-compensated layer: G = dY B^T, dX = dY Wr^T +
 * c G A^T (codes_nk, ent_nk; dX may be NULL), dA = c X^T G, dB = c xA^T dY,
 * dbias = column sums of dY (may be NULL).  The parameter gradients are the
 * passes of qlora_backward.  Deterministic. */
int qlora_outlier_backward(const qlora_layer_desc* d, int M, const void* X, const void* dY,
                           const qlora_outlier_kernel* q, const float* A, const float* B,
                           const float* xA, void* dX, float* dA, float* dB, float* dbias,
                           void* workspace, size_t workspace_bytes, void* stream);

/*
 * Lossy merge ("Introduce QLoRA-like technique", Results footnote: merging
 * LoRA weights into int8 kernels is lossy; "How to fine-tune the 4-bit
 * model?" thread: de-quantize, add the LoRA, re-quantize; the float merge
 * adds einsum(A, B) * alpha / rank, "Merge weights and generate text!"):
 *   W'[k,n] = fl(fl(Wq[n,k] * sw[n]) + fl(c * d)),
 *   d = A[k,0]*B[0,n] + ... + A[k,r-1]*B[r-1,n] summed in ascending j,
 * every operation a single fp32 rounding, then the per-output-channel
 * quantization of W' into Wq_out [N,K] and sw_out [N].  Bit-exact with that
 * order.  Wq_out and sw_out must not alias Wq and sw.
 */
int qlora_merge(const qlora_layer_desc* d, const int8_t* Wq, const float* sw,
                const float* A, const float* B, int8_t* Wq_out, float* sw_out,
                void* stream);

/*
 * The plain elementwise ReLU between the Dense layers of the MNIST MLP
 * ("Introduce QLoRA-like technique", benchmark.py: Dense + ReLU blocks).
 * Not part of the layer.  qlora_relu: Y[i] = max(Y[i], 0) in place, n
 * elements of `dtype`.  qlora_relu_backward: dY[i] = 0 where Y[i] <= 0 (Y is
 * the ReLU output), in place.  Device pointers; n == 0 is a no-op.
 */
int qlora_relu(void* Y, size_t n, qlora_dtype dtype, void* stream);
int qlora_relu_backward(void* dY, const void* Y, size_t n, qlora_dtype dtype, void* stream);

/*
 * Axis permutation of a row-major tensor (EinsumDense layouts: "Introduce
 * float8 training", the speed test's "abcde,aebf->adbcf"; an equation whose
 * operands are not a plain reshape of a Dense layer's is brought to
 * [batch, kept, contracted] order before the layer and back after it).
 * src has `ndim` (1..8) axes of extents shape[]; dst axis d is src axis
 * perm[d], i.e. dst[i_0, .., i_{ndim-1}] = src[j] with j_{perm[d]} = i_d.
 * elem_bytes is 1, 2, 4 or 8; both buffers are device memory aligned to it
 * and must not overlap.  Bit-exact (a copy).
 */
int qlora_permute(const void* src, void* dst, int ndim, const int64_t* shape, const int* perm,
                  int elem_bytes, void* stream);

/* ------------------------------------------------------------------------
 * The float8 training recipe ("Introduce float8 training", Keras PR 19488:
 * quantization mode "float8", per-tensor scale and amax_history updated
 * every step, the output-gradient scale, float8 matmuls on float8 tensor
 * cores).  The page gives no formula; the library's reading:
 *   formats   inputs and kernel E4M3 (largest finite 448), the output
 *             gradient E5M2 (largest finite 57344); codes as uint8
 *   quantize  q = fp8(satfinite(fl32(T / s))), round to nearest, ties to
 *             even, s the scale stored by the previous step (delayed
 *             scaling)
 *   state     after quantizing, s' = fl32(h / fp8_max) with h the largest
 *             entry of the amax history before this step (s' = s when h is
 *             0 or not finite), and the history becomes
 *             [amax(|T|), H[0], .., H[L-2]] (newest first, oldest dropped)
 *   layer     Y = (Xq Wq) s_x s_w + bias, dX = (dYq Wq^T) s_g s_w,
 *             dW = (Xq^T dYq) s_x s_g, dbias = column sums of dY
 * ------------------------------------------------------------------------ */
typedef enum { QLORA_FP8_E4M3 = 0, QLORA_FP8_E5M2 = 1 } qlora_fp8_format;

/* Scratch of qlora_fp8_quantize (one word; 256 for alignment). */
#define QLORA_FP8_WORKSPACE_BYTES 256

/* Quantizes T [rows, cols] (dtype) with the scale *scale_in into q [rows,
 * cols] and, if qt is not NULL, its transpose qt [cols, rows] (the K-major
 * operand of the backward GEMMs), then writes the next scale to *scale_out
 * and updates amax_history [history_len] in place, as above.  scale_in,
 * scale_out and amax_history are device memory; scale_out must not alias
 * scale_in (keep two and swap them every step).  Codes, scale and history
 * are bit-exact with the reading above. */
int qlora_fp8_quantize(const void* T, int rows, int cols, qlora_dtype dtype, qlora_fp8_format fmt,
                       const float* scale_in, float* scale_out, float* amax_history, int history_len,
                       uint8_t* q, uint8_t* qt, void* workspace, size_t workspace_bytes, void* stream);

/* Bytes of workspace qlora_fp8_quantize_colsum needs for T [rows, cols]
 * (0 for an empty shape). */
size_t qlora_fp8_colsum_workspace_bytes(int rows, int cols);

/* qlora_fp8_quantize plus colsum[c] = sum_r T[r, c] in fp32 (the bias
 * gradient when T is the output gradient dY), read in the same pass as the
 * codes.  The sum's order is fixed (within each 128-row tile, then over the
 * tiles by a second, small kernel), so repeated calls give the same bits.  Needs T
 * 16-byte aligned, cols % 8 == 0, q 8-byte aligned and qt NULL or 16-byte
 * aligned with rows % 16 == 0 (else QLORA_EUNSUPPORTED); workspace: device
 * memory, 256-byte aligned, of at least
 * qlora_fp8_colsum_workspace_bytes(rows, cols) bytes. */
int qlora_fp8_quantize_colsum(const void* T, int rows, int cols, qlora_dtype dtype, qlora_fp8_format fmt,
                              const float* scale_in, float* scale_out, float* amax_history, int history_len,
                              uint8_t* q, uint8_t* qt, float* colsum, void* workspace, size_t workspace_bytes,
                              void* stream);

/* C [M,N] = (A B^T) * (*scale_a) * (*scale_b) (+ bias[n]), A [M,K] and
 * B [N,K] float8 codes (both K-major, K a multiple of 16), products on
 * tcgen05.mma.kind::f8f6f4 with fp32 accumulation; C in c_dtype (bf16
 * rounded to nearest even).  bias may be NULL; scales are device pointers.
 * A, B and C 16-byte aligned. */
int qlora_fp8_gemm(const uint8_t* A, qlora_fp8_format fmt_a, const uint8_t* B, qlora_fp8_format fmt_b,
                   int M, int N, int K, const float* scale_a, const float* scale_b, const float* bias,
                   void* C, qlora_dtype c_dtype, void* stream);

/* Bytes of workspace qlora_fp8_gemm_ws uses at this shape on the current
 * device (0: it would not split; then it is qlora_fp8_gemm). */
size_t qlora_fp8_gemm_workspace_bytes(int M, int N, int K);

/* qlora_fp8_gemm with a workspace (device memory, 256-byte aligned; NULL or
 * too small: no split).  On CTA pairs, when the 256 x 256 output tiles leave
 * the pairs a partial last wave, that wave's tiles are computed as two halves
 * of the contraction each (one wave of half the length) and a second kernel
 * adds the halves' fp32 accumulators (in either order the same sum), scales
 * and adds the bias.  Results are deterministic; their fp32 sums are grouped
 * differently from qlora_fp8_gemm's on those tiles. */
int qlora_fp8_gemm_ws(const uint8_t* A, qlora_fp8_format fmt_a, const uint8_t* B, qlora_fp8_format fmt_b,
                      int M, int N, int K, const float* scale_a, const float* scale_b, const float* bias,
                      void* C, qlora_dtype c_dtype, void* workspace, size_t workspace_bytes, void* stream);

/* Message for the last non-OK status returned on the calling thread. */
const char* qlora_last_error(void);

/*
 * Synchronises `stream`, then reads and clears the library's device status
 * word on the current device: QLORA_OK, or QLORA_ETIMEOUT if a kernel gave up
 * a bounded wait (its outputs are then unspecified), or QLORA_ECUDA if the
 * synchronisation itself failed.
 */
int qlora_device_status(void* stream);

/*
 * Failure-path self test (no counterpart on the pages).  Enqueues one tiny
 * kernel whose bounded wait on a barrier that nothing signals gives up after
 * limit_us microseconds (1 .. 2e6) and records QLORA_ETIMEOUT in the device
 * status word, exactly as a stalled pipeline in the GEMM kernels would; the
 * kernel then exits normally and the context stays usable.  The following
 * qlora_device_status() returns QLORA_ETIMEOUT and clears the word.
 */
int qlora_selftest_wait_timeout(unsigned int limit_us, void* stream);

/* Library version, e.g. "qlora-b200 0.1 sm_100a". */
const char* qlora_version(void);

#ifdef __cplusplus
}
#endif

#endif /* QLORA_H */
