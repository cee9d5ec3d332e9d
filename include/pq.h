/*
 * pq.h - C ABI of the B200 (sm_100a) ParetoQ-style weight fake-quantizer.
 *
 * The library quantizes the fp32 "shadow" weights of one linear layer per
 * call, the way quantization-aware training does on every forward, and runs
 * the matching straight-through-estimator backward. All arithmetic runs in
 * CUDA kernels for sm_100a; there is no CPU fallback.
 *
 * Notation (one weight matrix):
 *   W      fp32 [rows, cols], row-major, contiguous; rows = output channels
 *   alpha  fp32 [rows], the learnable per-output-channel scale
 *   x      fl(w / alpha), IEEE fp32 division
 *   G      upstream gradient dWq, bf16 [rows, cols], row-major
 *
 * Conventions shared by every entry point:
 *   - All array arguments are DEVICE pointers owned by the caller. The
 *     library allocates nothing and keeps no state between calls.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL is the legacy
 *     default stream) and the call returns after the launch. Outputs are
 *     ready when the stream reaches that point.
 *   - rows == 0 or cols == 0 is valid and launches nothing (array pointers
 *     may then be NULL), except that the backward writes d(alpha) = 0 for
 *     rows > 0, cols == 0 (dalpha_out must then be valid).
 *   - Any alignment is accepted. The fast path needs cols % 8 == 0, 32-byte
 *     aligned fp32 arrays (weights, dW, moments), 16-byte aligned bf16 arrays
 *     and a packed buffer aligned to 2 bytes (2-bit codes) or 4 bytes (4-bit
 *     codes); otherwise a slower element path with the same results runs.
 *   - Preconditions not checked on the device: w finite, alpha finite and
 *     > 0, and output buffers that alias no input. Violations give
 *     unspecified results (no fault for in-bounds buffers).
 *   - Outputs are overwritten, never accumulated into. The same inputs give
 *     the same output bits on every run (fixed reduction order).
 *   - Errors: arguments are checked on the host before any launch; a bad
 *     argument returns PQ_ERR_INVALID_ARG or PQ_ERR_UNSUPPORTED and enqueues
 *     nothing. A failed launch returns PQ_ERR_CUDA; pq_last_cuda_error()
 *     then gives the cudaError_t value of the calling thread's last failure.
 *
 * Sources, by page title and section:
 *   [P1] "ParetoQ, the strongest low-bit QAT I could find" (modelfoundations.com)
 *   [P3] "ParetoQ: Improving Scaling Laws in Extremely Low-bit LLM
 *        Quantization" (paperhub.cn, authors' rebuttal)
 *   [P4] "Meta's ParetoQ compares five bit widths and puts the accuracy
 *        cliff at 1 bit" (llmobile ticker)
 */
#ifndef PQ_H_
#define PQ_H_

#include <stdint.h>

#if defined(__GNUC__)
#define PQ_API __attribute__((visibility("default")))
#else
#define PQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Quantizer (level set). [P1 "Finding 3"; P1 "Paper vs. code", the dispatch
 * SEQ for 1.58/2-bit, LSQ for 3/4-bit; P3 "why SEQ is better than LSQ"].
 *
 *   enum        clip on x          code c                         level (alpha units)
 *   PQ_BINARY   [-1, 1] mask only  x >= 0 ? +1 : -1               c
 *   PQ_TERNARY  [-0.99f, 0.99f]    rint(xc*1.5)                   c/1.5  = {-2/3, 0, 2/3}
 *   PQ_SEQ2     [-0.99f, 0.99f]    rint(xc*2 - 0.5)               (c+0.5)/2 = {+-0.25, +-0.75}
 *   PQ_SEQ2_B   [-0.99f, 0.99f]    rint(xc*1.5 - 0.5)             (c+0.5)/1.5 = {+-1/3, +-1}
 *   PQ_LSQ2/3/4 [-2^(b-1), 2^(b-1)-1]  rint(xc)                   c (integer grid)
 *
 * rint rounds half to even; each fp32 step rounds on its own (no FMA);
 * xc = min(max(x, lo), hi). PQ_SEQ2 is the 2-bit SEQ grid as printed on
 * [P1]; PQ_SEQ2_B is the alternative reading whose levels are
 * {-1.5,-0.5,0.5,1.5}/1.5. A negative argument that rounds to zero gives
 * the level -0.0 (and a dequantized -0.0), as the floating-point formula
 * does. The clip 0.99 is the code's 1 - 1e-2 [P1 "Paper vs. code"]. */
typedef enum {
    PQ_BINARY = 1,
    PQ_TERNARY = 2,
    PQ_SEQ2 = 3,
    PQ_SEQ2_B = 4,
    PQ_LSQ2 = 5,
    PQ_LSQ3 = 6,
    PQ_LSQ4 = 7
} pq_quant_t;

typedef enum {
    PQ_OK = 0,
    PQ_ERR_INVALID_ARG = 1, /* null pointer, negative size, bad enum, bad pack shape */
    PQ_ERR_UNSUPPORTED = 2, /* valid request the library does not serve */
    PQ_ERR_MISALIGNED = 3,  /* reserved: misaligned input is served by the element path */
    PQ_ERR_CUDA = 4,        /* a CUDA runtime call or launch failed */
    PQ_ERR_TIMEOUT = 5      /* reserved for bounded device-side waits */
} pq_status_t;

/* Forward fake-quantization of one weight matrix.
 * [P1 "Paper vs. code": SEQ formula alpha*(round(Clip(w/alpha)*k/2 - 0.5)
 *  + 0.5)/k*2, per-row scale of shape (rows, 1), cast of the quantized
 *  weight to the activation dtype; P1 "Finding 3": level sets.]
 *
 *   q            quantizer
 *   rows, cols   matrix shape (>= 0)
 *   w            fp32 [rows*cols], row-major
 *   alpha        fp32 [rows]
 *   wq_bf16_out  bf16 bit patterns [rows*cols]: bf16_rn(fl(level*alpha))
 *   packed_out   nullable; uint8 [rows * cols * bits / 8] with bits =
 *                pq_code_bits(q): two's-complement codes, 8/bits per byte,
 *                column k*(8/bits)+i of a row in bits [bits*i+bits-1 :
 *                bits*i] of byte k, rows back to back. Needs
 *                cols % (8/bits) == 0, else PQ_ERR_INVALID_ARG.
 *                [P4: ternary stored as 2-bit signed integers]
 *   stream       cudaStream_t
 * Algorithmic traffic: 4 B read + 2 B write per weight (+ bits/8 B packed).
 */
PQ_API pq_status_t pq_fakequant_fwd(pq_quant_t q, int64_t rows, int64_t cols,
                             const float* w, const float* alpha,
                             uint16_t* wq_bf16_out, uint8_t* packed_out,
                             void* stream);

/* Straight-through-estimator backward with the per-row scale gradient.
 * [P1 "QAT versus PTQ": gradient passed straight through inside the
 *  clipping range; P1 "The 2-bit recipe, in full": exactly zero outside,
 *  while alpha keeps a boundary-value gradient from the clipped weights;
 *  P1 "Paper vs. code": LSQ gradient for alpha with 1/sqrt(n*Qp) scaling,
 *  gradients in FP32 against the shadow weights.]
 *
 *   g_bf16       bf16 bit patterns [rows*cols], the upstream dWq
 *   dw_out       fp32 [rows*cols]: inside ? float(g) : +0.0f, where
 *                inside = (lo <= x <= hi) on the unclipped x (closed range)
 *   dalpha_out   fp32 [rows]: grad_scale * sum_j g_j*(level_j - inside_j*x_j),
 *                accumulated in fp64 in a fixed order, rounded once to fp32
 *   grad_scale   multiplies each row sum once; pq_default_grad_scale gives
 *                the LSQ rule 1/sqrt(cols*Qp)
 * Algorithmic traffic: 4 B + 2 B read, 4 B written per weight.
 */
PQ_API pq_status_t pq_fakequant_bwd(pq_quant_t q, int64_t rows, int64_t cols,
                             const float* w, const float* alpha,
                             const uint16_t* g_bf16, float* dw_out,
                             float* dalpha_out, float grad_scale,
                             void* stream);

/* Packed code export only (the forward's packed_out without the bf16
 * weights). Same layout and shape rule as packed_out above.
 * Algorithmic traffic: 4 B read + bits/8 B written per weight. */
PQ_API pq_status_t pq_pack_codes(pq_quant_t q, int64_t rows, int64_t cols,
                          const float* w, const float* alpha,
                          uint8_t* packed_out, void* stream);

/* One weight matrix of a batched call. The forward reads rows, cols, w,
 * alpha and writes wq_bf16_out and/or packed_out (at least one non-NULL when
 * the matrix is not empty); the backward reads rows, cols, w, alpha, g_bf16,
 * grad_scale and writes dw_out and dalpha_out. Fields a call does not use
 * are ignored. Layouts and rules are those of the single-matrix calls. */
typedef struct {
    int64_t rows;
    int64_t cols;
    const float* w;
    const float* alpha;
    uint16_t* wq_bf16_out;
    uint8_t* packed_out;
    const uint16_t* g_bf16;
    float* dw_out;
    float* dalpha_out;
    float grad_scale;
} pq_matrix_t;

/* Forward over n matrices in as few launches as possible (one per 256
 * matrices of the vector layout and output kind; the element path runs per
 * matrix). `mats` is a HOST array read during the call only; descriptors
 * travel as kernel parameters, so nothing is allocated. Equivalent to n
 * calls of pq_fakequant_fwd (or pq_pack_codes when wq_bf16_out is NULL)
 * on the same stream. All descriptors are validated before any launch. */
PQ_API pq_status_t pq_fakequant_fwd_batch(pq_quant_t q, int32_t n,
                                          const pq_matrix_t* mats, void* stream);

/* Backward over n matrices, batched like pq_fakequant_fwd_batch; equivalent
 * to n calls of pq_fakequant_bwd on the same stream. */
PQ_API pq_status_t pq_fakequant_bwd_batch(pq_quant_t q, int32_t n,
                                          const pq_matrix_t* mats, void* stream);

/* Hyperparameters of one AdamW step (decoupled weight decay). The library
 * forms its scalar factors once in double and rounds each to fp32:
 * decay = 1 - lr*weight_decay, beta1, 1 - beta1, beta2, 1 - beta2,
 * 1/sqrt(1 - beta2^step), lr/(1 - beta1^step), eps. Requires step >= 1,
 * 0 <= beta < 1, eps > 0, lr >= 0. [P1 "The 2-bit recipe, in full":
 * AdamW, weight decay 0; betas and eps are not stated there.] */
typedef struct {
    double lr;
    double beta1;
    double beta2;
    double eps;
    double weight_decay;
    int64_t step;
} pq_adamw_t;

/* One weight matrix of pq_fakequant_bwd_adamw (device pointers). */
typedef struct {
    int64_t rows;
    int64_t cols;
    float* w;                 /* fp32 [rows*cols], updated in place */
    float* alpha;             /* fp32 [rows], updated in place */
    const uint16_t* g_bf16;   /* bf16 [rows*cols], upstream dWq */
    float* m_w;               /* fp32 [rows*cols], AdamW first moments of w */
    float* v_w;               /* fp32 [rows*cols], second moments of w */
    float* m_alpha;           /* fp32 [rows], first moments of alpha */
    float* v_alpha;           /* fp32 [rows], second moments of alpha */
    float* dalpha_out;        /* fp32 [rows] or NULL: d(alpha) as computed */
    float grad_scale;         /* as in pq_fakequant_bwd */
} pq_adamw_matrix_t;

/* Backward fused with the optimizer step: for every matrix, the STE
 * gradient dW and d(alpha) of pq_fakequant_bwd are formed from the CURRENT
 * w and alpha, then one AdamW step updates every weight (gradient dW,
 * hyperparameters hp_w) and every row's alpha (gradient: the fp32
 * d(alpha), hyperparameters hp_alpha), in one pass: dW never goes to
 * memory. Per weight, element by element in fp32 (each step rounded on its
 * own): p = p*decay (if weight_decay != 0); m = beta1*m + (1-beta1)*g;
 * v = beta2*v + (1-beta2)*(g*g); p = p - (lr/bc1) * (m / (sqrt(v)/sqrt(bc2) +
 * eps)), with 1/sqrt(bc2) a precomputed factor. With data-parallel
 * replicas, all-reduce g_bf16 first: dW and d(alpha) are linear in it and
 * the STE mask is identical on every replica.
 * Traffic: 14 B read + 12 B written per weight (38 B for the backward
 * followed by a separate AdamW). Batched like pq_fakequant_bwd_batch; the
 * buffers of different matrices must not overlap. */
PQ_API pq_status_t pq_fakequant_bwd_adamw(pq_quant_t q, int32_t n,
                                          const pq_adamw_matrix_t* mats,
                                          const pq_adamw_t* hp_w,
                                          const pq_adamw_t* hp_alpha, void* stream);

/* One row shard of a weight matrix owned by this GPU (row-sharded,
 * owner-computes training): the shard's rows of w, alpha and the AdamW
 * moments live here; its upstream gradient rows sit at element offset
 * g_offset in every replica's gradient buffer (see pq_reduce_bwd_adamw). */
typedef struct {
    int64_t rows;
    int64_t cols;
    float* w;
    float* alpha;
    float* m_w;
    float* v_w;
    float* m_alpha;
    float* v_alpha;
    float* dalpha_out;        /* nullable */
    int64_t g_offset;         /* elements, >= 0 */
    float grad_scale;
} pq_shard_t;

/* Reduce-scatter fused with the backward and AdamW: for every shard, the
 * upstream gradient of each element is the fp32 sum, in source order, of
 * the bf16 gradients g_sources[0..n_src) (one per data-parallel replica,
 * all with the same layout; device pointers, local or another GPU's
 * memory reachable by peer access, e.g. mapped with pq_ipc_open), times
 * grad_mult (1/n_src for a mean); then the steps of
 * pq_fakequant_bwd_adamw run with that fp32 gradient. Each GPU calls this
 * on its own shards after every replica's gradient is complete (the
 * caller orders the launch after the replicas' writes, e.g. with a
 * collective or barrier on the stream); no data crosses GPUs except these
 * reads. 1 <= n_src <= 16. Traffic per weight: 2*n_src B gradient reads
 * (2*(n_src-1) over NVLink) + 12 B read + 12 B written locally. */
PQ_API pq_status_t pq_reduce_bwd_adamw(pq_quant_t q, int32_t n_src,
                                       const uint16_t* const* g_sources,
                                       float grad_mult, int32_t n,
                                       const pq_shard_t* shards,
                                       const pq_adamw_t* hp_w,
                                       const pq_adamw_t* hp_alpha, void* stream);

/* Peer-readable buffers across processes (the row-sharded step's plumbing;
 * no counterpart in the pages, which leave multi-GPU layout to the training
 * framework). A CUDA IPC handle of the device allocation that holds a
 * buffer; another process maps that allocation with pq_ipc_open and reads
 * the buffer at the exported offset from the mapped base. The mappings are
 * point-to-point peer mappings (peer access is enabled on first use): no
 * NVLink multicast object is created or bound.
 *   pq_ipc_export: dev_ptr is any address inside a cudaMalloc'd allocation
 *     of the current device (e.g. a tensor of a caching allocator; memory
 *     from virtual-memory or async pools is rejected with PQ_ERR_CUDA);
 *     handle_out receives the allocation's handle, offset_out the byte
 *     offset of dev_ptr from the allocation's base. Several buffers of one
 *     allocation share a handle: map it once per process.
 *   pq_ipc_open: maps an exported allocation into this process (current
 *     device) and returns its base; the owner must keep the allocation
 *     alive until every mapping is closed. Opening a handle exported by
 *     this same process fails (PQ_ERR_CUDA).
 *   pq_ipc_close: unmaps a base returned by pq_ipc_open, after this
 *     process's last kernel reading it has completed.
 * Host calls; nothing is enqueued and nothing is allocated. */
typedef struct {
    unsigned char bytes[64];
} pq_ipc_handle_t;

PQ_API pq_status_t pq_ipc_export(const void* dev_ptr, pq_ipc_handle_t* handle_out,
                                 int64_t* offset_out);
PQ_API pq_status_t pq_ipc_open(const pq_ipc_handle_t* handle, void** base_out);
PQ_API pq_status_t pq_ipc_close(void* base);

/* Dequantize packed codes back to bf16 weights: each stored code c (layout
 * of packed_out above) becomes bf16_rn(fl(level(c) * alpha_row)) with the
 * forward's level formulas, so the result equals the forward's
 * wq_bf16_out except that a zero level is +0.0 (the code does not keep the
 * sign of a rounded-to-zero weight). This is the consumer of exported
 * low-bit weights [P4: 2-bit kernels read packed weights; P1 "Paper vs.
 * code": the training code has no packed path].
 *   packed       uint8 [rows * cols * bits / 8], cols % (8/bits) == 0
 *   alpha        fp32 [rows]
 *   wq_bf16_out  bf16 bit patterns [rows*cols], overwritten
 * Fast path: cols % 8 == 0, packed aligned to 2 (2-bit) or 4 (4-bit)
 * bytes, wq_bf16_out to 16 bytes; any other layout takes an element path
 * with the same results. Traffic: bits/8 B read + 2 B written per weight. */
PQ_API pq_status_t pq_dequant_codes(pq_quant_t q, int64_t rows, int64_t cols,
                                    const uint8_t* packed, const float* alpha,
                                    uint16_t* wq_bf16_out, void* stream);

/* Dequantization over n matrices in as few launches as possible: for each
 * descriptor, packed_out is READ (the codes a forward wrote), alpha read,
 * wq_bf16_out written; other fields are ignored. Equivalent to n calls of
 * pq_dequant_codes on the same stream. */
PQ_API pq_status_t pq_dequant_codes_batch(pq_quant_t q, int32_t n,
                                          const pq_matrix_t* mats, void* stream);

/* Scaled weights x = fl(w / alpha_row): the first step of every quantizer,
 * computed by the same device routine as the forward and backward kernels
 * (the correctly rounded fp32 quotient; [P1 "Paper vs. code": the
 * quantizer clips and rounds w/alpha]). Useful to inspect a layer's
 * distribution in alpha units and to check the division on its own.
 *   w      fp32 [rows*cols] (any alignment), alpha fp32 [rows]
 *   x_out  fp32 [rows*cols], overwritten
 * Traffic: 4 B read + 4 B written per weight. */
PQ_API pq_status_t pq_scaled_weights(int64_t rows, int64_t cols, const float* w,
                                     const float* alpha, float* x_out, void* stream);

/* Weight-only low-bit matmul on the tensor cores (tcgen05, fp32 in TMEM):
 *   Y[m][n] = sum_k X[m][k] * level(code[n][k]) * alpha[n]
 * for the 2-bit quantizers (PQ_BINARY, PQ_TERNARY, PQ_SEQ2, PQ_SEQ2_B,
 * PQ_LSQ2; others return PQ_ERR_UNSUPPORTED). The pages' 2-bit inference
 * kernels consume packed weights in this way [P4: a 2-bit GEMM kernel on
 * CUTLASS; P3: the accuracy-latency trade-off]; this one is built for
 * sm_100a. The levels' integer numerators (SEQ2 2c+1, SEQ2_B 2c+1, ternary
 * 2c, LSQ2 and binary c) are affine in the code's offset-binary field
 * f' = c + 2; the factor (1/4, 1/3, 1/3, 1, 1) times alpha scales the sums,
 * which are rounded once to bf16. Two modes:
 *   m <= 16 (integer mode; m = 1 only for the grouped call): each activation
 *     row is scaled by a power of two to 30-bit fixed point and rounded to the
 *     nearest integer (exact for every value within 2^22 of the row's largest
 *     magnitude; otherwise off by at most 2^-30 of it); the tensor cores form
 *     the exact integer sums of those integers times the fields, combined in
 *     fp64. While every k <= 2^20 the integers go in as ten planes of
 *     balanced base-9 digits on block-scaled fp4 MMAs (kind::mxf4, unit
 *     scales; the weights as f'/2, every product and partial sum an exact
 *     fp32 value); beyond, as four signed base-256 digit planes on 8-bit MMAs
 *     (kind::i8, s32 sums). Both form the same exact integers and put them
 *     through the same formula.
 *   m > 16 (bf16 mode): weights decoded to bf16 1 + f'/4 (exact), products
 *     accumulated in fp32 by the tensor cores (kind::f16).
 * A lone matrix with m = 1 runs on the CUDA cores: below 2^27 weights with
 * fp32 fused multiply-adds, from 2^27 weights with the integer mode's
 * arithmetic (dp4a on the digit planes).
 * The bf16 and CUDA-core modes form y from sums over all k of x (1 + f'/4)
 * and of x, so their rounding scales with alpha sum_k |x|; where activations
 * far larger than the rest of their row meet zero levels (ternary, LSQ2),
 * that scale, not sum_k |x w|, bounds the error, as 2^-30 max_k |x|
 * sum_k |w| does in the integer mode.
 *   x_bf16   bf16 [m, k], row-major, 16-byte aligned, 1 <= m <= 128
 *   packed   codes [n, k/4] as pq_fakequant_fwd writes them, 16-byte aligned
 *   alpha    fp32 [n]
 *   y_bf16   bf16 [m, n], row-major, overwritten
 *   k        a multiple of 128
 *   workspace, workspace_bytes: device scratch of at least
 *            pq_wq_gemm_workspace_bytes(q, m, n, k) bytes, 256-byte
 *            aligned (may be NULL when that is 0). Split-K partial sums and
 *            counters, and in the integer mode the activations' digit planes
 *            (fp4: 10 mp k / 2 bytes, mp = 8 for m <= 8 else 16; 8-bit:
 *            4 m k bytes) and exponents, live there; calls that share a
 *            workspace must not overlap on the GPU. Results are deterministic.
 * Waits inside the kernel are bounded; pq_device_status() reports one that
 * gave up. Traffic: k/4 B of codes per output feature (+ x, y). */
PQ_API pq_status_t pq_wq_gemm(pq_quant_t q, int64_t m, int64_t n, int64_t k,
                              const uint16_t* x_bf16, const uint8_t* packed,
                              const float* alpha, uint16_t* y_bf16, void* workspace,
                              int64_t workspace_bytes, void* stream);

/* Workspace bytes pq_wq_gemm needs for this problem (0: none), -1 for an
 * unsupported quantizer or shape. */
PQ_API int64_t pq_wq_gemm_workspace_bytes(pq_quant_t q, int64_t m, int64_t n, int64_t k);

/* One matrix of a grouped weight-only matmul: Y = X (alpha * levels)^T with
 * the layouts and alignment of pq_wq_gemm; all matrices of a call share the
 * quantizer and the activation rows m (each may have its own X). */
typedef struct {
    int64_t n, k;               /* weight rows and columns (k a multiple of 128) */
    const uint16_t* x_bf16;     /* [m, k] bf16, 16-byte aligned */
    const uint8_t* packed;      /* [n, k/4] codes, 16-byte aligned */
    const float* alpha;         /* [n] */
    uint16_t* y_bf16;           /* [m, n] bf16, overwritten */
} pq_gemm_problem_t;

/* pq_wq_gemm over 1..64 matrices in one launch: their (row block, K chunk)
 * work items are split evenly over the GPU's SMs as one list, so the fixed
 * cost of a launch (pipeline fill, epilogue) is paid once for the group.
 * `problems` is a host array of `count` entries, read before the call
 * returns. Results equal separate pq_wq_gemm calls within rounding (the
 * split of K into partial sums may differ) and are deterministic.
 * Workspace: pq_wq_gemm_batch_workspace_bytes(...) bytes, 256-byte aligned
 * (NULL when 0); calls sharing a workspace must not overlap on the GPU.
 * count outside 1..64 or any bad matrix: PQ_ERR_INVALID_ARG, nothing run. */
PQ_API pq_status_t pq_wq_gemm_batch(pq_quant_t q, int64_t m, int32_t count,
                                    const pq_gemm_problem_t* problems, void* workspace,
                                    int64_t workspace_bytes, void* stream);

/* Workspace bytes pq_wq_gemm_batch needs (0: none), -1 if invalid. In the
 * integer mode it counts one digit-plane set per matrix; a call whose
 * matrices share activations (same x_bf16 and k) uses one set for them. */
PQ_API int64_t pq_wq_gemm_batch_workspace_bytes(pq_quant_t q, int64_t m, int32_t count,
                                                const pq_gemm_problem_t* problems);

/* Upper limit on the split-K scratch pq_wq_gemm_noalloc can use (8 MiB). */
#define PQ_WQ_GEMM_NOALLOC_SCRATCH_BYTES (8LL << 20)

/* pq_wq_gemm without a caller workspace and without allocating: the split-K
 * scratch is a fixed PQ_WQ_GEMM_NOALLOC_SCRATCH_BYTES array in the library's
 * device memory, one per device. The method's pages have no counterpart
 * to this entry point; it exists for callers that cannot allocate device
 * memory at call time: code inside an allocator's out-of-memory or free
 * callback (it must not re-enter the allocator), serving loops whose device
 * memory is reserved in full up front by a caching pool, and latency-bound
 * paths that cannot take the device-wide synchronisation of cudaFree.
 * Arguments, layouts and results are those of pq_wq_gemm (same kernel, same
 * split plan, same bits).
 *   Limit: a problem whose pq_wq_gemm_workspace_bytes(q, m, n, k) exceeds
 *          PQ_WQ_GEMM_NOALLOC_SCRATCH_BYTES returns PQ_ERR_UNSUPPORTED and
 *          enqueues nothing; call pq_wq_gemm with a workspace instead.
 *   Set-up: the first call on each device that passes the argument checks
 *          looks up the array's device address once (cudaGetSymbolAddress;
 *          a failure returns PQ_ERR_CUDA and the next call retries). Make
 *          that first call before any stream capture. The address is kept
 *          for the life of the process: after cudaDeviceReset on a device
 *          the library's module is loaded again and the kept address may
 *          be stale, so do not call this entry point on a device that has
 *          been reset since its first call.
 *   Zeroing: the split-K counters at the end of the used scratch must be
 *          zero when the kernel starts; every call clears them on `stream`
 *          (cudaMemsetAsync) before its launch. The partial sums need no
 *          clearing.
 *   Concurrency: all calls on one device share the one array, so calls that
 *          may overlap on the GPU (unordered streams, several host threads)
 *          race on it and give wrong results; order them on one stream.
 * No cudaMalloc, cudaFree or other allocating routine is called. */
PQ_API pq_status_t pq_wq_gemm_noalloc(pq_quant_t q, int64_t m, int64_t n, int64_t k,
                                      const uint16_t* x_bf16, const uint8_t* packed,
                                      const float* alpha, uint16_t* y_bf16, void* stream);

/* Device status of the library's bounded waits (the weight-only matmul
 * waits on mbarriers; every wait has an iteration cap): PQ_OK if none gave
 * up since the last call, PQ_ERR_TIMEOUT if one did (the status is then
 * cleared), PQ_ERR_CUDA if the status could not be read. A kernel whose wait
 * gave up stops all its roles, lets its copies and MMAs in flight finish,
 * frees its tensor memory and returns; its outputs are then undefined and
 * the CUDA context stays usable. Synchronises the device. */
PQ_API int pq_device_status(void);

/* Test switch for the timeout path: while on, every later launch of the
 * matmul's tensor-core path raises its abort flag at start, so its waits give
 * up as a wait that reached its cap does (roles stop, copies and MMAs in
 * flight drain, TMEM is freed) and pq_device_status reports PQ_ERR_TIMEOUT;
 * outputs of those launches are undefined. Off (0) by default. */
PQ_API pq_status_t pq_debug_abort_waits(int on);

/* Storage width in bits of one packed code: 2 (binary, ternary, SEQ2,
 * SEQ2_B, LSQ2) or 4 (LSQ3, LSQ4); 0 for an unknown quantizer. */
PQ_API int pq_code_bits(pq_quant_t q);

/* LSQ gradient scale 1/sqrt(cols*Qp) with n = cols weights per scale;
 * Qp = 1 (binary, ternary, LSQ2), 1.5 (SEQ2, SEQ2_B), 3 (LSQ3), 7 (LSQ4).
 * [P1 "Paper vs. code"]. Returns 0 for cols <= 0 or an unknown quantizer. */
PQ_API float pq_default_grad_scale(pq_quant_t q, int64_t cols);

/* Static description of a status code. */
PQ_API const char* pq_status_string(pq_status_t s);

/* cudaError_t of the calling thread's last PQ_ERR_CUDA (0 if none). */
PQ_API int pq_last_cuda_error(void);

/* Number of kernel launches the library has enqueued since it was loaded,
 * over all devices, streams and threads (a host-side counter, read without
 * synchronising). A call's launches are the difference of two readings;
 * under stream capture it counts the launches captured into the graph,
 * which every replay of the graph repeats. No counterpart in the pages:
 * it lets a caller report how many of this library's kernels a timed
 * region ran. */
PQ_API int64_t pq_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* PQ_H_ */
