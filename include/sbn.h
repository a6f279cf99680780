/*
 * sbn.h -- C ABI of libsbn: the Sparse-BitNet BitLinear forward on B200 (sm_100a).
 *
 * The BitLinear forward ("Microsoft BitNet 1.58: The Era of 1-Bit Large
 * Language Models", section "The BitLinear Layer") quantizes activations to
 * INT8 with an absmax scale, quantizes the latent weights to ternary
 * {-1, 0, +1} with an absmean scale, contracts the two in integer arithmetic
 * and dequantizes the result. Sparse-BitNet ("Sparse-BitNet: 1.58-bit LLMs
 * are Naturally Friendly to Semi-Structured Sparsity", Abstract) adds a
 * dynamic N:M magnitude mask on the latent weights, recomputed every forward.
 *
 * Three calls make the path:
 *   sbn_quantize_weights : mask + absmean ternary + pack   (latent bf16 W -> packed)
 *   sbn_quantize_acts    : per-token absmax INT8           (bf16 X -> Xq, s)
 *   sbn_bitlinear        : packed W x Xq, int32 accumulate, dequantize to bf16
 *
 * Conventions shared by every call
 *   - Sizes: T tokens, K in-features, N_out out-features; n:m keeps n of every
 *     m consecutive weights along K.
 *   - Layouts (row-major): X [T, K] bf16; W [N_out, K] bf16 (nn.Linear
 *     convention); Xq [T, K] int8; x_scale [T] fp32; Y [T, N_out] bf16;
 *     acc [T, N_out] int32.
 *   - Every pointer argument named "device" is device memory of the current
 *     CUDA device, owned by the caller, 16-byte aligned. The library never
 *     allocates or frees memory and never synchronizes, except
 *     sbn_get_device_error. All work is enqueued on `stream` (a cudaStream_t;
 *     NULL means the legacy default stream) and is asynchronous.
 *   - Argument errors are returned synchronously before anything is enqueued;
 *     outputs are then untouched. A failed launch returns SBN_ERR_CUDA.
 *     Device-side failures (a bounded wait that ran out) are recorded in a
 *     device error word and reported by sbn_get_device_error.
 *   - Non-finite inputs (inf, NaN) give unspecified outputs.
 *   - Per-device state: on its first call on a device the library caches,
 *     for that device, the result of its capability check, the kernels'
 *     shared-memory size attributes and the device address of the
 *     sbn_quantize_weights_noalloc scratch array. These belong to the
 *     device's primary context as it was then: after cudaDeviceReset (or any
 *     other end of that context) they are stale, and the library must not be
 *     called again on that device in the same process. Several host threads
 *     may make first calls at the same time; they store the same values.
 *
 * Packed weight format (canonical; produced by sbn_quantize_weights and read
 * by sbn_bitlinear):
 *   codes [N_out, codes_row_bytes]: per row, the ternary values of the kept
 *     positions in ascending k; value j sits in bits 2*(j%4)..2*(j%4)+1 of
 *     byte j/4, encoded 0 -> 00, +1 -> 01, -1 -> 11 (four 2-bit values per
 *     byte, as in the section "bitnet.cpp: Matrix-Free Inference" of the
 *     octagono page); codes_row_bytes = ceil(K*n/m/4) rounded up to 16, the
 *     padding bytes are zero.
 *   meta [N_out, meta_row_bytes]: per row, bit k%8 of byte k/8 is 1 iff
 *     position k is kept; meta_row_bytes = K/8 rounded up to 16; absent
 *     (0 bytes, pointer may be NULL) when n == m.
 *   gamma: one fp32 device scalar, the absmean scale.
 *
 * Supported patterns: m in {4, 8, 16} and 1 <= n <= m with 4*n divisible by
 * m (1:4 2:4 3:4 4:4, 2:8 4:8 6:8 8:8, 4:16 8:16 12:16 16:16). Shapes: K a
 * multiple of 128; T, N_out >= 1; T*K, N_out*K and T*N_out below 2^31.
 */
#ifndef SBN_H
#define SBN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  SBN_OK = 0,
  SBN_ERR_NULL = 1,      /* a required pointer is NULL */
  SBN_ERR_SHAPE = 2,     /* a size is out of the supported range */
  SBN_ERR_PATTERN = 3,   /* unsupported n:m */
  SBN_ERR_ALIGN = 4,     /* a pointer is not 16-byte aligned */
  SBN_ERR_WORKSPACE = 5, /* the workspace is smaller than required */
  SBN_ERR_CUDA = 6,      /* a CUDA runtime call or kernel launch failed */
  SBN_ERR_TIMEOUT = 7,   /* a bounded device-side wait gave up */
  SBN_ERR_DEVICE = 8     /* the current device is not sm_100 */
} sbn_status;

/* Human-readable name of a status code (static string, never NULL). */
const char* sbn_status_string(sbn_status s);

/* Library version as 10000*major + 100*minor + patch. */
int sbn_version(void);

/* Bytes of one packed code row, of the whole codes array, of one meta row and
 * of the whole meta array for the given shape and pattern (0 for an
 * unsupported pattern or shape). */
size_t sbn_codes_row_bytes(int32_t k, int32_t n, int32_t m);
size_t sbn_codes_bytes(int32_t n_out, int32_t k, int32_t n, int32_t m);
size_t sbn_meta_row_bytes(int32_t k, int32_t n, int32_t m);
size_t sbn_meta_bytes(int32_t n_out, int32_t k, int32_t n, int32_t m);

/* Device workspace that sbn_quantize_weights needs (exact-sum bins and the
 * derived threshold), in bytes. */
size_t sbn_quantize_weights_workspace_bytes(int32_t n_out, int32_t k);

/*
 * sbn_quantize_weights -- dynamic N:M mask, absmean ternary codes, packing.
 *
 * Defining passages: the absmean quantizer ("BitNet b1.58: How Ternary
 * Weights Cut LLM Memory by 82% Without Losing Accuracy", section "How
 * ternary quantization works during training": divide W by its mean absolute
 * value, round, clamp to [-1, 1]); the N:M magnitude mask (Sparse-BitNet page,
 * Abstract, and Figure 6: the per-block threshold t = |w|_(N+1)).
 *
 *   w_bf16     device, [n_out, k] bf16, read only.
 *   codes      device, sbn_codes_bytes(n_out, k, n, m) bytes, written.
 *   meta       device, sbn_meta_bytes(...) bytes, written; NULL allowed iff n == m.
 *   gamma      device, one float, written:
 *              gamma = max(fl32(fl64(S) / (n_out*k)), 1e-5) where S is the exact
 *              sum of |w| and fl64(S) its correctly rounded double.
 *   workspace  device, at least sbn_quantize_weights_workspace_bytes() bytes,
 *              scratch owned by the caller; its contents on entry do not matter
 *              and are overwritten. Calls that share a workspace must not
 *              overlap in time (same stream, or ordered by events).
 *
 * Mask: within every group of m consecutive positions of a row, the n
 * positions of largest |w| are kept; equal magnitudes keep the lower index.
 * Codes: clamp(rint(fl32(w / gamma)), -1, 1) (IEEE fp32 division, round half
 * to even) at kept positions; pruned positions are simply absent.
 * Errors: SBN_ERR_NULL, SBN_ERR_SHAPE, SBN_ERR_PATTERN, SBN_ERR_ALIGN,
 * SBN_ERR_WORKSPACE (returned before any work is enqueued); SBN_ERR_CUDA.
 */
sbn_status sbn_quantize_weights(const void* w_bf16, int32_t n_out, int32_t k,
                                int32_t n, int32_t m, uint8_t* codes,
                                uint8_t* meta, float* gamma, void* workspace,
                                size_t workspace_bytes, void* stream);

/*
 * sbn_quantize_weights_noalloc -- sbn_quantize_weights without a caller
 * workspace. (Library addition; the pages describe nothing like it.)
 *
 * For callers that cannot allocate device memory: a plugin or kernel library
 * that is handed only its input and output buffers, a real-time loop where
 * the device-wide synchronization of cudaMalloc/cudaFree is not acceptable,
 * or a process whose memory pool has already reserved all device memory.
 * The scratch lives in a fixed array of SBN_NOALLOC_SCRATCH_BYTES (64 KiB)
 * inside the library, reserved on every GPU that loads it until the process
 * exits. This call performs no allocation of any kind.
 *
 *   Arguments, outputs and results are those of sbn_quantize_weights, minus
 *   the workspace. Shapes whose workspace would exceed the fixed array are
 *   rejected with SBN_ERR_WORKSPACE before anything is enqueued.
 *   The first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress); make that first call before any stream capture.
 *   All calls on a device share the one array: two calls that may run at the
 *   same time on the GPU (different streams without ordering) race and give
 *   wrong results. Calls on one stream are safe.
 */
#define SBN_NOALLOC_SCRATCH_BYTES (64 * 1024)
sbn_status sbn_quantize_weights_noalloc(const void* w_bf16, int32_t n_out, int32_t k,
                                        int32_t n, int32_t m, uint8_t* codes,
                                        uint8_t* meta, float* gamma, void* stream);

/*
 * N_out-sharded (column-parallel) weight quantization.
 *
 * gamma is one scale for the whole tensor ("BitNet b1.58: How Ternary
 * Weights Cut LLM Memory by 82% Without Losing Accuracy", section "How
 * ternary quantization works during training": W is divided by the mean
 * absolute value of the weight tensor). When the rows of a layer are split
 * across devices, each shard computes the exact gamma bins of its rows, the
 * caller sums the bins over the shards (for example with an NCCL all-reduce of
 * SBN_GAMMA_BINS unsigned 64-bit integers: exact and independent of the order),
 * and each shard quantizes its rows with sbn_quantize_weights_from_bins. The
 * concatenated shards then equal sbn_quantize_weights on the whole tensor, byte
 * for byte, gamma included.
 *
 * Bins: SBN_GAMMA_BINS uint64 values B[e] with sum_e B[e] * 2^(e - 134)
 * equal to the exact sum of |w| over the rows. The split across e is not
 * unique, but the bins of two shards add up to bins of their union.
 */
#define SBN_GAMMA_BINS 256

/* Exact gamma bins of w_bf16 [n_out, k] (device, read only) into bins (device,
 * SBN_GAMMA_BINS uint64, 16-byte aligned, overwritten; cleared on `stream`
 * first). Errors: SBN_ERR_NULL, SBN_ERR_SHAPE (k a multiple of 128), SBN_ERR_ALIGN,
 * SBN_ERR_CUDA. */
sbn_status sbn_gamma_bins(const void* w_bf16, int32_t n_out, int32_t k,
                          unsigned long long* bins, void* stream);

/* Mask, codes and packing of w_bf16 [n_out, k] exactly as sbn_quantize_weights,
 * with gamma = max(fl32(fl64(S) / total_elems), 1e-5) where S is the exact sum
 * the bins (device, read only: the sum of every shard's bins) represent and
 * total_elems the element count of the whole tensor (n_out * k <= total_elems
 * <= 2^36). codes,
 * meta and gamma as in sbn_quantize_weights; no workspace. Errors: SBN_ERR_NULL,
 * SBN_ERR_SHAPE, SBN_ERR_PATTERN, SBN_ERR_ALIGN, SBN_ERR_CUDA. */
sbn_status sbn_quantize_weights_from_bins(const void* w_bf16, int32_t n_out,
                                          int32_t k, int32_t n, int32_t m,
                                          const unsigned long long* bins,
                                          int64_t total_elems, uint8_t* codes,
                                          uint8_t* meta, float* gamma, void* stream);

/*
 * sbn_quantize_acts -- per-token absmax INT8 activations.
 *
 * Defining passage: "The BitLinear Layer" (octagono page), second operation:
 * activations are quantized from bf16 to INT8 with absmax scaling and the
 * scale is kept for dequantization; the promptingindex page (same section as
 * above) makes the scale per token.
 *
 *   x_bf16   device, [t, k] bf16, read only (k a multiple of 16).
 *   xq       device, [t, k] int8, written:
 *            q = clamp(rint(fl32(x * fl32(127 / s_t))), -127, 127).
 *   x_scale  device, [t] fp32, written: s_t = max(max_k |x_tk|, 1e-5).
 * Errors: SBN_ERR_NULL, SBN_ERR_SHAPE, SBN_ERR_ALIGN; SBN_ERR_CUDA.
 */
sbn_status sbn_quantize_acts(const void* x_bf16, int32_t t, int32_t k,
                             int8_t* xq, float* x_scale, void* stream);

/*
 * sbn_bitlinear -- INT8 x ternary contraction with int32 accumulation and
 * dequantization to bf16.
 *
 * Defining passage: "The BitLinear Layer" (octagono page), fourth and fifth
 * operations: the product runs on the quantized values only (additions,
 * subtractions, zero-skips) and is rescaled by the preserved scales.
 *
 *   xq, x_scale   device, from sbn_quantize_acts ([t, k] int8, [t] fp32).
 *   codes, meta,  device, from sbn_quantize_weights for the same n_out, k, n, m
 *   gamma         (meta NULL allowed iff n == m).
 *   y_bf16        device, [t, n_out] bf16, written:
 *                 y = bf16_rne(acc * gamma * s_t / 127) evaluated in fp32, where
 *                 acc[t, o] = sum over kept k of xq[t, k] * code[o, k] (exact int32).
 *   workspace,    optional device scratch owned by the caller (the pages have
 *   ws_bytes      no counterpart). NULL: the packed weights are expanded
 *                 inside the contraction kernel. Non-NULL (16-byte aligned,
 *                 ws_bytes >= sbn_bitlinear_workspace_bytes(t, k, n_out)):
 *                 for t > 16 the packed weights are first expanded once into
 *                 it, and the tensor-core kernel then loads them by TMA like
 *                 the activations: for 2:4 as the compressed operand of the
 *                 sparse MMA (the kept int8 values [n_out, k/2] and their
 *                 4-bit position metadata [n_out rounded up to 256, k/8]),
 *                 for every other pattern as a dense int8 [n_out, k] matrix.
 *                 Ignored for t <= 16. Its contents are unspecified
 *                 afterwards. Both routes give the same acc and y.
 * Tensor-core routes (t > 16): 2:4 runs the sparse INT8 MMA
 * (tcgen05.mma.sp), which multiplies only the kept half of each group of
 * four ("Sparse-BitNet ...", Abstract: the 2:4 pattern suits the sparse
 * tensor cores); every other pattern runs the dense INT8 MMA on expanded
 * weights. With a workspace the MMAs run on CTA pairs (tcgen05 cta_group::2,
 * 256 weight rows per tile, clusters of two CTAs) where the device can hold
 * such clusters, else on single CTAs.
 * Errors: SBN_ERR_NULL, SBN_ERR_SHAPE, SBN_ERR_PATTERN, SBN_ERR_ALIGN,
 * SBN_ERR_WORKSPACE (before anything is enqueued); SBN_ERR_CUDA.
 */
sbn_status sbn_bitlinear(const int8_t* xq, const float* x_scale, int32_t t,
                         int32_t k, int32_t n_out, int32_t n, int32_t m,
                         const uint8_t* codes, const uint8_t* meta,
                         const float* gamma, void* y_bf16, void* workspace,
                         size_t ws_bytes, void* stream);

/* Bytes of sbn_bitlinear's optional workspace: when t > 16, the larger of
 * n_out * k (dense expansion) and the compressed 2:4 form
 * (round_up(n_out * k / 2, 128) + round_up(n_out, 256) * k / 8); else 0. */
size_t sbn_bitlinear_workspace_bytes(int32_t t, int32_t k, int32_t n_out);

/*
 * sbn_bitlinear_x -- sbn_quantize_acts and sbn_bitlinear in one call, from
 * the bf16 activations. For t <= 16 (when the layer's rows and X fit in
 * shared memory) it is one kernel: every CTA quantizes X per token with the
 * arithmetic of sbn_quantize_acts and contracts straight away, so the INT8
 * activations never go through HBM ("The BitLinear Layer" (octagono page),
 * second to fifth operations, run back to back). Otherwise it runs the two
 * calls in sequence.
 *
 *   x_bf16        device, [t, k] bf16.
 *   codes, meta,  as for sbn_bitlinear.
 *   gamma, y_bf16
 *   xq, x_scale   optional (NULL allowed) device outputs, [t, k] int8 and [t]
 *                 fp32: the INT8 activations and scales, bit-identical to
 *                 sbn_quantize_acts.
 *   workspace,    device scratch owned by the caller, 16-byte aligned, at
 *   ws_bytes      least sbn_bitlinear_x_workspace_bytes(t, k, n_out) bytes;
 *                 may be NULL when the one-kernel route applies (t <= 16 on
 *                 the configurations of this library's workloads), else
 *                 SBN_ERR_WORKSPACE. Contents unspecified afterwards.
 * Errors: SBN_ERR_NULL, SBN_ERR_SHAPE, SBN_ERR_PATTERN, SBN_ERR_ALIGN,
 * SBN_ERR_WORKSPACE (before anything is enqueued); SBN_ERR_CUDA.
 */
sbn_status sbn_bitlinear_x(const void* x_bf16, int32_t t, int32_t k,
                           int32_t n_out, int32_t n, int32_t m,
                           const uint8_t* codes, const uint8_t* meta,
                           const float* gamma, void* y_bf16, int8_t* xq,
                           float* x_scale, void* workspace, size_t ws_bytes,
                           void* stream);

/* Bytes of sbn_bitlinear_x's workspace (enough for its two-step route). */
size_t sbn_bitlinear_x_workspace_bytes(int32_t t, int32_t k, int32_t n_out);

/*
 * sbn_bitlinear_acc32 -- the same contraction, writing the exact int32
 * accumulators acc [t, n_out] (device, row-major) instead of y. Meant for
 * verification; same arguments (workspace included) and errors as
 * sbn_bitlinear.
 */
sbn_status sbn_bitlinear_acc32(const int8_t* xq, int32_t t, int32_t k,
                               int32_t n_out, int32_t n, int32_t m,
                               const uint8_t* codes, const uint8_t* meta,
                               int32_t* acc, void* workspace, size_t ws_bytes,
                               void* stream);

/*
 * sbn_mask_flips -- number of positions whose keep bit differs between two
 * keep masks of the same layer (two versions of sbn_quantize_weights' meta
 * for the same n_out, k, n, m), e.g. consecutive training steps.
 *
 * Defining passage: Sparse-BitNet page, Figure 3(b), the mask flip rate r_t
 * (its equation is missing from the page; read as the fraction of mask
 * positions that changed): r_t = flips / (n_out * k).
 *
 *   meta_a, meta_b  device, [n_out, sbn_meta_row_bytes] each, 16-byte aligned.
 *   flips           device, one uint64, 8-byte aligned, written (exact count).
 * Errors: SBN_ERR_NULL, SBN_ERR_SHAPE, SBN_ERR_PATTERN (also for n == m:
 * a dense layer has no mask), SBN_ERR_ALIGN; SBN_ERR_CUDA.
 */
sbn_status sbn_mask_flips(const uint8_t* meta_a, const uint8_t* meta_b,
                          int32_t n_out, int32_t k, int32_t n, int32_t m,
                          unsigned long long* flips, void* stream);

/*
 * Entropy-tight packed weights (the pages have no such format; the size of
 * its keep-pattern part follows "From 2:4 to 8:16 sparsity patterns in LLMs
 * for Outliers and Weights with Variance Correction", Abstract: 0.75 and
 * 0.875 bits per element for the 2:4 and 8:16 masks, i.e. ceil(log2 C(m, n))
 * / m, an index over the keep patterns of a group).
 *
 * Per group of m positions one word
 *     word = rank * 3^n + sum_i (code_i + 1) * 3^i
 * in ceil(log2(C(m, n) * 3^n)) bits, where rank = sum_i C(c_i, i) for the
 * kept offsets c_1 < ... < c_n (combinatorial number system, colex order)
 * and code_i are the kept ternary codes in ascending position. Words are
 * concatenated little-endian per row (bit b is bit b % 8 of byte b / 8);
 * rows are padded with zero bytes to a multiple of 16. 6:8 takes 15 bits per
 * 8 weights (1.875 bits/weight) instead of 2.5.
 */
size_t sbn_entropy_row_bytes(int32_t k, int32_t n, int32_t m);
size_t sbn_entropy_bytes(int32_t n_out, int32_t k, int32_t n, int32_t m);

/*
 * sbn_pack_entropy -- the canonical packed weights (codes, meta) of a layer,
 * as written by sbn_quantize_weights, into the entropy-tight format.
 *   ent   device, [n_out, sbn_entropy_row_bytes(k, n, m)], written.
 * Every supported pattern. Errors: SBN_ERR_NULL, SBN_ERR_SHAPE,
 * SBN_ERR_PATTERN, SBN_ERR_ALIGN; SBN_ERR_CUDA.
 */
sbn_status sbn_pack_entropy(const uint8_t* codes, const uint8_t* meta,
                            int32_t n_out, int32_t k, int32_t n, int32_t m,
                            uint8_t* ent, void* stream);

/*
 * sbn_bitlinear_entropy -- the decode contraction (1 <= t <= 16) reading
 * the entropy-tight weights: the same y as sbn_bitlinear on the canonical
 * weights, bit for bit. Patterns with m = 4 or 8 and n < m; other patterns
 * give SBN_ERR_PATTERN, t > 16 or rows that do not fit in shared memory
 * SBN_ERR_SHAPE. Other arguments and errors as sbn_bitlinear.
 */
sbn_status sbn_bitlinear_entropy(const int8_t* xq, const float* x_scale,
                                 int32_t t, int32_t k, int32_t n_out,
                                 int32_t n, int32_t m, const uint8_t* ent,
                                 const float* gamma, void* y_bf16,
                                 void* stream);

/* The same contraction writing the exact int32 accumulators (verification). */
sbn_status sbn_bitlinear_entropy_acc32(const int8_t* xq, int32_t t,
                                       int32_t k, int32_t n_out, int32_t n,
                                       int32_t m, const uint8_t* ent,
                                       int32_t* acc, void* stream);

/*
 * sbn_bitlinear_entropy_x -- sbn_quantize_acts fused into
 * sbn_bitlinear_entropy: y from the bf16 activations x_bf16 [t, k]
 * (device, 16-byte aligned), bit-identical to sbn_quantize_acts followed by
 * sbn_bitlinear_entropy. Every CTA quantizes X itself (per-token absmax
 * INT8, as sbn_quantize_acts) in its prologue.
 *   xq, x_scale   optional (NULL for none) device outputs [t, k] int8 and
 *                 [t] fp32: the INT8 activations and scales, bit-identical
 *                 to sbn_quantize_acts.
 *   workspace,    device scratch owned by the caller, 16-byte aligned, at
 *   ws_bytes      least sbn_bitlinear_entropy_x_workspace_bytes(t, k) bytes;
 *                 used only when the bf16 rows do not fit in shared memory
 *                 and xq or x_scale is NULL (two-step route: quantize, then
 *                 contract), else may be NULL. Contents unspecified after.
 * Patterns and shapes as sbn_bitlinear_entropy. Errors: SBN_ERR_NULL,
 * SBN_ERR_SHAPE, SBN_ERR_PATTERN, SBN_ERR_ALIGN, SBN_ERR_WORKSPACE (before
 * anything is enqueued); SBN_ERR_CUDA.
 */
sbn_status sbn_bitlinear_entropy_x(const void* x_bf16, int32_t t, int32_t k,
                                   int32_t n_out, int32_t n, int32_t m,
                                   const uint8_t* ent, const float* gamma,
                                   void* y_bf16, int8_t* xq, float* x_scale,
                                   void* workspace, size_t ws_bytes,
                                   void* stream);

/* Bytes of sbn_bitlinear_entropy_x's workspace (its two-step route). */
size_t sbn_bitlinear_entropy_x_workspace_bytes(int32_t t, int32_t k);

/*
 * Backward of the layer under the straight-through estimator ("Microsoft
 * BitNet 1.58: The Era of 1-Bit Large Language Models", section "Training
 * with the Straight-Through Estimator": gradients cross the quantizer as the
 * identity; the latent weights take them). The forward multiplies the
 * dequantized activations Xd = Xq * s_t / 127 by Wd = gamma * C (C the masked
 * ternary codes), so with dY = dL/dY [t, n_out] (device, bf16, row-major,
 * 16-byte aligned):
 *
 * sbn_bitlinear_grad_x -- dX = dY * (gamma C), [t, k] bf16 written to dx_bf16
 *   (device, 16-byte aligned). codes, meta, gamma as written by
 *   sbn_quantize_weights for (n_out, k, n, m). fp32 accumulation, one bf16
 *   rounding.
 * sbn_bitlinear_grad_w -- dW = dY^T * (Xq s / 127), [n_out, k] bf16 written
 *   to dw_bf16 (device, 16-byte aligned): the gradient of every latent
 *   weight, pruned positions included. xq [t, k] int8 and x_scale [t] fp32
 *   as written by sbn_quantize_acts for the forward's X. fp32
 *   accumulation, one bf16 rounding.
 * Shapes as sbn_bitlinear (k a multiple of 128). Errors: SBN_ERR_NULL,
 * SBN_ERR_SHAPE, SBN_ERR_PATTERN, SBN_ERR_ALIGN (before anything is
 * enqueued); SBN_ERR_CUDA.
 */
sbn_status sbn_bitlinear_grad_x(const void* dy_bf16, int32_t t, int32_t k,
                                int32_t n_out, int32_t n, int32_t m,
                                const uint8_t* codes, const uint8_t* meta,
                                const float* gamma, void* dx_bf16,
                                void* stream);
sbn_status sbn_bitlinear_grad_w(const void* dy_bf16, const int8_t* xq,
                                const float* x_scale, int32_t t, int32_t k,
                                int32_t n_out, void* dw_bf16, void* stream);

/*
 * Measurement helper (no counterpart in the method): the INT8 rate of the
 * tensor pipe. Launches one CTA per SM on `stream`, each issuing `iters`
 * back-to-back tcgen05.mma kind::i8 instructions of M = 128, N = 256,
 * K = 32 (2 * 128 * 256 * 32 operations each, int32 accumulation in tensor
 * memory) on shared-memory operands -- the instruction and tile shape of the
 * prefill contraction, with no loads in between. *ctas (host) receives the
 * number of CTAs; the caller times the launch. Errors: SBN_ERR_NULL,
 * SBN_ERR_SHAPE (iters outside 1..2^24), SBN_ERR_DEVICE, SBN_ERR_CUDA.
 */
sbn_status sbn_probe_i8_mma(int32_t iters, int32_t* ctas, void* stream);

/*
 * Measurement helper (no counterpart in the method): the sparse INT8 rate of
 * the tensor pipe on CTA pairs. Launches clusters of two CTAs (one per SM)
 * on `stream`; in each pair one thread issues `iters` back-to-back
 * tcgen05.mma.sp.cta_group::2.kind::i8 instructions of M = 256, N = 224,
 * K = 64 logical positions (2 * 256 * 224 * 64 logical operations each, half
 * of them products of kept weights; int32 accumulation in tensor memory) on
 * shared-memory operands with valid 2:4 metadata -- the instruction and tile
 * shape of the 2:4 prefill contraction, with no loads in between. *pairs
 * (host) receives the number of pairs; the caller times the launch. Errors:
 * SBN_ERR_NULL, SBN_ERR_SHAPE (iters outside 1..2^24), SBN_ERR_DEVICE (no
 * pair can be resident), SBN_ERR_CUDA.
 */
sbn_status sbn_probe_i8_sparse_mma(int32_t iters, int32_t* pairs, void* stream);

/*
 * Test hook of the failure detection (no counterpart in the method): runs one
 * of the library's bounded device waits on a condition that never comes, with
 * a limit of limit_ns (1e3..1e8) nanoseconds, on `stream`. which = 0: an
 * mbarrier wait (the kind every pipelined kernel uses); which = 1: the grid
 * barrier of the weight quantizer. The wait gives up, records the timeout in
 * the device error word and the kernel returns normally, so the next
 * sbn_get_device_error returns SBN_ERR_TIMEOUT (and clears the word). No
 * asynchronous copy or MMA is outstanding when the wait gives up. Errors:
 * SBN_ERR_SHAPE (which or limit out of range), SBN_ERR_DEVICE, SBN_ERR_CUDA.
 */
sbn_status sbn_selftest_wait_timeout(int32_t which, int64_t limit_ns, void* stream);

/*
 * sbn_set_programmatic_launch -- library-wide launch setting (no counterpart
 * in the method). Enabled (the default), the kernels of sbn_quantize_acts,
 * of the contraction for T > 16 with a workspace (the weight expansion and
 * the CTA-pair kernel) and of the decode GEMV are launched with CUDA's
 * programmatic stream serialization: such a kernel may be scheduled while
 * the previous kernel on the stream is finishing, and it waits on the device
 * for that kernel to complete before it reads or writes global memory. Outputs are identical
 * either way; only the gaps between kernels change. enable = 0 launches
 * them with plain stream order. Returns the previous setting (1 or 0).
 * Launches already enqueued keep the setting they were made with.
 */
int32_t sbn_set_programmatic_launch(int32_t enable);

/*
 * sbn_get_device_error -- synchronizes `stream`, then reads and clears the
 * device error word of the current device. Returns SBN_OK, SBN_ERR_TIMEOUT
 * (a bounded device wait gave up; the affected outputs are unspecified) or
 * SBN_ERR_CUDA (the synchronization itself failed).
 */
sbn_status sbn_get_device_error(void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SBN_H */
