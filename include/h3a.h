/*
 * h3a.h -- C ABI of the B200 (sm_100a) attention core for H3-style video DiTs.
 *
 * One DiT self-attention core per call sequence:
 *   h3a_qk_norm_rope  fused QK-RMSNorm + 3D RoPE over Q and K
 *   h3a_route         blockwise KV-block router (pool -> fp32 scores -> top-k)
 *   h3a_attention     bidirectional attention, dense or over routed KV blocks
 *
 * Conventions shared by every call
 *   - Tensors are bf16 (raw 16-bit words), laid out [B, N, heads, head_dim]
 *     with head_dim contiguous and element strides given by h3a_qkv_desc.
 *     Token n of the (T, H, W) grid is n = (t*H + h)*W + w.
 *   - head_dim must be 96 (hidden 5376 / 56 heads); the router and attention
 *     also take 128 (SubBlock's stated head size; the same hidden width as
 *     42 heads), the prologue does not (its 3D RoPE layout is defined for 96
 *     channels).  block must be 128.
 *   - All pointers are DEVICE pointers owned by the caller, 16-byte aligned;
 *     strides are multiples of 8 elements (16 bytes).  The library never
 *     allocates or frees device memory per call; the router's scratch is a
 *     caller workspace sized by h3a_route_workspace_size.  Its only device
 *     state is static: the status word below and the fixed scratch array of
 *     h3a_route_noalloc, both resident on every GPU that loads the library.
 *   - Calls are asynchronous on the caller's stream.  A status other than
 *     H3A_OK means nothing was launched, except H3A_ERR_CUDA, returned when a
 *     launch itself failed.  Device-side failures (a bounded pipeline wait that
 *     expired) are latched in a per-device status word and reported by
 *     h3a_last_device_error.
 *   - Thread safety: calls may be issued from several host threads.  A call
 *     writes only its arguments, except for two pieces of shared device state:
 *     kernels OR timeouts into the per-device status word (taken atomically by
 *     h3a_last_device_error), and h3a_route_noalloc works in one scratch array
 *     per device, so its calls race when they overlap on the GPU.
 */
#ifndef H3A_H_
#define H3A_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* h3a_stream_t; /* a cudaStream_t; NULL = legacy default stream */

typedef enum {
    H3A_OK = 0,
    H3A_ERR_INVALID_ARG = 1, /* null/misaligned pointer, inconsistent sizes, bad sparsity */
    H3A_ERR_UNSUPPORTED = 2, /* head_dim not supported by the call, block != 128, sizes beyond int32 range */
    H3A_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed (see h3a_last_cuda_error_string) */
    H3A_ERR_TIMEOUT = 4,     /* a bounded device-side wait expired; results are undefined */
    H3A_ERR_WORKSPACE = 5    /* router workspace null or too small */
} h3a_status;

/* Token grid of one clip latent: N = T*H*W tokens. */
typedef struct {
    int32_t T, H, W;
} h3a_grid;

/* Shape and element strides of a [B, N, heads, head_dim] bf16 tensor.
 * Q, K, V and O of one call share this descriptor. */
typedef struct {
    int32_t B, N, heads, head_dim;
    int64_t stride_b, stride_n, stride_h; /* in elements; head_dim is contiguous */
} h3a_qkv_desc;

/* Fused QK-RMSNorm + 3D RoPE.
 * Source: news.cocoloop.cn MiniMax-H3 SGLang report, section "Erst drei
 * übereinandergelegte Beschleunigungsebenen" (QK-RMSNorm with 3D RoPE fused
 * into one kernel, result unchanged); 3D multimodal RoPE and the 96-wide heads
 * from the 52hbtv.com H3-Image page, section 二, model table.
 * For every token n and head h of Q (and of K):
 *   y = x / sqrt(mean(x^2) + eps) * gamma        (over the head's 96 channels)
 *   then channels [0,32) turn with t, [32,64) with h, [64,96) with w: the pair
 *   (32a+2j, 32a+2j+1) rotates by pos_a * theta^(-2j/32), j = 0..15;
 *   computed in fp32, rounded once to bf16 (round to nearest even).
 * q, k      : input tensors (device, bf16, layout d).
 * gamma_q/k : fp32 [96] gains (device).
 * q_out/k_out: outputs (device, layout d); may equal q/k (in place), must not
 *             otherwise overlap them.
 * Errors: INVALID_ARG if any pointer is null or misaligned, T*H*W != N, or
 * eps < 0; UNSUPPORTED if head_dim != 96. */
h3a_status h3a_qk_norm_rope(const void* q, const void* k, const h3a_qkv_desc* d,
                            const float* gamma_q, const float* gamma_k, h3a_grid grid,
                            double theta, float eps, void* q_out, void* k_out,
                            h3a_stream_t stream);

/* Number of KV blocks kept per query block for a given sparsity:
 * k = clamp(ceil((1 - sparsity) * nkv - 1e-9), 1, nkv).
 * Returns -1 if sparsity is outside [0, 1) or nkv < 1. */
int64_t h3a_route_k(int64_t nkv, double sparsity);

/* h3a_qk_norm_rope with the RMSNorm spanning the token's whole hidden state:
 * the other reading of "QK-RMSNorm" on the same page (fused-operator
 * paragraph).  For every token n of Q (and of K):
 *   r = 1 / sqrt(mean over all heads x 96 channels of x^2 + eps)
 *   y[h, c] = x[h, c] * r * gamma[h * 96 + c], then the per-head 3D RoPE of
 *   h3a_qk_norm_rope; fp32 arithmetic, one rounding to bf16.
 * gamma_q/k : fp32 [heads * 96] gains (device, 16-byte aligned).
 * Other arguments, layouts and errors: as h3a_qk_norm_rope, and UNSUPPORTED
 * for more than 74 heads or B * N >= 2^31 (one CTA per token holds the
 * token's rows). */
h3a_status h3a_qk_fullnorm_rope(const void* q, const void* k, const h3a_qkv_desc* d,
                                const float* gamma_q, const float* gamma_k, h3a_grid grid,
                                double theta, float eps, void* q_out, void* k_out,
                                h3a_stream_t stream);

/* Sparsity to use at a denoising step: the router prunes KV blocks from the
 * first_sparse_step-th step on (news.cocoloop.cn MiniMax-H3 SGLang report,
 * SubBlock paragraph: from the 10th step), steps counted from 1.  Returns
 * `sparsity` when step >= first_sparse_step, 0.0 (dense attention) before,
 * and -1.0 if step < 1, first_sparse_step < 1 or sparsity is outside [0, 1).
 * Host only; no device work. */
double h3a_step_sparsity(int32_t step, int32_t first_sparse_step, double sparsity);

/* Bytes of device workspace h3a_route needs for the fp32 block means,
 * nblk = ceil(N / block), head_dim 96 or 128: Q's as [B, heads, nblk,
 * head_dim], then, from the next 256-byte boundary, K's channel-major as
 * [B, heads, head_dim, nblk rounded up to 4], each part rounded up to 256
 * bytes.  Returns INVALID_ARG/UNSUPPORTED for bad descriptors. */
h3a_status h3a_route_workspace_size(const h3a_qkv_desc* d, int32_t block, size_t* bytes);

/* Blockwise KV-block router.
 * Source: news.cocoloop.cn MiniMax-H3 SGLang report, SubBlock paragraph of
 * section "Erst drei übereinandergelegte Beschleunigungsebenen" (a blockwise
 * sparse router prunes the KV blocks, sparsity 0.75 or 0.80); pooling,
 * scoring and selection as fixed by the problem statement:
 *   qbar_i, kbar_j = fp32 means of the 128-token blocks (the tail block over
 *   its real length), score S_ij = (qbar_i . kbar_j) / sqrt(head_dim) in fp32,
 *   per (b, h, i) keep the k highest scores, ties to the lower j.
 * q, k       : prologue outputs (device, bf16, layout d).
 * block_idx  : device int32 [B, heads, nblk, k], each row ascending.
 * k_out      : host; receives k (may be NULL).
 * workspace  : device, at least h3a_route_workspace_size bytes, 16-B aligned.
 * Errors: INVALID_ARG for null pointers or sparsity outside [0, 1);
 * UNSUPPORTED for block != 128, head_dim other than 96 / 128, more key blocks
 * than the score kernel holds (each of its CTAs keeps 8 query blocks' fp32
 * scores against every key block in 200 KB of shared memory: ceil(N / 128)
 * <= 6,048 at head_dim 96, 6,016 at 128) or B * heads > 65,535; WORKSPACE if
 * the workspace is null or ws_bytes is too small.  Nothing is launched when a
 * check fails. */
h3a_status h3a_route(const void* q, const void* k, const h3a_qkv_desc* d, double sparsity,
                     int32_t block, int32_t* block_idx, int64_t* k_out, void* workspace,
                     size_t ws_bytes, h3a_stream_t stream);

/* h3a_qk_norm_rope that also pools its outputs for the router, so that
 * h3a_route_pooled can skip reading Q and K back from device memory.
 * Source: the fused prologue of h3a_qk_norm_rope and the block pooling of
 * h3a_route (news.cocoloop.cn MiniMax-H3 SGLang report: fused QK-RMSNorm +
 * 3D RoPE in section "Erst drei übereinandergelegte Beschleunigungsebenen",
 * SubBlock's blockwise router in the same section).
 * Writes q_out / k_out exactly as h3a_qk_norm_rope does, and into workspace
 * the fp32 means, over each 128-token block (the tail block over its real
 * length), of the rounded outputs: the same bytes h3a_route's pooling leaves
 * in its workspace (the layout h3a_route_workspace_size describes), bit for
 * bit.
 * workspace : device, at least h3a_route_workspace_size(d, 128) bytes,
 *             16-B aligned, owned by the caller; it must not overlap q, k,
 *             q_out or k_out.
 * Other arguments, layouts and errors: as h3a_qk_norm_rope; WORKSPACE if the
 * workspace is null, misaligned or too small; UNSUPPORTED if B > 65535.  Q
 * and K stream through shared memory with TMA; a bounded pipeline wait that
 * expired is reported by h3a_last_device_error (H3A_ERR_TIMEOUT). */
h3a_status h3a_qk_norm_rope_pool(const void* q, const void* k, const h3a_qkv_desc* d,
                                 const float* gamma_q, const float* gamma_k, h3a_grid grid,
                                 double theta, float eps, void* q_out, void* k_out,
                                 void* workspace, size_t ws_bytes, h3a_stream_t stream);

/* The scoring and top-k half of h3a_route, from block means that
 * h3a_qk_norm_rope_pool left in the workspace (same source and rule as
 * h3a_route).  d describes the Q/K tensors that were pooled; block_idx,
 * k_out and the result are those of h3a_route on the prologue's outputs.
 * The workspace is only read.  Errors: as h3a_route, and UNSUPPORTED for a
 * head_dim other than 96 (the prologue's only width). */
h3a_status h3a_route_pooled(const h3a_qkv_desc* d, double sparsity, int32_t block,
                            int32_t* block_idx, int64_t* k_out, const void* workspace,
                            size_t ws_bytes, h3a_stream_t stream);

/* Gated residual followed by the AdaLN update, one pass over device memory.
 * Source: news.cocoloop.cn MiniMax-H3 SGLang report, section "Erst drei
 * übereinandergelegte Beschleunigungsebenen", fused-operator paragraph (the
 * AdaLN update and the gated residual path fused like QK-RMSNorm + 3D RoPE,
 * no result changed); the page gives no formulas, these are the DiT block's.
 * For batch b and token row r of width C:
 *   h = x + gate[b] * f, rounded once to bf16 (f == NULL: h = x)
 *   y = (h - mean(h)) / sqrt(var(h) + eps) * (1 + scale[b]) + shift[b]
 *   (LayerNorm without affine, statistics over the C channels of the rounded
 *   h, fp32 arithmetic, y rounded once to bf16).
 * x, f        : device bf16 [B, rows, width], contiguous; f may be NULL.
 * gate, shift, scale: device fp32 [B, width] (gate only read when f != NULL).
 * h_out       : device bf16 [B, rows, width], written when f != NULL (then
 *               required; may equal x); ignored when f == NULL.
 * y_out       : device bf16 [B, rows, width]; must not overlap x, f or h_out.
 * All pointers 16-byte aligned.
 * Errors: INVALID_ARG for null/misaligned pointers, width not a positive
 * multiple of 8, eps < 0; UNSUPPORTED for width > 14336 or B*rows >= 2^31. */
h3a_status h3a_residual_adaln(const void* x, const void* f, const float* gate, const float* shift,
                              const float* scale, int32_t B, int64_t rows, int32_t width, float eps,
                              void* h_out, void* y_out, h3a_stream_t stream);

/* SwiGLU activation: out = silu(a) * b = a / (1 + exp(-a)) * b.
 * Source: the same fused-operator paragraph (the SwiGLU activation).
 * in  : device bf16 [rows, 2 * ffn_width], contiguous; each row is a (the
 *       first ffn_width channels) followed by b.
 * out : device bf16 [rows, ffn_width], contiguous; must not overlap in.
 * fp32 arithmetic, one rounding to bf16.  Both pointers 16-byte aligned.
 * Errors: INVALID_ARG for null/misaligned pointers or ffn_width not a
 * positive multiple of 8. */
h3a_status h3a_swiglu(const void* in, int64_t rows, int32_t ffn_width, void* out, h3a_stream_t stream);

/* Device workspace h3a_residual_diff needs: 32 KB (partial sums). */
#define H3A_RESIDUAL_DIFF_WORKSPACE_BYTES ((size_t)32768)

/* The Cache-DiT reuse decision between two denoising steps.
 * Source: news.cocoloop.cn MiniMax-H3 SGLang report, Cache-DiT paragraph
 * after the fused-operator one (results are reused between adjacent steps
 * when a residual-difference threshold allows: 0.04 conservative, 0.08 in
 * stride mode); read as the relative L1 difference
 *   rel = sum_i |cur_i - prev_i| / sum_i |prev_i|
 * (0 if both are zero, +inf if only prev is), reuse = rel < threshold.
 * cur, prev : device bf16 arrays of n values (n a positive multiple of 8),
 *             16-byte aligned.
 * workspace : device, >= H3A_RESIDUAL_DIFF_WORKSPACE_BYTES, 16-B aligned.
 * rel_out   : device fp64 scalar; reuse_out: device int32 scalar or NULL.
 * Sums: each 8 values in fp32, then fp64 in a fixed order (deterministic);
 * rel agrees with an fp64 sum to about 1e-7 relative, so a decision can only
 * differ from an exact one for rel within that band of the threshold.
 * Errors: INVALID_ARG for null/misaligned pointers, n not a positive multiple
 * of 8, threshold < 0 or NaN; WORKSPACE if the workspace is null or small. */
h3a_status h3a_residual_diff(const void* cur, const void* prev, int64_t n, double threshold,
                             void* workspace, size_t ws_bytes, double* rel_out, int32_t* reuse_out,
                             h3a_stream_t stream);

/* Capacity of the scratch built into h3a_route_noalloc: 64 MiB.  The router
 * keeps two fp32 block means of head_dim values per (batch, head, block) (the
 * layout h3a_route_workspace_size gives), so it holds about
 * B * heads * ceil(N / 128) <= 64 MiB / (8 * head_dim) blocks: some 87,000 at
 * head_dim 96 (e.g. 56 heads of a 124,992-token clip), 65,000 at 128; a shape
 * whose workspace size exceeds 64 MiB is refused. */
#define H3A_ROUTE_NOALLOC_MAX_BYTES ((size_t)64 << 20)

/* h3a_route for callers that cannot allocate device memory (no counterpart on
 * the pages).  Some callers have no allocator at hand where they route -- an
 * embedding runtime that hands out none after start-up, code inside a host
 * callback or another allocator's critical section, a serving loop with a
 * fixed memory budget -- so this variant takes no workspace: its scratch is a
 * file-scope device array of H3A_ROUTE_NOALLOC_MAX_BYTES that every GPU
 * loading the library holds until process exit.  It calls no cudaMalloc,
 * cudaFree or other allocating routine.  Arguments and results are those of
 * h3a_route.
 * The first call on a device resolves the array's device address for that
 * device (cudaGetSymbolAddress with the device current): make that first call
 * before any stream capture.  Every call shares the one array and overwrites
 * what it reads, so nothing needs clearing, but calls whose executions overlap
 * on the GPU (other streams, other host threads) race on it.
 * Errors: those of h3a_route; H3A_ERR_WORKSPACE when the shape needs more than
 * H3A_ROUTE_NOALLOC_MAX_BYTES of scratch (h3a_route_workspace_size bytes);
 * H3A_ERR_CUDA if the set-up fails. */
h3a_status h3a_route_noalloc(const void* q, const void* k, const h3a_qkv_desc* d, double sparsity,
                             int32_t block, int32_t* block_idx, int64_t* k_out, h3a_stream_t stream);

/* Bidirectional attention O = softmax(scale * Q K^T) V per (b, head).
 * Source: dense lossless path of the news.cocoloop.cn MiniMax-H3 SGLang
 * report (opening quote: no approximation; SSIM 1.0000) and its SubBlock
 * sparse attention (same page; "Ein paar Grenzen": long non-causal
 * attention, BF16).
 * block_idx == NULL: dense, every query attends to all N keys.
 * block_idx != NULL: device int32 [B, heads, nblk, k_blocks] routed lists
 *   (ascending, distinct, in [0, nblk)); the queries of block i attend exactly
 *   to the tokens of the KV blocks listed for (b, h, i), softmax renormalised
 *   over them.
 * scale: logit scale; 0 selects 1/sqrt(head_dim).
 * o: output (device, bf16, layout d), must not overlap q, k or v.
 * Tensor-core path: TMA tiles, tcgen05.mma with TMEM accumulators, fp32
 * online softmax, one rounding of O to bf16.
 * Errors: INVALID_ARG for null/misaligned pointers or k_blocks outside
 * [1, nblk] in sparse mode; UNSUPPORTED for head_dim other than 96 / 128,
 * block != 128, or N >= 2^31. */
h3a_status h3a_attention(const void* q, const void* k, const void* v, const h3a_qkv_desc* d,
                         const int32_t* block_idx, int32_t k_blocks, int32_t block, float scale,
                         void* o, h3a_stream_t stream);

/* Human-readable name of a status. Never NULL. */
const char* h3a_status_string(h3a_status s);

/* Text of the last CUDA error seen by the calling host thread ("" if none). */
const char* h3a_last_cuda_error_string(void);

/* Takes the current device's status word: after everything already queued
 * on `stream`, one atomic exchange reads the word and clears it, then the call
 * synchronises `stream` and returns H3A_OK, or H3A_ERR_TIMEOUT if a bounded
 * device wait expired since the word was last taken.  The word is shared by
 * every stream of the device: a timeout raised by a kernel on another stream is
 * reported to exactly one caller -- this one if that kernel had already raised
 * it, else a later one; it is never lost, and never reported twice.  Readers
 * in one process are serialised.  H3A_ERR_CUDA if the launch, the copy or the
 * synchronisation failed. */
h3a_status h3a_last_device_error(h3a_stream_t stream);

/* Self-check of the bounded-wait path (no counterpart on the pages): launches
 * one CTA that waits on a barrier nothing ever completes, with a limit of
 * `limit_us` microseconds, then synchronises.  Returns H3A_ERR_TIMEOUT when
 * the limit expired and was reported through the status word (the expected
 * result), H3A_OK if it was not, H3A_ERR_CUDA on a CUDA failure.  Clears the
 * status word afterwards. */
h3a_status h3a_selftest_wait_timeout(uint32_t limit_us, h3a_stream_t stream);

/* Self-check of the tensor-core building blocks used by h3a_attention (no
 * counterpart on the pages): one CTA loads a 128x96 tile A and a 128x96 tile
 * B (bf16, row-major, device) with TMA, computes S = A B^T (fp32 [128,128])
 * with tcgen05.mma into tensor memory, rounds S to bf16 into tensor memory and
 * computes R = bf16(S) C (fp32 [128,96]) with C = B read as a [128 kv, 96]
 * MN-major operand.  Writes S and R (device fp32).  For diagnosing a new
 * toolkit or driver. */
h3a_status h3a_selftest_mma(const void* a, const void* b, float* s_out, float* r_out,
                            h3a_stream_t stream);

/* Self-check of the exponential of the attention softmax (no counterpart on
 * the pages): y[i] = 2^x[i] for n device floats, by the instruction the
 * softmax evaluates every exponential with (ex2.approx.ftz.f32, in the log2
 * domain).  Asynchronous on `stream`.  INVALID_ARG for n < 0 or null /
 * misaligned pointers. */
h3a_status h3a_selftest_exp2(const float* x, float* y, int32_t n, h3a_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* H3A_H_ */
