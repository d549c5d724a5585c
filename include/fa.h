/*
 * fa.h -- C ABI of the B200 (sm_100a) exact attention library (libfa_sm100.so):
 * the forward (fa_fwd, fa_fwd_qkvpacked; with a local window and ALiBi
 * fa_fwd_ext, fa_fwd_qkvpacked_ext; over variable-length sequences
 * fa_fwd_varlen) and its gradient (fa_bwd, fa_bwd_noalloc).
 *
 * Operation.  For every batch b, head h and query row i:
 *
 *     s_j    = scale * sum_c q[b,h,i,c] * k[b,h,j,c]      (key j visible from i)
 *     O[i]   = sum_j exp(s_j) v[b,h,j,:] / sum_j exp(s_j)
 *     LSE[i] = ln sum_j exp(s_j)
 *
 * i.e. O = softmax(scale * Q K^T [+ causal mask]) V, the standard attention of
 * "2.3 FlashAttention与IO感知注意力(1)" (aiknowledge.cn), section 1.1, and of
 * standard_attention in "flash_attention.py" (forceinjection.github.io),
 * computed with the tiled online-softmax recurrence of flash_attention_forward
 * in the same file, so the N x N score matrix never reaches device memory.
 * With causal != 0, key j is visible from query i iff j <= i (lower triangle
 * including the diagonal).  LSE is the natural-log logsumexp of the scaled
 * scores over the visible keys, stored in fp32.
 *
 * Precision.  Inputs and O are fp16 or bf16; scores, the softmax state and the
 * O accumulator are fp32; the softmax weights P are rounded to the input type
 * before the P V product (as on the tensor cores of every FlashAttention).
 *
 * Memory.  Every pointer is device memory owned by the caller; the library
 * allocates nothing per call (fa_bwd_noalloc writes its row statistic into a
 * device array the library owns).  Tensor pointers must be 16-byte aligned.
 *
 * Execution.  Calls are asynchronous on `stream` (a cudaStream_t; NULL is the
 * legacy default stream) and never synchronise.  The returned status covers
 * argument checks and the launch only; a kernel whose bounded internal wait
 * ran out (which does not happen in correct operation) is reported by
 * fa_device_status().
 *
 * Errors are returned, never raised: no call aborts the process.
 */
#ifndef FA_SM100_H
#define FA_SM100_H

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st; /* cudaStream_t is `struct CUstream_st *` */

enum fa_status {
  FA_OK = 0,
  FA_ERR_ARG = -1,         /* null pointer, B/H/N < 1, bad scale, size overflow */
  FA_ERR_ALIGN = -2,       /* a tensor pointer is not 16-byte aligned */
  FA_ERR_HEADDIM = -3,     /* d is not 64, 128 or 256 */
  FA_ERR_DTYPE = -4,       /* dtype is not FA_FP16 or FA_BF16 (or FA_E4M3 where taken) */
  FA_ERR_UNSUPPORTED = -5, /* dropout_p != 0 */
  FA_ERR_CUDA = -6,        /* a CUDA runtime / driver call failed */
  FA_ERR_TIMEOUT = -7,     /* a kernel gave up on a bounded wait */
  FA_ERR_DEVICE = -8,      /* the current device is not sm_100 (B200 class) */
  FA_ERR_SEQLENS = -9      /* (fa_device_status) a kernel met cu_seqlens out of range */
};

/* FA_E4M3 (fp8 e4m3 operands) is accepted by fa_fwd_fp8 only. */
enum fa_dtype { FA_FP16 = 0, FA_BF16 = 1, FA_E4M3 = 2 };

/*
 * Attention forward on separate Q, K, V.
 *
 *   q, k, v : [B, H, N, d] contiguous, element type `dtype` (read only)
 *   o       : [B, H, N, d] contiguous, element type `dtype` (written)
 *   lse     : [B, H, N] fp32 (written), or NULL to skip it
 *   d       : 64, 128 or 256 (the head dims up to 256 that the feature list of
 *             "flash-attention与TensorRT 10集成", blog.gitcode.com, names)
 *   scale   : logit scale; 0 means 1/sqrt(d) (softmax_scale=None of the packed
 *             call in section 5.2 of the intelliparadigm.com build guide).
 *             Negative, NaN and infinite values are rejected.
 *   causal  : 0 or 1
 *
 * Signature as the flash_attn_func(q, k, v) call of section 11.1 of the
 * intelliparadigm.com guide, in the [B, H, N, d] layout of the aiknowledge.cn
 * page, section 1.1.
 */
int fa_fwd(const void *q, const void *k, const void *v, void *o, float *lse, int B, int H, int N,
           int d, float scale, int causal, int dtype, struct CUstream_st *stream);

/*
 * Attention forward on a packed QKV tensor, as flash_attn_qkvpacked_func in
 * section 5.2 (and the keyword list of section 10.1) of
 * "Windows下RTX 3090编译Flash Attention 2.8.3全指南" (intelliparadigm.com).
 *
 *   qkv       : [B, N, 3, H, d] contiguous; index 0 / 1 / 2 of axis 2 is q / k / v
 *   o         : [B, N, H, d] contiguous (written)
 *   lse       : [B, H, N] fp32 (written), or NULL
 *   dropout_p : must be 0 (dropout is not part of this forward); else FA_ERR_UNSUPPORTED
 *   other arguments as fa_fwd.
 */
int fa_fwd_qkvpacked(const void *qkv, void *o, float *lse, int B, int N, int H, int d, float scale,
                     int causal, float dropout_p, int dtype, struct CUstream_st *stream);

/*
 * fa_fwd with the two masks the packed call's keyword list names besides
 * `causal`: a local window (window_size) and an ALiBi bias (alibi_slopes);
 * section 10.1 (and 5.2) of "Windows下RTX 3090编译Flash Attention 2.8.3全指南"
 * (intelliparadigm.com).  The page lists both keywords without defining them;
 * the reading taken here:
 *
 *   window_left, window_right : key j is visible from query i iff
 *       i - window_left <= j <= i + window_right, intersected with the causal
 *       mask when causal != 0; -1 leaves that side unbounded (window_size =
 *       (-1, -1) is the plain forward).  Values below -1 give FA_ERR_ARG.
 *       Every row sees at least its own key.
 *   alibi_slopes : device pointer to H fp32 slopes, or NULL.  The scaled score
 *       of key j in head h becomes scale * q_i . k_j - alibi_slopes[h] * |i - j|
 *       (the softmax, O and LSE are taken over these biased scores).  Slopes
 *       must be finite.  4-byte alignment required.
 *
 * Other arguments, layouts, results and errors as fa_fwd; fa_fwd is this call
 * with (-1, -1, NULL).  Key blocks that lie wholly outside every row's window
 * are neither loaded nor multiplied.
 */
int fa_fwd_ext(const void *q, const void *k, const void *v, void *o, float *lse, int B, int H,
               int N, int d, float scale, int causal, int window_left, int window_right,
               const float *alibi_slopes, int dtype, struct CUstream_st *stream);

/*
 * fa_fwd_qkvpacked with the local window and ALiBi bias of fa_fwd_ext: the
 * full keyword list of flash_attn_qkvpacked_func in section 10.1 of the
 * intelliparadigm.com guide except `deterministic` (this forward is always
 * deterministic: one fixed reduction order per output element).
 */
int fa_fwd_qkvpacked_ext(const void *qkv, void *o, float *lse, int B, int N, int H, int d,
                         float scale, int causal, float dropout_p, int window_left,
                         int window_right, const float *alibi_slopes, int dtype,
                         struct CUstream_st *stream);

/*
 * Forward on fp8 (e4m3) Q, K, V with per-tensor dequantisation factors: the
 * low-precision inference path of item 4, "低精度推理支持" (INT8 / FP8), of
 * "flash-attention与TensorRT 10集成" (blog.gitcode.com).  The page names FP8
 * inference without fixing a format; the reading taken here:
 *
 *   q, k, v   : [B, H, N, d] contiguous e4m3 codes (1 byte each: sign, 4
 *               exponent bits with bias 7, 3 mantissa bits, no infinities;
 *               the OCP "E4M3FN" format), read only
 *   descale_q, descale_k, descale_v : the real tensors are descale_x * x;
 *               finite and > 0
 *   o         : [B, H, N, d] contiguous bf16 (written)
 *   lse       : [B, H, N] fp32 (written), or NULL
 *   d         : 128 or 256 (a row must fill a 128-byte line; else FA_ERR_HEADDIM)
 *   scale, causal, stream : as fa_fwd
 *
 * It computes O = softmax(scale * (descale_q Q)(descale_k K)^T [+ causal])
 * (descale_v V) and its logsumexp.  S = Q K^T is formed from the e4m3 codes
 * on the tensor cores with fp32 accumulation; the softmax weights P are
 * rounded to e4m3 (3 mantissa bits, values near or below 2^-9 of the row's
 * reference flush to zero) before P V, the row sum uses the unrounded fp32
 * weights.  That rounding, not the inputs, sets the output error: see the
 * per-element bound the tests state.
 */
int fa_fwd_fp8(const void *q, const void *k, const void *v, void *o, float *lse, int B, int H,
               int N, int d, float scale, float descale_q, float descale_k, float descale_v,
               int causal, struct CUstream_st *stream);

/*
 * Forward over a batch of sequences of different lengths packed back to back
 * (the dynamic sequence lengths of item 3, "动态形状优化", of
 * "flash-attention与TensorRT 10集成", blog.gitcode.com): sequence b holds the
 * tokens cu_seqlens[b] .. cu_seqlens[b+1]-1, attends only to itself, and
 * query and key lengths are equal (self-attention).
 *
 *   q, k, v    : [total, H, d] contiguous, element type `dtype`
 *   o          : [total, H, d] contiguous (written)
 *   lse        : [H, total] fp32 (written), or NULL
 *   cu_seqlens : device pointer to batch + 1 int32 offsets, nondecreasing,
 *                cu_seqlens[0] = 0, cu_seqlens[batch] <= total
 *   batch      : number of sequences (>= 1)
 *   max_seqlen : >= every sequence length (host value; sizes the grid)
 *   total      : rows of q, k, v, o (>= 1)
 *   causal, window_left, window_right, alibi_slopes : per sequence, positions
 *                counted from the sequence's first token; as fa_fwd_ext
 *   other arguments as fa_fwd.
 *
 * The offsets are read on the device only.  A sequence whose offsets are out
 * of range (negative, decreasing, longer than max_seqlen, or past total) is
 * skipped -- its rows of o and lse are not written -- and fa_device_status()
 * then returns FA_ERR_SEQLENS.  All rows of q, k, v must hold finite values.
 */
int fa_fwd_varlen(const void *q, const void *k, const void *v, void *o, float *lse,
                  const int *cu_seqlens, int batch, int max_seqlen, int total, int H, int d,
                  float scale, int causal, int window_left, int window_right,
                  const float *alibi_slopes, int dtype, struct CUstream_st *stream);

/*
 * Gradient of fa_fwd: dQ, dK, dV for an upstream gradient dO of O.  The score
 * tile is recomputed from q, k and the forward's logsumexp, the
 * recomputation in the backward pass that sections 1 and 7 of the
 * intelliparadigm.com build guide describe; the rest is the chain rule through
 * the forward (dV = P^T dO, dS = P * (dO V^T - rowsum(dO * O)),
 * dQ = scale dS K, dK = scale dS^T Q).
 *
 *   q, k, v, o : [B, H, N, d] contiguous, element type `dtype` (read only);
 *                o and lse are the outputs of fa_fwd on the same q, k, v,
 *                scale and causal
 *   lse        : [B, H, N] fp32 (read only; required)
 *   dout       : [B, H, N, d] contiguous, element type `dtype` (read only)
 *   dq, dk, dv : [B, H, N, d] contiguous, element type `dtype` (written)
 *   workspace  : [B, H, N] fp32, caller-owned scratch (overwritten); the
 *                library allocates nothing
 *   d          : 64 or 128 (else FA_ERR_HEADDIM)
 *   scale, causal, dtype, stream: as fa_fwd
 *
 * Asynchronous on `stream`: three kernels (row statistic, dK/dV, dQ); the
 * last two run on a persistent grid of at most one CTA per SM.  When dq, dk
 * and dv are all 32-byte aligned their rows are written with 32-byte stores
 * (whole L2 sectors), else with 16-byte stores; the results are the same.
 * Returns FA_OK or a negative status; FA_ERR_ALIGN if a tensor pointer is not
 * 16-byte aligned or lse / workspace not 4-byte aligned.
 */
int fa_bwd(const void *q, const void *k, const void *v, const void *o, const float *lse,
           const void *dout, void *dq, void *dk, void *dv, float *workspace, int B, int H, int N,
           int d, float scale, int causal, int dtype, struct CUstream_st *stream);

/*
 * fa_bwd without the workspace argument: the fp32 row statistic goes into a
 * device array the library owns (a file-scope __device__ array, one per
 * device), so the call allocates nothing and the caller provides no scratch.
 *
 *   B * H * N must not exceed 8,388,608 (the array's size), else FA_ERR_ARG.
 *   The array is shared by every call on the device: two calls that may run
 *   at the same time (on different streams) must not both use this entry
 *   point; calls ordered on one stream may.
 *   Other arguments, results and errors as fa_bwd.
 */
int fa_bwd_noalloc(const void *q, const void *k, const void *v, const void *o, const float *lse,
                   const void *dout, void *dq, void *dk, void *dv, int B, int H, int N, int d,
                   float scale, int causal, int dtype, struct CUstream_st *stream);

/* Static text for a status code. */
const char *fa_strerror(int status);

/*
 * Reads (and, if clear != 0, resets) the current device's watchdog word.
 * Synchronises the current device first.  Returns FA_OK, FA_ERR_TIMEOUT when a
 * kernel gave up on a bounded wait, FA_ERR_SEQLENS when fa_fwd_varlen met
 * offsets out of range (`*detail`, if not NULL, receives the (role << 8) | site
 * code), or FA_ERR_CUDA.
 */
int fa_device_status(int clear, unsigned int *detail);

/*
 * Launches a one-warp kernel that waits on a barrier nobody arrives at, with a
 * bound of `limit_ns` nanoseconds.  The wait gives up, records FA_ERR_TIMEOUT in
 * the watchdog word and the kernel returns normally.  For testing the failure
 * path without a hang.  Returns the launch status.
 */
int fa_debug_watchdog_selftest(unsigned long long limit_ns, struct CUstream_st *stream);

/*
 * Debug: bound of every mbarrier wait inside the attention kernels launched
 * after this call, in nanoseconds (100 ns .. 10 s; 0 restores the default of
 * 2 s).  With a bound far below a tile's load or product time, the kernels'
 * waits run out: each CTA raises its abort flag, drains the loads and products
 * it issued, frees tensor memory and returns, and fa_device_status() reports
 * FA_ERR_TIMEOUT with the (role << 8) | site of the first wait that gave up.
 * For testing that failure path on the real kernels; outputs of such launches
 * are undefined.  Applies to every device and thread of the process.
 * Returns FA_OK or FA_ERR_ARG.
 */
int fa_debug_set_wait_limit(unsigned long long limit_ns);

/*
 * Test hook: y[i] = the kernel's software 2^x (the FMA-pipe exponential used
 * for a quarter of the softmax weights at head dim 256) for n device floats x.  Not part of the
 * attention method; exposed so that its error against exp2f can be measured.
 */
int fa_debug_exp2_poly(const float *x, float *y, int n, struct CUstream_st *stream);

/* Grid size (CTAs) fa_fwd would launch for this problem on the current device, or < 0. */
int fa_launch_ctas(int B, int H, int N, int d, int causal);

/* Library version: major * 10000 + minor * 100 + patch. */
int fa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FA_SM100_H */
