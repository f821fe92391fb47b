/*
 * ss.h -- C ABI of libss: quantized matmul on the Blackwell (sm_100a) sparse
 * tensor cores for structured-sparse weights.
 *
 * The method (SlideSparse, "SlideSparse: 布局稀疏边界", 66bd.net, and the
 * "SlideSparse" write-up, omica.com.cn): a weight pattern (2Nh-2):2Nh --
 * 2:4, 4:6, 6:8, 8:10 -- keeps 2Nh-2 of every 2Nh consecutive weights along
 * K.  Nh-1 overlapping windows of width 4 and stride 2 cover each group; every
 * window holds at most two non-zeros, so the weight becomes hardware 2:4 over
 * a K grown by 2(Nh-1)/Nh (1.5x for 6:8).  The activation is "lifted" to match
 * by an index map fused into its per-token quantisation.
 *
 * Conventions for every call:
 *  - All data pointers are DEVICE pointers owned by the caller; the library
 *    allocates no device memory.  Pointers must be 16-byte aligned.
 *  - Matrices are row-major.  W is [N, K] (output channels x reduction),
 *    X is [M, K] (tokens x reduction), Y is [M, N].
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *    default stream).  Argument, alignment and architecture errors are
 *    returned before anything is launched.  Errors found on the device (a
 *    NaN/Inf weight, a bounded wait that ran out) are recorded in a device
 *    status word read by ss_get_device_status().
 *  - Only sm_100 devices are supported; others return SS_ERR_ARCH.  There is
 *    no CPU fallback.
 *  - Buffer sizes follow from ss_slide_shape() / ss_act_2to4_shape().
 */
#ifndef SS_H_
#define SS_H_

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *ss_stream_t; /* same type as cudaStream_t */

typedef enum {
    SS_OK = 0,
    SS_ERR_INVALID_ARG = 1, /* bad size, pattern, dtype or NULL pointer   */
    SS_ERR_UNSUPPORTED = 2, /* valid but beyond what the kernels handle   */
    SS_ERR_ALIGNMENT = 3,   /* pointer not 16-byte aligned                 */
    SS_ERR_ARCH = 4,        /* current device is not sm_100                */
    SS_ERR_CUDA = 5,        /* a CUDA runtime/driver call failed           */
    SS_ERR_TIMEOUT = 6,     /* a device-side bounded wait ran out          */
    SS_ERR_DATA = 7         /* NaN or Inf in a weight being compressed     */
} ss_status;

typedef enum { SS_IN_F32 = 0, SS_IN_BF16 = 1 } ss_in_dtype;
/* Stored operand type.  SS_BF16 is the 16-bit tier (the "2:4 + FP16" tier
 * of the "add 2:4 or drop a precision tier?" study, paper-daily 2610.28947,
 * section 1; the 16-bit rows of the SlideSparse precision list, 66bd.net):
 * values are kept as bf16 (round to nearest even from the input), two bytes
 * each, with no scale -- every s_w / s_x / s_a / s_b argument is then unused
 * and may be NULL, and the GEMM epilogue is y = fp32 acc (then bf16 RNE). */
typedef enum { SS_INT8 = 0, SS_FP8_E4M3 = 1, SS_BF16 = 2 } ss_qdtype;
typedef enum { SS_OUT_F32 = 0, SS_OUT_BF16 = 1 } ss_out_dtype;

/* Sparsity pattern keep:group; {2,4},{4,6},{6,8},{8,10}; {0,0} = dense. */
typedef struct {
    int32_t keep;
    int32_t group;
} ss_pattern;

/* Parse "2:4", "4:6", "6:8", "8:10" or "dense" (the pattern strings of the
 * SlideSparse write-up, omica.com.cn, 4.1 and 6.1). */
ss_status ss_parse_pattern(const char *s, ss_pattern *out);

/* Shapes for a reduction length K under pattern p (SlideSparse, 66bd.net,
 * Fig. 2: 8 elements become 12 for 6:8):
 *   K_pad  = 2Nh * ceil(K / 2Nh)          (zero padding of K)
 *   K_lift = 4 (Nh-1) * ceil(K / 2Nh)     (lifted reduction length)
 *   K_lp   = K_lift rounded up to 128     (what the GEMM consumes)
 * Dense: K_pad = K_lift = K, K_lp = K rounded up to 128. */
ss_status ss_slide_shape(ss_pattern p, int64_t K, int64_t *K_pad, int64_t *K_lift,
                         int64_t *K_lp);

/* K_lp of an online-pruned 2:4 activation: K rounded up to 4, then to 128. */
ss_status ss_act_2to4_shape(int64_t K, int64_t *K_lp);

/* Size in bytes of a metadata buffer (Wm, Xm) for `rows` rows of K_lp
 * lifted elements.  Metadata is stored tile-major so that the 2:4 selectors
 * of 128 rows x 128 K (the unit the GEMM stages) are one contiguous 2 KB
 * block, which the tensor-memory copy takes as is:
 *   byte b of row r (its nibbles as in the row layout [rows, K_lp/8]) is at
 *   ((r / 128) * (K_lp / 128) + b / 16) * 2048 + (r % 128) * 16 + b % 16.
 * Rows are padded to a multiple of 128; padding rows are zero.
 * SS_BF16 metadata adds one exchange inside each block: the 16-bit sparse
 * MMA reads the selectors of rows r and r + 8 (r % 16 < 8) for one MMA as
 * the two 2-byte halves of one 4-byte word, so bytes b of row r with
 * b % 4 in {2, 3} and r % 16 < 8 swap places with bytes b - 2 of row r + 8:
 * byte b of row r is at the offset above for row (r & ~8) | (b & 2) << 2 and
 * byte (b & ~2) | (r & 8) >> 2.
 * Returns 0 for rows < 1 or K_lp not a positive multiple of 128. */
int64_t ss_meta_bytes(int64_t rows, int64_t K_lp);

/* Offline weight compression (SlideSparse write-up, omica.com.cn, 2.2 weight
 * preprocessing and 3.1; LLM-Compressor W8A8 rows: channel-wise weights).
 * Per row of W[N, K] (f32 or bf16):
 *   1. magnitude prune each group of 2Nh along K to its 2Nh-2 largest |w|
 *      (ties keep the lower index; K zero-padded to K_pad);
 *   2. s_w[n] = absmax of the kept weights / Q (Q = 127 INT8, 448 E4M3);
 *      q = RNE(w * (Q / absmax)), INT8 clamped to [-127, 127], E4M3 saturated;
 *   3. assign every kept position to one of the Nh-1 windows by ascending
 *      first fit (window j covers 2j..2j+3 of its group);
 *   4. pack each window as two values (ascending local index, padded with the
 *      lowest unused indices, padded slots hold 0) and a nibble
 *      idx0 | idx1 << 2.
 * Outputs (pattern != dense):
 *   Wv  [N, K_lp/2] bytes   stored values, window w at bytes 2w, 2w+1
 *   Wm  ss_meta_bytes(N, K_lp) bytes, tile-major (see ss_meta_bytes): row n's
 *       nibbles, window w in its byte w/2, low nibble = even w
 *   s_w [N] fp32
 * Dense: Wv is [N, K_lp] (per-channel quantised W, zero padded), Wm unused
 * (may be NULL).  A NaN/Inf weight sets SS_ERR_DATA in the device status.
 * SS_BF16: step 2 is bf16 rounding with no scale; Wv holds 2-byte values
 * ([N, K_lp/2] bf16, dense [N, K_lp] bf16); s_w is not written. */
ss_status ss_compress_weight(const void *W, ss_in_dtype in_dtype, int64_t N, int64_t K,
                             ss_pattern p, ss_qdtype q, void *Wv, void *Wm, float *s_w,
                             ss_stream_t stream);

/* Fused per-token quantisation + activation lifting (SlideSparse, 66bd.net:
 * lifting is an index map fused into the per-token quant kernel; write-up
 * 3.2: window i reads 4 consecutive activations at
 * base = 2Nh * (i / (Nh-1)) + 2 * (i % (Nh-1)), four bytes packed per word).
 * Per token m of X[M, K]: a = max_k |x|, s_x[m] = a / Q, q = RNE(x * (Q / a));
 * Xq_lift[m, 4i + t] = q(X[m, base_i + t]) (0 past K and past K_lift).
 * Outputs: Xq_lift [M, K_lp] bytes, s_x [M] fp32.  Dense: identity map.
 * SS_BF16: no quantisation; Xq_lift [M, K_lp] holds the bf16 of X under the
 * same map (0 past K and K_lift); s_x is not written. */
ss_status ss_quant_lift_act(const void *X, ss_in_dtype in_dtype, int64_t M, int64_t K,
                            ss_pattern p, ss_qdtype q, void *Xq_lift, float *s_x,
                            ss_stream_t stream);

/* Online 2:4 prune + compress of an activation (the "add 2:4 or drop a
 * precision tier?" study, paper-daily 2610.28947, section 1: operands made on
 * the fly must be pruned and compressed before every matmul).  Per token m:
 * in each group of 4 along K keep the two largest |x| (ties keep the lower
 * index), s_x[m] = row absmax / Q, quantise the kept values, pack as in
 * ss_compress_weight.  Outputs Xv [M, K_lp/2], Xm (ss_meta_bytes(M, K_lp)
 * bytes, tile-major), s_x [M] with K_lp from ss_act_2to4_shape().
 * SS_BF16: the kept values are stored as bf16 (Xv [M, K_lp/2] bf16), no
 * scale; s_x is not written. */
ss_status ss_prune_act_2to4(const void *X, ss_in_dtype in_dtype, int64_t M, int64_t K,
                            ss_qdtype q, void *Xv, void *Xm, float *s_x, ss_stream_t stream);

/* Sparse GEMM on the sm_100a sparse tensor cores (tcgen05.mma.sp, TMEM
 * accumulators, TMA-staged tiles), with the dequant epilogue
 *   Y[m, n] = ((float)acc[m, n] * s_x[m]) * s_w[n]   (fp32, then bf16 RNE)
 * sparse_operand = 0: A = weight.  Av = Wv [N, K_lp/2], Am = Wm (tile-major),
 *                     s_a = s_w [N]; B = Xq_lift [M, K_lp], s_b = s_x [M].
 * sparse_operand = 1: A = activation.  Av = Xv [M, K_lp/2], Am = Xm
 *                     (tile-major), s_a = s_x [M]; B = Wq [N, K_lp] (dense),
 *                     s_b = s_w [N].
 * acc is exact int32 for INT8 and fp32 (tensor-core accumulation) for E4M3
 * and SS_BF16 (kind::f16; Av, B hold 2-byte values, s_a / s_b unused).
 * K_lp must be a positive multiple of 128; M, N in [1, 2^31) (SS_ERR_UNSUPPORTED when the
 * output-tile count passes 2^31).
 * Kernel shape: with more than 128 weight rows and bf16 Y, large problems
 * run output tiles of 256 channels x 2 token tiles (one A slice feeds two
 * MMAs), the rest (and every SS_BF16 problem) 256 x 1.  The choice follows the wave count; the
 * environment variable SS_SPARSE_KERNEL=narrow|wide pins it (same results). */
ss_status ss_sparse_gemm(int sparse_operand, const void *Av, const void *Am, const float *s_a,
                         const void *B, const float *s_b, int64_t M, int64_t N, int64_t K_lp,
                         ss_qdtype q, void *Y, ss_out_dtype out_dtype, ss_stream_t stream);

/* Dense GEMM of the same construction (tcgen05.mma), the like-for-like
 * comparison: Y = dequant(Xq [M, K_p] . Wq [N, K_p]^T) with the same
 * epilogue; Xq from ss_quant_lift_act(dense), Wq from
 * ss_compress_weight(dense).  K_p must be a positive multiple of 128.
 * SS_BF16: Xq, Wq hold bf16 ([M, K_p], [N, K_p]); s_x, s_w unused. */
ss_status ss_dense_gemm(const void *Xq, const float *s_x, const void *Wq, const float *s_w,
                        int64_t M, int64_t N, int64_t K_p, ss_qdtype q, void *Y,
                        ss_out_dtype out_dtype, ss_stream_t stream);

/* ------------------------------------------------------------------------
 * NVFP4 with pairwise sparsity (the Blackwell sparse FP4 of the "add 2:4 or
 * drop a precision tier?" study, paper-daily 2610.28947, 3.3: 2 of every 4
 * adjacent pairs in 8 elements kept; the NVFP4 row of the LLM-Compressor
 * compression-schemes page: E2M1 elements, a local scale per group of 16,
 * a global scale per tensor).
 *
 * Elements are E2M1 codes (sign << 3 | magnitude index of 0, .5, 1, 1.5, 2,
 * 3, 4, 6), two per byte, low nibble = lower K.  Local scales are UE4M3
 * (E4M3 with the sign clear).  With global scale g = amax / 2688 (fp32), a
 * block of absolute maximum a gets s = UE4M3(a / (6 g)), d = s * g,
 * inv = 1 / d (0 if d = 0) and codes E2M1(x * inv), round to nearest even,
 * saturating, each step one fp32 operation.
 *
 * A pattern keep:group counts PAIRS of adjacent elements: 2:4 is the
 * hardware's pairwise 4:8, and 4:6, 6:8, 8:10 slide windows of 4 pairs with
 * a stride of 2 pairs, exactly as the 8-bit patterns slide elements.  A
 * window of 4 pairs stores its 2 kept pairs (ascending) and the nibble
 * p0 | p1 << 2.  The sparse tensor-core instruction applies one scale per
 * 32 lifted K to both operands: 16 stored values of the sparse weight, 32
 * elements of the dense activation; the dense comparator uses 16.
 *
 * Scale storage is tile-major in 512-byte blocks, the source shape of the
 * tensor-memory copy: scale j (= k / block) of row r is at
 *   ((r / 128) * (n_blocks / 4) + j / 4) * 512 + (r % 32) * 16
 *     + ((r % 128) / 32) * 4 + j % 4,      n_blocks = K_lp / block,
 * rows padded to 128 (padding scales 0).  Sparse metadata is the tile-major
 * layout of ss_meta_bytes() over K_lp / 2 (16 bytes cover 256 lifted K).
 * ------------------------------------------------------------------------ */

/* Lifted and padded lengths for NVFP4 under pattern p (counted in pairs):
 * K_lift = 2 * (the pair slide's lifted length), K_lp = K_lift rounded up
 * to 256.  Dense: K_lift = K, K_lp = K rounded up to 256. */
ss_status ss_fp4_shape(ss_pattern p, int64_t K, int64_t *K_lift, int64_t *K_lp);

/* Bytes of a tile-major scale buffer for `rows` rows of K_lp lifted elements
 * with `block` (16 or 32) elements per scale; 0 for invalid shapes. */
int64_t ss_fp4_scale_bytes(int64_t rows, int64_t K_lp, int32_t block);

/* NVFP4 weight (offline).  Sparse pattern: prune pairs (keep the 2Nh-2 of
 * every 2Nh pairs of largest x0^2 + x1^2, ties keep the lower pair), slide
 * them into windows of 4 pairs (ascending first fit), store 2 pairs per
 * window, quantise the stored values in blocks of 16 with one global scale
 * for the tensor (amax of the kept weights).  Outputs: Wv [N, K_lp/4] bytes,
 * Wm ss_meta_bytes(N, K_lp/2) bytes, Ws ss_fp4_scale_bytes(N, K_lp, 32),
 * g_w[1].  Dense pattern: Wv [N, K_lp/2], Wm unused, Ws with block 16.
 * A NaN/Inf weight sets SS_ERR_DATA in the device status. */
ss_status ss_compress_weight_nvfp4(const void *W, ss_in_dtype in_dtype, int64_t N, int64_t K,
                                   ss_pattern p, void *Wv, void *Wm, void *Ws, float *g_w,
                                   ss_stream_t stream);

/* NVFP4 activation (M up to 2^30 rows): ONE global scale for the tensor, g_x[0] = amax(X) / 2688
 * (the NVFP4 row: a global scale per tensor; the page calibrates it on a
 * data set, and with none here it is taken from this call's X, so the call
 * first reduces |X| over all M x K elements), the pair lift of pattern p,
 * blocks of `block` lifted elements (32 for the sparse product -- the sparse
 * FP4 instruction scales 32 lifted K at a time, where the page's groups are
 * 16 -- and 16 for the dense one).  Outputs Xv [M, K_lp/2] bytes, Xs
 * ss_fp4_scale_bytes(M, K_lp, block), g_x [1].  g_x also serves as the
 * reduction's accumulator while the call runs (four launches: zero, amax,
 * quantise, g = amax / 2688). */
ss_status ss_quant_lift_act_nvfp4(const void *X, ss_in_dtype in_dtype, int64_t M, int64_t K,
                                  ss_pattern p, int32_t block, void *Xv, void *Xs, float *g_x,
                                  ss_stream_t stream);

/* Sparse NVFP4 GEMM (tcgen05.mma.sp kind::mxf4nvf4, block-scaled; one SM or a
 * CTA pair per MMA): Y[m, n] = ((float)acc[m, n] * g_x[0]) * g_w[0], acc the fp32
 * tensor-core sum of (codes x local scales) products; A = the compressed
 * weight, B = the lifted activation (block 32).  K_lp a positive multiple
 * of 256. */
ss_status ss_sparse_gemm_nvfp4(const void *Wv, const void *Wm, const void *Ws, const float *g_w,
                               const void *Xv, const void *Xs, const float *g_x, int64_t M,
                               int64_t N, int64_t K_lp, void *Y, ss_out_dtype out_dtype,
                               ss_stream_t stream);

/* Dense NVFP4 GEMM of the same construction (kind::mxf4nvf4, blocks of 16
 * on both operands), the comparator.  K_p a positive multiple of 256. */
ss_status ss_dense_gemm_nvfp4(const void *Xv, const void *Xs, const float *g_x, const void *Wv,
                              const void *Ws, const float *g_w, int64_t M, int64_t N,
                              int64_t K_p, void *Y, ss_out_dtype out_dtype, ss_stream_t stream);

/* Returns the first device-side error recorded since the last call
 * (SS_ERR_TIMEOUT, SS_ERR_DATA) or SS_OK, and clears it.  The status word is
 * one per device, shared by every stream: a kernel on `stream` takes it and
 * leaves zero in one atomic exchange after all work queued on `stream`
 * before the call, then the call waits for `stream`.  An error raised by a
 * kernel still running on ANOTHER stream is not lost -- it stays for the
 * next call -- but it is reported only if that kernel finished first, so
 * quiesce every stream that runs this library's kernels before relying on
 * the answer. */
ss_status ss_get_device_status(ss_stream_t stream);

/* Test hooks for the bounded waits (no counterpart in the pages).
 * ss_debug_set_wait_limit: every device-side wait gives up after `ns`
 *   nanoseconds (1 ms .. 60 s; 4 s by default) and records SS_ERR_TIMEOUT.
 * ss_debug_skip_stage: when kb >= 0, the producers of the 8-bit and bf16
 *   GEMM kernels issue no copies for K stage kb of their first output tile,
 *   so the MMA warp's bounded wait for that stage runs out: a wait that
 *   nothing satisfies, with no copy or MMA aimed at it.  The kernel then
 *   unwinds (lets issued copies land, drains issued MMAs, frees tensor
 *   memory) and the next call runs normally.  kb = -1 turns it off.
 * Both synchronise the device and set a device-wide value. */
ss_status ss_debug_set_wait_limit(uint64_t ns);
ss_status ss_debug_skip_stage(int32_t kb);

/* Human-readable name of a status code (static storage). */
const char *ss_status_string(ss_status s);

/* Number of kernels this library has launched in this process. */
int64_t ss_kernel_launches(void);

#ifdef __cplusplus
}
#endif

#endif /* SS_H_ */
