/*
 * ssref.c -- CPU oracle for structured-sparse quantized matmul.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the test suite, the smoke check and the CPU-baseline
 * leg of the benchmark use it.  It shares no code, header, table or helper
 * with the CUDA library; the two meet only through plain byte buffers that
 * the tests compare.
 *
 * Every function here is written to be checked by eye against the pages it
 * follows, not to be fast: plain loops, fp64 where the pages fix no
 * precision, no blocking, no reordering beyond what each definition states.
 * OpenMP is used only across independent output rows.
 *
 * Sources (page title -- section):
 *   [SS]  "SlideSparse: 布局稀疏边界" (66bd.net) -- sliding-window
 *         decomposition paragraph and Fig. 2, activation-lifting paragraph.
 *   [OM]  SlideSparse write-up (omica.com.cn) -- 2.1 pattern table,
 *         2.2 decomposition algorithm, 2.3 completeness theorem,
 *         3.2 vectorised byte packing and output-oriented iteration.
 *   [PD]  "Add 2:4 or drop a precision tier?" (paper-daily 2610.28947) --
 *         2.1 matched bits, 3.1 energy removed by 2:4, 3.3 Blackwell sparse FP4.
 *   [LC]  LLM-Compressor "compression schemes" -- W8A8 rows (channel-wise
 *         weights, dynamic per-token activations) and the 2:4 row.
 *   [OCP] OCP 8-bit floating point specification (E4M3: bias 7, max 448,
 *         no infinities, subnormals kept) -- used for the FP8 encoder.
 *
 * Readings where the pages are silent (each is a convention this oracle
 * fixes and the CUDA path must follow):
 *   R1 prune ties keep the lower index; NaN/Inf weights are rejected.
 *   R2 K is zero-padded to a multiple of the group 2Nh; the lifted K is then
 *      zero-padded to K_lp (a multiple of 128) in both operands.
 *   R3 non-zeros are assigned to windows by ascending first-fit, by mask
 *      (a kept weight that quantises to 0 is still kept).
 *   R4 2:4 packing: per window the assigned local indices ascending, padded
 *      with the lowest unused local indices; nibble = idx0 | idx1 << 2;
 *      two nibbles per byte, low nibble = even window; row-major.
 *   R5 symmetric absmax quantisation, RNE, INT8 clamp to [-127, 127],
 *      scale stored as fp32, inv = Q / a and s = a / Q as IEEE fp32
 *      divisions, zero rows give inv = s = 0.
 *   R6 four lifted bytes of a window sit at ascending addresses (the
 *      packed-word expression in [OM] 3.2 lost its operators; read as
 *      little-endian q0 | q1<<8 | q2<<16 | q3<<24).
 *   R7 epilogue y = ((float)acc * s_x[m]) * s_w[n] in fp32 round-to-nearest,
 *      then bf16 round-to-nearest-even (or fp32 out).
 *   R8 online 2:4 pruning of activations ranks on the input magnitudes and
 *      quantises afterwards with the row absmax.
 *   R9 the bf16 tier ([PD] 2.1 "2:4 + FP16", the 16-bit rows of the
 *      precision-tier tables): values are stored as bf16 (round to nearest
 *      even from the input), no scale; products of bf16 values are exact in
 *      double, summed in k order, rounded once to binary32.
 *   R10 NVFP4 ([LC] NVFP4 row: 4-bit floats, a local scale per group of 16
 *      elements and a global scale per tensor; [PD] 3.3: Blackwell's sparse
 *      FP4 keeps 2 of every 4 adjacent pairs in 8 elements):
 *      - elements are E2M1 (sign, 2 exponent bits with bias 1, 1 mantissa
 *        bit: 0, 0.5, 1, 1.5, 2, 3, 4, 6), round to nearest even, saturating;
 *        code = sign << 3 | magnitude index; two per byte, low nibble first;
 *      - local scales are E4M3 with the sign clear (UE4M3); global scale
 *        g = amax / (6 * 448) in fp32; a block with amax a gets
 *        s = UE4M3(a / (6 g)), divisor d = s * g, inv = 1 / d (0 if d = 0)
 *        and codes E2M1(x * inv), every step one fp32 operation;
 *      - one global scale per tensor, for weights and activations alike
 *        ([LC] NVFP4 row); the page calibrates the activation's global scale
 *        on a data set, and with none here it is taken dynamically from the
 *        amax of the whole activation tensor of the call;
 *      - sparsity is on pairs of adjacent elements: a pattern keep:group
 *        counts pairs (2:4 is the hardware's pairwise 4:8), pairs are ranked
 *        by x0^2 + x1^2 (ties keep the lower pair) and slid as units, and a
 *        window of 4 pairs stores its 2 kept pairs with the nibble
 *        p0 | p1 << 2;
 *      - block size: 16 stored values of a sparse operand (= 32 lifted
 *        elements), 32 lifted elements of the dense operand of a sparse
 *        product, 16 elements in a dense product -- the sparse FP4 tensor-core
 *        instruction applies one scale per 32 lifted K to both operands.  The
 *        page's own definition (16-element groups of the activation, along
 *        its original K) is computed too, by ssref_nvfp4_act_page, so that
 *        the tests can bound what the 32-element blocks cost.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define SSREF_OK 0
#define SSREF_EINVAL 1
#define SSREF_EINTERNAL 2

#define SSREF_INT8 0
#define SSREF_FP8_E4M3 1
#define SSREF_BF16 2
#define SSREF_NVFP4 3

#define SSREF_OUT_F32 0
#define SSREF_OUT_BF16 1

/* ------------------------------------------------------------------ */
/* Shapes: [SS] "8 elements become 12, a 1.5x expansion"; [OM] 2.1.     */
/* A (2Nh-2):2Nh group of 2Nh weights is covered by Nh-1 windows of 4.  */
/* ------------------------------------------------------------------ */
static int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }

/* keep/group = 0/0 means dense (no pattern). */
int ssref_slide_shape(int keep, int group, int64_t K, int64_t *K_pad,
                      int64_t *K_lift, int64_t *K_lp) {
    if (K <= 0) return SSREF_EINVAL;
    if (keep == 0 && group == 0) {
        *K_pad = K;
        *K_lift = K;
        *K_lp = round_up(K, 128);
        return SSREF_OK;
    }
    if (group < 4 || group % 2 != 0 || keep != group - 2) return SSREF_EINVAL;
    int64_t Nh = group / 2;
    int64_t G = (K + group - 1) / group;   /* number of groups */
    *K_pad = G * group;
    *K_lift = G * (Nh - 1) * 4;            /* Nh-1 windows of 4 per group */
    *K_lp = round_up(*K_lift, 128);
    return SSREF_OK;
}

/* [PD] 2.1: dense INTk costs k + 16/128 bits per element (one FP16 scale per
 * 128 elements); 2:4 keeps half the values and adds one index bit per
 * original element. */
double ssref_bits_per_element(int value_bits, int sparse_2to4) {
    double scale_bits = 16.0 / 128.0;
    if (sparse_2to4) return value_bits / 2.0 + 1.0 + scale_bits;
    return value_bits + scale_bits;
}

/* ------------------------------------------------------------------ */
/* Number formats                                                      */
/* ------------------------------------------------------------------ */

/* [OCP] E4M3: sign, 4 exponent bits (bias 7), 3 mantissa bits; normal
 * values (1 + m/8) * 2^(e-7) for e in 1..15 except e=15,m=7 (NaN);
 * subnormals (m/8) * 2^-6; no infinities.  Round to nearest even and
 * saturate to +-448 (the "satfinite" conversion). */
uint8_t ssref_e4m3_from_float(float v) {
    if (isnan(v)) return 0x7F;
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs((double)v);
    if (a >= 448.0) return sign | 0x7E;           /* saturate */
    if (a == 0.0) return sign;
    double quantum;
    if (a < ldexp(1.0, -6)) {
        quantum = ldexp(1.0, -9);                 /* subnormal spacing */
    } else {
        int e;
        frexp(a, &e);                             /* a = f * 2^e, f in [0.5,1) */
        quantum = ldexp(1.0, (e - 1) - 3);        /* 3 mantissa bits */
    }
    double r = nearbyint(a / quantum) * quantum;  /* RNE (default mode) */
    if (r >= 448.0) return sign | 0x7E;
    if (r == 0.0) return sign;
    if (r < ldexp(1.0, -6)) {
        int m = (int)(r / ldexp(1.0, -9));        /* 1..7 */
        return sign | (uint8_t)m;
    }
    int e;
    double f = frexp(r, &e);                      /* r = f * 2^e */
    int E = (e - 1) + 7;                          /* biased exponent */
    int m = (int)((f * 2.0 - 1.0) * 8.0);         /* exact */
    return sign | (uint8_t)(E << 3) | (uint8_t)m;
}

double ssref_e4m3_to_double(uint8_t b) {
    int s = b >> 7, E = (b >> 3) & 0xF, m = b & 7;
    double v;
    if (E == 15 && m == 7) return NAN;
    if (E == 0) v = ldexp((double)m / 8.0, -6);
    else v = ldexp(1.0 + (double)m / 8.0, E - 7);
    return s ? -v : v;
}

/* IEEE-754 binary32 -> bfloat16, round to nearest even (bfloat16 keeps the
 * top 16 bits of binary32). */
uint16_t ssref_bf16_from_float(float v) {
    uint32_t u;
    memcpy(&u, &v, 4);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)((u >> 16) | 0x40);
    uint32_t lower = u & 0xFFFFu;
    uint32_t upper = u >> 16;
    if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper += 1;
    return (uint16_t)upper;
}

/* ------------------------------------------------------------------ */
/* Quantisation ([LC] W8A8: channel-wise weights, dynamic per-token     */
/* activations, symmetric).  Readings R5.                              */
/* ------------------------------------------------------------------ */
static float q_max(int qdtype) { return qdtype == SSREF_INT8 ? 127.0f : 448.0f; }

static void scale_from_absmax(float a, int qdtype, float *inv, float *s) {
    volatile float Q = q_max(qdtype);
    if (a == 0.0f) { *inv = 0.0f; *s = 0.0f; return; }
    volatile float num = Q;
    *inv = num / a;   /* IEEE binary32 division */
    *s = a / Q;
}

static uint8_t quantize_one(float x, float inv, int qdtype) {
    volatile float p = x * inv;   /* binary32 multiply, rounded to nearest */
    if (qdtype == SSREF_INT8) {
        float r = rintf(p);        /* ties to even in the default mode */
        if (r > 127.0f) r = 127.0f;
        if (r < -127.0f) r = -127.0f;
        return (uint8_t)(int8_t)r;
    }
    return ssref_e4m3_from_float(p);
}

int ssref_quantize_value(float x, float inv, int qdtype, uint8_t *out) {
    *out = quantize_one(x, inv, qdtype);
    return SSREF_OK;
}

int ssref_scale_from_absmax(float a, int qdtype, float *inv, float *s) {
    scale_from_absmax(a, qdtype, inv, s);
    return SSREF_OK;
}

static double dequant_one(uint8_t q, int qdtype) {
    if (qdtype == SSREF_INT8) return (double)(int8_t)q;
    return ssref_e4m3_to_double(q);
}

/* ------------------------------------------------------------------ */
/* Magnitude pruning ([OM] 4.1 "magnitude pruning"; [PD] 2.3).          */
/* In each group of `group` consecutive elements along K keep the      */
/* `keep` largest |w|; rank = number of elements that come before it in */
/* the order (|w| descending, index ascending) -- reading R1.          */
/* ------------------------------------------------------------------ */
static void prune_group(const float *v, int group, int keep, uint8_t *kept) {
    for (int i = 0; i < group; i++) {
        int rank = 0;
        for (int j = 0; j < group; j++) {
            if (j == i) continue;
            float aj = fabsf(v[j]), ai = fabsf(v[i]);
            if (aj > ai || (aj == ai && j < i)) rank++;
        }
        kept[i] = rank < keep ? 1 : 0;
    }
}

/* mask[r*K_pad + k] = 1 where W[r,k] is kept; positions k >= K are the
 * zero padding of reading R2 and take part in the ranking as zeros. */
int ssref_prune_mask(const float *W, int64_t rows, int64_t K, int keep, int group,
                     uint8_t *mask) {
    if (group <= 0 || keep <= 0 || keep > group) return SSREF_EINVAL;
    int64_t K_pad = round_up(K, group);
    for (int64_t r = 0; r < rows; r++)
        for (int64_t k = 0; k < K; k++)
            if (!isfinite(W[r * K + k])) return SSREF_EINVAL;
    float *v = (float *)malloc(sizeof(float) * group);
    for (int64_t r = 0; r < rows; r++) {
        for (int64_t g = 0; g < K_pad / group; g++) {
            for (int i = 0; i < group; i++) {
                int64_t k = g * group + i;
                v[i] = k < K ? W[r * K + k] : 0.0f;
            }
            prune_group(v, group, keep, &mask[r * K_pad + g * group]);
        }
    }
    free(v);
    return SSREF_OK;
}

/* Blackwell sparse FP4 ([PD] 3.3): in each group of 8, keep 2 of the 4
 * adjacent pairs -- the two with the largest pair energy (sum of squares);
 * ties keep the lower pair index. */
int ssref_prune_pairwise_4of8(const float *W, int64_t rows, int64_t K, uint8_t *mask) {
    if (K % 8 != 0) return SSREF_EINVAL;
    for (int64_t r = 0; r < rows; r++) {
        for (int64_t g = 0; g < K / 8; g++) {
            const float *v = &W[r * K + g * 8];
            double e[4];
            for (int p = 0; p < 4; p++)
                e[p] = (double)v[2 * p] * v[2 * p] + (double)v[2 * p + 1] * v[2 * p + 1];
            for (int p = 0; p < 4; p++) {
                int rank = 0;
                for (int q = 0; q < 4; q++) {
                    if (q == p) continue;
                    if (e[q] > e[p] || (e[q] == e[p] && q < p)) rank++;
                }
                uint8_t k = rank < 2 ? 1 : 0;
                mask[r * K + g * 8 + 2 * p] = k;
                mask[r * K + g * 8 + 2 * p + 1] = k;
            }
        }
    }
    return SSREF_OK;
}

/* ------------------------------------------------------------------ */
/* Sliding-window decomposition ([SS] Fig. 2 and the paragraph before   */
/* it: Nh-1 windows of width 4, stride 2; window j of a group covers    */
/* local positions 2j..2j+3; an overflowing non-zero lies in the overlap */
/* with the next window and goes there).  Reading R3: ascending          */
/* first-fit.  win[r*K_pad+k] receives the window index j (0..Nh-2) of   */
/* each kept position and -1 elsewhere.                                 */
/* Returns SSREF_EINTERNAL if some kept position found no window (the   */
/* completeness theorem of [OM] 2.3 says that never happens for at most */
/* 2Nh-2 kept positions per group).                                     */
/* ------------------------------------------------------------------ */
int ssref_assign_windows(const uint8_t *mask, int64_t rows, int64_t K_pad, int group,
                         int8_t *win) {
    if (group < 4 || group % 2 != 0 || K_pad % group != 0) return SSREF_EINVAL;
    int Nh = group / 2;
    int status = SSREF_OK;
    for (int64_t r = 0; r < rows; r++) {
        for (int64_t g = 0; g < K_pad / group; g++) {
            const uint8_t *m = &mask[r * K_pad + g * group];
            int8_t *w = &win[r * K_pad + g * group];
            for (int i = 0; i < group; i++) w[i] = -1;
            for (int j = 0; j < Nh - 1; j++) {
                int taken = 0;
                for (int t = 0; t < 4 && taken < 2; t++) {
                    int pos = 2 * j + t;
                    if (m[pos] && w[pos] < 0) { w[pos] = (int8_t)j; taken++; }
                }
            }
            for (int i = 0; i < group; i++)
                if (m[i] && w[i] < 0) status = SSREF_EINTERNAL;
        }
    }
    return status;
}

/* ------------------------------------------------------------------ */
/* 2:4 packing of one window, reading R4.  `assigned[t]` marks the local */
/* positions t = 0..3 the window owns; q[t] their quantised bytes.      */
/* ------------------------------------------------------------------ */
static uint8_t window_slots(const uint8_t assigned[4], int idx[2]) {
    int n = 0;
    for (int t = 0; t < 4 && n < 2; t++)
        if (assigned[t]) idx[n++] = t;
    for (int t = 0; t < 4 && n < 2; t++) {       /* pad with lowest unused */
        int used = 0;
        for (int s = 0; s < n; s++) if (idx[s] == t) used = 1;
        if (!assigned[t] && !used) idx[n++] = t;
    }
    if (idx[0] > idx[1]) { int tmp = idx[0]; idx[0] = idx[1]; idx[1] = tmp; }
    return (uint8_t)(idx[0] | (idx[1] << 2));
}

static uint8_t pack_window(const uint8_t assigned[4], const uint8_t q[4], uint8_t val[2]) {
    int idx[2];
    uint8_t nib = window_slots(assigned, idx);
    for (int s = 0; s < 2; s++) val[s] = assigned[idx[s]] ? q[idx[s]] : 0;
    return nib;
}

/* The same packing for 16-bit values (the bf16 tier). */
static uint8_t pack_window16(const uint8_t assigned[4], const uint16_t q[4], uint16_t val[2]) {
    int idx[2];
    uint8_t nib = window_slots(assigned, idx);
    for (int s = 0; s < 2; s++) val[s] = assigned[idx[s]] ? q[idx[s]] : 0;
    return nib;
}

static void put_nibble(uint8_t *row_meta, int64_t w, uint8_t nib) {
    if (w % 2 == 0) row_meta[w / 2] = (uint8_t)((row_meta[w / 2] & 0xF0) | nib);
    else row_meta[w / 2] = (uint8_t)((row_meta[w / 2] & 0x0F) | (nib << 4));
}

static uint8_t get_nibble(const uint8_t *row_meta, int64_t w) {
    return w % 2 == 0 ? (row_meta[w / 2] & 0x0F) : (row_meta[w / 2] >> 4);
}

/* ------------------------------------------------------------------ */
/* Offline weight compression: prune -> per-channel quantise -> slide   */
/* decomposition -> 2:4 pack ([OM] 2.2 weight preprocessing, 3.1; [LC]  */
/* channel-wise weights).  Outputs:                                     */
/*   Wv [N, K_lp/2]  stored values, two per window                      */
/*   Wm [N, K_lp/8]  metadata nibbles (reading R4)                      */
/*   s_w[N]          per-channel scale                                  */
/* Dense (keep = group = 0): Wv = [N, K_lp] quantised W, Wm untouched.  */
/* ------------------------------------------------------------------ */
int ssref_compress_weight(const float *W, int64_t N, int64_t K, int keep, int group,
                          int qdtype, uint8_t *Wv, uint8_t *Wm, float *s_w) {
    int64_t K_pad, K_lift, K_lp;
    int st = ssref_slide_shape(keep, group, K, &K_pad, &K_lift, &K_lp);
    if (st) return st;
    for (int64_t i = 0; i < N * K; i++)
        if (!isfinite(W[i])) return SSREF_EINVAL;
    if (group == 0) {
        for (int64_t n = 0; n < N; n++) {
            float a = 0.0f, inv, s;
            for (int64_t k = 0; k < K; k++) a = fmaxf(a, fabsf(W[n * K + k]));
            scale_from_absmax(a, qdtype, &inv, &s);
            s_w[n] = s;
            for (int64_t k = 0; k < K_lp; k++)
                Wv[n * K_lp + k] = k < K ? quantize_one(W[n * K + k], inv, qdtype) : 0;
        }
        return SSREF_OK;
    }
    int Nh = group / 2;
    uint8_t *mask = (uint8_t *)malloc((size_t)(N * K_pad));
    int8_t *win = (int8_t *)malloc((size_t)(N * K_pad));
    st = ssref_prune_mask(W, N, K, keep, group, mask);
    if (!st) st = ssref_assign_windows(mask, N, K_pad, group, win);
    if (st) { free(mask); free(win); return st; }
    for (int64_t n = 0; n < N; n++) {
        /* absmax over the kept weights of this channel */
        float a = 0.0f, inv, s;
        for (int64_t k = 0; k < K; k++)
            if (mask[n * K_pad + k]) a = fmaxf(a, fabsf(W[n * K + k]));
        scale_from_absmax(a, qdtype, &inv, &s);
        s_w[n] = s;
        uint8_t *vrow = &Wv[n * (K_lp / 2)];
        uint8_t *mrow = &Wm[n * (K_lp / 8)];
        for (int64_t w = 0; w < K_lp / 4; w++) {
            uint8_t assigned[4] = {0, 0, 0, 0}, q[4] = {0, 0, 0, 0}, val[2];
            if (w < K_lift / 4) {
                int64_t g = w / (Nh - 1);
                int j = (int)(w % (Nh - 1));
                for (int t = 0; t < 4; t++) {
                    int64_t k = g * group + 2 * j + t;
                    if (win[n * K_pad + k] == j) {
                        assigned[t] = 1;
                        q[t] = quantize_one(k < K ? W[n * K + k] : 0.0f, inv, qdtype);
                    }
                }
            }
            uint8_t nib = pack_window(assigned, q, val);
            vrow[2 * w] = val[0];
            vrow[2 * w + 1] = val[1];
            put_nibble(mrow, w, nib);
        }
    }
    free(mask);
    free(win);
    return SSREF_OK;
}

/* ------------------------------------------------------------------ */
/* Activation quantisation with lifting ([SS] activation lifting is an  */
/* index map fused into the per-token quant kernel; [OM] 3.2: window    */
/* index -> group = idx / (Nh-1), offset = idx % (Nh-1),                 */
/* base = 2*Nh*group + 2*offset, load 4 consecutive activations).        */
/*   Xq[M, K_lp]   lifted quantised activations (R6 byte order)          */
/*   s_x[M]        per-token scale; the absmax runs over the original K  */
/* Dense (keep = group = 0): identity map onto K_lp.                     */
/* ------------------------------------------------------------------ */
int ssref_quant_lift_act(const float *X, int64_t M, int64_t K, int keep, int group,
                         int qdtype, uint8_t *Xq, float *s_x) {
    int64_t K_pad, K_lift, K_lp;
    int st = ssref_slide_shape(keep, group, K, &K_pad, &K_lift, &K_lp);
    if (st) return st;
    int Nh = group / 2;
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; m++) {
        const float *x = &X[m * K];
        float a = 0.0f, inv, s;
        for (int64_t k = 0; k < K; k++) a = fmaxf(a, fabsf(x[k]));
        scale_from_absmax(a, qdtype, &inv, &s);
        s_x[m] = s;
        uint8_t *out = &Xq[m * K_lp];
        if (group == 0) {
            for (int64_t k = 0; k < K_lp; k++)
                out[k] = k < K ? quantize_one(x[k], inv, qdtype) : 0;
            continue;
        }
        for (int64_t w = 0; w < K_lp / 4; w++) {
            for (int t = 0; t < 4; t++) {
                uint8_t q = 0;
                if (w < K_lift / 4) {
                    int64_t g = w / (Nh - 1), j = w % (Nh - 1);
                    int64_t base = 2 * Nh * g + 2 * j;
                    int64_t k = base + t;
                    q = k < K ? quantize_one(x[k], inv, qdtype) : 0;
                }
                out[4 * w + t] = q;
            }
        }
    }
    return SSREF_OK;
}

/* ------------------------------------------------------------------ */
/* Online 2:4 prune + compress of an activation ([PD] 1 and 2.3: an      */
/* operand produced on the fly must be pruned and compressed before      */
/* every matmul and that time counts).  Reading R8: rank on |x| (ties    */
/* keep the lower index), then quantise the kept values with the row     */
/* absmax.  K is zero-padded to K_lp = round_up(round_up(K,4),128).      */
/*   Xv[M, K_lp/2], Xm[M, K_lp/8], s_x[M]                                 */
/* ------------------------------------------------------------------ */
int ssref_prune_act_2to4(const float *X, int64_t M, int64_t K, int qdtype, uint8_t *Xv,
                         uint8_t *Xm, float *s_x) {
    if (K <= 0) return SSREF_EINVAL;
    int64_t K_lp = round_up(round_up(K, 4), 128);
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; m++) {
        const float *x = &X[m * K];
        float a = 0.0f, inv, s;
        for (int64_t k = 0; k < K; k++) a = fmaxf(a, fabsf(x[k]));
        scale_from_absmax(a, qdtype, &inv, &s);
        s_x[m] = s;
        for (int64_t w = 0; w < K_lp / 4; w++) {
            float v[4];
            uint8_t kept[4], q[4], val[2];
            for (int t = 0; t < 4; t++) {
                int64_t k = 4 * w + t;
                v[t] = k < K ? x[k] : 0.0f;
            }
            prune_group(v, 4, 2, kept);
            for (int t = 0; t < 4; t++) q[t] = kept[t] ? quantize_one(v[t], inv, qdtype) : 0;
            uint8_t nib = pack_window(kept, q, val);
            Xv[m * (K_lp / 2) + 2 * w] = val[0];
            Xv[m * (K_lp / 2) + 2 * w + 1] = val[1];
            put_nibble(&Xm[m * (K_lp / 8)], w, nib);
        }
    }
    return SSREF_OK;
}

/* Expand a 2:4 operand (values + nibbles) to its dense logical rows. */
int ssref_decompress_2to4(const uint8_t *Av, const uint8_t *Am, int64_t rows, int64_t K_lp,
                          uint8_t *A) {
    if (K_lp % 8 != 0) return SSREF_EINVAL;
    for (int64_t r = 0; r < rows; r++) {
        for (int64_t w = 0; w < K_lp / 4; w++) {
            uint8_t nib = get_nibble(&Am[r * (K_lp / 8)], w);
            int i0 = nib & 3, i1 = (nib >> 2) & 3;
            if (i0 >= i1) return SSREF_EINVAL;
            for (int t = 0; t < 4; t++) A[r * K_lp + 4 * w + t] = 0;
            A[r * K_lp + 4 * w + i0] = Av[r * (K_lp / 2) + 2 * w];
            A[r * K_lp + 4 * w + i1] = Av[r * (K_lp / 2) + 2 * w + 1];
        }
    }
    return SSREF_OK;
}

/* ------------------------------------------------------------------ */
/* The bf16 tier (reading R9): the same pruning, windows and packing,    */
/* with 16-bit stored values and no quantisation.                        */
/* ------------------------------------------------------------------ */
static double bf16_to_double(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Wv [N, K_lp/2] bf16 (dense: [N, K_lp]), Wm [N, K_lp/8] nibbles. */
int ssref_compress_weight_bf16(const float *W, int64_t N, int64_t K, int keep, int group,
                               uint16_t *Wv, uint8_t *Wm) {
    int64_t K_pad, K_lift, K_lp;
    int st = ssref_slide_shape(keep, group, K, &K_pad, &K_lift, &K_lp);
    if (st) return st;
    for (int64_t i = 0; i < N * K; i++)
        if (!isfinite(W[i])) return SSREF_EINVAL;
    if (group == 0) {
        for (int64_t n = 0; n < N; n++)
            for (int64_t k = 0; k < K_lp; k++)
                Wv[n * K_lp + k] = k < K ? ssref_bf16_from_float(W[n * K + k]) : 0;
        return SSREF_OK;
    }
    int Nh = group / 2;
    uint8_t *mask = (uint8_t *)malloc((size_t)(N * K_pad));
    int8_t *win = (int8_t *)malloc((size_t)(N * K_pad));
    st = ssref_prune_mask(W, N, K, keep, group, mask);
    if (!st) st = ssref_assign_windows(mask, N, K_pad, group, win);
    if (st) { free(mask); free(win); return st; }
    for (int64_t n = 0; n < N; n++) {
        uint16_t *vrow = &Wv[n * (K_lp / 2)];
        uint8_t *mrow = &Wm[n * (K_lp / 8)];
        for (int64_t w = 0; w < K_lp / 4; w++) {
            uint8_t assigned[4] = {0, 0, 0, 0};
            uint16_t q[4] = {0, 0, 0, 0}, val[2];
            if (w < K_lift / 4) {
                int64_t g = w / (Nh - 1);
                int j = (int)(w % (Nh - 1));
                for (int t = 0; t < 4; t++) {
                    int64_t k = g * group + 2 * j + t;
                    if (win[n * K_pad + k] == j) {
                        assigned[t] = 1;
                        q[t] = ssref_bf16_from_float(k < K ? W[n * K + k] : 0.0f);
                    }
                }
            }
            uint8_t nib = pack_window16(assigned, q, val);
            vrow[2 * w] = val[0];
            vrow[2 * w + 1] = val[1];
            put_nibble(mrow, w, nib);
        }
    }
    free(mask);
    free(win);
    return SSREF_OK;
}

/* Xl [M, K_lp] bf16: the lifted activation ([OM] 3.2 window map), no scale. */
int ssref_lift_act_bf16(const float *X, int64_t M, int64_t K, int keep, int group, uint16_t *Xl) {
    int64_t K_pad, K_lift, K_lp;
    int st = ssref_slide_shape(keep, group, K, &K_pad, &K_lift, &K_lp);
    if (st) return st;
    int Nh = group / 2;
    for (int64_t m = 0; m < M; m++) {
        const float *x = &X[m * K];
        uint16_t *out = &Xl[m * K_lp];
        if (group == 0) {
            for (int64_t k = 0; k < K_lp; k++) out[k] = k < K ? ssref_bf16_from_float(x[k]) : 0;
            continue;
        }
        for (int64_t w = 0; w < K_lp / 4; w++)
            for (int t = 0; t < 4; t++) {
                uint16_t q = 0;
                if (w < K_lift / 4) {
                    int64_t g = w / (Nh - 1), j = w % (Nh - 1);
                    int64_t k = 2 * Nh * g + 2 * j + t;
                    q = k < K ? ssref_bf16_from_float(x[k]) : 0;
                }
                out[4 * w + t] = q;
            }
    }
    return SSREF_OK;
}

int ssref_decompress_2to4_bf16(const uint16_t *Av, const uint8_t *Am, int64_t rows, int64_t K_lp,
                               uint16_t *A) {
    if (K_lp % 8 != 0) return SSREF_EINVAL;
    for (int64_t r = 0; r < rows; r++) {
        for (int64_t w = 0; w < K_lp / 4; w++) {
            uint8_t nib = get_nibble(&Am[r * (K_lp / 8)], w);
            int i0 = nib & 3, i1 = (nib >> 2) & 3;
            if (i0 >= i1) return SSREF_EINVAL;
            for (int t = 0; t < 4; t++) A[r * K_lp + 4 * w + t] = 0;
            A[r * K_lp + 4 * w + i0] = Av[r * (K_lp / 2) + 2 * w];
            A[r * K_lp + 4 * w + i1] = Av[r * (K_lp / 2) + 2 * w + 1];
        }
    }
    return SSREF_OK;
}

/* Y[r, n] = round_binary32(sum_k X[m_r, k] * W[n, k]) (double sum in k
 * order), then bf16 RNE or fp32 out. */
int ssref_matmul_bf16(const uint16_t *X, const uint16_t *W, int64_t M, int64_t N, int64_t K,
                      const int64_t *m_idx, int64_t n_rows, int out_dtype, void *Y) {
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t r = 0; r < n_rows; r++) {
        int64_t m = m_idx ? m_idx[r] : r;
        if (m < 0 || m >= M) continue;
        for (int64_t n = 0; n < N; n++) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; k++)
                acc += bf16_to_double(X[m * K + k]) * bf16_to_double(W[n * K + k]);
            volatile float y = (float)acc;
            if (out_dtype == SSREF_OUT_F32) ((float *)Y)[r * N + n] = y;
            else ((uint16_t *)Y)[r * N + n] = ssref_bf16_from_float(y);
        }
    }
    return SSREF_OK;
}

/* Sparse GEMM of the bf16 tier through decompression (sparse_operand as in
 * ssref_sparse_gemm). */
int ssref_sparse_gemm_bf16(int sparse_operand, const uint16_t *Av, const uint8_t *Am,
                           const uint16_t *B, int64_t M, int64_t N, int64_t K_lp,
                           const int64_t *m_idx, int64_t n_rows, int out_dtype, void *Y) {
    int64_t rowsA = sparse_operand == 0 ? N : M;
    uint16_t *A = (uint16_t *)malloc((size_t)(rowsA * K_lp) * sizeof(uint16_t));
    int st = ssref_decompress_2to4_bf16(Av, Am, rowsA, K_lp, A);
    if (!st) {
        if (sparse_operand == 0)
            st = ssref_matmul_bf16(B, A, M, N, K_lp, m_idx, n_rows, out_dtype, Y);
        else
            st = ssref_matmul_bf16(A, B, M, N, K_lp, m_idx, n_rows, out_dtype, Y);
    }
    free(A);
    return st;
}

/* ------------------------------------------------------------------ */
/* Matmul and epilogue.  acc[m,n] = sum_k X[m,k] * W[n,k].               */
/* INT8: exact integer sum (int64, then checked to fit int32).           */
/* E4M3: every product is exact in double; summed in double in k order,  */
/* then rounded once to binary32.                                        */
/* Epilogue R7.  m_idx selects output rows (NULL: all M rows).           */
/* ------------------------------------------------------------------ */
static void epilogue_store(double accd, int64_t acc_i, int qdtype, float sx, float sw,
                           int out_dtype, void *Y, int64_t off) {
    volatile float acc = qdtype == SSREF_INT8 ? (float)acc_i : (float)accd;
    volatile float t = acc * sx;
    volatile float y = t * sw;
    if (out_dtype == SSREF_OUT_F32) ((float *)Y)[off] = y;
    else ((uint16_t *)Y)[off] = ssref_bf16_from_float(y);
}

int ssref_matmul_q(int qdtype, const uint8_t *X, const float *s_x, const uint8_t *W,
                   const float *s_w, int64_t M, int64_t N, int64_t K,
                   const int64_t *m_idx, int64_t n_rows, int out_dtype, void *Y) {
    int64_t R = m_idx ? n_rows : M;
    int bad = 0;
    double lut[256];                        /* value of every 8-bit code */
    for (int b = 0; b < 256; b++) lut[b] = dequant_one((uint8_t)b, qdtype);
    #pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t r = 0; r < R; r++) {
        int64_t m = m_idx ? m_idx[r] : r;
        if (m < 0 || m >= M) { bad = 1; continue; }
        for (int64_t n = 0; n < N; n++) {
            int64_t acc_i = 0;
            double acc_d = 0.0;
            for (int64_t k = 0; k < K; k++) {
                if (qdtype == SSREF_INT8)
                    acc_i += (int64_t)(int8_t)X[m * K + k] * (int64_t)(int8_t)W[n * K + k];
                else
                    acc_d += lut[X[m * K + k]] * lut[W[n * K + k]];
            }
            if (acc_i > INT32_MAX || acc_i < INT32_MIN) bad = 1;
            epilogue_store(acc_d, acc_i, qdtype, s_x[m], s_w[n], out_dtype, Y, r * N + n);
        }
    }
    return bad ? SSREF_EINVAL : SSREF_OK;
}

/* Raw accumulators (no epilogue), for the integer identities. */
int ssref_matmul_acc(int qdtype, const uint8_t *X, const uint8_t *W, int64_t M, int64_t N,
                     int64_t K, int64_t *acc_i, double *acc_d) {
    #pragma omp parallel for schedule(static)
    for (int64_t m = 0; m < M; m++)
        for (int64_t n = 0; n < N; n++) {
            int64_t ai = 0;
            double ad = 0.0;
            for (int64_t k = 0; k < K; k++) {
                if (qdtype == SSREF_INT8)
                    ai += (int64_t)(int8_t)X[m * K + k] * (int64_t)(int8_t)W[n * K + k];
                else
                    ad += dequant_one(X[m * K + k], qdtype) * dequant_one(W[n * K + k], qdtype);
            }
            if (acc_i) acc_i[m * N + n] = ai;
            if (acc_d) acc_d[m * N + n] = ad;
        }
    return SSREF_OK;
}

/* Sparse GEMM over the packed 2:4 operand, mirroring the library call.
 * sparse_operand 0: A = W rows (N of them), B = lifted X [M, K_lp];
 * sparse_operand 1: A = X rows (M of them), B = dense W [N, K_lp].
 * Y[M, N] in both cases; scales s_a belong to A's rows, s_b to B's rows. */
int ssref_sparse_gemm(int sparse_operand, const uint8_t *Av, const uint8_t *Am,
                      const float *s_a, const uint8_t *B, const float *s_b, int64_t M,
                      int64_t N, int64_t K_lp, int qdtype, const int64_t *m_idx,
                      int64_t n_rows, int out_dtype, void *Y) {
    int64_t rowsA = sparse_operand == 0 ? N : M;
    uint8_t *A = (uint8_t *)malloc((size_t)(rowsA * K_lp));
    int st = ssref_decompress_2to4(Av, Am, rowsA, K_lp, A);
    if (!st) {
        if (sparse_operand == 0)
            st = ssref_matmul_q(qdtype, B, s_b, A, s_a, M, N, K_lp, m_idx, n_rows, out_dtype, Y);
        else
            st = ssref_matmul_q(qdtype, A, s_a, B, s_b, M, N, K_lp, m_idx, n_rows, out_dtype, Y);
    }
    free(A);
    return st;
}


/* ------------------------------------------------------------------ */
/* NVFP4 (reading R10).                                                  */
/* ------------------------------------------------------------------ */
static const double E2M1_MAG[8] = {0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};

/* Nearest E2M1 value, ties to the even code (the one with mantissa bit 0),
 * |v| above 6 saturating to 6; the sign is kept, so a negative value that
 * rounds to zero gives -0 (IEEE rounding keeps the sign of a zero result). */
uint8_t ssref_e2m1_from_float(float v) {
    double a = fabs((double)v);
    int best = 0;
    for (int i = 1; i < 8; i++) {
        double di = fabs(a - E2M1_MAG[i]), db = fabs(a - E2M1_MAG[best]);
        if (di < db || (di == db && (i & 1) == 0)) best = i;
    }
    if (a > 6.0) best = 7;
    uint8_t sign = signbit(v) ? 8 : 0;
    return (uint8_t)(sign | best);
}

double ssref_e2m1_to_double(uint8_t c) {
    double m = E2M1_MAG[c & 7];
    return (c & 8) ? -m : m;
}

float ssref_nvfp4_global(float amax) {
    volatile float g = amax / 2688.0f;   /* 6 * 448 */
    return g;
}

/* One block of n values with global scale g: codes[i] and the UE4M3 scale. */
static void nvfp4_block(const float *x, int n, float g, uint8_t *codes, uint8_t *sc) {
    float a = 0.0f;
    for (int i = 0; i < n; i++) a = fmaxf(a, fabsf(x[i]));
    *sc = 0;
    for (int i = 0; i < n; i++) codes[i] = 0;
    if (g == 0.0f) return;
    volatile float den = 6.0f * g;
    volatile float t = a / den;
    *sc = ssref_e4m3_from_float(t);
    volatile float d = (float)ssref_e4m3_to_double(*sc) * g;
    if (d == 0.0f) return;
    volatile float inv = 1.0f / d;
    for (int i = 0; i < n; i++) {
        volatile float y = x[i] * inv;
        codes[i] = ssref_e2m1_from_float(y);
    }
}

static void put_fp4(uint8_t *row, int64_t i, uint8_t c) {
    if (i & 1) row[i / 2] = (uint8_t)((row[i / 2] & 0x0F) | (c << 4));
    else row[i / 2] = (uint8_t)((row[i / 2] & 0xF0) | (c & 0x0F));
}

static uint8_t get_fp4(const uint8_t *row, int64_t i) {
    return (uint8_t)((row[i / 2] >> (4 * (i & 1))) & 0x0F);
}

/* Shapes on pairs: K_pairs = ceil(K / 2) is slid like K for elements; the
 * lifted length in elements is 2 * K_lift_pairs, padded to K_lp (a multiple
 * of 256: one metadata block of the GEMM).  Dense: K_lp = K rounded to 256. */
int ssref_fp4_shape(int keep, int group, int64_t K, int64_t *K_lift, int64_t *K_lp) {
    if (K <= 0) return SSREF_EINVAL;
    if (group == 0) {
        *K_lift = K;
        *K_lp = round_up(K, 256);
        return SSREF_OK;
    }
    int64_t Kp_pad, Kp_lift, Kp_lp;
    int st = ssref_slide_shape(keep, group, (K + 1) / 2, &Kp_pad, &Kp_lift, &Kp_lp);
    if (st) return st;
    *K_lift = 2 * Kp_lift;
    *K_lp = 2 * Kp_lp;
    return SSREF_OK;
}

/* Pair mask: per group of `group` pairs keep the `keep` pairs of largest
 * x0^2 + x1^2 (double), ties keep the lower pair.  mask[r * P_pad + p]. */
int ssref_prune_pairs(const float *W, int64_t rows, int64_t K, int keep, int group,
                      uint8_t *mask) {
    int64_t P = (K + 1) / 2, P_pad = round_up(P, group);
    for (int64_t r = 0; r < rows; r++)
        for (int64_t g = 0; g < P_pad / group; g++)
            for (int p = 0; p < group; p++) {
                double e[32];
                for (int q = 0; q < group; q++) {
                    int64_t k0 = 2 * (g * group + q);
                    double x0 = k0 < K ? W[r * K + k0] : 0.0;
                    double x1 = k0 + 1 < K ? W[r * K + k0 + 1] : 0.0;
                    e[q] = x0 * x0 + x1 * x1;
                }
                int rank = 0;
                for (int q = 0; q < group; q++)
                    if (q != p && (e[q] > e[p] || (e[q] == e[p] && q < p))) rank++;
                mask[r * P_pad + g * group + p] = rank < keep ? 1 : 0;
            }
    return SSREF_OK;
}

/* Sparse NVFP4 weight: prune pairs, slide them into windows of 4 pairs (the
 * first-fit of R3 on pairs), store each window's 2 kept pairs (4 values) and
 * a nibble, then quantise the stored values in blocks of 16 with one
 * global scale for the tensor.
 *   Wv [N, K_lp/4] bytes (K_lp/2 stored codes), Wm [N, K_lp/16] bytes
 *   (nibble per window of 8 lifted elements, low nibble first), Ws [N,
 *   K_lp/32] UE4M3, *g_w. */
int ssref_compress_weight_nvfp4(const float *W, int64_t N, int64_t K, int keep, int group,
                                uint8_t *Wv, uint8_t *Wm, uint8_t *Ws, float *g_w) {
    int64_t K_lift, K_lp;
    int st = ssref_fp4_shape(keep, group, K, &K_lift, &K_lp);
    if (st || group == 0) return SSREF_EINVAL;
    for (int64_t i = 0; i < N * K; i++)
        if (!isfinite(W[i])) return SSREF_EINVAL;
    int Nh = group / 2;
    int64_t P = (K + 1) / 2, P_pad = round_up(P, group);
    uint8_t *mask = (uint8_t *)malloc((size_t)(N * P_pad));
    int8_t *win = (int8_t *)malloc((size_t)(N * P_pad));
    float *stored = (float *)malloc((size_t)(K_lp / 2) * sizeof(float));
    ssref_prune_pairs(W, N, K, keep, group, mask);
    st = ssref_assign_windows(mask, N, P_pad, group, win);
    if (st) { free(mask); free(win); free(stored); return st; }
    /* global amax over the kept weights */
    float amax = 0.0f;
    for (int64_t r = 0; r < N; r++)
        for (int64_t p = 0; p < P; p++)
            if (mask[r * P_pad + p])
                for (int h = 0; h < 2; h++)
                    if (2 * p + h < K) amax = fmaxf(amax, fabsf(W[r * K + 2 * p + h]));
    float g = ssref_nvfp4_global(amax);
    *g_w = g;
    memset(Wv, 0, (size_t)(N * K_lp / 4));
    memset(Wm, 0, (size_t)(N * K_lp / 16));
    for (int64_t r = 0; r < N; r++) {
        for (int64_t i = 0; i < K_lp / 2; i++) stored[i] = 0.0f;
        for (int64_t w = 0; w < K_lp / 8; w++) {       /* windows of 4 pairs */
            uint8_t assigned[4] = {0, 0, 0, 0};
            int64_t pbase = 0;
            if (w < K_lift / 8) {
                int64_t gi = w / (Nh - 1);
                int j = (int)(w % (Nh - 1));
                pbase = gi * group + 2 * j;
                for (int t = 0; t < 4; t++)
                    if (win[r * P_pad + pbase + t] == j) assigned[t] = 1;
            }
            int idx[2];
            uint8_t nib = window_slots(assigned, idx);
            for (int s2 = 0; s2 < 2; s2++)
                for (int h = 0; h < 2; h++) {
                    int64_t k = 2 * (pbase + idx[s2]) + h;
                    stored[4 * w + 2 * s2 + h] = (assigned[idx[s2]] && k < K) ? W[r * K + k] : 0.0f;
                }
            put_nibble(&Wm[r * (K_lp / 16)], w, nib);
        }
        for (int64_t b = 0; b < K_lp / 32; b++) {        /* blocks of 16 stored */
            uint8_t codes[16];
            nvfp4_block(&stored[16 * b], 16, g, codes, &Ws[r * (K_lp / 32) + b]);
            for (int i = 0; i < 16; i++) put_fp4(&Wv[r * (K_lp / 4)], 16 * b + i, codes[i]);
        }
    }
    free(mask);
    free(win);
    free(stored);
    return SSREF_OK;
}

/* Source element of lifted position k under the pair slide of a pattern
 * with `group` pairs per group (window i of 4 pairs, element t of its 8):
 * [OM] 3.2's window map, base = 2Nh * (i / (Nh - 1)) + 2 * (i % (Nh - 1)),
 * applied to pairs.  -1 past the lifted length (zero padding). */
static int64_t pair_lift_src(int64_t k, int group, int64_t K_lift) {
    if (group == 0) return k;
    if (k >= K_lift) return -1;
    int64_t Nh = group / 2;
    int64_t wi = k / 8, t = k % 8;
    int64_t gi = wi / (Nh - 1), j = wi % (Nh - 1);
    return 2 * (gi * group + 2 * j) + t;
}

/* Dense NVFP4 matrix (the comparator's operands, or the dense operand of a
 * sparse product): rows of K (lifted on pairs for a pattern), zero-padded to
 * K_lp, blocks of `block` lifted elements, ONE global scale for the whole
 * matrix ([LC] NVFP4 row: a global scale per tensor), from the amax of all
 * its elements.  Xv [rows, K_lp/2] bytes, Xs [rows, K_lp/block], g_out[0]. */
int ssref_quant_nvfp4(const float *X, int64_t rows, int64_t K, int keep, int group, int block,
                      uint8_t *Xv, uint8_t *Xs, float *g_out) {
    int64_t K_lift, K_lp;
    int st = ssref_fp4_shape(keep, group, K, &K_lift, &K_lp);
    if (st || (block != 16 && block != 32)) return SSREF_EINVAL;
    float amax = 0.0f;
    for (int64_t i = 0; i < rows * K; i++) amax = fmaxf(amax, fabsf(X[i]));
    float g = ssref_nvfp4_global(amax);
    g_out[0] = g;
    float *lifted = (float *)malloc((size_t)K_lp * sizeof(float));
    memset(Xv, 0, (size_t)(rows * K_lp / 2));
    for (int64_t r = 0; r < rows; r++) {
        const float *x = &X[r * K];
        for (int64_t k = 0; k < K_lp; k++) {
            int64_t src = pair_lift_src(k, group, K_lift);
            lifted[k] = (src >= 0 && src < K) ? x[src] : 0.0f;
        }
        for (int64_t b = 0; b < K_lp / block; b++) {
            uint8_t codes[32];
            nvfp4_block(&lifted[block * b], block, g, codes, &Xs[r * (K_lp / block) + b]);
            for (int i = 0; i < block; i++) put_fp4(&Xv[r * (K_lp / 2)], block * b + i, codes[i]);
        }
    }
    free(lifted);
    return SSREF_OK;
}

/* The activation of a sparse NVFP4 product as the [LC] NVFP4 row defines
 * it: one global scale for the tensor, local scales per group of 16
 * elements along the ORIGINAL K (no lift, no padding to the lifted blocks).
 * The decoded values (codes times local scale, global scale not applied)
 * are then lifted to K_lp positions by the same pair window map, since
 * lifting only copies elements (the lossless decomposition, [SS] and
 * [OM] 2.3): Xlift [rows, K_lp] doubles, g_out[0].  The tensor-core path
 * cannot take this form (its sparse instruction scales 32 lifted K at a
 * time); the tests use it to measure what that costs. */
int ssref_nvfp4_act_page(const float *X, int64_t rows, int64_t K, int keep, int group,
                         double *Xlift, float *g_out) {
    int64_t K_lift, K_lp;
    int st = ssref_fp4_shape(keep, group, K, &K_lift, &K_lp);
    if (st) return st;
    float amax = 0.0f;
    for (int64_t i = 0; i < rows * K; i++) amax = fmaxf(amax, fabsf(X[i]));
    float g = ssref_nvfp4_global(amax);
    g_out[0] = g;
    int64_t K16 = round_up(K, 16);
    float *row = (float *)malloc((size_t)K16 * sizeof(float));
    double *dec = (double *)malloc((size_t)K16 * sizeof(double));
    for (int64_t r = 0; r < rows; r++) {
        for (int64_t k = 0; k < K16; k++) row[k] = k < K ? X[r * K + k] : 0.0f;
        for (int64_t b = 0; b < K16 / 16; b++) {
            uint8_t codes[16], sc;
            nvfp4_block(&row[16 * b], 16, g, codes, &sc);
            double s = ssref_e4m3_to_double(sc);
            for (int i = 0; i < 16; i++) dec[16 * b + i] = ssref_e2m1_to_double(codes[i]) * s;
        }
        for (int64_t k = 0; k < K_lp; k++) {
            int64_t src = pair_lift_src(k, group, K_lift);
            Xlift[r * K_lp + k] = (src >= 0 && src < K) ? dec[src] : 0.0;
        }
    }
    free(row);
    free(dec);
    return SSREF_OK;
}

/* Decode a sparse NVFP4 operand to lifted values (block scales applied, the
 * global scale not): A[r, k] for k < K_lp. */
int ssref_decode_sparse_nvfp4(const uint8_t *Av, const uint8_t *Am, const uint8_t *As,
                              int64_t rows, int64_t K_lp, double *A) {
    for (int64_t r = 0; r < rows; r++)
        for (int64_t w = 0; w < K_lp / 8; w++) {
            uint8_t nib = get_nibble(&Am[r * (K_lp / 16)], w);
            int p0 = nib & 3, p1 = (nib >> 2) & 3;
            if (p0 >= p1) return SSREF_EINVAL;
            for (int t = 0; t < 8; t++) A[r * K_lp + 8 * w + t] = 0.0;
            for (int s2 = 0; s2 < 2; s2++)
                for (int h = 0; h < 2; h++) {
                    int64_t i = 4 * w + 2 * s2 + h;          /* stored index */
                    double sc = ssref_e4m3_to_double(As[r * (K_lp / 32) + i / 16]);
                    double v = ssref_e2m1_to_double(get_fp4(&Av[r * (K_lp / 4)], i)) * sc;
                    A[r * K_lp + 8 * w + 2 * (s2 ? p1 : p0) + h] = v;
                }
        }
    return SSREF_OK;
}

int ssref_decode_dense_nvfp4(const uint8_t *Xv, const uint8_t *Xs, int64_t rows, int64_t K_lp,
                             int block, double *X) {
    for (int64_t r = 0; r < rows; r++)
        for (int64_t k = 0; k < K_lp; k++)
            X[r * K_lp + k] = ssref_e2m1_to_double(get_fp4(&Xv[r * (K_lp / 2)], k)) *
                              ssref_e4m3_to_double(Xs[r * (K_lp / block) + k / block]);
    return SSREF_OK;
}

/* Y[i, n] = ((float)sum_k Xd[m_i, k] Wd[n, k] * g_x[m_i]) * g_w[n] over
 * decoded operands (double sum of exact products, k order), bf16 RNE or
 * fp32 out. */
int ssref_matmul_nvfp4(const double *Xd, const float *g_x, const double *Wd, const float *g_w,
                       int64_t M, int64_t N, int64_t K, const int64_t *m_idx, int64_t n_rows,
                       int out_dtype, void *Y) {
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t i = 0; i < n_rows; i++) {
        int64_t m = m_idx ? m_idx[i] : i;
        if (m < 0 || m >= M) continue;
        for (int64_t n = 0; n < N; n++) {
            double acc = 0.0;
            for (int64_t k = 0; k < K; k++) acc += Xd[m * K + k] * Wd[n * K + k];
            volatile float a = (float)acc;
            volatile float t = a * g_x[m];
            volatile float y = t * g_w[n];
            if (out_dtype == SSREF_OUT_F32) ((float *)Y)[i * N + n] = y;
            else ((uint16_t *)Y)[i * N + n] = ssref_bf16_from_float(y);
        }
    }
    return SSREF_OK;
}
