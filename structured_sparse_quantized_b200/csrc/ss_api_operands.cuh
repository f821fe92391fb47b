// ss_api_operands.cuh -- the C entry points of libss (declared in
// include/ss.h) that prepare GEMM operands: weight compression
// (ss_compress_weight, ss_compress_weight_nvfp4), per-token activation
// quantisation with the lift (ss_quant_lift_act, ss_quant_lift_act_nvfp4)
// and the online 2:4 activation prune (ss_prune_act_2to4).  Included once, at
// the end of ss_api.cu, whose host helpers (device checks, launches) it uses.
#pragma once

extern "C" {

ss_status ss_compress_weight(const void* W, ss_in_dtype in_dtype, int64_t N, int64_t K,
                             ss_pattern p, ss_qdtype q, void* Wv, void* Wm, float* s_w,
                             ss_stream_t stream) {
    int64_t K_pad, K_lift, K_lp;
    ss_status st = ss_slide_shape(p, K, &K_pad, &K_lift, &K_lp);
    if (st != SS_OK) return st;
    const bool dense = p.group == 0;
    const int kq = kernel_q(q);
    if (kq < 0) return SS_ERR_INVALID_ARG;
    const bool scaled = kq != ss::kQBf16;  // the bf16 tier has no scale (s_w unused)
    if (!W || !Wv || (scaled && !s_w) || (!dense && !Wm) || N <= 0 || N > INT32_MAX)
        return SS_ERR_INVALID_ARG;
    if (in_dtype != SS_IN_F32 && in_dtype != SS_IN_BF16) return SS_ERR_INVALID_ARG;
    if (!aligned16(W) || !aligned16(Wv) || (scaled && !aligned16(s_w)) ||
        (!dense && !aligned16(Wm)))
        return SS_ERR_ALIGNMENT;
    const size_t smem = static_cast<size_t>((K_pad * 4 + 15) / 16 * 16) +
                        (dense ? 0 : 2 * static_cast<size_t>(K_pad / p.group)) + 16;
    if (smem > kMaxRowSmem) return SS_ERR_UNSUPPORTED;
    int dev;
    if ((st = check_device(&dev)) != SS_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* wv = static_cast<uint8_t*>(Wv);
    uint8_t* wm = static_cast<uint8_t*>(Wm);
    // sparse: one more CTA per padding row of the last 128-row metadata tile
    const int64_t rows_grid = dense ? N : (N + 127) / 128 * 128;
#define SS_COMPRESS(T, Q)                                                                      \
    do {                                                                                      \
        auto kern = ss::compress_weight_kernel<T, Q>;                                         \
        if ((st = set_smem(kern, dev, smem)) != SS_OK) return st;                             \
        st = launch_ex(kern, dim3(static_cast<unsigned>(rows_grid)), dim3(ss::kCompressThreads), \
                       smem, s, 1, static_cast<const T*>(W), N, K, p.keep, p.group, K_lift,   \
                       K_lp, wv, wm, s_w);                                                    \
    } while (0)
    if (in_dtype == SS_IN_BF16) {
        if (kq == ss::kQInt8) SS_COMPRESS(__nv_bfloat16, ss::kQInt8);
        else if (kq == ss::kQBf16) SS_COMPRESS(__nv_bfloat16, ss::kQBf16);
        else SS_COMPRESS(__nv_bfloat16, ss::kQE4M3);
    } else {
        if (kq == ss::kQInt8) SS_COMPRESS(float, ss::kQInt8);
        else if (kq == ss::kQBf16) SS_COMPRESS(float, ss::kQBf16);
        else SS_COMPRESS(float, ss::kQE4M3);
    }
#undef SS_COMPRESS
    return st;
}

ss_status ss_quant_lift_act(const void* X, ss_in_dtype in_dtype, int64_t M, int64_t K,
                            ss_pattern p, ss_qdtype q, void* Xq_lift, float* s_x,
                            ss_stream_t stream) {
    int64_t K_pad, K_lift, K_lp;
    ss_status st = ss_slide_shape(p, K, &K_pad, &K_lift, &K_lp);
    if (st != SS_OK) return st;
    const int kq = kernel_q(q);
    if (kq < 0) return SS_ERR_INVALID_ARG;
    const bool scaled = kq != ss::kQBf16;  // the bf16 tier only lifts (s_x unused)
    if (!X || !Xq_lift || (scaled && !s_x) || M <= 0 || M > INT32_MAX) return SS_ERR_INVALID_ARG;
    if (in_dtype != SS_IN_F32 && in_dtype != SS_IN_BF16) return SS_ERR_INVALID_ARG;
    if (!aligned16(X) || !aligned16(Xq_lift) || (scaled && !aligned16(s_x)))
        return SS_ERR_ALIGNMENT;
    if (!scaled) {
        int dev;
        if ((st = check_device(&dev)) != SS_OK) return st;
        cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
        const int Nh = p.group / 2;
        const int64_t units =
            Nh <= 2 ? K_lp / 8 : K_lift / (4 * (Nh - 1)) + (K_lp - K_lift) / 4;
        const dim3 grid(static_cast<unsigned>((units + ss::kLiftThreads - 1) / ss::kLiftThreads),
                        static_cast<unsigned>(M < 65535 ? M : 65535));
        uint16_t* xl = static_cast<uint16_t*>(Xq_lift);
        if (in_dtype == SS_IN_BF16)
            return launch_ex(ss::lift_bf16_kernel<__nv_bfloat16>, grid, dim3(ss::kLiftThreads), 0,
                             s, 1, static_cast<const __nv_bfloat16*>(X), M, K, Nh, K_lift, K_lp,
                             xl);
        return launch_ex(ss::lift_bf16_kernel<float>, grid, dim3(ss::kLiftThreads), 0, s, 1,
                         static_cast<const float*>(X), M, K, Nh, K_lift, K_lp, xl);
    }
    // one warp per token row; sliding patterns keep a quantised byte row per
    // warp in shared memory
    // one code row per row slot, with one zero chunk past the last group
    const int q_stride = p.group <= 4 ? 0 : static_cast<int>(round_up(K_pad, 16) + 16);
    int warps = ss::kWarpRowThreads / 32;
    if (q_stride > 0)
        while (warps > 1 && static_cast<size_t>(warps) * q_stride > kMaxRowSmem) warps /= 2;
    const size_t smem = static_cast<size_t>(warps) * q_stride;
    if (smem > kMaxRowSmem) return SS_ERR_UNSUPPORTED;
    int dev;
    if ((st = check_device(&dev)) != SS_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int Nh = p.group / 2;
    uint8_t* xq = static_cast<uint8_t*>(Xq_lift);
    const unsigned grid = static_cast<unsigned>((M + warps - 1) / warps);
#define SS_QLIFT(T, I8)                                                                        \
    do {                                                                                      \
        auto kern = ss::quant_lift_warp_kernel<T, I8>;                                        \
        if ((st = set_smem(kern, dev, smem)) != SS_OK) return st;                             \
        st = launch_ex(kern, dim3(grid), dim3(warps * 32), smem, s, 1,                        \
                       static_cast<const T*>(X), M, K, Nh, K_lift, K_lp, q_stride, xq, s_x);  \
    } while (0)
    // bf16 rows of up to kRegK = 16384 elements (K % 16 == 0) are read once, into registers
    const bool reg_path = in_dtype == SS_IN_BF16 && K % 16 == 0 && K <= ss::kRegK;
    if (reg_path) {
        // registers for the row: 1, 2 or 4 warps per row, each lane holding
        // just enough 16-element chunks
        const int wpr = K <= 4096 ? 1 : (K <= 8192 ? 2 : 4);
        const int chunks = static_cast<int>((K + 512 * wpr - 1) / (512 * wpr));
        const int rows_per_cta = (ss::kWarpRowThreads / 32) / wpr;
        const unsigned rgrid = static_cast<unsigned>((M + rows_per_cta - 1) / rows_per_cta);
        const auto* xb = static_cast<const __nv_bfloat16*>(X);
        // 6:8 lifts in registers; 4:6 and 8:10 keep one code row per row slot
        const size_t rsmem = Nh == 4 ? 0 : static_cast<size_t>(rows_per_cta) * q_stride;
#define SS_QREG(I8, C, W)                                                                      \
    do {                                                                                      \
        auto kern = ss::quant_lift_reg_kernel<I8, C, W>;                                      \
        if ((st = set_smem(kern, dev, rsmem)) != SS_OK) return st;                            \
        st = launch_ex(kern, dim3(rgrid), dim3(ss::kWarpRowThreads), rsmem, s, 1, xb, M, K,   \
                       Nh, K_lift, K_lp, q_stride, xq, s_x);                                 \
    } while (0)
#define SS_QREG_C(I8)                                                                          \
    do {                                                                                      \
        if (wpr == 1) {                                                                       \
            if (chunks <= 2) SS_QREG(I8, 2, 1);                                               \
            else if (chunks <= 4) SS_QREG(I8, 4, 1);                                          \
            else if (chunks <= 6) SS_QREG(I8, 6, 1);                                          \
            else if (chunks <= 7) SS_QREG(I8, 7, 1);                                          \
            else SS_QREG(I8, 8, 1);                                                           \
        } else if (wpr == 2) {                                                                \
            if (chunks <= 6) SS_QREG(I8, 6, 2);                                               \
            else if (chunks <= 7) SS_QREG(I8, 7, 2);                                          \
            else SS_QREG(I8, 8, 2);                                                           \
        } else {                                                                              \
            if (chunks <= 6) SS_QREG(I8, 6, 4);                                               \
            else if (chunks <= 7) SS_QREG(I8, 7, 4);                                          \
            else SS_QREG(I8, 8, 4);                                                           \
        }                                                                                     \
    } while (0)
        if (q == SS_INT8) SS_QREG_C(true);
        else SS_QREG_C(false);
#undef SS_QREG_C
#undef SS_QREG
    } else if (in_dtype == SS_IN_BF16) {
        if (q == SS_INT8) SS_QLIFT(__nv_bfloat16, true);
        else SS_QLIFT(__nv_bfloat16, false);
    } else {
        if (q == SS_INT8) SS_QLIFT(float, true);
        else SS_QLIFT(float, false);
    }
#undef SS_QLIFT
    return st;
}

ss_status ss_prune_act_2to4(const void* X, ss_in_dtype in_dtype, int64_t M, int64_t K,
                            ss_qdtype q, void* Xv, void* Xm, float* s_x, ss_stream_t stream) {
    int64_t K_lp;
    ss_status st = ss_act_2to4_shape(K, &K_lp);
    if (st != SS_OK) return st;
    const int kq = kernel_q(q);
    if (kq < 0) return SS_ERR_INVALID_ARG;
    const bool scaled = kq != ss::kQBf16;  // the bf16 tier has no scale (s_x unused)
    if (!X || !Xv || !Xm || (scaled && !s_x) || M <= 0 || M > INT32_MAX)
        return SS_ERR_INVALID_ARG;
    if (in_dtype != SS_IN_F32 && in_dtype != SS_IN_BF16) return SS_ERR_INVALID_ARG;
    if (!aligned16(X) || !aligned16(Xv) || !aligned16(Xm) || (scaled && !aligned16(s_x)))
        return SS_ERR_ALIGNMENT;
    int dev;
    if ((st = check_device(&dev)) != SS_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t* xv = static_cast<uint8_t*>(Xv);
    uint8_t* xm = static_cast<uint8_t*>(Xm);
    const int warps = ss::kWarpRowThreads / 32;
    // warps past M zero the padding rows of the last 128-row metadata tile
    const unsigned grid = static_cast<unsigned>(((M + 127) / 128 * 128 + warps - 1) / warps);
    // 8-bit tiers, bf16 rows split into 1, 2 or 4 chunks of up to 4096
    // elements (a multiple of 32): X streams through shared memory once, the
    // kept half of the row stays in registers
    const int wpr = K <= ss::kPruneChunkMax ? 1 : (K <= 2 * ss::kPruneChunkMax ? 2 : 4);
    if (in_dtype == SS_IN_BF16 && kq != ss::kQBf16 && K % (32 * wpr) == 0 &&
        K <= 4 * ss::kPruneChunkMax && M <= (int64_t{1} << 30)) {
        const int chunk_steps = static_cast<int>(K / wpr / 32);
        const int last_steps = static_cast<int>(K_lp / 32) - (wpr - 1) * chunk_steps;
        const int need = (std::max(chunk_steps, last_steps) + 31) / 32;
        int dev_sms = 148;
        cudaDeviceGetAttribute(&dev_sms, cudaDevAttrMultiProcessorCount, dev);
        const int rows_per_cta = (ss::kWarpRowThreads / 32) / wpr;
        const int64_t M_pad = (M + 127) / 128 * 128;
        const unsigned pgrid = static_cast<unsigned>(
            std::min<int64_t>(dev_sms, (M_pad + rows_per_cta - 1) / rows_per_cta));
        const auto* xb = static_cast<const __nv_bfloat16*>(X);
        const int Mi = static_cast<int>(M), Ki = static_cast<int>(K), Kl = static_cast<int>(K_lp);
#define SS_PRUNE_ST(Q, S, W, F)                                                               \
    do {                                                                                      \
        auto kern = ss::prune_act_stream_kernel<Q, S, W, F>;                                  \
        if ((st = set_smem(kern, dev, ss::kPruneSmem)) != SS_OK) return st;                   \
        return launch_ex(kern, dim3(pgrid), dim3(ss::kWarpRowThreads), ss::kPruneSmem, s, 1,  \
                         xb, Mi, Ki, Kl, xv, xm, s_x, 1u);                                    \
    } while (0)
        // full: the chunks fill exactly S steps per lane and there are no
        // padding steps
        const bool full2 = K_lp == K && chunk_steps == 64;
        const bool full4 = K_lp == K && chunk_steps == 128;
#define SS_PRUNE_ST_W(Q, W)                                                                   \
    do {                                                                                      \
        if (full2) SS_PRUNE_ST(Q, 2, W, true);                                                \
        if (full4) SS_PRUNE_ST(Q, 4, W, true);                                                \
        if (need <= 2) SS_PRUNE_ST(Q, 2, W, false);                                           \
        if (need <= 4) SS_PRUNE_ST(Q, 4, W, false);                                           \
        SS_PRUNE_ST(Q, 5, W, false);                                                          \
    } while (0)
#define SS_PRUNE_ST_Q(Q)                                                                      \
    do {                                                                                      \
        if (wpr == 1) SS_PRUNE_ST_W(Q, 1);                                                    \
        if (wpr == 2) SS_PRUNE_ST_W(Q, 2);                                                    \
        SS_PRUNE_ST_W(Q, 4);                                                                  \
    } while (0)
        if (kq == ss::kQInt8) SS_PRUNE_ST_Q(ss::kQInt8);
        SS_PRUNE_ST_Q(ss::kQE4M3);
#undef SS_PRUNE_ST_Q
#undef SS_PRUNE_ST_W
#undef SS_PRUNE_ST
    }
#define SS_PRUNE(T, Q)                                                                         \
    do {                                                                                      \
        st = launch_ex(ss::prune_act_warp_kernel<T, Q>, dim3(grid), dim3(ss::kWarpRowThreads), \
                       0, s, 1, static_cast<const T*>(X), M, K, K_lp, xv, xm, s_x);           \
    } while (0)
    if (in_dtype == SS_IN_BF16) {
        if (kq == ss::kQInt8) SS_PRUNE(__nv_bfloat16, ss::kQInt8);
        else if (kq == ss::kQBf16) SS_PRUNE(__nv_bfloat16, ss::kQBf16);
        else SS_PRUNE(__nv_bfloat16, ss::kQE4M3);
    } else {
        if (kq == ss::kQInt8) SS_PRUNE(float, ss::kQInt8);
        else if (kq == ss::kQBf16) SS_PRUNE(float, ss::kQBf16);
        else SS_PRUNE(float, ss::kQE4M3);
    }
#undef SS_PRUNE
    return st;
}

// ---------------------------------------------------------------- NVFP4

ss_status ss_compress_weight_nvfp4(const void* W, ss_in_dtype in_dtype, int64_t N, int64_t K,
                                   ss_pattern p, void* Wv, void* Wm, void* Ws, float* g_w,
                                   ss_stream_t stream) {
    int64_t K_lift, K_lp;
    ss_status st = ss_fp4_shape(p, K, &K_lift, &K_lp);
    if (st != SS_OK) return st;
    const bool dense = p.group == 0;
    if (!W || !Wv || !Ws || !g_w || (!dense && !Wm) || N <= 0 || N > INT32_MAX)
        return SS_ERR_INVALID_ARG;
    if (in_dtype != SS_IN_F32 && in_dtype != SS_IN_BF16) return SS_ERR_INVALID_ARG;
    if (!aligned16(W) || !aligned16(Wv) || !aligned16(Ws) || !aligned16(g_w) ||
        (!dense && !aligned16(Wm)))
        return SS_ERR_ALIGNMENT;
    const int64_t P_pad = dense ? (K + 1) / 2 : round_up((K + 1) / 2, p.group);
    const int64_t len = dense ? K_lp : 2 * P_pad;
    const size_t smem1 = static_cast<size_t>(round_up(2 * P_pad, 4) * 4);
    const size_t smem2 = static_cast<size_t>(round_up(len, 4) * 4) +
                         (dense ? 0 : static_cast<size_t>(K_lp / 2 * 4 + 2 * (P_pad / p.group) + 16));
    if (smem1 > kMaxRowSmem || smem2 > kMaxRowSmem) return SS_ERR_UNSUPPORTED;
    int dev;
    if ((st = check_device(&dev)) != SS_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    auto* amax = reinterpret_cast<unsigned int*>(g_w);  // pass 1 leaves the amax bits here
    if (cudaMemsetAsync(amax, 0, sizeof(unsigned int), s) != cudaSuccess) return SS_ERR_CUDA;
    const int64_t rows_grid = (N + 127) / 128 * 128;
    auto* wv = static_cast<uint8_t*>(Wv);
    auto* wm = static_cast<uint8_t*>(Wm);
    auto* ws = static_cast<uint8_t*>(Ws);
#define SS_FP4W(T)                                                                             \
    do {                                                                                      \
        auto k1 = ss::fp4_weight_amax_kernel<T>;                                               \
        auto k2 = ss::compress_weight_nvfp4_kernel<T>;                                         \
        if ((st = set_smem(k1, dev, smem1)) != SS_OK) return st;                              \
        if ((st = set_smem(k2, dev, smem2)) != SS_OK) return st;                              \
        const T* w = static_cast<const T*>(W);                                                \
        if ((st = launch_ex(k1, dim3(static_cast<unsigned>(N)), dim3(ss::kCompressThreads),   \
                            smem1, s, 1, w, N, K, p.keep, p.group, amax)) != SS_OK)           \
            return st;                                                                        \
        if ((st = launch_ex(k2, dim3(static_cast<unsigned>(rows_grid)),                       \
                            dim3(ss::kCompressThreads), smem2, s, 1, w, N, K, p.keep,          \
                            p.group, K_lift, K_lp, amax, wv, wm, ws)) != SS_OK)               \
            return st;                                                                        \
    } while (0)
    if (in_dtype == SS_IN_BF16) SS_FP4W(__nv_bfloat16);
    else SS_FP4W(float);
#undef SS_FP4W
    return launch_ex(ss::fp4_global_kernel, dim3(1), dim3(32), 0, s, 1, g_w);
}

ss_status ss_quant_lift_act_nvfp4(const void* X, ss_in_dtype in_dtype, int64_t M, int64_t K,
                                  ss_pattern p, int32_t block, void* Xv, void* Xs, float* g_x,
                                  ss_stream_t stream) {
    int64_t K_lift, K_lp;
    ss_status st = ss_fp4_shape(p, K, &K_lift, &K_lp);
    if (st != SS_OK) return st;
    if (!X || !Xv || !Xs || !g_x || M <= 0 || M > INT32_MAX || (block != 16 && block != 32))
        return SS_ERR_INVALID_ARG;
    if (in_dtype != SS_IN_F32 && in_dtype != SS_IN_BF16) return SS_ERR_INVALID_ARG;
    if (!aligned16(X) || !aligned16(Xv) || !aligned16(Xs) || !aligned16(g_x))
        return SS_ERR_ALIGNMENT;
    int dev;
    if ((st = check_device(&dev)) != SS_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // g_x[0] first accumulates the amax bits of X (zeroed, then atomicMax
    // over the tensor), pass 2 derives g from it, and the last launch turns
    // it into g = amax / 2688 in place.
    auto* amax = reinterpret_cast<unsigned int*>(g_x);
    if ((st = launch_ex(ss::zero_word_kernel, dim3(1), dim3(32), 0, s, 1, amax)) != SS_OK) return st;
    const int64_t n = M * K;
    const int64_t esz = in_dtype == SS_IN_BF16 ? 2 : 4;
    const int64_t nv = n * esz / 16;
    const unsigned agrid = static_cast<unsigned>(
        std::max<int64_t>(1, std::min<int64_t>((nv + 255) / 256, 148 * 8)));
    if (in_dtype == SS_IN_BF16)
        st = launch_ex(ss::fp4_act_amax_kernel<__nv_bfloat16>, dim3(agrid), dim3(256), 0, s, 1,
                       static_cast<const __nv_bfloat16*>(X), n, amax);
    else
        st = launch_ex(ss::fp4_act_amax_kernel<float>, dim3(agrid), dim3(256), 0, s, 1,
                       static_cast<const float*>(X), n, amax);
    if (st != SS_OK) return st;
    if (K_lp > INT32_MAX / 2 || M > (int64_t{1} << 30)) return SS_ERR_UNSUPPORTED;
    // one warp per row at a time: up to 8 row slots per SM
    const int64_t M_pad = (M + 127) / 128 * 128;
    const unsigned grid = static_cast<unsigned>(std::min<int64_t>((M_pad + 7) / 8, 148 * 8));
    const int Mi = static_cast<int>(M), Ki = static_cast<int>(K);
    const int Kl = static_cast<int>(K_lift), Kp = static_cast<int>(K_lp);
    const int Nh = p.group / 2;
    auto* xv = static_cast<uint8_t*>(Xv);
    auto* xs = static_cast<uint8_t*>(Xs);
#define SS_FP4X(T, B, NH)                                                                     \
    st = launch_ex(ss::quant_nvfp4_act_kernel<T, B, NH>, dim3(grid), dim3(256), 0, s, 1,     \
                   static_cast<const T*>(X), Mi, Ki, Kl, Kp, amax, xv, xs)
#define SS_FP4NH(T, B)                                                                        \
    switch (Nh) {                                                                             \
        case 3: SS_FP4X(T, B, 3); break;                                                      \
        case 4: SS_FP4X(T, B, 4); break;                                                      \
        case 5: SS_FP4X(T, B, 5); break;                                                      \
        default: SS_FP4X(T, B, 2); break;                                                     \
    }
    if (in_dtype == SS_IN_BF16) {
        if (block == 32) { SS_FP4NH(__nv_bfloat16, 32) }
        else { SS_FP4NH(__nv_bfloat16, 16) }
    } else {
        if (block == 32) { SS_FP4NH(float, 32) }
        else { SS_FP4NH(float, 16) }
    }
#undef SS_FP4NH
#undef SS_FP4X
    if (st != SS_OK) return st;
    return launch_ex(ss::fp4_global_kernel, dim3(1), dim3(32), 0, s, 1, g_x);
}

}  // extern "C"
