// ss_gemm.cuh -- persistent, warp-specialised tcgen05 GEMM for sm_100a, in a
// sparse (tcgen05.mma.sp, 2:4 A operand with metadata) and a dense
// (tcgen05.mma) variant of the same construction.
//
//   D[a, b] = sum_k A[a, k] * B[b, k]       (A, B both K-major bytes)
//   Y       = ((float)D * s_x) * s_w       (fp32 round-to-nearest, then
//                                          bf16 RNE or fp32 out)
//
// The sparse variant is the matmul the SlideSparse pages run on the sparse
// tensor cores after the sliding-window decomposition ("SlideSparse:
// 布局稀疏边界", 66bd.net: every window satisfies 2:4 and runs directly on the
// sparse tensor core; SlideSparse write-up, omica.com.cn, 2.2 sparse GEMM
// execution).  The dense variant is the like-for-like comparison.
//
// CTA = 6 warps, one CTA per SM, persistent over output tiles:
//   warp 0       TMA producer: A tile (128 rows), B tile (BN rows) and, for
//                the sparse variant, the 128 x 16-byte metadata tile of each
//                K stage, into a ring of shared-memory stages.
//   warp 1       allocates 512 TMEM columns; one lane issues the MMAs (and
//                the shared->tensor-memory metadata copies) into one of two
//                accumulator buffers and commits stage / accumulator
//                barriers.
//   warps 2-5    epilogue: tcgen05.ld the accumulator (lane = A row, column =
//                B row), scale, convert, store Y; release the buffer.
// Stage K is 128 logical elements: dense = 4 MMAs of K=32 (A and B 128-byte
// rows, 128B swizzle); sparse = 2 MMAs of K=64 (A holds 64 compressed bytes
// per row, 64B swizzle; B 128-byte rows, 128B swizzle; metadata 16 bytes per
// A row, one tcgen05.cp of 128 lanes x 128 bits).
// Every wait is bounded (ss_common.cuh); nothing here multicasts.
#pragma once

#include "ss_common.cuh"

namespace ss {

constexpr int kGemmThreads = 192;
constexpr int kTileA = 128;
constexpr int kTmemCols = 512;

template <bool kSparse>
struct GemmCfg {
    static constexpr int kStageK = 128;                    // logical K per stage
    static constexpr int kMmaK = kSparse ? 64 : 32;        // logical K per MMA
    static constexpr int kMmaPerStage = kStageK / kMmaK;   // 2 / 4
    static constexpr int kARowBytes = kSparse ? 64 : 128;  // A bytes per row per stage
    static constexpr int kABytes = kTileA * kARowBytes;
    static constexpr int kBnMax = kSparse ? 224 : 256;     // 2 accumulators (+ metadata) in TMEM
    static constexpr int kBBytes = kBnMax * 128;
    static constexpr int kEBytes = kSparse ? kTileA * 16 : 0;
    static constexpr int kStageBytes = kABytes + kBBytes + kEBytes;
    static constexpr int kStages = kSparse ? 5 : 4;
    static constexpr int kAccStride = kBnMax;              // TMEM columns between buffers
    static constexpr int kECol = 2 * kBnMax;               // metadata columns (sparse)
    static constexpr int kESlots = 4;                      // 4 columns each
    static constexpr int kSmemBytes = kStages * kStageBytes + 1024 /*align*/ + 256 /*barriers*/;
    static_assert(kStageBytes % 1024 == 0, "stage must keep 1024-byte alignment");
    static_assert(kABytes % 1024 == 0 && (kABytes + kBBytes) % 1024 == 0, "tile alignment");
    static_assert(!kSparse || kECol + kESlots * 4 <= kTmemCols, "TMEM budget");
};

struct GemmArgs {
    int rowsA;        // rows of A (128-row tiles)
    int rowsB;        // rows of B (BN-row tiles)
    int k_stages;     // K / 128
    int bn;           // B rows per tile (multiple of 32, <= kBnMax)
    int a_is_w;       // 1: A rows are output channels (Y[b, a]); 0: Y[a, b]
    int ldy;          // leading dimension of Y (= N)
    const float* s_a;
    const float* s_b;
    void* y;
};

__device__ __forceinline__ bool mbar_drain(uint64_t* bar, uint32_t parity) {
    const uint32_t b = smem_u32(bar);
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(b, parity))
        if (global_timer_ns() - t0 > 100000000ull) return false;  // 100 ms
    return true;
}

template <bool kInt8, bool kOutBf16>
__device__ __forceinline__ void store_scaled(void* y, int64_t off, uint32_t acc_bits, float sx,
                                             float sw) {
    const float acc = kInt8 ? __int2float_rn(static_cast<int32_t>(acc_bits))
                            : __uint_as_float(acc_bits);
    const float v = __fmul_rn(__fmul_rn(acc, sx), sw);
    if constexpr (kOutBf16)
        reinterpret_cast<__nv_bfloat16*>(y)[off] = __float2bfloat16_rn(v);
    else
        reinterpret_cast<float*>(y)[off] = v;
}

template <bool kSparse, bool kInt8, bool kOutBf16>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                const __grid_constant__ CUtensorMap tm_e, const GemmArgs args) {
    using C = GemmCfg<kSparse>;
    extern __shared__ __align__(1024) uint8_t smem_dyn[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStageBytes);
    uint64_t* empty = full + C::kStages;
    uint64_t* acc_full = empty + C::kStages;
    uint64_t* acc_empty = acc_full + 2;
    uint64_t* drain = acc_empty + 2;
    uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(drain + 1);
    __shared__ int abort_flag_storage;
    volatile int* abort_flag = &abort_flag_storage;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int nA = (args.rowsA + kTileA - 1) / kTileA;
    const int nB = (args.rowsB + args.bn - 1) / args.bn;
    const int n_tiles = nA * nB;

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 4);
        }
        mbar_init(drain, 1);
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_base_slot, kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_base_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            tma_prefetch_desc(&tm_a);
            tma_prefetch_desc(&tm_b);
            if (kSparse) tma_prefetch_desc(&tm_e);
            const uint32_t tx = C::kABytes + args.bn * 128 + C::kEBytes;
            int s = 0;
            uint32_t ph = 0, armed = 0, armed_par = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x) {
                const int a0 = (t % nA) * kTileA;
                const int b0 = (t / nA) * args.bn;
                for (int kb = 0; kb < args.k_stages; ++kb) {
                    if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    uint8_t* st = smem + s * C::kStageBytes;
                    mbar_arrive_expect_tx(&full[s], tx);
                    tma_load_2d(st, &tm_a, &full[s], kb * C::kARowBytes, a0);
                    tma_load_2d(st + C::kABytes, &tm_b, &full[s], kb * 128, b0);
                    if (kSparse)
                        tma_load_2d(st + C::kABytes + C::kBBytes, &tm_e, &full[s], kb * 16, a0);
                    armed |= 1u << s;
                    armed_par = (armed_par & ~(1u << s)) | (ph << s);
                    if (++s == C::kStages) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
            }
            if (!ok) {  // let every copy already issued land before the CTA exits
                for (int i = 0; i < C::kStages; ++i)
                    if ((armed >> i) & 1u) mbar_drain(&full[i], (armed_par >> i) & 1u);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            const uint32_t idesc = make_idesc(kSparse, kInt8, kTileA, args.bn);
            int s = 0;
            uint32_t ph = 0;
            uint32_t e_iter = 0;
            bool ok = true;
            int i = 0;
            for (int t = blockIdx.x; t < n_tiles && ok; t += gridDim.x, ++i) {
                const int buf = i & 1;
                const uint32_t aph = (i >> 1) & 1;
                if (!mbar_wait(&acc_empty[buf], aph ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + buf * C::kAccStride;
                for (int kb = 0; kb < args.k_stages; ++kb) {
                    if (!mbar_wait(&full[s], ph, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + s * C::kStageBytes);
                    const uint32_t b_addr = a_addr + C::kABytes;
                    uint32_t e_tmem = 0;
                    if constexpr (kSparse) {
                        e_tmem = tmem_base + C::kECol + 4 * (e_iter % C::kESlots);
                        ++e_iter;
                        const uint64_t e_desc =
                            smem_desc(b_addr + C::kBBytes, 128 * 16, 128, kSwizzleNone);
                        tc_cp_128x128b(e_tmem, e_desc);
                    }
#pragma unroll
                    for (int j = 0; j < C::kMmaPerStage; ++j) {
                        const uint32_t acc = (kb > 0 || j > 0) ? 1u : 0u;
                        if constexpr (kSparse) {
                            const uint64_t a_desc =
                                smem_desc(a_addr + j * 32, 16, 8 * 64, kSwizzle64B);
                            const uint64_t b_desc =
                                smem_desc(b_addr + j * 64, 16, 8 * 128, kSwizzle128B);
                            mma_sparse<kInt8>(d_tmem, a_desc, b_desc, e_tmem + 2 * j, idesc, acc);
                        } else {
                            const uint64_t a_desc =
                                smem_desc(a_addr + j * 32, 16, 8 * 128, kSwizzle128B);
                            const uint64_t b_desc =
                                smem_desc(b_addr + j * 32, 16, 8 * 128, kSwizzle128B);
                            mma_dense<kInt8>(d_tmem, a_desc, b_desc, idesc, acc);
                        }
                    }
                    tc_commit(&empty[s]);  // stage free once these MMAs have read it
                    if (++s == C::kStages) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) break;
                tc_commit(&acc_full[buf]);
            }
            if (!ok) {  // wait for every MMA already issued before TMEM is freed
                tc_commit(drain);
                mbar_drain(drain, 0);
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        const int lane_row = q * 32 + lane;
        int i = 0;
        for (int t = blockIdx.x; t < n_tiles; t += gridDim.x, ++i) {
            const int buf = i & 1;
            const uint32_t aph = (i >> 1) & 1;
            if (!mbar_wait(&acc_full[buf], aph, abort_flag)) break;
            tc_fence_after();
            const int a_row = (t % nA) * kTileA + lane_row;
            const int b0 = (t / nA) * args.bn;
            const bool row_ok = a_row < args.rowsA;
            const float sa = row_ok ? __ldg(args.s_a + a_row) : 0.0f;
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                   static_cast<uint32_t>(buf * C::kAccStride);
            for (int c = 0; c < args.bn; c += 32) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(t_row + c, r);
                tmem_ld_wait();
                if (row_ok) {
#pragma unroll
                    for (int u = 0; u < 32; ++u) {
                        const int b_row = b0 + c + u;
                        if (b_row < args.rowsB) {
                            const float sb = __ldg(args.s_b + b_row);
                            if (args.a_is_w)
                                store_scaled<kInt8, kOutBf16>(
                                    args.y, static_cast<int64_t>(b_row) * args.ldy + a_row, r[u],
                                    sb, sa);
                            else
                                store_scaled<kInt8, kOutBf16>(
                                    args.y, static_cast<int64_t>(a_row) * args.ldy + b_row, r[u],
                                    sa, sb);
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[buf]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

}  // namespace ss
