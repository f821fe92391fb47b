// ss_gemm_splitk.cuh -- split-K GEMM for decode-sized token counts (the
// weight-sparse and dense paths with A = weight, at most kSkBn tokens).
//
// At decode sizes the GEMM streams the weight: with one 128-row A tile per CTA
// a small weight (e.g. 4096 channels = 32 tiles) keeps only a fraction of the
// 148 SMs busy.  Here the K range of each A tile is cut into S parts that run
// on the S CTAs of one thread-block cluster (S = 2, 4 or 8).  Each CTA
// accumulates its part in tensor memory (tcgen05.mma(.sp), M = 128, single
// SM), writes the raw partial accumulator to its shared memory, and after a
// cluster barrier each CTA reduces 128/S of the tile's rows over the S
// partials through distributed shared memory (ld.shared::cluster), applies
// the epilogue of the one-pass kernels and stores Y.  INT8 partials are added
// as int32, so the result stays exact; fp32 partials are added in CTA order.
//
// CTA = 6 warps, one (tile, K part) per CTA:
//   warp 0     TMA producer into a ring of stages (A rows, B atoms, metadata),
//              as in gemm_kernel's single-SM form.
//   warp 1     TMEM allocation and the MMA loop (one elected lane issues).
//   warps 2-5  drain the accumulator into shared memory, then the reduction.
// Every wait is bounded; on a timeout each role skips its remaining work but
// still reaches both cluster barriers, so no CTA of the cluster is left
// waiting.  No load multicasts.
#pragma once

#include "ss_gemm.cuh"

namespace ss {

constexpr int kSplitKThreads = 192;  // warp 0 producer, warp 1 MMA, warps 2-5 epilogue
constexpr int kSkBn = 64;  // tokens (B rows) at most

template <bool kSparse, int kEb>
struct SplitKCfg {
    using G = GemmCfg<kSparse, 1, kEb>;
    static constexpr int kStageK = G::kStageK;
    static constexpr int kARowBytes = G::kARowBytes;
    static constexpr int kABytes = G::kABytes;  // 16 KB
    static constexpr int kBAtoms = G::kBAtoms;
    static constexpr int kBAtomBytes = kSkBn * 128;
    static constexpr int kBBytes = kBAtoms * kBAtomBytes;
    static constexpr int kEChunks = G::kEChunks;
    static constexpr int kEBytes = kEChunks * kTileA * 16;
    static constexpr int kBOffset = kABytes;
    static constexpr int kEOffset = kBOffset + kBBytes;
    static constexpr int kStageBytes = (kEOffset + kEBytes + 1023) / 1024 * 1024;
    static constexpr int kPartBytes = kSkBn * kTileA * 4;  // [column][128 rows] of 32-bit
    static constexpr int kStagesRaw = (225 * 1024 - 1024 - 256 - kPartBytes) / kStageBytes;
    static constexpr int kStages = kStagesRaw > 8 ? 8 : kStagesRaw;
    static constexpr int kPartOffset = kStages * kStageBytes;
    static constexpr int kBarOffset = kPartOffset + kPartBytes;
    static constexpr int kSmemBytes = kBarOffset + 256 + 1024;
    static constexpr int kECol = kSkBn;          // metadata slots after the accumulator
    static constexpr int kESlotCols = 4 * kEChunks;
    static constexpr int kTmemCols = 128;
    static_assert(kECol + kStages * kESlotCols <= kTmemCols, "TMEM budget");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
    static_assert(kStages >= 2, "pipeline depth");
    static_assert((2 * kStages + 2) * 8 + 4 <= 256, "barrier area");
    static_assert(kBAtomBytes % 1024 == 0 && kABytes % 1024 == 0, "tile alignment");
};

// args.k_stages: stages of the whole K; args.bn: B rows (a multiple of 32,
// <= kSkBn, covering every B row); args.a_is_w must be 1.
template <bool kSparse, int kQ, bool kOutBf16>
__global__ void __launch_bounds__(kSplitKThreads, 1)
    gemm_splitk_kernel(const __grid_constant__ CUtensorMap tm_a,
                       const __grid_constant__ CUtensorMap tm_b,
                       const __grid_constant__ CUtensorMap tm_e, const GemmArgs args) {
    constexpr bool kInt8 = kQ == kQInt8;
    constexpr bool kBf16 = kQ == kQBf16;
    using C = SplitKCfg<kSparse, kBf16 ? 2 : 1>;
    extern __shared__ __align__(1024) uint8_t smem_dyn[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~static_cast<uintptr_t>(1023));
    uint32_t* part = reinterpret_cast<uint32_t*>(smem + C::kPartOffset);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOffset);
    uint64_t* empty = full + C::kStages;
    uint64_t* acc_full = empty + C::kStages;
    uint64_t* drain = acc_full + 1;
    uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(drain + 1);
    __shared__ int abort_flag_storage;
    volatile int* abort_flag = &abort_flag_storage;
    pdl_trigger();

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int S = static_cast<int>(gridDim.x) / ((args.rowsA + kTileA - 1) / kTileA);
    const int split = static_cast<int>(cluster_ctarank());  // this CTA's K part
    const int a0 = static_cast<int>(blockIdx.x) / S * kTileA;
    const int kb0 = split * args.k_stages / S;
    const int kb1 = (split + 1) * args.k_stages / S;

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(drain, 1);
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_base_slot, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_base_slot;
    if (warp != 0) pdl_wait();

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (elect_one()) {
            tma_prefetch_desc(&tm_a);
            tma_prefetch_desc(&tm_b);
            if (kSparse) tma_prefetch_desc(&tm_e);
            for (int kb = kb0; kb < kb1 && kb < kb0 + kL2PrefetchStages; ++kb) {
                tma_prefetch_l2_2d(&tm_a, kb * C::kARowBytes, a0);  // the weight, into L2
#pragma unroll
                for (int u = 0; u < C::kEChunks; ++u)
                    tma_prefetch_l2_2d(&tm_e, 0,
                                       ((a0 >> 7) * args.e_chunks + kb * C::kEChunks + u) * 16);
            }
        }
        __syncwarp();
        pdl_wait();
        const uint32_t tx = C::kABytes + C::kEBytes + C::kBAtoms * args.bn * 128;
        int s = 0;
        uint32_t ph = 0, armed = 0, armed_par = 0;
        bool ok = true;
        for (int kb = kb0; kb < kb1; ++kb) {
            if (!__all_sync(0xffffffffu, mbar_wait(&empty[s], ph ^ 1u, abort_flag))) {
                ok = false;
                break;
            }
            if (elect_one()) {
                uint8_t* st = smem + s * C::kStageBytes;
                mbar_arrive_expect_tx(&full[s], tx);
                tma_load_2d(st, &tm_a, &full[s], kb * C::kARowBytes, a0);
#pragma unroll
                for (int u = 0; u < C::kBAtoms; ++u)
                    tma_load_2d(st + C::kBOffset + u * C::kBAtomBytes, &tm_b, &full[s],
                                (kb * C::kBAtoms + u) * 128, 0);
#pragma unroll
                for (int u = 0; u < C::kEChunks; ++u)
                    tma_load_2d(st + C::kEOffset + u * kTileA * 16, &tm_e, &full[s], 0,
                                ((a0 >> 7) * args.e_chunks + kb * C::kEChunks + u) * 16);
            }
            __syncwarp();
            armed |= 1u << s;
            armed_par = (armed_par & ~(1u << s)) | (ph << s);
            if (++s == C::kStages) {
                s = 0;
                ph ^= 1u;
            }
        }
        if (!ok && lane == 0) {  // let the copies already issued land
            for (int i = 0; i < C::kStages; ++i)
                if ((armed >> i) & 1u) mbar_drain(&full[i], (armed_par >> i) & 1u);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        const uint32_t idesc = make_idesc_q(kSparse, kQ, kTileA, args.bn);
        const uint32_t base = smem_u32(smem);
        const uint64_t a_desc0 = smem_desc(base, 16, 8 * C::kARowBytes, kSwizzle128B);
        const uint64_t b_desc0 = smem_desc(base + C::kBOffset, 16, 1024, kSwizzle128B);
        const uint64_t e_desc0 = smem_desc(base + C::kEOffset, 128 * 16, 128, kSwizzleNone);
        int s = 0;
        uint32_t ph = 0;
        bool ok = true;
        for (int kb = kb0; kb < kb1; ++kb) {
            if (!__all_sync(0xffffffffu, mbar_wait(&full[s], ph, abort_flag))) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint64_t soff = static_cast<uint64_t>((s * C::kStageBytes) >> 4);
            const uint32_t e_tmem = tmem_base + C::kECol + C::kESlotCols * s;
            if (elect_one()) {
#pragma unroll
                for (int j = 0; j < C::G::kMmaPerStage; ++j) {
                    const uint32_t accum = (kb > kb0 || j > 0) ? 1u : 0u;
                    const uint64_t a_desc = a_desc0 + soff + ((j * 32) >> 4);
                    if constexpr (kSparse) {
                        if (j == 0) {
#pragma unroll
                            for (int u = 0; u < C::kEChunks; ++u)
                                tc_cp_128x128b(e_tmem + 4 * u,
                                               e_desc0 + soff + ((u * kTileA * 16) >> 4));
                        }
                        const uint64_t b_desc =
                            b_desc0 + soff + (((j >> 1) * C::kBAtomBytes + (j & 1) * 64) >> 4);
                        if constexpr (kBf16)
                            mma_sparse_bf16_g<1>(tmem_base, a_desc, b_desc,
                                                 e_tmem + 2 * (j >> 1),
                                                 idesc | static_cast<uint32_t>(j & 1), accum);
                        else
                            mma_sparse_g<1, kInt8>(tmem_base, a_desc, b_desc, e_tmem + 2 * j,
                                                   idesc, accum);
                    } else {
                        const uint64_t b_desc = b_desc0 + soff + ((j * 32) >> 4);
                        if constexpr (kBf16)
                            mma_dense_bf16_g<1>(tmem_base, a_desc, b_desc, idesc, accum);
                        else
                            mma_dense_g<1, kInt8>(tmem_base, a_desc, b_desc, idesc, accum);
                    }
                }
            }
            __syncwarp();
            if (elect_one()) tc_commit(&empty[s]);
            __syncwarp();
            if (++s == C::kStages) {
                s = 0;
                ph ^= 1u;
            }
        }
        if (elect_one()) tc_commit(ok ? acc_full : drain);  // all issued MMAs done
        __syncwarp();
        if (!ok) {
            if (elect_one()) mbar_drain(drain, 0);
            __syncwarp();
        }
    } else {
        // ------------------------------------------------------------ drain to smem
        const int q = warp & 3;  // TMEM lane quarter
        const int row = q * 32 + lane;
        const bool got = kb1 > kb0 ? mbar_wait(acc_full, 0, abort_flag) : true;
        if (named_bar_and(1, 128, got)) {
            tc_fence_after();
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
            for (int c = 0; c < args.bn; c += 32) {
                uint32_t r[32];
                if (kb1 > kb0) {
                    tmem_ld_32x32b_x32(t_row + c, r);
                    tmem_ld_wait();
                } else {
#pragma unroll
                    for (int u = 0; u < 32; ++u) r[u] = 0u;  // empty K part: zero partial
                }
#pragma unroll
                for (int u = 0; u < 32; ++u) part[(c + u) * kTileA + row] = r[u];
            }
        }
    }
    tc_fence_before();
    cluster_sync_all();  // every partial of the cluster is in shared memory

    if (warp >= 2 && !*abort_flag) {
        // ------------------------------------------------------------ reduce + epilogue
        const int rows = kTileA / S;  // rows of the tile this CTA finishes
        const int r0 = split * rows;
        const int et = threadIdx.x - 64;  // 0..127
        uint32_t peer[8];
        for (int p = 0; p < S; ++p) peer[p] = map_to_rank(part, static_cast<uint32_t>(p));
        for (int f = et; f < rows * args.bn; f += 128) {
            const int rl = f % rows, col = f / rows;
            const int ch = a0 + r0 + rl;  // A row = output channel
            const int tok = col;          // B row = token
            if (ch >= args.rowsA || tok >= args.rowsB) continue;
            const uint32_t off = static_cast<uint32_t>((col * kTileA + r0 + rl) * 4);
            float accv;
            if constexpr (kInt8) {
                int32_t acc = 0;
                for (int p = 0; p < S; ++p) {
                    uint32_t v;
                    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(peer[p] + off));
                    acc += static_cast<int32_t>(v);
                }
                accv = __int2float_rn(acc);
            } else {
                accv = 0.0f;
                for (int p = 0; p < S; ++p) {
                    uint32_t v;
                    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(peer[p] + off));
                    accv = __fadd_rn(accv, __uint_as_float(v));
                }
            }
            const float sa = load_scale<kBf16>(args.s_a, ch, true);
            const float sb = load_scale<kBf16>(args.s_b, tok, true);
            const float y = __fmul_rn(__fmul_rn(accv, sb), sa);
            const int64_t o = static_cast<int64_t>(tok) * args.ldy + ch;
            if constexpr (kOutBf16)
                reinterpret_cast<__nv_bfloat16*>(args.y)[o] = __float2bfloat16_rn(y);
            else
                reinterpret_cast<float*>(args.y)[o] = y;
        }
    }
    cluster_sync_all();  // no CTA leaves while a peer may still read its partials
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, C::kTmemCols);
    }
}

}  // namespace ss
