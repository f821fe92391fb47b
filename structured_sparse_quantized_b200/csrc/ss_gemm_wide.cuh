// ss_gemm_wide.cuh -- the sparse GEMM of ss_gemm.cuh with output tiles two
// B tiles wide, for large problems.
//
// Same operation, same operands, same epilogue arithmetic as gemm_kernel:
//   D[a, b] = sum_k A[a, k] * B[b, k]
//   A = weight (rows = channels):   Y[b, a] = bf16(((float)D * s_b) * s_a)
//   A = activation (rows = tokens): Y[a, b] = bf16(((float)D * s_a) * s_b)
// (the sparse matmul after the sliding-window decomposition: SlideSparse
// write-up, omica.com.cn, 2.2 sparse GEMM execution).
//
// Why a second shape.  A pair of CTAs (tcgen05 cta_group::2, M = 256) with
// one B tile of N = 224 must bring 12 KB into each SM's shared memory per
// K = 64 MMA step (A 4 KB + metadata 1 KB + half the B tile 7 KB), about
// 107 bytes per tensor-core cycle at the sparse rate; an SM takes in ~68,
// so the tensor pipe idles ~40% of the time.  Here one output tile is
// 256 A rows x 2 B tiles: each A slice feeds two MMAs, the first reading it
// from shared memory into the tensor core's collector buffer
// (collector::a::fill) and the second taking it from there
// (collector::a::lastuse), so per MMA only 9.5 KB come in and the A slice is
// read from shared memory once.
//
// The two accumulators (2 x 224 columns) fill tensor memory, so they are
// single-buffered.  To free them quickly the epilogue runs 8 warps (two per
// TMEM lane quarter, one per B tile); each drains its 32 x up to 224 part of
// an accumulator into registers as packed bf16, releases the accumulator,
// and only then writes Y through shared memory with TMA stores while the
// next tile's MMAs run.
//
// Stages hold 128 logical K: A 128 rows x 64 compressed bytes (64B swizzle),
// two B half-tiles of up to 112 rows x 128 bytes (128B swizzle), metadata
// 128 rows x 16 bytes.  Five stages fit next to the Y staging buffers.
//
// Every wait is bounded (ss_common.cuh); no load multicasts.
#pragma once

#include "ss_common.cuh"
#include "ss_gemm.cuh"

// 1: large channel-row problems take the wide kernel; 0: always gemm_kernel.
#ifndef SS_SPARSE_WIDE
#define SS_SPARSE_WIDE 1
#endif

namespace ss {

constexpr int kWideThreads = 320;  // warp 0 producer, warp 1 MMA, warps 2-9 epilogue
constexpr int kWideBT = 2;         // B tiles per output tile

struct WideCfg {
    static constexpr int kStageK = 128;                   // logical K per stage
    static constexpr int kARowBytes = kStageK / 2;        // 64 compressed bytes
    static constexpr int kABytes = kTileA * kARowBytes;   // 8 KB
    static constexpr int kBnMax = 224;                    // MMA N (B rows of one B tile)
    static constexpr int kBRowsMax = kBnMax / 2;          // B rows per CTA per B tile
    static constexpr int kBTileBytes = kBRowsMax * 128;   // 14 KB
    static constexpr int kEBytes = kTileA * 16;           // 2 KB
    static constexpr int kBOffset = kABytes;
    static constexpr int kEOffset = kBOffset + kWideBT * kBTileBytes;
    static constexpr int kStageBytes = (kEOffset + kEBytes + 1023) / 1024 * 1024;
    static constexpr int kEpiBytes = 32 * kTileA * 2;     // one [32 tokens][128 channels] chunk
    static constexpr int kEpiGroupBytes = 2 * kEpiBytes;  // double buffer per B tile
    static constexpr int kBarBytes = 256;
    static constexpr int kStages =
        (227 * 1024 - 1024 - kBarBytes - 64 - kWideBT * kBnMax * 4 - kWideBT * kEpiGroupBytes) /
        kStageBytes;
    static constexpr int kEpiOffset = kStages * kStageBytes;
    static constexpr int kBarOffset = kEpiOffset + kWideBT * kEpiGroupBytes;
    static constexpr int kSbOffset = kBarOffset + kBarBytes;   // token scales of a tile
    static constexpr int kSbBytes = kWideBT * kBnMax * 4;
    static constexpr int kSmemBytes = kSbOffset + kSbBytes + 1024;
    static constexpr int kAccStride = kBnMax;             // TMEM columns per accumulator
    static constexpr int kECol = kWideBT * kBnMax;        // metadata: 4 columns per stage
    static_assert(kECol + 4 * kStages <= kTmemCols, "TMEM budget");
    static_assert(kStages >= 4, "pipeline depth");
    static_assert(kSmemBytes + 1024 <= 227 * 1024, "shared memory budget (with static)");
    static_assert(kBOffset % 1024 == 0 && kBTileBytes % 1024 == 0 && kEOffset % 16 == 0,
                  "stage alignment");
};

// Tile of pair `unit` in wave k.  Waves alternate direction, so the short
// tiles at the end of the list (the last, partial token tile of every channel
// tile) go to the pairs that took fewer full tiles in the wave before.
__device__ __forceinline__ int snake_tile(int k, int unit, int n_units) {
    return k * n_units + ((k & 1) ? (n_units - 1 - unit) : unit);
}

// kAIsW: A rows are output channels (weight-sparse, Y[b, a]); otherwise A
// rows are tokens (activation-sparse, Y[a, b]).
template <bool kInt8, bool kAIsW>
__global__ void __launch_bounds__(kWideThreads, 1)
    gemm_sparse_wide_kernel(const __grid_constant__ CUtensorMap tm_a,
                            const __grid_constant__ CUtensorMap tm_b,
                            const __grid_constant__ CUtensorMap tm_e,
                            const __grid_constant__ CUtensorMap tm_y, const GemmArgs args) {
    using C = WideCfg;
    extern __shared__ __align__(1024) uint8_t smem_dyn[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kBarOffset);
    uint64_t* empty = full + C::kStages;
    uint64_t* acc_full = empty + C::kStages;
    uint64_t* acc_empty = acc_full + 1;
    uint64_t* drain = acc_empty + 1;
    uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(drain + 1);
    __shared__ int abort_flag_storage;
    volatile int* abort_flag = &abort_flag_storage;
    pdl_trigger();

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    constexpr int kPairRows = 2 * kTileA;  // A rows of one output tile
    const int b_rows_cta = args.bn / 2;
    const int tile_b_rows = kWideBT * args.bn;
    const int nA = (args.rowsA + kPairRows - 1) / kPairRows;
    const int nB = (args.rowsB + tile_b_rows - 1) / tile_b_rows;
    const int n_tiles = nA * nB;
    const int unit = blockIdx.x / 2;
    const int n_units = gridDim.x / 2;

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(acc_full, 1);
        mbar_init(acc_empty, 8 * 2);  // 8 epilogue warps in each CTA of the pair
        mbar_init(drain, 1);
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc_g<2>(tmem_base_slot, kTmemCols);
        tmem_relinquish_g<2>();
    }
    tc_fence_before();
    cluster_sync_all();  // peer barriers initialised before any remote use
    tc_fence_after();
    const uint32_t tmem_base = *tmem_base_slot;
    // Every access to global memory waits for the previous kernel on the
    // stream (programmatic dependent launch); only the producer's L2
    // prefetches of the weight go first.
    if (warp != 0) pdl_wait();

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (elect_one()) {
            tma_prefetch_desc(&tm_a);
            tma_prefetch_desc(&tm_b);
            tma_prefetch_desc(&tm_e);
            const int t0 = snake_tile(0, unit, n_units);
            if (kAIsW && t0 < n_tiles) {  // the weight's first tile into L2
                int ta0, tb0;
                tile_coords(t0, nA, nB, args.a_groups, ta0, tb0);
                const int a0 = ta0 * kPairRows + static_cast<int>(rank) * kTileA;
                const int n_pre = args.k_stages < 2 * kL2PrefetchStages ? args.k_stages
                                                                        : 2 * kL2PrefetchStages;
                for (int kb = 0; kb < n_pre; ++kb) {
                    tma_prefetch_l2_2d(&tm_a, kb * C::kARowBytes, a0);
                    tma_prefetch_l2_2d(&tm_e, 0, ((a0 >> 7) * args.e_chunks + kb) * 16);
                }
            }
        }
        __syncwarp();
        pdl_wait();
        const uint32_t tx = 2 * (C::kABytes + C::kEBytes + kWideBT * b_rows_cta * 128);
        int s = 0;
        uint32_t ph = 0, armed = 0, armed_par = 0;
        bool ok = true;
        const int skip_kb = g_skip_stage;  // test hook, -1 in normal use
        for (int k = 0, t = snake_tile(0, unit, n_units); t < n_tiles && ok;
             ++k, t = snake_tile(k, unit, n_units)) {
            int ta, tb;
            tile_coords(t, nA, nB, args.a_groups, ta, tb);
            const int a0 = ta * kPairRows + static_cast<int>(rank) * kTileA;
            const int b0 = tb * tile_b_rows + static_cast<int>(rank) * b_rows_cta;
            for (int kb = 0; kb < args.k_stages; ++kb) {
                if (k == 0 && kb == skip_kb) {  // this stage is never loaded
                    ok = false;
                    break;
                }
                if (!__all_sync(0xffffffffu, mbar_wait(&empty[s], ph ^ 1u, abort_flag))) {
                    ok = false;
                    break;
                }
                if (elect_one()) {
                    uint8_t* st = smem + s * C::kStageBytes;
                    if (leader) mbar_arrive_expect_tx(&full[s], tx);
                    const uint32_t fb = map_to_rank(&full[s], 0);
                    const uint64_t keep = l2_policy_evict_last();
                    tma_load_2d_pair_hint(st, &tm_a, fb, kb * C::kARowBytes, a0, keep);
#pragma unroll
                    for (int u = 0; u < kWideBT; ++u)
                        tma_load_2d_pair_hint(st + C::kBOffset + u * C::kBTileBytes, &tm_b, fb,
                                              kb * C::kStageK, b0 + u * args.bn, keep);
                    tma_load_2d_pair_hint(st + C::kEOffset, &tm_e, fb, 0,
                                          ((a0 >> 7) * args.e_chunks + kb) * 16, keep);
                }
                __syncwarp();
                armed |= 1u << s;
                armed_par = (armed_par & ~(1u << s)) | (ph << s);
                if (++s == C::kStages) {
                    s = 0;
                    ph ^= 1u;
                }
            }
        }
        if (!ok && lane == 0) {  // let the copies already issued land before exiting
            if (leader) {
                for (int i = 0; i < C::kStages; ++i)
                    if ((armed >> i) & 1u) mbar_drain(&full[i], (armed_par >> i) & 1u);
            } else {  // the peer's copies count on the leader's barriers: wait 1 ms
                const uint64_t t0 = global_timer_ns();
                while (global_timer_ns() - t0 < 1000000ull) {
                }
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // Per stage: copy the metadata into tensor memory, then for each K = 64
        // step one MMA per B tile; the first fills the collector with the A
        // slice, the second uses and releases it.
        if (leader) {
            const uint32_t idesc = make_idesc(true, kInt8, kPairRows, args.bn);
            const uint32_t base = smem_u32(smem);
            const uint64_t a_desc0 = smem_desc(base, 16, 8 * C::kARowBytes, kSwizzle64B);
            const uint64_t b_desc0 = smem_desc(base + C::kBOffset, 16, 1024, kSwizzle128B);
            const uint64_t e_desc0 = smem_desc(base + C::kEOffset, 128 * 16, 128, kSwizzleNone);
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            int i = 0;
            for (int t = snake_tile(0, unit, n_units); t < n_tiles && ok;
                 ++i, t = snake_tile(i, unit, n_units)) {
                if (!__all_sync(0xffffffffu, mbar_wait(acc_empty, (i & 1) ^ 1u, abort_flag))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int kb = 0; kb < args.k_stages; ++kb) {
                    if (!__all_sync(0xffffffffu, mbar_wait(&full[s], ph, abort_flag))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t soff = static_cast<uint64_t>((s * C::kStageBytes) >> 4);
                    // metadata slot = stage index: a slot is rewritten only after
                    // the stage's "empty" commit, i.e. after its MMAs completed
                    const uint32_t e_tmem = tmem_base + C::kECol + 4 * s;
                    if (elect_one()) {
                        tc_cp_128x128b_g<2>(e_tmem, e_desc0 + soff);
#pragma unroll
                        for (int j = 0; j < C::kStageK / 64; ++j) {
                            const uint64_t a_desc = a_desc0 + soff + ((j * 32) >> 4);
                            const uint64_t b0_desc = b_desc0 + soff + ((j * 64) >> 4);
                            const uint64_t b1_desc =
                                b_desc0 + soff + ((C::kBTileBytes + j * 64) >> 4);
                            const uint32_t accum = (kb > 0 || j > 0) ? 1u : 0u;
                            mma_sparse_pair_coll<kInt8, 0>(tmem_base, a_desc, b0_desc,
                                                           e_tmem + 2 * j, idesc, accum);
                            mma_sparse_pair_coll<kInt8, 1>(tmem_base + C::kAccStride, a_desc,
                                                           b1_desc, e_tmem + 2 * j, idesc, accum);
                        }
                        tc_commit_g<2>(&empty[s]);  // stage free in both CTAs
                    }
                    __syncwarp();
                    if (++s == C::kStages) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) break;
                if (elect_one()) tc_commit_g<2>(acc_full);
                __syncwarp();
            }
            if (!ok) {  // wait for every MMA already issued before TMEM is freed
                if (elect_one()) {
                    tc_commit_g<2>(drain);
                    mbar_drain(drain, 0);
                }
                __syncwarp();
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        // Warp w (2..9) drains TMEM lane quarter w % 4 of accumulator (w - 2) / 4,
        // i.e. 32 A rows x up to 224 B rows.  The tile's scales are fetched
        // before its accumulators are ready (B-row scales through shared
        // memory), so the drain itself only reads tensor and shared memory.
        // Phase 1 reads every 32-column chunk, scales, and keeps the packed
        // bf16 pairs in registers; then the accumulator is released.  Phase 2
        // writes each chunk through shared memory with TMA stores while the
        // next tile's MMAs run:
        //   A = weight: m8n8 fragments (tcgen05.ld 16x256b) go through
        //     stmatrix.trans into a 128B-swizzled [32 tokens][64 channels]
        //     pair of halves shared by the four warps of the B tile;
        //   A = activation: each thread's own token row (tcgen05.ld 32x32b)
        //     goes to a [128 tokens][32 channels] box.
        constexpr int kChunks = C::kBnMax / 32;
        const int ew = warp - 2;
        const int et = ew * 32 + lane;  // 0..255
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        const int bt = ew >> 2;  // B tile (accumulator) of this warp
        const bool issuer = (ew & 3) == 0 && lane == 0;
        const uint32_t grp_bar = 2 + static_cast<uint32_t>(bt);
        const uint32_t acc_empty_leader = map_to_rank(acc_empty, 0);
        uint8_t* stage_y = smem + C::kEpiOffset + bt * C::kEpiGroupBytes;
        float* sb_smem = reinterpret_cast<float*>(smem + C::kSbOffset);
        const int t4 = lane >> 2, tm = lane & 3;
        const int mi = lane >> 3, mj = lane & 7;  // this thread's stmatrix matrix / row
        int i = 0;
        uint32_t chunk_iter = 0;
        for (int t = snake_tile(0, unit, n_units); t < n_tiles;
             ++i, t = snake_tile(i, unit, n_units)) {
            int ta, tb_;
            tile_coords(t, nA, nB, args.a_groups, ta, tb_);
            const int a_cta0 = ta * kPairRows + static_cast<int>(rank) * kTileA;
            const int tile_tok0 = tb_ * tile_b_rows;
            const int tok0 = tile_tok0 + bt * args.bn;
            // scales of this tile, fetched while its MMAs still run
            float sb_pre[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int j = et + 256 * u;
                const int tok = tile_tok0 + j;
                sb_pre[u] = (j < tile_b_rows && tok < args.rowsB) ? __ldg(args.s_b + tok) : 0.0f;
            }
            // A-row scales: channel-row path, the m8n8 fragment rows of this
            // thread; token-row path, this thread's own row
            float sa2[2][2];
            float sa_row = 0.0f;
            if constexpr (kAIsW) {
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int ch = a_cta0 + q * 32 + 16 * h + t4 + 8 * e;
                        sa2[h][e] = ch < args.rowsA ? __ldg(args.s_a + ch) : 0.0f;
                    }
            } else {
                const int ar = a_cta0 + q * 32 + lane;
                sa_row = ar < args.rowsA ? __ldg(args.s_a + ar) : 0.0f;
            }
            // all eight epilogue warps take the same decision, so none is left
            // behind at a named barrier if the wait gives up; passing it also
            // means every warp is done with the previous tile's token scales
            const bool got = mbar_wait(acc_full, static_cast<uint32_t>(i & 1), abort_flag);
            if (!named_bar_and(1, 256, got)) break;
#pragma unroll
            for (int u = 0; u < 2; ++u)
                if (et + 256 * u < kWideBT * C::kBnMax) sb_smem[et + 256 * u] = sb_pre[u];
            named_bar_sync(1, 256);
            tc_fence_after();
            const float* sb_tile = sb_smem + bt * args.bn;
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                   static_cast<uint32_t>(bt * C::kAccStride);
            uint32_t pk[kChunks][2][8];  // 16 packed bf16 pairs per chunk
            if constexpr (kAIsW) {
                // [chunk][half][token group r * 2 + channel block]
#pragma unroll
                for (int c = 0; c < kChunks; ++c) {
                    if (c * 32 < args.bn) {
                        uint32_t v[2][16];
                        tmem_ld_16x256b_x4(t_row + c * 32, v[0]);
                        tmem_ld_16x256b_x4(t_row + (16u << 16) + c * 32, v[1]);
                        // token scales of the chunk: tokens 8r + 2tm + {0, 1}
                        float2 sb[4];
#pragma unroll
                        for (int r = 0; r < 4; ++r)
                            sb[r] =
                                *reinterpret_cast<const float2*>(sb_tile + c * 32 + 8 * r + 2 * tm);
                        tmem_ld_wait();
#pragma unroll
                        for (int h = 0; h < 2; ++h)
#pragma unroll
                            for (int r = 0; r < 4; ++r)
#pragma unroll
                                for (int e = 0; e < 2; ++e) {
                                    const uint32_t b0 = v[h][4 * r + 2 * e];
                                    const uint32_t b1 = v[h][4 * r + 2 * e + 1];
                                    const float x0 = kInt8 ? __int2float_rn(static_cast<int32_t>(b0))
                                                           : __uint_as_float(b0);
                                    const float x1 = kInt8 ? __int2float_rn(static_cast<int32_t>(b1))
                                                           : __uint_as_float(b1);
                                    // ((acc * s_b) * s_a), both products rounded to fp32
                                    float y0, y1;
                                    mul_rn_f32x2(x0, x1, sb[r].x, sb[r].y, y0, y1);
                                    mul_rn_f32x2(y0, y1, sa2[h][e], sa2[h][e], y0, y1);
                                    const __nv_bfloat162 b2 = __floats2bfloat162_rn(y0, y1);
                                    pk[c][h][2 * r + e] = *reinterpret_cast<const uint32_t*>(&b2);
                                }
                    }
                }
            } else {
                // this thread's token row, 32 channels per chunk: [chunk][k / 8][k % 8]
#pragma unroll
                for (int c = 0; c < kChunks; ++c) {
                    if (c * 32 < args.bn) {
                        uint32_t r[32];
                        tmem_ld_32x32b_x32(t_row + c * 32, r);
                        float4 sb[8];  // channel scales of the chunk
#pragma unroll
                        for (int k = 0; k < 8; ++k)
                            sb[k] = *reinterpret_cast<const float4*>(sb_tile + c * 32 + 4 * k);
                        tmem_ld_wait();
#pragma unroll
                        for (int k = 0; k < 16; ++k) {
                            const float x0 = kInt8 ? __int2float_rn(static_cast<int32_t>(r[2 * k]))
                                                   : __uint_as_float(r[2 * k]);
                            const float x1 = kInt8 ? __int2float_rn(static_cast<int32_t>(r[2 * k + 1]))
                                                   : __uint_as_float(r[2 * k + 1]);
                            const float s0 = (k & 1) ? sb[k >> 1].z : sb[k >> 1].x;
                            const float s1 = (k & 1) ? sb[k >> 1].w : sb[k >> 1].y;
                            // ((acc * s_a) * s_b), both products rounded to fp32
                            float y0, y1;
                            mul_rn_f32x2(x0, x1, sa_row, sa_row, y0, y1);
                            mul_rn_f32x2(y0, y1, s0, s1, y0, y1);
                            const __nv_bfloat162 b2 = __floats2bfloat162_rn(y0, y1);
                            pk[c][k >> 3][k & 7] = *reinterpret_cast<const uint32_t*>(&b2);
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(acc_empty_leader);  // accumulator drained
#pragma unroll
            for (int c = 0; c < kChunks; ++c) {
                if (c * 32 < args.bn) {
                    uint8_t* sy = stage_y + (chunk_iter & 1) * C::kEpiBytes;
                    if (issuer) bulk_wait_read<1>();  // the stores of two chunks ago have read it
                    named_bar_sync(grp_bar, 128);
                    const uint32_t sy_u32 = smem_u32(sy);
                    if constexpr (kAIsW) {
#pragma unroll
                        for (int h = 0; h < 2; ++h)
#pragma unroll
                            for (int rp = 0; rp < 2; ++rp) {
                                // matrices: (r = 2rp, e = 0), (2rp, 1), (2rp+1, 0), (2rp+1, 1)
                                const int r = 2 * rp + (mi >> 1);
                                const int e = mi & 1;
                                const int tok = 8 * r + mj;              // row of the chunk
                                const int ch = q * 32 + 16 * h + 8 * e;  // 8-channel block
                                const int half = ch >> 6;
                                const int blk = (ch & 63) >> 3;
                                const uint32_t addr = sy_u32 + half * (32 * 128) + tok * 128 +
                                                      ((blk ^ (tok & 7)) << 4);
                                stmatrix_x4_trans(addr, pk[c][h][4 * rp + 0], pk[c][h][4 * rp + 1],
                                                  pk[c][h][4 * rp + 2], pk[c][h][4 * rp + 3]);
                            }
                    } else {
                        // [128 token rows][32 channels]: this thread's row is 64 bytes
                        uint4* dst = reinterpret_cast<uint4*>(sy + (q * 32 + lane) * 64);
#pragma unroll
                        for (int w = 0; w < 4; ++w)
                            dst[w] = make_uint4(pk[c][w >> 1][4 * (w & 1)], pk[c][w >> 1][4 * (w & 1) + 1],
                                                pk[c][w >> 1][4 * (w & 1) + 2],
                                                pk[c][w >> 1][4 * (w & 1) + 3]);
                    }
                    fence_async_shared();
                    named_bar_sync(grp_bar, 128);
                    if (issuer) {
                        const uint64_t stream = l2_policy_evict_first();
                        if constexpr (kAIsW) {
                            tma_store_2d_hint(&tm_y, sy, a_cta0, tok0 + c * 32, stream);
                            tma_store_2d_hint(&tm_y, sy + 32 * 128, a_cta0 + 64, tok0 + c * 32,
                                              stream);
                        } else {
                            tma_store_2d_hint(&tm_y, sy, tok0 + c * 32, a_cta0, stream);
                        }
                        bulk_commit_group();
                    }
                    ++chunk_iter;
                }
            }
        }
        if (issuer) bulk_wait_all();  // Y stores done reading shared memory
    }

    __syncwarp();
    tc_fence_before();
    cluster_sync_all();  // both CTAs done with barriers and tensor memory
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_g<2>(tmem_base, kTmemCols);
    }
}

}  // namespace ss
