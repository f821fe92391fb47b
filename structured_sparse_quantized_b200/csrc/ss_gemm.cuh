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
// kPair = 2 (problems with more than 128 A rows): a cluster of two CTAs on
// two SMs issues MMAs of M = 256 (tcgen05 cta_group::2).  Each CTA loads its
// own 128 A rows and its own half of the B rows into its own shared memory;
// the pair reads each B half once for both tensor cores, which is what lets
// the sparse MMA run at twice the dense rate.  D is split by A rows between
// the two tensor memories.  kPair = 1 is the single-SM form (M = 128).
//
// The accumulator is double-buffered in tensor memory: the epilogue drains
// one tile while the MMAs of the next fill the other buffer.  (For large
// problems the sparse GEMM also has a two-B-tile shape, ss_gemm_wide.cuh.)
//
// CTA = 10 warps, one CTA per SM, persistent over output tiles:
//   warp 0       TMA producer (whole warp, one elected lane issues): A tiles,
//                B atoms and, for the sparse variant, the 128 x 16-byte
//                metadata chunks of each K stage, into a ring of shared-memory
//                stages.  Both CTAs of a pair count their bytes on the leader
//                CTA's "full" barrier.
//   warp 1       allocates 512 TMEM columns (both CTAs); in the leader CTA the
//                whole warp runs the MMA loop and one elected lane issues the
//                metadata copies into tensor memory, the MMAs, and the commits
//                that release stages / accumulators in both CTAs.
//   warps 2-9    epilogue, two groups of four taking alternate 32-column
//                chunks: tcgen05.ld the accumulator (lane = A row, column =
//                B row), scale, convert, stage the chunk in the group's
//                shared-memory buffer and write it with one TMA tensor store;
//                release the accumulator on the leader's barrier.
// Every wait is bounded (ss_common.cuh); no load multicasts.
#pragma once

#include <type_traits>

#include "ss_common.cuh"

namespace ss {

constexpr int kGemmEpiWarps = 8;  // two groups of four, one warp per TMEM lane quarter each
constexpr int kGemmThreads = 64 + 32 * kGemmEpiWarps;
constexpr int kL2PrefetchStages = 16;  // weight stages a CTA prefetches before pdl_wait
constexpr int kTileA = 128;  // A rows per CTA per A tile
constexpr int kTmemCols = 512;

template <bool kSparse, int kPair, int kEb = 1>
struct GemmCfg {
    // One pipeline stage covers kStageK logical K: for 8-bit operands dense
    // 128 (4 MMAs of K=32) and sparse 256 (4 MMAs of K=64); for bf16 (kEb = 2
    // bytes) half of that, 4 MMAs of K=16 / K=32.  Either way an A row holds
    // 128 bytes of the stage (128B swizzle) and each MMA reads 32 bytes of an
    // A row and 32 (dense) or 64 (sparse) bytes of a B row.  (Stages of half
    // the K, with 64-byte A rows, measured slower: twice the handshakes per
    // byte cost more than the deeper ring gains.)
    static constexpr int kStageK = (kSparse ? 256 : 128) / kEb;
    static constexpr int kMmaK = (kSparse ? 64 : 32) / kEb;
    static constexpr int kMmaPerStage = kStageK / kMmaK;
    static constexpr int kARowBytes = kSparse ? kStageK * kEb / 2 : kStageK * kEb;  // 128
    static constexpr int kABytes = kTileA * kARowBytes;    // one A tile, 16 KB
    static constexpr int kBAtoms = kStageK * kEb / 128;    // 128-byte K atoms of B per stage
    // Metadata of a sparse MMA is addressed in tensor memory as aligned pairs
    // of 32-bit columns: an 8-bit MMA (K=64, 64 selector bits per row) uses a
    // whole pair, a bf16 MMA (K=32, 32 bits) one column of it, picked by the
    // sparsity selector of the instruction descriptor (bits 0-1).
    static constexpr int kBnMax = kSparse ? 224 : 256;     // MMA N; accumulators + metadata
    static constexpr int kBRowsMax = kBnMax / kPair;       // B rows held per CTA
    static constexpr int kBAtomBytes = kBRowsMax * 128;
    static constexpr int kBBytes = kBAtoms * kBAtomBytes;
    static constexpr int kEChunks = kSparse ? kStageK / 128 : 0;  // 16-byte chunks per A row
    static constexpr int kEBytes = kEChunks * kTileA * 16;  // one A tile
    // stage layout: [A tile | B atoms | E chunks]
    static constexpr int kBOffset = kABytes;
    static constexpr int kEOffset = kBOffset + kBBytes;
    static constexpr int kStageRaw = kEOffset + kEBytes;
    static constexpr int kStageBytes = (kStageRaw + 1023) / 1024 * 1024;
    static constexpr int kEpiBytes = 32 * kTileA * 2;      // one 32-column bf16 chunk of Y
    static constexpr int kSmemBudget = 225 * 1024 - 1024 - 256 - 2 * kEpiBytes;
    static constexpr int kStagesRaw = kSmemBudget / kStageBytes;
    static constexpr int kStages = kStagesRaw > 8 ? 8 : kStagesRaw;
    static constexpr int kAccBufs = 2;                     // accumulators in TMEM
    static constexpr int kSfStageBytes = 0;                // no block scales
    static constexpr int kAccStride = kBnMax;              // TMEM columns between accumulators
    static constexpr int kECol = 2 * kBnMax;               // metadata columns (sparse)
    static constexpr int kESlotCols = 4 * kEChunks;        // columns one stage's metadata takes
    // one metadata slot per stage: a slot is rewritten only after its stage's
    // "empty" commit, i.e. after the MMAs that read it completed
    static constexpr int kESlots = kStages;
    static constexpr int kEpiOffset = kStages * kStageBytes;  // 2 staging buffers for Y chunks
    static constexpr int kSmemBytes =
        kEpiOffset + 2 * kEpiBytes + 1024 /*align*/ + 256 /*barriers*/;
    static_assert(kABytes % 1024 == 0 && kBAtomBytes % 1024 == 0, "tile alignment");
    static_assert(kARowBytes == 128 && kMmaPerStage == 4, "stage geometry");
    static_assert(!kSparse || kECol + kESlots * kESlotCols <= kTmemCols, "TMEM budget");
    static_assert(kECol % 2 == 0 && kESlotCols % 2 == 0, "metadata column pairs stay aligned");
    static_assert(kSmemBytes <= 227 * 1024, "shared memory budget");
    static_assert(kStages >= (kPair == 2 ? 3 : 2), "pipeline depth");
    static_assert((2 * kStages + 5) * 8 + 4 <= 256, "barrier area");
};

// Stage layout of the block-scaled FP4 GEMM: per stage 4 MMAs (sparse: K =
// 128 lifted each, dense: K = 64), A 128 rows x 128 B, this CTA's B rows x
// 256 B (sparse) / 128 B (dense), sparse metadata 2 x 2 KB, the scale factors
// of A (512 B per MMA) and those of the whole B tile (512 B per MMA and
// 128-row scale tile).
//   single SM: MMA M = 128, N = 128; two 128-column accumulators in tensor
//     memory (the epilogue drains one while the next tile fills the other).
//   CTA pair:  MMA M = 256, N = 256 (128 B rows per CTA, two scale tiles);
//     one 256-column accumulator.  An FP4 MMA of N = 128 runs at about half
//     the rate of one of N = 256, so the pair takes the wide N and gives up
//     the second accumulator (the epilogue releases it as soon as it has
//     read it into registers).
// After the accumulators, tensor memory holds per stage a metadata slot (8
// columns, sparse) and a scale slot (4 columns per MMA for A, 4 per MMA and
// scale tile for B).
template <bool kSparse, int kPair = 1>
struct Fp4Cfg {
    static constexpr int kStageK = kSparse ? 512 : 256;
    static constexpr int kMmaK = kSparse ? 128 : 64;
    static constexpr int kMmaPerStage = kStageK / kMmaK;
    static constexpr int kARowBytes = 128;
    static constexpr int kABytes = kTileA * kARowBytes;
    static constexpr int kBAtoms = kSparse ? 2 : 1;
    static constexpr int kBnMax = 128 * kPair;
    static constexpr int kSfbTiles = kBnMax / 128;  // 128-row scale tiles per B tile
    static constexpr int kAccBufs = kPair == 2 ? 1 : 2;
    static constexpr int kBRowsMax = kBnMax / kPair;
    static constexpr int kBAtomBytes = kBRowsMax * 128;
    static constexpr int kBBytes = kBAtoms * kBAtomBytes;
    static constexpr int kEChunks = kSparse ? 2 : 0;
    static constexpr int kEBytes = kEChunks * kTileA * 16;
    static constexpr int kSfaBytes = kMmaPerStage * 512;   // A scales of a stage
    static constexpr int kSfbTileBytes = kMmaPerStage * 512;  // per 128-row scale tile
    static constexpr int kSfbBytes = kSfbTiles * kSfbTileBytes;  // B scales of a stage
    static constexpr int kSfStageBytes = kSfaBytes + kSfbBytes;
    static constexpr int kBOffset = kABytes;
    static constexpr int kEOffset = kBOffset + kBBytes;
    static constexpr int kSfaOffset = kEOffset + kEBytes;
    static constexpr int kSfbOffset = kSfaOffset + kSfaBytes;
    static constexpr int kStageBytes = (kSfbOffset + kSfbBytes + 1023) / 1024 * 1024;
    static constexpr int kEpiBytes = 32 * kTileA * 2;
    static constexpr int kSmemBudget = 225 * 1024 - 1024 - 256 - 2 * kEpiBytes;
    static constexpr int kStagesRaw = kSmemBudget / kStageBytes;
    static constexpr int kESlotCols = 4 * kEChunks;
    static constexpr int kSfaCols = 4 * kMmaPerStage;
    static constexpr int kSfbCols = 4 * kMmaPerStage * kSfbTiles;
    static constexpr int kSfSlotCols = kSfaCols + kSfbCols;
    static constexpr int kStagesTmem =
        (kTmemCols - kAccBufs * kBnMax) / (kESlotCols + kSfSlotCols);
    static constexpr int kStagesMin = kStagesRaw < kStagesTmem ? kStagesRaw : kStagesTmem;
    static constexpr int kStages = kStagesMin > 8 ? 8 : kStagesMin;
    static constexpr int kAccStride = kBnMax;
    static constexpr int kECol = kAccBufs * kBnMax;
    static constexpr int kESlots = kStages;
    static constexpr int kSfCol = kECol + kStages * kESlotCols;  // scale slots
    static constexpr int kEpiOffset = kStages * kStageBytes;
    static constexpr int kSmemBytes = kEpiOffset + 2 * kEpiBytes + 1024 + 256;
    static_assert(kSfCol % 4 == 0 && kSfCol + kSfSlotCols * kStages <= kTmemCols, "TMEM budget");
    static_assert(kSmemBytes <= 227 * 1024 && kStages >= 3, "shared memory budget");
    static_assert((2 * kStages + 5) * 8 + 4 <= 256, "barrier area");
};

struct GemmArgs {
    int rowsA;        // rows of A
    int rowsB;        // rows of B
    int k_stages;     // ceil(K_lp / kStageK)
    int bn;           // B rows per tile (MMA N; multiple of 32, <= kBnMax)
    int a_is_w;       // 1: A rows are output channels (Y[b, a]); 0: Y[a, b]
    int ldy;          // leading dimension of Y (= N)
    int tma_store;    // 1: Y written by TMA tensor stores through shared memory
                      //    (A rows = channels: 128B-swizzled [32][64] halves)
    int e_chunks;     // K_lp / 128: 2 KB metadata tiles per 128 rows (tile-major)
                      // (block-scaled FP4: K_lp / 256)
    int sf_k;         // FP4: MMA k-blocks per 128-row scale tile (4 scales each)
    int a_groups;     // A tiles are walked in this many groups (tile_coords)
    const float* s_a;
    const float* s_b;
    void* y;
};

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

// Output tile t -> (A tile ta, B tile tb).  Consecutive tiles (the ones a
// wave of CTA pairs works on together) take consecutive A tiles for the same
// B tile(s), so each B tile is read from L2 by many pairs at once.  With
// a_groups > 1 the A tiles are split into that many groups and a group's A
// tiles are walked for every B tile before the next group starts: the slice
// of A that every wave re-reads is 1/a_groups of it, small enough to stay in
// L2 while the B tiles and Y stream through (the host picks a_groups from the
// size of A).
__device__ __forceinline__ void tile_coords(int t, int nA, int nB, int groups, int& ta, int& tb) {
    if (groups <= 1) {
        ta = t % nA;
        tb = t / nA;
        return;
    }
    const int G = (nA + groups - 1) / groups;  // A tiles per group (the last may have fewer)
    const int g = t / (G * nB);
    const int rows = min(G, nA - g * G);
    const int r = t - g * G * nB;
    ta = g * G + r % rows;
    tb = r / rows;
}

// Scale of row i, or 1 for the unscaled bf16 tier (the product with 1.0f
// is exact, so both tiers share the epilogue arithmetic).
template <bool kUnit>
__device__ __forceinline__ float load_scale(const float* s, int i, bool in_range) {
    if constexpr (kUnit) return 1.0f;
    else return in_range ? __ldg(s + i) : 0.0f;
}

// Scale of B row i: per row, 1 for the bf16 tier, or the one global scale
// of the NVFP4 activation tensor.
template <int kQ>
__device__ __forceinline__ float load_b_scale(const float* s, int i, bool in_range) {
    if constexpr (kQ == kQNvfp4) return in_range ? __ldg(s) : 0.0f;
    else return load_scale<kQ == kQBf16>(s, i, in_range);
}

// kQ: kQE4M3, kQInt8 (kind::f8f6f4 / kind::i8), kQBf16 (kind::f16) or kQNvfp4
// (kind::mxf4nvf4, block-scaled; tm_sfa / tm_sfb are its scale-factor maps,
// unused otherwise, and s_a is one global scale).
template <bool kSparse, int kQ, bool kOutBf16, int kPair>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                const __grid_constant__ CUtensorMap tm_e, const __grid_constant__ CUtensorMap tm_y,
                const __grid_constant__ CUtensorMap tm_sfa,
                const __grid_constant__ CUtensorMap tm_sfb, const GemmArgs args) {
    constexpr bool kInt8 = kQ == kQInt8;
    constexpr bool kBf16 = kQ == kQBf16;
    constexpr bool kFp4 = kQ == kQNvfp4;
    using C = std::conditional_t<kFp4, Fp4Cfg<kSparse, kPair>, GemmCfg<kSparse, kPair, kBf16 ? 2 : 1>>;
    extern __shared__ __align__(1024) uint8_t smem_dyn[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_dyn) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::kEpiOffset + 2 * C::kEpiBytes);
    uint64_t* empty = full + C::kStages;
    uint64_t* acc_full = empty + C::kStages;  // [2]: one per accumulator buffer
    uint64_t* acc_empty = acc_full + 2;
    uint64_t* drain = acc_empty + 2;
    uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(drain + 1);
    __shared__ int abort_flag_storage;
    volatile int* abort_flag = &abort_flag_storage;
    pdl_trigger();

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = kPair == 2 ? cluster_ctarank() : 0u;
    const bool leader = rank == 0;
    const int pair_rows = kTileA * kPair;     // A rows one MMA covers
    const int tile_a_rows = pair_rows;        // A rows of one output tile
    const int b_rows_cta = args.bn / kPair;
    const int nA = (args.rowsA + tile_a_rows - 1) / tile_a_rows;
    const int nB = (args.rowsB + args.bn - 1) / args.bn;
    const int n_tiles = nA * nB;
    const int unit = blockIdx.x / kPair;   // cluster index
    const int n_units = gridDim.x / kPair;

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        for (int s = 0; s < C::kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], kGemmEpiWarps * kPair);
        }
        mbar_init(drain, 1);
        fence_barrier_init();
    }
    if (warp == 1) {
        tmem_alloc_g<kPair>(tmem_base_slot, kTmemCols);
        tmem_relinquish_g<kPair>();
    }
    tc_fence_before();
    if constexpr (kPair == 2)
        cluster_sync_all();  // peer barriers initialised before any remote use
    else
        __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_base_slot;
    // Until the previous kernel on the stream has finished, only the weight
    // operand may be touched, and only through L2 prefetches (the producer's,
    // below); every other access waits here.
    if (warp != 0) pdl_wait();

    // The producer and MMA roles run as whole, converged warps: every lane
    // takes the barrier waits (the outcome is made warp-uniform) and one
    // elected lane issues the TMA copies / tensor-core instructions.  A lone
    // diverged lane issuing MMAs stalls on every memory operation and leaves
    // the tensor pipe idle between stages.
    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (elect_one()) {
            tma_prefetch_desc(&tm_a);
            tma_prefetch_desc(&tm_b);
            if (kSparse) tma_prefetch_desc(&tm_e);
            if (args.a_is_w && unit < n_tiles) {
                // A (and its metadata) is the weight: start streaming the first
                // tile's K stages into L2 while the previous kernel finishes.
                int ta0, tb0;
                tile_coords(unit, nA, nB, args.a_groups, ta0, tb0);
                const int a0 = ta0 * tile_a_rows + static_cast<int>(rank) * kTileA;
                const int n_pre = args.k_stages < kL2PrefetchStages ? args.k_stages
                                                                    : kL2PrefetchStages;
                for (int kb = 0; kb < n_pre; ++kb) {
                    tma_prefetch_l2_2d(&tm_a, kb * C::kARowBytes, a0);
#pragma unroll
                    for (int u = 0; u < C::kEChunks; ++u)
                        tma_prefetch_l2_2d(&tm_e, 0,
                                           ((a0 >> 7) * args.e_chunks + kb * C::kEChunks + u) * 16);
                }
            }
        }
        __syncwarp();
        pdl_wait();
        // FP4: each CTA also loads its A scales and the B tile's scales
        const uint32_t tx = kPair * (C::kABytes + C::kEBytes + C::kBAtoms * b_rows_cta * 128 +
                                     C::kSfStageBytes);
        int s = 0;
        uint32_t ph = 0, armed = 0, armed_par = 0;
        bool ok = true;
        const int skip_kb = g_skip_stage;  // test hook, -1 in normal use
        for (int t = unit; t < n_tiles && ok; t += n_units) {
            int ta, tb;
            tile_coords(t, nA, nB, args.a_groups, ta, tb);
            const int a0 = ta * tile_a_rows + static_cast<int>(rank) * kTileA;
            const int b0 = tb * args.bn + static_cast<int>(rank) * b_rows_cta;
            for (int kb = 0; kb < args.k_stages; ++kb) {
                if (t == unit && kb == skip_kb) {  // this stage is never loaded
                    ok = false;
                    break;
                }
                if (!__all_sync(0xffffffffu, mbar_wait(&empty[s], ph ^ 1u, abort_flag))) {
                    ok = false;
                    break;
                }
                if (elect_one()) {
                    uint8_t* st = smem + s * C::kStageBytes;
                    if constexpr (kPair == 2) {
                        if (leader) mbar_arrive_expect_tx(&full[s], tx);
                        const uint32_t fb = map_to_rank(&full[s], 0);
                        const uint64_t keep = l2_policy_evict_last();
                        tma_load_2d_pair_hint(st, &tm_a, fb, kb * C::kARowBytes, a0, keep);
#pragma unroll
                        for (int u = 0; u < C::kBAtoms; ++u)
                            tma_load_2d_pair_hint(st + C::kBOffset + u * C::kBAtomBytes, &tm_b,
                                                  fb, (kb * C::kBAtoms + u) * 128, b0, keep);
#pragma unroll
                        for (int u = 0; u < C::kEChunks; ++u)
                            tma_load_2d_pair_hint(st + C::kEOffset + u * kTileA * 16, &tm_e, fb, 0,
                                                  ((a0 >> 7) * args.e_chunks + kb * C::kEChunks + u) * 16,
                                                  keep);
                        if constexpr (kFp4) {  // this CTA's A scales, the whole B tile's scales
                            tma_load_2d_pair_hint(
                                st + C::kSfaOffset, &tm_sfa, fb, 0,
                                ((a0 >> 7) * args.sf_k + kb * C::kMmaPerStage) * 4, keep);
                            const int sfb_tile = tb * args.bn >> 7;
#pragma unroll
                            for (int u = 0; u < C::kSfbTiles; ++u)  // past the last: zero fill
                                tma_load_2d_pair_hint(
                                    st + C::kSfbOffset + C::kSfbTileBytes * u, &tm_sfb, fb, 0,
                                    ((sfb_tile + u) * args.sf_k + kb * C::kMmaPerStage) * 4, keep);
                        }
                    } else {
                        mbar_arrive_expect_tx(&full[s], tx);
                        tma_load_2d(st, &tm_a, &full[s], kb * C::kARowBytes, a0);
#pragma unroll
                        for (int u = 0; u < C::kBAtoms; ++u)
                            tma_load_2d(st + C::kBOffset + u * C::kBAtomBytes, &tm_b, &full[s],
                                        (kb * C::kBAtoms + u) * 128, b0);
#pragma unroll
                        for (int u = 0; u < C::kEChunks; ++u)
                            tma_load_2d(st + C::kEOffset + u * kTileA * 16, &tm_e, &full[s], 0,
                                        ((a0 >> 7) * args.e_chunks + kb * C::kEChunks + u) * 16);
                        if constexpr (kFp4) {
                            // 4 MMAs' scales of A and of B: 2 KB each, as 16 rows of 128 B
                            tma_load_2d(st + C::kSfaOffset, &tm_sfa, &full[s], 0,
                                        ((a0 >> 7) * args.sf_k + kb * C::kMmaPerStage) * 4);
#pragma unroll
                            for (int u = 0; u < C::kSfbTiles; ++u)
                                tma_load_2d(st + C::kSfbOffset + C::kSfbTileBytes * u, &tm_sfb,
                                            &full[s], 0,
                                            (((b0 >> 7) + u) * args.sf_k + kb * C::kMmaPerStage) * 4);
                        }
                    }
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
            if (kPair == 1 || leader) {
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
        // Descriptors are built once; a stage, A tile or K step only adds its
        // byte offset (>> 4) to the start-address field.
        if (leader) {
            const uint32_t idesc = make_idesc_q(kSparse, kQ, pair_rows, args.bn);
            const uint32_t base = smem_u32(smem);
            const uint64_t a_desc0 = smem_desc(base, 16, 8 * C::kARowBytes, kSwizzle128B);
            const uint64_t b_desc0 = smem_desc(base + C::kBOffset, 16, 1024, kSwizzle128B);
            const uint64_t e_desc0 =
                smem_desc(base + C::kEOffset, 128 * 16, 128, kSwizzleNone);
            const uint64_t sf_desc0 = smem_desc(base, 512, 128, kSwizzleNone);  // + stage offsets
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            int i = 0;
            for (int t = unit; t < n_tiles && ok; t += n_units, ++i) {
                // accumulator buffer of this tile (two: i & 1; one: 0), one
                // phase per use
                const int buf = C::kAccBufs == 2 ? (i & 1) : 0;
                const uint32_t aph = C::kAccBufs == 2 ? ((i >> 1) & 1) : (i & 1);
                if (!__all_sync(0xffffffffu, mbar_wait(&acc_empty[buf], aph ^ 1u, abort_flag))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int kb = 0; kb < args.k_stages && ok; ++kb) {
                    if (!__all_sync(0xffffffffu, mbar_wait(&full[s], ph, abort_flag))) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t soff = static_cast<uint64_t>((s * C::kStageBytes) >> 4);
                    const uint32_t e_tmem =
                        tmem_base + C::kECol + C::kESlotCols * s;
                    const uint32_t d_tmem = tmem_base + buf * C::kAccStride;
                    if (elect_one()) {
                        if constexpr (kFp4) {
                            // scale slot: A's 4 columns per MMA, then B's 4
                            // per MMA and 128-row scale tile
                            const uint32_t sf_tmem = tmem_base + C::kSfCol + C::kSfSlotCols * s;
                            const uint32_t sfb_tmem = sf_tmem + C::kSfaCols;
#pragma unroll
                            for (int t = 0; t < C::kMmaPerStage; ++t) {
                                tc_cp_32x128b_warpx4_g<kPair>(
                                    sf_tmem + 4 * t, sf_desc0 + soff + ((C::kSfaOffset + 512 * t) >> 4));
#pragma unroll
                                for (int u = 0; u < C::kSfbTiles; ++u)
                                    tc_cp_32x128b_warpx4_g<kPair>(
                                        sfb_tmem + 4 * (C::kSfbTiles * t + u),
                                        sf_desc0 + soff +
                                            ((C::kSfbOffset + C::kSfbTileBytes * u + 512 * t) >> 4));
                            }
                            if constexpr (kSparse) {
#pragma unroll
                                for (int u = 0; u < C::kEChunks; ++u)
                                    tc_cp_128x128b_g<kPair>(e_tmem + 4 * u,
                                                            e_desc0 + soff + ((u * kTileA * 16) >> 4));
                            }
#pragma unroll
                            for (int j = 0; j < C::kMmaPerStage; ++j) {
                                const uint64_t a_desc = a_desc0 + soff + ((j * 32) >> 4);
                                const uint32_t accum = (kb > 0 || j > 0) ? 1u : 0u;
                                if constexpr (kSparse) {
                                    const uint64_t b_desc =
                                        b_desc0 + soff +
                                        (((j >> 1) * C::kBAtomBytes + (j & 1) * 64) >> 4);
                                    mma_fp4_sparse_g<kPair>(d_tmem, a_desc, b_desc, e_tmem + 2 * j,
                                                            idesc, sf_tmem + 4 * j,
                                                            sfb_tmem + 4 * C::kSfbTiles * j, accum);
                                } else {
                                    const uint64_t b_desc = b_desc0 + soff + ((j * 32) >> 4);
                                    mma_fp4_g<kPair>(d_tmem, a_desc, b_desc, idesc, sf_tmem + 4 * j,
                                                     sfb_tmem + 4 * C::kSfbTiles * j, accum);
                                }
                            }
                        } else if constexpr (kSparse) {
#pragma unroll
                            for (int u = 0; u < C::kEChunks; ++u)
                                tc_cp_128x128b_g<kPair>(e_tmem + 4 * u,
                                                        e_desc0 + soff + ((u * kTileA * 16) >> 4));
#pragma unroll
                            for (int j = 0; j < C::kMmaPerStage; ++j) {
                                const uint64_t a_desc = a_desc0 + soff + ((j * 32) >> 4);
                                const uint64_t b_desc =
                                    b_desc0 + soff +
                                    (((j >> 1) * C::kBAtomBytes + (j & 1) * 64) >> 4);
                                const uint32_t accum = (kb > 0 || j > 0) ? 1u : 0u;
                                if constexpr (kBf16)  // 32 selector bits: half j & 1 of a pair
                                    mma_sparse_bf16_g<kPair>(d_tmem, a_desc, b_desc,
                                                             e_tmem + 2 * (j >> 1),
                                                             idesc | static_cast<uint32_t>(j & 1),
                                                             accum);
                                else
                                    mma_sparse_g<kPair, kInt8>(d_tmem, a_desc, b_desc,
                                                               e_tmem + 2 * j, idesc, accum);
                            }
                        } else {
#pragma unroll
                            for (int j = 0; j < C::kMmaPerStage; ++j) {
                                const uint64_t a_desc = a_desc0 + soff + ((j * 32) >> 4);
                                const uint64_t b_desc = b_desc0 + soff + ((j * 32) >> 4);
                                const uint32_t accum = (kb > 0 || j > 0) ? 1u : 0u;
                                if constexpr (kBf16)
                                    mma_dense_bf16_g<kPair>(d_tmem, a_desc, b_desc, idesc, accum);
                                else
                                    mma_dense_g<kPair, kInt8>(d_tmem, a_desc, b_desc, idesc,
                                                              accum);
                            }
                        }
                    }
                    __syncwarp();
                    if (!ok) break;
                    if (elect_one()) tc_commit_g<kPair>(&empty[s]);  // stage free in both CTAs
                    __syncwarp();
                    if (++s == C::kStages) {
                        s = 0;
                        ph ^= 1u;
                    }
                }
                if (!ok) break;
                if (elect_one()) tc_commit_g<kPair>(&acc_full[buf]);
                __syncwarp();
            }
            if (!ok) {  // wait for every MMA already issued before TMEM is freed
                if (elect_one()) {
                    tc_commit_g<kPair>(drain);
                    mbar_drain(drain, 0);
                }
                __syncwarp();
            }
        }
    } else {
        // ------------------------------------------------------------ epilogue
        // Two groups of four warps (one warp per TMEM lane quarter in each);
        // group g takes the 32-column chunks g, g + 2, ... of an accumulator.
        // A chunk is scaled, converted and written to the group's own
        // shared-memory staging buffer, laid out as the chunk's box of Y, then
        // stored by one TMA tensor store (clipped at the edges of Y).  The two
        // groups' load / convert / store latencies overlap, which is what
        // keeps the epilogue shorter than the MMAs of a tile when K is short.
        // Without TMA stores (fp32 Y, or Y rows not 16-byte aligned) the
        // values go straight to global memory.
        const int ew = warp - 2;
        const int grp = ew >> 2;  // chunk parity of this group
        const uint32_t grp_bar = 1 + static_cast<uint32_t>(grp);
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        const int lane_row = q * 32 + lane;
        const bool issuer = (ew & 3) == 0 && lane == 0;
        const uint32_t acc_empty_leader = kPair == 2 ? map_to_rank(acc_empty, 0) : 0u;
        constexpr int kEsz = 2;  // TMA-store staging is used for bf16 output only
        uint8_t* sy = smem + C::kEpiOffset + grp * C::kEpiBytes;
        int i = 0;
        bool ok = true;
        for (int t = unit; t < n_tiles && ok; t += n_units, ++i) {
            int ta, tb;
            tile_coords(t, nA, nB, args.a_groups, ta, tb);
            const int a_tile0 = ta * tile_a_rows + static_cast<int>(rank) * kTileA;
            const int b0 = tb * args.bn;
            const int acc = C::kAccBufs == 2 ? (i & 1) : 0;
            const uint32_t aph = C::kAccBufs == 2 ? ((i >> 1) & 1) : (i & 1);
            // the four warps of a group take the same decision, so none is
            // left behind at the group's named barrier if the wait gives up
            const bool got = mbar_wait(&acc_full[acc], aph, abort_flag);
            if (!named_bar_and(grp_bar, 128, got)) {
                ok = false;
                break;
            }
            tc_fence_after();
            if (32 * grp >= args.bn) {  // no chunk for this group (bn = 32)
                __syncwarp();
                if (lane == 0) {
                    if constexpr (kPair == 2)
                        mbar_arrive_cluster(acc_empty_leader + acc * sizeof(uint64_t));
                    else
                        mbar_arrive(&acc_empty[acc]);
                }
                continue;
            }
            const int a_cta0 = a_tile0;
            const int a_row = a_cta0 + lane_row;
            const bool row_ok = a_row < args.rowsA;
            const float sa = kFp4 ? __ldg(args.s_a) : load_scale<kBf16>(args.s_a, a_row, row_ok);
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                   static_cast<uint32_t>(acc * C::kAccStride);
            if (args.tma_store && args.a_is_w) {
                // Transposed store path.  Each warp reads its 32 channels x 32
                // tokens of a chunk as m8n8 fragments (two 16-lane halves),
                // scales them, packs bf16 pairs and writes 8x8 blocks with
                // stmatrix.trans into [token][channel] staging, 128B-swizzled
                // in two 64-channel halves, stored by two TMA stores.
                const int t4 = lane >> 2, tm = lane & 3;
                float sa2[2][2];
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int ch = a_cta0 + q * 32 + 16 * h + t4 + 8 * e;
                        sa2[h][e] = kFp4 ? __ldg(args.s_a)
                                         : load_scale<kBf16>(args.s_a, ch, ch < args.rowsA);
                    }
                // this thread's stmatrix row: matrix mi, row mj
                const int mi = lane >> 3, mj = lane & 7;
                // Chunks go through registers in batches: with two accumulators
                // one chunk at a time (its stores overlap the next chunk's
                // reads); with one accumulator the whole group's part is read
                // first, so that it is released before any store is waited for.
                constexpr int kCpg = (C::kBnMax + 63) / 64;  // chunks per group, at most
                constexpr int kBatch = C::kAccBufs == 1 ? kCpg : 1;
#pragma unroll
                for (int cb = 0; cb < kCpg; cb += kBatch) {
                    // 1) the batch's chunks into registers as packed bf16
                    //    ([chunk][half][column group r * 2 + channel block]):
                    //    every tensor-memory read of the batch is issued first and
                    //    waited for once; with one accumulator it is released right
                    //    then (2), before the conversion, so the next tile's MMAs
                    //    need not wait for it
                    uint32_t pk[kBatch][2][8];
                    uint32_t v[kBatch][2][16];
#pragma unroll
                    for (int cc = 0; cc < kBatch; ++cc) {
                        const int c = 32 * grp + 64 * (cb + cc);
                        if (c < args.bn) {
                            tmem_ld_16x256b_x4(t_row + c, v[cc][0]);
                            tmem_ld_16x256b_x4(t_row + (16u << 16) + c, v[cc][1]);
                        }
                    }
                    tmem_ld_wait();
                    // 2) after the group's last read of the accumulator: release its part
                    if (32 * grp + 64 * (cb + kBatch) >= args.bn &&
                        32 * grp + 64 * cb < args.bn) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) {
                            if constexpr (kPair == 2)
                                mbar_arrive_cluster(acc_empty_leader + acc * sizeof(uint64_t));
                            else
                                mbar_arrive(&acc_empty[acc]);
                        }
                    }
#pragma unroll
                    for (int cc = 0; cc < kBatch; ++cc) {
                        const int c = 32 * grp + 64 * (cb + cc);
                        if (c < args.bn) {
                            float sb[4][2];  // the chunk's token scales
#pragma unroll
                            for (int r = 0; r < 4; ++r)
#pragma unroll
                                for (int e = 0; e < 2; ++e) {
                                    const int tok = b0 + c + 8 * r + 2 * tm + e;
                                    sb[r][e] = load_b_scale<kQ>(args.s_b, tok, tok < args.rowsB);
                                }
#pragma unroll
                            for (int h = 0; h < 2; ++h)
#pragma unroll
                                for (int r = 0; r < 4; ++r)
#pragma unroll
                                    for (int e = 0; e < 2; ++e) {
                                        float y2[2];
#pragma unroll
                                        for (int k = 0; k < 2; ++k) {
                                            const uint32_t bits = v[cc][h][4 * r + 2 * e + k];
                                            const float accv =
                                                kInt8 ? __int2float_rn(static_cast<int32_t>(bits))
                                                      : __uint_as_float(bits);
                                            y2[k] = __fmul_rn(__fmul_rn(accv, sb[r][k]), sa2[h][e]);
                                        }
                                        const __nv_bfloat162 b2 =
                                            __floats2bfloat162_rn(y2[0], y2[1]);
                                        pk[cc][h][2 * r + e] =
                                            *reinterpret_cast<const uint32_t*>(&b2);
                                    }
                        }
                    }
                    // 3) stage and store the batch
#pragma unroll
                    for (int cc = 0; cc < kBatch; ++cc) {
                        const int c = 32 * grp + 64 * (cb + cc);
                        if (c < args.bn) {
                            if (issuer) bulk_wait_read<0>();  // the group's last stores have read it
                            named_bar_sync(grp_bar, 128);
                            const uint32_t sy_u32 = smem_u32(sy);
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
                                    stmatrix_x4_trans(addr, pk[cc][h][4 * rp + 0],
                                                      pk[cc][h][4 * rp + 1], pk[cc][h][4 * rp + 2],
                                                      pk[cc][h][4 * rp + 3]);
                                }
                            fence_async_shared();
                            named_bar_sync(grp_bar, 128);
                            if (issuer) {
                                const uint64_t stream = l2_policy_evict_first();
                                tma_store_2d_hint(&tm_y, sy, a_cta0, b0 + c, stream);
                                tma_store_2d_hint(&tm_y, sy + 32 * 128, a_cta0 + 64, b0 + c,
                                                  stream);
                                bulk_commit_group();
                            }
                        }
                    }
                }
                continue;
            }
            for (int c = 32 * grp; c < args.bn; c += 64) {
                const int bc = b0 + c + lane;  // this lane's B row of the chunk
                const float sb_lane = load_b_scale<kQ>(args.s_b, bc, bc < args.rowsB);
                uint32_t r[32];
                tmem_ld_32x32b_x32(t_row + c, r);
                tmem_ld_wait();
                if (c + 64 >= args.bn) {  // this group's last read: release its part
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) {
                        if constexpr (kPair == 2)
                            mbar_arrive_cluster(acc_empty_leader + acc * sizeof(uint64_t));
                        else
                            mbar_arrive(&acc_empty[acc]);
                    }
                }
                if (args.tma_store) {
                    if (issuer) bulk_wait_read<0>();  // the group's last store has read it
                    named_bar_sync(grp_bar, 128);
                    if (args.a_is_w) {
                        // box [32 B rows][128 A rows]: element (u, lane_row)
#pragma unroll
                        for (int u = 0; u < 32; ++u) {
                            const float sb = __shfl_sync(0xffffffffu, sb_lane, u);
                            const float accv = kInt8
                                                   ? __int2float_rn(static_cast<int32_t>(r[u]))
                                                   : __uint_as_float(r[u]);
                            const float v = __fmul_rn(__fmul_rn(accv, sb), sa);
                            reinterpret_cast<__nv_bfloat16*>(sy)[u * kTileA + lane_row] =
                                __float2bfloat16_rn(v);
                        }
                    } else {
                        // box [128 A rows][32 B rows]: this lane's row is contiguous
                        uint32_t packed[32 * kEsz / 4];
#pragma unroll
                        for (int u = 0; u < 32; ++u) {
                            const float sb = __shfl_sync(0xffffffffu, sb_lane, u);
                            const float accv = kInt8
                                                   ? __int2float_rn(static_cast<int32_t>(r[u]))
                                                   : __uint_as_float(r[u]);
                            const float v = __fmul_rn(__fmul_rn(accv, sa), sb);
                            const uint32_t h = __bfloat16_as_ushort(__float2bfloat16_rn(v));
                            if (u & 1)
                                packed[u >> 1] |= h << 16;
                            else
                                packed[u >> 1] = h;
                        }
                        uint4* dst = reinterpret_cast<uint4*>(sy + lane_row * 32 * kEsz);
#pragma unroll
                        for (int w = 0; w < 32 * kEsz / 16; ++w)
                            dst[w] = make_uint4(packed[4 * w], packed[4 * w + 1],
                                                packed[4 * w + 2], packed[4 * w + 3]);
                    }
                    fence_async_shared();
                    named_bar_sync(grp_bar, 128);
                    if (issuer) {
                        const uint64_t stream = l2_policy_evict_first();
                        if (args.a_is_w)
                            tma_store_2d_hint(&tm_y, sy, a_cta0, b0 + c, stream);
                        else
                            tma_store_2d_hint(&tm_y, sy, b0 + c, a_cta0, stream);
                        bulk_commit_group();
                    }
                } else {
#pragma unroll
                    for (int u = 0; u < 32; ++u) {
                        const int b_row = b0 + c + u;
                        const float sb = __shfl_sync(0xffffffffu, sb_lane, u);
                        if (row_ok && b_row < args.rowsB) {
                            if (args.a_is_w)
                                store_scaled<kInt8, kOutBf16>(
                                    args.y, static_cast<int64_t>(b_row) * args.ldy + a_row,
                                    r[u], sb, sa);
                            else
                                store_scaled<kInt8, kOutBf16>(
                                    args.y, static_cast<int64_t>(a_row) * args.ldy + b_row,
                                    r[u], sa, sb);
                        }
                    }
                }
            }
        }
        if (issuer) bulk_wait_all();  // Y stores done reading shared memory
    }

    __syncwarp();
    tc_fence_before();
    if constexpr (kPair == 2)
        cluster_sync_all();  // both CTAs done with barriers and tensor memory
    else
        __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_g<kPair>(tmem_base, kTmemCols);
    }
}

}  // namespace ss
