// ss_common.cuh -- sm_100a building blocks shared by the libss kernels:
// device status word, bounded mbarrier waits, TMA loads, tcgen05 (TMEM
// allocation, MMA, copies, loads) and shared-memory matrix descriptors.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <stdint.h>

namespace ss {

// Device status word: the first device-side error since the last read.
__device__ int g_status;
// Written by ss_get_device_status()'s exchange kernel: the status it took.
__device__ int g_status_taken;

__device__ __forceinline__ void record_status(int code) { atomicCAS(&g_status, 0, code); }

// Take the status word and leave zero, in one atomic exchange, so that an
// error recorded concurrently is either taken now or left for the next read.
__global__ void status_exchange_kernel() { g_status_taken = atomicExch(&g_status, 0); }

// ---------------------------------------------------------------------------
// Time and bounded waits.  Every spin in these kernels gives up after
// g_wait_limit_ns (4 s unless a test shortens it through
// ss_debug_set_wait_limit) or when the CTA-wide abort flag is raised,
// records SS_ERR_TIMEOUT and lets the caller unwind; nothing traps or hangs.
// ---------------------------------------------------------------------------
constexpr uint64_t kWaitLimitNs = 4000000000ull;  // 4 s
__device__ uint64_t g_wait_limit_ns = kWaitLimitNs;
// Test hook (ss_debug_skip_stage): when >= 0, the GEMM producers issue no
// copies for K stage g_skip_stage of their first tile, so the MMA warp's wait
// for that stage can only run out.  -1 (off) in normal use.
__device__ int g_skip_stage = -1;
constexpr int kErrTimeout = 6;                    // SS_ERR_TIMEOUT
constexpr int kErrData = 7;                       // SS_ERR_DATA

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_async_shared() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for the phase with parity `parity` of `bar` to complete.  Returns
// false (after recording SS_ERR_TIMEOUT) if the time limit passes or another
// role of the CTA has raised `abort_flag`.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity,
                                          volatile int* abort_flag) {
    const uint32_t b = smem_u32(bar);
    if (mbar_try_wait(b, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(b, parity)) return true;
        if ((i & 255u) == 0) {
            if (*abort_flag) return false;
            if (global_timer_ns() - t0 > *reinterpret_cast<volatile uint64_t*>(&g_wait_limit_ns)) {
                record_status(kErrTimeout);
                *abort_flag = 1;
                return false;
            }
        }
    }
}

// Wait up to 100 ms for a phase on an exit path (copies or MMAs already
// issued must land before their shared or tensor memory is given back).
__device__ __forceinline__ bool mbar_drain(uint64_t* bar, uint32_t parity) {
    const uint32_t b = smem_u32(bar);
    const uint64_t t0 = global_timer_ns();
    while (!mbar_try_wait(b, parity))
        if (global_timer_ns() - t0 > 100000000ull) return false;  // 100 ms
    return true;
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

// Tile-major metadata: byte b of row r of a [rows, K_lp/8] selector matrix is
// stored at this offset, so the selectors of 128 rows x 128 K (one GEMM
// stage's metadata tile) form one contiguous 2 KB block ([128 rows][16 B]).
__host__ __device__ __forceinline__ int64_t meta_offset(int64_t r, int64_t b, int64_t K_lp) {
    return ((r >> 7) * (K_lp >> 7) + (b >> 4)) * 2048 + (r & 127) * 16 + (b & 15);
}

// The 16-bit sparse MMA (kind::f16) reads the 32 selector bits of one MMA for
// rows r and r + 8 of each 16-row group from one tensor-memory column as two
// 16-bit halves (the pairing of the warp-level 16-bit sparse MMA's metadata
// register).  The bf16 tier therefore stores the selectors with row bit 3 and
// byte bit 1 exchanged inside that layout: the 2-byte half h of 4-byte word c
// of row r lands in row (r & ~8) | 8h, half ((r >> 3) & 1) of the same word.
__host__ __device__ __forceinline__ int64_t meta_offset_i16(int64_t r, int64_t b, int64_t K_lp) {
    const int64_t r2 = (r & ~int64_t{8}) | (((b >> 1) & 1) << 3);
    const int64_t b2 = (b & ~int64_t{2}) | (((r >> 3) & 1) << 1);
    return meta_offset(r2, b2, K_lp);
}

// ---------------------------------------------------------------------------
// Programmatic dependent launch.  Every kernel of this library is launched
// with programmatic stream serialisation allowed: it may start while the
// previous kernel on the stream is still running, and pdl_wait() -- taken by
// every thread before its first access to memory that other work may write --
// returns once that kernel has completed and its writes are visible.
// pdl_trigger() lets the next kernel start early; it takes effect once every
// CTA of this grid has issued it (or exited), i.e. when all of them are
// already resident, so an early dependent cannot keep this grid from running.
// Without the launch attribute both are no-ops.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ void pdl_trigger() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------------------
// TMA (no multicast anywhere in this library).
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Prefetch one box of a 2-D tensor map into L2 (no shared-memory write, no
// barrier).  L2 is the point of coherence, so this is safe even before
// pdl_wait(): a later load still sees any write made in between.
__device__ __forceinline__ void tma_prefetch_l2_2d(const CUtensorMap* map, int32_t x, int32_t y) {
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global [%0, {%1, %2}];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(x), "r"(y)
                 : "memory");
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t x, int32_t y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

// 1-D bulk copy global -> this CTA's shared memory, completion counted on
// `bar` (both addresses 16-byte aligned, bytes a multiple of 16).
__device__ __forceinline__ void bulk_load_1d(void* dst, const void* src, uint32_t bytes,
                                             uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// L2 cache policies: operands the GEMM re-reads stay (evict_last); the output
// streams through (evict_first) so it does not push the operands out of L2.
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ void tma_store_2d_hint(const CUtensorMap* map, const void* src,
                                                  int32_t x, int32_t y, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group.L2::cache_hint"
        " [%0, {%2, %3}], [%1], %4;" ::"l"(reinterpret_cast<uint64_t>(map)),
        "r"(smem_u32(src)), "r"(x), "r"(y), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void tma_load_2d_pair_hint(void* dst, const CUtensorMap* map,
                                                      uint32_t bar_cluster_addr, int32_t x,
                                                      int32_t y, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster_addr), "r"(x), "r"(y), "l"(policy)
        : "memory");
}

// TMA tensor store from this CTA's shared memory (bulk-group completion).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int32_t x,
                                             int32_t y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
            reinterpret_cast<uint64_t>(map)),
        "r"(smem_u32(src)), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ void bulk_commit_group() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Wait until at most N committed bulk groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void bulk_wait_all() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// Named barrier over `count` threads that also ANDs a predicate across them.
__device__ __forceinline__ bool named_bar_and(uint32_t id, uint32_t count, bool pred) {
    uint32_t out;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(out)
        : "r"(static_cast<uint32_t>(pred)), "r"(id), "r"(count)
        : "memory");
    return out != 0;
}

// Named barrier over `count` threads (id 0 is __syncthreads).
__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: tensor memory, MMA, copies, loads.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Arrive on `bar` once every tcgen05 operation issued so far by this thread
// has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}

// Shared-memory matrix descriptor (tcgen05 "matrix descriptor"): start
// address, leading/stride byte offsets (>> 4), version 1, swizzle mode.
enum : uint32_t { kSwizzleNone = 0, kSwizzle128B = 2, kSwizzle64B = 4, kSwizzle32B = 6 };

__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo,
                                              uint32_t swizzle) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
    d |= 1ull << 46;
    d |= static_cast<uint64_t>(swizzle & 7u) << 61;
    return d;
}

// Instruction descriptor for kind::i8 / kind::f8f6f4, both operands K-major.
//   bits 0-1   sparsity selector (which part of an aligned metadata column
//              pair a sparse MMA reads; 0 for the 8-bit kinds)
//   bit 2      sparse flag
//   bits 4-5   accumulator format (1 = f32, 2 = s32)
//   bits 7-9   A format, 10-12 B format (i8: 1 = signed; f8f6f4: 0 = E4M3)
//   bits 17-22 N >> 3, bits 24-28 M >> 4
__host__ __device__ constexpr uint32_t make_idesc(bool sparse, bool is_int8, uint32_t M,
                                                  uint32_t N) {
    return (sparse ? (1u << 2) : 0u) | ((is_int8 ? 2u : 1u) << 4) | ((is_int8 ? 1u : 0u) << 7) |
           ((is_int8 ? 1u : 0u) << 10) | ((N >> 3) << 17) | ((M >> 4) << 24);
}

// Operand types of the GEMM kernels: the two 8-bit kinds and the 16-bit tier
// (bf16 operands, kind::f16, fp32 accumulator, no scales).
constexpr int kQE4M3 = 0;
constexpr int kQInt8 = 1;
constexpr int kQBf16 = 2;
constexpr int kQNvfp4 = 3;  // E2M1 with UE4M3 block scales (kind::mxf4nvf4)

// Instruction descriptor for kind::f16 with bf16 A and B (format 1 in bits
// 7-9 and 10-12), fp32 accumulator, both operands K-major.
__host__ __device__ constexpr uint32_t make_idesc_bf16(bool sparse, uint32_t M, uint32_t N) {
    return (sparse ? (1u << 2) : 0u) | (1u << 4) | (1u << 7) | (1u << 10) | ((N >> 3) << 17) |
           ((M >> 4) << 24);
}

// Instruction descriptor for kind::mxf4nvf4 (block-scaled): E2M1 A and B
// (format 1 in bits 7-9 and 10-12), UE4M3 scales (bit 23 clear), scale IDs 0
// (bits 4-5, 29-30: each MMA's scales start a tensor-memory column), K-major.
__host__ __device__ constexpr uint32_t make_idesc_fp4(bool sparse, uint32_t M, uint32_t N) {
    return (sparse ? (1u << 2) : 0u) | (1u << 7) | (1u << 10) | ((N >> 3) << 17) | ((M >> 4) << 24);
}

__host__ __device__ constexpr uint32_t make_idesc_q(bool sparse, int q, uint32_t M, uint32_t N) {
    return q == kQBf16    ? make_idesc_bf16(sparse, M, N)
           : q == kQNvfp4 ? make_idesc_fp4(sparse, M, N)
                          : make_idesc(sparse, q == kQInt8, M, N);
}

template <bool kInt8>
__device__ __forceinline__ void mma_dense(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
    if constexpr (kInt8) {
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
            "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
            : "memory");
    } else {
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
            "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
            : "memory");
    }
}

template <bool kInt8>
__device__ __forceinline__ void mma_sparse(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                           uint32_t e_tmem, uint32_t idesc,
                                           uint32_t accumulate) {
    if constexpr (kInt8) {
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %5, 0;\n\t"
            "tcgen05.mma.sp.cta_group::1.kind::i8 [%0], %1, %2, [%3], %4, p;\n\t}" ::"r"(
                d_tmem),
            "l"(a_desc), "l"(b_desc), "r"(e_tmem), "r"(idesc), "r"(accumulate)
            : "memory");
    } else {
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %5, 0;\n\t"
            "tcgen05.mma.sp.cta_group::1.kind::f8f6f4 [%0], %1, %2, [%3], %4, p;\n\t}" ::"r"(
                d_tmem),
            "l"(a_desc), "l"(b_desc), "r"(e_tmem), "r"(idesc), "r"(accumulate)
            : "memory");
    }
}

// Shared memory -> tensor memory, 128 lanes x 128 bits (one 16-byte row of
// the source per lane).
__device__ __forceinline__ void tc_cp_128x128b(uint32_t taddr, uint64_t src_desc) {
    asm volatile("tcgen05.cp.cta_group::1.128x128b [%0], %1;" ::"r"(taddr), "l"(src_desc)
                 : "memory");
}

// Each thread of the warp reads 32 consecutive 32-bit columns of its lane.
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, "
        "[%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr)
        : "memory");
}

// 16 TMEM lanes x 256 bits, repeated 4 times along the columns: with lane
// base L and column base C, thread t receives, for r = 0..3,
//   v[4r + 0] = D[L + t/4][C + 8r + 2(t%4)],  v[4r + 1] = ...[... + 1],
//   v[4r + 2] = D[L + t/4 + 8][C + 8r + 2(t%4)], v[4r + 3] = ...[... + 1],
// i.e. the layout of the m8n8 matrix fragments that stmatrix stores.
__device__ __forceinline__ void tmem_ld_16x256b_x4(uint32_t taddr, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x4.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
          "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
          "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr)
        : "memory");
}

// Four 8x8 b16 matrices stored transposed: thread 8i + j gives the address of
// row j of matrix i; register i holds this thread's fragment of matrix i.
__device__ __forceinline__ void stmatrix_x4_trans(uint32_t saddr, uint32_t r0, uint32_t r1,
                                                  uint32_t r2, uint32_t r3) {
    asm volatile("stmatrix.sync.aligned.m8n8.x4.trans.shared.b16 [%0], {%1, %2, %3, %4};" ::"r"(
                     saddr),
                 "r"(r0), "r"(r1), "r"(r2), "r"(r3)
                 : "memory");
}

__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ bool elect_one() {
    uint32_t pred = 0;
    asm volatile(
        "{\n\t.reg .b32 r;\n\t.reg .pred p;\n\t"
        "elect.sync r|p, 0xffffffff;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(pred));
    return pred != 0;
}

// ---------------------------------------------------------------------------
// Thread-block clusters of two CTAs (cta_group::2): the pair shares one MMA of
// M = 256; each CTA holds half of A and half of B in its own shared memory
// and half of D in its own tensor memory.  Nothing here multicasts a load.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Address of `p` (in this CTA's shared memory) in CTA `rank`'s shared memory,
// as a shared::cluster address.
__device__ __forceinline__ uint32_t map_to_rank(const void* p, uint32_t rank) {
    uint32_t out;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(smem_u32(p)), "r"(rank));
    return out;
}

__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

// Arrive on an mbarrier given by its shared::cluster address (possibly in the
// peer CTA).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
                 : "memory");
}

// TMA load into this CTA's shared memory whose completion is counted on an
// mbarrier that may live in the peer CTA of the pair (given as a
// shared::cluster address).
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* map,
                                                 uint32_t bar_cluster_addr, int32_t x, int32_t y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster_addr), "r"(x), "r"(y)
        : "memory");
}

template <int kPair>
__device__ __forceinline__ void tmem_alloc_g(uint32_t* dst_smem, uint32_t ncols) {
    if constexpr (kPair == 2)
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(dst_smem)),
                     "r"(ncols)
                     : "memory");
    else
        tmem_alloc(dst_smem, ncols);
}

template <int kPair>
__device__ __forceinline__ void tmem_relinquish_g() {
    if constexpr (kPair == 2)
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    else
        tmem_relinquish();
}

template <int kPair>
__device__ __forceinline__ void tmem_dealloc_g(uint32_t taddr, uint32_t ncols) {
    if constexpr (kPair == 2)
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr),
                     "r"(ncols)
                     : "memory");
    else
        tmem_dealloc(taddr, ncols);
}

// Commit: arrive on `bar` (same shared-memory offset in both CTAs of the
// pair) once the tcgen05 operations issued so far have completed.
template <int kPair>
__device__ __forceinline__ void tc_commit_g(uint64_t* bar) {
    if constexpr (kPair == 2)
        asm volatile(
            "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
            " [%0], %1;" ::"r"(smem_u32(bar)),
            "h"(static_cast<uint16_t>(3))
            : "memory");
    else
        tc_commit(bar);
}

template <int kPair, bool kInt8>
__device__ __forceinline__ void mma_dense_g(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
    if constexpr (kPair == 1) {
        mma_dense<kInt8>(d_tmem, a_desc, b_desc, idesc, accumulate);
    } else if constexpr (kInt8) {
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
            "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
            : "memory");
    } else {
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
            "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
            : "memory");
    }
}

template <int kPair, bool kInt8>
__device__ __forceinline__ void mma_sparse_g(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                             uint32_t e_tmem, uint32_t idesc,
                                             uint32_t accumulate) {
    if constexpr (kPair == 1) {
        mma_sparse<kInt8>(d_tmem, a_desc, b_desc, e_tmem, idesc, accumulate);
    } else if constexpr (kInt8) {
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %5, 0;\n\t"
            "tcgen05.mma.sp.cta_group::2.kind::i8 [%0], %1, %2, [%3], %4, p;\n\t}" ::"r"(d_tmem),
            "l"(a_desc), "l"(b_desc), "r"(e_tmem), "r"(idesc), "r"(accumulate)
            : "memory");
    } else {
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %5, 0;\n\t"
            "tcgen05.mma.sp.cta_group::2.kind::f8f6f4 [%0], %1, %2, [%3], %4, p;\n\t}" ::"r"(
                d_tmem),
            "l"(a_desc), "l"(b_desc), "r"(e_tmem), "r"(idesc), "r"(accumulate)
            : "memory");
    }
}

// kind::f16 MMAs of the bf16 tier (dense K = 16, sparse K = 32 per MMA).
template <int kPair>
__device__ __forceinline__ void mma_dense_bf16_g(uint32_t d_tmem, uint64_t a_desc,
                                                 uint64_t b_desc, uint32_t idesc,
                                                 uint32_t accumulate) {
    if constexpr (kPair == 2)
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
            "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
            : "memory");
    else
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
            "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
            "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
            : "memory");
}

template <int kPair>
__device__ __forceinline__ void mma_sparse_bf16_g(uint32_t d_tmem, uint64_t a_desc,
                                                  uint64_t b_desc, uint32_t e_tmem,
                                                  uint32_t idesc, uint32_t accumulate) {
    if constexpr (kPair == 2)
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %5, 0;\n\t"
            "tcgen05.mma.sp.cta_group::2.kind::f16 [%0], %1, %2, [%3], %4, p;\n\t}" ::"r"(
                d_tmem),
            "l"(a_desc), "l"(b_desc), "r"(e_tmem), "r"(idesc), "r"(accumulate)
            : "memory");
    else
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %5, 0;\n\t"
            "tcgen05.mma.sp.cta_group::1.kind::f16 [%0], %1, %2, [%3], %4, p;\n\t}" ::"r"(
                d_tmem),
            "l"(a_desc), "l"(b_desc), "r"(e_tmem), "r"(idesc), "r"(accumulate)
            : "memory");
}

// Block-scaled FP4 MMAs (cta_group::1 form): scale factors of A and B in tensor
// memory, one 32-bit column per 32 rows (4 scales) with the rows of each
// 32-lane quarter repeated in all four quarters (tcgen05.cp .32x128b.warpx4).
__device__ __forceinline__ void mma_fp4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                        uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                        uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %6, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%4], "
        "[%5], p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(sfa), "r"(sfb), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void mma_fp4_sparse(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                               uint32_t e_tmem, uint32_t idesc, uint32_t sfa,
                                               uint32_t sfb, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %7, 0;\n\t"
        "tcgen05.mma.sp.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, [%3], "
        "%4, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(e_tmem), "r"(idesc), "r"(sfa), "r"(sfb), "r"(accumulate)
        : "memory");
}

// Shared memory -> tensor memory, 32 lanes x 128 bits copied to all four
// lane quarters (the scale-factor source: [32 rows][16 B], 512 bytes).  The
// pair form, issued by the leader, copies each CTA's shared memory into its
// own tensor memory.
template <int kPair>
__device__ __forceinline__ void tc_cp_32x128b_warpx4_g(uint32_t taddr, uint64_t src_desc) {
    if constexpr (kPair == 2)
        asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(src_desc)
                     : "memory");
    else
        asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(src_desc)
                     : "memory");
}

// Block-scaled FP4 MMAs in either CTA-group form.
template <int kPair>
__device__ __forceinline__ void mma_fp4_g(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                          uint32_t accumulate) {
    if constexpr (kPair == 2)
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %6, 0;\n\t"
            "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, "
            "[%4], [%5], p;\n\t}" ::"r"(d_tmem),
            "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(sfa), "r"(sfb), "r"(accumulate)
            : "memory");
    else
        mma_fp4(d_tmem, a_desc, b_desc, idesc, sfa, sfb, accumulate);
}

template <int kPair>
__device__ __forceinline__ void mma_fp4_sparse_g(uint32_t d_tmem, uint64_t a_desc,
                                                 uint64_t b_desc, uint32_t e_tmem, uint32_t idesc,
                                                 uint32_t sfa, uint32_t sfb, uint32_t accumulate) {
    if constexpr (kPair == 2)
        asm volatile(
            "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %7, 0;\n\t"
            "tcgen05.mma.sp.cta_group::2.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, "
            "[%3], %4, [%5], [%6], p;\n\t}" ::"r"(d_tmem),
            "l"(a_desc), "l"(b_desc), "r"(e_tmem), "r"(idesc), "r"(sfa), "r"(sfb), "r"(accumulate)
            : "memory");
    else
        mma_fp4_sparse(d_tmem, a_desc, b_desc, e_tmem, idesc, sfa, sfb, accumulate);
}

// Two fp32 products in one instruction (mul.rn.f32x2): (a0 * b0, a1 * b1),
// each rounded to nearest even as __fmul_rn would.
__device__ __forceinline__ void mul_rn_f32x2(float a0, float a1, float b0, float b1, float& r0,
                                             float& r1) {
    uint64_t a, b, r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(a) : "f"(a0), "f"(a1));
    asm("mov.b64 %0, {%1, %2};" : "=l"(b) : "f"(b0), "f"(b1));
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    asm("mov.b64 {%0, %1}, %2;" : "=f"(r0), "=f"(r1) : "l"(r));
}

// Pair sparse MMA that keeps its A operand in the tensor core's collector
// buffer: kUse = 0 reads A from shared memory and keeps it (fill), kUse = 1
// takes A from the collector and releases it (lastuse).  Two MMAs that share
// one A tile then read it from shared memory once.
template <bool kInt8, int kUse>
__device__ __forceinline__ void mma_sparse_pair_coll(uint32_t d_tmem, uint64_t a_desc,
                                                     uint64_t b_desc, uint32_t e_tmem,
                                                     uint32_t idesc, uint32_t accumulate) {
#define SS_MMA_SP_COLL(KIND, USE)                                                             \
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %5, 0;\n\t"                         \
                 "tcgen05.mma.sp.cta_group::2.kind::" KIND ".collector::a::" USE             \
                 " [%0], %1, %2, [%3], %4, p;\n\t}" ::"r"(d_tmem),                          \
                 "l"(a_desc), "l"(b_desc), "r"(e_tmem), "r"(idesc), "r"(accumulate)          \
                 : "memory")
    if constexpr (kInt8) {
        if constexpr (kUse == 0) SS_MMA_SP_COLL("i8", "fill");
        else SS_MMA_SP_COLL("i8", "lastuse");
    } else {
        if constexpr (kUse == 0) SS_MMA_SP_COLL("f8f6f4", "fill");
        else SS_MMA_SP_COLL("f8f6f4", "lastuse");
    }
#undef SS_MMA_SP_COLL
}

template <int kPair>
__device__ __forceinline__ void tc_cp_128x128b_g(uint32_t taddr, uint64_t src_desc) {
    if constexpr (kPair == 2)
        asm volatile("tcgen05.cp.cta_group::2.128x128b [%0], %1;" ::"r"(taddr), "l"(src_desc)
                     : "memory");
    else
        tc_cp_128x128b(taddr, src_desc);
}

// ---------------------------------------------------------------------------
// Quantisation shared by the activation and weight kernels (IEEE fp32
// division and multiply, round to nearest even; INT8 clamped to +-127,
// E4M3 saturated to +-448).
// ---------------------------------------------------------------------------
template <bool kInt8>
__device__ __forceinline__ float q_max() {
    return kInt8 ? 127.0f : 448.0f;
}

template <bool kInt8>
__device__ __forceinline__ void scale_from_absmax(float a, float& inv, float& s) {
    if (a == 0.0f) {
        inv = 0.0f;
        s = 0.0f;
    } else {
        inv = __fdiv_rn(q_max<kInt8>(), a);
        s = __fdiv_rn(a, q_max<kInt8>());
    }
}

template <bool kInt8>
__device__ __forceinline__ uint32_t quantize(float x, float inv) {
    const float p = __fmul_rn(x, inv);
    if constexpr (kInt8) {
        float r = rintf(p);
        r = fminf(fmaxf(r, -127.0f), 127.0f);
        return static_cast<uint32_t>(static_cast<uint8_t>(static_cast<int8_t>(r)));
    } else {
        return static_cast<uint32_t>(__nv_cvt_float_to_fp8(p, __NV_SATFINITE, __NV_E4M3));
    }
}

// bf16 bits of x, rounded to nearest even (the stored values of the bf16 tier).
__device__ __forceinline__ uint32_t bf16_bits(float x) {
    return static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(x)));
}

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) {
    return v;
}
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
    return __bfloat162float(v);
}

}  // namespace ss
