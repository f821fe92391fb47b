// ss_api.cu -- the C ABI of libss (declared in include/ss.h): host-side
// argument checks, TMA tensor-map construction and kernel launches.  All
// kernels are compiled into this one translation unit.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <algorithm>
#include <mutex>
#include <vector>

#include "ss.h"
#include "ss_common.cuh"
#include "ss_compress.cuh"
#include "ss_fp4.cuh"
#include "ss_gemm.cuh"
#include "ss_gemm_splitk.cuh"
#include "ss_gemm_wide.cuh"
#include "ss_quant.cuh"

namespace {

std::atomic<int64_t> g_launches{0};

constexpr int kMaxDevices = 64;
int g_arch_ok[kMaxDevices];  // 0 unknown, 1 sm_100, -1 other
int g_num_sms[kMaxDevices];
std::mutex g_mu;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }

ss_status check_device(int* dev_out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return SS_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return SS_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_arch_ok[dev] == 0) {
        int major = 0, minor = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return SS_ERR_CUDA;
        g_arch_ok[dev] = (major == 10 && minor == 0) ? 1 : -1;
        g_num_sms[dev] = sms;
    }
    if (g_arch_ok[dev] != 1) return SS_ERR_ARCH;
    *dev_out = dev;
    return SS_OK;
}

ss_status launched() {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cudaGetLastError() == cudaSuccess ? SS_OK : SS_ERR_CUDA;
}

// Programmatic dependent launch for every kernel (SS_PDL=0 turns it off).
// Each kernel takes griddepcontrol.wait before touching memory that earlier
// work on the stream may write, so results do not depend on this switch.
bool pdl_enabled() {
    static const bool on = [] {
        const char* v = std::getenv("SS_PDL");
        return !(v && std::strcmp(v, "0") == 0);
    }();
    return on;
}

// Launch `kern` on `stream` with programmatic stream serialisation allowed
// and, for cluster > 1, that cluster size.
template <typename... KArgs, typename... Args>
ss_status launch_ex(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                    cudaStream_t stream, int cluster, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    unsigned n = 0;
    if (cluster > 1) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = static_cast<unsigned>(cluster);
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    if (pdl_enabled()) {
        attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[n].val.programmaticStreamSerializationAllowed = 1;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    if (cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...) != cudaSuccess) {
        cudaGetLastError();
        return SS_ERR_CUDA;
    }
    return launched();
}

bool valid_pattern(ss_pattern p) {
    if (p.keep == 0 && p.group == 0) return true;
    return (p.group == 4 || p.group == 6 || p.group == 8 || p.group == 10) &&
           p.keep == p.group - 2;
}

// ---------------------------------------------------------------- tensor maps
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// 2-D row-major matrix [rows, cols] of `esz`-byte elements, box [box_rows, box_cols].
bool make_map_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                 uint32_t box_rows, uint32_t box_cols, CUtensorMapSwizzle swizzle,
                 CUtensorMapDataType dtype = CU_TENSOR_MAP_DATA_TYPE_UINT8, uint32_t esz = 1) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * esz};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tensor map of Y [M, N] for the epilogue's TMA stores of one 32-column chunk:
// box [32 tokens][128 channels] when A rows are channels, [128 tokens][32
// channels] otherwise.  Returns false (direct stores instead) when the rows
// of Y are not 16-byte aligned.
bool make_y_map(CUtensorMap* map, void* Y, int64_t M, int64_t N, bool out_bf16, bool a_is_w) {
    const uint32_t esz = out_bf16 ? 2 : 4;
    if (!out_bf16 || (N * esz) % 16 != 0) return false;  // fp32 Y: direct stores
    const CUtensorMapDataType dt =
        out_bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
    // A rows = channels: one TMA store per 64-channel half of a chunk, staged
    // [32 tokens][64 channels] with 128B swizzle; otherwise [128 tokens][32
    // channels] unswizzled.
    return a_is_w ? make_map_2d(map, Y, M, N, 32, 64, CU_TENSOR_MAP_SWIZZLE_128B, dt, esz)
                  : make_map_2d(map, Y, M, N, ss::kTileA, 32, CU_TENSOR_MAP_SWIZZLE_NONE, dt, esz);
}

template <bool kSparse, int kQ, bool kOutBf16, int kPair>
ss_status launch_gemm(int dev, const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& e,
                      const CUtensorMap& y, const ss::GemmArgs& args, cudaStream_t stream,
                      const CUtensorMap* sfa = nullptr, const CUtensorMap* sfb = nullptr) {
    using C = std::conditional_t<kQ == ss::kQNvfp4, ss::Fp4Cfg<kSparse, kPair>,
                                 ss::GemmCfg<kSparse, kPair, kQ == ss::kQBf16 ? 2 : 1>>;
    auto kern = ss::gemm_kernel<kSparse, kQ, kOutBf16, kPair>;
    static std::once_flag once[kMaxDevices];
    static cudaError_t attr_err[kMaxDevices];
    std::call_once(once[dev], [&] {
        attr_err[dev] =
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    });
    if (attr_err[dev] != cudaSuccess) return SS_ERR_CUDA;
    const int64_t tile_rows = static_cast<int64_t>(ss::kTileA) * kPair;
    const int64_t tiles =
        ((args.rowsA + tile_rows - 1) / tile_rows) * ((args.rowsB + args.bn - 1) / args.bn);
    const int64_t units = g_num_sms[dev] / kPair;
    const int grid = static_cast<int>((tiles < units ? tiles : units) * kPair);
    return launch_ex(kern, dim3(grid), dim3(ss::kGemmThreads), C::kSmemBytes, stream, kPair, a, b,
                     e, y, sfa ? *sfa : a, sfb ? *sfb : a, args);
}

// q: ss::kQE4M3, kQInt8 or kQBf16; bf16: Y element type.
template <bool kSparse, int kPair>
ss_status dispatch_gemm(int dev, int q, bool bf16, const CUtensorMap& a, const CUtensorMap& b,
                        const CUtensorMap& e, const CUtensorMap& y, const ss::GemmArgs& args,
                        cudaStream_t st) {
    using namespace ss;
    if (q == kQInt8)
        return bf16 ? launch_gemm<kSparse, kQInt8, true, kPair>(dev, a, b, e, y, args, st)
                    : launch_gemm<kSparse, kQInt8, false, kPair>(dev, a, b, e, y, args, st);
    if (q == kQBf16)
        return bf16 ? launch_gemm<kSparse, kQBf16, true, kPair>(dev, a, b, e, y, args, st)
                    : launch_gemm<kSparse, kQBf16, false, kPair>(dev, a, b, e, y, args, st);
    return bf16 ? launch_gemm<kSparse, kQE4M3, true, kPair>(dev, a, b, e, y, args, st)
                : launch_gemm<kSparse, kQE4M3, false, kPair>(dev, a, b, e, y, args, st);
}

// Split-K GEMM (decode sizes, A = weight): S K parts on the S CTAs of a
// cluster.  Returns the number of clusters of S CTAs that can be resident at
// once (0 if the kernel cannot run), cached per device.
template <bool kSparse, int kQ, bool kOutBf16>
int splitk_max_clusters(int dev, int S) {
    using C = ss::SplitKCfg<kSparse, kQ == ss::kQBf16 ? 2 : 1>;
    auto kern = ss::gemm_splitk_kernel<kSparse, kQ, kOutBf16>;
    static std::once_flag once[kMaxDevices];
    static int cached[kMaxDevices][4];  // S = 2, 4, 8
    std::call_once(once[dev], [&] {
        for (int i = 0; i < 4; ++i) cached[dev][i] = 0;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 C::kSmemBytes) != cudaSuccess) {
            cudaGetLastError();
            return;
        }
        for (int i = 1; i < 4; ++i) {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(1 << i);
            cfg.blockDim = dim3(ss::kSplitKThreads);
            cfg.dynamicSmemBytes = C::kSmemBytes;
            cudaLaunchAttribute attr[1];
            attr[0].id = cudaLaunchAttributeClusterDimension;
            attr[0].val.clusterDim.x = 1u << i;
            attr[0].val.clusterDim.y = 1;
            attr[0].val.clusterDim.z = 1;
            cfg.attrs = attr;
            cfg.numAttrs = 1;
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
                cudaGetLastError();
                n = 0;
            }
            cached[dev][i] = n;
        }
    });
    return S == 2 ? cached[dev][1] : (S == 4 ? cached[dev][2] : (S == 8 ? cached[dev][3] : 0));
}

template <bool kSparse, int kQ, bool kOutBf16>
ss_status launch_splitk(int S, int64_t tiles, const CUtensorMap& a, const CUtensorMap& b,
                        const CUtensorMap& e, const ss::GemmArgs& args, cudaStream_t stream) {
    using C = ss::SplitKCfg<kSparse, kQ == ss::kQBf16 ? 2 : 1>;
    return launch_ex(ss::gemm_splitk_kernel<kSparse, kQ, kOutBf16>,
                     dim3(static_cast<unsigned>(tiles * S)), dim3(ss::kSplitKThreads), C::kSmemBytes,
                     stream, S, a, b, e, args);
}

// The K split for a decode-sized problem (A = weight, every B row in one
// tile of at most ss::kSkBn): the largest S in {8, 4, 2} whose tiles x S CTAs
// are all resident at once, with at least one K stage per part, and which
// keeps more SMs busy than the one-pass kernel's CTA pairs.  0: no split.
template <bool kSparse, int kQ, bool kOutBf16>
int choose_split(int dev, int64_t rowsA, int64_t rowsB, int k_stages) {
    if (rowsB > ss::kSkBn) return 0;
    const int64_t tiles = (rowsA + ss::kTileA - 1) / ss::kTileA;
    const int64_t pair_ctas = rowsA > ss::kTileA ? (rowsA + 2 * ss::kTileA - 1) / (2 * ss::kTileA) * 2
                                                 : 1;
    for (int S = 8; S >= 2; S /= 2) {
        if (S > k_stages || tiles * S > g_num_sms[dev] || tiles * S <= pair_ctas) continue;
        if (tiles <= splitk_max_clusters<kSparse, kQ, kOutBf16>(dev, S)) return S;
    }
    return 0;
}

// Split-K dispatch on the operand type and Y type; returns SS_ERR_UNSUPPORTED
// (nothing launched) when no split applies.
template <bool kSparse>
ss_status try_splitk(int dev, int q, bool bf16, int64_t rowsA, int64_t rowsB,
                     const void* Av, int64_t a_cols, const void* B, int64_t b_cols,
                     const CUtensorMap& e, const ss::GemmArgs& args, cudaStream_t stream) {
    using namespace ss;
    int S = 0;
#define SS_SK_PICK(Q, BF) S = choose_split<kSparse, Q, BF>(dev, rowsA, rowsB, args.k_stages)
    if (q == kQInt8) { if (bf16) SS_SK_PICK(kQInt8, true); else SS_SK_PICK(kQInt8, false); }
    else if (q == kQBf16) { if (bf16) SS_SK_PICK(kQBf16, true); else SS_SK_PICK(kQBf16, false); }
    else { if (bf16) SS_SK_PICK(kQE4M3, true); else SS_SK_PICK(kQE4M3, false); }
#undef SS_SK_PICK
    if (S == 0) return SS_ERR_UNSUPPORTED;
    ss::GemmArgs a2 = args;
    a2.bn = static_cast<int>(round_up(rowsB, 32));
    CUtensorMap ta, tb;
    if (!make_map_2d(&ta, Av, rowsA, a_cols, ss::kTileA, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d(&tb, B, rowsB, b_cols, a2.bn, 128, CU_TENSOR_MAP_SWIZZLE_128B))
        return SS_ERR_CUDA;
    const int64_t tiles = (rowsA + ss::kTileA - 1) / ss::kTileA;
#define SS_SK_GO(Q, BF) return launch_splitk<kSparse, Q, BF>(S, tiles, ta, tb, e, a2, stream)
    if (q == kQInt8) { if (bf16) SS_SK_GO(kQInt8, true); SS_SK_GO(kQInt8, false); }
    if (q == kQBf16) { if (bf16) SS_SK_GO(kQBf16, true); SS_SK_GO(kQBf16, false); }
    if (bf16) SS_SK_GO(kQE4M3, true);
    SS_SK_GO(kQE4M3, false);
#undef SS_SK_GO
}

// Operand type of the kernels for a public ss_qdtype (-1: not one).
int kernel_q(ss_qdtype q) {
    switch (q) {
        case SS_INT8: return ss::kQInt8;
        case SS_FP8_E4M3: return ss::kQE4M3;
        case SS_BF16: return ss::kQBf16;
    }
    return -1;
}

template <bool kInt8, bool kAIsW>
ss_status launch_gemm_wide(int dev, const CUtensorMap& a, const CUtensorMap& b,
                           const CUtensorMap& e, const CUtensorMap& y, const ss::GemmArgs& args,
                           cudaStream_t stream) {
    using C = ss::WideCfg;
    auto kern = ss::gemm_sparse_wide_kernel<kInt8, kAIsW>;
    static std::once_flag once[kMaxDevices];
    static cudaError_t attr_err[kMaxDevices];
    std::call_once(once[dev], [&] {
        attr_err[dev] =
            cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
    });
    if (attr_err[dev] != cudaSuccess) return SS_ERR_CUDA;
    const int64_t tile_b = static_cast<int64_t>(ss::kWideBT) * args.bn;
    const int64_t tiles = ((args.rowsA + 2 * ss::kTileA - 1) / (2 * ss::kTileA)) *
                          ((args.rowsB + tile_b - 1) / tile_b);
    const int64_t units = g_num_sms[dev] / 2;
    const int grid = static_cast<int>((tiles < units ? tiles : units) * 2);
    return launch_ex(kern, dim3(grid), dim3(ss::kWideThreads), C::kSmemBytes, stream, 2, a, b, e,
                     y, args);
}

// B-tile width of the wide sparse GEMM: the multiple of 32 (<= 224) whose
// tile schedule (persistent pairs, snake order) finishes first.  A tile's time
// is taken as proportional to the bytes a K step brings into each SM (A and
// metadata 5 KB shared by the two B tiles, plus 32 bytes per token of the
// tile), which is what bounds the mainloop.
int choose_bn_wide(int64_t rowsA, int64_t rowsB, int units) {
    const int64_t nA = (rowsA + 2 * ss::kTileA - 1) / (2 * ss::kTileA);
    int best = ss::WideCfg::kBnMax;
    double best_cost = 0.0;
    std::vector<double> load(static_cast<size_t>(units));
    for (int bn = ss::WideCfg::kBnMax; bn >= 64; bn -= 32) {
        const int64_t nB = (rowsB + 2 * bn - 1) / (2 * bn);
        const int64_t tiles = nA * nB;
        std::fill(load.begin(), load.end(), 0.0);
        for (int64_t t = 0; t < tiles; ++t) {
            const int64_t k = t / units, r = t % units;
            const int64_t u = (k & 1) ? units - 1 - r : r;
            const int64_t tok = std::min<int64_t>(2 * bn, rowsB - (t / nA) * 2 * bn);
            load[static_cast<size_t>(u)] += 5120.0 + 32.0 * static_cast<double>(tok);
        }
        const double cost = *std::max_element(load.begin(), load.end());
        if (bn == ss::WideCfg::kBnMax || cost < best_cost * 0.98) {
            best = bn;
            best_cost = cost;
        }
    }
    return best;
}

// SS_SPARSE_KERNEL=narrow|wide|splitk pins the GEMM shape where it applies
// (for tests and measurements; "narrow" also keeps decode-sized problems off
// the split-K kernel); unset or anything else: chosen per problem.
int forced_sparse_kernel() {
    const char* v = std::getenv("SS_SPARSE_KERNEL");
    if (!v) return 0;
    if (std::strcmp(v, "narrow") == 0) return 1;
    if (std::strcmp(v, "wide") == 0) return 2;
    if (std::strcmp(v, "splitk") == 0) return 3;
    return 0;
}

// Wide or narrow sparse GEMM: compare the waves each needs, a wide tile
// (256 channels x 448 tokens) counting as 1.8 narrow ones (256 x 224).  The
// factor is measured on B200 (Qwen2.5-7B gate/up and Llama-3.1-8B q_proj
// shapes at 8192 tokens): a wide K step moves 19 KB into each SM against
// 2 x 12 KB, but its accumulators drain with the tensor pipe idle.
bool prefer_wide(int64_t rowsA, int64_t rowsB, int bn_narrow, int units) {
    const int64_t nA = (rowsA + 2 * ss::kTileA - 1) / (2 * ss::kTileA);
    const int64_t waves_n = (nA * ((rowsB + bn_narrow - 1) / bn_narrow) + units - 1) / units;
    const int64_t tile_w = 2 * ss::WideCfg::kBnMax;
    const int64_t waves_w = (nA * ((rowsB + tile_w - 1) / tile_w) + units - 1) / units;
    return 1.8 * static_cast<double>(waves_w) < static_cast<double>(waves_n);
}

// B rows per tile: the whole of a small B, else the largest width <= max.
int choose_bn(int64_t rowsB, int bn_max) {
    const int64_t r = round_up(rowsB, 32);
    return static_cast<int>(r < bn_max ? r : bn_max);
}

// Groups the GEMM kernels walk the A tiles in (tile_coords).  A wave of CTA
// pairs works on consecutive tiles: with g groups it re-reads 1/g of A and
// touches about units * g / nA B tiles.  The smallest g whose per-wave set
// (A / g plus those B tiles) fits in 40 MB keeps A in L2 across waves at the
// cost of reading B g times; if no g fits (B tiles of long rows), one group
// reads B once.  Measured on B200: Llama-3.1-8B gate/up 6:8 INT8, M = 16384
// (A 55 MB, B tiles 2.75 MB): one group 551-561 us, two 528-535 us, four
// 549 us; the down projection (B tiles 9.6 MB) runs best as one group.
int a_groups_for(int64_t a_bytes, int64_t nA, int64_t units, int64_t b_tile_bytes) {
    const int64_t budget = int64_t{40} << 20;
    for (int64_t g = 1; g <= 8 && g <= nA; ++g) {
        const int64_t b_tiles = (units * g + nA - 1) / nA;
        if ((a_bytes + g - 1) / g + b_tiles * b_tile_bytes <= budget) return static_cast<int>(g);
    }
    return 1;
}

// The GEMM kernels count output tiles (A tiles of 128 or 256 rows x B tiles
// of bn rows) in 32-bit integers.
bool tiles_overflow(int64_t rowsA, int64_t rowsB, int bn) {
    return (rowsA + 127) / 128 * ((rowsB + bn - 1) / bn) > INT32_MAX;
}

// Opt a row kernel into more than 48 KB of dynamic shared memory when needed.
template <typename Kern>
ss_status set_smem(Kern kern, int /*dev*/, size_t bytes) {
    if (bytes <= 48 * 1024) return SS_OK;
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(bytes)) == cudaSuccess
               ? SS_OK
               : SS_ERR_CUDA;
}

constexpr size_t kMaxRowSmem = 200 * 1024;

}  // namespace

extern "C" {

const char* ss_status_string(ss_status s) {
    switch (s) {
        case SS_OK: return "SS_OK";
        case SS_ERR_INVALID_ARG: return "SS_ERR_INVALID_ARG";
        case SS_ERR_UNSUPPORTED: return "SS_ERR_UNSUPPORTED";
        case SS_ERR_ALIGNMENT: return "SS_ERR_ALIGNMENT";
        case SS_ERR_ARCH: return "SS_ERR_ARCH";
        case SS_ERR_CUDA: return "SS_ERR_CUDA";
        case SS_ERR_TIMEOUT: return "SS_ERR_TIMEOUT";
        case SS_ERR_DATA: return "SS_ERR_DATA";
    }
    return "SS_ERR_UNKNOWN";
}

int64_t ss_kernel_launches(void) { return g_launches.load(); }

ss_status ss_parse_pattern(const char* s, ss_pattern* out) {
    if (!s || !out) return SS_ERR_INVALID_ARG;
    if (std::strcmp(s, "dense") == 0) {
        *out = ss_pattern{0, 0};
        return SS_OK;
    }
    static const char* names[] = {"2:4", "4:6", "6:8", "8:10"};
    for (int i = 0; i < 4; ++i)
        if (std::strcmp(s, names[i]) == 0) {
            *out = ss_pattern{2 * i + 2, 2 * i + 4};
            return SS_OK;
        }
    return SS_ERR_INVALID_ARG;
}

ss_status ss_slide_shape(ss_pattern p, int64_t K, int64_t* K_pad, int64_t* K_lift,
                         int64_t* K_lp) {
    if (!valid_pattern(p) || K <= 0 || K > (int64_t{1} << 30) || !K_pad || !K_lift || !K_lp)
        return SS_ERR_INVALID_ARG;
    if (p.group == 0) {
        *K_pad = K;
        *K_lift = K;
        *K_lp = round_up(K, 128);
        return SS_OK;
    }
    const int64_t G = (K + p.group - 1) / p.group;
    const int64_t Nh = p.group / 2;
    *K_pad = G * p.group;
    *K_lift = G * (Nh - 1) * 4;
    *K_lp = round_up(*K_lift, 128);
    return SS_OK;
}

ss_status ss_act_2to4_shape(int64_t K, int64_t* K_lp) {
    if (K <= 0 || K > (int64_t{1} << 30) || !K_lp) return SS_ERR_INVALID_ARG;
    *K_lp = round_up(round_up(K, 4), 128);
    return SS_OK;
}

int64_t ss_meta_bytes(int64_t rows, int64_t K_lp) {
    if (rows < 1 || rows > INT32_MAX || K_lp <= 0 || K_lp % 128 != 0 || K_lp > (int64_t{1} << 30))
        return 0;
    return (rows + 127) / 128 * 128 * (K_lp / 8);
}

ss_status ss_sparse_gemm(int sparse_operand, const void* Av, const void* Am, const float* s_a,
                         const void* B, const float* s_b, int64_t M, int64_t N, int64_t K_lp,
                         ss_qdtype q, void* Y, ss_out_dtype out_dtype, ss_stream_t stream) {
    if (sparse_operand != 0 && sparse_operand != 1) return SS_ERR_INVALID_ARG;
    const int kq = kernel_q(q);
    if (kq < 0) return SS_ERR_INVALID_ARG;
    const bool scaled = kq != ss::kQBf16;  // bf16 tier: s_a, s_b unused
    if (!Av || !Am || (scaled && (!s_a || !s_b)) || !B || !Y) return SS_ERR_INVALID_ARG;
    if (M <= 0 || N <= 0 || M > INT32_MAX || N > INT32_MAX || K_lp <= 0 || K_lp % 128 != 0 ||
        K_lp > (int64_t{1} << 30))
        return SS_ERR_INVALID_ARG;
    if (out_dtype != SS_OUT_F32 && out_dtype != SS_OUT_BF16) return SS_ERR_INVALID_ARG;
    if (!aligned16(Av) || !aligned16(Am) || !aligned16(B) || !aligned16(Y)) return SS_ERR_ALIGNMENT;
    int dev;
    ss_status st = check_device(&dev);
    if (st != SS_OK) return st;
    const int64_t rowsA = sparse_operand == 0 ? N : M;
    const int64_t rowsB = sparse_operand == 0 ? M : N;
    const int pair = rowsA > ss::kTileA ? 2 : 1;
    const int bn = choose_bn(rowsB, ss::GemmCfg<true, 1>::kBnMax);
    if (tiles_overflow(rowsA, rowsB, bn)) return SS_ERR_UNSUPPORTED;
    // operand element bytes: the maps address bytes, so a bf16 row is twice as wide
    const int64_t eb = scaled ? 1 : 2;
    CUtensorMap ta, tb, te;
    using CS = ss::GemmCfg<true, 1>;
    if (!make_map_2d(&ta, Av, rowsA, K_lp / 2 * eb, ss::kTileA, CS::kARowBytes,
                     CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d(&tb, B, rowsB, K_lp * eb, bn / pair, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d(&te, Am, (rowsA + 127) / 128 * (K_lp / 128) * 16, 128, 16, 128,
                     CU_TENSOR_MAP_SWIZZLE_NONE))
        return SS_ERR_CUDA;
    ss::GemmArgs args;
    args.rowsA = static_cast<int>(rowsA);
    args.rowsB = static_cast<int>(rowsB);
    // 8-bit: a last half stage (K_lp an odd multiple of 128) reads zeros past
    // the rows; bf16 stages are 128 K
    const int64_t stage_k = scaled ? CS::kStageK : ss::GemmCfg<true, 1, 2>::kStageK;
    args.k_stages = static_cast<int>((K_lp + stage_k - 1) / stage_k);
    args.bn = bn;
    args.a_is_w = sparse_operand == 0 ? 1 : 0;
    args.ldy = static_cast<int>(N);
    args.e_chunks = static_cast<int>(K_lp / 128);
    args.sf_k = 0;
    // values + selectors of A; B tiles of bn rows (the wide kernel sets its own)
    args.a_groups = a_groups_for(rowsA * (K_lp / 2 * eb + K_lp / 8), (rowsA + 255) / 256,
                                 g_num_sms[dev] / 2, static_cast<int64_t>(bn) * K_lp * eb);
    args.s_a = s_a;
    args.s_b = s_b;
    args.y = Y;
    CUtensorMap ty;
    args.tma_store = make_y_map(&ty, Y, M, N, out_dtype == SS_OUT_BF16, args.a_is_w) ? 1 : 0;
    if (!args.tma_store) ty = ta;  // unused
    cudaStream_t st_ = reinterpret_cast<cudaStream_t>(stream);
    const bool i8 = q == SS_INT8, bf = out_dtype == SS_OUT_BF16;
    const int forced = forced_sparse_kernel();
    if (args.a_is_w && forced != 1 && forced != 2) {  // decode sizes: split K over a cluster
        const ss_status sk = try_splitk<true>(dev, kq, bf, rowsA, rowsB, Av, K_lp / 2 * eb, B,
                                              K_lp * eb, te, args, st_);
        if (sk != SS_ERR_UNSUPPORTED) return sk;
    }
#if SS_SPARSE_WIDE
    // (8-bit operands only: the bf16 tier runs the one-B-tile kernel)
    // Large problems with bf16 Y may take two B tiles per output tile: fewer
    // bytes per MMA, but single-buffered accumulators.
    if (scaled && pair == 2 && args.tma_store && forced != 1 &&
        (forced == 2 || (rowsB > 2 * ss::WideCfg::kBnMax &&
                         prefer_wide(rowsA, rowsB, bn, g_num_sms[dev] / 2)))) {
        using CW = ss::WideCfg;
        const int bnw = choose_bn_wide(rowsA, rowsB, g_num_sms[dev] / 2);
        CUtensorMap wa, wb;
        if (!make_map_2d(&wa, Av, rowsA, K_lp / 2, ss::kTileA, CW::kARowBytes,
                         CU_TENSOR_MAP_SWIZZLE_64B) ||
            !make_map_2d(&wb, B, rowsB, K_lp, bnw / 2, 128, CU_TENSOR_MAP_SWIZZLE_128B))
            return SS_ERR_CUDA;
        ss::GemmArgs wargs = args;
        wargs.bn = bnw;
        wargs.a_groups = a_groups_for(rowsA * (K_lp / 2 + K_lp / 8), (rowsA + 255) / 256,
                                      g_num_sms[dev] / 2, 2 * static_cast<int64_t>(bnw) * K_lp);
        wargs.k_stages = static_cast<int>(K_lp / CW::kStageK);
        if (args.a_is_w)
            return i8 ? launch_gemm_wide<true, true>(dev, wa, wb, te, ty, wargs, st_)
                      : launch_gemm_wide<false, true>(dev, wa, wb, te, ty, wargs, st_);
        return i8 ? launch_gemm_wide<true, false>(dev, wa, wb, te, ty, wargs, st_)
                  : launch_gemm_wide<false, false>(dev, wa, wb, te, ty, wargs, st_);
    }
#endif
    if (pair == 1) return dispatch_gemm<true, 1>(dev, kq, bf, ta, tb, te, ty, args, st_);
    return dispatch_gemm<true, 2>(dev, kq, bf, ta, tb, te, ty, args, st_);
}

ss_status ss_dense_gemm(const void* Xq, const float* s_x, const void* Wq, const float* s_w,
                        int64_t M, int64_t N, int64_t K_p, ss_qdtype q, void* Y,
                        ss_out_dtype out_dtype, ss_stream_t stream) {
    const int kq = kernel_q(q);
    if (kq < 0) return SS_ERR_INVALID_ARG;
    const bool scaled = kq != ss::kQBf16;  // bf16 tier: s_x, s_w unused
    if (!Xq || (scaled && (!s_x || !s_w)) || !Wq || !Y) return SS_ERR_INVALID_ARG;
    if (M <= 0 || N <= 0 || M > INT32_MAX || N > INT32_MAX || K_p <= 0 || K_p % 128 != 0 ||
        K_p > (int64_t{1} << 30))
        return SS_ERR_INVALID_ARG;
    if (out_dtype != SS_OUT_F32 && out_dtype != SS_OUT_BF16) return SS_ERR_INVALID_ARG;
    if (!aligned16(Xq) || !aligned16(Wq) || !aligned16(Y)) return SS_ERR_ALIGNMENT;
    int dev;
    ss_status st = check_device(&dev);
    if (st != SS_OK) return st;
    const int pair = N > ss::kTileA ? 2 : 1;
    const int bn = choose_bn(M, ss::GemmCfg<false, 1>::kBnMax);
    if (tiles_overflow(N, M, bn)) return SS_ERR_UNSUPPORTED;
    const int64_t eb = scaled ? 1 : 2;  // operand element bytes
    CUtensorMap ta, tb;
    if (!make_map_2d(&ta, Wq, N, K_p * eb, ss::kTileA, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d(&tb, Xq, M, K_p * eb, bn / pair, 128, CU_TENSOR_MAP_SWIZZLE_128B))
        return SS_ERR_CUDA;
    ss::GemmArgs args;
    args.rowsA = static_cast<int>(N);
    args.rowsB = static_cast<int>(M);
    args.k_stages = static_cast<int>(K_p * eb / 128);  // 128 bytes of K per stage
    args.bn = bn;
    args.a_is_w = 1;
    args.ldy = static_cast<int>(N);
    args.e_chunks = 0;
    args.sf_k = 0;
    args.a_groups = a_groups_for(N * K_p * eb, (N + 255) / 256, g_num_sms[dev] / 2,
                                 static_cast<int64_t>(bn) * K_p * eb);
    args.s_a = s_w;
    args.s_b = s_x;
    args.y = Y;
    CUtensorMap ty;
    args.tma_store = make_y_map(&ty, Y, M, N, out_dtype == SS_OUT_BF16, true) ? 1 : 0;
    if (!args.tma_store) ty = ta;  // unused
    cudaStream_t st_ = reinterpret_cast<cudaStream_t>(stream);
    const bool bf = out_dtype == SS_OUT_BF16;
    if (forced_sparse_kernel() != 1) {  // decode sizes: split K over a cluster
        const ss_status sk =
            try_splitk<false>(dev, kq, bf, N, M, Wq, K_p * eb, Xq, K_p * eb, ta, args, st_);
        if (sk != SS_ERR_UNSUPPORTED) return sk;
    }
    return pair == 2 ? dispatch_gemm<false, 2>(dev, kq, bf, ta, tb, ta, ty, args, st_)
                     : dispatch_gemm<false, 1>(dev, kq, bf, ta, tb, ta, ty, args, st_);
}

// ---------------------------------------------------------------- NVFP4

ss_status ss_fp4_shape(ss_pattern p, int64_t K, int64_t* K_lift, int64_t* K_lp) {
    if (!valid_pattern(p) || K <= 0 || K > (int64_t{1} << 30) || !K_lift || !K_lp)
        return SS_ERR_INVALID_ARG;
    if (p.group == 0) {
        *K_lift = K;
        *K_lp = round_up(K, 256);
        return SS_OK;
    }
    int64_t kp_pad, kp_lift, kp_lp;
    const ss_status st = ss_slide_shape(p, (K + 1) / 2, &kp_pad, &kp_lift, &kp_lp);
    if (st != SS_OK) return st;
    *K_lift = 2 * kp_lift;
    *K_lp = 2 * kp_lp;
    return SS_OK;
}

int64_t ss_fp4_scale_bytes(int64_t rows, int64_t K_lp, int32_t block) {
    if (rows < 1 || rows > INT32_MAX || K_lp <= 0 || K_lp % 256 != 0 || K_lp > (int64_t{1} << 30) ||
        (block != 16 && block != 32))
        return 0;
    return (rows + 127) / 128 * 128 * (K_lp / block);
}


}  // extern "C"

namespace {

// Shared by the two NVFP4 GEMMs: tiles of 128 weight rows per CTA x up to 128
// tokens (single SM), or, above 128 weight rows, a CTA pair with MMA M = 256 x
// up to 256 tokens (two 128-row scale tiles of B).  One B tile covers small M.
template <bool kSparse>
ss_status gemm_nvfp4(const void* Av, const void* Am, const void* As, const float* g_w,
                     const void* Bv, const void* Bs, const float* g_x, int64_t M, int64_t N,
                     int64_t K_lp, void* Y, ss_out_dtype out_dtype, ss_stream_t stream) {
    if (!Av || (kSparse && !Am) || !As || !g_w || !Bv || !Bs || !g_x || !Y)
        return SS_ERR_INVALID_ARG;
    if (M <= 0 || N <= 0 || M > INT32_MAX || N > INT32_MAX || K_lp <= 0 || K_lp % 256 != 0 ||
        K_lp > (int64_t{1} << 30))
        return SS_ERR_INVALID_ARG;
    if (out_dtype != SS_OUT_F32 && out_dtype != SS_OUT_BF16) return SS_ERR_INVALID_ARG;
    if (!aligned16(Av) || (kSparse && !aligned16(Am)) || !aligned16(As) || !aligned16(Bv) ||
        !aligned16(Bs) || !aligned16(Y))
        return SS_ERR_ALIGNMENT;
    int dev;
    ss_status st = check_device(&dev);
    if (st != SS_OK) return st;
    using C = ss::Fp4Cfg<kSparse>;
    const int block = kSparse ? 32 : 16;
    // CTA pairs (MMA M = 256, N up to 256 tokens) above one 128-row A tile;
    // for the sparse product only from K_lp > 2048: with fewer K stages per
    // tile the pair's single accumulator leaves the MMAs waiting on the
    // epilogue, and the single-SM form (two accumulators) is faster (measured
    // at M = 8192, N = 14336: K_lp = 2048 106.6 us single vs 123.0 us pair;
    // K_lp = 4096 190.7 vs 166.8 us)
    const int pair = N > ss::kTileA && (!kSparse || K_lp > 2048) ? 2 : 1;
    const int bn_max = pair == 2 ? ss::Fp4Cfg<kSparse, 2>::kBnMax : C::kBnMax;
    const int bn = M <= bn_max ? static_cast<int>(round_up(M, 32)) : bn_max;
    if (tiles_overflow(N, M, bn)) return SS_ERR_UNSUPPORTED;
    const int64_t a_bytes = kSparse ? K_lp / 4 : K_lp / 2;  // bytes per A row
    const int64_t nblk = K_lp / block;
    CUtensorMap ta, tb, te, tsa, tsb;
    if (!make_map_2d(&ta, Av, N, a_bytes, ss::kTileA, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d(&tb, Bv, M, K_lp / 2, bn / pair, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map_2d(&tsa, As, (N + 127) / 128 * nblk, 128, 16, 128, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map_2d(&tsb, Bs, (M + 127) / 128 * nblk, 128, 16, 128, CU_TENSOR_MAP_SWIZZLE_NONE))
        return SS_ERR_CUDA;
    if (kSparse) {
        if (!make_map_2d(&te, Am, (N + 127) / 128 * (K_lp / 256) * 16, 128, 16, 128,
                         CU_TENSOR_MAP_SWIZZLE_NONE))
            return SS_ERR_CUDA;
    } else {
        te = ta;  // unused
    }
    ss::GemmArgs args;
    args.rowsA = static_cast<int>(N);
    args.rowsB = static_cast<int>(M);
    args.k_stages = static_cast<int>((K_lp + C::kStageK - 1) / C::kStageK);
    args.bn = bn;
    args.a_is_w = 1;
    args.ldy = static_cast<int>(N);
    args.e_chunks = static_cast<int>(K_lp / 256);
    args.sf_k = static_cast<int>(nblk / 4);
    // codes, block scales and (sparse) selectors of the weight
    args.a_groups = a_groups_for(N * (kSparse ? K_lp / 4 + K_lp / 16 : K_lp / 2) + N * nblk,
                                 (N + 255) / 256, g_num_sms[dev] / 2,
                                 static_cast<int64_t>(bn) * (K_lp / 2 + K_lp / 16));
    args.s_a = g_w;
    args.s_b = g_x;
    args.y = Y;
    CUtensorMap ty;
    args.tma_store = make_y_map(&ty, Y, M, N, out_dtype == SS_OUT_BF16, true) ? 1 : 0;
    if (!args.tma_store) ty = ta;  // unused
    cudaStream_t st_ = reinterpret_cast<cudaStream_t>(stream);
    const bool bf = out_dtype == SS_OUT_BF16;
    if (pair == 2)
        return bf ? launch_gemm<kSparse, ss::kQNvfp4, true, 2>(dev, ta, tb, te, ty, args, st_, &tsa,
                                                               &tsb)
                  : launch_gemm<kSparse, ss::kQNvfp4, false, 2>(dev, ta, tb, te, ty, args, st_,
                                                                &tsa, &tsb);
    return bf ? launch_gemm<kSparse, ss::kQNvfp4, true, 1>(dev, ta, tb, te, ty, args, st_, &tsa, &tsb)
              : launch_gemm<kSparse, ss::kQNvfp4, false, 1>(dev, ta, tb, te, ty, args, st_, &tsa,
                                                            &tsb);
}

}  // namespace

extern "C" {

ss_status ss_sparse_gemm_nvfp4(const void* Wv, const void* Wm, const void* Ws, const float* g_w,
                               const void* Xv, const void* Xs, const float* g_x, int64_t M,
                               int64_t N, int64_t K_lp, void* Y, ss_out_dtype out_dtype,
                               ss_stream_t stream) {
    return gemm_nvfp4<true>(Wv, Wm, Ws, g_w, Xv, Xs, g_x, M, N, K_lp, Y, out_dtype, stream);
}

ss_status ss_dense_gemm_nvfp4(const void* Xv, const void* Xs, const float* g_x, const void* Wv,
                              const void* Ws, const float* g_w, int64_t M, int64_t N,
                              int64_t K_p, void* Y, ss_out_dtype out_dtype, ss_stream_t stream) {
    return gemm_nvfp4<false>(Wv, nullptr, Ws, g_w, Xv, Xs, g_x, M, N, K_p, Y, out_dtype, stream);
}

ss_status ss_get_device_status(ss_stream_t stream) {
    int dev;
    ss_status st = check_device(&dev);
    if (st != SS_OK) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // one thread takes the word and leaves zero in one atomic exchange, after
    // everything queued on `s` before it (plain launch: full serialisation)
    ss::status_exchange_kernel<<<1, 1, 0, s>>>();
    if (cudaGetLastError() != cudaSuccess) return SS_ERR_CUDA;
    int code = 0;
    if (cudaMemcpyFromSymbolAsync(&code, ss::g_status_taken, sizeof(int), 0,
                                  cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return SS_ERR_CUDA;
    return static_cast<ss_status>(code);
}

ss_status ss_debug_set_wait_limit(uint64_t ns) {
    if (ns < 1000000ull || ns > 60000000000ull) return SS_ERR_INVALID_ARG;  // 1 ms .. 60 s
    int dev;
    ss_status st = check_device(&dev);
    if (st != SS_OK) return st;
    if (cudaDeviceSynchronize() != cudaSuccess) return SS_ERR_CUDA;
    if (cudaMemcpyToSymbol(ss::g_wait_limit_ns, &ns, sizeof(ns)) != cudaSuccess) return SS_ERR_CUDA;
    return SS_OK;
}

ss_status ss_debug_skip_stage(int32_t kb) {
    if (kb < -1) return SS_ERR_INVALID_ARG;
    int dev;
    ss_status st = check_device(&dev);
    if (st != SS_OK) return st;
    if (cudaDeviceSynchronize() != cudaSuccess) return SS_ERR_CUDA;
    if (cudaMemcpyToSymbol(ss::g_skip_stage, &kb, sizeof(kb)) != cudaSuccess) return SS_ERR_CUDA;
    return SS_OK;
}

}  // extern "C"

// The entry points that prepare the GEMM operands (weight compression,
// activation quantisation, lifting and pruning, and their NVFP4 forms).
#include "ss_api_operands.cuh"
