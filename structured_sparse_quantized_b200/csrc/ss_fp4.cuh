// ss_fp4.cuh -- NVFP4 with pairwise sparsity: weight compression (offline)
// and the per-token quantisation + pair lift of activations.
//
// Format ("add 2:4 or drop a precision tier?", paper-daily 2610.28947, 3.3:
// Blackwell's sparse FP4 keeps 2 of every 4 adjacent pairs in 8 elements;
// LLM-Compressor compression schemes, NVFP4 row: E2M1 elements, a local
// scale per group of 16, a global scale per tensor):
//   E2M1 codes, two per byte (low nibble first), UE4M3 local scales,
//   g = amax / 2688, block scale s = UE4M3(a / (6 g)), d = s * g,
//   inv = 1 / d, codes = E2M1(x * inv) (round to nearest even, saturating).
// Sparse patterns count pairs; a window of 4 pairs stores 2 pairs and the
// nibble p0 | p1 << 2.  The sparse instruction scales per 32 lifted K on
// both operands (16 stored weight values, 32 activation elements); the
// dense product per 16.
#pragma once

#include "ss_common.cuh"
#include "ss_compress.cuh"
#include "ss_quant.cuh"

namespace ss {

// Two E2M1 codes in one byte: lo in bits 0-3, hi in bits 4-7
// (cvt.rn.satfinite.e2m1x2.f32 puts its first source in the high nibble).
__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi) {
    uint32_t out;
    asm("{\n\t.reg .b8 b;\n\tcvt.rn.satfinite.e2m1x2.f32 b, %1, %2;\n\tcvt.u32.u8 %0, b;\n\t}"
        : "=r"(out)
        : "f"(hi), "f"(lo));
    return out & 0xFFu;
}

// UE4M3 code of t >= 0 (round to nearest even, saturating at 448) and its
// value: e = c >> 3, m = c & 7 gives (8 + m) 2^(e - 10), or m 2^-9 for e = 0.
__device__ __forceinline__ uint32_t ue4m3_code(float t) {
    return static_cast<uint32_t>(__nv_cvt_float_to_fp8(t, __NV_SATFINITE, __NV_E4M3)) & 0x7Fu;
}

__device__ __forceinline__ float ue4m3_value(uint32_t c) {
    const uint32_t e = (c >> 3) & 15u, m = c & 7u;
    // normal: 2^(e - 7) (1 + m / 8) as fp32 bits; subnormal: m 2^-9 (exact)
    return e == 0 ? __fmul_rn(static_cast<float>(m), 0.001953125f)
                  : __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// Tile-major scale offset (512-byte blocks: 128 rows x 4 consecutive scales,
// the source shape of tcgen05.cp.32x128b.warpx4): scale j of row r.
__host__ __device__ __forceinline__ int64_t fp4_scale_offset(int64_t r, int64_t j, int64_t nblk) {
    return ((r >> 7) * (nblk >> 2) + (j >> 2)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (j & 3);
}

// One block of n (16 or 32) values: the UE4M3 scale code and the packed codes
// (n / 2 bytes into out), global scale g.
template <int kN>
__device__ __forceinline__ uint32_t nvfp4_block(const float (&x)[kN], float g, uint8_t* out) {
    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < kN; ++i) a = fmaxf(a, fabsf(x[i]));
    uint32_t sc = 0;
    float inv = 0.0f;
    if (g != 0.0f) {
        sc = ue4m3_code(__fdiv_rn(a, __fmul_rn(6.0f, g)));
        const float d = __fmul_rn(ue4m3_value(sc), g);
        inv = d == 0.0f ? 0.0f : __fdiv_rn(1.0f, d);
    }
    uint32_t w[kN / 8];
#pragma unroll
    for (int q = 0; q < kN / 8; ++q) {
        uint32_t v = 0;
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            const int i = 8 * q + 2 * h;
            const uint32_t b = inv == 0.0f ? 0u : e2m1x2(__fmul_rn(x[i], inv), __fmul_rn(x[i + 1], inv));
            v |= b << (8 * h);
        }
        w[q] = v;
    }
    if constexpr (kN == 16) {
        *reinterpret_cast<uint2*>(out) = make_uint2(w[0], w[1]);
    } else {
        *reinterpret_cast<uint4*>(out) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    return sc;
}

// Kept pairs of one group of `group` pairs starting at pair p0 of a staged
// row (srow, K_pad floats): bit q set for the `keep` pairs of largest
// x0^2 + x1^2 (double, as the ranking must not depend on rounding), ties
// keep the lower pair.
__device__ __forceinline__ uint32_t kept_pairs(const float* srow, int64_t p0, int group,
                                               int keep) {
    double e[kMaxGroup];
    for (int q = 0; q < group; ++q) {
        const double x0 = srow[2 * (p0 + q)], x1 = srow[2 * (p0 + q) + 1];
        e[q] = x0 * x0 + x1 * x1;
    }
    uint32_t bits = 0;
    for (int q = 0; q < group; ++q) {
        int rank = 0;
        for (int o = 0; o < group; ++o)
            if (o != q && (e[o] > e[q] || (e[o] == e[q] && o < q))) ++rank;
        if (rank < keep) bits |= 1u << q;
    }
    return bits;
}

// Stage row n of W (K elements, zero padded to 2 * P_pad) in shared memory;
// returns false (and records SS_ERR_DATA) if it holds a NaN or Inf.
template <typename T>
__device__ __forceinline__ bool stage_row_fp4(const T* __restrict__ w, int64_t K, int64_t len,
                                              float* srow) {
    __shared__ int bad;
    if (threadIdx.x == 0) bad = 0;
    __syncthreads();
    for (int64_t k = threadIdx.x; k < len; k += blockDim.x) {
        const float v = k < K ? to_f32<T>(w[k]) : 0.0f;
        if (!isfinite(v)) bad = 1;
        srow[k] = v;
    }
    __syncthreads();
    return bad == 0;
}

// Pass 1 of the weight compression: absolute maximum of the kept weights of
// every row, combined with atomicMax on the float bits (non-negative floats
// order as their bit patterns).
template <typename T>
__global__ void __launch_bounds__(kCompressThreads) fp4_weight_amax_kernel(
    const T* __restrict__ W, int64_t N, int64_t K, int keep, int group,
    unsigned int* __restrict__ amax_bits) {
    pdl_trigger();
    pdl_wait();
    extern __shared__ __align__(16) uint8_t smem_raw[];
    __shared__ float red[32];
    float* srow = reinterpret_cast<float*>(smem_raw);
    const int64_t n = blockIdx.x;
    const int64_t P = (K + 1) / 2;
    const int64_t P_pad = group ? (P + group - 1) / group * group : P;
    if (!stage_row_fp4<T>(W + n * K, K, 2 * P_pad, srow)) {
        if (threadIdx.x == 0) record_status(kErrData);
        return;
    }
    float a = 0.0f;
    if (group == 0) {
        for (int64_t k = threadIdx.x; k < K; k += blockDim.x) a = fmaxf(a, fabsf(srow[k]));
    } else {
        for (int64_t gi = threadIdx.x; gi < P_pad / group; gi += blockDim.x) {
            const uint32_t bits = kept_pairs(srow, gi * group, group, keep);
            for (int q = 0; q < group; ++q)
                if ((bits >> q) & 1u)
                    a = fmaxf(a, fmaxf(fabsf(srow[2 * (gi * group + q)]),
                                       fabsf(srow[2 * (gi * group + q) + 1])));
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = a;
    __syncthreads();
    if (threadIdx.x < 32) {
        a = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.0f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
        if (threadIdx.x == 0) atomicMax(amax_bits, __float_as_uint(a));
    }
}

// g = amax / 2688 in place (one thread).
__global__ void fp4_global_kernel(float* g) {
    pdl_trigger();
    pdl_wait();
    if (threadIdx.x == 0 && blockIdx.x == 0) g[0] = __fdiv_rn(g[0], 2688.0f);
}

// Pass 2: one CTA per (padded) row.  Sparse: prune pairs, slide them into
// windows of 4 pairs (ascending first fit), store 2 pairs per window in a
// shared row, then quantise it in blocks of 16 stored values.  Dense: the
// row itself in blocks of 16.  amax_bits holds pass 1's result.
template <typename T>
__global__ void __launch_bounds__(kCompressThreads) compress_weight_nvfp4_kernel(
    const T* __restrict__ W, int64_t N, int64_t K, int keep, int group, int64_t K_lift,
    int64_t K_lp, const unsigned int* __restrict__ amax_bits, uint8_t* __restrict__ Wv,
    uint8_t* __restrict__ Wm, uint8_t* __restrict__ Ws) {
    pdl_trigger();
    pdl_wait();
    extern __shared__ __align__(16) uint8_t smem_raw[];
    const int64_t n = blockIdx.x;
    const bool dense = group == 0;
    const int block = dense ? 16 : 32;         // lifted elements per scale
    const int64_t nblk = K_lp / block;
    if (n >= N) {  // padding row of the last 128-row scale / metadata tile
        for (int64_t j = threadIdx.x; j < nblk; j += blockDim.x) Ws[fp4_scale_offset(n, j, nblk)] = 0;
        if (!dense)
            for (int64_t b = threadIdx.x; b < K_lp / 16; b += blockDim.x)
                Wm[meta_offset(n, b, K_lp / 2)] = 0;
        return;
    }
    const float g = __fdiv_rn(__uint_as_float(*amax_bits), 2688.0f);
    const int64_t P = (K + 1) / 2;
    const int64_t P_pad = dense ? P : (P + group - 1) / group * group;
    const int64_t len = dense ? K_lp : 2 * P_pad;
    float* srow = reinterpret_cast<float*>(smem_raw);                       // len floats
    float* stored = srow + ((len + 3) / 4 * 4);                             // K_lp / 2 floats
    if (!stage_row_fp4<T>(W + n * K, K, len, srow)) return;  // pass 1 recorded it
    const float* vals = srow;
    if (!dense) {
        const int Nh = group / 2;
        uint8_t* kept = reinterpret_cast<uint8_t*>(stored + K_lp / 2);      // 2 bytes per group
        for (int64_t gi = threadIdx.x; gi < P_pad / group; gi += blockDim.x) {
            const uint32_t bits = kept_pairs(srow, gi * group, group, keep);
            kept[2 * gi] = static_cast<uint8_t>(bits & 0xFFu);
            kept[2 * gi + 1] = static_cast<uint8_t>(bits >> 8);
        }
        __syncthreads();
        // two windows per metadata byte
        for (int64_t pr = threadIdx.x; pr < K_lp / 16; pr += blockDim.x) {
            uint32_t meta = 0;
            for (int h = 0; h < 2; ++h) {
                const int64_t w = 2 * pr + h;
                uint32_t own = 0;
                int64_t pbase = 0;
                if (w < K_lift / 8) {
                    const int64_t gi = w / (Nh - 1);
                    const int j = static_cast<int>(w - gi * (Nh - 1));
                    const uint32_t kb = kept[2 * gi] | (static_cast<uint32_t>(kept[2 * gi + 1]) << 8);
                    own = window_bits(kb, Nh, j);
                    pbase = gi * group + 2 * j;
                }
                int i0, i1;
                window_indices(own, i0, i1);
                const bool k0 = (own >> i0) & 1u, k1 = (own >> i1) & 1u;
                stored[4 * w + 0] = k0 ? srow[2 * (pbase + i0)] : 0.0f;
                stored[4 * w + 1] = k0 ? srow[2 * (pbase + i0) + 1] : 0.0f;
                stored[4 * w + 2] = k1 ? srow[2 * (pbase + i1)] : 0.0f;
                stored[4 * w + 3] = k1 ? srow[2 * (pbase + i1) + 1] : 0.0f;
                meta |= static_cast<uint32_t>(i0 | (i1 << 2)) << (4 * h);
            }
            Wm[meta_offset(n, pr, K_lp / 2)] = static_cast<uint8_t>(meta);
        }
        __syncthreads();
        vals = stored;
    }
    // blocks of 16 values (stored values, or the dense row)
    const int64_t nval = dense ? K_lp : K_lp / 2;
    uint8_t* vrow = Wv + n * (nval / 2);
    for (int64_t b = threadIdx.x; b < nval / 16; b += blockDim.x) {
        float x[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) x[i] = vals[16 * b + i];
        const uint32_t sc = nvfp4_block<16>(x, g, vrow + 8 * b);
        Ws[fp4_scale_offset(n, b, nblk)] = static_cast<uint8_t>(sc);
    }
}

// L2 cache policies for the two passes over X: pass 1 keeps it resident for
// pass 2 (evict_last), pass 2 is its last use (evict_first).
__device__ __forceinline__ uint4 ldg_policy(const void* p, uint64_t pol) {
    uint4 v;
    asm volatile("ld.global.nc.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p), "l"(pol));
    return v;
}

__device__ __forceinline__ uint2 ldg_policy2(const void* p, uint64_t pol) {
    uint2 v;
    asm volatile("ld.global.nc.L2::cache_hint.v2.u32 {%0, %1}, [%2], %3;"
                 : "=r"(v.x), "=r"(v.y)
                 : "l"(p), "l"(pol));
    return v;
}

// NVFP4 activation, pass 1: the absolute maximum of the whole tensor X
// (M * K elements, contiguous), combined with atomicMax on the float bits
// into *amax_bits, which the caller has zeroed.  The global scale is per
// tensor (LLM-Compressor compression schemes, NVFP4 row); with no
// calibration set it is taken from this call's activation.
template <typename T>
__global__ void __launch_bounds__(256) fp4_act_amax_kernel(const T* __restrict__ X, int64_t n,
                                                           unsigned int* __restrict__ amax_bits) {
    pdl_trigger();
    pdl_wait();
    __shared__ float red[8];
    constexpr int kPer = 16 / sizeof(T);  // elements per 16-byte load
    constexpr int kUnroll = 8;            // loads in flight per thread
    const int64_t nv = n / kPer;
    const uint4* xv = reinterpret_cast<const uint4*>(X);  // X is 16-byte aligned
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    const uint64_t keep = l2_policy_evict_last();
    float a = 0.0f;
    int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    for (; i + (kUnroll - 1) * stride < nv; i += kUnroll * stride) {
        uint4 v[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) v[u] = ldg_policy(xv + i + u * stride, keep);
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) a = fmaxf(a, chunk_absmax<T>(v[u]));
    }
    for (; i < nv; i += stride) a = fmaxf(a, chunk_absmax<T>(ldg_policy(xv + i, keep)));
    const int64_t t = nv * kPer + static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (t < n) a = fmaxf(a, fabsf(to_f32<T>(X[t])));  // the tail (< kPer elements)
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = a;
    __syncthreads();
    if (threadIdx.x < 32) {
        a = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.0f;
#pragma unroll
        for (int o = 4; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
        if (threadIdx.x == 0) atomicMax(amax_bits, __float_as_uint(a));
    }
}

// Zero one 32-bit word (the amax accumulator of the next pass).
__global__ void zero_word_kernel(unsigned int* p) {
    pdl_trigger();
    pdl_wait();
    if (threadIdx.x == 0 && blockIdx.x == 0) *p = 0u;
}

// The 8 lifted elements of window wi (8 consecutive inputs from src0; zero
// past K and for padding windows, src0 < 0).
template <typename T>
__device__ __forceinline__ void load_window8(const T* __restrict__ x, int src0, int K,
                                             uint64_t pol, float (&v)[8]) {
    bool done = false;
    if (src0 >= 0 && src0 + 8 <= K) {
        const uintptr_t addr = reinterpret_cast<uintptr_t>(x + src0);
        if constexpr (sizeof(T) == 2) {
            uint32_t u[4];
            if ((addr & 15u) == 0) {
                const uint4 q = ldg_policy(x + src0, pol);
                u[0] = q.x, u[1] = q.y, u[2] = q.z, u[3] = q.w;
                done = true;
            } else if ((addr & 7u) == 0) {
                const uint2 q0 = ldg_policy2(x + src0, pol);
                const uint2 q1 = ldg_policy2(x + src0 + 4, pol);
                u[0] = q0.x, u[1] = q0.y, u[2] = q1.x, u[3] = q1.y;
                done = true;
            }
            if (done) {
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    v[2 * h] = __uint_as_float(u[h] << 16);
                    v[2 * h + 1] = __uint_as_float(u[h] & 0xFFFF0000u);
                }
            }
        } else {
            if ((addr & 15u) == 0) {
                const uint4 q0 = ldg_policy(x + src0, pol);
                const uint4 q1 = ldg_policy(x + src0 + 4, pol);
                v[0] = __uint_as_float(q0.x), v[1] = __uint_as_float(q0.y);
                v[2] = __uint_as_float(q0.z), v[3] = __uint_as_float(q0.w);
                v[4] = __uint_as_float(q1.x), v[5] = __uint_as_float(q1.y);
                v[6] = __uint_as_float(q1.z), v[7] = __uint_as_float(q1.w);
                done = true;
            }
        }
    }
    if (!done) {
#pragma unroll
        for (int t = 0; t < 8; ++t) {
            const int src = src0 + t;
            v[t] = (src0 >= 0 && src < K) ? to_f32<T>(x[src]) : 0.0f;
        }
    }
}

// NVFP4 activation, pass 2: one warp per token row at a time, lane l taking
// the blocks of kBlock lifted elements l, l + 32, ... (kBlock / 8 windows of
// 8 lifted elements each).  g = amax / 2688 from pass 1; the block scale
// s = UE4M3(a / (6 g)), d = s g, codes E2M1(x * (1 / d)) (the reciprocal
// correctly rounded, as 1 / d).  kNh: the pattern's half group (pair windows
// slide by 2 pairs, Nh - 1 windows per group of 2 Nh pairs); 0 or 2 for the
// identity map (dense, pair 2:4).  Warps of the padding rows
// (M <= m < M_pad) only zero their scales.
template <typename T, int kBlock, int kNh>
__global__ void __launch_bounds__(256) quant_nvfp4_act_kernel(
    const T* __restrict__ X, int M, int K, int K_lift, int K_lp,
    const unsigned int* __restrict__ amax_bits, uint8_t* __restrict__ Xv,
    uint8_t* __restrict__ Xs) {
    pdl_trigger();
    pdl_wait();
    constexpr int kWin = kBlock / 8;  // windows per block
    const int lane = threadIdx.x & 31;
    const int warps = static_cast<int>(gridDim.x * (blockDim.x >> 5));
    const int M_pad = (M + 127) / 128 * 128;
    const int nblk = K_lp / kBlock;
    const float g = __fdiv_rn(__uint_as_float(__ldg(amax_bits)), 2688.0f);
    const float g6 = __fmul_rn(6.0f, g);
    const uint64_t last = l2_policy_evict_first();
    for (int m = static_cast<int>(blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)); m < M_pad;
         m += warps) {
        if (m >= M) {
            for (int j = lane; j < nblk; j += 32) Xs[fp4_scale_offset(m, j, nblk)] = 0;
            continue;
        }
        const T* x = X + static_cast<int64_t>(m) * K;
        uint8_t* vrow = Xv + static_cast<int64_t>(m) * (K_lp / 2);
        for (int b = lane; b < nblk; b += 32) {
            float v[kWin][8];
#pragma unroll
            for (int q = 0; q < kWin; ++q) {
                const int wi = b * kWin + q;
                int src0;
                if constexpr (kNh <= 2) {
                    src0 = 8 * wi;
                } else {
                    const int gi = wi / (kNh - 1), j = wi - gi * (kNh - 1);
                    src0 = 8 * wi < K_lift ? 2 * (gi * 2 * kNh + 2 * j) : -1;
                }
                load_window8<T>(x, src0, K, last, v[q]);
            }
            float a = 0.0f;
#pragma unroll
            for (int q = 0; q < kWin; ++q)
#pragma unroll
                for (int t = 0; t < 8; ++t) a = fmaxf(a, fabsf(v[q][t]));
            uint32_t sc = 0;
            float inv = 0.0f;
            if (g != 0.0f) {
                sc = ue4m3_code(__fdiv_rn(a, g6));
                const float d = __fmul_rn(ue4m3_value(sc), g);
                inv = d == 0.0f ? 0.0f : __frcp_rn(d);
            }
            uint32_t w[kWin];
#pragma unroll
            for (int q = 0; q < kWin; ++q) {
                uint32_t word = 0;
                if (inv != 0.0f) {
#pragma unroll
                    for (int h = 0; h < 4; ++h)
                        word |= e2m1x2(__fmul_rn(v[q][2 * h], inv), __fmul_rn(v[q][2 * h + 1], inv))
                                << (8 * h);
                }
                w[q] = word;
            }
            if constexpr (kWin == 4)
                __stcs(reinterpret_cast<uint4*>(vrow) + b, make_uint4(w[0], w[1], w[2], w[3]));
            else
                __stcs(reinterpret_cast<uint2*>(vrow) + b, make_uint2(w[0], w[1]));
            Xs[fp4_scale_offset(m, b, nblk)] = static_cast<uint8_t>(sc);
        }
    }
}

}  // namespace ss
