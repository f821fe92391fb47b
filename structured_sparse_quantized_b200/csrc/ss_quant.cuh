// ss_quant.cuh -- memory-bound activation kernels.
//
//  quant_lift_reg_kernel    fused per-token absmax, quantisation and activation
//                           lifting for bf16 rows of up to 16384 elements: the
//                           row is read once, into registers (1, 2 or 4 warps
//                           per row) (SlideSparse, 66bd.net: lifting is an
//                           index map fused into the per-token quant kernel;
//                           SlideSparse write-up, omica.com.cn, 3.2: one kernel
//                           computes the absmax, the scale, the clamped
//                           quantised values, the window remap and the packed
//                           stores, iterating over output windows).
//  quant_lift_warp_kernel   the same for any other row (fp32 rows, longer or
//                           ragged K): pass 1 streams the row with 16-byte loads
//                           for its absmax, pass 2 streams it again (from L2)
//                           and quantises.
//  prune_act_stream_kernel  online 2:4 prune + compress of bf16 rows for the
//                           8-bit tiers, single pass: rows stream through shared
//                           memory, the kept half stays in registers ("add 2:4
//                           or drop a precision tier?", paper-daily 2610.28947,
//                           sections 1 and 2.3).
//  prune_act_warp_kernel    the same for other rows and for the bf16 tier, in
//                           two passes like quant_lift_warp_kernel.
//  lift_bf16_kernel         the lift alone, for the bf16 tier (no scale).
//
// One warp (or a few) per token row, no block-wide barrier on the path;
// outputs leave in 16-byte stores -- four lifted windows (or sixteen identity
// bytes) per store for the lift, eight 2:4 groups (16 value bytes + one 32-bit
// nibble word) per step for the prune.
#pragma once

#include "ss_common.cuh"

namespace ss {

// Largest |v| over the eight values of a 16-byte chunk.
template <typename T>
__device__ __forceinline__ float chunk_absmax(const uint4& v);
template <>
__device__ __forceinline__ float chunk_absmax<__nv_bfloat16>(const uint4& v) {
    // max of |bf16| pairs is exact in bf16; one packed op per two values
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
    __nv_bfloat162 m = __habs2(h[0]);
    m = __hmax2(m, __habs2(h[1]));
    m = __hmax2(m, __habs2(h[2]));
    m = __hmax2(m, __habs2(h[3]));
    return fmaxf(__low2float(m), __high2float(m));
}
template <>
__device__ __forceinline__ float chunk_absmax<float>(const uint4& v) {
    return fmaxf(fmaxf(fabsf(__uint_as_float(v.x)), fabsf(__uint_as_float(v.y))),
                 fmaxf(fabsf(__uint_as_float(v.z)), fabsf(__uint_as_float(v.w))));
}

// INT8 code of x * inv as the low byte of a 32-bit word: the product is
// rounded to fp32 and then to the nearest integer (ties to even) by adding
// 1.5 * 2^23, after which the integer sits in the low mantissa bits -- the
// IEEE round-to-nearest-even of the fp32 product, without the low-throughput
// float-to-int conversion unit.  No clamp is needed: |x| <= a and
// inv = RN(127 / a) give |x * inv| <= 127 (1 + 2^-24), which rounds into
// [-127, 127].
__device__ __forceinline__ uint32_t int8_code(float x, float inv) {
    return __float_as_uint(__fadd_rn(__fmul_rn(x, inv), 12582912.0f));  // low byte = code
}

// Quantise sixteen values into sixteen bytes (byte j = value j).
template <bool kInt8>
__device__ __forceinline__ uint4 quant16(const float (&f)[16], float inv) {
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        if constexpr (kInt8) {
            const uint32_t b0 = int8_code(f[4 * j], inv), b1 = int8_code(f[4 * j + 1], inv);
            const uint32_t b2 = int8_code(f[4 * j + 2], inv), b3 = int8_code(f[4 * j + 3], inv);
            // bytes b0.0, b1.0, b2.0, b3.0
            w[j] = __byte_perm(__byte_perm(b0, b1, 0x0040), __byte_perm(b2, b3, 0x0040), 0x5410);
        } else {
            const float2 lo = make_float2(__fmul_rn(f[4 * j], inv), __fmul_rn(f[4 * j + 1], inv));
            const float2 hi =
                make_float2(__fmul_rn(f[4 * j + 2], inv), __fmul_rn(f[4 * j + 3], inv));
            const uint32_t l = __nv_cvt_float2_to_fp8x2(lo, __NV_SATFINITE, __NV_E4M3);
            const uint32_t h = __nv_cvt_float2_to_fp8x2(hi, __NV_SATFINITE, __NV_E4M3);
            w[j] = (l & 0xFFFFu) | (h << 16);
        }
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

// Keep the two largest |v| of a group of four (ties keep the lower index);
// returns the two local indices in ascending order.  For j < i, j beats i
// iff |v_j| >= |v_i|; a position is kept iff fewer than two others beat it.
__device__ __forceinline__ void top2_of4(const float* v, int& i0, int& i1) {
    const float a0 = fabsf(v[0]), a1 = fabsf(v[1]), a2 = fabsf(v[2]), a3 = fabsf(v[3]);
    const int g01 = a0 >= a1, g02 = a0 >= a2, g03 = a0 >= a3;
    const int g12 = a1 >= a2, g13 = a1 >= a3, g23 = a2 >= a3;
    const int r0 = (1 - g01) + (1 - g02) + (1 - g03);
    const int r1 = g01 + (1 - g12) + (1 - g13);
    const int r2 = g02 + g12 + (1 - g23);
    const bool k0 = r0 < 2, k1 = r1 < 2, k2 = r2 < 2;  // exactly two are kept
    i0 = k0 ? 0 : (k1 ? 1 : 2);
    i1 = k0 ? (k1 ? 1 : (k2 ? 2 : 3)) : (k1 ? (k2 ? 2 : 3) : 3);
}

// top2_of4 on four bf16 values given as two 32-bit words (element i in bits
// 16(i%2) of word i/2), in integer arithmetic: key_i = |x_i| bits * 4 +
// (3 - i) orders by magnitude and, among equal magnitudes, by lower index --
// the same order as top2_of4 for every non-NaN input (|bf16| bit patterns
// are monotone in the value).  Returns the two kept bf16 values, lower index
// in the low half, picked with one byte permute.
__device__ __forceinline__ uint32_t top2_of4_bf16(uint32_t lo, uint32_t hi, int& i0, int& i1,
                                                  uint32_t& top) {
    const uint32_t k0 = (lo & 0x7FFFu) * 4u + 3u;
    const uint32_t k1 = ((lo >> 16) & 0x7FFFu) * 4u + 2u;
    const uint32_t k2 = (hi & 0x7FFFu) * 4u + 1u;
    const uint32_t k3 = ((hi >> 16) & 0x7FFFu) * 4u;
    const uint32_t a = max(k0, k1), b = min(k0, k1), c = max(k2, k3), d = min(k2, k3);
    const uint32_t first = max(a, c);                   // the largest key
    const uint32_t second = max(min(a, c), max(b, d));  // the second largest
    top = first;  // |x| bits of the group's largest magnitude, times 4, plus a tie tag
    const int ia = static_cast<int>((first & 3u) ^ 3u), ib = static_cast<int>((second & 3u) ^ 3u);
    i0 = min(ia, ib);
    i1 = max(ia, ib);
    // bytes 2 i0, 2 i0 + 1 -> low half; 2 i1, 2 i1 + 1 -> high half
    const uint32_t sel = static_cast<uint32_t>(i0) * 0x22u + static_cast<uint32_t>(i1) * 0x2200u + 0x1010u;
    return __byte_perm(lo, hi, sel);
}

__device__ __forceinline__ uint32_t top2_of4_bf16(uint32_t lo, uint32_t hi, int& i0, int& i1) {
    uint32_t top;
    return top2_of4_bf16(lo, hi, i0, i1, top);
}

// top2_of4_bf16 for the streaming prune kernel, which is bound by the
// integer ALU pipe: the keys are built with multiply-adds (FMA pipe) by the
// multipliers c2 = 2 and c17 = 2^17, which the caller passes in registers the
// compiler cannot fold.  key_i = |x_i| bits in bits 31..17, tie tag 3 - i in
// bits 1..0 (x_0 * 2^17 drops its sign bit and x_1; (x_1's half) * 2 drops
// its sign bit): the same order as top2_of4_bf16.  Returns the kept pair
// (lower index in the low half), the nibble i0 | i1 << 2 and the largest key.
__device__ __forceinline__ uint32_t top2_of4_bf16_keys(uint32_t lo, uint32_t hi, uint32_t c2,
                                                       uint32_t c17, uint32_t& nib,
                                                       uint32_t& top) {
    const uint32_t k0 = lo * c17 + 3u;
    const uint32_t k1 = (lo & 0xFFFF0000u) * c2 + 2u;
    const uint32_t k2 = hi * c17 + 1u;
    const uint32_t k3 = (hi & 0xFFFF0000u) * c2;
    const uint32_t a = max(k0, k1), b = min(k0, k1), c = max(k2, k3), d = min(k2, k3);
    const uint32_t first = max(a, c);
    const uint32_t second = max(min(a, c), max(b, d));
    top = first;
    const uint32_t ia = (first & 3u) ^ 3u, ib = (second & 3u) ^ 3u;
    const uint32_t i0 = min(ia, ib), i1 = max(ia, ib);
    nib = i1 * 4u + i0;
    return __byte_perm(lo, hi, i0 * 0x22u + i1 * 0x2200u + 0x1010u);
}

// Value at local index i (0..3) of a group, without indexing registers
// dynamically.
__device__ __forceinline__ float pick4(const float* v, int i) {
    return i == 0 ? v[0] : (i == 1 ? v[1] : (i == 2 ? v[2] : v[3]));
}

template <bool kInt8>
__device__ __forceinline__ uint32_t quantize_pair(float x0, float x1, float inv) {
    if constexpr (kInt8) {
        return __byte_perm(int8_code(x0, inv), int8_code(x1, inv), 0x0040) & 0xFFFFu;
    } else {
        return __nv_cvt_float2_to_fp8x2(make_float2(__fmul_rn(x0, inv), __fmul_rn(x1, inv)),
                                        __NV_SATFINITE, __NV_E4M3) &
               0xFFFFu;
    }
}

// ---------------------------------------------------------------------------
// Warp-per-row kernels.  One warp owns one token row; no block-wide barrier
// is on the path, so many rows are in flight per SM.  Pass 1 streams the row
// (16-byte loads, four in flight per lane) for its absmax; pass 2 streams it
// again -- the row was just read, so this comes from L2 -- and quantises.
// ---------------------------------------------------------------------------
constexpr int kWarpRowThreads = 256;  // 8 rows per CTA

// Sixteen inputs at k0 straight from global memory (zero past K); `vec`
// means the row is 16-byte aligned with K * sizeof(T) a multiple of 16.
template <typename T>
__device__ __forceinline__ void gload16(const T* __restrict__ x, int k0, int K, bool vec,
                                        float (&f)[16]) {
    if (vec && k0 + 16 <= K) {
        if constexpr (sizeof(T) == 2) {
            const uint4* p = reinterpret_cast<const uint4*>(x + k0);
            const uint4 v0 = __ldg(p), v1 = __ldg(p + 1);
            const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                f[2 * j] = __uint_as_float(w[j] << 16);
                f[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
            }
        } else {
            const float4* p = reinterpret_cast<const float4*>(x + k0);
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const float4 v = __ldg(p + h);
                f[4 * h] = v.x;
                f[4 * h + 1] = v.y;
                f[4 * h + 2] = v.z;
                f[4 * h + 3] = v.w;
            }
        }
    } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) f[j] = (k0 + j < K) ? to_f32<T>(x[k0 + j]) : 0.0f;
    }
}

template <typename T>
__device__ __forceinline__ float warp_row_absmax(const T* __restrict__ x, int K, bool vec,
                                                 int lane) {
    float a = 0.0f;
    if (vec) {
        constexpr int kVec = 16 / sizeof(T);
        const int nv = K / kVec;
        const uint4* xv = reinterpret_cast<const uint4*>(x);
        int i = lane;
        for (; i + 96 < nv; i += 128) {
            const uint4 v0 = __ldg(xv + i), v1 = __ldg(xv + i + 32);
            const uint4 v2 = __ldg(xv + i + 64), v3 = __ldg(xv + i + 96);
            a = fmaxf(a, fmaxf(fmaxf(chunk_absmax<T>(v0), chunk_absmax<T>(v1)),
                               fmaxf(chunk_absmax<T>(v2), chunk_absmax<T>(v3))));
        }
        for (; i < nv; i += 32) a = fmaxf(a, chunk_absmax<T>(__ldg(xv + i)));
    } else {
        for (int k = lane; k < K; k += 32) a = fmaxf(a, fabsf(to_f32<T>(x[k])));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    return a;
}

template <typename T, bool kInt8>
__global__ void __launch_bounds__(kWarpRowThreads) quant_lift_warp_kernel(
    const T* __restrict__ X, int64_t M, int64_t K64, int Nh, int64_t K_lift64, int64_t K_lp64,
    int q_stride, uint8_t* __restrict__ Xq, float* __restrict__ s_x) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    pdl_trigger();
    pdl_wait();
    const int64_t m = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + warp;
    if (m >= M) return;
    const int K = static_cast<int>(K64);
    const int K_lift = static_cast<int>(K_lift64);
    const int K_lp = static_cast<int>(K_lp64);
    const T* x = X + m * K64;
    const bool vec = (K * static_cast<int>(sizeof(T))) % 16 == 0 &&
                     (reinterpret_cast<uintptr_t>(X) & 15) == 0;
    const float a = warp_row_absmax<T>(x, K, vec, lane);
    float inv, s;
    scale_from_absmax<kInt8>(a, inv, s);
    if (lane == 0) s_x[m] = s;
    uint4* out = reinterpret_cast<uint4*>(Xq + m * K_lp64);
    const int n_chunks = K_lp / 16;  // 16 output bytes per chunk
    if (Nh <= 2) {                   // identity map (dense, 2:4)
        int c = lane;
        for (; c + 32 < n_chunks; c += 64) {  // two chunks of loads in flight
            float f0[16], f1[16];
            gload16<T>(x, c * 16, K, vec, f0);
            gload16<T>(x, (c + 32) * 16, K, vec, f1);
            __stcs(out + c, quant16<kInt8>(f0, inv));
            __stcs(out + c + 32, quant16<kInt8>(f1, inv));
        }
        if (c < n_chunks) {
            float f[16];
            gload16<T>(x, c * 16, K, vec, f);
            __stcs(out + c, quant16<kInt8>(f, inv));
        }
        return;
    }
    // sliding patterns: quantised byte row of this warp, then window gather
    uint4* qrow = reinterpret_cast<uint4*>(smem_raw + warp * q_stride);
    const int q_chunks = ((K_lift / (4 * (Nh - 1))) * 2 * Nh + 15) / 16;
    {
        int c = lane;
        for (; c + 32 < q_chunks; c += 64) {  // two chunks of loads in flight
            float f0[16], f1[16];
            gload16<T>(x, c * 16, K, vec, f0);
            gload16<T>(x, (c + 32) * 16, K, vec, f1);
            qrow[c] = quant16<kInt8>(f0, inv);
            qrow[c + 32] = quant16<kInt8>(f1, inv);
        }
        if (c < q_chunks) {
            float f[16];
            gload16<T>(x, c * 16, K, vec, f);
            qrow[c] = quant16<kInt8>(f, inv);
        }
    }
    __syncwarp();
    const uint16_t* q16 = reinterpret_cast<const uint16_t*>(qrow);
    const uint32_t n_win = static_cast<uint32_t>(K_lift / 4);
    const uint32_t per_group = static_cast<uint32_t>(Nh - 1);
    for (int c = lane; c < n_chunks; c += 32) {
        uint32_t win = static_cast<uint32_t>(c) * 4u;
        uint32_t g = win / per_group;
        uint32_t j = win - g * per_group;
        uint32_t w[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint32_t word = 0;
            if (win < n_win) {
                const uint32_t half = Nh * g + j;  // base / 2, base = 2Nh g + 2j
                word = static_cast<uint32_t>(q16[half]) |
                       (static_cast<uint32_t>(q16[half + 1]) << 16);
            }
            w[i] = word;
            ++win;
            if (++j == per_group) {
                j = 0;
                ++g;
            }
        }
        __stcs(out + c, make_uint4(w[0], w[1], w[2], w[3]));
    }
}

// Online 2:4 prune + compress of one token row per warp.  The 8-bit tiers
// take the row absmax first and quantise the kept values; the bf16 tier
// (kQ = kQBf16) keeps them as bf16 (two bytes each, no scale, one pass).
template <typename T, int kQ>
__global__ void __launch_bounds__(kWarpRowThreads) prune_act_warp_kernel(
    const T* __restrict__ X, int64_t M, int64_t K64, int64_t K_lp64, uint8_t* __restrict__ Xv,
    uint8_t* __restrict__ Xm, float* __restrict__ s_x) {
    constexpr bool kInt8 = kQ == kQInt8;
    constexpr bool kBf16 = kQ == kQBf16;
    pdl_trigger();
    pdl_wait();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t m = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + warp;
    const int64_t M_pad = (M + 127) / 128 * 128;
    if (m >= M_pad) return;
    // the 4 selector bytes of step st (one word; the bf16 tier stores its two
    // halves in rows m and m ^ 8, see meta_offset_i16)
    auto put_meta = [&](int64_t st, uint32_t nibs) {
        if constexpr (kBf16) {
            __stcs(reinterpret_cast<uint16_t*>(Xm + meta_offset_i16(m, 4 * st, K_lp64)),
                   static_cast<uint16_t>(nibs & 0xFFFFu));
            __stcs(reinterpret_cast<uint16_t*>(Xm + meta_offset_i16(m, 4 * st + 2, K_lp64)),
                   static_cast<uint16_t>(nibs >> 16));
        } else {
            __stcs(reinterpret_cast<uint32_t*>(Xm + meta_offset(m, 4 * st, K_lp64)), nibs);
        }
    };
    if (m >= M) {  // padding row of the last 128-row metadata tile
        for (int64_t st = lane; st < K_lp64 / 32; st += 32) put_meta(st, 0u);
        return;
    }
    const int K = static_cast<int>(K64);
    const int K_lp = static_cast<int>(K_lp64);
    const T* x = X + m * K64;
    const bool vec = (K * static_cast<int>(sizeof(T))) % 16 == 0 &&
                     (reinterpret_cast<uintptr_t>(X) & 15) == 0;
    float inv = 0.0f;
    if constexpr (!kBf16) {
        const float a = warp_row_absmax<T>(x, K, vec, lane);
        float s;
        scale_from_absmax<kInt8>(a, inv, s);
        if (lane == 0) s_x[m] = s;
    }
    // One step = 8 groups of 4 = 32 inputs -> 16 values (16 bytes, 32 for
    // bf16) + 4 nibble bytes.
    constexpr int kVq = kBf16 ? 2 : 1;  // uint4 of values per step
    uint4* vout = reinterpret_cast<uint4*>(Xv + m * (K_lp64 / 2) * (kBf16 ? 2 : 1));
    const int n_steps = K_lp / 32;
    for (int st = lane; st < n_steps; st += 32) {
        if constexpr (sizeof(T) == 2) {
            if (vec && st * 32 + 32 <= K) {  // bf16: select on the raw words
                const uint4* p = reinterpret_cast<const uint4*>(x) + 4 * st;
                const uint4 c0 = __ldg(p), c1 = __ldg(p + 1), c2 = __ldg(p + 2), c3 = __ldg(p + 3);
                const uint32_t w[16] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w,
                                        c2.x, c2.y, c2.z, c2.w, c3.x, c3.y, c3.z, c3.w};
                uint32_t vals[8];
                uint32_t nibs = 0;
#pragma unroll
                for (int gi = 0; gi < 8; ++gi) {
                    int i0, i1;
                    const uint32_t kept = top2_of4_bf16(w[2 * gi], w[2 * gi + 1], i0, i1);
                    if constexpr (kBf16) {
                        vals[gi] = kept;
                    } else {
                        const uint32_t q = quantize_pair<kInt8>(
                            __uint_as_float(kept << 16), __uint_as_float(kept & 0xFFFF0000u), inv);
                        if (gi & 1)
                            vals[gi >> 1] |= q << 16;
                        else
                            vals[gi >> 1] = q;
                    }
                    nibs |= static_cast<uint32_t>(i0 | (i1 << 2)) << (4 * gi);
                }
#pragma unroll
                for (int v = 0; v < kVq; ++v)
                    __stcs(vout + kVq * st + v,
                           make_uint4(vals[4 * v], vals[4 * v + 1], vals[4 * v + 2], vals[4 * v + 3]));
                put_meta(st, nibs);
                continue;
            }
        }
        float f[32];
        gload16<T>(x, st * 32, K, vec, *reinterpret_cast<float(*)[16]>(f));
        gload16<T>(x, st * 32 + 16, K, vec, *reinterpret_cast<float(*)[16]>(f + 16));
        uint32_t vals[8];
        uint32_t nibs = 0;
#pragma unroll
        for (int gi = 0; gi < 8; ++gi) {
            int i0, i1;
            top2_of4(f + 4 * gi, i0, i1);
            if constexpr (kBf16) {
                vals[gi] = bf16_bits(pick4(f + 4 * gi, i0)) |
                           (bf16_bits(pick4(f + 4 * gi, i1)) << 16);
            } else {
                const uint32_t q =
                    quantize_pair<kInt8>(pick4(f + 4 * gi, i0), pick4(f + 4 * gi, i1), inv);
                if (gi & 1)
                    vals[gi >> 1] |= q << 16;
                else
                    vals[gi >> 1] = q;
            }
            nibs |= static_cast<uint32_t>(i0 | (i1 << 2)) << (4 * gi);
        }
#pragma unroll
        for (int v = 0; v < kVq; ++v)
            __stcs(vout + kVq * st + v,
                   make_uint4(vals[4 * v], vals[4 * v + 1], vals[4 * v + 2], vals[4 * v + 3]));
        put_meta(st, nibs);
    }
}

// Single-pass online 2:4 prune of bf16 rows (8-bit tiers), streamed through
// shared memory.  A row is split into kWpr chunks of C = K / kWpr elements
// (C a multiple of 32, at most kPruneChunkMax); the kWpr warps of a row slot
// each take one chunk.  Each warp owns kPruneSlots shared-memory slots and keeps the
// 1-D bulk copies of its next chunks in flight while it works on the current
// one, so X is read from HBM once at full overlap:
//   - select: lane l takes the 32-element steps l, l + 32, ... of the chunk
//     (8 groups of 4 each) from shared memory, keeps the top-2 of every group
//     in registers as bf16 pairs, and the nibbles;
//   - the row absmax is the largest kept magnitude (the largest element of
//     every group is kept), combined across the row's warps through shared
//     memory;
//   - quantise the kept values from registers and store values and nibbles.
// Steps past K up to K_lp are groups of zeros: values 0, nibble 0x4.  Rows
// are taken in a grid-stride loop; padding rows (M <= m < M_pad) only zero
// their metadata.
constexpr int kPruneChunkMax = 4096;  // elements per chunk (8 KB of bf16)
constexpr int kPruneSlots = 3;
constexpr int kPruneSmem = 8 * kPruneSlots * kPruneChunkMax * 2;  // 8 warps

// kFull: every warp's chunk is exactly kSteps steps per lane and K_lp = K
// (no bounds test on the loads, no padding steps).  `one` is 1: the
// multipliers built from it are opaque to the compiler, so that products
// with them stay multiply-adds on the FMA pipe.
template <int kQ, int kSteps, int kWpr, bool kFull>
__global__ void __launch_bounds__(kWarpRowThreads, 1) prune_act_stream_kernel(
    const __nv_bfloat16* __restrict__ X, int M, int K, int K_lp, uint8_t* __restrict__ Xv,
    uint8_t* __restrict__ Xm, float* __restrict__ s_x, uint32_t one) {
    constexpr bool kInt8 = kQ == kQInt8;
    const uint32_t c2 = one << 1, c16 = one << 4, c17 = one << 17;
    const uint32_t c65536 = one << 16;
    constexpr int kRowsPerCta = kWarpRowThreads / (32 * kWpr);
    extern __shared__ __align__(16) uint8_t smem_raw[];
    __shared__ uint64_t full[8][kPruneSlots];
    __shared__ float part[2][kRowsPerCta][kWpr];
    __shared__ int abort_flag_storage;
    volatile int* abort_flag = &abort_flag_storage;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int slot = warp / kWpr, sub = warp % kWpr;
    const int chunk = K / kWpr;           // elements of this warp's chunk
    const int chunk_steps = chunk / 32;   // full steps in the chunk
    const int n_steps = K_lp / 32;        // steps of a row (K and its padding)
    const int M_pad = (M + 127) / 128 * 128;
    const int rows_total = static_cast<int>(gridDim.x) * kRowsPerCta;
    uint8_t* my_smem = smem_raw + warp * (kPruneSlots * kPruneChunkMax * 2);
    if (threadIdx.x == 0) *abort_flag = 0;
    if (lane == 0) {
        for (int b = 0; b < kPruneSlots; ++b) mbar_init(&full[warp][b], 1);
        fence_barrier_init();
    }
    __syncthreads();
    pdl_trigger();
    pdl_wait();
    const int m0 = static_cast<int>(blockIdx.x) * kRowsPerCta + slot;
    // the copy of this warp's chunk of row m into buffer b
    uint32_t pending = 0;  // buffers with a copy in flight (lane 0's view)
    bool ok = true;
    auto issue = [&](int m, int b) {
        if (m < M && ok && lane == 0) {
            fence_async_shared();  // this warp's reads of the buffer come first
            pending |= 1u << b;
            mbar_arrive_expect_tx(&full[warp][b], static_cast<uint32_t>(chunk * 2));
            bulk_load_1d(my_smem + b * (kPruneChunkMax * 2),
                         X + static_cast<int64_t>(m) * K + static_cast<int64_t>(sub) * chunk,
                         static_cast<uint32_t>(chunk * 2), &full[warp][b]);
        }
    };
#pragma unroll
    for (int b = 0; b < kPruneSlots - 1; ++b) issue(m0 + b * rows_total, b);
    int it = 0;
    for (int m = m0; m < M_pad; m += rows_total, ++it) {
        const int b = it % kPruneSlots;
        // the slot of item it + kPruneSlots - 1 was last read in iteration it - 1
        __syncwarp();
        issue(m + (kPruneSlots - 1) * rows_total, (it + kPruneSlots - 1) % kPruneSlots);
        if (m >= M) {  // padding row of the last 128-row metadata tile
            for (int st = sub * 32 + lane; st < n_steps; st += 32 * kWpr)
                __stcs(reinterpret_cast<uint32_t*>(Xm + meta_offset(m, 4 * st, K_lp)), 0u);
            continue;
        }
        const bool got = ok && mbar_wait(&full[warp][b],
                                         static_cast<uint32_t>((it / kPruneSlots) & 1), abort_flag);
        if (!__all_sync(0xffffffffu, got)) ok = false;
        if (got) pending &= ~(1u << b);
        const uint4* c4s = reinterpret_cast<const uint4*>(my_smem + b * (kPruneChunkMax * 2));
        uint32_t kept[kSteps][8];
        uint32_t nib[kSteps];
        // the largest selection key (|bf16| bits << 17 + tie tag): |bf16| bit
        // patterns order as the magnitudes, and the largest of every group is kept
        uint32_t amax_key = 0;
#pragma unroll
        for (int i = 0; i < kSteps; ++i) {
            const int ls = 32 * i + lane;  // step within the chunk
            uint32_t w[16];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint4 v = (kFull || ls < chunk_steps) ? c4s[4 * ls + j]
                                                             : make_uint4(0u, 0u, 0u, 0u);
                w[4 * j] = v.x, w[4 * j + 1] = v.y, w[4 * j + 2] = v.z, w[4 * j + 3] = v.w;
            }
            // the nibbles of groups 7 .. 0, Horner-style in multiply-adds
            uint32_t nibs = 0;
#pragma unroll
            for (int gi = 7; gi >= 0; --gi) {
                uint32_t top, n;
                kept[i][gi] = top2_of4_bf16_keys(w[2 * gi], w[2 * gi + 1], c2, c17, n, top);
                amax_key = max(amax_key, top);
                nibs = nibs * c16 + n;
            }
            nib[i] = nibs;  // steps past the chunk: zeros, indices 0, 1
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
            amax_key = max(amax_key, __shfl_xor_sync(0xffffffffu, amax_key, o));
        float a = __uint_as_float((amax_key >> 17) << 16);
        if constexpr (kWpr > 1) {
            if (lane == 0) part[it & 1][slot][sub] = a;
            named_bar_sync(1 + slot, 32 * kWpr);
#pragma unroll
            for (int w = 0; w < kWpr; ++w) a = fmaxf(a, part[it & 1][slot][w]);
        }
        float inv, s;
        scale_from_absmax<kInt8>(a, inv, s);
        if (lane == 0 && sub == 0) s_x[m] = s;
        // this lane's first step; a step 32 further is 16 value bytes x 32 and
        // eight 2 KB metadata tiles further
        const int st0 = sub * chunk_steps + lane;
        uint4* vout = reinterpret_cast<uint4*>(Xv + static_cast<int64_t>(m) * (K_lp / 2)) + st0;
        uint32_t* mout = reinterpret_cast<uint32_t*>(Xm + meta_offset(m, 4 * st0, K_lp));
#pragma unroll
        for (int i = 0; i < kSteps; ++i) {
            // the chunk's steps, then (last warp of the row) the padding steps
            const int ls = 32 * i + lane;
            const bool mine =
                kFull || ls < chunk_steps || (sub == kWpr - 1 && st0 + 32 * i < n_steps);
            if (mine) {
                uint32_t vals[4];
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const uint32_t p0 = kept[i][2 * h], p1 = kept[i][2 * h + 1];
                    if constexpr (kInt8) {
                        const uint32_t b0 = int8_code(__uint_as_float(p0 * c65536), inv);
                        const uint32_t b1 = int8_code(__uint_as_float(p0 & 0xFFFF0000u), inv);
                        const uint32_t b2 = int8_code(__uint_as_float(p1 * c65536), inv);
                        const uint32_t b3 = int8_code(__uint_as_float(p1 & 0xFFFF0000u), inv);
                        vals[h] = __byte_perm(__byte_perm(b0, b1, 0x0040),
                                              __byte_perm(b2, b3, 0x0040), 0x5410);
                    } else {
                        const uint32_t q0 = quantize_pair<false>(
                            __uint_as_float(p0 * c65536), __uint_as_float(p0 & 0xFFFF0000u), inv);
                        const uint32_t q1 = quantize_pair<false>(
                            __uint_as_float(p1 * c65536), __uint_as_float(p1 & 0xFFFF0000u), inv);
                        vals[h] = q1 * c65536 + q0;
                    }
                }
                __stcs(vout + 32 * i, make_uint4(vals[0], vals[1], vals[2], vals[3]));
                __stcs(mout + 4096 * i, nib[i]);
            }
        }
    }
    // after a wait that ran out: copies still in flight land before exit
    __syncwarp();
    if (lane == 0 && pending) {
        for (int b = 0; b < kPruneSlots; ++b)
            if ((pending >> b) & 1u) {
                const uint64_t t0 = global_timer_ns();
                while (global_timer_ns() - t0 < 1000000ull) {  // 1 ms
                }
            }
    }
}

// ---------------------------------------------------------------------------
// Single-pass variants for bf16 rows of up to kRegK elements: the whole row
// sits in registers (16 bytes x 2 x 8 per lane), so X is read from HBM once.
// ---------------------------------------------------------------------------
constexpr int kRegChunks = 8;                     // 16-element chunks per lane, at most
constexpr int kRegK = 4 * 32 * 16 * kRegChunks;   // 16384 elements (4 warps per row)

__device__ __forceinline__ void bf16x16_to_f32(const uint4& a, const uint4& b, float (&f)[16]) {
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        f[2 * j] = __uint_as_float(w[j] << 16);
        f[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
    }
}

// Requires K % 16 == 0, K <= 512 * kChunks * kWpr and a 16-byte aligned X.
// A row is held by kWpr warps (kWpr = 1, 2 or 4), each lane keeping kChunks
// 16-element chunks: chunk c of the row sits with warp c / (32 kChunks), lane
// c % 32.  The warps of a row combine their absmax through shared memory;
// 256 / (32 kWpr) rows per CTA.
template <bool kInt8, int kChunks, int kWpr = 1>
__global__ void __launch_bounds__(kWarpRowThreads) quant_lift_reg_kernel(
    const __nv_bfloat16* __restrict__ X, int64_t M, int64_t K64, int Nh, int64_t K_lift64,
    int64_t K_lp64, int q_stride, uint8_t* __restrict__ Xq, float* __restrict__ s_x) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    pdl_trigger();
    pdl_wait();
    constexpr int kRowsPerCta = kWarpRowThreads / (32 * kWpr);
    __shared__ float part[kRowsPerCta][kWpr];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int slot = warp / kWpr;            // row slot of this CTA
    const int sub = warp % kWpr;             // part of the row this warp holds
    const int rt = sub * 32 + lane;          // thread index within the row
    constexpr int kRowThreads = 32 * kWpr;
    const int64_t m = static_cast<int64_t>(blockIdx.x) * kRowsPerCta + slot;
    // rows are whole per warp group, so a group leaves (or stays) together
    if (m >= M) return;
    const int K = static_cast<int>(K64);
    const int K_lift = static_cast<int>(K_lift64);
    const int K_lp = static_cast<int>(K_lp64);
    const uint4* xv = reinterpret_cast<const uint4*>(X + m * K64);
    const int n16 = K / 16;
    const int c0 = sub * 32 * kChunks + lane;  // this lane's first chunk
    uint4 v[2 * kChunks];
#pragma unroll
    for (int i = 0; i < kChunks; ++i) {
        const int c = c0 + 32 * i;
        if (c < n16) {
            v[2 * i] = __ldcs(xv + 2 * c);
            v[2 * i + 1] = __ldcs(xv + 2 * c + 1);
        } else {
            v[2 * i] = make_uint4(0, 0, 0, 0);
            v[2 * i + 1] = make_uint4(0, 0, 0, 0);
        }
    }
    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < 2 * kChunks; ++i) a = fmaxf(a, chunk_absmax<__nv_bfloat16>(v[i]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if constexpr (kWpr > 1) {
        if (lane == 0) part[slot][sub] = a;
        named_bar_sync(1 + slot, kRowThreads);
#pragma unroll
        for (int w = 0; w < kWpr; ++w) a = fmaxf(a, part[slot][w]);
    }
    float inv, s;
    scale_from_absmax<kInt8>(a, inv, s);
    if (rt == 0) s_x[m] = s;
    uint4* out = reinterpret_cast<uint4*>(Xq + m * K_lp64);
    const int n_chunks = K_lp / 16;
    if (Nh <= 2) {  // identity map: chunk c of the output is chunk c of the input
#pragma unroll
        for (int i = 0; i < kChunks; ++i) {
            const int c = c0 + 32 * i;
            if (c < n16) {
                float f[16];
                bf16x16_to_f32(v[2 * i], v[2 * i + 1], f);
                __stcs(out + c, quant16<kInt8>(f, inv));
            }
        }
        for (int c = n16 + rt; c < n_chunks; c += kRowThreads) __stcs(out + c, make_uint4(0, 0, 0, 0));
        return;
    }
    if (Nh == 4) {
        // 6:8: a 16-element chunk is exactly two groups of 8, and its six
        // windows (elements 0-3, 2-5, 4-7 of each group) are made of its own
        // codes: 24 lifted bytes at 24c, no other lane's data involved.
#pragma unroll
        for (int i = 0; i < kChunks; ++i) {
            const int c = c0 + 32 * i;
            if (c < n16) {
                float f[16];
                bf16x16_to_f32(v[2 * i], v[2 * i + 1], f);
                const uint4 w = quant16<kInt8>(f, inv);
                uint2* o = reinterpret_cast<uint2*>(Xq + m * K_lp64 + 24 * static_cast<int64_t>(c));
                __stcs(o, make_uint2(w.x, __byte_perm(w.x, w.y, 0x5432)));
                __stcs(o + 1, make_uint2(w.y, w.z));
                __stcs(o + 2, make_uint2(__byte_perm(w.z, w.w, 0x5432), w.w));
            }
        }
        // zero windows past the last group up to K_lp (8-byte aligned: K_lift = 24 K / 16)
        uint2* z = reinterpret_cast<uint2*>(Xq + m * K_lp64);
        for (int c8 = K_lift / 8 + rt; c8 < K_lp / 8; c8 += kRowThreads)
            __stcs(z + c8, make_uint2(0, 0));
        return;
    }
    // 4:6, 8:10: the row's codes go to a shared-memory row; each 16-byte output
    // word (four windows) is then built from the 12 code bytes its windows
    // span -- two 6-byte groups (4:6) or one 10-byte group (8:10) -- read as
    // three aligned 32-bit words and recombined with byte permutes.
    uint4* qrow = reinterpret_cast<uint4*>(smem_raw + slot * q_stride);
    const int q_chunks = ((K_lift / (4 * (Nh - 1))) * 2 * Nh + 15) / 16;
#pragma unroll
    for (int i = 0; i < kChunks; ++i) {
        const int c = c0 + 32 * i;
        if (c < n16) {
            float f[16];
            bf16x16_to_f32(v[2 * i], v[2 * i + 1], f);
            qrow[c] = quant16<kInt8>(f, inv);
        }
    }
    // zero codes from K to one chunk past the last group: the word reads below
    // may run up to 6 bytes past K_pad
    for (int c = n16 + rt; c <= q_chunks; c += kRowThreads) qrow[c] = make_uint4(0, 0, 0, 0);
    if constexpr (kWpr > 1)
        named_bar_sync(1 + slot, kRowThreads);
    else
        __syncwarp();
    const uint32_t* q32 = reinterpret_cast<const uint32_t*>(qrow);
    const int n_words = (K_lift + 15) / 16;  // output words holding windows (the rest are zero)
    for (int c = rt; c < n_chunks; c += kRowThreads) {
        uint4 o = make_uint4(0, 0, 0, 0);
        if (c < n_words) {
            if (Nh == 3) {
                // groups 2c, 2c+1: code bytes 12c .. 12c+11; windows at 0, 2, 6, 8
                const uint32_t u0 = q32[3 * c], u1 = q32[3 * c + 1], u2 = q32[3 * c + 2];
                o = make_uint4(u0, __byte_perm(u0, u1, 0x5432), __byte_perm(u1, u2, 0x5432), u2);
            } else {
                // 8:10, group c: code bytes 10c .. 10c+9; windows at 0, 2, 4, 6
                const int w0 = (10 * c) >> 2;  // first aligned word
                const uint32_t u0 = q32[w0], u1 = q32[w0 + 1], u2 = q32[w0 + 2];
                if ((c & 1) == 0)
                    o = make_uint4(u0, __byte_perm(u0, u1, 0x5432), u1, __byte_perm(u1, u2, 0x5432));
                else  // the group starts 2 bytes into u0
                    o = make_uint4(__byte_perm(u0, u1, 0x5432), u1, __byte_perm(u1, u2, 0x5432), u2);
            }
        }
        __stcs(out + c, o);
    }
}


}  // namespace ss

namespace ss {

// ---------------------------------------------------------------------------
// Activation lift of the bf16 tier: the same window map as the 8-bit tiers
// (SlideSparse write-up, omica.com.cn, 3.2: window i of group g reads the
// four activations at 2Nh g + 2(i % (Nh-1))), no quantisation, bf16 out.
// Window j of a group is the word pair (u_j, u_{j+1}) of the group's Nh
// 32-bit words of bf16 pairs, so a group of 2Nh inputs becomes 2(Nh-1)
// output words.  Dense and 2:4 are the identity (zero padded to K_lp).
//
// One thread per unit, grid-strided over rows: a unit is a group (sliding
// patterns) or 8 outputs (identity); the zero tail [K_lift, K_lp) goes in
// units of 4 outputs.
// ---------------------------------------------------------------------------
constexpr int kLiftThreads = 256;

template <typename T>
__device__ __forceinline__ uint32_t bf16_pair_at(const T* __restrict__ x, int64_t k, int64_t K) {
    const uint32_t lo = k < K ? bf16_bits(to_f32<T>(x[k])) : 0u;
    const uint32_t hi = k + 1 < K ? bf16_bits(to_f32<T>(x[k + 1])) : 0u;
    return lo | (hi << 16);
}

template <typename T>
__global__ void __launch_bounds__(kLiftThreads) lift_bf16_kernel(
    const T* __restrict__ X, int64_t M, int64_t K, int Nh, int64_t K_lift, int64_t K_lp,
    uint16_t* __restrict__ Xl) {
    pdl_trigger();
    pdl_wait();
    const int64_t u = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    // bf16 words can be read straight from X when every pair is whole
    constexpr bool kRaw = sizeof(T) == 2;
    const bool raw_ok = kRaw && (K % 2 == 0);
    if (Nh <= 2) {
        if (u >= K_lp / 8) return;
        const int64_t k0 = u * 8;
        for (int64_t m = blockIdx.y; m < M; m += gridDim.y) {
            const T* x = X + m * K;
            uint4 v;
            if (kRaw && K % 8 == 0 && k0 + 8 <= K) {
                v = __ldg(reinterpret_cast<const uint4*>(x + k0));
            } else {
                v = make_uint4(bf16_pair_at<T>(x, k0, K), bf16_pair_at<T>(x, k0 + 2, K),
                               bf16_pair_at<T>(x, k0 + 4, K), bf16_pair_at<T>(x, k0 + 6, K));
            }
            __stcs(reinterpret_cast<uint4*>(Xl + m * K_lp + k0), v);
        }
        return;
    }
    const int64_t G = K_lift / (4 * (Nh - 1));
    const int64_t tail_units = (K_lp - K_lift) / 4;
    if (u >= G + tail_units) return;
    for (int64_t m = blockIdx.y; m < M; m += gridDim.y) {
        uint16_t* out_row = Xl + m * K_lp;
        if (u >= G) {  // zero tail, 4 outputs (8 bytes) per unit
            __stcs(reinterpret_cast<uint2*>(out_row + K_lift + 4 * (u - G)), make_uint2(0u, 0u));
            continue;
        }
        const T* x = X + m * K;
        const int64_t k0 = u * 2 * Nh;
        uint32_t w[5];
        if (raw_ok && k0 + 2 * Nh <= K) {
            const uint32_t* xw = reinterpret_cast<const uint32_t*>(x + k0);
#pragma unroll
            for (int i = 0; i < 5; ++i)
                if (i < Nh) w[i] = __ldg(xw + i);
        } else {
#pragma unroll
            for (int i = 0; i < 5; ++i)
                if (i < Nh) w[i] = bf16_pair_at<T>(x, k0 + 2 * i, K);
        }
        uint2* o = reinterpret_cast<uint2*>(out_row + u * 4 * (Nh - 1));
#pragma unroll
        for (int j = 0; j < 4; ++j)
            if (j < Nh - 1) __stcs(o + j, make_uint2(w[j], w[j + 1]));
    }
}

}  // namespace ss
