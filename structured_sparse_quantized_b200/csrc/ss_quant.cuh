// ss_quant.cuh -- memory-bound activation kernels.
//
//  quant_lift_kernel   fused per-token absmax, quantisation and activation
//                      lifting (SlideSparse, 66bd.net: lifting is an index map
//                      fused into the per-token quant kernel; SlideSparse
//                      write-up, omica.com.cn, 3.2: one pass computes the
//                      absmax, the scale, the clamped quantised values, the
//                      window remap and the packed 32-bit stores, iterating
//                      over output windows).
//  prune_act_kernel    online 2:4 prune + compress of an activation ("add 2:4
//                      or drop a precision tier?", paper-daily 2610.28947,
//                      sections 1 and 2.3).
//
// One CTA per token row.  The row is read from HBM once into shared memory
// (16-byte loads), the absmax is reduced there, and the output is produced in
// 16-byte stores: four lifted windows (or sixteen identity bytes) per store
// for the lift, eight 2:4 groups (16 value bytes + one 32-bit nibble word)
// per step for the prune.
#pragma once

#include "ss_common.cuh"

namespace ss {

constexpr int kRowThreads = 256;

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

// Stage one row of X into shared memory as raw input elements and return the
// row absmax (block-wide).  Rows are read once, 16 bytes per load.
template <typename T>
__device__ __forceinline__ float stage_row_absmax(const T* __restrict__ x, int64_t K64, T* srow,
                                                  float* red) {
    const int K = static_cast<int>(K64);
    float a = 0.0f;
    constexpr int kVec = 16 / sizeof(T);
    const bool vec_ok = (K % kVec == 0) && ((reinterpret_cast<uintptr_t>(x) & 15) == 0);
    if (vec_ok) {
        const int nv = K / kVec;
        const uint4* xv = reinterpret_cast<const uint4*>(x);
        uint4* sv = reinterpret_cast<uint4*>(srow);
        int i = threadIdx.x;
        for (; i + 3 * static_cast<int>(blockDim.x) < nv; i += 4 * blockDim.x) {
            uint4 v[4];  // four loads in flight per thread
#pragma unroll
            for (int u = 0; u < 4; ++u) v[u] = __ldcs(xv + i + u * blockDim.x);
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                sv[i + u * blockDim.x] = v[u];
                a = fmaxf(a, chunk_absmax<T>(v[u]));
            }
        }
        for (; i < nv; i += blockDim.x) {
            const uint4 v = __ldcs(xv + i);
            sv[i] = v;
            a = fmaxf(a, chunk_absmax<T>(v));
        }
    } else {
        for (int i = threadIdx.x; i < K; i += blockDim.x) {
            T v = x[i];
            srow[i] = v;
            a = fmaxf(a, fabsf(to_f32<T>(v)));
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = a;
    __syncthreads();
    if (warp == 0) {
        a = lane < static_cast<int>(blockDim.x >> 5) ? red[lane] : 0.0f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
        if (lane == 0) red[0] = a;
    }
    __syncthreads();
    return red[0];
}

template <typename T>
__device__ __forceinline__ float row_at(const T* srow, int64_t k, int64_t K) {
    return k < K ? to_f32<T>(srow[k]) : 0.0f;
}

// Sixteen consecutive inputs of the staged row (zero past K) as floats.
template <typename T>
__device__ __forceinline__ void load16(const T* srow, int k0, int K, float (&f)[16]) {
    if (k0 + 16 <= K) {
        if constexpr (sizeof(T) == 2) {
            const uint4* p = reinterpret_cast<const uint4*>(srow + k0);  // 16-byte aligned
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint4 v = p[h];
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    f[8 * h + 2 * j] = __uint_as_float(w[j] << 16);         // bf16 -> f32 (exact)
                    f[8 * h + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
                }
            }
        } else {
            const float4* p = reinterpret_cast<const float4*>(srow + k0);
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const float4 v = p[h];
                f[4 * h] = v.x;
                f[4 * h + 1] = v.y;
                f[4 * h + 2] = v.z;
                f[4 * h + 3] = v.w;
            }
        }
    } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) f[j] = (k0 + j < K) ? to_f32<T>(srow[k0 + j]) : 0.0f;
    }
}

// INT8 code of x * inv as the low byte of a 32-bit word: the product is
// rounded to fp32, clamped to [-127, 127], and rounded to the nearest integer
// (ties to even) by adding 1.5 * 2^23, after which the integer sits in the
// low mantissa bits.  This is the IEEE round-to-nearest-even of the fp32
// product, without the low-throughput float-to-int conversion unit.
__device__ __forceinline__ uint32_t int8_code(float x, float inv) {
    const float p = fminf(fmaxf(__fmul_rn(x, inv), -127.0f), 127.0f);
    return __float_as_uint(__fadd_rn(p, 12582912.0f));  // low byte = code
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

// Xq[m, :] for pattern with half-group Nh (Nh = 0: dense identity map).
// Pass 1 stages the row and reduces the absmax.  Identity maps (dense and
// 2:4, whose single window per group is the group itself) then quantise
// sixteen inputs into one 16-byte store each.  Sliding patterns quantise
// every input once into a byte row in shared memory and build the lifted
// windows from it: each window starts at an even position, so it is two
// 16-bit shared loads, and four windows make one 16-byte store.
template <typename T, bool kInt8>
__global__ void __launch_bounds__(kRowThreads) quant_lift_kernel(
    const T* __restrict__ X, int64_t K64, int Nh, int64_t K_lift64, int64_t K_lp64,
    uint8_t* __restrict__ Xq, float* __restrict__ s_x) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    __shared__ float red[32];
    const int K = static_cast<int>(K64);
    const int K_lift = static_cast<int>(K_lift64);
    const int K_lp = static_cast<int>(K_lp64);
    T* srow = reinterpret_cast<T*>(smem_raw);
    const int row_bytes = (K * static_cast<int>(sizeof(T)) + 15) / 16 * 16;
    const int64_t m = blockIdx.x;
    const float a = stage_row_absmax<T>(X + m * K64, K64, srow, red);
    float inv, s;
    scale_from_absmax<kInt8>(a, inv, s);
    if (threadIdx.x == 0) s_x[m] = s;

    uint4* out = reinterpret_cast<uint4*>(Xq + m * K_lp64);
    const int n_chunks = K_lp / 16;  // 16 output bytes
    if (Nh <= 2) {                   // identity map
        for (int c = threadIdx.x; c < n_chunks; c += blockDim.x) {
            float f[16];
            load16<T>(srow, c * 16, K, f);
            __stcs(out + c, quant16<kInt8>(f, inv));
        }
        return;
    }
    // quantised byte row covering K_pad = (K_lift / (4 (Nh-1))) * 2Nh positions
    uint4* qrow = reinterpret_cast<uint4*>(smem_raw + row_bytes);
    const int q_chunks = ((K_lift / (4 * (Nh - 1))) * 2 * Nh + 15) / 16;
    for (int c = threadIdx.x; c < q_chunks; c += blockDim.x) {
        float f[16];
        load16<T>(srow, c * 16, K, f);
        qrow[c] = quant16<kInt8>(f, inv);
    }
    __syncthreads();
    const uint16_t* q16 = reinterpret_cast<const uint16_t*>(qrow);
    const uint32_t n_win = static_cast<uint32_t>(K_lift / 4);
    const uint32_t per_group = static_cast<uint32_t>(Nh - 1);
    for (int c = threadIdx.x; c < n_chunks; c += blockDim.x) {
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
            w[i] = word;  // byte t of the window at ascending address
            ++win;
            if (++j == per_group) {
                j = 0;
                ++g;
            }
        }
        __stcs(out + c, make_uint4(w[0], w[1], w[2], w[3]));
    }
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

template <typename T, bool kInt8>
__global__ void __launch_bounds__(kRowThreads) prune_act_kernel(
    const T* __restrict__ X, int64_t K64, int64_t K_lp64, uint8_t* __restrict__ Xv,
    uint8_t* __restrict__ Xm, float* __restrict__ s_x) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    __shared__ float red[32];
    const int K = static_cast<int>(K64);
    const int K_lp = static_cast<int>(K_lp64);
    T* srow = reinterpret_cast<T*>(smem_raw);
    const int64_t m = blockIdx.x;
    const float a = stage_row_absmax<T>(X + m * K64, K64, srow, red);
    float inv, s;
    scale_from_absmax<kInt8>(a, inv, s);
    if (threadIdx.x == 0) s_x[m] = s;

    // One step = 8 groups of 4 = 32 inputs -> 16 value bytes + 4 nibble bytes.
    uint4* vout = reinterpret_cast<uint4*>(Xv + m * (K_lp64 / 2));
    uint32_t* mout = reinterpret_cast<uint32_t*>(Xm + m * (K_lp64 / 8));
    const int n_steps = K_lp / 32;
    for (int st = threadIdx.x; st < n_steps; st += blockDim.x) {
        float f[32];
        load16<T>(srow, st * 32, K, *reinterpret_cast<float(*)[16]>(f));
        load16<T>(srow, st * 32 + 16, K, *reinterpret_cast<float(*)[16]>(f + 16));
        uint32_t vals[4];
        uint32_t nibs = 0;
#pragma unroll
        for (int gi = 0; gi < 8; ++gi) {
            int i0, i1;
            top2_of4(f + 4 * gi, i0, i1);
            const uint32_t q =
                quantize_pair<kInt8>(pick4(f + 4 * gi, i0), pick4(f + 4 * gi, i1), inv);
            if (gi & 1)
                vals[gi >> 1] |= q << 16;
            else
                vals[gi >> 1] = q;
            nibs |= static_cast<uint32_t>(i0 | (i1 << 2)) << (4 * gi);
        }
        __stcs(vout + st, make_uint4(vals[0], vals[1], vals[2], vals[3]));
        __stcs(mout + st, nibs);
    }
}

}  // namespace ss
