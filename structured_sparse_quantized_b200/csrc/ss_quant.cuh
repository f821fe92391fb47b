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

// Stage row `m` of X into shared memory as raw input elements and return the
// row absmax (block-wide).
template <typename T>
__device__ __forceinline__ float stage_row_absmax(const T* __restrict__ x, int64_t K, T* srow,
                                                  float* red) {
    float a = 0.0f;
    constexpr int kVec = 16 / sizeof(T);
    const bool vec_ok = (K % kVec == 0) && ((reinterpret_cast<uintptr_t>(x) & 15) == 0);
    if (vec_ok) {
        const int64_t nv = K / kVec;
        const uint4* xv = reinterpret_cast<const uint4*>(x);
        uint4* sv = reinterpret_cast<uint4*>(srow);
        for (int64_t i = threadIdx.x; i < nv; i += blockDim.x) {
            uint4 v = __ldcs(xv + i);  // streamed once
            sv[i] = v;
            const T* e = reinterpret_cast<const T*>(&v);
#pragma unroll
            for (int t = 0; t < kVec; ++t) a = fmaxf(a, fabsf(to_f32<T>(e[t])));
        }
    } else {
        for (int64_t i = threadIdx.x; i < K; i += blockDim.x) {
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
        a = lane < (blockDim.x >> 5) ? red[lane] : 0.0f;
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

// Xq[m, :] for pattern with half-group Nh (Nh = 0: dense identity map).
// Pass 1 stages the row and reduces the absmax; pass 2 quantises every input
// element once into a byte row in shared memory (zero past K); pass 3 builds
// the lifted windows from that byte row (each window starts at an even
// position, so it is two 16-bit shared loads) and writes 16-byte chunks.
template <typename T, bool kInt8>
__global__ void __launch_bounds__(kRowThreads) quant_lift_kernel(
    const T* __restrict__ X, int64_t K, int Nh, int64_t K_lift, int64_t K_lp,
    uint8_t* __restrict__ Xq, float* __restrict__ s_x) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    __shared__ float red[32];
    T* srow = reinterpret_cast<T*>(smem_raw);
    const int64_t row_bytes = (K * static_cast<int64_t>(sizeof(T)) + 15) / 16 * 16;
    uint32_t* qrow = reinterpret_cast<uint32_t*>(smem_raw + row_bytes);
    const int64_t m = blockIdx.x;
    const float a = stage_row_absmax<T>(X + m * K, K, srow, red);
    float inv, s;
    scale_from_absmax<kInt8>(a, inv, s);
    if (threadIdx.x == 0) s_x[m] = s;

    // quantised byte row, length q_len (a multiple of 16 covering every
    // position a window or the identity map can touch)
    const int64_t q_len = Nh == 0 ? K_lp : (K_lift / (4 * (Nh - 1))) * 2 * Nh;
    const int64_t q_words = (q_len + 15) / 16 * 4;
    for (int64_t i = threadIdx.x; i < q_words; i += blockDim.x) {
        uint32_t word = 0;
#pragma unroll
        for (int t = 0; t < 4; ++t) {
            const int64_t k = i * 4 + t;
            const uint32_t q = k < K ? quantize<kInt8>(to_f32<T>(srow[k]), inv) : 0u;
            word |= q << (8 * t);
        }
        qrow[i] = word;
    }
    __syncthreads();

    uint4* out = reinterpret_cast<uint4*>(Xq + m * K_lp);
    const int64_t n_chunks = K_lp / 16;  // 16 output bytes = 4 windows
    if (Nh == 0) {
        const uint4* q4 = reinterpret_cast<const uint4*>(qrow);
        for (int64_t c = threadIdx.x; c < n_chunks; c += blockDim.x) __stcs(out + c, q4[c]);
        return;
    }
    const uint16_t* q16 = reinterpret_cast<const uint16_t*>(qrow);
    const uint32_t n_win = static_cast<uint32_t>(K_lift / 4);
    const uint32_t per_group = static_cast<uint32_t>(Nh - 1);
    for (int64_t c = threadIdx.x; c < n_chunks; c += blockDim.x) {
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

// Keep the two largest |v| of a group of four (ties keep the lower index);
// returns the two local indices in ascending order.
__device__ __forceinline__ void top2_of4(const float (&v)[4], int& i0, int& i1) {
    float a[4];
#pragma unroll
    for (int t = 0; t < 4; ++t) a[t] = fabsf(v[t]);
    int sel[2], n = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int rank = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            if (j == i) continue;
            rank += (a[j] > a[i] || (a[j] == a[i] && j < i)) ? 1 : 0;
        }
        if (rank < 2 && n < 2) sel[n++] = i;
    }
    i0 = sel[0];
    i1 = sel[1];
}

template <typename T, bool kInt8>
__global__ void __launch_bounds__(kRowThreads) prune_act_kernel(
    const T* __restrict__ X, int64_t K, int64_t K_lp, uint8_t* __restrict__ Xv,
    uint8_t* __restrict__ Xm, float* __restrict__ s_x) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    __shared__ float red[32];
    T* srow = reinterpret_cast<T*>(smem_raw);
    const int64_t m = blockIdx.x;
    const float a = stage_row_absmax<T>(X + m * K, K, srow, red);
    float inv, s;
    scale_from_absmax<kInt8>(a, inv, s);
    if (threadIdx.x == 0) s_x[m] = s;

    // One step = 8 groups of 4 = 32 inputs -> 16 value bytes + 4 nibble bytes.
    uint4* vout = reinterpret_cast<uint4*>(Xv + m * (K_lp / 2));
    uint32_t* mout = reinterpret_cast<uint32_t*>(Xm + m * (K_lp / 8));
    const int64_t n_steps = K_lp / 32;
    for (int64_t st = threadIdx.x; st < n_steps; st += blockDim.x) {
        uint32_t vals[4] = {0, 0, 0, 0};
        uint32_t nibs = 0;
#pragma unroll
        for (int gi = 0; gi < 8; ++gi) {
            const int64_t k0 = st * 32 + gi * 4;
            float v[4];
#pragma unroll
            for (int t = 0; t < 4; ++t) v[t] = row_at<T>(srow, k0 + t, K);
            int i0, i1;
            top2_of4(v, i0, i1);
            const uint32_t q0 = quantize<kInt8>(v[i0], inv);
            const uint32_t q1 = quantize<kInt8>(v[i1], inv);
            // value bytes 2*gi, 2*gi+1 of the 16-byte chunk
            vals[gi >> 1] |= (q0 | (q1 << 8)) << (16 * (gi & 1));
            nibs |= static_cast<uint32_t>(i0 | (i1 << 2)) << (4 * gi);
        }
        __stcs(vout + st, make_uint4(vals[0], vals[1], vals[2], vals[3]));
        __stcs(mout + st, nibs);
    }
}

}  // namespace ss
