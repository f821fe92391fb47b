// ss_compress.cuh -- offline weight compression kernel (not on the timed
// path): magnitude prune to the (2Nh-2):2Nh pattern, per-channel scale,
// sliding-window decomposition and 2:4 packing (SlideSparse write-up,
// omica.com.cn, 2.2 weight preprocessing and 2.3; SlideSparse, 66bd.net,
// Fig. 2: windows 0-3, 2-5, 4-7 of each group of 8 for 6:8; LLM-Compressor
// W8A8: channel-wise weight scales).
//
// The bf16 tier (kQ = kQBf16) stores the kept weights as bf16 (round to
// nearest even), two bytes per value, and has no scale.
//
// One CTA per output channel.  Pass 1 stages the row in shared memory, marks
// the kept positions of every group (keep the 2Nh-2 largest |w|, ties keep the
// lower index) and reduces the absmax of the kept weights.  Pass 2 walks the
// output windows in pairs (one metadata byte per pair), assigns the kept
// positions of a window's group to windows by ascending first fit, and packs
// two values and a nibble per window.
#pragma once

#include "ss_common.cuh"

namespace ss {

constexpr int kCompressThreads = 256;
constexpr int kMaxGroup = 10;

// kept bits of group g (bit i = local position i), ranking on |w|.
__device__ __forceinline__ uint32_t kept_bits(const float* v, int group, int keep) {
    uint32_t bits = 0;
    for (int i = 0; i < group; ++i) {
        int rank = 0;
        const float ai = fabsf(v[i]);
        for (int j = 0; j < group; ++j) {
            if (j == i) continue;
            const float aj = fabsf(v[j]);
            rank += (aj > ai || (aj == ai && j < i)) ? 1 : 0;
        }
        if (rank < keep) bits |= 1u << i;
    }
    return bits;
}

// Ascending first fit of the kept positions of one group into its Nh-1
// windows; returns, for window j, the 4-bit set of local positions (0..3
// relative to 2j) it owns.
__device__ __forceinline__ uint32_t window_bits(uint32_t kept, int Nh, int j_target) {
    uint32_t free_ = kept;
    uint32_t result = 0;
    for (int j = 0; j < Nh - 1; ++j) {
        uint32_t own = 0;
        int taken = 0;
        for (int t = 0; t < 4 && taken < 2; ++t) {
            const int pos = 2 * j + t;
            if ((free_ >> pos) & 1u) {
                own |= 1u << t;
                free_ &= ~(1u << pos);
                ++taken;
            }
        }
        if (j == j_target) result = own;
    }
    return result;
}

// Two local indices (ascending) for a window owning `own` (bits 0..3):
// the owned ones, padded with the lowest unused.
__device__ __forceinline__ void window_indices(uint32_t own, int& i0, int& i1) {
    int idx[2], n = 0;
    for (int t = 0; t < 4 && n < 2; ++t)
        if ((own >> t) & 1u) idx[n++] = t;
    for (int t = 0; t < 4 && n < 2; ++t) {
        const bool used = (n > 0 && idx[0] == t);
        if (!((own >> t) & 1u) && !used) idx[n++] = t;
    }
    i0 = min(idx[0], idx[1]);
    i1 = max(idx[0], idx[1]);
}

template <typename T, int kQ>
__global__ void __launch_bounds__(kCompressThreads) compress_weight_kernel(
    const T* __restrict__ W, int64_t N, int64_t K, int keep, int group, int64_t K_lift,
    int64_t K_lp, uint8_t* __restrict__ Wv, uint8_t* __restrict__ Wm, float* __restrict__ s_w) {
    constexpr bool kInt8 = kQ == kQInt8;
    constexpr bool kBf16 = kQ == kQBf16;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    pdl_trigger();
    pdl_wait();
    __shared__ float red[32];
    __shared__ int bad;
    const int64_t n = blockIdx.x;
    // selector byte b of row n in the storage layout of this tier
    auto meta_at = [&](int64_t b) -> uint8_t& {
        return Wm[kQ == kQBf16 ? meta_offset_i16(n, b, K_lp) : meta_offset(n, b, K_lp)];
    };
    if (n >= N) {  // padding row of the last 128-row metadata tile
        for (int64_t b = threadIdx.x; b < K_lp / 8; b += blockDim.x) meta_at(b) = 0;
        return;
    }
    const T* w = W + n * K;
    float* srow = reinterpret_cast<float*>(smem_raw);  // K_pad floats
    const bool dense = (group == 0);
    const int64_t K_pad = dense ? K : (K + group - 1) / group * group;
    uint8_t* kept = smem_raw + ((K_pad * 4 + 15) / 16 * 16);  // one byte per group
    if (threadIdx.x == 0) bad = 0;
    for (int64_t k = threadIdx.x; k < K_pad; k += blockDim.x) {
        const float v = k < K ? to_f32<T>(w[k]) : 0.0f;
        if (!isfinite(v)) bad = 1;
        srow[k] = v;
    }
    __syncthreads();
    float a = 0.0f;
    if (dense) {
        for (int64_t k = threadIdx.x; k < K; k += blockDim.x) a = fmaxf(a, fabsf(srow[k]));
    } else {
        for (int64_t g = threadIdx.x; g < K_pad / group; g += blockDim.x) {
            const uint32_t bits = kept_bits(srow + g * group, group, keep);
            kept[g] = static_cast<uint8_t>(bits & 0xFFu);
            reinterpret_cast<uint8_t*>(kept + K_pad / group)[g] = static_cast<uint8_t>(bits >> 8);
            for (int i = 0; i < group; ++i)
                if ((bits >> i) & 1u) a = fmaxf(a, fabsf(srow[g * group + i]));
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
        if (threadIdx.x == 0) red[0] = a;
    }
    __syncthreads();
    a = red[0];
    if (bad) {
        if (threadIdx.x == 0) record_status(kErrData);
        return;
    }
    float inv = 0.0f, s;
    if constexpr (!kBf16) {
        scale_from_absmax<kInt8>(a, inv, s);
        if (threadIdx.x == 0) s_w[n] = s;
    }
    // stored code of one kept value
    auto code = [&](float v) -> uint32_t {
        if constexpr (kBf16) return bf16_bits(v);
        else return quantize<kInt8>(v, inv);
    };

    if (dense) {
        if constexpr (kBf16) {
            uint16_t* out = reinterpret_cast<uint16_t*>(Wv) + n * K_lp;
            for (int64_t k = threadIdx.x; k < K_lp; k += blockDim.x)
                out[k] = k < K ? static_cast<uint16_t>(code(srow[k])) : 0;
        } else {
            uint8_t* out = Wv + n * K_lp;
            for (int64_t k = threadIdx.x; k < K_lp; k += blockDim.x)
                out[k] = k < K ? static_cast<uint8_t>(code(srow[k])) : 0;
        }
        return;
    }
    const int Nh = group / 2;
    const int64_t n_win = K_lift / 4;
    uint8_t* vrow = Wv + n * (K_lp / 2) * (kBf16 ? 2 : 1);
    const uint8_t* kept_hi = kept + K_pad / group;
    for (int64_t pr = threadIdx.x; pr < K_lp / 8; pr += blockDim.x) {
        uint32_t vals[2] = {0u, 0u};  // 8-bit: vals[0] holds both windows
        uint32_t meta = 0;
        for (int h = 0; h < 2; ++h) {
            const int64_t win = pr * 2 + h;
            uint32_t own = 0;
            int64_t base = 0;
            if (win < n_win) {
                const int64_t g = win / (Nh - 1);
                const int j = static_cast<int>(win - g * (Nh - 1));
                const uint32_t kb = kept[g] | (static_cast<uint32_t>(kept_hi[g]) << 8);
                own = window_bits(kb, Nh, j);
                base = g * group + 2 * j;
            }
            int i0, i1;
            window_indices(own, i0, i1);
            const uint32_t q0 = ((own >> i0) & 1u) ? code(srow[base + i0]) : 0u;
            const uint32_t q1 = ((own >> i1) & 1u) ? code(srow[base + i1]) : 0u;
            if constexpr (kBf16)
                vals[h] = q0 | (q1 << 16);
            else
                vals[0] |= (q0 | (q1 << 8)) << (16 * h);
            meta |= static_cast<uint32_t>(i0 | (i1 << 2)) << (4 * h);
        }
        if constexpr (kBf16)
            reinterpret_cast<uint2*>(vrow)[pr] = make_uint2(vals[0], vals[1]);  // 4 values
        else
            reinterpret_cast<uint32_t*>(vrow)[pr] = vals[0];  // 4 value bytes
        meta_at(pr) = static_cast<uint8_t>(meta);
    }
}

}  // namespace ss
