// rb_pack kernels: residual sign planes and scales from one shared weight.
//
// RaBiT (arXiv 2602.05367) section 4.2 and appendix G: the paths are derived
// in turn from one shared full-precision weight, the residual updated after
// each path. The scale of a path is mean |R| over its row or 128-column group
// (QBB summary, cascaded analytical residual initialisation); sign(0) = +1.
//
// Two kernels, both HBM-bound streams that read W once and keep the residual
// of a row (or group) in registers across the N paths:
//  * one scale per row: one CTA per row, each thread holding CPT chunks of 8
//    consecutive columns; the fp64 sum of |R| is reduced over the CTA.
//  * one scale per 128 columns: four lanes per group, each lane holding the 32
//    columns of one output word; the sum is reduced over the four lanes.
// |R| is summed in fp32 over at most 8 (row) or 32 (group) values in a
// balanced tree, then in fp64, so alpha keeps ~2e-7 relative accuracy; the
// residual stays in fp32 and is updated with the fp32-rounded alpha.
#include "rb_internal.cuh"

namespace rb {
namespace {

__device__ __forceinline__ void load8(const __half* p, float (&v)[8]) {
    const uint4 u = __ldcs(reinterpret_cast<const uint4*>(p));
    const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __half22float2(h[i]);
        v[2 * i] = f.x;
        v[2 * i + 1] = f.y;
    }
}

__device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
    const float4 a = __ldcs(reinterpret_cast<const float4*>(p));
    const float4 b = __ldcs(reinterpret_cast<const float4*>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// Balanced fp32 sum of |v[0..8)|.
__device__ __forceinline__ float abs_sum8(const float* v) {
    return ((fabsf(v[0]) + fabsf(v[1])) + (fabsf(v[2]) + fabsf(v[3]))) +
           ((fabsf(v[4]) + fabsf(v[5])) + (fabsf(v[6]) + fabsf(v[7])));
}

// Pairs of fp32 values in one 64-bit register, added with one add.f32x2.
__device__ __forceinline__ uint64_t pack_f2(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void unpack_f2(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t add_f2(uint64_t a, uint64_t b) {
    uint64_t r;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
    return r;
}

// 32 weights as fp32 with -0.0 turned into +0.0 (sign(0) = +1): fp16 values
// are widened and added to +0.0 in one mixed-precision add.
__device__ __forceinline__ void load32_nz(const __half* p, float (&v)[32]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint4 u = __ldcs(reinterpret_cast<const uint4*>(p) + i);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const unsigned short h = static_cast<unsigned short>(w[j >> 1] >> (16 * (j & 1)));
            asm("add.rn.f32.f16 %0, %1, %2;" : "=f"(v[8 * i + j]) : "h"(h), "f"(0.0f));
        }
    }
}
__device__ __forceinline__ void load32_nz(const float* p, float (&v)[32]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float t[8];
        load8(p + 8 * i, t);
#pragma unroll
        for (int e = 0; e < 8; ++e) v[8 * i + e] = __fadd_rn(t[e], 0.0f);
    }
}

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(FULL_MASK, v, o);
    return v;
}

// Sum over the CTA; every thread gets the same value (same order everywhere).
__device__ __forceinline__ double block_sum(double v, double* red) {
    v = warp_sum(v);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    if (lane == 0) red[warp] = v;
    __syncthreads();
    double t = lane < nw ? red[lane] : 0.0;
    t = warp_sum(t);
    __syncthreads();
    return t;
}

// B = +1 when R >= 0 (so -0.0 and +0.0 give +1); returns the packed bits of
// 8 columns and, unless it is the last path, moves R to R - alpha * B.
__device__ __forceinline__ uint32_t sign_and_update8(float* r, float a, bool update) {
    uint32_t bits = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        const bool pos = !(r[e] < 0.0f);
        bits |= static_cast<uint32_t>(pos) << e;
        if (update) r[e] -= pos ? a : -a;
    }
    return bits;
}

template <typename WT, int CPT, int MAXT>
__global__ void __launch_bounds__(MAXT)
pack_row_kernel(const WT* __restrict__ W, int64_t ldw, int M, int K, int N, bool sliced,
                uint32_t* __restrict__ planes, float* __restrict__ alpha,
                __half* __restrict__ alpha16) {
    __shared__ double red[32];
    const int row = blockIdx.x;
    const int chunks = K >> 3;
    const WT* wrow = W + static_cast<int64_t>(row) * ldw;
    uint8_t* pb = reinterpret_cast<uint8_t*>(planes);
    const size_t S = (static_cast<size_t>(K) + 511) / 512;
    // byte `idx` (columns 8 idx .. 8 idx + 7) of path k of this row
    auto byte_at = [&](int k, int idx) -> uint8_t* {
        if (!sliced) return pb + (static_cast<size_t>(k) * M + row) * chunks + idx;
        const int w = idx >> 2;
        return pb + ((static_cast<size_t>(k) * S + (w >> 4)) * M + row) * 64 + 4 * (w & 15) + (idx & 3);
    };

    float r[CPT][8];
#pragma unroll
    for (int c = 0; c < CPT; ++c) {
        const int idx = threadIdx.x + c * blockDim.x;
        if (idx < chunks) {
            load8(wrow + 8 * idx, r[c]);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) r[c][e] = 0.0f;
        }
    }
    for (int k = 0; k < N; ++k) {
        double s = 0.0;
#pragma unroll
        for (int c = 0; c < CPT; ++c)
            if (threadIdx.x + c * blockDim.x < chunks) s += static_cast<double>(abs_sum8(r[c]));
        s = block_sum(s, red);
        const float a = static_cast<float>(s / static_cast<double>(K));
        if (threadIdx.x == 0) {
            alpha[static_cast<size_t>(k) * M + row] = a;
            if (alpha16) alpha16[static_cast<size_t>(k) * M + row] = __float2half_rn(a);
        }
        const bool update = k + 1 < N;
#pragma unroll
        for (int c = 0; c < CPT; ++c) {
            const int idx = threadIdx.x + c * blockDim.x;
            if (idx < chunks) {
                const uint32_t bits = sign_and_update8(r[c], a, update);
                *byte_at(k, idx) = static_cast<uint8_t>(bits);
            }
        }
    }
}

template <typename WT>
__device__ __forceinline__ void load32(const WT* p, float (&v)[32]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float t[8];
        load8(p + 8 * i, t);
#pragma unroll
        for (int e = 0; e < 8; ++e) v[8 * i + e] = t[e];
    }
}

// One scale per row, K <= 32768: thread tr of a row's `tpr` threads owns
// plane word tr (columns 32 tr .. 32 tr + 31) for every path, so the sign
// bits of a word are packed in registers and stored as one 32-bit word. A
// CTA packs rows_per_cta rows; |R| is summed in fp32 over the 32 values of
// a word (balanced tree), then in fp64 over the words of the row (warp
// shuffles, then the row's warps through shared memory, in a fixed order).
// NPC: the path count as a compile-time constant (1..4), 0 to read N
template <typename WT, int NPC>
__global__ void __launch_bounds__(1024)
pack_words_kernel(const WT* __restrict__ W, int64_t ldw, int M, int K, int N_rt, bool sliced, int tpr,
                  int rows_per_cta, uint32_t* __restrict__ planes, float* __restrict__ alpha,
                  __half* __restrict__ alpha16) {
    __shared__ double red[2][32];
    const int N = NPC > 0 ? NPC : N_rt;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int rl = tid / tpr, tr = tid - rl * tpr;
    const int row = blockIdx.x * rows_per_cta + rl;
    const int words = K >> 5;
    const bool active = row < M && tr < words;
    const int wpr = tpr >> 5;   // warps per row when tpr >= 32
    const size_t S = (static_cast<size_t>(K) + 511) / 512;

    // mean = sum / K; for K a power of two the product with 1/K is the same
    // number and avoids the fp64 division
    const bool k_pow2 = (K & (K - 1)) == 0;
    const double inv_k = 1.0 / static_cast<double>(K);
    float r[32];
    if (active) {
        load32_nz(W + static_cast<int64_t>(row) * ldw + 32 * tr, r);   // -0.0 -> +0.0 (sign(0) = +1)
    } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) r[e] = 0.0f;
    }
    for (int k = 0; k < N; ++k) {
        // balanced tree: |r| of neighbours, then pairs of partial sums in
        // f32x2 registers (lane e with lane e + 8), then the two lanes
        uint64_t t2[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
            t2[e] = pack_f2(fabsf(r[2 * e]) + fabsf(r[2 * e + 1]), fabsf(r[2 * e + 16]) + fabsf(r[2 * e + 17]));
#pragma unroll
        for (int w = 4; w >= 1; w >>= 1)
#pragma unroll
            for (int e = 0; e < w; ++e) t2[e] = add_f2(t2[e], t2[e + w]);
        float tlo, thi;
        unpack_f2(t2[0], tlo, thi);
        double sum = static_cast<double>(tlo + thi);
        if (tpr <= 32) {
            for (int o = 1; o < tpr; o <<= 1) sum += __shfl_xor_sync(FULL_MASK, sum, o);
        } else {
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) sum += __shfl_xor_sync(FULL_MASK, sum, o);
            if (lane == 0) red[k & 1][warp] = sum;
            __syncthreads();
            sum = 0.0;
            if (wpr > 8) {
                // long rows: the row's partials as a shuffle tree (five
                // levels instead of wpr dependent adds); a + b == b + a, so
                // every lane ends with the same sum
                double v = lane < wpr ? red[k & 1][rl * wpr + lane] : 0.0;
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(FULL_MASK, v, o);
                sum = v;
            } else {
                for (int w = 0; w < wpr; ++w) sum += red[k & 1][rl * wpr + w];
            }
        }
        // every lane of a row holds the same sum; one lane per warp divides
        float a = 0.0f;
        if ((lane & (min(tpr, 32) - 1)) == 0)
            a = static_cast<float>(k_pow2 ? sum * inv_k : sum / static_cast<double>(K));
        a = __shfl_sync(FULL_MASK, a, lane & ~(min(tpr, 32) - 1));
        if (active && tr == 0) {
            alpha[static_cast<size_t>(k) * M + row] = a;
            if (alpha16) alpha16[static_cast<size_t>(k) * M + row] = __float2half_rn(a);
        }
        // B = +1 where R >= 0 (R is never -0.0: the input was cleared of it
        // and x + (-x) rounds to +0.0); R <- R + (-a B)
        // The sign bits are gathered with one funnel shift per value (bit e of
        // `neg` = sign of R[e]); the word is their complement.
        uint32_t neg = 0;
#pragma unroll
        for (int e = 31; e >= 0; --e) neg = __funnelshift_l(__float_as_uint(r[e]), neg, 1);
        const uint32_t word = ~neg;
        // threads past the row's last word keep R = 0, so they add nothing
        // to the next path's sum
        if (active && k + 1 < N) {
            const uint32_t neg_a = __float_as_uint(-a);
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const float q0 = __uint_as_float((__float_as_uint(r[2 * e]) & 0x80000000u) ^ neg_a);
                const float q1 = __uint_as_float((__float_as_uint(r[2 * e + 1]) & 0x80000000u) ^ neg_a);
                unpack_f2(add_f2(pack_f2(r[2 * e], r[2 * e + 1]), pack_f2(q0, q1)), r[2 * e], r[2 * e + 1]);
            }
        }
        if (active) {
            const size_t wo = sliced ? ((static_cast<size_t>(k) * S + (tr >> 4)) * M + row) * 16 + (tr & 15)
                                     : (static_cast<size_t>(k) * M + row) * words + tr;
            planes[wo] = word;
        }
    }
}

// One scale per (path, row, 128 columns): lanes 4g..4g+3 of a warp own group g
// (eight groups per warp per step); lane (4g + q) holds columns 32q..32q+31.
template <typename WT>
__global__ void __launch_bounds__(128)
pack_g128_kernel(const WT* __restrict__ W, int64_t ldw, int M, int K, int N, bool sliced,
                 uint32_t* __restrict__ planes, float* __restrict__ alpha,
                 __half* __restrict__ alpha16) {
    const int gpr = K >> 7;
    const int words = K >> 5;
    const int64_t S = (K + 511) / 512;
    const int64_t total = static_cast<int64_t>(M) * gpr;
    const int lane = threadIdx.x & 31;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    for (int64_t g0 = warp * 8; g0 < total; g0 += nwarps * 8) {
        const int64_t grp = g0 + (lane >> 2);
        const bool valid = grp < total;
        const int64_t row = valid ? grp / gpr : 0;
        const int gi = valid ? static_cast<int>(grp - row * gpr) : 0;
        const int wi = gi * 4 + (lane & 3);
        float r[32];
        if (valid) {
            load32_nz(W + row * ldw + 32 * wi, r);   // -0.0 -> +0.0 (sign(0) = +1)
        } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) r[e] = 0.0f;
        }
        for (int k = 0; k < N; ++k) {
            float p8[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) p8[i] = abs_sum8(r + 8 * i);
            double s = static_cast<double>((p8[0] + p8[1]) + (p8[2] + p8[3]));
            s += __shfl_xor_sync(FULL_MASK, s, 1);
            s += __shfl_xor_sync(FULL_MASK, s, 2);
            const float a = static_cast<float>(s * (1.0 / 128.0));
            // sign bits by one funnel shift per value; R <- R + (-a B)
            uint32_t neg = 0;
#pragma unroll
            for (int e = 31; e >= 0; --e) neg = __funnelshift_l(__float_as_uint(r[e]), neg, 1);
            const uint32_t word = ~neg;
            if (k + 1 < N) {
                const uint32_t neg_a = __float_as_uint(-a);
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float q0 = __uint_as_float((__float_as_uint(r[2 * e]) & 0x80000000u) ^ neg_a);
                    const float q1 = __uint_as_float((__float_as_uint(r[2 * e + 1]) & 0x80000000u) ^ neg_a);
                    unpack_f2(add_f2(pack_f2(r[2 * e], r[2 * e + 1]), pack_f2(q0, q1)), r[2 * e], r[2 * e + 1]);
                }
            }
            if (valid) {
                const int64_t wo = sliced ? ((k * S + (wi >> 4)) * M + row) * 16 + (wi & 15)
                                          : (static_cast<int64_t>(k) * M + row) * words + wi;
                planes[wo] = word;
                if ((lane & 3) == 0) {
                    const int64_t ai = (static_cast<int64_t>(k) * M + row) * gpr + gi;
                    alpha[ai] = a;
                    if (alpha16) alpha16[ai] = __float2half_rn(a);
                }
            }
        }
    }
}

template <typename WT, int CPT, int MAXT = 1024>
cudaError_t launch_row(const PackArgs& a, int threads, cudaStream_t s) {
    pack_row_kernel<WT, CPT, MAXT><<<static_cast<unsigned>(a.M), threads, 0, s>>>(
        static_cast<const WT*>(a.W), a.ldw, static_cast<int>(a.M), static_cast<int>(a.K),
        a.n_paths, a.sliced, a.planes, a.alpha, a.alpha16);
    return cudaGetLastError();
}

template <typename WT>
cudaError_t launch_words(const PackArgs& a, cudaStream_t s) {
    const int words = static_cast<int>(a.K >> 5);
    int tpr = 4;
    if (words <= 32) {
        while (tpr < words) tpr <<= 1;
    } else {
        tpr = (words + 31) & ~31;
    }
    // 128-thread CTAs (one row for K >= 4096): many small CTAs per SM hide the
    // load latency of one behind the arithmetic of others (512-thread CTAs
    // were 15 % slower on 11008 x 4096)
    const int rows_per_cta = tpr >= 128 ? 1 : 128 / tpr;
    const int64_t blocks = (a.M + rows_per_cta - 1) / rows_per_cta;
    auto kern = a.n_paths == 1   ? pack_words_kernel<WT, 1>
                : a.n_paths == 2 ? pack_words_kernel<WT, 2>
                : a.n_paths == 3 ? pack_words_kernel<WT, 3>
                : a.n_paths == 4 ? pack_words_kernel<WT, 4>
                                 : pack_words_kernel<WT, 0>;
    kern<<<static_cast<unsigned>(blocks), rows_per_cta * tpr, 0, s>>>(
        static_cast<const WT*>(a.W), a.ldw, static_cast<int>(a.M), static_cast<int>(a.K), a.n_paths, a.sliced, tpr,
        rows_per_cta, a.planes, a.alpha, a.alpha16);
    return cudaGetLastError();
}

template <typename WT>
cudaError_t launch_row_any(const PackArgs& a, cudaStream_t s) {
    if (a.K <= 32768) return launch_words<WT>(a, s);
    const int chunks = static_cast<int>(a.K >> 3);
    int cpt = 1;
    while (cpt < 8 && (chunks + cpt - 1) / cpt > 512) cpt *= 2;
    int threads = (chunks + cpt - 1) / cpt;
    threads = (threads + 31) & ~31;
    if (threads > 1024) return cudaErrorInvalidConfiguration;
    switch (cpt) {
        case 1: return launch_row<WT, 1>(a, threads, s);
        case 2: return launch_row<WT, 2>(a, threads, s);
        case 4: return launch_row<WT, 4>(a, threads, s);
        default:   // 8 chunks (64 values) per thread: give it 128 registers when it fits in 512 threads
            return threads <= 512 ? launch_row<WT, 8, 512>(a, threads, s) : launch_row<WT, 8, 1024>(a, threads, s);
    }
}

template <typename WT>
cudaError_t launch_g128(const PackArgs& a, cudaStream_t s) {
    const int64_t groups = a.M * (a.K >> 7);
    const int64_t warps_needed = (groups + 7) / 8;
    // 128-thread CTAs, one group of 8 per warp: many small CTAs per SM hide
    // load latency (a grid capped at 8 CTAs of 256 per SM was 2 % slower)
    int64_t blocks = (warps_needed + 3) / 4;
    if (blocks < 1) blocks = 1;
    pack_g128_kernel<WT><<<static_cast<unsigned>(blocks), 128, 0, s>>>(
        static_cast<const WT*>(a.W), a.ldw, static_cast<int>(a.M), static_cast<int>(a.K),
        a.n_paths, a.sliced, a.planes, a.alpha, a.alpha16);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_pack(const PackArgs& a, cudaStream_t s) {
    if (a.sliced && a.K % 512 != 0) {
        // zero the last slice of every path (its words past K/32 are padding)
        const size_t S = static_cast<size_t>((a.K + 511) / 512);
        const size_t pitch = S * static_cast<size_t>(a.M) * 64;
        char* last = reinterpret_cast<char*>(a.planes) + (S - 1) * static_cast<size_t>(a.M) * 64;
        cudaError_t e = cudaMemset2DAsync(last, pitch, 0, static_cast<size_t>(a.M) * 64, a.n_paths, s);
        if (e != cudaSuccess) return e;
    }
    if (a.group == 0)
        return a.w_f16 ? launch_row_any<__half>(a, s) : launch_row_any<float>(a, s);
    return a.w_f16 ? launch_g128<__half>(a, s) : launch_g128<float>(a, s);
}

}  // namespace rb
