// The dual-scale binary block with caller-given scales (RaBiT, arXiv
// 2602.05367, section 4.1: binary cores with per-channel output and input
// scaling vectors, W^_k = diag(h_k) B_k diag(g_k); section 4.2: the paths are
// derived in turn from the shared weight and their scales are learned).
//
//   pack_fixed:  B_k = sign(R_{k-1}),  R_k = R_{k-1} - h_k[i] g_k[j] B_k
//                (signs only; the scales are the caller's)
//   dual gemv:   y = sum_k h_k (.) (B_k x_k),  x_k = RN_fp16(g_k (.) x)
//                (the input scaling is an fp16 activation, A16), evaluated by
//                the table matvec as one grouped launch of N single-path
//                descriptors (alpha = h_k, x = x_k) into fp32 per-path rows,
//                then summed over the paths.
#include "rb_internal.cuh"

namespace rb {
namespace {

template <typename WT>
__device__ __forceinline__ void load32f(const WT* p, float (&v)[32]);

template <>
__device__ __forceinline__ void load32f<__half>(const __half* p, float (&v)[32]) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint4 u = __ldcs(reinterpret_cast<const uint4*>(p) + q);
        const __half2* h = reinterpret_cast<const __half2*>(&u);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float2 f = __half22float2(h[i]);
            v[8 * q + 2 * i] = f.x;
            v[8 * q + 2 * i + 1] = f.y;
        }
    }
}

template <>
__device__ __forceinline__ void load32f<float>(const float* p, float (&v)[32]) {
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const float4 u = __ldcs(reinterpret_cast<const float4*>(p) + q);
        v[4 * q] = u.x; v[4 * q + 1] = u.y; v[4 * q + 2] = u.z; v[4 * q + 3] = u.w;
    }
}

// One thread per (row, 32-column word): the residual of its 32 columns stays
// in registers across the N paths. R is kept in fp32; the product
// h_k[i] g_k[j] is rounded to fp32 once.
template <typename WT>
__global__ void __launch_bounds__(256) pack_fixed_kernel(const WT* __restrict__ W, int64_t ldw, int M, int K, int N,
                                                         bool sliced, const float* __restrict__ h,
                                                         const float* __restrict__ g, uint32_t* __restrict__ planes) {
    const int words = K >> 5;
    const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (idx >= static_cast<int64_t>(M) * words) return;
    const int row = static_cast<int>(idx / words), w = static_cast<int>(idx - static_cast<int64_t>(row) * words);
    const size_t S = (static_cast<size_t>(K) + 511) / 512;
    float r[32];
    load32f<WT>(W + static_cast<int64_t>(row) * ldw + 32 * w, r);
#pragma unroll
    for (int e = 0; e < 32; ++e) r[e] = __fadd_rn(r[e], 0.0f);   // -0.0 -> +0.0 (sign(0) = +1)
    for (int k = 0; k < N; ++k) {
        uint32_t word = 0;
#pragma unroll
        for (int e = 0; e < 32; ++e) word |= static_cast<uint32_t>(!(r[e] < 0.0f)) << e;
        if (k + 1 < N) {
            const float hk = h[static_cast<size_t>(k) * M + row];
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                const float sc = g ? __fmul_rn(hk, g[static_cast<size_t>(k) * K + 32 * w + e]) : hk;
                r[e] = (word >> e) & 1u ? __fsub_rn(r[e], sc) : __fadd_rn(r[e], sc);
            }
        }
        const size_t wo = sliced ? ((static_cast<size_t>(k) * S + (w >> 4)) * M + row) * 16 + (w & 15)
                                 : (static_cast<size_t>(k) * M + row) * words + w;
        planes[wo] = word;
    }
}

// x_k[t][j] = RN_fp16(g_k[j] x[t][j]) for every path, from the exact fp64
// product (one rounding); with g null, one dense copy of x. Output [N][T][K].
__global__ void scale_inputs_kernel(const __half* __restrict__ x, int64_t ldx, int T, int64_t K, int N,
                                    const float* __restrict__ g, __half* __restrict__ xk) {
    const int64_t n = static_cast<int64_t>(N) * T * K;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const int64_t j = i % K, t = (i / K) % T, k = i / (K * T);
        const __half xv = x[t * ldx + j];
        xk[i] = g ? __double2half(static_cast<double>(g[k * K + j]) * static_cast<double>(__half2float(xv))) : xv;
    }
}

// The N single-path descriptors of the grouped matvec, written on the device
// (so that a call enqueues no host-to-device copy).
__global__ void fill_descs_kernel(GvJob* descs, const uint32_t* planes, size_t path_words, const float* h,
                                  int64_t M, int64_t K, const __half* xk, size_t x_stride, float* yk, int T, int N) {
    const int k = threadIdx.x;
    if (k < N) {
        descs[k].planes = planes + static_cast<size_t>(k) * path_words;
        descs[k].alpha = h + static_cast<size_t>(k) * M;
        descs[k].x = xk + static_cast<size_t>(k) * x_stride;
        descs[k].y = yk + static_cast<size_t>(k) * T * M;
        descs[k].M = M;
        descs[k].K = K;
    }
}

// y[t][i] = sum_k yk[k][t][i] (in path order), stored as fp16 or fp32.
__global__ void combine_paths_kernel(const float* __restrict__ yk, int N, int T, int64_t M, void* y, int64_t ldy,
                                     bool y_f16) {
    const int64_t n = static_cast<int64_t>(T) * M;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        float s = 0.0f;
        for (int k = 0; k < N; ++k) s += yk[static_cast<int64_t>(k) * n + i];
        const int64_t t = i / M, row = i - t * M;
        if (y_f16) static_cast<__half*>(y)[t * ldy + row] = __float2half_rn(s);
        else static_cast<float*>(y)[t * ldy + row] = s;
    }
}

unsigned grid_for(int64_t n, int threads) {
    const int64_t cap = static_cast<int64_t>(device_sm_count()) * 8;
    int64_t b = (n + threads - 1) / threads;
    if (b > cap) b = cap;
    return static_cast<unsigned>(b < 1 ? 1 : b);
}

}  // namespace

cudaError_t launch_pack_fixed(const void* W, bool w_f16, int64_t ldw, int64_t M, int64_t K, int N, bool sliced,
                              const float* h, const float* g, uint32_t* planes, cudaStream_t s) {
    if (sliced && K % 512 != 0) {
        // zero the padding words of the last slice of every path
        const size_t S = static_cast<size_t>((K + 511) / 512);
        const size_t pitch = S * static_cast<size_t>(M) * 64;
        char* last = reinterpret_cast<char*>(planes) + (S - 1) * static_cast<size_t>(M) * 64;
        cudaError_t e = cudaMemset2DAsync(last, pitch, 0, static_cast<size_t>(M) * 64, N, s);
        if (e != cudaSuccess) return e;
    }
    const int64_t n = M * (K >> 5);
    const unsigned blocks = static_cast<unsigned>((n + 255) / 256);
    if (w_f16)
        pack_fixed_kernel<__half><<<blocks, 256, 0, s>>>(static_cast<const __half*>(W), ldw, static_cast<int>(M),
                                                         static_cast<int>(K), N, sliced, h, g, planes);
    else
        pack_fixed_kernel<float><<<blocks, 256, 0, s>>>(static_cast<const float*>(W), ldw, static_cast<int>(M),
                                                        static_cast<int>(K), N, sliced, h, g, planes);
    return cudaGetLastError();
}

DualPlan dual_plan(int64_t M, int64_t K, int N, int T, bool scaled_x) {
    DualPlan d{};
    GvJob* jobs = new GvJob[N];
    for (int k = 0; k < N; ++k) jobs[k] = GvJob{nullptr, nullptr, nullptr, nullptr, M, K};
    d.gv = gemv_plan_grouped(jobs, N, 1, 0, T);
    delete[] jobs;
    auto a256 = [](size_t b) { return (b + 255) & ~size_t(255); };
    const size_t gv_ws = (d.gv.counters == 0 && d.gv.partials == 0)
                             ? GV_HEADER_BYTES
                             : GV_HEADER_BYTES + GV_CTR_ZONE_BYTES + d.gv.partials * 4;
    d.gv_bytes = a256(gv_ws);
    d.desc_bytes = a256(static_cast<size_t>(N) * sizeof(GvJob));
    d.xk_bytes = scaled_x ? a256(static_cast<size_t>(N) * T * K * 2) : a256(static_cast<size_t>(T) * K * 2);
    d.yk_bytes = a256(static_cast<size_t>(N) * T * M * 4);
    d.total = d.gv_bytes + d.desc_bytes + d.xk_bytes + d.yk_bytes;
    return d;
}

cudaError_t launch_dual_gemv(const uint32_t* planes, bool sliced, int64_t M, int64_t K, int N, const float* h,
                             const float* g, const void* x, int64_t ldx, int T, void* y, bool y_f16, int64_t ldy,
                             void* workspace, const DualPlan& d, cudaStream_t s) {
    char* ws = static_cast<char*>(workspace);
    GvJob* descs = reinterpret_cast<GvJob*>(ws + d.gv_bytes);
    __half* xk = reinterpret_cast<__half*>(ws + d.gv_bytes + d.desc_bytes);
    float* yk = reinterpret_cast<float*>(ws + d.gv_bytes + d.desc_bytes + d.xk_bytes);
    // this workspace carries no zeroed-once contract: clear header and counters
    const size_t zone = GV_HEADER_BYTES + GV_CTR_ZONE_BYTES;
    const size_t clear = d.gv_bytes < zone ? d.gv_bytes : zone;
    cudaError_t e = cudaMemsetAsync(workspace, 0, clear, s);
    if (e != cudaSuccess) return e;
    // the grouped descriptors take dense [T][K] activations: per path x_k with
    // input scales; without them x itself (or one dense copy of a pitched x)
    const __half* xin = static_cast<const __half*>(x);
    size_t x_stride = 0;   // elements between the x of consecutive paths
    if (g || (ldx != K && T > 1)) {
        const int copies = g ? N : 1;
        const int64_t n = static_cast<int64_t>(copies) * T * K;
        scale_inputs_kernel<<<grid_for(n, 256), 256, 0, s>>>(xin, ldx, T, K, copies, g, xk);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        xin = xk;
        x_stride = g ? static_cast<size_t>(T) * K : 0;
    }
    const size_t S = static_cast<size_t>((K + 511) / 512);
    const size_t path_words = sliced ? S * static_cast<size_t>(M) * 16 : static_cast<size_t>(M) * (K / 32);
    fill_descs_kernel<<<1, 32, 0, s>>>(descs, planes, path_words, h, M, K, xin, x_stride, yk, T, N);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    GvArgs a{};
    a.one = GvJob{};
    a.jobs = descs;
    a.n_jobs = N;
    a.n_paths = 1;
    a.group = 0;
    a.sliced = sliced;
    a.alpha_f16 = false;
    a.y_f16 = false;
    a.T = T;
    a.chunk_slices = d.gv.chunk_slices;
    a.workspace = workspace;
    a.ws_bytes = d.gv_bytes;
    a.expect_units = static_cast<uint32_t>(d.gv.units);
    a.expect_ctrs = static_cast<uint32_t>(d.gv.counters);
    a.expect_parts = static_cast<uint32_t>(d.gv.partials);
    if ((e = launch_gemv(a, d.gv, s)) != cudaSuccess) return e;
    combine_paths_kernel<<<grid_for(static_cast<int64_t>(T) * M, 256), 256, 0, s>>>(yk, N, T, M, y, ldy, y_f16);
    return cudaGetLastError();
}

}  // namespace rb
