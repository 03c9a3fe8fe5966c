// Host side of the C ABI declared in include/rb_api.h: argument validation,
// launch planning and error reporting. Every check runs before anything is
// enqueued; the kernels live in rb_pack.cu, rb_gemv.cu, rb_gemm.cu (prefill
// blocks) and rb_gemm_dec.cu (decode batches).
#include "../../include/rb_api.h"
#include "rb_internal.cuh"

#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

namespace rb {

static thread_local std::string g_last_error;

static rb_status fail(rb_status s, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return s;
}

void set_error_message(const char* msg) { g_last_error = msg; }

static rb_status cuda_fail(cudaError_t e, const char* where) {
    return fail(RB_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

int device_sm_count() {
    static std::mutex mu;
    static std::vector<int> cache;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    std::lock_guard<std::mutex> lk(mu);
    if (static_cast<int>(cache.size()) <= dev) cache.resize(dev + 1, 0);
    if (cache[dev] == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cache[dev] = n;
    }
    return cache[dev];
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

static rb_status check_layout(const rb_layout& L) {
    if (L.M <= 0 || L.K <= 0) return fail(RB_ERR_INVALID_ARG, "M and K must be positive (M=%lld K=%lld)",
                                          (long long)L.M, (long long)L.K);
    if (L.K % 128 != 0) return fail(RB_ERR_UNSUPPORTED, "K=%lld is not a multiple of 128", (long long)L.K);
    if (L.n_paths < 1 || L.n_paths > 8) return fail(RB_ERR_UNSUPPORTED, "n_paths=%d outside 1..8", L.n_paths);
    if (L.group != 0 && L.group != 128) return fail(RB_ERR_UNSUPPORTED, "group=%d (0 or 128)", L.group);
    if (L.order != RB_ROWS && L.order != RB_SLICED) return fail(RB_ERR_INVALID_ARG, "order=%d", L.order);
    if (L.reserved != 0) return fail(RB_ERR_INVALID_ARG, "reserved field must be 0");
    // byte offsets within one path's planes and scale indices are 32-bit on the device
    if (static_cast<double>(L.M) * 64.0 * ((L.K + 511) / 512) >= 4294967296.0 || L.M >= (1ll << 31) ||
        static_cast<double>(L.n_paths) * L.M * (L.K / 128) >= 4294967296.0)
        return fail(RB_ERR_UNSUPPORTED, "layout too large (planes of one path must stay below 4 GiB)");
    return RB_OK;
}

static size_t dtype_size(rb_dtype d) { return d == RB_F16 ? 2 : 4; }

static bool valid_dtype(rb_dtype d) { return d == RB_F16 || d == RB_F32; }

static size_t gv_ws_bytes(const GvPlan& pl) {
    if (pl.counters == 0 && pl.partials == 0) return GV_HEADER_BYTES;
    return GV_HEADER_BYTES + GV_CTR_ZONE_BYTES + pl.partials * 4;
}

}  // namespace rb

using namespace rb;

extern "C" {

size_t rb_planes_words(rb_layout L) {
    if (check_layout(L) != RB_OK) return 0;
    if (L.order == RB_SLICED) return static_cast<size_t>(L.n_paths) * L.M * 16 * ((L.K + 511) / 512);
    return static_cast<size_t>(L.n_paths) * L.M * (L.K / 32);
}

size_t rb_scales_count(rb_layout L) {
    if (check_layout(L) != RB_OK) return 0;
    const int64_t G = L.group ? L.group : L.K;
    return static_cast<size_t>(L.n_paths) * L.M * (L.K / G);
}

const char* rb_status_string(rb_status s) {
    switch (s) {
        case RB_OK: return "RB_OK";
        case RB_ERR_INVALID_ARG: return "RB_ERR_INVALID_ARG";
        case RB_ERR_UNSUPPORTED: return "RB_ERR_UNSUPPORTED";
        case RB_ERR_ALIGNMENT: return "RB_ERR_ALIGNMENT";
        case RB_ERR_WORKSPACE: return "RB_ERR_WORKSPACE";
        case RB_ERR_CUDA: return "RB_ERR_CUDA";
        case RB_ERR_DEVICE: return "RB_ERR_DEVICE";
    }
    return "RB_ERR_UNKNOWN";
}

const char* rb_last_error(void) { return g_last_error.c_str(); }

rb_status rb_pack(const void* W, rb_dtype w_dtype, int64_t ldw, rb_layout L,
                  uint32_t* planes, float* alpha, void* alpha_f16, void* stream) {
    g_last_error.clear();
    rb_status st = check_layout(L);
    if (st != RB_OK) return st;
    if (!W || !planes || !alpha) return fail(RB_ERR_INVALID_ARG, "null W, planes or alpha");
    if (!valid_dtype(w_dtype)) return fail(RB_ERR_INVALID_ARG, "bad w_dtype %d", (int)w_dtype);
    if (ldw < L.K) return fail(RB_ERR_INVALID_ARG, "ldw=%lld < K=%lld", (long long)ldw, (long long)L.K);
    if (!aligned16(W) || (ldw * dtype_size(w_dtype)) % 16 != 0)
        return fail(RB_ERR_ALIGNMENT, "W and its row pitch must be 16-byte aligned");
    if (!aligned16(planes)) return fail(RB_ERR_ALIGNMENT, "planes must be 16-byte aligned");
    if ((reinterpret_cast<uintptr_t>(alpha) & 3u) || (reinterpret_cast<uintptr_t>(alpha_f16) & 1u))
        return fail(RB_ERR_ALIGNMENT, "alpha must be 4-byte aligned, alpha_f16 2-byte aligned");
    if (L.group == 0 && L.K > 65536) return fail(RB_ERR_UNSUPPORTED, "one scale per row supports K <= 65536");
    PackArgs a{W, ldw, L.M, L.K, L.n_paths, L.group, w_dtype == RB_F16, L.order == RB_SLICED, planes, alpha,
               static_cast<__half*>(alpha_f16)};
    cudaError_t e = launch_pack(a, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "rb_pack launch");
    return RB_OK;
}

size_t rb_gemv_workspace_bytes(rb_layout L, int32_t T) {
    if (check_layout(L) != RB_OK || T < 1) return 0;
    GvPlan pl = gemv_plan_single(L.M, L.K, L.n_paths, L.group, T, device_sm_count());
    return gv_ws_bytes(pl);
}

static rb_status check_gemv_common(const void* alpha, rb_dtype alpha_dtype, rb_dtype y_dtype, int32_t T) {
    if (!valid_dtype(alpha_dtype) || !valid_dtype(y_dtype)) return fail(RB_ERR_INVALID_ARG, "bad dtype");
    if (T < 1 || T > 64) return fail(RB_ERR_UNSUPPORTED, "T=%d outside 1..64", T);
    if (reinterpret_cast<uintptr_t>(alpha) & (dtype_size(alpha_dtype) - 1))
        return fail(RB_ERR_ALIGNMENT, "alpha misaligned for its dtype");
    return RB_OK;
}

// rb_gemv, and rb_gemv_swiglu with `gated` (the planes and scales then hold
// 2 L.n_paths paths: the gate's, then the up projection's)
static rb_status gemv_one(const uint32_t* planes, const void* alpha, rb_dtype alpha_dtype, rb_layout L,
                          const void* x, int64_t ldx, int32_t T, void* y, rb_dtype y_dtype, int64_t ldy,
                          void* workspace, size_t ws_bytes, void* stream, bool gated) {
    g_last_error.clear();
    rb_status st = check_layout(L);
    if (st != RB_OK) return st;
    if (gated && L.n_paths > 4) return fail(RB_ERR_UNSUPPORTED, "rb_gemv_swiglu takes 1..4 paths per matrix");
    if (!planes || !alpha || !x || !y) return fail(RB_ERR_INVALID_ARG, "null planes, alpha, x or y");
    if ((st = check_gemv_common(alpha, alpha_dtype, y_dtype, T)) != RB_OK) return st;
    if (ldx < L.K || ldy < L.M) return fail(RB_ERR_INVALID_ARG, "ldx < K or ldy < M");
    if (!aligned16(planes) || !aligned16(x) || (ldx * 2) % 16 != 0)
        return fail(RB_ERR_ALIGNMENT, "planes, x and the row pitch of x must be 16-byte aligned");
    if (reinterpret_cast<uintptr_t>(y) & (dtype_size(y_dtype) - 1)) return fail(RB_ERR_ALIGNMENT, "y misaligned");
    const int sms = device_sm_count();
    const int np = gated ? 2 * L.n_paths : L.n_paths;
    GvPlan pl = gemv_plan_single(L.M, L.K, np, L.group, T, sms, gated);
    const size_t need = gv_ws_bytes(pl);
    if (!workspace || ws_bytes < need || !aligned16(workspace))
        return fail(RB_ERR_WORKSPACE, "workspace needs %zu bytes (16-byte aligned), got %zu", need, ws_bytes);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    GvArgs a{};
    a.one = GvJob{planes, alpha, x, y, L.M, L.K};
    a.jobs = nullptr;
    a.n_jobs = 1;
    a.n_paths = np;
    a.swiglu = gated ? 1 : 0;
    a.group = L.group;
    a.sliced = L.order == RB_SLICED;
    a.alpha_f16 = alpha_dtype == RB_F16;
    a.y_f16 = y_dtype == RB_F16;
    a.T = T;
    a.ldx = ldx;
    a.ldy = ldy;
    a.chunk_slices = pl.chunk_slices;
    a.workspace = workspace;
    a.ws_bytes = ws_bytes;
    a.expect_units = static_cast<uint32_t>(pl.units);
    a.expect_ctrs = static_cast<uint32_t>(pl.counters);
    a.expect_parts = static_cast<uint32_t>(pl.partials);
    const cudaError_t e = launch_gemv(a, pl, s);
    if (e != cudaSuccess) return cuda_fail(e, gated ? "rb_gemv_swiglu launch" : "rb_gemv launch");
    return RB_OK;
}

rb_status rb_gemv(const uint32_t* planes, const void* alpha, rb_dtype alpha_dtype, rb_layout L, const void* x,
                  int64_t ldx, int32_t T, void* y, rb_dtype y_dtype, int64_t ldy, void* workspace, size_t ws_bytes,
                  void* stream) {
    return gemv_one(planes, alpha, alpha_dtype, L, x, ldx, T, y, y_dtype, ldy, workspace, ws_bytes, stream, false);
}

rb_status rb_gemv_swiglu(const uint32_t* planes, const void* alpha, rb_dtype alpha_dtype, rb_layout L,
                         const void* x, int64_t ldx, int32_t T, void* h, rb_dtype h_dtype, int64_t ldh,
                         void* workspace, size_t ws_bytes, void* stream) {
    return gemv_one(planes, alpha, alpha_dtype, L, x, ldx, T, h, h_dtype, ldh, workspace, ws_bytes, stream, true);
}

size_t rb_gemv_swiglu_workspace_bytes(rb_layout L, int32_t T) {
    if (check_layout(L) != RB_OK || L.n_paths > 4 || T < 1) return 0;
    GvPlan pl = gemv_plan_single(L.M, L.K, 2 * L.n_paths, L.group, T, device_sm_count(), true);
    return gv_ws_bytes(pl);
}

static rb_status check_descs(const rb_gemv_desc* d, int32_t n, int32_t n_paths, int32_t group, int32_t order,
                             rb_dtype alpha_dtype, rb_dtype y_dtype) {
    if (!d) return fail(RB_ERR_INVALID_ARG, "null descriptors");
    if (n < 1 || n > gemv_max_jobs()) return fail(RB_ERR_UNSUPPORTED, "n=%d outside 1..%d", n, gemv_max_jobs());
    if (!valid_dtype(alpha_dtype) || !valid_dtype(y_dtype)) return fail(RB_ERR_INVALID_ARG, "bad dtype");
    for (int32_t i = 0; i < n; ++i) {
        rb_layout L{d[i].M, d[i].K, n_paths, group, order, 0};
        rb_status st = check_layout(L);
        if (st != RB_OK) return fail(st, "descriptor %d: %s", i, g_last_error.c_str());
        if (!d[i].planes || !d[i].alpha || !d[i].x || !d[i].y)
            return fail(RB_ERR_INVALID_ARG, "descriptor %d has a null pointer", i);
        if (!aligned16(d[i].planes) || !aligned16(d[i].x))
            return fail(RB_ERR_ALIGNMENT, "descriptor %d: planes and x must be 16-byte aligned", i);
        if (reinterpret_cast<uintptr_t>(d[i].alpha) & (dtype_size(alpha_dtype) - 1))
            return fail(RB_ERR_ALIGNMENT, "descriptor %d: alpha misaligned for its dtype", i);
        if (reinterpret_cast<uintptr_t>(d[i].y) & (dtype_size(y_dtype) - 1))
            return fail(RB_ERR_ALIGNMENT, "descriptor %d: y misaligned for its dtype", i);
    }
    return RB_OK;
}

size_t rb_gemv_grouped_workspace_bytes(const rb_gemv_desc* descs_host, int32_t n, int32_t n_paths, int32_t T) {
    if (!descs_host || n < 1 || n_paths < 1 || n_paths > 8 || T < 1) return 0;
    // the scale granularity does not change the plan's size bound: use the
    // larger of the two row-block sizes' counts
    size_t best = 0;
    for (int group : {0, 128}) {
        GvPlan pl = gemv_plan_grouped(reinterpret_cast<const GvJob*>(descs_host), n, n_paths, group, T);
        const size_t b = gv_ws_bytes(pl);
        if (b > best) best = b;
    }
    return best;
}

rb_status rb_gemv_grouped(const rb_gemv_desc* descs_host, const rb_gemv_desc* descs_dev,
                          int32_t n, int32_t n_paths, int32_t group, int32_t order,
                          rb_dtype alpha_dtype, rb_dtype y_dtype, int32_t T,
                          void* workspace, size_t ws_bytes, void* stream) {
    g_last_error.clear();
    static_assert(sizeof(rb_gemv_desc) == sizeof(GvJob), "descriptor layout");
    rb_status st = check_descs(descs_host, n, n_paths, group, order, alpha_dtype, y_dtype);
    if (st != RB_OK) return st;
    if (!descs_dev || (reinterpret_cast<uintptr_t>(descs_dev) & 7u))
        return fail(RB_ERR_INVALID_ARG, "descs_dev must be a non-null, 8-byte aligned device pointer");
    if ((st = check_gemv_common(descs_host[0].alpha, alpha_dtype, y_dtype, T)) != RB_OK) return st;
    GvPlan pl = gemv_plan_grouped(reinterpret_cast<const GvJob*>(descs_host), n, n_paths, group, T);
    const size_t need = gv_ws_bytes(pl);
    if (!workspace || ws_bytes < need || !aligned16(workspace))
        return fail(RB_ERR_WORKSPACE, "workspace needs %zu bytes (16-byte aligned), got %zu", need, ws_bytes);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    GvArgs a{};
    a.one = GvJob{};
    a.jobs = reinterpret_cast<const GvJob*>(descs_dev);
    a.n_jobs = n;
    a.n_paths = n_paths;
    a.group = group;
    a.sliced = order == RB_SLICED;
    a.alpha_f16 = alpha_dtype == RB_F16;
    a.y_f16 = y_dtype == RB_F16;
    a.T = T;
    a.ldx = 0;
    a.ldy = 0;
    a.chunk_slices = pl.chunk_slices;
    a.workspace = workspace;
    a.ws_bytes = ws_bytes;
    a.expect_units = static_cast<uint32_t>(pl.units);
    a.expect_ctrs = static_cast<uint32_t>(pl.counters);
    a.expect_parts = static_cast<uint32_t>(pl.partials);
    const cudaError_t e = launch_gemv(a, pl, s);
    if (e != cudaSuccess) return cuda_fail(e, "rb_gemv_grouped launch");
    return RB_OK;
}

rb_status rb_pack_fixed(const void* W, rb_dtype w_dtype, int64_t ldw, rb_layout L, const float* h, const float* g,
                        uint32_t* planes, void* stream) {
    g_last_error.clear();
    rb_status st = check_layout(L);
    if (st != RB_OK) return st;
    if (!W || !h || !planes) return fail(RB_ERR_INVALID_ARG, "null W, h or planes");
    if (L.group != 0) return fail(RB_ERR_UNSUPPORTED, "given scales are per row (h) and per column (g): group must be 0");
    if (!valid_dtype(w_dtype)) return fail(RB_ERR_INVALID_ARG, "bad w_dtype %d", (int)w_dtype);
    if (ldw < L.K) return fail(RB_ERR_INVALID_ARG, "ldw=%lld < K=%lld", (long long)ldw, (long long)L.K);
    if (!aligned16(W) || (ldw * dtype_size(w_dtype)) % 16 != 0)
        return fail(RB_ERR_ALIGNMENT, "W and its row pitch must be 16-byte aligned");
    if (!aligned16(planes)) return fail(RB_ERR_ALIGNMENT, "planes must be 16-byte aligned");
    if ((reinterpret_cast<uintptr_t>(h) & 3u) || (reinterpret_cast<uintptr_t>(g) & 3u))
        return fail(RB_ERR_ALIGNMENT, "h and g must be 4-byte aligned");
    cudaError_t e = launch_pack_fixed(W, w_dtype == RB_F16, ldw, L.M, L.K, L.n_paths, L.order == RB_SLICED, h, g, planes,
                                      static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "rb_pack_fixed launch");
    return RB_OK;
}

size_t rb_dual_gemv_workspace_bytes(rb_layout L, int32_t T) {
    if (check_layout(L) != RB_OK || L.group != 0 || T < 1 || T > 64) return 0;
    return dual_plan(L.M, L.K, L.n_paths, T, true).total;
}

rb_status rb_dual_gemv(const uint32_t* planes, rb_layout L, const float* h, const float* g, const void* x, int64_t ldx,
                       int32_t T, void* y, rb_dtype y_dtype, int64_t ldy, void* workspace, size_t ws_bytes,
                       void* stream) {
    g_last_error.clear();
    rb_status st = check_layout(L);
    if (st != RB_OK) return st;
    if (!planes || !h || !x || !y) return fail(RB_ERR_INVALID_ARG, "null planes, h, x or y");
    if (L.group != 0) return fail(RB_ERR_UNSUPPORTED, "given scales are per row (h) and per column (g): group must be 0");
    if ((st = check_gemv_common(h, RB_F32, y_dtype, T)) != RB_OK) return st;
    if ((reinterpret_cast<uintptr_t>(g) & 3u)) return fail(RB_ERR_ALIGNMENT, "g must be 4-byte aligned");
    if (ldx < L.K || ldy < L.M) return fail(RB_ERR_INVALID_ARG, "ldx < K or ldy < M");
    if (!aligned16(planes) || !aligned16(x) || (ldx * 2) % 16 != 0)
        return fail(RB_ERR_ALIGNMENT, "planes, x and the row pitch of x must be 16-byte aligned");
    if (reinterpret_cast<uintptr_t>(y) & (dtype_size(y_dtype) - 1)) return fail(RB_ERR_ALIGNMENT, "y misaligned");
    const DualPlan d = dual_plan(L.M, L.K, L.n_paths, T, true);
    if (!workspace || ws_bytes < d.total || !aligned16(workspace))
        return fail(RB_ERR_WORKSPACE, "workspace needs %zu bytes (16-byte aligned), got %zu", d.total, ws_bytes);
    cudaError_t e = launch_dual_gemv(planes, L.order == RB_SLICED, L.M, L.K, L.n_paths, h, g, x, ldx, T, y,
                                     y_dtype == RB_F16, ldy, workspace, d, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "rb_dual_gemv launch");
    return RB_OK;
}

// rb_gemm_from_weight workspace: the rb_gemm workspace, then the planes, the
// fp32 scales and (one scale per 128 columns) their fp16 copy, each
// starting on a 256-byte boundary
struct FromWeightLayout {
    size_t gemm, planes, alpha, alpha16, total;
};
static FromWeightLayout from_weight_layout(rb_layout L, int32_t T) {
    auto a256 = [](size_t b) { return (b + 255) & ~size_t(255); };
    FromWeightLayout f{};
    f.gemm = a256(rb_gemm_workspace_bytes(L, T));
    f.planes = a256(rb_planes_words(L) * 4);
    f.alpha = a256(rb_scales_count(L) * 4);
    f.alpha16 = L.group ? a256(rb_scales_count(L) * 2) : 0;
    f.total = (f.gemm && f.planes) ? f.gemm + f.planes + f.alpha + f.alpha16 : 0;
    return f;
}

size_t rb_gemm_from_weight_workspace_bytes(rb_layout L, int32_t T) {
    if (check_layout(L) != RB_OK || T < 1 || L.n_paths > 4) return 0;
    return from_weight_layout(L, T).total;
}

rb_status rb_gemm_from_weight(const void* W, rb_dtype w_dtype, int64_t ldw, rb_layout L, const void* X, int64_t ldx,
                              int32_t T, void* Y, rb_dtype y_dtype, int64_t ldy, void* workspace, size_t ws_bytes,
                              void* stream) {
    g_last_error.clear();
    rb_status st = check_layout(L);
    if (st != RB_OK) return st;
    // everything rb_pack and rb_gemm would refuse is refused here, before
    // either is enqueued
    if (!W || !X || !Y) return fail(RB_ERR_INVALID_ARG, "null W, X or Y");
    if (!valid_dtype(w_dtype) || !valid_dtype(y_dtype)) return fail(RB_ERR_INVALID_ARG, "bad dtype");
    if (L.n_paths > 4) return fail(RB_ERR_UNSUPPORTED, "rb_gemm supports 1..4 paths");
    if (ldw < L.K) return fail(RB_ERR_INVALID_ARG, "ldw=%lld < K=%lld", (long long)ldw, (long long)L.K);
    if (!aligned16(W) || (ldw * dtype_size(w_dtype)) % 16 != 0)
        return fail(RB_ERR_ALIGNMENT, "W and its row pitch must be 16-byte aligned");
    if (L.group == 0 && L.K > 65536) return fail(RB_ERR_UNSUPPORTED, "one scale per row supports K <= 65536");
    if (T < 1 || T > (1 << 22)) return fail(RB_ERR_UNSUPPORTED, "T=%d outside 1..2^22", T);
    if (ldx < L.K || ldy < L.M) return fail(RB_ERR_INVALID_ARG, "ldx < K or ldy < M");
    if (!aligned16(X) || (ldx * 2) % 16 != 0) return fail(RB_ERR_ALIGNMENT, "X and its row pitch must be 16-byte aligned");
    if (reinterpret_cast<uintptr_t>(Y) & (dtype_size(y_dtype) - 1)) return fail(RB_ERR_ALIGNMENT, "Y misaligned");
    const FromWeightLayout f = from_weight_layout(L, T);
    if (!workspace || ws_bytes < f.total || !aligned16(workspace))
        return fail(RB_ERR_WORKSPACE, "workspace needs %zu bytes (16-byte aligned), got %zu", f.total, ws_bytes);
    char* ws = static_cast<char*>(workspace);
    uint32_t* planes = reinterpret_cast<uint32_t*>(ws + f.gemm);
    float* alpha = reinterpret_cast<float*>(ws + f.gemm + f.planes);
    void* alpha16 = L.group ? ws + f.gemm + f.planes + f.alpha : nullptr;
    if ((st = rb_pack(W, w_dtype, ldw, L, planes, alpha, alpha16, stream)) != RB_OK) return st;
    return rb_gemm(planes, L.group ? alpha16 : alpha, L.group ? RB_F16 : RB_F32, L, X, ldx, T, Y, y_dtype, ldy,
                   workspace, f.gemm, stream);
}

size_t rb_gemm_workspace_bytes(rb_layout L, int32_t T) {
    if (check_layout(L) != RB_OK || T < 1) return 0;
    if (T > GEMM_DEC_MAX_T) return GEMM_HEADER_BYTES;
    const GemmDecPlan pl = gemm_dec_plan(L.M, L.K, L.n_paths, L.group, T, device_sm_count());
    return GEMM_HEADER_BYTES + pl.counters_bytes + pl.partials_bytes + pl.xp_bytes;
}

rb_status rb_gemm(const uint32_t* planes, const void* alpha, rb_dtype alpha_dtype, rb_layout L,
                  const void* X, int64_t ldx, int32_t T, void* Y, rb_dtype y_dtype, int64_t ldy,
                  void* workspace, size_t ws_bytes, void* stream) {
    g_last_error.clear();
    rb_status st = check_layout(L);
    if (st != RB_OK) return st;
    if (!planes || !alpha || !X || !Y) return fail(RB_ERR_INVALID_ARG, "null planes, alpha, X or Y");
    if (!valid_dtype(alpha_dtype) || !valid_dtype(y_dtype)) return fail(RB_ERR_INVALID_ARG, "bad dtype");
    if (L.n_paths > 4) return fail(RB_ERR_UNSUPPORTED, "rb_gemm supports 1..4 paths");
    if (L.group == 128 && alpha_dtype != RB_F16)
        return fail(RB_ERR_UNSUPPORTED, "rb_gemm with one scale per 128 columns takes fp16 scales "
                                        "(they are folded exactly into the fp16 operand)");
    if (T < 1 || T > (1 << 22)) return fail(RB_ERR_UNSUPPORTED, "T=%d outside 1..2^22", T);
    if (ldx < L.K || ldy < L.M) return fail(RB_ERR_INVALID_ARG, "ldx < K or ldy < M");
    if (!aligned16(planes) || !aligned16(X) || (ldx * 2) % 16 != 0)
        return fail(RB_ERR_ALIGNMENT, "planes, X and the row pitch of X must be 16-byte aligned");
    if (reinterpret_cast<uintptr_t>(alpha) & (dtype_size(alpha_dtype) - 1))
        return fail(RB_ERR_ALIGNMENT, "alpha misaligned for its dtype");
    if (reinterpret_cast<uintptr_t>(Y) & (dtype_size(y_dtype) - 1)) return fail(RB_ERR_ALIGNMENT, "Y misaligned");
    const bool dec = T <= GEMM_DEC_MAX_T;
    GemmDecPlan pl{};
    size_t need = GEMM_HEADER_BYTES;
    if (dec) {
        pl = gemm_dec_plan(L.M, L.K, L.n_paths, L.group, T, device_sm_count());
        need += pl.counters_bytes + pl.partials_bytes + pl.xp_bytes;
    }
    if (!workspace || ws_bytes < need || !aligned16(workspace))
        return fail(RB_ERR_WORKSPACE, "workspace needs %zu bytes (16-byte aligned), got %zu", need, ws_bytes);
    // no memset: the decode path's operand pre-pass clears the error word
    // and the arrival counters, the prefill kernel clears the error word
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (dec)
        e = launch_gemm_dec(planes, alpha, alpha_dtype == RB_F16, L.M, L.K, L.n_paths, L.group, L.order == RB_SLICED,
                            X, ldx, T, Y, y_dtype == RB_F16, ldy, workspace, pl, s);
    else
        e = launch_gemm_prefill(planes, alpha, alpha_dtype == RB_F16, L.M, L.K, L.n_paths, L.group,
                                L.order == RB_SLICED, X, ldx, T, Y, y_dtype == RB_F16, ldy,
                                static_cast<uint32_t*>(workspace) + 1, false, s);
    if (e == cudaErrorNotSupported) return fail(RB_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
    if (e != cudaSuccess) return cuda_fail(e, "rb_gemm launch");
    return RB_OK;
}

rb_status rb_gemm_reconstruct(const uint32_t* planes, const void* alpha, rb_dtype alpha_dtype, rb_layout L,
                              const void* X, int64_t ldx, int32_t T, void* Y, rb_dtype y_dtype, int64_t ldy,
                              void* workspace, size_t ws_bytes, void* stream) {
    g_last_error.clear();
    rb_status st = check_layout(L);
    if (st != RB_OK) return st;
    if (!planes || !alpha || !X || !Y) return fail(RB_ERR_INVALID_ARG, "null planes, alpha, X or Y");
    if (!valid_dtype(alpha_dtype) || !valid_dtype(y_dtype)) return fail(RB_ERR_INVALID_ARG, "bad dtype");
    if (L.n_paths != 2 || L.group != 0)
        return fail(RB_ERR_UNSUPPORTED, "rb_gemm_reconstruct takes two paths with one scale per row");
    if (T < 1 || T > (1 << 22)) return fail(RB_ERR_UNSUPPORTED, "T=%d outside 1..2^22", T);
    if (ldx < L.K || ldy < L.M) return fail(RB_ERR_INVALID_ARG, "ldx < K or ldy < M");
    if (!aligned16(planes) || !aligned16(X) || (ldx * 2) % 16 != 0)
        return fail(RB_ERR_ALIGNMENT, "planes, X and the row pitch of X must be 16-byte aligned");
    if (reinterpret_cast<uintptr_t>(alpha) & (dtype_size(alpha_dtype) - 1))
        return fail(RB_ERR_ALIGNMENT, "alpha misaligned for its dtype");
    if (reinterpret_cast<uintptr_t>(Y) & (dtype_size(y_dtype) - 1)) return fail(RB_ERR_ALIGNMENT, "Y misaligned");
    if (!workspace || ws_bytes < GEMM_HEADER_BYTES || !aligned16(workspace))
        return fail(RB_ERR_WORKSPACE, "workspace needs %zu bytes (16-byte aligned), got %zu",
                    (size_t)GEMM_HEADER_BYTES, ws_bytes);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const cudaError_t e = launch_gemm_prefill(planes, alpha, alpha_dtype == RB_F16, L.M, L.K, 2, 0, L.order == RB_SLICED, X, ldx, T, Y,
                            y_dtype == RB_F16, ldy, static_cast<uint32_t*>(workspace) + 1, true, s);
    if (e == cudaErrorNotSupported) return fail(RB_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
    if (e != cudaSuccess) return cuda_fail(e, "rb_gemm_reconstruct launch");
    return RB_OK;
}

// Wait for `stream`, then read word 1 (the error flags) of a workspace header.
static rb_status read_flags(const void* header, void* stream, const char* who, uint32_t* flags) {
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(flags, static_cast<const uint32_t*>(header) + 1, sizeof(uint32_t),
                                    cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_fail(e, who);
    return RB_OK;
}

rb_status rb_gemm_check(const void* workspace, void* stream) {
    g_last_error.clear();
    if (!workspace) return fail(RB_ERR_INVALID_ARG, "null workspace");
    uint32_t flag = 0;
    rb_status st = read_flags(workspace, stream, "rb_gemm_check", &flag);
    if (st != RB_OK) return st;
    if (flag)
        return fail(RB_ERR_DEVICE, "rb_gemm kernel flag 0x%x: a pipeline wait ran out in (%s%s%s%s)", flag,
                    (flag & 1u) ? "X-tile producer " : "", (flag & 2u) ? "MMA issuer " : "",
                    (flag & 4u) ? "operand expansion " : "", (flag & 8u) ? "epilogue" : "");
    return RB_OK;
}

rb_status rb_gemv_check(const void* workspace, void* stream) {
    g_last_error.clear();
    const void* header = workspace;
    if (!header) {
        // the static scratch of rb_gemv_noalloc on the current device
        void* p = nullptr;
        cudaError_t e = noalloc_scratch(&p);
        if (e != cudaSuccess) return cuda_fail(e, "rb_gemv_check (static scratch)");
        header = p;
    }
    uint32_t flag = 0;
    rb_status st = read_flags(header, stream, "rb_gemv_check", &flag);
    if (st != RB_OK) return st;
    if (flag)
        return fail(RB_ERR_DEVICE, "matvec kernel flag 0x%x (%s%s%s%s)", flag,
                    (flag & GV_ERR_SMEM_LAYOUT) ? "shared-memory window not where the tables need it; " : "",
                    (flag & GV_ERR_BAD_JOB) ? "device descriptors differ from the host copy the launch was "
                                              "planned on; " : "",
                    (flag & GV_ERR_TOO_MANY_JOBS) ? "more descriptors than a launch takes; " : "",
                    (flag & GV_ERR_COUNTER) ? "an arrival counter was not zero (workspace not zeroed before its "
                                              "first use)" : "");
    return RB_OK;
}

}  // extern "C"
