// Internal declarations shared by the CUDA sources of librb (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace rb {

constexpr unsigned FULL_MASK = 0xffffffffu;

// 32-bit shared-window address of a generic pointer into shared memory.
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------- rb_pack
struct PackArgs {
    const void* W;
    int64_t ldw;
    int64_t M, K;
    int n_paths;
    int group;          // 0 or 128
    bool w_f16;
    bool sliced;        // plane words in the sliced order
    uint32_t* planes;
    float* alpha;
    __half* alpha16;    // nullable
};
cudaError_t launch_pack(const PackArgs& a, cudaStream_t s);

// ---------------------------------------------------------------- rb_gemv
// Must match rb_gemv_desc in include/rb_api.h field by field.
struct GvJob {
    const uint32_t* planes;
    const void* alpha;
    const void* x;
    void* y;
    int64_t M;
    int64_t K;
};

struct GvArgs {
    GvJob one;              // the matrix when `jobs` is null
    const GvJob* jobs;      // device array of n_jobs descriptors (grouped)
    int n_jobs;
    int n_paths;
    int group;              // 0 or 128
    bool sliced;            // plane words in the sliced order
    bool alpha_f16;
    bool y_f16;
    int T;
    int64_t ldx, ldy;       // pitches of the single matrix (grouped: K and M)
    int chunk_slices;       // 512-column slices per K chunk
    void* workspace;
    size_t ws_bytes;
    // the plan the host sized the workspace for; a launch whose device
    // descriptors give another plan flags GV_ERR_BAD_JOB and does nothing
    uint32_t expect_units, expect_ctrs, expect_parts;
    // SiLU-gated pair: the job's paths are those of two matrices of the same
    // shape, [0, n_paths/2) the gate G and [n_paths/2, n_paths) the up
    // projection U, and the output is y = silu(G x) * (U x) (K-split
    // units keep two partial sums per row)
    int swiglu;
};

// Workspace layout: a 256-byte header (word 1: error flags), then one
// arrival counter per (job, row block, token) of every K-split job, then the
// fp32 partial sums of the split jobs.
constexpr size_t GV_HEADER_BYTES = 256;
// Arrival counters of K-split units live in a zone of fixed size right after
// the header, the fp32 partial sums after it: a workspace zeroed once keeps
// zero counters whatever plans later calls use (every call leaves its
// counters at zero, and no plan writes partial sums into the zone). A plan
// with more counters than the zone holds does not split K.
constexpr size_t GV_CTR_ZONE_BYTES = 65536;
constexpr size_t GV_MAX_COUNTERS = GV_CTR_ZONE_BYTES / 4;
// GV_ERR_BAD_JOB: the device descriptors do not give the plan the host sized
// the workspace for (they differ from the host copy)
// GV_ERR_COUNTER: an arrival counter held more than its K chunks (the
// workspace was not zeroed before its first use).
enum : uint32_t { GV_ERR_SMEM_LAYOUT = 1u, GV_ERR_BAD_JOB = 2u, GV_ERR_TOO_MANY_JOBS = 4u, GV_ERR_COUNTER = 8u };

struct GvPlan {
    int rows_per_cta;       // R
    int chunk_slices;
    size_t counters;        // number of uint32 counters
    size_t partials;        // number of fp32 partial sums
    size_t units;
};
int gemv_rows_per_cta(int n_paths, int group);
GvPlan gemv_plan_single(int64_t M, int64_t K, int n_paths, int group, int T, int num_sms, bool swiglu = false);
GvPlan gemv_plan_grouped(const GvJob* host_jobs, int n, int n_paths, int group, int T);
cudaError_t launch_gemv(const GvArgs& a, const GvPlan& plan, cudaStream_t s);
int gemv_max_jobs();

// ---------------------------------------------------------------- rb_gemm
// Workspace: a 256-byte header (word 1: error flags of the call's kernels);
// for decode batches (T <= GEMM_DEC_MAX_T) then the row-tile arrival
// counters, the fp32 partial sums of tiles shared by two CTAs, and the
// column-permuted copy of X.
constexpr size_t GEMM_HEADER_BYTES = 256;
constexpr int GEMM_DEC_MAX_T = 64;

struct GemmDecPlan {
    int64_t tiles, total;   // row tiles, stages (tiles * K / stage width)
    int grid, bn;
    bool f8;                // fp8 operands with X split into four e5m2 terms
    size_t counters_bytes, partials_bytes, xp_bytes;
};
GemmDecPlan gemm_dec_plan(int64_t M, int64_t K, int n_paths, int group, int T, int num_sms);
cudaError_t launch_gemm_dec(const uint32_t* planes, const void* alpha, bool alpha_f16, int64_t M, int64_t K,
                            int n_paths, int group, bool sliced, const void* X, int64_t ldx, int T, void* Y,
                            bool y_f16, int64_t ldy, void* workspace, const GemmDecPlan& plan, cudaStream_t s);
cudaError_t launch_gemm_prefill(const uint32_t* planes, const void* alpha, bool alpha_f16, int64_t M, int64_t K,
                                int n_paths, int group, bool sliced, const void* X, int64_t ldx, int T, void* Y,
                                bool y_f16, int64_t ldy, uint32_t* err, bool reconstruct, cudaStream_t s);

// ------------------------------------------------------- dual-scale block
cudaError_t launch_pack_fixed(const void* W, bool w_f16, int64_t ldw, int64_t M, int64_t K, int N, bool sliced,
                              const float* h, const float* g, uint32_t* planes, cudaStream_t s);

// Workspace of the dual-scale matvec: the grouped matvec's own workspace
// (header with the error word first), N single-path descriptors, the scaled
// activations x_k and the fp32 per-path outputs.
struct DualPlan {
    GvPlan gv;
    size_t gv_bytes, desc_bytes, xk_bytes, yk_bytes, total;
};
DualPlan dual_plan(int64_t M, int64_t K, int N, int T, bool scaled_x);
cudaError_t launch_dual_gemv(const uint32_t* planes, bool sliced, int64_t M, int64_t K, int N, const float* h,
                             const float* g, const void* x, int64_t ldx, int T, void* y, bool y_f16, int64_t ldy,
                             void* workspace, const DualPlan& d, cudaStream_t s);

int device_sm_count();

// Device address of the static scratch array of rb_gemv_noalloc on the
// current device (looked up once per device).
cudaError_t noalloc_scratch(void** out);

}  // namespace rb
