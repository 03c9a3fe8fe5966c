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
};

// Workspace layout: a 256-byte header (word 1: error flags), then one
// arrival counter per (job, row block, token) of every K-split job, then the
// fp32 partial sums of the split jobs.
constexpr size_t GV_HEADER_BYTES = 256;
enum : uint32_t { GV_ERR_SMEM_LAYOUT = 1u, GV_ERR_BAD_JOB = 2u, GV_ERR_TOO_MANY_JOBS = 4u, GV_ERR_WAIT = 8u };

struct GvPlan {
    int rows_per_cta;       // R
    int chunk_slices;
    size_t counters;        // number of uint32 counters
    size_t partials;        // number of fp32 partial sums
    size_t units;
};
int gemv_rows_per_cta(int n_paths, int group);
GvPlan gemv_plan_single(int64_t M, int64_t K, int n_paths, int group, int T, int num_sms);
GvPlan gemv_plan_grouped(const GvJob* host_jobs, int n, int n_paths, int group, int T);
cudaError_t launch_gemv(const GvArgs& a, const GvPlan& plan, cudaStream_t s);
int gemv_max_jobs();

// ---------------------------------------------------------------- rb_gemm
bool gemm_supported(int n_paths, int group);
cudaError_t launch_gemm(const uint32_t* planes, const void* alpha, bool alpha_f16, int64_t M, int64_t K, int n_paths,
                        int group, bool sliced, const void* X, int64_t ldx, int T, void* Y, bool y_f16, int64_t ldy,
                        cudaStream_t s);
cudaError_t gemm_read_error(unsigned int* code);

int device_sm_count();

}  // namespace rb
