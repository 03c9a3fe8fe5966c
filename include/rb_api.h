/*
 * rb_api.h -- C ABI of the residual-binary-weight linear layer on B200 (sm_100a).
 *
 * A linear layer W (M x K) is stored as W ~= sum_k alpha_k (.) B_k with N binary
 * planes B_k in {-1, +1}^(M x K) and non-negative scales alpha_k, one per row
 * or one per 128 input columns of each row.
 *
 *   RaBiT: Residual-Aware Binarization Training (arXiv 2602.05367),
 *     section 4.1  -- binary cores with per-channel scale vectors, evaluated
 *                     with additions and subtractions, k = 2 paths;
 *     section 4.2  -- every path derived in turn from one shared
 *                     full-precision weight, the residual updated after each;
 *     appendix A   -- R1 = W_FP - W^_1, B2 = sign(R1);
 *     appendix D   -- bit-packed binary GEMV, 32 columns per uint32.
 *   QBB: Quantization with Binary Bases for LLMs (atlas.scime.ai summary),
 *     Approach / Key results -- N = 4 binary bases, fp16 scales, one scale
 *     per 128 input columns (W(4x1)A16g128), cascaded analytical residual
 *     initialisation.
 *
 * Conventions shared by every call
 * --------------------------------
 * - Pointers marked "device" must be CUDA device memory of the current device;
 *   the caller owns every buffer. Calls never allocate device memory.
 * - Every call that takes `stream` (a cudaStream_t, NULL for the legacy
 *   default stream) only enqueues work and returns; results are ready when the
 *   stream reaches that point. Stream order holds for the inputs: a call sees
 *   everything earlier work on the stream wrote. (The matvec and decode
 *   kernels are programmatic dependent launches that start while the
 *   previous kernel ends; before they wait for it they only set up, and a
 *   single-matrix matvec prefetches its first planes into L2, which reads
 *   no stale data.)
 * - Arguments are validated on the host before anything is enqueued; a call
 *   that returns an error has enqueued nothing, except where stated.
 * - Plane words: bit j of word w of a row holds column 32*w + j (least
 *   significant bit first); a set bit means +1; sign(0) = +1, including -0.0.
 *   (The paper fixes 32 columns per uint32 but not the bit order or the
 *   polarity; this is the reading the library uses.) Two word orders:
 *     RB_ROWS    [N][M][K/32], row-major: the interchange order.
 *     RB_SLICED  the order the matvec kernels stream: for each path k and each
 *                512-column slice s (S = ceil(K/512) slices), the 16 words of
 *                that slice of every row, row after row. Word v of slice s of
 *                row i of path k sits at ((k*S + s)*M + i)*16 + v. In the last
 *                slice the words past K/32 are padding (rb_pack writes 0).
 * - Scales: [N][M][K/G] with G = K (group = 0) or G = 128 (group = 128).
 * - K must be a positive multiple of 128, M positive, N in 1..8.
 * - Non-finite weights or activations are outside the contract.
 */
#ifndef RB_API_H
#define RB_API_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define RB_API __attribute__((visibility("default")))
#else
#define RB_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    RB_OK = 0,
    RB_ERR_INVALID_ARG = 1,   /* null pointer, bad size or leading dimension */
    RB_ERR_UNSUPPORTED = 2,   /* valid request the kernels do not implement */
    RB_ERR_ALIGNMENT = 3,     /* pointer or row pitch not 16-byte aligned */
    RB_ERR_WORKSPACE = 4,     /* workspace missing or smaller than required */
    RB_ERR_CUDA = 5,          /* a CUDA runtime call or kernel launch failed */
    RB_ERR_DEVICE = 6         /* a kernel reported a failure through its flag */
} rb_status;

typedef enum { RB_F32 = 0, RB_F16 = 1 } rb_dtype;

typedef enum { RB_ROWS = 0, RB_SLICED = 1 } rb_order;

typedef struct {
    int64_t M;        /* output rows (> 0) */
    int64_t K;        /* input columns (> 0, multiple of 128) */
    int32_t n_paths;  /* N, 1..8 */
    int32_t group;    /* 0: one scale per row; 128: one scale per 128 columns */
    int32_t order;    /* plane word order, an rb_order */
    int32_t reserved; /* must be 0 */
} rb_layout;

/* Number of uint32 plane words: N*M*K/32 (RB_ROWS) or N*M*16*ceil(K/512)
 * (RB_SLICED); 0 for an invalid layout. */
RB_API size_t rb_planes_words(rb_layout L);

/* Number of scales, N * M * (K / G) (0 for an invalid layout). */
RB_API size_t rb_scales_count(rb_layout L);

/* Human-readable name of a status code (static string). */
RB_API const char* rb_status_string(rb_status s);

/* Detail of the last error returned on the calling host thread ("" if none). */
RB_API const char* rb_last_error(void);

/*
 * rb_pack -- derive N residual sign planes and their scales from one shared
 * full-precision weight (RaBiT section 4.2 and appendix G; QBB cascaded
 * analytical residual initialisation). For each row, or each 128-column
 * group of a row:
 *     R_0 = W;  for k = 1..N:  B_k = sign(R_{k-1})  (sign(0) = +1),
 *     alpha_k = mean |R_{k-1}| over the row or group,
 *     R_k = R_{k-1} - alpha_k * B_k.
 * Arithmetic: residuals in fp32, sums of |R| accumulated in fp64, alpha_k
 * rounded to fp32 and that fp32 value used in the residual update.
 *
 * W         device, M rows of K elements, row pitch `ldw` elements (>= K);
 *           w_dtype RB_F16 or RB_F32. Base and row pitch 16-byte aligned.
 * planes    device, out, rb_planes_words(L) words in L.order, 16-byte aligned.
 * alpha     device, out, rb_scales_count(L) fp32 scales.
 * alpha_f16 device, out, nullable: the same scales rounded to nearest fp16.
 * Errors: RB_ERR_INVALID_ARG / UNSUPPORTED / ALIGNMENT before launch;
 *         RB_ERR_CUDA if the launch fails. One scale per row supports
 *         K <= 65536.
 */
RB_API rb_status rb_pack(const void* W, rb_dtype w_dtype, int64_t ldw, rb_layout L,
                  uint32_t* planes, float* alpha, void* alpha_f16, void* stream);

/*
 * rb_gemv -- y_t = sum_k alpha_k (.) (B_k x_t) for a small batch of tokens
 * (RaBiT section 4.1, appendix D: matmul-free evaluation, all paths in one
 * pass). Runs on CUDA cores: each 8-column block of x is expanded once into a
 * shared-memory table of its 256 signed sums (built as 2 * masked sum - block
 * sum), and every plane byte then costs one table lookup and one add.
 *
 * planes    device, rb_planes_words(L) words in L.order (RB_SLICED streams
 *           contiguous 32 KB tiles; RB_ROWS reads 64-byte pieces per row).
 * alpha     device, rb_scales_count(L) scales of type alpha_dtype.
 * x         device, T rows of K fp16 values, row pitch ldx elements (>= K);
 *           base and row pitch 16-byte aligned.
 * y         device, out, T rows of M values of type y_dtype, pitch ldy >= M.
 * T         tokens, 1..64.
 * workspace device scratch of at least rb_gemv_workspace_bytes(L, T) bytes,
 *           16-byte aligned, ZEROED ONCE before its first use (cudaMemset);
 *           every call leaves its arrival counters at zero again, so no
 *           clearing is needed between calls (the kernel clears the error
 *           word itself; no memset is enqueued). A workspace zeroed once
 *           serves any later shape that fits it. It must not be shared by
 *           calls that may overlap on the GPU. May be NULL when that size is
 *           0. A counter found non-zero is flagged (rb_gemv_check).
 * Errors: as rb_pack; RB_ERR_WORKSPACE if the workspace is too small. A
 *         kernel-side failure is recorded in the workspace; rb_gemv_check()
 *         reads it back.
 */
RB_API rb_status rb_gemv(const uint32_t* planes, const void* alpha, rb_dtype alpha_dtype,
                  rb_layout L, const void* x, int64_t ldx, int32_t T,
                  void* y, rb_dtype y_dtype, int64_t ldy,
                  void* workspace, size_t ws_bytes, void* stream);

RB_API size_t rb_gemv_workspace_bytes(rb_layout L, int32_t T);

/*
 * rb_gemv_swiglu -- h_t = silu(G x_t) (.) (U x_t) for the gated MLP block of
 * the Llama models whose decode speed RaBiT section 5 reports (the pages do
 * not print the block; silu(z) = z / (1 + e^-z) is that architecture's gate),
 * with G and U both residual-binary matrices of layout L:
 *     G x = sum_k alpha^G_k (.) (B^G_k x),   U x = sum_k alpha^U_k (.) (B^U_k x).
 * One launch of the rb_gemv kernel: each unit evaluates the rows of both
 * matrices and its epilogue applies the gate, so G x and U x never reach
 * memory. The down projection that consumes h is a plain rb_gemv.
 *
 * planes    device, 2 * rb_planes_words(L) words: G's L.n_paths planes, then
 *           U's (two rb_pack outputs stored back to back), in L.order.
 * alpha     device, 2 * rb_scales_count(L) scales of type alpha_dtype: G's,
 *           then U's.
 * L         M, K, group, order of both matrices; n_paths = paths of each
 *           (1..4).
 * x, T      as rb_gemv.
 * h         device, out, T rows of M values of type h_dtype, pitch ldh >= M:
 *           silu(g) * u computed in fp32 from the fp32 sums g, u, then
 *           rounded to h_dtype.
 * workspace as rb_gemv, of rb_gemv_swiglu_workspace_bytes(L, T) bytes
 *           (zeroed once before its first use).
 * Errors: as rb_gemv; RB_ERR_UNSUPPORTED for more than 4 paths per matrix.
 */
RB_API rb_status rb_gemv_swiglu(const uint32_t* planes, const void* alpha, rb_dtype alpha_dtype, rb_layout L,
                                const void* x, int64_t ldx, int32_t T, void* h, rb_dtype h_dtype, int64_t ldh,
                                void* workspace, size_t ws_bytes, void* stream);
RB_API size_t rb_gemv_swiglu_workspace_bytes(rb_layout L, int32_t T);

/* One matrix of a grouped matvec; x is [T][K] and y is [T][M], both dense. */
typedef struct {
    const uint32_t* planes;  /* device, rb_planes_words words in the call's order */
    const void* alpha;       /* device, [N][M][K/G] */
    const void* x;           /* device, fp16 [T][K], 16-byte aligned; or pinned
                                host memory mapped for the device (its device
                                address), which the kernel then reads over the
                                bus (zero-copy; on the 7B stack this is slower
                                than one host-to-device copy of all x before
                                the launch: 2.95 against 3.63 TB/s end to end) */
    void* y;                 /* device, [T][M]; or pinned host memory mapped for
                                the device (its device address), which the
                                kernel then writes over the bus */
    int64_t M;
    int64_t K;
} rb_gemv_desc;

/*
 * rb_gemv_grouped -- the same operation over n independent matrices in one
 * persistent launch (a decode step through a stack of layers). The work
 * units (row block, K chunk, token) of all matrices are dealt to the CTAs
 * round robin, in descriptor order; a CTA moves from one unit to the next
 * without draining its load pipeline, so listing the longest matrices
 * first and keeping related matrices adjacent helps.
 *
 * descs_host  host, n descriptors, read for validation and sizing only:
 *             every descriptor's planes and x must be 16-byte aligned, its
 *             alpha and y aligned for their dtypes.
 * descs_dev   device, the same n descriptors (the caller uploads them once).
 *             A device copy that gives another work plan than the host copy
 *             is detected by the kernel, which then does nothing and records
 *             a flag for rb_gemv_check().
 * n           1..2047.  n_paths, group, order (an rb_order), alpha_dtype,
 *             y_dtype: shared by all.
 * T           tokens, 1..64.
 * workspace   device scratch of rb_gemv_grouped_workspace_bytes(...) bytes,
 *             zeroed once before its first use, as for rb_gemv.
 */
RB_API rb_status rb_gemv_grouped(const rb_gemv_desc* descs_host, const rb_gemv_desc* descs_dev,
                          int32_t n, int32_t n_paths, int32_t group, int32_t order,
                          rb_dtype alpha_dtype, rb_dtype y_dtype, int32_t T,
                          void* workspace, size_t ws_bytes, void* stream);

RB_API size_t rb_gemv_grouped_workspace_bytes(const rb_gemv_desc* descs_host, int32_t n,
                                       int32_t n_paths, int32_t T);

/*
 * rb_gemm -- Y_t = sum_k alpha_k (.) (B_k X_t) for a block of T tokens on the
 * tcgen05 tensor cores (RaBiT section 4.1: binary cores with per-channel
 * scales; QBB W(4x1)A16g128 for one scale per 128 columns). The plane bits
 * are expanded exactly to fp16 +-1 (one scale per row: one fp32 accumulator
 * per path in tensor memory, scaled by alpha_k at the end) or to +-alpha_k in
 * fp16 (one scale per 128 columns), multiplied with fp16 X, accumulated in
 * fp32. Two kernels: decode batches (T <= 64) run on a persistent grid that
 * splits the rows x K work evenly over the SMs; prefill blocks (T > 64) run
 * one 128-row x up-to-256-token tile per CTA.
 *
 * planes    device, rb_planes_words(L) words in L.order; 16-byte aligned.
 * alpha     device, rb_scales_count(L) scales of type alpha_dtype. With
 *           group = 128 the scales must be RB_F16 (they become operand
 *           values, which is exact only for fp16); RB_F32 group scales are
 *           refused with RB_ERR_UNSUPPORTED.
 * X         device, fp16 [T][ldx], ldx >= K, base and row pitch 16-byte aligned.
 * Y         device, out, [T][ldy] of type y_dtype, ldy >= M.
 * L         1..4 paths.  T in 1..2^22.
 * workspace device scratch of at least rb_gemm_workspace_bytes(L, T) bytes,
 *           16-byte aligned, owned by the caller: a 256-byte header (word 1
 *           is the call's device error word) and, for T <= 64, arrival
 *           counters, fp32 partial sums and a column-permuted copy of X.
 *           Nothing needs to be zero beforehand: for T <= 64 the call's
 *           operand pre-pass clears the error word and the counters, the
 *           prefill kernel clears the error word (no memset is enqueued).
 *           Calls that may overlap on the GPU need separate workspaces.
 * Errors: validation as rb_gemv (RB_ERR_WORKSPACE if the workspace is too
 *         small); RB_ERR_CUDA if the tensor-map encoder or a launch fails. A
 *         kernel whose bounded pipeline waits ran out records a code in the
 *         workspace header; rb_gemm_check() reports it.
 */
RB_API rb_status rb_gemm(const uint32_t* planes, const void* alpha, rb_dtype alpha_dtype, rb_layout L,
                         const void* X, int64_t ldx, int32_t T, void* Y, rb_dtype y_dtype, int64_t ldy,
                         void* workspace, size_t ws_bytes, void* stream);

/*
 * rb_gemm_reconstruct -- Y_t = W^ X_t with the reconstructed weight
 * W^[i][j] = RN_fp16(alpha_0[i] B_0[i][j] + alpha_1[i] B_1[i][j]) (RaBiT
 * section 4.1, W ~= sum_k alpha_k (.) B_k): the two paths are folded into one
 * fp16 operand per weight (rounded once from the exact sum of the two scales)
 * and contracted in one tcgen05 MMA chain, half the tensor work of rb_gemm.
 * Each weight differs from sum_k alpha_k B_k by at most 2^-11 of its
 * magnitude, so the result is within 2^-11 sum_j |W^_ij x_j| (plus the
 * output rounding) of rb_gemm's. For prefill-sized blocks (any T >= 1).
 *
 * Arguments as rb_gemm; L: two paths, one scale per row (RB_ERR_UNSUPPORTED
 * otherwise). workspace: at least 256 bytes (the header with the error word,
 * read by rb_gemm_check).
 */
RB_API rb_status rb_gemm_reconstruct(const uint32_t* planes, const void* alpha, rb_dtype alpha_dtype, rb_layout L,
                                     const void* X, int64_t ldx, int32_t T, void* Y, rb_dtype y_dtype, int64_t ldy,
                                     void* workspace, size_t ws_bytes, void* stream);

/*
 * rb_gemm_from_weight -- the training forward of a residual-binary layer:
 * the planes and scales are derived afresh from the shared full-precision
 * weight W and contracted with X in one call, as every training step
 * re-derives every path from W_FP (RaBiT section 4.2 and appendix G):
 *     rb_pack(W) into the workspace, then rb_gemm(planes, scales, X).
 * The planes and scales live only in the call's workspace (with one scale
 * per 128 columns the fp16 copy is contracted, as rb_gemm requires). The
 * result equals rb_pack followed by rb_gemm bit for bit.
 *
 * W, w_dtype, ldw  as rb_pack.   X, ldx, T, Y, y_dtype, ldy  as rb_gemm.
 * L         1..4 paths.
 * workspace device scratch of rb_gemm_from_weight_workspace_bytes(L, T)
 *           bytes, 16-byte aligned: the rb_gemm workspace, then the planes
 *           and scales, each on a 256-byte boundary. Nothing needs to be
 *           zero beforehand.
 * Errors: everything rb_pack or rb_gemm would refuse, before either is
 *         enqueued; rb_gemm_check(workspace) reads the device error word.
 */
RB_API rb_status rb_gemm_from_weight(const void* W, rb_dtype w_dtype, int64_t ldw, rb_layout L, const void* X,
                                     int64_t ldx, int32_t T, void* Y, rb_dtype y_dtype, int64_t ldy, void* workspace,
                                     size_t ws_bytes, void* stream);
RB_API size_t rb_gemm_from_weight_workspace_bytes(rb_layout L, int32_t T);

/* Workspace bytes rb_gemm needs for layout L and T tokens on the current
 * device (0 for an invalid layout or T < 1). */
RB_API size_t rb_gemm_workspace_bytes(rb_layout L, int32_t T);

/* rb_gemm_check -- wait for `stream`, then report RB_ERR_DEVICE if the
 * rb_gemm call that used `workspace` recorded a failure, else RB_OK. */
RB_API rb_status rb_gemm_check(const void* workspace, void* stream);

/*
 * rb_pack_fixed -- the sign planes of the dual-scale binary block for scales
 * the caller gives (RaBiT section 4.1: binary cores with per-channel output
 * and input scaling vectors, W^_k = diag(h_k) B_k diag(g_k); section 4.2:
 * paths derived in turn from the shared weight, scales learned). Signs only:
 *     R_0 = W;  for k = 1..N:  B_k = sign(R_{k-1})  (sign(0) = +1),
 *     R_k[i][j] = R_{k-1}[i][j] - h_k[i] g_k[j] B_k[i][j].
 * Arithmetic: residuals in fp32, h_k[i] g_k[j] rounded to fp32 once.
 *
 * W       device, as rb_pack (fp16 or fp32, pitch ldw, 16-byte aligned).
 * L       group must be 0 (the scales are per row and per column).
 * h       device, fp32 [N][M] output-channel scales, 4-byte aligned.
 * g       device, fp32 [N][K] input-channel scales, or NULL for all ones.
 * planes  device, out, rb_planes_words(L) words in L.order.
 * Errors: as rb_pack; RB_ERR_UNSUPPORTED for group != 0.
 */
RB_API rb_status rb_pack_fixed(const void* W, rb_dtype w_dtype, int64_t ldw, rb_layout L, const float* h,
                               const float* g, uint32_t* planes, void* stream);

/*
 * rb_dual_gemv -- the dual-scale block's output for T <= 64 tokens,
 *     y_t = sum_k h_k (.) (B_k x_{k,t}),   x_{k,t} = RN_fp16(g_k (.) x_t)
 * (RaBiT section 4.1). The input scaling is taken as an fp16 activation (the
 * A16 reading): each product g_k[j] x_t[j] is rounded to the nearest fp16
 * (from its exact value) before the binary core sees it. Runs the CUDA-core
 * table matvec once per path (one grouped launch; alpha = h_k), then sums
 * the paths in fp32.
 *
 * planes  device, rb_planes_words(L) words in L.order (group 0).
 * h, g    device fp32 scales as in rb_pack_fixed (g may be NULL).
 * x, y    as rb_gemv (x fp16 [T][ldx]; y [T][ldy] of y_dtype).
 * workspace  device scratch of rb_dual_gemv_workspace_bytes(L, T) bytes,
 *         16-byte aligned, not shared by calls that may overlap on the GPU;
 *         its header's error word is read by rb_gemv_check(workspace, s).
 */
RB_API rb_status rb_dual_gemv(const uint32_t* planes, rb_layout L, const float* h, const float* g, const void* x,
                              int64_t ldx, int32_t T, void* y, rb_dtype y_dtype, int64_t ldy, void* workspace,
                              size_t ws_bytes, void* stream);

RB_API size_t rb_dual_gemv_workspace_bytes(rb_layout L, int32_t T);

/*
 * rb_gemv_noalloc -- rb_gemv for callers that cannot allocate device memory.
 * (An addition of this library; the paper has no counterpart.) Some callers
 * have no way to obtain a workspace: code that runs where cudaMalloc is not
 * allowed or not wanted -- a real-time decode loop that must not take the
 * implicit device synchronisation of an allocation, a plug-in inside a host
 * framework that owns every device buffer, or a fixed-budget deployment that
 * forbids allocations after start-up. For them the scratch rb_gemv keeps in
 * the workspace (error word, arrival counters and K-split partial sums) lives in one static
 * 1 MiB device array per GPU, held by every GPU that loads the library until
 * the process exits. The caller still passes planes, scales, x and y, with
 * the same meaning, layout and checks as rb_gemv.
 *
 * - Shapes whose scratch would exceed 1 MiB (rb_gemv_workspace_bytes(L, T) >
 *   1 MiB) are refused with RB_ERR_UNSUPPORTED before any CUDA call.
 * - The first call on a device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call
 *   before any stream capture.
 * - Every call on a device shares the array (zero-initialised storage; each
 *   call leaves its counters at zero again). Calls whose work may overlap
 *   on the GPU -- on different streams of one device -- race on the array and
 *   must be ordered by the caller.
 * - Nothing here calls cudaMalloc, cudaFree or any allocating routine.
 * - A kernel-side failure is recorded in the array's header like rb_gemv's;
 *   rb_gemv_check(NULL, stream) reports it.
 */
RB_API rb_status rb_gemv_noalloc(const uint32_t* planes, const void* alpha, rb_dtype alpha_dtype,
                                 rb_layout L, const void* x, int64_t ldx, int32_t T,
                                 void* y, rb_dtype y_dtype, int64_t ldy, void* stream);

/*
 * rb_gemv_check -- wait for `stream`, then report RB_ERR_DEVICE if a matvec
 * kernel that used `workspace` recorded a failure, else RB_OK. With
 * workspace = NULL it reads the error word of rb_gemv_noalloc's static
 * scratch on the current device (the last noalloc call there).
 */
RB_API rb_status rb_gemv_check(const void* workspace, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* RB_API_H */
