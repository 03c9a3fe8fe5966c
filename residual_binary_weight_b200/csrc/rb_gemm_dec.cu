// rb_gemm for decode batches: Y = sum_k alpha_k (.) (B_k X^T) for T <= 64
// tokens on the tcgen05 tensor cores, one persistent CTA per SM.
//
// RaBiT (arXiv 2602.05367) section 4.1: y = sum_k alpha_k (.) (B_k x) with
// B_k in {-1, +1}; QBB W(4x1)A16g128 for the per-128-column scales.
//
// At a few tokens the tensor core has little to do (an M=128, N=16, K=16 MMA
// takes ~14 cycles); what bounds the contraction is turning plane bits into
// fp16 operands, one value per weight and path, and handing stages between
// the warps. The expansion is one shift and one LOP3 per two weights:
//   * The columns of X are permuted once per call (a small pre-pass into the
//     workspace) so that inside every 32-column block position 2k holds
//     column k and position 2k + 1 holds column k + 16.
//   * The fp16x2 operand of positions (2k, 2k + 1) then takes its two signs
//     from bits k and k + 16 of the plane word: shifting the word left by
//     15 - k puts them at bits 15 and 31, the two fp16 sign bits, and
//     ((w << (15 - k)) & 0x80008000) ^ (-v, -v) is +-v in each half
//     (v = 1.0, or alpha_k in fp16 with one scale per 128 columns: exact).
//   * The expanded operand goes to tensor memory (tcgen05.st), so the MMA
//     reads only the small X tile from shared memory.
// A stage is SW = 128 columns (64 with more than two paths, for tensor-memory
// room); the two groups of expansion warps take alternate stages, so each
// warp synchronises once per two stages.
//
// Work split (stream-K): the row tiles (128 rows) x K stages are one sequence
// of tiles * K/SW stages, cut into gridDim.x equal contiguous ranges, one per
// CTA. A CTA's range covers whole tiles and at most two partial tiles (its
// first and last); a partial tile's rows are written as fp32 partial sums
// into the workspace, and the last of its CTAs to finish adds the parts in
// CTA order (deterministic) and stores Y.
//
// Roles (NG = 3 expansion groups where the plane words come by TMA, else 2):
//   warps 0 .. 4 NG - 1   expansion: warp w writes rows 32 (w % 4) .. + 31
//               (its tensor-memory lane quarter) of every path, for the
//               stages i of the CTA's range with i % NG == w / 4;
//   next 4 warps  epilogue: tcgen05.ld of the accumulators, per-row scales,
//               store or partial sums;
//   next warp   TMA loads of the permuted X tiles;
//   next 2      MMA issue, alternate stages (the first allocates tensor memory);
//   last warp   TMA loads of the plane words (per-row scales, >= 4 words per
//               row and stage) into an 8-stage shared-memory ring, so that
//               the expansion warps issue no global loads.
// The TMA, MMA and plane warps run their loops converged (warp-uniform operands) and issue
// through one elected lane. mbarriers: full[s] (TMA bytes + the 4 warps of
// the stage's group), empty[s] (MMAs of stage s done), acc_full[b] /
// acc_empty[b] (accumulator buffer b filled / read), pfull[k] / pempty[k]
// (plane ring), baton[u] (issue order between the two MMA warps). Every wait
// is bounded; a wait that runs out records a code in the call's error word
// and the CTA winds down after draining what it issued.
#include "rb_tc.cuh"

#include <cuda_fp8.h>

#include <type_traits>
#include <utility>

namespace rb {
namespace {

using namespace tc;

// Warp roles for NG expansion groups of 4 warps: [0, 4 NG) expansion, then 4
// epilogue warps, the X TMA warp, two MMA warps and the plane-word TMA warp.
__host__ __device__ constexpr int epi_warp0(int ng) { return 4 * ng; }
__host__ __device__ constexpr int tma_warp(int ng) { return 4 * ng + 4; }
__host__ __device__ constexpr int mma_warp(int ng) { return 4 * ng + 5; }   // and the next one
__host__ __device__ constexpr int pl_warp(int ng) { return 4 * ng + 7; }

struct DecArgs {
    uint32_t* err;          // the call's device error word
    uint32_t* counters;     // one arrival counter per row tile (cleared by the host)
    float* partials;        // [gridDim.x][2][BN][128] fp32 partial sums
    const uint32_t* planes;
    const void* alpha;
    void* y;
    int64_t M, K, ldy;
    int64_t tiles;          // row tiles
    int64_t total;          // tiles * K / SW stages
    int T;
    bool sliced, alpha_f16, y_f16;
};

__host__ __device__ constexpr int stage_cols(int np, bool f8) { return f8 ? 256 : np <= 2 ? 128 : 64; }

// F8: fp8 operands (kind::f8f6f4): the weights as e4m3 +-1, X as four
// scaled e5m2 terms (TERMS rows per token, see split_x_f8_kernel),
// 256-column stages.
template <int NP, int BN, bool G128, bool F8>
struct DecCfg {
    static constexpr int SW = stage_cols(NP, F8);         // K columns per stage
    static constexpr int WPS = SW / 32;                    // plane words per row, path and stage
    static constexpr int TERMS = F8 ? 4 : 1;               // B rows per token
    static constexpr int NMMA = TERMS * BN;                // MMA N
    static constexpr int SUB = F8 ? SW / 128 : SW / BK;    // 128-byte X boxes per stage
    static constexpr int NACC = G128 ? 1 : NP;             // accumulators per buffer
    static constexpr int ACC_STRIDE = NMMA;                // MMA N: 16, 32 or 64 columns
    static constexpr int COLS_PER_WORD = F8 ? 8 : 16;      // tensor-memory columns of one plane word
    static constexpr int A_STAGE_COLS = NP * WPS * COLS_PER_WORD;
    // two accumulator buffers (the epilogue of one tile overlaps the next
    // tile's MMAs) when that still leaves three operand stages
    static constexpr int ACC_BUF = (512 - 2 * NACC * ACC_STRIDE) / A_STAGE_COLS >= 3 ? 2 : 1;
    static constexpr int ACC_COLS = ACC_BUF * NACC * ACC_STRIDE;
    static constexpr int STAGES_FIT = (512 - ACC_COLS) / A_STAGE_COLS;
    static constexpr int STAGES = STAGES_FIT < 8 ? STAGES_FIT : 8;
    // Expansion groups: three where the plane words come by TMA (no register
    // ring, so 640 threads fit), else two. A group waits on slot s for the
    // MMAs of stage i - STAGES; its previous stage (i - NG) waited for those
    // of i - NG - STAGES, and MMAs complete in issue order, so with
    // NG <= STAGES the barrier is never two phases behind the waiter (which
    // would let a parity wait pass early).
    static constexpr int NG = (!G128 && SW / 32 >= 4) ? 3 : 2;
    static constexpr int THREADS = 32 * (4 * NG + 8);
    static constexpr uint32_t SUB_BYTES = NMMA * 128;      // one 128-byte-wide box of NMMA rows
    static constexpr uint32_t B_TILE_BYTES = SUB * SUB_BYTES;
    // plane words through TMA into a shared-memory ring (per-row scales, at
    // least 4 words per row and stage: the TMA x coordinate stays 16-byte aligned)
    static constexpr bool PTMA = !G128 && WPS >= 4;
    static constexpr int PS = PTMA ? 8 : 0;                            // plane ring stages
    static constexpr uint32_t P_PATH_BYTES = BM * WPS * 4;             // [128 rows][WPS words]
    static constexpr uint32_t P_STAGE_BYTES = NP * P_PATH_BYTES;
    static constexpr uint32_t SMEM_USED = STAGES * B_TILE_BYTES + PS * P_STAGE_BYTES + 1024 /*align*/ + 512 /*barriers*/;
    // at least 120 KB, so that two CTAs never share an SM's tensor memory
    static constexpr uint32_t SMEM_BYTES = SMEM_USED < 120u * 1024u ? 120u * 1024u : SMEM_USED;
    static_assert(STAGES >= 2, "operand stages do not fit beside the accumulators");
    static_assert(NG <= STAGES, "an expansion group could run two phases ahead of a stage slot");
    static_assert(F8 ? (BN == 4 || BN == 8 || BN == 16) : (BN == 16 || BN == 32 || BN == 64), "token tile");
    static_assert(!F8 || (!G128 && NP <= 2), "fp8 operands: per-row scales, 1-2 paths");
    static_assert(SUB_BYTES % 1024 == 0, "X box must keep the 1024-byte swizzle alignment");
};

// first stage of CTA c's range and the CTA whose range holds stage g
__device__ __forceinline__ int64_t range_lo(int64_t c, int64_t total, int64_t G) { return c * total / G; }
__device__ __forceinline__ int64_t cta_of(int64_t g, int64_t total, int64_t G) { return ((g + 1) * G - 1) / total; }

template <int NP, int BN, bool G128, bool F8>
__global__ void __launch_bounds__(DecCfg<NP, BN, G128, F8>::THREADS, 1)
gemm_dec_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap pmap, DecArgs a) {
    using C = DecCfg<NP, BN, G128, F8>;
    constexpr int STAGES = C::STAGES, ACC_BUF = C::ACC_BUF, SW = C::SW, WPS = C::WPS, NG = C::NG;
    constexpr int EPI_WARP0 = epi_warp0(NG), TMA_WARP = tma_warp(NG), MMA_WARP = mma_warp(NG), PL_WARP = pl_warp(NG);
    extern __shared__ __align__(1024) unsigned char dsm[];
    const uint32_t raw = smem_addr(dsm);
    const uint32_t tiles_s = (raw + 1023u) & ~1023u;
    const uint32_t planes_s = tiles_s + STAGES * C::B_TILE_BYTES;
    const uint32_t bars = planes_s + C::PS * C::P_STAGE_BYTES;
    auto full_bar = [&](int s) { return bars + 8u * s; };
    auto empty_bar = [&](int s) { return bars + 8u * (STAGES + s); };
    auto acc_full = [&](int b) { return bars + 8u * (2 * STAGES + b); };
    auto acc_empty = [&](int b) { return bars + 8u * (2 * STAGES + 2 + b); };
    const uint32_t fin_bar = bars + 8u * (2 * STAGES + 4);
    auto baton = [&](int u) { return bars + 8u * (2 * STAGES + 5 + u); };
    auto pfull = [&](int k) { return bars + 8u * (2 * STAGES + 7 + k); };
    auto pempty = [&](int k) { return bars + 8u * (2 * STAGES + 7 + C::PS + k); };
    const uint32_t tmem_slot = bars + 8u * (2 * STAGES + 7 + 2 * C::PS);
    const uint32_t abort_slot = tmem_slot + 4u;
    const uint32_t last_slot = abort_slot + 4u;
    volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(dsm + (abort_slot - raw));
    volatile uint32_t* last_flag = reinterpret_cast<volatile uint32_t*>(dsm + (last_slot - raw));
    auto b_tile = [&](int s) { return tiles_s + static_cast<uint32_t>(s) * C::B_TILE_BYTES; };
    auto a_col = [&](int s, int p) {
        return static_cast<uint32_t>(C::ACC_COLS + (s * NP + p) * (WPS * C::COLS_PER_WORD));
    };

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t M = a.M, K = a.K, S = K / SW, total = a.total, G = gridDim.x, me = blockIdx.x;
    const int64_t lo = range_lo(me, total, G), hi = range_lo(me + 1, total, G);
    uint32_t* err = a.err;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full_bar(s), 1 + 4);
            mbar_init(empty_bar(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(acc_full(b), 2);
            mbar_init(acc_empty(b), 4);
            mbar_init(baton(b), 1);
        }
        mbar_init(fin_bar, 2);
        for (int k = 0; k < C::PS; ++k) {
            mbar_init(pfull(k), 1);
            mbar_init(pempty(k), 4);   // the four warps of the expansion group that reads it
        }
        *abort_flag = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == MMA_WARP) tmem_alloc(tmem_slot, 512);
    fence_before();
    __syncthreads();
    fence_after();
    const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t*>(dsm + (tmem_slot - raw));
    // programmatic dependent launch: the barriers and tensor memory above are
    // set up while the operand pre-pass may still run; wait for it (and
    // everything before it) here, before the first global access
    asm volatile("griddepcontrol.wait;" ::: "memory");

    if (warp == TMA_WARP) {
        // ------------------------------------------------------------ X tiles
        int64_t issued = 0;
        int s = 0, kb = static_cast<int>(lo % S);
        uint32_t ph = 0;
        for (int64_t i = 0; i < hi - lo; ++i) {
            if (!__all_sync(FULL_MASK, mbar_wait(empty_bar(s), ph ^ 1u, abort_flag, err, 1u))) break;
            if (elect_one()) {
                mbar_arrive_expect_tx(full_bar(s), C::B_TILE_BYTES);
#pragma unroll
                for (int u = 0; u < C::SUB; ++u) {
                    if (F8) tma_load_3d(b_tile(s) + u * C::SUB_BYTES, &xmap, kb * SW + u * 128, 0, 0, full_bar(s));
                    else tma_load_2d(b_tile(s) + u * C::SUB_BYTES, &xmap, kb * SW + u * BK, 0, full_bar(s));
                }
            }
            __syncwarp();
            issued = i + 1;
            if (++kb == S) kb = 0;
            if (++s == STAGES) {
                s = 0;
                ph ^= 1u;
            }
        }
        if (*abort_flag)   // loads still in flight land before the CTA exits
            for (int64_t i = issued - 1; i >= 0 && i >= issued - STAGES; --i)
                mbar_drain(full_bar(static_cast<int>(i % STAGES)), static_cast<uint32_t>(i / STAGES) & 1u);
    } else if (warp == PL_WARP) {
        // ------------------------------------------------------ plane words
        // One TMA load per path and stage: the WPS words of the stage for the
        // tile's 128 rows (rows past M read as zero), into ring slot i % PS.
        if constexpr (C::PTMA) {
            int64_t issued = 0;
            int64_t lt = lo / S;
            int lkb = static_cast<int>(lo - lt * S);
            for (int64_t i = 0; i < hi - lo; ++i) {
                const int ps = static_cast<int>(i % C::PS);
                const uint32_t pph = static_cast<uint32_t>(i / C::PS) & 1u;
                if (!__all_sync(FULL_MASK, mbar_wait(pempty(ps), pph ^ 1u, abort_flag, err, 1u))) break;
                if (elect_one()) {
                    mbar_arrive_expect_tx(pfull(ps), C::P_STAGE_BYTES);
                    const int w = lkb * WPS;
                    const int row0 = static_cast<int>(lt * BM);
#pragma unroll
                    for (int p = 0; p < NP; ++p)
                        tma_load_4d(planes_s + ps * C::P_STAGE_BYTES + p * C::P_PATH_BYTES, &pmap,
                                    a.sliced ? (w & 15) : w, row0, a.sliced ? (w >> 4) : 0, p, pfull(ps));
                }
                __syncwarp();
                issued = i + 1;
                if (++lkb == S) {
                    lkb = 0;
                    ++lt;
                }
            }
            if (*abort_flag)   // loads still in flight land before the CTA exits
                for (int64_t i = issued - 1; i >= 0 && i >= issued - C::PS; --i)
                    mbar_drain(pfull(static_cast<int>(i % C::PS)), static_cast<uint32_t>(i / C::PS) & 1u);
        }
    } else if (warp == MMA_WARP || warp == MMA_WARP + 1) {
        // ---------------------------------------------------------------- MMA
        // Two issuers take alternate stages of the range (issuer u the
        // stages i with i % 2 == u), so that one does its bookkeeping
        // (barrier waits, commit) while the other's MMAs keep the tensor pipe
        // busy. Both add into the same accumulators, so the order of issue
        // is handed over: after issuing stage i the issuer fences
        // (tcgen05.fence::before_thread_sync) and arrives on its baton
        // barrier; the issuer of stage i + 1 waits for that arrival and
        // fences (after_thread_sync) before its first MMA. Each issuer
        // commits its own MMAs: empty[s] for its stages, and acc_full / the
        // final barrier (two arrivals each) for every tile.
        const int u = warp - MMA_WARP;
        constexpr uint32_t idesc = F8 ? instr_desc_f8(C::NMMA) : instr_desc(BN);
        int st = 0;          // stage slot and phase of the next stage
        uint32_t sph = 0;
        uint32_t bph = 0;    // phase of the other issuer's baton waited for next
        int64_t i = 0;       // stage ordinal in the CTA's range
        int j = 0;           // segment counter
        bool ok = true;
        for (int64_t t = lo / S; ok && t * S < hi; ++t, ++j) {
            const int64_t k0 = (lo > t * S ? lo - t * S : 0), k1 = (hi < (t + 1) * S ? hi - t * S : S);
            const int b = j % ACC_BUF;
            const uint32_t dbase = tmem_base + static_cast<uint32_t>(b * C::NACC * C::ACC_STRIDE);
            for (int64_t kb = k0; kb < k1; ++kb, ++i) {
                const int s = st;
                const uint32_t ph = sph;
                if (++st == STAGES) {
                    st = 0;
                    sph ^= 1u;
                }
                if ((i & 1) != u) continue;
                // the tile's first stage: its accumulator buffer must have been read out
                if (kb == k0 && j >= ACC_BUF &&
                    !__all_sync(FULL_MASK, mbar_wait(acc_empty(b), static_cast<uint32_t>(j / ACC_BUF - 1) & 1u,
                                                     abort_flag, err, 2u))) {
                    ok = false;
                    break;
                }
                if (!__all_sync(FULL_MASK, mbar_wait(full_bar(s), ph, abort_flag, err, 2u))) {
                    ok = false;
                    break;
                }
                if (i > 0) {
                    if (!__all_sync(FULL_MASK, mbar_wait(baton(u ^ 1), bph, abort_flag, err, 2u))) {
                        ok = false;
                        break;
                    }
                    bph ^= 1u;
                }
                fence_after();
                const uint64_t bd0 = smem_desc(b_tile(s));
                const uint32_t acc0 = kb > k0 ? 1u : 0u;
                if (elect_one()) {
#pragma unroll
                    for (int p = 0; p < NP; ++p) {
                        const uint32_t d = dbase + static_cast<uint32_t>(G128 ? 0 : p * C::ACC_STRIDE);
                        // one MMA per 32 bytes of K (16 fp16 or 32 fp8 columns):
                        // box kk / 4, and +32 bytes inside a swizzled box is +2
                        // in the descriptor's address field
#pragma unroll
                        for (int kk = 0; kk < WPS * C::COLS_PER_WORD / 8; ++kk) {
                            const uint64_t bd = bd0 + ((kk >> 2) * C::SUB_BYTES >> 4) + 2u * (kk & 3);
                            const uint32_t acc = (kk > 0 || (G128 && p > 0)) ? 1u : acc0;
                            if (F8) umma_f8_ta(d, tmem_base + a_col(s, p) + 8u * kk, bd, idesc, acc);
                            else umma_f16_ta(d, tmem_base + a_col(s, p) + 8u * kk, bd, idesc, acc);
                        }
                    }
                    fence_before();
                    mbar_arrive(baton(u));
                    umma_commit(empty_bar(s));
                }
                __syncwarp();
            }
            if (ok) {
                if (elect_one()) umma_commit(acc_full(b));
                __syncwarp();
            }
        }
        if (elect_one()) umma_commit(fin_bar);   // every MMA issued above has completed once both arrive
        __syncwarp();
    } else if (warp < 4 * NG) {
        // ---------------------------------------------------------- expansion
        // Thread = one row of the tile (its tensor-memory lane), all paths,
        // the stages i with i % NG == grp. The plane words of a stage (SW / 32
        // per path) come from the TMA ring in shared memory (PTMA) or are
        // loaded PR of the group's stages ahead into registers.
        const int q = warp & 3, grp = warp >> 2;
        const int r = 32 * q + lane;
        const uint32_t lane_q = static_cast<uint32_t>(32 * q) << 16;
        const uint32_t uM = static_cast<uint32_t>(M);
        const uint32_t W32 = static_cast<uint32_t>(K >> 5), SL = static_cast<uint32_t>((K + 511) >> 9);
        const uint32_t gpr = static_cast<uint32_t>(K >> 7);
        const uint32_t path_words = a.sliced ? SL * uM * 16u : uM * W32;   // < 2^30 (checked by the host)
        using WV = typename std::conditional<WPS == 2, uint2, uint4>::type;
        constexpr int NV = WPS == 2 ? 1 : WPS / 4;   // vector loads per path and stage
        constexpr int PR = F8 ? 2 : NP <= 2 ? 4 : 2;   // stages of this group loaded ahead
        const int64_t n = hi - lo;
        // (tile, stage-in-tile) of the next stage to load, stepping by 2
        int64_t lt = (lo + grp) / S;   // (tile, stage) of the next register-ring load
        int lkb = static_cast<int>(lo + grp - lt * S);
        WV ring[C::PTMA ? 1 : PR][NP][NV];
        uint32_t nring[C::PTMA ? 1 : PR][NP];
        auto load_stage = [&](WV (&dst)[NP][NV], uint32_t (&ndst)[NP]) {
            const int64_t row64 = lt * BM + r;
            const uint32_t row = static_cast<uint32_t>(row64 < M ? row64 : M - 1);   // rows past M read a real row
            const uint32_t w = static_cast<uint32_t>(lkb) * WPS;
            const uint32_t off = a.sliced ? ((w >> 4) * uM + row) * 16u + (w & 15u) : row * W32 + w;
#pragma unroll
            for (int p = 0; p < NP; ++p) {
#pragma unroll
                for (int v = 0; v < NV; ++v)
                    dst[p][v] = __ldg(reinterpret_cast<const WV*>(a.planes + static_cast<size_t>(p) * path_words + off) + v);
                if (G128) {
                    const uint32_t g = static_cast<uint32_t>(lkb) * SW / 128u;
                    const uint32_t hv = static_cast<const unsigned short*>(a.alpha)[(p * uM + row) * gpr + g] | 0x8000u;
                    ndst[p] = hv | (hv << 16);
                } else {
                    ndst[p] = 0xBC00BC00u;   // -1.0 in both halves
                }
            }
            lkb += NG;
            while (lkb >= S) {
                lkb -= static_cast<int>(S);
                ++lt;
            }
        };
        // fp16: +-v pairs of one plane word into 16 tensor-memory columns
        auto expand_store = [&](uint32_t w, uint32_t ng, uint32_t col) {
            uint32_t h[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) h[k] = ((w << (15 - k)) & 0x80008000u) ^ ng;
            tmem_store16(tmem_base + lane_q + col, h);
        };
        // fp8: two plane words into 16 tensor-memory columns of e4m3 +-1.
        // The columns of X'' are ordered so that byte b of column r of a
        // word holds column 8b + r: shifting left by 7 - r puts bits r,
        // 8 + r, 16 + r, 24 + r at the four byte sign bits, and xor with
        // four e4m3 -1.0 (0xB8) gives +1.0 (0x38) where the bit is set.
        auto expand_store8 = [&](uint32_t w0, uint32_t w1, uint32_t col) {
            uint32_t h[16];
#pragma unroll
            for (int r = 0; r < 8; ++r) {
                h[r] = ((w0 << (7 - r)) & 0x80808080u) ^ 0xB8B8B8B8u;
                h[8 + r] = ((w1 << (7 - r)) & 0x80808080u) ^ 0xB8B8B8B8u;
            }
            tmem_store16(tmem_base + lane_q + col, h);
        };
        auto word = [](const WV (&v)[NV], int i) -> uint32_t {
            if constexpr (WPS == 2) return i == 0 ? v[0].x : v[0].y;
            else {
                const uint4& u = v[i >> 2];
                const int j = i & 3;
                return j == 0 ? u.x : j == 1 ? u.y : j == 2 ? u.z : u.w;
            }
        };
        // expand the words of stage slot s into tensor memory and hand the slot to the MMA
        auto expand_stage = [&](const WV (&cur)[NP][NV], const uint32_t (&ng)[NP], int s) {
#pragma unroll
            for (int p = 0; p < NP; ++p) {
                if constexpr (F8) {
#pragma unroll
                    for (int wi = 0; wi < WPS; wi += 2)
                        expand_store8(word(cur[p], wi), word(cur[p], wi + 1), a_col(s, p) + 8u * wi);
                } else {
#pragma unroll
                    for (int wi = 0; wi < WPS; ++wi) expand_store(word(cur[p], wi), ng[p], a_col(s, p) + 16u * wi);
                }
            }
            tmem_store_wait();
            fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(full_bar(s));
        };
        int s = grp % STAGES;
        uint32_t ph = static_cast<uint32_t>(grp / STAGES) & 1u;
        if constexpr (C::PTMA) {
            const unsigned char* prow = dsm + (planes_s - raw) + static_cast<uint32_t>(r) * (WPS * 4);
            uint32_t ng[NP];
#pragma unroll
            for (int p = 0; p < NP; ++p) ng[p] = 0xBC00BC00u;   // -1.0 in both halves
            for (int64_t i = grp; i < n; i += NG) {
                const int ps = static_cast<int>(i % C::PS);
                if (!__all_sync(FULL_MASK, mbar_wait(pfull(ps), static_cast<uint32_t>(i / C::PS) & 1u, abort_flag,
                                                     err, 4u)))
                    break;
                WV cur[NP][NV];
#pragma unroll
                for (int p = 0; p < NP; ++p)
#pragma unroll
                    for (int v = 0; v < NV; ++v)
                        cur[p][v] = *reinterpret_cast<const WV*>(prow + ps * C::P_STAGE_BYTES + p * C::P_PATH_BYTES +
                                                                 v * sizeof(WV));
                __syncwarp();
                if (lane == 0) mbar_arrive(pempty(ps));   // the words are in registers: the slot may refill
                // warp-uniform: the tensor-memory stores are .sync.aligned
                if (!__all_sync(FULL_MASK, mbar_wait(empty_bar(s), ph ^ 1u, abort_flag, err, 4u))) break;
                expand_stage(cur, ng, s);
                s += NG;
                while (s >= STAGES) {
                    s -= STAGES;
                    ph ^= 1u;
                }
            }
        } else {
#pragma unroll
            for (int d = 0; d < PR; ++d)
                if (grp + NG * d < n) load_stage(ring[d], nring[d]);
            bool go = true;
            for (int64_t i0 = grp; i0 < n && go; i0 += NG * PR) {
#pragma unroll
                for (int d = 0; d < PR; ++d) {
                    const int64_t i = i0 + NG * d;
                    if (i < n && go) {
                        WV cur[NP][NV];
                        uint32_t ng[NP];
#pragma unroll
                        for (int p = 0; p < NP; ++p) {
#pragma unroll
                            for (int v = 0; v < NV; ++v) cur[p][v] = ring[d][p][v];
                            ng[p] = nring[d][p];
                        }
                        if (i + NG * PR < n) load_stage(ring[d], nring[d]);
                        // warp-uniform: the tensor-memory stores are .sync.aligned
                        if (!__all_sync(FULL_MASK, mbar_wait(empty_bar(s), ph ^ 1u, abort_flag, err, 4u))) {
                            go = false;
                        } else {
                            expand_stage(cur, ng, s);
                        }
                        s += NG;
                        while (s >= STAGES) {
                            s -= STAGES;
                            ph ^= 1u;
                        }
                    }
                }
            }
        }
    } else if (warp >= EPI_WARP0 && warp < EPI_WARP0 + 4) {
        // ----------------------------------------------------------- epilogue
        const int q = warp & 3;
        const int r = 32 * q + lane;
        const uint32_t lane_q = static_cast<uint32_t>(32 * q) << 16;
        constexpr int CW = BN < 32 ? BN : 32;
        int j = 0;
        for (int64_t t = lo / S; t * S < hi; ++t, ++j) {
            const int64_t k0 = (lo > t * S ? lo - t * S : 0), k1 = (hi < (t + 1) * S ? hi - t * S : S);
            const int b = j % ACC_BUF;
            const int64_t row = t * BM + r;
            const int64_t crow = row < M ? row : M - 1;
            const bool ok =   // warp-uniform: tcgen05.ld is .sync.aligned
                __all_sync(FULL_MASK, mbar_wait(acc_full(b), static_cast<uint32_t>(j / ACC_BUF) & 1u, abort_flag, err, 8u));
            fence_after();
            const bool full = k0 == 0 && k1 == S;
            const int T = a.T;
            const int slot = (t == lo / S) ? 0 : 1;
            float* mine = a.partials + ((me * 2 + slot) * BN) * BM;
            // one output value of token column c of this thread's row
            auto store_y1 = [&](int c, float v) {
                if (row < M && c < T) {
                    if (a.y_f16) static_cast<__half*>(a.y)[c * a.ldy + row] = __float2half_rn(v);
                    else static_cast<float*>(a.y)[c * a.ldy + row] = v;
                }
            };
            if (ok) {
                float al[C::NACC];
#pragma unroll
                for (int p = 0; p < C::NACC; ++p) {
                    if (G128) al[p] = 1.0f;
                    else al[p] = a.alpha_f16 ? __half2float(static_cast<const __half*>(a.alpha)[p * M + crow])
                                             : static_cast<const float*>(a.alpha)[p * M + crow];
                }
                // CW token columns at a time: sum_k alpha_k acc_k, then Y or
                // the partial-sum slot of this CTA. With one chunk (BN <= 32)
                // the accumulator buffer is released before the stores, so
                // the next tile's MMAs need not wait for them.
#pragma unroll 1
                for (int c0 = 0; c0 < BN; c0 += CW) {
                    float yv[CW];
#pragma unroll
                    for (int c = 0; c < CW; ++c) yv[c] = 0.0f;
#pragma unroll
                    for (int p = 0; p < C::NACC; ++p) {
                        // token c0 + c of term m sits at column m * BN + c0 + c
                        float acc[CW];
#pragma unroll
                        for (int c = 0; c < CW; ++c) acc[c] = 0.0f;
#pragma unroll
                        for (int m = 0; m < C::TERMS; ++m) {
                            uint32_t v[CW];
                            tmem_load<CW>(tmem_base + lane_q +
                                              static_cast<uint32_t>((b * C::NACC + p) * C::ACC_STRIDE + m * BN + c0), v);
                            const float wm = F8 ? 1.0f / static_cast<float>(1 << (2 * m)) : 1.0f;   // 4^-m
#pragma unroll
                            for (int c = 0; c < CW; ++c) acc[c] = fmaf(wm, __uint_as_float(v[c]), acc[c]);
                        }
#pragma unroll
                        for (int c = 0; c < CW; ++c) yv[c] = fmaf(al[p], acc[c], yv[c]);
                    }
                    if (CW == BN) {
                        fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(acc_empty(b));   // the buffer may take the next tile
                    }
#pragma unroll
                    for (int c = 0; c < CW; ++c) {
                        if (full) store_y1(c0 + c, yv[c]);
                        else if (c0 + c < T) mine[(c0 + c) * BM + r] = yv[c];
                    }
                }
            }
            if (!ok || CW != BN) {
                fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(acc_empty(b));   // the buffer may take the next tile
            }
            if (full) continue;
            // partial tile: the same sequence of named barriers whatever happened
            const int64_t first = cta_of(t * S, total, G), last = cta_of((t + 1) * S - 1, total, G);
            if (ok) __threadfence();
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (threadIdx.x == EPI_WARP0 * 32) {
                uint32_t prev = 0;
                if (!*abort_flag) prev = atomicAdd(a.counters + t, 1u);
                *last_flag = (!*abort_flag && prev == static_cast<uint32_t>(last - first)) ? 1u : 0u;
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (*last_flag && ok) {
                // every part, this CTA's own included, is read back from the
                // workspace and added in CTA order: the result does not
                // depend on which CTA finished last
                __threadfence();
#pragma unroll 1
                for (int c0 = 0; c0 < BN; c0 += CW) {
                    float yv[CW];
#pragma unroll
                    for (int c = 0; c < CW; ++c) yv[c] = 0.0f;
                    for (int64_t cc = first; cc <= last; ++cc) {
                        const int sl = (t == range_lo(cc, total, G) / S) ? 0 : 1;
                        const float* part = a.partials + ((cc * 2 + sl) * BN) * BM;
#pragma unroll
                        for (int c = 0; c < CW; ++c)
                            if (c0 + c < T) yv[c] += __ldcg(part + (c0 + c) * BM + r);
                    }
#pragma unroll
                    for (int c = 0; c < CW; ++c) store_y1(c0 + c, yv[c]);
                }
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");   // last_flag is reused by the next tile
        }
    }

    __syncwarp();
    fence_before();
    __syncthreads();
    if (warp == MMA_WARP) {
        mbar_drain(fin_bar, 0u);   // no MMA still reads or writes tensor memory
        __syncwarp();
        fence_after();
        tmem_dealloc(tmem_base, 512);
    }
}

// X' = X with the columns of every 32-column block reordered so that
// position 2k holds column k and position 2k + 1 column k + 16 (the operand
// order the expansion above produces). One thread per (token, block).
// The pre-pass also clears the call's error word and the arrival counters
// of the main kernel (it runs before it on the same stream).
__device__ __forceinline__ void clear_call_state(uint32_t* err, uint32_t* counters, int64_t n_ctr, int64_t idx) {
    // programmatic dependent launch: let the main kernel launch and set up;
    // wait for the previous kernel of the stream (which may still read this
    // workspace) before the first global access
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (idx == 0) *err = 0u;
    const int64_t step = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = idx; i < n_ctr; i += step) counters[i] = 0u;
}

__global__ void permute_x_kernel(const __half* __restrict__ X, int64_t ldx, int T, int64_t K,
                                 __half* __restrict__ Xp, uint32_t* err, uint32_t* counters, int64_t n_ctr) {
    const int64_t blocks = K >> 5;
    const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    clear_call_state(err, counters, n_ctr, idx);
    if (idx >= blocks * T) return;
    const int64_t t = idx / blocks, bl = idx - t * blocks;
    const uint4* src = reinterpret_cast<const uint4*>(X + t * ldx + 32 * bl);
    const uint4 l0 = __ldg(src), l1 = __ldg(src + 1), h0 = __ldg(src + 2), h1 = __ldg(src + 3);
    const uint32_t lw[8] = {l0.x, l0.y, l0.z, l0.w, l1.x, l1.y, l1.z, l1.w};   // columns 2m, 2m + 1
    const uint32_t hw[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};   // columns 16 + 2m, 17 + 2m
    uint32_t o[16];
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        o[2 * m] = __byte_perm(lw[m], hw[m], 0x5410);       // (column 2m, column 16 + 2m)
        o[2 * m + 1] = __byte_perm(lw[m], hw[m], 0x7632);   // (column 2m + 1, column 17 + 2m)
    }
    uint4* dst = reinterpret_cast<uint4*>(Xp + t * K + 32 * bl);
    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
    dst[2] = make_uint4(o[8], o[9], o[10], o[11]);
    dst[3] = make_uint4(o[12], o[13], o[14], o[15]);
}

// X'' for the fp8 operands: every fp16 value x is written as four e5m2
// terms, each the rounding of the previous residual scaled by 4:
//   s1 = RN(x), s2 = RN(4 (x - s1)), s3 = RN(4 (4 (x - s1) - s2)), ...
// so that x = s1 + s2/4 + s3/16 + s4/64 + e. e5m2 has the exponent range of
// fp16 and 3 significant bits, each residual is at most 2^-3 of the value it
// was taken from, and the scaled residuals are exact in fp16 and stay below
// |x| / 2 (no overflow): |e| <= 2^-12 |x| + 2^-23, and e = 0 for every normal
// fp16 x (4 x 3 bits cover its 11). The epilogue weights the accumulators of
// the four terms by 1, 1/4, 1/16, 1/64. Layout: [term][token][K] bytes, and
// inside every 32-column block byte 4r + b holds column 8b + r (the order
// the fp8 expansion produces). One thread per (token, block).
__global__ void split_x_f8_kernel(const __half* __restrict__ X, int64_t ldx, int T, int64_t K,
                                  uint8_t* __restrict__ Xq, uint32_t* err, uint32_t* counters, int64_t n_ctr) {
    const int64_t blocks = K >> 5;
    const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    clear_call_state(err, counters, n_ctr, idx);
    if (idx >= blocks * T) return;
    const int64_t t = idx / blocks, bl = idx - t * blocks;
    const uint4* src = reinterpret_cast<const uint4*>(X + t * ldx + 32 * bl);
    __half res[32];
#pragma unroll
    for (int v = 0; v < 4; ++v) {
        const uint4 u = __ldg(src + v);
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __half2_raw h2;
            h2.x = static_cast<unsigned short>(w[i] & 0xFFFFu);
            h2.y = static_cast<unsigned short>(w[i] >> 16);
            res[8 * v + 2 * i] = __half(__half_raw{h2.x});
            res[8 * v + 2 * i + 1] = __half(__half_raw{h2.y});
        }
    }
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        uint32_t q[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) {
            const __nv_fp8_storage_t b8 = __nv_cvt_halfraw_to_fp8(static_cast<__half_raw>(res[c]), __NV_SATFINITE, __NV_E5M2);
            q[c] = b8;
            if (m < 3)   // exact: the residual and its product with 4
                res[c] = __hmul(__hsub(res[c], __half(__nv_cvt_fp8_to_halfraw(b8, __NV_E5M2))), __float2half(4.0f));
        }
        uint32_t o[8];
#pragma unroll
        for (int r = 0; r < 8; ++r) o[r] = q[r] | (q[8 + r] << 8) | (q[16 + r] << 16) | (q[24 + r] << 24);
        uint4* dst = reinterpret_cast<uint4*>(Xq + (static_cast<int64_t>(m) * T + t) * K + 32 * bl);
        dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
        dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
    }
}

// Plane words as a 4-D uint32 tensor {word, row, slice, path}: in the sliced
// order 16 words per 512-column slice (rows 64 bytes apart, slices M rows
// apart); in the row order all K/32 words of a row and one slice. A box is
// the stage's `words` words of 128 rows of one path.
cudaError_t make_plane_map(CUtensorMap* map, const uint32_t* planes, int64_t M, int64_t K, int n_paths, bool sliced,
                           int words) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    const int64_t W32 = K / 32, SL = (K + 511) / 512;
    const cuuint64_t wpr = static_cast<cuuint64_t>(sliced ? 16 : W32);   // words per row and slice
    const cuuint64_t dims[4] = {wpr, static_cast<cuuint64_t>(M), static_cast<cuuint64_t>(sliced ? SL : 1),
                                static_cast<cuuint64_t>(n_paths)};
    const cuuint64_t row_b = wpr * 4, slice_b = row_b * static_cast<cuuint64_t>(M);
    const cuuint64_t strides[3] = {row_b, slice_b, slice_b * dims[2]};
    const cuuint32_t box[4] = {static_cast<cuuint32_t>(words), static_cast<cuuint32_t>(tc::BM), 1u, 1u};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    if (enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, const_cast<uint32_t*>(planes), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    return cudaSuccess;
}

// Launch as a programmatic dependent of the stream's previous kernel (the
// kernels wait for it with griddepcontrol.wait before any global access).
template <typename... P, typename... A>
cudaError_t launch_pdl(void (*kern)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, A&&... args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<A>(args)...);
}

template <int NP, int BN, bool G128, bool F8>
cudaError_t launch_dec(const DecArgs& a, const void* Xp, int grid, cudaStream_t s) {
    using C = DecCfg<NP, BN, G128, F8>;
    CUtensorMap map, pmap;
    cudaError_t e = F8 ? make_x8_map(&map, Xp, a.K, a.T, 4, BN) : make_x_map(&map, Xp, a.K, a.T, a.K, BN);
    if (e != cudaSuccess) return e;
    if constexpr (C::PTMA) {
        e = make_plane_map(&pmap, a.planes, a.M, a.K, NP, a.sliced, C::WPS);
        if (e != cudaSuccess) return e;
    } else {
        pmap = map;   // unused
    }
    auto kern = gemm_dec_kernel<NP, BN, G128, F8>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    return launch_pdl(kern, dim3(grid), dim3(C::THREADS), C::SMEM_BYTES, s, map, pmap, a);
}

template <int NP, bool G128>
cudaError_t launch_dec_np(const DecArgs& a, const void* Xp, int grid, bool f8, cudaStream_t s) {
    if constexpr (NP <= 2 && !G128) {
        if (f8) {
            if (a.T <= 4) return launch_dec<NP, 4, false, true>(a, Xp, grid, s);
            if (a.T <= 8) return launch_dec<NP, 8, false, true>(a, Xp, grid, s);
            return launch_dec<NP, 16, false, true>(a, Xp, grid, s);
        }
    }
    if (a.T <= 16) return launch_dec<NP, 16, G128, false>(a, Xp, grid, s);
    if (a.T <= 32) return launch_dec<NP, 32, G128, false>(a, Xp, grid, s);
    return launch_dec<NP, 64, G128, false>(a, Xp, grid, s);
}

}  // namespace

static size_t align256(size_t b) { return (b + 255) & ~size_t(255); }

// tokens per tile: fp16 operands 16/32/64; fp8 operands 4/8/16 (x 4 terms)
static int dec_bn(int T, bool f8) {
    if (f8) return T <= 4 ? 4 : T <= 8 ? 8 : 16;
    return T <= 16 ? 16 : T <= 32 ? 32 : 64;
}

// fp8 operands for T <= 16 tokens with one or two paths and per-row scales
// (the scales stay out of the operands), when K splits into 256-column stages
static bool dec_f8(int64_t K, int n_paths, int group, int T) {
    return T <= 16 && n_paths <= 2 && group == 0 && K % 256 == 0;
}

GemmDecPlan gemm_dec_plan(int64_t M, int64_t K, int n_paths, int group, int T, int num_sms) {
    GemmDecPlan pl{};
    const bool f8 = dec_f8(K, n_paths, group, T);
    const int64_t tiles = (M + tc::BM - 1) / tc::BM;
    const int64_t total = tiles * (K / stage_cols(n_paths, f8));
    pl.tiles = tiles;
    pl.total = total;
    pl.grid = static_cast<int>(total < num_sms ? total : num_sms);
    pl.bn = dec_bn(T, f8);
    pl.f8 = f8;
    pl.counters_bytes = align256(static_cast<size_t>(tiles) * 4);
    pl.partials_bytes = align256(static_cast<size_t>(pl.grid) * 2 * pl.bn * tc::BM * 4);
    pl.xp_bytes = align256(static_cast<size_t>(T) * K * (f8 ? 4 : 2));
    return pl;
}

cudaError_t launch_gemm_dec(const uint32_t* planes, const void* alpha, bool alpha_f16, int64_t M, int64_t K,
                            int n_paths, int group, bool sliced, const void* X, int64_t ldx, int T, void* Y,
                            bool y_f16, int64_t ldy, void* workspace, const GemmDecPlan& pl, cudaStream_t s) {
    // workspace: header | counters | partial sums | permuted X
    char* ws = static_cast<char*>(workspace);
    uint32_t* counters = reinterpret_cast<uint32_t*>(ws + GEMM_HEADER_BYTES);
    float* partials = reinterpret_cast<float*>(ws + GEMM_HEADER_BYTES + pl.counters_bytes);
    __half* Xp = reinterpret_cast<__half*>(ws + GEMM_HEADER_BYTES + pl.counters_bytes + pl.partials_bytes);
    const int64_t nthr = (K >> 5) * T;
    uint32_t* err = reinterpret_cast<uint32_t*>(ws) + 1;
    cudaError_t e;
    if (pl.f8)
        e = launch_pdl(split_x_f8_kernel, dim3(static_cast<unsigned>((nthr + 127) / 128)), dim3(128), 0, s,
                       static_cast<const __half*>(X), ldx, T, K, reinterpret_cast<uint8_t*>(Xp), err, counters,
                       static_cast<int64_t>(pl.tiles));
    else
        e = launch_pdl(permute_x_kernel, dim3(static_cast<unsigned>((nthr + 255) / 256)), dim3(256), 0, s,
                       static_cast<const __half*>(X), ldx, T, K, Xp, err, counters, static_cast<int64_t>(pl.tiles));
    if (e != cudaSuccess) return e;
    DecArgs a{err, counters, partials, planes, alpha, Y, M, K, ldy, pl.tiles,
              pl.total, T, sliced, alpha_f16, y_f16};
    const bool g128 = group == 128;
    switch (n_paths) {
        case 1: return g128 ? launch_dec_np<1, true>(a, Xp, pl.grid, pl.f8, s)
                     : launch_dec_np<1, false>(a, Xp, pl.grid, pl.f8, s);
        case 2: return g128 ? launch_dec_np<2, true>(a, Xp, pl.grid, pl.f8, s)
                     : launch_dec_np<2, false>(a, Xp, pl.grid, pl.f8, s);
        case 3: return g128 ? launch_dec_np<3, true>(a, Xp, pl.grid, pl.f8, s)
                     : launch_dec_np<3, false>(a, Xp, pl.grid, pl.f8, s);
        case 4: return g128 ? launch_dec_np<4, true>(a, Xp, pl.grid, pl.f8, s)
                     : launch_dec_np<4, false>(a, Xp, pl.grid, pl.f8, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace rb
