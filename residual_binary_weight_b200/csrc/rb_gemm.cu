// rb_gemm, prefill blocks: Y = sum_k alpha_k (.) (B_k X^T) for a block of
// T > 64 tokens on the tcgen05 tensor cores (sm_100a). Decode batches of at
// most 64 tokens go to the persistent kernel of rb_gemm_dec.cu.
//
// The per-path contraction B_k X^T is a dense GEMM with a +-1 operand: the
// plane bits are expanded exactly to fp16 +-1.0 (or, with one scale per 128
// columns, to +-alpha_k in fp16, which is exact because alpha_k is stored in
// fp16) and multiplied on the tensor cores with fp32 accumulation in tensor
// memory; per-row scales multiply the per-path accumulators in the epilogue
// (RaBiT section 4.1: y = sum_k alpha_k (.) (B_k x); QBB W(4x1)A16g128).
//
// One CTA computes a 128-row x BN-token tile over all of K:
//   warp 0     one thread issues TMA loads of X tiles (BN tokens x 64 columns,
//              128-byte swizzle) into a STAGES-deep ring;
//   warp 1     allocates tensor memory and one thread issues
//              tcgen05.mma.cta_group::1.kind::f16 (M=128, N=BN, K=16), one
//              accumulator per path (per-row scales) or one in all;
//   warps 4-7  expand the plane bits of their row (thread = row) into the
//              K-major 128-byte-swizzled fp16 A tile of every path, then run
//              the epilogue: tcgen05.ld of the accumulators, scale, fp16/fp32
//              store.
// Stages are handed over with mbarriers: full_x[s] (TMA bytes), full_a[s]
// (128 expansion arrivals) and empty[s] (tcgen05.commit after the MMAs that
// read stage s). Every wait is bounded; a wait that runs out records an error
// code in the call's error word, raises a CTA-wide abort flag and the kernel
// winds down instead of hanging (after draining its issued MMAs and loads).
#include "rb_tc.cuh"

namespace rb {
namespace {

using namespace tc;

constexpr int THREADS = 256;
constexpr int EXP_WARP0 = 4;     // first expansion/epilogue warp
constexpr uint32_t A_TILE_BYTES = BM * BK * 2;   // 16 KB

__device__ __forceinline__ uint32_t elect_lane0() { return (threadIdx.x & 31) == 0; }

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
                 : "memory");
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

__device__ __forceinline__ uint32_t lop_sign(uint32_t value, uint32_t mask) {
    // value | (~mask & 0x80008000): clear bit -> negative half
    return value | (~mask & 0x80008000u);
}

// Expand one 32-column word of plane bits into 16 half2 (+-v, v = `val2`
// in both halves): half2 i holds columns 2i, 2i+1. Bit c sits at the most
// significant bit of byte c/8 of (w << (7 - c % 8)); PRMT replicates those
// sign bits into a mask, which decides the sign of each half.
__device__ __forceinline__ void expand_word(uint32_t w, uint32_t val2, uint32_t (&h)[16]) {
    uint32_t s[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) s[k] = w << (7 - k);
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int m = i & 3, b = i >> 2;
        // byte 1 <- sign of byte b of s[2m] (column 2i); byte 3 <- sign of byte b of s[2m+1] (column 2i+1)
        const uint32_t sel = (static_cast<uint32_t>(8 | b) << 4) | (static_cast<uint32_t>(8 | (4 + b)) << 12);
        h[i] = lop_sign(val2, prmt(s[2 * m], s[2 * m + 1], sel));
    }
}

// Reconstruct-once expansion of one 32-column word pair (paths 0 and 1) into
// 16 half2 of W^ = alpha_0 B_0 + alpha_1 B_1: the magnitude is p2 (both
// signs equal) or q2 (signs differ), chosen by a full-width mask of
// ~(w0 ^ w1); the sign is that of path 0 (q may itself be negative, and the
// sign flip of an fp16 is exact). Half2 i holds columns 2i, 2i+1.
__device__ __forceinline__ void expand_word_rec(uint32_t w0, uint32_t w1, uint32_t p2, uint32_t q2,
                                                uint32_t (&h)[16]) {
    const uint32_t e = ~(w0 ^ w1);
    uint32_t s0[8], se[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        s0[k] = w0 << (7 - k);
        se[k] = e << (7 - k);
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int m = i & 3, b = i >> 2;
        const uint32_t lo = 8u | b, hi = 8u | (4u + b);
        // bytes 0-1 <- sign of byte b of se[2m] (column 2i), bytes 2-3 <- sign of byte b of se[2m+1]
        const uint32_t mask = prmt(se[2 * m], se[2 * m + 1], lo | (lo << 4) | (hi << 8) | (hi << 12));
        const uint32_t mag = (mask & p2) | (~mask & q2);
        const uint32_t sgn = prmt(s0[2 * m], s0[2 * m + 1], (lo << 4) | (hi << 12));
        h[i] = mag ^ (~sgn & 0x80008000u);
    }
}

struct GemmArgs {
    uint32_t* err;          // device error word of the call (workspace header word 1)
    const uint32_t* planes;
    const void* alpha;
    void* y;
    int64_t M, K, ldy;
    int T;
    int n_paths;
    bool g128;
    bool sliced;
    bool alpha_f16;
    bool y_f16;
};

// ATM: the expanded A operand goes to tensor memory (tcgen05.st) instead of
// shared memory, so shared memory only carries the X tiles; used for token
// tiles of at most 128, where the accumulators leave room for A stages.
// REC: reconstruct-once -- one fp16 operand W^ = sum_k alpha_k B_k per
// weight (two paths, per-row scales), one accumulator, one MMA chain.
template <int NP, int BN, int STAGES, bool G128, bool ATM, bool REC = false>
struct GemmCfg {
    static constexpr int NA = REC ? 1 : NP;                            // operand tiles per stage
    static constexpr int NACC = (G128 || REC) ? 1 : NP;                // accumulators
    // tensor-memory columns between accumulators: BN rounded up to a power of two
    static constexpr int ACC_STRIDE = BN <= 16 ? 16 : BN <= 32 ? 32 : BN <= 64 ? 64 : BN <= 128 ? 128 : 256;
    static constexpr uint32_t B_TILE_BYTES = BN * BK * 2;
    static constexpr uint32_t STAGE_BYTES = (ATM ? 0 : NA * A_TILE_BYTES) + B_TILE_BYTES;
    static constexpr int ACC_COLS = NACC * ACC_STRIDE;
    static constexpr int A_BASE = ACC_COLS;               // first tensor-memory column of the A stages
    static constexpr int A_STAGE_COLS = NA * BK / 2;      // fp16 pairs of all operand tiles of one stage
    static constexpr uint32_t TMEM_COLS = ATM ? 512 : (ACC_COLS <= 32) ? 32 : (ACC_COLS <= 64) ? 64 :
                                          (ACC_COLS <= 128) ? 128 : (ACC_COLS <= 256) ? 256 : 512;
    // with A in tensor memory the shared memory is small; ask for enough that
    // two CTAs never share an SM (the second would wait for tensor memory)
    static constexpr uint32_t SMEM_USED = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;
    static constexpr uint32_t SMEM_BYTES = ATM && SMEM_USED < 120u * 1024u ? 120u * 1024u : SMEM_USED;
    static_assert(!ATM || A_BASE + STAGES * A_STAGE_COLS <= 512, "A stages exceed tensor memory");
    static_assert(ACC_COLS <= 512, "accumulators exceed tensor memory");
    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "MMA N for M = 128");
    static_assert(B_TILE_BYTES % 1024 == 0, "B tile must keep the 1024-byte swizzle alignment");
    static_assert(!REC || (NP == 2 && !G128), "reconstruct-once: two paths, per-row scales");
};

template <int NP, int BN, int STAGES, bool G128, bool ATM, bool REC>
__global__ void __launch_bounds__(THREADS, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap xmap, GemmArgs a) {
    using C = GemmCfg<NP, BN, STAGES, G128, ATM, REC>;
    constexpr int NA = C::NA;
    extern __shared__ __align__(1024) unsigned char dsm[];
    // 1024-byte aligned tile area (the 128-byte swizzle repeats every 1024 B)
    const uint32_t raw = smem_addr(dsm);
    const uint32_t tiles = (raw + 1023u) & ~1023u;
    // barriers: full_x[STAGES] (X tile landed), full_a[STAGES] (A expanded),
    // empty[STAGES] (MMAs of the stage done), acc (all MMAs done)
    const uint32_t bars = tiles + STAGES * C::STAGE_BYTES;
    auto full_x = [&](int s) { return bars + 8u * s; };
    auto full_a = [&](int s) { return bars + 8u * (STAGES + s); };
    auto empty_bar = [&](int s) { return bars + 8u * (2 * STAGES + s); };
    const uint32_t acc_bar = bars + 8u * (3 * STAGES);
    const uint32_t tmem_slot = acc_bar + 8u;
    const uint32_t abort_slot = tmem_slot + 4u;
    volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(dsm + (abort_slot - raw));
    auto a_tile = [&](int s, int p) { return tiles + s * C::STAGE_BYTES + p * A_TILE_BYTES; };
    auto b_tile = [&](int s) { return tiles + s * C::STAGE_BYTES + (ATM ? 0u : NA * A_TILE_BYTES); };
    // tensor-memory column of stage s, operand tile p of the A operand (ATM)
    auto a_col = [&](int s, int p) { return static_cast<uint32_t>(C::A_BASE + (s * NA + p) * (BK / 2)); };

    // the call's error word is cleared here rather than by a memset before
    // the launch: flags are raised only by waits that ran out, seconds after
    // the first CTA started
    if (blockIdx.x == 0 && blockIdx.y == 0 && threadIdx.x == 0) *a.err = 0u;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row_tile = blockIdx.x, tok_tile = blockIdx.y;
    const int64_t M = a.M, K = a.K;
    const int nk = static_cast<int>(K / BK);

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full_x(s), 1);
            mbar_init(full_a(s), 128);
            mbar_init(empty_bar(s), 1);
        }
        mbar_init(acc_bar, 1);
        *abort_flag = 0u;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) tmem_alloc(tmem_slot, C::TMEM_COLS);
    fence_before();
    __syncthreads();
    fence_after();
    uint32_t* err = a.err;
    const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t*>(dsm + (tmem_slot - raw));

    if (warp == 0) {
        // ---------------------------------------------------------- TMA producer
        if (elect_lane0()) {
            int issued = 0;
            for (int kb = 0; kb < nk; ++kb) {
                const int s = kb % STAGES;
                const uint32_t ph = static_cast<uint32_t>(kb / STAGES) & 1u;
                if (!mbar_wait(empty_bar(s), ph ^ 1u, abort_flag, err, 1u)) break;
                mbar_arrive_expect_tx(full_x(s), C::B_TILE_BYTES);
                tma_load_2d(b_tile(s), &xmap, kb * BK, tok_tile * BN, full_x(s));
                issued = kb + 1;
            }
            // after an abort, the loads still in flight land before the CTA
            // releases its shared memory: wait for the last load of each stage
            if (*abort_flag)
                for (int kb = issued - 1; kb >= 0 && kb >= issued - STAGES; --kb)
                    mbar_drain(full_x(kb % STAGES), static_cast<uint32_t>(kb / STAGES) & 1u);
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        // the whole warp runs the loop (warp-uniform operands); one elected
        // lane issues each MMA
        // The last token tile of a block may be narrower than BN: its MMAs
        // compute only the columns that hold tokens, rounded up to 16 (the
        // TMA box still fills BN rows, zeros past T; the epilogue stores
        // tokens < T only). With 240-wide tiles over 2048 tokens the ninth
        // tile holds 128 tokens, and those CTAs run last.
        const int t_left = a.T - tok_tile * BN;
        const uint32_t idesc = instr_desc(t_left >= BN ? BN : ((t_left + 15) & ~15));
        bool ok = true;
        for (int kb = 0; kb < nk && ok; ++kb) {
            const int s = kb % STAGES;
            const uint32_t ph = static_cast<uint32_t>(kb / STAGES) & 1u;
            if (!__all_sync(FULL_MASK, mbar_wait(full_x(s), ph, abort_flag, err, 2u) &&
                                           mbar_wait(full_a(s), ph, abort_flag, err, 2u))) {
                ok = false;
                break;
            }
            fence_after();
            const uint64_t bd0 = smem_desc(b_tile(s));
#pragma unroll
            for (int p = 0; p < NA; ++p) {
                const uint32_t d = tmem_base + static_cast<uint32_t>((G128 || REC) ? 0 : p * C::ACC_STRIDE);
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk) {
                    // +32 bytes along K inside the swizzled tile: +2 in the address field
                    const uint32_t acc = (kb > 0 || kk > 0 || (G128 && p > 0)) ? 1u : 0u;
                    if (ATM) umma_f16_ta_elect(d, tmem_base + a_col(s, p) + 8u * kk, bd0 + 2u * kk, idesc, acc);
                    else umma_f16_elect(d, smem_desc(a_tile(s, p)) + 2u * kk, bd0 + 2u * kk, idesc, acc);
                }
            }
            umma_commit_elect(empty_bar(s));      // stage s is free once these MMAs completed
        }
        umma_commit_elect(acc_bar);               // accumulators complete (also after an abort:
                                                  // the teardown waits on it before freeing TMEM)
    } else if (warp >= EXP_WARP0) {
        // ------------------------------------------------- expansion, then epilogue
        const int r = (warp - EXP_WARP0) * 32 + lane;            // row within the tile
        const int64_t row = static_cast<int64_t>(row_tile) * BM + r;
        const int64_t crow = row < M ? row : M - 1;               // rows past M read a real row
        const int64_t W32 = K >> 5;
        const int64_t S = (K + 511) >> 9;
        const int64_t gpr = K >> 7;
        // the two words (64 columns) of stage kb of path p of this row
        auto words_at = [&](int p, int kb) -> uint2 {
            const int64_t w = 2 * static_cast<int64_t>(kb);
            const uint32_t* src = a.sliced ? a.planes + ((p * S + (w >> 4)) * M + crow) * 16 + (w & 15)
                                           : a.planes + (p * M + crow) * W32 + w;
            return __ldg(reinterpret_cast<const uint2*>(src));
        };
        auto alpha_h2 = [&](int p, int kb) -> uint32_t {
            if (!G128) return 0x3C003C00u;                             // +1.0 in both halves
            const int64_t ai = (p * M + crow) * gpr + (static_cast<int64_t>(kb) * BK >> 7);
            // group scales are fp16 (the host refuses fp32 ones): +-alpha is exact
            const uint32_t hv = static_cast<const unsigned short*>(a.alpha)[ai];
            return hv | (hv << 16);
        };
        const uint32_t rsw = static_cast<uint32_t>(r & 7);
        const uint32_t row_off = static_cast<uint32_t>(r >> 3) * 1024u + rsw * 128u;
        const uint32_t lane_addr_q = static_cast<uint32_t>((warp - EXP_WARP0) * 32) << 16;   // this warp's lanes
        // The words (and group scales) of stage kb are loaded PD stages ahead
        // into a register ring, so a stage never waits for global memory even
        // when the tensor-core work per stage is short (few tokens).
        constexpr int PD = 16 / NP;
        // reconstruct-once: this row's two weight magnitudes, each the fp16
        // rounding of the exact sum or difference of its fp32 scales
        uint2 pq2 = make_uint2(0u, 0u);
        if (REC) {
            const double a0 = a.alpha_f16 ? __half2float(static_cast<const __half*>(a.alpha)[crow])
                                          : static_cast<const float*>(a.alpha)[crow];
            const double a1 = a.alpha_f16 ? __half2float(static_cast<const __half*>(a.alpha)[M + crow])
                                          : static_cast<const float*>(a.alpha)[M + crow];
            const uint32_t p = __half_as_ushort(__double2half(a0 + a1)), q = __half_as_ushort(__double2half(a0 - a1));
            pq2 = make_uint2(p | (p << 16), q | (q << 16));
        }
        uint2 ring[PD][NP];
        uint32_t aring[PD][NP];
#pragma unroll
        for (int i = 0; i < PD; ++i)
#pragma unroll
            for (int p = 0; p < NP; ++p) {
                if (i < nk) {
                    ring[i][p] = words_at(p, i);
                    aring[i][p] = alpha_h2(p, i);
                } else {
                    ring[i][p] = make_uint2(0u, 0u);
                    aring[i][p] = 0u;
                }
            }
        bool go = true;
        for (int kb0 = 0; kb0 < nk && go; kb0 += PD) {
#pragma unroll
            for (int i = 0; i < PD; ++i) {
                const int kb = kb0 + i;
                if (kb < nk && go) {
                    const int s = kb % STAGES;
                    const uint32_t ph = static_cast<uint32_t>(kb / STAGES) & 1u;
                    uint2 cur[NP];
                    uint32_t v2[NP];
#pragma unroll
                    for (int p = 0; p < NP; ++p) {
                        cur[p] = ring[i][p];
                        v2[p] = aring[i][p];
                        if (kb + PD < nk) {
                            ring[i][p] = words_at(p, kb + PD);
                            aring[i][p] = alpha_h2(p, kb + PD);
                        }
                    }
                    // warp-uniform: the tensor-memory stores below are .sync.aligned
                    if (!__all_sync(FULL_MASK, mbar_wait(empty_bar(s), ph ^ 1u, abort_flag, err, 4u))) {
                        go = false;
                    } else {
#pragma unroll
                        for (int p = 0; p < NA; ++p) {
                            const uint32_t base = a_tile(s, p) + row_off;
#pragma unroll
                            for (int half = 0; half < 2; ++half) {
                                uint32_t h[16];
                                if (REC) expand_word_rec(half ? cur[0].y : cur[0].x, half ? cur[1].y : cur[1].x, pq2.x,
                                                         pq2.y, h);
                                else expand_word(half ? cur[p].y : cur[p].x, v2[p], h);
                                if (ATM) {
                                    // row r is tensor-memory lane r; column j holds K-columns 2j, 2j+1
                                    tmem_store16(tmem_base + lane_addr_q + a_col(s, p) + 16u * half, h);
                                } else {
#pragma unroll
                                    for (int c4 = 0; c4 < 4; ++c4) {
                                        const uint32_t chunk = static_cast<uint32_t>(4 * half + c4);   // 16-byte chunk
                                        sts128(base + ((chunk ^ rsw) << 4), h[4 * c4], h[4 * c4 + 1], h[4 * c4 + 2],
                                               h[4 * c4 + 3]);
                                    }
                                }
                            }
                        }
                        if (ATM) {
                            tmem_store_wait();   // stores done first
                            fence_before();
                        } else {
                            fence_proxy_async_smem();   // make the generic-proxy stores visible to the tensor core
                        }
                        mbar_arrive(full_a(s));
                    }
                }
            }
        }

        // ------------------------------------------------------------ epilogue
        const bool ok = __all_sync(FULL_MASK, mbar_wait(acc_bar, 0u, abort_flag, err, 8u));
        fence_after();
        if (ok) {
            float al[C::NACC];
#pragma unroll
            for (int p = 0; p < C::NACC; ++p) {
                if (G128 || REC) al[p] = 1.0f;
                else al[p] = a.alpha_f16 ? __half2float(static_cast<const __half*>(a.alpha)[p * M + crow])
                                         : static_cast<const float*>(a.alpha)[p * M + crow];
            }
            const uint32_t lane_addr = static_cast<uint32_t>((warp - EXP_WARP0) * 32) << 16;
            const int t_base = tok_tile * BN;
            // columns per tensor-memory load (a divisor of BN)
            constexpr int CW = BN < 32 ? BN : (BN % 32 == 0 ? 32 : 16);
            for (int c0 = 0; c0 < BN; c0 += CW) {
                float yv[CW];
#pragma unroll
                for (int i = 0; i < CW; ++i) yv[i] = 0.0f;
#pragma unroll
                for (int p = 0; p < C::NACC; ++p) {
                    uint32_t v[CW];
                    const uint32_t taddr = tmem_base + lane_addr + static_cast<uint32_t>(p * C::ACC_STRIDE + c0);
                    tmem_load<CW>(taddr, v);
#pragma unroll
                    for (int i = 0; i < CW; ++i) yv[i] = fmaf(al[p], __uint_as_float(v[i]), yv[i]);
                }
                if (row < M) {
#pragma unroll
                    for (int i = 0; i < CW; ++i) {
                        const int t = t_base + c0 + i;
                        if (t < a.T) {
                            if (a.y_f16) static_cast<__half*>(a.y)[t * a.ldy + row] = __float2half_rn(yv[i]);
                            else static_cast<float*>(a.y)[t * a.ldy + row] = yv[i];
                        }
                    }
                }
            }
        }
    }

    __syncwarp();            // lanes 1..31 of warp 0 wait for their lane 0
    fence_before();
    __syncthreads();
    if (warp == 1) {
        // after an abort, the MMAs already issued finish before their tensor
        // memory is released (the MMA warp committed them to acc_bar)
        if (*abort_flag) mbar_drain(acc_bar, 0u);
        __syncwarp();
        fence_after();
        tmem_dealloc(tmem_base, C::TMEM_COLS);
    }
}

// ---------------------------------------------------------------- host side
template <int NP, int BN, int STAGES, bool G128, bool ATM, bool REC>
cudaError_t launch_cfg(const GemmArgs& a, const void* X, int64_t ldx, cudaStream_t s) {
    using C = GemmCfg<NP, BN, STAGES, G128, ATM, REC>;
    CUtensorMap map;
    cudaError_t me = make_x_map(&map, X, a.K, a.T, ldx, BN);
    if (me != cudaSuccess) return me;
    auto kern = gemm_tc_kernel<NP, BN, STAGES, G128, ATM, REC>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    dim3 grid(static_cast<unsigned>((a.M + BM - 1) / BM), static_cast<unsigned>((a.T + BN - 1) / BN));
    kern<<<grid, THREADS, C::SMEM_BYTES, s>>>(map, a);
    return cudaGetLastError();
}

}  // namespace

// stages that fit in shared memory for a configuration (at most 8); na
// operand tiles per stage
constexpr int stages_for(int na, int bn) {
    return ((210 * 1024) / static_cast<int>(na * A_TILE_BYTES + bn * BK * 2)) < 8
               ? ((210 * 1024) / static_cast<int>(na * A_TILE_BYTES + bn * BK * 2))
               : 8;
}

// stages of the A operand (na tiles) that fit in tensor memory beside nacc
// accumulators of a token tile (0: fewer than two, use shared memory for A)
constexpr int atm_stages(int na, int nacc, int bn) {
    const int stride = bn <= 16 ? 16 : bn <= 32 ? 32 : bn <= 64 ? 64 : bn <= 128 ? 128 : 256;
    const int st = (512 - nacc * stride) / (na * BK / 2);
    return st >= 2 ? (st < 8 ? st : 8) : 0;
}

// A in tensor memory when it fits (always for token tiles up to 128; for
// wider tiles with a single accumulator), else in shared memory
template <int NP, int BN, bool G128, bool REC>
cudaError_t launch_tile(const GemmArgs& a, const void* X, int64_t ldx, cudaStream_t s) {
    constexpr int NA = REC ? 1 : NP, NACC = (G128 || REC) ? 1 : NP;
    // with A in tensor memory a stage is only the X tile: also bounded by shared memory
    constexpr int SX = (210 * 1024) / (BN * BK * 2);
    constexpr int SA = atm_stages(NA, NACC, BN) < SX ? atm_stages(NA, NACC, BN) : SX;
    if constexpr (SA >= 2 && (BN <= 128 || REC)) return launch_cfg<NP, BN, SA, G128, true, REC>(a, X, ldx, s);
    else return launch_cfg<NP, BN, stages_for(NA, BN), G128, false, REC>(a, X, ldx, s);
}

template <int NP, bool G128, bool REC = false>
cudaError_t launch_np(const GemmArgs& a, const void* X, int64_t ldx, cudaStream_t s) {
    // token tile: the narrowest of 16..256 that covers T (MMA N), so small
    // batches do not pay for unused columns; the accumulators must fit in
    // 512 tensor-memory columns
    constexpr int BN_MAX = (G128 || REC) ? 256 : (NP <= 2 ? 256 : 128);
    const int T = a.T;
    if (T <= 16) return launch_tile<NP, 16, G128, REC>(a, X, ldx, s);
    if (T <= 32) return launch_tile<NP, 32, G128, REC>(a, X, ldx, s);
    if (T <= 64) return launch_tile<NP, 64, G128, REC>(a, X, ldx, s);
    if constexpr (BN_MAX == 128) {
        return launch_tile<NP, 128, G128, REC>(a, X, ldx, s);
    } else {
    if (T <= 128) return launch_tile<NP, 128, G128, REC>(a, X, ldx, s);
    // Wide token tiles: 240 instead of 256 when the last wave of 256-wide
    // tiles would leave most SMs idle and 240 needs no extra wave: e.g. 112
    // row tiles x 2048 tokens are 896 tiles of 256 (6 full waves on 148 SMs
    // and 8 tiles in a seventh) or 1008 of 240 (7 waves, the last 81 % full).
    // Measured: 14336 x 4096 x 2048 tokens 374 -> 350 us; 4096 x 14336 (256
    // tiles of 256, last wave 73 % full) is slower with 240 and keeps 256.
    const int64_t rows = (a.M + BM - 1) / BM, sms = device_sm_count();
    const int64_t tiles256 = rows * ((T + 255) / 256), tiles240 = rows * ((T + 239) / 240);
    const int64_t waves256 = (tiles256 + sms - 1) / sms, waves240 = (tiles240 + sms - 1) / sms;
    const int64_t last256 = tiles256 - (waves256 - 1) * sms;
    if (waves240 <= waves256 && 2 * last256 < sms) return launch_tile<NP, 240, G128, REC>(a, X, ldx, s);
    return launch_tile<NP, BN_MAX, G128, REC>(a, X, ldx, s);
    }
}

cudaError_t launch_gemm_prefill(const uint32_t* planes, const void* alpha, bool alpha_f16, int64_t M, int64_t K,
                                int n_paths, int group, bool sliced, const void* X, int64_t ldx, int T, void* Y,
                                bool y_f16, int64_t ldy, uint32_t* err, bool reconstruct, cudaStream_t s) {
    GemmArgs a{err, planes, alpha, Y, M, K, ldy, T, n_paths, group == 128, sliced, alpha_f16, y_f16};
    if (reconstruct) {
        if (n_paths != 2 || group != 0) return cudaErrorInvalidValue;
        return launch_np<2, false, true>(a, X, ldx, s);
    }
    if (group == 0) {
        switch (n_paths) {
            case 1: return launch_np<1, false>(a, X, ldx, s);
            case 2: return launch_np<2, false>(a, X, ldx, s);
            case 3: return launch_np<3, false>(a, X, ldx, s);
            case 4: return launch_np<4, false>(a, X, ldx, s);
        }
    } else {
        switch (n_paths) {
            case 1: return launch_np<1, true>(a, X, ldx, s);
            case 2: return launch_np<2, true>(a, X, ldx, s);
            case 3: return launch_np<3, true>(a, X, ldx, s);
            case 4: return launch_np<4, true>(a, X, ldx, s);
        }
    }
    return cudaErrorInvalidValue;
}

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

cudaError_t make_x_map(CUtensorMap* map, const void* X, int64_t cols, int64_t rows, int64_t ld, int box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(tc::BK), static_cast<cuuint32_t>(box_rows)};
    const cuuint32_t estr[2] = {1, 1};
    if (enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(X), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    return cudaSuccess;
}

cudaError_t make_x8_map(CUtensorMap* map, const void* X, int64_t cols, int64_t rows, int terms, int box_rows) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    const cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows),
                                static_cast<cuuint64_t>(terms)};
    const cuuint64_t strides[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(cols) * rows};
    const cuuint32_t box[3] = {128u, static_cast<cuuint32_t>(box_rows), static_cast<cuuint32_t>(terms)};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(X), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    return cudaSuccess;
}

}  // namespace rb
