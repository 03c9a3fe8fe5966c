// rb_gemv: y_t = sum_k alpha_k (.) (B_k x_t) on CUDA cores, all paths in one pass.
//
// RaBiT (arXiv 2602.05367) section 4.1 and appendix D evaluate the layer
// without multiplications, with additions and subtractions over bit-packed
// planes. Here every 8-column block c of x is expanded once per CTA into a
// shared-memory table of its 256 signed sums
//     T[b][c] = sum_e (bit e of b ? +x[8c+e] : -x[8c+e])
// (2 * masked sum - block sum, built from two 16-entry nibble tables), so a
// plane byte b costs one PRMT (which forms the table address from the byte
// and a per-lane base), one LDS and one FADD: 3 instructions per 8 weight
// bits instead of >= 1 per bit for a select-and-add.
//
// Table layout: 256 rows of 64 fp32 entries (one 512-column slice of x),
// 64 KB, at shared-window address 0x10000 (a second one, for double
// buffering, at 0x20000). With the table 64 KB aligned the address of entry
// (b, c) is 0x10000 | b << 8 | 4c: PRMT takes byte 0 (4c) and bytes 2-3 from
// the lane's base register and byte 1 from the plane word.
//
// Work split. A CTA (32 warps) owns R rows of one matrix for a K chunk and
// walks its 512-column slices. An item (row, path) of a slice is 16 plane
// words; 8 lanes hold one item, two consecutive words per lane, so one
// warp-wide 64-bit load covers 4 items: 4 consecutive rows of one path, which
// in the sliced plane layout are 256 contiguous bytes (and the items of one
// path sit at immediate offsets from one pointer). Each lane issues J such
// loads per slice. Lanes whose words would share banks process their two
// words in opposite order and rotate the byte order, which puts the 32 lanes
// of every LDS on 32 distinct banks. Partial sums stay in registers across
// the slices of the chunk and are reduced over the 8 lanes of each item at
// the end.
//
// Per-row scales are applied once per row at the end; per-128-column scales
// (the QBB layout) multiply each word's partial sum as it is accumulated.
// A K chunk that is only part of the row writes fp32 partial sums to the
// workspace; the last CTA to finish a row block adds them in chunk order.
#include "rb_internal.cuh"

namespace rb {
namespace {

constexpr int THREADS = 1024;
constexpr int WARPS = THREADS / 32;
constexpr int SLICE_COLS = 512;
constexpr uint32_t TBL0 = 0x10000u;
constexpr uint32_t TBL_TOGGLE = 0x30000u;   // 0x10000 <-> 0x20000
constexpr int SMEM_BYTES = 0x30000;          // covers both tables whatever the window base
constexpr int MAX_JOBS = 2 * THREADS - 1;    // each thread scans two descriptors

// Low shared region (below 0x10000): totals, job prefix sums, staged x.
struct __align__(16) LowSmem {
    float tot[WARPS][32];
    uint32_t unit_prefix[MAX_JOBS + 1];
    uint32_t ctr_prefix[MAX_JOBS + 1];
    uint32_t part_prefix[MAX_JOBS + 1];
    uint32_t wsum[3][WARPS];
    uint4 xstage[2][64];      // x of the next slices, staged by cp.async
    uint32_t bcast;
    uint32_t last;
};

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

__device__ __forceinline__ float lds(uint32_t addr) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ void sts(uint32_t addr, float v) {
    asm volatile("st.shared.f32 [%0], %1;" ::"r"(addr), "f"(v));
}

// CTA barrier that also orders the inline-asm shared accesses around it.
__device__ __forceinline__ void cta_sync() { asm volatile("bar.sync 0;" ::: "memory"); }

// The same barrier for code that warps reach from different branches (the
// full and the partial copy of the slice loop): the non-aligned form.
__device__ __forceinline__ void cta_sync_any() { asm volatile("barrier.sync 0;" ::: "memory"); }

// base + a * b bytes as one 32x32 -> 64-bit multiply-add
__device__ __forceinline__ const char* mad_ptr(uint32_t a, uint32_t b, const void* base) {
    uint64_t r;
    asm("mad.wide.u32 %0, %1, %2, %3;" : "=l"(r) : "r"(a), "r"(b), "l"(base));
    return reinterpret_cast<const char*>(r);
}

// m ? b : a, bitwise (m is all ones or all zeros): one LOP3
__device__ __forceinline__ uint32_t sel_mask(uint32_t a, uint32_t b, uint32_t m) {
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, %3, 0xD8;" : "=r"(d) : "r"(a), "r"(b), "r"(m));
    return d;
}

__device__ __forceinline__ uint2 ldg_words2(const void* p) {
    uint2 v;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t ldg_word(const void* p) {
    uint32_t v;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

template <bool B>
struct BoolC { static constexpr bool value = B; };

template <int J>
struct Log2 { static constexpr int v = J == 16 ? 4 : J == 8 ? 3 : J == 4 ? 2 : J == 2 ? 1 : 0; };

// A warp-wide 64-bit load reads 4 items (consecutive rows of one path, 8
// lanes per item, 2 words per lane); J such loads per lane and slice.
template <int NP, bool G128>
struct Cfg {
    static constexpr int J = G128 && NP <= 4 ? 4 : 8;  // item loads per lane per slice (>= NP)
    static constexpr int HR = J / NP > 0 ? J / NP : 1; // row quads per path per warp
    static constexpr int RW = 4 * HR;                 // rows per warp
    static constexpr int JV = NP * HR <= J ? NP * HR : J;   // loads in use
    static constexpr int R = WARPS * RW;              // rows per CTA
};

__device__ __forceinline__ int slices_of(int64_t K) { return static_cast<int>((K + SLICE_COLS - 1) / SLICE_COLS); }

// Stage the 512 x values of slice `s` into `dst` (64 x 16 bytes): threads
// 0..63 each copy one 16-byte block with cp.async; blocks past K are zeroed,
// so the table entries of columns past K are 0 and unused plane bits add 0.
__device__ __forceinline__ void stage_x(const __half* __restrict__ xt, int64_t K, int s, uint4* dst) {
    const int c = threadIdx.x;
    if (c < 64) {
        const int64_t col = static_cast<int64_t>(s) * SLICE_COLS + 8 * c;
        if (col < K) {
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_addr(dst + c)), "l"(xt + col) : "memory");
        } else {
            dst[c] = make_uint4(0u, 0u, 0u, 0u);
        }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
}

// Wait until this thread's staged copies are complete (the CTA barrier that
// follows makes them visible to every thread).
__device__ __forceinline__ void stage_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Write the signed-sum table of one slice into the table at `tbl`: thread
// (c = tid % 64, hi = tid / 64) writes the 16 entries whose high nibble is hi.
__device__ __forceinline__ void build_table(const uint4* xs, uint32_t tbl) {
    const int c = threadIdx.x & 63;
    const int hi = threadIdx.x >> 6;
    const uint4 xv = xs[c];
    const __half2* h2 = reinterpret_cast<const __half2*>(&xv);
    float x[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 f = __half22float2(h2[i]);
        x[2 * i] = f.x;
        x[2 * i + 1] = f.y;
    }
    // nibble tables of signed sums: bit e set -> +x_e, clear -> -x_e
    float p01[4], p23[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        p01[i] = ((i & 1) ? x[0] : -x[0]) + ((i & 2) ? x[1] : -x[1]);
        p23[i] = ((i & 1) ? x[2] : -x[2]) + ((i & 2) ? x[3] : -x[3]);
    }
    const float hsum = (((hi & 1) ? x[4] : -x[4]) + ((hi & 2) ? x[5] : -x[5])) +
                       (((hi & 4) ? x[6] : -x[6]) + ((hi & 8) ? x[7] : -x[7]));
    float q01[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) q01[i] = p01[i] + hsum;
    const uint32_t a0 = tbl + (static_cast<uint32_t>(hi) << 12) + 4u * c;
#pragma unroll
    for (int lo = 0; lo < 16; ++lo) sts(a0 + (lo << 8), q01[lo & 3] + p23[lo >> 2]);
}

// Reduce acc[0..J) over the 8 lanes of an item group (lane bits 0-2); J is
// a power of two <= 8. Afterwards lane t of the group holds the sum of item
// load j = t >> (3 - log2 J) in acc[0].
template <int J>
__device__ __forceinline__ void group8_transpose_reduce(float (&acc)[J], int t) {
    int cnt = J;
#pragma unroll
    for (int off = 4; off >= 1; off >>= 1) {
        if (cnt > 1) {
            const int half = cnt >> 1;
            const bool up = (t & off) != 0;
#pragma unroll
            for (int i = 0; i < J / 2; ++i) {
                if (i < half) {
                    const float send = up ? acc[i] : acc[i + half];
                    const float keep = up ? acc[i + half] : acc[i];
                    acc[i] = keep + __shfl_xor_sync(FULL_MASK, send, off);
                }
            }
            cnt = half;
        } else {
            acc[0] += __shfl_xor_sync(FULL_MASK, acc[0], off);
        }
    }
}

struct UnitInfo {
    GvJob jb;
    int j, t, ch, rb, nch, s_begin, s_end;
    int64_t ldx, ldy;
};

// Unit u -> job (binary search of the prefix), then (row block, chunk, token)
// with the token fastest, so CTAs that run together share plane rows in L2.
__device__ __forceinline__ UnitInfo decode_unit(const GvArgs& p, const LowSmem& lo, int n_jobs, uint32_t u) {
    UnitInfo ui;
    int jlo = 0, jhi = n_jobs - 1;
    while (jlo < jhi) {
        const int mid = (jlo + jhi + 1) >> 1;
        if (lo.unit_prefix[mid] <= u) jlo = mid; else jhi = mid - 1;
    }
    ui.j = jlo;
    ui.jb = p.jobs ? p.jobs[jlo] : p.one;
    ui.ldx = p.jobs ? ui.jb.K : p.ldx;
    ui.ldy = p.jobs ? ui.jb.M : p.ldy;
    const int S = slices_of(ui.jb.K);
    ui.nch = (S + p.chunk_slices - 1) / p.chunk_slices;
    uint32_t r = u - lo.unit_prefix[jlo];
    ui.t = static_cast<int>(r % static_cast<uint32_t>(p.T));
    r /= static_cast<uint32_t>(p.T);
    ui.ch = static_cast<int>(r % static_cast<uint32_t>(ui.nch));
    ui.rb = static_cast<int>(r / static_cast<uint32_t>(ui.nch));
    ui.s_begin = ui.ch * p.chunk_slices;
    ui.s_end = min(S, ui.s_begin + p.chunk_slices);
    return ui;
}

// Every CTA computes the same unit prefix sums over the jobs: each thread
// counts two descriptors, then one block-wide scan.
template <int R>
__device__ __forceinline__ void scan_jobs(const GvArgs& p, LowSmem& lo, int n_jobs) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int T = p.T;
    uint32_t cu[2] = {0, 0}, cc[2] = {0, 0}, cq[2] = {0, 0};
#pragma unroll
    for (int e = 0; e < 2; ++e) {
        const int j = 2 * tid + e;
        if (j < n_jobs) {
            const int64_t jM = p.jobs ? p.jobs[j].M : p.one.M;
            const int64_t jK = p.jobs ? p.jobs[j].K : p.one.K;
            const int nrb = static_cast<int>((jM + R - 1) / R);
            const int nch = (slices_of(jK) + p.chunk_slices - 1) / p.chunk_slices;
            cu[e] = static_cast<uint32_t>(nrb * nch * T);
            if (nch > 1) {
                cc[e] = static_cast<uint32_t>(nrb * T);
                cq[e] = static_cast<uint32_t>(nch * T) * static_cast<uint32_t>(jM);
            }
        }
    }
    uint32_t su = cu[0] + cu[1], sc = cc[0] + cc[1], sq = cq[0] + cq[1];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const uint32_t a1 = __shfl_up_sync(FULL_MASK, su, off);
        const uint32_t a2 = __shfl_up_sync(FULL_MASK, sc, off);
        const uint32_t a3 = __shfl_up_sync(FULL_MASK, sq, off);
        if (lane >= off) { su += a1; sc += a2; sq += a3; }
    }
    if (lane == 31) { lo.wsum[0][warp] = su; lo.wsum[1][warp] = sc; lo.wsum[2][warp] = sq; }
    cta_sync();
    if (warp == 0) {
        uint32_t v0 = lo.wsum[0][lane], v1 = lo.wsum[1][lane], v2 = lo.wsum[2][lane];
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const uint32_t a1 = __shfl_up_sync(FULL_MASK, v0, off);
            const uint32_t a2 = __shfl_up_sync(FULL_MASK, v1, off);
            const uint32_t a3 = __shfl_up_sync(FULL_MASK, v2, off);
            if (lane >= off) { v0 += a1; v1 += a2; v2 += a3; }
        }
        lo.wsum[0][lane] = v0; lo.wsum[1][lane] = v1; lo.wsum[2][lane] = v2;   // inclusive
    }
    cta_sync();
    const uint32_t bu = warp ? lo.wsum[0][warp - 1] : 0u;
    const uint32_t bc = warp ? lo.wsum[1][warp - 1] : 0u;
    const uint32_t bq = warp ? lo.wsum[2][warp - 1] : 0u;
    const uint32_t eu = bu + su - (cu[0] + cu[1]);
    const uint32_t ec = bc + sc - (cc[0] + cc[1]);
    const uint32_t eq = bq + sq - (cq[0] + cq[1]);
    const int j0 = 2 * tid;
    if (j0 <= n_jobs) { lo.unit_prefix[j0] = eu; lo.ctr_prefix[j0] = ec; lo.part_prefix[j0] = eq; }
    if (j0 + 1 <= n_jobs) {
        lo.unit_prefix[j0 + 1] = eu + cu[0]; lo.ctr_prefix[j0 + 1] = ec + cc[0]; lo.part_prefix[j0 + 1] = eq + cq[0];
    }
    cta_sync();
}

template <int NP, bool G128, bool A16, bool SLICED>
__global__ void __launch_bounds__(THREADS, 1) gemv_lut_kernel(GvArgs p, uint32_t* __restrict__ hdr,
                                                              uint32_t* __restrict__ ctrs,
                                                              float* __restrict__ parts) {
    using C = Cfg<NP, G128>;
    constexpr int J = C::J, HR = C::HR;
    extern __shared__ __align__(16) unsigned char dsm[];
    LowSmem& lo = *reinterpret_cast<LowSmem*>(dsm);

    const uint32_t s0 = smem_addr(dsm);
    if (s0 + sizeof(LowSmem) > TBL0 || s0 + SMEM_BYTES < TBL0 + 2 * 0x10000u) {
        if (threadIdx.x == 0) atomicOr(hdr + 1, GV_ERR_SMEM_LAYOUT);
        return;
    }
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // lane -> item q4 of each 4-item load, word pair t (words 2t, 2t + 1)
    const int q4 = lane >> 3, t8 = lane & 7;
    const int T = p.T;
    const int n_jobs = p.jobs ? p.n_jobs : 1;
    if (n_jobs > MAX_JOBS) {
        if (tid == 0) atomicOr(hdr + 1, GV_ERR_TOO_MANY_JOBS);
        return;
    }
    scan_jobs<C::R>(p, lo, n_jobs);
    const uint32_t total_units = lo.unit_prefix[n_jobs];

    // The 8 lanes sharing t8 & 3 (t8 in {a, a + 4}, 4 items) would hit the
    // same banks; lane z = (t8 >> 2) + 2 q4 swaps its two words when z is odd
    // (rv) and rotates the byte order by rq = z >> 1, so every LDS touches 32
    // distinct banks.
    const uint32_t zr = static_cast<uint32_t>((t8 >> 2) + 2 * q4);
    const uint32_t rv = zr & 1u, rq = zr >> 1;
    const uint32_t swap_mask = 0u - rv;
    uint32_t sel[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) sel[q] = 0x7604u | (((static_cast<uint32_t>(q) + rq) & 3u) << 4);

    uint32_t iter = 0;
    while (true) {
        uint32_t u;
        if (p.dynamic) {
            if (tid == 0) lo.bcast = atomicAdd(hdr, 1u);
            cta_sync();
            u = lo.bcast;
            cta_sync();
        } else {
            u = blockIdx.x + iter * gridDim.x;
        }
        ++iter;
        if (u >= total_units) break;

        const UnitInfo ui = decode_unit(p, lo, n_jobs, u);
        const GvJob& jb = ui.jb;
        const int64_t M = jb.M, K = jb.K;
        const int S = slices_of(K);
        const int s_begin = ui.s_begin, s_end = ui.s_end;
        const uint32_t uM = static_cast<uint32_t>(M);
        const uint32_t uW32 = static_cast<uint32_t>(K >> 5);
        const uint32_t gpr = static_cast<uint32_t>(K >> 7);
        const uint32_t row0 = static_cast<uint32_t>(ui.rb) * C::R + warp * C::RW;
        const __half* xt = static_cast<const __half*>(jb.x) + ui.t * ui.ldx;
        // plane bytes per path in each layout
        const uint32_t path_bytes = SLICED ? static_cast<uint32_t>(S) * 64u * uM : uM * uW32 * 4u;
        // a full warp has every row of its items below M; others clamp rows
        // (the sums of the extra rows are computed and dropped)
        const bool full = row0 + C::RW <= uM;

        float acc[J];
        uint2 wv[J];
        float av[J];
#pragma unroll
        for (int j = 0; j < J; ++j) {
            acc[j] = 0.0f;
            av[j] = 0.0f;
        }
        // table address base of step (word v, byte q): column 8 t8 + 4 (v ^ rv) + (q + rq) & 3
        uint32_t cur_base[8];
#pragma unroll
        for (int v = 0; v < 2; ++v)
#pragma unroll
            for (int q = 0; q < 4; ++q)
                cur_base[4 * v + q] = TBL0 + 4u * (8u * t8 + 4u * (static_cast<uint32_t>(v) ^ rv) +
                                                   ((static_cast<uint32_t>(q) + rq) & 3u));

        // word pair of lane t8 in slice s, clamped in a partial last slice
        // (the table entries past K are 0, so a clamped pair adds nothing);
        // the sliced layout pads the last slice, so only the scale index and
        // the row layout need it
        auto lane_pair = [&](int s) -> uint32_t {
            const int ws = min(16, static_cast<int>((K - static_cast<int64_t>(s) * SLICE_COLS) >> 5));
            return 2 * t8 < ws ? static_cast<uint32_t>(t8) : 0u;
        };
        auto alpha_at = [&](size_t ai) -> float {
            return A16 ? __half2float(static_cast<const __half*>(jb.alpha)[ai]) : static_cast<const float*>(jb.alpha)[ai];
        };
        // Item load j: path j / HR, rows row0 + 4 (j % HR) + q4. Its lane
        // pointer = path pointer + (j % HR) * (4 rows): an immediate offset in
        // the sliced layout. The per-slice row goes through an empty asm so
        // the compiler cannot hoist per-item values.
        struct SliceAddr {
            const char* slice0;   // (path 0, row 0, pair tsel) of the slice
            const char* lane0;    // (path 0, row r0 + q4, pair tsel): full warps
            uint32_t r0, tp;
        };
        const uint32_t row_bytes = SLICED ? 64u : uW32 * 4u;
        auto slice_addr = [&](int s) {
            SliceAddr a;
            a.tp = lane_pair(s);
            a.r0 = row0;
            asm volatile("" : "+r"(a.r0));
            const uint32_t tsel = SLICED ? static_cast<uint32_t>(t8) : a.tp;
            a.slice0 = reinterpret_cast<const char*>(jb.planes) +
                       (SLICED ? (static_cast<size_t>(s) * uM * 16u + 2u * tsel) * 4u
                               : (16u * static_cast<uint32_t>(s) + 2u * tsel) * 4u);
            a.lane0 = mad_ptr(a.r0 + q4, row_bytes, a.slice0);
            return a;
        };
        // load item j of the slice at `a` (words swapped on lanes with rv)
        auto fetch = [&](int j, int s, const SliceAddr& a, auto full_tag) {
            constexpr bool F = decltype(full_tag)::value;
            const uint32_t path = j / HR, rr = j % HR;
            uint32_t row;
            const char* wp;
            if (F) {
                row = a.r0 + q4 + 4u * rr;
                const char* pb = path ? mad_ptr(path, path_bytes, a.lane0) : a.lane0;
                wp = SLICED ? pb + rr * 256u : mad_ptr(4u * rr, row_bytes, pb);
            } else {
                // rows past M are clamped to the last row (absolute address)
                row = min(a.r0 + q4 + 4u * rr, uM - 1u);
                wp = mad_ptr(row, row_bytes, path ? mad_ptr(path, path_bytes, a.slice0) : a.slice0);
            }
            // K is a multiple of 128, so rows of either layout are a multiple
            // of 16 bytes, the planes are 16-byte aligned and a slice holds an
            // even number of words: the pair is one aligned 8-byte load
            wv[j] = ldg_words2(wp);
            if (G128) av[j] = alpha_at(static_cast<size_t>(path * uM + row) * gpr + 4u * s + (a.tp >> 1));
        };
        auto fetch_slice = [&](int s, auto full_tag) {
            const SliceAddr a = slice_addr(s);
#pragma unroll
            for (int j = 0; j < J; ++j)
                if (j < C::JV) fetch(j, s, a, full_tag);
        };
        // consume slice s from the current table; with PF, item j of slice
        // s + 1 is loaded right after item j of slice s was used, so each load
        // has about one slice of time to arrive
        auto consume = [&](int s, auto full_tag, auto pf_tag) {
            constexpr bool PF = decltype(pf_tag)::value;
            SliceAddr an;
            if (PF) an = slice_addr(s + 1);
#pragma unroll
            for (int j = 0; j < J; ++j) {
                if (j >= C::JV) continue;
                // the word swap of lanes with rv happens here, where the words
                // are used, not where they are loaded (a use right after the
                // load would wait for it)
                const uint32_t w0 = sel_mask(wv[j].x, wv[j].y, swap_mask);
                const uint32_t w1 = sel_mask(wv[j].y, wv[j].x, swap_mask);
                const float v0 = lds(prmt(w0, cur_base[0], sel[0]));
                const float v1 = lds(prmt(w0, cur_base[1], sel[1]));
                const float v2 = lds(prmt(w0, cur_base[2], sel[2]));
                const float v3 = lds(prmt(w0, cur_base[3], sel[3]));
                const float v4 = lds(prmt(w1, cur_base[4], sel[0]));
                const float v5 = lds(prmt(w1, cur_base[5], sel[1]));
                const float v6 = lds(prmt(w1, cur_base[6], sel[2]));
                const float v7 = lds(prmt(w1, cur_base[7], sel[3]));
                const float ps = ((v0 + v1) + (v2 + v3)) + ((v4 + v5) + (v6 + v7));
                if (G128) acc[j] = fmaf(av[j], ps, acc[j]);
                else acc[j] += ps;
                if (PF) fetch(j, s + 1, an, full_tag);
            }
        };

        // ---- slice pipeline: table of slice s in buffer (s - s_begin) & 1;
        // the x of slice s + 2 is staged while slice s is consumed, so each
        // slice needs one CTA barrier. Full and partial warps run separate
        // copies of the whole loop (non-aligned barriers), the last slice is
        // peeled, so the steady-state loop is one straight-line block.
        auto run_unit = [&](auto full_tag) {
            fetch_slice(s_begin, full_tag);
            stage_x(xt, K, s_begin, lo.xstage[0]);
            stage_wait_all();
            cta_sync_any();
            build_table(lo.xstage[0], TBL0);
            if (s_begin + 1 < s_end) stage_x(xt, K, s_begin + 1, lo.xstage[1]);
            stage_wait_all();
            cta_sync_any();
            for (int s = s_begin; s < s_end - 1; ++s) {
                const int par = (s - s_begin) & 1;
                build_table(lo.xstage[par ^ 1], par ? TBL0 : TBL0 + 0x10000u);
                if (s + 2 < s_end) stage_x(xt, K, s + 2, lo.xstage[par]);
                consume(s, full_tag, BoolC<true>{});
#pragma unroll
                for (int q = 0; q < 8; ++q) cur_base[q] ^= TBL_TOGGLE;
                stage_wait_all();
                cta_sync_any();
            }
            consume(s_end - 1, full_tag, BoolC<false>{});
            cta_sync_any();
        };
        if (full) run_unit(BoolC<true>{});
        else run_unit(BoolC<false>{});

        // the unit's indices are decoded again rather than kept live across
        // the slice loop, which leaves the registers to the accumulators
        asm volatile("" : "+r"(u));
        const UnitInfo ue = decode_unit(p, lo, n_jobs, u);

        // ---- reduce over the 8 lanes of each item; lane t8 owns load j = t8 >> shift
        group8_transpose_reduce<J>(acc, t8);
        constexpr int shift = 3 - Log2<J>::v;
        if ((t8 & ((1 << shift) - 1)) == 0) lo.tot[warp][4 * (t8 >> shift) + q4] = acc[0];
        __syncwarp();

        // ---- per-row output of this chunk: lane r < RW owns row r of the warp,
        // whose path-k item is load k * HR + r / 4 of item group r % 4
        float yv = 0.0f;
        const int64_t my_row = static_cast<int64_t>(ue.rb) * C::R + warp * C::RW + lane;
        const bool row_ok = lane < C::RW && my_row < ue.jb.M;
        if (row_ok) {
#pragma unroll
            for (int k = 0; k < NP; ++k) {
                const float tk = lo.tot[warp][4 * (k * HR + (lane >> 2)) + (lane & 3)];
                if (G128) {
                    yv += tk;
                } else {
                    const size_t ai = static_cast<size_t>(k) * ue.jb.M + my_row;
                    const float a = p.alpha_f16 ? __half2float(static_cast<const __half*>(ue.jb.alpha)[ai])
                                                : static_cast<const float*>(ue.jb.alpha)[ai];
                    yv = fmaf(a, tk, yv);
                }
            }
        }
        if (ue.nch == 1) {
            if (row_ok) {
                if (p.y_f16) static_cast<__half*>(ue.jb.y)[ue.t * ue.ldy + my_row] = __float2half_rn(yv);
                else static_cast<float*>(ue.jb.y)[ue.t * ue.ldy + my_row] = yv;
            }
        } else {
            float* part = parts + lo.part_prefix[ue.j] + (static_cast<size_t>(ue.t) * ue.nch) * ue.jb.M;
            if (row_ok) part[static_cast<size_t>(ue.ch) * ue.jb.M + my_row] = yv;
            __threadfence();
            cta_sync();
            if (tid == 0) {
                const uint32_t prev = atomicAdd(ctrs + lo.ctr_prefix[ue.j] + ue.rb * T + ue.t, 1u);
                lo.last = (prev == static_cast<uint32_t>(ue.nch - 1)) ? 1u : 0u;
            }
            cta_sync();
            if (lo.last) {
                __threadfence();
                const int64_t rbase = static_cast<int64_t>(ue.rb) * C::R;
                for (int i = tid; i < C::R; i += THREADS) {
                    const int64_t row = rbase + i;
                    if (row < ue.jb.M) {
                        float sum = 0.0f;
                        for (int c = 0; c < ue.nch; ++c) sum += __ldcg(part + static_cast<size_t>(c) * ue.jb.M + row);
                        if (p.y_f16) static_cast<__half*>(ue.jb.y)[ue.t * ue.ldy + row] = __float2half_rn(sum);
                        else static_cast<float*>(ue.jb.y)[ue.t * ue.ldy + row] = sum;
                    }
                }
            }
        }
        cta_sync();
    }
}

template <int NP, bool G128, bool A16, bool SLICED>
cudaError_t launch_one(const GvArgs& a, const GvPlan& plan, cudaStream_t s) {
    auto kern = gemv_lut_kernel<NP, G128, A16, SLICED>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    uint32_t* hdr = static_cast<uint32_t*>(a.workspace);
    uint32_t* ctrs = reinterpret_cast<uint32_t*>(static_cast<char*>(a.workspace) + GV_HEADER_BYTES);
    float* parts = reinterpret_cast<float*>(ctrs + ((plan.counters + 3) & ~size_t(3)));
    const int sms = device_sm_count();
    size_t grid = a.dynamic ? static_cast<size_t>(sms) : plan.units;
    if (grid > static_cast<size_t>(sms)) grid = sms;
    if (grid < 1) grid = 1;
    kern<<<static_cast<unsigned>(grid), THREADS, SMEM_BYTES, s>>>(a, hdr, ctrs, parts);
    return cudaGetLastError();
}

template <int NP, bool SLICED>
cudaError_t launch_np(const GvArgs& a, const GvPlan& plan, cudaStream_t s) {
    if (a.group == 0) return launch_one<NP, false, false, SLICED>(a, plan, s);   // scale dtype read at run time
    return a.alpha_f16 ? launch_one<NP, true, true, SLICED>(a, plan, s) : launch_one<NP, true, false, SLICED>(a, plan, s);
}

template <bool SLICED>
cudaError_t launch_order(const GvArgs& a, const GvPlan& plan, cudaStream_t s) {
    switch (a.n_paths) {
        case 1: return launch_np<1, SLICED>(a, plan, s);
        case 2: return launch_np<2, SLICED>(a, plan, s);
        case 3: return launch_np<3, SLICED>(a, plan, s);
        case 4: return launch_np<4, SLICED>(a, plan, s);
        case 5: return launch_np<5, SLICED>(a, plan, s);
        case 6: return launch_np<6, SLICED>(a, plan, s);
        case 7: return launch_np<7, SLICED>(a, plan, s);
        case 8: return launch_np<8, SLICED>(a, plan, s);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

int gemv_max_jobs() { return MAX_JOBS; }

int gemv_rows_per_cta(int n_paths, int group) {
    const int J = group && n_paths <= 4 ? 4 : 8;
    const int hr = J / n_paths > 0 ? J / n_paths : 1;
    return WARPS * 4 * hr;
}

static void count_job(int64_t M, int64_t K, int R, int chunk, int T, GvPlan& pl) {
    const int64_t nrb = (M + R - 1) / R;
    const int64_t S = (K + SLICE_COLS - 1) / SLICE_COLS;
    const int64_t nch = (S + chunk - 1) / chunk;
    pl.units += static_cast<size_t>(nrb * nch * T);
    if (nch > 1) {
        pl.counters += static_cast<size_t>(nrb * T);
        pl.partials += static_cast<size_t>(nch * T * M);
    }
}

GvPlan gemv_plan_single(int64_t M, int64_t K, int n_paths, int group, int T, int num_sms) {
    const int R = gemv_rows_per_cta(n_paths, group);
    const int64_t S = (K + SLICE_COLS - 1) / SLICE_COLS;
    const int64_t nrb = (M + R - 1) / R;
    // split K until there are at least two units per SM (or one slice per unit)
    int64_t nch = 1;
    while (nch < S && nrb * nch * T < 2 * num_sms) ++nch;
    const int chunk = static_cast<int>((S + nch - 1) / nch);
    GvPlan pl{R, chunk, 0, 0, 0};
    count_job(M, K, R, chunk, T, pl);
    return pl;
}

GvPlan gemv_plan_grouped(const GvJob* jobs, int n, int n_paths, int group, int T) {
    const int R = gemv_rows_per_cta(n_paths, group);
    const int chunk = 8;   // 4096 columns: wider matrices are split so units stay small
    GvPlan pl{R, chunk, 0, 0, 0};
    for (int i = 0; i < n; ++i) count_job(jobs[i].M, jobs[i].K, R, chunk, T, pl);
    return pl;
}

cudaError_t launch_gemv(const GvArgs& a, const GvPlan& plan, cudaStream_t s) {
    return a.sliced ? launch_order<true>(a, plan, s) : launch_order<false>(a, plan, s);
}

}  // namespace rb
