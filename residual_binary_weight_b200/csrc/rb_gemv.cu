// rb_gemv: y_t = sum_k alpha_k (.) (B_k x_t) on CUDA cores, all paths in one pass.
//
// RaBiT (arXiv 2602.05367) section 4.1 and appendix D evaluate the layer
// without multiplications, with additions and subtractions over bit-packed
// planes. Here every 8-column block c of x is expanded once per CTA into a
// shared-memory table of its 256 signed sums
//     T[b][c] = sum_e (bit e of b ? +x[8c+e] : -x[8c+e])
// (2 * masked sum - block sum, built from two 16-entry nibble tables), so a
// plane byte b costs one PRMT (which forms the table address from the byte
// and a per-lane base), one LDS and half of a packed fp32x2 add: about 2.5
// instructions per 8 weight bits instead of >= 1 per bit for a select-and-add.
//
// Table layout: 256 rows of 64 fp32 entries (one 512-column slice of x),
// 64 KB, at shared-window address 0x10000 (a second one, for double
// buffering, at 0x20000). With the table 64 KB aligned the address of entry
// (b, c) is 0x10000 | b << 8 | 4c: PRMT takes byte 1 from the plane word,
// byte 0 (4c) from byte 0 or 1 of a base register that holds the columns of
// two lookup steps, and bytes 2-3 (the table page) from the same register.
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
// Scheduling. Units (row block, K chunk, token) are dealt to CTAs round robin
// and decoded once into shared memory, so each CTA knows its whole sequence
// of (unit, slice) steps: the last step of a unit already loads the next
// unit's first plane words, builds its first table and stages its x, and the
// unit's epilogue overlaps those loads.
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

// One work unit of a CTA, decoded once into shared memory: (job, row block,
// K chunk, token), with the token fastest, so CTAs that run together share
// plane rows in L2.
struct __align__(16) UnitRec {
    const uint32_t* planes;
    const void* alpha;
    const __half* x;        // the unit's token row of x
    void* y;                // the unit's token row of y
    int64_t M, K;
    uint32_t rb, j, t, ch, nch, s_begin, s_end, pad;
};

constexpr int UCAP = 128;   // unit records held at a time (a ring)

// Low shared region (below 0x10000): totals, job prefix sums, unit records,
// staged x.
struct __align__(16) LowSmem {
    float tot[WARPS][32];
    uint32_t unit_prefix[MAX_JOBS + 1];
    uint32_t ctr_prefix[MAX_JOBS + 1];
    uint32_t part_prefix[MAX_JOBS + 1];
    uint32_t wsum[3][WARPS];
    uint4 xstage[2][64];      // x of the next slices, staged by cp.async
    UnitRec units[UCAP];      // this CTA's units k at k % UCAP
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

// Packed fp32 pairs (sm_100 add/fma .f32x2): one instruction adds two
// independent sums.
__device__ __forceinline__ uint64_t pack_f2(float lo, float hi) {
    uint64_t d;
    asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(lo), "f"(hi));
    return d;
}

__device__ __forceinline__ void unpack_f2(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

__device__ __forceinline__ uint64_t add_f2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

__device__ __forceinline__ uint64_t fma_f2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

__device__ __forceinline__ uint2 ldg_words2(const void* p) {
    uint2 v;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
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
    // item loads per lane per slice (>= NP); 8 for every layout (with group
    // scales 4 loads per lane halved the rows per table and was ~20 % slower)
    static constexpr int J = 8;
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

// silu(g) * u = g u / (1 + e^-g) in fp32 (expf; for g -> -inf the quotient
// tends to -0)
__device__ __forceinline__ float silu_mul(float g, float u) { return g / (1.0f + expf(-g)) * u; }

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

__device__ __forceinline__ void decode_rec(const GvArgs& p, const uint32_t* unit_prefix, int n_jobs, uint32_t u,
                                           UnitRec& r) {
    int jlo = 0, jhi = n_jobs - 1;
    while (jlo < jhi) {
        const int mid = (jlo + jhi + 1) >> 1;
        if (unit_prefix[mid] <= u) jlo = mid; else jhi = mid - 1;
    }
    const GvJob jb = p.jobs ? p.jobs[jlo] : p.one;
    const int64_t ldx = p.jobs ? jb.K : p.ldx;
    const int64_t ldy = p.jobs ? jb.M : p.ldy;
    const int S = slices_of(jb.K);
    const uint32_t nch = static_cast<uint32_t>((S + p.chunk_slices - 1) / p.chunk_slices);
    uint32_t q = u - unit_prefix[jlo];
    const uint32_t t = q % static_cast<uint32_t>(p.T);
    q /= static_cast<uint32_t>(p.T);
    const uint32_t ch = q % nch;
    r.planes = jb.planes;
    r.alpha = jb.alpha;
    r.x = static_cast<const __half*>(jb.x) + t * ldx;
    r.y = static_cast<char*>(jb.y) + t * ldy * (p.y_f16 ? 2 : 4);
    r.M = jb.M;
    r.K = jb.K;
    r.rb = q / nch;
    r.j = static_cast<uint32_t>(jlo);
    r.t = t;
    r.ch = ch;
    r.nch = nch;
    // the S slices split into nch chunks of equal size (+-1)
    r.s_begin = (ch * static_cast<uint32_t>(S)) / nch;
    r.s_end = ((ch + 1) * static_cast<uint32_t>(S)) / nch;
    r.pad = 0;
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
                cq[e] = static_cast<uint32_t>(nch * T * (p.swiglu ? 2 : 1)) * static_cast<uint32_t>(jM);
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

// A single matrix (descriptor in the kernel parameters, sliced planes):
// bring the first two slices of this CTA's first unit into L2 with bulk
// prefetches, so that their HBM reads overlap the end of the previous kernel
// in the stream. A prefetch to L2 only moves lines into the point of
// coherence and hands no data to the thread, so it may run before the
// dependent-launch wait even if an earlier kernel still writes the planes.
// The unit follows the numbering of decode_rec: (row block, chunk, token),
// token fastest; units of token t > 0 read the planes of token 0's unit and
// skip it.
template <int R, int NP>
__device__ __forceinline__ void prefetch_first_unit(const GvArgs& p) {
    const int64_t M = p.one.M, K = p.one.K;
    const uint32_t S = static_cast<uint32_t>(slices_of(K));
    const uint32_t nch = (S + static_cast<uint32_t>(p.chunk_slices) - 1) / static_cast<uint32_t>(p.chunk_slices);
    const uint64_t nrb = static_cast<uint64_t>((M + R - 1) / R);
    const uint64_t u = blockIdx.x, T = static_cast<uint64_t>(p.T);
    if (u >= nrb * nch * T || u % T != 0) return;
    const uint64_t q = u / T;
    const uint32_t ch = static_cast<uint32_t>(q % nch);
    const uint64_t rb = q / nch;
    const uint32_t s_begin = (ch * S) / nch, s_end = ((ch + 1) * S) / nch;
    const uint32_t ns = min(2u, s_end - s_begin);
    const uint64_t row0 = rb * R;
    const uint32_t bytes = static_cast<uint32_t>(min(static_cast<uint64_t>(R), static_cast<uint64_t>(M) - row0)) * 64u;
    const uint32_t i = threadIdx.x;
    if (i < NP * ns) {
        // sliced layout: path k, slice s, row m at ((k S + s) M + m) * 64 bytes
        const uint64_t k = i / ns, s = s_begin + i % ns;
        const char* a = reinterpret_cast<const char*>(p.one.planes) + ((k * S + s) * static_cast<uint64_t>(M) + row0) * 64u;
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(a), "r"(bytes) : "memory");
    }
}

// GATE: the SiLU-gated pair (GvArgs::swiglu), a separate instantiation so
// that the plain kernel's epilogue carries none of it
template <int NP, bool G128, bool A16, bool SLICED, bool GATE = false>
__global__ void __launch_bounds__(THREADS, 1) gemv_lut_kernel(GvArgs p, uint32_t* __restrict__ hdr,
                                                              uint32_t* __restrict__ ctrs,
                                                              float* __restrict__ parts) {
    using C = Cfg<NP, G128>;
    constexpr int J = C::J, HR = C::HR;
    extern __shared__ __align__(16) unsigned char dsm[];
    LowSmem& lo = *reinterpret_cast<LowSmem*>(dsm);

    // Programmatic dependent launch: the next kernel of the stream may be
    // launched now (its CTAs start as this grid's CTAs leave their SMs and
    // wait in join() until this grid has finished). join() waits for the
    // kernel before this one. Everything before it reads only the kernel
    // parameters and shared memory: the grouped descriptors are device
    // memory, so a grouped call joins first; a single matrix scans its plan,
    // decodes its first units and prefetches its first planes to L2 (a
    // prefetch hands no data to the CTA) while the previous kernel ends.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const bool single = p.jobs == nullptr;
    if (SLICED && single) prefetch_first_unit<C::R, NP>(p);
    // The call's error word is cleared in join(), not by a memset before
    // the launch: every condition below is detected by every CTA, CTA 0
    // included, after CTA 0's join, so a flag another CTA raised before the
    // clear is raised again. Every global access and every return follows a
    // join() (a second griddepcontrol.wait returns at once).
    bool joined = false;
    auto join = [&]() {
        if (joined) return;
        asm volatile("griddepcontrol.wait;" ::: "memory");
        if (blockIdx.x == 0 && threadIdx.x == 0) hdr[1] = 0u;
        joined = true;
    };
    if (!single) join();
    const uint32_t s0 = smem_addr(dsm);
    if (s0 + sizeof(LowSmem) > TBL0 || s0 + SMEM_BYTES < TBL0 + 2 * 0x10000u) {
        join();
        if (threadIdx.x == 0) atomicOr(hdr + 1, GV_ERR_SMEM_LAYOUT);
        return;
    }
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // lane -> item q4 of each 4-item load, word pair t (words 2t, 2t + 1)
    const int q4 = lane >> 3, t8 = lane & 7;
    const int T = p.T;
    const int n_jobs = p.jobs ? p.n_jobs : 1;
    if (n_jobs > MAX_JOBS) {
        join();
        if (tid == 0) atomicOr(hdr + 1, GV_ERR_TOO_MANY_JOBS);
        return;
    }
    scan_jobs<C::R>(p, lo, n_jobs);
    const uint32_t total_units = lo.unit_prefix[n_jobs];
    // the device descriptors must give the plan the host sized the workspace
    // for (they are a copy the caller uploaded; a stale copy would write
    // counters and partial sums past the workspace)
    if (total_units != p.expect_units || lo.ctr_prefix[n_jobs] != p.expect_ctrs ||
        lo.part_prefix[n_jobs] != p.expect_parts) {
        join();
        if (tid == 0) atomicOr(hdr + 1, GV_ERR_BAD_JOB);
        return;   // uniform: every thread read the same shared values
    }

    // The 8 lanes sharing t8 & 3 (t8 in {a, a + 4}, 4 items) would hit the
    // same banks; lane z = (t8 >> 2) + 2 q4 swaps its two words when z is odd
    // (rv) and rotates the byte order by rq = z >> 1, so every LDS touches 32
    // distinct banks. One PRMT per word does both: word v' of the lane is
    // (rv ? word 1 - v : word v) with byte q taken from byte (q + rq) & 3.
    const uint32_t zr = static_cast<uint32_t>((t8 >> 2) + 2 * q4);
    const uint32_t rv = zr & 1u, rq = zr >> 1;
    uint32_t perm0 = 0, perm1 = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const uint32_t byte = (static_cast<uint32_t>(q) + rq) & 3u;
        perm0 |= (byte + 4u * rv) << (4 * q);
        perm1 |= (byte + 4u * (rv ^ 1u)) << (4 * q);
    }

    // ---- this CTA's units: u = blockIdx.x + k * gridDim.x, k < n_my, decoded
    // into the ring of unit records ahead of use
    const uint32_t G = gridDim.x, bid = blockIdx.x;
    const uint32_t n_my = total_units > bid ? (total_units - bid + G - 1) / G : 0u;
    if (n_my == 0) {   // uniform over the CTA
        join();
        return;
    }
    uint32_t decoded = 0;
    auto decode_upto = [&](uint32_t to) {
        for (uint32_t k = decoded + tid; k < to; k += THREADS)
            decode_rec(p, lo.unit_prefix, n_jobs, bid + k * G, lo.units[k % UCAP]);
        decoded = to;
        cta_sync();
    };
    decode_upto(min(n_my, static_cast<uint32_t>(UCAP)));
    join();

    // The step `d` steps after (unit k, slice s) in this CTA's sequence of
    // (unit, slice) steps; false past the last unit. Needs units up to k + d
    // decoded (every unit has at least one slice).
    auto step_after = [&](uint32_t k, int s, int d, uint32_t& ko, int& so) -> bool {
        while (true) {
            const UnitRec& r = lo.units[k % UCAP];
            if (s + d < static_cast<int>(r.s_end)) {
                ko = k;
                so = s + d;
                return true;
            }
            d -= static_cast<int>(r.s_end) - s;
            if (++k >= n_my) return false;
            s = static_cast<int>(lo.units[k % UCAP].s_begin);
        }
    };
    // threads 0..63 stage the x of step (k, s) + d into `dst`
    auto stage_step = [&](uint32_t k, int s, int d, uint4* dst) {
        if (tid < 64) {
            uint32_t ko;
            int so;
            if (step_after(k, s, d, ko, so)) {
                const UnitRec& r = lo.units[ko % UCAP];
                stage_x(r.x, r.K, so, dst);
            }
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };

    // items 2i and 2i + 1 accumulate as one fp32 pair (add.f32x2)
    uint64_t acc2[J / 2];
    uint2 wv[J];
    float av[J];
#pragma unroll
    for (int j = 0; j < J; ++j) av[j] = 0.0f;
    // Table address of lookup step i = 4 v + q (byte q of permuted word
    // v): TBL | b << 8 | 4c with c = 8 t8 + 4 (v ^ rv) + (q + rq) & 3.
    // Register pb[i / 2] holds 4c of steps i and i + 1 in bytes 0 and 1,
    // the table's 64 KB page in byte 2 and 0 in byte 3; the address PRMT
    // takes byte 0 or 1 of it, the plane byte, then bytes 2 and 3.
    uint32_t pb[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        uint32_t r = TBL0;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const uint32_t v = static_cast<uint32_t>((2 * k + h) >> 2), q = static_cast<uint32_t>((2 * k + h) & 3);
            r |= (4u * (8u * t8 + 4u * (v ^ rv) + ((q + rq) & 3u))) << (8 * h);
        }
        pb[k] = r;
    }
    uint32_t tbl_next = TBL0 + 0x10000u;   // buffer of the next step's table

    // Where item loads of one slice of one unit come from. Item load j: path
    // j / HR, rows r0 + 4 (j % HR) + q4. In a full warp its lane pointer is
    // the path pointer + (j % HR) * (4 rows), an immediate offset in the
    // sliced layout; other warps clamp rows to M - 1 (absolute addresses).
    struct SliceAddr {
        const char* slice0;   // (path 0, row 0, pair tsel) of the slice
        const char* lane0;    // (path 0, row r0 + q4, pair tsel)
        const void* alpha;
        uint32_t r0, tp, uM, path_bytes, row_bytes, aoff, gpr;
    };
    auto make_addr = [&](const uint32_t* planes, const void* alpha, uint32_t uM, int64_t K, uint32_t rb, int s) {
        SliceAddr a;
        // word pair of lane t8, clamped in a partial last slice (the table
        // entries past K are 0, so a clamped pair adds nothing); the sliced
        // layout pads the last slice, so only the scale index and the row
        // layout need it
        const int ws = min(16, static_cast<int>((K - static_cast<int64_t>(s) * SLICE_COLS) >> 5));
        a.tp = 2 * t8 < ws ? static_cast<uint32_t>(t8) : 0u;
        a.r0 = rb * C::R + warp * C::RW;
        asm volatile("" : "+r"(a.r0));
        a.uM = uM;
        const uint32_t S = static_cast<uint32_t>(slices_of(K));
        const uint32_t uW32 = static_cast<uint32_t>(K >> 5);
        a.path_bytes = SLICED ? S * 64u * uM : uM * uW32 * 4u;
        a.row_bytes = SLICED ? 64u : uW32 * 4u;
        a.alpha = alpha;
        a.gpr = static_cast<uint32_t>(K >> 7);
        a.aoff = 4u * static_cast<uint32_t>(s) + (a.tp >> 1);
        const uint32_t tsel = SLICED ? static_cast<uint32_t>(t8) : a.tp;
        a.slice0 = reinterpret_cast<const char*>(planes) +
                   (SLICED ? (static_cast<size_t>(s) * uM * 16u + 2u * tsel) * 4u
                           : (16u * static_cast<uint32_t>(s) + 2u * tsel) * 4u);
        a.lane0 = mad_ptr(a.r0 + q4, a.row_bytes, a.slice0);
        return a;
    };
    auto fetch = [&](int j, const SliceAddr& a, auto full_tag) {
        constexpr bool F = decltype(full_tag)::value;
        const uint32_t path = j / HR, rr = j % HR;
        uint32_t row;
        const char* wp;
        if (F) {
            row = a.r0 + q4 + 4u * rr;
            const char* pp = path ? mad_ptr(path, a.path_bytes, a.lane0) : a.lane0;
            wp = SLICED ? pp + rr * 256u : mad_ptr(4u * rr, a.row_bytes, pp);
        } else {
            row = min(a.r0 + q4 + 4u * rr, a.uM - 1u);
            wp = mad_ptr(row, a.row_bytes, path ? mad_ptr(path, a.path_bytes, a.slice0) : a.slice0);
        }
        // K is a multiple of 128, so rows of either layout are a multiple
        // of 16 bytes, the planes are 16-byte aligned and a slice holds an
        // even number of words: the pair is one aligned 8-byte load
        wv[j] = ldg_words2(wp);
        if (G128) {
            const size_t ai = static_cast<size_t>(path * a.uM + row) * a.gpr + a.aoff;
            av[j] = A16 ? __half2float(static_cast<const __half*>(a.alpha)[ai]) : static_cast<const float*>(a.alpha)[ai];
        }
    };
    auto fetch_all = [&](const SliceAddr& a, auto full_tag) {
#pragma unroll
        for (int j = 0; j < J; ++j)
            if (j < C::JV) fetch(j, a, full_tag);
    };
    // consume the current slice from the current table; with PF, items of
    // the next step (at `an`) are loaded right after the same items of this
    // slice were used, so each load has about one slice of time to arrive
    auto consume = [&](const SliceAddr& an, auto pf_tag, auto full_tag) {
        constexpr bool PF = decltype(pf_tag)::value;
#pragma unroll
        for (int i = 0; i < J / 2; ++i) {
            const int j0 = 2 * i, j1 = 2 * i + 1;
            if (j0 >= C::JV) continue;
            const bool has1 = j1 < C::JV;
            // the word permutation happens here, where the words are
            // used, not where they are loaded (a use right after the load
            // would wait for it)
            const uint32_t a0 = prmt(wv[j0].x, wv[j0].y, perm0), a1 = prmt(wv[j0].x, wv[j0].y, perm1);
            uint32_t b0 = 0, b1 = 0;
            if (has1) {
                b0 = prmt(wv[j1].x, wv[j1].y, perm0);
                b1 = prmt(wv[j1].x, wv[j1].y, perm1);
            }
            uint64_t pr[8];
#pragma unroll
            for (int st = 0; st < 8; ++st) {
                const uint32_t q = st & 3;
                const uint32_t sel = 0x7600u | (q << 4) | (4u + (st & 1));
                const float e0 = lds(prmt(st < 4 ? a0 : a1, pb[st >> 1], sel));
                const float e1 = has1 ? lds(prmt(st < 4 ? b0 : b1, pb[st >> 1], sel)) : 0.0f;
                pr[st] = pack_f2(e0, e1);
            }
            const uint64_t ps = add_f2(add_f2(add_f2(pr[0], pr[1]), add_f2(pr[2], pr[3])),
                                       add_f2(add_f2(pr[4], pr[5]), add_f2(pr[6], pr[7])));
            if (G128) acc2[i] = fma_f2(pack_f2(av[j0], av[j1]), ps, acc2[i]);
            else acc2[i] = add_f2(acc2[i], ps);
            if (PF) {
                fetch(j0, an, full_tag);
                if (has1) fetch(j1, an, full_tag);
            }
        }
    };

    // ---- prologue: words, x and table of the first step, x of the second
    uint32_t g = 0;   // global step counter: x of step g in xstage[g & 1]
    {
        const UnitRec& r = lo.units[0];
        fetch_all(make_addr(r.planes, r.alpha, static_cast<uint32_t>(r.M), r.K, r.rb, static_cast<int>(r.s_begin)),
                  BoolC<false>{});
        stage_step(0, static_cast<int>(r.s_begin), 0, lo.xstage[0]);
        stage_step(0, static_cast<int>(r.s_begin), 1, lo.xstage[1]);
        stage_wait_all();
        cta_sync();
        build_table(lo.xstage[0], TBL0);
        cta_sync();
    }

    for (uint32_t k = 0; k < n_my; ++k) {
        if (decoded < n_my && decoded < k + 3) decode_upto(min(n_my, decoded + UCAP / 2));
        const UnitRec& ur = lo.units[k % UCAP];
        const uint32_t* planes = ur.planes;
        const void* alpha = ur.alpha;
        const uint32_t uM = static_cast<uint32_t>(ur.M);
        const int64_t K = ur.K;
        const uint32_t rb = ur.rb;
        const int s_begin = static_cast<int>(ur.s_begin), s_end = static_cast<int>(ur.s_end);
        const bool has_next = k + 1 < n_my;
        const uint32_t row0 = rb * C::R + warp * C::RW;
        // a full warp has every row of its items below M
        const bool full = row0 + C::RW <= uM;
#pragma unroll
        for (int i = 0; i < J / 2; ++i) acc2[i] = 0ull;
        // the per-row scales of this warp's rows, read in the epilogue, are
        // brought into L1 now
        if (!G128 && lane < 2 * NP) {
            const uint32_t row = min(row0 + (lane & 1) * (C::RW - 1), uM - 1u);
            const size_t ai = static_cast<size_t>(lane >> 1) * uM + row;
            const char* ap = static_cast<const char*>(alpha) + ai * (p.alpha_f16 ? 2 : 4);
            asm volatile("prefetch.global.L1 [%0];" ::"l"(ap));
        }

        // one step: build the next step's table, stage x two steps ahead,
        // consume this slice (loading the next step's words), one barrier
        auto step = [&](int s, bool build_next, const SliceAddr& an, auto pf_tag, auto full_tag) {
            if (build_next) build_table(lo.xstage[(g + 1) & 1], tbl_next);
            stage_step(k, s, 2, lo.xstage[g & 1]);
            consume(an, pf_tag, full_tag);
#pragma unroll
            for (int q = 0; q < 4; ++q) pb[q] ^= TBL_TOGGLE;
            tbl_next ^= TBL_TOGGLE;
            ++g;
            stage_wait_all();
            cta_sync_any();
        };
        // Full and partial warps run separate copies of the unit's steps
        // (non-aligned barriers); the last step is peeled: it loads the next
        // unit's first words (rows clamped, whatever that unit's shape)
        auto run_unit = [&](auto full_tag) {
            for (int s = s_begin; s < s_end - 1; ++s)
                step(s, true, make_addr(planes, alpha, uM, K, rb, s + 1), BoolC<true>{}, full_tag);
            if (has_next) {
                const UnitRec& rn = lo.units[(k + 1) % UCAP];
                step(s_end - 1, true,
                     make_addr(rn.planes, rn.alpha, static_cast<uint32_t>(rn.M), rn.K, rn.rb,
                               static_cast<int>(rn.s_begin)),
                     BoolC<true>{}, BoolC<false>{});
            } else {
                SliceAddr none{};
                step(s_end - 1, false, none, BoolC<false>{}, full_tag);
            }
        };
        if (full) run_unit(BoolC<true>{});
        else run_unit(BoolC<false>{});

        // ---- reduce over the 8 lanes of each item; lane t8 owns load j = t8 >> shift
        float acc[J];
#pragma unroll
        for (int i = 0; i < J / 2; ++i) unpack_f2(acc2[i], acc[2 * i], acc[2 * i + 1]);
        group8_transpose_reduce<J>(acc, t8);
        constexpr int shift = 3 - Log2<J>::v;
        if ((t8 & ((1 << shift) - 1)) == 0) lo.tot[warp][4 * (t8 >> shift) + q4] = acc[0];
        __syncwarp();

        // ---- per-row output of this chunk: lane r < RW owns row r of the warp,
        // whose path-k item is load k * HR + r / 4 of item group r % 4
        const UnitRec& ue = lo.units[k % UCAP];
        const int64_t M = ue.M;
        // yv: sum over the paths (with the SiLU gate: over the gate's paths,
        // yv2 over the up projection's)
        float yv = 0.0f, yv2 = 0.0f;
        constexpr bool gated = GATE;
        const int64_t my_row = static_cast<int64_t>(ue.rb) * C::R + warp * C::RW + lane;
        const bool row_ok = lane < C::RW && my_row < M;
        if (row_ok) {
#pragma unroll
            for (int kk = 0; kk < NP; ++kk) {
                const float tk = lo.tot[warp][4 * (kk * HR + (lane >> 2)) + (lane & 3)];
                float& dst = (gated && kk >= NP / 2) ? yv2 : yv;
                if (G128) {
                    dst += tk;
                } else {
                    const size_t ai = static_cast<size_t>(kk) * M + my_row;
                    const float a = p.alpha_f16 ? __half2float(static_cast<const __half*>(ue.alpha)[ai])
                                                : static_cast<const float*>(ue.alpha)[ai];
                    dst = fmaf(a, tk, dst);
                }
            }
        }
        auto store_y = [&](int64_t row, float v, float v2) {
            if (gated) v = silu_mul(v, v2);
            if (p.y_f16) static_cast<__half*>(ue.y)[row] = __float2half_rn(v);
            else static_cast<float*>(ue.y)[row] = v;
        };
        const uint32_t nch = ue.nch;
        if (nch == 1) {
            if (row_ok) store_y(my_row, yv, yv2);
        } else {
            // partial sums [t][chunk][1 or 2][M]
            const uint32_t W = gated ? 2u : 1u;
            float* part = parts + lo.part_prefix[ue.j] + (static_cast<size_t>(ue.t) * nch * W) * M;
            if (row_ok) {
                part[static_cast<size_t>(ue.ch * W) * M + my_row] = yv;
                if (gated) part[static_cast<size_t>(ue.ch * W + 1) * M + my_row] = yv2;
            }
            __threadfence();
            cta_sync();
            if (tid == 0) {
                uint32_t* ctr = ctrs + lo.ctr_prefix[ue.j] + ue.rb * T + ue.t;
                const uint32_t prev = atomicAdd(ctr, 1u);
                lo.last = (prev == nch - 1) ? 1u : 0u;
                // the last arrival puts the counter back to zero, so the
                // workspace needs no clearing between calls
                if (prev == nch - 1) *ctr = 0u;
                if (prev >= nch) atomicOr(hdr + 1, GV_ERR_COUNTER);
            }
            cta_sync();
            if (lo.last) {
                __threadfence();
                const int64_t rbase = static_cast<int64_t>(ue.rb) * C::R;
                for (int i = tid; i < C::R; i += THREADS) {
                    const int64_t row = rbase + i;
                    if (row < M) {
                        float sum = 0.0f, sum2 = 0.0f;
                        for (uint32_t c = 0; c < nch; ++c) {
                            sum += __ldcg(part + static_cast<size_t>(c * W) * M + row);
                            if (gated) sum2 += __ldcg(part + static_cast<size_t>(c * W + 1) * M + row);
                        }
                        store_y(row, sum, sum2);
                    }
                }
            }
        }
        cta_sync();
    }
}

template <int NP, bool G128, bool A16, bool SLICED, bool GATE = false>
cudaError_t launch_one(const GvArgs& a, const GvPlan& plan, cudaStream_t s) {
    auto kern = gemv_lut_kernel<NP, G128, A16, SLICED, GATE>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    uint32_t* hdr = static_cast<uint32_t*>(a.workspace);
    uint32_t* ctrs = reinterpret_cast<uint32_t*>(static_cast<char*>(a.workspace) + GV_HEADER_BYTES);
    float* parts = reinterpret_cast<float*>(ctrs + GV_MAX_COUNTERS);
    const int sms = device_sm_count();
    size_t grid = plan.units;
    if (grid > static_cast<size_t>(sms)) grid = sms;
    if (grid < 1) grid = 1;
    // launched as a programmatic dependent of the stream's previous kernel
    // (the kernel waits for it with griddepcontrol.wait before any global
    // access), so the launch overlaps that kernel's tail
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, a, hdr, ctrs, parts);
}

template <int NP, bool SLICED>
cudaError_t launch_np(const GvArgs& a, const GvPlan& plan, cudaStream_t s) {
    if (a.swiglu) {
        if constexpr (NP % 2 == 0) {
            if (a.group == 0) return launch_one<NP, false, false, SLICED, true>(a, plan, s);
            return a.alpha_f16 ? launch_one<NP, true, true, SLICED, true>(a, plan, s)
                               : launch_one<NP, true, false, SLICED, true>(a, plan, s);
        } else {
            return cudaErrorInvalidValue;   // a gated pair has an even number of paths
        }
    }
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

int gemv_rows_per_cta(int n_paths, int /*group*/) {
    const int J = 8;   // Cfg::J
    const int hr = J / n_paths > 0 ? J / n_paths : 1;
    return WARPS * 4 * hr;
}

static void count_job(int64_t M, int64_t K, int R, int chunk, int T, GvPlan& pl, int sums_per_row = 1) {
    const int64_t nrb = (M + R - 1) / R;
    const int64_t S = (K + SLICE_COLS - 1) / SLICE_COLS;
    const int64_t nch = (S + chunk - 1) / chunk;
    pl.units += static_cast<size_t>(nrb * nch * T);
    if (nch > 1) {
        pl.counters += static_cast<size_t>(nrb * T);
        pl.partials += static_cast<size_t>(nch * T * M * sums_per_row);
    }
}

GvPlan gemv_plan_single(int64_t M, int64_t K, int n_paths, int group, int T, int num_sms, bool swiglu) {
    const int R = gemv_rows_per_cta(n_paths, group);
    const int64_t S = (K + SLICE_COLS - 1) / SLICE_COLS;
    const int64_t nrb = (M + R - 1) / R;
    // Choose the number of K chunks that minimises the busiest CTA's work:
    // (units it gets) x (slices per unit + about half a slice for the
    // partial-sum epilogue of a split unit); ties go to fewer chunks.
    const int64_t sms = num_sms > 0 ? num_sms : 1;
    int64_t best_nch = 1;
    double best = -1.0;
    // a split needs nrb * T arrival counters, at most GV_MAX_COUNTERS
    const int64_t max_nch = nrb * T <= static_cast<int64_t>(GV_MAX_COUNTERS) ? S : 1;
    for (int64_t nch = 1; nch <= max_nch; ++nch) {
        const int64_t units = nrb * nch * T;
        const int64_t per_cta = (units + sms - 1) / sms;
        const int64_t slices = (S + nch - 1) / nch;
        const double cost = static_cast<double>(per_cta) * (static_cast<double>(slices) + (nch > 1 ? 0.5 : 0.0));
        if (best < 0.0 || cost < best) {
            best = cost;
            best_nch = nch;
        }
    }
    const int chunk = static_cast<int>((S + best_nch - 1) / best_nch);
    GvPlan pl{R, chunk, 0, 0, 0};
    count_job(M, K, R, chunk, T, pl, swiglu ? 2 : 1);
    return pl;
}

GvPlan gemv_plan_grouped(const GvJob* jobs, int n, int n_paths, int group, int T) {
    const int R = gemv_rows_per_cta(n_paths, group);
    // up to 12 slices (6144 columns) per unit: wider matrices are split in
    // equal parts. Each split adds a partial-sum epilogue (fp32 partials, an
    // arrival counter, the last CTA's reduction), which costs more than the
    // load imbalance of longer units (7B stack: 8 -> 408 us, 12 -> 402 us;
    // 4 or 6, which split the 4096-wide matrices too: 519 and 506 us)
    GvPlan pl{R, 12, 0, 0, 0};
    for (int i = 0; i < n; ++i) count_job(jobs[i].M, jobs[i].K, R, pl.chunk_slices, T, pl);
    if (pl.counters > GV_MAX_COUNTERS) {   // more splits than the counter zone holds: split nothing
        pl = GvPlan{R, 1 << 20, 0, 0, 0};
        for (int i = 0; i < n; ++i) count_job(jobs[i].M, jobs[i].K, R, pl.chunk_slices, T, pl);
    }
    return pl;
}

cudaError_t launch_gemv(const GvArgs& a, const GvPlan& plan, cudaStream_t s) {
    return a.sliced ? launch_order<true>(a, plan, s) : launch_order<false>(a, plan, s);
}

}  // namespace rb
