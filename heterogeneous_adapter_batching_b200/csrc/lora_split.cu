// Split gather path for short segments: a shrink kernel and an expand kernel.
//
// Page "Multi-LoRA Serving in Production" (llms.blog), section "Segmented
// Gather Matrix-Vector Multiplication (SGMV)": the shrink v = x A and the
// scaled expand y += (alpha/r) v B are two steps over tokens grouped by
// adapter; section "Multi-Size Batched Gather Kernels (MBGMV and MBGMM)": the
// decode kernels gather each token's adapter pages without padding to the
// largest rank.  Page "Multi-LoRA Serving Architecture ... (2026)", section
// "Heterogeneous batching: the core compute trick": the branch is
// memory-bound, its cost the adapter bytes read.
//
// The two steps run as two persistent kernels so that every SM streams
// adapter pages back to back, with no exchange inside a unit of work:
//
//   shrink_part_kernel   units = (gather job, quarter s of d_in).  A producer
//                        warp streams the quarter's A^T pages (TMA boxes of 16
//                        rank rows x 4 x 64 columns, 128-byte swizzle) and the
//                        job's X rows (bulk copies) into a ring of stages; 15
//                        consumer warps run warp-level bf16 MMAs and write the
//                        quarter's fp32 partial v into the workspace.
//   expand_part_kernel   units = (gather job, part e of d_out).  Launched as a
//                        programmatic dependent of the shrink kernel: its
//                        producer streams the part's B pages and the old Y rows
//                        before it waits for the shrink grid, then fetches the
//                        four partials; consumers add them, split v into a
//                        bf16 high and low part, run the expand MMAs, update Y
//                        in shared memory and write the rows back.
//
// The arithmetic is that of the cluster gather kernel, step for step: the d_in
// quarters are the same, within a quarter warp w owns the 16-column steps
// congruent to w mod 15 in increasing order, the warps' partials are added in
// warp order and the quarters in quarter order, and the expand takes pages in
// order with the high part before the low part.  The two paths therefore give
// bit-identical Y, and the library picks between them for speed alone.
//
// Consumers learn their work only from a per-stage header the producer writes
// before arming the stage, so they never wait on global memory.  Every wait,
// including the consumers' own synchronisation, is an mbarrier wait with a
// bound (about a second); a wait that runs out sets LORA_DEV_ERR_TIMEOUT, the
// CTA's abort flag makes every later wait return at once, and each role
// leaves its loop; the producer then waits (bounded) for its own copies in
// flight before it exits.  No kernel traps.  No cluster multicast is used.
#include "lora_internal.cuh"
#include "lora_ptx.cuh"

namespace lora {
namespace {

using namespace ptx;

constexpr int kSlices = 4;                      // d_in quarters (the cluster gather kernel's CTAs per cluster)
constexpr int kCW = 15;                         // consumer warps
constexpr int kConsumers = kCW * 32;
constexpr int kThreads = kConsumers + 32;       // + one producer warp
constexpr int kNTok = 8;                        // tokens per MMA (the N side)
constexpr int kMaxNT = LORA_MAX_JOB_TOKENS / kNTok;
constexpr int kMaxPages = LORA_MAX_RANK / LORA_PAGE_ROWS;
constexpr int kSlots = 8;                                  // chunks in flight at most (barrier and header ring)
constexpr int kBoxCols = 64;
constexpr int kBoxBytes = LORA_PAGE_ROWS * kBoxCols * 2;   // 2 KB
constexpr int kRowRegion = 16640;                          // most bytes of X or Y rows in one chunk: 16 rows x 1040 B
constexpr int kMaxBoxes = 32;                              // page boxes in one chunk at most (64 KB)
constexpr int kMaxChunk = kMaxBoxes * kBoxBytes + kRowRegion;
constexpr int kTilesPerWarp = 3;                           // expand: m-tiles a warp runs at once
constexpr int kShrinkArena = 159 * 1024;                   // byte rings the chunks are packed into
constexpr int kExpandArena = 180 * 1024;
constexpr int kTableSlots = 128;                           // slot tables up to this size live in shared memory
constexpr long long kWaitLimit = 2000000000LL;             // cycles (~1 s)
constexpr int kVPartFloats = LORA_MAX_JOB_TOKENS * LORA_MAX_RANK;
constexpr int kVTileBytes = LORA_MAX_JOB_TOKENS * LORA_MAX_RANK * 2;   // one bf16 part of v

static_assert(kShrinkArena / 2 >= kMaxPages * kBoxBytes + LORA_MAX_JOB_TOKENS * (kBoxCols * 2 + 16) &&
                  kExpandArena >= 2 * kMaxChunk,
              "the rings hold at least two chunks");
static_assert(kMaxNT * kNTok == LORA_MAX_JOB_TOKENS, "job size must be a whole number of MMA tiles");

// What the producer tells the consumers about one chunk.
struct ChunkHdr {
    int unit;          // >= 0: a chunk of a unit; -1: no more work
    int off;           // byte offset of the chunk in the ring (1 KB aligned): page boxes, then rows
    int first, last;   // first / last chunk of its unit
    int c0, cols;      // first column, valid columns (a multiple of 8)
    int nb;            // 64-column boxes per page
    int np, r, n, nt;  // pages per matrix, rank, tokens, 8-token MMA tiles
    int lo, hi;        // the unit's column range (d_in quarter, or d_out part)
    int q0;            // shrink: position of the job's first token in the plan's token list
    int slice;         // shrink: quarter s; expand: v staging buffer
    float scale;       // expand: alpha / r
    int tok[LORA_MAX_JOB_TOKENS];   // expand: the job's token indices
};

struct __align__(1024) ShrinkSmem {
    unsigned char ring[kShrinkArena];
    float red[kCW * kMaxPages * kMaxNT * 128];   // the warps' partial sums of a unit
    ChunkHdr hdr[kSlots];
    int4 pt[kTableSlots * 2];
    int ranks[kTableSlots];
    int asz[kSlots];                             // producer: ring bytes each chunk in flight holds
    uint64_t full[kSlots], empty[kSlots];
    uint64_t red_full, red_free;
    int abort;
};

struct __align__(1024) ExpandSmem {
    unsigned char ring[kExpandArena];
    float vst[2][kSlices][kVPartFloats];          // the four partials of a unit, double-buffered
    unsigned char vt[2 * kVTileBytes];            // v: bf16 high part [t][k] (16-byte groups swizzled), then low part
    ChunkHdr hdr[kSlots];
    int4 pt[kTableSlots * 2];
    int ranks[kTableSlots];
    float scales[kTableSlots];
    int asz[kSlots];
    uint64_t full[kSlots], empty[kSlots];
    uint64_t vfull[2], vempty[2];
    uint64_t vt_full, vt_free;
    int abort;
};



static_assert(sizeof(ShrinkSmem) + 1024 <= 227 * 1024, "shrink kernel: shared memory beyond the per-block limit");
static_assert(sizeof(ExpandSmem) + 1024 <= 227 * 1024, "expand kernel: shared memory beyond the per-block limit");

struct KSplit {
    const uint16_t *X;
    float *Y;
    int T, d_in, d_out, S;
    const int32_t *ranks;
    const float *scales;
    const int32_t *pt;
    long long rowsA, rowsB;
    const int32_t *perm;     // the plan's short-token list (gather jobs index it)
    const int4 *jobs;
    const PlanHeader *hdr;
    float *vpart;            // [kSlices][T][LORA_MAX_RANK] fp32
    int32_t *err;
    int e_max;               // most d_out parts (each keeps >= 64 columns)
    bool wide_in, wide_out;  // the 3D page maps are valid (width >= 256)
};

// Bounded wait on an mbarrier phase; false when it ran out or the CTA aborted.
template <class Sm>
__device__ __forceinline__ bool wait_b(uint64_t *bar, uint32_t parity, Sm &sm, int32_t *err) {
    const uint32_t a = smem_u32(bar);
    if (mbar_try(a, parity)) return true;
    const long long t0 = clock64();
    while (!mbar_try(a, parity)) {
        if (*(volatile int *)&sm.abort) return false;
        if (clock64() - t0 > kWaitLimit) {
            *(volatile int *)&sm.abort = 1;
            if (err) atomicOr(err, LORA_DEV_ERR_TIMEOUT);
            return false;
        }
    }
    return true;
}

// The same, with one outcome for the whole warp.
template <class Sm>
__device__ __forceinline__ bool wait_w(uint64_t *bar, uint32_t parity, Sm &sm, int32_t *err) {
    const bool ok = wait_b(bar, parity, sm, err);
    return __all_sync(0xffffffffu, ok);
}

// Bounded wait for copies this thread issued, before the CTA exits; not cut
// short by the abort flag.
__device__ __forceinline__ void drain_wait(uint64_t *bar, uint32_t parity) {
    const uint32_t a = smem_u32(bar);
    const long long t0 = clock64();
    while (!mbar_try(a, parity) && clock64() - t0 < kWaitLimit / 8) {
    }
}

// The producer's side of a ring of chunks: chunk i uses barrier and header
// slot i mod kSlots and a 1 KB aligned byte range of the arena; ranges are
// handed out in order and come back in order (the consumers release chunks in
// the order they take them), so the producer waits for the oldest chunks'
// release until the next range and slot are free.
struct Ring {
    long long produced;   // bytes handed out (a chunk that would cross the end skips to the start)
    long long released;   // bytes returned
    int chunk;            // chunks handed out
    int popped;           // chunks whose release the producer has seen
};

// Free the oldest chunk: wait for its release (all consumer warps arrived).
template <class Sm>
__device__ __forceinline__ bool ring_pop(Ring &rg, Sm &sm, int32_t *err) {
    const int ps = rg.popped % kSlots;
    if (!wait_w(&sm.empty[ps], (uint32_t)((rg.popped / kSlots) & 1), sm, err)) return false;
    rg.released += sm.asz[ps];
    ++rg.popped;
    return true;
}

// Hand out `bytes` (rounded up to 1 KB) and the next slot; `before_block` runs
// once, before the first wait this call would make.  Returns the byte offset,
// or -1 when a wait failed.
template <int kArena, class Sm, class F>
__device__ __forceinline__ int ring_alloc(Ring &rg, Sm &sm, int bytes, int32_t *err, F &&before_block) {
    const int need = (bytes + 1023) & ~1023;
    const int at = (int)(rg.produced % kArena);
    const int pad = at + need > kArena ? kArena - at : 0;
    bool called = false;
    while (rg.produced + pad + need - rg.released > kArena || rg.chunk - rg.popped >= kSlots) {
        if (!called) {
            before_block();
            called = true;
        }
        if (rg.popped == rg.chunk || !ring_pop(rg, sm, err)) return -1;
    }
    if (threadIdx.x % 32 == 0) sm.asz[rg.chunk % kSlots] = pad + need;
    __syncwarp();
    rg.produced += pad + need;
    return pad ? 0 : at;
}

// One slot's rank, pages and scale, validated against both pools (a unit is
// skipped in both kernels when either matrix is out of range, so the expand
// never reads a partial that the shrink did not write).  The loads (RawMeta)
// are issued one unit ahead of their use, the checks (Meta) at the use.
struct RawMeta {
    int r;
    int4 pga, pgb;
    float scale;
};

struct Meta {
    int r, np;
    int4 pga, pgb;
    float scale;
    bool bad;
};

__device__ __forceinline__ RawMeta raw_meta(const KSplit &a, const int4 *spt, const int *srk, const float *ssc,
                                            bool staged, int slot) {
    RawMeta m;
    if (staged) {
        m.r = srk[slot];
        m.pga = spt[2 * slot];
        m.pgb = spt[2 * slot + 1];
        m.scale = ssc ? ssc[slot] : 0.f;
    } else {
        m.r = a.ranks[slot];
        m.pga = reinterpret_cast<const int4 *>(a.pt)[2 * slot];
        m.pgb = reinterpret_cast<const int4 *>(a.pt)[2 * slot + 1];
        m.scale = ssc ? a.scales[slot] : 0.f;
    }
    return m;
}

__device__ __forceinline__ Meta check_meta(const KSplit &a, const RawMeta &raw) {
    Meta m;
    int r = raw.r;
    m.pga = raw.pga;
    m.pgb = raw.pgb;
    m.scale = raw.scale;
    m.bad = r > LORA_MAX_RANK;
    if (r <= 0 || m.bad) r = 0;
    const int np = (r + LORA_PAGE_ROWS - 1) / LORA_PAGE_ROWS;
    const int pa[4] = {m.pga.x, m.pga.y, m.pga.z, m.pga.w};
    const int pb[4] = {m.pgb.x, m.pgb.y, m.pgb.z, m.pgb.w};
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        if (p < np) {
            if (pa[p] < 0 || (long long)(pa[p] + 1) * LORA_PAGE_ROWS > a.rowsA) m.bad = true;
            if (pb[p] < 0 || (long long)(pb[p] + 1) * LORA_PAGE_ROWS > a.rowsB) m.bad = true;
        }
    }
    m.r = m.bad ? 0 : r;
    m.np = m.bad ? 0 : np;
    return m;
}

// Token t of a job: the first four are in the job record, the rest in the
// plan's token list.  -1 past the job's end.
__device__ __forceinline__ int job_token(const KSplit &a, const int4 &tk, int q0, int n, int t) {
    if (t >= n) return -1;
    if (t < 4) return t == 0 ? tk.x : t == 1 ? tk.y : t == 2 ? tk.z : tk.w;
    return ld_cg_s32(a.perm + q0 + t);
}

// Stage the slot tables of up to kTableSlots slots (caller state, read before
// the kernel waits for its predecessor).
template <class Sm>
__device__ __forceinline__ bool stage_tables(const KSplit &a, Sm &sm, float *scales) {
    const bool staged = a.S <= kTableSlots;
    if (staged) {
        for (int i = threadIdx.x; i < a.S; i += kThreads) {
            sm.pt[2 * i] = reinterpret_cast<const int4 *>(a.pt)[2 * i];
            sm.pt[2 * i + 1] = reinterpret_cast<const int4 *>(a.pt)[2 * i + 1];
            sm.ranks[i] = a.ranks[i];
            if (scales) scales[i] = a.scales[i];
        }
    }
    return staged;
}

// ---------------------------------------------------------------------------
// Shrink: partial v of one d_in quarter per unit.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads, 1)
shrink_part_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmA4,
                   const __grid_constant__ KSplit a) {
    extern __shared__ unsigned char smem_raw[];
    ShrinkSmem &sm = *reinterpret_cast<ShrinkSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kSlots; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], kCW);
        }
        mbar_init(&sm.red_full, kCW);
        mbar_init(&sm.red_free, kCW);
        sm.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA4)) : "memory");
    }
    const bool staged = stage_tables(a, sm, (float *)nullptr);
    // The plan (job list) may come from the kernel just before this one: wait
    // for it, then let the expand kernel get resident.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");
    __syncthreads();

    if (warp == kCW) {
        // ------------------------------ producer ------------------------------
        const int n_jobs = a.hdr->n_jobs;
        const int n_units = n_jobs * kSlices;
        const unsigned Gi = (unsigned)a.d_in >> 3;
        const int G = gridDim.x;
        Ring rg = {0, 0, 0, 0};
        bool ok = true;
        // the job record two units ahead and the slot tables one unit ahead are
        // in flight while the current unit streams
        int4 jobA = make_int4(0, 0, 0, 0), tkA = jobA, jobB = jobA, tkB = jobA;
        RawMeta rmA = {};
        int tokA = -1;
        const int u0 = blockIdx.x;
        if (u0 < n_units) { jobA = a.jobs[2 * (u0 / kSlices)]; tkA = a.jobs[2 * (u0 / kSlices) + 1]; }
        if (u0 + G < n_units) { jobB = a.jobs[2 * ((u0 + G) / kSlices)]; tkB = a.jobs[2 * ((u0 + G) / kSlices) + 1]; }
        if (u0 < n_units) {
            rmA = raw_meta(a, sm.pt, sm.ranks, nullptr, staged, jobA.x);
            tokA = job_token(a, tkA, jobA.z, min(jobA.y, LORA_MAX_JOB_TOKENS), lane);
        }
        for (int u = u0; u < n_units && ok; u += G) {
            const int s = u - (u / kSlices) * kSlices;
            const int4 job = jobA;
            const RawMeta rm = rmA;
            const int mytok = tokA;
            jobA = jobB;
            tkA = tkB;
            if (u + G < n_units) {
                rmA = raw_meta(a, sm.pt, sm.ranks, nullptr, staged, jobA.x);
                tokA = job_token(a, tkA, jobA.z, min(jobA.y, LORA_MAX_JOB_TOKENS), lane);
            }
            if (u + 2 * G < n_units) {
                jobB = a.jobs[2 * ((u + 2 * G) / kSlices)];
                tkB = a.jobs[2 * ((u + 2 * G) / kSlices) + 1];
            }
            const int n = min(job.y, LORA_MAX_JOB_TOKENS), q0 = job.z;
            const Meta m = check_meta(a, rm);
            if (m.r == 0 || n <= 0) continue;
            const int nt = (n + kNTok - 1) / kNTok;
            const int in0 = 8 * (int)(Gi * s / kSlices), in1 = 8 * (int)(Gi * (s + 1) / kSlices);
            if (in1 <= in0) continue;
            // as many 64-column blocks per page as keep two chunks in the ring
            int nb = max(1, min(kMaxBoxes / m.np, nt > 1 ? 8 : 16));
            while (nb > 1 && m.np * nb * kBoxBytes + nt * kNTok * (nb * kBoxCols * 2 + 16) > kShrinkArena / 2) --nb;
            const int cw = nb * kBoxCols, px = cw * 2 + 16;
            const int nch = (in1 - in0 + cw - 1) / cw;
            const int box_bytes = m.np * nb * kBoxBytes;
            for (int c = 0; c < nch; ++c) {
                const int off = ring_alloc<kShrinkArena>(rg, sm, box_bytes + nt * kNTok * px, a.err, [] {});
                if (off < 0) { ok = false; break; }
                const int st = rg.chunk % kSlots;
                const int c0 = in0 + c * cw, c1 = min(c0 + cw, in1);
                const int boxes = (c1 - c0 + kBoxCols - 1) / kBoxCols;
                if (lane == 0) {
                    ChunkHdr &h = sm.hdr[st];
                    h.unit = u; h.off = off; h.first = c == 0; h.last = c == nch - 1;
                    h.c0 = c0; h.cols = c1 - c0; h.nb = nb; h.np = m.np; h.r = m.r; h.n = n; h.nt = nt;
                    h.lo = in0; h.hi = in1; h.q0 = q0; h.slice = s; h.scale = 0.f;
                    mbar_expect_tx(&sm.full[st], (uint32_t)(m.np * boxes * kBoxBytes + n * (c1 - c0) * 2));
                }
                __syncwarp();
                unsigned char *sb = sm.ring + off;
                // lanes 16..31 issue the page boxes (a group of four 64-column
                // blocks per lane), lanes 0..n-1 the X rows
                if (lane >= 16)
                    issue_page_boxes(lane - 16, sb, &tmA, &tmA4, a.wide_in, a.d_in, m.np, nb, boxes, c0, m.pga,
                                     &sm.full[st]);
                if (lane < n)
                    bulk_load(sb + box_bytes + lane * px, a.X + (size_t)mytok * a.d_in + c0, (uint32_t)((c1 - c0) * 2),
                              &sm.full[st]);
                ++rg.chunk;
            }
        }
        if (ok && ring_alloc<kShrinkArena>(rg, sm, 0, a.err, [] {}) >= 0) {   // end marker
            const int st = rg.chunk % kSlots;
            if (lane == 0) {
                sm.hdr[st].unit = -1;
                mbar_arrive(&sm.full[st]);
            }
            ++rg.chunk;
        }
        if (lane == 0)
            for (int i = max(rg.popped, rg.chunk - kSlots); i < rg.chunk; ++i)
                drain_wait(&sm.full[i % kSlots], (i / kSlots) & 1);
        return;
    }

    // ------------------------------ consumers ------------------------------
    const int li = lane & 7, lj = lane >> 3, g8 = lane >> 2;
    float acc[kMaxPages][kMaxNT][4];
    int chunk = 0, nred = 0;
    while (true) {
        const int st = chunk % kSlots;
        if (!wait_w(&sm.full[st], (chunk / kSlots) & 1, sm, a.err)) break;
        const ChunkHdr &h = sm.hdr[st];
        if (h.unit < 0) break;
        const int first = h.first, last = h.last, c0 = h.c0, cols = h.cols, nb = h.nb, np = h.np, r = h.r;
        const int n = h.n, nt = h.nt, lo = h.lo, hi = h.hi, q0 = h.q0, slice = h.slice, off = h.off;
        if (first) {
#pragma unroll
            for (int p = 0; p < kMaxPages; ++p)
#pragma unroll
                for (int j = 0; j < kMaxNT; ++j)
#pragma unroll
                    for (int i = 0; i < 4; ++i) acc[p][j][i] = 0.f;
        }
        const int px = nb * kBoxCols * 2 + 16;
        const int nks = (cols + 15) >> 4;
        const int kbase = (c0 - lo) >> 4;
        const uint32_t sb = smem_u32(sm.ring + off);
        const uint32_t xb = sb + np * nb * kBoxBytes;
        const bool tok0 = g8 < n, tok1 = kNTok + g8 < n;
        int kk = warp - kbase % kCW;
        if (kk < 0) kk += kCW;
        for (; kk < nks; kk += kCW) {
            // X fragments (B side) of both token tiles; tokens past n and
            // columns past the quarter's end enter as zeros
            uint32_t bx[kMaxNT][2];
            {
                const int t = (lj >> 1) * kNTok + li;
                const uint32_t ad = xb + (uint32_t)(t * px + (2 * kk + (lj & 1)) * 16);
                if (nt > 1) {
                    uint32_t r4[4];
                    ldsm_x4(ad, r4);
                    bx[0][0] = r4[0]; bx[0][1] = r4[1];
                    bx[1][0] = r4[2]; bx[1][1] = r4[3];
                } else {
                    ldsm_x2(ad, bx[0][0], bx[0][1]);
                    bx[1][0] = bx[1][1] = 0u;
                }
                const int col = c0 + 16 * kk;
                const bool lo_ok = col < hi, hi_ok = col + 8 < hi;
                bx[0][0] = (lo_ok && tok0) ? bx[0][0] : 0u;
                bx[0][1] = (hi_ok && tok0) ? bx[0][1] : 0u;
                bx[1][0] = (lo_ok && tok1) ? bx[1][0] : 0u;
                bx[1][1] = (hi_ok && tok1) ? bx[1][1] : 0u;
            }
            const int b = kk >> 2, ks = kk & 3;
#pragma unroll
            for (int p = 0; p < kMaxPages; ++p) {
                if (p < np) {
                    uint32_t af[4];
                    const int row = li + 8 * (lj & 1);
                    ldsm_x4(sb + (uint32_t)((p * nb + b) * kBoxBytes + row * 128 + (((2 * ks + (lj >> 1)) ^ li) << 4)),
                            af);
                    mma_bf16(acc[p][0], af, bx[0][0], bx[0][1]);
                    if (nt > 1) mma_bf16(acc[p][1], af, bx[1][0], bx[1][1]);
                }
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.empty[st]);
        ++chunk;
        if (!last) continue;

        // the warps' partials of this quarter, added in warp order
        if (nred > 0 && !wait_w(&sm.red_free, (nred - 1) & 1, sm, a.err)) break;
#pragma unroll
        for (int p = 0; p < kMaxPages; ++p)
#pragma unroll
            for (int j = 0; j < kMaxNT; ++j)
                if (p < np && j < nt)
                    *reinterpret_cast<float4 *>(sm.red + ((warp * kMaxPages + p) * kMaxNT + j) * 128 + lane * 4) =
                        make_float4(acc[p][j][0], acc[p][j][1], acc[p][j][2], acc[p][j][3]);
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.red_full);
        if (!wait_w(&sm.red_full, nred & 1, sm, a.err)) break;
        for (int idx = threadIdx.x; idx < np * nt * 128; idx += kConsumers) {
            const int p = idx / (nt * 128), rest = idx - p * nt * 128;
            const int j = rest >> 7, el = rest & 127;
            // element el of a fragment: lane el / 4, register el % 4
            const int fl = el >> 2, fr = el & 3;
            const int k = p * LORA_PAGE_ROWS + (fl >> 2) + 8 * (fr >> 1);
            const int t = j * kNTok + 2 * (fl & 3) + (fr & 1);
            if (t < n && k < r) {
                float sum = 0.f;
#pragma unroll 5
                for (int w = 0; w < kCW; ++w) sum += sm.red[((w * kMaxPages + p) * kMaxNT + j) * 128 + el];
                a.vpart[((size_t)slice * a.T + q0 + t) * LORA_MAX_RANK + k] = sum;
            }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.red_free);
        ++nred;
    }
}

// Quarters of d_in that hold columns (d_in below 32 leaves some empty; an
// empty quarter adds +0 to v in the cluster kernel, so skipping it in the sum
// gives the same bits).
__device__ __forceinline__ unsigned quarter_mask(int d_in) {
    const unsigned Gi = (unsigned)d_in >> 3;
    unsigned m = 0;
#pragma unroll
    for (int q = 0; q < kSlices; ++q)
        if (Gi * (q + 1) / kSlices > Gi * q / kSlices) m |= 1u << q;
    return m;
}

// d_out parts per job for this launch: enough units to fill the grid, few
// enough that each unit still streams a long run of B columns.
__device__ __forceinline__ int choose_parts(int n_jobs, int grid, int e_max) {
    int E = 1;
    if (n_jobs < grid) {
        E = grid / n_jobs;
    } else {
        float best = 1e30f;
        for (int e = 1; e <= 4; ++e) {
            const int rounds = (n_jobs * e + grid - 1) / grid;
            const float cost = rounds * (1.f / e + 0.03f);
            if (cost < best - 1e-6f) { best = cost; E = e; }
        }
    }
    return max(1, min(E, e_max));
}

// ---------------------------------------------------------------------------
// Expand: Y += s * v B over one d_out part per unit.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads, 1)
expand_part_kernel(const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmB4,
                   const __grid_constant__ KSplit a) {
    extern __shared__ unsigned char smem_raw[];
    ExpandSmem &sm = *reinterpret_cast<ExpandSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kSlots; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], kCW);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.vfull[b], 1);
            mbar_init(&sm.vempty[b], kCW);
        }
        mbar_init(&sm.vt_full, kCW);
        mbar_init(&sm.vt_free, kCW);
        sm.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB4)) : "memory");
    }
    // The shrink kernel ahead of this one waited for the plan before it let
    // this grid start, so the plan, the slot tables, the pages and Y may be
    // read now; only the partials need the shrink grid to have finished.
    const bool staged = stage_tables(a, sm, sm.scales);
    __syncthreads();

    if (warp == kCW) {
        // ------------------------------ producer ------------------------------
        const int n_jobs = ld_cg_s32(&a.hdr->n_jobs);
        const int E = n_jobs > 0 ? choose_parts(n_jobs, gridDim.x, a.e_max) : 1;
        const int n_units = n_jobs * E;
        const long long Go = a.d_out >> 3;
        const unsigned qmask = quarter_mask(a.d_in);
        Ring rg = {0, 0, 0, 0};
        int nv = 0;
        bool ok = true, waited = false;
        auto wait_shrink = [&]() {
            asm volatile("griddepcontrol.wait;" ::: "memory");
            asm volatile("griddepcontrol.launch_dependents;");
            waited = true;
        };
        const int G = gridDim.x;
        int4 jobA = make_int4(0, 0, 0, 0), tkA = jobA, jobB = jobA, tkB = jobA;
        RawMeta rmA = {};
        int tokA = -1;
        const int u0 = blockIdx.x;
        if (u0 < n_units) { jobA = ld_cg_v4(a.jobs + 2 * (u0 / E)); tkA = ld_cg_v4(a.jobs + 2 * (u0 / E) + 1); }
        if (u0 + G < n_units) {
            jobB = ld_cg_v4(a.jobs + 2 * ((u0 + G) / E));
            tkB = ld_cg_v4(a.jobs + 2 * ((u0 + G) / E) + 1);
        }
        if (u0 < n_units) {
            rmA = raw_meta(a, sm.pt, sm.ranks, sm.scales, staged, jobA.x);
            tokA = job_token(a, tkA, jobA.z, min(jobA.y, LORA_MAX_JOB_TOKENS), lane);
        }
        for (int u = u0; u < n_units && ok; u += G) {
            const int ji = u / E, e = u - ji * E;
            const int4 job = jobA;
            const RawMeta rm = rmA;
            const int mytok = tokA;
            jobA = jobB;
            tkA = tkB;
            if (u + G < n_units) {
                rmA = raw_meta(a, sm.pt, sm.ranks, sm.scales, staged, jobA.x);
                tokA = job_token(a, tkA, jobA.z, min(jobA.y, LORA_MAX_JOB_TOKENS), lane);
            }
            if (u + 2 * G < n_units) {
                jobB = ld_cg_v4(a.jobs + 2 * ((u + 2 * G) / E));
                tkB = ld_cg_v4(a.jobs + 2 * ((u + 2 * G) / E) + 1);
            }
            const int n = min(job.y, LORA_MAX_JOB_TOKENS), q0 = job.z;
            const Meta m = check_meta(a, rm);
            if (m.bad && e == 0 && lane == 0 && a.err) atomicOr(a.err, LORA_DEV_ERR_BAD_PAGE);
            if (m.r == 0 || n <= 0) continue;
            const int out0 = 8 * (int)(Go * e / E), out1 = 8 * (int)(Go * (e + 1) / E);
            if (out1 <= out0) continue;
            const int nt = (n + kNTok - 1) / kNTok;
            const int ylim = ((kRowRegion / n) - 16) / 4 / kBoxCols;   // Y rows of a chunk fit the row region
            // as many 64-column blocks per page as keep two chunks in the ring
            int nb = max(1, min(16, ylim));
            while (nb > 1 && m.np * nb * kBoxBytes + n * (nb * kBoxCols * 4 + 16) > kExpandArena / 2) --nb;
            const int cw = nb * kBoxCols, py = cw * 4 + 16;
            const int nch = (out1 - out0 + cw - 1) / cw;
            const int vb = nv & 1;
            auto issue_v = [&]() {
                if (!wait_w(&sm.vempty[vb], ((nv >> 1) & 1) ^ 1, sm, a.err)) return false;
                if (lane == 0) mbar_expect_tx(&sm.vfull[vb], (uint32_t)(__popc(qmask) * n * LORA_MAX_RANK * 4));
                __syncwarp();
                if (lane < kSlices && ((qmask >> lane) & 1u))
                    bulk_load(sm.vst[vb][lane], a.vpart + ((size_t)lane * a.T + q0) * LORA_MAX_RANK,
                              (uint32_t)(n * LORA_MAX_RANK * 4), &sm.vfull[vb]);
                ++nv;
                return true;
            };
            // The first unit's partials are fetched (after waiting for the
            // shrink grid) just before the producer would first have to wait
            // for ring space, or after its last chunk: until then its B pages and
            // Y rows stream in while the shrink kernel still runs.
            bool pending_v = true;
            if (waited) {
                if (!issue_v()) { ok = false; break; }
                pending_v = false;
            }
            auto before_block = [&]() {
                if (!pending_v) return;
                if (!waited) wait_shrink();
                if (!issue_v()) ok = false;
                pending_v = false;
            };
            const int box_bytes = m.np * nb * kBoxBytes;
            for (int c = 0; c < nch && ok; ++c) {
                const int off = ring_alloc<kExpandArena>(rg, sm, box_bytes + n * py, a.err, before_block);
                if (off < 0 || !ok) { ok = false; break; }
                const int st = rg.chunk % kSlots;
                const int c0 = out0 + c * cw, c1 = min(c0 + cw, out1);
                const int boxes = (c1 - c0 + kBoxCols - 1) / kBoxCols;
                if (lane == 0) {
                    ChunkHdr &h = sm.hdr[st];
                    h.unit = u; h.off = off; h.first = c == 0; h.last = c == nch - 1;
                    h.c0 = c0; h.cols = c1 - c0; h.nb = nb; h.np = m.np; h.r = m.r; h.n = n; h.nt = nt;
                    h.lo = out0; h.hi = out1; h.q0 = q0; h.slice = vb; h.scale = m.scale;
                }
                if (lane < LORA_MAX_JOB_TOKENS) sm.hdr[st].tok[lane] = mytok;
                __syncwarp();
                if (lane == 0)
                    mbar_expect_tx(&sm.full[st], (uint32_t)(m.np * boxes * kBoxBytes + n * (c1 - c0) * 4));
                __syncwarp();
                unsigned char *sb = sm.ring + off;
                // lanes 16..31 issue the page boxes (a group of four 64-column
                // blocks per lane), lanes 0..n-1 the Y rows
                if (lane >= 16)
                    issue_page_boxes(lane - 16, sb, &tmB, &tmB4, a.wide_out, a.d_out, m.np, nb, boxes, c0, m.pgb,
                                     &sm.full[st]);
                if (lane < n)
                    bulk_load(sb + box_bytes + lane * py, a.Y + (size_t)mytok * a.d_out + c0,
                              (uint32_t)((c1 - c0) * 4), &sm.full[st]);
                ++rg.chunk;
            }
            if (ok) before_block();   // a unit whose chunks all fit without waiting
        }
        if (!waited) wait_shrink();
        if (ok && ring_alloc<kExpandArena>(rg, sm, 0, a.err, [] {}) >= 0) {   // end marker
            const int st = rg.chunk % kSlots;
            if (lane == 0) {
                sm.hdr[st].unit = -1;
                mbar_arrive(&sm.full[st]);
            }
            ++rg.chunk;
        }
        if (lane == 0) {
            for (int i = max(rg.popped, rg.chunk - kSlots); i < rg.chunk; ++i)
                drain_wait(&sm.full[i % kSlots], (i / kSlots) & 1);
            for (int i = (nv > 2 ? nv - 2 : 0); i < nv; ++i) drain_wait(&sm.vfull[i & 1], (i >> 1) & 1);
        }
        return;
    }

    // ------------------------------ consumers ------------------------------
    const int li = lane & 7, lj = lane >> 3, g8 = lane >> 2, tig = lane & 3;
    const uint32_t vt_base = smem_u32(sm.vt);
    const unsigned qmask = quarter_mask(a.d_in);
    int chunk = 0, nunit = 0;
    while (true) {
        const int st = chunk % kSlots;
        if (!wait_w(&sm.full[st], (chunk / kSlots) & 1, sm, a.err)) break;
        const ChunkHdr &h = sm.hdr[st];
        if (h.unit < 0) break;
        const int first = h.first, last = h.last, c0 = h.c0, cols = h.cols, nb = h.nb, np = h.np, r = h.r;
        const int n = h.n, nt = h.nt, hi = h.hi, vb = h.slice, off = h.off;
        const float sc = h.scale;
        if (first) {
            // v = the four quarters' partials added in quarter order, split into
            // a bf16 high part and a bf16 low part (v - high)
            if (nunit > 0 && !wait_w(&sm.vt_free, (nunit - 1) & 1, sm, a.err)) break;
            if (!wait_w(&sm.vfull[vb], (nunit >> 1) & 1, sm, a.err)) break;
            for (int idx = threadIdx.x; idx < n * r; idx += kConsumers) {
                const int t = idx / r, k = idx - t * r;
                const int o = t * LORA_MAX_RANK + k;
                float v = 0.f;
#pragma unroll
                for (int q = 0; q < kSlices; ++q)
                    if ((qmask >> q) & 1u) v += sm.vst[vb][q][o];
                const uint16_t hv = bf16_rn(v);
                const uint16_t lv = bf16_rn(v - __uint_as_float((uint32_t)hv << 16));
                const uint32_t so = swz(t, LORA_MAX_RANK * 2, k >> 3) + (k & 7) * 2;
                *reinterpret_cast<uint16_t *>(sm.vt + so) = hv;
                *reinterpret_cast<uint16_t *>(sm.vt + kVTileBytes + so) = lv;
            }
            // rank rows past r (up to the page end) and token rows past n hold
            // zeros: 0 * v must not meet a stale non-finite value
            for (int idx = threadIdx.x; idx < nt * kNTok * np * LORA_PAGE_ROWS; idx += kConsumers) {
                const int t = idx / (np * LORA_PAGE_ROWS), k = idx - t * (np * LORA_PAGE_ROWS);
                if (t >= n || k >= r) {
                    const uint32_t so = swz(t, LORA_MAX_RANK * 2, k >> 3) + (k & 7) * 2;
                    *reinterpret_cast<uint16_t *>(sm.vt + so) = 0;
                    *reinterpret_cast<uint16_t *>(sm.vt + kVTileBytes + so) = 0;
                }
            }
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&sm.vempty[vb]);
                mbar_arrive(&sm.vt_full);
            }
            if (!wait_w(&sm.vt_full, nunit & 1, sm, a.err)) break;
        }

        // expand-add over this chunk: 16-column m-tiles, warp w takes m-tiles
        // congruent to w mod 15; Y rows of the chunk sit in the stage
        const int cw = nb * kBoxCols, py4 = cw + 4;   // Y row pitch in floats
        const int nmt = (cols + 15) >> 4;
        const uint32_t sb = smem_u32(sm.ring + off);
        float *ys = reinterpret_cast<float *>(sm.ring + off + np * nb * kBoxBytes);
        const uint32_t vbase = vt_base + ((lj >> 1) ? kVTileBytes : 0);
        const int krow = li + 8 * (lj >> 1);
        // A warp runs up to kTilesPerWarp of its m-tiles (mt, mt + 15, mt + 30)
        // at once: their MMA chains are independent and interleave, while each
        // accumulator still sees pages in order, high part before low part.
        for (int mt0 = warp; mt0 < nmt; mt0 += kTilesPerWarp * kCW) {
            float d[kTilesPerWarp][kMaxNT][4];
            uint32_t offA[kTilesPerWarp];
            bool has[kTilesPerWarp];
#pragma unroll
            for (int q = 0; q < kTilesPerWarp; ++q) {
                const int mt = mt0 + q * kCW;
                has[q] = mt < nmt;
                offA[q] = (uint32_t)((mt >> 2) * kBoxBytes + krow * 128 + (((2 * (mt & 3) + (lj & 1)) ^ li) << 4));
#pragma unroll
                for (int jj = 0; jj < kMaxNT; ++jj)
#pragma unroll
                    for (int i = 0; i < 4; ++i) d[q][jj][i] = 0.f;
            }
#pragma unroll 1
            for (int p = 0; p < np; ++p) {
                uint32_t af[kTilesPerWarp][4];
#pragma unroll
                for (int q = 0; q < kTilesPerWarp; ++q)
                    if (has[q]) ldsm_x4_t(sb + (uint32_t)(p * nb * kBoxBytes) + offA[q], af[q]);
#pragma unroll
                for (int jj = 0; jj < kMaxNT; ++jj) {
                    if (jj < nt) {
                        uint32_t bv[4];
                        ldsm_x4(vbase + swz(jj * kNTok + li, LORA_MAX_RANK * 2, 2 * p + (lj & 1)), bv);
#pragma unroll
                        for (int q = 0; q < kTilesPerWarp; ++q)
                            if (has[q]) mma_bf16(d[q][jj], af[q], bv[0], bv[1]);
#pragma unroll
                        for (int q = 0; q < kTilesPerWarp; ++q)
                            if (has[q]) mma_bf16(d[q][jj], af[q], bv[2], bv[3]);
                    }
                }
            }
            // y = fmaf(s, acc, y) for column g8 / g8 + 8 and tokens 2 tig,
            // 2 tig + 1, the old value from the staged Y rows, the new one
            // straight to global memory (eight consecutive columns of a row per
            // store)
#pragma unroll
            for (int jj = 0; jj < kMaxNT; ++jj) {
                if (jj < nt) {
                    const int t0 = jj * kNTok + 2 * tig;
                    const int tok0 = t0 < n ? h.tok[t0] : 0, tok1 = t0 + 1 < n ? h.tok[t0 + 1] : 0;
#pragma unroll
                    for (int q = 0; q < kTilesPerWarp; ++q) {
                        if (!has[q]) continue;
                        const int mt = mt0 + q * kCW;
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const int t = t0 + (i & 1), cc = mt * 16 + g8 + 8 * (i >> 1);
                            if (t < n && c0 + cc < hi)
                                a.Y[(size_t)((i & 1) ? tok1 : tok0) * a.d_out + c0 + cc] =
                                    fmaf(sc, d[q][jj][i], ys[t * py4 + cc]);
                        }
                    }
                }
            }
        }
        // the staged Y rows were only read
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.empty[st]);
        ++chunk;
        if (last) {
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.vt_free);
            ++nunit;
        }
    }
}

constexpr size_t kShrinkSmemBytes = sizeof(ShrinkSmem) + 1024;
constexpr size_t kExpandSmemBytes = sizeof(ExpandSmem) + 1024;
int g_split_sms[64] = {};

int split_grid(int *out) {
    int dev = 0;
    if (int rc = cuda_check(cudaGetDevice(&dev))) return rc;
    if (dev < 0 || dev >= 64) return LORA_ERR_INVALID_ARG;
    if (g_split_sms[dev] == 0) {
        if (int rc = cuda_check(cudaFuncSetAttribute(shrink_part_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                     (int)kShrinkSmemBytes)))
            return rc;
        if (int rc = cuda_check(cudaFuncSetAttribute(expand_part_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                     (int)kExpandSmemBytes)))
            return rc;
        int sms = 0, occ = 0;
        if (int rc = cuda_check(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev))) return rc;
        if (int rc = cuda_check(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, shrink_part_kernel, kThreads,
                                                                                kShrinkSmemBytes)))
            return rc;
        g_split_sms[dev] = max(1, sms * max(1, occ));
    }
    *out = g_split_sms[dev];
    return LORA_OK;
}

}  // namespace

size_t split_vpart_bytes(int T) { return (size_t)kSlices * (size_t)(T > 0 ? T : 1) * LORA_MAX_RANK * sizeof(float); }

int launch_split(const SplitArgs &s, lora_pool_s *pa, lora_pool_s *pb, cudaStream_t st) {
    int grid = 1;
    if (int rc = split_grid(&grid)) return rc;
    CUtensorMap tmA, tmB, tmA4, tmB4;
    if (int rc = pool_tensor_map(pa, &tmA)) return rc;
    if (int rc = pool_tensor_map(pb, &tmB)) return rc;
    const bool wide_in = pa->width >= 256, wide_out = pb->width >= 256;
    if (wide_in) {
        if (int rc = pool_tensor_map4(pa, &tmA4)) return rc;
    } else {
        tmA4 = tmA;
    }
    if (wide_out) {
        if (int rc = pool_tensor_map4(pb, &tmB4)) return rc;
    } else {
        tmB4 = tmB;
    }
    KSplit k;
    k.X = s.X; k.Y = s.Y; k.T = s.T; k.d_in = s.d_in; k.d_out = s.d_out; k.S = s.S;
    k.ranks = s.ranks; k.scales = s.scales; k.pt = s.pt;
    k.rowsA = (long long)pa->num_pages * LORA_PAGE_ROWS;
    k.rowsB = (long long)pb->num_pages * LORA_PAGE_ROWS;
    k.perm = s.perm; k.jobs = s.jobs; k.hdr = s.hdr; k.vpart = s.vpart; k.err = s.err;
    k.e_max = max(1, (s.d_out >> 3) / 8);
    k.wide_in = wide_in;
    k.wide_out = wide_out;

    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.blockDim = dim3(kThreads);
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const long long t = s.T > 0 ? s.T : 1;
    cfg.gridDim = dim3((unsigned)(t * kSlices < grid ? t * kSlices : grid));
    cfg.dynamicSmemBytes = kShrinkSmemBytes;
    if (int rc = cuda_check(cudaLaunchKernelEx(&cfg, shrink_part_kernel, tmA, tmA4, k))) return rc;
    count_launch();
    cfg.gridDim = dim3((unsigned)(t * k.e_max < grid ? t * k.e_max : grid));
    cfg.dynamicSmemBytes = kExpandSmemBytes;
    if (int rc = cuda_check(cudaLaunchKernelEx(&cfg, expand_part_kernel, tmB, tmB4, k))) return rc;
    count_launch();
    note_launch(st, false);
    return LORA_OK;
}

}  // namespace lora
