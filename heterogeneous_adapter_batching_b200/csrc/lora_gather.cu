// Gather path for short segments (decode: a few tokens per adapter).
//
// Page "Multi-LoRA Serving in Production" (llms.blog), section "Multi-Size
// Batched Gather Kernels (MBGMV and MBGMM)": in decode each sequence
// contributes one token, and the kernel gathers every token's adapter
// weights from non-contiguous rank buffers of different sizes without padding
// to the largest rank.  Section "Segmented Gather Matrix-Vector
// Multiplication (SGMV)": shrink v = x A, then expand v B scaled by alpha/r and
// added to the base output.  Section "Unified Paging Architecture": the
// weights are read straight out of the physical pages the page table names.
//
// Work unit = one gather job (an adapter slot and up to 16 of its tokens, from
// the plan kernel) times one projection (a launch may cover up to 8 that read
// the same X) times one part e of an E-way split of d_out.  A cluster of kCS
// CTAs (one per SM) runs one unit at a time and loops over the units in
// rounds of one unit per cluster, each round in the opposite direction to the
// last (persistent grid sized from the occupancy of the cluster shape).  Per
// CTA:
//   * a producer warp streams the adapter's pages into a ring of shared-memory
//     stages with 2D TMA loads of 16 rank rows x 64 columns (128-byte
//     swizzled): first the CTA's 1/kCS slice of d_in (rows of A^T), then its
//     slice of d_out (rows of B).  It runs ahead into the next unit while the
//     consumers finish the current one.  Only the pages the adapter has are
//     read; a rank that is not a multiple of 16 reads the zeroed rows of its
//     last page;
//   * 15 consumer warps copy the tokens' X columns of each chunk into shared
//     memory (cp.async, issued one chunk ahead) and run the shrink on the
//     tensor cores with warp-level bf16 MMAs (m16n8k16, fp32 accumulate): a
//     page's 16 rank rows are the M side, 8 tokens the N side (two N tiles
//     for a 16-token job), and each warp owns every 15th 16-column step of
//     the slice.  The warps' partial sums are added in warp order; each CTA
//     pushes its partial into its peers' shared memory with asynchronous
//     DSMEM stores that complete on the peer's mbarrier, and adds the kCS
//     partials in rank order, so all CTAs hold the same fp32 v and a token's
//     result does not depend on the job it landed in;
//   * v is split into a bf16 high part and a bf16 low part (v - high), and the
//     expand runs as two MMAs per page (output columns on the M side, read
//     with transposing ldmatrix), which keeps v to about 16 significant bits;
//     each warp owns every 15th 16-column tile of the d_out slice, takes its
//     tiles in pairs whose MMA chains interleave, turns the results into rows
//     through small shared tiles and updates Y in place with float4 rows.
// Slot tables of up to 128 (projection, slot) entries are staged in shared
// memory before the kernel waits for its predecessor, so a unit's metadata
// costs one global read (the job record).  The hardware cluster barrier is
// used once, at start-up.  Every wait is bounded; a wait that runs out sets
// LORA_DEV_ERR_TIMEOUT in the error word and the kernel runs to completion
// without trapping.  No cluster multicast is used.
#include "lora_internal.cuh"
#include "lora_ptx.cuh"

namespace lora {
namespace {

constexpr int kCS = 4;                       // CTAs per cluster
constexpr int kConsumerWarps = 15;           // + 1 producer = 16 warps: 4 per SM sub-partition
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32;    // + one producer warp
constexpr int kNTok = 8;                     // tokens per MMA (the N side)
constexpr int kMaxNTiles = LORA_MAX_JOB_TOKENS / kNTok;
constexpr int kMaxJobTokens = kMaxNTiles * kNTok;
constexpr int kMaxPages = LORA_MAX_RANK / LORA_PAGE_ROWS;
constexpr int kStages = 2;
constexpr int kBoxCols = 64;                 // TMA box: 16 rows x 64 columns of bf16 = 2 KB, 128B swizzle
constexpr int kBoxBytes = LORA_PAGE_ROWS * kBoxCols * 2;
constexpr int kStageBoxes = 32;              // a stage holds 32 boxes = 64 KB
constexpr int kMaxPageBoxes = 16;            // 64-column blocks of one page in a chunk at most
constexpr int kMaxChunkCols = kMaxPageBoxes * kBoxCols;   // widest chunk (1024 columns)
constexpr int kTableSlots = 128;             // page tables up to this many slots live in shared memory
constexpr long long kWaitLimit = 2000000000LL;   // cycles (~1 s)
constexpr int kMaxSplit = 64;                // most parts d_out is split into

static_assert(kMaxJobTokens == LORA_MAX_JOB_TOKENS, "job size must be a whole number of MMA tiles");
// After the shrink the X buffers hold the warps' partial sums (kRedBytes),
// then this CTA's partial; after the exchange, v in bf16 (high and low parts).
constexpr int kRedBytes = kConsumerWarps * kMaxPages * kMaxNTiles * 128 * 4;
constexpr int kPartFloats = kMaxJobTokens * LORA_MAX_RANK;
constexpr int kVBytes = kMaxJobTokens * LORA_MAX_RANK * 2;   // one bf16 part of v
// During the expand each warp turns its MMA results into rows of Y through two
// 16-token x 16-column fp32 tiles in the X buffers, after the two parts of v.
constexpr int kYTileBytes = kMaxJobTokens * 16 * 4;
constexpr int kYTileOff = 2 * kVBytes;
static_assert(kRedBytes + kPartFloats * 4 <= 2 * kMaxJobTokens * kMaxChunkCols * 2,
              "the partial sums must fit in the X buffers");
static_assert(kYTileOff + kConsumerWarps * 2 * kYTileBytes <= 2 * kMaxJobTokens * kMaxChunkCols * 2,
              "the warps' Y tiles must fit in the X buffers");

struct __align__(1024) GatherSmem {
    // stage s, box (page p, column block b) at (p * nb + b) * 2 KB, each box
    // 1024-byte aligned in the TMA's 128-byte swizzle
    unsigned char stage[kStages][kStageBoxes * kBoxBytes];
    // X of a chunk: one row of the chunk's columns per token (bf16, the
    // 16-byte groups XOR-swizzled by token row), double-buffered.  After the
    // shrink: the warps' partial sums at 0, this CTA's partial [t][k] at
    // kRedBytes; after the exchange: v's bf16 high part [t][k] (groups
    // swizzled) at 0 and its low part at kVBytes.
    unsigned char xs[2][kMaxJobTokens * kMaxChunkCols * 2];
    // the peers' partial sums [t][k] of the current unit, written by their
    // asynchronous DSMEM stores that complete on rbar; double-buffered over
    // units (slot (q - this rank - 1) mod kCS holds rank q's)
    float R[2][kCS - 1][kPartFloats];
    int4 pt[kTableSlots * 2];                         // staged page-table rows (A pages, B pages)
    int ranks[kTableSlots];
    float scales[kTableSlots];
    int ebound[LORA_MAX_PROJECTIONS][kMaxSplit + 1];  // d_out split: first 8-column group of part e
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t rbar[2];
    int abort;
};

static_assert(sizeof(GatherSmem) + 1024 <= 227 * 1024, "shared memory beyond the per-block limit");

// Kernel parameters for launches of up to NP projections: single-projection
// launches pass one record and one pair of TMA descriptors, not the maximum.
template <int NP>
struct GatherMaps {
    CUtensorMap A[NP];
    CUtensorMap B[NP];
    CUtensorMap A4[NP];   // the pools seen in 3D (four 64-column blocks per box); a copy of A/B for widths below 256
    CUtensorMap B4[NP];
};

template <int NP>
struct KArgs {
    const uint16_t *X;
    float *V;
    int T, d_in;
    int S;
    int nproj;
    GatherProj proj[NP];
    const int32_t *perm;
    const int4 *jobs;
    const PlanHeader *hdr;
    int32_t *err;
    int early;           // the plan was complete before this launch started (see plan_was_last_launch)
};

// The unit a cluster runs in its round k.  Rounds alternate direction, so the
// cluster that took one of the heaviest units first (jobs come heaviest rank
// class first) takes one of the lightest in the next round.  Once a round's
// unit is past the end, every later round's is too.
__device__ __forceinline__ int unit_of(int k, int cluster_id, int n_clusters) {
    return k * n_clusters + ((k & 1) ? n_clusters - 1 - cluster_id : cluster_id);
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ bool mbar_try(uint32_t addr, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(addr), "r"(parity) : "memory");
    return ok != 0;
}

// Bounded wait.  On timeout the CTA-wide abort flag is raised (later waits
// return at once) and the error word records it; execution continues so
// that no peer is left waiting for this CTA.
__device__ __forceinline__ void mbar_wait(uint64_t *bar, uint32_t parity, GatherSmem &sm, int32_t *err) {
    const uint32_t a = smem_u32(bar);
    if (mbar_try(a, parity)) return;
    const long long t0 = clock64();
    while (!mbar_try(a, parity)) {
        if (*(volatile int *)&sm.abort) return;
        if (clock64() - t0 > kWaitLimit) {
            *(volatile int *)&sm.abort = 1;
            if (err) atomicOr(err, LORA_DEV_ERR_TIMEOUT);
            return;
        }
    }
}

// Bounded wait for this thread's own copies before it exits, not cut short
// by the abort flag.
__device__ __forceinline__ void drain_wait(uint64_t *bar, uint32_t parity) {
    const uint32_t a = smem_u32(bar);
    const long long t0 = clock64();
    while (!mbar_try(a, parity) && clock64() - t0 < kWaitLimit / 8) {
    }
}

// A consumer warp frees a stage: its reads of the stage have completed (the
// MMAs that use them issued earlier), and nothing else this arrival would
// order must reach the producer, so the arrive is relaxed: a release here
// would wait for the warp's outstanding global stores of Y.
__device__ __forceinline__ void mbar_arrive_relaxed(uint64_t *bar) {
    asm volatile("mbarrier.arrive.relaxed.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}


__device__ __forceinline__ uint32_t map_peer(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

// Asynchronous 4-byte store into a peer CTA's shared memory that completes
// its transaction count on the peer's mbarrier (no fence needed).
__device__ __forceinline__ void st_async_peer(uint32_t addr, float v, uint32_t bar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];"
                 ::"r"(addr), "r"(__float_as_uint(v)), "r"(bar) : "memory");
}

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_arrive_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }

__device__ __forceinline__ void consumer_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(kConsumers) : "memory");
}

// 16-byte asynchronous copy global -> shared; src_bytes = 0 writes zeros.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t &r0, uint32_t &r1) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr) : "memory");
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr) : "memory");
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr) : "memory");
}

// d += a (16 x 16, row) * b (16 x 8, col); bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
                 "{%0, %1, %2, %3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint16_t bf16_rn(float f) {
    uint16_t h;
    asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(h) : "f"(f));
    return h;
}

// Byte offset of 16-byte group j of row t in a row-major shared array whose
// rows are a multiple of 128 bytes: groups are XOR-swizzled by row so that
// the eight rows an ldmatrix reads sit in different banks.
__device__ __forceinline__ uint32_t swz(int t, int pitch, int j) { return (uint32_t)(t * pitch + ((j ^ (t & 7)) << 4)); }

// Per-slot data of this call, from the shared-memory copy when staged.
struct SlotMeta {
    int r;           // rank, or 0 to skip the unit
    int np;          // pages per matrix
    int4 pga, pgb;   // page ids of A^T and B
    float scale;
    bool bad;
};

template <int MODE, class Args>
__device__ __forceinline__ SlotMeta slot_meta(const Args &a, const GatherSmem &sm, bool staged, int pj,
                                              int slot) {
    SlotMeta m;
    int r;
    const GatherProj &pr = a.proj[pj];
    if (staged) {
        const int i = pj * a.S + slot;
        r = sm.ranks[i];
        m.pga = sm.pt[2 * i];
        m.pgb = sm.pt[2 * i + 1];
        m.scale = sm.scales[i];
    } else {
        r = pr.ranks[slot];
        m.pga = reinterpret_cast<const int4 *>(pr.pt)[2 * slot];
        m.pgb = reinterpret_cast<const int4 *>(pr.pt)[2 * slot + 1];
        m.scale = (MODE == kShrink) ? 0.f : pr.scales[slot];
    }
    m.bad = r > LORA_MAX_RANK;
    if (r <= 0 || m.bad) r = 0;
    const int np = (r + LORA_PAGE_ROWS - 1) / LORA_PAGE_ROWS;
    const int pa[4] = {m.pga.x, m.pga.y, m.pga.z, m.pga.w};
    const int pb[4] = {m.pgb.x, m.pgb.y, m.pgb.z, m.pgb.w};
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        if (p < np) {
            if (MODE != kExpand && (pa[p] < 0 || (long long)(pa[p] + 1) * LORA_PAGE_ROWS > pr.rowsA)) m.bad = true;
            if (MODE != kShrink && (pb[p] < 0 || (long long)(pb[p] + 1) * LORA_PAGE_ROWS > pr.rowsB)) m.bad = true;
        }
    }
    m.r = m.bad ? 0 : r;
    m.np = m.bad ? 0 : np;
    return m;
}

// Column geometry of one unit for this CTA (columns, multiples of 8).
struct UnitGeom {
    int in0, in1;        // d_in slice
    int out0, out1;      // d_out slice
    int nb;              // 64-column boxes per page in a chunk (chunk width nb * 64)
    int n_shrink, n_expand;
};

template <int MODE, class Args>
__device__ __forceinline__ UnitGeom unit_geom(const Args &a, const GatherSmem &sm, int pj, int np, int e,
                                              int crank) {
    UnitGeom g;
    // 32-bit arithmetic: column groups fit easily (d <= 2^24 checked on the host)
    const unsigned Gi = (unsigned)a.d_in >> 3;
    g.in0 = 8 * (int)(Gi * crank / kCS);
    g.in1 = 8 * (int)(Gi * (crank + 1) / kCS);
    const unsigned ge0 = (unsigned)sm.ebound[pj][e], ge1 = (unsigned)sm.ebound[pj][e + 1];
    g.out0 = 8 * (int)(ge0 + (ge1 - ge0) * crank / kCS);
    g.out1 = 8 * (int)(ge0 + (ge1 - ge0) * (crank + 1) / kCS);
    // As many boxes per page as fit in a stage (at most 16 per page, the width
    // of the X buffers): the chunk width depends on the rank only.  A token's
    // fp32 summation order depends on neither the chunk width nor the job it
    // lands in: 16-column steps and tiles are numbered across the whole slice.
    g.nb = np > 0 ? min(kStageBoxes / np, kMaxPageBoxes) : 1;
    const int cw = g.nb * kBoxCols;
    const int win = g.in1 - g.in0, wout = g.out1 - g.out0;
    g.n_shrink = (MODE == kExpand || win <= 0 || np == 0) ? 0 : (win + cw - 1) / cw;
    g.n_expand = (MODE == kShrink || wout <= 0 || np == 0) ? 0 : (wout + cw - 1) / cw;
    return g;
}

// Plan data, read through L2 (it may come from a kernel before the one ahead).
__device__ __forceinline__ int4 ld_v4_now(const int4 *p) {
    int4 v;
    asm volatile("ld.global.cg.v4.s32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}
__device__ __forceinline__ int ld_s32_now(const int *p) {
    int v;
    asm volatile("ld.global.cg.s32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

// Token index t of a job: the first four are in the job record, the rest
// in the plan's slot-ordered token list.  -1 past the job's end.
template <class Args>
__device__ __forceinline__ int job_token(const Args &a, const int4 &tk, int q0, int n, int t) {
    if (t >= n) return -1;
    if (t < 4) return t == 0 ? tk.x : t == 1 ? tk.y : t == 2 ? tk.z : tk.w;
    return __ldg(a.perm + q0 + t);
}

template <int MODE, int NP>
__global__ void __launch_bounds__(kThreads, 1)
gather_kernel(const __grid_constant__ GatherMaps<NP> maps, const __grid_constant__ KArgs<NP> a, int e_max) {
    extern __shared__ unsigned char smem_raw[];
    GatherSmem &sm = *reinterpret_cast<GatherSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int crank = (int)cluster_rank();
    const int cluster_id = blockIdx.x / kCS;
    const int n_clusters = gridDim.x / kCS;
    const int nproj = (NP == 1) ? 1 : a.nproj;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], kConsumerWarps);
        }
        // one arrival per unit (this CTA's expect_tx) plus the peers' bytes
        mbar_init(&sm.rbar[0], 1);
        mbar_init(&sm.rbar[1], 1);
        sm.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // The cluster barrier is used once: every thread arrives here (thread 0
    // after initialising the barriers above and fencing that for the
    // cluster), and waits before its CTA first stores into a peer (or before
    // it exits).  Peers store into this CTA only for units this CTA also runs
    // and waits on, so no CTA exits while a store into it is pending.
    cluster_arrive_relaxed();
    // Every launch's parameters sit in memory this SM has not read yet: fetch
    // them and both tensor maps now, while the previous kernel drains, rather
    // than on first use.
    if (warp == kConsumerWarps && lane < 4 * nproj) {
        const int q = lane >> 2, k = lane & 3;
        const CUtensorMap *m = k == 0 ? &maps.A[q] : k == 1 ? &maps.B[q] : k == 2 ? &maps.A4[q] : &maps.B4[q];
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
    }
    asm volatile("" ::"l"(a.X), "l"(a.V), "r"(a.T), "r"(a.d_in), "r"(a.S), "r"(nproj), "l"(a.perm), "l"(a.jobs),
                 "l"(a.hdr), "l"(a.err), "r"(e_max));
    if (threadIdx.x < nproj) {
        const GatherProj &pr = a.proj[threadIdx.x];
        asm volatile("" ::"l"(pr.Y), "r"(pr.d_out), "r"(pr.ldy), "l"(pr.ranks), "l"(pr.scales), "l"(pr.pt), "l"(pr.rowsA),
                     "l"(pr.rowsB));
    }
    // Small page tables, ranks and scales are staged in shared memory.  They
    // are the caller's slot state, not the plan's output, so they are read
    // before this kernel waits for the kernels ahead of it (the library's own
    // kernels, the only ones here that let a dependent start early, never
    // write them).
    const bool staged = nproj * a.S <= kTableSlots;
    if (staged) {
        for (int i = threadIdx.x; i < nproj * a.S; i += kThreads) {
            const int pj = i / a.S, k = i - pj * a.S;
            const GatherProj &pr = a.proj[pj];
            sm.pt[2 * i] = reinterpret_cast<const int4 *>(pr.pt)[2 * k];
            sm.pt[2 * i + 1] = reinterpret_cast<const int4 *>(pr.pt)[2 * k + 1];
            sm.ranks[i] = pr.ranks[k];
            sm.scales[i] = (MODE == kShrink) ? 0.f : pr.scales[k];
        }
    }
    // Wait for the kernels ahead of this one, then let the next kernel on the
    // stream get its CTAs resident (it reads nothing this grid writes before
    // its own wait, which returns only when this grid has completed).  When
    // the plan was complete before this launch started (a.early), only the
    // consumer warps wait, before they read X and Y: the producer reads the
    // plan and streams the adapter pages while the kernel ahead drains.
    const bool early = a.early != 0;
    auto wait_and_release = []() {
        asm volatile("griddepcontrol.wait;" ::: "memory");
        asm volatile("griddepcontrol.launch_dependents;");
    };
    if (!early) wait_and_release();

    // Issue the first job record (a guess that holds whenever there are at
    // least half as many jobs as clusters) and the job count together, so
    // their latencies overlap.
    const int spec = min(cluster_id / nproj, a.T - 1);
    const int4 spec_job = ld_v4_now(a.jobs + 2 * spec);
    const int4 spec_tok = ld_v4_now(a.jobs + 2 * spec + 1);
    const int n_jobs = ld_s32_now(&a.hdr->n_jobs);
    int E = 1;
    if (MODE != kShrink && n_jobs > 0) {
        E = n_clusters / (n_jobs * nproj);
        E = E < 1 ? 1 : (E > e_max ? e_max : E);
        E = E > kMaxSplit ? kMaxSplit : E;
    }
    // part e of projection p's d_out split starts at 8-column group floor(Go * e / E)
    for (int i = threadIdx.x; i < nproj * (E + 1); i += kThreads) {
        const int pj = i / (E + 1), e = i - pj * (E + 1);
        sm.ebound[pj][e] = (int)((long long)(a.proj[pj].d_out >> 3) * e / E);
    }
    __syncthreads();
    if (n_jobs <= 0) {   // uniform over the grid; no peer traffic has happened
        if (early) wait_and_release();
        cluster_wait();
        return;
    }
    const int upj = nproj * E;   // units per job: (projection, d_out part)
    const int n_units = n_jobs * upj;

    // Cluster exchange of the shrink partials (apply and shrink modes).
    constexpr bool kXchg = MODE != kExpand;

    if (warp == kConsumerWarps) {
        // ------------------------------------------------------------------
        // Producer warp: lane 0 issues the TMA loads of the adapter's pages;
        // the whole warp takes part in the cluster barriers.
        // ------------------------------------------------------------------
        int chunk = 0;
        for (int k = 0, u = cluster_id; u < n_units; ++k, u = unit_of(k, cluster_id, n_clusters)) {
            const int ji = u / upj;
            const int4 job = (ji == spec) ? spec_job : ld_v4_now(a.jobs + 2 * ji);
            const int pj = (NP == 1) ? 0 : (u - ji * upj) / E, e = u - ji * upj - pj * E;
            const SlotMeta m = slot_meta<MODE>(a, sm, staged, pj, job.x);
            const UnitGeom g = unit_geom<MODE>(a, sm, pj, m.np, e, crank);
            const CUtensorMap *tmA = &maps.A[pj], *tmB = &maps.B[pj];
            const CUtensorMap *tmA4 = &maps.A4[pj], *tmB4 = &maps.B4[pj];
            const int d_out = a.proj[pj].d_out;
            // Shrink chunks, then expand chunks, in the order the consumers use
            // them; the ring lets the loads run up to kStages chunks ahead,
            // into the next unit.  Lane 0 arms the stage; lanes 0..15 each issue
            // one page's group of four 64-column blocks (one 3D box, or 2D
            // boxes at the row's end).
            const int cw = g.nb * kBoxCols;
            for (int c = 0; c < g.n_shrink + g.n_expand; ++c) {
                const int s = chunk % kStages;
                mbar_wait(&sm.empty[s], ((chunk / kStages) & 1) ^ 1, sm, a.err);
                const bool shrink = c < g.n_shrink;
                const int c0 = shrink ? g.in0 + c * cw : g.out0 + (c - g.n_shrink) * cw;
                const int c1 = shrink ? g.in1 : g.out1;
                const int boxes = min(g.nb, (c1 - c0 + kBoxCols - 1) / kBoxCols);
                if (lane == 0) mbar_expect_tx(&sm.full[s], (uint32_t)(m.np * boxes * kBoxBytes));
                __syncwarp();
                if (shrink)
                    ptx::issue_page_boxes(lane, sm.stage[s], tmA, tmA4, a.d_in >= 256, a.d_in, m.np, g.nb, boxes, c0,
                                          m.pga, &sm.full[s]);
                else
                    ptx::issue_page_boxes(lane, sm.stage[s], tmB, tmB4, d_out >= 256, d_out, m.np, g.nb, boxes, c0,
                                          m.pgb, &sm.full[s]);
                ++chunk;
            }
            __syncwarp();
        }
        if (lane == 0) {
            // the loads armed last on each stage have landed before this thread exits
            for (int i = (chunk > kStages ? chunk - kStages : 0); i < chunk; ++i)
                drain_wait(&sm.full[i % kStages], (i / kStages) & 1);
        }
        __syncwarp();
        cluster_wait();
        return;
    }

    // ----------------------------------------------------------------------
    // Consumer warps.
    // ----------------------------------------------------------------------
    if (early) wait_and_release();
    const int g8 = lane >> 2, tig = lane & 3;    // MMA fragment coordinates
    const int li = lane & 7, lj = lane >> 3;     // ldmatrix: row within a matrix, matrix index
    int chunk = 0;
    int iter = 0;
    bool joined = false;   // passed the start-up cluster barrier
    for (int u = cluster_id; u < n_units; ++iter, u = unit_of(iter, cluster_id, n_clusters)) {
        const int ji = u / upj;
        const int4 job = (ji == spec) ? spec_job : a.jobs[2 * ji];
        const int4 tk = (ji == spec) ? spec_tok : a.jobs[2 * ji + 1];
        const int pj = (NP == 1) ? 0 : (u - ji * upj) / E, e = u - ji * upj - pj * E;
        const int slot = job.x, n = min(job.y, kMaxJobTokens), q0 = job.z;
        const SlotMeta m = slot_meta<MODE>(a, sm, staged, pj, slot);
        if (m.bad && threadIdx.x == 0 && crank == 0 && e == 0 && a.err) atomicOr(a.err, LORA_DEV_ERR_BAD_PAGE);
        const int r = m.r, np = m.np;
        const UnitGeom g = unit_geom<MODE>(a, sm, pj, np, e, crank);
        float *const Yp = a.proj[pj].Y;
        const int ldy = a.proj[pj].ldy;   // row stride of Y (d_out unless the caller passed a column block)
        const int buf = iter & 1;
        const int cw = g.nb * kBoxCols;
        const int nt = (n + kNTok - 1) / kNTok;   // token tiles of 8
        const int rows = nt * kNTok;
        const int pitch = cw * 2;                   // bytes per token row of a staged X chunk
        if (kXchg && threadIdx.x == 0)   // the peers' partials of this unit: (kCS - 1) * n * r floats
            mbar_expect_tx(&sm.rbar[buf], (uint32_t)((kCS - 1) * n * r * 4));
        // Y is read and written in rows: lane = (token rt of an 8-token tile,
        // 4-column group rc of a 16-column tile), one float4 each.
        const int rt = lane >> 2, rc = lane & 3;
        int rtok[kMaxNTiles];
#pragma unroll
        for (int j = 0; j < kMaxNTiles; ++j) rtok[j] = job_token(a, tk, q0, n, j * kNTok + rt);
        // Old Y of a 16-column tile: token tile 0 one pair of tiles ahead (the
        // warp's first pair of the first expand chunk before the exchange),
        // token tile 1 with its pair.  Each (token, column) belongs to exactly
        // one unit.
        auto load_y = [&](int c0, int mt, int nmt, int j) {
            const int col = c0 + mt * 16 + 4 * rc;
            return (mt < nmt && rtok[j] >= 0 && col < g.out1)
                       ? *reinterpret_cast<const float4 *>(Yp + (size_t)rtok[j] * ldy + col)
                       : make_float4(0.f, 0.f, 0.f, 0.f);
        };
        float4 ya = make_float4(0.f, 0.f, 0.f, 0.f), yb = ya;   // token tile 0 of this tile and the next
        auto load_y0 = [&]() {
            if (g.n_expand > 0) {
                const int nmt0 = (min(cw, g.out1 - g.out0) + 15) >> 4;
                ya = load_y(g.out0, warp, nmt0, 0);
                yb = load_y(g.out0, warp + kConsumerWarps, nmt0, 0);
            }
        };

        if (MODE != kExpand) {
            // ---- shrink: partial sums over this CTA's d_in slice ----
            float acc[kMaxPages][kMaxNTiles][4];
#pragma unroll
            for (int p = 0; p < kMaxPages; ++p)
#pragma unroll
                for (int j = 0; j < kMaxNTiles; ++j)
#pragma unroll
                    for (int i = 0; i < 4; ++i) acc[p][j][i] = 0.f;
            const int gq = cw >> 3;   // 16-byte groups per token row
            auto stage_x = [&](int c) {
                const int c0 = g.in0 + c * cw;
                const uint32_t base = smem_u32(sm.xs[c & 1]);
                for (int i = threadIdx.x; i < rows * gq; i += kConsumers) {
                    const int t = i / gq, q = i - t * gq;
                    const int col = c0 + q * 8;
                    const int tok = (col < g.in1) ? job_token(a, tk, q0, n, t) : -1;
                    const uint16_t *src = tok >= 0 ? a.X + (size_t)tok * a.d_in + col : a.X;
                    cp_async16(base + swz(t, pitch, q), src, tok >= 0 ? 16 : 0);
                }
                cp_async_commit();
            };
            if (g.n_shrink > 0) stage_x(0);
            int kbase = 0;   // 16-column steps of the slice before this chunk
            for (int c = 0; c < g.n_shrink; ++c, ++chunk) {
                const int s = chunk % kStages;
                const int c0 = g.in0 + c * cw;
                const int nks = (min(cw, g.in1 - c0) + 15) >> 4;
                cp_async_wait_all();
                mbar_wait(&sm.full[s], (chunk / kStages) & 1, sm, a.err);
                consumer_sync();   // every thread's X copies of chunk c are in; chunk c-1 is done
                if (c + 1 < g.n_shrink) stage_x(c + 1);
                const uint32_t xb = smem_u32(sm.xs[c & 1]);
                const uint32_t sb = smem_u32(sm.stage[s]);
                int kk = warp - kbase % kConsumerWarps;
                if (kk < 0) kk += kConsumerWarps;
                for (; kk < nks; kk += kConsumerWarps) {
                    // X fragments (B side) of this step for both token tiles
                    uint32_t bx[kMaxNTiles][2];
                    {
                        const int t = (lj >> 1) * kNTok + li;
                        const uint32_t ad = xb + swz(t, pitch, 2 * kk + (lj & 1));
                        if (nt > 1) {
                            uint32_t r4[4];
                            ldsm_x4(ad, r4);
                            bx[0][0] = r4[0]; bx[0][1] = r4[1];
                            bx[kMaxNTiles - 1][0] = r4[2]; bx[kMaxNTiles - 1][1] = r4[3];
                        } else {
                            ldsm_x2(ad, bx[0][0], bx[0][1]);
                        }
                    }
                    const int b = kk >> 2, ks = kk & 3;
#pragma unroll
                    for (int p = 0; p < kMaxPages; ++p) {
                        if (p < np) {
                            uint32_t af[4];
                            const int row = li + 8 * (lj & 1);
                            ldsm_x4(sb + (uint32_t)((p * g.nb + b) * kBoxBytes + row * 128 +
                                                    (((2 * ks + (lj >> 1)) ^ li) << 4)),
                                    af);
                            mma_bf16(acc[p][0], af, bx[0][0], bx[0][1]);
                            if (kMaxNTiles > 1 && nt > 1)
                                mma_bf16(acc[p][kMaxNTiles - 1], af, bx[kMaxNTiles - 1][0], bx[kMaxNTiles - 1][1]);
                        }
                    }
                }
                kbase += nks;
                __syncwarp();
                if (lane == 0) mbar_arrive_relaxed(&sm.empty[s]);
            }
            // the warps' partial sums, added in warp order, become this CTA's
            // partial; it goes to its own slot and into every peer's
            consumer_sync();   // every warp is done with the X buffers
            float *red = reinterpret_cast<float *>(sm.xs);
#pragma unroll
            for (int p = 0; p < kMaxPages; ++p)
#pragma unroll
                for (int j = 0; j < kMaxNTiles; ++j)
                    if (p < np && j < nt)
                        *reinterpret_cast<float4 *>(red + ((warp * kMaxPages + p) * kMaxNTiles + j) * 128 + lane * 4) =
                            make_float4(acc[p][j][0], acc[p][j][1], acc[p][j][2], acc[p][j][3]);
            consumer_sync();
            if (MODE == kApply) load_y0();
            if (!joined) {   // the peers' barriers are initialised
                cluster_wait();
                joined = true;
            }
            float *own = reinterpret_cast<float *>(reinterpret_cast<unsigned char *>(&sm.xs) + kRedBytes);
            const uint32_t own_bar = smem_u32(&sm.rbar[buf]);
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
                    for (int w = 0; w < kConsumerWarps; ++w)
                        sum += red[((w * kMaxPages + p) * kMaxNTiles + j) * 128 + el];
                    const int o = t * LORA_MAX_RANK + k;
                    own[o] = sum;
#pragma unroll
                    for (int d = 1; d < kCS; ++d) {   // into slot (crank - peer - 1) mod kCS = kCS - 1 - d of peer
                        const uint32_t peer = (uint32_t)((crank + d) % kCS);
                        st_async_peer(map_peer(smem_u32(&sm.R[buf][kCS - 1 - d][o]), peer), sum, map_peer(own_bar, peer));
                    }
                }
            }
            mbar_wait(&sm.rbar[buf], (uint32_t)((iter >> 1) & 1), sm, a.err);
            consumer_sync();   // this CTA's own partial is complete too; the warps' sums are read
            // v[t][k] = sum of the CTAs' partials in rank order
            const int nv = n * r;
            for (int idx = threadIdx.x; idx < nv; idx += kConsumers) {
                const int t = idx / r, k = idx - t * r;
                const int o = t * LORA_MAX_RANK + k;
                float v = 0.f;
#pragma unroll
                for (int q = 0; q < kCS; ++q) v += (q == crank) ? own[o] : sm.R[buf][(q - crank - 1 + kCS) % kCS][o];
                if (MODE == kShrink) {
                    if (crank == 0) a.V[(size_t)job_token(a, tk, q0, n, t) * LORA_MAX_RANK + k] = v;
                } else {
                    const uint16_t h = bf16_rn(v);
                    const uint16_t l = bf16_rn(v - __uint_as_float((uint32_t)h << 16));
                    const uint32_t so = swz(t, LORA_MAX_RANK * 2, k >> 3) + (k & 7) * 2;
                    *reinterpret_cast<uint16_t *>(reinterpret_cast<unsigned char *>(&sm.xs) + so) = h;
                    *reinterpret_cast<uint16_t *>(reinterpret_cast<unsigned char *>(&sm.xs) + kVBytes + so) = l;
                }
            }
            if (MODE == kShrink) {
                consumer_sync();
                continue;
            }
        } else {
            load_y0();
            for (int idx = threadIdx.x; idx < n * r; idx += kConsumers) {
                const int t = idx / r, k = idx - t * r;
                const float v = a.V[(size_t)job_token(a, tk, q0, n, t) * LORA_MAX_RANK + k];
                const uint16_t h = bf16_rn(v);
                const uint16_t l = bf16_rn(v - __uint_as_float((uint32_t)h << 16));
                const uint32_t so = swz(t, LORA_MAX_RANK * 2, k >> 3) + (k & 7) * 2;
                *reinterpret_cast<uint16_t *>(reinterpret_cast<unsigned char *>(&sm.xs) + so) = h;
                *reinterpret_cast<uint16_t *>(reinterpret_cast<unsigned char *>(&sm.xs) + kVBytes + so) = l;
            }
        }
        // rank rows past r (up to the page end) and token rows past n of the
        // tiles hold zeros: the weights' padding rows are zero in the pool,
        // and 0 * v must not meet a stale non-finite value
        for (int idx = threadIdx.x; idx < rows * np * LORA_PAGE_ROWS; idx += kConsumers) {
            const int t = idx / (np * LORA_PAGE_ROWS), k = idx - t * (np * LORA_PAGE_ROWS);
            if (t >= n || k >= r) {
                const uint32_t so = swz(t, LORA_MAX_RANK * 2, k >> 3) + (k & 7) * 2;
                *reinterpret_cast<uint16_t *>(reinterpret_cast<unsigned char *>(&sm.xs) + so) = 0;
                *reinterpret_cast<uint16_t *>(reinterpret_cast<unsigned char *>(&sm.xs) + kVBytes + so) = 0;
            }
        }
        consumer_sync();

        // ---- expand-add over this CTA's d_out slice ----
        // v fragments (B side) are read from shared memory per page and token
        // tile: high part (matrices 0, 1) and low part (matrices 2, 3)
        const uint32_t vbase = smem_u32(&sm.xs) + ((lj >> 1) ? kVBytes : 0);
        const float sc = m.scale;
        float *ytile = reinterpret_cast<float *>(reinterpret_cast<unsigned char *>(&sm.xs) + kYTileOff +
                                                 warp * 2 * kYTileBytes);
        for (int c = 0; c < g.n_expand; ++c, ++chunk) {
            const int s = chunk % kStages;
            const int c0 = g.out0 + c * cw;
            const int nmt = (min(cw, g.out1 - c0) + 15) >> 4;
            mbar_wait(&sm.full[s], (chunk / kStages) & 1, sm, a.err);
            const uint32_t sb = smem_u32(sm.stage[s]);
            int mt = warp - (c * (cw >> 4)) % kConsumerWarps;
            if (mt < 0) mt += kConsumerWarps;
            if (c > 0) {
                ya = load_y(c0, mt, nmt, 0);
                yb = load_y(c0, mt + kConsumerWarps, nmt, 0);
            }
            const int krow = li + 8 * (lj >> 1);
            // The warp's tiles are taken in pairs (mt, mt + 15) whose fragment
            // loads and MMAs interleave, so the two dependent chains overlap.
#pragma unroll 1
            for (; mt < nmt; mt += 2 * kConsumerWarps) {
                const int mtB = mt + kConsumerWarps;
                const bool hasB = mtB < nmt;
                // token tile 0 rows of the next pair; token tile 1 rows of this one
                const float4 yc = load_y(c0, mt + 2 * kConsumerWarps, nmt, 0);
                const float4 yd = load_y(c0, mt + 3 * kConsumerWarps, nmt, 0);
                float4 y1[2] = {make_float4(0.f, 0.f, 0.f, 0.f), make_float4(0.f, 0.f, 0.f, 0.f)};
                if (kMaxNTiles > 1 && nt > 1) {
                    y1[0] = load_y(c0, mt, nmt, kMaxNTiles - 1);
                    y1[1] = load_y(c0, mtB, nmt, kMaxNTiles - 1);
                }
                float d[2][kMaxNTiles][4];
#pragma unroll
                for (int h = 0; h < 2; ++h)
#pragma unroll
                    for (int jj = 0; jj < kMaxNTiles; ++jj)
#pragma unroll
                        for (int e2 = 0; e2 < 4; ++e2) d[h][jj][e2] = 0.f;
                const uint32_t offA = (uint32_t)((mt >> 2) * kBoxBytes + krow * 128 + (((2 * (mt & 3) + (lj & 1)) ^ li) << 4));
                const uint32_t offB = (uint32_t)((mtB >> 2) * kBoxBytes + krow * 128 + (((2 * (mtB & 3) + (lj & 1)) ^ li) << 4));
#pragma unroll 1
                for (int p = 0; p < np; ++p) {
                    const uint32_t pb0 = sb + (uint32_t)(p * g.nb * kBoxBytes);
                    uint32_t afA[4], afB[4] = {0u, 0u, 0u, 0u};
                    ldsm_x4_t(pb0 + offA, afA);
                    if (hasB) ldsm_x4_t(pb0 + offB, afB);
#pragma unroll
                    for (int jj = 0; jj < kMaxNTiles; ++jj) {
                        if (jj < nt) {
                            uint32_t bv[4];
                            ldsm_x4(vbase + swz(jj * kNTok + li, LORA_MAX_RANK * 2, 2 * p + (lj & 1)), bv);
                            mma_bf16(d[0][jj], afA, bv[0], bv[1]);
                            if (hasB) mma_bf16(d[1][jj], afB, bv[0], bv[1]);
                            mma_bf16(d[0][jj], afA, bv[2], bv[3]);
                            if (hasB) mma_bf16(d[1][jj], afB, bv[2], bv[3]);
                        }
                    }
                }
                // fragments (column g8 / g8 + 8, tokens 2 tig, 2 tig + 1) -> rows:
                // per tile [token][16 columns], 4-column groups swizzled by token
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    if (h == 0 || hasB) {
#pragma unroll
                        for (int jj = 0; jj < kMaxNTiles; ++jj) {
                            if (jj < nt) {
#pragma unroll
                                for (int e2 = 0; e2 < 4; ++e2) {
                                    const int t = jj * kNTok + 2 * tig + (e2 & 1), cc = g8 + 8 * (e2 >> 1);
                                    ytile[h * (kYTileBytes / 4) + t * 16 + (((cc >> 2) ^ (t & 3)) << 2) + (cc & 3)] =
                                        d[h][jj][e2];
                                }
                            }
                        }
                    }
                }
                __syncwarp();
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int col = c0 + (mt + h * kConsumerWarps) * 16 + 4 * rc;
                    if ((h == 0 || hasB) && col < g.out1) {
#pragma unroll
                        for (int jj = 0; jj < kMaxNTiles; ++jj) {
                            const int t = jj * kNTok + rt;
                            const int tok = rtok[jj];
                            if (jj < nt && tok >= 0) {
                                const float4 dv = *reinterpret_cast<const float4 *>(
                                    ytile + h * (kYTileBytes / 4) + t * 16 + ((rc ^ (t & 3)) << 2));
                                const float4 y = (jj == 0) ? (h == 0 ? ya : yb) : y1[h];
                                *reinterpret_cast<float4 *>(Yp + (size_t)tok * ldy + col) =
                                    make_float4(fmaf(sc, dv.x, y.x), fmaf(sc, dv.y, y.y), fmaf(sc, dv.z, y.z),
                                                fmaf(sc, dv.w, y.w));
                            }
                        }
                    }
                }
                __syncwarp();   // the tiles are rewritten for the next pair
                ya = yc;
                yb = yd;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive_relaxed(&sm.empty[s]);
        }
        consumer_sync();   // v is rewritten by the next unit
    }
    if (!joined) cluster_wait();
}

constexpr size_t kGatherSmemBytes = sizeof(GatherSmem) + 1024;   // + room to align the base to 1 KB
int g_max_clusters[64] = {};

// Occupancy in clusters of the gather kernel (every mode has the same shape).
int max_clusters(int *out) {
    int dev = 0;
    if (int rc = cuda_check(cudaGetDevice(&dev))) return rc;
    if (dev < 0 || dev >= 64) return LORA_ERR_INVALID_ARG;
    if (g_max_clusters[dev] == 0) {
        const void *fns[4] = {(const void *)gather_kernel<kApply, 1>, (const void *)gather_kernel<kShrink, 1>,
                              (const void *)gather_kernel<kExpand, 1>,
                              (const void *)gather_kernel<kApply, LORA_MAX_PROJECTIONS>};
        for (const void *f : fns)
            if (int rc = cuda_check(cudaFuncSetAttribute(f, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                         (int)kGatherSmemBytes)))
                return rc;
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = kCS;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = kGatherSmemBytes;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        cfg.gridDim = dim3(kCS * 256);
        int ncl = 0;
        if (int rc = cuda_check(cudaOccupancyMaxActiveClusters(&ncl, gather_kernel<kApply, 1>, &cfg))) return rc;
        g_max_clusters[dev] = ncl > 0 ? ncl : 1;
    }
    *out = g_max_clusters[dev];
    return LORA_OK;
}

template <int MODE, int NP>
int launch_mode(const GatherArgs &ga, lora_pool_s *const *pa, lora_pool_s *const *pb, cudaStream_t st, bool pdl) {
    if (ga.nproj < 1 || ga.nproj > NP) return LORA_ERR_INVALID_ARG;
    int mcl = 1;
    if (int rc = max_clusters(&mcl)) return rc;
    const size_t smem = kGatherSmemBytes;
    KArgs<NP> a;
    a.X = ga.X; a.V = ga.V; a.T = ga.T; a.d_in = ga.d_in; a.S = ga.S; a.nproj = ga.nproj;
    for (int p = 0; p < NP; ++p) a.proj[p] = ga.proj[p < ga.nproj ? p : 0];
    a.perm = ga.perm; a.jobs = ga.jobs; a.hdr = ga.hdr; a.err = ga.err;
    a.early = (pdl && !plan_was_last_launch(st)) ? 1 : 0;
    GatherMaps<NP> maps;
    int e_max = 1 << 30;
    for (int p = 0; p < a.nproj; ++p) {
        if (MODE != kExpand) {
            if (int rc = pool_tensor_map(pa[p], &maps.A[p])) return rc;
        }
        if (MODE != kShrink) {
            if (int rc = pool_tensor_map(pb[p], &maps.B[p])) return rc;
        }
        if (MODE == kExpand) maps.A[p] = maps.B[p];
        if (MODE == kShrink) maps.B[p] = maps.A[p];
        maps.A4[p] = maps.A[p];
        maps.B4[p] = maps.B[p];
        if (MODE != kExpand && pa[p]->width >= 256) {
            if (int rc = pool_tensor_map4(pa[p], &maps.A4[p])) return rc;
        }
        if (MODE != kShrink && pb[p]->width >= 256) {
            if (int rc = pool_tensor_map4(pb[p], &maps.B4[p])) return rc;
        }
        // a d_out part keeps at least kCS x 8 column groups (8 per CTA)
        const int em = (a.proj[p].d_out >> 3) / (kCS * 8);
        e_max = min(e_max, em < 1 ? 1 : em);
    }
    for (int p = a.nproj; p < NP; ++p) {   // unused slots: valid copies, never read
        maps.A[p] = maps.A[0];
        maps.B[p] = maps.B[0];
        maps.A4[p] = maps.A4[0];
        maps.B4[p] = maps.B4[0];
    }

    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kCS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    long long want = (long long)(a.T > 0 ? a.T : 1) * a.nproj * (MODE == kShrink ? 1 : e_max);
    int ncl = (int)(want < mcl ? want : mcl);
    if (ncl < 1) ncl = 1;
    cfg.gridDim = dim3(kCS * ncl);
    cfg.numAttrs = pdl ? 2 : 1;
    if (int rc = cuda_check(cudaLaunchKernelEx(&cfg, gather_kernel<MODE, NP>, maps, a, e_max))) return rc;
    count_launch();
    note_launch(st, false);
    return LORA_OK;
}

}  // namespace

int gather_clusters(int *out) { return max_clusters(out); }

int launch_gather(GatherMode mode, const GatherArgs &a, lora_pool_s *const *pa, lora_pool_s *const *pb,
                  cudaStream_t st, bool pdl) {
    if (a.nproj > 1) {   // several projections: apply mode only
        if (mode != kApply) return LORA_ERR_INVALID_ARG;
        return launch_mode<kApply, LORA_MAX_PROJECTIONS>(a, pa, pb, st, pdl);
    }
    switch (mode) {
        case kApply: return launch_mode<kApply, 1>(a, pa, pb, st, pdl);
        case kShrink: return launch_mode<kShrink, 1>(a, pa, pb, st, pdl);
        case kExpand: return launch_mode<kExpand, 1>(a, pa, pb, st, pdl);
    }
    return LORA_ERR_INVALID_ARG;
}

}  // namespace lora
