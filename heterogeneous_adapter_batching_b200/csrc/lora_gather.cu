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
// Work unit = one gather job (an adapter slot and up to 4 of its tokens, from
// the plan kernel) times one part e of an E-way split of d_out.  A cluster of
// kCS CTAs (one per SM) runs one unit at a time and loops over the units
// (persistent grid sized from the occupancy of the cluster shape).  Per CTA:
//   * a producer warp streams the adapter's pages into a ring of shared-memory
//     stages with 2D TMA loads, one page (16 rank rows) by 256 columns per
//     instruction: first the CTA's 1/kCS slice of d_in (rows of A^T), then its
//     slice of d_out (rows of B).  It runs ahead into the next unit while the
//     consumers finish the current one.  Only the pages the adapter has are
//     read; a rank that is not a multiple of 16 reads the zeroed rows of its
//     last page;
//   * 8 consumer warps read the tokens' X and Y values straight from global
//     memory (coalesced, issued before they wait for the weights), compute the
//     shrink partial sums over the d_in slice (warps take rank rows, lanes take
//     8-column groups, warp shuffles reduce the lanes) and push them into
//     every peer CTA's shared memory (distributed shared memory stores, then a
//     release arrive on the peer's mbarrier);
//   * each CTA sums the kCS partials in rank order, so all CTAs hold the same
//     fp32 v and the result is bit-reproducible, then expands its d_out slice:
//     threads take columns, read B from the stage and store the new Y values
//     with coalesced stores.
// Small page tables (<= 256 slots) are staged in shared memory before the
// kernel waits for the plan, so a unit's metadata costs one global read (the
// job record).  Every wait is bounded; a wait that runs out sets
// LORA_DEV_ERR_TIMEOUT in the error word and the kernel runs to completion
// without trapping.  No cluster multicast is used.
#include "lora_internal.cuh"

namespace lora {
namespace {

constexpr int kCS = 4;                       // CTAs per cluster
constexpr int kConsumerWarps = 8;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32;    // + one producer warp
constexpr int kNT = 4;                       // max tokens per job
constexpr int kStages = 4;
constexpr int kBoxCols = 256;                // TMA box: 16 rows x 256 columns of bf16 = 8 KB
constexpr int kBoxBytes = LORA_PAGE_ROWS * kBoxCols * 2;
constexpr int kStageBoxes = 4;               // a stage holds 4 boxes = 32 KB
constexpr int kTableSlots = 256;             // page tables up to this many slots live in shared memory
constexpr long long kWaitLimit = 2000000000LL;   // cycles (~1 s)

struct __align__(128) GatherSmem {
    unsigned char stage[kStages][kStageBoxes * kBoxBytes];   // box (page p, column block b) at (p * nb + b) * 8 KB
    float P[2][kCS][kNT * LORA_MAX_RANK];     // partial sums pushed by each peer, [t * r + k]
    float4 v[LORA_MAX_RANK];                  // reduced v: v[k] holds tokens 0..3
    uint4 xs[2][kNT][kStageBoxes * kBoxCols / 8];   // the chunk's X columns per token (double-buffered)
    int4 pt[kTableSlots * 2];                 // staged page-table rows (A pages, B pages)
    int ranks[kTableSlots];
    float scales[kTableSlots];
    uint64_t full[kStages];
    uint64_t empty[kStages];
    uint64_t xbar[2];
    int abort;
};

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

__device__ __forceinline__ bool mbar_try_cluster(uint32_t addr, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok) : "r"(addr), "r"(parity) : "memory");
    return ok != 0;
}

// Bounded wait.  On timeout the CTA-wide abort flag is raised (later waits
// return at once) and the error word records it; execution continues so
// that no peer is left waiting for this CTA.
template <bool kCluster>
__device__ __forceinline__ void mbar_wait(uint64_t *bar, uint32_t parity, GatherSmem &sm, int32_t *err) {
    const uint32_t a = smem_u32(bar);
    if (kCluster ? mbar_try_cluster(a, parity) : mbar_try(a, parity)) return;
    const long long t0 = clock64();
    while (!(kCluster ? mbar_try_cluster(a, parity) : mbar_try(a, parity))) {
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

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ void tma_load_box(void *dst, const CUtensorMap *m, int x, int y, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(y), "r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ uint32_t map_peer(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

__device__ __forceinline__ void st_peer_v4(uint32_t addr, float4 v) {
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};"
                 ::"r"(addr), "f"(v.x), "f"(v.y), "f"(v.z), "f"(v.w) : "memory");
}

__device__ __forceinline__ void arrive_peer_release(uint32_t addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(addr) : "memory");
}

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void consumer_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(kConsumers) : "memory");
}

__device__ __forceinline__ void bf16x8(const uint4 &v, float f[8]) {
    f[0] = __uint_as_float(v.x << 16); f[1] = __uint_as_float(v.x & 0xffff0000u);
    f[2] = __uint_as_float(v.y << 16); f[3] = __uint_as_float(v.y & 0xffff0000u);
    f[4] = __uint_as_float(v.z << 16); f[5] = __uint_as_float(v.z & 0xffff0000u);
    f[6] = __uint_as_float(v.w << 16); f[7] = __uint_as_float(v.w & 0xffff0000u);
}

// Per-slot data of this call, from the shared-memory copy when staged.
struct SlotMeta {
    int r;           // rank, or 0 to skip the unit
    int np;          // pages per matrix
    int4 pga, pgb;   // page ids of A^T and B
    float scale;
    bool bad;
};

template <int MODE>
__device__ __forceinline__ SlotMeta slot_meta(const GatherArgs &a, const GatherSmem &sm, bool staged, int slot) {
    SlotMeta m;
    int r;
    if (staged) {
        r = sm.ranks[slot];
        m.pga = sm.pt[2 * slot];
        m.pgb = sm.pt[2 * slot + 1];
        m.scale = sm.scales[slot];
    } else {
        r = a.ranks[slot];
        m.pga = reinterpret_cast<const int4 *>(a.pt)[2 * slot];
        m.pgb = reinterpret_cast<const int4 *>(a.pt)[2 * slot + 1];
        m.scale = (MODE == kShrink) ? 0.f : a.scales[slot];
    }
    m.bad = r > LORA_MAX_RANK;
    if (r <= 0 || m.bad) r = 0;
    const int np = (r + LORA_PAGE_ROWS - 1) / LORA_PAGE_ROWS;
    const int pa[4] = {m.pga.x, m.pga.y, m.pga.z, m.pga.w};
    const int pb[4] = {m.pgb.x, m.pgb.y, m.pgb.z, m.pgb.w};
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        if (p < np) {
            if (MODE != kExpand && (pa[p] < 0 || (long long)(pa[p] + 1) * LORA_PAGE_ROWS > a.rowsA)) m.bad = true;
            if (MODE != kShrink && (pb[p] < 0 || (long long)(pb[p] + 1) * LORA_PAGE_ROWS > a.rowsB)) m.bad = true;
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
    int nb;              // 256-column boxes per chunk (chunk width nb * 256)
    int n_shrink, n_expand;
};

template <int MODE>
__device__ __forceinline__ UnitGeom unit_geom(const GatherArgs &a, int np, int e, int E, int crank) {
    UnitGeom g;
    const int Gi = a.d_in >> 3, Go = a.d_out >> 3;
    g.in0 = 8 * (int)((long long)Gi * crank / kCS);
    g.in1 = 8 * (int)((long long)Gi * (crank + 1) / kCS);
    const int ge0 = (int)((long long)Go * e / E), ge1 = (int)((long long)Go * (e + 1) / E);
    g.out0 = 8 * (ge0 + (int)((long long)(ge1 - ge0) * crank / kCS));
    g.out1 = 8 * (ge0 + (int)((long long)(ge1 - ge0) * (crank + 1) / kCS));
    // As many 256-column boxes per chunk as fit next to the rank's pages: the
    // chunk width depends on the rank only, so a token's fp32 summation order
    // does not depend on which job it lands in.
    g.nb = np > 0 ? kStageBoxes / np : 1;
    const int cw = g.nb * kBoxCols;
    const int win = g.in1 - g.in0, wout = g.out1 - g.out0;
    g.n_shrink = (MODE == kExpand || win <= 0 || np == 0) ? 0 : (win + cw - 1) / cw;
    g.n_expand = (MODE == kShrink || wout <= 0 || np == 0) ? 0 : (wout + cw - 1) / cw;
    return g;
}

__device__ __forceinline__ int4 ld_v4_now(const int4 *p) {
    int4 v;
    asm volatile("ld.global.v4.s32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}
__device__ __forceinline__ int ld_s32_now(const int *p) {
    int v;
    asm volatile("ld.global.s32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

// 8-term dot product summed as a tree (a fixed order, shorter dependency chains).
__device__ __forceinline__ float dot8(const float a[8], const float x[8]) {
    const float p0 = fmaf(a[1], x[1], a[0] * x[0]);
    const float p1 = fmaf(a[3], x[3], a[2] * x[2]);
    const float p2 = fmaf(a[5], x[5], a[4] * x[4]);
    const float p3 = fmaf(a[7], x[7], a[6] * x[6]);
    return (p0 + p1) + (p2 + p3);
}

// One staged chunk of the shrink: this warp's rank rows k = warp + 8 j for
// j < RPW, lanes over the chunk's 8-column groups.
template <int RPW>
__device__ __forceinline__ void shrink_chunk(const unsigned char *st, const uint4 (*xs)[kStageBoxes * kBoxCols / 8],
                                             int ng, int nb, int warp, int lane, int r, int n, float (&acc)[8][kNT]) {
    // tokens in groups of TG: all four at once for few rank rows per warp, two
    // at a time for 8 rows (the rows' values are re-read from shared memory)
    constexpr int TG = RPW >= 8 ? 2 : kNT;
    for (int q = lane; q < ng; q += 32) {
        const int b = (q * 8) / kBoxCols, cb = q * 8 - b * kBoxCols;
#pragma unroll
        for (int t0 = 0; t0 < kNT; t0 += TG) {
            if (t0 >= n) break;
            float xf[TG][8];
#pragma unroll
            for (int t = 0; t < TG; ++t) {
                if (t0 + t < n) bf16x8(xs[t0 + t][q], xf[t]);
                else {
#pragma unroll
                    for (int i = 0; i < 8; ++i) xf[t][i] = 0.f;
                }
            }
#pragma unroll
            for (int j = 0; j < RPW; ++j) {
                const int k = warp + j * kConsumerWarps;
                if (k < r) {
                    float af[8];
                    bf16x8(*reinterpret_cast<const uint4 *>(st + (size_t)((k >> 4) * nb + b) * kBoxBytes +
                                                            (k & 15) * (kBoxCols * 2) + cb * 2),
                           af);
#pragma unroll
                    for (int t = 0; t < TG; ++t) acc[j][t0 + t] += dot8(af, xf[t]);
                }
            }
        }
    }
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
gather_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, GatherArgs a,
              int e_max) {
    extern __shared__ __align__(128) unsigned char smem_raw[];
    GatherSmem &sm = *reinterpret_cast<GatherSmem *>(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int crank = (int)cluster_rank();
    const int cluster_id = blockIdx.x / kCS;
    const int n_clusters = gridDim.x / kCS;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], kConsumerWarps);
        }
        // every consumer warp of every CTA of the cluster arrives once per unit
        mbar_init(&sm.xbar[0], kCS * kConsumerWarps);
        mbar_init(&sm.xbar[1], kCS * kConsumerWarps);
        sm.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // Announce this CTA's barriers to its peers; the matching wait comes just
    // before the first push into a peer.
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");

    // The plan kernel runs before this one; wait for its output.  Then let the
    // next kernel on the stream get its CTAs resident: it reads nothing the
    // kernels write before its own wait, which returns only when this grid has
    // completed.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");

    // Issue the first job record (a guess that holds whenever there are at
    // least half as many jobs as clusters), the job count and the slot tables
    // together, so their latencies overlap.
    const int spec = cluster_id < a.T ? cluster_id : a.T - 1;
    const int4 spec_job = ld_v4_now(a.jobs + 2 * spec);
    const int4 spec_tok = ld_v4_now(a.jobs + 2 * spec + 1);
    const int n_jobs = ld_s32_now(&a.hdr->n_jobs);
    // Small page tables, ranks and scales are staged in shared memory.
    const bool staged = a.S <= kTableSlots;
    if (staged) {
        for (int i = threadIdx.x; i < a.S; i += kThreads) {
            sm.pt[2 * i] = reinterpret_cast<const int4 *>(a.pt)[2 * i];
            sm.pt[2 * i + 1] = reinterpret_cast<const int4 *>(a.pt)[2 * i + 1];
            sm.ranks[i] = a.ranks[i];
            sm.scales[i] = (MODE == kShrink) ? 0.f : a.scales[i];
        }
    }
    __syncthreads();
    if (n_jobs <= 0) return;   // uniform over the grid; no peer traffic has happened
    int E = 1;
    if (MODE != kShrink) {
        E = n_clusters / n_jobs;
        E = E < 1 ? 1 : (E > e_max ? e_max : E);
    }
    const int n_units = n_jobs * E;

    if (warp == kConsumerWarps) {
        // ------------------------------------------------------------------
        // Producer warp (lane 0): TMA loads of the adapter's pages.
        // ------------------------------------------------------------------
        if (lane == 0) {
            int chunk = 0;
            for (int u = cluster_id; u < n_units; u += n_clusters) {
                const int ji = u / E;
                const int4 job = (ji == spec) ? spec_job : a.jobs[2 * ji];
                const int e = u - ji * E;
                const SlotMeta m = slot_meta<MODE>(a, sm, staged, job.x);
                const UnitGeom g = unit_geom<MODE>(a, m.np, e, E, crank);
                const int pa[4] = {m.pga.x, m.pga.y, m.pga.z, m.pga.w};
                const int pb[4] = {m.pgb.x, m.pgb.y, m.pgb.z, m.pgb.w};
                for (int c = 0; c < g.n_shrink + g.n_expand; ++c, ++chunk) {
                    const int s = chunk % kStages;
                    mbar_wait<false>(&sm.empty[s], ((chunk / kStages) & 1) ^ 1, sm, a.err);
                    const bool shrink = c < g.n_shrink;
                    const int c0 = shrink ? g.in0 + c * g.nb * kBoxCols : g.out0 + (c - g.n_shrink) * g.nb * kBoxCols;
                    const int c1 = shrink ? g.in1 : g.out1;
                    const int boxes = min(g.nb, (c1 - c0 + kBoxCols - 1) / kBoxCols);
                    mbar_expect_tx(&sm.full[s], (uint32_t)(m.np * boxes * kBoxBytes));
                    for (int p = 0; p < m.np; ++p)
                        for (int b = 0; b < boxes; ++b)
                            tma_load_box(sm.stage[s] + (size_t)(p * g.nb + b) * kBoxBytes, shrink ? &tmA : &tmB,
                                         c0 + b * kBoxCols, (shrink ? pa[p] : pb[p]) * LORA_PAGE_ROWS, &sm.full[s]);
                }
            }
            // the loads armed last on each stage have landed before this thread exits
            for (int i = (chunk > kStages ? chunk - kStages : 0); i < chunk; ++i)
                drain_wait(&sm.full[i % kStages], (i / kStages) & 1);
        }
        return;
    }

    // ----------------------------------------------------------------------
    // Consumer warps.
    // ----------------------------------------------------------------------
    int chunk = 0;
    int iter = 0;
    bool joined = false;   // waited on the start-up cluster barrier
    for (int u = cluster_id; u < n_units; u += n_clusters, ++iter) {
        const int ji = u / E;
        const int4 job = (ji == spec) ? spec_job : a.jobs[2 * ji];
        const int4 tk = (ji == spec) ? spec_tok : a.jobs[2 * ji + 1];
        const int e = u - ji * E;
        const int slot = job.x, n = job.y;
        const int tok[kNT] = {tk.x, tk.y, tk.z, tk.w};
        const SlotMeta m = slot_meta<MODE>(a, sm, staged, slot);
        if (m.bad && threadIdx.x == 0 && crank == 0 && e == 0 && a.err) atomicOr(a.err, LORA_DEV_ERR_BAD_PAGE);
        const int r = m.r;
        const UnitGeom g = unit_geom<MODE>(a, m.np, e, E, crank);
        const int buf = iter & 1;
        const int cw = g.nb * kBoxCols;
        // old Y of this thread's columns of the first expand chunk, fetched early
        float yv[kStageBoxes][kNT];
        auto load_y = [&](int c0, int wcols) {
#pragma unroll
            for (int i = 0; i < kStageBoxes; ++i) {
                const int col = threadIdx.x + i * kConsumers;
#pragma unroll
                for (int t = 0; t < kNT; ++t)
                    yv[i][t] = (t < n && col < wcols) ? a.Y[(size_t)tok[t] * a.d_out + c0 + col] : 0.f;
            }
        };

        if (MODE != kExpand) {
            // ---- shrink: partial sums over this CTA's d_in slice ----
            float acc[8][kNT];
#pragma unroll
            for (int j = 0; j < 8; ++j)
#pragma unroll
                for (int t = 0; t < kNT; ++t) acc[j][t] = 0.f;
            const int rpw = (r + kConsumerWarps - 1) / kConsumerWarps;
            for (int c = 0; c < g.n_shrink; ++c, ++chunk) {
                const int s = chunk % kStages;
                const int c0 = g.in0 + c * cw;
                const int wcols = min(cw, g.in1 - c0);
                const int ng = wcols >> 3;   // 8-column groups in this chunk
                uint4 (*xs)[kStageBoxes * kBoxCols / 8] = sm.xs[c & 1];
                // stage the tokens' X columns of this chunk (coalesced, before the weights arrive)
                for (int i = threadIdx.x; i < n * ng; i += kConsumers) {
                    const int t = i / ng, q = i - t * ng;
                    xs[t][q] = __ldg(reinterpret_cast<const uint4 *>(a.X + (size_t)tok[t] * a.d_in + c0 + q * 8));
                }
                mbar_wait<false>(&sm.full[s], (chunk / kStages) & 1, sm, a.err);
                consumer_sync();
                const unsigned char *st = sm.stage[s];
                if (rpw <= 1) shrink_chunk<1>(st, xs, ng, g.nb, warp, lane, r, n, acc);
                else if (rpw <= 2) shrink_chunk<2>(st, xs, ng, g.nb, warp, lane, r, n, acc);
                else if (rpw <= 4) shrink_chunk<4>(st, xs, ng, g.nb, warp, lane, r, n, acc);
                else shrink_chunk<8>(st, xs, ng, g.nb, warp, lane, r, n, acc);
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.empty[s]);
            }
            if (MODE == kApply && g.n_expand > 0) load_y(g.out0, min(cw, g.out1 - g.out0));
            if (!joined) {
                asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
                joined = true;
            }
            // reduce over lanes (every lane gets the sum), then lane q stores the
            // value into peer q's slot `crank` and arrives on peer q's barrier
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const int k = warp + j * kConsumerWarps;
                if (k < r) {
#pragma unroll
                    for (int t = 0; t < kNT; ++t) {
                        if (t < n) {
                            float x = acc[j][t];
#pragma unroll
                            for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
                            if (lane < kCS)
                                asm volatile("st.shared::cluster.f32 [%0], %1;"
                                             ::"r"(map_peer(smem_u32(&sm.P[buf][crank][t * r + k]), (uint32_t)lane)),
                                             "f"(x) : "memory");
                        }
                    }
                }
            }
            __syncwarp();
            if (lane < kCS) arrive_peer_release(map_peer(smem_u32(&sm.xbar[buf]), (uint32_t)lane));
            mbar_wait<true>(&sm.xbar[buf], (uint32_t)((iter >> 1) & 1), sm, a.err);
            // v[k][t] = sum over peers in rank order
            const int nv = n * r;
            for (int idx = threadIdx.x; idx < nv; idx += kConsumers) {
                const int t = idx / r, k = idx - t * r;
                float sum = 0.f;
#pragma unroll
                for (int q = 0; q < kCS; ++q) sum += sm.P[buf][q][idx];
                reinterpret_cast<float *>(&sm.v[k])[t] = sum;
            }
            consumer_sync();
            if (MODE == kShrink) {
                if (crank == 0) {
                    for (int idx = threadIdx.x; idx < nv; idx += kConsumers) {
                        const int t = idx / r, k = idx - t * r;
                        a.V[(size_t)tok[t] * LORA_MAX_RANK + k] = reinterpret_cast<const float *>(&sm.v[k])[t];
                    }
                }
                consumer_sync();
                continue;
            }
        } else {
            for (int idx = threadIdx.x; idx < n * r; idx += kConsumers) {
                const int t = idx / r, k = idx - t * r;
                reinterpret_cast<float *>(&sm.v[k])[t] = a.V[(size_t)tok[t] * LORA_MAX_RANK + k];
            }
            if (g.n_expand > 0) load_y(g.out0, min(cw, g.out1 - g.out0));
            consumer_sync();
        }

        // ---- expand-add over this CTA's d_out slice ----
        const float sc = m.scale;
        for (int c = 0; c < g.n_expand; ++c, ++chunk) {
            const int s = chunk % kStages;
            const int c0 = g.out0 + c * cw;
            const int wcols = min(cw, g.out1 - c0);
            if (c > 0) load_y(c0, wcols);   // the first chunk's Y was fetched before the exchange
            mbar_wait<false>(&sm.full[s], (chunk / kStages) & 1, sm, a.err);
            const unsigned char *st = sm.stage[s];
#pragma unroll
            for (int i = 0; i < kStageBoxes; ++i) {
                const int col = threadIdx.x + i * kConsumers;
                if (col < wcols) {
                    const int b = col / kBoxCols, cb = col - b * kBoxCols;
                    float accv[kNT];
#pragma unroll
                    for (int t = 0; t < kNT; ++t) accv[t] = 0.f;
#pragma unroll 4
                    for (int k = 0; k < r; ++k) {
                        const uint16_t braw = *reinterpret_cast<const uint16_t *>(
                            st + (size_t)((k >> 4) * g.nb + b) * kBoxBytes + (k & 15) * (kBoxCols * 2) + cb * 2);
                        const float bk = __uint_as_float((uint32_t)braw << 16);
                        const float4 v0 = sm.v[k];
                        accv[0] = fmaf(v0.x, bk, accv[0]); accv[1] = fmaf(v0.y, bk, accv[1]);
                        accv[2] = fmaf(v0.z, bk, accv[2]); accv[3] = fmaf(v0.w, bk, accv[3]);
                    }
#pragma unroll
                    for (int t = 0; t < kNT; ++t)
                        if (t < n) a.Y[(size_t)tok[t] * a.d_out + c0 + col] = fmaf(sc, accv[t], yv[i][t]);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.empty[s]);
        }
        consumer_sync();   // sm.v is rewritten by the next unit
    }
    if (!joined) asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

template <int MODE>
int launch_mode(const GatherArgs &a, lora_pool_s *pa, lora_pool_s *pb, cudaStream_t st, bool pdl) {
    static int max_clusters[64] = {};
    int dev = 0;
    if (int rc = cuda_check(cudaGetDevice(&dev))) return rc;
    if (dev < 0 || dev >= 64) return LORA_ERR_INVALID_ARG;
    const size_t smem = sizeof(GatherSmem);
    CUtensorMap ma, mb;
    if (MODE != kExpand) {
        if (int rc = pool_tensor_map(pa, kPoolMapGather, &ma)) return rc;
    }
    if (MODE != kShrink) {
        if (int rc = pool_tensor_map(pb, kPoolMapGather, &mb)) return rc;
    }
    if (MODE == kExpand) ma = mb;
    if (MODE == kShrink) mb = ma;

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
    if (max_clusters[dev] == 0) {
        if (int rc = cuda_check(cudaFuncSetAttribute(gather_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                     (int)smem)))
            return rc;
        int ncl = 0;
        cfg.gridDim = dim3(kCS * 256);
        if (int rc = cuda_check(cudaOccupancyMaxActiveClusters(&ncl, gather_kernel<MODE>, &cfg))) return rc;
        max_clusters[dev] = ncl > 0 ? ncl : 1;
    }
    const int G = a.d_out >> 3;
    int e_max = G / (kCS * 8);
    if (e_max < 1) e_max = 1;
    long long want = (long long)(a.T > 0 ? a.T : 1) * (MODE == kShrink ? 1 : e_max);
    int ncl = (int)(want < max_clusters[dev] ? want : max_clusters[dev]);
    if (ncl < 1) ncl = 1;
    cfg.gridDim = dim3(kCS * ncl);
    cfg.numAttrs = pdl ? 2 : 1;
    if (int rc = cuda_check(cudaLaunchKernelEx(&cfg, gather_kernel<MODE>, ma, mb, a, e_max))) return rc;
    count_launch();
    return LORA_OK;
}

}  // namespace

int launch_gather(GatherMode mode, const GatherArgs &a, lora_pool_s *pa, lora_pool_s *pb, cudaStream_t st, bool pdl) {
    switch (mode) {
        case kApply: return launch_mode<kApply>(a, pa, pb, st, pdl);
        case kShrink: return launch_mode<kShrink>(a, pa, pb, st, pdl);
        case kExpand: return launch_mode<kExpand>(a, pa, pb, st, pdl);
    }
    return LORA_ERR_INVALID_ARG;
}

}  // namespace lora
