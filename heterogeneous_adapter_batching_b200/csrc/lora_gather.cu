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
// Work unit = one gather job (an adapter slot and up to 8 of its tokens, from
// the plan kernel) times one part e of an E-way split of d_out.  A cluster of
// kCS CTAs runs one unit at a time and loops over the units (persistent grid
// sized from the occupancy of the cluster shape).  Per CTA:
//   * a producer warp streams the unit's rows into a ring of shared-memory
//     stages with bulk asynchronous copies (cp.async.bulk, completion on an
//     mbarrier): first the CTA's 1/kCS slice of d_in (rank rows of A^T from
//     the pages, and the tokens' X rows), then its slice of d_out (rank rows
//     of B, and the tokens' Y rows).  Only the r_i rows the adapter has are
//     copied.  The producer runs ahead into the next unit while the
//     consumers finish the current one, so B and Y are in flight during the
//     shrink;
//   * 8 consumer warps compute the shrink partial sums over the d_in slice
//     (warps take rank rows, lanes take 8-column groups, warp shuffles reduce
//     the lanes) and push them into every peer CTA's shared memory
//     (distributed shared memory stores, then a release arrive on the peer's
//     mbarrier);
//   * each CTA sums the kCS partials in rank order, so all CTAs hold the same
//     fp32 v and the result is bit-reproducible, then expands its d_out slice:
//     threads take columns, read B and the old Y from the stage and store the
//     new Y row segments with coalesced stores.
// Every wait is bounded; a wait that runs out sets LORA_DEV_ERR_TIMEOUT in the
// error word and the kernel runs to completion without trapping.
#include "lora_internal.cuh"

namespace lora {
namespace {

constexpr int kCS = 8;                 // CTAs per cluster
constexpr int kConsumerWarps = 8;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kNT = 4;                 // max tokens per job
constexpr int kStages = 4;
constexpr int kStageBytes = 16384;
constexpr long long kWaitLimit = 2000000000LL;   // cycles (~1 s)

struct __align__(16) GatherSmem {
    unsigned char stage[kStages][kStageBytes];
    float P[2][kCS][kNT * LORA_MAX_RANK];     // partial sums pushed by each peer, [t * r + k]
    float4 v[LORA_MAX_RANK];                  // reduced v, [k] holds tokens 0..3
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

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
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

__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ void consumer_sync() {
    asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
}

__device__ __forceinline__ void bf16x8(const uint4 &v, float f[8]) {
    f[0] = __uint_as_float(v.x << 16); f[1] = __uint_as_float(v.x & 0xffff0000u);
    f[2] = __uint_as_float(v.y << 16); f[3] = __uint_as_float(v.y & 0xffff0000u);
    f[4] = __uint_as_float(v.z << 16); f[5] = __uint_as_float(v.z & 0xffff0000u);
    f[6] = __uint_as_float(v.w << 16); f[7] = __uint_as_float(v.w & 0xffff0000u);
}

// Column ranges, in units of 8 columns (16 bytes of bf16), of the CTA's
// slices and the chunk widths that fit one stage.
struct UnitGeom {
    int r, n;
    int in_g0, in_g1, kw;    // d_in slice [in_g0, in_g1) groups; shrink chunk width in groups
    int out_g0, out_g1, cw;  // d_out slice; expand chunk width in groups
    int n_shrink, n_expand;
};

// The slot's rank for this call, or 0 when the rank or any page it needs is
// out of range (the unit is then skipped: its Y rows stay untouched).  Every
// thread of the CTA evaluates it on the same data, so all agree.
template <int MODE>
__device__ __forceinline__ int checked_rank(const GatherArgs &a, int slot, bool &bad) {
    int r = a.ranks[slot];
    bad = false;
    if (r <= 0) return 0;
    if (r > LORA_MAX_RANK) { bad = true; return 0; }
    const int np = (r + LORA_PAGE_ROWS - 1) / LORA_PAGE_ROWS;
    for (int p = 0; p < np; ++p) {
        if (MODE != kExpand) {
            const int pg = a.pt[slot * 8 + p];
            if (pg < 0 || (long long)(pg + 1) * LORA_PAGE_ROWS > a.rowsA) bad = true;
        }
        if (MODE != kShrink) {
            const int pg = a.pt[slot * 8 + 4 + p];
            if (pg < 0 || (long long)(pg + 1) * LORA_PAGE_ROWS > a.rowsB) bad = true;
        }
    }
    return bad ? 0 : r;
}

template <int MODE>
__device__ __forceinline__ UnitGeom unit_geom(const GatherArgs &a, int r, int n, int e, int E, int crank) {
    UnitGeom g;
    g.r = r;
    g.n = n;
    const int Gi = a.d_in >> 3, Go = a.d_out >> 3;
    g.in_g0 = (int)((long long)Gi * crank / kCS);
    g.in_g1 = (int)((long long)Gi * (crank + 1) / kCS);
    const int ge0 = (int)((long long)Go * e / E), ge1 = (int)((long long)Go * (e + 1) / E);
    g.out_g0 = ge0 + (int)((long long)(ge1 - ge0) * crank / kCS);
    g.out_g1 = ge0 + (int)((long long)(ge1 - ge0) * (crank + 1) / kCS);
    // Chunk widths (in 16-byte column groups) sized for the largest job, so that
    // they depend on the rank only: a token's fp32 summation order is then the
    // same whichever job it lands in, and results do not depend on batch order.
    // Shrink: r + kNT rows of 16 B per group; expand: r rows of 16 B + kNT rows of 32 B.
    g.kw = kStageBytes / ((r + kNT) * 16);
    g.cw = kStageBytes / (r * 16 + kNT * 32);
    const int win = g.in_g1 - g.in_g0, wout = g.out_g1 - g.out_g0;
    g.n_shrink = (MODE == kExpand || win <= 0 || r == 0) ? 0 : (win + g.kw - 1) / g.kw;
    g.n_expand = (MODE == kShrink || wout <= 0 || r == 0) ? 0 : (wout + g.cw - 1) / g.cw;
    return g;
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 2)
gather_kernel(GatherArgs a, int e_max) {
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
        mbar_init(&sm.xbar[0], kCS);
        mbar_init(&sm.xbar[1], kCS);
        sm.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // Peers push into this CTA's barriers only after every CTA initialised them.
    cluster_sync_all();

    // The plan kernel runs just before this one; wait for its output.
    asm volatile("griddepcontrol.wait;" ::: "memory");

    const int n_jobs = a.hdr->n_jobs;
    if (n_jobs <= 0) return;   // uniform over the grid; no peer traffic has happened
    int E = 1;
    if (MODE != kShrink) {
        E = n_clusters / n_jobs;
        E = E < 1 ? 1 : (E > e_max ? e_max : E);
    }
    const int n_units = n_jobs * E;

    if (warp == kConsumerWarps) {
        // ------------------------------------------------------------------
        // Producer warp: bulk copies of row segments into the stage ring.
        // ------------------------------------------------------------------
        int chunk = 0;
        for (int u = cluster_id; u < n_units; u += n_clusters) {
            const int4 job = a.jobs[u / E];
            const int e = u - (u / E) * E;
            const int slot = job.x, p0 = job.y, n = job.z;
            bool bad;
            const int r = checked_rank<MODE>(a, slot, bad);
            const UnitGeom g = unit_geom<MODE>(a, r, n, e, E, crank);
            // shrink chunks: rows of A^T (r) then X (n), each kw groups wide
            for (int c = 0; c < g.n_shrink; ++c, ++chunk) {
                const int s = chunk % kStages;
                const uint32_t par = ((chunk / kStages) & 1) ^ 1;
                const int c0 = g.in_g0 + c * g.kw;
                const int w = min(g.kw, g.in_g1 - c0);
                mbar_wait<false>(&sm.empty[s], par, sm, a.err);
                if (lane == 0) mbar_expect_tx(&sm.full[s], (uint32_t)((r + n) * w * 16));
                __syncwarp();
                for (int i = lane; i < r + n; i += 32) {
                    const uint16_t *src;
                    if (i < r) {
                        const int page = a.pt[slot * 8 + (i >> 4)];
                        src = a.poolA + ((size_t)page * LORA_PAGE_ROWS + (i & 15)) * a.d_in + (size_t)c0 * 8;
                    } else {
                        const int t = i - r;
                        src = a.X + (size_t)a.perm[p0 + t] * a.d_in + (size_t)c0 * 8;
                    }
                    bulk_g2s(sm.stage[s] + (size_t)i * w * 16, src, (uint32_t)(w * 16), &sm.full[s]);
                }
            }
            // expand chunks: rows of B (r, bf16) then Y (n, fp32)
            for (int c = 0; c < g.n_expand; ++c, ++chunk) {
                const int s = chunk % kStages;
                const uint32_t par = ((chunk / kStages) & 1) ^ 1;
                const int c0 = g.out_g0 + c * g.cw;
                const int w = min(g.cw, g.out_g1 - c0);
                mbar_wait<false>(&sm.empty[s], par, sm, a.err);
                if (lane == 0) mbar_expect_tx(&sm.full[s], (uint32_t)((r * 16 + n * 32) * w));
                __syncwarp();
                for (int i = lane; i < r + n; i += 32) {
                    if (i < r) {
                        const int page = a.pt[slot * 8 + 4 + (i >> 4)];
                        const uint16_t *src = a.poolB + ((size_t)page * LORA_PAGE_ROWS + (i & 15)) * a.d_out + (size_t)c0 * 8;
                        bulk_g2s(sm.stage[s] + (size_t)i * w * 16, src, (uint32_t)(w * 16), &sm.full[s]);
                    } else {
                        const int t = i - r;
                        const float *src = a.Y + (size_t)a.perm[p0 + t] * a.d_out + (size_t)c0 * 8;
                        bulk_g2s(sm.stage[s] + (size_t)r * w * 16 + (size_t)t * w * 32, src, (uint32_t)(w * 32),
                                 &sm.full[s]);
                    }
                }
            }
        }
        return;
    }

    // ----------------------------------------------------------------------
    // Consumer warps.
    // ----------------------------------------------------------------------
    int chunk = 0;
    int iter = 0;
    for (int u = cluster_id; u < n_units; u += n_clusters, ++iter) {
        const int4 job = a.jobs[u / E];
        const int e = u - (u / E) * E;
        const int slot = job.x, p0 = job.y, n = job.z;
        bool bad;
        const int r = checked_rank<MODE>(a, slot, bad);
        if (bad && threadIdx.x == 0 && crank == 0 && e == 0 && a.err) atomicOr(a.err, LORA_DEV_ERR_BAD_PAGE);
        const UnitGeom g = unit_geom<MODE>(a, r, n, e, E, crank);
        const int buf = iter & 1;

        if (MODE != kExpand) {
            // ---- shrink: partial sums over this CTA's d_in slice ----
            float acc[8][kNT];
#pragma unroll
            for (int j = 0; j < 8; ++j)
#pragma unroll
                for (int t = 0; t < kNT; ++t) acc[j][t] = 0.f;
            for (int c = 0; c < g.n_shrink; ++c, ++chunk) {
                const int s = chunk % kStages;
                const uint32_t par = (chunk / kStages) & 1;
                const int w = min(g.kw, g.in_g1 - (g.in_g0 + c * g.kw));
                mbar_wait<false>(&sm.full[s], par, sm, a.err);
                const uint4 *rows = reinterpret_cast<const uint4 *>(sm.stage[s]);
                for (int q = lane; q < w; q += 32) {
                    float xf[kNT][8];
#pragma unroll
                    for (int t = 0; t < kNT; ++t)
                        if (t < n) bf16x8(rows[(size_t)(r + t) * w + q], xf[t]);
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const int k = warp + j * kConsumerWarps;
                        if (k < r) {
                            float af[8];
                            bf16x8(rows[(size_t)k * w + q], af);
#pragma unroll
                            for (int t = 0; t < kNT; ++t) {
                                if (t < n) {
                                    float sum = acc[j][t];
#pragma unroll
                                    for (int i = 0; i < 8; ++i) sum = fmaf(af[i], xf[t][i], sum);
                                    acc[j][t] = sum;
                                }
                            }
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&sm.empty[s]);
            }
            // reduce over lanes; lane 0 keeps the warp's sums
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
                            if (lane == 0) sm.P[buf][crank][t * r + k] = x;   // own slot, local copy
                        }
                    }
                }
            }
            consumer_sync();
            // push the partial vector [t * r + k] to every peer's slot `crank`
            const int nv = n * r;
            for (int idx = threadIdx.x; idx < kCS * ((nv + 3) / 4); idx += kConsumerWarps * 32) {
                const int q = idx / ((nv + 3) / 4);
                const int v4 = idx - q * ((nv + 3) / 4);
                if (q == crank) continue;
                const float *srcp = &sm.P[buf][crank][v4 * 4];
                const float4 val = make_float4(srcp[0], v4 * 4 + 1 < nv ? srcp[1] : 0.f,
                                               v4 * 4 + 2 < nv ? srcp[2] : 0.f, v4 * 4 + 3 < nv ? srcp[3] : 0.f);
                st_peer_v4(map_peer(smem_u32(&sm.P[buf][crank][v4 * 4]), (uint32_t)q), val);
            }
            consumer_sync();
            if (threadIdx.x == 0) {
                for (int q = 0; q < kCS; ++q) arrive_peer_release(map_peer(smem_u32(&sm.xbar[buf]), (uint32_t)q));
            }
            mbar_wait<true>(&sm.xbar[buf], (uint32_t)((iter >> 1) & 1), sm, a.err);
            // v[k][t] = sum over peers in rank order
            for (int idx = threadIdx.x; idx < nv; idx += kConsumerWarps * 32) {
                const int t = idx / r, k = idx - t * r;
                float sum = 0.f;
#pragma unroll
                for (int q = 0; q < kCS; ++q) sum += sm.P[buf][q][idx];
                reinterpret_cast<float *>(&sm.v[k])[t] = sum;
            }
            consumer_sync();
            if (MODE == kShrink) {
                if (crank == 0) {
                    for (int idx = threadIdx.x; idx < nv; idx += kConsumerWarps * 32) {
                        const int t = idx / r, k = idx - t * r;
                        a.V[(size_t)a.perm[p0 + t] * LORA_MAX_RANK + k] = reinterpret_cast<const float *>(&sm.v[k])[t];
                    }
                }
                consumer_sync();
                continue;
            }
        } else {
            for (int idx = threadIdx.x; idx < n * r; idx += kConsumerWarps * 32) {
                const int t = idx / r, k = idx - t * r;
                reinterpret_cast<float *>(&sm.v[k])[t] = a.V[(size_t)a.perm[p0 + t] * LORA_MAX_RANK + k];
            }
            consumer_sync();
        }

        // ---- expand-add over this CTA's d_out slice ----
        const float sc = a.scales[slot];
        int tok[kNT];
#pragma unroll
        for (int t = 0; t < kNT; ++t) tok[t] = t < n ? a.perm[p0 + t] : 0;
        for (int c = 0; c < g.n_expand; ++c, ++chunk) {
            const int s = chunk % kStages;
            const uint32_t par = (chunk / kStages) & 1;
            const int c0 = g.out_g0 + c * g.cw;
            const int w = min(g.cw, g.out_g1 - c0);
            mbar_wait<false>(&sm.full[s], par, sm, a.err);
            const uint16_t *Bs = reinterpret_cast<const uint16_t *>(sm.stage[s]);
            const float *Ys = reinterpret_cast<const float *>(sm.stage[s] + (size_t)r * w * 16);
            const int ncol = w * 8;
            for (int col = threadIdx.x; col < ncol; col += kConsumerWarps * 32) {
                float accv[kNT];
#pragma unroll
                for (int t = 0; t < kNT; ++t) accv[t] = 0.f;
#pragma unroll 4
                for (int k = 0; k < r; ++k) {
                    const float b = __uint_as_float((uint32_t)Bs[(size_t)k * ncol + col] << 16);
                    const float4 v0 = sm.v[k];
                    accv[0] = fmaf(v0.x, b, accv[0]); accv[1] = fmaf(v0.y, b, accv[1]);
                    accv[2] = fmaf(v0.z, b, accv[2]); accv[3] = fmaf(v0.w, b, accv[3]);
                }
#pragma unroll
                for (int t = 0; t < kNT; ++t) {
                    if (t < n) {
                        const float y = fmaf(sc, accv[t], Ys[(size_t)t * ncol + col]);
                        a.Y[(size_t)tok[t] * a.d_out + (size_t)c0 * 8 + col] = y;
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.empty[s]);
        }
        consumer_sync();   // sm.v is rewritten by the next unit
    }
}

template <int MODE>
int launch_mode(const GatherArgs &a, cudaStream_t st, bool pdl) {
    static int max_clusters[64] = {};
    int dev = 0;
    if (int rc = cuda_check(cudaGetDevice(&dev))) return rc;
    if (dev < 0 || dev >= 64) return LORA_ERR_INVALID_ARG;
    const size_t smem = sizeof(GatherSmem);

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
    if (int rc = cuda_check(cudaLaunchKernelEx(&cfg, gather_kernel<MODE>, a, e_max))) return rc;
    count_launch();
    return LORA_OK;
}

}  // namespace

int launch_gather(GatherMode mode, const GatherArgs &a, cudaStream_t st, bool pdl) {
    switch (mode) {
        case kApply: return launch_mode<kApply>(a, st, pdl);
        case kShrink: return launch_mode<kShrink>(a, st, pdl);
        case kExpand: return launch_mode<kExpand>(a, st, pdl);
    }
    return LORA_ERR_INVALID_ARG;
}

}  // namespace lora
