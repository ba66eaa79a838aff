// Tensor-core path for long contiguous segments (prefill).
//
// Page "Multi-LoRA Serving in Production" (llms.blog), section "Multi-Size
// Batched Gather Kernels (MBGMV and MBGMM)": in prefill a sequence brings a
// variable-length chunk of tokens that all use one adapter, and the kernel
// indexes that adapter's rank-specific weights dynamically.  Section
// "Segmented Gather Matrix-Vector Multiplication (SGMV)": shrink v = x A on
// the tensor cores, then expand v B scaled by alpha/r into the base output.
//
// Work: a tile is up to 128 consecutive tokens of one run (from the plan
// kernel); an item is one tile times one projection (a launch may cover up to
// 8 projections that read the same X) times one 64-column n-tile of that
// projection's d_out.  Every CTA (one per SM) takes an equal contiguous share
// of the items in (tile, projection, n-tile) order and works through it as
// units of one (tile, projection) each, recomputing the small shrink of a
// unit whose items it shares with a neighbour.  Warp-specialised:
//   warp 0     TMA producer of the shrink operands: X tile [128 x 64] and the
//              adapter's A^T pages [16 x 64] per page, 128-byte swizzled;
//   warp 1     TMA producer of the expand operands: B pages [16 x 64] of the
//              current 64-column n-tile and the Y tile [128 x 64] fp32;
//   warp 2     allocates tensor memory and issues tcgen05.mma:
//                shrink  D1[128 x N1] = X[128 x d_in] A[d_in x N1]   (N1 = r rounded up to 16)
//                expand  D2[128 x 64] = Vhi[128 x N1] B[N1 x 64] + Vlo[128 x N1] B[N1 x 64]
//                        (B read MN-major)
//   warps 4-7  epilogue: read D1 from tensor memory, split v into a bf16 high
//              part and a bf16 low part in two swizzled shared tiles (the A
//              operands of the expand's two products), then per
//              n-tile read D2, add s * D2 to the Y tile and write it back with
//              a TMA store (or row stores for a tile with fewer than 128 tokens).
// Pages hold 16 rank-rows; ranks that are not a multiple of 16 read the
// zero-filled rows of their last page, so padding exists only inside the
// page and in shared memory, never in the pool.  Every mbarrier wait is
// bounded (LORA_DEV_ERR_TIMEOUT).  No cluster multicast is used.
#include <cuda.h>
#include <cuda_bf16.h>

#include "lora_internal.cuh"

namespace lora {
namespace {

constexpr int kM = 128;              // tokens per tile (MMA M)
constexpr int kKB = 64;              // shrink K block: one 128-byte swizzle row of bf16
constexpr int kNB = 64;              // expand n-tile width (MMA N)
constexpr int kStages = 3;           // shrink pipeline depth
constexpr int kThreads = 256;
constexpr long long kWaitLimit = 2000000000LL;

// Launch modes.  kFused: one kernel does a unit's shrink and its expand (any
// number of projections).  kShrinkQ + kExpandV: the shrink of every (tile,
// quarter of d_in) once, into fp32 partials in the workspace, then a kernel
// that only streams B and Y and rebuilds v from the partials (one projection).
constexpr int kFused = 0, kShrinkQ = 1, kExpandV = 2;
constexpr int kSlicesQ = 4;          // d_in quarters of the shrink-only launch

// Shared memory of a mode: STAGES shrink stages, BUF expand buffers (B
// n-tile, its accumulator, the Y tile).  Every array is a whole number of KB,
// so each starts 1024-byte aligned as the 128-byte swizzle needs.
template <int STAGES, int BUF>
struct TileSmemT {
    static constexpr int kBufN = BUF;
    static constexpr int kStageN = STAGES;
    __nv_bfloat16 xs[STAGES][kM * kKB];       // 16 KB each, K-major SW128
    __nv_bfloat16 as[STAGES][64 * kKB];       //  8 KB each, up to 4 pages x 16 rows
    __nv_bfloat16 vs[kM * 64];                // 16 KB, v high part (expand A operand), K-major SW128
    __nv_bfloat16 vl[kM * 64];                // 16 KB, v low part (v - high), same layout
    __nv_bfloat16 bs[BUF][64 * kNB];          //  8 KB each, B n-tile, rank rows x 64 cols (MN-major SW128)
    float ys[BUF][kM * kNB];                  // 32 KB each, two SW128 boxes of [128 rows x 32 cols]
    uint64_t full[STAGES], empty[STAGES];
    uint64_t bfull[BUF], bempty[BUF], yfull[BUF], yempty[BUF], accfull[BUF], accempty[BUF];
    uint64_t shrink_done, d1_empty, v_ready, v_full, v_empty, mma_drain;
    uint32_t tmem_base;
    int reduce;   // kShrinkQ: this CTA finishes the current tile's v
    int abort;
};

template <int MODE>
struct SmemOf {
    using type = TileSmemT<MODE == kExpandV ? 1 : (MODE == kShrinkQ ? 6 : kStages), MODE == kShrinkQ ? 1 : (MODE == kExpandV ? 4 : 3)>;
};
// Tensor-memory columns: the shrink's D1 of quarter q at [64 q, 64 q + 64);
// expand accumulator b at
// [kAccCol + 64 b, kAccCol + 64 b + 64).
constexpr int kAccCol = 64 * kSlicesQ;
template <int MODE>
constexpr uint32_t tmem_cols() { return MODE == kShrinkQ ? 256u : 512u; }

static_assert(sizeof(SmemOf<kFused>::type) + 1024 <= 227 * 1024, "tiles kernel: shared memory beyond the per-block limit");
static_assert(sizeof(SmemOf<kShrinkQ>::type) + 1024 <= 227 * 1024, "tiles kernel: shared memory beyond the per-block limit");
static_assert(sizeof(SmemOf<kExpandV>::type) + 1024 <= 227 * 1024, "tiles kernel: shared memory beyond the per-block limit");
static_assert(kAccCol + 64 * SmemOf<kExpandV>::type::kBufN <= (int)tmem_cols<kExpandV>() &&
              kAccCol + 64 * SmemOf<kFused>::type::kBufN <= (int)tmem_cols<kFused>(), "accumulators beyond the allocation");

__device__ __forceinline__ uint32_t su32(const void *p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }

__device__ __forceinline__ void mbar_init(uint64_t *b, uint32_t n) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(su32(b)), "r"(n));
}
__device__ __forceinline__ bool mbar_try(uint32_t a, uint32_t par) {
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(a), "r"(par) : "memory");
    return ok != 0;
}
// Bounded wait: true when the phase completed.  On timeout it raises the
// CTA's abort flag and records LORA_DEV_ERR_TIMEOUT; once the flag is up every
// wait returns false at once and each role stops issuing work.
template <class Sm>
__device__ __forceinline__ bool mbar_wait(uint64_t *b, uint32_t par, Sm &sm, int32_t *err) {
    const uint32_t a = su32(b);
    if (mbar_try(a, par)) return true;
    const long long t0 = clock64();
    while (!mbar_try(a, par)) {
        if (*(volatile int *)&sm.abort) return false;
        if (clock64() - t0 > kWaitLimit) {
            *(volatile int *)&sm.abort = 1;
            if (err) atomicOr(err, LORA_DEV_ERR_TIMEOUT);
            return false;
        }
    }
    return true;
}
// Drain wait for this thread's own asynchronous operations before the CTA
// exits: bounded, and not cut short by the abort flag.
__device__ __forceinline__ void drain_wait(uint64_t *b, uint32_t par) {
    const uint32_t a = su32(b);
    const long long t0 = clock64();
    while (!mbar_try(a, par) && clock64() - t0 < kWaitLimit / 8) {
    }
}
// A plan field read through L2 (the plan may come from a kernel before the one ahead).
__device__ __forceinline__ int ld_l2(const int *p) {
    int v;
    asm volatile("ld.global.cg.s32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}
template <class Sm>
__device__ __forceinline__ bool aborted(const Sm &sm) { return *(volatile const int *)&sm.abort != 0; }
__device__ __forceinline__ void mbar_arrive(uint64_t *b) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(su32(b)) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t *b, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(su32(b)), "r"(bytes) : "memory");
}

__device__ __forceinline__ void tma_load(void *dst, const CUtensorMap *m, int x, int y, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(su32(dst)), "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(y), "r"(su32(bar)) : "memory");
}
__device__ __forceinline__ void tma_store(const CUtensorMap *m, int x, int y, const void *src) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%1, %2}], [%3];"
                 ::"l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(y), "r"(su32(src)) : "memory");
}

// tcgen05 shared-memory matrix descriptor, 128-byte swizzle (layout type 2),
// descriptor version 1, base offset 0 (atoms are 1024-byte aligned).
__device__ __forceinline__ uint64_t sdesc(const void *p, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((su32(p) >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

// Instruction descriptor of kind::f16: bf16 x bf16 -> fp32.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int a_mn, int b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "r"(acc));
}
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(su32(bar)) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

#define TMEM_LD16(taddr, r)                                                                                   \
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];" \
                 : "=f"(r[0]), "=f"(r[1]), "=f"(r[2]), "=f"(r[3]), "=f"(r[4]), "=f"(r[5]), "=f"(r[6]), "=f"(r[7]),     \
                   "=f"(r[8]), "=f"(r[9]), "=f"(r[10]), "=f"(r[11]), "=f"(r[12]), "=f"(r[13]), "=f"(r[14]), "=f"(r[15]) \
                 : "r"(taddr))
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
// AND of `ok` over the 128 epilogue threads (a barrier too): every epilogue
// thread takes the same branch after a wait that may have been cut short.
__device__ __forceinline__ bool epi_all(bool ok) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 q, %1, 0;\n\t"
        "bar.red.and.pred p, 2, 128, q;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(r) : "r"((uint32_t)ok) : "memory");
    return r != 0;
}

// One projection of a launch, as the kernel sees it.
struct KTileProj {
    float *Y;
    int d_out;
    const int32_t *ranks;
    const float *scales;
    const int32_t *pt;
    long long rowsA;     // rows in the A pool (pages * 16)
    long long rowsB;     // rows in the B pool
};

template <int NP>
struct KTile {
    const uint16_t *X;
    int T, d_in;
    int nproj;
    KTileProj proj[NP];
    int jpre[NP + 1];    // n-tiles of the projections before p, within one tile
    int4 *tiles;         // the plan's tiles; kShrinkQ counts a tile's finished quarters in .w (0 between launches)
    const PlanHeader *hdr;
    int32_t *err;
    float *vpart;        // kShrinkQ / kExpandV: [kSlicesQ][T][LORA_MAX_RANK] fp32 partials of v; the finished
                         // v of row t as bf16 high part, low part in the first 256 bytes of quarter 0's row t
};

template <int NP>
struct TileMaps {
    CUtensorMap V;       // kExpandV: quarter 0 of the partials seen as bf16 [T][128] (v high | v low), SW128 boxes
    CUtensorMap X;
    CUtensorMap A[NP];
    CUtensorMap B[NP];
    CUtensorMap Y[NP];
};

struct UnitInfo {
    int tile;
    int slot, row0, ntok, r, n1, np, j0, j1;
    int p;       // projection
    bool skip;
    bool bad;    // rank above 64 or a page outside its pool (LORA_DEV_ERR_BAD_PAGE); rank 0 is not bad
};

template <int NP>
__device__ __forceinline__ UnitInfo unit_info(const KTile<NP> &a, int tile, int pj, int j0, int j1) {
    UnitInfo ui;
    const int4 t = a.tiles[tile];
    const KTileProj &pr = a.proj[pj];
    ui.tile = tile;
    ui.slot = t.x;
    ui.row0 = t.y;
    ui.ntok = t.z;
    ui.j0 = j0;
    ui.j1 = j1;
    ui.p = pj;
    int r = pr.ranks[ui.slot];
    bool bad = r > LORA_MAX_RANK;
    const int np = (bad || r <= 0) ? 0 : (r + 15) >> 4;
    for (int p = 0; p < np; ++p) {
        const int pa = pr.pt[ui.slot * 8 + p], pb = pr.pt[ui.slot * 8 + 4 + p];
        if (pa < 0 || (long long)(pa + 1) * LORA_PAGE_ROWS > pr.rowsA) bad = true;
        if (pb < 0 || (long long)(pb + 1) * LORA_PAGE_ROWS > pr.rowsB) bad = true;
    }
    ui.bad = bad;
    bad = bad || r <= 0;
    ui.skip = bad || ui.j0 >= ui.j1;
    ui.r = bad ? 0 : r;
    ui.np = bad ? 0 : np;
    ui.n1 = ui.np * 16;
    return ui;
}

// Items are (tile, projection, 64-column n-tile) in that order; every CTA
// takes an equal contiguous share and walks it as units of one (tile,
// projection) each, so a CTA's consecutive units read the same X tile (the
// second and later projections find it in L2).  A CTA whose share starts or
// ends inside a unit recomputes that unit's (small) shrink.  Even CTAs walk
// their share forward and odd CTAs backward, so the two CTAs that share a
// unit reach it at the same time (both first, or both last) and the second
// reader of its X rows and adapter pages finds them in L2.
struct UnitIter {
    long long lo, hi;   // items not yet walked
    int nj;             // items per tile (all projections)
    bool back;
};

__device__ __forceinline__ UnitIter unit_range(int n_tiles, int nj) {
    UnitIter u;
    const long long total = (long long)n_tiles * nj;
    u.lo = total * blockIdx.x / gridDim.x;
    u.hi = total * (blockIdx.x + 1) / gridDim.x;
    u.nj = nj;
    u.back = (blockIdx.x & 1) != 0;
    return u;
}

template <int NP>
__device__ __forceinline__ int proj_of(const KTile<NP> &a, int off) {
    int pj = 0;
#pragma unroll
    for (int q = 1; q < NP; ++q)
        if (q < a.nproj && off >= a.jpre[q]) pj = q;
    return pj;
}

template <int NP>
__device__ __forceinline__ bool next_unit(const KTile<NP> &a, UnitIter &u, UnitInfo &ui) {
    if (u.lo >= u.hi) return false;
    int tile, pj, j0, j1;
    if (!u.back) {
        tile = (int)(u.lo / u.nj);
        const int off = (int)(u.lo - (long long)tile * u.nj);
        pj = proj_of(a, off);
        j0 = off - a.jpre[pj];
        j1 = (int)min((long long)(a.jpre[pj + 1] - a.jpre[pj]), j0 + (u.hi - u.lo));
        u.lo += j1 - j0;
    } else {
        tile = (int)((u.hi - 1) / u.nj);
        const long long ts = (long long)tile * u.nj;
        const int off = (int)(u.hi - 1 - ts);
        pj = proj_of(a, off);
        const long long us = ts + a.jpre[pj];
        const long long st = u.lo > us ? u.lo : us;
        j0 = (int)(st - us);
        j1 = off - a.jpre[pj] + 1;
        u.hi = st;
    }
    ui = unit_info(a, tile, pj, j0, j1);
    return true;
}

// Units of the shrink-only launch: (tile, quarter q of the K blocks), in
// that order; every CTA takes an equal contiguous range, so a CTA mostly
// holds all four quarters of its tiles and the reductions that finish the
// tiles (done by whichever CTA completes a tile's last quarter) spread evenly
// instead of piling up on CTAs that fell behind.  Quarter q covers K blocks
// [nkb q / 4, nkb (q + 1) / 4); with fewer than four K blocks some quarters
// are empty and hold no partial.
__device__ __forceinline__ void quarter_blocks(int nkb, int q, int &kb0, int &kb1) {
    kb0 = nkb * q / kSlicesQ;
    kb1 = nkb * (q + 1) / kSlicesQ;
}

struct QIter {
    int u0, u, u1;   // start of this CTA's range, next unit, end of the range
};

__device__ __forceinline__ QIter qunit_range(int n_tiles) {
    const long long total = (long long)n_tiles * kSlicesQ;
    QIter it;
    it.u0 = it.u = (int)(total * blockIdx.x / gridDim.x);
    it.u1 = (int)(total * (blockIdx.x + 1) / gridDim.x);
    return it;
}

template <int NP>
__device__ __forceinline__ bool next_qunit(const KTile<NP> &a, QIter &it, UnitInfo &ui, int &q) {
    if (it.u >= it.u1) return false;
    const int tile = it.u / kSlicesQ;
    q = it.u - tile * kSlicesQ;
    ui = unit_info(a, tile, 0, 0, 1);
    ++it.u;
    return true;
}

template <int NP, int MODE>
__global__ void __launch_bounds__(kThreads, 1)
tiles_kernel(const __grid_constant__ TileMaps<NP> maps, const __grid_constant__ KTile<NP> a) {
    using Sm = typename SmemOf<MODE>::type;
    constexpr int kBuf = Sm::kBufN;
    constexpr int kSt = Sm::kStageN;
    extern __shared__ unsigned char smem_raw[];
    Sm &sm = *reinterpret_cast<Sm *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // Fetch this launch's parameters and tensor maps while the previous
    // kernel drains.
    const int nproj = NP == 1 ? 1 : a.nproj;
    if (threadIdx.x == 0) {
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.X)) : "memory");
        if (MODE == kExpandV) asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&maps.V)) : "memory");
    }
    if (threadIdx.x >= 32 && threadIdx.x < 32 + 3 * nproj) {
        const int i = threadIdx.x - 32, q = i / 3;
        const CUtensorMap *m = (i % 3 == 0) ? &maps.A[q] : (i % 3 == 1) ? &maps.B[q] : &maps.Y[q];
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
    }
    asm volatile("" ::"l"(a.X), "r"(a.T), "r"(a.d_in), "l"(a.tiles), "l"(a.hdr), "l"(a.err));
    // The kernels before this one on the stream produce the plan (and, for
    // kExpandV, v).  The shrink launch lets its dependent (the expand launch)
    // get resident once it has waited.  In the expand launch only the producer
    // waits, after it has issued its first unit's B and Y loads and before it
    // loads v: when it starts, every kernel before the shrink launch, the plan
    // included, has completed (the shrink launch released it only after its
    // own wait), and the shrink launch writes nothing else it reads.  A batch
    // without long runs has no tiles: leave (after waiting) before touching
    // tensor memory.
    if (MODE != kExpandV) {
        asm volatile("griddepcontrol.wait;" ::: "memory");
        if (MODE == kShrinkQ) asm volatile("griddepcontrol.launch_dependents;");
    }
    const int n_tiles = ld_l2(&a.hdr->n_tiles);
    if (n_tiles <= 0) {   // uniform over the grid
        if (MODE == kExpandV) asm volatile("griddepcontrol.wait;" ::: "memory");
        return;
    }

    if (threadIdx.x == 0) {
        for (int s = 0; s < kSt; ++s) { mbar_init(&sm.full[s], 1); mbar_init(&sm.empty[s], 1); }
        for (int b = 0; b < kBuf; ++b) {
            mbar_init(&sm.bfull[b], 1); mbar_init(&sm.bempty[b], 1);
            mbar_init(&sm.yfull[b], 1); mbar_init(&sm.yempty[b], 1);
            mbar_init(&sm.accfull[b], 1); mbar_init(&sm.accempty[b], 128);
        }
        mbar_init(&sm.shrink_done, 1);
        mbar_init(&sm.d1_empty, 128);
        mbar_init(&sm.v_ready, 128);
        mbar_init(&sm.v_full, 1);
        mbar_init(&sm.v_empty, 1);
        mbar_init(&sm.mma_drain, 1);
        sm.abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 2) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(su32(&sm.tmem_base)),
                     "r"(tmem_cols<MODE>()));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem_base;

    const int nj = a.jpre[nproj];     // items per tile over all projections
    const int nkb = (a.d_in + kKB - 1) / kKB;
    int nq = 0;                       // quarters of d_in that hold K blocks
    for (int q = 0; q < kSlicesQ; ++q) {
        int kb0, kb1;
        quarter_blocks(nkb, q, kb0, kb1);
        nq += kb1 > kb0;
    }

    if (warp == 0 && lane == 0) {
        // ---------------- shrink operand producer ----------------
        int it = 0;
        auto load_kblocks = [&](const UnitInfo &ui, int kb0, int kb1) {
            int pg[4];
            const int32_t *pt = a.proj[ui.p].pt;
            for (int p = 0; p < 4; ++p) pg[p] = p < ui.np ? pt[ui.slot * 8 + p] : 0;
            const CUtensorMap *tmA = &maps.A[ui.p];
            for (int kb = kb0; kb < kb1; ++kb, ++it) {
                const int s = it % kSt;
                if (!mbar_wait(&sm.empty[s], ((it / kSt) & 1) ^ 1, sm, a.err)) return false;
                mbar_expect_tx(&sm.full[s], (uint32_t)(kM * kKB * 2 + ui.np * 16 * kKB * 2));
                tma_load(sm.xs[s], &maps.X, kb * kKB, ui.row0, &sm.full[s]);
                for (int p = 0; p < ui.np; ++p)
                    tma_load(&sm.as[s][p * 16 * kKB], tmA, kb * kKB, pg[p] * LORA_PAGE_ROWS, &sm.full[s]);
            }
            return true;
        };
        if constexpr (MODE == kFused) {
            UnitIter ur = unit_range(n_tiles, nj);
            UnitInfo ui;
            while (next_unit(a, ur, ui) && !aborted(sm)) {
                if (ui.bad && a.err) atomicOr(a.err, LORA_DEV_ERR_BAD_PAGE);
                if (ui.skip) continue;
                if (!load_kblocks(ui, 0, nkb)) break;
            }
        } else if constexpr (MODE == kShrinkQ) {
            QIter u = qunit_range(n_tiles);
            int q = 0, kb0, kb1;
            UnitInfo ui;
            while (next_qunit(a, u, ui, q) && !aborted(sm)) {
                if (ui.bad && q == 0 && a.err) atomicOr(a.err, LORA_DEV_ERR_BAD_PAGE);
                quarter_blocks(nkb, q, kb0, kb1);
                if (ui.skip || kb1 <= kb0) continue;
                if (!load_kblocks(ui, kb0, kb1)) break;
            }
        }
        // the loads this thread armed last on each stage have landed before exit
        for (int i = (it > kSt ? it - kSt : 0); i < it; ++i) drain_wait(&sm.full[i % kSt], (i / kSt) & 1);
    } else if (warp == 1 && lane == 0) {
        // ---------------- expand operand producer: v (kExpandV), B and Y ----------------
        if constexpr (MODE != kShrinkQ) {
            int it = 0, itv = 0;
            bool waited = MODE != kExpandV;
            UnitIter ur = unit_range(n_tiles, nj);
            UnitInfo ui;
            // kExpandV: the unit's v, high and low part, straight into the MMA's
            // operand tiles (the first one after waiting for the shrink launch)
            bool v_done = true;
            auto issue_v = [&]() {
                if (!waited) {
                    asm volatile("griddepcontrol.wait;" ::: "memory");
                    waited = true;
                }
                if (!mbar_wait(&sm.v_empty, (itv & 1) ^ 1, sm, a.err)) return false;
                mbar_expect_tx(&sm.v_full, (uint32_t)(2 * kM * 64 * 2));
                tma_load(sm.vs, &maps.V, 0, ui.row0, &sm.v_full);
                tma_load(sm.vl, &maps.V, 64, ui.row0, &sm.v_full);
                ++itv;
                v_done = true;
                return true;
            };
            bool ok = true;
            while (ok && next_unit(a, ur, ui) && !aborted(sm)) {
                if constexpr (MODE == kExpandV)
                    if (ui.bad && a.err) atomicOr(a.err, LORA_DEV_ERR_BAD_PAGE);
                if (ui.skip) continue;
                if constexpr (MODE == kExpandV) {
                    v_done = false;
                    if (waited && !issue_v()) break;
                }
                int pg[4];
                const int32_t *pt = a.proj[ui.p].pt;
                for (int p = 0; p < 4; ++p) pg[p] = p < ui.np ? pt[ui.slot * 8 + 4 + p] : 0;
                const CUtensorMap *tmB = &maps.B[ui.p], *tmY = &maps.Y[ui.p];
                for (int j = ui.j0; j < ui.j1; ++j, ++it) {
                    // the first unit's first kBuf items need nothing from the shrink launch
                    if (!v_done && j - ui.j0 == kBuf && !issue_v()) {
                        ok = false;
                        break;
                    }
                    const int b = it % kBuf;
                    const uint32_t par = ((it / kBuf) & 1) ^ 1;
                    if (!mbar_wait(&sm.bempty[b], par, sm, a.err)) break;
                    mbar_expect_tx(&sm.bfull[b], (uint32_t)(ui.np * 16 * kNB * 2));
                    for (int p = 0; p < ui.np; ++p)
                        tma_load(&sm.bs[b][p * 16 * kNB], tmB, j * kNB, pg[p] * LORA_PAGE_ROWS, &sm.bfull[b]);
                    if (!mbar_wait(&sm.yempty[b], par, sm, a.err)) break;
                    mbar_expect_tx(&sm.yfull[b], (uint32_t)(kM * kNB * 4));
                    tma_load(&sm.ys[b][0], tmY, j * kNB, ui.row0, &sm.yfull[b]);
                    tma_load(&sm.ys[b][kM * 32], tmY, j * kNB + 32, ui.row0, &sm.yfull[b]);
                }
                if (ok && !v_done && !issue_v()) ok = false;   // a first unit of at most kBuf items
            }
            if (!waited) asm volatile("griddepcontrol.wait;" ::: "memory");   // before the CTA can finish
            for (int i = (it > kBuf ? it - kBuf : 0); i < it; ++i) {
                drain_wait(&sm.bfull[i % kBuf], (i / kBuf) & 1);
                drain_wait(&sm.yfull[i % kBuf], (i / kBuf) & 1);
            }
            if (itv > 0) drain_wait(&sm.v_full, (itv - 1) & 1);
        }
    } else if (warp == 2 && lane == 0) {
        // ---------------- MMA issuer ----------------
        int it = 0, ite = 0, itt = 0;
        bool issued = false;
        const uint32_t idesc2 = idesc_bf16(kM, kNB, 0, 1);
        // shrink: for each quarter q in [q0, q1), D1_q = X A over its K blocks,
        // into columns 64 q (spread) or 0
        auto shrink = [&](const UnitInfo &ui, int q0, int q1, bool spread) {
            const uint32_t idesc1 = idesc_bf16(kM, ui.n1, 0, 0);
            if (!mbar_wait(&sm.d1_empty, (itt & 1) ^ 1, sm, a.err)) return false;
            tc_fence_after();
            for (int q = q0; q < q1; ++q) {
                int kb0, kb1;
                quarter_blocks(nkb, q, kb0, kb1);
                const uint32_t d1 = tmem + (spread ? 64u * (uint32_t)q : 0u);
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const int s = it % kSt;
                    if (!mbar_wait(&sm.full[s], (it / kSt) & 1, sm, a.err)) return false;
                    tc_fence_after();
                    issued = true;
                    const uint64_t da = sdesc(sm.xs[s], 16, 1024);
                    const uint64_t db = sdesc(sm.as[s], 16, 1024);
#pragma unroll
                    for (int k = 0; k < kKB / 16; ++k)
                        mma_bf16(d1, da + (uint64_t)(k * 2), db + (uint64_t)(k * 2), idesc1, (kb != kb0) || (k != 0));
                    mma_commit(&sm.empty[s]);
                }
            }
            if (aborted(sm)) return false;
            mma_commit(&sm.shrink_done);
            return true;
        };
        // expand: one 64-column n-tile at a time into a buffered accumulator
        auto expand = [&](const UnitInfo &ui) {
            if (!mbar_wait(MODE == kExpandV ? &sm.v_full : &sm.v_ready, itt & 1, sm, a.err)) return false;
            tc_fence_after();
            const uint64_t dv = sdesc(sm.vs, 16, 1024);
            const uint64_t dvl = sdesc(sm.vl, 16, 1024);
            for (int j = ui.j0; j < ui.j1; ++j, ++ite) {
                const int b = ite % kBuf;
                const uint32_t par = (ite / kBuf) & 1;
                if (!mbar_wait(&sm.accempty[b], par ^ 1, sm, a.err)) return false;
                if (!mbar_wait(&sm.bfull[b], par, sm, a.err)) return false;
                tc_fence_after();
                issued = true;
                const uint64_t dbb = sdesc(sm.bs[b], (uint32_t)(ui.n1 * 128), 1024);
                for (int k = 0; k < ui.np; ++k)
                    mma_bf16(tmem + kAccCol + 64 * b, dv + (uint64_t)(k * 2), dbb + (uint64_t)(k * (2048 >> 4)),
                             idesc2, k != 0);
                for (int k = 0; k < ui.np; ++k)
                    mma_bf16(tmem + kAccCol + 64 * b, dvl + (uint64_t)(k * 2), dbb + (uint64_t)(k * (2048 >> 4)),
                             idesc2, 1);
                mma_commit(&sm.bempty[b]);
                mma_commit(&sm.accfull[b]);
            }
            if (aborted(sm)) return false;
            mma_commit(&sm.v_empty);
            return true;
        };
        if constexpr (MODE == kShrinkQ) {
            QIter u = qunit_range(n_tiles);
            int q = 0, kb0, kb1;
            UnitInfo ui;
            while (next_qunit(a, u, ui, q) && !aborted(sm)) {
                quarter_blocks(nkb, q, kb0, kb1);
                if (ui.skip || kb1 <= kb0) continue;
                if (!shrink(ui, q, q + 1, true)) break;
                ++itt;
            }
        } else {
            UnitIter ur = unit_range(n_tiles, nj);
            UnitInfo ui;
            while (next_unit(a, ur, ui) && !aborted(sm)) {
                if (ui.skip) continue;
                if constexpr (MODE == kFused)
                    if (!shrink(ui, 0, kSlicesQ, true)) break;
                if (!expand(ui)) break;
                ++itt;
            }
        }
        // every MMA this thread issued has completed before tensor memory is freed
        if (issued) {
            mma_commit(&sm.mma_drain);
            drain_wait(&sm.mma_drain, 0);
        }
    } else if (warp >= 4) {
        // ---------------- epilogue ----------------
        const int q = warp & 3;              // tensor-memory lane quarter of this warp
        const int m = q * 32 + lane;         // tile row = accumulator lane
        const uint32_t trow = tmem + ((uint32_t)(q * 32) << 16);
        const bool leader = (warp == 4 && lane == 0);
        int pending = -1;   // Y buffer whose TMA store may still be reading it
        int ite = 0, itt = 0;
        // row m of v (fp32) -> its bf16 high part (bytes 0..127 of quarter 0's
        // workspace row) and low part (bytes 128..255), one 16-byte group of
        // eight values at a time
        auto store_v_row = [&](const float (&v)[64], int np, float *row) {
            uint4 *dst = reinterpret_cast<uint4 *>(row);
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                if (c < np * 2) {
                    uint32_t hw[4], lw[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float f0 = v[c * 8 + 2 * e], f1 = v[c * 8 + 2 * e + 1];
                        const __nv_bfloat162 h = __floats2bfloat162_rn(f0, f1);
                        const __nv_bfloat162 l = __floats2bfloat162_rn(f0 - __low2float(h), f1 - __high2float(h));
                        hw[e] = *reinterpret_cast<const uint32_t *>(&h);
                        lw[e] = *reinterpret_cast<const uint32_t *>(&l);
                    }
                    dst[c] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
                    dst[8 + c] = make_uint4(lw[0], lw[1], lw[2], lw[3]);
                }
            }
        };
        // v (fp32, row m) -> bf16 high part and low part (v - high), the two
        // 16-significant-bit halves the expand multiplies by B
        auto split_v = [&](const float (&v)[64], int np, uint32_t (&hw)[32], uint32_t (&lw)[32]) {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
                if (e < np * 8) {
                    const __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * e], v[2 * e + 1]);
                    const __nv_bfloat162 l = __floats2bfloat162_rn(v[2 * e] - __low2float(h), v[2 * e + 1] - __high2float(h));
                    hw[e] = *reinterpret_cast<const uint32_t *>(&h);
                    lw[e] = *reinterpret_cast<const uint32_t *>(&l);
                }
            }
        };
        if constexpr (MODE == kShrinkQ) {
            // A tile whose four quarters all lie in this CTA's range keeps each
            // quarter's D1 in its own tensor-memory block; at its last quarter
            // the epilogue adds the blocks in quarter order and leaves v (bf16
            // high, low) in quarter 0's rows of the workspace.  Any other tile:
            // D1 rows of its tokens -> the quarter's fp32 partials, and the CTA
            // that finishes the tile's last quarter adds the quarters in order
            // from there.  Both give the same sums.
            QIter u = qunit_range(n_tiles);
            int qq = 0, kb0, kb1, last_q = 0;
            for (int q2 = 0; q2 < kSlicesQ; ++q2) {
                quarter_blocks(nkb, q2, kb0, kb1);
                if (kb1 > kb0) last_q = q2;
            }
            UnitInfo ui;
            while (next_qunit(a, u, ui, qq)) {
                if (!epi_all(!aborted(sm))) break;
                quarter_blocks(nkb, qq, kb0, kb1);
                if (ui.skip || kb1 <= kb0) continue;
                if (!epi_all(mbar_wait(&sm.shrink_done, itt & 1, sm, a.err))) break;
                tc_fence_after();
                const bool owned = ui.tile * kSlicesQ >= u.u0 && ui.tile * kSlicesQ + kSlicesQ <= u.u1;
                if (owned) {
                    if (qq == last_q) {
                        float v[64];
#pragma unroll
                        for (int c = 0; c < 64; ++c) v[c] = 0.f;
                        for (int q2 = 0; q2 < kSlicesQ; ++q2) {
                            int b0, b1;
                            quarter_blocks(nkb, q2, b0, b1);
                            if (b1 <= b0) continue;
#pragma unroll
                            for (int c = 0; c < 4; ++c) {
                                if (c < ui.np) {
                                    float t16[16];
                                    TMEM_LD16(trow + 64 * q2 + c * 16, t16);
                                    tmem_wait_ld();
#pragma unroll
                                    for (int i = 0; i < 16; ++i) v[c * 16 + i] += t16[i];
                                }
                            }
                        }
                        tc_fence_before();
                        mbar_arrive(&sm.d1_empty);
                        if (m < ui.ntok) store_v_row(v, ui.np, a.vpart + ((size_t)ui.row0 + m) * LORA_MAX_RANK);
                    } else {
                        // the block stays until the tile's last quarter reads it
                        tc_fence_before();
                        mbar_arrive(&sm.d1_empty);
                    }
                    ++itt;
                    continue;
                }
                float d1[64];
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    if (c < ui.np) TMEM_LD16(trow + 64 * qq + c * 16, (&d1[c * 16]));
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(&sm.d1_empty);
                if (m < ui.ntok) {
                    float4 *dst = reinterpret_cast<float4 *>(a.vpart + ((size_t)qq * a.T + ui.row0 + m) * LORA_MAX_RANK);
#pragma unroll
                    for (int c = 0; c < 16; ++c)
                        if (c < ui.np * 4)
                            dst[c] = make_float4(d1[4 * c], d1[4 * c + 1], d1[4 * c + 2], d1[4 * c + 3]);
                }
                __threadfence();   // this quarter's rows are visible before it is counted
                epi_sync();
                if (leader) sm.reduce = atomicAdd(&a.tiles[ui.tile].w, 1) == nq - 1;
                epi_sync();
                if (sm.reduce) {
                    __threadfence();
                    if (m < ui.ntok) {
                        float v[64];
#pragma unroll
                        for (int c = 0; c < 64; ++c) v[c] = 0.f;
                        // all four quarters' loads in flight at once; added in quarter order
#pragma unroll
                        for (int q2 = 0; q2 < kSlicesQ; ++q2) {
                            int b0, b1;
                            quarter_blocks(nkb, q2, b0, b1);
                            const float4 *src =
                                reinterpret_cast<const float4 *>(a.vpart + ((size_t)q2 * a.T + ui.row0 + m) * LORA_MAX_RANK);
#pragma unroll
                            for (int c = 0; c < 16; ++c) {
                                if (b1 > b0 && c < ui.np * 4) {
                                    const float4 w = __ldcg(src + c);
                                    v[4 * c] += w.x;
                                    v[4 * c + 1] += w.y;
                                    v[4 * c + 2] += w.z;
                                    v[4 * c + 3] += w.w;
                                }
                            }
                        }
                        store_v_row(v, ui.np, a.vpart + ((size_t)ui.row0 + m) * LORA_MAX_RANK);
                    }
                    if (leader) a.tiles[ui.tile].w = 0;   // ready for the next launch over this plan
                }
                ++itt;
            }
        } else {
            UnitIter ur = unit_range(n_tiles, nj);
            UnitInfo ui;
            while (next_unit(a, ur, ui)) {
                if (!epi_all(!aborted(sm))) break;   // same decision in all 128 epilogue threads
                if (ui.skip) continue;
                const KTileProj &pr = a.proj[ui.p];
                const float sc = pr.scales[ui.slot];
                if constexpr (MODE == kFused) {
                    // v = row m of the quarters' D1 added in quarter order: the
                    // same fp32 sums, and the same bf16 parts, as the two-launch form
                    if (!epi_all(mbar_wait(&sm.shrink_done, itt & 1, sm, a.err))) break;
                    tc_fence_after();
                    float d1[64];
#pragma unroll
                    for (int c = 0; c < 64; ++c) d1[c] = 0.f;
                    for (int qq = 0; qq < kSlicesQ; ++qq) {
                        int kb0, kb1;
                        quarter_blocks(nkb, qq, kb0, kb1);
                        if (kb1 <= kb0) continue;
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            if (c < ui.np) {
                                float t16[16];
                                TMEM_LD16(trow + 64 * qq + c * 16, t16);
                                tmem_wait_ld();
#pragma unroll
                                for (int i = 0; i < 16; ++i) d1[c * 16 + i] += t16[i];
                            }
                        }
                    }
                    tc_fence_before();
                    mbar_arrive(&sm.d1_empty);
                    uint32_t hw[32], lw[32];
                    split_v(d1, ui.np, hw, lw);
                    if (!epi_all(mbar_wait(&sm.v_empty, (itt & 1) ^ 1, sm, a.err))) break;
                    unsigned char *vrow = reinterpret_cast<unsigned char *>(sm.vs) + m * 128;
                    unsigned char *lrow = reinterpret_cast<unsigned char *>(sm.vl) + m * 128;
#pragma unroll
                    for (int c = 0; c < 8; ++c) {
                        if (c < ui.np * 2) {
                            *reinterpret_cast<uint4 *>(vrow + ((c ^ (m & 7)) << 4)) =
                                make_uint4(hw[4 * c], hw[4 * c + 1], hw[4 * c + 2], hw[4 * c + 3]);
                            *reinterpret_cast<uint4 *>(lrow + ((c ^ (m & 7)) << 4)) =
                                make_uint4(lw[4 * c], lw[4 * c + 1], lw[4 * c + 2], lw[4 * c + 3]);
                        }
                    }
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    mbar_arrive(&sm.v_ready);
                }
                // n-tiles: y = s * D2 + y on the Y tile in shared memory (row m
                // per thread); a full tile goes back with two TMA stores issued by
                // one thread (its buffer is released once the store has read it,
                // one item later), a tile of fewer than 128 tokens with coalesced
                // row stores of its tokens from all 128 threads
                const bool full_tile = ui.ntok == kM;
                for (int j = ui.j0; j < ui.j1; ++j, ++ite) {
                    const int b = ite % kBuf;
                    const uint32_t par = (ite / kBuf) & 1;
                    bool ok = mbar_wait(&sm.accfull[b], par, sm, a.err);
                    ok = mbar_wait(&sm.yfull[b], par, sm, a.err) && ok;
                    if (!epi_all(ok)) break;
                    tc_fence_after();
                    float acc[64];
#pragma unroll
                    for (int c = 0; c < 4; ++c) TMEM_LD16(trow + kAccCol + 64 * b + c * 16, (&acc[c * 16]));
                    tmem_wait_ld();
                    tc_fence_before();
                    mbar_arrive(&sm.accempty[b]);
                    unsigned char *yt = reinterpret_cast<unsigned char *>(&sm.ys[b][0]);
#pragma unroll
                    for (int c = 0; c < 16; ++c) {
                        const int h = c >> 3, cc = c & 7;
                        float4 *yp = reinterpret_cast<float4 *>(yt + h * kM * 128 + m * 128 + ((cc ^ (m & 7)) << 4));
                        float4 y = *yp;
                        y.x = fmaf(sc, acc[c * 4 + 0], y.x);
                        y.y = fmaf(sc, acc[c * 4 + 1], y.y);
                        y.z = fmaf(sc, acc[c * 4 + 2], y.z);
                        y.w = fmaf(sc, acc[c * 4 + 3], y.w);
                        *yp = y;
                    }
                    // the tile was written through the generic proxy; order that
                    // before the TMA store or the producer's next TMA load into it
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                    epi_sync();
                    if (full_tile) {
                        if (leader) {
                            tma_store(&maps.Y[ui.p], j * kNB, ui.row0, &sm.ys[b][0]);
                            tma_store(&maps.Y[ui.p], j * kNB + 32, ui.row0, &sm.ys[b][kM * 32]);
                            asm volatile("cp.async.bulk.commit_group;" ::: "memory");
                            // the previous store has left its buffer once at most one
                            // group (this one) is still reading
                            asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
                            if (pending >= 0) mbar_arrive(&sm.yempty[pending]);
                            pending = b;
                        }
                    } else {
                        // 16 threads per row, one 16-byte group each: row r, group g
                        const int tid = threadIdx.x - 128;
#pragma unroll 4
                        for (int i = 0; i < 16; ++i) {
                            const int idx = tid + 128 * i, r = idx >> 4, g = idx & 15;
                            const int col = j * kNB + 4 * g;
                            if (r < ui.ntok && col < pr.d_out) {
                                const int h = g >> 3, cc = g & 7;
                                const float4 y =
                                    *reinterpret_cast<const float4 *>(yt + h * kM * 128 + r * 128 + ((cc ^ (r & 7)) << 4));
                                *reinterpret_cast<float4 *>(pr.Y + (size_t)(ui.row0 + r) * pr.d_out + col) = y;
                            }
                        }
                        epi_sync();
                        if (leader) {
                            // a buffer whose store is still pending would otherwise wait
                            // for the next full tile, which may never come on this CTA
                            if (pending >= 0) {
                                asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
                                mbar_arrive(&sm.yempty[pending]);
                                pending = -1;
                            }
                            mbar_arrive(&sm.yempty[b]);
                        }
                    }
                }
                ++itt;
            }
            if (leader) {
                asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
                if (pending >= 0) mbar_arrive(&sm.yempty[pending]);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 2)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(tmem_cols<MODE>()));
}

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------
}  // namespace

bool tiles_supported() { return tma_supported(); }

namespace {

template <int NP, int MODE>
int launch_np(const TileArgs &a, cudaStream_t st, bool pdl, int sms) {
    const size_t smem = sizeof(typename SmemOf<MODE>::type) + 1024;
    TileMaps<NP> maps;
    KTile<NP> k;
    k.X = a.X; k.T = a.T; k.d_in = a.d_in; k.nproj = a.nproj;
    k.tiles = const_cast<int4 *>(a.tiles); k.hdr = a.hdr; k.err = a.err; k.vpart = a.vpart;
    if (int rc = make_tensor_map(&maps.X, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.X, (uint64_t)a.d_in, (uint64_t)a.T,
                                 kKB, kM, true))
        return rc;
    maps.V = maps.X;
    if (MODE == kExpandV) {
        // quarter 0 of the partials, row t = 256 bytes = v high [64] | v low [64] in bf16
        if (int rc = make_tensor_map(&maps.V, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.vpart, 2 * LORA_MAX_RANK,
                                     (uint64_t)a.T, 64, kM, true))
            return rc;
    }
    k.jpre[0] = 0;
    for (int p = 0; p < NP; ++p) {
        const TileProj &q = a.proj[p < a.nproj ? p : 0];
        k.proj[p].Y = q.Y; k.proj[p].d_out = q.d_out; k.proj[p].ranks = q.ranks; k.proj[p].scales = q.scales;
        k.proj[p].pt = q.pt;
        k.proj[p].rowsA = (long long)q.pa->num_pages * LORA_PAGE_ROWS;
        k.proj[p].rowsB = (long long)q.pb->num_pages * LORA_PAGE_ROWS;
        if (int rc = make_tensor_map(&maps.Y[p], CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, q.Y, (uint64_t)q.d_out,
                                     (uint64_t)a.T, 32, kM, true))
            return rc;
        if (int rc = pool_tensor_map(const_cast<lora_pool_s *>(q.pa), &maps.A[p])) return rc;
        if (int rc = pool_tensor_map(const_cast<lora_pool_s *>(q.pb), &maps.B[p])) return rc;
        k.jpre[p + 1] = k.jpre[p] + (p < a.nproj ? (q.d_out + kNB - 1) / kNB : 0);
    }
    // one CTA per SM (never more than there can be units)
    const long long max_tiles = (a.T + kM - 1) / kM + (a.long_thresh > 0 ? a.T / a.long_thresh : 0);
    long long grid = sms;
    const long long units = MODE == kShrinkQ ? max_tiles * kSlicesQ : max_tiles * k.jpre[NP];
    if (grid > units) grid = units;
    if (grid < 1) grid = 1;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    if (int rc = cuda_check(cudaLaunchKernelEx(&cfg, tiles_kernel<NP, MODE>, maps, k))) return rc;
    count_launch();
    note_launch(st, false);
    return LORA_OK;
}

template <int NP, int MODE>
int set_smem_attr() {
    return cuda_check(cudaFuncSetAttribute(tiles_kernel<NP, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)(sizeof(typename SmemOf<MODE>::type) + 1024)));
}

}  // namespace

int launch_tiles(const TileArgs &a, cudaStream_t st, bool pdl) {
    static int num_sms[64] = {};
    int dev = 0;
    if (a.nproj < 1 || a.nproj > LORA_MAX_PROJECTIONS) return LORA_ERR_INVALID_ARG;
    if (int rc = cuda_check(cudaGetDevice(&dev))) return rc;
    if (dev < 0 || dev >= 64) return LORA_ERR_INVALID_ARG;
    if (num_sms[dev] == 0) {
        if (int rc = set_smem_attr<1, kFused>()) return rc;
        if (int rc = set_smem_attr<LORA_MAX_PROJECTIONS, kFused>()) return rc;
        if (int rc = set_smem_attr<1, kShrinkQ>()) return rc;
        if (int rc = set_smem_attr<1, kExpandV>()) return rc;
        int n = 0;
        if (int rc = cuda_check(cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev))) return rc;
        num_sms[dev] = n > 0 ? n : 1;
    }
    const int sms = num_sms[dev];
    if (a.nproj == 1 && a.vpart) {
        if (int rc = launch_np<1, kShrinkQ>(a, st, pdl, sms)) return rc;
        return launch_np<1, kExpandV>(a, st, true, sms);
    }
    return a.nproj == 1 ? launch_np<1, kFused>(a, st, pdl, sms)
                        : launch_np<LORA_MAX_PROJECTIONS, kFused>(a, st, pdl, sms);
}

}  // namespace lora
