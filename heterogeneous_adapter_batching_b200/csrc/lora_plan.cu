// Segment plan: stable grouping of the batch's tokens by adapter slot, and the
// work lists of the two compute paths.
//
// Page "Multi-LoRA Serving in Production" (llms.blog), section "Segmented
// Gather Matrix-Vector Multiplication (SGMV)": the kernel groups the requests
// of the batch by their target adapter so that each adapter's weights serve
// all of its tokens.  Section "Multi-Size Batched Gather Kernels (MBGMV and
// MBGMM)": decode tokens (one per sequence) and prefill chunks (many
// consecutive tokens of one sequence) take different kernels.
//
// Outputs (all in the workspace):
//   perm [n_valid]      every token with a valid adapter, by slot ascending and
//                       token index ascending (a stable counting sort);
//   seg_start [S+1]     slot i owns perm[seg_start[i] .. seg_start[i+1]);
//   tiles               every maximal run of >= long_thresh consecutive tokens
//                       with the same slot, cut into tiles of kTileM tokens in
//                       token order: (slot, first token, count, 0);
//   perm_short          perm without the tokens of such runs (a stable
//                       compaction, so still grouped by slot);
//   jobs                the short tokens of every slot, split into gather
//                       jobs of balanced size, at most the size chosen for
//                       the batch (4, 8 or the cap job_tokens <=
//                       LORA_MAX_JOB_TOKENS, from the job counts and the
//                       gather kernel's cluster count), heaviest rank class
//                       first: two int4 per job, {slot, count, first index
//                       into perm_short, 0} and the job's first four token
//                       indices (-1 padded), so a decode consumer needs a
//                       single read to know its work (a larger job's further
//                       tokens follow in perm_short); the header records the
//                       job size chosen.
// Invalid ids (outside [-1, S) or an empty slot) are dropped and flagged.
//
// One CTA (256 threads for up to 1024 tokens, 512 up to 4096, 1024 beyond).
// Up to 4096 tokens the kernel keeps ids, ranks, perm, perm_short, the run
// bounds and seg_start in shared memory: the inputs cross from global memory
// once and the outputs are written once, so the plan costs one memory round
// trip plus its barriers.  W warps (W * S <= 16384) own contiguous token
// ranges; per-warp counts live in a [slot][warp] table in shared memory whose
// exclusive scan in slot-major order gives every warp the first output
// position of its tokens of each slot; __match_any_sync ranks the lanes that
// share a slot inside a warp, so the scatter keeps token order without
// atomics on the output.  Runs are delimited by "breaks" (a token that starts
// a run or has no valid adapter): a per-warp prefix max of break positions
// (left to right) gives each token its run start and a suffix min (right to
// left) the next break, both seeded by carries combined across warps.
#include <climits>

#include "lora_internal.cuh"

namespace lora {
namespace {

constexpr int kPlanMaxThreads = 1024;
constexpr int kTableEntries = 16384;
constexpr int kSmemTokens = 4096;      // batches up to this size plan in shared memory
constexpr int kScanVals = 8;           // most values one block scan carries

// Exclusive scan of N values per thread across the block (thread order);
// totals[i] receives the sum of value i.  Every thread must call it.
template <int N>
__device__ __forceinline__ void block_scan(int (&v)[N], int *wsum, int *totals) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int x[N];
#pragma unroll
    for (int i = 0; i < N; ++i) {
        x[i] = v[i];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x[i], o);
            if (lane >= o) x[i] += y;
        }
        if (lane == 31) wsum[i * 32 + wid] = x[i];
    }
    __syncthreads();
    if (wid == 0) {
#pragma unroll
        for (int i = 0; i < N; ++i) {
            const int w = lane < nw ? wsum[i * 32 + lane] : 0;
            int s = w;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, s, o);
                if (lane >= o) s += y;
            }
            wsum[i * 32 + lane] = s - w;   // exclusive warp offsets
            if (lane == 31) totals[i] = s;
        }
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < N; ++i) v[i] = wsum[i * 32 + wid] + x[i] - v[i];
    __syncthreads();   // wsum is reused by the next scan
}

__device__ __forceinline__ int block_exclusive_scan(int v, int *wsum, int *total) {
    int a[1] = {v};
    block_scan<1>(a, wsum, total);
    return a[0];
}

__device__ __forceinline__ bool valid_id(int id, int S, const int32_t *ranks) {
    return id >= 0 && id < S && ranks[id] > 0;
}

// Gather jobs are ordered by rank class: 0 = 4 pages per matrix (rank 49-64;
// an out-of-range rank counts here too), 1 = 3 pages, 2 = 2, 3 = 1 page.
constexpr int kPlanRankClasses = 4;
__device__ __forceinline__ int rank_class(int r) {
    const int np = (r + LORA_PAGE_ROWS - 1) / LORA_PAGE_ROWS;
    return np >= 4 ? 0 : (np <= 1 ? 3 : 4 - np);
}

// A break: token t starts a run of one slot, or has no valid adapter.
__device__ __forceinline__ bool is_break(const int32_t *ids, int t, int id, bool ok) {
    return !ok || t == 0 || ids[t - 1] != id;
}

// Dynamic shared memory of the kernel (ints).
__host__ __device__ constexpr size_t plan_smem_ints(int T, int S, int W, bool in_smem) {
    return (((size_t)S * W + 3) & ~(size_t)3) + (size_t)S + (in_smem ? (size_t)5 * T + 2 * (size_t)S + 1 : 0);
}

template <bool SMEM>
__global__ void __launch_bounds__(kPlanMaxThreads, 1)
plan_kernel(const int32_t *__restrict__ ids_g, int T, const int32_t *__restrict__ ranks_g, int S, int W,
            int long_thresh, int job_tokens, int clusters, PlanOut out, int32_t *err_dev) {
    // Let the dependent kernel's CTAs get resident while the plan runs; they
    // wait for this grid's completion before reading its output.
    asm volatile("griddepcontrol.launch_dependents;");

    extern __shared__ int smem[];
    int *cnt = smem;                       // [S][W] per-warp counts, then scan offsets (padded to 4 entries)
    int *scnt = cnt + (((size_t)S * W + 3) & ~(size_t)3);   // [S] short tokens per slot
    int *ids_s = scnt + S;                 // SMEM only: [T] ids, [S] ranks, [T] perm, [T] perm_short,
    int *ranks_s = ids_s + T;              //   [T] run starts, [T] run ends, [S + 1] seg_start
    int *perm_s = ranks_s + S;
    int *psh_s = perm_s + T;
    int *rs_s = psh_s + T;
    int *re_s = rs_s + T;
    int *seg_s = re_s + T;
    __shared__ int wsum[kScanVals * 32];
    __shared__ int s_total[16];
    __shared__ int wfirst[32], wlast[32], carry_l[32], carry_r[32];

    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5, nthr = blockDim.x;
    const int n_entries = S * W;
    const bool runs = long_thresh > 0 && T >= long_thresh;

    const int32_t *ids = SMEM ? ids_s : ids_g;
    const int32_t *ranks = SMEM ? ranks_s : ranks_g;
    int32_t *perm = SMEM ? perm_s : out.perm;
    int32_t *perm_short = SMEM ? psh_s : out.perm_short;
    int32_t *run_start = SMEM ? rs_s : out.run_start;
    int32_t *run_end = SMEM ? re_s : out.run_end;
    int32_t *seg_start = SMEM ? seg_s : out.seg_start;

    if (SMEM) {
        for (int t = tid; t < T; t += nthr) ids_s[t] = ids_g[t];
        for (int k = tid; k < S; k += nthr) ranks_s[k] = ranks_g[k];
    }
    for (int e = tid; e < ((n_entries + 3) & ~3); e += nthr) cnt[e] = 0;
    for (int k = tid; k < S; k += nthr) scnt[k] = 0;
    __syncthreads();

    const int chunk = ((T + W - 1) / W + 31) / 32 * 32;
    int err = 0;

    // Phase 1: per-warp histograms; first and last break of each warp's range.
    if (wid < W) {
        const int lo = wid * chunk, hi = min(T, lo + chunk);
        int first = T, last = -1;
        for (int base = lo; base < hi; base += 32) {
            const int t = base + lane;
            int id = -1;
            bool ok = false, brk = false;
            if (t < hi) {
                id = ids[t];
                if (id < -1 || id >= S) err |= LORA_DEV_ERR_BAD_ID;
                else if (id >= 0) {
                    if (ranks[id] > 0) ok = true;
                    else err |= LORA_DEV_ERR_EMPTY_SLOT;
                }
                brk = is_break(ids, t, id, ok);
            }
            const unsigned bm = __ballot_sync(0xffffffffu, brk);
            if (bm) {
                first = min(first, base + __ffs(bm) - 1);
                last = max(last, base + 31 - __clz(bm));
            }
            const unsigned act = __ballot_sync(0xffffffffu, ok);
            if (ok) {
                const unsigned m = __match_any_sync(act, id);
                if (lane == __ffs(m) - 1) cnt[id * W + wid] += __popc(m);
            }
        }
        if (lane == 0) { wfirst[wid] = first; wlast[wid] = last; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) err |= __shfl_xor_sync(0xffffffffu, err, o);
    if (lane == 0 && err && err_dev) atomicOr(err_dev, err);
    __syncthreads();

    // Phase 2: exclusive scan of cnt in slot-major order; carries of the run scans.
    {
        // each thread a contiguous run of 4-entry groups (the table is padded
        // to a multiple of 4 entries with zeros)
        const int n4 = (n_entries + 3) >> 2;
        const int per = (n4 + nthr - 1) / nthr;
        const int g0 = tid * per, g1 = min(n4, g0 + per);
        int4 *cnt4 = reinterpret_cast<int4 *>(cnt);
        int local = 0;
        for (int g = g0; g < g1; ++g) {
            const int4 c = cnt4[g];
            local += c.x + c.y + c.z + c.w;
        }
        int run = block_exclusive_scan(local, wsum, &s_total[0]);
        for (int g = g0; g < g1; ++g) {
            const int4 c = cnt4[g];
            int4 o;
            o.x = run; run += c.x;
            o.y = run; run += c.y;
            o.z = run; run += c.z;
            o.w = run; run += c.w;
            cnt4[g] = o;
        }
        if (tid < W) {
            int cl = -1, cr = T;
            for (int w = 0; w < tid; ++w) cl = max(cl, wlast[w]);
            for (int w = tid + 1; w < W; ++w) cr = min(cr, wfirst[w]);
            carry_l[tid] = cl;
            carry_r[tid] = cr;
        }
    }
    __syncthreads();
    const int n_valid = s_total[0];
    for (int k = tid; k < S; k += nthr) {
        const int st = cnt[k * W];
        seg_start[k] = st;
        if (SMEM) out.seg_start[k] = st;
        if (out.seg_start_copy) out.seg_start_copy[k] = st;
    }
    if (tid == 0) {
        seg_start[S] = n_valid;
        if (SMEM) out.seg_start[S] = n_valid;
        if (out.seg_start_copy) out.seg_start_copy[S] = n_valid;
    }
    __syncthreads();   // the scatter below advances cnt in place

    // Phase 3: stable scatter (perm) and, when tiles are wanted, the runs.
    if (wid < W) {
        const unsigned lt_mask = (1u << lane) - 1u;
        const int lo = wid * chunk, hi = min(T, lo + chunk);
        for (int base = lo; base < hi; base += 32) {
            const int t = base + lane;
            int id = -1;
            bool ok = false;
            if (t < hi) {
                id = ids[t];
                ok = valid_id(id, S, ranks);
            }
            const unsigned act = __ballot_sync(0xffffffffu, ok);
            unsigned m = 0;
            if (ok) {
                m = __match_any_sync(act, id);
                const int pos = cnt[id * W + wid] + __popc(m & lt_mask);
                perm[pos] = t;
                if (out.perm_copy) out.perm_copy[pos] = t;
            }
            __syncwarp();
            if (ok && lane == __ffs(m) - 1) cnt[id * W + wid] += __popc(m);
            __syncwarp();
        }
        if (runs) {
            // run start of every token: prefix max of break positions, left to right
            int carry = carry_l[wid];
            for (int base = lo; base < hi; base += 32) {
                const int t = base + lane;
                int v = -1;
                if (t < hi) {
                    const int id = ids[t];
                    if (is_break(ids, t, id, valid_id(id, S, ranks))) v = t;
                }
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int y = __shfl_up_sync(0xffffffffu, v, o);
                    if (lane >= o) v = max(v, y);
                }
                v = max(v, carry);
                if (t < hi) run_start[t] = v;
                carry = __shfl_sync(0xffffffffu, v, 31);
            }
            // next break after every token: suffix min, right to left.  The same
            // lane wrote run_start[t] above, so it reads its own value.
            int rc = carry_r[wid];
            const int nch = (hi - lo + 31) / 32;
            for (int c = nch - 1; c >= 0; --c) {
                const int t = lo + c * 32 + lane;
                int id = -1;
                bool ok = false;
                int v = T;
                if (t < hi) {
                    id = ids[t];
                    ok = valid_id(id, S, ranks);
                    if (is_break(ids, t, id, ok)) v = t;
                }
                int incl = v;   // inclusive suffix min over lanes >= this one
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int y = __shfl_down_sync(0xffffffffu, incl, o);
                    if (lane + o < 32) incl = min(incl, y);
                }
                int nxt = __shfl_down_sync(0xffffffffu, incl, 1);
                if (lane == 31) nxt = T;
                nxt = min(nxt, rc);
                if (t < hi) {
                    int end = -1;
                    if (ok && nxt - run_start[t] >= long_thresh) end = nxt - 1;
                    run_end[t] = end;
                }
                rc = min(rc, __shfl_sync(0xffffffffu, incl, 0));
            }
        }
    }
    __syncthreads();

    // Phase 4: compact perm to the tokens outside long runs (perm_short) and
    // count them per slot.
    {
        const int per = (n_valid + nthr - 1) / nthr;
        const int p0 = tid * per, p1 = min(n_valid, p0 + per);
        int local = 0;
        for (int p = p0; p < p1; ++p) {
            const int t = perm[p];
            if (!runs || run_end[t] < 0) ++local;
        }
        int pos = block_exclusive_scan(local, wsum, &s_total[1]);
        for (int p = p0; p < p1; ++p) {
            const int t = perm[p];
            if (!runs || run_end[t] < 0) {
                perm_short[pos] = t;
                if (SMEM) out.perm_short[pos] = t;
                atomicAdd(&scnt[ids[t]], 1);
                ++pos;
            }
        }
    }
    __syncthreads();

    // Phase 5: gather jobs (per slot) and tensor tiles (per long run, token order).
    {
        const int per = (S + nthr - 1) / nthr;
        const int k0 = tid * per, k1 = min(S, k0 + per);
        // Job size: the candidates are 4, 8 and the cap job_tokens (each at
        // most the cap).  The largest is taken that still gives min(jobs at
        // the smallest size, clusters) jobs: a batch with fewer jobs than the
        // gather kernel has clusters keeps its parallelism, a larger one gets
        // fewer reads of each adapter.
        const int cand[3] = {min(4, job_tokens), min(8, job_tokens), job_tokens};
        int njc[3] = {0, 0, 0};
        for (int k = k0; k < k1; ++k) {
            const int c = scnt[k];
#pragma unroll
            for (int i = 0; i < 3; ++i)
                if (c > 0) njc[i] += (c + cand[i] - 1) / cand[i];
        }
        block_scan<3>(njc, wsum, &s_total[6]);
        {
            const int want = min(s_total[6], clusters);
            int jt = cand[0];
#pragma unroll
            for (int i = 1; i < 3; ++i)
                if (cand[i] <= job_tokens && s_total[6 + i] >= want) jt = cand[i];
            job_tokens = jt;
        }
        // Jobs are written heaviest first: by pages per matrix (4, 3, 2, 1),
        // then slot order.  The gather kernels hand units out round robin, so
        // this order places the long units first and the short ones fill in
        // after them.  One scan carries the short tokens before each slot, the
        // jobs of each rank class before it and the slots present.
        int vals[kPlanRankClasses + 2] = {0, 0, 0, 0, 0, 0};   // jobs per class, short tokens, slots present
        for (int k = k0; k < k1; ++k) {
            const int c = scnt[k];
            vals[kPlanRankClasses] += c;
            if (c > 0) vals[rank_class(ranks[k])] += (c + job_tokens - 1) / job_tokens;
            if (seg_start[k + 1] > seg_start[k]) ++vals[kPlanRankClasses + 1];
        }
        block_scan<kPlanRankClasses + 2>(vals, wsum, &s_total[6]);
        int sh_off = vals[kPlanRankClasses];
        int j_off[kPlanRankClasses];
        {
            int base = 0;   // classes in order 0 (heaviest) .. 3
#pragma unroll
            for (int i = 0; i < kPlanRankClasses; ++i) {
                j_off[i] = vals[i] + base;
                base += s_total[6 + i];
            }
            if (tid == 0) {
                s_total[3] = base;
                s_total[4] = s_total[6 + kPlanRankClasses + 1];
            }
        }
        for (int k = k0; k < k1; ++k) {
            const int c = scnt[k];
            if (c > 0) {
                const int nj = (c + job_tokens - 1) / job_tokens;
                const int b = c / nj, rem = c % nj;
                int &jo = j_off[rank_class(ranks[k])];
                for (int j = 0; j < nj; ++j) {
                    const int cc = b + (j < rem ? 1 : 0);
                    const int q0 = sh_off + j * b + min(j, rem);
                    int tk[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) tk[i] = i < cc ? perm_short[q0 + i] : -1;
                    out.jobs[2 * (jo + j)] = make_int4(k, cc, q0, 0);
                    out.jobs[2 * (jo + j) + 1] = make_int4(tk[0], tk[1], tk[2], tk[3]);
                }
                jo += nj;
            }
            sh_off += c;
        }
        __syncthreads();   // s_total[3], s_total[4] are read below
        // a token starts a tile when it lies in a long run at a multiple of kTileM
        // from the run's start
        int nt_local = 0;
        const int tper = (T + nthr - 1) / nthr;
        const int t0 = tid * tper, t1 = min(T, t0 + tper);
        if (runs) {
            for (int t = t0; t < t1; ++t) {
                const int e = run_end[t];
                if (e >= 0 && ((t - run_start[t]) % kTileM) == 0) ++nt_local;
            }
        }
        int t_off = block_exclusive_scan(nt_local, wsum, &s_total[5]);
        if (runs) {
            for (int t = t0; t < t1; ++t) {
                const int e = run_end[t];
                if (e >= 0 && ((t - run_start[t]) % kTileM) == 0)
                    out.tiles[t_off++] = make_int4(ids[t], t, min(kTileM, e - t + 1), 0);
            }
        }
        if (tid == 0) {
            out.header->n_valid = n_valid;
            out.header->n_seg = s_total[4];
            out.header->n_jobs = s_total[3];
            out.header->n_tiles = runs ? s_total[5] : 0;
            out.header->T = T;
            out.header->S = S;
            out.header->job_tokens = job_tokens;
            out.header->long_thresh = long_thresh;
        }
    }
}

// Small batches without long runs (T <= kSmallTokens, S <= kSmallSlots): the
// same outputs as plan_kernel<true>, bit for bit, from one warp.  The
// block-wide scans and barriers of the general kernel cost more than the
// work at these sizes; here every step is a warp scan over shared tables,
// with two passes over the tokens (counts, then the stable scatter) and two
// over the slots (offsets and job-size counts, then the jobs).
constexpr int kSmallTokens = 256;
constexpr int kSmallSlots = 128;   // with more slots the warp's two slot passes cost more than the block's scans

__device__ __forceinline__ int warp_incl_scan(int v, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += y;
    }
    return v;
}

__global__ void __launch_bounds__(32, 1)
plan_small_kernel(const int32_t *__restrict__ ids_g, int T, const int32_t *__restrict__ ranks_g, int S,
                  int long_thresh, int job_tokens, int clusters, PlanOut out, int32_t *err_dev) {
    asm volatile("griddepcontrol.launch_dependents;");
    __shared__ int ids_s[kSmallTokens];
    __shared__ int perm_s[kSmallTokens];    // perm (the workspace copy is not written, as in plan_kernel<true>)
    __shared__ int rk[kSmallSlots];
    __shared__ int pos[kSmallSlots];      // tokens per slot, then the next output position of each slot
    __shared__ int seg[kSmallSlots + 1];
    const int lane = threadIdx.x;
    const unsigned lt_mask = (1u << lane) - 1u;

    for (int k = lane; k < S; k += 32) {
        rk[k] = ranks_g[k];
        pos[k] = 0;
    }
    for (int t = lane; t < T; t += 32) ids_s[t] = ids_g[t];
    __syncwarp();

    // tokens per slot, and the error bits
    int err = 0;
    for (int base = 0; base < T; base += 32) {
        const int t = base + lane;
        int id = -1;
        bool ok = false;
        if (t < T) {
            id = ids_s[t];
            if (id < -1 || id >= S) err |= LORA_DEV_ERR_BAD_ID;
            else if (id >= 0) {
                if (rk[id] > 0) ok = true;
                else err |= LORA_DEV_ERR_EMPTY_SLOT;
            }
        }
        const unsigned act = __ballot_sync(0xffffffffu, ok);
        if (ok) {
            const unsigned m = __match_any_sync(act, id);
            if (lane == __ffs(m) - 1) pos[id] += __popc(m);
        }
        __syncwarp();
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) err |= __shfl_xor_sync(0xffffffffu, err, o);
    if (lane == 0 && err && err_dev) atomicOr(err_dev, err);

    // slot offsets; the job counts of the three candidate sizes; the jobs of
    // each rank class under each candidate
    const int cand[3] = {min(4, job_tokens), min(8, job_tokens), job_tokens};
    int run = 0, n_seg = 0;
    int njc[3] = {0, 0, 0};
    int ncls[3][kPlanRankClasses] = {};
    for (int base = 0; base < S; base += 32) {
        const int k = base + lane;
        const int c = k < S ? pos[k] : 0;
        const int inc = warp_incl_scan(c, lane);
        if (k < S) {
            const int st = run + inc - c;
            seg[k] = st;
            pos[k] = st;
            out.seg_start[k] = st;
            if (out.seg_start_copy) out.seg_start_copy[k] = st;
            if (c > 0) {
                const int cl = rank_class(rk[k]);
#pragma unroll
                for (int i = 0; i < 3; ++i) {
                    const int nj = (c + cand[i] - 1) / cand[i];
                    njc[i] += nj;
#pragma unroll
                    for (int q = 0; q < kPlanRankClasses; ++q) ncls[i][q] += cl == q ? nj : 0;
                }
            }
        }
        n_seg += __popc(__ballot_sync(0xffffffffu, k < S && c > 0));
        run += __shfl_sync(0xffffffffu, inc, 31);
    }
    const int n_valid = run;
    if (lane == 0) {
        seg[S] = n_valid;
        out.seg_start[S] = n_valid;
        if (out.seg_start_copy) out.seg_start_copy[S] = n_valid;
    }
#pragma unroll
    for (int i = 0; i < 3; ++i) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) njc[i] += __shfl_xor_sync(0xffffffffu, njc[i], o);
#pragma unroll
        for (int q = 0; q < kPlanRankClasses; ++q)
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) ncls[i][q] += __shfl_xor_sync(0xffffffffu, ncls[i][q], o);
    }
    __syncwarp();

    // stable scatter: perm = perm_short (no long runs)
    for (int base = 0; base < T; base += 32) {
        const int t = base + lane;
        int id = -1;
        bool ok = false;
        if (t < T) {
            id = ids_s[t];
            ok = valid_id(id, S, rk);
        }
        const unsigned act = __ballot_sync(0xffffffffu, ok);
        unsigned m = 0;
        if (ok) {
            m = __match_any_sync(act, id);
            const int p = pos[id] + __popc(m & lt_mask);
            perm_s[p] = t;
            out.perm_short[p] = t;
            if (out.perm_copy) out.perm_copy[p] = t;
        }
        __syncwarp();
        if (ok && lane == __ffs(m) - 1) pos[id] += __popc(m);
        __syncwarp();
    }

    // job size: the largest candidate that still gives min(jobs at the
    // smallest size, clusters) jobs (the general kernel's rule)
    const int want = min(njc[0], clusters);
    int ci = 0;
#pragma unroll
    for (int i = 1; i < 3; ++i)
        if (cand[i] <= job_tokens && njc[i] >= want) ci = i;
    const int jt = cand[ci];
    int cls_base[kPlanRankClasses], n_jobs = 0;
#pragma unroll
    for (int q = 0; q < kPlanRankClasses; ++q) {
        cls_base[q] = n_jobs;
        n_jobs += ncls[ci][q];
    }

    // jobs: heaviest rank class first, slot order within a class
    for (int base = 0; base < S; base += 32) {
        const int k = base + lane;
        const int c = k < S ? seg[k + 1] - seg[k] : 0;
        const int cl = (k < S && c > 0) ? rank_class(rk[k]) : 0;
        const int nj = c > 0 ? (c + jt - 1) / jt : 0;
        int jo = 0;
#pragma unroll
        for (int q = 0; q < kPlanRankClasses; ++q) {
            const int v = cl == q ? nj : 0;
            const int inc = warp_incl_scan(v, lane);
            if (cl == q) jo = cls_base[q] + inc - v;
            cls_base[q] += __shfl_sync(0xffffffffu, inc, 31);
        }
        if (c > 0) {
            const int b = c / nj, rem = c % nj;
            for (int j = 0; j < nj; ++j) {
                const int cc = b + (j < rem ? 1 : 0);
                const int q0 = seg[k] + j * b + min(j, rem);
                int tk[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) tk[i] = i < cc ? perm_s[q0 + i] : -1;
                out.jobs[2 * (jo + j)] = make_int4(k, cc, q0, 0);
                out.jobs[2 * (jo + j) + 1] = make_int4(tk[0], tk[1], tk[2], tk[3]);
            }
        }
    }
    if (lane == 0) {
        out.header->n_valid = n_valid;
        out.header->n_seg = n_seg;
        out.header->n_jobs = n_jobs;
        out.header->n_tiles = 0;
        out.header->T = T;
        out.header->S = S;
        out.header->job_tokens = jt;
        out.header->long_thresh = long_thresh;
    }
}

}  // namespace

int launch_plan(const int32_t *ids, int T, const int32_t *ranks, int S, int long_thresh, int job_tokens,
                const PlanOut &out, int32_t *err_dev, cudaStream_t st, int units_per_job) {
    const bool in_smem = T <= kSmemTokens;
    const int threads = T <= 1024 ? 256 : (in_smem ? 512 : kPlanMaxThreads);
    // warps that own tokens: no more than there are 32-token groups (the
    // [slot][warp] table and its scan shrink with them)
    int W = threads / 32;
    if (W > (T + 31) / 32) W = (T + 31) / 32 > 0 ? (T + 31) / 32 : 1;
    while (W > 1 && W * S > kTableEntries) W >>= 1;
    const size_t smem = sizeof(int) * plan_smem_ints(T, S, W, in_smem);
    static bool attr_set[64] = {};
    int dev = 0;
    if (int rc = cuda_check(cudaGetDevice(&dev))) return rc;
    if (dev < 0 || dev >= 64) return LORA_ERR_INVALID_ARG;
    if (!attr_set[dev]) {
        // the largest each variant asks for: a full table (W * S = 16384) and, in
        // shared memory, kSmemTokens tokens and LORA_MAX_SLOTS slots
        const int big = (int)(sizeof(int) * (kTableEntries + LORA_MAX_SLOTS));
        const int big_s = (int)(sizeof(int) * (kTableEntries + LORA_MAX_SLOTS + 5 * kSmemTokens + 2 * LORA_MAX_SLOTS + 1));
        if (int rc = cuda_check(cudaFuncSetAttribute(plan_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, big)))
            return rc;
        if (int rc = cuda_check(cudaFuncSetAttribute(plan_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, big_s)))
            return rc;
        attr_set[dev] = true;
    }
    int clusters = 1;
    if (int rc = gather_clusters(&clusters)) return rc;
    clusters = max(1, clusters / max(1, units_per_job));
    const bool runs = long_thresh > 0 && T >= long_thresh;
    if (!runs && T <= kSmallTokens && S <= kSmallSlots && opt_plan_kernel() != LORA_PLAN_GENERAL) {
        plan_small_kernel<<<1, 32, 0, st>>>(ids, T, ranks, S, long_thresh, job_tokens, clusters, out, err_dev);
        count_launch();
        note_launch(st, true);
        return cuda_check(cudaGetLastError());
    }
    if (in_smem)
        plan_kernel<true><<<1, threads, smem, st>>>(ids, T, ranks, S, W, long_thresh, job_tokens, clusters, out, err_dev);
    else
        plan_kernel<false><<<1, threads, smem, st>>>(ids, T, ranks, S, W, long_thresh, job_tokens, clusters, out, err_dev);
    count_launch();
    note_launch(st, true);
    return cuda_check(cudaGetLastError());
}

}  // namespace lora
