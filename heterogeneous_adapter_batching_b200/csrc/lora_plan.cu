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
// One CTA of 1024 threads.  W warps (W * S <= 16384) own contiguous token
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

constexpr int kPlanThreads = 1024;
constexpr int kTableEntries = 16384;

__device__ __forceinline__ int block_exclusive_scan(int v, int *warp_tot, int *total) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[wid] = x;
    __syncthreads();
    if (wid == 0) {
        int w = (lane < (int)(blockDim.x >> 5)) ? warp_tot[lane] : 0;
        int s = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int y = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += y;
        }
        warp_tot[lane] = s - w;  // exclusive warp offsets
        if (lane == 31) *total = s;
    }
    __syncthreads();
    int r = warp_tot[wid] + x - v;
    __syncthreads();
    return r;
}

__device__ __forceinline__ bool valid_id(int id, int S, const int32_t *ranks) {
    return id >= 0 && id < S && ranks[id] > 0;
}

// A break: token t starts a run of one slot, or has no valid adapter.
// Gather jobs are ordered by rank class: 0 = 4 pages per matrix (rank 49-64;
// an out-of-range rank counts here too), 1 = 3 pages, 2 = 2, 3 = 1 page.
constexpr int kPlanRankClasses = 4;
__device__ __forceinline__ int rank_class(int r) {
    const int np = (r + LORA_PAGE_ROWS - 1) / LORA_PAGE_ROWS;
    return np >= 4 ? 0 : (np <= 1 ? 3 : 4 - np);
}

__device__ __forceinline__ bool is_break(const int32_t *ids, int t, int id, bool ok) {
    return !ok || t == 0 || ids[t - 1] != id;
}

__global__ void __launch_bounds__(kPlanThreads, 1)
plan_kernel(const int32_t *__restrict__ ids, int T, const int32_t *__restrict__ ranks, int S, int W,
            int long_thresh, int job_tokens, int clusters, PlanOut out, int32_t *err_dev) {
    // Let the dependent kernel's CTAs get resident while the plan runs; they
    // wait for this grid's completion before reading its output.
    asm volatile("griddepcontrol.launch_dependents;");

    extern __shared__ int smem[];
    int *cnt = smem;                       // [S][W] per-warp counts, then scan offsets
    int *scnt = cnt + (size_t)S * W;       // [S] short tokens per slot
    __shared__ int warp_tot[32];
    __shared__ int s_total[12];
    __shared__ int wfirst[32], wlast[32], carry_l[32], carry_r[32];

    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int n_entries = S * W;
    const bool runs = long_thresh > 0 && T >= long_thresh;

    for (int e = tid; e < n_entries; e += blockDim.x) cnt[e] = 0;
    for (int k = tid; k < S; k += blockDim.x) scnt[k] = 0;
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
        const int per = (n_entries + blockDim.x - 1) / blockDim.x;
        const int e0 = tid * per, e1 = min(n_entries, e0 + per);
        int local = 0;
        for (int e = e0; e < e1; ++e) local += cnt[e];
        int run = block_exclusive_scan(local, warp_tot, &s_total[0]);
        for (int e = e0; e < e1; ++e) { int c = cnt[e]; cnt[e] = run; run += c; }
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
    for (int k = tid; k < S; k += blockDim.x) {
        const int st = cnt[k * W];
        out.seg_start[k] = st;
        if (out.seg_start_copy) out.seg_start_copy[k] = st;
    }
    if (tid == 0) {
        out.seg_start[S] = n_valid;
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
                out.perm[pos] = t;
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
                if (t < hi) out.run_start[t] = v;
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
                    if (ok && nxt - out.run_start[t] >= long_thresh) end = nxt - 1;
                    out.run_end[t] = end;
                }
                rc = min(rc, __shfl_sync(0xffffffffu, incl, 0));
            }
        }
    }
    __syncthreads();

    // Phase 4: compact perm to the tokens outside long runs (perm_short) and
    // count them per slot.
    {
        const int per = (n_valid + blockDim.x - 1) / blockDim.x;
        const int p0 = tid * per, p1 = min(n_valid, p0 + per);
        int local = 0;
        for (int p = p0; p < p1; ++p) {
            const int t = out.perm[p];
            if (!runs || out.run_end[t] < 0) ++local;
        }
        int pos = block_exclusive_scan(local, warp_tot, &s_total[1]);
        for (int p = p0; p < p1; ++p) {
            const int t = out.perm[p];
            if (!runs || out.run_end[t] < 0) {
                out.perm_short[pos++] = t;
                atomicAdd(&scnt[ids[t]], 1);
            }
        }
    }
    __syncthreads();

    // Phase 5: gather jobs (per slot) and tensor tiles (per long run, token order).
    {
        const int per = (S + blockDim.x - 1) / blockDim.x;   // <= 4 for S <= 4096
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
#pragma unroll
        for (int i = 0; i < 3; ++i) (void)block_exclusive_scan(njc[i], warp_tot, &s_total[6 + i]);
        {
            const int want = min(s_total[6], clusters);
            int jt = cand[0];
#pragma unroll
            for (int i = 1; i < 3; ++i)
                if (cand[i] <= job_tokens && s_total[6 + i] >= want) jt = cand[i];
            job_tokens = jt;
        }
        // Jobs are written heaviest first: by pages per matrix (4, 3, 2, 1),
        // then slot order.  The gather kernel hands units to clusters round
        // robin, so this order places the long units first and the short ones
        // fill in after them.
        int sh_local = 0, ns_local = 0;
        int njp[kPlanRankClasses] = {0, 0, 0, 0};
        for (int k = k0; k < k1; ++k) {
            const int c = scnt[k];
            sh_local += c;
            if (c > 0) njp[rank_class(ranks[k])] += (c + job_tokens - 1) / job_tokens;
            if (out.seg_start[k + 1] > out.seg_start[k]) ++ns_local;
        }
        int sh_off = block_exclusive_scan(sh_local, warp_tot, &s_total[2]);
        int j_off[kPlanRankClasses];
#pragma unroll
        for (int i = 0; i < kPlanRankClasses; ++i) j_off[i] = block_exclusive_scan(njp[i], warp_tot, &s_total[6 + i]);
        (void)block_exclusive_scan(ns_local, warp_tot, &s_total[4]);
        {
            int base = 0;   // classes in order 0 (heaviest) .. 3
#pragma unroll
            for (int i = 0; i < kPlanRankClasses; ++i) {
                j_off[i] += base;
                base += s_total[6 + i];
            }
            if (tid == 0) s_total[3] = base;
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
                    for (int i = 0; i < 4; ++i) tk[i] = i < cc ? out.perm_short[q0 + i] : -1;
                    out.jobs[2 * (jo + j)] = make_int4(k, cc, q0, 0);
                    out.jobs[2 * (jo + j) + 1] = make_int4(tk[0], tk[1], tk[2], tk[3]);
                }
                jo += nj;
            }
            sh_off += c;
        }
        __syncthreads();   // s_total[3] (the job count) is read below
        // a token starts a tile when it lies in a long run at a multiple of kTileM
        // from the run's start
        int nt_local = 0;
        const int tper = (T + blockDim.x - 1) / blockDim.x;
        const int t0 = tid * tper, t1 = min(T, t0 + tper);
        if (runs) {
            for (int t = t0; t < t1; ++t) {
                const int e = out.run_end[t];
                if (e >= 0 && ((t - out.run_start[t]) % kTileM) == 0) ++nt_local;
            }
        }
        int t_off = block_exclusive_scan(nt_local, warp_tot, &s_total[5]);
        if (runs) {
            for (int t = t0; t < t1; ++t) {
                const int e = out.run_end[t];
                if (e >= 0 && ((t - out.run_start[t]) % kTileM) == 0)
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

}  // namespace

int launch_plan(const int32_t *ids, int T, const int32_t *ranks, int S, int long_thresh, int job_tokens,
                const PlanOut &out, int32_t *err_dev, cudaStream_t st, int units_per_job) {
    int W = 32;
    while (W > 1 && W * S > kTableEntries) W >>= 1;
    const size_t smem = sizeof(int) * ((size_t)S * W + (size_t)S);
    static bool attr_set[64] = {};
    int dev = 0;
    if (int rc = cuda_check(cudaGetDevice(&dev))) return rc;
    if (dev < 0 || dev >= 64) return LORA_ERR_INVALID_ARG;
    if (!attr_set[dev]) {
        int rc = cuda_check(cudaFuncSetAttribute(plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)(sizeof(int) * (kTableEntries + LORA_MAX_SLOTS))));
        if (rc) return rc;
        attr_set[dev] = true;
    }
    int clusters = 1;
    if (int rc = gather_clusters(&clusters)) return rc;
    clusters = max(1, clusters / max(1, units_per_job));
    plan_kernel<<<1, kPlanThreads, smem, st>>>(ids, T, ranks, S, W, long_thresh, job_tokens, clusters, out, err_dev);
    count_launch();
    return cuda_check(cudaGetLastError());
}

}  // namespace lora
