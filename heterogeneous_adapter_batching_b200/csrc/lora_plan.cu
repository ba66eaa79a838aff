// Segment plan: stable grouping of the batch's tokens by adapter slot.
//
// Page "Multi-LoRA Serving in Production" (llms.blog), section "Segmented
// Gather Matrix-Vector Multiplication (SGMV)": the kernel groups the requests
// of the batch by their target adapter so that each adapter's weights serve
// all of its tokens.  This kernel computes that grouping on the device as a
// stable counting sort (slot ascending, token index ascending within a slot)
// and, from it, the work lists of the two compute paths:
//   * gather jobs  (slot, first perm index, token count) for short segments;
//   * tensor tiles (slot, first X row, token count, first perm index) for
//     segments of at least `long_thresh` tokens whose tokens are contiguous in
//     the batch (a prefill sequence), cut into tiles of kTileM tokens.
//
// One CTA of 1024 threads.  W warps (W * S <= 16384) own contiguous token
// ranges; per-warp counts live in a [slot][warp] table in shared memory, whose
// exclusive scan in slot-major order gives every warp the first output
// position of its tokens of each slot.  Inside a warp, __match_any_sync ranks
// the lanes that share a slot, so the scatter keeps token order without
// atomics on the output.
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

__global__ void __launch_bounds__(kPlanThreads, 1)
plan_kernel(const int32_t *__restrict__ ids, int T, const int32_t *__restrict__ ranks, int S,
            int W, int long_thresh, int job_tokens, PlanHeader *hdr, int32_t *seg_start,
            int32_t *perm, int4 *jobs, int4 *tiles, int32_t *perm2, int32_t *seg_start2,
            int32_t *err_dev) {
    // Let the dependent kernel's CTAs get resident while the plan runs; they
    // wait for this grid's completion before reading its output.
    asm volatile("griddepcontrol.launch_dependents;");

    extern __shared__ int smem[];
    int *cnt = smem;                      // [S][W]
    int *tmin = cnt + (size_t)S * W;      // [S]
    int *tmax = tmin + S;                 // [S]
    __shared__ int warp_tot[32];
    __shared__ int s_total[4];

    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int n_entries = S * W;

    for (int e = tid; e < n_entries; e += blockDim.x) cnt[e] = 0;
    for (int k = tid; k < S; k += blockDim.x) { tmin[k] = INT_MAX; tmax[k] = -1; }
    __syncthreads();

    const int chunk = ((T + W - 1) / W + 31) / 32 * 32;
    int err = 0;

    // Phase 1: per-warp histograms and first/last token of every slot.
    if (wid < W) {
        const int lo = wid * chunk, hi = min(T, lo + chunk);
        for (int base = lo; base < hi; base += 32) {
            const int t = base + lane;
            int id = -1;
            bool ok = false;
            if (t < hi) {
                id = ids[t];
                if (id < -1 || id >= S) err |= LORA_DEV_ERR_BAD_ID;
                else if (id >= 0) {
                    if (ranks[id] > 0) ok = true;
                    else err |= LORA_DEV_ERR_EMPTY_SLOT;
                }
            }
            const unsigned act = __ballot_sync(0xffffffffu, ok);
            if (ok) {
                const unsigned m = __match_any_sync(act, id);
                const int leader = __ffs(m) - 1;
                if (lane == leader) {
                    cnt[id * W + wid] += __popc(m);
                    atomicMin(&tmin[id], base + leader);
                    atomicMax(&tmax[id], base + 31 - __clz(m));
                }
            }
        }
    }
    // error bits: one atomic per warp
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) err |= __shfl_xor_sync(0xffffffffu, err, o);
    if (lane == 0 && err && err_dev) atomicOr(err_dev, err);
    __syncthreads();

    // Phase 2: exclusive scan of cnt in slot-major order.
    {
        const int per = (n_entries + blockDim.x - 1) / blockDim.x;
        const int e0 = tid * per, e1 = min(n_entries, e0 + per);
        int local = 0;
        for (int e = e0; e < e1; ++e) local += cnt[e];
        int run = block_exclusive_scan(local, warp_tot, &s_total[0]);
        for (int e = e0; e < e1; ++e) { int c = cnt[e]; cnt[e] = run; run += c; }
    }
    __syncthreads();
    const int n_valid = s_total[0];

    // Phase 2b: segment boundaries and work lists, a few slots per thread.
    {
        const int per = (S + blockDim.x - 1) / blockDim.x;   // <= 4 for S <= 4096
        const int k0 = tid * per, k1 = min(S, k0 + per);
        int nj_local = 0, nt_local = 0, ns_local = 0;
        for (int k = k0; k < k1; ++k) {
            const int st = cnt[k * W];
            const int en = (k + 1 < S) ? cnt[(k + 1) * W] : n_valid;
            const int c = en - st;
            if (c > 0) {
                ++ns_local;
                const bool contiguous = (tmax[k] - tmin[k] + 1) == c;
                const bool is_long = long_thresh > 0 && c >= long_thresh && contiguous;
                if (is_long) nt_local += (c + kTileM - 1) / kTileM;
                else nj_local += (c + job_tokens - 1) / job_tokens;
            }
        }
        int j_off = block_exclusive_scan(nj_local, warp_tot, &s_total[1]);
        int t_off = block_exclusive_scan(nt_local, warp_tot, &s_total[2]);
        (void)block_exclusive_scan(ns_local, warp_tot, &s_total[3]);
        for (int k = k0; k < k1; ++k) {
            const int st = cnt[k * W];
            const int en = (k + 1 < S) ? cnt[(k + 1) * W] : n_valid;
            const int c = en - st;
            seg_start[k] = st;
            if (seg_start2) seg_start2[k] = st;
            if (c <= 0) continue;
            const bool contiguous = (tmax[k] - tmin[k] + 1) == c;
            const bool is_long = long_thresh > 0 && c >= long_thresh && contiguous;
            if (is_long) {
                const int nt = (c + kTileM - 1) / kTileM;
                for (int j = 0; j < nt; ++j) {
                    const int cc = min(kTileM, c - j * kTileM);
                    tiles[t_off + j] = make_int4(k, tmin[k] + j * kTileM, cc, st + j * kTileM);
                }
                t_off += nt;
            } else {
                const int nj = (c + job_tokens - 1) / job_tokens;
                const int b = c / nj, rem = c % nj;
                for (int j = 0; j < nj; ++j) {
                    const int cc = b + (j < rem ? 1 : 0);
                    jobs[j_off + j] = make_int4(k, st + j * b + min(j, rem), cc, 0);
                }
                j_off += nj;
            }
        }
        if (tid == 0) {
            seg_start[S] = n_valid;
            if (seg_start2) seg_start2[S] = n_valid;
            hdr->n_valid = n_valid;
            hdr->n_seg = s_total[3];
            hdr->n_jobs = s_total[1];
            hdr->n_tiles = s_total[2];
            hdr->T = T;
            hdr->S = S;
            hdr->job_tokens = job_tokens;
            hdr->long_thresh = long_thresh;
        }
    }
    __syncthreads();

    // Phase 3: stable scatter of token indices.
    if (wid < W) {
        const unsigned lt_mask = (1u << lane) - 1u;
        const int lo = wid * chunk, hi = min(T, lo + chunk);
        for (int base = lo; base < hi; base += 32) {
            const int t = base + lane;
            int id = -1;
            bool ok = false;
            if (t < hi) {
                id = ids[t];
                ok = id >= 0 && id < S && ranks[id] > 0;
            }
            const unsigned act = __ballot_sync(0xffffffffu, ok);
            unsigned m = 0;
            int pos = 0;
            if (ok) {
                m = __match_any_sync(act, id);
                pos = cnt[id * W + wid] + __popc(m & lt_mask);
                perm[pos] = t;
                if (perm2) perm2[pos] = t;
            }
            __syncwarp();
            if (ok && lane == __ffs(m) - 1) cnt[id * W + wid] += __popc(m);
            __syncwarp();
        }
    }
}

}  // namespace

int launch_plan(const int32_t *ids, int T, const int32_t *ranks, int S, int long_thresh,
                int job_tokens, const PlanOut &out, int32_t *err_dev, cudaStream_t st) {
    int W = 32;
    while (W > 1 && W * S > kTableEntries) W >>= 1;
    const size_t smem = sizeof(int) * ((size_t)S * W + 2 * (size_t)S);
    static bool attr_set[64] = {};
    int dev = 0;
    if (int rc = cuda_check(cudaGetDevice(&dev))) return rc;
    if (dev < 0 || dev >= 64) return LORA_ERR_INVALID_ARG;
    if (!attr_set[dev]) {
        int rc = cuda_check(cudaFuncSetAttribute(plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)(sizeof(int) * (kTableEntries + 2 * LORA_MAX_SLOTS))));
        if (rc) return rc;
        attr_set[dev] = true;
    }
    plan_kernel<<<1, kPlanThreads, smem, st>>>(ids, T, ranks, S, W, long_thresh, job_tokens, out.header,
                                               out.seg_start, out.perm, out.jobs, out.tiles, out.perm_copy,
                                               out.seg_start_copy, err_dev);
    count_launch();
    return cuda_check(cudaGetLastError());
}

}  // namespace lora
