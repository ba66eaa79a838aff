// C-ABI entry points of liblora: page pools, argument validation, workspace
// layout and the launch sequence of each call.  See include/lora.h for the
// contract of every function.
#include <atomic>
#include <cstring>

#include <mutex>
#include <unordered_map>

#include "lora_internal.cuh"

namespace lora {

namespace {
std::atomic<int> g_long_segment{128};
std::atomic<int> g_job_tokens{LORA_MAX_JOB_TOKENS};
std::atomic<int> g_gather_path{LORA_GATHER_AUTO};
std::atomic<int> g_plan_kernel{LORA_PLAN_AUTO};
thread_local int t_launches = 0;
thread_local const char *t_last_cuda_error = "no error";

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Writes one slot's table row: page ids of A and B, scale and rank.
__global__ void set_slot_kernel(int32_t *pt, float *scale, int32_t *rank, int slot, int4 pa, int4 pb,
                                float s, int r) {
    if (threadIdx.x == 0) {
        int32_t *row = pt + (size_t)slot * 2 * LORA_MAX_PAGES_PER_MATRIX;
        row[0] = pa.x; row[1] = pa.y; row[2] = pa.z; row[3] = pa.w;
        row[4] = pb.x; row[5] = pb.y; row[6] = pb.z; row[7] = pb.w;
        scale[slot] = s;
        rank[slot] = r;
    }
}

// Resolves (slot, matrix, rank-row) through the page table and copies the row.
__global__ void read_row_kernel(const uint16_t *pool, int width, const int32_t *pt, int slot, int m, int k,
                                uint16_t *out) {
    const int page = pt[((size_t)slot * 2 + m) * LORA_MAX_PAGES_PER_MATRIX + k / LORA_PAGE_ROWS];
    const uint16_t *row = pool + ((size_t)page * LORA_PAGE_ROWS + (k % LORA_PAGE_ROWS)) * width;
    for (int c = threadIdx.x + blockIdx.x * blockDim.x; c < width; c += blockDim.x * gridDim.x) out[c] = row[c];
}
}  // namespace

int opt_long_segment() { return g_long_segment.load(); }
int opt_job_tokens() { return g_job_tokens.load(); }
int opt_gather_path() { return g_gather_path.load(); }
int opt_plan_kernel() { return g_plan_kernel.load(); }

namespace {
std::mutex g_last_mu;
std::unordered_map<cudaStream_t, bool> g_plan_last;   // stream -> its last library launch was the plan
}  // namespace

bool plan_was_last_launch(cudaStream_t st) {
    std::lock_guard<std::mutex> g(g_last_mu);
    const auto it = g_plan_last.find(st);
    return it != g_plan_last.end() && it->second;
}

void note_launch(cudaStream_t st, bool is_plan) {
    std::lock_guard<std::mutex> g(g_last_mu);
    g_plan_last[st] = is_plan;
}

int cuda_check(cudaError_t e) {
    if (e == cudaSuccess) return LORA_OK;
    t_last_cuda_error = cudaGetErrorString(e);
    return LORA_ERR_CUDA;
}
void count_launch(int n) { t_launches += n; }
void reset_launch_count() { t_launches = 0; }

// Page allocation helpers (caller holds the pool mutex).
static int take_pages(lora_pool_s *p, int n, const int32_t *want, std::vector<int> &got) {
    got.clear();
    if (want) {
        for (int i = 0; i < n; ++i) {
            const int id = want[i];
            if (id < 0 || id >= p->num_pages || p->used[id]) return LORA_ERR_BAD_SLOT;
            for (int j = 0; j < i; ++j)
                if (want[j] == id) return LORA_ERR_BAD_SLOT;
        }
        for (int i = 0; i < n; ++i) {
            p->used[want[i]] = 1;
            got.push_back(want[i]);
        }
        // drop the taken ids from the free stack
        std::vector<int> keep;
        keep.reserve(p->free_stack.size());
        for (int id : p->free_stack)
            if (!p->used[id]) keep.push_back(id);
        p->free_stack.swap(keep);
        return LORA_OK;
    }
    if ((int)p->free_stack.size() < n) return LORA_ERR_POOL_OOM;
    for (int i = 0; i < n; ++i) {
        const int id = p->free_stack.back();
        p->free_stack.pop_back();
        p->used[id] = 1;
        got.push_back(id);
    }
    return LORA_OK;
}

static void give_pages(lora_pool_s *p, const std::vector<int> &pages) {
    for (int id : pages) {
        if (id >= 0 && id < p->num_pages && p->used[id] == 1) {
            p->used[id] = 0;
            p->free_stack.push_back(id);
        }
    }
}

}  // namespace lora

using namespace lora;

extern "C" {

int lora_pool_create(void *dev_buf, size_t bytes, int width, int page_rows, lora_pool_t *out) {
    if (!out || !dev_buf || width <= 0 || (width % 8) != 0 || width > (1 << 24) || page_rows != LORA_PAGE_ROWS)
        return LORA_ERR_INVALID_ARG;
    if (!aligned(dev_buf, 256)) return LORA_ERR_INVALID_ARG;
    const size_t page_bytes = (size_t)page_rows * width * 2;
    const size_t np = bytes / page_bytes;
    if (np < 1 || np > (size_t)INT32_MAX / LORA_PAGE_ROWS) return LORA_ERR_INVALID_ARG;
    lora_pool_s *p = new lora_pool_s();
    p->base = static_cast<uint16_t *>(dev_buf);
    p->bytes = bytes;
    p->width = width;
    p->page_rows = page_rows;
    p->num_pages = (int)np;
    p->used.assign(np, 0);
    p->free_stack.reserve(np);
    for (int i = (int)np - 1; i >= 0; --i) p->free_stack.push_back(i);  // pop order 0, 1, 2, ...
    *out = p;
    return LORA_OK;
}

int lora_pool_destroy(lora_pool_t pool) {
    delete pool;
    return LORA_OK;
}

int lora_pool_free_pages(lora_pool_t pool) {
    if (!pool) return -1;
    std::lock_guard<std::mutex> g(pool->mu);
    return (int)pool->free_stack.size();
}

int lora_pool_num_pages(lora_pool_t pool) { return pool ? pool->num_pages : -1; }

int lora_pool_alloc_pages(lora_pool_t pool, int n, int32_t *ids_out) {
    if (!pool || n < 0 || (n > 0 && !ids_out)) return LORA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> g(pool->mu);
    if ((int)pool->free_stack.size() < n) return LORA_ERR_POOL_OOM;
    for (int i = 0; i < n; ++i) {
        const int id = pool->free_stack.back();
        pool->free_stack.pop_back();
        pool->used[id] = 2;
        ids_out[i] = id;
    }
    return LORA_OK;
}

int lora_pool_free_page_list(lora_pool_t pool, const int32_t *ids, int n) {
    if (!pool || n < 0 || (n > 0 && !ids)) return LORA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> g(pool->mu);
    for (int i = 0; i < n; ++i) {   // all or nothing
        const int id = ids[i];
        if (id < 0 || id >= pool->num_pages || pool->used[id] != 2) return LORA_ERR_BAD_SLOT;
        for (int j = 0; j < i; ++j)
            if (ids[j] == id) return LORA_ERR_BAD_SLOT;
    }
    for (int i = 0; i < n; ++i) {
        pool->used[ids[i]] = 0;
        pool->free_stack.push_back(ids[i]);
    }
    return LORA_OK;
}

int lora_pool_usage(lora_pool_t pool, int *adapter_pages, int *other_pages) {
    if (!pool || !adapter_pages || !other_pages) return LORA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> g(pool->mu);
    int a = 0, o = 0;
    for (char u : pool->used) {
        a += u == 1;
        o += u == 2;
    }
    *adapter_pages = a;
    *other_pages = o;
    return LORA_OK;
}

int lora_pool_load(lora_pool_t pa, lora_pool_t pb, int slot, int num_slots, int rank, float alpha,
                   const uint16_t *a_t, const uint16_t *b, const int32_t *page_ids,
                   int32_t *page_table_dev, float *scale_dev, int32_t *rank_dev, lora_stream_t stream) {
    if (!pa || !pb || !a_t || !b || !page_table_dev || !scale_dev || !rank_dev) return LORA_ERR_INVALID_ARG;
    if (num_slots < 1 || num_slots > LORA_MAX_SLOTS) return LORA_ERR_INVALID_ARG;
    if (slot < 0 || slot >= num_slots) return LORA_ERR_BAD_SLOT;
    if (rank < 1 || rank > LORA_MAX_RANK) return LORA_ERR_BAD_RANK;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const int np = (rank + LORA_PAGE_ROWS - 1) / LORA_PAGE_ROWS;
    lora_pool_s *pools[2] = {pa, pb};
    const uint16_t *src[2] = {a_t, b};
    std::vector<int> got[2];
    // Lock both pools (in address order when distinct) for the allocation.
    std::unique_lock<std::mutex> l1, l2;
    if (pa == pb) {
        l1 = std::unique_lock<std::mutex>(pa->mu);
    } else if (pa < pb) {
        l1 = std::unique_lock<std::mutex>(pa->mu);
        l2 = std::unique_lock<std::mutex>(pb->mu);
    } else {
        l1 = std::unique_lock<std::mutex>(pb->mu);
        l2 = std::unique_lock<std::mutex>(pa->mu);
    }
    for (int m = 0; m < 2; ++m)
        if (pools[m]->owners.count(std::make_tuple((const void *)page_table_dev, slot, m))) return LORA_ERR_BAD_SLOT;
    for (int m = 0; m < 2; ++m) {
        int rc = take_pages(pools[m], np, page_ids ? page_ids + m * LORA_MAX_PAGES_PER_MATRIX : nullptr, got[m]);
        if (rc) {
            if (m == 1) give_pages(pools[0], got[0]);
            return rc;
        }
    }
    int rc = LORA_OK;
    for (int m = 0; m < 2 && rc == LORA_OK; ++m) {
        lora_pool_s *p = pools[m];
        const size_t row_bytes = (size_t)p->width * 2;
        for (int q = 0; q < np && rc == LORA_OK; ++q) {
            const int rows = (rank - q * LORA_PAGE_ROWS) < LORA_PAGE_ROWS ? (rank - q * LORA_PAGE_ROWS) : LORA_PAGE_ROWS;
            char *dst = reinterpret_cast<char *>(p->base) + (size_t)got[m][q] * LORA_PAGE_ROWS * row_bytes;
            const char *s = reinterpret_cast<const char *>(src[m]) + (size_t)q * LORA_PAGE_ROWS * row_bytes;
            rc = cuda_check(cudaMemcpyAsync(dst, s, rows * row_bytes, cudaMemcpyDefault, st));
            if (rc == LORA_OK && rows < LORA_PAGE_ROWS)
                rc = cuda_check(cudaMemsetAsync(dst + rows * row_bytes, 0, (LORA_PAGE_ROWS - rows) * row_bytes, st));
        }
    }
    if (rc != LORA_OK) {
        give_pages(pools[0], got[0]);
        give_pages(pools[1], got[1]);
        return rc;
    }
    int32_t ids[2][4] = {{-1, -1, -1, -1}, {-1, -1, -1, -1}};
    for (int m = 0; m < 2; ++m)
        for (int q = 0; q < np; ++q) ids[m][q] = got[m][q];
    set_slot_kernel<<<1, 32, 0, st>>>(page_table_dev, scale_dev, rank_dev, slot,
                                      make_int4(ids[0][0], ids[0][1], ids[0][2], ids[0][3]),
                                      make_int4(ids[1][0], ids[1][1], ids[1][2], ids[1][3]),
                                      alpha / (float)rank, rank);
    rc = cuda_check(cudaGetLastError());
    if (rc != LORA_OK) {
        give_pages(pools[0], got[0]);
        give_pages(pools[1], got[1]);
        return rc;
    }
    for (int m = 0; m < 2; ++m) pools[m]->owners[std::make_tuple((const void *)page_table_dev, slot, m)] = got[m];
    return LORA_OK;
}

int lora_pool_evict(lora_pool_t pa, lora_pool_t pb, int slot, int num_slots, int32_t *page_table_dev,
                    float *scale_dev, int32_t *rank_dev, lora_stream_t stream) {
    if (!pa || !pb || !page_table_dev || !scale_dev || !rank_dev) return LORA_ERR_INVALID_ARG;
    if (num_slots < 1 || num_slots > LORA_MAX_SLOTS) return LORA_ERR_INVALID_ARG;
    if (slot < 0 || slot >= num_slots) return LORA_ERR_BAD_SLOT;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    lora_pool_s *pools[2] = {pa, pb};
    std::unique_lock<std::mutex> l1, l2;
    if (pa == pb) {
        l1 = std::unique_lock<std::mutex>(pa->mu);
    } else if (pa < pb) {
        l1 = std::unique_lock<std::mutex>(pa->mu);
        l2 = std::unique_lock<std::mutex>(pb->mu);
    } else {
        l1 = std::unique_lock<std::mutex>(pb->mu);
        l2 = std::unique_lock<std::mutex>(pa->mu);
    }
    bool found = false;
    for (int m = 0; m < 2; ++m) {
        auto key = std::make_tuple((const void *)page_table_dev, slot, m);
        auto it = pools[m]->owners.find(key);
        if (it != pools[m]->owners.end()) {
            found = true;
            give_pages(pools[m], it->second);
            pools[m]->owners.erase(it);
        }
    }
    if (!found) return LORA_ERR_BAD_SLOT;
    set_slot_kernel<<<1, 32, 0, st>>>(page_table_dev, scale_dev, rank_dev, slot, make_int4(-1, -1, -1, -1),
                                      make_int4(-1, -1, -1, -1), 0.f, 0);
    return cuda_check(cudaGetLastError());
}

int lora_pool_read_row(lora_pool_t pool, const int32_t *page_table_dev, int num_slots, int slot, int m, int k,
                       uint16_t *out_dev, lora_stream_t stream) {
    if (!pool || !page_table_dev || !out_dev || m < 0 || m > 1 || k < 0 || k >= LORA_MAX_RANK) return LORA_ERR_INVALID_ARG;
    if (slot < 0 || slot >= num_slots) return LORA_ERR_BAD_SLOT;
    {
        std::lock_guard<std::mutex> g(pool->mu);
        auto it = pool->owners.find(std::make_tuple((const void *)page_table_dev, slot, m));
        if (it == pool->owners.end() || k >= (int)it->second.size() * LORA_PAGE_ROWS) return LORA_ERR_BAD_SLOT;
    }
    read_row_kernel<<<4, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(pool->base, pool->width, page_table_dev,
                                                                           slot, m, k, out_dev);
    return cuda_check(cudaGetLastError());
}

size_t lora_workspace_size(int T, int num_slots) {
    if (T < 0 || num_slots < 1) return 0;
    return ws_layout(T, num_slots).total;
}

static int check_common(int T, int num_slots, const int32_t *ids, const int32_t *ranks, void *ws, size_t ws_bytes) {
    if (T < 0 || num_slots < 1 || num_slots > LORA_MAX_SLOTS) return LORA_ERR_INVALID_ARG;
    if (T > 0 && (!ids || !ranks)) return LORA_ERR_INVALID_ARG;
    if (!ws || ws_bytes < ws_layout(T, num_slots).total || !aligned(ws, 256)) return LORA_ERR_WORKSPACE;
    return LORA_OK;
}

static PlanOut plan_out(void *ws, int T, int S, int32_t *perm_out, int32_t *seg_out) {
    PlanOut o = plan_in_ws(ws, T, S);
    o.perm_copy = perm_out;
    o.seg_start_copy = seg_out;
    return o;
}

static bool plan_uses_tiles(int T) {
    return tiles_supported() && opt_long_segment() > 0 && T >= opt_long_segment();
}

static GatherProj gather_proj(float *Y, int d_out, const int32_t *ranks, const float *scales,
                              const int32_t *page_table, const lora_pool_s *pa, const lora_pool_s *pb) {
    GatherProj g = {};
    g.Y = Y; g.d_out = d_out; g.ldy = d_out; g.ranks = ranks; g.scales = scales; g.pt = page_table;
    g.rowsA = pa ? (long long)pa->num_pages * LORA_PAGE_ROWS : 0;
    g.rowsB = pb ? (long long)pb->num_pages * LORA_PAGE_ROWS : 0;
    return g;
}

// The tensor-core launch of a plan with long runs: one for all projections.
static int run_tiles(const uint16_t *X, int T, int d_in, const lora_projection_t *pr, int nproj, const PlanOut &o,
                     float *vpart, int32_t *err_dev, cudaStream_t st) {
    if (!plan_uses_tiles(T)) return LORA_OK;
    TileArgs ta = {};
    ta.X = X; ta.T = T; ta.d_in = d_in; ta.nproj = nproj;
    for (int p = 0; p < nproj; ++p) {
        TileProj &q = ta.proj[p];
        q.Y = pr[p].Y; q.d_out = pr[p].d_out; q.ranks = pr[p].ranks; q.scales = pr[p].scales;
        q.pt = pr[p].page_table; q.pa = pr[p].pa; q.pb = pr[p].pb;
    }
    ta.tiles = o.tiles; ta.hdr = o.header; ta.err = err_dev; ta.long_thresh = opt_long_segment();
    ta.vpart = vpart;
    return launch_tiles(ta, st, true);
}

// Which gather path a call takes (both give bit-identical results).
// LORA_GATHER_AUTO: the split path where many distinct adapters are likely
// (a pool of at least kSplitMinSlots slots and at least kSplitMinTokens
// tokens, one projection).  Measured on B200 at the 7B/8B shapes, the cluster
// kernel takes 18-30 % less time with few gather jobs (decode over a small
// pool, one shared adapter, mixed-rank MLPs over 128 slots), the split pair
// with many (64 and 512 distinct rank-64 adapters at d_out 14336: 7 % and 26 %
// less).  The job count itself is known only on the device, so the host
// decides from the pool size and the token count (one shared adapter over a
// large pool at 64 tokens takes the split pair and 27 % longer).
constexpr int kSplitMinSlots = 256;
constexpr int kSplitMinTokens = 64;

static bool use_split(int nproj, int T, int num_slots) {
    const int p = opt_gather_path();
    if (p == LORA_GATHER_SPLIT) return true;
    if (p == LORA_GATHER_CLUSTER) return false;
    return nproj == 1 && num_slots >= kSplitMinSlots && T >= kSplitMinTokens;
}

// The apply kernels over a plan already in ws: the short segments of every
// projection through the gather path (one cluster-kernel launch for all
// projections, or a shrink + expand pair per projection), then (when the plan
// has long runs) one tile launch per projection.
static int run_planned(const uint16_t *X, int T, int d_in, int num_slots, const lora_projection_t *pr, int nproj,
                       void *ws, int32_t *err_dev, cudaStream_t st) {
    const PlanOut o = plan_out(ws, T, num_slots, nullptr, nullptr);
    // per-quarter partials of v: the split gather pair's (by short-token
    // position), then the tile shrink's (by token); the tile launches wait for
    // the gather kernels before they write
    float *vpart = reinterpret_cast<float *>(static_cast<char *>(ws) + ws_layout(T, num_slots).vpart);
    if (use_split(nproj, T, num_slots)) {
        for (int p = 0; p < nproj; ++p) {
            SplitArgs s = {};
            s.X = X; s.Y = pr[p].Y; s.T = T; s.d_in = d_in; s.d_out = pr[p].d_out; s.S = num_slots;
            s.ranks = pr[p].ranks; s.scales = pr[p].scales; s.pt = pr[p].page_table;
            s.perm = o.perm_short; s.jobs = o.jobs; s.hdr = o.header; s.vpart = vpart; s.err = err_dev;
            if (int rc = launch_split(s, pr[p].pa, pr[p].pb, st)) return rc;
        }
        return run_tiles(X, T, d_in, pr, nproj, o, vpart, err_dev, st);
    }
    GatherArgs a = {};
    a.X = X; a.T = T; a.d_in = d_in; a.S = num_slots; a.nproj = nproj;
    lora_pool_s *pa[LORA_MAX_PROJECTIONS], *pb[LORA_MAX_PROJECTIONS];
    for (int p = 0; p < nproj; ++p) {
        a.proj[p] = gather_proj(pr[p].Y, pr[p].d_out, pr[p].ranks, pr[p].scales, pr[p].page_table, pr[p].pa, pr[p].pb);
        pa[p] = pr[p].pa;
        pb[p] = pr[p].pb;
    }
    a.perm = o.perm_short; a.jobs = o.jobs; a.hdr = o.header; a.err = err_dev;
    if (int rc = launch_gather(kApply, a, pa, pb, st, true)) return rc;
    return run_tiles(X, T, d_in, pr, nproj, o, vpart, err_dev, st);
}

static lora_projection_t one_proj(float *Y, int d_out, const int32_t *ranks, const float *scales,
                                  const int32_t *page_table, lora_pool_t pa, lora_pool_t pb) {
    lora_projection_t p;
    p.Y = Y; p.d_out = d_out; p.ranks = ranks; p.scales = scales; p.page_table = page_table; p.pa = pa; p.pb = pb;
    return p;
}

int lora_plan(const int32_t *ids, int T, const int32_t *ranks, int num_slots, int32_t *perm_out,
              int32_t *seg_start_out, void *ws, size_t ws_bytes, int32_t *err_dev, lora_stream_t stream) {
    reset_launch_count();
    if (int rc = check_common(T, num_slots, ids, ranks, ws, ws_bytes)) return rc;
    const PlanOut o = plan_out(ws, T, num_slots, perm_out, seg_start_out);
    return launch_plan(ids, T, ranks, num_slots, plan_uses_tiles(T) ? opt_long_segment() : 0, opt_job_tokens(),
                       o, err_dev, reinterpret_cast<cudaStream_t>(stream));
}

int lora_apply_planned(const uint16_t *X, float *Y, int T, int d_in, int d_out, int num_slots, const int32_t *ranks,
                       const float *scales, const int32_t *page_table, lora_pool_t pa, lora_pool_t pb, void *ws,
                       size_t ws_bytes, int32_t *err_dev, lora_stream_t stream) {
    reset_launch_count();
    if (T < 0 || num_slots < 1 || num_slots > LORA_MAX_SLOTS || !ranks) return LORA_ERR_INVALID_ARG;
    if (!ws || ws_bytes < ws_layout(T, num_slots).total || !aligned(ws, 256)) return LORA_ERR_WORKSPACE;
    if (!pa || !pb) return LORA_ERR_INVALID_ARG;
    if (pa->width != d_in || pb->width != d_out) return LORA_ERR_WIDTH_MISMATCH;
    if (T == 0) return LORA_OK;
    if (!X || !Y || !scales || !page_table || !aligned(X, 16) || !aligned(Y, 16)) return LORA_ERR_INVALID_ARG;
    const lora_projection_t pr = one_proj(Y, d_out, ranks, scales, page_table, pa, pb);
    return run_planned(X, T, d_in, num_slots, &pr, 1, ws, err_dev, reinterpret_cast<cudaStream_t>(stream));
}

int lora_shrink(const uint16_t *X, int T, int d_in, const int32_t *ids, int num_slots, const int32_t *ranks,
                const int32_t *page_table, lora_pool_t pa, float *V, void *ws, size_t ws_bytes, int32_t *err_dev,
                lora_stream_t stream) {
    reset_launch_count();
    if (int rc = check_common(T, num_slots, ids, ranks, ws, ws_bytes)) return rc;
    if (!pa) return LORA_ERR_INVALID_ARG;
    if (pa->width != d_in) return LORA_ERR_WIDTH_MISMATCH;
    if (T == 0) return LORA_OK;
    if (!X || !V || !page_table || !aligned(X, 16)) return LORA_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const PlanOut o = plan_out(ws, T, num_slots, nullptr, nullptr);
    if (int rc = launch_plan(ids, T, ranks, num_slots, 0, opt_job_tokens(), o, err_dev, st)) return rc;
    GatherArgs a = {};
    a.X = X; a.V = V; a.T = T; a.d_in = d_in; a.S = num_slots; a.nproj = 1;
    a.proj[0] = gather_proj(nullptr, 8, ranks, nullptr, page_table, pa, nullptr);
    a.perm = o.perm_short; a.jobs = o.jobs; a.hdr = o.header; a.err = err_dev;
    lora_pool_s *pp[1] = {pa};
    return launch_gather(kShrink, a, pp, pp, st, true);
}

int lora_expand_add(const float *V, float *Y, int T, int d_out, const int32_t *ids, int num_slots,
                    const int32_t *ranks, const float *scales, const int32_t *page_table, lora_pool_t pb, void *ws,
                    size_t ws_bytes, int32_t *err_dev, lora_stream_t stream) {
    return lora_expand_add_strided(V, Y, d_out, T, d_out, ids, num_slots, ranks, scales, page_table, pb, ws, ws_bytes,
                                   err_dev, stream);
}

int lora_expand_add_strided(const float *V, float *Y, int ldy, int T, int d_out, const int32_t *ids, int num_slots,
                            const int32_t *ranks, const float *scales, const int32_t *page_table, lora_pool_t pb,
                            void *ws, size_t ws_bytes, int32_t *err_dev, lora_stream_t stream) {
    reset_launch_count();
    if (int rc = check_common(T, num_slots, ids, ranks, ws, ws_bytes)) return rc;
    if (!pb) return LORA_ERR_INVALID_ARG;
    if (pb->width != d_out) return LORA_ERR_WIDTH_MISMATCH;
    if (ldy < d_out || (ldy % 4) != 0) return LORA_ERR_INVALID_ARG;
    if (T == 0) return LORA_OK;
    if (!V || !Y || !scales || !page_table || !aligned(Y, 16)) return LORA_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const PlanOut o = plan_out(ws, T, num_slots, nullptr, nullptr);
    if (int rc = launch_plan(ids, T, ranks, num_slots, 0, opt_job_tokens(), o, err_dev, st)) return rc;
    GatherArgs a = {};
    a.V = const_cast<float *>(V); a.T = T; a.d_in = 8; a.S = num_slots; a.nproj = 1;
    a.proj[0] = gather_proj(Y, d_out, ranks, scales, page_table, nullptr, pb);
    a.proj[0].ldy = ldy;
    a.perm = o.perm_short; a.jobs = o.jobs; a.hdr = o.header; a.err = err_dev;
    lora_pool_s *pp[1] = {pb};
    return launch_gather(kExpand, a, pp, pp, st, true);
}

int lora_apply(const uint16_t *X, float *Y, int T, int d_in, int d_out, const int32_t *ids, int num_slots,
               const int32_t *ranks, const float *scales, const int32_t *page_table, lora_pool_t pa, lora_pool_t pb,
               void *ws, size_t ws_bytes, int32_t *err_dev, lora_stream_t stream) {
    reset_launch_count();
    if (int rc = check_common(T, num_slots, ids, ranks, ws, ws_bytes)) return rc;
    if (!pa || !pb) return LORA_ERR_INVALID_ARG;
    if (pa->width != d_in || pb->width != d_out) return LORA_ERR_WIDTH_MISMATCH;
    if (T == 0) return LORA_OK;
    if (!X || !Y || !scales || !page_table || !aligned(X, 16) || !aligned(Y, 16)) return LORA_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const PlanOut o = plan_out(ws, T, num_slots, nullptr, nullptr);
    const int long_thresh = plan_uses_tiles(T) ? opt_long_segment() : 0;
    if (int rc = launch_plan(ids, T, ranks, num_slots, long_thresh, opt_job_tokens(), o, err_dev, st)) return rc;
    const lora_projection_t pr = one_proj(Y, d_out, ranks, scales, page_table, pa, pb);
    return run_planned(X, T, d_in, num_slots, &pr, 1, ws, err_dev, st);
}

// Checks of the projection list shared by the two multi-projection calls
// (the sizes, ids and workspace are checked by the caller).
static int check_projs(const uint16_t *X, int T, int d_in, const lora_projection_t *projs, int num_projs) {
    for (int p = 0; p < num_projs; ++p) {
        const lora_projection_t &q = projs[p];
        if (!q.pa || !q.pb || !q.ranks) return LORA_ERR_INVALID_ARG;
        if (q.pa->width != d_in || q.pb->width != q.d_out) return LORA_ERR_WIDTH_MISMATCH;
    }
    if (T == 0) return LORA_OK;
    if (!X || !aligned(X, 16)) return LORA_ERR_INVALID_ARG;
    for (int p = 0; p < num_projs; ++p) {
        const lora_projection_t &q = projs[p];
        if (!q.Y || !q.scales || !q.page_table || !aligned(q.Y, 16)) return LORA_ERR_INVALID_ARG;
    }
    return LORA_OK;
}

int lora_apply_multi_planned(const uint16_t *X, int T, int d_in, int num_slots, const lora_projection_t *projs,
                             int num_projs, void *ws, size_t ws_bytes, int32_t *err_dev, lora_stream_t stream) {
    reset_launch_count();
    if (!projs || num_projs < 1 || num_projs > LORA_MAX_PROJECTIONS) return LORA_ERR_INVALID_ARG;
    if (T < 0 || num_slots < 1 || num_slots > LORA_MAX_SLOTS) return LORA_ERR_INVALID_ARG;
    if (!ws || ws_bytes < ws_layout(T, num_slots).total || !aligned(ws, 256)) return LORA_ERR_WORKSPACE;
    if (int rc = check_projs(X, T, d_in, projs, num_projs)) return rc;
    if (T == 0) return LORA_OK;
    return run_planned(X, T, d_in, num_slots, projs, num_projs, ws, err_dev, reinterpret_cast<cudaStream_t>(stream));
}

int lora_apply_multi(const uint16_t *X, int T, int d_in, const int32_t *ids, int num_slots,
                     const lora_projection_t *projs, int num_projs, void *ws, size_t ws_bytes, int32_t *err_dev,
                     lora_stream_t stream) {
    reset_launch_count();
    if (!projs || num_projs < 1 || num_projs > LORA_MAX_PROJECTIONS) return LORA_ERR_INVALID_ARG;
    if (int rc = check_common(T, num_slots, ids, projs[0].ranks, ws, ws_bytes)) return rc;
    if (int rc = check_projs(X, T, d_in, projs, num_projs)) return rc;
    if (T == 0) return LORA_OK;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    const PlanOut o = plan_out(ws, T, num_slots, nullptr, nullptr);
    const int long_thresh = plan_uses_tiles(T) ? opt_long_segment() : 0;
    if (int rc = launch_plan(ids, T, projs[0].ranks, num_slots, long_thresh, opt_job_tokens(), o, err_dev, st,
                             num_projs))
        return rc;
    return run_planned(X, T, d_in, num_slots, projs, num_projs, ws, err_dev, st);
}

int lora_set_option(int key, int value) {
    switch (key) {
        case LORA_OPT_LONG_SEGMENT:
            if (value < 0) return LORA_ERR_INVALID_ARG;
            g_long_segment.store(value);
            return LORA_OK;
        case LORA_OPT_DECODE_JOB_TOKENS:
            if (value < 1 || value > LORA_MAX_JOB_TOKENS) return LORA_ERR_INVALID_ARG;
            g_job_tokens.store(value);
            return LORA_OK;
        case LORA_OPT_GATHER_PATH:
            if (value < LORA_GATHER_AUTO || value > LORA_GATHER_SPLIT) return LORA_ERR_INVALID_ARG;
            g_gather_path.store(value);
            return LORA_OK;
        case LORA_OPT_PLAN_KERNEL:
            if (value < LORA_PLAN_AUTO || value > LORA_PLAN_GENERAL) return LORA_ERR_INVALID_ARG;
            g_plan_kernel.store(value);
            return LORA_OK;
    }
    return LORA_ERR_INVALID_ARG;
}

int lora_get_option(int key) {
    switch (key) {
        case LORA_OPT_LONG_SEGMENT: return g_long_segment.load();
        case LORA_OPT_DECODE_JOB_TOKENS: return g_job_tokens.load();
        case LORA_OPT_GATHER_PATH: return g_gather_path.load();
        case LORA_OPT_PLAN_KERNEL: return g_plan_kernel.load();
    }
    return LORA_ERR_INVALID_ARG;
}

const char *lora_last_cuda_error(void) { return t_last_cuda_error; }

int lora_last_launch_count(void) { return t_launches; }

}  // extern "C"
