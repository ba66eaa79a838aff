// Internal declarations shared by the liblora translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <map>
#include <mutex>
#include <tuple>
#include <vector>

#include "lora.h"

namespace lora {

// ---------------------------------------------------------------------------
// Workspace layout.  All offsets are 256-byte aligned.
// ---------------------------------------------------------------------------
struct PlanHeader {
    int n_valid;      // tokens with a valid adapter
    int n_seg;        // distinct slots present
    int n_jobs;       // gather jobs (short segments)
    int n_tiles;      // tensor-core tiles (long, contiguous segments)
    int T;
    int S;
    int job_tokens;
    int long_thresh;
};

struct WsLayout {
    size_t header, seg_start, perm, perm_short, run_start, run_end, jobs, tiles;
    size_t plan_total;   // bytes of the plan (everything above)
    size_t vpart;        // split gather path: fp32 partials [4][T][LORA_MAX_RANK]
    size_t total;
};

constexpr size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// constexpr so that the fixed scratch of lora_apply_noalloc can be sized from it.
constexpr WsLayout ws_layout(int T, int S) {
    WsLayout l{};
    const size_t t = (size_t)(T > 0 ? T : 1);
    size_t o = 0;
    l.header = o;     o = align_up(o + sizeof(PlanHeader), 256);
    l.seg_start = o;  o = align_up(o + sizeof(int32_t) * (size_t)(S + 1), 256);
    l.perm = o;       o = align_up(o + sizeof(int32_t) * t, 256);
    l.perm_short = o; o = align_up(o + sizeof(int32_t) * t, 256);
    l.run_start = o;  o = align_up(o + sizeof(int32_t) * t, 256);
    l.run_end = o;    o = align_up(o + sizeof(int32_t) * t, 256);
    l.jobs = o;       o = align_up(o + 2 * sizeof(int4) * t, 256);   // two int4 per job
    l.tiles = o;      o = align_up(o + sizeof(int4) * t, 256);
    l.plan_total = o;
    l.vpart = o;      o = align_up(o + 4 * t * LORA_MAX_RANK * sizeof(float), 256);
    l.total = o;
    return l;
}

// Tile height of the tensor-core path (tokens per tile).
constexpr int kTileM = 128;

// ---------------------------------------------------------------------------
// Page pool (host side).
// ---------------------------------------------------------------------------
}  // namespace lora

struct lora_pool_s {
    uint16_t *base = nullptr;
    size_t bytes = 0;
    int width = 0;
    int page_rows = 0;
    int num_pages = 0;
    std::vector<int> free_stack;            // free page ids
    std::vector<char> used;                 // per page: 0 free, 1 an adapter's, 2 taken by lora_pool_alloc_pages
    // (page table identity, slot, matrix) -> pages owned
    std::map<std::tuple<const void *, int, int>, std::vector<int>> owners;
    std::mutex mu;
    // TMA descriptors of the pool, built on first use (see pool_tensor_map)
    CUtensorMap tmap;
    bool tmap_ok = false;
    CUtensorMap tmap4;       // 4 consecutive 64-column blocks per box (pool_tensor_map4)
    bool tmap4_ok = false;
};

namespace lora {

// TMA tensor maps (cuTensorMapEncodeTiled through the runtime's driver entry point).
bool tma_supported();
int make_tensor_map(CUtensorMap *m, CUtensorMapDataType dt, int esize, const void *base, uint64_t cols,
                    uint64_t rows, uint32_t box_cols, uint32_t box_rows, bool swizzle128);
// The pool's map: a box is 64 columns x 16 rows (one page high), 128-byte swizzle.
int pool_tensor_map(lora_pool_s *pool, CUtensorMap *out);
// The pool seen in 3D, (column, row, 64-column step): one box (64, 16, 4) lands
// the same shared-memory bytes as four boxes of the 2D map at columns x, x+64,
// x+128, x+192 (valid for x + 256 <= width), with one TMA operation instead of
// four.  Only for widths of at least 256 (LORA_ERR_INVALID_ARG otherwise).
int pool_tensor_map4(lora_pool_s *pool, CUtensorMap *out);

// Process-wide options.
int opt_long_segment();
int opt_job_tokens();
int opt_gather_path();
int opt_plan_kernel();

// Record a CUDA error and return LORA_ERR_CUDA, or LORA_OK.
int cuda_check(cudaError_t e);

// Programmatic launches.  Every library kernel that lets its dependents start
// early (griddepcontrol.launch_dependents) does so only after its own
// griddepcontrol.wait, and waits before it exits; the plan kernel, which
// triggers at once, is launched without the programmatic attribute.  So when
// a library kernel starts, everything launched on its stream before the
// kernel just ahead of it has completed and is visible.  The library records,
// per stream, whether its last launch there was the plan: if not, the plan
// a launch reads is complete before the launch starts, and the kernel may
// read it (and the adapter pages it names) before its own wait.
bool plan_was_last_launch(cudaStream_t st);
void note_launch(cudaStream_t st, bool is_plan);

// Per-thread launch counter for diagnostics.
void count_launch(int n = 1);
void reset_launch_count();

// Kernel launchers (each returns LORA_OK or an error code).
struct PlanOut {
    PlanHeader *header;
    int32_t *seg_start;
    int32_t *perm;
    int32_t *perm_short;       // perm without the tokens of long runs (gather jobs index it)
    int32_t *run_start;        // per token: first token of its run (scratch)
    int32_t *run_end;          // per token: last token of its run if the run is long, else -1
    int4 *jobs;                // per job: {slot, count, 0, 0}, {token 0..3 (-1 pad)}
    int4 *tiles;
    int32_t *perm_copy;        // optional second destination of perm (caller's buffer)
    int32_t *seg_start_copy;   // optional second destination of seg_start
};

// Pointers of the plan inside a workspace laid out by ws_layout(T, S).
inline PlanOut plan_in_ws(void *ws, int T, int S) {
    const WsLayout l = ws_layout(T, S);
    char *b = static_cast<char *>(ws);
    PlanOut o;
    o.header = reinterpret_cast<PlanHeader *>(b + l.header);
    o.seg_start = reinterpret_cast<int32_t *>(b + l.seg_start);
    o.perm = reinterpret_cast<int32_t *>(b + l.perm);
    o.perm_short = reinterpret_cast<int32_t *>(b + l.perm_short);
    o.run_start = reinterpret_cast<int32_t *>(b + l.run_start);
    o.run_end = reinterpret_cast<int32_t *>(b + l.run_end);
    o.jobs = reinterpret_cast<int4 *>(b + l.jobs);
    o.tiles = reinterpret_cast<int4 *>(b + l.tiles);
    o.perm_copy = nullptr;
    o.seg_start_copy = nullptr;
    return o;
}
// units_per_job: gather units each job becomes (projections sharing the plan);
// the job size rule then counts clusters / units_per_job.
int launch_plan(const int32_t *ids, int T, const int32_t *ranks, int S, int long_thresh,
                int job_tokens, const PlanOut &out, int32_t *err_dev, cudaStream_t st, int units_per_job = 1);

enum GatherMode { kApply = 0, kShrink = 1, kExpand = 2 };

// One adapted projection of a gather launch: its output and slot tables.
struct GatherProj {
    float *Y;           // [T][ldy] fp32, columns [0, d_out) updated in place
    int d_out;
    int ldy;            // row stride of Y in elements (>= d_out, a multiple of 4)
    const int32_t *ranks;
    const float *scales;
    const int32_t *pt;
    long long rowsA;    // rows in the A pool (pages * 16); 0 when unused
    long long rowsB;
};

struct GatherArgs {
    const uint16_t *X;
    float *V;
    int T, d_in;
    int S;              // slots in every projection's tables
    int nproj;          // projections sharing X and the plan (1..LORA_MAX_PROJECTIONS)
    GatherProj proj[LORA_MAX_PROJECTIONS];
    const int32_t *perm;
    const int4 *jobs;
    const PlanHeader *hdr;
    int32_t *err;
};
// pa[p], pb[p]: the pools of projection p.
int launch_gather(GatherMode mode, const GatherArgs &a, lora_pool_s *const *pa, lora_pool_s *const *pb,
                  cudaStream_t st, bool pdl);
// Clusters the gather kernel keeps resident on the current device (its grid
// size in clusters when there is enough work).
int gather_clusters(int *out);

// One projection of a tile launch: its output, slot tables and pools.
struct TileProj {
    float *Y;            // [T][d_out] fp32, in place
    int d_out;
    const int32_t *ranks;
    const float *scales;
    const int32_t *pt;
    const lora_pool_s *pa;
    const lora_pool_s *pb;
};

struct TileArgs {
    const uint16_t *X;
    int T, d_in;
    int nproj;           // projections sharing X and the plan (1..LORA_MAX_PROJECTIONS)
    TileProj proj[LORA_MAX_PROJECTIONS];
    const int4 *tiles;
    const PlanHeader *hdr;
    int32_t *err;
    int long_thresh;     // long-segment threshold the plan used
    float *vpart;        // workspace for v's per-quarter partials ([4][T][64] fp32), or null: with one
                         // projection and vpart set, the shrink of every tile runs once in its own
                         // launch and a second launch streams B and Y; else one fused launch
};
int launch_tiles(const TileArgs &a, cudaStream_t st, bool pdl);
bool tiles_supported();

// Split gather path (shrink kernel writing per-quarter partials, then an
// expand kernel), bit-identical to the cluster gather kernel in apply mode.
struct SplitArgs {
    const uint16_t *X;
    float *Y;
    int T, d_in, d_out, S;
    const int32_t *ranks;
    const float *scales;
    const int32_t *pt;
    const int32_t *perm;     // the plan's short-token list
    const int4 *jobs;
    const PlanHeader *hdr;
    float *vpart;            // workspace region WsLayout::vpart
    int32_t *err;
};
int launch_split(const SplitArgs &s, lora_pool_s *pa, lora_pool_s *pb, cudaStream_t st);

}  // namespace lora
