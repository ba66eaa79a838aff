// Internal declarations shared by the liblora translation units.
#pragma once

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
    size_t header, seg_start, perm, jobs, tiles, total;
};

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

inline WsLayout ws_layout(int T, int S) {
    WsLayout l;
    size_t o = 0;
    l.header = o;    o = align_up(o + sizeof(PlanHeader), 256);
    l.seg_start = o; o = align_up(o + sizeof(int32_t) * (size_t)(S + 1), 256);
    l.perm = o;      o = align_up(o + sizeof(int32_t) * (size_t)(T > 0 ? T : 1), 256);
    l.jobs = o;      o = align_up(o + sizeof(int4) * (size_t)(T > 0 ? T : 1), 256);
    l.tiles = o;     o = align_up(o + sizeof(int4) * (size_t)(T > 0 ? T : 1), 256);
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
    std::vector<char> used;                 // per page
    // (page table identity, slot, matrix) -> pages owned
    std::map<std::tuple<const void *, int, int>, std::vector<int>> owners;
    std::mutex mu;
};

namespace lora {

// Process-wide options.
int opt_long_segment();
int opt_job_tokens();

// Record a CUDA error and return LORA_ERR_CUDA, or LORA_OK.
int cuda_check(cudaError_t e);

// Per-thread launch counter for diagnostics.
void count_launch(int n = 1);
void reset_launch_count();

// Kernel launchers (each returns LORA_OK or an error code).
struct PlanOut {
    PlanHeader *header;
    int32_t *seg_start;
    int32_t *perm;
    int4 *jobs;
    int4 *tiles;
    int32_t *perm_copy;        // optional second destination of perm (caller's buffer)
    int32_t *seg_start_copy;   // optional second destination of seg_start
};
int launch_plan(const int32_t *ids, int T, const int32_t *ranks, int S, int long_thresh,
                int job_tokens, const PlanOut &out, int32_t *err_dev, cudaStream_t st);

enum GatherMode { kApply = 0, kShrink = 1, kExpand = 2 };

struct GatherArgs {
    const uint16_t *X;
    float *Y;
    float *V;
    int T, d_in, d_out;
    const int32_t *ranks;
    const float *scales;
    const int32_t *pt;
    const uint16_t *poolA;
    const uint16_t *poolB;
    const int32_t *perm;
    const int4 *jobs;
    const PlanHeader *hdr;
    int32_t *err;
    long long rowsA;   // rows in the A pool (pages * 16); 0 when unused
    long long rowsB;
};
int launch_gather(GatherMode mode, const GatherArgs &a, cudaStream_t st, bool pdl);

struct TileArgs {
    const uint16_t *X;
    float *Y;
    int T, d_in, d_out;
    const int32_t *ranks;
    const float *scales;
    const int32_t *pt;
    const lora_pool_s *pa;
    const lora_pool_s *pb;
    const int4 *tiles;
    const PlanHeader *hdr;
    int32_t *err;
    long long rowsA;     // rows in the A pool (pages * 16)
    long long rowsB;     // rows in the B pool
    int long_thresh;     // long-segment threshold the plan used
};
int launch_tiles(const TileArgs &a, cudaStream_t st, bool pdl);
bool tiles_supported();

}  // namespace lora
