// lora_apply_noalloc: the fused adapter branch for callers that cannot
// allocate device memory.
//
// lora_apply needs a caller-provided workspace for the segment plan.  Some
// callers have no way to get one: a plug-in running inside a host framework
// that owns every byte of device memory through its own pool and forbids
// outside allocations, or a latency-critical serving loop that must not call
// cudaMalloc/cudaFree because those calls can synchronise the whole device.
// This entry point serves them: it keeps the plan in a fixed scratch array
// that is part of the library's device image, so the library itself never
// allocates.  The array is a file-scope __device__ variable; each GPU that
// loads the library holds it (LORA_NOALLOC_SCRATCH_BYTES) until the process
// exits.
#include <mutex>

#include "lora_internal.cuh"

namespace lora {
namespace {

// The shared scratch.  In host code the name g_noalloc_scratch is only a
// host-side stand-in, not a device address: its device address is taken
// once per device with cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[LORA_NOALLOC_SCRATCH_BYTES];

// The scratch holds the whole plan of the largest call the entry point admits.
static_assert(ws_layout(LORA_NOALLOC_MAX_TOKENS, LORA_MAX_SLOTS).plan_total <= (size_t)LORA_NOALLOC_SCRATCH_BYTES,
              "LORA_NOALLOC_SCRATCH_BYTES is smaller than the plan of LORA_NOALLOC_MAX_TOKENS tokens and "
              "LORA_MAX_SLOTS slots");

std::mutex g_noalloc_mu;
void *g_noalloc_ptr[64] = {};

// Device address of the scratch array on the current device, looked up on the
// first call made on that device and kept for the life of the process.  The
// address belongs to the device's primary context: a cudaDeviceReset makes it
// stale, so a process that resets a device must not call this entry point on
// that device again.
int noalloc_scratch(void **out) {
    int dev = 0;
    if (int rc = cuda_check(cudaGetDevice(&dev))) return rc;
    if (dev < 0 || dev >= 64) return LORA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> g(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        if (int rc = cuda_check(cudaGetSymbolAddress(&p, g_noalloc_scratch))) return rc;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return LORA_OK;
}

bool is_aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace
}  // namespace lora

using namespace lora;

extern "C" int lora_apply_noalloc(const uint16_t *X, float *Y, int T, int d_in, int d_out, const int32_t *ids,
                                  int num_slots, const int32_t *ranks, const float *scales,
                                  const int32_t *page_table, lora_pool_t pa, lora_pool_t pb, int32_t *err_dev,
                                  lora_stream_t stream) {
    reset_launch_count();
    if (T < 0 || num_slots < 1 || num_slots > LORA_MAX_SLOTS) return LORA_ERR_INVALID_ARG;
    if (T > LORA_NOALLOC_MAX_TOKENS) return LORA_ERR_TOO_LARGE;
    const WsLayout l = ws_layout(T, num_slots);
    if (l.plan_total > (size_t)LORA_NOALLOC_SCRATCH_BYTES) return LORA_ERR_TOO_LARGE;
    if (T > 0 && (!ids || !ranks)) return LORA_ERR_INVALID_ARG;
    if (!pa || !pb) return LORA_ERR_INVALID_ARG;
    if (pa->width != d_in || pb->width != d_out) return LORA_ERR_WIDTH_MISMATCH;
    if (T == 0) return LORA_OK;
    if (!X || !Y || !scales || !page_table || !is_aligned(X, 16) || !is_aligned(Y, 16)) return LORA_ERR_INVALID_ARG;

    void *ws = nullptr;
    if (int rc = noalloc_scratch(&ws)) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

    // The launch sequence of lora_apply with the cluster gather kernel, which
    // needs nothing beyond the plan (lora_apply may take the split gather path
    // instead, whose result is bit-identical), and the plan kept in the
    // scratch.  Every word the compute kernels read is written by the plan
    // kernel of the same call first, so nothing in the scratch has to start at
    // zero.
    const PlanOut o = plan_in_ws(ws, T, num_slots);
    const bool use_tiles = tiles_supported() && opt_long_segment() > 0 && T >= opt_long_segment();
    const int long_thresh = use_tiles ? opt_long_segment() : 0;
    if (int rc = launch_plan(ids, T, ranks, num_slots, long_thresh, opt_job_tokens(), o, err_dev, st)) return rc;

    GatherArgs a = {};
    a.X = X; a.T = T; a.d_in = d_in; a.S = num_slots; a.nproj = 1;
    a.proj[0].Y = Y; a.proj[0].d_out = d_out; a.proj[0].ldy = d_out; a.proj[0].ranks = ranks;
    a.proj[0].scales = scales;
    a.proj[0].pt = page_table;
    a.proj[0].rowsA = (long long)pa->num_pages * LORA_PAGE_ROWS;
    a.proj[0].rowsB = (long long)pb->num_pages * LORA_PAGE_ROWS;
    a.perm = o.perm_short; a.jobs = o.jobs; a.hdr = o.header; a.err = err_dev;
    lora_pool_s *ppa[1] = {pa}, *ppb[1] = {pb};
    if (int rc = launch_gather(kApply, a, ppa, ppb, st, true)) return rc;
    if (use_tiles) {
        TileArgs ta = {};
        ta.X = X; ta.T = T; ta.d_in = d_in; ta.nproj = 1;
        ta.proj[0].Y = Y; ta.proj[0].d_out = d_out; ta.proj[0].ranks = ranks; ta.proj[0].scales = scales;
        ta.proj[0].pt = page_table; ta.proj[0].pa = pa; ta.proj[0].pb = pb;
        ta.tiles = o.tiles; ta.hdr = o.header; ta.err = err_dev; ta.long_thresh = long_thresh;
        if (int rc = launch_tiles(ta, st, true)) return rc;
    }
    return LORA_OK;
}
