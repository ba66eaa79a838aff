// TMA tensor maps: host-side encoding of the 2D tiled descriptors that the
// kernels' cp.async.bulk.tensor loads and stores use.  The encoder is the
// driver's cuTensorMapEncodeTiled, reached through the runtime's driver entry
// point so that the library does not link libcuda directly.
#include "lora_internal.cuh"

namespace lora {
namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static bool tried = false;
    if (!tried) {
        tried = true;
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

}  // namespace

bool tma_supported() { return encode_fn() != nullptr; }

// Row-major [rows][cols] tensor of esize-byte elements; a box is box_rows x
// box_cols.  Out-of-bounds elements of a box read as zero.
int make_tensor_map(CUtensorMap *m, CUtensorMapDataType dt, int esize, const void *base, uint64_t cols, uint64_t rows,
                    uint32_t box_cols, uint32_t box_rows, bool swizzle128) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return LORA_ERR_CUDA;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * (uint64_t)esize};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t es[2] = {1, 1};
    CUresult r = enc(m, dt, 2, const_cast<void *>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? LORA_OK : LORA_ERR_CUDA;
}

int pool_tensor_map(lora_pool_s *pool, CUtensorMap *out) {
    if (!pool) return LORA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> g(pool->mu);
    if (!pool->tmap_ok) {
        const uint64_t rows = (uint64_t)pool->num_pages * LORA_PAGE_ROWS;
        if (int rc = make_tensor_map(&pool->tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, pool->base,
                                     (uint64_t)pool->width, rows, 64, LORA_PAGE_ROWS, true))
            return rc;
        pool->tmap_ok = true;
    }
    *out = pool->tmap;
    return LORA_OK;
}

int pool_tensor_map4(lora_pool_s *pool, CUtensorMap *out) {
    if (!pool || pool->width < 256) return LORA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> g(pool->mu);
    if (!pool->tmap4_ok) {
        EncodeTiledFn enc = encode_fn();
        if (!enc) return LORA_ERR_CUDA;
        // element (x, y, z) at base + 2 x + 2 width y + 128 z; x < width - 192 keeps
        // every element of a box (x + 64 z + 63 < width) inside its row
        const cuuint64_t rows = (cuuint64_t)pool->num_pages * LORA_PAGE_ROWS;
        cuuint64_t dims[3] = {(cuuint64_t)pool->width - 192, rows, 4};
        cuuint64_t strides[2] = {(cuuint64_t)pool->width * 2, 128};
        cuuint32_t box[3] = {64, LORA_PAGE_ROWS, 4};
        cuuint32_t es[3] = {1, 1, 1};
        CUresult r = enc(&pool->tmap4, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, pool->base, dims, strides, box, es,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (r != CUDA_SUCCESS) return LORA_ERR_CUDA;
        pool->tmap4_ok = true;
    }
    *out = pool->tmap4;
    return LORA_OK;
}

}  // namespace lora
