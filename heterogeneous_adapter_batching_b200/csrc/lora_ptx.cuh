// Thin inline-PTX wrappers used by the split shrink / expand kernels: mbarriers
// with bounded waits, TMA tile loads, bulk copies, warp-level MMA fragments.
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace lora {
namespace ptx {

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

// Arrive (release at CTA scope) without a transaction count.
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

// 2D tiled TMA load of one box into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *m, int x, int y, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
        ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(y), "r"(smem_u32(bar)) : "memory");
}

// 3D tiled TMA load of one box into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *m, int x, int y, int z, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
        "[%5];" ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
        : "memory");
}

// The page boxes of one chunk: for page p (rows pg * 16 ...) the 64-column
// blocks b = 0 .. boxes-1 starting at column c0, written at dst + (p * nb + b)
// * 2 KB.  Lane i (< np * ceil(boxes / 4)) takes page i / ng, blocks 4 g ..
// 4 g + 3 of it: one 3D box when all four lie inside the row (m4 valid and
// c0 + 64 (4 g + 4) <= width), else one 2D box per block.
__device__ __forceinline__ void issue_page_boxes(int i, unsigned char *dst, const CUtensorMap *m2,
                                                 const CUtensorMap *m4, bool use4, int width, int np, int nb,
                                                 int boxes, int c0, int4 pages, uint64_t *bar) {
    const int ng = (boxes + 3) >> 2;
    if (i >= np * ng) return;
    const int p = i / ng, g = i - p * ng;
    const int pg = p == 0 ? pages.x : p == 1 ? pages.y : p == 2 ? pages.z : pages.w;
    const int b0 = 4 * g, b1 = b0 + 4 < boxes ? b0 + 4 : boxes;
    unsigned char *d = dst + (p * nb + b0) * 2048;
    if (use4 && b1 - b0 == 4 && c0 + 64 * b1 <= width) {
        tma_load_3d(d, m4, c0 + 64 * b0, pg * 16, 0, bar);
    } else {
        for (int b = b0; b < b1; ++b) tma_load_2d(dst + (p * nb + b) * 2048, m2, c0 + 64 * b, pg * 16, bar);
    }
}

// Contiguous bulk copy global -> shared (both 16-byte aligned, bytes a
// multiple of 16), completing on `bar`.
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t &r0, uint32_t &r1) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(addr) : "memory");
}
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr) : "memory");
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr) : "memory");
}

// d += a (16 x 16, row) * b (16 x 8, col); bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
                 "{%0, %1, %2, %3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint16_t bf16_rn(float f) {
    uint16_t h;
    asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(h) : "f"(f));
    return h;
}

__device__ __forceinline__ int4 ld_cg_v4(const int4 *p) {
    int4 v;
    asm volatile("ld.global.cg.v4.s32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}
__device__ __forceinline__ int ld_cg_s32(const int *p) {
    int v;
    asm volatile("ld.global.cg.s32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

// Byte offset of 16-byte group j of row t in a row-major shared array whose
// rows are a multiple of 128 bytes: groups XOR-swizzled by row, so the eight
// rows an ldmatrix reads sit in different banks.
__device__ __forceinline__ uint32_t swz(int t, int pitch, int j) { return (uint32_t)(t * pitch + ((j ^ (t & 7)) << 4)); }

}  // namespace ptx
}  // namespace lora
