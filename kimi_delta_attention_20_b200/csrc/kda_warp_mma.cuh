// Warp-level tensor-core helpers of the micro-chunk kernels (forward and backward):
// m16n8k16 bf16 MMA with fp32 accumulate, ldmatrix fragment loads from row-major bf16
// tiles (and their transposed forms), a zero-filling 16-byte cp.async, and small
// packing and exp2 helpers.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

#include "kda_sm100.cuh"
#include "kda_tc_util.cuh"

namespace kda {
namespace cw {

constexpr float kL2e = 1.4426950408889634f;

// ---- warp-level MMA
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldsm4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void ldsm4t(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
// Four 8 x 8 bf16 matrices from the MMA accumulator layout (lane: row lane / 4, columns
// 2 (lane % 4), + 1; register i = matrix i) to shared memory; lane l gives the address of
// stored row l % 8 of matrix l / 8. The .trans form stores each matrix transposed.
__device__ __forceinline__ void stsm4(uint32_t addr, uint32_t r0, uint32_t r1, uint32_t r2, uint32_t r3) {
    asm volatile("stmatrix.sync.aligned.m8n8.x4.shared.b16 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(r0), "r"(r1),
                 "r"(r2), "r"(r3)
                 : "memory");
}
__device__ __forceinline__ void stsm4t(uint32_t addr, uint32_t r0, uint32_t r1, uint32_t r2, uint32_t r3) {
    asm volatile("stmatrix.sync.aligned.m8n8.x4.trans.shared.b16 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(r0),
                 "r"(r1), "r"(r2), "r"(r3)
                 : "memory");
}
// Fragment loads of a row-major bf16 tile with rows of `ld` elements at shared address
// `base`. A (16 x 16 at (m0, k0)) from [M][K] storage, or from [K][M] storage (trans).
__device__ __forceinline__ void frag_a(uint32_t base, int ld, int m0, int k0, int lane, uint32_t (&a)[4]) {
    ldsm4(base + 2 * ((m0 + (lane & 7) + 8 * ((lane >> 3) & 1)) * ld + k0 + 8 * (lane >> 4)), a);
}
__device__ __forceinline__ void frag_at(uint32_t base, int ld, int m0, int k0, int lane, uint32_t (&a)[4]) {
    ldsm4t(base + 2 * ((k0 + (lane & 7) + 8 * (lane >> 4)) * ld + m0 + 8 * ((lane >> 3) & 1)), a);
}
// B for two n-tiles (n0 .. n0 + 15) x k0 .. k0 + 15: from [N][K] storage, or [K][N] (trans).
// b[0], b[1]: n-tile n0; b[2], b[3]: n-tile n0 + 8.
__device__ __forceinline__ void frag_b(uint32_t base, int ld, int n0, int k0, int lane, uint32_t (&b)[4]) {
    ldsm4(base + 2 * ((n0 + (lane & 7) + 8 * (lane >> 4)) * ld + k0 + 8 * ((lane >> 3) & 1)), b);
}
__device__ __forceinline__ void frag_bt(uint32_t base, int ld, int n0, int k0, int lane, uint32_t (&b)[4]) {
    ldsm4t(base + 2 * ((k0 + (lane & 7) + 8 * ((lane >> 3) & 1)) * ld + n0 + 8 * (lane >> 4)), b);
}
// 16-byte cp.async that zero-fills the destination when `valid` is false (no bytes read;
// the source address is still a valid one)
__device__ __forceinline__ void cp16z(void *sdst, const void *gsrc, bool valid) {
    const uint32_t d = sm100::smem_u32(sdst);
    const int n = valid ? 16 : 0;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(gsrc), "r"(n) : "memory");
}
__device__ __forceinline__ void stb2(uint8_t *p, float a, float b) {
    *reinterpret_cast<__nv_bfloat162 *>(p) = __floats2bfloat162_rn(a, b);
}
__device__ __forceinline__ float e2(float x) { return tcu::ex2a(x * kL2e); }

}  // namespace cw
}  // namespace kda
