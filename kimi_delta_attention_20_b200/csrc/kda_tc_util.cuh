// Device and host helpers shared by the tensor-core chunk kernels: bf16
// packing, 128-bit shared-memory access, special-function-unit exp2/log2, the
// in-kernel gate on those units, a Newton reciprocal, and the TMA descriptor
// of a [T_total, H, 128] bf16 tensor.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include "kda_common.cuh"
#include "kda_sm100.cuh"

namespace kda {
namespace tcu {

using namespace sm100;

__device__ __forceinline__ void unpack8(const uint4 &u, float (&f)[8]) {
    const __nv_bfloat162 *b = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 t = __bfloat1622float2(b[i]);
        f[2 * i] = t.x;
        f[2 * i + 1] = t.y;
    }
}
__device__ __forceinline__ uint4 pack8(const float *f) {
    return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                      pack_bf16x2(f[6], f[7]));
}
__device__ __forceinline__ void sts128(uint8_t *base, uint32_t off, const uint4 &v) {
    *reinterpret_cast<uint4 *>(base + off) = v;
}
__device__ __forceinline__ uint4 lds128(const uint8_t *base, uint32_t off) {
    return *reinterpret_cast<const uint4 *>(base + off);
}
__device__ __forceinline__ float bf(const uint8_t *base, uint32_t off) {
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(base + off));
}
__device__ __forceinline__ void st_bf(uint8_t *base, uint32_t off, float x) {
    *reinterpret_cast<__nv_bfloat16 *>(base + off) = __float2bfloat16_rn(x);
}
__device__ __forceinline__ uint32_t pack2(float2 v) {
    __nv_bfloat162 b = __float22bfloat162_rn(v);
    return *reinterpret_cast<uint32_t *>(&b);
}
__device__ __forceinline__ void unpack8x2(const uint4 &u, float2 (&f)[4]) {
    const __nv_bfloat162 *b = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) f[i] = __bfloat1622float2(b[i]);
}
__device__ __forceinline__ uint4 pack8x2(const float2 (&f)[4]) {
    return make_uint4(pack2(f[0]), pack2(f[1]), pack2(f[2]), pack2(f[3]));
}
// 2^x on the special-function unit (the approximate exp2 instruction)
__device__ __forceinline__ float ex2a(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// log2(x) on the special-function unit (the approximate log2 instruction)
__device__ __forceinline__ float lg2a(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// In-kernel gate (page "atlas_core/kimi_k3/kda.rs", `bounded_gate`) for this bf16
// path, on the special-function unit: with x = x_in + bias,
//   kGateSoftplus: -rate (max(x, 0) + ln 2 * log2(1 + 2^(-|x| log2 e)))
//   kGateSafe:     lb / (1 + 2^(-rate x log2 e)), exponent capped at 64 so the
//                  denominator stays finite (the capped tail is below 1e-19 |lb|)
// The absolute error of g is a few 1e-7 * rate, far inside bf16 input rounding.
__device__ __forceinline__ float gate_fast(float x_in, float bias, float rate, int mode, float lb) {
    constexpr float kL2e = 1.4426950408889634f, kLn2 = 0.6931471805599453f;
    const float x = x_in + bias;
    if (mode == kGateSoftplus) {
        const float e = ex2a(-fabsf(x) * kL2e);
        return -rate * fmaf(lg2a(1.f + e), kLn2, fmaxf(x, 0.f));
    }
    return __fdividef(lb, 1.f + ex2a(fminf(-rate * x * kL2e, 64.f)));
}

// 1/x for normal positive x on the FMA pipe: a bit-pattern first estimate
// (reciprocal ~ 2^(2*127) / x read off the exponent/mantissa bits) refined by two
// Newton-Raphson steps y <- y (2 - x y); relative error ~1e-5.
__device__ __forceinline__ float2 rcp2_nr(float2 x) {
    float2 y = make_float2(__int_as_float(0x7EF311C3 - __float_as_int(x.x)),
                           __int_as_float(0x7EF311C3 - __float_as_int(x.y)));
    const float2 nx = make_float2(-x.x, -x.y), two = make_float2(2.f, 2.f);
    y = __fmul2_rn(y, __ffma2_rn(nx, y, two));
    y = __fmul2_rn(y, __ffma2_rn(nx, y, two));
    return y;
}

// 16 fp32 values of one TMEM row to two 16-byte chunks of a swizzled bf16 tile row
__device__ __forceinline__ void row16_to_tile(uint8_t *sm, uint32_t tile, int row, int col0, int rows,
                                              const float (&x)[16]) {
    sts128(sm, tile + sw128_chunk(row, col0, rows), pack8(x));
    sts128(sm, tile + sw128_chunk(row, col0 + 8, rows), pack8(x + 8));
}


inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// [T_total, H, 128] bf16 viewed as a 3-D tensor (channel, head, token); one
// box = 64 channels x 1 head x 64 tokens, 128-byte swizzled.
inline bool make_map(CUtensorMap *m, const void *base, long long ttot, int H) {
    auto fn = encode_fn();
    if (!fn) return false;
    constexpr cuuint64_t kD = 128;
    cuuint64_t dims[3] = {kD, (cuuint64_t)H, (cuuint64_t)ttot};
    cuuint64_t strides[2] = {kD * 2, (cuuint64_t)H * kD * 2};
    cuuint32_t box[3] = {64, 1, 64};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace tcu
}  // namespace kda
