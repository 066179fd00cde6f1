// Staging helpers shared by the kernels that walk a sequence in stretches of
// tokens: 16-byte cp.async copies from global into shared memory, and the
// widening of staged bf16 / fp32 elements to fp32 with vector shared loads.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace kda {

__device__ __forceinline__ void cp_async16(void *sdst, const void *gsrc) {
    const unsigned d = (unsigned)__cvta_generic_to_shared(sdst);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }
// wait until at most N of this thread's committed groups are still in flight
template <int N>
__device__ __forceinline__ void cp_async_wait_group() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// E consecutive staged elements to fp32, with vector shared loads (bf16 widens exactly).
template <int E>
__device__ __forceinline__ void stage_cvt(const float *src, float (&out)[E]) {
    static_assert(E % 2 == 0, "pairs");
    if constexpr (E % 4 == 0) {
#pragma unroll
        for (int j = 0; j < E; j += 4) {
            const float4 x = *reinterpret_cast<const float4 *>(src + j);
            out[j] = x.x; out[j + 1] = x.y; out[j + 2] = x.z; out[j + 3] = x.w;
        }
    } else {
#pragma unroll
        for (int j = 0; j < E; j += 2) {
            const float2 x = *reinterpret_cast<const float2 *>(src + j);
            out[j] = x.x; out[j + 1] = x.y;
        }
    }
}
template <int E>
__device__ __forceinline__ void stage_cvt(const __nv_bfloat16 *src, float (&out)[E]) {
    static_assert(E % 2 == 0, "pairs");
    if constexpr (E % 8 == 0) {
#pragma unroll
        for (int j = 0; j < E; j += 8) {
            const uint4 x = *reinterpret_cast<const uint4 *>(src + j);
            const unsigned w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                out[j + 2 * e] = __uint_as_float(w[e] << 16);
                out[j + 2 * e + 1] = __uint_as_float(w[e] & 0xffff0000u);
            }
        }
    } else {
#pragma unroll
        for (int j = 0; j < E; j += 2) {
            const unsigned w = *reinterpret_cast<const unsigned *>(src + j);
            out[j] = __uint_as_float(w << 16);
            out[j + 1] = __uint_as_float(w & 0xffff0000u);
        }
    }
}
template <int E>
__device__ __forceinline__ void store_vec(float *dst, const float (&x)[E]) {
    if constexpr (E % 4 == 0) {
#pragma unroll
        for (int j = 0; j < E; j += 4) *reinterpret_cast<float4 *>(dst + j) = make_float4(x[j], x[j + 1], x[j + 2], x[j + 3]);
    } else {
#pragma unroll
        for (int j = 0; j < E; j += 2) *reinterpret_cast<float2 *>(dst + j) = make_float2(x[j], x[j + 1]);
    }
}

}  // namespace kda
