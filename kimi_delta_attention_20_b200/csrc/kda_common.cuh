// Shared device helpers and launch-parameter structs of the KDA library.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kda {

constexpr float kL2Eps = 1e-6f;  // x / sqrt(sum x^2 + 1e-6), "atlas_core/kimi_k3/kda.rs" l2norm_rows

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

__device__ __forceinline__ float sigmoidf_(float x) { return 1.0f / (1.0f + expf(-x)); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Streaming 128-bit global accesses for data touched once per launch.
__device__ __forceinline__ float4 ld_stream(const float4 *p) { return __ldcs(p); }
__device__ __forceinline__ void st_stream(float4 *p, float4 v) { __stcs(p, v); }

// Launch parameters of the chunkwise forward (device pointers).
struct ChunkParams {
    const void *q, *k, *v, *g, *beta;
    void *o;
    const float *S0;
    float *S_out;
    const int32_t *cu_seqlens;  // may be null: sequence n = tokens [n*T, (n+1)*T)
    int T;                      // tokens per batch row when cu_seqlens is null
    int N, H;
    float scale;
    int use_l2;
    int has_lb;
    float lb;
};

// Launch parameters of the recurrent decode step.
struct StepParams {
    const void *q, *k, *v, *g, *beta;
    float *state;
    void *o;
    int N, H;
    float scale;
    int use_l2;
    int has_lb;
    float lb;
};

}  // namespace kda
