// Shared device helpers and launch-parameter structs of the KDA library.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace kda {

// Counts one kernel launch queued by the library (kda_launch_count of the C ABI).
void count_launch();

constexpr float kL2Eps = 1e-6f;  // x / sqrt(sum x^2 + 1e-6), "atlas_core/kimi_k3/kda.rs" l2norm_rows

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

__device__ __forceinline__ float sigmoidf_(float x) { return 1.0f / (1.0f + expf(-x)); }

// How g is obtained from the g input (kda_gate_mode of the C ABI).
enum : int { kGateLog = 0, kGateSoftplus = 1, kGateSafe = 2 };

// The per-channel log-decay from the g input x_in (page "atlas_core/kimi_k3/kda.rs",
// `bounded_gate`): rate = exp(A_log[h]) and bias = dt_bias[h, c].
//   kGateLog:      x_in, clamped below by lb when has_lb
//   kGateSoftplus: -rate * log(1 + e^x), x = x_in + bias (overflow-free split)
//   kGateSafe:     lb * sigmoid(rate * x)
__device__ __forceinline__ float gate_value(float x_in, float bias, float rate, int mode, int has_lb,
                                            float lb) {
    if (mode == kGateSoftplus) {
        const float x = x_in + bias;
        return -rate * (fmaxf(x, 0.f) + log1pf(expf(-fabsf(x))));
    }
    if (mode == kGateSafe) return lb / (1.f + expf(-rate * (x_in + bias)));
    return has_lb ? fmaxf(x_in, lb) : x_in;
}

// beta as the recurrence uses it: sigmoid of a logit, or the probability as given.
__device__ __forceinline__ float beta_value(float b, int is_prob) { return is_prob ? b : sigmoidf_(b); }

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
    int gate_mode;              // kGate*
    const float *A_log;         // [H], in-kernel gate forms
    const float *dt_bias;       // [H, Dk] or null
    int beta_prob;              // 1: beta is a probability
    int stall_first_wait;       // test of the bounded waits: the first input copy is not issued
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
    int gate_mode;
    const float *A_log;
    const float *dt_bias;
    int beta_prob;
};

// Launch parameters of the fused decode token (conv + SiLU, recurrent step, output gate).
struct TokenParams {
    StepParams step;            // q, k, v unused: they come from the convolution
    const void *x;              // [N, H*(2Dk+Dv)]
    const float *conv_w;        // [H*(2Dk+Dv), K]
    float *conv_state;          // [N, H*(2Dk+Dv), K]
    int K;
    const void *g_out;          // [N, H, Dv] or null
    float norm_eps;
};

}  // namespace kda
