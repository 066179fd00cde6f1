// Segments of long sequences, for the chunk forward when there are too few
// (sequence, head) state chains to fill the GPU. Every sequence is cut into P
// segments aligned to `align` tokens; the state after a segment is affine in the
// state before it, S_end = M S_start + N (each token's update is affine in S), so
// the forward runs over the segments with v = 0 from the identity (the final
// states are the M), from zero (the N), and, once `kda_seg_chain` has walked each
// sequence's segments to their true entering states, from those states for the
// outputs. Internal linkage: every file that includes this has its own copies.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "kda_stage.cuh"

namespace kda {
namespace {

// cu_v[n P + s] = first token of segment s of sequence n (segment length: the
// sequence's length / P rounded up to whole `align` blocks; trailing segments may be
// empty); cu_v[N P] = the total.
__global__ void kda_seg_setup(const int32_t *cu, int T, int N, int P, int align, int32_t *cu_v) {
    for (int n = blockIdx.x * blockDim.x + threadIdx.x; n < N; n += gridDim.x * blockDim.x) {
        const long long bos = cu ? cu[n] : (long long)n * T, len = cu ? (long long)cu[n + 1] - cu[n] : T;
        const long long L = ((len + P - 1) / P + align - 1) / align * align;
        for (int sg = 0; sg < P; ++sg) cu_v[(long long)n * P + sg] = (int32_t)(bos + (sg * L < len ? sg * L : len));
        if (n == N - 1) cu_v[(long long)N * P] = (int32_t)(bos + len);
    }
}

// count identity states [D][D]
__global__ void kda_seg_identity(float *S, long long count, int D) {
    const long long total = count * D * D;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total; i += (long long)gridDim.x * blockDim.x) {
        const long long e = i % ((long long)D * D);
        S[i] = (e / D) == (e % D) ? 1.f : 0.f;
    }
}

// One CTA of 256 threads per (sequence, head, 16-column slice): walk the P segments
// of the sequence, S_start(s) = S, S <- M_s S + N_s, from the caller's initial state
// (or zero); the last S is the final state. M_s is staged in shared memory by
// cp.async while the previous segment is applied (rows padded to D + 4 floats:
// 16-byte aligned, and the rows a warp reads at one k spread over the banks).
// Thread t holds row t / TPR and CPT = 16 / TPR columns of the slice (TPR = 256 / D).
template <int D>
struct SegChainSmem {
    static constexpr int LD = D + 4;
    float4 sc[2][D][4];  // the state slice, rows of 16 columns
    float m[2][D][LD];
};

template <int D>
__global__ void __launch_bounds__(256) kda_seg_chain(const float *S0, const float *M, const float *Nst, float *S_start,
                                                     float *S_out, int N, int H, int P) {
    constexpr int TPR = 256 / D, CPT = 16 / TPR, LD = SegChainSmem<D>::LD, SL = D / 16;
    static_assert(TPR * D == 256 && CPT % 2 == 0, "chain tiling");
    extern __shared__ __align__(16) uint8_t smraw[];
    SegChainSmem<D> &sm = *reinterpret_cast<SegChainSmem<D> *>(smraw);
    const int tid = threadIdx.x;
    const int slice = blockIdx.x % SL, nh = blockIdx.x / SL;
    const int n = nh / H, h = nh % H, j0 = 16 * slice;
    const int r = tid / TPR, cb = (tid % TPR) * CPT;  // row r, slice columns cb .. cb + CPT - 1
    const long long DD = (long long)D * D;
    auto stage_m = [&](int sg, int b) {  // start the copy of M_sg into buffer b
        const float *src = M + (((long long)n * P + sg) * H + h) * DD;
        for (int e = tid; e < D * (D / 4); e += 256) cp_async16(&sm.m[b][e / (D / 4)][(e % (D / 4)) * 4], src + (long long)e * 4);
        cp_async_commit();
    };
    float *sc0 = reinterpret_cast<float *>(sm.sc[0]);
    for (int e = tid; e < D * 16; e += 256) {
        const int rr = e / 16, cc = e % 16;
        sc0[rr * 16 + cc] = S0 ? S0[((long long)nh * D + rr) * D + j0 + cc] : 0.f;
    }
    if (P > 0) stage_m(0, 0);
    int cur = 0;
    for (int sg = 0; sg < P; ++sg) {
        const long long vs = ((long long)n * P + sg) * H + h;  // virtual (segment, head) state index
        cp_async_wait_all();
        __syncthreads();  // M_sg and the current state are in shared memory; the other M buffer is free
        if (sg + 1 < P) stage_m(sg + 1, (sg + 1) & 1);
        const float (*m)[LD] = sm.m[sg & 1];
        const float *scc = reinterpret_cast<const float *>(sm.sc[cur]);
        float *scn = reinterpret_cast<float *>(sm.sc[cur ^ 1]);
        float2 acc[CPT / 2];
#pragma unroll
        for (int q = 0; q < CPT / 2; ++q) {
            const float2 x = make_float2(scc[r * 16 + cb + 2 * q], scc[r * 16 + cb + 2 * q + 1]);
            *reinterpret_cast<float2 *>(S_start + (vs * D + r) * D + j0 + cb + 2 * q) = x;
            acc[q] = *reinterpret_cast<const float2 *>(Nst + (vs * D + r) * D + j0 + cb + 2 * q);
        }
#pragma unroll 8
        for (int k = 0; k < D; ++k) {
            const float mv = m[r][k];
            const float2 m2 = make_float2(mv, mv);
#pragma unroll
            for (int q = 0; q < CPT / 2; ++q)
                acc[q] = __ffma2_rn(m2, *reinterpret_cast<const float2 *>(scc + k * 16 + cb + 2 * q), acc[q]);
        }
#pragma unroll
        for (int q = 0; q < CPT / 2; ++q) *reinterpret_cast<float2 *>(scn + r * 16 + cb + 2 * q) = acc[q];
        cur ^= 1;
    }
    __syncthreads();
    if (S_out) {
        const float *scc = reinterpret_cast<const float *>(sm.sc[cur]);
#pragma unroll
        for (int q = 0; q < CPT / 2; ++q)
            *reinterpret_cast<float2 *>(S_out + ((long long)nh * D + r) * D + j0 + cb + 2 * q) =
                make_float2(scc[r * 16 + cb + 2 * q], scc[r * 16 + cb + 2 * q + 1]);
    }
}

// Launch the chain for N sequences x H heads of D x D states.
template <int D>
cudaError_t seg_chain_launch(const float *S0, const float *M, const float *Nst, float *S_start, float *S_out, int N, int H,
                             int P, cudaStream_t st) {
    cudaError_t e = cudaFuncSetAttribute(kda_seg_chain<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)sizeof(SegChainSmem<D>));
    if (e != cudaSuccess) return e;
    kda_seg_chain<D><<<(unsigned)((long long)N * H * (D / 16)), 256, sizeof(SegChainSmem<D>), st>>>(S0, M, Nst, S_start,
                                                                                                    S_out, N, H, P);
    return cudaGetLastError();
}

}  // namespace
}  // namespace kda
