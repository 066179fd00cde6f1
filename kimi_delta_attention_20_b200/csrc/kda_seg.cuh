// Segments of long sequences, for the chunk forward when there are too few
// (sequence, head) state chains to fill the GPU. Every sequence is cut into P
// segments aligned to `align` tokens; the state after a segment is affine in the
// state before it, S_end = M S_start + N (each token's update is affine in S). The
// caller obtains every segment's transition M and offset N (runs of its forward over
// the segments), `kda_seg_chain` walks each sequence's segments to their true
// entering states, and the caller forms the outputs from those. Internal linkage:
// every file that includes this has its own copies.
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

// One CTA of 4 D / R threads per (sequence, head, 16-column slice): walk the P segments of
// the sequence, S_start(s) = S, S <- M_s S + N_s, from the caller's initial state (or
// zero); the last S is the final state. M_s and the slice of N_s are staged in shared
// memory by cp.async in a ring of NB buffers (all segments at once for d = 32), so the
// copies run ahead of the sequential products. Lane (rg, cg) = (lane / 4, lane % 4) of
// warp w holds rows 8 R w + rg + 8 j (j < R) and columns 4 cg .. 4 cg + 3: per
// key it reads R values of M (rows padded to D + 4 floats, so the 8 rows a warp reads
// at once fall on distinct banks) and one 16-byte piece of the state slice, and does
// 4 R multiply-adds. The register tile trades shared-memory wavefronts per
// multiply-add (a 16-byte load costs about four, broadcast or not) against warps to
// hide the load latency. Measured (B1 T8192 H16, 9 segments, d = 128): R = 2 with 8
// warps 38 us, R = 4 with 4 warps 41 us, R = 8 with 2 warps 48 us; at d = 32 (B4 T2048
// H8, 16 segments) R = 1 with 4 warps 12.5 us, R = 2 with 2 warps 17 us.
template <int D>
struct SegChainCfg {
    static constexpr int R = D >= 128 ? 2 : 1, NT = 4 * D / R, LD = D + 4;
    static constexpr int NB = D == 32 ? 16 : D == 64 ? 6 : 2;  // ring depth
};

template <int D>
struct SegChainSmem {
    float sc[2][D][16];                   // the state slice (current, next)
    float nb[SegChainCfg<D>::NB][D][16];  // slices of N_s
    float m[SegChainCfg<D>::NB][D][SegChainCfg<D>::LD];
};

// M_s and N_s are read at M + vs pitch and Nst + vs pitch (vs = (n P + s) H + h), rows
// ld floats apart; S_start is written as packed D x D states. rev walks the segments
// from the last to the first (the backward's cotangent, entering at each segment's end:
// S0 is then the final-state cotangent, S_start(s) the cotangent at the end of segment
// s, and S_out the cotangent of the initial state).
template <int D>
__global__ void __launch_bounds__(SegChainCfg<D>::NT) kda_seg_chain(const float *S0, const float *M, const float *Nst, int ld,
                                                    long long pitch, float *S_start, float *S_out, int N, int H, int P,
                                                    int rev) {
    using Cfg = SegChainCfg<D>;
    constexpr int NT = Cfg::NT, R = Cfg::R, NB = Cfg::NB, SL = D / 16;
    extern __shared__ __align__(16) uint8_t smraw[];
    SegChainSmem<D> &sm = *reinterpret_cast<SegChainSmem<D> *>(smraw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int slice = blockIdx.x % SL, nh = blockIdx.x / SL;
    const int n = nh / H, h = nh % H, j0 = 16 * slice;
    const int rb = warp * 8 * R + (lane >> 2), c = 4 * (lane & 3);  // rows rb + 8 j
    auto stage = [&](int sg) {  // start the copies of M_sg and N_sg's slice into buffer sg % NB
        if (sg < P) {
            const int b = sg % NB;
            const long long vs = ((long long)n * P + (rev ? P - 1 - sg : sg)) * H + h;
            const float *src = M + vs * pitch;
            for (int e = tid; e < D * (D / 4); e += NT)
                cp_async16(&sm.m[b][e / (D / 4)][(e % (D / 4)) * 4], src + (long long)(e / (D / 4)) * ld + (e % (D / 4)) * 4);
            const float *ns = Nst + vs * pitch + j0;
            for (int e = tid; e < D * 4; e += NT) cp_async16(&sm.nb[b][e / 4][(e % 4) * 4], ns + (long long)(e / 4) * ld + (e % 4) * 4);
        }
        cp_async_commit();  // empty past the last segment: one group per call keeps the count
    };
    for (int e = tid; e < D * 4; e += NT) {
        const int rr = e / 4, cc = (e % 4) * 4;
        *reinterpret_cast<float4 *>(&sm.sc[0][rr][cc]) =
            S0 ? *reinterpret_cast<const float4 *>(S0 + ((long long)nh * D + rr) * D + j0 + cc) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll 1
    for (int sg = 0; sg < NB - 1; ++sg) stage(sg);
    int cur = 0;
#pragma unroll 1
    for (int sg = 0; sg < P; ++sg) {
        const long long vs = ((long long)n * P + (rev ? P - 1 - sg : sg)) * H + h;  // virtual (segment, head) state index
        cp_async_wait_group<NB - 2>();
        __syncthreads();  // M_sg, N_sg and the current state are in place; buffer (sg - 1) % NB is free
        stage(sg + NB - 1);
        const int b = sg % NB;
        const float(*scc)[16] = sm.sc[cur];
        float(*scn)[16] = sm.sc[cur ^ 1];
        float2 acc[R][2];
#pragma unroll
        for (int j = 0; j < R; ++j) {
            const int r = rb + 8 * j;
            const float4 x = *reinterpret_cast<const float4 *>(&scc[r][c]);
            *reinterpret_cast<float4 *>(S_start + (vs * D + r) * D + j0 + c) = x;
            const float4 nv = *reinterpret_cast<const float4 *>(&sm.nb[b][r][c]);
            acc[j][0] = make_float2(nv.x, nv.y);
            acc[j][1] = make_float2(nv.z, nv.w);
        }
#pragma unroll 2
        for (int k = 0; k < D; k += 4) {
            float4 mv[R];
#pragma unroll
            for (int j = 0; j < R; ++j) mv[j] = *reinterpret_cast<const float4 *>(&sm.m[b][rb + 8 * j][k]);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const float4 sv = *reinterpret_cast<const float4 *>(&scc[k + kk][c]);
                const float2 s01 = make_float2(sv.x, sv.y), s23 = make_float2(sv.z, sv.w);
#pragma unroll
                for (int j = 0; j < R; ++j) {
                    const float mk = kk == 0 ? mv[j].x : kk == 1 ? mv[j].y : kk == 2 ? mv[j].z : mv[j].w;
                    const float2 m2 = make_float2(mk, mk);
                    acc[j][0] = __ffma2_rn(m2, s01, acc[j][0]);
                    acc[j][1] = __ffma2_rn(m2, s23, acc[j][1]);
                }
            }
        }
#pragma unroll
        for (int j = 0; j < R; ++j)
            *reinterpret_cast<float4 *>(&scn[rb + 8 * j][c]) = make_float4(acc[j][0].x, acc[j][0].y, acc[j][1].x, acc[j][1].y);
        cur ^= 1;
    }
    cp_async_wait_all();  // only empty groups can remain; nothing is left in flight at exit
    __syncthreads();
    if (S_out)
        for (int e = tid; e < D * 4; e += NT) {
            const int rr = e / 4, cc = (e % 4) * 4;
            *reinterpret_cast<float4 *>(S_out + ((long long)nh * D + rr) * D + j0 + cc) =
                *reinterpret_cast<const float4 *>(&sm.sc[cur][rr][cc]);
        }
}

// Launch the chain for N sequences x H heads of D x D states.
template <int D>
cudaError_t seg_chain_launch(const float *S0, const float *M, const float *Nst, int ld, long long pitch, float *S_start,
                             float *S_out, int N, int H, int P, cudaStream_t st, int rev = 0) {
    cudaError_t e = cudaFuncSetAttribute(kda_seg_chain<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)sizeof(SegChainSmem<D>));
    if (e != cudaSuccess) return e;
    count_launch();
    kda_seg_chain<D><<<(unsigned)((long long)N * H * (D / 16)), SegChainCfg<D>::NT, sizeof(SegChainSmem<D>), st>>>(
        S0, M, Nst, ld, pitch, S_start, S_out, N, H, P, rev);
    return cudaGetLastError();
}

}  // namespace
}  // namespace kda
