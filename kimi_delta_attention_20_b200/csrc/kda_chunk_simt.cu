// Chunkwise KDA forward in fp32 on CUDA cores.
//
// This is the fp32 path (fp32 inputs need ~1e-4 relative accuracy, which
// tensor-core tf32 cannot give) and the reference shape of the chunk
// algorithm the tensor-core path follows. One CTA owns one (sequence, head,
// 64-column slab of d_v) and walks the sequence one chunk of C = 64 tokens
// at a time, with the state slab S (d_k x 64, fp32) resident in shared
// memory across chunks (C = 64, or 32 when the caller asks for 32-token
// chunks). Per chunk, with G the inclusive in-chunk cumsum of
// the gate (clamped, or formed in the kernel from A_log and dt_bias) and
// beta = sigmoid(logit) (or a given probability):
//
//   A_kk[r,s] = sum_c k_r k_s exp(G_r - G_s)       (s < r)
//   A_qk[r,s] = sum_c q_r k_s exp(G_r - G_s)       (s <= r)
//   Delta: (I + diag(beta) A_kk) Delta = diag(beta) (V - (k . e^G) S),
//          solved by forward substitution row by row
//   O     = scale ((q . e^G) S + A_qk Delta)
//   S    <- diag(e^{G_last}) S + (k . e^{G_last - G})^T Delta
//
// which is the token recurrence of page "atlas_core/kimi_k3/kda.rs" regrouped
// by chunk (the boundary is `chunk_kda` of page "K3/kda/ops/api.py"). Every
// exponent is a difference G_r - G_s with r >= s, or G_last - G_s, so no
// factor exceeds 1 and none can overflow. A partial last chunk is padded with
// zero q, k, v, g and beta = 0, which leaves the state and the real rows
// untouched.
#include "kda_common.cuh"

namespace kda {

template <int DK, int DV, int CC>
struct SimtCfg {
    static constexpr int C = CC;                  // tokens per chunk: 32 or 64
    static constexpr int VS = DV < 64 ? DV : 64;  // state columns per CTA
    static constexpr int kSlabs = DV / VS;
    static constexpr int kThreads = 256;
    static constexpr int kWarps = kThreads / 32;
    // shared memory, in floats
    static constexpr int oQ = 0, oK = oQ + C * DK, oG = oK + C * DK, oV = oG + C * DK;
    static constexpr int oS = oV + C * VS, oAkk = oS + DK * VS, oAqk = oAkk + C * C;
    static constexpr int oB = oAqk + C * C, oGL = oB + C, kFloats = oGL + DK;
    static constexpr size_t kSmemBytes = sizeof(float) * kFloats;
};

template <typename Tin, int DK, int DV, int CC>
__global__ void __launch_bounds__(256, 1) kda_chunk_simt_kernel(ChunkParams p) {
    using Cfg = SimtCfg<DK, DV, CC>;
    constexpr int C = Cfg::C, VS = Cfg::VS, NT = Cfg::kThreads, NW = Cfg::kWarps;
    extern __shared__ float smem[];
    float *qs = smem + Cfg::oQ, *ks = smem + Cfg::oK, *Gs = smem + Cfg::oG;
    float *vs = smem + Cfg::oV, *Ss = smem + Cfg::oS;
    float *Akk = smem + Cfg::oAkk, *Aqk = smem + Cfg::oAqk;
    float *sb = smem + Cfg::oB, *GL = smem + Cfg::oGL;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int slab = blockIdx.x % Cfg::kSlabs;
    const int nh = blockIdx.x / Cfg::kSlabs;
    const int h = nh % p.H, n = nh / p.H;
    long long bos, eos;
    if (p.cu_seqlens) { bos = p.cu_seqlens[n]; eos = p.cu_seqlens[n + 1]; }
    else { bos = (long long)n * p.T; eos = bos + p.T; }
    const int H = p.H;
    const int col0 = slab * VS;

    // state slab in
    const long long sbase = (long long)nh * DK * DV + col0;
    for (int i = tid; i < DK * VS; i += NT) {
        const int c = i / VS, j = i % VS;
        Ss[i] = p.S0 ? p.S0[sbase + (long long)c * DV + j] : 0.f;
    }

    const Tin *Q = static_cast<const Tin *>(p.q), *K = static_cast<const Tin *>(p.k);
    const Tin *Vv = static_cast<const Tin *>(p.v), *Gg = static_cast<const Tin *>(p.g);
    const Tin *Bt = static_cast<const Tin *>(p.beta);
    Tin *O = static_cast<Tin *>(p.o);

    const float rate = p.gate_mode != kGateLog ? expf(p.A_log[h]) : 0.f;
    const float *dtb = p.gate_mode != kGateLog && p.dt_bias ? p.dt_bias + (long long)h * DK : nullptr;

    for (long long t0 = bos; t0 < eos; t0 += C) {
        const int L = (int)((eos - t0) < C ? (eos - t0) : C);
        __syncthreads();  // previous chunk done with every buffer
        // 1. load the chunk; rows >= L are zero padding with beta = 0
        for (int i = tid; i < C * DK; i += NT) {
            const int r = i / DK, c = i % DK;
            float qv = 0.f, kv = 0.f, gv = 0.f;
            if (r < L) {
                const long long off = ((t0 + r) * H + h) * DK + c;
                qv = to_f32(Q[off]); kv = to_f32(K[off]);
                gv = gate_value(to_f32(Gg[off]), dtb ? dtb[c] : 0.f, rate, p.gate_mode, p.has_lb, p.lb);
            }
            qs[i] = qv; ks[i] = kv; Gs[i] = gv;
        }
        for (int i = tid; i < C * VS; i += NT) {
            const int r = i / VS, j = i % VS;
            vs[i] = r < L ? to_f32(Vv[((t0 + r) * H + h) * DV + col0 + j]) : 0.f;
        }
        for (int r = tid; r < C; r += NT)
            sb[r] = r < L ? beta_value(to_f32(Bt[(t0 + r) * H + h]), p.beta_prob) : 0.f;
        __syncthreads();

        // 2. row L2 norms of q and k (warp per row), cumsum of g (thread per channel)
        if (p.use_l2) {
            for (int r = warp; r < C; r += NW) {
                float sq = 0.f, sk = 0.f;
                for (int c = lane; c < DK; c += 32) {
                    sq += qs[r * DK + c] * qs[r * DK + c];
                    sk += ks[r * DK + c] * ks[r * DK + c];
                }
                sq = warp_sum(sq); sk = warp_sum(sk);
                const float iq = rsqrtf(sq + kL2Eps), ik = rsqrtf(sk + kL2Eps);
                for (int c = lane; c < DK; c += 32) { qs[r * DK + c] *= iq; ks[r * DK + c] *= ik; }
            }
        }
        for (int c = tid; c < DK; c += NT) {
            float acc = 0.f;
            for (int r = 0; r < C; ++r) { acc += Gs[r * DK + c]; Gs[r * DK + c] = acc; }
        }
        __syncthreads();

        // 3. gated A_kk and A_qk, lower triangle, one warp per row
        for (int c = tid; c < DK; c += NT) GL[c] = Gs[(C - 1) * DK + c];
        for (int r = warp; r < C; r += NW) {
            constexpr int PL = DK / 32;
            float kr[PL], qr[PL], gr[PL];
#pragma unroll
            for (int u = 0; u < PL; ++u) {
                const int c = lane + 32 * u;
                kr[u] = ks[r * DK + c]; qr[u] = qs[r * DK + c]; gr[u] = Gs[r * DK + c];
            }
            for (int s = 0; s <= r; ++s) {
                float akk = 0.f, aqk = 0.f;
#pragma unroll
                for (int u = 0; u < PL; ++u) {
                    const int c = lane + 32 * u;
                    const float e = expf(gr[u] - Gs[s * DK + c]) * ks[s * DK + c];
                    akk = fmaf(kr[u], e, akk);
                    aqk = fmaf(qr[u], e, aqk);
                }
                akk = warp_sum(akk); aqk = warp_sum(aqk);
                if (lane == 0) { Akk[r * C + s] = (s < r) ? akk : 0.f; Aqk[r * C + s] = aqk; }
            }
        }
        __syncthreads();

        // 4. gated operands: q <- q.e^G, k <- k.e^G, G <- k.e^{G_last - G}
        for (int i = tid; i < C * DK; i += NT) {
            const int c = i % DK;
            const float gg = Gs[i], kk = ks[i];
            qs[i] *= expf(gg);
            ks[i] = kk * expf(gg);
            Gs[i] = kk * expf(GL[c] - gg);
        }
        __syncthreads();

        // 5. V <- V - (k.e^G) S
        for (int i = tid; i < C * VS; i += NT) {
            const int r = i / VS, j = i % VS;
            float acc = 0.f;
#pragma unroll 8
            for (int c = 0; c < DK; ++c) acc = fmaf(ks[r * DK + c], Ss[c * VS + j], acc);
            vs[i] -= acc;
        }
        __syncthreads();

        // 6. forward substitution, in place: Delta_r = beta_r (V_r - sum_{s<r} A_kk[r,s] Delta_s);
        //    each warp owns VS/NW columns, the sum over s is split across lanes
        {
            constexpr int CPW = VS / NW;       // columns per warp
            constexpr int NPART = 32 / CPW;    // lanes sharing a column
            const int j = warp * CPW + (lane % CPW);
            const int part = lane / CPW;
            for (int r = 0; r < C; ++r) {
                float acc = 0.f;
                for (int s = part; s < r; s += NPART) acc = fmaf(Akk[r * C + s], vs[s * VS + j], acc);
#pragma unroll
                for (int o = CPW; o < 32; o <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
                const float d = sb[r] * (vs[r * VS + j] - acc);
                __syncwarp();
                if (part == 0) vs[r * VS + j] = d;
                __syncwarp();
            }
        }
        __syncthreads();

        // 7. O = scale ((q.e^G) S + A_qk Delta)
        for (int i = tid; i < C * VS; i += NT) {
            const int r = i / VS, j = i % VS;
            float acc = 0.f;
#pragma unroll 8
            for (int c = 0; c < DK; ++c) acc = fmaf(qs[r * DK + c], Ss[c * VS + j], acc);
            for (int s = 0; s <= r; ++s) acc = fmaf(Aqk[r * C + s], vs[s * VS + j], acc);
            if (r < L) O[((t0 + r) * H + h) * DV + col0 + j] = from_f32<Tin>(p.scale * acc);
        }
        __syncthreads();

        // 8. S <- diag(e^{G_last}) S + (k.e^{G_last - G})^T Delta
        for (int i = tid; i < DK * VS; i += NT) {
            const int c = i / VS, j = i % VS;
            float acc = expf(GL[c]) * Ss[i];
#pragma unroll 8
            for (int s = 0; s < C; ++s) acc = fmaf(Gs[s * DK + c], vs[s * VS + j], acc);
            Ss[i] = acc;
        }
    }
    __syncthreads();
    if (p.S_out) {
        for (int i = tid; i < DK * VS; i += NT) {
            const int c = i / VS, j = i % VS;
            p.S_out[sbase + (long long)c * DV + j] = Ss[i];
        }
    }
}

template <typename Tin, int DK, int DV, int CC>
cudaError_t launch_simt_t(const ChunkParams &p, cudaStream_t st) {
    using Cfg = SimtCfg<DK, DV, CC>;
    const long long blocks = (long long)p.N * p.H * Cfg::kSlabs;
    if (blocks == 0) return cudaSuccess;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    auto kern = kda_chunk_simt_kernel<Tin, DK, DV, CC>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)Cfg::kSmemBytes);
    if (e != cudaSuccess) return e;
    count_launch();
    kern<<<(unsigned)blocks, Cfg::kThreads, Cfg::kSmemBytes, st>>>(p);
    return cudaGetLastError();
}

template <typename Tin, int CC>
cudaError_t launch_simt_dt(const ChunkParams &p, int Dk, int Dv, cudaStream_t st) {
#define KDA_SIMT_CASE(DK_, DV_) \
    if (Dk == DK_ && Dv == DV_) return launch_simt_t<Tin, DK_, DV_, CC>(p, st);
    KDA_SIMT_CASE(32, 32) KDA_SIMT_CASE(32, 64) KDA_SIMT_CASE(32, 128)
    KDA_SIMT_CASE(64, 32) KDA_SIMT_CASE(64, 64) KDA_SIMT_CASE(64, 128)
    KDA_SIMT_CASE(128, 32) KDA_SIMT_CASE(128, 64) KDA_SIMT_CASE(128, 128)
#undef KDA_SIMT_CASE
    return cudaErrorInvalidValue;
}

cudaError_t launch_chunk_simt(const ChunkParams &p, bool bf16, int Dk, int Dv, int chunk, cudaStream_t st) {
    if (chunk == 32)
        return bf16 ? launch_simt_dt<__nv_bfloat16, 32>(p, Dk, Dv, st) : launch_simt_dt<float, 32>(p, Dk, Dv, st);
    return bf16 ? launch_simt_dt<__nv_bfloat16, 64>(p, Dk, Dv, st) : launch_simt_dt<float, 64>(p, Dk, Dv, st);
}

}  // namespace kda
