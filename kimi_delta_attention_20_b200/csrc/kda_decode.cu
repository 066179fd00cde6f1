// Recurrent decode step: one token for each of N sequences, state updated in
// place (page "atlas_core/kimi_k3/kda.rs", `kda_recurrent_step`).
//
// The step is a read-modify-write of the fp32 state [N,H,Dk,Dv] (64 KiB per
// head at 128x128) against ~1 KiB of per-token vectors, so it is bound by HBM
// bandwidth. Each CTA owns a 32-column slab of one head's state: 128 bytes of
// every key row, read and written back as float4 with streaming cache hints,
// kept in registers between the read and the write (one pass over HBM). The
// write goes back in place, or to `state_out` when the caller keeps the old state.
//
// g is the log-decay as given (clamped) or formed from the gate input in the
// kernel; beta a logit or a given probability. Per head, with S' = diag(exp g) S, the two column reductions over the key
// axis r_k = S'^T k and r_q = S'^T q are taken in the same pass; then
//   delta = sigmoid(beta) (v - r_k),
//   S     = S' + k delta^T,
//   o     = scale S^T q = scale (r_q + delta (k.q)),
// the last line being the output of the updated state rewritten with the
// values already at hand, so the state is not read twice.
#include "kda_common.cuh"

namespace kda {

template <typename Tin, int DK, int DV>
struct DecodeCfg {
    static constexpr int kCols = 32;            // state columns per CTA
    static constexpr int kSlabs = DV / kCols;
    static constexpr int kThreads = 256;
    static constexpr int kRowsPerPass = kThreads / 8;  // 8 threads x float4 per row
    static constexpr int kPasses = (DK + kRowsPerPass - 1) / kRowsPerPass;
    static constexpr int kWarps = kThreads / 32;
};

template <typename Tin, int DK, int DV>
__global__ void __launch_bounds__(256) kda_decode_kernel(StepParams p, float *state_out) {
    using Cfg = DecodeCfg<Tin, DK, DV>;
    constexpr int NP = Cfg::kPasses, RP = Cfg::kRowsPerPass, NW = Cfg::kWarps;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int slab = blockIdx.x % Cfg::kSlabs;
    const long long nh = blockIdx.x / Cfg::kSlabs;  // n * H + h
    const int cg = tid & 7;                          // float4 column group in the slab
    const int rg = tid >> 3;                         // first key row of this thread

    const long long tile = nh * (long long)(DK * DV) + slab * Cfg::kCols + cg * 4;
    const float *S = p.state + tile;
    float *So = (state_out ? state_out : p.state) + tile;
    const int h = nh % p.H;

    // The token's vectors first: they are few bytes, but every step after the state
    // read waits on them, and a new token's vectors come from HBM. Raw values now,
    // converted once the state reads are in flight.
    static_assert(DK <= Cfg::kThreads, "one key channel per thread");
    Tin q_raw = Tin(0.f), k_raw = Tin(0.f), g_raw = Tin(0.f), b_raw = Tin(0.f), v_raw = Tin(0.f);
    float bias = 0.f, rate = 0.f;
    if (tid < DK) {
        q_raw = static_cast<const Tin *>(p.q)[nh * DK + tid];
        k_raw = static_cast<const Tin *>(p.k)[nh * DK + tid];
        g_raw = static_cast<const Tin *>(p.g)[nh * DK + tid];
        if (p.gate_mode != kGateLog) {
            rate = expf(p.A_log[h]);
            if (p.dt_bias) bias = p.dt_bias[h * DK + tid];
        }
    }
    if (warp == 0) {
        b_raw = static_cast<const Tin *>(p.beta)[nh];
        v_raw = static_cast<const Tin *>(p.v)[nh * DV + slab * Cfg::kCols + lane];
    }

    // then the state reads, held in registers until the write-back
    float4 s[NP];
#pragma unroll
    for (int i = 0; i < NP; ++i) {
        const int c = rg + i * RP;
        if (c < DK) s[i] = ld_stream(reinterpret_cast<const float4 *>(S + (long long)c * DV));
        else s[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }

    __shared__ float sq[DK], sk[DK], sa[DK];
    __shared__ float sred[3];
    __shared__ float rk_part[NW][32], rq_part[NW][32];
    __shared__ float sdelta[32];

    if (tid < DK) {
        sq[tid] = to_f32(q_raw);
        sk[tid] = to_f32(k_raw);
        sa[tid] = expf(gate_value(to_f32(g_raw), bias, rate, p.gate_mode, p.has_lb, p.lb));
    }
    __syncthreads();
    if (warp == 0) {
        float qq = 0.f, kk = 0.f, qk = 0.f;
        for (int c = lane; c < DK; c += 32) {
            const float a = sq[c], b = sk[c];
            qq += a * a; kk += b * b; qk += a * b;
        }
        qq = warp_sum(qq); kk = warp_sum(kk); qk = warp_sum(qk);
        if (lane == 0) { sred[0] = qq; sred[1] = kk; sred[2] = qk; }
    }

    // Decay and both column reductions over this thread's key rows.
    float4 rk = make_float4(0.f, 0.f, 0.f, 0.f), rq = rk;
#pragma unroll
    for (int i = 0; i < NP; ++i) {
        const int c = rg + i * RP;
        if (c < DK) {
            const float a = sa[c], kc = sk[c], qc = sq[c];
            s[i].x *= a; s[i].y *= a; s[i].z *= a; s[i].w *= a;
            rk.x += s[i].x * kc; rk.y += s[i].y * kc; rk.z += s[i].z * kc; rk.w += s[i].w * kc;
            rq.x += s[i].x * qc; rq.y += s[i].y * qc; rq.z += s[i].z * qc; rq.w += s[i].w * qc;
        }
    }
    // Lanes sharing a column group differ in lane bits 3 and 4.
#pragma unroll
    for (int o = 8; o < 32; o <<= 1) {
        rk.x += __shfl_xor_sync(0xffffffffu, rk.x, o); rk.y += __shfl_xor_sync(0xffffffffu, rk.y, o);
        rk.z += __shfl_xor_sync(0xffffffffu, rk.z, o); rk.w += __shfl_xor_sync(0xffffffffu, rk.w, o);
        rq.x += __shfl_xor_sync(0xffffffffu, rq.x, o); rq.y += __shfl_xor_sync(0xffffffffu, rq.y, o);
        rq.z += __shfl_xor_sync(0xffffffffu, rq.z, o); rq.w += __shfl_xor_sync(0xffffffffu, rq.w, o);
    }
    if (lane < 8) {
        rk_part[warp][lane * 4 + 0] = rk.x; rk_part[warp][lane * 4 + 1] = rk.y;
        rk_part[warp][lane * 4 + 2] = rk.z; rk_part[warp][lane * 4 + 3] = rk.w;
        rq_part[warp][lane * 4 + 0] = rq.x; rq_part[warp][lane * 4 + 1] = rq.y;
        rq_part[warp][lane * 4 + 2] = rq.z; rq_part[warp][lane * 4 + 3] = rq.w;
    }
    __syncthreads();

    const float inv_q = p.use_l2 ? rsqrtf(sred[0] + kL2Eps) : 1.f;
    const float inv_k = p.use_l2 ? rsqrtf(sred[1] + kL2Eps) : 1.f;
    if (warp == 0) {
        float a = 0.f, b = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) { a += rk_part[w][lane]; b += rq_part[w][lane]; }
        const int col = slab * Cfg::kCols + lane;
        const float bsig = beta_value(to_f32(b_raw), p.beta_prob);
        const float vj = to_f32(v_raw);
        const float delta = bsig * (vj - inv_k * a);
        sdelta[lane] = delta;
        const float kq = inv_k * inv_q * sred[2];
        const float o = p.scale * (inv_q * b + delta * kq);
        static_cast<Tin *>(p.o)[nh * DV + col] = from_f32<Tin>(o);
    }
    __syncthreads();

    const float d0 = sdelta[cg * 4 + 0], d1 = sdelta[cg * 4 + 1];
    const float d2 = sdelta[cg * 4 + 2], d3 = sdelta[cg * 4 + 3];
#pragma unroll
    for (int i = 0; i < NP; ++i) {
        const int c = rg + i * RP;
        if (c < DK) {
            const float kc = inv_k * sk[c];
            float4 u;
            u.x = fmaf(kc, d0, s[i].x); u.y = fmaf(kc, d1, s[i].y);
            u.z = fmaf(kc, d2, s[i].z); u.w = fmaf(kc, d3, s[i].w);
            st_stream(reinterpret_cast<float4 *>(So + (long long)c * DV), u);
        }
    }
}

template <typename Tin, int DK, int DV>
cudaError_t launch_decode_t(const StepParams &p, float *state_out, cudaStream_t st) {
    using Cfg = DecodeCfg<Tin, DK, DV>;
    const long long blocks = (long long)p.N * p.H * Cfg::kSlabs;
    if (blocks == 0) return cudaSuccess;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    count_launch();
    kda_decode_kernel<Tin, DK, DV><<<(unsigned)blocks, Cfg::kThreads, 0, st>>>(p, state_out);
    return cudaGetLastError();
}

template <typename Tin>
cudaError_t launch_decode_dt(const StepParams &p, float *state_out, int Dk, int Dv, cudaStream_t st) {
#define KDA_DEC_CASE(DK_, DV_) \
    if (Dk == DK_ && Dv == DV_) return launch_decode_t<Tin, DK_, DV_>(p, state_out, st);
    KDA_DEC_CASE(32, 32) KDA_DEC_CASE(32, 64) KDA_DEC_CASE(32, 128)
    KDA_DEC_CASE(64, 32) KDA_DEC_CASE(64, 64) KDA_DEC_CASE(64, 128)
    KDA_DEC_CASE(128, 32) KDA_DEC_CASE(128, 64) KDA_DEC_CASE(128, 128)
#undef KDA_DEC_CASE
    return cudaErrorInvalidValue;
}

cudaError_t launch_decode(const StepParams &p, float *state_out, bool bf16, int Dk, int Dv, cudaStream_t st) {
    return bf16 ? launch_decode_dt<__nv_bfloat16>(p, state_out, Dk, Dv, st)
                : launch_decode_dt<float>(p, state_out, Dk, Dv, st);
}

}  // namespace kda
