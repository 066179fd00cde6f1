// Fused serving decode token: causal depthwise conv + SiLU, the recurrent step and
// the full-rank output gate for one token of each of N sequences (page
// "atlas_core/kimi_k3/kda.rs": `conv_update`, `kda_decode_token`,
// `full_rank_output_gate`).
//
// One CTA of 256 threads per (sequence, head). Like the plain step it is a
// read-modify-write of the fp32 state (64 KiB per head at 128x128), so it is bound
// by HBM bandwidth; the conv windows of the head's 2 Dk + Dv channels (6 KiB at
// K = 4) and the token vectors add about 10 %. Thread (kg, vg) holds rows
// kg*RP .. kg*RP+RP-1 and columns 4 vg .. 4 vg + 3 of the state as float4 in
// registers between the read and the write, which goes back in place or to
// `state_out` when the caller keeps the old state. The per-head steps:
//   conv:   window <- (window[1:], x), y = silu(w . window) for q, k, v channels
//   step:   S' = diag(exp g) S, r_k = S'^T k, r_q = S'^T q (one pass),
//           delta = sigmoid(beta) (v - r_k / |k|), S = S' + (k/|k|) delta^T,
//           core = scale S^T q^ = scale (r_q / |q| + delta (k^.q^))
//   gate:   o = sigmoid(g_out) core / sqrt(mean(core^2) + eps)   (when g_out is given)
#include "kda_common.cuh"

namespace kda {

namespace {

constexpr int kTokThreads = 256;
constexpr int kMaxConv = 8;

template <typename Tin, int DK, int DV>
__global__ void __launch_bounds__(kTokThreads) kda_token_kernel(TokenParams tp, float *state_out) {
    constexpr int NT = kTokThreads, VG = DV / 4, KG = NT / VG, RP = DK / KG, NW = NT / 32;
    static_assert(VG * KG == NT && RP * KG == DK && RP >= 1, "state tiling");
    const StepParams &p = tp.step;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int vg = tid % VG, kg = tid / VG;
    const long long nh = blockIdx.x;  // n * H + h
    const int H = p.H, h = (int)(nh % H);
    const long long n = nh / H;

    const long long tile = nh * (long long)(DK * DV) + 4 * vg;
    const float *S = p.state + tile;
    float *So = (state_out ? state_out : p.state) + tile;
    // the token's gate, beta and output-gate values first (a few bytes each, but the
    // steps after the state read wait on them), raw until used
    const Tin *gop = static_cast<const Tin *>(tp.g_out);
    Tin g_raw = Tin(0.f), b_raw = Tin(0.f), go_raw = Tin(0.f);
    if (tid < DK) g_raw = static_cast<const Tin *>(p.g)[nh * DK + tid];
    if (tid < DV) {
        b_raw = static_cast<const Tin *>(p.beta)[nh];
        if (gop) go_raw = gop[nh * DV + tid];
    }
    static_assert(DK <= kTokThreads && DV <= kTokThreads, "one channel per thread");
    // then the state reads, whose latency hides the conv and vector work
    float4 s[RP];
#pragma unroll
    for (int i = 0; i < RP; ++i) s[i] = ld_stream(reinterpret_cast<const float4 *>(S + (long long)(kg * RP + i) * DV));

    __shared__ float sq[DK], sk[DK], sv[DV], sa[DK];
    __shared__ float rk_part[KG][DV + 1], rq_part[KG][DV + 1];
    __shared__ float sdelta[DV];
    __shared__ float sred[4];
    __shared__ float swarp[NW];

    // ---- causal depthwise conv + SiLU over this head's q, k, v channels
    const int K = tp.K;
    const long long C = (long long)H * (2 * DK + DV);
    const Tin *xp = static_cast<const Tin *>(tp.x) + n * C;
    float *cs_n = tp.conv_state + n * C * K;
    for (int j = tid; j < 2 * DK + DV; j += NT) {
        long long c;
        float *dst;
        if (j < DK) { c = (long long)h * DK + j; dst = sq + j; }
        else if (j < 2 * DK) { c = (long long)H * DK + (long long)h * DK + (j - DK); dst = sk + (j - DK); }
        else { c = 2LL * H * DK + (long long)h * DV + (j - 2 * DK); dst = sv + (j - 2 * DK); }
        float win[kMaxConv];
        float *cs = cs_n + c * K;
        const float *w = tp.conv_w + c * K;
#pragma unroll
        for (int t = 0; t < kMaxConv; ++t)
            if (t + 1 < K) win[t] = cs[t + 1];
        const float xv = to_f32(xp[c]);
        float acc = 0.f;
#pragma unroll
        for (int t = 0; t < kMaxConv; ++t) {
            if (t < K) {
                const float e = t + 1 < K ? win[t] : xv;
                cs[t] = e;
                acc = fmaf(w[t], e, acc);
            }
        }
        *dst = acc / (1.f + expf(-acc));  // SiLU
    }
    const float rate = p.gate_mode != kGateLog ? expf(p.A_log[h]) : 0.f;
    if (tid < DK) {
        const float bias = p.gate_mode != kGateLog && p.dt_bias ? p.dt_bias[h * DK + tid] : 0.f;
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

    // ---- decay and both column reductions over this thread's key rows
    float4 rk = make_float4(0.f, 0.f, 0.f, 0.f), rq = rk;
#pragma unroll
    for (int i = 0; i < RP; ++i) {
        const int c = kg * RP + i;
        const float a = sa[c], kc = sk[c], qc = sq[c];
        s[i].x *= a; s[i].y *= a; s[i].z *= a; s[i].w *= a;
        rk.x = fmaf(s[i].x, kc, rk.x); rk.y = fmaf(s[i].y, kc, rk.y);
        rk.z = fmaf(s[i].z, kc, rk.z); rk.w = fmaf(s[i].w, kc, rk.w);
        rq.x = fmaf(s[i].x, qc, rq.x); rq.y = fmaf(s[i].y, qc, rq.y);
        rq.z = fmaf(s[i].z, qc, rq.z); rq.w = fmaf(s[i].w, qc, rq.w);
    }
    rk_part[kg][4 * vg + 0] = rk.x; rk_part[kg][4 * vg + 1] = rk.y;
    rk_part[kg][4 * vg + 2] = rk.z; rk_part[kg][4 * vg + 3] = rk.w;
    rq_part[kg][4 * vg + 0] = rq.x; rq_part[kg][4 * vg + 1] = rq.y;
    rq_part[kg][4 * vg + 2] = rq.z; rq_part[kg][4 * vg + 3] = rq.w;
    __syncthreads();

    const float inv_q = p.use_l2 ? rsqrtf(sred[0] + kL2Eps) : 1.f;
    const float inv_k = p.use_l2 ? rsqrtf(sred[1] + kL2Eps) : 1.f;
    float core = 0.f;
    if (tid < DV) {
        float a = 0.f, b = 0.f;
#pragma unroll 8
        for (int g = 0; g < KG; ++g) { a += rk_part[g][tid]; b += rq_part[g][tid]; }
        const float bsig = beta_value(to_f32(b_raw), p.beta_prob);
        const float delta = bsig * (sv[tid] - inv_k * a);
        sdelta[tid] = delta;
        core = p.scale * (inv_q * b + delta * inv_k * inv_q * sred[2]);
    }
    // ---- output gate: RMS of the head's core output (threads tid < DV hold it)
    if (gop) {
        float ss = warp_sum(tid < DV ? core * core : 0.f);
        if (lane == 0) swarp[warp] = ss;
    }
    __syncthreads();
    if (tid < DV) {
        float out = core;
        if (gop) {
            float tot = 0.f;
#pragma unroll
            for (int w = 0; w < NW; ++w) tot += swarp[w];
            const float inv = rsqrtf(tot / DV + tp.norm_eps);
            const float gv = to_f32(go_raw);
            out = core * inv / (1.f + expf(-gv));
        }
        static_cast<Tin *>(p.o)[nh * DV + tid] = from_f32<Tin>(out);
    }

    // ---- state write-back: S = S' + (k / |k|) delta^T
    const float d0 = sdelta[4 * vg + 0], d1 = sdelta[4 * vg + 1];
    const float d2 = sdelta[4 * vg + 2], d3 = sdelta[4 * vg + 3];
#pragma unroll
    for (int i = 0; i < RP; ++i) {
        const int c = kg * RP + i;
        const float kc = inv_k * sk[c];
        float4 u;
        u.x = fmaf(kc, d0, s[i].x); u.y = fmaf(kc, d1, s[i].y);
        u.z = fmaf(kc, d2, s[i].z); u.w = fmaf(kc, d3, s[i].w);
        st_stream(reinterpret_cast<float4 *>(So + (long long)c * DV), u);
    }
}

template <typename Tin, int DK, int DV>
cudaError_t launch_token_t(const TokenParams &tp, float *state_out, cudaStream_t st) {
    const long long blocks = (long long)tp.step.N * tp.step.H;
    if (blocks == 0) return cudaSuccess;
    if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    count_launch();
    kda_token_kernel<Tin, DK, DV><<<(unsigned)blocks, kTokThreads, 0, st>>>(tp, state_out);
    return cudaGetLastError();
}

template <typename Tin>
cudaError_t launch_token_dt(const TokenParams &tp, float *state_out, int Dk, int Dv, cudaStream_t st) {
#define KDA_TOK_CASE(DK_, DV_) \
    if (Dk == DK_ && Dv == DV_) return launch_token_t<Tin, DK_, DV_>(tp, state_out, st);
    KDA_TOK_CASE(32, 32) KDA_TOK_CASE(32, 64) KDA_TOK_CASE(32, 128)
    KDA_TOK_CASE(64, 32) KDA_TOK_CASE(64, 64) KDA_TOK_CASE(64, 128)
    KDA_TOK_CASE(128, 32) KDA_TOK_CASE(128, 64) KDA_TOK_CASE(128, 128)
#undef KDA_TOK_CASE
    return cudaErrorInvalidValue;
}

}  // namespace

bool token_conv_supported(int K) { return K >= 1 && K <= kMaxConv; }

cudaError_t launch_token(const TokenParams &tp, float *state_out, bool bf16, int Dk, int Dv, cudaStream_t st) {
    return bf16 ? launch_token_dt<__nv_bfloat16>(tp, state_out, Dk, Dv, st)
                : launch_token_dt<float>(tp, state_out, Dk, Dv, st);
}

}  // namespace kda
