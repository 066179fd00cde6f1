// Backward of the chunkwise forward: the derivatives of the token recurrence of
// page "atlas_core/kimi_k3/kda.rs" (the pages give no backward formulas).
//
// Per token t of one (sequence, head), with k^, q^ the normalised rows,
// a = exp(max(g, lb)), b the write strength and S the entering state:
//   S' = diag(a) S,  u = S'^T k^,  delta = b (v - u),  S_t = S' + k^ delta^T,
//   o = scale S_t^T q^.
// Walking the tokens backwards with dS the cotangent of S_t (starting from the
// final-state cotangent):
//   dS      += scale q^ do^T
//   dq^      = scale S_t do = scale (S' do + k^ (delta . do))
//   ddelta   = dS^T k^,            dv = b ddelta
//   dk^      = dS delta - b S' ddelta
//   db       = ddelta . (v - u)    (dbeta = db b (1 - b) for a logit)
//   dS'      = dS - b k^ ddelta^T
//   dg_c     = a_c sum_j dS'_cj S_cj = sum_j dS'_cj S'_cj   (zero where g_c < lb)
//   dS      <- diag(a) dS'          (the cotangent of the previous token's state)
//   dq       = r_q (dq^ - q^ (q^ . dq^)) for q^ = r_q q, likewise dk.
// The entering state of every token comes from a checkpoint written every kCB
// tokens by a recompute of the forward (`kda_bwd_ckpt_kernel`): per sub-chunk of
// kCB tokens the reverse sweep (`kda_bwd_kernel`) runs the forward once from the
// checkpoint, keeping each token's entering state in a per-head scratch (each
// thread stores and later reloads only its own tile), then walks the tokens back.
//
// One CTA of 256 threads per (sequence, head). Thread (kg, vg) keeps rows
// kg*RP .. kg*RP+RP-1, columns 4 vg .. 4 vg+3 of S and of dS as float4 in
// registers; sums over the key axis go through shared memory across row groups,
// sums over the value axis through shuffles among the VG lanes of a row group.
#include "kda_common.cuh"

namespace kda {

namespace {

constexpr int kBwdThreads = 256;
constexpr int kCB = 16;  // tokens per checkpoint

template <int DK, int DV>
struct BwdTile {
    static constexpr int NT = kBwdThreads, VG = DV / 4, KG = NT / VG, RP = DK / KG;
    static_assert(VG * KG == NT && RP * KG == DK && RP >= 1 && VG <= 32, "state tiling");
};

// Shared memory of both kernels: one sub-chunk of token vectors and the reduction
// scratch. Vectors are fp32; k^, q^ already normalised.
template <int DK, int DV>
struct BwdSmem {
    static constexpr int KG = BwdTile<DK, DV>::KG;
    float kh[kCB][DK], qh[kCB][DK], al[kCB][DK], graw[kCB][DK];
    float v[kCB][DV], dout[kCB][DV];
    float b[kCB], rq[kCB], rk[kCB];
    float red0[KG][DV + 1], red1[KG][DV + 1];
    float u[DV], delta[DV], ddelta[DV];
    float dqh[DK], dkh[DK];
    float wred[8];  // per-warp partials of delta . do and ddelta . (v - u)
    float scal[8];
};

__device__ __forceinline__ long long seq_begin(const BwdParams &p, int n) {
    return p.cu_seqlens ? (long long)p.cu_seqlens[n] : (long long)n * p.T;
}
__device__ __forceinline__ long long seq_end(const BwdParams &p, int n) {
    return p.cu_seqlens ? (long long)p.cu_seqlens[n + 1] : (long long)(n + 1) * p.T;
}
__device__ __forceinline__ long long first_ckpt(const BwdParams &p, int n) {
    return p.cu_seqlens ? (long long)p.ckpt_off[n] : (long long)n * ((p.T + kCB - 1) / kCB);
}

// Load tokens [t0, t0 + cnt) of head h into shared memory: k^, q^ (normalised when
// use_l2), the decay a = exp(max(g, lb)), the raw gate, v, the output cotangent and
// the write strength b. Ends with a block barrier.
template <typename Tin, int DK, int DV>
__device__ void load_tokens(const BwdParams &p, BwdSmem<DK, DV> &sm, long long t0, int cnt, int h, bool with_q) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int H = p.H;
    for (int e = tid; e < cnt * DK; e += kBwdThreads) {
        const int i = e / DK, c = e % DK;
        const long long gi = ((t0 + i) * H + h) * DK + c;
        sm.kh[i][c] = to_f32(static_cast<const Tin *>(p.k)[gi]);
        if (with_q) sm.qh[i][c] = to_f32(static_cast<const Tin *>(p.q)[gi]);
        const float gr = to_f32(static_cast<const Tin *>(p.g)[gi]);
        sm.graw[i][c] = gr;
        sm.al[i][c] = expf(p.has_lb ? fmaxf(gr, p.lb) : gr);
    }
    for (int e = tid; e < cnt * DV; e += kBwdThreads) {
        const int i = e / DV, c = e % DV;
        const long long gi = ((t0 + i) * H + h) * DV + c;
        sm.v[i][c] = to_f32(static_cast<const Tin *>(p.v)[gi]);
        if (with_q) sm.dout[i][c] = to_f32(static_cast<const Tin *>(p.dout)[gi]);
    }
    if (tid < cnt) sm.b[tid] = beta_value(to_f32(static_cast<const Tin *>(p.beta)[(t0 + tid) * H + h]), p.beta_prob);
    __syncthreads();
    // row norms: warp w takes tokens w, w + 8
    for (int i = warp; i < cnt; i += kBwdThreads / 32) {
        float kk = 0.f, qq = 0.f;
        for (int c = lane; c < DK; c += 32) {
            kk = fmaf(sm.kh[i][c], sm.kh[i][c], kk);
            if (with_q) qq = fmaf(sm.qh[i][c], sm.qh[i][c], qq);
        }
        kk = warp_sum(kk);
        qq = warp_sum(qq);
        const float rk = p.use_l2 ? rsqrtf(kk + kL2Eps) : 1.f, rq = p.use_l2 ? rsqrtf(qq + kL2Eps) : 1.f;
        for (int c = lane; c < DK; c += 32) {
            sm.kh[i][c] *= rk;
            if (with_q) sm.qh[i][c] *= rq;
        }
        if (lane == 0) { sm.rk[i] = rk; sm.rq[i] = rq; }
    }
    __syncthreads();
}

// One forward step of token i of the loaded sub-chunk on the register tile s.
template <int DK, int DV>
__device__ __forceinline__ void fwd_step(BwdSmem<DK, DV> &sm, int i, float4 (&s)[BwdTile<DK, DV>::RP]) {
    using Tl = BwdTile<DK, DV>;
    constexpr int RP = Tl::RP, KG = Tl::KG;
    const int tid = threadIdx.x, vg = tid % Tl::VG, kg = tid / Tl::VG;
    float4 pu = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int r = 0; r < RP; ++r) {
        const int c = kg * RP + r;
        const float a = sm.al[i][c], kc = sm.kh[i][c];
        s[r].x *= a; s[r].y *= a; s[r].z *= a; s[r].w *= a;
        pu.x = fmaf(s[r].x, kc, pu.x); pu.y = fmaf(s[r].y, kc, pu.y);
        pu.z = fmaf(s[r].z, kc, pu.z); pu.w = fmaf(s[r].w, kc, pu.w);
    }
    sm.red0[kg][4 * vg] = pu.x; sm.red0[kg][4 * vg + 1] = pu.y;
    sm.red0[kg][4 * vg + 2] = pu.z; sm.red0[kg][4 * vg + 3] = pu.w;
    __syncthreads();
    if (tid < DV) {
        float u = 0.f;
#pragma unroll 8
        for (int g = 0; g < KG; ++g) u += sm.red0[g][tid];
        sm.delta[tid] = sm.b[i] * (sm.v[i][tid] - u);
    }
    __syncthreads();
    const float d0 = sm.delta[4 * vg], d1 = sm.delta[4 * vg + 1], d2 = sm.delta[4 * vg + 2], d3 = sm.delta[4 * vg + 3];
#pragma unroll
    for (int r = 0; r < RP; ++r) {
        const float kc = sm.kh[i][kg * RP + r];
        s[r].x = fmaf(kc, d0, s[r].x); s[r].y = fmaf(kc, d1, s[r].y);
        s[r].z = fmaf(kc, d2, s[r].z); s[r].w = fmaf(kc, d3, s[r].w);
    }
    __syncthreads();  // delta and red0 are rewritten by the next step
}

template <int DK, int DV>
__device__ __forceinline__ float *tile_ptr(float *base, int row, int vg) {
    return base + (long long)row * DV + 4 * vg;
}

// Recompute of the forward, storing the entering state of tokens 0, kCB, 2 kCB, ...
template <typename Tin, int DK, int DV>
__global__ void __launch_bounds__(kBwdThreads, 1) kda_bwd_ckpt_kernel(BwdParams p) {
    using Tl = BwdTile<DK, DV>;
    constexpr int RP = Tl::RP;
    extern __shared__ __align__(16) uint8_t smraw[];
    BwdSmem<DK, DV> &sm = *reinterpret_cast<BwdSmem<DK, DV> *>(smraw);
    const int tid = threadIdx.x, vg = tid % Tl::VG, kg = tid / Tl::VG;
    const long long nh = blockIdx.x;
    const int n = (int)(nh / p.H), h = (int)(nh % p.H);
    const long long bos = seq_begin(p, n), eos = seq_end(p, n);
    float4 s[RP];
#pragma unroll
    for (int r = 0; r < RP; ++r)
        s[r] = p.S0 ? *reinterpret_cast<const float4 *>(tile_ptr<DK, DV>(const_cast<float *>(p.S0) + nh * DK * DV,
                                                                          kg * RP + r, vg))
                    : make_float4(0.f, 0.f, 0.f, 0.f);
    const long long c0 = first_ckpt(p, n);
    for (long long t0 = bos; t0 < eos; t0 += kCB) {
        const int cnt = (int)min((long long)kCB, eos - t0);
        float *ck = p.ckpt + ((c0 + (t0 - bos) / kCB) * p.H + h) * DK * DV;
#pragma unroll
        for (int r = 0; r < RP; ++r) *reinterpret_cast<float4 *>(tile_ptr<DK, DV>(ck, kg * RP + r, vg)) = s[r];
        load_tokens<Tin, DK, DV>(p, sm, t0, cnt, h, false);
        for (int i = 0; i < cnt; ++i) fwd_step<DK, DV>(sm, i, s);
    }
}

// Reverse sweep.
template <typename Tin, int DK, int DV>
__global__ void __launch_bounds__(kBwdThreads, 1) kda_bwd_kernel(BwdParams p) {
    using Tl = BwdTile<DK, DV>;
    constexpr int RP = Tl::RP, VG = Tl::VG, KG = Tl::KG;
    extern __shared__ __align__(16) uint8_t smraw[];
    BwdSmem<DK, DV> &sm = *reinterpret_cast<BwdSmem<DK, DV> *>(smraw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, vg = tid % VG, kg = tid / VG;
    const long long nh = blockIdx.x;
    const int n = (int)(nh / p.H), h = (int)(nh % p.H);
    const int H = p.H;
    const long long bos = seq_begin(p, n), eos = seq_end(p, n);
    const long long c0 = first_ckpt(p, n);
    float *scr = p.scratch + nh * (long long)kCB * DK * DV;  // this head's per-token states

    float4 ds[RP], s[RP];
#pragma unroll
    for (int r = 0; r < RP; ++r)
        ds[r] = p.dSf ? *reinterpret_cast<const float4 *>(tile_ptr<DK, DV>(const_cast<float *>(p.dSf) + nh * DK * DV,
                                                                           kg * RP + r, vg))
                      : make_float4(0.f, 0.f, 0.f, 0.f);
    const long long len = eos - bos;
    for (long long cs = (len + kCB - 1) / kCB - 1; cs >= 0; --cs) {
        const long long t0 = bos + cs * kCB;
        const int cnt = (int)min((long long)kCB, eos - t0);
        const float *ck = p.ckpt + ((c0 + cs) * H + h) * DK * DV;
        load_tokens<Tin, DK, DV>(p, sm, t0, cnt, h, true);
        // forward from the checkpoint, keeping every token's entering state
#pragma unroll
        for (int r = 0; r < RP; ++r)
            s[r] = *reinterpret_cast<const float4 *>(tile_ptr<DK, DV>(const_cast<float *>(ck), kg * RP + r, vg));
        for (int i = 0; i < cnt; ++i) {
#pragma unroll
            for (int r = 0; r < RP; ++r) *reinterpret_cast<float4 *>(tile_ptr<DK, DV>(scr + (long long)i * DK * DV, kg * RP + r, vg)) = s[r];
            if (i + 1 < cnt) fwd_step<DK, DV>(sm, i, s);
        }
        for (int i = cnt - 1; i >= 0; --i) {
            // the entering state of token i, stored by the forward pass over this sub-chunk
#pragma unroll
            for (int r = 0; r < RP; ++r) s[r] = *reinterpret_cast<const float4 *>(tile_ptr<DK, DV>(scr + (long long)i * DK * DV,
                                                                                                    kg * RP + r, vg));

            // ---- token i: S', u = S'^T k^, dS += scale q^ do^T, ddelta = dS^T k^
            const float b = sm.b[i];
            const float4 dov = *reinterpret_cast<const float4 *>(&sm.dout[i][4 * vg]);
            float4 pu = make_float4(0.f, 0.f, 0.f, 0.f), pd = pu;
#pragma unroll
            for (int r = 0; r < RP; ++r) {
                const int c = kg * RP + r;
                const float a = sm.al[i][c], kc = sm.kh[i][c], qs = p.scale * sm.qh[i][c];
                s[r].x *= a; s[r].y *= a; s[r].z *= a; s[r].w *= a;
                pu.x = fmaf(s[r].x, kc, pu.x); pu.y = fmaf(s[r].y, kc, pu.y);
                pu.z = fmaf(s[r].z, kc, pu.z); pu.w = fmaf(s[r].w, kc, pu.w);
                ds[r].x = fmaf(qs, dov.x, ds[r].x); ds[r].y = fmaf(qs, dov.y, ds[r].y);
                ds[r].z = fmaf(qs, dov.z, ds[r].z); ds[r].w = fmaf(qs, dov.w, ds[r].w);
                pd.x = fmaf(ds[r].x, kc, pd.x); pd.y = fmaf(ds[r].y, kc, pd.y);
                pd.z = fmaf(ds[r].z, kc, pd.z); pd.w = fmaf(ds[r].w, kc, pd.w);
            }
            sm.red0[kg][4 * vg] = pu.x; sm.red0[kg][4 * vg + 1] = pu.y;
            sm.red0[kg][4 * vg + 2] = pu.z; sm.red0[kg][4 * vg + 3] = pu.w;
            sm.red1[kg][4 * vg] = pd.x; sm.red1[kg][4 * vg + 1] = pd.y;
            sm.red1[kg][4 * vg + 2] = pd.z; sm.red1[kg][4 * vg + 3] = pd.w;
            __syncthreads();
            if (tid < DV) {
                float u = 0.f, dd = 0.f;
#pragma unroll 8
                for (int g = 0; g < KG; ++g) { u += sm.red0[g][tid]; dd += sm.red1[g][tid]; }
                const float vv = sm.v[i][tid];
                const float delta = b * (vv - u);
                sm.u[tid] = u;
                sm.delta[tid] = delta;
                sm.ddelta[tid] = dd;
                // dv, and the two value-axis dot products delta . do and ddelta . (v - u)
                static_cast<Tin *>(p.dv)[((t0 + i) * H + h) * DV + tid] = from_f32<Tin>(b * dd);
                float x0 = delta * sm.dout[i][tid], x1 = dd * (vv - u);
                x0 = warp_sum(x0);
                x1 = warp_sum(x1);
                if (lane == 0) { sm.wred[2 * warp] = x0; sm.wred[2 * warp + 1] = x1; }
            }
            __syncthreads();
            if (tid == 0) {
                float ddo = 0.f, db = 0.f;
                for (int w = 0; w < DV / 32; ++w) { ddo += sm.wred[2 * w]; db += sm.wred[2 * w + 1]; }
                sm.scal[0] = ddo;
                const float dbeta = p.beta_prob ? db : db * b * (1.f - b);
                static_cast<Tin *>(p.dbeta)[(t0 + i) * H + h] = from_f32<Tin>(dbeta);
            }
            // ---- row sums over the value axis: S' do, dS delta, S' ddelta, dS (.) S'
            const float4 dl = *reinterpret_cast<const float4 *>(&sm.delta[4 * vg]);
            const float4 ddl = *reinterpret_cast<const float4 *>(&sm.ddelta[4 * vg]);
            float ra[RP], rb[RP], re[RP], rh[RP];
#pragma unroll
            for (int r = 0; r < RP; ++r) {
                ra[r] = s[r].x * dov.x + s[r].y * dov.y + s[r].z * dov.z + s[r].w * dov.w;
                rb[r] = ds[r].x * dl.x + ds[r].y * dl.y + ds[r].z * dl.z + ds[r].w * dl.w;
                re[r] = s[r].x * ddl.x + s[r].y * ddl.y + s[r].z * ddl.z + s[r].w * ddl.w;
                rh[r] = ds[r].x * s[r].x + ds[r].y * s[r].y + ds[r].z * s[r].z + ds[r].w * s[r].w;
            }
#pragma unroll
            for (int o = 1; o < VG; o <<= 1) {
#pragma unroll
                for (int r = 0; r < RP; ++r) {
                    ra[r] += __shfl_xor_sync(0xffffffffu, ra[r], o);
                    rb[r] += __shfl_xor_sync(0xffffffffu, rb[r], o);
                    re[r] += __shfl_xor_sync(0xffffffffu, re[r], o);
                    rh[r] += __shfl_xor_sync(0xffffffffu, rh[r], o);
                }
            }
            __syncthreads();  // scal[0] is written
            const float ddo = sm.scal[0];
            if (vg == 0) {
#pragma unroll
                for (int r = 0; r < RP; ++r) {
                    const int c = kg * RP + r;
                    const float kc = sm.kh[i][c];
                    sm.dqh[c] = p.scale * (ra[r] + kc * ddo);
                    sm.dkh[c] = rb[r] - b * re[r];
                    const bool pass = !p.has_lb || sm.graw[i][c] >= p.lb;
                    const float dg = pass ? rh[r] - b * kc * re[r] : 0.f;
                    static_cast<Tin *>(p.dg)[((t0 + i) * H + h) * DK + c] = from_f32<Tin>(dg);
                }
            }
            // ---- dS <- diag(a) (dS - b k^ ddelta^T), the cotangent of the entering state
#pragma unroll
            for (int r = 0; r < RP; ++r) {
                const int c = kg * RP + r;
                const float a = sm.al[i][c], bk = b * sm.kh[i][c];
                ds[r].x = a * fmaf(-bk, ddl.x, ds[r].x); ds[r].y = a * fmaf(-bk, ddl.y, ds[r].y);
                ds[r].z = a * fmaf(-bk, ddl.z, ds[r].z); ds[r].w = a * fmaf(-bk, ddl.w, ds[r].w);
            }
            __syncthreads();
            // ---- through the L2 norm: dq = r (dq^ - q^ (q^ . dq^)), likewise k
            if (warp == 0) {
                float qd = 0.f, kd = 0.f;
                for (int c = lane; c < DK; c += 32) {
                    qd = fmaf(sm.qh[i][c], sm.dqh[c], qd);
                    kd = fmaf(sm.kh[i][c], sm.dkh[c], kd);
                }
                qd = warp_sum(qd);
                kd = warp_sum(kd);
                if (lane == 0) { sm.scal[1] = qd; sm.scal[2] = kd; }
            }
            __syncthreads();
            {
                const float qd = p.use_l2 ? sm.scal[1] : 0.f, kd = p.use_l2 ? sm.scal[2] : 0.f;
                const float rq = sm.rq[i], rk = sm.rk[i];
                for (int c = tid; c < DK; c += kBwdThreads) {
                    const long long gi = ((t0 + i) * H + h) * DK + c;
                    static_cast<Tin *>(p.dq)[gi] = from_f32<Tin>(rq * (sm.dqh[c] - sm.qh[i][c] * qd));
                    static_cast<Tin *>(p.dk)[gi] = from_f32<Tin>(rk * (sm.dkh[c] - sm.kh[i][c] * kd));
                }
            }
            __syncthreads();  // dqh / dkh / scal / red are rewritten by the next token
        }
    }
    if (p.dS0) {
#pragma unroll
        for (int r = 0; r < RP; ++r) *reinterpret_cast<float4 *>(tile_ptr<DK, DV>(p.dS0 + nh * DK * DV, kg * RP + r, vg)) = ds[r];
    }
}

// First checkpoint of every sequence: ckpt_off[n] = sum_{m<n} ceil(len_m / kCB). One block.
__global__ void kda_bwd_offsets(const int32_t *cu, int N, int *off) {
    if (threadIdx.x == 0) {
        int acc = 0;
        for (int n = 0; n < N; ++n) {
            off[n] = acc;
            acc += (int)(((long long)cu[n + 1] - cu[n] + kCB - 1) / kCB);
        }
        off[N] = acc;
    }
}

template <typename Tin, int DK, int DV>
cudaError_t launch_bwd_t(const BwdParams &p, cudaStream_t st) {
    const long long blocks = (long long)p.N * p.H;
    if (blocks == 0) return cudaSuccess;
    const int smem = (int)sizeof(BwdSmem<DK, DV>);
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(kda_bwd_ckpt_kernel<Tin, DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) != cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(kda_bwd_kernel<Tin, DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) != cudaSuccess)
        return e;
    if (p.cu_seqlens) {
        kda_bwd_offsets<<<1, 32, 0, st>>>(p.cu_seqlens, p.N, p.ckpt_off);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    kda_bwd_ckpt_kernel<Tin, DK, DV><<<(unsigned)blocks, kBwdThreads, smem, st>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    kda_bwd_kernel<Tin, DK, DV><<<(unsigned)blocks, kBwdThreads, smem, st>>>(p);
    return cudaGetLastError();
}

template <typename Tin>
cudaError_t launch_bwd_dt(const BwdParams &p, int Dk, int Dv, cudaStream_t st) {
#define KDA_BWD_CASE(DK_, DV_) \
    if (Dk == DK_ && Dv == DV_) return launch_bwd_t<Tin, DK_, DV_>(p, st);
    KDA_BWD_CASE(32, 32) KDA_BWD_CASE(32, 64) KDA_BWD_CASE(32, 128)
    KDA_BWD_CASE(64, 32) KDA_BWD_CASE(64, 64) KDA_BWD_CASE(64, 128)
    KDA_BWD_CASE(128, 32) KDA_BWD_CASE(128, 64) KDA_BWD_CASE(128, 128)
#undef KDA_BWD_CASE
    return cudaErrorInvalidValue;
}

}  // namespace

// Workspace: [ckpt_off: N+1 ints, 256-byte block][per-head scratch: kCB states][checkpoints]
size_t bwd_workspace_bytes(bool varlen, long long T, int N, int H, int Dk, int Dv) {
    const long long nck = varlen ? (T + kCB - 1) / kCB + N : (long long)N * ((T + kCB - 1) / kCB);
    const size_t head = (((size_t)(N + 1) * 4 + 255) / 256) * 256;
    return head + (size_t)N * H * kCB * Dk * Dv * 4 + (size_t)nck * H * Dk * Dv * 4;
}

cudaError_t launch_bwd(BwdParams p, bool bf16, int Dk, int Dv, void *workspace, cudaStream_t st) {
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    p.ckpt_off = reinterpret_cast<int *>(ws);
    p.scratch = reinterpret_cast<float *>(ws + (((size_t)(p.N + 1) * 4 + 255) / 256) * 256);
    p.ckpt = p.scratch + (size_t)p.N * p.H * kCB * Dk * Dv;
    return bf16 ? launch_bwd_dt<__nv_bfloat16>(p, Dk, Dv, st) : launch_bwd_dt<float>(p, Dk, Dv, st);
}

}  // namespace kda
