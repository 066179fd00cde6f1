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
//
// Column split. The value columns of S and of dS evolve independently (u, delta,
// ddelta and the decay act column by column), so each (sequence, head) runs as a
// cluster of Dv/16 CTAs, one per 16-column slice. What sums over the value axis
// (dq^, dk^, dg, db) is linear in the per-slice terms: every CTA keeps its slice's
// terms for the kCB tokens of a stretch in shared memory, and after the stretch
// the cluster adds them across its CTAs through distributed shared memory (a
// fixed rank order, so the result is deterministic) and applies the L2-norm and
// sigmoid chain rules once per token.
//
// The entering state of every token comes from a checkpoint written every kCB
// tokens by a recompute of the forward (`kda_bwd_ckpt_kernel`): per stretch of kCB
// tokens the reverse sweep (`kda_bwd_kernel`) runs the forward once from the
// checkpoint, keeping each token's entering state in a per-CTA scratch (each
// thread stores and later reloads only its own tile), then walks the tokens back.
//
// 128 threads per CTA. Thread (kg, vg) = (tid / 4, tid % 4) keeps rows
// kg*RP .. kg*RP+RP-1 and slice columns 4 vg .. 4 vg+3 of S and of dS as float4
// in registers. Key-axis sums go through shuffles among the 8 row groups of a
// warp, then shared memory across the 4 warps (one block barrier per token, the
// buffers alternating between tokens); value-axis sums within the slice go
// through shuffles among the 4 lanes of a row group.
#include <cooperative_groups.h>

#include "kda_common.cuh"

namespace kda {

namespace {

namespace cg = cooperative_groups;

constexpr int kBwdThreads = 128;
constexpr int kWarps = kBwdThreads / 32;
constexpr int kCB = 16;   // tokens per checkpoint (one stretch)
constexpr int kDVC = 16;  // value columns per CTA

template <int DK, int DV>
struct BwdTile {
    static constexpr int VG = kDVC / 4, KG = kBwdThreads / VG, RP = DK / KG, NS = DV / kDVC;
    static_assert(VG == 4 && KG == 32 && RP * KG == DK && RP >= 1 && NS >= 1 && NS <= 8, "state tiling");
};

// Raw inputs of one stretch, copied in by cp.async while the previous stretch runs.
template <typename Tin, int DK>
struct Stage {
    Tin k[kCB][DK], g[kCB][DK], q[kCB][DK];  // q: reverse sweep only
    Tin v[kCB][kDVC], dout[kCB][kDVC];       // this CTA's value columns; dout: reverse sweep only
};

// Token vectors of one stretch (fp32; k^ normalised) and the key-axis reduction
// buffers: what the forward recompute needs.
template <typename Tin, int DK>
struct FwdSmem {
    Stage<Tin, DK> st;
    float kh[kCB][DK], al[kCB][DK];
    float v[kCB][kDVC];
    float b[kCB], rk[kCB];
    float4 red[2][kWarps][2][4];  // [token parity][warp][u or ddelta][column group]
};

// The reverse sweep adds q^, the raw gate (for the clamp mask), the output
// cotangent, and the per-slice terms of dq^, dk^, dg and db, double-buffered
// across stretches so that one cluster barrier per stretch suffices.
template <typename Tin, int DK>
struct BwdSmem : FwdSmem<Tin, DK> {
    float qh[kCB][DK], graw[kCB][DK];
    float dout[kCB][kDVC];
    float rq[kCB];
    float pdq[2][kCB][DK], pdk[2][kCB][DK], pdg[2][kCB][DK];
    float pdb[2][kCB];
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

template <int RP>
__device__ __forceinline__ void load_rows(const float *src, float (&out)[RP]) {
    if constexpr (RP == 4) {
        const float4 x = *reinterpret_cast<const float4 *>(src);
        out[0] = x.x; out[1] = x.y; out[2] = x.z; out[3] = x.w;
    } else if constexpr (RP == 2) {
        const float2 x = *reinterpret_cast<const float2 *>(src);
        out[0] = x.x; out[1] = x.y;
    } else {
        out[0] = src[0];
    }
}

__device__ __forceinline__ float4 f4_add(float4 a, float4 b) { return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w); }
__device__ __forceinline__ float dot4(float4 a, float4 b) { return a.x * b.x + a.y * b.y + a.z * b.z + a.w * b.w; }

// Sum over the 8 row groups of a warp (lane bits 2..4).
__device__ __forceinline__ float4 rowgroup_sum(float4 x) {
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
        x.x += __shfl_xor_sync(0xffffffffu, x.x, o);
        x.y += __shfl_xor_sync(0xffffffffu, x.y, o);
        x.z += __shfl_xor_sync(0xffffffffu, x.z, o);
        x.w += __shfl_xor_sync(0xffffffffu, x.w, o);
    }
    return x;
}
// Sum over the 4 column groups of a row group (lane bits 0..1).
__device__ __forceinline__ float colgroup_sum(float x) {
    x += __shfl_xor_sync(0xffffffffu, x, 1);
    x += __shfl_xor_sync(0xffffffffu, x, 2);
    return x;
}

__device__ __forceinline__ void cp_async16(void *sdst, const void *gsrc) {
    const unsigned d = (unsigned)__cvta_generic_to_shared(sdst);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// Start the copy of tokens [t0, t0 + cnt) of head h into the stage: k, g (and q
// for the reverse sweep) rows, and this CTA's columns of v (and of the output
// cotangent), in 16-byte pieces. Returns this thread's raw beta (thread i < cnt
// holds token i's); the load completes in the background like the copies.
template <typename Tin, int DK, int DV, bool kRev>
__device__ __forceinline__ float issue_stretch(const BwdParams &p, Stage<Tin, DK> &st, long long t0, int cnt, int h,
                                               int col0) {
    constexpr int EP = 16 / (int)sizeof(Tin);  // elements per piece
    constexpr int RK = DK / EP, RV = kDVC / EP;
    const int tid = threadIdx.x, H = p.H;
    for (int e = tid; e < cnt * RK; e += kBwdThreads) {
        const int i = e / RK, c = (e % RK) * EP;
        const long long gi = ((t0 + i) * H + h) * DK + c;
        cp_async16(&st.k[i][c], static_cast<const Tin *>(p.k) + gi);
        cp_async16(&st.g[i][c], static_cast<const Tin *>(p.g) + gi);
        if constexpr (kRev) cp_async16(&st.q[i][c], static_cast<const Tin *>(p.q) + gi);
    }
    for (int e = tid; e < cnt * RV; e += kBwdThreads) {
        const int i = e / RV, c = (e % RV) * EP;
        const long long gi = ((t0 + i) * H + h) * DV + col0 + c;
        cp_async16(&st.v[i][c], static_cast<const Tin *>(p.v) + gi);
        if constexpr (kRev) cp_async16(&st.dout[i][c], static_cast<const Tin *>(p.dout) + gi);
    }
    cp_async_commit();
    return tid < cnt ? to_f32(static_cast<const Tin *>(p.beta)[(t0 + tid) * H + h]) : 0.f;
}

// Turn the staged stretch into the fp32 token vectors: k^ (and q^; normalised
// when use_l2), the decay a = exp(max(g, lb)), v (and the output cotangent), the
// write strength b. The first barrier publishes the copies and also separates
// these writes from the previous stretch's last readers; on return the vectors
// are complete and the stage is free for the next copy.
template <typename Tin, int DK, bool kRev, typename Sm>
__device__ void take_stretch(const BwdParams &p, Sm &sm, int cnt, float beta_raw) {
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    cp_async_wait_all();
    __syncthreads();
    for (int e = tid; e < cnt * DK; e += kBwdThreads) {
        const int i = e / DK, c = e % DK;
        sm.kh[i][c] = to_f32(sm.st.k[i][c]);
        const float gr = to_f32(sm.st.g[i][c]);
        sm.al[i][c] = expf(p.has_lb ? fmaxf(gr, p.lb) : gr);
        if constexpr (kRev) {
            sm.qh[i][c] = to_f32(sm.st.q[i][c]);
            sm.graw[i][c] = gr;
        }
    }
    for (int e = tid; e < cnt * kDVC; e += kBwdThreads) {
        const int i = e / kDVC, c = e % kDVC;
        sm.v[i][c] = to_f32(sm.st.v[i][c]);
        if constexpr (kRev) sm.dout[i][c] = to_f32(sm.st.dout[i][c]);
    }
    if (tid < cnt) sm.b[tid] = beta_value(beta_raw, p.beta_prob);
    __syncthreads();
    for (int i = warp; i < cnt; i += kWarps) {
        float kk = 0.f, qq = 0.f;
        for (int c = lane; c < DK; c += 32) {
            kk = fmaf(sm.kh[i][c], sm.kh[i][c], kk);
            if constexpr (kRev) qq = fmaf(sm.qh[i][c], sm.qh[i][c], qq);
        }
        kk = warp_sum(kk);
        const float rk = p.use_l2 ? rsqrtf(kk + kL2Eps) : 1.f;
        for (int c = lane; c < DK; c += 32) sm.kh[i][c] *= rk;
        if (lane == 0) sm.rk[i] = rk;
        if constexpr (kRev) {
            qq = warp_sum(qq);
            const float rq = p.use_l2 ? rsqrtf(qq + kL2Eps) : 1.f;
            for (int c = lane; c < DK; c += 32) sm.qh[i][c] *= rq;
            if (lane == 0) sm.rq[i] = rq;
        }
    }
    __syncthreads();
}

// One forward step of token i of the loaded stretch on the register tile s; ph
// selects the reduction buffer (alternating between consecutive steps).
template <typename Tin, int DK, int DV>
__device__ __forceinline__ void fwd_step(FwdSmem<Tin, DK> &sm, int i, int ph, float4 (&s)[BwdTile<DK, DV>::RP]) {
    constexpr int RP = BwdTile<DK, DV>::RP;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, vg = tid & 3, kg = tid >> 2;
    float kr[RP], ar[RP];
    load_rows<RP>(&sm.kh[i][kg * RP], kr);
    load_rows<RP>(&sm.al[i][kg * RP], ar);
    float4 pu = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int r = 0; r < RP; ++r) {
        s[r].x *= ar[r]; s[r].y *= ar[r]; s[r].z *= ar[r]; s[r].w *= ar[r];
        pu.x = fmaf(s[r].x, kr[r], pu.x); pu.y = fmaf(s[r].y, kr[r], pu.y);
        pu.z = fmaf(s[r].z, kr[r], pu.z); pu.w = fmaf(s[r].w, kr[r], pu.w);
    }
    pu = rowgroup_sum(pu);
    if (lane < 4) sm.red[ph][warp][0][vg] = pu;
    __syncthreads();
    float4 u = sm.red[ph][0][0][vg];
#pragma unroll
    for (int w = 1; w < kWarps; ++w) u = f4_add(u, sm.red[ph][w][0][vg]);
    const float b = sm.b[i];
    const float4 vv = *reinterpret_cast<const float4 *>(&sm.v[i][4 * vg]);
    const float4 d = make_float4(b * (vv.x - u.x), b * (vv.y - u.y), b * (vv.z - u.z), b * (vv.w - u.w));
#pragma unroll
    for (int r = 0; r < RP; ++r) {
        s[r].x = fmaf(kr[r], d.x, s[r].x); s[r].y = fmaf(kr[r], d.y, s[r].y);
        s[r].z = fmaf(kr[r], d.z, s[r].z); s[r].w = fmaf(kr[r], d.w, s[r].w);
    }
}

// Row `row`, slice column 4 vg of a [DK, DV] state tile whose slice starts at col0.
template <int DV>
__device__ __forceinline__ float4 *state_ptr(float *base, int row, int col0, int vg) {
    return reinterpret_cast<float4 *>(base + (long long)row * DV + col0 + 4 * vg);
}

// Recompute of the forward, storing the entering state of tokens 0, kCB, 2 kCB, ...
// One CTA per (sequence, head, 16-column slice); no cross-CTA traffic.
template <typename Tin, int DK, int DV>
__global__ void __launch_bounds__(kBwdThreads) kda_bwd_ckpt_kernel(BwdParams p) {
    using Tl = BwdTile<DK, DV>;
    constexpr int RP = Tl::RP, NS = Tl::NS;
    extern __shared__ __align__(16) uint8_t smraw[];
    FwdSmem<Tin, DK> &sm = *reinterpret_cast<FwdSmem<Tin, DK> *>(smraw);
    const int tid = threadIdx.x, vg = tid & 3, kg = tid >> 2;
    const long long nh = blockIdx.x / NS;
    const int col0 = (int)(blockIdx.x % NS) * kDVC;
    const int n = (int)(nh / p.H), h = (int)(nh % p.H);
    const long long bos = seq_begin(p, n), eos = seq_end(p, n);
    float4 s[RP];
#pragma unroll
    for (int r = 0; r < RP; ++r)
        s[r] = p.S0 ? *state_ptr<DV>(const_cast<float *>(p.S0) + nh * DK * DV, kg * RP + r, col0, vg)
                    : make_float4(0.f, 0.f, 0.f, 0.f);
    const long long c0 = first_ckpt(p, n);
    int ph = 0;
    float braw = bos < eos ? issue_stretch<Tin, DK, DV, false>(p, sm.st, bos, (int)min((long long)kCB, eos - bos), h, col0) : 0.f;
    for (long long t0 = bos; t0 < eos; t0 += kCB) {
        const int cnt = (int)min((long long)kCB, eos - t0);
        float *ck = p.ckpt + ((c0 + (t0 - bos) / kCB) * p.H + h) * DK * DV;
#pragma unroll
        for (int r = 0; r < RP; ++r) *state_ptr<DV>(ck, kg * RP + r, col0, vg) = s[r];
        take_stretch<Tin, DK, false>(p, sm, cnt, braw);
        if (t0 + kCB < eos) braw = issue_stretch<Tin, DK, DV, false>(p, sm.st, t0 + kCB, (int)min((long long)kCB, eos - t0 - kCB), h, col0);
        for (int i = 0; i < cnt; ++i, ph ^= 1) fwd_step<Tin, DK, DV>(sm, i, ph, s);
    }
}

// Reverse sweep: one cluster of NS CTAs per (sequence, head), CTA rank r owning
// value columns 16 r .. 16 r + 15.
template <typename Tin, int DK, int DV>
__global__ void __launch_bounds__(kBwdThreads) kda_bwd_kernel(BwdParams p) {
    using Tl = BwdTile<DK, DV>;
    constexpr int RP = Tl::RP, NS = Tl::NS;
    extern __shared__ __align__(16) uint8_t smraw[];
    BwdSmem<Tin, DK> &sm = *reinterpret_cast<BwdSmem<Tin, DK> *>(smraw);
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, vg = tid & 3, kg = tid >> 2;
    const long long nh = blockIdx.x / NS;
    const int col0 = rank * kDVC;
    const int n = (int)(nh / p.H), h = (int)(nh % p.H);
    const int H = p.H;
    const long long bos = seq_begin(p, n), eos = seq_end(p, n);
    const long long c0 = first_ckpt(p, n);
    // this CTA's per-token entering states, thread-major: slot i, row part r at ((i RP + r) 128 + tid)
    float4 *scr = reinterpret_cast<float4 *>(p.scratch) + (long long)blockIdx.x * kCB * RP * kBwdThreads;

    float4 ds[RP], s[RP];
#pragma unroll
    for (int r = 0; r < RP; ++r)
        ds[r] = p.dSf ? *state_ptr<DV>(const_cast<float *>(p.dSf) + nh * DK * DV, kg * RP + r, col0, vg)
                      : make_float4(0.f, 0.f, 0.f, 0.f);
    int ph = 0;
    const long long len = eos - bos;
    const long long nst = (len + kCB - 1) / kCB;
    float braw = nst > 0 ? issue_stretch<Tin, DK, DV, true>(p, sm.st, bos + (nst - 1) * kCB,
                                                            (int)(len - (nst - 1) * kCB), h, col0) : 0.f;
    for (long long cs = nst - 1; cs >= 0; --cs) {
        const long long t0 = bos + cs * kCB;
        const int cnt = (int)min((long long)kCB, eos - t0);
        const int pb = (int)(cs & 1);
        const float *ck = p.ckpt + ((c0 + cs) * H + h) * DK * DV;
        take_stretch<Tin, DK, true>(p, sm, cnt, braw);
        if (cs > 0) braw = issue_stretch<Tin, DK, DV, true>(p, sm.st, t0 - kCB, kCB, h, col0);
        // forward from the checkpoint, keeping every token's entering state; the
        // last one stays in s
#pragma unroll
        for (int r = 0; r < RP; ++r) s[r] = *state_ptr<DV>(const_cast<float *>(ck), kg * RP + r, col0, vg);
        for (int i = 0; i + 1 < cnt; ++i, ph ^= 1) {
#pragma unroll
            for (int r = 0; r < RP; ++r) scr[(i * RP + r) * kBwdThreads + tid] = s[r];
            fwd_step<Tin, DK, DV>(sm, i, ph, s);
        }
        for (int i = cnt - 1; i >= 0; --i, ph ^= 1) {
            // the previous token's entering state, fetched while this token runs
            float4 sn[RP];
            if (i > 0) {
#pragma unroll
                for (int r = 0; r < RP; ++r) sn[r] = scr[((i - 1) * RP + r) * kBwdThreads + tid];
            }
            float kr[RP], ar[RP], qr[RP];
            load_rows<RP>(&sm.kh[i][kg * RP], kr);
            load_rows<RP>(&sm.al[i][kg * RP], ar);
            load_rows<RP>(&sm.qh[i][kg * RP], qr);
            const float b = sm.b[i];
            const float4 dov = *reinterpret_cast<const float4 *>(&sm.dout[i][4 * vg]);

            // ---- S', u = S'^T k^, dS += scale q^ do^T, ddelta = dS^T k^
            float4 pu = make_float4(0.f, 0.f, 0.f, 0.f), pd = pu;
#pragma unroll
            for (int r = 0; r < RP; ++r) {
                const float qs = p.scale * qr[r];
                s[r].x *= ar[r]; s[r].y *= ar[r]; s[r].z *= ar[r]; s[r].w *= ar[r];
                pu.x = fmaf(s[r].x, kr[r], pu.x); pu.y = fmaf(s[r].y, kr[r], pu.y);
                pu.z = fmaf(s[r].z, kr[r], pu.z); pu.w = fmaf(s[r].w, kr[r], pu.w);
                ds[r].x = fmaf(qs, dov.x, ds[r].x); ds[r].y = fmaf(qs, dov.y, ds[r].y);
                ds[r].z = fmaf(qs, dov.z, ds[r].z); ds[r].w = fmaf(qs, dov.w, ds[r].w);
                pd.x = fmaf(ds[r].x, kr[r], pd.x); pd.y = fmaf(ds[r].y, kr[r], pd.y);
                pd.z = fmaf(ds[r].z, kr[r], pd.z); pd.w = fmaf(ds[r].w, kr[r], pd.w);
            }
            pu = rowgroup_sum(pu);
            pd = rowgroup_sum(pd);
            if (lane < 4) { sm.red[ph][warp][0][vg] = pu; sm.red[ph][warp][1][vg] = pd; }
            __syncthreads();
            float4 u = sm.red[ph][0][0][vg], dd = sm.red[ph][0][1][vg];
#pragma unroll
            for (int w = 1; w < kWarps; ++w) { u = f4_add(u, sm.red[ph][w][0][vg]); dd = f4_add(dd, sm.red[ph][w][1][vg]); }
            const float4 vv = *reinterpret_cast<const float4 *>(&sm.v[i][4 * vg]);
            const float4 vu = make_float4(vv.x - u.x, vv.y - u.y, vv.z - u.z, vv.w - u.w);
            const float4 dl = make_float4(b * vu.x, b * vu.y, b * vu.z, b * vu.w);
            if (tid < 4) {  // dv = b ddelta for this slice
                Tin *dv = static_cast<Tin *>(p.dv) + ((t0 + i) * H + h) * DV + col0 + 4 * tid;
                dv[0] = from_f32<Tin>(b * dd.x); dv[1] = from_f32<Tin>(b * dd.y);
                dv[2] = from_f32<Tin>(b * dd.z); dv[3] = from_f32<Tin>(b * dd.w);
            }
            // slice terms of delta . do and ddelta . (v - u)
            const float ddo = colgroup_sum(dot4(dl, dov));
            const float db = colgroup_sum(dot4(dd, vu));

            // ---- slice terms of the row sums: S' do, dS delta, S' ddelta, dS (.) S'
            float ra[RP], rb[RP], re[RP], rh[RP];
#pragma unroll
            for (int r = 0; r < RP; ++r) {
                ra[r] = colgroup_sum(dot4(s[r], dov));
                rb[r] = colgroup_sum(dot4(ds[r], dl));
                re[r] = colgroup_sum(dot4(s[r], dd));
                rh[r] = colgroup_sum(dot4(ds[r], s[r]));
            }
            if (vg == 0) {
                float g4[RP];
                load_rows<RP>(&sm.graw[i][kg * RP], g4);
#pragma unroll
                for (int r = 0; r < RP; ++r) {
                    const int c = kg * RP + r;
                    sm.pdq[pb][i][c] = p.scale * fmaf(kr[r], ddo, ra[r]);
                    sm.pdk[pb][i][c] = fmaf(-b, re[r], rb[r]);
                    const bool pass = !p.has_lb || g4[r] >= p.lb;
                    sm.pdg[pb][i][c] = pass ? fmaf(-b * kr[r], re[r], rh[r]) : 0.f;
                }
            }
            if (tid == 0) sm.pdb[pb][i] = db;
            // ---- dS <- diag(a) (dS - b k^ ddelta^T), the cotangent of the entering state
#pragma unroll
            for (int r = 0; r < RP; ++r) {
                const float bk = b * kr[r];
                ds[r].x = ar[r] * fmaf(-bk, dd.x, ds[r].x); ds[r].y = ar[r] * fmaf(-bk, dd.y, ds[r].y);
                ds[r].z = ar[r] * fmaf(-bk, dd.z, ds[r].z); ds[r].w = ar[r] * fmaf(-bk, dd.w, ds[r].w);
            }
            if (i > 0) {
#pragma unroll
                for (int r = 0; r < RP; ++r) s[r] = sn[r];
            }
        }
        // ---- the stretch's slice terms are complete in every CTA of the cluster:
        // rank r finishes tokens r, r + NS, ... (warp w takes every kWarps-th of them)
        cluster.sync();
        for (int i = rank + NS * warp; i < cnt; i += NS * kWarps) {
            constexpr int CP = DK / 32;
            float sq[CP], sk[CP], sg[CP];
            float qd = 0.f, kd = 0.f;
#pragma unroll
            for (int j = 0; j < CP; ++j) {
                const int c = lane + 32 * j;
                sq[j] = 0.f; sk[j] = 0.f; sg[j] = 0.f;
#pragma unroll
                for (int q = 0; q < NS; ++q) {
                    const BwdSmem<Tin, DK> *rs = cluster.map_shared_rank(&sm, q);
                    sq[j] += rs->pdq[pb][i][c];
                    sk[j] += rs->pdk[pb][i][c];
                    sg[j] += rs->pdg[pb][i][c];
                }
                qd = fmaf(sm.qh[i][c], sq[j], qd);
                kd = fmaf(sm.kh[i][c], sk[j], kd);
            }
            qd = p.use_l2 ? warp_sum(qd) : 0.f;
            kd = p.use_l2 ? warp_sum(kd) : 0.f;
            const float rq = sm.rq[i], rk = sm.rk[i];
#pragma unroll
            for (int j = 0; j < CP; ++j) {
                const int c = lane + 32 * j;
                const long long gi = ((t0 + i) * H + h) * DK + c;
                static_cast<Tin *>(p.dq)[gi] = from_f32<Tin>(rq * fmaf(-sm.qh[i][c], qd, sq[j]));
                static_cast<Tin *>(p.dk)[gi] = from_f32<Tin>(rk * fmaf(-sm.kh[i][c], kd, sk[j]));
                static_cast<Tin *>(p.dg)[gi] = from_f32<Tin>(sg[j]);
            }
            if (lane == 0) {
                float db = 0.f;
#pragma unroll
                for (int q = 0; q < NS; ++q) db += cluster.map_shared_rank(&sm, q)->pdb[pb][i];
                const float b = sm.b[i];
                static_cast<Tin *>(p.dbeta)[(t0 + i) * H + h] = from_f32<Tin>(p.beta_prob ? db : db * b * (1.f - b));
            }
        }
    }
    // no CTA leaves while another rank may still read its shared memory
    cluster.sync();
    if (p.dS0) {
#pragma unroll
        for (int r = 0; r < RP; ++r) *state_ptr<DV>(p.dS0 + nh * DK * DV, kg * RP + r, col0, vg) = ds[r];
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
    constexpr int NS = BwdTile<DK, DV>::NS;
    const long long heads = (long long)p.N * p.H;
    if (heads == 0) return cudaSuccess;
    const int smem_f = (int)sizeof(FwdSmem<Tin, DK>), smem_b = (int)sizeof(BwdSmem<Tin, DK>);
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(kda_bwd_ckpt_kernel<Tin, DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_f)) != cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(kda_bwd_kernel<Tin, DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_b)) != cudaSuccess)
        return e;
    if (p.cu_seqlens) {
        kda_bwd_offsets<<<1, 32, 0, st>>>(p.cu_seqlens, p.N, p.ckpt_off);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    kda_bwd_ckpt_kernel<Tin, DK, DV><<<(unsigned)(heads * NS), kBwdThreads, smem_f, st>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(heads * NS));
    cfg.blockDim = dim3(kBwdThreads);
    cfg.dynamicSmemBytes = (size_t)smem_b;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = NS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kda_bwd_kernel<Tin, DK, DV>, p);
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

// Workspace: [ckpt_off: N+1 ints, 256-byte block][per-CTA scratch: kCB states per head][checkpoints]
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
