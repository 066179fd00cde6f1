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
// cluster of Dv/32 CTAs, one per 32-column slice; inside a CTA each of the 4 warps
// owns 8 columns over all Dk rows, and lane (rg, cg) = (lane / 2, lane % 2) keeps
// rows rg*RP .. rg*RP+RP-1 (RP = Dk / 16) of columns 4 cg .. 4 cg + 3 of its warp's
// block, of S and of dS, as column pairs for the paired fp32 FMA pipe. Key-axis
// sums (u, ddelta) are reductions over the 16 row groups of a warp (no block
// barrier; the forward recompute needs none at all); value-axis sums are lane-local
// over 4 columns and then added across the 2 column groups of a warp. What sums
// over the value axis across warps and CTAs (dq^, dk^, dg, db) is linear in the
// per-warp terms: the 4 warps' terms of a token meet in shared memory (one block
// barrier per token), every CTA keeps its slice's terms for the kCB tokens of a
// stretch, and after the stretch the cluster adds them across its CTAs through
// distributed shared memory (a fixed rank order, so the result is deterministic)
// and applies the L2-norm and sigmoid chain rules once per token.
//
// The entering state of every token comes from a checkpoint written every kCB
// tokens by a recompute of the forward (`kda_bwd_ckpt_kernel`, one warp group
// stepping while another takes in the next stretch). Per stretch of kCB tokens the
// reverse sweep (`kda_bwd_kernel`) prepares the stretch (intake, then the forward
// once from its checkpoint, keeping each token's decayed state S' = diag(a) S in
// a per-CTA scratch that stays in L2 and u = S'^T k^ in shared memory), walks the
// tokens back, and lets the cluster add the slice terms. When the grid has at most
// one CTA per SM a CTA has two warp groups, one preparing the next stretch into a
// second buffer set while the other walks the current one; otherwise one group
// does both in turn and two CTAs share an SM. Checkpoints and scratch are
// thread-major per CTA (coalesced).
#include <cooperative_groups.h>

#include <algorithm>

#include "kda_common.cuh"
#include "kda_bwd.cuh"
#include "kda_stage.cuh"
#include "kda_seg.cuh"

namespace kda {

namespace {

namespace cg = cooperative_groups;

constexpr int kGrp = 128;              // threads of one warp group
constexpr int kGW = kGrp / 32;         // warps per group
constexpr int kRevThreads = 2 * kGrp;  // reverse sweep: a walking group and a preparing group
constexpr int kCB = 16;                // tokens per checkpoint (one stretch)
constexpr int kDVC = 32;               // value columns per CTA: 8 per warp of a group

// Lane (rg, cg) = (lane / 2, lane % 2) of group warp w holds rows rg*RP .. rg*RP+RP-1
// and columns 8 w + 4 cg .. 8 w + 4 cg + 3 of its CTA's slice.
template <int DK, int DV>
struct BwdTile {
    static constexpr int RP = DK / 16, NS = DV / kDVC;
    static_assert(kGW * 8 == kDVC && RP * 16 == DK && RP >= 2 && RP <= 8 && NS >= 1 && NS <= 8, "state tiling");
};

// Raw inputs of one stretch, copied in by cp.async while the previous stretch runs.
template <typename Tin, int DK>
struct Stage {
    Tin k[kCB][DK], g[kCB][DK], q[kCB][DK];  // q: reverse sweep only
    Tin v[kCB][kDVC], dout[kCB][kDVC];       // this CTA's value columns; dout: reverse sweep only
};

// Token vectors of one stretch (fp32; k^ normalised): what the forward recompute
// needs. al holds the decay a = exp(max(g, lb)), negated where g < lb (the clamp
// is taken there and the gate gets no gradient).
template <int DK>
struct FwdVec {
    float kh[kCB][DK], al[kCB][DK];
    float v[kCB][kDVC];
    float b[kCB], rk[kCB];
};

// The reverse sweep adds q^, the output cotangent and u = S'^T k^ of every token
// (from the stretch's forward recompute).
template <int DK>
struct RevVec : FwdVec<DK> {
    float qh[kCB][DK];
    float dout[kCB][kDVC];
    float u[kCB][kDVC];
    float rq[kCB];
};

template <typename Tin, int DK>
struct CkptSmem {
    Stage<Tin, DK> st;
    FwdVec<DK> tv[2];
};

// Reverse sweep: two sets of token vectors (the walked stretch and the one being
// prepared), the walking group's per-warp terms of the current token (alternating
// between tokens), and the per-CTA terms of dq^, dk^, dg ([0], [1], [2]) and db of
// the walked stretch.
template <typename Tin, int DK>
struct RevSmem {
    Stage<Tin, DK> st;
    RevVec<DK> tv[2];
    float wp[2][kGW][3][DK];
    float wdb[2][kGW];
    float pd[3][kCB][DK];
    float pdb[kCB];
};

// Thread and warp index within the thread's group of 128.
__device__ __forceinline__ int gtid() { return threadIdx.x & (kGrp - 1); }
__device__ __forceinline__ int gwarp() { return (threadIdx.x >> 5) & (kGW - 1); }
// Barrier of the whole block (id 0) or of one group of 128 threads (named barrier id).
__device__ __forceinline__ void grp_sync(int id) {
    if (id == 0) __syncthreads();
    else asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(kGrp) : "memory");
}

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
    if constexpr (RP % 4 == 0) {
#pragma unroll
        for (int j = 0; j < RP; j += 4) {
            const float4 x = *reinterpret_cast<const float4 *>(src + j);
            out[j] = x.x; out[j + 1] = x.y; out[j + 2] = x.z; out[j + 3] = x.w;
        }
    } else if constexpr (RP == 2) {
        const float2 x = *reinterpret_cast<const float2 *>(src);
        out[0] = x.x; out[1] = x.y;
    } else {
        out[0] = src[0];
    }
}

template <int RP>
__device__ __forceinline__ void store_rows(float *dst, const float (&x)[RP]) {
    if constexpr (RP == 4) {
        *reinterpret_cast<float4 *>(dst) = make_float4(x[0], x[1], x[2], x[3]);
    } else if constexpr (RP == 2) {
        *reinterpret_cast<float2 *>(dst) = make_float2(x[0], x[1]);
    } else {
        dst[0] = x[0];
    }
}

__device__ __forceinline__ float dot4(float4 a, float4 b) { return a.x * b.x + a.y * b.y + a.z * b.z + a.w * b.w; }

// Sum of 4 column values over the 16 row groups of a warp (lane bits 4..1), returned
// to every lane of the column group: reduce-scatter over bits 4 and 3 (each lane
// keeps half of its values at each step), butterfly over bits 2 and 1, then each
// sum is gathered from the lanes that hold it (value v sits in lanes with bits
// 4..3 = v). 9 shuffles.
__device__ __forceinline__ float4 colsum4(float4 x) {
    const int lane = threadIdx.x & 31, cg = lane & 1;
    const bool h4 = lane & 16, h3 = lane & 8;
    float a0 = h4 ? x.z : x.x, a1 = h4 ? x.w : x.y;
    a0 += __shfl_xor_sync(0xffffffffu, h4 ? x.x : x.z, 16);
    a1 += __shfl_xor_sync(0xffffffffu, h4 ? x.y : x.w, 16);
    float m = h3 ? a1 : a0;
    m += __shfl_xor_sync(0xffffffffu, h3 ? a0 : a1, 8);
    m += __shfl_xor_sync(0xffffffffu, m, 4);
    m += __shfl_xor_sync(0xffffffffu, m, 2);
    return make_float4(__shfl_sync(0xffffffffu, m, cg), __shfl_sync(0xffffffffu, m, 8 + cg),
                       __shfl_sync(0xffffffffu, m, 16 + cg), __shfl_sync(0xffffffffu, m, 24 + cg));
}

// Start the copy of tokens [t0, t0 + cnt) of head h into the stage: k, g (and q
// for the reverse sweep) rows, and this CTA's columns of v (and of the output
// cotangent), in 16-byte pieces, by the calling group. Returns this thread's raw
// beta (thread i < cnt of the group holds token i's), left unconverted so that its
// load completes in the background like the copies.
template <typename Tin, int DK, int DV, bool kRev>
__device__ __forceinline__ Tin issue_stretch(const BwdParams &p, Stage<Tin, DK> &st, long long t0, int cnt, int h,
                                             int col0) {
    constexpr int EP = 16 / (int)sizeof(Tin);  // elements per piece
    constexpr int RK = DK / EP, RV = kDVC / EP;
    const int tid = gtid(), H = p.H;
    for (int e = tid; e < cnt * RK; e += kGrp) {
        const int i = e / RK, c = (e % RK) * EP;
        const long long gi = ((t0 + i) * H + h) * DK + c;
        cp_async16(&st.k[i][c], static_cast<const Tin *>(p.k) + gi);
        cp_async16(&st.g[i][c], static_cast<const Tin *>(p.g) + gi);
        if constexpr (kRev) cp_async16(&st.q[i][c], static_cast<const Tin *>(p.q) + gi);
    }
    for (int e = tid; e < cnt * RV; e += kGrp) {
        const int i = e / RV, c = (e % RV) * EP;
        const long long gi = ((t0 + i) * H + h) * DV + col0 + c;
        cp_async16(&st.v[i][c], static_cast<const Tin *>(p.v) + gi);
        if constexpr (kRev) cp_async16(&st.dout[i][c], static_cast<const Tin *>(p.dout) + gi);
    }
    cp_async_commit();
    return tid < cnt ? static_cast<const Tin *>(p.beta)[(t0 + tid) * H + h] : Tin(0.f);
}

// Turn the staged stretch into the fp32 token vectors tv: k^ (and q^; normalised
// when use_l2), the signed decay al, v (and the output cotangent), the write
// strength b. Each key row is taken by 16 threads (DK / 16 elements each) that form
// its squared norm with shuffles. The first barrier (`bar`, the calling group's)
// publishes the copies and separates these writes from earlier readers of tv; on
// return the vectors are complete and the stage is free for the next copy.
template <typename Tin, int DK, bool kRev, typename TV>
__device__ void take_stretch(const BwdParams &p, Stage<Tin, DK> &st, TV &tv, int cnt, Tin beta_raw, int bar) {
    constexpr int TPR = 16, E = DK / TPR;
    const int tid = gtid();
    cp_async_wait_all();
    grp_sync(bar);
    const int c = (tid % TPR) * E;
    // uniform trip count: every lane joins the shuffles; rows past cnt read row 0
    // and store nothing
    for (int i0 = 0; i0 < cnt; i0 += kGrp / TPR) {
        const int i = i0 + tid / TPR;
        const bool live = i < cnt;
        const int ir = live ? i : 0;
        float kx[E], gx[E];
        stage_cvt<E>(&st.k[ir][c], kx);
        stage_cvt<E>(&st.g[ir][c], gx);
        float kk = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) kk = fmaf(kx[e], kx[e], kk);
#pragma unroll
        for (int o = TPR / 2; o > 0; o >>= 1) kk += __shfl_xor_sync(0xffffffffu, kk, o);
        const float rk = p.use_l2 ? rsqrtf(kk + kL2Eps) : 1.f;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            kx[e] *= rk;
            const bool pass = !p.has_lb || gx[e] >= p.lb;
            const float a = expf(pass ? gx[e] : p.lb);
            gx[e] = pass ? a : -a;
        }
        if (live) {
            store_vec<E>(&tv.kh[i][c], kx);
            store_vec<E>(&tv.al[i][c], gx);
            if (tid % TPR == 0) tv.rk[i] = rk;
        }
        if constexpr (kRev) {
            float qx[E];
            stage_cvt<E>(&st.q[ir][c], qx);
            float qq = 0.f;
#pragma unroll
            for (int e = 0; e < E; ++e) qq = fmaf(qx[e], qx[e], qq);
#pragma unroll
            for (int o = TPR / 2; o > 0; o >>= 1) qq += __shfl_xor_sync(0xffffffffu, qq, o);
            const float rq = p.use_l2 ? rsqrtf(qq + kL2Eps) : 1.f;
#pragma unroll
            for (int e = 0; e < E; ++e) qx[e] *= rq;
            if (live) {
                store_vec<E>(&tv.qh[i][c], qx);
                if (tid % TPR == 0) tv.rq[i] = rq;
            }
        }
    }
    for (int e = tid; e < cnt * kDVC; e += kGrp) {
        const int i = e / kDVC, cc = e % kDVC;
        tv.v[i][cc] = to_f32(st.v[i][cc]);
        if constexpr (kRev) tv.dout[i][cc] = to_f32(st.dout[i][cc]);
    }
    if (tid < cnt) tv.b[tid] = beta_value(to_f32(beta_raw), p.beta_prob);
    grp_sync(bar);
}

// One forward step of token i of the stretch in tv on this lane's register tile s
// (rows rg*RP.., slice columns 8 w + 4 cg .. of group warp w). Warp-local. With
// keep_s, the decayed state S' = diag(a) S goes to keep_s[r * 128] (this thread's
// slots) and u = S'^T k^ of the lane's columns to keep_u[0..3] (lanes 0 and 1).
template <typename Tin, int DK, int DV, typename TV>
__device__ __forceinline__ void fwd_step(const TV &tv, int i, float4 (&s)[BwdTile<DK, DV>::RP],
                                         float4 *keep_s = nullptr, float *keep_u = nullptr) {
    constexpr int RP = BwdTile<DK, DV>::RP;
    const int lane = threadIdx.x & 31, warp = gwarp(), rg = lane >> 1, cg = lane & 1;
    float kr[RP], ar[RP];
    load_rows<RP>(&tv.kh[i][rg * RP], kr);
    load_rows<RP>(&tv.al[i][rg * RP], ar);
    const float b = tv.b[i];
    const float4 vv = *reinterpret_cast<const float4 *>(&tv.v[i][8 * warp + 4 * cg]);
    // decay and this lane's part of u on the paired fp32 FMA pipe (two chains)
    const float2 z2 = make_float2(0.f, 0.f);
    float2 pu[2][2] = {{z2, z2}, {z2, z2}};
#pragma unroll
    for (int r = 0; r < RP; ++r) {
        const float a = fabsf(ar[r]);
        const float2 a2 = make_float2(a, a), k2 = make_float2(kr[r], kr[r]);
        const float2 lo = __fmul2_rn(make_float2(s[r].x, s[r].y), a2), hi = __fmul2_rn(make_float2(s[r].z, s[r].w), a2);
        s[r] = make_float4(lo.x, lo.y, hi.x, hi.y);
        pu[r & 1][0] = __ffma2_rn(lo, k2, pu[r & 1][0]);
        pu[r & 1][1] = __ffma2_rn(hi, k2, pu[r & 1][1]);
    }
    if (keep_s) {
#pragma unroll
        for (int r = 0; r < RP; ++r) keep_s[r * kGrp] = s[r];
    }
    const float2 u01 = __fadd2_rn(pu[0][0], pu[1][0]), u23 = __fadd2_rn(pu[0][1], pu[1][1]);
    const float4 u = colsum4(make_float4(u01.x, u01.y, u23.x, u23.y));
    if (keep_u && lane < 2) *reinterpret_cast<float4 *>(keep_u + 4 * cg) = u;
    const float2 d01 = make_float2(b * (vv.x - u.x), b * (vv.y - u.y)), d23 = make_float2(b * (vv.z - u.z), b * (vv.w - u.w));
#pragma unroll
    for (int r = 0; r < RP; ++r) {
        const float2 k2 = make_float2(kr[r], kr[r]);
        const float2 lo = __ffma2_rn(k2, d01, make_float2(s[r].x, s[r].y));
        const float2 hi = __ffma2_rn(k2, d23, make_float2(s[r].z, s[r].w));
        s[r] = make_float4(lo.x, lo.y, hi.x, hi.y);
    }
}

// This lane's element (row, first of its 4 columns) of a user [DK, DV] state whose
// CTA slice starts at col0.
template <int DV>
__device__ __forceinline__ float4 *state_ptr(float *base, int row, int col0) {
    const int lane = threadIdx.x & 31;
    return reinterpret_cast<float4 *>(base + (long long)row * DV + col0 + 8 * gwarp() + 4 * (lane & 1));
}

// Recompute of the forward, storing the entering state of tokens 0, kCB, 2 kCB, ...
// (thread-major: checkpoint j of CTA slice r at ((j H + h) NS + r) RP 128 float4).
// One CTA of two warp groups per (sequence, head, 32-column slice), no cross-CTA
// traffic: warps 0..3 step stretch j - 1 forward from one token-vector buffer while
// warps 4..7 take stretch j into the other (and start the copy of stretch j + 1).
template <typename Tin, int DK, int DV>
__global__ void __launch_bounds__(2 * kGrp) kda_bwd_ckpt_kernel(BwdParams p) {
    using Tl = BwdTile<DK, DV>;
    constexpr int RP = Tl::RP, NS = Tl::NS;
    constexpr int kIntakeBar = 1;
    extern __shared__ __align__(16) uint8_t smraw[];
    CkptSmem<Tin, DK> &sm = *reinterpret_cast<CkptSmem<Tin, DK> *>(smraw);
    const bool stepper = threadIdx.x < kGrp;
    const int ltid = gtid(), rg = (threadIdx.x & 31) >> 1;
    const long long nh = blockIdx.x / NS;
    const int rank = (int)(blockIdx.x % NS), col0 = rank * kDVC;
    const int n = (int)(nh / p.H), h = (int)(nh % p.H);
    const long long bos = seq_begin(p, n), eos = seq_end(p, n);
    const long long nst = (eos - bos + kCB - 1) / kCB;
    float4 s[RP];
    if (stepper) {
#pragma unroll
        for (int r = 0; r < RP; ++r)
            s[r] = p.S0 ? *state_ptr<DV>(const_cast<float *>(p.S0) + nh * DK * DV, rg * RP + r, col0)
                        : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    const long long c0 = first_ckpt(p, n);
    float4 *ckb = reinterpret_cast<float4 *>(p.ckpt);
    Tin braw = Tin(0.f);
    if (!stepper && nst > 0)
        braw = issue_stretch<Tin, DK, DV, false>(p, sm.st, bos, (int)min((long long)kCB, eos - bos), h, col0);
    for (long long j = 0; j <= nst; ++j) {
        if (stepper) {
            if (j >= 1) {
                const long long t0 = bos + (j - 1) * kCB;
                const int cnt = (int)min((long long)kCB, eos - t0);
                float4 *ck = ckb + (((c0 + j - 1) * p.H + h) * NS + rank) * (RP * kGrp);
#pragma unroll
                for (int r = 0; r < RP; ++r) ck[r * kGrp + ltid] = s[r];
                const FwdVec<DK> &tv = sm.tv[(j - 1) & 1];
                for (int i = 0; i < cnt; ++i) fwd_step<Tin, DK, DV>(tv, i, s);
            }
        } else if (j < nst) {
            const long long t0 = bos + j * kCB;
            const int cnt = (int)min((long long)kCB, eos - t0);
            take_stretch<Tin, DK, false>(p, sm.st, sm.tv[j & 1], cnt, braw, kIntakeBar);
            if (t0 + kCB < eos)
                braw = issue_stretch<Tin, DK, DV, false>(p, sm.st, t0 + kCB, (int)min((long long)kCB, eos - t0 - kCB), h, col0);
        }
        __syncthreads();
    }
}

__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }

// Reverse sweep: one cluster of NS CTAs per (sequence, head), CTA rank r owning
// value columns 32 r .. 32 r + 31. A CTA has two groups of 4 warps. The preparing
// group (warps 4..7) takes in the next stretch to walk and reruns it forward from
// its checkpoint, keeping every token's decayed state S' (a scratch buffer) and
// u = S'^T k^ (its token vectors); meanwhile the walking group (warps 0..3) walks
// the previous stretch back from the other buffer set. Iteration it prepares
// stretch nst-1-it and walks stretch nst-it; the walking group then adds, with the
// cluster, the slice terms of the stretch it walked at the start of the next
// iteration. Cluster barriers: B (arrive and wait, all threads) at the start of an
// iteration, after those adds, frees the slice-term buffers and the token vectors
// that the adds read; A at the end, after a block barrier, publishes every rank's
// terms of the walked stretch.
// With kSplit false the CTA is one group of 128 threads that does both jobs in
// turn (same order, same buffers): the form for grids of more than one CTA per SM,
// where two such CTAs share an SM.
template <typename Tin, int DK, int DV, bool kSplit>
__global__ void __launch_bounds__(kSplit ? kRevThreads : kGrp) kda_bwd_kernel(BwdParams p) {
    using Tl = BwdTile<DK, DV>;
    constexpr int RP = Tl::RP, NS = Tl::NS, RH = RP / 2;
    constexpr int kWalkBar = 1, kPrepBar = 2;
    extern __shared__ __align__(16) uint8_t smraw[];
    RevSmem<Tin, DK> &sm = *reinterpret_cast<RevSmem<Tin, DK> *>(smraw);
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const bool walker = !kSplit || threadIdx.x < kGrp, preparer = !kSplit || threadIdx.x >= kGrp;
    const int ltid = gtid(), lane = threadIdx.x & 31, lwarp = gwarp(), rg = lane >> 1, cgp = lane & 1;
    const int cs0 = 8 * lwarp + 4 * cgp;  // this lane's first column within the CTA slice
    const long long nh = blockIdx.x / NS;
    const int col0 = rank * kDVC;
    const int n = (int)(nh / p.H), h = (int)(nh % p.H);
    const int H = p.H;
    const long long bos = seq_begin(p, n), eos = seq_end(p, n);
    const long long c0 = first_ckpt(p, n);
    const float4 *ckb = reinterpret_cast<const float4 *>(p.ckpt);
    // two scratch buffers per CTA; slot i, row part r of group thread t at ((i RP + r) 128 + t)
    float4 *scr = reinterpret_cast<float4 *>(p.scratch) + (long long)blockIdx.x * 2 * kCB * RP * kGrp + ltid;
    const long long len = eos - bos;
    const long long nst = (len + kCB - 1) / kCB;

    float4 ds[RP], s[RP];
    if (walker) {
#pragma unroll
        for (int r = 0; r < RP; ++r)
            ds[r] = p.dSf ? *state_ptr<DV>(const_cast<float *>(p.dSf) + nh * DK * DV, rg * RP + r, col0)
                          : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    Tin braw = Tin(0.f);
    if (preparer && nst > 0)
        braw = issue_stretch<Tin, DK, DV, true>(p, sm.st, bos + (nst - 1) * kCB, (int)(len - (nst - 1) * kCB), h, col0);

    // the cluster's terms of the stretch walked last (buffer b): rank r finishes tokens
    // r, r + NS, ... (group warp w takes every kGW-th of them)
    auto finish_stretch = [&](long long cs, int b) {
        const RevVec<DK> &tv = sm.tv[b];
        const long long t0 = bos + cs * kCB;
        const int cnt = (int)min((long long)kCB, eos - t0);
        for (int i = rank + NS * lwarp; i < cnt; i += NS * kGW) {
            constexpr int CP = DK / 32;  // channels per lane, contiguous: c0 .. c0 + CP - 1
            const int cb = CP * lane;
            float sq[CP], sk[CP], sg[CP], qv[CP], kv[CP];
#pragma unroll
            for (int j = 0; j < CP; ++j) { sq[j] = 0.f; sk[j] = 0.f; sg[j] = 0.f; }
#pragma unroll
            for (int q = 0; q < NS; ++q) {
                const RevSmem<Tin, DK> *rs = cluster.map_shared_rank(&sm, q);
                float x[CP], y[CP], z[CP];
                load_rows<CP>(&rs->pd[0][i][cb], x);
                load_rows<CP>(&rs->pd[1][i][cb], y);
                load_rows<CP>(&rs->pd[2][i][cb], z);
#pragma unroll
                for (int j = 0; j < CP; ++j) { sq[j] += x[j]; sk[j] += y[j]; sg[j] += z[j]; }
            }
            load_rows<CP>(&tv.qh[i][cb], qv);
            load_rows<CP>(&tv.kh[i][cb], kv);
            float qd = 0.f, kd = 0.f;
#pragma unroll
            for (int j = 0; j < CP; ++j) { qd = fmaf(qv[j], sq[j], qd); kd = fmaf(kv[j], sk[j], kd); }
            qd = p.use_l2 ? warp_sum(qd) : 0.f;
            kd = p.use_l2 ? warp_sum(kd) : 0.f;
            const float rq = tv.rq[i], rk = tv.rk[i];
            const long long gi = ((t0 + i) * H + h) * DK + cb;
#pragma unroll
            for (int j = 0; j < CP; ++j) {
                static_cast<Tin *>(p.dq)[gi + j] = from_f32<Tin>(rq * fmaf(-qv[j], qd, sq[j]));
                static_cast<Tin *>(p.dk)[gi + j] = from_f32<Tin>(rk * fmaf(-kv[j], kd, sk[j]));
                static_cast<Tin *>(p.dg)[gi + j] = from_f32<Tin>(sg[j]);
            }
            if (lane == 0) {
                float db = 0.f;
#pragma unroll
                for (int q = 0; q < NS; ++q) db += cluster.map_shared_rank(&sm, q)->pdb[i];
                const float b = tv.b[i];
                static_cast<Tin *>(p.dbeta)[(t0 + i) * H + h] = from_f32<Tin>(p.beta_prob ? db : db * b * (1.f - b));
            }
        }
    };

    // prepare stretch cs into buffer b: intake, then the forward from its checkpoint
    auto prepare = [&](long long cs, int b) {
        const long long t0 = bos + cs * kCB;
        const int cnt = (int)min((long long)kCB, eos - t0);
        take_stretch<Tin, DK, true>(p, sm.st, sm.tv[b], cnt, braw, kPrepBar);
        if (cs > 0) braw = issue_stretch<Tin, DK, DV, true>(p, sm.st, t0 - kCB, kCB, h, col0);
        const float4 *ck = ckb + (((c0 + cs) * H + h) * NS + rank) * (RP * kGrp);
#pragma unroll
        for (int r = 0; r < RP; ++r) s[r] = ck[r * kGrp + ltid];
        float4 *sb = scr + b * kCB * RP * kGrp;
        for (int i = 0; i < cnt; ++i) fwd_step<Tin, DK, DV>(sm.tv[b], i, s, sb + i * RP * kGrp, &sm.tv[b].u[i][8 * lwarp]);
    };

    int ph = 0;  // alternates between the per-warp term buffers token by token
    // walk stretch cs back from buffer b (the walking threads)
    auto walk = [&](long long cs, int b) {
        const RevVec<DK> &tv = sm.tv[b];
        const long long t0 = bos + cs * kCB;
        const int cnt = (int)min((long long)kCB, eos - t0);
        const float4 *sb = scr + b * kCB * RP * kGrp;
        float4 sp[RP];  // S' of the current token, fetched one token ahead
#pragma unroll
        for (int r = 0; r < RP; ++r) sp[r] = sb[((cnt - 1) * RP + r) * kGrp];
        for (int i = cnt - 1; i >= 0; --i, ph ^= 1) {
#pragma unroll
            for (int r = 0; r < RP; ++r) s[r] = sp[r];
            if (i > 0) {
#pragma unroll
                for (int r = 0; r < RP; ++r) sp[r] = sb[((i - 1) * RP + r) * kGrp];
            }
            float kr[RP], ar[RP], qr[RP];
            load_rows<RP>(&tv.kh[i][rg * RP], kr);
            load_rows<RP>(&tv.al[i][rg * RP], ar);
            load_rows<RP>(&tv.qh[i][rg * RP], qr);
            const float bt = tv.b[i];
            const float4 dov = *reinterpret_cast<const float4 *>(&tv.dout[i][cs0]);
            const float4 vv = *reinterpret_cast<const float4 *>(&tv.v[i][cs0]);
            const float4 u = *reinterpret_cast<const float4 *>(&tv.u[i][cs0]);

            // ---- dS += scale q^ do^T, then ddelta = dS^T k^ (column sums); column
            // pairs on the paired fp32 FMA pipe, two chains
            const float2 do01 = make_float2(dov.x, dov.y), do23 = make_float2(dov.z, dov.w);
            const float2 z2 = make_float2(0.f, 0.f);
            float2 pd[2][2] = {{z2, z2}, {z2, z2}};
#pragma unroll
            for (int r = 0; r < RP; ++r) {
                const float qs = p.scale * qr[r];
                const float2 qs2 = make_float2(qs, qs), k2 = make_float2(kr[r], kr[r]);
                const float2 lo = __ffma2_rn(qs2, do01, make_float2(ds[r].x, ds[r].y));
                const float2 hi = __ffma2_rn(qs2, do23, make_float2(ds[r].z, ds[r].w));
                ds[r] = make_float4(lo.x, lo.y, hi.x, hi.y);
                pd[r & 1][0] = __ffma2_rn(lo, k2, pd[r & 1][0]);
                pd[r & 1][1] = __ffma2_rn(hi, k2, pd[r & 1][1]);
            }
            const float2 e01 = __fadd2_rn(pd[0][0], pd[1][0]), e23 = __fadd2_rn(pd[0][1], pd[1][1]);
            const float4 dd = colsum4(make_float4(e01.x, e01.y, e23.x, e23.y));
            const float4 vu = make_float4(vv.x - u.x, vv.y - u.y, vv.z - u.z, vv.w - u.w);
            const float4 dl = make_float4(bt * vu.x, bt * vu.y, bt * vu.z, bt * vu.w);
            if (lane < 2) {  // dv = b ddelta for this lane's columns
                Tin *dv = static_cast<Tin *>(p.dv) + ((t0 + i) * H + h) * DV + col0 + cs0;
                dv[0] = from_f32<Tin>(bt * dd.x); dv[1] = from_f32<Tin>(bt * dd.y);
                dv[2] = from_f32<Tin>(bt * dd.z); dv[3] = from_f32<Tin>(bt * dd.w);
            }
            // this lane's terms of delta . do and ddelta . (v - u) (its 4 columns)
            const float ddo = dot4(dl, dov);
            float db = dot4(dd, vu);

            // ---- this lane's terms of the row sums S' do, dS delta, S' ddelta, dS (.) S'
            const float2 dl01 = make_float2(dl.x, dl.y), dl23 = make_float2(dl.z, dl.w);
            const float2 dd01 = make_float2(dd.x, dd.y), dd23 = make_float2(dd.z, dd.w);
            float tq[RP], tk[RP], tg[RP];
#pragma unroll
            for (int r = 0; r < RP; ++r) {
                const float2 s01 = make_float2(s[r].x, s[r].y), s23 = make_float2(s[r].z, s[r].w);
                const float2 g01 = make_float2(ds[r].x, ds[r].y), g23 = make_float2(ds[r].z, ds[r].w);
                const float2 xa = __ffma2_rn(s23, do23, __fmul2_rn(s01, do01));
                const float2 xb = __ffma2_rn(g23, dl23, __fmul2_rn(g01, dl01));
                const float2 xe = __ffma2_rn(s23, dd23, __fmul2_rn(s01, dd01));
                const float2 xh = __ffma2_rn(g23, s23, __fmul2_rn(g01, s01));
                const float ra = xa.x + xa.y, rb = xb.x + xb.y, re = xe.x + xe.y, rh = xh.x + xh.y;
                tq[r] = p.scale * fmaf(kr[r], ddo, ra);
                tk[r] = fmaf(-bt, re, rb);
                tg[r] = ar[r] > 0.f ? fmaf(-bt * kr[r], re, rh) : 0.f;
            }
            // ---- the warp's terms: add the two column groups (lane bit 0), each lane
            // keeping half of its rows (cg 0 the first RH, cg 1 the last RH)
            float wq[RH], wk[RH], wg[RH];
#pragma unroll
            for (int j = 0; j < RH; ++j) {
                const float kq = cgp ? tq[RH + j] : tq[j], sq = cgp ? tq[j] : tq[RH + j];
                const float kk = cgp ? tk[RH + j] : tk[j], sk = cgp ? tk[j] : tk[RH + j];
                const float kg = cgp ? tg[RH + j] : tg[j], sg = cgp ? tg[j] : tg[RH + j];
                wq[j] = kq + __shfl_xor_sync(0xffffffffu, sq, 1);
                wk[j] = kk + __shfl_xor_sync(0xffffffffu, sk, 1);
                wg[j] = kg + __shfl_xor_sync(0xffffffffu, sg, 1);
            }
            db += __shfl_xor_sync(0xffffffffu, db, 1);
            const int row0 = rg * RP + cgp * RH;
            store_rows<RH>(&sm.wp[ph][lwarp][0][row0], wq);
            store_rows<RH>(&sm.wp[ph][lwarp][1][row0], wk);
            store_rows<RH>(&sm.wp[ph][lwarp][2][row0], wg);
            if (lane == 0) sm.wdb[ph][lwarp] = db;
            // ---- dS <- diag(a) (dS - b k^ ddelta^T), the cotangent of the entering state
#pragma unroll
            for (int r = 0; r < RP; ++r) {
                const float nbk = -bt * kr[r], a = fabsf(ar[r]);
                const float2 nbk2 = make_float2(nbk, nbk), a2 = make_float2(a, a);
                const float2 lo = __fmul2_rn(a2, __ffma2_rn(nbk2, dd01, make_float2(ds[r].x, ds[r].y)));
                const float2 hi = __fmul2_rn(a2, __ffma2_rn(nbk2, dd23, make_float2(ds[r].z, ds[r].w)));
                ds[r] = make_float4(lo.x, lo.y, hi.x, hi.y);
            }
            // ---- the CTA's terms of token i: the 4 warps' terms added in a fixed order
            grp_sync(kWalkBar);
            constexpr int Q4 = DK / 4;  // float4 per quantity row
            if (ltid < 3 * Q4) {
                const int qn = ltid / Q4, c = (ltid % Q4) * 4;
                float4 acc = *reinterpret_cast<const float4 *>(&sm.wp[ph][0][qn][c]);
#pragma unroll
                for (int w = 1; w < kGW; ++w) {
                    const float4 x = *reinterpret_cast<const float4 *>(&sm.wp[ph][w][qn][c]);
                    acc.x += x.x; acc.y += x.y; acc.z += x.z; acc.w += x.w;
                }
                *reinterpret_cast<float4 *>(&sm.pd[qn][i][c]) = acc;
            } else if (ltid == kGrp - 1) {
                float acc = sm.wdb[ph][0];
#pragma unroll
                for (int w = 1; w < kGW; ++w) acc += sm.wdb[ph][w];
                sm.pdb[i] = acc;
            }
        }
    };

    if constexpr (kSplit) {
        // iteration it prepares stretch nst-1-it and walks stretch nst-it
        for (long long it = 0; it <= nst; ++it) {
            if (walker) {
                if (it >= 2) finish_stretch(nst - it + 1, (int)((it - 2) & 1));
                cluster_arrive();  // B
                cluster_wait();
                if (it >= 1) walk(nst - it, (int)((it - 1) & 1));
            } else {
                cluster_arrive();  // B: the walking group's adds have read the token vectors
                cluster_wait();
                if (it < nst) prepare(nst - 1 - it, (int)(it & 1));
            }
            __syncthreads();
            cluster_arrive();  // A: every rank's terms of the stretch walked in this iteration are complete
            cluster_wait();
        }
        if (walker && nst >= 1) finish_stretch(0, (int)((nst - 1) & 1));
    } else {
        // one buffer set: prepare a stretch (overlapping the B wait), walk it, add its terms
        for (long long cs = nst - 1; cs >= 0; --cs) {
            prepare(cs, 0);
            if (cs != nst - 1) cluster_wait();  // B: every rank has added the previous stretch's terms
            walk(cs, 0);
            cluster_arrive();  // A
            cluster_wait();
            finish_stretch(cs, 0);
            cluster_arrive();  // B
        }
        if (nst > 0) cluster_wait();
    }
    // no CTA leaves while another may still read its shared memory
    cluster_arrive();
    cluster_wait();
    if (walker && p.dS0) {
#pragma unroll
        for (int r = 0; r < RP; ++r) *state_ptr<DV>(p.dS0 + nh * DK * DV, rg * RP + r, col0) = ds[r];
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
    const int smem_f = (int)sizeof(CkptSmem<Tin, DK>), smem_b = (int)sizeof(RevSmem<Tin, DK>);
    static_assert(sizeof(RevSmem<Tin, DK>) <= 232448, "shared memory of the reverse sweep");
    cudaError_t e;
    int dev = 0, sms = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    // one CTA per SM or fewer: walking and preparing groups side by side; more: one
    // group doing both, two CTAs per SM
    const bool split = heads * NS <= (long long)sms;
    auto rev = split ? kda_bwd_kernel<Tin, DK, DV, true> : kda_bwd_kernel<Tin, DK, DV, false>;
    if ((e = cudaFuncSetAttribute(kda_bwd_ckpt_kernel<Tin, DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_f)) != cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(rev, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_b)) != cudaSuccess)
        return e;
    if (p.cu_seqlens) {
        count_launch();
        kda_bwd_offsets<<<1, 32, 0, st>>>(p.cu_seqlens, p.N, p.ckpt_off);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    count_launch();
    kda_bwd_ckpt_kernel<Tin, DK, DV><<<(unsigned)(heads * NS), 2 * kGrp, smem_f, st>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(heads * NS));
    cfg.blockDim = dim3(split ? kRevThreads : kGrp);
    cfg.dynamicSmemBytes = (size_t)smem_b;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = NS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    count_launch();
    return cudaLaunchKernelEx(&cfg, rev, p);
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

// Workspace: [ckpt_off: N+1 ints, 256-byte block][per-CTA scratch: two stretches of states][checkpoints]
size_t bwd_workspace_bytes_min(bool varlen, long long T, int N, int H, int Dk, int Dv) {
    const long long nck = varlen ? (T + kCB - 1) / kCB + N : (long long)N * ((T + kCB - 1) / kCB);
    const size_t head = (((size_t)(N + 1) * 4 + 255) / 256) * 256;
    return head + 2 * (size_t)N * H * kCB * Dk * Dv * 4 + (size_t)nck * H * Dk * Dv * 4;
}

// Segments: with few (sequence, head) chains the sweeps would leave most SMs idle, so
// every sequence is cut into P segments that run as a varlen batch of N P sequences.
// Per token the forward map is S -> A S + b k^ v^T with A = (I - b k^ k^T) diag(a), and
// the cotangent map is dS -> A^T (dS + scale q^ do^T): A^T = diag(a) (I - b k^ k^T). So
// over a segment S_end = M S_start + N and dS_start = M^T dS_end + N', where M = A_last
// ... A_first, N' = sum_t w_t do_t^T and w_t = scale M_t^T q^_t (M_t = A_t ... A_first,
// the map up to token t) is the output of the run that gives M. M, N and w come from
// the two-pass tensor-core kernel's auxiliary passes (bf16, d = 128) or from a widened
// run of the recurrence (kda_chunk_rec.cu); `kda_seg_chain` walks them forwards to each
// segment's entering state and, with M^T and N', backwards to each segment's leaving
// cotangent (and the initial-state gradient); the two sweeps then run over the
// segments. P fills about two waves of the reverse sweep at two CTAs per SM, with at
// least 64 tokens per segment on average; square heads only.
constexpr int kBwdMaxSeg = 16;
constexpr int kBwdSms = 148;

int bwd_seg_count(bool varlen, long long T, int N, int H, int Dk, int Dv) {
    if (Dk != Dv || (Dk != 32 && Dk != 64 && Dk != 128)) return 1;
    const long long ctas = (long long)N * H * (Dv / kDVC);
    if (ctas <= 0 || ctas * 2 > 4 * kBwdSms) return 1;
    const long long avg = varlen ? T / (N > 0 ? N : 1) : T;
    long long P = std::min<long long>(kBwdMaxSeg, 4 * kBwdSms / ctas);
    P = std::min<long long>(P, avg / 64);
    return P < 2 ? 1 : (int)P;
}

size_t chunk_2pass_base_bytes(const ChunkParams &q);
cudaError_t chunk_2pass_transitions(const ChunkParams &q, void *workspace, float *M, float *Nst, float *w,
                                    cudaStream_t st);
cudaError_t rec_widened_run(const ChunkParams &q, bool bf16, int D, cudaStream_t st);

namespace {

// MT[s] = M[s]^T (packed D x D) for the states at M + s pitch, rows ld floats apart; one
// 32 x 32 tile per CTA through shared memory.
template <int D>
__global__ void __launch_bounds__(256) kda_seg_transpose(const float *M, int ld, long long pitch, float *MT) {
    constexpr int TB = D / 32;
    __shared__ float tile[32][33];
    const long long b = blockIdx.x, s = b / (TB * TB);
    const int tr = (int)(b % (TB * TB)) / TB, tc = (int)(b % TB);
    const float *src = M + s * pitch;
    float *dst = MT + s * (long long)D * D;
    const int x = threadIdx.x & 31, y = threadIdx.x >> 5;
    for (int i = y; i < 32; i += 8) tile[i][x] = src[(long long)(32 * tr + i) * ld + 32 * tc + x];
    __syncthreads();
    for (int i = y; i < 32; i += 8) dst[(long long)(32 * tc + i) * D + 32 * tr + x] = tile[x][i];
}

__device__ __forceinline__ float4 load4_f32(const float *p) { return *reinterpret_cast<const float4 *>(p); }
__device__ __forceinline__ float4 load4_f32(const __nv_bfloat16 *p) {
    const uint2 u = *reinterpret_cast<const uint2 *>(p);
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
    return make_float4(a.x, a.y, b.x, b.y);
}

// N'[v H + h] = sum over the tokens t of segment v of w_t do_t^T, w_t = row t H + h of w
// (wstride floats apart), do_t = row t H + h of dout. One CTA per (segment, head, 32
// rows k of N'); tokens in tiles of 32 staged in shared memory; thread (kr, cc) = (warp,
// lane) sums rows 4 kr .. of its block and columns CC cc .. (CC = D / 32).
template <typename Tin, int D>
__global__ void __launch_bounds__(256) kda_seg_cot_offset(const float *w, int wstride, const Tin *dout,
                                                          const int32_t *cu_v, float *Nrev, int H) {
    constexpr int TT = 32, CC = D / 32;
    __shared__ __align__(16) float wsm[TT][36];
    __shared__ __align__(16) float dsm[TT][D + 4];
    const int v = blockIdx.x / H, h = blockIdx.x % H, kb = blockIdx.y;
    const int tid = threadIdx.x, kr = tid >> 5, cc = tid & 31;
    const long long bos = cu_v[v], eos = cu_v[v + 1];
    float acc[4][CC];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int j = 0; j < CC; ++j) acc[r][j] = 0.f;
    for (long long t0 = bos; t0 < eos; t0 += TT) {
        const int cnt = (int)min((long long)TT, eos - t0);
        __syncthreads();  // the previous tile is consumed
        for (int e = tid; e < TT * 8; e += 256) {
            const int i = e >> 3, q4 = (e & 7) * 4;
            *reinterpret_cast<float4 *>(&wsm[i][q4]) =
                i < cnt ? load4_f32(w + ((t0 + i) * H + h) * wstride + 32 * kb + q4) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        for (int e = tid; e < TT * (D / 4); e += 256) {
            const int i = e / (D / 4), c4 = (e % (D / 4)) * 4;
            *reinterpret_cast<float4 *>(&dsm[i][c4]) =
                i < cnt ? load4_f32(dout + ((t0 + i) * H + h) * D + c4) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        __syncthreads();
        for (int i = 0; i < cnt; ++i) {
            const float4 wk = *reinterpret_cast<const float4 *>(&wsm[i][4 * kr]);
            const float wv[4] = {wk.x, wk.y, wk.z, wk.w};
            float dc[CC];  // one vector load of the lane's CC consecutive columns (no bank conflicts)
            if constexpr (CC == 4) {
                const float4 x = *reinterpret_cast<const float4 *>(&dsm[i][4 * cc]);
                dc[0] = x.x; dc[1] = x.y; dc[2] = x.z; dc[3] = x.w;
            } else if constexpr (CC == 2) {
                const float2 x = *reinterpret_cast<const float2 *>(&dsm[i][2 * cc]);
                dc[0] = x.x; dc[1] = x.y;
            } else {
                dc[0] = dsm[i][cc];
            }
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int j = 0; j < CC; ++j) acc[r][j] = fmaf(wv[r], dc[j], acc[r][j]);
        }
    }
    float *dst = Nrev + ((long long)blockIdx.x * D + 32 * kb + 4 * kr) * D + CC * cc;
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int j = 0; j < CC; ++j) dst[(long long)r * D + j] = acc[r][j];
}

}  // namespace

// The segment view of a backward call as forward parameters (cu_v: the segment offsets).
ChunkParams bwd_seg_view(const BwdParams &b, int P, const int32_t *cu_v) {
    ChunkParams q{};
    q.q = b.q; q.k = b.k; q.v = b.v; q.g = b.g; q.beta = b.beta;
    q.cu_seqlens = cu_v;
    q.T = b.cu_seqlens ? b.T : b.N * b.T;
    q.N = b.N * P; q.H = b.H;
    q.scale = b.scale; q.use_l2 = b.use_l2; q.has_lb = b.has_lb; q.lb = b.lb;
    q.gate_mode = kGateLog; q.beta_prob = b.beta_prob;
    return q;
}

// Workspace: [cu_v][M, N (or [M | N] rows)][entering states][leaving cotangents]
// [M^T, N'][w rows][shared] where "shared" holds first the two-pass kernel's records
// (when it gives the maps), then the sweeps' own workspace.
struct BwdSegLayout {
    size_t cu, maps, states, w, shared, total;
};
BwdSegLayout bwd_seg_layout(bool varlen, long long T, int N, int H, int D, int P, bool tc) {
    auto r256 = [](size_t b) { return (b + 255) / 256 * 256; };
    const long long total = varlen ? T : (long long)N * T;
    const size_t nv = (size_t)N * P;
    BwdSegLayout L;
    L.cu = r256((nv + 1) * 4);
    L.maps = r256(nv * H * D * 2 * D * 4);
    L.states = r256(nv * H * D * D * 4);
    L.w = r256((size_t)total * H * D * (tc ? 1 : 2) * 4);
    L.shared = bwd_workspace_bytes_min(true, total, (int)nv, H, D, D);
    if (tc) {
        ChunkParams q{};
        q.cu_seqlens = reinterpret_cast<const int32_t *>(16);  // only its presence is read
        q.T = (int)total; q.N = (int)nv; q.H = H;
        L.shared = std::max(L.shared, chunk_2pass_base_bytes(q));
    }
    L.total = L.cu + L.maps + 4 * L.states + L.w + L.shared;
    return L;
}

cudaError_t launch_bwd_ws(BwdParams p, bool bf16, int Dk, int Dv, uint8_t *ws, cudaStream_t st) {
    p.ckpt_off = reinterpret_cast<int *>(ws);
    p.scratch = reinterpret_cast<float *>(ws + (((size_t)(p.N + 1) * 4 + 255) / 256) * 256);
    p.ckpt = p.scratch + 2 * (size_t)p.N * p.H * kCB * Dk * Dv;
    return bf16 ? launch_bwd_dt<__nv_bfloat16>(p, Dk, Dv, st) : launch_bwd_dt<float>(p, Dk, Dv, st);
}

template <int D>
cudaError_t bwd_segments(const BwdParams &p, bool bf16, int P, const BwdSegLayout &L, uint8_t *ws, bool tc,
                         cudaStream_t st) {
    uint8_t *cur = ws;
    int32_t *cu_v = reinterpret_cast<int32_t *>(cur); cur += L.cu;
    float *maps = reinterpret_cast<float *>(cur); cur += L.maps;
    float *S_start = reinterpret_cast<float *>(cur); cur += L.states;
    float *dS_end = reinterpret_cast<float *>(cur); cur += L.states;
    float *MT = reinterpret_cast<float *>(cur); cur += L.states;
    float *Nrev = reinterpret_cast<float *>(cur); cur += L.states;
    float *w = reinterpret_cast<float *>(cur); cur += L.w;
    uint8_t *shared = cur;
    const ChunkParams q = bwd_seg_view(p, P, cu_v);
    const long long nst = (long long)q.N * q.H;
    cudaError_t e;
    // segments of whole 64-token chunks for the two-pass kernel, of 16-token stretches otherwise
    count_launch();
    kda_seg_setup<<<(p.N + 255) / 256, 256, 0, st>>>(p.cu_seqlens, p.T, p.N, P, tc ? 64 : 16, cu_v);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    // the forward maps and w, then the entering states
    const float *M, *Nf;
    int ld, wstride;
    long long pitch;
    if (tc) {
        M = maps; Nf = maps + nst * D * D; ld = D; pitch = (long long)D * D; wstride = D;
        if ((e = chunk_2pass_transitions(q, shared, maps, maps + nst * D * D, w, st)) != cudaSuccess) return e;
    } else {
        M = maps; Nf = maps + D; ld = 2 * D; pitch = 2LL * D * D; wstride = 2 * D;
        ChunkParams r = q;
        r.S_out = maps;
        r.o = w;
        if ((e = rec_widened_run(r, bf16, D, st)) != cudaSuccess) return e;
    }
    if ((e = seg_chain_launch<D>(p.S0, M, Nf, ld, pitch, S_start, nullptr, p.N, p.H, P, st)) != cudaSuccess) return e;
    // the cotangent maps M^T and N', then the leaving cotangents and the initial-state gradient
    count_launch();
    kda_seg_transpose<D><<<(unsigned)(nst * (D / 32) * (D / 32)), 256, 0, st>>>(M, ld, pitch, MT);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    count_launch();
    if (bf16)
        kda_seg_cot_offset<__nv_bfloat16, D><<<dim3((unsigned)nst, D / 32), 256, 0, st>>>(
            w, wstride, static_cast<const __nv_bfloat16 *>(p.dout), cu_v, Nrev, p.H);
    else
        kda_seg_cot_offset<float, D><<<dim3((unsigned)nst, D / 32), 256, 0, st>>>(
            w, wstride, static_cast<const float *>(p.dout), cu_v, Nrev, p.H);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = seg_chain_launch<D>(p.dSf, MT, Nrev, D, (long long)D * D, dS_end, p.dS0, p.N, p.H, P, st, 1)) != cudaSuccess)
        return e;
    BwdParams b = p;  // the sweeps over the segments; dS0 came from the cotangent chain
    b.cu_seqlens = cu_v;
    b.T = q.T;
    b.N = q.N;
    b.S0 = S_start;
    b.dSf = dS_end;
    b.dS0 = nullptr;
    return launch_bwd_ws(b, bf16, D, D, shared, st);
}

size_t bwd_chunked_workspace_bytes(const BwdParams &p, bool bf16, int Dk, int Dv);
cudaError_t launch_bwd_chunked(const BwdParams &p, void *workspace, cudaStream_t st);
bool bwd_warp_supported(const BwdParams &p, bool bf16, int Dk, int Dv);
size_t bwd_warp_workspace_bytes(const BwdParams &p, int Dv);
cudaError_t launch_bwd_warp(const BwdParams &p, int Dv, void *workspace, cudaStream_t st);
size_t bwd_workspace_bytes(bool varlen, long long T, int N, int H, int Dk, int Dv);

// The workspace with which kda_chunk_bwd runs its fastest form: the chunked form
// (kda_bwd_chunk.cu, d = 128) or the micro-chunk form (kda_bwd_warp.cu, d_k = 32) where
// they apply, else the segments when they apply.
size_t bwd_workspace_bytes(const BwdParams &p, bool bf16, int Dk, int Dv) {
    const bool varlen = p.cu_seqlens != nullptr;
    const size_t chunked = bwd_chunked_workspace_bytes(p, bf16, Dk, Dv);
    if (chunked) return std::max(chunked, bwd_workspace_bytes_min(varlen, p.T, p.N, p.H, Dk, Dv));
    if (bwd_warp_supported(p, bf16, Dk, Dv))
        return std::max(bwd_warp_workspace_bytes(p, Dv), bwd_workspace_bytes_min(varlen, p.T, p.N, p.H, Dk, Dv));
    return bwd_workspace_bytes(varlen, p.T, p.N, p.H, Dk, Dv);
}

// The workspace of the token-recurrence form (the segments when they apply).
size_t bwd_workspace_bytes(bool varlen, long long T, int N, int H, int Dk, int Dv) {
    const size_t plain = bwd_workspace_bytes_min(varlen, T, N, H, Dk, Dv);
    const int P = bwd_seg_count(varlen, T, N, H, Dk, Dv);
    if (P < 2) return plain;
    // the larger of the two map sources, so that either dtype fits
    return std::max({plain, bwd_seg_layout(varlen, T, N, H, Dk, P, false).total,
                     Dk == 128 ? bwd_seg_layout(varlen, T, N, H, Dk, P, true).total : (size_t)0});
}

cudaError_t launch_bwd(BwdParams p, bool bf16, int Dk, int Dv, void *workspace, size_t workspace_bytes, cudaStream_t st) {
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    const bool varlen = p.cu_seqlens != nullptr;
    const size_t chunked = bwd_chunked_workspace_bytes(p, bf16, Dk, Dv);
    if (chunked && workspace_bytes >= chunked && (reinterpret_cast<uintptr_t>(ws) & 255) == 0)
        return launch_bwd_chunked(p, ws, st);
    if (bwd_warp_supported(p, bf16, Dk, Dv) && workspace_bytes >= bwd_warp_workspace_bytes(p, Dv) &&
        (reinterpret_cast<uintptr_t>(ws) & 255) == 0)
        return launch_bwd_warp(p, Dv, ws, st);
    const int P = bwd_seg_count(varlen, p.T, p.N, p.H, Dk, Dv);
    if (P >= 2 && (reinterpret_cast<uintptr_t>(ws) & 255) == 0) {
        const bool tc = bf16 && Dk == 128;
        const BwdSegLayout L = bwd_seg_layout(varlen, p.T, p.N, p.H, Dk, P, tc);
        if (workspace_bytes >= L.total) {
            if (Dk == 32) return bwd_segments<32>(p, bf16, P, L, ws, tc, st);
            if (Dk == 64) return bwd_segments<64>(p, bf16, P, L, ws, tc, st);
            return bwd_segments<128>(p, bf16, P, L, ws, tc, st);
        }
    }
    return launch_bwd_ws(p, bf16, Dk, Dv, ws, st);
}

}  // namespace kda
