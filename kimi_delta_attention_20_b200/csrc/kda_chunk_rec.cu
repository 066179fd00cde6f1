// Chunk forward for the shapes the tensor-core path does not take (fp32 inputs,
// d_k or d_v other than 128): the token recurrence of page
// "atlas_core/kimi_k3/kda.rs" run directly, with the fp32 state in registers.
//
// Per token, with k^, q^ the normalised rows, a = exp(g) (g clamped, or formed
// in the kernel from A_log and dt_bias) and b the write strength:
//   S' = diag(a) S,  u = S'^T k^,  S = S' + k^ (b (v - u))^T,  o = scale S^T q^.
// The result is that of `chunk_kda` (page "K3/kda/ops/api.py") for any chunk
// size: regrouping the recurrence by chunks changes the order of the
// arithmetic, not its value. For small head dims the recurrence also takes
// fewer operations than the chunked form (no C x C blocks, no inverse).
//
// One CTA per (sequence, head). A warp holds WC value columns of the state over all
// d_k rows: lane (rg, cg) = (lane / CGN, lane % CGN) keeps the RP = 16 key rows
// rg*RP .. rg*RP+15 of columns CG cg .. CG cg + CG - 1 of its warp's block in registers,
// as column pairs for the paired fp32 FMA pipe. For d_k <= 64 the warp has d_k / 16
// row groups and CG = 2, so the key-axis sums u and o are a butterfly of one or two
// shuffle levels that leaves every lane with the totals of its own columns; for
// d_k = 128 there are 8 row groups and CG = 4, and the sums are a reduce-scatter
// followed by a gather for u. Nothing else crosses lanes, and no barrier is taken
// per token. Tokens arrive in stretches of CT: the raw rows of the next
// stretch are copied by cp.async while the current one runs, turned into fp32
// (L2 norms, gate, sigmoid) once per stretch, and the stretch's outputs leave
// from shared memory as whole rows.
#include <algorithm>

#include <type_traits>

#include "kda_common.cuh"
#include "kda_stage.cuh"
#include "kda_seg.cuh"
#include "kda_tc_util.cuh"

namespace kda {

namespace {

template <int DK, int DV>
struct RecCfg {
    // 16 key rows per lane. Small key dims take the butterfly layout (d_k / 16 row groups,
    // 2 value columns per lane); d_k = 128 keeps 8 row groups of 4 value columns, where
    // a butterfly would need three levels and twice the warps' columns.
    static constexpr bool BFLY = DK <= 64;
    static constexpr int RGN = BFLY ? DK / 16 : 8;  // row groups per warp
    static constexpr int CGN = 32 / RGN;            // column groups per warp (lanes per row group)
    static constexpr int CG = BFLY ? 2 : 4;         // value columns per lane
    static constexpr int WC = CGN * CG;             // value columns per warp
    static constexpr int NW = DV / WC, NT = NW * 32;
    static constexpr int RP = DK / RGN;             // rows per lane
    static constexpr int CT = DK >= 128 ? 16 : 32;  // tokens per stretch
    static constexpr int TPR = 8, E = DK / TPR;     // intake: threads per key row, elements each
    static_assert(NW >= 1 && NW * WC == DV && RP == 16 && NT >= CT, "recurrent tiling");
};

template <typename Tin, int DK, int DV>
struct RecSmem {
    static constexpr int CT = RecCfg<DK, DV>::CT;
    Tin rk[CT][DK], rq[CT][DK], rg[CT][DK], rv[CT][DV];  // raw rows, copied in by cp.async
    float kh[CT][DK], qh[CT][DK], al[CT][DK];           // k^, q^, a = exp(g)
    float vo[CT][DV];  // v of token i, then its output: a warp reads v[i] of its own columns
                       // before its shuffles and writes o[i] of the same columns after them
    float b[CT];
    float dtb[DK];                                       // dt_bias of the head (in-kernel gate)
};

// Start the copy of tokens [t0, t0 + cnt) of head h; returns this thread's raw
// beta (thread i < cnt holds token i's), left unconverted so that the load
// completes in the background.
// (The CTA holds state columns c0 .. c0 + CB - 1 of DV.)
template <typename Tin, int DK, int DV, bool AUG, int CB>
__device__ __forceinline__ Tin rec_issue(const ChunkParams &p, RecSmem<Tin, DK, CB> &sm, long long t0, int cnt, int h,
                                         int c0) {
    constexpr int NT = RecCfg<DK, CB>::NT, EP = 16 / (int)sizeof(Tin);
    constexpr int VOFF = AUG ? DK : 0, DVR = DV - VOFF;  // augmented: v occupies columns DK .. DV - 1
    constexpr int RK = DK / EP;
    const int tid = threadIdx.x, H = p.H;
    for (int e = tid; e < cnt * RK; e += NT) {
        const int i = e / RK, c = (e % RK) * EP;
        const long long gi = ((t0 + i) * H + h) * DK + c;
        cp_async16(&sm.rk[i][c], static_cast<const Tin *>(p.k) + gi);
        cp_async16(&sm.rq[i][c], static_cast<const Tin *>(p.q) + gi);
        cp_async16(&sm.rg[i][c], static_cast<const Tin *>(p.g) + gi);
    }
    // the CTA's columns that see v: local vlo .. CB - 1 (none for a block of M columns)
    const int vlo = max(c0, VOFF) - c0, rv = (CB - vlo) / EP;
    for (int e = tid; e < cnt * rv; e += NT) {
        const int i = e / rv, c = (e % rv) * EP;
        cp_async16(&sm.rv[i][vlo + c], static_cast<const Tin *>(p.v) + ((t0 + i) * H + h) * DVR + (c0 + vlo - VOFF) + c);
    }
    cp_async_commit();
    return tid < cnt ? static_cast<const Tin *>(p.beta)[(t0 + tid) * H + h] : Tin(0.f);
}

// The staged stretch as fp32 token vectors. Each key row is taken by TPR
// threads that form its squared norms with shuffles (uniform trip count: rows
// past cnt read row 0 and store nothing). Barriers on both sides.
template <typename Tin, int DK, bool AUG, int CB>
__device__ void rec_take(const ChunkParams &p, RecSmem<Tin, DK, CB> &sm, int cnt, Tin beta_raw, float rate, int c0) {
    using Cfg = RecCfg<DK, CB>;
    constexpr int NT = Cfg::NT, TPR = Cfg::TPR, E = Cfg::E;
    const int tid = threadIdx.x;
    cp_async_wait_all();
    __syncthreads();
    const int c = (tid % TPR) * E;
    for (int i0 = 0; i0 < cnt; i0 += NT / TPR) {
        const int i = i0 + tid / TPR;
        const bool live = i < cnt;
        const int ir = live ? i : 0;
        float kx[E], qx[E], gx[E];
        stage_cvt<E>(&sm.rk[ir][c], kx);
        stage_cvt<E>(&sm.rq[ir][c], qx);
        stage_cvt<E>(&sm.rg[ir][c], gx);
        float kk = 0.f, qq = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) { kk = fmaf(kx[e], kx[e], kk); qq = fmaf(qx[e], qx[e], qq); }
#pragma unroll
        for (int o = TPR / 2; o > 0; o >>= 1) {
            kk += __shfl_xor_sync(0xffffffffu, kk, o);
            qq += __shfl_xor_sync(0xffffffffu, qq, o);
        }
        const float rk = p.use_l2 ? rsqrtf(kk + kL2Eps) : 1.f, rq = p.use_l2 ? rsqrtf(qq + kL2Eps) : 1.f;
#pragma unroll
        for (int e = 0; e < E; ++e) {
            kx[e] *= rk;
            qx[e] *= rq;
            if constexpr (std::is_same<Tin, __nv_bfloat16>::value) {
                // bf16 inputs: the gate and the decay on the special-function unit (the
                // forms of the tensor-core path; their error is far below bf16 rounding)
                constexpr float kL2e = 1.4426950408889634f;
                const float gv = p.gate_mode == kGateLog ? (p.has_lb ? fmaxf(gx[e], p.lb) : gx[e])
                                                         : tcu::gate_fast(gx[e], sm.dtb[c + e], rate, p.gate_mode, p.lb);
                gx[e] = tcu::ex2a(gv * kL2e);
            } else {
                gx[e] = expf(gate_value(gx[e], sm.dtb[c + e], rate, p.gate_mode, p.has_lb, p.lb));
            }
        }
        if (live) {
            store_vec<E>(&sm.kh[i][c], kx);
            store_vec<E>(&sm.qh[i][c], qx);
            store_vec<E>(&sm.al[i][c], gx);
        }
    }
    for (int e = tid; e < cnt * CB; e += NT) {
        const int i = e / CB, cc = e % CB;
        sm.vo[i][cc] = (AUG && c0 + cc < DK) ? 0.f : to_f32(sm.rv[i][cc]);
    }
    if (tid < cnt) sm.b[tid] = beta_value(to_f32(beta_raw), p.beta_prob);
    __syncthreads();
}

template <int RP>
__device__ __forceinline__ void rows_in(const float *src, float (&out)[RP]) {
#pragma unroll
    for (int j = 0; j < RP; j += 4) {
        const float4 x = *reinterpret_cast<const float4 *>(src + j);
        out[j] = x.x; out[j + 1] = x.y; out[j + 2] = x.z; out[j + 3] = x.w;
    }
}

// Sum of CG values over the 8 row groups of a warp (lane bits 4, 3, 2) by
// reduce-scatter: at lane bit 16, 8, ... each lane keeps the upper or lower half of
// its values and adds the partner's copy of that half. Returns the total of value
// v = lane / (32 / CG) of this lane's column group (for CG = 4, bit 2 is a plain
// butterfly and lanes with bit 2 = 0 and 1 hold the same).
template <int CG>
__device__ __forceinline__ float rowgroup_scatter(const float (&x)[CG]) {
    const int lane = threadIdx.x & 31;
    float a[CG];
#pragma unroll
    for (int j = 0; j < CG; ++j) a[j] = x[j];
#pragma unroll
    for (int n = CG, bit = 16; n > 1; n >>= 1, bit >>= 1) {
        const bool hi = lane & bit;
#pragma unroll
        for (int j = 0; j < n / 2; ++j) {
            const float keep = hi ? a[n / 2 + j] : a[j], send = hi ? a[j] : a[n / 2 + j];
            a[j] = keep + __shfl_xor_sync(0xffffffffu, send, bit);
        }
    }
    if constexpr (CG == 4) a[0] += __shfl_xor_sync(0xffffffffu, a[0], 4);
    return a[0];
}

// AUG: the augmented run of the segment form. Its state is [M | N] (d_k x (d_k + d_v)):
// the first d_k columns start from the identity and see v = 0, the others start from
// zero and see v; the outputs [scale M^T q^ | scale N^T q^] go out in fp32, rows of
// d_k + d_v, and the final state as [d_k][d_k + d_v].
// CB: state columns per CTA; the DV / CB CTAs of one (sequence, head) (blockIdx.y) need
// nothing from one another, since the columns of S evolve independently.
template <typename Tin, int DK, int DV, bool AUG, int CB = DV>
__global__ void __launch_bounds__(RecCfg<DK, CB>::NT) kda_chunk_rec_kernel(ChunkParams p) {
    using Cfg = RecCfg<DK, CB>;
    constexpr int RP = Cfg::RP, CT = Cfg::CT, NT = Cfg::NT, CG = Cfg::CG, CP = CG / 2, CGN = Cfg::CGN;
    constexpr bool BFLY = Cfg::BFLY;
    constexpr int NACC = BFLY ? 4 : 2;  // independent accumulation chains per column pair
    constexpr int VS = 32 / CG;  // lanes between the holders of consecutive reduced values (reduce-scatter)
    extern __shared__ __align__(16) uint8_t smraw[];
    RecSmem<Tin, DK, CB> &sm = *reinterpret_cast<RecSmem<Tin, DK, CB> *>(smraw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int rg = lane / CGN, cg = lane % CGN;
    const int c0 = blockIdx.y * CB;            // the CTA's first state column
    const int col = Cfg::WC * warp + CG * cg;  // this lane's first value column within the CTA's
    const int gcol = c0 + col;
    const long long nh = blockIdx.x;
    const int n = (int)(nh / p.H), h = (int)(nh % p.H), H = p.H;
    long long bos, eos;
    if (p.cu_seqlens) { bos = p.cu_seqlens[n]; eos = p.cu_seqlens[n + 1]; }
    else { bos = (long long)n * p.T; eos = bos + p.T; }

    const float rate = p.gate_mode != kGateLog ? expf(p.A_log[h]) : 0.f;
    for (int c = tid; c < DK; c += NT)
        sm.dtb[c] = (p.gate_mode != kGateLog && p.dt_bias) ? p.dt_bias[(long long)h * DK + c] : 0.f;

    // the state as column pairs (col + 2 j, col + 2 j + 1), for the paired fp32 FMA pipe
    float2 s[RP][CP];
#pragma unroll
    for (int r = 0; r < RP; ++r) {
        const int row = rg * RP + r;
        if constexpr (CP == 1) {
            s[r][0] = AUG ? make_float2(row == gcol, row == gcol + 1)
                    : p.S0 ? *reinterpret_cast<const float2 *>(p.S0 + (nh * DK + row) * DV + gcol)
                           : make_float2(0.f, 0.f);
        } else {
#pragma unroll
            for (int j = 0; j < CP; j += 2) {
                const int cj = gcol + 2 * j;
                const float4 x = AUG ? make_float4(row == cj, row == cj + 1, row == cj + 2, row == cj + 3)
                                 : p.S0 ? *reinterpret_cast<const float4 *>(p.S0 + (nh * DK + row) * DV + cj)
                                        : make_float4(0.f, 0.f, 0.f, 0.f);
                s[r][j] = make_float2(x.x, x.y);
                s[r][j + 1] = make_float2(x.z, x.w);
            }
        }
    }

    long long t0 = bos;  // stretches of CT tokens
    int cnt = (int)min((long long)CT, eos - bos);
    Tin braw = cnt > 0 ? rec_issue<Tin, DK, DV, AUG, CB>(p, sm, t0, cnt, h, c0) : Tin(0.f);
    while (cnt > 0) {
        rec_take<Tin, DK, AUG, CB>(p, sm, cnt, braw, rate, c0);
        const long long t0n = t0 + CT;
        const int cntn = (int)max(0LL, min((long long)CT, eos - t0n));
        if (cntn > 0) braw = rec_issue<Tin, DK, DV, AUG, CB>(p, sm, t0n, cntn, h, c0);
#pragma unroll 2
        for (int i = 0; i < cnt; ++i) {
            float kr[RP], ar[RP], qr[RP];
            rows_in<RP>(&sm.kh[i][rg * RP], kr);
            rows_in<RP>(&sm.al[i][rg * RP], ar);
            rows_in<RP>(&sm.qh[i][rg * RP], qr);
            const float b = sm.b[i];
            float2 vv[CP];
            if constexpr (CP == 1) {
                vv[0] = *reinterpret_cast<const float2 *>(&sm.vo[i][col]);
            } else {
#pragma unroll
                for (int j = 0; j < CP; j += 2) {
                    const float4 x = *reinterpret_cast<const float4 *>(&sm.vo[i][col + 2 * j]);
                    vv[j] = make_float2(x.x, x.y);
                    vv[j + 1] = make_float2(x.z, x.w);
                }
            }
            // S' = diag(a) S and this lane's part of u = S'^T k^ (NACC chains per pair)
            const float2 z2 = make_float2(0.f, 0.f);
            float2 acc[NACC][CP];
#pragma unroll
            for (int a = 0; a < NACC; ++a)
#pragma unroll
                for (int j = 0; j < CP; ++j) acc[a][j] = z2;
#pragma unroll
            for (int r = 0; r < RP; ++r) {
                const float2 a2 = make_float2(ar[r], ar[r]), k2 = make_float2(kr[r], kr[r]);
#pragma unroll
                for (int j = 0; j < CP; ++j) {
                    s[r][j] = __fmul2_rn(s[r][j], a2);
                    acc[r % NACC][j] = __ffma2_rn(s[r][j], k2, acc[r % NACC][j]);
                }
            }
            float2 d[CP];
            const float2 b2 = make_float2(b, b);
            if constexpr (BFLY) {
                // u of the lane's two columns: its chains, then the other row groups
                float2 u = __fadd2_rn(acc[0][0], acc[1][0]);
#pragma unroll
                for (int a = 2; a < NACC; ++a) u = __fadd2_rn(u, acc[a][0]);
#pragma unroll
                for (int bit = 16; bit >= CGN; bit >>= 1)
                    u = __fadd2_rn(u, make_float2(__shfl_xor_sync(0xffffffffu, u.x, bit),
                                                  __shfl_xor_sync(0xffffffffu, u.y, bit)));
                d[0] = __fmul2_rn(b2, __fadd2_rn(vv[0], make_float2(-u.x, -u.y)));
            } else {
                float part[CG];
#pragma unroll
                for (int j = 0; j < CP; ++j) {
                    const float2 t = __fadd2_rn(acc[0][j], acc[1][j]);
                    part[2 * j] = t.x; part[2 * j + 1] = t.y;
                }
                const float m = rowgroup_scatter<CG>(part);
                // gather u of the lane's columns from the lanes that hold them
#pragma unroll
                for (int j = 0; j < CP; ++j) {
                    const float2 u = make_float2(__shfl_sync(0xffffffffu, m, (2 * j) * VS + cg),
                                                 __shfl_sync(0xffffffffu, m, (2 * j + 1) * VS + cg));
                    d[j] = __fmul2_rn(b2, __fadd2_rn(vv[j], make_float2(-u.x, -u.y)));
                }
            }
            // S = S' + k^ d^T and this lane's part of S^T q^
#pragma unroll
            for (int a = 0; a < NACC; ++a)
#pragma unroll
                for (int j = 0; j < CP; ++j) acc[a][j] = z2;
#pragma unroll
            for (int r = 0; r < RP; ++r) {
                const float2 k2 = make_float2(kr[r], kr[r]), q2 = make_float2(qr[r], qr[r]);
#pragma unroll
                for (int j = 0; j < CP; ++j) {
                    s[r][j] = __ffma2_rn(k2, d[j], s[r][j]);
                    acc[r % NACC][j] = __ffma2_rn(s[r][j], q2, acc[r % NACC][j]);
                }
            }
            if constexpr (BFLY) {
                float2 ov = __fadd2_rn(acc[0][0], acc[1][0]);
#pragma unroll
                for (int a = 2; a < NACC; ++a) ov = __fadd2_rn(ov, acc[a][0]);
#pragma unroll
                for (int bit = 16; bit >= CGN; bit >>= 1)
                    ov = __fadd2_rn(ov, make_float2(__shfl_xor_sync(0xffffffffu, ov.x, bit),
                                                    __shfl_xor_sync(0xffffffffu, ov.y, bit)));
                if (rg == 0) *reinterpret_cast<float2 *>(&sm.vo[i][col]) = make_float2(p.scale * ov.x, p.scale * ov.y);
            } else {
                float part[CG];
#pragma unroll
                for (int j = 0; j < CP; ++j) {
                    const float2 t = __fadd2_rn(acc[0][j], acc[1][j]);
                    part[2 * j] = t.x; part[2 * j + 1] = t.y;
                }
                const float ov = rowgroup_scatter<CG>(part);
                if (CG == 8 || (lane & 4) == 0) sm.vo[i][col + lane / VS] = p.scale * ov;
            }
        }
        if (p.o) {
            // the stretch's output rows, from shared memory
            __syncthreads();
            for (int e = 4 * tid; e < cnt * CB; e += 4 * NT) {
                const int i = e / CB, c = e % CB;
                const float4 x = *reinterpret_cast<const float4 *>(&sm.vo[i][c]);
                if constexpr (AUG) {
                    *reinterpret_cast<float4 *>(static_cast<float *>(p.o) + ((t0 + i) * H + h) * DV + c0 + c) = x;
                } else {
                    Tin *dst = static_cast<Tin *>(p.o) + ((t0 + i) * H + h) * DV + c0 + c;
                    dst[0] = from_f32<Tin>(x.x); dst[1] = from_f32<Tin>(x.y);
                    dst[2] = from_f32<Tin>(x.z); dst[3] = from_f32<Tin>(x.w);
                }
            }
    
        }
        t0 = t0n;
        cnt = cntn;
    }
    if (p.S_out) {
#pragma unroll
        for (int r = 0; r < RP; ++r) {
            float *dst = p.S_out + (nh * DK + rg * RP + r) * DV + gcol;
            if constexpr (CP == 1) {
                *reinterpret_cast<float2 *>(dst) = s[r][0];
            } else {
#pragma unroll
                for (int j = 0; j < CP; j += 2)
                    *reinterpret_cast<float4 *>(dst + 2 * j) = make_float4(s[r][j].x, s[r][j].y, s[r][j + 1].x, s[r][j + 1].y);
            }
        }
    }
}

template <typename Tin, int DK, int DV, bool AUG = false, int CB = DV>
cudaError_t launch_rec_t(const ChunkParams &p, cudaStream_t st) {
    static_assert(DV % CB == 0 && (!AUG || DK % CB == 0 || CB == DV), "a column block lies inside the M or the N block, or holds both");
    const long long blocks = (long long)p.N * p.H;
    if (blocks == 0) return cudaSuccess;
    const int smem = (int)sizeof(RecSmem<Tin, DK, CB>);
    auto kern = kda_chunk_rec_kernel<Tin, DK, DV, AUG, CB>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    count_launch();
    kern<<<dim3((unsigned)blocks, DV / CB), RecCfg<DK, CB>::NT, smem, st>>>(p);
    return cudaGetLastError();
}

template <typename Tin>
cudaError_t launch_rec_dt(const ChunkParams &p, int Dk, int Dv, cudaStream_t st) {
#define KDA_REC_CASE(DK_, DV_) \
    if (Dk == DK_ && Dv == DV_) return launch_rec_t<Tin, DK_, DV_>(p, st);
    KDA_REC_CASE(32, 32) KDA_REC_CASE(32, 64) KDA_REC_CASE(32, 128)
    KDA_REC_CASE(64, 32) KDA_REC_CASE(64, 64) KDA_REC_CASE(64, 128)
    KDA_REC_CASE(128, 32) KDA_REC_CASE(128, 64) KDA_REC_CASE(128, 128)
#undef KDA_REC_CASE
    return cudaErrorInvalidValue;
}

// ---- segments (kda_seg.cuh): with few (sequence, head) chains and square states, each
// sequence is cut into P segments. One augmented launch runs every segment with the
// state [M | N] (columns of S evolve independently, so the transition M, from the
// identity with v = 0, and the offset N, from zero with v, are extra columns of one
// state); it also writes w_t = scale M_t^T q^_t and scale N_t^T q^_t per token, M_t, N_t
// being the maps up to token t within the segment. `kda_seg_chain` then walks the
// segments to their entering states S_s, and since S_t = M_t S_s + N_t the outputs are
// o_t = S_s^T w_t + scale N_t^T q^_t, a product per token with no sequential dependence.
constexpr int kRecMaxSeg = 16;
constexpr int kRecChains = 8 * 148;  // chains wanted in flight: several small CTAs per SM

int rec_seg_count(const ChunkParams &p, int Dk, int Dv, bool bf16) {
    if (Dk != Dv || (Dk != 32 && Dk != 64)) return 1;
    const long long chains = (long long)p.N * p.H;
    if (chains <= 0 || chains * 2 > kRecChains) return 1;
    // bf16 d = 64: from 128 chains on, the micro-chunk form (kda_chunk_warp.cu) beats the
    // segments, whose widened run is the recurrence at twice the width (B T2048 H8:
    // 128 chains 0.41 against 0.64 ms, 512 chains 0.52 against 2.13 ms; 64 chains 0.37
    // against 0.34 ms)
    if (bf16 && Dk == 64 && chains >= 128) return 1;
    const long long avg = p.cu_seqlens ? (long long)p.T / (p.N > 0 ? p.N : 1) : (long long)p.T;
    long long P = std::min<long long>(kRecMaxSeg, kRecChains / chains);
    P = std::min<long long>(P, avg / 64);  // at least 64 tokens per segment on average
    if (P < 2) return 1;
    const long long seg_max = (((long long)p.T + P - 1) / P + 15) / 16 * 16;
    return (seg_max + 31) / 32 > 65535 ? 1 : (int)P;  // the fixup grid's second dimension (32-token tiles)
}

size_t rk1(size_t b) { return (b + 1023) / 1024 * 1024; }

// Tiles of kFixTok tokens in the longest segment: ceil(len / P) rounded up to 16 tokens,
// len <= T (T is the tokens of a batch row, or the total of a varlen call)
constexpr int kFixTok = 32;
long long rec_fix_tiles(const ChunkParams &p, int P) {
    const long long seg_max = (((long long)p.T + P - 1) / P + 15) / 16 * 16;
    return (seg_max + kFixTok - 1) / kFixTok;
}

struct RecSegLayout {
    size_t cu, oaug, saug, sstart, total;
};
RecSegLayout rec_seg_layout(const ChunkParams &p, int P, int D) {
    const long long total = p.cu_seqlens ? (long long)p.T : (long long)p.N * p.T;
    const size_t states = (size_t)p.N * P * p.H;
    RecSegLayout L;
    L.cu = rk1((states / p.H + 1) * 4);
    L.oaug = rk1((size_t)total * p.H * 2 * D * 4);
    L.saug = rk1(states * D * 2 * D * 4);
    L.sstart = rk1(states * D * D * 4);
    L.total = L.cu + L.oaug + L.saug + L.sstart;
    return L;
}

__device__ __forceinline__ void store_o4(float *dst, float4 x) { *reinterpret_cast<float4 *>(dst) = x; }
__device__ __forceinline__ void store_o4(__nv_bfloat16 *dst, float4 x) {
    __nv_bfloat162 a = __floats2bfloat162_rn(x.x, x.y), b = __floats2bfloat162_rn(x.z, x.w);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t *>(&a);
    u.y = *reinterpret_cast<uint32_t *>(&b);
    *reinterpret_cast<uint2 *>(dst) = u;
}

// One CTA of 128 threads per (segment, head, 32-token tile): o_t = S_s^T w_t +
// (scale N_t^T q^_t) for the tile's tokens, from the augmented outputs (rows
// [w_t | scale N_t^T q^_t], fp32) and the entering state S_s (packed D x D). S_s and the
// tile's w rows are copied into shared memory by cp.async while each thread loads its
// offset terms; thread t then takes tokens t / (D / 4) + (128 / (D / 4)) i and 4 output
// columns. Tiles past the segment's end exit at once (the grid covers the longest
// segment any sequence can have).
template <typename To, int D>
__global__ void __launch_bounds__(128) kda_rec_seg_fixup(const float *oaug, const float *S_start, const int32_t *cu_v,
                                                         To *o, int H) {
    constexpr int NT = 128, Q = D / 4, TT = kFixTok, TPP = NT / Q, NTOK = TT / TPP, LW = D + 4;
    __shared__ __align__(16) float S[D][D];
    __shared__ __align__(16) float w[TT][LW];
    const int v = blockIdx.x / H, h = blockIdx.x % H, tid = threadIdx.x;
    const long long eos = cu_v[v + 1], t0 = cu_v[v] + (long long)blockIdx.y * TT;
    if (t0 >= eos) return;
    const int cnt = (int)min((long long)TT, eos - t0);
    const float *Ss = S_start + (long long)blockIdx.x * D * D;  // state index v H + h
    for (int e = tid; e < D * Q; e += NT) cp_async16(&S[e / Q][(e % Q) * 4], Ss + (long long)e * 4);
    for (int e = tid; e < cnt * Q; e += NT) {
        const int i = e / Q, k4 = (e % Q) * 4;
        cp_async16(&w[i][k4], oaug + ((t0 + i) * H + h) * (2 * D) + k4);
    }
    cp_async_commit();
    const int tb = tid / Q, c = (tid % Q) * 4;
    float4 acc[NTOK];
#pragma unroll
    for (int i = 0; i < NTOK; ++i) {
        const int ti = tb + TPP * i;
        acc[i] = ti < cnt ? *reinterpret_cast<const float4 *>(oaug + ((t0 + ti) * H + h) * (2 * D) + D + c)
                          : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    cp_async_wait_all();
    __syncthreads();
#pragma unroll 2
    for (int k = 0; k < D; k += 4) {
        float4 sv[4];
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) sv[kk] = *reinterpret_cast<const float4 *>(&S[k + kk][c]);
#pragma unroll
        for (int i = 0; i < NTOK; ++i) {
            const float4 wv = *reinterpret_cast<const float4 *>(&w[tb + TPP * i][k]);
            const float wk[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                acc[i].x = fmaf(wk[kk], sv[kk].x, acc[i].x);
                acc[i].y = fmaf(wk[kk], sv[kk].y, acc[i].y);
                acc[i].z = fmaf(wk[kk], sv[kk].z, acc[i].z);
                acc[i].w = fmaf(wk[kk], sv[kk].w, acc[i].w);
            }
        }
    }
#pragma unroll
    for (int i = 0; i < NTOK; ++i) {
        const int ti = tb + TPP * i;
        if (ti < cnt) store_o4(o + ((t0 + ti) * H + h) * D + c, acc[i]);
    }
}

}  // namespace
cudaError_t launch_chunk_warp_widened(const ChunkParams &q, cudaStream_t st);
namespace {

template <typename Tin, int D>
cudaError_t launch_rec_seg(const ChunkParams &p, int P, uint8_t *ws, cudaStream_t st) {
    const RecSegLayout L = rec_seg_layout(p, P, D);
    int32_t *cu_v = reinterpret_cast<int32_t *>(ws);
    float *oaug = reinterpret_cast<float *>(ws + L.cu);
    float *saug = reinterpret_cast<float *>(ws + L.cu + L.oaug);
    float *sstart = reinterpret_cast<float *>(ws + L.cu + L.oaug + L.saug);
    ChunkParams q = p;  // the segment view: P segments per sequence as a varlen batch
    q.T = p.cu_seqlens ? p.T : p.N * p.T;
    q.N = p.N * P;
    q.cu_seqlens = cu_v;
    q.S0 = nullptr;
    q.S_out = saug;
    q.o = oaug;
    cudaError_t e;
    count_launch();
    kda_seg_setup<<<(p.N + 255) / 256, 256, 0, st>>>(p.cu_seqlens, p.T, p.N, P, 16, cu_v);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if constexpr (std::is_same<Tin, __nv_bfloat16>::value && D == 32)  // the widened run on tensor cores
        e = launch_chunk_warp_widened(q, st);
    else
        e = launch_rec_t<Tin, D, 2 * D, true>(q, st);
    if (e != cudaSuccess) return e;
    if ((e = seg_chain_launch<D>(p.S0, saug, saug + D, 2 * D, 2LL * D * D, sstart, p.S_out, p.N, p.H, P, st)) !=
        cudaSuccess)
        return e;
    const dim3 fgrid((unsigned)((long long)q.N * p.H), (unsigned)rec_fix_tiles(p, P));
    count_launch();
    kda_rec_seg_fixup<Tin, D><<<fgrid, 128, 0, st>>>(oaug, sstart, cu_v, static_cast<Tin *>(p.o), p.H);
    return cudaGetLastError();
}

template <typename Tin>
cudaError_t launch_rec_seg_dt(const ChunkParams &p, int P, int D, uint8_t *ws, cudaStream_t st) {
    if (D == 32) return launch_rec_seg<Tin, 32>(p, P, ws, st);
    if (D == 64) return launch_rec_seg<Tin, 64>(p, P, ws, st);
    return cudaErrorInvalidValue;
}

}  // namespace

// One widened run over a segment view q (kda_bwd.cu's segment form): final states
// [M | N] to q.S_out as [d][2d] and, when q.o is given, the fp32 outputs
// [scale M_t^T q^_t | scale N_t^T q^_t] as rows of 2d.
cudaError_t rec_widened_run(const ChunkParams &q, bool bf16, int D, cudaStream_t st) {
#define KDA_WIDE(D_) \
    if (D == D_) return bf16 ? launch_rec_t<__nv_bfloat16, D_, 2 * D_, true>(q, st) : launch_rec_t<float, D_, 2 * D_, true>(q, st);
    KDA_WIDE(32) KDA_WIDE(64) KDA_WIDE(128)
#undef KDA_WIDE
    return cudaErrorInvalidValue;
}

// Workspace the recurrent forward can use (0: it needs none).
size_t chunk_rec_workspace_bytes(const ChunkParams &p, bool bf16, int Dk, int Dv) {
    const int P = rec_seg_count(p, Dk, Dv, bf16);
    return P < 2 ? 0 : rec_seg_layout(p, P, Dk).total;
}

bool chunk_warp_supported(bool bf16, int Dk, int Dv);
cudaError_t launch_chunk_warp(const ChunkParams &p, int Dk, int Dv, cudaStream_t st);

// Few chains of long sequences: the segment form of the recurrence; otherwise, for bf16
// with d_k 32 or 64 and d_v 32 or 64, the tensor-core micro-chunk form (kda_chunk_warp.cu);
// otherwise the recurrence.
cudaError_t launch_chunk_rec(const ChunkParams &p, bool bf16, int Dk, int Dv, void *workspace, size_t workspace_bytes,
                             cudaStream_t st) {
    const int P = rec_seg_count(p, Dk, Dv, bf16);
    if (P >= 2 && workspace && (reinterpret_cast<uintptr_t>(workspace) & 255) == 0 &&
        workspace_bytes >= rec_seg_layout(p, P, Dk).total) {
        uint8_t *ws = static_cast<uint8_t *>(workspace);
        return bf16 ? launch_rec_seg_dt<__nv_bfloat16>(p, P, Dk, ws, st) : launch_rec_seg_dt<float>(p, P, Dk, ws, st);
    }
    if (P < 2 && chunk_warp_supported(bf16, Dk, Dv)) return launch_chunk_warp(p, Dk, Dv, st);
    return bf16 ? launch_rec_dt<__nv_bfloat16>(p, Dk, Dv, st) : launch_rec_dt<float>(p, Dk, Dv, st);
}

}  // namespace kda
