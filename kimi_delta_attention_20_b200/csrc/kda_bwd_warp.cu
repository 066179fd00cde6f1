// Backward of the chunkwise forward for bf16 inputs with d_k = 32 (d_v 32 or 64) and a
// gate lower bound >= -10, in the micro-chunk form of the forward (kda_chunk_warp.cu):
// one warp per (sequence, head) walks its 16-token micro-chunks from the last, with
// the state cotangent dS (32 x d_v, fp32) in its accumulator registers.
//
// The pages give no backward formulas; these are the derivatives of the chunk form of
// `chunk_kda` (page "K3/kda/ops/api.py"; the result is the token recurrence of page
// "atlas_core/kimi_k3/kda.rs"), the same as in kda_bwd_chunk.cu with 16-token chunks:
// per micro-chunk, with the forward's S (the entering state, saved by the forward as a
// bf16 tile), T' = (I + diag(b) A_kk)^-1 diag(b), W = T' Ktil, D = T'V - W S and dO' =
// scale dO:
//   dD = A_qk^T dO' + Khat dS_C,   dS <- diag(gamma) dS_C + Qtil^T dO' - W^T dD,
//   dQtil = dO' S^T, dW = -dD S^T, dKhat = D dS_C^T, dA_qk = dO' D^T (its diagonal apart),
//   dT' = dD V^T + dW Ktil^T, dV = T'^T dD, dKtil = T'^T dW,
//   db_s = sum_r dT'_rs T_rs, dM = -T^T (dT' diag(b)) T^T, dA_kk = diag(b) dM (s < r),
//   db_r += sum_{s<r} dM_rs A_rs,
// the gated products split at the middle row (factors e^{+-(G - G_7)}, within e^80 for a
// lower bound >= -10), the elementwise factors of Qtil, Ktil, Khat and gamma, the reverse
// in-micro-chunk cumsum of dG for dg (zero where the clamp is active) and the L2-norm and
// sigmoid chain rules. Products are warp-level bf16 MMAs (m16n8k16, fp32 accumulate);
// the 16 x 16 inverse's backward runs on the CUDA cores in fp32. Every [16][32] product
// shares one fragment layout, so the contributions to dq^, dk^ and dG of an element stay
// in one lane's registers until the end of the micro-chunk.
#include <algorithm>

#include "kda_common.cuh"
#include "kda_bwd.cuh"
#include "kda_stage.cuh"
#include "kda_tc_util.cuh"
#include "kda_sm100.cuh"
#include "kda_warp_mma.cuh"

namespace kda {

cudaError_t launch_chunk_warp_save(const ChunkParams &p, int Dv, __nv_bfloat16 *save, cudaStream_t st);

namespace cbw {

using namespace tcu;
using namespace cw;

constexpr int CW = 16, DK = 32;
constexpr int LK = DK + 8;  // [16][32] row-major bf16 tiles (-W, dW)
constexpr int LT = 24;      // [*][16] bf16 tiles (T', A_qk, dA, the transposed operand tiles)
constexpr int LF = 17;      // [16][16] fp32 tiles
constexpr int LG = 40;      // G / dG fp32 [16][LG]: 64-bit fragment reads conflict-free

template <int DV>
struct Lay {
    static constexpr int LV = DV + 8;
    static constexpr uint32_t TT = DK * LT * 2;  // a transposed [32][16] tile
    // inputs: raw q, k, g [16][32]; v and dO [16][LV]; the saved entering state S [32][LV]
    static constexpr uint32_t Q = 0, K = Q + CW * DK * 2, G = K + CW * DK * 2, V = G + CW * DK * 2;
    static constexpr uint32_t DO = V + CW * LV * 2, S = DO + CW * LV * 2;
    // operand tiles (transposed: row = key channel): k^ e^{G-M}, k^ e^{M-G}, q^ e^{G-M},
    // k^ e^G, q^ e^G, k^ e^{G_last-G}
    static constexpr uint32_t XT = S + DK * LV * 2, YT = XT + TT, XQT = YT + TT, KTT = XQT + TT, QTT = KTT + TT,
                              KHT = QTT + TT;
    static constexpr uint32_t TP = KHT + TT, AQ = TP + CW * LT * 2, DAQ = AQ + CW * LT * 2, DA = DAQ + CW * LT * 2;
    static constexpr uint32_t WN = DA + CW * LT * 2, DW = WN + CW * LK * 2;  // -W, dW
    static constexpr uint32_t D = DW + CW * LK * 2, DD = D + CW * LV * 2, DS = DD + CW * LV * 2;
    static constexpr uint32_t AF = DS + DK * LV * 2, TF = AF + CW * LF * 4, DTP = TF + CW * LF * 4, X1 = DTP + CW * LF * 4,
                              DM = X1 + CW * LF * 4;
    static constexpr uint32_t GS = DM + CW * LF * 4;  // G, later dG
    static constexpr uint32_t RK = GS + CW * LG * 4, RQ = RK + 64, BB = RQ + 64, DBS = BB + 64, DAD = DBS + 64,
                              MSK = DAD + 64, GAM = MSK + 64, DGC = GAM + DK * 4;
    static constexpr uint32_t BYTES = (DGC + DK * 4 + 127) / 128 * 128;
};

template <int DV>
__global__ void __launch_bounds__(32) kda_bwd_warp_kernel(const BwdParams p, const __nv_bfloat16 *save) {
    using Ly = Lay<DV>;
    constexpr int LV = Ly::LV, NVT = DV / 8;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    uint8_t *sm = smem_raw;
    const uint32_t sb = sm100::smem_u32(sm);
    const int lane = threadIdx.x, g8 = lane >> 2, t4 = lane & 3;
    const long long chain = blockIdx.x;
    const int n = (int)(chain / p.H), h = (int)(chain % p.H), H = p.H;
    float *rk = reinterpret_cast<float *>(sm + Ly::RK), *rq = reinterpret_cast<float *>(sm + Ly::RQ);
    float *bb = reinterpret_cast<float *>(sm + Ly::BB), *dbs = reinterpret_cast<float *>(sm + Ly::DBS);
    float *dad = reinterpret_cast<float *>(sm + Ly::DAD), *gam = reinterpret_cast<float *>(sm + Ly::GAM);
    float *dgc = reinterpret_cast<float *>(sm + Ly::DGC);
    uint32_t *msk = reinterpret_cast<uint32_t *>(sm + Ly::MSK);
    float *Gs = reinterpret_cast<float *>(sm + Ly::GS);
    float *AF = reinterpret_cast<float *>(sm + Ly::AF), *TF = reinterpret_cast<float *>(sm + Ly::TF);
    float *DTP = reinterpret_cast<float *>(sm + Ly::DTP), *X1 = reinterpret_cast<float *>(sm + Ly::X1);
    float *DMf = reinterpret_cast<float *>(sm + Ly::DM);
    long long bos, eos;
    if (p.cu_seqlens) { bos = p.cu_seqlens[n]; eos = p.cu_seqlens[n + 1]; }
    else { bos = (long long)n * p.T; eos = bos + p.T; }
    const int nmc = (int)((eos - bos + CW - 1) / CW);
    const __nv_bfloat16 *qg = static_cast<const __nv_bfloat16 *>(p.q), *kg = static_cast<const __nv_bfloat16 *>(p.k);
    const __nv_bfloat16 *gg = static_cast<const __nv_bfloat16 *>(p.g), *vg = static_cast<const __nv_bfloat16 *>(p.v);
    const __nv_bfloat16 *dog = static_cast<const __nv_bfloat16 *>(p.dout);
    const __nv_bfloat16 *betag = static_cast<const __nv_bfloat16 *>(p.beta);
    __nv_bfloat16 *dqg = static_cast<__nv_bfloat16 *>(p.dq), *dkg = static_cast<__nv_bfloat16 *>(p.dk);
    __nv_bfloat16 *dvg = static_cast<__nv_bfloat16 *>(p.dv), *dgg = static_cast<__nv_bfloat16 *>(p.dg);
    __nv_bfloat16 *dbg = static_cast<__nv_bfloat16 *>(p.dbeta);
    const float lb = p.lb;

    // the state cotangent: rows c = 16 mk + g8 (+ 8), columns 8 j + 2 t4 (+ 1)
    float dS[2][NVT][4];
    const long long sbase = ((long long)n * H + h) * DK * DV;
#pragma unroll
    for (int mk = 0; mk < 2; ++mk)
#pragma unroll
        for (int j = 0; j < NVT; ++j)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int c = 16 * mk + g8 + 8 * (i >> 1), v = 8 * j + 2 * t4 + (i & 1);
                dS[mk][j][i] = p.dSf ? p.dSf[sbase + (long long)c * DV + v] : 0.f;
            }

    // the inputs of micro-chunk mc, lane (row r = lane / 2, half hf): part 0 the v and dO rows
    // and the saved state's row `lane` (last read by dV), part 1 the raw q, k, g rows (last
    // read by the dq, dk outputs); each part is copied in for the next micro-chunk as soon as
    // this one is done with it
    auto issue = [&](int mc, int part) {
        const long long t0 = bos + (long long)mc * CW;
        const int L = (int)min((long long)CW, eos - t0);
        const int r = lane >> 1, hf = lane & 1;
        const bool ok = r < L;
        const long long row = (t0 + (ok ? r : 0)) * H + h;
        if (part == 0) {
            const uint32_t ov = (r * LV + (DV / 2) * hf) * 2;
#pragma unroll
            for (int c2 = 0; c2 < DV / 16; ++c2) {
                cp16z(sm + Ly::V + ov + 16 * c2, vg + row * DV + (DV / 2) * hf + 8 * c2, ok);
                cp16z(sm + Ly::DO + ov + 16 * c2, dog + row * DV + (DV / 2) * hf + 8 * c2, ok);
            }
            const long long slot = (bos >> 4) + n + mc;
            const __nv_bfloat16 *srow = save + ((slot * H + h) * DK + lane) * DV;
#pragma unroll
            for (int c2 = 0; c2 < DV / 8; ++c2) cp16z(sm + Ly::S + (lane * LV + 8 * c2) * 2, srow + 8 * c2, true);
        } else {
            const uint32_t o = (r * DK + 16 * hf) * 2;
#pragma unroll
            for (int c2 = 0; c2 < 2; ++c2) {
                cp16z(sm + Ly::Q + o + 16 * c2, qg + row * DK + 16 * hf + 8 * c2, ok);
                cp16z(sm + Ly::K + o + 16 * c2, kg + row * DK + 16 * hf + 8 * c2, ok);
                cp16z(sm + Ly::G + o + 16 * c2, gg + row * DK + 16 * hf + 8 * c2, ok);
            }
        }
        cp_async_commit();
    };
    if (nmc > 0) { issue(nmc - 1, 0); issue(nmc - 1, 1); }

    for (int mc = nmc - 1; mc >= 0; --mc) {
        const long long t0 = bos + (long long)mc * CW;
        const int L = (int)min((long long)CW, eos - t0);
        const float braw = lane < L ? __bfloat162float(betag[(t0 + lane) * H + h]) : 0.f;
        cp_async_wait_all();
        __syncwarp();
        // dO' = scale dO in place
        for (int e = lane; e < CW * DV / 8; e += 32) {
            const int r = e / (DV / 8), c8 = e % (DV / 8);
            const uint32_t off = Ly::DO + (r * LV + 8 * c8) * 2;
            float y[8];
            unpack8(lds128(sm, off), y);
#pragma unroll
            for (int u = 0; u < 8; ++u) y[u] *= p.scale;
            sts128(sm, off, pack8(y));
        }
        // ---- G (lane = channel), the clamp mask, row norms, write strengths
        float G[CW];
#pragma unroll
        for (int r = 0; r < CW; ++r) {
            const float x = __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(sm + Ly::G)[r * DK + lane]);
            const uint32_t m = __ballot_sync(0xffffffffu, x >= lb);
            if (lane == 0) msk[r] = m;
            G[r] = r < L ? fmaxf(x, lb) : 0.f;
        }
#pragma unroll
        for (int r = 1; r < CW; ++r) G[r] += G[r - 1];
#pragma unroll
        for (int r = 0; r < CW; ++r) Gs[r * LG + lane] = G[r];
        {
            const int r = lane & 15;
            const uint32_t row = (lane < 16 ? Ly::K : Ly::Q) + r * DK * 2;
            float s = 0.f;
#pragma unroll
            for (int c8 = 0; c8 < DK / 8; ++c8) {
                float f[8];
                unpack8(lds128(sm, row + 16 * c8), f);
#pragma unroll
                for (int e = 0; e < 8; ++e) s = fmaf(f[e], f[e], s);
            }
            const float inv = r < L ? (p.use_l2 ? rsqrtf(s + 1e-6f) : 1.f) : 0.f;
            if (lane < 16) {
                rk[r] = inv;
                bb[r] = r < L ? beta_value(braw, p.beta_prob) : 0.f;
            } else {
                rq[r] = inv;
            }
        }
        __syncwarp();
        // ---- operand tiles, row `lane` of each transposed tile
        const float Gm = G[7], GC = G[CW - 1];
        {
            const __nv_bfloat16 *kr = reinterpret_cast<const __nv_bfloat16 *>(sm + Ly::K);
            const __nv_bfloat16 *qr = reinterpret_cast<const __nv_bfloat16 *>(sm + Ly::Q);
#pragma unroll
            for (int h8 = 0; h8 < 2; ++h8) {
                float x[8], y[8], xq[8], kt[8], qt[8], kc[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int r = 8 * h8 + u;
                    const float kh = __bfloat162float(kr[r * DK + lane]) * rk[r];
                    const float qh = __bfloat162float(qr[r * DK + lane]) * rq[r];
                    const float dm = G[r] - Gm;
                    const float em = e2(dm), en = e2(-dm), eg = e2(G[r]), ec = e2(GC - G[r]);
                    x[u] = kh * em; y[u] = kh * en; xq[u] = qh * em;
                    kt[u] = kh * eg; qt[u] = qh * eg; kc[u] = kh * ec;
                }
                const uint32_t o = (lane * LT + 8 * h8) * 2;
                sts128(sm, Ly::XT + o, pack8(x));
                sts128(sm, Ly::YT + o, pack8(y));
                sts128(sm, Ly::XQT + o, pack8(xq));
                sts128(sm, Ly::KTT + o, pack8(kt));
                sts128(sm, Ly::QTT + o, pack8(qt));
                sts128(sm, Ly::KHT + o, pack8(kc));
            }
            gam[lane] = e2(GC);
        }
        __syncwarp();
        // ---- A_kk (s < r, unscaled, fp32) and A_qk (s <= r, bf16 tile)
        {
            float akk[2][4] = {}, aqk[2][4] = {};
#pragma unroll
            for (int k0 = 0; k0 < DK; k0 += 16) {
                uint32_t a[4], aq[4], b[4];
                frag_at(sb + Ly::XT, LT, 0, k0, lane, a);
                frag_at(sb + Ly::XQT, LT, 0, k0, lane, aq);
                frag_bt(sb + Ly::YT, LT, 0, k0, lane, b);
                mma16816(akk[0], a, b[0], b[1]);
                mma16816(akk[1], a, b[2], b[3]);
                mma16816(aqk[0], aq, b[0], b[1]);
                mma16816(aqk[1], aq, b[2], b[3]);
            }
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int hi = 0; hi < 2; ++hi) {
                    const int r = g8 + 8 * hi, s_ = 8 * j + 2 * t4;
                    AF[r * LF + s_] = s_ < r ? akk[j][2 * hi] : 0.f;
                    AF[r * LF + s_ + 1] = s_ + 1 < r ? akk[j][2 * hi + 1] : 0.f;
                    stb2(sm + Ly::AQ + (r * LT + s_) * 2, s_ <= r ? aqk[j][2 * hi] : 0.f,
                         s_ + 1 <= r ? aqk[j][2 * hi + 1] : 0.f);
                }
        }
        __syncwarp();
        // ---- T = (I + diag(b) A_kk)^-1 (lane j < 16: column j), T' = T diag(b)
        if (lane < CW) {
            const int j = lane;
            float t[CW];
#pragma unroll
            for (int i = 0; i < CW; ++i) {
                float acc = i == j ? 1.f : 0.f;
                const float bi = bb[i];
#pragma unroll
                for (int k = 0; k < i; ++k) acc = fmaf(-bi * AF[i * LF + k], t[k], acc);
                t[i] = acc;
            }
            const float bj = bb[j];
#pragma unroll
            for (int i = 0; i < CW; ++i) {
                TF[i * LF + j] = t[i];
                reinterpret_cast<__nv_bfloat16 *>(sm + Ly::TP)[i * LT + j] = __float2bfloat16_rn(t[i] * bj);
            }
        }
        __syncwarp();
        // ---- D = T'V - W S (registers -> bf16 tile); -W (bf16 tile)
        {
            float U[NVT][4];
            uint32_t a[4];
            frag_a(sb + Ly::TP, LT, 0, 0, lane, a);
#pragma unroll
            for (int j = 0; j < NVT; j += 2) {
                uint32_t b[4];
                frag_bt(sb + Ly::V, LV, 8 * j, 0, lane, b);
                U[j][0] = U[j][1] = U[j][2] = U[j][3] = 0.f;
                U[j + 1][0] = U[j + 1][1] = U[j + 1][2] = U[j + 1][3] = 0.f;
                mma16816(U[j], a, b[0], b[1]);
                mma16816(U[j + 1], a, b[2], b[3]);
            }
            float wv[4][4] = {};
#pragma unroll
            for (int j = 0; j < 4; j += 2) {
                uint32_t b[4];
                frag_b(sb + Ly::KTT, LT, 8 * j, 0, lane, b);
                mma16816(wv[j], a, b[0], b[1]);
                mma16816(wv[j + 1], a, b[2], b[3]);
            }
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int hi = 0; hi < 2; ++hi)
                    stb2(sm + Ly::WN + ((g8 + 8 * hi) * LK + 8 * j + 2 * t4) * 2, -wv[j][2 * hi], -wv[j][2 * hi + 1]);
            __syncwarp();
#pragma unroll
            for (int k0 = 0; k0 < DK; k0 += 16) {
                uint32_t aw[4];
                frag_a(sb + Ly::WN, LK, 0, k0, lane, aw);
#pragma unroll
                for (int j = 0; j < NVT; j += 2) {
                    uint32_t b[4];
                    frag_bt(sb + Ly::S, LV, 8 * j, k0, lane, b);
                    mma16816(U[j], aw, b[0], b[1]);
                    mma16816(U[j + 1], aw, b[2], b[3]);
                }
            }
#pragma unroll
            for (int j = 0; j < NVT; ++j)
#pragma unroll
                for (int hi = 0; hi < 2; ++hi)
                    stb2(sm + Ly::D + ((g8 + 8 * hi) * LV + 8 * j + 2 * t4) * 2, U[j][2 * hi], U[j][2 * hi + 1]);
        }
        // ---- dS_C as a bf16 operand; gamma_c sum_v S dS_C (from the fp32 registers)
#pragma unroll
        for (int mk = 0; mk < 2; ++mk) {
            float rs[2] = {0.f, 0.f};
#pragma unroll
            for (int j = 0; j < NVT; ++j)
#pragma unroll
                for (int hi = 0; hi < 2; ++hi) {
                    const int c = 16 * mk + g8 + 8 * hi, v = 8 * j + 2 * t4;
                    stb2(sm + Ly::DS + (c * LV + v) * 2, dS[mk][j][2 * hi], dS[mk][j][2 * hi + 1]);
                    const float2 s2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(sm + Ly::S + (c * LV + v) * 2));
                    rs[hi] = fmaf(s2.x, dS[mk][j][2 * hi], fmaf(s2.y, dS[mk][j][2 * hi + 1], rs[hi]));
                }
#pragma unroll
            for (int hi = 0; hi < 2; ++hi) {
                rs[hi] += __shfl_xor_sync(0xffffffffu, rs[hi], 1);
                rs[hi] += __shfl_xor_sync(0xffffffffu, rs[hi], 2);
                const int c = 16 * mk + g8 + 8 * hi;
                if (t4 == 0) dgc[c] = gam[c] * rs[hi];
            }
        }
        __syncwarp();
        // ---- dD = A_qk^T dO' + Khat dS_C -> bf16 tile
        {
            float dd[NVT][4];
#pragma unroll
            for (int j = 0; j < NVT; ++j) dd[j][0] = dd[j][1] = dd[j][2] = dd[j][3] = 0.f;
            uint32_t a[4];
            frag_at(sb + Ly::AQ, LT, 0, 0, lane, a);
#pragma unroll
            for (int j = 0; j < NVT; j += 2) {
                uint32_t b[4];
                frag_bt(sb + Ly::DO, LV, 8 * j, 0, lane, b);
                mma16816(dd[j], a, b[0], b[1]);
                mma16816(dd[j + 1], a, b[2], b[3]);
            }
#pragma unroll
            for (int k0 = 0; k0 < DK; k0 += 16) {
                frag_at(sb + Ly::KHT, LT, 0, k0, lane, a);
#pragma unroll
                for (int j = 0; j < NVT; j += 2) {
                    uint32_t b[4];
                    frag_bt(sb + Ly::DS, LV, 8 * j, k0, lane, b);
                    mma16816(dd[j], a, b[0], b[1]);
                    mma16816(dd[j + 1], a, b[2], b[3]);
                }
            }
#pragma unroll
            for (int j = 0; j < NVT; ++j)
#pragma unroll
                for (int hi = 0; hi < 2; ++hi)
                    stb2(sm + Ly::DD + ((g8 + 8 * hi) * LV + 8 * j + 2 * t4) * 2, dd[j][2 * hi], dd[j][2 * hi + 1]);
        }
        __syncwarp();
        // ---- dS <- diag(gamma) dS_C + Qtil^T dO' + (-W)^T dD  (the cotangent entering)
#pragma unroll
        for (int mk = 0; mk < 2; ++mk) {
            const float ga = gam[16 * mk + g8], gb2 = gam[16 * mk + g8 + 8];
#pragma unroll
            for (int j = 0; j < NVT; ++j) {
                dS[mk][j][0] *= ga; dS[mk][j][1] *= ga;
                dS[mk][j][2] *= gb2; dS[mk][j][3] *= gb2;
            }
            uint32_t a[4], aw[4];
            frag_a(sb + Ly::QTT, LT, 16 * mk, 0, lane, a);
            frag_at(sb + Ly::WN, LK, 16 * mk, 0, lane, aw);
#pragma unroll
            for (int j = 0; j < NVT; j += 2) {
                uint32_t b[4], bd[4];
                frag_bt(sb + Ly::DO, LV, 8 * j, 0, lane, b);
                frag_bt(sb + Ly::DD, LV, 8 * j, 0, lane, bd);
                mma16816(dS[mk][j], a, b[0], b[1]);
                mma16816(dS[mk][j + 1], a, b[2], b[3]);
                mma16816(dS[mk][j], aw, bd[0], bd[1]);
                mma16816(dS[mk][j + 1], aw, bd[2], bd[3]);
            }
        }

        // ---- chunk-local gradients. Element e = 4 j + 2 hi (+1): row g8 + 8 hi, column
        // 8 j + 2 t4 (+1) of a [16][32] result.
        float dq_[16], dk_[16], dG_[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) dq_[e] = dk_[e] = dG_[e] = 0.f;
        auto G2 = [&](int r, int c) { return *reinterpret_cast<const float2 *>(Gs + r * LG + c); };
        auto kh2 = [&](int r, int c) {
            const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(sm + Ly::K + (r * DK + c) * 2));
            return make_float2(x.x * rk[r], x.y * rk[r]);
        };
        auto qh2 = [&](int r, int c) {
            const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(sm + Ly::Q + (r * DK + c) * 2));
            return make_float2(x.x * rq[r], x.y * rq[r]);
        };
        // [16][32] = A (16 x K) B (K x 32), A from [M][K] (or [K][M] when AT), B from [N][K]
        // (or [K][N] when BT)
        auto prod32 = [&](float (&acc)[4][4], uint32_t A, int lda, bool at, uint32_t B, int ldb, bool bt, int K) {
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
            for (int k0 = 0; k0 < K; k0 += 16) {
                uint32_t a[4];
                if (at) frag_at(sb + A, lda, 0, k0, lane, a);
                else frag_a(sb + A, lda, 0, k0, lane, a);
#pragma unroll
                for (int j = 0; j < 4; j += 2) {
                    uint32_t b[4];
                    if (bt) frag_bt(sb + B, ldb, 8 * j, k0, lane, b);
                    else frag_b(sb + B, ldb, 8 * j, k0, lane, b);
                    mma16816(acc[j], a, b[0], b[1]);
                    mma16816(acc[j + 1], a, b[2], b[3]);
                }
            }
        };
        float acc[4][4];
        // dQtil = dO' S^T: dq^ += dQtil e^G, dG += dQtil Qtil
        prod32(acc, Ly::DO, LV, false, Ly::S, LV, false, DV);
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int hi = 0; hi < 2; ++hi) {
                const int r = g8 + 8 * hi, c = 8 * j + 2 * t4, e = 4 * j + 2 * hi;
                const float2 Gv = G2(r, c), q = qh2(r, c);
                const float xa = acc[j][2 * hi] * e2(Gv.x), xb = acc[j][2 * hi + 1] * e2(Gv.y);
                dq_[e] += xa; dq_[e + 1] += xb;
                dG_[e] += xa * q.x; dG_[e + 1] += xb * q.y;
            }
        // dW = -dD S^T -> bf16 tile
        prod32(acc, Ly::DD, LV, false, Ly::S, LV, false, DV);
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int hi = 0; hi < 2; ++hi)
                stb2(sm + Ly::DW + ((g8 + 8 * hi) * LK + 8 * j + 2 * t4) * 2, -acc[j][2 * hi], -acc[j][2 * hi + 1]);
        // dKhat = D dS_C^T: dk^ += dKhat e^{G_C-G}, dG -= dKhat Khat, dG_C += sum_r dKhat Khat
        prod32(acc, Ly::D, LV, false, Ly::DS, LV, false, DV);
        {
            float cs_[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int c = 8 * j + 2 * t4;
                const float2 Gc = G2(CW - 1, c);
                cs_[2 * j] = cs_[2 * j + 1] = 0.f;
#pragma unroll
                for (int hi = 0; hi < 2; ++hi) {
                    const int r = g8 + 8 * hi, e = 4 * j + 2 * hi;
                    const float2 Gv = G2(r, c), k = kh2(r, c);
                    const float ea = e2(Gc.x - Gv.x), eb = e2(Gc.y - Gv.y);
                    dk_[e] += acc[j][2 * hi] * ea; dk_[e + 1] += acc[j][2 * hi + 1] * eb;
                    const float pa = acc[j][2 * hi] * k.x * ea, pb = acc[j][2 * hi + 1] * k.y * eb;
                    dG_[e] -= pa; dG_[e + 1] -= pb;
                    cs_[2 * j] += pa; cs_[2 * j + 1] += pb;
                }
            }
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                cs_[i] += __shfl_xor_sync(0xffffffffu, cs_[i], 4);
                cs_[i] += __shfl_xor_sync(0xffffffffu, cs_[i], 8);
                cs_[i] += __shfl_xor_sync(0xffffffffu, cs_[i], 16);
            }
            __syncwarp();
            if (g8 == 0)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    dgc[8 * j + 2 * t4] += cs_[2 * j];
                    dgc[8 * j + 2 * t4 + 1] += cs_[2 * j + 1];
                }
        }
        // dA_qk = dO' D^T: the diagonal apart, the part below it -> bf16 tile
        {
            float aq[2][4] = {};
            for (int k0 = 0; k0 < DV; k0 += 16) {
                uint32_t a[4], b[4];
                frag_a(sb + Ly::DO, LV, 0, k0, lane, a);
                frag_b(sb + Ly::D, LV, 0, k0, lane, b);
                mma16816(aq[0], a, b[0], b[1]);
                mma16816(aq[1], a, b[2], b[3]);
            }
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int hi = 0; hi < 2; ++hi) {
                    const int r = g8 + 8 * hi, s_ = 8 * j + 2 * t4;
                    stb2(sm + Ly::DAQ + (r * LT + s_) * 2, s_ < r ? aq[j][2 * hi] : 0.f, s_ + 1 < r ? aq[j][2 * hi + 1] : 0.f);
                    if (s_ == r) dad[r] = aq[j][2 * hi];
                    if (s_ + 1 == r) dad[r] = aq[j][2 * hi + 1];
                }
        }
        __syncwarp();
        // dT' = dD V^T + dW Ktil^T (fp32)
        {
            float tq[2][4] = {};
            for (int k0 = 0; k0 < DV; k0 += 16) {
                uint32_t a[4], b[4];
                frag_a(sb + Ly::DD, LV, 0, k0, lane, a);
                frag_b(sb + Ly::V, LV, 0, k0, lane, b);
                mma16816(tq[0], a, b[0], b[1]);
                mma16816(tq[1], a, b[2], b[3]);
            }
#pragma unroll
            for (int k0 = 0; k0 < DK; k0 += 16) {
                uint32_t a[4], b[4];
                frag_a(sb + Ly::DW, LK, 0, k0, lane, a);
                frag_bt(sb + Ly::KTT, LT, 0, k0, lane, b);
                mma16816(tq[0], a, b[0], b[1]);
                mma16816(tq[1], a, b[2], b[3]);
            }
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int hi = 0; hi < 2; ++hi) {
                    const int r = g8 + 8 * hi, s_ = 8 * j + 2 * t4;
                    DTP[r * LF + s_] = tq[j][2 * hi];
                    DTP[r * LF + s_ + 1] = tq[j][2 * hi + 1];
                }
        }
        // dV = T'^T dD -> dv
        {
            float dv_[NVT][4];
            uint32_t a[4];
            frag_at(sb + Ly::TP, LT, 0, 0, lane, a);
#pragma unroll
            for (int j = 0; j < NVT; j += 2) {
                uint32_t b[4];
                frag_bt(sb + Ly::DD, LV, 8 * j, 0, lane, b);
                dv_[j][0] = dv_[j][1] = dv_[j][2] = dv_[j][3] = 0.f;
                dv_[j + 1][0] = dv_[j + 1][1] = dv_[j + 1][2] = dv_[j + 1][3] = 0.f;
                mma16816(dv_[j], a, b[0], b[1]);
                mma16816(dv_[j + 1], a, b[2], b[3]);
            }
#pragma unroll
            for (int hi = 0; hi < 2; ++hi) {
                const int r = g8 + 8 * hi;
                if (r < L) {
                    __nv_bfloat16 *orow = dvg + ((t0 + r) * H + h) * DV + 2 * t4;
#pragma unroll
                    for (int j = 0; j < NVT; ++j)
                        *reinterpret_cast<__nv_bfloat162 *>(orow + 8 * j) = __floats2bfloat162_rn(dv_[j][2 * hi], dv_[j][2 * hi + 1]);
                }
            }
        }
        __syncwarp();  // v, dO and the saved state are read: the previous micro-chunk's come in
        if (mc > 0) issue(mc - 1, 0);
        // dKtil = T'^T dW: dk^ += dKtil e^G, dG += dKtil Ktil
        prod32(acc, Ly::TP, LT, true, Ly::DW, LK, true, CW);
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int hi = 0; hi < 2; ++hi) {
                const int r = g8 + 8 * hi, c = 8 * j + 2 * t4, e = 4 * j + 2 * hi;
                const float2 Gv = G2(r, c), k = kh2(r, c);
                const float xa = acc[j][2 * hi] * e2(Gv.x), xb = acc[j][2 * hi + 1] * e2(Gv.y);
                dk_[e] += xa; dk_[e + 1] += xb;
                dG_[e] += xa * k.x; dG_[e + 1] += xb * k.y;
            }
        __syncwarp();
        // ---- the inverse's backward: db_s = sum_r dT'_rs T_rs (lane s < 16), then the two
        // 16 x 16 x 16 products X1 = (dT' diag(b)) T^T and dM = -T^T X1 as tf32 warp MMAs
        if (lane < CW) {
            float s = 0.f;
#pragma unroll
            for (int r = 0; r < CW; ++r) s = fmaf(DTP[r * LF + lane], TF[r * LF + lane], s);
            dbs[lane] = s;
        }
        {
            float x1[2][4] = {};
#pragma unroll
            for (int k0 = 0; k0 < CW; k0 += 8) {
                const uint32_t a[4] = {to_tf32(DTP[g8 * LF + k0 + t4] * bb[k0 + t4]),
                                       to_tf32(DTP[(g8 + 8) * LF + k0 + t4] * bb[k0 + t4]),
                                       to_tf32(DTP[g8 * LF + k0 + t4 + 4] * bb[k0 + t4 + 4]),
                                       to_tf32(DTP[(g8 + 8) * LF + k0 + t4 + 4] * bb[k0 + t4 + 4])};
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const uint32_t b[2] = {to_tf32(TF[(8 * j + g8) * LF + k0 + t4]), to_tf32(TF[(8 * j + g8) * LF + k0 + t4 + 4])};
                    mma_tf32_16x8x8(x1[j], a, b);
                }
            }
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                X1[g8 * LF + 8 * j + 2 * t4] = x1[j][0];
                X1[g8 * LF + 8 * j + 2 * t4 + 1] = x1[j][1];
                X1[(g8 + 8) * LF + 8 * j + 2 * t4] = x1[j][2];
                X1[(g8 + 8) * LF + 8 * j + 2 * t4 + 1] = x1[j][3];
            }
        }
        __syncwarp();
        {
            float dm[2][4] = {};
#pragma unroll
            for (int k0 = 0; k0 < CW; k0 += 8) {
                const uint32_t a[4] = {to_tf32(TF[(k0 + t4) * LF + g8]), to_tf32(TF[(k0 + t4) * LF + g8 + 8]),
                                       to_tf32(TF[(k0 + t4 + 4) * LF + g8]), to_tf32(TF[(k0 + t4 + 4) * LF + g8 + 8])};
#pragma unroll
                for (int j = 0; j < 2; ++j) {
                    const uint32_t b[2] = {to_tf32(X1[(k0 + t4) * LF + 8 * j + g8]), to_tf32(X1[(k0 + t4 + 4) * LF + 8 * j + g8])};
                    mma_tf32_16x8x8(dm[j], a, b);
                }
            }
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                DMf[g8 * LF + 8 * j + 2 * t4] = -dm[j][0];
                DMf[g8 * LF + 8 * j + 2 * t4 + 1] = -dm[j][1];
                DMf[(g8 + 8) * LF + 8 * j + 2 * t4] = -dm[j][2];
                DMf[(g8 + 8) * LF + 8 * j + 2 * t4 + 1] = -dm[j][3];
            }
        }
        __syncwarp();
        if (lane < CW) {  // row r = lane: dA_kk = b_r dM (s < r), db_r += sum_{s<r} dM_rs A_rs
            const int r = lane;
            float db = 0.f;
            float da[CW];
#pragma unroll
            for (int s_ = 0; s_ < CW; ++s_) {
                const float m_ = s_ < r ? DMf[r * LF + s_] : 0.f;
                db = fmaf(m_, AF[r * LF + s_], db);
                da[s_] = bb[r] * m_;
            }
            dbs[r] += db;
            sts128(sm, Ly::DA + r * LT * 2, pack8(da));
            sts128(sm, Ly::DA + r * LT * 2 + 16, pack8(da + 8));
        }
        __syncwarp();
        // ---- the gated products, split at the middle row M = G_7
        // x side (rows r): Zx = dA Y -> dk^ (and dG += k^ Zx); Zqx = dA_qk Y -> dq^ (dG += q^ Zqx)
        // y side (rows s): Zy = dA^T X, Zqy = dA_qk^T XQ -> dk^ (dG -= k^ Z)
#pragma unroll 1
        for (int which = 0; which < 4; ++which) {
            const bool yside = which >= 2, qa = which & 1;
            prod32(acc, qa ? Ly::DAQ : Ly::DA, LT, yside, yside ? (qa ? Ly::XQT : Ly::XT) : Ly::YT, LT, false, CW);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int c = 8 * j + 2 * t4;
                const float2 Mv = G2(7, c);
#pragma unroll
                for (int hi = 0; hi < 2; ++hi) {
                    const int r = g8 + 8 * hi, e = 4 * j + 2 * hi;
                    const float2 Gv = G2(r, c);
                    const float fa = yside ? e2(Mv.x - Gv.x) : e2(Gv.x - Mv.x);
                    const float fb = yside ? e2(Mv.y - Gv.y) : e2(Gv.y - Mv.y);
                    const float za = acc[j][2 * hi] * fa, zb = acc[j][2 * hi + 1] * fb;
                    if (!yside && qa) {
                        const float2 q = qh2(r, c);
                        dq_[e] += za; dq_[e + 1] += zb;
                        dG_[e] += za * q.x; dG_[e + 1] += zb * q.y;
                    } else {
                        const float2 k = kh2(r, c);
                        dk_[e] += za; dk_[e + 1] += zb;
                        if (yside) { dG_[e] -= za * k.x; dG_[e + 1] -= zb * k.y; }
                        else { dG_[e] += za * k.x; dG_[e + 1] += zb * k.y; }
                    }
                }
            }
        }
        // ---- outputs
        {
            float sk2[2] = {0.f, 0.f}, sq2[2] = {0.f, 0.f};
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int hi = 0; hi < 2; ++hi) {
                    const int r = g8 + 8 * hi, c = 8 * j + 2 * t4, e = 4 * j + 2 * hi;
                    const float2 k = kh2(r, c), q = qh2(r, c);
                    const float d = dad[r];  // the diagonal of dA_qk
                    dq_[e] += d * k.x; dq_[e + 1] += d * k.y;
                    dk_[e] += d * q.x; dk_[e + 1] += d * q.y;
                    sk2[hi] += k.x * dk_[e] + k.y * dk_[e + 1];
                    sq2[hi] += q.x * dq_[e] + q.y * dq_[e + 1];
                }
#pragma unroll
            for (int hi = 0; hi < 2; ++hi) {
                sk2[hi] += __shfl_xor_sync(0xffffffffu, sk2[hi], 1);
                sk2[hi] += __shfl_xor_sync(0xffffffffu, sk2[hi], 2);
                sq2[hi] += __shfl_xor_sync(0xffffffffu, sq2[hi], 1);
                sq2[hi] += __shfl_xor_sync(0xffffffffu, sq2[hi], 2);
            }
#pragma unroll
            for (int hi = 0; hi < 2; ++hi) {
                const int r = g8 + 8 * hi;
                if (r >= L) continue;
                const long long o = ((t0 + r) * H + h) * DK + 2 * t4;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int c = 8 * j + 2 * t4, e = 4 * j + 2 * hi;
                    const float2 k = kh2(r, c), q = qh2(r, c);
                    float ka = dk_[e], kb = dk_[e + 1], qa = dq_[e], qb = dq_[e + 1];
                    if (p.use_l2) {
                        ka = rk[r] * (ka - k.x * sk2[hi]); kb = rk[r] * (kb - k.y * sk2[hi]);
                        qa = rq[r] * (qa - q.x * sq2[hi]); qb = rq[r] * (qb - q.y * sq2[hi]);
                    }
                    *reinterpret_cast<__nv_bfloat162 *>(dkg + o + 8 * j) = __floats2bfloat162_rn(ka, kb);
                    *reinterpret_cast<__nv_bfloat162 *>(dqg + o + 8 * j) = __floats2bfloat162_rn(qa, qb);
                }
            }
            __syncwarp();  // every read of G and of the raw rows is done: dG in its place
            if (mc > 0) issue(mc - 1, 1);
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int hi = 0; hi < 2; ++hi) {
                    const int e = 4 * j + 2 * hi;
                    *reinterpret_cast<float2 *>(Gs + (g8 + 8 * hi) * LG + 8 * j + 2 * t4) = make_float2(dG_[e], dG_[e + 1]);
                }
            __syncwarp();
            // dg: reverse cumsum over the rows (lane = channel), dG_C on the last row
            float run = dgc[lane];
#pragma unroll
            for (int r = CW - 1; r >= 0; --r) {
                run += Gs[r * LG + lane];
                if (r < L) {
                    const bool pass = (msk[r] >> lane) & 1u;
                    dgg[((t0 + r) * H + h) * DK + lane] = __float2bfloat16_rn(pass ? run : 0.f);
                }
            }
            if (lane < L) {
                const float b = bb[lane], d = dbs[lane];
                dbg[(t0 + lane) * H + h] = __float2bfloat16_rn(p.beta_prob ? d : d * b * (1.f - b));
            }
        }
        __syncwarp();
    }
    if (p.dS0) {
#pragma unroll
        for (int mk = 0; mk < 2; ++mk)
#pragma unroll
            for (int j = 0; j < NVT; ++j)
#pragma unroll
                for (int hi = 0; hi < 2; ++hi) {
                    const int c = 16 * mk + g8 + 8 * hi, v = 8 * j + 2 * t4;
                    *reinterpret_cast<float2 *>(p.dS0 + sbase + (long long)c * DV + v) =
                        make_float2(dS[mk][j][2 * hi], dS[mk][j][2 * hi + 1]);
                }
    }
}

template <int DV>
cudaError_t launch_t(const BwdParams &p, const __nv_bfloat16 *save, cudaStream_t st) {
    const long long chains = (long long)p.N * p.H;
    if (chains <= 0) return cudaSuccess;
    const uint32_t smem = Lay<DV>::BYTES;
    cudaError_t e = cudaFuncSetAttribute(kda_bwd_warp_kernel<DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    count_launch();
    kda_bwd_warp_kernel<DV><<<(unsigned)chains, 32, smem, st>>>(p, save);
    return cudaGetLastError();
}

}  // namespace cbw

// The micro-chunk backward applies to bf16 d_k = 32 (d_v 32 or 64) with a lower bound
// >= -10 (the middle-row split stays within e^80) and enough chains to fill the part.
bool bwd_warp_supported(const BwdParams &p, bool bf16, int Dk, int Dv) {
    return bf16 && Dk == 32 && (Dv == 32 || Dv == 64) && p.has_lb && p.lb >= -10.f && (long long)p.N * p.H >= 256;
}

// Workspace: the saved states, one bf16 [32][d_v] tile per (micro-chunk slot, head).
size_t bwd_warp_workspace_bytes(const BwdParams &p, int Dv) {
    const long long total = p.cu_seqlens ? (long long)p.T : (long long)p.N * p.T;
    const long long slots = total / 16 + p.N + 1;
    return (size_t)slots * p.H * 32 * Dv * 2;
}

cudaError_t launch_bwd_warp(const BwdParams &p, int Dv, void *workspace, cudaStream_t st) {
    __nv_bfloat16 *save = static_cast<__nv_bfloat16 *>(workspace);
    ChunkParams f{};
    f.q = p.q; f.k = p.k; f.v = p.v; f.g = p.g; f.beta = p.beta;
    f.o = nullptr;
    f.S0 = p.S0;
    f.S_out = nullptr;
    f.cu_seqlens = p.cu_seqlens;
    f.T = p.T; f.N = p.N; f.H = p.H;
    f.scale = p.scale;
    f.use_l2 = p.use_l2;
    f.has_lb = p.has_lb;
    f.lb = p.lb;
    f.gate_mode = kGateLog;
    f.beta_prob = p.beta_prob;
    cudaError_t e = launch_chunk_warp_save(f, Dv, save, st);
    if (e != cudaSuccess) return e;
    return Dv == 32 ? cbw::launch_t<32>(p, save, st) : cbw::launch_t<64>(p, save, st);
}

}  // namespace kda
