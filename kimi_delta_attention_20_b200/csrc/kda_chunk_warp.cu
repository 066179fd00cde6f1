// Chunk forward for bf16 inputs with d_k 32 or 64 (d_v 32 or 64) when there are many
// (sequence, head) chains: the WY/UT chunk form on 16-token micro-chunks, every product
// a warp-level tensor-core MMA (m16n8k16, bf16 operands, fp32 accumulate) and the fp32
// state in accumulator registers.
//
// The operator is the `chunk_kda` boundary of page "K3/kda/ops/api.py" (the token
// recurrence of page "atlas_core/kimi_k3/kda.rs"). The chunk form is exact for any
// chunk size -- grouping tokens changes the order of the arithmetic, not its value --
// and with 16 tokens the UT inverse is a 16 x 16 unit-triangular solve inside one
// warp, every product is one MMA tile high, and a 32 x d_v state fits in the registers
// of one or two warps, so a chain needs no record. Per micro-chunk (G the in-chunk
// cumsum of the gate, k^, q^ the normalised rows, b the write strengths):
//   A_kk[r,s] = sum_c k^_rc k^_sc e^{G_rc - G_sc} (s < r),  A_qk likewise with q^ (s <= r)
//   T' = (I + diag(b) A_kk)^-1 diag(b),  U = T' V,  W = T' (k^ e^G)
//   D = U - W S,  O = scale ((q^ e^G) S + A_qk D),  S <- diag(e^{G_last}) S + (k^ e^{G_last - G})^T D.
// The gated products split e^{G_r - G_s} at the micro-chunk's middle row (both parts
// <= e^80 while the gate moves by at most 80 over half a micro-chunk); a micro-chunk
// whose gate moves further takes A_kk and A_qk from exponent differences on the CUDA
// cores. Lane = key channel for the gate, its cumsum and the operand tiles.
//
// Three kernels, each one CTA of two warps per chain (the chains are serial, so the
// time is set by per-chain latency while every chain is in flight):
//   d_k = 32 by default: w2 -- the warps split the value columns and the rows of the
//     key-side work, meeting at block barriers;
//   d_k = 32 with the log-decay gate and up to four chains per SM: pc -- a producer warp
//     forms the key side of the next micro-chunk while a consumer warp runs the state chain
//     of the current one;
//   d_k = 64: w64 -- as w2, over 64 key channels.
#include <algorithm>

#include "kda_common.cuh"
#include "kda_stage.cuh"
#include "kda_tc_util.cuh"
#include "kda_sm100.cuh"
#include "kda_warp_mma.cuh"

namespace kda {
namespace cw {

using namespace tcu;

constexpr int CW = 16;      // tokens per micro-chunk
constexpr int DK = 32;      // key dim (lane = key channel)
constexpr int LK = DK + 8;  // padded row of a [16][32] bf16 tile (elements): 80 B, conflict-free fragments
constexpr int LT = 24;      // padded row of a [16][16] bf16 tile: 48 B
constexpr int LL = 20;      // row of the fp32 L tile: 80 B, so a row is read four values at a time
constexpr float kSpan = 80.f;  // largest |G - G_mid| of the split products

// ---- d_k = 64: one CTA of two warps per chain. Warp w owns the value columns
// [VW w, VW w + VW) of the 64 x d_v state (VW = d_v / 2), held transposed (S^T) in
// accumulator registers as in the d_k = 32 forms below, and the key channels
// [32 w, 32 w + 32) of the gate and of the transposed operand tiles; the 16 x 16 blocks
// are split between the warps (warp 0 A_kk and the inverse, warp 1 A_qk and then its
// (q^ e^G) S), and block barriers separate the phases that read the other warp's half.
// O^T leaves through transposing matrix stores into this step's v stage.
namespace w64 {
constexpr int DK2 = 64;
constexpr int LKR = DK2 + 8;  // padded raw row (elements): 144 B, conflict-free row reads
constexpr int LW = DK2 + 8;   // the -W tile [16][LW]
template <int DV>
struct Lay {
    static constexpr int LV = DV + 8;
    // two input stages: raw q, k, g [16][LKR] and v [16][LV] (v's stage then stages O)
    static constexpr uint32_t Q = 0, K = Q + CW * LKR * 2, G = K + CW * LKR * 2, V = G + CW * LKR * 2;
    static constexpr uint32_t IN = (V + CW * LV * 2 + 127) / 128 * 128;
    static constexpr uint32_t TT = DK2 * LT * 2;  // a transposed tile [64][LT]
    static constexpr uint32_t X = 2 * IN, Y = X + TT, XQ = Y + TT, KT = XQ + TT, QT = KT + TT, KH = QT + TT;
    static constexpr uint32_t W = X;                                // -W [16][LW] over X^T
    static constexpr uint32_t TP = KH + TT, AQ = TP + CW * LT * 2;  // T'^T [16][LT], A_qk [16][LT]
    static constexpr uint32_t L = AQ + CW * LT * 2;                 // L = diag(b) A_kk, f32 [16][LL]
    static constexpr uint32_t RK = L + CW * LL * 4, RQ = RK + 64, BB = RQ + 64, PART = BB + 64, GAM = PART + 256;
    static constexpr uint32_t BYTES = (GAM + DK2 * 4 + 127) / 128 * 128;
    static_assert(CW * LW * 2 <= TT && CW * 65 * 4 <= 2 * TT, "aliases over X^T (and Y^T)");
    static_assert(L % 16 == 0 && RK % 16 == 0 && RQ % 16 == 0, "rows read 16 bytes at a time");
};

template <int DV>
__global__ void __launch_bounds__(64, 5) kda_chunk_warp64_kernel(const ChunkParams p) {
    using Ly = Lay<DV>;
    constexpr int LV = Ly::LV, VW = DV / 2, MT = VW / 16;  // own value columns and their m-tiles
    extern __shared__ __align__(16) uint8_t smem_raw[];
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const long long chain = blockIdx.x;
    const int n = (int)(chain / p.H), h = (int)(chain % p.H);
    uint8_t *sm = smem_raw;
    const uint32_t sb = sm100::smem_u32(sm);
    float *rk = reinterpret_cast<float *>(sm + Ly::RK), *rq = reinterpret_cast<float *>(sm + Ly::RQ);
    float *bb = reinterpret_cast<float *>(sm + Ly::BB), *gam = reinterpret_cast<float *>(sm + Ly::GAM);
    float *part = reinterpret_cast<float *>(sm + Ly::PART);
    float *Lf = reinterpret_cast<float *>(sm + Ly::L);
    const int H = p.H, g8 = lane >> 2, t4 = lane & 3, mi = lane >> 3, mr = lane & 7;
    const int c = 32 * w + lane;  // this thread's key channel
    long long bos, eos;
    if (p.cu_seqlens) { bos = p.cu_seqlens[n]; eos = p.cu_seqlens[n + 1]; }
    else { bos = (long long)n * p.T; eos = bos + p.T; }
    const int nmc = (int)((eos - bos + CW - 1) / CW);
    const __nv_bfloat16 *qg = static_cast<const __nv_bfloat16 *>(p.q), *kg = static_cast<const __nv_bfloat16 *>(p.k);
    const __nv_bfloat16 *gg = static_cast<const __nv_bfloat16 *>(p.g), *vg = static_cast<const __nv_bfloat16 *>(p.v);
    const __nv_bfloat16 *betag = static_cast<const __nv_bfloat16 *>(p.beta);
    __nv_bfloat16 *og = static_cast<__nv_bfloat16 *>(p.o);
    const float rate = p.gate_mode != kGateLog ? expf(p.A_log[h]) : 0.f;
    const float bias = (p.gate_mode != kGateLog && p.dt_bias) ? p.dt_bias[(long long)h * DK2 + c] : 0.f;

    // thread (row r = tid / 4, quarter qq = tid % 4): q, k, g pieces 2 qq, 2 qq + 1 and its
    // share of the v row; thread r < 16 also loads token r's beta into braw
    float braw = 0.f;
    auto issue = [&](int mc) {
        const long long t0 = bos + (long long)mc * CW;
        const int L = (int)min((long long)CW, eos - t0);
        const int r = tid >> 2, qq = tid & 3;
        const bool ok = r < L;
        const long long row = (t0 + (ok ? r : 0)) * H + h;
        const uint32_t in = (mc & 1) * Ly::IN, o = in + (r * LKR + 16 * qq) * 2;
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
            cp16z(sm + Ly::Q + o + 16 * cc, qg + row * DK2 + 16 * qq + 8 * cc, ok);
            cp16z(sm + Ly::K + o + 16 * cc, kg + row * DK2 + 16 * qq + 8 * cc, ok);
            cp16z(sm + Ly::G + o + 16 * cc, gg + row * DK2 + 16 * qq + 8 * cc, ok);
        }
        constexpr int VP = DV / 32;  // 16-byte v pieces per thread
#pragma unroll
        for (int cc = 0; cc < VP; ++cc) {
            const int piece = VP * qq + cc;
            cp16z(sm + in + Ly::V + (r * LV + 8 * piece) * 2, vg + row * DV + 8 * piece, ok);
        }
        braw = tid < L ? __bfloat162float(betag[(t0 + tid) * H + h]) : 0.f;
        cp_async_commit();
    };

    // S^T, own value columns: rows (values) VW w + 16 mt + g8 (+ 8), columns (keys) 8 nk + 2 t4 (+ 1)
    float ST[MT][8][4];
    const long long sbase = ((long long)n * H + h) * DK2 * DV;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int nk = 0; nk < 8; ++nk)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int v = VW * w + 16 * mt + g8 + 8 * (i >> 1), cr = 8 * nk + 2 * t4 + (i & 1);
                ST[mt][nk][i] = p.S0 ? p.S0[sbase + (long long)cr * DV + v] : 0.f;
            }
    // A fragment of S^T (bf16) for own value m-tile mt and key step kk
    auto sfrag = [&](int mt, int kk, uint32_t (&a)[4]) {
        a[0] = pack_bf16x2(ST[mt][2 * kk][0], ST[mt][2 * kk][1]);
        a[1] = pack_bf16x2(ST[mt][2 * kk][2], ST[mt][2 * kk][3]);
        a[2] = pack_bf16x2(ST[mt][2 * kk + 1][0], ST[mt][2 * kk + 1][1]);
        a[3] = pack_bf16x2(ST[mt][2 * kk + 1][2], ST[mt][2 * kk + 1][3]);
    };

    if (nmc > 0) issue(0);
    for (int mc = 0; mc < nmc; ++mc) {
        const long long t0 = bos + (long long)mc * CW;
        const int L = (int)min((long long)CW, eos - t0);
        const float bcur = braw;
        const uint32_t in = (mc & 1) * Ly::IN;
        cp_async_wait_all();
        __syncthreads();  // this micro-chunk's rows, from both warps' copies
        // gate and cumsum for channel c
        float G[CW];
#pragma unroll
        for (int r = 0; r < CW; ++r) {
            const float x = __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(sm + in + Ly::G)[r * LKR + c]);
            const float gv = p.gate_mode == kGateLog ? (p.has_lb ? fmaxf(x, p.lb) : x)
                                                     : gate_fast(x, bias, rate, p.gate_mode, p.lb);
            G[r] = r < L ? gv : 0.f;
        }
#pragma unroll
        for (int r = 1; r < CW; ++r) G[r] += G[r - 1];
        // row norms: each warp sums its 32 channels (lanes 0..15 k rows, 16..31 q rows)
        {
            const int r = lane & 15;
            const uint32_t row = in + (lane < 16 ? Ly::K : Ly::Q) + (r * LKR + 32 * w) * 2;
            float sacc = 0.f;
#pragma unroll
            for (int c8 = 0; c8 < 4; ++c8) {
                float f[8];
                unpack8(lds128(sm, row + 16 * c8), f);
#pragma unroll
                for (int e = 0; e < 8; ++e) sacc = fmaf(f[e], f[e], sacc);
            }
            part[w * 32 + lane] = sacc;
        }
        __syncthreads();
        if (tid < 32) {
            const int r = tid & 15;
            const float ssum = part[tid] + part[32 + tid];
            const float inv = r < L ? (p.use_l2 ? rsqrtf(ssum + 1e-6f) : 1.f) : 0.f;
            if (tid < 16) {
                rk[r] = inv;
                bb[r] = r < L ? beta_value(bcur, p.beta_prob) : 0.f;
            } else {
                rq[r] = inv;
            }
        }
        __syncthreads();
        // operand tiles, row c of each transposed tile
        const float Gm = G[7], GC = G[CW - 1];
        bool steep = false;
        {
            const __nv_bfloat16 *kr = reinterpret_cast<const __nv_bfloat16 *>(sm + in + Ly::K);
            const __nv_bfloat16 *qr = reinterpret_cast<const __nv_bfloat16 *>(sm + in + Ly::Q);
#pragma unroll
            for (int h8 = 0; h8 < 2; ++h8) {
                const float4 rka = *reinterpret_cast<const float4 *>(rk + 8 * h8);
                const float4 rkb = *reinterpret_cast<const float4 *>(rk + 8 * h8 + 4);
                const float4 rqa = *reinterpret_cast<const float4 *>(rq + 8 * h8);
                const float4 rqb = *reinterpret_cast<const float4 *>(rq + 8 * h8 + 4);
                const float rkv[8] = {rka.x, rka.y, rka.z, rka.w, rkb.x, rkb.y, rkb.z, rkb.w};
                const float rqv[8] = {rqa.x, rqa.y, rqa.z, rqa.w, rqb.x, rqb.y, rqb.z, rqb.w};
                float x[8], y[8], xq[8], kt[8], qt[8], kc[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int r = 8 * h8 + u;
                    const float kh = __bfloat162float(kr[r * LKR + c]) * rkv[u];
                    const float qh = __bfloat162float(qr[r * LKR + c]) * rqv[u];
                    const float dm = G[r] - Gm;
                    steep |= fabsf(dm) > kSpan;
                    const float em = e2(dm), en = e2(-dm), eg = e2(G[r]), ec = e2(GC - G[r]);
                    x[u] = kh * em; y[u] = kh * en; xq[u] = qh * em;
                    kt[u] = kh * eg; qt[u] = qh * eg; kc[u] = kh * ec;
                }
                const uint32_t o = (c * LT + 8 * h8) * 2;
                sts128(sm, Ly::X + o, pack8(x));
                sts128(sm, Ly::Y + o, pack8(y));
                sts128(sm, Ly::XQ + o, pack8(xq));
                sts128(sm, Ly::KT + o, pack8(kt));
                sts128(sm, Ly::QT + o, pack8(qt));
                sts128(sm, Ly::KH + o, pack8(kc));
            }
            gam[c] = e2(GC);
        }
        steep = __syncthreads_or(steep) != 0;
        // the next micro-chunk's rows into the other stage (read, and its O staging copied
        // out, in the previous micro-chunk, which both warps finished before this one's
        // first barrier)
        if (mc + 1 < nmc) issue(mc + 1);
        // A_kk (warp 0) -> L = diag(b) A_kk; A_qk (warp 1) -> bf16 tile
        {
            float acc[2][4] = {};
            const uint32_t xa = w == 0 ? Ly::X : Ly::XQ;
#pragma unroll
            for (int k0 = 0; k0 < DK2; k0 += 16) {
                uint32_t a[4], bf[4];
                frag_at(sb + xa, LT, 0, k0, lane, a);
                frag_bt(sb + Ly::Y, LT, 0, k0, lane, bf);
                mma16816(acc[0], a, bf[0], bf[1]);
                mma16816(acc[1], a, bf[2], bf[3]);
            }
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int hi = 0; hi < 2; ++hi) {
                    const int r = g8 + 8 * hi, s_ = 8 * j + 2 * t4;
                    if (w == 0) {
                        const float br = bb[r];
                        *reinterpret_cast<float2 *>(Lf + r * LL + s_) = make_float2(
                            s_ < r ? br * acc[j][2 * hi] : 0.f, s_ + 1 < r ? br * acc[j][2 * hi + 1] : 0.f);
                    } else {
                        stb2(sm + Ly::AQ + (r * LT + s_) * 2, s_ <= r ? acc[j][2 * hi] : 0.f,
                             s_ + 1 <= r ? acc[j][2 * hi + 1] : 0.f);
                    }
                }
        }
        if (steep) {  // exponent differences (never positive) on the CUDA cores
            __syncthreads();  // X^T and Y^T are read by both warps: the scratch goes over them
            float *Gs = reinterpret_cast<float *>(sm + Ly::X);
#pragma unroll
            for (int r = 0; r < CW; ++r) Gs[r * 65 + c] = G[r];
            __syncthreads();
            const __nv_bfloat16 *kr = reinterpret_cast<const __nv_bfloat16 *>(sm + in + Ly::K);
            const __nv_bfloat16 *qr = reinterpret_cast<const __nv_bfloat16 *>(sm + in + Ly::Q);
            for (int e = tid; e < CW * CW; e += 64) {
                const int r = e >> 4, s_ = e & 15;
                if (s_ > r) continue;
                float akk = 0.f, aqk = 0.f;
                for (int cc = 0; cc < DK2; ++cc) {
                    const float ed = expf(Gs[r * 65 + cc] - Gs[s_ * 65 + cc]);
                    const float ks = __bfloat162float(kr[s_ * LKR + cc]) * ed;
                    akk = fmaf(__bfloat162float(kr[r * LKR + cc]), ks, akk);
                    aqk = fmaf(__bfloat162float(qr[r * LKR + cc]), ks, aqk);
                }
                akk *= rk[r] * rk[s_];
                aqk *= rq[r] * rk[s_];
                if (s_ < r) Lf[r * LL + s_] = bb[r] * akk;
                reinterpret_cast<__nv_bfloat16 *>(sm + Ly::AQ)[r * LT + s_] = __float2bfloat16_rn(aqk);
            }
        }
        __syncthreads();
        // T' by forward substitution (warp 0, lane j < 16: column j, a row of L four values at
        // a time); row j of T'^T = column j of T diag(b) (two 16-byte stores)
        if (w == 0 && lane < CW) {
            const int j = lane;
            float t[CW];
#pragma unroll
            for (int i = 0; i < CW; ++i) {
                float acc = i == j ? 1.f : 0.f;
#pragma unroll
                for (int k4 = 0; k4 < i; k4 += 4) {
                    const float4 l4 = *reinterpret_cast<const float4 *>(Lf + i * LL + k4);
                    acc = fmaf(-l4.x, t[k4], acc);
                    if (k4 + 1 < i) acc = fmaf(-l4.y, t[k4 + 1], acc);
                    if (k4 + 2 < i) acc = fmaf(-l4.z, t[k4 + 2], acc);
                    if (k4 + 3 < i) acc = fmaf(-l4.w, t[k4 + 3], acc);
                }
                t[i] = acc;
            }
            const float bj = bb[j];
#pragma unroll
            for (int i = 0; i < CW; ++i) t[i] *= bj;
            sts128(sm, Ly::TP + (j * LT) * 2, pack8(t));
            sts128(sm, Ly::TP + (j * LT + 8) * 2, pack8(t + 8));
        }
        // O^T = S^T Qtil^T for own value columns (warp 1 while the inverse runs)
        float OT[MT][2][4];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int i = 0; i < 4; ++i) OT[mt][0][i] = OT[mt][1][i] = 0.f;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            uint32_t bq[4];
            frag_bt(sb + Ly::QT, LT, 0, 16 * kk, lane, bq);
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                uint32_t a[4];
                sfrag(mt, kk, a);
                mma16816(OT[mt][0], a, bq[0], bq[1]);
                mma16816(OT[mt][1], a, bq[2], bq[3]);
            }
        }
        __syncthreads();  // T'
        // U^T = V^T T'^T (own value columns); -W = -T' Ktil for key channels [32 w, 32 w + 32)
        float UT[MT][2][4];
        {
            uint32_t bt[4];
            frag_bt(sb + Ly::TP, LT, 0, 0, lane, bt);
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                uint32_t a[4];
                frag_at(sb + in + Ly::V, LV, VW * w + 16 * mt, 0, lane, a);
#pragma unroll
                for (int i = 0; i < 4; ++i) UT[mt][0][i] = UT[mt][1][i] = 0.f;
                mma16816(UT[mt][0], a, bt[0], bt[1]);
                mma16816(UT[mt][1], a, bt[2], bt[3]);
            }
            uint32_t a[4];
            frag_at(sb + Ly::TP, LT, 0, 0, lane, a);
#pragma unroll
            for (int jb = 0; jb < 4; jb += 2) {
                uint32_t bf[4];
                frag_b(sb + Ly::KT, LT, 32 * w + 8 * jb, 0, lane, bf);
                float wv[2][4] = {};
                mma16816(wv[0], a, bf[0], bf[1]);
                mma16816(wv[1], a, bf[2], bf[3]);
                // matrix mi: row half mi % 2, key n-tile 4 w + jb + mi / 2
                stsm4(sb + Ly::W + ((8 * (mi & 1) + mr) * LW + 32 * w + 8 * (jb + (mi >> 1))) * 2,
                      pack_bf16x2(-wv[0][0], -wv[0][1]), pack_bf16x2(-wv[0][2], -wv[0][3]),
                      pack_bf16x2(-wv[1][0], -wv[1][1]), pack_bf16x2(-wv[1][2], -wv[1][3]));
            }
        }
        __syncthreads();  // -W complete
        // D^T = U^T + S^T (-W)^T (own value columns), as bf16 A fragments over the tokens
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            uint32_t bw[4];
            frag_b(sb + Ly::W, LW, 0, 16 * kk, lane, bw);
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                uint32_t a[4];
                sfrag(mt, kk, a);
                mma16816(UT[mt][0], a, bw[0], bw[1]);
                mma16816(UT[mt][1], a, bw[2], bw[3]);
            }
        }
        uint32_t DA[MT][4];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            DA[mt][0] = pack_bf16x2(UT[mt][0][0], UT[mt][0][1]);
            DA[mt][1] = pack_bf16x2(UT[mt][0][2], UT[mt][0][3]);
            DA[mt][2] = pack_bf16x2(UT[mt][1][0], UT[mt][1][1]);
            DA[mt][3] = pack_bf16x2(UT[mt][1][2], UT[mt][1][3]);
        }
        // O^T += D^T A_qk^T; out through the staging tile over this stage's own v columns
        {
            uint32_t baq[4];
            frag_b(sb + Ly::AQ, LT, 0, 0, lane, baq);
            const float f = p.scale;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                mma16816(OT[mt][0], DA[mt], baq[0], baq[1]);
                mma16816(OT[mt][1], DA[mt], baq[2], baq[3]);
                // matrix mi: token rows 8 (mi / 2) + mr, value columns VW w + 16 mt + 8 (mi % 2)
                stsm4t(sb + in + Ly::V + ((8 * (mi >> 1) + mr) * LV + VW * w + 16 * mt + 8 * (mi & 1)) * 2,
                       pack_bf16x2(f * OT[mt][0][0], f * OT[mt][0][1]), pack_bf16x2(f * OT[mt][0][2], f * OT[mt][0][3]),
                       pack_bf16x2(f * OT[mt][1][0], f * OT[mt][1][1]), pack_bf16x2(f * OT[mt][1][2], f * OT[mt][1][3]));
            }
        }
        // S^T <- S^T diag(e^{G_last}) + D^T Khat (own value columns)
#pragma unroll
        for (int nk = 0; nk < 8; ++nk) {
            const float2 gk = *reinterpret_cast<const float2 *>(gam + 8 * nk + 2 * t4);
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                ST[mt][nk][0] *= gk.x; ST[mt][nk][1] *= gk.y;
                ST[mt][nk][2] *= gk.x; ST[mt][nk][3] *= gk.y;
            }
        }
#pragma unroll
        for (int nk = 0; nk < 8; nk += 2) {
            uint32_t bk[4];
            frag_b(sb + Ly::KH, LT, 8 * nk, 0, lane, bk);
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                mma16816(ST[mt][nk], DA[mt], bk[0], bk[1]);
                mma16816(ST[mt][nk + 1], DA[mt], bk[2], bk[3]);
            }
        }
        if (og) {  // rows < L of the staged O, own columns, 16 bytes per lane and step
            __syncwarp();
            constexpr int PR = VW / 8;
#pragma unroll
            for (int q = lane; q < CW * PR; q += 32) {
                const int r = q / PR, cq = q % PR;
                if (r < L)
                    *reinterpret_cast<uint4 *>(og + ((t0 + r) * H + h) * DV + VW * w + 8 * cq) =
                        lds128(sm, in + Ly::V + (r * LV + VW * w + 8 * cq) * 2);
            }
        }
        // no barrier here: the next micro-chunk writes shared tiles only after its first
        // barrier, which both warps reach only when done with this one (the O staging is
        // this warp's own columns)
    }
    cp_async_wait_all();
    if (p.S_out) {
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int nk = 0; nk < 8; ++nk)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int v = VW * w + 16 * mt + g8 + 8 * (i >> 1), cr = 8 * nk + 2 * t4 + (i & 1);
                    p.S_out[sbase + (long long)cr * DV + v] = ST[mt][nk][i];
                }
    }
}

template <int DV>
cudaError_t launch_t(const ChunkParams &p, cudaStream_t st) {
    const long long chains = (long long)p.N * p.H;
    if (chains <= 0) return cudaSuccess;
    const uint32_t smem = Lay<DV>::BYTES;
    cudaError_t e = cudaFuncSetAttribute(kda_chunk_warp64_kernel<DV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    count_launch();
    kda_chunk_warp64_kernel<DV><<<(unsigned)chains, 64, smem, st>>>(p);
    return cudaGetLastError();
}
}  // namespace w64


// ---- d_k = 32 on a pair of warps per chain (one 64-thread CTA): warp w owns the value
// columns [VW w, VW w + VW) of the state, held transposed (S^T, registers) as in the
// consumer of the pc form below, and rows [8 w, 8 w + 8) of the gate values and of the
// transposed operand tiles (the warps exchange one running gate sum per channel); warp 0
// forms A_kk and the inverse, warp 1 A_qk and then its (q^ e^G) S while the inverse runs.
// S^T and D^T never pass through shared memory, and O^T leaves through transposing matrix
// stores into this step's v stage (each warp its own columns); save as in the pc form. AUG: the widened run of the segment form (kda_chunk_rec.cu): the state is [M | N]
// (32 x DV, DV = 32 + d_v; warp 0 owns M, warp 1 N), M starts from the identity and sees
// v = 0, N starts from zero and sees v; the outputs [scale M^T q^ | scale N^T q^] go out
// in fp32 rows of DV and the final state as [32][DV].
namespace w2 {
template <int DV>
struct Lay {
    static constexpr int LV = DV + 8;
    // two input stages: raw q, k, g [16][32] and v [16][LV] (v's stage then stages O)
    static constexpr uint32_t Q = 0, K = Q + CW * DK * 2, G = K + CW * DK * 2, V = G + CW * DK * 2;
    static constexpr uint32_t IN = (V + CW * LV * 2 + 127) / 128 * 128;
    static constexpr uint32_t TT = DK * LT * 2;
    static constexpr uint32_t X = 2 * IN, Y = X + TT, XQ = Y + TT, KT = XQ + TT, QT = KT + TT, KH = QT + TT;
    static constexpr uint32_t W = X;  // -W [16][LK] over X^T (after the A products)
    static constexpr uint32_t TP = KH + TT, AQ = TP + CW * LT * 2;  // T'^T [16][LT], A_qk [16][LT]
    static constexpr uint32_t L = AQ + CW * LT * 2;                  // L = diag(b) A_kk, f32 [16][LL]
    static constexpr uint32_t RK = L + CW * LL * 4, RQ = RK + 64, BB = RQ + 64, GAM = BB + 64, XG = GAM + DK * 4;
    static constexpr uint32_t BYTES = (XG + 2 * DK * 4 + 127) / 128 * 128;
    static_assert(CW * LK * 2 <= TT && CW * 33 * 4 <= 2 * TT, "aliases over X^T (and Y^T)");
    static_assert(L % 16 == 0 && RK % 16 == 0 && RQ % 16 == 0, "rows read 16 bytes at a time");
};

template <int DV, bool AUG, bool SAVE>
__global__ void __launch_bounds__(64, 7) kda_chunk_pair_kernel(const ChunkParams p, __nv_bfloat16 *save) {
    using Ly = Lay<DV>;
    constexpr int LV = Ly::LV, VW = DV / 2, MT = VW / 16;  // own value columns and their m-tiles
    constexpr int VOFF = AUG ? DK : 0, DVR = DV - VOFF;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const long long chain = blockIdx.x;
    const int n = (int)(chain / p.H), h = (int)(chain % p.H);
    uint8_t *sm = smem_raw;
    const uint32_t sb = sm100::smem_u32(sm);
    float *rk = reinterpret_cast<float *>(sm + Ly::RK), *rq = reinterpret_cast<float *>(sm + Ly::RQ);
    float *bb = reinterpret_cast<float *>(sm + Ly::BB), *gam = reinterpret_cast<float *>(sm + Ly::GAM);
    float *Lf = reinterpret_cast<float *>(sm + Ly::L), *XG = reinterpret_cast<float *>(sm + Ly::XG);
    const int H = p.H, g8 = lane >> 2, t4 = lane & 3, mi = lane >> 3, mr = lane & 7;
    long long bos, eos;
    if (p.cu_seqlens) { bos = p.cu_seqlens[n]; eos = p.cu_seqlens[n + 1]; }
    else { bos = (long long)n * p.T; eos = bos + p.T; }
    const int nmc = (int)((eos - bos + CW - 1) / CW);
    const __nv_bfloat16 *qg = static_cast<const __nv_bfloat16 *>(p.q), *kg = static_cast<const __nv_bfloat16 *>(p.k);
    const __nv_bfloat16 *gg = static_cast<const __nv_bfloat16 *>(p.g), *vg = static_cast<const __nv_bfloat16 *>(p.v);
    const __nv_bfloat16 *betag = static_cast<const __nv_bfloat16 *>(p.beta);
    __nv_bfloat16 *og = static_cast<__nv_bfloat16 *>(p.o);
    const float rate = p.gate_mode != kGateLog ? expf(p.A_log[h]) : 0.f;
    const float bias = (p.gate_mode != kGateLog && p.dt_bias) ? p.dt_bias[(long long)h * DK + lane] : 0.f;

    // thread (row r = tid / 4, quarter qq = tid % 4): 16-byte piece qq of its q, k and g rows
    // and DVR / 32 pieces of its v row; thread r < 16 also loads token r's beta into braw
    float braw = 0.f;
    auto issue = [&](int mc) {
        const long long t0 = bos + (long long)mc * CW;
        const int L = (int)min((long long)CW, eos - t0);
        const int r = tid >> 2, qq = tid & 3;
        const bool ok = r < L;
        const long long row = (t0 + (ok ? r : 0)) * H + h;
        const uint32_t in = (mc & 1) * Ly::IN, o = in + (r * DK + 8 * qq) * 2;
        cp16z(sm + Ly::Q + o, qg + row * DK + 8 * qq, ok);
        cp16z(sm + Ly::K + o, kg + row * DK + 8 * qq, ok);
        cp16z(sm + Ly::G + o, gg + row * DK + 8 * qq, ok);
        constexpr int VP = DVR / 32;
#pragma unroll
        for (int cc = 0; cc < VP; ++cc) {
            const int piece = VP * qq + cc;
            cp16z(sm + in + Ly::V + (r * LV + VOFF + 8 * piece) * 2, vg + row * DVR + 8 * piece, ok);
        }
        braw = tid < L ? __bfloat162float(betag[(t0 + tid) * H + h]) : 0.f;
        cp_async_commit();
    };

    // S^T, own value columns: rows (values) VW w + 16 mt + g8 (+ 8), columns (keys) 8 nk + 2 t4 (+ 1)
    float ST[MT][4][4];
    const long long sbase = ((long long)n * H + h) * DK * DV;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int nk = 0; nk < 4; ++nk)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int v = VW * w + 16 * mt + g8 + 8 * (i >> 1), c = 8 * nk + 2 * t4 + (i & 1);
                ST[mt][nk][i] = AUG ? (c == v ? 1.f : 0.f) : p.S0 ? p.S0[sbase + (long long)c * DV + v] : 0.f;
            }
    if constexpr (AUG) {  // the identity block sees v = 0: its columns of both v tiles stay zero
        const uint32_t z = ((tid >> 2) * LV + 8 * (tid & 3)) * 2;
        sts128(sm, Ly::V + z, make_uint4(0u, 0u, 0u, 0u));
        sts128(sm, Ly::IN + Ly::V + z, make_uint4(0u, 0u, 0u, 0u));
    }
    // A fragment of S^T (bf16) for own value m-tile mt and key step kk
    auto sfrag = [&](int mt, int kk, uint32_t (&a)[4]) {
        a[0] = pack_bf16x2(ST[mt][2 * kk][0], ST[mt][2 * kk][1]);
        a[1] = pack_bf16x2(ST[mt][2 * kk][2], ST[mt][2 * kk][3]);
        a[2] = pack_bf16x2(ST[mt][2 * kk + 1][0], ST[mt][2 * kk + 1][1]);
        a[3] = pack_bf16x2(ST[mt][2 * kk + 1][2], ST[mt][2 * kk + 1][3]);
    };

    if (nmc > 0) issue(0);
    for (int mc = 0; mc < nmc; ++mc) {
        const long long t0 = bos + (long long)mc * CW;
        const int L = (int)min((long long)CW, eos - t0);
        const float bcur = braw;
        const uint32_t in = (mc & 1) * Ly::IN;
        cp_async_wait_all();
        __syncthreads();  // this micro-chunk's rows, from both warps' copies
        // ---- gate values of rows 8 w .. 8 w + 7 for channel `lane` and their running sum
        // (this warp's total to XG); row norms (thread pair per row: rows 0..15 of k, then
        // of q; 16 channels each) and write strengths
        float G8[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int r = 8 * w + u;
            const float x = __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(sm + in + Ly::G)[r * DK + lane]);
            const float gv = p.gate_mode == kGateLog ? (p.has_lb ? fmaxf(x, p.lb) : x)
                                                     : gate_fast(x, bias, rate, p.gate_mode, p.lb);
            G8[u] = r < L ? gv : 0.f;
        }
#pragma unroll
        for (int u = 1; u < 8; ++u) G8[u] += G8[u - 1];
        XG[w * DK + lane] = G8[7];
        {
            const int rr = tid >> 1, half = tid & 1, r = rr & 15;
            const uint32_t row = in + (rr < 16 ? Ly::K : Ly::Q) + r * DK * 2 + 32 * half;
            float s = 0.f;
#pragma unroll
            for (int c8 = 0; c8 < 2; ++c8) {
                float f[8];
                unpack8(lds128(sm, row + 16 * c8), f);
#pragma unroll
                for (int e = 0; e < 8; ++e) s = fmaf(f[e], f[e], s);
            }
            s += __shfl_xor_sync(0xffffffffu, s, 1);
            const float inv = r < L ? (p.use_l2 ? rsqrtf(s + 1e-6f) : 1.f) : 0.f;
            if (half == 0) (rr < 16 ? rk : rq)[r] = inv;
            if (tid < CW) bb[tid] = tid < L ? beta_value(bcur, p.beta_prob) : 0.f;
        }
        __syncthreads();
        // ---- the in-chunk cumsum of channel `lane` on rows 8 w .. 8 w + 7 (warp 1 adds warp
        // 0's total G_7); operand tiles, those rows of row `lane` of each transposed tile
        const float Gm = XG[lane];
        if (w) {
#pragma unroll
            for (int u = 0; u < 8; ++u) G8[u] += Gm;
        }
        const float GC = w ? G8[7] : Gm + XG[DK + lane];
        bool steep = false;
        {
            const __nv_bfloat16 *kr = reinterpret_cast<const __nv_bfloat16 *>(sm + in + Ly::K);
            const __nv_bfloat16 *qr = reinterpret_cast<const __nv_bfloat16 *>(sm + in + Ly::Q);
            const float4 rka = *reinterpret_cast<const float4 *>(rk + 8 * w), rkb = *reinterpret_cast<const float4 *>(rk + 8 * w + 4);
            const float4 rqa = *reinterpret_cast<const float4 *>(rq + 8 * w), rqb = *reinterpret_cast<const float4 *>(rq + 8 * w + 4);
            const float rkv[8] = {rka.x, rka.y, rka.z, rka.w, rkb.x, rkb.y, rkb.z, rkb.w};
            const float rqv[8] = {rqa.x, rqa.y, rqa.z, rqa.w, rqb.x, rqb.y, rqb.z, rqb.w};
            float x[8], y[8], xq[8], kt[8], qt[8], kc[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int r = 8 * w + u;
                const float kh = __bfloat162float(kr[r * DK + lane]) * rkv[u];
                const float qh = __bfloat162float(qr[r * DK + lane]) * rqv[u];
                const float dm = G8[u] - Gm;
                steep |= fabsf(dm) > kSpan;
                const float em = e2(dm), en = e2(-dm), eg = e2(G8[u]), ec = e2(GC - G8[u]);
                x[u] = kh * em; y[u] = kh * en; xq[u] = qh * em;
                kt[u] = kh * eg; qt[u] = qh * eg; kc[u] = kh * ec;
            }
            const uint32_t o = (lane * LT + 8 * w) * 2;
            sts128(sm, Ly::X + o, pack8(x));
            sts128(sm, Ly::Y + o, pack8(y));
            sts128(sm, Ly::XQ + o, pack8(xq));
            sts128(sm, Ly::KT + o, pack8(kt));
            sts128(sm, Ly::QT + o, pack8(qt));
            sts128(sm, Ly::KH + o, pack8(kc));
            if (w == 0) gam[lane] = e2(GC);
        }
        steep = __syncthreads_or(steep) != 0;
        // the next micro-chunk's rows into the other stage (last read before the previous
        // micro-chunk's sixth barrier, its O staging copied out before this one's first);
        // issued here rather than at the top of the step, where they would queue ahead of
        // this step's first shared-memory reads
        if (mc + 1 < nmc) issue(mc + 1);
        // ---- A_kk (warp 0) -> L = diag(b) A_kk (s < r); A_qk (warp 1) -> bf16 tile (s <= r)
        {
            float acc[2][4] = {};
            const uint32_t xa = w == 0 ? Ly::X : Ly::XQ;
#pragma unroll
            for (int k0 = 0; k0 < DK; k0 += 16) {
                uint32_t a[4], bf[4];
                frag_at(sb + xa, LT, 0, k0, lane, a);
                frag_bt(sb + Ly::Y, LT, 0, k0, lane, bf);
                mma16816(acc[0], a, bf[0], bf[1]);
                mma16816(acc[1], a, bf[2], bf[3]);
            }
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int hi = 0; hi < 2; ++hi) {
                    const int r = g8 + 8 * hi, s_ = 8 * j + 2 * t4;
                    if (w == 0) {
                        const float br = bb[r];
                        *reinterpret_cast<float2 *>(Lf + r * LL + s_) = make_float2(
                            s_ < r ? br * acc[j][2 * hi] : 0.f, s_ + 1 < r ? br * acc[j][2 * hi + 1] : 0.f);
                    } else {
                        stb2(sm + Ly::AQ + (r * LT + s_) * 2, s_ <= r ? acc[j][2 * hi] : 0.f,
                             s_ + 1 <= r ? acc[j][2 * hi + 1] : 0.f);
                    }
                }
        }
        if (steep) {  // exponent differences (never positive) on the CUDA cores
            __syncthreads();  // X^T and Y^T are read by both warps: the scratch goes over them
            float *Gs = reinterpret_cast<float *>(sm + Ly::X);
#pragma unroll
            for (int u = 0; u < 8; ++u) Gs[(8 * w + u) * 33 + lane] = G8[u];
            __syncthreads();
            const __nv_bfloat16 *kr = reinterpret_cast<const __nv_bfloat16 *>(sm + in + Ly::K);
            const __nv_bfloat16 *qr = reinterpret_cast<const __nv_bfloat16 *>(sm + in + Ly::Q);
            for (int e = tid; e < CW * CW; e += 64) {
                const int r = e >> 4, s_ = e & 15;
                if (s_ > r) continue;
                float akk = 0.f, aqk = 0.f;
                for (int c = 0; c < DK; ++c) {
                    const float ed = expf(Gs[r * 33 + c] - Gs[s_ * 33 + c]);
                    const float ks = __bfloat162float(kr[s_ * DK + c]) * ed;
                    akk = fmaf(__bfloat162float(kr[r * DK + c]), ks, akk);
                    aqk = fmaf(__bfloat162float(qr[r * DK + c]), ks, aqk);
                }
                akk *= rk[r] * rk[s_];
                aqk *= rq[r] * rk[s_];
                if (s_ < r) Lf[r * LL + s_] = bb[r] * akk;
                reinterpret_cast<__nv_bfloat16 *>(sm + Ly::AQ)[r * LT + s_] = __float2bfloat16_rn(aqk);
            }
        }
        __syncthreads();
        // ---- T = (I + L)^-1 by forward substitution (warp 0, lane j < 16: column j, a row of
        // L four values at a time); row j of T'^T = column j of T diag(b) (two 16-byte stores)
        if (w == 0 && lane < CW) {
            const int j = lane;
            float t[CW];
#pragma unroll
            for (int i = 0; i < CW; ++i) {
                float acc = i == j ? 1.f : 0.f;
#pragma unroll
                for (int k4 = 0; k4 < i; k4 += 4) {
                    const float4 l4 = *reinterpret_cast<const float4 *>(Lf + i * LL + k4);
                    acc = fmaf(-l4.x, t[k4], acc);
                    if (k4 + 1 < i) acc = fmaf(-l4.y, t[k4 + 1], acc);
                    if (k4 + 2 < i) acc = fmaf(-l4.z, t[k4 + 2], acc);
                    if (k4 + 3 < i) acc = fmaf(-l4.w, t[k4 + 3], acc);
                }
                t[i] = acc;
            }
            const float bj = bb[j];
#pragma unroll
            for (int i = 0; i < CW; ++i) t[i] *= bj;
            sts128(sm, Ly::TP + (j * LT) * 2, pack8(t));
            sts128(sm, Ly::TP + (j * LT + 8) * 2, pack8(t + 8));
        }
        // ---- O^T = S^T Qtil^T for own value columns (warp 1 while the inverse runs)
        float OT[MT][2][4];
        {
            uint32_t bq[2][4];
            frag_bt(sb + Ly::QT, LT, 0, 0, lane, bq[0]);
            frag_bt(sb + Ly::QT, LT, 0, 16, lane, bq[1]);
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
#pragma unroll
                for (int i = 0; i < 4; ++i) OT[mt][0][i] = OT[mt][1][i] = 0.f;
#pragma unroll
                for (int kk = 0; kk < 2; ++kk) {
                    uint32_t a[4];
                    sfrag(mt, kk, a);
                    mma16816(OT[mt][0], a, bq[kk][0], bq[kk][1]);
                    mma16816(OT[mt][1], a, bq[kk][2], bq[kk][3]);
                }
            }
        }
        __syncthreads();  // T'
        // ---- U^T = V^T T'^T (own value columns); -W = -T' Ktil for key channels [16 w, 16 w + 16)
        float UT[MT][2][4];
        {
            uint32_t bt[4];
            frag_bt(sb + Ly::TP, LT, 0, 0, lane, bt);
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                uint32_t a[4];
                frag_at(sb + in + Ly::V, LV, VW * w + 16 * mt, 0, lane, a);
#pragma unroll
                for (int i = 0; i < 4; ++i) UT[mt][0][i] = UT[mt][1][i] = 0.f;
                mma16816(UT[mt][0], a, bt[0], bt[1]);
                mma16816(UT[mt][1], a, bt[2], bt[3]);
            }
            if constexpr (SAVE) {  // own columns of the entering state S (bf16 [32][DV]), 16 key rows at a time
                __syncwarp();  // own v columns are read: they stage the rows
                const long long slot = (bos >> 4) + n + mc;
#pragma unroll
                for (int kh = 0; kh < 2; ++kh) {
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt)  // matrix mi: key n-tile 2 kh + mi / 2, value half mi % 2
                        stsm4t(sb + in + Ly::V + ((8 * (mi >> 1) + mr) * LV + VW * w + 16 * mt + 8 * (mi & 1)) * 2,
                               pack_bf16x2(ST[mt][2 * kh][0], ST[mt][2 * kh][1]),
                               pack_bf16x2(ST[mt][2 * kh][2], ST[mt][2 * kh][3]),
                               pack_bf16x2(ST[mt][2 * kh + 1][0], ST[mt][2 * kh + 1][1]),
                               pack_bf16x2(ST[mt][2 * kh + 1][2], ST[mt][2 * kh + 1][3]));
                    __syncwarp();
                    constexpr int PR = VW / 8;
#pragma unroll
                    for (int q = lane; q < CW * PR; q += 32) {
                        const int r = q / PR, c = q % PR;
                        *reinterpret_cast<uint4 *>(save + ((slot * H + h) * DK + 16 * kh + r) * DV + VW * w + 8 * c) =
                            lds128(sm, in + Ly::V + (r * LV + VW * w + 8 * c) * 2);
                    }
                    __syncwarp();
                }
            }
            uint32_t a[4], bf[4];
            frag_at(sb + Ly::TP, LT, 0, 0, lane, a);
            frag_b(sb + Ly::KT, LT, 16 * w, 0, lane, bf);
            float wv[2][4] = {};
            mma16816(wv[0], a, bf[0], bf[1]);
            mma16816(wv[1], a, bf[2], bf[3]);
            // matrix mi: row half mi % 2, key n-tile 2 w + mi / 2
            stsm4(sb + Ly::W + ((8 * (mi & 1) + mr) * LK + 16 * w + 8 * (mi >> 1)) * 2,
                  pack_bf16x2(-wv[0][0], -wv[0][1]), pack_bf16x2(-wv[0][2], -wv[0][3]),
                  pack_bf16x2(-wv[1][0], -wv[1][1]), pack_bf16x2(-wv[1][2], -wv[1][3]));
        }
        __syncthreads();  // -W complete
        // ---- D^T = U^T + S^T (-W)^T (own value columns), as bf16 A fragments over the tokens
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
            uint32_t bw[4];
            frag_b(sb + Ly::W, LK, 0, 16 * kk, lane, bw);
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                uint32_t a[4];
                sfrag(mt, kk, a);
                mma16816(UT[mt][0], a, bw[0], bw[1]);
                mma16816(UT[mt][1], a, bw[2], bw[3]);
            }
        }
        uint32_t DA[MT][4];
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            DA[mt][0] = pack_bf16x2(UT[mt][0][0], UT[mt][0][1]);
            DA[mt][1] = pack_bf16x2(UT[mt][0][2], UT[mt][0][3]);
            DA[mt][2] = pack_bf16x2(UT[mt][1][0], UT[mt][1][1]);
            DA[mt][3] = pack_bf16x2(UT[mt][1][2], UT[mt][1][3]);
        }
        // ---- O^T += D^T A_qk^T; out through the staging tile over this stage's own v columns
        // (rows = tokens), or in fp32 rows of DV (AUG)
        {
            uint32_t baq[4];
            frag_b(sb + Ly::AQ, LT, 0, 0, lane, baq);
            const float f = p.scale;
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                mma16816(OT[mt][0], DA[mt], baq[0], baq[1]);
                mma16816(OT[mt][1], DA[mt], baq[2], baq[3]);
                if constexpr (AUG) {
                    if (p.o) {
#pragma unroll
                        for (int nr = 0; nr < 2; ++nr)
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                const int r = 8 * nr + 2 * t4 + (i & 1), v = VW * w + 16 * mt + g8 + 8 * (i >> 1);
                                if (r < L) static_cast<float *>(p.o)[((t0 + r) * H + h) * DV + v] = f * OT[mt][nr][i];
                            }
                    }
                } else {  // matrix mi: token rows 8 (mi / 2) + mr, value columns VW w + 16 mt + 8 (mi % 2)
                    stsm4t(sb + in + Ly::V + ((8 * (mi >> 1) + mr) * LV + VW * w + 16 * mt + 8 * (mi & 1)) * 2,
                           pack_bf16x2(f * OT[mt][0][0], f * OT[mt][0][1]), pack_bf16x2(f * OT[mt][0][2], f * OT[mt][0][3]),
                           pack_bf16x2(f * OT[mt][1][0], f * OT[mt][1][1]), pack_bf16x2(f * OT[mt][1][2], f * OT[mt][1][3]));
                }
            }
        }
        // ---- S^T <- S^T diag(e^{G_last}) + D^T Khat (own value columns)
#pragma unroll
        for (int nk = 0; nk < 4; ++nk) {
            const float2 gk = *reinterpret_cast<const float2 *>(gam + 8 * nk + 2 * t4);
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                ST[mt][nk][0] *= gk.x; ST[mt][nk][1] *= gk.y;
                ST[mt][nk][2] *= gk.x; ST[mt][nk][3] *= gk.y;
            }
        }
#pragma unroll
        for (int nk = 0; nk < 4; nk += 2) {
            uint32_t bk[4];
            frag_b(sb + Ly::KH, LT, 8 * nk, 0, lane, bk);
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                mma16816(ST[mt][nk], DA[mt], bk[0], bk[1]);
                mma16816(ST[mt][nk + 1], DA[mt], bk[2], bk[3]);
            }
        }
        if (!AUG && p.o) {  // rows < L of the staged O, own columns, 16 bytes per lane and step
            __syncwarp();
            constexpr int PR = VW / 8;
#pragma unroll
            for (int q = lane; q < CW * PR; q += 32) {
                const int r = q / PR, c = q % PR;
                if (r < L)
                    *reinterpret_cast<uint4 *>(og + ((t0 + r) * H + h) * DV + VW * w + 8 * c) =
                        lds128(sm, in + Ly::V + (r * LV + VW * w + 8 * c) * 2);
            }
        }
        // no barrier here: every shared tile the next micro-chunk writes before its third
        // barrier was last read before this one's sixth (the O staging is this warp's own)
    }
    cp_async_wait_all();
    if (p.S_out) {
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int nk = 0; nk < 4; ++nk)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int v = VW * w + 16 * mt + g8 + 8 * (i >> 1), c = 8 * nk + 2 * t4 + (i & 1);
                    p.S_out[sbase + (long long)c * DV + v] = ST[mt][nk][i];
                }
    }
}

template <int DV, bool AUG = false, bool SAVE = false>
cudaError_t launch_t(const ChunkParams &p, cudaStream_t st, __nv_bfloat16 *save = nullptr) {
    const long long chains = (long long)p.N * p.H;
    if (chains <= 0) return cudaSuccess;
    const uint32_t smem = Lay<DV>::BYTES;
    cudaError_t e = cudaFuncSetAttribute(kda_chunk_pair_kernel<DV, AUG, SAVE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    count_launch();
    kda_chunk_pair_kernel<DV, AUG, SAVE><<<(unsigned)chains, 64, smem, st>>>(p, save);
    return cudaGetLastError();
}
}  // namespace w2


// ---- d_k = 32 on a producer warp and a consumer warp per chain (one 64-thread CTA).
// Warp 0 forms, micro-chunk after micro-chunk, everything that does not depend on the
// state -- the gate and its cumsum, the row norms, the operand tiles, A_kk and A_qk, the
// inverse and -W -- and hands Qtil^T, Khat^T, A_qk, T'^T, -W and e^{G_last} to warp 1
// through one of two buffers, then goes on with the next micro-chunk. Warp 1 holds S^T
// (d_v x 32, fp32) in accumulator registers and runs the state chain:
//   U^T = V^T T'^T,  D^T = U^T + S^T (-W)^T,  O^T = S^T Qtil^T + D^T A_qk^T,
//   S^T <- S^T diag(e^{G_last}) + D^T Khat.
// Held transposed, S^T and D^T are A operands of the next products as they stand (two
// adjacent 8-column accumulator tiles are one 16-wide A fragment), so neither goes
// through shared memory; O^T leaves through transposing matrix stores. Hand-off: named
// barrier 1 + b (buffer b full: the producer arrives, the consumer waits) and 3 + b
// (buffer b free again), 64 threads each. AUG as in w2. save (or null): the state entering
// every micro-chunk, bf16 [32][d_v], at save + ((slot * H + h) * 32 + row) * d_v with
// slot = bos / 16 + n + micro-chunk (distinct across sequences: sequence n's slots end
// before bos_{n+1} / 16 + n + 1); read by the micro-chunk backward.
namespace pc {
template <int DV>
struct Lay {
    static constexpr int LV = DV + 8;                           // v stage / output staging row
    static constexpr uint32_t QKG = 3 * CW * DK * 2;            // one q, k, g stage
    static constexpr uint32_t Q = 0, K = CW * DK * 2, G = 2 * CW * DK * 2;
    static constexpr uint32_t VS = 2 * QKG, VSZ = CW * LV * 2;  // two v stages [16][LV]
    static constexpr uint32_t TT = DK * LT * 2;                 // a transposed tile [32][LT]
    static constexpr uint32_t X = VS + 2 * VSZ, Y = X + TT, XQ = Y + TT, KT = XQ + TT;
    static constexpr uint32_t L = KT + TT;                      // f32 [16][LL]
    static constexpr uint32_t RK = L + CW * LL * 4, RQ = RK + 64, BB = RQ + 64;
    // hand-off buffer b at HB + b HSZ: Qtil^T [32][LT], Khat^T [32][LT], A_qk [16][LT],
    // T'^T [16][LT], -W [16][LK], e^{G_last} [32]
    static constexpr uint32_t HB = BB + 64;
    static constexpr uint32_t HQT = 0, HKH = TT, HAQ = 2 * TT, HTP = HAQ + CW * LT * 2, HW = HTP + CW * LT * 2,
                              HGAM = HW + CW * LK * 2, HSZ = HGAM + DK * 4;
    static constexpr uint32_t BYTES = HB + 2 * HSZ;
    static_assert(CW * 33 * 4 <= 2 * TT, "exponent scratch over X^T and Y^T");
    static_assert(VSZ % 16 == 0 && L % 16 == 0 && RK % 16 == 0 && HB % 16 == 0 && HSZ % 16 == 0, "alignment");
};

template <int DV, bool AUG>
__global__ void __maxnreg__(144) kda_chunk_pc_kernel(const ChunkParams p, __nv_bfloat16 *save) {
    using Ly = Lay<DV>;
    constexpr int LV = Ly::LV, MT = DV / 16;  // value m-tiles of S^T
    constexpr int VOFF = AUG ? DK : 0, DVR = DV - VOFF;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const long long chain = blockIdx.x;
    const int n = (int)(chain / p.H), h = (int)(chain % p.H);
    uint8_t *sm = smem_raw;
    const uint32_t sb = sm100::smem_u32(sm);
    const int H = p.H, g8 = lane >> 2, t4 = lane & 3;
    long long bos, eos;
    if (p.cu_seqlens) { bos = p.cu_seqlens[n]; eos = p.cu_seqlens[n + 1]; }
    else { bos = (long long)n * p.T; eos = bos + p.T; }
    const int nmc = (int)((eos - bos + CW - 1) / CW);

    if (warp == 0) {
        // ================= producer: lane = key channel for the gate and the operand tiles
        const __nv_bfloat16 *qg = static_cast<const __nv_bfloat16 *>(p.q), *kg = static_cast<const __nv_bfloat16 *>(p.k);
        const __nv_bfloat16 *gg = static_cast<const __nv_bfloat16 *>(p.g);
        const __nv_bfloat16 *betag = static_cast<const __nv_bfloat16 *>(p.beta);
        float *rk = reinterpret_cast<float *>(sm + Ly::RK), *rq = reinterpret_cast<float *>(sm + Ly::RQ);
        float *bb = reinterpret_cast<float *>(sm + Ly::BB), *Lf = reinterpret_cast<float *>(sm + Ly::L);
        const float rate = p.gate_mode != kGateLog ? expf(p.A_log[h]) : 0.f;
        const float bias = (p.gate_mode != kGateLog && p.dt_bias) ? p.dt_bias[(long long)h * DK + lane] : 0.f;
        // q, k, g rows of micro-chunk mc into stage mc % 2 (lane: row lane / 2, half lane % 2);
        // lane r < 16 also loads token r's beta into braw (used one micro-chunk later)
        float braw = 0.f;
        auto issue = [&](int mc) {
            const long long t0 = bos + (long long)mc * CW;
            const int L = (int)min((long long)CW, eos - t0);
            const int r = lane >> 1, hf = lane & 1;
            const bool ok = r < L;
            const long long row = (t0 + (ok ? r : 0)) * H + h;
            const uint32_t o = (mc & 1) * Ly::QKG + (r * DK + 16 * hf) * 2;
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                cp16z(sm + Ly::Q + o + 16 * c, qg + row * DK + 16 * hf + 8 * c, ok);
                cp16z(sm + Ly::K + o + 16 * c, kg + row * DK + 16 * hf + 8 * c, ok);
                cp16z(sm + Ly::G + o + 16 * c, gg + row * DK + 16 * hf + 8 * c, ok);
            }
            braw = lane < L ? __bfloat162float(betag[(t0 + lane) * H + h]) : 0.f;
            cp_async_commit();
        };
        if (nmc > 0) issue(0);
        for (int mc = 0; mc < nmc; ++mc) {
            const long long t0 = bos + (long long)mc * CW;
            const int L = (int)min((long long)CW, eos - t0);
            const float bcur = braw;
            const uint32_t st = (mc & 1) * Ly::QKG;
            const int b = mc & 1;
            const uint32_t hb = Ly::HB + b * Ly::HSZ;
            cp_async_wait_all();
            __syncwarp();
            // gate and its cumsum
            float G[CW];
#pragma unroll
            for (int r = 0; r < CW; ++r) {
                const float x = __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(sm + st + Ly::G)[r * DK + lane]);
                const float gv = p.gate_mode == kGateLog ? (p.has_lb ? fmaxf(x, p.lb) : x)
                                                         : gate_fast(x, bias, rate, p.gate_mode, p.lb);
                G[r] = r < L ? gv : 0.f;
            }
#pragma unroll
            for (int r = 1; r < CW; ++r) G[r] += G[r - 1];
            // row norms (lanes 0..15: k rows, 16..31: q rows) and write strengths
            {
                const int r = lane & 15;
                const uint32_t row = st + (lane < 16 ? Ly::K : Ly::Q) + r * DK * 2;
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
                    bb[r] = r < L ? beta_value(bcur, p.beta_prob) : 0.f;
                } else {
                    rq[r] = inv;
                }
            }
            __syncwarp();
            if (mc >= 2) {  // hand-off buffer b read by the consumer (micro-chunk mc - 2)
                if (b == 0) sm100::bar_sync(3, 64); else sm100::bar_sync(4, 64);
            }
            // operand tiles, row `lane` of each transposed tile: X = k^ e^{G-M}, Y = k^ e^{M-G},
            // XQ = q^ e^{G-M}, KT = k^ e^G (own); QT = q^ e^G, KH = k^ e^{G_last-G} (hand-off)
            const float Gm = G[7], GC = G[CW - 1];
            bool steep = false;
            {
                const __nv_bfloat16 *kr = reinterpret_cast<const __nv_bfloat16 *>(sm + st + Ly::K);
                const __nv_bfloat16 *qr = reinterpret_cast<const __nv_bfloat16 *>(sm + st + Ly::Q);
#pragma unroll
                for (int h8 = 0; h8 < 2; ++h8) {
                    const float4 rka = *reinterpret_cast<const float4 *>(rk + 8 * h8);
                    const float4 rkb = *reinterpret_cast<const float4 *>(rk + 8 * h8 + 4);
                    const float4 rqa = *reinterpret_cast<const float4 *>(rq + 8 * h8);
                    const float4 rqb = *reinterpret_cast<const float4 *>(rq + 8 * h8 + 4);
                    const float rkv[8] = {rka.x, rka.y, rka.z, rka.w, rkb.x, rkb.y, rkb.z, rkb.w};
                    const float rqv[8] = {rqa.x, rqa.y, rqa.z, rqa.w, rqb.x, rqb.y, rqb.z, rqb.w};
                    float x[8], y[8], xq[8], kt[8], qt[8], kc[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const int r = 8 * h8 + u;
                        const float kh = __bfloat162float(kr[r * DK + lane]) * rkv[u];
                        const float qh = __bfloat162float(qr[r * DK + lane]) * rqv[u];
                        const float dm = G[r] - Gm;
                        steep |= fabsf(dm) > kSpan;
                        const float em = e2(dm), en = e2(-dm), eg = e2(G[r]), ec = e2(GC - G[r]);
                        x[u] = kh * em; y[u] = kh * en; xq[u] = qh * em;
                        kt[u] = kh * eg; qt[u] = qh * eg; kc[u] = kh * ec;
                    }
                    const uint32_t o = (lane * LT + 8 * h8) * 2;
                    sts128(sm, Ly::X + o, pack8(x));
                    sts128(sm, Ly::Y + o, pack8(y));
                    sts128(sm, Ly::XQ + o, pack8(xq));
                    sts128(sm, Ly::KT + o, pack8(kt));
                    sts128(sm, hb + Ly::HQT + o, pack8(qt));
                    sts128(sm, hb + Ly::HKH + o, pack8(kc));
                }
                reinterpret_cast<float *>(sm + hb + Ly::HGAM)[lane] = e2(GC);
            }
            steep = __any_sync(0xffffffffu, steep);
            if (mc + 1 < nmc) issue(mc + 1);  // into the other stage, read in the previous step
            __syncwarp();
            // A_kk (s < r) -> L = diag(b) A_kk (fp32), A_qk (s <= r) -> bf16 (hand-off)
            {
                float akk[2][4] = {}, aqk[2][4] = {};
#pragma unroll
                for (int k0 = 0; k0 < DK; k0 += 16) {
                    uint32_t a[4], aq[4], bf[4];
                    frag_at(sb + Ly::X, LT, 0, k0, lane, a);
                    frag_at(sb + Ly::XQ, LT, 0, k0, lane, aq);
                    frag_bt(sb + Ly::Y, LT, 0, k0, lane, bf);
                    mma16816(akk[0], a, bf[0], bf[1]);
                    mma16816(akk[1], a, bf[2], bf[3]);
                    mma16816(aqk[0], aq, bf[0], bf[1]);
                    mma16816(aqk[1], aq, bf[2], bf[3]);
                }
#pragma unroll
                for (int j = 0; j < 2; ++j)
#pragma unroll
                    for (int hi = 0; hi < 2; ++hi) {
                        const int r = g8 + 8 * hi, s_ = 8 * j + 2 * t4;
                        const float br = bb[r];
                        *reinterpret_cast<float2 *>(Lf + r * LL + s_) =
                            make_float2(s_ < r ? br * akk[j][2 * hi] : 0.f, s_ + 1 < r ? br * akk[j][2 * hi + 1] : 0.f);
                        stb2(sm + hb + Ly::HAQ + (r * LT + s_) * 2, s_ <= r ? aqk[j][2 * hi] : 0.f,
                             s_ + 1 <= r ? aqk[j][2 * hi + 1] : 0.f);
                    }
            }
            if (steep) {  // exponent differences (never positive) on the CUDA cores
                __syncwarp();  // X^T and Y^T are read: the scratch goes over them
                float *Gs = reinterpret_cast<float *>(sm + Ly::X);
#pragma unroll
                for (int r = 0; r < CW; ++r) Gs[r * 33 + lane] = G[r];
                __syncwarp();
                const __nv_bfloat16 *kr = reinterpret_cast<const __nv_bfloat16 *>(sm + st + Ly::K);
                const __nv_bfloat16 *qr = reinterpret_cast<const __nv_bfloat16 *>(sm + st + Ly::Q);
                for (int e = lane; e < CW * CW; e += 32) {
                    const int r = e >> 4, s_ = e & 15;
                    if (s_ > r) continue;
                    float akk = 0.f, aqk = 0.f;
                    for (int c = 0; c < DK; ++c) {
                        const float ed = expf(Gs[r * 33 + c] - Gs[s_ * 33 + c]);
                        const float ks = __bfloat162float(kr[s_ * DK + c]) * ed;
                        akk = fmaf(__bfloat162float(kr[r * DK + c]), ks, akk);
                        aqk = fmaf(__bfloat162float(qr[r * DK + c]), ks, aqk);
                    }
                    akk *= rk[r] * rk[s_];
                    aqk *= rq[r] * rk[s_];
                    if (s_ < r) Lf[r * LL + s_] = bb[r] * akk;
                    reinterpret_cast<__nv_bfloat16 *>(sm + hb + Ly::HAQ)[r * LT + s_] = __float2bfloat16_rn(aqk);
                }
            }
            __syncwarp();
            // T = (I + L)^-1 by forward substitution (lane j < 16: column j, a row of L four
            // values at a time); row j of T'^T = column j of T diag(b) (two 16-byte stores)
            if (lane < CW) {
                const int j = lane;
                float t[CW];
#pragma unroll
                for (int i = 0; i < CW; ++i) {
                    float acc = i == j ? 1.f : 0.f;
#pragma unroll
                    for (int k4 = 0; k4 < i; k4 += 4) {
                        const float4 l4 = *reinterpret_cast<const float4 *>(Lf + i * LL + k4);
                        acc = fmaf(-l4.x, t[k4], acc);
                        if (k4 + 1 < i) acc = fmaf(-l4.y, t[k4 + 1], acc);
                        if (k4 + 2 < i) acc = fmaf(-l4.z, t[k4 + 2], acc);
                        if (k4 + 3 < i) acc = fmaf(-l4.w, t[k4 + 3], acc);
                    }
                    t[i] = acc;
                }
                const float bj = bb[j];
#pragma unroll
                for (int i = 0; i < CW; ++i) t[i] *= bj;
                sts128(sm, hb + Ly::HTP + (j * LT) * 2, pack8(t));
                sts128(sm, hb + Ly::HTP + (j * LT + 8) * 2, pack8(t + 8));
            }
            __syncwarp();
            // -W = -T' Ktil (hand-off, [16][LK]) by matrix stores
            {
                uint32_t a[4];
                frag_at(sb + hb + Ly::HTP, LT, 0, 0, lane, a);
                float w[4][4] = {};
#pragma unroll
                for (int j = 0; j < 4; j += 2) {
                    uint32_t bf[4];
                    frag_b(sb + Ly::KT, LT, 8 * j, 0, lane, bf);
                    mma16816(w[j], a, bf[0], bf[1]);
                    mma16816(w[j + 1], a, bf[2], bf[3]);
                }
                const int i = lane >> 3;  // matrix i of a store: row half i & 1, n-tile jb + (i >> 1)
#pragma unroll
                for (int jb = 0; jb < 4; jb += 2)
                    stsm4(sb + hb + Ly::HW + ((8 * (i & 1) + (lane & 7)) * LK + 8 * (jb + (i >> 1))) * 2,
                          pack_bf16x2(-w[jb][0], -w[jb][1]), pack_bf16x2(-w[jb][2], -w[jb][3]),
                          pack_bf16x2(-w[jb + 1][0], -w[jb + 1][1]), pack_bf16x2(-w[jb + 1][2], -w[jb + 1][3]));
            }
            if (b == 0) sm100::bar_arrive(1, 64); else sm100::bar_arrive(2, 64);  // hand-off buffer b full
        }
        cp_async_wait_all();
    } else {
        // ================= consumer: S^T in accumulator registers
        const __nv_bfloat16 *vg = static_cast<const __nv_bfloat16 *>(p.v);
        __nv_bfloat16 *og = static_cast<__nv_bfloat16 *>(p.o);
        // S^T: rows (value channels) 16 mt + g8 (+ 8), columns (key channels) 8 nk + 2 t4 (+ 1)
        float ST[MT][4][4];
        const long long sbase = ((long long)n * H + h) * DK * DV;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int nk = 0; nk < 4; ++nk)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int v = 16 * mt + g8 + 8 * (i >> 1), c = 8 * nk + 2 * t4 + (i & 1);
                    ST[mt][nk][i] = AUG ? (c == v ? 1.f : 0.f) : p.S0 ? p.S0[sbase + (long long)c * DV + v] : 0.f;
                }
        // v rows of micro-chunk mc into v stage mc % 2 (lane: row lane / 2, half lane % 2)
        auto issue_v = [&](int mc) {
            const long long t0 = bos + (long long)mc * CW;
            const int L = (int)min((long long)CW, eos - t0);
            const int r = lane >> 1, hf = lane & 1;
            const bool ok = r < L;
            const long long row = (t0 + (ok ? r : 0)) * H + h;
            const uint32_t o = Ly::VS + (mc & 1) * Ly::VSZ + (r * LV + VOFF + (DVR / 2) * hf) * 2;
#pragma unroll
            for (int c = 0; c < DVR / 16; ++c) cp16z(sm + o + 16 * c, vg + row * DVR + (DVR / 2) * hf + 8 * c, ok);
            cp_async_commit();
        };
        if constexpr (AUG) {  // the identity block sees v = 0: its columns of both v stages stay zero
            const uint32_t z = Ly::VS + ((lane >> 1) * LV + 16 * (lane & 1)) * 2;
#pragma unroll
            for (int s2 = 0; s2 < 2; ++s2) {
                sts128(sm, z + s2 * Ly::VSZ, make_uint4(0u, 0u, 0u, 0u));
                sts128(sm, z + s2 * Ly::VSZ + 16, make_uint4(0u, 0u, 0u, 0u));
            }
        }
        // A fragment of S^T (bf16) for value m-tile mt and key step kk
        auto sfrag = [&](int mt, int kk, uint32_t (&a)[4]) {
            a[0] = pack_bf16x2(ST[mt][2 * kk][0], ST[mt][2 * kk][1]);
            a[1] = pack_bf16x2(ST[mt][2 * kk][2], ST[mt][2 * kk][3]);
            a[2] = pack_bf16x2(ST[mt][2 * kk + 1][0], ST[mt][2 * kk + 1][1]);
            a[3] = pack_bf16x2(ST[mt][2 * kk + 1][2], ST[mt][2 * kk + 1][3]);
        };
        const int mi = lane >> 3, mr = lane & 7;  // matrix and stored row of a matrix store
        if (nmc > 0) issue_v(0);
        for (int mc = 0; mc < nmc; ++mc) {
            const long long t0 = bos + (long long)mc * CW;
            const int L = (int)min((long long)CW, eos - t0);
            const int b = mc & 1;
            const uint32_t hb = Ly::HB + b * Ly::HSZ, vs = Ly::VS + b * Ly::VSZ;
            cp_async_wait_all();
            __syncwarp();
            if (b == 0) sm100::bar_sync(1, 64); else sm100::bar_sync(2, 64);  // hand-off buffer b full
            // U^T = V^T T'^T
            float UT[MT][2][4];
            {
                uint32_t bt[4];
                frag_bt(sb + hb + Ly::HTP, LT, 0, 0, lane, bt);
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    uint32_t a[4];
                    frag_at(sb + vs, LV, 16 * mt, 0, lane, a);
#pragma unroll
                    for (int i = 0; i < 4; ++i) UT[mt][0][i] = UT[mt][1][i] = 0.f;
                    mma16816(UT[mt][0], a, bt[0], bt[1]);
                    mma16816(UT[mt][1], a, bt[2], bt[3]);
                }
            }
            if (mc + 1 < nmc) issue_v(mc + 1);  // into the other stage, read in the previous step
            __syncwarp();  // v stage b is read: it stages the saved state and then O
            if (save) {  // the entering state S (bf16 [32][DV]), 16 key rows at a time
                const long long slot = (bos >> 4) + n + mc;
#pragma unroll
                for (int kh = 0; kh < 2; ++kh) {
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt)  // matrix mi: key n-tile 2 kh + mi / 2, value half mi % 2
                        stsm4t(sb + vs + ((8 * (mi >> 1) + mr) * LV + 16 * mt + 8 * (mi & 1)) * 2,
                               pack_bf16x2(ST[mt][2 * kh][0], ST[mt][2 * kh][1]),
                               pack_bf16x2(ST[mt][2 * kh][2], ST[mt][2 * kh][3]),
                               pack_bf16x2(ST[mt][2 * kh + 1][0], ST[mt][2 * kh + 1][1]),
                               pack_bf16x2(ST[mt][2 * kh + 1][2], ST[mt][2 * kh + 1][3]));
                    __syncwarp();
                    constexpr int PR = DV / 8;
#pragma unroll
                    for (int q = lane; q < CW * PR; q += 32) {
                        const int r = q / PR, c = q % PR;
                        *reinterpret_cast<uint4 *>(save + ((slot * H + h) * DK + 16 * kh + r) * DV + 8 * c) =
                            lds128(sm, vs + (r * LV + 8 * c) * 2);
                    }
                    __syncwarp();
                }
            }
            // D^T = U^T + S^T (-W)^T
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
                uint32_t bw[4];
                frag_b(sb + hb + Ly::HW, LK, 0, 16 * kk, lane, bw);
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    uint32_t a[4];
                    sfrag(mt, kk, a);
                    mma16816(UT[mt][0], a, bw[0], bw[1]);
                    mma16816(UT[mt][1], a, bw[2], bw[3]);
                }
            }
            // D^T as bf16 A fragments over the 16 tokens
            uint32_t DA[MT][4];
#pragma unroll
            for (int mt = 0; mt < MT; ++mt) {
                DA[mt][0] = pack_bf16x2(UT[mt][0][0], UT[mt][0][1]);
                DA[mt][1] = pack_bf16x2(UT[mt][0][2], UT[mt][0][3]);
                DA[mt][2] = pack_bf16x2(UT[mt][1][0], UT[mt][1][1]);
                DA[mt][3] = pack_bf16x2(UT[mt][1][2], UT[mt][1][3]);
            }
            // O^T = S^T Qtil^T + D^T A_qk^T, one value m-tile at a time, stored transposed
            // (rows = tokens) into the staging tile over v stage b
            {
                uint32_t bq[2][4], baq[4];
                frag_bt(sb + hb + Ly::HQT, LT, 0, 0, lane, bq[0]);
                frag_bt(sb + hb + Ly::HQT, LT, 0, 16, lane, bq[1]);
                frag_b(sb + hb + Ly::HAQ, LT, 0, 0, lane, baq);
                const float f = p.scale;
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    float OT[2][4] = {};
#pragma unroll
                    for (int kk = 0; kk < 2; ++kk) {
                        uint32_t a[4];
                        sfrag(mt, kk, a);
                        mma16816(OT[0], a, bq[kk][0], bq[kk][1]);
                        mma16816(OT[1], a, bq[kk][2], bq[kk][3]);
                    }
                    mma16816(OT[0], DA[mt], baq[0], baq[1]);
                    mma16816(OT[1], DA[mt], baq[2], baq[3]);
                    if constexpr (AUG) {  // fp32 rows of DV: element (value 16 mt + g8 (+8), token 8 nr + 2 t4 (+1))
                        if (p.o) {
#pragma unroll
                            for (int nr = 0; nr < 2; ++nr)
#pragma unroll
                                for (int i = 0; i < 4; ++i) {
                                    const int r = 8 * nr + 2 * t4 + (i & 1), v = 16 * mt + g8 + 8 * (i >> 1);
                                    if (r < L) static_cast<float *>(p.o)[((t0 + r) * H + h) * DV + v] = f * OT[nr][i];
                                }
                        }
                    } else {  // matrix mi = 2 nr + vh: stored rows = tokens 8 nr + mr, columns 16 mt + 8 vh
                        stsm4t(sb + vs + ((8 * (mi >> 1) + mr) * LV + 16 * mt + 8 * (mi & 1)) * 2,
                               pack_bf16x2(f * OT[0][0], f * OT[0][1]), pack_bf16x2(f * OT[0][2], f * OT[0][3]),
                               pack_bf16x2(f * OT[1][0], f * OT[1][1]), pack_bf16x2(f * OT[1][2], f * OT[1][3]));
                    }
                }
            }
            // S^T <- S^T diag(e^{G_last}) + D^T Khat
            {
                const float *gam = reinterpret_cast<const float *>(sm + hb + Ly::HGAM);
#pragma unroll
                for (int nk = 0; nk < 4; ++nk) {
                    const float2 gk = *reinterpret_cast<const float2 *>(gam + 8 * nk + 2 * t4);
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt) {
                        ST[mt][nk][0] *= gk.x; ST[mt][nk][1] *= gk.y;
                        ST[mt][nk][2] *= gk.x; ST[mt][nk][3] *= gk.y;
                    }
                }
#pragma unroll
                for (int nk = 0; nk < 4; nk += 2) {
                    uint32_t bk[4];
                    frag_b(sb + hb + Ly::HKH, LT, 8 * nk, 0, lane, bk);
#pragma unroll
                    for (int mt = 0; mt < MT; ++mt) {
                        mma16816(ST[mt][nk], DA[mt], bk[0], bk[1]);
                        mma16816(ST[mt][nk + 1], DA[mt], bk[2], bk[3]);
                    }
                }
            }
            __syncwarp();
            if (mc + 2 < nmc) {  // hand-off buffer b free (its next use: mc + 2)
                if (b == 0) sm100::bar_arrive(3, 64); else sm100::bar_arrive(4, 64);
            }
            if (!AUG && p.o) {  // rows < L of the staged O, 16 bytes per lane and step
                constexpr int PR = DV / 8;
#pragma unroll
                for (int q = lane; q < CW * PR; q += 32) {
                    const int r = q / PR, c = q % PR;
                    if (r < L)
                        *reinterpret_cast<uint4 *>(og + ((t0 + r) * H + h) * DV + 8 * c) = lds128(sm, vs + (r * LV + 8 * c) * 2);
                }
            }
            __syncwarp();  // the staging tile is read before the next v copies reuse the stage
        }
        cp_async_wait_all();
        if (p.S_out) {
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int nk = 0; nk < 4; ++nk)
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int v = 16 * mt + g8 + 8 * (i >> 1), c = 8 * nk + 2 * t4 + (i & 1);
                        p.S_out[sbase + (long long)c * DV + v] = ST[mt][nk][i];
                    }
        }
    }
}

template <int DV, bool AUG = false>
cudaError_t launch_t(const ChunkParams &p, cudaStream_t st, __nv_bfloat16 *save = nullptr) {
    const long long chains = (long long)p.N * p.H;
    if (chains <= 0) return cudaSuccess;
    const uint32_t smem = Lay<DV>::BYTES;
    cudaError_t e = cudaFuncSetAttribute(kda_chunk_pc_kernel<DV, AUG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    count_launch();
    kda_chunk_pc_kernel<DV, AUG><<<(unsigned)chains, 64, smem, st>>>(p, save);
    return cudaGetLastError();
}
}  // namespace pc

}  // namespace cw

bool chunk_warp_supported(bool bf16, int Dk, int Dv) { return bf16 && (Dk == 32 || Dk == 64) && (Dv == 32 || Dv == 64); }

// d_k = 32: the producer/consumer form for the log-decay gate while every SM holds at most
// four chains (latency per chain decides), the split form otherwise: with more chains, or
// with an in-kernel gate form (16 gate evaluations per lane and micro-chunk on the
// producer), the producer warp's serial key-side work would set the pace. B T2048 H8 d_k 32
// d_v 64, 10 calls, L2 flushed: log gate 128 chains 0.25 against 0.29 ms, 512 chains 0.30
// against 0.34 ms, 1,024 chains 0.57 against 0.47 ms; softplus gate 128 chains 0.35 against
// 0.31 ms, 1,024 chains 0.75 against 0.48 ms.
static bool pc_form(const ChunkParams &p) { return p.gate_mode == kGateLog && (long long)p.N * p.H <= 4LL * 148; }

cudaError_t launch_chunk_warp(const ChunkParams &p, int Dk, int Dv, cudaStream_t st) {
    if (Dk == 64) return Dv == 32 ? cw::w64::launch_t<32>(p, st) : cw::w64::launch_t<64>(p, st);
    if (pc_form(p)) return Dv == 32 ? cw::pc::launch_t<32>(p, st) : cw::pc::launch_t<64>(p, st);
    return Dv == 32 ? cw::w2::launch_t<32>(p, st) : cw::w2::launch_t<64>(p, st);
}

// The d_k = 32 forward saving every micro-chunk's entering state for the backward.
cudaError_t launch_chunk_warp_save(const ChunkParams &p, int Dv, __nv_bfloat16 *save, cudaStream_t st) {
    if (pc_form(p)) return Dv == 32 ? cw::pc::launch_t<32>(p, st, save) : cw::pc::launch_t<64>(p, st, save);
    return Dv == 32 ? cw::w2::launch_t<32, false, true>(p, st, save) : cw::w2::launch_t<64, false, true>(p, st, save);
}

// The widened run of the segment form for bf16 d_k = d_v = 32 (outputs fp32 rows of 64,
// final states [32][64]); q is the segment view.
cudaError_t launch_chunk_warp_widened(const ChunkParams &q, cudaStream_t st) {
    return pc_form(q) ? cw::pc::launch_t<64, true>(q, st) : cw::w2::launch_t<64, true>(q, st);
}

}  // namespace kda
