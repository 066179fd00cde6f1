// Chunk forward for bf16 inputs with d_k = 32 (d_v = 32 or 64) when there are many
// (sequence, head) chains: one warp per chain, the WY/UT chunk form on 16-token
// micro-chunks, every product a warp-level tensor-core MMA (m16n8k16, bf16 operands,
// fp32 accumulate) and the fp32 state in the warp's accumulator registers.
//
// The operator is the `chunk_kda` boundary of page "K3/kda/ops/api.py" (the token
// recurrence of page "atlas_core/kimi_k3/kda.rs"). The chunk form is exact for any
// chunk size -- grouping tokens changes the order of the arithmetic, not its value --
// and with 16 tokens the UT inverse is a 16 x 16 unit-triangular solve inside one
// warp, every product is one MMA tile high, and a 32 x d_v state fits in 64 registers
// per lane, so a chain needs no block barrier and no record. Per micro-chunk (G the
// in-chunk cumsum of the gate, k^, q^ the normalised rows, b the write strengths):
//   A_kk[r,s] = sum_c k^_rc k^_sc e^{G_rc - G_sc} (s < r),  A_qk likewise with q^ (s <= r)
//   T' = (I + diag(b) A_kk)^-1 diag(b),  U = T' V,  W = T' (k^ e^G)
//   D = U - W S,  O = scale ((q^ e^G) S + A_qk D),  S <- diag(e^{G_last}) S + (k^ e^{G_last - G})^T D.
// The gated products split e^{G_r - G_s} at the micro-chunk's middle row (both parts
// <= e^80 while the gate moves by at most 80 over half a micro-chunk); a micro-chunk
// whose gate moves further takes A_kk and A_qk from exponent differences on the CUDA
// cores. Lane = key channel for the gate, its cumsum and the operand tiles.
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
constexpr int LL = 17;      // row of the fp32 L tile
constexpr int NWARP = 4;    // chains per CTA
constexpr float kSpan = 80.f;  // largest |G - G_mid| of the split products

template <int DV>
struct Lay {
    static constexpr int LV = DV + 8;                      // padded row of [*][DV] bf16 tiles
    // two input stages (micro-chunk parity): raw q, k, g rows [16][32] (read by column or
    // whole rows: no padding) and v [16][LV]
    static constexpr uint32_t Q = 0, K = Q + CW * DK * 2, G = K + CW * DK * 2, V = G + CW * DK * 2;
    static constexpr uint32_t IN = (V + CW * LV * 2 + 127) / 128 * 128;
    static constexpr uint32_t B = 2 * IN;
    // the operand tiles, stored transposed ([32 channels][16 rows], rows of LT): X^T of
    // k^ e^{G-M} (later the -W tile, [16][LK]), Y^T of k^ e^{M-G}, XQ^T of q^ e^{G-M},
    // KT^T of k^ e^G, QT^T of q^ e^G, KH^T of k^ e^{G_last-G}
    static constexpr uint32_t TT = DK * LT * 2;
    static constexpr uint32_t X = B;
    static constexpr uint32_t Y = X + TT;
    static constexpr uint32_t XQ = Y + TT;
    static constexpr uint32_t D = Y;                         // D (bf16 [16][LV]) over Y and XQ
    static constexpr uint32_t KT = XQ + TT;
    static constexpr uint32_t QT = KT + TT;
    static constexpr uint32_t KH = QT + TT;
    static constexpr uint32_t TP = KH + TT;                  // T' [16][LT]
    static constexpr uint32_t AQ = TP + CW * LT * 2;         // A_qk [16][LT]
    static constexpr uint32_t S = AQ + CW * LT * 2;          // S (bf16 [32][LV]); exponent scratch G [16][33] f32
    static constexpr uint32_t L = S + DK * LV * 2;           // L = diag(b) A_kk, f32 [16][LL]
    static constexpr uint32_t RK = L + CW * LL * 4, RQ = RK + 64, BB = RQ + 64, GAM = BB + 64;
    static constexpr uint32_t BYTES = (GAM + DK * 4 + 127) / 128 * 128;
    static_assert(D + CW * LV * 2 <= KT && CW * LK * 2 <= TT && CW * 33 * 4 <= DK * LV * 2, "aliases");
};


// AUG: the widened run of the segment form (kda_chunk_rec.cu): the state is [M | N]
// (32 x DV, DV = 32 + d_v), the first 32 columns start from the identity and see v = 0,
// the others start from zero and see v; the outputs [scale M^T q^ | scale N^T q^] go
// out in fp32 as rows of DV and the final state as [32][DV].
// save (or null): the state entering every micro-chunk, bf16 [32][DV], at
// save + ((slot * H + h) * 32 + row) * DV with slot = bos / 16 + n + micro-chunk (distinct
// across sequences: sequence n's slots end before bos_{n+1} / 16 + n + 1); read by the
// micro-chunk backward.
template <int DV, bool AUG>
__global__ void __launch_bounds__(NWARP * 32, 2) kda_chunk_warp_kernel(const ChunkParams p, __nv_bfloat16 *save) {
    using Ly = Lay<DV>;
    constexpr int LV = Ly::LV, NVT = DV / 8;
    constexpr int VOFF = AUG ? DK : 0, DVR = DV - VOFF;  // v's columns in the state, and its width
    extern __shared__ __align__(16) uint8_t smem_raw[];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const long long chain = (long long)blockIdx.x * NWARP + warp;
    if (chain >= (long long)p.N * p.H) return;  // no block barriers below: the warps are independent
    const int n = (int)(chain / p.H), h = (int)(chain % p.H);
    uint8_t *sm = smem_raw + warp * Ly::BYTES;
    const uint32_t sb = sm100::smem_u32(sm);
    float *rk = reinterpret_cast<float *>(sm + Ly::RK), *rq = reinterpret_cast<float *>(sm + Ly::RQ);
    float *bb = reinterpret_cast<float *>(sm + Ly::BB), *gam = reinterpret_cast<float *>(sm + Ly::GAM);
    float *Lf = reinterpret_cast<float *>(sm + Ly::L);
    const int H = p.H, g8 = lane >> 2, t4 = lane & 3;
    long long bos, eos;
    if (p.cu_seqlens) { bos = p.cu_seqlens[n]; eos = p.cu_seqlens[n + 1]; }
    else { bos = (long long)n * p.T; eos = bos + p.T; }
    const int nmc = (int)((eos - bos + CW - 1) / CW);
    const __nv_bfloat16 *qg = static_cast<const __nv_bfloat16 *>(p.q), *kg = static_cast<const __nv_bfloat16 *>(p.k);
    const __nv_bfloat16 *gg = static_cast<const __nv_bfloat16 *>(p.g), *vg = static_cast<const __nv_bfloat16 *>(p.v);
    const __nv_bfloat16 *betag = static_cast<const __nv_bfloat16 *>(p.beta);
    __nv_bfloat16 *og = static_cast<__nv_bfloat16 *>(p.o);
    // in-kernel gate: rate and this lane's channel bias
    const float rate = p.gate_mode != kGateLog ? expf(p.A_log[h]) : 0.f;
    const float bias = (p.gate_mode != kGateLog && p.dt_bias) ? p.dt_bias[(long long)h * DK + lane] : 0.f;

    // raw rows of micro-chunk mc (rows past the sequence zero-filled) into input stage
    // mc % 2: q, k, g, v by cp.async; lane r < 16 also loads token r's beta into braw
    // (a register, used one micro-chunk later, so the load does not stall the warp)
    float braw = 0.f;
    // lane (row r = lane / 2, half hf = lane % 2): pieces hf*2, hf*2+1 of its q, k, g rows
    // and hf*DV/16 .. of its v row (16-byte pieces)
    auto issue = [&](int mc) {
        const long long t0 = bos + (long long)mc * CW;
        const int L = (int)min((long long)CW, eos - t0);
        const int r = lane >> 1, hf = lane & 1;
        const bool ok = r < L;
        const long long row = (t0 + (ok ? r : 0)) * H + h;
        const __nv_bfloat16 *qs = qg + row * DK + 16 * hf, *ks = kg + row * DK + 16 * hf, *gs = gg + row * DK + 16 * hf;
        const __nv_bfloat16 *vs = vg + row * DVR + (DVR / 2) * hf;
        const uint32_t in = (mc & 1) * Ly::IN;
        const uint32_t o = in + (r * DK + 16 * hf) * 2, ov = in + (r * LV + VOFF + (DVR / 2) * hf) * 2;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
            cp16z(sm + Ly::Q + o + 16 * c, qs + 8 * c, ok);
            cp16z(sm + Ly::K + o + 16 * c, ks + 8 * c, ok);
            cp16z(sm + Ly::G + o + 16 * c, gs + 8 * c, ok);
        }
#pragma unroll
        for (int c = 0; c < DVR / 16; ++c) cp16z(sm + Ly::V + ov + 16 * c, vs + 8 * c, ok);
        braw = lane < L ? __bfloat162float(betag[(t0 + lane) * H + h]) : 0.f;
        cp_async_commit();
    };

    // the state: rows c = 16 mk + g8 (+ 8), columns 8 j + 2 t4 (+ 1), in MMA accumulator layout
    float S[2][NVT][4];
    const long long sbase = ((long long)n * H + h) * DK * DV;
#pragma unroll
    for (int mk = 0; mk < 2; ++mk)
#pragma unroll
        for (int j = 0; j < NVT; ++j)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int c = 16 * mk + g8 + 8 * (i >> 1), v = 8 * j + 2 * t4 + (i & 1);
                S[mk][j][i] = AUG ? (c == v ? 1.f : 0.f) : p.S0 ? p.S0[sbase + (long long)c * DV + v] : 0.f;
            }
    if constexpr (AUG) {  // the identity block sees v = 0: its columns of both v tiles stay zero
        const uint32_t z = ((lane >> 1) * LV + 16 * (lane & 1)) * 2;
#pragma unroll
        for (int st2 = 0; st2 < 2; ++st2) {
            sts128(sm, st2 * Ly::IN + Ly::V + z, make_uint4(0u, 0u, 0u, 0u));
            sts128(sm, st2 * Ly::IN + Ly::V + z + 16, make_uint4(0u, 0u, 0u, 0u));
        }
    }

    if (nmc > 0) issue(0);
    for (int mc = 0; mc < nmc; ++mc) {
        const long long t0 = bos + (long long)mc * CW;
        const int L = (int)min((long long)CW, eos - t0);
        const float bcur = braw;  // beta of this micro-chunk's row `lane` (lane < 16)
        const uint32_t in = (mc & 1) * Ly::IN;
        if (mc + 1 < nmc) {  // the next micro-chunk's rows into the other stage, then wait for ours
            issue(mc + 1);
            cp_async_wait_group<1>();
        } else {
            cp_async_wait_all();
        }
        __syncwarp();
        // ---- gate and its in-chunk cumsum: lane = channel, G[r] for the 16 rows (the 16
        // gate values first, independently, then the running sum)
        float G[CW];
        {
#pragma unroll
            for (int r = 0; r < CW; ++r) {
                const float x = __bfloat162float(reinterpret_cast<const __nv_bfloat16 *>(sm + in + Ly::G)[r * DK + lane]);
                const float gv = p.gate_mode == kGateLog ? (p.has_lb ? fmaxf(x, p.lb) : x)
                                                         : gate_fast(x, bias, rate, p.gate_mode, p.lb);
                G[r] = r < L ? gv : 0.f;
            }
#pragma unroll
            for (int r = 1; r < CW; ++r) G[r] += G[r - 1];
        }
        // ---- row norms (lanes 0..15: k rows, 16..31: q rows) and write strengths
        {
            const int r = lane & 15;
            const uint32_t row = in + (lane < 16 ? Ly::K : Ly::Q) + r * DK * 2;
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
        // ---- operand tiles, row `lane` of each transposed tile (16 values = two 16-byte
        // stores): X = k^ e^{G-M}, Y = k^ e^{M-G}, XQ = q^ e^{G-M}, KT = k^ e^G,
        // QT = q^ e^G, KH = k^ e^{G_last-G}
        const float Gm = G[7], GC = G[CW - 1];
        bool steep = false;
        {
            const __nv_bfloat16 *kr = reinterpret_cast<const __nv_bfloat16 *>(sm + in + Ly::K);
            const __nv_bfloat16 *qr = reinterpret_cast<const __nv_bfloat16 *>(sm + in + Ly::Q);
#pragma unroll
            for (int h8 = 0; h8 < 2; ++h8) {
                float x[8], y[8], xq[8], kt[8], qt[8], kc[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int r = 8 * h8 + u;
                    const float kh = __bfloat162float(kr[r * DK + lane]) * rk[r];
                    const float qh = __bfloat162float(qr[r * DK + lane]) * rq[r];
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
                sts128(sm, Ly::QT + o, pack8(qt));
                sts128(sm, Ly::KH + o, pack8(kc));
            }
            gam[lane] = e2(GC);
        }
        steep = __any_sync(0xffffffffu, steep);
        __syncwarp();
        // ---- A_kk (s < r) -> L = diag(b) A_kk (fp32), A_qk (s <= r) -> bf16 tile
        {
            float akk[2][4] = {}, aqk[2][4] = {};
#pragma unroll
            for (int k0 = 0; k0 < DK; k0 += 16) {
                uint32_t a[4], aq[4], b[4];
                frag_at(sb + Ly::X, LT, 0, k0, lane, a);
                frag_at(sb + Ly::XQ, LT, 0, k0, lane, aq);
                frag_bt(sb + Ly::Y, LT, 0, k0, lane, b);
                mma16816(akk[0], a, b[0], b[1]);
                mma16816(akk[1], a, b[2], b[3]);
                mma16816(aqk[0], aq, b[0], b[1]);
                mma16816(aqk[1], aq, b[2], b[3]);
            }
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int hi = 0; hi < 2; ++hi) {
                    const int r = g8 + 8 * hi, s = 8 * j + 2 * t4;
                    const float br = bb[r];
                    Lf[r * LL + s] = s < r ? br * akk[j][2 * hi] : 0.f;
                    Lf[r * LL + s + 1] = s + 1 < r ? br * akk[j][2 * hi + 1] : 0.f;
                    stb2(sm + Ly::AQ + (r * LT + s) * 2, s <= r ? aqk[j][2 * hi] : 0.f,
                         s + 1 <= r ? aqk[j][2 * hi + 1] : 0.f);
                }
        }
        if (steep) {  // exponent differences (never positive) on the CUDA cores
            float *Gs = reinterpret_cast<float *>(sm + Ly::S);
#pragma unroll
            for (int r = 0; r < CW; ++r) Gs[r * 33 + lane] = G[r];
            __syncwarp();
            const __nv_bfloat16 *kr = reinterpret_cast<const __nv_bfloat16 *>(sm + in + Ly::K);
            const __nv_bfloat16 *qr = reinterpret_cast<const __nv_bfloat16 *>(sm + in + Ly::Q);
            for (int e = lane; e < CW * CW; e += 32) {
                const int r = e >> 4, s = e & 15;
                if (s > r) continue;
                float akk = 0.f, aqk = 0.f;
                for (int c = 0; c < DK; ++c) {
                    const float ed = expf(Gs[r * 33 + c] - Gs[s * 33 + c]);
                    const float ks = __bfloat162float(kr[s * DK + c]) * ed;
                    akk = fmaf(__bfloat162float(kr[r * DK + c]), ks, akk);
                    aqk = fmaf(__bfloat162float(qr[r * DK + c]), ks, aqk);
                }
                akk *= rk[r] * rk[s];
                aqk *= rq[r] * rk[s];
                if (s < r) Lf[r * LL + s] = bb[r] * akk;
                reinterpret_cast<__nv_bfloat16 *>(sm + Ly::AQ)[r * LT + s] = __float2bfloat16_rn(aqk);
            }
        }
        __syncwarp();
        // ---- T = (I + L)^-1 by forward substitution (lane j < 16: column j), T' = T diag(b)
        if (lane < CW) {
            const int j = lane;
            float t[CW];
#pragma unroll
            for (int i = 0; i < CW; ++i) {
                float acc = i == j ? 1.f : 0.f;
#pragma unroll
                for (int k = 0; k < i; ++k) acc = fmaf(-Lf[i * LL + k], t[k], acc);
                t[i] = acc;
            }
            const float bj = bb[j];
#pragma unroll
            for (int i = 0; i < CW; ++i)
                reinterpret_cast<__nv_bfloat16 *>(sm + Ly::TP)[i * LT + j] = __float2bfloat16_rn(t[i] * bj);
        }
        __syncwarp();
        // ---- U = T' V (registers), -W = -T' Ktil (bf16 tile over X)
        float U[NVT][4];
        {
            uint32_t a[4];
            frag_a(sb + Ly::TP, LT, 0, 0, lane, a);
#pragma unroll
            for (int j = 0; j < NVT; j += 2) {
                uint32_t b[4];
                frag_bt(sb + in + Ly::V, LV, 8 * j, 0, lane, b);
                U[j][0] = U[j][1] = U[j][2] = U[j][3] = 0.f;
                U[j + 1][0] = U[j + 1][1] = U[j + 1][2] = U[j + 1][3] = 0.f;
                mma16816(U[j], a, b[0], b[1]);
                mma16816(U[j + 1], a, b[2], b[3]);
            }
            float w[4][4] = {};
#pragma unroll
            for (int j = 0; j < 4; j += 2) {
                uint32_t b[4];
                frag_b(sb + Ly::KT, LT, 8 * j, 0, lane, b);
                mma16816(w[j], a, b[0], b[1]);
                mma16816(w[j + 1], a, b[2], b[3]);
            }
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int hi = 0; hi < 2; ++hi)
                    stb2(sm + Ly::X + ((g8 + 8 * hi) * LK + 8 * j + 2 * t4) * 2, -w[j][2 * hi], -w[j][2 * hi + 1]);
        }
        // the state as a bf16 operand
#pragma unroll
        for (int mk = 0; mk < 2; ++mk)
#pragma unroll
            for (int j = 0; j < NVT; ++j)
#pragma unroll
                for (int hi = 0; hi < 2; ++hi)
                    stb2(sm + Ly::S + ((16 * mk + g8 + 8 * hi) * LV + 8 * j + 2 * t4) * 2, S[mk][j][2 * hi],
                         S[mk][j][2 * hi + 1]);
        __syncwarp();
        if (save) {  // row `lane` of the entering state
            const long long slot = (bos >> 4) + n + mc;
            uint4 *dst = reinterpret_cast<uint4 *>(save + ((slot * H + h) * DK + lane) * DV);
#pragma unroll
            for (int q8 = 0; q8 < DV / 8; ++q8) dst[q8] = lds128(sm, Ly::S + (lane * LV + 8 * q8) * 2);
        }
        // ---- D = U - W S (in U's registers) -> bf16 tile
#pragma unroll
        for (int k0 = 0; k0 < DK; k0 += 16) {
            uint32_t a[4];
            frag_a(sb + Ly::X, LK, 0, k0, lane, a);
#pragma unroll
            for (int j = 0; j < NVT; j += 2) {
                uint32_t b[4];
                frag_bt(sb + Ly::S, LV, 8 * j, k0, lane, b);
                mma16816(U[j], a, b[0], b[1]);
                mma16816(U[j + 1], a, b[2], b[3]);
            }
        }
#pragma unroll
        for (int j = 0; j < NVT; ++j)
#pragma unroll
            for (int hi = 0; hi < 2; ++hi)
                stb2(sm + Ly::D + ((g8 + 8 * hi) * LV + 8 * j + 2 * t4) * 2, U[j][2 * hi], U[j][2 * hi + 1]);
        __syncwarp();
        // ---- O = scale ((q^ e^G) S + A_qk D), rows < L to o
        {
            float O[NVT][4];
#pragma unroll
            for (int j = 0; j < NVT; ++j) O[j][0] = O[j][1] = O[j][2] = O[j][3] = 0.f;
#pragma unroll
            for (int k0 = 0; k0 < DK; k0 += 16) {
                uint32_t a[4];
                frag_at(sb + Ly::QT, LT, 0, k0, lane, a);
#pragma unroll
                for (int j = 0; j < NVT; j += 2) {
                    uint32_t b[4];
                    frag_bt(sb + Ly::S, LV, 8 * j, k0, lane, b);
                    mma16816(O[j], a, b[0], b[1]);
                    mma16816(O[j + 1], a, b[2], b[3]);
                }
            }
            {
                uint32_t a[4];
                frag_a(sb + Ly::AQ, LT, 0, 0, lane, a);
#pragma unroll
                for (int j = 0; j < NVT; j += 2) {
                    uint32_t b[4];
                    frag_bt(sb + Ly::D, LV, 8 * j, 0, lane, b);
                    mma16816(O[j], a, b[0], b[1]);
                    mma16816(O[j + 1], a, b[2], b[3]);
                }
            }
            if (p.o) {
                const float f = p.scale;  // Qtil and A_qk are built from q^
#pragma unroll
                for (int hi = 0; hi < 2; ++hi) {
                    const int r = g8 + 8 * hi;
                    if (r < L) {
                        const long long ob = ((t0 + r) * H + h) * DV + 2 * t4;
#pragma unroll
                        for (int j = 0; j < NVT; ++j) {
                            if constexpr (AUG)
                                *reinterpret_cast<float2 *>(static_cast<float *>(p.o) + ob + 8 * j) =
                                    make_float2(f * O[j][2 * hi], f * O[j][2 * hi + 1]);
                            else
                                *reinterpret_cast<__nv_bfloat162 *>(og + ob + 8 * j) =
                                    __floats2bfloat162_rn(f * O[j][2 * hi], f * O[j][2 * hi + 1]);
                        }
                    }
                }
            }
        }
        // ---- S <- diag(e^{G_last}) S + Khat^T D
#pragma unroll
        for (int mk = 0; mk < 2; ++mk) {
            const float ga = gam[16 * mk + g8], gb = gam[16 * mk + g8 + 8];
#pragma unroll
            for (int j = 0; j < NVT; ++j) {
                S[mk][j][0] *= ga; S[mk][j][1] *= ga;
                S[mk][j][2] *= gb; S[mk][j][3] *= gb;
            }
            uint32_t a[4];
            frag_a(sb + Ly::KH, LT, 16 * mk, 0, lane, a);
#pragma unroll
            for (int j = 0; j < NVT; j += 2) {
                uint32_t b[4];
                frag_bt(sb + Ly::D, LV, 8 * j, 0, lane, b);
                mma16816(S[mk][j], a, b[0], b[1]);
                mma16816(S[mk][j + 1], a, b[2], b[3]);
            }
        }
        __syncwarp();  // every tile of this micro-chunk is read
    }
    cp_async_wait_all();
    if (p.S_out) {
#pragma unroll
        for (int mk = 0; mk < 2; ++mk)
#pragma unroll
            for (int j = 0; j < NVT; ++j)
#pragma unroll
                for (int hi = 0; hi < 2; ++hi) {
                    const int c = 16 * mk + g8 + 8 * hi, v = 8 * j + 2 * t4;
                    *reinterpret_cast<float2 *>(p.S_out + sbase + (long long)c * DV + v) =
                        make_float2(S[mk][j][2 * hi], S[mk][j][2 * hi + 1]);
                }
    }
}

template <int DV, bool AUG = false>
cudaError_t launch_t(const ChunkParams &p, cudaStream_t st, __nv_bfloat16 *save = nullptr) {
    const long long chains = (long long)p.N * p.H;
    if (chains <= 0) return cudaSuccess;
    const uint32_t smem = NWARP * Lay<DV>::BYTES;
    cudaError_t e = cudaFuncSetAttribute(kda_chunk_warp_kernel<DV, AUG>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    count_launch();
    kda_chunk_warp_kernel<DV, AUG><<<(unsigned)((chains + NWARP - 1) / NWARP), NWARP * 32, smem, st>>>(p, save);
    return cudaGetLastError();
}


// ---- d_k = 64: one CTA of two warps per chain. Warp w owns the value columns
// [VW w, VW w + VW) of the 64 x d_v state (VW = d_v / 2, registers) and the key channels
// [32 w, 32 w + 32) of the gate and of the transposed operand tiles; the 16 x 16 blocks
// are split between the warps (warp 0 A_kk and the inverse, warp 1 A_qk), and block
// barriers separate the phases that read the other warp's half.
namespace w64 {
constexpr int DK2 = 64;
constexpr int LKR = DK2 + 8;  // padded raw row (elements): 144 B, conflict-free row reads
constexpr int LW = DK2 + 8;   // the -W tile [16][LW]
template <int DV>
struct Lay {
    static constexpr int LV = DV + 8;
    static constexpr uint32_t Q = 0, K = Q + CW * LKR * 2, G = K + CW * LKR * 2, V = G + CW * LKR * 2;
    static constexpr uint32_t IN = (V + CW * LV * 2 + 127) / 128 * 128;
    static constexpr uint32_t TT = DK2 * LT * 2;             // a transposed tile [64][LT]
    static constexpr uint32_t X = 2 * IN, Y = X + TT, XQ = Y + TT, KT = XQ + TT, QT = KT + TT, KH = QT + TT;
    static constexpr uint32_t W = X;                          // -W [16][LW] over X^T
    static constexpr uint32_t D = Y;                          // D [16][LV] over Y^T
    static constexpr uint32_t TP = KH + TT, AQ = TP + CW * LT * 2;
    static constexpr uint32_t S = AQ + CW * LT * 2;           // S bf16 [64][LV]; exponent scratch [16][65] f32
    static constexpr uint32_t L = S + DK2 * LV * 2;
    static constexpr uint32_t RK = L + CW * LL * 4, RQ = RK + 64, BB = RQ + 64, PART = BB + 64, GAM = PART + 256;
    static constexpr uint32_t BYTES = (GAM + DK2 * 4 + 127) / 128 * 128;
    static_assert(CW * LW * 2 <= TT && CW * LV * 2 <= TT && CW * 65 * 4 <= DK2 * LV * 2, "aliases");
};

template <int DV>
__global__ void __launch_bounds__(64, 4) kda_chunk_warp64_kernel(const ChunkParams p) {
    using Ly = Lay<DV>;
    constexpr int LV = Ly::LV, VW = DV / 2, NVT = VW / 8;
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
    const int H = p.H, g8 = lane >> 2, t4 = lane & 3, c = 32 * w + lane;  // this thread's key channel
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

    float S[4][NVT][4];  // rows 16 mk + g8 (+ 8), columns VW w + 8 j + 2 t4 (+ 1)
    const long long sbase = ((long long)n * H + h) * DK2 * DV;
#pragma unroll
    for (int mk = 0; mk < 4; ++mk)
#pragma unroll
        for (int j = 0; j < NVT; ++j)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int cr = 16 * mk + g8 + 8 * (i >> 1), v = VW * w + 8 * j + 2 * t4 + (i & 1);
                S[mk][j][i] = p.S0 ? p.S0[sbase + (long long)cr * DV + v] : 0.f;
            }

    if (nmc > 0) issue(0);
    for (int mc = 0; mc < nmc; ++mc) {
        const long long t0 = bos + (long long)mc * CW;
        const int L = (int)min((long long)CW, eos - t0);
        const float bcur = braw;
        const uint32_t in = (mc & 1) * Ly::IN;
        if (mc + 1 < nmc) {
            issue(mc + 1);
            cp_async_wait_group<1>();
        } else {
            cp_async_wait_all();
        }
        __syncthreads();
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
                float x[8], y[8], xq[8], kt[8], qt[8], kc[8];
#pragma unroll
                for (int u = 0; u < 8; ++u) {
                    const int r = 8 * h8 + u;
                    const float kh = __bfloat162float(kr[r * LKR + c]) * rk[r];
                    const float qh = __bfloat162float(qr[r * LKR + c]) * rq[r];
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
        // A_kk (warp 0) -> L = diag(b) A_kk; A_qk (warp 1) -> bf16 tile
        {
            float acc[2][4] = {};
            const uint32_t xa = w == 0 ? Ly::X : Ly::XQ;
#pragma unroll
            for (int k0 = 0; k0 < DK2; k0 += 16) {
                uint32_t a[4], b[4];
                frag_at(sb + xa, LT, 0, k0, lane, a);
                frag_bt(sb + Ly::Y, LT, 0, k0, lane, b);
                mma16816(acc[0], a, b[0], b[1]);
                mma16816(acc[1], a, b[2], b[3]);
            }
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int hi = 0; hi < 2; ++hi) {
                    const int r = g8 + 8 * hi, s_ = 8 * j + 2 * t4;
                    if (w == 0) {
                        const float br = bb[r];
                        Lf[r * LL + s_] = s_ < r ? br * acc[j][2 * hi] : 0.f;
                        Lf[r * LL + s_ + 1] = s_ + 1 < r ? br * acc[j][2 * hi + 1] : 0.f;
                    } else {
                        stb2(sm + Ly::AQ + (r * LT + s_) * 2, s_ <= r ? acc[j][2 * hi] : 0.f,
                             s_ + 1 <= r ? acc[j][2 * hi + 1] : 0.f);
                    }
                }
        }
        if (steep) {  // exponent differences (never positive) on the CUDA cores
            float *Gs = reinterpret_cast<float *>(sm + Ly::S);
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
        // T' by forward substitution (warp 0, lane j < 16: column j)
        if (w == 0 && lane < CW) {
            const int j = lane;
            float t[CW];
#pragma unroll
            for (int i = 0; i < CW; ++i) {
                float acc = i == j ? 1.f : 0.f;
#pragma unroll
                for (int k = 0; k < i; ++k) acc = fmaf(-Lf[i * LL + k], t[k], acc);
                t[i] = acc;
            }
            const float bj = bb[j];
#pragma unroll
            for (int i = 0; i < CW; ++i)
                reinterpret_cast<__nv_bfloat16 *>(sm + Ly::TP)[i * LT + j] = __float2bfloat16_rn(t[i] * bj);
        }
        __syncthreads();
        // U (own value columns, registers); -W for own key channels into the shared tile
        float U[NVT][4];
        {
            uint32_t a[4];
            frag_a(sb + Ly::TP, LT, 0, 0, lane, a);
#pragma unroll
            for (int j = 0; j < NVT; j += 2) {
                uint32_t b[4];
                frag_bt(sb + in + Ly::V, LV, VW * w + 8 * j, 0, lane, b);
                U[j][0] = U[j][1] = U[j][2] = U[j][3] = 0.f;
                U[j + 1][0] = U[j + 1][1] = U[j + 1][2] = U[j + 1][3] = 0.f;
                mma16816(U[j], a, b[0], b[1]);
                mma16816(U[j + 1], a, b[2], b[3]);
            }
            float wv[4][4] = {};
#pragma unroll
            for (int j = 0; j < 4; j += 2) {
                uint32_t b[4];
                frag_b(sb + Ly::KT, LT, 32 * w + 8 * j, 0, lane, b);
                mma16816(wv[j], a, b[0], b[1]);
                mma16816(wv[j + 1], a, b[2], b[3]);
            }
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int hi = 0; hi < 2; ++hi)
                    stb2(sm + Ly::W + ((g8 + 8 * hi) * LW + 32 * w + 8 * j + 2 * t4) * 2, -wv[j][2 * hi],
                         -wv[j][2 * hi + 1]);
        }
        // own columns of the state as a bf16 operand
#pragma unroll
        for (int mk = 0; mk < 4; ++mk)
#pragma unroll
            for (int j = 0; j < NVT; ++j)
#pragma unroll
                for (int hi = 0; hi < 2; ++hi)
                    stb2(sm + Ly::S + ((16 * mk + g8 + 8 * hi) * LV + VW * w + 8 * j + 2 * t4) * 2, S[mk][j][2 * hi],
                         S[mk][j][2 * hi + 1]);
        __syncthreads();  // -W complete
        // D = U - W S (own columns) -> bf16 tile
#pragma unroll
        for (int k0 = 0; k0 < DK2; k0 += 16) {
            uint32_t a[4];
            frag_a(sb + Ly::W, LW, 0, k0, lane, a);
#pragma unroll
            for (int j = 0; j < NVT; j += 2) {
                uint32_t b[4];
                frag_bt(sb + Ly::S, LV, VW * w + 8 * j, k0, lane, b);
                mma16816(U[j], a, b[0], b[1]);
                mma16816(U[j + 1], a, b[2], b[3]);
            }
        }
#pragma unroll
        for (int j = 0; j < NVT; ++j)
#pragma unroll
            for (int hi = 0; hi < 2; ++hi)
                stb2(sm + Ly::D + ((g8 + 8 * hi) * LV + VW * w + 8 * j + 2 * t4) * 2, U[j][2 * hi], U[j][2 * hi + 1]);
        __syncwarp();
        // O = scale (Qtil S + A_qk D), own columns
        {
            float O[NVT][4];
#pragma unroll
            for (int j = 0; j < NVT; ++j) O[j][0] = O[j][1] = O[j][2] = O[j][3] = 0.f;
#pragma unroll
            for (int k0 = 0; k0 < DK2; k0 += 16) {
                uint32_t a[4];
                frag_at(sb + Ly::QT, LT, 0, k0, lane, a);
#pragma unroll
                for (int j = 0; j < NVT; j += 2) {
                    uint32_t b[4];
                    frag_bt(sb + Ly::S, LV, VW * w + 8 * j, k0, lane, b);
                    mma16816(O[j], a, b[0], b[1]);
                    mma16816(O[j + 1], a, b[2], b[3]);
                }
            }
            {
                uint32_t a[4];
                frag_a(sb + Ly::AQ, LT, 0, 0, lane, a);
#pragma unroll
                for (int j = 0; j < NVT; j += 2) {
                    uint32_t b[4];
                    frag_bt(sb + Ly::D, LV, VW * w + 8 * j, 0, lane, b);
                    mma16816(O[j], a, b[0], b[1]);
                    mma16816(O[j + 1], a, b[2], b[3]);
                }
            }
            if (og) {
#pragma unroll
                for (int hi = 0; hi < 2; ++hi) {
                    const int r = g8 + 8 * hi;
                    if (r < L) {
                        __nv_bfloat16 *orow = og + ((t0 + r) * H + h) * DV + VW * w + 2 * t4;
#pragma unroll
                        for (int j = 0; j < NVT; ++j)
                            *reinterpret_cast<__nv_bfloat162 *>(orow + 8 * j) =
                                __floats2bfloat162_rn(p.scale * O[j][2 * hi], p.scale * O[j][2 * hi + 1]);
                    }
                }
            }
        }
        // S <- diag(e^{G_last}) S + Khat^T D (own columns)
#pragma unroll
        for (int mk = 0; mk < 4; ++mk) {
            const float ga = gam[16 * mk + g8], gb = gam[16 * mk + g8 + 8];
#pragma unroll
            for (int j = 0; j < NVT; ++j) {
                S[mk][j][0] *= ga; S[mk][j][1] *= ga;
                S[mk][j][2] *= gb; S[mk][j][3] *= gb;
            }
            uint32_t a[4];
            frag_a(sb + Ly::KH, LT, 16 * mk, 0, lane, a);
#pragma unroll
            for (int j = 0; j < NVT; j += 2) {
                uint32_t b[4];
                frag_bt(sb + Ly::D, LV, VW * w + 8 * j, 0, lane, b);
                mma16816(S[mk][j], a, b[0], b[1]);
                mma16816(S[mk][j + 1], a, b[2], b[3]);
            }
        }
        __syncthreads();  // every tile of this micro-chunk is read
    }
    cp_async_wait_all();
    if (p.S_out) {
#pragma unroll
        for (int mk = 0; mk < 4; ++mk)
#pragma unroll
            for (int j = 0; j < NVT; ++j)
#pragma unroll
                for (int hi = 0; hi < 2; ++hi) {
                    const int cr = 16 * mk + g8 + 8 * hi, v = VW * w + 8 * j + 2 * t4;
                    *reinterpret_cast<float2 *>(p.S_out + sbase + (long long)cr * DV + v) =
                        make_float2(S[mk][j][2 * hi], S[mk][j][2 * hi + 1]);
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

}  // namespace cw

bool chunk_warp_supported(bool bf16, int Dk, int Dv) { return bf16 && (Dk == 32 || Dk == 64) && (Dv == 32 || Dv == 64); }

cudaError_t launch_chunk_warp(const ChunkParams &p, int Dk, int Dv, cudaStream_t st) {
    if (Dk == 64) return Dv == 32 ? cw::w64::launch_t<32>(p, st) : cw::w64::launch_t<64>(p, st);
    return Dv == 32 ? cw::launch_t<32>(p, st) : cw::launch_t<64>(p, st);
}

// The d_k = 32 forward saving every micro-chunk's entering state for the backward.
cudaError_t launch_chunk_warp_save(const ChunkParams &p, int Dv, __nv_bfloat16 *save, cudaStream_t st) {
    return Dv == 32 ? cw::launch_t<32>(p, st, save) : cw::launch_t<64>(p, st, save);
}

// The widened run of the segment form for bf16 d_k = d_v = 32 (outputs fp32 rows of 64,
// final states [32][64]); q is the segment view.
cudaError_t launch_chunk_warp_widened(const ChunkParams &q, cudaStream_t st) { return cw::launch_t<64, true>(q, st); }

}  // namespace kda
