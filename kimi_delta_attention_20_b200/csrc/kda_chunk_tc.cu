// Chunkwise KDA forward on the 5th-generation tensor cores (tcgen05 + TMEM,
// inputs staged by TMA), bf16 inputs, d_k = d_v = 128, chunk C = 64.
//
// The operator is the `chunk_kda` boundary of page "K3/kda/ops/api.py"; its
// result is the token recurrence of page "atlas_core/kimi_k3/kda.rs". One CTA
// owns one (sequence, head) and walks its chunks in order. The fp32 state is
// kept transposed, S^T (value channel v = TMEM lane, key channel c = column),
// in tensor memory for the whole sequence, so every state contraction is an
// M = 128 MMA whose accumulator row is a value channel:
//
//   per chunk, with G the inclusive in-chunk cumsum of the gate (clamped, or
//   formed in the kernel from A_log and dt_bias), beta = sigmoid(logit) (or a
//   given probability), k^/q^ the L2-normalised rows and T' = T diag(beta),
//   T = (I + diag(beta) A_kk)^-1:
//     A_kk[r,s] = sum_c k^_r k^_s e^{G_r-G_s} (s<r), A_qk likewise with q^_r (s<=r)
//     U^T   = V^T T'^T                   (MMA, M=v)
//     W^T   = (k^ e^G)^T T'^T            (MMA, M=c)
//     D^T   = U^T - S^T W^T              (MMA into the U accumulator, B negated)
//     O^T   = S^T (q^ e^G)^T + D^T A_qk^T   (two MMAs, one accumulator)
//     S^T  <- S^T diag(e^{G_last}) + D^T (k^ e^{G_last-G})   (MMA into the state)
//
// A_kk and A_qk come from two tensor-core products over the key channels. The
// gated product k_r k_s e^{G_r - G_s} is split as (k_r e^{G_r-R}) (k_s e^{R-G_s})
// with a per-channel reference R: for the two diagonal 32x32 blocks R is the
// block's middle row, for the off-diagonal block the boundary row 31 (both
// factors <= 1 there). A middle-row factor can reach e^{span}; when some
// channel's span exceeds kSpanMax the chunk computes A_kk and A_qk exactly on
// CUDA cores instead (no overflow, any gate).
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <vector>

#include "kda_common.cuh"
#include "kda_sm100.cuh"
#include "kda_tc_util.cuh"

namespace kda {
namespace tc {

using namespace sm100;
using namespace tcu;

constexpr int C = 64;
constexpr int D = 128;
constexpr int NT = 512;                      // 16 warps
constexpr float kSpanMax = 80.f;             // e^80 = 5.5e34 stays finite in bf16 and fp32
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // bounded waits: 2 s

// ---- shared memory map (bytes from the 1024-aligned base) ----
constexpr uint32_t STG_Q = 0, STG_K = 16384, STG_G = 32768, STG_V = 49152;  // TMA staging, [64][128]
constexpr uint32_t AOPS = 65536;                                            // 72 KiB, two views:
// view 1, operands of the A_kk / A_qk products
constexpr uint32_t YD_H0 = AOPS + 0, YD_H1 = AOPS + 8192, YO_H0 = AOPS + 16384, YO_H1 = AOPS + 20480;
constexpr uint32_t XKQD = AOPS + 40960;  // 2 halves x [128 rows][128 B]: rows 0..63 k, 64..127 q
constexpr uint32_t NRM = AOPS + 24576;   // [q|k][16 warps][64 rows] f32 partial squared norms
// view 2, after those products: fp32 solve buffers, T' tiles, then W^T, D^T and the output tile
constexpr int LDS = 65;  // padded fp32 row stride of L (64x64)
constexpr int LDT = 68;  // fp32 row stride of T (64x64)
constexpr int LDR = 52;  // fp32 row stride of the 16x48 block-row buffer
// (the k rows of XKQD, 40960..49152 and 57344..65536, stay live until the W products)
constexpr uint32_t LF = AOPS + 0, TF = AOPS + 16896, RF = AOPS + 34304, AQK = AOPS + 49152;
constexpr uint32_t WT = AOPS + 0, DT = AOPS + 16384, OT = AOPS + 57344;  // OT: [64][128] bf16, plain
constexpr uint32_t QT = AOPS + 73728, TPU = QT + 16384, TPW = TPU + 8192;  // T diag(beta), T diag(beta/|k|)
constexpr uint32_t KH = TPW + 8192, ST = KH + 16384;                       // ST: 32 KiB
constexpr uint32_t MISC = ST + 32768;
constexpr uint32_t M_BETA = MISC, M_INVQ = MISC + 256, M_INVK = MISC + 512, M_GAM = MISC + 768,
                   M_BAR = MISC + 1280, M_TMEM = MISC + 1312,
                   M_EW = MISC + 1536,    // [2][128] f32: e^{G_15}, e^{G_47} per channel
                   M_DTB = M_EW + 1024;   // [128] f32: dt_bias of this head (in-kernel gate)
constexpr uint32_t SMEM_BYTES = M_DTB + 512;
constexpr uint32_t SMEM_ALLOC = SMEM_BYTES + 1024;  // slack for 1024-byte alignment
static_assert(YO_H1 + 4096 <= NRM && NRM + 8192 <= XKQD, "view 1");
static_assert(LF + 64 * LDS * 4 <= TF && TF + 64 * LDT * 4 <= RF && RF + 16 * LDR * 4 <= XKQD, "view 2");
static_assert(AQK + 8192 <= XKQD + 16384 + 8192 && DT + 16384 <= XKQD && OT + 16384 <= AOPS + 73728, "view 2 tiles");
static_assert(SMEM_ALLOC <= 232448, "shared memory budget");

// ---- tensor memory columns ----
constexpr uint32_t TM_S = 0, TM_U = 128, TM_W = 192, TM_O = 256, TM_A = 320, TM_W1 = 416, TM_COLS = 512;

// ---- instruction descriptors ----
constexpr uint32_t ID_A1 = idesc_bf16(128, 64, false, false);
constexpr uint32_t ID_A2 = idesc_bf16(128, 32, false, false);
constexpr uint32_t ID_UW = idesc_bf16(128, 64, true, false);
constexpr uint32_t ID_DL = idesc_bf16(128, 64, false, true, /*neg_b=*/true);
constexpr uint32_t ID_O = idesc_bf16(128, 64, false, false);
constexpr uint32_t ID_S = idesc_bf16(128, 128, false, true);

constexpr int kMaxPerm = 256;

struct TcParams {
    CUtensorMap tq, tk, tg, tv;
    ChunkParams p;
    int *status;
    int nperm;
    int perm[kMaxPerm];
};

// Normalisation of q and k is deferred: the products use the raw rows and the
// per-row factors 1/|q_r|, 1/|k_r| are applied where they act linearly --
//   L[r,s]  = beta_r |k_r|^-1 |k_s|^-1 A_kk,raw[r,s]
//   W       = T diag(beta_s |k_s|^-1) (k e^G)_raw            (second T' tile)
//   D~      = D with column s scaled by |k_s|^-1, which feeds O += A_qk,raw D~ and
//             S += Khat_raw^T D~
//   o_r     = scale |q_r|^-1 (Qtil_raw S + A_qk,raw D~)_r
// which is algebraically identical to normalising first.
__global__ void __launch_bounds__(NT, 1) kda_chunk_tc_kernel(const __grid_constant__ TcParams P) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const ChunkParams &p = P.p;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = p.H;
    const int rank = blockIdx.x / H, h = blockIdx.x % H;
    const int n = rank < P.nperm ? P.perm[rank] : rank;
    long long bos, eos;
    if (p.cu_seqlens) { bos = p.cu_seqlens[n]; eos = p.cu_seqlens[n + 1]; }
    else { bos = (long long)n * p.T; eos = bos + p.T; }
    const int nchunks = (int)((eos - bos + C - 1) / C);

    uint64_t *bar_qkg = reinterpret_cast<uint64_t *>(sm + M_BAR);
    uint64_t *bar_v = bar_qkg + 1, *bar_mma = bar_qkg + 2;
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(sm + M_TMEM);
    float *sbeta = reinterpret_cast<float *>(sm + M_BETA);
    float *sinvq = reinterpret_cast<float *>(sm + M_INVQ);
    float *sinvk = reinterpret_cast<float *>(sm + M_INVK);
    float *sGam = reinterpret_cast<float *>(sm + M_GAM);
    float *sEw = reinterpret_cast<float *>(sm + M_EW);
    float *sDtb = reinterpret_cast<float *>(sm + M_DTB);
    const int gmode = p.gate_mode;
    const float rate = gmode != kGateLog ? expf(p.A_log[h]) : 0.f;
    if (tid < D) sDtb[tid] = gmode != kGateLog && p.dt_bias ? p.dt_bias[h * D + tid] : 0.f;
    float *Lf = reinterpret_cast<float *>(sm + LF);
    float *Tf = reinterpret_cast<float *>(sm + TF);

    if (warp == 0) { tmem_alloc(s_tmem, TM_COLS); tmem_relinquish(); }
    if (tid == 32) {
        mbar_init(bar_qkg, 1); mbar_init(bar_v, 1); mbar_init(bar_mma, 1);
        fence_mbar_init();
        tma_prefetch_desc(&P.tq); tma_prefetch_desc(&P.tk); tma_prefetch_desc(&P.tg); tma_prefetch_desc(&P.tv);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tb = *s_tmem;
    const uint32_t sb = smem_u32(sm);
    // descriptor of byte offset `off` from the tile base: the start-address field is the
    // only one that changes, so each descriptor is one add on a precomputed base
    const uint64_t dK = sdesc_sw128(sb, 16, 1024);    // K-major operands
    const uint64_t dM = sdesc_sw128(sb, 8192, 1024);  // MN-major operands (atoms 8 KiB apart)
    const uint64_t dX = sdesc_sw128(sb, 16384, 1024); // MN-major view of XKQD (halves 16 KiB apart)
    auto dk = [&](uint32_t off) { return dK + (uint64_t)(off >> 4); };
    auto dm = [&](uint32_t off) { return dM + (uint64_t)(off >> 4); };
    auto dx = [&](uint32_t off) { return dX + (uint64_t)(off >> 4); };
    const int quarter = warp & 3;                               // TMEM lanes 32*quarter .. +31
    const uint32_t lane_sel = (uint32_t)(32 * quarter) << 16;
    const int cgrp = warp >> 2;                                  // column group of TMEM phases

    auto issue_qkg = [&](long long t) {
        mbar_arrive_expect_tx(bar_qkg, 3 * 16384);
        for (int hf = 0; hf < 2; ++hf) {
            tma_load_3d(sm + STG_Q + hf * 8192, &P.tq, bar_qkg, hf * 64, h, (int)t);
            tma_load_3d(sm + STG_K + hf * 8192, &P.tk, bar_qkg, hf * 64, h, (int)t);
            tma_load_3d(sm + STG_G + hf * 8192, &P.tg, bar_qkg, hf * 64, h, (int)t);
        }
    };
    auto issue_v = [&](long long t) {
        mbar_arrive_expect_tx(bar_v, 16384);
        for (int hf = 0; hf < 2; ++hf) tma_load_3d(sm + STG_V + hf * 8192, &P.tv, bar_v, hf * 64, h, (int)t);
    };
    // a bounded wait on an mbarrier phase: one warp polls, the others park in the
    // CTA barrier (no issue slots spent polling); true if the CTA must stop
    // (the phase advances only when it completed, so an abort waits on the pending one)
    auto wait_all = [&](uint64_t *bar, uint32_t &ph) -> bool {
        bool ok = true;
        if (warp == 0) ok = mbar_wait(bar, ph, kWaitLimitNs);
        const bool stop = __syncthreads_or(!ok) != 0;
        if (!stop) ph ^= 1;
        return stop;
    };

    // thread kMma issues the MMAs, thread kTma (another warp) the TMA loads
    constexpr int kMma = 0, kTma = NT - 32;
    uint32_t ph_qkg = 0, ph_v = 0, ph_mma = 0;
    bool qkg_out = false, v_out = false, mma_out = false;  // outstanding async work of this thread
    bool aborted = false;
    // (a test of the bounded waits leaves the first copies unissued: the first wait gives up)
    if (tid == kTma && nchunks > 0 && !p.stall_first_wait) { issue_qkg(bos); issue_v(bos); qkg_out = v_out = true; }

    const long long sbase_state = ((long long)n * H + h) * D * D;
    const __nv_bfloat16 *bt = static_cast<const __nv_bfloat16 *>(p.beta);
    // beta logits run one chunk ahead in registers of threads 0..63
    float beta_next = 0.f;
    if (tid < C && bos + tid < eos) beta_next = __bfloat162float(bt[(bos + tid) * H + h]);

    // thread -> (16-byte chunk of 8 channels, 2 consecutive rows) for the row-layout phases:
    // warp w owns channels 8w .. 8w+7 for all 64 rows, lane l rows 2l and 2l+1, so the
    // in-chunk cumsum is a scan across the lanes of one warp.
    const int jch = warp;
    const int row0 = 2 * lane;
    const int blk = lane >> 4;                     // 32-row block of those rows

    for (int ci = 0; ci < nchunks && !aborted; ++ci) {
        const long long t0 = bos + (long long)ci * C;
        const int L = (int)((eos - t0) < C ? (eos - t0) : C);
        const bool has_next = ci + 1 < nchunks;

        if (tid < C) {
            sbeta[tid] = tid < L ? beta_value(beta_next, p.beta_prob) : 0.f;
            beta_next = 0.f;
            if (has_next && t0 + C + tid < eos) beta_next = __bfloat162float(bt[(t0 + C + tid) * H + h]);
        }

        // ---------------- inputs of this chunk
        {
            bool ok = true;
            if (warp == 0) ok = mbar_wait(bar_qkg, ph_qkg, kWaitLimitNs) && mbar_wait(bar_v, ph_v, kWaitLimitNs);
            if (__syncthreads_or(!ok)) { aborted = true; break; }
            ph_qkg ^= 1; ph_v ^= 1;
            if (tid == kTma) qkg_out = v_out = false;
        }

        // ---------------- P1: gate cumsum, in-warp scan over the 64 rows
        float G[2][8], Gm[8], G47[8], G63[8];
        bool span_bad = false;
        {
            float tot[8];
            {
                float2 tt[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) tt[e] = make_float2(0.f, 0.f);
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const int r = row0 + u;
                    float2 gg[4];
                    unpack8x2(lds128(sm + STG_G, sw128_chunk(r, 8 * jch, 64)), gg);
                    if (gmode != kGateLog) {
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 b = *reinterpret_cast<const float2 *>(sDtb + 8 * jch + 2 * e);
                            gg[e] = make_float2(gate_fast(gg[e].x, b.x, rate, gmode, p.lb),
                                                gate_fast(gg[e].y, b.y, rate, gmode, p.lb));
                        }
                    } else if (p.has_lb) {
#pragma unroll
                        for (int e = 0; e < 4; ++e) gg[e] = make_float2(fmaxf(gg[e].x, p.lb), fmaxf(gg[e].y, p.lb));
                    }
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 gv = r < L ? gg[e] : make_float2(0.f, 0.f);
                        tt[e] = __fadd2_rn(tt[e], gv);
                        G[u][2 * e] = tt[e].x;
                        G[u][2 * e + 1] = tt[e].y;
                    }
                }
#pragma unroll
                for (int e = 0; e < 4; ++e) { tot[2 * e] = tt[e].x; tot[2 * e + 1] = tt[e].y; }
            }
            float G15[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                float inc = tot[e];
#pragma unroll
                for (int d = 1; d < 32; d <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, inc, d);
                    if (lane >= d) inc += y;
                }
                G[0][e] += inc - tot[e];
                G[1][e] += inc - tot[e];
                G15[e] = __shfl_sync(0xffffffffu, inc, 7);
                G47[e] = __shfl_sync(0xffffffffu, inc, 23);
                G63[e] = __shfl_sync(0xffffffffu, inc, 31);
                Gm[e] = blk ? G47[e] : G15[e];
                span_bad |= fabsf(G[0][e] - Gm[e]) > kSpanMax;
                span_bad |= fabsf(G[1][e] - Gm[e]) > kSpanMax;
            }
            if (lane < 8) {  // lane e writes channel 8*jch + e
                float a = G63[0], b = G15[0], c = G47[0];
#pragma unroll
                for (int e = 1; e < 8; ++e)
                    if (lane == e) { a = G63[e]; b = G15[e]; c = G47[e]; }
                sGam[8 * jch + lane] = expf(a);
                sEw[8 * jch + lane] = expf(b);
                sEw[128 + 8 * jch + lane] = expf(c);
            }
        }
        const bool fb = __syncthreads_or(span_bad) != 0;

        // ---------------- P2: bf16 operand tiles from the raw rows
        {
            const int hf = jch >> 3, jc = 8 * (jch & 7);
            constexpr float kLog2e = 1.4426950408889634f;
            float2 ngm[4], emid[4], fkh[4], foff[4];
            if (!fb) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float m0 = Gm[2 * e], m1 = Gm[2 * e + 1];
                    ngm[e] = make_float2(-m0, -m1);
                    emid[e] = make_float2(__expf(m0), __expf(m1));
                    fkh[e] = make_float2(__expf(G63[2 * e] - m0), __expf(G63[2 * e + 1] - m1));
                    foff[e] = make_float2(__expf(G47[2 * e] - m0), __expf(G47[2 * e + 1] - m1));
                }
            }
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int r = row0 + u;
                const uint32_t off = sw128_chunk(r, 8 * jch, 64);
                float2 qq[4], kk[4];
                unpack8x2(lds128(sm + STG_Q, off), qq);
                unpack8x2(lds128(sm + STG_K, off), kk);
                if (r >= L) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) { qq[e] = make_float2(0.f, 0.f); kk[e] = qq[e]; }
                }
                {   // this thread's 8 channels of |q_r|^2 and |k_r|^2
                    float2 a = __fmul2_rn(qq[0], qq[0]), b = __fmul2_rn(kk[0], kk[0]);
#pragma unroll
                    for (int e = 1; e < 4; ++e) { a = __ffma2_rn(qq[e], qq[e], a); b = __ffma2_rn(kk[e], kk[e], b); }
                    float *nrm = reinterpret_cast<float *>(sm + NRM);
                    nrm[jch * 64 + r] = a.x + a.y;
                    nrm[1024 + jch * 64 + r] = b.x + b.y;
                }
                float2 t1[4], t3[4];
                if (!fb) {
                    float2 xk[4], xq[4], y[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        // a = G - G_m; ed = e^a (SFU), yd = e^-a = 1/ed (FMA pipe)
                        const float2 a = __fmul2_rn(__fadd2_rn(make_float2(G[u][2 * e], G[u][2 * e + 1]), ngm[e]),
                                                    make_float2(kLog2e, kLog2e));
                        const float2 ed = make_float2(ex2a(a.x), ex2a(a.y));
                        const float2 yd = rcp2_nr(ed);
                        xk[e] = __fmul2_rn(kk[e], ed);
                        xq[e] = __fmul2_rn(qq[e], ed);
                        y[e] = __fmul2_rn(kk[e], yd);
                        t1[e] = __fmul2_rn(xq[e], emid[e]);
                        t3[e] = __fmul2_rn(y[e], fkh[e]);
                    }
                    sts128(sm, XKQD + sw128_chunk(r, 8 * jch, 128), pack8x2(xk));
                    sts128(sm, XKQD + sw128_chunk(64 + r, 8 * jch, 128), pack8x2(xq));
                    sts128(sm, (hf ? YD_H1 : YD_H0) + sw128_chunk(r, jc, 64), pack8x2(y));
                    if (blk == 0) {
                        // off-diagonal column operand k_s e^{G_47 - G_s}, paired with the block-1 rows
#pragma unroll
                        for (int e = 0; e < 4; ++e) y[e] = __fmul2_rn(y[e], foff[e]);
                        sts128(sm, (hf ? YO_H1 : YO_H0) + sw128_chunk(r, jc, 32), pack8x2(y));
                    }
                } else {
                    // exact path: no block reference, the k rows of XKQD hold k e^G (<= 1)
                    float2 t2[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 eg = make_float2(expf(G[u][2 * e]), expf(G[u][2 * e + 1]));
                        const float2 ek = make_float2(expf(G63[2 * e] - G[u][2 * e]), expf(G63[2 * e + 1] - G[u][2 * e + 1]));
                        t1[e] = __fmul2_rn(qq[e], eg);
                        t2[e] = __fmul2_rn(kk[e], eg);
                        t3[e] = __fmul2_rn(kk[e], ek);
                    }
                    sts128(sm, XKQD + sw128_chunk(r, 8 * jch, 128), pack8x2(t2));
                }
                sts128(sm, QT + off, pack8x2(t1));
                sts128(sm, KH + off, pack8x2(t3));
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // ---------------- A_kk / A_qk products; next chunk's q, k, g loads
        // D1 (cols 0..63): rows 0..63 = A_kk, rows 64..127 = A_qk (diagonal 32-blocks valid).
        // D2 (cols 64..95): A rows start at row 32, so lanes 0..31 = A_kk[32+i][0..31] and
        // lanes 64..95 = A_qk[32+i][0..31]; the other lanes are unused.
        if (tid == kTma && !fb && has_next) { issue_qkg(t0 + C); qkg_out = true; }
        if (tid == kMma && !fb) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t ko = (kk >> 2) * 16384 + (kk & 3) * 32;
                const uint32_t yb = (kk >> 2) ? YD_H1 : YD_H0, ob = (kk >> 2) ? YO_H1 : YO_H0;
                mma_bf16(tb + TM_A, dk(XKQD + ko),
                         dk(yb + (kk & 3) * 32), ID_A1, kk > 0);
                mma_bf16(tb + TM_A + 64, dk(XKQD + ko + 32 * 128),
                         dk(ob + (kk & 3) * 32), ID_A2, kk > 0);
            }
            mma_commit(bar_mma);
            mma_out = true;
        }

        if (tid < 128) {  // row norms from the 16 per-warp partials
            const int r = tid & 63, which = tid >> 6;
            const float *nrm = reinterpret_cast<const float *>(sm + NRM) + which * 1024 + r;
            float ssum = 0.f;
#pragma unroll
            for (int w = 0; w < 16; ++w) ssum += nrm[w * 64];
            const float inv = r < L ? (p.use_l2 ? rsqrtf(ssum + kL2Eps) : 1.f) : 0.f;
            (which ? sinvk : sinvq)[r] = inv;
        }

        // ---------------- state refresh (overlaps the products above):
        // bf16 copy of S^T for this chunk's MMAs, and S^T diag(e^{G_last}) back into TMEM
        {
            const int v = 32 * quarter + lane;
            const int c0 = 32 * cgrp;
            float x[32];
            if (ci == 0) {
#pragma unroll
                for (int j = 0; j < 32; ++j) x[j] = p.S0 ? p.S0[sbase_state + (long long)(c0 + j) * D + v] : 0.f;
            } else {
                tmem_ld32(tb + TM_S + lane_sel + c0, x);
                tmem_ld_wait();
            }
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) sts128(sm, ST + sw128_chunk(v, c0 + 8 * q4, 128), pack8(x + 8 * q4));
#pragma unroll
            for (int j = 0; j < 32; j += 2) {
                const float2 v2 = __fmul2_rn(make_float2(x[j], x[j + 1]),
                                             *reinterpret_cast<const float2 *>(sGam + c0 + j));
                x[j] = v2.x; x[j + 1] = v2.y;
            }
            tmem_st32(tb + TM_S + lane_sel + c0, x);
            tmem_st_wait();
        }

        // ---------------- A results -> L (fp32, beta and key norms applied) and raw A_qk (bf16 tile)
        if (!fb) {
            if (wait_all(bar_mma, ph_mma)) { aborted = true; break; }
            if (tid == kMma) mma_out = false;
            tc_fence_after();
            const int i = lane;
            // (quarter, column group) -> a 32-row x 16-column piece of D1 / D2
            const bool has = (quarter & 1) == 0 || cgrp < 2;
            const int col = (quarter & 1) ? 32 + 16 * cgrp : (cgrp < 2 ? 16 * cgrp : 64 + 16 * (cgrp - 2));
            float va[16];
            if (has) {
                tmem_ld16(tb + TM_A + lane_sel + col, va);
                tmem_ld_wait();
            }
            if (quarter == 0) {
                if (cgrp < 2) {  // A_kk rows 0..31, cols 16*cgrp..: s < i
                    const float f = sbeta[i] * sinvk[i];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int s = 16 * cgrp + j;
                        Lf[i * LDS + s] = s < i ? f * sinvk[s] * va[j] : 0.f;
                    }
                } else {         // A_kk rows 32..63, cols 0..31 (all below the diagonal)
                    const float f = sbeta[32 + i] * sinvk[32 + i];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int s = 16 * (cgrp - 2) + j;
                        Lf[(32 + i) * LDS + s] = f * sinvk[s] * va[j];
                    }
                }
            } else if (quarter == 1) {
                if (cgrp < 2) {  // A_kk rows 32..63, cols 32..63: s < i
                    const float f = sbeta[32 + i] * sinvk[32 + i];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int s = 16 * cgrp + j;
                        Lf[(32 + i) * LDS + 32 + s] = s < i ? f * sinvk[32 + s] * va[j] : 0.f;
                    }
                }
            } else if (quarter == 2) {
                if (cgrp < 2) {  // A_qk rows 0..31, cols 0..31: s <= i
#pragma unroll
                    for (int j = 0; j < 16; ++j) va[j] = 16 * cgrp + j <= i ? va[j] : 0.f;
                    row16_to_tile(sm, AQK, i, 16 * cgrp, 64, va);
                } else {         // A_qk rows 32..63, cols 0..31
                    row16_to_tile(sm, AQK, 32 + i, 16 * (cgrp - 2), 64, va);
                }
            } else {
                if (cgrp < 2) {  // A_qk rows 32..63, cols 32..63: s <= i
#pragma unroll
                    for (int j = 0; j < 16; ++j) va[j] = 16 * cgrp + j <= i ? va[j] : 0.f;
                    row16_to_tile(sm, AQK, 32 + i, 32 + 16 * cgrp, 64, va);
                } else {         // A_qk rows 0..31, cols 32..63 are zero
                    const int c0 = 32 + 16 * (cgrp - 2);
                    sts128(sm, AQK + sw128_chunk(i, c0, 64), make_uint4(0u, 0u, 0u, 0u));
                    sts128(sm, AQK + sw128_chunk(i, c0 + 8, 64), make_uint4(0u, 0u, 0u, 0u));
                }
            }
        } else {
            __syncthreads();  // the row norms above are read below
            // exact A_kk / A_qk on CUDA cores (raw rows): warp per row r, lanes over channels,
            // walking s downwards while accumulating the gate between s and r
            for (int r = warp; r < C; r += NT / 32) {
                float kr[4], qr[4], dg[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const uint32_t o = sw128(r, lane + 32 * u, 64);
                    kr[u] = r < L ? bf(sm + STG_K, o) : 0.f;
                    qr[u] = r < L ? bf(sm + STG_Q, o) : 0.f;
                    dg[u] = 0.f;
                }
                for (int s = r; s >= 0; --s) {
                    float akk = 0.f, aqk = 0.f;
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const uint32_t o = sw128(s, lane + 32 * u, 64);
                        const float e = expf(dg[u]) * (s < L ? bf(sm + STG_K, o) : 0.f);
                        akk = fmaf(kr[u], e, akk);
                        aqk = fmaf(qr[u], e, aqk);
                        float gv = 0.f;
                        if (s < L) {
                            gv = bf(sm + STG_G, o);
                            if (gmode != kGateLog) gv = gate_fast(gv, sDtb[lane + 32 * u], rate, gmode, p.lb);
                            else if (p.has_lb) gv = fmaxf(gv, p.lb);
                        }
                        dg[u] += gv;
                    }
                    akk = warp_sum(akk); aqk = warp_sum(aqk);
                    if (lane == 0) {
                        Lf[r * LDS + s] = s < r ? sbeta[r] * sinvk[r] * sinvk[s] * akk : 0.f;
                        st_bf(sm, AQK + sw128(r, s, 64), aqk);
                    }
                }
                for (int s = r + 1 + lane; s < C; s += 32) st_bf(sm, AQK + sw128(r, s, 64), 0.f);
            }
            fence_proxy_async_smem();
            __syncthreads();
            if (tid == kTma && has_next) { issue_qkg(t0 + C); qkg_out = true; }
        }
        __syncthreads();

        // ---------------- T = (I + L)^-1 on 16x16 blocks, written straight into the bf16
        // tiles T_u = T diag(beta) and T_w = T diag(beta / |k|) (rows r, columns s <= r)
        if (warp < 4) {
            // diagonal blocks by a column sweep (lane j = column j): once t[k] is final it
            // updates every later row, so the dependent chain is 16 steps long
            if (lane < 16) {
                const int b = warp, j = lane;
                float t[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) t[i] = i == j ? 1.f : 0.f;
#pragma unroll
                for (int k = 0; k < 15; ++k) {
#pragma unroll
                    for (int i = k + 1; i < 16; ++i) t[i] = fmaf(-Lf[(16 * b + i) * LDS + 16 * b + k], t[k], t[i]);
                }
#pragma unroll
                for (int i = 0; i < 16; ++i) Tf[(16 * b + i) * LDT + 16 * b + j] = t[i];
            }
        } else {
            // blocks above the block diagonal: zero in T (read by the block products) and in
            // both bf16 tiles
            // 6 blocks x 16 rows x 2 chunks of 8 columns = 192 items for 384 threads
            const int e = tid - 128;
            if (e < 192) {
                const int bid = e >> 5, i = (e >> 1) & 15, half = e & 1;
                const int bi = bid < 3 ? 0 : bid < 5 ? 1 : 2;
                const int bj = bid < 3 ? bid + 1 : bid < 5 ? bid - 1 : 3;
                const int r = 16 * bi + i, c = 16 * bj + 8 * half;
                *reinterpret_cast<float4 *>(Tf + r * LDT + c) = make_float4(0.f, 0.f, 0.f, 0.f);
                *reinterpret_cast<float4 *>(Tf + r * LDT + c + 4) = make_float4(0.f, 0.f, 0.f, 0.f);
                sts128(sm, TPU + sw128_chunk(r, c, 64), make_uint4(0u, 0u, 0u, 0u));
                sts128(sm, TPW + sw128_chunk(r, c, 64), make_uint4(0u, 0u, 0u, 0u));
            }
        }
        __syncthreads();
        // block rows I = 1..3:  T[I, J<I] = -T_II sum_{K<I} L_IK T_KJ on warp-level tf32 MMAs;
        // warp w < 2I owns output columns 8w .. 8w+7; the step-1 accumulator is transposed
        // into the step-2 operand with shuffles inside the warp
        if (warp >= 8) {
            // diagonal blocks of T -> both bf16 tiles (s <= r), 4 blocks x 16 rows x 2 chunks
            const int e = tid - 256;
            if (e < 128) {
                const int b = e >> 5, i = (e >> 1) & 15, half = e & 1;
                const int r = 16 * b + i, c = 16 * b + 8 * half;
                float mu[8], mw[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const int s_ = c + q;
                    mu[q] = s_ <= r ? Tf[r * LDT + s_] * sbeta[s_] : 0.f;
                    mw[q] = mu[q] * sinvk[s_];
                }
                sts128(sm, TPU + sw128_chunk(r, c, 64), pack8(mu));
                sts128(sm, TPW + sw128_chunk(r, c, 64), pack8(mw));
            }
        }
        {
            const int g = lane >> 2, t4 = lane & 3;
#pragma unroll
            for (int I = 1; I < 4; ++I) {
                if (warp < 2 * I) {
                    const int n0 = 8 * warp;
                    float d[4] = {0.f, 0.f, 0.f, 0.f};
                    const float *La = Lf + (16 * I + g) * LDS, *Lb = Lf + (16 * I + g + 8) * LDS;
#pragma unroll
                    for (int ks = 0; ks < 2 * I; ++ks) {
                        const int k0 = 8 * ks;
                        const uint32_t a[4] = {to_tf32(La[k0 + t4]), to_tf32(Lb[k0 + t4]), to_tf32(La[k0 + t4 + 4]),
                                               to_tf32(Lb[k0 + t4 + 4])};
                        const uint32_t b[2] = {to_tf32(Tf[(k0 + t4) * LDT + n0 + g]),
                                               to_tf32(Tf[(k0 + t4 + 4) * LDT + n0 + g])};
                        mma_tf32_16x8x8(d, a, b);
                    }
                    // R[row][col] sits in lane 4*(row % 8) + col/2, component (row >= 8) * 2 + col % 2
                    const int srcA = 4 * t4 + (g >> 1), srcB = 4 * (t4 + 4) + (g >> 1);
                    const bool odd = g & 1;
                    float v[8];
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        v[c] = __shfl_sync(0xffffffffu, d[c], srcA);
                        v[4 + c] = __shfl_sync(0xffffffffu, d[c], srcB);
                    }
                    const uint32_t b0[2] = {to_tf32(odd ? v[1] : v[0]), to_tf32(odd ? v[5] : v[4])};  // rows t, t+4
                    const uint32_t b1[2] = {to_tf32(odd ? v[3] : v[2]), to_tf32(odd ? v[7] : v[6])};  // rows 8+t, 12+t
                    float e[4] = {0.f, 0.f, 0.f, 0.f};
                    const float *Ta = Tf + (16 * I + g) * LDT + 16 * I, *Tb = Tf + (16 * I + g + 8) * LDT + 16 * I;
                    {
                        const uint32_t a[4] = {to_tf32(Ta[t4]), to_tf32(Tb[t4]), to_tf32(Ta[t4 + 4]), to_tf32(Tb[t4 + 4])};
                        mma_tf32_16x8x8(e, a, b0);
                    }
                    {
                        const uint32_t a[4] = {to_tf32(Ta[8 + t4]), to_tf32(Tb[8 + t4]), to_tf32(Ta[12 + t4]),
                                               to_tf32(Tb[12 + t4])};
                        mma_tf32_16x8x8(e, a, b1);
                    }
                    const int r0 = 16 * I + g, c0 = n0 + 2 * t4;
                    Tf[r0 * LDT + c0] = -e[0];
                    Tf[r0 * LDT + c0 + 1] = -e[1];
                    Tf[(r0 + 8) * LDT + c0] = -e[2];
                    Tf[(r0 + 8) * LDT + c0 + 1] = -e[3];
                    const float b0s = sbeta[c0], b1s = sbeta[c0 + 1];
                    const float w0s = b0s * sinvk[c0], w1s = b1s * sinvk[c0 + 1];
                    *reinterpret_cast<uint32_t *>(sm + TPU + sw128(r0, c0, 64)) =
                        pack_bf16x2(-e[0] * b0s, -e[1] * b1s);
                    *reinterpret_cast<uint32_t *>(sm + TPU + sw128(r0 + 8, c0, 64)) =
                        pack_bf16x2(-e[2] * b0s, -e[3] * b1s);
                    *reinterpret_cast<uint32_t *>(sm + TPW + sw128(r0, c0, 64)) =
                        pack_bf16x2(-e[0] * w0s, -e[1] * w1s);
                    *reinterpret_cast<uint32_t *>(sm + TPW + sw128(r0 + 8, c0, 64)) =
                        pack_bf16x2(-e[2] * w0s, -e[3] * w1s);
                }
                if (I < 3) __syncthreads();
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // ---------------- U^T = V^T T_u^T, W^T = Ktil^T T_w^T
        if (tid == kMma) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                mma_bf16(tb + TM_U, dm(STG_V + kk * 2048), dk(TPU + kk * 32), ID_UW, kk > 0);
                // W in two K halves (token blocks 0..31 and 32..63), each with its own
                // block reference; recombined per key channel when W is read back
                mma_bf16(tb + (kk < 2 ? TM_W : TM_W1), dx(XKQD + kk * 2048), dk(TPW + kk * 32), ID_UW,
                         (kk & 1) != 0);
            }
            mma_commit(bar_mma);
            mma_out = true;
        }
        if (wait_all(bar_mma, ph_mma)) { aborted = true; break; }
        if (tid == kMma) mma_out = false;
        tc_fence_after();
        {   // W^T (lane c, columns r) = e^{G_15[c]} W0 + e^{G_47[c]} W1 -> bf16 tile [c][r]
            float x[16], x1[16];
            const int c = 32 * quarter + lane;
            tmem_ld16(tb + TM_W + lane_sel + 16 * cgrp, x);
            tmem_ld16(tb + TM_W1 + lane_sel + 16 * cgrp, x1);
            tmem_ld_wait();
            const float e0 = fb ? 1.f : sEw[c], e1 = fb ? 1.f : sEw[128 + c];
#pragma unroll
            for (int j = 0; j < 16; ++j) x[j] = fmaf(e0, x[j], e1 * x1[j]);
            row16_to_tile(sm, WT, c, 16 * cgrp, 128, x);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // ---------------- D^T = U^T - S^T W^T ; O^T = S^T Qtil^T ; next chunk's v load
        if (tid == kTma && has_next) { issue_v(t0 + C); v_out = true; }
        if (tid == kMma) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint64_t adesc = dk(ST + (kk >> 2) * 16384 + (kk & 3) * 32);
                mma_bf16(tb + TM_U, adesc, dm(WT + kk * 2048), ID_DL, 1);
                mma_bf16(tb + TM_O, adesc, dk(QT + (kk >> 2) * 8192 + (kk & 3) * 32),
                         ID_O, kk > 0);
            }
            mma_commit(bar_mma);
            mma_out = true;
        }
        if (wait_all(bar_mma, ph_mma)) { aborted = true; break; }
        if (tid == kMma) mma_out = false;
        tc_fence_after();
        {   // D^T (lane v, columns s), times |k_s|^-1 -> bf16 tile [v][s]
            float x[16];
            const int s0 = 16 * cgrp;
            tmem_ld16(tb + TM_U + lane_sel + s0, x);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 16; ++j) x[j] *= sinvk[s0 + j];
            row16_to_tile(sm, DT, 32 * quarter + lane, s0, 128, x);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // ---------------- O^T += D~^T A_qk^T ; S^T += D~^T Khat
        if (tid == kMma) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint64_t adesc = dk(DT + kk * 32);
                mma_bf16(tb + TM_O, adesc, dk(AQK + kk * 32), ID_O, 1);
                mma_bf16(tb + TM_S, adesc, dm(KH + kk * 2048), ID_S, 1);
            }
            mma_commit(bar_mma);
            mma_out = true;
        }
        if (wait_all(bar_mma, ph_mma)) { aborted = true; break; }
        if (tid == kMma) mma_out = false;
        tc_fence_after();
        {   // O^T (lane v, columns r) -> plain [r][v] tile, scale and 1/|q_r| applied
            float x[16];
            const int v = 32 * quarter + lane, r0 = 16 * cgrp;
            tmem_ld16(tb + TM_O + lane_sel + r0, x);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                const int r = r0 + j;
                *reinterpret_cast<__nv_bfloat16 *>(sm + OT + r * 256 + v * 2) =
                    __float2bfloat16_rn(p.scale * sinvq[r] * x[j]);
            }
        }
        __syncthreads();
        {   // coalesced 16-byte stores of the rows that belong to this sequence
            __nv_bfloat16 *O = static_cast<__nv_bfloat16 *>(p.o);
#pragma unroll
            for (int m = 0; m < 2; ++m) {
                const int qd = tid + NT * m, r = qd >> 4, c16 = qd & 15;
                if (r < L) {
                    const uint4 val = lds128(sm + OT, r * 256 + c16 * 16);
                    *reinterpret_cast<uint4 *>(O + ((t0 + r) * H + h) * D + c16 * 8) = val;
                }
            }
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }

    if (!aborted && p.S_out) {
        const int v = 32 * quarter + lane;
        const int c0 = 32 * cgrp;
        float x[32];
        if (nchunks == 0) {
#pragma unroll
            for (int j = 0; j < 32; ++j) x[j] = p.S0 ? p.S0[sbase_state + (long long)(c0 + j) * D + v] : 0.f;
        } else {
            tmem_ld32(tb + TM_S + lane_sel + c0, x);
            tmem_ld_wait();
        }
#pragma unroll
        for (int j = 0; j < 32; ++j) p.S_out[sbase_state + (long long)(c0 + j) * D + v] = x[j];
    }

    if (aborted && (tid == kMma || tid == kTma)) {
        // let copies and products already in flight land before the CTA leaves
        if (qkg_out) mbar_wait(bar_qkg, ph_qkg, kWaitLimitNs);
        if (v_out) mbar_wait(bar_v, ph_v, kWaitLimitNs);
        if (mma_out) mbar_wait(bar_mma, ph_mma, kWaitLimitNs);
        if (P.status && tid == kMma) atomicOr(P.status, 1);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tb, TM_COLS);
    }
}

// ------------------------------------------------------------------ host side

}  // namespace tc

bool chunk_tc_supported(bool bf16, int Dk, int Dv, int chunk_size) {
    return bf16 && Dk == 128 && Dv == 128 && (chunk_size == 0 || chunk_size == 64);
}

size_t chunk_tc_workspace_bytes(int, int, int, int) { return 256; }

cudaError_t launch_chunk_tc(const ChunkParams &p, int, int, void *workspace, size_t, const int32_t *cu_host,
                            cudaStream_t st) {
    using namespace tc;
    // tokens in the packed [T_total, H, 128] tensors: B*T, with B == 1 when varlen
    const long long total = p.cu_seqlens ? (long long)p.T : (long long)p.N * p.T;
    static_assert(sizeof(TcParams) <= 4096, "kernel parameter block");
    TcParams P;
    memset(&P, 0, sizeof(P));
    P.p = p;
    P.status = static_cast<int *>(workspace);
    // Longest sequences first, so the block scheduler hands them out early.
    P.nperm = 0;
    if (cu_host && p.N <= kMaxPerm) {
        std::vector<int> idx(p.N);
        for (int i = 0; i < p.N; ++i) idx[i] = i;
        std::stable_sort(idx.begin(), idx.end(), [&](int a, int b) {
            return (cu_host[a + 1] - cu_host[a]) > (cu_host[b + 1] - cu_host[b]);
        });
        for (int i = 0; i < p.N; ++i) P.perm[i] = idx[i];
        P.nperm = p.N;
    }
    if (total <= 0) return cudaErrorInvalidValue;
    if (!make_map(&P.tq, p.q, total, p.H) || !make_map(&P.tk, p.k, total, p.H) ||
        !make_map(&P.tg, p.g, total, p.H) || !make_map(&P.tv, p.v, total, p.H))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaMemsetAsync(workspace, 0, sizeof(int), st);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kda_chunk_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_ALLOC);
    if (e != cudaSuccess) return e;
    const long long blocks = (long long)p.N * p.H;
    count_launch();
    kda_chunk_tc_kernel<<<(unsigned)blocks, NT, SMEM_ALLOC, st>>>(P);
    return cudaGetLastError();
}

}  // namespace kda
