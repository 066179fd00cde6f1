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
//   per chunk, with G the inclusive in-chunk cumsum of the clamped gate,
//   beta = sigmoid(logit), k^/q^ the L2-normalised rows and T' = T diag(beta),
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

namespace kda {
namespace tc {

using namespace sm100;

constexpr int C = 64;
constexpr int D = 128;
constexpr int NT = 256;
constexpr float kSpanMax = 80.f;           // e^80 = 5.5e34 stays finite in bf16 and fp32
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // bounded waits: 2 s

// ---- shared memory map (bytes from the 1024-aligned base) ----
constexpr uint32_t STG_Q = 0, STG_K = 16384, STG_G = 32768, STG_V = 49152;  // TMA staging, [64][128]
constexpr uint32_t AOPS = 65536;                                            // 72 KiB, two views:
// view 1, operands of the A_kk / A_qk products
constexpr uint32_t XKQO_H0 = AOPS + 0, YD_H0 = AOPS + 8192, XKQO_H1 = AOPS + 16384, YD_H1 = AOPS + 24576;
constexpr uint32_t YO_H0 = AOPS + 32768, YO_H1 = AOPS + 36864, XKQD = AOPS + 40960;  // XKQD: 2 x 16 KiB
// view 2, after those products: fp32 solve buffers, then W^T and D^T tiles
constexpr int LDS = 65;  // padded fp32 row stride of the 64x64 solve buffers
constexpr uint32_t LF = AOPS + 0, TF = AOPS + 16896, MF = AOPS + 33792, AQK = AOPS + 40960, TP = AOPS + 49152;
constexpr uint32_t WT = AOPS + 0, DT = AOPS + 16384;
constexpr uint32_t QT = AOPS + 73728, KT = QT + 16384, KH = KT + 16384, ST = KH + 16384;  // ST: 32 KiB
constexpr uint32_t MISC = ST + 32768;
constexpr uint32_t M_BETA = MISC, M_INVQ = MISC + 256, M_INVK = MISC + 512, M_G31 = MISC + 768,
                   M_G63 = MISC + 1280, M_GAM = MISC + 1792, M_BAR = MISC + 2304, M_TMEM = MISC + 2336;
constexpr uint32_t SMEM_BYTES = MISC + 2560;
constexpr uint32_t SMEM_ALLOC = SMEM_BYTES + 1024;  // slack for 1024-byte alignment
static_assert(LF + 64 * LDS * 4 <= TF && TF + 64 * LDS * 4 <= MF && MF + 32 * 33 * 4 <= AQK, "view 2");
static_assert(TP + 8192 <= AOPS + 73728 && DT + 16384 <= AQK, "view 2 tiles");
static_assert(SMEM_ALLOC <= 232448, "shared memory budget");

// ---- tensor memory columns ----
constexpr uint32_t TM_S = 0, TM_U = 128, TM_W = 192, TM_O = 256, TM_A = 320, TM_COLS = 512;

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

__device__ __forceinline__ float bf(const uint8_t *base, uint32_t off) {
    return __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(base + off));
}
__device__ __forceinline__ void st_bf(uint8_t *base, uint32_t off, float x) {
    *reinterpret_cast<__nv_bfloat16 *>(base + off) = __float2bfloat16_rn(x);
}

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
    float *sG31 = reinterpret_cast<float *>(sm + M_G31);
    float *sG63 = reinterpret_cast<float *>(sm + M_G63);
    float *sGam = reinterpret_cast<float *>(sm + M_GAM);
    float *Lf = reinterpret_cast<float *>(sm + LF);
    float *Tf = reinterpret_cast<float *>(sm + TF);
    float *Mf = reinterpret_cast<float *>(sm + MF);

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
    const uint32_t lane_sel = (uint32_t)(32 * (warp & 3)) << 16;  // this warp's TMEM lane quarter

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

    uint32_t ph_qkg = 0, ph_v = 0, ph_mma = 0;
    bool qkg_out = false, v_out = false, mma_out = false;  // thread 0's outstanding async work
    bool aborted = false;
    if (tid == 0 && nchunks > 0) { issue_qkg(bos); issue_v(bos); qkg_out = v_out = true; }

    const long long sbase_state = ((long long)n * H + h) * D * D;

    for (int ci = 0; ci < nchunks && !aborted; ++ci) {
        const long long t0 = bos + (long long)ci * C;
        const int L = (int)((eos - t0) < C ? (eos - t0) : C);
        const bool has_next = ci + 1 < nchunks;

        // ---------------- inputs of this chunk
        {
            bool ok = mbar_wait(bar_qkg, ph_qkg, kWaitLimitNs) && mbar_wait(bar_v, ph_v, kWaitLimitNs);
            ph_qkg ^= 1; ph_v ^= 1;
            if (tid == 0) qkg_out = v_out = false;
            if (__syncthreads_or(!ok)) { aborted = true; break; }
        }

        // ---------------- P1: beta, row norms of q and k (warp per row)
        if (tid < C) {
            const __nv_bfloat16 *bt = static_cast<const __nv_bfloat16 *>(p.beta);
            sbeta[tid] = tid < L ? sigmoidf_(__bfloat162float(bt[(t0 + tid) * H + h])) : 0.f;
        }
        for (int r = warp; r < C; r += NT / 32) {
            const int hf = lane >> 4, cc = (lane & 15) * 4;
            const uint32_t off = hf * 8192 + r * 128 + ((((cc >> 3) ^ (r & 7)) << 4) | ((cc & 7) << 1));
            const uint2 qv = *reinterpret_cast<const uint2 *>(sm + STG_Q + off);
            const uint2 kv = *reinterpret_cast<const uint2 *>(sm + STG_K + off);
            const __nv_bfloat162 *q2 = reinterpret_cast<const __nv_bfloat162 *>(&qv);
            const __nv_bfloat162 *k2 = reinterpret_cast<const __nv_bfloat162 *>(&kv);
            float sq = 0.f, sk = 0.f;
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const float2 a = __bfloat1622float2(q2[e]), b = __bfloat1622float2(k2[e]);
                sq += a.x * a.x + a.y * a.y;
                sk += b.x * b.x + b.y * b.y;
            }
            sq = warp_sum(sq); sk = warp_sum(sk);
            if (lane == 0) {
                sinvq[r] = r < L ? (p.use_l2 ? rsqrtf(sq + kL2Eps) : 1.f) : 0.f;
                sinvk[r] = r < L ? (p.use_l2 ? rsqrtf(sk + kL2Eps) : 1.f) : 0.f;
            }
        }

        // ---------------- P2: in-chunk cumsum of the gate, thread per (channel, 32-row block)
        const int c = tid & 127, blk = tid >> 7;
        float Gl[32];
        {
            float acc = 0.f;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const int r = 32 * blk + i;
                float gv = 0.f;
                if (r < L) {
                    gv = bf(sm + STG_G, sw128(r, c, 64));
                    if (p.has_lb) gv = fmaxf(gv, p.lb);
                }
                acc += gv;
                Gl[i] = acc;
            }
        }
        if (blk == 0) sG31[c] = Gl[31];
        __syncthreads();
        if (blk == 1) {
            const float b = sG31[c];
#pragma unroll
            for (int i = 0; i < 32; ++i) Gl[i] += b;
            sG63[c] = Gl[31];
            sGam[c] = expf(Gl[31]);
        }
        const float Gm = Gl[15];
        const int span_bad = fmaxf(Gl[0] - Gm, Gm - Gl[31]) > kSpanMax;
        const bool fb = __syncthreads_or(span_bad) != 0;  // also publishes sG63 / sGam

        // ---------------- P3: bf16 operand tiles
        {
            const float G31 = blk == 0 ? Gl[31] : sG31[c];
            const float G63 = sG63[c];
            const int hf = c >> 6, cc = c & 63;
            if (!fb) {
                const float Emid = __expf(Gm);
                const float Fkh = __expf(G63 - Gm);
                const float Foff = blk == 0 ? __expf(G31 - Gm) : __expf(Gm - G31);
                const uint32_t yd = hf ? YD_H1 : YD_H0, yo = hf ? YO_H1 : YO_H0, xo = hf ? XKQO_H1 : XKQO_H0;
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int r = 32 * blk + i;
                    const uint32_t o64 = sw128(r, c, 64);
                    const float kh = bf(sm + STG_K, o64) * sinvk[r];
                    const float qh = bf(sm + STG_Q, o64) * sinvq[r];
                    const float a = Gl[i] - Gm;
                    const float ed = __expf(a), ydf = __expf(-a);
                    const float xk = kh * ed, xq = qh * ed, y = kh * ydf;
                    st_bf(sm, XKQD + sw128(r, c, 128), xk);
                    st_bf(sm, XKQD + sw128(64 + r, c, 128), xq);
                    st_bf(sm, yd + sw128(r, cc, 64), y);
                    st_bf(sm, QT + o64, xq * Emid);
                    st_bf(sm, KT + o64, xk * Emid);
                    st_bf(sm, KH + o64, y * Fkh);
                    if (blk == 0) {
                        st_bf(sm, yo + sw128(r, cc, 32), y * Foff);
                    } else {
                        st_bf(sm, xo + sw128(i, cc, 64), xk * Foff);
                        st_bf(sm, xo + sw128(32 + i, cc, 64), xq * Foff);
                    }
                }
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int r = 32 * blk + i;
                    const uint32_t o64 = sw128(r, c, 64);
                    const float kh = bf(sm + STG_K, o64) * sinvk[r];
                    const float qh = bf(sm + STG_Q, o64) * sinvq[r];
                    const float eg = expf(Gl[i]);
                    st_bf(sm, QT + o64, qh * eg);
                    st_bf(sm, KT + o64, kh * eg);
                    st_bf(sm, KH + o64, kh * expf(G63 - Gl[i]));
                }
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // ---------------- A_kk / A_qk products; next chunk's q, k, g loads
        if (tid == 0 && !fb) {
            if (has_next) { issue_qkg(t0 + C); qkg_out = true; }
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t ko = (kk >> 2) * 16384 + (kk & 3) * 32;
                const uint32_t yb = (kk >> 2) ? YD_H1 : YD_H0, ob = (kk >> 2) ? YO_H1 : YO_H0;
                mma_bf16(tb + TM_A, sdesc_sw128(sb + XKQD + ko, 16, 1024),
                         sdesc_sw128(sb + yb + (kk & 3) * 32, 16, 1024), ID_A1, kk > 0);
                mma_bf16(tb + TM_A + 64, sdesc_sw128(sb + XKQO_H0 + ko, 16, 1024),
                         sdesc_sw128(sb + ob + (kk & 3) * 32, 16, 1024), ID_A2, kk > 0);
            }
            mma_commit(bar_mma);
            mma_out = true;
        }

        // ---------------- state refresh (overlaps the products above):
        // bf16 copy of S^T for this chunk's MMAs, and S^T diag(e^{G_last}) back into TMEM
        {
            const int v = 32 * (warp & 3) + lane;
            const int cb = (warp >> 2) * 64;
#pragma unroll
            for (int b = 0; b < 2; ++b) {
                const int c0 = cb + 32 * b;
                float x[32];
                if (ci == 0) {
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        x[j] = p.S0 ? p.S0[sbase_state + (long long)(c0 + j) * D + v] : 0.f;
                } else {
                    tmem_ld32(tb + TM_S + lane_sel + c0, x);
                    tmem_ld_wait();
                }
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    uint4 pk;
                    pk.x = pack_bf16x2(x[8 * q4 + 0], x[8 * q4 + 1]);
                    pk.y = pack_bf16x2(x[8 * q4 + 2], x[8 * q4 + 3]);
                    pk.z = pack_bf16x2(x[8 * q4 + 4], x[8 * q4 + 5]);
                    pk.w = pack_bf16x2(x[8 * q4 + 6], x[8 * q4 + 7]);
                    *reinterpret_cast<uint4 *>(sm + ST + sw128_chunk(v, c0 + 8 * q4, 128)) = pk;
                }
#pragma unroll
                for (int j = 0; j < 32; ++j) x[j] *= sGam[c0 + j];
                tmem_st32(tb + TM_S + lane_sel + c0, x);
            }
            tmem_st_wait();
        }

        // ---------------- A results -> beta-scaled L (fp32) and A_qk (bf16 tile)
        if (!fb) {
            bool ok = mbar_wait(bar_mma, ph_mma, kWaitLimitNs);
            ph_mma ^= 1;
            if (tid == 0) mma_out = false;
            if (__syncthreads_or(!ok)) { aborted = true; break; }
            tc_fence_after();
            if (warp < 4) {
                const int i = lane;
                float va[32], vb[32];
                if (warp == 0 || warp == 2) tmem_ld32(tb + TM_A + lane_sel + 0, va);
                else tmem_ld32(tb + TM_A + lane_sel + 32, va);
                if (warp < 2) tmem_ld32(tb + TM_A + lane_sel + 64, vb);
                tmem_ld_wait();
                if (warp == 0) {
                    const float b0 = sbeta[i], b1 = sbeta[32 + i];
#pragma unroll
                    for (int s = 0; s < 32; ++s) {
                        Lf[i * LDS + s] = s < i ? b0 * va[s] : 0.f;
                        Lf[i * LDS + 32 + s] = 0.f;
                        Lf[(32 + i) * LDS + s] = b1 * vb[s];
                    }
                } else if (warp == 1) {
                    const float b1 = sbeta[32 + i];
#pragma unroll
                    for (int s = 0; s < 32; ++s) Lf[(32 + i) * LDS + 32 + s] = s < i ? b1 * va[s] : 0.f;
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        uint4 pk;
                        pk.x = pack_bf16x2(vb[8 * q4 + 0], vb[8 * q4 + 1]);
                        pk.y = pack_bf16x2(vb[8 * q4 + 2], vb[8 * q4 + 3]);
                        pk.z = pack_bf16x2(vb[8 * q4 + 4], vb[8 * q4 + 5]);
                        pk.w = pack_bf16x2(vb[8 * q4 + 6], vb[8 * q4 + 7]);
                        *reinterpret_cast<uint4 *>(sm + AQK + sw128_chunk(32 + i, 8 * q4, 64)) = pk;
                    }
                } else {
                    const int row = warp == 2 ? i : 32 + i;
                    const int col0 = warp == 2 ? 0 : 32;
                    float m[32];
#pragma unroll
                    for (int s = 0; s < 32; ++s) m[s] = s <= i ? va[s] : 0.f;
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        uint4 pk;
                        pk.x = pack_bf16x2(m[8 * q4 + 0], m[8 * q4 + 1]);
                        pk.y = pack_bf16x2(m[8 * q4 + 2], m[8 * q4 + 3]);
                        pk.z = pack_bf16x2(m[8 * q4 + 4], m[8 * q4 + 5]);
                        pk.w = pack_bf16x2(m[8 * q4 + 6], m[8 * q4 + 7]);
                        *reinterpret_cast<uint4 *>(sm + AQK + sw128_chunk(row, col0 + 8 * q4, 64)) = pk;
                        if (warp == 2)
                            *reinterpret_cast<uint4 *>(sm + AQK + sw128_chunk(row, 32 + 8 * q4, 64)) =
                                make_uint4(0u, 0u, 0u, 0u);
                    }
                }
            }
        } else {
            // exact A_kk / A_qk on CUDA cores: warp per row r, lanes over channels,
            // walking s downwards while accumulating the gate between s and r
            for (int r = warp; r < C; r += NT / 32) {
                float kr[4], qr[4], dg[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const uint32_t o = sw128(r, lane + 32 * u, 64);
                    kr[u] = bf(sm + STG_K, o) * sinvk[r];
                    qr[u] = bf(sm + STG_Q, o) * sinvq[r];
                    dg[u] = 0.f;
                }
                for (int s = r; s >= 0; --s) {
                    float akk = 0.f, aqk = 0.f;
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const uint32_t o = sw128(s, lane + 32 * u, 64);
                        const float e = expf(dg[u]) * bf(sm + STG_K, o) * sinvk[s];
                        akk = fmaf(kr[u], e, akk);
                        aqk = fmaf(qr[u], e, aqk);
                        float gv = 0.f;
                        if (s < L) {
                            gv = bf(sm + STG_G, o);
                            if (p.has_lb) gv = fmaxf(gv, p.lb);
                        }
                        dg[u] += gv;
                    }
                    akk = warp_sum(akk); aqk = warp_sum(aqk);
                    if (lane == 0) {
                        Lf[r * LDS + s] = s < r ? sbeta[r] * akk : 0.f;
                        st_bf(sm, AQK + sw128(r, s, 64), aqk);
                    }
                }
                for (int s = r + 1 + lane; s < C; s += 32) {
                    Lf[r * LDS + s] = 0.f;
                    st_bf(sm, AQK + sw128(r, s, 64), 0.f);
                }
            }
            fence_proxy_async_smem();
            __syncthreads();
            if (tid == 0 && has_next) { issue_qkg(t0 + C); qkg_out = true; }
        }
        __syncthreads();

        // ---------------- T = (I + L)^-1 by blocks: diagonal 32x32 by forward substitution
        if (warp < 2) {
            const int b = warp, j = lane;
            float t[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                float s = i == j ? 1.f : 0.f;
                const float *Lrow = Lf + (32 * b + i) * LDS + 32 * b;
#pragma unroll
                for (int k = 0; k < i; ++k) s = fmaf(-Lrow[k], t[k], s);
                t[i] = s;
            }
#pragma unroll
            for (int i = 0; i < 32; ++i) Tf[(32 * b + i) * LDS + 32 * b + j] = t[i];
        }
        __syncthreads();
        {   // M1 = L10 T00
            const int j = lane;
#pragma unroll
            for (int ii = 0; ii < 4; ++ii) {
                const int i = warp * 4 + ii;
                float acc = 0.f;
#pragma unroll 8
                for (int k = 0; k < 32; ++k) acc = fmaf(Lf[(32 + i) * LDS + k], Tf[k * LDS + j], acc);
                Mf[i * 33 + j] = acc;
            }
        }
        __syncthreads();
        {   // T10 = -T11 M1
            const int j = lane;
#pragma unroll
            for (int ii = 0; ii < 4; ++ii) {
                const int i = warp * 4 + ii;
                float acc = 0.f;
#pragma unroll 8
                for (int k = 0; k < 32; ++k) acc = fmaf(Tf[(32 + i) * LDS + 32 + k], Mf[k * 33 + j], acc);
                Tf[(32 + i) * LDS + j] = -acc;
            }
        }
        __syncthreads();
        // T' = T diag(beta) as a bf16 tile [r][s]
        for (int q = tid; q < 512; q += NT) {
            const int r = q >> 3, s0 = (q & 7) * 8;
            float m[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int s = s0 + e;
                m[e] = s <= r ? Tf[r * LDS + s] * sbeta[s] : 0.f;
            }
            uint4 pk;
            pk.x = pack_bf16x2(m[0], m[1]); pk.y = pack_bf16x2(m[2], m[3]);
            pk.z = pack_bf16x2(m[4], m[5]); pk.w = pack_bf16x2(m[6], m[7]);
            *reinterpret_cast<uint4 *>(sm + TP + sw128_chunk(r, s0, 64)) = pk;
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // ---------------- U^T = V^T T'^T, W^T = Ktil^T T'^T
        if (tid == 0) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint64_t bdesc = sdesc_sw128(sb + TP + kk * 32, 16, 1024);
                mma_bf16(tb + TM_U, sdesc_sw128(sb + STG_V + kk * 2048, 8192, 1024), bdesc, ID_UW, kk > 0);
                mma_bf16(tb + TM_W, sdesc_sw128(sb + KT + kk * 2048, 8192, 1024), bdesc, ID_UW, kk > 0);
            }
            mma_commit(bar_mma);
            mma_out = true;
        }
        {
            bool ok = mbar_wait(bar_mma, ph_mma, kWaitLimitNs);
            ph_mma ^= 1;
            if (tid == 0) mma_out = false;
            if (__syncthreads_or(!ok)) { aborted = true; break; }
        }
        tc_fence_after();
        {   // W^T (lane c, columns r) -> bf16 tile [c][r]
            const int cr = 32 * (warp & 3) + lane, r0 = (warp >> 2) * 32;
            float x[32];
            tmem_ld32(tb + TM_W + lane_sel + r0, x);
            tmem_ld_wait();
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                uint4 pk;
                pk.x = pack_bf16x2(x[8 * q4 + 0], x[8 * q4 + 1]);
                pk.y = pack_bf16x2(x[8 * q4 + 2], x[8 * q4 + 3]);
                pk.z = pack_bf16x2(x[8 * q4 + 4], x[8 * q4 + 5]);
                pk.w = pack_bf16x2(x[8 * q4 + 6], x[8 * q4 + 7]);
                *reinterpret_cast<uint4 *>(sm + WT + sw128_chunk(cr, r0 + 8 * q4, 128)) = pk;
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // ---------------- D^T = U^T - S^T W^T ; O^T = S^T Qtil^T ; next chunk's v load
        if (tid == 0) {
            if (has_next) { issue_v(t0 + C); v_out = true; }
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint64_t adesc = sdesc_sw128(sb + ST + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
                mma_bf16(tb + TM_U, adesc, sdesc_sw128(sb + WT + kk * 2048, 8192, 1024), ID_DL, 1);
                mma_bf16(tb + TM_O, adesc, sdesc_sw128(sb + QT + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024),
                         ID_O, kk > 0);
            }
            mma_commit(bar_mma);
            mma_out = true;
        }
        {
            bool ok = mbar_wait(bar_mma, ph_mma, kWaitLimitNs);
            ph_mma ^= 1;
            if (tid == 0) mma_out = false;
            if (__syncthreads_or(!ok)) { aborted = true; break; }
        }
        tc_fence_after();
        {   // D^T (lane v, columns s) -> bf16 tile [v][s]
            const int v = 32 * (warp & 3) + lane, s0 = (warp >> 2) * 32;
            float x[32];
            tmem_ld32(tb + TM_U + lane_sel + s0, x);
            tmem_ld_wait();
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                uint4 pk;
                pk.x = pack_bf16x2(x[8 * q4 + 0], x[8 * q4 + 1]);
                pk.y = pack_bf16x2(x[8 * q4 + 2], x[8 * q4 + 3]);
                pk.z = pack_bf16x2(x[8 * q4 + 4], x[8 * q4 + 5]);
                pk.w = pack_bf16x2(x[8 * q4 + 6], x[8 * q4 + 7]);
                *reinterpret_cast<uint4 *>(sm + DT + sw128_chunk(v, s0 + 8 * q4, 128)) = pk;
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // ---------------- O^T += D^T A_qk^T ; S^T += D^T Khat
        if (tid == 0) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint64_t adesc = sdesc_sw128(sb + DT + kk * 32, 16, 1024);
                mma_bf16(tb + TM_O, adesc, sdesc_sw128(sb + AQK + kk * 32, 16, 1024), ID_O, 1);
                mma_bf16(tb + TM_S, adesc, sdesc_sw128(sb + KH + kk * 2048, 8192, 1024), ID_S, 1);
            }
            mma_commit(bar_mma);
            mma_out = true;
        }
        {
            bool ok = mbar_wait(bar_mma, ph_mma, kWaitLimitNs);
            ph_mma ^= 1;
            if (tid == 0) mma_out = false;
            if (__syncthreads_or(!ok)) { aborted = true; break; }
        }
        tc_fence_after();
        {   // O^T (lane v, columns r) -> o[t0 + r, h, v]
            const int v = 32 * (warp & 3) + lane, r0 = (warp >> 2) * 32;
            float x[32];
            tmem_ld32(tb + TM_O + lane_sel + r0, x);
            tmem_ld_wait();
            __nv_bfloat16 *O = static_cast<__nv_bfloat16 *>(p.o);
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int r = r0 + j;
                if (r < L) O[((t0 + r) * H + h) * D + v] = __float2bfloat16_rn(p.scale * x[j]);
            }
        }
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
    }

    if (!aborted && p.S_out) {
        const int v = 32 * (warp & 3) + lane;
        const int cb = (warp >> 2) * 64;
#pragma unroll
        for (int b = 0; b < 2; ++b) {
            const int c0 = cb + 32 * b;
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
    }

    if (aborted && tid == 0) {
        // let copies and products already in flight land before the CTA leaves
        if (qkg_out) mbar_wait(bar_qkg, ph_qkg, kWaitLimitNs);
        if (v_out) mbar_wait(bar_v, ph_v, kWaitLimitNs);
        if (mma_out) mbar_wait(bar_mma, ph_mma, kWaitLimitNs);
        if (P.status) atomicOr(P.status, 1);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tb, TM_COLS);
    }
}

// ------------------------------------------------------------------ host side

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// [T_total, H, 128] bf16 viewed as a 3-D tensor (channel, head, token); one
// box = 64 channels x 1 head x 64 tokens, 128-byte swizzled.
bool make_map(CUtensorMap *m, const void *base, long long ttot, int H) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)H, (cuuint64_t)ttot};
    cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)H * D * 2};
    cuuint32_t box[3] = {64, 1, 64};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

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
    kda_chunk_tc_kernel<<<(unsigned)blocks, NT, SMEM_ALLOC, st>>>(P);
    return cudaGetLastError();
}

}  // namespace kda
