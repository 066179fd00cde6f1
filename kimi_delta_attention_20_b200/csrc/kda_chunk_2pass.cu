// Chunkwise KDA forward in two passes on the 5th-generation tensor cores, bf16
// inputs, d_k = d_v = 128, chunk C = 64.
//
// The operator is the `chunk_kda` boundary of page "K3/kda/ops/api.py"; its
// result is the token recurrence of page "atlas_core/kimi_k3/kda.rs". Per chunk
// (G the inclusive in-chunk cumsum of the gate, beta the write strengths, T' =
// (I + diag(beta) A_kk)^-1 diag(beta)), everything that does not involve the
// state S depends on that chunk alone:
//   A_kk[r,s] = sum_c k^_r k^_s e^{G_r-G_s} (s<r), A_qk likewise with q^_r (s<=r)
//   W = T' (k^ e^G),  Qtil = q^ e^G,  Khat = k^ e^{G_last-G}
// and only four products carry the state from chunk to chunk:
//   D = T'V - W S,  O = Qtil S + A_qk D,  S <- diag(e^{G_last}) S + Khat^T D.
//
// Pass 1 (`kda_tp_intra_kernel`) computes the chunk-local part of every
// (chunk, head) at once -- all chunks of all sequences are independent -- with
// two 256-thread CTAs per SM walking a flat list of work items, and writes one
// record per (chunk, head): W^T, Qtil^T, Khat^T, T' and A_qk as bf16 tiles
// already laid out as the 128-byte-swizzled shared-memory images the tensor
// cores read, plus e^{G_last} and the row norms. Its layout is by key channel:
// three tensor-core products against constant tiles put the in-chunk cumsum
// G^T = g^T Tri^T and the transposes k^T, q^T into tensor memory (lane = key
// channel), so each thread holds one channel for a run of rows, takes its block
// references from its own registers and writes every operand tile as whole
// 128-byte rows; the tiles go to the record with bulk copies.
// Pass 2 (`kda_tp_state_kernel`) walks each (sequence, head) through its
// chunks with the fp32 state S^T resident in tensor memory; per chunk it
// bulk-copies the record and the v tile (TMA) into a double-buffered stage and
// issues the four state products, so the sequential part of the work is short.
//
// Normalisation of q and k is deferred: the products use raw rows, and 1/|k_s|
// scales the columns of D, 1/|q_r| the output rows, beta/|k_s| the columns of
// the W factor (all algebraically identical to normalising first). The gated
// products use 32-row blocks with middle references (factors up to e^{span});
// a chunk whose gate moves by more than kSpanMax inside a block is queued and
// its record is rewritten by `kda_tp_exact_kernel`, which computes every
// product on CUDA cores from exponent differences alone (any gate).
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <functional>
#include <queue>
#include <vector>

#include "kda_common.cuh"
#include "kda_sm100.cuh"
#include "kda_tc_util.cuh"
#include "kda_stage.cuh"
#include "kda_seg.cuh"
#include "kda_record.cuh"

namespace kda {
namespace tp {

using namespace sm100;
using namespace tcu;

constexpr int C = 64;
constexpr int D = 128;
constexpr float kSpanMax = 80.f;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // bounded waits: 2 s

// the record of one (chunk, head): kda_record.cuh

// ============================================================== pass 1
constexpr int NT1 = 256;  // 8 warps, two CTAs per SM
// Shared memory (bytes from a 1024-aligned base). Phases reuse regions:
//   inputs      KQ: 2 channel halves x [128 rows: k tokens 0..63, q tokens 0..63][128 B]
//               GS: 2 channel halves x [64 tokens][128 B] (the gate)
//               TRI, IDT: [64][64] bf16 constant tiles (bulk-copied with the inputs);
//               GLO: low part of a split gate
//   operands    XK, XQ: X^T images [128 c][64 r] of k e^{G-G_m}, q e^{G-G_m}
//               YT: Y^T [128 c][64 s] of k e^{G_m-G};  YP: Y'^T of k e^{G_47-G} (s < 32)
//               QT, KH: the record's Qtil^T and Khat^T images
//   inverse     LF: fp32 L [64][68];  TF: fp32 T [64][72];  TW: bf16 T diag(beta/|k|)
//               AQK, TPU: the record's A_qk and T' images;  WT: the record's W^T image
constexpr uint32_t KQ = 0, GS = 32768;
constexpr uint32_t XK = 0, XQ = 16384, YT = 32768;
constexpr uint32_t R2 = 49152;
constexpr uint32_t TRI = R2, IDT = R2 + 8192, GLO = R2 + 16384;
constexpr uint32_t QT = R2, KH = R2 + 16384, YP = R2 + 32768;
constexpr int LDS = 68, LDT = 72;  // row strides (floats) of L and T: 16-byte rows, fragment loads conflict-free
constexpr uint32_t LF = 16384, TF = 33792, TW = 53248;
constexpr uint32_t AQK = YP, TPU = YP + 8192, WT = KH;
constexpr uint32_t MISC1 = 98304;
constexpr uint32_t M1_REC = MISC1,           // record misc image: gamma[128], invq[64], invk[64]
    M1_GAM = MISC1, M1_INVQ = MISC1 + 512, M1_INVK = MISC1 + 768,
                   M1_BETA = MISC1 + 1024,   // [64] f32
                   M1_GX = MISC1 + 1280,     // [128] f32: gate totals of rows 0..31 (gate forms)
                   M1_DTB = MISC1 + 1792,    // [128] f32: dt_bias of the item's head
                   M1_BAR = MISC1 + 2304, M1_TMEM = MISC1 + 2336,
                   M1_XS = MISC1 + 2432;     // fp32 X [32][LDX] of the inverse's last step
constexpr int LDXS = 40;  // row stride (floats) of X: fragment loads conflict-free
constexpr uint32_t SMEM1_BYTES = M1_XS + 32 * LDXS * 4;
constexpr uint32_t SMEM1_ALLOC = SMEM1_BYTES + 1024;
static_assert(LF + 64 * LDS * 4 <= TF && TF + 64 * LDT * 4 <= TW && TW + 8192 <= KH, "inverse scratch");
static_assert(TW % 1024 == 0 && AQK % 1024 == 0 && TPU % 1024 == 0 && TPU + 8192 == MISC1, "tile alignment");
static_assert(2 * (SMEM1_ALLOC + 1024) <= 233472, "two CTAs per SM");

// tensor memory (256 columns): G^T, k^T, q^T; then the A products (one N = 128 product
// against [Y | Y']: D1 in columns 0..63, D2 in 64..127); then W in two K halves
constexpr uint32_t TM_G = 0, TM_K = 64, TM_Q = 128;
constexpr uint32_t TM_A1 = 0, TM_A2 = 64, TM_W0 = 128, TM_W1 = 192, TM1_COLS = 256;
static_assert(YP - YT == 49152, "Y and Y' are the two N groups of one operand (LBO 48 KB)");

constexpr uint32_t ID_T = idesc_bf16(128, 64, true, false);   // g^T Tri^T, k^T I, q^T I
constexpr uint32_t ID_A = idesc_bf16(128, 128, true, true);   // [X_k; X_q] [Y | Y']^T
constexpr uint32_t ID_W = idesc_bf16(128, 64, false, false);  // X_k^T T_w^T

struct IntraParams {
    CUtensorMap tq, tk, tg;
    ChunkParams p;
    uint8_t *rec;            // records, index (global chunk) * H + head
    const int2 *chunk_tok;   // varlen: per global chunk (first token, valid rows)
    const int *n_chunks;     // varlen: device count of global chunks
    int cpr;                 // batch: chunks per batch row
    long long n_items;       // upper bound of (global chunk, head) items
    int split_gate;          // the clamped gate needs a low bf16 part (bound not a bf16 value)
    const uint8_t *consts;   // the Tri and I tile images (16 KB, written by kda_tp_prep)
    int *fix_count;          // items whose gate span needs the exact kernel
    int *fix_list;
    int *status;
};

struct Item {
    int h;
    int t0;        // first token of the chunk
    int L;         // valid rows
    long long gc;  // global chunk index
};

// The chunk's tokens of work item (global chunk gc, head h); false past the end
__device__ __forceinline__ bool decode_chunk(const IntraParams &P, long long gc, int h, int nch, Item &it) {
    const ChunkParams &p = P.p;
    it.h = h;
    it.gc = gc;
    if (P.chunk_tok) {  // every table entry has rows: the result does not wait for the load
        if (gc >= nch) return false;
        const int2 e = P.chunk_tok[gc];
        it.t0 = e.x;
        it.L = e.y;
        return true;
    } else {  // gc < 2^31 (checked on the host): 32-bit division
        const unsigned n = (unsigned)gc / (unsigned)P.cpr;
        if ((int)n >= p.N) return false;
        const int ci = (int)((unsigned)gc - n * (unsigned)P.cpr);
        it.t0 = (int)n * p.T + ci * C;
        it.L = min(C, p.T - ci * C);
    }
    return it.L > 0;
}
// (global chunk, head) of flat item index `item` (= gc * H + h)
__device__ __forceinline__ bool decode_item(const IntraParams &P, long long item, int nch, Item &it) {
    if (item >= P.n_items) return false;
    return decode_chunk(P, item / P.p.H, (int)(item % P.p.H), nch, it);
}

// 8 bf16 of an unpacked register pair set -> one 16-byte chunk
__device__ __forceinline__ uint4 pack16B(const float2 (&f)[4]) { return pack8x2(f); }

__global__ void __launch_bounds__(NT1, 2) kda_tp_intra_kernel(const __grid_constant__ IntraParams P) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const ChunkParams &p = P.p;
    const int tid = threadIdx.x, lane = tid & 31;
    const int warp = __shfl_sync(0xffffffffu, tid >> 5, 0);  // warp-uniform by construction
    const int H = p.H;
    constexpr int kMma = 0, kTma = NT1 - 32;  // warp 0 issues the MMAs, thread kTma the copies
    constexpr float kL2e = 1.4426950408889634f;

    uint64_t *bar_in = reinterpret_cast<uint64_t *>(sm + M1_BAR);
    uint64_t *bar_mma = bar_in + 1;
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(sm + M1_TMEM);
    float *sbeta = reinterpret_cast<float *>(sm + M1_BETA);
    float *sinvq = reinterpret_cast<float *>(sm + M1_INVQ);
    float *sinvk = reinterpret_cast<float *>(sm + M1_INVK);
    float *sgam = reinterpret_cast<float *>(sm + M1_GAM);
    float *sGX = reinterpret_cast<float *>(sm + M1_GX);
    float *sDtb = reinterpret_cast<float *>(sm + M1_DTB);
    float *Lf = reinterpret_cast<float *>(sm + LF);
    float *Tf = reinterpret_cast<float *>(sm + TF);
    float *Xs = reinterpret_cast<float *>(sm + M1_XS);

    if (warp == 0) { tmem_alloc(s_tmem, TM1_COLS); tmem_relinquish(); }
    if (tid == 32) {
        mbar_init(bar_in, 1); mbar_init(bar_mma, 1);
        fence_mbar_init();
        tma_prefetch_desc(&P.tq); tma_prefetch_desc(&P.tk); tma_prefetch_desc(&P.tg);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tb = *s_tmem;
    const uint32_t sb = smem_u32(sm);
    // 128-byte-swizzled operand at `off`: K-major (lbo unused) or MN-major (lbo = step
    // between 64-element groups along M/N); 8-row groups 1024 bytes apart
    const uint64_t dK = sdesc_sw128(sb, 16, 1024), dA8 = sdesc_sw128(sb, 8192, 1024),
                   dA16 = sdesc_sw128(sb, 16384, 1024), dYY = sdesc_sw128(sb, YP - YT, 1024);
    auto desc = [&](uint32_t off, uint32_t lbo) {
        return (lbo == 16 ? dK : lbo == 8192 ? dA8 : dA16) + (uint64_t)(off >> 4);
    };
    // channel layout: thread (quarter, hw) owns key channel c (tensor-memory lane c)
    // and rows 32 hw .. 32 hw + 31; hw also splits columns in the row-layout phases
    const int quarter = warp & 3, hw = warp >> 2;
    const int c = 32 * quarter + lane;
    const uint32_t lane_sel = (uint32_t)(32 * quarter) << 16;
    const int gmode = p.gate_mode;
    const int nch = P.chunk_tok ? *P.n_chunks : 0;

    uint32_t ph_in = 0, ph_mma = 0;
    bool in_out = false, mma_out = false, aborted = false;
    // the phase advances only when it completed, so an abort waits on the pending one
    auto wait_all = [&](uint64_t *bar, uint32_t &ph) -> bool {
        bool ok = true;
        if (warp == 0) ok = mbar_wait(bar, ph, kWaitLimitNs);
        const bool stop = __syncthreads_or(!ok) != 0;
        if (!stop) ph ^= 1;
        return stop;
    };
    auto issue_in = [&](const Item &it) {
        mbar_arrive_expect_tx(bar_in, 4 * 16384);
        bulk_load(sm + TRI, P.consts, 16384, bar_in);
        for (int hf = 0; hf < 2; ++hf) {
            tma_load_3d(sm + KQ + hf * 16384, &P.tk, bar_in, hf * 64, it.h, it.t0);
            tma_load_3d(sm + KQ + hf * 16384 + 8192, &P.tq, bar_in, hf * 64, it.h, it.t0);
            tma_load_3d(sm + GS + hf * 8192, &P.tg, bar_in, hf * 64, it.h, it.t0);
        }
    };

    // raw bits: the load is consumed (converted) only when the item starts
    const unsigned short *bt16 = reinterpret_cast<const unsigned short *>(p.beta);
    auto load_beta = [&](const Item &it) -> unsigned short {
        return tid < it.L ? bt16[((long long)it.t0 + tid) * H + it.h] : (unsigned short)0;
    };

    // items blockIdx.x + k gridDim.x, walked as (global chunk, head) with the stride split once
    const int step_h = (int)(gridDim.x % H);
    const long long step_c = gridDim.x / H;
    long long item = blockIdx.x;
    Item cur;
    bool have = decode_item(P, item, nch, cur);
    // (a test of the bounded waits leaves the first copy unissued: the first wait gives up)
    if (have && tid == kTma && !p.stall_first_wait) { issue_in(cur); in_out = true; }
    unsigned short beta_raw = (have && tid < C) ? load_beta(cur) : (unsigned short)0;

    while (have) {
        const long long nitem = item + gridDim.x;
        Item nxt;
        bool have_next = false;
        if (nitem < P.n_items) {
            int nh = cur.h + step_h;
            long long ngc = cur.gc + step_c;
            if (nh >= H) { nh -= H; ++ngc; }
            have_next = decode_chunk(P, ngc, nh, nch, nxt);
        }
        const int h = cur.h, L = cur.L;
        uint8_t *rec = P.rec + (cur.gc * H + h) * (long long)REC_BYTES;

        // ---------------- per-item scalars (beta was loaded one item ahead)
        if (tid < C) sbeta[tid] = tid < L ? beta_value(__uint_as_float((uint32_t)beta_raw << 16), p.beta_prob) : 0.f;
        const float rate = gmode != kGateLog ? expf(p.A_log[h]) : 0.f;
        if (gmode != kGateLog && tid < D) sDtb[tid] = p.dt_bias ? p.dt_bias[h * D + tid] : 0.f;
        // the previous item's record stores must have read their sources (GLO, misc)
        if (tid == kTma) bulk_wait_read_all();
        if (wait_all(bar_in, ph_in)) { aborted = true; break; }
        if (tid == kTma) in_out = false;

        // ---------------- rows past the sequence end: zero k, q and the gate input
        if (L < C) {
            for (int e = tid; e < 3072; e += NT1) {
                uint32_t off;
                int tok;
                if (e < 2048) {
                    const int row = (e >> 3) & 127;
                    tok = row & 63;
                    off = KQ + (e >> 10) * 16384 + row * 128 + (e & 7) * 16;
                } else {
                    const int e2 = e - 2048, row = (e2 >> 3) & 63;
                    tok = row;
                    off = GS + (e2 >> 9) * 8192 + row * 128 + (e2 & 7) * 16;
                }
                if (tok >= L) sts128(sm, off, make_uint4(0u, 0u, 0u, 0u));
            }
            __syncthreads();
        }

        // ---------------- the gate: clamp in place for the tensor-core cumsum (a low bf16
        // part when the bound is not a bf16 value), or the in-kernel gate forms summed in
        // fp32 on the CUDA cores straight into tensor memory
        if (gmode == kGateLog) {
            if (p.has_lb && !P.split_gate) {
                const __nv_bfloat162 lb2 = __float2bfloat162_rn(p.lb);
#pragma unroll
                for (int e = tid; e < 1024; e += NT1) {
                    uint4 u = lds128(sm + GS, e * 16);
                    __nv_bfloat162 *b2 = reinterpret_cast<__nv_bfloat162 *>(&u);
#pragma unroll
                    for (int q = 0; q < 4; ++q) b2[q] = __hmax2(b2[q], lb2);
                    sts128(sm, GS + e * 16, u);
                }
            } else if (p.has_lb) {
                for (int e = tid; e < 1024; e += NT1) {
                    float2 f[4], hi[4], lo[4];
                    unpack8x2(lds128(sm + GS, e * 16), f);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const float2 v = make_float2(fmaxf(f[q].x, p.lb), fmaxf(f[q].y, p.lb));
                        const __nv_bfloat162 hb = __float22bfloat162_rn(v);
                        hi[q] = __bfloat1622float2(hb);
                        lo[q] = make_float2(v.x - hi[q].x, v.y - hi[q].y);
                    }
                    sts128(sm, GS + e * 16, pack8x2(hi));
                    sts128(sm, GLO + e * 16, pack8x2(lo));
                }
            }
        } else {
            const float bias = sDtb[c];
            float Gv[32];
            float run = 0.f;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int r = 32 * hw + j;
                const float x = bf(sm + GS, sw128(r, c, 64));
                run += r < L ? gate_fast(x, bias, rate, gmode, p.lb) : 0.f;
                Gv[j] = run;
            }
            if (hw == 0) sGX[c] = run;
            __syncthreads();
            if (hw == 1) {
                const float off = sGX[c];
#pragma unroll
                for (int j = 0; j < 32; ++j) Gv[j] += off;
            }
            tmem_st32(tb + lane_sel + TM_G + 32 * hw, Gv);
            tmem_st_wait();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // ---------------- tensor core: G^T = g^T Tri^T, k^T = k^T I, q^T = q^T I (lane = channel)
        if (warp == 0) {
            const uint32_t ld = elect_one();
            if (gmode == kGateLog) {
#pragma unroll
                for (int kq = 0; kq < 4; ++kq)
                    mma_bf16_by(ld, tb + TM_G, desc(GS + kq * 2048, 8192), desc(TRI + kq * 32, 16), ID_T, kq > 0);
                if (p.has_lb && P.split_gate) {
#pragma unroll
                    for (int kq = 0; kq < 4; ++kq)
                        mma_bf16_by(ld, tb + TM_G, desc(GLO + kq * 2048, 8192), desc(TRI + kq * 32, 16), ID_T, 1);
                }
            }
#pragma unroll
            for (int kq = 0; kq < 4; ++kq)
                mma_bf16_by(ld, tb + TM_K, desc(KQ + kq * 2048, 16384), desc(IDT + kq * 32, 16), ID_T, kq > 0);
#pragma unroll
            for (int kq = 0; kq < 4; ++kq)
                mma_bf16_by(ld, tb + TM_Q, desc(KQ + 8192 + kq * 2048, 16384), desc(IDT + kq * 32, 16), ID_T, kq > 0);
            mma_commit_by(ld, bar_mma);
            mma_out = true;
        }
        // row norms of k and q from the staged rows while the products run: four
        // threads per row, 32 channels each
        {
            const int r = tid >> 2, part = tid & 3, half = part >> 1, cb = (part & 1) * 4;
            float2 ak = make_float2(0.f, 0.f), aq = ak;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t off = KQ + half * 16384 + r * 128 + ((((cb + j) ^ (r & 7))) << 4);
                float2 fk[4], fq[4];
                unpack8x2(lds128(sm, off), fk);
                unpack8x2(lds128(sm, off + 8192), fq);
#pragma unroll
                for (int e = 0; e < 4; ++e) { ak = __ffma2_rn(fk[e], fk[e], ak); aq = __ffma2_rn(fq[e], fq[e], aq); }
            }
            float sk = ak.x + ak.y, sq = aq.x + aq.y;
            sk += __shfl_xor_sync(0xffffffffu, sk, 1);
            sq += __shfl_xor_sync(0xffffffffu, sq, 1);
            sk += __shfl_xor_sync(0xffffffffu, sk, 2);
            sq += __shfl_xor_sync(0xffffffffu, sq, 2);
            if (part == 0) {
                sinvk[r] = r < L ? (p.use_l2 ? rsqrtf(sk + kL2Eps) : 1.f) : 0.f;
                sinvq[r] = r < L ? (p.use_l2 ? rsqrtf(sq + kL2Eps) : 1.f) : 0.f;
            }
        }
        if (wait_all(bar_mma, ph_mma)) { aborted = true; break; }
        if (warp == 0) mma_out = false;
        tc_fence_after();

        // ---------------- operands, channel layout: thread (c, hw) turns its 32 rows of
        // G, k, q into the bf16 rows c of X_k^T, X_q^T, Y^T (block reference G_m = G_15
        // or G_47 by hw), Y'^T (reference G_47, hw = 0), Qtil^T and Khat^T
        float e15, e47;
        bool span_bad;
        {
            const float g15 = tmem_ld1(tb + lane_sel + TM_G + 15);
            const float g47 = tmem_ld1(tb + lane_sel + TM_G + 47);
            const float g63 = tmem_ld1(tb + lane_sel + TM_G + 63);
            tmem_ld_wait();
            const float gm = hw ? g47 : g15;
            e15 = ex2a(g15 * kL2e);
            e47 = ex2a(g47 * kL2e);
            if (hw == 0) sgam[c] = ex2a(g63 * kL2e);
            const float2 l2e2 = make_float2(kL2e, kL2e), nb = make_float2(-gm * kL2e, -gm * kL2e);
            const float em = ex2a(gm * kL2e), fk = ex2a((g63 - gm) * kL2e);
            const float2 em2 = make_float2(em, em), fk2 = make_float2(fk, fk);
            // Y' takes its own exponent G_47 - G_s (>= -80 - |g_32| next to the block
            // boundary, where it matters): a factor e^{G_47 - G_15} spans 32 tokens and
            // would leave the fp32 range for steep gates
            const float2 nl2e2 = make_float2(-kL2e, -kL2e), b47 = make_float2(g47 * kL2e, g47 * kL2e);
            float amax = 0.f;  // largest |G - G_m| in log2 units
#pragma unroll
            for (int sb2 = 0; sb2 < 2; ++sb2) {
                const int r0 = 32 * hw + 16 * sb2;
                float Gv[16], Kv[16], Qv[16];
                tmem_ld16(tb + lane_sel + TM_G + r0, Gv);
                tmem_ld16(tb + lane_sel + TM_K + r0, Kv);
                tmem_ld16(tb + lane_sel + TM_Q + r0, Qv);
                tmem_ld_wait();
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    float2 xk[4], xq[4], y[4], qt[4], kh[4], yo[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int i = 8 * u + 2 * j;
                        const float2 g2 = make_float2(Gv[i], Gv[i + 1]);
                        const float2 k2 = make_float2(Kv[i], Kv[i + 1]);
                        const float2 q2 = make_float2(Qv[i], Qv[i + 1]);
                        const float2 a = __ffma2_rn(g2, l2e2, nb);
                        amax = fmaxf(amax, fmaxf(fabsf(a.x), fabsf(a.y)));
                        const float2 ed = make_float2(ex2a(a.x), ex2a(a.y));
                        const float2 yd = rcp2_nr(ed);  // e^{G_m - G} on the FMA pipe (ed >= 2^-116 here)
                        xk[j] = __fmul2_rn(k2, ed);
                        xq[j] = __fmul2_rn(q2, ed);
                        y[j] = __fmul2_rn(k2, yd);
                        qt[j] = __fmul2_rn(xq[j], em2);
                        kh[j] = __fmul2_rn(y[j], fk2);
                        if (hw == 0) {
                            const float2 a47 = __ffma2_rn(g2, nl2e2, b47);
                            yo[j] = __fmul2_rn(k2, make_float2(ex2a(a47.x), ex2a(a47.y)));
                        }
                    }
                    const uint32_t off = c * 128 + ((((r0 >> 3) + u) ^ (c & 7)) << 4);
                    sts128(sm, XK + off, pack8x2(xk));
                    sts128(sm, XQ + off, pack8x2(xq));
                    sts128(sm, YT + off, pack8x2(y));
                    sts128(sm, QT + off, pack8x2(qt));
                    sts128(sm, KH + off, pack8x2(kh));
                    if (hw == 0) sts128(sm, YP + off, pack8x2(yo));
                }
            }
            span_bad = !(amax <= kSpanMax * kL2e);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        const bool fb = __syncthreads_or(span_bad) != 0;
        tc_fence_after();
        // a chunk whose gate moves too far inside a block: its record is rewritten exactly
        if (fb && tid == kMma) P.fix_list[atomicAdd(P.fix_count, 1)] = (int)item;
        if (tid == kTma) {
            bulk_store(rec + R_QT, sm + QT, 16384);
            bulk_store(rec + R_KH, sm + KH, 16384);
            bulk_commit();
        }

        // ---------------- A products: D1 = [X_k; X_q] Y^T (diagonal 32-blocks valid),
        // D2 = [X_k; X_q] Y'^T (rows 32..63 against columns 0..31 valid)
        if (warp == 0) {
            const uint32_t ld = elect_one();
#pragma unroll
            for (int kq = 0; kq < 8; ++kq)
                mma_bf16_by(ld, tb + TM_A1, desc(XK + kq * 2048, 16384), dYY + (uint64_t)((YT + kq * 2048) >> 4), ID_A,
                            kq > 0);
            mma_commit_by(ld, bar_mma);
            mma_out = true;
        }
        if (wait_all(bar_mma, ph_mma)) { aborted = true; break; }
        if (warp == 0) mma_out = false;
        tc_fence_after();

        // ---------------- read-back, row layout (lane = row): L = beta_r |k_r|^-1 |k_s|^-1 A_kk
        // (fp32 rows of 16-byte groups; only its strictly lower part is read later) and the
        // raw A_qk tile (bf16, zero above the diagonal)
        {
            const int i = lane;
            if (quarter < 2) {  // A_kk rows 32 quarter + i
                const int r = 32 * quarter + i;
                const float f = sbeta[r] * sinvk[r];
                float va[32];
                int s0, nv;
                if (quarter == 0) {  // block 0: columns 16 hw ..
                    float v16[16];
                    tmem_ld16(tb + lane_sel + TM_A1 + 16 * hw, v16);
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 16; ++j) va[j] = v16[j];
                    s0 = 16 * hw;
                    nv = 16;
                } else {  // hw 0: the diagonal block (columns 32..63), hw 1: columns 0..31
                    tmem_ld32(tb + lane_sel + (hw ? TM_A2 : TM_A1 + 32), va);
                    tmem_ld_wait();
                    s0 = hw ? 0 : 32;
                    nv = 32;
                }
#pragma unroll
                for (int j = 0; j < 32; j += 4) {
                    if (j < nv) {
                        const float4 ik = *reinterpret_cast<const float4 *>(sinvk + s0 + j);
                        *reinterpret_cast<float4 *>(Lf + r * LDS + s0 + j) =
                            make_float4(f * ik.x * va[j], f * ik.y * va[j + 1], f * ik.z * va[j + 2], f * ik.w * va[j + 3]);
                    }
                }
            } else if (quarter == 2) {  // A_qk rows 0..31: columns 16 hw .. (s <= i), zeros right of 32
                float va[16];
                tmem_ld16(tb + lane_sel + TM_A1 + 16 * hw, va);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 16; ++j) va[j] = 16 * hw + j <= i ? va[j] : 0.f;
                row16_to_tile(sm, AQK, i, 16 * hw, 64, va);
                sts128(sm, AQK + sw128_chunk(i, 32 + 16 * hw, 64), make_uint4(0u, 0u, 0u, 0u));
                sts128(sm, AQK + sw128_chunk(i, 40 + 16 * hw, 64), make_uint4(0u, 0u, 0u, 0u));
            } else {  // A_qk rows 32..63: hw 0 the diagonal block (s <= i), hw 1 columns 0..31
                float va[32];
                tmem_ld32(tb + lane_sel + (hw ? TM_A2 : TM_A1 + 32), va);
                tmem_ld_wait();
                if (!hw) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) va[j] = j <= i ? va[j] : 0.f;
                }
                float v16[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) v16[j] = va[j];
                row16_to_tile(sm, AQK, 32 + i, hw ? 0 : 32, 64, v16);
#pragma unroll
                for (int j = 0; j < 16; ++j) v16[j] = va[16 + j];
                row16_to_tile(sm, AQK, 32 + i, hw ? 16 : 48, 64, v16);
            }
        }
        // the Qtil^T / Khat^T stores must have read their sources before T and T_w overwrite them
        if (tid == kTma) bulk_wait_read_all();
        __syncthreads();

        // ---------------- T = (I + L)^-1, written straight into the bf16 tiles T' = T diag(beta)
        // (record) and T_w = T diag(beta / |k|) (rows r, columns s <= r):
        //   1. the four 16x16 diagonal blocks by forward substitution (lane j = column j, the
        //      updates of step k applied to all later rows at once);
        //   2. T_10 = -T_11 L_10 T_00 and T_32 = -T_33 L_32 T_22;
        //   3. X = L_[23][01] T_[01][01], then T_[23][01] = -T_[23][23] X  (32x32 blocks).
        // Steps 2 and 3 run on warp-level tf32 MMAs.
        if (warp < 4) {
            if (lane < 16) {
                const int b = warp, j = lane;
                float t[16];
#pragma unroll
                for (int i = 0; i < 16; ++i) t[i] = i == j ? 1.f : 0.f;
                const float *Lb = Lf + 16 * b * LDS + 16 * b;
#pragma unroll
                for (int kg = 0; kg < 4; ++kg) {
                    float lv[16][4];
#pragma unroll
                    for (int i = 4 * kg + 1; i < 16; ++i) {
                        const float4 l4 = *reinterpret_cast<const float4 *>(Lb + i * LDS + 4 * kg);
                        lv[i][0] = l4.x; lv[i][1] = l4.y; lv[i][2] = l4.z; lv[i][3] = l4.w;
                    }
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int k = 4 * kg + u;
#pragma unroll
                        for (int i = k + 1; i < 16; ++i) t[i] = fmaf(-lv[i][u], t[k], t[i]);
                    }
                }
#pragma unroll
                for (int i = 0; i < 16; ++i) Tf[(16 * b + i) * LDT + 16 * b + j] = t[i];
            }
        } else {
            // blocks above the block diagonal: zero in T and in both bf16 tiles
            // (6 blocks x 16 rows x 2 chunks of 8 columns = 192 items for 128 threads)
            for (int e = tid - 128; e < 192; e += 128) {
                const int bid = e >> 5, i = (e >> 1) & 15, hf = e & 1;
                const int bi = bid < 3 ? 0 : bid < 5 ? 1 : 2;
                const int bj = bid < 3 ? bid + 1 : bid < 5 ? bid - 1 : 3;
                const int r = 16 * bi + i, cc = 16 * bj + 8 * hf;
                *reinterpret_cast<float4 *>(Tf + r * LDT + cc) = make_float4(0.f, 0.f, 0.f, 0.f);
                *reinterpret_cast<float4 *>(Tf + r * LDT + cc + 4) = make_float4(0.f, 0.f, 0.f, 0.f);
                sts128(sm, TPU + sw128_chunk(r, cc, 64), make_uint4(0u, 0u, 0u, 0u));
                sts128(sm, TW + sw128_chunk(r, cc, 64), make_uint4(0u, 0u, 0u, 0u));
            }
        }
        __syncthreads();
        const int g8 = lane >> 2, t4 = lane & 3;
        // -T[r][c], -T[r][c+1] of an MMA output pair into T and both bf16 tiles
        auto put_pair = [&](int r, int c0, float e0, float e1) {
            Tf[r * LDT + c0] = -e0;
            Tf[r * LDT + c0 + 1] = -e1;
            const float b0s = sbeta[c0], b1s = sbeta[c0 + 1];
            *reinterpret_cast<uint32_t *>(sm + TPU + sw128(r, c0, 64)) = pack_bf16x2(-e0 * b0s, -e1 * b1s);
            *reinterpret_cast<uint32_t *>(sm + TW + sw128(r, c0, 64)) =
                pack_bf16x2(-e0 * b0s * sinvk[c0], -e1 * b1s * sinvk[c0 + 1]);
        };
        if (warp < 4) {
            // step 2: block row I (1 or 3) against block column J = I - 1; warp w owns
            // output columns n0 .. n0 + 7
            const int I = warp < 2 ? 1 : 3, jb = 16 * (I - 1), n0 = jb + 8 * (warp & 1);
            float d[4] = {0.f, 0.f, 0.f, 0.f};
            const float *La = Lf + (16 * I + g8) * LDS, *Lb2 = Lf + (16 * I + g8 + 8) * LDS;
#pragma unroll
            for (int ks = 0; ks < 2; ++ks) {
                const int k0 = jb + 8 * ks;
                const uint32_t a[4] = {to_tf32(La[k0 + t4]), to_tf32(Lb2[k0 + t4]), to_tf32(La[k0 + t4 + 4]),
                                       to_tf32(Lb2[k0 + t4 + 4])};
                const uint32_t b[2] = {to_tf32(Tf[(k0 + t4) * LDT + n0 + g8]), to_tf32(Tf[(k0 + t4 + 4) * LDT + n0 + g8])};
                mma_tf32_16x8x8(d, a, b);
            }
            // R[row][col] sits in lane 4*(row % 8) + col/2, component (row >= 8) * 2 + col % 2
            const int srcA = 4 * t4 + (g8 >> 1), srcB = 4 * (t4 + 4) + (g8 >> 1);
            const bool odd = g8 & 1;
            float vv[8];
#pragma unroll
            for (int cq = 0; cq < 4; ++cq) {
                vv[cq] = __shfl_sync(0xffffffffu, d[cq], srcA);
                vv[4 + cq] = __shfl_sync(0xffffffffu, d[cq], srcB);
            }
            const uint32_t b0[2] = {to_tf32(odd ? vv[1] : vv[0]), to_tf32(odd ? vv[5] : vv[4])};
            const uint32_t b1[2] = {to_tf32(odd ? vv[3] : vv[2]), to_tf32(odd ? vv[7] : vv[6])};
            float e4[4] = {0.f, 0.f, 0.f, 0.f};
            const float *Ta = Tf + (16 * I + g8) * LDT + 16 * I, *Tb = Tf + (16 * I + g8 + 8) * LDT + 16 * I;
            {
                const uint32_t a[4] = {to_tf32(Ta[t4]), to_tf32(Tb[t4]), to_tf32(Ta[t4 + 4]), to_tf32(Tb[t4 + 4])};
                mma_tf32_16x8x8(e4, a, b0);
            }
            {
                const uint32_t a[4] = {to_tf32(Ta[8 + t4]), to_tf32(Tb[8 + t4]), to_tf32(Ta[12 + t4]), to_tf32(Tb[12 + t4])};
                mma_tf32_16x8x8(e4, a, b1);
            }
            put_pair(16 * I + g8, n0 + 2 * t4, e4[0], e4[1]);
            put_pair(16 * I + g8 + 8, n0 + 2 * t4, e4[2], e4[3]);
        } else if (warp >= 6) {
            // meanwhile: the diagonal blocks into both bf16 tiles
            for (int e = tid - 192; e < 128; e += 64) {
                const int b = e >> 5, i = (e >> 1) & 15, hf = e & 1;
                const int r = 16 * b + i, cc = 16 * b + 8 * hf;
                float mu[8], mw[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const int s_ = cc + q;
                    mu[q] = s_ <= r ? Tf[r * LDT + s_] * sbeta[s_] : 0.f;
                    mw[q] = mu[q] * sinvk[s_];
                }
                sts128(sm, TPU + sw128_chunk(r, cc, 64), pack8(mu));
                sts128(sm, TW + sw128_chunk(r, cc, 64), pack8(mw));
            }
        }
        __syncthreads();
        // step 3: warp w owns rows 32 + 16 mt .. (mt = w / 4) and columns 8 nt .. (nt = w % 4)
        const int mt = warp >> 2, n0 = 8 * (warp & 3);
        {
            float d[4] = {0.f, 0.f, 0.f, 0.f};
            const float *La = Lf + (32 + 16 * mt + g8) * LDS, *Lb2 = Lf + (32 + 16 * mt + g8 + 8) * LDS;
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const int k0 = 8 * ks;
                const uint32_t a[4] = {to_tf32(La[k0 + t4]), to_tf32(Lb2[k0 + t4]), to_tf32(La[k0 + t4 + 4]),
                                       to_tf32(Lb2[k0 + t4 + 4])};
                const uint32_t b[2] = {to_tf32(Tf[(k0 + t4) * LDT + n0 + g8]), to_tf32(Tf[(k0 + t4 + 4) * LDT + n0 + g8])};
                mma_tf32_16x8x8(d, a, b);
            }
            float *xr = Xs + (16 * mt + g8) * LDXS + n0 + 2 * t4;
            xr[0] = d[0]; xr[1] = d[1];
            xr[8 * LDXS] = d[2]; xr[8 * LDXS + 1] = d[3];
        }
        __syncthreads();
        {
            float e4[4] = {0.f, 0.f, 0.f, 0.f};
            const float *Ta = Tf + (32 + 16 * mt + g8) * LDT, *Tb = Tf + (32 + 16 * mt + g8 + 8) * LDT;
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                if (ks < 2 + 2 * mt) {  // T_[23][23] is zero right of its block diagonal
                    const int k0 = 32 + 8 * ks;
                    const uint32_t a[4] = {to_tf32(Ta[k0 + t4]), to_tf32(Tb[k0 + t4]), to_tf32(Ta[k0 + t4 + 4]),
                                           to_tf32(Tb[k0 + t4 + 4])};
                    const uint32_t b[2] = {to_tf32(Xs[(k0 - 32 + t4) * LDXS + n0 + g8]),
                                           to_tf32(Xs[(k0 - 32 + t4 + 4) * LDXS + n0 + g8])};
                    mma_tf32_16x8x8(e4, a, b);
                }
            }
            put_pair(32 + 16 * mt + g8, n0 + 2 * t4, e4[0], e4[1]);
            put_pair(32 + 16 * mt + g8 + 8, n0 + 2 * t4, e4[2], e4[3]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();

        // ---------------- W^T = X_k^T T_w^T in two K halves (token blocks 0..31, 32..63, each
        // with its own block reference), recombined per key channel at read-back
        if (warp == 0) {
            const uint32_t ld = elect_one();
#pragma unroll
            for (int kq = 0; kq < 4; ++kq)
                mma_bf16_by(ld, tb + (kq < 2 ? TM_W0 : TM_W1), desc(XK + kq * 32, 16), desc(TW + kq * 32, 16), ID_W,
                            (kq & 1) != 0);
            mma_commit_by(ld, bar_mma);
            mma_out = true;
        }
        if (tid == kTma) {
            bulk_store(rec + R_AQK, sm + AQK, 8192);
            bulk_store(rec + R_TPU, sm + TPU, 8192);
            bulk_commit();
        }
        if (tid < C) beta_raw = have_next ? load_beta(nxt) : (unsigned short)0;  // consumed by the next item
        if (wait_all(bar_mma, ph_mma)) { aborted = true; break; }
        if (warp == 0) mma_out = false;
        tc_fence_after();
        // the input area is free again: the next item's inputs load during the read-back
        if (tid == kTma && have_next) { issue_in(nxt); in_out = true; }
        {   // thread (c, hw): -W^T[c][r], r = 32 hw .., = -(e^{G_15} W0 + e^{G_47} W1)
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int r0 = 32 * hw + 16 * u;
                float w0[16], w1[16];
                tmem_ld16(tb + lane_sel + TM_W0 + r0, w0);
                tmem_ld16(tb + lane_sel + TM_W1 + r0, w1);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 16; ++j) w0[j] = -fmaf(e15, w0[j], e47 * w1[j]);
                sts128(sm, WT + c * 128 + (((r0 >> 3) ^ (c & 7)) << 4), pack8(w0));
                sts128(sm, WT + c * 128 + ((((r0 >> 3) + 1) ^ (c & 7)) << 4), pack8(w0 + 8));
            }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (tid == kTma) {
            bulk_store(rec + R_WT, sm + WT, 16384);
            bulk_store(rec + R_MISC, sm + M1_REC, 1024);
            bulk_commit();
        }

        item = nitem;
        cur = nxt;
        have = have_next;
    }

    if (aborted && (tid == kMma || tid == kTma)) {
        if (in_out) mbar_wait(bar_in, ph_in, kWaitLimitNs);
        if (mma_out) mbar_wait(bar_mma, ph_mma, kWaitLimitNs);
        if (P.status && tid == kMma) atomicOr(P.status, 1);
    }
    if (tid == kTma) bulk_wait_all();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tb, TM1_COLS);
    }
}

// ============================================================== exact records
// Rewrites the record of every queued (chunk, head) on CUDA cores in fp32 from
// exponent differences that are never positive (gate <= 0), so no factor can
// overflow whatever the gate: A_kk and A_qk term by term, T by row-wise forward
// substitution, W = T diag(beta/|k|) (k e^G) (stored negated), Qtil = q e^G,
// Khat = k e^{G_last-G}.
constexpr int NTX = 256;
constexpr int LDX = 65;
constexpr uint32_t X_Q = 0, X_K = 32768, X_G = 65536;           // fp32 [64][128]
constexpr uint32_t X_AKK = 98304, X_AQK = X_AKK + 64 * LDX * 4;  // fp32 [64][65]
constexpr uint32_t X_T = X_AQK + 64 * LDX * 4;
constexpr uint32_t X_MISC = X_T + 64 * LDX * 4;                  // beta, invq, invk [64] each
constexpr uint32_t SMEMX_BYTES = X_MISC + 768;

__global__ void __launch_bounds__(NTX, 1) kda_tp_exact_kernel(const __grid_constant__ IntraParams P) {
    extern __shared__ uint8_t smx[];
    const ChunkParams &p = P.p;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = p.H;
    float *qf = reinterpret_cast<float *>(smx + X_Q), *kf = reinterpret_cast<float *>(smx + X_K);
    float *Gf = reinterpret_cast<float *>(smx + X_G);
    float *Akk = reinterpret_cast<float *>(smx + X_AKK), *Aqk = reinterpret_cast<float *>(smx + X_AQK);
    float *Tm = reinterpret_cast<float *>(smx + X_T);
    float *sbeta = reinterpret_cast<float *>(smx + X_MISC), *sinvq = sbeta + 64, *sinvk = sbeta + 128;
    const __nv_bfloat16 *qb = static_cast<const __nv_bfloat16 *>(p.q), *kb = static_cast<const __nv_bfloat16 *>(p.k);
    const __nv_bfloat16 *gb = static_cast<const __nv_bfloat16 *>(p.g), *bt = static_cast<const __nv_bfloat16 *>(p.beta);
    const int nch = P.chunk_tok ? *P.n_chunks : 0;
    const int count = *P.fix_count;

    for (int idx = blockIdx.x; idx < count; idx += gridDim.x) {
        Item it;
        if (!decode_item(P, P.fix_list[idx], nch, it)) continue;
        const int h = it.h, L = it.L;
        const long long t0 = it.t0;
        uint8_t *rec = P.rec + (it.gc * H + h) * (long long)REC_BYTES;
        const float rate = p.gate_mode != kGateLog ? expf(p.A_log[h]) : 0.f;

        __syncthreads();  // the previous item's shared data is no longer read
        for (int e = tid; e < C * D; e += NTX) {
            const int r = e >> 7, cc = e & 127;
            const long long gi = ((t0 + r) * H + h) * D + cc;
            float x = 0.f, y = 0.f, gv = 0.f;
            if (r < L) {
                x = __bfloat162float(qb[gi]);
                y = __bfloat162float(kb[gi]);
                const float bias = (p.gate_mode != kGateLog && p.dt_bias) ? p.dt_bias[h * D + cc] : 0.f;
                gv = gate_value(__bfloat162float(gb[gi]), bias, rate, p.gate_mode, p.has_lb, p.lb);
            }
            qf[e] = x;
            kf[e] = y;
            Gf[e] = gv;
        }
        if (tid < C) {
            const float b = tid < L ? __bfloat162float(bt[(t0 + tid) * H + h]) : 0.f;
            sbeta[tid] = tid < L ? beta_value(b, p.beta_prob) : 0.f;
        }
        __syncthreads();
        if (tid < D) {  // inclusive cumsum per channel
            float run = 0.f;
            for (int r = 0; r < C; ++r) { run += Gf[r * D + tid]; Gf[r * D + tid] = run; }
        }
        for (int r = warp; r < C; r += NTX / 32) {  // row norms
            float sq = 0.f, sk = 0.f;
            for (int cc = lane; cc < D; cc += 32) {
                sq = fmaf(qf[r * D + cc], qf[r * D + cc], sq);
                sk = fmaf(kf[r * D + cc], kf[r * D + cc], sk);
            }
            sq = warp_sum(sq);
            sk = warp_sum(sk);
            if (lane == 0) {
                sinvq[r] = r < L ? (p.use_l2 ? rsqrtf(sq + kL2Eps) : 1.f) : 0.f;
                sinvk[r] = r < L ? (p.use_l2 ? rsqrtf(sk + kL2Eps) : 1.f) : 0.f;
            }
        }
        __syncthreads();
        // raw A_kk[r][s] and A_qk[r][s] for s <= r: warp per pair, lanes over channels
        for (int pr = warp; pr < C * (C + 1) / 2; pr += NTX / 32) {
            int r = (int)((sqrtf(8.f * pr + 1.f) - 1.f) * 0.5f);
            while ((r + 1) * (r + 2) / 2 <= pr) ++r;
            while (r * (r + 1) / 2 > pr) --r;
            const int s = pr - r * (r + 1) / 2;
            float akk = 0.f, aqk = 0.f;
            for (int cc = lane; cc < D; cc += 32) {
                const float e = expf(Gf[r * D + cc] - Gf[s * D + cc]) * kf[s * D + cc];
                akk = fmaf(kf[r * D + cc], e, akk);
                aqk = fmaf(qf[r * D + cc], e, aqk);
            }
            akk = warp_sum(akk);
            aqk = warp_sum(aqk);
            if (lane == 0) {
                Akk[r * LDX + s] = s < r ? sbeta[r] * sinvk[r] * sinvk[s] * akk : 0.f;  // L
                Aqk[r * LDX + s] = aqk;
            }
        }
        __syncthreads();
        // T = (I + L)^-1, row by row: T[i][j] = delta_ij - sum_{j<=k<i} L[i][k] T[k][j]
        for (int i = 0; i < C; ++i) {
            if (tid <= i) {
                float t = tid == i ? 1.f : 0.f;
                for (int k = tid; k < i; ++k) t = fmaf(-Akk[i * LDX + k], Tm[k * LDX + tid], t);
                Tm[i * LDX + tid] = t;
            }
            __syncthreads();
        }
        // record: A_qk, T' tiles (bf16 images, zero above the diagonal)
        for (int e = tid; e < C * C; e += NTX) {
            const int r = e >> 6, s = e & 63;
            const float aq = s <= r ? Aqk[r * LDX + s] : 0.f;
            const float tp = s <= r ? Tm[r * LDX + s] * sbeta[s] : 0.f;
            *reinterpret_cast<__nv_bfloat16 *>(rec + R_AQK + sw128(r, s, 64)) = __float2bfloat16_rn(aq);
            *reinterpret_cast<__nv_bfloat16 *>(rec + R_TPU + sw128(r, s, 64)) = __float2bfloat16_rn(tp);
        }
        // Qtil^T, Khat^T, then k e^G in place of k
        for (int e = tid; e < C * D; e += NTX) {
            const int r = e >> 7, cc = e & 127;
            const float g = Gf[e], gl = Gf[(C - 1) * D + cc];
            *reinterpret_cast<__nv_bfloat16 *>(rec + R_QT + sw128(cc, r, 128)) = __float2bfloat16_rn(qf[e] * expf(g));
            *reinterpret_cast<__nv_bfloat16 *>(rec + R_KH + sw128(cc, r, 128)) =
                __float2bfloat16_rn(kf[e] * expf(gl - g));
        }
        __syncthreads();
        for (int e = tid; e < C * D; e += NTX) kf[e] *= expf(Gf[e]);
        __syncthreads();
        // W^T[c][r] = sum_{s<=r} T[r][s] beta_s |k_s|^-1 (k e^G)[s][c]
        for (int e = tid; e < C * D; e += NTX) {
            const int cc = e & 127, r = e >> 7;
            float w = 0.f;
            for (int s = 0; s <= r; ++s) w = fmaf(Tm[r * LDX + s] * sbeta[s] * sinvk[s], kf[s * D + cc], w);
            *reinterpret_cast<__nv_bfloat16 *>(rec + R_WT + sw128(cc, r, 128)) = __float2bfloat16_rn(-w);
        }
        float *misc = reinterpret_cast<float *>(rec + R_MISC);
        if (tid < D) misc[tid] = expf(Gf[(C - 1) * D + tid]);
        else if (tid < D + C) misc[128 + tid - D] = sinvq[tid - D];
        else misc[192 + tid - D - C] = sinvk[tid - D - C];
    }
}

// ============================================================== pass 2
// One CTA per (sequence, head), 16 warps in two groups:
//   warps 0..7 (the state chain): per chunk, a bf16 copy of S^T for the products
//     and the decayed state written back; [O^T | D^T] = S^T [Qtil^T | -W^T] and
//     D^T += V^T T'^T; D~^T = D^T diag(|k|^-1) to shared memory; S^T += D~^T Khat
//     (its own commit, which the next chunk waits for) and O^T += D~^T A_qk^T;
//   warps 8..15 (output): one chunk behind, read O^T, let the consumed stage be
//     refilled two chunks ahead, and write the output rows.
// O^T and D^T are double-buffered in tensor memory, so the output work of chunk i
// overlaps the state chain of chunk i + 1.
constexpr int NT2 = 512;
constexpr int kGroup = 256;  // threads per warp group
constexpr uint32_t STAGE_BYTES = REC_BYTES + 16384;  // record image + v tile
constexpr uint32_t S_V = REC_BYTES;                  // v tile [64 r][128 v] as two halves (MN-major A)
constexpr uint32_t ST2 = 2 * STAGE_BYTES;            // bf16 S^T [128 v][128 c], K-major A (halves 16 KiB apart)
constexpr uint32_t DT2 = ST2 + 32768;                // bf16 D~^T [128 v][64 s], K-major A
constexpr uint32_t MISC2 = DT2 + 16384;
constexpr uint32_t M2_BAR = MISC2, M2_TMEM = MISC2 + 96;
constexpr uint32_t SMEM2_BYTES = MISC2 + 128;
constexpr uint32_t SMEM2_ALLOC = SMEM2_BYTES + 1024;
static_assert(STAGE_BYTES % 1024 == 0 && SMEM2_ALLOC <= 232448, "pass 2 shared memory");

// tensor memory (512 columns): S^T, then per buffer b: O^T at 128 + 128 b and D^T
// right after it, so [O^T | D^T] is the accumulator of one N = 128 product
constexpr uint32_t TM2_S = 0, TM2_COLS = 512;
__host__ __device__ constexpr uint32_t tm2_o(int b) { return 128 + 128 * b; }
__host__ __device__ constexpr uint32_t tm2_d(int b) { return 192 + 128 * b; }
constexpr uint32_t ID2_QW = idesc_bf16(128, 128, false, true);  // S^T [Qtil^T | -W^T]
constexpr uint32_t ID2_UW = idesc_bf16(128, 64, true, false);   // + V^T T'^T
constexpr uint32_t ID2_KS = idesc_bf16(128, 128, false, false); // D~^T Khat
constexpr uint32_t ID2_KA = idesc_bf16(128, 64, false, false);  // D~^T A_qk^T
constexpr int kMaxPerm = 256;

struct StateParams {
    CUtensorMap tv;
    ChunkParams p;
    const uint8_t *rec;
    const int *chunk_off;
    int cpr;
    int *status;
    int s0_identity;  // start every chain from the identity (S0 is not read)
    int o_f32;        // outputs in fp32 (rows of D floats) instead of bf16
    int v_zero;       // v = 0: no v tiles are copied (tv is not read) and the stage's v area stays zero
    uint8_t *save;    // or null: per (chunk, head) backward record, the S^T and D~^T images go there
    int nperm;
    int perm[kMaxPerm];
};

__global__ void __launch_bounds__(NT2, 1) kda_tp_state_kernel(const __grid_constant__ StateParams P) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const ChunkParams &p = P.p;
    const int tid = threadIdx.x, lane = tid & 31;
    const int warp = __shfl_sync(0xffffffffu, tid >> 5, 0);  // warp-uniform by construction
    const int H = p.H;
    const int rank = blockIdx.x / H, h = blockIdx.x % H;
    const int n = rank < P.nperm ? P.perm[rank] : rank;
    long long bos, eos, c_first;
    if (p.cu_seqlens) { bos = p.cu_seqlens[n]; eos = p.cu_seqlens[n + 1]; c_first = P.chunk_off[n]; }
    else { bos = (long long)n * p.T; eos = bos + p.T; c_first = (long long)n * P.cpr; }
    const int nchunks = (int)((eos - bos + C - 1) / C);
    constexpr int kTma = kGroup;  // first thread of the output group issues the stage copies
    constexpr int kSave = 32;     // stores the chain's images to the backward record

    uint64_t *bar_full = reinterpret_cast<uint64_t *>(sm + M2_BAR);  // [2] stage s loaded
    uint64_t *bar_m1 = bar_full + 2;                                 // first products done
    uint64_t *bar_s = bar_full + 3;                                  // state update done
    uint64_t *bar_o = bar_full + 4;                                  // [2] O^T buffer b complete
    uint64_t *bar_of = bar_full + 6;                                 // [2] O^T buffer b read
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(sm + M2_TMEM);

    if (warp == 0) { tmem_alloc(s_tmem, TM2_COLS); tmem_relinquish(); }
    if (tid == 32) {
        for (int i = 0; i < 6; ++i) mbar_init(bar_full + i, 1);
        mbar_init(bar_of, kGroup); mbar_init(bar_of + 1, kGroup);
        fence_mbar_init();
        if (!P.v_zero) tma_prefetch_desc(&P.tv);
    }
    if (P.v_zero) {  // the v areas of both stages, read by the products as zeros
        for (int e = tid; e < 2 * 1024; e += NT2)
            sts128(sm, (e >> 10) * STAGE_BYTES + S_V + (e & 1023) * 16, make_uint4(0u, 0u, 0u, 0u));
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tb = *s_tmem;
    const uint32_t sb = smem_u32(sm);
    const uint64_t dK = sdesc_sw128(sb, 16, 1024);    // K-major operands
    const uint64_t dM = sdesc_sw128(sb, 8192, 1024);  // MN-major operands (atoms 8 KiB apart)
    const uint64_t dQW = sdesc_sw128(sb, R_WT - R_QT, 1024);  // [Qtil^T | -W^T], groups 16 KiB apart
    auto dk = [&](uint32_t off) { return dK + (uint64_t)(off >> 4); };
    auto dm = [&](uint32_t off) { return dM + (uint64_t)(off >> 4); };
    const int quarter = warp & 3;
    const uint32_t lane_sel = (uint32_t)(32 * quarter) << 16;
    const int v = 32 * quarter + lane;   // value channel = tensor-memory lane of this thread
    const int half = (warp >> 2) & 1;    // column half within the group

    uint32_t full_out = 0;  // stage copies in flight (thread kTma)
    bool aborted = false;
    auto issue_stage = [&](int ci) {
        const int s = ci & 1;
        uint8_t *dst = sm + s * STAGE_BYTES;
        const uint8_t *src = P.rec + ((c_first + ci) * H + h) * (long long)REC_BYTES;
        mbar_arrive_expect_tx(bar_full + s, P.v_zero ? REC_BYTES : STAGE_BYTES);
        bulk_load(dst, src, REC_BYTES, bar_full + s);
        const int t = (int)(bos + (long long)ci * C);
        if (!P.v_zero)
            for (int hf = 0; hf < 2; ++hf) tma_load_3d(dst + S_V + hf * 8192, &P.tv, bar_full + s, hf * 64, h, t);
        full_out |= 1u << s;
    };
    if (tid == kTma) {
        if (nchunks > 0) issue_stage(0);
        if (nchunks > 1) issue_stage(1);
    }
    const long long sbase_state = ((long long)n * H + h) * D * D;

    if (warp < 8) {
        // ================= the state chain
        int issued = -1;  // last chunk whose products were issued (warp 0)
        for (int ci = 0; ci < nchunks; ++ci) {
            const int s = ci & 1, b = ci & 1;
            uint8_t *stg = sm + s * STAGE_BYTES;
            const uint32_t so = s * STAGE_BYTES;
            if (tid == kSave && P.save) bulk_wait_read_all();  // the previous chunk's images were copied out
            {
                bool ok = true;
                if (warp == 0) {
                    ok = mbar_wait(bar_full + s, (ci >> 1) & 1, kWaitLimitNs);
                    if (ok && ci > 0) ok = mbar_wait(bar_s, (ci - 1) & 1, kWaitLimitNs);
                }
                if (bar_or(1, kGroup, !ok)) { aborted = true; break; }
            }
            tc_fence_after();
            // bf16 copy of S^T for the products; the decayed S^T diag(e^{G_last}) back into
            // tensor memory (the update product accumulates onto it)
            const float *gam = reinterpret_cast<const float *>(stg + R_GAM);
#pragma unroll
            for (int jc = 0; jc < 2; ++jc) {
                const int c0 = 64 * half + 32 * jc;
                float x[32];
                if (ci == 0) {
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        x[j] = P.s0_identity ? (c0 + j == v ? 1.f : 0.f)
                                             : p.S0 ? p.S0[sbase_state + (long long)(c0 + j) * D + v] : 0.f;
                } else {
                    tmem_ld32(tb + TM2_S + lane_sel + c0, x);
                    tmem_ld_wait();
                }
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) sts128(sm, ST2 + sw128_chunk(v, c0 + 8 * q4, 128), pack8(x + 8 * q4));
#pragma unroll
                for (int j = 0; j < 32; j += 2) {
                    const float2 v2 = __fmul2_rn(make_float2(x[j], x[j + 1]),
                                                 *reinterpret_cast<const float2 *>(gam + c0 + j));
                    x[j] = v2.x; x[j + 1] = v2.y;
                }
                tmem_st32(tb + TM2_S + lane_sel + c0, x);
            }
            tmem_st_wait();
            fence_proxy_async_smem();
            tc_fence_before();
            bar_sync(1, kGroup);
            tc_fence_after();
            uint8_t *bsave = P.save ? P.save + ((c_first + ci) * H + h) * (long long)BR_BYTES : nullptr;
            if (tid == kSave && bsave) { bulk_store(bsave + BR_S0, sm + ST2, 32768); bulk_commit(); }

            // [O^T | D^T] = S^T [Qtil^T | -W^T], then D^T += V^T T'^T
            if (warp == 0) {
                bool ok = true;
                if (ci >= 2) ok = mbar_wait(bar_of + b, ((ci - 2) >> 1) & 1, kWaitLimitNs);  // O^T buffer read
                if (ok) {
                    const uint32_t ld = elect_one();
#pragma unroll
                    for (int kq = 0; kq < 8; ++kq)
                        mma_bf16_by(ld, tb + tm2_o(b), dk(ST2 + (kq >> 2) * 16384 + (kq & 3) * 32),
                                    dQW + (uint64_t)((so + R_QT + kq * 2048) >> 4), ID2_QW, kq > 0);
#pragma unroll
                    for (int kq = 0; kq < 4; ++kq)
                        mma_bf16_by(ld, tb + tm2_d(b), dm(so + S_V + kq * 2048), dk(so + R_TPU + kq * 32), ID2_UW, 1);
                    mma_commit_by(ld, bar_m1);
                    ok = mbar_wait(bar_m1, ci & 1, kWaitLimitNs);
                }
                if (!ok) aborted = true;
            }
            if (bar_or(1, kGroup, aborted)) { aborted = true; break; }
            tc_fence_after();
            {   // D^T (lane v, columns s), times |k_s|^-1 -> bf16 tile [v][s]
                const float *invk = reinterpret_cast<const float *>(stg + R_INVK);
                float x[32];
                const int s0 = 32 * half;
                tmem_ld32(tb + tm2_d(b) + lane_sel + s0, x);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 32; j += 4) {
                    const float4 f = *reinterpret_cast<const float4 *>(invk + s0 + j);
                    x[j] *= f.x; x[j + 1] *= f.y; x[j + 2] *= f.z; x[j + 3] *= f.w;
                }
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) sts128(sm, DT2 + sw128_chunk(v, s0 + 8 * q4, 128), pack8(x + 8 * q4));
            }
            fence_proxy_async_smem();
            tc_fence_before();
            bar_sync(1, kGroup);
            tc_fence_after();
            if (tid == kSave && bsave) { bulk_store(bsave + BR_DL, sm + DT2, 16384); bulk_commit(); }

            // S^T += D~^T Khat (committed on its own: the next chunk waits for it), then
            // O^T += D~^T A_qk^T (the output group waits for that one)
            if (warp == 0) {
                const uint32_t ld = elect_one();
#pragma unroll
                for (int kq = 0; kq < 4; ++kq)
                    mma_bf16_by(ld, tb + TM2_S, dk(DT2 + kq * 32), dk(so + R_KH + kq * 32), ID2_KS, 1);
                mma_commit_by(ld, bar_s);
#pragma unroll
                for (int kq = 0; kq < 4; ++kq)
                    mma_bf16_by(ld, tb + tm2_o(b), dk(DT2 + kq * 32), dk(so + R_AQK + kq * 32), ID2_KA, 1);
                mma_commit_by(ld, bar_o + b);
                issued = ci;
            }
        }
        if (!aborted && p.S_out) {
            bool ok = true;
            if (warp == 0 && nchunks > 0) ok = mbar_wait(bar_s, (nchunks - 1) & 1, kWaitLimitNs);
            if (bar_or(1, kGroup, !ok)) aborted = true;
            tc_fence_after();
            if (!aborted) {
#pragma unroll
                for (int jc = 0; jc < 2; ++jc) {
                    const int c0 = 64 * half + 32 * jc;
                    float x[32];
                    if (nchunks == 0) {
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            x[j] = P.s0_identity ? (c0 + j == v ? 1.f : 0.f)
                                                 : p.S0 ? p.S0[sbase_state + (long long)(c0 + j) * D + v] : 0.f;
                    } else {
                        tmem_ld32(tb + TM2_S + lane_sel + c0, x);
                        tmem_ld_wait();
                    }
#pragma unroll
                    for (int j = 0; j < 32; ++j) p.S_out[sbase_state + (long long)(c0 + j) * D + v] = x[j];
                }
            }
        }
        if (aborted && warp == 0 && issued >= 0) {  // let the issued products finish before exit
            mbar_wait(bar_o + (issued & 1), (issued >> 1) & 1, kWaitLimitNs);
            if (P.status && lane == 0) atomicOr(P.status, 1);
        }
        if (tid == kSave && P.save) bulk_wait_all();
    } else {
        // ================= output rows, one chunk behind
        __nv_bfloat16 *O = static_cast<__nv_bfloat16 *>(p.o);
        float *Of = P.o_f32 ? static_cast<float *>(p.o) : nullptr;
        for (int ci = 0; ci < nchunks; ++ci) {
            const int s = ci & 1, b = ci & 1;
            const uint8_t *stg = sm + s * STAGE_BYTES;
            {
                bool ok = true;
                if (warp == 8) ok = mbar_wait(bar_o + b, (ci >> 1) & 1, kWaitLimitNs);
                if (bar_or(2, kGroup, !ok)) { aborted = true; break; }
            }
            tc_fence_after();
            const int r0 = 32 * half;
            float x[32], iq[32];
            tmem_ld32(tb + tm2_o(b) + lane_sel + r0, x);
            const float *invq = reinterpret_cast<const float *>(stg + R_INVQ);
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
                const float4 f = *reinterpret_cast<const float4 *>(invq + r0 + j);
                iq[j] = f.x; iq[j + 1] = f.y; iq[j + 2] = f.z; iq[j + 3] = f.w;
            }
            tmem_ld_wait();
            tc_fence_before();
            bar_sync(2, kGroup);  // O^T buffer and the stage are no longer read by this group
            if (tid == kTma) {
                if ((full_out >> s) & 1u) full_out &= ~(1u << s);  // chunk ci's copies completed (waited above)
                if (ci + 2 < nchunks) issue_stage(ci + 2);
            }
            mbar_arrive(bar_of + b);
            const long long t0 = bos + (long long)ci * C;
            const int L = (int)((eos - t0) < C ? (eos - t0) : C);
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int r = r0 + j;
                if (r < L && O) {
                    const float ov = p.scale * iq[j] * x[j];
                    if (Of) Of[((t0 + r) * H + h) * D + v] = ov;
                    else O[((t0 + r) * H + h) * D + v] = __float2bfloat16_rn(ov);
                }
            }
        }
        if (aborted && tid == kTma) {  // copies still in flight finish before exit
            for (int s = 0; s < 2; ++s)
                if ((full_out >> s) & 1u) mbar_wait(bar_full + s, 0, kWaitLimitNs), mbar_wait(bar_full + s, 1, kWaitLimitNs);
            if (P.status) atomicOr(P.status, 1);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tb, TM2_COLS);
    }
}

// Set-up of a forward call, one block of 1024 threads:
//  * the constant tile images of pass 1 (bf16, 128-byte swizzle): Tri[r][s] = 1 for
//    s <= r (B operand of the in-chunk cumsum) and the identity (the transposes);
//  * for a varlen batch, the chunk table: chunk_off[n] = sum_{m<n} ceil(len_m / C)
//    (the first global chunk of sequence n; chunk_off[N] = the total) and, per global
//    chunk, its first token and number of valid rows (sequences in tiles of 1024).
__global__ void __launch_bounds__(1024) kda_tp_prep(uint8_t *consts, const int32_t *cu, int N, int *chunk_off,
                                                    int2 *chunk_tok) {
    __shared__ int warp_tot[32];
    __shared__ int carry;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nw = blockDim.x >> 5;
    {
        const int tile = tid >> 9, r = (tid >> 3) & 63, j = tid & 7;
        float v[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const int s_ = 8 * j + q;
            v[q] = tile ? (s_ == r ? 1.f : 0.f) : (s_ <= r ? 1.f : 0.f);
        }
        *reinterpret_cast<uint4 *>(consts + tile * 8192 + sw128_chunk(r, 8 * j, 64)) = pack8(v);
    }
    if (!cu) return;
    if (tid == 0) { carry = 0; chunk_off[0] = 0; }
    __syncthreads();
    for (int base = 0; base < N; base += blockDim.x) {
        const int n = base + tid;
        int c = 0;
        if (n < N) c = (int)(((long long)cu[n + 1] - cu[n] + C - 1) / C);
        int inc = c;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, inc, d);
            if (lane >= d) inc += y;
        }
        if (lane == 31) warp_tot[warp] = inc;
        __syncthreads();
        int before = 0;
        for (int w = 0; w < warp; ++w) before += warp_tot[w];
        const int c0 = carry;
        if (n < N) chunk_off[n + 1] = c0 + before + inc;
        __syncthreads();
        if (tid == blockDim.x - 1) {
            int tot = 0;
            for (int w = 0; w < nw; ++w) tot += warp_tot[w];
            carry = c0 + tot;
        }
        __syncthreads();
    }
    // chunk_off is complete (written by this block before the barriers above)
    for (int n = warp; n < N; n += nw) {
        const int first = chunk_off[n], bos = cu[n], len = cu[n + 1] - bos;
        const int nc = (len + C - 1) / C;
        for (int ci = lane; ci < nc; ci += 32) chunk_tok[first + ci] = make_int2(bos + ci * C, min(C, len - ci * C));
    }
}

// ---- workspace: [header 1 KB: status word, exact-queue count][constant tiles 16 KB]
// [chunk offsets][chunk table][exact queue][records], every part 1024-aligned
long long max_chunks(const ChunkParams &p) {
    if (p.cu_seqlens) return ((long long)p.T + C - 1) / C + p.N;
    return (long long)p.N * (((long long)p.T + C - 1) / C);
}
size_t round1k(size_t b) { return (b + 1023) / 1024 * 1024; }
size_t offsets_bytes(const ChunkParams &p) { return p.cu_seqlens ? round1k((size_t)(p.N + 1) * 4) : 0; }
size_t table_bytes(const ChunkParams &p) { return p.cu_seqlens ? round1k((size_t)max_chunks(p) * 8) : 0; }
size_t queue_bytes(const ChunkParams &p) { return round1k((size_t)max_chunks(p) * p.H * 4); }

}  // namespace tp

namespace tp {

size_t base_workspace_bytes(const ChunkParams &p) {
    return 1024 + 16384 + offsets_bytes(p) + table_bytes(p) + queue_bytes(p) + (size_t)max_chunks(p) * p.H * REC_BYTES;
}

// prep, pass 1 and the exact records of p into the workspace ws (its layout follows p)
cudaError_t run_pass1(const ChunkParams &p, uint8_t *ws, cudaStream_t st) {
    const long long total = p.cu_seqlens ? (long long)p.T : (long long)p.N * p.T;
    if (total <= 0) return cudaErrorInvalidValue;
    const long long n_items = max_chunks(p) * p.H;
    if (n_items >= (1LL << 31) || total >= (1LL << 31)) return cudaErrorInvalidValue;
    int *status = reinterpret_cast<int *>(ws);
    int *fix_count = reinterpret_cast<int *>(ws + 64);
    uint8_t *consts = ws + 1024;
    const size_t base = 1024 + 16384;
    int *chunk_off = reinterpret_cast<int *>(ws + base);
    int2 *chunk_tok = reinterpret_cast<int2 *>(ws + base + offsets_bytes(p));
    int *fix_list = reinterpret_cast<int *>(ws + base + offsets_bytes(p) + table_bytes(p));
    uint8_t *rec = ws + base + offsets_bytes(p) + table_bytes(p) + queue_bytes(p);

    static_assert(sizeof(IntraParams) <= 4096 && sizeof(StateParams) <= 4096, "kernel parameter blocks");
    IntraParams A;
    memset(&A, 0, sizeof(A));
    A.p = p;
    A.rec = rec;
    A.chunk_tok = p.cu_seqlens ? chunk_tok : nullptr;
    A.n_chunks = p.cu_seqlens ? chunk_off + p.N : nullptr;
    A.cpr = (int)(((long long)p.T + C - 1) / C);
    A.n_items = n_items;
    A.split_gate = (p.gate_mode == kGateLog && p.has_lb &&
                    __bfloat162float(__float2bfloat16_rn(p.lb)) != p.lb) ? 1 : 0;
    A.consts = consts;
    A.fix_count = fix_count;
    A.fix_list = fix_list;
    A.status = status;
    if (!make_map(&A.tq, p.q, total, p.H) || !make_map(&A.tk, p.k, total, p.H) ||
        !make_map(&A.tg, p.g, total, p.H))
        return cudaErrorInvalidValue;

    cudaError_t e = cudaMemsetAsync(ws, 0, 256, st);
    if (e != cudaSuccess) return e;
    count_launch();
    kda_tp_prep<<<1, 1024, 0, st>>>(consts, p.cu_seqlens, p.N, chunk_off, chunk_tok);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    int dev = 0, nsm = 148;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kda_tp_intra_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM1_ALLOC);
    if (e != cudaSuccess) return e;
    const long long grid1 = std::min<long long>(n_items, 2LL * nsm);
    count_launch();
    kda_tp_intra_kernel<<<(unsigned)grid1, NT1, SMEM1_ALLOC, st>>>(A);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kda_tp_exact_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEMX_BYTES);
    if (e != cudaSuccess) return e;
    count_launch();
    kda_tp_exact_kernel<<<(unsigned)std::min<long long>(n_items, nsm), NTX, SMEMX_BYTES, st>>>(A);
    return cudaGetLastError();
}

// Finish time of pass 2 when its CTAs -- the sequences in the order `ord`, all heads of
// a sequence in a row -- go in that order to whichever of `slots` SMs frees first (one
// CTA per SM), a CTA taking one unit per chunk of its sequence (at least one).
long long dispatch_makespan(const std::vector<int> &ord, const std::vector<long long> &units, int H, int slots) {
    std::priority_queue<long long, std::vector<long long>, std::greater<long long>> free_at;
    for (int i = 0; i < slots; ++i) free_at.push(0);
    long long end = 0;
    for (int n : ord)
        for (int h = 0; h < H; ++h) {
            const long long t = free_at.top() + units[n];
            free_at.pop();
            free_at.push(t);
            end = std::max(end, t);
        }
    return end;
}

// The launch order of pass 2's sequences: longest first, then pairwise swaps that
// shorten the simulated finish time (few sequences of a few lengths leave a ragged
// last wave under longest-first: lengths 4096/8192/12288/7168 at H = 96 finish at 368
// chunk units longest-first and at 352 with 7168 moved ahead of 8192).
std::vector<int> pass2_order(const int32_t *cu_host, int N, int H, int slots) {
    std::vector<int> ord(N);
    std::vector<long long> units(N);
    for (int i = 0; i < N; ++i) {
        ord[i] = i;
        units[i] = std::max<long long>(1, ((long long)cu_host[i + 1] - cu_host[i] + C - 1) / C);
    }
    std::stable_sort(ord.begin(), ord.end(), [&](int a, int b) { return units[a] > units[b]; });
    if (N < 2 || N > 16 || (long long)N * H <= slots || (long long)N * H > 16384) return ord;
    // the search (tens of microseconds) runs once per set of lengths on this thread
    thread_local std::vector<long long> last_units;
    thread_local std::vector<int> last_ord;
    thread_local int last_H = -1, last_slots = -1;
    if (H == last_H && slots == last_slots && units == last_units) return last_ord;
    long long best = dispatch_makespan(ord, units, H, slots);
    long long total = 0;
    for (int i = 0; i < N; ++i) total += units[i] * H;
    const long long lower = std::max(units[ord[0]], (total + slots - 1) / slots);
    for (int round = 0; round < 4 && best * 50 > lower * 51; ++round) {  // more than 2 % above the bound
        bool better = false;
        for (int i = 0; i < N; ++i)
            for (int j = i + 1; j < N; ++j) {
                if (units[ord[i]] == units[ord[j]]) continue;
                std::swap(ord[i], ord[j]);
                const long long m = dispatch_makespan(ord, units, H, slots);
                if (m < best) { best = m; better = true; }
                else std::swap(ord[i], ord[j]);
            }
        if (!better) break;
    }
    last_H = H;
    last_slots = slots;
    last_units = units;
    last_ord = ord;
    return ord;
}

// pass 2 of p (v, S0, S_out and o as p gives them; o may be null) over the records in ws;
// s0_identity starts every chain from the identity, v_zero takes v = 0 (p.v is not read)
cudaError_t run_pass2(const ChunkParams &p, uint8_t *ws, const int32_t *cu_host, cudaStream_t st, int s0_identity = 0,
                      int v_zero = 0, int o_f32 = 0, uint8_t *save = nullptr) {
    const long long total = p.cu_seqlens ? (long long)p.T : (long long)p.N * p.T;
    int *status = reinterpret_cast<int *>(ws);
    const size_t base = 1024 + 16384;
    int *chunk_off = reinterpret_cast<int *>(ws + base);
    uint8_t *rec = ws + base + offsets_bytes(p) + table_bytes(p) + queue_bytes(p);
    StateParams B;
    memset(&B, 0, sizeof(B));
    B.p = p;
    B.rec = rec;
    B.chunk_off = p.cu_seqlens ? chunk_off : nullptr;
    B.cpr = (int)(((long long)p.T + C - 1) / C);
    B.status = status;
    B.s0_identity = s0_identity;
    B.v_zero = v_zero;
    B.o_f32 = o_f32;
    B.save = save;
    if (!v_zero && !make_map(&B.tv, p.v, total, p.H)) return cudaErrorInvalidValue;
    B.nperm = 0;
    cudaError_t e;
    if (cu_host && p.N <= kMaxPerm) {  // the launch order of the sequences (longest first, tail balanced)
        int dev = 0, nsm = 148;
        if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
        if ((e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
        const std::vector<int> ord = pass2_order(cu_host, p.N, p.H, nsm);
        for (int i = 0; i < p.N; ++i) B.perm[i] = ord[i];
        B.nperm = p.N;
    }
    e = cudaFuncSetAttribute(kda_tp_state_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM2_ALLOC);
    if (e != cudaSuccess) return e;
    count_launch();
    kda_tp_state_kernel<<<(unsigned)((long long)p.N * p.H), NT2, SMEM2_ALLOC, st>>>(B);
    return cudaGetLastError();
}

// ---- segments: with few (sequence, head) state chains, every sequence is cut into
// P chunk-aligned segments whose chains run side by side. The state after a segment
// is affine in the state before it, S_end = M S_start + N (the chunk update
// S <- diag(e^{G_last}) S + Khat^T (U - W S) is affine in S), so pass 2 runs three
// times over the segments: with v = 0 and S_start = I (its final states are the
// M; the identity is formed in the kernel and no v is read), with S_start = 0 (the N;
// neither run writes outputs), and, once `kda_seg_chain` has walked the segments
// of each sequence to their true entering states, with those states for the
// outputs. Pass 1's records do not depend on the state and serve all three runs.
constexpr int kMaxSeg = 16;
constexpr int kChainSms = 148;  // chains wanted in flight: the SM count of the part

int seg_count(const ChunkParams &p) {
    const long long chains = (long long)p.N * p.H;
    if (chains >= kChainSms) return 1;
    const long long avg = p.cu_seqlens ? (long long)p.T / (p.N > 0 ? p.N : 1) : (long long)p.T;
    long long P = std::min<long long>(kMaxSeg, kChainSms / chains);  // one wave of pass-2 CTAs (one per SM)
    P = std::min<long long>(P, avg / (4 * C));  // at least four chunks per segment on average
    return P < 2 ? 1 : (int)P;
}

// The segment view of p: P segments per sequence as a varlen batch.
ChunkParams seg_view(const ChunkParams &p, int P, const int32_t *cu_v) {
    ChunkParams q = p;
    q.T = p.cu_seqlens ? p.T : p.N * p.T;  // total tokens (varlen convention)
    q.N = p.N * P;
    q.cu_seqlens = cu_v;
    return q;
}

size_t seg_state_bytes(const ChunkParams &p, int P) { return round1k((size_t)p.N * P * p.H * 128 * 128 * 4); }

}  // namespace tp

size_t chunk_2pass_workspace_bytes(const ChunkParams &p) {
    using namespace tp;
    const int P = seg_count(p);
    if (P == 1) return base_workspace_bytes(p);
    const ChunkParams q = seg_view(p, P, reinterpret_cast<const int32_t *>(16));  // only its presence is read
    return base_workspace_bytes(q) + round1k(((size_t)p.N * P + 1) * 4) + 3 * seg_state_bytes(p, P);
}

// For kda_bwd.cu's segment form: the transitions and offsets of every sequence of the
// (segment) view q, from pass 1 over q and pass 2 from the identity with v = 0 (final
// states to M; per token, w_t = scale M_t^T q^_t to w in fp32 rows of D when w is given,
// M_t the map up to token t) and from zero (final states to Nst, no outputs).
// ws: chunk_2pass_base_bytes(q).
size_t chunk_2pass_base_bytes(const ChunkParams &q) { return tp::base_workspace_bytes(q); }

cudaError_t chunk_2pass_transitions(const ChunkParams &q, void *workspace, float *M, float *Nst, float *w,
                                    cudaStream_t st) {
    using namespace tp;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    cudaError_t e;
    if ((e = run_pass1(q, ws, st)) != cudaSuccess) return e;
    ChunkParams pm = q;
    pm.v = nullptr; pm.S0 = nullptr; pm.S_out = M; pm.o = w;
    if ((e = run_pass2(pm, ws, nullptr, st, 1, 1, 1)) != cudaSuccess) return e;
    ChunkParams pn = q;
    pn.S0 = nullptr; pn.S_out = Nst; pn.o = nullptr;
    return run_pass2(pn, ws, nullptr, st);
}

// The records of the forward run in ws (its layout follows the segment view when p is
// segmented); chunk numbering is the same either way, as segments are chunk-aligned.
uint8_t *chunk_2pass_records(const ChunkParams &p, void *workspace) {
    using namespace tp;
    const int P = seg_count(p);
    const ChunkParams q = P == 1 ? p : seg_view(p, P, reinterpret_cast<const int32_t *>(16));
    return static_cast<uint8_t *>(workspace) + 1024 + 16384 + offsets_bytes(q) + table_bytes(q) + queue_bytes(q);
}

// The forward of p; with save non-null, the pass that forms the outputs also writes
// every (chunk, head)'s S^T and D~^T images to its backward record (save + (chunk * H
// + head) * BR_BYTES, global chunk numbering).
cudaError_t launch_chunk_2pass_save(const ChunkParams &p, void *workspace, const int32_t *cu_host, uint8_t *save,
                                    cudaStream_t st) {
    using namespace tp;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    const int P = seg_count(p);
    cudaError_t e;
    if (P == 1) {
        if ((e = run_pass1(p, ws, st)) != cudaSuccess) return e;
        return run_pass2(p, ws, cu_host, st, 0, 0, 0, save);
    }
    // workspace: [two-pass workspace of the segment view][cu_v][M][N][S_start]
    int32_t *cu_v = reinterpret_cast<int32_t *>(ws + base_workspace_bytes(seg_view(p, P, reinterpret_cast<const int32_t *>(16))));
    const ChunkParams q = seg_view(p, P, cu_v);
    uint8_t *cursor = reinterpret_cast<uint8_t *>(cu_v) + round1k(((size_t)p.N * P + 1) * 4);
    float *Mbuf = reinterpret_cast<float *>(cursor);
    cursor += seg_state_bytes(p, P);
    float *Nbuf = reinterpret_cast<float *>(cursor);
    cursor += seg_state_bytes(p, P);
    float *Sbuf = reinterpret_cast<float *>(cursor);

    count_launch();
    kda_seg_setup<<<(p.N + 255) / 256, 256, 0, st>>>(p.cu_seqlens, p.T, p.N, P, C, cu_v);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = run_pass1(q, ws, st)) != cudaSuccess) return e;
    ChunkParams pm = q;  // the transitions: v = 0 from the identity, no outputs
    pm.v = nullptr; pm.S0 = nullptr; pm.S_out = Mbuf; pm.o = nullptr;
    if ((e = run_pass2(pm, ws, nullptr, st, 1, 1)) != cudaSuccess) return e;
    ChunkParams pn = q;  // the offsets: from zero, no outputs
    pn.S0 = nullptr; pn.S_out = Nbuf; pn.o = nullptr;
    if ((e = run_pass2(pn, ws, nullptr, st)) != cudaSuccess) return e;
    if ((e = seg_chain_launch<128>(p.S0, Mbuf, Nbuf, 128, 128LL * 128, Sbuf, p.S_out, p.N, p.H, P, st)) != cudaSuccess) return e;
    ChunkParams pf = q;  // the outputs, from the true entering states
    pf.S0 = Sbuf; pf.S_out = nullptr;
    return run_pass2(pf, ws, nullptr, st, 0, 0, 0, save);
}

int chunk_2pass_seg_count(const ChunkParams &p) { return tp::seg_count(p); }

// Where a segmented forward of p keeps its segment view in ws: returns P (1 when p is not
// segmented, and nothing is set), the view's cu_seqlens and chunk offsets, and the
// segment transitions M ([N P, H, 128, 128], S_end = M S_start + N).
int chunk_2pass_seg_info(const ChunkParams &p, void *workspace, const int32_t **cu_v, const int **chunk_off_v,
                         const float **M) {
    using namespace tp;
    const int P = seg_count(p);
    if (P == 1) return 1;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    const ChunkParams q = seg_view(p, P, reinterpret_cast<const int32_t *>(16));
    uint8_t *cv = ws + base_workspace_bytes(q);
    *cu_v = reinterpret_cast<const int32_t *>(cv);
    *chunk_off_v = reinterpret_cast<const int *>(ws + 1024 + 16384);
    *M = reinterpret_cast<const float *>(cv + round1k(((size_t)p.N * P + 1) * 4));
    return P;
}

// The chunk offsets and table of a varlen batch (the prep kernel also writes the constant
// tiles to consts, 16 KB).
cudaError_t chunk_2pass_chunk_table(const int32_t *cu, int N, int *chunk_off, int2 *chunk_tok, uint8_t *consts,
                                    cudaStream_t st) {
    count_launch();
    tp::kda_tp_prep<<<1, 1024, 0, st>>>(consts, cu, N, chunk_off, chunk_tok);
    return cudaGetLastError();
}

cudaError_t launch_chunk_2pass(const ChunkParams &p, void *workspace, const int32_t *cu_host, cudaStream_t st) {
    return launch_chunk_2pass_save(p, workspace, cu_host, nullptr, st);
}

}  // namespace kda
