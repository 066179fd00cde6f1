// Backward of the chunkwise forward in chunk form, bf16 inputs, d_k = d_v = 128,
// chunk C = 64, a lower-bounded gate (lower_bound >= -5).
//
// The pages give no backward formulas; this differentiates the chunk form of the
// operator (`chunk_kda` of page "K3/kda/ops/api.py", whose result is the token
// recurrence of page "atlas_core/kimi_k3/kda.rs"). Per chunk, with the notation
// of the two-pass forward (G the in-chunk cumsum of the clamped gate, k^, q^ the
// normalised rows, b the write strengths, T = (I + diag(b) A_kk)^-1, T' = T diag(b),
// Ktil = k^ e^G, Qtil = q^ e^G, Khat = k^ e^{G_C - G}, gamma = e^{G_C}):
//   W = T' Ktil,  U = T' V,  D = U - W S,  O = scale (Qtil S + A_qk D),
//   S_C = diag(gamma) S + Khat^T D.
// Given the output cotangent dO and dS_C (the cotangent of the state leaving the
// chunk), the state-dependent part is a chain walked from the last chunk back:
//   dD  = scale A_qk^T dO + Khat dS_C,
//   dS  = diag(gamma) dS_C + scale Qtil^T dO - W^T dD     (the cotangent entering)
// (`kda_cb_dstate_kernel`, tensor cores, dS^T resident in tensor memory), and the
// rest is local to each chunk (`kda_cb_intra_kernel`, all chunks at once):
//   dQtil = scale dO S^T,  dW = -dD S^T,  dKhat = D dS_C^T,  dA_qk = scale dO D^T (s <= r),
//   dT' = dD V^T + dW Ktil^T,  dV = T'^T dD,  dKtil = T'^T dW,
//   T = I - T' A_kk,  db_s += sum_r dT'_rs T_rs,  dM = -T^T (dT' diag(b)) T^T,
//   dA_kk = diag(b) dM (s < r),  db_r += sum_s dM_rs A_rs,
// the gated products A[r,s] = sum_c x_rc y_sc e^{G_rc - G_sc} give
//   dx_r += sum_s dA_rs y_s e^{G_r - G_s},  dy_s += sum_r dA_rs x_r e^{G_r - G_s},
//   dG_r += x_r . (that first sum), dG_s -= y_s . (the second),
// the elementwise factors give dq^ += dQtil e^G, dk^ += dKtil e^G + dKhat e^{G_C - G},
// dG += dQtil Qtil + dKtil Ktil - dKhat Khat, dG_C += sum_s dKhat Khat + gamma sum_v S dS_C,
// and dg is the reverse in-chunk cumsum of dG (zero where the clamp is active), dk and
// dq go through the L2 norm, dbeta through the sigmoid.
//
// The factor e^{G_r - G_s} of a gated product is split at a reference so that neither
// part leaves the fp32 range: for rows and columns in different 16-row blocks at the
// block boundary between them (both parts <= 1, whatever the gate), inside a 16-row
// block at its middle row (parts <= e^{8 |lower_bound|}).
#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>

#include "kda_common.cuh"
#include "kda_bwd.cuh"
#include "kda_sm100.cuh"
#include "kda_tc_util.cuh"
#include "kda_stage.cuh"
#include "kda_record.cuh"
#include "kda_seg.cuh"

namespace kda {

// from kda_chunk_2pass.cu
size_t chunk_2pass_workspace_bytes(const ChunkParams &p);
uint8_t *chunk_2pass_records(const ChunkParams &p, void *workspace);
cudaError_t launch_chunk_2pass_save(const ChunkParams &p, void *workspace, const int32_t *cu_host, uint8_t *save,
                                    cudaStream_t st);
int chunk_2pass_seg_info(const ChunkParams &p, void *workspace, const int32_t **cu_v, const int **chunk_off_v,
                         const float **M);
int chunk_2pass_seg_count(const ChunkParams &p);

namespace cb {

using namespace sm100;
using namespace tcu;
using tp::BR_BYTES;
using tp::BR_DD;
using tp::BR_DL;
using tp::BR_DS;
using tp::BR_S0;
using tp::REC_BYTES;

constexpr int C = 64;
constexpr int D = 128;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // bounded waits: 2 s
constexpr float kL2e = 1.4426950408889634f;

// ============================================================== cotangent chain
// One CTA of 256 threads per (sequence, head), walking its chunks from the last.
// Per chunk the stage holds the forward's record and the dO tile (TMA, two 64-column
// halves, the MN-major A operand dO^T); thread (quarter, half) owns tensor-memory
// lanes 32 quarter .. (value channel v) and a half of the columns.
//   products 1-3:  dD~^T  = dO'^T A_qk + dS^T Khat^T        (dO' = diag(scale/|q_r|) dO)
//                  dS^T  += dO'^T Qtil                      (onto diag(gamma)-decayed dS^T)
//   product 4:     dS^T  += dD^T (-W)                       (dD = diag(1/|k_s|) dD~)
// with the record's raw rows (Qtil, Khat, A_qk without the norms) and its normalised W.
constexpr int NTC = 256;
constexpr uint32_t C_STAGE = REC_BYTES + 16384;  // record + dO tile
constexpr uint32_t C_DO = REC_BYTES;
constexpr uint32_t C_DST = 2 * C_STAGE;          // bf16 dS^T [128 v][128 k], K-major A (halves 16 KiB apart)
constexpr uint32_t C_DDT = C_DST + 32768;        // bf16 dD^T [128 v][64 s], K-major A
constexpr uint32_t C_MISC = C_DDT + 16384;
constexpr uint32_t C_BAR = C_MISC, C_TMEM = C_MISC + 64;
constexpr uint32_t SMEMC_ALLOC = C_MISC + 128 + 1024;
static_assert(C_STAGE % 1024 == 0 && SMEMC_ALLOC <= 232448, "cotangent chain shared memory");
constexpr uint32_t TMC_S = 0, TMC_D = 128, TMC_COLS = 256;
constexpr uint32_t IDC_1 = idesc_bf16(128, 64, true, true);    // dO'^T A_qk
constexpr uint32_t IDC_2 = idesc_bf16(128, 64, false, true);   // dS^T Khat^T
constexpr uint32_t IDC_3 = idesc_bf16(128, 128, true, false);  // dO'^T Qtil
constexpr uint32_t IDC_4 = idesc_bf16(128, 128, false, false); // dD^T (-W)

struct DStateParams {
    CUtensorMap tdo;
    const uint8_t *rec;     // the forward's records
    uint8_t *bsave;         // backward records (dS^T, dD^T images written here)
    const int32_t *cu_seqlens;
    const int *chunk_off;   // varlen: first global chunk of each sequence
    int T, N, H, cpr;
    float scale;
    const float *dSf;       // [N,H,128,128] or null
    float *dS0;             // [N,H,128,128] or null
    int *status;
};

__global__ void __launch_bounds__(NTC, 1) kda_cb_dstate_kernel(const __grid_constant__ DStateParams P) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, lane = tid & 31;
    const int warp = __shfl_sync(0xffffffffu, tid >> 5, 0);
    const int H = P.H;
    const int n = blockIdx.x / H, h = blockIdx.x % H;
    long long bos, eos, c_first;
    if (P.cu_seqlens) { bos = P.cu_seqlens[n]; eos = P.cu_seqlens[n + 1]; c_first = P.chunk_off[n]; }
    else { bos = (long long)n * P.T; eos = bos + P.T; c_first = (long long)n * P.cpr; }
    const int nchunks = (int)((eos - bos + C - 1) / C);
    constexpr int kTma = 32, kSave = 64;

    uint64_t *bar_full = reinterpret_cast<uint64_t *>(sm + C_BAR);  // [2] stage loaded
    uint64_t *bar_m = bar_full + 2;                                 // products 1-3 done
    uint64_t *bar_s = bar_full + 3;                                 // product 4 done
    uint32_t *s_tmem = reinterpret_cast<uint32_t *>(sm + C_TMEM);
    if (warp == 0) { tmem_alloc(s_tmem, TMC_COLS); tmem_relinquish(); }
    if (tid == kTma) {
        for (int i = 0; i < 4; ++i) mbar_init(bar_full + i, 1);
        fence_mbar_init();
        tma_prefetch_desc(&P.tdo);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tb = *s_tmem;
    const uint32_t sb = smem_u32(sm);
    const uint64_t dK = sdesc_sw128(sb, 16, 1024);
    const uint64_t dM = sdesc_sw128(sb, 8192, 1024);
    auto dk = [&](uint32_t off) { return dK + (uint64_t)(off >> 4); };
    auto dm = [&](uint32_t off) { return dM + (uint64_t)(off >> 4); };
    const int quarter = warp & 3, half = warp >> 2;
    const uint32_t lane_sel = (uint32_t)(32 * quarter) << 16;
    const int v = 32 * quarter + lane;

    uint32_t full_out = 0;  // stage copies in flight (thread kTma)
    auto issue_stage = [&](int i) {  // step i = chunk nchunks - 1 - i
        const int s = i & 1, ci = nchunks - 1 - i;
        uint8_t *dst = sm + s * C_STAGE;
        mbar_arrive_expect_tx(bar_full + s, C_STAGE);
        bulk_load(dst, P.rec + ((c_first + ci) * H + h) * (long long)REC_BYTES, REC_BYTES, bar_full + s);
        const int t = (int)(bos + (long long)ci * C);
        for (int hf = 0; hf < 2; ++hf) tma_load_3d(dst + C_DO + hf * 8192, &P.tdo, bar_full + s, hf * 64, h, t);
        full_out |= 1u << s;
    };
    if (tid == kTma) {
        if (nchunks > 0) issue_stage(0);
        if (nchunks > 1) issue_stage(1);
    }
    const long long sbase = ((long long)n * H + h) * D * D;
    bool aborted = false;
    int issued_m = -1, issued_s = -1;  // last step whose products 1-3 / product 4 were issued (warp 0)
    for (int i = 0; i < nchunks; ++i) {
        const int s = i & 1, ci = nchunks - 1 - i;
        const uint32_t so = s * C_STAGE;
        uint8_t *stg = sm + so;
        if (tid == kSave && P.bsave) bulk_wait_read_all();  // the previous chunk's images were copied out
        {
            bool ok = true;
            if (warp == 0) {
                ok = mbar_wait(bar_full + s, (i >> 1) & 1, kWaitLimitNs);
                if (ok && i > 0) ok = mbar_wait(bar_s, (i - 1) & 1, kWaitLimitNs);
            }
            if (bar_or(1, NTC, !ok)) { aborted = true; break; }
        }
        tc_fence_after();
        if (tid == kTma) {
            full_out &= ~(1u << s);
            if (i >= 1 && i + 1 < nchunks) issue_stage(i + 1);  // into the stage step i - 1 used
        }
        // bf16 image of dS^T (the cotangent leaving this chunk), then dS^T diag(gamma) back
        const float *gam = reinterpret_cast<const float *>(stg + tp::R_GAM);
#pragma unroll
        for (int jc = 0; jc < 2; ++jc) {
            const int c0 = 64 * half + 32 * jc;
            float x[32];
            if (i == 0) {
#pragma unroll
                for (int j = 0; j < 32; ++j) x[j] = P.dSf ? P.dSf[sbase + (long long)(c0 + j) * D + v] : 0.f;
            } else {
                tmem_ld32(tb + TMC_S + lane_sel + c0, x);
                tmem_ld_wait();
            }
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) sts128(sm, C_DST + sw128_chunk(v, c0 + 8 * q4, 128), pack8(x + 8 * q4));
#pragma unroll
            for (int j = 0; j < 32; ++j) x[j] *= gam[c0 + j];
            tmem_st32(tb + TMC_S + lane_sel + c0, x);
        }
        // dO' = diag(scale / |q_r|) dO in place: the tile's 128 rows of 128 bytes (two
        // halves of 64 token rows), a half row of 4 chunks per thread
        {
            const float *invq = reinterpret_cast<const float *>(stg + tp::R_INVQ);
            const int rr = tid >> 1, r = rr & 63;
            const float f = P.scale * invq[r];
            const uint32_t off = so + C_DO + (uint32_t)rr * 128 + (uint32_t)(tid & 1) * 64;
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) {
                float y[8];
                unpack8(lds128(sm, off + 16 * q4), y);
#pragma unroll
                for (int j = 0; j < 8; ++j) y[j] *= f;
                sts128(sm, off + 16 * q4, pack8(y));
            }
        }
        tmem_st_wait();
        fence_proxy_async_smem();
        tc_fence_before();
        bar_sync(1, NTC);
        tc_fence_after();
        uint8_t *bsave = P.bsave ? P.bsave + ((c_first + ci) * H + h) * (long long)BR_BYTES : nullptr;
        if (tid == kSave && bsave) { bulk_store(bsave + BR_DS, sm + C_DST, 32768); bulk_commit(); }
        if (warp == 0) {
            const uint32_t ld = elect_one();
#pragma unroll
            for (int kq = 0; kq < 4; ++kq)
                mma_bf16_by(ld, tb + TMC_D, dm(so + C_DO + kq * 2048), dm(so + tp::R_AQK + kq * 2048), IDC_1, kq > 0);
#pragma unroll
            for (int kq = 0; kq < 8; ++kq)
                mma_bf16_by(ld, tb + TMC_D, dk(C_DST + (kq >> 2) * 16384 + (kq & 3) * 32), dm(so + tp::R_KH + kq * 2048),
                            IDC_2, 1);
#pragma unroll
            for (int kq = 0; kq < 4; ++kq)
                mma_bf16_by(ld, tb + TMC_S, dm(so + C_DO + kq * 2048), dk(so + tp::R_QT + kq * 32), IDC_3, 1);
            mma_commit_by(ld, bar_m);
            issued_m = i;
            if (!mbar_wait(bar_m, i & 1, kWaitLimitNs)) aborted = true;
        }
        if (bar_or(1, NTC, aborted)) { aborted = true; break; }
        tc_fence_after();
        {   // dD^T = dD~^T diag(1/|k_s|) -> bf16 image
            const float *invk = reinterpret_cast<const float *>(stg + tp::R_INVK);
            const int s0 = 32 * half;
            float x[32];
            tmem_ld32(tb + TMC_D + lane_sel + s0, x);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) x[j] *= invk[s0 + j];
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) sts128(sm, C_DDT + sw128_chunk(v, s0 + 8 * q4, 128), pack8(x + 8 * q4));
        }
        fence_proxy_async_smem();
        tc_fence_before();
        bar_sync(1, NTC);
        tc_fence_after();
        if (tid == kSave && bsave) { bulk_store(bsave + BR_DD, sm + C_DDT, 16384); bulk_commit(); }
        if (warp == 0) {
            const uint32_t ld = elect_one();
#pragma unroll
            for (int kq = 0; kq < 4; ++kq)
                mma_bf16_by(ld, tb + TMC_S, dk(C_DDT + kq * 32), dk(so + tp::R_WT + kq * 32), IDC_4, 1);
            mma_commit_by(ld, bar_s);
            issued_s = i;
        }
    }
    if (!aborted && P.dS0) {
        bool ok = true;
        if (warp == 0 && nchunks > 0) ok = mbar_wait(bar_s, (nchunks - 1) & 1, kWaitLimitNs);
        if (bar_or(1, NTC, !ok)) aborted = true;
        tc_fence_after();
        if (!aborted) {
#pragma unroll
            for (int jc = 0; jc < 2; ++jc) {
                const int c0 = 64 * half + 32 * jc;
                float x[32];
                if (nchunks == 0) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) x[j] = P.dSf ? P.dSf[sbase + (long long)(c0 + j) * D + v] : 0.f;
                } else {
                    tmem_ld32(tb + TMC_S + lane_sel + c0, x);
                    tmem_ld_wait();
                }
#pragma unroll
                for (int j = 0; j < 32; ++j) P.dS0[sbase + (long long)(c0 + j) * D + v] = x[j];
            }
        }
    }
    if (aborted) {
        if (warp == 0) {  // the products issued last complete before exit
            if (issued_s >= 0 && issued_s == issued_m) mbar_wait(bar_s, issued_s & 1, kWaitLimitNs);
            else if (issued_m >= 0) mbar_wait(bar_m, issued_m & 1, kWaitLimitNs);
        }
        if (tid == kTma) {
            for (int s = 0; s < 2; ++s)
                if ((full_out >> s) & 1u) mbar_wait(bar_full + s, 0, kWaitLimitNs), mbar_wait(bar_full + s, 1, kWaitLimitNs);
            if (P.status) atomicOr(P.status, 1);
        }
    }
    if (tid == kSave && P.bsave) bulk_wait_all();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        tmem_dealloc(tb, TMC_COLS);
    }
}

// MT[s] = M[s]^T for packed 128 x 128 states; one 32 x 32 tile per CTA.
__global__ void __launch_bounds__(256) kda_cb_transpose(const float *M, float *MT) {
    __shared__ float tile[32][33];
    const long long b = blockIdx.x, s = b >> 4;
    const int tr = (int)(b & 15) >> 2, tc = (int)(b & 3);
    const float *src = M + s * D * D;
    float *dst = MT + s * D * D;
    const int x = threadIdx.x & 31, y = threadIdx.x >> 5;
    for (int i = y; i < 32; i += 8) tile[i][x] = src[(32 * tr + i) * D + 32 * tc + x];
    __syncthreads();
    for (int i = y; i < 32; i += 8) dst[(32 * tc + i) * D + 32 * tr + x] = tile[x][i];
}

// ============================================================== chunk-local gradients
// One item = one (chunk, head); persistent CTAs of 512 threads (16 warps) walk the
// items. Products are warp-level bf16 tensor-core MMAs (m16n8k16, fp32 accumulate)
// on tiles in shared memory: the backward record's images (128-byte swizzle) and the
// raw rows (padded to 136 elements, 272-byte rows, so the eight rows of a fragment
// load fall on distinct banks); the three 64 x 64 x 64 products of the inverse run as
// tf32 MMAs on fp32 tiles. Every [64][128] result uses one warp layout -- warp w
// owns rows 16 (w % 4) .. and columns 32 (w / 4) .. -- so the contributions to dq^,
// dk^ and dG of an element stay in the registers of one thread until the end.
constexpr int NTI = 512;
constexpr int LP = 136;                  // padded row of a bf16 [64][128] tile (elements)
constexpr uint32_t PT = 64 * LP * 2;     // bytes of such a tile: 17,408
constexpr int LG = 136;                  // fp32 row of G / dG (floats)
constexpr int LF = 68, LT = 72;          // fp32 rows of the 64 x 64 tiles
constexpr int LA = 72;                   // bf16 row of the 64 x 64 dA tiles
// persistent regions
constexpr uint32_t X_Q = 0, X_K = PT, X_G = 2 * PT;               // raw q, raw k, G (fp32)
constexpr uint32_t X_DAQ = X_G + 64 * LG * 4;                     // dA_qk bf16 [64][72]
constexpr uint32_t X_MISC = X_DAQ + 64 * LA * 2;
constexpr uint32_t XM_RK = X_MISC, XM_RQ = X_MISC + 256, XM_B = X_MISC + 512, XM_DB = X_MISC + 768,
                   XM_DGC = X_MISC + 1024,   // [4][128] column partials of sum_s dKhat Khat
                   XM_DGAM = X_MISC + 3072,  // [128] gamma_c sum_v S dS_C
                   XM_RED = X_MISC + 3584,   // [16][128] f32 reduction scratch
                   XM_BAR = XM_RED + 8192,
                   XM_DAD = XM_BAR + 64,      // [64] the diagonal of dA_qk
                   XM_MSK = XM_DAD + 256,     // [64][4] u32: g >= lower bound (the clamp passes the gradient)
                   XM_KN = XM_MSK + 1024;     // [64] |k_r| (with the norm's eps; 1 without the norm, 0 past L)
constexpr uint32_t X_R = (XM_KN + 256 + 1023) / 1024 * 1024;      // phase region
// phase A/B
constexpr uint32_t Y_SV = X_R, Y_S0 = Y_SV + BR_S0, Y_DL = Y_SV + BR_DL, Y_DS = Y_SV + BR_DS, Y_DD = Y_SV + BR_DD;
constexpr uint32_t Y_DO = X_R + BR_BYTES, Y_DW = Y_DO + PT;       // raw dO; dW (bf16) -- raw g before it
// phase C (in the S0 and dS image areas, and dO's)
constexpr uint32_t Y_V = X_R, Y_TP = X_R + PT, Y_KT = Y_DS, Y_DTP = Y_DO;
// phase D: the k tiles for A, then the inverse's fp32 tiles
constexpr uint32_t Y_KYD = X_R, Y_KB1 = X_R + 25600, Y_KB2 = Y_KB1 + PT, Y_KB3 = Y_KB2 + PT, Y_KXD = Y_KB3 + PT,
                   Y_AF = Y_DW;
constexpr uint32_t Y_TF = X_R + 25600, Y_X1 = Y_TF + 64 * LT * 4, Y_DA = Y_X1 + 64 * LF * 4;
// phase E: the k tiles again, then the q tiles in their places
constexpr uint32_t Z_YD = X_R, Z_XD = X_R + PT, Z_B1 = Y_DA + 64 * LA * 2, Z_B2 = Z_B1 + PT, Z_B3 = Z_B2 + PT;
constexpr uint32_t X_END = Y_DW + PT;
constexpr uint32_t SMEMI_ALLOC = X_END + 1024;
static_assert(Y_TP + 8192 <= Y_DL && Y_KT + PT <= Y_DD && Y_DTP + 64 * LF * 4 <= Y_DW, "phase C layout");
static_assert(Y_KXD + PT <= Y_DO && Y_AF + 64 * LF * 4 <= X_END, "phase D layout (tiles)");
static_assert(Y_TF >= Y_TP + 8192 && Y_DA + 64 * LA * 2 <= Y_DTP, "phase D layout (inverse)");
static_assert(Z_XD + PT <= Y_DA && Z_B1 >= Y_DA + 64 * LA * 2 && Z_B3 + PT <= X_END, "phase E layout");
static_assert(SMEMI_ALLOC <= 232448, "intra backward shared memory");

struct IntraBwdParams {
    const __nv_bfloat16 *q, *k, *v, *g, *dout;
    const void *beta;
    int beta_f32;
    __nv_bfloat16 *dq, *dk, *dv, *dg;
    void *dbeta;
    const uint8_t *bsave;   // backward records
    const uint8_t *rec;     // the forward's records (T')
    const int32_t *cu_seqlens;
    const int *chunk_off;   // varlen: [N+1]
    int T, N, H, cpr;
    long long n_items;      // chunks x H
    float scale, lb;
    int use_l2, beta_prob;
    int *status;
};

// ---- warp-level bf16 MMA on shared-memory tiles
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void ldsm4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void ldsm4t(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
// Operand tiles: at(row, col) is the shared address of the 16-byte piece at (row, col),
// col % 8 == 0; kRow16 / kCol16 the address step of 16 rows / 16 columns where that step
// is a constant (kColLinear: along the columns too).
// A padded bf16 tile: element (row, col) at base + row * 2 LP + 2 col.
struct Pad {
    uint32_t base;
    static constexpr uint32_t kRow16 = 16 * 2 * LP, kCol16 = 32;
    static constexpr bool kColLinear = true;
    __device__ __forceinline__ uint32_t at(int row, int col) const { return base + (uint32_t)(row * (2 * LP) + 2 * col); }
};
// A padded bf16 64 x 64 tile with rows of LA elements.
struct PadA {
    uint32_t base;
    static constexpr uint32_t kRow16 = 16 * 2 * LA, kCol16 = 32;
    static constexpr bool kColLinear = true;
    __device__ __forceinline__ uint32_t at(int row, int col) const { return base + (uint32_t)(row * (2 * LA) + 2 * col); }
};
// A swizzled image with `rows` rows (64-column halves): linear along the rows only.
struct Img {
    uint32_t base;
    int rows;
    static constexpr uint32_t kRow16 = 16 * 128, kCol16 = 0;
    static constexpr bool kColLinear = false;
    __device__ __forceinline__ uint32_t at(int row, int col) const { return base + sw128_chunk(row, col, rows); }
};

// acc[NT] (+)= A[m0..m0+16][k0..k1] B[k0..k1][n0..n0+8 NT]; AT: A stored [K][M], BT: B
// stored [K][N] (else [M][K] and [N][K]); k0, k1 multiples of 16, NT even.
template <int NT, bool AT, bool BT, class OA, class OB>
__device__ __forceinline__ void wgemm(float (&acc)[NT][4], const OA &A, const OB &B, int m0, int n0, int k0, int k1,
                                      int lane) {
    const int li = lane & 7, l3 = (lane >> 3) & 1, l4 = lane >> 4;
    static_assert(AT || OA::kColLinear, "A read along its columns needs a column-linear tile");
    // this lane's fragment addresses at k0 and their step per 16 of k
    const uint32_t a0 = AT ? A.at(k0 + li + 8 * l4, m0 + 8 * l3) : A.at(m0 + li + 8 * l3, k0 + 8 * l4);
    constexpr uint32_t da = AT ? OA::kRow16 : OA::kCol16;
    constexpr bool b_lin = BT || OB::kColLinear;
    constexpr uint32_t db = BT ? OB::kRow16 : OB::kCol16;
    uint32_t b0[NT / 2];
#pragma unroll
    for (int p = 0; p < NT / 2; ++p)
        b0[p] = BT ? B.at(k0 + li + 8 * l3, n0 + 16 * p + 8 * l4) : B.at(n0 + 16 * p + li + 8 * l4, k0 + 8 * l3);
    const int nk = (k1 - k0) >> 4;
#pragma unroll 2
    for (int i = 0; i < nk; ++i) {
        uint32_t a[4];
        if (!AT) ldsm4(a0 + i * da, a);
        else ldsm4t(a0 + i * da, a);
#pragma unroll
        for (int p = 0; p < NT / 2; ++p) {
            uint32_t b[4];
            const uint32_t ba = b_lin ? b0[p] + i * db : B.at(n0 + 16 * p + li + 8 * l4, k0 + 16 * i + 8 * l3);
            if (!BT) ldsm4(ba, b);
            else ldsm4t(ba, b);
            mma16816(acc[2 * p], a, b[0], b[1]);
            mma16816(acc[2 * p + 1], a, b[2], b[3]);
        }
    }
}
template <int NT>
__device__ __forceinline__ void zero(float (&acc)[NT][4]) {
#pragma unroll
    for (int j = 0; j < NT; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
}
// 64 x 64 x 64 tf32 product, warp tile rows m0.., columns n0.. (NT n-tiles)
template <int NT, class FA, class FB>
__device__ __forceinline__ void tgemm(float (&acc)[NT][4], FA a, FB b, int m0, int n0, int g, int t) {
#pragma unroll 2
    for (int k0 = 0; k0 < 64; k0 += 8) {
        const uint32_t af[4] = {to_tf32(a(m0 + g, k0 + t)), to_tf32(a(m0 + g + 8, k0 + t)), to_tf32(a(m0 + g, k0 + t + 4)),
                                to_tf32(a(m0 + g + 8, k0 + t + 4))};
#pragma unroll
        for (int j = 0; j < NT; ++j) {
            const uint32_t bf[2] = {to_tf32(b(k0 + t, n0 + 8 * j + g)), to_tf32(b(k0 + t + 4, n0 + 8 * j + g))};
            mma_tf32_16x8x8(acc[j], af, bf);
        }
    }
}

__device__ __forceinline__ float2 ldf2(const uint8_t *sm, uint32_t off) { return *reinterpret_cast<const float2 *>(sm + off); }
__device__ __forceinline__ float2 ldb2(const uint8_t *sm, uint32_t off) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(sm + off));
}
__device__ __forceinline__ void stb2(uint8_t *sm, uint32_t off, float a, float b) {
    *reinterpret_cast<__nv_bfloat162 *>(sm + off) = __floats2bfloat162_rn(a, b);
}
__device__ __forceinline__ float e2(float x) { return ex2a(x * kL2e); }

__global__ void __launch_bounds__(NTI, 1) kda_cb_intra_kernel(const __grid_constant__ IntraBwdParams P) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, lane = tid & 31;
    const int warp = __shfl_sync(0xffffffffu, tid >> 5, 0);
    const int g8 = lane >> 2, t4 = lane & 3;
    const int mt = warp & 3, nq = warp >> 2;
    const int m0 = 16 * mt, n0 = 32 * nq, n0s = 16 * nq;  // [64][128] and [64][64] warp tiles
    const int H = P.H;
    const uint32_t sb = smem_u32(sm);
    float *rk = reinterpret_cast<float *>(sm + XM_RK), *rq = reinterpret_cast<float *>(sm + XM_RQ);
    float *bb = reinterpret_cast<float *>(sm + XM_B), *dbs = reinterpret_cast<float *>(sm + XM_DB);
    float *dgc = reinterpret_cast<float *>(sm + XM_DGC), *dgam = reinterpret_cast<float *>(sm + XM_DGAM);
    float *red = reinterpret_cast<float *>(sm + XM_RED);
    float *dad = reinterpret_cast<float *>(sm + XM_DAD);
    float *knorm = reinterpret_cast<float *>(sm + XM_KN);
    uint32_t *gmask = reinterpret_cast<uint32_t *>(sm + XM_MSK);
    float *Gs = reinterpret_cast<float *>(sm + X_G);
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + XM_BAR);
    if (tid == 0) { mbar_init(bar, 1); fence_mbar_init(); }
    __syncthreads();
    uint32_t phase = 0;
    const float lb = P.lb;
    const long long n_items = P.n_items >= 0 ? P.n_items : (long long)P.chunk_off[P.N] * H;

    const long long rowstride = (long long)H * D;  // elements between token rows
    // first token and rows of an item's chunk
    auto locate = [&](long long it, long long &t0_, int &L_) {  // item counts are below 2^31
        const int gc_ = (int)it / H;
        if (P.cu_seqlens) {  // the sequence holding global chunk gc_
            int lo = 0, hi = P.N - 1;
            while (lo < hi) { const int mid = (lo + hi + 1) >> 1; if (P.chunk_off[mid] <= gc_) lo = mid; else hi = mid - 1; }
            const int ci = gc_ - P.chunk_off[lo];
            t0_ = P.cu_seqlens[lo] + ci * C;
            L_ = (int)min((long long)C, (long long)P.cu_seqlens[lo + 1] - t0_);
        } else {
            const int n = gc_ / P.cpr, ci = gc_ - n * P.cpr;
            t0_ = (long long)n * P.T + ci * C;
            L_ = min(C, P.T - ci * C);
        }
    };
    // an item's inputs: the backward record (bulk), then raw rows (cp.async, one group);
    // which: 0 = record, dO and g;  1 = q and k
    auto issue_loads = [&](long long it, int which) {
        long long t0_;
        int L_;
        locate(it, t0_, L_);
        const int h_ = (int)it % H;
        if (which == 0 && tid == 0) {
            mbar_arrive_expect_tx(bar, BR_BYTES);
            bulk_load(sm + Y_SV, P.bsave + it * (long long)BR_BYTES, BR_BYTES, bar);
        }
        for (int e = tid; e < 2 * 64 * 16; e += NTI) {
            const int sel = e >> 10, r = (e >> 4) & 63, ch = e & 15;
            const uint32_t base = which ? (sel ? X_K : X_Q) : (sel ? Y_DW : Y_DO);
            const __nv_bfloat16 *src = which ? (sel ? P.k : P.q) : (sel ? P.g : P.dout);
            const uint32_t dst = base + r * (2 * LP) + ch * 16;
            if (r < L_) cp_async16(sm + dst, src + (t0_ + r) * rowstride + (long long)h_ * D + ch * 8);
            else *reinterpret_cast<uint4 *>(sm + dst) = make_uint4(0u, 0u, 0u, 0u);
        }
        cp_async_commit();
    };
    if (blockIdx.x < n_items) { issue_loads(blockIdx.x, 0); issue_loads(blockIdx.x, 1); }

    for (long long item = blockIdx.x; item < n_items; item += gridDim.x) {
        const int h = (int)item % H;
        long long t0;
        int L;
        locate(item, t0, L);
        const long long next = item + gridDim.x;
        auto grow = [&](const __nv_bfloat16 *base, int r) { return base + (t0 + r) * rowstride + (long long)h * D; };

        // ---------------- this item's inputs were issued before (the previous item's tail)
        if (tid < C) {
            float b = 0.f;
            if (tid < L) {
                const long long bi = (t0 + tid) * H + h;
                const float x = P.beta_f32 ? static_cast<const float *>(P.beta)[bi]
                                           : __bfloat162float(static_cast<const __nv_bfloat16 *>(P.beta)[bi]);
                b = P.beta_prob ? x : 1.f / (1.f + __expf(-x));
            }
            bb[tid] = b;
        }
        cp_async_wait_all();
        __syncthreads();
        // ---------------- norms (8 threads per row); G: 4 threads per channel, 16 rows each
        {
            const int r = tid >> 3, part = tid & 7;
            float sk = 0.f, sq = 0.f;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
                float fk[8], fq[8];
                unpack8(lds128(sm, X_K + r * (2 * LP) + (part * 2 + j) * 16), fk);
                unpack8(lds128(sm, X_Q + r * (2 * LP) + (part * 2 + j) * 16), fq);
#pragma unroll
                for (int e = 0; e < 8; ++e) { sk = fmaf(fk[e], fk[e], sk); sq = fmaf(fq[e], fq[e], sq); }
            }
#pragma unroll
            for (int o = 1; o < 8; o <<= 1) {
                sk += __shfl_xor_sync(0xffffffffu, sk, o);
                sq += __shfl_xor_sync(0xffffffffu, sq, o);
            }
            if (part == 0) {
                rk[r] = r < L ? (P.use_l2 ? rsqrtf(sk + 1e-6f) : 1.f) : 0.f;
                rq[r] = r < L ? (P.use_l2 ? rsqrtf(sq + 1e-6f) : 1.f) : 0.f;
                knorm[r] = r < L ? (P.use_l2 ? sqrtf(sk + 1e-6f) : 1.f) : 0.f;
            }
        }
        {   // a warp: 32 channels of one 16-row part; the clamp mask by ballot
            const int c = tid & 127, part = tid >> 7;
            float run = 0.f;
#pragma unroll 4
            for (int r = 16 * part; r < 16 * part + 16; ++r) {
                const float x = __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(sm + Y_DW + r * (2 * LP) + 2 * c));
                run += r < L ? fmaxf(x, lb) : 0.f;
                Gs[r * LG + c] = run;
                const uint32_t m = __ballot_sync(0xffffffffu, x >= lb);
                if (lane == 0) gmask[r * 4 + (c >> 5)] = m;
            }
            red[part * 128 + c] = run;
        }
        const bool ok = mbar_wait(bar, phase, kWaitLimitNs);
        phase ^= 1;
        if (__syncthreads_or(!ok)) {  // give up: the copy in flight gets one more bounded wait
            if (tid == 0) {
                mbar_wait(bar, phase ^ 1, kWaitLimitNs);
                if (P.status) atomicOr(P.status, 1);
            }
            return;
        }
        {   // carries of the G parts
            const int c = tid & 127, part = tid >> 7;
            float carry = 0.f;
            for (int p2 = 0; p2 < part; ++p2) carry += red[p2 * 128 + c];
            if (part > 0)
                for (int r = 16 * part; r < 16 * part + 16; ++r) Gs[r * LG + c] += carry;
        }
        // D~^T -> D^T (times |k_s|, zero for rows past the chunk)
        for (int e = tid; e < 128 * 8; e += NTI) {
            const int vv = e >> 3, cs = e & 7;
            const uint32_t off = Y_DL + sw128_chunk(vv, 8 * cs, 128);
            float y[8];
            unpack8(lds128(sm, off), y);
#pragma unroll
            for (int j = 0; j < 8; ++j) y[j] *= knorm[8 * cs + j];
            sts128(sm, off, pack8(y));
        }

        float dq_[16], dk_[16], dG_[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) dq_[e] = dk_[e] = dG_[e] = 0.f;
        // element pair (j, hi) of the [64][128] warp tile: row m0 + g8 + 8 hi, columns c, c + 1
        auto erow = [&](int hi) { return m0 + g8 + 8 * hi; };
        auto ecol = [&](int j) { return n0 + 8 * j + 2 * t4; };
        auto G2 = [&](int r, int c) { return *reinterpret_cast<const float2 *>(Gs + r * LG + c); };
        auto kh2 = [&](int r, int c) { const float2 x = ldb2(sm, X_K + r * (2 * LP) + 2 * c); const float s = rk[r]; return make_float2(x.x * s, x.y * s); };
        auto qh2 = [&](int r, int c) { const float2 x = ldb2(sm, X_Q + r * (2 * LP) + 2 * c); const float s = rq[r]; return make_float2(x.x * s, x.y * s); };

        __syncthreads();
        // ---------------- P1: dQtil = scale dO S^T;  P2: dW = -dD S^T -> bf16 tile
        {
            float acc[4][4];
            zero(acc);
            wgemm<4, false, true>(acc, Pad{sb + Y_DO}, Img{sb + Y_S0, 128}, m0, n0, 0, 128, lane);
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int hi = 0; hi < 2; ++hi) {
                    const int r = erow(hi), c = ecol(j), e = 4 * j + 2 * hi;
                    const float2 G = G2(r, c), q = qh2(r, c);
                    const float va = P.scale * acc[j][2 * hi] * e2(G.x), vb = P.scale * acc[j][2 * hi + 1] * e2(G.y);
                    dq_[e] += va; dq_[e + 1] += vb;
                    dG_[e] += va * q.x; dG_[e + 1] += vb * q.y;
                }
        }
        {
            float acc[4][4];
            zero(acc);
            wgemm<4, true, true>(acc, Img{sb + Y_DD, 128}, Img{sb + Y_S0, 128}, m0, n0, 0, 128, lane);
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int hi = 0; hi < 2; ++hi)
                    stb2(sm, Y_DW + erow(hi) * (2 * LP) + 2 * ecol(j), -acc[j][2 * hi], -acc[j][2 * hi + 1]);
        }
        // ---------------- gamma_c sum_v S[c][v] dS_C[c][v]: thread (8 channels, 4 values)
        {
            const int cs = tid & 15, vg = tid >> 4;
            float a8[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) a8[j] = 0.f;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int vv = 4 * vg + u;
                float s8[8], d8[8];
                unpack8(lds128(sm, Y_S0 + sw128_chunk(vv, 8 * cs, 128)), s8);
                unpack8(lds128(sm, Y_DS + sw128_chunk(vv, 8 * cs, 128)), d8);
#pragma unroll
                for (int j = 0; j < 8; ++j) a8[j] = fmaf(s8[j], d8[j], a8[j]);
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                a8[j] += __shfl_xor_sync(0xffffffffu, a8[j], 16);
                if (lane < 16) red[warp * 128 + 8 * cs + j] = a8[j];
            }
        }
        __syncthreads();
        if (tid < D) {
            float s = 0.f;
#pragma unroll
            for (int w = 0; w < NTI / 32; ++w) s += red[w * 128 + tid];
            dgam[tid] = s * e2(Gs[63 * LG + tid]);
        }
        // ---------------- P4: dKhat = D dS_C^T
        {
            float acc[4][4];
            zero(acc);
            wgemm<4, true, true>(acc, Img{sb + Y_DL, 128}, Img{sb + Y_DS, 128}, m0, n0, 0, 128, lane);
            float cs_[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int c = ecol(j);
                const float2 GC = G2(63, c);
                cs_[2 * j] = cs_[2 * j + 1] = 0.f;
#pragma unroll
                for (int hi = 0; hi < 2; ++hi) {
                    const int r = erow(hi), e = 4 * j + 2 * hi;
                    const float2 G = G2(r, c), k = kh2(r, c);
                    const float ea = e2(GC.x - G.x), eb = e2(GC.y - G.y);
                    const float xa = acc[j][2 * hi], xb = acc[j][2 * hi + 1];
                    dk_[e] += xa * ea; dk_[e + 1] += xb * eb;
                    const float pa = xa * k.x * ea, pb = xb * k.y * eb;
                    dG_[e] -= pa; dG_[e + 1] -= pb;
                    cs_[2 * j] += pa; cs_[2 * j + 1] += pb;
                }
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                float x = cs_[j];
                x += __shfl_xor_sync(0xffffffffu, x, 4);
                x += __shfl_xor_sync(0xffffffffu, x, 8);
                x += __shfl_xor_sync(0xffffffffu, x, 16);
                cs_[j] = x;
            }
            if (g8 == 0)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    dgc[mt * 128 + ecol(j)] = cs_[2 * j];
                    dgc[mt * 128 + ecol(j) + 1] = cs_[2 * j + 1];
                }
        }
        __syncthreads();  // S and dS_C images are free
        // ---------------- raw v and T' (cp.async into the freed areas), while P3 runs
        {
            const uint8_t *tp_src = P.rec + item * (long long)REC_BYTES + tp::R_TPU;
            for (int e = tid; e < 64 * 16 + 512; e += NTI) {
                if (e < 1024) {
                    const int r = e >> 4, ch = e & 15;
                    const uint32_t dst = Y_V + r * (2 * LP) + ch * 16;
                    if (r < L) cp_async16(sm + dst, grow(P.v, r) + ch * 8);
                    else *reinterpret_cast<uint4 *>(sm + dst) = make_uint4(0u, 0u, 0u, 0u);
                } else {
                    const int c16 = e - 1024;
                    cp_async16(sm + Y_TP + c16 * 16, tp_src + c16 * 16);
                }
            }
            cp_async_commit();
        }
        // ---------------- P3: dA_qk = scale dO D^T: the part below the diagonal -> bf16, the
        // diagonal apart (A_qk[r,r] = q^_r . k^_r has no gate factor, so its cotangent goes to
        // q^ and k^ directly and to no dG: the gated split would leave a rounding residue)
        {
            float acc[2][4];
            zero(acc);
            wgemm<2, false, true>(acc, Pad{sb + Y_DO}, Img{sb + Y_DL, 128}, m0, n0s, 0, 128, lane);
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int hi = 0; hi < 2; ++hi) {
                    const int r = erow(hi), c = n0s + 8 * j + 2 * t4;
                    const float va = P.scale * acc[j][2 * hi], vb = P.scale * acc[j][2 * hi + 1];
                    stb2(sm, X_DAQ + (r * LA + c) * 2, c < r ? va : 0.f, c + 1 < r ? vb : 0.f);
                    if (c == r) dad[r] = va;
                    if (c + 1 == r) dad[r] = vb;
                }
        }
        cp_async_wait_all();
        __syncthreads();  // v, T' in place; dO free
        // Ktil = k^ e^G -> bf16 tile
        for (int e = tid; e < 64 * 64; e += NTI) {
            const int r = e >> 6, c = 2 * (e & 63);
            const float2 G = G2(r, c), k = kh2(r, c);
            stb2(sm, Y_KT + r * (2 * LP) + 2 * c, k.x * e2(G.x), k.y * e2(G.y));
        }
        __syncthreads();
        // ---------------- P5: dT' = dD V^T + dW Ktil^T -> fp32
        float *dtp = reinterpret_cast<float *>(sm + Y_DTP);
        {
            float acc[2][4];
            zero(acc);
            wgemm<2, true, false>(acc, Img{sb + Y_DD, 128}, Pad{sb + Y_V}, m0, n0s, 0, 128, lane);
            wgemm<2, false, false>(acc, Pad{sb + Y_DW}, Pad{sb + Y_KT}, m0, n0s, 0, 128, lane);
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int hi = 0; hi < 2; ++hi) {
                    const int r = erow(hi), c = n0s + 8 * j + 2 * t4;
                    *reinterpret_cast<float2 *>(dtp + r * LF + c) = make_float2(acc[j][2 * hi], acc[j][2 * hi + 1]);
                }
        }
        // ---------------- P6: dV = T'^T dD (out); dKtil = T'^T dW
        {
            float acc[4][4];
            zero(acc);
            wgemm<4, true, false>(acc, Img{sb + Y_TP, 64}, Img{sb + Y_DD, 128}, m0, n0, 0, 64, lane);
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int hi = 0; hi < 2; ++hi) {
                    const int r = erow(hi);
                    if (r < L)
                        *reinterpret_cast<__nv_bfloat162 *>(P.dv + (t0 + r) * rowstride + (long long)h * D + ecol(j)) =
                            __floats2bfloat162_rn(acc[j][2 * hi], acc[j][2 * hi + 1]);
                }
        }
        {
            float acc[4][4];
            zero(acc);
            wgemm<4, true, true>(acc, Img{sb + Y_TP, 64}, Pad{sb + Y_DW}, m0, n0, 0, 64, lane);
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int hi = 0; hi < 2; ++hi) {
                    const int r = erow(hi), c = ecol(j), e = 4 * j + 2 * hi;
                    const float2 G = G2(r, c), k = kh2(r, c);
                    const float xa = acc[j][2 * hi] * e2(G.x), xb = acc[j][2 * hi + 1] * e2(G.y);
                    dk_[e] += xa; dk_[e + 1] += xb;
                    dG_[e] += xa * k.x; dG_[e + 1] += xb * k.y;
                }
        }
        __syncthreads();  // v, Ktil, dD, dW free
        // ---------------- the k tiles of the block-referenced products
        // B_j (j = 1..3): rows s < 16 j hold k^_s e^{E_j - G_s}, rows r >= 16 j hold
        // k^_r e^{G_r - E_j} (E_j = G_{16 j - 1}); XD / YD: k^ e^{+-(G - M_b)}, M_b = G_{16 b + 7}.
        // The q side (q_side) writes only XD and the rows r >= 16 j of the B_j, from q^.
        auto build_k = [&](uint32_t yd, uint32_t xd, uint32_t b1, uint32_t b2, uint32_t b3, bool q_side) {
            for (int e = tid; e < 64 * 64; e += NTI) {
                const int r = e >> 6, c = 2 * (e & 63), blk = r >> 4;
                const float2 G = G2(r, c), x = q_side ? qh2(r, c) : kh2(r, c), M = G2(16 * blk + 7, c);
                const float2 dm = make_float2(G.x - M.x, G.y - M.y);
                if (!q_side) stb2(sm, yd + r * (2 * LP) + 2 * c, x.x * e2(-dm.x), x.y * e2(-dm.y));
                stb2(sm, xd + r * (2 * LP) + 2 * c, x.x * e2(dm.x), x.y * e2(dm.y));
#pragma unroll
                for (int j = 1; j < 4; ++j) {
                    const uint32_t bt = j == 1 ? b1 : j == 2 ? b2 : b3;
                    const float2 E = G2(16 * j - 1, c);
                    const bool lo = r < 16 * j;
                    if (q_side && lo) continue;
                    const float fa = lo ? E.x - G.x : G.x - E.x, fb = lo ? E.y - G.y : G.y - E.y;
                    stb2(sm, bt + r * (2 * LP) + 2 * c, x.x * e2(fa), x.y * e2(fb));
                }
            }
        };
        build_k(Y_KYD, Y_KXD, Y_KB1, Y_KB2, Y_KB3, false);
        __syncthreads();
        // ---------------- A_kk (strict lower) -> fp32: warp (mt, nq) forms block (mt, nq)
        float *af = reinterpret_cast<float *>(sm + Y_AF);
        {
            const int cbk = nq;
            float acc[2][4];
            zero(acc);
            if (cbk < mt) {
                const uint32_t bt = mt == 1 ? Y_KB1 : mt == 2 ? Y_KB2 : Y_KB3;
                wgemm<2, false, false>(acc, Pad{sb + bt}, Pad{sb + bt}, m0, 16 * cbk, 0, 128, lane);
            } else if (cbk == mt) {
                wgemm<2, false, false>(acc, Pad{sb + Y_KXD}, Pad{sb + Y_KYD}, m0, 16 * cbk, 0, 128, lane);
            }
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int hi = 0; hi < 2; ++hi) {
                    const int r = erow(hi), c = 16 * cbk + 8 * j + 2 * t4;
                    *reinterpret_cast<float2 *>(af + r * LF + c) =
                        make_float2(c < r ? acc[j][2 * hi] : 0.f, c + 1 < r ? acc[j][2 * hi + 1] : 0.f);
                }
        }
        __syncthreads();  // the k tiles are free
        // ---------------- T = I - T' A_kk (tf32)
        float *tf = reinterpret_cast<float *>(sm + Y_TF);
        float *x1 = reinterpret_cast<float *>(sm + Y_X1);
        {
            float acc[2][4];
            zero(acc);
            tgemm(acc, [&](int m, int k) { return bf(sm, Y_TP + sw128(m, k, 64)); },
                  [&](int k, int n) { return af[k * LF + n]; }, m0, n0s, g8, t4);
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int hi = 0; hi < 2; ++hi) {
                    const int r = erow(hi), c = n0s + 8 * j + 2 * t4;
                    tf[r * LT + c] = (c == r ? 1.f : 0.f) - acc[j][2 * hi];
                    tf[r * LT + c + 1] = (c + 1 == r ? 1.f : 0.f) - acc[j][2 * hi + 1];
                }
        }
        __syncthreads();
        // db_s = sum_r dT'_rs T_rs (eight threads per column); dT' <- dT' diag(b)
        {
            const int c = tid >> 3, part = tid & 7;
            float s = 0.f;
#pragma unroll
            for (int r = 8 * part; r < 8 * part + 8; ++r) s = fmaf(dtp[r * LF + c], tf[r * LT + c], s);
            s += __shfl_xor_sync(0xffffffffu, s, 1);
            s += __shfl_xor_sync(0xffffffffu, s, 2);
            s += __shfl_xor_sync(0xffffffffu, s, 4);
            if (part == 0) dbs[c] = s;
        }
        // X1 = (dT' diag(b)) T^T
        {
            float acc[2][4];
            zero(acc);
            tgemm(acc, [&](int m, int k) { return dtp[m * LF + k] * bb[k]; }, [&](int k, int n) { return tf[n * LT + k]; },
                  m0, n0s, g8, t4);
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int hi = 0; hi < 2; ++hi) {
                    const int r = erow(hi), c = n0s + 8 * j + 2 * t4;
                    *reinterpret_cast<float2 *>(x1 + r * LF + c) = make_float2(acc[j][2 * hi], acc[j][2 * hi + 1]);
                }
        }
        __syncthreads();
        // dM = -T^T X1;  dA = diag(b) dM (s < r) -> bf16;  db_r += sum_{s<r} dM_rs A_rs
        {
            float acc[2][4];
            zero(acc);
            tgemm(acc, [&](int m, int k) { return tf[k * LT + m]; }, [&](int k, int n) { return x1[k * LF + n]; }, m0, n0s,
                  g8, t4);
            float rs[2] = {0.f, 0.f};
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int hi = 0; hi < 2; ++hi) {
                    const int r = erow(hi), c = n0s + 8 * j + 2 * t4;
                    const float ma = c < r ? -acc[j][2 * hi] : 0.f, mb = c + 1 < r ? -acc[j][2 * hi + 1] : 0.f;
                    rs[hi] += ma * af[r * LF + c] + mb * af[r * LF + c + 1];
                    stb2(sm, Y_DA + (r * LA + c) * 2, bb[r] * ma, bb[r] * mb);
                }
#pragma unroll
            for (int hi = 0; hi < 2; ++hi) {
                rs[hi] += __shfl_xor_sync(0xffffffffu, rs[hi], 1);
                rs[hi] += __shfl_xor_sync(0xffffffffu, rs[hi], 2);
                if (t4 == 0) red[nq * 64 + erow(hi)] = rs[hi];
            }
        }
        __syncthreads();
        if (tid < C) dbs[tid] += red[tid] + red[64 + tid] + red[128 + tid] + red[192 + tid];
        // ---------------- the k tiles again (A_kk's area is reused), then the gated gradients
        build_k(Z_YD, Z_XD, Z_B1, Z_B2, Z_B3, false);
        __syncthreads();
        const PadA pda{sb + Y_DA}, pdaq{sb + X_DAQ};
        // x side, rows of block mt: Zx = sum_s dA_rs y_s e^{G_r - G_s}, likewise Zqx with dA_qk
#pragma unroll 1
        for (int which = 0; which < 2; ++which) {
            const PadA dA = which ? pdaq : pda;
            float acc[4][4];
#pragma unroll 1
            for (int part = mt > 0 ? 0 : 1; part < 2; ++part) {  // 0: columns below the block, 1: the block
                zero(acc);
                const uint32_t bt = part ? Z_YD : mt == 1 ? Z_B1 : mt == 2 ? Z_B2 : Z_B3;
                wgemm<4, false, true>(acc, dA, Pad{sb + bt}, m0, n0, part ? 16 * mt : 0, part ? 16 * mt + 16 : 16 * mt, lane);
                const int refrow = part ? 16 * mt + 7 : 16 * mt - 1;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int c = ecol(j);
                    const float2 E = G2(refrow, c);
#pragma unroll
                    for (int hi = 0; hi < 2; ++hi) {
                        const int r = erow(hi), e = 4 * j + 2 * hi;
                        const float2 G = G2(r, c), x = which ? qh2(r, c) : kh2(r, c);
                        const float za = acc[j][2 * hi] * e2(G.x - E.x), zb = acc[j][2 * hi + 1] * e2(G.y - E.y);
                        if (which) { dq_[e] += za; dq_[e + 1] += zb; } else { dk_[e] += za; dk_[e + 1] += zb; }
                        dG_[e] += za * x.x; dG_[e + 1] += zb * x.y;
                    }
                }
            }
        }
        // y side, rows s of block mt: Zy = sum_r dA_rs x_r e^{G_r - G_s}, x = k^ (dA_kk), then q^ (dA_qk)
#pragma unroll 1
        for (int which = 0; which < 2; ++which) {
            if (which) {  // the q tiles in the places of the k tiles
                __syncthreads();
                build_k(Z_YD, Z_XD, Z_B1, Z_B2, Z_B3, true);
                __syncthreads();
            }
            const PadA dA = which ? pdaq : pda;
            float acc[4][4];
#pragma unroll 1
            for (int part = mt < 3 ? 0 : 1; part < 2; ++part) {  // 0: rows above the block, 1: the block
                zero(acc);
                const uint32_t bt = part ? Z_XD : mt == 0 ? Z_B1 : mt == 1 ? Z_B2 : Z_B3;
                wgemm<4, true, true>(acc, dA, Pad{sb + bt}, m0, n0, part ? 16 * mt : 16 * mt + 16, part ? 16 * mt + 16 : 64,
                                     lane);
                const int refrow = part ? 16 * mt + 7 : 16 * mt + 15;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int c = ecol(j);
                    const float2 E = G2(refrow, c);
#pragma unroll
                    for (int hi = 0; hi < 2; ++hi) {
                        const int r = erow(hi), e = 4 * j + 2 * hi;
                        const float2 G = G2(r, c), k = kh2(r, c);
                        const float za = acc[j][2 * hi] * e2(E.x - G.x), zb = acc[j][2 * hi + 1] * e2(E.y - G.y);
                        dk_[e] += za; dk_[e + 1] += zb;
                        dG_[e] -= za * k.x; dG_[e + 1] -= zb * k.y;
                    }
                }
            }
        }
        __syncthreads();  // the tile areas (record, dO, dW) are free: the next item's record, dO and g
        if (next < n_items) issue_loads(next, 0);
        // the diagonal of dA_qk: dq^_r += dA_qk[r,r] k^_r, dk^_r += dA_qk[r,r] q^_r
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int hi = 0; hi < 2; ++hi) {
                const int r = erow(hi), c = ecol(j), e = 4 * j + 2 * hi;
                const float2 k = kh2(r, c), q = qh2(r, c);
                const float d = dad[r];
                dq_[e] += d * k.x; dq_[e + 1] += d * k.y;
                dk_[e] += d * q.x; dk_[e + 1] += d * q.y;
            }
        // ---------------- outputs
        // row dots k^ . dk^ and q^ . dq^ (quad sums, then the four column quarters)
        {
            float sk2[2] = {0.f, 0.f}, sq2[2] = {0.f, 0.f};
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int hi = 0; hi < 2; ++hi) {
                    const int r = erow(hi), c = ecol(j), e = 4 * j + 2 * hi;
                    const float2 k = kh2(r, c), q = qh2(r, c);
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
            __syncthreads();  // red and G's readers are done
            if (t4 == 0)
#pragma unroll
                for (int hi = 0; hi < 2; ++hi) {
                    red[nq * 64 + erow(hi)] = sk2[hi];
                    red[256 + nq * 64 + erow(hi)] = sq2[hi];
                }
            // dG into G's area (every read of G is behind the barrier above)
#pragma unroll
            for (int j = 0; j < 4; ++j)
#pragma unroll
                for (int hi = 0; hi < 2; ++hi) {
                    const int e = 4 * j + 2 * hi;
                    *reinterpret_cast<float2 *>(Gs + erow(hi) * LG + ecol(j)) = make_float2(dG_[e], dG_[e + 1]);
                }
        }
        __syncthreads();
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int hi = 0; hi < 2; ++hi) {
                const int r = erow(hi), c = ecol(j), e = 4 * j + 2 * hi;
                if (r >= L) continue;
                const float dotk = red[r] + red[64 + r] + red[128 + r] + red[192 + r];
                const float dotq = red[256 + r] + red[320 + r] + red[384 + r] + red[448 + r];
                const float2 k = kh2(r, c), q = qh2(r, c);
                float ka = dk_[e], kb = dk_[e + 1], qa = dq_[e], qb = dq_[e + 1];
                if (P.use_l2) {
                    ka = rk[r] * (ka - k.x * dotk); kb = rk[r] * (kb - k.y * dotk);
                    qa = rq[r] * (qa - q.x * dotq); qb = rq[r] * (qb - q.y * dotq);
                }
                const long long o = (t0 + r) * rowstride + (long long)h * D + c;
                *reinterpret_cast<__nv_bfloat162 *>(P.dk + o) = __floats2bfloat162_rn(ka, kb);
                *reinterpret_cast<__nv_bfloat162 *>(P.dq + o) = __floats2bfloat162_rn(qa, qb);
            }
        __syncthreads();  // raw q and k are no longer read: the next item's
        if (next < n_items) issue_loads(next, 1);
        // dg: reverse in-chunk cumsum of dG (with dG_C on the last row), clamp mask; four
        // threads per channel, 16 rows each
        {
            const int c = tid & 127, part = tid >> 7;
            const float *gcol = Gs + c;
            float sfx[16];
            float run = part == 3 ? dgc[c] + dgc[128 + c] + dgc[256 + c] + dgc[384 + c] + dgam[c] : 0.f;
#pragma unroll
            for (int i = 15; i >= 0; --i) { run += gcol[(16 * part + i) * LG]; sfx[i] = run; }
            red[512 + part * 128 + c] = run;
            __syncthreads();
            float carry = 0.f;
            for (int p2 = part + 1; p2 < 4; ++p2) carry += red[512 + p2 * 128 + c];
            __nv_bfloat16 *dgp = P.dg + (t0 + 16 * part) * rowstride + (long long)h * D + c;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int r = 16 * part + i;
                const bool pass = (gmask[r * 4 + (c >> 5)] >> (c & 31)) & 1u;
                if (r < L) dgp[i * rowstride] = __float2bfloat16_rn(pass ? sfx[i] + carry : 0.f);
            }
        }
        if (tid < L) {
            const float b = bb[tid], d = dbs[tid];
            const float db = P.beta_prob ? d : d * b * (1.f - b);
            const long long bi = (t0 + tid) * H + h;
            if (P.beta_f32) static_cast<float *>(P.dbeta)[bi] = db;
            else static_cast<__nv_bfloat16 *>(P.dbeta)[bi] = __float2bfloat16_rn(db);
        }
        __syncthreads();  // before the next item's loads overwrite the tiles
    }
}

// ============================================================== host
bool cb_supported(const BwdParams &p, bool bf16, int Dk, int Dv) {
    return bf16 && Dk == D && Dv == D && p.has_lb && p.lb >= -5.f && p.H > 0;
}

ChunkParams cb_fwd_params(const BwdParams &p) {
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
    return f;
}

size_t round1k(size_t b) { return (b + 1023) / 1024 * 1024; }
long long cb_max_chunks(const BwdParams &p) {
    return p.cu_seqlens ? ((long long)p.T + C - 1) / C + p.N : (long long)p.N * (((long long)p.T + C - 1) / C);
}

// Workspace: [the forward's two-pass workspace][backward records][chunk offsets][chunk
// table][segment form: per (segment, head) the cotangent offsets N', M^T and the
// leaving cotangents]
struct CbLayout {
    size_t fwd, save, offs, table, seg, total;
};
int cb_seg_count(const BwdParams &p) { return chunk_2pass_seg_count(cb_fwd_params(p)); }
CbLayout cb_layout(const BwdParams &p) {
    CbLayout L;
    L.fwd = round1k(chunk_2pass_workspace_bytes(cb_fwd_params(p)));
    L.save = (size_t)cb_max_chunks(p) * p.H * BR_BYTES;
    L.offs = p.cu_seqlens ? round1k((size_t)(p.N + 1) * 4) : 0;
    L.table = p.cu_seqlens ? round1k((size_t)cb_max_chunks(p) * 8) + 16384 : 0;
    const int P = cb_seg_count(p);
    L.seg = P > 1 ? 3 * round1k((size_t)p.N * P * p.H * D * D * 4) : 0;
    L.total = L.fwd + L.save + L.offs + L.table + L.seg;
    return L;
}

}  // namespace cb

cudaError_t chunk_2pass_chunk_table(const int32_t *cu, int N, int *chunk_off, int2 *chunk_tok, uint8_t *consts,
                                    cudaStream_t st);

size_t bwd_chunked_workspace_bytes(const BwdParams &p, bool bf16, int Dk, int Dv) {
    if (!cb::cb_supported(p, bf16, Dk, Dv)) return 0;
    return cb::cb_layout(p).total;
}

// The chunked backward: the forward (records, and every chunk's entering state and D
// saved), the cotangent chain, then the chunk-local gradients. Needs
// bwd_chunked_workspace_bytes(p) bytes of workspace, 256-byte aligned.
cudaError_t launch_bwd_chunked(const BwdParams &p, void *workspace, cudaStream_t st) {
    using namespace cb;
    const CbLayout Lo = cb_layout(p);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    uint8_t *save = ws + Lo.fwd;
    int *chunk_off = reinterpret_cast<int *>(save + Lo.save);
    int2 *chunk_tok = reinterpret_cast<int2 *>(save + Lo.save + Lo.offs + 16384);
    uint8_t *consts = save + Lo.save + Lo.offs;
    const long long total = p.cu_seqlens ? (long long)p.T : (long long)p.N * p.T;
    const long long nchunks_max = cb_max_chunks(p);
    if (total <= 0 || nchunks_max * p.H >= (1LL << 31)) return cudaErrorInvalidValue;
    const ChunkParams f = cb_fwd_params(p);
    cudaError_t e;
    if ((e = launch_chunk_2pass_save(f, ws, nullptr, save, st)) != cudaSuccess) return e;
    int *status = reinterpret_cast<int *>(ws);  // the forward's status word (cleared by its first pass)
    if (p.cu_seqlens && (e = chunk_2pass_chunk_table(p.cu_seqlens, p.N, chunk_off, chunk_tok, consts, st)) != cudaSuccess)
        return e;
    const int cpr = (int)(((long long)p.T + C - 1) / C);
    // the cotangent chain
    DStateParams B;
    memset(&B, 0, sizeof(B));
    if (!make_map(&B.tdo, p.dout, total, p.H)) return cudaErrorInvalidValue;
    B.rec = chunk_2pass_records(f, ws);
    B.bsave = save;
    B.cu_seqlens = p.cu_seqlens;
    B.chunk_off = chunk_off;
    B.T = p.T; B.N = p.N; B.H = p.H; B.cpr = cpr;
    B.scale = p.scale;
    B.dSf = p.dSf;
    B.dS0 = p.dS0;
    B.status = status;
    if ((e = cudaFuncSetAttribute(kda_cb_dstate_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEMC_ALLOC)) !=
        cudaSuccess)
        return e;
    const int32_t *cu_v = nullptr;
    const int *chunk_off_v = nullptr;
    const float *Mseg = nullptr;
    const int P = chunk_2pass_seg_info(f, ws, &cu_v, &chunk_off_v, &Mseg);
    if (P == 1) {
        count_launch();
        kda_cb_dstate_kernel<<<(unsigned)((long long)p.N * p.H), NTC, SMEMC_ALLOC, st>>>(B);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    } else {
        // the segments of the forward's view: the cotangent over a segment is affine in the
        // cotangent leaving it, dS_start = M^T dS_end + N', so the chain runs once over all
        // segments from zero (the N'), the segments are walked back with M^T to their
        // leaving cotangents, and the chain runs again from those (writing the records)
        const size_t sb = round1k((size_t)p.N * P * p.H * D * D * 4);
        float *Nrev = reinterpret_cast<float *>(save + Lo.save + Lo.offs + Lo.table);
        float *MT = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(Nrev) + sb);
        float *dSend = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(Nrev) + 2 * sb);
        const long long nv = (long long)p.N * P * p.H;
        DStateParams Bv = B;
        Bv.cu_seqlens = cu_v;
        Bv.chunk_off = chunk_off_v;
        Bv.T = p.cu_seqlens ? p.T : p.N * p.T;
        Bv.N = p.N * P;
        Bv.bsave = nullptr;
        Bv.dSf = nullptr;
        Bv.dS0 = Nrev;
        count_launch();
        kda_cb_dstate_kernel<<<(unsigned)nv, NTC, SMEMC_ALLOC, st>>>(Bv);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        count_launch();
        kda_cb_transpose<<<(unsigned)(nv * 16), 256, 0, st>>>(Mseg, MT);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        if ((e = seg_chain_launch<D>(p.dSf, MT, Nrev, D, (long long)D * D, dSend, p.dS0, p.N, p.H, P, st, 1)) !=
            cudaSuccess)
            return e;
        Bv.bsave = save;
        Bv.dSf = dSend;
        Bv.dS0 = nullptr;
        count_launch();
        kda_cb_dstate_kernel<<<(unsigned)nv, NTC, SMEMC_ALLOC, st>>>(Bv);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    // the chunk-local gradients: every (chunk, head) of the chunk numbering (varlen: the
    // table's count; slots past it belong to no sequence and are skipped by count)
    IntraBwdParams I;
    memset(&I, 0, sizeof(I));
    I.q = static_cast<const __nv_bfloat16 *>(p.q);
    I.k = static_cast<const __nv_bfloat16 *>(p.k);
    I.v = static_cast<const __nv_bfloat16 *>(p.v);
    I.g = static_cast<const __nv_bfloat16 *>(p.g);
    I.dout = static_cast<const __nv_bfloat16 *>(p.dout);
    I.beta = p.beta;
    I.beta_f32 = 0;
    I.dq = static_cast<__nv_bfloat16 *>(p.dq);
    I.dk = static_cast<__nv_bfloat16 *>(p.dk);
    I.dv = static_cast<__nv_bfloat16 *>(p.dv);
    I.dg = static_cast<__nv_bfloat16 *>(p.dg);
    I.dbeta = p.dbeta;
    I.bsave = save;
    I.rec = B.rec;
    I.cu_seqlens = p.cu_seqlens;
    I.chunk_off = chunk_off;
    I.T = p.T; I.N = p.N; I.H = p.H; I.cpr = cpr;
    I.n_items = p.cu_seqlens ? -1 : (long long)p.N * cpr * p.H;
    I.scale = p.scale;
    I.lb = p.lb;
    I.use_l2 = p.use_l2;
    I.beta_prob = p.beta_prob;
    I.status = status;
    int dev = 0, nsm = 148;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(kda_cb_intra_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEMI_ALLOC)) !=
        cudaSuccess)
        return e;
    const long long items_max = nchunks_max * p.H;
    count_launch();
    kda_cb_intra_kernel<<<(unsigned)std::min<long long>(items_max, nsm), NTI, SMEMI_ALLOC, st>>>(I);
    return cudaGetLastError();
}

}  // namespace kda
