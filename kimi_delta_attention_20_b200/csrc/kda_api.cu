// Host side of the C ABI declared in include/kda.h: argument validation,
// kernel selection and launch. No allocation, no synchronisation.
#include <math.h>
#include <stdint.h>

#include <atomic>

#include "../../include/kda.h"
#include "kda_common.cuh"
#include "kda_bwd.cuh"

namespace kda {
cudaError_t launch_decode(const StepParams &p, float *state_out, bool bf16, int Dk, int Dv, cudaStream_t st);
cudaError_t launch_chunk_simt(const ChunkParams &p, bool bf16, int Dk, int Dv, int chunk, cudaStream_t st);
cudaError_t launch_chunk_rec(const ChunkParams &p, bool bf16, int Dk, int Dv, void *workspace, size_t workspace_bytes,
                             cudaStream_t st);
size_t chunk_rec_workspace_bytes(const ChunkParams &p, bool bf16, int Dk, int Dv);
bool chunk_tc_supported(bool bf16, int Dk, int Dv, int chunk_size);
size_t chunk_tc_workspace_bytes(int N, int H, int Dk, int Dv);
cudaError_t launch_chunk_tc(const ChunkParams &p, int Dk, int Dv, void *workspace,
                            size_t workspace_bytes, const int32_t *cu_host, cudaStream_t st);
size_t chunk_2pass_workspace_bytes(const ChunkParams &p);
cudaError_t launch_chunk_2pass(const ChunkParams &p, void *workspace, const int32_t *cu_host, cudaStream_t st);
bool token_conv_supported(int K);
size_t bwd_workspace_bytes(const BwdParams &p, bool bf16, int Dk, int Dv);
size_t bwd_workspace_bytes_min(bool varlen, long long T, int N, int H, int Dk, int Dv);
cudaError_t launch_bwd(BwdParams p, bool bf16, int Dk, int Dv, void *workspace, size_t workspace_bytes, cudaStream_t st);
cudaError_t launch_token(const TokenParams &tp, float *state_out, bool bf16, int Dk, int Dv, cudaStream_t st);
}  // namespace kda

namespace {

thread_local int g_last_cuda_error = 0;

kda_status cuda_status(cudaError_t e) {
    if (e == cudaSuccess) return KDA_OK;
    g_last_cuda_error = (int)e;
    return KDA_ERR_CUDA;
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// An out-of-place decode state: 16-byte aligned and either the state itself or
// disjoint from it (a partial overlap would let one CTA read what another wrote).
bool state_out_ok(const float *state, const float *out, long long N, int H, int Dk, int Dv) {
    if (!out || out == state) return true;
    if (!aligned(out, 16)) return false;
    const uintptr_t bytes = (uintptr_t)(N * H * (long long)Dk * Dv) * sizeof(float);
    const uintptr_t a = reinterpret_cast<uintptr_t>(state), b = reinterpret_cast<uintptr_t>(out);
    return a + bytes <= b || b + bytes <= a;
}

bool head_dim_ok(int d) { return d == 32 || d == 64 || d == 128; }

float resolve_scale(float s, int Dk) {
    if (!(s > 0.f)) return 1.0f / sqrtf((float)Dk);  // also catches NaN
    return s;
}

// Gate mode against the lower-bound flag: the unbounded in-kernel form has no
// lower bound and the safe form needs one.
kda_status check_gate_mode(int mode, int has_lb) {
    if (mode == KDA_GATE_LOG) return KDA_OK;
    if (mode == KDA_GATE_SOFTPLUS) return has_lb ? KDA_ERR_INVALID_ARGUMENT : KDA_OK;
    if (mode == KDA_GATE_SAFE) return has_lb ? KDA_OK : KDA_ERR_INVALID_ARGUMENT;
    return KDA_ERR_INVALID_ARGUMENT;
}

// Gate parameter pointers, when the in-kernel gate will read them.
kda_status check_gate_ptrs(int mode, const float *A_log, const float *dt_bias) {
    if (mode == KDA_GATE_LOG) return KDA_OK;
    if (!A_log || !aligned(A_log, 4) || (dt_bias && !aligned(dt_bias, 4))) return KDA_ERR_INVALID_ARGUMENT;
    return KDA_OK;
}

// Shapes and flags only (shared by the workspace query and the launch).
kda_status check_chunk_shape(const kda_chunk_args *a, int *N_out) {
    if (!a) return KDA_ERR_INVALID_ARGUMENT;
    if (a->dtype != KDA_DTYPE_F32 && a->dtype != KDA_DTYPE_BF16) return KDA_ERR_INVALID_ARGUMENT;
    if (a->B < 1 || a->T < 0 || a->H < 1 || a->Dk < 1 || a->Dv < 1) return KDA_ERR_INVALID_ARGUMENT;
    if (!head_dim_ok(a->Dk) || !head_dim_ok(a->Dv)) return KDA_ERR_UNSUPPORTED;
    if (a->chunk_size != 0 && a->chunk_size != 32 && a->chunk_size != 64) return KDA_ERR_UNSUPPORTED;
    if (a->has_lower_bound && !(a->lower_bound < 0.f)) return KDA_ERR_INVALID_ARGUMENT;
    if (check_gate_mode(a->gate_mode, a->has_lower_bound) != KDA_OK) return KDA_ERR_INVALID_ARGUMENT;
    if ((long long)a->B * a->T * a->H * (a->Dk > a->Dv ? a->Dk : a->Dv) >= (1LL << 40))
        return KDA_ERR_INVALID_ARGUMENT;
    int N = a->N;
    if (a->cu_seqlens) {
        if (a->B != 1 || N < 1) return KDA_ERR_INVALID_ARGUMENT;
    } else {
        if (N == 0) N = a->B;
        if (N != a->B) return KDA_ERR_INVALID_ARGUMENT;
    }
    if ((long long)N * a->H * 4 >= 0x7fffffffLL) return KDA_ERR_INVALID_ARGUMENT;
    *N_out = N;
    return KDA_OK;
}

}  // namespace

namespace kda {
void record_cuda_error(int e) { g_last_cuda_error = e; }

std::atomic<unsigned long long> g_launches{0};
void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

// The status word at `word` (device memory) once `st` has drained: non-zero means a
// bounded device wait gave up.
kda_status read_status_word(const void *word, cudaStream_t st) {
    int v = 0;
    cudaError_t e = cudaMemcpyAsync(&v, word, sizeof(int), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_status(e);
    return v ? KDA_ERR_TIMEOUT : KDA_OK;
}
}  // namespace kda

namespace {
// The forward's shape view of backward arguments (shared validation).
kda_chunk_args fwd_view(const kda_chunk_bwd_args *a) {
    kda_chunk_args f{};
    f.dtype = a->dtype;
    f.B = a->B; f.T = a->T; f.H = a->H; f.Dk = a->Dk; f.Dv = a->Dv;
    f.cu_seqlens = a->cu_seqlens; f.cu_seqlens_host = a->cu_seqlens_host; f.N = a->N;
    f.has_lower_bound = a->has_lower_bound; f.lower_bound = a->lower_bound;
    f.gate_mode = KDA_GATE_LOG;
    return f;
}
}  // namespace

namespace kda {
// Smallest workspace kda_chunk_fwd accepts for these arguments (the single-pass
// tensor-core kernel's status word, or 0 where no kernel needs scratch).
kda_status chunk_workspace_min_bytes(const kda_chunk_args *a, size_t *bytes) {
    int N = 0;
    kda_status s = check_chunk_shape(a, &N);
    if (s != KDA_OK) return s;
    *bytes = 0;
    if (chunk_tc_supported(a->dtype == KDA_DTYPE_BF16, a->Dk, a->Dv, a->chunk_size) &&
        (long long)a->B * a->T > 0)
        *bytes = chunk_tc_workspace_bytes(N, a->H, a->Dk, a->Dv);
    return KDA_OK;
}
}  // namespace kda

extern "C" {

const char *kda_status_string(kda_status s) {
    switch (s) {
    case KDA_OK: return "ok";
    case KDA_ERR_INVALID_ARGUMENT: return "invalid argument";
    case KDA_ERR_UNSUPPORTED: return "unsupported configuration";
    case KDA_ERR_CUDA: return "CUDA error";
    case KDA_ERR_TIMEOUT: return "device-side wait timed out";
    case KDA_ERR_WORKSPACE: return "workspace missing or too small";
    }
    return "unknown status";
}

int kda_last_cuda_error(void) { return g_last_cuda_error; }

int kda_version(void) { return KDA_VERSION; }

unsigned long long kda_launch_count(void) { return kda::g_launches.load(std::memory_order_relaxed); }

kda_status kda_chunk_fwd_workspace_size(const kda_chunk_args *a, size_t *bytes) {
    if (!bytes) return KDA_ERR_INVALID_ARGUMENT;
    int N = 0;
    kda_status s = check_chunk_shape(a, &N);
    if (s != KDA_OK) return s;
    *bytes = 0;
    if (kda::chunk_tc_supported(a->dtype == KDA_DTYPE_BF16, a->Dk, a->Dv, a->chunk_size) &&
        (long long)a->B * a->T > 0) {
        kda::ChunkParams p{};
        p.cu_seqlens = a->cu_seqlens;  // only its presence is read
        p.T = a->T; p.N = N; p.H = a->H;
        *bytes = kda::chunk_2pass_workspace_bytes(p);
    } else if (a->chunk_size != 32 && (long long)a->B * a->T > 0) {
        kda::ChunkParams p{};
        p.cu_seqlens = a->cu_seqlens;  // only its presence is read
        p.T = a->T; p.N = N; p.H = a->H;
        *bytes = kda::chunk_rec_workspace_bytes(p, a->dtype == KDA_DTYPE_BF16, a->Dk, a->Dv);
    }
    return KDA_OK;
}


kda_status kda_chunk_fwd(const kda_chunk_args *a, void *stream) {
    int N = 0;
    kda_status s = check_chunk_shape(a, &N);
    if (s != KDA_OK) return s;
    const bool bf16 = a->dtype == KDA_DTYPE_BF16;
    const size_t esz = bf16 ? 2 : 4;
    const long long ntok = (long long)a->B * a->T;
    if (ntok > 0) {
        if (!a->q || !a->k || !a->v || !a->g || !a->beta || !a->o) return KDA_ERR_INVALID_ARGUMENT;
        if (!aligned(a->q, 16) || !aligned(a->k, 16) || !aligned(a->v, 16) || !aligned(a->g, 16) ||
            !aligned(a->o, 16) || !aligned(a->beta, esz))
            return KDA_ERR_INVALID_ARGUMENT;
        if (check_gate_ptrs(a->gate_mode, a->A_log, a->dt_bias) != KDA_OK) return KDA_ERR_INVALID_ARGUMENT;
    }
    if ((a->initial_state && !aligned(a->initial_state, 16)) ||
        (a->final_state && !aligned(a->final_state, 16)))
        return KDA_ERR_INVALID_ARGUMENT;
    if (a->cu_seqlens_host) {
        const int32_t *cu = a->cu_seqlens_host;
        if (cu[0] != 0 || cu[N] != a->T) return KDA_ERR_INVALID_ARGUMENT;
        for (int n = 0; n < N; ++n)
            if (cu[n + 1] < cu[n]) return KDA_ERR_INVALID_ARGUMENT;
    }
    if (!a->cu_seqlens && a->cu_seqlens_host) return KDA_ERR_INVALID_ARGUMENT;

    kda::ChunkParams p{};
    p.q = a->q; p.k = a->k; p.v = a->v; p.g = a->g; p.beta = a->beta; p.o = a->o;
    p.S0 = a->initial_state; p.S_out = a->final_state;
    p.cu_seqlens = a->cu_seqlens; p.T = a->T; p.N = N; p.H = a->H;
    p.scale = resolve_scale(a->scale, a->Dk);
    p.use_l2 = a->use_qk_l2norm ? 1 : 0;
    p.has_lb = a->has_lower_bound ? 1 : 0;
    p.lb = a->lower_bound;
    p.gate_mode = a->gate_mode;
    p.A_log = a->A_log;
    p.dt_bias = a->dt_bias;
    p.beta_prob = a->beta_is_prob ? 1 : 0;
    p.stall_first_wait = (a->debug_flags & KDA_DEBUG_STALL_FIRST_WAIT) ? 1 : 0;
    cudaStream_t st = static_cast<cudaStream_t>(stream);

    if (ntok > 0 && kda::chunk_tc_supported(bf16, a->Dk, a->Dv, a->chunk_size)) {
        // two passes when the workspace holds the per-chunk records, else the single-pass kernel
        if (a->workspace && aligned(a->workspace, 256) &&
            a->workspace_bytes >= kda::chunk_2pass_workspace_bytes(p))
            return cuda_status(kda::launch_chunk_2pass(p, a->workspace, a->cu_seqlens_host, st));
        const size_t need = kda::chunk_tc_workspace_bytes(N, a->H, a->Dk, a->Dv);
        if (need > 0 && (!a->workspace || a->workspace_bytes < need || !aligned(a->workspace, 256)))
            return KDA_ERR_WORKSPACE;
        return cuda_status(kda::launch_chunk_tc(p, a->Dk, a->Dv, a->workspace, a->workspace_bytes,
                                                a->cu_seqlens_host, st));
    }
    // other shapes: the register-resident recurrence; an explicit 32-token chunk
    // request runs the chunked CUDA-core kernel with C = 32 (same result)
    if (a->chunk_size == 32) return cuda_status(kda::launch_chunk_simt(p, bf16, a->Dk, a->Dv, 32, st));
    return cuda_status(kda::launch_chunk_rec(p, bf16, a->Dk, a->Dv, a->workspace, a->workspace_bytes, st));
}

kda_status kda_chunk_fwd_status(const kda_chunk_args *a, void *stream) {
    if (!a) return KDA_ERR_INVALID_ARGUMENT;
    size_t need = 0;
    kda_status s = kda::chunk_workspace_min_bytes(a, &need);
    if (s != KDA_OK) return s;
    if (need == 0) return KDA_OK;  // a kernel without device waits
    if (!a->workspace) return KDA_ERR_WORKSPACE;
    return kda::read_status_word(a->workspace, static_cast<cudaStream_t>(stream));
}

kda_status kda_recurrent_step(const kda_step_args *a, void *stream) {
    if (!a) return KDA_ERR_INVALID_ARGUMENT;
    if (a->dtype != KDA_DTYPE_F32 && a->dtype != KDA_DTYPE_BF16) return KDA_ERR_INVALID_ARGUMENT;
    if (a->N < 0 || a->H < 1 || a->Dk < 1 || a->Dv < 1) return KDA_ERR_INVALID_ARGUMENT;
    if (!head_dim_ok(a->Dk) || !head_dim_ok(a->Dv)) return KDA_ERR_UNSUPPORTED;
    if (a->has_lower_bound && !(a->lower_bound < 0.f)) return KDA_ERR_INVALID_ARGUMENT;
    if (check_gate_mode(a->gate_mode, a->has_lower_bound) != KDA_OK) return KDA_ERR_INVALID_ARGUMENT;
    if ((long long)a->N * a->H * 4 >= 0x7fffffffLL) return KDA_ERR_INVALID_ARGUMENT;
    if (a->N == 0) return KDA_OK;
    const bool bf16 = a->dtype == KDA_DTYPE_BF16;
    const size_t esz = bf16 ? 2 : 4;
    if (!a->q || !a->k || !a->v || !a->g || !a->beta || !a->state || !a->o)
        return KDA_ERR_INVALID_ARGUMENT;
    if (!aligned(a->q, 16) || !aligned(a->k, 16) || !aligned(a->v, 16) || !aligned(a->g, 16) ||
        !aligned(a->o, 16) || !aligned(a->state, 16) || !aligned(a->beta, esz))
        return KDA_ERR_INVALID_ARGUMENT;
    if (check_gate_ptrs(a->gate_mode, a->A_log, a->dt_bias) != KDA_OK) return KDA_ERR_INVALID_ARGUMENT;
    if (!state_out_ok(a->state, a->state_out, a->N, a->H, a->Dk, a->Dv)) return KDA_ERR_INVALID_ARGUMENT;
    kda::StepParams p;
    p.q = a->q; p.k = a->k; p.v = a->v; p.g = a->g; p.beta = a->beta;
    p.state = a->state; p.o = a->o; p.N = a->N; p.H = a->H;
    p.scale = resolve_scale(a->scale, a->Dk);
    p.use_l2 = a->use_qk_l2norm ? 1 : 0;
    p.has_lb = a->has_lower_bound ? 1 : 0;
    p.lb = a->lower_bound;
    p.gate_mode = a->gate_mode;
    p.A_log = a->A_log;
    p.dt_bias = a->dt_bias;
    p.beta_prob = a->beta_is_prob ? 1 : 0;
    return cuda_status(kda::launch_decode(p, a->state_out, bf16, a->Dk, a->Dv, static_cast<cudaStream_t>(stream)));
}

kda_status kda_decode_token(const kda_token_args *a, void *stream) {
    if (!a) return KDA_ERR_INVALID_ARGUMENT;
    if (a->dtype != KDA_DTYPE_F32 && a->dtype != KDA_DTYPE_BF16) return KDA_ERR_INVALID_ARGUMENT;
    if (a->N < 0 || a->H < 1 || a->Dk < 1 || a->Dv < 1) return KDA_ERR_INVALID_ARGUMENT;
    if (!head_dim_ok(a->Dk) || !head_dim_ok(a->Dv)) return KDA_ERR_UNSUPPORTED;
    if (!kda::token_conv_supported(a->conv_kernel)) return KDA_ERR_UNSUPPORTED;
    if (a->has_lower_bound && !(a->lower_bound < 0.f)) return KDA_ERR_INVALID_ARGUMENT;
    if (check_gate_mode(a->gate_mode, a->has_lower_bound) != KDA_OK) return KDA_ERR_INVALID_ARGUMENT;
    if (!(a->norm_eps >= 0.f)) return KDA_ERR_INVALID_ARGUMENT;
    if ((long long)a->N * a->H * 4 >= 0x7fffffffLL) return KDA_ERR_INVALID_ARGUMENT;
    if (a->N == 0) return KDA_OK;
    const bool bf16 = a->dtype == KDA_DTYPE_BF16;
    const size_t esz = bf16 ? 2 : 4;
    if (!a->x || !a->conv_w || !a->conv_state || !a->g || !a->beta || !a->state || !a->o)
        return KDA_ERR_INVALID_ARGUMENT;
    if (!aligned(a->x, esz) || !aligned(a->g, esz) || !aligned(a->beta, esz) || !aligned(a->o, esz) ||
        (a->g_out && !aligned(a->g_out, esz)) || !aligned(a->conv_w, 4) || !aligned(a->conv_state, 4) ||
        !aligned(a->state, 16))
        return KDA_ERR_INVALID_ARGUMENT;
    if (check_gate_ptrs(a->gate_mode, a->A_log, a->dt_bias) != KDA_OK) return KDA_ERR_INVALID_ARGUMENT;
    if (!state_out_ok(a->state, a->state_out, a->N, a->H, a->Dk, a->Dv)) return KDA_ERR_INVALID_ARGUMENT;
    kda::TokenParams tp;
    kda::StepParams &p = tp.step;
    p.q = p.k = p.v = nullptr;
    p.g = a->g; p.beta = a->beta;
    p.state = a->state; p.o = a->o; p.N = a->N; p.H = a->H;
    p.scale = resolve_scale(a->scale, a->Dk);
    p.use_l2 = a->use_qk_l2norm ? 1 : 0;
    p.has_lb = a->has_lower_bound ? 1 : 0;
    p.lb = a->lower_bound;
    p.gate_mode = a->gate_mode;
    p.A_log = a->A_log;
    p.dt_bias = a->dt_bias;
    p.beta_prob = a->beta_is_prob ? 1 : 0;
    tp.x = a->x;
    tp.conv_w = a->conv_w;
    tp.conv_state = a->conv_state;
    tp.K = a->conv_kernel;
    tp.g_out = a->g_out;
    tp.norm_eps = a->norm_eps;
    return cuda_status(kda::launch_token(tp, a->state_out, bf16, a->Dk, a->Dv, static_cast<cudaStream_t>(stream)));
}

namespace {
kda::BwdParams bwd_params(const kda_chunk_bwd_args *a, int N) {
    kda::BwdParams p{};
    p.q = a->q; p.k = a->k; p.v = a->v; p.g = a->g; p.beta = a->beta; p.dout = a->dout;
    p.S0 = a->initial_state; p.dSf = a->dfinal_state;
    p.dq = a->dq; p.dk = a->dk; p.dv = a->dv; p.dg = a->dg; p.dbeta = a->dbeta; p.dS0 = a->dinitial_state;
    p.cu_seqlens = a->cu_seqlens; p.T = a->T; p.N = N; p.H = a->H;
    p.scale = resolve_scale(a->scale, a->Dk);
    p.use_l2 = a->use_qk_l2norm ? 1 : 0;
    p.has_lb = a->has_lower_bound ? 1 : 0;
    p.lb = a->lower_bound;
    p.beta_prob = a->beta_is_prob ? 1 : 0;
    return p;
}
}  // namespace

kda_status kda_chunk_bwd_workspace_size(const kda_chunk_bwd_args *a, size_t *bytes) {
    if (!a || !bytes) return KDA_ERR_INVALID_ARGUMENT;
    const kda_chunk_args f = fwd_view(a);
    int N = 0;
    kda_status s = check_chunk_shape(&f, &N);
    if (s != KDA_OK) return s;
    *bytes = kda::bwd_workspace_bytes(bwd_params(a, N), a->dtype == KDA_DTYPE_BF16, a->Dk, a->Dv);
    return KDA_OK;
}

kda_status kda_chunk_bwd(const kda_chunk_bwd_args *a, void *stream) {
    if (!a) return KDA_ERR_INVALID_ARGUMENT;
    const kda_chunk_args f = fwd_view(a);
    int N = 0;
    kda_status s = check_chunk_shape(&f, &N);
    if (s != KDA_OK) return s;
    const bool bf16 = a->dtype == KDA_DTYPE_BF16;
    const size_t esz = bf16 ? 2 : 4;
    const long long ntok = (long long)a->B * a->T;
    if (ntok > 0) {
        const void *rows[] = {a->q, a->k, a->v, a->g, a->dout, a->dq, a->dk, a->dv, a->dg};
        for (const void *ptr : rows)
            if (!ptr || !aligned(ptr, 16)) return KDA_ERR_INVALID_ARGUMENT;
        if (!a->beta || !aligned(a->beta, esz) || !a->dbeta || !aligned(a->dbeta, esz)) return KDA_ERR_INVALID_ARGUMENT;
    }
    if ((a->initial_state && !aligned(a->initial_state, 16)) || (a->dfinal_state && !aligned(a->dfinal_state, 16)) ||
        (a->dinitial_state && !aligned(a->dinitial_state, 16)))
        return KDA_ERR_INVALID_ARGUMENT;
    if (a->cu_seqlens_host) {
        const int32_t *cu = a->cu_seqlens_host;
        if (cu[0] != 0 || cu[N] != a->T) return KDA_ERR_INVALID_ARGUMENT;
        for (int n = 0; n < N; ++n)
            if (cu[n + 1] < cu[n]) return KDA_ERR_INVALID_ARGUMENT;
    }
    if (!a->cu_seqlens && a->cu_seqlens_host) return KDA_ERR_INVALID_ARGUMENT;
    const size_t need_ws = kda::bwd_workspace_bytes_min(a->cu_seqlens != nullptr, a->T, N, a->H, a->Dk, a->Dv);
    if (!a->workspace || a->workspace_bytes < need_ws || !aligned(a->workspace, 16)) return KDA_ERR_WORKSPACE;
    const kda::BwdParams p = bwd_params(a, N);
    return cuda_status(
        kda::launch_bwd(p, bf16, a->Dk, a->Dv, a->workspace, a->workspace_bytes, static_cast<cudaStream_t>(stream)));
}

}  // extern "C"
