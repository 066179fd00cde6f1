// kda_chunk_fwd_noalloc: the chunkwise forward for callers that cannot allocate
// device memory.
//
// Some callers run under a fixed device-memory plan and may not allocate once
// they are running: an inference engine that reserves all of its memory at start-
// up, a plug-in whose host application owns every device buffer, or a C host
// that has no allocator handle at the call site. kda_chunk_fwd asks such callers
// for a workspace they have no way to obtain. This entry point instead uses a
// small scratch array that lives in the library's own device memory (a
// file-scope __device__ array, created when the library is loaded on a device
// and held until the process exits). Inputs and outputs are still the caller's.
//
// The array's name, seen from host code, is only a host-side stand-in and not a
// device address; its device address is looked up with cudaGetSymbolAddress (with
// the caller's device current) on every call -- a host-side lookup, cheap once the
// library's device code is loaded, and never stale after a device reset reloads
// it -- and that address is what the kernels receive.

#include "../../include/kda.h"
#include "kda_common.cuh"

// Scratch of the no-allocation entry point: the tensor-core chunk kernel keeps
// its device status word here (it needs 256 bytes whatever the problem size).
static constexpr size_t kScratchBytes = 4096;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

namespace kda {
void record_cuda_error(int e);  // kda_api.cu: value returned by kda_last_cuda_error()
// kda_api.cu: the smallest workspace kda_chunk_fwd accepts for these arguments
kda_status chunk_workspace_min_bytes(const kda_chunk_args *a, size_t *bytes);
// kda_api.cu: the status word at a device address, after the stream drains
kda_status read_status_word(const void *word, cudaStream_t st);
}  // namespace kda

namespace {
// Device address of the scratch array on the current device.
kda_status scratch_address(void **out) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) {
        kda::record_cuda_error((int)e);
        return KDA_ERR_CUDA;
    }
    *out = p;
    return KDA_OK;
}
}  // namespace

extern "C" {

KDA_API kda_status kda_chunk_fwd_noalloc(const kda_chunk_args *args, void *stream) {
    if (!args) return KDA_ERR_INVALID_ARGUMENT;
    size_t need = 0;
    // the smallest workspace the forward accepts: with it, kda_chunk_fwd runs the
    // single-pass kernel, which keeps only a status word in scratch
    kda_status s = kda::chunk_workspace_min_bytes(args, &need);
    if (s != KDA_OK) return s;
    if (need > kScratchBytes) return KDA_ERR_WORKSPACE;  // beyond the fixed scratch size

    void *scratch = nullptr;
    if (need) {
        s = scratch_address(&scratch);
        if (s != KDA_OK) return s;
    }
    kda_chunk_args a = *args;
    a.workspace = need ? scratch : nullptr;
    a.workspace_bytes = need ? kScratchBytes : 0;
    return kda_chunk_fwd(&a, stream);
}

KDA_API kda_status kda_chunk_fwd_noalloc_status(const kda_chunk_args *args, void *stream) {
    if (!args) return KDA_ERR_INVALID_ARGUMENT;
    size_t need = 0;
    kda_status s = kda::chunk_workspace_min_bytes(args, &need);
    if (s != KDA_OK) return s;
    if (need == 0) return KDA_OK;  // that call ran a kernel without device waits
    void *scratch = nullptr;
    s = scratch_address(&scratch);
    if (s != KDA_OK) return s;
    return kda::read_status_word(scratch, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
