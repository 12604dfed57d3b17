// kda_chunk_fwd_noalloc: chunked prefill for callers that cannot allocate.
//
// Some callers have no way to hand the library a workspace: a plugin hosted by
// a runtime that owns all device memory and exposes no allocator to it, or a
// latency-critical serving loop that must not call cudaMalloc (which can
// synchronise the whole device) in the middle of a step.  This entry point runs
// exactly the kernels of kda_chunk_fwd, but takes its scratch from a file-scope
// device array instead of a caller workspace.
//
// The array is kNoAllocScratchBytes per GPU, reserved on every device that
// loads this library and held until the process exits.  Host code cannot pass
// the array's name to a kernel (on the host it is only a stand-in, not a device
// address), so each call looks the device address up with cudaGetSymbolAddress
// on the current device.  Once the library's device code is loaded on a device
// that is a host-side table lookup; the first call on a device loads it, so
// that first call should come before any stream capture.  Looking the address
// up on every call (rather than caching it) keeps it right after a device
// reset, which can move the array.  Nothing here calls cudaMalloc, cudaFree or
// any allocating library routine.
//
// All calls share the one array: two calls whose kernels overlap on the GPU
// (different streams, no ordering between them) race on it and corrupt each
// other's results.  Calls on one stream, or otherwise ordered, are safe.  The
// array keeps the last call's contents; the chunk path writes every scratch
// word it reads (segment table, segment states) before reading it, so nothing
// needs clearing between calls.
#include "kda_common.cuh"

namespace kda {

constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;  // 64 MiB per device

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

size_t chunk_workspace_bytes(int B, int T, int H, int num_seqs, int dtype, int l2norm);
size_t chunk_workspace_bytes_min(int B, int T, int H, int num_seqs, int dtype, int l2norm);

// Device address of g_noalloc_scratch on the current device.
static void* noalloc_scratch(const char** why) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
        *why = e != cudaSuccess ? cudaGetErrorString(e) : "no device address for the static scratch array";
        return nullptr;
    }
    return p;
}

}  // namespace kda

extern "C" int kda_chunk_fwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
                             const float* initial_state, float* final_state, void* o, const int32_t* cu_seqlens,
                             int num_seqs, int B, int T, int H, int dtype, float scale, int l2norm_qk,
                             void* workspace, size_t workspace_bytes, void* stream);

extern "C" int kda_chunk_fwd_noalloc(const void* q, const void* k, const void* v, const float* g, const float* beta,
                                     const float* initial_state, float* final_state, void* o,
                                     const int32_t* cu_seqlens, int num_seqs, int B, int T, int H, int dtype,
                                     float scale, int l2norm_qk, void* stream) {
    using namespace kda;
    if (B < 0 || T < 0 || H < 0 || num_seqs < 0)
        return kda_chunk_fwd(q, k, v, g, beta, initial_state, final_state, o, cu_seqlens, num_seqs, B, T, H, dtype,
                             scale, l2norm_qk, nullptr, 0, stream);  // reports the bad size
    // the full workspace if it fits (the fastest schedule), else the smallest accepted one
    const int ns = cu_seqlens ? num_seqs : 0;
    size_t need = chunk_workspace_bytes(B, T, H, ns, dtype, l2norm_qk);
    if (need > kNoAllocScratchBytes) need = chunk_workspace_bytes_min(B, T, H, ns, dtype, l2norm_qk);
    if (need > kNoAllocScratchBytes) {
        snprintf(t_last_error, sizeof(t_last_error),
                 "kda_chunk_fwd_noalloc: this call needs %zu bytes of scratch, more than the %zu-byte static "
                 "array; use kda_chunk_fwd with a workspace",
                 need, kNoAllocScratchBytes);
        return KDA_ERR_UNSUPPORTED;
    }
    const char* why = "";
    void* scratch = noalloc_scratch(&why);
    if (!scratch) {
        snprintf(t_last_error, sizeof(t_last_error), "kda_chunk_fwd_noalloc: %s", why);
        return KDA_ERR_CUDA;
    }
    return kda_chunk_fwd(q, k, v, g, beta, initial_state, final_state, o, cu_seqlens, num_seqs, B, T, H, dtype,
                         scale, l2norm_qk, scratch, need, stream);
}
