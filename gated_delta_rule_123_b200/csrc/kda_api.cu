// extern "C" entry points of libkda: host-side argument validation, then
// launches on the caller's stream.  Declared and documented in include/kda.h.
#include <stdio.h>
#include <string.h>

#include "kda_gemm.cuh"

namespace kda {

size_t dplr_workspace_bytes(int B, int T, int H, int num_seqs, int dtype);
int launch_dplr_chunk_fwd(const void* q, const void* k, const void* v, const void* a, const void* b, const float* g,
                          const float* beta, const float* init, float* fin, void* o, const int32_t* cu, int num_seqs,
                          int B, int T, int H, int dtype, float scale, void* ws, size_t ws_bytes, cudaStream_t stream,
                          const char** why);
size_t recurrent_bwd_workspace_bytes(int B, int T, int H);
int launch_recurrent_bwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
                         const float* init, const void* dout, const float* dfinal, float* dq, float* dk, float* dv,
                         float* dg, float* dbeta, float* dinit, int B, int Tn, int H, int dtype, float scale,
                         void* ws, size_t ws_bytes, cudaStream_t stream, const char** why);
int chunk_segment_tokens(int B, int T, int H, int num_seqs, int* middle);
int chunk_plan_items(const void* ws, int B, int T, int H, int num_seqs, int* rows, int max_rows);
size_t chunk_workspace_bytes_min(int B, int T, int H, int num_seqs, int dtype, int l2norm);
int launch_recurrent_fwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
                         float* state, void* o, int B, int Tn, int H, int dtype, float scale, int l2norm,
                         cudaStream_t stream, int out_f32);
int launch_decode_step(const void* q, const void* k, const void* v, const float* g, const float* beta,
                       float* state, void* o, int B, int H, int dtype, float scale, int l2norm, cudaStream_t stream);
int launch_chunk_fwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
                     const float* init, float* fin, void* o, const int32_t* cu, int num_seqs, int B, int T, int H,
                     int dtype, float scale, int l2norm, void* ws, size_t ws_bytes, cudaStream_t stream,
                     const char** why, int scalar_gate, int out_f32);
size_t chunk_workspace_bytes(int B, int T, int H, int num_seqs, int dtype, int l2norm);
size_t layer_workspace_bytes(int total_tokens, int d_model, int H, int rank, int num_seqs);
int launch_layer_fwd(const void* x, const kda_layer_weights* w, const int32_t* cu, int nseq, int ntok,
                     const float* init, float* fin, const void* conv_in, void* conv_out, void* y, void* ws,
                     size_t ws_bytes, cudaStream_t stream, const char** why);
size_t layer_decode_workspace_bytes(int B, int T, int d_model, int H, int rank);
int launch_layer_decode(const void* x, const kda_layer_weights* w, void* conv_state, float* state, void* y, int B,
                        int T, void* ws, size_t ws_bytes, cudaStream_t stream, const char** why);

static thread_local char t_last_error[256] = "";
thread_local cudaEvent_t* g_trace_events = nullptr;

static int fail(int code, const char* msg) {
    snprintf(t_last_error, sizeof(t_last_error), "%s", msg ? msg : "");
    return code;
}
static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace kda

using namespace kda;

extern "C" {

const char* kda_status_string(int s) {
    switch (s) {
        case KDA_OK: return "KDA_OK";
        case KDA_ERR_INVALID_ARG: return "KDA_ERR_INVALID_ARG";
        case KDA_ERR_UNSUPPORTED: return "KDA_ERR_UNSUPPORTED";
        case KDA_ERR_WORKSPACE: return "KDA_ERR_WORKSPACE";
        case KDA_ERR_CUDA: return "KDA_ERR_CUDA";
        case KDA_ERR_TIMEOUT: return "KDA_ERR_TIMEOUT";
        default: return "KDA_ERR_UNKNOWN";
    }
}

int kda_head_dim(void) { return kD; }

const char* kda_last_error(void) { return t_last_error; }

int kda_set_trace_events(void* events, int n_events) {
    if (events && n_events < 5) return fail(KDA_ERR_INVALID_ARG, "need 5 events");
    g_trace_events = static_cast<cudaEvent_t*>(events);
    return KDA_OK;
}

int kda_device_status(void* stream) {
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int val = 0;
    const int zero = 0;
    if (cudaMemcpyFromSymbolAsync(&val, g_device_status, sizeof(int), 0, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return fail(KDA_ERR_CUDA, cudaGetErrorString(cudaGetLastError()));
    if (val != 0) {
        cudaMemcpyToSymbolAsync(g_device_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice, s);
        cudaStreamSynchronize(s);
        char msg[64];
        snprintf(msg, sizeof(msg), "device wait gave up (site mask 0x%x)", val);
        return fail(KDA_ERR_TIMEOUT, msg);
    }
    return KDA_OK;
}

int kda_debug_fault_injection(long long wait_limit_cycles, int skip_chunk) {
    t_last_error[0] = 0;
    const long long lim = wait_limit_cycles > 0 ? wait_limit_cycles : (1ll << 31);
    const int skip = skip_chunk >= 0 ? skip_chunk : -1;
    cudaError_t e = cudaMemcpyToSymbol(c_wait_limit, &lim, sizeof(lim));
    if (e == cudaSuccess) e = cudaMemcpyToSymbol(c_skip_chunk_load, &skip, sizeof(skip));
    return e == cudaSuccess ? KDA_OK : fail(KDA_ERR_CUDA, cudaGetErrorString(e));
}

int kda_chunk_fwd_segment_tokens(int B, int T, int H, int num_seqs, int* middle_tokens) {
    if (middle_tokens) *middle_tokens = 0;
    if (B < 0 || T < 0 || H < 0 || num_seqs < 0) return 0;
    return chunk_segment_tokens(B, T, H, num_seqs, middle_tokens);
}

int kda_chunk_fwd_plan_items(const void* workspace, int B, int T, int H, int num_seqs, int* rows, int max_rows) {
    if (!workspace || !rows || max_rows < 0 || B < 0 || T < 0 || H < 0 || num_seqs < 0) return -1;
    if (cudaDeviceSynchronize() != cudaSuccess) return -1;  // the call may have run on any stream
    return chunk_plan_items(workspace, B, T, H, num_seqs, rows, max_rows);
}

size_t kda_chunk_fwd_workspace_min(int B, int T, int H, int num_seqs, int dtype, int l2norm_qk) {
    if (B < 0 || T < 0 || H < 0 || num_seqs < 0) return 0;
    return chunk_workspace_bytes_min(B, T, H, num_seqs, dtype, l2norm_qk);
}

size_t kda_chunk_fwd_workspace(int B, int T, int H, int num_seqs, int dtype, int l2norm_qk) {
    if (B < 0 || T < 0 || H < 0 || num_seqs < 0) return 0;
    return chunk_workspace_bytes(B, T, H, num_seqs, dtype, l2norm_qk);
}

// Shared body of kda_chunk_fwd (per-channel g, [.., H, 128]) and kda_gdn_chunk_fwd
// (one g per token and head, [.., H]).
static int chunk_fwd_impl(const void* q, const void* k, const void* v, const float* g, const float* beta,
                          const float* initial_state, float* final_state, void* o, const int32_t* cu_seqlens,
                          int num_seqs, int B, int T, int H, int dtype, float scale, int l2norm_qk, void* workspace,
                          size_t workspace_bytes, void* stream, int scalar_gate) {
    t_last_error[0] = 0;
    if (dtype != KDA_BF16 && dtype != KDA_FP32) return fail(KDA_ERR_INVALID_ARG, "dtype must be KDA_BF16 or KDA_FP32");
    if (B < 0 || T < 0 || H < 0) return fail(KDA_ERR_INVALID_ARG, "negative size");
    if (cu_seqlens) {
        if (B != 1) return fail(KDA_ERR_INVALID_ARG, "cu_seqlens requires B == 1");
        if (num_seqs < 1) return fail(KDA_ERR_INVALID_ARG, "cu_seqlens requires num_seqs >= 1");
    } else if (num_seqs != 0) {
        return fail(KDA_ERR_INVALID_ARG, "num_seqs must be 0 for dense input");
    }
    const long long N = cu_seqlens ? num_seqs : B;
    if ((long long)(cu_seqlens ? 1 : B) * T * H * kD >= (1ll << 31))
        return fail(KDA_ERR_UNSUPPORTED, "more than 2^31 elements per token tensor");
    if ((long long)T * H * kD == 0 || N == 0 || H == 0) {
        // nothing to compute except the state pass-through
        if (final_state && N * H > 0) {
            const size_t bytes = size_t(N) * H * kD * kD * sizeof(float);
            cudaError_t e = initial_state
                                ? (initial_state == final_state
                                       ? cudaSuccess
                                       : cudaMemcpyAsync(final_state, initial_state, bytes, cudaMemcpyDeviceToDevice,
                                                         static_cast<cudaStream_t>(stream)))
                                : cudaMemsetAsync(final_state, 0, bytes, static_cast<cudaStream_t>(stream));
            if (e != cudaSuccess) return fail(KDA_ERR_CUDA, cudaGetErrorString(e));
        }
        return KDA_OK;
    }
    if (!q || !k || !v || !g || !beta || !o) return fail(KDA_ERR_INVALID_ARG, "NULL tensor pointer");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(g) || !aligned16(o) ||
        (initial_state && !aligned16(initial_state)) || (final_state && !aligned16(final_state)))
        return fail(KDA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
    if (o == q || o == k || o == v) return fail(KDA_ERR_INVALID_ARG, "o must not alias q, k or v");
    if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return fail(KDA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    const char* why = "";
    const int rc = launch_chunk_fwd(q, k, v, g, beta, initial_state, final_state, o, cu_seqlens, num_seqs, B, T, H,
                                    dtype, scale, l2norm_qk, workspace, workspace_bytes,
                                    static_cast<cudaStream_t>(stream), &why, scalar_gate, 0);
    return rc == KDA_OK ? KDA_OK : fail(rc, why);
}

int kda_chunk_fwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
                  const float* initial_state, float* final_state, void* o, const int32_t* cu_seqlens, int num_seqs,
                  int B, int T, int H, int dtype, float scale, int l2norm_qk, void* workspace,
                  size_t workspace_bytes, void* stream) {
    return chunk_fwd_impl(q, k, v, g, beta, initial_state, final_state, o, cu_seqlens, num_seqs, B, T, H, dtype,
                          scale, l2norm_qk, workspace, workspace_bytes, stream, 0);
}

int kda_gdn_chunk_fwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
                      const float* initial_state, float* final_state, void* o, const int32_t* cu_seqlens,
                      int num_seqs, int B, int T, int H, int dtype, float scale, int l2norm_qk, void* workspace,
                      size_t workspace_bytes, void* stream) {
    return chunk_fwd_impl(q, k, v, g, beta, initial_state, final_state, o, cu_seqlens, num_seqs, B, T, H, dtype,
                          scale, l2norm_qk, workspace, workspace_bytes, stream, 1);
}

int kda_decode_step(const void* q, const void* k, const void* v, const float* g, const float* beta, float* state,
                    void* o, int B, int H, int dtype, float scale, int l2norm_qk, void* stream) {
    t_last_error[0] = 0;
    if (dtype != KDA_BF16 && dtype != KDA_FP32) return fail(KDA_ERR_INVALID_ARG, "dtype must be KDA_BF16 or KDA_FP32");
    if (B < 0 || H < 0) return fail(KDA_ERR_INVALID_ARG, "negative size");
    if ((long long)B * H == 0) return KDA_OK;
    if ((long long)B * H >= (1ll << 31)) return fail(KDA_ERR_UNSUPPORTED, "too many heads");
    if (!q || !k || !v || !g || !beta || !state || !o) return fail(KDA_ERR_INVALID_ARG, "NULL tensor pointer");
    if (!aligned16(state) || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(g) || !aligned16(o))
        return fail(KDA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
    const int rc = launch_decode_step(q, k, v, g, beta, state, o, B, H, dtype, scale, l2norm_qk,
                                      static_cast<cudaStream_t>(stream));
    return rc == KDA_OK ? KDA_OK : fail(rc, cudaGetErrorString(cudaGetLastError()));
}

size_t kda_recurrent_bwd_workspace(int B, int T, int H) {
    if (B < 0 || T < 0 || H < 0) return 0;
    return recurrent_bwd_workspace_bytes(B, T, H);
}

int kda_recurrent_bwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
                      const float* initial_state, const void* d_o, const float* d_final_state, float* dq, float* dk,
                      float* dv, float* dg, float* dbeta, float* d_initial_state, int B, int T, int H, int dtype,
                      float scale, void* workspace, size_t workspace_bytes, void* stream) {
    t_last_error[0] = 0;
    if (dtype != KDA_BF16 && dtype != KDA_FP32) return fail(KDA_ERR_INVALID_ARG, "dtype must be KDA_BF16 or KDA_FP32");
    if (B < 0 || T < 0 || H < 0) return fail(KDA_ERR_INVALID_ARG, "negative size");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if ((long long)B * H == 0) return KDA_OK;
    if ((long long)B * H >= (1ll << 31) || (long long)B * T * H * kD >= (1ll << 40))
        return fail(KDA_ERR_UNSUPPORTED, "too many heads or tokens");
    if (T == 0) {  // the initial-state gradient is the final-state gradient
        if (d_initial_state) {
            const size_t bytes = size_t(B) * H * kD * kD * sizeof(float);
            const cudaError_t e = d_final_state ? cudaMemcpyAsync(d_initial_state, d_final_state, bytes,
                                                                  cudaMemcpyDeviceToDevice, s)
                                                : cudaMemsetAsync(d_initial_state, 0, bytes, s);
            if (e != cudaSuccess) return fail(KDA_ERR_CUDA, cudaGetErrorString(e));
        }
        return KDA_OK;
    }
    if (!q || !k || !v || !g || !beta || !d_o || !dq || !dk || !dv || !dg || !dbeta)
        return fail(KDA_ERR_INVALID_ARG, "NULL tensor pointer");
    const void* p16[] = {q, k, v, g, d_o, dq, dk, dv, dg, initial_state, d_final_state, d_initial_state};
    for (const void* ptr : p16)
        if (ptr && !aligned16(ptr)) return fail(KDA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
    if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return fail(KDA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    const char* why = "";
    const int rc = launch_recurrent_bwd(q, k, v, g, beta, initial_state, d_o, d_final_state, dq, dk, dv, dg, dbeta,
                                        d_initial_state, B, T, H, dtype, scale, workspace, workspace_bytes, s, &why);
    return rc == KDA_OK ? KDA_OK : fail(rc, why);
}

size_t kda_dplr_chunk_fwd_workspace(int B, int T, int H, int num_seqs, int dtype) {
    if (B < 0 || T < 0 || H < 0 || num_seqs < 0) return 0;
    return dplr_workspace_bytes(B, T, H, num_seqs, dtype);
}

int kda_dplr_chunk_fwd(const void* q, const void* k, const void* v, const void* a, const void* b, const float* g,
                       const float* beta, const float* initial_state, float* final_state, void* o,
                       const int32_t* cu_seqlens, int num_seqs, int B, int T, int H, int dtype, float scale,
                       void* workspace, size_t workspace_bytes, void* stream) {
    t_last_error[0] = 0;
    if (dtype != KDA_BF16 && dtype != KDA_FP32) return fail(KDA_ERR_INVALID_ARG, "dtype must be KDA_BF16 or KDA_FP32");
    if (B < 0 || T < 0 || H < 0) return fail(KDA_ERR_INVALID_ARG, "negative size");
    if (cu_seqlens) {
        if (B != 1) return fail(KDA_ERR_INVALID_ARG, "cu_seqlens requires B == 1");
        if (num_seqs < 1) return fail(KDA_ERR_INVALID_ARG, "cu_seqlens requires num_seqs >= 1");
    } else if (num_seqs != 0) {
        return fail(KDA_ERR_INVALID_ARG, "num_seqs must be 0 for dense input");
    }
    const long long N = cu_seqlens ? num_seqs : B;
    if ((long long)(cu_seqlens ? 1 : B) * T * H * kD >= (1ll << 31))
        return fail(KDA_ERR_UNSUPPORTED, "more than 2^31 elements per token tensor");
    if (N > 65535 || H > 65535) return fail(KDA_ERR_UNSUPPORTED, "more than 65535 sequences or heads");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if ((long long)T * H == 0 || N == 0) {
        if (final_state && N * H > 0) {
            const size_t bytes = size_t(N) * H * kD * kD * sizeof(float);
            cudaError_t e = initial_state ? (initial_state == final_state
                                                 ? cudaSuccess
                                                 : cudaMemcpyAsync(final_state, initial_state, bytes,
                                                                   cudaMemcpyDeviceToDevice, s))
                                          : cudaMemsetAsync(final_state, 0, bytes, s);
            if (e != cudaSuccess) return fail(KDA_ERR_CUDA, cudaGetErrorString(e));
        }
        return KDA_OK;
    }
    if (!q || !k || !v || !a || !b || !g || !beta || !o) return fail(KDA_ERR_INVALID_ARG, "NULL tensor pointer");
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(a) || !aligned16(b) || !aligned16(g) ||
        !aligned16(o) || (initial_state && !aligned16(initial_state)) || (final_state && !aligned16(final_state)))
        return fail(KDA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
    if (o == q || o == k || o == v || o == a || o == b) return fail(KDA_ERR_INVALID_ARG, "o must not alias an input");
    if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return fail(KDA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    const char* why = "";
    const int rc = launch_dplr_chunk_fwd(q, k, v, a, b, g, beta, initial_state, final_state, o, cu_seqlens, num_seqs,
                                         B, T, H, dtype, scale, workspace, workspace_bytes, s, &why);
    return rc == KDA_OK ? KDA_OK : fail(rc, why);
}

int kda_recurrent_fwd(const void* q, const void* k, const void* v, const float* g, const float* beta, float* state,
                      void* o, int B, int T, int H, int dtype, float scale, int l2norm_qk, void* stream) {
    t_last_error[0] = 0;
    if (dtype != KDA_BF16 && dtype != KDA_FP32) return fail(KDA_ERR_INVALID_ARG, "dtype must be KDA_BF16 or KDA_FP32");
    if (B < 0 || T < 0 || H < 0) return fail(KDA_ERR_INVALID_ARG, "negative size");
    if ((long long)B * H == 0 || T == 0) return KDA_OK;
    if ((long long)B * H >= (1ll << 31) || (long long)B * T * H * kD >= (1ll << 40))
        return fail(KDA_ERR_UNSUPPORTED, "too many heads or tokens");
    if (!q || !k || !v || !g || !beta || !state || !o) return fail(KDA_ERR_INVALID_ARG, "NULL tensor pointer");
    if (!aligned16(state) || !aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(g) || !aligned16(o))
        return fail(KDA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
    if (o == q || o == k || o == v) return fail(KDA_ERR_INVALID_ARG, "o must not alias q, k or v");
    const int rc = launch_recurrent_fwd(q, k, v, g, beta, state, o, B, T, H, dtype, scale, l2norm_qk,
                                        static_cast<cudaStream_t>(stream), 0);
    return rc == KDA_OK ? KDA_OK : fail(rc, cudaGetErrorString(cudaGetLastError()));
}

int kda_linear_bf16(const void* x, int ldx, const void* W, int ldw, void* y, int ldy, int M, int N, int K,
                    void* stream) {
    t_last_error[0] = 0;
    if (M < 0 || N < 0 || K < 0) return fail(KDA_ERR_INVALID_ARG, "negative size");
    if ((long long)M * N == 0) return KDA_OK;
    if (K == 0) return fail(KDA_ERR_UNSUPPORTED, "K must be positive");
    if (!x || !W || !y) return fail(KDA_ERR_INVALID_ARG, "NULL tensor pointer");
    if (ldx < K || ldw < K || ldy < N) return fail(KDA_ERR_INVALID_ARG, "row stride smaller than the row");
    if (!aligned16(x) || !aligned16(W) || !aligned16(y) || ldx % 8 || ldw % 8 || ldy % 8)
        return fail(KDA_ERR_INVALID_ARG, "pointers and row strides must be 16-byte aligned");
    if (y == x || y == W) return fail(KDA_ERR_INVALID_ARG, "y must not alias x or W");
    const char* why = "";
    const int rc = launch_gemm(x, ldx, W, ldw, y, ldy, M, N, K, GemmEpilogue{}, static_cast<cudaStream_t>(stream),
                               &why);
    return rc == KDA_OK ? KDA_OK : fail(rc, why);
}

size_t kda_layer_fwd_workspace(int total_tokens, int d_model, int H, int rank, int num_seqs) {
    if (total_tokens < 0 || d_model <= 0 || H <= 0 || rank <= 0 || num_seqs < 1) return 0;
    return layer_workspace_bytes(total_tokens, d_model, H, rank, num_seqs);
}

// Weight checks shared by the layer entry points.
static int check_layer_weights(const kda_layer_weights* w) {
    if (!w) return fail(KDA_ERR_INVALID_ARG, "NULL weights");
    if (w->d_model <= 0 || w->H <= 0 || w->rank <= 0) return fail(KDA_ERR_INVALID_ARG, "bad sizes");
    if (w->d_model % 8 || w->rank % 8) return fail(KDA_ERR_UNSUPPORTED, "d_model and rank must be multiples of 8");
    if (!w->W_in || !w->W_aup || !w->W_gup || !w->conv_w || !w->norm_w || !w->W_o)
        return fail(KDA_ERR_INVALID_ARG, "NULL weight pointer");
    if (!aligned16(w->W_in) || !aligned16(w->W_aup) || !aligned16(w->W_gup) || !aligned16(w->W_o) ||
        !aligned16(w->conv_w))
        return fail(KDA_ERR_INVALID_ARG, "weight pointers must be 16-byte aligned");
    return KDA_OK;
}

int kda_layer_fwd(const void* x, const kda_layer_weights* w, const int32_t* cu_seqlens, int num_seqs,
                  int total_tokens, const float* initial_state, float* final_state, const void* conv_state_in,
                  void* conv_state_out, void* y, void* workspace, size_t workspace_bytes, void* stream) {
    t_last_error[0] = 0;
    const int wc = check_layer_weights(w);
    if (wc != KDA_OK) return wc;
    if (total_tokens < 0 || num_seqs < 1) return fail(KDA_ERR_INVALID_ARG, "bad sizes");
    if (!cu_seqlens) return fail(KDA_ERR_INVALID_ARG, "cu_seqlens is required");
    if ((initial_state && !aligned16(initial_state)) || (final_state && !aligned16(final_state)) ||
        (conv_state_in && !aligned16(conv_state_in)) || (conv_state_out && !aligned16(conv_state_out)))
        return fail(KDA_ERR_INVALID_ARG, "state pointers must be 16-byte aligned");
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (total_tokens == 0) {  // every sequence is empty: the states pass through
        const size_t sb = size_t(num_seqs) * w->H * kD * kD * sizeof(float);
        const size_t cb = size_t(num_seqs) * 3 * 3 * w->H * kD * 2;
        cudaError_t e = cudaSuccess;
        if (final_state && final_state != initial_state)
            e = initial_state ? cudaMemcpyAsync(final_state, initial_state, sb, cudaMemcpyDeviceToDevice, s)
                              : cudaMemsetAsync(final_state, 0, sb, s);
        if (e == cudaSuccess && conv_state_out && conv_state_out != conv_state_in)
            e = conv_state_in ? cudaMemcpyAsync(conv_state_out, conv_state_in, cb, cudaMemcpyDeviceToDevice, s)
                              : cudaMemsetAsync(conv_state_out, 0, cb, s);
        return e == cudaSuccess ? KDA_OK : fail(KDA_ERR_CUDA, cudaGetErrorString(e));
    }
    if (!x || !y) return fail(KDA_ERR_INVALID_ARG, "NULL tensor pointer");
    if (!aligned16(x) || !aligned16(y)) return fail(KDA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
    if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return fail(KDA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    const char* why = "";
    const int rc = launch_layer_fwd(x, w, cu_seqlens, num_seqs, total_tokens, initial_state, final_state,
                                    conv_state_in, conv_state_out, y, workspace, workspace_bytes, s, &why);
    return rc == KDA_OK ? KDA_OK : fail(rc, why);
}

size_t kda_layer_decode_workspace(int B, int T, int d_model, int H, int rank) {
    if (B <= 0 || T <= 0 || d_model <= 0 || H <= 0 || rank <= 0) return 0;
    return layer_decode_workspace_bytes(B, T, d_model, H, rank);
}

int kda_layer_decode(const void* x, const kda_layer_weights* w, void* conv_state, float* state, void* y, int B,
                     int T, void* workspace, size_t workspace_bytes, void* stream) {
    t_last_error[0] = 0;
    const int wc = check_layer_weights(w);
    if (wc != KDA_OK) return wc;
    if (B < 0 || T < 0) return fail(KDA_ERR_INVALID_ARG, "negative size");
    if ((long long)B * T == 0) return KDA_OK;
    if ((long long)B * T * (3 * w->H * kD + 2 * w->rank + w->H) >= (1ll << 31))
        return fail(KDA_ERR_UNSUPPORTED, "too many tokens");
    if (!x || !y || !conv_state || !state) return fail(KDA_ERR_INVALID_ARG, "NULL tensor pointer");
    if (!aligned16(x) || !aligned16(y) || !aligned16(conv_state) || !aligned16(state))
        return fail(KDA_ERR_INVALID_ARG, "tensor pointers must be 16-byte aligned");
    if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return fail(KDA_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
    const char* why = "";
    const int rc = launch_layer_decode(x, w, conv_state, state, y, B, T, workspace, workspace_bytes,
                                       static_cast<cudaStream_t>(stream), &why);
    return rc == KDA_OK ? KDA_OK : fail(rc, why);
}

}  // extern "C"
