// KDA layer forward around the chunk operator.
//
// "Kimi Linear: An Expressive, Efficient Attention Architecture", section
// "Neural Parameterization" (bias-free Q/K/V projections, depthwise ShortConv
// of kernel 4, SiLU, L2-normalised q and k, a rank-128 low-rank per-channel
// decay, a sigmoid beta per token and head, RMSNorm with a low-rank sigmoid
// output gate) and section "Code Verification" (three ShortConvolutions, b_proj
// followed by sigmoid, hidden -> 128 -> H*128 alpha gate, FusedRMSNormGated with
// a sigmoid activation).
//
// Pipeline (all on the caller's stream; every step is a kernel of this library):
//   z, beta = x W_in^T                  tcgen05 GEMM: z = [q|k|v|a_down|g_down|b] in bf16,
//                                        and beta = sigmoid(b) in fp32 from its epilogue
//   q,k,v = SiLU(conv4(z_qkv))          causal, restarts at each packed sequence;
//   q,k <- q,k / ||.||                  fused into the convolution kernel
//   g     = -softplus(a_down W_aup^T)   tcgen05 GEMM, fp32 from its epilogue
//   o     = KDA(q, k, v, g, beta)       the chunk kernels (varlen), o kept in fp32
//   on    = RMSNorm_head(o) * norm_w * sigmoid(g_down W_gup^T)
//                                        tcgen05 GEMM with the norm and gate in its epilogue
//   y     = on W_o^T                    tcgen05 GEMM
#include "kda_gemm.cuh"

namespace kda {

int launch_chunk_fwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
                     const float* init, float* fin, void* o, const int32_t* cu, int num_seqs, int B, int T, int H,
                     int dtype, float scale, int l2norm, void* ws, size_t ws_bytes, cudaStream_t stream,
                     const char** why, int scalar_gate, int out_f32);
size_t chunk_workspace_bytes(int B, int T, int H, int num_seqs, int dtype, int l2norm);
int launch_recurrent_fwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
                         float* state, void* o, int B, int Tn, int H, int dtype, float scale, int l2norm,
                         cudaStream_t stream, int out_f32);

// Sequence of token t: packed (cu[n] <= t < cu[n+1]), or dense with seq_len
// tokens per sequence when cu is NULL.
__device__ __forceinline__ int seq_of(const int32_t* cu, int nseq, int seq_len, int t) {
    if (!cu) return t / seq_len;
    int lo = 0, hi = nseq;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (cu[mid] <= t) lo = mid; else hi = mid;
    }
    return lo;
}
__device__ __forceinline__ int seq_begin(const int32_t* cu, int seq_len, int n) { return cu ? cu[n] : n * seq_len; }

// ShortConv + SiLU (+ L2 norm of q and k per head).  A CTA of 256 threads runs
// one tensor (blockIdx.y: q, k or v) over kConvTok consecutive tokens and 2048
// of its channels (blockIdx.z); thread i owns channels [8i, 8i + 8) of that
// block (its 4 taps stay in registers), and a head's 128 channels are one
// half-warp.  The last three inputs of each
// channel are kept in registers as the window slides over the tokens, so every
// projection row is read once; at a sequence start the window restarts from the
// cached history conv_in [nseq][3][3 H 128] (row 2 = the token just before) or
// from zero.  Loads and stores are 16 bytes, and all of a block's rows are
// requested before the first is used (the kernel is bound by memory latency
// otherwise).  Each block also re-reads the three rows before it: 12 tokens per
// block read 15/12 of the rows (8 tokens: 11/8) and still fit 128 registers
// (16 tokens spill).
constexpr int kConvTok = 12;

__device__ __forceinline__ void unpack8(const uint4& r, float* f) {
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&r);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        f[2 * u] = __low2float(p[u]);
        f[2 * u + 1] = __high2float(p[u]);
    }
}

__global__ void __launch_bounds__(256) conv_silu_norm_kernel(
    const __nv_bfloat16* __restrict__ z, int ldz, const __nv_bfloat16* __restrict__ conv_w,
    const int32_t* __restrict__ cu, int nseq, int seq_len, int ntok, int H, const __nv_bfloat16* __restrict__ conv_in,
    __nv_bfloat16* __restrict__ q, __nv_bfloat16* __restrict__ k, __nv_bfloat16* __restrict__ v) {
    const int HD = H * kD;
    const int which = blockIdx.y;
    const int c0 = (blockIdx.z * 256 + threadIdx.x) * 8;  // channel inside the tensor
    if (c0 >= HD) return;  // whole half-warps (heads) drop out together
    const unsigned hmask = 0xffffu << (threadIdx.x & 16);  // this half-warp
    const int col = which * HD + c0;  // column of z and of the conv taps
    const int t0 = blockIdx.x * kConvTok, t1 = min(ntok, t0 + kConvTok);
    float w[8][4];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
        const uint2 raw = *reinterpret_cast<const uint2*>(conv_w + (size_t)(col + u) * 4);
        const __nv_bfloat162* pr = reinterpret_cast<const __nv_bfloat162*>(&raw);
        w[u][0] = __low2float(pr[0]);
        w[u][1] = __high2float(pr[0]);
        w[u][2] = __low2float(pr[1]);
        w[u][3] = __high2float(pr[1]);
    }
    __nv_bfloat16* dst = which == 0 ? q : (which == 1 ? k : v);
    int n = seq_of(cu, nseq, seq_len, t0);
    int s_beg = seq_begin(cu, seq_len, n), s_end = seq_begin(cu, seq_len, n + 1);
    float hist[3][8];  // inputs at t-3, t-2, t-1
    auto load_hist = [&](int t) {  // window for token t, which starts at or after s_beg
#pragma unroll
        for (int j = 0; j < 3; ++j) {
            const int tt = t - 3 + j;
            if (tt >= s_beg) {
                unpack8(*reinterpret_cast<const uint4*>(z + (size_t)tt * ldz + col), hist[j]);
            } else if (conv_in) {
                unpack8(*reinterpret_cast<const uint4*>(conv_in + ((size_t)n * 3 + (3 + tt - s_beg)) * (3 * HD) + col),
                        hist[j]);
            } else {
#pragma unroll
                for (int u = 0; u < 8; ++u) hist[j][u] = 0.f;
            }
        }
    };
    uint4 rows[kConvTok];
#pragma unroll
    for (int j = 0; j < kConvTok; ++j)
        if (t0 + j < t1) rows[j] = *reinterpret_cast<const uint4*>(z + (size_t)(t0 + j) * ldz + col);
    load_hist(t0);
#pragma unroll
    for (int j = 0; j < kConvTok; ++j) {
        const int t = t0 + j;
        if (t >= t1) break;
        while (t >= s_end) {  // a new sequence starts at t (empty ones are skipped)
            ++n;
            s_beg = s_end;
            s_end = seq_begin(cu, seq_len, n + 1);
            load_hist(t);
        }
        float x[8];
        unpack8(rows[j], x);
        float acc[8], ss = 0.f;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            float a = w[u][0] * hist[0][u] + w[u][1] * hist[1][u] + w[u][2] * hist[2][u] + w[u][3] * x[u];
            a = __fdividef(a, 1.f + __expf(-a));  // SiLU
            acc[u] = a;
            ss += a * a;
            hist[0][u] = hist[1][u];
            hist[1][u] = hist[2][u];
            hist[2][u] = x[u];
        }
        if (which < 2) {  // L2 norm over the head's 128 channels = this half-warp
#pragma unroll
            for (int off = 8; off > 0; off >>= 1) ss += __shfl_xor_sync(hmask, ss, off);
            const float f = rsqrtf(ss + 1e-6f);
#pragma unroll
            for (int u = 0; u < 8; ++u) acc[u] *= f;
        }
        uint4 o;
        o.x = pack_bf16x2(acc[0], acc[1]);
        o.y = pack_bf16x2(acc[2], acc[3]);
        o.z = pack_bf16x2(acc[4], acc[5]);
        o.w = pack_bf16x2(acc[6], acc[7]);
        *reinterpret_cast<uint4*>(dst + (size_t)t * HD + c0) = o;
    }
}

// conv_out[n] = the last 3 conv inputs (q, k, v pre-activations) up to the end of
// sequence n, oldest first, taken from this call's tokens and, for a sequence
// shorter than 3, from the history conv_in (or zero).  One thread per (n,
// column) reads its three sources before writing, so conv_out may equal conv_in.
__global__ void conv_cache_out_kernel(const __nv_bfloat16* __restrict__ z, int ldz, const int32_t* __restrict__ cu,
                                      int nseq, int seq_len, int C, const __nv_bfloat16* conv_in,
                                      __nv_bfloat16* conv_out) {
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (long long)nseq * C) return;
    const int n = int(i / C), c = int(i % C);
    const int s0 = seq_begin(cu, seq_len, n), e0 = seq_begin(cu, seq_len, n + 1);
    __nv_bfloat16 r[3];
#pragma unroll
    for (int j = 0; j < 3; ++j) {
        const int p = e0 - 3 + j;
        r[j] = p >= s0 ? z[(size_t)p * ldz + c]
                       : (conv_in ? conv_in[((size_t)n * 3 + (3 + p - s0)) * C + c] : __float2bfloat16_rn(0.f));
    }
#pragma unroll
    for (int j = 0; j < 3; ++j) conv_out[((size_t)n * 3 + j) * C + c] = r[j];
}

struct LayerPlan {
    int HD, nz, ldz;  // ldz: row stride of z, padded to 8 elements so every row is 16-byte aligned
    size_t off_z, off_q, off_k, off_v, off_g, off_beta, off_o, off_chunk, chunk_bytes, total;
};

static size_t up256l(size_t x) { return (x + 255) & ~size_t(255); }

static LayerPlan make_layer_plan(int ntok, int d_model, int H, int rank, int nseq, bool chunked = true) {
    (void)d_model;
    LayerPlan p{};
    p.HD = H * kD;
    p.nz = 3 * p.HD + 2 * rank + H;
    p.ldz = (p.nz + 7) & ~7;
    size_t off = 0;
    const size_t tokHD = size_t(ntok) * p.HD;
    p.off_z = off; off = up256l(off + size_t(ntok) * p.ldz * 2);
    p.off_q = off; off = up256l(off + tokHD * 2);  // q, then the normed and gated output
    p.off_k = off; off = up256l(off + tokHD * 2);
    p.off_v = off; off = up256l(off + tokHD * 2);
    p.off_g = off; off = up256l(off + tokHD * 4);
    p.off_beta = off; off = up256l(off + size_t(ntok) * H * 4);
    p.off_o = off; off = up256l(off + tokHD * 4);  // the operator's output, fp32
    p.chunk_bytes = chunked ? chunk_workspace_bytes(1, ntok, H, nseq, KDA_BF16, 0) : 0;
    p.off_chunk = off; off = up256l(off + p.chunk_bytes);
    p.total = off;
    return p;
}

size_t layer_workspace_bytes(int ntok, int d_model, int H, int rank, int nseq) {
    return make_layer_plan(ntok, d_model, H, rank, nseq).total;
}
size_t layer_decode_workspace_bytes(int B, int T, int d_model, int H, int rank) {
    return make_layer_plan(B * T, d_model, H, rank, B, false).total;
}

// Shared by the prefill (cu = packed offsets, KDA by the chunk kernels) and the
// decode step (cu = NULL, B sequences of seq_len tokens, KDA by the fused
// recurrent kernel on the state in place).
static int layer_pipeline(const void* x, const kda_layer_weights* w, const int32_t* cu, int nseq, int seq_len,
                          int ntok, const float* init, float* fin, float* state_inplace, const void* conv_in,
                          void* conv_out, void* y, void* ws, size_t ws_bytes, cudaStream_t stream, const char** why) {
    const int H = w->H, D = w->d_model, R = w->rank;
    const bool decode = cu == nullptr;
    const LayerPlan pl = make_layer_plan(ntok, D, H, R, nseq, !decode);
    if (!ws || ws_bytes < pl.total) {
        *why = decode ? "workspace smaller than kda_layer_decode_workspace()"
                      : "workspace smaller than kda_layer_fwd_workspace()";
        return KDA_ERR_WORKSPACE;
    }
    uint8_t* b = static_cast<uint8_t*>(ws);
    __nv_bfloat16* z = reinterpret_cast<__nv_bfloat16*>(b + pl.off_z);
    __nv_bfloat16* q = reinterpret_cast<__nv_bfloat16*>(b + pl.off_q);
    __nv_bfloat16* k = reinterpret_cast<__nv_bfloat16*>(b + pl.off_k);
    __nv_bfloat16* v = reinterpret_cast<__nv_bfloat16*>(b + pl.off_v);
    float* g = reinterpret_cast<float*>(b + pl.off_g);
    float* beta = reinterpret_cast<float*>(b + pl.off_beta);
    float* o = reinterpret_cast<float*>(b + pl.off_o);
    const int HD = pl.HD, nz = pl.nz, ldz = pl.ldz;
    const __nv_bfloat16* zb = z;

    GemmEpilogue ep_in;  // z in bf16; the beta columns also as sigmoid in fp32
    ep_in.beta_out = beta;
    ep_in.beta_col0 = 3 * HD + 2 * R;
    ep_in.H = H;
    int rc = launch_gemm(x, D, w->W_in, D, z, ldz, ntok, nz, D, ep_in, stream, why);
    if (rc != KDA_OK) return rc;
    {
        const dim3 grid(unsigned((ntok + kConvTok - 1) / kConvTok), 3, unsigned((HD + 2047) / 2048));
        conv_silu_norm_kernel<<<grid, 256, 0, stream>>>(zb, ldz, static_cast<const __nv_bfloat16*>(w->conv_w), cu,
                                                        nseq, seq_len, ntok, H,
                                                        static_cast<const __nv_bfloat16*>(conv_in), q, k, v);
    }
    if (conv_out) {
        const long long n = (long long)nseq * 3 * HD;
        conv_cache_out_kernel<<<unsigned((n + 255) / 256), 256, 0, stream>>>(
            zb, ldz, cu, nseq, seq_len, 3 * HD, static_cast<const __nv_bfloat16*>(conv_in),
            static_cast<__nv_bfloat16*>(conv_out));
    }
    GemmEpilogue ep_decay;  // g = -softplus(a_down W_aup^T), fp32
    ep_decay.kind = GemmEpilogue::kNegSoftplus;
    rc = launch_gemm(zb + 3 * HD, ldz, w->W_aup, R, g, HD, ntok, HD, R, ep_decay, stream, why);
    if (rc != KDA_OK) return rc;
    if (decode) {
        rc = launch_recurrent_fwd(q, k, v, g, beta, state_inplace, o, nseq, seq_len, H, KDA_BF16, 1.f, 0, stream, 1);
        if (rc != KDA_OK) {
            *why = "recurrent kernel launch failed";
            return rc;
        }
    } else {
        rc = launch_chunk_fwd(q, k, v, g, beta, init, fin, o, cu, nseq, 1, ntok, H, KDA_BF16, 1.f, 0,
                              b + pl.off_chunk, pl.chunk_bytes, stream, why, 0, 1);
        if (rc != KDA_OK) return rc;
    }
    GemmEpilogue ep_gate;  // RMSNorm_head(o) * norm_w * sigmoid(g_down W_gup^T), bf16 (over q)
    ep_gate.kind = GemmEpilogue::kNormGate;
    ep_gate.o_in = o;
    ep_gate.ldo = HD;
    ep_gate.norm_w = w->norm_w;
    rc = launch_gemm(zb + 3 * HD + R, ldz, w->W_gup, R, q, HD, ntok, HD, R, ep_gate, stream, why);
    if (rc != KDA_OK) return rc;
    rc = launch_gemm(q, HD, w->W_o, HD, y, D, ntok, D, HD, GemmEpilogue{}, stream, why);
    if (rc != KDA_OK) return rc;
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        *why = cudaGetErrorString(e);
        return KDA_ERR_CUDA;
    }
    return KDA_OK;
}

int launch_layer_fwd(const void* x, const kda_layer_weights* w, const int32_t* cu, int nseq, int ntok,
                     const float* init, float* fin, const void* conv_in, void* conv_out, void* y, void* ws,
                     size_t ws_bytes, cudaStream_t stream, const char** why) {
    return layer_pipeline(x, w, cu, nseq, 0, ntok, init, fin, nullptr, conv_in, conv_out, y, ws, ws_bytes, stream,
                          why);
}

int launch_layer_decode(const void* x, const kda_layer_weights* w, void* conv_state, float* state, void* y, int B,
                        int T, void* ws, size_t ws_bytes, cudaStream_t stream, const char** why) {
    return layer_pipeline(x, w, nullptr, B, T, B * T, nullptr, nullptr, state, conv_state, conv_state, y, ws,
                          ws_bytes, stream, why);
}

}  // namespace kda
