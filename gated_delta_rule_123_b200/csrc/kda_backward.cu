// KDA backward (reverse mode of the recurrence): dq, dk, dv, dg, dbeta and the
// initial-state gradient, given the output gradient and the final-state gradient.
//
// The forward is the token recurrence ("Kimi Linear: An Expressive, Efficient
// Attention Architecture", section Method, "From Linear Attention to KDA"):
//     S~ = Diag(a) S_{t-1} (a = e^g),  y = S~^T k,  u = beta (v - y),
//     S_t = S~ + k u^T,  o = S_t^T (scale q).
// Its reverse, token t from T down to 1, with G the running gradient of S_t:
//     G += (scale q) do^T;  dq = scale (S~ do + k (u . do))
//     du = G^T k;  dv = beta du;  dbeta = du . (v - y);  dy = -beta du
//     dk = G u + S~ dy;  G~ = G + k dy^T;  dg = rowsum(G~ (.) S~);  G <- Diag(a) G~.
// Training needs these gradients ("Training and Inference": training runs the
// chunk form, with FLA's tests covering q/k/v/g/beta and initial-state
// gradients); this kernel computes them exactly (fp32) by recurrence.
//
// Layout: one CTA (256 threads) per (sequence, head); warp w owns key rows
// [16w, 16w+16), lane l value columns [4l, 4l+4); S, G and S~ live in
// registers.  Phase 1 runs the forward and stores the state at every 64-token
// boundary (checkpoints in the workspace).  Phase 2 walks the chunks backwards:
// it recomputes the chunk's 64 intermediate states from its checkpoint into a
// per-CTA scratch (4 MB, L2-resident), then runs the reverse steps reading them
// back.  Column sums (y, du) go through shared memory, one barrier each; row sums
// (dq, dk, dg) are butterfly reductions over the 32 lanes: 16 partial row sums
// per lane become one full sum per lane pair in 16 shuffles.
#include "kda_common.cuh"

namespace kda {

// Sum x[i] (i < 16, the 16 rows of this warp) over the 32 lanes.  Returns the
// full sum of row (lane >> 1) & 15 (each lane pair holds the same row).
__device__ __forceinline__ float rowsum_16x32(float (&x)[16], int lane) {
#pragma unroll
    for (int half = 8, off = 16; half >= 1; half >>= 1, off >>= 1) {
        const bool hi = (lane & off) != 0;
#pragma unroll
        for (int j = 0; j < half; ++j) {
            const float send = hi ? x[j] : x[j + half];
            const float recv = __shfl_xor_sync(0xffffffffu, send, off);
            x[j] = (hi ? x[j + half] : x[j]) + recv;
        }
    }
    return x[0] + __shfl_xor_sync(0xffffffffu, x[0], 1);
}

template <typename T>
__global__ void __launch_bounds__(256, 1)
    recurrent_bwd_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                         const float* __restrict__ g, const float* __restrict__ beta, const float* __restrict__ init,
                         const T* __restrict__ dout, const float* __restrict__ dfinal, float* __restrict__ dq,
                         float* __restrict__ dk, float* __restrict__ dv, float* __restrict__ dg,
                         float* __restrict__ dbeta, float* __restrict__ dinit, float4* __restrict__ ckpt,
                         float4* __restrict__ scratch, int Tn, int H, float scale) {
    __shared__ __align__(16) float sk[2][kD], sq[2][kD], sa[2][kD], sv[2][kD], sdo[2][kD];
    __shared__ float sb[2];
    __shared__ float4 sy[2][8][32], sdu[2][8][32];

    const int bh = blockIdx.x, b = bh / H, h = bh - b * H;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nchunks = (Tn + kC - 1) / kC;
    auto row = [&](int t) { return (size_t(b) * Tn + t) * H + h; };
    auto sidx4 = [&](int i) { return (warp * 16 + i) * 32 + lane; };  // float4 index of (row 16w+i, cols 4l..)
    float4* ck = ckpt + size_t(bh) * nchunks * (kD * kD / 4);
    float4* sc = scratch + size_t(bh) * kC * (kD * kD / 4);

    // token vectors into buffer p (threads < 128: one channel each); q is pre-scaled
    auto load_tok = [&](int t, int p, bool with_bwd) {
        if (tid < kD) {
            const size_t e = row(t) * kD + tid;
            sk[p][tid] = to_f32(k[e]);
            sa[p][tid] = expf(g[e]);
            sv[p][tid] = to_f32(v[e]);
            if (with_bwd) {
                sq[p][tid] = to_f32(q[e]) * scale;
                sdo[p][tid] = to_f32(dout[e]);
            }
            if (tid == 0) sb[p] = beta[row(t)];
        }
    };
    // one forward step on s with the token in buffer p (two barriers: vectors, partials)
    auto fwd_step = [&](float4 (&s)[16], int p) {
        __syncthreads();
        float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int r = warp * 16 + i;
            const float a = sa[p][r], kr = sk[p][r];
            s[i].x *= a; s[i].y *= a; s[i].z *= a; s[i].w *= a;
            y.x += s[i].x * kr; y.y += s[i].y * kr; y.z += s[i].z * kr; y.w += s[i].w * kr;
        }
        sy[p][warp][lane] = y;
        __syncthreads();
        float4 ys = sy[p][0][lane];
#pragma unroll
        for (int w = 1; w < 8; ++w) {
            const float4 t4 = sy[p][w][lane];
            ys.x += t4.x; ys.y += t4.y; ys.z += t4.z; ys.w += t4.w;
        }
        const float bt = sb[p];
        const float4 v4 = reinterpret_cast<const float4*>(sv[p])[lane];
        const float4 u = make_float4(bt * (v4.x - ys.x), bt * (v4.y - ys.y), bt * (v4.z - ys.z), bt * (v4.w - ys.w));
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float kr = sk[p][warp * 16 + i];
            s[i].x += kr * u.x; s[i].y += kr * u.y; s[i].z += kr * u.z; s[i].w += kr * u.w;
        }
    };

    // ---- phase 1: forward, checkpoint at every chunk start
    float4 s[16];
    {
        const float4* s0 = init ? reinterpret_cast<const float4*>(init) + size_t(bh) * (kD * kD / 4) : nullptr;
#pragma unroll
        for (int i = 0; i < 16; ++i) s[i] = s0 ? s0[sidx4(i)] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll 1
    for (int t = 0; t < Tn; ++t) {
        if ((t & (kC - 1)) == 0) {
            float4* dst = ck + size_t(t / kC) * (kD * kD / 4);
#pragma unroll
            for (int i = 0; i < 16; ++i) dst[sidx4(i)] = s[i];
        }
        load_tok(t, t & 1, false);
        fwd_step(s, t & 1);
    }

    // ---- phase 2: chunks in reverse; G is the running gradient of the state
    float4 G[16];
    {
        const float4* d0 = dfinal ? reinterpret_cast<const float4*>(dfinal) + size_t(bh) * (kD * kD / 4) : nullptr;
#pragma unroll
        for (int i = 0; i < 16; ++i) G[i] = d0 ? d0[sidx4(i)] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll 1
    for (int c = nchunks - 1; c >= 0; --c) {
        const int t0 = c * kC, t1 = min(Tn, t0 + kC);
        __syncthreads();  // the previous token's readers of the vector buffers are done
        {  // recompute S_{t-1} for every token of the chunk into the scratch
            const float4* src = ck + size_t(c) * (kD * kD / 4);
#pragma unroll
            for (int i = 0; i < 16; ++i) s[i] = src[sidx4(i)];
#pragma unroll 1
            for (int t = t0; t < t1; ++t) {
                float4* dst = sc + size_t(t - t0) * (kD * kD / 4);
#pragma unroll
                for (int i = 0; i < 16; ++i) dst[sidx4(i)] = s[i];
                load_tok(t, t & 1, false);
                fwd_step(s, t & 1);
            }
        }
        __syncthreads();  // as above, before the reverse loop reuses the buffers (each thread reads back only its own scratch)
#pragma unroll 1
        for (int t = t1 - 1; t >= t0; --t) {
            const int p = t & 1;
            float4 St[16];
            const float4* src = sc + size_t(t - t0) * (kD * kD / 4);
#pragma unroll
            for (int i = 0; i < 16; ++i) St[i] = src[sidx4(i)];
            load_tok(t, p, true);
            __syncthreads();
            float4 y = make_float4(0.f, 0.f, 0.f, 0.f), du = y;
            const float4 do4 = reinterpret_cast<const float4*>(sdo[p])[lane];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int r = warp * 16 + i;
                const float a = sa[p][r], kr = sk[p][r], qr = sq[p][r];
                St[i].x *= a; St[i].y *= a; St[i].z *= a; St[i].w *= a;  // S~ = Diag(a) S_{t-1}
                y.x += St[i].x * kr; y.y += St[i].y * kr; y.z += St[i].z * kr; y.w += St[i].w * kr;
                G[i].x += qr * do4.x; G[i].y += qr * do4.y; G[i].z += qr * do4.z; G[i].w += qr * do4.w;
                du.x += G[i].x * kr; du.y += G[i].y * kr; du.z += G[i].z * kr; du.w += G[i].w * kr;
            }
            sy[p][warp][lane] = y;
            sdu[p][warp][lane] = du;
            __syncthreads();
            float4 ys = sy[p][0][lane], dus = sdu[p][0][lane];
#pragma unroll
            for (int w = 1; w < 8; ++w) {
                const float4 a4 = sy[p][w][lane], b4 = sdu[p][w][lane];
                ys.x += a4.x; ys.y += a4.y; ys.z += a4.z; ys.w += a4.w;
                dus.x += b4.x; dus.y += b4.y; dus.z += b4.z; dus.w += b4.w;
            }
            const float bt = sb[p];
            const float4 v4 = reinterpret_cast<const float4*>(sv[p])[lane];
            const float4 r4 = make_float4(v4.x - ys.x, v4.y - ys.y, v4.z - ys.z, v4.w - ys.w);  // v - y
            const float4 u = make_float4(bt * r4.x, bt * r4.y, bt * r4.z, bt * r4.w);
            const float4 dy = make_float4(-bt * dus.x, -bt * dus.y, -bt * dus.z, -bt * dus.w);
            float udo = u.x * do4.x + u.y * do4.y + u.z * do4.z + u.w * do4.w;
            float dbt = dus.x * r4.x + dus.y * r4.y + dus.z * r4.z + dus.w * r4.w;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                udo += __shfl_xor_sync(0xffffffffu, udo, off);
                dbt += __shfl_xor_sync(0xffffffffu, dbt, off);
            }
            if (warp == 0) {
                *reinterpret_cast<float4*>(dv + row(t) * kD + 4 * lane) =
                    make_float4(bt * dus.x, bt * dus.y, bt * dus.z, bt * dus.w);
                if (lane == 0) dbeta[row(t)] = dbt;
            }
            const int rr = warp * 16 + ((lane >> 1) & 15);  // the row this lane pair reduces
            const bool writer = (lane & 1) == 0;
            float x[16];
            // dq = scale (S~ do + k (u . do))
#pragma unroll
            for (int i = 0; i < 16; ++i) x[i] = St[i].x * do4.x + St[i].y * do4.y + St[i].z * do4.z + St[i].w * do4.w;
            float sum = rowsum_16x32(x, lane);
            if (writer) dq[row(t) * kD + rr] = scale * (sum + sk[p][rr] * udo);
            // dk = G u + S~ dy
#pragma unroll
            for (int i = 0; i < 16; ++i)
                x[i] = G[i].x * u.x + G[i].y * u.y + G[i].z * u.z + G[i].w * u.w + St[i].x * dy.x + St[i].y * dy.y +
                       St[i].z * dy.z + St[i].w * dy.w;
            sum = rowsum_16x32(x, lane);
            if (writer) dk[row(t) * kD + rr] = sum;
            // G~ = G + k dy^T;  dg = rowsum(G~ (.) S~);  G <- Diag(a) G~
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int r = warp * 16 + i;
                const float kr = sk[p][r], a = sa[p][r];
                G[i].x += kr * dy.x; G[i].y += kr * dy.y; G[i].z += kr * dy.z; G[i].w += kr * dy.w;
                x[i] = G[i].x * St[i].x + G[i].y * St[i].y + G[i].z * St[i].z + G[i].w * St[i].w;
                G[i].x *= a; G[i].y *= a; G[i].z *= a; G[i].w *= a;
            }
            sum = rowsum_16x32(x, lane);
            if (writer) dg[row(t) * kD + rr] = sum;
        }
    }
    if (dinit) {
        float4* d = reinterpret_cast<float4*>(dinit) + size_t(bh) * (kD * kD / 4);
#pragma unroll
        for (int i = 0; i < 16; ++i) d[sidx4(i)] = G[i];
    }
}

size_t recurrent_bwd_workspace_bytes(int B, int T, int H) {
    const size_t nchunks = (size_t(T) + kC - 1) / kC;
    return (size_t(B) * H * (nchunks + kC)) * kD * kD * sizeof(float);
}

int launch_recurrent_bwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
                         const float* init, const void* dout, const float* dfinal, float* dq, float* dk, float* dv,
                         float* dg, float* dbeta, float* dinit, int B, int Tn, int H, int dtype, float scale,
                         void* ws, size_t ws_bytes, cudaStream_t stream, const char** why) {
    const int nbh = B * H;
    if (nbh == 0) return KDA_OK;
    if (ws_bytes < recurrent_bwd_workspace_bytes(B, Tn, H) || ws == nullptr) {
        *why = "workspace smaller than kda_recurrent_bwd_workspace()";
        return KDA_ERR_WORKSPACE;
    }
    const size_t nchunks = (size_t(Tn) + kC - 1) / kC;
    float4* ckpt = static_cast<float4*>(ws);
    float4* scr = ckpt + size_t(nbh) * nchunks * (kD * kD / 4);
    if (dtype == KDA_BF16) {
        using Tb = __nv_bfloat16;
        recurrent_bwd_kernel<Tb><<<nbh, 256, 0, stream>>>(
            static_cast<const Tb*>(q), static_cast<const Tb*>(k), static_cast<const Tb*>(v), g, beta, init,
            static_cast<const Tb*>(dout), dfinal, dq, dk, dv, dg, dbeta, dinit, ckpt, scr, Tn, H, scale);
    } else {
        recurrent_bwd_kernel<float><<<nbh, 256, 0, stream>>>(
            static_cast<const float*>(q), static_cast<const float*>(k), static_cast<const float*>(v), g, beta, init,
            static_cast<const float*>(dout), dfinal, dq, dk, dv, dg, dbeta, dinit, ckpt, scr, Tn, H, scale);
    }
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        *why = cudaGetErrorString(e);
        return KDA_ERR_CUDA;
    }
    return KDA_OK;
}

}  // namespace kda
