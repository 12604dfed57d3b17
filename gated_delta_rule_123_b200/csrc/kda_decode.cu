// KDA recurrent decode step: one token per sequence, each head's fp32 state
// read once and written once, in place.
//
// Residual form of the KDA recurrence ("Kimi Linear: An Expressive, Efficient
// Attention Architecture", section Method, "From Linear Attention to KDA":
// S~ = Diag(alpha) S, S = S~ + beta k (v - S~^T k)^T, o = S^T q), evaluated in
// one pass over S:
//     y = S~^T k,  z = S~^T q,  u = beta (v - y),  S <- S~ + k u^T,
//     o = S^T q = z + (k^T q) u.
// Bandwidth-bound: 64 KB read + 64 KB written per head, 128-bit coalesced.
#include "kda_common.cuh"

namespace kda {

// One CTA (256 threads) per (sequence, head).  Warp w owns key rows
// [16w, 16w+16); lane l owns value columns [4l, 4l+4), so every row is read
// and written as one 512-byte coalesced warp access.
template <typename T>
__global__ void __launch_bounds__(256, 2)
    decode_step_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                       const float* __restrict__ g, const float* __restrict__ beta, float* __restrict__ state,
                       T* __restrict__ o, float scale, int l2norm) {
    __shared__ float sk[kD], sq[kD], sa[kD];
    __shared__ float4 sy[8][32], sz[8][32];
    __shared__ float4 su[32];
    __shared__ float s_coef[3];  // k scale, q scale, (k^T q) with both scales

    const int bh = blockIdx.x;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const size_t vec = size_t(bh) * kD;
    float4* S4 = reinterpret_cast<float4*>(state) + size_t(bh) * (kD * kD / 4);

    // Issue all 16 row loads of this thread first (64 KB in flight per CTA).
    float4 s[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) s[i] = __ldcs(&S4[(warp * 16 + i) * 32 + lane]);

    if (tid < kD) {
        sk[tid] = to_f32(k[vec + tid]);
        sq[tid] = to_f32(q[vec + tid]);
        sa[tid] = expf(g[vec + tid]);
    }
    __syncthreads();
    if (warp == 0) {
        float kk = 0.f, qq = 0.f, kq = 0.f;
#pragma unroll
        for (int j = lane; j < kD; j += 32) {
            kk += sk[j] * sk[j];
            qq += sq[j] * sq[j];
            kq += sk[j] * sq[j];
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            kk += __shfl_xor_sync(0xffffffffu, kk, off);
            qq += __shfl_xor_sync(0xffffffffu, qq, off);
            kq += __shfl_xor_sync(0xffffffffu, kq, off);
        }
        if (lane == 0) {
            const float nk = l2norm ? rsqrtf(kk + 1e-6f) : 1.f;
            const float nq = (l2norm ? rsqrtf(qq + 1e-6f) : 1.f) * scale;
            s_coef[0] = nk;
            s_coef[1] = nq;
            s_coef[2] = kq * nk * nq;
        }
    }
    __syncthreads();
    const float nk = s_coef[0], nq = s_coef[1];

    float4 y = make_float4(0.f, 0.f, 0.f, 0.f), z = y;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int r = warp * 16 + i;
        const float a = sa[r], kr = sk[r] * nk, qr = sq[r] * nq;
        s[i].x *= a;
        s[i].y *= a;
        s[i].z *= a;
        s[i].w *= a;
        y.x += s[i].x * kr;
        y.y += s[i].y * kr;
        y.z += s[i].z * kr;
        y.w += s[i].w * kr;
        z.x += s[i].x * qr;
        z.y += s[i].y * qr;
        z.z += s[i].z * qr;
        z.w += s[i].w * qr;
    }
    sy[warp][lane] = y;
    sz[warp][lane] = z;
    __syncthreads();
    if (tid < 32) {
        float4 ys = sy[0][tid], zs = sz[0][tid];
#pragma unroll
        for (int w = 1; w < 8; ++w) {
            ys.x += sy[w][tid].x; ys.y += sy[w][tid].y; ys.z += sy[w][tid].z; ys.w += sy[w][tid].w;
            zs.x += sz[w][tid].x; zs.y += sz[w][tid].y; zs.z += sz[w][tid].z; zs.w += sz[w][tid].w;
        }
        const float b = beta[bh];
        const size_t vb = vec + 4 * tid;
        float4 u;
        u.x = b * (to_f32(v[vb + 0]) - ys.x);
        u.y = b * (to_f32(v[vb + 1]) - ys.y);
        u.z = b * (to_f32(v[vb + 2]) - ys.z);
        u.w = b * (to_f32(v[vb + 3]) - ys.w);
        su[tid] = u;
        const float kq = s_coef[2];
        o[vb + 0] = from_f32<T>(zs.x + kq * u.x);
        o[vb + 1] = from_f32<T>(zs.y + kq * u.y);
        o[vb + 2] = from_f32<T>(zs.z + kq * u.z);
        o[vb + 3] = from_f32<T>(zs.w + kq * u.w);
    }
    __syncthreads();
    const float4 u = su[lane];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const float kr = sk[warp * 16 + i] * nk;
        float4 t = s[i];
        t.x += kr * u.x;
        t.y += kr * u.y;
        t.z += kr * u.z;
        t.w += kr * u.w;
        __stcs(&S4[(warp * 16 + i) * 32 + lane], t);
    }
}

int launch_decode_step(const void* q, const void* k, const void* v, const float* g, const float* beta,
                       float* state, void* o, int B, int H, int dtype, float scale, int l2norm,
                       cudaStream_t stream) {
    const int nbh = B * H;
    if (nbh == 0) return KDA_OK;
    if (dtype == KDA_BF16) {
        decode_step_kernel<__nv_bfloat16><<<nbh, 256, 0, stream>>>(
            static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
            static_cast<const __nv_bfloat16*>(v), g, beta, state, static_cast<__nv_bfloat16*>(o), scale, l2norm);
    } else {
        decode_step_kernel<float><<<nbh, 256, 0, stream>>>(
            static_cast<const float*>(q), static_cast<const float*>(k), static_cast<const float*>(v), g, beta, state,
            static_cast<float*>(o), scale, l2norm);
    }
    return cudaGetLastError() == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

// ---------------------------------------------------------------- recurrent segments
// kda_recurrent_fwd: T tokens per sequence (the pages' fused recurrent path for
// single steps and segments of up to 64 tokens), each head's state read once,
// carried in registers across the segment and written once.
//
// One CTA (256 threads) per (sequence, head); warp w owns key rows [16w, 16w+16),
// lane l value columns [4l, 4l+4), as in decode_step_kernel.  Per token there is
// one barrier: every warp writes its partial S~^T k and S~^T q (16 rows) and then
// reduces all eight partials itself for its lane's columns, so u = beta (v - y)
// needs no second broadcast.  Token vectors are loaded one token ahead by
// threads 0..127 (global -> registers -> shared), into a triple buffer; partials
// are double-buffered.  Buffer reuse distances: a token buffer written during
// token t (for t+1) was last read during token t-2, and every warp has passed
// token t-1's barrier before any warp starts token t.
template <typename T, typename OutT>
__global__ void __launch_bounds__(256, 2)
    recurrent_fwd_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                         const float* __restrict__ g, const float* __restrict__ beta, float* __restrict__ state,
                         OutT* __restrict__ o, int Tn, int H, float scale, int l2norm) {
    __shared__ __align__(16) float sk[3][kD], sq[3][kD], sa[3][kD], sv[3][kD];
    __shared__ float sdot[3][4][3];  // per loader warp: k.k, q.q, k.q
    __shared__ float sb[3];
    __shared__ float4 sy[2][8][32], sz[2][8][32];

    const int bh = blockIdx.x, b = bh / H, h = bh - b * H;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    float4* S4 = reinterpret_cast<float4*>(state) + size_t(bh) * (kD * kD / 4);
    auto row = [&](int t) { return (size_t(b) * Tn + t) * H + h; };  // (token, head) row index

    float4 s[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) s[i] = __ldcs(&S4[(warp * 16 + i) * 32 + lane]);

    // token vectors: thread c < 128 handles channel c
    float rk = 0.f, rq = 0.f, rg = 0.f, rv = 0.f, rb = 0.f;
    auto load = [&](int t) {
        if (tid < kD && t < Tn) {
            const size_t e = row(t) * kD + tid;
            rk = to_f32(k[e]);
            rq = to_f32(q[e]);
            rg = g[e];
            rv = to_f32(v[e]);
            if (tid == 0) rb = beta[row(t)];
        }
    };
    auto put = [&](int t) {
        if (tid < kD && t < Tn) {
            const int p = t % 3;
            sk[p][tid] = rk;
            sq[p][tid] = rq;
            sa[p][tid] = expf(rg);
            sv[p][tid] = rv;
            if (tid == 0) sb[p] = rb;
            float kk = rk * rk, qq = rq * rq, kq = rk * rq;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                kk += __shfl_xor_sync(0xffffffffu, kk, off);
                qq += __shfl_xor_sync(0xffffffffu, qq, off);
                kq += __shfl_xor_sync(0xffffffffu, kq, off);
            }
            if (lane == 0) {
                sdot[p][warp][0] = kk;
                sdot[p][warp][1] = qq;
                sdot[p][warp][2] = kq;
            }
        }
    };
    load(0);
    put(0);
    __syncthreads();

#pragma unroll 1
    for (int t = 0; t < Tn; ++t) {
        const int p = t % 3, pp = t & 1;
        load(t + 1);  // in flight during this token's work
        const float kk = sdot[p][0][0] + sdot[p][1][0] + sdot[p][2][0] + sdot[p][3][0];
        const float qq = sdot[p][0][1] + sdot[p][1][1] + sdot[p][2][1] + sdot[p][3][1];
        const float kq = sdot[p][0][2] + sdot[p][1][2] + sdot[p][2][2] + sdot[p][3][2];
        const float nk = l2norm ? rsqrtf(kk + 1e-6f) : 1.f;
        const float nq = (l2norm ? rsqrtf(qq + 1e-6f) : 1.f) * scale;
        float4 y = make_float4(0.f, 0.f, 0.f, 0.f), z = y;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int r = warp * 16 + i;
            const float a = sa[p][r], kr = sk[p][r] * nk, qr = sq[p][r] * nq;
            s[i].x *= a;
            s[i].y *= a;
            s[i].z *= a;
            s[i].w *= a;
            y.x += s[i].x * kr;
            y.y += s[i].y * kr;
            y.z += s[i].z * kr;
            y.w += s[i].w * kr;
            z.x += s[i].x * qr;
            z.y += s[i].y * qr;
            z.z += s[i].z * qr;
            z.w += s[i].w * qr;
        }
        sy[pp][warp][lane] = y;
        sz[pp][warp][lane] = z;
        put(t + 1);
        __syncthreads();
        float4 ys = sy[pp][0][lane], zs = sz[pp][0][lane];
#pragma unroll
        for (int w = 1; w < 8; ++w) {
            const float4 a4 = sy[pp][w][lane], b4 = sz[pp][w][lane];
            ys.x += a4.x; ys.y += a4.y; ys.z += a4.z; ys.w += a4.w;
            zs.x += b4.x; zs.y += b4.y; zs.z += b4.z; zs.w += b4.w;
        }
        const float bt = sb[p];
        const float4 v4 = reinterpret_cast<const float4*>(sv[p])[lane];
        float4 u;
        u.x = bt * (v4.x - ys.x);
        u.y = bt * (v4.y - ys.y);
        u.z = bt * (v4.z - ys.z);
        u.w = bt * (v4.w - ys.w);
        if (warp == 0) {  // o = S_new^T q = z + (k^T q) u, scales folded in
            const float c = kq * nk * nq;
            OutT* op = o + row(t) * kD + 4 * lane;
            op[0] = from_f32<OutT>(zs.x + c * u.x);
            op[1] = from_f32<OutT>(zs.y + c * u.y);
            op[2] = from_f32<OutT>(zs.z + c * u.z);
            op[3] = from_f32<OutT>(zs.w + c * u.w);
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const float kr = sk[p][warp * 16 + i] * nk;
            s[i].x += kr * u.x;
            s[i].y += kr * u.y;
            s[i].z += kr * u.z;
            s[i].w += kr * u.w;
        }
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) __stcs(&S4[(warp * 16 + i) * 32 + lane], s[i]);
}

// out_f32 != 0 writes o in fp32 whatever the input dtype (the layer's use).
int launch_recurrent_fwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
                         float* state, void* o, int B, int Tn, int H, int dtype, float scale, int l2norm,
                         cudaStream_t stream, int out_f32) {
    const int nbh = B * H;
    if (nbh == 0) return KDA_OK;
    if (dtype == KDA_BF16) {
        auto qb = static_cast<const __nv_bfloat16*>(q);
        auto kb = static_cast<const __nv_bfloat16*>(k);
        auto vb = static_cast<const __nv_bfloat16*>(v);
        if (out_f32)
            recurrent_fwd_kernel<__nv_bfloat16, float><<<nbh, 256, 0, stream>>>(
                qb, kb, vb, g, beta, state, static_cast<float*>(o), Tn, H, scale, l2norm);
        else
            recurrent_fwd_kernel<__nv_bfloat16, __nv_bfloat16><<<nbh, 256, 0, stream>>>(
                qb, kb, vb, g, beta, state, static_cast<__nv_bfloat16*>(o), Tn, H, scale, l2norm);
    } else {
        recurrent_fwd_kernel<float, float><<<nbh, 256, 0, stream>>>(
            static_cast<const float*>(q), static_cast<const float*>(k), static_cast<const float*>(v), g, beta, state,
            static_cast<float*>(o), Tn, H, scale, l2norm);
    }
    return cudaGetLastError() == cudaSuccess ? KDA_OK : KDA_ERR_CUDA;
}

}  // namespace kda
