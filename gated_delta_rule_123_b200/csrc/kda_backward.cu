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
// Parallel layout.  The recurrence never mixes value columns: column j of S and
// of G evolves on its own (y, u, du and dy are per-column).  So every (sequence,
// head) is split into kSlices = 16 CTAs of kSliceCols = 8 value columns each, and a
// CTA is one warp that runs the whole sequence for its columns, lane l holding key
// rows 4l..4l+3.  The per-column sums y = S~^T k and du = G^T k are a shuffle
// reduce-scatter inside the warp (no barrier), and the per-row sums dq, dk, dg (and
// the scalar dbeta) are in-thread partial sums over the CTA's columns.  Those
// partials go to the workspace and a second kernel adds the slices up (in a fixed
// order, so results are deterministic); dv and the initial-state gradient are
// per-column and written directly.
//   Phase 1 runs the forward and stores the state slice at every kSub-token
//   boundary.  Phase 2 walks the sub-chunks backwards: it recomputes the kSub
//   states S_{t-1} of a sub-chunk from its checkpoint into shared memory, then
//   runs the reverse steps reading them back.  Each sub-chunk's token inputs (k,
//   q, g per row; the slice's v and dO; beta) are staged into shared memory with
//   cp.async one sub-chunk ahead, so a step reads nothing from global memory.
#include "kda_common.cuh"

namespace kda {
namespace bwd {

constexpr int kSliceCols = 8;                  // value columns per CTA
constexpr int kSlices = kD / kSliceCols;       // CTAs per (sequence, head)
constexpr int kSub = 16;                       // tokens per recomputed / staged sub-chunk
constexpr int kThreads = 32;                   // one warp: lane l holds key rows 4l..4l+3
constexpr int kRows = kD / kThreads;           // key rows per lane
constexpr uint32_t kStateBytes = kSub * kSliceCols * kD * sizeof(float);  // states [kSub][col][row]

// One sub-chunk of token inputs in shared memory (element type E of q, k, v, dO):
// k, q [kSub][128]; g fp32 [kSub][128]; the slice's v, dO [kSub][8]; beta [kSub].
template <typename E>
struct Stage {
    static constexpr uint32_t K = 0, Q = kSub * kD * sizeof(E), G = 2 * Q, V = G + kSub * kD * 4,
                              DO = V + kSub * kSliceCols * sizeof(E), B = DO + kSub * kSliceCols * sizeof(E),
                              kBytes = (B + kSub * 4 + 127) & ~127u;
};
template <typename E>
constexpr uint32_t smem_bytes() { return kStateBytes + 2 * Stage<E>::kBytes; }

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_4(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_wait_1() { asm volatile("cp.async.wait_group 1;" ::: "memory"); }
__device__ __forceinline__ void cp_wait_0() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// Sum x[c] (c < 8) over the 32 lanes of the warp.  Returns, in every lane, the full
// sum of column lane >> 2 (lanes 4c..4c+3 hold column c): a reduce-scatter that halves
// the values per lane at each step (7 shuffles), then two plain sums.
__device__ __forceinline__ float colsum8(float (&x)[8], int lane) {
    int off = 16;
#pragma unroll
    for (int half = 4; half >= 1; half >>= 1, off >>= 1) {
        const bool hi = (lane & off) != 0;
#pragma unroll
        for (int j = 0; j < half; ++j) {
            const float send = hi ? x[j] : x[j + half];
            const float recv = __shfl_xor_sync(0xffffffffu, send, off);
            x[j] = (hi ? x[j + half] : x[j]) + recv;
        }
    }
    float sum = x[0];
    sum += __shfl_xor_sync(0xffffffffu, sum, 2);
    sum += __shfl_xor_sync(0xffffffffu, sum, 1);
    return sum;
}

template <typename T>
__device__ __forceinline__ void load4(const uint8_t* p, float* out) {  // 4 consecutive elements of type T
    if constexpr (sizeof(T) == 2) {
        const uint2 raw = *reinterpret_cast<const uint2*>(p);
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
        out[0] = __low2float(h2[0]);
        out[1] = __high2float(h2[0]);
        out[2] = __low2float(h2[1]);
        out[3] = __high2float(h2[1]);
    } else {
        const float4 f = *reinterpret_cast<const float4*>(p);
        out[0] = f.x; out[1] = f.y; out[2] = f.z; out[3] = f.w;
    }
}
template <typename T>
__device__ __forceinline__ void load8(const uint8_t* p, float* out) {  // 8 consecutive elements of type T
    load4<T>(p, out);
    load4<T>(p + 4 * sizeof(T), out + 4);
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
    recurrent_bwd_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                         const float* __restrict__ g, const float* __restrict__ beta, const float* __restrict__ init,
                         const T* __restrict__ dout, const float* __restrict__ dfinal, float* __restrict__ dv,
                         float* __restrict__ dinit, float* __restrict__ part, float* __restrict__ ckpt, int Tn, int H,
                         float scale) {
    extern __shared__ __align__(128) uint8_t smem[];
    float* sst = reinterpret_cast<float*>(smem);  // [kSub][kSliceCols][kD]: S_{t-1} of the sub-chunk's tokens
    using S = Stage<T>;

    const int bh = blockIdx.x, sl = blockIdx.y, b = bh / H, h = bh - b * H;
    const int lane = threadIdx.x, r0 = kRows * lane;
    const int c0 = sl * kSliceCols;
    const int nsub = (Tn + kSub - 1) / kSub;
    const size_t TH = size_t(gridDim.x) * Tn;  // (sequence, token, head) rows: [B][Tn][H]
    auto row = [&](int t) { return (size_t(b) * Tn + t) * H + h; };
    // per-slice partial sums: [slice][dq | dk | dg][B*Tn*H][kD], then dbeta [slice][B*Tn*H]
    float* p_dq = part + (size_t(sl) * 3 + 0) * TH * kD;
    float* p_dk = part + (size_t(sl) * 3 + 1) * TH * kD;
    float* p_dg = part + (size_t(sl) * 3 + 2) * TH * kD;
    float* p_db = part + size_t(kSlices) * 3 * TH * kD + size_t(sl) * TH;
    float* ck = ckpt + (size_t(bh) * kSlices + sl) * size_t(nsub) * (kSliceCols * kD);  // [nsub][col][row]
    const uint32_t stage0 = smem_u32(smem + kStateBytes);

    // Stage sub-chunk sc into buffer buf with cp.async (tokens past the end read as zero).
    auto stage = [&](int sc, int buf, bool with_bwd) {
        const uint32_t base = stage0 + uint32_t(buf) * S::kBytes;
        constexpr int per_row = kD * sizeof(T) / 16;           // 16-byte pieces of a 128-wide row
        constexpr int per_slice = kSliceCols * sizeof(T) / 16;  // of the slice's 8 values
        for (int i = lane; i < kSub * per_row; i += kThreads) {
            const int j = i / per_row, piece = i % per_row, t = sc * kSub + j;
            const bool ok = t < Tn;
            const size_t e = (ok ? row(t) : 0) * kD;
            const uint32_t off = uint32_t(j * kD * sizeof(T) + piece * 16);
            cp_async16(base + S::K + off, reinterpret_cast<const uint8_t*>(k + e) + piece * 16, ok ? 16u : 0u);
            if (with_bwd)
                cp_async16(base + S::Q + off, reinterpret_cast<const uint8_t*>(q + e) + piece * 16, ok ? 16u : 0u);
        }
        for (int i = lane; i < kSub * (kD * 4 / 16); i += kThreads) {
            const int j = i / (kD * 4 / 16), piece = i % (kD * 4 / 16), t = sc * kSub + j;
            const bool ok = t < Tn;
            const size_t e = (ok ? row(t) : 0) * kD;
            cp_async16(base + S::G + uint32_t(j * kD * 4 + piece * 16),
                       reinterpret_cast<const uint8_t*>(g + e) + piece * 16, ok ? 16u : 0u);
        }
        for (int i = lane; i < kSub * per_slice; i += kThreads) {
            const int j = i / per_slice, piece = i % per_slice, t = sc * kSub + j;
            const bool ok = t < Tn;
            const size_t e = (ok ? row(t) : 0) * kD + c0;
            const uint32_t off = uint32_t(j * kSliceCols * sizeof(T) + piece * 16);
            cp_async16(base + S::V + off, reinterpret_cast<const uint8_t*>(v + e) + piece * 16, ok ? 16u : 0u);
            if (with_bwd)
                cp_async16(base + S::DO + off, reinterpret_cast<const uint8_t*>(dout + e) + piece * 16,
                           ok ? 16u : 0u);
        }
        if (lane < kSub) {
            const int t = sc * kSub + lane;
            const bool ok = t < Tn;
            cp_async_4(base + S::B + lane * 4, beta + (ok ? row(t) : 0), ok ? 4u : 0u);
        }
        cp_commit();
    };
    auto sbuf = [&](int buf) { return smem + kStateBytes + buf * S::kBytes; };

    // y[c] (c < 8) = sum over all 128 rows of x[r][c] * w[r]: the warp's column sums, in every lane
    auto colsums = [&](const float (&x)[kRows][kSliceCols], const float (&w)[kRows], float (&y)[kSliceCols]) {
        float p[kSliceCols];
#pragma unroll
        for (int c = 0; c < kSliceCols; ++c) {
            p[c] = x[0][c] * w[0];
#pragma unroll
            for (int rr = 1; rr < kRows; ++rr) p[c] = fmaf(x[rr][c], w[rr], p[c]);
        }
        const float tot = colsum8(p, lane);
#pragma unroll
        for (int c = 0; c < kSliceCols; ++c) y[c] = __shfl_sync(0xffffffffu, tot, 4 * c);
    };
    // the token's per-row k and a = e^g (this lane's 4 rows), from staged buffer sb
    auto rows_ka = [&](const uint8_t* sb, int j, float (&kr)[kRows], float (&a)[kRows]) {
        load4<T>(sb + S::K + (j * kD + r0) * sizeof(T), kr);
        const float4 g4 = *reinterpret_cast<const float4*>(sb + S::G + (j * kD + r0) * 4);
        a[0] = expf(g4.x); a[1] = expf(g4.y); a[2] = expf(g4.z); a[3] = expf(g4.w);
    };
    // one forward step of this lane's 4 rows of the slice, token j of staged buffer sb
    auto fwd_step = [&](float (&s)[kRows][kSliceCols], const uint8_t* sb, int j) {
        float kr[kRows], a[kRows], vv[kSliceCols], y[kSliceCols];
        rows_ka(sb, j, kr, a);
        load8<T>(sb + S::V + j * kSliceCols * sizeof(T), vv);
        const float bt = reinterpret_cast<const float*>(sb + S::B)[j];
#pragma unroll
        for (int rr = 0; rr < kRows; ++rr)
#pragma unroll
            for (int c = 0; c < kSliceCols; ++c) s[rr][c] *= a[rr];
        colsums(s, kr, y);
#pragma unroll
        for (int c = 0; c < kSliceCols; ++c) {
            const float u = bt * (vv[c] - y[c]);
#pragma unroll
            for (int rr = 0; rr < kRows; ++rr) s[rr][c] = fmaf(kr[rr], u, s[rr][c]);
        }
    };

    // ---- phase 1: forward, checkpoint at every sub-chunk start
    float s[kRows][kSliceCols];
#pragma unroll
    for (int rr = 0; rr < kRows; ++rr)
#pragma unroll
        for (int c = 0; c < kSliceCols; ++c)
            s[rr][c] = init ? init[(size_t(bh) * kD + r0 + rr) * kD + c0 + c] : 0.f;
    stage(0, 0, false);
#pragma unroll 1
    for (int sc = 0; sc < nsub; ++sc) {
        if (sc + 1 < nsub) {
            stage(sc + 1, (sc + 1) & 1, false);
            cp_wait_1();
        } else {
            cp_wait_0();
        }
        __syncwarp();  // sub-chunk sc has landed for every lane
        float* dst = ck + size_t(sc) * (kSliceCols * kD);
#pragma unroll
        for (int c = 0; c < kSliceCols; ++c)
            *reinterpret_cast<float4*>(dst + c * kD + r0) = make_float4(s[0][c], s[1][c], s[2][c], s[3][c]);
        const uint8_t* sb = sbuf(sc & 1);
        const int len = min(kSub, Tn - sc * kSub);
#pragma unroll 1
        for (int j = 0; j < len; ++j) fwd_step(s, sb, j);
        __syncwarp();  // every lane is done with buffer sc & 1 before it is restaged
    }

    // ---- phase 2: sub-chunks in reverse; G is the running gradient of the state
    float G[kRows][kSliceCols];
#pragma unroll
    for (int rr = 0; rr < kRows; ++rr)
#pragma unroll
        for (int c = 0; c < kSliceCols; ++c)
            G[rr][c] = dfinal ? dfinal[(size_t(bh) * kD + r0 + rr) * kD + c0 + c] : 0.f;
    stage(nsub - 1, (nsub - 1) & 1, true);
#pragma unroll 1
    for (int sc = nsub - 1; sc >= 0; --sc) {
        if (sc > 0) {
            stage(sc - 1, (sc - 1) & 1, true);
            cp_wait_1();
        } else {
            cp_wait_0();
        }
        __syncwarp();  // sub-chunk sc has landed for every lane
        const uint8_t* sb = sbuf(sc & 1);
        const int t0 = sc * kSub, len = min(kSub, Tn - t0);
        {  // recompute S_{t-1} of every token of the sub-chunk into shared memory (own rows only)
            const float* src = ck + size_t(sc) * (kSliceCols * kD);
#pragma unroll
            for (int c = 0; c < kSliceCols; ++c) {
                const float4 x4 = *reinterpret_cast<const float4*>(src + c * kD + r0);
                s[0][c] = x4.x; s[1][c] = x4.y; s[2][c] = x4.z; s[3][c] = x4.w;
            }
#pragma unroll 1
            for (int j = 0; j < len; ++j) {
                float* dst = sst + j * (kSliceCols * kD);
#pragma unroll
                for (int c = 0; c < kSliceCols; ++c)
                    *reinterpret_cast<float4*>(dst + c * kD + r0) = make_float4(s[0][c], s[1][c], s[2][c], s[3][c]);
                fwd_step(s, sb, j);
            }
        }
#pragma unroll 1
        for (int j = len - 1; j >= 0; --j) {
            const int t = t0 + j;
            float kr[kRows], a[kRows], qr[kRows], d[kSliceCols], vv[kSliceCols];
            rows_ka(sb, j, kr, a);
            load4<T>(sb + S::Q + (j * kD + r0) * sizeof(T), qr);
            load8<T>(sb + S::DO + j * kSliceCols * sizeof(T), d);
            load8<T>(sb + S::V + j * kSliceCols * sizeof(T), vv);
            const float bt = reinterpret_cast<const float*>(sb + S::B)[j];
            const float* src = sst + j * (kSliceCols * kD);
            float St[kRows][kSliceCols];
#pragma unroll
            for (int c = 0; c < kSliceCols; ++c) {
                const float4 x4 = *reinterpret_cast<const float4*>(src + c * kD + r0);
                St[0][c] = x4.x * a[0]; St[1][c] = x4.y * a[1]; St[2][c] = x4.z * a[2]; St[3][c] = x4.w * a[3];
            }
#pragma unroll
            for (int rr = 0; rr < kRows; ++rr) {
                const float qs = qr[rr] * scale;
#pragma unroll
                for (int c = 0; c < kSliceCols; ++c) G[rr][c] = fmaf(qs, d[c], G[rr][c]);
            }
            float y[kSliceCols], du[kSliceCols];
            colsums(St, kr, y);
            colsums(G, kr, du);
            float udo = 0.f, dbt = 0.f, u[kSliceCols], dy[kSliceCols];
#pragma unroll
            for (int c = 0; c < kSliceCols; ++c) {
                const float rr = vv[c] - y[c];  // v - y
                u[c] = bt * rr;
                dy[c] = -bt * du[c];
                udo = fmaf(u[c], d[c], udo);
                dbt = fmaf(du[c], rr, dbt);
            }
            float xq[kRows], xk[kRows], xg[kRows];
#pragma unroll
            for (int rr = 0; rr < kRows; ++rr) {
                float aq = 0.f, ak = 0.f, ag = 0.f;
#pragma unroll
                for (int c = 0; c < kSliceCols; ++c) {
                    aq = fmaf(St[rr][c], d[c], aq);
                    ak = fmaf(G[rr][c], u[c], fmaf(St[rr][c], dy[c], ak));
                    const float gt = fmaf(kr[rr], dy[c], G[rr][c]);  // G~ = G + k dy^T
                    ag = fmaf(gt, St[rr][c], ag);
                    G[rr][c] = gt * a[rr];  // G <- Diag(a) G~
                }
                xq[rr] = scale * (aq + kr[rr] * udo);
                xk[rr] = ak;
                xg[rr] = ag;
            }
            const size_t e = row(t);
            float dur = 0.f;
#pragma unroll
            for (int c = 0; c < kSliceCols; ++c) dur = (c == lane) ? du[c] : dur;
            if (lane < kSliceCols) dv[e * kD + c0 + lane] = bt * dur;  // dv = beta du: lane c writes column c0 + c
            if (lane == 0) p_db[e] = dbt;
            *reinterpret_cast<float4*>(p_dq + e * kD + r0) = make_float4(xq[0], xq[1], xq[2], xq[3]);
            *reinterpret_cast<float4*>(p_dk + e * kD + r0) = make_float4(xk[0], xk[1], xk[2], xk[3]);
            *reinterpret_cast<float4*>(p_dg + e * kD + r0) = make_float4(xg[0], xg[1], xg[2], xg[3]);
        }
        __syncwarp();  // every lane is done with buffer sc & 1 before it is restaged
    }
    if (dinit) {
#pragma unroll
        for (int rr = 0; rr < kRows; ++rr)
#pragma unroll
            for (int c = 0; c < kSliceCols; ++c) dinit[(size_t(bh) * kD + r0 + rr) * kD + c0 + c] = G[rr][c];
    }
}

// dq, dk, dg, dbeta = the sum of the slices' partials, in slice order.
__global__ void bwd_reduce_kernel(const float* __restrict__ part, float* __restrict__ dq, float* __restrict__ dk,
                                  float* __restrict__ dg, float* __restrict__ dbeta, size_t rows) {
    const size_t n4 = rows * (kD / 4);
    const float4* p4 = reinterpret_cast<const float4*>(part);
    const size_t stride = rows * (kD / 4);  // one (slice, which) plane in float4
    for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n4; i += size_t(gridDim.x) * blockDim.x) {
        float4 a[3];
#pragma unroll
        for (int w = 0; w < 3; ++w) a[w] = p4[size_t(w) * stride + i];
#pragma unroll 1
        for (int s = 1; s < kSlices; ++s) {
#pragma unroll
            for (int w = 0; w < 3; ++w) {
                const float4 x = p4[(size_t(s) * 3 + w) * stride + i];
                a[w].x += x.x; a[w].y += x.y; a[w].z += x.z; a[w].w += x.w;
            }
        }
        reinterpret_cast<float4*>(dq)[i] = a[0];
        reinterpret_cast<float4*>(dk)[i] = a[1];
        reinterpret_cast<float4*>(dg)[i] = a[2];
    }
    const float* pb = part + size_t(kSlices) * 3 * rows * kD;
    for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < rows; i += size_t(gridDim.x) * blockDim.x) {
        float acc = pb[i];
#pragma unroll 1
        for (int s = 1; s < kSlices; ++s) acc += pb[size_t(s) * rows + i];
        dbeta[i] = acc;
    }
}

}  // namespace bwd

// checkpoints [B*H][slices][ceil(T/kSub)][cols][rows] fp32, then the slices' partial sums
// [slices][3][B*T*H][128] and [slices][B*T*H] fp32
static size_t bwd_ckpt_bytes(int B, int T, int H) {
    const size_t nsub = (size_t(T) + bwd::kSub - 1) / bwd::kSub;
    return (size_t(B) * H * bwd::kSlices * nsub * bwd::kSliceCols * kD * sizeof(float) + 255) & ~size_t(255);
}

size_t recurrent_bwd_workspace_bytes(int B, int T, int H) {
    const size_t rows = size_t(B) * T * H;
    return bwd_ckpt_bytes(B, T, H) + size_t(bwd::kSlices) * (3 * kD + 1) * rows * sizeof(float);
}

int launch_recurrent_bwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
                         const float* init, const void* dout, const float* dfinal, float* dq, float* dk, float* dv,
                         float* dg, float* dbeta, float* dinit, int B, int Tn, int H, int dtype, float scale,
                         void* ws, size_t ws_bytes, cudaStream_t stream, const char** why) {
    using namespace bwd;
    const int nbh = B * H;
    if (nbh == 0) return KDA_OK;
    if (ws_bytes < recurrent_bwd_workspace_bytes(B, Tn, H) || ws == nullptr) {
        *why = "workspace smaller than kda_recurrent_bwd_workspace()";
        return KDA_ERR_WORKSPACE;
    }
    float* ckpt = static_cast<float*>(ws);
    float* part = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + bwd_ckpt_bytes(B, Tn, H));
    const dim3 grid(unsigned(nbh), unsigned(bwd::kSlices));
    if (dtype == KDA_BF16) {
        using Tb = __nv_bfloat16;
        if (!set_smem_attr(recurrent_bwd_kernel<Tb>, smem_bytes<Tb>())) {
            *why = "cudaFuncSetAttribute failed for the backward kernel";
            return KDA_ERR_CUDA;
        }
        recurrent_bwd_kernel<Tb><<<grid, bwd::kThreads, smem_bytes<Tb>(), stream>>>(
            static_cast<const Tb*>(q), static_cast<const Tb*>(k), static_cast<const Tb*>(v), g, beta, init,
            static_cast<const Tb*>(dout), dfinal, dv, dinit, part, ckpt, Tn, H, scale);
    } else {
        if (!set_smem_attr(recurrent_bwd_kernel<float>, smem_bytes<float>())) {
            *why = "cudaFuncSetAttribute failed for the backward kernel";
            return KDA_ERR_CUDA;
        }
        recurrent_bwd_kernel<float><<<grid, bwd::kThreads, smem_bytes<float>(), stream>>>(
            static_cast<const float*>(q), static_cast<const float*>(k), static_cast<const float*>(v), g, beta, init,
            static_cast<const float*>(dout), dfinal, dv, dinit, part, ckpt, Tn, H, scale);
    }
    const size_t rows = size_t(B) * Tn * H;
    const unsigned rgrid = unsigned(std::min<size_t>((rows * (kD / 4) + 255) / 256, size_t(148) * 16));
    bwd_reduce_kernel<<<rgrid, 256, 0, stream>>>(part, dq, dk, dg, dbeta, rows);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        *why = cudaGetErrorString(e);
        return KDA_ERR_CUDA;
    }
    return KDA_OK;
}

}  // namespace kda
