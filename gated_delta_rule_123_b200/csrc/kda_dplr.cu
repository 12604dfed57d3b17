// Generic (untied) DPLR chunkwise prefill on sm_100a, for comparison with KDA.
//
// The recurrence ("Kimi Linear: An Expressive, Efficient Attention
// Architecture", section "Chunkwise Algorithm": KDA is a constrained
// diagonal-plus-low-rank transition; its tied a = b = sqrt(beta) k form needs
// two gated gram matrices per chunk where the general form needs four, "the
// 4 -> 2" of the pages' kernel comparison):
//     S_t = (I - a_t b_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,
//     o_t = S_t^T (scale q_t),
// with a_t, b_t free per (token, head).  KDA is the case a = beta k, b = k.
//
// Chunk form (derived here; per chunk of C = 64 tokens, b the in-chunk
// cumulative log decay, Gamma_{rj} = exp(b_r - b_j) per channel, w_r the
// rank-1 read-out b_r^T Diag(alpha_r) S_{r-1}):
//     M_ba[r,j] = sum_c b_rc a_jc Gamma_rjc            (j < r)
//     M_bk[r,j] = beta_j sum_c b_rc k_jc Gamma_rjc     (j < r)
//     P_qa[r,j] = sum_c q_rc a_jc Gamma_rjc            (j <= r)
//     P_qk[r,j] = beta_j sum_c q_rc k_jc Gamma_rjc     (j <= r)
//     T = (I + M_ba)^{-1},  W = T (B (.) e^b) S + T M_bk V,   U~ = -W,
//     O = (Q (.) e^b) S + P_qk V + P_qa U~,
//     S' = Diag(e^{b_C}) S + (K beta (.) e^{b_C - b})^T V + (A (.) e^{b_C - b})^T U~.
// (With a = beta k, b = k this is the KDA chunk form with U~ = -W = its U~.)
//
// B200 mapping, following the KDA kernel (kda_chunk.cu): transposed tiles with
// M = 128 and the fp32 state S^T resident in TMEM; per-channel reference point
// m = (b_0 + b_63)/2 giving Bp = B e^{b-m}, Qp = Q e^{b-m}, Am = A e^{m-b},
// Kbm = K beta e^{m-b}; one N = 128 MMA [Bp;Qp] x [Am;Kbm]^T yields all four
// grams; the UT transform is the KDA one (without beta); T'' = -T M_bk on tf32
// warp MMAs; then U^T = V^T T''^T and R^T = Bp^T T^T (one MMA group),
// [U~ | O] += S'^T [-R^T | Qp], and two N = 192 MMAs [O | S] += U~^T [P_qa | Am]
// + V^T [P_qk | Kbm].  Chunks whose decay range exceeds kRangeMax compute the
// four grams on CUDA cores with one exp per term and use the references 0 and
// b_C, as in the KDA kernel.  One CTA per (sequence, head) -- no segment scan --
// and the next chunk's q, k, a, b, g are loaded once the U~/O MMA has released
// the tiles that alias them.
#include "kda_common.cuh"

namespace kda {

namespace dplr {
// Shared memory (bytes).  The raw tiles q, k, a, b, g are dead after the
// operand stage; the UT scratch, T, T'', -R^T and S' then live over them.
constexpr uint32_t RAW_Q = 0, RAW_K = 16384, RAW_A = 32768, RAW_B = 49152, RAW_G = 65536;  // g: fp32 32 KB
constexpr uint32_t S_A = 0;          // fp32 [64][64] M_ba (UT input), then -R^T (bf16 [128 k][64 tok])
constexpr uint32_t S_WN = 0;
constexpr uint32_t S_T = 16384;      // fp32 [64][64] T
constexpr uint32_t S_MBK = 32768;    // fp32 [64][64] M_bk
constexpr uint32_t S_TB = 49152;     // bf16 [64][64] T (B operand of R^T)
constexpr uint32_t S_TB2 = 57344;    // bf16 [64][64] T'' = -T M_bk (B operand of U^T)
constexpr uint32_t S_ST = 65536;     // 2 x bf16 [128 v][64 k] S'^T
constexpr uint32_t S_V = 98304;      // bf16 [64 tok][128 v] (TMA)
constexpr uint32_t S_BP = 114688;    // bf16 [128 c][64 tok] Bp
constexpr uint32_t S_QP = 131072;    // Qp ([Bp;Qp] M=128 stack; [-R^T|Qp] N=128 stack)
constexpr uint32_t S_PQA = 147456;   // bf16 [64][64] P_qa, then Am: one N=192 operand
constexpr uint32_t S_AM = 155648;
constexpr uint32_t S_PQK = 172032;   // bf16 [64][64] P_qk, then Kbm: one N=192 operand
constexpr uint32_t S_KBM = 180224;
constexpr uint32_t S_UT = 196608;    // bf16 [128 v][64 tok] U~^T, then the O tile for the TMA store
constexpr uint32_t S_MISC = 212992;
constexpr uint32_t kSmem = S_MISC + 7 * 1024;
static_assert(S_AM - S_PQA == 8192 && S_KBM - S_PQK == 8192 && kSmem <= 232448, "dplr shared memory plan");
// TMEM columns: U^T | O^T | S^T as in the KDA kernel (TM_U, TM_O, TM_S), then the
// four grams (128 columns) and R^T
constexpr uint32_t TM_G = 256, TM_R = 384;
static_assert(TM_U == 0 && TM_O == 64 && TM_S == 128, "[U|O] and [O|S] stacks");

struct Args {
    const float* beta;
    const float* init_state;
    float* final_state;
    void* o;
    const SegItem* items;
    const int* n_items;
    int H;
    float scale;
};
}  // namespace dplr

template <typename OutT>
__global__ void __launch_bounds__(kThreads, 1)
    dplr_chunk_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_a,
                      const __grid_constant__ CUtensorMap tm_b, const __grid_constant__ CUtensorMap tm_g,
                      const __grid_constant__ CUtensorMap tm_o, const dplr::Args p) {
    using namespace dplr;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = smem_raw;
    const uint32_t sbase = smem_u32(sm);
    if (sbase & 1023u) {
        if (threadIdx.x == 0) report_timeout(15);
        return;
    }
    constexpr bool kStageO = sizeof(OutT) == 2;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, part = warp >> 2;
    const int item_id = blockIdx.x, h = blockIdx.y, H = p.H;
    if (item_id >= *p.n_items) return;
    const SegItem it = p.items[item_id];

    float* sBeta2 = reinterpret_cast<float*>(sm + S_MISC);  // [2][64]
    float* sFrOp = sBeta2 + 128;                            // [128]
    float* sFrAcc = sFrOp + 128;                            // [128]
    float* sPost = sFrAcc + 128;                            // [2][128]
    float* sCarry = sPost + 256;                            // [4][128]
    uint64_t* bars = reinterpret_cast<uint64_t*>(sCarry + 512);  // raw, v, mma
    uint32_t* sTmem = reinterpret_cast<uint32_t*>(bars + 4);
    float* sA = reinterpret_cast<float*>(sm + S_A);
    float* sT = reinterpret_cast<float*>(sm + S_T);
    float* sMbk = reinterpret_cast<float*>(sm + S_MBK);
    constexpr int kLoader = 96;

    if (warp == 0) {
        tmem_alloc(sTmem, 512);
        tmem_relinquish();
    }
    if (tid == 32) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        mbar_init(&bars[2], 1);
        fence_mbar_init();
    }
    if (tid == 64) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        prefetch_tmap(&tm_a);
        prefetch_tmap(&tm_b);
        prefetch_tmap(&tm_g);
    }
    if (tid < 128) sPost[128 + tid] = 1.f;
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *sTmem;
    const uint32_t lane_off = uint32_t(quad * 32) << 16;
    const int vrow = quad * 32 + lane;
    const int t_begin = it.tok_begin, t_end = it.tok_end;
    const int nchunks = (t_end - t_begin + kC - 1) / kC;

    auto issue_raw = [&](int c) {
        const int t0 = t_begin + c * kC;
        mbar_arrive_expect_tx(&bars[0], 4 * 16384u + 32768u);
        tma_load_3d(sm + RAW_Q, &tm_q, &bars[0], 0, h, t0);
        tma_load_3d(sm + RAW_Q + 8192, &tm_q, &bars[0], 64, h, t0);
        tma_load_3d(sm + RAW_K, &tm_k, &bars[0], 0, h, t0);
        tma_load_3d(sm + RAW_K + 8192, &tm_k, &bars[0], 64, h, t0);
        tma_load_3d(sm + RAW_A, &tm_a, &bars[0], 0, h, t0);
        tma_load_3d(sm + RAW_A + 8192, &tm_a, &bars[0], 64, h, t0);
        tma_load_3d(sm + RAW_B, &tm_b, &bars[0], 0, h, t0);
        tma_load_3d(sm + RAW_B + 8192, &tm_b, &bars[0], 64, h, t0);
        tma_load_3d(sm + RAW_G, &tm_g, &bars[0], 0, h, t0);
    };
    auto issue_v = [&](int c) {
        const int t0 = t_begin + c * kC;
        mbar_arrive_expect_tx(&bars[1], 16384u);
        tma_load_3d(sm + S_V, &tm_v, &bars[1], 0, h, t0);
        tma_load_3d(sm + S_V + 8192, &tm_v, &bars[1], 64, h, t0);
    };
    bool pend_raw = false, pend_v = false;
    if (tid == kLoader && nchunks > 0) {
        issue_raw(0);
        issue_v(0);
        pend_raw = pend_v = true;
    }
    {  // start state into TMEM (S^T: lane = v, column = k)
        const float* src = p.init_state ? p.init_state + (size_t(it.seq) * H + h) * (kD * kD) : nullptr;
#pragma unroll 1
        for (int cb = 0; cb < 2; ++cb) {
            float buf[16];
            const int k0 = part * 32 + cb * 16;
#pragma unroll
            for (int j = 0; j < 16; ++j) buf[j] = src ? src[size_t(k0 + j) * kD + vrow] : 0.f;
            tmem_st16(tbase + TM_S + lane_off + k0, buf);
        }
        tmem_wait_st();
    }
    uint32_t ph_raw = 0, ph_v = 0, ph_mma = 0;
    bool aborted = false;
    auto fetch_beta = [&](int cc) {
        const int tn = t_begin + cc * kC + tid;
        const bool valid = cc < nchunks && tn < t_end;
        cp_async4(sBeta2 + (cc & 1) * 64 + tid, p.beta + (valid ? size_t(tn) * H + h : 0), valid ? 4u : 0u);
    };
    if (tid < 64) fetch_beta(0);
    const uint32_t id_g = idesc_bf16(128, 128, 1, 1);    // [Bp;Qp] (MN) x [Am;Kbm] (MN)
    const uint32_t id_r = idesc_bf16(128, 64, 0, 0);     // Bp^T (K) x T^T (K)
    const uint32_t id_u = idesc_bf16(128, 64, 1, 0);     // V^T (MN) x T''^T (K)
    const uint32_t id_so2 = idesc_bf16(128, 128, 0, 1);  // S'^T (K) x [-R^T | Qp] (MN)
    const uint32_t id_os = idesc_bf16(128, 192, 0, 0);   // U~^T (K) x [P_qa | Am] (K)
    const uint32_t id_vs = idesc_bf16(128, 192, 1, 0);   // V^T (MN) x [P_qk | Kbm] (K)
    // T, T'' strictly-upper 16x16 blocks are zero: one 16-byte chunk per thread < 192 for each
    uint32_t tb_zero = 0;
    if (tid < 192) {
        const int I = tid < 96 ? 0 : (tid < 160 ? 1 : 2);
        const int e0 = tid - (I == 0 ? 0 : (I == 1 ? 96 : 160)), per = 6 - 2 * I;
        tb_zero = sw128_chunk(16 * I + e0 / per, 2 * (I + 1) + e0 % per);
    }
    const int ch = tid & 127, rq = tid >> 7;

#pragma unroll 1
    for (int c = 0; c < nchunks; ++c) {
        const int t0 = t_begin + c * kC;
        const int len = min(kC, t_end - t0);
        const int cur = c & 1, prev = cur ^ 1;
        const float* sBeta = sBeta2 + cur * 64;

        // ===== operands =====
        bool ok = mbar_wait(&bars[0], ph_raw, 1);
        ph_raw ^= 1;
        if (tid == kLoader) pend_raw = false;
        if (__syncthreads_or(!ok)) { aborted = true; break; }
        if (len < kC) {  // rows past the end: g = q = k = a = b = 0
            for (int e = tid; e < (kC - len) * 32; e += kThreads) {
                const int r = len + (e >> 5), w = e & 31;
                reinterpret_cast<float4*>(sm + RAW_G)[r * 32 + w] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (w < 16) {
                    const uint32_t off = (w >> 3) * 8192 + r * 128 + (w & 7) * 16;
                    st_shared_v4(sbase + RAW_Q + off, 0u, 0u, 0u, 0u);
                    st_shared_v4(sbase + RAW_K + off, 0u, 0u, 0u, 0u);
                    st_shared_v4(sbase + RAW_A + off, 0u, 0u, 0u, 0u);
                    st_shared_v4(sbase + RAW_B + off, 0u, 0u, 0u, 0u);
                }
            }
            __syncthreads();
        }
        float bl[16];
        {
            const float* sG = reinterpret_cast<const float*>(sm + RAW_G);
            float acc = 0.f;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                acc += fmaxf(sG[(rq * 16 + j) * kD + ch], kGateFloor);
                bl[j] = acc;
            }
            sCarry[rq * 128 + ch] = acc;
        }
        if (tid < 64) {
            cp_async_wait_all();
            fetch_beta(c + 1);
        }
        const float b0 = fmaxf(reinterpret_cast<const float*>(sm + RAW_G)[ch], kGateFloor);
        __syncthreads();
        float carry = 0.f, bC = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float cq = sCarry[q * 128 + ch];
            carry += (q < rq) ? cq : 0.f;
            bC += cq;
        }
        const bool fast = __syncthreads_and((b0 - bC) <= kRangeMax) != 0;
        const float m = 0.5f * (b0 + bC);
        const float mp = fast ? m : 0.f, mk = fast ? m : bC;
        {
            const uint32_t box = uint32_t(ch >> 6) * 8192u;
            const float y0 = (carry - mp) * kLog2e, y1 = (mk - carry) * kLog2e;
#pragma unroll
            for (int jj = 0; jj < 16; jj += 8) {
                uint32_t pb[4], pq[4], pa[4], pk[4];
#pragma unroll
                for (int e = 0; e < 8; e += 2) {
                    float bv[2], qv[2], av[2], kv[2];
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const int j = jj + e + u, r = rq * 16 + j;
                        const uint32_t off = box + sw128_off(r, ch & 63);
                        const float e1 = ex2_approx(fmaf(bl[j], kLog2e, y0));   // e^{b - mp}
                        const float e2 = ex2_approx(fmaf(bl[j], -kLog2e, y1));  // e^{mk - b}
                        bv[u] = bf16_at(sm + RAW_B, off) * e1;
                        qv[u] = bf16_at(sm + RAW_Q, off) * p.scale * e1;
                        av[u] = bf16_at(sm + RAW_A, off) * e2;
                        kv[u] = bf16_at(sm + RAW_K, off) * sBeta[r] * e2;
                    }
                    pb[e >> 1] = pack_bf16x2(bv[0], bv[1]);
                    pq[e >> 1] = pack_bf16x2(qv[0], qv[1]);
                    pa[e >> 1] = pack_bf16x2(av[0], av[1]);
                    pk[e >> 1] = pack_bf16x2(kv[0], kv[1]);
                }
                const int j8 = (rq * 16 + jj) >> 3;
                st_shared_v4(sbase + S_BP + sw128_chunk(ch, j8), pb[0], pb[1], pb[2], pb[3]);
                st_shared_v4(sbase + S_QP + sw128_chunk(ch, j8), pq[0], pq[1], pq[2], pq[3]);
                st_shared_v4(sbase + S_AM + sw128_chunk(ch, j8), pa[0], pa[1], pa[2], pa[3]);
                st_shared_v4(sbase + S_KBM + sw128_chunk(ch, j8), pk[0], pk[1], pk[2], pk[3]);
            }
            if (tid < 128) {
                const float postp = sPost[prev * 128 + ch];
                sFrOp[ch] = postp * ex2_approx(mp * kLog2e);
                sFrAcc[ch] = postp * ex2_approx(mk * kLog2e);
                sPost[cur * 128 + ch] = ex2_approx((bC - mk) * kLog2e);
            }
        }
        fence_async_smem();

        // ===== exact grams (CUDA cores) for a wide chunk, before anything overwrites the raw tiles =====
        if (!fast) {
            constexpr int kPairs = 64 * 65 / 2, kPer = (kPairs + kThreads - 1) / kThreads;
            float gba[kPer], gbk[kPer], gqa[kPer], gqk[kPer];
            float* sB = reinterpret_cast<float*>(sm + RAW_G);
            __syncthreads();  // every thread has read g
#pragma unroll
            for (int j = 0; j < 16; ++j) sB[(rq * 16 + j) * kD + ch] = bl[j] + carry;
            __syncthreads();
#pragma unroll
            for (int u = 0; u < kPer; ++u) {
                const int pidx = tid + u * kThreads;
                gba[u] = gbk[u] = gqa[u] = gqk[u] = 0.f;
                if (pidx >= kPairs) continue;
                int r = int((sqrtf(8.f * pidx + 1.f) - 1.f) * 0.5f);
                while (r * (r + 1) / 2 > pidx) --r;
                while ((r + 1) * (r + 2) / 2 <= pidx) ++r;
                const int j = pidx - r * (r + 1) / 2;
                if (r >= len) continue;
                for (int cc = 0; cc < kD; ++cc) {
                    const float f = __expf(sB[r * kD + cc] - sB[j * kD + cc]);
                    const uint32_t offr = uint32_t(cc >> 6) * 8192u + sw128_off(r, cc & 63);
                    const uint32_t offj = uint32_t(cc >> 6) * 8192u + sw128_off(j, cc & 63);
                    const float aj = bf16_at(sm + RAW_A, offj) * f, kj = bf16_at(sm + RAW_K, offj) * f;
                    const float br = bf16_at(sm + RAW_B, offr), qr = bf16_at(sm + RAW_Q, offr);
                    gba[u] += br * aj;
                    gbk[u] += br * kj;
                    gqa[u] += qr * aj;
                    gqk[u] += qr * kj;
                }
            }
            __syncthreads();  // the raw tiles are read: the grams go over them
            for (int e = tid; e < 64 * 64; e += kThreads) {
                sA[e] = 0.f;
                sMbk[e] = 0.f;
            }
            for (int e = tid; e < 512; e += kThreads) {
                st_shared_v4(sbase + S_PQA + e * 16, 0u, 0u, 0u, 0u);
                st_shared_v4(sbase + S_PQK + e * 16, 0u, 0u, 0u, 0u);
            }
            __syncthreads();
#pragma unroll
            for (int u = 0; u < kPer; ++u) {
                const int pidx = tid + u * kThreads;
                if (pidx >= kPairs) continue;
                int r = int((sqrtf(8.f * pidx + 1.f) - 1.f) * 0.5f);
                while (r * (r + 1) / 2 > pidx) --r;
                while ((r + 1) * (r + 2) / 2 <= pidx) ++r;
                const int j = pidx - r * (r + 1) / 2;
                if (j < r) {
                    sA[((r >> 4) == (j >> 4)) ? sidx(j, r) : sidx(r, j)] = gba[u];
                    sMbk[sidx(r, j)] = sBeta[j] * gbk[u];
                }
                *reinterpret_cast<__nv_bfloat16*>(sm + S_PQA + sw128_off(r, j)) = __float2bfloat16_rn(gqa[u] * p.scale);
                *reinterpret_cast<__nv_bfloat16*>(sm + S_PQK + sw128_off(r, j)) =
                    __float2bfloat16_rn(gqk[u] * p.scale * sBeta[j]);
            }
        }
        __syncthreads();  // raw tiles read; operands, frame factors (and exact grams) visible

        // ===== gram MMA (fast) overlapped with the state frame pass =====
        if (fast && tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint64_t a = sdesc_sw128(sbase + S_BP + ks * 2048, S_QP - S_BP, 1024);
                const uint64_t b = sdesc_sw128(sbase + S_AM + ks * 2048, S_KBM - S_AM, 1024);
                umma_bf16(tbase + TM_G, a, b, id_g, ks > 0);
            }
            umma_commit(&bars[2]);
        }
        {  // S <- S * post(prev); bf16 operand S' = S e^{mp}; TMEM S = S e^{mk}; O^T = 0
            float x[32];
#pragma unroll
            for (int cb = 0; cb < 2; ++cb) tmem_ld16(tbase + TM_S + lane_off + part * 32 + cb * 16, x + cb * 16);
            tmem_wait_ld();
            const uint32_t dst = sbase + S_ST + ((part >> 1) ? 16384u : 0u);
#pragma unroll
            for (int cb = 0; cb < 2; ++cb) {
                const int k0 = part * 32 + cb * 16, ck = (part & 1) * 4 + cb * 2;
                uint32_t pk[8];
#pragma unroll
                for (int j = 0; j < 16; j += 4) {
                    const float4 fo = *reinterpret_cast<const float4*>(sFrOp + k0 + j);
                    const float4 fa = *reinterpret_cast<const float4*>(sFrAcc + k0 + j);
                    float* xx = x + cb * 16 + j;
                    pk[j >> 1] = pack_bf16x2(xx[0] * fo.x, xx[1] * fo.y);
                    pk[(j >> 1) + 1] = pack_bf16x2(xx[2] * fo.z, xx[3] * fo.w);
                    xx[0] *= fa.x;
                    xx[1] *= fa.y;
                    xx[2] *= fa.z;
                    xx[3] *= fa.w;
                }
                st_shared_v4(dst + sw128_chunk(vrow, ck), pk[0], pk[1], pk[2], pk[3]);
                st_shared_v4(dst + sw128_chunk(vrow, ck + 1), pk[4], pk[5], pk[6], pk[7]);
            }
#pragma unroll
            for (int cb = 0; cb < 2; ++cb) tmem_st16(tbase + TM_S + lane_off + part * 32 + cb * 16, x + cb * 16);
            float z[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) z[j] = 0.f;
            tmem_st16(tbase + TM_O + lane_off + part * 16, z);
            tmem_wait_st();
        }
        if (tid == 0) bulk_wait_read0();  // the previous O tile (over U~^T) is read out
        if (fast) {
            ok = mbar_wait(&bars[2], ph_mma, 2);
            ph_mma ^= 1;
            tc_fence_after();
            if (__syncthreads_or(!ok)) { aborted = true; break; }
            // lanes 0..63: Bp rows -> M_ba (cols 0..63), M_bk (cols 64..127);
            // lanes 64..127: Qp rows -> P_qa, P_qk.  Thread part p reads columns [32p, 32p+32).
            float vals[32];
            tmem_ld16(tbase + TM_G + lane_off + part * 32, vals);
            tmem_ld16(tbase + TM_G + lane_off + part * 32 + 16, vals + 16);
            tmem_wait_ld();
            const int cb0 = (part & 1) * 32;  // first column inside its 64-column gram
            if (vrow < 64) {
                if (part < 2) {  // M_ba, strictly lower; the diagonal 16x16 block stored transposed
#pragma unroll
                    for (int j = 0; j < 32; j += 4) {
                        const int i = cb0 + j;
                        if ((i >> 4) == (vrow >> 4)) {
#pragma unroll
                            for (int u = 0; u < 4; ++u) sA[sidx(i + u, vrow)] = (i + u < vrow) ? vals[j + u] : 0.f;
                        } else {
                            float4 w4;
                            w4.x = (i + 0 < vrow) ? vals[j + 0] : 0.f;
                            w4.y = (i + 1 < vrow) ? vals[j + 1] : 0.f;
                            w4.z = (i + 2 < vrow) ? vals[j + 2] : 0.f;
                            w4.w = (i + 3 < vrow) ? vals[j + 3] : 0.f;
                            *reinterpret_cast<float4*>(&sA[sidx(vrow, i)]) = w4;
                        }
                    }
                } else {  // M_bk, strictly lower
#pragma unroll
                    for (int j = 0; j < 32; j += 4) {
                        const int i = cb0 + j;
                        float4 w4;
                        w4.x = (i + 0 < vrow) ? vals[j + 0] : 0.f;
                        w4.y = (i + 1 < vrow) ? vals[j + 1] : 0.f;
                        w4.z = (i + 2 < vrow) ? vals[j + 2] : 0.f;
                        w4.w = (i + 3 < vrow) ? vals[j + 3] : 0.f;
                        *reinterpret_cast<float4*>(&sMbk[sidx(vrow, i)]) = w4;
                    }
                }
            } else {  // P_qa / P_qk (lower incl. diagonal), bf16 [64 r][64 j]
                const int r = vrow - 64;
                const uint32_t dstp = sbase + (part < 2 ? S_PQA : S_PQK);
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    uint32_t w[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int i0 = cb0 + q4 * 8 + 2 * u;
                        w[u] = pack_bf16x2(i0 <= r ? vals[q4 * 8 + 2 * u] : 0.f,
                                           i0 + 1 <= r ? vals[q4 * 8 + 2 * u + 1] : 0.f);
                    }
                    st_shared_v4(dstp + sw128_chunk(r, (cb0 >> 3) + q4), w[0], w[1], w[2], w[3]);
                }
            }
        }
        __syncthreads();

        // ===== UT transform: T = (I + M_ba)^{-1} (as in the KDA kernel, without beta) =====
        if (warp < 4 && lane < 16) {
            const int base = 16 * warp, jc = lane;
            const float4* at4 = reinterpret_cast<const float4*>(sA);
            float4 win[3][4];
            auto ld_row = [&](float4* dst, const int r) {
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    if (4 * q + 3 > r) dst[q] = at4[sidx(base + r, base + 4 * q) >> 2];
            };
            ld_row(win[0], 0);
            ld_row(win[1], 1);
            float ps[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) ps[r] = (r == jc) ? 1.f : 0.f;
#pragma unroll
            for (int r = 0; r < 15; ++r) {
                if (r + 2 < 15) ld_row(win[(r + 2) % 3], r + 2);
                const float tr = ps[r];
                const float4* w = win[r % 3];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    if (4 * q + 0 > r) ps[4 * q + 0] = fmaf(-w[q].x, tr, ps[4 * q + 0]);
                    if (4 * q + 1 > r) ps[4 * q + 1] = fmaf(-w[q].y, tr, ps[4 * q + 1]);
                    if (4 * q + 2 > r) ps[4 * q + 2] = fmaf(-w[q].z, tr, ps[4 * q + 2]);
                    if (4 * q + 3 > r) ps[4 * q + 3] = fmaf(-w[q].w, tr, ps[4 * q + 3]);
                }
            }
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                sT[sidx(base + r, base + jc)] = ps[r];
                *reinterpret_cast<uint16_t*>(sm + S_TB + sw128_off(base + r, base + jc)) =
                    uint16_t((__float_as_uint(ps[r]) + 0x8000u) >> 16);
            }
        }
        if (tid < 192) {  // strictly-upper blocks of T and T''
            st_shared_v4(sbase + S_TB + tb_zero, 0u, 0u, 0u, 0u);
            st_shared_v4(sbase + S_TB2 + tb_zero, 0u, 0u, 0u, 0u);
        }
        __syncthreads();
        const int gq = lane >> 2, tq = lane & 3;
        // y (16x16 in two fragments) += L (16x16 at (lr0, lk0) of srcL) x R (16x16 at (rk0, rn0) of srcR)
        auto mm16 = [&](float* y, const float* srcL, int lr0, int lk0, const float* srcR, int rk0, int rn0) {
#pragma unroll
            for (int kc = 0; kc < 16; kc += 8) {
                const uint32_t a0 = f32_to_tf32(srcL[sidx(lr0 + gq, lk0 + kc + tq)]);
                const uint32_t a1 = f32_to_tf32(srcL[sidx(lr0 + gq + 8, lk0 + kc + tq)]);
                const uint32_t a2 = f32_to_tf32(srcL[sidx(lr0 + gq, lk0 + kc + tq + 4)]);
                const uint32_t a3 = f32_to_tf32(srcL[sidx(lr0 + gq + 8, lk0 + kc + tq + 4)]);
#pragma unroll
                for (int nb = 0; nb < 2; ++nb)
                    mma_tf32_16x8x8(y + nb * 4, a0, a1, a2, a3,
                                    f32_to_tf32(srcR[sidx(rk0 + kc + tq, rn0 + nb * 8 + gq)]),
                                    f32_to_tf32(srcR[sidx(rk0 + kc + tq + 4, rn0 + nb * 8 + gq)]));
            }
        };
        // acc (16x8) += y (registers) x sT rows [rk0, rk0+16), columns [rn0, rn0+8) (k-paired order)
        auto mm_reg = [&](float* acc, const float* y, int rk0, int rn0) {
#pragma unroll
            for (int nb = 0; nb < 2; ++nb)
                mma_tf32_16x8x8(acc, f32_to_tf32(y[nb * 4 + 0]), f32_to_tf32(y[nb * 4 + 2]), f32_to_tf32(y[nb * 4 + 1]),
                                f32_to_tf32(y[nb * 4 + 3]), f32_to_tf32(sT[sidx(rk0 + nb * 8 + 2 * tq, rn0 + gq)]),
                                f32_to_tf32(sT[sidx(rk0 + nb * 8 + 2 * tq + 1, rn0 + gq)]));
        };
        auto put_t = [&](int r0, int c0, const float* acc) {  // T block piece = -acc (fp32 and bf16)
            const int cc = c0 + 2 * tq;
            sT[sidx(r0 + gq, cc)] = -acc[0];
            sT[sidx(r0 + gq, cc + 1)] = -acc[1];
            sT[sidx(r0 + gq + 8, cc)] = -acc[2];
            sT[sidx(r0 + gq + 8, cc + 1)] = -acc[3];
            *reinterpret_cast<uint32_t*>(sm + S_TB + sw128_off(r0 + gq, cc)) = pack_bf16x2(-acc[0], -acc[1]);
            *reinterpret_cast<uint32_t*>(sm + S_TB + sw128_off(r0 + gq + 8, cc)) = pack_bf16x2(-acc[2], -acc[3]);
        };
        if (warp < 6) {  // T_IJ = -(D_I A_IJ) D_J, (I, J) = (1,0), (2,1), (3,2)
            const int J = warp >> 1, I = J + 1, cn = 16 * J + 8 * (warp & 1);
            float y[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            mm16(y, sT, 16 * I, 16 * I, sA, 16 * I, 16 * J);
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            mm_reg(acc, y, 16 * J, cn);
            put_t(16 * I, cn, acc);
        }
        __syncthreads();
        if (warp < 6) {  // T_20, T_31, T_30 as in the KDA kernel
            const int task = warp >> 1, cn = 8 * (warp & 1);
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            float z0[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            float z1[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            if (task == 0) {
                mm16(z0, sT, 32, 32, sA, 32, 0);
                mm16(z1, sT, 32, 32, sA, 32, 16);
                mm_reg(acc, z0, 0, cn);
                mm_reg(acc, z1, 16, cn);
                put_t(32, cn, acc);
            } else if (task == 1) {
                mm16(z1, sT, 48, 32, sA, 32, 16);
                mm16(z1, sT, 48, 48, sA, 48, 16);
                mm_reg(acc, z1, 16, 16 + cn);
                put_t(48, 16 + cn, acc);
            } else {
                mm16(z0, sT, 48, 32, sA, 32, 0);
                mm16(z1, sT, 48, 32, sA, 32, 16);
                mm16(z0, sT, 48, 48, sA, 48, 0);
                mm16(z1, sT, 48, 48, sA, 48, 16);
                mm_reg(acc, z0, 0, cn);
                mm_reg(acc, z1, 16, cn);
                put_t(48, cn, acc);
            }
        }
        __syncthreads();
        // ===== T'' = -T M_bk (lower triangular), bf16: warp = (row block I, column block J <= I) =====
        if (warp < 10) {
            // warps 0..9 -> (I, J) = (0,0) (1,0) (1,1) (2,0) (2,1) (2,2) (3,0) (3,1) (3,2) (3,3)
            const int I = warp < 1 ? 0 : (warp < 3 ? 1 : (warp < 6 ? 2 : 3));
            const int J = warp - (I * (I + 1)) / 2;
            float y[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            for (int L = J; L <= I; ++L) mm16(y, sT, 16 * I, 16 * L, sMbk, 16 * L, 16 * J);
#pragma unroll
            for (int nb = 0; nb < 2; ++nb) {
                const int cc = 16 * J + nb * 8 + 2 * tq;
                *reinterpret_cast<uint32_t*>(sm + S_TB2 + sw128_off(16 * I + gq, cc)) =
                    pack_bf16x2(-y[nb * 4 + 0], -y[nb * 4 + 1]);
                *reinterpret_cast<uint32_t*>(sm + S_TB2 + sw128_off(16 * I + gq + 8, cc)) =
                    pack_bf16x2(-y[nb * 4 + 2], -y[nb * 4 + 3]);
            }
        }
        fence_async_smem();
        ok = mbar_wait(&bars[1], ph_v, 3);
        ph_v ^= 1;
        if (tid == kLoader) pend_v = false;
        if (__syncthreads_or(!ok)) { aborted = true; break; }

        // ===== R^T = Bp^T T^T, U^T = V^T T''^T =====
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                umma_bf16(tbase + TM_R, sdesc_sw128(sbase + S_BP + ks * 32, 16, 1024),
                          sdesc_sw128(sbase + S_TB + ks * 32, 16, 1024), id_r, ks > 0);
                umma_bf16(tbase + TM_U, sdesc_sw128(sbase + S_V + ks * 2048, 8192, 1024),
                          sdesc_sw128(sbase + S_TB2 + ks * 32, 16, 1024), id_u, ks > 0);
            }
            umma_commit(&bars[2]);
        }
        ok = mbar_wait(&bars[2], ph_mma, 4);
        ph_mma ^= 1;
        tc_fence_after();
        if (__syncthreads_or(!ok)) { aborted = true; break; }
        {  // -R^T -> smem (over the dead M_ba scratch)
            float w[16];
            tmem_ld16(tbase + TM_R + lane_off + part * 16, w);
            tmem_wait_ld();
#pragma unroll
            for (int q4 = 0; q4 < 2; ++q4)
                st_shared_v4(sbase + S_WN + sw128_chunk(vrow, part * 2 + q4),
                             pack_bf16x2(-w[q4 * 8 + 0], -w[q4 * 8 + 1]), pack_bf16x2(-w[q4 * 8 + 2], -w[q4 * 8 + 3]),
                             pack_bf16x2(-w[q4 * 8 + 4], -w[q4 * 8 + 5]), pack_bf16x2(-w[q4 * 8 + 6], -w[q4 * 8 + 7]));
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();

        // ===== [U~ | O] += S'^T [-R^T | Qp] =====
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint64_t a = sdesc_sw128(sbase + S_ST + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
                umma_bf16(tbase + TM_U, a, sdesc_sw128(sbase + S_WN + ks * 2048, S_QP - S_WN, 1024), id_so2, 1);
            }
            umma_commit(&bars[2]);
        }
        ok = mbar_wait(&bars[2], ph_mma, 5);
        ph_mma ^= 1;
        tc_fence_after();
        if (__syncthreads_or(!ok)) { aborted = true; break; }
        if (tid == kLoader && c + 1 < nchunks) {  // the raw tiles and everything over them are free
            issue_raw(c + 1);
            pend_raw = true;
        }
        {  // U~^T -> smem
            float u[16];
            tmem_ld16(tbase + TM_U + lane_off + part * 16, u);
            tmem_wait_ld();
#pragma unroll
            for (int q4 = 0; q4 < 2; ++q4)
                st_shared_v4(sbase + S_UT + sw128_chunk(vrow, part * 2 + q4),
                             pack_bf16x2(u[q4 * 8 + 0], u[q4 * 8 + 1]), pack_bf16x2(u[q4 * 8 + 2], u[q4 * 8 + 3]),
                             pack_bf16x2(u[q4 * 8 + 4], u[q4 * 8 + 5]), pack_bf16x2(u[q4 * 8 + 6], u[q4 * 8 + 7]));
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();

        // ===== [O | S] += U~^T [P_qa | Am] + V^T [P_qk | Kbm] =====
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                umma_bf16(tbase + TM_O, sdesc_sw128(sbase + S_UT + ks * 32, 16, 1024),
                          sdesc_sw128(sbase + S_PQA + ks * 32, 16, 1024), id_os, 1);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                umma_bf16(tbase + TM_O, sdesc_sw128(sbase + S_V + ks * 2048, 8192, 1024),
                          sdesc_sw128(sbase + S_PQK + ks * 32, 16, 1024), id_vs, 1);
            umma_commit(&bars[2]);
        }
        ok = mbar_wait(&bars[2], ph_mma, 6);
        ph_mma ^= 1;
        tc_fence_after();
        if (__syncthreads_or(!ok)) { aborted = true; break; }
        if (tid == kLoader && c + 1 < nchunks) {  // V of this chunk is consumed
            issue_v(c + 1);
            pend_v = true;
        }
        bool staged = false;
        {  // O^T -> o[t0 + r, h, v]
            float ov[16];
            tmem_ld16(tbase + TM_O + lane_off + part * 16, ov);
            tmem_wait_ld();
            if (kStageO && len == kC) {
                uint8_t* so = sm + S_UT + (vrow >> 6) * 8192;
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    *reinterpret_cast<__nv_bfloat16*>(so + sw128_off(part * 16 + j, vrow & 63)) =
                        __float2bfloat16_rn(ov[j]);
                fence_async_smem();
                staged = true;
            } else {
                OutT* o = static_cast<OutT*>(p.o);
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int r = part * 16 + j;
                    if (r < len) o[(size_t(t0 + r) * H + h) * kD + vrow] = from_f32<OutT>(ov[j]);
                }
            }
        }
        tc_fence_before();
        __syncthreads();
        if (staged && tid == 0) {
            tma_store_3d(&tm_o, sm + S_UT, 0, h, t0);
            tma_store_3d(&tm_o, sm + S_UT + 8192, 64, h, t0);
            bulk_commit();
        }
    }

    if (!aborted) {
        const int last = (nchunks - 1) & 1;
        float* dstS = p.final_state ? p.final_state + (size_t(it.seq) * H + h) * (kD * kD) : nullptr;
        tc_fence_after();
        if (dstS) {
#pragma unroll 1
            for (int cb = 0; cb < 2; ++cb) {
                const int k0 = part * 32 + cb * 16;
                float x[16];
                tmem_ld16(tbase + TM_S + lane_off + k0, x);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j)
                    dstS[size_t(k0 + j) * kD + vrow] = x[j] * (nchunks > 0 ? sPost[last * 128 + k0 + j] : 1.f);
            }
        }
    } else {
        if (tid == kLoader) {
            if (pend_raw) mbar_wait(&bars[0], ph_raw, 7);
            if (pend_v) mbar_wait(&bars[1], ph_v, 7);
        }
        if (tid == 0) mbar_wait(&bars[2], ph_mma, 7);
    }
    if (tid == 0) bulk_wait0();
    if (tid < 64) cp_async_wait_all();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, 512);
}

template <typename O>
static cudaError_t dplr_smem_attr() {
    return set_smem_attr(dplr_chunk_kernel<O>, dplr::kSmem) ? cudaSuccess : cudaErrorInvalidValue;
}

size_t dplr_workspace_bytes(int B, int T, int H, int num_seqs, int dtype) {
    const long long N = num_seqs > 0 ? num_seqs : B, Ttot = num_seqs > 0 ? T : (long long)B * T;
    size_t off = up256(size_t(N) * sizeof(SegItem)) + 256;  // items + count
    if (dtype == KDA_FP32) off += 5 * up256(size_t(Ttot) * H * kD * 2);  // bf16 copies of q, k, v, a, b
    return off;
}

int launch_dplr_chunk_fwd(const void* q, const void* k, const void* v, const void* a, const void* b, const float* g,
                          const float* beta, const float* init, float* fin, void* o, const int32_t* cu, int num_seqs,
                          int B, int T, int H, int dtype, float scale, void* ws, size_t ws_bytes, cudaStream_t stream,
                          const char** why) {
    const int N = cu ? num_seqs : B;
    const long long Ttot = cu ? T : (long long)B * T;
    if (ws_bytes < dplr_workspace_bytes(B, T, H, cu ? num_seqs : 0, dtype) || ws == nullptr) {
        *why = "workspace smaller than kda_dplr_chunk_fwd_workspace()";
        return KDA_ERR_WORKSPACE;
    }
    if (N == 0 || H == 0) return KDA_OK;
    uint8_t* w = static_cast<uint8_t*>(ws);
    SegItem* items = reinterpret_cast<SegItem*>(w);
    int* n_items = reinterpret_cast<int*>(w + up256(size_t(N) * sizeof(SegItem)));
    size_t off = up256(size_t(N) * sizeof(SegItem)) + 256;
    const void* in[5] = {q, k, v, a, b};
    if (dtype == KDA_FP32) {
        const long long rows = Ttot * H;
        for (int i = 0; i < 5; ++i) {
            __nv_bfloat16* d = reinterpret_cast<__nv_bfloat16*>(w + off);
            off += up256(size_t(rows) * kD * 2);
            if (rows > 0)
                prep_rows_kernel<float><<<unsigned((rows + 7) / 8), 256, 0, stream>>>(static_cast<const float*>(in[i]),
                                                                                      d, rows, 0);
            in[i] = d;
        }
    }
    CUtensorMap mq, mk, mv, ma, mb, mg, mo;
    const long long Tmap = Ttot > 0 ? Ttot : 1;
    if (!make_map(&mq, in[0], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, H, Tmap, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mk, in[1], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, H, Tmap, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mv, in[2], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, H, Tmap, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&ma, in[3], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, H, Tmap, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mb, in[4], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, H, Tmap, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mg, g, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, H, Tmap, 128, CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map(&mo, dtype == KDA_FP32 ? in[2] : o, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, H, Tmap, 64,
                  CU_TENSOR_MAP_SWIZZLE_128B)) {
        *why = "cuTensorMapEncodeTiled failed";
        return KDA_ERR_CUDA;
    }
    // one segment per sequence
    plan_kernel<<<1, 1024, 0, stream>>>(cu, N, T, 1 << 24, items, n_items, N, 1 << 24, nullptr);
    dplr::Args p{};
    p.beta = beta;
    p.init_state = init;
    p.final_state = fin;
    p.o = o;
    p.items = items;
    p.n_items = n_items;
    p.H = H;
    p.scale = scale;
    const dim3 grid(static_cast<unsigned>(N), static_cast<unsigned>(H));
    if (dtype == KDA_FP32) {
        if (dplr_smem_attr<float>() != cudaSuccess) return KDA_ERR_CUDA;
        dplr_chunk_kernel<float><<<grid, kThreads, dplr::kSmem, stream>>>(mq, mk, mv, ma, mb, mg, mo, p);
    } else {
        if (dplr_smem_attr<__nv_bfloat16>() != cudaSuccess) return KDA_ERR_CUDA;
        dplr_chunk_kernel<__nv_bfloat16><<<grid, kThreads, dplr::kSmem, stream>>>(mq, mk, mv, ma, mb, mg, mo, p);
    }
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        *why = cudaGetErrorString(e);
        return KDA_ERR_CUDA;
    }
    return KDA_OK;
}

}  // namespace kda
