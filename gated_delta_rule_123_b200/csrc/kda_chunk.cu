// KDA chunkwise prefill on sm_100a: TMA-fed tcgen05 tiles, fp32 state in TMEM.
//
// The method ("Kimi Linear: An Expressive, Efficient Attention Architecture",
// section "Chunkwise Algorithm"; the news rewrite "Kimi Linear", section on the
// hardware-efficient chunkwise algorithm): split every sequence into chunks of
// C = 64 tokens; inside a chunk unroll the per-channel decay and the rank-1
// corrections (WY representation), invert the unit lower-triangular system by
// forward substitution (UT transform), and carry only the 128x128 state from
// chunk to chunk.  Per chunk, with b the in-chunk cumulative log decay
// (gamma^{i->j} = prod_{k=i+1}^{j} alpha^k, the corrected definition from the
// section "Mathematical Rigor"):
//     A[r,i] = beta_r sum_c k_rc k_ic exp(b_rc - b_ic)      (i < r)
//     P[r,i] =        sum_c q_rc k_ic exp(b_rc - b_ic)      (i <= r)
//     T = (I + A)^{-1}
//     W = T diag(beta) (K (.) e^b),   U = T diag(beta) V     (one T for both:
//                                      the a = b = sqrt(beta) k binding)
//     U~ = U - W S,   O = (Q (.) e^b) S + P U~,
//     S' = Diag(e^{b_C}) S + (K (.) e^{b_C - b})^T U~.
//
// B200 design (what differs from the pages' GPU design):
//  * Everything is computed transposed so that every tensor-core tile has
//    M = 128 (one TMEM lane per key or value channel): S^T lives in TMEM as the
//    fp32 accumulator (lane = value channel, column = key channel) for the
//    whole sequence segment; one thread per lane owns its row.
//  * The gated operands are formed ONCE per chunk from a per-channel reference
//    point m_c = (b_0c + b_63c)/2: Kp = K (.) e^{b-m}, Qp = Q (.) e^{b-m},
//    Km = K (.) e^{m-b}.  Then A = diag(beta) Kp Km^T and P = Qp Km^T (one
//    stacked M=128 MMA), W S = (T beta Kp) (Diag(e^m) S), Q e^b S = Qp
//    (Diag(e^m) S), and the state update becomes
//    S' = Diag(e^{b_C - m}) [Diag(e^m) S + Km^T U~]: the Diag factors are
//    per-lane scalings folded into the one TMEM pass per chunk that also
//    writes the bf16 copy of S used as the MMA operand.  Every exponent is
//    bounded by half the chunk's decay range (checked per chunk); chunks whose
//    range exceeds kRangeMax take an exact fallback (A, P on CUDA cores with
//    one exp per term; the other products with m = 0 / b_C references, whose
//    factors are all <= 1).
//  * Long sequences with few (sequence, head) pairs are cut into segments so
//    that ~one CTA per SM has work: a summary pass computes each segment's
//    affine map S_end = X S_start + N (X carried like a second state with
//    U = 0), a short combine pass chains the maps, and the output pass runs
//    every segment from its true start state.  Only the state crosses chunks.
#include <cmath>

#include <cub/block/block_scan.cuh>

#include "kda_common.cuh"

namespace kda {

extern thread_local cudaEvent_t* g_trace_events;

struct SegItem {
    int seq;        // sequence index n
    int tok_begin;  // first token of this segment (packed index)
    int tok_end;    // one past its last token
    int g;          // segment index inside the sequence
    int G;          // number of segments of the sequence
    int first;      // item index of segment 0 of the sequence
    int slot;       // product-image slot of its chunk 0 (chunk c of the segment uses slot + c)
    int pad1;
};

// Optional per-stage cycle counters, compiled in only with -DKDA_STAGE_TIMING for
// profiling builds.  Thread 0 (stages) and lane 0 of each warp (marks) accumulate
// in shared memory; each CTA adds its totals to the device arrays once, at exit.
#ifdef KDA_STAGE_TIMING
__device__ unsigned long long g_stage_cycles[64];
__device__ unsigned long long g_warp_cycles[2 * 8 * 16];
#define KDA_STAGE(i)                                  \
    do {                                              \
        if (tid == 0) {                               \
            const long long t_ = clock64();           \
            s_stage_cyc[(i)] += (unsigned long long)(t_ - ts_); \
            ts_ = t_;                                 \
        }                                             \
    } while (0)
#define KDA_WMARK(k)                                                                        \
    do {                                                                                    \
        if (lane == 0) s_warp_cyc[(k) * 16 + warp] += (unsigned long long)(clock64() - tw0_); \
    } while (0)
#else
#define KDA_STAGE(i) \
    do {             \
    } while (0)
#define KDA_WMARK(k) \
    do {             \
    } while (0)
#endif

constexpr float kRangeMax = 64.f;   // max in-chunk decay range (nats) for the factored path
constexpr float kGateFloor = -1e4f; // log-gates below this are treated as this

// Shared-memory plan (bytes from a 1024-aligned base).  Tiles are bf16 with
// 128-byte swizzled rows unless noted.
constexpr uint32_t OFF_Q = 0;         // [64 tok][128 c]  (two 64-column boxes, TMA)
constexpr uint32_t OFF_K = 16384;     // [64 tok][128 c]  (TMA)
constexpr uint32_t OFF_V = 32768;     // [64 tok][128 v]  (TMA; MN-major A of U^T)
constexpr uint32_t OFF_G = 49152;     // fp32 [64 tok][128 c] (TMA, no swizzle)
constexpr uint32_t OFF_KP = 81920;    // [128 c][64 tok]  Kp
constexpr uint32_t OFF_WN = 98304;    // [128 k][64 tok]  -W^T
constexpr uint32_t OFF_QP = 114688;   // [128 c][64 tok]  Qp: Kp + 32 KB ([Kp;Qp] stack), -W^T + 16 KB ([-W^T|Qp])
constexpr uint32_t OFF_TB = 131072;   // [64 r][64 i]     T diag(beta)
constexpr uint32_t OFF_P = 139264;    // [64 r][64 i]     P (lower incl. diagonal)
constexpr uint32_t OFF_KM = 147456;   // [128 c][64 tok]  Km: right after P ([P|Km] as one N=192 operand)
constexpr uint32_t OFF_ST = 163840;   // 2 x [128 v][64 k] S'^T (operand copy)
constexpr uint32_t OFF_UT = 196608;   // [128 v][64 tok]  U~^T (then the O tile for the TMA store)
constexpr uint32_t OFF_MISC = 212992;
static_assert(OFF_QP - OFF_KP == 32768 && OFF_QP - OFF_WN == 16384 && OFF_KM - OFF_P == 8192, "operand stacks");
constexpr uint32_t MISC_BYTES = 7 * 1024;
constexpr uint32_t kSmemBytes = OFF_MISC + MISC_BYTES;
static_assert(kSmemBytes <= 232448, "shared memory plan");
// The map pass keeps X' in TMEM (over [A;P]) and U_X~^T at OFF_TB (16 KB).

// TMEM columns (512 allocated): U^T | O^T (or U_X^T) | S^T | [A;P] | W^T | X^T.
// [U|O] and [O|S] are contiguous so one N=128 and one N=192 MMA can fill them.
constexpr uint32_t TM_U = 0, TM_O = 64, TM_S = 128, TM_AP = 256, TM_W = 320, TM_X = 384;

// Per-chunk products of a segment's map pass, reused by its output pass: one
// image per (segment item, chunk, head), laid out as the output kernel's tiles
// so that it loads straight into MMA operands: -W^T | Qp (adjacent: one N=128
// operand), T beta, P | Km (adjacent: one N=192 operand), then the chunk's
// frame factors post(prev) e^{mp}, post(prev) e^{mk}, e^{b_C - mk} (fp32 [3][128]).
constexpr uint32_t PI_WN = 0, PI_QP = 16384, PI_TB = 32768, PI_P = 40960, PI_KM = 49152, PI_FR = 65536;
constexpr uint32_t kProdBytes = 67584;
static_assert(PI_QP - PI_WN == OFF_QP - OFF_WN && PI_KM - PI_P == OFF_KM - OFF_P && PI_P - PI_TB == OFF_P - OFF_TB,
              "product image keeps the operand stacks");

struct ChunkArgs {
    const float* beta;
    uint8_t* prod;    // product images [slot][H] (segmented calls; SegItem::slot)
    const float* gs;  // per-head scalar log-gates [Ttot][H] (scalar-gate kernels only)
    const float* init_state;
    float* final_state;
    void* o;
    const SegItem* items;
    const int* n_items;
    float* segN;
    float* segX;
    float* segS;  // per-segment start states (phase 1 writes segment 1's, the combine pass the rest)
    const int* order;    // balanced plans: the launch order of the items (heaviest first), else null
    const int* n_order;  // the number of items in that order
    int seg0_whole;      // balanced plans: segment 0 runs its output in phase 1 from the initial state
    int H;
    float scale;
};

// Column swizzle of the segment maps' X^T rows in global memory (and, by a linear
// copy, in the combine pass's shared memory): column k of row k' sits at k ^ this.
// Rows k' .. k'+3 of one MMA fragment then spread one column over 4 x 8 banks.
__device__ __forceinline__ int xt_swizzle(int kp) { return (kp & 3) << 3; }

// fp32 -> tf32 operand, rounded to nearest (ties away from zero) on the integer
// pipe: add half an ulp of the 10-bit mantissa to the magnitude bits, then drop
// the 13 low bits.  Finite inputs only.
__device__ __forceinline__ uint32_t f32_to_tf32(float x) {
    return (__float_as_uint(x) + 0x1000u) & 0xffffe000u;
}

// Warp-level D += A(16x8, row) * B(8x8, col) in tf32 with fp32 accumulation.
__device__ __forceinline__ void mma_tf32_16x8x8(float* d, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                                uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, const void* src, int c0, int c1, int c2) {
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(map),
                 "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2)
                 : "memory");
}
// 4-byte asynchronous global->shared copy; src_bytes = 0 writes zero.
__device__ __forceinline__ void cp_async4(void* dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
                 : "memory");
    asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// Global -> shared bulk copy completing on an mbarrier (16-byte aligned addresses and size).
__device__ __forceinline__ void bulk_load_1d(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}
// Shared -> global bulk copy (16-byte aligned addresses and size), in the current bulk group.
__device__ __forceinline__ void bulk_store_1d(void* gdst, const void* ssrc, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst), "r"(smem_u32(ssrc)),
                 "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// fp32 [64][64] scratch tiles of the UT transform, XOR-swizzled by row so that
// the tf32 mma fragment loads and the row-vector stores are bank-conflict free.
__device__ __forceinline__ int sidx(int r, int c) { return r * 64 + (c ^ ((r & 7) << 2)); }

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
constexpr float kLog2e = 1.4426950408889634f;  // exp(x) = 2^(x log2 e)

// ---- exact A and P for a chunk whose decay range fails the factored path's bound:
// one exp per (r, i, c) term with every exponent <= 0, one (r, i) pair of the 64 x 65 / 2
// lower-triangle pairs per thread and step (kThreads = 512 threads)
constexpr int kExactPairs = 64 * 65 / 2, kExactPer = (kExactPairs + 511) / 512;
struct ExactAP {
    float ra[kExactPer], rp[kExactPer];  // the thread's A and P terms
};
__device__ __forceinline__ void exact_pair(int pidx, int& r, int& i) {  // pidx = r (r + 1) / 2 + i, i <= r
    r = int((sqrtf(8.f * pidx + 1.f) - 1.f) * 0.5f);
    while (r * (r + 1) / 2 > pidx) --r;
    while ((r + 1) * (r + 2) / 2 <= pidx) ++r;
    i = pidx - r * (r + 1) / 2;
}


// The terms, from the q, k and cumulative-gate tiles (rows >= len are zero).
__device__ __noinline__ void exact_ap_terms(const uint8_t* sm, int tid, int len, ExactAP* acc) {
    const float* sB = reinterpret_cast<const float*>(sm + OFF_G);
    const uint8_t* sQb = sm + OFF_Q;
    const uint8_t* sKb = sm + OFF_K;
    for (int u = 0; u < kExactPer; ++u) {
        const int pidx = tid + u * 512;
        acc->ra[u] = acc->rp[u] = 0.f;
        if (pidx >= kExactPairs) continue;
        int r, i;
        exact_pair(pidx, r, i);
        if (r < len) {
            float ra = 0.f, rp = 0.f;
            for (int cc = 0; cc < kD; ++cc) {
                const float f = __expf(sB[r * kD + cc] - sB[i * kD + cc]);
                const uint32_t offr = uint32_t(cc >> 6) * 8192u + sw128_off(r, cc & 63);
                const uint32_t offi = uint32_t(cc >> 6) * 8192u + sw128_off(i, cc & 63);
                const float ki = bf16_at(sKb, offi) * f;
                ra += bf16_at(sKb, offr) * ki;
                rp += bf16_at(sQb, offr) * ki;
            }
            acc->ra[u] = ra;
            acc->rp[u] = rp;
        }
    }
}
// A (beta-scaled, strictly lower; diagonal blocks transposed for the UT solve) into sA and
// P (bf16, lower incl. the diagonal, times scale) into its tile; every thread of the CTA calls it.
__device__ __noinline__ void exact_ap_store(uint8_t* sm, uint32_t sbase, float* sA, const float* sBeta, float scale,
                                            int tid, const ExactAP* acc) {
    for (int e = tid; e < 64 * 64; e += 512) sA[e] = 0.f;
    for (int e = tid; e < 512; e += 512) st_shared_v4(sbase + OFF_P + e * 16, 0u, 0u, 0u, 0u);
    __syncthreads();
    for (int u = 0; u < kExactPer; ++u) {
        const int pidx = tid + u * 512;
        if (pidx >= kExactPairs) continue;
        int r, i;
        exact_pair(pidx, r, i);
        if (i < r) sA[((r >> 4) == (i >> 4)) ? sidx(i, r) : sidx(r, i)] = sBeta[r] * acc->ra[u];
        *reinterpret_cast<__nv_bfloat16*>(sm + OFF_P + sw128_off(r, i)) = __float2bfloat16_rn(acc->rp[u] * scale);
    }
}

// kSummary = true : segment summary (zero start state, identity X, no output).
// kSummary = false: output from the segment's true start state (the initial state
//                   for segment 0, the combine pass's result for the others).
// A segmented sequence runs in two phases of launches: phase 1 computes the maps
// of its G equal segments (exporting each chunk's products when the workspace has
// room); after the combine pass has chained the maps from the initial state,
// phase 2 computes every segment's output.  Both keep G CTAs per (sequence, head)
// busy (G-1 in phase 1 without the export: the last segment needs no map).
// kScalarGate = true: one log-gate per (token, head) (gated DeltaNet); every key
// channel shares it, so the decay factors are per row instead of per element.
constexpr int kThreads = 512;  // 16 warps; 4 threads per TMEM lane (one per column quarter)

// kChain = false (summary only): the last segment's map in a balanced plan, which
// runs only to export its chunk products (they do not depend on the state) and so
// skips the state and transition chains, which no later pass reads.
template <bool kSummary, typename OutT, bool kScalarGate, bool kChain = true>
__device__ __forceinline__ void chunk_body(const CUtensorMap& tm_q, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                                           const CUtensorMap& tm_g, const CUtensorMap& tm_o, const ChunkArgs& p,
                                           const SegItem it, const int item_id, const int h) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* sm = smem_raw;
    const uint32_t sbase = smem_u32(sm);
    if (sbase & 1023u) {  // the swizzled layouts need a 1024-byte aligned base
        if (threadIdx.x == 0) report_timeout(15);
        return;
    }

    constexpr bool kStageO = sizeof(OutT) == 2;  // bf16 output leaves through TMA stores
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int quad = warp & 3, part = warp >> 2;  // TMEM lane quadrant; column quarter
    const int H = p.H;

    float* sBeta2 = reinterpret_cast<float*>(sm + OFF_MISC);  // [2][64] beta per chunk parity
    float* sFrOp = sBeta2 + 128;                               // [128] post(prev) * e^{mp}
    float* sFrAcc = sFrOp + 128;                               // [128] post(prev) * e^{mk}
    float* sPost = sFrAcc + 128;                               // [2][128] e^{b_C - mk} per chunk
    float* sCarry = sPost + 256;                               // [4][128] row-quarter sums of g
    uint64_t* bars = reinterpret_cast<uint64_t*>(sCarry + 512);  // qkg, v, mma
    uint32_t* sTmem = reinterpret_cast<uint32_t*>(bars + 4);
    // scalar gates: [2][64] raw log-gates per chunk parity, and [2][64] per-row
    // factors e^{b_r - m}, e^{m - b_r} of the chunk being built
    float* sGs2 = reinterpret_cast<float*>(sm + OFF_MISC + 4864);
    float* sFac = sGs2 + 128;
    // UT-transform scratch, in tiles that are dead from the A/P readout until the
    // W^T spill: fp32 A over U~^T, fp32 T over -W^T.
    float* sA = reinterpret_cast<float*>(sm + OFF_UT);
    float* sT = reinterpret_cast<float*>(sm + OFF_WN);
    constexpr int kLoader = 96;    // the thread that issues every TMA load (warp 3, lane 0)
    constexpr int kExporter = 32;  // the thread that issues the map pass's product exports (warp 1)

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
        if (!kScalarGate) prefetch_tmap(&tm_g);
    }
    if (tid < 128) sPost[128 + tid] = 1.f;  // the "previous chunk" of chunk 0 scales by 1
#ifdef KDA_STAGE_TIMING
    __shared__ unsigned long long s_stage_cyc[32], s_warp_cyc[128];
    if (tid < 32) s_stage_cyc[tid] = 0;
    if (tid < 128) s_warp_cyc[tid] = 0;
#endif
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *sTmem;
    const uint32_t lane_off = uint32_t(quad * 32) << 16;
    const int vrow = quad * 32 + lane;  // TMEM lane owned by this thread

    const int t_begin = it.tok_begin, t_end = it.tok_end;
    const int nchunks = (t_end - t_begin + kC - 1) / kC;
    static_assert(kChain || kSummary, "only a map pass may skip the chains");
    constexpr bool chain = kChain;

    auto issue_qkg = [&](int c) -> bool {  // false: skipped by the failure-test hook
        if (c == c_skip_chunk_load) return false;
        const int t0 = t_begin + c * kC;
        mbar_arrive_expect_tx(&bars[0], 65536u - (kScalarGate ? 32768u : 0u));
        tma_load_3d(sm + OFF_Q, &tm_q, &bars[0], 0, h, t0);
        tma_load_3d(sm + OFF_Q + 8192, &tm_q, &bars[0], 64, h, t0);
        tma_load_3d(sm + OFF_K, &tm_k, &bars[0], 0, h, t0);
        tma_load_3d(sm + OFF_K + 8192, &tm_k, &bars[0], 64, h, t0);
        if (!kScalarGate) tma_load_3d(sm + OFF_G, &tm_g, &bars[0], 0, h, t0);
        return true;
    };
    auto issue_v = [&](int c) {
        const int t0 = t_begin + c * kC;
        mbar_arrive_expect_tx(&bars[1], 16384u);
        tma_load_3d(sm + OFF_V, &tm_v, &bars[1], 0, h, t0);
        tma_load_3d(sm + OFF_V + 8192, &tm_v, &bars[1], 64, h, t0);
    };
    bool pend_qkg = false, pend_v = false;  // meaningful in the loader thread only
    if (tid == kLoader && nchunks > 0) {
        pend_qkg = issue_qkg(0);
        issue_v(0);
        pend_v = true;
    }

    // ---- start state into TMEM: S^T (lane = v, column = k); X^T = I for the summary.
    {
        const float* src = nullptr;
        if (!kSummary) {
            // segment 0 starts from the initial state (read in phase 1, before any
            // final state is written, so the two may alias); the others from the
            // combine pass
            if (it.g == 0)
                src = p.init_state ? p.init_state + (size_t(it.seq) * H + h) * (kD * kD) : nullptr;
            else
                src = p.segS + (size_t(item_id) * H + h) * (kD * kD);
        }
#pragma unroll 1
        for (int cb = 0; cb < 2; ++cb) {
            float buf[16];
            const int k0 = part * 32 + cb * 16;
#pragma unroll
            for (int j = 0; j < 16; ++j) buf[j] = src ? src[size_t(k0 + j) * kD + vrow] : 0.f;
            tmem_st16(tbase + TM_S + lane_off + k0, buf);
            if (kSummary) {
#pragma unroll
                for (int j = 0; j < 16; ++j) buf[j] = (k0 + j == vrow) ? 1.f : 0.f;
                tmem_st16(tbase + TM_X + lane_off + k0, buf);
            }
        }
        tmem_wait_st();
    }

    uint32_t ph_qkg = 0, ph_v = 0, ph_mma = 0;
    bool aborted = false;
    auto fetch_beta = [&](int cc) {  // beta of chunk cc's rows into sBeta2[cc & 1], asynchronously (tid < 64)
        const int tn = t_begin + cc * kC + tid;
        const bool valid = cc < nchunks && tn < t_end;
        cp_async4(sBeta2 + (cc & 1) * 64 + tid, p.beta + (valid ? size_t(tn) * H + h : 0), valid ? 4u : 0u);
        if (kScalarGate)  // rows past the end read as g = 0
            cp_async4(sGs2 + (cc & 1) * 64 + tid, p.gs + (valid ? size_t(tn) * H + h : 0), valid ? 4u : 0u);
    };
    if (tid < 64) fetch_beta(0);
    const uint32_t id_ap = idesc_bf16(128, 64, 1, 1);   // [Kp;Qp] (MN) x Km (MN)
    const uint32_t id_w = idesc_bf16(128, 64, 0, 0);    // Kp^T (K) x (T beta)^T (K)
    const uint32_t id_u = idesc_bf16(128, 64, 1, 0);    // V^T (MN) x (T beta)^T (K)
    const uint32_t id_so = idesc_bf16(128, 64, 0, 1);   // S^T (K) x {-W^T, Qp} (MN)
    const uint32_t id_s = idesc_bf16(128, 128, 0, 0);   // U~^T (K) x Km (K)
    const uint32_t id_so2 = idesc_bf16(128, 128, 0, 1); // S'^T (K) x [-W^T | Qp] (MN)
    const uint32_t id_os = idesc_bf16(128, 192, 0, 0);  // U~^T (K) x [P^T | Km] (K)
    // Summary pass: X'^T in TMEM over the [A;P] columns once they are read out (A operand of
    // the U_X~ MMA); U_X~^T over T beta + P once both are exported.
    const uint32_t UXT = OFF_TB;
    const uint32_t TM_XP = TM_AP;

    // ---- gated operands of a chunk.  Chunk c+1's are built while chunk c's last
    // tensor-core MMAs run, in pieces placed by which tiles those MMAs still read:
    //   e_prep : wait for q, k, g; cumulative log decay per channel (registers);
    //            row-quarter sums to shared memory (a barrier must follow);
    //   e_head : carry, chunk total b_C, reference point m, this channel's decay range;
    //   e_rows : factored operands of 8 rows, packed to bf16 in registers;
    //   e_put_kq / e_put_m : into the Kp, Qp tiles (free once the U~/O MMA is done)
    //            and the Km tile (free once the O/S MMA is done);
    //   e_exact: the rare chunk whose decay range failed the vote, rebuilt with the
    //            exact references (mp = 0, mk = b_C);
    //   e_frame: per-channel frame factors.
    const int ch = tid & 127, rq = tid >> 7;  // channel; row quarter (16 rows)
    const uint32_t e_box = uint32_t(ch >> 6) * 8192u;
    float bl[16];
    float e_carry = 0.f, e_bC = 0.f, e_m = 0.f, e_b0 = 0.f;
    bool e_fast_here = true;
    uint32_t opk[8], opq[8], opm[8];
    auto e_prep = [&](int cc) -> bool {  // false: a bounded wait gave up
        const int len = min(kC, t_end - (t_begin + cc * kC));
        bool okw = mbar_wait(&bars[0], ph_qkg, 1);
        ph_qkg ^= 1;
        if (tid == kLoader) pend_qkg = false;
        if (__syncthreads_or(!okw)) return false;
        if (len < kC) {  // rows past the end of the sequence: g = k = q = 0 (beta = 0)
            for (int e = tid; e < (kC - len) * 32; e += kThreads) {
                const int r = len + (e >> 5), w = e & 31;
                if (!kScalarGate) reinterpret_cast<float4*>(sm + OFF_G)[r * 32 + w] = make_float4(0.f, 0.f, 0.f, 0.f);
                if (w < 16) {
                    const int box = w >> 3, j = w & 7;
                    st_shared_v4(sbase + OFF_K + box * 8192 + r * 128 + j * 16, 0u, 0u, 0u, 0u);
                    st_shared_v4(sbase + OFF_Q + box * 8192 + r * 128 + j * 16, 0u, 0u, 0u, 0u);
                }
            }
            __syncthreads();
        }
        if (kScalarGate) {
            if (tid < 64) {  // this chunk's beta and g have landed: inclusive scan of g per warp
                cp_async_wait_all();
                float x = fmaxf(sGs2[(cc & 1) * 64 + tid], kGateFloor);
#pragma unroll
                for (int d = 1; d < 32; d <<= 1) {
                    const float y = __shfl_up_sync(0xffffffffu, x, d);
                    if (lane >= d) x += y;
                }
                sCarry[tid] = x;  // rows 32..63 still lack rows 0..31's total
                fetch_beta(cc + 1);
            }
            return true;
        }
        const float* sG = reinterpret_cast<const float*>(sm + OFF_G);
        float acc = 0.f;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            acc += fmaxf(sG[(rq * 16 + j) * kD + ch], kGateFloor);
            bl[j] = acc;
        }
        sCarry[rq * 128 + ch] = acc;
        e_b0 = fmaxf(sG[ch], kGateFloor);
        if (tid < 64) {  // this chunk's beta has landed; start the one after it
            cp_async_wait_all();
            fetch_beta(cc + 1);
        }
        return true;
    };
    // scalar gates: b of row r from the per-warp scans (valid between e_prep and the
    // next chunk's e_prep)
    auto b_row = [&](int r) { return sCarry[r] + (r >= 32 ? sCarry[31] : 0.f); };
    auto e_head = [&]() {
        if (kScalarGate) {
            e_carry = rq ? b_row(rq * 16 - 1) : 0.f;
#pragma unroll
            for (int j = 0; j < 16; ++j) bl[j] = b_row(rq * 16 + j) - e_carry;
            e_b0 = b_row(0);
            e_bC = b_row(63);
            e_fast_here = (e_b0 - e_bC) <= kRangeMax;
            e_m = 0.5f * (e_b0 + e_bC);
            return;
        }
        e_carry = 0.f;
        e_bC = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float cq = sCarry[q * 128 + ch];
            e_carry += (q < rq) ? cq : 0.f;
            e_bC += cq;
        }
        e_fast_here = (e_b0 - e_bC) <= kRangeMax;
        e_m = 0.5f * (e_b0 + e_bC);
    };
    // Kp = k e^{b-mp}, Qp = q e^{b-mp}, Km = k e^{mk-b} for rows [8 h8, 8 h8 + 8) of the
    // quarter; factored (mp = mk = m): one product y = (b - m) log2 e feeds both factors.
    auto e_rows = [&](const int h8, const bool factored) {
        const uint8_t* sQb = sm + OFF_Q;
        const uint8_t* sKb = sm + OFF_K;
        const float sc = p.scale;
        const bool unit_scale = sc == 1.f;
        const float y0 = (factored ? e_carry - e_m : e_carry) * kLog2e;
        const float y1 = (e_bC - e_carry) * kLog2e;
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
            float kv[2], qv[2], e1[2], e2[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int j = h8 * 8 + e + u, r = rq * 16 + j;
                const uint32_t off = e_box + sw128_off(r, ch & 63);
                kv[u] = bf16_at(sKb, off);
                qv[u] = unit_scale ? bf16_at(sQb, off) : bf16_at(sQb, off) * sc;
                if (factored && kScalarGate) {  // per-row factors, shared by every channel
                    e1[u] = sFac[r];
                    e2[u] = sFac[64 + r];
                } else if (factored) {
                    const float y = fmaf(bl[j], kLog2e, y0);
                    e1[u] = ex2_approx(y);
                    e2[u] = ex2_approx(-y);
                } else {
                    e1[u] = ex2_approx(fmaf(bl[j], kLog2e, y0));
                    e2[u] = ex2_approx(fmaf(bl[j], -kLog2e, y1));
                }
            }
            const int slot = h8 * 4 + (e >> 1);
            opk[slot] = pack_bf16x2(kv[0] * e1[0], kv[1] * e1[1]);
            opq[slot] = pack_bf16x2(qv[0] * e1[0], qv[1] * e1[1]);
            opm[slot] = pack_bf16x2(kv[0] * e2[0], kv[1] * e2[1]);
        }
    };
    auto e_put_kq = [&](const int h8) {
        const int j8 = (rq * 16 + h8 * 8) >> 3;
        st_shared_v4(sbase + OFF_KP + sw128_chunk(ch, j8), opk[h8 * 4], opk[h8 * 4 + 1], opk[h8 * 4 + 2],
                     opk[h8 * 4 + 3]);
        st_shared_v4(sbase + OFF_QP + sw128_chunk(ch, j8), opq[h8 * 4], opq[h8 * 4 + 1], opq[h8 * 4 + 2],
                     opq[h8 * 4 + 3]);
    };
    auto e_put_m = [&]() {
#pragma unroll
        for (int h8 = 0; h8 < 2; ++h8) {
            const int j8 = (rq * 16 + h8 * 8) >> 3;
            st_shared_v4(sbase + OFF_KM + sw128_chunk(ch, j8), opm[h8 * 4], opm[h8 * 4 + 1], opm[h8 * 4 + 2],
                         opm[h8 * 4 + 3]);
        }
    };
    // Exact rebuild; the g tile still holds this chunk's gates, so b is recomputed from it
    // (bl need not stay live) and then kept there for the exact A / P.
    auto e_exact = [&]() {
        float* sB = reinterpret_cast<float*>(sm + OFF_G);
        if (kScalarGate) {  // the g tile is not loaded: b comes from the scans
#pragma unroll
            for (int j = 0; j < 16; ++j) bl[j] = b_row(rq * 16 + j) - e_carry;
        } else {
            float acc = 0.f;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                acc += fmaxf(sB[(rq * 16 + j) * kD + ch], kGateFloor);
                bl[j] = acc;
            }
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) sB[(rq * 16 + j) * kD + ch] = bl[j] + e_carry;
        e_rows(0, false);
        e_rows(1, false);
        e_put_kq(0);
        e_put_kq(1);
    };
    auto e_factors = [&]() {  // scalar gates, factored references: row tid's e^{b-m}, e^{m-b}
        if (kScalarGate && tid < 64) {
            const float y = (b_row(tid) - e_m) * kLog2e;
            sFac[tid] = ex2_approx(y);
            sFac[64 + tid] = ex2_approx(-y);
        }
    };
    auto e_frame = [&](const int cc, const bool fastc) {
        if (tid < 128) {
            const float mp = fastc ? e_m : 0.f, mk = fastc ? e_m : e_bC;
            const float postp = sPost[((cc & 1) ^ 1) * 128 + ch];
            sFrOp[ch] = postp * ex2_approx(mp * kLog2e);
            sFrAcc[ch] = postp * ex2_approx(mk * kLog2e);
            sPost[(cc & 1) * 128 + ch] = ex2_approx((e_bC - mk) * kLog2e);
        }
    };

    // T beta's strictly-upper 16x16 blocks are zeroed every chunk, one 16-byte chunk
    // per thread < 192: rows of block I hold 6 - 2I zero chunks past column 16 (I + 1).
    uint32_t tb_zero_addr = 0;
    if (tid < 192) {
        const int I = tid < 96 ? 0 : (tid < 160 ? 1 : 2);
        const int e0 = tid - (I == 0 ? 0 : (I == 1 ? 96 : 160)), per = 6 - 2 * I;
        tb_zero_addr = sbase + OFF_TB + sw128_chunk(16 * I + e0 / per, 2 * (I + 1) + e0 % per);
    }

    bool fast_next = true;
    if (nchunks > 0) {
        if (!e_prep(0)) {
            aborted = true;
        } else {
            __syncthreads();
            e_head();
            e_factors();
            fast_next = __syncthreads_and(e_fast_here) != 0;
            if (fast_next) {
                e_rows(0, true);
                e_rows(1, true);
                e_put_kq(0);
                e_put_kq(1);
            } else {
                e_exact();
            }
            e_put_m();
            e_frame(0, fast_next);
            fence_async_smem();
            __syncthreads();
            if (fast_next && tid == kLoader && nchunks > 1) {  // q, k, g of chunk 0 are consumed
                pend_qkg = issue_qkg(1);
            }
        }
    }

#pragma unroll 1
    for (int c = 0; c < nchunks && !aborted; ++c) {
        const int t0 = t_begin + c * kC;
        const int len = min(kC, t_end - t0);
        const float* sBeta = sBeta2 + (c & 1) * 64;
        const bool fast = fast_next;
        bool ok = true;
#ifdef KDA_STAGE_TIMING
        long long ts_ = clock64(), tw0_ = ts_;
#endif
        KDA_STAGE(1);
        // the map pass exports what the output pass of this segment reuses
        uint8_t* img = (kSummary && p.prod) ? p.prod + ((size_t(it.slot) + c) * H + h) * kProdBytes : nullptr;
        if (img) {
            if (tid == kExporter) {  // Qp and Km of this chunk are final (built before the last barrier)
                bulk_store_1d(img + PI_QP, sm + OFF_QP, 16384u);
                bulk_store_1d(img + PI_KM, sm + OFF_KM, 16384u);
                bulk_commit();
            }
            if (tid < 128) {
                float* fr = reinterpret_cast<float*>(img + PI_FR);
                fr[tid] = sFrOp[tid];
                fr[128 + tid] = sFrAcc[tid];
                fr[256 + tid] = sPost[(c & 1) * 128 + tid];
            }
        }

        // ===== A (scaled by beta, strictly lower) and P (lower incl. diagonal) =====
        if (fast && tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint64_t a = sdesc_sw128(sbase + OFF_KP + ks * 2048, OFF_QP - OFF_KP, 1024);
                const uint64_t b = sdesc_sw128(sbase + OFF_KM + ks * 2048, 8192, 1024);
                umma_bf16(tbase + TM_AP, a, b, id_ap, ks > 0);
            }
            umma_commit(&bars[2]);
        }
        // ===== S frame (needs only the previous chunk's state; overlaps the A/P MMA):
        //   S <- S * post(prev);  bf16 operand = S * e^{mp};  TMEM = S * e^{mk}
        {
            auto frame = [&](uint32_t tcol, uint32_t st_off0, uint32_t st_off1) {
                float x[32];  // key columns [32 part, 32 part + 32) of this lane
#pragma unroll
                for (int cb = 0; cb < 2; ++cb) tmem_ld16(tbase + tcol + lane_off + part * 32 + cb * 16, x + cb * 16);
                tmem_wait_ld();
                const uint32_t dst = sbase + ((part >> 1) ? st_off1 : st_off0);
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
                for (int cb = 0; cb < 2; ++cb) tmem_st16(tbase + tcol + lane_off + part * 32 + cb * 16, x + cb * 16);
            };
            if (chain) frame(TM_S, OFF_ST, OFF_ST + 16384);
            if (!kSummary) {  // O^T starts at zero: the merged [U~|O] MMA below accumulates into both halves
                float z[16];
#pragma unroll
                for (int j = 0; j < 16; ++j) z[j] = 0.f;
                tmem_st16(tbase + TM_O + lane_off + part * 16, z);
            }
            tmem_wait_st();
        }
        // the previous O tile (over U~^T / sA) has been read out.  The exporter's groups are
        // waited for after the U~/O MMA: that wait covers the previous chunk's -W^T (under T)
        // before this chunk's solve, and this chunk's Qp / Km before they are rewritten.
        if (tid == 0) bulk_wait_read0();
        if (fast) {
            ok = mbar_wait(&bars[2], ph_mma, 2);
            ph_mma ^= 1;
            tc_fence_after();
            if (__syncthreads_or(!ok)) { aborted = true; break; }
            KDA_STAGE(2);
#ifdef KDA_STAGE_TIMING
            tw0_ = clock64();
#endif
            float vals[16];  // columns [16 part, 16 part + 16)
            tmem_ld16(tbase + TM_AP + lane_off + part * 16, vals);
            tmem_wait_ld();
            if (vrow < 64 && part == (vrow >> 4)) {
                // diagonal 16x16 block of A, stored transposed (A_{r i} at [i][r]) for the
                // column-per-lane solve below
                const float br = sBeta[vrow];
#pragma unroll
                for (int j = 0; j < 16; ++j) {
                    const int i = part * 16 + j;
                    sA[sidx(i, vrow)] = (i < vrow) ? br * vals[j] : 0.f;
                }
            } else if (vrow < 64) {
                const float br = sBeta[vrow];
#pragma unroll
                for (int j = 0; j < 16; j += 4) {
                    const int i = part * 16 + j;
                    float4 w4;
                    w4.x = (i + 0 < vrow) ? br * vals[j + 0] : 0.f;
                    w4.y = (i + 1 < vrow) ? br * vals[j + 1] : 0.f;
                    w4.z = (i + 2 < vrow) ? br * vals[j + 2] : 0.f;
                    w4.w = (i + 3 < vrow) ? br * vals[j + 3] : 0.f;
                    *reinterpret_cast<float4*>(&sA[sidx(vrow, i)]) = w4;
                }
            } else {
                const int r = vrow - 64;
#pragma unroll
                for (int q4 = 0; q4 < 2; ++q4) {
                    uint32_t w[4];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int i0 = part * 16 + q4 * 8 + 2 * u;
                        w[u] = pack_bf16x2(i0 <= r ? vals[q4 * 8 + 2 * u] : 0.f,
                                           i0 + 1 <= r ? vals[q4 * 8 + 2 * u + 1] : 0.f);
                    }
                    st_shared_v4(sbase + OFF_P + sw128_chunk(r, part * 2 + q4), w[0], w[1], w[2], w[3]);
                }
            }
        } else {
            // Exact fallback: one exp per (r, i, c) term, all exponents <= 0.  Out of line: it is
            // rare, and inline it would sit in the middle of the chunk loop's instruction stream.
            ExactAP ex;
            exact_ap_terms(sm, tid, len, &ex);
            __syncthreads();  // the q / k / b tiles are read
            if (tid == kLoader && c + 1 < nchunks) {
                pend_qkg = issue_qkg(c + 1);
            }
            exact_ap_store(sm, sbase, sA, sBeta, p.scale, tid, &ex);
        }
        KDA_WMARK(0);
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        KDA_WMARK(1);
        KDA_STAGE(3);
        if (kSummary && chain && warp >= 4) {
            // X' = X e^{mp} as bf16 pairs into the [A;P] columns (read out by now): the A operand
            // of the U_X~ MMA; TMEM X <- X e^{mk}.  Warps 4..15 do it while warps 0..3 run the
            // diagonal UT solves: the three warps of a TMEM lane quadrant take key columns
            // [0, 64), [64, 96) and [96, 128).
            const int slot = (warp >> 2) - 1;
            for (int kb = slot == 0 ? 0 : 32 * (slot + 1); kb < (slot == 0 ? 64 : 32 * (slot + 2)); kb += 32) {
                float x[32];
                tmem_ld16(tbase + TM_X + lane_off + kb, x);
                tmem_ld16(tbase + TM_X + lane_off + kb + 16, x + 16);
                tmem_wait_ld();
                float xp[16];
#pragma unroll
                for (int j = 0; j < 32; j += 2) {
                    const int k0 = kb + j;
                    xp[j >> 1] = __uint_as_float(pack_bf16x2(x[j] * sFrOp[k0], x[j + 1] * sFrOp[k0 + 1]));
                    x[j] *= sFrAcc[k0];
                    x[j + 1] *= sFrAcc[k0 + 1];
                }
                tmem_st16(tbase + TM_X + lane_off + kb, x);
                tmem_st16(tbase + TM_X + lane_off + kb + 16, x + 16);
                tmem_st16(tbase + TM_XP + lane_off + kb / 2, xp);
            }
            tmem_wait_st();
        }

        // ===== UT transform: T = (I + A)^{-1}, blocked forward substitution =====
        if (warp < 4 && lane < 16) {
            // 16x16 diagonal blocks D_I = (I + A_II)^{-1}: warp I, lane jc solves column jc.
            // Right-looking: once t_r is final, every later row r2 subtracts A_{r2 r} t_r.
            // Column r of A_II is row r of the transposed block the readout stored, so
            // each step reads up to four float4 (the same for all lanes), loaded two
            // steps ahead so that the chain is one FMA per step.
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
            const float bj = sBeta[base + jc];
#pragma unroll
            for (int r = 0; r < 16; ++r) {
                sT[sidx(base + r, base + jc)] = ps[r];
                *reinterpret_cast<uint16_t*>(sm + OFF_TB + sw128_off(base + r, base + jc)) =
                    uint16_t((__float_as_uint(ps[r] * bj) + 0x8000u) >> 16);
            }
        }
        if (tid < 192) st_shared_v4(tb_zero_addr, 0u, 0u, 0u, 0u);  // strictly-upper blocks of T beta
        KDA_STAGE(15);
        KDA_WMARK(2);
        __syncthreads();
        KDA_WMARK(3);
        KDA_STAGE(4);
        // Off-diagonal 16x16 blocks on tf32 warp MMAs, each as (L A) R so that the
        // product L A stays in registers: an accumulator fragment (row g, columns 2t and
        // 2t+1) is the A operand of the next MMA when the k index is permuted the same
        // way in the B operand (k slot t <-> row 2t, k slot t+4 <-> row 2t+1).
        // Level 1: T_IJ = -(D_I A_IJ) D_J for (I, J) = (1,0), (2,1), (3,2).
        // Level 2 (needs T_10, T_32), with Z_2K = D_2 A_2K and Z_3K = T_32 A_2K + D_3 A_3K:
        //   T_20 = -(Z_20 D_0 + Z_21 T_10),  T_31 = -Z_31 D_1,  T_30 = -(Z_30 D_0 + Z_31 T_10).
        // Warp task = (output block, 8-column half).
        {
            const int gq = lane >> 2, tq = lane & 3;
            // y (16x16: fragments for columns [0, 8) and [8, 16)) += L (16x16 at row lr0,
            // column lk0 of srcL) x R (16x16 at row rk0, column rn0 of srcR)
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
            // acc (16x8) += y (16x16, registers) x sT rows [rk0, rk0+16), columns [rn0, rn0+8)
            auto mm_reg = [&](float* acc, const float* y, int rk0, int rn0) {
#pragma unroll
                for (int nb = 0; nb < 2; ++nb)
                    mma_tf32_16x8x8(acc, f32_to_tf32(y[nb * 4 + 0]), f32_to_tf32(y[nb * 4 + 2]),
                                    f32_to_tf32(y[nb * 4 + 1]), f32_to_tf32(y[nb * 4 + 3]),
                                    f32_to_tf32(sT[sidx(rk0 + nb * 8 + 2 * tq, rn0 + gq)]),
                                    f32_to_tf32(sT[sidx(rk0 + nb * 8 + 2 * tq + 1, rn0 + gq)]));
            };
            auto put_t = [&](int r0, int c0, const float* acc) {  // T block piece = -acc, and its T beta
                const int cc = c0 + 2 * tq;
                sT[sidx(r0 + gq, cc)] = -acc[0];
                sT[sidx(r0 + gq, cc + 1)] = -acc[1];
                sT[sidx(r0 + gq + 8, cc)] = -acc[2];
                sT[sidx(r0 + gq + 8, cc + 1)] = -acc[3];
                const float b0c = sBeta[cc], b1c = sBeta[cc + 1];
                *reinterpret_cast<uint32_t*>(sm + OFF_TB + sw128_off(r0 + gq, cc)) =
                    pack_bf16x2(-acc[0] * b0c, -acc[1] * b1c);
                *reinterpret_cast<uint32_t*>(sm + OFF_TB + sw128_off(r0 + gq + 8, cc)) =
                    pack_bf16x2(-acc[2] * b0c, -acc[3] * b1c);
            };
            if (warp < 6) {
                const int J = warp >> 1, I = J + 1, cn = 16 * J + 8 * (warp & 1);
                float y[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                mm16(y, sT, 16 * I, 16 * I, sA, 16 * I, 16 * J);
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
                mm_reg(acc, y, 16 * J, cn);
                put_t(16 * I, cn, acc);
            }
            KDA_WMARK(4);
            __syncthreads();
            KDA_WMARK(5);
            if (warp < 6) {
                const int task = warp >> 1, cn = 8 * (warp & 1);
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
                float z0[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                float z1[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
                if (task == 0) {  // T_20
                    mm16(z0, sT, 32, 32, sA, 32, 0);
                    mm16(z1, sT, 32, 32, sA, 32, 16);
                    mm_reg(acc, z0, 0, cn);
                    mm_reg(acc, z1, 16, cn);
                    put_t(32, cn, acc);
                } else if (task == 1) {  // T_31
                    mm16(z1, sT, 48, 32, sA, 32, 16);
                    mm16(z1, sT, 48, 48, sA, 48, 16);
                    mm_reg(acc, z1, 16, 16 + cn);
                    put_t(48, 16 + cn, acc);
                } else {  // T_30
                    mm16(z0, sT, 48, 32, sA, 32, 0);
                    mm16(z1, sT, 48, 32, sA, 32, 16);
                    mm16(z0, sT, 48, 48, sA, 48, 0);
                    mm16(z1, sT, 48, 48, sA, 48, 16);
                    mm_reg(acc, z0, 0, cn);
                    mm_reg(acc, z1, 16, cn);
                    put_t(48, cn, acc);
                }
            }
            KDA_WMARK(6);
            __syncthreads();
            KDA_WMARK(7);
        }
        KDA_STAGE(5);
        KDA_STAGE(14);
        fence_async_smem();
        ok = mbar_wait(&bars[1], ph_v, 3);
        ph_v ^= 1;
        if (tid == kLoader) pend_v = false;
        if (__syncthreads_or(!ok)) { aborted = true; break; }
        if (img && tid == kExporter) {  // T beta and P (adjacent tiles) are final
            bulk_store_1d(img + PI_TB, sm + OFF_TB, 16384u);
            bulk_commit();
        }
        KDA_STAGE(6);

        // ===== W^T = Kp^T (T beta)^T and U^T = V^T (T beta)^T =====
        if (tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t bt = sdesc_sw128(sbase + OFF_TB + ks * 32, 16, 1024);
                umma_bf16(tbase + TM_W, sdesc_sw128(sbase + OFF_KP + ks * 32, 16, 1024), bt, id_w, ks > 0);
                umma_bf16(tbase + TM_U, sdesc_sw128(sbase + OFF_V + ks * 2048, 8192, 1024), bt, id_u, ks > 0);
            }
            umma_commit(&bars[2]);
        }

        KDA_STAGE(7);
        ok = mbar_wait(&bars[2], ph_mma, 4);
        ph_mma ^= 1;
        tc_fence_after();
        if (__syncthreads_or(!ok)) { aborted = true; break; }
        KDA_STAGE(8);
        if (tid == kLoader && c + 1 < nchunks) {  // V of this chunk is consumed
            issue_v(c + 1);
            pend_v = true;
        }
        {  // -W^T -> smem (lane = key channel k, 16 tokens per thread)
            float w[16];
            tmem_ld16(tbase + TM_W + lane_off + part * 16, w);
            tmem_wait_ld();
#pragma unroll
            for (int q4 = 0; q4 < 2; ++q4)
                st_shared_v4(sbase + OFF_WN + sw128_chunk(vrow, part * 2 + q4),
                             pack_bf16x2(-w[q4 * 8 + 0], -w[q4 * 8 + 1]), pack_bf16x2(-w[q4 * 8 + 2], -w[q4 * 8 + 3]),
                             pack_bf16x2(-w[q4 * 8 + 4], -w[q4 * 8 + 5]), pack_bf16x2(-w[q4 * 8 + 6], -w[q4 * 8 + 7]));
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        if (img && tid == kExporter) {  // -W^T is final
            bulk_store_1d(img + PI_WN, sm + OFF_WN, 16384u);
            bulk_commit();
        }

        KDA_STAGE(9);
        // ===== U~^T = U^T - S'^T W^T ;  O^T = S'^T Qp  (or U_X~^T = -X'^T W^T) =====
        if (chain && tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 8; ++ks) {
                const uint64_t a = sdesc_sw128(sbase + OFF_ST + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
                if (!kSummary) {
                    // [U~ | O] += S'^T [-W^T | Qp]: one N=128 MMA per K step
                    umma_bf16(tbase + TM_U, a, sdesc_sw128(sbase + OFF_WN + ks * 2048, OFF_QP - OFF_WN, 1024),
                              id_so2, 1);
                } else {
                    umma_bf16(tbase + TM_U, a, sdesc_sw128(sbase + OFF_WN + ks * 2048, 8192, 1024), id_so, 1);
                    umma_bf16_tmem_a(tbase + TM_O, tbase + TM_XP + ks * 8,
                                     sdesc_sw128(sbase + OFF_WN + ks * 2048, 8192, 1024), id_so, ks > 0);
                }
            }
            umma_commit(&bars[2]);
        }
        // next chunk's operands, first part (the MMA above reads S', -W, Qp)
        const bool has_next = c + 1 < nchunks;
        if (has_next) {
            if (!e_prep(c + 1)) { aborted = true; break; }
            __syncthreads();  // row-quarter sums (scalar gates: per-warp scans)
            e_head();
            if (kScalarGate) {
                e_factors();
                __syncthreads();  // every row's factors are in sFac
            }
            e_rows(0, true);
        }
        KDA_STAGE(16);
        if (chain) {
            ok = mbar_wait(&bars[2], ph_mma, 5);
            ph_mma ^= 1;
        }
        tc_fence_after();
        // the exports have read Qp (rewritten next) and T beta + P (U_X~^T goes over them)
        if (img && tid == kExporter) bulk_wait_read0();
        if (__syncthreads_or(!ok)) { aborted = true; break; }
        KDA_STAGE(10);
        if (has_next) e_put_kq(0);  // Kp, Qp are free: the A/P, W and U~/O MMAs are done
        {  // U~^T (and U_X~^T) -> smem, lane = value channel, 16 tokens per thread
            auto spill = [&](uint32_t tcol, uint32_t dst_off) {
                float u[16];
                tmem_ld16(tbase + tcol + lane_off + part * 16, u);
                tmem_wait_ld();
#pragma unroll
                for (int q4 = 0; q4 < 2; ++q4)
                    st_shared_v4(sbase + dst_off + sw128_chunk(vrow, part * 2 + q4),
                                 pack_bf16x2(u[q4 * 8 + 0], u[q4 * 8 + 1]), pack_bf16x2(u[q4 * 8 + 2], u[q4 * 8 + 3]),
                                 pack_bf16x2(u[q4 * 8 + 4], u[q4 * 8 + 5]), pack_bf16x2(u[q4 * 8 + 6], u[q4 * 8 + 7]));
            };
            if (chain) spill(TM_U, OFF_UT);
            if (kSummary && chain) spill(TM_O, UXT);
        }
        fence_async_smem();
        tc_fence_before();
        fast_next = __syncthreads_and(e_fast_here) != 0;  // next chunk's decay-range vote

        KDA_STAGE(11);
        // ===== O^T += U~^T P^T ;  S^T += U~^T Km  (X^T += U_X~^T Km) =====
        if (chain && tid == 0) {
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                const uint64_t a = sdesc_sw128(sbase + OFF_UT + ks * 32, 16, 1024);
                if (!kSummary)  // [O | S] += U~^T [P^T | Km]: one N=192 MMA per K step
                    umma_bf16(tbase + TM_O, a, sdesc_sw128(sbase + OFF_P + ks * 32, 16, 1024), id_os, 1);
                else
                    umma_bf16(tbase + TM_S, a, sdesc_sw128(sbase + OFF_KM + ks * 32, 16, 1024), id_s, 1);
                if (kSummary)
                    umma_bf16(tbase + TM_X, sdesc_sw128(sbase + UXT + ks * 32, 16, 1024),
                              sdesc_sw128(sbase + OFF_KM + ks * 32, 16, 1024), id_s, 1);
            }
            umma_commit(&bars[2]);
        }
        if (has_next && fast_next) {  // second part, overlapping the MMA above (reads U~, P, Km)
            e_rows(1, true);
            e_put_kq(1);
        }
        KDA_STAGE(18);
        if (chain) {
            ok = mbar_wait(&bars[2], ph_mma, 6);
            ph_mma ^= 1;
        }
        tc_fence_after();
        if (__syncthreads_or(!ok)) { aborted = true; break; }
        KDA_STAGE(12);
        if (has_next) {  // last part: Km is free now
            if (!fast_next) e_exact();
            e_put_m();
            e_frame(c + 1, fast_next);
            fence_async_smem();
        }
        KDA_STAGE(19);

        bool staged = false;
        if (!kSummary) {  // O^T -> o[t0 + r, h, v]
            float ov[16];  // tokens [16 part, 16 part + 16) of value channel vrow
            tmem_ld16(tbase + TM_O + lane_off + part * 16, ov);
            tmem_wait_ld();
            if (kStageO && len == kC) {
                // full chunk: transpose through a swizzled [64 tok][128 v] tile (over U~^T,
                // consumed by now) and write it with one TMA store
                uint8_t* so = sm + OFF_UT + (vrow >> 6) * 8192;
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
            tma_store_3d(&tm_o, sm + OFF_UT, 0, h, t0);
            tma_store_3d(&tm_o, sm + OFF_UT + 8192, 64, h, t0);
            bulk_commit();
        }
        if (has_next && fast_next && tid == kLoader && c + 2 < nchunks) {  // q, k, g of chunk c+1 are consumed
            pend_qkg = issue_qkg(c + 2);
        }
        KDA_STAGE(13);
    }

    if (!aborted) {
        // ---- end state: S = S^T(TMEM) * post(last chunk)
        const int last = (nchunks - 1) & 1;
        float* dstS = nullptr;
        float* dstX = nullptr;
        if (kSummary) {
            if (chain) {
                dstS = p.segN + (size_t(item_id) * H + h) * (kD * kD);
                dstX = p.segX + (size_t(item_id) * H + h) * (kD * kD);
            }
        } else if (it.g == it.G - 1) {
            if (p.final_state) dstS = p.final_state + (size_t(it.seq) * H + h) * (kD * kD);
        } else if (p.seg0_whole && it.g == 0 && item_id + 1 < *p.n_items) {  // the start state of segment 1
            dstS = p.segS + (size_t(item_id + 1) * H + h) * (kD * kD);
        }
        tc_fence_after();
        auto store = [&](uint32_t tcol, float* dst) {
#pragma unroll 1
            for (int cb = 0; cb < 2; ++cb) {
                const int k0 = part * 32 + cb * 16;
                float x[16];
                tmem_ld16(tbase + tcol + lane_off + k0, x);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) dst[size_t(k0 + j) * kD + vrow] = x[j] * sPost[last * 128 + k0 + j];
            }
        };
        if (dstS) store(TM_S, dstS);
        if (dstX) {  // X stored transposed, [k'][k] (TMEM lane k' owns a row), for the combine pass, with
                     // column k of row k' at k ^ xt_swizzle(k') (see the combine pass)
            float* row = dstX + size_t(vrow) * kD;
            const int sw = xt_swizzle(vrow);
#pragma unroll 1
            for (int cb = 0; cb < 2; ++cb) {
                const int k0 = part * 32 + cb * 16;
                float x[16];
                tmem_ld16(tbase + TM_X + lane_off + k0, x);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; j += 4)
                    *reinterpret_cast<float4*>(row + ((k0 + j) ^ sw)) =
                        make_float4(x[j] * sPost[last * 128 + k0 + j], x[j + 1] * sPost[last * 128 + k0 + j + 1],
                                    x[j + 2] * sPost[last * 128 + k0 + j + 2], x[j + 3] * sPost[last * 128 + k0 + j + 3]);
            }
        }
    } else {
        // let copies and MMAs still in flight land before shared memory and TMEM are released
        if (tid == kLoader) {
            if (pend_qkg) mbar_wait(&bars[0], ph_qkg, 7);
            if (pend_v) mbar_wait(&bars[1], ph_v, 7);
        }
        if (tid == 0) mbar_wait(&bars[2], ph_mma, 7);
    }
    if (tid == 0 || tid == kExporter) bulk_wait0();  // O tiles and exported products are written
    if (tid < 64) cp_async_wait_all();
    tc_fence_before();
    __syncthreads();
#ifdef KDA_STAGE_TIMING
    if (tid < 32) atomicAdd(&g_stage_cycles[(kSummary ? 32 : 0) + tid], s_stage_cyc[tid]);
    if (tid < 128) atomicAdd(&g_warp_cycles[(kSummary ? 128 : 0) + tid], s_warp_cyc[tid]);
#endif
    if (warp == 0) tmem_dealloc(tbase, 512);
}

// Output pass of a segment whose map pass exported its per-chunk products: per
// chunk it loads the product image (double-buffered, one bulk copy) and V, and
// runs only the state chain -- the frame pass, U^T = V^T (T beta)^T followed by
// [U~ | O] += S'^T [-W^T | Qp] in one MMA group, the U~ spill, [O | S] +=
// U~^T [P | Km], and the O store.  Only the last segment's end state is stored
// (the combine pass produced the other segments' successors' start states).
namespace light {
constexpr uint32_t PROD = 0;                          // 2 product images
constexpr uint32_t V = 2 * kProdBytes;                // 2 x [64 tok][128 v]
constexpr uint32_t ST = V + 32768;                    // S'^T, 2 x [128 v][64 k]
constexpr uint32_t UT = ST + 32768;                   // U~^T, then the O tile
constexpr uint32_t MISC = UT + 16384;                 // barriers, TMEM address
static_assert(MISC + 256 <= kSmemBytes && (2 * kProdBytes) % 1024 == 0, "light shared memory plan");
}  // namespace light

template <typename OutT>
__device__ __forceinline__ void chunk_light_body(const CUtensorMap& tm_v, const CUtensorMap& tm_o, const ChunkArgs& p,
                                                 const SegItem it, const int item_id, const int h) {
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
    const int H = p.H;
    uint64_t* bars = reinterpret_cast<uint64_t*>(sm + light::MISC);  // [0],[1]: buffer loads; [2]: MMA
    uint32_t* sTmem = reinterpret_cast<uint32_t*>(bars + 4);
    constexpr int kLoader = 96;

    if (warp == 0) {
        tmem_alloc(sTmem, 256);
        tmem_relinquish();
    }
    if (tid == 32) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        mbar_init(&bars[2], 1);
        fence_mbar_init();
    }
    if (tid == 64) {
        prefetch_tmap(&tm_v);
        prefetch_tmap(&tm_o);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *sTmem;
    const uint32_t lane_off = uint32_t(quad * 32) << 16;
    const int vrow = quad * 32 + lane;
    const int t_begin = it.tok_begin, t_end = it.tok_end;
    const int nchunks = (t_end - t_begin + kC - 1) / kC;
    auto image = [&](int c) { return p.prod + ((size_t(it.slot) + c) * H + h) * kProdBytes; };
    auto issue = [&](int c) {  // chunk c's image and V into buffer c & 1
        const int b = c & 1;
        mbar_arrive_expect_tx(&bars[b], kProdBytes + 16384u);
        bulk_load_1d(sm + light::PROD + b * kProdBytes, image(c), kProdBytes, &bars[b]);
        tma_load_3d(sm + light::V + b * 16384, &tm_v, &bars[b], 0, h, t_begin + c * kC);
        tma_load_3d(sm + light::V + b * 16384 + 8192, &tm_v, &bars[b], 64, h, t_begin + c * kC);
    };
    int pend[2] = {-1, -1};  // loader thread: the chunk whose load into buffer b is in flight
    if (tid == kLoader) {
        for (int c = 0; c < 2 && c < nchunks; ++c) {
            issue(c);
            pend[c] = c;
        }
    }
    {  // start state into TMEM (S^T: lane = v, column = k): the initial state (or zero) for segment 0
        const float* src = it.g > 0 ? p.segS + (size_t(item_id) * H + h) * (kD * kD)
                                    : (p.init_state ? p.init_state + (size_t(it.seq) * H + h) * (kD * kD) : nullptr);
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
    const uint32_t id_u = idesc_bf16(128, 64, 1, 0);     // V^T (MN) x (T beta)^T (K)
    const uint32_t id_so2 = idesc_bf16(128, 128, 0, 1);  // S'^T (K) x [-W^T | Qp] (MN)
    const uint32_t id_os = idesc_bf16(128, 192, 0, 0);   // U~^T (K) x [P^T | Km] (K)
    uint32_t ph_mma = 0;
    bool aborted = false;

#pragma unroll 1
    for (int c = 0; c < nchunks; ++c) {
        const int b = c & 1, t0 = t_begin + c * kC, len = min(kC, t_end - t0);
        uint8_t* img = sm + light::PROD + b * kProdBytes;
        const uint32_t simg = sbase + light::PROD + b * kProdBytes;
        bool ok = mbar_wait(&bars[b], uint32_t((c >> 1) & 1), 1);
        if (tid == kLoader) pend[b] = -1;
        if (__syncthreads_or(!ok)) { aborted = true; break; }
        {  // S <- S post(prev); bf16 S' = S e^{mp}; TMEM S = S e^{mk}; O^T = 0
            const float* frOp = reinterpret_cast<const float*>(img + PI_FR);
            const float* frAcc = frOp + 128;
            float x[32];
#pragma unroll
            for (int cb = 0; cb < 2; ++cb) tmem_ld16(tbase + TM_S + lane_off + part * 32 + cb * 16, x + cb * 16);
            tmem_wait_ld();
            const uint32_t dst = sbase + light::ST + ((part >> 1) ? 16384u : 0u);
#pragma unroll
            for (int cb = 0; cb < 2; ++cb) {
                const int k0 = part * 32 + cb * 16, ck = (part & 1) * 4 + cb * 2;
                uint32_t pk[8];
#pragma unroll
                for (int j = 0; j < 16; j += 4) {
                    const float4 fo = *reinterpret_cast<const float4*>(frOp + k0 + j);
                    const float4 fa = *reinterpret_cast<const float4*>(frAcc + k0 + j);
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
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {  // U^T = V^T (T beta)^T, then [U~ | O] += S'^T [-W^T | Qp]
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                umma_bf16(tbase + TM_U, sdesc_sw128(sbase + light::V + b * 16384 + ks * 2048, 8192, 1024),
                          sdesc_sw128(simg + PI_TB + ks * 32, 16, 1024), id_u, ks > 0);
#pragma unroll
            for (int ks = 0; ks < 8; ++ks)
                umma_bf16(tbase + TM_U, sdesc_sw128(sbase + light::ST + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024),
                          sdesc_sw128(simg + PI_WN + ks * 2048, PI_QP - PI_WN, 1024), id_so2, 1);
            umma_commit(&bars[2]);
        }
        ok = mbar_wait(&bars[2], ph_mma, 5);
        ph_mma ^= 1;
        tc_fence_after();
        if (tid == 0) bulk_wait_read0();  // the previous O tile (over U~^T) is read out
        if (__syncthreads_or(!ok)) { aborted = true; break; }
        {  // U~^T -> smem
            float u[16];
            tmem_ld16(tbase + TM_U + lane_off + part * 16, u);
            tmem_wait_ld();
#pragma unroll
            for (int q4 = 0; q4 < 2; ++q4)
                st_shared_v4(sbase + light::UT + sw128_chunk(vrow, part * 2 + q4), pack_bf16x2(u[q4 * 8 + 0], u[q4 * 8 + 1]),
                             pack_bf16x2(u[q4 * 8 + 2], u[q4 * 8 + 3]), pack_bf16x2(u[q4 * 8 + 4], u[q4 * 8 + 5]),
                             pack_bf16x2(u[q4 * 8 + 6], u[q4 * 8 + 7]));
        }
        fence_async_smem();
        tc_fence_before();
        __syncthreads();
        if (tid == 0) {  // [O | S] += U~^T [P^T | Km]
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                umma_bf16(tbase + TM_O, sdesc_sw128(sbase + light::UT + ks * 32, 16, 1024),
                          sdesc_sw128(simg + PI_P + ks * 32, 16, 1024), id_os, 1);
            umma_commit(&bars[2]);
        }
        ok = mbar_wait(&bars[2], ph_mma, 6);
        ph_mma ^= 1;
        tc_fence_after();
        if (__syncthreads_or(!ok)) { aborted = true; break; }
        if (tid == kLoader && c + 2 < nchunks) {  // buffer b is consumed: chunk c+2 goes there
            issue(c + 2);
            pend[b] = c + 2;
        }
        bool staged = false;
        {  // O^T -> o[t0 + r, h, v]
            float ov[16];
            tmem_ld16(tbase + TM_O + lane_off + part * 16, ov);
            tmem_wait_ld();
            if (kStageO && len == kC) {
                uint8_t* so = sm + light::UT + (vrow >> 6) * 8192;
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
            tma_store_3d(&tm_o, sm + light::UT, 0, h, t0);
            tma_store_3d(&tm_o, sm + light::UT + 8192, 64, h, t0);
            bulk_commit();
        }
    }
    if (aborted) {  // let copies and MMAs still in flight land before shared memory and TMEM are released
        if (tid == kLoader) {
            for (int b = 0; b < 2; ++b)
                if (pend[b] >= 0) mbar_wait(&bars[b], uint32_t((pend[b] >> 1) & 1), 7);
        }
        if (tid == 0) mbar_wait(&bars[2], ph_mma, 7);
    } else if (it.g == it.G - 1 && p.final_state && nchunks > 0) {
        // end state = S^T(TMEM) x post(last chunk); the last image (never reloaded) holds post
        const float* post = reinterpret_cast<const float*>(sm + light::PROD + ((nchunks - 1) & 1) * kProdBytes + PI_FR) + 256;
        float* dst = p.final_state + (size_t(it.seq) * H + h) * (kD * kD);
#pragma unroll 1
        for (int cb = 0; cb < 2; ++cb) {
            const int k0 = part * 32 + cb * 16;
            float x[16];
            tmem_ld16(tbase + TM_S + lane_off + k0, x);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 16; ++j) dst[size_t(k0 + j) * kD + vrow] = x[j] * post[k0 + j];
        }
    }
    if (tid == 0) bulk_wait0();
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, 256);
}

// The (item, head) pair a CTA of a phase launch runs; false when it has none.
// Uniform plans map blockIdx.x to the item and blockIdx.y to the head.  Balanced
// plans list their items heaviest first, and consecutive CTAs (in launch order)
// take the heads of one item in turn: the longest items start first and the
// shorter ones fill the SMs that free up.
__device__ __forceinline__ bool cta_item(const ChunkArgs& p, int& item, int& h) {
    if (p.order) {
        const int lin = int(blockIdx.x + blockIdx.y * gridDim.x);
        const int r = lin / p.H;
        if (r >= *p.n_order) return false;
        item = p.order[r];
        h = lin - r * p.H;
        return true;
    }
    item = int(blockIdx.x);
    h = int(blockIdx.y);
    return item < *p.n_items;
}

// Phase 1 (and the only launch of an unsegmented call): the maps of every
// segment of a segmented sequence (the last segment's map only exports its chunk
// products, and runs only when there is room for them), and the whole output of
// an unsegmented one.  Segmented calls of a uniform plan thus run one code path
// on every SM.  In a balanced plan segment 0 needs no map: it runs its output
// from the initial state here and leaves its end state as segment 1's start.
template <typename OutT, bool kScalarGate>
__global__ void __launch_bounds__(kThreads, 1)
    chunk_phase1_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                        const __grid_constant__ CUtensorMap tm_o, const ChunkArgs p) {
    int item, h;
    if (!cta_item(p, item, h)) return;
    const SegItem it = p.items[item];
    if (it.G == 1 || (p.seg0_whole && it.g == 0))
        chunk_body<false, OutT, kScalarGate>(tm_q, tm_k, tm_v, tm_g, tm_o, p, it, item, h);
    else if (it.g < it.G - 1 || (p.prod && !p.seg0_whole))
        chunk_body<true, __nv_bfloat16, kScalarGate>(tm_q, tm_k, tm_v, tm_g, tm_o, p, it, item, h);
    else if (p.prod)  // a balanced plan's last segment: chunk products only.  (A uniform plan's segments are
                      // equal, so its phase 1 lasts as long as a full map whatever the last one does; it keeps
                      // one code path for every CTA.)
        chunk_body<true, __nv_bfloat16, kScalarGate, false>(tm_q, tm_k, tm_v, tm_g, tm_o, p, it, item, h);
}

// Phase 2: the outputs of every segment of a segmented sequence from its start
// state (the initial state, or the combine pass's), reusing the chunk products
// the map pass exported when there was room for them.
template <typename OutT, bool kScalarGate>
__global__ void __launch_bounds__(kThreads, 1)
    chunk_phase2_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                        const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_g,
                        const __grid_constant__ CUtensorMap tm_o, const ChunkArgs p) {
    int item, h;
    if (!cta_item(p, item, h)) return;
    const SegItem it = p.items[item];
    if (it.G == 1 || (p.seg0_whole && it.g == 0)) return;  // its output was written in phase 1
    if (p.prod)
        chunk_light_body<OutT>(tm_v, tm_o, p, it, item, h);
    else
        chunk_body<false, OutT, kScalarGate>(tm_q, tm_k, tm_v, tm_g, tm_o, p, it, item, h);
}

// ---------------------------------------------------------------- plan
// One CTA: per sequence n, G_n = max(1, ceil(chunks_n / L)) segments; writes the
// segment table in sequence order, the item count and (if asked) each sequence's
// first item.
// Segment 0 of a sequence has L0 chunks, the others L (the last one the rest).
__global__ void __launch_bounds__(1024) plan_kernel(const int32_t* cu, int N, int T, int L, SegItem* items,
                                                    int* n_items, int max_items, int L0, int* seq_first) {
    using Scan = cub::BlockScan<int, 1024>;
    __shared__ typename Scan::TempStorage tmp;
    __shared__ int s_base;
    if (threadIdx.x == 0) s_base = 0;
    __syncthreads();
    for (int n0 = 0; n0 < N; n0 += 1024) {
        const int n = n0 + threadIdx.x;
        int sb = 0, se = 0, G = 0;
        if (n < N) {
            sb = cu ? cu[n] : n * T;
            se = cu ? cu[n + 1] : (n + 1) * T;
            const long long nch = (se - sb + kC - 1) / kC;
            G = nch > L0 ? 1 + int((nch - L0 + L - 1) / L) : 1;
        }
        int off = 0, tot = 0;
        Scan(tmp).ExclusiveSum(G, off, tot);
        off += s_base;
        if (seq_first && n < N) seq_first[n] = off;  // the item of its first segment
        if (n < N) {
            for (int g = 0; g < G; ++g) {
                const int id = off + g;
                if (id >= max_items) break;
                SegItem s;
                s.seq = n;
                const long long c0 = g == 0 ? 0 : L0 + (long long)(g - 1) * L;
                const long long c1 = g == 0 ? L0 : c0 + L;
                s.tok_begin = int(min((long long)se, sb + c0 * kC));
                s.tok_end = int(min((long long)se, sb + c1 * kC));
                s.g = g;
                s.G = G;
                s.first = off;
                s.slot = L < (1 << 30) ? id * L : 0;  // image slots exist only in segmented plans
                s.pad1 = 0;
                items[id] = s;
            }
        }
        __syncthreads();
        if (threadIdx.x == 0) s_base += tot;
        __syncthreads();
    }
    if (threadIdx.x == 0) *n_items = min(s_base, max_items);
}

// ---------------------------------------------------------------- balanced plan
// Packed sequences whose (sequence, head) pairs are too many for the uniform plan
// (which cuts every sequence into G equal segments, G CTAs per pair) but whose
// lengths differ: unsegmented, the longest sequence alone sets the time while
// most SMs idle.  The balanced plan cuts each sequence at a common target
// length lam: segment 0 runs its output from the initial state in phase 1 (no
// map, no second pass), the later ones run a map in phase 1 and an output pass
// in phase 2, and short sequences stay whole.  lam is chosen on the device, from
// the lengths in cu_seqlens, among 16 candidates (one warp each), by a closed-form
// estimate of each phase's time: the longer of its longest CTA and its mean load
// per SM plus half a mean CTA (the tail), plus the combine pass's waves.  The
// launch order puts the longest items first, so shorter ones fill the SMs that
// free up.
constexpr int kBalMaxSeqs = 64;    // sequences a balanced plan takes
constexpr int kBalMaxItems = 128;  // segments it may cut them into
constexpr int kBalMinChunks = 16;  // shortest target segment length
constexpr int kBalCands = 16;      // target lengths tried: ceil(longest / (w + 1)), w < 16

// Costs that the plan weighs, in thousands of SM cycles on B200 (fitted to the
// phase times of forced target lengths 16-128 over three length mixes of 65536
// packed tokens, H=16, bf16 and fp32 o, all SMs busy).
struct BalCost {
    float whole;  // per chunk of an output pass from a known start state (segment 0, whole sequences)
    float map;    // per chunk of a map pass
    float prod;   // per chunk of the last segment's map pass (chunk products only, no chains)
    float item;   // per phase-1 CTA: TMEM and barriers, the start state in, the end state out
    float light;  // per chunk of a later segment's output pass
    float litem;  // per phase-2 CTA
    float comb;   // per combine step of one CTA (sequence, head, 16 columns), SMs full
    float seg;    // the extra launches' cost when anything is cut
};

// Cuts a sequence of n chunks at target length lam: segment 0 takes l0 chunks
// (r = map / whole cost: as long as a map of the others' length takes), the
// others lm (the last one the rest).  Returns the segment count G <= ceil(n/lam).
__device__ __forceinline__ int bal_split(int n, int lam, float r, int& l0, int& lm) {
    if (n <= lam) {
        l0 = n;
        lm = 0;
        return 1;
    }
    const int G0 = (n + lam - 1) / lam;
    l0 = int(roundf(float(n) * r / (r + float(G0 - 1))));
    l0 = max(1, min(l0, n - 1));
    const int rest = n - l0;
    lm = (rest + G0 - 2) / (G0 - 1);
    return 1 + (rest + lm - 1) / lm;
}

// One CTA of 512 threads (16 warps), N <= kBalMaxSeqs.  Warp w scores the target
// length of candidate w; then the best one (ties to the longer length) is cut and
// written: the segment table in sequence order (segments of a sequence adjacent,
// as the combine pass expects), each sequence's first item, the phase-1 launch
// order (all items, heaviest first), the phase-2 launch order (segments g >= 1,
// longest first) and the two counts.
__global__ void __launch_bounds__(32 * kBalCands) plan_balanced_kernel(const int32_t* cu, int N, int H, int nsm,
                                                                       BalCost cost, int max_items, SegItem* items,
                                                                       int* counts, int* seq_first, int* order1,
                                                                       int* order2) {
    __shared__ int s_n[kBalMaxSeqs], s_off[kBalMaxSeqs + 1];
    __shared__ unsigned long long s_key[kBalCands];
    __shared__ float s_k1[kBalMaxItems], s_k2[kBalMaxItems];
    __shared__ int s_maxn, s_lam, s_total;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (warp == 0) {
        int mx = 0;
        for (int n = lane; n < N; n += 32) {
            const int c = (cu[n + 1] - cu[n] + kC - 1) / kC;
            s_n[n] = c;
            mx = max(mx, c);
        }
        mx = int(__reduce_max_sync(0xffffffffu, unsigned(mx)));
        if (lane == 0) s_maxn = mx;
    }
    __syncthreads();
    const int maxn = s_maxn;
    const float r = cost.map / cost.whole;
    const int cap = min(max_items, kBalMaxItems);
    {  // this warp's candidate: sums and maxima of both phases' CTA costs
        const int w = warp;
        const int lam = max(kBalMinChunks, (maxn + w) / (w + 1));
        const bool repeat = w > 0 && lam == max(kBalMinChunks, (maxn + w - 1) / w);
        float sum1 = 0.f, max1 = 0.f, sum2 = 0.f, max2 = 0.f;
        int n1 = 0, n2 = 0, maxG = 1, steps = 0;
        for (int n = lane; n < N; n += 32) {
            int l0, lm;
            const int nch = s_n[n];
            const int G = bal_split(nch, lam, r, l0, lm);
            const float c0 = float(G == 1 ? nch : l0) * cost.whole + cost.item;
            sum1 += c0;
            max1 = fmaxf(max1, c0);
            for (int g = 1; g < G; ++g) {
                const int len = min(lm, nch - l0 - (g - 1) * lm);
                const float cm = float(len) * (g == G - 1 ? cost.prod : cost.map) + cost.item;
                const float cl = float(len) * cost.light + cost.litem;
                sum1 += cm;
                max1 = fmaxf(max1, cm);
                sum2 += cl;
                max2 = fmaxf(max2, cl);
            }
            n1 += G;
            n2 += G - 1;
            maxG = max(maxG, G);
            steps += max(0, G - 2);
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
            sum1 += __shfl_xor_sync(0xffffffffu, sum1, off);
            sum2 += __shfl_xor_sync(0xffffffffu, sum2, off);
            max1 = fmaxf(max1, __shfl_xor_sync(0xffffffffu, max1, off));
            max2 = fmaxf(max2, __shfl_xor_sync(0xffffffffu, max2, off));
        }
        n1 = __reduce_add_sync(0xffffffffu, n1);
        n2 = __reduce_add_sync(0xffffffffu, n2);
        maxG = __reduce_max_sync(0xffffffffu, maxG);
        steps = __reduce_add_sync(0xffffffffu, steps);
        float est = 3.0e38f;
        if (!repeat && n1 <= cap) {
            const float per_sm = float(H) / float(nsm);
            est = fmaxf(max1, sum1 * per_sm + 0.5f * sum1 / float(n1));
            if (n2 > 0) {  // the combine runs H x 8 CTAs per chained sequence: waves of nsm
                const int waves = max(maxG - 2, (steps * H * (kD / 16) + nsm - 1) / nsm);
                est += fmaxf(max2, sum2 * per_sm + 0.5f * sum2 / float(n2)) + cost.comb * float(waves) + cost.seg;
            }
        }
        // the lowest estimate, ties to the lowest w (the longest target length)
        if (lane == 0) s_key[w] = (static_cast<unsigned long long>(__float_as_uint(est)) << 32) | unsigned(lam);
    }
    __syncthreads();
    if (tid == 0) {
        unsigned long long best = s_key[0];
        for (int w = 1; w < kBalCands; ++w)
            if ((s_key[w] >> 32) < (best >> 32)) best = s_key[w];
        s_lam = int(best & 0xffffffffu);
    }
    __syncthreads();
    const int lam = s_lam;
    int G = 0, l0 = 0, lm = 0, nch = 0;
    if (tid < N) {
        nch = s_n[tid];
        G = bal_split(nch, lam, r, l0, lm);
        s_off[tid] = G;
    }
    __syncthreads();
    if (tid == 0) {
        int off = 0;
        for (int n = 0; n < N; ++n) {
            const int g = s_off[n];
            s_off[n] = off;
            off += g;
        }
        s_off[N] = off;
        s_total = min(off, cap);
    }
    __syncthreads();
    const int total = s_total;
    if (tid < N) {
        const int off = s_off[tid], sb = cu[tid], se = cu[tid + 1];
        seq_first[tid] = off;
        for (int g = 0; g < G && off + g < total; ++g) {
            const int c0 = g == 0 ? 0 : l0 + (g - 1) * lm;
            const int c1 = g == 0 ? (G == 1 ? nch : l0) : min(nch, c0 + lm);
            SegItem s;
            s.seq = tid;
            s.tok_begin = min(se, sb + c0 * kC);
            s.tok_end = min(se, sb + c1 * kC);
            s.g = g;
            s.G = G;
            s.first = off;
            s.slot = sb / kC + tid + c0;  // distinct for every chunk of every sequence
            s.pad1 = 0;
            items[off + g] = s;
            s_k1[off + g] = float(c1 - c0) * (g == 0 ? cost.whole : (g == G - 1 ? cost.prod : cost.map));
            s_k2[off + g] = g == 0 ? -1.f : float(c1 - c0);
        }
    }
    __syncthreads();
    if (tid < total) {  // ranks: heavier first, ties in item order
        const float a = s_k1[tid], b = s_k2[tid];
        int r1 = 0, r2 = 0;
        for (int j = 0; j < total; ++j) {
            r1 += (s_k1[j] > a) || (s_k1[j] == a && j < tid);
            r2 += s_k2[j] >= 0.f && ((s_k2[j] > b) || (s_k2[j] == b && j < tid));
        }
        order1[r1] = tid;
        if (b >= 0.f) order2[r2] = tid;
    }
    if (tid == 0) {
        counts[0] = total;
        counts[1] = total - N;
    }
}

// ---------------------------------------------------------------- combine
// Chains the segment maps of one (sequence, head, 16-column slice):
// S_{g+1} = X_g S_g + N_g, written as the start state of segment g+1 (segment 0
// gets the initial state).  With s0 = 1 (balanced plans) phase 1 has already
// written S_1, the end state of segment 0's output pass, and the chain starts there.
// X_g^T (64 KB, written transposed and column-swizzled by the summary pass) streams
// into shared memory with one 1-D bulk copy per step, double-buffered.  Each of the 8
// warps owns 16 rows of the 128 x 16 product and runs them on tf32 warp MMAs split
// three ways (hi*hi + hi*lo + lo*hi, with x = hi + lo both tf32): fp32-level
// accuracy at tensor-core latency.  The swizzle makes the A-fragment loads (4 rows
// of X^T x 8 columns per warp) hit 32 distinct banks; the slice of S is
// double-buffered with rows padded to 24 floats (conflict-free B fragments), so one
// barrier per step orders both buffers; N_{g+1}'s slice is loaded a step ahead.
constexpr int kCombCols = 16;
constexpr int kCombThreads = 256;  // 8 warps, one 16-row tile of the 128 x 16 slice each
constexpr int kCombSs = 24;        // S slice row stride in shared memory (floats)
constexpr uint32_t kCombSmem = 2 * 65536 + 2 * kD * kCombSs * 4 + 64;

// x = hi + lo, both exactly representable in tf32 (hi rounded to nearest).
__device__ __forceinline__ void split_tf32(float x, uint32_t& hi, uint32_t& lo) {
    hi = f32_to_tf32(x);
    lo = f32_to_tf32(x - __uint_as_float(hi));
}

__global__ void __launch_bounds__(kCombThreads, 1) combine_kernel(const SegItem* items, const int* n_items,
                                                                  const int* seq_first, int N, const float* init,
                                                                  const float* segN, const float* segXt,
                                                                  float* segS, int H, int s0) {
    const int n = blockIdx.x, h = blockIdx.y, z = blockIdx.z;  // one CTA per (sequence, head, slice)
    if (n >= N) return;
    const int item = seq_first[n];
    if (item < 0 || item >= *n_items) return;
    const SegItem it = items[item];
    if (it.g != 0 || it.G < 2 + s0) return;
    extern __shared__ __align__(128) uint8_t csm[];
    float* sX = reinterpret_cast<float*>(csm);                            // [2][128 k'][128 k]: X_g^T, swizzled
    float* sS = sX + 2 * kD * kD;                                         // [2][128 k][kCombSs]: S_g's slice
    uint64_t* bar = reinterpret_cast<uint64_t*>(sS + 2 * kD * kCombSs);  // [2]
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int gq = lane >> 2, tq = lane & 3;
    const int m0 = warp * 16;  // this warp's rows k
    const int c0 = kCombCols * z;
    const size_t hs = size_t(h) * (kD * kD);
    if (tid == 0) {
        mbar_init(&bar[0], 1);
        mbar_init(&bar[1], 1);
        fence_mbar_init();
    }
    __syncthreads();
    // step j = 0, 1, ..., G-2-s0 maps S_{s0+j} to S_{s0+j+1} with segment s0+j's map
    // (S_0 = the initial state; S_1 = segment 0's end state when s0 = 1)
    auto fetch = [&](int j) {
        mbar_arrive_expect_tx(&bar[j & 1], 65536u);
        bulk_load_1d(sX + (j & 1) * kD * kD, segXt + size_t(item + s0 + j) * H * (kD * kD) + hs, 65536u,
                     &bar[j & 1]);
    };
    if (tid == 0) fetch(0);
    const float* s_in = s0 ? segS + size_t(item + 1) * H * (kD * kD) + hs
                           : (init ? init + size_t(it.seq) * H * (kD * kD) + hs : nullptr);
    for (int e = tid; e < kD * kCombCols; e += kCombThreads) {
        const int kk = e / kCombCols, jj = e % kCombCols;
        sS[kk * kCombSs + jj] = s_in ? s_in[size_t(kk) * kD + c0 + jj] : 0.f;
    }
    const int steps = it.G - 1 - s0;
    // this thread's accumulators: rows m0 + gq (+8), columns 8 nt + 2 tq (+1), nt = 0, 1
    auto load_n = [&](int g, float* v) {
        const float* b = segN + size_t(item + g) * H * (kD * kD) + hs + size_t(m0 + gq) * kD + c0 + 2 * tq;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const float2 a = *reinterpret_cast<const float2*>(b + 8 * nt);
            const float2 c = *reinterpret_cast<const float2*>(b + 8 * kD + 8 * nt);
            v[nt * 4 + 0] = a.x;
            v[nt * 4 + 1] = a.y;
            v[nt * 4 + 2] = c.x;
            v[nt * 4 + 3] = c.y;
        }
    };
    float nxt[8];
    load_n(s0, nxt);
    __syncthreads();
    // A-fragment columns: k = m0 + gq (+8), swizzled by row k' = kp + tq (+4), whose low two bits are tq
    const int sw = tq << 3;
    const int ca = (m0 + gq) ^ sw, cb = (m0 + gq + 8) ^ sw;
    bool ok = true;
    int fetched = 1, j = 0;  // fetches issued (thread 0) and the step being consumed
    for (; j < steps; ++j) {
        const int g = s0 + j;  // the segment whose map this step applies
        if (tid == 0 && j + 1 < steps) {
            fetch(j + 1);
            fetched = j + 2;
        }
        float acc[8], x1[8], x2[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            acc[e] = nxt[e];
            x1[e] = x2[e] = 0.f;
        }
        if (j + 1 < steps) load_n(g + 1, nxt);
        ok = mbar_wait(&bar[j & 1], uint32_t((j >> 1) & 1), 8);
        if (__syncthreads_or(!ok)) break;
        const float* X = sX + (j & 1) * kD * kD;  // X^T: row k', column k (swizzled)
        const float* S = sS + (j & 1) * kD * kCombSs;
#pragma unroll 2
        for (int kp = 0; kp < kD; kp += 8) {
            // A (16 x 8): A[m][kk] = X^T[kp + kk][m0 + m];  B (8 x 8) per column tile: S[kp + kk][8 nt + n]
            const float* r0 = X + (kp + tq) * kD;
            const float* r4 = r0 + 4 * kD;
            uint32_t ah[4], al[4];
            split_tf32(r0[ca], ah[0], al[0]);
            split_tf32(r0[cb], ah[1], al[1]);
            split_tf32(r4[ca], ah[2], al[2]);
            split_tf32(r4[cb], ah[3], al[3]);
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                uint32_t bh[2], bl[2];
                split_tf32(S[(kp + tq) * kCombSs + 8 * nt + gq], bh[0], bl[0]);
                split_tf32(S[(kp + tq + 4) * kCombSs + 8 * nt + gq], bh[1], bl[1]);
                mma_tf32_16x8x8(acc + 4 * nt, ah[0], ah[1], ah[2], ah[3], bh[0], bh[1]);
                mma_tf32_16x8x8(x1 + 4 * nt, ah[0], ah[1], ah[2], ah[3], bl[0], bl[1]);
                mma_tf32_16x8x8(x2 + 4 * nt, al[0], al[1], al[2], al[3], bh[0], bh[1]);
            }
        }
        float* Sn = sS + ((j + 1) & 1) * kD * kCombSs;
        float* out = segS + size_t(item + g + 1) * H * (kD * kD) + hs;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            const int r = m0 + gq, cc = 8 * nt + 2 * tq;
            const float* a = acc + 4 * nt;
            const float* p1 = x1 + 4 * nt;
            const float* p2 = x2 + 4 * nt;
            const float2 v0 = make_float2(a[0] + (p1[0] + p2[0]), a[1] + (p1[1] + p2[1]));
            const float2 v1 = make_float2(a[2] + (p1[2] + p2[2]), a[3] + (p1[3] + p2[3]));
            *reinterpret_cast<float2*>(Sn + r * kCombSs + cc) = v0;
            *reinterpret_cast<float2*>(Sn + (r + 8) * kCombSs + cc) = v1;
            *reinterpret_cast<float2*>(out + size_t(r) * kD + c0 + cc) = v0;
            *reinterpret_cast<float2*>(out + size_t(r + 8) * kD + c0 + cc) = v1;
        }
        __syncthreads();  // every warp has read this X buffer and S buffer; S_{g+1} is complete
    }
    if (tid == 0 && !ok) {  // let copies still in flight land before the shared memory is released
        for (int f = j; f < fetched; ++f) mbar_wait(&bar[f & 1], uint32_t((f >> 1) & 1), 8);
    }
}

// ---------------------------------------------------------------- prep
// One warp per (token, head) row: optional L2 normalisation of q / k and a
// cast to bf16 (used for fp32 inputs or l2norm_qk).
template <typename T>
__global__ void prep_rows_kernel(const T* __restrict__ src, __nv_bfloat16* __restrict__ dst, long long rows,
                                 int normalize) {
    const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    float x[4];
    float ss = 0.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        x[u] = to_f32(src[row * kD + lane * 4 + u]);
        ss += x[u] * x[u];
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
    const float f = normalize ? rsqrtf(ss + 1e-6f) : 1.f;
#pragma unroll
    for (int u = 0; u < 4; ++u) dst[row * kD + lane * 4 + u] = __float2bfloat16_rn(x[u] * f);
}

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// [Ttot, H, 128] token tensor as a 3-D map (c, h, t); box = (bc, 1, 64).
static bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int esize, int H, long long Ttot,
                     int bc, CUtensorMapSwizzle sw) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {cuuint64_t(kD), cuuint64_t(H), cuuint64_t(Ttot)};
    cuuint64_t strides[2] = {cuuint64_t(kD) * esize, cuuint64_t(H) * kD * esize};
    cuuint32_t box[3] = {cuuint32_t(bc), 1, cuuint32_t(kC)};
    cuuint32_t es[3] = {1, 1, 1};
    return fn(m, dt, 3, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int device_sm_count() {
    int dev = 0, n = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    return n > 0 ? n : 148;
}

struct ChunkPlan {
    size_t off_prod, prod_bytes, total_min;  // product images; workspace without them
    int L0;                                  // chunks of segment 0 (L for the others)
    int N, L, max_items;
    long long Ttot;
    bool scan;
    bool balanced;  // per-sequence cuts chosen on the device (plan_balanced_kernel)
    size_t off_items, off_count, off_first, off_order1, off_order2, off_segN, off_segX, off_segS, off_q, off_k,
        off_v, total;
};

static size_t up256(size_t x) { return (x + 255) & ~size_t(255); }
constexpr size_t kPlanHead = 16;  // the item counts

// balanced_ok = false leaves packed calls with many pairs unsegmented (for workspaces
// too small for the balanced plan's per-segment states).
ChunkPlan make_chunk_plan(int B, int T, int H, int num_seqs, int dtype, int l2norm, bool varlen, int nsm,
                          bool balanced_ok = true) {
    ChunkPlan pl{};
    pl.N = varlen ? num_seqs : B;
    pl.Ttot = varlen ? (long long)T : (long long)B * T;
    const long long chunks_bound = (pl.Ttot + kC - 1) / kC + pl.N;
    const long long pairs = (long long)pl.N * H;
    int L = 1 << 30, L0 = 1 << 30;
    if (pairs > 0 && pairs * 3 <= nsm) {
        // G equal segments per sequence: one CTA per segment and pair in each phase
        const long long G = nsm / pairs;
        const long long per_seq = (chunks_bound + pl.N - 1) / pl.N;
        L = int((per_seq + G - 1) / G);
        if (L < 1) L = 1;
        L0 = L;
        if (per_seq < 3 * (long long)L) L = L0 = 1 << 30;  // too short to pay for the map pass
    }
    pl.L = L;
    pl.L0 = L0;
    pl.scan = L < (1 << 30);
    pl.max_items = int(pl.N + (pl.scan ? (chunks_bound + L - 1) / L : 0));
    // Packed sequences with too many pairs for the uniform plan: the balanced plan,
    // when the call is long enough for some sequence to be cut.  It makes at most
    // sum_n ceil(chunks_n / kBalMinChunks) <= N + chunks_bound / kBalMinChunks segments.
    if (balanced_ok && !pl.scan && varlen && pairs > 0 && pl.N <= kBalMaxSeqs &&
        (pl.Ttot + kC - 1) / kC > kBalMinChunks) {
        const long long bound = pl.N + (chunks_bound + kBalMinChunks - 1) / kBalMinChunks;
        pl.balanced = true;
        pl.scan = true;
        pl.max_items = int(bound < kBalMaxItems ? bound : kBalMaxItems);
    }
    size_t off = 0;  // the counts and the segment table first, where every plan has them
    pl.off_count = off; off = up256(off + kPlanHead);
    pl.off_items = off; off = up256(off + sizeof(SegItem) * size_t(pl.max_items));
    pl.off_first = off; off = up256(off + (pl.scan ? sizeof(int) * size_t(pl.N) : 0));
    pl.off_order1 = off; off = up256(off + (pl.balanced ? sizeof(int) * size_t(pl.max_items) : 0));
    pl.off_order2 = off; off = up256(off + (pl.balanced ? sizeof(int) * size_t(pl.max_items) : 0));
    const size_t st = size_t(pl.max_items) * H * kD * kD * sizeof(float);
    pl.off_segN = off; off = up256(off + (pl.scan ? st : 0));
    pl.off_segX = off; off = up256(off + (pl.scan ? st : 0));
    pl.off_segS = off; off = up256(off + (pl.scan ? st : 0));
    const size_t tok = size_t(pl.Ttot) * H * kD * sizeof(__nv_bfloat16);
    const bool need_qk = (dtype == KDA_FP32) || l2norm;
    pl.off_q = off; off = up256(off + (need_qk ? tok : 0));
    pl.off_k = off; off = up256(off + (need_qk ? tok : 0));
    pl.off_v = off; off = up256(off + (dtype == KDA_FP32 ? tok : 0));
    pl.total_min = off;
    // image slots: L per item in a uniform plan; one per chunk of the call in a balanced one
    const size_t slots = pl.balanced ? size_t(chunks_bound) : size_t(pl.max_items) * size_t(L);
    pl.prod_bytes = pl.scan ? slots * H * kProdBytes : 0;
    pl.off_prod = off; off = up256(off + pl.prod_bytes);
    pl.total = off;
    return pl;
}

template <int kPhase, typename O, bool G>
static int launch_phase(dim3 grid, const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                        const CUtensorMap& mg, const CUtensorMap& mo, const ChunkArgs& a, cudaStream_t stream) {
    auto kern = kPhase == 1 ? chunk_phase1_kernel<O, G> : chunk_phase2_kernel<O, G>;
    if (!set_smem_attr(kern, kSmemBytes)) return KDA_ERR_CUDA;
    kern<<<grid, kThreads, kSmemBytes, stream>>>(mq, mk, mv, mg, mo, a);
    return KDA_OK;
}

template <int kPhase>
static int launch_phase_for(int dtype, int scalar_gate, dim3 grid, const CUtensorMap& mq, const CUtensorMap& mk,
                            const CUtensorMap& mv, const CUtensorMap& mg, const CUtensorMap& mo, const ChunkArgs& a,
                            cudaStream_t stream) {
    if (dtype == KDA_FP32)
        return scalar_gate ? launch_phase<kPhase, float, true>(grid, mq, mk, mv, mg, mo, a, stream)
                           : launch_phase<kPhase, float, false>(grid, mq, mk, mv, mg, mo, a, stream);
    return scalar_gate ? launch_phase<kPhase, __nv_bfloat16, true>(grid, mq, mk, mv, mg, mo, a, stream)
                       : launch_phase<kPhase, __nv_bfloat16, false>(grid, mq, mk, mv, mg, mo, a, stream);
}

// Trace events are recorded as external event nodes when the stream is being
// captured into a CUDA graph (so a replayed graph still times each launch), and
// plainly otherwise (the external flag is refused outside a capture).
static inline void trace_record(cudaEvent_t e, cudaStream_t stream) {
    cudaStreamCaptureStatus st = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &st) == cudaSuccess && st == cudaStreamCaptureStatusActive)
        cudaEventRecordWithFlags(e, stream, cudaEventRecordExternal);
    else
        cudaEventRecord(e, stream);
}

// out_f32 != 0 writes o in fp32 whatever the input dtype (the layer's use).
int launch_chunk_fwd(const void* q, const void* k, const void* v, const float* g, const float* beta,
                     const float* init, float* fin, void* o, const int32_t* cu, int num_seqs, int B, int T, int H,
                     int dtype, float scale, int l2norm, void* ws, size_t ws_bytes, cudaStream_t stream,
                     const char** why, int scalar_gate, int out_f32) {
    const int out_dtype = (dtype == KDA_FP32 || out_f32) ? KDA_FP32 : KDA_BF16;
    ChunkPlan pl = make_chunk_plan(B, T, H, num_seqs, dtype, l2norm, cu != nullptr, device_sm_count());
    // A workspace of kda_chunk_fwd_workspace() bytes holds the exported chunk products of
    // segmented calls; one of only total_min bytes runs the same schedule recomputing them.
    // Below a balanced plan's total_min the call runs unsegmented.
    if (pl.balanced && ws_bytes < pl.total_min)
        pl = make_chunk_plan(B, T, H, num_seqs, dtype, l2norm, true, device_sm_count(), false);
    const bool products = pl.scan && ws_bytes >= pl.total;
    if (ws_bytes < pl.total_min || (pl.total_min > 0 && ws == nullptr)) {
        *why = "workspace smaller than kda_chunk_fwd_workspace()";
        return KDA_ERR_WORKSPACE;
    }
    if (pl.N == 0 || H == 0) return KDA_OK;
    uint8_t* w = static_cast<uint8_t*>(ws);
    SegItem* items = reinterpret_cast<SegItem*>(w + pl.off_items);
    int* n_items = reinterpret_cast<int*>(w + pl.off_count);
    const long long rows = pl.Ttot * H;

    const void *qb = q, *kb = k, *vb = v;
    if (dtype == KDA_FP32 || l2norm) {
        const unsigned grid = unsigned((rows + 7) / 8);
        __nv_bfloat16* dq = reinterpret_cast<__nv_bfloat16*>(w + pl.off_q);
        __nv_bfloat16* dk = reinterpret_cast<__nv_bfloat16*>(w + pl.off_k);
        if (rows > 0) {
            if (dtype == KDA_FP32) {
                prep_rows_kernel<float><<<grid, 256, 0, stream>>>(static_cast<const float*>(q), dq, rows, l2norm);
                prep_rows_kernel<float><<<grid, 256, 0, stream>>>(static_cast<const float*>(k), dk, rows, l2norm);
            } else {
                prep_rows_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(q), dq,
                                                                          rows, l2norm);
                prep_rows_kernel<__nv_bfloat16><<<grid, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(k), dk,
                                                                          rows, l2norm);
            }
        }
        qb = dq;
        kb = dk;
        if (dtype == KDA_FP32) {
            __nv_bfloat16* dv = reinterpret_cast<__nv_bfloat16*>(w + pl.off_v);
            if (rows > 0)
                prep_rows_kernel<float><<<grid, 256, 0, stream>>>(static_cast<const float*>(v), dv, rows, 0);
            vb = dv;
        }
    }

    CUtensorMap mq, mk, mv, mg, mo;
    const long long Tmap = pl.Ttot > 0 ? pl.Ttot : 1;
    if (!make_map(&mq, qb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, H, Tmap, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mk, kb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, H, Tmap, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !make_map(&mv, vb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, H, Tmap, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        // scalar gates are fetched per row, not by TMA: the g map is then a placeholder
        !make_map(&mg, scalar_gate ? kb : g, scalar_gate ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                  scalar_gate ? 2 : 4, H, Tmap, scalar_gate ? 64 : 128,
                  scalar_gate ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE) ||
        !make_map(&mo, out_dtype == KDA_FP32 ? vb : o, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, H, Tmap, 64,
                  CU_TENSOR_MAP_SWIZZLE_128B)) {
        *why = "cuTensorMapEncodeTiled failed";
        return KDA_ERR_CUDA;
    }

    cudaEvent_t* ev = g_trace_events;
    if (ev) trace_record(ev[0], stream);
    int* seq_first = pl.scan ? reinterpret_cast<int*>(w + pl.off_first) : nullptr;
    int* order1 = pl.balanced ? reinterpret_cast<int*>(w + pl.off_order1) : nullptr;
    int* order2 = pl.balanced ? reinterpret_cast<int*>(w + pl.off_order2) : nullptr;
    if (pl.balanced) {
        // per-chunk costs of the three passes, measured at d = 128 on B200 (the output
        // passes a little dearer with an fp32 o).  The later segments' output passes
        // are costed as reading back exported products even when the workspace has
        // no room for them: the cuts, and so the results, do not depend on its size.
        BalCost cost;
        const bool f32 = out_dtype == KDA_FP32;
        cost.whole = f32 ? 14.7f : 13.4f;
        cost.map = 17.0f;
        cost.prod = 13.0f;
        cost.item = 20.0f;
        cost.light = f32 ? 6.4f : 4.8f;
        cost.litem = f32 ? 13.0f : 10.0f;
        cost.comb = 8.45f;
        cost.seg = 20.0f;
        plan_balanced_kernel<<<1, 32 * kBalCands, 0, stream>>>(cu, pl.N, H, device_sm_count(), cost, pl.max_items,
                                                                items, n_items, seq_first, order1, order2);
    } else {
        plan_kernel<<<1, 1024, 0, stream>>>(cu, pl.N, T, pl.L, items, n_items, pl.max_items, pl.L0, seq_first);
    }
    if (ev) trace_record(ev[1], stream);

    ChunkArgs a{};
    a.beta = beta;
    a.prod = products ? w + pl.off_prod : nullptr;
    a.gs = scalar_gate ? g : nullptr;
    a.init_state = init;
    a.final_state = fin;
    a.o = o;
    a.items = items;
    a.n_items = n_items;
    a.segN = reinterpret_cast<float*>(w + pl.off_segN);
    a.segX = reinterpret_cast<float*>(w + pl.off_segX);
    a.segS = reinterpret_cast<float*>(w + pl.off_segS);
    a.order = order1;
    a.n_order = n_items;
    a.seg0_whole = pl.balanced ? 1 : 0;
    a.H = H;
    a.scale = scale;
    const dim3 grid(unsigned(pl.max_items), unsigned(H));
    if (!pl.scan && ev) {  // one launch: it is timed as the output pass
        trace_record(ev[2], stream);
        trace_record(ev[3], stream);
    }
    const int r1 = launch_phase_for<1>(out_dtype, scalar_gate, grid, mq, mk, mv, mg, mo, a, stream);
    if (r1 != KDA_OK) return r1;
    if (pl.scan) {
        if (ev) trace_record(ev[2], stream);
        if (!set_smem_attr(combine_kernel, kCombSmem)) return KDA_ERR_CUDA;
        combine_kernel<<<dim3(unsigned(pl.N), unsigned(H), kD / kCombCols), kCombThreads, kCombSmem, stream>>>(
            items, n_items, seq_first, pl.N, init, a.segN, a.segX, reinterpret_cast<float*>(w + pl.off_segS), H,
            pl.balanced ? 1 : 0);
        if (ev) trace_record(ev[3], stream);
        ChunkArgs a2 = a;  // a balanced plan launches only the segments g >= 1, longest first
        a2.order = order2;
        a2.n_order = n_items + 1;
        const dim3 grid2 = pl.balanced ? dim3(unsigned(pl.max_items > pl.N ? pl.max_items - pl.N : 1), unsigned(H)) : grid;
        const int r2 = launch_phase_for<2>(out_dtype, scalar_gate, grid2, mq, mk, mv, mg, mo, a2, stream);
        if (r2 != KDA_OK) return r2;
    }
    if (ev) trace_record(ev[4], stream);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        *why = cudaGetErrorString(e);
        return KDA_ERR_CUDA;
    }
    return KDA_OK;
}

#ifdef KDA_STAGE_TIMING
extern "C" int kda_debug_stage_cycles(unsigned long long* out, int reset) {
    if (cudaMemcpyFromSymbol(out, g_stage_cycles, sizeof(unsigned long long) * 64) != cudaSuccess) return 1;
    if (reset) {
        unsigned long long z[64] = {};
        cudaMemcpyToSymbol(g_stage_cycles, z, sizeof(z));
    }
    return 0;
}
extern "C" int kda_debug_warp_cycles(unsigned long long* out, int reset) {
    if (cudaMemcpyFromSymbol(out, g_warp_cycles, sizeof(unsigned long long) * 256) != cudaSuccess) return 1;
    if (reset) {
        unsigned long long z[256] = {};
        cudaMemcpyToSymbol(g_warp_cycles, z, sizeof(z));
    }
    return 0;
}
#endif

int chunk_segment_tokens(int B, int T, int H, int num_seqs, int* middle) {
    const ChunkPlan pl = make_chunk_plan(B, T, H, num_seqs, KDA_BF16, 0, num_seqs > 0, device_sm_count());
    if (pl.balanced) {  // cut per sequence on the device
        if (middle) *middle = -1;
        return -1;
    }
    if (middle) *middle = pl.scan ? pl.L * kC : 0;
    return pl.scan ? pl.L0 * kC : 0;
}

// The segment table a call with these sizes left in its workspace (it sits at the
// workspace's start, so dtype and l2norm do not move it).
int chunk_plan_items(const void* ws, int B, int T, int H, int num_seqs, int* rows, int max_rows) {
    ChunkPlan pl = make_chunk_plan(B, T, H, num_seqs, KDA_BF16, 0, num_seqs > 0, device_sm_count());
    const ChunkPlan flat = make_chunk_plan(B, T, H, num_seqs, KDA_BF16, 0, num_seqs > 0, device_sm_count(), false);
    if (flat.max_items > pl.max_items) pl.max_items = flat.max_items;  // either may have run
    const uint8_t* w = static_cast<const uint8_t*>(ws);
    int n = 0;
    if (cudaMemcpy(&n, w + pl.off_count, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return -1;
    if (n < 0 || n > pl.max_items) return -1;
    const int k = n < max_rows ? n : max_rows;
    for (int i = 0; i < k; ++i) {
        SegItem it;
        if (cudaMemcpy(&it, w + pl.off_items + sizeof(SegItem) * size_t(i), sizeof(SegItem), cudaMemcpyDeviceToHost) !=
            cudaSuccess)
            return -1;
        const int r[5] = {it.seq, it.tok_begin, it.tok_end, it.g, it.G};
        for (int j = 0; j < 5; ++j) rows[5 * i + j] = r[j];
    }
    return n;
}

size_t chunk_workspace_bytes(int B, int T, int H, int num_seqs, int dtype, int l2norm) {
    return make_chunk_plan(B, T, H, num_seqs, dtype, l2norm, num_seqs > 0, device_sm_count()).total;
}

// The smallest workspace kda_chunk_fwd accepts (a uniform segmented schedule then
// recomputes the chunk products in its output pass instead of reading them back; a
// call that would take the balanced plan runs unsegmented).
size_t chunk_workspace_bytes_min(int B, int T, int H, int num_seqs, int dtype, int l2norm) {
    return make_chunk_plan(B, T, H, num_seqs, dtype, l2norm, num_seqs > 0, device_sm_count(), false).total_min;
}

}  // namespace kda
