// The KDA layer's projection GEMMs on sm_100a: C = A W^T with A [M, K] and
// W [N, K] bf16 row-major (both K-major), fp32 accumulation in tensor memory.
//
// "Kimi Linear: An Expressive, Efficient Attention Architecture", section
// "Neural Parameterization" and "Code Verification": the layer's bias-free
// Q/K/V projections (with the low-rank gate down-projections and the beta
// projection stacked into one input GEMM), the rank-128 up-projections of the
// decay and of the output gate, and the output projection.  These are ~94% of
// the layer's FLOPs, so they run on the 5th-generation tensor cores:
//
//  * Persistent kernel, one CTA per SM, tiles of 128 x 256 walked in row-major
//    tile order (all N tiles of an M block before the next M block) so that
//    the CTAs running at one time share the A rows in L2 and the weights stay
//    L2-resident.
//  * Warp roles: warp 0 issues the TMA loads (128B-swizzled 64-wide K slices
//    of A and W into a 4-stage ring), one thread of warp 1 issues
//    tcgen05.mma (M = 128, N = 256, K = 16 per instruction) into one of two
//    256-column fp32 accumulators in TMEM, and 8 epilogue warps drain the
//    other accumulator meanwhile (warp w reads TMEM lanes 32 (w % 4) ..
//    + 31, i.e. 32 rows, and one 128-column half).  A tile narrower than 256
//    at the right edge issues MMAs of the width it needs (N a multiple of 16).
//  * Epilogues (the layer's elementwise steps fused into the GEMM that makes
//    their input, so the intermediate never goes to HBM):
//      kStoreBf16  : C in bf16 through a swizzled staging tile and TMA stores;
//                    optionally the columns [beta_col0, beta_col0 + H) are also
//                    written as beta = sigmoid(c) in fp32 ([M, H]).
//      kNegSoftplus: g = -softplus(c) in fp32 (the per-channel log decay,
//                    alpha = exp(-softplus(a))).
//      kNormGate   : out = RMSNorm_head(o) * norm_w * sigmoid(c), o in fp32
//                    from the operator; each 128-column half of a tile is one
//                    head.  Each epilogue warp TMA-loads its 32 x 128 block of
//                    o into shared memory, so every thread reads its row there,
//                    and stores the result from the same buffer.
// Every wait is bounded (kda_common.cuh); a wait that gives up records
// KDA_ERR_TIMEOUT and the kernel winds down without a trap.
#include "kda_gemm.cuh"

namespace kda {

int device_sm_count();

namespace gemm {

constexpr int BM = 128, BN = 256, BK = 64;
constexpr uint32_t kABytes = BM * BK * 2;           // 16 KB
constexpr uint32_t kBBytes = BN * BK * 2;           // 32 KB
constexpr uint32_t kStageBytes = kABytes + kBBytes;  // 48 KB
constexpr int kEpiWarps = 8;
constexpr int kThreads = 64 + kEpiWarps * 32;  // producer warp, MMA warp, epilogue warps

constexpr int kStoreBf16 = GemmEpilogue::kStoreBf16, kNegSoftplus = GemmEpilogue::kNegSoftplus,
              kNormGate = GemmEpilogue::kNormGate;

// Shared-memory plan per epilogue: the operand ring, one staging area per epilogue warp,
// barriers.  kStoreBf16 (the K = d_model projections): four stages, one 32 x 128 B output
// tile per warp.  The two rank-128 GEMMs have K = 128 (two K slices), so two stages hold a
// whole tile's operands and each warp gets 16 KB: kNegSoftplus four output tiles (one per
// 32 columns, so a tile's stores never wait for each other), kNormGate its 32 x 128 fp32
// block of o (which its output then reuses).
template <int kEpi> struct Plan {
    static constexpr int kStages = kEpi == kStoreBf16 ? 4 : 2;
    static constexpr uint32_t kStagingBytes = kEpi == kStoreBf16 ? 4096 : 16384;
    static constexpr uint32_t OFF_STAGING = kStages * kStageBytes;
    static constexpr uint32_t OFF_BARS = OFF_STAGING + kEpiWarps * kStagingBytes;
    static constexpr uint32_t kSmem = OFF_BARS + 256 + 1024;  // + slack to align the base to 1024 B
    static_assert(kSmem <= 232448, "GEMM shared-memory plan");
};

struct Args {
    int M, N, K;
    int tiles_m, tiles_n;
    float* beta_out;  // kStoreBf16: sigmoid of columns [beta_col0, beta_col0 + H), [M][H] fp32
    int beta_col0, H;
    const float* o_in;  // kNormGate: operator output fp32 [M][ldo]
    int ldo;
    const float* norm_w;  // kNormGate: [128]
};

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
            smem_u32(dst)),
        "l"(map), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
        : "memory");
}
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int c0, int c1) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(map),
                 "r"(smem_u32(src)), "r"(c0), "r"(c1)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
// 32 lanes x 32 consecutive fp32 columns of TMEM (this warp's lane quadrant).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%"
        "19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
          "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
          "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi) {
    const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&p);
}
// One row of 128 bytes (8 chunks of 16 B) into a 128B-swizzled staging tile.
__device__ __forceinline__ void stage_row(uint32_t tile, int row, const uint32_t* w32) {
#pragma unroll
    for (int j = 0; j < 8; ++j)
        st_shared_v4(tile + sw128_chunk(row, j), w32[4 * j], w32[4 * j + 1], w32[4 * j + 2], w32[4 * j + 3]);
}

template <int kEpi>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                const __grid_constant__ CUtensorMap map_c, const __grid_constant__ CUtensorMap map_o,
                const Args p) {
    constexpr int kStages = Plan<kEpi>::kStages;
    constexpr uint32_t kStagingBytes = Plan<kEpi>::kStagingBytes;
    constexpr uint32_t OFF_STAGING = Plan<kEpi>::OFF_STAGING;
    constexpr uint32_t OFF_BARS = Plan<kEpi>::OFF_BARS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(sm);
    uint64_t* full = reinterpret_cast<uint64_t*>(sm + OFF_BARS);
    uint64_t* empty = full + kStages;
    uint64_t* acc_full = empty + kStages;
    uint64_t* acc_empty = acc_full + 2;
    uint64_t* obar = acc_empty + 2;  // kNormGate: per epilogue warp, its block of o has landed
    uint32_t* sTmem = reinterpret_cast<uint32_t*>(obar + kEpiWarps);
    volatile int* sAbort = reinterpret_cast<volatile int*>(sTmem + 1);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int total = p.tiles_m * p.tiles_n;
    const int nkb = (p.K + BK - 1) / BK;

    if (warp == 0) {
        tmem_alloc(sTmem, 512);
        tmem_relinquish();
    }
    if (tid == 32) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], kEpiWarps);
        }
        for (int w = 0; w < kEpiWarps; ++w) mbar_init(&obar[w], 1);
        *sAbort = 0;
        fence_mbar_init();
    }
    if (tid == 64) {
        prefetch_tmap(&map_a);
        prefetch_tmap(&map_b);
        prefetch_tmap(&map_c);
        if (kEpi == kNormGate) prefetch_tmap(&map_o);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *sTmem;

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int issued = 0;  // loads whose full barrier may still be pending at exit
            for (int t = blockIdx.x; t < total && !*sAbort; t += gridDim.x) {
                const int m0 = (t / p.tiles_n) * BM, n0 = (t % p.tiles_n) * BN;
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait(&empty[stage], phase ^ 1, 8)) {
                        *sAbort = 1;
                        break;
                    }
                    uint8_t* sa = sm + stage * kStageBytes;
                    mbar_arrive_expect_tx(&full[stage], kStageBytes);
                    tma_load_2d(sa, &map_a, &full[stage], kb * BK, m0);
                    tma_load_2d(sa + kABytes, &map_b, &full[stage], kb * BK, n0);
                    ++issued;
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
            if (*sAbort) {  // let every load this thread issued land before the CTA exits
                for (int s = 0; s < kStages && issued > 0; ++s, --issued) {
                    if (--stage < 0) {
                        stage = kStages - 1;
                        phase ^= 1;
                    }
                    mbar_wait(&full[stage], phase, 9);
                }
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int i = 0;
            bool pending = false;  // a commit whose barrier may not have arrived yet
            for (int t = blockIdx.x; t < total && !*sAbort; t += gridDim.x, ++i) {
                const int buf = i & 1;
                const uint32_t aph = (i >> 1) & 1;
                const int n0 = (t % p.tiles_n) * BN;
                int nw = p.N - n0;
                nw = nw >= BN ? BN : ((nw + 15) & ~15);
                const uint32_t idesc = idesc_bf16(BM, nw, 0, 0);
                if (!mbar_wait(&acc_empty[buf], aph ^ 1, 10)) {
                    *sAbort = 1;
                    break;
                }
                tc_fence_after();
                const uint32_t dtm = tbase + uint32_t(buf * BN);
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!mbar_wait(&full[stage], phase, 11)) {
                        *sAbort = 1;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = sbase + stage * kStageBytes;
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)
                        umma_bf16(dtm, sdesc_sw128(sa + k * 32, 16, 1024), sdesc_sw128(sa + kABytes + k * 32, 16, 1024),
                                  idesc, (kb | k) != 0);
                    umma_commit(&empty[stage]);
                    pending = true;
                    if (++stage == kStages) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                if (*sAbort) break;
                umma_commit(&acc_full[buf]);
            }
            if (*sAbort && pending) {  // the last MMAs still read shared memory: let them finish
                const int last = (stage + kStages - 1) % kStages;
                mbar_wait(&empty[last], stage == 0 ? phase ^ 1 : phase, 12);
            }
        }
    } else {
        // ---------------------------------------------------------------- epilogue
        const int ew = warp - 2;             // 0..7
        const int quad = warp & 3;           // TMEM lane quadrant this warp may read
        const int half = ew >> 2;            // column half of the 256-wide tile
        const uint32_t stg = sbase + OFF_STAGING + uint32_t(ew) * kStagingBytes;
        uint8_t* stg_p = sm + OFF_STAGING + ew * kStagingBytes;
        // kNormGate: this warp's 32 x 128 fp32 block of o for tile t (its 32 rows, its head),
        // as four 32 x 32 boxes (128B-swizzled rows), landing on obar[ew].  The next tile's
        // block is requested as soon as this tile's output stores have read the buffer.
        auto has_o = [&](int t) { return t < total && ((t % p.tiles_n) * BN + half * 128) < p.N; };
        auto load_o = [&](int t) {
            const int r0 = (t / p.tiles_n) * BM + quad * 32, c0 = (t % p.tiles_n) * BN + half * 128;
            mbar_arrive_expect_tx(&obar[ew], 16384u);
#pragma unroll
            for (int b = 0; b < 4; ++b) tma_load_2d(stg_p + b * 4096, &map_o, &obar[ew], c0 + 32 * b, r0);
        };
        bool o_pend = false;  // lane 0: a load of o issued and not yet waited for
        uint32_t o_ph = 0;    // phase of obar[ew] the next load completes
        if (kEpi == kNormGate && lane == 0 && has_o(blockIdx.x)) {
            load_o(blockIdx.x);
            o_pend = true;
        }
        int i = 0;
        for (int t = blockIdx.x; t < total; t += gridDim.x, ++i) {
            const int buf = i & 1;
            const uint32_t aph = (i >> 1) & 1;
            const int m0 = (t / p.tiles_n) * BM, n0 = (t % p.tiles_n) * BN;
            const bool ok = mbar_wait(&acc_full[buf], aph, 13);
            if (__any_sync(0xffffffffu, !ok) || *sAbort) {
                *sAbort = 1;
                break;
            }
            tc_fence_after();
            const uint32_t tacc = tbase + uint32_t(buf * BN) + (uint32_t(quad * 32) << 16);
            const int row = m0 + quad * 32 + lane;  // output row of this thread
            const int cols = min(BN, p.N - n0);     // valid columns of this tile
            if constexpr (kEpi == kStoreBf16) {
#pragma unroll 1
                for (int ch = 0; ch < 2; ++ch) {
                    const int c0 = half * 128 + ch * 64;  // tile column of this 64-wide chunk
                    if (c0 >= cols) break;
                    float v[64];
                    tmem_ld32(tacc + c0, v);
                    tmem_ld32(tacc + c0 + 32, v + 32);
                    tmem_wait_ld();
                    if (p.beta_out) {  // the beta columns: sigmoid in fp32 as well
                        const int b0 = p.beta_col0 - (n0 + c0);
                        if (b0 < 64 && b0 + p.H > 0 && row < p.M) {
#pragma unroll
                            for (int j = 0; j < 64; ++j) {
                                const int hcol = j - b0;
                                if (hcol >= 0 && hcol < p.H)
                                    p.beta_out[size_t(row) * p.H + hcol] = __fdividef(1.f, 1.f + __expf(-v[j]));
                            }
                        }
                    }
                    uint32_t w32[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j) w32[j] = bf16x2_rn(v[2 * j], v[2 * j + 1]);
                    if (lane == 0) bulk_wait_read0();  // the previous store has read the staging tile
                    __syncwarp();
                    stage_row(stg, lane, w32);
                    fence_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(&map_c, sm + OFF_STAGING + ew * kStagingBytes, n0 + c0, m0 + quad * 32);
                        bulk_commit();
                    }
                }
            } else if constexpr (kEpi == kNegSoftplus) {
                if (lane == 0) bulk_wait_read0();  // the previous tile's stores have read their tiles
                __syncwarp();
#pragma unroll 1
                for (int ch = 0; ch < 4; ++ch) {
                    const int c0 = half * 128 + ch * 32;
                    if (c0 >= cols) break;
                    float v[32];
                    tmem_ld32(tacc + c0, v);
                    tmem_wait_ld();
                    uint32_t w32[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const float x = v[j];
                        // softplus(x) = max(x, 0) + log(1 + e^-|x|); below e^-|x| ~ 6e-8 the log
                        // term rounds to 0, an absolute error under 1e-7 in the log decay
                        w32[j] = __float_as_uint(-(fmaxf(x, 0.f) + __logf(1.f + __expf(-fabsf(x)))));
                    }
                    stage_row(stg + ch * 4096, lane, w32);
                    fence_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(&map_c, stg_p + ch * 4096, n0 + c0, m0 + quad * 32);
                        bulk_commit();
                    }
                }
            } else {  // kNormGate: this warp's half is one head of 128 channels, for its 32 rows
                if (half * 128 < cols) {
                    const bool okw = mbar_wait(&obar[ew], o_ph, 14);
                    o_ph ^= 1;
                    o_pend = false;
                    if (__any_sync(0xffffffffu, !okw)) {
                        *sAbort = 1;
                        break;
                    }
                    // the row's sum of squares over the head (its 128 B rows in the four boxes)
                    float ss = 0.f;
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const float4 x = *reinterpret_cast<const float4*>(stg_p + (j >> 3) * 4096 + sw128_chunk(lane, j & 7));
                        ss += x.x * x.x + x.y * x.y + x.z * x.z + x.w * x.w;
                    }
                    const float rs = rsqrtf(ss * (1.f / 128.f) + 1e-5f);
#pragma unroll 1
                    for (int cp = 0; cp < 2; ++cp) {  // 64 channels: boxes 2cp and 2cp+1 of the block
#pragma unroll
                        for (int hb = 0; hb < 2; ++hb) {
                            const int b = 2 * cp + hb;
                            float v[32];
                            tmem_ld32(tacc + half * 128 + b * 32, v);
                            tmem_wait_ld();
                            uint32_t w16[16];
#pragma unroll
                            for (int j = 0; j < 8; ++j) {
                                const float4 x = *reinterpret_cast<const float4*>(stg_p + b * 4096 + sw128_chunk(lane, j));
                                const float4 nw = reinterpret_cast<const float4*>(p.norm_w + b * 32)[j];
                                const float r0 = __fdividef(x.x * rs * nw.x, 1.f + __expf(-v[4 * j]));
                                const float r1 = __fdividef(x.y * rs * nw.y, 1.f + __expf(-v[4 * j + 1]));
                                const float r2 = __fdividef(x.z * rs * nw.z, 1.f + __expf(-v[4 * j + 2]));
                                const float r3 = __fdividef(x.w * rs * nw.w, 1.f + __expf(-v[4 * j + 3]));
                                w16[2 * j] = bf16x2_rn(r0, r1);
                                w16[2 * j + 1] = bf16x2_rn(r2, r3);
                            }
                            // bf16 output (32 channels, 64 B) into this lane's own row of box 2cp,
                            // which it has finished reading (box 2cp+1 is read after box 2cp)
#pragma unroll
                            for (int c = 0; c < 4; ++c)
                                st_shared_v4(stg + 2 * cp * 4096 + sw128_chunk(lane, 4 * hb + c), w16[4 * c],
                                             w16[4 * c + 1], w16[4 * c + 2], w16[4 * c + 3]);
                        }
                        // one TMA store per 64 channels
                        fence_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_2d(&map_c, stg_p + 2 * cp * 4096, n0 + half * 128 + 64 * cp, m0 + quad * 32);
                            bulk_commit();
                        }
                    }
                    // the stores must have read the buffer before the next block of o lands in it
                    const int tn = t + gridDim.x;
                    if (lane == 0 && has_o(tn)) {
                        bulk_wait_read0();
                        load_o(tn);
                        o_pend = true;
                    }
                }
            }
            // this warp has read its part of the accumulator: hand it back to the MMA warp
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[buf]);
        }
        if (lane == 0) {
            if (o_pend) mbar_wait(&obar[ew], o_ph, 15);  // after an abort: let a load still in flight land
            bulk_wait0();  // every store of this warp has completed
        }
        __syncwarp();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) tmem_dealloc(tbase, 512);
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

// Row-major [rows, cols] matrix with row stride ld elements as a 2-D map (col, row), 128B swizzle.
static bool map_2d(CUtensorMap* m, const void* base, bool f32, long long rows, long long cols, long long ld,
                   int box_cols, int box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const int es = f32 ? 4 : 2;
    cuuint64_t dims[2] = {cuuint64_t(cols), cuuint64_t(rows)};
    cuuint64_t strides[1] = {cuuint64_t(ld) * es};
    cuuint32_t box[2] = {cuuint32_t(box_cols), cuuint32_t(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base),
              dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace gemm

// Requirements (checked): 16-byte aligned bases and row strides; for kNegSoftplus and
// kNormGate N a multiple of 128, and (kNormGate) o 16-byte aligned with ldo a multiple of 4.
int launch_gemm(const void* A, int lda, const void* W, int ldw, void* C, int ldc, int M, int N, int K,
                const GemmEpilogue& ep, cudaStream_t stream, const char** why) {
    using namespace gemm;
    if (M <= 0 || N <= 0) return KDA_OK;
    const bool f32_out = ep.kind == kNegSoftplus;
    if (K <= 0 || lda < K || ldw < K || ldc < N || !aligned(A, 16) || !aligned(W, 16) || !aligned(C, 16) ||
        (lda * 2) % 16 || (ldw * 2) % 16 || (ldc * (f32_out ? 4 : 2)) % 16) {
        *why = "GEMM operands must be 16-byte aligned with 16-byte row strides";
        return KDA_ERR_INVALID_ARG;
    }
    if (ep.kind != kStoreBf16 && N % 128) {
        *why = "fused GEMM epilogues need N to be a multiple of 128";
        return KDA_ERR_INVALID_ARG;
    }
    if (ep.kind == kNormGate && (!ep.o_in || !ep.norm_w || ep.ldo % 4 || ep.ldo < N || !aligned(ep.o_in, 16) ||
                                 !aligned(ep.norm_w, 16))) {
        *why = "norm-gate epilogue needs 16-byte aligned o and norm_w";
        return KDA_ERR_INVALID_ARG;
    }
    CUtensorMap ma, mb, mc, mo;
    if (!map_2d(&ma, A, false, M, K, lda, BK, BM) || !map_2d(&mb, W, false, N, K, ldw, BK, BN) ||
        !map_2d(&mc, C, f32_out, M, N, ldc, f32_out ? 32 : 64, 32) ||
        !(ep.kind == kNormGate ? map_2d(&mo, ep.o_in, true, M, N, ep.ldo, 32, 32) : (mo = mc, true))) {
        *why = "cuTensorMapEncodeTiled failed for a GEMM operand";
        return KDA_ERR_CUDA;
    }
    Args a{};
    a.M = M;
    a.N = N;
    a.K = K;
    a.tiles_m = (M + BM - 1) / BM;
    a.tiles_n = (N + BN - 1) / BN;
    a.beta_out = ep.beta_out;
    a.beta_col0 = ep.beta_col0;
    a.H = ep.H;
    a.o_in = ep.o_in;
    a.ldo = ep.ldo;
    a.norm_w = ep.norm_w;
    const long long tiles = (long long)a.tiles_m * a.tiles_n;
    const int grid = int(tiles < device_sm_count() ? tiles : device_sm_count());
    auto kern = ep.kind == kStoreBf16 ? gemm_kernel<kStoreBf16>
                                      : (ep.kind == kNegSoftplus ? gemm_kernel<kNegSoftplus> : gemm_kernel<kNormGate>);
    const uint32_t smem = ep.kind == kStoreBf16 ? Plan<kStoreBf16>::kSmem
                                                : (ep.kind == kNegSoftplus ? Plan<kNegSoftplus>::kSmem
                                                                           : Plan<kNormGate>::kSmem);
    if (!set_smem_attr(kern, smem)) {
        *why = "cudaFuncSetAttribute failed for the GEMM kernel";
        return KDA_ERR_CUDA;
    }
    kern<<<grid, gemm::kThreads, smem, stream>>>(ma, mb, mc, mo, a);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        *why = cudaGetErrorString(e);
        return KDA_ERR_CUDA;
    }
    return KDA_OK;
}

}  // namespace kda
