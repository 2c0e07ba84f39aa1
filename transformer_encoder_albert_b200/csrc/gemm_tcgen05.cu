// gemm_tcgen05.cu -- persistent BF16 GEMM for sm_100a: Y = epi(A W^T + bias).
//
// The dense contractions of the encoder (the fused Q|K|V projection, the
// attention output projection, both FFN matrices and the 768->512 final
// projection; "ALBERT: How Kokoro's Phoneme Encoder Works", section "Inside One
// Real ALBERT Layer", steps 3-6) run here; the 128->768 input projection (step
// 2) runs inside the embedding kernel (embed_proj.cu) and, through the test
// entry, here as well.
// A linear layer is y_j = b_j + sum_i x_i W_{j,i} with W stored [out, in]
// ("Qwen3-TTS and Kokoro", section A), i.e. both operands are K-major.
//
// Design (one CTA per SM, persistent over output tiles; three variants):
//   * single CTA per 128x256 tile: 3-stage ring of {A 128x64, B 256x64};
//   * single CTA per 128x128 tile ("narrow"): 5-stage ring of {A 128x64,
//     B 128x64}, epilogue on one warp per lane quadrant -- for few rows, where
//     256x256 pair tiles would leave SMs idle;
//   * CTA pair (cluster of 2, tcgen05.mma cta_group::2) per 256x256 tile: each
//     CTA stages its 128 rows of A and 128 rows of B, 5-stage ring of
//     {A 128x64, B 128x64} per CTA (the pair is used whenever A has more than
//     one 128-row block).
//   warp 0      : TMA producer of the ring (bf16 tiles, 128-byte swizzle, no
//                 multicast);
//   warp 1      : TMEM allocator + single-thread tcgen05.mma issuer into two
//                 128x256 fp32 accumulators (512 TMEM columns), so the epilogue
//                 of one tile overlaps the main loop of the next;
//   warps 2..9  : epilogue, 2 warps per TMEM lane quadrant (column halves);
//                 tcgen05.ld -> epilogue math -> bf16 32x32 tile in a swizzled
//                 shared staging buffer (two, used alternately, when the
//                 epilogue has no residual) -> TMA bulk tensor store
//                 (coalesced, asynchronous; one-row-per-lane global stores
//                 would contend with the tensor core's shared-memory operand
//                 reads in the unified L1/shared array).
//
// Post-LN LayerNorms (steps 5 and 6) are deferred to the consumers of their
// output, so every epilogue is a single pass with no cross-CTA dependency:
//   * the GEMM that forms the pre-norm row z = acc + bias + residual writes
//     z * gamma (bf16) and, per row and 128-column slice, exact (mean, M2)
//     statistics of z (two-pass inside each 32-column chunk, Chan's merge
//     across chunks);
//   * a GEMM that reads z * gamma as its A operand merges the six partial
//     statistics of its row into (mu, rstd) and applies
//     LN(z) W^T = rstd * (z*gamma) W^T - rstd * mu * (W gamma) + W beta;
//   * a GEMM whose residual is LN(z) rebuilds it from the z*gamma tile as
//     rstd * (z*gamma) - rstd * mu * gamma + beta.
// Residual tiles arrive by TMA into a second per-warp staging tile, one
// 32-column chunk ahead.  Every wait is bounded (%globaltimer); on expiry the
// CTA records ALBERT_ERR_TIMEOUT, drains its in-flight copies and MMAs, frees
// TMEM and exits.
#include "kernels.h"
#include "sm100_ptx.cuh"

namespace albert {
namespace {

using namespace gemm;

// Shared-memory plan of one kernel instance: {A, B} pipeline stages, then 2 KB
// staging tiles per epilogue warp (output, residual or second output, and for
// the residual epilogue a second output tile, paid for with one stage), then
// barriers; 1 KiB slack for the 1 KiB alignment of the stages.
template <int EPI, bool PAIR, bool F8 = false, int TBN = BN>
struct Plan {
    static constexpr bool kRes = EPI == kEpiResStats;
    static constexpr bool kLnIn = EPI == kEpiLnIn || EPI == kEpiLnInGelu || EPI == kEpiLnInScatter;
    // (128-column tiles halve the B stage, which buys two more stages)
    static constexpr int NST = PAIR ? PAIR_STAGES - 1 : (TBN == 128 ? STAGES + 1 : STAGES - 1);
    static constexpr int BSTAGE = PAIR ? B_HALF_BYTES : TBN * 128;  // TBN rows of 128 bytes
    static constexpr int NSTG = kRes ? 3 : 2;
    // per-column vectors of a unit: bias, then W gamma (LayerNorm input) or
    // out_g and res_g (residual epilogue), then for E4M3 operands the weight
    // row scales; two buffers (this unit, the next)
    static constexpr int NVEC_BASE = kLnIn ? 2 : (kRes ? 3 : 1);
    static constexpr int NVEC = NVEC_BASE + (F8 ? 1 : 0);
    static constexpr int VEC_BYTES = 2 * NVEC * TBN * 4;
    static constexpr int SMEM = 1024 + NST * (A_BYTES + BSTAGE) + NSTG * EPI_WARPS * STG_BYTES + VEC_BYTES + 1024;
    static_assert(SMEM <= 232448, "shared memory per CTA");
};

struct Smem {
    uint8_t *a, *b;
    uint8_t *stg;            // 2 KB output staging tile per epilogue warp
    uint8_t *rstg;           // 2 KB residual (or second output) staging tile per epilogue warp
    uint8_t *stg2;           // residual epilogue: second 2 KB output staging tile per warp
    float *vec;              // [2][NVEC][TBN] per-column vectors of this unit and the next
    uint64_t *vec_full;      // [2]: a unit's vectors are in shared memory
    uint64_t *full, *empty, *tfull, *tempty, *drain, *rbar;
    uint32_t *tmem_slot;
    volatile int *abort_flag;
    int *misc;               // [0] n_rows, [1] status at entry
};

template <int EPI, bool PAIR, bool F8, int TBN>
__device__ __forceinline__ Smem carve(uint8_t *raw) {
    using P = Plan<EPI, PAIR, F8, TBN>;
    constexpr int NST = P::NST;
    Smem s;
    uint8_t *p = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
    s.a = p;
    s.b = p + NST * A_BYTES;
    s.stg = s.b + NST * P::BSTAGE;
    s.rstg = s.stg + EPI_WARPS * STG_BYTES;
    s.stg2 = s.rstg + EPI_WARPS * STG_BYTES;
    s.vec = reinterpret_cast<float *>(s.stg + P::NSTG * EPI_WARPS * STG_BYTES);
    uint8_t *ctrl = reinterpret_cast<uint8_t *>(s.vec) + P::VEC_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(ctrl);
    s.full = bars;
    s.empty = bars + NST;
    s.tfull = bars + 2 * NST;
    s.tempty = bars + 2 * NST + 2;
    s.drain = bars + 2 * NST + 4;
    s.rbar = bars + 2 * NST + 5;
    s.vec_full = bars + 2 * NST + 5 + EPI_WARPS;
    uint32_t *u = reinterpret_cast<uint32_t *>(bars + 2 * NST + 5 + EPI_WARPS + 2);
    s.tmem_slot = u;
    s.abort_flag = reinterpret_cast<volatile int *>(u + 1);
    s.misc = reinterpret_cast<int *>(u + 2);
    return s;
}

// 32 values held as 16 fp32 pairs -> 4 x 16 bytes of bf16.
__device__ __forceinline__ uint32_t pack_pair(uint64_t v) {
    const float2 f = f2_split(v);
    return pack_bf16x2(f.x, f.y);
}

__device__ __forceinline__ void store_bf16x32(bf16 *dst, const uint64_t (&v)[16]) {
    uint4 *d = reinterpret_cast<uint4 *>(dst);
#pragma unroll
    for (int q = 0; q < 4; ++q)
        d[q] = make_uint4(pack_pair(v[4 * q]), pack_pair(v[4 * q + 1]), pack_pair(v[4 * q + 2]), pack_pair(v[4 * q + 3]));
}

// Byte offset of 16-byte chunk q of row r in a 32x32 bf16 tile (64-byte rows)
// stored with the TMA 64-byte swizzle: chunk index XOR ((r >> 1) & 3).  A warp
// writing one chunk per lane (lane = row) hits 32 distinct banks per 8 lanes.
__device__ __forceinline__ uint32_t stg_off(int r, int q) {
    return (uint32_t)(r * 64 + ((q ^ ((r >> 1) & 3)) << 4));
}

__device__ __forceinline__ void st_shared_v4(uint32_t a, uint4 v) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}
__device__ __forceinline__ uint4 ld_shared_v4(uint32_t a) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a) : "memory");
    return v;
}
__device__ __forceinline__ float4 ld_shared_f4(uint32_t a) {
    float4 v;
    asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "r"(a) : "memory");
    return v;
}

// Write this lane's 32 values (its row of the warp's 32x32 tile) as bf16 into
// the staging tile, then one lane stores the tile to global memory by TMA.
// The previous store from the same tile must have finished reading it: with
// two tiles used alternately (double_buffered) that store is the one before
// the most recent.
__device__ __forceinline__ void stage_and_store(uint32_t stg, const uint64_t (&v)[16], const CUtensorMap *tm,
                                                int x, int y, int lane, bool double_buffered) {
    uint4 w[4];
#pragma unroll
    for (int q = 0; q < 4; ++q)
        w[q] = make_uint4(pack_pair(v[4 * q]), pack_pair(v[4 * q + 1]), pack_pair(v[4 * q + 2]), pack_pair(v[4 * q + 3]));
    if (lane == 0) {
        if (double_buffered) bulk_wait_read1();
        else bulk_wait_read0();
    }
    __syncwarp();
#pragma unroll
    for (int q = 0; q < 4; ++q) st_shared_v4(stg + stg_off(lane, q), w[q]);
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
        tma_store_2d(tm, stg, x, y);
        bulk_commit();
    }
}

// Chan's merge: (mean, m2) over cnt values absorbs a group (cm, cq) of cn values.
__device__ __forceinline__ void chan_merge(float &mean, float &m2, float cnt, float cm, float cq, float cn) {
    const float nn = cnt + cn, d = cm - mean;
    mean = fmaf(d, cn / nn, mean);
    m2 += cq + d * d * (cnt * cn / nn);
}

// Mean and 1/sqrt(var + eps) of a 768-wide row from its six 128-column partials.
__device__ __forceinline__ void row_stats_merge(const float2 (&q)[LN_PARTS], float eps, float &mu, float &rstd) {
    float m = 0.f;
#pragma unroll
    for (int i = 0; i < LN_PARTS; ++i) m += q[i].x;
    m *= (1.0f / LN_PARTS);
    float m2 = 0.f;
#pragma unroll
    for (int i = 0; i < LN_PARTS; ++i) {
        const float d = q[i].x - m;
        m2 += q[i].y + (float)(LN_N / LN_PARTS) * d * d;
    }
    mu = m;
    rstd = rsqrtf(m2 * (1.0f / LN_N) + eps);
}

// F8: both operands are E4M3 (tiles of 128 bytes = 128 elements along K, products
// with tcgen05.mma kind::f8f6f4, K = 32 per instruction) with fp32 row scales:
// the epilogue starts from acc * a_scale[row] * w_scale[col].
template <int EPI, bool PAIR, bool F8, int TBN>
__global__ void __launch_bounds__(THREADS, 1)
gemm_bf16_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const __grid_constant__ CUtensorMap tmOut, const __grid_constant__ CUtensorMap tmRes,
                 const GemmArgs p) {
    constexpr bool kLnIn = EPI == kEpiLnIn || EPI == kEpiLnInGelu || EPI == kEpiLnInScatter;
    constexpr bool kGelu = EPI == kEpiGelu || EPI == kEpiLnInGelu;
    constexpr bool kScatter = EPI == kEpiScatter || EPI == kEpiLnInScatter;
    constexpr bool kRes = EPI == kEpiResStats;
    constexpr int NST = Plan<EPI, PAIR, F8, TBN>::NST;
    constexpr int BSTAGE = Plan<EPI, PAIR, F8, TBN>::BSTAGE;
    static_assert(TBN == 256 || (TBN == 128 && !PAIR), "tile widths: 256, or 128 for one CTA");
    constexpr int NH = TBN / 128;      // 128-column halves of a tile
    constexpr int AEW = 4 * NH;        // epilogue warps with columns (one per lane quadrant and half)
    constexpr int KB = F8 ? 128 : BK;  // K elements per stage (a 128-byte swizzle row)
    constexpr int UM = PAIR ? 2 * BM : BM;  // rows of A (and D) per unit
    extern __shared__ uint8_t smem_raw[];
    Smem sm = carve<EPI, PAIR, F8, TBN>(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // A pair works on one unit at a time; rank 0 issues the MMAs for both CTAs.
    const uint32_t rank = PAIR ? cluster_ctarank() : 0;
    const int slot = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
    const int nslots = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;

    if (p.trigger) griddep_launch_dependents();  // the next kernel may take SMs as this grid frees them
    if (threadIdx.x == 0) {
        *sm.abort_flag = 0;
        wait_limit_init(p.wait_ns);
        for (int i = 0; i < NST; ++i) {
            mbar_init(smem_u32(&sm.full[i]), 1);
            mbar_init(smem_u32(&sm.empty[i]), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(&sm.tfull[i]), 1);
            // the pair's accumulator is released by the epilogues of both CTAs
            mbar_init(smem_u32(&sm.tempty[i]), PAIR ? 2 * AEW : AEW);
        }
        mbar_init(smem_u32(sm.drain), 1);
        for (int i = 0; i < EPI_WARPS; ++i) mbar_init(smem_u32(&sm.rbar[i]), 1);
        // every epilogue thread arrives once it has stored its columns
        for (int i = 0; i < 2; ++i) mbar_init(smem_u32(&sm.vec_full[i]), 32 * AEW);
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
        if (!kScatter) prefetch_tmap(&tmOut);
        if (kRes) prefetch_tmap(&tmRes);

    }
    if (warp == 1) {
        if (PAIR) {
            tmem_alloc_pair(smem_u32(sm.tmem_slot), TMEM_COLS);
            tmem_relinquish_pair();
        } else {
            tmem_alloc(smem_u32(sm.tmem_slot), TMEM_COLS);
            tmem_relinquish();
        }
    }
    // The weights do not depend on the previous kernel: before waiting for it,
    // the producer starts the B tiles of the first stages of its first unit
    // (their A tiles follow the wait).  A pair's copies count on rank 0's
    // barriers, so their initialisation must be visible to both CTAs first.
    if (PAIR) cluster_sync();
    else __syncthreads();
    const int pre = p.withhold_loads ? 0 : (p.K / KB < NST ? p.K / KB : NST);  // stages started early
    if (warp == 0 && lane == 0 && pre > 0) {
        const uint64_t keep = policy_evict_last();
        const int n = slot % (p.N / TBN);
        for (int st = 0; st < pre; ++st) {
            const uint32_t fb = smem_u32(&sm.full[st]);
            const uint32_t b_dst = smem_u32(sm.b + st * BSTAGE);
            if (PAIR) {
                if (rank == 0) mbar_expect_tx(fb, 2 * B_HALF_BYTES);
                tma_load_2d_pair_hint(b_dst, &tmB, mapa_shared(fb, 0), st * KB, n * BN + (int)rank * B_BOX, keep);
            } else {
                mbar_expect_tx(fb, BSTAGE);
                tma_load_2d_hint(b_dst, &tmB, fb, st * KB, n * TBN, keep);
                if (TBN == 256) tma_load_2d_hint(b_dst + B_HALF_BYTES, &tmB, fb, st * KB, n * TBN + B_BOX, keep);
            }
        }
    }
    // The prologue above overlaps the previous kernel; its results are used from here on.
    griddep_wait();
    if (threadIdx.x == 0) {
        sm.misc[0] = *reinterpret_cast<const volatile int *>(p.n_rows);
        sm.misc[1] = *reinterpret_cast<const volatile int *>(p.status);
    }
    tc_fence_before();
    // barrier initialisation (and, for a pair, the peer's) is visible before any use
    if (PAIR) cluster_sync();
    else __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *sm.tmem_slot;

    // An earlier kernel of this forward failed, or the row count is out of range:
    // no units (every role still reaches the teardown, which a pair shares).
    const bool skip = sm.misc[1] != 0 || sm.misc[0] < 0 || sm.misc[0] > p.rows_cap;
    const int n_rows = skip ? 0 : sm.misc[0];
    const int m_blocks = (n_rows + UM - 1) / UM;
    const int n_sub = p.N / TBN;
    const int units = m_blocks * n_sub;  // unit u = tile (u / n_sub, u % n_sub), row-block major
    const int kblocks = p.K / KB;

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer --
        if (lane == 0) {
            const uint64_t keep = policy_evict_last();  // weights: reused by every CTA
            int stage = 0, issued = 0;
            uint32_t phase = 0;
            bool ok = true;
            const int units_loaded = p.withhold_loads ? 0 : units;
            for (int u = slot; u < units_loaded && ok; u += nslots) {
                const int m = u / n_sub, n = u % n_sub;
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!mbar_wait(smem_u32(&sm.empty[stage]), phase ^ 1, sm.abort_flag)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_u32(&sm.full[stage]);
                    const uint32_t a_dst = smem_u32(sm.a + stage * A_BYTES);
                    const uint32_t b_dst = smem_u32(sm.b + stage * BSTAGE);
                    if (issued < pre) {
                        // the first unit's B tiles of this stage are already on their way
                        if (PAIR) {
                            if (rank == 0) mbar_arrive_expect_tx(fb, 2 * A_BYTES);
                            tma_load_2d_pair(a_dst, &tmA, mapa_shared(fb, 0), kb * KB, m * UM + (int)rank * BM);
                        } else {
                            mbar_arrive_expect_tx(fb, A_BYTES);
                            tma_load_2d(a_dst, &tmA, fb, kb * KB, m * BM);
                        }
                    } else if (PAIR) {
                        // both CTAs' copies count on rank 0's barrier, which expects them all
                        const uint32_t fb0 = mapa_shared(fb, 0);
                        if (rank == 0) mbar_arrive_expect_tx(fb, 2 * (A_BYTES + B_HALF_BYTES));
                        tma_load_2d_pair(a_dst, &tmA, fb0, kb * KB, m * UM + (int)rank * BM);
                        tma_load_2d_pair_hint(b_dst, &tmB, fb0, kb * KB, n * TBN + (int)rank * B_BOX, keep);
                    } else {
                        mbar_arrive_expect_tx(fb, A_BYTES + BSTAGE);
                        tma_load_2d(a_dst, &tmA, fb, kb * KB, m * BM);
                        tma_load_2d_hint(b_dst, &tmB, fb, kb * KB, n * TBN, keep);
                        if (TBN == 256)
                            tma_load_2d_hint(b_dst + B_HALF_BYTES, &tmB, fb, kb * KB, n * TBN + B_BOX, keep);
                    }
                    ++issued;
                    if (++stage == NST) { stage = 0; phase ^= 1; }
                }
            }
            if (issued < pre && (!PAIR || rank == 0)) {
                // no unit to load (few rows, or an earlier kernel failed): the early
                // weight tiles still land before the CTA's shared memory goes away
                for (int st = issued; st < pre; ++st) mbar_arrive(smem_u32(&sm.full[st]));
                for (int st = issued; st < pre; ++st) mbar_wait_drain(smem_u32(&sm.full[st]), 0);
            }
            if (!ok && (!PAIR || rank == 0)) {
                // Drain: every stage whose load may still be in flight completes
                // its transaction count before the CTA's shared memory goes away.
                // (A pair's rank 1 counts its copies on rank 0's barriers; rank 0
                // drains them before the pair's closing cluster barrier.)
                for (int i = 0; i < NST && i < issued; ++i) {
                    if (--stage < 0) { stage = NST - 1; phase ^= 1; }
                    mbar_wait_drain(smem_u32(&sm.full[stage]), phase);
                }
            }
        }
    } else if (warp == 1) {
        // -------------------------------------------------------- MMA issuer --
        if (lane == 0 && rank == 0) {
            const uint32_t idesc = F8 ? idesc_e4m3_f32(UM, TBN) : idesc_bf16_f32(UM, TBN);
            int stage = 0, acc = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int u = slot; u < units && ok; u += nslots) {
                const int ab = acc & 1;
                const uint32_t aph = (acc >> 1) & 1;
                if (!mbar_wait(smem_u32(&sm.tempty[ab]), aph ^ 1, sm.abort_flag)) break;
                tc_fence_after();
                const uint32_t d = tmem_base + ab * TBN;
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!mbar_wait(smem_u32(&sm.full[stage]), phase, sm.abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(sm.a + stage * A_BYTES);
                    const uint32_t b0 = smem_u32(sm.b + stage * BSTAGE);
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k) {
                        // each product consumes 32 bytes of K: 16 bf16 or 32 E4M3 elements
                        if (PAIR && F8)
                            umma_e4m3_pair(d, sw128_kmajor_desc(a0 + k * 32), sw128_kmajor_desc(b0 + k * 32), idesc,
                                           (kb | k) != 0);
                        else if (F8)
                            umma_e4m3(d, sw128_kmajor_desc(a0 + k * 32), sw128_kmajor_desc(b0 + k * 32), idesc,
                                      (kb | k) != 0);
                        else if (PAIR)
                            umma_bf16_pair(d, sw128_kmajor_desc(a0 + k * 32), sw128_kmajor_desc(b0 + k * 32), idesc,
                                           (kb | k) != 0);
                        else
                            umma_bf16(d, sw128_kmajor_desc(a0 + k * 32), sw128_kmajor_desc(b0 + k * 32), idesc,
                                      (kb | k) != 0);
                    }
                    // the stage is free in both CTAs once these MMAs have read it
                    if (PAIR) umma_commit_pair(smem_u32(&sm.empty[stage]), 3);
                    else umma_commit(smem_u32(&sm.empty[stage]));
                    if (++stage == NST) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                if (PAIR) umma_commit_pair(smem_u32(&sm.tfull[ab]), 3);
                else umma_commit(smem_u32(&sm.tfull[ab]));
                ++acc;
            }
            // All MMAs issued by this thread complete before TMEM is released.
            if (PAIR) umma_commit_pair(smem_u32(sm.drain), 1);
            else umma_commit(smem_u32(sm.drain));
            mbar_wait_drain(smem_u32(sm.drain), 0);
        }
    } else if (warp - 2 < AEW) {
        // ---------------------------------------------------------- epilogue --
        // (a 128-column tile keeps warps 6..9 idle: one warp per lane quadrant)
        const int ew = warp - 2;            // 0..AEW-1
        const int quad = warp & 3;          // TMEM lanes 32*quad .. 32*quad+31
        const int half = ew >> 2;           // 128-column half of the tile
        const int r_local = quad * 32 + lane;
        const int row_off = (int)rank * BM;  // this CTA's rows within a unit
        const uint32_t stg = smem_u32(sm.stg + ew * STG_BYTES);
        const uint32_t rstg = smem_u32(sm.rstg + ew * STG_BYTES);  // residual tile (kRes) or second output tile
        const uint32_t stg2 = smem_u32(sm.stg2 + ew * STG_BYTES);  // kRes only: second output tile
        const uint32_t rbar = smem_u32(&sm.rbar[ew]);
        const bool res_ln = kRes && p.res_stats != nullptr;
        uint32_t rph = 0;
        bool res_pending = false;
        // residual chunk c (0..3) of unit u -> TMA load into this warp's residual tile
        auto res_issue = [&](int u, int c) {
            if (lane == 0) {
                mbar_arrive_expect_tx(rbar, STG_BYTES);
                tma_load_2d(rstg, &tmRes, rbar, (u % n_sub) * TBN + half * 128 + c * 32,
                            (u / n_sub) * UM + row_off + quad * 32);
            }
            res_pending = true;
        };
        int acc = 0;
        bool ok = true;
        if (kRes && slot < units) res_issue(slot, 0);
        // row statistics of the next unit are fetched while the current one runs
        float2 qin[LN_PARTS], qres[LN_PARTS];
        // (rows past rows_cap, reachable in a pair's last unit, read as zeros)
        auto fetch_stats = [&](int u) {
            const int row = (u / n_sub) * UM + row_off + r_local;
            const bool in = row < p.rows_cap;
#pragma unroll
            for (int i = 0; i < LN_PARTS; ++i) {
                if (kLnIn) qin[i] = in ? __ldg(p.in_stats + (size_t)row * LN_PARTS + i) : make_float2(0.f, 0.f);
                if (res_ln) qres[i] = in ? __ldg(p.res_stats + (size_t)row * LN_PARTS + i) : make_float2(0.f, 0.f);
            }
        };
        if ((kLnIn || res_ln) && slot < units) fetch_stats(slot);
        // The per-column vectors of each unit are staged in shared memory: every
        // epilogue thread loads one column of each a unit ahead (registers),
        // stores it at the end of the current unit, and arrives on vec_full.
        // (Read from global memory inside the chunk loop, these uniform loads
        // stalled every chunk on their latency.)
        constexpr int NVEC = Plan<EPI, PAIR, F8, TBN>::NVEC;
        constexpr int NVEC_BASE = Plan<EPI, PAIR, F8, TBN>::NVEC_BASE;
        const int et = ew * 32 + lane;  // 0..TBN-1: the column this thread stages
        float vreg[NVEC];
        auto vec_load = [&](int un) {
            const int col = (un % n_sub) * TBN + et;
            vreg[0] = __ldg(p.bias + col);
            if (kLnIn) vreg[1] = __ldg(p.fold_s + col);
            if (kRes) {
                vreg[1] = __ldg(p.out_g + col);
                vreg[NVEC_BASE - 1] = res_ln ? __ldg(p.res_g + col) : 0.f;
            }
            if (F8) vreg[NVEC - 1] = __ldg(p.w_scale + col);
        };
        auto vec_store = [&](int b) {
#pragma unroll
            for (int i = 0; i < NVEC; ++i) sm.vec[(b * NVEC + i) * TBN + et] = vreg[i];
            mbar_arrive(smem_u32(&sm.vec_full[b]));
        };
        if (slot < units) {
            vec_load(slot);
            vec_store(0);
            if (slot + nslots < units) vec_load(slot + nslots);
        }
        int j = 0;  // unit iteration of this CTA
        for (int u = slot; u < units && ok; u += nslots) {
            const int m = u / n_sub, n = u % n_sub;
            const int row = m * UM + row_off + r_local;
            const bool row_ok = row < n_rows;
            const int tile_row = m * UM + row_off + quad * 32;
            int dst = row;
            if (kScatter) dst = row_ok ? __ldg(p.row_dst + row) : -1;
            // E4M3 operands: the A row's scale (rows past rows_cap, reachable in a
            // pair's last unit, are never stored)
            const float asc = F8 ? (row < p.rows_cap ? __ldg(p.a_scale + row) : 0.f) : 1.f;
            float mu = 0.f, rstd = 1.f;        // LayerNorm of the A operand
            if (kLnIn) row_stats_merge(qin, p.eps, mu, rstd);
            float rmu = 0.f, rrstd = 1.f;      // LayerNorm of the residual
            if (res_ln) row_stats_merge(qres, p.eps, rmu, rrstd);
            if ((kLnIn || res_ln) && u + nslots < units) fetch_stats(u + nslots);
            const float nmu = -rstd * mu, rnmu = -rrstd * rmu;

            const int ab = acc & 1;
            const uint32_t aph = (acc >> 1) & 1;
            const int vb = j & 1;
            bool got = mbar_wait(smem_u32(&sm.vec_full[vb]), (j >> 1) & 1, sm.abort_flag) &&
                       mbar_wait(smem_u32(&sm.tfull[ab]), aph, sm.abort_flag);
            got = __all_sync(0xffffffffu, got);
            if (!got) { ok = false; break; }
            tc_fence_after();
            // shared addresses of this warp's 128 columns of each vector
            const uint32_t vbias = smem_u32(sm.vec + (vb * NVEC) * TBN + half * 128);
            const uint32_t vsec = vbias + TBN * 4;          // W gamma or out_g
            const uint32_t vres = smem_u32(sm.vec + (vb * NVEC + NVEC_BASE - 1) * TBN + half * 128);  // res_g
            const uint32_t vws = smem_u32(sm.vec + (vb * NVEC + NVEC - 1) * TBN + half * 128);  // w_scale (F8)
            const uint32_t tbase = tmem_base + ((uint32_t)(quad * 32) << 16) + ab * TBN + half * 128;
            const int ncol0 = n * TBN + half * 128;  // first output column of this warp
            float mean = 0.f, m2 = 0.f;
            // chunk c + 1 loads from TMEM while chunk c is processed
            uint32_t r[2][32];
            tmem_ld32(tbase, r[0]);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint4 rr[4];
                if (kRes) {
                    bool rok = mbar_wait(rbar, rph, sm.abort_flag);
                    rok = __all_sync(0xffffffffu, rok);
                    if (!rok) { ok = false; tmem_ld_wait(); break; }
                    rph ^= 1;
                    res_pending = false;
#pragma unroll
                    for (int q = 0; q < 4; ++q) rr[q] = ld_shared_v4(rstg + stg_off(lane, q));
                }
                tmem_ld_wait();
                if (c < 3) {
                    tmem_ld32(tbase + (c + 1) * 32, r[(c + 1) & 1]);
                } else {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) {
                        if (PAIR) mbar_arrive_cluster(mapa_shared(smem_u32(&sm.tempty[ab]), 0));
                        else mbar_arrive(smem_u32(&sm.tempty[ab]));
                    }
                }
                const uint32_t *rc = r[c & 1];
                uint32_t rsc[32];
                if (F8) {
                    // acc * a_scale[row] * w_scale[col]: the product of the unscaled E4M3 codes
                    const uint32_t ws4 = vws + c * 128;
                    const uint64_t a2 = f2_make(asc, asc);
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const float4 w = ld_shared_f4(ws4 + q * 16);
                        const float2 x0 = f2_split(f2_mul(f2_mul(f2_make_u(rc[4 * q], rc[4 * q + 1]), f2_make(w.x, w.y)), a2));
                        const float2 x1 =
                            f2_split(f2_mul(f2_mul(f2_make_u(rc[4 * q + 2], rc[4 * q + 3]), f2_make(w.z, w.w)), a2));
                        rsc[4 * q] = __float_as_uint(x0.x);
                        rsc[4 * q + 1] = __float_as_uint(x0.y);
                        rsc[4 * q + 2] = __float_as_uint(x1.x);
                        rsc[4 * q + 3] = __float_as_uint(x1.y);
                    }
                    rc = rsc;
                }
                const int col0 = ncol0 + c * 32;
                uint64_t v[16];  // columns col0 + 2j, col0 + 2j + 1
                const uint32_t bias4 = vbias + c * 128;  // 32 floats per chunk
                if (kLnIn) {
                    const uint32_t s4 = vsec + c * 128;
                    const uint64_t rstd2 = f2_make(rstd, rstd), nmu2 = f2_make(nmu, nmu);
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const float4 bb = ld_shared_f4(bias4 + q * 16), ss = ld_shared_f4(s4 + q * 16);
                        v[2 * q] = f2_fma(rstd2, f2_make_u(rc[4 * q], rc[4 * q + 1]),
                                          f2_fma(nmu2, f2_make(ss.x, ss.y), f2_make(bb.x, bb.y)));
                        v[2 * q + 1] = f2_fma(rstd2, f2_make_u(rc[4 * q + 2], rc[4 * q + 3]),
                                              f2_fma(nmu2, f2_make(ss.z, ss.w), f2_make(bb.z, bb.w)));
                    }
                } else {
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const float4 bb = ld_shared_f4(bias4 + q * 16);
                        v[2 * q] = f2_add(f2_make_u(rc[4 * q], rc[4 * q + 1]), f2_make(bb.x, bb.y));
                        v[2 * q + 1] = f2_add(f2_make_u(rc[4 * q + 2], rc[4 * q + 3]), f2_make(bb.z, bb.w));
                    }
                }
                if (kGelu) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) v[j] = gelu_tanh_f2(v[j]);
                }
                if (kRes) {
                    // residual: plain, or rebuilt LayerNorm output (its beta is folded into bias);
                    // bf16 -> fp32 is the high half of a 32-bit word
                    uint64_t x[16];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint32_t w4[4] = {rr[q].x, rr[q].y, rr[q].z, rr[q].w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) x[4 * q + e] = f2_make_u(w4[e] << 16, w4[e] & 0xffff0000u);
                    }
                    // the residual tile has been read: prefetch the next chunk
                    __syncwarp();
                    if (c < 3) res_issue(u, c + 1);
                    else if (u + nslots < units) res_issue(u + nslots, 0);
                    if (res_ln) {
                        const uint32_t rg4 = vres + c * 128;
                        const uint64_t rrstd2 = f2_make(rrstd, rrstd), rnmu2 = f2_make(rnmu, rnmu);
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const float4 g = ld_shared_f4(rg4 + q * 16);
                            v[2 * q] = f2_fma(rrstd2, x[2 * q], f2_fma(rnmu2, f2_make(g.x, g.y), v[2 * q]));
                            v[2 * q + 1] = f2_fma(rrstd2, x[2 * q + 1], f2_fma(rnmu2, f2_make(g.z, g.w), v[2 * q + 1]));
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 16; ++j) v[j] = f2_add(v[j], x[j]);
                    }
                    // exact chunk statistics of z (four independent chains each),
                    // merged into the running ones
                    uint64_t s4[4] = {v[0], v[1], v[2], v[3]};
#pragma unroll
                    for (int j = 4; j < 16; ++j) s4[j & 3] = f2_add(s4[j & 3], v[j]);
                    const float2 sf = f2_split(f2_add(f2_add(s4[0], s4[1]), f2_add(s4[2], s4[3])));
                    const float cm = (sf.x + sf.y) * (1.0f / 32.0f);
                    const uint64_t ncm2 = f2_make(-cm, -cm);
                    uint64_t q4[4];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const uint64_t d = f2_add(v[j], ncm2);
                        q4[j & 3] = j < 4 ? f2_mul(d, d) : f2_fma(d, d, q4[j & 3]);
                    }
                    const float2 qf = f2_split(f2_add(f2_add(q4[0], q4[1]), f2_add(q4[2], q4[3])));
                    const float cq = qf.x + qf.y;
                    if (c == 0) { mean = cm; m2 = cq; }
                    else chan_merge(mean, m2, 32.f * c, cm, cq, 32.f);
                    // output z * gamma of the LayerNorm that will normalize z
                    const uint32_t og4 = vsec + c * 128;
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const float4 g = ld_shared_f4(og4 + q * 16);
                        v[2 * q] = f2_mul(v[2 * q], f2_make(g.x, g.y));
                        v[2 * q + 1] = f2_mul(v[2 * q + 1], f2_make(g.z, g.w));
                    }
                }
                if (kScatter) {
                    if (dst >= 0) store_bf16x32(p.out + (size_t)dst * p.ld_out + col0, v);
                } else if (kRes) {
                    stage_and_store((c & 1) ? stg2 : stg, v, &tmOut, col0, tile_row, lane, true);
                } else {
                    // the residual tile is free here: alternate the two staging tiles
                    stage_and_store((c & 1) ? rstg : stg, v, &tmOut, col0, tile_row, lane, true);
                }
            }
            if (!ok) break;
            if (kRes && row < p.rows_cap) p.out_stats[(size_t)row * LN_PARTS + n * NH + half] = make_float2(mean, m2);
            ++acc;
            // the next unit's vectors: buffer (j + 1) & 1 was last read in unit j - 1,
            // which every epilogue thread finished before arriving for unit j
            if (u + nslots < units) {
                vec_store((j + 1) & 1);
                if (u + 2 * nslots < units) vec_load(u + 2 * nslots);
            }
            ++j;
        }
        // outstanding copies finish before the CTA's shared memory goes away
        if (lane == 0) bulk_wait0();
        if (res_pending && lane == 0) mbar_wait_drain(rbar, rph);
        __syncwarp();
    }

    // A pair's CTAs leave together: rank 1's shared memory and tensor memory are
    // operands of rank 0's MMAs, and its epilogue arrives on rank 0's barriers.
    tc_fence_before();
    if (PAIR) cluster_sync();
    else __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        if (PAIR) tmem_dealloc_pair(tmem_base, TMEM_COLS);
        else tmem_dealloc(tmem_base, TMEM_COLS);
    }
    if (threadIdx.x == 0 && *sm.abort_flag) set_status(p.status, kStatusTimeout);
}

}  // namespace


// The kernel instance's shared-memory limit, raised once per device.
template <int EPI, bool PAIR, bool F8, int TBN = BN>
static cudaError_t configure(int smem) {
    static std::atomic<unsigned long long> configured{0};
    return ensure_smem_attr(reinterpret_cast<const void *>(gemm_bf16_kernel<EPI, PAIR, F8, TBN>), smem, configured);
}

// Clusters of two GEMM CTAs that fit on the device at once (every epilogue
// instance has the same footprint), per device ordinal.
static int pair_clusters(int num_sms) {
    static std::atomic<int> cached[64];  // zero-initialised (static storage)
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return num_sms / 2;
    const int known = cached[dev].load(std::memory_order_acquire);
    if (known > 0) return known;
    int n = 0;
    if (configure<kEpiBias, true, false>(Plan<kEpiBias, true>::SMEM) == cudaSuccess) {
        cudaLaunchConfig_t cfg = {};
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.gridDim = dim3(2 * (num_sms / 2));
        cfg.blockDim = dim3(THREADS);
        cfg.dynamicSmemBytes = Plan<kEpiBias, true>::SMEM;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaOccupancyMaxActiveClusters(&n, gemm_bf16_kernel<kEpiBias, true, false, BN>, &cfg) != cudaSuccess) n = 0;
    }
    cudaGetLastError();
    if (n <= 0 || n > num_sms / 2) n = num_sms / 2;
    cached[dev].store(n, std::memory_order_release);
    return n;
}

// The kernel a launch takes.  Auto: one CTA per 128x256 tile for a single
// 128-row block; otherwise the CTA pair per 256x256 tile, unless that leaves
// clusters idle while 128x128 tiles on one CTA each would all run at once
// (few rows: the narrower tile halves each unit's main loop and spreads the
// work over more SMs).
int gemm_resolve(int rows_cap, int N, int num_sms, int variant) {
    if (variant != kGemmAuto) return variant;
    if (rows_cap <= BM) return kGemmSingle;
    const int pair_units = ((rows_cap + 2 * BM - 1) / (2 * BM)) * (N / BN);
    const int narrow_units = ((rows_cap + BM - 1) / BM) * (N / 128);
    if (N % 128 == 0 && pair_units < pair_clusters(num_sms) && narrow_units <= num_sms) return kGemmNarrow;
    return kGemmPair;
}

int gemm_grid(int epi, int rows_cap, int N, int num_sms, int variant) {
    (void)epi;
    const int v = gemm_resolve(rows_cap, N, num_sms, variant);
    if (v == kGemmPair) {
        const int units = ((rows_cap + 2 * BM - 1) / (2 * BM)) * (N / BN);
        const int clusters = pair_clusters(num_sms);
        return 2 * (units < clusters ? (units > 0 ? units : 1) : clusters);
    }
    const int units = ((rows_cap + BM - 1) / BM) * (N / (v == kGemmNarrow ? 128 : BN));
    return units < num_sms ? (units > 0 ? units : 1) : num_sms;
}

template <int EPI, bool F8, int TBN>
static cudaError_t launch_single(const CUtensorMap &tmA, const CUtensorMap &tmB, const CUtensorMap &tmOut,
                                 const CUtensorMap &tmRes, const GemmArgs &a, int grid, cudaStream_t s, bool pdl) {
    constexpr int smem = Plan<EPI, false, F8, TBN>::SMEM;
    cudaError_t e = configure<EPI, false, F8, TBN>(smem);
    if (e != cudaSuccess) return e;
    if (!pdl) {
        gemm_bf16_kernel<EPI, false, F8, TBN><<<grid, THREADS, smem, s>>>(tmA, tmB, tmOut, tmRes, a);
        return cudaGetLastError();
    }
    return launch_pdl(gemm_bf16_kernel<EPI, false, F8, TBN>, dim3(grid), dim3(THREADS), smem, s, tmA, tmB, tmOut,
                      tmRes, a);
}

template <int EPI, bool F8>
static cudaError_t launch_one(const CUtensorMap &tmA, const CUtensorMap &tmB, const CUtensorMap &tmOut,
                              const CUtensorMap &tmRes, const GemmArgs &a, int grid, cudaStream_t s, int v,
                              bool pdl) {
    if (v == kGemmSingle) return launch_single<EPI, F8, BN>(tmA, tmB, tmOut, tmRes, a, grid, s, pdl);
    if (v == kGemmNarrow) {
        if (a.N % 128) return cudaErrorInvalidValue;
        return launch_single<EPI, F8, 128>(tmA, tmB, tmOut, tmRes, a, grid, s, pdl);
    }
    if (grid < 2 || grid % 2) return cudaErrorInvalidConfiguration;
    cudaError_t e = configure<EPI, true, F8>(Plan<EPI, true, F8>::SMEM);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;  // see launch_pdl
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = Plan<EPI, true, F8>::SMEM;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, gemm_bf16_kernel<EPI, true, F8, BN>, tmA, tmB, tmOut, tmRes, a);
}

cudaError_t launch_gemm(int epi, const CUtensorMap &tmA, const CUtensorMap &tmB, const CUtensorMap &tmOut,
                        const CUtensorMap &tmRes, const GemmArgs &a, int grid, int num_sms, cudaStream_t s,
                        int variant, bool pdl) {
    const int v = gemm_resolve(a.rows_cap, a.N, num_sms, variant);
    if (a.e4m3) {
        // the E4M3 variant serves the four layer GEMMs and the single-kernel tests
        switch (epi) {
            case kEpiBias: return launch_one<kEpiBias, true>(tmA, tmB, tmOut, tmRes, a, grid, s, v, pdl);
            case kEpiGelu: return launch_one<kEpiGelu, true>(tmA, tmB, tmOut, tmRes, a, grid, s, v, pdl);
            case kEpiResStats: return launch_one<kEpiResStats, true>(tmA, tmB, tmOut, tmRes, a, grid, s, v, pdl);
            case kEpiScatter: return launch_one<kEpiScatter, true>(tmA, tmB, tmOut, tmRes, a, grid, s, v, pdl);
            case kEpiLnIn: return launch_one<kEpiLnIn, true>(tmA, tmB, tmOut, tmRes, a, grid, s, v, pdl);
            case kEpiLnInGelu: return launch_one<kEpiLnInGelu, true>(tmA, tmB, tmOut, tmRes, a, grid, s, v, pdl);
        }
        return cudaErrorInvalidValue;
    }
    switch (epi) {
        case kEpiBias: return launch_one<kEpiBias, false>(tmA, tmB, tmOut, tmRes, a, grid, s, v, pdl);
        case kEpiGelu: return launch_one<kEpiGelu, false>(tmA, tmB, tmOut, tmRes, a, grid, s, v, pdl);
        case kEpiResStats: return launch_one<kEpiResStats, false>(tmA, tmB, tmOut, tmRes, a, grid, s, v, pdl);
        case kEpiScatter: return launch_one<kEpiScatter, false>(tmA, tmB, tmOut, tmRes, a, grid, s, v, pdl);
        case kEpiLnIn: return launch_one<kEpiLnIn, false>(tmA, tmB, tmOut, tmRes, a, grid, s, v, pdl);
        case kEpiLnInGelu: return launch_one<kEpiLnInGelu, false>(tmA, tmB, tmOut, tmRes, a, grid, s, v, pdl);
        case kEpiLnInScatter: return launch_one<kEpiLnInScatter, false>(tmA, tmB, tmOut, tmRes, a, grid, s, v, pdl);
    }
    return cudaErrorInvalidValue;
}

// ------------------------------------------------------------ tensor maps --
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    }
    return fn;
}

static int encode_bf16(CUtensorMap *tm, const void *base, uint64_t rows, uint64_t cols, uint32_t box_cols,
                       uint32_t box_rows, CUtensorMapSwizzle swz) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return -1;
    if ((reinterpret_cast<uintptr_t>(base) & 15) || (cols * 2) % 16) return -2;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t es[2] = {1, 1};
    CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides,
                    box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? 0 : -3;
}

int make_tmap_bf16(CUtensorMap *tm, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    return encode_bf16(tm, base, rows, cols, BK, box_rows, CU_TENSOR_MAP_SWIZZLE_128B);
}

int make_tmap_e4m3(CUtensorMap *tm, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return -1;
    if ((reinterpret_cast<uintptr_t>(base) & 15) || cols % 16) return -2;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols};
    cuuint32_t box[2] = {128, box_rows};
    cuuint32_t es[2] = {1, 1};
    CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? 0 : -3;
}

int make_tmap_bf16_tile32(CUtensorMap *tm, const void *base, uint64_t rows, uint64_t cols) {
    return encode_bf16(tm, base, rows, cols, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B);
}

}  // namespace albert
