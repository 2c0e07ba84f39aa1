// gemm_tcgen05.cu -- persistent BF16 GEMM for sm_100a: Y = epi(A W^T + bias).
//
// The dense contractions of the encoder (the 128->768 input projection, the
// fused Q|K|V projection, the attention output projection, both FFN matrices
// and the 768->512 final projection; "ALBERT: How Kokoro's Phoneme Encoder
// Works", section "Inside One Real ALBERT Layer", steps 2-6) all run here.
// A linear layer is y_j = b_j + sum_i x_i W_{j,i} with W stored [out, in]
// ("Qwen3-TTS and Kokoro", section A), i.e. both operands are K-major.
//
// Design (one CTA per SM, persistent over 128x256 output tiles):
//   warp 0      : TMA producer, 4-stage ring of {A 128x64, B 256x64} bf16 tiles
//                 (128-byte swizzle, no multicast);
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

struct Smem {
    uint8_t *a, *b;
    uint8_t *stg;            // one 2 KB output staging tile per epilogue warp
    uint8_t *rstg;           // one 2 KB residual staging tile per epilogue warp
    uint64_t *full, *empty, *tfull, *tempty, *drain, *rbar;
    uint32_t *tmem_slot;
    volatile int *abort_flag;
    int *misc;               // [0] n_rows, [1] status at entry
};

__device__ __forceinline__ Smem carve(uint8_t *raw) {
    Smem s;
    uint8_t *p = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
    s.a = p;
    s.b = p + STAGES * A_BYTES;
    s.stg = s.b + STAGES * B_BYTES;
    s.rstg = s.stg + EPI_WARPS * STG_BYTES;
    uint8_t *ctrl = s.rstg + EPI_WARPS * STG_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(ctrl);
    s.full = bars;
    s.empty = bars + STAGES;
    s.tfull = bars + 2 * STAGES;
    s.tempty = bars + 2 * STAGES + 2;
    s.drain = bars + 2 * STAGES + 4;
    s.rbar = bars + 2 * STAGES + 5;
    uint32_t *u = reinterpret_cast<uint32_t *>(bars + 2 * STAGES + 5 + EPI_WARPS);
    s.tmem_slot = u;
    s.abort_flag = reinterpret_cast<volatile int *>(u + 1);
    s.misc = reinterpret_cast<int *>(u + 2);
    return s;
}

__device__ __forceinline__ void store_bf16x32(bf16 *dst, const float (&v)[32]) {
    uint4 *d = reinterpret_cast<uint4 *>(dst);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint4 w;
        w.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
        w.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
        w.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
        w.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
        d[q] = w;
    }
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

// Write this lane's 32 values (its row of the warp's 32x32 tile) as bf16 into
// the staging tile, then one lane stores the tile to global memory by TMA.
// The previous store from the same tile must have finished reading it: with
// two tiles used alternately (double_buffered) that store is the one before
// the most recent.
__device__ __forceinline__ void stage_and_store(uint32_t stg, const float (&v)[32], const CUtensorMap *tm,
                                                int x, int y, int lane, bool double_buffered) {
    if (lane == 0) {
        if (double_buffered) bulk_wait_read1();
        else bulk_wait_read0();
    }
    __syncwarp();
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint4 w;
        w.x = pack_bf16x2(v[8 * q + 0], v[8 * q + 1]);
        w.y = pack_bf16x2(v[8 * q + 2], v[8 * q + 3]);
        w.z = pack_bf16x2(v[8 * q + 4], v[8 * q + 5]);
        w.w = pack_bf16x2(v[8 * q + 6], v[8 * q + 7]);
        st_shared_v4(stg + stg_off(lane, q), w);
    }
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

template <int EPI>
__global__ void __launch_bounds__(THREADS, 1)
gemm_bf16_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const __grid_constant__ CUtensorMap tmOut, const __grid_constant__ CUtensorMap tmRes,
                 const GemmArgs p) {
    constexpr bool kLnIn = EPI == kEpiLnIn || EPI == kEpiLnInGelu || EPI == kEpiLnInScatter;
    constexpr bool kGelu = EPI == kEpiGelu || EPI == kEpiLnInGelu;
    constexpr bool kScatter = EPI == kEpiScatter || EPI == kEpiLnInScatter;
    constexpr bool kRes = EPI == kEpiResStats;
    extern __shared__ uint8_t smem_raw[];
    Smem sm = carve(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        sm.misc[0] = *reinterpret_cast<const volatile int *>(p.n_rows);
        sm.misc[1] = *reinterpret_cast<const volatile int *>(p.status);
        *sm.abort_flag = 0;
        for (int i = 0; i < STAGES; ++i) {
            mbar_init(smem_u32(&sm.full[i]), 1);
            mbar_init(smem_u32(&sm.empty[i]), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(&sm.tfull[i]), 1);
            mbar_init(smem_u32(&sm.tempty[i]), EPI_WARPS);
        }
        mbar_init(smem_u32(sm.drain), 1);
        for (int i = 0; i < EPI_WARPS; ++i) mbar_init(smem_u32(&sm.rbar[i]), 1);
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
        if (!kScatter) prefetch_tmap(&tmOut);
        if (kRes) prefetch_tmap(&tmRes);
    }
    __syncthreads();
    // An earlier kernel of this forward failed, or the row count is out of range.
    if (sm.misc[1] != 0 || sm.misc[0] < 0 || sm.misc[0] > p.rows_cap) return;

    if (warp == 1) {
        tmem_alloc(smem_u32(sm.tmem_slot), TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *sm.tmem_slot;

    const int n_rows = sm.misc[0];
    const int m_blocks = (n_rows + BM - 1) / BM;
    const int n_sub = p.N / BN;
    const int units = m_blocks * n_sub;  // unit u = tile (u / n_sub, u % n_sub), row-block major
    const int kblocks = p.K / BK;

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer --
        if (lane == 0) {
            const uint64_t keep = policy_evict_last();  // weights: reused by every CTA
            int stage = 0, issued = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
                const int m = u / n_sub, n = u % n_sub;
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!mbar_wait(smem_u32(&sm.empty[stage]), phase ^ 1, sm.abort_flag)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_u32(&sm.full[stage]);
                    mbar_arrive_expect_tx(fb, A_BYTES + B_BYTES);
                    tma_load_2d(smem_u32(sm.a + stage * A_BYTES), &tmA, fb, kb * BK, m * BM);
                    tma_load_2d_hint(smem_u32(sm.b + stage * B_BYTES), &tmB, fb, kb * BK, n * BN, keep);
                    ++issued;
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
            }
            if (!ok) {
                // Drain: every stage whose load may still be in flight completes
                // its transaction count before the CTA's shared memory goes away.
                for (int i = 0; i < STAGES && i < issued; ++i) {
                    if (--stage < 0) { stage = STAGES - 1; phase ^= 1; }
                    mbar_wait_drain(smem_u32(&sm.full[stage]), phase);
                }
            }
        }
    } else if (warp == 1) {
        // -------------------------------------------------------- MMA issuer --
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16_f32(BM, BN);
            int stage = 0, acc = 0;
            uint32_t phase = 0;
            bool ok = true;
            for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
                const int ab = acc & 1;
                const uint32_t aph = (acc >> 1) & 1;
                if (!mbar_wait(smem_u32(&sm.tempty[ab]), aph ^ 1, sm.abort_flag)) break;
                tc_fence_after();
                const uint32_t d = tmem_base + ab * BN;
                for (int kb = 0; kb < kblocks; ++kb) {
                    if (!mbar_wait(smem_u32(&sm.full[stage]), phase, sm.abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(sm.a + stage * A_BYTES);
                    const uint32_t b0 = smem_u32(sm.b + stage * B_BYTES);
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)
                        umma_bf16(d, sw128_kmajor_desc(a0 + k * 32), sw128_kmajor_desc(b0 + k * 32), idesc,
                                  (kb | k) != 0);
                    umma_commit(smem_u32(&sm.empty[stage]));
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                umma_commit(smem_u32(&sm.tfull[ab]));
                ++acc;
            }
            // All MMAs issued by this thread complete before TMEM is released.
            umma_commit(smem_u32(sm.drain));
            mbar_wait_drain(smem_u32(sm.drain), 0);
        }
    } else {
        // ---------------------------------------------------------- epilogue --
        const int ew = warp - 2;            // 0..7
        const int quad = warp & 3;          // TMEM lanes 32*quad .. 32*quad+31
        const int half = ew >> 2;           // column half of the 256-wide tile
        const int r_local = quad * 32 + lane;
        const uint32_t stg = smem_u32(sm.stg + ew * STG_BYTES);
        const uint32_t rstg = smem_u32(sm.rstg + ew * STG_BYTES);
        const uint32_t rbar = smem_u32(&sm.rbar[ew]);
        const bool res_ln = kRes && p.res_stats != nullptr;
        uint32_t rph = 0;
        bool res_pending = false;
        // residual chunk c (0..3) of unit u -> TMA load into this warp's residual tile
        auto res_issue = [&](int u, int c) {
            if (lane == 0) {
                mbar_arrive_expect_tx(rbar, STG_BYTES);
                tma_load_2d(rstg, &tmRes, rbar, (u % n_sub) * BN + half * 128 + c * 32,
                            (u / n_sub) * BM + quad * 32);
            }
            res_pending = true;
        };
        int acc = 0;
        bool ok = true;
        if (kRes && (int)blockIdx.x < units) res_issue(blockIdx.x, 0);
        // row statistics of the next unit are fetched while the current one runs
        float2 qin[LN_PARTS], qres[LN_PARTS];
        auto fetch_stats = [&](int u) {
            const size_t row = (size_t)(u / n_sub) * BM + r_local;
#pragma unroll
            for (int i = 0; i < LN_PARTS; ++i) {
                if (kLnIn) qin[i] = __ldg(p.in_stats + row * LN_PARTS + i);
                if (res_ln) qres[i] = __ldg(p.res_stats + row * LN_PARTS + i);
            }
        };
        if ((kLnIn || res_ln) && (int)blockIdx.x < units) fetch_stats(blockIdx.x);
        for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
            const int m = u / n_sub, n = u % n_sub;
            const int row = m * BM + r_local;  // < rows_cap
            const bool row_ok = row < n_rows;
            const int tile_row = m * BM + quad * 32;
            int dst = row;
            if (kScatter) dst = row_ok ? __ldg(p.row_dst + row) : -1;
            float mu = 0.f, rstd = 1.f;        // LayerNorm of the A operand
            if (kLnIn) row_stats_merge(qin, p.eps, mu, rstd);
            float rmu = 0.f, rrstd = 1.f;      // LayerNorm of the residual
            if (res_ln) row_stats_merge(qres, p.eps, rmu, rrstd);
            if ((kLnIn || res_ln) && u + (int)gridDim.x < units) fetch_stats(u + gridDim.x);
            const float nmu = -rstd * mu, rnmu = -rrstd * rmu;

            const int ab = acc & 1;
            const uint32_t aph = (acc >> 1) & 1;
            bool got = mbar_wait(smem_u32(&sm.tfull[ab]), aph, sm.abort_flag);
            got = __all_sync(0xffffffffu, got);
            if (!got) { ok = false; break; }
            tc_fence_after();
            const uint32_t tbase = tmem_base + ((uint32_t)(quad * 32) << 16) + ab * BN + half * 128;
            const int ncol0 = n * BN + half * 128;  // first output column of this warp
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
                    if (lane == 0) mbar_arrive(smem_u32(&sm.tempty[ab]));
                }
                const uint32_t *rc = r[c & 1];
                const int col0 = ncol0 + c * 32;
                float v[32];
                const float4 *bias4 = reinterpret_cast<const float4 *>(p.bias + col0);
                if (kLnIn) {
                    const float4 *s4 = reinterpret_cast<const float4 *>(p.fold_s + col0);
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const float4 bb = __ldg(bias4 + q), ss = __ldg(s4 + q);
                        v[4 * q + 0] = fmaf(rstd, __uint_as_float(rc[4 * q + 0]), fmaf(nmu, ss.x, bb.x));
                        v[4 * q + 1] = fmaf(rstd, __uint_as_float(rc[4 * q + 1]), fmaf(nmu, ss.y, bb.y));
                        v[4 * q + 2] = fmaf(rstd, __uint_as_float(rc[4 * q + 2]), fmaf(nmu, ss.z, bb.z));
                        v[4 * q + 3] = fmaf(rstd, __uint_as_float(rc[4 * q + 3]), fmaf(nmu, ss.w, bb.w));
                    }
                } else {
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const float4 bb = __ldg(bias4 + q);
                        v[4 * q + 0] = __uint_as_float(rc[4 * q + 0]) + bb.x;
                        v[4 * q + 1] = __uint_as_float(rc[4 * q + 1]) + bb.y;
                        v[4 * q + 2] = __uint_as_float(rc[4 * q + 2]) + bb.z;
                        v[4 * q + 3] = __uint_as_float(rc[4 * q + 3]) + bb.w;
                    }
                }
                if (kGelu) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) v[j] = gelu_tanh_fast(v[j]);
                }
                if (kRes) {
                    // residual: plain, or rebuilt LayerNorm output (its beta is folded into bias)
                    float x[32];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        float2 f;
                        f = unpack_bf16x2(rr[q].x); x[8 * q + 0] = f.x; x[8 * q + 1] = f.y;
                        f = unpack_bf16x2(rr[q].y); x[8 * q + 2] = f.x; x[8 * q + 3] = f.y;
                        f = unpack_bf16x2(rr[q].z); x[8 * q + 4] = f.x; x[8 * q + 5] = f.y;
                        f = unpack_bf16x2(rr[q].w); x[8 * q + 6] = f.x; x[8 * q + 7] = f.y;
                    }
                    // the residual tile has been read: prefetch the next chunk
                    __syncwarp();
                    if (c < 3) res_issue(u, c + 1);
                    else if (u + (int)gridDim.x < units) res_issue(u + gridDim.x, 0);
                    if (res_ln) {
                        const float4 *rg4 = reinterpret_cast<const float4 *>(p.res_g + col0);
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const float4 g = __ldg(rg4 + q);
                            v[4 * q + 0] += fmaf(rrstd, x[4 * q + 0], rnmu * g.x);
                            v[4 * q + 1] += fmaf(rrstd, x[4 * q + 1], rnmu * g.y);
                            v[4 * q + 2] += fmaf(rrstd, x[4 * q + 2], rnmu * g.z);
                            v[4 * q + 3] += fmaf(rrstd, x[4 * q + 3], rnmu * g.w);
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 32; ++j) v[j] += x[j];
                    }
                    // exact chunk statistics of z, merged into the running ones
                    float cs = 0.f;
#pragma unroll
                    for (int j = 0; j < 32; ++j) cs += v[j];
                    const float cm = cs * (1.0f / 32.0f);
                    float cq = 0.f;
#pragma unroll
                    for (int j = 0; j < 32; ++j) { const float d = v[j] - cm; cq = fmaf(d, d, cq); }
                    if (c == 0) { mean = cm; m2 = cq; }
                    else chan_merge(mean, m2, 32.f * c, cm, cq, 32.f);
                    // output z * gamma of the LayerNorm that will normalize z
                    const float4 *og4 = reinterpret_cast<const float4 *>(p.out_g + col0);
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const float4 g = __ldg(og4 + q);
                        v[4 * q + 0] *= g.x; v[4 * q + 1] *= g.y; v[4 * q + 2] *= g.z; v[4 * q + 3] *= g.w;
                    }
                }
                if (kScatter) {
                    if (dst >= 0) store_bf16x32(p.out + (size_t)dst * p.ld_out + col0, v);
                } else if (kRes) {
                    stage_and_store(stg, v, &tmOut, col0, tile_row, lane, false);
                } else {
                    // the residual tile is free here: alternate the two staging tiles
                    stage_and_store((c & 1) ? rstg : stg, v, &tmOut, col0, tile_row, lane, true);
                }
            }
            if (!ok) break;
            if (kRes) p.out_stats[(size_t)row * LN_PARTS + n * 2 + half] = make_float2(mean, m2);
            ++acc;
        }
        // outstanding copies finish before the CTA's shared memory goes away
        if (lane == 0) bulk_wait0();
        if (res_pending && lane == 0) mbar_wait_drain(rbar, rph);
        __syncwarp();
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
    if (threadIdx.x == 0 && *sm.abort_flag) set_status(p.status, kStatusTimeout);
}

}  // namespace

int gemm_grid(int epi, int rows_cap, int N, int num_sms) {
    (void)epi;
    const int units = ((rows_cap + BM - 1) / BM) * (N / BN);
    return units < num_sms ? (units > 0 ? units : 1) : num_sms;
}

template <int EPI>
static cudaError_t launch_one(const CUtensorMap &tmA, const CUtensorMap &tmB, const CUtensorMap &tmOut,
                              const CUtensorMap &tmRes, const GemmArgs &a, int grid, cudaStream_t s) {
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(gemm_bf16_kernel<EPI>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    gemm_bf16_kernel<EPI><<<grid, THREADS, SMEM_BYTES, s>>>(tmA, tmB, tmOut, tmRes, a);
    return cudaGetLastError();
}

cudaError_t launch_gemm(int epi, const CUtensorMap &tmA, const CUtensorMap &tmB, const CUtensorMap &tmOut,
                        const CUtensorMap &tmRes, const GemmArgs &a, int grid, cudaStream_t s) {
    switch (epi) {
        case kEpiBias: return launch_one<kEpiBias>(tmA, tmB, tmOut, tmRes, a, grid, s);
        case kEpiGelu: return launch_one<kEpiGelu>(tmA, tmB, tmOut, tmRes, a, grid, s);
        case kEpiResStats: return launch_one<kEpiResStats>(tmA, tmB, tmOut, tmRes, a, grid, s);
        case kEpiScatter: return launch_one<kEpiScatter>(tmA, tmB, tmOut, tmRes, a, grid, s);
        case kEpiLnIn: return launch_one<kEpiLnIn>(tmA, tmB, tmOut, tmRes, a, grid, s);
        case kEpiLnInGelu: return launch_one<kEpiLnInGelu>(tmA, tmB, tmOut, tmRes, a, grid, s);
        case kEpiLnInScatter: return launch_one<kEpiLnInScatter>(tmA, tmB, tmOut, tmRes, a, grid, s);
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

int make_tmap_bf16_tile32(CUtensorMap *tm, const void *base, uint64_t rows, uint64_t cols) {
    return encode_bf16(tm, base, rows, cols, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B);
}

}  // namespace albert
