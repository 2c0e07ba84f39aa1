// attention_tc_long.cu -- masked bidirectional attention on the 5th-generation
// tensor cores (tcgen05) for batches whose longest sequence has 129..512 tokens.
//
// Per sequence b and head h ("ALBERT: How Kokoro's Phoneme Encoder Works",
// section "Inside One Real ALBERT Layer", step 4; "How Kokoro TTS Works and
// Where CKE Stands", section "What ALBERT does here"):
//     C_h = softmax(Q_h K_h^T / sqrt(64) + mask) V_h,
// key u of sequence b takes part iff u < L_b, every query sees both sides.
//
// One work item = (sequence b, query block qb of 128 rows, head h).  All of the
// item's scores (128 rows x L_b <= 512 keys, fp32) fit in the SM's tensor
// memory at once -- 512 columns, key block j in columns 128j..128j+127 -- so
// the softmax is the exact two-pass one of the definition (row maximum, then
// exponentials and their sum), with no running rescale of the output:
//   warp 0      : TMA producer: the item's Q tile and its ceil(L_b/128) key
//                 tiles into one stage, its value tiles into one of two stages
//                 (128 rows x 64, 128-byte swizzle, from the packed
//                 [rows, 3*768] buffer);
//   warp 1      : tcgen05.mma issuer: S_j = Q K_j^T per key block (M=128,
//                 N=128, K=64; one commit per block so the softmax starts on
//                 block 0 early), then O = sum_j P_j V_j (M=128, N=64) with P_j
//                 read from tensor memory as soon as block j's softmax is done;
//   warps 2..9  : softmax, two halves of four warps (one per TMEM lane
//                 quadrant); half w owns key blocks w and w+2; each thread owns
//                 one query row.  The halves exchange their row maxima through
//                 shared memory (one mbarrier per lane quadrant), then each
//                 writes P_j as packed bf16 over the first 64 columns of its
//                 block (scores already read) and its partial row sum to
//                 shared memory;
//   warps 10..13: output: O sits in columns 64..127 (the second half of block
//                 0, free once P_0 is written); it is scaled by 1 / (sum of the
//                 two halves' sums) and stored.
// Tensor memory is the item's, so the next item's S waits until the output
// warps have read O; its Q, K and V loads run ahead.  A warp whose 32 query rows
// all lie past the sequence's end reads and writes nothing but still takes part
// in every barrier.  Every wait is bounded (%globaltimer).
#include "kernels.h"
#include "sm100_ptx.cuh"

namespace albert {
namespace {

constexpr int LQ = 128;                        // query rows per item; keys per block
constexpr int LKB = 4;                         // key blocks: L <= 512
constexpr int LTILE = LQ * 128;                // 128 rows x 64 bf16 = 16 KB
constexpr int NVS = 2;                         // value stages (LKB tiles each)
constexpr int LA_THREADS = 32 * 14;
constexpr uint32_t LTM_O = 64;                 // O: columns 64..127
constexpr int LA_SMEM = 1024 + (1 + LKB) * LTILE + NVS * LKB * LTILE + 4 * LQ * 4 + 256;
static_assert(LA_SMEM <= 232448, "shared memory per CTA");

struct LongSmem {
    uint8_t *q, *k, *v;                        // Q tile; [LKB] K tiles; [NVS][LKB] V tiles
    float *xmax, *xsum;                        // [2][LQ]: each half's row maxima / row sums
    uint64_t *qk_full, *qk_empty;              // one stage
    uint64_t *v_full, *v_empty;                // [NVS]
    uint64_t *s_full, *p_full;                 // [LKB]
    uint64_t *o_full, *o_empty;
    uint64_t *x_bar;                           // [4]: row-maximum exchange, per lane quadrant
    uint64_t *drain;
    uint32_t *tmem_slot;
    volatile int *abort_flag;
    int *misc;
};

__device__ __forceinline__ LongSmem long_carve(uint8_t *raw) {
    LongSmem s;
    uint8_t *p = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
    s.q = p;
    s.k = p + LTILE;
    s.v = p + (1 + LKB) * LTILE;
    s.xmax = reinterpret_cast<float *>(p + (1 + LKB + NVS * LKB) * LTILE);
    s.xsum = s.xmax + 2 * LQ;
    uint64_t *b = reinterpret_cast<uint64_t *>(s.xsum + 2 * LQ);
    s.qk_full = b;
    s.qk_empty = b + 1;
    s.v_full = b + 2;
    s.v_empty = b + 2 + NVS;
    s.s_full = b + 2 + 2 * NVS;
    s.p_full = s.s_full + LKB;
    s.o_full = s.s_full + 2 * LKB;
    s.o_empty = s.o_full + 1;
    s.x_bar = s.o_full + 2;
    s.drain = s.x_bar + 4;
    uint32_t *u = reinterpret_cast<uint32_t *>(s.drain + 1);
    s.tmem_slot = u;
    s.abort_flag = reinterpret_cast<volatile int *>(u + 1);
    s.misc = reinterpret_cast<int *>(u + 2);
    return s;
}

struct LongItem {
    int h, qb, L, start;
};

// The CTA's items: slots id = blockIdx.x + k * gridDim.x of nseq * LKB * 12,
// slot = (b, qb, h); query blocks past the sequence's end are skipped.  Every
// role walks the same list.
__device__ __forceinline__ bool next_long_item(int &id, int total, const int *__restrict__ seq_start,
                                               const int *__restrict__ seq_len, LongItem &it) {
    for (; id < total; id += gridDim.x) {
        const int b = id / (LKB * kHeads), rem = id - b * (LKB * kHeads);
        const int qb = rem / kHeads;
        // lengths are validated against max_len <= 512 before this kernel runs; the
        // clamp only keeps every tile and TMEM column in bounds regardless
        const int L = min(__ldg(seq_len + b), LKB * LQ);
        if (qb * LQ < L) {
            it.h = rem - qb * kHeads;
            it.qb = qb;
            it.L = L;
            it.start = __ldg(seq_start + b);
            id += gridDim.x;
            return true;
        }
    }
    return false;
}

__device__ __forceinline__ int key_blocks(int L) { return (L + LQ - 1) / LQ; }

__global__ void __launch_bounds__(LA_THREADS, 1)
attn_tc_long_kernel(const __grid_constant__ CUtensorMap tmQKV, bf16 *__restrict__ ctx,
                    const int *__restrict__ seq_start, const int *__restrict__ seq_len, int nseq, int *status,
                    int trigger, unsigned long long wait_ns) {
    if (trigger) griddep_launch_dependents();  // the next kernel may take SMs as this grid frees them
    griddep_wait();               // the previous kernel has completed

    extern __shared__ uint8_t smem_raw[];
    LongSmem sm = long_carve(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        sm.misc[0] = *reinterpret_cast<const volatile int *>(status);
        *sm.abort_flag = 0;
        wait_limit_init(wait_ns);
        mbar_init(smem_u32(sm.qk_full), 1);
        mbar_init(smem_u32(sm.qk_empty), 1);
        for (int i = 0; i < NVS; ++i) {
            mbar_init(smem_u32(&sm.v_full[i]), 1);
            mbar_init(smem_u32(&sm.v_empty[i]), 1);
        }
        for (int j = 0; j < LKB; ++j) {
            mbar_init(smem_u32(&sm.s_full[j]), 1);
            mbar_init(smem_u32(&sm.p_full[j]), 4);  // the four warps of the owning half
        }
        mbar_init(smem_u32(sm.o_full), 1);
        mbar_init(smem_u32(sm.o_empty), 4);
        for (int q = 0; q < 4; ++q) mbar_init(smem_u32(&sm.x_bar[q]), 2);  // one warp of each half
        mbar_init(smem_u32(sm.drain), 1);
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) prefetch_tmap(&tmQKV);
    __syncthreads();
    if (sm.misc[0] != 0) return;  // an earlier kernel of this forward failed
    if (warp == 1) {
        tmem_alloc(smem_u32(sm.tmem_slot), LKB * LQ);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *sm.tmem_slot;
    const int total = nseq * LKB * kHeads;

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer --
        if (lane == 0) {
            int nq = 0, nv = 0;  // stages filled so far
            int id = blockIdx.x;
            LongItem it;
            while (next_long_item(id, total, seq_start, seq_len, it)) {
                const int nkb = key_blocks(it.L);
                // Q and K: free once the previous item's S products have read them
                if (!mbar_wait(smem_u32(sm.qk_empty), (nq & 1) ^ 1, sm.abort_flag)) break;
                const uint32_t fq = smem_u32(sm.qk_full);
                mbar_arrive_expect_tx(fq, (1 + nkb) * LTILE);
                tma_load_2d(smem_u32(sm.q), &tmQKV, fq, it.h * kHeadDim, it.start + it.qb * LQ);
                for (int j = 0; j < nkb; ++j)
                    tma_load_2d(smem_u32(sm.k + j * LTILE), &tmQKV, fq, kHidden + it.h * kHeadDim, it.start + j * LQ);
                ++nq;
                // V: free once the O product of the item two back has completed
                const int vs = nv % NVS;
                if (!mbar_wait(smem_u32(&sm.v_empty[vs]), ((nv / NVS) & 1) ^ 1, sm.abort_flag)) break;
                const uint32_t fv = smem_u32(&sm.v_full[vs]);
                mbar_arrive_expect_tx(fv, nkb * LTILE);
                for (int j = 0; j < nkb; ++j)
                    tma_load_2d(smem_u32(sm.v + (vs * LKB + j) * LTILE), &tmQKV, fv, 2 * kHidden + it.h * kHeadDim,
                                it.start + j * LQ);
                ++nv;
            }
            if (*sm.abort_flag) {
                // loads still in flight complete before the CTA's shared memory goes away
                if (nq > 0) mbar_wait_drain(smem_u32(sm.qk_full), (nq - 1) & 1);
                for (int j = nv > NVS ? nv - NVS : 0; j < nv; ++j)
                    mbar_wait_drain(smem_u32(&sm.v_full[j % NVS]), (j / NVS) & 1);
            }
        }
    } else if (warp == 1) {
        // -------------------------------------------------------- MMA issuer --
        if (lane == 0) {
            const uint32_t idesc_s = idesc_bf16_f32(LQ, LQ);
            const uint32_t idesc_o = idesc_bf16_f32(LQ, kHeadDim) | (1u << 16);  // B (= V) MN-major
            uint32_t par = 0;  // bit j: phase parity of s_full[j] / p_full[j] for the next item using block j
            int id = blockIdx.x, i = 0;
            LongItem it;
            while (next_long_item(id, total, seq_start, seq_len, it)) {
                const int nkb = key_blocks(it.L);
                // tensor memory is free once the output warps have read the previous item's O
                if (!mbar_wait(smem_u32(sm.qk_full), i & 1, sm.abort_flag)) break;
                if (!mbar_wait(smem_u32(sm.o_empty), (i & 1) ^ 1, sm.abort_flag)) break;
                tc_fence_after();
                const uint32_t q = smem_u32(sm.q);
                for (int j = 0; j < nkb; ++j) {
                    const uint32_t k = smem_u32(sm.k + j * LTILE);
#pragma unroll
                    for (int kk = 0; kk < kHeadDim / 16; ++kk)
                        umma_bf16(tmem_base + j * LQ, sw128_kmajor_desc(q + kk * 32), sw128_kmajor_desc(k + kk * 32),
                                  idesc_s, kk != 0);
                    umma_commit(smem_u32(&sm.s_full[j]));
                }
                umma_commit(smem_u32(sm.qk_empty));  // Q, K consumed: stage free
                const int vs = i % NVS;
                if (!mbar_wait(smem_u32(&sm.v_full[vs]), (i / NVS) & 1, sm.abort_flag)) break;
                bool ok = true;
                for (int j = 0; j < nkb && ok; ++j) {
                    ok = mbar_wait(smem_u32(&sm.p_full[j]), (par >> j) & 1, sm.abort_flag);
                    if (!ok) break;
                    tc_fence_after();
                    const int Lj = min(LQ, it.L - j * LQ);
                    const int ksteps = (Lj + 15) >> 4;
                    const uint32_t vb = smem_u32(sm.v + (vs * LKB + j) * LTILE);
                    const uint32_t pcol = tmem_base + j * LQ;
                    for (int kk = 0; kk < ksteps; ++kk) {
                        // P: 16 keys = 8 packed TMEM columns; V: 16 keys = 16 rows of 128 B
                        umma_bf16_ts(tmem_base + LTM_O, pcol + kk * 8, sw128_kmajor_desc(vb + kk * 2048), idesc_o,
                                     (j | kk) != 0);
                    }
                }
                if (!ok) break;
                umma_commit(smem_u32(sm.o_full));
                umma_commit(smem_u32(&sm.v_empty[vs]));  // V consumed: stage free
                par ^= (1u << nkb) - 1;
                ++i;
            }
            umma_commit(smem_u32(sm.drain));
            mbar_wait_drain(smem_u32(sm.drain), 0);
        }
    } else if (warp < 10) {
        // ------------------------------------------------------ softmax warps --
        const int half = (warp - 2) >> 2;  // key blocks half, half + 2
        const int quad = warp & 3;
        const int r = quad * 32 + lane;    // query row within the item
        const float sl2 = 0.125f * 1.4426950408889634f;
        const uint32_t trow = tmem_base + ((uint32_t)(quad * 32) << 16);
        uint32_t par = 0, xpar = 0;
        int id = blockIdx.x;
        LongItem it;
        bool ok = true;
        while (ok && next_long_item(id, total, seq_start, seq_len, it)) {
            const int L = it.L, nkb = key_blocks(L);
            const bool live = it.qb * LQ + quad * 32 < L;  // some row of this warp is a real query
            // pass 1: row maximum over the valid keys of this half's blocks
            // (four independent chains: a single chain is latency-bound)
            float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
            uint32_t v[2][32];
            for (int j = half; j < nkb; j += 2) {
                bool got = mbar_wait(smem_u32(&sm.s_full[j]), (par >> j) & 1, sm.abort_flag);
                got = __all_sync(0xffffffffu, got);
                if (!got) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (!live) continue;
                const int Lj = min(LQ, L - j * LQ), nch = (Lj + 31) >> 5;
                const uint32_t sb = trow + j * LQ;
#pragma unroll 1
                for (int c = 0; c < nch; c += 2) {
                    tmem_ld32(sb + c * 32, v[0]);
                    if (c + 1 < nch) tmem_ld32(sb + (c + 1) * 32, v[1]);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int base = (c + e) * 32;
                        if (c + e >= nch) continue;
                        if (base + 32 <= Lj) {
#pragma unroll
                            for (int t = 0; t < 32; t += 2)
                                mx[(t >> 1) & 3] = fmax3(mx[(t >> 1) & 3], __uint_as_float(v[e][t]),
                                                           __uint_as_float(v[e][t + 1]));
                        } else {
#pragma unroll
                            for (int t = 0; t < 32; ++t)
                                if (base + t < Lj) mx[t & 3] = fmaxf(mx[t & 3], __uint_as_float(v[e][t]));
                        }
                    }
                }
            }
            if (!ok) break;
            float m = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
            if (live && nkb >= 2) {
                // both halves own a block: exchange the partial maxima of each row
                sm.xmax[half * LQ + r] = m;
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&sm.x_bar[quad]));
                bool got = mbar_wait(smem_u32(&sm.x_bar[quad]), xpar, sm.abort_flag);
                got = __all_sync(0xffffffffu, got);
                if (!got) break;
                xpar ^= 1;
                m = fmaxf(m, sm.xmax[(half ^ 1) * LQ + r]);
            }
            // pass 2: P = exp(scale * (s - max)) packed as bf16 pairs; chunk c of block j
            // goes to columns 128j + 16c .. +15, which hold scores already read
            const uint64_t sl2x2 = f2_make(sl2, sl2), nms2 = f2_make(-m * sl2, -m * sl2);
            uint64_t lsum[2] = {f2_make(0.f, 0.f), f2_make(0.f, 0.f)};
            for (int j = half; j < nkb; j += 2) {
                if (live) {
                    const int Lj = min(LQ, L - j * LQ), nch = (Lj + 31) >> 5;
                    const uint32_t sb = trow + j * LQ;
#pragma unroll 1
                    for (int c = 0; c < nch; c += 2) {
                        tmem_ld32(sb + c * 32, v[0]);
                        if (c + 1 < nch) tmem_ld32(sb + (c + 1) * 32, v[1]);
                        tmem_ld_wait();
#pragma unroll
                        for (int e = 0; e < 2; ++e) {
                            const int cc = c + e;
                            if (cc >= nch) continue;
                            const bool full = cc * 32 + 32 <= Lj;
                            uint32_t pk[16];
#pragma unroll
                            for (int t = 0; t < 16; ++t) {
                                const int k0 = cc * 32 + 2 * t;
                                const float2 x =
                                    f2_split(f2_fma(f2_make_u(v[e][2 * t], v[e][2 * t + 1]), sl2x2, nms2));
                                float p0 = ex2_approx(x.x), p1 = ex2_approx(x.y);
                                if (!full) {
                                    p0 = k0 < Lj ? p0 : 0.f;
                                    p1 = k0 + 1 < Lj ? p1 : 0.f;
                                }
                                lsum[t & 1] = f2_add(lsum[t & 1], f2_make(p0, p1));
                                pk[t] = pack_bf16x2(p0, p1);
                            }
                            tmem_st16(sb + cc * 16, pk);
                        }
                    }
                    if (j + 2 >= nkb) {
                        // the half's last block: its row sum, read by the output warps
                        // after they have waited on p_full
                        const float2 ls = f2_split(f2_add(lsum[0], lsum[1]));
                        sm.xsum[half * LQ + r] = ls.x + ls.y;
                    }
                    tmem_st_wait();
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&sm.p_full[j]));
            }
            par ^= (1u << nkb) - 1;
        }
    } else {
        // ------------------------------------------------------- output warps --
        const int quad = warp & 3;
        const int r = quad * 32 + lane;  // query row within the item
        const uint32_t trow = tmem_base + ((uint32_t)(quad * 32) << 16);
        uint32_t par = 0;
        int id = blockIdx.x, i = 0;
        LongItem it;
        while (next_long_item(id, total, seq_start, seq_len, it)) {
            const int L = it.L, nkb = key_blocks(L);
            const bool live = it.qb * LQ + quad * 32 < L;
            // the p_full phases (complete before O is) make both halves' sums visible here
            bool got = mbar_wait(smem_u32(sm.o_full), i & 1, sm.abort_flag);
            for (int j = 0; j < nkb && got; ++j) got = mbar_wait(smem_u32(&sm.p_full[j]), (par >> j) & 1, sm.abort_flag);
            got = __all_sync(0xffffffffu, got);
            if (!got) break;
            par ^= (1u << nkb) - 1;
            tc_fence_after();
            uint32_t o[2][32];
            float inv = 0.f;
            if (live) {
                tmem_ld32(trow + LTM_O, o[0]);
                tmem_ld32(trow + LTM_O + 32, o[1]);
                inv = 1.f / (sm.xsum[r] + (nkb >= 2 ? sm.xsum[LQ + r] : 0.f));
                tmem_ld_wait();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(sm.o_empty));
            const int qi = it.qb * LQ + r;
            if (qi < L) {
                uint4 *dst = reinterpret_cast<uint4 *>(ctx + (size_t)(it.start + qi) * kHidden + it.h * kHeadDim);
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const uint32_t *x = o[q >> 2] + (q & 3) * 8;
                    dst[q] = make_uint4(pack_bf16x2(__uint_as_float(x[0]) * inv, __uint_as_float(x[1]) * inv),
                                        pack_bf16x2(__uint_as_float(x[2]) * inv, __uint_as_float(x[3]) * inv),
                                        pack_bf16x2(__uint_as_float(x[4]) * inv, __uint_as_float(x[5]) * inv),
                                        pack_bf16x2(__uint_as_float(x[6]) * inv, __uint_as_float(x[7]) * inv));
                }
            }
            ++i;
        }
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, LKB * LQ);
    }
    if (threadIdx.x == 0 && *sm.abort_flag) set_status(status, kStatusTimeout);
}

}  // namespace

cudaError_t launch_attention_tc_long(const CUtensorMap &tmQKV, bf16 *ctx, const int *seq_start, const int *seq_len,
                                     int nseq, int *status, int num_sms, cudaStream_t s, bool trigger,
                                     unsigned long long wait_ns) {
    if (nseq <= 0) return cudaSuccess;
    static std::atomic<unsigned long long> configured{0};
    cudaError_t e = ensure_smem_attr(reinterpret_cast<const void *>(attn_tc_long_kernel), LA_SMEM, configured);
    if (e != cudaSuccess) return e;
    const int total = nseq * LKB * kHeads;
    const int grid = total < num_sms ? total : num_sms;
    return launch_pdl(attn_tc_long_kernel, dim3(grid), dim3(LA_THREADS), LA_SMEM, s, tmQKV, ctx, seq_start, seq_len,
                      nseq, status, trigger ? 1 : 0, wait_ns);
}

}  // namespace albert
