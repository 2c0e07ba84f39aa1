// attention_tc.cu -- masked bidirectional attention on the 5th-generation tensor
// cores (tcgen05) for sequences of at most 128 tokens.
//
// Per sequence b and head h ("ALBERT: How Kokoro's Phoneme Encoder Works",
// section "Inside One Real ALBERT Layer", step 4; "How Kokoro TTS Works and
// Where CKE Stands", section "What ALBERT does here"):
//     C_h = softmax(Q_h K_h^T / sqrt(64) + mask) V_h,
// key u of sequence b takes part iff u < L_b, every query sees both sides.
//
// One work item = (group, head), all of the group's <= 128 queries and keys at
// once.  A group is one sequence, or two sequences of at most 64 tokens (paired
// by the prep kernels) loaded as the two 64-row halves of the item's tiles:
// queries, keys and values of the first in rows 0..63, of the second in rows
// 64..127, each query taking only the keys of its own half.  Every softmax warp
// then has real rows, where a lone short sequence leaves half of them idle.
// The group entries of every item of the CTA are read into shared memory once,
// before the roles start (a global load per item on the issuing threads' path
// cost about as much as the item itself).
//   warp 0      : TMA producer of the head's Q and K tiles (128 or 64 rows x
//                 64, or two 64-row halves; 128-byte swizzle) from the packed
//                 [rows, 3*768] buffer
//                 into a ring of stages; a Q/K stage is free again as soon as
//                 the S product has read it, so Q/K loads run well ahead.  It
//                 also loads the V tiles of the first four items; the V tile
//                 of item n + 4 is loaded by the output group as soon as the O
//                 product of item n, the last reader of that V stage, is
//                 complete;
//   warp 1      : tcgen05.mma issuer of the score products S = Q K^T (M=128,
//                 N=128 or 64, K=64) into a TMEM buffer, item after item;
//   warp 14     : tcgen05.mma issuer of the output products O = P V (M=128,
//                 N=64, K = L rounded up to 16) with P read from TMEM and V
//                 from shared memory as an MN-major operand.  Two issuing
//                 threads: the cost of issuing, committing and polling on one
//                 thread (about as much per MMA as the MMA itself) no longer
//                 serializes the two products of successive items;
//   warps 2..9  : two softmax groups of 4 warps (items alternate between
//                 them): each thread owns one query row, reads its scores from
//                 TMEM, applies the mask (keys of the row's own sequence) and
//                 a max-subtracted softmax in registers (no cross-thread
//                 reductions), writes P as packed bf16 back into TMEM over
//                 scores it has read (zeros for every other key of the item)
//                 and 1/sum into shared memory, and moves on to its next item;
//   warps 10..13: output group: per item, reads its rows of O from TMEM once
//                 O = P V is complete, scales them by 1/sum and stores them.
// TMEM holds four 128-column item buffers: S fills a buffer, P is packed into
// its first 64 columns and O lands in the last 64 (scores already consumed),
// so four items are in flight between the S product and the output, and a
// softmax group finds its next scores ready when it finishes an item.  A warp
// whose 32 query rows all lie past the sequence's end skips its softmax and
// output.  Every wait is bounded (%globaltimer).
#include "kernels.h"
#include "sm100_ptx.cuh"

namespace albert {
namespace {

constexpr int TROWS = 128;                     // query rows / keys per item
constexpr int TILE = TROWS * 128;              // 128 rows x 64 bf16 = 16 KB
constexpr int NQK = 4;                         // Q/K stages (2 tiles each)
constexpr int NV = 4;                          // V stages (1 tile each)
constexpr int NBUF = 4;                        // TMEM item buffers (128 columns each)
constexpr int ATC_THREADS = 32 * 15;
constexpr int ATC_O_WARP = 14;                 // issuer of the O = P V products
constexpr int ATC_ITEM_CAP = 512;              // items whose (start, length) are kept in shared memory
constexpr int ATC_SMEM = 1024 + (2 * NQK + NV) * TILE + NBUF * TROWS * 4 + ATC_ITEM_CAP * 16 + 512;
constexpr uint32_t TM_O = 64;                  // O's first column within an item buffer
// Item n uses Q/K stage, V stage and TMEM buffer n % 4 alike, so a Q/K stage is
// free when the S product of the item four back completes (s_full) and a V
// stage when its O product completes (o_full): no separate release barriers,
// and two fewer tcgen05.commit per item on the issuing thread.
static_assert(NQK == NBUF && NV == NBUF, "stages and TMEM buffers share one index");

struct AttSmem {
    uint8_t *qk, *v;                           // [NQK][Q tile, K tile], [NV][V tile]
    uint64_t *qk_full;                         // [NQK]
    uint64_t *v_full;                          // [NV]
    uint64_t *s_full, *p_full, *o_full, *o_empty;  // [NBUF]
    uint64_t *drain, *drain_o;                 // each issuer's products complete
    uint32_t *tmem_slot;
    volatile int *abort_flag;
    int *misc;
    int *qk_len, *v_len;                       // length of the item a stage holds
    float *inv_sum;                            // [NBUF][TROWS]
    int4 *item;                                // [ATC_ITEM_CAP] group entries of the CTA's items
    int *n_issued;                             // [0] Q/K, [1] V loads issued (read by the teardown)
};

__device__ __forceinline__ AttSmem att_carve(uint8_t *raw) {
    AttSmem s;
    uint8_t *p = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
    s.qk = p;
    s.v = p + 2 * NQK * TILE;
    s.inv_sum = reinterpret_cast<float *>(s.v + NV * TILE);
    s.item = reinterpret_cast<int4 *>(s.v + NV * TILE + NBUF * TROWS * 4);
    uint64_t *b = reinterpret_cast<uint64_t *>(s.item + ATC_ITEM_CAP);
    s.qk_full = b;
    s.v_full = b + 2 * NQK;
    s.s_full = b + 2 * NQK + 2 * NV;
    s.p_full = s.s_full + NBUF;
    s.o_full = s.s_full + 2 * NBUF;
    s.o_empty = s.s_full + 3 * NBUF;
    s.drain = s.s_full + 4 * NBUF;
    s.drain_o = s.drain + 1;
    uint32_t *u = reinterpret_cast<uint32_t *>(s.drain + 2);
    s.tmem_slot = u;
    s.abort_flag = reinterpret_cast<volatile int *>(u + 1);
    s.misc = reinterpret_cast<int *>(u + 2);
    s.qk_len = s.misc + 2;
    s.v_len = s.qk_len + NQK;
    s.n_issued = s.v_len + NV;
    return s;
}

// Group entry {start, length, partner start, partner length} of the CTA's item j
// (id = blockIdx.x + j * gridDim.x = group * 12 + head).
__device__ __forceinline__ int4 item_info(const AttSmem &sm, int j, const int4 *groups) {
    if (j < ATC_ITEM_CAP) return sm.item[j];
    return groups[(blockIdx.x + j * gridDim.x) / kHeads];
}
__device__ __forceinline__ bool item_pair(int4 it) { return it.w > 0; }
// rows (and keys) of the item's tiles: a pair fills both 64-row halves
__device__ __forceinline__ int item_rows(int4 it) { return it.w > 0 ? TROWS : it.y; }

// TMA load of 64 columns (one head) of the item's rows into a 128-row tile: one
// box, or one 64-row box per half for a pair (the second lands 64 rows = 8 KB in,
// a multiple of the 1 KB swizzle period).
__device__ __forceinline__ void load_item_tile(uint32_t dst, int4 it, int col, const CUtensorMap *tmQKV,
                                               const CUtensorMap *tmQKV64, uint32_t bar) {
    if (item_pair(it)) {
        tma_load_2d(dst, tmQKV64, bar, col, it.x);
        tma_load_2d(dst + TILE / 2, tmQKV64, bar, col, it.z);
    } else {
        tma_load_2d(dst, it.y <= 64 ? tmQKV64 : tmQKV, bar, col, it.x);
    }
}

// TMA load of the V tile of the CTA's item n into V stage n % NV (one thread).
__device__ __forceinline__ void issue_v(const AttSmem &sm, int n, int4 it, const CUtensorMap *tmQKV,
                                        const CUtensorMap *tmQKV64) {
    const int h = (blockIdx.x + n * gridDim.x) % kHeads;
    const int st = n % NV;
    const int rows = item_rows(it);
    sm.v_len[st] = rows;  // read by the O issuer once the stage is full
    const uint32_t fb = smem_u32(&sm.v_full[st]);
    mbar_arrive_expect_tx(fb, rows <= 64 ? TILE / 2 : TILE);
    load_item_tile(smem_u32(sm.v + st * TILE), it, 2 * kHidden + h * kHeadDim, tmQKV, tmQKV64, fb);
}

__global__ void __launch_bounds__(ATC_THREADS, 1)
attn_tc_kernel(const __grid_constant__ CUtensorMap tmQKV, const __grid_constant__ CUtensorMap tmQKV64,
               bf16 *__restrict__ ctx, const int4 *__restrict__ groups, const int *__restrict__ n_groups,
               int max_groups, int *status, int trigger, unsigned long long wait_ns) {
    if (trigger) griddep_launch_dependents();  // the next kernel may take SMs as this grid frees them
    griddep_wait();               // the previous kernel has completed

    extern __shared__ uint8_t smem_raw[];
    AttSmem sm = att_carve(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        sm.misc[0] = *reinterpret_cast<const volatile int *>(status);
        const int ng = *reinterpret_cast<const volatile int *>(n_groups);
        sm.misc[1] = ng < 0 ? 0 : (ng > max_groups ? max_groups : ng);
        *sm.abort_flag = 0;
        wait_limit_init(wait_ns);
        for (int i = 0; i < NQK; ++i) mbar_init(smem_u32(&sm.qk_full[i]), 1);
        for (int i = 0; i < NV; ++i) mbar_init(smem_u32(&sm.v_full[i]), 1);
        for (int i = 0; i < NBUF; ++i) {
            mbar_init(smem_u32(&sm.s_full[i]), 1);
            mbar_init(smem_u32(&sm.p_full[i]), 4);
            mbar_init(smem_u32(&sm.o_full[i]), 1);
            mbar_init(smem_u32(&sm.o_empty[i]), 4);
        }
        mbar_init(smem_u32(sm.drain), 1);
        mbar_init(smem_u32(sm.drain_o), 1);
        fence_mbar_init();
        sm.n_issued[0] = sm.n_issued[1] = sm.n_issued[2] = 0;
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmQKV);
        prefetch_tmap(&tmQKV64);
    }
    __syncthreads();
    if (sm.misc[0] != 0) return;  // an earlier kernel of this forward failed
    const int total = sm.misc[1] * kHeads;  // item id = group * 12 + h
    // items of this CTA: id = blockIdx.x + j * gridDim.x, j < n_items
    const int n_items = (int)blockIdx.x < total ? (total - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    for (int j = threadIdx.x; j < n_items && j < ATC_ITEM_CAP; j += blockDim.x)
        sm.item[j] = groups[(blockIdx.x + j * gridDim.x) / kHeads];
    if (warp == 1) {
        tmem_alloc(smem_u32(sm.tmem_slot), NBUF * TROWS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *sm.tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------ TMA producer --
        // Q/K of item n into stage n % 4 once the S product of item n - 4 has read
        // it; the V tiles of items 0..3 alongside.
        if (lane == 0) {
            int nq = 0;
            for (; nq < n_items; ++nq) {
                const int st = nq % NQK;
                if (!mbar_wait(smem_u32(&sm.s_full[st]), ((nq / NQK) & 1) ^ 1, sm.abort_flag)) break;
                const int4 it = item_info(sm, nq, groups);
                const int h = (blockIdx.x + nq * gridDim.x) % kHeads;
                const int rows = item_rows(it);
                sm.qk_len[st] = rows;  // read by the issuer once the stage is full
                // a lone sequence of at most 64 tokens moves 64-row tiles
                const uint32_t dst = smem_u32(sm.qk + st * 2 * TILE);
                const uint32_t fb = smem_u32(&sm.qk_full[st]);
                mbar_arrive_expect_tx(fb, rows <= 64 ? TILE : 2 * TILE);
                load_item_tile(dst, it, h * kHeadDim, &tmQKV, &tmQKV64, fb);
                load_item_tile(dst + TILE, it, kHidden + h * kHeadDim, &tmQKV, &tmQKV64, fb);
                sm.n_issued[0] = nq + 1;
                if (nq < NV) {
                    issue_v(sm, nq, it, &tmQKV, &tmQKV64);
                    sm.n_issued[1] = nq + 1;
                }
            }
        }
    } else if (warp == 1) {
        // --------------------------------------------- score-product issuer --
        // S of item n goes into TMEM buffer n % 4 once its Q/K stage is full and
        // the output group has read O of item n - 4 from that buffer.
        if (lane == 0) {
            const uint32_t idesc_s128 = idesc_bf16_f32(TROWS, TROWS);
            const uint32_t idesc_s64 = idesc_bf16_f32(TROWS, 64);
            for (int ns = 0; ns < n_items; ++ns) {
                const int tb = ns % NBUF, st = ns % NQK;
                if (!mbar_wait(smem_u32(&sm.qk_full[st]), (ns / NQK) & 1, sm.abort_flag) ||
                    !mbar_wait(smem_u32(&sm.o_empty[tb]), ((ns / NBUF) & 1) ^ 1, sm.abort_flag))
                    break;
                tc_fence_after();
                const int L = sm.qk_len[st];
                const uint32_t q = smem_u32(sm.qk + st * 2 * TILE), k = q + TILE;
#pragma unroll
                for (int kk = 0; kk < kHeadDim / 16; ++kk)
                    umma_bf16(tmem_base + tb * TROWS, sw128_kmajor_desc(q + kk * 32), sw128_kmajor_desc(k + kk * 32),
                              L <= 64 ? idesc_s64 : idesc_s128, kk != 0);
                umma_commit(smem_u32(&sm.s_full[tb]));  // also frees Q/K stage st (== tb)
            }
            umma_commit(smem_u32(sm.drain));
            mbar_wait_drain(smem_u32(sm.drain), 0);
        }
    } else if (warp == ATC_O_WARP) {
        // -------------------------------------------- output-product issuer --
        // O of item n once the softmax has written P over its scores (p_full, which
        // also means every score of the buffer has been read) and its V stage is full.
        if (lane == 0) {
            const uint32_t idesc_o = idesc_bf16_f32(TROWS, kHeadDim) | (1u << 16);  // B (= V) MN-major
            for (int no = 0; no < n_items; ++no) {
                const int tb = no % NBUF, st = no % NV;
                if (!mbar_wait(smem_u32(&sm.p_full[tb]), (no / NBUF) & 1, sm.abort_flag) ||
                    !mbar_wait(smem_u32(&sm.v_full[st]), (no / NV) & 1, sm.abort_flag))
                    break;
                tc_fence_after();
                const int L = sm.v_len[st];
                const int ksteps = (L + 15) >> 4;
                const uint32_t vbase = smem_u32(sm.v + st * TILE);
                const uint32_t buf = tmem_base + tb * TROWS;
                for (int kk = 0; kk < ksteps; ++kk) {
                    // P: 16 keys = 8 packed TMEM columns; V: 16 keys = 16 rows of 128 B
                    umma_bf16_ts(buf + TM_O, buf + kk * 8, sw128_kmajor_desc(vbase + kk * 2048), idesc_o, kk != 0);
                }
                umma_commit(smem_u32(&sm.o_full[tb]));  // also frees V stage st (== tb)
            }
            umma_commit(smem_u32(sm.drain_o));
            mbar_wait_drain(smem_u32(sm.drain_o), 0);
        }
    } else if (warp < 10) {
        // ------------------------------------------------------ softmax warps --
        const int g = (warp - 2) >> 2;   // items i with i % 2 == g
        const int quad = warp & 3;
        const int r = quad * 32 + lane;  // query row within the item
        const float sl2 = 0.125f * 1.4426950408889634f;
        const uint32_t trow = tmem_base + ((uint32_t)(quad * 32) << 16);
        int i = 0;
        for (int id = blockIdx.x; id < total; id += gridDim.x, ++i) {
            if ((i & 1) != g) continue;
            const int tb = i % NBUF;
            const uint32_t ph = (i / NBUF) & 1;
            const int4 it = item_info(sm, i, groups);
            // A pair's second sequence holds rows and keys 64..127: its warps read
            // scores from column 64 and write P from column 32 (keys 64..127), and
            // otherwise run as for a sequence of their own.
            const bool pair = item_pair(it), hi = pair && quad >= 2;
            const int L = hi ? it.w : it.y;  // keys of this warp's sequence
            const uint32_t srow = trow + tb * TROWS + (hi ? 64u : 0u);
            const uint32_t prow = trow + tb * TROWS + (hi ? 32u : 0u);
            const int nch = (L + 31) >> 5;  // 32-key chunks holding valid keys
            const bool live = (hi ? quad * 32 - 64 : quad * 32) < L;  // some row of this warp is a real query
            bool got = mbar_wait(smem_u32(&sm.s_full[tb]), ph, sm.abort_flag);
            got = __all_sync(0xffffffffu, got);
            if (!got) break;
            tc_fence_after();
            if (live) {
                // pass 1: row maximum over the valid keys (two 32-key chunks per TMEM wait)
                // (four independent max / sum chains: a single chain is latency-bound)
                float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
                uint32_t v[2][32];
#pragma unroll 1
                for (int c = 0; c < nch; c += 2) {
                    tmem_ld32(srow + c * 32, v[0]);
                    if (c + 1 < nch) tmem_ld32(srow + (c + 1) * 32, v[1]);
                    tmem_ld_wait();
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int base = (c + e) * 32;
                        if (c + e >= nch) continue;
                        if (base + 32 <= L) {
#pragma unroll
                            for (int j = 0; j < 32; j += 2)
                                mx[(j >> 1) & 3] = fmax3(mx[(j >> 1) & 3], __uint_as_float(v[e][j]),
                                                           __uint_as_float(v[e][j + 1]));
                        } else {
#pragma unroll
                            for (int j = 0; j < 32; ++j)
                                if (base + j < L) mx[j & 3] = fmaxf(mx[j & 3], __uint_as_float(v[e][j]));
                        }
                    }
                }
                const float m = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
                // pass 2: P = exp(scale * (s - max)) packed as bf16 pairs; chunk c goes to
                // columns 16c..16c+15 of the same buffer, which hold scores already read
                const uint64_t sl2x2 = f2_make(sl2, sl2), nms2 = f2_make(-m * sl2, -m * sl2);
                uint64_t lsum[2] = {f2_make(0.f, 0.f), f2_make(0.f, 0.f)};
#pragma unroll 1
                for (int c = 0; c < nch; c += 2) {
                    if (nch > 2) {  // up to 64 keys the row is still in registers
                        tmem_ld32(srow + c * 32, v[0]);
                        if (c + 1 < nch) tmem_ld32(srow + (c + 1) * 32, v[1]);
                        tmem_ld_wait();
                    }
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int cc = c + e;
                        if (cc >= nch) continue;
                        const bool full = cc * 32 + 32 <= L;
                        uint32_t pk[16];
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            const int k0 = cc * 32 + 2 * j;
                            const float2 x = f2_split(f2_fma(f2_make_u(v[e][2 * j], v[e][2 * j + 1]), sl2x2, nms2));
                            float p0 = ex2_approx(x.x), p1 = ex2_approx(x.y);
                            if (!full) {
                                p0 = k0 < L ? p0 : 0.f;
                                p1 = k0 + 1 < L ? p1 : 0.f;
                            }
                            lsum[j & 1] = f2_add(lsum[j & 1], f2_make(p0, p1));
                            pk[j] = pack_bf16x2(p0, p1);
                        }
                        tmem_st16(prow + cc * 16, pk);
                    }
                }
                if (pair) {
                    // the O product reads P for all 128 keys: the other half's keys
                    // (and those past this sequence's end) get P = 0
                    uint32_t z[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) z[j] = 0u;
                    const uint32_t p0row = trow + tb * TROWS;
                    for (int cc = 0; cc < 4; ++cc) {
                        const int rel = cc - (hi ? 2 : 0);  // chunk within this warp's half
                        if (rel < 0 || rel >= nch) tmem_st16(p0row + cc * 16, z);
                    }
                }
                const float2 ls = f2_split(f2_add(lsum[0], lsum[1]));
                // read by the output group after it has waited on p_full
                sm.inv_sum[tb * TROWS + r] = 1.f / (ls.x + ls.y);
                tmem_st_wait();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&sm.p_full[tb]));
        }
    } else {
        // ------------------------------------------------------- output warps --
        const int quad = warp & 3;
        const int r = quad * 32 + lane;  // query row within the item
        const uint32_t trow = tmem_base + ((uint32_t)(quad * 32) << 16);
        int i = 0;
        for (int id = blockIdx.x; id < total; id += gridDim.x, ++i) {
            const int tb = i % NBUF;
            const uint32_t ph = (i / NBUF) & 1;
            const int h = id % kHeads;
            const int4 it = item_info(sm, i, groups);
            // this warp's rows belong to the pair's second sequence (rows 64..127) or
            // to the item's first (or only) one
            const bool hi = item_pair(it) && quad >= 2;
            const int start = hi ? it.z : it.x, n_valid = hi ? it.w : it.y;
            const int rs = hi ? r - 64 : r;  // row within its sequence
            const bool live = (hi ? quad * 32 - 64 : quad * 32) < n_valid;
            // p_full (complete before O is) makes the softmax's 1/sum visible here
            bool got = mbar_wait(smem_u32(&sm.o_full[tb]), ph, sm.abort_flag) &&
                       mbar_wait(smem_u32(&sm.p_full[tb]), ph, sm.abort_flag);
            got = __all_sync(0xffffffffu, got);
            if (!got) break;
            tc_fence_after();
            // O of item i is complete: its V stage takes the V tile of item i + 4
            if (warp == 10 && lane == 0 && i + NV < n_items) {
                issue_v(sm, i + NV, item_info(sm, i + NV, groups), &tmQKV, &tmQKV64);
                sm.n_issued[2] = i + 1;
            }
            uint32_t o[2][32];
            float inv = 0.f;
            if (live) {
                tmem_ld32(trow + tb * TROWS + TM_O, o[0]);
                tmem_ld32(trow + tb * TROWS + TM_O + 32, o[1]);
                inv = sm.inv_sum[tb * TROWS + r];
                tmem_ld_wait();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(&sm.o_empty[tb]));
            if (rs < n_valid) {
                uint4 *dst = reinterpret_cast<uint4 *>(ctx + (size_t)(start + rs) * kHidden + h * kHeadDim);
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    const uint32_t *x = o[q >> 2] + (q & 3) * 8;
                    dst[q] = make_uint4(pack_bf16x2(__uint_as_float(x[0]) * inv, __uint_as_float(x[1]) * inv),
                                        pack_bf16x2(__uint_as_float(x[2]) * inv, __uint_as_float(x[3]) * inv),
                                        pack_bf16x2(__uint_as_float(x[4]) * inv, __uint_as_float(x[5]) * inv),
                                        pack_bf16x2(__uint_as_float(x[6]) * inv, __uint_as_float(x[7]) * inv));
                }
            }
        }
    }

    __syncthreads();
    if (threadIdx.x == 0 && *sm.abort_flag) {
        // loads still in flight land before the CTA's shared memory goes away (the
        // last four issued of each ring; the V tiles issued are items 0..last)
        const int nq = sm.n_issued[0];
        for (int j = nq > NQK ? nq - NQK : 0; j < nq; ++j)
            mbar_wait_drain(smem_u32(&sm.qk_full[j % NQK]), (j / NQK) & 1);
        const int nv = sm.n_issued[2] > 0 ? NV + sm.n_issued[2] : sm.n_issued[1];
        for (int j = nv > NV ? nv - NV : 0; j < nv; ++j)
            mbar_wait_drain(smem_u32(&sm.v_full[j % NV]), (j / NV) & 1);
    }
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, NBUF * TROWS);
    }
    if (threadIdx.x == 0 && *sm.abort_flag) set_status(status, kStatusTimeout);
}

}  // namespace

cudaError_t launch_attention_tc(const CUtensorMap &tmQKV, const CUtensorMap &tmQKV64, bf16 *ctx, const int4 *groups,
                                const int *n_groups, int max_groups, int *status, int num_sms, cudaStream_t s,
                                bool trigger, unsigned long long wait_ns) {
    if (max_groups <= 0) return cudaSuccess;
    static std::atomic<unsigned long long> configured{0};
    cudaError_t e = ensure_smem_attr(reinterpret_cast<const void *>(attn_tc_kernel), ATC_SMEM, configured);
    if (e != cudaSuccess) return e;
    // sized for one group per sequence; CTAs past the groups' items have none
    const int total = max_groups * kHeads;
    const int grid = total < num_sms ? total : num_sms;
    return launch_pdl(attn_tc_kernel, dim3(grid), dim3(ATC_THREADS), ATC_SMEM, s, tmQKV, tmQKV64, ctx, groups,
                      n_groups, max_groups, status, trigger ? 1 : 0, wait_ns);
}

}  // namespace albert
