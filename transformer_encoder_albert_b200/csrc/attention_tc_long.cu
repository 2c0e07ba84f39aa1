// attention_tc_long.cu -- masked bidirectional attention on the 5th-generation
// tensor cores (tcgen05) for batches whose longest sequence has 129..512 tokens.
//
// Per sequence b and head h ("ALBERT: How Kokoro's Phoneme Encoder Works",
// section "Inside One Real ALBERT Layer", step 4; "How Kokoro TTS Works and
// Where CKE Stands", section "What ALBERT does here"):
//     C_h = softmax(Q_h K_h^T / sqrt(64) + mask) V_h,
// key u of sequence b takes part iff u < L_b, every query sees both sides.
//
// One work item = (sequence b, query block qb of 128 rows, head h).  The keys
// are taken in blocks of 64 with a running row maximum m: for block j,
// S_j = Q K_j^T, P_j = exp(S_j - m), O += P_j V_j and l += rowsum(P_j); the
// result is O / l.  m is raised only when a block's maximum exceeds it by more
// than 2^8 in the exponential (O and l are then rescaled in place); otherwise
// P_j may reach 2^8, which bf16 P and fp32 O and l hold as precisely as values
// below 1, and O / l is the softmax of the definition whichever m was used.
//
// Two items are in flight per CTA, in two slots that share nothing but the SM:
// each has its own TMA producer (Q double-buffered, a ring of {K, V} 64-row
// block tiles), its own tcgen05.mma issuing thread and its own four softmax
// warps (one per TMEM lane quadrant, each thread one query row).  Per slot,
// tensor memory holds two 64-column score buffers and a 64-column O
// accumulator: the issuer computes S_{j+1} (and S_{j+2} once P_j V_j is issued)
// while the softmax works on block j, so the softmax never waits for a product
// of its own item once the pipeline is full.  P_j is written as packed bf16 over
// the first 32 columns of its score buffer.  A slot's products run in its
// thread's issue order, so S_{j+2} cannot overwrite P_j before P_j V_j has read
// it.  A rescale of O while on block j waits for S_{j+1}: the issuer issues it
// right after P_{j-1} V_{j-1}, and its completion covers every earlier product
// of the slot (after the slot's last S, a commit with no product stands in for
// it).  After an item's last block its softmax warps read O, scale it by 1 / l
// and store it.  A warp whose 32 query rows all lie past the sequence's end
// skips the arithmetic but takes part in every barrier.  Every wait is bounded
// (%globaltimer).
#include "kernels.h"
#include "sm100_ptx.cuh"

namespace albert {
namespace {

constexpr int LQ = 128;                        // query rows per item
constexpr int LKB = 4;                         // 128-key spans: L <= 512
constexpr int KB = 64;                         // keys per block
constexpr int QTILE = LQ * 128;                // 128 rows x 64 bf16 = 16 KB
constexpr int KVTILE = KB * 128;               // 64 rows x 64 bf16 = 8 KB
constexpr int NKV = 4;                         // {K, V} block stages per slot
constexpr int LA_THREADS = 32 * 12;            // producer 0 / 10, issuer 1 / 11, softmax 2..9
// per slot s: score buffers at 192 s + {0, 64}, O at 192 s + 128
constexpr uint32_t SLOT_COLS = 192;
constexpr float kRescaleLog2 = 8.0f;
constexpr int SLOT_BYTES = 2 * QTILE + NKV * 2 * KVTILE;  // 96 KB
constexpr int LA_ITEM_CAP = 512;               // items of a CTA kept in shared memory
constexpr int LA_SMEM = 1024 + 2 * SLOT_BYTES + 512 + LA_ITEM_CAP * 16;
static_assert(LA_SMEM <= 232448, "shared memory per CTA");

struct SlotSmem {
    uint8_t *q, *kv;                           // [2] Q tiles; [NKV] {K tile, V tile}
    uint64_t *q_full, *q_empty;                // [2]
    uint64_t *kv_full, *kv_empty;              // [NKV]
    uint64_t *s_full, *p_full;                 // [2] per score buffer
    uint64_t *o_full, *o_empty, *drain;
};

__device__ __forceinline__ uint8_t *smem_base(uint8_t *raw) {
    return reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
}

__device__ __forceinline__ SlotSmem slot_carve(uint8_t *raw, int slot, uint64_t **bars_end) {
    uint8_t *p = smem_base(raw);
    SlotSmem s;
    s.q = p + slot * SLOT_BYTES;
    s.kv = s.q + 2 * QTILE;
    uint64_t *b = reinterpret_cast<uint64_t *>(p + 2 * SLOT_BYTES) + slot * (4 + 2 * NKV + 7);
    s.q_full = b;
    s.q_empty = b + 2;
    s.kv_full = b + 4;
    s.kv_empty = b + 4 + NKV;
    s.s_full = b + 4 + 2 * NKV;
    s.p_full = s.s_full + 2;
    s.o_full = s.s_full + 4;
    s.o_empty = s.s_full + 5;
    s.drain = s.s_full + 6;
    if (bars_end) *bars_end = reinterpret_cast<uint64_t *>(p + 2 * SLOT_BYTES) + 2 * (4 + 2 * NKV + 7);
    return s;
}

struct LongItem {
    int h, qb, L, start;
};

// The CTA's items: slots id = blockIdx.x + k * gridDim.x of nseq * LKB * 12,
// slot = (b, qb, h); query blocks past the sequence's end are skipped.
__device__ __forceinline__ bool next_long_item(int &id, int total, const int *__restrict__ seq_start,
                                               const int *__restrict__ seq_len, LongItem &it) {
    for (; id < total; id += gridDim.x) {
        const int b = id / (LKB * kHeads), rem = id - b * (LKB * kHeads);
        const int qb = rem / kHeads;
        // lengths are validated against max_len <= 512 before this kernel runs; the
        // clamp only keeps every tile in bounds regardless
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

__device__ __forceinline__ int key_blocks(int L) { return (L + KB - 1) / KB; }

// The CTA's first LA_ITEM_CAP items (h, qb, L, start), built in shared memory
// before the roles start: walking the candidates through global memory at every
// item boundary put a chain of dependent loads on each role's path.  resume is
// the candidate index of the first item past the table, or -1 if there is none.
struct ItemTable {
    const int4 *tab;
    int n, resume;
};

// The items of one slot: the CTA's items k with k % 2 == slot, from the table,
// then (past it) from the candidates in global memory.
struct SlotCursor {
    ItemTable t;
    int k;      // next table index of this slot
    int id, c;  // past the table: next candidate id and the CTA item index it would get
    __device__ void start(int slot, const ItemTable &tb) {
        t = tb;
        k = slot;
        id = -1;
        c = 0;
    }
    __device__ bool next(int slot, int total, const int *seq_start, const int *seq_len, LongItem &it) {
        if (k < t.n) {
            const int4 e = t.tab[k];
            k += 2;
            it.h = e.x;
            it.qb = e.y;
            it.L = e.z;
            it.start = e.w;
            return true;
        }
        if (t.resume < 0) return false;
        if (id < 0) {
            id = blockIdx.x + t.resume * gridDim.x;
            c = t.n;
        }
        LongItem u;
        while (next_long_item(id, total, seq_start, seq_len, u)) {
            if ((c++ & 1) == slot) {
                it = u;
                return true;
            }
        }
        return false;
    }
};

// A slot's key blocks over all of its items, in order: block counter b (the
// score buffer is b & 1, the {K, V} stage b % NKV), item counter n (the Q
// buffer is n & 1), the item and the block's index j within it.
struct SlotBlocks {
    SlotCursor cur;
    LongItem it;
    bool has;
    int j, n, b;
    __device__ void start(int slot, int total, const int *seq_start, const int *seq_len, const ItemTable &tb) {
        cur.start(slot, tb);
        has = cur.next(slot, total, seq_start, seq_len, it);
        j = 0;
        n = 0;
        b = 0;
    }
    __device__ void advance(int slot, int total, const int *seq_start, const int *seq_len) {
        ++b;
        if (++j == key_blocks(it.L)) {
            has = cur.next(slot, total, seq_start, seq_len, it);
            j = 0;
            ++n;
        }
    }
};

__global__ void __launch_bounds__(LA_THREADS, 1)
attn_tc_long_kernel(const __grid_constant__ CUtensorMap tmQKV, const __grid_constant__ CUtensorMap tmQKV64,
                    bf16 *__restrict__ ctx, const int *__restrict__ seq_start, const int *__restrict__ seq_len,
                    int nseq, int *status, int trigger, unsigned long long wait_ns) {
    if (trigger) griddep_launch_dependents();  // the next kernel may take SMs as this grid frees them
    griddep_wait();               // the previous kernel has completed

    extern __shared__ uint8_t smem_raw[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // roles: slot 0 -- producer warp 0, issuer warp 1, softmax warps 2..5;
    //        slot 1 -- producer warp 10, issuer warp 11, softmax warps 6..9
    const int slot = (warp == 0 || warp == 1 || (warp >= 2 && warp < 6)) ? 0 : 1;
    uint64_t *bars_end = nullptr;
    SlotSmem sm = slot_carve(smem_raw, slot, &bars_end);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars_end);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    int *misc = reinterpret_cast<int *>(tmem_slot + 2);

    if (threadIdx.x == 0) {
        misc[0] = *reinterpret_cast<const volatile int *>(status);
        *abort_flag = 0;
        wait_limit_init(wait_ns);
        for (int s = 0; s < 2; ++s) {
            SlotSmem t = slot_carve(smem_raw, s, nullptr);
            for (int i = 0; i < 2; ++i) {
                mbar_init(smem_u32(&t.q_full[i]), 1);
                mbar_init(smem_u32(&t.q_empty[i]), 1);
                mbar_init(smem_u32(&t.s_full[i]), 1);
                // per score buffer: a warp may arrive for block j + 1 before the others
                // finish block j, never for block j + 2 (its S follows P_j V)
                mbar_init(smem_u32(&t.p_full[i]), 4);  // the slot's four softmax warps
            }
            for (int i = 0; i < NKV; ++i) {
                mbar_init(smem_u32(&t.kv_full[i]), 1);
                mbar_init(smem_u32(&t.kv_empty[i]), 1);
            }
            mbar_init(smem_u32(t.o_full), 1);
            mbar_init(smem_u32(t.o_empty), 4);
            mbar_init(smem_u32(t.drain), 1);
        }
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&tmQKV);
        prefetch_tmap(&tmQKV64);
    }
    __syncthreads();
    if (misc[0] != 0) return;  // an earlier kernel of this forward failed
    const int total = nseq * LKB * kHeads;
    ItemTable items;
    {
        // candidates blockIdx.x + c * gridDim.x, c = 0 .. ncand - 1, compacted in order:
        // per chunk of LA_THREADS candidates, warp ballots, then the warps' counts
        int4 *tab = reinterpret_cast<int4 *>(smem_base(smem_raw) + 2 * SLOT_BYTES + 512);
        int *wcount = misc + 4;  // [LA_THREADS / 32]
        const int ncand = total > (int)blockIdx.x ? (total - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x : 0;
        int found = 0;
        for (int c0 = 0; c0 < ncand; c0 += LA_THREADS) {
            const int c = c0 + threadIdx.x;
            int4 e = make_int4(0, 0, 0, 0);
            bool valid = false;
            if (c < ncand) {
                const int id = blockIdx.x + c * gridDim.x;
                const int sb = id / (LKB * kHeads), rem = id - sb * (LKB * kHeads);
                const int qb = rem / kHeads;
                // lengths are validated against max_len <= 512 before this kernel runs;
                // the clamp only keeps every tile in bounds regardless
                const int L = min(__ldg(seq_len + sb), LKB * LQ);
                valid = qb * LQ < L;
                if (valid) e = make_int4(rem - qb * kHeads, qb, L, __ldg(seq_start + sb));
            }
            const unsigned bal = __ballot_sync(0xffffffffu, valid);
            if (lane == 0) wcount[warp] = __popc(bal);
            __syncthreads();
            int before = found, chunk = 0;
            for (int w = 0; w < LA_THREADS / 32; ++w) {
                before += w < warp ? wcount[w] : 0;
                chunk += wcount[w];
            }
            const int rank = before + __popc(bal & ((1u << lane) - 1));
            if (valid && rank < LA_ITEM_CAP) tab[rank] = e;
            if (valid && rank == LA_ITEM_CAP) misc[2] = c;
            found += chunk;
            __syncthreads();  // wcount is rewritten by the next chunk
        }
        items.tab = tab;
        items.n = min(found, LA_ITEM_CAP);
        items.resume = found > LA_ITEM_CAP ? misc[2] : -1;
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const uint32_t sbase = tmem_base + slot * SLOT_COLS;

    if (warp == 0 || warp == 10) {
        // ------------------------------------------------------ TMA producer --
        if (lane == 0) {
            SlotBlocks bl;
            bl.start(slot, total, seq_start, seq_len, items);
            int nq = 0;
            while (bl.has) {
                if (bl.j == 0) {
                    // Q buffer n & 1: free once the last S of the slot's item n - 2 has read it
                    const int qb = bl.n & 1;
                    if (!mbar_wait(smem_u32(&sm.q_empty[qb]), ((bl.n >> 1) & 1) ^ 1, abort_flag)) break;
                    const uint32_t fq = smem_u32(&sm.q_full[qb]);
                    mbar_arrive_expect_tx(fq, QTILE);
                    tma_load_2d(smem_u32(sm.q + qb * QTILE), &tmQKV, fq, bl.it.h * kHeadDim,
                                bl.it.start + bl.it.qb * LQ);
                    ++nq;
                }
                // a {K, V} stage is free once the P V product of its block has completed
                const int st = bl.b % NKV;
                if (!mbar_wait(smem_u32(&sm.kv_empty[st]), ((bl.b / NKV) & 1) ^ 1, abort_flag)) break;
                const uint32_t fb = smem_u32(&sm.kv_full[st]);
                const uint32_t kd = smem_u32(sm.kv + st * 2 * KVTILE);
                mbar_arrive_expect_tx(fb, 2 * KVTILE);
                tma_load_2d(kd, &tmQKV64, fb, kHidden + bl.it.h * kHeadDim, bl.it.start + bl.j * KB);
                tma_load_2d(kd + KVTILE, &tmQKV64, fb, 2 * kHidden + bl.it.h * kHeadDim, bl.it.start + bl.j * KB);
                bl.advance(slot, total, seq_start, seq_len);
            }
            if (*abort_flag) {
                // loads still in flight complete before the CTA's shared memory goes away
                for (int n = nq > 2 ? nq - 2 : 0; n < nq; ++n)
                    mbar_wait_drain(smem_u32(&sm.q_full[n & 1]), (n >> 1) & 1);
                for (int b = bl.b > NKV ? bl.b - NKV : 0; b < bl.b; ++b)
                    mbar_wait_drain(smem_u32(&sm.kv_full[b % NKV]), (b / NKV) & 1);
            }
        }
    } else if (warp == 1 || warp == 11) {
        // -------------------------------------------------------- MMA issuer --
        // S of blocks b and b + 1 ahead; for each block in order: P V once the
        // softmax has written P, then S of block b + 2 into the same buffer.
        if (lane == 0) {
            const uint32_t idesc_s = idesc_bf16_f32(LQ, KB);
            const uint32_t idesc_o = idesc_bf16_f32(LQ, kHeadDim) | (1u << 16);  // B (= V) MN-major
            SlotBlocks gs, gp;  // next block for S, next block for P V
            gs.start(slot, total, seq_start, seq_len, items);
            gp.start(slot, total, seq_start, seq_len, items);
            bool ok = true;
            uint32_t oph = 0;
            auto issue_s = [&]() -> bool {
                const int qb = gs.n & 1;
                if (gs.j == 0) {
                    if (!mbar_wait(smem_u32(&sm.q_full[qb]), (gs.n >> 1) & 1, abort_flag)) return false;
                }
                const int st = gs.b % NKV;
                if (!mbar_wait(smem_u32(&sm.kv_full[st]), (gs.b / NKV) & 1, abort_flag)) return false;
                tc_fence_after();
                const uint32_t q = smem_u32(sm.q + qb * QTILE), k = smem_u32(sm.kv + st * 2 * KVTILE);
#pragma unroll
                for (int kk = 0; kk < kHeadDim / 16; ++kk)
                    umma_bf16(sbase + (gs.b & 1) * KB, sw128_kmajor_desc(q + kk * 32),
                              sw128_kmajor_desc(k + kk * 32), idesc_s, kk != 0);
                umma_commit(smem_u32(&sm.s_full[gs.b & 1]));
                if (gs.j == key_blocks(gs.it.L) - 1) umma_commit(smem_u32(&sm.q_empty[qb]));
                gs.advance(slot, total, seq_start, seq_len);
                return true;
            };
            for (int i = 0; i < 2 && gs.has && ok; ++i) ok = issue_s();
            bool sentinel = false;  // the commit that stands in for S after the slot's last
            while (ok && gp.has) {
                ok = mbar_wait(smem_u32(&sm.p_full[gp.b & 1]), (gp.b >> 1) & 1, abort_flag);
                if (!ok) break;
                if (gp.j == 0) {
                    // O holds the slot's previous item until its softmax warps have read it
                    ok = mbar_wait(smem_u32(sm.o_empty), oph ^ 1, abort_flag);
                    if (!ok) break;
                    oph ^= 1;
                }
                tc_fence_after();
                const int st = gp.b % NKV;
                const int Lj = min(KB, gp.it.L - gp.j * KB);
                const int ksteps = (Lj + 15) >> 4;
                const uint32_t vb = smem_u32(sm.kv + st * 2 * KVTILE + KVTILE);
                const uint32_t pcol = sbase + (gp.b & 1) * KB;
                for (int kk = 0; kk < ksteps; ++kk) {
                    // P: 16 keys = 8 packed TMEM columns; V: 16 keys = 16 rows of 128 B
                    umma_bf16_ts(sbase + 2 * KB, pcol + kk * 8, sw128_kmajor_desc(vb + kk * 2048), idesc_o,
                                 (gp.j | kk) != 0);
                }
                umma_commit(smem_u32(&sm.kv_empty[st]));  // K, V of the block consumed
                if (gp.j == key_blocks(gp.it.L) - 1) umma_commit(smem_u32(sm.o_full));
                gp.advance(slot, total, seq_start, seq_len);
                if (gs.has) {
                    ok = issue_s();  // into the score buffer P V has just read
                } else if (!sentinel) {
                    // no S of block gs.b: its phase of s_full completes once P V of block
                    // gs.b - 2 has, for a rescale on the slot's last block
                    umma_commit(smem_u32(&sm.s_full[gs.b & 1]));
                    sentinel = true;
                }
            }
            umma_commit(smem_u32(sm.drain));
            mbar_wait_drain(smem_u32(sm.drain), 0);
        }
    } else {
        // ------------------------------------------------------ softmax warps --
        const int quad = warp & 3;
        const int r = quad * 32 + lane;    // query row within the item
        const float sl2 = 0.125f * 1.4426950408889634f;
        const uint32_t lanes = (uint32_t)(quad * 32) << 16;
        const uint32_t orow = sbase + lanes + 2 * KB;
        uint32_t oph = 0;
        int b = 0;  // block counter of the slot (score buffer b & 1)
        SlotCursor cur;
        cur.start(slot, items);
        LongItem it;
        bool ok = true;
        while (ok && cur.next(slot, total, seq_start, seq_len, it)) {
            const int L = it.L, nkb = key_blocks(L);
            const bool live = it.qb * LQ + quad * 32 < L;  // some row of this warp is a real query
            float m_used = -INFINITY, l = 0.f;
            for (int j = 0; j < nkb; ++j, ++b) {
                const uint32_t srow = sbase + lanes + (b & 1) * KB;
                bool got = mbar_wait(smem_u32(&sm.s_full[b & 1]), (b >> 1) & 1, abort_flag);
                got = __all_sync(0xffffffffu, got);
                if (!got) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (live) {
                    const int Lj = min(KB, L - j * KB), nch = (Lj + 31) >> 5;
                    // the block's scores stay in registers for both passes
                    uint32_t v[2][32];
                    tmem_ld32(srow, v[0]);
                    if (nch > 1) tmem_ld32(srow + 32, v[1]);
                    tmem_ld_wait();
                    float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const int base = e * 32;
                        if (e >= nch) continue;
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
                    const float mb = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
                    // raise the running maximum only when this block would exceed it by
                    // more than 2^8; O and l follow.  O needs the slot's P V of block b - 1,
                    // which S of block b + 1 (or the commit after the slot's last S)
                    // follows in the issuer's order.  This warp has seen that barrier's
                    // previous phase (block b - 1), and its next needs this warp's arrival
                    // on P of block b + 1: the parity wait is exact.
                    const bool raise = j == 0 || (mb - m_used) * sl2 > kRescaleLog2;
                    const float m_new = raise ? mb : m_used;
                    if (j > 0 && __any_sync(0xffffffffu, raise)) {
                        bool d = mbar_wait(smem_u32(&sm.s_full[(b + 1) & 1]), ((b + 1) >> 1) & 1, abort_flag);
                        d = __all_sync(0xffffffffu, d);
                        if (!d) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const float sc = raise ? ex2_approx((m_used - m_new) * sl2) : 1.f;
#pragma unroll 1
                        for (int hcol = 0; hcol < kHeadDim; hcol += 32) {
                            uint32_t o[32];
                            tmem_ld32(orow + hcol, o);
                            tmem_ld_wait();
#pragma unroll
                            for (int t = 0; t < 32; ++t) o[t] = __float_as_uint(__uint_as_float(o[t]) * sc);
                            tmem_st32(orow + hcol, o);
                        }
                        l *= sc;
                    }
                    m_used = m_new;
                    // P_j = exp(scale * (s - m)) packed as bf16 pairs over the block's first columns
                    const uint64_t sl2x2 = f2_make(sl2, sl2), nms2 = f2_make(-m_used * sl2, -m_used * sl2);
                    uint64_t lsum[2] = {f2_make(0.f, 0.f), f2_make(0.f, 0.f)};
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        if (e >= nch) continue;
                        const bool full = e * 32 + 32 <= Lj;
                        uint32_t pk[16];
#pragma unroll
                        for (int t = 0; t < 16; ++t) {
                            const int k0 = e * 32 + 2 * t;
                            const float2 x = f2_split(f2_fma(f2_make_u(v[e][2 * t], v[e][2 * t + 1]), sl2x2, nms2));
                            float p0 = ex2_approx(x.x), p1 = ex2_approx(x.y);
                            if (!full) {
                                p0 = k0 < Lj ? p0 : 0.f;
                                p1 = k0 + 1 < Lj ? p1 : 0.f;
                            }
                            lsum[t & 1] = f2_add(lsum[t & 1], f2_make(p0, p1));
                            pk[t] = pack_bf16x2(p0, p1);
                        }
                        tmem_st16(srow + e * 16, pk);
                    }
                    const float2 ls = f2_split(f2_add(lsum[0], lsum[1]));
                    l += ls.x + ls.y;
                    tmem_st_wait();
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(&sm.p_full[b & 1]));
            }
            if (!ok) break;
            bool got = mbar_wait(smem_u32(sm.o_full), oph, abort_flag);
            got = __all_sync(0xffffffffu, got);
            if (!got) break;
            oph ^= 1;
            tc_fence_after();
            // O / l as bf16, read 32 columns at a time (packed as they arrive)
            uint32_t ob[32];
            if (live) {
                const float inv = 1.f / l;
#pragma unroll
                for (int hcol = 0; hcol < kHeadDim; hcol += 32) {
                    uint32_t o[32];
                    tmem_ld32(orow + hcol, o);
                    tmem_ld_wait();
#pragma unroll
                    for (int t = 0; t < 16; ++t)
                        ob[hcol / 2 + t] =
                            pack_bf16x2(__uint_as_float(o[2 * t]) * inv, __uint_as_float(o[2 * t + 1]) * inv);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_u32(sm.o_empty));
            const int qi = it.qb * LQ + r;
            if (live && qi < L) {
                uint4 *dst = reinterpret_cast<uint4 *>(ctx + (size_t)(it.start + qi) * kHidden + it.h * kHeadDim);
#pragma unroll
                for (int q = 0; q < 8; ++q) dst[q] = make_uint4(ob[4 * q], ob[4 * q + 1], ob[4 * q + 2], ob[4 * q + 3]);
            }
        }
    }

    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
    if (threadIdx.x == 0 && *abort_flag) set_status(status, kStatusTimeout);
}

}  // namespace

cudaError_t launch_attention_tc_long(const CUtensorMap &tmQKV, const CUtensorMap &tmQKV64, bf16 *ctx,
                                     const int *seq_start, const int *seq_len, int nseq, int *status, int num_sms,
                                     cudaStream_t s, bool trigger, unsigned long long wait_ns) {
    if (nseq <= 0) return cudaSuccess;
    static std::atomic<unsigned long long> configured{0};
    cudaError_t e = ensure_smem_attr(reinterpret_cast<const void *>(attn_tc_long_kernel), LA_SMEM, configured);
    if (e != cudaSuccess) return e;
    const int total = nseq * LKB * kHeads;
    const int grid = total < num_sms ? total : num_sms;
    return launch_pdl(attn_tc_long_kernel, dim3(grid), dim3(LA_THREADS), LA_SMEM, s, tmQKV, tmQKV64, ctx, seq_start,
                      seq_len, nseq, status, trigger ? 1 : 0, wait_ns);
}

}  // namespace albert
