// forward_small.cu -- the whole encoder forward for a batch of at most 128
// token rows in ONE persistent kernel (batch-1 latency).
//
// What it computes is the forward of the rest of the library ("ALBERT: How
// Kokoro's Phoneme Encoder Works", section "Inside One Real ALBERT Layer",
// steps 2-6 and the paragraph after them; "2. Cross-layer parameter sharing"
// for the one weight set reused by every execution):
//   X  = E W_in^T + b_in
//   n_exec x { QKV = X Wqkv^T + b;  C = per head softmax(Q K^T / 8 + mask) V;
//              X1 = LN(X + C Wo^T + bo);  X = LN(X1 + GELU(X1 W1^T + b1) W2^T + b2) }
//   Y  = X W_out^T + b_out  (or the hidden states when out_dim == 0).
// With at most 128 rows every GEMM is a single 128-row tile, so the per-layer
// kernels of the large-batch path leave most SMs idle and the forward is the
// sum of ~65 launch latencies.  Here a cooperative grid of G CTAs (one per SM,
// all resident) runs the forward as a sequence of phases separated by grid
// barriers; inside a phase each CTA takes jobs round robin:
//   in-proj     12 jobs: a 64-column tile of X (K = 128);
//   per execution:
//   Q|K|V       36 jobs: a 64-column tile of QKV (K = 768);
//   attention   one job per (sequence, head): S = Q K^T on tcgen05 into TMEM,
//               softmax by one thread per query row, P written back to TMEM
//               as bf16, O = P V (P from TMEM, V from shared memory);
//   out-proj    12 jobs: a 64-column tile of z1 = C Wo^T + bo + residual,
//               stored as z1 * gamma1 with the tile's per-row (mean, M2);
//   FFN         32 jobs, the FFN fused per hidden chunk: job j computes
//               H_j = GELU(LN1(z1) W1[64j..64j+63]^T + b1) (K = 768) into
//               TMEM, keeps it on chip (bf16, shared memory, in the layout
//               of a tensor-core A operand) and multiplies it straight into
//               its partial of the down projection, H_j W2[:, 64j..]^T (three
//               256-column products), stored as fp32 partial sums;
//   reduce      per (row, 64-column slice): z2 = sum_j partial_j + b2 + LN1(z1),
//               stored as z2 * gamma2 with its (mean, M2);
//   final       8 jobs: a 64-column tile of Y = LN2(z2) W_out^T + b_out,
//               scattered to the caller's rows (or LN2(z2) itself).
// The LayerNorms are applied where their input is consumed, as in the rest of
// the library: a consumer merges the twelve 64-column (mean, M2) partials of a
// row and uses LN(z) W^T = rstd (z gamma) W^T - rstd mu (W gamma) + W beta + b
// with W gamma and W beta + b folded once per weight set.  The partial sums of
// the down projection are reduced in a fixed order: the result does not
// depend on scheduling.
//
// Roles inside a CTA (192 threads): warp 0 lane 0 issues TMA loads into a
// 3-stage ring of 64 KB stages (a stage carries up to four 64-wide K blocks of
// both operands, so a 64-column tile with K = 768 and at most 64 rows has all
// of K in flight at once: the phases are bound by load latency, not
// bandwidth), warp 1 lane 0 allocates TMEM and issues tcgen05.mma, warps
// 2..5 (one per TMEM lane quadrant, one thread per tile row) run epilogues and
// the softmax; every warp takes rows of the reduce phase.  Every wait is
// bounded (mbarriers and the grid barrier alike); on expiry the kernel records
// ALBERT_ERR_TIMEOUT, every CTA leaves at its next grid barrier, and in-flight
// copies and products are drained before TMEM is freed.
#include "kernels.h"
#include "sm100_ptx.cuh"

namespace albert {
namespace {

constexpr int SB_THREADS = 192;
constexpr int SB_NS = 3;                      // ring stages
constexpr int SB_BOX = 64 * 64 * 2;           // one {64 cols, 64 rows} bf16 box, 128-byte swizzle: 8 KB
constexpr int SB_A_BYTES = 4 * SB_BOX;        // A: up to four 64-row K blocks (two of 128 rows)
constexpr int SB_B_BYTES = 4 * SB_BOX;        // B: up to four 64-row K blocks, or one of 256 rows
constexpr int SB_H_BYTES = 2 * SB_BOX;        // FFN hidden chunk, 128 rows x 64 bf16
constexpr int SB_STG_BYTES = 4 * 32 * 32 * 4; // FFN partial sums: a 32 x 32 fp32 staging tile per epilogue warp
constexpr int SB_SMEM = 1024 + SB_NS * (SB_A_BYTES + SB_B_BYTES) + SB_H_BYTES + SB_STG_BYTES + 128 * 4 + 512;
static_assert(SB_SMEM <= 232448, "shared memory per CTA");
constexpr int SB_PARTS = kSmallParts;         // 64-column statistics slices of a 768-wide row
constexpr int SB_CHUNKS = kFfn / 64;          // FFN hidden chunks
constexpr uint32_t SB_TM_O = 64;              // attention: O's columns within the item's TMEM columns

struct SbSmem {
    uint8_t *a, *b, *h, *stg;
    float *inv_sum;                           // [128] attention: 1 / row sum
    uint64_t *full, *empty;                   // [SB_NS]
    uint64_t *acc_full, *acc_empty, *h_ready, *drain;
    uint32_t *tmem_slot;
    volatile int *abort_flag;
    int *misc;                                // [0] rows, [1] status at entry
};

__device__ __forceinline__ SbSmem sb_carve(uint8_t *raw) {
    SbSmem s;
    uint8_t *p = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
    s.a = p;
    s.b = p + SB_NS * SB_A_BYTES;
    s.h = s.b + SB_NS * SB_B_BYTES;
    s.stg = s.h + SB_H_BYTES;
    s.inv_sum = reinterpret_cast<float *>(s.stg + SB_STG_BYTES);
    uint64_t *bars = reinterpret_cast<uint64_t *>(s.inv_sum + 128);
    s.full = bars;
    s.empty = bars + SB_NS;
    s.acc_full = bars + 2 * SB_NS;
    s.acc_empty = s.acc_full + 1;
    s.h_ready = s.acc_full + 2;
    s.drain = s.acc_full + 3;
    uint32_t *u = reinterpret_cast<uint32_t *>(s.acc_full + 4);
    s.tmem_slot = u;
    s.abort_flag = reinterpret_cast<volatile int *>(u + 1);
    s.misc = reinterpret_cast<int *>(u + 2);
    return s;
}

__device__ __forceinline__ void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

// (mean, rstd) of a 768-wide row from its twelve 64-column (mean, M2) partials
// (Chan's merge of equal-size groups).
__device__ __forceinline__ void merge_parts(const float2 *q, float eps, float &mu, float &rstd) {
    float2 v[SB_PARTS];
#pragma unroll
    for (int i = 0; i < SB_PARTS; ++i) v[i] = q[i];
    float m = 0.f;
#pragma unroll
    for (int i = 0; i < SB_PARTS; ++i) m += v[i].x;
    m *= 1.0f / SB_PARTS;
    float m2 = 0.f;
#pragma unroll
    for (int i = 0; i < SB_PARTS; ++i) {
        const float d = v[i].x - m;
        m2 += v[i].y + 64.0f * d * d;
    }
    mu = m;
    rstd = rsqrtf(m2 * (1.0f / kHidden) + eps);
}

// Grid barrier of the cooperative launch: every thread of every CTA calls it.
// The counter only grows (zeroed before the launch); barrier e completes when
// it reaches e * gridDim.x.  Returns false when the kernel is failing (this or
// another CTA saw a wait run out): the CTA then leaves.
__device__ bool grid_sync(int *ctr, int &epoch, int *status, volatile int *abort) {
    fence_proxy_async_global();  // this thread's stores, before other CTAs' TMA reads of them
    __syncthreads();
    if (threadIdx.x == 0) {
        ++epoch;
        if (*abort) set_status(status, kStatusTimeout);
        __threadfence();
        atomicAdd(ctr, 1);
        const int target = epoch * (int)gridDim.x;
        unsigned long long t0 = 0;
        unsigned polls = 0;
        while (!*abort && ld_acquire_gpu(ctr) < target) {
            if ((++polls & 63) == 0) {
                if (*reinterpret_cast<volatile int *>(status) != 0) { *abort = 1; break; }
                const unsigned long long now = globaltimer_ns();
                if (t0 == 0) t0 = now;
                else if (now - t0 > wait_limit()) {
                    *abort = 1;
                    set_status(status, kStatusTimeout);
                }
            }
        }
        __threadfence();
        fence_proxy_async_global();
    }
    __syncthreads();
    return !*abort;
}

// ---------------------------------------------------------------- phases ----
enum SbPhase : int { kPhIn = 0, kPhQKV, kPhAttn, kPhOut, kPhFfn, kPhReduce, kPhFinal };

__device__ __forceinline__ int phase_jobs(int ph, const SmallFwdArgs &p) {
    switch (ph) {
        case kPhIn: return kHidden / 64;
        case kPhQKV: return kQKV / 64;
        case kPhAttn: return p.nseq * kHeads;
        case kPhOut: return kHidden / 64;
        case kPhFfn: return SB_CHUNKS;
        case kPhFinal: return p.out_dim > 0 ? p.out_dim / 64 : 0;
    }
    return 0;
}

// Loads of one job, in the order the MMA issuer consumes them.  Each load step
// fills one ring stage with nk consecutive 64-wide K blocks; K block j holds
// a_boxes boxes of 64 rows of A at j * a_boxes * 8 KB and b_boxes boxes of 64
// rows of B at j * b_boxes * 8 KB.  The FFN's second products load B only.
struct LoadStep {
    const CUtensorMap *ta, *tb;
    int a_boxes, b_boxes, nk;
    int ax, ay, bx, by;       // coordinates of the first boxes (x = column, y = row)
};

__global__ void __launch_bounds__(SB_THREADS, 1) fwd_small_kernel(const __grid_constant__ SmallFwdArgs p) {
    extern __shared__ uint8_t smem_raw[];
    SbSmem sm = sb_carve(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        *sm.abort_flag = 0;
        wait_limit_init(p.wait_ns);
        for (int i = 0; i < SB_NS; ++i) {
            mbar_init(smem_u32(&sm.full[i]), 1);
            mbar_init(smem_u32(&sm.empty[i]), 1);
        }
        mbar_init(smem_u32(sm.acc_full), 1);
        mbar_init(smem_u32(sm.acc_empty), 4);  // one arrive per epilogue warp
        mbar_init(smem_u32(sm.h_ready), 4);
        mbar_init(smem_u32(sm.drain), 1);
        fence_mbar_init();
        sm.misc[0] = *reinterpret_cast<const volatile int *>(p.n_rows);
        sm.misc[1] = *reinterpret_cast<const volatile int *>(p.status);
    }
    if (warp == 0 && lane == 0) {
        prefetch_tmap(&p.tmE);
        prefetch_tmap(&p.tmX);
        prefetch_tmap(&p.tmC);
        prefetch_tmap(&p.tmX1);
        prefetch_tmap(&p.tmZ);
        prefetch_tmap(&p.tmQKV);
        prefetch_tmap(&p.tmQKV64);
        prefetch_tmap(&p.tmWin);
        prefetch_tmap(&p.tmWqkv);
        prefetch_tmap(&p.tmWo);
        prefetch_tmap(&p.tmW1);
        prefetch_tmap(&p.tmW2);
        prefetch_tmap(&p.tmWout);
        prefetch_tmap(&p.tmPart);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(sm.tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *sm.tmem_slot;
    const int M = sm.misc[0];
    // an earlier kernel of this forward failed (or the row count is out of range): nothing to do
    const bool skip = sm.misc[1] != 0 || M < 1 || M > 128;
    const int a_boxes = M > 64 ? 2 : 1;
    const int kb_step = M > 64 ? 2 : 4;  // 64-wide K blocks per ring stage in the GEMM phases
    const int n_phases = 1 + 5 * p.n_exec + 1;

    int epoch = 0;
    // ring and accumulator progress, advanced identically by the roles that use them
    uint32_t ring = 0;   // load steps issued (producer) / consumed (MMA issuer)
    uint32_t units = 0;  // accumulations committed (MMA issuer) / read (epilogue)
    uint32_t hcnt = 0;   // FFN hidden chunks handed over through shared memory
    bool ok = !skip;

    for (int phi = 0; phi < n_phases && ok; ++phi) {
        const int ph = phi == 0 ? kPhIn : phi == n_phases - 1 ? kPhFinal : 1 + (phi - 1) % 5;
        const int l = phi == 0 ? -1 : (phi - 1) / 5;  // execution of the shared layer
        const int njobs = phase_jobs(ph, p);

        if (ph == kPhReduce || (ph == kPhFinal && p.out_dim == 0)) {
            // ------------------------------------------------ row phases (all warps) --
            // item = (row, 64-column slice); one warp per item, two columns per lane
            const int items = M * SB_PARTS;
            for (int it = blockIdx.x * (SB_THREADS / 32) + warp; it < items; it += gridDim.x * (SB_THREADS / 32)) {
                const int r = it / SB_PARTS, s = it % SB_PARTS;
                const int c = s * 64 + 2 * lane;
                if (ph == kPhReduce) {
                    // z2 = sum of the FFN partials + (b2 + beta1) + rstd1 * x1 - rstd1 * mu1 * gamma1
                    // every partial's load is issued before the first add (one round trip)
                    float2 pv[SB_CHUNKS];
#pragma unroll
                    for (int j = 0; j < SB_CHUNKS; ++j)
                        pv[j] = *reinterpret_cast<const float2 *>(p.part + ((size_t)j * 128 + r) * kHidden + c);
                    float ax = 0.f, ay = 0.f;
#pragma unroll
                    for (int j = 0; j < SB_CHUNKS; ++j) {
                        ax += pv[j].x;
                        ay += pv[j].y;
                    }
                    float mu1, rstd1;
                    merge_parts(p.st1 + (size_t)r * SB_PARTS, p.eps, mu1, rstd1);
                    const float2 x1 = unpack_bf16x2(*reinterpret_cast<const uint32_t *>(p.X1 + (size_t)r * kHidden + c));
                    const float2 g1 = *reinterpret_cast<const float2 *>(p.ln1_g + c);
                    const float2 bb = *reinterpret_cast<const float2 *>(p.bias_21 + c);
                    const float z0 = ax + bb.x + rstd1 * x1.x - rstd1 * mu1 * g1.x;
                    const float z1 = ay + bb.y + rstd1 * x1.y - rstd1 * mu1 * g1.y;
                    // exact (mean, M2) of the slice: two passes over the warp's 64 values
                    float sum = z0 + z1;
#pragma unroll
                    for (int o = 16; o; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
                    const float mean = sum * (1.0f / 64);
                    float q = (z0 - mean) * (z0 - mean) + (z1 - mean) * (z1 - mean);
#pragma unroll
                    for (int o = 16; o; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
                    const float2 g2 = *reinterpret_cast<const float2 *>(p.ln2_g + c);
                    *reinterpret_cast<uint32_t *>(p.Z + (size_t)r * kHidden + c) = pack_bf16x2(z0 * g2.x, z1 * g2.y);
                    if (lane == 0) p.st2[(size_t)r * SB_PARTS + s] = make_float2(mean, q);
                } else {
                    // hidden-state output: LN2(z2) = rstd2 * zg - rstd2 * mu2 * gamma2 + beta2
                    const int dst = p.row_dst[r];
                    if (dst < 0) continue;
                    if (dst >= p.out_rows) { set_status(p.status, kStatusShape); continue; }
                    float mu2, rstd2;
                    merge_parts(p.st2 + (size_t)r * SB_PARTS, p.eps, mu2, rstd2);
                    const float2 zg = unpack_bf16x2(*reinterpret_cast<const uint32_t *>(p.Z + (size_t)r * kHidden + c));
                    const float2 g2 = *reinterpret_cast<const float2 *>(p.ln2_g + c);
                    const float2 b2 = *reinterpret_cast<const float2 *>(p.ln2_b + c);
                    *reinterpret_cast<uint32_t *>(p.out + (size_t)dst * kHidden + c) =
                        pack_bf16x2(rstd2 * zg.x - rstd2 * mu2 * g2.x + b2.x, rstd2 * zg.y - rstd2 * mu2 * g2.y + b2.y);
                }
            }
        } else if (warp == 0) {
            // ------------------------------------------------------------ producer --
            if (lane == 0) {
                const uint64_t keep = policy_evict_last();  // weights: read by every execution
                for (int job = p.withhold_loads ? njobs : blockIdx.x; job < njobs && ok; job += gridDim.x) {
                    LoadStep st[12];  // at most 6 + 3 (FFN)
                    int ns = 0;
                    if (ph == kPhIn) {
                        st[ns++] = {&p.tmE, &p.tmWin, a_boxes, 1, kEmb / 64, 0, 0, 0, job * 64};
                    } else if (ph == kPhQKV || ph == kPhOut || ph == kPhFinal || ph == kPhFfn) {
                        const CUtensorMap *ta = ph == kPhOut ? &p.tmC : ph == kPhFfn ? &p.tmX1
                                                : (ph == kPhQKV && l == 0) ? &p.tmX : &p.tmZ;
                        const CUtensorMap *tb = ph == kPhQKV ? &p.tmWqkv : ph == kPhOut ? &p.tmWo
                                                : ph == kPhFfn ? &p.tmW1 : &p.tmWout;
                        // every CTA of the phase reads the same A rows: each starts at another
                        // stage of K, so that they do not all ask L2 for the same lines at once
                        // (the sum over K is then taken in a rotated, fixed order per job)
                        const int nsteps = (kHidden / 64) / kb_step;
                        for (int i = 0; i < nsteps; ++i) {
                            const int kb = ((i + job) % nsteps) * kb_step;
                            st[ns++] = {ta, tb, a_boxes, 1, kb_step, kb * 64, 0, kb * 64, job * 64};
                        }
                        if (ph == kPhFfn)
                            for (int nb = 0; nb < 3; ++nb)
                                st[ns++] = {nullptr, &p.tmW2, 0, 4, 1, 0, 0, job * 64, nb * 256};
                    } else {  // attention: Q and K of (sequence, head), then V
                        const int b = job / kHeads, h = job % kHeads;
                        const int L = __ldg(p.seq_len + b), start = __ldg(p.seq_start + b);
                        const CUtensorMap *tq = L <= 64 ? &p.tmQKV64 : &p.tmQKV;
                        st[ns++] = {tq, tq, 1, 1, 1, h * kHeadDim, start, kHidden + h * kHeadDim, start};
                        st[ns++] = {nullptr, tq, 0, 1, 1, 0, 0, 2 * kHidden + h * kHeadDim, start};
                    }
                    for (int i = 0; i < ns && ok; ++i, ++ring) {
                        const int s = ring % SB_NS;
                        if (!mbar_wait(smem_u32(&sm.empty[s]), ((ring / SB_NS) & 1) ^ 1, sm.abort_flag)) {
                            ok = false;
                            break;
                        }
                        const LoadStep &d = st[i];
                        const bool attn = ph == kPhAttn;
                        // attention boxes are 128 rows unless the sequence fits in 64
                        const uint32_t box_bytes = attn && d.tb == &p.tmQKV ? 2 * SB_BOX : SB_BOX;
                        const uint32_t fb = smem_u32(&sm.full[s]);
                        mbar_arrive_expect_tx(fb, box_bytes * (uint32_t)(d.nk * (d.a_boxes + d.b_boxes)));
                        const uint32_t a_dst = smem_u32(sm.a + s * SB_A_BYTES), b_dst = smem_u32(sm.b + s * SB_B_BYTES);
                        if (attn) {
                            if (d.a_boxes) tma_load_2d(a_dst, d.ta, fb, d.ax, d.ay);
                            tma_load_2d(b_dst, d.tb, fb, d.bx, d.by);
                        } else {
                            for (int j = 0; j < d.nk; ++j) {
                                for (int q = 0; q < d.a_boxes; ++q)
                                    tma_load_2d(a_dst + (j * d.a_boxes + q) * SB_BOX, d.ta, fb, d.ax + 64 * j, d.ay + 64 * q);
                                for (int q = 0; q < d.b_boxes; ++q)
                                    tma_load_2d_hint(b_dst + (j * d.b_boxes + q) * SB_BOX, d.tb, fb, d.bx + 64 * j,
                                                     d.by + 64 * q, keep);
                            }
                        }
                    }
                }
            }
        } else if (warp == 1) {
            // ---------------------------------------------------------- MMA issuer --
            if (lane == 0) {
                auto wait_stage = [&](uint32_t &s) -> bool {
                    s = ring % SB_NS;
                    if (!mbar_wait(smem_u32(&sm.full[s]), (ring / SB_NS) & 1, sm.abort_flag)) return false;
                    tc_fence_after();
                    return true;
                };
                // the accumulator columns are free once the epilogue has read the previous unit
                auto wait_acc_free = [&]() -> bool {
                    if (!mbar_wait(smem_u32(sm.acc_empty), (units & 1) ^ 1, sm.abort_flag)) return false;
                    tc_fence_after();
                    return true;
                };
                auto finish_unit = [&]() {
                    umma_commit(smem_u32(sm.acc_full));
                    ++units;
                };
                for (int job = blockIdx.x; job < njobs && ok; job += gridDim.x) {
                    if (ph == kPhAttn) {
                        const int L = __ldg(p.seq_len + job / kHeads);
                        uint32_t s;
                        if (!wait_acc_free() || !wait_stage(s)) { ok = false; break; }
                        const uint32_t q = smem_u32(sm.a + s * SB_A_BYTES), k = smem_u32(sm.b + s * SB_B_BYTES);
                        const uint32_t idesc = idesc_bf16_f32(128, L <= 64 ? 64 : 128);
#pragma unroll
                        for (int kk = 0; kk < kHeadDim / 16; ++kk)
                            umma_bf16(tmem_base, sw128_kmajor_desc(q + kk * 32), sw128_kmajor_desc(k + kk * 32), idesc,
                                      kk != 0);
                        umma_commit(smem_u32(&sm.empty[s]));
                        ++ring;
                        finish_unit();
                        // O = P V once the softmax has written P over the scores
                        if (!wait_acc_free() || !wait_stage(s)) { ok = false; break; }
                        const uint32_t vbase = smem_u32(sm.b + s * SB_B_BYTES);
                        const uint32_t idesc_o = idesc_bf16_f32(128, kHeadDim) | (1u << 16);  // V MN-major
                        for (int kk = 0; kk < (L + 15) / 16; ++kk)
                            umma_bf16_ts(tmem_base + SB_TM_O, tmem_base + kk * 8, sw128_kmajor_desc(vbase + kk * 2048),
                                         idesc_o, kk != 0);
                        umma_commit(smem_u32(&sm.empty[s]));
                        ++ring;
                        finish_unit();
                        continue;
                    }
                    // one stage per kb_step K blocks (the in-projection's two in one stage)
                    const int nsteps = ph == kPhIn ? 1 : (kHidden / 64) / kb_step;
                    const int nk = ph == kPhIn ? kEmb / 64 : kb_step;
                    if (!wait_acc_free()) { ok = false; break; }
                    const uint32_t idesc = idesc_bf16_f32(128, 64);
                    for (int stp = 0; stp < nsteps && ok; ++stp) {
                        uint32_t s;
                        if (!wait_stage(s)) { ok = false; break; }
                        const uint32_t a0 = smem_u32(sm.a + s * SB_A_BYTES), b0 = smem_u32(sm.b + s * SB_B_BYTES);
                        for (int j = 0; j < nk; ++j) {
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                umma_bf16(tmem_base, sw128_kmajor_desc(a0 + j * a_boxes * SB_BOX + kk * 32),
                                          sw128_kmajor_desc(b0 + j * SB_BOX + kk * 32), idesc, (stp | j | kk) != 0);
                        }
                        umma_commit(smem_u32(&sm.empty[s]));
                        ++ring;
                    }
                    if (!ok) break;
                    finish_unit();
                    if (ph == kPhFfn) {
                        // the down projection of this hidden chunk: three 256-column products
                        // with H (bf16, shared memory) as the A operand, K = 64
                        if (!mbar_wait(smem_u32(sm.h_ready), hcnt & 1, sm.abort_flag)) { ok = false; break; }
                        ++hcnt;
                        const uint32_t hb = smem_u32(sm.h);
                        const uint32_t idesc2 = idesc_bf16_f32(128, 256);
                        for (int nb = 0; nb < 3; ++nb) {
                            uint32_t s;
                            if (!wait_acc_free() || !wait_stage(s)) { ok = false; break; }
                            const uint32_t b0 = smem_u32(sm.b + s * SB_B_BYTES);
#pragma unroll
                            for (int kk = 0; kk < 4; ++kk)
                                umma_bf16(tmem_base, sw128_kmajor_desc(hb + kk * 32), sw128_kmajor_desc(b0 + kk * 32),
                                          idesc2, kk != 0);
                            umma_commit(smem_u32(&sm.empty[s]));
                            ++ring;
                            finish_unit();
                        }
                    }
                }
            }
        } else {
            // ------------------------------------------------ epilogue warps 2..5 --
            const int quad = warp & 3;
            const int r = quad * 32 + lane;  // tile row
            const uint32_t trow = tmem_base + ((uint32_t)(quad * 32) << 16);
            auto wait_unit = [&]() -> bool {
                bool got = mbar_wait(smem_u32(sm.acc_full), units & 1, sm.abort_flag);
                got = __all_sync(0xffffffffu, got);
                if (got) tc_fence_after();
                return got;
            };
            auto release_unit = [&]() {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_u32(sm.acc_empty));
                ++units;
            };
            for (int job = blockIdx.x; job < njobs && ok; job += gridDim.x) {
                if (ph == kPhAttn) {
                    const int b = job / kHeads, h = job % kHeads;
                    const int L = __ldg(p.seq_len + b), start = __ldg(p.seq_start + b);
                    const bool live = quad * 32 < L;
                    if (!wait_unit()) { ok = false; break; }
                    if (live) {
                        // scores of this query row over the valid keys: max, then
                        // exponentials packed as bf16 pairs over the columns already read
                        // (all four 32-column chunks are read, so that the register
                        // arrays are indexed statically; keys >= L are masked)
                        const float sl2 = 0.125f * 1.4426950408889634f;
                        const int nch = (L + 31) >> 5;
                        uint32_t v[4][32];
#pragma unroll
                        for (int c = 0; c < 4; ++c) tmem_ld32(trow + c * 32, v[c]);
                        tmem_ld_wait();
                        float m = -INFINITY;
#pragma unroll
                        for (int c = 0; c < 4; ++c)
#pragma unroll
                            for (int j = 0; j < 32; ++j)
                                if (c * 32 + j < L) m = fmaxf(m, __uint_as_float(v[c][j]));
                        float sum = 0.f;
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            if (c >= nch) break;
                            uint32_t pk[16];
#pragma unroll
                            for (int j = 0; j < 16; ++j) {
                                const int k0 = c * 32 + 2 * j;
                                float p0 = ex2_approx((__uint_as_float(v[c][2 * j]) - m) * sl2);
                                float p1 = ex2_approx((__uint_as_float(v[c][2 * j + 1]) - m) * sl2);
                                p0 = k0 < L ? p0 : 0.f;
                                p1 = k0 + 1 < L ? p1 : 0.f;
                                sum += p0 + p1;
                                pk[j] = pack_bf16x2(p0, p1);
                            }
                            tmem_st16(trow + c * 16, pk);
                        }
                        sm.inv_sum[r] = 1.f / sum;
                        tmem_st_wait();
                    }
                    release_unit();  // P is in TMEM: the O product may run
                    if (!wait_unit()) { ok = false; break; }
                    uint32_t o[2][32];
                    if (live) {
                        tmem_ld32(trow + SB_TM_O, o[0]);
                        tmem_ld32(trow + SB_TM_O + 32, o[1]);
                        tmem_ld_wait();
                    }
                    release_unit();
                    if (r < L) {
                        const float inv = sm.inv_sum[r];
                        uint4 *dst = reinterpret_cast<uint4 *>(p.C + (size_t)(start + r) * kHidden + h * kHeadDim);
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const uint32_t *x = o[q >> 2] + (q & 3) * 8;
                            dst[q] = make_uint4(pack_bf16x2(__uint_as_float(x[0]) * inv, __uint_as_float(x[1]) * inv),
                                                pack_bf16x2(__uint_as_float(x[2]) * inv, __uint_as_float(x[3]) * inv),
                                                pack_bf16x2(__uint_as_float(x[4]) * inv, __uint_as_float(x[5]) * inv),
                                                pack_bf16x2(__uint_as_float(x[6]) * inv, __uint_as_float(x[7]) * inv));
                        }
                    }
                    continue;
                }
                // 64-column tile of a GEMM: this thread's row, columns n0..n0+63
                const int n0 = job * 64;
                uint32_t v[2][32];
                if (!wait_unit()) { ok = false; break; }
                tmem_ld32(trow, v[0]);
                tmem_ld32(trow + 32, v[1]);
                tmem_ld_wait();
                release_unit();
                const bool row_ok = r < M;
                float y[64];
#pragma unroll
                for (int j = 0; j < 64; ++j) y[j] = __uint_as_float(v[j >> 5][j & 31]);
                // LayerNorm of the A operand (z * gamma held in A, statistics per row)
                const float2 *in_st = nullptr;
                const float *fs = nullptr, *bias = nullptr;
                if (ph == kPhIn) bias = p.b_in;
                else if (ph == kPhQKV) {
                    bias = l == 0 ? p.bqkv0 : p.bqkv;
                    if (l > 0) { in_st = p.st2; fs = p.s_qkv; }
                } else if (ph == kPhOut) bias = l == 0 ? p.bo0 : p.bo;
                else if (ph == kPhFfn) { bias = p.c_1; in_st = p.st1; fs = p.s_1; }
                else { bias = p.c_out; in_st = p.st2; fs = p.s_out; }  // final
                float mu = 0.f, rstd = 1.f;
                if (in_st && row_ok) merge_parts(in_st + (size_t)r * SB_PARTS, p.eps, mu, rstd);
#pragma unroll
                for (int j = 0; j < 64; j += 4) {
                    const float4 bb = __ldg(reinterpret_cast<const float4 *>(bias + n0 + j));
                    if (in_st) {
                        const float4 ss = __ldg(reinterpret_cast<const float4 *>(fs + n0 + j));
                        y[j] = rstd * y[j] - rstd * mu * ss.x + bb.x;
                        y[j + 1] = rstd * y[j + 1] - rstd * mu * ss.y + bb.y;
                        y[j + 2] = rstd * y[j + 2] - rstd * mu * ss.z + bb.z;
                        y[j + 3] = rstd * y[j + 3] - rstd * mu * ss.w + bb.w;
                    } else {
                        y[j] += bb.x;
                        y[j + 1] += bb.y;
                        y[j + 2] += bb.z;
                        y[j + 3] += bb.w;
                    }
                }
                if (ph == kPhFfn) {
                    // H chunk = GELU(...) as bf16 into shared memory, the layout TMA
                    // would give a 128 x 64 tile with the 128-byte swizzle (row r: 128 B,
                    // 16-byte chunk q at position q ^ (r & 7)), for the down products
#pragma unroll
                    for (int j = 0; j < 64; ++j) y[j] = gelu_tanh_fast(y[j]);
                    // the previous chunk's down products have read H (its last unit was waited for)
                    const uint32_t hrow = smem_u32(sm.h) + r * 128;
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        const uint32_t w0 = pack_bf16x2(y[8 * q], y[8 * q + 1]), w1 = pack_bf16x2(y[8 * q + 2], y[8 * q + 3]);
                        const uint32_t w2 = pack_bf16x2(y[8 * q + 4], y[8 * q + 5]), w3 = pack_bf16x2(y[8 * q + 6], y[8 * q + 7]);
                        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(hrow + ((q ^ (r & 7)) << 4)),
                                     "r"(w0), "r"(w1), "r"(w2), "r"(w3)
                                     : "memory");
                    }
                    fence_proxy_async_smem();  // generic writes, read by the tensor core (async proxy)
                    __syncwarp();
                    if (lane == 0) mbar_arrive(smem_u32(sm.h_ready));
                    // the three down products: fp32 partial sums of this chunk, each warp's
                    // 32 x 32 tiles staged in shared memory (128-byte swizzle) and stored
                    // by TMA (rows of the partial buffer are 3 KB apart: one row per lane
                    // would scatter every store)
                    const bool any_row = quad * 32 < M;
                    const uint32_t stg = smem_u32(sm.stg) + (uint32_t)quad * 4096u;
                    for (int nb = 0; nb < 3; ++nb) {
                        if (!wait_unit()) { ok = false; break; }
                        for (int c = 0; c < 8; ++c) {
                            uint32_t t[32];
                            if (any_row) {
                                tmem_ld32(trow + c * 32, t);
                                tmem_ld_wait();
                                if (lane == 0) bulk_wait_read0();  // the previous tile has left the staging
                                __syncwarp();
#pragma unroll
                                for (int q = 0; q < 8; ++q)
                                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                                                 ::"r"(stg + lane * 128 + ((q ^ (lane & 7)) << 4)), "r"(t[4 * q]),
                                                 "r"(t[4 * q + 1]), "r"(t[4 * q + 2]), "r"(t[4 * q + 3])
                                                 : "memory");
                                fence_proxy_async_smem();
                                __syncwarp();
                                if (lane == 0) {
                                    tma_store_2d(&p.tmPart, stg, nb * 256 + c * 32, job * 128 + quad * 32);
                                    bulk_commit();
                                }
                            }
                        }
                        release_unit();
                    }
                    // the partial sums are in global memory before the phase's barrier
                    if (lane == 0) bulk_wait0();
                    __syncwarp();
                    if (!ok) break;
                    continue;
                }
                if (!row_ok) continue;
                if (ph == kPhOut) {
                    // z1 = acc + bias + residual (the layer input: X plain in the first
                    // execution, else LN2(z2) rebuilt from z2 * gamma2 and its statistics)
                    const bf16 *res = (l == 0 ? p.X : p.Z) + (size_t)r * kHidden + n0;
                    float rmu = 0.f, rrstd = 1.f;
                    if (l > 0) merge_parts(p.st2 + (size_t)r * SB_PARTS, p.eps, rmu, rrstd);
#pragma unroll
                    for (int j = 0; j < 64; j += 8) {
                        const uint4 w = *reinterpret_cast<const uint4 *>(res + j);
                        const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 x = unpack_bf16x2(wv[e]);
                            if (l == 0) {
                                y[j + 2 * e] += x.x;
                                y[j + 2 * e + 1] += x.y;
                            } else {
                                const float g0 = __ldg(p.ln2_g + n0 + j + 2 * e), g1 = __ldg(p.ln2_g + n0 + j + 2 * e + 1);
                                y[j + 2 * e] += rrstd * x.x - rrstd * rmu * g0;
                                y[j + 2 * e + 1] += rrstd * x.y - rrstd * rmu * g1;
                            }
                        }
                    }
                    float sum = 0.f;
#pragma unroll
                    for (int j = 0; j < 64; ++j) sum += y[j];
                    const float mean = sum * (1.0f / 64);
                    float m2 = 0.f;
#pragma unroll
                    for (int j = 0; j < 64; ++j) m2 += (y[j] - mean) * (y[j] - mean);
                    p.st1[(size_t)r * SB_PARTS + job] = make_float2(mean, m2);
#pragma unroll
                    for (int j = 0; j < 64; ++j) y[j] *= __ldg(p.ln1_g + n0 + j);
                }
                bf16 *dst;
                if (ph == kPhFinal) {
                    const int d = p.row_dst[r];
                    if (d < 0) continue;
                    if (d >= p.out_rows) { set_status(p.status, kStatusShape); continue; }
                    dst = p.out + (size_t)d * p.out_dim + n0;
                } else {
                    bf16 *base = ph == kPhIn ? p.X : ph == kPhQKV ? p.QKV : p.X1;
                    const int ld = ph == kPhQKV ? kQKV : kHidden;
                    dst = base + (size_t)r * ld + n0;
                }
                uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    d4[q] = make_uint4(pack_bf16x2(y[8 * q], y[8 * q + 1]), pack_bf16x2(y[8 * q + 2], y[8 * q + 3]),
                                       pack_bf16x2(y[8 * q + 4], y[8 * q + 5]), pack_bf16x2(y[8 * q + 6], y[8 * q + 7]));
            }
        }
        // a failed wait in any role stops the CTA at this barrier; the others
        // see the status word and leave at theirs
        if (!ok) *sm.abort_flag = 1;
        if (phi + 1 < n_phases) ok = grid_sync(p.bar, epoch, p.status, sm.abort_flag) && ok;
    }

    // ----------------------------------------------------------------- teardown --
    __syncthreads();
    if (*sm.abort_flag) {
        if (warp == 0 && lane == 0) {
            // loads still in flight land before the CTA's shared memory goes away
            for (int i = 0; i < SB_NS && (uint32_t)i < ring; ++i) {
                const uint32_t c = ring - 1 - i;
                mbar_wait_drain(smem_u32(&sm.full[c % SB_NS]), (c / SB_NS) & 1);
            }
        }
        if (warp == 1 && lane == 0) {
            umma_commit(smem_u32(sm.drain));
            mbar_wait_drain(smem_u32(sm.drain), 0);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
    if (threadIdx.x == 0 && *sm.abort_flag) set_status(p.status, kStatusTimeout);
}

}  // namespace

int small_forward_grid(int num_sms) {
    // the widest GEMM phase has 36 jobs; more CTAs only make the grid barrier slower
    return num_sms < 36 ? num_sms : 36;
}

cudaError_t launch_forward_small(const SmallFwdArgs &a, int grid, cudaStream_t s) {
    static std::atomic<unsigned long long> configured{0};
    cudaError_t e = ensure_smem_attr(reinterpret_cast<const void *>(fwd_small_kernel), SB_SMEM, configured);
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(a.bar, 0, sizeof(int), s);
    if (e != cudaSuccess) return e;
    // cooperative: every CTA is resident at once, which the grid barriers need
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(SB_THREADS);
    cfg.dynamicSmemBytes = SB_SMEM;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, fwd_small_kernel, a);
}

}  // namespace albert
