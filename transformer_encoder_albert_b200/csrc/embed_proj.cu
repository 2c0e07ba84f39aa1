// embed_proj.cu -- the factorized embedding and the input projection in one
// kernel (bf16 activations, batches beyond the small-batch kernel's 128 rows).
//
// "ALBERT: How Kokoro's Phoneme Encoder Works", section "Inside One Real ALBERT
// Layer", steps 1-2 (and "1. Factorized embedding" for the sizes):
//     E = LN_128(word[id] + pos[t] + type[0]; gamma, beta, eps)
//     X = E W_in^T + b_in                         (128 -> 768)
// Each CTA takes 128-row blocks of the packed rows.  Its eight warps gather and
// normalize the block's embedding rows (sixteen rows per warp, four at a time,
// four features per lane) straight into shared memory, in the 128-byte-swizzled
// K-major layout the tensor core reads, so E never goes to global memory.  One thread then issues the products against W_in, which
// every CTA loads once by TMA (192 KB, resident for all of its blocks) before
// waiting on the previous kernel: two passes of M=128 x N=256 x K=128 tcgen05
// products into tensor memory (output columns 0..511, then 512..767), each read
// back by all eight warps (two per TMEM lane quadrant), plus b_in, and stored
// as bf16 rows of X.  Rows past the batch's end are zero in E and never stored.
// Invalid ids are reported as in the standalone kernel (ALBERT_ERR_ID for a
// valid slot); the later kernels of the forward then do nothing.  Every wait is
// bounded (%globaltimer); on expiry the kernel records ALBERT_ERR_TIMEOUT.
#include "kernels.h"
#include "sm100_ptx.cuh"

namespace albert {
namespace {

constexpr int EP_THREADS = 256;
constexpr int EP_BOX = 128 * 128;                 // {64 cols, 128 rows} bf16 box: 16 KB
constexpr int EP_WBOXES = 2 * (kHidden / 128);    // two 64-column K blocks x six 128-row blocks of W_in
constexpr int EP_W_BYTES = EP_WBOXES * EP_BOX;    // 192 KB
constexpr int EP_E_BYTES = 2 * EP_BOX;            // 128 rows x 128 features: two K blocks
constexpr int EP_SMEM = 1024 + EP_W_BYTES + EP_E_BYTES + 256;
static_assert(EP_SMEM <= 232448, "shared memory per CTA");
static_assert(kEmb == 128, "two 64-column K blocks");

// Byte offset of feature pair (4 lane .. 4 lane + 3) of local row r in the
// swizzled E tile: K block lane / 16, 16-byte chunk (lane % 16) / 2 XOR (r % 8).
__device__ __forceinline__ uint32_t e_offset(int r, int lane) {
    const int kb = lane >> 4, chunk = (lane & 15) >> 1;
    return (uint32_t)(kb * EP_BOX + r * 128 + (((chunk ^ (r & 7)) << 4) | ((lane & 1) << 3)));
}

__global__ void __launch_bounds__(EP_THREADS, 1)
embed_proj_kernel(const __grid_constant__ CUtensorMap tmW, const EmbedArgs a, const float *__restrict__ b_in,
                  bf16 *__restrict__ X, unsigned long long wait_ns, int withhold_w) {
    if (a.trigger) griddep_launch_dependents();  // the next kernel may take SMs as this grid frees them

    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *wsm = base, *esm = base + EP_W_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(esm + EP_E_BYTES);  // [0] W_in landed, [1] products done
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_blocks_cap = a.rows_cap / 128;
    // (withhold_w: failure-path tests; W_in never arrives and the products' wait runs out)
    const bool loads_w = (int)blockIdx.x < n_blocks_cap && !withhold_w;

    if (threadIdx.x == 0) {
        *abort_flag = 0;
        wait_limit_init(wait_ns);
        mbar_init(smem_u32(&bars[0]), 1);
        mbar_init(smem_u32(&bars[1]), 1);
        fence_mbar_init();
    }
    __syncthreads();
    // W_in does not depend on the previous kernel: its load starts before the wait
    if (threadIdx.x == 0 && loads_w) {
        const uint32_t fb = smem_u32(&bars[0]);
        const uint64_t keep = policy_evict_last();  // read by every CTA
        mbar_arrive_expect_tx(fb, EP_W_BYTES);
        for (int kb = 0; kb < 2; ++kb)
            for (int nb = 0; nb < kHidden / 128; ++nb)
                tma_load_2d_hint(smem_u32(wsm + (kb * (kHidden / 128) + nb) * EP_BOX), &tmW, fb, kb * 64, nb * 128,
                                 keep);
    }
    griddep_wait();               // the previous kernel has completed
    const int status0 = *reinterpret_cast<const volatile int *>(a.status);
    const int n_rows = *reinterpret_cast<const volatile int *>(a.n_rows);
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_slot), 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const uint32_t lanes = (uint32_t)((warp & 3) * 32) << 16;
    const int half = warp >> 2;  // column half of each pass's products read by this warp
    bool ok = status0 == 0 && n_rows >= 0 && n_rows <= a.rows_cap;
    bool w_waited = false;
    uint32_t mph = 0;
    const uint32_t idesc = idesc_bf16_f32(128, 256);

    for (int rb = blockIdx.x; ok && rb * 128 < n_rows; rb += gridDim.x) {
        // ---- E rows of this block into shared memory: 16 per warp ----
        // The warp finds the sequence of its first row with a 32-way search (one
        // load per lane and level instead of a chain of dependent loads), then
        // lane i < 16 takes row i: its sequence is that one plus the sequences
        // that start within the sixteen rows, counted from the next 16 starts.
        const int r0 = rb * 128 + warp * 16;
        int b0 = 0;
        {
            int lo = 0, n = a.nseq;  // the answer lies in [lo, lo + n)
            while (n > 1) {
                const int step = (n + 31) / 32;
                const int k = lo + lane * step;
                const bool le = lane * step < n && __ldg(a.seq_start + k) <= r0;
                const unsigned m = __ballot_sync(0xffffffffu, le);  // lane 0 always (seq_start[lo] <= r0)
                const int h = 31 - __clz(m);
                lo += h * step;
                n = min(step, n - h * step);
            }
            b0 = lo;
        }
        const int nb = b0 + 1 + (lane & 15);
        const int next_start = nb < a.nseq ? __ldg(a.seq_start + nb) : 0x7fffffff;
        int my_t = 0, my_dst = -1;
        long long my_id = 0;
        {
            const int r = r0 + (lane & 15);
            int b = b0;
#pragma unroll
            for (int j = 0; j < 16; ++j) b += __shfl_sync(0xffffffffu, next_start, j) <= r ? 1 : 0;
            if (r < n_rows) {
                my_t = r - __ldg(a.seq_start + b);
                const bool valid = my_t < __ldg(a.seq_len + b);
                my_dst = valid ? (a.dst_padded ? b * a.T + my_t : r) : -1;
                if (!a.emb_in) {
                    my_id = a.ids_padded ? a.ids[(size_t)b * a.T + my_t] : a.ids[r];
                    if (my_id < 0 || my_id >= a.vocab) {
                        if (valid && lane < 16) set_status(a.status, kStatusId);
                        my_id = 0;  // padding slot: any id; its row never reaches a valid output
                    }
                }
                if (lane < 16) a.row_dst[r] = my_dst;
            }
        }
        const float4 g = __ldg(reinterpret_cast<const float4 *>(a.g) + lane);
        const float4 bb = __ldg(reinterpret_cast<const float4 *>(a.b) + lane);
        const float4 ty = __ldg(reinterpret_cast<const float4 *>(a.type) + lane);
#pragma unroll 1
        for (int i0 = 0; i0 < 16; i0 += 4) {
            float4 x[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int i = i0 + j, r = r0 + i;
                const long long id = __shfl_sync(0xffffffffu, my_id, i);
                const int t = __shfl_sync(0xffffffffu, my_t, i);
                if (r >= n_rows) {
                    x[j] = make_float4(0.f, 0.f, 0.f, 0.f);
                } else if (a.emb_in) {
                    // the caller supplies the post-LayerNorm embedding rows themselves
                    x[j] = reinterpret_cast<const float4 *>(a.emb_in + (size_t)r * kEmb)[lane];
                } else {
                    const float4 w = __ldg(reinterpret_cast<const float4 *>(a.word + id * kEmb) + lane);
                    const float4 ps = __ldg(reinterpret_cast<const float4 *>(a.pos + (size_t)t * kEmb) + lane);
                    x[j] = make_float4(w.x + ps.x + ty.x, w.y + ps.y + ty.y, w.z + ps.z + ty.z, w.w + ps.w + ty.w);
                }
            }
            if (a.emb_in) {
                // the caller supplies the post-LayerNorm embedding rows themselves
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    uint2 u;
                    u.x = pack_bf16x2(x[j].x, x[j].y);
                    u.y = pack_bf16x2(x[j].z, x[j].w);
                    *reinterpret_cast<uint2 *>(esm + e_offset(warp * 16 + i0 + j, lane)) = u;
                }
                continue;
            }
            // LayerNorm over the 128 features of each of the four rows (two passes,
            // the four rows' reductions interleaved)
            float sm[4], sq[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) sm[j] = x[j].x + x[j].y + x[j].z + x[j].w;
#pragma unroll
            for (int o = 16; o; o >>= 1)
#pragma unroll
                for (int j = 0; j < 4; ++j) sm[j] += __shfl_xor_sync(0xffffffffu, sm[j], o);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float mu = sm[j] * (1.0f / kEmb);
                x[j] = make_float4(x[j].x - mu, x[j].y - mu, x[j].z - mu, x[j].w - mu);
                sq[j] = x[j].x * x[j].x + x[j].y * x[j].y + x[j].z * x[j].z + x[j].w * x[j].w;
            }
#pragma unroll
            for (int o = 16; o; o >>= 1)
#pragma unroll
                for (int j = 0; j < 4; ++j) sq[j] += __shfl_xor_sync(0xffffffffu, sq[j], o);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                float y0 = 0.f, y1 = 0.f, y2 = 0.f, y3 = 0.f;
                if (r0 + i0 + j < n_rows) {
                    const float rstd = rsqrtf(sq[j] * (1.0f / kEmb) + a.eps);
                    y0 = fmaf(x[j].x * rstd, g.x, bb.x); y1 = fmaf(x[j].y * rstd, g.y, bb.y);
                    y2 = fmaf(x[j].z * rstd, g.z, bb.z); y3 = fmaf(x[j].w * rstd, g.w, bb.w);
                }
                uint2 u;
                u.x = pack_bf16x2(y0, y1);
                u.y = pack_bf16x2(y2, y3);
                *reinterpret_cast<uint2 *>(esm + e_offset(warp * 16 + i0 + j, lane)) = u;
            }
        }
        fence_proxy_async_smem();  // the tensor core reads E through the async proxy
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        // ---- two passes of products: columns 0..511, then 512..767 ----
        for (int pass = 0; pass < 2 && ok; ++pass) {
            if (threadIdx.x == 32) {
                bool ready = true;
                if (!w_waited) {
                    ready = mbar_wait(smem_u32(&bars[0]), 0, abort_flag);
                    w_waited = true;
                }
                if (ready) {
                    tc_fence_after();
                    const int nt0 = pass ? 2 : 0, nt = pass ? 1 : 2;
                    for (int t = 0; t < nt; ++t) {
#pragma unroll
                        for (int kb = 0; kb < 2; ++kb) {
                            const uint32_t ea = smem_u32(esm + kb * EP_BOX);
                            const uint32_t wb = smem_u32(wsm + (kb * (kHidden / 128) + 2 * (nt0 + t)) * EP_BOX);
#pragma unroll
                            for (int k = 0; k < 4; ++k)
                                umma_bf16(tmem_base + t * 256, sw128_kmajor_desc(ea + k * 32),
                                          sw128_kmajor_desc(wb + k * 32), idesc, (kb | k) != 0);
                        }
                    }
                }
                umma_commit(smem_u32(&bars[1]));  // (also when nothing was issued: the wait below ends)
            }
            bool got = mbar_wait(smem_u32(&bars[1]), mph, abort_flag);
            mph ^= 1;
            got = __syncthreads_and(got && !*abort_flag) != 0;
            if (!got) {
                ok = false;
                break;
            }
            tc_fence_after();
            // ---- epilogue: + b_in, bf16, rows of X ----
            // (chunk c + 1's accumulator and bias load while chunk c is processed)
            const int r = rb * 128 + (warp & 3) * 32 + lane;
            const int ncol = pass ? 128 : 256;  // TMEM columns per warp in this pass
            const int nch = ncol / 32;
            uint32_t v[2][32];
            float4 bv[2][8];
            auto fetch = [&](int c, int slot) {
                const int tcol = half * ncol + c * 32;
                tmem_ld32(tmem_base + lanes + tcol, v[slot]);
#pragma unroll
                for (int q = 0; q < 8; ++q)
                    bv[slot][q] = __ldg(reinterpret_cast<const float4 *>(b_in + pass * 512 + tcol) + q);
            };
            fetch(0, 0);
#pragma unroll 1
            for (int c = 0; c < nch; c += 2) {
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    tmem_ld_wait();
                    if (c + e + 1 < nch) fetch(c + e + 1, e ^ 1);
                    const int col = pass * 512 + half * ncol + (c + e) * 32;
                    if (r < n_rows) {
                        uint32_t pk[16];
#pragma unroll
                        for (int q = 0; q < 8; ++q) {
                            const float4 bb = bv[e][q];
                            pk[2 * q] = pack_bf16x2(__uint_as_float(v[e][4 * q]) + bb.x,
                                                    __uint_as_float(v[e][4 * q + 1]) + bb.y);
                            pk[2 * q + 1] = pack_bf16x2(__uint_as_float(v[e][4 * q + 2]) + bb.z,
                                                        __uint_as_float(v[e][4 * q + 3]) + bb.w);
                        }
                        uint4 *dst = reinterpret_cast<uint4 *>(X + (size_t)r * kHidden + col);
#pragma unroll
                        for (int q = 0; q < 4; ++q)
                            dst[q] = make_uint4(pk[4 * q], pk[4 * q + 1], pk[4 * q + 2], pk[4 * q + 3]);
                    }
                }
            }
            tmem_ld_wait();
            // the TMEM columns (next pass) and E (next block) are free once every warp is here
            tc_fence_before();
            __syncthreads();
            tc_fence_after();
        }
    }

    // W_in lands before the CTA's shared memory goes away, waited for or not
    if (threadIdx.x == 0 && loads_w) mbar_wait_drain(smem_u32(&bars[0]), 0);
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
    if (threadIdx.x == 0 && *abort_flag) set_status(a.status, kStatusTimeout);
}

}  // namespace

cudaError_t launch_embed_proj(const CUtensorMap &tmWin, const EmbedArgs &a, const float *b_in, bf16 *X, int num_sms,
                              cudaStream_t s, unsigned long long wait_ns, bool withhold_w) {
    static std::atomic<unsigned long long> configured{0};
    cudaError_t e = ensure_smem_attr(reinterpret_cast<const void *>(embed_proj_kernel), EP_SMEM, configured);
    if (e != cudaSuccess) return e;
    const int blocks = a.rows_cap / 128;
    const int grid = blocks < num_sms ? (blocks > 0 ? blocks : 1) : num_sms;
    return launch_pdl(embed_proj_kernel, dim3(grid), dim3(EP_THREADS), EP_SMEM, s, tmWin, a, b_in, X, wait_ns,
                      withhold_w ? 1 : 0);
}

}  // namespace albert
