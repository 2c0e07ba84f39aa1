// attention.cu -- bidirectional multi-head attention with a key-padding mask.
//
// Per sequence b and head h ("ALBERT: How Kokoro's Phoneme Encoder Works",
// section "Inside One Real ALBERT Layer", step 4; "How Kokoro TTS Works and
// Where CKE Stands", section "What ALBERT does here"):
//     C_h = softmax(Q_h K_h^T / sqrt(64) + mask) V_h,
// where key u of sequence b takes part iff u < L_b (additive -inf mask) and
// every query attends to keys on both sides.  Q, K, V live in one packed
// [rows, 3*768] buffer (Q | K | V); head h is the 64-column slice 64h..64h+63
// of each; the context goes to [rows, 768] with the same head layout.
//
// The forward pass runs the tcgen05 kernels (attention_tc.cu, attention_tc_long.cu)
// for bf16; the bf16 kernel here is an independent mma.sync implementation of
// the same operation, reachable through albert_test_attention as a cross-check.
//
// bf16 kernel: one CTA per (sequence, head, query tile of 16 rows per warp;
// 4 warps for T <= 128, 8 warps above).  The head's whole K and V (L_b <= 512
// rows of 64 bf16) are staged in shared memory by cp.async, one commit group
// per 64-key block, so the first block's math overlaps the later blocks'
// loads; each warp runs an online (max-subtracted) softmax over the 64-key
// blocks with mma.sync m16n8k16 (bf16 in, fp32 accumulate), keeping P in
// registers between the two products.
#include "kernels.h"
#include "sm100_ptx.cuh"

namespace albert {
namespace {

constexpr int KBLK = 64;     // keys per online-softmax block
constexpr int LDS = 72;      // shared row stride in bf16 (144 B): conflict-free ldmatrix

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const bf16 *p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const bf16 *p) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(smem_u32(p)));
}
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                               uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// 16-byte global -> shared copy; src_bytes = 0 writes zeros and reads nothing.
__device__ __forceinline__ void cp_async16(bf16 *dst, const bf16 *src, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// Wait until at most n of this thread's cp.async groups are still pending (n <= 7).
__device__ __forceinline__ void cp_async_wait_pending(int n) {
    switch (n) {
        case 0: asm volatile("cp.async.wait_group 0;" ::: "memory"); break;
        case 1: asm volatile("cp.async.wait_group 1;" ::: "memory"); break;
        case 2: asm volatile("cp.async.wait_group 2;" ::: "memory"); break;
        case 3: asm volatile("cp.async.wait_group 3;" ::: "memory"); break;
        case 4: asm volatile("cp.async.wait_group 4;" ::: "memory"); break;
        case 5: asm volatile("cp.async.wait_group 5;" ::: "memory"); break;
        case 6: asm volatile("cp.async.wait_group 6;" ::: "memory"); break;
        default: asm volatile("cp.async.wait_group 7;" ::: "memory"); break;
    }
}

template <int NW>
__global__ void __launch_bounds__(NW * 32)
attn_bf16_kernel(const bf16 *__restrict__ qkv, bf16 *__restrict__ ctx, const int *__restrict__ seq_start,
                 const int *__restrict__ seq_len, const int *__restrict__ status, int trigger) {
    if (trigger) griddep_launch_dependents();  // the next kernel may take SMs as this grid frees them
    griddep_wait();               // the previous kernel has completed

    constexpr int QT = 16 * NW, NT = 32 * NW;
    if (*reinterpret_cast<const volatile int *>(status) != 0) return;
    const int b = blockIdx.z, h = blockIdx.y, q0 = blockIdx.x * QT;
    const int L = seq_len[b];
    if (q0 >= L) return;
    const int start = seq_start[b];
    const int nkb = (L + KBLK - 1) / KBLK;

    extern __shared__ uint4 smem4[];
    bf16 *sQ = reinterpret_cast<bf16 *>(smem4);
    bf16 *sK = sQ + QT * LDS;
    bf16 *sV = sK + nkb * KBLK * LDS;
    const bf16 *base = qkv + (size_t)start * kQKV + h * kHeadDim;

    // group 0: the query tile and key/value block 0; group j: key/value block j
    for (int j = 0; j < nkb; ++j) {
        if (j == 0) {
            for (int i = threadIdx.x; i < QT * 8; i += NT) {
                const int t = i >> 3, c = i & 7, row = q0 + t;
                cp_async16(sQ + t * LDS + c * 8, base + (size_t)min(row, L - 1) * kQKV + c * 8, row < L ? 16 : 0);
            }
        }
        for (int i = threadIdx.x; i < 2 * KBLK * 8; i += NT) {
            const int which = i >> 9, r = (i >> 3) & (KBLK - 1), c = i & 7, u = j * KBLK + r;
            const bf16 *src = base + (size_t)min(u, L - 1) * kQKV + (1 + which) * kHidden + c * 8;
            cp_async16((which ? sV : sK) + u * LDS + c * 8, src, u < L ? 16 : 0);
        }
        cp_async_commit();
    }

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int qw = q0 + warp * 16;
    const bool active = qw < L;
    const int g = lane >> 2, tig = lane & 3;
    const int j8 = lane >> 3, r8 = lane & 7;
    // scores are kept in log2 units: s * (1/8) * log2(e)
    const float sl2 = 0.125f * 1.4426950408889634f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    float o[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    uint32_t qf[4][4];

    for (int j = 0; j < nkb; ++j) {
        cp_async_wait_pending(nkb - 1 - j);
        __syncthreads();
        if (!active) continue;
        if (j == 0) {
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                ldsm_x4(qf[ks], sQ + (warp * 16 + (lane & 15)) * LDS + ks * 16 + (lane >> 4) * 8);
        }
        const int kb = j * KBLK;
        float s[8][4];
#pragma unroll
        for (int i = 0; i < 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
            for (int np = 0; np < 4; ++np) {
                uint32_t kf[4];
                ldsm_x4(kf, sK + (kb + np * 16 + (j8 >> 1) * 8 + r8) * LDS + ks * 16 + (j8 & 1) * 8);
                mma_bf16_16816(s[2 * np], qf[ks], kf[0], kf[1]);
                mma_bf16_16816(s[2 * np + 1], qf[ks], kf[2], kf[3]);
            }
        }
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            const int key = kb + nt * 8 + tig * 2;
            s[nt][0] = key < L ? s[nt][0] * sl2 : -INFINITY;
            s[nt][1] = key + 1 < L ? s[nt][1] * sl2 : -INFINITY;
            s[nt][2] = key < L ? s[nt][2] * sl2 : -INFINITY;
            s[nt][3] = key + 1 < L ? s[nt][3] * sl2 : -INFINITY;
            mx0 = fmaxf(mx0, fmaxf(s[nt][0], s[nt][1]));
            mx1 = fmaxf(mx1, fmaxf(s[nt][2], s[nt][3]));
        }
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);  // finite: block holds a valid key
        const float a0 = ex2_approx(m0 - mn0), a1 = ex2_approx(m1 - mn1);
        m0 = mn0;
        m1 = mn1;
        float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            s[nt][0] = ex2_approx(s[nt][0] - mn0);
            s[nt][1] = ex2_approx(s[nt][1] - mn0);
            s[nt][2] = ex2_approx(s[nt][2] - mn1);
            s[nt][3] = ex2_approx(s[nt][3] - mn1);
            rs0 += s[nt][0] + s[nt][1];
            rs1 += s[nt][2] + s[nt][3];
        }
        l0 = l0 * a0 + rs0;
        l1 = l1 * a1 + rs1;
#pragma unroll
        for (int nd = 0; nd < 8; ++nd) {
            o[nd][0] *= a0; o[nd][1] *= a0;
            o[nd][2] *= a1; o[nd][3] *= a1;
        }
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            uint32_t pa[4];
            pa[0] = pack_bf16x2(s[2 * jj][0], s[2 * jj][1]);
            pa[1] = pack_bf16x2(s[2 * jj][2], s[2 * jj][3]);
            pa[2] = pack_bf16x2(s[2 * jj + 1][0], s[2 * jj + 1][1]);
            pa[3] = pack_bf16x2(s[2 * jj + 1][2], s[2 * jj + 1][3]);
#pragma unroll
            for (int dp = 0; dp < 4; ++dp) {
                uint32_t vf[4];
                ldsm_x4_t(vf, sV + (kb + jj * 16 + (j8 & 1) * 8 + r8) * LDS + dp * 16 + (j8 >> 1) * 8);
                mma_bf16_16816(o[2 * dp], pa, vf[0], vf[1]);
                mma_bf16_16816(o[2 * dp + 1], pa, vf[2], vf[3]);
            }
        }
    }
    if (!active) return;
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    const float i0 = 1.f / l0, i1 = 1.f / l1;
    const int t0 = qw + g, t1 = qw + g + 8;
#pragma unroll
    for (int nd = 0; nd < 8; ++nd) {
        const int col = h * kHeadDim + nd * 8 + tig * 2;
        if (t0 < L)
            *reinterpret_cast<uint32_t *>(ctx + (size_t)(start + t0) * kHidden + col) =
                pack_bf16x2(o[nd][0] * i0, o[nd][1] * i0);
        if (t1 < L)
            *reinterpret_cast<uint32_t *>(ctx + (size_t)(start + t1) * kHidden + col) =
                pack_bf16x2(o[nd][2] * i1, o[nd][3] * i1);
    }
}

// fp32 kernel: one warp per query row; scores of the row in shared memory.
constexpr int F32_ROWS = 8;
__global__ void __launch_bounds__(32 * F32_ROWS)
attn_f32_kernel(const float *__restrict__ qkv, float *__restrict__ ctx, const int *__restrict__ seq_start,
                const int *__restrict__ seq_len, const int *__restrict__ status, int max_len) {
    if (*reinterpret_cast<const volatile int *>(status) != 0) return;
    const int b = blockIdx.z, h = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = blockIdx.x * F32_ROWS + warp;
    const int L = seq_len[b];
    if (t >= L) return;
    const int start = seq_start[b];
    extern __shared__ float fsm[];
    float *sc = fsm + warp * max_len;
    float *qs = fsm + F32_ROWS * max_len + warp * kHeadDim;
    const float *qrow = qkv + (size_t)(start + t) * kQKV + h * kHeadDim;
    qs[lane] = qrow[lane];
    qs[lane + 32] = qrow[lane + 32];
    __syncwarp();
    const float scale = 0.125f;
    float mx = -INFINITY;
    for (int u = lane; u < L; u += 32) {
        const float *k = qkv + (size_t)(start + u) * kQKV + kHidden + h * kHeadDim;
        float d = 0.f;
        for (int i = 0; i < kHeadDim; ++i) d = fmaf(qs[i], k[i], d);
        d *= scale;
        sc[u] = d;
        mx = fmaxf(mx, d);
    }
    for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float den = 0.f;
    for (int u = lane; u < L; u += 32) {
        const float e = expf(sc[u] - mx);
        sc[u] = e;
        den += e;
    }
    for (int o = 16; o; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    __syncwarp();
    const float inv = 1.f / den;
    float a0 = 0.f, a1 = 0.f;
    for (int u = 0; u < L; ++u) {
        const float *v = qkv + (size_t)(start + u) * kQKV + 2 * kHidden + h * kHeadDim;
        a0 = fmaf(sc[u], v[lane], a0);
        a1 = fmaf(sc[u], v[lane + 32], a1);
    }
    float *crow = ctx + (size_t)(start + t) * kHidden + h * kHeadDim;
    crow[lane] = a0 * inv;
    crow[lane + 32] = a1 * inv;
}

}  // namespace

static size_t attn_bf16_smem(int max_len, int qt) {
    const int lpad = (max_len + KBLK - 1) / KBLK * KBLK;
    return (size_t)(qt + 2 * lpad) * LDS * sizeof(bf16);
}

template <int NW>
static cudaError_t launch_attn_nw(const bf16 *qkv, bf16 *ctx, const int *seq_start, const int *seq_len, int nseq,
                                  int max_len, const int *status, cudaStream_t s, bool trigger) {
    constexpr int QT = 16 * NW;
    static std::atomic<unsigned long long> configured{0};
    cudaError_t e = ensure_smem_attr(reinterpret_cast<const void *>(attn_bf16_kernel<NW>),
                                     (int)attn_bf16_smem(kMaxPos, QT), configured);
    if (e != cudaSuccess) return e;
    dim3 grid((max_len + QT - 1) / QT, kHeads, nseq);
    return launch_pdl(attn_bf16_kernel<NW>, grid, dim3(NW * 32), attn_bf16_smem(max_len, QT), s, qkv, ctx, seq_start,
                      seq_len, status, trigger ? 1 : 0);
}

cudaError_t launch_attention_bf16(const bf16 *qkv, bf16 *ctx, const int *seq_start,
                                  const int *seq_len, int nseq, int max_len, const int *status,
                                  cudaStream_t s, bool trigger) {
    if (nseq <= 0) return cudaSuccess;
    if (max_len <= 128) return launch_attn_nw<4>(qkv, ctx, seq_start, seq_len, nseq, max_len, status, s, trigger);
    return launch_attn_nw<8>(qkv, ctx, seq_start, seq_len, nseq, max_len, status, s, trigger);
}

cudaError_t launch_attention_f32(const float *qkv, float *ctx, const int *seq_start,
                                 const int *seq_len, int nseq, int max_len, const int *status,
                                 cudaStream_t s) {
    if (nseq <= 0) return cudaSuccess;
    const size_t smem = (size_t)F32_ROWS * (max_len + kHeadDim) * sizeof(float);
    static std::atomic<unsigned long long> configured{0};
    cudaError_t e = ensure_smem_attr(reinterpret_cast<const void *>(attn_f32_kernel),
                                     (int)((size_t)F32_ROWS * (kMaxPos + kHeadDim) * sizeof(float)), configured);
    if (e != cudaSuccess) return e;
    dim3 grid((max_len + F32_ROWS - 1) / F32_ROWS, kHeads, nseq);
    attn_f32_kernel<<<grid, 32 * F32_ROWS, smem, s>>>(qkv, ctx, seq_start, seq_len, status, max_len);
    return cudaGetLastError();
}

}  // namespace albert
