// prep_embed.cu -- batch preparation (rows per sequence, the attention groups),
// the standalone three-table embedding + LayerNorm (small batches and the fp32
// path; larger bf16 batches use embed_proj.cu), and the output-side kernels
// (padding rows, row scatter).
//
// Embedding ("ALBERT: How Kokoro's Phoneme Encoder Works", section "Inside One
// Real ALBERT Layer", step 1; section "1. Factorized embedding" for the table
// sizes): e = word[id] + pos[t] + type[0], E = LN_128(e; gamma, beta, eps).
// Checked-input convention ("How Kokoro TTS Works and Where CKE Stands":
// invalid ids and arena rejection are detected before any output is written;
// a failed check stops downstream work): these kernels record an error in
// the device status word and every later kernel of the forward returns
// without writing.
#include "kernels.h"
#include "sm100_ptx.cuh"

namespace albert {
namespace {

constexpr int PREP_THREADS = 1024;

// Block-wide exclusive scan of rows[b] (b < n) into start[b]; returns the total.
__device__ int block_exclusive_scan(const int *rows, int n, int *start, int *sh) {
    const int tid = threadIdx.x;
    const int chunk = (n + PREP_THREADS - 1) / PREP_THREADS;
    const int lo = min(n, tid * chunk), hi = min(n, lo + chunk);
    int local = 0;
    for (int i = lo; i < hi; ++i) local += rows[i];
    sh[tid] = local;
    __syncthreads();
    for (int off = 1; off < PREP_THREADS; off <<= 1) {
        const int v = tid >= off ? sh[tid - off] : 0;
        __syncthreads();
        sh[tid] += v;
        __syncthreads();
    }
    int run = sh[tid] - local;  // exclusive prefix of this thread's chunk
    for (int i = lo; i < hi; ++i) {
        const int v = rows[i];  // rows and start may be the same array
        start[i] = run;
        run += v;
    }
    const int total = sh[PREP_THREADS - 1];
    __syncthreads();
    return total;
}

// Attention groups (launch_attention_tc): the k-th and (k+1)-th sequences of at
// most 64 tokens (k even, in batch order) share one item, as its two 64-row
// halves; longer sequences, and a last short one without a partner, have an item
// each.  groups[g] = {start, length, partner start, partner length} (partner
// length 0: one sequence): the pairs first, then the longer sequences in batch
// order, then the unpaired short one.  One warp, 32 sequences per step, ranks
// from ballots.  Warp 0 only; seq_start / seq_len are final and visible to it.
__device__ void build_attention_groups(const int *seq_start, const int *seq_len, int n, int4 *groups,
                                       int *n_groups) {
    const int lane = threadIdx.x & 31;
    const unsigned below = (1u << lane) - 1u;
    int n_short = 0;
    for (int base = 0; base < n; base += 32) {
        const int b = base + lane;
        n_short += __popc(__ballot_sync(0xffffffffu, b < n && seq_len[b] <= kAttnHalfRows));
    }
    const int n_pairs = n_short >> 1;
    const int n_long = n - n_short;
    int2 *half = reinterpret_cast<int2 *>(groups);  // {start, length} halves of the entries
    int short_seen = 0, long_seen = 0;
    for (int base = 0; base < n; base += 32) {
        const int b = base + lane;
        const int len = b < n ? seq_len[b] : 0, st = b < n ? seq_start[b] : 0;
        const bool is_short = b < n && len <= kAttnHalfRows, is_long = b < n && !is_short;
        const unsigned S = __ballot_sync(0xffffffffu, is_short), Lg = __ballot_sync(0xffffffffu, is_long);
        if (is_short) {
            const int k = short_seen + __popc(S & below);
            if (k < 2 * n_pairs) half[k] = make_int2(st, len);  // entry k / 2, half k % 2
            else groups[n_pairs + n_long] = make_int4(st, len, 0, 0);
        } else if (is_long) {
            groups[n_pairs + long_seen + __popc(Lg & below)] = make_int4(st, len, 0, 0);
        }
        short_seen += __popc(S);
        long_seen += __popc(Lg);
    }
    if (lane == 0) *n_groups = n_pairs + n_long + (n_short & 1);
}

// Padded batch: mask[B, T] must hold, per row, a non-empty prefix of non-zero
// bytes followed only by zeros.  L_b = prefix length.  Packed mode gives
// sequence b L_b rows, padded mode T rows.
__global__ void __launch_bounds__(PREP_THREADS)
prep_padded_kernel(const uint8_t *__restrict__ mask, int B, int T, int pack, int rows_cap,
                   int *seq_start, int *seq_len, int *n_rows, int *status, int4 *groups, int *n_groups, int trigger) {
    if (trigger) griddep_launch_dependents();  // the next kernel may take SMs as this grid frees them
    griddep_wait();               // the previous kernel has completed

    __shared__ int sh[PREP_THREADS];
    __shared__ int bad;
    if (threadIdx.x == 0) { *status = 0; bad = 0; }
    __syncthreads();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int b = warp; b < B; b += PREP_THREADS / 32) {
        const uint8_t *m = mask + (size_t)b * T;
        int first_zero = T, last_one = -1;
        for (int t = lane; t < T; t += 32) {
            const bool on = m[t] != 0;
            if (!on) first_zero = min(first_zero, t);
            else last_one = max(last_one, t);
        }
        for (int o = 16; o; o >>= 1) {
            first_zero = min(first_zero, __shfl_xor_sync(0xffffffffu, first_zero, o));
            last_one = max(last_one, __shfl_xor_sync(0xffffffffu, last_one, o));
        }
        const bool ok = first_zero >= 1 && last_one < first_zero;
        if (lane == 0) {
            seq_len[b] = ok ? first_zero : 0;
            if (!ok) bad = 1;
        }
    }
    __syncthreads();
    if (bad) {
        if (threadIdx.x == 0) { set_status(status, kStatusMask); *n_rows = 0; *n_groups = 0; }
        return;
    }
    // rows per sequence, reusing seq_start as the input of the scan
    for (int b = threadIdx.x; b < B; b += PREP_THREADS) seq_start[b] = pack ? seq_len[b] : T;
    __syncthreads();
    const int total = block_exclusive_scan(seq_start, B, seq_start, sh);  // ends with a block barrier
    if (threadIdx.x == 0) {
        *n_rows = total;
        if (total > rows_cap) set_status(status, kStatusShape);
    }
    if (warp == 0) build_attention_groups(seq_start, seq_len, B, groups, n_groups);
}

// Packed batch: cu[0] == 0, 1 <= cu[s+1]-cu[s] <= max_len, cu[nseq] <= rows_cap.
__global__ void __launch_bounds__(PREP_THREADS)
prep_varlen_kernel(const int32_t *__restrict__ cu, int nseq, int max_len, int rows_cap,
                   int *seq_start, int *seq_len, int *n_rows, int *status, int4 *groups, int *n_groups,
                   int trigger) {
    if (trigger) griddep_launch_dependents();  // the next kernel may take SMs as this grid frees them
    griddep_wait();               // the previous kernel has completed

    __shared__ int bad;
    if (threadIdx.x == 0) { *status = 0; bad = 0; }
    __syncthreads();
    for (int s = threadIdx.x; s < nseq; s += PREP_THREADS) {
        const int a = cu[s], e = cu[s + 1];
        const int len = e - a;
        seq_start[s] = a;
        seq_len[s] = len;
        if (len < 1 || len > max_len || (s == 0 && a != 0)) bad = 1;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const int total = cu[nseq];
        if (bad) {
            set_status(status, kStatusSeqlens);
            *n_rows = 0;
        } else if (total > rows_cap) {
            set_status(status, kStatusShape);
            *n_rows = 0;
        } else {
            *n_rows = total;
        }
    }
    if (threadIdx.x < 32) {
        if (bad) {
            if (threadIdx.x == 0) *n_groups = 0;
        } else {
            build_attention_groups(seq_start, seq_len, nseq, groups, n_groups);
        }
    }
}

// One warp per row: gather the three table rows, LayerNorm over 128 (two-pass,
// fp32), write E (bf16 or fp32) and the row's destination in the output.
__global__ void __launch_bounds__(256)
embed_ln_kernel(const EmbedArgs a) {
    if (a.trigger) griddep_launch_dependents();  // the next kernel may take SMs as this grid frees them
    griddep_wait();               // the previous kernel has completed

    if (*reinterpret_cast<const volatile int *>(a.status) != 0) return;
    const int n_rows = *a.n_rows;
    const int r = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (r >= n_rows) return;
    // sequence of row r: last b with seq_start[b] <= r
    int lo = 0, hi = a.nseq - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (__ldg(a.seq_start + mid) <= r) lo = mid; else hi = mid - 1;
    }
    const int b = lo;
    const int t = r - __ldg(a.seq_start + b);
    const bool valid = t < __ldg(a.seq_len + b);
    float y0, y1, y2, y3;
    if (a.emb_in) {
        // the caller supplies the post-LayerNorm embedding rows themselves
        const float4 e = reinterpret_cast<const float4 *>(a.emb_in + (size_t)r * kEmb)[lane];
        y0 = e.x; y1 = e.y; y2 = e.z; y3 = e.w;
    } else {
        long long id = a.ids_padded ? a.ids[(size_t)b * a.T + t] : a.ids[r];
        if (id < 0 || id >= a.vocab) {
            if (valid) set_status(a.status, kStatusId);
            id = 0;  // padding slot: any id; its row never reaches a valid output
        }
        const float4 w = __ldg(reinterpret_cast<const float4 *>(a.word + id * kEmb) + lane);
        const float4 ps = __ldg(reinterpret_cast<const float4 *>(a.pos + (size_t)t * kEmb) + lane);
        const float4 ty = __ldg(reinterpret_cast<const float4 *>(a.type) + lane);
        float x[4] = {w.x + ps.x + ty.x, w.y + ps.y + ty.y, w.z + ps.z + ty.z, w.w + ps.w + ty.w};
        float s = x[0] + x[1] + x[2] + x[3];
        for (int o = 16; o; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        const float mu = s * (1.0f / kEmb);
        float q = 0.f;
        for (int i = 0; i < 4; ++i) { const float d = x[i] - mu; q = fmaf(d, d, q); }
        for (int o = 16; o; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
        const float rstd = rsqrtf(q * (1.0f / kEmb) + a.eps);
        const float4 g = __ldg(reinterpret_cast<const float4 *>(a.g) + lane);
        const float4 bb = __ldg(reinterpret_cast<const float4 *>(a.b) + lane);
        y0 = fmaf((x[0] - mu) * rstd, g.x, bb.x); y1 = fmaf((x[1] - mu) * rstd, g.y, bb.y);
        y2 = fmaf((x[2] - mu) * rstd, g.z, bb.z); y3 = fmaf((x[3] - mu) * rstd, g.w, bb.w);
    }
    if (a.out_f32) {
        reinterpret_cast<float4 *>(static_cast<float *>(a.E) + (size_t)r * kEmb)[lane] = make_float4(y0, y1, y2, y3);
    } else {
        uint2 u;
        u.x = pack_bf16x2(y0, y1);
        u.y = pack_bf16x2(y2, y3);
        reinterpret_cast<uint2 *>(static_cast<bf16 *>(a.E) + (size_t)r * kEmb)[lane] = u;
    }
    if (lane == 0) a.row_dst[r] = valid ? (a.dst_padded ? b * a.T + t : r) : -1;
}

__global__ void zero_pad_kernel(uint4 *out, int B, int T, int chunks_per_row, const int *seq_len,
                                const int *status) {
    // last kernel of a forward: no early trigger, so that whatever follows in the
    // stream waits for its completion (and, through the chain, the whole forward's)
    griddep_wait();               // the previous kernel has completed

    if (*reinterpret_cast<const volatile int *>(status) != 0) return;
    const size_t n = (size_t)B * T * chunks_per_row;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        const size_t row = i / chunks_per_row;
        const int b = (int)(row / T), t = (int)(row % T);
        if (t >= __ldg(seq_len + b)) out[i] = make_uint4(0, 0, 0, 0);
    }
}

// Per sequence b: a [T, D] block of token-major rows -> [D, T], through 32x32
// shared tiles (reads along d, writes along t, both coalesced); padding slots 0.
template <typename E>
__global__ void __launch_bounds__(256)
transpose_out_kernel(const E *__restrict__ src, E *__restrict__ out, int T, int D, const int *__restrict__ seq_len,
                     const int *status) {
    // last kernel of a forward: no early trigger
    griddep_wait();               // the previous kernel has completed
    if (*reinterpret_cast<const volatile int *>(status) != 0) return;
    __shared__ E tile[32][33];
    const int b = blockIdx.z, t0 = blockIdx.x * 32, d0 = blockIdx.y * 32;
    const int L = __ldg(seq_len + b);
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8
    for (int k = ty; k < 32; k += 8) {
        const int t = t0 + k, d = d0 + tx;
        tile[k][tx] = (t < L && d < D) ? src[((size_t)b * T + t) * D + d] : E(0);
    }
    __syncthreads();
    for (int k = ty; k < 32; k += 8) {
        const int d = d0 + k, t = t0 + tx;
        if (d < D && t < T) out[((size_t)b * D + d) * T + t] = tile[tx][k];
    }
}

__global__ void scatter_rows_kernel(const uint4 *X, uint4 *out, int chunks_per_row, int rows_cap,
                                    const int *n_rows, const int *row_dst, const int *status) {
    // last kernel of a forward: no early trigger, so that whatever follows in the
    // stream waits for its completion (and, through the chain, the whole forward's)
    griddep_wait();               // the previous kernel has completed

    if (*reinterpret_cast<const volatile int *>(status) != 0) return;
    const int rows = *n_rows;
    const size_t n = (size_t)rows * chunks_per_row;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
        const int r = (int)(i / chunks_per_row), c = (int)(i % chunks_per_row);
        const int d = __ldg(row_dst + r);
        if (d >= 0) out[(size_t)d * chunks_per_row + c] = X[i];
    }
}

__global__ void f32_to_bf16_kernel(const float *src, bf16 *dst, size_t n) {
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
        dst[i] = __float2bfloat16_rn(src[i]);
}

}  // namespace

cudaError_t launch_prep_padded(const uint8_t *mask, int B, int T, int pack, int rows_cap,
                               int *seq_start, int *seq_len, int *n_rows, int *status,
                               int4 *groups, int *n_groups, cudaStream_t s, bool trigger) {
    // The first kernel of a forward: a plain launch, so that it is ordered after
    // every earlier operation of the stream (copies of the inputs included).
    prep_padded_kernel<<<1, PREP_THREADS, 0, s>>>(mask, B, T, pack, rows_cap, seq_start, seq_len, n_rows, status,
                                                  groups, n_groups, trigger ? 1 : 0);
    return cudaGetLastError();
}

cudaError_t launch_prep_varlen(const int32_t *cu, int nseq, int max_len, int rows_cap,
                               int *seq_start, int *seq_len, int *n_rows, int *status,
                               int4 *groups, int *n_groups, cudaStream_t s, bool trigger) {
    // first kernel of a forward: plain launch (see launch_prep_padded)
    prep_varlen_kernel<<<1, PREP_THREADS, 0, s>>>(cu, nseq, max_len, rows_cap, seq_start, seq_len, n_rows, status,
                                                  groups, n_groups, trigger ? 1 : 0);
    return cudaGetLastError();
}

cudaError_t launch_embed(const EmbedArgs &a, cudaStream_t s) {
    const int blocks = (a.rows_cap + 7) / 8;
    return launch_pdl(embed_ln_kernel, dim3(blocks), dim3(256), 0, s, a);
}

static int grid_for(size_t n, int threads) {
    size_t b = (n + threads - 1) / threads;
    if (b > 148 * 16) b = 148 * 16;
    return b < 1 ? 1 : (int)b;
}

cudaError_t launch_zero_pad(void *out, int B, int T, int D, int elem_bytes, const int *seq_len,
                            const int *status, cudaStream_t s) {
    const int cpr = D * elem_bytes / 16;
    const size_t n = (size_t)B * T * cpr;
    return launch_pdl(zero_pad_kernel, dim3(grid_for(n, 256)), dim3(256), 0, s, static_cast<uint4 *>(out), B, T, cpr,
                      seq_len, status);
}

cudaError_t launch_transpose_out(const void *src, void *out, int B, int T, int D, int elem_bytes,
                                 const int *seq_len, const int *status, cudaStream_t s) {
    const dim3 grid((T + 31) / 32, (D + 31) / 32, B);
    if (elem_bytes == 2)
        return launch_pdl(transpose_out_kernel<uint16_t>, grid, dim3(256), 0, s, static_cast<const uint16_t *>(src),
                          static_cast<uint16_t *>(out), T, D, seq_len, status);
    return launch_pdl(transpose_out_kernel<float>, grid, dim3(256), 0, s, static_cast<const float *>(src),
                      static_cast<float *>(out), T, D, seq_len, status);
}

cudaError_t launch_scatter_rows(const void *X, void *out, int D, int elem_bytes, int rows_cap,
                                const int *n_rows, const int *row_dst, const int *status,
                                cudaStream_t s) {
    const int cpr = D * elem_bytes / 16;
    const size_t n = (size_t)rows_cap * cpr;
    return launch_pdl(scatter_rows_kernel, dim3(grid_for(n, 256)), dim3(256), 0, s, static_cast<const uint4 *>(X),
                      static_cast<uint4 *>(out), cpr, rows_cap, n_rows, row_dst, status);
}

cudaError_t launch_f32_to_bf16(const float *src, bf16 *dst, size_t n, cudaStream_t s) {
    f32_to_bf16_kernel<<<grid_for(n, 256), 256, 0, s>>>(src, dst, n);
    return cudaGetLastError();
}

}  // namespace albert
