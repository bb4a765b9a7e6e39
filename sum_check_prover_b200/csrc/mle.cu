// Multilinear-extension kernels: eq tables, the eq-weighted row contraction
// ("partial evaluation") of int4 / int8 matrices, and the per-site output
// claims of the matmul sum-check.
//
// The partial evaluation is the matmul sum-check's weight decode ("How fast
// can FlashProve go", 4 Tighter Rooflines: weights decoded once for the
// matmuls' sum-checks). out[c] = sum_i eq[i] * W_eff[i][c] streams W once.
// Weights are small integers, so no modular reduction happens in the inner
// loop: with u = W_eff + off >= 0 and eq[i] = eh * 2^32 + el, the two exact
// 64-bit sums  Lo = sum el * u  and  Hi = sum eh * u  are kept per column and
// folded into the field once per row block: Lo + 2^32 Hi - off * sum eq.
#include <vector>

#include "fp_field.cuh"
#include "fp_internal.h"

namespace {

constexpr int PR_THREADS = 128;
constexpr int PR_COLS = 16;                   // columns per thread
constexpr int PR_ROWS_PER_SPLIT_MAX = 1 << 14;  // keeps every 64-bit sum exact

__global__ void eq_build_kernel(FpPoint z, uint64_t* out, uint64_t n) {
    uint64_t x = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (x >= n) return;
    uint64_t e = 1;
    for (int b = 0; b < z.v; b++) e = gl_mul(e, gl_eq1(z.z[b], (int)((x >> (z.v - 1 - b)) & 1)));
    out[x] = e;
}

// Sum of eq[0..n) into *out (single block).
__global__ void sum_kernel(const uint64_t* v, uint64_t n, uint64_t* out) {
    __shared__ uint64_t red[32];
    uint64_t acc = 0;
    for (uint64_t i = threadIdx.x; i < n; i += blockDim.x) acc = gl_add(acc, v[i]);
    acc = warp_sum_gl(acc);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x < 32) {
        uint64_t a = (threadIdx.x < (blockDim.x >> 5)) ? red[threadIdx.x] : 0;
        a = warp_sum_gl(a);
        if (threadIdx.x == 0) *out = a;
    }
}

__device__ __forceinline__ int nib(uint64_t w, int c) { return (int)((w >> (4 * c)) & 15); }

// Lo + 2^32 * Hi (mod p)
__device__ __forceinline__ uint64_t fold_lohi(uint64_t lo, uint64_t hi) {
    return gl_add(gl_canon(lo), gl_mul_2_32(gl_canon(hi)));
}

// One thread: PR_COLS consecutive columns starting at col0 over rows [r0, r1).
template <bool W4, bool SCALED, bool ALIGNED>
__global__ void __launch_bounds__(PR_THREADS)
    partial_acc_kernel(const uint8_t* __restrict__ mat, const int8_t* __restrict__ scales, int rows, int cols,
                       int64_t pitch, const uint64_t* __restrict__ eq, int rows_per_split,
                       uint64_t* __restrict__ part) {
    const int col0 = (blockIdx.x * PR_THREADS + threadIdx.x) * PR_COLS;
    const int r0 = blockIdx.y * rows_per_split;
    const int r1 = min(rows, r0 + rows_per_split);
    if (col0 >= cols) return;
    const int G = (cols + 63) / 64;
    const uint32_t off = SCALED ? (W4 ? 1024u : 16384u) : (W4 ? 8u : 128u);
    uint64_t lo[PR_COLS], hi[PR_COLS];
#pragma unroll
    for (int c = 0; c < PR_COLS; c++) lo[c] = hi[c] = 0;

    for (int i = r0; i < r1; i++) {
        const uint64_t e = __ldg(eq + i);
        const uint32_t el = (uint32_t)e, eh = (uint32_t)(e >> 32);
        const int32_t sc = SCALED ? (int32_t)__ldg(scales + (int64_t)i * G + (col0 >> 6)) : 1;
        int32_t w[PR_COLS];
        if (ALIGNED) {
            if (W4) {
                const uint2 v = __ldg(reinterpret_cast<const uint2*>(mat + (int64_t)i * pitch + (col0 >> 1)));
                const uint64_t b = ((uint64_t)v.y << 32) | v.x;
#pragma unroll
                for (int c = 0; c < PR_COLS; c++) {
                    int n = nib(b, c);
                    w[c] = n >= 8 ? n - 16 : n;
                }
            } else {
                const uint4 v = __ldg(reinterpret_cast<const uint4*>(mat + (int64_t)i * pitch + col0));
                const uint32_t wd[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int c = 0; c < PR_COLS; c++) w[c] = (int32_t)(int8_t)(wd[c >> 2] >> (8 * (c & 3)));
            }
        } else {
#pragma unroll
            for (int c = 0; c < PR_COLS; c++) {
                const int cc = col0 + c;
                int v = 0;
                if (cc < cols) {
                    if (W4) {
                        uint8_t b = mat[(int64_t)i * pitch + (cc >> 1)];
                        int n = (cc & 1) ? (b >> 4) : (b & 15);
                        v = n >= 8 ? n - 16 : n;
                    } else {
                        v = (int8_t)mat[(int64_t)i * pitch + cc];
                    }
                    if (SCALED) v *= (int32_t)__ldg(scales + (int64_t)i * G + (cc >> 6));
                }
                w[c] = v;
            }
        }
#pragma unroll
        for (int c = 0; c < PR_COLS; c++) {
            const uint32_t u = (uint32_t)((ALIGNED && SCALED ? w[c] * sc : w[c]) + (int32_t)off);
            lo[c] += (uint64_t)el * u;
            hi[c] += (uint64_t)eh * u;
        }
    }
    uint64_t* o = part + (int64_t)blockIdx.y * cols;
#pragma unroll
    for (int c = 0; c < PR_COLS; c++)
        if (col0 + c < cols) o[col0 + c] = fold_lohi(lo[c], hi[c]);
}

// out[c] = sum_s part[s][c] - off * E for c < cols; 0 up to cols_pad.
__global__ void partial_fin_kernel(const uint64_t* __restrict__ part, int splits, int cols, int64_t cols_pad,
                                   const uint64_t* __restrict__ esum, uint64_t off, uint64_t* __restrict__ out) {
    int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= cols_pad) return;
    if (c >= cols) {
        out[c] = 0;
        return;
    }
    uint64_t a = 0;
    for (int s = 0; s < splits; s++) a = gl_add(a, part[(int64_t)s * cols + c]);
    out[c] = gl_sub(a, gl_mul(off, *esum));
}

// ---- output claims ------------------------------------------------------------

struct ClaimSite {
    const int32_t* q;
    const int32_t* r;
    const uint64_t* eq_row;
    const uint64_t* eq_col;
    int32_t M, N, k;
    int32_t pad;
    int64_t first_block;
};

constexpr int CL_THREADS = 256;
constexpr int CL_ELEMS = 4096;  // flat elements per block

__global__ void __launch_bounds__(CL_THREADS)
    claim_kernel(const ClaimSite* __restrict__ sites, int nsites, uint64_t* __restrict__ part) {
    __shared__ uint64_t red[CL_THREADS / 32];
    const int64_t b = blockIdx.x;
    int lo = 0, hi = nsites - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (sites[mid].first_block <= b)
            lo = mid;
        else
            hi = mid - 1;
    }
    const ClaimSite S = sites[lo];
    const int64_t total = (int64_t)S.M * S.N;
    const int64_t e0 = (b - S.first_block) * CL_ELEMS;
    const int64_t e1 = min(total, e0 + CL_ELEMS);
    uint64_t acc = 0;
    for (int64_t e = e0 + threadIdx.x; e < e1; e += CL_THREADS) {
        int j, i;
        if (total < (1ll << 32)) {
            const uint32_t e32 = (uint32_t)e, m32 = (uint32_t)S.M;
            j = (int)(e32 / m32);
            i = (int)(e32 - (uint32_t)j * m32);
        } else {
            j = (int)(e / S.M);
            i = (int)(e - (int64_t)j * S.M);
        }
        const int64_t yv = ((int64_t)S.q[e] << S.k) + (int64_t)S.r[e];
        acc = gl_add(acc, gl_mul(gl_mul(S.eq_row[i], S.eq_col[j]), gl_from_i64(yv)));
    }
    acc = warp_sum_gl(acc);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x < 32) {
        uint64_t a = threadIdx.x < CL_THREADS / 32 ? red[threadIdx.x] : 0;
        a = warp_sum_gl(a);
        if (threadIdx.x == 0) part[b] = a;
    }
}

// out[s] = sum of part[first[s] .. first[s+1])
__global__ void segment_sum_kernel(const uint64_t* __restrict__ part, const int64_t* __restrict__ first,
                                   int nseg, uint64_t* __restrict__ out) {
    __shared__ uint64_t red[32];
    const int s = blockIdx.x;
    if (s >= nseg) return;
    uint64_t acc = 0;
    for (int64_t i = first[s] + threadIdx.x; i < first[s + 1]; i += blockDim.x) acc = gl_add(acc, part[i]);
    acc = warp_sum_gl(acc);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = acc;
    __syncthreads();
    if (threadIdx.x < 32) {
        uint64_t a = (threadIdx.x < (blockDim.x >> 5)) ? red[threadIdx.x] : 0;
        a = warp_sum_gl(a);
        if (threadIdx.x == 0) out[s] = a;
    }
}

}  // namespace

int fp_eq_table(fp_ctx* c, const FpPoint& z, uint64_t* out, cudaStream_t s) {
    uint64_t n = 1ull << z.v;
    int slot;
    fp_tic(c, s, K_EQ_BUILD, 8.0 * n, &slot);
    eq_build_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(z, out, n);
    fp_toc(c, s, slot);
    FP_CUDA(c, cudaGetLastError());
    return FP_OK;
}

// row splits of the partial evaluation: about two waves of blocks, every
// split short enough for the exact 64-bit column sums
static int pr_rows_per_split(int num_sms, int rows, int cols) {
    int col_blocks = (cols + PR_THREADS * PR_COLS - 1) / (PR_THREADS * PR_COLS);
    int want_splits = (2 * num_sms * 4 + col_blocks - 1) / col_blocks;
    int rps = (rows + want_splits - 1) / want_splits;
    if (rps < 64) rps = 64;
    if (rps > PR_ROWS_PER_SPLIT_MAX) rps = PR_ROWS_PER_SPLIT_MAX;
    return rps;
}

size_t fp_partial_rows_scratch(const fp_ctx* c, int rows, int cols) {
    int rps = pr_rows_per_split(c->num_sms, rows, cols);
    int splits = (rows + rps - 1) / rps;
    return fp_align_up((size_t)8 * splits * cols, 256) + 512;
}

int fp_partial_rows(fp_ctx* c, const void* mat, int bits, const int8_t* scales, int rows, int cols,
                    const uint64_t* eq, uint64_t* out, int64_t out_len, cudaStream_t s) {
    const bool w4 = bits == 4, sc = scales != nullptr;
    const int64_t pitch = w4 ? (cols + 1) / 2 : cols;
    const int col_blocks = (cols + PR_THREADS * PR_COLS - 1) / (PR_THREADS * PR_COLS);
    const int rps = pr_rows_per_split(c->num_sms, rows, cols);
    const int splits = (rows + rps - 1) / rps;
    uint64_t* part = (uint64_t*)fp_alloc(c->dev, (size_t)8 * splits * cols);
    uint64_t* esum = (uint64_t*)fp_alloc(c->dev, 256);
    if (!part || !esum) return fp_fail(c, FP_ERR_OOM, "partial evaluation: scratch exhausted");
    const bool al = ((uintptr_t)mat % 16 == 0) && (cols % PR_COLS == 0) && (w4 ? (pitch % 8 == 0) : (pitch % 16 == 0));
    dim3 grid(col_blocks, splits);
    double bytes = (double)rows * pitch + (sc ? (double)rows * ((cols + 63) / 64) : 0.0) + 8.0 * rows;
    int slot;
    fp_tic(c, s, K_PARTIAL_ACC, bytes, &slot);
#define PR_LAUNCH(A, B, C)                                                                                    \
    partial_acc_kernel<A, B, C><<<grid, PR_THREADS, 0, s>>>((const uint8_t*)mat, scales, rows, cols, pitch, eq, \
                                                            rps, part)
    if (w4) {
        if (sc) {
            if (al) PR_LAUNCH(true, true, true); else PR_LAUNCH(true, true, false);
        } else {
            if (al) PR_LAUNCH(true, false, true); else PR_LAUNCH(true, false, false);
        }
    } else {
        if (sc) {
            if (al) PR_LAUNCH(false, true, true); else PR_LAUNCH(false, true, false);
        } else {
            if (al) PR_LAUNCH(false, false, true); else PR_LAUNCH(false, false, false);
        }
    }
#undef PR_LAUNCH
    fp_toc(c, s, slot);
    FP_CUDA(c, cudaGetLastError());
    fp_tic(c, s, K_REDUCE, 8.0 * rows, &slot);
    sum_kernel<<<1, 1024, 0, s>>>(eq, (uint64_t)rows, esum);
    fp_toc(c, s, slot);
    FP_CUDA(c, cudaGetLastError());
    const int64_t cols_pad = out_len;
    const uint64_t off = sc ? (w4 ? 1024u : 16384u) : (w4 ? 8u : 128u);
    fp_tic(c, s, K_PARTIAL_FIN, 8.0 * splits * cols + 8.0 * cols_pad, &slot);
    partial_fin_kernel<<<(unsigned)((cols_pad + 255) / 256), 256, 0, s>>>(part, splits, cols, cols_pad, esum, off,
                                                                          out);
    fp_toc(c, s, slot);
    FP_CUDA(c, cudaGetLastError());
    return FP_OK;
}

size_t fp_claims_scratch(const fp_site* sites, int nsites) {
    int64_t blocks = 0;
    for (int s = 0; s < nsites; s++) blocks += ((int64_t)sites[s].M * sites[s].N + CL_ELEMS - 1) / CL_ELEMS;
    return fp_align_up(sizeof(ClaimSite) * nsites, 256) + fp_align_up(8 * (size_t)(nsites + 1), 256) +
           fp_align_up(8 * (size_t)blocks, 256) + 1024;
}

int fp_claims(fp_ctx* c, const fp_site* sites, int nsites, const uint64_t* const* eq_rows,
              const uint64_t* const* eq_cols, uint64_t* dev_out, cudaStream_t s) {
    std::vector<ClaimSite> h(nsites);
    std::vector<int64_t> first(nsites + 1);
    int64_t blocks = 0;
    double bytes = 0;
    for (int i = 0; i < nsites; i++) {
        h[i].q = sites[i].q;
        h[i].r = sites[i].r;
        h[i].eq_row = eq_rows[i];
        h[i].eq_col = eq_cols[i];
        h[i].M = sites[i].M;
        h[i].N = sites[i].N;
        h[i].k = sites[i].k_shift;
        h[i].pad = 0;
        h[i].first_block = blocks;
        first[i] = blocks;
        blocks += ((int64_t)sites[i].M * sites[i].N + CL_ELEMS - 1) / CL_ELEMS;
        bytes += 8.0 * sites[i].M * sites[i].N;
    }
    first[nsites] = blocks;
    size_t szs = sizeof(ClaimSite) * nsites, szf = 8 * (size_t)(nsites + 1);
    ClaimSite* dsites = (ClaimSite*)fp_alloc(c->dev, szs);
    int64_t* dfirst = (int64_t*)fp_alloc(c->dev, szf);
    uint64_t* part = (uint64_t*)fp_alloc(c->dev, 8 * (size_t)blocks);
    char* hs = (char*)fp_alloc(c->host, szs + szf);
    if (!dsites || !dfirst || !part || !hs) return fp_fail(c, FP_ERR_OOM, "claims: scratch exhausted");
    memcpy(hs, h.data(), szs);
    memcpy(hs + szs, first.data(), szf);
    FP_CUDA(c, cudaMemcpyAsync(dsites, hs, szs, cudaMemcpyHostToDevice, s));
    FP_CUDA(c, cudaMemcpyAsync(dfirst, hs + szs, szf, cudaMemcpyHostToDevice, s));
    int slot;
    fp_tic(c, s, K_CLAIM, bytes, &slot);
    claim_kernel<<<(unsigned)blocks, CL_THREADS, 0, s>>>(dsites, nsites, part);
    fp_toc(c, s, slot);
    FP_CUDA(c, cudaGetLastError());
    fp_tic(c, s, K_REDUCE, 8.0 * blocks, &slot);
    segment_sum_kernel<<<nsites, 256, 0, s>>>(part, dfirst, nsites, dev_out);
    fp_toc(c, s, slot);
    FP_CUDA(c, cudaGetLastError());
    return FP_OK;
}
