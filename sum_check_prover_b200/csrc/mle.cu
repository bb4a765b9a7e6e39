// Multilinear-extension kernels: eq tables and the per-site output claims of
// the matmul sum-check (the claim c_s is the MLE of 2^k q + r, the committed
// stand-in for the unrounded product, at (r_row, r_col): "How fast can
// FlashProve go", 3.1).
#include <vector>

#include "fp_field.cuh"
#include "fp_internal.h"

namespace {


__global__ void eq_build_kernel(FpPoint z, uint64_t* out, uint64_t n) {
    uint64_t x = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (x >= n) return;
    uint64_t e = 1;
    for (int b = 0; b < z.v; b++) e = gl_mul(e, gl_eq1(z.z[b], (int)((x >> (z.v - 1 - b)) & 1)));
    out[x] = e;
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
