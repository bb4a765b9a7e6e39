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
// three blocks per SM (80 registers): the claim waits on memory latency, and two blocks of 90
// registers left it at a quarter of the warps (MoE layer with 32 experts: 0.313 -> 0.239 ms)
#ifndef FP_CLAIM_MIN_BLOCKS
#define FP_CLAIM_MIN_BLOCKS 3
#endif
constexpr int CL_ELEMS = 32768;  // flat elements per block (128 per thread: the block's set-up is amortised)

__global__ void __launch_bounds__(CL_THREADS, FP_CLAIM_MIN_BLOCKS)
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
    // Row j of the N x M output is contiguous: sum_i eq_row[i] (2^k q + r) over a thread's
    // elements of row j is kept exactly (q + 2^31 and r + 2^31 as 32-bit factors, the offsets
    // removed with the sum of the weights) and weighted by eq_col[j] once the thread leaves row j.
    GlAcc tot, aq, ar, es;
    int64_t e = e0 + threadIdx.x;
    int64_t j = e / S.M, i = e - j * S.M;
    int64_t jcur = j;
    const uint64_t k2 = 1ull << S.k;
    auto flush = [&]() {
        const uint64_t w = es.value();
        const uint64_t off = gl_mul(1ull << 31, w);
        const uint64_t vq = gl_sub(aq.value(), off), vr = gl_sub(ar.value(), off);
        tot.mac(__ldg(S.eq_col + jcur), gl_add(gl_mul(k2, vq), vr));
        aq = GlAcc();
        ar = GlAcc();
        es = GlAcc();
    };
    const bool vec = S.M % 4 == 0 && S.M >= 8 * CL_THREADS &&
                     (((uintptr_t)S.q | (uintptr_t)S.r | (uintptr_t)S.eq_row) & 15) == 0;
    if (vec) {
        // four consecutive elements (one row: M is a multiple of 4) per step, two steps' loads in
        // flight: thread t takes elements 4 t .. 4 t + 3 of every 4 CL_THREADS
        e = e0 + 4 * (int64_t)threadIdx.x;
        j = e / S.M;
        i = e - j * S.M;
        jcur = j;
        const bool any = e < e1;
        for (; e < e1; e += 8 * CL_THREADS) {
            const int64_t eb = e + 4 * CL_THREADS;
            int64_t jb = j, ib = i + 4 * CL_THREADS;
            if (ib >= S.M) {
                ib -= S.M;
                jb++;
            }
            const bool two = eb < e1;
            const int4 qa = __ldcs(reinterpret_cast<const int4*>(S.q + e));
            const int4 ra = __ldcs(reinterpret_cast<const int4*>(S.r + e));
            const ulonglong2 wa0 = __ldg(reinterpret_cast<const ulonglong2*>(S.eq_row + i));
            const ulonglong2 wa1 = __ldg(reinterpret_cast<const ulonglong2*>(S.eq_row + i + 2));
            int4 qb = make_int4(0, 0, 0, 0), rb = qb;
            ulonglong2 wb0 = make_ulonglong2(0, 0), wb1 = wb0;
            if (two) {
                qb = __ldcs(reinterpret_cast<const int4*>(S.q + eb));
                rb = __ldcs(reinterpret_cast<const int4*>(S.r + eb));
                wb0 = __ldg(reinterpret_cast<const ulonglong2*>(S.eq_row + ib));
                wb1 = __ldg(reinterpret_cast<const ulonglong2*>(S.eq_row + ib + 2));
            }
            if (j != jcur) {
                flush();
                jcur = j;
            }
            aq.mac32(wa0.x, (uint32_t)qa.x ^ 0x80000000u);
            aq.mac32(wa0.y, (uint32_t)qa.y ^ 0x80000000u);
            aq.mac32(wa1.x, (uint32_t)qa.z ^ 0x80000000u);
            aq.mac32(wa1.y, (uint32_t)qa.w ^ 0x80000000u);
            ar.mac32(wa0.x, (uint32_t)ra.x ^ 0x80000000u);
            ar.mac32(wa0.y, (uint32_t)ra.y ^ 0x80000000u);
            ar.mac32(wa1.x, (uint32_t)ra.z ^ 0x80000000u);
            ar.mac32(wa1.y, (uint32_t)ra.w ^ 0x80000000u);
            es.add(wa0.x);
            es.add(wa0.y);
            es.add(wa1.x);
            es.add(wa1.y);
            if (two) {
                if (jb != jcur) {
                    flush();
                    jcur = jb;
                }
                aq.mac32(wb0.x, (uint32_t)qb.x ^ 0x80000000u);
                aq.mac32(wb0.y, (uint32_t)qb.y ^ 0x80000000u);
                aq.mac32(wb1.x, (uint32_t)qb.z ^ 0x80000000u);
                aq.mac32(wb1.y, (uint32_t)qb.w ^ 0x80000000u);
                ar.mac32(wb0.x, (uint32_t)rb.x ^ 0x80000000u);
                ar.mac32(wb0.y, (uint32_t)rb.y ^ 0x80000000u);
                ar.mac32(wb1.x, (uint32_t)rb.z ^ 0x80000000u);
                ar.mac32(wb1.y, (uint32_t)rb.w ^ 0x80000000u);
                es.add(wb0.x);
                es.add(wb0.y);
                es.add(wb1.x);
                es.add(wb1.y);
            }
            j = jb;
            i = ib + 4 * CL_THREADS;
            while (i >= S.M) {
                i -= S.M;
                j++;
            }
        }
        if (any) flush();
        e = e1;  // the scalar loop below has nothing left
    }
    for (; e < e1; e += CL_THREADS) {
        if (j != jcur) {
            flush();
            jcur = j;
        }
        const uint64_t w = __ldg(S.eq_row + i);
        aq.mac32(w, (uint32_t)S.q[e] ^ 0x80000000u);
        ar.mac32(w, (uint32_t)S.r[e] ^ 0x80000000u);
        es.add(w);
        i += CL_THREADS;
        if (i >= S.M) {
            if (S.M >= CL_THREADS) {
                i -= S.M;
                j++;
            } else {
                j += i / S.M;
                i %= S.M;
            }
        }
    }
    if (!vec && e0 + threadIdx.x < e1) flush();
    uint64_t acc = tot.value();
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
