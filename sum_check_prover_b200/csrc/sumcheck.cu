// Matmul sum-check with claims batched by a random linear combination
// ("How fast can FlashProve go", 2 Background: sum-check reduces each
// polynomial operation to claims on committed values and weights; 2 and 2.1:
// claims are merged into one).
//
// Statement per site s: sum_k A_s[k] B_s[k] = c_s with A_s = W~_s(r_row, .),
// B_s = X~_s(., r_col), c_s = MLE of 2^k q + r at (r_row, r_col) ("How fast
// can FlashProve go", 3.1: 2^k g + r stands in for the unrounded product).
// The batched claim sum_s rho_s c_s is proven in n = max ceil(log2 K_s)
// rounds of the degree-2 polynomial g(X) = sum_s rho_s sum_b A_s(X,b) B_s(X,b).
//
// One kernel per round: it folds the previous round's vectors by the
// previous challenge (MSB binding) and evaluates g at 0, 1, 2 in the same
// pass; warp shuffles + a block tree + the last block finish the sums.
#include <string.h>

#include <map>
#include <vector>

#include "fp_internal.h"
#include "fp_reduce.cuh"

namespace {

constexpr int SC_THREADS = 256;

// Round t of the matmul sum-check over `nsites` site vectors of current length
// 2*half. FOLD: the inputs have length 4*half per site (round t-1's vectors)
// and are folded by rprev first, the folded halves being written to out.
template <bool FOLD, bool MULTI>
__global__ void __launch_bounds__(SC_THREADS)
    sc_round_kernel(const uint64_t* __restrict__ Ain, const uint64_t* __restrict__ Bin, uint64_t* __restrict__ Aout,
                    uint64_t* __restrict__ Bout, int64_t half, int logh, int64_t npairs, uint64_t rprev,
                    const uint64_t* __restrict__ rho, uint64_t* part, unsigned int* ticket,
                    uint64_t* __restrict__ gout) {
    uint64_t acc[3] = {0, 0, 0};
    for (int64_t p = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; p < npairs; p += (int64_t)gridDim.x * blockDim.x) {
        const int64_t s = p >> logh, b = p & (half - 1);
        uint64_t a0, a1, b0, b1;
        if (FOLD) {
            const int64_t bi = s * 4 * half + b;
            a0 = gl_fold(Ain[bi], Ain[bi + 2 * half], rprev);
            a1 = gl_fold(Ain[bi + half], Ain[bi + 3 * half], rprev);
            b0 = gl_fold(Bin[bi], Bin[bi + 2 * half], rprev);
            b1 = gl_fold(Bin[bi + half], Bin[bi + 3 * half], rprev);
            const int64_t bo = s * 2 * half + b;
            Aout[bo] = a0;
            Aout[bo + half] = a1;
            Bout[bo] = b0;
            Bout[bo + half] = b1;
        } else {
            const int64_t bi = s * 2 * half + b;
            a0 = Ain[bi];
            a1 = Ain[bi + half];
            b0 = Bin[bi];
            b1 = Bin[bi + half];
        }
        const uint64_t a2 = gl_sub(gl_add(a1, a1), a0);
        const uint64_t b2 = gl_sub(gl_add(b1, b1), b0);
        uint64_t t0 = gl_mul(a0, b0), t1 = gl_mul(a1, b1), t2 = gl_mul(a2, b2);
        if (MULTI) {
            const uint64_t rs = rho[s];
            t0 = gl_mul(t0, rs);
            t1 = gl_mul(t1, rs);
            t2 = gl_mul(t2, rs);
        }
        acc[0] = gl_add(acc[0], t0);
        acc[1] = gl_add(acc[1], t1);
        acc[2] = gl_add(acc[2], t2);
    }
    if (grid_sum_gl<3>(acc, part, ticket) && threadIdx.x == 0) {
        gout[0] = acc[0];
        gout[1] = acc[1];
        gout[2] = acc[2];
    }
}

// A_s(rho), B_s(rho): fold the length-2 vectors by the last challenge (len == 2),
// or copy them (n == 0, len == 1).
__global__ void sc_final_kernel(const uint64_t* A, const uint64_t* B, int nsites, int len, uint64_t r,
                                uint64_t* out) {
    int s = blockIdx.x * blockDim.x + threadIdx.x;
    if (s >= nsites) return;
    if (len == 2) {
        out[2 * s] = gl_fold(A[2 * s], A[2 * s + 1], r);
        out[2 * s + 1] = gl_fold(B[2 * s], B[2 * s + 1], r);
    } else {
        out[2 * s] = A[s];
        out[2 * s + 1] = B[s];
    }
}

void put_u64s(uint8_t* p, const uint64_t* v, size_t n) {
    for (size_t i = 0; i < n; i++)
        for (int b = 0; b < 8; b++) p[8 * i + b] = (uint8_t)(v[i] >> (8 * b));
}

}  // namespace

int sumcheck_prove_matmul(fp_ctx* c, fp_tx* tx, const fp_site* sites, int nsites, uint8_t* proof, size_t* proof_len,
                          void* stream) {
    if (!c || !tx || !proof_len) return fp_fail(c, FP_ERR_ARG, "sumcheck_prove_matmul: null argument");
    int rc = fp_check_sites(c, sites, nsites, true);
    if (rc) return rc;
    size_t mm_bytes, lu_bytes;
    fp_proof_size(sites, nsites, &mm_bytes, &lu_bytes);
    if (!proof || *proof_len < mm_bytes) {
        *proof_len = mm_bytes;
        return fp_fail(c, FP_ERR_ARG, "sumcheck_prove_matmul: proof buffer too small");
    }
    FP_CUDA(c, cudaSetDevice(c->device));
    cudaStream_t st = (cudaStream_t)stream;

    int vM = 0, vN = 0, n = 0;
    for (int s = 0; s < nsites; s++) {
        vM = std::max(vM, fp_log2_ceil((uint64_t)sites[s].M));
        vN = std::max(vN, fp_log2_ceil((uint64_t)sites[s].N));
        n = std::max(n, fp_log2_ceil((uint64_t)sites[s].K));
    }
    const int64_t L = 1ll << n;

    // ---- scratch ----
    std::map<int, uint64_t*> eqr, eqc;  // eq tables by prefix length
    size_t need = 0;
    std::map<int, int> lens_r, lens_c;
    for (int s = 0; s < nsites; s++) {
        lens_r[fp_log2_ceil((uint64_t)sites[s].M)] = 1;
        lens_c[fp_log2_ceil((uint64_t)sites[s].N)] = 1;
    }
    for (auto& kv : lens_r) need += fp_align_up((size_t)8 << kv.first, 256);
    for (auto& kv : lens_c) need += fp_align_up((size_t)8 << kv.first, 256);
    need += fp_claims_scratch(sites, nsites);
    const size_t vec = (size_t)8 * nsites * L;
    need += 4 * fp_align_up(vec, 256);
    size_t pr = 0;
    for (int s = 0; s < nsites; s++)
        pr = std::max(pr, std::max(fp_partial_rows_scratch(c, sites[s].M, sites[s].K),
                                   fp_partial_rows_scratch(c, sites[s].N, sites[s].K)));
    need += pr;
    const int max_blocks = 4 * c->num_sms;
    need += fp_align_up((size_t)8 * 3 * max_blocks, 256) + fp_align_up(8 * (size_t)nsites, 256) * 3 + (1 << 16);
    if ((rc = fp_reserve(c, c->dev, need))) return rc;
    if ((rc = fp_reserve(c, c->host, fp_align_up(sizeof(uint64_t) * (4 * (size_t)nsites + 64), 256) + 8192 +
                                         (size_t)160 * nsites)))
        return rc;
    fp_reset(c->dev);
    fp_reset(c->host);

    // ---- challenges for the output point ----
    FpPoint zr, zc;
    zr.v = vM;
    zc.v = vN;
    for (int i = 0; i < vM; i++) zr.z[i] = fp_tx_squeeze_one(tx, "r_row");
    for (int i = 0; i < vN; i++) zc.z[i] = fp_tx_squeeze_one(tx, "r_col");
    for (auto& kv : lens_r) {
        uint64_t* t = (uint64_t*)fp_alloc(c->dev, (size_t)8 << kv.first);
        FpPoint p = zr;
        p.v = kv.first;
        if ((rc = fp_eq_table(c, p, t, st))) return rc;
        eqr[kv.first] = t;
    }
    for (auto& kv : lens_c) {
        uint64_t* t = (uint64_t*)fp_alloc(c->dev, (size_t)8 << kv.first);
        FpPoint p = zc;
        p.v = kv.first;
        if ((rc = fp_eq_table(c, p, t, st))) return rc;
        eqc[kv.first] = t;
    }
    std::vector<const uint64_t*> er(nsites), ec(nsites);
    for (int s = 0; s < nsites; s++) {
        er[s] = eqr[fp_log2_ceil((uint64_t)sites[s].M)];
        ec[s] = eqc[fp_log2_ceil((uint64_t)sites[s].N)];
    }

    // ---- claims ----
    uint64_t* dclaims = (uint64_t*)fp_alloc(c->dev, 8 * (size_t)nsites);
    if ((rc = fp_claims(c, sites, nsites, er.data(), ec.data(), dclaims, st))) return rc;
    uint64_t* hbuf = (uint64_t*)fp_alloc(c->host, sizeof(uint64_t) * (4 * (size_t)nsites + 64));
    FP_CUDA(c, cudaMemcpyAsync(hbuf, dclaims, 8 * (size_t)nsites, cudaMemcpyDeviceToHost, st));
    FP_CUDA(c, cudaStreamSynchronize(st));
    size_t pos = 0;
    put_u64s(proof + pos, hbuf, nsites);
    fp_tx_absorb_raw(tx, "claims", proof + pos, 8 * (size_t)nsites);
    pos += 8 * (size_t)nsites;

    // ---- batching coefficients ----
    std::vector<uint64_t> rho(nsites, 1);
    if (nsites > 1)
        for (int s = 0; s < nsites; s++) rho[s] = fp_tx_squeeze_one(tx, "rho");
    uint64_t* drho = (uint64_t*)fp_alloc(c->dev, 8 * (size_t)nsites);
    uint64_t* hrho = (uint64_t*)fp_alloc(c->host, 8 * (size_t)nsites);
    memcpy(hrho, rho.data(), 8 * (size_t)nsites);
    FP_CUDA(c, cudaMemcpyAsync(drho, hrho, 8 * (size_t)nsites, cudaMemcpyHostToDevice, st));

    // ---- partial evaluations A_s = W~_s(r_row, .), B_s = X~_s(., r_col) ----
    uint64_t* bufA[2] = {(uint64_t*)fp_alloc(c->dev, vec), (uint64_t*)fp_alloc(c->dev, vec)};
    uint64_t* bufB[2] = {(uint64_t*)fp_alloc(c->dev, vec), (uint64_t*)fp_alloc(c->dev, vec)};
    const size_t mark = c->dev.top;
    for (int s = 0; s < nsites; s++) {
        c->dev.top = mark;  // partial-evaluation scratch is reused site after site
        if ((rc = fp_partial_rows(c, sites[s].w, sites[s].w_bits, sites[s].scales, sites[s].M, sites[s].K, er[s],
                                  bufA[0] + (size_t)s * L, L, st)))
            return rc;
        c->dev.top = mark;
        if ((rc = fp_partial_rows(c, sites[s].xt, 8, nullptr, sites[s].N, sites[s].K, ec[s],
                                  bufB[0] + (size_t)s * L, L, st)))
            return rc;
    }
    c->dev.top = mark + pr;
    uint64_t* part = (uint64_t*)fp_alloc(c->dev, (size_t)8 * 3 * max_blocks);
    uint64_t* dg = (uint64_t*)fp_alloc(c->dev, 64);
    uint64_t* dfin = (uint64_t*)fp_alloc(c->dev, 16 * (size_t)nsites);
    if (!bufA[1] || !bufB[1] || !part || !dg || !dfin) return fp_fail(c, FP_ERR_OOM, "sumcheck: scratch exhausted");

    // ---- rounds ----
    int cur = 0;
    uint64_t rprev = 0;
    for (int t = 1; t <= n; t++) {
        const int64_t half = 1ll << (n - t);
        const int64_t npairs = (int64_t)nsites * half;
        int blocks = (int)std::min<int64_t>(max_blocks, (npairs + SC_THREADS - 1) / SC_THREADS);
        const bool fold = t > 1;
        const int nxt = fold ? 1 - cur : cur;
        double bytes = fold ? 48.0 * npairs : 32.0 * npairs;
        int slot;
        fp_tic(c, st, K_SC_ROUND, bytes, &slot);
#define SC_LAUNCH(F, M)                                                                                    \
    sc_round_kernel<F, M><<<blocks, SC_THREADS, 0, st>>>(bufA[cur], bufB[cur], bufA[nxt], bufB[nxt], half, \
                                                         n - t, npairs, rprev, drho, part, c->tickets, dg)
        if (fold) {
            if (nsites > 1) SC_LAUNCH(true, true); else SC_LAUNCH(true, false);
        } else {
            if (nsites > 1) SC_LAUNCH(false, true); else SC_LAUNCH(false, false);
        }
#undef SC_LAUNCH
        fp_toc(c, st, slot);
        FP_CUDA(c, cudaGetLastError());
        cur = nxt;
        FP_CUDA(c, cudaMemcpyAsync(hbuf, dg, 24, cudaMemcpyDeviceToHost, st));
        FP_CUDA(c, cudaStreamSynchronize(st));
        put_u64s(proof + pos, hbuf, 3);
        fp_tx_absorb_raw(tx, "sc_round", proof + pos, 24);
        pos += 24;
        rprev = fp_tx_squeeze_one(tx, "sc_chal");
    }
    // ---- final evaluations ----
    int slot;
    fp_tic(c, st, K_SC_FINAL, 32.0 * nsites, &slot);
    sc_final_kernel<<<(nsites + 127) / 128, 128, 0, st>>>(bufA[cur], bufB[cur], nsites, n > 0 ? 2 : 1, rprev, dfin);
    fp_toc(c, st, slot);
    FP_CUDA(c, cudaGetLastError());
    FP_CUDA(c, cudaMemcpyAsync(hbuf, dfin, 16 * (size_t)nsites, cudaMemcpyDeviceToHost, st));
    FP_CUDA(c, cudaStreamSynchronize(st));
    put_u64s(proof + pos, hbuf, 2 * (size_t)nsites);
    fp_tx_absorb_raw(tx, "sc_final", proof + pos, 16 * (size_t)nsites);
    pos += 16 * (size_t)nsites;
    *proof_len = pos;
    return FP_OK;
}
