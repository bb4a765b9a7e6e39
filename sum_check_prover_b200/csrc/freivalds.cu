// Freivalds' check of a weight matmul: the prover's side.
//
// "Towards Proving Frontier-Scale LLM Inference", The proof system: the matmuls
// with the weights are checked by Freivalds' algorithm, the verifier testing
// A (B r) = C r for a random vector r instead of recomputing C = A B. For one
// site Y = W_eff X with the committed witness Y = 2^k q + r:
//   absorb "frv_site" D(W) || D(S) || D(Xt) || D(q) || D(r); squeeze rho
//   ("frv_rho"); send u = X rho^(.) ("frv_u", K values), u_k = sum_j X[k][j] rho^j.
// The verifier checks u against X and W_eff u = Y rho^(.) row by row. It is the
// comparison statement for the sum-check of the same matmul: this prover reads
// only the activations (N K bytes), the verifier reads the weights.
//
// Kernels: the powers rho^j (one exponentiation each), then the row contraction of
// Xt (N x K int8) with them, which is the partial evaluation's contraction with the
// powers as its row weights (the tensor-core byte-limb kernel: Xt streamed once by
// TMA, the weights split into byte limbs).
#include <string.h>

#include <algorithm>

#include "fp_internal.h"

namespace {

__global__ void frv_pow_kernel(uint64_t rho, int64_t n, uint64_t* __restrict__ pw) {
    for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < n; j += (int64_t)gridDim.x * blockDim.x)
        pw[j] = gl_pow(rho, (uint64_t)j);
}

}  // namespace

int freivalds_prove_matmul(fp_ctx* c, fp_tx* tx, const fp_site* site, uint8_t* proof, size_t* proof_len,
                           void* stream) {
    if (!c || !tx || !proof_len || !site) return fp_fail(c, FP_ERR_ARG, "freivalds_prove_matmul: null argument");
    int rc;
    if ((rc = fp_check_sites(c, site, 1, true))) return rc;
    const fp_site& s = *site;
    const size_t need_len = 8 * (size_t)s.K;
    if (!proof || *proof_len < need_len) {
        *proof_len = need_len;
        return fp_fail(c, FP_ERR_ARG, "freivalds_prove_matmul: proof buffer too small");
    }
    FP_CUDA(c, cudaSetDevice(c->device));
    cudaStream_t st = (cudaStream_t)stream;
    {
        uint8_t d[160];
        if ((rc = fp_site_digest160(c, s, d, st))) return rc;
        fp_tx_absorb_raw(tx, "frv_site", d, 160);
    }
    const uint64_t rho = fp_tx_squeeze_one(tx, "frv_rho");
    // u = sum_j rho^j Xt[j][.]: the row contraction of Xt with the powers as row weights
    FpPeJob job{s.xt, 8, nullptr, s.N, s.K, nullptr, 0, nullptr, (int64_t)s.K};
    const size_t need = fp_align_up((size_t)8 * s.N, 256) + fp_align_up((size_t)8 * s.K, 256) +
                        fp_partial_scratch(c, &job, 1) + 4096;
    if ((rc = fp_reserve(c, c->dev, need))) return rc;
    if ((rc = fp_reserve(c, c->host, fp_align_up((size_t)8 * s.K, 256) + fp_partial_host_scratch(&job, 1) + 4096)))
        return rc;
    fp_reset(c->dev);
    fp_reset(c->host);
    uint64_t* pw = (uint64_t*)fp_alloc(c->dev, (size_t)8 * s.N);
    uint64_t* u = (uint64_t*)fp_alloc(c->dev, (size_t)8 * s.K);
    uint64_t* hu = (uint64_t*)fp_alloc(c->host, (size_t)8 * s.K);
    if (!pw || !u || !hu) return fp_fail(c, FP_ERR_OOM, "freivalds_prove_matmul: scratch exhausted");
    job.out = u;
    job.wts = pw;
    int slot;
    fp_tic(c, st, K_FRV_U, (double)s.N * s.K + 8.0 * s.K, &slot);
    frv_pow_kernel<<<fp_grid256(c, s.N), 256, 0, st>>>(rho, s.N, pw);
    FP_CUDA(c, cudaGetLastError());
    if ((rc = fp_partial_many(c, &job, 1, st))) return rc;
    fp_toc(c, st, slot);  // the powers and the contraction's launches under one slot
    FP_CUDA(c, cudaMemcpyAsync(hu, u, (size_t)8 * s.K, cudaMemcpyDeviceToHost, st));
    FP_CUDA(c, cudaStreamSynchronize(st));
    put_u64s(proof, hu, (size_t)s.K);
    fp_tx_absorb_raw(tx, "frv_u", proof, 8 * (uint64_t)s.K);
    *proof_len = need_len;
    return FP_OK;
}
