// MoE dispatch: the experts' inputs are the routed rows of the layer input.
//
// "How fast can FlashProve go", 2 Background (the note on MoE layers): the
// routing computation and the choice of expert are proven; the routing proof
// (route.cu) covers the choice, this statement the moving of every token's
// activations to its expert. With X the layer input (T x K int8, token-major),
// e_t the expert of token t and D the experts' inputs stacked expert by expert
// (each expert's tokens in token order), D = Pi X for the permutation sending
// token t to pos(t) = #{t' : e_t' < e_t} + #{t' < t : e_t' = e_t}, so
// D~(r, c) = sum_t eq(r, pos(t)) X~(t, c):
//   absorb "dsp_site" D(X) || D(e, int32) || D(D); squeeze r_row ("dsp_row",
//   vT coordinates) and r_col ("dsp_col", vK); send c = D~(r_row, r_col)
//   ("dsp_claim"); vT degree-2 rounds of sum_t P(t) B(t) with
//   P(t) = eq(r_row, pos(t)), B(t) = X~(t, r_col) ("dsp_round", "dsp_chal");
//   send P(rho), B(rho) ("dsp_final").
//
// Kernels: the claim through the partial evaluation (D's rows weighted by the
// eq table of r_row, then a dot product with the eq table of r_col); pos(t) by
// one block per expert (a count of the tokens of lower experts, then a stable
// scan of its own tokens) writing P(t); B(t) as a warp per row of X with exact
// 64 x 32-bit sums; the rounds on the matmul sum-check's kernel.
#include <string.h>

#include <algorithm>

#include "fp_internal.h"
#include "fp_reduce.cuh"

namespace {

constexpr int DSP_THREADS = 256;

// Block x handles expert x: pos(t) for its tokens and P(t) = eq_row[pos(t)]. A token whose
// expert lies outside [0, E) is counted in *bad.
__global__ void __launch_bounds__(DSP_THREADS) dsp_pos_kernel(const int32_t* __restrict__ e, int64_t T, int E,
                                                              const uint64_t* __restrict__ eq_row,
                                                              uint64_t* __restrict__ P, uint32_t* __restrict__ bad) {
    __shared__ uint32_t wcnt[DSP_THREADS / 32];
    __shared__ uint64_t s_base;
    const int x = blockIdx.x, lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // tokens of lower experts
    uint64_t below = 0;
    for (int64_t t = threadIdx.x; t < T; t += DSP_THREADS) {
        const int32_t v = e[t];
        below += (v >= 0 && v < x) ? 1 : 0;
        if (x == 0 && (v < 0 || v >= E)) atomicAdd(bad, 1u);
    }
    for (int o = 16; o > 0; o >>= 1) below += __shfl_xor_sync(0xffffffffu, below, o);
    if (threadIdx.x == 0) s_base = 0;
    __syncthreads();
    if (lane == 0) atomicAdd((unsigned long long*)&s_base, (unsigned long long)below);
    __syncthreads();
    uint64_t run = s_base;
    // a stable scan of the block's tokens, 256 at a time
    for (int64_t t0 = 0; t0 < T; t0 += DSP_THREADS) {
        const int64_t t = t0 + threadIdx.x;
        const bool mine = t < T && e[t] == x;
        const unsigned bal = __ballot_sync(0xffffffffu, mine);
        if (lane == 0) wcnt[warp] = (uint32_t)__popc(bal);
        __syncthreads();
        uint64_t before = run;
        for (int w = 0; w < warp; w++) before += wcnt[w];
        before += (uint64_t)__popc(bal & ((1u << lane) - 1u));
        if (mine) P[t] = __ldg(eq_row + before);
        uint64_t tot = 0;
        for (int w = 0; w < DSP_THREADS / 32; w++) tot += wcnt[w];
        run += tot;
        __syncthreads();  // wcnt is rewritten by the next chunk
    }
}

// B(t) = sum_k eq_col[k] X[t][k] for t < T: a warp per row, exact sums of eq_col (x + 128), the
// offset removed with the sum of eq_col over k < K (ecsum)
__global__ void __launch_bounds__(DSP_THREADS) dsp_rowdot_kernel(const int8_t* __restrict__ X, int64_t T, int64_t K,
                                                                 const uint64_t* __restrict__ eq_col, uint64_t ecsum,
                                                                 uint64_t* __restrict__ B) {
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (DSP_THREADS / 32);
    for (int64_t t = (int64_t)blockIdx.x * (DSP_THREADS / 32) + (threadIdx.x >> 5); t < T; t += warps) {
        GlAcc a;
        const int8_t* row = X + t * K;
        for (int64_t k = lane; k < K; k += 32) a.mac32(__ldg(eq_col + k), (uint32_t)((int32_t)row[k] + 128));
        uint64_t v = a.value();
        v = warp_sum_gl(v);
        if (lane == 0) B[t] = gl_sub(v, gl_mul(128, ecsum));
    }
}

// out[0] = sum_k a[k] b[k] over n entries, out[1] = sum_k b[k] (one block)
__global__ void __launch_bounds__(DSP_THREADS) dsp_dot_kernel(const uint64_t* __restrict__ a,
                                                              const uint64_t* __restrict__ b, int64_t n, int64_t nb,
                                                              uint64_t* __restrict__ out) {
    GlAcc s, sb;
    for (int64_t k = threadIdx.x; k < n; k += DSP_THREADS) s.mac(a[k], b[k]);
    for (int64_t k = threadIdx.x; k < nb; k += DSP_THREADS) sb.add(b[k]);
    uint64_t v[2] = {s.value(), sb.value()};
    block_sum_gl<2>(v);
    if (threadIdx.x == 0) {
        out[0] = v[0];
        out[1] = v[1];
    }
}

size_t dsp_proof_len(int vT) { return 8 + 24 * (size_t)vT + 16; }

}  // namespace

int sumcheck_prove_dispatch(fp_ctx* c, fp_tx* tx, const int8_t* X, const int32_t* e, const int8_t* D, int64_t T,
                            int64_t K, int E, uint8_t* proof, size_t* proof_len, void* stream) {
    if (!c || !tx || !X || !e || !D || !proof_len) return fp_fail(c, FP_ERR_ARG, "sumcheck_prove_dispatch: null argument");
    if (T < 1 || K < 1 || E < 1 || T > (1ll << 24) || K > (1ll << 24) || E > (1 << 20))
        return fp_fail(c, FP_ERR_SHAPE, "sumcheck_prove_dispatch: need 1 <= T, K <= 2^24 and 1 <= E <= 2^20");
    const int vT = fp_log2_ceil((uint64_t)T), vK = fp_log2_ceil((uint64_t)K);
    const size_t need_len = dsp_proof_len(vT);
    if (!proof || *proof_len < need_len) {
        *proof_len = need_len;
        return fp_fail(c, FP_ERR_ARG, "sumcheck_prove_dispatch: proof buffer too small");
    }
    FP_CUDA(c, cudaSetDevice(c->device));
    cudaStream_t st = (cudaStream_t)stream;
    const int64_t LT = 1ll << vT, LK = 1ll << vK;
    FpPeJob job{D, 8, nullptr, (int)T, (int)K, nullptr, 0, nullptr, LK};
    size_t need = fp_align_up((size_t)8 * LT, 256) * 3 + fp_align_up((size_t)8 * LK, 256) * 2 +
                  fp_partial_scratch(c, &job, 1) + fp_two_vector_scratch(c, vT) + 4096;
    int rc;
    if ((rc = fp_reserve(c, c->dev, need))) return rc;
    if ((rc = fp_reserve(c, c->host, fp_partial_host_scratch(&job, 1) + fp_two_vector_host_scratch() + 4096))) return rc;
    fp_reset(c->dev);
    fp_reset(c->host);
    uint64_t* erow = (uint64_t*)fp_alloc(c->dev, (size_t)8 * LT);
    uint64_t* ecol = (uint64_t*)fp_alloc(c->dev, (size_t)8 * LK);
    uint64_t* Ad = (uint64_t*)fp_alloc(c->dev, (size_t)8 * LK);
    uint64_t* P = (uint64_t*)fp_alloc(c->dev, (size_t)8 * LT);
    uint64_t* B = (uint64_t*)fp_alloc(c->dev, (size_t)8 * LT);
    uint64_t* small = (uint64_t*)fp_alloc(c->dev, 256);
    uint64_t* hs = (uint64_t*)fp_alloc(c->host, 256);
    if (!erow || !ecol || !Ad || !P || !B || !small || !hs)
        return fp_fail(c, FP_ERR_OOM, "sumcheck_prove_dispatch: scratch exhausted");

    // ---- the statement's digests ----
    {
        FpDigestJob jobs[3] = {{(const uint8_t*)X, (uint64_t)(T * K)}, {(const uint8_t*)e, 4 * (uint64_t)T},
                               {(const uint8_t*)D, (uint64_t)(T * K)}};
        uint8_t d[96];
        if ((rc = fp_digest_many(c, jobs, 3, d, st))) return rc;  // synchronises the stream
        fp_tx_absorb_raw(tx, "dsp_site", d, 96);
    }
    FpPoint zr, zc;
    zr.v = vT;
    zc.v = vK;
    for (int i = 0; i < vT; i++) zr.z[i] = fp_tx_squeeze_one(tx, "dsp_row");
    for (int i = 0; i < vK; i++) zc.z[i] = fp_tx_squeeze_one(tx, "dsp_col");
    if ((rc = fp_eq_table(c, zr, erow, st))) return rc;
    if ((rc = fp_eq_table(c, zc, ecol, st))) return rc;

    // ---- claim: D's rows weighted by eq(r_row, .), dotted with eq(r_col, .) ----
    job.out = Ad;
    job.wts = erow;
    int slot;
    fp_tic(c, st, K_DSP_CLAIM, (double)T * K, &slot);
    if ((rc = fp_partial_many(c, &job, 1, st))) return rc;
    dsp_dot_kernel<<<1, DSP_THREADS, 0, st>>>(Ad, ecol, K, K, small);
    fp_toc(c, st, slot);
    FP_CUDA(c, cudaGetLastError());

    // ---- the vectors: P(t) = eq(r_row, pos(t)), B(t) = X~(t, r_col); zero past T ----
    FP_CUDA(c, cudaMemsetAsync(P, 0, (size_t)8 * LT, st));
    FP_CUDA(c, cudaMemsetAsync(B, 0, (size_t)8 * LT, st));
    FP_CUDA(c, cudaMemsetAsync(small + 8, 0, 8, st));
    FP_CUDA(c, cudaMemcpyAsync(hs, small, 16, cudaMemcpyDeviceToHost, st));
    FP_CUDA(c, cudaStreamSynchronize(st));
    const uint64_t claim = hs[0], ecsum = hs[1];
    fp_tic(c, st, K_DSP_VECTORS, 4.0 * T + (double)T * K + 16.0 * T, &slot);
    dsp_pos_kernel<<<E, DSP_THREADS, 0, st>>>(e, T, E, erow, P, (uint32_t*)(small + 8));
    const unsigned rgrid = (unsigned)std::max<int64_t>(1, std::min<int64_t>((T + 7) / 8, 8ll * c->num_sms));
    dsp_rowdot_kernel<<<rgrid, DSP_THREADS, 0, st>>>(X, T, K, ecol, ecsum, B);
    fp_toc(c, st, slot);
    FP_CUDA(c, cudaGetLastError());
    c->launches++;  // two kernels under one slot
    FP_CUDA(c, cudaMemcpyAsync(hs + 2, small + 8, 8, cudaMemcpyDeviceToHost, st));
    FP_CUDA(c, cudaStreamSynchronize(st));
    if ((uint32_t)hs[2] != 0) return fp_fail(c, FP_ERR_ARG, "sumcheck_prove_dispatch: an expert index outside [0, E)");

    size_t pos = 0;
    put_u64s(proof + pos, &claim, 1);
    fp_tx_absorb_raw(tx, "dsp_claim", proof + pos, 8);
    pos += 8;
    uint64_t fin[2];
    if ((rc = fp_two_vector_sumcheck(c, tx, P, B, vT, claim, "dsp_round", "dsp_chal", proof, &pos, fin, st))) return rc;
    put_u64s(proof + pos, fin, 2);
    fp_tx_absorb_raw(tx, "dsp_final", proof + pos, 16);
    pos += 16;
    *proof_len = pos;
    return FP_OK;
}
