// Product sum-checks for products that are never committed: the gated product
// h = s (.) u and the per-group scaled weights W_eff = S (.) w.
//
// "How fast can FlashProve go", 3.1 Committing intermediate values: the MLP's
// gated product is a plain product, so the prover never commits to it; a
// sum-check reduces a claim on its MLE to claims on the committed factors. The
// grouped-scale weights of the FFN are the same kind of product (the scales and
// the int4 weights are committed, their product is not), reduced the same way.
// Both run the degree-3 sum-check of eq(z, .) s u over v variables:
//   send c = sum_x eq(z, x) s(x) u(x) ("<p>_claim");
//   round t = 1..v: send g_t(0..3) ("<p>_round"); squeeze rho_t ("<p>_chal");
//   send s~(rho), u~(rho) ("<p>_final"),
// with p = "had" (absorb "had_site" D(s) || D(u), squeeze z: sumcheck_prove_hadamard)
// or p = "scl" (absorb "scl_site" D(W) || D(S), z from the caller:
// sumcheck_reduce_scales, factors Se(i, k) = S[i][k >> 6] and w(i, k), row bits first).
//
// g_t(X) = eq(z_<t, rho_<t) eq(z_t, X) h_t(X) with h_t(X) =
// sum_b eq(z_>t, b) s(X, b) u(X, b) over the factors folded by rho_<t; h_t has
// degree 2, so the device returns h_t(0), h_t(1), h_t(2) and the host forms the
// four values of g_t (h_t(3) = h_t(0) - 3 h_t(1) + 3 h_t(2)). g_t(0) + g_t(1)
// must equal the running claim; the host checks it on every round.
//
// All rounds run in one resident cooperative launch (the handshake of
// fp_session.cuh). Round 1 reads the factors as small integers and writes the
// suffix eq table E[b] = eq(z_>1, b); round 2 folds them by rho_1 into field
// vectors; later rounds fold those in place (each thread owns positions b,
// b + h, b + 2h, b + 3h) and sum E in place. One pair per thread per pass.
#include <string.h>

#include <algorithm>

#include "fp_eqchunks.cuh"
#include "fp_internal.h"
#include "fp_reduce.cuh"
#include "fp_session.cuh"

namespace {

constexpr int HAD_THREADS = 256;
constexpr int HAD_MAX_V = 30;

// the gated product's factors: two int8 vectors of n entries, zero-padded
struct HadSrc {
    const int8_t* s;
    const int8_t* u;
    int64_t n;
    __device__ __forceinline__ int s_at(int64_t x) const { return x < n ? (int)s[x] : 0; }
    __device__ __forceinline__ int u_at(int64_t x) const { return x < n ? (int)u[x] : 0; }
};

// the scaled weights' factors over x = i 2^vK + k: Se(i, k) = S[i][k >> 6] (zero past the
// M x G scales) and w(i, k) (int4: two per byte, low nibble = even k; zero past M x K)
struct SclSrc {
    const uint8_t* w;
    const int8_t* sc;
    int64_t pitch;  // bytes per weight row
    int M, K, G, vK, bits;
    __device__ __forceinline__ int s_at(int64_t x) const {
        const int64_t i = x >> vK, g = (x & ((1ll << vK) - 1)) >> 6;
        return (i < M && g < G) ? (int)sc[i * G + g] : 0;
    }
    __device__ __forceinline__ int u_at(int64_t x) const {
        const int64_t i = x >> vK, k = x & ((1ll << vK) - 1);
        if (i >= M || k >= K) return 0;
        if (bits == 8) return (int)(int8_t)w[i * pitch + k];
        const int b = w[i * pitch + (k >> 1)];
        const int nib = (k & 1) ? (b >> 4) : (b & 15);
        return nib >= 8 ? nib - 16 : nib;
    }
};

template <class Src>
struct ProdArgs {
    Src src;
    uint64_t* S;  // folded factors from round 2 on (2^(v-1) entries each)
    uint64_t* U;
    uint64_t* E;  // suffix eq table (2^(v-1) entries)
    const uint64_t* z;  // device copy of z_1..z_v
    int v;
    int grid;
    int per_block;
    int pad;
    uint64_t seq0;  // round t publishes seq0 + t, the final values seq0 + v + 1
    int t_begin;    // rounds run by this launch: [t_begin, t_end]; t_end > v includes the final values
    int t_end;
};

// a small signed integer as a field element
__device__ __forceinline__ uint64_t lifti(int x) { return x < 0 ? GL_P - (uint64_t)(-(int64_t)x) : (uint64_t)x; }

// X = 2 on the line through (a, b) at 0 and 1
__device__ __forceinline__ uint64_t at2(uint64_t a, uint64_t b) { return gl_sub(gl_add(b, b), a); }

// c = sum_{x < len} eq(z, x) s(x) u(x), eq split as EH[x >> vl] EL[x & (2^vl - 1)]; the factors'
// product is a small integer (|s u| <= 2^14)
template <class Src>
__global__ void __launch_bounds__(256) prod_claim_kernel(Src src, int64_t len, const uint64_t* __restrict__ EH,
                                                         const uint64_t* __restrict__ EL, int vl, uint64_t* part,
                                                         unsigned int* ticket, uint64_t* out) {
    GlAcc acc;
    const int64_t mask = (1ll << vl) - 1;
    for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < len; x += (int64_t)gridDim.x * blockDim.x) {
        const int p = src.s_at(x) * src.u_at(x);
        if (p == 0) continue;
        const uint64_t e = gl_mul(__ldg(EH + (x >> vl)), __ldg(EL + (x & mask)));
        acc.mac(e, lifti(p));
    }
    uint64_t v[1] = {acc.value()};
    if (grid_sum_gl<1>(v, part, ticket) && threadIdx.x == 0) *out = v[0];
}

// v = 0: the single entries are the final values
template <class Src>
__global__ void prod_final0_kernel(Src src, uint64_t* out) {
    out[0] = lifti(src.s_at(0));
    out[1] = lifti(src.u_at(0));
}

template <class Src>
__global__ void __launch_bounds__(HAD_THREADS, 2) prod_session_kernel(ProdArgs<Src> A, FpMailbox* mb, FpRelay* rl,
                                                                     uint64_t* part) {
    __shared__ uint64_t zs[32];
    __shared__ uint64_t eq_tab[3 << kEqChunk];
    if (threadIdx.x < A.v) zs[threadIdx.x] = A.z[threadIdx.x];
    __syncthreads();
    uint64_t rprev = 0;
    for (int t = A.t_begin; t <= A.v && t <= A.t_end; t++) {
        if (t > 1 && !session_wait(mb, rl, A.seq0 + t - 1, rprev)) return;
        const int64_t h = 1ll << (A.v - t);
        const int64_t want = (h + A.per_block - 1) / A.per_block;
        const unsigned active = (unsigned)(want < 1 ? 1 : (want > A.grid ? A.grid : want));
        if (blockIdx.x >= active) return;  // no pairs for this block in this or any later round
        EqChunks EC{0, 0, 0};
        if (t == 1) EC = eq_chunks_build(eq_tab, zs, A.v);
        GlAcc a0, a1, a2;
        for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < h; b += (int64_t)active * blockDim.x) {
            if (t == 1) {
                // the factors as they are: the three products are small integers
                // (|s u| <= 2^14, |(2 s1 - s0)(2 u1 - u0)| < 2^18)
                const int s0 = A.src.s_at(b), s1 = A.src.s_at(b + h);
                const int u0 = A.src.u_at(b), u1 = A.src.u_at(b + h);
                const uint64_t e = eq_chunks_at(EC, eq_tab, b);  // eq(z_2..z_v, b)
                if (A.v > 1) A.E[b] = e;
                a0.mac(e, lifti(s0 * u0));
                a1.mac(e, lifti(s1 * u1));
                a2.mac(e, lifti((2 * s1 - s0) * (2 * u1 - u0)));
                continue;
            }
            uint64_t s0, s1, u0, u1;
            if (t == 2) {
                // the factors (length 4h) folded by rho_1: a + rho_1 (b - a) with b - a small
                const int sa = A.src.s_at(b), sb = A.src.s_at(b + 2 * h);
                const int sc = A.src.s_at(b + h), sd = A.src.s_at(b + 3 * h);
                const int ua = A.src.u_at(b), ub = A.src.u_at(b + 2 * h);
                const int uc = A.src.u_at(b + h), ud = A.src.u_at(b + 3 * h);
                s0 = gl_add(lifti(sa), gl_mul_small(rprev, sb - sa));
                s1 = gl_add(lifti(sc), gl_mul_small(rprev, sd - sc));
                u0 = gl_add(lifti(ua), gl_mul_small(rprev, ub - ua));
                u1 = gl_add(lifti(uc), gl_mul_small(rprev, ud - uc));
            } else {
                s0 = gl_fold_fast(__ldcg(A.S + b), __ldcg(A.S + b + 2 * h), rprev);
                s1 = gl_fold_fast(__ldcg(A.S + b + h), __ldcg(A.S + b + 3 * h), rprev);
                u0 = gl_fold_fast(__ldcg(A.U + b), __ldcg(A.U + b + 2 * h), rprev);
                u1 = gl_fold_fast(__ldcg(A.U + b + h), __ldcg(A.U + b + 3 * h), rprev);
            }
            A.S[b] = s0;
            A.S[b + h] = s1;
            A.U[b] = u0;
            A.U[b + h] = u1;
            const uint64_t e = gl_add(__ldcg(A.E + b), __ldcg(A.E + b + h));  // eq(z_>t, b)
            A.E[b] = e;
            a0.mac(e, gl_mul_weak(s0, u0));
            a1.mac(e, gl_mul_weak(s1, u1));
            a2.mac(e, gl_mul_weak(at2(s0, s1), at2(u0, u1)));
        }
        uint64_t acc[3] = {a0.value(), a1.value(), a2.value()};
        bool last;
        if (active == 1) {
            block_sum_gl<3>(acc);
            last = true;
        } else {
            last = grid_sum_gl_n<3>(acc, part, &rl->ticket, active);
        }
        if (last && threadIdx.x == 0) session_publish(mb, acc, A.seq0 + t);  // {h(0), h(1), h(2)}
    }
    // block 0 folds the last pair by the last challenge: s~(rho), u~(rho)
    if (A.t_end <= A.v || blockIdx.x != 0) return;
    if (!session_wait(mb, rl, A.seq0 + A.v, rprev)) return;
    if (threadIdx.x == 0) {
        uint64_t s0, s1, u0, u1;
        if (A.v == 1) {
            s0 = lifti(A.src.s_at(0));
            s1 = lifti(A.src.s_at(1));
            u0 = lifti(A.src.u_at(0));
            u1 = lifti(A.src.u_at(1));
        } else {
            s0 = __ldcg(A.S);
            s1 = __ldcg(A.S + 1);
            u0 = __ldcg(A.U);
            u1 = __ldcg(A.U + 1);
        }
        const uint64_t fin[2] = {gl_fold_fast(s0, s1, rprev), gl_fold_fast(u0, u1, rprev)};
        session_publish(mb, fin, A.seq0 + A.v + 1);
    }
}

struct ProdLabels {
    const char* claim;
    const char* round;
    const char* chal;
    const char* fin;
};

// Claim, rounds and final values of the product sum-check at the point z (v coordinates),
// written to proof (8 + 32 v + 16 bytes) and absorbed under the labels. The factors are
// read at x < len (zero beyond).
template <class Src>
int prod_sumcheck(fp_ctx* c, fp_tx* tx, const Src& src, int64_t len, const FpPoint& z, const ProdLabels& lab,
                  uint8_t* proof, size_t* proof_len, cudaStream_t st, const char* who) {
    const int v = z.v;
    int rc;
    const int vl = v / 2, vh = v - vl;
    const int64_t half = v > 0 ? 1ll << (v - 1) : 0;
    int occ = 0;
    FP_CUDA(c, cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, prod_session_kernel<Src>, HAD_THREADS, 0));
    const int cap_grid = std::max(1, occ) * c->num_sms;
    const size_t part_n = (size_t)3 * std::max(cap_grid, 2 * c->num_sms);
    size_t need = fp_align_up((size_t)8 << vh, 256) + fp_align_up((size_t)8 << vl, 256) +
                  3 * fp_align_up((size_t)8 * std::max<int64_t>(half, 1), 256) + fp_align_up(8 * part_n, 256) +
                  fp_align_up(8 * 64, 256) + 4096;
    if ((rc = fp_reserve(c, c->dev, need))) return rc;
    if ((rc = fp_reserve(c, c->host, 4096))) return rc;
    fp_reset(c->dev);
    fp_reset(c->host);
    uint64_t* EH = (uint64_t*)fp_alloc(c->dev, (size_t)8 << vh);
    uint64_t* EL = (uint64_t*)fp_alloc(c->dev, (size_t)8 << vl);
    uint64_t* S = (uint64_t*)fp_alloc(c->dev, (size_t)8 * std::max<int64_t>(half, 1));
    uint64_t* U = (uint64_t*)fp_alloc(c->dev, (size_t)8 * std::max<int64_t>(half, 1));
    uint64_t* E = (uint64_t*)fp_alloc(c->dev, (size_t)8 * std::max<int64_t>(half, 1));
    uint64_t* part = (uint64_t*)fp_alloc(c->dev, 8 * part_n);
    uint64_t* small = (uint64_t*)fp_alloc(c->dev, 8 * 64);  // [0] claim, [2..3] final values (v = 0), [8..] z
    uint64_t* hs = (uint64_t*)fp_alloc(c->host, 8 * 64);
    if (!EH || !EL || !S || !U || !E || !part || !small || !hs)
        return fp_fail(c, FP_ERR_OOM, std::string(who) + ": scratch exhausted");

    // ---- the claim c = sum_x eq(z, x) s(x) u(x) ----
    {
        FpPoint zh, zl;
        zh.v = vh;
        zl.v = vl;
        for (int i = 0; i < vh; i++) zh.z[i] = z.z[i];
        for (int i = 0; i < vl; i++) zl.z[i] = z.z[vh + i];
        if ((rc = fp_eq_table(c, zh, EH, st))) return rc;
        if ((rc = fp_eq_table(c, zl, EL, st))) return rc;
        const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>((len + 255) / 256, 2 * (int64_t)c->num_sms));
        int slot;
        fp_tic(c, st, K_HAD_CLAIM, 2.0 * (double)len, &slot);
        prod_claim_kernel<Src><<<(unsigned)blocks, 256, 0, st>>>(src, len, EH, EL, vl, part, c->tickets, small);
        fp_toc(c, st, slot);
        FP_CUDA(c, cudaGetLastError());
        if (v == 0) {
            prod_final0_kernel<Src><<<1, 1, 0, st>>>(src, small + 2);
            FP_CUDA(c, cudaGetLastError());
        }
        for (int i = 0; i < v; i++) hs[8 + i] = z.z[i];
        FP_CUDA(c, cudaMemcpyAsync(small + 8, hs + 8, 8 * (size_t)std::max(v, 1), cudaMemcpyHostToDevice, st));
        FP_CUDA(c, cudaMemcpyAsync(hs, small, 32, cudaMemcpyDeviceToHost, st));
        FP_CUDA(c, cudaStreamSynchronize(st));
    }
    size_t pos = 0;
    uint64_t claim = hs[0];
    put_u64s(proof + pos, &claim, 1);
    fp_tx_absorb_raw(tx, lab.claim, proof + pos, 8);
    pos += 8;

    uint64_t fin[2] = {hs[2], hs[3]};
    if (v > 0) {
        ProdArgs<Src> A;
        memset(&A, 0, sizeof A);
        A.src = src;
        A.S = S;
        A.U = U;
        A.E = E;
        A.z = small + 8;
        A.v = v;
        A.per_block = HAD_THREADS;  // one pair per thread
        A.grid = (int)std::max<int64_t>(1, std::min<int64_t>((half + A.per_block - 1) / A.per_block, cap_grid));
        A.seq0 = fp_seq_reserve(c, (uint64_t)v + 2);
        if ((rc = fp_session_begin(c, st))) return rc;
        fp_session_expect(c, 3);  // before any launch: round 1 publishes without a challenge
        void* args[] = {&A, &c->mb_dev, &c->relay, &part};
        const void* kern = (const void*)prod_session_kernel<Src>;
        auto round_bytes = [&](int t) {
            const double pairs = (double)(1ll << (v - t));
            return t == 1 ? 12.0 * pairs : (t == 2 ? 64.0 * pairs : 120.0 * pairs);
        };
        if (!c->stepped) {
            A.t_begin = 1;
            A.t_end = v + 1;
            double bytes = 0;
            for (int t = 1; t <= v; t++) bytes += round_bytes(t);
            int slot;
            fp_tic(c, st, K_HAD_ROUND, bytes, &slot);
            FP_CUDA(c, cudaLaunchCooperativeKernel(kern, dim3(A.grid), dim3(HAD_THREADS), args, 0, st));
            fp_toc(c, st, slot);
        }
        uint64_t pre = 1;  // eq(z_<t, rho_<t)
        for (int t = 1; t <= v; t++) {
            if (c->stepped) {
                A.t_begin = A.t_end = t;
                int slot;
                fp_tic(c, st, K_HAD_ROUND, round_bytes(t), &slot);
                FP_CUDA(c, cudaLaunchCooperativeKernel(kern, dim3(A.grid), dim3(HAD_THREADS), args, 0, st));
                fp_toc(c, st, slot);
            }
            if ((rc = fp_session_wait(c, A.seq0 + t, st))) return rc;
            const uint64_t h0 = c->mb->res[0], h1 = c->mb->res[1], h2 = c->mb->res[2];
            const uint64_t zt = z.z[t - 1];
            const uint64_t h3 = gl_add(gl_sub(h0, gl_mul(3, h1)), gl_mul(3, h2));
            uint64_t g[4];
            g[0] = gl_mul(pre, gl_mul(gl_sub(1, zt), h0));
            g[1] = gl_mul(pre, gl_mul(zt, h1));
            g[2] = gl_mul(pre, gl_mul(gl_sub(gl_mul(3, zt), 1), h2));
            g[3] = gl_mul(pre, gl_mul(gl_sub(gl_mul(5, zt), 2), h3));
            if (gl_add(g[0], g[1]) != claim) {
                fp_session_abandon(c, st);
                return fp_fail(c, FP_ERR_CUDA, std::string(who) + ": round values inconsistent with the claim");
            }
            put_u64s(proof + pos, g, 4);
            fp_tx_absorb_raw(tx, lab.round, proof + pos, 32);
            pos += 32;
            fp_session_expect(c, t < v ? 3 : 2);  // the last challenge triggers the final values
            const uint64_t r = fp_tx_squeeze_one(tx, lab.chal);
            fp_session_post(c, A.seq0 + t, r);
            claim = fp_lagrange4(g, r);
            pre = gl_mul(pre, gl_add(gl_mul(zt, r), gl_mul(gl_sub(1, zt), gl_sub(1, r))));
        }
        if (c->stepped) {
            A.t_begin = A.t_end = v + 1;
            int slot;
            fp_tic(c, st, K_HAD_FINAL, 32.0, &slot);
            FP_CUDA(c, cudaLaunchCooperativeKernel(kern, dim3(1), dim3(HAD_THREADS), args, 0, st));
            fp_toc(c, st, slot);
        }
        if ((rc = fp_session_wait(c, A.seq0 + v + 1, st))) return rc;
        fin[0] = c->mb->res[0];
        fin[1] = c->mb->res[1];
        FP_CUDA(c, cudaStreamSynchronize(st));
    }
    put_u64s(proof + pos, fin, 2);
    fp_tx_absorb_raw(tx, lab.fin, proof + pos, 16);
    pos += 16;
    *proof_len = pos;
    return FP_OK;
}

}  // namespace

int sumcheck_prove_hadamard(fp_ctx* c, fp_tx* tx, const int8_t* s, const int8_t* u, int64_t n, uint8_t* proof,
                            size_t* proof_len, void* stream) {
    if (!c || !tx || !proof_len) return fp_fail(c, FP_ERR_ARG, "sumcheck_prove_hadamard: null argument");
    if (!s || !u) return fp_fail(c, FP_ERR_ARG, "sumcheck_prove_hadamard: null factor");
    if (n < 1 || n > (1ll << HAD_MAX_V))
        return fp_fail(c, FP_ERR_SHAPE, "sumcheck_prove_hadamard: need 1 <= n <= 2^30");
    const int v = fp_log2_ceil((uint64_t)n);
    const size_t need_len = 8 + 32 * (size_t)v + 16;
    if (!proof || *proof_len < need_len) {
        *proof_len = need_len;
        return fp_fail(c, FP_ERR_ARG, "sumcheck_prove_hadamard: proof buffer too small");
    }
    FP_CUDA(c, cudaSetDevice(c->device));
    cudaStream_t st = (cudaStream_t)stream;
    int rc;
    {
        FpDigestJob jobs[2] = {{(const uint8_t*)s, (uint64_t)n}, {(const uint8_t*)u, (uint64_t)n}};
        uint8_t d[64];
        if ((rc = fp_digest_many(c, jobs, 2, d, st))) return rc;  // synchronises the stream
        fp_tx_absorb_raw(tx, "had_site", d, 64);
    }
    FpPoint z;
    z.v = v;
    for (int i = 0; i < v; i++) z.z[i] = fp_tx_squeeze_one(tx, "had_z");
    HadSrc src{s, u, n};
    return prod_sumcheck(c, tx, src, n, z, ProdLabels{"had_claim", "had_round", "had_chal", "had_final"}, proof,
                         proof_len, st, "sumcheck_prove_hadamard");
}

int sumcheck_reduce_scales(fp_ctx* c, fp_tx* tx, const void* w, int w_bits, const int8_t* scales, int M, int K,
                           const uint64_t* point, uint8_t* proof, size_t* proof_len, void* stream) {
    if (!c || !tx || !proof_len || !point) return fp_fail(c, FP_ERR_ARG, "sumcheck_reduce_scales: null argument");
    if (!w || !scales) return fp_fail(c, FP_ERR_ARG, "sumcheck_reduce_scales: null weights or scales");
    if (w_bits != 4 && w_bits != 8) return fp_fail(c, FP_ERR_ARG, "sumcheck_reduce_scales: w_bits must be 4 or 8");
    if (M < 1 || K < 1) return fp_fail(c, FP_ERR_SHAPE, "sumcheck_reduce_scales: need M, K >= 1");
    const int vM = fp_log2_ceil((uint64_t)M), vK = fp_log2_ceil((uint64_t)K), v = vM + vK;
    if (v > HAD_MAX_V)
        return fp_fail(c, FP_ERR_SHAPE, "sumcheck_reduce_scales: need ceil(log2 M) + ceil(log2 K) <= 30");
    const size_t need_len = 8 + 32 * (size_t)v + 16;
    if (!proof || *proof_len < need_len) {
        *proof_len = need_len;
        return fp_fail(c, FP_ERR_ARG, "sumcheck_reduce_scales: proof buffer too small");
    }
    for (int i = 0; i < v; i++)
        if (point[i] >= GL_P) return fp_fail(c, FP_ERR_ARG, "sumcheck_reduce_scales: point not canonical");
    FP_CUDA(c, cudaSetDevice(c->device));
    cudaStream_t st = (cudaStream_t)stream;
    int rc;
    const int64_t pitch = w_bits == 4 ? (K + 1) / 2 : K;
    const int G = (K + 63) / 64;
    {
        FpDigestJob jobs[2] = {{(const uint8_t*)w, (uint64_t)M * (uint64_t)pitch},
                               {(const uint8_t*)scales, (uint64_t)M * (uint64_t)G}};
        uint8_t d[64];
        if ((rc = fp_digest_many(c, jobs, 2, d, st))) return rc;  // synchronises the stream
        fp_tx_absorb_raw(tx, "scl_site", d, 64);
    }
    FpPoint z;
    z.v = v;
    for (int i = 0; i < v; i++) z.z[i] = point[i];
    SclSrc src{(const uint8_t*)w, scales, pitch, M, K, G, vK, w_bits};
    return prod_sumcheck(c, tx, src, (int64_t)M << vK, z,
                         ProdLabels{"scl_claim", "scl_round", "scl_chal", "scl_final"}, proof, proof_len, st,
                         "sumcheck_reduce_scales");
}
