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
//
// The scale reduction takes a shorter road to the same bytes. Se(i, k) does not depend on
// the vL = min(6, vK) low column bits kl, and those are the last variables bound, so for the
// first v' = v - vL rounds every sum over kl can be taken first: with x = (i, kh, kl),
//   sum_kl eq(z, x) Se(x) w(x) = eq(z', (i, kh)) S[i][kh] W'(i, kh),
//   W'(i, kh) = sum_kl eq(z_kl, kl) w(i, kh 2^vL + kl),
// so rounds 1..v' are the product sum-check of S and W' (a 64th of the entries) at
// z' = z_1..z_v'. The last vL rounds need w~(rho', kl) for the 2^vL values of kl: one row
// contraction of w with the weights eq(rho_rows, i) (the partial evaluation), paired on the
// host with eq(rho_kh, kh); Se~ is the constant S~(rho') there, and the host runs those
// rounds on 2^vL values.
#include <string.h>

#include <algorithm>
#include <vector>

#include "fp_eqchunks.cuh"
#include "fp_internal.h"
#include "fp_reduce.cuh"
#include "fp_session.cuh"

namespace {

constexpr int HAD_THREADS = 256;
constexpr int HAD_MAX_V = 30;

// the gated product's factors: two int8 vectors of n entries, zero-padded
struct HadSrc {
    static constexpr bool kFieldU = false;
    const int8_t* s;
    const int8_t* u;
    int64_t n;
    __device__ __forceinline__ int s_at(int64_t x) const { return x < n ? (int)s[x] : 0; }
    __device__ __forceinline__ int u_at(int64_t x) const { return x < n ? (int)u[x] : 0; }
    __device__ __forceinline__ uint64_t uf(int64_t) const { return 0; }
};

// the scale reduction's first v' rounds over x' = i 2^vH + kh: the scales S[i][kh] (zero
// past the M x G scales) and W'(i, kh), a field vector of M 2^vH entries (zero beyond)
struct SclRedSrc {
    static constexpr bool kFieldU = true;
    const int8_t* sc;
    const uint64_t* wp;
    int64_t n;  // M 2^vH
    int G, vH;
    __device__ __forceinline__ int s_at(int64_t x) const {
        const int64_t kh = x & ((1ll << vH) - 1);
        return (x < n && kh < G) ? (int)sc[(x >> vH) * G + kh] : 0;
    }
    __device__ __forceinline__ int u_at(int64_t) const { return 0; }
    __device__ __forceinline__ uint64_t uf(int64_t x) const { return x < n ? wp[x] : 0ull; }
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

// W'(i, kh) = sum_{kl < 2^vL} eq(z_kl, kl) w(i, kh 2^vL + kl), i < M, kh < 2^vH (w zero past K):
// one output per thread, the weights' small values biased to unsigned (w + 8 for int4, w + 128
// for int8) and summed exactly, the bias times the sum of the used weights taken off once
struct SclGroupArgs {
    const uint8_t* w;
    int64_t pitch;  // bytes per weight row
    int M, K, bits, vL, vH;
};

__global__ void __launch_bounds__(256) scl_group_kernel(SclGroupArgs a, const uint64_t* __restrict__ eqL,
                                                        uint64_t* __restrict__ wp) {
    __shared__ uint64_t e[64];
    __shared__ uint64_t esum;
    const int L = 1 << a.vL;
    if (threadIdx.x < L) e[threadIdx.x] = eqL[threadIdx.x];
    __syncthreads();
    if (threadIdx.x == 0) {
        uint64_t t = 0;
        for (int j = 0; j < L; j++) t = gl_add(t, e[j]);
        esum = gl_mul(t, a.bits == 4 ? 8ull : 128ull);
    }
    __syncthreads();
    const int64_t n = (int64_t)a.M << a.vH;
    for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < n; x += (int64_t)gridDim.x * blockDim.x) {
        const int64_t i = x >> a.vH, k0 = (x & ((1ll << a.vH) - 1)) << a.vL;
        const uint8_t* row = a.w + i * a.pitch;
        GlAcc acc;
        uint64_t corr = esum;
        if (k0 + L <= a.K) {
            if (a.bits == 4) {
                const uint8_t* p = row + (k0 >> 1);
                for (int j = 0; j < L; j += 2) {
                    const uint32_t b = p[j >> 1];
                    acc.mac32(e[j], (b & 15) ^ 8);  // nibble n stands for n - 16 when n >= 8: n ^ 8 = w + 8
                    if (j + 1 < L) acc.mac32(e[j + 1], (b >> 4) ^ 8);
                }
            } else {
                const uint8_t* p = row + k0;
                for (int j = 0; j < L; j++) acc.mac32(e[j], (uint32_t)p[j] ^ 0x80u);  // w + 128
            }
        } else {
            // the ragged last group: only k < K contributes, and only its weights carry the bias
            uint64_t used = 0;
            for (int j = 0; j < L && k0 + j < a.K; j++) {
                const int64_t k = k0 + j;
                uint32_t u;
                if (a.bits == 4) {
                    const uint32_t b = row[k >> 1];
                    u = ((k & 1) ? (b >> 4) : (b & 15)) ^ 8;
                } else {
                    u = (uint32_t)row[k] ^ 0x80u;
                }
                acc.mac32(e[j], u);
                used = gl_add(used, e[j]);
            }
            corr = gl_mul(used, a.bits == 4 ? 8ull : 128ull);
        }
        wp[x] = gl_sub(acc.value(), corr);
    }
}

// c' = sum_{x' < n} eq(z', x') S(x') W'(x'), eq split as EH[x' >> vl] EL[x' & (2^vl - 1)]
__global__ void __launch_bounds__(256) scl_red_claim_kernel(SclRedSrc src, const uint64_t* __restrict__ EH,
                                                            const uint64_t* __restrict__ EL, int vl, uint64_t* part,
                                                            unsigned int* ticket, uint64_t* out) {
    GlAcc acc;
    const int64_t mask = (1ll << vl) - 1;
    for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < src.n; x += (int64_t)gridDim.x * blockDim.x) {
        const int sv = src.s_at(x);
        if (sv == 0) continue;
        const uint64_t e = gl_mul(__ldg(EH + (x >> vl)), __ldg(EL + (x & mask)));
        acc.mac(gl_mul_small(gl_mul(e, src.uf(x)), sv), 1ull);
    }
    uint64_t v[1] = {acc.value()};
    if (grid_sum_gl<1>(v, part, ticket) && threadIdx.x == 0) *out = v[0];
}

template <class Src>
// four blocks per SM (64 registers, no spill): the rounds wait on memory latency, and more
// warps hide it (2^26 entries: gated product 1.29 -> 1.02 ms, SiLU layers 1.66 -> 1.58 ms)
#ifndef FP_HAD_MIN_BLOCKS
#define FP_HAD_MIN_BLOCKS 4
#endif
__global__ void __launch_bounds__(HAD_THREADS, FP_HAD_MIN_BLOCKS) prod_session_kernel(ProdArgs<Src> A, FpMailbox* mb, FpRelay* rl,
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
                const int s0 = A.src.s_at(b), s1 = A.src.s_at(b + h);
                const uint64_t e = eq_chunks_at(EC, eq_tab, b);  // eq(z_2..z_v, b)
                if (A.v > 1) A.E[b] = e;
                if constexpr (Src::kFieldU) {
                    // a small integer s times a field element u
                    const uint64_t u0 = A.src.uf(b), u1 = A.src.uf(b + h);
                    a0.mac(e, gl_mul_small(u0, s0));
                    a1.mac(e, gl_mul_small(u1, s1));
                    a2.mac(e, gl_mul_small(at2(u0, u1), 2 * s1 - s0));
                } else {
                    // the factors as they are: the three products are small integers
                    // (|s u| <= 2^14, |(2 s1 - s0)(2 u1 - u0)| < 2^18)
                    const int u0 = A.src.u_at(b), u1 = A.src.u_at(b + h);
                    a0.mac(e, lifti(s0 * u0));
                    a1.mac(e, lifti(s1 * u1));
                    a2.mac(e, lifti((2 * s1 - s0) * (2 * u1 - u0)));
                }
                continue;
            }
            uint64_t s0, s1, u0, u1;
            if (t == 2) {
                // the factors (length 4h) folded by rho_1: a + rho_1 (b - a) with b - a small
                const int sa = A.src.s_at(b), sb = A.src.s_at(b + 2 * h);
                const int sc = A.src.s_at(b + h), sd = A.src.s_at(b + 3 * h);
                s0 = gl_add(lifti(sa), gl_mul_small(rprev, sb - sa));
                s1 = gl_add(lifti(sc), gl_mul_small(rprev, sd - sc));
                if constexpr (Src::kFieldU) {
                    u0 = gl_fold_fast(A.src.uf(b), A.src.uf(b + 2 * h), rprev);
                    u1 = gl_fold_fast(A.src.uf(b + h), A.src.uf(b + 3 * h), rprev);
                } else {
                    const int ua = A.src.u_at(b), ub = A.src.u_at(b + 2 * h);
                    const int uc = A.src.u_at(b + h), ud = A.src.u_at(b + 3 * h);
                    u0 = gl_add(lifti(ua), gl_mul_small(rprev, ub - ua));
                    u1 = gl_add(lifti(uc), gl_mul_small(rprev, ud - uc));
                }
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
            if constexpr (Src::kFieldU) {
                u0 = A.src.uf(0);
                u1 = A.src.uf(1);
            } else {
                u0 = lifti(A.src.u_at(0));
                u1 = lifti(A.src.u_at(1));
            }
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

// g_t(0..3) = eq(z_<t, rho_<t) eq(z_t, X) h_t(X) from h_t(0), h_t(1), h_t(2) (h_t has degree 2:
// h_t(3) = h_t(0) - 3 h_t(1) + 3 h_t(2)); eq(z_t, 2) = 3 z_t - 1, eq(z_t, 3) = 5 z_t - 2
void prod_round_values(const uint64_t h[3], uint64_t zt, uint64_t pre, uint64_t g[4]) {
    const uint64_t h3 = gl_add(gl_sub(h[0], gl_mul(3, h[1])), gl_mul(3, h[2]));
    g[0] = gl_mul(pre, gl_mul(gl_sub(1, zt), h[0]));
    g[1] = gl_mul(pre, gl_mul(zt, h[1]));
    g[2] = gl_mul(pre, gl_mul(gl_sub(gl_mul(3, zt), 1), h[2]));
    g[3] = gl_mul(pre, gl_mul(gl_sub(gl_mul(5, zt), 2), h3));
}

// Rounds 1..v (v >= 1) of the product sum-check of src at the point z, from the running claim:
// the round values written at proof + pos and absorbed, the challenges into rho, the final
// values s~(rho), u~(rho) into fin; claim and pre (eq(z_<t, rho_<t)) carried on. S, U, E
// (2^(v-1) entries), part (3 words per block of cap_grid), small (64 words; z goes to small + 8)
// and hs (64 host words) are the caller's scratch.
template <class Src>
int prod_rounds(fp_ctx* c, fp_tx* tx, const Src& src, const FpPoint& z, const ProdLabels& lab, int cap_grid,
                uint64_t* S, uint64_t* U, uint64_t* E, uint64_t* part, uint64_t* small, uint64_t* hs,
                uint64_t& claim, uint64_t& pre, uint8_t* proof, size_t& pos, uint64_t* rho, uint64_t fin[2],
                cudaStream_t st, const char* who) {
    const int v = z.v;
    int rc;
    const int64_t half = 1ll << (v - 1);
    for (int i = 0; i < v; i++) hs[8 + i] = z.z[i];
    FP_CUDA(c, cudaMemcpyAsync(small + 8, hs + 8, 8 * (size_t)v, cudaMemcpyHostToDevice, st));
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
        if (Src::kFieldU) return t == 1 ? 20.0 * pairs : (t == 2 ? 72.0 * pairs : 120.0 * pairs);
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
    for (int t = 1; t <= v; t++) {
        if (c->stepped) {
            A.t_begin = A.t_end = t;
            int slot;
            fp_tic(c, st, K_HAD_ROUND, round_bytes(t), &slot);
            FP_CUDA(c, cudaLaunchCooperativeKernel(kern, dim3(A.grid), dim3(HAD_THREADS), args, 0, st));
            fp_toc(c, st, slot);
        }
        if ((rc = fp_session_wait(c, A.seq0 + t, st))) return rc;
        const uint64_t h[3] = {c->mb->res[0], c->mb->res[1], c->mb->res[2]};
        uint64_t g[4];
        prod_round_values(h, z.z[t - 1], pre, g);
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
        rho[t - 1] = r;
        claim = fp_lagrange4(g, r);
        pre = gl_mul(pre, gl_add(gl_mul(z.z[t - 1], r), gl_mul(gl_sub(1, z.z[t - 1]), gl_sub(1, r))));
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
    return FP_OK;
}

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
        std::vector<uint64_t> rho(v);
        uint64_t pre = 1;
        if ((rc = prod_rounds(c, tx, src, z, lab, cap_grid, S, U, E, part, small, hs, claim, pre, proof, pos, rho.data(),
                              fin, st, who)))
            return rc;
    }
    put_u64s(proof + pos, fin, 2);
    fp_tx_absorb_raw(tx, lab.fin, proof + pos, 16);
    pos += 16;
    *proof_len = pos;
    return FP_OK;
}

// eq(z, x) for the 2^v indices x (z_0 the weight of the top bit), on the host
std::vector<uint64_t> host_eq_table(const uint64_t* z, int v) {
    std::vector<uint64_t> e((size_t)1 << v, 1);
    for (int j = 0; j < v; j++) {
        const size_t n = (size_t)1 << j;  // entries so far, over the first j coordinates
        for (size_t x = n; x-- > 0;) {
            e[2 * x + 1] = gl_mul(e[x], z[j]);
            e[2 * x] = gl_mul(e[x], gl_sub(1, z[j]));
        }
    }
    return e;
}

// The scale reduction by the grouped road (see the head of the file): W' on the device, the
// first v' = v - vL rounds as the product sum-check of S and W', then the last vL rounds on the
// host from w~(rho', kl). The bytes are those of the product sum-check of Se and w.
int scl_grouped_sumcheck(fp_ctx* c, fp_tx* tx, const uint8_t* w, int bits, const int8_t* sc, int M, int K,
                         int64_t pitch, int G, const FpPoint& z, const ProdLabels& lab, uint8_t* proof,
                         size_t* proof_len, cudaStream_t st, const char* who) {
    const int vM = fp_log2_ceil((uint64_t)M), vK = fp_log2_ceil((uint64_t)K), v = z.v;
    const int vL = std::min(6, vK), vH = vK - vL, vp = vM + vH;
    const int64_t nW = (int64_t)M << vH;
    const int vl = vp / 2, vh = vp - vl;
    const int64_t half = vp > 0 ? 1ll << (vp - 1) : 1;
    int rc, occ = 0;
    FP_CUDA(c, cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, prod_session_kernel<SclRedSrc>, HAD_THREADS, 0));
    const int cap_grid = std::max(1, occ) * c->num_sms;
    const size_t part_n = (size_t)3 * std::max(cap_grid, 2 * c->num_sms);
    const int64_t kpad = 1ll << vK;
    std::vector<uint64_t> zrow(z.z, z.z + vM);  // replaced by rho_rows before the contraction
    FpPeJob job{w, bits, nullptr, M, K, nullptr, vM, nullptr, kpad};
    size_t need = fp_align_up((size_t)8 << vh, 256) + fp_align_up((size_t)8 << vl, 256) +
                  3 * fp_align_up((size_t)8 * half, 256) + fp_align_up(8 * part_n, 256) + fp_align_up(8 * 64, 256) +
                  fp_align_up((size_t)8 * nW, 256) + fp_align_up((size_t)8 * kpad, 256) + fp_align_up(8 * 64, 256) +
                  fp_partial_scratch(c, &job, 1) + 8192;
    if ((rc = fp_reserve(c, c->dev, need))) return rc;
    if ((rc = fp_reserve(c, c->host, 4096 + (size_t)8 * kpad + fp_partial_host_scratch(&job, 1) + 4096))) return rc;
    fp_reset(c->dev);
    fp_reset(c->host);
    uint64_t* EH = (uint64_t*)fp_alloc(c->dev, (size_t)8 << vh);
    uint64_t* EL = (uint64_t*)fp_alloc(c->dev, (size_t)8 << vl);
    uint64_t* S = (uint64_t*)fp_alloc(c->dev, (size_t)8 * half);
    uint64_t* U = (uint64_t*)fp_alloc(c->dev, (size_t)8 * half);
    uint64_t* E = (uint64_t*)fp_alloc(c->dev, (size_t)8 * half);
    uint64_t* part = (uint64_t*)fp_alloc(c->dev, 8 * part_n);
    uint64_t* small = (uint64_t*)fp_alloc(c->dev, 8 * 64);  // [0] claim, [2..3] S, W' at v' = 0, [8..] z'
    uint64_t* wp = (uint64_t*)fp_alloc(c->dev, (size_t)8 * std::max<int64_t>(nW, 1));
    uint64_t* acol = (uint64_t*)fp_alloc(c->dev, (size_t)8 * kpad);
    uint64_t* eqd = (uint64_t*)fp_alloc(c->dev, 8 * 64);
    uint64_t* hs = (uint64_t*)fp_alloc(c->host, 8 * 64);
    uint64_t* hcol = (uint64_t*)fp_alloc(c->host, (size_t)8 * kpad);
    if (!EH || !EL || !S || !U || !E || !part || !small || !wp || !acol || !eqd || !hs || !hcol)
        return fp_fail(c, FP_ERR_OOM, std::string(who) + ": scratch exhausted");

    // ---- W'(i, kh) with eq over the low column coordinates z_v'+1..z_v ----
    const std::vector<uint64_t> eqL = host_eq_table(z.z + vp, vL);
    for (int j = 0; j < (1 << vL); j++) hs[j] = eqL[j];
    FP_CUDA(c, cudaMemcpyAsync(eqd, hs, 8 * ((size_t)1 << vL), cudaMemcpyHostToDevice, st));
    {
        SclGroupArgs ga{w, pitch, M, K, bits, vL, vH};
        int slot;
        fp_tic(c, st, K_SCL_GROUP, (double)M * (double)pitch + 8.0 * (double)nW, &slot);
        scl_group_kernel<<<fp_grid256(c, nW), 256, 0, st>>>(ga, eqd, wp);
        fp_toc(c, st, slot);
        FP_CUDA(c, cudaGetLastError());
    }
    const SclRedSrc src{sc, wp, nW, G, vH};

    // ---- the claim c = sum_x' eq(z', x') S(x') W'(x') ----
    {
        FpPoint zh, zl;
        zh.v = vh;
        zl.v = vl;
        for (int i = 0; i < vh; i++) zh.z[i] = z.z[i];
        for (int i = 0; i < vl; i++) zl.z[i] = z.z[vh + i];
        if ((rc = fp_eq_table(c, zh, EH, st))) return rc;
        if ((rc = fp_eq_table(c, zl, EL, st))) return rc;
        FP_CUDA(c, cudaMemsetAsync(small, 0, 8 * 4, st));
        const int64_t blocks = std::max<int64_t>(1, std::min<int64_t>((nW + 255) / 256, 2 * (int64_t)c->num_sms));
        int slot;
        fp_tic(c, st, K_HAD_CLAIM, 9.0 * (double)nW, &slot);
        scl_red_claim_kernel<<<(unsigned)blocks, 256, 0, st>>>(src, EH, EL, vl, part, c->tickets, small);
        fp_toc(c, st, slot);
        FP_CUDA(c, cudaGetLastError());
        FP_CUDA(c, cudaMemcpyAsync(hs, small, 8, cudaMemcpyDeviceToHost, st));
        FP_CUDA(c, cudaStreamSynchronize(st));
    }
    size_t pos = 0;
    uint64_t claim = hs[0], pre = 1;
    put_u64s(proof + pos, &claim, 1);
    fp_tx_absorb_raw(tx, lab.claim, proof + pos, 8);
    pos += 8;

    // ---- rounds 1..v' on the device: S~(rho') and W'~(rho') at the end ----
    std::vector<uint64_t> rho(std::max(vp, 1));
    uint64_t fin1[2];
    if (vp > 0) {
        FpPoint zp;
        zp.v = vp;
        for (int i = 0; i < vp; i++) zp.z[i] = z.z[i];
        if ((rc = prod_rounds(c, tx, src, zp, lab, cap_grid, S, U, E, part, small, hs, claim, pre, proof, pos,
                              rho.data(), fin1, st, who)))
            return rc;
    } else {
        // one row, one group: S[0][0] and W'(0)
        int8_t s00 = 0;
        FP_CUDA(c, cudaMemcpyAsync(&s00, sc, 1, cudaMemcpyDeviceToHost, st));
        FP_CUDA(c, cudaMemcpyAsync(hs, wp, 8, cudaMemcpyDeviceToHost, st));
        FP_CUDA(c, cudaStreamSynchronize(st));
        fin1[0] = gl_from_i64(s00);
        fin1[1] = hs[0];
    }

    // ---- w~(rho', kl): the rows contracted with eq(rho_rows, i), the groups paired with eq(rho_kh, kh) ----
    for (int i = 0; i < vM; i++) zrow[i] = rho[i];
    job.z = zrow.data();
    job.out = acol;
    if ((rc = fp_partial_many(c, &job, 1, st))) return rc;
    FP_CUDA(c, cudaMemcpyAsync(hcol, acol, (size_t)8 * kpad, cudaMemcpyDeviceToHost, st));
    FP_CUDA(c, cudaStreamSynchronize(st));
    const std::vector<uint64_t> eqH = host_eq_table(rho.data() + vM, vH);
    std::vector<uint64_t> wl((size_t)1 << vL, 0);
    for (int64_t kh = 0; kh < (1ll << vH); kh++)
        for (int j = 0; j < (1 << vL); j++) {
            const int64_t k = (kh << vL) + j;
            if (k < K) wl[j] = gl_add(wl[j], gl_mul(eqH[kh], gl_canon(hcol[k])));
        }
    {
        // W'~(rho') = sum_kl eq(z_kl, kl) w~(rho', kl): the device's two roads must meet
        uint64_t chk = 0;
        for (int j = 0; j < (1 << vL); j++) chk = gl_add(chk, gl_mul(eqL[j], wl[j]));
        if (chk != fin1[1]) return fp_fail(c, FP_ERR_CUDA, std::string(who) + ": grouped and row contractions disagree");
    }

    // ---- rounds v'+1..v on the host: Se~ is the constant S~(rho'), w runs over kl ----
    const uint64_t sfin = fin1[0];
    for (int t = vp + 1; t <= v; t++) {
        const size_t hlen = wl.size() / 2;
        const std::vector<uint64_t> e = host_eq_table(z.z + t, v - t);  // eq(z_>t, b), b < hlen
        uint64_t h[3] = {0, 0, 0};
        for (size_t b = 0; b < hlen; b++) {
            h[0] = gl_add(h[0], gl_mul(e[b], wl[b]));
            h[1] = gl_add(h[1], gl_mul(e[b], wl[b + hlen]));
            h[2] = gl_add(h[2], gl_mul(e[b], gl_sub(gl_add(wl[b + hlen], wl[b + hlen]), wl[b])));
        }
        for (int i = 0; i < 3; i++) h[i] = gl_mul(sfin, h[i]);
        uint64_t g[4];
        prod_round_values(h, z.z[t - 1], pre, g);
        if (gl_add(g[0], g[1]) != claim)
            return fp_fail(c, FP_ERR_CUDA, std::string(who) + ": round values inconsistent with the claim");
        put_u64s(proof + pos, g, 4);
        fp_tx_absorb_raw(tx, lab.round, proof + pos, 32);
        pos += 32;
        const uint64_t r = fp_tx_squeeze_one(tx, lab.chal);
        claim = fp_lagrange4(g, r);
        pre = gl_mul(pre, gl_add(gl_mul(z.z[t - 1], r), gl_mul(gl_sub(1, z.z[t - 1]), gl_sub(1, r))));
        for (size_t b = 0; b < hlen; b++) wl[b] = gl_fold(wl[b], wl[b + hlen], r);
        wl.resize(hlen);
    }
    const uint64_t fin[2] = {sfin, wl[0]};
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
                           const uint64_t* point, const uint8_t* w_digest, uint8_t* proof, size_t* proof_len,
                           void* stream) {
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
    if (w_digest) {
        fp_tx_absorb_raw(tx, "scl_site", w_digest, 64);  // committed in advance
    } else {
        FpDigestJob jobs[2] = {{(const uint8_t*)w, (uint64_t)M * (uint64_t)pitch},
                               {(const uint8_t*)scales, (uint64_t)M * (uint64_t)G}};
        uint8_t d[64];
        if ((rc = fp_digest_many(c, jobs, 2, d, st))) return rc;  // synchronises the stream
        fp_tx_absorb_raw(tx, "scl_site", d, 64);
    }
    FpPoint z;
    z.v = v;
    for (int i = 0; i < v; i++) z.z[i] = point[i];
    return scl_grouped_sumcheck(c, tx, (const uint8_t*)w, w_bits, scales, M, K, pitch, G, z,
                                ProdLabels{"scl_claim", "scl_round", "scl_chal", "scl_final"}, proof, proof_len, st,
                                "sumcheck_reduce_scales");
}
