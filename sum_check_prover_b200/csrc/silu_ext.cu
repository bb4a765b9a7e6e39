// The 16-bit function lookups (SiLU, softmax numerator) over the quadratic extension.
//
// "How fast can FlashProve go", 2 Background and 3.1 (non-polynomial steps are
// proven by lookups; the SiLU's output is committed), 4 (Tighter Rooflines: the
// key side is a binary tree of fractions, every level proven by sum-check; the
// note on soundness: challenges from an extension field). The statement of
// logup_prove_silu / logup_prove_exp with gamma, alpha, mu, lambda, every round
// challenge and every value sent in F_p[phi]/(phi^2 - 7) (16 bytes each), and
// the tree's fractions in the extension; labels "silu2_*" / "exp2_*".
//
// Kernels follow silu.cu with 16-byte vectors: a histogram of g (the padding
// keys added by one thread), the leaves P = 1, Q = alpha - (g + gamma s), one
// level of the tree per launch, each layer's sum-check of
// eq(z, x) (pL qR + pR qL + lambda qL qR) as one resident cooperative launch
// (h(0), h(1), h(2) as six words; the host forms g(0..3) with eq(z_t, X) and the
// eq prefix), and the leaf claims g~(z), s~(z) as eq-weighted sums of the int16
// columns (the s column's padding adds pad_s (1 - sum_{x < n} eq(z, x))).
//
// The host half (x16_protocol) takes its device values from a source: the
// kernels here, or a caller's callback (fp_lookup16x_protocol_drive).
#include <string.h>

#include <algorithm>
#include <vector>

#include "fp_ext2.cuh"
#include "fp_ext2_host.h"
#include "fp_hist.cuh"
#include "fp_internal.h"
#include "fp_reduce.cuh"
#include "fp_session.cuh"

namespace {

constexpr int X16_THREADS = 256;
constexpr int X16_MAX_V = 30;
constexpr int X16_CHUNK = 8;  // four eq chunk tables of at most 2^8 entries (z_2..z_d, d <= 29)

__device__ __forceinline__ uint64_t x16_lift(int64_t x) { return x < 0 ? GL_P - (uint64_t)(-x) : (uint64_t)x; }

// leaves: P = 1, Q = alpha - (g + gamma s); past n the padding key (0, pad_s)
__global__ void x16_leaf_kernel(const int16_t* __restrict__ g, const int16_t* __restrict__ s, int64_t n, int64_t L,
                                Ext2 alpha, Ext2 gamma, int64_t pad_s, Ext2* __restrict__ P, Ext2* __restrict__ Q) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < L; i += (int64_t)gridDim.x * blockDim.x) {
        const uint64_t gv = i < n ? x16_lift(g[i]) : 0, sv = i < n ? x16_lift(s[i]) : x16_lift(pad_s);
        const Ext2 f = e2_make(gl_add(gv, gl_mul(gamma.a, sv)), gl_mul(gamma.b, sv));
        P[i] = e2_make(1, 0);
        Q[i] = e2_sub(alpha, f);
    }
}

// one level up: P'[x] = P[2x] Q[2x+1] + P[2x+1] Q[2x], Q'[x] = Q[2x] Q[2x+1], x < c
__global__ void x16_level_kernel(const Ext2* __restrict__ P, const Ext2* __restrict__ Q, int64_t c,
                                 Ext2* __restrict__ Po, Ext2* __restrict__ Qo) {
    for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < c; x += (int64_t)gridDim.x * blockDim.x) {
        const Ext2 pl = P[2 * x], pr = P[2 * x + 1], ql = Q[2 * x], qr = Q[2 * x + 1];
        Po[x] = e2_add(e2_mul(pl, qr), e2_mul(pr, ql));
        Qo[x] = e2_mul(ql, qr);
    }
}

// the eq table of an extension point (by value): out[x] = eq(z, x), z_1 on the top bit
struct X16Point {
    Ext2 z[32];
    int v;
};

__global__ void x16_eq_kernel(X16Point p, Ext2* __restrict__ out) {
    const int64_t len = 1ll << p.v;
    for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < len; x += (int64_t)gridDim.x * blockDim.x) {
        Ext2 e = e2_make(1, 0);
        for (int b = 0; b < p.v; b++) e = e2_mul(e, e2_eq1(p.z[b], (int)((x >> (p.v - 1 - b)) & 1)));
        out[x] = e;
    }
}

// out[0..1] = sum_{x < n} eq(z, x) a(x), out[2..3] = sum_{x < n} eq(z, x) (eq split as EH[x >> vl] EL[...])
template <class T>
__global__ void __launch_bounds__(256) x16_mle_kernel(const T* __restrict__ a, int64_t n,
                                                      const Ext2* __restrict__ EH, const Ext2* __restrict__ EL, int vl,
                                                      uint64_t* part, unsigned int* ticket, uint64_t* out) {
    E2Acc acc;
    GlAcc ea, eb;
    const int64_t mask = (1ll << vl) - 1;
    for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < n; x += (int64_t)gridDim.x * blockDim.x) {
        const Ext2 e = e2_mul(EH[x >> vl], EL[x & mask]);
        ea.add(e.a);
        eb.add(e.b);
        const int64_t v = (int64_t)a[x];
        if (v != 0) acc.mac_base(e, x16_lift(v));
    }
    uint64_t v[4] = {acc.a.value(), acc.b.value(), ea.value(), eb.value()};
    if (grid_sum_gl<4>(v, part, ticket) && threadIdx.x == 0)
        for (int i = 0; i < 4; i++) out[i] = v[i];
}

struct X16Layer {
    const Ext2* P;  // tree layer d + 1 (2^(d+1) entries): child x of node b is entry 2 b + x
    const Ext2* Q;
    Ext2* pl;       // folded children from round 2 on (2^(d-1) entries each)
    Ext2* pr;
    Ext2* ql;
    Ext2* qr;
    Ext2* E;        // suffix eq table (2^(d-1) entries)
    X16Point z;     // the layer's point z_1..z_d
    Ext2 lam;
    int d;
    int grid;
    int per_block;
    int pad;
    uint64_t seq0;  // round t publishes seq0 + t, the final values seq0 + d + 1
    int t_begin;    // rounds run by this launch: [t_begin, t_end]; t_end > d includes the final values
    int t_end;
};

// pL qR + pR qL + lambda qL qR
__device__ __forceinline__ Ext2 x16_f(Ext2 a, Ext2 b, Ext2 c, Ext2 e, Ext2 lam) {
    return e2_add(e2_add(e2_mul(a, e), e2_mul(b, c)), e2_mul(lam, e2_mul(c, e)));
}

// the chunk tables of eq(z_2..z_d, .) (table j at tab + 2^8 j; the first coordinate on the top bit)
__device__ __forceinline__ void x16_tables(Ext2* tab, const Ext2* zs, int d, int (&w)[4]) {
    int rest = d - 1;
#pragma unroll
    for (int j = 0; j < 4; j++) {
        w[j] = rest < X16_CHUNK ? rest : X16_CHUNK;
        rest -= w[j];
    }
    for (int x = threadIdx.x; x < (4 << X16_CHUNK); x += blockDim.x) {
        const int j = x >> X16_CHUNK, y = x & ((1 << X16_CHUNK) - 1);
        if (y >= (1 << w[j])) continue;
        int first = 1;
        for (int q = 0; q < j; q++) first += w[q];
        Ext2 e = e2_make(1, 0);
        for (int i = 0; i < w[j]; i++) e = e2_mul(e, e2_eq1(zs[first + i], (y >> (w[j] - 1 - i)) & 1));
        tab[x] = e;
    }
    __syncthreads();
}

__device__ __forceinline__ Ext2 x16_eq_at(const Ext2* tab, const int (&w)[4], int64_t b) {
    const int s2 = w[3], s1 = w[3] + w[2], s0 = s1 + w[1];
    Ext2 e = tab[(int)((b >> s0) & ((1 << w[0]) - 1))];
    if (w[1]) e = e2_mul(e, tab[(1 << X16_CHUNK) + (int)((b >> s1) & ((1 << w[1]) - 1))]);
    if (w[2]) e = e2_mul(e, tab[(2 << X16_CHUNK) + (int)((b >> s2) & ((1 << w[2]) - 1))]);
    if (w[3]) e = e2_mul(e, tab[(3 << X16_CHUNK) + (int)(b & ((1 << w[3]) - 1))]);
    return e;
}

__global__ void __launch_bounds__(X16_THREADS, 2) x16_layer_kernel(X16Layer A, FpMailbox* mb, FpRelay* rl,
                                                                  uint64_t* part) {
    __shared__ Ext2 tab[4 << X16_CHUNK];
    Ext2 rho = e2_make(0, 0);
    for (int t = A.t_begin; t <= A.d && t <= A.t_end; t++) {
        if (t > 1) {
            uint64_t ra, rb;
            if (!session_wait2(mb, rl, A.seq0 + t - 1, ra, rb)) return;
            rho = e2_make(ra, rb);
        }
        const int64_t h = 1ll << (A.d - t);
        const int64_t want = (h + A.per_block - 1) / A.per_block;
        const unsigned active = (unsigned)(want < 1 ? 1 : (want > A.grid ? A.grid : want));
        if (blockIdx.x >= active) return;  // no pairs for this block in this or any later round
        int w[4] = {0, 0, 0, 0};
        if (t == 1) x16_tables(tab, A.z.z, A.d, w);
        // h(1) only when z_t = 0: otherwise the host takes it from the running claim
        const bool need1 = A.z.z[t - 1].a == 0 && A.z.z[t - 1].b == 0;
        E2Acc a0, a1, a2;
        for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < h; b += (int64_t)active * blockDim.x) {
            Ext2 p0, p1, r0, r1, q0, q1, s0, s1, e;  // pL, pR, qL, qR at the pair's two points
            if (t == 1) {
                p0 = e2_ldcg(A.P + 2 * b);
                r0 = e2_ldcg(A.P + 2 * b + 1);
                q0 = e2_ldcg(A.Q + 2 * b);
                s0 = e2_ldcg(A.Q + 2 * b + 1);
                p1 = e2_ldcg(A.P + 2 * (b + h));
                r1 = e2_ldcg(A.P + 2 * (b + h) + 1);
                q1 = e2_ldcg(A.Q + 2 * (b + h));
                s1 = e2_ldcg(A.Q + 2 * (b + h) + 1);
                e = x16_eq_at(tab, w, b);  // eq(z_2..z_d, b)
                if (A.d > 1) A.E[b] = e;
            } else {
                if (t == 2) {
                    // the children vectors (length 4h, read from the tree layer) folded by rho_1
                    p0 = e2_fold(e2_ldcg(A.P + 2 * b), e2_ldcg(A.P + 2 * (b + 2 * h)), rho);
                    r0 = e2_fold(e2_ldcg(A.P + 2 * b + 1), e2_ldcg(A.P + 2 * (b + 2 * h) + 1), rho);
                    q0 = e2_fold(e2_ldcg(A.Q + 2 * b), e2_ldcg(A.Q + 2 * (b + 2 * h)), rho);
                    s0 = e2_fold(e2_ldcg(A.Q + 2 * b + 1), e2_ldcg(A.Q + 2 * (b + 2 * h) + 1), rho);
                    p1 = e2_fold(e2_ldcg(A.P + 2 * (b + h)), e2_ldcg(A.P + 2 * (b + 3 * h)), rho);
                    r1 = e2_fold(e2_ldcg(A.P + 2 * (b + h) + 1), e2_ldcg(A.P + 2 * (b + 3 * h) + 1), rho);
                    q1 = e2_fold(e2_ldcg(A.Q + 2 * (b + h)), e2_ldcg(A.Q + 2 * (b + 3 * h)), rho);
                    s1 = e2_fold(e2_ldcg(A.Q + 2 * (b + h) + 1), e2_ldcg(A.Q + 2 * (b + 3 * h) + 1), rho);
                } else {
                    p0 = e2_fold(e2_ldcg(A.pl + b), e2_ldcg(A.pl + b + 2 * h), rho);
                    r0 = e2_fold(e2_ldcg(A.pr + b), e2_ldcg(A.pr + b + 2 * h), rho);
                    q0 = e2_fold(e2_ldcg(A.ql + b), e2_ldcg(A.ql + b + 2 * h), rho);
                    s0 = e2_fold(e2_ldcg(A.qr + b), e2_ldcg(A.qr + b + 2 * h), rho);
                    p1 = e2_fold(e2_ldcg(A.pl + b + h), e2_ldcg(A.pl + b + 3 * h), rho);
                    r1 = e2_fold(e2_ldcg(A.pr + b + h), e2_ldcg(A.pr + b + 3 * h), rho);
                    q1 = e2_fold(e2_ldcg(A.ql + b + h), e2_ldcg(A.ql + b + 3 * h), rho);
                    s1 = e2_fold(e2_ldcg(A.qr + b + h), e2_ldcg(A.qr + b + 3 * h), rho);
                }
                A.pl[b] = p0;
                A.pr[b] = r0;
                A.ql[b] = q0;
                A.qr[b] = s0;
                A.pl[b + h] = p1;
                A.pr[b + h] = r1;
                A.ql[b + h] = q1;
                A.qr[b + h] = s1;
                e = e2_add(e2_ldcg(A.E + b), e2_ldcg(A.E + b + h));  // eq(z_>t, b)
                A.E[b] = e;
            }
            const uint64_t e7 = gl_mul7(e.b);
            a0.mac(e, e7, x16_f(p0, r0, q0, s0, A.lam));
            if (need1) a1.mac(e, e7, x16_f(p1, r1, q1, s1, A.lam));
            a2.mac(e, e7, x16_f(e2_at2(p0, p1), e2_at2(r0, r1), e2_at2(q0, q1), e2_at2(s0, s1), A.lam));
        }
        uint64_t acc[6] = {a0.a.value(), a0.b.value(), a1.a.value(), a1.b.value(), a2.a.value(), a2.b.value()};
        bool last;
        if (active == 1) {
            block_sum_gl<6>(acc);
            last = true;
        } else {
            last = grid_sum_gl_n<6>(acc, part, &rl->ticket, active);
        }
        if (last && threadIdx.x == 0) session_publish(mb, acc, A.seq0 + t);  // {h(0), h(1), h(2)}
    }
    // block 0 folds the last pair of each vector by the last challenge: pL, pR, qL, qR at rho
    if (A.t_end <= A.d || blockIdx.x != 0) return;
    uint64_t ra, rb;
    if (!session_wait2(mb, rl, A.seq0 + A.d, ra, rb)) return;
    rho = e2_make(ra, rb);
    if (threadIdx.x == 0) {
        Ext2 f[4];
        if (A.d == 1) {
            f[0] = e2_fold(e2_ldcg(A.P), e2_ldcg(A.P + 2), rho);
            f[1] = e2_fold(e2_ldcg(A.P + 1), e2_ldcg(A.P + 3), rho);
            f[2] = e2_fold(e2_ldcg(A.Q), e2_ldcg(A.Q + 2), rho);
            f[3] = e2_fold(e2_ldcg(A.Q + 1), e2_ldcg(A.Q + 3), rho);
        } else {
            f[0] = e2_fold(e2_ldcg(A.pl), e2_ldcg(A.pl + 1), rho);
            f[1] = e2_fold(e2_ldcg(A.pr), e2_ldcg(A.pr + 1), rho);
            f[2] = e2_fold(e2_ldcg(A.ql), e2_ldcg(A.ql + 1), rho);
            f[3] = e2_fold(e2_ldcg(A.qr), e2_ldcg(A.qr + 1), rho);
        }
        const uint64_t fin[8] = {f[0].a, f[0].b, f[1].a, f[1].b, f[2].a, f[2].b, f[3].a, f[3].b};
        session_publish(mb, fin, A.seq0 + A.d + 1);
    }
}

// ---- the host half ------------------------------------------------------------

struct X16Labels {
    const char *site, *gamma, *m, *alpha, *l1, *mu, *lambda, *round, *chal, *fin, *leaf;
};
const X16Labels kSilu2 = {"silu2_site", "silu2_gamma", "silu2_m", "silu2_alpha", "silu2_l1", "silu2_mu",
                          "silu2_lambda", "silu2_round", "silu2_chal", "silu2_final", "silu2_leaf"};
const X16Labels kExp2 = {"exp2_site", "exp2_gamma", "exp2_m", "exp2_alpha", "exp2_l1", "exp2_mu",
                         "exp2_lambda", "exp2_round", "exp2_chal", "exp2_final", "exp2_leaf"};

// Where the device values come from. Each call returns FP_OK or an error status.
struct X16Source {
    virtual ~X16Source() {}
    virtual void abandon() {}  // the host stopped early: let a waiting kernel finish
    virtual int tree(Ext2 gamma, Ext2 alpha, Ext2 l1[4]) = 0;           // build the tree, layer one's values
    virtual int layer(int d, const Ext2* z, Ext2 lam) = 0;              // layer d's sum-check begins
    virtual int round(int d, int t, Ext2 h[3]) = 0;                     // its h(0), h(1), h(2)
    virtual int answer(int d, int t, Ext2 rho) = 0;
    virtual int finals(int d, Ext2 fin[4]) = 0;                         // pL, pR, qL, qR at rho
    virtual int leaf(const Ext2* z, int v, Ext2 out[2]) = 0;            // g~(z), s~(z) of the padded columns
};

size_t x16_proof_len(int64_t n) {
    int v = fp_log2_ceil((uint64_t)n);
    if (v < 1) v = 1;
    size_t len = 4 * 65536 + 64 + 32;
    for (int d = 1; d < v; d++) len += 64 * (size_t)d + 64;
    return len;
}

// The protocol after the site is absorbed and gamma squeezed, from the multiplicities on.
int x16_protocol(fp_ctx* c, fp_tx* tx, const X16Labels& lab, int v, Ext2 gamma, const uint32_t* m,
                 const uint8_t m_digest[32], X16Source& src, uint8_t* proof, size_t* proof_len) {
    int rc;
    size_t pos = 0;
    for (size_t j = 0; j < 65536; j++)
        for (int b = 0; b < 4; b++) proof[4 * j + b] = (uint8_t)(m[j] >> (8 * b));
    pos += 4 * 65536;
    fp_tx_absorb_raw(tx, lab.m, m_digest, 32);
    const Ext2 alpha = e2_squeeze_host(tx, lab.alpha);
    Ext2 l1[4];
    if ((rc = src.tree(gamma, alpha, l1))) return rc;
    e2_send_host(tx, lab.l1, l1, 4, proof, pos);
    Ext2 z[X16_MAX_V + 1];
    z[0] = e2_squeeze_host(tx, lab.mu);
    Ext2 cP = e2_fold_host(l1[0], l1[1], z[0]), cQ = e2_fold_host(l1[2], l1[3], z[0]);
    const Ext2 one = e2_make(1, 0);
    for (int d = 1; d < v; d++) {
        const Ext2 lam = e2_squeeze_host(tx, lab.lambda);
        Ext2 claim = e2_add(cP, e2_mul(lam, cQ));
        if ((rc = src.layer(d, z, lam))) return rc;
        Ext2 pre = one;  // eq(z_<t, rho_<t)
        Ext2 rho[X16_MAX_V];
        for (int t = 1; t <= d; t++) {
            Ext2 h[3];
            if ((rc = src.round(d, t, h))) return rc;
            const Ext2 zt = z[t - 1];
            Ext2 g[4];
            e2_layer_round_values(h, pre, zt, claim, g);  // h(1) only from the device when z_t = 0
            if (!e2_same(e2_add(g[0], g[1]), claim)) {
                src.abandon();
                return fp_fail(c, FP_ERR_CUDA, "lookup over the extension: round values inconsistent with the claim");
            }
            e2_send_host(tx, lab.round, g, 4, proof, pos);
            const Ext2 r = e2_squeeze_host(tx, lab.chal);
            if ((rc = src.answer(d, t, r))) return rc;
            rho[t - 1] = r;
            claim = e2_lagrange4(g, r);
            pre = e2_mul(pre, e2_eq(zt, r));
        }
        Ext2 fin[4];
        if ((rc = src.finals(d, fin))) return rc;
        e2_send_host(tx, lab.fin, fin, 4, proof, pos);
        const Ext2 mu = e2_squeeze_host(tx, lab.mu);
        cP = e2_fold_host(fin[0], fin[1], mu);
        cQ = e2_fold_host(fin[2], fin[3], mu);
        for (int i = 0; i < d; i++) z[i] = rho[i];
        z[d] = mu;
    }
    Ext2 leaf[2];
    if ((rc = src.leaf(z, v, leaf))) return rc;
    e2_send_host(tx, lab.leaf, leaf, 2, proof, pos);
    *proof_len = pos;
    return FP_OK;
}


// ---- the rescale LogUp over the extension: two trees batched in one GKR ----------------
//
// The remainder table R_k (keys r) and the clamp table C16 (keys q + gamma y) as in
// logup_prove_rescale, every challenge and value in the extension, as a statement of
// its own over the sites' key columns (labels "lu2_*"). Each layer's summand is
// sum_tau lambda^(2 tau) (pL qR + pR qL + lambda qL qR) over both trees; a pair's two
// trees are folded one after the other to keep the live values few.

// m[key + off] += 1 for the keys inside [0, T); the rest counted in *outside
__global__ void lu2_hist_kernel(const int32_t* __restrict__ keys, int64_t n, int64_t T, int64_t off,
                                uint32_t* __restrict__ m, uint32_t* __restrict__ outside) {
    uint32_t out_local = 0;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t j = (int64_t)keys[i] + off;
        if (j >= 0 && j < T)
            atomicAdd(m + j, 1u);
        else
            out_local++;
    }
    if (out_local) atomicAdd(outside, out_local);
}

// m[q + 2^15] += 1 for q in [-2^15, 2^15); keys outside, and outputs y != clamp(q), counted in *outside
__global__ void lu2_hist_clamp_kernel(const int32_t* __restrict__ q, const int8_t* __restrict__ y, int64_t n,
                                      uint32_t* __restrict__ m, uint32_t* __restrict__ outside) {
    uint32_t out_local = 0;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t qv = q[i], j = qv + 32768;
        if (j >= 0 && j < 65536)
            atomicAdd(m + j, 1u);
        else
            out_local++;
        if ((int64_t)y[i] != (qv < -128 ? -128 : (qv > 127 ? 127 : qv))) out_local++;
    }
    if (out_local) atomicAdd(outside, out_local);
}

__global__ void lu2_add_pad_kernel(uint32_t* m_rem, int64_t half, uint32_t* m_clamp, uint32_t pad) {
    m_rem[half] += pad;
    m_clamp[32768] += pad;
}

// leaves of both trees: P = 1, Q_0 = alpha_0 - r, Q_1 = alpha_1 - (q + gamma y); zero keys past n
__global__ void lu2_leaf_kernel(const int32_t* __restrict__ r, const int32_t* __restrict__ q,
                                const int8_t* __restrict__ y, int64_t n, int64_t L, Ext2 alpha0, Ext2 alpha1,
                                Ext2 gamma, Ext2* __restrict__ P0, Ext2* __restrict__ Q0, Ext2* __restrict__ P1,
                                Ext2* __restrict__ Q1) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < L; i += (int64_t)gridDim.x * blockDim.x) {
        const uint64_t rv = i < n ? x16_lift(r[i]) : 0, qv = i < n ? x16_lift(q[i]) : 0;
        const uint64_t yv = i < n ? x16_lift(y[i]) : 0;
        P0[i] = e2_make(1, 0);
        P1[i] = e2_make(1, 0);
        Q0[i] = e2_sub(alpha0, e2_make(rv, 0));
        Q1[i] = e2_sub(alpha1, e2_make(gl_add(qv, gl_mul(gamma.a, yv)), gl_mul(gamma.b, yv)));
    }
}

struct Lu2Layer {
    const Ext2* P[2];  // tree layer d + 1 of each table: child x of node b is entry 2 b + x
    const Ext2* Q[2];
    Ext2* pl[2];       // folded children from round 2 on (2^(d-1) entries each)
    Ext2* pr[2];
    Ext2* ql[2];
    Ext2* qr[2];
    Ext2* E;           // suffix eq table (2^(d-1) entries)
    X16Point z;        // the layer's point z_1..z_d
    Ext2 lam, lam2;
    int d;
    int grid;
    int per_block;
    int pad;
    uint64_t seq0;  // round t publishes seq0 + t, the final values seq0 + d + 1
    int t_begin;    // rounds run by this launch: [t_begin, t_end]; t_end > d includes the final values
    int t_end;
};

__global__ void __launch_bounds__(X16_THREADS, 2) lu2_layer_kernel(Lu2Layer A, FpMailbox* mb, FpRelay* rl,
                                                                  uint64_t* part) {
    __shared__ Ext2 tab[4 << X16_CHUNK];
    Ext2 rho = e2_make(0, 0);
    for (int t = A.t_begin; t <= A.d && t <= A.t_end; t++) {
        if (t > 1) {
            uint64_t ra, rb;
            if (!session_wait2(mb, rl, A.seq0 + t - 1, ra, rb)) return;
            rho = e2_make(ra, rb);
        }
        const int64_t h = 1ll << (A.d - t);
        const int64_t want = (h + A.per_block - 1) / A.per_block;
        const unsigned active = (unsigned)(want < 1 ? 1 : (want > A.grid ? A.grid : want));
        if (blockIdx.x >= active) return;  // no pairs for this block in this or any later round
        int w[4] = {0, 0, 0, 0};
        if (t == 1) x16_tables(tab, A.z.z, A.d, w);
        // h(1) only when z_t = 0: otherwise the host takes it from the running claim
        const bool need1 = A.z.z[t - 1].a == 0 && A.z.z[t - 1].b == 0;
        E2Acc a0, a1, a2;
        for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < h; b += (int64_t)active * blockDim.x) {
            Ext2 F[3] = {e2_make(0, 0), e2_make(0, 0), e2_make(0, 0)};
#pragma unroll 1
            for (int tau = 0; tau < 2; tau++) {
                const Ext2* P = A.P[tau];
                const Ext2* Q = A.Q[tau];
                Ext2 p0, p1, r0, r1, q0, q1, s0, s1;  // pL, pR, qL, qR at the pair's two points
                if (t == 1) {
                    p0 = e2_ldcg(P + 2 * b);
                    r0 = e2_ldcg(P + 2 * b + 1);
                    q0 = e2_ldcg(Q + 2 * b);
                    s0 = e2_ldcg(Q + 2 * b + 1);
                    p1 = e2_ldcg(P + 2 * (b + h));
                    r1 = e2_ldcg(P + 2 * (b + h) + 1);
                    q1 = e2_ldcg(Q + 2 * (b + h));
                    s1 = e2_ldcg(Q + 2 * (b + h) + 1);
                } else {
                    if (t == 2) {
                        p0 = e2_fold(e2_ldcg(P + 2 * b), e2_ldcg(P + 2 * (b + 2 * h)), rho);
                        r0 = e2_fold(e2_ldcg(P + 2 * b + 1), e2_ldcg(P + 2 * (b + 2 * h) + 1), rho);
                        q0 = e2_fold(e2_ldcg(Q + 2 * b), e2_ldcg(Q + 2 * (b + 2 * h)), rho);
                        s0 = e2_fold(e2_ldcg(Q + 2 * b + 1), e2_ldcg(Q + 2 * (b + 2 * h) + 1), rho);
                        p1 = e2_fold(e2_ldcg(P + 2 * (b + h)), e2_ldcg(P + 2 * (b + 3 * h)), rho);
                        r1 = e2_fold(e2_ldcg(P + 2 * (b + h) + 1), e2_ldcg(P + 2 * (b + 3 * h) + 1), rho);
                        q1 = e2_fold(e2_ldcg(Q + 2 * (b + h)), e2_ldcg(Q + 2 * (b + 3 * h)), rho);
                        s1 = e2_fold(e2_ldcg(Q + 2 * (b + h) + 1), e2_ldcg(Q + 2 * (b + 3 * h) + 1), rho);
                    } else {
                        p0 = e2_fold(e2_ldcg(A.pl[tau] + b), e2_ldcg(A.pl[tau] + b + 2 * h), rho);
                        r0 = e2_fold(e2_ldcg(A.pr[tau] + b), e2_ldcg(A.pr[tau] + b + 2 * h), rho);
                        q0 = e2_fold(e2_ldcg(A.ql[tau] + b), e2_ldcg(A.ql[tau] + b + 2 * h), rho);
                        s0 = e2_fold(e2_ldcg(A.qr[tau] + b), e2_ldcg(A.qr[tau] + b + 2 * h), rho);
                        p1 = e2_fold(e2_ldcg(A.pl[tau] + b + h), e2_ldcg(A.pl[tau] + b + 3 * h), rho);
                        r1 = e2_fold(e2_ldcg(A.pr[tau] + b + h), e2_ldcg(A.pr[tau] + b + 3 * h), rho);
                        q1 = e2_fold(e2_ldcg(A.ql[tau] + b + h), e2_ldcg(A.ql[tau] + b + 3 * h), rho);
                        s1 = e2_fold(e2_ldcg(A.qr[tau] + b + h), e2_ldcg(A.qr[tau] + b + 3 * h), rho);
                    }
                    A.pl[tau][b] = p0;
                    A.pr[tau][b] = r0;
                    A.ql[tau][b] = q0;
                    A.qr[tau][b] = s0;
                    A.pl[tau][b + h] = p1;
                    A.pr[tau][b + h] = r1;
                    A.ql[tau][b + h] = q1;
                    A.qr[tau][b + h] = s1;
                }
                Ext2 f0 = x16_f(p0, r0, q0, s0, A.lam), f1 = e2_make(0, 0);
                if (need1) f1 = x16_f(p1, r1, q1, s1, A.lam);
                Ext2 f2 = x16_f(e2_at2(p0, p1), e2_at2(r0, r1), e2_at2(q0, q1), e2_at2(s0, s1), A.lam);
                if (tau == 1) {
                    f0 = e2_mul(A.lam2, f0);
                    if (need1) f1 = e2_mul(A.lam2, f1);
                    f2 = e2_mul(A.lam2, f2);
                }
                F[0] = e2_add(F[0], f0);
                F[1] = e2_add(F[1], f1);
                F[2] = e2_add(F[2], f2);
            }
            Ext2 e;
            if (t == 1) {
                e = x16_eq_at(tab, w, b);  // eq(z_2..z_d, b)
                if (A.d > 1) A.E[b] = e;
            } else {
                e = e2_add(e2_ldcg(A.E + b), e2_ldcg(A.E + b + h));  // eq(z_>t, b)
                A.E[b] = e;
            }
            const uint64_t e7 = gl_mul7(e.b);
            a0.mac(e, e7, F[0]);
            if (need1) a1.mac(e, e7, F[1]);
            a2.mac(e, e7, F[2]);
        }
        uint64_t acc[6] = {a0.a.value(), a0.b.value(), a1.a.value(), a1.b.value(), a2.a.value(), a2.b.value()};
        bool last;
        if (active == 1) {
            block_sum_gl<6>(acc);
            last = true;
        } else {
            last = grid_sum_gl_n<6>(acc, part, &rl->ticket, active);
        }
        if (last && threadIdx.x == 0) session_publish(mb, acc, A.seq0 + t);  // {h(0), h(1), h(2)}
    }
    // block 0 folds the last pair of each of the eight vectors by the last challenge
    if (A.t_end <= A.d || blockIdx.x != 0) return;
    uint64_t ra, rb;
    if (!session_wait2(mb, rl, A.seq0 + A.d, ra, rb)) return;
    rho = e2_make(ra, rb);
    if (threadIdx.x == 0) {
        uint64_t fin[16];
        for (int tau = 0; tau < 2; tau++) {
            Ext2 f[4];
            if (A.d == 1) {
                f[0] = e2_fold(e2_ldcg(A.P[tau]), e2_ldcg(A.P[tau] + 2), rho);
                f[1] = e2_fold(e2_ldcg(A.P[tau] + 1), e2_ldcg(A.P[tau] + 3), rho);
                f[2] = e2_fold(e2_ldcg(A.Q[tau]), e2_ldcg(A.Q[tau] + 2), rho);
                f[3] = e2_fold(e2_ldcg(A.Q[tau] + 1), e2_ldcg(A.Q[tau] + 3), rho);
            } else {
                f[0] = e2_fold(e2_ldcg(A.pl[tau]), e2_ldcg(A.pl[tau] + 1), rho);
                f[1] = e2_fold(e2_ldcg(A.pr[tau]), e2_ldcg(A.pr[tau] + 1), rho);
                f[2] = e2_fold(e2_ldcg(A.ql[tau]), e2_ldcg(A.ql[tau] + 1), rho);
                f[3] = e2_fold(e2_ldcg(A.qr[tau]), e2_ldcg(A.qr[tau] + 1), rho);
            }
            for (int i = 0; i < 4; i++) {
                fin[8 * tau + 2 * i] = f[i].a;
                fin[8 * tau + 2 * i + 1] = f[i].b;
            }
        }
        session_publish(mb, fin, A.seq0 + A.d + 1);
    }
}

// Where the device values come from. Each call returns FP_OK or an error status.
struct Lu2Source {
    virtual ~Lu2Source() {}
    virtual void abandon() {}
    virtual int tree(Ext2 gamma, Ext2 alpha0, Ext2 alpha1, Ext2 l1[8]) = 0;  // both trees, layer one
    virtual int layer(int d, const Ext2* z, Ext2 lam) = 0;
    virtual int round(int t, Ext2 h[3]) = 0;
    virtual int answer(int d, int t, Ext2 rho) = 0;
    virtual int finals(int d, Ext2 fin[8]) = 0;                               // both trees' children at rho
    virtual int leaf(const Ext2* z, int v, Ext2 out[3]) = 0;                  // r~(z), q~(z), y~(z)
};

size_t lu2_proof_len(int v, int k) {
    size_t len = 4 * ((size_t)1 << k) + 4 * 65536 + 128 + 48;
    for (int d = 1; d < v; d++) len += 64 * (size_t)d + 128;
    return len;
}

// The protocol after "lu2_site" is absorbed, from the multiplicities on.
int lu2_protocol(fp_ctx* c, fp_tx* tx, int v, int k, const uint32_t* m_rem, const uint8_t d_rem[32],
                 const uint32_t* m_clamp, const uint8_t d_clamp[32], Lu2Source& src, uint8_t* proof,
                 size_t* proof_len) {
    int rc;
    size_t pos = 0;
    const size_t T = (size_t)1 << k;
    for (size_t j = 0; j < T; j++)
        for (int b = 0; b < 4; b++) proof[pos + 4 * j + b] = (uint8_t)(m_rem[j] >> (8 * b));
    pos += 4 * T;
    fp_tx_absorb_raw(tx, "lu2_m_rem", d_rem, 32);
    const Ext2 gamma = e2_squeeze_host(tx, "lu2_gamma");
    for (size_t j = 0; j < 65536; j++)
        for (int b = 0; b < 4; b++) proof[pos + 4 * j + b] = (uint8_t)(m_clamp[j] >> (8 * b));
    pos += 4 * 65536;
    fp_tx_absorb_raw(tx, "lu2_m_clamp", d_clamp, 32);
    const Ext2 alpha0 = e2_squeeze_host(tx, "lu2_alpha");
    const Ext2 alpha1 = e2_squeeze_host(tx, "lu2_alpha");
    Ext2 l1[8];
    if ((rc = src.tree(gamma, alpha0, alpha1, l1))) return rc;
    e2_send_host(tx, "lu2_l1", l1, 8, proof, pos);
    Ext2 z[X16_MAX_V + 1];
    z[0] = e2_squeeze_host(tx, "lu2_mu");
    Ext2 cP[2], cQ[2];
    for (int tau = 0; tau < 2; tau++) {
        cP[tau] = e2_fold_host(l1[4 * tau], l1[4 * tau + 1], z[0]);
        cQ[tau] = e2_fold_host(l1[4 * tau + 2], l1[4 * tau + 3], z[0]);
    }
    const Ext2 one = e2_make(1, 0);
    for (int d = 1; d < v; d++) {
        const Ext2 lam = e2_squeeze_host(tx, "lu2_lambda");
        const Ext2 lam2 = e2_mul(lam, lam), lam3 = e2_mul(lam2, lam);
        Ext2 claim = e2_add(e2_add(cP[0], e2_mul(lam, cQ[0])), e2_add(e2_mul(lam2, cP[1]), e2_mul(lam3, cQ[1])));
        if ((rc = src.layer(d, z, lam))) return rc;
        Ext2 pre = one;
        Ext2 rho[X16_MAX_V];
        for (int t = 1; t <= d; t++) {
            Ext2 h[3];
            if ((rc = src.round(t, h))) return rc;
            const Ext2 zt = z[t - 1];
            Ext2 g[4];
            e2_layer_round_values(h, pre, zt, claim, g);  // h(1) only from the device when z_t = 0
            if (!e2_same(e2_add(g[0], g[1]), claim)) {
                src.abandon();
                return fp_fail(c, FP_ERR_CUDA, "logup_prove_rescale_ext2: round values inconsistent with the claim");
            }
            e2_send_host(tx, "lu2_round", g, 4, proof, pos);
            const Ext2 r = e2_squeeze_host(tx, "lu2_chal");
            if ((rc = src.answer(d, t, r))) return rc;
            rho[t - 1] = r;
            claim = e2_lagrange4(g, r);
            pre = e2_mul(pre, e2_eq(zt, r));
        }
        Ext2 fin[8];
        if ((rc = src.finals(d, fin))) return rc;
        e2_send_host(tx, "lu2_final", fin, 8, proof, pos);
        const Ext2 mu = e2_squeeze_host(tx, "lu2_mu");
        for (int tau = 0; tau < 2; tau++) {
            cP[tau] = e2_fold_host(fin[4 * tau], fin[4 * tau + 1], mu);
            cQ[tau] = e2_fold_host(fin[4 * tau + 2], fin[4 * tau + 3], mu);
        }
        for (int i = 0; i < d; i++) z[i] = rho[i];
        z[d] = mu;
    }
    Ext2 leaf[3];
    if ((rc = src.leaf(z, v, leaf))) return rc;
    e2_send_host(tx, "lu2_leaf", leaf, 3, proof, pos);
    *proof_len = pos;
    return FP_OK;
}

// Device values from the kernels above.
struct X16Device : X16Source {
    fp_ctx* c;
    cudaStream_t st;
    const int16_t* g;
    const int16_t* s;
    int64_t n;
    int64_t pad_s;
    int v;
    std::vector<Ext2*> TP, TQ;
    Ext2* vecs[5];
    Ext2 *EH, *EL;
    uint64_t *part, *small, *hs;
    X16Layer A;
    int cap_grid = 1;

    void abandon() override { fp_session_abandon(c, st); }

    int tree(Ext2 gamma, Ext2 alpha, Ext2 l1[4]) override {
        const int64_t L = 1ll << v;
        int slot;
        fp_tic(c, st, K_X16_TREE, 4.0 * (double)n + 64.0 * (double)L, &slot);
        x16_leaf_kernel<<<fp_grid256(c, L), 256, 0, st>>>(g, s, n, L, alpha, gamma, pad_s, TP[v], TQ[v]);
        FP_CUDA(c, cudaGetLastError());
        for (int d = v - 1; d >= 1; d--) {
            x16_level_kernel<<<fp_grid256(c, 1ll << d), 256, 0, st>>>(TP[d + 1], TQ[d + 1], 1ll << d, TP[d], TQ[d]);
            FP_CUDA(c, cudaGetLastError());
            c->launches++;
        }
        fp_toc(c, st, slot);
        FP_CUDA(c, cudaMemcpyAsync(hs, TP[1], 32, cudaMemcpyDeviceToHost, st));
        FP_CUDA(c, cudaMemcpyAsync(hs + 4, TQ[1], 32, cudaMemcpyDeviceToHost, st));
        FP_CUDA(c, cudaStreamSynchronize(st));
        l1[0] = e2_make(hs[0], hs[1]);
        l1[1] = e2_make(hs[2], hs[3]);
        l1[2] = e2_make(hs[4], hs[5]);
        l1[3] = e2_make(hs[6], hs[7]);
        return FP_OK;
    }

    double round_bytes(int t) const {
        const double pairs = (double)(1ll << (A.d - t));
        return (t == 1 ? 160.0 : 320.0) * pairs;  // four 16-byte child vectors and the eq table
    }

    int launch(int t_begin, int t_end, unsigned grid, double bytes) {
        A.t_begin = t_begin;
        A.t_end = t_end;
        void* args[] = {&A, &c->mb_dev, &c->relay, &part};
        int slot;
        fp_tic(c, st, K_X16_ROUND, bytes, &slot);
        FP_CUDA(c, cudaLaunchCooperativeKernel((const void*)x16_layer_kernel, dim3(grid), dim3(X16_THREADS), args, 0,
                                               st));
        fp_toc(c, st, slot);
        return FP_OK;
    }

    int layer(int d, const Ext2* z, Ext2 lam) override {
        int rc;
        memset(&A, 0, sizeof A);
        A.P = TP[d + 1];
        A.Q = TQ[d + 1];
        A.pl = vecs[0];
        A.pr = vecs[1];
        A.ql = vecs[2];
        A.qr = vecs[3];
        A.E = vecs[4];
        for (int i = 0; i < d; i++) A.z.z[i] = z[i];
        A.z.v = d;
        A.lam = lam;
        A.d = d;
        A.per_block = X16_THREADS;  // one pair per thread
        const int64_t half = 1ll << (d - 1);
        A.grid = (int)std::max<int64_t>(1, std::min<int64_t>((half + A.per_block - 1) / A.per_block, cap_grid));
        A.seq0 = fp_seq_reserve(c, (uint64_t)d + 2);
        if ((rc = fp_session_begin(c, st))) return rc;
        fp_session_expect(c, 6);  // before any launch: round 1 publishes without a challenge
        if (!c->stepped) {
            double bytes = 0;
            for (int t = 1; t <= d; t++) bytes += round_bytes(t);
            return launch(1, d + 1, (unsigned)A.grid, bytes);
        }
        return FP_OK;
    }

    int round(int d, int t, Ext2 h[3]) override {
        (void)d;
        int rc;
        if (c->stepped && (rc = launch(t, t, (unsigned)A.grid, round_bytes(t)))) return rc;
        if ((rc = fp_session_wait(c, A.seq0 + t, st))) return rc;
        for (int i = 0; i < 3; i++) h[i] = e2_make(c->mb->res[2 * i], c->mb->res[2 * i + 1]);
        return FP_OK;
    }

    int answer(int d, int t, Ext2 rho) override {
        fp_session_expect(c, t < d ? 6 : 8);  // the last challenge triggers the four final values
        fp_session_post2(c, A.seq0 + t, rho.a, rho.b);
        return FP_OK;
    }

    int finals(int d, Ext2 fin[4]) override {
        int rc;
        if (c->stepped && (rc = launch(d + 1, d + 1, 1, 128.0))) return rc;
        if ((rc = fp_session_wait(c, A.seq0 + d + 1, st))) return rc;
        for (int i = 0; i < 4; i++) fin[i] = e2_make(c->mb->res[2 * i], c->mb->res[2 * i + 1]);
        FP_CUDA(c, cudaStreamSynchronize(st));
        return FP_OK;
    }

    int leaf(const Ext2* z, int vv, Ext2 out[2]) override {
        const int vl = vv / 2, vh = vv - vl;
        X16Point ph, pl;
        memset(&ph, 0, sizeof ph);
        memset(&pl, 0, sizeof pl);
        ph.v = vh;
        pl.v = vl;
        for (int i = 0; i < vh; i++) ph.z[i] = z[i];
        for (int i = 0; i < vl; i++) pl.z[i] = z[vh + i];
        const unsigned blocks =
            (unsigned)std::max<int64_t>(1, std::min<int64_t>((n + 255) / 256, 2 * (int64_t)c->num_sms));
        int slot;
        fp_tic(c, st, K_X16_LEAF, 4.0 * (double)n, &slot);
        x16_eq_kernel<<<fp_grid256(c, 1ll << vh), 256, 0, st>>>(ph, EH);
        x16_eq_kernel<<<fp_grid256(c, 1ll << vl), 256, 0, st>>>(pl, EL);
        x16_mle_kernel<int16_t><<<blocks, 256, 0, st>>>(g, n, EH, EL, vl, part, c->tickets, small);
        x16_mle_kernel<int16_t><<<blocks, 256, 0, st>>>(s, n, EH, EL, vl, part, c->tickets, small + 4);
        fp_toc(c, st, slot);
        FP_CUDA(c, cudaGetLastError());
        c->launches += 3;  // four kernels under one timing slot
        FP_CUDA(c, cudaMemcpyAsync(hs, small, 64, cudaMemcpyDeviceToHost, st));
        FP_CUDA(c, cudaStreamSynchronize(st));
        out[0] = e2_make(hs[0], hs[1]);
        // the s column past n holds the padding value: it adds pad_s (1 - sum_{x < n} eq(z, x))
        const Ext2 eqsum = e2_make(hs[6], hs[7]);
        const uint64_t padf = gl_from_i64(pad_s);
        out[1] = e2_add(e2_make(hs[4], hs[5]), e2_scal(e2_sub(e2_make(1, 0), eqsum), padf));
        return FP_OK;
    }
};

// Device values from a caller's callback (no device).
struct X16Callback : X16Source {
    fp_values_fn fn;
    void* user;
    int call(int kind, int t, const uint64_t* in, uint64_t* out) { return fn(user, kind, t, in, out) ? FP_ERR_ARG : FP_OK; }
    static Ext2 ext(const uint64_t* w) { return e2_make(gl_canon(w[0]), gl_canon(w[1])); }
    int tree(Ext2 gamma, Ext2 alpha, Ext2 l1[4]) override {
        const uint64_t in[4] = {gamma.a, gamma.b, alpha.a, alpha.b};
        uint64_t out[8] = {0};
        const int rc = call(FP_VAL_COLUMN, 0, in, out);
        for (int i = 0; i < 4; i++) l1[i] = ext(out + 2 * i);
        return rc;
    }
    int layer(int d, const Ext2* z, Ext2 lam) override {
        uint64_t in[2 * X16_MAX_V + 4];
        for (int i = 0; i < d; i++) {
            in[2 * i] = z[i].a;
            in[2 * i + 1] = z[i].b;
        }
        in[2 * d] = lam.a;
        in[2 * d + 1] = lam.b;
        return call(FP_VAL_START, d, in, nullptr);
    }
    int round(int d, int t, Ext2 h[3]) override {
        (void)d;
        uint64_t out[6] = {0};
        const int rc = call(FP_VAL_ROUND, t, nullptr, out);
        for (int i = 0; i < 3; i++) h[i] = ext(out + 2 * i);
        return rc;
    }
    int answer(int d, int t, Ext2 rho) override {
        (void)d;
        const uint64_t in[2] = {rho.a, rho.b};
        return call(FP_VAL_ANSWER, t, in, nullptr);
    }
    int finals(int d, Ext2 fin[4]) override {
        (void)d;
        uint64_t out[8] = {0};
        const int rc = call(FP_VAL_FINALS, 0, nullptr, out);
        for (int i = 0; i < 4; i++) fin[i] = ext(out + 2 * i);
        return rc;
    }
    int leaf(const Ext2* z, int v, Ext2 out2[2]) override {
        uint64_t in[2 * X16_MAX_V + 2];
        for (int i = 0; i < v; i++) {
            in[2 * i] = z[i].a;
            in[2 * i + 1] = z[i].b;
        }
        uint64_t out[4] = {0};
        const int rc = call(FP_VAL_CLAIM, v, in, out);
        out2[0] = ext(out);
        out2[1] = ext(out + 2);
        return rc;
    }
};


// Device values from the kernels above.
struct Lu2Device : Lu2Source {
    fp_ctx* c;
    cudaStream_t st;
    const int32_t* r;
    const int32_t* q;
    const int8_t* y;
    int64_t n;
    int v;
    std::vector<Ext2*> TP[2], TQ[2];
    Ext2* vec[9];  // pl, pr, ql, qr of table 0, then of table 1, then E
    Ext2 *EH, *EL;
    uint64_t *part, *small, *hs;
    Lu2Layer A;
    int cap_grid = 1;

    void abandon() override { fp_session_abandon(c, st); }

    int tree(Ext2 gamma, Ext2 alpha0, Ext2 alpha1, Ext2 l1[8]) override {
        const int64_t L = 1ll << v;
        int slot;
        fp_tic(c, st, K_LU2_TREE, 9.0 * (double)n + 128.0 * (double)L, &slot);
        lu2_leaf_kernel<<<fp_grid256(c, L), 256, 0, st>>>(r, q, y, n, L, alpha0, alpha1, gamma, TP[0][v], TQ[0][v],
                                                         TP[1][v], TQ[1][v]);
        FP_CUDA(c, cudaGetLastError());
        for (int tau = 0; tau < 2; tau++)
            for (int d = v - 1; d >= 1; d--) {
                x16_level_kernel<<<fp_grid256(c, 1ll << d), 256, 0, st>>>(TP[tau][d + 1], TQ[tau][d + 1], 1ll << d,
                                                                        TP[tau][d], TQ[tau][d]);
                FP_CUDA(c, cudaGetLastError());
                c->launches++;
            }
        fp_toc(c, st, slot);
        for (int tau = 0; tau < 2; tau++) {
            FP_CUDA(c, cudaMemcpyAsync(hs + 8 * tau, TP[tau][1], 32, cudaMemcpyDeviceToHost, st));
            FP_CUDA(c, cudaMemcpyAsync(hs + 8 * tau + 4, TQ[tau][1], 32, cudaMemcpyDeviceToHost, st));
        }
        FP_CUDA(c, cudaStreamSynchronize(st));
        for (int i = 0; i < 8; i++) l1[i] = e2_make(hs[2 * i], hs[2 * i + 1]);  // P(0), P(1), Q(0), Q(1) per table
        return FP_OK;
    }

    double round_bytes(int t) const {
        const double pairs = (double)(1ll << (A.d - t));
        return (t == 1 ? 288.0 : 576.0) * pairs;  // eight 16-byte child vectors and the eq table
    }

    int launch(int t_begin, int t_end, unsigned grid, double bytes) {
        A.t_begin = t_begin;
        A.t_end = t_end;
        void* args[] = {&A, &c->mb_dev, &c->relay, &part};
        int slot;
        fp_tic(c, st, K_LU2_ROUND, bytes, &slot);
        FP_CUDA(c, cudaLaunchCooperativeKernel((const void*)lu2_layer_kernel, dim3(grid), dim3(X16_THREADS), args, 0,
                                               st));
        fp_toc(c, st, slot);
        return FP_OK;
    }

    int layer(int d, const Ext2* z, Ext2 lam) override {
        int rc;
        memset(&A, 0, sizeof A);
        for (int tau = 0; tau < 2; tau++) {
            A.P[tau] = TP[tau][d + 1];
            A.Q[tau] = TQ[tau][d + 1];
            A.pl[tau] = vec[4 * tau];
            A.pr[tau] = vec[4 * tau + 1];
            A.ql[tau] = vec[4 * tau + 2];
            A.qr[tau] = vec[4 * tau + 3];
        }
        A.E = vec[8];
        for (int i = 0; i < d; i++) A.z.z[i] = z[i];
        A.z.v = d;
        A.lam = lam;
        A.lam2 = e2_mul(lam, lam);
        A.d = d;
        A.per_block = X16_THREADS;  // one pair per thread
        const int64_t half = 1ll << (d - 1);
        A.grid = (int)std::max<int64_t>(1, std::min<int64_t>((half + A.per_block - 1) / A.per_block, cap_grid));
        A.seq0 = fp_seq_reserve(c, (uint64_t)d + 2);
        if ((rc = fp_session_begin(c, st))) return rc;
        fp_session_expect(c, 6);  // before any launch: round 1 publishes without a challenge
        if (!c->stepped) {
            double bytes = 0;
            for (int t = 1; t <= d; t++) bytes += round_bytes(t);
            return launch(1, d + 1, (unsigned)A.grid, bytes);
        }
        return FP_OK;
    }

    int round(int t, Ext2 h[3]) override {
        int rc;
        if (c->stepped && (rc = launch(t, t, (unsigned)A.grid, round_bytes(t)))) return rc;
        if ((rc = fp_session_wait(c, A.seq0 + t, st))) return rc;
        for (int i = 0; i < 3; i++) h[i] = e2_make(c->mb->res[2 * i], c->mb->res[2 * i + 1]);
        return FP_OK;
    }

    int answer(int d, int t, Ext2 rho) override {
        fp_session_expect(c, t < d ? 6 : 16);  // the last challenge triggers the sixteen final words
        fp_session_post2(c, A.seq0 + t, rho.a, rho.b);
        return FP_OK;
    }

    int finals(int d, Ext2 fin[8]) override {
        int rc;
        if (c->stepped && (rc = launch(d + 1, d + 1, 1, 256.0))) return rc;
        if ((rc = fp_session_wait(c, A.seq0 + d + 1, st))) return rc;
        for (int i = 0; i < 8; i++) fin[i] = e2_make(c->mb->res[2 * i], c->mb->res[2 * i + 1]);
        FP_CUDA(c, cudaStreamSynchronize(st));
        return FP_OK;
    }

    int leaf(const Ext2* z, int vv, Ext2 out[3]) override {
        const int vl = vv / 2, vh = vv - vl;
        X16Point ph, pl;
        memset(&ph, 0, sizeof ph);
        memset(&pl, 0, sizeof pl);
        ph.v = vh;
        pl.v = vl;
        for (int i = 0; i < vh; i++) ph.z[i] = z[i];
        for (int i = 0; i < vl; i++) pl.z[i] = z[vh + i];
        const unsigned blocks =
            (unsigned)std::max<int64_t>(1, std::min<int64_t>((n + 255) / 256, 2 * (int64_t)c->num_sms));
        int slot;
        fp_tic(c, st, K_LU2_LEAF, 9.0 * (double)n, &slot);
        x16_eq_kernel<<<fp_grid256(c, 1ll << vh), 256, 0, st>>>(ph, EH);
        x16_eq_kernel<<<fp_grid256(c, 1ll << vl), 256, 0, st>>>(pl, EL);
        x16_mle_kernel<int32_t><<<blocks, 256, 0, st>>>(r, n, EH, EL, vl, part, c->tickets, small);
        x16_mle_kernel<int32_t><<<blocks, 256, 0, st>>>(q, n, EH, EL, vl, part, c->tickets, small + 4);
        x16_mle_kernel<int8_t><<<blocks, 256, 0, st>>>(y, n, EH, EL, vl, part, c->tickets, small + 8);
        fp_toc(c, st, slot);
        FP_CUDA(c, cudaGetLastError());
        c->launches += 4;  // five kernels under one timing slot
        FP_CUDA(c, cudaMemcpyAsync(hs, small, 96, cudaMemcpyDeviceToHost, st));
        FP_CUDA(c, cudaStreamSynchronize(st));
        // the padding keys are zero in all three columns: no correction
        for (int i = 0; i < 3; i++) out[i] = e2_make(hs[4 * i], hs[4 * i + 1]);
        return FP_OK;
    }
};

// Device values from a caller's callback (no device).
struct Lu2Callback : Lu2Source {
    fp_values_fn fn;
    void* user;
    int call(int kind, int t, const uint64_t* in, uint64_t* out) { return fn(user, kind, t, in, out) ? FP_ERR_ARG : FP_OK; }
    static Ext2 ext(const uint64_t* w) { return e2_make(gl_canon(w[0]), gl_canon(w[1])); }
    int tree(Ext2 gamma, Ext2 alpha0, Ext2 alpha1, Ext2 l1[8]) override {
        const uint64_t in[6] = {gamma.a, gamma.b, alpha0.a, alpha0.b, alpha1.a, alpha1.b};
        uint64_t out[16] = {0};
        const int rc = call(FP_VAL_COLUMN, 0, in, out);
        for (int i = 0; i < 8; i++) l1[i] = ext(out + 2 * i);
        return rc;
    }
    int layer(int d, const Ext2* z, Ext2 lam) override {
        uint64_t in[2 * X16_MAX_V + 4];
        for (int i = 0; i < d; i++) {
            in[2 * i] = z[i].a;
            in[2 * i + 1] = z[i].b;
        }
        in[2 * d] = lam.a;
        in[2 * d + 1] = lam.b;
        return call(FP_VAL_START, d, in, nullptr);
    }
    int round(int t, Ext2 h[3]) override {
        uint64_t out[6] = {0};
        const int rc = call(FP_VAL_ROUND, t, nullptr, out);
        for (int i = 0; i < 3; i++) h[i] = ext(out + 2 * i);
        return rc;
    }
    int answer(int d, int t, Ext2 rho) override {
        (void)d;
        const uint64_t in[2] = {rho.a, rho.b};
        return call(FP_VAL_ANSWER, t, in, nullptr);
    }
    int finals(int d, Ext2 fin[8]) override {
        (void)d;
        uint64_t out[16] = {0};
        const int rc = call(FP_VAL_FINALS, 0, nullptr, out);
        for (int i = 0; i < 8; i++) fin[i] = ext(out + 2 * i);
        return rc;
    }
    int leaf(const Ext2* z, int v, Ext2 out3[3]) override {
        uint64_t in[2 * X16_MAX_V + 2];
        for (int i = 0; i < v; i++) {
            in[2 * i] = z[i].a;
            in[2 * i + 1] = z[i].b;
        }
        uint64_t out[6] = {0};
        const int rc = call(FP_VAL_CLAIM, v, in, out);
        for (int i = 0; i < 3; i++) out3[i] = ext(out + 2 * i);
        return rc;
    }
};

int x16_prove(fp_ctx* c, fp_tx* tx, const X16Labels& lab, int64_t pad_s, const int16_t* g, const int16_t* s, int64_t n,
              uint8_t* proof, size_t* proof_len, void* stream, const char* who) {
    if (!c || !tx || !proof_len) return fp_fail(c, FP_ERR_ARG, std::string(who) + ": null argument");
    if (!g || !s) return fp_fail(c, FP_ERR_ARG, std::string(who) + ": null column");
    if (n < 1 || n > (1ll << X16_MAX_V)) return fp_fail(c, FP_ERR_SHAPE, std::string(who) + ": need 1 <= n <= 2^30");
    const size_t need_len = x16_proof_len(n);
    if (!proof || *proof_len < need_len) {
        *proof_len = need_len;
        return fp_fail(c, FP_ERR_ARG, std::string(who) + ": proof buffer too small");
    }
    FP_CUDA(c, cudaSetDevice(c->device));
    cudaStream_t st = (cudaStream_t)stream;
    int rc;
    int v = fp_log2_ceil((uint64_t)n);
    if (v < 1) v = 1;
    const int64_t L = 1ll << v;
    {
        FpDigestJob jobs[2] = {{(const uint8_t*)g, 2 * (uint64_t)n}, {(const uint8_t*)s, 2 * (uint64_t)n}};
        uint8_t d[64];
        if ((rc = fp_digest_many(c, jobs, 2, d, st))) return rc;  // synchronises the stream
        fp_tx_absorb_raw(tx, lab.site, d, 64);
    }
    const Ext2 gamma = e2_squeeze_host(tx, lab.gamma);

    X16Device dev;
    dev.c = c;
    dev.st = st;
    dev.g = g;
    dev.s = s;
    dev.n = n;
    dev.pad_s = pad_s;
    dev.v = v;
    int occ = 0;
    FP_CUDA(c, cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, x16_layer_kernel, X16_THREADS, 0));
    dev.cap_grid = std::max(1, occ) * c->num_sms;
    const size_t part_n = (size_t)6 * std::max(dev.cap_grid, 4 * c->num_sms);
    const int64_t hv = v >= 2 ? 1ll << (v - 2) : 1;  // the largest layer's vectors: 2^(d-1) for d = v - 1
    const int vl = v / 2, vh = v - vl;
    size_t need = fp_align_up(4 * 65536, 256) + fp_align_up(8 * part_n, 256) + fp_align_up(8 * 64, 256) +
                  fp_align_up((size_t)16 << vh, 256) + fp_align_up((size_t)16 << vl, 256) +
                  5 * fp_align_up((size_t)16 * hv, 256) + 4096;
    for (int d = 1; d <= v; d++) need += 2 * fp_align_up((size_t)16 << d, 256);
    need += fp_hist::hist16_scratch();
    if ((rc = fp_reserve(c, c->dev, need))) return rc;
    if ((rc = fp_reserve(c, c->host, 4 * 65536 + 8192))) return rc;
    fp_reset(c->dev);
    fp_reset(c->host);
    uint32_t* m = (uint32_t*)fp_alloc(c->dev, 4 * 65536);
    uint32_t* hpart = (uint32_t*)fp_alloc(c->dev, fp_hist::hist16_scratch());
    dev.part = (uint64_t*)fp_alloc(c->dev, 8 * part_n);
    dev.small = (uint64_t*)fp_alloc(c->dev, 8 * 64);
    dev.EH = (Ext2*)fp_alloc(c->dev, (size_t)16 << vh);
    dev.EL = (Ext2*)fp_alloc(c->dev, (size_t)16 << vl);
    for (int i = 0; i < 5; i++) dev.vecs[i] = (Ext2*)fp_alloc(c->dev, (size_t)16 * hv);
    dev.TP.assign(v + 1, nullptr);
    dev.TQ.assign(v + 1, nullptr);
    for (int d = 1; d <= v; d++) {
        dev.TP[d] = (Ext2*)fp_alloc(c->dev, (size_t)16 << d);
        dev.TQ[d] = (Ext2*)fp_alloc(c->dev, (size_t)16 << d);
        if (!dev.TP[d] || !dev.TQ[d]) return fp_fail(c, FP_ERR_OOM, std::string(who) + ": scratch exhausted");
    }
    uint32_t* hm = (uint32_t*)fp_alloc(c->host, 4 * 65536);
    dev.hs = (uint64_t*)fp_alloc(c->host, 8 * 64);
    if (!m || !hpart || !dev.part || !dev.small || !dev.EH || !dev.EL || !dev.vecs[4] || !hm || !dev.hs)
        return fp_fail(c, FP_ERR_OOM, std::string(who) + ": scratch exhausted");

    // ---- multiplicities ----
    {
        int slot;
        fp_tic(c, st, K_SILU_HIST, 2.0 * (double)n, &slot);
        rc = fp_hist::hist16(c, g, n, (uint32_t)(L - n), m, hpart, st);
        fp_toc(c, st, slot);
        if (rc) return rc;
    }
    FP_CUDA(c, cudaMemcpyAsync(hm, m, 4 * 65536, cudaMemcpyDeviceToHost, st));
    uint8_t dm[32];
    {
        FpDigestJob job = {(const uint8_t*)m, 4 * 65536ull};
        if ((rc = fp_digest_many(c, &job, 1, dm, st))) return rc;  // synchronises the stream
    }
    return x16_protocol(c, tx, lab, v, gamma, hm, dm, dev, proof, proof_len);
}

}  // namespace

int logup_prove_silu_ext2(fp_ctx* c, fp_tx* tx, const int16_t* g, const int16_t* s, int64_t n, uint8_t* proof,
                          size_t* proof_len, void* stream) {
    // keys are padded with the table's row for input 0: silu(0) = 0
    return x16_prove(c, tx, kSilu2, 0, g, s, n, proof, proof_len, stream, "logup_prove_silu_ext2");
}

int logup_prove_exp_ext2(fp_ctx* c, fp_tx* tx, const int16_t* g, const int16_t* s, int64_t n, uint8_t* proof,
                         size_t* proof_len, void* stream) {
    // keys are padded with the table's row for input 0: e^0 scaled to the 9-bit numerator, 511
    return x16_prove(c, tx, kExp2, 511, g, s, n, proof, proof_len, stream, "logup_prove_exp_ext2");
}

int fp_lookup16x_protocol_drive(fp_tx* tx, int table, int v, const uint64_t* gamma, const uint32_t* m,
                                const uint8_t* m_digest, fp_values_fn fn, void* user, uint8_t* proof,
                                size_t* proof_len) {
    if (!tx || !fn || !proof_len || !m || !m_digest || !gamma) return FP_ERR_ARG;
    if (table != 0 && table != 1) return FP_ERR_ARG;
    if (v < 1 || v > X16_MAX_V) return FP_ERR_SHAPE;
    const size_t need_len = x16_proof_len(1ll << v);
    if (!proof || *proof_len < need_len) {
        *proof_len = need_len;
        return FP_ERR_ARG;
    }
    X16Callback cb;
    cb.fn = fn;
    cb.user = user;
    return x16_protocol(nullptr, tx, table == 0 ? kSilu2 : kExp2, v, e2_make(gamma[0], gamma[1]), m, m_digest, cb,
                        proof, proof_len);
}

int logup_prove_rescale_ext2(fp_ctx* c, fp_tx* tx, const fp_site* sites, int nsites, uint8_t* proof,
                             size_t* proof_len, void* stream) {
    if (!c || !tx || !proof_len) return fp_fail(c, FP_ERR_ARG, "logup_prove_rescale_ext2: null argument");
    int rc;
    if ((rc = fp_check_sites(c, sites, nsites, true))) return rc;
    const int k = sites[0].k_shift;
    int64_t nk = 0;
    for (int i = 0; i < nsites; i++) {
        if (sites[i].k_shift != k)
            return fp_fail(c, FP_ERR_ARG, "logup_prove_rescale_ext2: every site needs the same k_shift");
        nk += (int64_t)sites[i].M * sites[i].N;
    }
    if (nk > (1ll << X16_MAX_V)) return fp_fail(c, FP_ERR_SHAPE, "logup_prove_rescale_ext2: more than 2^30 keys");
    const int v = std::max(1, fp_log2_ceil((uint64_t)nk));
    const size_t need_len = lu2_proof_len(v, k);
    if (!proof || *proof_len < need_len) {
        *proof_len = need_len;
        return fp_fail(c, FP_ERR_ARG, "logup_prove_rescale_ext2: proof buffer too small");
    }
    FP_CUDA(c, cudaSetDevice(c->device));
    cudaStream_t st = (cudaStream_t)stream;
    const int64_t L = 1ll << v, T = 1ll << k;
    Lu2Device dev;
    dev.c = c;
    dev.st = st;
    dev.n = nk;
    dev.v = v;
    int occ = 0;
    FP_CUDA(c, cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, lu2_layer_kernel, X16_THREADS, 0));
    dev.cap_grid = std::max(1, occ) * c->num_sms;
    const size_t part_n = (size_t)6 * std::max(dev.cap_grid, 4 * c->num_sms);
    const int64_t hv = v >= 2 ? 1ll << (v - 2) : 1;
    const int vl = v / 2, vh = v - vl;
    size_t need = 2 * fp_align_up((size_t)4 * nk, 256) + fp_align_up((size_t)nk, 256) + fp_align_up((size_t)4 * T, 256) +
                  fp_align_up(4 * 65536, 256) + fp_align_up(8 * part_n, 256) + 2 * fp_align_up(8 * 64, 256) +
                  fp_align_up((size_t)16 << vh, 256) + fp_align_up((size_t)16 << vl, 256) +
                  9 * fp_align_up((size_t)16 * hv, 256) + 4096;
    for (int d = 1; d <= v; d++) need += 4 * fp_align_up((size_t)16 << d, 256);
    if ((rc = fp_reserve(c, c->dev, need))) return rc;
    if ((rc = fp_reserve(c, c->host, fp_align_up((size_t)4 * T, 256) + 4 * 65536 + 8192))) return rc;
    fp_reset(c->dev);
    fp_reset(c->host);
    int32_t* r_all = (int32_t*)fp_alloc(c->dev, (size_t)4 * nk);
    int32_t* q_all = (int32_t*)fp_alloc(c->dev, (size_t)4 * nk);
    int8_t* y_all = (int8_t*)fp_alloc(c->dev, (size_t)nk);
    uint32_t* m_rem = (uint32_t*)fp_alloc(c->dev, (size_t)4 * T);
    uint32_t* m_cl = (uint32_t*)fp_alloc(c->dev, 4 * 65536);
    dev.part = (uint64_t*)fp_alloc(c->dev, 8 * part_n);
    dev.small = (uint64_t*)fp_alloc(c->dev, 8 * 64);
    uint32_t* outside = (uint32_t*)fp_alloc(c->dev, 8 * 64);
    dev.EH = (Ext2*)fp_alloc(c->dev, (size_t)16 << vh);
    dev.EL = (Ext2*)fp_alloc(c->dev, (size_t)16 << vl);
    bool ok = r_all && q_all && y_all && m_rem && m_cl && dev.part && dev.small && outside && dev.EH && dev.EL;
    for (int i = 0; i < 9; i++) ok = ok && (dev.vec[i] = (Ext2*)fp_alloc(c->dev, (size_t)16 * hv));
    for (int tau = 0; tau < 2; tau++) {
        dev.TP[tau].assign(v + 1, nullptr);
        dev.TQ[tau].assign(v + 1, nullptr);
        for (int d = 1; d <= v; d++) {
            ok = ok && (dev.TP[tau][d] = (Ext2*)fp_alloc(c->dev, (size_t)16 << d));
            ok = ok && (dev.TQ[tau][d] = (Ext2*)fp_alloc(c->dev, (size_t)16 << d));
        }
    }
    uint32_t* hm = (uint32_t*)fp_alloc(c->host, (size_t)4 * T + 4 * 65536);
    dev.hs = (uint64_t*)fp_alloc(c->host, 8 * 64);
    if (!ok || !hm || !dev.hs) return fp_fail(c, FP_ERR_OOM, "logup_prove_rescale_ext2: scratch exhausted");
    dev.r = r_all;
    dev.q = q_all;
    dev.y = y_all;

    // ---- the key columns, concatenated in site order ----
    int64_t o = 0;
    for (int i = 0; i < nsites; i++) {
        const int64_t mn = (int64_t)sites[i].M * sites[i].N;
        FP_CUDA(c, cudaMemcpyAsync(r_all + o, sites[i].r, 4 * (size_t)mn, cudaMemcpyDeviceToDevice, st));
        FP_CUDA(c, cudaMemcpyAsync(q_all + o, sites[i].q, 4 * (size_t)mn, cudaMemcpyDeviceToDevice, st));
        FP_CUDA(c, cudaMemcpyAsync(y_all + o, sites[i].y, (size_t)mn, cudaMemcpyDeviceToDevice, st));
        o += mn;
    }
    {
        FpDigestJob jobs[3] = {{(const uint8_t*)r_all, 4 * (uint64_t)nk}, {(const uint8_t*)q_all, 4 * (uint64_t)nk},
                               {(const uint8_t*)y_all, (uint64_t)nk}};
        uint8_t d[96];
        if ((rc = fp_digest_many(c, jobs, 3, d, st))) return rc;  // synchronises the stream
        fp_tx_absorb_raw(tx, "lu2_site", d, 96);
    }
    // ---- multiplicities ----
    FP_CUDA(c, cudaMemsetAsync(m_rem, 0, (size_t)4 * T, st));
    FP_CUDA(c, cudaMemsetAsync(m_cl, 0, 4 * 65536, st));
    FP_CUDA(c, cudaMemsetAsync(outside, 0, 4, st));
    {
        int slot;
        fp_tic(c, st, K_LU2_HIST, 9.0 * (double)nk, &slot);
        lu2_hist_kernel<<<fp_grid256(c, nk), 256, 0, st>>>(r_all, nk, T, T / 2, m_rem, outside);
        lu2_hist_clamp_kernel<<<fp_grid256(c, nk), 256, 0, st>>>(q_all, y_all, nk, m_cl, outside);
        if (L > nk) lu2_add_pad_kernel<<<1, 1, 0, st>>>(m_rem, T / 2, m_cl, (uint32_t)(L - nk));
        fp_toc(c, st, slot);
        FP_CUDA(c, cudaGetLastError());
        c->launches += L > nk ? 2 : 1;
    }
    FP_CUDA(c, cudaMemcpyAsync(hm, m_rem, (size_t)4 * T, cudaMemcpyDeviceToHost, st));
    FP_CUDA(c, cudaMemcpyAsync(hm + T, m_cl, 4 * 65536, cudaMemcpyDeviceToHost, st));
    FP_CUDA(c, cudaMemcpyAsync(dev.hs, outside, 4, cudaMemcpyDeviceToHost, st));
    uint8_t dm[64];
    {
        FpDigestJob jobs[2] = {{(const uint8_t*)m_rem, 4 * (uint64_t)T}, {(const uint8_t*)m_cl, 4 * 65536ull}};
        if ((rc = fp_digest_many(c, jobs, 2, dm, st))) return rc;  // synchronises the stream
    }
    uint32_t n_outside;
    memcpy(&n_outside, dev.hs, 4);
    if ((rc = lu2_protocol(c, tx, v, k, hm, dm, hm + T, dm + 32, dev, proof, proof_len))) return rc;
    return n_outside ? 1 : FP_OK;
}

int fp_lu2_protocol_drive(fp_tx* tx, int v, int k, const uint32_t* m_rem, const uint8_t* d_rem, const uint32_t* m_clamp,
                          const uint8_t* d_clamp, fp_values_fn fn, void* user, uint8_t* proof, size_t* proof_len) {
    if (!tx || !fn || !proof_len || !m_rem || !d_rem || !m_clamp || !d_clamp) return FP_ERR_ARG;
    if (v < 1 || v > X16_MAX_V) return FP_ERR_SHAPE;
    if (k < 1 || k > 20) return FP_ERR_ARG;
    const size_t need_len = lu2_proof_len(v, k);
    if (!proof || *proof_len < need_len) {
        *proof_len = need_len;
        return FP_ERR_ARG;
    }
    Lu2Callback cb;
    cb.fn = fn;
    cb.user = user;
    return lu2_protocol(nullptr, tx, v, k, m_rem, d_rem, m_clamp, d_clamp, cb, proof, proof_len);
}
