// SiLU by lookup: one LogUp-GKR fraction tree over the keys f = g + gamma s.
//
// "How fast can FlashProve go", 2 Background and 3.1: the SiLU is not a
// polynomial, so its 16-bit outputs are committed and proven by a lookup. The
// table reads a 16-bit input v with 8 fractional bits and stores
// silu_q(v) = floor(v / (1 + e^(-v/256)) + 1/2) (evaluated in double precision on
// the host, where the verifier evaluates it too). The statement:
//   absorb "silu_site" D(g) || D(s) (int16 little-endian); squeeze gamma;
//   keys padded to 2^v (v >= 1) with (0, 0); m_j = #{keys with g = j - 2^15};
//   send m (2^16 u32, its digest absorbed as "silu_m"); squeeze alpha;
//   the fraction tree of leaves (1, alpha - f): send layer one ("silu_l1"),
//   squeeze mu; layers d = 1..v-1: squeeze lambda, sum-check of
//   eq(z, x)(pL qR + pR qL + lambda qL qR) over d variables ("silu_round" /
//   "silu_chal"), send the four child values at rho ("silu_final"), squeeze
//   mu, z = (rho, mu); send g~(z), s~(z) ("silu_leaf").
// A layer's round values come as in the product sum-checks: the device returns
// h(0), h(1), h(2) of h(X) = sum_b eq(z_>t, b) F(X, b) (F has degree 2) and the
// host multiplies in eq(z_<t, rho_<t) eq(z_t, X), checking g(0) + g(1) against
// the running claim.
#include <math.h>
#include <string.h>

#include <algorithm>
#include <vector>

#include "fp_eqchunks.cuh"
#include "fp_hist.cuh"
#include "fp_internal.h"
#include "fp_reduce.cuh"
#include "fp_session.cuh"

namespace {

constexpr int SL_THREADS = 256;
constexpr int SL_MAX_V = 30;

__device__ __forceinline__ uint64_t lift_i(int64_t x) { return x < 0 ? GL_P - (uint64_t)(-x) : (uint64_t)x; }

// leaves: P = 1, Q = alpha - (g + gamma s); past n the padding key fpad (the table's row for input 0)
__global__ void silu_leaf_kernel(const int16_t* __restrict__ g, const int16_t* __restrict__ s, int64_t n, int64_t L,
                                 uint64_t alpha, uint64_t gamma, uint64_t fpad, uint64_t* __restrict__ P,
                                 uint64_t* __restrict__ Q) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < L; i += (int64_t)gridDim.x * blockDim.x) {
        uint64_t f = fpad;
        if (i < n) f = gl_add(lift_i(g[i]), gl_mul(gamma, lift_i(s[i])));
        P[i] = 1;
        Q[i] = gl_sub(alpha, f);
    }
}

// one level up: P'[x] = P[2x] Q[2x+1] + P[2x+1] Q[2x], Q'[x] = Q[2x] Q[2x+1], x < c
__global__ void silu_level_kernel(const uint64_t* __restrict__ P, const uint64_t* __restrict__ Q, int64_t c,
                                  uint64_t* __restrict__ Po, uint64_t* __restrict__ Qo) {
    for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < c; x += (int64_t)gridDim.x * blockDim.x) {
        const uint64_t pl = P[2 * x], pr = P[2 * x + 1], ql = Q[2 * x], qr = Q[2 * x + 1];
        Po[x] = gl_add(gl_mul(pl, qr), gl_mul(pr, ql));
        Qo[x] = gl_mul(ql, qr);
    }
}

// out[0] = sum_{x < n} eq(z, x) a(x) for an int16 column a of n entries, out[1] = sum_{x < n} eq(z, x)
// (so that a padding value past n adds pad (1 - out[1])); eq split as EH[x >> vl] EL[x & (2^vl - 1)]
__global__ void __launch_bounds__(256) silu_mle_kernel(const int16_t* __restrict__ a, int64_t n,
                                                       const uint64_t* __restrict__ EH, const uint64_t* __restrict__ EL,
                                                       int vl, uint64_t* part, unsigned int* ticket, uint64_t* out) {
    GlAcc acc, eacc;
    const int64_t mask = (1ll << vl) - 1;
    for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < n; x += (int64_t)gridDim.x * blockDim.x) {
        const uint64_t e = gl_mul(__ldg(EH + (x >> vl)), __ldg(EL + (x & mask)));
        eacc.add(e);
        const int v = a[x];
        if (v != 0) acc.mac(e, lift_i(v));
    }
    uint64_t v[2] = {acc.value(), eacc.value()};
    if (grid_sum_gl<2>(v, part, ticket) && threadIdx.x == 0) {
        out[0] = v[0];
        out[1] = v[1];
    }
}

struct LayerArgs {
    const ulonglong2* P;  // tree layer d + 1 as child pairs: (pL, pR) of node b at entry b
    const ulonglong2* Q;  // (qL, qR)
    ulonglong2* pp;       // the child pairs folded, from round 2 on (2^(d-1) pairs each)
    ulonglong2* qq;
    uint64_t* E;          // suffix eq table (2^(d-1) entries)
    const uint64_t* z;  // device copy of the layer's point z_1..z_d
    uint64_t lam;
    int d;
    int grid;
    int per_block;
    int pad;
    uint64_t seq0;  // round t publishes seq0 + t, the final values seq0 + d + 1
    int t_begin;    // rounds run by this launch: [t_begin, t_end]; t_end > d includes the final values
    int t_end;
};

__device__ __forceinline__ uint64_t at2(uint64_t a, uint64_t b) { return gl_sub(gl_add(b, b), a); }

// pL qR + pR qL + lambda qL qR = pL qR + qL (pR + lambda qR), weakly reduced (< 2^64, congruent)
__device__ __forceinline__ uint64_t layer_f(ulonglong2 p, ulonglong2 q, uint64_t lam) {
    const uint64_t u = gl_add(p.y, gl_mul_weak(lam, q.y));
    return gl_muladd_weak(q.x, u, gl_mul_weak(p.x, q.y));
}

__device__ __forceinline__ ulonglong2 fold2(ulonglong2 a, ulonglong2 b, uint64_t r) {
    return make_ulonglong2(gl_fold_fast(a.x, b.x, r), gl_fold_fast(a.y, b.y, r));
}

__device__ __forceinline__ ulonglong2 at2v(ulonglong2 a, ulonglong2 b) { return make_ulonglong2(at2(a.x, b.x), at2(a.y, b.y)); }

// four blocks per SM (64 registers, no spill): the rounds wait on memory latency, and more
// warps hide it (2^26 entries: gated product 1.29 -> 1.02 ms, SiLU layers 1.66 -> 1.58 ms)
#ifndef FP_SILU_MIN_BLOCKS
#define FP_SILU_MIN_BLOCKS 4
#endif
__global__ void __launch_bounds__(SL_THREADS, FP_SILU_MIN_BLOCKS) silu_layer_kernel(LayerArgs A, FpMailbox* mb, FpRelay* rl,
                                                                  uint64_t* part) {
    __shared__ uint64_t zs[32];
    __shared__ uint64_t eq_tab[3 << kEqChunk];
    if (threadIdx.x < A.d) zs[threadIdx.x] = A.z[threadIdx.x];
    __syncthreads();
    uint64_t rprev = 0;
    for (int t = A.t_begin; t <= A.d && t <= A.t_end; t++) {
        if (t > 1 && !session_wait(mb, rl, A.seq0 + t - 1, rprev)) return;
        const int64_t h = 1ll << (A.d - t);
        const int64_t want = (h + A.per_block - 1) / A.per_block;
        const unsigned active = (unsigned)(want < 1 ? 1 : (want > A.grid ? A.grid : want));
        if (blockIdx.x >= active) return;  // no pairs for this block in this or any later round
        EqChunks EC{0, 0, 0};
        if (t == 1) EC = eq_chunks_build(eq_tab, zs, A.d);
        // h(1) only where the host cannot take it from the running claim (z_t = 0)
        const bool need1 = zs[t - 1] == 0;
        GlAcc a0, a1, a2;
        for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < h; b += (int64_t)active * blockDim.x) {
            ulonglong2 p0, p1, q0, q1;  // (pL, pR), (qL, qR) at the pair's two points
            uint64_t e;
            if (t == 1) {
                p0 = __ldcg(A.P + b);
                q0 = __ldcg(A.Q + b);
                p1 = __ldcg(A.P + b + h);
                q1 = __ldcg(A.Q + b + h);
                e = eq_chunks_at(EC, eq_tab, b);  // eq(z_2..z_d, b)
                if (A.d > 1) A.E[b] = e;
            } else {
                // the children (the tree layer in round 2, the folded pairs after) folded by rho_(t-1)
                const ulonglong2* sp = t == 2 ? A.P : A.pp;
                const ulonglong2* sq = t == 2 ? A.Q : A.qq;
                p0 = fold2(__ldcg(sp + b), __ldcg(sp + b + 2 * h), rprev);
                q0 = fold2(__ldcg(sq + b), __ldcg(sq + b + 2 * h), rprev);
                p1 = fold2(__ldcg(sp + b + h), __ldcg(sp + b + 3 * h), rprev);
                q1 = fold2(__ldcg(sq + b + h), __ldcg(sq + b + 3 * h), rprev);
                A.pp[b] = p0;
                A.qq[b] = q0;
                A.pp[b + h] = p1;
                A.qq[b + h] = q1;
                e = gl_add(__ldcg(A.E + b), __ldcg(A.E + b + h));  // eq(z_>t, b)
                A.E[b] = e;
            }
            a0.mac(e, layer_f(p0, q0, A.lam));
            if (need1) a1.mac(e, layer_f(p1, q1, A.lam));
            a2.mac(e, layer_f(at2v(p0, p1), at2v(q0, q1), A.lam));
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
    // block 0 folds the last pair of each vector by the last challenge: pL, pR, qL, qR at rho
    if (A.t_end <= A.d || blockIdx.x != 0) return;
    if (!session_wait(mb, rl, A.seq0 + A.d, rprev)) return;
    if (threadIdx.x == 0) {
        const ulonglong2* sp = A.d == 1 ? A.P : A.pp;
        const ulonglong2* sq = A.d == 1 ? A.Q : A.qq;
        const ulonglong2 pf = fold2(__ldcg(sp), __ldcg(sp + 1), rprev), qf = fold2(__ldcg(sq), __ldcg(sq + 1), rprev);
        const uint64_t fin[4] = {pf.x, pf.y, qf.x, qf.y};
        session_publish(mb, fin, A.seq0 + A.d + 1);
    }
}

// 1 / z_i for every nonzero coordinate (one inversion for all), 0 where z_i = 0
std::vector<uint64_t> inverses_or_zero(const uint64_t* z, int n) {
    std::vector<uint64_t> inv(n, 0);
    uint64_t run = 1;
    for (int i = 0; i < n; i++) {
        inv[i] = run;
        if (z[i]) run = gl_mul(run, z[i]);
    }
    uint64_t r = gl_inv(run);
    for (int i = n - 1; i >= 0; i--) {
        if (!z[i]) {
            inv[i] = 0;
            continue;
        }
        inv[i] = gl_mul(inv[i], r);
        r = gl_mul(r, z[i]);
    }
    return inv;
}

int64_t silu_q_host(int64_t v) { return (int64_t)floor((double)v / (1.0 + exp(-(double)v / 256.0)) + 0.5); }

// the softmax numerator: floor(511 e^(v/256) + 1/2) for v = score - row maximum <= 0, 511 above
int64_t exp_q_host(int64_t v) { return v >= 0 ? 511 : (int64_t)floor(511.0 * exp((double)v / 256.0) + 0.5); }

struct LookupLabels {
    const char *site, *gamma, *m, *alpha, *l1, *mu, *lambda, *round, *chal, *fin, *leaf;
};
const LookupLabels kSiluLabels = {"silu_site", "silu_gamma", "silu_m", "silu_alpha", "silu_l1", "silu_mu",
                                  "silu_lambda", "silu_round", "silu_chal", "silu_final", "silu_leaf"};
const LookupLabels kExpLabels = {"exp_site", "exp_gamma", "exp_m", "exp_alpha", "exp_l1", "exp_mu",
                                 "exp_lambda", "exp_round", "exp_chal", "exp_final", "exp_leaf"};

unsigned grid_of(const fp_ctx* c, int64_t work) {
    return (unsigned)std::max<int64_t>(1, std::min<int64_t>((work + 255) / 256, 4 * (int64_t)c->num_sms));
}

// m (2^16 u32), layer one (4), per layer d = 1..v-1 its d rounds (4 each) and 4 final values, 2 leaf values
size_t silu_proof_len(int64_t n) {
    int v = fp_log2_ceil((uint64_t)n);
    if (v < 1) v = 1;
    size_t len = 4 * 65536 + 32 + 16;
    for (int d = 1; d < v; d++) len += 32 * (size_t)d + 32;
    return len;
}

// One 16-bit function lookup: the argument is the same for every table; the table enters
// only through its row for input 0 (pad_s = table(0)), which pads the keys, and the labels.
int lookup16_prove(fp_ctx* c, fp_tx* tx, const LookupLabels& lab, int64_t pad_s, const int16_t* g, const int16_t* s,
                   int64_t n, uint8_t* proof, size_t* proof_len, void* stream) {
    if (!c || !tx || !proof_len) return fp_fail(c, FP_ERR_ARG, "logup_prove_silu: null argument");
    if (!g || !s) return fp_fail(c, FP_ERR_ARG, "logup_prove_silu: null column");
    if (n < 1 || n > (1ll << SL_MAX_V)) return fp_fail(c, FP_ERR_SHAPE, "logup_prove_silu: need 1 <= n <= 2^30");
    const size_t need_len = silu_proof_len(n);
    if (!proof || *proof_len < need_len) {
        *proof_len = need_len;
        return fp_fail(c, FP_ERR_ARG, "logup_prove_silu: proof buffer too small");
    }
    FP_CUDA(c, cudaSetDevice(c->device));
    cudaStream_t st = (cudaStream_t)stream;
    int rc;
    int v = fp_log2_ceil((uint64_t)n);
    if (v < 1) v = 1;
    const int64_t L = 1ll << v;

    // ---- commit ----
    {
        FpDigestJob jobs[2] = {{(const uint8_t*)g, 2 * (uint64_t)n}, {(const uint8_t*)s, 2 * (uint64_t)n}};
        uint8_t d[64];
        if ((rc = fp_digest_many(c, jobs, 2, d, st))) return rc;  // synchronises the stream
        fp_tx_absorb_raw(tx, lab.site, d, 64);
    }
    const uint64_t gamma = fp_tx_squeeze_one(tx, lab.gamma);

    // ---- scratch: multiplicities, tree layers 1..v, layer vectors, eq tables, reductions ----
    int occ = 0;
    FP_CUDA(c, cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, silu_layer_kernel, SL_THREADS, 0));
    const int cap_grid = std::max(1, occ) * c->num_sms;
    const size_t part_n = (size_t)3 * std::max(cap_grid, 4 * c->num_sms);
    const int64_t hv = v >= 2 ? 1ll << (v - 2) : 1;  // the largest layer's vectors: 2^(d-1) for d = v - 1
    const int vl = v / 2, vh = v - vl;
    size_t need = fp_align_up(4 * 65536, 256) + fp_align_up(8 * part_n, 256) + fp_align_up(8 * 64, 256) +
                  fp_align_up((size_t)8 << vh, 256) + fp_align_up((size_t)8 << vl, 256) +
                  2 * fp_align_up((size_t)16 * hv, 256) + fp_align_up((size_t)8 * hv, 256) + 4096;
    for (int d = 1; d <= v; d++) need += 2 * fp_align_up((size_t)8 << d, 256);
    need += fp_hist::hist16_scratch();
    if ((rc = fp_reserve(c, c->dev, need))) return rc;
    if ((rc = fp_reserve(c, c->host, 4 * 65536 + 8192))) return rc;
    fp_reset(c->dev);
    fp_reset(c->host);
    uint32_t* m = (uint32_t*)fp_alloc(c->dev, 4 * 65536);
    uint32_t* hpart = (uint32_t*)fp_alloc(c->dev, fp_hist::hist16_scratch());
    uint64_t* part = (uint64_t*)fp_alloc(c->dev, 8 * part_n);
    uint64_t* small = (uint64_t*)fp_alloc(c->dev, 8 * 64);  // [0..1] leaf values, [8..] the layer's point
    uint64_t* EH = (uint64_t*)fp_alloc(c->dev, (size_t)8 << vh);
    uint64_t* EL = (uint64_t*)fp_alloc(c->dev, (size_t)8 << vl);
    // the layer's folded child pairs (p and q: 16 bytes per pair each) and its suffix eq table
    ulonglong2* fpp = (ulonglong2*)fp_alloc(c->dev, (size_t)16 * hv);
    ulonglong2* fqq = (ulonglong2*)fp_alloc(c->dev, (size_t)16 * hv);
    uint64_t* fE = (uint64_t*)fp_alloc(c->dev, (size_t)8 * hv);
    std::vector<uint64_t*> TP(v + 1, nullptr), TQ(v + 1, nullptr);
    for (int d = 1; d <= v; d++) {
        TP[d] = (uint64_t*)fp_alloc(c->dev, (size_t)8 << d);
        TQ[d] = (uint64_t*)fp_alloc(c->dev, (size_t)8 << d);
        if (!TP[d] || !TQ[d]) return fp_fail(c, FP_ERR_OOM, "logup_prove_silu: scratch exhausted");
    }
    uint8_t* hm = (uint8_t*)fp_alloc(c->host, 4 * 65536);
    uint64_t* hs = (uint64_t*)fp_alloc(c->host, 8 * 64);
    if (!m || !hpart || !part || !small || !EH || !EL || !fpp || !fqq || !fE || !hm || !hs)
        return fp_fail(c, FP_ERR_OOM, "logup_prove_silu: scratch exhausted");

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
    size_t pos = 0;
    memcpy(proof + pos, hm, 4 * 65536);  // device words are little-endian u32
    pos += 4 * 65536;
    fp_tx_absorb_raw(tx, lab.m, dm, 32);
    const uint64_t alpha = fp_tx_squeeze_one(tx, lab.alpha);

    // ---- the fraction tree, layers v (leaves) .. 1 ----
    {
        int slot;
        fp_tic(c, st, K_SILU_TREE, 4.0 * (double)n + 32.0 * (double)L, &slot);
        const uint64_t fpad = gl_mul(gamma, pad_s < 0 ? GL_P - (uint64_t)(-pad_s) : (uint64_t)pad_s);
        silu_leaf_kernel<<<grid_of(c, L), 256, 0, st>>>(g, s, n, L, alpha, gamma, fpad, TP[v], TQ[v]);
        FP_CUDA(c, cudaGetLastError());
        for (int d = v - 1; d >= 1; d--) {
            silu_level_kernel<<<grid_of(c, 1ll << d), 256, 0, st>>>(TP[d + 1], TQ[d + 1], 1ll << d, TP[d], TQ[d]);
            FP_CUDA(c, cudaGetLastError());
        }
        fp_toc(c, st, slot);
    }
    FP_CUDA(c, cudaMemcpyAsync(hs, TP[1], 16, cudaMemcpyDeviceToHost, st));
    FP_CUDA(c, cudaMemcpyAsync(hs + 2, TQ[1], 16, cudaMemcpyDeviceToHost, st));
    FP_CUDA(c, cudaStreamSynchronize(st));
    uint64_t l1[4] = {hs[0], hs[1], hs[2], hs[3]};
    put_u64s(proof + pos, l1, 4);
    fp_tx_absorb_raw(tx, lab.l1, proof + pos, 32);
    pos += 32;
    FpPoint z;
    z.v = 1;
    z.z[0] = fp_tx_squeeze_one(tx, lab.mu);
    uint64_t cP = gl_fold(l1[0], l1[1], z.z[0]), cQ = gl_fold(l1[2], l1[3], z.z[0]);

    // ---- layer sum-checks d = 1 .. v - 1 ----
    for (int d = 1; d < v; d++) {
        const uint64_t lam = fp_tx_squeeze_one(tx, lab.lambda);
        uint64_t claim = gl_add(cP, gl_mul(lam, cQ));
        for (int i = 0; i < d; i++) hs[8 + i] = z.z[i];
        FP_CUDA(c, cudaMemcpyAsync(small + 8, hs + 8, 8 * (size_t)d, cudaMemcpyHostToDevice, st));
        LayerArgs A;
        memset(&A, 0, sizeof A);
        A.P = reinterpret_cast<const ulonglong2*>(TP[d + 1]);
        A.Q = reinterpret_cast<const ulonglong2*>(TQ[d + 1]);
        A.pp = fpp;
        A.qq = fqq;
        A.E = fE;
        A.z = small + 8;
        A.lam = lam;
        A.d = d;
        A.per_block = SL_THREADS;  // one pair per thread
        const int64_t half = 1ll << (d - 1);
        A.grid = (int)std::max<int64_t>(1, std::min<int64_t>((half + A.per_block - 1) / A.per_block, cap_grid));
        A.seq0 = fp_seq_reserve(c, (uint64_t)d + 2);
        if ((rc = fp_session_begin(c, st))) return rc;
        fp_session_expect(c, 3);  // before any launch: round 1 publishes without a challenge
        void* args[] = {&A, &c->mb_dev, &c->relay, &part};
        auto round_bytes = [&](int t) { return 80.0 * (double)(1ll << (d - t)) * (t == 1 ? 1.0 : 2.0); };
        if (!c->stepped) {
            A.t_begin = 1;
            A.t_end = d + 1;
            double bytes = 0;
            for (int t = 1; t <= d; t++) bytes += round_bytes(t);
            int slot;
            fp_tic(c, st, K_SILU_ROUND, bytes, &slot);
            FP_CUDA(c, cudaLaunchCooperativeKernel((const void*)silu_layer_kernel, dim3(A.grid), dim3(SL_THREADS),
                                                   args, 0, st));
            fp_toc(c, st, slot);
        }
        uint64_t pre = 1;  // eq(z_<t, rho_<t)
        std::vector<uint64_t> rho(d);
        const std::vector<uint64_t> zinv = inverses_or_zero(z.z, d);
        for (int t = 1; t <= d; t++) {
            if (c->stepped) {
                A.t_begin = A.t_end = t;
                int slot;
                fp_tic(c, st, K_SILU_ROUND, round_bytes(t), &slot);
                FP_CUDA(c, cudaLaunchCooperativeKernel((const void*)silu_layer_kernel, dim3(A.grid),
                                                       dim3(SL_THREADS), args, 0, st));
                fp_toc(c, st, slot);
            }
            if ((rc = fp_session_wait(c, A.seq0 + t, st))) return rc;
            // g(X) = pre eq(z_t, X) h(X); g(1) = claim - g(0), and h(1) = g(1) / (pre z_t) gives
            // h(3) = h(0) - 3 h(1) + 3 h(2) (the device sends h(1) only when z_t = 0)
            const uint64_t zt = z.z[t - 1];
            const uint64_t ph0 = gl_mul(pre, c->mb->res[0]), ph2 = gl_mul(pre, c->mb->res[2]);
            uint64_t gr[4];
            gr[0] = gl_mul(gl_sub(1, zt), ph0);
            gr[1] = gl_sub(claim, gr[0]);
            const uint64_t ph1 = zt ? gl_mul(gr[1], zinv[t - 1]) : gl_mul(pre, c->mb->res[1]);
            gr[2] = gl_mul(gl_sub(gl_mul(3, zt), 1), ph2);
            gr[3] = gl_mul(gl_sub(gl_mul(5, zt), 2), gl_add(gl_sub(ph0, gl_mul(3, ph1)), gl_mul(3, ph2)));
            put_u64s(proof + pos, gr, 4);
            fp_tx_absorb_raw(tx, lab.round, proof + pos, 32);
            pos += 32;
            fp_session_expect(c, t < d ? 3 : 4);  // the last challenge triggers the four final values
            const uint64_t r = fp_tx_squeeze_one(tx, lab.chal);
            fp_session_post(c, A.seq0 + t, r);
            rho[t - 1] = r;
            claim = fp_lagrange4(gr, r);
            pre = gl_mul(pre, gl_add(gl_mul(zt, r), gl_mul(gl_sub(1, zt), gl_sub(1, r))));
        }
        if (c->stepped) {
            A.t_begin = A.t_end = d + 1;
            int slot;
            fp_tic(c, st, K_SILU_ROUND, 64.0, &slot);
            FP_CUDA(c, cudaLaunchCooperativeKernel((const void*)silu_layer_kernel, dim3(1), dim3(SL_THREADS), args, 0,
                                                   st));
            fp_toc(c, st, slot);
        }
        if ((rc = fp_session_wait(c, A.seq0 + d + 1, st))) return rc;
        uint64_t fin[4] = {c->mb->res[0], c->mb->res[1], c->mb->res[2], c->mb->res[3]};
        FP_CUDA(c, cudaStreamSynchronize(st));
        put_u64s(proof + pos, fin, 4);
        fp_tx_absorb_raw(tx, lab.fin, proof + pos, 32);
        pos += 32;
        const uint64_t mu = fp_tx_squeeze_one(tx, lab.mu);
        cP = gl_fold(fin[0], fin[1], mu);
        cQ = gl_fold(fin[2], fin[3], mu);
        for (int i = 0; i < d; i++) z.z[i] = rho[i];
        z.z[d] = mu;
        z.v = d + 1;
    }

    // ---- leaf claims: g~(z), s~(z) over the padded columns ----
    {
        FpPoint zh, zl;
        zh.v = vh;
        zl.v = vl;
        for (int i = 0; i < vh; i++) zh.z[i] = z.z[i];
        for (int i = 0; i < vl; i++) zl.z[i] = z.z[vh + i];
        if ((rc = fp_eq_table(c, zh, EH, st))) return rc;
        if ((rc = fp_eq_table(c, zl, EL, st))) return rc;
        const unsigned blocks = (unsigned)std::max<int64_t>(1, std::min<int64_t>((n + 255) / 256, 2 * (int64_t)c->num_sms));
        int slot;
        fp_tic(c, st, K_SILU_LEAF, 4.0 * (double)n, &slot);
        silu_mle_kernel<<<blocks, 256, 0, st>>>(g, n, EH, EL, vl, part, c->tickets, small);
        FP_CUDA(c, cudaGetLastError());
        silu_mle_kernel<<<blocks, 256, 0, st>>>(s, n, EH, EL, vl, part, c->tickets, small + 2);
        fp_toc(c, st, slot);
        FP_CUDA(c, cudaGetLastError());
        FP_CUDA(c, cudaMemcpyAsync(hs, small, 32, cudaMemcpyDeviceToHost, st));
        FP_CUDA(c, cudaStreamSynchronize(st));
    }
    // the s column past n holds the padding value: it adds pad_s (1 - sum_{x < n} eq(z, x))
    const uint64_t padf = pad_s < 0 ? GL_P - (uint64_t)(-pad_s) : (uint64_t)pad_s;
    const uint64_t leaf[2] = {hs[0], gl_add(hs[2], gl_mul(padf, gl_sub(1, hs[3])))};
    put_u64s(proof + pos, leaf, 2);
    fp_tx_absorb_raw(tx, lab.leaf, proof + pos, 16);
    pos += 16;
    *proof_len = pos;
    return FP_OK;
}

}  // namespace

int logup_prove_silu(fp_ctx* c, fp_tx* tx, const int16_t* g, const int16_t* s, int64_t n, uint8_t* proof,
                     size_t* proof_len, void* stream) {
    return lookup16_prove(c, tx, kSiluLabels, silu_q_host(0), g, s, n, proof, proof_len, stream);
}

int logup_prove_exp(fp_ctx* c, fp_tx* tx, const int16_t* g, const int16_t* s, int64_t n, uint8_t* proof,
                    size_t* proof_len, void* stream) {
    return lookup16_prove(c, tx, kExpLabels, exp_q_host(0), g, s, n, proof, proof_len, stream);
}

namespace {

// The SiLU's inputs and outputs for 8-bit inputs (the gate projection's outputs): g = y widened,
// s = silu_q(y) as 16-bit and as 8-bit values (silu_q maps [-128, 127] into [-48, 79])
struct SiluTab8 {
    int16_t v[256];
};

__global__ void silu_inputs_kernel(const int8_t* __restrict__ y, int64_t n, SiluTab8 tab, int16_t* __restrict__ g,
                                   int16_t* __restrict__ s, int8_t* __restrict__ s8) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const int v = y[i];
        const int16_t o = tab.v[v + 128];
        g[i] = (int16_t)v;
        s[i] = o;
        s8[i] = (int8_t)o;
    }
}

// The FFN's hidden activations h = s u rescaled by 2^kh (round half up, as every site's
// witness): q = floor((h + 2^(kh-1)) / 2^kh) (an arithmetic shift), r = h - 2^kh q,
// y = clamp(q, -128, 127). Sixteen entries per thread step from 16-byte loads when every
// buffer is 16-byte aligned; the rest entry by entry.
__device__ __forceinline__ void hidden_one(int sv, int uv, int kh, int32_t& q, int32_t& r, int8_t& y) {
    const int h = sv * uv;
    const int qq = (h + (1 << (kh - 1))) >> kh;
    q = qq;
    r = h - qq * (1 << kh);
    y = (int8_t)(qq < -128 ? -128 : (qq > 127 ? 127 : qq));
}

__global__ void ffn_hidden_kernel(const int8_t* __restrict__ s, const int8_t* __restrict__ u, int64_t n, int kh,
                                  int32_t* __restrict__ q, int32_t* __restrict__ r, int8_t* __restrict__ y,
                                  bool vec) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    int64_t done = 0;
    if (vec) {
        const int64_t n16 = n / 16;
        for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < n16; j += stride) {
            const int4 sv = reinterpret_cast<const int4*>(s)[j];
            const int4 uv = reinterpret_cast<const int4*>(u)[j];
            const int8_t* sb = reinterpret_cast<const int8_t*>(&sv);
            const int8_t* ub = reinterpret_cast<const int8_t*>(&uv);
            int4 qv[4], rv[4], yv;
            int32_t* qo = reinterpret_cast<int32_t*>(qv);
            int32_t* ro = reinterpret_cast<int32_t*>(rv);
            int8_t* yo = reinterpret_cast<int8_t*>(&yv);
#pragma unroll
            for (int e = 0; e < 16; e++) hidden_one(sb[e], ub[e], kh, qo[e], ro[e], yo[e]);
#pragma unroll
            for (int w = 0; w < 4; w++) {
                reinterpret_cast<int4*>(q)[4 * j + w] = qv[w];
                reinterpret_cast<int4*>(r)[4 * j + w] = rv[w];
            }
            reinterpret_cast<int4*>(y)[j] = yv;
        }
        done = n16 * 16;
    }
    for (int64_t i = done + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
        hidden_one(s[i], u[i], kh, q[i], r[i], y[i]);
}

}  // namespace

int fp_ffn_hidden(fp_ctx* c, const int8_t* s, const int8_t* u, int64_t n, int kh, int32_t* q, int32_t* r, int8_t* y,
                  void* stream) {
    if (!c || !s || !u || !q || !r || !y || n < 1) return fp_fail(c, FP_ERR_ARG, "fp_ffn_hidden: bad argument");
    if (kh < 1 || kh > 16) return fp_fail(c, FP_ERR_ARG, "fp_ffn_hidden: kh outside [1, 16]");
    FP_CUDA(c, cudaSetDevice(c->device));
    cudaStream_t st = (cudaStream_t)stream;
    const bool vec = ((uintptr_t)s | (uintptr_t)u | (uintptr_t)q | (uintptr_t)r | (uintptr_t)y) % 16 == 0;
    const int64_t items = vec ? std::max<int64_t>(n / 16, 1) : n;
    const unsigned grid = (unsigned)std::min<int64_t>((items + 255) / 256, 8ll * c->num_sms);
    int slot;
    fp_tic(c, st, K_FFN_HIDDEN, 11.0 * (double)n, &slot);  // two int8 factors in, q and r int32 and y out
    ffn_hidden_kernel<<<grid, 256, 0, st>>>(s, u, n, kh, q, r, y, vec);
    fp_toc(c, st, slot);
    FP_CUDA(c, cudaGetLastError());
    return FP_OK;
}

int fp_silu_inputs(fp_ctx* c, const int8_t* y, int64_t n, int16_t* g, int16_t* s, int8_t* s8, void* stream) {
    if (!c || !y || !g || !s || !s8 || n < 1) return fp_fail(c, FP_ERR_ARG, "fp_silu_inputs: bad argument");
    FP_CUDA(c, cudaSetDevice(c->device));
    SiluTab8 tab;
    for (int v = -128; v < 128; v++) tab.v[v + 128] = (int16_t)silu_q_host(v);
    cudaStream_t st = (cudaStream_t)stream;
    const unsigned grid = (unsigned)std::min<int64_t>((n + 255) / 256, 8ll * c->num_sms);
    int slot;
    fp_tic(c, st, K_SILU_INPUTS, 6.0 * (double)n, &slot);  // y in; g, s (int16) and s8 out
    silu_inputs_kernel<<<grid, 256, 0, st>>>(y, n, tab, g, s, s8);
    fp_toc(c, st, slot);
    FP_CUDA(c, cudaGetLastError());
    return FP_OK;
}

int fp_silu_table(int32_t* out) {
    if (!out) return FP_ERR_ARG;
    for (int64_t v = -32768; v < 32768; v++) out[v + 32768] = (int32_t)silu_q_host(v);
    return FP_OK;
}

int fp_exp_table(int32_t* out) {
    if (!out) return FP_ERR_ARG;
    for (int64_t v = -32768; v < 32768; v++) out[v + 32768] = (int32_t)exp_q_host(v);
    return FP_OK;
}
