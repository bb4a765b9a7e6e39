// MoE routing: the top-1 choice of expert, proven.
//
// "How fast can FlashProve go", 2 Background (the note on MoE layers: the
// routing computation and each token's choice of expert are proven too). Token
// t goes to e_t, the first index of its largest router logit (int8, token-major
// T x E, E a power of two). The prover commits the one-hot H[t][e] = [e = e_t]
// (u8) and D[t][e] = l[t][e_t] - l[t][e] - [e < e_t] (int32), which lies in
// [0, 256) for every e exactly when e_t is the first maximum. With x = t E + e
// (token bits first) and rows zero-padded to 2^vT:
//   absorb "route_site" D(l) || D(H) || D(D); squeeze z, w (vT + vE each,
//   "route_z", "route_w"), lambda1, lambda2 ("route_lambda"); send D~(z), l~(z)
//   ("route_open"); sum-check of
//     F(x) = eq(z_t, t) H (l - G(e)) + lambda1 eq(w, x) H (1 - H) + lambda2 eq(w_t, t) H,
//   G(e) = sum_{e' < e} eq(z_e, e'), claim D~(z) + l~(z) + lambda2 sum_{t < T} eq(w_t, t)
//   (rounds g(0..3), "route_round", "route_chal"); send H~(rho), l~(rho)
//   ("route_final"); then the helper-inverse LogUp of the keys D - 128 on R_8.
//
// Kernels: one warp per token finds the first maximum and writes H, D and the
// keys; the six factors of F are laid out as vectors over x (eq tables from
// mle.cu, G as prefix sums of eq(z_e, .)); one pass gives the two openings and
// the row-sum weight; every round runs in one resident cooperative launch that
// folds the six vectors in place and sums F at X = 0..3 exactly. T E is at most
// 2^26 here (the MoE layer's 8192 x 128 is 2^20), so the vectors stay small.
//
// The host half (route_protocol) takes its device values from a source: the
// kernels here, or a caller's callback (fp_route_protocol_drive).
#include <string.h>

#include <algorithm>

#include "fp_internal.h"
#include "fp_reduce.cuh"
#include "fp_session.cuh"

namespace {

constexpr int RT_THREADS = 256;
constexpr int RT_MAX_N = 26;      // vT + vE
constexpr int RT_MAX_E = 4096;

// one warp per token row: the first maximum, then H, D and the keys D - 128 of the row
__global__ void route_witness_kernel(const int8_t* __restrict__ l, int64_t T, int E, uint8_t* __restrict__ H,
                                     int32_t* __restrict__ D, int32_t* __restrict__ keys) {
    const int lane = threadIdx.x & 31;
    const int64_t warp = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t t = warp; t < T; t += nwarps) {  // warp-uniform
        const int8_t* row = l + t * E;
        int bv = -1000, be = 0x7fffffff;
        for (int e = lane; e < E; e += 32) {  // increasing e: a strict > keeps the first maximum
            const int x = row[e];
            if (x > bv) {
                bv = x;
                be = e;
            }
        }
#pragma unroll
        for (int m = 16; m > 0; m >>= 1) {
            const int ov = __shfl_xor_sync(0xffffffffu, bv, m), oe = __shfl_xor_sync(0xffffffffu, be, m);
            if (ov > bv || (ov == bv && oe < be)) {
                bv = ov;
                be = oe;
            }
        }
        for (int e = lane; e < E; e += 32) {
            const int d = bv - (int)row[e] - (e < be ? 1 : 0);
            H[t * E + e] = (uint8_t)(e == be);
            D[t * E + e] = d;
            keys[t * E + e] = d - 128;
        }
    }
}

// G[e] = sum_{e' < e} eq(z_e, e') from the eq table of z_e (E entries; one thread)
__global__ void route_prefix_kernel(const uint64_t* __restrict__ eqe, int E, uint64_t* __restrict__ G) {
    if (blockIdx.x != 0 || threadIdx.x != 0) return;
    uint64_t acc = 0;
    for (int e = 0; e < E; e++) {
        G[e] = acc;
        acc = gl_add(acc, eqe[e]);
    }
}

// the factor vectors over x < 2^n: eq(z_t, t), H, l, G(e), eq(w_t, t) (eq(w, x) is built in place by
// the eq-table builder)
__global__ void route_vectors_kernel(const int8_t* __restrict__ l, const uint8_t* __restrict__ H, int64_t TE, int vE,
                                     int64_t L, const uint64_t* __restrict__ et, const uint64_t* __restrict__ ewt,
                                     const uint64_t* __restrict__ G, uint64_t* __restrict__ Et,
                                     uint64_t* __restrict__ Hv, uint64_t* __restrict__ lv, uint64_t* __restrict__ Gv,
                                     uint64_t* __restrict__ Ewt) {
    const int64_t emask = (1ll << vE) - 1;
    for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < L; x += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = x >> vE;
        Et[x] = et[t];
        Ewt[x] = ewt[t];
        Gv[x] = G[x & emask];
        Hv[x] = x < TE ? (uint64_t)H[x] : 0;
        lv[x] = x < TE ? gl_from_i64(l[x]) : 0;
    }
}

// out[0] = D~(z), out[1] = l~(z) (eq(z, x) = EH[x >> vl] EL[x & (2^vl - 1)]), out[2] = sum_{t < T} ewt[t]
__global__ void __launch_bounds__(RT_THREADS) route_open_kernel(const int32_t* __restrict__ D,
                                                                const int8_t* __restrict__ l, int64_t TE,
                                                                const uint64_t* __restrict__ EH,
                                                                const uint64_t* __restrict__ EL, int vl,
                                                                const uint64_t* __restrict__ ewt, int64_t T,
                                                                uint64_t* part, unsigned int* ticket, uint64_t* out) {
    GlAcc a, b, s;
    const int64_t mask = (1ll << vl) - 1;
    const int64_t tid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x, stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t x = tid; x < TE; x += stride) {
        const uint64_t e = gl_mul(EH[x >> vl], EL[x & mask]);
        a.mac(e, gl_from_i64(D[x]));
        b.mac(e, gl_from_i64(l[x]));
    }
    for (int64_t t = tid; t < T; t += stride) s.add(ewt[t]);
    uint64_t v[3] = {a.value(), b.value(), s.value()};
    if (grid_sum_gl<3>(v, part, ticket) && threadIdx.x == 0) {
        out[0] = v[0];
        out[1] = v[1];
        out[2] = v[2];
    }
}

struct RouteArgs {
    uint64_t* V[6];  // eq(z_t, t), H, l, G, eq(w, x), eq(w_t, t): 2^n entries each, folded in place
    uint64_t lam1, lam2;
    int n;
    int grid;
    int per_block;
    int pad;
    uint64_t seq0;  // round t publishes seq0 + t, the final values seq0 + n + 1
    int t_begin;    // rounds run by this launch: [t_begin, t_end]; t_end > n includes the final values
    int t_end;
};

__device__ __forceinline__ uint64_t rt_at2(uint64_t a, uint64_t b) { return gl_sub(gl_add(b, b), a); }

__global__ void __launch_bounds__(RT_THREADS, 2) route_session_kernel(RouteArgs A, FpMailbox* mb, FpRelay* rl,
                                                                     uint64_t* part) {
    uint64_t rprev = 0;
    for (int t = A.t_begin; t <= A.n && t <= A.t_end; t++) {
        if (t > 1 && !session_wait(mb, rl, A.seq0 + t - 1, rprev)) return;
        const int64_t h = 1ll << (A.n - t);
        const int64_t want = (h + A.per_block - 1) / A.per_block;
        const unsigned active = (unsigned)(want < 1 ? 1 : (want > A.grid ? A.grid : want));
        if (blockIdx.x >= active) return;  // no pairs for this block in this or any later round
        GlAcc g0, g1, g2, g3;
        for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < h; b += (int64_t)active * blockDim.x) {
            uint64_t lo[6], hi[6];
#pragma unroll
            for (int k = 0; k < 6; k++) {
                uint64_t* V = A.V[k];
                if (t == 1) {
                    lo[k] = __ldcg(V + b);
                    hi[k] = __ldcg(V + b + h);
                } else {
                    // the vectors of length 4h folded by rho_{t-1}
                    lo[k] = gl_fold_fast(__ldcg(V + b), __ldcg(V + b + 2 * h), rprev);
                    hi[k] = gl_fold_fast(__ldcg(V + b + h), __ldcg(V + b + 3 * h), rprev);
                    V[b] = lo[k];
                    V[b + h] = hi[k];
                }
            }
#pragma unroll
            for (int X = 0; X < 4; X++) {
                uint64_t at[6];
#pragma unroll
                for (int k = 0; k < 6; k++)
                    at[k] = X == 0 ? lo[k] : (X == 1 ? hi[k] : (X == 2 ? rt_at2(lo[k], hi[k])
                                                                       : rt_at2(hi[k], rt_at2(lo[k], hi[k]))));
                const uint64_t Hx = at[1];
                uint64_t f = gl_mul(at[0], gl_mul(Hx, gl_sub(at[2], at[3])));
                f = gl_add(f, gl_mul(A.lam1, gl_mul(at[4], gl_mul(Hx, gl_sub(1, Hx)))));
                f = gl_add(f, gl_mul(A.lam2, gl_mul(at[5], Hx)));
                if (X == 0) g0.add(f);
                else if (X == 1) g1.add(f);
                else if (X == 2) g2.add(f);
                else g3.add(f);
            }
        }
        uint64_t acc[4] = {g0.value(), g1.value(), g2.value(), g3.value()};
        bool last;
        if (active == 1) {
            block_sum_gl<4>(acc);
            last = true;
        } else {
            last = grid_sum_gl_n<4>(acc, part, &rl->ticket, active);
        }
        if (last && threadIdx.x == 0) session_publish(mb, acc, A.seq0 + t);  // {g(0), g(1), g(2), g(3)}
    }
    // block 0 folds the last pair by the last challenge: H~(rho), l~(rho)
    if (A.t_end <= A.n || blockIdx.x != 0) return;
    if (!session_wait(mb, rl, A.seq0 + A.n, rprev)) return;
    if (threadIdx.x == 0) {
        const uint64_t fin[2] = {gl_fold_fast(__ldcg(A.V[1]), __ldcg(A.V[1] + 1), rprev),
                                 gl_fold_fast(__ldcg(A.V[2]), __ldcg(A.V[2] + 1), rprev)};
        session_publish(mb, fin, A.seq0 + A.n + 1);
    }
}

// ---- the host half ------------------------------------------------------------

// Where the device values come from. Each call returns FP_OK or an error status.
struct RouteSource {
    virtual ~RouteSource() {}
    virtual void abandon() {}  // the host stopped early: let a waiting kernel finish
    virtual int start(const uint64_t* z, const uint64_t* w, int n, uint64_t lam1, uint64_t lam2) = 0;
    virtual int opens(uint64_t out[3]) = 0;  // D~(z), l~(z), sum_{t < T} eq(w_t, t)
    virtual int round(int t, uint64_t g[4]) = 0;
    virtual int answer(int t, uint64_t rho) = 0;
    virtual int finals(uint64_t fin[2]) = 0;  // H~(rho), l~(rho)
};

// The routing sum-check after "route_site" is absorbed: 16 + 32 n + 16 proof bytes.
int route_protocol(fp_ctx* c, fp_tx* tx, int n, RouteSource& src, uint8_t* proof, size_t* proof_len) {
    uint64_t z[RT_MAX_N] = {}, w[RT_MAX_N] = {};
    for (int i = 0; i < n; i++) z[i] = fp_tx_squeeze_one(tx, "route_z");
    for (int i = 0; i < n; i++) w[i] = fp_tx_squeeze_one(tx, "route_w");
    const uint64_t lam1 = fp_tx_squeeze_one(tx, "route_lambda");
    const uint64_t lam2 = fp_tx_squeeze_one(tx, "route_lambda");
    int rc;
    if ((rc = src.start(z, w, n, lam1, lam2))) return rc;
    uint64_t o[3];
    if ((rc = src.opens(o))) return rc;
    size_t pos = 0;
    put_u64s(proof + pos, o, 2);
    fp_tx_absorb_raw(tx, "route_open", proof + pos, 16);
    pos += 16;
    uint64_t claim = gl_add(gl_add(o[0], o[1]), gl_mul(lam2, o[2]));
    for (int t = 1; t <= n; t++) {
        uint64_t g[4];
        if ((rc = src.round(t, g))) return rc;
        if (gl_add(g[0], g[1]) != claim) {
            src.abandon();
            return fp_fail(c, FP_ERR_CUDA, "sumcheck_prove_routing: round values inconsistent with the claim");
        }
        put_u64s(proof + pos, g, 4);
        fp_tx_absorb_raw(tx, "route_round", proof + pos, 32);
        pos += 32;
        const uint64_t r = fp_tx_squeeze_one(tx, "route_chal");
        if ((rc = src.answer(t, r))) return rc;
        claim = fp_lagrange4(g, r);
    }
    uint64_t fin[2];
    if ((rc = src.finals(fin))) return rc;
    put_u64s(proof + pos, fin, 2);
    fp_tx_absorb_raw(tx, "route_final", proof + pos, 16);
    pos += 16;
    *proof_len = pos;
    return FP_OK;
}

// Device values from the kernels above.
struct RouteDevice : RouteSource {
    fp_ctx* c;
    cudaStream_t st;
    const int8_t* l;
    const uint8_t* H;
    const int32_t* D;
    int64_t T;
    int E, vT, vE;
    uint64_t* V[6];
    uint64_t *et, *ewt, *eqe, *G, *EH, *EL, *part, *small, *hs;
    RouteArgs A;
    int cap_grid = 1;

    void abandon() override { fp_session_abandon(c, st); }

    int start(const uint64_t* z, const uint64_t* w, int n, uint64_t lam1, uint64_t lam2) override {
        int rc;
        const int64_t L = 1ll << n, TE = T * (int64_t)E;
        // eq tables: z_t, z_e, w (whole), w_t, and z split in halves for the openings
        FpPoint p;
        p.v = vT;
        for (int i = 0; i < vT; i++) p.z[i] = z[i];
        if ((rc = fp_eq_table(c, p, et, st))) return rc;
        p.v = vE;
        for (int i = 0; i < vE; i++) p.z[i] = z[vT + i];
        if ((rc = fp_eq_table(c, p, eqe, st))) return rc;
        p.v = n;
        for (int i = 0; i < n; i++) p.z[i] = w[i];
        if ((rc = fp_eq_table(c, p, V[4], st))) return rc;
        p.v = vT;
        if ((rc = fp_eq_table(c, p, ewt, st))) return rc;  // w_1..w_vT
        const int vl = n / 2, vh = n - vl;
        p.v = vh;
        for (int i = 0; i < vh; i++) p.z[i] = z[i];
        if ((rc = fp_eq_table(c, p, EH, st))) return rc;
        p.v = vl;
        for (int i = 0; i < vl; i++) p.z[i] = z[vh + i];
        if ((rc = fp_eq_table(c, p, EL, st))) return rc;
        int slot;
        fp_tic(c, st, K_ROUTE_VECTORS, 48.0 * (double)L + 9.0 * (double)TE, &slot);
        route_prefix_kernel<<<1, 1, 0, st>>>(eqe, E, G);
        route_vectors_kernel<<<fp_grid256(c, L), 256, 0, st>>>(l, H, TE, vE, L, et, ewt, G, V[0], V[1], V[2], V[3], V[5]);
        fp_toc(c, st, slot);
        FP_CUDA(c, cudaGetLastError());
        c->launches++;  // two kernels under one timing slot
        fp_tic(c, st, K_ROUTE_OPEN, 5.0 * (double)TE, &slot);
        route_open_kernel<<<fp_grid256(c, TE), RT_THREADS, 0, st>>>(D, l, TE, EH, EL, vl, ewt, T, part, c->tickets, small);
        fp_toc(c, st, slot);
        FP_CUDA(c, cudaGetLastError());
        memset(&A, 0, sizeof A);
        for (int k = 0; k < 6; k++) A.V[k] = V[k];
        A.lam1 = lam1;
        A.lam2 = lam2;
        A.n = n;
        return FP_OK;
    }

    double round_bytes(int t) const {
        const double pairs = (double)(1ll << (A.n - t));
        // six vectors: round 1 reads two values of each per pair, later rounds read four and write two
        return t == 1 ? 96.0 * pairs : 288.0 * pairs;
    }

    int launch(int t_begin, int t_end, unsigned grid, int kernel, double bytes) {
        A.t_begin = t_begin;
        A.t_end = t_end;
        void* args[] = {&A, &c->mb_dev, &c->relay, &part};
        int slot;
        fp_tic(c, st, kernel, bytes, &slot);
        FP_CUDA(c, cudaLaunchCooperativeKernel((const void*)route_session_kernel, dim3(grid), dim3(RT_THREADS), args,
                                               0, st));
        fp_toc(c, st, slot);
        return FP_OK;
    }

    int opens(uint64_t out[3]) override {
        FP_CUDA(c, cudaMemcpyAsync(hs, small, 24, cudaMemcpyDeviceToHost, st));
        FP_CUDA(c, cudaStreamSynchronize(st));
        out[0] = hs[0];
        out[1] = hs[1];
        out[2] = hs[2];
        if (A.n == 0) return FP_OK;
        int rc;
        A.per_block = RT_THREADS;  // one pair per thread
        const int64_t half = 1ll << (A.n - 1);
        A.grid = (int)std::max<int64_t>(1, std::min<int64_t>((half + A.per_block - 1) / A.per_block, cap_grid));
        A.seq0 = fp_seq_reserve(c, (uint64_t)A.n + 2);
        if ((rc = fp_session_begin(c, st))) return rc;
        fp_session_expect(c, 4);  // before any launch: round 1 publishes without a challenge
        if (!c->stepped) {
            double bytes = 0;
            for (int t = 1; t <= A.n; t++) bytes += round_bytes(t);
            return launch(1, A.n + 1, (unsigned)A.grid, K_ROUTE_ROUND, bytes);
        }
        return FP_OK;
    }

    int round(int t, uint64_t g[4]) override {
        int rc;
        if (c->stepped && (rc = launch(t, t, (unsigned)A.grid, K_ROUTE_ROUND, round_bytes(t)))) return rc;
        if ((rc = fp_session_wait(c, A.seq0 + t, st))) return rc;
        for (int i = 0; i < 4; i++) g[i] = c->mb->res[i];
        return FP_OK;
    }

    int answer(int t, uint64_t rho) override {
        fp_session_expect(c, t < A.n ? 4 : 2);  // the last challenge triggers the final values
        fp_session_post(c, A.seq0 + t, rho);
        return FP_OK;
    }

    int finals(uint64_t fin[2]) override {
        if (A.n == 0) {  // one token, one expert: the single entries
            FP_CUDA(c, cudaMemcpyAsync(hs, V[1], 8, cudaMemcpyDeviceToHost, st));
            FP_CUDA(c, cudaMemcpyAsync(hs + 1, V[2], 8, cudaMemcpyDeviceToHost, st));
            FP_CUDA(c, cudaStreamSynchronize(st));
            fin[0] = hs[0];
            fin[1] = hs[1];
            return FP_OK;
        }
        int rc;
        if (c->stepped && (rc = launch(A.n + 1, A.n + 1, 1, K_ROUTE_FINAL, 32.0))) return rc;
        if ((rc = fp_session_wait(c, A.seq0 + A.n + 1, st))) return rc;
        fin[0] = c->mb->res[0];
        fin[1] = c->mb->res[1];
        FP_CUDA(c, cudaStreamSynchronize(st));
        return FP_OK;
    }
};

// Device values from a caller's callback (no device).
struct RouteCallback : RouteSource {
    fp_values_fn fn;
    void* user;
    int call(int kind, int t, const uint64_t* in, uint64_t* out) { return fn(user, kind, t, in, out) ? FP_ERR_ARG : FP_OK; }
    int start(const uint64_t* z, const uint64_t* w, int n, uint64_t lam1, uint64_t lam2) override {
        uint64_t in[2 * RT_MAX_N + 2];
        for (int i = 0; i < n; i++) {
            in[i] = z[i];
            in[n + i] = w[i];
        }
        in[2 * n] = lam1;
        in[2 * n + 1] = lam2;
        return call(FP_VAL_START, n, in, nullptr);
    }
    int opens(uint64_t out[3]) override {
        out[0] = out[1] = out[2] = 0;
        const int rc = call(FP_VAL_CLAIM, 0, nullptr, out);
        for (int i = 0; i < 3; i++) out[i] = gl_canon(out[i]);
        return rc;
    }
    int round(int t, uint64_t g[4]) override {
        for (int i = 0; i < 4; i++) g[i] = 0;
        const int rc = call(FP_VAL_ROUND, t, nullptr, g);
        for (int i = 0; i < 4; i++) g[i] = gl_canon(g[i]);
        return rc;
    }
    int answer(int t, uint64_t rho) override { return call(FP_VAL_ANSWER, t, &rho, nullptr); }
    int finals(uint64_t fin[2]) override {
        fin[0] = fin[1] = 0;
        const int rc = call(FP_VAL_FINALS, 0, nullptr, fin);
        fin[0] = gl_canon(fin[0]);
        fin[1] = gl_canon(fin[1]);
        return rc;
    }
};

size_t route_part_len(int n) { return 16 + 32 * (size_t)n + 16; }

}  // namespace

int sumcheck_prove_routing(fp_ctx* c, fp_tx* tx, const int8_t* logits, int64_t T, int E, uint8_t* H, int32_t* D,
                           uint8_t* proof, size_t* proof_len, void* stream) {
    if (!c || !tx || !proof_len || !logits || !H || !D)
        return fp_fail(c, FP_ERR_ARG, "sumcheck_prove_routing: null argument");
    if (E < 1 || E > RT_MAX_E || (E & (E - 1)))
        return fp_fail(c, FP_ERR_SHAPE, "sumcheck_prove_routing: E must be a power of two in [1, 4096]");
    const int vE = fp_log2_ceil((uint64_t)E);
    if (T < 1 || fp_log2_ceil((uint64_t)T) + vE > RT_MAX_N)
        return fp_fail(c, FP_ERR_SHAPE, "sumcheck_prove_routing: need T >= 1 and ceil(log2 T) + log2 E <= 26");
    const int vT = fp_log2_ceil((uint64_t)T), n = vT + vE;
    const int64_t TE = T * (int64_t)E, L = 1ll << n;
    const size_t need_len = route_part_len(n) + fp_lhi_proof_len(TE, 8);
    if (!proof || *proof_len < need_len) {
        *proof_len = need_len;
        return fp_fail(c, FP_ERR_ARG, "sumcheck_prove_routing: proof buffer too small");
    }
    FP_CUDA(c, cudaSetDevice(c->device));
    cudaStream_t st = (cudaStream_t)stream;
    int rc;
    RouteDevice dev;
    dev.c = c;
    dev.st = st;
    dev.l = logits;
    dev.H = H;
    dev.D = D;
    dev.T = T;
    dev.E = E;
    dev.vT = vT;
    dev.vE = vE;
    int occ = 0;
    FP_CUDA(c, cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, route_session_kernel, RT_THREADS, 0));
    dev.cap_grid = std::max(1, occ) * c->num_sms;
    const size_t part_n = (size_t)4 * std::max(dev.cap_grid, 4 * c->num_sms);
    size_t lhi_host = 0;
    const size_t lhi_dev = fp_lhi_scratch(c, TE, 8, &lhi_host);
    const int vl = n / 2, vh = n - vl;
    const size_t need = 6 * fp_align_up((size_t)8 * L, 256) + 2 * fp_align_up((size_t)8 << vT, 256) +
                        2 * fp_align_up((size_t)8 * E, 256) + fp_align_up((size_t)8 << vh, 256) +
                        fp_align_up((size_t)8 << vl, 256) + fp_align_up(8 * part_n, 256) + fp_align_up(8 * 64, 256) +
                        fp_align_up((size_t)4 * TE, 256) + lhi_dev + 8192;
    if ((rc = fp_reserve(c, c->dev, need))) return rc;
    if ((rc = fp_reserve(c, c->host, fp_align_up(8 * 64, 256) + lhi_host + 8192))) return rc;
    fp_reset(c->dev);
    fp_reset(c->host);
    for (int k = 0; k < 6; k++) dev.V[k] = (uint64_t*)fp_alloc(c->dev, (size_t)8 * L);
    dev.et = (uint64_t*)fp_alloc(c->dev, (size_t)8 << vT);
    dev.ewt = (uint64_t*)fp_alloc(c->dev, (size_t)8 << vT);
    dev.eqe = (uint64_t*)fp_alloc(c->dev, (size_t)8 * E);
    dev.G = (uint64_t*)fp_alloc(c->dev, (size_t)8 * E);
    dev.EH = (uint64_t*)fp_alloc(c->dev, (size_t)8 << vh);
    dev.EL = (uint64_t*)fp_alloc(c->dev, (size_t)8 << vl);
    dev.part = (uint64_t*)fp_alloc(c->dev, 8 * part_n);
    dev.small = (uint64_t*)fp_alloc(c->dev, 8 * 64);
    int32_t* keys = (int32_t*)fp_alloc(c->dev, (size_t)4 * TE);
    dev.hs = (uint64_t*)fp_alloc(c->host, 8 * 64);
    bool ok = dev.et && dev.ewt && dev.eqe && dev.G && dev.EH && dev.EL && dev.part && dev.small && keys && dev.hs;
    for (int k = 0; k < 6; k++) ok = ok && dev.V[k];
    if (!ok) return fp_fail(c, FP_ERR_OOM, "sumcheck_prove_routing: scratch exhausted");

    // ---- the witness: the first argmax of every row ----
    {
        int slot;
        fp_tic(c, st, K_ROUTE_WITNESS, 10.0 * (double)TE, &slot);
        const int64_t warps = std::min<int64_t>(T, 8ll * c->num_sms * 8);
        route_witness_kernel<<<(unsigned)((warps + 7) / 8), 256, 0, st>>>(logits, T, E, H, D, keys);
        fp_toc(c, st, slot);
        FP_CUDA(c, cudaGetLastError());
    }
    {
        FpDigestJob jobs[3] = {{(const uint8_t*)logits, (uint64_t)TE}, {(const uint8_t*)H, (uint64_t)TE},
                               {(const uint8_t*)D, 4 * (uint64_t)TE}};
        uint8_t d[96];
        if ((rc = fp_digest_many(c, jobs, 3, d, st))) return rc;  // synchronises the stream
        fp_tx_absorb_raw(tx, "route_site", d, 96);
    }
    size_t part_len = 0;
    if ((rc = route_protocol(c, tx, n, dev, proof, &part_len))) return rc;
    // ---- the range of D: the helper-inverse LogUp of D - 128 on R_8 ----
    size_t lhi_len = *proof_len - part_len;
    rc = fp_lhi_run(c, tx, keys, TE, 8, proof + part_len, &lhi_len, st);
    if (rc < 0) return rc;
    *proof_len = part_len + lhi_len;
    return rc;  // 1 only if some key lies outside R_8, which the first argmax never gives
}

int fp_route_protocol_drive(fp_tx* tx, int n, fp_values_fn fn, void* user, uint8_t* proof, size_t* proof_len) {
    if (!tx || !fn || !proof_len) return FP_ERR_ARG;
    if (n < 0 || n > RT_MAX_N) return FP_ERR_SHAPE;
    const size_t need_len = route_part_len(n);
    if (!proof || *proof_len < need_len) {
        *proof_len = need_len;
        return FP_ERR_ARG;
    }
    RouteCallback cb;
    cb.fn = fn;
    cb.user = user;
    return route_protocol(nullptr, tx, n, cb, proof, proof_len);
}
