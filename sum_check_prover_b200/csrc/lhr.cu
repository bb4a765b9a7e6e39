// The rescale lookups by helper inverses: the lookup section of the layer proof
// in the form of LogUp after Haboeck 2022 ("Towards Proving Frontier-Scale LLM
// Inference", The proof system), set against the fraction tree with one
// sum-check per level ("How fast can FlashProve go", 4 Tighter Rooflines).
//
// The same keys, tables and multiplicities as logup_prove_rescale (remainder
// table R_k with key r, clamp table C16 with key q + gamma y); instead of the
// tree, two committed helper columns and one degree-3 sum-check:
//   send m_rem (2^k u32; digest absorbed, "lhr_m_rem"); squeeze gamma
//   ("lhr_gamma"); send m_clamp (2^16 u32, "lhr_m_clamp"); squeeze alpha0,
//   alpha1 ("lhr_alpha"); commit h0_i = 1 / (alpha0 - r_i) and
//   h1_i = 1 / (alpha1 - q_i - gamma y_i): absorb "lhr_h" D(h0) || D(h1);
//   squeeze z_1..z_v ("lhr_z"), beta ("lhr_beta"); send S0 = sum h0,
//   S1 = sum h1 ("lhr_sum"); sum-check over v variables of
//     G = h0 + beta h1 + eq(z, .) (beta^2 (h0 (alpha0 - r) - 1)
//                                  + beta^3 (h1 (alpha1 - q - gamma y) - 1))
//   with claim S0 + beta S1: rounds g(0..3) ("lhr_round"), "lhr_chal"; send
//   h0, h1, r, q, y at rho ("lhr_final").
// v rounds (one host round trip each) instead of the tree's v (v - 1) / 2, for
// two committed columns: 16 bytes a key written and hashed.
//
// Kernels: the inverses of the 2^k + 2^16 table rows (one exponentiation each);
// the two helper columns as gathers from them (a key that is no row of its
// table takes its own inverse, so the columns are right for any witness); their
// digests; then every round in one resident cooperative launch. With
// A0_t(X) = sum_b h0_t(X, b), A1_t likewise (linear in X), and
// Q0_t(X) = sum_b eq(z_>t, b) h0_t(X, b) (alpha0 - r_t(X, b)), Q1_t with
// h1 (alpha1 - q - gamma y) (quadratic), the device returns A0(0), A0(1),
// A1(0), A1(1), Q0(0..2), Q1(0..2) and the host forms
//   g_t(X) = A0(X) + beta A1(X)
//            + eq(z_<t, rho_<t) eq(z_t, X) (beta^2 (Q0(X) - 1) + beta^3 (Q1(X) - 1)),
// the weights eq(z_>t, .) summing to 1. Round 1 gives S0 = A0(0) + A0(1) and
// S1 likewise, and g_1(0) + g_1(1) = S0 + beta S1 is checked like every round.
//
// The host half (lhr_protocol) takes its device values from a source: the
// kernels here, or a caller's callback (fp_lhr_protocol_drive).
#include <string.h>

#include <algorithm>

#include "fp_eqchunks.cuh"
#include "fp_internal.h"
#include "fp_reduce.cuh"
#include "fp_session.cuh"

namespace {

constexpr int LR_THREADS = 256;
constexpr int LR_MAX_V = 30;

struct LhrChal {
    uint64_t a0, a1, gamma;
};

// inv0[j] = 1 / (alpha0 - (j - 2^(k-1))), j < 2^k; inv1[j] = 1 / (alpha1 - v_j - gamma clamp(v_j)),
// v_j = j - 2^15, j < 2^16 (the inverse of 0 is taken as 0)
__global__ void lhr_inv_kernel(LhrChal C, int k, uint64_t* __restrict__ inv0, uint64_t* __restrict__ inv1) {
    const int64_t T0 = 1ll << k, half = T0 >> 1, n = T0 + 65536;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        if (i < T0) {
            inv0[i] = gl_inv(gl_sub(C.a0, gl_from_i64(i - half)));
        } else {
            const int32_t v = (int32_t)(i - T0) - 32768;
            const int32_t cv = v < -128 ? -128 : (v > 127 ? 127 : v);
            inv1[i - T0] = gl_inv(gl_sub(C.a1, gl_add(gl_from_i64(v), gl_mul_small(C.gamma, cv))));
        }
    }
}

__device__ __forceinline__ void lr_key(const FpKeyCols& K, int64_t i, int32_t& r, int32_t& q, int32_t& y) {
    if (i < K.n) {
        r = K.r[i];
        q = K.q[i];
        y = K.y[i];
    } else {
        r = q = y = 0;
    }
}

// the helper columns over the 2^v padded keys: a key that is a row of its table takes the row's
// inverse, any other key its own
__global__ void lhr_column_kernel(FpKeyCols K, int64_t L, int k, LhrChal C, const uint64_t* __restrict__ inv0,
                                  const uint64_t* __restrict__ inv1, uint64_t* __restrict__ h0,
                                  uint64_t* __restrict__ h1) {
    const int64_t T0 = 1ll << k, half = T0 >> 1;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < L; i += (int64_t)gridDim.x * blockDim.x) {
        int32_t r, q, y;
        lr_key(K, i, r, q, y);
        const int64_t j0 = (int64_t)r + half, j1 = (int64_t)q + 32768;
        h0[i] = (j0 >= 0 && j0 < T0) ? __ldg(inv0 + j0) : gl_inv(gl_sub(C.a0, gl_from_i64(r)));
        const int32_t cq = q < -128 ? -128 : (q > 127 ? 127 : q);
        h1[i] = (j1 >= 0 && j1 < 65536 && y == cq)
                    ? __ldg(inv1 + j1)
                    : gl_inv(gl_sub(C.a1, gl_add(gl_from_i64(q), gl_mul_small(C.gamma, y))));
    }
}

struct LhrArgs {
    FpKeyCols keys;
    const uint64_t* h0;  // the helper columns (2^v entries each)
    const uint64_t* h1;
    uint64_t* V[5];      // h0, h1, r, q, y folded, from round 2 on (2^(v-1) entries each)
    uint64_t* E;         // eq(z_>t, .) (2^(v-1) entries)
    const uint64_t* z;   // device copy of z_1..z_v
    LhrChal C;
    int v;
    int grid;
    int per_block;
    int pad;
    uint64_t seq0;  // round t publishes seq0 + t, the final values seq0 + v + 1
    int t_begin;    // rounds run by this launch: [t_begin, t_end]; t_end > v includes the final values
    int t_end;
};

// the five column values at position i of the unfolded columns: h0, h1, r, q, y
__device__ __forceinline__ void lr_raw(const LhrArgs& A, int64_t i, uint64_t (&c)[5]) {
    int32_t r, q, y;
    lr_key(A.keys, i, r, q, y);
    c[0] = __ldg(A.h0 + i);
    c[1] = __ldg(A.h1 + i);
    c[2] = gl_from_i64(r);
    c[3] = gl_from_i64(q);
    c[4] = gl_from_i64(y);
}

// X = 2 on the line through (a, b) at 0 and 1
__device__ __forceinline__ uint64_t lr_at2(uint64_t a, uint64_t b) { return gl_sub(gl_add(b, b), a); }

__global__ void __launch_bounds__(LR_THREADS, 2) lhr_session_kernel(LhrArgs A, FpMailbox* mb, FpRelay* rl,
                                                                   uint64_t* part) {
    __shared__ uint64_t zs[32];
    __shared__ uint64_t eq_tab[3 << kEqChunk];
    if (threadIdx.x < A.v) zs[threadIdx.x] = A.z[threadIdx.x];
    __syncthreads();
    const uint64_t a0 = A.C.a0, a1 = A.C.a1, gamma = A.C.gamma;
    uint64_t rprev = 0;
    for (int t = A.t_begin; t <= A.v && t <= A.t_end; t++) {
        if (t > 1 && !session_wait(mb, rl, A.seq0 + t - 1, rprev)) return;
        const int64_t h = 1ll << (A.v - t);
        const int64_t want = (h + A.per_block - 1) / A.per_block;
        const unsigned active = (unsigned)(want < 1 ? 1 : (want > A.grid ? A.grid : want));
        if (blockIdx.x >= active) return;  // no pairs for this block in this or any later round
        EqChunks EC{0, 0, 0};
        if (t == 1) EC = eq_chunks_build(eq_tab, zs, A.v);
        GlAcc S00, S01, S10, S11, Q0[3], Q1[3];
        for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < h; b += (int64_t)active * blockDim.x) {
            uint64_t c0[5], c1[5], e;
            if (t == 1) {
                lr_raw(A, b, c0);
                lr_raw(A, b + h, c1);
                e = eq_chunks_at(EC, eq_tab, b);  // eq(z_2..z_v, b)
                if (A.v > 1) A.E[b] = e;
            } else {
                uint64_t s0[5], s1[5], s2[5], s3[5];
                if (t == 2) {  // the columns and the keys (length 4h) folded by rho_1
                    lr_raw(A, b, s0);
                    lr_raw(A, b + h, s1);
                    lr_raw(A, b + 2 * h, s2);
                    lr_raw(A, b + 3 * h, s3);
                } else {
#pragma unroll
                    for (int i = 0; i < 5; i++) {
                        s0[i] = __ldcg(A.V[i] + b);
                        s1[i] = __ldcg(A.V[i] + b + h);
                        s2[i] = __ldcg(A.V[i] + b + 2 * h);
                        s3[i] = __ldcg(A.V[i] + b + 3 * h);
                    }
                }
#pragma unroll
                for (int i = 0; i < 5; i++) {
                    c0[i] = gl_fold_fast(s0[i], s2[i], rprev);
                    c1[i] = gl_fold_fast(s1[i], s3[i], rprev);
                    A.V[i][b] = c0[i];
                    A.V[i][b + h] = c1[i];
                }
                e = gl_add(__ldcg(A.E + b), __ldcg(A.E + b + h));  // eq(z_>t, b)
                A.E[b] = e;
            }
            S00.add(c0[0]);
            S01.add(c1[0]);
            S10.add(c0[1]);
            S11.add(c1[1]);
#pragma unroll
            for (int X = 0; X < 3; X++) {
                uint64_t c[5];
#pragma unroll
                for (int i = 0; i < 5; i++) c[i] = X == 0 ? c0[i] : (X == 1 ? c1[i] : lr_at2(c0[i], c1[i]));
                Q0[X].mac(e, gl_mul_weak(c[0], gl_sub(a0, c[2])));
                Q1[X].mac(e, gl_mul_weak(c[1], gl_sub(a1, gl_add(c[3], gl_mul(gamma, c[4])))));
            }
        }
        uint64_t acc[10] = {S00.value(), S01.value(), S10.value(), S11.value(), Q0[0].value(), Q0[1].value(),
                            Q0[2].value(), Q1[0].value(), Q1[1].value(), Q1[2].value()};
        bool last;
        if (active == 1) {
            block_sum_gl<10>(acc);
            last = true;
        } else {
            last = grid_sum_gl_n<10>(acc, part, &rl->ticket, active);
        }
        if (last && threadIdx.x == 0) session_publish(mb, acc, A.seq0 + t);
    }
    // block 0 folds the last pair by the last challenge: h0, h1, r, q, y at rho
    if (A.t_end <= A.v || blockIdx.x != 0) return;
    if (!session_wait(mb, rl, A.seq0 + A.v, rprev)) return;
    if (threadIdx.x == 0) {
        uint64_t c0[5], c1[5];
        if (A.v == 1) {
            lr_raw(A, 0, c0);
            lr_raw(A, 1, c1);
        } else {
#pragma unroll
            for (int i = 0; i < 5; i++) {
                c0[i] = __ldcg(A.V[i]);
                c1[i] = __ldcg(A.V[i] + 1);
            }
        }
        uint64_t fin[5];
#pragma unroll
        for (int i = 0; i < 5; i++) fin[i] = gl_fold_fast(c0[i], c1[i], rprev);
        session_publish(mb, fin, A.seq0 + A.v + 1);
    }
}

// ---- the host half ------------------------------------------------------------

struct LhrSource {
    virtual ~LhrSource() {}
    virtual void abandon() {}                                         // the host stopped early
    virtual int column(const LhrChal& C, uint8_t digest[64]) = 0;     // commit h0, h1: D(h0) || D(h1)
    virtual int start(const uint64_t* z, int v, uint64_t beta) = 0;  // the point is known
    virtual int round(int t, uint64_t vals[10]) = 0;                 // A0(0), A0(1), A1(0), A1(1), Q0(0..2), Q1(0..2)
    virtual int answer(int t, uint64_t rho) = 0;                     // the challenge rho_t
    virtual int finals(uint64_t fin[5]) = 0;                         // h0, h1, r, q, y at rho
};

size_t lhr_proof_len(int v, int k) { return 4 * ((size_t)1 << k) + 4 * 65536 + 16 + 32 * (size_t)v + 40; }

// The section from the multiplicities on. hm: 2^k u32 of m_rem, then 2^16 of m_clamp.
int lhr_protocol(fp_ctx* c, fp_tx* tx, int v, int k, const uint8_t* hm, const uint8_t dg_rem[32],
                 const uint8_t dg_cl[32], LhrSource& src, uint8_t* proof, size_t* proof_len) {
    int rc;
    size_t pos = 0;
    const size_t T = (size_t)1 << k;
    memcpy(proof + pos, hm, 4 * T);  // little-endian u32 words
    pos += 4 * T;
    fp_tx_absorb_raw(tx, "lhr_m_rem", dg_rem, 32);
    LhrChal C;
    C.gamma = fp_tx_squeeze_one(tx, "lhr_gamma");
    memcpy(proof + pos, hm + 4 * T, 4 * 65536);
    pos += 4 * 65536;
    fp_tx_absorb_raw(tx, "lhr_m_clamp", dg_cl, 32);
    C.a0 = fp_tx_squeeze_one(tx, "lhr_alpha");
    C.a1 = fp_tx_squeeze_one(tx, "lhr_alpha");
    {
        uint8_t hd[64];
        if ((rc = src.column(C, hd))) return rc;
        fp_tx_absorb_raw(tx, "lhr_h", hd, 64);
    }
    uint64_t z[LR_MAX_V];
    for (int i = 0; i < v; i++) z[i] = fp_tx_squeeze_one(tx, "lhr_z");
    const uint64_t beta = fp_tx_squeeze_one(tx, "lhr_beta");
    const uint64_t b2 = gl_mul(beta, beta), b3 = gl_mul(b2, beta);
    if ((rc = src.start(z, v, beta))) return rc;
    uint64_t claim = 0, pre = 1;  // pre = eq(z_<t, rho_<t)
    for (int t = 1; t <= v; t++) {
        uint64_t w[10];
        if ((rc = src.round(t, w))) return rc;
        if (t == 1) {
            const uint64_t S[2] = {gl_add(w[0], w[1]), gl_add(w[2], w[3])};
            put_u64s(proof + pos, S, 2);
            fp_tx_absorb_raw(tx, "lhr_sum", proof + pos, 16);
            pos += 16;
            claim = gl_add(S[0], gl_mul(beta, S[1]));
        }
        const uint64_t zt = z[t - 1];
        // the linear sums at 0..3, the quadratic ones extended to 3: q(3) = q(0) - 3 q(1) + 3 q(2)
        uint64_t A0[4], A1[4], Q0[4], Q1[4];
        for (int X = 0; X < 4; X++) {
            A0[X] = gl_add(w[0], gl_mul(X, gl_sub(w[1], w[0])));
            A1[X] = gl_add(w[2], gl_mul(X, gl_sub(w[3], w[2])));
        }
        for (int X = 0; X < 3; X++) {
            Q0[X] = w[4 + X];
            Q1[X] = w[7 + X];
        }
        Q0[3] = gl_add(gl_sub(w[4], gl_mul(3, w[5])), gl_mul(3, w[6]));
        Q1[3] = gl_add(gl_sub(w[7], gl_mul(3, w[8])), gl_mul(3, w[9]));
        const uint64_t eqX[4] = {gl_sub(1, zt), zt, gl_sub(gl_mul(3, zt), 1), gl_sub(gl_mul(5, zt), 2)};
        uint64_t g[4];
        for (int X = 0; X < 4; X++) {
            const uint64_t zero = gl_add(gl_mul(b2, gl_sub(Q0[X], 1)), gl_mul(b3, gl_sub(Q1[X], 1)));
            g[X] = gl_add(gl_add(A0[X], gl_mul(beta, A1[X])), gl_mul(pre, gl_mul(eqX[X], zero)));
        }
        if (gl_add(g[0], g[1]) != claim) {
            src.abandon();
            return fp_fail(c, FP_ERR_CUDA, "logup_prove_rescale_hi: round values inconsistent with the claim");
        }
        put_u64s(proof + pos, g, 4);
        fp_tx_absorb_raw(tx, "lhr_round", proof + pos, 32);
        pos += 32;
        const uint64_t r = fp_tx_squeeze_one(tx, "lhr_chal");
        if ((rc = src.answer(t, r))) return rc;
        claim = fp_lagrange4(g, r);
        pre = gl_mul(pre, gl_add(gl_mul(zt, r), gl_mul(gl_sub(1, zt), gl_sub(1, r))));
    }
    uint64_t fin[5];
    if ((rc = src.finals(fin))) return rc;
    put_u64s(proof + pos, fin, 5);
    fp_tx_absorb_raw(tx, "lhr_final", proof + pos, 40);
    pos += 40;
    *proof_len = pos;
    return FP_OK;
}

// Device values from the kernels above.
struct LhrDevice : LhrSource {
    fp_ctx* c;
    cudaStream_t st;
    FpKeyCols K;
    int k, v;
    uint64_t *h0 = nullptr, *h1 = nullptr, *inv0 = nullptr, *inv1 = nullptr;
    uint64_t* part = nullptr;
    uint64_t* small = nullptr;  // device: [8 .. 8 + v) z
    uint64_t* hs = nullptr;     // pinned host staging
    LhrArgs A;
    int cap_grid = 1;

    int launch(int t_begin, int t_end, unsigned grid, int kernel, double bytes) {
        A.t_begin = t_begin;
        A.t_end = t_end;
        void* args[] = {&A, &c->mb_dev, &c->relay, &part};
        int slot;
        fp_tic(c, st, kernel, bytes, &slot);
        FP_CUDA(c, cudaLaunchCooperativeKernel((const void*)lhr_session_kernel, dim3(grid), dim3(LR_THREADS), args,
                                               0, st));
        fp_toc(c, st, slot);
        return FP_OK;
    }

    double round_bytes(int t) const {
        const double pairs = (double)(1ll << (v - t));
        // round 1: both columns and the keys at 2 positions (50 B) and one E write; round 2:
        // columns and keys at 4 positions, the five folded vectors written at 2, E read twice
        // and written; later rounds read the folded vectors at 4 positions instead
        return t == 1 ? 58.0 * pairs : (t == 2 ? 204.0 * pairs : 264.0 * pairs);
    }

    void abandon() override { fp_session_abandon(c, st); }

    int column(const LhrChal& C, uint8_t digest[64]) override {
        const int64_t L = 1ll << v, T0 = 1ll << k;
        int slot;
        fp_tic(c, st, K_LHR_COLUMN, 8.0 * (double)(T0 + 65536) + 9.0 * (double)K.n + 16.0 * (double)L, &slot);
        lhr_inv_kernel<<<fp_grid256(c, T0 + 65536), 256, 0, st>>>(C, k, inv0, inv1);
        lhr_column_kernel<<<fp_grid256(c, L), 256, 0, st>>>(K, L, k, C, inv0, inv1, h0, h1);
        fp_toc(c, st, slot);
        FP_CUDA(c, cudaGetLastError());
        c->launches++;  // two kernels under one timing slot
        A.C = C;
        FpDigestJob jobs[2] = {{(const uint8_t*)h0, 8 * (uint64_t)L}, {(const uint8_t*)h1, 8 * (uint64_t)L}};
        return fp_digest_many(c, jobs, 2, digest, st);  // synchronises the stream
    }

    int start(const uint64_t* z, int vv, uint64_t beta) override {
        (void)beta;  // the host alone applies beta
        int rc;
        for (int i = 0; i < vv; i++) hs[8 + i] = z[i];
        FP_CUDA(c, cudaMemcpyAsync(small + 8, hs + 8, 8 * (size_t)vv, cudaMemcpyHostToDevice, st));
        A.z = small + 8;
        A.v = vv;
        A.per_block = LR_THREADS;  // one pair per thread
        const int64_t half = 1ll << (vv - 1);
        A.grid = (int)std::max<int64_t>(1, std::min<int64_t>((half + A.per_block - 1) / A.per_block, cap_grid));
        A.seq0 = fp_seq_reserve(c, (uint64_t)vv + 2);
        if ((rc = fp_session_begin(c, st))) return rc;
        fp_session_expect(c, 10);  // before any launch: round 1 publishes without a challenge
        if (!c->stepped) {
            double bytes = 0;
            for (int t = 1; t <= vv; t++) bytes += round_bytes(t);
            return launch(1, vv + 1, (unsigned)A.grid, K_LHR_ROUND, bytes);
        }
        return FP_OK;
    }

    int round(int t, uint64_t vals[10]) override {
        int rc;
        if (c->stepped && (rc = launch(t, t, (unsigned)A.grid, K_LHR_ROUND, round_bytes(t)))) return rc;
        if ((rc = fp_session_wait(c, A.seq0 + t, st))) return rc;
        for (int i = 0; i < 10; i++) vals[i] = c->mb->res[i];
        return FP_OK;
    }

    int answer(int t, uint64_t rho) override {
        fp_session_expect(c, t < v ? 10 : 5);  // the last challenge triggers the final values
        fp_session_post(c, A.seq0 + t, rho);
        return FP_OK;
    }

    int finals(uint64_t fin[5]) override {
        int rc;
        if (c->stepped && (rc = launch(v + 1, v + 1, 1, K_LHR_FINAL, 80.0))) return rc;
        if ((rc = fp_session_wait(c, A.seq0 + v + 1, st))) return rc;
        for (int i = 0; i < 5; i++) fin[i] = c->mb->res[i];
        FP_CUDA(c, cudaStreamSynchronize(st));
        return FP_OK;
    }
};

// Device values from a caller's callback (no device).
struct LhrCallback : LhrSource {
    fp_values_fn fn;
    void* user;
    int call(int kind, int t, const uint64_t* in, uint64_t* out) { return fn(user, kind, t, in, out) ? FP_ERR_ARG : FP_OK; }
    int column(const LhrChal& C, uint8_t digest[64]) override {
        uint64_t in[3] = {C.a0, C.a1, C.gamma}, out[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        const int rc = call(FP_VAL_COLUMN, 0, in, out);
        for (int i = 0; i < 8; i++)
            for (int b = 0; b < 8; b++) digest[8 * i + b] = (uint8_t)(out[i] >> (8 * b));
        return rc;
    }
    int start(const uint64_t* z, int v, uint64_t beta) override {
        uint64_t in[LR_MAX_V + 1];
        for (int i = 0; i < v; i++) in[i] = z[i];
        in[v] = beta;
        return call(FP_VAL_START, v, in, nullptr);
    }
    int round(int t, uint64_t vals[10]) override {
        for (int i = 0; i < 10; i++) vals[i] = 0;
        const int rc = call(FP_VAL_ROUND, t, nullptr, vals);
        for (int i = 0; i < 10; i++) vals[i] = gl_canon(vals[i]);
        return rc;
    }
    int answer(int t, uint64_t rho) override { return call(FP_VAL_ANSWER, t, &rho, nullptr); }
    int finals(uint64_t fin[5]) override {
        for (int i = 0; i < 5; i++) fin[i] = 0;
        const int rc = call(FP_VAL_FINALS, 0, nullptr, fin);
        for (int i = 0; i < 5; i++) fin[i] = gl_canon(fin[i]);
        return rc;
    }
};

}  // namespace

int logup_prove_rescale_hi(fp_ctx* c, fp_tx* tx, const fp_site* sites, int nsites, uint8_t* proof,
                           size_t* proof_len, void* stream) {
    if (!c || !tx || !proof_len) return fp_fail(c, FP_ERR_ARG, "logup_prove_rescale_hi: null argument");
    int rc = fp_check_sites(c, sites, nsites, true);
    if (rc) return rc;
    for (int s = 1; s < nsites; s++)
        if (sites[s].k_shift != sites[0].k_shift)
            return fp_fail(c, FP_ERR_SHAPE, "logup_prove_rescale_hi: all sites must share k_shift");
    const int k = sites[0].k_shift;
    int64_t nk = 0;
    for (int s = 0; s < nsites; s++) nk += (int64_t)sites[s].M * sites[s].N;
    const int v = std::max(1, fp_log2_ceil((uint64_t)nk));
    if (v > LR_MAX_V) return fp_fail(c, FP_ERR_SHAPE, "logup_prove_rescale_hi: more than 2^30 keys");
    const size_t need_len = lhr_proof_len(v, k);
    if (!proof || *proof_len < need_len) {
        *proof_len = need_len;
        return fp_fail(c, FP_ERR_ARG, "logup_prove_rescale_hi: proof buffer too small");
    }
    FP_CUDA(c, cudaSetDevice(c->device));
    cudaStream_t st = (cudaStream_t)stream;
    const int64_t L = 1ll << v, T0 = 1ll << k, half = L / 2;
    int occ = 0;
    FP_CUDA(c, cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, lhr_session_kernel, LR_THREADS, 0));
    const int cap_grid = std::max(1, occ) * c->num_sms;
    const size_t part_n = (size_t)10 * cap_grid;
    size_t need = fp_lookup_keys_scratch(nsites, nk) + fp_lookup_mults_scratch(k);
    need += 2 * fp_align_up((size_t)8 * L, 256) + 6 * fp_align_up((size_t)8 * half, 256);
    need += fp_align_up((size_t)8 * T0, 256) + fp_align_up((size_t)8 * 65536, 256);
    need += fp_align_up(8 * part_n, 256) + fp_align_up(8 * 64, 256) + 4096;
    if ((rc = fp_reserve(c, c->dev, need))) return rc;
    // host: the multiplicities, the staging words, the gather table of the key columns
    if ((rc = fp_reserve(c, c->host, 4 * (size_t)T0 + 4 * 65536 + 256 + fp_align_up(8 * 64, 256) + 4096 +
                                         64 * (size_t)nsites)))
        return rc;
    fp_reset(c->dev);
    fp_reset(c->host);

    LhrDevice dev;
    dev.c = c;
    dev.st = st;
    dev.k = k;
    dev.v = v;
    dev.cap_grid = cap_grid;
    if ((rc = fp_lookup_keys(c, sites, nsites, st, &dev.K))) return rc;
    uint8_t* hm = (uint8_t*)fp_alloc(c->host, 4 * (size_t)T0 + 4 * 65536 + 256);
    uint8_t dg_rem[32], dg_cl[32];
    if ((rc = fp_lookup_mults(c, dev.K, k, L, st, hm, dg_rem, dg_cl))) return rc;
    uint32_t n_outside;
    memcpy(&n_outside, hm + 4 * T0 + 4 * 65536, 4);
    dev.h0 = (uint64_t*)fp_alloc(c->dev, (size_t)8 * L);
    dev.h1 = (uint64_t*)fp_alloc(c->dev, (size_t)8 * L);
    memset(&dev.A, 0, sizeof dev.A);
    for (int i = 0; i < 5; i++) dev.A.V[i] = (uint64_t*)fp_alloc(c->dev, (size_t)8 * half);
    dev.A.E = (uint64_t*)fp_alloc(c->dev, (size_t)8 * half);
    dev.inv0 = (uint64_t*)fp_alloc(c->dev, (size_t)8 * T0);
    dev.inv1 = (uint64_t*)fp_alloc(c->dev, (size_t)8 * 65536);
    dev.part = (uint64_t*)fp_alloc(c->dev, 8 * part_n);
    dev.small = (uint64_t*)fp_alloc(c->dev, 8 * 64);
    dev.hs = (uint64_t*)fp_alloc(c->host, 8 * 64);
    bool ok = dev.h0 && dev.h1 && dev.A.E && dev.inv0 && dev.inv1 && dev.part && dev.small && dev.hs;
    for (int i = 0; i < 5; i++) ok = ok && dev.A.V[i];
    if (!ok) return fp_fail(c, FP_ERR_OOM, "logup_prove_rescale_hi: scratch exhausted");
    dev.A.keys = dev.K;
    dev.A.h0 = dev.h0;
    dev.A.h1 = dev.h1;
    if ((rc = lhr_protocol(c, tx, v, k, hm, dg_rem, dg_cl, dev, proof, proof_len))) return rc;
    return n_outside ? FP_WARN_KEYS_OUTSIDE_TABLE : FP_OK;
}

int fp_lhr_protocol_drive(fp_tx* tx, int v, int k, const uint32_t* m, const uint8_t* m_digests, fp_values_fn fn,
                          void* user, uint8_t* proof, size_t* proof_len) {
    if (!tx || !fn || !proof_len || !m || !m_digests) return FP_ERR_ARG;
    if (v < 1 || v > LR_MAX_V) return FP_ERR_SHAPE;
    if (k < 1 || k > 20) return FP_ERR_ARG;
    const size_t need_len = lhr_proof_len(v, k);
    if (!proof || *proof_len < need_len) {
        *proof_len = need_len;
        return FP_ERR_ARG;
    }
    LhrCallback cb;
    cb.fn = fn;
    cb.user = user;
    return lhr_protocol(nullptr, tx, v, k, (const uint8_t*)m, m_digests, m_digests + 32, cb, proof, proof_len);
}
