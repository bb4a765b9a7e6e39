// The helper-inverse LogUp on the remainder table R_k.
//
// "Towards Proving Frontier-Scale LLM Inference", The proof system: lookups use
// LogUp (Haboeck 2022), whose key side is a committed column of inverses checked
// by one sum-check; the GKR form ("How fast can FlashProve go", 4 Tighter
// Rooflines) builds a fraction tree instead and proves every level. For the
// remainder table R_k = {j - 2^(k-1) : j < 2^k} and one key column r (int32,
// n keys, padded to 2^v, v >= 1, with the key 0):
//   absorb "lhi_site" D(r); send m_j = #{keys = j - 2^(k-1)} (2^k u32; the
//   digest of their bytes is absorbed, "lhi_m"); squeeze alpha ("lhi_alpha");
//   commit h_i = 1 / (alpha - r_i): absorb "lhi_h" D(h); squeeze z_1..z_v
//   ("lhi_z") and beta ("lhi_beta"); send S = sum_i h_i ("lhi_sum");
//   sum-check of F(x) = h(x) + beta eq(z, x) (h(x) (alpha - f(x)) - 1) with
//   claim S: rounds g_t(0..3) ("lhi_round"), rho_t ("lhi_chal");
//   send h~(rho), f~(rho) ("lhi_final").
//
// Kernels: a histogram of the keys (shared-memory bins for 2^k <= 2^14); the
// inverses of the 2^k table rows alpha - t_j, one exponentiation each; the
// helper column as a gather from them (a key outside the table takes its own
// inverse); then every round in one resident cooperative launch, as for the
// gated product. With H_t(X) = sum_b h_t(X, b) (linear in X) and
// Q_t(X) = sum_b eq(z_>t, b) h_t(X, b) (alpha - f_t(X, b)) (quadratic), the
// device returns H_t(0), H_t(1), Q_t(0), Q_t(1), Q_t(2) and the host forms
//   g_t(X) = H_t(X) + beta eq(z_<t, rho_<t) eq(z_t, X) (Q_t(X) - 1),
// since the weights eq(z_>t, b) sum to 1. Round 1's values also give
// S = H_1(0) + H_1(1), and g_1(0) + g_1(1) = S is checked like every later round.
//
// The host half (lhi_protocol) takes its device values from a source: the
// kernels here, or a caller's callback (fp_lhi_protocol_drive), so the transcript
// order and the round polynomials can be checked without a GPU.
//
// The same statement over the quadratic extension ("How fast can FlashProve go",
// 4, the note on soundness) follows the base-field kernels with 16-byte vectors
// (lhi2_*, logup_prove_helper_inverse_ext2); fp_lhi_run is the base-field
// statement from "lhi_site" on, for callers (the MoE routing proof) that reserve
// the arenas themselves.
#include <string.h>

#include <algorithm>

#include "fp_eqchunks.cuh"
#include "fp_ext2.cuh"
#include "fp_ext2_host.h"
#include "fp_internal.h"
#include "fp_reduce.cuh"
#include "fp_session.cuh"

namespace {

constexpr int LH_THREADS = 256;
constexpr int LH_MAX_V = 30;
constexpr int LH_MAX_K = 24;
constexpr int LH_SMEM_BINS = 1 << 14;  // histograms of up to 2^14 bins are kept in shared memory

__device__ __forceinline__ int64_t lh_key(const int32_t* r, int64_t n, int64_t i) { return i < n ? (int64_t)r[i] : 0; }

// m_j = #{keys = j - 2^(k-1)} over the n keys and the L - n padding keys 0; keys outside
// the table are counted in *outside only
__global__ void __launch_bounds__(1024) lhi_hist_kernel(const int32_t* __restrict__ r, int64_t n, int64_t L, int k,
                                                        uint32_t* __restrict__ m, uint32_t* __restrict__ outside,
                                                        int in_smem) {
    extern __shared__ uint32_t bins[];
    const int64_t T = 1ll << k, half = 1ll << (k - 1);
    if (in_smem)
        for (int64_t i = threadIdx.x; i < T; i += blockDim.x) bins[i] = 0;
    __syncthreads();
    uint32_t out_local = 0;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t j = (int64_t)r[i] + half;
        if (j >= 0 && j < T) {
            if (in_smem)
                atomicAdd(&bins[j], 1u);
            else
                atomicAdd(&m[j], 1u);
        } else {
            out_local++;
        }
    }
    if (out_local) atomicAdd(outside, out_local);
    __syncthreads();
    if (in_smem)
        for (int64_t i = threadIdx.x; i < T; i += blockDim.x)
            if (bins[i]) atomicAdd(&m[i], bins[i]);
    if (blockIdx.x == 0 && threadIdx.x == 0 && L > n) atomicAdd(&m[half], (uint32_t)(L - n));
}

// inv[j] = 1 / (alpha - (j - 2^(k-1))) (0 where alpha is that row: the inverse of 0 is taken as 0)
__global__ void lhi_inv_kernel(uint64_t alpha, int k, uint64_t* __restrict__ inv) {
    const int64_t T = 1ll << k, half = 1ll << (k - 1);
    for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < T; j += (int64_t)gridDim.x * blockDim.x)
        inv[j] = gl_inv(gl_sub(alpha, gl_from_i64(j - half)));
}

// h_i = 1 / (alpha - key_i) for i < L: the table's inverse where the key is a row, else its own
__global__ void lhi_column_kernel(const int32_t* __restrict__ r, int64_t n, int64_t L, int k, uint64_t alpha,
                                  const uint64_t* __restrict__ inv, uint64_t* __restrict__ h) {
    const int64_t T = 1ll << k, half = 1ll << (k - 1);
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < L; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t key = lh_key(r, n, i), j = key + half;
        h[i] = (j >= 0 && j < T) ? __ldg(inv + j) : gl_inv(gl_sub(alpha, gl_from_i64(key)));
    }
}

struct LhiArgs {
    const int32_t* r;
    int64_t n;
    const uint64_t* h;  // the helper column (2^v entries)
    uint64_t* Hv;       // h and f folded, from round 2 on (2^(v-1) entries each)
    uint64_t* Fv;
    uint64_t* E;        // eq(z_>t, .) (2^(v-1) entries)
    const uint64_t* z;  // device copy of z_1..z_v
    uint64_t alpha;
    int v;
    int grid;
    int per_block;
    int pad;
    uint64_t seq0;  // round t publishes seq0 + t, the final values seq0 + v + 1
    int t_begin;    // rounds run by this launch: [t_begin, t_end]; t_end > v includes the final values
    int t_end;
};

// X = 2 on the line through (a, b) at 0 and 1
__device__ __forceinline__ uint64_t lh_at2(uint64_t a, uint64_t b) { return gl_sub(gl_add(b, b), a); }

// four blocks per SM (64 registers, no spill): 2^26 keys of R_12 1.47 -> 1.35 ms
#ifndef FP_LHI_MIN_BLOCKS
#define FP_LHI_MIN_BLOCKS 4
#endif
__global__ void __launch_bounds__(LH_THREADS, FP_LHI_MIN_BLOCKS) lhi_session_kernel(LhiArgs A, FpMailbox* mb, FpRelay* rl,
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
        GlAcc H0, H1, q0, q1, q2;
        for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < h; b += (int64_t)active * blockDim.x) {
            uint64_t h0, h1, f0, f1, e;
            if (t == 1) {
                h0 = __ldg(A.h + b);
                h1 = __ldg(A.h + b + h);
                f0 = gl_from_i64(lh_key(A.r, A.n, b));
                f1 = gl_from_i64(lh_key(A.r, A.n, b + h));
                e = eq_chunks_at(EC, eq_tab, b);  // eq(z_2..z_v, b)
                if (A.v > 1) A.E[b] = e;
            } else {
                if (t == 2) {
                    // the column and the keys (length 4h) folded by rho_1
                    h0 = gl_fold_fast(__ldg(A.h + b), __ldg(A.h + b + 2 * h), rprev);
                    h1 = gl_fold_fast(__ldg(A.h + b + h), __ldg(A.h + b + 3 * h), rprev);
                    f0 = gl_fold_fast(gl_from_i64(lh_key(A.r, A.n, b)), gl_from_i64(lh_key(A.r, A.n, b + 2 * h)),
                                      rprev);
                    f1 = gl_fold_fast(gl_from_i64(lh_key(A.r, A.n, b + h)),
                                      gl_from_i64(lh_key(A.r, A.n, b + 3 * h)), rprev);
                } else {
                    h0 = gl_fold_fast(__ldcg(A.Hv + b), __ldcg(A.Hv + b + 2 * h), rprev);
                    h1 = gl_fold_fast(__ldcg(A.Hv + b + h), __ldcg(A.Hv + b + 3 * h), rprev);
                    f0 = gl_fold_fast(__ldcg(A.Fv + b), __ldcg(A.Fv + b + 2 * h), rprev);
                    f1 = gl_fold_fast(__ldcg(A.Fv + b + h), __ldcg(A.Fv + b + 3 * h), rprev);
                }
                A.Hv[b] = h0;
                A.Hv[b + h] = h1;
                A.Fv[b] = f0;
                A.Fv[b + h] = f1;
                e = gl_add(__ldcg(A.E + b), __ldcg(A.E + b + h));  // eq(z_>t, b)
                A.E[b] = e;
            }
            H0.add(h0);
            H1.add(h1);
            q0.mac(e, gl_mul_weak(h0, gl_sub(A.alpha, f0)));
            q1.mac(e, gl_mul_weak(h1, gl_sub(A.alpha, f1)));
            q2.mac(e, gl_mul_weak(lh_at2(h0, h1), gl_sub(A.alpha, lh_at2(f0, f1))));
        }
        uint64_t acc[5] = {H0.value(), H1.value(), q0.value(), q1.value(), q2.value()};
        bool last;
        if (active == 1) {
            block_sum_gl<5>(acc);
            last = true;
        } else {
            last = grid_sum_gl_n<5>(acc, part, &rl->ticket, active);
        }
        if (last && threadIdx.x == 0) session_publish(mb, acc, A.seq0 + t);  // {H(0), H(1), Q(0), Q(1), Q(2)}
    }
    // block 0 folds the last pair by the last challenge: h~(rho), f~(rho)
    if (A.t_end <= A.v || blockIdx.x != 0) return;
    if (!session_wait(mb, rl, A.seq0 + A.v, rprev)) return;
    if (threadIdx.x == 0) {
        uint64_t h0, h1, f0, f1;
        if (A.v == 1) {
            h0 = __ldg(A.h);
            h1 = __ldg(A.h + 1);
            f0 = gl_from_i64(lh_key(A.r, A.n, 0));
            f1 = gl_from_i64(lh_key(A.r, A.n, 1));
        } else {
            h0 = __ldcg(A.Hv);
            h1 = __ldcg(A.Hv + 1);
            f0 = __ldcg(A.Fv);
            f1 = __ldcg(A.Fv + 1);
        }
        const uint64_t fin[2] = {gl_fold_fast(h0, h1, rprev), gl_fold_fast(f0, f1, rprev)};
        session_publish(mb, fin, A.seq0 + A.v + 1);
    }
}

// ---- the host half ------------------------------------------------------------

// Where the device values come from. Each call returns FP_OK or an error status.
struct LhiSource {
    virtual ~LhiSource() {}
    virtual void abandon() {}  // the host stopped early: let a waiting kernel finish
    virtual int column(uint64_t alpha, uint8_t digest[32]) = 0;      // commit h, return D(h)
    virtual int start(const uint64_t* z, int v, uint64_t beta) = 0;  // the point is known
    virtual int round(int t, uint64_t vals[5]) = 0;                  // H(0), H(1), Q(0), Q(1), Q(2)
    virtual int answer(int t, uint64_t rho) = 0;                     // the challenge rho_t
    virtual int finals(uint64_t fin[2]) = 0;                         // h~(rho), f~(rho)
};

// The protocol after "lhi_site" is absorbed, from the multiplicities on: proof of
// 4 2^k + 8 + 32 v + 16 bytes.
int lhi_protocol(fp_ctx* c, fp_tx* tx, int v, int k, const uint32_t* m, const uint8_t m_digest[32],
                 LhiSource& src, uint8_t* proof, size_t* proof_len) {
    int rc;
    size_t pos = 0;
    const size_t T = (size_t)1 << k;
    for (size_t j = 0; j < T; j++)
        for (int b = 0; b < 4; b++) proof[4 * j + b] = (uint8_t)(m[j] >> (8 * b));
    pos += 4 * T;
    fp_tx_absorb_raw(tx, "lhi_m", m_digest, 32);
    const uint64_t alpha = fp_tx_squeeze_one(tx, "lhi_alpha");
    {
        uint8_t hd[32];
        if ((rc = src.column(alpha, hd))) return rc;
        fp_tx_absorb_raw(tx, "lhi_h", hd, 32);
    }
    uint64_t z[LH_MAX_V];
    for (int i = 0; i < v; i++) z[i] = fp_tx_squeeze_one(tx, "lhi_z");
    const uint64_t beta = fp_tx_squeeze_one(tx, "lhi_beta");
    if ((rc = src.start(z, v, beta))) return rc;
    uint64_t claim = 0, pre = 1;  // pre = eq(z_<t, rho_<t)
    for (int t = 1; t <= v; t++) {
        uint64_t w[5];
        if ((rc = src.round(t, w))) return rc;
        if (t == 1) {
            claim = gl_add(w[0], w[1]);  // S = sum of h over the whole cube
            put_u64s(proof + pos, &claim, 1);
            fp_tx_absorb_raw(tx, "lhi_sum", proof + pos, 8);
            pos += 8;
        }
        const uint64_t zt = z[t - 1], scale = gl_mul(beta, pre);
        const uint64_t H[4] = {w[0], w[1], gl_sub(gl_add(w[1], w[1]), w[0]),
                               gl_sub(gl_mul(3, w[1]), gl_add(w[0], w[0]))};
        const uint64_t Q[4] = {w[2], w[3], w[4], gl_add(gl_sub(w[2], gl_mul(3, w[3])), gl_mul(3, w[4]))};
        const uint64_t eqX[4] = {gl_sub(1, zt), zt, gl_sub(gl_mul(3, zt), 1), gl_sub(gl_mul(5, zt), 2)};
        uint64_t g[4];
        for (int X = 0; X < 4; X++) g[X] = gl_add(H[X], gl_mul(scale, gl_mul(eqX[X], gl_sub(Q[X], 1))));
        if (gl_add(g[0], g[1]) != claim) {
            src.abandon();
            return fp_fail(c, FP_ERR_CUDA, "logup_prove_helper_inverse: round values inconsistent with the claim");
        }
        put_u64s(proof + pos, g, 4);
        fp_tx_absorb_raw(tx, "lhi_round", proof + pos, 32);
        pos += 32;
        const uint64_t r = fp_tx_squeeze_one(tx, "lhi_chal");
        if ((rc = src.answer(t, r))) return rc;
        claim = fp_lagrange4(g, r);
        pre = gl_mul(pre, gl_add(gl_mul(zt, r), gl_mul(gl_sub(1, zt), gl_sub(1, r))));
    }
    uint64_t fin[2];
    if ((rc = src.finals(fin))) return rc;
    put_u64s(proof + pos, fin, 2);
    fp_tx_absorb_raw(tx, "lhi_final", proof + pos, 16);
    pos += 16;
    *proof_len = pos;
    return FP_OK;
}

// Device values from the kernels above.
struct LhiDevice : LhiSource {
    fp_ctx* c;
    cudaStream_t st;
    const int32_t* r;
    int64_t n;
    int k;
    int v;
    uint64_t* hcol = nullptr;
    uint64_t* inv = nullptr;
    uint64_t* part = nullptr;
    uint64_t* small = nullptr;  // device: [8 .. 8 + v) z
    uint64_t* hs = nullptr;     // pinned host staging
    LhiArgs A;
    int cap_grid = 1;

    int launch(int t_begin, int t_end, unsigned grid, int kernel, double bytes) {
        A.t_begin = t_begin;
        A.t_end = t_end;
        void* args[] = {&A, &c->mb_dev, &c->relay, &part};
        int slot;
        fp_tic(c, st, kernel, bytes, &slot);
        FP_CUDA(c, cudaLaunchCooperativeKernel((const void*)lhi_session_kernel, dim3(grid), dim3(LH_THREADS), args,
                                               0, st));
        fp_toc(c, st, slot);
        return FP_OK;
    }

    double round_bytes(int t) const {
        const double pairs = (double)(1ll << (v - t));
        // round 1: two column and two key reads and one E write per pair; round 2: four
        // column and four key reads, two E reads, four folded writes and one E write; later
        // rounds read eight folded values instead
        return t == 1 ? 32.0 * pairs : (t == 2 ? 104.0 * pairs : 120.0 * pairs);
    }

    void abandon() override { fp_session_abandon(c, st); }

    int column(uint64_t alpha, uint8_t digest[32]) override {
        const int64_t L = 1ll << v, T = 1ll << k;
        int slot;
        fp_tic(c, st, K_LHI_COLUMN, 8.0 * (double)T + 12.0 * (double)L, &slot);
        lhi_inv_kernel<<<fp_grid256(c, T), 256, 0, st>>>(alpha, k, inv);
        lhi_column_kernel<<<fp_grid256(c, L), 256, 0, st>>>(r, n, L, k, alpha, inv, hcol);
        fp_toc(c, st, slot);
        FP_CUDA(c, cudaGetLastError());
        c->launches++;  // two kernels under one timing slot
        FpDigestJob job = {(const uint8_t*)hcol, 8 * (uint64_t)L};
        A.alpha = alpha;
        return fp_digest_many(c, &job, 1, digest, st);  // synchronises the stream
    }

    int start(const uint64_t* z, int vv, uint64_t beta) override {
        (void)beta;  // the host alone applies beta
        int rc;
        for (int i = 0; i < vv; i++) hs[8 + i] = z[i];
        FP_CUDA(c, cudaMemcpyAsync(small + 8, hs + 8, 8 * (size_t)vv, cudaMemcpyHostToDevice, st));
        A.z = small + 8;
        A.v = vv;
        A.per_block = LH_THREADS;  // one pair per thread
        const int64_t half = 1ll << (vv - 1);
        A.grid = (int)std::max<int64_t>(1, std::min<int64_t>((half + A.per_block - 1) / A.per_block, cap_grid));
        A.seq0 = fp_seq_reserve(c, (uint64_t)vv + 2);
        if ((rc = fp_session_begin(c, st))) return rc;
        fp_session_expect(c, 5);  // before any launch: round 1 publishes without a challenge
        if (!c->stepped) {
            double bytes = 0;
            for (int t = 1; t <= vv; t++) bytes += round_bytes(t);
            return launch(1, vv + 1, (unsigned)A.grid, K_LHI_ROUND, bytes);
        }
        return FP_OK;
    }

    int round(int t, uint64_t vals[5]) override {
        int rc;
        if (c->stepped && (rc = launch(t, t, (unsigned)A.grid, K_LHI_ROUND, round_bytes(t)))) return rc;
        if ((rc = fp_session_wait(c, A.seq0 + t, st))) return rc;
        for (int i = 0; i < 5; i++) vals[i] = c->mb->res[i];
        return FP_OK;
    }

    int answer(int t, uint64_t rho) override {
        fp_session_expect(c, t < v ? 5 : 2);  // the last challenge triggers the final values
        fp_session_post(c, A.seq0 + t, rho);
        return FP_OK;
    }

    int finals(uint64_t fin[2]) override {
        int rc;
        if (c->stepped && (rc = launch(v + 1, v + 1, 1, K_LHI_FINAL, 32.0))) return rc;
        if ((rc = fp_session_wait(c, A.seq0 + v + 1, st))) return rc;
        fin[0] = c->mb->res[0];
        fin[1] = c->mb->res[1];
        FP_CUDA(c, cudaStreamSynchronize(st));
        return FP_OK;
    }
};

// Device values from a caller's callback (no device).
struct LhiCallback : LhiSource {
    fp_values_fn fn;
    void* user;
    int call(int kind, int t, const uint64_t* in, uint64_t* out) { return fn(user, kind, t, in, out) ? FP_ERR_ARG : FP_OK; }
    int column(uint64_t alpha, uint8_t digest[32]) override {
        uint64_t out[4] = {0, 0, 0, 0};
        const int rc = call(FP_VAL_COLUMN, 0, &alpha, out);
        for (int i = 0; i < 4; i++)
            for (int b = 0; b < 8; b++) digest[8 * i + b] = (uint8_t)(out[i] >> (8 * b));
        return rc;
    }
    int start(const uint64_t* z, int v, uint64_t beta) override {
        uint64_t in[LH_MAX_V + 1];
        for (int i = 0; i < v; i++) in[i] = z[i];
        in[v] = beta;
        return call(FP_VAL_START, v, in, nullptr);
    }
    int round(int t, uint64_t vals[5]) override {
        for (int i = 0; i < 5; i++) vals[i] = 0;
        const int rc = call(FP_VAL_ROUND, t, nullptr, vals);
        for (int i = 0; i < 5; i++) vals[i] = gl_canon(vals[i]);
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

size_t lhi_proof_len(int v, int k) { return 4 * ((size_t)1 << k) + 8 + 32 * (size_t)v + 16; }

// ---- the same statement over the extension F_p[phi]/(phi^2 - 7) ---------------------
//
// alpha, z, beta and every challenge are extension elements, the helper column
// holds the extension inverses 1 / (alpha - r_i) = (a - b phi) / (a^2 - 7 b^2)
// (16 bytes each), and every value sent is an extension element; the labels
// are "lhi2_*". The kernels are the base-field ones with 16-byte vectors: the
// eq weights of round 1 come from four 2^8-entry chunk tables in shared memory,
// and the device returns H(0), H(1), Q(0), Q(1), Q(2) as ten words.

constexpr int LH2_CHUNK = 8;

// 1 / x in the extension (0 for 0)
__device__ __forceinline__ Ext2 e2_inv_dev(Ext2 x) {
    const uint64_t ni = gl_inv(gl_sub(gl_mul(x.a, x.a), gl_mul7(gl_mul(x.b, x.b))));
    return e2_make(gl_mul(x.a, ni), gl_sub(0, gl_mul(x.b, ni)));
}

__global__ void lhi2_inv_kernel(Ext2 alpha, int k, Ext2* __restrict__ inv) {
    const int64_t T = 1ll << k, half = 1ll << (k - 1);
    for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < T; j += (int64_t)gridDim.x * blockDim.x)
        inv[j] = e2_inv_dev(e2_make(gl_sub(alpha.a, gl_from_i64(j - half)), alpha.b));
}

__global__ void lhi2_column_kernel(const int32_t* __restrict__ r, int64_t n, int64_t L, int k, Ext2 alpha,
                                   const Ext2* __restrict__ inv, Ext2* __restrict__ h) {
    const int64_t T = 1ll << k, half = 1ll << (k - 1);
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < L; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t key = lh_key(r, n, i), j = key + half;
        h[i] = (j >= 0 && j < T) ? inv[j] : e2_inv_dev(e2_make(gl_sub(alpha.a, gl_from_i64(key)), alpha.b));
    }
}

struct Lhi2Args {
    const int32_t* r;
    int64_t n;
    const Ext2* h;  // the helper column (2^v entries)
    Ext2* Hv;       // h and f folded, from round 2 on (2^(v-1) entries each)
    Ext2* Fv;
    Ext2* E;        // eq(z_>t, .) (2^(v-1) entries)
    const Ext2* z;  // device copy of z_1..z_v
    Ext2 alpha;
    int v;
    int grid;
    int per_block;
    int pad;
    uint64_t seq0;  // round t publishes seq0 + t, the final values seq0 + v + 1
    int t_begin;    // rounds run by this launch: [t_begin, t_end]; t_end > v includes the final values
    int t_end;
};

// Table j (at tab + 2^8 j): for y < 2^w[j], the product of eq(z_c, bit) over its coordinates
// (the first on y's top bit); the four tables cover z_2..z_v. Called by every thread of the block.
__device__ __forceinline__ void lh2_tables(Ext2* tab, const Ext2* zs, int v, int (&w)[4]) {
    int rest = v - 1;
#pragma unroll
    for (int j = 0; j < 4; j++) {
        w[j] = rest < LH2_CHUNK ? rest : LH2_CHUNK;
        rest -= w[j];
    }
    for (int x = threadIdx.x; x < (4 << LH2_CHUNK); x += blockDim.x) {
        const int j = x >> LH2_CHUNK, y = x & ((1 << LH2_CHUNK) - 1);
        if (y >= (1 << w[j])) continue;
        int first = 1;
        for (int q = 0; q < j; q++) first += w[q];
        Ext2 e = e2_make(1, 0);
        for (int i = 0; i < w[j]; i++) e = e2_mul(e, e2_eq1(zs[first + i], (y >> (w[j] - 1 - i)) & 1));
        tab[x] = e;
    }
    __syncthreads();
}

__device__ __forceinline__ Ext2 lh2_eq_at(const Ext2* tab, const int (&w)[4], int64_t b) {
    const int s2 = w[3], s1 = w[3] + w[2], s0 = s1 + w[1];
    Ext2 e = tab[(int)((b >> s0) & ((1 << w[0]) - 1))];
    if (w[1]) e = e2_mul(e, tab[(1 << LH2_CHUNK) + (int)((b >> s1) & ((1 << w[1]) - 1))]);
    if (w[2]) e = e2_mul(e, tab[(2 << LH2_CHUNK) + (int)((b >> s2) & ((1 << w[2]) - 1))]);
    if (w[3]) e = e2_mul(e, tab[(3 << LH2_CHUNK) + (int)(b & ((1 << w[3]) - 1))]);
    return e;
}

// ka + rho (kb - ka) for two keys (any int32)
__device__ __forceinline__ Ext2 lh2_fold_keys(int64_t ka, int64_t kb, Ext2 rho) {
    const uint64_t d = gl_from_i64(kb - ka);
    return e2_make(gl_add(gl_from_i64(ka), gl_mul(rho.a, d)), gl_mul(rho.b, d));
}

__global__ void __launch_bounds__(LH_THREADS, 2) lhi2_session_kernel(Lhi2Args A, FpMailbox* mb, FpRelay* rl,
                                                                    uint64_t* part) {
    __shared__ Ext2 zs[32];
    __shared__ Ext2 tab[4 << LH2_CHUNK];
    if (threadIdx.x < A.v) zs[threadIdx.x] = A.z[threadIdx.x];
    __syncthreads();
    Ext2 rho = e2_make(0, 0);
    for (int t = A.t_begin; t <= A.v && t <= A.t_end; t++) {
        if (t > 1) {
            uint64_t ra, rb;
            if (!session_wait2(mb, rl, A.seq0 + t - 1, ra, rb)) return;
            rho = e2_make(ra, rb);
        }
        const int64_t h = 1ll << (A.v - t);
        const int64_t want = (h + A.per_block - 1) / A.per_block;
        const unsigned active = (unsigned)(want < 1 ? 1 : (want > A.grid ? A.grid : want));
        if (blockIdx.x >= active) return;  // no pairs for this block in this or any later round
        int w[4] = {0, 0, 0, 0};
        if (t == 1) lh2_tables(tab, zs, A.v, w);
        GlAcc H0a, H0b, H1a, H1b;
        E2Acc q0, q1, q2;
        for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < h; b += (int64_t)active * blockDim.x) {
            Ext2 h0, h1, f0, f1, e;
            if (t == 1) {
                h0 = e2_ldcg(A.h + b);
                h1 = e2_ldcg(A.h + b + h);
                f0 = e2_make(gl_from_i64(lh_key(A.r, A.n, b)), 0);
                f1 = e2_make(gl_from_i64(lh_key(A.r, A.n, b + h)), 0);
                e = lh2_eq_at(tab, w, b);  // eq(z_2..z_v, b)
                if (A.v > 1) A.E[b] = e;
            } else {
                if (t == 2) {
                    // the column and the keys (length 4h) folded by rho_1
                    h0 = e2_fold(e2_ldcg(A.h + b), e2_ldcg(A.h + b + 2 * h), rho);
                    h1 = e2_fold(e2_ldcg(A.h + b + h), e2_ldcg(A.h + b + 3 * h), rho);
                    f0 = lh2_fold_keys(lh_key(A.r, A.n, b), lh_key(A.r, A.n, b + 2 * h), rho);
                    f1 = lh2_fold_keys(lh_key(A.r, A.n, b + h), lh_key(A.r, A.n, b + 3 * h), rho);
                } else {
                    h0 = e2_fold(e2_ldcg(A.Hv + b), e2_ldcg(A.Hv + b + 2 * h), rho);
                    h1 = e2_fold(e2_ldcg(A.Hv + b + h), e2_ldcg(A.Hv + b + 3 * h), rho);
                    f0 = e2_fold(e2_ldcg(A.Fv + b), e2_ldcg(A.Fv + b + 2 * h), rho);
                    f1 = e2_fold(e2_ldcg(A.Fv + b + h), e2_ldcg(A.Fv + b + 3 * h), rho);
                }
                A.Hv[b] = h0;
                A.Hv[b + h] = h1;
                A.Fv[b] = f0;
                A.Fv[b + h] = f1;
                e = e2_add(e2_ldcg(A.E + b), e2_ldcg(A.E + b + h));  // eq(z_>t, b)
                A.E[b] = e;
            }
            H0a.add(h0.a);
            H0b.add(h0.b);
            H1a.add(h1.a);
            H1b.add(h1.b);
            const uint64_t e7 = gl_mul7(e.b);
            q0.mac(e, e7, e2_mul(h0, e2_sub(A.alpha, f0)));
            q1.mac(e, e7, e2_mul(h1, e2_sub(A.alpha, f1)));
            q2.mac(e, e7, e2_mul(e2_at2(h0, h1), e2_sub(A.alpha, e2_at2(f0, f1))));
        }
        uint64_t acc[10] = {H0a.value(), H0b.value(), H1a.value(), H1b.value(), q0.a.value(),
                            q0.b.value(), q1.a.value(), q1.b.value(), q2.a.value(), q2.b.value()};
        bool last;
        if (active == 1) {
            block_sum_gl<10>(acc);
            last = true;
        } else {
            last = grid_sum_gl_n<10>(acc, part, &rl->ticket, active);
        }
        if (last && threadIdx.x == 0) session_publish(mb, acc, A.seq0 + t);  // {H(0), H(1), Q(0), Q(1), Q(2)}
    }
    // block 0 folds the last pair by the last challenge: h~(rho), f~(rho)
    if (A.t_end <= A.v || blockIdx.x != 0) return;
    uint64_t ra, rb;
    if (!session_wait2(mb, rl, A.seq0 + A.v, ra, rb)) return;
    rho = e2_make(ra, rb);
    if (threadIdx.x == 0) {
        Ext2 hf, ff;
        if (A.v == 1) {
            hf = e2_fold(e2_ldcg(A.h), e2_ldcg(A.h + 1), rho);
            ff = lh2_fold_keys(lh_key(A.r, A.n, 0), lh_key(A.r, A.n, 1), rho);
        } else {
            hf = e2_fold(e2_ldcg(A.Hv), e2_ldcg(A.Hv + 1), rho);
            ff = e2_fold(e2_ldcg(A.Fv), e2_ldcg(A.Fv + 1), rho);
        }
        const uint64_t fin[4] = {hf.a, hf.b, ff.a, ff.b};
        session_publish(mb, fin, A.seq0 + A.v + 1);
    }
}

struct Lhi2Source {
    virtual ~Lhi2Source() {}
    virtual void abandon() {}  // the host stopped early: let a waiting kernel finish
    virtual int column(Ext2 alpha, uint8_t digest[32]) = 0;   // commit h, return D(h)
    virtual int start(const Ext2* z, int v, Ext2 beta) = 0;   // the point is known
    virtual int round(int t, Ext2 vals[5]) = 0;               // H(0), H(1), Q(0), Q(1), Q(2)
    virtual int answer(int t, Ext2 rho) = 0;
    virtual int finals(Ext2 fin[2]) = 0;                      // h~(rho), f~(rho)
};

// The statement over the extension after "lhi2_site" is absorbed, from the multiplicities on:
// 4 2^k + 16 + 64 v + 32 proof bytes.
int lhi2_protocol(fp_ctx* c, fp_tx* tx, int v, int k, const uint32_t* m, const uint8_t m_digest[32],
                  Lhi2Source& src, uint8_t* proof, size_t* proof_len) {
    int rc;
    size_t pos = 0;
    const size_t T = (size_t)1 << k;
    for (size_t j = 0; j < T; j++)
        for (int b = 0; b < 4; b++) proof[4 * j + b] = (uint8_t)(m[j] >> (8 * b));
    pos += 4 * T;
    fp_tx_absorb_raw(tx, "lhi2_m", m_digest, 32);
    const Ext2 alpha = e2_squeeze_host(tx, "lhi2_alpha");
    {
        uint8_t hd[32];
        if ((rc = src.column(alpha, hd))) return rc;
        fp_tx_absorb_raw(tx, "lhi2_h", hd, 32);
    }
    Ext2 z[LH_MAX_V];
    for (int i = 0; i < v; i++) z[i] = e2_squeeze_host(tx, "lhi2_z");
    const Ext2 beta = e2_squeeze_host(tx, "lhi2_beta");
    if ((rc = src.start(z, v, beta))) return rc;
    const Ext2 one = e2_make(1, 0);
    Ext2 claim = e2_make(0, 0), pre = one;  // pre = eq(z_<t, rho_<t)
    for (int t = 1; t <= v; t++) {
        Ext2 w[5];
        if ((rc = src.round(t, w))) return rc;
        if (t == 1) {
            claim = e2_add(w[0], w[1]);  // S = the sum of h over the whole cube
            e2_send_host(tx, "lhi2_sum", &claim, 1, proof, pos);
        }
        const Ext2 zt = z[t - 1], scale = e2_mul(beta, pre);
        const Ext2 H[4] = {w[0], w[1], e2_at2(w[0], w[1]), e2_sub(e2_scal(w[1], 3), e2_add(w[0], w[0]))};
        const Ext2 Q[4] = {w[2], w[3], w[4], e2_add(e2_sub(w[2], e2_scal(w[3], 3)), e2_scal(w[4], 3))};
        const Ext2 eqX[4] = {e2_sub(one, zt), zt, e2_sub(e2_scal(zt, 3), one), e2_sub(e2_scal(zt, 5), e2_make(2, 0))};
        Ext2 g[4];
        for (int X = 0; X < 4; X++) g[X] = e2_add(H[X], e2_mul(scale, e2_mul(eqX[X], e2_sub(Q[X], one))));
        if (!e2_same(e2_add(g[0], g[1]), claim)) {
            src.abandon();
            return fp_fail(c, FP_ERR_CUDA, "logup_prove_helper_inverse_ext2: round values inconsistent with the claim");
        }
        e2_send_host(tx, "lhi2_round", g, 4, proof, pos);
        const Ext2 r = e2_squeeze_host(tx, "lhi2_chal");
        if ((rc = src.answer(t, r))) return rc;
        claim = e2_lagrange4(g, r);
        pre = e2_mul(pre, e2_eq(zt, r));
    }
    Ext2 fin[2];
    if ((rc = src.finals(fin))) return rc;
    e2_send_host(tx, "lhi2_final", fin, 2, proof, pos);
    *proof_len = pos;
    return FP_OK;
}

struct Lhi2Device : Lhi2Source {
    fp_ctx* c;
    cudaStream_t st;
    const int32_t* r;
    int64_t n;
    int k;
    int v;
    Ext2* hcol = nullptr;
    Ext2* inv = nullptr;
    uint64_t* part = nullptr;
    uint64_t* small = nullptr;  // device: [8 .. 8 + 2 v) z
    uint64_t* hs = nullptr;
    Lhi2Args A;
    int cap_grid = 1;

    void abandon() override { fp_session_abandon(c, st); }

    int launch(int t_begin, int t_end, unsigned grid, int kernel, double bytes) {
        A.t_begin = t_begin;
        A.t_end = t_end;
        void* args[] = {&A, &c->mb_dev, &c->relay, &part};
        int slot;
        fp_tic(c, st, kernel, bytes, &slot);
        FP_CUDA(c, cudaLaunchCooperativeKernel((const void*)lhi2_session_kernel, dim3(grid), dim3(LH_THREADS), args,
                                               0, st));
        fp_toc(c, st, slot);
        return FP_OK;
    }

    double round_bytes(int t) const {
        const double pairs = (double)(1ll << (v - t));
        // round 1: two 16-byte column reads, two key reads and one E write per pair; round 2:
        // four column and four key reads, two E reads, four folded writes, one E write; later
        // rounds read eight folded values instead
        return t == 1 ? 56.0 * pairs : (t == 2 ? 176.0 * pairs : 240.0 * pairs);
    }

    int column(Ext2 alpha, uint8_t digest[32]) override {
        const int64_t L = 1ll << v, T = 1ll << k;
        int slot;
        fp_tic(c, st, K_LHI2_COLUMN, 16.0 * (double)T + 20.0 * (double)L, &slot);
        lhi2_inv_kernel<<<fp_grid256(c, T), 256, 0, st>>>(alpha, k, inv);
        lhi2_column_kernel<<<fp_grid256(c, L), 256, 0, st>>>(r, n, L, k, alpha, inv, hcol);
        fp_toc(c, st, slot);
        FP_CUDA(c, cudaGetLastError());
        c->launches++;  // two kernels under one timing slot
        A.alpha = alpha;
        FpDigestJob job = {(const uint8_t*)hcol, 16 * (uint64_t)L};
        return fp_digest_many(c, &job, 1, digest, st);  // synchronises the stream
    }

    int start(const Ext2* z, int vv, Ext2 beta) override {
        (void)beta;  // the host alone applies beta
        int rc;
        for (int i = 0; i < vv; i++) {
            hs[8 + 2 * i] = z[i].a;
            hs[9 + 2 * i] = z[i].b;
        }
        FP_CUDA(c, cudaMemcpyAsync(small + 8, hs + 8, 16 * (size_t)vv, cudaMemcpyHostToDevice, st));
        A.z = (const Ext2*)(small + 8);
        A.v = vv;
        A.per_block = LH_THREADS;  // one pair per thread
        const int64_t half = 1ll << (vv - 1);
        A.grid = (int)std::max<int64_t>(1, std::min<int64_t>((half + A.per_block - 1) / A.per_block, cap_grid));
        A.seq0 = fp_seq_reserve(c, (uint64_t)vv + 2);
        if ((rc = fp_session_begin(c, st))) return rc;
        fp_session_expect(c, 10);  // before any launch: round 1 publishes without a challenge
        if (!c->stepped) {
            double bytes = 0;
            for (int t = 1; t <= vv; t++) bytes += round_bytes(t);
            return launch(1, vv + 1, (unsigned)A.grid, K_LHI2_ROUND, bytes);
        }
        return FP_OK;
    }

    int round(int t, Ext2 vals[5]) override {
        int rc;
        if (c->stepped && (rc = launch(t, t, (unsigned)A.grid, K_LHI2_ROUND, round_bytes(t)))) return rc;
        if ((rc = fp_session_wait(c, A.seq0 + t, st))) return rc;
        for (int i = 0; i < 5; i++) vals[i] = e2_make(c->mb->res[2 * i], c->mb->res[2 * i + 1]);
        return FP_OK;
    }

    int answer(int t, Ext2 rho) override {
        fp_session_expect(c, t < v ? 10 : 4);  // the last challenge triggers the final values
        fp_session_post2(c, A.seq0 + t, rho.a, rho.b);
        return FP_OK;
    }

    int finals(Ext2 fin[2]) override {
        int rc;
        if (c->stepped && (rc = launch(v + 1, v + 1, 1, K_LHI2_FINAL, 64.0))) return rc;
        if ((rc = fp_session_wait(c, A.seq0 + v + 1, st))) return rc;
        fin[0] = e2_make(c->mb->res[0], c->mb->res[1]);
        fin[1] = e2_make(c->mb->res[2], c->mb->res[3]);
        FP_CUDA(c, cudaStreamSynchronize(st));
        return FP_OK;
    }
};

struct Lhi2Callback : Lhi2Source {
    fp_values_fn fn;
    void* user;
    int call(int kind, int t, const uint64_t* in, uint64_t* out) { return fn(user, kind, t, in, out) ? FP_ERR_ARG : FP_OK; }
    static Ext2 ext(const uint64_t* w) { return e2_make(gl_canon(w[0]), gl_canon(w[1])); }
    int column(Ext2 alpha, uint8_t digest[32]) override {
        const uint64_t in[2] = {alpha.a, alpha.b};
        uint64_t out[4] = {0, 0, 0, 0};
        const int rc = call(FP_VAL_COLUMN, 0, in, out);
        for (int i = 0; i < 4; i++)
            for (int b = 0; b < 8; b++) digest[8 * i + b] = (uint8_t)(out[i] >> (8 * b));
        return rc;
    }
    int start(const Ext2* z, int v, Ext2 beta) override {
        uint64_t in[2 * LH_MAX_V + 2];
        for (int i = 0; i < v; i++) {
            in[2 * i] = z[i].a;
            in[2 * i + 1] = z[i].b;
        }
        in[2 * v] = beta.a;
        in[2 * v + 1] = beta.b;
        return call(FP_VAL_START, v, in, nullptr);
    }
    int round(int t, Ext2 vals[5]) override {
        uint64_t out[10] = {0};
        const int rc = call(FP_VAL_ROUND, t, nullptr, out);
        for (int i = 0; i < 5; i++) vals[i] = ext(out + 2 * i);
        return rc;
    }
    int answer(int t, Ext2 rho) override {
        const uint64_t in[2] = {rho.a, rho.b};
        return call(FP_VAL_ANSWER, t, in, nullptr);
    }
    int finals(Ext2 fin[2]) override {
        uint64_t out[4] = {0, 0, 0, 0};
        const int rc = call(FP_VAL_FINALS, 0, nullptr, out);
        fin[0] = ext(out);
        fin[1] = ext(out + 2);
        return rc;
    }
};

size_t lhi2_proof_len(int v, int k) { return 4 * ((size_t)1 << k) + 16 + 64 * (size_t)v + 32; }

}  // namespace

size_t fp_lhi_proof_len(int64_t n, int k) { return lhi_proof_len(std::max(1, fp_log2_ceil((uint64_t)n)), k); }

size_t fp_lhi_scratch(fp_ctx* c, int64_t n, int k, size_t* host_bytes) {
    const int v = std::max(1, fp_log2_ceil((uint64_t)n));
    const int64_t L = 1ll << v, T = 1ll << k, half = L / 2;
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, lhi_session_kernel, LH_THREADS, 0) != cudaSuccess) occ = 2;
    const size_t part_n = (size_t)5 * std::max(1, occ) * c->num_sms;
    if (host_bytes) *host_bytes = fp_align_up((size_t)4 * T, 256) + fp_align_up(8 * 64, 256);
    return fp_align_up((size_t)8 * L, 256) + 3 * fp_align_up((size_t)8 * half, 256) + fp_align_up((size_t)8 * T, 256) +
           fp_align_up((size_t)4 * T, 256) + fp_align_up(8 * part_n, 256) + 2 * fp_align_up(8 * 64, 256);
}

int fp_lhi_run(fp_ctx* c, fp_tx* tx, const int32_t* r, int64_t n, int k, uint8_t* proof, size_t* proof_len,
               cudaStream_t st) {
    int rc;
    {
        FpDigestJob job = {(const uint8_t*)r, 4 * (uint64_t)n};
        uint8_t d[32];
        if ((rc = fp_digest_many(c, &job, 1, d, st))) return rc;  // synchronises the stream
        fp_tx_absorb_raw(tx, "lhi_site", d, 32);
    }
    const int v = std::max(1, fp_log2_ceil((uint64_t)n));
    const int64_t L = 1ll << v, T = 1ll << k, half = L / 2;
    LhiDevice dev;
    dev.c = c;
    dev.st = st;
    dev.r = r;
    dev.n = n;
    dev.k = k;
    dev.v = v;
    int occ = 0;
    FP_CUDA(c, cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, lhi_session_kernel, LH_THREADS, 0));
    dev.cap_grid = std::max(1, occ) * c->num_sms;
    const size_t part_n = (size_t)5 * dev.cap_grid;
    dev.hcol = (uint64_t*)fp_alloc(c->dev, (size_t)8 * L);
    uint64_t* Hv = (uint64_t*)fp_alloc(c->dev, (size_t)8 * half);
    uint64_t* Fv = (uint64_t*)fp_alloc(c->dev, (size_t)8 * half);
    uint64_t* E = (uint64_t*)fp_alloc(c->dev, (size_t)8 * half);
    dev.inv = (uint64_t*)fp_alloc(c->dev, (size_t)8 * T);
    uint32_t* m = (uint32_t*)fp_alloc(c->dev, (size_t)4 * T);
    dev.part = (uint64_t*)fp_alloc(c->dev, 8 * part_n);
    dev.small = (uint64_t*)fp_alloc(c->dev, 8 * 64);
    uint32_t* outside = (uint32_t*)fp_alloc(c->dev, 8 * 64);
    uint32_t* hm = (uint32_t*)fp_alloc(c->host, (size_t)4 * T);
    dev.hs = (uint64_t*)fp_alloc(c->host, 8 * 64);
    if (!dev.hcol || !Hv || !Fv || !E || !dev.inv || !m || !dev.part || !dev.small || !outside || !hm || !dev.hs)
        return fp_fail(c, FP_ERR_OOM, "helper-inverse LogUp: scratch exhausted");
    memset(&dev.A, 0, sizeof dev.A);
    dev.A.r = r;
    dev.A.n = n;
    dev.A.h = dev.hcol;
    dev.A.Hv = Hv;
    dev.A.Fv = Fv;
    dev.A.E = E;

    // ---- multiplicities ----
    FP_CUDA(c, cudaMemsetAsync(m, 0, (size_t)4 * T, st));
    FP_CUDA(c, cudaMemsetAsync(outside, 0, 4, st));
    {
        const int in_smem = T <= LH_SMEM_BINS;
        const int smem = in_smem ? 4 * (int)T : 0;
        if (smem > 48 * 1024)
            FP_CUDA(c, cudaFuncSetAttribute(lhi_hist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
        int slot;
        fp_tic(c, st, K_LHI_HIST, 4.0 * (double)n + 4.0 * (double)T, &slot);
        lhi_hist_kernel<<<c->num_sms, 1024, smem, st>>>(r, n, L, k, m, outside, in_smem);
        fp_toc(c, st, slot);
        FP_CUDA(c, cudaGetLastError());
    }
    FP_CUDA(c, cudaMemcpyAsync(hm, m, (size_t)4 * T, cudaMemcpyDeviceToHost, st));
    FP_CUDA(c, cudaMemcpyAsync(dev.hs, outside, 4, cudaMemcpyDeviceToHost, st));
    uint8_t md[32];
    {
        FpDigestJob job = {(const uint8_t*)m, 4 * (uint64_t)T};
        if ((rc = fp_digest_many(c, &job, 1, md, st))) return rc;  // synchronises the stream
    }
    uint32_t n_outside;
    memcpy(&n_outside, dev.hs, 4);
    if ((rc = lhi_protocol(c, tx, v, k, hm, md, dev, proof, proof_len))) return rc;
    return n_outside ? 1 : FP_OK;
}

int logup_prove_helper_inverse(fp_ctx* c, fp_tx* tx, const int32_t* r, int64_t n, int k, uint8_t* proof,
                               size_t* proof_len, void* stream) {
    if (!c || !tx || !proof_len || !r) return fp_fail(c, FP_ERR_ARG, "logup_prove_helper_inverse: null argument");
    if (k < 1 || k > LH_MAX_K) return fp_fail(c, FP_ERR_ARG, "logup_prove_helper_inverse: need 1 <= k <= 24");
    if (n < 1 || n > (1ll << LH_MAX_V))
        return fp_fail(c, FP_ERR_SHAPE, "logup_prove_helper_inverse: need 1 <= n <= 2^30");
    const size_t need_len = fp_lhi_proof_len(n, k);
    if (!proof || *proof_len < need_len) {
        *proof_len = need_len;
        return fp_fail(c, FP_ERR_ARG, "logup_prove_helper_inverse: proof buffer too small");
    }
    FP_CUDA(c, cudaSetDevice(c->device));
    cudaStream_t st = (cudaStream_t)stream;
    int rc;
    size_t hb = 0;
    const size_t need = fp_lhi_scratch(c, n, k, &hb) + 4096;
    if ((rc = fp_reserve(c, c->dev, need))) return rc;
    if ((rc = fp_reserve(c, c->host, hb + 4096))) return rc;
    fp_reset(c->dev);
    fp_reset(c->host);
    return fp_lhi_run(c, tx, r, n, k, proof, proof_len, st);
}

int fp_lhi_protocol_drive(fp_tx* tx, int v, int k, const uint32_t* m, const uint8_t* m_digest, fp_values_fn fn,
                          void* user, uint8_t* proof, size_t* proof_len) {
    if (!tx || !fn || !proof_len || !m || !m_digest) return FP_ERR_ARG;
    if (v < 1 || v > LH_MAX_V) return FP_ERR_SHAPE;
    if (k < 1 || k > LH_MAX_K) return FP_ERR_ARG;
    const size_t need_len = lhi_proof_len(v, k);
    if (!proof || *proof_len < need_len) {
        *proof_len = need_len;
        return FP_ERR_ARG;
    }
    LhiCallback cb;
    cb.fn = fn;
    cb.user = user;
    return lhi_protocol(nullptr, tx, v, k, m, m_digest, cb, proof, proof_len);
}

int logup_prove_helper_inverse_ext2(fp_ctx* c, fp_tx* tx, const int32_t* r, int64_t n, int k, uint8_t* proof,
                                    size_t* proof_len, void* stream) {
    if (!c || !tx || !proof_len || !r)
        return fp_fail(c, FP_ERR_ARG, "logup_prove_helper_inverse_ext2: null argument");
    if (k < 1 || k > LH_MAX_K) return fp_fail(c, FP_ERR_ARG, "logup_prove_helper_inverse_ext2: need 1 <= k <= 24");
    if (n < 1 || n > (1ll << LH_MAX_V))
        return fp_fail(c, FP_ERR_SHAPE, "logup_prove_helper_inverse_ext2: need 1 <= n <= 2^30");
    const int v = std::max(1, fp_log2_ceil((uint64_t)n));
    const size_t need_len = lhi2_proof_len(v, k);
    if (!proof || *proof_len < need_len) {
        *proof_len = need_len;
        return fp_fail(c, FP_ERR_ARG, "logup_prove_helper_inverse_ext2: proof buffer too small");
    }
    FP_CUDA(c, cudaSetDevice(c->device));
    cudaStream_t st = (cudaStream_t)stream;
    int rc;
    {
        FpDigestJob job = {(const uint8_t*)r, 4 * (uint64_t)n};
        uint8_t d[32];
        if ((rc = fp_digest_many(c, &job, 1, d, st))) return rc;  // synchronises the stream
        fp_tx_absorb_raw(tx, "lhi2_site", d, 32);
    }
    const int64_t L = 1ll << v, T = 1ll << k, half = L / 2;
    Lhi2Device dev;
    dev.c = c;
    dev.st = st;
    dev.r = r;
    dev.n = n;
    dev.k = k;
    dev.v = v;
    int occ = 0;
    FP_CUDA(c, cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, lhi2_session_kernel, LH_THREADS, 0));
    dev.cap_grid = std::max(1, occ) * c->num_sms;
    const size_t part_n = (size_t)10 * dev.cap_grid;
    const size_t need = fp_align_up((size_t)16 * L, 256) + 3 * fp_align_up((size_t)16 * half, 256) +
                        fp_align_up((size_t)16 * T, 256) + fp_align_up((size_t)4 * T, 256) +
                        fp_align_up(8 * part_n, 256) + 2 * fp_align_up(8 * 128, 256) + 4096;
    if ((rc = fp_reserve(c, c->dev, need))) return rc;
    if ((rc = fp_reserve(c, c->host, fp_align_up((size_t)4 * T, 256) + fp_align_up(8 * 128, 256) + 4096))) return rc;
    fp_reset(c->dev);
    fp_reset(c->host);
    dev.hcol = (Ext2*)fp_alloc(c->dev, (size_t)16 * L);
    Ext2* Hv = (Ext2*)fp_alloc(c->dev, (size_t)16 * half);
    Ext2* Fv = (Ext2*)fp_alloc(c->dev, (size_t)16 * half);
    Ext2* E = (Ext2*)fp_alloc(c->dev, (size_t)16 * half);
    dev.inv = (Ext2*)fp_alloc(c->dev, (size_t)16 * T);
    uint32_t* m = (uint32_t*)fp_alloc(c->dev, (size_t)4 * T);
    dev.part = (uint64_t*)fp_alloc(c->dev, 8 * part_n);
    dev.small = (uint64_t*)fp_alloc(c->dev, 8 * 128);
    uint32_t* outside = (uint32_t*)fp_alloc(c->dev, 8 * 128);
    uint32_t* hm = (uint32_t*)fp_alloc(c->host, (size_t)4 * T);
    dev.hs = (uint64_t*)fp_alloc(c->host, 8 * 128);
    if (!dev.hcol || !Hv || !Fv || !E || !dev.inv || !m || !dev.part || !dev.small || !outside || !hm || !dev.hs)
        return fp_fail(c, FP_ERR_OOM, "logup_prove_helper_inverse_ext2: scratch exhausted");
    memset(&dev.A, 0, sizeof dev.A);
    dev.A.r = r;
    dev.A.n = n;
    dev.A.h = dev.hcol;
    dev.A.Hv = Hv;
    dev.A.Fv = Fv;
    dev.A.E = E;
    FP_CUDA(c, cudaMemsetAsync(m, 0, (size_t)4 * T, st));
    FP_CUDA(c, cudaMemsetAsync(outside, 0, 4, st));
    {
        const int in_smem = T <= LH_SMEM_BINS;
        const int smem = in_smem ? 4 * (int)T : 0;
        if (smem > 48 * 1024)
            FP_CUDA(c, cudaFuncSetAttribute(lhi_hist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
        int slot;
        fp_tic(c, st, K_LHI_HIST, 4.0 * (double)n + 4.0 * (double)T, &slot);
        lhi_hist_kernel<<<c->num_sms, 1024, smem, st>>>(r, n, L, k, m, outside, in_smem);
        fp_toc(c, st, slot);
        FP_CUDA(c, cudaGetLastError());
    }
    FP_CUDA(c, cudaMemcpyAsync(hm, m, (size_t)4 * T, cudaMemcpyDeviceToHost, st));
    FP_CUDA(c, cudaMemcpyAsync(dev.hs, outside, 4, cudaMemcpyDeviceToHost, st));
    uint8_t md[32];
    {
        FpDigestJob job = {(const uint8_t*)m, 4 * (uint64_t)T};
        if ((rc = fp_digest_many(c, &job, 1, md, st))) return rc;  // synchronises the stream
    }
    uint32_t n_outside;
    memcpy(&n_outside, dev.hs, 4);
    if ((rc = lhi2_protocol(c, tx, v, k, hm, md, dev, proof, proof_len))) return rc;
    return n_outside ? 1 : FP_OK;
}

int fp_lhi2_protocol_drive(fp_tx* tx, int v, int k, const uint32_t* m, const uint8_t* m_digest, fp_values_fn fn,
                           void* user, uint8_t* proof, size_t* proof_len) {
    if (!tx || !fn || !proof_len || !m || !m_digest) return FP_ERR_ARG;
    if (v < 1 || v > LH_MAX_V) return FP_ERR_SHAPE;
    if (k < 1 || k > LH_MAX_K) return FP_ERR_ARG;
    const size_t need_len = lhi2_proof_len(v, k);
    if (!proof || *proof_len < need_len) {
        *proof_len = need_len;
        return FP_ERR_ARG;
    }
    Lhi2Callback cb;
    cb.fn = fn;
    cb.user = user;
    return lhi2_protocol(nullptr, tx, v, k, m, m_digest, cb, proof, proof_len);
}
