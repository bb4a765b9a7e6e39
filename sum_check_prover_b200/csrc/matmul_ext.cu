// The matmul sum-check of one site with challenges in the quadratic extension.
//
// "How fast can FlashProve go", 2 Background (sum-check reduces the matmul
// Y = W X to claims on the committed operands), 3.1 (Y enters as 2^k q + r)
// and 4 (the note on soundness: challenges from an extension field). The
// statement of sumcheck_prove_matmul for one site with every challenge, claim,
// round value and final value in F_p[phi]/(phi^2 - 7) (fp_ext2.cuh):
//   absorb "mm2_site" D(W) || D(S) || D(Xt) || D(q) || D(r); squeeze r_row
//   (vM coordinates, "mm2_row") and r_col (vN, "mm2_col"); send
//   c = Y~(r_row, r_col) ("mm2_claim"); n = ceil(log2 K) rounds of g(0), g(1),
//   g(2) of sum_b A(X, b) B(X, b) with A = W_eff~(r_row, .) and
//   B = X~(., r_col) ("mm2_round"), rho_t ("mm2_chal"); send A(rho), B(rho)
//   ("mm2_final").
//
// An extension point's eq weights are extension elements e_i = a_i + b_i phi and the
// matrices hold base-field integers, so each partial evaluation
// A[k] = sum_i eq(r_row, i) W_eff[i][k] (and B[k] = sum_j eq(r_col, j) Xt[j][k]) is two
// base-field row contractions, sum_i a_i W_eff[i][k] and sum_i b_i W_eff[i][k]: the
// partial evaluation's tensor-core kernel with the two coordinate vectors as its row
// weights (all four contractions of a call in one launch), then a pass pairing the
// coordinates into extension elements. The claim
// is a flat eq_row x eq_col weighted sum of 2^k q + r. The rounds run in one
// resident cooperative launch over the two length-2^n vectors, folding in place
// as the base-field matmul kernel does.
//
// The host half (mm2_protocol) takes its device values from a source: the
// kernels here, or a caller's callback (fp_mm2_protocol_drive).
#include <string.h>

#include <algorithm>
#include <vector>

#include "fp_ext2.cuh"
#include "fp_ext2_host.h"
#include "fp_internal.h"
#include "fp_reduce.cuh"
#include "fp_session.cuh"

namespace {

constexpr int M2_THREADS = 256;

// out[x] = eq(z, x) for x < 2^v, z_1 on the most significant bit
__global__ void e2_eq_kernel(const Ext2* __restrict__ z, int v, Ext2* __restrict__ out) {
    const int64_t len = 1ll << v;
    for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < len; x += (int64_t)gridDim.x * blockDim.x) {
        Ext2 e = e2_make(1, 0);
        for (int b = 0; b < v; b++) e = e2_mul(e, e2_eq1(z[b], (int)((x >> (v - 1 - b)) & 1)));
        out[x] = e;
    }
}

// c = sum over the N x M token-major witness of eq(r_col, j) eq(r_row, i) (2^k q + r)
__global__ void __launch_bounds__(M2_THREADS) mm2_claim_kernel(const int32_t* __restrict__ q,
                                                               const int32_t* __restrict__ r, int M, int64_t total,
                                                               int kshift, const Ext2* __restrict__ Erow,
                                                               const Ext2* __restrict__ Ecol, uint64_t* part,
                                                               unsigned int* ticket, uint64_t* out) {
    E2Acc acc;
    for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < total; x += (int64_t)gridDim.x * blockDim.x) {
        const int64_t y = (int64_t)q[x] * (1ll << kshift) + (int64_t)r[x];  // |y| < 2^52
        if (y == 0) continue;
        const int64_t j = x / M, i = x - j * M;
        acc.mac_base(e2_mul(Ecol[j], Erow[i]), gl_from_i64(y));
    }
    uint64_t v[2] = {acc.a.value(), acc.b.value()};
    if (grid_sum_gl<2>(v, part, ticket) && threadIdx.x == 0) {
        out[0] = v[0];
        out[1] = v[1];
    }
}

// out[k] = (a[k], b[k]): the two coordinates of the contractions paired into extension elements
__global__ void e2_pair_kernel(const uint64_t* __restrict__ a, const uint64_t* __restrict__ b, int64_t len,
                               Ext2* __restrict__ out) {
    for (int64_t k = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; k < len; k += (int64_t)gridDim.x * blockDim.x)
        out[k] = e2_make(a[k], b[k]);
}

struct Mm2Args {
    Ext2* A;  // 2^n entries each, folded in place
    Ext2* B;
    int n;
    int grid;
    int per_block;
    int pad;
    uint64_t seq0;  // round t publishes seq0 + t, the final values seq0 + n + 1
    int t_begin;    // rounds run by this launch: [t_begin, t_end]; t_end > n includes the final values
    int t_end;
};

__global__ void __launch_bounds__(M2_THREADS, 2) mm2_session_kernel(Mm2Args P, FpMailbox* mb, FpRelay* rl,
                                                                   uint64_t* part) {
    Ext2 rho = e2_make(0, 0);
    for (int t = P.t_begin; t <= P.n && t <= P.t_end; t++) {
        if (t > 1) {
            uint64_t ra, rb;
            if (!session_wait2(mb, rl, P.seq0 + t - 1, ra, rb)) return;
            rho = e2_make(ra, rb);
        }
        const int64_t h = 1ll << (P.n - t);
        const int64_t want = (h + P.per_block - 1) / P.per_block;
        const unsigned active = (unsigned)(want < 1 ? 1 : (want > P.grid ? P.grid : want));
        if (blockIdx.x >= active) return;  // no pairs for this block in this or any later round
        E2Acc c0, c1, c2;
        for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < h; b += (int64_t)active * blockDim.x) {
            Ext2 a0, a1, b0, b1;
            if (t == 1) {
                a0 = e2_ldcg(P.A + b);
                a1 = e2_ldcg(P.A + b + h);
                b0 = e2_ldcg(P.B + b);
                b1 = e2_ldcg(P.B + b + h);
            } else {
                // the vectors of length 4h folded by rho_{t-1}
                a0 = e2_fold(e2_ldcg(P.A + b), e2_ldcg(P.A + b + 2 * h), rho);
                a1 = e2_fold(e2_ldcg(P.A + b + h), e2_ldcg(P.A + b + 3 * h), rho);
                b0 = e2_fold(e2_ldcg(P.B + b), e2_ldcg(P.B + b + 2 * h), rho);
                b1 = e2_fold(e2_ldcg(P.B + b + h), e2_ldcg(P.B + b + 3 * h), rho);
                P.A[b] = a0;
                P.A[b + h] = a1;
                P.B[b] = b0;
                P.B[b + h] = b1;
            }
            c0.mac(a0, gl_mul7(a0.b), b0);
            c1.mac(a1, gl_mul7(a1.b), b1);
            const Ext2 a2 = e2_at2(a0, a1);
            c2.mac(a2, gl_mul7(a2.b), e2_at2(b0, b1));
        }
        uint64_t acc[6] = {c0.a.value(), c0.b.value(), c1.a.value(), c1.b.value(), c2.a.value(), c2.b.value()};
        bool last;
        if (active == 1) {
            block_sum_gl<6>(acc);
            last = true;
        } else {
            last = grid_sum_gl_n<6>(acc, part, &rl->ticket, active);
        }
        if (last && threadIdx.x == 0) session_publish(mb, acc, P.seq0 + t);  // {g(0), g(1), g(2)}
    }
    // block 0 folds the last pair by the last challenge: A(rho), B(rho)
    if (P.t_end <= P.n || blockIdx.x != 0) return;
    uint64_t ra, rb;
    if (!session_wait2(mb, rl, P.seq0 + P.n, ra, rb)) return;
    rho = e2_make(ra, rb);
    if (threadIdx.x == 0) {
        const Ext2 fa = e2_fold(e2_ldcg(P.A), e2_ldcg(P.A + 1), rho);
        const Ext2 fb = e2_fold(e2_ldcg(P.B), e2_ldcg(P.B + 1), rho);
        const uint64_t fin[4] = {fa.a, fa.b, fb.a, fb.b};
        session_publish(mb, fin, P.seq0 + P.n + 1);
    }
}

// ---- the host half ------------------------------------------------------------

// Where the device values come from. Each call returns FP_OK or an error status.
struct Mm2Source {
    virtual ~Mm2Source() {}
    virtual void abandon() {}  // the host stopped early: let a waiting kernel finish
    virtual int start(const Ext2* zr, int vM, const Ext2* zc, int vN) = 0;  // the point is known
    virtual int claim(Ext2& c) = 0;                                          // Y~(r_row, r_col)
    virtual int round(int t, Ext2 g[3]) = 0;                                 // g_t(0), g_t(1), g_t(2)
    virtual int answer(int t, Ext2 rho) = 0;                                 // the challenge rho_t
    virtual int finals(Ext2 fin[2]) = 0;                                     // A(rho), B(rho)
};

constexpr int M2_MAX_V = 32;

// The protocol after "mm2_site" is absorbed: proof of 16 + 48 n + 32 bytes.
int mm2_protocol(fp_ctx* c, fp_tx* tx, int vM, int vN, int n, Mm2Source& src, uint8_t* proof, size_t* proof_len) {
    Ext2 zr[M2_MAX_V] = {}, zc[M2_MAX_V] = {};
    for (int i = 0; i < vM; i++) zr[i] = e2_squeeze_host(tx, "mm2_row");
    for (int i = 0; i < vN; i++) zc[i] = e2_squeeze_host(tx, "mm2_col");
    int rc;
    if ((rc = src.start(zr, vM, zc, vN))) return rc;
    size_t pos = 0;
    Ext2 claim;
    if ((rc = src.claim(claim))) return rc;
    e2_send_host(tx, "mm2_claim", &claim, 1, proof, pos);
    for (int t = 1; t <= n; t++) {
        Ext2 g[3];
        if ((rc = src.round(t, g))) return rc;
        if (!e2_same(e2_add(g[0], g[1]), claim)) {
            src.abandon();
            return fp_fail(c, FP_ERR_CUDA, "sumcheck_prove_matmul_ext2: round values inconsistent with the claim");
        }
        e2_send_host(tx, "mm2_round", g, 3, proof, pos);
        const Ext2 r = e2_squeeze_host(tx, "mm2_chal");
        if ((rc = src.answer(t, r))) return rc;
        claim = e2_lagrange3(g, r);
    }
    Ext2 fin[2];
    if ((rc = src.finals(fin))) return rc;
    e2_send_host(tx, "mm2_final", fin, 2, proof, pos);
    *proof_len = pos;
    return FP_OK;
}

// Device values from the kernels above.
struct Mm2Device : Mm2Source {
    fp_ctx* c;
    cudaStream_t st;
    const fp_site* s;
    int n;
    Ext2* A = nullptr;
    Ext2* B = nullptr;
    Ext2* Erow = nullptr;
    Ext2* Ecol = nullptr;
    uint64_t* coord[4] = {nullptr, nullptr, nullptr, nullptr};  // A.a, A.b, B.a, B.b (2^n each)
    uint64_t* part = nullptr;   // reduction partials
    uint64_t* small = nullptr;  // device: [0..2) claim, [8..) the point
    uint64_t* hs = nullptr;     // pinned host staging
    Mm2Args P;
    int cap_grid = 1;

    // the four base-field contractions: W and Xt, each with the a and the b coordinates of its
    // eq weights (row i's weight at E[i].a or E[i].b, a stride of two words)
    std::vector<FpPeJob> jobs() const {
        const int64_t L = 1ll << n;
        std::vector<FpPeJob> j(4);
        for (int h = 0; h < 2; h++) {
            j[h] = FpPeJob{s->w, s->w_bits, s->scales, s->M, s->K, nullptr, 0, coord[h], L};
            j[h].wts = reinterpret_cast<const uint64_t*>(Erow) + h;
            j[h].wts_stride = 2;
            j[2 + h] = FpPeJob{s->xt, 8, nullptr, s->N, s->K, nullptr, 0, coord[2 + h], L};
            j[2 + h].wts = reinterpret_cast<const uint64_t*>(Ecol) + h;
            j[2 + h].wts_stride = 2;
        }
        return j;
    }

    // A and B from the four contractions, in one partial-evaluation launch per kernel variant
    int contract() {
        const int64_t L = 1ll << n;
        const double bytes = (double)s->M * (s->w_bits == 4 ? (s->K + 1) / 2 : s->K) + (double)s->N * s->K;
        int slot, rc;
        fp_tic(c, st, K_MM2_CONTRACT, bytes, &slot);
        const std::vector<FpPeJob> j = jobs();
        if ((rc = fp_partial_many(c, j.data(), 4, st))) return rc;
        e2_pair_kernel<<<fp_grid256(c, L), 256, 0, st>>>(coord[0], coord[1], L, A);
        e2_pair_kernel<<<fp_grid256(c, L), 256, 0, st>>>(coord[2], coord[3], L, B);
        fp_toc(c, st, slot);
        FP_CUDA(c, cudaGetLastError());
        c->launches++;  // the two pairing kernels under one slot (the slot counts one)
        return FP_OK;
    }

    void abandon() override { fp_session_abandon(c, st); }

    int start(const Ext2* zr, int vM, const Ext2* zc, int vN) override {
        for (int i = 0; i < vM; i++) {
            hs[8 + 2 * i] = zr[i].a;
            hs[9 + 2 * i] = zr[i].b;
        }
        for (int i = 0; i < vN; i++) {
            hs[8 + 2 * (vM + i)] = zc[i].a;
            hs[9 + 2 * (vM + i)] = zc[i].b;
        }
        FP_CUDA(c, cudaMemcpyAsync(small + 8, hs + 8, 16 * (size_t)(vM + vN), cudaMemcpyHostToDevice, st));
        const Ext2* dzr = (const Ext2*)(small + 8);
        const Ext2* dzc = dzr + vM;
        int slot;
        fp_tic(c, st, K_MM2_EQ, 16.0 * (double)((1ll << vM) + (1ll << vN)), &slot);
        e2_eq_kernel<<<fp_grid256(c, 1ll << vM), 256, 0, st>>>(dzr, vM, Erow);
        e2_eq_kernel<<<fp_grid256(c, 1ll << vN), 256, 0, st>>>(dzc, vN, Ecol);
        fp_toc(c, st, slot);
        FP_CUDA(c, cudaGetLastError());
        c->launches++;
        return contract();
    }

    int claim(Ext2& cl) override {
        const int64_t total = (int64_t)s->M * s->N;
        int slot;
        fp_tic(c, st, K_MM2_CLAIM, 8.0 * (double)total, &slot);
        mm2_claim_kernel<<<fp_grid256(c, total), M2_THREADS, 0, st>>>(s->q, s->r, s->M, total, s->k_shift, Erow, Ecol, part,
                                                                c->tickets, small);
        fp_toc(c, st, slot);
        FP_CUDA(c, cudaGetLastError());
        FP_CUDA(c, cudaMemcpyAsync(hs, small, 16, cudaMemcpyDeviceToHost, st));
        FP_CUDA(c, cudaStreamSynchronize(st));
        cl = e2_make(hs[0], hs[1]);
        if (n == 0) return FP_OK;
        int rc;
        memset(&P, 0, sizeof P);
        P.A = A;
        P.B = B;
        P.n = n;
        P.per_block = M2_THREADS;  // one pair per thread
        const int64_t half = 1ll << (n - 1);
        P.grid = (int)std::max<int64_t>(1, std::min<int64_t>((half + P.per_block - 1) / P.per_block, cap_grid));
        P.seq0 = fp_seq_reserve(c, (uint64_t)n + 2);
        if ((rc = fp_session_begin(c, st))) return rc;
        fp_session_expect(c, 6);  // before any launch: round 1 publishes without a challenge
        if (!c->stepped) {
            double bytes = 0;
            for (int t = 1; t <= n; t++) bytes += round_bytes(t);
            return launch(1, n + 1, (unsigned)P.grid, K_MM2_ROUND, bytes);
        }
        return FP_OK;
    }

    double round_bytes(int t) const {
        const double pairs = (double)(1ll << (n - t));
        // round 1 reads two 16-byte values of A and B per pair; later rounds read four and write two
        return t == 1 ? 64.0 * pairs : 192.0 * pairs;
    }

    int launch(int t_begin, int t_end, unsigned grid, int kernel, double bytes) {
        P.t_begin = t_begin;
        P.t_end = t_end;
        void* args[] = {&P, &c->mb_dev, &c->relay, &part};
        int slot;
        fp_tic(c, st, kernel, bytes, &slot);
        FP_CUDA(c, cudaLaunchCooperativeKernel((const void*)mm2_session_kernel, dim3(grid), dim3(M2_THREADS), args, 0,
                                               st));
        fp_toc(c, st, slot);
        return FP_OK;
    }

    int round(int t, Ext2 g[3]) override {
        int rc;
        if (c->stepped && (rc = launch(t, t, (unsigned)P.grid, K_MM2_ROUND, round_bytes(t)))) return rc;
        if ((rc = fp_session_wait(c, P.seq0 + t, st))) return rc;
        for (int i = 0; i < 3; i++) g[i] = e2_make(c->mb->res[2 * i], c->mb->res[2 * i + 1]);
        return FP_OK;
    }

    int answer(int t, Ext2 rho) override {
        fp_session_expect(c, t < n ? 6 : 4);  // the last challenge triggers the final values
        fp_session_post2(c, P.seq0 + t, rho.a, rho.b);
        return FP_OK;
    }

    int finals(Ext2 fin[2]) override {
        if (n == 0) {  // K = 1: the single entries
            FP_CUDA(c, cudaMemcpyAsync(hs, A, 16, cudaMemcpyDeviceToHost, st));
            FP_CUDA(c, cudaMemcpyAsync(hs + 2, B, 16, cudaMemcpyDeviceToHost, st));
            FP_CUDA(c, cudaStreamSynchronize(st));
            fin[0] = e2_make(hs[0], hs[1]);
            fin[1] = e2_make(hs[2], hs[3]);
            return FP_OK;
        }
        int rc;
        if (c->stepped && (rc = launch(n + 1, n + 1, 1, K_MM2_FINAL, 64.0))) return rc;
        if ((rc = fp_session_wait(c, P.seq0 + n + 1, st))) return rc;
        fin[0] = e2_make(c->mb->res[0], c->mb->res[1]);
        fin[1] = e2_make(c->mb->res[2], c->mb->res[3]);
        FP_CUDA(c, cudaStreamSynchronize(st));
        return FP_OK;
    }
};

// Device values from a caller's callback (no device).
struct Mm2Callback : Mm2Source {
    fp_values_fn fn;
    void* user;
    int call(int kind, int t, const uint64_t* in, uint64_t* out) { return fn(user, kind, t, in, out) ? FP_ERR_ARG : FP_OK; }
    static Ext2 ext(const uint64_t* w) { return e2_make(gl_canon(w[0]), gl_canon(w[1])); }
    int start(const Ext2* zr, int vM, const Ext2* zc, int vN) override {
        uint64_t in[4 * M2_MAX_V];
        for (int i = 0; i < vM; i++) {
            in[2 * i] = zr[i].a;
            in[2 * i + 1] = zr[i].b;
        }
        for (int i = 0; i < vN; i++) {
            in[2 * (vM + i)] = zc[i].a;
            in[2 * (vM + i) + 1] = zc[i].b;
        }
        return call(FP_VAL_START, vM + vN, in, nullptr);
    }
    int claim(Ext2& cl) override {
        uint64_t out[2] = {0, 0};
        const int rc = call(FP_VAL_CLAIM, 0, nullptr, out);
        cl = ext(out);
        return rc;
    }
    int round(int t, Ext2 g[3]) override {
        uint64_t out[6] = {0, 0, 0, 0, 0, 0};
        const int rc = call(FP_VAL_ROUND, t, nullptr, out);
        for (int i = 0; i < 3; i++) g[i] = ext(out + 2 * i);
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

size_t mm2_proof_len(int n) { return 16 + 48 * (size_t)n + 32; }

}  // namespace

int fp_site_digest160(fp_ctx* c, const fp_site& s, uint8_t d[160], cudaStream_t st) {
    const uint64_t mn = (uint64_t)s.M * s.N;
    const uint64_t wb = (uint64_t)s.M * (s.w_bits == 4 ? (uint64_t)((s.K + 1) / 2) : (uint64_t)s.K);
    const uint64_t sb = s.scales ? (uint64_t)s.M * ((s.K + 63) / 64) : 0;
    FpDigestJob jobs[5] = {{(const uint8_t*)s.w, wb},
                           {(const uint8_t*)s.scales, sb},
                           {(const uint8_t*)s.xt, (uint64_t)s.N * s.K},
                           {(const uint8_t*)s.q, 4 * mn},
                           {(const uint8_t*)s.r, 4 * mn}};
    if (s.w_digest) {
        memcpy(d, s.w_digest, 64);
        return fp_digest_many(c, jobs + 2, 3, d + 64, st);  // synchronises the stream
    }
    return fp_digest_many(c, jobs, 5, d, st);
}

int sumcheck_prove_matmul_ext2(fp_ctx* c, fp_tx* tx, const fp_site* site, uint8_t* proof, size_t* proof_len,
                               void* stream) {
    if (!c || !tx || !proof_len || !site) return fp_fail(c, FP_ERR_ARG, "sumcheck_prove_matmul_ext2: null argument");
    int rc;
    if ((rc = fp_check_sites(c, site, 1, true))) return rc;
    const fp_site& s = *site;
    const int vM = fp_log2_ceil((uint64_t)s.M), vN = fp_log2_ceil((uint64_t)s.N), n = fp_log2_ceil((uint64_t)s.K);
    const size_t need_len = mm2_proof_len(n);
    if (!proof || *proof_len < need_len) {
        *proof_len = need_len;
        return fp_fail(c, FP_ERR_ARG, "sumcheck_prove_matmul_ext2: proof buffer too small");
    }
    FP_CUDA(c, cudaSetDevice(c->device));
    cudaStream_t st = (cudaStream_t)stream;
    {
        uint8_t d[160];
        if ((rc = fp_site_digest160(c, s, d, st))) return rc;
        fp_tx_absorb_raw(tx, "mm2_site", d, 160);
    }
    Mm2Device dev;
    dev.c = c;
    dev.st = st;
    dev.s = &s;
    dev.n = n;
    int occ = 0;
    FP_CUDA(c, cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, mm2_session_kernel, M2_THREADS, 0));
    dev.cap_grid = std::max(1, occ) * c->num_sms;
    const int64_t L = 1ll << n;
    const size_t part_n = (size_t)6 * std::max(dev.cap_grid, 4 * c->num_sms);
    const std::vector<FpPeJob> pj = dev.jobs();  // shapes only, for the partial evaluation's scratch
    const size_t need = 2 * fp_align_up((size_t)16 * L, 256) + fp_align_up((size_t)16 << vM, 256) +
                        fp_align_up((size_t)16 << vN, 256) + 4 * fp_align_up((size_t)8 * L, 256) +
                        fp_partial_scratch(c, pj.data(), 4) + fp_align_up(8 * part_n, 256) +
                        fp_align_up(8 * 160, 256) + 4096;
    if ((rc = fp_reserve(c, c->dev, need))) return rc;
    if ((rc = fp_reserve(c, c->host, fp_partial_host_scratch(pj.data(), 4) + fp_align_up(8 * 160, 256) + 4096)))
        return rc;
    fp_reset(c->dev);
    fp_reset(c->host);
    dev.A = (Ext2*)fp_alloc(c->dev, (size_t)16 * L);
    dev.B = (Ext2*)fp_alloc(c->dev, (size_t)16 * L);
    dev.Erow = (Ext2*)fp_alloc(c->dev, (size_t)16 << vM);
    dev.Ecol = (Ext2*)fp_alloc(c->dev, (size_t)16 << vN);
    for (int h = 0; h < 4; h++) dev.coord[h] = (uint64_t*)fp_alloc(c->dev, (size_t)8 * L);
    dev.part = (uint64_t*)fp_alloc(c->dev, 8 * part_n);
    dev.small = (uint64_t*)fp_alloc(c->dev, 8 * 160);
    dev.hs = (uint64_t*)fp_alloc(c->host, 8 * 160);
    if (!dev.A || !dev.B || !dev.Erow || !dev.Ecol || !dev.coord[3] || !dev.part || !dev.small || !dev.hs)
        return fp_fail(c, FP_ERR_OOM, "sumcheck_prove_matmul_ext2: scratch exhausted");
    return mm2_protocol(c, tx, vM, vN, n, dev, proof, proof_len);
}

int fp_mm2_protocol_drive(fp_tx* tx, int vM, int vN, int n, fp_values_fn fn, void* user, uint8_t* proof,
                          size_t* proof_len) {
    if (!tx || !fn || !proof_len) return FP_ERR_ARG;
    if (vM < 0 || vN < 0 || vM > 24 || vN > 24 || n < 0 || n > 20) return FP_ERR_SHAPE;
    const size_t need_len = mm2_proof_len(n);
    if (!proof || *proof_len < need_len) {
        *proof_len = need_len;
        return FP_ERR_ARG;
    }
    Mm2Callback cb;
    cb.fn = fn;
    cb.user = user;
    return mm2_protocol(nullptr, tx, vM, vN, n, cb, proof, proof_len);
}
