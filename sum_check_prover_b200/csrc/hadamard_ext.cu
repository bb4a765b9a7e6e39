// The gated-product sum-check with challenges in the quadratic extension.
//
// "How fast can FlashProve go", 3.1 (the gated product h = s (.) u is proven by
// sum-check, never committed) and 4 (the note on soundness: challenges from an
// extension field). The statement is sumcheck_prove_hadamard's with every
// challenge, claim, round value and final value in F_p[phi]/(phi^2 - 7)
// (fp_ext2.cuh), an extension element sent as 16 bytes:
//   absorb "had2_site" D(s) || D(u); squeeze z_1..z_v ("had2_z", two base
//   squeezes each); send c = sum_x eq(z, x) s(x) u(x) ("had2_claim");
//   round t = 1..v: send g_t(0..3) ("had2_round"), squeeze rho_t ("had2_chal");
//   send s~(rho), u~(rho) ("had2_final").
//
// The device computes h_t(X) = sum_b eq(z_>t, b) s_t(X, b) u_t(X, b) at
// X = 0, 1, 2 (s_t, u_t the factors folded by rho_<t); the host forms
// g_t(X) = eq(z_<t, rho_<t) eq(z_t, X) h_t(X). Round 1's values need no
// challenge, so the claim is taken from them: c = g_1(0) + g_1(1). Every later
// round is checked against the running claim on the host.
//
// All rounds run in one resident cooperative launch, as in hadamard.cu: round 1
// reads the int8 factors and writes E[b] = eq(z_>1, b) from four chunk tables of
// at most 2^8 entries each (built per block in shared memory); round 2 folds the
// int8 factors by rho_1 (small differences times an extension element); later
// rounds fold the extension vectors in place. Each vector element is 16 bytes
// (a, b interleaved), read and written as one 16-byte access.
//
// The host half (had2_protocol) takes its round values from a source: the
// device session here, or a caller's callback (fp_had2_protocol_drive), so the
// transcript order and the round polynomials can be checked without a GPU.
#include <string.h>

#include <algorithm>

#include "fp_ext2.cuh"
#include "fp_ext2_host.h"
#include "fp_internal.h"
#include "fp_reduce.cuh"
#include "fp_session.cuh"

namespace {

constexpr int H2_THREADS = 256;
constexpr int H2_MAX_V = 30;
constexpr int H2_CHUNK = 8;  // four tables of at most 2^8 entries cover z_2..z_v for v <= 33

struct Had2Args {
    const int8_t* s;
    const int8_t* u;
    int64_t n;
    Ext2* S;  // folded factors from round 2 on (2^(v-1) entries each)
    Ext2* U;
    Ext2* E;  // eq(z_>t, .) (2^(v-1) entries)
    const Ext2* z;  // device copy of z_1..z_v
    int v;
    int grid;
    int per_block;
    int pad;
    uint64_t seq0;  // round t publishes seq0 + t, the final values seq0 + v + 1
    int t_begin;    // rounds run by this launch: [t_begin, t_end]; t_end > v includes the final values
    int t_end;
};

__device__ __forceinline__ int h2_at(const int8_t* p, int64_t n, int64_t x) { return x < n ? (int)p[x] : 0; }

__device__ __forceinline__ uint64_t h2_lift(int x) { return x < 0 ? GL_P - (uint64_t)(-(int64_t)x) : (uint64_t)x; }

// sa + rho (sb - sa) for small integers sa, sb
__device__ __forceinline__ Ext2 h2_fold_small(int sa, int sb, Ext2 rho) {
    const int d = sb - sa;
    return e2_make(gl_add(h2_lift(sa), gl_mul_small(rho.a, d)), gl_mul_small(rho.b, d));
}

// Widths of the chunk tables of eq(z_2..z_v, .), most significant chunk first.
__device__ __forceinline__ void h2_widths(int v, int (&w)[4]) {
    int rest = v - 1;
#pragma unroll
    for (int j = 0; j < 4; j++) {
        w[j] = rest < H2_CHUNK ? rest : H2_CHUNK;
        rest -= w[j];
    }
}

// Table j (at tab + 2^8 j) holds, for each y < 2^w[j], the product of eq(z_c, bit) over
// its w[j] coordinates (the first one on y's top bit). Called by every thread of the block.
__device__ __forceinline__ void h2_tables(Ext2* tab, const Ext2* zs, const int (&w)[4]) {
    for (int x = threadIdx.x; x < (4 << H2_CHUNK); x += blockDim.x) {
        const int j = x >> H2_CHUNK, y = x & ((1 << H2_CHUNK) - 1);
        if (y >= (1 << w[j])) continue;
        int first = 1;  // z_2 is zs[1]
        for (int k = 0; k < j; k++) first += w[k];
        Ext2 e = e2_make(1, 0);
        for (int i = 0; i < w[j]; i++) e = e2_mul(e, e2_eq1(zs[first + i], (y >> (w[j] - 1 - i)) & 1));
        tab[x] = e;
    }
    __syncthreads();
}

// eq(z_2..z_v, b) for b < 2^(v-1): one entry of each table
__device__ __forceinline__ Ext2 h2_eq_at(const Ext2* tab, const int (&w)[4], int64_t b) {
    const int s2 = w[3], s1 = w[3] + w[2], s0 = s1 + w[1];
    Ext2 e = tab[(int)((b >> s0) & ((1 << w[0]) - 1))];
    if (w[1]) e = e2_mul(e, tab[(1 << H2_CHUNK) + (int)((b >> s1) & ((1 << w[1]) - 1))]);
    if (w[2]) e = e2_mul(e, tab[(2 << H2_CHUNK) + (int)((b >> s2) & ((1 << w[2]) - 1))]);
    if (w[3]) e = e2_mul(e, tab[(3 << H2_CHUNK) + (int)(b & ((1 << w[3]) - 1))]);
    return e;
}

// v = 0: the claim s(0) u(0) and the final values s(0), u(0)
__global__ void had2_single_kernel(const int8_t* s, const int8_t* u, uint64_t* out) {
    const int a = s[0], b = u[0];
    out[0] = h2_lift(a * b);
    out[1] = 0;
    out[2] = h2_lift(a);
    out[3] = 0;
    out[4] = h2_lift(b);
    out[5] = 0;
}

// two blocks per SM: bounded to three (80 registers) the extension products spill and the
// 2^26-entry rounds slow down (3.56 -> 3.74 ms)
#ifndef FP_HAD2_MIN_BLOCKS
#define FP_HAD2_MIN_BLOCKS 2
#endif
__global__ void __launch_bounds__(H2_THREADS, FP_HAD2_MIN_BLOCKS) had2_session_kernel(Had2Args A, FpMailbox* mb, FpRelay* rl,
                                                                    uint64_t* part) {
    __shared__ Ext2 zs[32];
    __shared__ Ext2 tab[4 << H2_CHUNK];
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
        if (t == 1) {
            h2_widths(A.v, w);
            h2_tables(tab, zs, w);
        }
        E2Acc a0, a1, a2;
        for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < h; b += (int64_t)active * blockDim.x) {
            if (t == 1) {
                // the factors as they are: the three products are small integers
                const int s0 = h2_at(A.s, A.n, b), s1 = h2_at(A.s, A.n, b + h);
                const int u0 = h2_at(A.u, A.n, b), u1 = h2_at(A.u, A.n, b + h);
                const Ext2 e = h2_eq_at(tab, w, b);  // eq(z_2..z_v, b)
                if (A.v > 1) A.E[b] = e;
                a0.mac_base(e, h2_lift(s0 * u0));
                a1.mac_base(e, h2_lift(s1 * u1));
                a2.mac_base(e, h2_lift((2 * s1 - s0) * (2 * u1 - u0)));
                continue;
            }
            Ext2 s0, s1, u0, u1;
            if (t == 2) {
                // the int8 factors (length 4h) folded by rho_1
                s0 = h2_fold_small(h2_at(A.s, A.n, b), h2_at(A.s, A.n, b + 2 * h), rho);
                s1 = h2_fold_small(h2_at(A.s, A.n, b + h), h2_at(A.s, A.n, b + 3 * h), rho);
                u0 = h2_fold_small(h2_at(A.u, A.n, b), h2_at(A.u, A.n, b + 2 * h), rho);
                u1 = h2_fold_small(h2_at(A.u, A.n, b + h), h2_at(A.u, A.n, b + 3 * h), rho);
            } else {
                s0 = e2_fold(e2_ldcg(A.S + b), e2_ldcg(A.S + b + 2 * h), rho);
                s1 = e2_fold(e2_ldcg(A.S + b + h), e2_ldcg(A.S + b + 3 * h), rho);
                u0 = e2_fold(e2_ldcg(A.U + b), e2_ldcg(A.U + b + 2 * h), rho);
                u1 = e2_fold(e2_ldcg(A.U + b + h), e2_ldcg(A.U + b + 3 * h), rho);
            }
            A.S[b] = s0;
            A.S[b + h] = s1;
            A.U[b] = u0;
            A.U[b + h] = u1;
            const Ext2 e = e2_add(e2_ldcg(A.E + b), e2_ldcg(A.E + b + h));  // eq(z_>t, b)
            A.E[b] = e;
            const uint64_t e7 = gl_mul7(e.b);
            a0.mac(e, e7, e2_mul(s0, u0));
            a1.mac(e, e7, e2_mul(s1, u1));
            a2.mac(e, e7, e2_mul(e2_at2(s0, s1), e2_at2(u0, u1)));
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
    // block 0 folds the last pair by the last challenge: s~(rho), u~(rho)
    if (A.t_end <= A.v || blockIdx.x != 0) return;
    uint64_t ra, rb;
    if (!session_wait2(mb, rl, A.seq0 + A.v, ra, rb)) return;
    rho = e2_make(ra, rb);
    if (threadIdx.x == 0) {
        Ext2 sf, uf;
        if (A.v == 1) {
            sf = h2_fold_small(h2_at(A.s, A.n, 0), h2_at(A.s, A.n, 1), rho);
            uf = h2_fold_small(h2_at(A.u, A.n, 0), h2_at(A.u, A.n, 1), rho);
        } else {
            sf = e2_fold(e2_ldcg(A.S), e2_ldcg(A.S + 1), rho);
            uf = e2_fold(e2_ldcg(A.U), e2_ldcg(A.U + 1), rho);
        }
        const uint64_t fin[4] = {sf.a, sf.b, uf.a, uf.b};
        session_publish(mb, fin, A.seq0 + A.v + 1);
    }
}

// ---- the host half ------------------------------------------------------------

// Where the round values come from. Each call returns FP_OK or an error status.
struct Had2Source {
    virtual ~Had2Source() {}
    virtual void abandon() {}  // the host stopped early: let a waiting kernel finish
    virtual int start(const Ext2* z, int v) = 0;         // the point is known
    virtual int single(Ext2& claim, Ext2 fin[2]) = 0;    // v = 0: no rounds
    virtual int round(int t, Ext2 h[3]) = 0;             // h_t(0), h_t(1), h_t(2)
    virtual int answer(int t, Ext2 rho) = 0;             // the challenge rho_t
    virtual int finals(Ext2 fin[2]) = 0;                 // s~(rho), u~(rho)
};

// The protocol after "had2_site" is absorbed: proof of 16 + 64 v + 32 bytes.
int had2_protocol(fp_ctx* c, fp_tx* tx, int v, Had2Source& src, uint8_t* proof, size_t* proof_len) {
    Ext2 z[H2_MAX_V] = {};
    for (int i = 0; i < v; i++) z[i] = e2_squeeze_host(tx, "had2_z");
    int rc;
    if ((rc = src.start(z, v))) return rc;
    size_t pos = 0;
    Ext2 fin[2];
    if (v == 0) {
        Ext2 claim;
        if ((rc = src.single(claim, fin))) return rc;
        e2_send_host(tx, "had2_claim", &claim, 1, proof, pos);
    } else {
        const Ext2 one = e2_make(1, 0);
        Ext2 claim = e2_make(0, 0), pre = one;  // pre = eq(z_<t, rho_<t)
        for (int t = 1; t <= v; t++) {
            Ext2 h[3];
            if ((rc = src.round(t, h))) return rc;
            const Ext2 zt = z[t - 1];
            const Ext2 h3 = e2_add(e2_sub(h[0], e2_scal(h[1], 3)), e2_scal(h[2], 3));
            Ext2 g[4];
            g[0] = e2_mul(pre, e2_mul(e2_sub(one, zt), h[0]));
            g[1] = e2_mul(pre, e2_mul(zt, h[1]));
            g[2] = e2_mul(pre, e2_mul(e2_sub(e2_scal(zt, 3), one), h[2]));
            g[3] = e2_mul(pre, e2_mul(e2_sub(e2_scal(zt, 5), e2_make(2, 0)), h3));
            if (t == 1) {
                claim = e2_add(g[0], g[1]);
                e2_send_host(tx, "had2_claim", &claim, 1, proof, pos);
            } else if (!e2_same(e2_add(g[0], g[1]), claim)) {
                src.abandon();
                return fp_fail(c, FP_ERR_CUDA, "sumcheck_prove_hadamard_ext2: round values inconsistent with the claim");
            }
            e2_send_host(tx, "had2_round", g, 4, proof, pos);
            const Ext2 r = e2_squeeze_host(tx, "had2_chal");
            if ((rc = src.answer(t, r))) return rc;
            claim = e2_lagrange4(g, r);
            pre = e2_mul(pre, e2_eq(zt, r));
        }
        if ((rc = src.finals(fin))) return rc;
    }
    e2_send_host(tx, "had2_final", fin, 2, proof, pos);
    *proof_len = pos;
    return FP_OK;
}

// Round values from the resident kernel.
struct Had2Device : Had2Source {
    fp_ctx* c;
    cudaStream_t st;
    const int8_t* s;
    const int8_t* u;
    int64_t n;
    Had2Args A;
    uint64_t* part = nullptr;
    uint64_t* small = nullptr;  // device: [0..6) single-entry values, [8..8 + 2v) z
    uint64_t* hs = nullptr;     // pinned host staging
    int cap_grid = 1;

    int launch(int t_begin, int t_end, unsigned grid, int kernel, double bytes) {
        A.t_begin = t_begin;
        A.t_end = t_end;
        void* args[] = {&A, &c->mb_dev, &c->relay, &part};
        int slot;
        fp_tic(c, st, kernel, bytes, &slot);
        FP_CUDA(c, cudaLaunchCooperativeKernel((const void*)had2_session_kernel, dim3(grid), dim3(H2_THREADS), args,
                                               0, st));
        fp_toc(c, st, slot);
        return FP_OK;
    }

    double round_bytes(int t) const {
        const double pairs = (double)(1ll << (A.v - t));
        // round 1: four int8 reads and one E write per pair; round 2: eight int8 reads, two E
        // reads, four factor writes and one E write; later rounds: eight factor reads instead
        return t == 1 ? 20.0 * pairs : (t == 2 ? 120.0 * pairs : 240.0 * pairs);
    }

    void abandon() override { fp_session_abandon(c, st); }

    int start(const Ext2* z, int v) override {
        int rc;
        const int64_t half = v > 0 ? 1ll << (v - 1) : 0;
        int occ = 0;
        FP_CUDA(c, cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, had2_session_kernel, H2_THREADS, 0));
        cap_grid = std::max(1, occ) * c->num_sms;
        const size_t part_n = (size_t)6 * cap_grid;
        const size_t vec = fp_align_up((size_t)16 * std::max<int64_t>(half, 1), 256);
        const size_t need = 3 * vec + fp_align_up(8 * part_n, 256) + fp_align_up(8 * 128, 256) + 4096;
        if ((rc = fp_reserve(c, c->dev, need))) return rc;
        if ((rc = fp_reserve(c, c->host, 4096))) return rc;
        fp_reset(c->dev);
        fp_reset(c->host);
        Ext2* S = (Ext2*)fp_alloc(c->dev, vec);
        Ext2* U = (Ext2*)fp_alloc(c->dev, vec);
        Ext2* E = (Ext2*)fp_alloc(c->dev, vec);
        part = (uint64_t*)fp_alloc(c->dev, 8 * part_n);
        small = (uint64_t*)fp_alloc(c->dev, 8 * 128);
        hs = (uint64_t*)fp_alloc(c->host, 8 * 128);
        if (!S || !U || !E || !part || !small || !hs)
            return fp_fail(c, FP_ERR_OOM, "sumcheck_prove_hadamard_ext2: scratch exhausted");
        if (v == 0) return FP_OK;
        for (int i = 0; i < v; i++) {
            hs[8 + 2 * i] = z[i].a;
            hs[8 + 2 * i + 1] = z[i].b;
        }
        FP_CUDA(c, cudaMemcpyAsync(small + 8, hs + 8, 16 * (size_t)v, cudaMemcpyHostToDevice, st));
        memset(&A, 0, sizeof A);
        A.s = s;
        A.u = u;
        A.n = n;
        A.S = S;
        A.U = U;
        A.E = E;
        A.z = (const Ext2*)(small + 8);
        A.v = v;
        A.per_block = H2_THREADS;  // one pair per thread
        A.grid = (int)std::max<int64_t>(1, std::min<int64_t>((half + A.per_block - 1) / A.per_block, cap_grid));
        A.seq0 = fp_seq_reserve(c, (uint64_t)v + 2);
        if ((rc = fp_session_begin(c, st))) return rc;
        fp_session_expect(c, 6);  // before any launch: round 1 publishes without a challenge
        if (!c->stepped) {
            double bytes = 0;
            for (int t = 1; t <= v; t++) bytes += round_bytes(t);
            return launch(1, v + 1, (unsigned)A.grid, K_HAD2_ROUND, bytes);
        }
        return FP_OK;
    }

    int single(Ext2& claim, Ext2 fin[2]) override {
        int slot;
        fp_tic(c, st, K_HAD2_FINAL, 2.0 + 48.0, &slot);
        had2_single_kernel<<<1, 1, 0, st>>>(s, u, small);
        fp_toc(c, st, slot);
        FP_CUDA(c, cudaGetLastError());
        FP_CUDA(c, cudaMemcpyAsync(hs, small, 48, cudaMemcpyDeviceToHost, st));
        FP_CUDA(c, cudaStreamSynchronize(st));
        claim = e2_make(hs[0], hs[1]);
        fin[0] = e2_make(hs[2], hs[3]);
        fin[1] = e2_make(hs[4], hs[5]);
        return FP_OK;
    }

    int round(int t, Ext2 h[3]) override {
        int rc;
        if (c->stepped && (rc = launch(t, t, (unsigned)A.grid, K_HAD2_ROUND, round_bytes(t)))) return rc;
        if ((rc = fp_session_wait(c, A.seq0 + t, st))) return rc;
        for (int i = 0; i < 3; i++) h[i] = e2_make(c->mb->res[2 * i], c->mb->res[2 * i + 1]);
        return FP_OK;
    }

    int answer(int t, Ext2 rho) override {
        fp_session_expect(c, t < A.v ? 6 : 4);  // the last challenge triggers the final values
        fp_session_post2(c, A.seq0 + t, rho.a, rho.b);
        return FP_OK;
    }

    int finals(Ext2 fin[2]) override {
        int rc;
        if (c->stepped && (rc = launch(A.v + 1, A.v + 1, 1, K_HAD2_FINAL, 64.0))) return rc;
        if ((rc = fp_session_wait(c, A.seq0 + A.v + 1, st))) return rc;
        fin[0] = e2_make(c->mb->res[0], c->mb->res[1]);
        fin[1] = e2_make(c->mb->res[2], c->mb->res[3]);
        FP_CUDA(c, cudaStreamSynchronize(st));
        return FP_OK;
    }
};

// Round values from a caller's callback (no device).
struct Had2Callback : Had2Source {
    fp_values_fn fn;
    void* user;
    int call(int kind, int t, const uint64_t* in, uint64_t* out) {
        return fn(user, kind, t, in, out) ? FP_ERR_ARG : FP_OK;
    }
    int start(const Ext2* z, int v) override {
        uint64_t in[2 * H2_MAX_V + 2];
        for (int i = 0; i < v; i++) {
            in[2 * i] = z[i].a;
            in[2 * i + 1] = z[i].b;
        }
        return call(FP_VAL_START, v, in, nullptr);
    }
    int single(Ext2& claim, Ext2 fin[2]) override {
        uint64_t out[6] = {0, 0, 0, 0, 0, 0};
        int rc = call(FP_VAL_SINGLE, 0, nullptr, out);
        claim = e2_make(gl_canon(out[0]), gl_canon(out[1]));
        fin[0] = e2_make(gl_canon(out[2]), gl_canon(out[3]));
        fin[1] = e2_make(gl_canon(out[4]), gl_canon(out[5]));
        return rc;
    }
    int round(int t, Ext2 h[3]) override {
        uint64_t out[6] = {0, 0, 0, 0, 0, 0};
        int rc = call(FP_VAL_ROUND, t, nullptr, out);
        for (int i = 0; i < 3; i++) h[i] = e2_make(gl_canon(out[2 * i]), gl_canon(out[2 * i + 1]));
        return rc;
    }
    int answer(int t, Ext2 rho) override {
        const uint64_t in[2] = {rho.a, rho.b};
        return call(FP_VAL_ANSWER, t, in, nullptr);
    }
    int finals(Ext2 fin[2]) override {
        uint64_t out[4] = {0, 0, 0, 0};
        int rc = call(FP_VAL_FINALS, 0, nullptr, out);
        fin[0] = e2_make(gl_canon(out[0]), gl_canon(out[1]));
        fin[1] = e2_make(gl_canon(out[2]), gl_canon(out[3]));
        return rc;
    }
};

}  // namespace

int sumcheck_prove_hadamard_ext2(fp_ctx* c, fp_tx* tx, const int8_t* s, const int8_t* u, int64_t n, uint8_t* proof,
                                 size_t* proof_len, void* stream) {
    if (!c || !tx || !proof_len) return fp_fail(c, FP_ERR_ARG, "sumcheck_prove_hadamard_ext2: null argument");
    if (!s || !u) return fp_fail(c, FP_ERR_ARG, "sumcheck_prove_hadamard_ext2: null factor");
    if (n < 1 || n > (1ll << H2_MAX_V))
        return fp_fail(c, FP_ERR_SHAPE, "sumcheck_prove_hadamard_ext2: need 1 <= n <= 2^30");
    const int v = fp_log2_ceil((uint64_t)n);
    const size_t need_len = 16 + 64 * (size_t)v + 32;
    if (!proof || *proof_len < need_len) {
        *proof_len = need_len;
        return fp_fail(c, FP_ERR_ARG, "sumcheck_prove_hadamard_ext2: proof buffer too small");
    }
    FP_CUDA(c, cudaSetDevice(c->device));
    cudaStream_t st = (cudaStream_t)stream;
    int rc;
    {
        FpDigestJob jobs[2] = {{(const uint8_t*)s, (uint64_t)n}, {(const uint8_t*)u, (uint64_t)n}};
        uint8_t d[64];
        if ((rc = fp_digest_many(c, jobs, 2, d, st))) return rc;  // synchronises the stream
        fp_tx_absorb_raw(tx, "had2_site", d, 64);
    }
    Had2Device dev;
    dev.c = c;
    dev.st = st;
    dev.s = s;
    dev.u = u;
    dev.n = n;
    return had2_protocol(c, tx, v, dev, proof, proof_len);
}

int fp_had2_protocol_drive(fp_tx* tx, int v, fp_values_fn fn, void* user, uint8_t* proof, size_t* proof_len) {
    if (!tx || !fn || !proof_len) return FP_ERR_ARG;
    if (v < 0 || v > H2_MAX_V) return FP_ERR_SHAPE;
    const size_t need_len = 16 + 64 * (size_t)v + 32;
    if (!proof || *proof_len < need_len) {
        *proof_len = need_len;
        return FP_ERR_ARG;
    }
    Had2Callback cb;
    cb.fn = fn;
    cb.user = user;
    return had2_protocol(nullptr, tx, v, cb, proof, proof_len);
}
