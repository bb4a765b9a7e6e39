// LogUp proof of the rescale remainders and clamps.
//
// "How fast can FlashProve go", 3.1: every rescale commits its remainder r and
// a lookup shows that r is small; clamps are non-polynomial and are proven by
// lookup as well. Same page, 4 Tighter Rooflines: a lookup compares a product
// over the keys with one over the table; the key side is built as a binary
// tree and every level of the tree is proven with sum-check (keys are small
// integers, so the leaf level is cheap). "Towards Proving Frontier-Scale LLM
// Inference", The proof system: lookups by logarithmic derivatives (LogUp).
// Here the tree holds LogUp fractions: leaves (1, alpha - f), parents
// (pL qR + pR qL, qL qR). Two tables share one tree shape -- the remainder range
// table (key r) and the clamp table (key q + gamma y, which also bounds q to 16
// bits) -- and every layer of both trees is proven by one degree-3 sum-check.
//
// Layer d (point z of d coordinates, challenges lambda): round t sends
// g(X) = sum_b eq(z, (rho_<t, X, b)) F(rho_<t, X, b) at X = 0..3 with
// F = sum_tau lambda^(2 tau) (pL qR + pR qL + lambda qL qR)_tau. The kernels
// compute h(X) = sum_b eq(z_>t, b) F(., X, b) at X = 0, 1, 2 and the last block
// forms g(X) = eq(z_<t, rho_<t) eq(z_t, X) h(X) (h has degree 2). The vectors are
// folded in place by the previous challenge in the same pass; the suffix eq
// table is kept in place too (E_t[b] = E_(t-1)[b] + E_(t-1)[b + h]).
#include <string.h>

#include <vector>

#include "fp_internal.h"
#include "fp_reduce.cuh"

namespace {

constexpr int LU_THREADS = 256;

struct KeySrc {
    const int32_t* r;
    const int32_t* q;
    const int8_t* y;
    int64_t n;  // real keys; indices in [n, 2^v) are the neutral key 0
};

struct Chal {
    uint64_t alpha0, alpha1, gamma;
};

__device__ __forceinline__ void key_at(const KeySrc& K, int64_t i, int32_t& r, int32_t& q, int32_t& y) {
    if (i < K.n) {
        r = K.r[i];
        q = K.q[i];
        y = K.y[i];
    } else {
        r = q = y = 0;
    }
}

// leaf denominators alpha - f of key i for both tables
__device__ __forceinline__ void leaf_den(const KeySrc& K, const Chal& C, int64_t i, uint64_t& d0, uint64_t& d1) {
    int32_t r, q, y;
    key_at(K, i, r, q, y);
    d0 = gl_sub(C.alpha0, gl_from_i64(r));
    d1 = gl_sub(C.alpha1, gl_add(gl_from_i64(q), gl_mul(C.gamma, gl_from_i64(y))));
}

// ---- histograms --------------------------------------------------------------

constexpr int HIST_WIN = 1 << 14;  // q in [-2^14, 2^14) counted in shared memory

__global__ void __launch_bounds__(1024) hist_kernel(KeySrc K, int k, int64_t L, uint32_t* __restrict__ m_rem,
                                                    uint32_t* __restrict__ m_clamp, uint32_t* __restrict__ outside,
                                                    int rem_in_smem) {
    extern __shared__ uint32_t sh[];
    uint32_t* sq = sh;                   // 2 * HIST_WIN bins
    uint32_t* sr = sh + 2 * HIST_WIN;    // 2^k bins when rem_in_smem
    const int64_t T = 1ll << k;
    const int32_t half = 1 << (k - 1);
    for (int i = threadIdx.x; i < 2 * HIST_WIN; i += blockDim.x) sq[i] = 0;
    if (rem_in_smem)
        for (int i = threadIdx.x; i < T; i += blockDim.x) sr[i] = 0;
    __syncthreads();
    uint32_t out_local = 0;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < K.n; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t jr = (int64_t)K.r[i] + half;
        if (jr >= 0 && jr < T) {
            if (rem_in_smem)
                atomicAdd(&sr[jr], 1u);
            else
                atomicAdd(&m_rem[jr], 1u);
        } else {
            out_local++;
        }
        const int64_t q = K.q[i];
        if (q >= -HIST_WIN && q < HIST_WIN)
            atomicAdd(&sq[q + HIST_WIN], 1u);
        else if (q >= -32768 && q < 32768)
            atomicAdd(&m_clamp[q + 32768], 1u);
        else
            out_local++;
        if ((int32_t)K.y[i] != (q < -128 ? -128 : (q > 127 ? 127 : (int32_t)q))) out_local++;
    }
    if (out_local) atomicAdd(outside, out_local);
    __syncthreads();
    for (int i = threadIdx.x; i < 2 * HIST_WIN; i += blockDim.x)
        if (sq[i]) atomicAdd(&m_clamp[i - HIST_WIN + 32768], sq[i]);
    if (rem_in_smem)
        for (int i = threadIdx.x; i < T; i += blockDim.x)
            if (sr[i]) atomicAdd(&m_rem[i], sr[i]);
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        // the padding keys are the neutral key 0 of both tables
        const uint32_t pad = (uint32_t)(L - K.n);
        atomicAdd(&m_rem[half], pad);
        atomicAdd(&m_clamp[32768], pad);
    }
}

// ---- key gather (several sites) ---------------------------------------------

struct GatherSite {
    const int32_t* q;
    const int32_t* r;
    const int8_t* y;
    int64_t first;  // offset in the concatenated key vector
};

__global__ void gather_kernel(const GatherSite* __restrict__ gs, int nsites, int64_t n, int32_t* __restrict__ r,
                              int32_t* __restrict__ q, int8_t* __restrict__ y) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        int lo = 0, hi = nsites - 1;
        while (lo < hi) {
            int mid = (lo + hi + 1) >> 1;
            if (gs[mid].first <= i)
                lo = mid;
            else
                hi = mid - 1;
        }
        const int64_t e = i - gs[lo].first;
        r[i] = gs[lo].r[e];
        q[i] = gs[lo].q[e];
        y[i] = gs[lo].y[e];
    }
}

// ---- tree --------------------------------------------------------------------

struct TreeLayer {
    uint64_t* P[2];
    uint64_t* Q[2];
};

// layer v-1 from the leaves: p = qL + qR (leaf numerators are 1), q = qL qR
__global__ void tree_leaf_kernel(KeySrc K, Chal C, TreeLayer out, int64_t n) {
    for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < n; x += (int64_t)gridDim.x * blockDim.x) {
        uint64_t l0, l1, r0, r1;
        leaf_den(K, C, 2 * x, l0, l1);
        leaf_den(K, C, 2 * x + 1, r0, r1);
        out.P[0][x] = gl_add(l0, r0);
        out.Q[0][x] = gl_mul(l0, r0);
        out.P[1][x] = gl_add(l1, r1);
        out.Q[1][x] = gl_mul(l1, r1);
    }
}

__global__ void tree_up_kernel(TreeLayer in, TreeLayer out, int64_t n) {
    for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < n; x += (int64_t)gridDim.x * blockDim.x) {
#pragma unroll
        for (int tau = 0; tau < 2; tau++) {
            const ulonglong2 p = reinterpret_cast<const ulonglong2*>(in.P[tau])[x];
            const ulonglong2 q = reinterpret_cast<const ulonglong2*>(in.Q[tau])[x];
            out.P[tau][x] = gl_add(gl_mul(p.x, q.y), gl_mul(p.y, q.x));
            out.Q[tau][x] = gl_mul(q.x, q.y);
        }
    }
}

// layer one when the leaves themselves are the two-node layer (v == 1)
__global__ void l1_from_keys_kernel(KeySrc K, Chal C, uint64_t* out) {
    uint64_t a0, a1, b0, b1;
    leaf_den(K, C, 0, a0, a1);
    leaf_den(K, C, 1, b0, b1);
    out[0] = 1; out[1] = 1; out[2] = a0; out[3] = b0;
    out[4] = 1; out[5] = 1; out[6] = a1; out[7] = b1;
}

__global__ void l1_from_layer_kernel(TreeLayer one, uint64_t* out) {
    for (int tau = 0; tau < 2; tau++) {
        out[4 * tau + 0] = one.P[tau][0];
        out[4 * tau + 1] = one.P[tau][1];
        out[4 * tau + 2] = one.Q[tau][0];
        out[4 * tau + 3] = one.Q[tau][1];
    }
}

// ---- layer sum-check rounds ----------------------------------------------------

struct GkrArgs {
    // pair vectors (x: left child, y: right child); LEAF layers have no p vectors
    ulonglong2* pp[2];
    ulonglong2* qq[2];
    const ulonglong2* src_pp[2];  // round 1 / round 2 source when not from keys
    const ulonglong2* src_qq[2];
    uint64_t* E;
    uint64_t* state;  // [0] = eq(z_<t, rho_<t)
    KeySrc keys;
    Chal chal;
    FpPoint z;        // the layer's point (d coordinates)
    int d, t;
    int64_t h;        // pairs this round: 2^(d - t)
    uint64_t rprev, lam;
};

// F(X) of one pair position for the two tables
template <bool LEAF>
__device__ __forceinline__ uint64_t layer_F(const uint64_t (&pl)[2], const uint64_t (&pr)[2], const uint64_t (&ql)[2],
                                            const uint64_t (&qr)[2], uint64_t lam, uint64_t lam2) {
    uint64_t f[2];
#pragma unroll
    for (int tau = 0; tau < 2; tau++) {
        const uint64_t qq = gl_mul(ql[tau], qr[tau]);
        const uint64_t cross = LEAF ? gl_add(qr[tau], ql[tau]) : gl_add(gl_mul(pl[tau], qr[tau]), gl_mul(pr[tau], ql[tau]));
        f[tau] = gl_add(cross, gl_mul(lam, qq));
    }
    return gl_add(f[0], gl_mul(lam2, f[1]));
}

// Source pair at position x of the layer's initial vectors.
template <bool KEYS>
__device__ __forceinline__ void src_pair(const GkrArgs& A, int64_t x, ulonglong2 (&pp)[2], ulonglong2 (&qq)[2]) {
    if (KEYS) {
        uint64_t l0, l1, r0, r1;
        leaf_den(A.keys, A.chal, 2 * x, l0, l1);
        leaf_den(A.keys, A.chal, 2 * x + 1, r0, r1);
        pp[0] = make_ulonglong2(1, 1);
        pp[1] = make_ulonglong2(1, 1);
        qq[0] = make_ulonglong2(l0, r0);
        qq[1] = make_ulonglong2(l1, r1);
    } else {
#pragma unroll
        for (int tau = 0; tau < 2; tau++) {
            pp[tau] = A.src_pp[tau][x];
            qq[tau] = A.src_qq[tau][x];
        }
    }
}

__device__ __forceinline__ ulonglong2 fold2(ulonglong2 a, ulonglong2 b, uint64_t r) {
    return make_ulonglong2(gl_fold(a.x, b.x, r), gl_fold(a.y, b.y, r));
}

// MODE 0: round 1 (no fold). MODE 1: fold from the source (round 2).
// MODE 2: fold in place in pp/qq (round >= 3). KEYS: the source is the key columns.
template <bool LEAF, bool KEYS, int MODE>
__global__ void __launch_bounds__(LU_THREADS) gkr_round_kernel(GkrArgs A, uint64_t* part, unsigned int* ticket,
                                                               uint64_t* __restrict__ gout) {
    uint64_t acc[3] = {0, 0, 0};
    const int64_t h = A.h;
    const uint64_t lam2 = gl_mul(A.lam, A.lam);
    for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < h; b += (int64_t)gridDim.x * blockDim.x) {
        ulonglong2 c0p[2], c0q[2], c1p[2], c1q[2];  // current pairs at b and b + h
        uint64_t e;
        if (MODE == 0) {
            src_pair<KEYS>(A, b, c0p, c0q);
            src_pair<KEYS>(A, b + h, c1p, c1q);
            // E_1[b] = eq(z_2..z_d, b)
            e = 1;
            const int nb = A.d - 1;
            for (int i = 0; i < nb; i++) e = gl_mul(e, gl_eq1(A.z.z[1 + i], (int)((b >> (nb - 1 - i)) & 1)));
            if (A.d > 1) A.E[b] = e;
        } else {
            ulonglong2 s0p[2], s0q[2], s1p[2], s1q[2], s2p[2], s2q[2], s3p[2], s3q[2];
            if (MODE == 1) {
                src_pair<KEYS>(A, b, s0p, s0q);
                src_pair<KEYS>(A, b + h, s1p, s1q);
                src_pair<KEYS>(A, b + 2 * h, s2p, s2q);
                src_pair<KEYS>(A, b + 3 * h, s3p, s3q);
            } else {
#pragma unroll
                for (int tau = 0; tau < 2; tau++) {
                    if (!LEAF) {
                        s0p[tau] = A.pp[tau][b];
                        s1p[tau] = A.pp[tau][b + h];
                        s2p[tau] = A.pp[tau][b + 2 * h];
                        s3p[tau] = A.pp[tau][b + 3 * h];
                    } else {
                        s0p[tau] = s1p[tau] = s2p[tau] = s3p[tau] = make_ulonglong2(1, 1);
                    }
                    s0q[tau] = A.qq[tau][b];
                    s1q[tau] = A.qq[tau][b + h];
                    s2q[tau] = A.qq[tau][b + 2 * h];
                    s3q[tau] = A.qq[tau][b + 3 * h];
                }
            }
#pragma unroll
            for (int tau = 0; tau < 2; tau++) {
                if (LEAF) {
                    c0p[tau] = c1p[tau] = make_ulonglong2(1, 1);
                } else {
                    c0p[tau] = fold2(s0p[tau], s2p[tau], A.rprev);
                    c1p[tau] = fold2(s1p[tau], s3p[tau], A.rprev);
                    A.pp[tau][b] = c0p[tau];
                    A.pp[tau][b + h] = c1p[tau];
                }
                c0q[tau] = fold2(s0q[tau], s2q[tau], A.rprev);
                c1q[tau] = fold2(s1q[tau], s3q[tau], A.rprev);
                A.qq[tau][b] = c0q[tau];
                A.qq[tau][b + h] = c1q[tau];
            }
            e = gl_add(A.E[b], A.E[b + h]);
            A.E[b] = e;
        }
        // h(X) at X = 0, 1, 2
        uint64_t pl[2], pr[2], ql[2], qr[2];
#pragma unroll
        for (int X = 0; X < 3; X++) {
#pragma unroll
            for (int tau = 0; tau < 2; tau++) {
                if (X == 0) {
                    pl[tau] = c0p[tau].x; pr[tau] = c0p[tau].y; ql[tau] = c0q[tau].x; qr[tau] = c0q[tau].y;
                } else if (X == 1) {
                    pl[tau] = c1p[tau].x; pr[tau] = c1p[tau].y; ql[tau] = c1q[tau].x; qr[tau] = c1q[tau].y;
                } else {
                    pl[tau] = gl_sub(gl_add(c1p[tau].x, c1p[tau].x), c0p[tau].x);
                    pr[tau] = gl_sub(gl_add(c1p[tau].y, c1p[tau].y), c0p[tau].y);
                    ql[tau] = gl_sub(gl_add(c1q[tau].x, c1q[tau].x), c0q[tau].x);
                    qr[tau] = gl_sub(gl_add(c1q[tau].y, c1q[tau].y), c0q[tau].y);
                }
            }
            acc[X] = gl_add(acc[X], gl_mul(e, layer_F<LEAF>(pl, pr, ql, qr, A.lam, lam2)));
        }
    }
    if (grid_sum_gl<3>(acc, part, ticket) && threadIdx.x == 0) {
        // prefix eq(z_<t, rho_<t), updated with the previous round's challenge
        uint64_t pre = 1;
        if (A.t > 1) {
            const uint64_t zp = A.z.z[A.t - 2];
            pre = gl_mul(A.state[0], gl_add(gl_mul(zp, A.rprev), gl_mul(gl_sub(1, zp), gl_sub(1, A.rprev))));
        }
        A.state[0] = pre;
        const uint64_t zt = A.z.z[A.t - 1];
        // h(3) from the third finite difference of a quadratic
        const uint64_t h3 = gl_add(gl_sub(gl_mul(3, acc[2]), gl_mul(3, acc[1])), acc[0]);
        const uint64_t hv[4] = {acc[0], acc[1], acc[2], h3};
        const uint64_t one_m = gl_sub(1, zt), slope = gl_sub(gl_add(zt, zt), 1);  // eq(z_t, X) = (1 - z_t) + X (2 z_t - 1)
#pragma unroll
        for (int X = 0; X < 4; X++) {
            const uint64_t ex = gl_add(one_m, gl_mul((uint64_t)X, slope));
            gout[X] = gl_mul(pre, gl_mul(ex, hv[X]));
        }
    }
}

// The eight child values at the layer's last challenge.
template <bool LEAF, bool KEYS>
__global__ void gkr_final_kernel(GkrArgs A, uint64_t rlast, uint64_t* out) {
    if (threadIdx.x != 0) return;
    ulonglong2 p0[2], q0[2], p1[2], q1[2];
    if (KEYS) {
        src_pair<true>(A, 0, p0, q0);
        src_pair<true>(A, 1, p1, q1);
    } else {
#pragma unroll
        for (int tau = 0; tau < 2; tau++) {
            p0[tau] = LEAF ? make_ulonglong2(1, 1) : A.pp[tau][0];
            p1[tau] = LEAF ? make_ulonglong2(1, 1) : A.pp[tau][1];
            q0[tau] = A.qq[tau][0];
            q1[tau] = A.qq[tau][1];
        }
    }
#pragma unroll
    for (int tau = 0; tau < 2; tau++) {
        out[4 * tau + 0] = gl_fold(p0[tau].x, p1[tau].x, rlast);
        out[4 * tau + 1] = gl_fold(p0[tau].y, p1[tau].y, rlast);
        out[4 * tau + 2] = gl_fold(q0[tau].x, q1[tau].x, rlast);
        out[4 * tau + 3] = gl_fold(q0[tau].y, q1[tau].y, rlast);
    }
}

// ---- leaf claims: MLEs of the key columns at z (split eq: hi x lo) ----------------

__global__ void __launch_bounds__(LU_THREADS) leaf_eval_kernel(KeySrc K, const uint64_t* __restrict__ ehi,
                                                               const uint64_t* __restrict__ elo, int lo_bits, int64_t L,
                                                               uint64_t* part, unsigned int* ticket,
                                                               uint64_t* __restrict__ out) {
    uint64_t acc[3] = {0, 0, 0};
    const int64_t mask = (1ll << lo_bits) - 1;
    for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < K.n && x < L;
         x += (int64_t)gridDim.x * blockDim.x) {
        const uint64_t e = gl_mul(ehi[x >> lo_bits], elo[x & mask]);
        acc[0] = gl_add(acc[0], gl_mul(e, gl_from_i64(K.r[x])));
        acc[1] = gl_add(acc[1], gl_mul(e, gl_from_i64(K.q[x])));
        acc[2] = gl_add(acc[2], gl_mul(e, gl_from_i64(K.y[x])));
    }
    if (grid_sum_gl<3>(acc, part, ticket) && threadIdx.x == 0) {
        out[0] = acc[0];
        out[1] = acc[1];
        out[2] = acc[2];
    }
}

void put_le(uint8_t* p, uint64_t v, int nb) {
    for (int i = 0; i < nb; i++) p[i] = (uint8_t)(v >> (8 * i));
}

int grid_for(fp_ctx* c, int64_t work, int threads) {
    int64_t b = (work + threads - 1) / threads;
    int64_t cap = 8ll * c->num_sms;
    if (b > cap) b = cap;
    if (b < 1) b = 1;
    return (int)b;
}

}  // namespace

int logup_prove_rescale(fp_ctx* c, fp_tx* tx, const fp_site* sites, int nsites, uint8_t* proof, size_t* proof_len,
                        void* stream) {
    if (!c || !tx || !proof_len) return fp_fail(c, FP_ERR_ARG, "logup_prove_rescale: null argument");
    int rc = fp_check_sites(c, sites, nsites, true);
    if (rc) return rc;
    for (int s = 1; s < nsites; s++)
        if (sites[s].k_shift != sites[0].k_shift)
            return fp_fail(c, FP_ERR_SHAPE, "logup_prove_rescale: all sites must share k_shift");
    size_t mm_bytes, lu_bytes;
    fp_proof_size(sites, nsites, &mm_bytes, &lu_bytes);
    if (!proof || *proof_len < lu_bytes) {
        *proof_len = lu_bytes;
        return fp_fail(c, FP_ERR_ARG, "logup_prove_rescale: proof buffer too small");
    }
    FP_CUDA(c, cudaSetDevice(c->device));
    cudaStream_t st = (cudaStream_t)stream;

    const int k = sites[0].k_shift;
    int64_t nk = 0;
    for (int s = 0; s < nsites; s++) nk += (int64_t)sites[s].M * sites[s].N;
    int v = fp_log2_ceil((uint64_t)nk);
    if (v < 1) v = 1;
    if (v > 31) return fp_fail(c, FP_ERR_SHAPE, "logup_prove_rescale: more than 2^31 keys");
    const int64_t L = 1ll << v;
    const int64_t T = 1ll << k;

    // ---- scratch ----
    size_t need = 0;
    if (nsites > 1) need += fp_align_up(9 * (size_t)nk + 1024, 256) + fp_align_up(sizeof(GatherSite) * nsites, 256);
    need += fp_align_up(4 * (size_t)T, 256) + fp_align_up(4 * 65536, 256) + 256;
    size_t tree = 0;
    for (int d = 1; d <= v - 1; d++) tree += 4 * fp_align_up((size_t)8 << d, 256);
    need += tree;
    if (v >= 2) need += 2 * fp_align_up((size_t)16 << (v - 2), 256);          // leaf-layer fold buffers
    need += fp_align_up((size_t)8 << (v >= 2 ? v - 2 : 0), 256);              // suffix eq table
    const int lo_bits = v / 2;
    need += fp_align_up((size_t)8 << lo_bits, 256) + fp_align_up((size_t)8 << (v - lo_bits), 256);
    need += fp_align_up((size_t)8 * 3 * 8 * c->num_sms, 256) + 4096;
    if ((rc = fp_reserve(c, c->dev, need + (1 << 20)))) return rc;
    if ((rc = fp_reserve(c, c->host, 4 * (size_t)T + 4 * 65536 + 4096 + sizeof(GatherSite) * nsites))) return rc;
    fp_reset(c->dev);
    fp_reset(c->host);

    // ---- keys ----
    KeySrc K;
    K.n = nk;
    if (nsites == 1) {
        K.r = sites[0].r;
        K.q = sites[0].q;
        K.y = sites[0].y;
    } else {
        int32_t* r = (int32_t*)fp_alloc(c->dev, 4 * (size_t)nk);
        int32_t* q = (int32_t*)fp_alloc(c->dev, 4 * (size_t)nk);
        int8_t* y = (int8_t*)fp_alloc(c->dev, (size_t)nk);
        std::vector<GatherSite> gs(nsites);
        int64_t off = 0;
        for (int s = 0; s < nsites; s++) {
            gs[s] = GatherSite{sites[s].q, sites[s].r, sites[s].y, off};
            off += (int64_t)sites[s].M * sites[s].N;
        }
        GatherSite* dgs = (GatherSite*)fp_alloc(c->dev, sizeof(GatherSite) * nsites);
        GatherSite* hgs = (GatherSite*)fp_alloc(c->host, sizeof(GatherSite) * nsites);
        memcpy(hgs, gs.data(), sizeof(GatherSite) * nsites);
        FP_CUDA(c, cudaMemcpyAsync(dgs, hgs, sizeof(GatherSite) * nsites, cudaMemcpyHostToDevice, st));
        int slot;
        fp_tic(c, st, K_KEYS_GATHER, 18.0 * nk, &slot);
        gather_kernel<<<grid_for(c, nk, 256), 256, 0, st>>>(dgs, nsites, nk, r, q, y);
        fp_toc(c, st, slot);
        FP_CUDA(c, cudaGetLastError());
        K.r = r;
        K.q = q;
        K.y = y;
    }

    // ---- multiplicities ----
    uint32_t* m_rem = (uint32_t*)fp_alloc(c->dev, 4 * (size_t)T);
    uint32_t* m_cl = (uint32_t*)fp_alloc(c->dev, 4 * 65536);
    uint32_t* outside = (uint32_t*)fp_alloc(c->dev, 256);
    FP_CUDA(c, cudaMemsetAsync(m_rem, 0, 4 * (size_t)T, st));
    FP_CUDA(c, cudaMemsetAsync(m_cl, 0, 4 * 65536, st));
    FP_CUDA(c, cudaMemsetAsync(outside, 0, 4, st));
    {
        const int rem_smem = T <= 16384;
        const int smem = 4 * (2 * HIST_WIN) + (rem_smem ? 4 * (int)T : 0);
        FP_CUDA(c, cudaFuncSetAttribute(hist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
        int slot;
        fp_tic(c, st, K_HIST, 9.0 * nk, &slot);
        hist_kernel<<<c->num_sms, 1024, smem, st>>>(K, k, L, m_rem, m_cl, outside, rem_smem);
        fp_toc(c, st, slot);
        FP_CUDA(c, cudaGetLastError());
    }
    uint8_t* hm = (uint8_t*)fp_alloc(c->host, 4 * (size_t)T + 4 * 65536 + 256);
    FP_CUDA(c, cudaMemcpyAsync(hm, m_rem, 4 * (size_t)T, cudaMemcpyDeviceToHost, st));
    FP_CUDA(c, cudaMemcpyAsync(hm + 4 * T, m_cl, 4 * 65536, cudaMemcpyDeviceToHost, st));
    FP_CUDA(c, cudaMemcpyAsync(hm + 4 * T + 4 * 65536, outside, 4, cudaMemcpyDeviceToHost, st));
    uint8_t dg_rem[32], dg_cl[32];
    {
        FpDigestJob jobs[2] = {{(const uint8_t*)m_rem, 4 * (uint64_t)T}, {(const uint8_t*)m_cl, 4 * 65536ull}};
        uint8_t both[64];
        if ((rc = fp_digest_many(c, jobs, 2, both, st))) return rc;  // synchronises the stream
        memcpy(dg_rem, both, 32);
        memcpy(dg_cl, both + 32, 32);
    }
    uint32_t n_outside;
    memcpy(&n_outside, hm + 4 * T + 4 * 65536, 4);
    size_t pos = 0;
    memcpy(proof + pos, hm, 4 * (size_t)T);  // device words are little-endian u32
    pos += 4 * (size_t)T;
    fp_tx_absorb_raw(tx, "logup_m_rem", dg_rem, 32);
    Chal C;
    C.gamma = fp_tx_squeeze_one(tx, "logup_gamma");
    memcpy(proof + pos, hm + 4 * T, 4 * 65536);
    pos += 4 * 65536;
    fp_tx_absorb_raw(tx, "logup_m_clamp", dg_cl, 32);
    C.alpha0 = fp_tx_squeeze_one(tx, "logup_alpha");
    C.alpha1 = fp_tx_squeeze_one(tx, "logup_alpha");

    // ---- fraction trees (layers 1 .. v-1) ----
    std::vector<TreeLayer> lay(v + 1);
    for (int d = 1; d <= v - 1; d++)
        for (int tau = 0; tau < 2; tau++) {
            lay[d].P[tau] = (uint64_t*)fp_alloc(c->dev, (size_t)8 << d);
            lay[d].Q[tau] = (uint64_t*)fp_alloc(c->dev, (size_t)8 << d);
        }
    ulonglong2* leafq[2] = {nullptr, nullptr};
    if (v >= 2)
        for (int tau = 0; tau < 2; tau++) leafq[tau] = (ulonglong2*)fp_alloc(c->dev, (size_t)16 << (v - 2));
    uint64_t* E = (uint64_t*)fp_alloc(c->dev, (size_t)8 << (v >= 2 ? v - 2 : 0));
    uint64_t* part = (uint64_t*)fp_alloc(c->dev, (size_t)8 * 3 * 8 * c->num_sms);
    uint64_t* small = (uint64_t*)fp_alloc(c->dev, 256);  // [0..8) outputs, [16] state
    uint64_t* hsmall = (uint64_t*)fp_alloc(c->host, 256);
    if (!part || !small || !hsmall || !E) return fp_fail(c, FP_ERR_OOM, "logup: scratch exhausted");

    if (v >= 2) {
        int slot;
        const int64_t n = L / 2;
        fp_tic(c, st, K_TREE_LEAF, 9.0 * L + 32.0 * n, &slot);
        tree_leaf_kernel<<<grid_for(c, n, 256), 256, 0, st>>>(K, C, lay[v - 1], n);
        fp_toc(c, st, slot);
        FP_CUDA(c, cudaGetLastError());
        for (int d = v - 2; d >= 1; d--) {
            const int64_t nn = 1ll << d;
            fp_tic(c, st, K_TREE_UP, 64.0 * nn + 32.0 * nn, &slot);
            tree_up_kernel<<<grid_for(c, nn, 256), 256, 0, st>>>(lay[d + 1], lay[d], nn);
            fp_toc(c, st, slot);
            FP_CUDA(c, cudaGetLastError());
        }
        int s2;
        fp_tic(c, st, K_REDUCE, 64.0, &s2);
        l1_from_layer_kernel<<<1, 1, 0, st>>>(lay[1], small);
        fp_toc(c, st, s2);
    } else {
        int s2;
        fp_tic(c, st, K_REDUCE, 64.0, &s2);
        l1_from_keys_kernel<<<1, 1, 0, st>>>(K, C, small);
        fp_toc(c, st, s2);
    }
    FP_CUDA(c, cudaGetLastError());
    FP_CUDA(c, cudaMemcpyAsync(hsmall, small, 64, cudaMemcpyDeviceToHost, st));
    FP_CUDA(c, cudaStreamSynchronize(st));
    for (int i = 0; i < 8; i++) put_le(proof + pos + 8 * i, hsmall[i], 8);
    fp_tx_absorb_raw(tx, "gkr_l1", proof + pos, 64);
    pos += 64;
    FpPoint z;
    z.v = 1;
    z.z[0] = fp_tx_squeeze_one(tx, "gkr_mu");

    // ---- layer sum-checks ----
    for (int d = 1; d <= v - 1; d++) {
        const bool leaf = (d == v - 1);
        GkrArgs A;
        memset(&A, 0, sizeof A);
        for (int tau = 0; tau < 2; tau++) {
            if (leaf) {
                A.pp[tau] = nullptr;
                A.qq[tau] = leafq[tau];
            } else {
                A.pp[tau] = reinterpret_cast<ulonglong2*>(lay[d + 1].P[tau]);
                A.qq[tau] = reinterpret_cast<ulonglong2*>(lay[d + 1].Q[tau]);
            }
            A.src_pp[tau] = A.pp[tau];
            A.src_qq[tau] = A.qq[tau];
        }
        A.E = E;
        A.state = small + 16;
        A.keys = K;
        A.chal = C;
        A.z = z;
        A.d = d;
        A.lam = fp_tx_squeeze_one(tx, "gkr_lambda");
        std::vector<uint64_t> rho(d);
        uint64_t rprev = 0;
        for (int t = 1; t <= d; t++) {
            A.t = t;
            A.h = 1ll << (d - t);
            A.rprev = rprev;
            const int mode = t == 1 ? 0 : (t == 2 ? 1 : 2);
            const int blocks = grid_for(c, A.h, LU_THREADS);
            double bytes = (leaf ? 36.0 : 128.0) * A.h * (mode == 0 ? 1 : 2) + (mode ? 24.0 * A.h : 8.0 * A.h);
            int slot;
            fp_tic(c, st, K_GKR_ROUND, bytes, &slot);
            if (leaf) {
                if (mode == 0) gkr_round_kernel<true, true, 0><<<blocks, LU_THREADS, 0, st>>>(A, part, c->tickets, small);
                else if (mode == 1) gkr_round_kernel<true, true, 1><<<blocks, LU_THREADS, 0, st>>>(A, part, c->tickets, small);
                else gkr_round_kernel<true, false, 2><<<blocks, LU_THREADS, 0, st>>>(A, part, c->tickets, small);
            } else {
                if (mode == 0) gkr_round_kernel<false, false, 0><<<blocks, LU_THREADS, 0, st>>>(A, part, c->tickets, small);
                else if (mode == 1) gkr_round_kernel<false, false, 1><<<blocks, LU_THREADS, 0, st>>>(A, part, c->tickets, small);
                else gkr_round_kernel<false, false, 2><<<blocks, LU_THREADS, 0, st>>>(A, part, c->tickets, small);
            }
            fp_toc(c, st, slot);
            FP_CUDA(c, cudaGetLastError());
            FP_CUDA(c, cudaMemcpyAsync(hsmall, small, 32, cudaMemcpyDeviceToHost, st));
            FP_CUDA(c, cudaStreamSynchronize(st));
            for (int i = 0; i < 4; i++) put_le(proof + pos + 8 * i, hsmall[i], 8);
            fp_tx_absorb_raw(tx, "gkr_round", proof + pos, 32);
            pos += 32;
            rprev = rho[t - 1] = fp_tx_squeeze_one(tx, "gkr_chal");
        }
        int slot;
        fp_tic(c, st, K_GKR_FINAL, 128.0, &slot);
        if (leaf) {
            if (d == 1) gkr_final_kernel<true, true><<<1, 32, 0, st>>>(A, rprev, small);
            else gkr_final_kernel<true, false><<<1, 32, 0, st>>>(A, rprev, small);
        } else {
            gkr_final_kernel<false, false><<<1, 32, 0, st>>>(A, rprev, small);
        }
        fp_toc(c, st, slot);
        FP_CUDA(c, cudaGetLastError());
        FP_CUDA(c, cudaMemcpyAsync(hsmall, small, 64, cudaMemcpyDeviceToHost, st));
        FP_CUDA(c, cudaStreamSynchronize(st));
        for (int i = 0; i < 8; i++) put_le(proof + pos + 8 * i, hsmall[i], 8);
        fp_tx_absorb_raw(tx, "gkr_final", proof + pos, 64);
        pos += 64;
        const uint64_t mu = fp_tx_squeeze_one(tx, "gkr_mu");
        for (int t = 0; t < d; t++) z.z[t] = rho[t];
        z.z[d] = mu;
        z.v = d + 1;
    }

    // ---- leaf claims ----
    {
        const int hi_bits = v - lo_bits;
        uint64_t* ehi = (uint64_t*)fp_alloc(c->dev, (size_t)8 << hi_bits);
        uint64_t* elo = (uint64_t*)fp_alloc(c->dev, (size_t)8 << lo_bits);
        if (!ehi || !elo) return fp_fail(c, FP_ERR_OOM, "logup: scratch exhausted");
        FpPoint zh, zl;
        zh.v = hi_bits;
        zl.v = lo_bits;
        for (int i = 0; i < hi_bits; i++) zh.z[i] = z.z[i];
        for (int i = 0; i < lo_bits; i++) zl.z[i] = z.z[hi_bits + i];
        if ((rc = fp_eq_table(c, zh, ehi, st))) return rc;
        if ((rc = fp_eq_table(c, zl, elo, st))) return rc;
        int slot;
        fp_tic(c, st, K_LEAF_EVAL, 9.0 * nk, &slot);
        leaf_eval_kernel<<<grid_for(c, nk, LU_THREADS), LU_THREADS, 0, st>>>(K, ehi, elo, lo_bits, L, part, c->tickets,
                                                                             small);
        fp_toc(c, st, slot);
        FP_CUDA(c, cudaGetLastError());
        FP_CUDA(c, cudaMemcpyAsync(hsmall, small, 24, cudaMemcpyDeviceToHost, st));
        FP_CUDA(c, cudaStreamSynchronize(st));
        for (int i = 0; i < 3; i++) put_le(proof + pos + 8 * i, hsmall[i], 8);
        fp_tx_absorb_raw(tx, "leaf", proof + pos, 24);
        pos += 24;
    }
    *proof_len = pos;
    return n_outside ? FP_WARN_KEYS_OUTSIDE_TABLE : FP_OK;
}
