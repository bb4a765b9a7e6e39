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
// compute h(X) = sum_b eq(z_>t, b) F(., X, b) at X = 0 and 2 (and at 1 only when
// z_t = 0); the host forms g(X) = eq(z_<t, rho_<t) eq(z_t, X) h(X) (h has degree
// 2), taking g(1) from the running claim. The vectors are folded in place by the
// previous challenge in the same pass; the suffix eq table is kept in place too
// (E_t[b] = E_(t-1)[b] + E_(t-1)[b + h]).
#include <string.h>

#include <algorithm>
#include <vector>

#include "fp_eqchunks.cuh"
#include "fp_hist.cuh"
#include "fp_internal.h"
#include "fp_reduce.cuh"
#include "fp_session.cuh"

namespace {

// Launch shapes of the layer kernels (block threads; the blocks per SM the register budget is
// sized for). The leaf layer's kernel runs 512-thread blocks: its big rounds, read from the key
// columns, ran about 3% faster as one 512-thread block per SM than as two 256-thread blocks.
#ifndef FP_GKR_THREADS
#define FP_GKR_THREADS 256
#endif
#ifndef FP_GKR_MIN_BLOCKS
#define FP_GKR_MIN_BLOCKS 2
#endif
#ifndef FP_GKR_LEAF_THREADS
#define FP_GKR_LEAF_THREADS 512
#endif
#ifndef FP_GKR_LEAF_MIN_BLOCKS
#define FP_GKR_LEAF_MIN_BLOCKS 1
#endif
#ifndef FP_TREE_KEYS_MIN_BLOCKS
#define FP_TREE_KEYS_MIN_BLOCKS 3
#endif
constexpr int LU_THREADS = FP_GKR_THREADS;
constexpr int LU_LEAF_THREADS = FP_GKR_LEAF_THREADS;

using KeySrc = FpKeyCols;

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

// alpha - v for a canonical alpha and a signed 32-bit v, canonical
__device__ __forceinline__ uint64_t sub_i32(uint64_t alpha, int32_t v) {
    const uint64_t x = alpha - (uint64_t)(int64_t)v;
    if (v >= 0) return alpha >= (uint64_t)v ? x : x - GL_EPS;  // a borrow is worth + p
    return x >= GL_P ? x - GL_P : x;                            // alpha + |v| < 2^64
}

// alpha - v for a canonical alpha and a signed v with |v| < 2^62, canonical
__device__ __forceinline__ uint64_t sub_i64(uint64_t alpha, int64_t v) {
    if (v >= 0) {
        const uint64_t u = (uint64_t)v, x = alpha - u;
        return alpha >= u ? x : x - GL_EPS;
    }
    const uint64_t u = (uint64_t)(-v);
    uint64_t x = alpha + u;
    if (x < u) x += GL_EPS;  // the lost 2^64 is worth EPS; the sum is then alpha + u - p < u
    return x >= GL_P ? x - GL_P : x;
}

// Round 1 of the leaf layer sends, in place of h(2), the X^2 coefficient of h: the host takes
// h(2) = 2 h(1) - h(0) + 2 C2 (h has degree 2, h(1) from the running claim or the device). With
// leaves q = alpha - f and p = 1, the X^2 coefficient of a pair's F is
// lambda dL0 dR0 + lambda^3 dL1 dR1, d = q(1) - q(0): for the remainder table the integer
// r(0) - r(1), for the clamp table -((q'(1) - q'(0)) + gamma (y(1) - y(0))). So C2 needs no field
// product for the remainder table (an exact integer product below 2^64) and one for the clamp.
// e dL0 dR0 into ca, e dL1 dR1 into cb.
__device__ __forceinline__ void leaf_c2(uint64_t e, const int32_t (&r0)[2], const int32_t (&q0)[2],
                                        const int32_t (&y0)[2], const int32_t (&r1)[2], const int32_t (&q1)[2],
                                        const int32_t (&y1)[2], uint64_t gamma, GlAcc& ca, GlAcc& cb) {
    const int64_t dl = (int64_t)r0[0] - r1[0], dr = (int64_t)r0[1] - r1[1];
    const uint64_t u = (uint64_t)(uint32_t)(dl < 0 ? -dl : dl) * (uint32_t)(dr < 0 ? -dr : dr);
    const uint64_t uc = u >= GL_P ? u - GL_P : u;
    ca.mac(e, ((dl < 0) != (dr < 0)) ? gl_sub(0, uc) : uc);
    const uint64_t dL = sub_i64(gl_mul_small(gamma, y1[0] - y0[0]), (int64_t)q0[0] - q1[0]);
    const uint64_t dR = sub_i64(gl_mul_small(gamma, y1[1] - y0[1]), (int64_t)q0[1] - q1[1]);
    cb.mac(e, gl_mul_weak(dL, dR));
}

// lambda ca + lambda^3 cb as this thread's share of C2, in acc (cleared first)
__device__ __forceinline__ void leaf_c2_close(GlAcc& acc, const GlAcc& cb, uint64_t lam, uint64_t lam2) {
    const uint64_t a = acc.value(), b = cb.value();
    acc = GlAcc();
    acc.add(gl_mul(lam, gl_add(a, gl_mul(lam2, b))));
}

// leaf denominators alpha - f of key i for both tables
__device__ __forceinline__ void leaf_den(const KeySrc& K, const Chal& C, int64_t i, uint64_t& d0, uint64_t& d1) {
    int32_t r, q, y;
    key_at(K, i, r, q, y);
    d0 = sub_i32(C.alpha0, r);
    d1 = sub_i32(gl_sub(C.alpha1, gl_mul_small(C.gamma, y)), q);
}

// ytab[y + 128] = alpha1 - gamma y for every int8 y (one block fills it)
__device__ __forceinline__ void leaf_ytab_build(const Chal& C, uint64_t* ytab) {
    for (int j = threadIdx.x; j < 256; j += blockDim.x) ytab[j] = gl_sub(C.alpha1, gl_mul_small(C.gamma, j - 128));
}

// The layer sum-check's table: alpha1 - gamma y for y in [-384, 384) at index y + 384, which
// covers the int8 outputs and their extrapolations 2 y1 - y0 to the point X = 2
constexpr int kYWide = 768;
__device__ __forceinline__ void leaf_ytabw_build(const Chal& C, uint64_t* ytab) {
    for (int j = threadIdx.x; j < kYWide; j += blockDim.x) ytab[j] = gl_sub(C.alpha1, gl_mul_small(C.gamma, j - 384));
}

// keys 2x and 2x + 1 (one pair position of the leaf layer), with 8-byte loads of r and q and a
// 2-byte load of y when the columns allow it
__device__ __forceinline__ void key_pair(const KeySrc& K, bool vec, int64_t x, int32_t (&r)[2], int32_t (&q)[2],
                                         int32_t (&y)[2]) {
    const int64_t i = 2 * x;
    if (vec && i + 1 < K.n) {
        const int2 rv = __ldcg(reinterpret_cast<const int2*>(K.r + i));
        const int2 qv = __ldcg(reinterpret_cast<const int2*>(K.q + i));
        const unsigned short yv = __ldcg(reinterpret_cast<const unsigned short*>(K.y + i));
        r[0] = rv.x; r[1] = rv.y;
        q[0] = qv.x; q[1] = qv.y;
        y[0] = (int8_t)(yv & 0xFF);
        y[1] = (int8_t)(yv >> 8);
    } else {
        key_at(K, i, r[0], q[0], y[0]);
        key_at(K, i + 1, r[1], q[1], y[1]);
    }
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
    auto count = [&](int32_t rv, int32_t qv, int32_t yv) {
        const int64_t jr = (int64_t)rv + half;
        if (jr >= 0 && jr < T) {
            if (rem_in_smem)
                atomicAdd(&sr[jr], 1u);
            else
                atomicAdd(&m_rem[jr], 1u);
        } else {
            out_local++;
        }
        const int64_t q = qv;
        if (q >= -HIST_WIN && q < HIST_WIN)
            atomicAdd(&sq[q + HIST_WIN], 1u);
        else if (q >= -32768 && q < 32768)
            atomicAdd(&m_clamp[q + 32768], 1u);
        else
            out_local++;
        if (yv != (q < -128 ? -128 : (q > 127 ? 127 : (int32_t)q))) out_local++;
    };
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    int64_t done = 0;  // keys below this index are counted by the vector loop
    if (((uintptr_t)K.r | (uintptr_t)K.q) % 16 == 0 && (uintptr_t)K.y % 4 == 0) {
        // four keys per load (r, q as int4, y as one word), two groups in flight per iteration
        const int64_t ng = K.n / 4;
        const int4* r4 = reinterpret_cast<const int4*>(K.r);
        const int4* q4 = reinterpret_cast<const int4*>(K.q);
        const uint32_t* y4 = reinterpret_cast<const uint32_t*>(K.y);
        for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < ng; g += 2 * stride) {
            const bool two = g + stride < ng;
            const int4 ra = __ldcs(r4 + g), qa = __ldcs(q4 + g);
            const uint32_t ya = __ldcs(y4 + g);
            int4 rb = make_int4(0, 0, 0, 0), qb = rb;
            uint32_t yb = 0;
            if (two) {
                rb = __ldcs(r4 + g + stride);
                qb = __ldcs(q4 + g + stride);
                yb = __ldcs(y4 + g + stride);
            }
            count(ra.x, qa.x, (int8_t)(ya & 0xFF));
            count(ra.y, qa.y, (int8_t)((ya >> 8) & 0xFF));
            count(ra.z, qa.z, (int8_t)((ya >> 16) & 0xFF));
            count(ra.w, qa.w, (int8_t)(ya >> 24));
            if (two) {
                count(rb.x, qb.x, (int8_t)(yb & 0xFF));
                count(rb.y, qb.y, (int8_t)((yb >> 8) & 0xFF));
                count(rb.z, qb.z, (int8_t)((yb >> 16) & 0xFF));
                count(rb.w, qb.w, (int8_t)(yb >> 24));
            }
        }
        done = 4 * ng;
    }
    for (int64_t i = done + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < K.n; i += stride)
        count(K.r[i], K.q[i], (int32_t)K.y[i]);
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

// The same counts for remainder tables of 2^15 to 2^18 rows, too large for one block: a cluster
// of 2^(k-15) CTAs holds the table in distributed shared memory, 2^15 rows per CTA (each
// remainder counted on its owner's shared memory), next to a clamp window [-2^12, 2^12) of its
// own. Every cluster writes its remainder rows to part (row = cluster index, 2^k words) with
// plain stores; hist_rows_sum_kernel adds the rows (and the padding keys) into m_rem.
constexpr int HIST_CL_WIN = 1 << 12;

__global__ void __launch_bounds__(1024) hist_cluster_kernel(KeySrc K, int k, int64_t L, uint32_t* __restrict__ part,
                                                            uint32_t* __restrict__ m_clamp,
                                                            uint32_t* __restrict__ outside) {
    extern __shared__ uint32_t sh[];
    namespace cg = cooperative_groups;
    cg::cluster_group cl = cg::this_cluster();
    constexpr int SB = fp_hist::kShareBits;
    const unsigned crank = cl.block_rank(), csize = cl.num_blocks();
    uint32_t* sr = sh;               // remainder rows [crank 2^15, (crank + 1) 2^15)
    uint32_t* sq = sh + (1 << SB);   // 2 HIST_CL_WIN clamp rows around q = 0
    const int64_t T = 1ll << k;
    const int32_t half = 1 << (k - 1);
    for (int i = threadIdx.x; i < (1 << SB); i += blockDim.x) sr[i] = 0;
    for (int i = threadIdx.x; i < 2 * HIST_CL_WIN; i += blockDim.x) sq[i] = 0;
    cl.sync();  // every CTA's rows are zero before any CTA counts into them
    uint32_t out_local = 0;
    auto count = [&](int32_t rv, int32_t qv, int32_t yv) {
        const int64_t jr = (int64_t)rv + half;
        if (jr >= 0 && jr < T)
            atomicAdd(cl.map_shared_rank(sr, (unsigned)(jr >> SB)) + (jr & ((1 << SB) - 1)), 1u);
        else
            out_local++;
        const int64_t q = qv;
        if (q >= -HIST_CL_WIN && q < HIST_CL_WIN)
            atomicAdd(&sq[q + HIST_CL_WIN], 1u);
        else if (q >= -32768 && q < 32768)
            atomicAdd(&m_clamp[q + 32768], 1u);
        else
            out_local++;
        if (yv != (q < -128 ? -128 : (q > 127 ? 127 : (int32_t)q))) out_local++;
    };
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    int64_t done = 0;
    if (((uintptr_t)K.r | (uintptr_t)K.q) % 16 == 0 && (uintptr_t)K.y % 4 == 0) {
        const int64_t ng = K.n / 4;
        const int4* r4 = reinterpret_cast<const int4*>(K.r);
        const int4* q4 = reinterpret_cast<const int4*>(K.q);
        const uint32_t* y4 = reinterpret_cast<const uint32_t*>(K.y);
        for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < ng; g += stride) {
            const int4 ra = __ldcs(r4 + g), qa = __ldcs(q4 + g);
            const uint32_t ya = __ldcs(y4 + g);
            count(ra.x, qa.x, (int8_t)(ya & 0xFF));
            count(ra.y, qa.y, (int8_t)((ya >> 8) & 0xFF));
            count(ra.z, qa.z, (int8_t)((ya >> 16) & 0xFF));
            count(ra.w, qa.w, (int8_t)(ya >> 24));
        }
        done = 4 * ng;
    }
    for (int64_t i = done + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < K.n; i += stride)
        count(K.r[i], K.q[i], (int32_t)K.y[i]);
    if (out_local) atomicAdd(outside, out_local);
    cl.sync();  // every count has landed; no CTA leaves while another may still count into it
    uint32_t* row = part + (size_t)(blockIdx.x / csize) * (size_t)T + ((size_t)crank << SB);
    for (int i = threadIdx.x; i < (1 << SB); i += blockDim.x) row[i] = sr[i];
    for (int i = threadIdx.x; i < 2 * HIST_CL_WIN; i += blockDim.x)
        if (sq[i]) atomicAdd(&m_clamp[i - HIST_CL_WIN + 32768], sq[i]);
    if (blockIdx.x == 0 && threadIdx.x == 0) atomicAdd(&m_clamp[32768], (uint32_t)(L - K.n));
}

// remainder tables counted by hist_cluster_kernel, and the partial rows they may write (one
// per cluster; at most one cluster per SM)
constexpr int kHistClMinK = 15, kHistClMaxK = 18, kHistClMaxRows = 160;

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

// Up to kTreeLevels layers per launch. Block b takes 2^levels consecutive
// nodes of layer L0 (the leaves when KEYS, else a stored layer) and builds its
// subtree down to one node of layer L0 - levels in shared memory, writing
// every layer it passes to global memory. Parent of children 2x, 2x+1:
// (pL qR + pR qL, qL qR); at the leaves p = 1, so the first level is (qL + qR, qL qR).
constexpr int kTreeLevels = 10;

struct TreeOut {
    TreeLayer lay[kTreeLevels];  // lay[l]: layer L0 - 1 - l
};

template <bool KEYS>
__global__ void __launch_bounds__(512) tree_chunk_kernel(KeySrc K, Chal C, TreeLayer in, TreeOut out, int levels) {
    extern __shared__ uint64_t sm[];  // [2 buffers][4 values: P0 Q0 P1 Q1][n1]
    const int n1 = 1 << (levels - 1);
    uint64_t* buf[2] = {sm, sm + 4 * n1};
    for (int x = threadIdx.x; x < n1; x += blockDim.x) {
        const int64_t gx = (int64_t)blockIdx.x * n1 + x;
        uint64_t P[2], Q[2];
        if (KEYS) {
            uint64_t l0, l1, r0, r1;
            leaf_den(K, C, 2 * gx, l0, l1);
            leaf_den(K, C, 2 * gx + 1, r0, r1);
            P[0] = gl_add(l0, r0);
            Q[0] = gl_mul(l0, r0);
            P[1] = gl_add(l1, r1);
            Q[1] = gl_mul(l1, r1);
        } else {
#pragma unroll
            for (int tau = 0; tau < 2; tau++) {
                const ulonglong2 p = reinterpret_cast<const ulonglong2*>(in.P[tau])[gx];
                const ulonglong2 q = reinterpret_cast<const ulonglong2*>(in.Q[tau])[gx];
                P[tau] = gl_add(gl_mul(p.x, q.y), gl_mul(p.y, q.x));
                Q[tau] = gl_mul(q.x, q.y);
            }
        }
#pragma unroll
        for (int tau = 0; tau < 2; tau++) {
            out.lay[0].P[tau][gx] = P[tau];
            out.lay[0].Q[tau][gx] = Q[tau];
            buf[0][(2 * tau) * n1 + x] = P[tau];
            buf[0][(2 * tau + 1) * n1 + x] = Q[tau];
        }
    }
    for (int l = 1; l < levels; l++) {
        __syncthreads();
        const int nl = n1 >> l;
        const uint64_t* src = buf[(l - 1) & 1];
        uint64_t* dst = buf[l & 1];
        for (int x = threadIdx.x; x < nl; x += blockDim.x) {
            const int64_t gx = (int64_t)blockIdx.x * nl + x;
#pragma unroll
            for (int tau = 0; tau < 2; tau++) {
                const uint64_t pl = src[(2 * tau) * n1 + 2 * x], pr = src[(2 * tau) * n1 + 2 * x + 1];
                const uint64_t ql = src[(2 * tau + 1) * n1 + 2 * x], qr = src[(2 * tau + 1) * n1 + 2 * x + 1];
                const uint64_t P = gl_add(gl_mul(pl, qr), gl_mul(pr, ql)), Q = gl_mul(ql, qr);
                out.lay[l].P[tau][gx] = P;
                out.lay[l].Q[tau][gx] = Q;
                dst[(2 * tau) * n1 + x] = P;
                dst[(2 * tau + 1) * n1 + x] = Q;
            }
        }
    }
}

// The first twelve levels above the leaves (v - 1 .. v - 12) from the keys, for v >= 13. A block
// takes 4096-leaf chunks in turn: each thread builds the four levels above its 16 consecutive
// leaves in registers, each warp the next five by shuffles (a lane per node and table), and warp
// 0 the last three from the block's 8 warp nodes; every level is written as it is formed. The
// kernel is bound by the integer pipes, so the leaves' denominators take a branch-light
// subtraction and a parent's P one exact two-product sum and a single reduction.
constexpr int kKeyTreeLevels = 12;
constexpr int kKeyTreeThreads = 256;  // 16 leaves per thread: 4096 leaves per chunk

struct KeyTreeOut {
    TreeLayer lay[kKeyTreeLevels];  // lay[l]: level v - 1 - l
};

// (P, Q) of a parent from its children: (pL qR + pR qL, qL qR), canonical
__device__ __forceinline__ void tree_up(uint64_t pl, uint64_t ql, uint64_t pr, uint64_t qr, uint64_t& p, uint64_t& q) {
    GlAcc a;
    a.mac(pl, qr);
    a.mac(pr, ql);
    p = a.value();
    q = gl_mul(ql, qr);
}

// The four levels above a thread's 16 consecutive leaves in one table (v - 1 .. v - 4), each
// written as it is formed; the level v - 4 node is returned. One table at a time keeps the
// thread's live values to one table's keys and nodes.
template <int T>
__device__ __forceinline__ void key_subtree(const KeySrc& K, const Chal& C, const uint64_t* ytab, const KeyTreeOut& out,
                                            int64_t ch, int64_t leaf0, uint64_t& p4, uint64_t& q4) {
    uint64_t P[8], Q[8];
    if (leaf0 + 16 <= K.n) {
        int32_t k[16];  // r (table 0) or q (table 1)
        const int32_t* col = T == 0 ? K.r : K.q;
#pragma unroll
        for (int u = 0; u < 4; u++) {
            const int4 kv = __ldcs(reinterpret_cast<const int4*>(col + leaf0) + u);
            k[4 * u] = kv.x; k[4 * u + 1] = kv.y; k[4 * u + 2] = kv.z; k[4 * u + 3] = kv.w;
        }
        uint32_t yw[4] = {0, 0, 0, 0};
        if (T == 1) {
            const uint4 yv = __ldcs(reinterpret_cast<const uint4*>(K.y + leaf0));
            yw[0] = yv.x; yw[1] = yv.y; yw[2] = yv.z; yw[3] = yv.w;
        }
#pragma unroll
        for (int j = 0; j < 8; j++) {
            uint64_t a, b;
            if (T == 0) {
                a = sub_i32(C.alpha0, k[2 * j]);
                b = sub_i32(C.alpha0, k[2 * j + 1]);
            } else {
                const int ya = (int8_t)((yw[j >> 1] >> (16 * (j & 1))) & 0xFF);
                const int yb = (int8_t)((yw[j >> 1] >> (16 * (j & 1) + 8)) & 0xFF);
                a = sub_i32(ytab[ya + 128], k[2 * j]);
                b = sub_i32(ytab[yb + 128], k[2 * j + 1]);
            }
            P[j] = gl_add(a, b);
            Q[j] = gl_mul(a, b);
        }
    } else {
#pragma unroll
        for (int j = 0; j < 8; j++) {
            int32_t r0, q0, y0, r1, q1, y1;
            key_at(K, leaf0 + 2 * j, r0, q0, y0);
            key_at(K, leaf0 + 2 * j + 1, r1, q1, y1);
            const uint64_t a = T == 0 ? sub_i32(C.alpha0, r0) : sub_i32(ytab[y0 + 128], q0);
            const uint64_t b = T == 0 ? sub_i32(C.alpha0, r1) : sub_i32(ytab[y1 + 128], q1);
            P[j] = gl_add(a, b);
            Q[j] = gl_mul(a, b);
        }
    }
    // write level l's n (8, 4, 2, 1) consecutive nodes, then form level l + 1
#pragma unroll
    for (int l = 0; l < 4; l++) {
        const int n = 8 >> l;
        const int64_t g = (ch * 256 + threadIdx.x) * (int64_t)n;  // the thread's first node of level l
        if (n >= 2) {
#pragma unroll
            for (int j = 0; j < n; j += 2) {
                reinterpret_cast<ulonglong2*>(out.lay[l].P[T] + g)[j / 2] = make_ulonglong2(P[j], P[j + 1]);
                reinterpret_cast<ulonglong2*>(out.lay[l].Q[T] + g)[j / 2] = make_ulonglong2(Q[j], Q[j + 1]);
            }
#pragma unroll
            for (int j = 0; j < n / 2; j++) tree_up(P[2 * j], Q[2 * j], P[2 * j + 1], Q[2 * j + 1], P[j], Q[j]);
        } else {
            out.lay[l].P[T][g] = P[0];
            out.lay[l].Q[T][g] = Q[0];
        }
    }
    p4 = P[0];
    q4 = Q[0];
}

__global__ void __launch_bounds__(kKeyTreeThreads, FP_TREE_KEYS_MIN_BLOCKS) tree_keys_kernel(KeySrc K, Chal C, KeyTreeOut out, int64_t nchunks) {
    __shared__ uint64_t ytab[256];
    __shared__ uint64_t wnode[2][2][8];  // [table][P, Q][warp]: each warp's level v - 9 node
    // every node over padding keys only (the neutral key 0: leaf alpha0, and alpha1 - gamma 0) has
    // one value per level and table: [level][table][P, Q]
    __shared__ uint64_t padc[kKeyTreeLevels][2][2];
    leaf_ytab_build(C, ytab);
    __syncthreads();
    if (threadIdx.x < 2) {
        const int t = threadIdx.x;
        const uint64_t a = t == 0 ? sub_i32(C.alpha0, 0) : sub_i32(ytab[128], 0);
        uint64_t p = gl_add(a, a), q = gl_mul(a, a);
        for (int l = 0; l < kKeyTreeLevels; l++) {
            padc[l][t][0] = p;
            padc[l][t][1] = q;
            uint64_t np, nq;
            tree_up(p, q, p, q, np, nq);
            p = np;
            q = nq;
        }
    }
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int64_t ch = blockIdx.x; ch < nchunks; ch += gridDim.x) {
        if (ch * 4096 >= K.n) {
            // a chunk of padding only: every level's nodes are the level's constants (block-uniform)
#pragma unroll 1
            for (int l = 0; l < kKeyTreeLevels; l++) {
                const int nl = 2048 >> l;  // the chunk's nodes at level v - 1 - l
                const int64_t g0 = ch * nl;
#pragma unroll
                for (int t = 0; t < 2; t++)
                    for (int i = threadIdx.x; i < nl; i += blockDim.x) {
                        out.lay[l].P[t][g0 + i] = padc[l][t][0];
                        out.lay[l].Q[t][g0 + i] = padc[l][t][1];
                    }
            }
            continue;
        }
        const int64_t leaf0 = ch * 4096 + 16 * (int64_t)threadIdx.x;
        uint64_t P[2][1], Q[2][1];  // the thread's level v - 4 node per table
        key_subtree<0>(K, C, ytab, out, ch, leaf0, P[0][0], Q[0][0]);
        key_subtree<1>(K, C, ytab, out, ch, leaf0, P[1][0], Q[1][0]);
        // each lane now holds its level v - 4 node of both tables in P[t][0], Q[t][0]. Levels v - 5 ..
        // v - 9 in the warp: at level v - 5 lane L forms node x = L & 15 of table L >> 4 from lanes
        // 2x, 2x + 1; below, a level's items sit on lanes 0 .. 2 nl - 1, table-major
        uint64_t mp, mq;  // this lane's item of the current level
        {
            const int t = lane >> 4, x = lane & 15, src = 2 * x;
            const uint64_t pl0 = shfl_u64(P[0][0], src), ql0 = shfl_u64(Q[0][0], src);
            const uint64_t pr0 = shfl_u64(P[0][0], src + 1), qr0 = shfl_u64(Q[0][0], src + 1);
            const uint64_t pl1 = shfl_u64(P[1][0], src), ql1 = shfl_u64(Q[1][0], src);
            const uint64_t pr1 = shfl_u64(P[1][0], src + 1), qr1 = shfl_u64(Q[1][0], src + 1);
            tree_up(t ? pl1 : pl0, t ? ql1 : ql0, t ? pr1 : pr0, t ? qr1 : qr0, mp, mq);
            const int64_t g = (ch * 8 + warp) * 16 + x;
            out.lay[4].P[t][g] = mp;
            out.lay[4].Q[t][g] = mq;
        }
#pragma unroll
        for (int l = 5; l < 9; l++) {
            const int nl = 16 >> (l - 4);  // nodes per table of level v - 1 - l in the warp
            const int t = lane / nl, x = lane % nl;
            const int src = (t * 2 * nl + 2 * x) & 31;  // children: items 2x, 2x + 1 of table t one level down
            const uint64_t pl = shfl_u64(mp, src), ql = shfl_u64(mq, src);
            const uint64_t pr = shfl_u64(mp, src + 1), qr = shfl_u64(mq, src + 1);
            uint64_t np, nq;
            tree_up(pl, ql, pr, qr, np, nq);
            mp = np;
            mq = nq;
            if (lane < 2 * nl) {
                const int64_t g = (ch * 8 + warp) * (int64_t)nl + x;
                out.lay[l].P[t][g] = np;
                out.lay[l].Q[t][g] = nq;
            }
        }
        if (lane < 2) {  // lane t holds the warp's level v - 9 node of table t
            wnode[lane][0][warp] = mp;
            wnode[lane][1][warp] = mq;
        }
        __syncthreads();
        // levels v - 10 .. v - 12 from the 8 warp nodes per table, in warp 0 (item i = table i >> 3)
        if (warp == 0) {
            uint64_t bp = lane < 16 ? wnode[lane >> 3][0][lane & 7] : 0ull;
            uint64_t bq = lane < 16 ? wnode[lane >> 3][1][lane & 7] : 0ull;
#pragma unroll
            for (int l = 9; l < kKeyTreeLevels; l++) {
                const int nl = 8 >> (l - 8);
                const int t = lane / nl, x = lane % nl;
                const int src = (t * 2 * nl + 2 * x) & 31;
                const uint64_t pl = shfl_u64(bp, src), ql = shfl_u64(bq, src);
                const uint64_t pr = shfl_u64(bp, src + 1), qr = shfl_u64(bq, src + 1);
                uint64_t np, nq;
                tree_up(pl, ql, pr, qr, np, nq);
                bp = np;
                bq = nq;
                if (lane < 2 * nl) {
                    out.lay[l].P[t][ch * nl + x] = np;
                    out.lay[l].Q[t][ch * nl + x] = nq;
                }
            }
        }
        __syncthreads();  // wnode is rewritten by the next chunk
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

// ---- layer sum-check: one persistent kernel per layer ---------------------------------

struct GkrLayer {
    // pair vectors (x: left child, y: right child): rounds 1 and 2 read the children's level
    // (sp, sq), round 2 writes the folded halves to pp, qq, later rounds fold pp, qq in place.
    // pp == sp everywhere except in the layer above the leaf layer, which must leave its
    // children's level intact (the leaf layer's first round reads it) and folds into the leaf
    // layer's buffer instead. The leaf layer has no p vectors (all ones), reads its keys in
    // rounds 1 and 2 and folds its q pairs into a buffer.
    const ulonglong2* sp[2];
    const ulonglong2* sq[2];
    ulonglong2* pp[2];
    ulonglong2* qq[2];
    // leaf layer: the tree's level above the leaves, (dL + dR, dL dR) of every node per table
    const uint64_t* parP[2];
    const uint64_t* parQ[2];
    uint64_t* E;       // suffix eq table, kept in place
    KeySrc keys;
    int keys_vec;      // r, q 8-byte and y 2-byte aligned: key pairs by vector loads
    int piped;         // the leaf layer's rounds 1 and 2 stream their operands through the
                       // per-warp cp.async stages (16-byte aligned key columns)
    Chal chal;
    // Challenge points by layer parity: layer d reads its point from zin
    // (z_1..z_(d-1) = the previous layer's round challenges, z_d = mu written
    // by this layer's first launch) and writes its own round challenges to
    // zout, which is the next layer's zin. lam[0] keeps lambda for later launches.
    uint64_t* zin;
    uint64_t* zout;
    uint64_t* lam;
    int d;
    int threads;       // threads per block (<= LU_THREADS, LU_LEAF_THREADS in the leaf layer)
    int grid;          // blocks launched (all co-resident)
    int per_block;     // pairs one block covers in a round
    uint64_t seq0;     // {mu, lambda} arrive as challenge seq0; round t publishes seq0 + t
    int t_begin;       // rounds run by this launch: [t_begin, t_end]; t_end > d includes
    int t_end;         // the final values (one launch per layer, or one per round)
};

// F at one pair position for both tables: sum_tau lambda^(2 tau) (pL qR + pR qL + lambda qL qR),
// each table's term as pL qR + qL (pR + lambda qR) (qR + qL (1 + lambda qR) when p = 1),
// weakly reduced (it only feeds the product with the eq weight)
template <bool LEAF>
__device__ __forceinline__ uint64_t layer_F(const uint64_t (&pl)[2], const uint64_t (&pr)[2], const uint64_t (&ql)[2],
                                            const uint64_t (&qr)[2], uint64_t lam, uint64_t lam2) {
    uint64_t f[2];
#pragma unroll
    for (int tau = 0; tau < 2; tau++) {
        const uint64_t u = gl_add(LEAF ? 1ull : pr[tau], gl_mul_weak(lam, qr[tau]));
        f[tau] = gl_muladd_weak(ql[tau], u, LEAF ? qr[tau] : gl_mul_weak(pl[tau], qr[tau]));
    }
    return gl_muladd_weak(lam2, f[1], f[0]);
}

// pair x of the layer's vectors: before any fold (from_src) from the key columns or the
// children's level, afterwards from the fold buffers pp/qq
template <bool LEAF>
__device__ __forceinline__ void layer_pair(const GkrLayer& A, const uint64_t* ytab, bool from_src, int64_t x,
                                           ulonglong2 (&pp)[2], ulonglong2 (&qq)[2]) {
    if (LEAF && from_src) {
        int32_t r[2], q[2], y[2];
        key_pair(A.keys, A.keys_vec != 0, x, r, q, y);
        qq[0] = make_ulonglong2(sub_i32(A.chal.alpha0, r[0]), sub_i32(A.chal.alpha0, r[1]));
        qq[1] = make_ulonglong2(sub_i32(ytab[y[0] + 384], q[0]), sub_i32(ytab[y[1] + 384], q[1]));
        pp[0] = pp[1] = make_ulonglong2(1, 1);
    } else {
#pragma unroll
        for (int tau = 0; tau < 2; tau++) {
            pp[tau] = LEAF ? make_ulonglong2(1, 1) : __ldcg((from_src ? A.sp[tau] : A.pp[tau]) + x);
            qq[tau] = __ldcg((!LEAF && from_src ? A.sq[tau] : A.qq[tau]) + x);
        }
    }
}

__device__ __forceinline__ ulonglong2 fold2(ulonglong2 a, ulonglong2 b, uint64_t r) {
    return make_ulonglong2(gl_fold_fast(a.x, b.x, r), gl_fold_fast(a.y, b.y, r));
}

// F of a node of the level above the leaves from its stored (P, Q) = (dL + dR, dL dR):
// sum_tau lambda^(2 tau) (P + lambda Q), weakly reduced
__device__ __forceinline__ uint64_t parent_F(const GkrLayer& A, int64_t x, uint64_t lam, uint64_t lam2) {
    const uint64_t f0 = gl_muladd_weak(lam, __ldcg(A.parQ[0] + x), __ldcg(A.parP[0] + x));
    const uint64_t f1 = gl_muladd_weak(lam, __ldcg(A.parQ[1] + x), __ldcg(A.parP[1] + x));
    return gl_muladd_weak(lam2, f1, f0);
}

// The leaf layer's denominators at X = 2 of the pair positions (b, b + h): the children's keys
// on the line through b and b + h, 2 k(b + h) - k(b), formed in integers (alpha1 - gamma y for
// the extrapolated y from the wide table). ql, qr: left and right leaf, per table.
__device__ __forceinline__ void leaf_pair_at2(const GkrLayer& A, const uint64_t* ytab, int64_t b, int64_t h,
                                              uint64_t (&ql)[2], uint64_t (&qr)[2]) {
    int32_t r0[2], q0[2], y0[2], r1[2], q1[2], y1[2];
    key_pair(A.keys, A.keys_vec != 0, b, r0, q0, y0);
    key_pair(A.keys, A.keys_vec != 0, b + h, r1, q1, y1);
    uint64_t d[2][2];  // [leaf][table]
#pragma unroll
    for (int j = 0; j < 2; j++) {
        d[j][0] = sub_i64(A.chal.alpha0, 2 * (int64_t)r1[j] - r0[j]);
        d[j][1] = sub_i64(ytab[2 * y1[j] - y0[j] + 384], 2 * (int64_t)q1[j] - q0[j]);
    }
    ql[0] = d[0][0];
    ql[1] = d[0][1];
    qr[0] = d[1][0];
    qr[1] = d[1][1];
}

// ---- the leaf layer's rounds 1 and 2 through per-warp cp.async stages ------------------------
//
// Both rounds read their operands once, from places h pairs apart (the keys of pair positions b,
// b + h (and b + 2h, b + 3h), the level above the leaves or the eq table at b), with a few field
// products per pair: the warps are too few (one 512-thread block of 126 registers per SM) to hide
// the loads' latency by themselves. So each warp streams its 32-pair chunks through three
// shared-memory stages by cp.async, two chunks ahead of the one it computes on.
constexpr int kPipeStages = 3;
constexpr int kPipeStage = 1024 + 4 * 576;  // parents or eq (4 x 256 B), then 4 positions x (r, q, y of 64 keys)
constexpr int kPipeWarps = LU_LEAF_THREADS / 32;
constexpr size_t kPipeBytes = (size_t)kPipeWarps * kPipeStages * kPipeStage;

__device__ __forceinline__ void cp_async16_zfill(uint32_t dst, const void* src, int bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(bytes) : "memory");
}

// the keys of pair positions x0 .. x0 + 31 (64 keys from 2 x0) into a stage: r and q by 16 lanes
// each, y by 4 lanes; keys past the column's end read as zero
__device__ __forceinline__ void pipe_keys(const KeySrc& K, int64_t x0, uint32_t dst, int lane) {
    const int64_t i0 = 2 * x0;
    if (lane < 16) {
        const int64_t i = i0 + 4 * lane;
        const int64_t left = K.n - i;
        const int nb = left >= 4 ? 16 : (left > 0 ? (int)left * 4 : 0);
        cp_async16_zfill(dst + 16 * lane, nb ? (const void*)(K.r + i) : (const void*)K.r, nb);
    } else {
        const int64_t i = i0 + 4 * (lane - 16);
        const int64_t left = K.n - i;
        const int nb = left >= 4 ? 16 : (left > 0 ? (int)left * 4 : 0);
        cp_async16_zfill(dst + 256 + 16 * (lane - 16), nb ? (const void*)(K.q + i) : (const void*)K.q, nb);
    }
    if (lane < 4) {
        const int64_t i = i0 + 16 * lane;
        const int64_t left = K.n - i;
        const int nb = left >= 16 ? 16 : (left > 0 ? (int)left : 0);
        cp_async16_zfill(dst + 512 + 16 * lane, nb ? (const void*)(K.y + i) : (const void*)K.y, nb);
    }
}

// 32 consecutive 8-byte values from v + x0 into a stage slot (16 lanes, one 16-byte copy each)
__device__ __forceinline__ void pipe_u64x32(const uint64_t* v, int64_t x0, uint32_t dst, int l16) {
    cp_async16_zfill(dst + 16 * l16, v + x0 + 2 * l16, 16);
}

// issue chunk x0's copies for round t into stage address st
template <int T>
__device__ __forceinline__ void pipe_issue(const GkrLayer& A, int64_t x0, int64_t h, uint32_t st, int lane) {
    if (T == 1) {
        // the level above the leaves at x0: P of table 0 at 0, of table 1 at 256, Q at 512 and 768
        const int arr = lane >> 4, l16 = lane & 15;
        pipe_u64x32(arr == 0 ? A.parP[0] : A.parQ[0], x0, st + 512 * arr, l16);
        pipe_u64x32(arr == 0 ? A.parP[1] : A.parQ[1], x0, st + 256 + 512 * arr, l16);
        pipe_keys(A.keys, x0, st + 1024, lane);
        pipe_keys(A.keys, x0 + h, st + 1024 + 576, lane);
    } else {
        // the eq table at x0 and x0 + h, then the keys of four positions
        pipe_u64x32(A.E, x0 + (lane >> 4) * h, st + 256 * (lane >> 4), lane & 15);
#pragma unroll
        for (int p = 0; p < 4; p++) pipe_keys(A.keys, x0 + p * h, st + 1024 + 576 * p, lane);
    }
    asm volatile("cp.async.commit_group;\n" ::: "memory");
}

// keys 2 lane, 2 lane + 1 of position slot p of a stage
__device__ __forceinline__ void pipe_key_pair(const uint8_t* st, int p, int lane, int32_t (&r)[2], int32_t (&q)[2],
                                              int32_t (&y)[2]) {
    const uint8_t* kb = st + 1024 + 576 * p;
    const int2 rv = *reinterpret_cast<const int2*>(kb + 8 * lane);
    const int2 qv = *reinterpret_cast<const int2*>(kb + 256 + 8 * lane);
    const unsigned short yv = *reinterpret_cast<const unsigned short*>(kb + 512 + 2 * lane);
    r[0] = rv.x; r[1] = rv.y;
    q[0] = qv.x; q[1] = qv.y;
    y[0] = (int8_t)(yv & 0xFF);
    y[1] = (int8_t)(yv >> 8);
}

// Rounds 1 and 2 of the leaf layer by the stages (h >= 32: every chunk is 32 whole pairs).
template <int T>
__device__ __forceinline__ void leaf_round_piped(const GkrLayer& A, const uint64_t* ytab, uint8_t* pipe,
                                                 const EqChunks& EC, const uint64_t* eq_tab, int64_t h,
                                                 unsigned active, uint64_t rprev, uint64_t lam, uint64_t lam2,
                                                 bool need1, GlAcc (&acc)[3]) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    GlAcc c2b;  // round 1: the clamp table's share of C2
    uint8_t* wbuf = pipe + (size_t)warp * kPipeStages * kPipeStage;
    const uint32_t wsa = (uint32_t)__cvta_generic_to_shared(wbuf);
    const int64_t first = (int64_t)blockIdx.x * blockDim.x + 32 * warp, stride = (int64_t)active * blockDim.x;
    // prologue: chunks 0 .. kPipeStages - 2 in flight (an empty group keeps the count uniform)
#pragma unroll
    for (int i = 0; i < kPipeStages - 1; i++) {
        const int64_t x0 = first + i * stride;
        if (x0 < h)
            pipe_issue<T>(A, x0, h, wsa + i * kPipeStage, lane);
        else
            asm volatile("cp.async.commit_group;\n" ::: "memory");
    }
    int64_t x0 = first;
    for (int i = 0; x0 < h; i++, x0 += stride) {
        {
            const int64_t xn = x0 + (kPipeStages - 1) * stride;
            const int sn = (i + kPipeStages - 1) % kPipeStages;
            if (xn < h)
                pipe_issue<T>(A, xn, h, wsa + sn * kPipeStage, lane);
            else
                asm volatile("cp.async.commit_group;\n" ::: "memory");
        }
        asm volatile("cp.async.wait_group %0;\n" ::"n"(kPipeStages - 1) : "memory");
        __syncwarp();  // every lane's copies of chunk i have landed
        const uint8_t* st = wbuf + (i % kPipeStages) * kPipeStage;
        const int64_t b = x0 + lane;
        if (T == 1) {
            // X = 0 (and 1) from the level above the leaves; X = 2 from the keys extrapolated
            const uint64_t e = eq_chunks_at(EC, eq_tab, b);  // E_1[b] = eq(z_2..z_d, b)
            if (A.d > 1) A.E[b] = e;
            const uint64_t* pv = reinterpret_cast<const uint64_t*>(st);  // P0, P1, Q0, Q1: 32 each
            const uint64_t f0 = gl_muladd_weak(lam, pv[64 + lane], pv[lane]);
            const uint64_t f1 = gl_muladd_weak(lam, pv[96 + lane], pv[32 + lane]);
            acc[0].mac(e, gl_muladd_weak(lam2, f1, f0));
            if (need1) acc[2].mac(e, parent_F(A, b + h, lam, lam2));
            int32_t r0[2], q0[2], y0[2], r1[2], q1[2], y1[2];
            pipe_key_pair(st, 0, lane, r0, q0, y0);
            pipe_key_pair(st, 1, lane, r1, q1, y1);
            leaf_c2(e, r0, q0, y0, r1, q1, y1, A.chal.gamma, acc[1], c2b);
        } else {
            // fold positions (b, b + 2h) and (b + h, b + 3h) by the round-1 challenge
            uint64_t c0[2][2], c1[2][2];  // [table][leaf] at X = 0 (position b) and X = 1 (b + h)
#pragma unroll
            for (int half = 0; half < 2; half++) {
                int32_t ra[2], qa[2], ya[2], rb[2], qb[2], yb[2];
                pipe_key_pair(st, half, lane, ra, qa, ya);
                pipe_key_pair(st, half + 2, lane, rb, qb, yb);
                uint64_t (&c)[2][2] = half ? c1 : c0;
#pragma unroll
                for (int j = 0; j < 2; j++) {
                    c[0][j] = gl_fold_fast(sub_i32(A.chal.alpha0, ra[j]), sub_i32(A.chal.alpha0, rb[j]), rprev);
                    c[1][j] = gl_fold_fast(sub_i32(ytab[ya[j] + 384], qa[j]), sub_i32(ytab[yb[j] + 384], qb[j]), rprev);
                }
            }
#pragma unroll
            for (int tau = 0; tau < 2; tau++) {
                A.qq[tau][b] = make_ulonglong2(c0[tau][0], c0[tau][1]);
                A.qq[tau][b + h] = make_ulonglong2(c1[tau][0], c1[tau][1]);
            }
            const uint64_t* ev = reinterpret_cast<const uint64_t*>(st);
            const uint64_t e = gl_add(ev[lane], ev[32 + lane]);
            A.E[b] = e;
            uint64_t pl[2] = {1, 1}, pr[2] = {1, 1}, ql[2], qr[2];
#pragma unroll
            for (int tau = 0; tau < 2; tau++) {
                ql[tau] = c0[tau][0];
                qr[tau] = c0[tau][1];
            }
            acc[0].mac(e, layer_F<true>(pl, pr, ql, qr, lam, lam2));
            if (need1) {
#pragma unroll
                for (int tau = 0; tau < 2; tau++) {
                    ql[tau] = c1[tau][0];
                    qr[tau] = c1[tau][1];
                }
                acc[2].mac(e, layer_F<true>(pl, pr, ql, qr, lam, lam2));
            }
#pragma unroll
            for (int tau = 0; tau < 2; tau++) {
                ql[tau] = gl_add(gl_sub(c1[tau][0], c0[tau][0]), c1[tau][0]);
                qr[tau] = gl_add(gl_sub(c1[tau][1], c0[tau][1]), c1[tau][1]);
            }
            acc[1].mac(e, layer_F<true>(pl, pr, ql, qr, lam, lam2));
        }
        __syncwarp();  // the stage is refilled two chunks on
    }
    asm volatile("cp.async.wait_group 0;\n" ::: "memory");
    if (T == 1) leaf_c2_close(acc[1], c2b, lam, lam2);
}

// Round t of layer d over the pairs b < h handled by this block.
// t == 1: the vectors as they are. t >= 2: fold the previous round's vectors
// (length 4h) by rprev first and store the folded halves in place.
template <bool LEAF>
__device__ __forceinline__ void layer_round(const GkrLayer& A, const uint64_t* ytab, uint8_t* pipe, const EqChunks& EC,
                                            const uint64_t* eq_tab, int t,
                                            int64_t h, unsigned active, uint64_t rprev, uint64_t lam, uint64_t lam2,
                                            bool need1, GlAcc (&acc)[3]) {
    const bool from_keys = t <= 2;  // the unfolded vectors (keys or the children's level)
    if (LEAF && t <= 2 && A.piped && h >= 32) {
        if (t == 1)
            leaf_round_piped<1>(A, ytab, pipe, EC, eq_tab, h, active, rprev, lam, lam2, need1, acc);
        else
            leaf_round_piped<2>(A, ytab, pipe, EC, eq_tab, h, active, rprev, lam, lam2, need1, acc);
        return;
    }
    GlAcc c2b;  // the leaf layer's round 1: the clamp table's share of C2
    for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < h; b += (int64_t)active * blockDim.x) {
        if (LEAF && t == 1) {
            // X = 0 (and 1) from the stored level above the leaves; the X^2 coefficient C2 from
            // the keys' differences
            const uint64_t e = eq_chunks_at(EC, eq_tab, b);  // E_1[b] = eq(z_2..z_d, b)
            if (A.d > 1) A.E[b] = e;
            acc[0].mac(e, parent_F(A, b, lam, lam2));
            if (need1) acc[2].mac(e, parent_F(A, b + h, lam, lam2));
            int32_t r0[2], q0[2], y0[2], r1[2], q1[2], y1[2];
            key_pair(A.keys, A.keys_vec != 0, b, r0, q0, y0);
            key_pair(A.keys, A.keys_vec != 0, b + h, r1, q1, y1);
            leaf_c2(e, r0, q0, y0, r1, q1, y1, A.chal.gamma, acc[1], c2b);
            continue;
        }
        ulonglong2 c0p[2], c0q[2], c1p[2], c1q[2];
        uint64_t e;
        if (t == 1) {
            layer_pair<LEAF>(A, ytab, from_keys, b, c0p, c0q);
            layer_pair<LEAF>(A, ytab, from_keys, b + h, c1p, c1q);
            e = eq_chunks_at(EC, eq_tab, b);  // E_1[b] = eq(z_2..z_d, b)
            if (A.d > 1) A.E[b] = e;
        } else {
            ulonglong2 s0p[2], s0q[2], s1p[2], s1q[2], s2p[2], s2q[2], s3p[2], s3q[2];
            layer_pair<LEAF>(A, ytab, from_keys, b, s0p, s0q);
            layer_pair<LEAF>(A, ytab, from_keys, b + h, s1p, s1q);
            layer_pair<LEAF>(A, ytab, from_keys, b + 2 * h, s2p, s2q);
            layer_pair<LEAF>(A, ytab, from_keys, b + 3 * h, s3p, s3q);
#pragma unroll
            for (int tau = 0; tau < 2; tau++) {
                if (LEAF) {
                    c0p[tau] = c1p[tau] = make_ulonglong2(1, 1);
                } else {
                    c0p[tau] = fold2(s0p[tau], s2p[tau], rprev);
                    c1p[tau] = fold2(s1p[tau], s3p[tau], rprev);
                    A.pp[tau][b] = c0p[tau];
                    A.pp[tau][b + h] = c1p[tau];
                }
                c0q[tau] = fold2(s0q[tau], s2q[tau], rprev);
                c1q[tau] = fold2(s1q[tau], s3q[tau], rprev);
                A.qq[tau][b] = c0q[tau];
                A.qq[tau][b + h] = c1q[tau];
            }
            e = gl_add(__ldcg(A.E + b), __ldcg(A.E + b + h));
            A.E[b] = e;
        }
        // h(0) and h(2) always; h(1) only when z_t = 0 (otherwise the host takes it
        // from the running claim). Products with the eq weight are summed exactly.
        uint64_t pl[2], pr[2], ql[2], qr[2];
#pragma unroll
        for (int tau = 0; tau < 2; tau++) {
            pl[tau] = c0p[tau].x; pr[tau] = c0p[tau].y; ql[tau] = c0q[tau].x; qr[tau] = c0q[tau].y;
        }
        acc[0].mac(e, layer_F<LEAF>(pl, pr, ql, qr, lam, lam2));
        if (need1) {
#pragma unroll
            for (int tau = 0; tau < 2; tau++) {
                pl[tau] = c1p[tau].x; pr[tau] = c1p[tau].y; ql[tau] = c1q[tau].x; qr[tau] = c1q[tau].y;
            }
            acc[2].mac(e, layer_F<LEAF>(pl, pr, ql, qr, lam, lam2));
        }
#pragma unroll
        for (int tau = 0; tau < 2; tau++) {
            if (!LEAF) {
                pl[tau] = gl_add(gl_sub(c1p[tau].x, c0p[tau].x), c1p[tau].x);
                pr[tau] = gl_add(gl_sub(c1p[tau].y, c0p[tau].y), c1p[tau].y);
            }
            ql[tau] = gl_add(gl_sub(c1q[tau].x, c0q[tau].x), c1q[tau].x);
            qr[tau] = gl_add(gl_sub(c1q[tau].y, c0q[tau].y), c1q[tau].y);
        }
        acc[1].mac(e, layer_F<LEAF>(pl, pr, ql, qr, lam, lam2));
    }
    if (LEAF && t == 1) leaf_c2_close(acc[1], c2b, lam, lam2);
}

// The rest of a layer once one block holds all its pairs (h <= kTailPairs): the
// pair vectors move to shared memory (folded there by each new challenge) and
// each (pair, table, evaluation point) is its own task, so a round is a few
// short dependency chains per thread instead of one long one.
constexpr int kTailPairs = 128;

template <bool LEAF>
__device__ __forceinline__ void layer_tail(const GkrLayer& A, const uint64_t* ytab, const uint64_t* zs,
                                           const EqChunks& EC, const uint64_t* eq_tab, int t0, uint64_t rprev,
                                           uint64_t lam, uint64_t lam2, FpMailbox* mb, FpRelay* rl) {
    __shared__ uint64_t S[8][2 * kTailPairs];  // position x: p0L p0R q0L q0R p1L p1R q1L q1R
    __shared__ uint64_t Et[kTailPairs];
    const int d = A.d;
    int h = 1 << (d - t0);
    const bool from_keys = t0 <= 2;  // the unfolded vectors (keys or the children's level)
    for (int x = threadIdx.x; x < 2 * h; x += blockDim.x) {
        ulonglong2 pp[2], qq[2];
        layer_pair<LEAF>(A, ytab, from_keys, x, pp, qq);
        if (t0 > 1) {
            ulonglong2 p2[2], q2[2];
            layer_pair<LEAF>(A, ytab, from_keys, x + 2 * h, p2, q2);
#pragma unroll
            for (int tau = 0; tau < 2; tau++) {
                if (!LEAF) pp[tau] = fold2(pp[tau], p2[tau], rprev);
                qq[tau] = fold2(qq[tau], q2[tau], rprev);
            }
        }
#pragma unroll
        for (int tau = 0; tau < 2; tau++) {
            S[4 * tau + 0][x] = pp[tau].x;
            S[4 * tau + 1][x] = pp[tau].y;
            S[4 * tau + 2][x] = qq[tau].x;
            S[4 * tau + 3][x] = qq[tau].y;
        }
    }
    for (int b = threadIdx.x; b < h; b += blockDim.x)
        Et[b] = t0 == 1 ? eq_chunks_at(EC, eq_tab, b) : gl_add(__ldcg(A.E + b), __ldcg(A.E + b + h));
    __syncthreads();
    for (int t = t0; t <= d; t++) {
        if (t > t0) {
            if (!session_wait(mb, rl, A.seq0 + t - 1, rprev)) return;
            if (threadIdx.x == 0) A.zout[t - 2] = rprev;
            h >>= 1;
            // fold the most significant position bit: x < 2h takes x + 2h (p stays 1 on the leaf layer)
            for (int i = threadIdx.x; i < 8 * 2 * h; i += blockDim.x) {
                const int c = i / (2 * h), x = i - c * (2 * h);
                if (LEAF && (c & 2) == 0) continue;
                S[c][x] = gl_fold_fast(S[c][x], S[c][x + 2 * h], rprev);
            }
            for (int b = threadIdx.x; b < h; b += blockDim.x) Et[b] = gl_add(Et[b], Et[b + h]);
            __syncthreads();
        }
        const int nx = zs[t - 1] == 0 ? 3 : 2;  // X = 0, 2 (and 1 when z_t = 0)
        GlAcc acc0, acc2, acc1;  // by evaluation point (separate variables: no dynamic indexing)
        for (int task = threadIdx.x; task < h * 2 * nx; task += blockDim.x) {
            const int b = task % h, rest = task / h, tau = rest & 1, xi = rest >> 1;
            uint64_t v[4];
#pragma unroll
            for (int k = 0; k < 4; k++) {
                const uint64_t c0 = S[4 * tau + k][b], c1 = S[4 * tau + k][b + h];
                v[k] = xi == 0 ? c0 : xi == 1 ? gl_add(gl_sub(c1, c0), c1) : c1;
            }
            // v = pL, pR, qL, qR at X
            uint64_t f;
            if (LEAF && t == 1 && xi == 1) {
                // the leaf layer's round 1 sends C2: lambda (qL(1) - qL(0)) (qR(1) - qR(0))
                const uint64_t dl = gl_sub(S[4 * tau + 2][b + h], S[4 * tau + 2][b]);
                const uint64_t dr = gl_sub(S[4 * tau + 3][b + h], S[4 * tau + 3][b]);
                f = gl_mul_weak(lam, gl_mul(dl, dr));
            } else {
                const uint64_t u = gl_add(LEAF ? 1ull : v[1], gl_mul_weak(lam, v[3]));
                f = gl_muladd_weak(v[2], u, LEAF ? v[3] : gl_mul_weak(v[0], v[3]));
            }
            if (tau) f = gl_mul_weak(lam2, f);
            if (xi == 0)
                acc0.mac(Et[b], f);
            else if (xi == 1)
                acc2.mac(Et[b], f);
            else
                acc1.mac(Et[b], f);
        }
        uint64_t out[3] = {acc0.value(), acc2.value(), acc1.value()};
        block_sum_gl<3>(out);
        if (threadIdx.x == 0) session_publish(mb, out, A.seq0 + t);
    }
    if (!session_wait(mb, rl, A.seq0 + d, rprev)) return;
    if (threadIdx.x == 0) {
        A.zout[d - 1] = rprev;
        uint64_t out[8];
#pragma unroll
        for (int c = 0; c < 8; c++) out[c] = gl_fold(S[c][0], S[c][1], rprev);
        session_publish(mb, out, A.seq0 + d + 1);
    }
}

// Rounds [t_begin, t_end] of one layer (t_end > d: and its final child values).
template <bool LEAF>
__global__ void __launch_bounds__(LEAF ? LU_LEAF_THREADS : LU_THREADS, LEAF ? FP_GKR_LEAF_MIN_BLOCKS : FP_GKR_MIN_BLOCKS) gkr_layer_kernel(GkrLayer A, FpMailbox* mb, FpRelay* rl, uint64_t* part) {
    __shared__ uint64_t zs[32];
    __shared__ uint64_t s_lam;
    __shared__ uint64_t eq_tab[3 << kEqChunk];
    extern __shared__ __align__(16) uint64_t gkr_dyn_smem[];  // the leaf layer's wide y table, then its stages
    uint64_t* ytab = gkr_dyn_smem;
    uint8_t* pipe = reinterpret_cast<uint8_t*>(gkr_dyn_smem + kYWide);
    const int d = A.d;
    if (LEAF) leaf_ytabw_build(A.chal, ytab);  // visible after the first barrier below
    if (A.t_begin == 1) {
        // the layer's own challenges: mu (last point coordinate) and lambda
        uint64_t mu, lam;
        if (!session_wait2(mb, rl, A.seq0, mu, lam)) return;
        if (threadIdx.x == 0) {
            for (int i = 0; i < d - 1; i++) zs[i] = __ldcg(A.zin + i);
            zs[d - 1] = mu;
            s_lam = lam;
            if (blockIdx.x == 0) {
                A.zin[d - 1] = mu;
                A.lam[0] = lam;
            }
        }
    } else if (threadIdx.x == 0) {
        for (int i = 0; i < d; i++) zs[i] = __ldcg(A.zin + i);
        s_lam = __ldcg(A.lam);
    }
    __syncthreads();
    const uint64_t lam = s_lam, lam2 = gl_mul(lam, lam);
    uint64_t rprev = 0;
    for (int t = A.t_begin; t <= d && t <= A.t_end; t++) {
        if (t > 1) {
            if (!session_wait(mb, rl, A.seq0 + t - 1, rprev)) return;
            if (blockIdx.x == 0 && threadIdx.x == 0) A.zout[t - 2] = rprev;
        }
        const int64_t h = 1ll << (d - t);
        int64_t want = (h + A.per_block - 1) / A.per_block;
        const unsigned active = (unsigned)(want < 1 ? 1 : (want > A.grid ? A.grid : want));
        if (blockIdx.x >= active) return;  // this block has no pairs in this or any later round
        EqChunks EC{0, 0, 0};
        if (t == 1) EC = eq_chunks_build(eq_tab, zs, d);
        if (active == 1 && h <= kTailPairs && A.t_end > d) {
            // one block left, and this launch runs to the end of the layer
            layer_tail<LEAF>(A, ytab, zs, EC, eq_tab, t, rprev, lam, lam2, mb, rl);
            return;
        }
        GlAcc sums[3];
        layer_round<LEAF>(A, ytab, pipe, EC, eq_tab, t, h, active, rprev, lam, lam2, zs[t - 1] == 0, sums);
        uint64_t acc[3] = {sums[0].value(), sums[1].value(), sums[2].value()};
        bool last;
        if (active == 1) {
            block_sum_gl<3>(acc);
            last = true;
        } else {
            last = grid_sum_gl_n<3>(acc, part, &rl->ticket, active);
        }
        // {h(0), h(2), h(1) or 0} of h(X) = sum_b eq(z_>t, b) F(rho_<t, X, b); the host
        // forms g(X) = eq(z_<t, rho_<t) eq(z_t, X) h(X)
        if (last && threadIdx.x == 0) session_publish(mb, acc, A.seq0 + t);
    }
    // only block 0 is left: fold the last pair by the last challenge
    if (A.t_end <= d || blockIdx.x != 0) return;
    if (!session_wait(mb, rl, A.seq0 + d, rprev)) return;
    if (threadIdx.x == 0) {
        A.zout[d - 1] = rprev;
        ulonglong2 p0[2], q0[2], p1[2], q1[2];
        layer_pair<LEAF>(A, ytab, d == 1, 0, p0, q0);  // a one-round layer never folded
        layer_pair<LEAF>(A, ytab, d == 1, 1, p1, q1);
        uint64_t out[8];
#pragma unroll
        for (int tau = 0; tau < 2; tau++) {
            out[4 * tau + 0] = gl_fold(p0[tau].x, p1[tau].x, rprev);
            out[4 * tau + 1] = gl_fold(p0[tau].y, p1[tau].y, rprev);
            out[4 * tau + 2] = gl_fold(q0[tau].x, q1[tau].x, rprev);
            out[4 * tau + 3] = gl_fold(q0[tau].y, q1[tau].y, rprev);
        }
        session_publish(mb, out, 8, A.seq0 + d + 1);
    }
}

// ---- leaf claims: MLEs of the key columns at z (split eq: hi x lo) ----------------

// Leaf claims: the MLEs of the padded key columns at z, sum_x eq(z, x) f(x) with the eq split
// as eq_hi[x >> lo] eq_lo[x & (2^lo - 1)]. A block takes groups of 2^lo consecutive keys in turn
// (eq_hi constant within one): each thread sums eq_lo[.] (f + off) exactly over its keys of the
// group (64 x 32-bit products, f + off >= 0: off = 2^31 for r and q, 128 for y), removes
// off sum eq_lo, and weights the group's value by eq_hi once. Padding keys are 0 and add nothing.
__global__ void __launch_bounds__(LU_THREADS) leaf_eval_kernel(KeySrc K, const uint64_t* __restrict__ ehi,
                                                               const uint64_t* __restrict__ elo, int lo_bits,
                                                               uint64_t* part, unsigned int* ticket,
                                                               uint64_t* __restrict__ out) {
    const int64_t G = 1ll << lo_bits;
    const int64_t ngroups = (K.n + G - 1) >> lo_bits;
    const bool vec = lo_bits >= 2 && ((uintptr_t)K.r | (uintptr_t)K.q | (uintptr_t)elo) % 16 == 0 && (uintptr_t)K.y % 4 == 0;
    GlAcc tot[3];
    for (int64_t g = blockIdx.x; g < ngroups; g += gridDim.x) {
        const int64_t x0 = g << lo_bits;
        const int64_t xe = x0 + G < K.n ? x0 + G : K.n;
        GlAcc a[3], es;
        auto key = [&](uint64_t e, int32_t rv, int32_t qv, int32_t yv) {
            a[0].mac32(e, (uint32_t)rv ^ 0x80000000u);
            a[1].mac32(e, (uint32_t)qv ^ 0x80000000u);
            a[2].mac32(e, (uint32_t)(yv + 128));
            es.add(e);
        };
        int64_t xs = x0;  // keys from here on by the scalar loop
        if (vec) {
            // quads of keys (r, q as int4, y as one word, the weights as two 16-byte loads), two in flight
            const int64_t xq = x0 + ((xe - x0) & ~3ll);
            const int64_t step = 4 * (int64_t)blockDim.x;
            for (int64_t x = x0 + 4 * threadIdx.x; x < xq; x += 2 * step) {
                const bool two = x + step < xq;
                const int4 ra = __ldcs(reinterpret_cast<const int4*>(K.r + x));
                const int4 qa = __ldcs(reinterpret_cast<const int4*>(K.q + x));
                const uint32_t ya = __ldcs(reinterpret_cast<const uint32_t*>(K.y + x));
                const ulonglong2 ea0 = __ldg(reinterpret_cast<const ulonglong2*>(elo + (x - x0)));
                const ulonglong2 ea1 = __ldg(reinterpret_cast<const ulonglong2*>(elo + (x - x0) + 2));
                int4 rb = make_int4(0, 0, 0, 0), qb = rb;
                uint32_t yb = 0;
                ulonglong2 eb0 = make_ulonglong2(0, 0), eb1 = eb0;
                if (two) {
                    rb = __ldcs(reinterpret_cast<const int4*>(K.r + x + step));
                    qb = __ldcs(reinterpret_cast<const int4*>(K.q + x + step));
                    yb = __ldcs(reinterpret_cast<const uint32_t*>(K.y + x + step));
                    eb0 = __ldg(reinterpret_cast<const ulonglong2*>(elo + (x + step - x0)));
                    eb1 = __ldg(reinterpret_cast<const ulonglong2*>(elo + (x + step - x0) + 2));
                }
                key(ea0.x, ra.x, qa.x, (int8_t)(ya & 0xFF));
                key(ea0.y, ra.y, qa.y, (int8_t)((ya >> 8) & 0xFF));
                key(ea1.x, ra.z, qa.z, (int8_t)((ya >> 16) & 0xFF));
                key(ea1.y, ra.w, qa.w, (int8_t)(ya >> 24));
                if (two) {
                    key(eb0.x, rb.x, qb.x, (int8_t)(yb & 0xFF));
                    key(eb0.y, rb.y, qb.y, (int8_t)((yb >> 8) & 0xFF));
                    key(eb1.x, rb.z, qb.z, (int8_t)((yb >> 16) & 0xFF));
                    key(eb1.y, rb.w, qb.w, (int8_t)(yb >> 24));
                }
            }
            xs = xq;
        }
        for (int64_t x = xs + threadIdx.x; x < xe; x += blockDim.x) key(__ldg(elo + (x - x0)), K.r[x], K.q[x], K.y[x]);
        const uint64_t esum = es.value(), eh = __ldg(ehi + g);
        const uint64_t off[3] = {1ull << 31, 1ull << 31, 128ull};
#pragma unroll
        for (int i = 0; i < 3; i++) tot[i].mac(eh, gl_sub(a[i].value(), gl_mul(off[i], esum)));
    }
    uint64_t acc[3] = {tot[0].value(), tot[1].value(), tot[2].value()};
    if (grid_sum_gl<3>(acc, part, ticket) && threadIdx.x == 0) {
        out[0] = acc[0];
        out[1] = acc[1];
        out[2] = acc[2];
    }
}

// Algorithmic bytes of round t of a layer with h pairs: the pair vectors
// (p and q of both tables, 16 B per pair entry; the leaf layer has only q and
// reads its first two rounds from the keys, 9 B per key, and in round 1 the
// stored level above the leaves, 32 B per node), read at 2 (t = 1) or 4
// positions and written at 2, plus the suffix eq table.
double gkr_round_bytes(bool leaf, int t, double h) {
    const double entry = leaf ? 32.0 : 64.0;  // one position of all pair vectors
    // the leaf layer's round 1 reads the four children's keys and the stored parent of b
    if (t == 1) return (leaf ? 4 * 9.0 + 32.0 : 2 * entry) * h + 8.0 * h;
    if (leaf && t == 2) return 8 * 9.0 * h + 2 * entry * h + 24.0 * h;
    return 4 * entry * h + 2 * entry * h + 24.0 * h;
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

size_t fp_lookup_keys_scratch(int nsites, int64_t nk) {
    return nsites > 1 ? fp_align_up(9 * (size_t)nk + 1024, 256) + fp_align_up(sizeof(GatherSite) * nsites, 256) : 0;
}

int fp_lookup_keys(fp_ctx* c, const fp_site* sites, int nsites, cudaStream_t st, FpKeyCols* K) {
    int64_t nk = 0;
    for (int s = 0; s < nsites; s++) nk += (int64_t)sites[s].M * sites[s].N;
    K->n = nk;
    // the sites' columns already back to back in site order (one site, or buffers laid out so):
    // read in place, no copy
    bool in_place = true;
    int64_t off = 0;
    for (int s = 0; s < nsites && in_place; s++) {
        in_place = sites[s].q == sites[0].q + off && sites[s].r == sites[0].r + off && sites[s].y == sites[0].y + off;
        off += (int64_t)sites[s].M * sites[s].N;
    }
    if (in_place) {
        K->r = sites[0].r;
        K->q = sites[0].q;
        K->y = sites[0].y;
        return FP_OK;
    }
    int32_t* r = (int32_t*)fp_alloc(c->dev, 4 * (size_t)nk);
    int32_t* q = (int32_t*)fp_alloc(c->dev, 4 * (size_t)nk);
    int8_t* y = (int8_t*)fp_alloc(c->dev, (size_t)nk);
    GatherSite* dgs = (GatherSite*)fp_alloc(c->dev, sizeof(GatherSite) * nsites);
    GatherSite* hgs = (GatherSite*)fp_alloc(c->host, sizeof(GatherSite) * nsites);
    if (!r || !q || !y || !dgs || !hgs) return fp_fail(c, FP_ERR_OOM, "lookup keys: scratch exhausted");
    off = 0;
    for (int s = 0; s < nsites; s++) {
        hgs[s] = GatherSite{sites[s].q, sites[s].r, sites[s].y, off};
        off += (int64_t)sites[s].M * sites[s].N;
    }
    FP_CUDA(c, cudaMemcpyAsync(dgs, hgs, sizeof(GatherSite) * nsites, cudaMemcpyHostToDevice, st));
    int slot;
    fp_tic(c, st, K_KEYS_GATHER, 18.0 * nk, &slot);
    gather_kernel<<<grid_for(c, nk, 256), 256, 0, st>>>(dgs, nsites, nk, r, q, y);
    fp_toc(c, st, slot);
    FP_CUDA(c, cudaGetLastError());
    K->r = r;
    K->q = q;
    K->y = y;
    return FP_OK;
}

size_t fp_lookup_mults_scratch(int k) {
    size_t b = fp_align_up(4 * ((size_t)1 << k), 256) + fp_align_up(4 * 65536, 256) + 256;
    if (k >= kHistClMinK && k <= kHistClMaxK) b += fp_align_up((size_t)4 * (kHistClMaxRows << fp_hist::kShareBits), 256);
    return b;
}

int fp_lookup_mults(fp_ctx* c, const FpKeyCols& K, int k, int64_t L, cudaStream_t st, uint8_t* hm, uint8_t dg_rem[32],
                    uint8_t dg_cl[32]) {
    const int64_t T = 1ll << k;
    int rc;
    uint32_t* m_rem = (uint32_t*)fp_alloc(c->dev, 4 * (size_t)T);
    uint32_t* m_cl = (uint32_t*)fp_alloc(c->dev, 4 * 65536);
    uint32_t* outside = (uint32_t*)fp_alloc(c->dev, 256);
    if (!m_rem || !m_cl || !outside || !hm) return fp_fail(c, FP_ERR_OOM, "lookup multiplicities: scratch exhausted");
    FP_CUDA(c, cudaMemsetAsync(m_rem, 0, 4 * (size_t)T, st));
    FP_CUDA(c, cudaMemsetAsync(m_cl, 0, 4 * 65536, st));
    FP_CUDA(c, cudaMemsetAsync(outside, 0, 4, st));
    bool counted = false;
    if (k >= kHistClMinK && k <= kHistClMaxK) {
        // the remainder table over a cluster's shared memory (2^(k-15) CTAs of 2^15 rows)
        const int csize = 1 << (k - fp_hist::kShareBits);
        const size_t rows_bytes = (size_t)4 * (kHistClMaxRows << fp_hist::kShareBits);
        uint32_t* part = (uint32_t*)fp_alloc(c->dev, rows_bytes);
        if (!part) return fp_fail(c, FP_ERR_OOM, "lookup multiplicities: scratch exhausted");
        const int smem = 4 * ((1 << fp_hist::kShareBits) + 2 * HIST_CL_WIN);
        int clusters = 0, slot;
        fp_tic(c, st, K_HIST, 9.0 * K.n, &slot);
        if (fp_hist::launch_clusters(hist_cluster_kernel, csize, smem, kHistClMaxRows / csize, st, &clusters, K, k, L,
                                     part, m_cl, outside) == cudaSuccess) {
            fp_hist::hist_rows_sum_kernel<<<fp_grid256(c, T), 256, 0, st>>>(part, clusters, T, m_rem, T / 2,
                                                                            (uint32_t)(L - K.n));
            c->launches++;
            counted = true;
        } else {
            (void)cudaGetLastError();  // no cluster of that size fits here: the global-atomic path below
        }
        fp_toc(c, st, slot);
        FP_CUDA(c, cudaGetLastError());
    }
    if (!counted) {
        const int rem_smem = T <= 16384;
        const int smem = 4 * (2 * HIST_WIN) + (rem_smem ? 4 * (int)T : 0);
        FP_CUDA(c, cudaFuncSetAttribute(hist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
        int slot;
        fp_tic(c, st, K_HIST, 9.0 * K.n, &slot);
        hist_kernel<<<c->num_sms, 1024, smem, st>>>(K, k, L, m_rem, m_cl, outside, rem_smem);
        fp_toc(c, st, slot);
        FP_CUDA(c, cudaGetLastError());
    }
    FP_CUDA(c, cudaMemcpyAsync(hm, m_rem, 4 * (size_t)T, cudaMemcpyDeviceToHost, st));
    FP_CUDA(c, cudaMemcpyAsync(hm + 4 * T, m_cl, 4 * 65536, cudaMemcpyDeviceToHost, st));
    FP_CUDA(c, cudaMemcpyAsync(hm + 4 * T + 4 * 65536, outside, 4, cudaMemcpyDeviceToHost, st));
    FpDigestJob jobs[2] = {{(const uint8_t*)m_rem, 4 * (uint64_t)T}, {(const uint8_t*)m_cl, 4 * 65536ull}};
    uint8_t both[64];
    if ((rc = fp_digest_many(c, jobs, 2, both, st))) return rc;  // synchronises the stream
    memcpy(dg_rem, both, 32);
    memcpy(dg_cl, both + 32, 32);
    return FP_OK;
}

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
    size_t need = fp_lookup_keys_scratch(nsites, nk) + fp_lookup_mults_scratch(k);
    size_t tree = 0;
    for (int d = 1; d <= v - 1; d++) tree += 4 * fp_align_up((size_t)8 << d, 256);
    need += tree;
    if (v >= 2) need += 2 * fp_align_up((size_t)16 << (v - 2), 256);          // leaf-layer fold buffers
    need += fp_align_up((size_t)8 << (v >= 2 ? v - 2 : 0), 256);              // suffix eq table
    const int lo_bits = v / 2;
    need += fp_align_up((size_t)8 << lo_bits, 256) + fp_align_up((size_t)8 << (v - lo_bits), 256);
    need += fp_align_up((size_t)8 * 3 * 16 * c->num_sms, 256) + 3 * 512 + 8192;
    if ((rc = fp_reserve(c, c->dev, need + (1 << 20)))) return rc;
    if ((rc = fp_reserve(c, c->host, 4 * (size_t)T + 4 * 65536 + 4096 + sizeof(GatherSite) * nsites))) return rc;
    fp_reset(c->dev);
    fp_reset(c->host);

    // ---- keys, multiplicities ----
    KeySrc K;
    if ((rc = fp_lookup_keys(c, sites, nsites, st, &K))) return rc;
    uint8_t* hm = (uint8_t*)fp_alloc(c->host, 4 * (size_t)T + 4 * 65536 + 256);
    uint8_t dg_rem[32], dg_cl[32];
    if ((rc = fp_lookup_mults(c, K, k, L, st, hm, dg_rem, dg_cl))) return rc;
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
    uint64_t* part = (uint64_t*)fp_alloc(c->dev, (size_t)8 * 3 * 16 * c->num_sms);
    uint64_t* small = (uint64_t*)fp_alloc(c->dev, 256);  // [0..8) outputs
    uint64_t* zb[3] = {(uint64_t*)fp_alloc(c->dev, 8 * 64), (uint64_t*)fp_alloc(c->dev, 8 * 64),
                       (uint64_t*)fp_alloc(c->dev, 8 * 64)};
    uint64_t* hsmall = (uint64_t*)fp_alloc(c->host, 256);
    if (!part || !small || !hsmall || !E || !zb[2]) return fp_fail(c, FP_ERR_OOM, "logup: scratch exhausted");

    if (v >= 2) {
        // layers v-1 .. 1: the first twelve from the keys in one persistent launch (v >= 13), the
        // rest kTreeLevels per launch
        int L0 = v;
        // the vector loads of 16 keys need 16-byte aligned key columns
        const bool keys_aligned = (uintptr_t)K.r % 16 == 0 && (uintptr_t)K.q % 16 == 0 && (uintptr_t)K.y % 16 == 0;
        if (v >= kKeyTreeLevels + 1 && keys_aligned) {
            KeyTreeOut ko;
            for (int l = 0; l < kKeyTreeLevels; l++) ko.lay[l] = lay[v - 1 - l];
            const int64_t nchunks = (1ll << v) / 4096;
            int occ_t = 0;
            FP_CUDA(c, cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ_t, tree_keys_kernel, kKeyTreeThreads, 0));
            const unsigned blocks = (unsigned)std::min<int64_t>(nchunks, (int64_t)std::max(1, occ_t) * c->num_sms);
            const double nodes = (double)(1ll << v) - (double)(1ll << (v - kKeyTreeLevels));
            int slot;
            fp_tic(c, st, K_TREE_LEAF, 9.0 * (double)(1ll << v) + 32.0 * nodes, &slot);
            tree_keys_kernel<<<blocks, kKeyTreeThreads, 0, st>>>(K, C, ko, nchunks);
            fp_toc(c, st, slot);
            FP_CUDA(c, cudaGetLastError());
            L0 = v - kKeyTreeLevels;
        }
        while (L0 > 1) {
            const int levels = std::min(kTreeLevels, L0 - 1);
            TreeOut to;
            memset(&to, 0, sizeof to);
            for (int l = 0; l < levels; l++) to.lay[l] = lay[L0 - 1 - l];
            const unsigned blocks = 1u << (L0 - levels);
            const int n1 = 1 << (levels - 1);
            const int threads = std::min(512, n1);
            const size_t smem = (size_t)8 * 8 * n1;
            const double nodes = (double)(1ll << (L0 - 1)) * 2.0;
            int slot;
            if (L0 == v) {
                fp_tic(c, st, K_TREE_LEAF, 9.0 * (double)(1ll << L0) + 32.0 * nodes, &slot);
                tree_chunk_kernel<true><<<blocks, threads, smem, st>>>(K, C, lay[L0 - 1], to, levels);
            } else {
                fp_tic(c, st, K_TREE_UP, 32.0 * (double)(1ll << L0) + 32.0 * nodes, &slot);
                tree_chunk_kernel<false><<<blocks, threads, smem, st>>>(K, C, lay[L0], to, levels);
            }
            fp_toc(c, st, slot);
            FP_CUDA(c, cudaGetLastError());
            L0 -= levels;
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

    // ---- layer sum-checks: one resident kernel per layer, all queued up front ----
    int occ[2] = {0, 0};
    // the leaf layer's kernel takes its wide y table as dynamic shared memory (above the 48 KB
    // of static shared memory a kernel may declare)
    const size_t leaf_smem = (size_t)8 * kYWide + kPipeBytes;
    FP_CUDA(c, cudaFuncSetAttribute(gkr_layer_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)leaf_smem));
    FP_CUDA(c, cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ[0], gkr_layer_kernel<false>, LU_THREADS, 0));
    FP_CUDA(c, cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ[1], gkr_layer_kernel<true>, LU_LEAF_THREADS, leaf_smem));
    std::vector<GkrLayer> layers(v > 1 ? v - 1 : 0);
    for (int d = 1; d <= v - 1; d++) {
        const bool leaf = (d == v - 1);
        GkrLayer& A = layers[d - 1];
        memset(&A, 0, sizeof A);
        for (int tau = 0; tau < 2; tau++) {
            if (leaf) {
                A.pp[tau] = nullptr;
                A.qq[tau] = leafq[tau];
                A.parP[tau] = lay[d].P[tau];  // the level above the leaves (d = v - 1)
                A.parQ[tau] = lay[d].Q[tau];
            } else {
                A.sp[tau] = reinterpret_cast<const ulonglong2*>(lay[d + 1].P[tau]);
                A.sq[tau] = reinterpret_cast<const ulonglong2*>(lay[d + 1].Q[tau]);
                if (d == v - 2) {
                    // keep level v - 1 for the leaf layer: fold into its (not yet used) q buffer,
                    // 2^(v-3) positions of p and q pairs per table = 16 << (v - 2) bytes
                    A.pp[tau] = leafq[tau];
                    A.qq[tau] = leafq[tau] + ((size_t)1 << (v - 3));
                } else {
                    A.pp[tau] = reinterpret_cast<ulonglong2*>(lay[d + 1].P[tau]);
                    A.qq[tau] = reinterpret_cast<ulonglong2*>(lay[d + 1].Q[tau]);
                }
            }
        }
        A.E = E;
        A.keys = K;
        A.keys_vec = (uintptr_t)K.r % 8 == 0 && (uintptr_t)K.q % 8 == 0 && (uintptr_t)K.y % 2 == 0;
        A.chal = C;
        A.zin = zb[d & 1];
        A.zout = zb[(d + 1) & 1];
        A.lam = zb[2];
        A.d = d;
        const int64_t h1 = 1ll << (d - 1);
        // small layers: fewer threads, so single-block rounds reduce over fewer warps
        A.threads = (int)std::min<int64_t>(leaf ? LU_LEAF_THREADS : LU_THREADS, std::max<int64_t>(64, h1));
        A.per_block = A.threads;  // one pair per thread: the single-block rounds stay short chains
        A.piped = leaf && (uintptr_t)K.r % 16 == 0 && (uintptr_t)K.q % 16 == 0 && (uintptr_t)K.y % 16 == 0 &&
                  A.threads == LU_LEAF_THREADS;
        const int64_t want = (h1 + A.per_block - 1) / A.per_block;
        const int cap = std::max(1, occ[leaf ? 1 : 0]) * c->num_sms;
        A.grid = (int)std::max<int64_t>(1, std::min<int64_t>(want, cap));
        A.seq0 = fp_seq_reserve(c, d + 2);
    }
    if ((rc = fp_session_begin(c, st))) return rc;
    if (!c->stepped) {
        for (int d = 1; d <= v - 1; d++) {
            GkrLayer& A = layers[d - 1];
            A.t_begin = 1;
            A.t_end = d + 1;
            void* args[] = {&A, &c->mb_dev, &c->relay, &part};
            const bool leaf = (d == v - 1);
            double bytes = 0;
            for (int t = 1; t <= d; t++) bytes += gkr_round_bytes(leaf, t, (double)(1ll << (d - t)));
            int slot;
            fp_tic(c, st, K_GKR_ROUND, bytes, &slot);
            FP_CUDA(c, cudaLaunchCooperativeKernel(leaf ? (const void*)gkr_layer_kernel<true>
                                                        : (const void*)gkr_layer_kernel<false>,
                                                   dim3(A.grid), dim3(A.threads), args, leaf ? leaf_smem : 0, st));
            fp_toc(c, st, slot);
        }
    }
    // The host assembles each round polynomial g(X) = pre eq(z_t, X) h(X) from the
    // device's h(0), h(2): g(1) follows from the running claim (g(0) + g(1) = claim),
    // h(1) = g(1) / (pre z_t) gives g(3) through h(3) = h(0) - 3 h(1) + 3 h(2).
    // The next claim is g(rho_t) (Lagrange on the nodes 0..3).
    uint64_t prev[8];  // the two-node layer's values, then each layer's child values at its point
    memcpy(prev, hsmall, sizeof prev);
    std::vector<uint64_t> zpt, rhos, zinv;
    uint64_t mu = z.z[0];
    for (int d = 1; d <= v - 1; d++) {
        GkrLayer A = layers[d - 1];
        const bool leaf = (d == v - 1);
        const void* kern = leaf ? (const void*)gkr_layer_kernel<true> : (const void*)gkr_layer_kernel<false>;
        const uint64_t lam = fp_tx_squeeze_one(tx, "gkr_lambda");
        // point (previous rounds' challenges, mu) and claim sum_tau lam^(2 tau) (p~_tau + lam q~_tau)
        zpt = rhos;
        zpt.push_back(mu);
        rhos.clear();
        uint64_t claim = 0, lp = 1;
        for (int tau = 0; tau < 2; tau++) {
            const uint64_t pz = gl_fold(prev[4 * tau], prev[4 * tau + 1], mu);
            const uint64_t qz = gl_fold(prev[4 * tau + 2], prev[4 * tau + 3], mu);
            claim = gl_add(claim, gl_mul(lp, gl_add(pz, gl_mul(lam, qz))));
            lp = gl_mul(lam, lam);
        }
        // 1 / z_t for every coordinate at once (zero coordinates are left to the device)
        zinv.assign(d, 0);
        {
            uint64_t run = 1;
            for (int i = 0; i < d; i++) {
                zinv[i] = run;
                if (zpt[i]) run = gl_mul(run, zpt[i]);
            }
            uint64_t inv = gl_inv(run);
            for (int i = d - 1; i >= 0; i--) {
                if (!zpt[i]) continue;
                zinv[i] = gl_mul(zinv[i], inv);
                inv = gl_mul(inv, zpt[i]);
            }
        }
        uint64_t pre = 1;
        fp_session_expect(c, 3);
        fp_session_post2(c, A.seq0, mu, lam);
        for (int t = 1; t <= d + 1; t++) {
            if (c->stepped) {
                // one launch per round (its challenge is already in the mailbox), then the final values
                A.t_begin = A.t_end = t;
                void* args[] = {&A, &c->mb_dev, &c->relay, &part};
                const int64_t h = t <= d ? 1ll << (d - t) : 0;
                int slot;
                if (t <= d)
                    fp_tic(c, st, K_GKR_ROUND, gkr_round_bytes(leaf, t, (double)h), &slot);
                else
                    fp_tic(c, st, K_GKR_FINAL, 128.0, &slot);
                FP_CUDA(c, cudaLaunchCooperativeKernel(kern, dim3(t <= d ? A.grid : 1), dim3(A.threads), args,
                                                       leaf ? leaf_smem : 0, st));
                fp_toc(c, st, slot);
            }
            if ((rc = fp_session_wait(c, A.seq0 + t, st))) return rc;
            if (t <= d) {
                const uint64_t h0 = c->mb->res[0], h2 = c->mb->res[1], h1 = c->mb->res[2];
                const uint64_t zt = zpt[t - 1];
                const uint64_t ph0 = gl_mul(pre, h0);
                uint64_t g[4];
                g[0] = gl_mul(gl_sub(1, zt), ph0);
                g[1] = gl_sub(claim, g[0]);
                const uint64_t ph1 = zt ? gl_mul(g[1], zinv[t - 1]) : gl_mul(pre, h1);
                // the leaf layer's round 1 sends the X^2 coefficient C2: h(2) = 2 h(1) - h(0) + 2 C2
                const uint64_t ph2 = (leaf && t == 1) ? gl_add(gl_sub(gl_add(ph1, ph1), ph0), gl_mul(pre, gl_add(h2, h2)))
                                                      : gl_mul(pre, h2);
                g[2] = gl_mul(gl_sub(gl_add(zt, gl_add(zt, zt)), 1), ph2);                  // eq(z_t, 2) = 3 z_t - 1
                const uint64_t ph3 = gl_add(gl_sub(ph0, gl_add(ph1, gl_add(ph1, ph1))), gl_add(ph2, gl_add(ph2, ph2)));
                g[3] = gl_mul(gl_sub(gl_add(gl_add(zt, zt), gl_add(zt, gl_add(zt, zt))), 2), ph3);  // 5 z_t - 2
                for (int i = 0; i < 4; i++) put_le(proof + pos + 8 * i, g[i], 8);
                fp_tx_absorb_raw(tx, "gkr_round", proof + pos, 32);
                pos += 32;
                fp_session_expect(c, t < d ? 3 : 8);  // the last challenge triggers the final values
                const uint64_t r = fp_tx_squeeze_one(tx, "gkr_chal");
                fp_session_post(c, A.seq0 + t, r);
                claim = fp_lagrange4(g, r);
                pre = gl_mul(pre, gl_add(gl_mul(zt, r), gl_mul(gl_sub(1, zt), gl_sub(1, r))));
                rhos.push_back(r);
            } else {
                for (int i = 0; i < 8; i++) {
                    prev[i] = c->mb->res[i];
                    put_le(proof + pos + 8 * i, prev[i], 8);
                }
                fp_tx_absorb_raw(tx, "gkr_final", proof + pos, 64);
                pos += 64;
                mu = fp_tx_squeeze_one(tx, "gkr_mu");
            }
        }
    }
    // the leaf point: the last layer's round challenges, then its mu
    for (int i = 0; i < v - 1; i++) z.z[i] = rhos[i];
    z.z[v - 1] = mu;
    z.v = v;

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
        const int64_t ngroups = (nk + (1ll << lo_bits) - 1) >> lo_bits;
        const unsigned lgrid = (unsigned)std::max<int64_t>(1, std::min<int64_t>(ngroups, 8ll * c->num_sms));
        leaf_eval_kernel<<<lgrid, LU_THREADS, 0, st>>>(K, ehi, elo, lo_bits, part, c->tickets, small);
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
