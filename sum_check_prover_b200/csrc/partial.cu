// Multilinear partial evaluation: the eq-weighted row contraction
// out[c] = sum_i eq(z, i) M_eff[i][c] of int4 / int8 matrices.
//
// This is the matmul sum-check's weight decode ("How fast can FlashProve go",
// 4 Tighter Rooflines: each weight is decoded once for the matmuls'
// sum-checks): A_s = W~_s(r_row, .) streams W once, B_s = X~_s(., r_col)
// streams the token-major activations once. Weights are small integers, so the
// inner loop does no modular reduction: with u = M_eff + off >= 0 and
// eq(z, i) = eh * 2^32 + el, the exact 64-bit sums Lo = sum el u and
// Hi = sum eh u are kept per column, and folded into the field once per block:
// Lo + 2^32 Hi - off * (sum of the block's eq values). int4 nibbles are
// unpacked in registers.
//
// Tensor-core path (matrices whose rows hold whole 32-byte warp slices): the
// field weights are split into 8 byte limbs, e = sum_l e_l 2^(8 l), and
// C[c][l] = sum_i u[i][c] e_l[i] is an exact 8-bit -> s32 matrix product
// (mma m16n8k32: 16 matrix columns as the A rows, matrix rows as K, limbs as
// N). TMA streams 32-row chunks into shared memory; each warp takes its 32-byte
// slice with transposing ldmatrix loads, which hand it A fragments directly.
// int8 bytes enter as signed operands; an int4 byte b ^ 0x88 =
// 16 (w_odd + 8) + (w_even + 8) enters whole and as its low nibble, and the
// odd column is the difference over 16. The limbs are recombined mod p once
// per block. With scales, the weight of row i in column group g is
// e_i s[i][g] (a warp's columns lie in one group).
//
// All contractions of a call go into one launch per kernel variant (a job
// list; the MoE layer has hundreds of sites). eq(z, i) for the block's rows
// is computed in the block from the point, so no eq table is materialised. A
// job may give its row weights as a device vector instead (the coordinates of
// extension-field eq weights, the powers of a Freivalds challenge): the same
// contraction with w_i read per row.
#include <cuda.h>  // CUtensorMap and its enums; the encoder is fetched through the runtime
#include <cudaTypedefs.h>
#include <string.h>

#include <algorithm>
#include <vector>

#include "fp_field.cuh"
#include "fp_internal.h"

namespace {

struct PeJob {
    const uint8_t* mat;
    const int8_t* scales;
    const uint64_t* z;   // device, v coordinates
    const uint64_t* wts; // device row weights (row i at wts[i * wstride]), or null: eq(z, i)
    uint64_t* part;      // splits x cols block sums
    uint64_t* out;
    int64_t out_len;
    int32_t rows, cols, v, rows_per_block;
    int32_t col_blocks, splits;
    int32_t aligned;
    int32_t wstride;
    int64_t first_block;
    // tensor-core path: the matrix as a 2-D byte tensor (rows x pitch), 32-row x 128-byte
    // boxes with 128-byte swizzle, read by TMA from this device copy of the job
    alignas(64) CUtensorMap tmap;
};

constexpr int PE_THREADS = 256;              // 8 warps share the block's columns, split its rows
constexpr int PE_COLS = 8;                   // columns per lane: one 32-bit (int4) or 64-bit (int8) load per row
constexpr int PE_BLOCK_COLS = 32 * PE_COLS;  // 256 columns per block
constexpr int PE_UNROLL = 8;                 // rows whose loads a warp issues before using any of them
constexpr int PE_MAX_ROWS = 256;             // 256 rows x 2^32 x 2^15 < 2^64: the sums stay exact
constexpr int PE_TC_THREADS = PE_THREADS + 32;  // tensor-core path: 8 consumer warps and a TMA producer warp

// D (16 columns x 8 limbs) += A (16 columns x 32 rows of the matrix) . B (32 rows x 8 limbs)
__device__ __forceinline__ void mma_u8(uint32_t (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                       uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.u8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D (16 columns x 8 limbs) += A (signed bytes) . B (unsigned limbs)
__device__ __forceinline__ void mma_s8u8(uint32_t (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.u8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Two 16 x 16-byte matrices (rows named by lanes 0-15 and 16-31), transposed on the way in: the
// lane gets, per matrix, column gid of rows 4 tig .. 4 tig + 3 and column gid + 8 of the same rows
// (four bytes per register, row 4 tig in the low byte): the m16n8k32 A fragment of a row-major
// (K rows x 16 columns) tile.
__device__ __forceinline__ void ldsm_x2_trans(uint32_t (&f)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m16n16.x2.trans.shared.b8 {%0, %1, %2, %3}, [%4];\n"
                 : "=r"(f[0]), "=r"(f[1]), "=r"(f[2]), "=r"(f[3])
                 : "r"(addr)
                 : "memory");
}

// ---- TMA pipeline (shared-memory stages filled by cp.async.bulk.tensor, tracked by mbarriers) ----
constexpr int PE_STAGES = 6;               // 32-row chunks in flight per block
constexpr int PE_STAGE = 2 * 32 * 128;     // one chunk: two 32 x 128-byte boxes
constexpr int PE_DYN = PE_STAGES * PE_STAGE + 1024;  // + alignment slack
constexpr uint32_t PE_WAIT_LIMIT = 1u << 24;

__device__ __forceinline__ uint32_t pe_saddr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

// barrier 1 among the 8 consumer warps only (the producer warp never joins it)
__device__ __forceinline__ void pe_consumers_sync() { asm volatile("bar.sync 1, %0;\n" ::"n"(PE_THREADS) : "memory"); }

__device__ __forceinline__ bool pe_wait(uint32_t mbar, uint32_t parity) {
    for (uint32_t it = 0; it < PE_WAIT_LIMIT; it++) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}\n"
            : "=r"(ok)
            : "r"(mbar), "r"(parity)
            : "memory");
        if (ok) return true;
    }
    return false;
}

__device__ __forceinline__ uint64_t fold_lohi(uint64_t lo, uint64_t hi) {
    return gl_add(gl_canon(lo), gl_mul_2_32(gl_canon(hi)));
}

__device__ __forceinline__ int find_job(const PeJob* jobs, int njobs, int64_t b) {
    int lo = 0, hi = njobs - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (jobs[mid].first_block <= b)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

template <bool W4, bool SCALED>
__global__ void __launch_bounds__(PE_THREADS, 3) partial_many_kernel(const PeJob* __restrict__ jobs, int njobs) {
    __shared__ uint64_t eqs[PE_MAX_ROWS];
    __shared__ uint64_t red[2][8][PE_BLOCK_COLS / 2];
    __shared__ uint64_t wsum[8];
    const PeJob J = jobs[find_job(jobs, njobs, blockIdx.x)];
    const int64_t lb = blockIdx.x - J.first_block;
    const int cb = (int)(lb % J.col_blocks), split = (int)(lb / J.col_blocks);
    const int r0 = split * J.rows_per_block;
    const int nr = min(J.rows_per_block, J.rows - r0);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // eq(z, i) of the block's rows and their sum
    uint64_t es = 0;
    for (int k = threadIdx.x; k < nr; k += PE_THREADS) {
        const uint64_t i = (uint64_t)(r0 + k);
        uint64_t e = 1;
        if (J.wts)
            e = __ldg(J.wts + (int64_t)i * J.wstride);
        else
            for (int b = 0; b < J.v; b++) e = gl_mul(e, gl_eq1(J.z[b], (int)((i >> (J.v - 1 - b)) & 1)));
        eqs[k] = e;
        es = gl_add(es, e);
    }
    es = warp_sum_gl(es);
    if (lane == 0) wsum[warp] = es;
    __syncthreads();
    uint64_t esum = 0;
#pragma unroll
    for (int w = 0; w < PE_THREADS / 32; w++) esum = gl_add(esum, wsum[w]);

    const int col0 = cb * PE_BLOCK_COLS + lane * PE_COLS;
    const int64_t pitch = W4 ? (J.cols + 1) / 2 : J.cols;
    const int G = (J.cols + 63) / 64;
    const uint32_t off = SCALED ? (W4 ? 1024u : 16384u) : (W4 ? 8u : 128u);
    uint64_t lo[PE_COLS], hi[PE_COLS];
#pragma unroll
    for (int c = 0; c < PE_COLS; c++) lo[c] = hi[c] = 0;
    if (col0 < J.cols && J.aligned) {
        // u = M_eff + off >= 0 from the stored bits: an int4 nibble n holds w = n - 16 [n >= 8],
        // so n ^ 8 = w + 8; an int8 byte b gives b ^ 0x80 = w + 128. With a scale s,
        // w s + off = (n ^ 8) s + (off - 8 s) (int4) or (b ^ 0x80) s + (off - 128 s) (int8).
        const uint8_t* base = J.mat + (int64_t)r0 * pitch + (W4 ? (col0 >> 1) : col0);
        for (int kb = warp; kb < nr; kb += (PE_THREADS / 32) * PE_UNROLL) {
            uint32_t wv[PE_UNROLL][W4 ? 1 : 2];
            int32_t sv[PE_UNROLL];
            uint64_t ev[PE_UNROLL];
#pragma unroll
            for (int u = 0; u < PE_UNROLL; u++) {
                const int k = kb + (PE_THREADS / 32) * u;
                const bool in = k < nr;
                const uint8_t* rp = base + (int64_t)(in ? k : 0) * pitch;
                if (W4) {
                    wv[u][0] = in ? __ldcs(reinterpret_cast<const uint32_t*>(rp)) : 0u;
                } else {
                    const uint2 q = in ? __ldcs(reinterpret_cast<const uint2*>(rp)) : make_uint2(0, 0);
                    wv[u][0] = q.x;
                    wv[u][W4 ? 0 : 1] = q.y;
                }
                sv[u] = SCALED && in ? (int32_t)__ldg(J.scales + (int64_t)(r0 + k) * G + (col0 >> 6)) : 1;
                ev[u] = in ? eqs[k] : 0ull;  // rows past the end weigh nothing
            }
#pragma unroll
            for (int u = 0; u < PE_UNROLL; u++) {
                const uint32_t el = (uint32_t)ev[u], eh = (uint32_t)(ev[u] >> 32);
                const int32_t sc = sv[u];
                const uint32_t base_u = SCALED ? (uint32_t)((int32_t)off - (W4 ? 8 : 128) * sc) : 0u;
#pragma unroll
                for (int c = 0; c < PE_COLS; c++) {
                    uint32_t n;
                    if (W4)
                        n = ((wv[u][0] ^ 0x88888888u) >> (4 * c)) & 15u;
                    else
                        n = ((wv[u][c >> 2] ^ 0x80808080u) >> (8 * (c & 3))) & 255u;
                    const uint32_t uu = SCALED ? n * (uint32_t)sc + base_u : n;
                    lo[c] += (uint64_t)el * uu;
                    hi[c] += (uint64_t)eh * uu;
                }
            }
        }
    } else if (col0 < J.cols) {
        for (int k = warp; k < nr; k += PE_THREADS / 32) {
            const int64_t i = r0 + k;
            const uint64_t e = eqs[k];
            const uint32_t el = (uint32_t)e, eh = (uint32_t)(e >> 32);
#pragma unroll
            for (int c = 0; c < PE_COLS; c++) {
                const int cc = col0 + c;
                int x = 0;
                if (cc < J.cols) {
                    if (W4) {
                        const uint8_t bt = J.mat[i * pitch + (cc >> 1)];
                        const int n = (cc & 1) ? (bt >> 4) : (bt & 15);
                        x = n >= 8 ? n - 16 : n;
                    } else {
                        x = (int8_t)J.mat[i * pitch + cc];
                    }
                    if (SCALED) x *= (int32_t)__ldg(J.scales + i * G + (cc >> 6));
                }
                const uint32_t u = (uint32_t)(x + (int32_t)off);
                lo[c] += (uint64_t)el * u;
                hi[c] += (uint64_t)eh * u;
            }
        }
    }
    // the 8 warps' sums meet in shared memory, half of every lane's columns at a time
    const uint64_t corr = gl_mul(off, esum);
#pragma unroll
    for (int half = 0; half < 2; half++) {
        __syncthreads();
#pragma unroll
        for (int c = 0; c < PE_COLS / 2; c++) {
            red[0][warp][lane * (PE_COLS / 2) + c] = lo[half * (PE_COLS / 2) + c];
            red[1][warp][lane * (PE_COLS / 2) + c] = hi[half * (PE_COLS / 2) + c];
        }
        __syncthreads();
        for (int x = threadIdx.x; x < PE_BLOCK_COLS / 2; x += PE_THREADS) {
            uint64_t sl = 0, sh = 0;
#pragma unroll
            for (int w2 = 0; w2 < PE_THREADS / 32; w2++) {
                sl += red[0][w2][x];
                sh += red[1][w2][x];
            }
            const int ln = x / (PE_COLS / 2), cc = x % (PE_COLS / 2);
            const int col = cb * PE_BLOCK_COLS + ln * PE_COLS + half * (PE_COLS / 2) + cc;
            if (col < J.cols) J.part[(int64_t)split * J.cols + col] = gl_sub(fold_lohi(sl, sh), corr);
        }
    }
}

// Tensor-core partial evaluation. A warp owns 32 bytes of every row (64 int4 or
// 32 int8 columns); 8 warps side by side, up to PE_TC_ROWS rows per block.
//
// eq(z, i) of the block's rows comes from two small tables: with i = 32 m + n,
// eq(z, i) = H[m - m0] T[n], H over the high coordinates of the block's row
// groups and T over the last five coordinates; one product per row. Without
// scales every warp reads one limb table of the block's rows; with scales the
// weight of row i is e_i s[i][g] for the warp's column group g, so each warp
// forms its chunk's 32 scaled weights as it goes (the scales one chunk ahead).
constexpr int PE_TC_ROWS = 2048;  // exact s32 sums: 2048 x 255 x 255 < 2^31

template <bool W4, bool SCALED>
__global__ void __launch_bounds__(PE_TC_THREADS, 3) partial_tc_kernel(const PeJob* __restrict__ jobs, int njobs) {
    constexpr int WCOLS = W4 ? 64 : 32;
    constexpr int NG = W4 ? 4 : 2;  // MMAs per 32-row chunk: 16 columns each
    constexpr int ROWS = PE_TC_ROWS;
    // unscaled: limb l of row k's weight eq(z, i); scaled: eq(z, i) of the block's rows, and per
    // warp the limbs of the current chunk's scaled weights
    __shared__ __align__(16) uint8_t et[8][SCALED ? 16 : ROWS];
    __shared__ uint64_t eqs[SCALED ? ROWS : 1];
    __shared__ __align__(16) uint8_t lt[SCALED ? PE_THREADS / 32 : 1][8][32];
    __shared__ uint64_t htab[ROWS / 32], ttab[32];
    __shared__ uint64_t wsum[8];
    __shared__ __align__(8) uint64_t full[PE_STAGES], empty[PE_STAGES];
    extern __shared__ uint8_t dyn_raw[];  // PE_STAGES chunks (1024-byte aligned); then the per-warp sums
    uint8_t* stg = dyn_raw + ((1024 - (pe_saddr(dyn_raw) & 1023)) & 1023);
    uint32_t(*red)[64 * 8] = reinterpret_cast<uint32_t(*)[64 * 8]>(stg);
    const int jidx = find_job(jobs, njobs, blockIdx.x);
    const PeJob J = jobs[jidx];
    const int64_t lb = blockIdx.x - J.first_block;
    const int cb = (int)(lb % J.col_blocks), split = (int)(lb / J.col_blocks);
    const int r0 = split * J.rows_per_block;  // a multiple of 32
    const int nr = min(J.rows_per_block, J.rows - r0);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gid = lane >> 2, tig = lane & 3;
    const int wc0 = (cb * (PE_THREADS / 32) + warp) * WCOLS;
    if (threadIdx.x == 0) {
        for (int st = 0; st < PE_STAGES; st++) {
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(pe_saddr(&full[st])));
            asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(pe_saddr(&empty[st])), "r"(PE_THREADS / 32));
        }
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::);
    }
    __syncthreads();  // the barriers are initialised
    const int nch = (nr + 31) >> 5;
    if (warp == PE_THREADS / 32) {
        // producer warp: one lane streams the block's 32-row chunks of its 256-byte column slice into
        // the stages, two TMA boxes (32 rows x 128 bytes, 128-byte swizzle) per chunk, each stage once
        // the consumer warps have released the chunk it held. Rows past the block are read too: their
        // eq limbs are zero. A release that never comes ends the stream (the consumers' waits then
        // run out too: wrong sums, no hang).
        if (lane == 0) {
            const CUtensorMap* tm = &jobs[jidx].tmap;
            asm volatile("fence.proxy.tensormap::generic.acquire.gpu [%0], 128;\n" ::"l"(tm) : "memory");
            int st = 0;
            uint32_t par = 0;
            for (int i = 0; i < nch; i++) {
                if (i >= PE_STAGES && !pe_wait(pe_saddr(&empty[st]), par ^ 1u)) break;
                const uint32_t fb = pe_saddr(&full[st]);
                asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(fb), "r"(PE_STAGE) : "memory");
#pragma unroll
                for (int half = 0; half < 2; half++)
                    asm volatile(
                        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
                        "%3}], [%4];\n" ::"r"(pe_saddr(stg + st * PE_STAGE + half * (PE_STAGE / 2))),
                        "l"(tm), "r"(cb * 256 + half * 128), "r"(r0 + 32 * i), "r"(fb)
                        : "memory");
                if (++st == PE_STAGES) {
                    st = 0;
                    par ^= 1u;
                }
            }
        }
        return;
    }
    const bool wactive = wc0 < J.cols;
    const int G = (J.cols + 63) / 64;

    // the two eq tables (v < 5: T covers every coordinate and H is the single entry 1)
    const int tb = J.v < 5 ? J.v : 5;  // coordinates in T (the last tb of z)
    const int hb = J.v - tb;
    const int ngroups = (nr + 31) >> 5;
    for (int x = threadIdx.x; x < ngroups + 32; x += PE_THREADS) {
        uint64_t e = 1;
        if (x < ngroups) {
            const uint64_t m = (uint64_t)(r0 >> 5) + x;  // row group: the rows' high bits
            for (int b = 0; b < hb; b++) e = gl_mul(e, gl_eq1(J.z[b], (int)((m >> (hb - 1 - b)) & 1)));
            htab[x] = e;
        } else {
            const int n = x - ngroups;
            for (int b = 0; b < tb; b++) e = gl_mul(e, gl_eq1(J.z[hb + b], (n >> (tb - 1 - b)) & 1));
            ttab[n] = e;
        }
    }
    pe_consumers_sync();
    uint64_t es = 0;  // sum of the weights this warp's columns see
    const int kend = (nr + 31) & ~31;  // whole chunks: positions past nr read zero limbs
    if (!SCALED) {
        for (int k = threadIdx.x; k < kend; k += PE_THREADS) {
            // with v < 5 the rows are i = n < 2^v and H = {1}
            const uint64_t e = k >= nr ? 0ull
                               : J.wts ? __ldg(J.wts + (int64_t)(r0 + k) * J.wstride)
                                       : gl_mul(htab[k >> 5], ttab[k & 31]);
#pragma unroll
            for (int l = 0; l < 8; l++) et[l][k] = (uint8_t)(e >> (8 * l));
            es = gl_add(es, e);
        }
        es = warp_sum_gl(es);
        if (lane == 0) wsum[warp] = es;
        pe_consumers_sync();
        es = 0;
#pragma unroll
        for (int w = 0; w < PE_THREADS / 32; w++) es = gl_add(es, wsum[w]);
    } else {
        for (int k = threadIdx.x; k < kend; k += PE_THREADS)
            eqs[k] = k >= nr ? 0ull
                     : J.wts ? __ldg(J.wts + (int64_t)(r0 + k) * J.wstride)
                             : gl_mul(htab[k >> 5], ttab[k & 31]);
        pe_consumers_sync();
    }
    // scaled: the scale of row 32 i + lane in the warp's column group, loaded a chunk ahead
    const int8_t* srow = SCALED ? J.scales + (int64_t)r0 * G + wc0 / 64 : nullptr;
    int32_t sv = 0;
    if (SCALED && wactive && lane < nr) sv = (int32_t)__ldg(srow + (int64_t)lane * G);

    uint32_t acc[NG][4];
#pragma unroll
    for (int g = 0; g < NG; g++) acc[g][0] = acc[g][1] = acc[g][2] = acc[g][3] = 0;
    {
        // every warp waits for a chunk, loads its 32-byte slice as two transposed 32 x 16-byte A
        // fragments, and releases the stage
        const uint8_t* lp = &et[gid][0];
        // ldmatrix row addresses: lane L names row L of the chunk (lanes 0-15 the first 16 x 16-byte
        // matrix, lanes 16-31 the second); the warp's slice is 16-byte chunks c0 and c0 + 1 of its
        // 128-byte half, and 128-byte swizzle puts chunk c of row r at c ^ (r % 8)
        const int c0 = (warp & 3) * 2;
        const uint32_t hoff = (uint32_t)((warp >> 2) * (PE_STAGE / 2) + lane * 128);
        const uint32_t o0 = hoff + ((c0 ^ (lane & 7)) << 4), o1 = hoff + (((c0 + 1) ^ (lane & 7)) << 4);
        const uint32_t sbase = pe_saddr(stg);
        int st = 0;
        uint32_t par = 0;
        for (int i = 0; i < nch; i++) {
            const bool got = pe_wait(pe_saddr(&full[st]), par);
            __syncwarp();  // ldmatrix is warp-wide
            // f[h][0..3]: the A fragment of bytes 16 h .. 16 h + 15 of the slice: f[h][0] holds byte
            // column gid of rows 4 tig .. 4 tig + 3, f[h][1] column gid + 8, f[h][2], f[h][3] the same
            // for rows 16 + 4 tig ..
            uint32_t f[2][4];
            const uint32_t sp = sbase + (uint32_t)(st * PE_STAGE);
            ldsm_x2_trans(f[0], sp + o0);
            ldsm_x2_trans(f[1], sp + o1);
            __syncwarp();
            if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(pe_saddr(&empty[st])) : "memory");
            const int ch = 32 * i;
            if (++st == PE_STAGES) {
                st = 0;
                par ^= 1u;
            }
            // a stalled copy leaves this block's sums wrong, not hung (the same decision in every lane)
            if (!__all_sync(0xffffffffu, got) || !wactive) continue;
            // B: limb gid of rows tig*4 .. +3 and 16 + tig*4 .. +3
            uint32_t b0, b1;
            if (SCALED) {
                // lane r forms row r's weight e s (zero past the block: eqs is zero there) and
                // spreads its limbs; the warp's previous reads of lt ended before the wait above
                const int k = ch + lane;
                const uint64_t w = gl_mul_small(eqs[k], sv);
                sv = k + 32 < nr ? (int32_t)__ldg(srow + (int64_t)(k + 32) * G) : 0;
                es = gl_add(es, w);
#pragma unroll
                for (int l = 0; l < 8; l++) lt[warp][l][lane] = (uint8_t)(w >> (8 * l));
                __syncwarp();
                b0 = *reinterpret_cast<const uint32_t*>(&lt[warp][gid][tig * 4]);
                b1 = *reinterpret_cast<const uint32_t*>(&lt[warp][gid][16 + tig * 4]);
            } else {
                b0 = *reinterpret_cast<const uint32_t*>(lp + ch + tig * 4);
                b1 = *reinterpret_cast<const uint32_t*>(lp + ch + 16 + tig * 4);
            }
#pragma unroll
            for (int h = 0; h < 2; h++) {
                if (W4) {
                    // byte ^ 0x88 = 16 (w_odd + 8) + (w_even + 8): the whole byte (P) and its low
                    // nibble (Q) give both columns, the odd one as (P - Q) / 16
                    uint32_t x[4], lo[4];
#pragma unroll
                    for (int r = 0; r < 4; r++) {
                        x[r] = f[h][r] ^ 0x88888888u;
                        lo[r] = x[r] & 0x0F0F0F0Fu;
                    }
                    mma_u8(acc[2 * h], x[0], x[1], x[2], x[3], b0, b1);
                    mma_u8(acc[2 * h + 1], lo[0], lo[1], lo[2], lo[3], b0, b1);
                } else {
                    mma_s8u8(acc[h], f[h][0], f[h][1], f[h][2], f[h][3], b0, b1);
                }
            }
        }
    }
    pe_consumers_sync();  // every consumer warp is done with the stages, which now hold the sums
    // D[m][n]: m = byte column of the 16-byte half h (m = gid in c0, c1; gid + 8 in c2, c3),
    // n = 2 tig + e = limb. int4: byte b holds columns 2 b (low nibble) and 2 b + 1.
    if (!wactive) return;
    if (SCALED) es = warp_sum_gl(es);  // this warp's sum of e s
#pragma unroll
    for (int h = 0; h < 2; h++) {
#pragma unroll
        for (int e = 0; e < 2; e++) {
#pragma unroll
            for (int hm = 0; hm < 2; hm++) {
                const int byte = 16 * h + gid + 8 * hm;
                const int limb = 2 * tig + e;
                if (W4) {
                    const uint32_t P = acc[2 * h][2 * hm + e], Q = acc[2 * h + 1][2 * hm + e];
                    red[warp][(2 * byte) * 8 + limb] = Q;
                    red[warp][(2 * byte + 1) * 8 + limb] = (P - Q) >> 4;
                } else {
                    red[warp][byte * 8 + limb] = acc[h][2 * hm + e];
                }
            }
        }
    }
    __syncwarp();
    // int4 sums are of w + 8 (corrected by 8 times the weight sum); int8 limb sums are signed
    // (s8 matrix bytes): each is read with 2^31 added, and the added 2^31 sum_l 2^(8 l) is removed
    const uint64_t corr = W4 ? gl_mul(8u, es) : gl_mul(1ull << 31, 0x0101010101010101ull);
    const uint32_t flip = W4 ? 0u : 0x80000000u;
    for (int c = lane; c < WCOLS; c += 32) {
        const int gc = wc0 + c;
        if (gc >= J.cols) break;
        // sum_l C_l 2^(8 l) for C_l < 2^32: a = limbs 0..3, b = limbs 4..7 (each < 2^57), a + 2^32 b
        const uint32_t* C = &red[warp][c * 8];
        const uint64_t a = (uint64_t)(C[0] ^ flip) + ((uint64_t)(C[1] ^ flip) << 8) + ((uint64_t)(C[2] ^ flip) << 16) +
                           ((uint64_t)(C[3] ^ flip) << 24);
        const uint64_t bq = (uint64_t)(C[4] ^ flip) + ((uint64_t)(C[5] ^ flip) << 8) + ((uint64_t)(C[6] ^ flip) << 16) +
                            ((uint64_t)(C[7] ^ flip) << 24);
        uint64_t lo = a, hi = bq >> 32;
        asm("add.cc.u64 %0, %0, %2;\n\taddc.u64 %1, %1, 0;" : "+l"(lo), "+l"(hi) : "l"(bq << 32));
        J.part[(int64_t)split * J.cols + gc] = gl_sub(gl_canon(gl_reduce_weak(lo, hi)), corr);
    }
}

// out[c] = sum over the splits of part[split][c] (c < cols), 0 up to out_len; job blockIdx.y
__global__ void partial_fin_kernel(const PeJob* __restrict__ jobs) {
    const PeJob J = jobs[blockIdx.y];
    for (int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; c < J.out_len;
         c += (int64_t)gridDim.x * blockDim.x) {
        if (c >= J.cols) {
            J.out[c] = 0;
            continue;
        }
        uint64_t a = 0;
        for (int s = 0; s < J.splits; s++) a = gl_add(a, J.part[(int64_t)s * J.cols + c]);
        J.out[c] = a;
    }
}

template <bool W4, bool SCALED>
cudaError_t pe_tc_launch(const PeJob* dj, int n, int64_t blocks, cudaStream_t s) {
    cudaError_t e = cudaFuncSetAttribute(partial_tc_kernel<W4, SCALED>, cudaFuncAttributeMaxDynamicSharedMemorySize, PE_DYN);
    if (e != cudaSuccess) return e;
    partial_tc_kernel<W4, SCALED><<<(unsigned)blocks, PE_TC_THREADS, PE_DYN, s>>>(dj, n);
    return cudaGetLastError();
}

// About `waves` blocks per SM, at most max_rows rows per block (a multiple of row_step): the
// CUDA-core fallback for a job whose tensor map could not be made.
void pe_plan_shape(int num_sms, int rows, int cols, int block_cols, int max_rows, int row_step, int waves,
                   int& col_blocks, int& rpb, int& splits) {
    col_blocks = (cols + block_cols - 1) / block_cols;
    int want = (waves * num_sms + col_blocks - 1) / col_blocks;
    rpb = (rows + want - 1) / want;
    rpb = (rpb + row_step - 1) / row_step * row_step;
    if (rpb < row_step) rpb = row_step;
    if (rpb > max_rows) rpb = max_rows;
    splits = (rows + rpb - 1) / rpb;
}

// cuTensorMapEncodeTiled through the runtime (no link-time dependency on the driver library)
PFN_cuTensorMapEncodeTiled_v12000 tmap_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess) {
            cudaGetLastError();
            p = nullptr;
        }
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }();
    return fn;
}

// The matrix as a 2-D byte tensor for TMA: 32-row x 128-byte boxes, 128-byte swizzle, zero fill
bool pe_make_tmap(const FpPeJob& q, CUtensorMap* tm) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tmap_encoder();
    if (!enc) return false;
    const cuuint64_t pitch = q.bits == 4 ? (cuuint64_t)(q.cols + 1) / 2 : (cuuint64_t)q.cols;
    const cuuint64_t dims[2] = {pitch, (cuuint64_t)q.rows};
    const cuuint64_t strides[1] = {pitch};
    const cuuint32_t box[2] = {128, 32}, estr[2] = {1, 1};
    return enc(tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(q.mat), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The tensor-core path needs whole 32-byte warp slices in every row and a matrix that TMA can
// read (16-byte aligned base and row pitch).
bool pe_tc_ok(const FpPeJob& q) {
    const int64_t pitch = q.bits == 4 ? (q.cols + 1) / 2 : q.cols;
    return ((uintptr_t)q.mat % 16 == 0) && (q.cols % (q.bits == 4 ? 64 : 32) == 0) && (pitch % 16 == 0) &&
           tmap_encoder() != nullptr;
}

void pe_plan_cuda_core(int num_sms, const FpPeJob& q, int& col_blocks, int& rpb, int& splits) {
    pe_plan_shape(num_sms, q.rows, q.cols, PE_BLOCK_COLS, PE_MAX_ROWS, 8, 2, col_blocks, rpb, splits);
}

struct PePlan {
    bool tc;
    int col_blocks, rpb, splits;
};

int pe_variant(bool tc, const FpPeJob& q) { return (tc ? 4 : 0) + (q.bits == 4 ? 2 : 0) + (q.scales ? 1 : 0); }

// Every job of a call is planned together: the jobs of one kernel variant share one grid, so one
// row count per block is chosen for all of them, the smallest (a multiple of the row step, at most
// the exact-sum limit) that keeps the whole grid within about `waves` blocks per SM. A lone large
// matrix gets about two rounds of three resident blocks per SM; a batch of many matrices (a MoE
// layer) gets long blocks instead of many short ones, each of which would pay the block's set-up
// and its first copy's latency over a few chunks.
std::vector<PePlan> pe_plan_all(int num_sms, const FpPeJob* jobs, int njobs) {
    std::vector<PePlan> P(njobs);
    for (int j = 0; j < njobs; j++) {
        const FpPeJob& q = jobs[j];
        P[j].tc = pe_tc_ok(q);
        const int bc = P[j].tc ? (PE_THREADS / 32) * (q.bits == 4 ? 64 : 32) : PE_BLOCK_COLS;
        P[j].col_blocks = (q.cols + bc - 1) / bc;
    }
    for (int var = 0; var < 8; var++) {
        const bool tc = var >= 4;
        const int64_t step = tc ? 32 : 8, cap = tc ? PE_TC_ROWS : PE_MAX_ROWS;
        const int64_t target = (int64_t)(tc ? 6 : 2) * num_sms;
        auto blocks = [&](int64_t R) {
            int64_t n = 0;
            for (int j = 0; j < njobs; j++)
                if (pe_variant(P[j].tc, jobs[j]) == var) n += (int64_t)P[j].col_blocks * ((jobs[j].rows + R - 1) / R);
            return n;
        };
        if (blocks(cap) == 0) continue;  // no job of this variant
        int64_t lo = 1, hi = cap / step;  // the answer in row steps
        if (blocks(cap) > target) {
            lo = hi;
        } else {
            while (lo < hi) {
                const int64_t mid = (lo + hi) / 2;
                if (blocks(mid * step) <= target)
                    hi = mid;
                else
                    lo = mid + 1;
            }
        }
        const int R = (int)(lo * step);
        for (int j = 0; j < njobs; j++)
            if (pe_variant(P[j].tc, jobs[j]) == var) {
                P[j].rpb = R;
                P[j].splits = (jobs[j].rows + R - 1) / R;
            }
    }
    return P;
}

}  // namespace

bool fp_tmap_u8_2d(void* tmap, const void* base, uint64_t inner, uint64_t rows, uint64_t pitch, uint32_t box_inner,
                   uint32_t box_rows, bool swizzle128) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tmap_encoder();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)pitch};
    const cuuint32_t box[2] = {box_inner, box_rows}, estr[2] = {1, 1};
    return enc(reinterpret_cast<CUtensorMap*>(tmap), CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims,
               strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t fp_partial_scratch(const fp_ctx* c, const FpPeJob* jobs, int njobs) {
    size_t need = 4 * fp_align_up(sizeof(PeJob) * (size_t)njobs, 256) + 4096;
    const std::vector<PePlan> P = pe_plan_all(c->num_sms, jobs, njobs);
    for (int j = 0; j < njobs; j++) {
        int cbk, rpb, sp;
        pe_plan_cuda_core(c->num_sms, jobs[j], cbk, rpb, sp);  // the fallback of a job without a tensor map
        sp = std::max(sp, P[j].splits);
        need += fp_align_up((size_t)8 * sp * jobs[j].cols, 256) + fp_align_up(8 * (size_t)std::max(1, jobs[j].v), 256);
    }
    return need;
}

size_t fp_partial_host_scratch(const FpPeJob* jobs, int njobs) {
    size_t zt = 0;
    for (int j = 0; j < njobs; j++) zt += (size_t)jobs[j].v;
    return fp_align_up(8 * (zt + 1), 256) + 4 * fp_align_up(sizeof(PeJob) * (size_t)njobs, 256) + 4096;
}

int fp_partial_many(fp_ctx* c, const FpPeJob* jobs, int njobs, cudaStream_t s) {
    if (njobs <= 0) return FP_OK;
    std::vector<PeJob> h(njobs);
    std::vector<int> order[8];  // (tensor-core path, int4, scaled)
    const std::vector<PePlan> P = pe_plan_all(c->num_sms, jobs, njobs);
    size_t zt = 0;
    for (int j = 0; j < njobs; j++) zt += (size_t)jobs[j].v;
    uint64_t* hz = (uint64_t*)fp_alloc(c->host, 8 * (zt + 1));
    uint64_t* dz = (uint64_t*)fp_alloc(c->dev, 8 * (zt + 1));
    if (!hz || !dz) return fp_fail(c, FP_ERR_OOM, "partial evaluation: scratch exhausted");
    size_t zo = 0;
    for (int j = 0; j < njobs; j++) {
        const FpPeJob& q = jobs[j];
        PeJob& d = h[j];
        d.mat = (const uint8_t*)q.mat;
        d.scales = q.scales;
        d.out = q.out;
        d.out_len = q.out_len;
        d.rows = q.rows;
        d.cols = q.cols;
        d.v = q.v;
        bool tc = P[j].tc;
        d.col_blocks = P[j].col_blocks;
        d.rows_per_block = P[j].rpb;
        d.splits = P[j].splits;
        memset(&d.tmap, 0, sizeof d.tmap);
        if (tc && !pe_make_tmap(q, &d.tmap)) {  // no tensor map: the CUDA-core kernel
            tc = false;
            pe_plan_cuda_core(c->num_sms, q, d.col_blocks, d.rows_per_block, d.splits);
        }
        const int64_t pitch = q.bits == 4 ? (q.cols + 1) / 2 : q.cols;
        // the fast path loads 4 (int4) or 8 (int8) bytes per lane and row
        d.aligned = ((uintptr_t)q.mat % 16 == 0) && (q.cols % PE_COLS == 0) &&
                    (q.bits == 4 ? (pitch % 4 == 0) : (pitch % 8 == 0));
        d.wts = q.wts;
        d.wstride = q.wts_stride;
        d.first_block = 0;
        d.part = (uint64_t*)fp_alloc(c->dev, (size_t)8 * d.splits * q.cols);
        if (!d.part) return fp_fail(c, FP_ERR_OOM, "partial evaluation: scratch exhausted");
        if (q.v) memcpy(hz + zo, q.z, 8 * (size_t)q.v);
        d.z = dz + zo;
        zo += (size_t)q.v;
        order[pe_variant(tc, q)].push_back(j);
    }
    FP_CUDA(c, cudaMemcpyAsync(dz, hz, 8 * (zt + 1), cudaMemcpyHostToDevice, s));
    for (int var = 0; var < 8; var++) {
        if (order[var].empty()) continue;
        std::vector<PeJob> g;
        int64_t blocks = 0;
        double bytes = 0;
        for (int j : order[var]) {
            PeJob d = h[j];
            d.first_block = blocks;
            blocks += (int64_t)d.col_blocks * d.splits;
            g.push_back(d);
            const double pitch = jobs[j].bits == 4 ? (jobs[j].cols + 1) / 2 : jobs[j].cols;
            bytes += jobs[j].rows * pitch + (jobs[j].scales ? (double)jobs[j].rows * ((jobs[j].cols + 63) / 64) : 0.0);
        }
        const size_t sz = sizeof(PeJob) * g.size();
        PeJob* dj = (PeJob*)fp_alloc(c->dev, sz);
        PeJob* hj = (PeJob*)fp_alloc(c->host, sz);
        if (!dj || !hj) return fp_fail(c, FP_ERR_OOM, "partial evaluation: scratch exhausted");
        memcpy(hj, g.data(), sz);
        FP_CUDA(c, cudaMemcpyAsync(dj, hj, sz, cudaMemcpyHostToDevice, s));
        int slot;
        fp_tic(c, s, K_PARTIAL_ACC, bytes, &slot);
        const int n = (int)g.size();
        if (var == 0) partial_many_kernel<false, false><<<(unsigned)blocks, PE_THREADS, 0, s>>>(dj, n);
        if (var == 1) partial_many_kernel<false, true><<<(unsigned)blocks, PE_THREADS, 0, s>>>(dj, n);
        if (var == 2) partial_many_kernel<true, false><<<(unsigned)blocks, PE_THREADS, 0, s>>>(dj, n);
        if (var == 3) partial_many_kernel<true, true><<<(unsigned)blocks, PE_THREADS, 0, s>>>(dj, n);
        static_assert(PE_STAGES * PE_STAGE >= 8 * 64 * 8 * 4, "the stages must hold the per-warp sums");
        if (var == 4) FP_CUDA(c, (pe_tc_launch<false, false>(dj, n, blocks, s)));
        if (var == 5) FP_CUDA(c, (pe_tc_launch<false, true>(dj, n, blocks, s)));
        if (var == 6) FP_CUDA(c, (pe_tc_launch<true, false>(dj, n, blocks, s)));
        if (var == 7) FP_CUDA(c, (pe_tc_launch<true, true>(dj, n, blocks, s)));
        fp_toc(c, s, slot);
        FP_CUDA(c, cudaGetLastError());
    }
    const size_t sz = sizeof(PeJob) * (size_t)njobs;
    PeJob* dj = (PeJob*)fp_alloc(c->dev, sz);
    PeJob* hj = (PeJob*)fp_alloc(c->host, sz);
    if (!dj || !hj) return fp_fail(c, FP_ERR_OOM, "partial evaluation: scratch exhausted");
    memcpy(hj, h.data(), sz);
    FP_CUDA(c, cudaMemcpyAsync(dj, hj, sz, cudaMemcpyHostToDevice, s));
    int64_t maxlen = 0;
    double fbytes = 0;
    for (auto& d : h) {
        maxlen = std::max<int64_t>(maxlen, d.out_len);
        fbytes += 8.0 * d.splits * d.cols + 8.0 * d.out_len;
    }
    const unsigned gx = (unsigned)std::max<int64_t>(1, std::min<int64_t>((maxlen + 255) / 256, 64));
    int slot;
    fp_tic(c, s, K_PARTIAL_FIN, fbytes, &slot);
    partial_fin_kernel<<<dim3(gx, njobs), 256, 0, s>>>(dj);
    fp_toc(c, s, slot);
    FP_CUDA(c, cudaGetLastError());
    return FP_OK;
}
