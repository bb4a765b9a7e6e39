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
// All contractions of a call go into one launch per operand variant (a job
// list; the MoE layer has hundreds of sites): a block owns 512 columns x up
// to 256 rows of one job, its 8 warps split the rows, and their sums meet in
// shared memory. eq(z, i) for the block's rows is computed in the block from
// the point, so no eq table is materialised.
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
    uint64_t* part;      // splits x cols block sums
    uint64_t* out;
    int64_t out_len;
    int32_t rows, cols, v, rows_per_block;
    int32_t col_blocks, splits;
    int32_t aligned;
    int32_t pad;
    int64_t first_block;
};

constexpr int PE_THREADS = 256;              // 8 warps share the block's columns, split its rows
constexpr int PE_COLS = 8;                   // columns per lane: one 32-bit (int4) or 64-bit (int8) load per row
constexpr int PE_BLOCK_COLS = 32 * PE_COLS;  // 256 columns per block
constexpr int PE_UNROLL = 8;                 // rows whose loads a warp issues before using any of them
constexpr int PE_MAX_ROWS = 256;             // 256 rows x 2^32 x 2^15 < 2^64: the sums stay exact

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

// About two waves of 8-warp blocks, at most PE_MAX_ROWS rows per block.
void pe_plan(int num_sms, int rows, int cols, int& col_blocks, int& rpb, int& splits) {
    col_blocks = (cols + PE_BLOCK_COLS - 1) / PE_BLOCK_COLS;
    int want = (2 * num_sms + col_blocks - 1) / col_blocks;
    rpb = (rows + want - 1) / want;
    rpb = (rpb + 7) / 8 * 8;
    if (rpb < 8) rpb = 8;
    if (rpb > PE_MAX_ROWS) rpb = PE_MAX_ROWS;
    splits = (rows + rpb - 1) / rpb;
}

}  // namespace

size_t fp_partial_scratch(const fp_ctx* c, const FpPeJob* jobs, int njobs) {
    size_t need = 4 * fp_align_up(sizeof(PeJob) * (size_t)njobs, 256) + 4096;
    for (int j = 0; j < njobs; j++) {
        int cbk, rpb, sp;
        pe_plan(c->num_sms, jobs[j].rows, jobs[j].cols, cbk, rpb, sp);
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
    std::vector<int> order[4];
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
        pe_plan(c->num_sms, q.rows, q.cols, d.col_blocks, d.rows_per_block, d.splits);
        const int64_t pitch = q.bits == 4 ? (q.cols + 1) / 2 : q.cols;
        // the fast path loads 4 (int4) or 8 (int8) bytes per lane and row
        d.aligned = ((uintptr_t)q.mat % 16 == 0) && (q.cols % PE_COLS == 0) &&
                    (q.bits == 4 ? (pitch % 4 == 0) : (pitch % 8 == 0));
        d.pad = 0;
        d.first_block = 0;
        d.part = (uint64_t*)fp_alloc(c->dev, (size_t)8 * d.splits * q.cols);
        if (!d.part) return fp_fail(c, FP_ERR_OOM, "partial evaluation: scratch exhausted");
        if (q.v) memcpy(hz + zo, q.z, 8 * (size_t)q.v);
        d.z = dz + zo;
        zo += (size_t)q.v;
        order[(q.bits == 4 ? 2 : 0) + (q.scales ? 1 : 0)].push_back(j);
    }
    FP_CUDA(c, cudaMemcpyAsync(dz, hz, 8 * (zt + 1), cudaMemcpyHostToDevice, s));
    for (int var = 0; var < 4; var++) {
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
