// mle_partial_eval_noalloc: the multilinear partial evaluation without any
// device allocation.
//
// Who needs this: code that runs where cudaMalloc is off limits -- inside a
// host callback or a custom allocator hook, under a memory pool that forbids
// out-of-band allocations, or in a process that has already reserved every
// byte of device memory for other work. mle_partial_eval needs an fp_ctx,
// whose scratch arena grows with cudaMalloc; this variant needs neither. Its
// scratch is one file-scope device array of fixed size (kNoallocWords 64-bit
// words = 16 MiB). The CUDA runtime loads this file's module on a device the
// first time it is used there (lazy loading, the default since CUDA 12): that
// first call reserves the 16 MiB, which the device then holds until the
// process exits. Make the first call on each device outside the context that
// must not allocate.
//
// The caller still passes the matrix, the point and the output buffer. The
// result is the same as mle_partial_eval's: out[c] = sum_i eq(point, i) *
// M_eff[i][c], with M_eff = scales[i][c/64] * mat[i][c] when scales are given.
#include "fp_field.cuh"
#include "fp_internal.h"

namespace {

constexpr int kNaThreads = 128;
constexpr int kNaCols = 8;                  // columns per thread
constexpr int kNaRows = 1024;               // rows per split (block), eq of those rows kept in shared memory
constexpr uint64_t kNoallocWords = 1u << 21;  // 16 MiB of per-split column partials

// The scratch array. Host code must not pass its name to a kernel (on the host
// the name is only a stand-in for the device symbol); the entry point passes
// the device address obtained with cudaGetSymbolAddress instead.
static __device__ __align__(256) uint64_t g_noalloc_scratch[kNoallocWords];

struct NaPoint {
    uint64_t z[24];
    int v;
};

// One block: kNaRows rows (one split) x kNaThreads * kNaCols columns.
// part[split][c] = sum over the split's rows of eq[i] * (M_eff[i][c] + off) - off * sum eq[i]
// computed with exact 64-bit sums of the 32-bit halves of eq, then reduced mod p.
template <bool W4, bool SCALED>
__global__ void __launch_bounds__(kNaThreads)
    pe_noalloc_acc_kernel(const uint8_t* __restrict__ mat, const int8_t* __restrict__ scales, int rows, int cols,
                          NaPoint z, uint64_t* __restrict__ part) {
    __shared__ uint64_t eqs[kNaRows];
    __shared__ uint64_t esum_w[kNaThreads / 32];
    const int r0 = blockIdx.y * kNaRows;
    const int nr = min(kNaRows, rows - r0);
    uint64_t es = 0;
    for (int k = threadIdx.x; k < nr; k += kNaThreads) {
        const uint64_t i = (uint64_t)(r0 + k);
        uint64_t e = 1;
        for (int b = 0; b < z.v; b++) e = gl_mul(e, gl_eq1(z.z[b], (int)((i >> (z.v - 1 - b)) & 1)));
        eqs[k] = e;
        es = gl_add(es, e);
    }
    es = warp_sum_gl(es);
    if ((threadIdx.x & 31) == 0) esum_w[threadIdx.x >> 5] = es;
    __syncthreads();
    uint64_t esum = 0;
#pragma unroll
    for (int w = 0; w < kNaThreads / 32; w++) esum = gl_add(esum, esum_w[w]);

    const int col0 = (blockIdx.x * kNaThreads + threadIdx.x) * kNaCols;
    if (col0 >= cols) return;
    const int64_t pitch = W4 ? (cols + 1) / 2 : cols;
    const int G = (cols + 63) / 64;
    const uint32_t off = SCALED ? (W4 ? 1024u : 16384u) : (W4 ? 8u : 128u);
    uint64_t lo[kNaCols], hi[kNaCols];
#pragma unroll
    for (int c = 0; c < kNaCols; c++) lo[c] = hi[c] = 0;
    for (int k = 0; k < nr; k++) {
        const int64_t i = r0 + k;
        const uint64_t e = eqs[k];
        const uint32_t el = (uint32_t)e, eh = (uint32_t)(e >> 32);
#pragma unroll
        for (int c = 0; c < kNaCols; c++) {
            const int cc = col0 + c;
            int v = 0;
            if (cc < cols) {
                if (W4) {
                    const uint8_t b = mat[i * pitch + (cc >> 1)];
                    const int n = (cc & 1) ? (b >> 4) : (b & 15);
                    v = n >= 8 ? n - 16 : n;
                } else {
                    v = (int8_t)mat[i * pitch + cc];
                }
                if (SCALED) v *= (int32_t)scales[i * G + (cc >> 6)];
            }
            const uint32_t u = (uint32_t)(v + (int32_t)off);
            lo[c] += (uint64_t)el * u;
            hi[c] += (uint64_t)eh * u;
        }
    }
    const uint64_t corr = gl_mul(off, esum);
    uint64_t* o = part + (uint64_t)blockIdx.y * cols;
#pragma unroll
    for (int c = 0; c < kNaCols; c++)
        if (col0 + c < cols) o[col0 + c] = gl_sub(gl_add(gl_canon(lo[c]), gl_mul_2_32(gl_canon(hi[c]))), corr);
}

// out[c] = sum over splits of part[s][c] for c < cols, 0 for cols <= c < out_len.
__global__ void pe_noalloc_fin_kernel(const uint64_t* __restrict__ part, int splits, int cols, int64_t out_len,
                                      uint64_t* __restrict__ out) {
    const int64_t c = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (c >= out_len) return;
    if (c >= cols) {
        out[c] = 0;
        return;
    }
    uint64_t a = 0;
    for (int s = 0; s < splits; s++) a = gl_add(a, part[(int64_t)s * cols + c]);
    out[c] = a;
}

// Device address of the scratch array in the current device's context. Looked
// up on every call (once the module is loaded the lookup allocates nothing), so
// a context that was torn down and created again never gets a stale address.
int scratch_for_current_device(uint64_t** ptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
        cudaGetLastError();
        return FP_ERR_CUDA;
    }
    *ptr = (uint64_t*)p;
    return FP_OK;
}

}  // namespace

int mle_partial_eval_noalloc(const void* mat, int bits, const int8_t* scales, int rows, int cols,
                             const uint64_t* point, int npoint, uint64_t* out, void* stream) {
    if (!mat || !out || (npoint && !point)) return FP_ERR_ARG;
    if (bits != 4 && bits != 8) return FP_ERR_ARG;
    if (rows < 1 || cols < 1 || rows > (1 << 24) || cols > (1 << 24)) return FP_ERR_SHAPE;
    if (npoint != fp_log2_ceil((uint64_t)rows) || npoint > 24) return FP_ERR_SHAPE;
    for (int i = 0; i < npoint; i++)
        if (point[i] >= 0xFFFFFFFF00000001ull) return FP_ERR_ARG;
    const int splits = (rows + kNaRows - 1) / kNaRows;
    if ((uint64_t)splits * (uint64_t)cols > kNoallocWords) return FP_ERR_SHAPE;  // beyond the fixed scratch
    uint64_t* scratch = nullptr;
    int rc = scratch_for_current_device(&scratch);
    if (rc) return rc;

    NaPoint z;
    z.v = npoint;
    for (int i = 0; i < npoint; i++) z.z[i] = point[i];
    cudaStream_t s = (cudaStream_t)stream;
    dim3 grid((cols + kNaThreads * kNaCols - 1) / (kNaThreads * kNaCols), splits);
    const bool w4 = bits == 4, sc = scales != nullptr;
    const uint8_t* m = (const uint8_t*)mat;
    if (w4) {
        if (sc)
            pe_noalloc_acc_kernel<true, true><<<grid, kNaThreads, 0, s>>>(m, scales, rows, cols, z, scratch);
        else
            pe_noalloc_acc_kernel<true, false><<<grid, kNaThreads, 0, s>>>(m, scales, rows, cols, z, scratch);
    } else {
        if (sc)
            pe_noalloc_acc_kernel<false, true><<<grid, kNaThreads, 0, s>>>(m, scales, rows, cols, z, scratch);
        else
            pe_noalloc_acc_kernel<false, false><<<grid, kNaThreads, 0, s>>>(m, scales, rows, cols, z, scratch);
    }
    if (cudaGetLastError() != cudaSuccess) return FP_ERR_CUDA;
    const int64_t out_len = 1ll << fp_log2_ceil((uint64_t)cols);
    pe_noalloc_fin_kernel<<<(unsigned)((out_len + 255) / 256), 256, 0, s>>>(scratch, splits, cols, out_len, out);
    if (cudaGetLastError() != cudaSuccess) return FP_ERR_CUDA;
    return FP_OK;
}
