// Histograms of lookup keys over tables larger than one block's shared memory.
//
// A lookup's multiplicities m_j count the keys equal to table row j ("How fast can FlashProve
// go", 4: LogUp compares the keys' fractions with the table's, weighted by m). Counting with
// one global atomic per key is bound by same-address atomics whenever the keys are
// concentrated (a SiLU lookup's inputs are a projection's int8 outputs: a few hundred rows of
// 65536). Here a thread-block cluster holds the whole table in distributed shared memory:
// CTA c of a cluster owns rows [c 2^s, (c + 1) 2^s) and every key is counted by an atomic on
// its owner's shared memory. Keys in a small window around zero, where concentrated keys sit,
// are counted in the counting CTA's own shared memory first. At the end every cluster writes
// its rows to a partial table with plain stores and one pass sums the partial tables.
#pragma once

#include <cooperative_groups.h>

#include "fp_internal.h"

namespace fp_hist {
namespace {

namespace cg = cooperative_groups;

// rows per CTA of the distributed table, and the local window [-kWin16, kWin16) of the
// 16-bit key histogram
constexpr int kShareBits = 15;
constexpr int kWin16 = 1 << 11;
constexpr int kThreads = 1024;

// m[key + 2^15] counts of n int16 keys, table of 2^16 rows held by a cluster of two CTAs.
// part: (gridDim.x / 2) rows of 2^16 words, written in full; the window's counts go to m
// by global atomics (m zeroed by the caller).
__global__ void __launch_bounds__(kThreads) hist16_cluster_kernel(const int16_t* __restrict__ g, int64_t n,
                                                                  uint32_t* __restrict__ part,
                                                                  uint32_t* __restrict__ m) {
    extern __shared__ uint32_t sh[];
    cg::cluster_group cl = cg::this_cluster();
    const unsigned crank = cl.block_rank();
    uint32_t* share = sh;                     // 2^15 rows: [crank 2^15, (crank + 1) 2^15)
    uint32_t* win = sh + (1 << kShareBits);  // 2 kWin16 rows around key 0
    for (int i = threadIdx.x; i < (1 << kShareBits); i += blockDim.x) share[i] = 0;
    for (int i = threadIdx.x; i < 2 * kWin16; i += blockDim.x) win[i] = 0;
    cl.sync();  // every CTA's share is zero before any CTA counts into it
    uint32_t* const own0 = cl.map_shared_rank(share, 0);
    uint32_t* const own1 = cl.map_shared_rank(share, 1);
    auto count = [&](int v) {
        if (v >= -kWin16 && v < kWin16) {
            atomicAdd(&win[v + kWin16], 1u);
        } else {
            const int j = v + 32768;
            atomicAdd(((j >> kShareBits) ? own1 : own0) + (j & ((1 << kShareBits) - 1)), 1u);
        }
    };
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    int64_t done = 0;
    if ((uintptr_t)g % 16 == 0) {
        const int64_t n8 = n / 8;
        const int4* g8 = reinterpret_cast<const int4*>(g);
        for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n8; i += stride) {
            const int4 w = __ldcs(g8 + i);
            const uint32_t u[4] = {(uint32_t)w.x, (uint32_t)w.y, (uint32_t)w.z, (uint32_t)w.w};
#pragma unroll
            for (int e = 0; e < 4; e++) {
                count((int16_t)(u[e] & 0xFFFF));
                count((int16_t)(u[e] >> 16));
            }
        }
        done = 8 * n8;
    }
    for (int64_t i = done + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) count(g[i]);
    cl.sync();  // every count has landed; no CTA leaves while another may still count into it
    uint32_t* row = part + (size_t)(blockIdx.x >> 1) * 65536 + ((size_t)crank << kShareBits);
    for (int i = threadIdx.x; i < (1 << kShareBits); i += blockDim.x) row[i] = share[i];
    for (int i = threadIdx.x; i < 2 * kWin16; i += blockDim.x)
        if (win[i]) atomicAdd(&m[i - kWin16 + 32768], win[i]);
}

// one global atomic per key: the fallback when no cluster of two fits
__global__ void hist16_global_kernel(const int16_t* __restrict__ g, int64_t n, uint32_t* __restrict__ m) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        atomicAdd(m + ((int)g[i] + 32768), 1u);
}

// m[j] += sum over the rows of part[row][j] (+ pad at row pad_at), j < T
__global__ void hist_rows_sum_kernel(const uint32_t* __restrict__ part, int rows, int64_t T, uint32_t* __restrict__ m,
                                     int64_t pad_at, uint32_t pad) {
    for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < T; j += (int64_t)gridDim.x * blockDim.x) {
        uint32_t s = m[j];
        for (int r = 0; r < rows; r++) s += __ldcs(part + (size_t)r * T + j);
        if (j == pad_at) s += pad;
        m[j] = s;
    }
}

// Launch `kernel` on clusters of `csize` CTAs of kThreads threads with `smem` bytes of dynamic
// shared memory each, as many clusters as fit on the GPU at once (at most max_clusters); the
// cluster count launched in *clusters. Returns cudaSuccess or the launch's error (the caller
// then takes its fallback path).
template <typename... Args, typename... Act>
cudaError_t launch_clusters(void (*kernel)(Args...), int csize, int smem, int max_clusters, cudaStream_t st,
                                   int* clusters, Act... args) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = csize;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.blockDim = dim3(kThreads);
    cfg.gridDim = dim3(csize);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    int nc = 0;
    e = cudaOccupancyMaxActiveClusters(&nc, kernel, &cfg);
    if (e != cudaSuccess) return e;
    if (nc < 1) return cudaErrorInvalidConfiguration;
    nc = nc < max_clusters ? nc : max_clusters;
    cfg.gridDim = dim3(nc * csize);
    *clusters = nc;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Rows of the partial tables a cluster histogram may write: one per cluster, at most one
// cluster per SM pair for the 16-bit table.
constexpr int kMaxClusters16 = 128;
inline size_t hist16_scratch() { return fp_align_up((size_t)kMaxClusters16 * 65536 * 4, 256); }

// The 2^16-row histogram of n int16 keys into m (zeroed here), the padding keys (pad of them,
// all key 0) included. part: hist16_scratch() bytes of device scratch. Two launches, on st.
inline int hist16(fp_ctx* c, const int16_t* g, int64_t n, uint32_t pad, uint32_t* m, uint32_t* part,
                         cudaStream_t st) {
    FP_CUDA(c, cudaMemsetAsync(m, 0, 4 * 65536, st));
    int clusters = 0;
    const int smem = 4 * ((1 << kShareBits) + 2 * kWin16);
    if (launch_clusters(hist16_cluster_kernel, 2, smem, kMaxClusters16, st, &clusters, g, n, part, m) != cudaSuccess) {
        (void)cudaGetLastError();  // no cluster launch here: count with global atomics
        clusters = 0;
        hist16_global_kernel<<<fp_grid256(c, n), 256, 0, st>>>(g, n, m);
        FP_CUDA(c, cudaGetLastError());
    }
    hist_rows_sum_kernel<<<fp_grid256(c, 65536), 256, 0, st>>>(part, clusters, 65536, m, 32768, pad);
    FP_CUDA(c, cudaGetLastError());
    c->launches += 1;  // the summing pass; the caller's timing counts the histogram launch
    return FP_OK;
}

}  // namespace
}  // namespace fp_hist
