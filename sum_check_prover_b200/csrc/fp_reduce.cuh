// Grid-wide sums of field elements: warp shuffles, a block tree in shared
// memory, then the last block to finish (atomic ticket) adds every block's
// partial. The ticket is left at zero for the next launch on the stream.
#pragma once
#include "fp_field.cuh"

// Sum NV values over the block; the totals are returned in every thread of warp 0
// (and are undefined elsewhere).
template <int NV>
__device__ __forceinline__ void block_sum_gl(uint64_t (&v)[NV]) {
    __shared__ uint64_t red[NV][32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = (blockDim.x + 31) >> 5;
#pragma unroll
    for (int k = 0; k < NV; k++) v[k] = warp_sum_gl(v[k]);
    __syncthreads();  // red may still be read by a previous call
    if (lane == 0) {
#pragma unroll
        for (int k = 0; k < NV; k++) red[k][warp] = v[k];
    }
    __syncthreads();
    if (warp == 0) {
#pragma unroll
        for (int k = 0; k < NV; k++) {
            uint64_t a = lane < nwarps ? red[k][lane] : 0ull;
            v[k] = warp_sum_gl(a);
        }
    }
}

// Every block contributes v; returns true in the last block, whose warp 0 then
// holds the grid totals in v. part needs NV * gridDim.x entries.
template <int NV>
__device__ __forceinline__ bool grid_sum_gl(uint64_t (&v)[NV], uint64_t* part, unsigned int* ticket) {
    __shared__ bool am_last;
    block_sum_gl<NV>(v);
    if (threadIdx.x == 0) {
#pragma unroll
        for (int k = 0; k < NV; k++) part[(size_t)blockIdx.x * NV + k] = v[k];
        __threadfence();
        unsigned int t = atomicAdd(ticket, 1u);
        am_last = (t == gridDim.x - 1);
    }
    __syncthreads();
    if (!am_last) return false;
    __threadfence();
    uint64_t acc[NV];
#pragma unroll
    for (int k = 0; k < NV; k++) acc[k] = 0;
    for (unsigned b = threadIdx.x; b < gridDim.x; b += blockDim.x)
#pragma unroll
        for (int k = 0; k < NV; k++) acc[k] = gl_add(acc[k], __ldcg(part + (size_t)b * NV + k));
    block_sum_gl<NV>(acc);
#pragma unroll
    for (int k = 0; k < NV; k++) v[k] = acc[k];
    if (threadIdx.x == 0) *ticket = 0u;
    return true;
}
