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

// The first `nblocks` blocks contribute v; returns true in the last of them to
// finish, whose warp 0 then holds the totals in v. part needs NV * nblocks
// entries; *ticket must be zero on entry and is zero again on return.
template <int NV>
__device__ __forceinline__ bool grid_sum_gl_n(uint64_t (&v)[NV], uint64_t* part, unsigned int* ticket,
                                              unsigned int nblocks) {
    __shared__ bool am_last;
    block_sum_gl<NV>(v);
    if (threadIdx.x == 0) {
#pragma unroll
        for (int k = 0; k < NV; k++) part[(size_t)blockIdx.x * NV + k] = v[k];
        __threadfence();
        unsigned int t = atomicAdd(ticket, 1u);
        am_last = (t == nblocks - 1);
    }
    __syncthreads();
    if (!am_last) return false;
    __threadfence();
    uint64_t acc[NV];
#pragma unroll
    for (int k = 0; k < NV; k++) acc[k] = 0;
    for (unsigned b = threadIdx.x; b < nblocks; b += blockDim.x)
#pragma unroll
        for (int k = 0; k < NV; k++) acc[k] = gl_add(acc[k], __ldcg(part + (size_t)b * NV + k));
    block_sum_gl<NV>(acc);
#pragma unroll
    for (int k = 0; k < NV; k++) v[k] = acc[k];
    if (threadIdx.x == 0) *ticket = 0u;
    return true;
}

// Every block of the grid contributes v (see grid_sum_gl_n).
template <int NV>
__device__ __forceinline__ bool grid_sum_gl(uint64_t (&v)[NV], uint64_t* part, unsigned int* ticket) {
    return grid_sum_gl_n<NV>(v, part, ticket, gridDim.x);
}
