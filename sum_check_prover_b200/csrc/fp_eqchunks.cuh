// eq weights of a sum-check's first round from three small shared-memory tables.
//
// Round one of a sum-check over v variables with an eq(z, .) factor needs
// E_1[b] = eq(z_2..z_v, b) for every pair b. Splitting b's bits (most
// significant first) into chunks of widths w0 >= w1 >= w2 (each at most
// kEqChunk) gives E_1[b] as the product of three table entries, so each block
// builds the tables once (by doubling) and each pair costs two multiplications. Used by the
// LogUp-GKR layer sum-checks ("How fast can FlashProve go", 4 Tighter
// Rooflines: every tree level proven by sum-check) and by the gated-product
// sum-check (same page, 3.1: the gated product is handled by sum-check alone).
#pragma once
#include "fp_field.cuh"

// A table of width 0 is the single entry 1; the tables take 3 << kEqChunk
// entries of shared memory, so they cover up to 3 kEqChunk + 1 variables.
constexpr int kEqChunk = 10;

struct EqChunks {
    int w0, w1, w2;
};

__device__ __forceinline__ EqChunks eq_chunks_build(uint64_t* tab, const uint64_t* zs, int d) {
    const int nb = d - 1;  // coordinates z_2..z_d, i.e. zs[1..d-1]
    EqChunks C;
    C.w0 = nb < kEqChunk ? nb : kEqChunk;
    C.w1 = nb - C.w0 < kEqChunk ? nb - C.w0 : kEqChunk;
    C.w2 = nb - C.w0 - C.w1;
    const int b1 = 1 << C.w0, b2 = (1 << C.w0) + (1 << C.w1);  // where tables 1 and 2 start
    // Each table by doubling, in place: after step i the entry of prefix j (the first i of the
    // table's coordinates) sits at j 2^(w - i); step i splits it on the next coordinate z into
    // (1 - z) e at the same place and z e half a stride further. One product per entry.
    if (threadIdx.x < 3) tab[threadIdx.x == 0 ? 0 : (threadIdx.x == 1 ? b1 : b2)] = 1;
    __syncthreads();
    for (int i = 0; i < kEqChunk; i++) {
        const int n0 = i < C.w0 ? 1 << i : 0, n1 = i < C.w1 ? 1 << i : 0, n2 = i < C.w2 ? 1 << i : 0;
        if (n0 + n1 + n2 == 0) break;
        for (int x = threadIdx.x; x < n0 + n1 + n2; x += blockDim.x) {
            int j = x, w = C.w0, base = 0, first = 1;
            if (x >= n0 + n1) {
                j = x - n0 - n1; w = C.w2; base = b2; first = 1 + C.w0 + C.w1;
            } else if (x >= n0) {
                j = x - n0; w = C.w1; base = b1; first = 1 + C.w0;
            }
            const int stride = 1 << (w - i);
            uint64_t* e = tab + base + j * stride;
            const uint64_t hi = gl_mul(*e, zs[first + i]);
            e[stride >> 1] = hi;
            e[0] = gl_sub(e[0], hi);
        }
        __syncthreads();
    }
    return C;
}

__device__ __forceinline__ uint64_t eq_chunks_at(const EqChunks& C, const uint64_t* tab, int64_t b) {
    const int64_t i2 = b & ((1 << C.w2) - 1);
    const int64_t i1 = (b >> C.w2) & ((1 << C.w1) - 1);
    const int64_t i0 = b >> (C.w1 + C.w2);
    return gl_canon(gl_mul_weak(gl_mul_weak(tab[i0], tab[(1 << C.w0) + i1]), tab[(1 << C.w0) + (1 << C.w1) + i2]));
}

