// Goldilocks field arithmetic for sm_100a device code.
//
// p = 2^64 - 2^32 + 1 ("How fast can FlashProve go", 3.1: FlashProve's field).
// The reduction uses only the prime's shape: 2^64 = 2^32 - 1 (mod p) and
// 2^96 = -1 (mod p). A 128-bit product hi*2^64 + lo with hi = hh*2^32 + hl is
// therefore congruent to lo - hh + hl*(2^32 - 1); two conditional corrections
// by EPS = 2^32 - 1 absorb the 64-bit borrow and carry.
//
// Values are canonical (< p) unless a function says otherwise. gl_mul accepts
// any 64-bit inputs and returns a canonical value.
#pragma once
#include <stdint.h>

#define GL_P 0xFFFFFFFF00000001ull
#define GL_EPS 0x00000000FFFFFFFFull

__device__ __forceinline__ uint64_t gl_add(uint64_t a, uint64_t b) {
    uint64_t s = a + b;
    // carry out of 64 bits: the lost 2^64 is worth EPS; the result is then < p
    s += (s < a) ? GL_EPS : 0ull;
    return (s >= GL_P) ? s - GL_P : s;
}

__device__ __forceinline__ uint64_t gl_sub(uint64_t a, uint64_t b) {
    uint64_t d = a - b;
    // borrow: a - b + p = a - b + 2^64 - EPS
    return (a < b) ? d - GL_EPS : d;
}

__device__ __forceinline__ uint64_t gl_reduce128(uint64_t lo, uint64_t hi) {
    uint64_t hh = hi >> 32;
    uint64_t hl = hi & GL_EPS;
    uint64_t t0 = lo - hh;
    if (lo < hh) t0 -= GL_EPS;               // borrow worth -2^64 = -EPS
    uint64_t t1 = (hl << 32) - hl;           // hl * EPS, fits in 64 bits
    uint64_t r = t0 + t1;
    if (r < t1) r += GL_EPS;                 // carry worth EPS; cannot carry again
    return (r >= GL_P) ? r - GL_P : r;
}

__device__ __forceinline__ uint64_t gl_mul(uint64_t a, uint64_t b) {
    return gl_reduce128(a * b, __umul64hi(a, b));
}

// Reduce an arbitrary 64-bit value into [0, p).
__device__ __forceinline__ uint64_t gl_canon(uint64_t a) { return (a >= GL_P) ? a - GL_P : a; }

// A signed 64-bit integer lifted into the field.
__device__ __forceinline__ uint64_t gl_from_i64(int64_t v) {
    return v >= 0 ? gl_canon((uint64_t)v) : gl_sub(0ull, gl_canon((uint64_t)(-(v + 1)) + 1ull));
}

// 2^32 * a (mod p) for a canonical a, via the reduction of (a >> 32, a << 32).
__device__ __forceinline__ uint64_t gl_mul_2_32(uint64_t a) { return gl_reduce128(a << 32, a >> 32); }

// a + r * (b - a): the sum-check fold of a pair by the challenge r.
__device__ __forceinline__ uint64_t gl_fold(uint64_t a, uint64_t b, uint64_t r) {
    return gl_add(a, gl_mul(r, gl_sub(b, a)));
}

// eq(z, x) for one Boolean x_b: x ? z : 1 - z
__device__ __forceinline__ uint64_t gl_eq1(uint64_t z, int bit) { return bit ? z : gl_sub(1ull, z); }

// 64-bit warp shuffles of field elements
__device__ __forceinline__ uint64_t shfl_xor_u64(uint64_t v, int m) {
    uint32_t lo = (uint32_t)v, hi = (uint32_t)(v >> 32);
    lo = __shfl_xor_sync(0xffffffffu, lo, m);
    hi = __shfl_xor_sync(0xffffffffu, hi, m);
    return ((uint64_t)hi << 32) | lo;
}

__device__ __forceinline__ uint64_t warp_sum_gl(uint64_t v) {
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) v = gl_add(v, shfl_xor_u64(v, m));
    return v;
}
