// Goldilocks field arithmetic for sm_100a device code.
//
// p = 2^64 - 2^32 + 1 ("How fast can FlashProve go", 3.1: FlashProve's field).
// The reduction uses only the prime's shape: 2^64 = 2^32 - 1 (mod p) and
// 2^96 = -1 (mod p). A 128-bit product hi*2^64 + lo with hi = hh*2^32 + hl is
// therefore congruent to lo - hh + hl*(2^32 - 1); two conditional corrections
// by EPS = 2^32 - 1 absorb the 64-bit borrow and carry.
//
// Values are canonical (< p) unless a function says otherwise. gl_mul accepts
// any 64-bit inputs and returns a canonical value. The scalar operations also
// compile for the host, where the library assembles round polynomials and
// tracks running claims.
#pragma once
#include <stdint.h>

#ifdef __CUDACC__
#define GL_HD __host__ __device__ __forceinline__
#else
#define GL_HD inline
#endif

#define GL_P 0xFFFFFFFF00000001ull
#define GL_EPS 0x00000000FFFFFFFFull

GL_HD uint64_t gl_add(uint64_t a, uint64_t b) {
    uint64_t s = a + b;
    // carry out of 64 bits: the lost 2^64 is worth EPS; the result is then < p
    s += (s < a) ? GL_EPS : 0ull;
    return (s >= GL_P) ? s - GL_P : s;
}

GL_HD uint64_t gl_sub(uint64_t a, uint64_t b) {
    uint64_t d = a - b;
    // borrow: a - b + p = a - b + 2^64 - EPS
    return (a < b) ? d - GL_EPS : d;
}

GL_HD uint64_t gl_reduce128(uint64_t lo, uint64_t hi) {
    uint64_t hh = hi >> 32;
    uint64_t hl = hi & GL_EPS;
    uint64_t t0 = lo - hh;
    if (lo < hh) t0 -= GL_EPS;               // borrow worth -2^64 = -EPS
    uint64_t t1 = (hl << 32) - hl;           // hl * EPS, fits in 64 bits
    uint64_t r = t0 + t1;
    if (r < t1) r += GL_EPS;                 // carry worth EPS; cannot carry again
    return (r >= GL_P) ? r - GL_P : r;
}

GL_HD uint64_t gl_mul(uint64_t a, uint64_t b) {
#ifdef __CUDA_ARCH__
    return gl_reduce128(a * b, __umul64hi(a, b));
#else
    const unsigned __int128 x = (unsigned __int128)a * b;
    return gl_reduce128((uint64_t)x, (uint64_t)(x >> 64));
#endif
}

// a^e, and the inverse a^(p-2) (0 for a = 0)
GL_HD uint64_t gl_pow(uint64_t a, uint64_t e) {
    uint64_t r = 1;
    for (; e; e >>= 1) {
        if (e & 1) r = gl_mul(r, a);
        a = gl_mul(a, a);
    }
    return r;
}

GL_HD uint64_t gl_inv(uint64_t a) { return gl_pow(a, GL_P - 2); }

// Reduce an arbitrary 64-bit value into [0, p).
GL_HD uint64_t gl_canon(uint64_t a) { return (a >= GL_P) ? a - GL_P : a; }

// A signed 64-bit integer lifted into the field.
GL_HD uint64_t gl_from_i64(int64_t v) {
    return v >= 0 ? gl_canon((uint64_t)v) : gl_sub(0ull, gl_canon((uint64_t)(-(v + 1)) + 1ull));
}

// 2^32 * a (mod p) for a canonical a, via the reduction of (a >> 32, a << 32).
GL_HD uint64_t gl_mul_2_32(uint64_t a) { return gl_reduce128(a << 32, a >> 32); }

// a + r * (b - a): the sum-check fold of a pair by the challenge r.
GL_HD uint64_t gl_fold(uint64_t a, uint64_t b, uint64_t r) {
    return gl_add(a, gl_mul(r, gl_sub(b, a)));
}

// eq(z, x) for one Boolean x_b: x ? z : 1 - z
GL_HD uint64_t gl_eq1(uint64_t z, int bit) { return bit ? z : gl_sub(1ull, z); }

#ifdef __CUDACC__
// ---- throughput forms (device only) ------------------------------------------
//
// The hot loops are bound by integer ALU issue, not by the multiplier, so they
// avoid canonicalising intermediates: products are summed as exact 128-bit
// values in a 192-bit accumulator (GlAcc) and reduced once at the end, and a
// "weak" reduction returns a value < 2^64 that is congruent mod p but may be
// >= p. Carries go through PTX carry chains.

// Weakly reduced lo + 2^64 hi: congruent mod p, < 2^64 (not necessarily < p).
// lo - hh (+ 2^64 on borrow, worth -EPS) + hl * EPS (- 2^64 on carry, worth +EPS);
// neither correction can wrap again.
__device__ __forceinline__ uint64_t gl_reduce_weak(uint64_t lo, uint64_t hi) {
    const uint32_t hl = (uint32_t)hi, hh = (uint32_t)(hi >> 32);
    uint64_t r;
    asm("{\n\t"
        ".reg .u64 t0, t1, m64;\n\t"
        ".reg .u32 m;\n\t"
        "sub.cc.u64 t0, %1, %2;\n\t"
        "subc.u32 m, 0, 0;\n\t"
        "cvt.u64.u32 m64, m;\n\t"
        "sub.u64 t0, t0, m64;\n\t"
        "mul.wide.u32 t1, %3, 0xFFFFFFFF;\n\t"
        "add.cc.u64 %0, t0, t1;\n\t"
        "addc.u32 m, 0, 0;\n\t"
        "mul.wide.u32 m64, m, 0xFFFFFFFF;\n\t"
        "add.u64 %0, %0, m64;\n\t"
        "}"
        : "=l"(r)
        : "l"(lo), "l"((uint64_t)hh), "r"(hl));
    return r;
}

__device__ __forceinline__ uint64_t gl_mul_weak(uint64_t a, uint64_t b) {
    return gl_reduce_weak(a * b, __umul64hi(a, b));
}

// a + r (b - a) for canonical a, b: the 128-bit r (b - a) + a is reduced once.
__device__ __forceinline__ uint64_t gl_fold_fast(uint64_t a, uint64_t b, uint64_t r) {
    const uint64_t d = gl_sub(b, a);
    uint64_t lo = r * d, hi = __umul64hi(r, d);
    asm("add.cc.u64 %0, %0, %2;\n\taddc.u64 %1, %1, 0;" : "+l"(lo), "+l"(hi) : "l"(a));
    return gl_canon(gl_reduce_weak(lo, hi));
}

// a b + c for any 64-bit a, b, c (the 128-bit sum cannot overflow), weakly reduced
__device__ __forceinline__ uint64_t gl_muladd_weak(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t lo = a * b, hi = __umul64hi(a, b);
    asm("add.cc.u64 %0, %0, %2;\n\taddc.u64 %1, %1, 0;" : "+l"(lo), "+l"(hi) : "l"(c));
    return gl_reduce_weak(lo, hi);
}

// a v for canonical a and a small signed v (|v| < 2^31), canonical: the product
// of a and |v| has a high word below 2^31, worth hi * EPS
__device__ __forceinline__ uint64_t gl_mul_small(uint64_t a, int32_t v) {
    const uint32_t m = v < 0 ? (uint32_t)(-(int64_t)v) : (uint32_t)v;
    const uint64_t lo = a * m, hi = __umul64hi(a, (uint64_t)m);
    uint64_t r = lo + hi * GL_EPS;
    r += (r < lo) ? GL_EPS : 0ull;
    r = gl_canon(r);
    return v < 0 ? gl_sub(0ull, r) : r;
}

// Exact sum of up to 2^32 products of 64-bit values: lo + 2^64 hi + 2^128 top.
struct GlAcc {
    uint64_t lo = 0, hi = 0;
    uint32_t top = 0;
    __device__ __forceinline__ void mac(uint64_t a, uint64_t b) {
        const uint64_t plo = a * b, phi = __umul64hi(a, b);
        asm("add.cc.u64 %0, %0, %3;\n\taddc.cc.u64 %1, %1, %4;\n\taddc.u32 %2, %2, 0;"
            : "+l"(lo), "+l"(hi), "+r"(top)
            : "l"(plo), "l"(phi));
    }
    // a b for a 64-bit a and a 32-bit b: two 32 x 32 products, a_lo b + 2^32 a_hi b
    __device__ __forceinline__ void mac32(uint64_t a, uint32_t b) {
        const uint64_t p0 = (uint64_t)(uint32_t)a * b, p1 = (uint64_t)(uint32_t)(a >> 32) * b;
        const uint64_t plo = p0 + (p1 << 32);
        const uint64_t phi = (p1 >> 32) + (plo < p0 ? 1ull : 0ull);
        asm("add.cc.u64 %0, %0, %3;\n\taddc.cc.u64 %1, %1, %4;\n\taddc.u32 %2, %2, 0;"
            : "+l"(lo), "+l"(hi), "+r"(top)
            : "l"(plo), "l"(phi));
    }
    __device__ __forceinline__ void add(uint64_t a) {
        asm("add.cc.u64 %0, %0, %3;\n\taddc.cc.u64 %1, %1, 0;\n\taddc.u32 %2, %2, 0;"
            : "+l"(lo), "+l"(hi), "+r"(top)
            : "l"(a));
    }
    // canonical value: 2^128 = -2^32 (mod p)
    __device__ __forceinline__ uint64_t value() const {
        const uint64_t r = gl_canon(gl_reduce_weak(lo, hi));
        return gl_sub(r, gl_canon((uint64_t)top << 32));
    }
};

// 64-bit warp shuffles of field elements
__device__ __forceinline__ uint64_t shfl_xor_u64(uint64_t v, int m) {
    uint32_t lo = (uint32_t)v, hi = (uint32_t)(v >> 32);
    lo = __shfl_xor_sync(0xffffffffu, lo, m);
    hi = __shfl_xor_sync(0xffffffffu, hi, m);
    return ((uint64_t)hi << 32) | lo;
}

// lane src's 64-bit value
__device__ __forceinline__ uint64_t shfl_u64(uint64_t v, int src) {
    uint32_t lo = (uint32_t)v, hi = (uint32_t)(v >> 32);
    lo = __shfl_sync(0xffffffffu, lo, src);
    hi = __shfl_sync(0xffffffffu, hi, src);
    return ((uint64_t)hi << 32) | lo;
}

__device__ __forceinline__ uint64_t warp_sum_gl(uint64_t v) {
#pragma unroll
    for (int m = 16; m > 0; m >>= 1) v = gl_add(v, shfl_xor_u64(v, m));
    return v;
}
#endif
