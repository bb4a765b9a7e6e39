// The quadratic extension F_p[phi]/(phi^2 - 7) of the Goldilocks field.
//
// "How fast can FlashProve go", 4 (the note on soundness): challenges drawn
// from an extension of the base field make a sum-check's soundness error
// deg v / p^2 instead of deg v / p. 7 is not a square mod p (Euler's
// criterion: 7^((p-1)/2) = -1), so phi^2 = 7 defines the field of p^2
// elements; an element is a + b phi with a, b canonical, sent as a then b.
// A product takes three base multiplications (Karatsuba):
//   (a + b phi)(c + d phi) = (ac + 7 bd) + ((a + b)(c + d) - ac - bd) phi.
// The scalar forms compile for the host too, where round polynomials and
// running claims are assembled.
#pragma once
#include "fp_field.cuh"

struct alignas(16) Ext2 {
    uint64_t a, b;
};

GL_HD Ext2 e2_make(uint64_t a, uint64_t b) {
    Ext2 r;
    r.a = a;
    r.b = b;
    return r;
}

GL_HD Ext2 e2_add(Ext2 x, Ext2 y) { return e2_make(gl_add(x.a, y.a), gl_add(x.b, y.b)); }
GL_HD Ext2 e2_sub(Ext2 x, Ext2 y) { return e2_make(gl_sub(x.a, y.a), gl_sub(x.b, y.b)); }

// 7 x = 8 x - x for a canonical x
GL_HD uint64_t gl_mul7(uint64_t x) {
    const uint64_t x2 = gl_add(x, x), x4 = gl_add(x2, x2);
    return gl_sub(gl_add(x4, x4), x);
}

GL_HD Ext2 e2_mul(Ext2 x, Ext2 y) {
    const uint64_t ac = gl_mul(x.a, y.a), bd = gl_mul(x.b, y.b);
    const uint64_t m = gl_mul(gl_add(x.a, x.b), gl_add(y.a, y.b));
    return e2_make(gl_add(ac, gl_mul7(bd)), gl_sub(gl_sub(m, ac), bd));
}

// a base-field multiple
GL_HD Ext2 e2_scal(Ext2 x, uint64_t k) { return e2_make(gl_mul(x.a, k), gl_mul(x.b, k)); }

GL_HD bool e2_same(Ext2 x, Ext2 y) { return x.a == y.a && x.b == y.b; }

// eq(z, x) for one Boolean x: x ? z : 1 - z
GL_HD Ext2 e2_eq1(Ext2 z, int bit) { return bit ? z : e2_sub(e2_make(1, 0), z); }

// eq(z, r) = z r + (1 - z)(1 - r) for two extension elements
GL_HD Ext2 e2_eq(Ext2 z, Ext2 r) {
    const Ext2 one = e2_make(1, 0);
    return e2_add(e2_mul(z, r), e2_mul(e2_sub(one, z), e2_sub(one, r)));
}

// X = 2 on the line through (x, y) at 0 and 1
GL_HD Ext2 e2_at2(Ext2 x, Ext2 y) { return e2_sub(e2_add(y, y), x); }

#ifdef __CUDACC__
// ---- device forms ---------------------------------------------------------------

__device__ __forceinline__ Ext2 e2_ldcg(const Ext2* p) {
    const ulonglong2 q = __ldcg(reinterpret_cast<const ulonglong2*>(p));
    return e2_make(q.x, q.y);
}

// x + r (y - x): the fold of a pair by an extension challenge
__device__ __forceinline__ Ext2 e2_fold(Ext2 x, Ext2 y, Ext2 r) { return e2_add(x, e2_mul(r, e2_sub(y, x))); }

// Exact sums of extension products e p, kept as two base accumulators:
// a += e.a p.a + 7 e.b p.b, b += e.a p.b + e.b p.a.
struct E2Acc {
    GlAcc a, b;
    // e times a full extension element; e7b = 7 e.b (computed once per e)
    __device__ __forceinline__ void mac(Ext2 e, uint64_t e7b, Ext2 p) {
        a.mac(e.a, p.a);
        a.mac(e7b, p.b);
        b.mac(e.a, p.b);
        b.mac(e.b, p.a);
    }
    // e times a base-field element
    __device__ __forceinline__ void mac_base(Ext2 e, uint64_t p) {
        a.mac(e.a, p);
        b.mac(e.b, p);
    }
};
#endif
