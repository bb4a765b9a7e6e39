// Host-side helpers of the extension-field statements: extension challenges and
// values through the Fiat-Shamir transcript, and Lagrange interpolation at an
// extension point. An extension element a + b phi is squeezed as two base
// challenges under one label and sent as a then b (16 bytes, u64 little-endian).
#pragma once
#include "fp_ext2.cuh"
#include "fp_internal.h"

// a + r (b - a): a pair folded by an extension challenge
static inline Ext2 e2_fold_host(Ext2 a, Ext2 b, Ext2 r) { return e2_add(a, e2_mul(r, e2_sub(b, a))); }

// 1 / x = (a - b phi) / (a^2 - 7 b^2) (0 for 0)
static inline Ext2 e2_inv_host(Ext2 x) {
    const uint64_t ni = gl_inv(gl_sub(gl_mul(x.a, x.a), gl_mul(7, gl_mul(x.b, x.b))));
    return e2_make(gl_mul(x.a, ni), gl_sub(0, gl_mul(x.b, ni)));
}

// The round values g(0..3) of a layer round from the device's h(0), h(2) (and h(1), used only
// when z_t = 0): g(X) = pre eq(z_t, X) h(X), h of degree 2, and g(1) = claim - g(0), so that
// pre h(1) = g(1) / z_t. With ph = pre h: g(0) = (1 - z_t) ph(0), g(2) = (3 z_t - 1) ph(2),
// g(3) = (5 z_t - 2) ph(3), ph(3) = ph(0) - 3 ph(1) + 3 ph(2).
static inline void e2_layer_round_values(const Ext2 h[3], Ext2 pre, Ext2 zt, Ext2 claim, Ext2 g[4]) {
    const Ext2 one = e2_make(1, 0);
    const Ext2 ph0 = e2_mul(pre, h[0]), ph2 = e2_mul(pre, h[2]);
    g[0] = e2_mul(e2_sub(one, zt), ph0);
    g[1] = e2_sub(claim, g[0]);
    const bool z0 = zt.a == 0 && zt.b == 0;
    const Ext2 ph1 = z0 ? e2_mul(pre, h[1]) : e2_mul(g[1], e2_inv_host(zt));
    if (z0) g[1] = e2_make(0, 0);  // eq(0, 1) = 0
    g[2] = e2_mul(e2_sub(e2_scal(zt, 3), one), ph2);
    const Ext2 ph3 = e2_add(e2_sub(ph0, e2_scal(ph1, 3)), e2_scal(ph2, 3));
    g[3] = e2_mul(e2_sub(e2_scal(zt, 5), e2_make(2, 0)), ph3);
}

static inline Ext2 e2_squeeze_host(fp_tx* tx, const char* label) {
    const uint64_t a = fp_tx_squeeze_one(tx, label);
    const uint64_t b = fp_tx_squeeze_one(tx, label);
    return e2_make(a, b);
}

// n <= 8 extension elements into the proof at pos, absorbed under one label
static inline void e2_send_host(fp_tx* tx, const char* label, const Ext2* v, int n, uint8_t* proof, size_t& pos) {
    uint64_t w[16];
    for (int i = 0; i < n; i++) {
        w[2 * i] = v[i].a;
        w[2 * i + 1] = v[i].b;
    }
    put_u64s(proof + pos, w, 2 * (size_t)n);
    fp_tx_absorb_raw(tx, label, proof + pos, 16 * (uint64_t)n);
    pos += 16 * (size_t)n;
}

// the degree-2 polynomial through (i, g[i]), i = 0..2, at r:
// L0 = (r-1)(r-2)/2, L1 = -r(r-2), L2 = r(r-1)/2
static inline Ext2 e2_lagrange3(const Ext2 g[3], Ext2 r) {
    static const uint64_t inv2 = gl_inv(2);
    const Ext2 r1 = e2_sub(r, e2_make(1, 0)), r2 = e2_sub(r, e2_make(2, 0));
    const Ext2 l0 = e2_scal(e2_mul(r1, r2), inv2);
    const Ext2 l1 = e2_sub(e2_make(0, 0), e2_mul(r, r2));
    const Ext2 l2 = e2_scal(e2_mul(r, r1), inv2);
    return e2_add(e2_add(e2_mul(g[0], l0), e2_mul(g[1], l1)), e2_mul(g[2], l2));
}

// the degree-3 polynomial through (i, g[i]), i = 0..3, at r:
// L0 = -(r-1)(r-2)(r-3)/6, L1 = r(r-2)(r-3)/2, L2 = -r(r-1)(r-3)/2, L3 = r(r-1)(r-2)/6
static inline Ext2 e2_lagrange4(const Ext2 g[4], Ext2 r) {
    static const uint64_t inv2 = gl_inv(2), inv6 = gl_inv(6);
    const Ext2 r1 = e2_sub(r, e2_make(1, 0)), r2 = e2_sub(r, e2_make(2, 0)), r3 = e2_sub(r, e2_make(3, 0));
    const Ext2 zero = e2_make(0, 0);
    const Ext2 l0 = e2_sub(zero, e2_scal(e2_mul(e2_mul(r1, r2), r3), inv6));
    const Ext2 l1 = e2_scal(e2_mul(e2_mul(r, r2), r3), inv2);
    const Ext2 l2 = e2_sub(zero, e2_scal(e2_mul(e2_mul(r, r1), r3), inv2));
    const Ext2 l3 = e2_scal(e2_mul(e2_mul(r, r1), r2), inv6);
    return e2_add(e2_add(e2_mul(g[0], l0), e2_mul(g[1], l1)), e2_add(e2_mul(g[2], l2), e2_mul(g[3], l3)));
}
