/*
 * oracle.c -- reference prover and verifier for the quantised-matmul sum-check
 * with LogUp rescale/clamp lookups.
 *
 * TEST INFRASTRUCTURE ONLY. This file is the slow, obviously-correct CPU
 * statement of what the CUDA library computes. Only the test-suite, the smoke
 * check and the benchmark's CPU-baseline / reference arm load it. It shares no
 * code, header, table or helper with the CUDA library: the library must reach
 * the same bytes on its own.
 *
 * Style rules kept on purpose: single-threaded; every field operation is
 * (unsigned __int128 arithmetic) % P; every sum is the plain loop of its
 * definition; no blocking, fusion or reordering.
 *
 * Sources (page title, section):
 *  - "How fast can FlashProve go", 2 Background: the prover commits the
 *    intermediate values; sum-check reduces each polynomial operation (the
 *    matmuls) to claims on committed values and weights; non-polynomial steps
 *    (rescale, clamp) are proven by lookups; Fiat-Shamir makes each challenge
 *    a hash of everything sent so far.
 *  - same page, 3.1 Committing intermediate values: a rescale
 *    g = round(g_hat / 2^k) is proven by committing the remainder
 *    r = g_hat - 2^k g, using 2^k g + r in place of g_hat in the matmul
 *    sum-check, and looking r up to show it is small; the field is Goldilocks
 *    2^64 - 2^32 + 1.
 *  - same page, 2 Background and 2.1 Batching: many claims are merged into one
 *    (here: random linear combination of per-matmul claims).
 *  - same page, 4 Tighter Rooflines: a lookup compares a product over the keys
 *    with one over the table; the key side is a binary tree whose every level
 *    is proven with sum-check.
 *  - "Towards Proving Frontier-Scale LLM Inference", How the prover works /
 *    The proof system: lookups by logarithmic derivatives (LogUp), whose
 *    fractions we sum in the same binary tree.
 * Every point the pages leave open (transcript encoding, bit order, rounding
 * tie, table layout, batching of the two lookups) follows the protocol
 * specification written out in the repository's design notes; the choices
 * are repeated next to the code that makes them.
 */
#include <stdint.h>
#include <math.h>
#include <stdlib.h>
#include <string.h>

typedef uint64_t u64;
typedef uint32_t u32;
typedef unsigned __int128 u128;

#define ORC_P 0xFFFFFFFF00000001ull

/* ------------------------------------------------------------------------ */
/* Goldilocks field: canonical representatives in [0, P).                    */
/* ------------------------------------------------------------------------ */

u64 orc_fadd(u64 a, u64 b) { return (u64)(((u128)a + (u128)b) % ORC_P); }
u64 orc_fsub(u64 a, u64 b) { return (u64)(((u128)a + (u128)ORC_P - (u128)(b % ORC_P)) % ORC_P); }
u64 orc_fmul(u64 a, u64 b) { return (u64)(((u128)a * (u128)b) % ORC_P); }

u64 orc_fpow(u64 a, u64 e) {
    u64 r = 1, b = a % ORC_P;
    while (e) {
        if (e & 1) r = orc_fmul(r, b);
        b = orc_fmul(b, b);
        e >>= 1;
    }
    return r;
}

/* Fermat: a^(P-2) is the inverse of a non-zero a. */
u64 orc_finv(u64 a) { return orc_fpow(a, ORC_P - 2); }

/* A signed integer lifted into the field: v mod P in [0, P). */
u64 orc_fint(int64_t v) {
    if (v >= 0) return (u64)v % ORC_P;
    u64 mag = (u64)(-(v + 1)) + 1u; /* |v| without overflow */
    return orc_fsub(0, mag % ORC_P);
}

/* ------------------------------------------------------------------------ */
/* SHA-256, written from FIPS 180-4 (sections 4.1.2, 4.2.2, 5.1.1, 6.2).      */
/* ------------------------------------------------------------------------ */

static const u32 SHA_K[64] = {
    0x428a2f98, 0x71374491, 0xb5c0fbcf, 0xe9b5dba5, 0x3956c25b, 0x59f111f1, 0x923f82a4, 0xab1c5ed5,
    0xd807aa98, 0x12835b01, 0x243185be, 0x550c7dc3, 0x72be5d74, 0x80deb1fe, 0x9bdc06a7, 0xc19bf174,
    0xe49b69c1, 0xefbe4786, 0x0fc19dc6, 0x240ca1cc, 0x2de92c6f, 0x4a7484aa, 0x5cb0a9dc, 0x76f988da,
    0x983e5152, 0xa831c66d, 0xb00327c8, 0xbf597fc7, 0xc6e00bf3, 0xd5a79147, 0x06ca6351, 0x14292967,
    0x27b70a85, 0x2e1b2138, 0x4d2c6dfc, 0x53380d13, 0x650a7354, 0x766a0abb, 0x81c2c92e, 0x92722c85,
    0xa2bfe8a1, 0xa81a664b, 0xc24b8b70, 0xc76c51a3, 0xd192e819, 0xd6990624, 0xf40e3585, 0x106aa070,
    0x19a4c116, 0x1e376c08, 0x2748774c, 0x34b0bcb5, 0x391c0cb3, 0x4ed8aa4a, 0x5b9cca4f, 0x682e6ff3,
    0x748f82ee, 0x78a5636f, 0x84c87814, 0x8cc70208, 0x90befffa, 0xa4506ceb, 0xbef9a3f7, 0xc67178f2};

typedef struct {
    u32 h[8];
    uint8_t buf[64];
    u64 total; /* bytes fed so far */
    u32 fill;  /* bytes waiting in buf */
} sha_ctx;

static u32 rotr32(u32 x, int n) { return (x >> n) | (x << (32 - n)); }

static void sha_compress(u32 h[8], const uint8_t blk[64]) {
    u32 w[64];
    for (int t = 0; t < 16; t++)
        w[t] = ((u32)blk[4 * t] << 24) | ((u32)blk[4 * t + 1] << 16) | ((u32)blk[4 * t + 2] << 8) |
               (u32)blk[4 * t + 3];
    for (int t = 16; t < 64; t++) {
        u32 s0 = rotr32(w[t - 15], 7) ^ rotr32(w[t - 15], 18) ^ (w[t - 15] >> 3);
        u32 s1 = rotr32(w[t - 2], 17) ^ rotr32(w[t - 2], 19) ^ (w[t - 2] >> 10);
        w[t] = w[t - 16] + s0 + w[t - 7] + s1;
    }
    u32 a = h[0], b = h[1], c = h[2], d = h[3], e = h[4], f = h[5], g = h[6], hh = h[7];
    for (int t = 0; t < 64; t++) {
        u32 S1 = rotr32(e, 6) ^ rotr32(e, 11) ^ rotr32(e, 25);
        u32 ch = (e & f) ^ (~e & g);
        u32 T1 = hh + S1 + ch + SHA_K[t] + w[t];
        u32 S0 = rotr32(a, 2) ^ rotr32(a, 13) ^ rotr32(a, 22);
        u32 mj = (a & b) ^ (a & c) ^ (b & c);
        u32 T2 = S0 + mj;
        hh = g; g = f; f = e; e = d + T1; d = c; c = b; b = a; a = T1 + T2;
    }
    h[0] += a; h[1] += b; h[2] += c; h[3] += d; h[4] += e; h[5] += f; h[6] += g; h[7] += hh;
}

static void sha_init(sha_ctx* c) {
    static const u32 H0[8] = {0x6a09e667, 0xbb67ae85, 0x3c6ef372, 0xa54ff53a,
                              0x510e527f, 0x9b05688c, 0x1f83d9ab, 0x5be0cd19};
    memcpy(c->h, H0, sizeof H0);
    c->total = 0;
    c->fill = 0;
}

static void sha_update(sha_ctx* c, const void* data, u64 n) {
    const uint8_t* p = (const uint8_t*)data;
    c->total += n;
    while (n > 0) {
        u32 take = 64 - c->fill;
        if (take > n) take = (u32)n;
        memcpy(c->buf + c->fill, p, take);
        c->fill += take;
        p += take;
        n -= take;
        if (c->fill == 64) {
            sha_compress(c->h, c->buf);
            c->fill = 0;
        }
    }
}

static void sha_final(sha_ctx* c, uint8_t out[32]) {
    u64 bits = c->total * 8u;
    uint8_t one = 0x80, zero = 0;
    sha_update(c, &one, 1);
    while (c->fill != 56) sha_update(c, &zero, 1);
    uint8_t lenb[8];
    for (int i = 0; i < 8; i++) lenb[i] = (uint8_t)(bits >> (56 - 8 * i));
    sha_update(c, lenb, 8);
    for (int i = 0; i < 8; i++) {
        out[4 * i] = (uint8_t)(c->h[i] >> 24);
        out[4 * i + 1] = (uint8_t)(c->h[i] >> 16);
        out[4 * i + 2] = (uint8_t)(c->h[i] >> 8);
        out[4 * i + 3] = (uint8_t)(c->h[i]);
    }
}

void orc_sha256(const void* data, u64 n, uint8_t out[32]) {
    sha_ctx c;
    sha_init(&c);
    sha_update(&c, data, n);
    sha_final(&c, out);
}

static void put_le(uint8_t* p, u64 v, int nbytes) {
    for (int i = 0; i < nbytes; i++) p[i] = (uint8_t)(v >> (8 * i));
}

static u64 get_le(const uint8_t* p, int nbytes) {
    u64 v = 0;
    for (int i = 0; i < nbytes; i++) v |= (u64)p[i] << (8 * i);
    return v;
}

/*
 * Tree digest of a byte string (binds the committed buffers into the
 * transcript; the pages' commitment scheme itself is out of scope).
 *   level 0: SHA-256 of each 1024-byte chunk (the last one may be short; an
 *            empty string has one empty chunk);
 *   level l+1: SHA-256 of each run of up to 32 consecutive level-l digests;
 *   until one digest is left; result = SHA-256(u64le(len) || that digest).
 */
#define ORC_CHUNK 1024u
void orc_tree_digest(const void* data, u64 len, uint8_t out[32]) {
    const uint8_t* p = (const uint8_t*)data;
    u64 cnt = len == 0 ? 1 : (len + ORC_CHUNK - 1) / ORC_CHUNK;
    uint8_t* lv = (uint8_t*)malloc(cnt * 32);
    for (u64 c = 0; c < cnt; c++) {
        u64 off = c * ORC_CHUNK;
        u64 n = len - off < ORC_CHUNK ? len - off : ORC_CHUNK;
        if (len == 0) n = 0;
        orc_sha256(p + off, n, lv + 32 * c);
    }
    while (cnt > 1) {
        u64 nc = (cnt + 31) / 32;
        uint8_t* nx = (uint8_t*)malloc(nc * 32);
        for (u64 g = 0; g < nc; g++) {
            u64 m = cnt - 32 * g < 32 ? cnt - 32 * g : 32;
            orc_sha256(lv + 32 * 32 * g, 32 * m, nx + 32 * g);
        }
        free(lv);
        lv = nx;
        cnt = nc;
    }
    uint8_t fin[40];
    put_le(fin, len, 8);
    memcpy(fin + 8, lv, 32);
    orc_sha256(fin, 40, out);
    free(lv);
}

/* ------------------------------------------------------------------------ */
/* Fiat-Shamir transcript ("How fast can FlashProve go", 2 Background: each   */
/* challenge hashes everything the prover sent; SHA-256 instead of BLAKE2b).  */
/*   state0 = SHA256("FPSC-v1" || u64le(seed))                                */
/*   absorb: state = SHA256(state || u32le(|label|) || label || u64le(n) || data) */
/*   squeeze: h = SHA256(state || "sq" || u32le(|label|) || label || u32le(ctr)) */
/*            for ctr = 0, 1, ...; the first h whose low 8 bytes (LE) are < P  */
/*            becomes the state and that value the challenge.                 */
/* ------------------------------------------------------------------------ */

typedef struct {
    uint8_t st[32];
} orc_tx;

void orc_tx_init(orc_tx* t, u64 seed) {
    uint8_t b[15];
    memcpy(b, "FPSC-v1", 7);
    put_le(b + 7, seed, 8);
    orc_sha256(b, 15, t->st);
}

void orc_tx_absorb(orc_tx* t, const char* label, const void* data, u64 n) {
    sha_ctx c;
    uint8_t l4[4], l8[8];
    u32 ll = (u32)strlen(label);
    sha_init(&c);
    sha_update(&c, t->st, 32);
    put_le(l4, ll, 4);
    sha_update(&c, l4, 4);
    sha_update(&c, label, ll);
    put_le(l8, n, 8);
    sha_update(&c, l8, 8);
    sha_update(&c, data, n);
    sha_final(&c, t->st);
}

u64 orc_tx_squeeze(orc_tx* t, const char* label) {
    u32 ll = (u32)strlen(label);
    for (u32 ctr = 0;; ctr++) {
        sha_ctx c;
        uint8_t l4[4], c4[4], h[32];
        sha_init(&c);
        sha_update(&c, t->st, 32);
        sha_update(&c, "sq", 2);
        put_le(l4, ll, 4);
        sha_update(&c, l4, 4);
        sha_update(&c, label, ll);
        put_le(c4, ctr, 4);
        sha_update(&c, c4, 4);
        sha_final(&c, h);
        u64 v = get_le(h, 8);
        if (v < ORC_P) {
            memcpy(t->st, h, 32);
            return v;
        }
    }
}

/* ctypes-facing transcript handle */
void* orc_tx_new(u64 seed) {
    orc_tx* t = (orc_tx*)malloc(sizeof(orc_tx));
    orc_tx_init(t, seed);
    return t;
}
void orc_tx_free(void* t) { free(t); }
void orc_tx_state(const void* t, uint8_t out[32]) { memcpy(out, ((const orc_tx*)t)->st, 32); }
void orc_tx_absorb_h(void* t, const char* label, const void* d, u64 n) { orc_tx_absorb((orc_tx*)t, label, d, n); }
u64 orc_tx_squeeze_h(void* t, const char* label) { return orc_tx_squeeze((orc_tx*)t, label); }

/* ------------------------------------------------------------------------ */
/* Multilinear extensions. A vector of length 2^v is indexed by             */
/* x = sum_b x_b 2^(v-b): the first coordinate z_1 of a point binds the MSB. */
/* eq(z, x) = prod_b (z_b x_b + (1 - z_b)(1 - x_b)).                          */
/* ------------------------------------------------------------------------ */

int orc_log2_ceil(u64 n) {
    int v = 0;
    while (((u64)1 << v) < n) v++;
    return v;
}

/* eq table by doubling: start [1]; step b maps entry j to 2j (times 1 - z_b)
 * and 2j+1 (times z_b), so z_1 ends up on the most significant bit. */
void orc_eq_table(const u64* z, int v, u64* out) {
    out[0] = 1;
    for (int b = 0; b < v; b++) {
        u64 len = (u64)1 << b;
        for (u64 j = len; j-- > 0;) {
            u64 o = out[j];
            out[2 * j] = orc_fmul(o, orc_fsub(1, z[b]));
            out[2 * j + 1] = orc_fmul(o, z[b]);
        }
    }
}

/* MLE of vals (length n, zero-padded to 2^v) at z: sum_x eq(z, x) vals[x]. */
u64 orc_mle_eval(const u64* vals, u64 n, const u64* z, int v) {
    u64 sz = (u64)1 << v;
    u64* e = (u64*)malloc(sz * sizeof(u64));
    orc_eq_table(z, v, e);
    u64 acc = 0;
    for (u64 x = 0; x < n && x < sz; x++) acc = orc_fadd(acc, orc_fmul(e[x], vals[x]));
    free(e);
    return acc;
}

/* Evaluate the polynomial of degree npts-1 through (i, g[i]), i = 0..npts-1, at x. */
u64 orc_lagrange(const u64* g, int npts, u64 x) {
    u64 acc = 0;
    for (int i = 0; i < npts; i++) {
        u64 num = 1, den = 1;
        for (int j = 0; j < npts; j++) {
            if (j == i) continue;
            num = orc_fmul(num, orc_fsub(x, (u64)j));
            den = orc_fmul(den, orc_fsub((u64)i, (u64)j));
        }
        acc = orc_fadd(acc, orc_fmul(g[i], orc_fmul(num, orc_finv(den))));
    }
    return acc;
}

/* ------------------------------------------------------------------------ */
/* Sites: one matrix product Y = W . X per site.                              */
/*   W: M x K, int8, or int4 packed two per byte along K (low nibble = even   */
/*      k, two's complement, ceil(K/2) bytes per row); optional int8 scales  */
/*      per 64-column group: W_eff[i][k] = S[i][k/64] * w[i][k].             */
/*   X: stored transposed, xt = N x K int8 (token-major).                    */
/*   outputs q, r (int32) and y (int8), stored N x M (token-major).          */
/* ------------------------------------------------------------------------ */

typedef struct {
    const void* w;
    const int8_t* scales;
    const int8_t* xt;
    int32_t w_bits, M, K, N, k_shift, pad;
} orc_site;

typedef struct {
    int32_t* q;
    int32_t* r;
    int8_t* y;
} orc_wit;

static int64_t w_eff(const orc_site* s, int i, int k) {
    int64_t w;
    if (s->w_bits == 8) {
        w = ((const int8_t*)s->w)[(u64)i * s->K + k];
    } else {
        const uint8_t* row = (const uint8_t*)s->w + (u64)i * ((s->K + 1) / 2);
        int nib = (k & 1) ? (row[k / 2] >> 4) : (row[k / 2] & 15);
        w = nib >= 8 ? nib - 16 : nib;
    }
    if (s->scales) w *= s->scales[(u64)i * ((s->K + 63) / 64) + k / 64];
    return w;
}

static int64_t floordiv_pow2(int64_t a, int k) {
    int64_t d = (int64_t)1 << k;
    int64_t q = a / d;
    if (a % d != 0 && a < 0) q -= 1;
    return q;
}

/* Witness of one site ("How fast can FlashProve go", 3.1): Y = W_eff . X in
 * integers; q = floor((Y + 2^(k-1)) / 2^k) (round half up), r = Y - 2^k q,
 * y = clamp(q, -128, 127). Returns 0, or -1 if some |Y| needs more than 31
 * bits (the accepted input domain). */
int orc_witness(const orc_site* s, int32_t* q, int32_t* r, int8_t* y) {
    int M = s->M, K = s->K, N = s->N, k = s->k_shift;
    int64_t* wrow = (int64_t*)malloc(sizeof(int64_t) * (K > 0 ? K : 1));
    int bad = 0;
    for (int i = 0; i < M; i++) {
        for (int kk = 0; kk < K; kk++) wrow[kk] = w_eff(s, i, kk);
        for (int j = 0; j < N; j++) {
            const int8_t* xr = s->xt + (u64)j * K;
            int64_t acc = 0;
            for (int kk = 0; kk < K; kk++) acc += wrow[kk] * (int64_t)xr[kk];
            if (acc > 2147483647LL || acc < -2147483648LL) bad = 1;
            int64_t qq = floordiv_pow2(acc + ((int64_t)1 << (k - 1)), k);
            int64_t rr = acc - (qq << k);
            u64 o = (u64)j * M + i;
            q[o] = (int32_t)qq;
            r[o] = (int32_t)rr;
            y[o] = (int8_t)(qq < -128 ? -128 : (qq > 127 ? 127 : qq));
        }
    }
    free(wrow);
    return bad ? -1 : 0;
}

/* A_s[k] = sum_i eq(z, i) W_eff[i][k] for k < K, zero up to 2^ceil(log2 K).
 * z has ceil(log2 M) coordinates. */
void orc_partial_w(const orc_site* s, const u64* z, int v, u64* out) {
    u64 Kp = (u64)1 << orc_log2_ceil((u64)s->K);
    u64* e = (u64*)malloc(sizeof(u64) << v);
    orc_eq_table(z, v, e);
    for (u64 k = 0; k < Kp; k++) out[k] = 0;
    for (int i = 0; i < s->M; i++)
        for (int k = 0; k < s->K; k++) out[k] = orc_fadd(out[k], orc_fmul(e[i], orc_fint(w_eff(s, i, k))));
    free(e);
}

/* B_s[k] = sum_j eq(z, j) X[k][j] = sum_j eq(z, j) xt[j][k]; z has ceil(log2 N) coordinates. */
void orc_partial_x(const orc_site* s, const u64* z, int v, u64* out) {
    u64 Kp = (u64)1 << orc_log2_ceil((u64)s->K);
    u64* e = (u64*)malloc(sizeof(u64) << v);
    orc_eq_table(z, v, e);
    for (u64 k = 0; k < Kp; k++) out[k] = 0;
    for (int j = 0; j < s->N; j++)
        for (int k = 0; k < s->K; k++)
            out[k] = orc_fadd(out[k], orc_fmul(e[j], orc_fint(s->xt[(u64)j * s->K + k])));
    free(e);
}

/* Generic row contraction used by the library's partial-evaluation entry
 * point: out[c] = sum_{i<rows} eq(z, i) (S[i][c/64] *) mat[i][c]. */
void orc_partial_rows(const void* mat, int bits, const int8_t* scales, int rows, int cols,
                      const u64* z, int v, u64* out) {
    orc_site s;
    memset(&s, 0, sizeof s);
    s.w = mat;
    s.w_bits = bits;
    s.scales = scales;
    s.M = rows;
    s.K = cols;
    orc_partial_w(&s, z, v, out);
}

/* Output claim c = sum_{i,j} eq(zr, i) eq(zc, j) (2^k q[i,j] + r[i,j]): the MLE
 * of Y = 2^k q + r at (zr, zc), row bits first ("How fast can FlashProve go", 3.1). */
u64 orc_claim(const int32_t* q, const int32_t* r, int M, int N, int k, const u64* zr, int vr,
              const u64* zc, int vc) {
    u64* er = (u64*)malloc(sizeof(u64) << vr);
    u64* ec = (u64*)malloc(sizeof(u64) << vc);
    orc_eq_table(zr, vr, er);
    orc_eq_table(zc, vc, ec);
    u64 two_k = orc_fint((int64_t)1 << k);
    u64 acc = 0;
    for (int i = 0; i < M; i++)
        for (int j = 0; j < N; j++) {
            u64 o = (u64)j * M + i;
            u64 yv = orc_fadd(orc_fmul(two_k, orc_fint(q[o])), orc_fint(r[o]));
            acc = orc_fadd(acc, orc_fmul(orc_fmul(er[i], ec[j]), yv));
        }
    free(er);
    free(ec);
    return acc;
}

/* Direct MLE of W_eff (padded to 2^vr x 2^n) at (zr, rho): sum_{i,k} eq eq W. */
static u64 mle_w_direct(const orc_site* s, const u64* zr, int vr, const u64* rho, int n) {
    u64* er = (u64*)malloc(sizeof(u64) << vr);
    u64* ek = (u64*)malloc(sizeof(u64) << n);
    orc_eq_table(zr, vr, er);
    orc_eq_table(rho, n, ek);
    u64 acc = 0;
    for (int i = 0; i < s->M; i++)
        for (int k = 0; k < s->K; k++)
            acc = orc_fadd(acc, orc_fmul(orc_fmul(er[i], ek[k]), orc_fint(w_eff(s, i, k))));
    free(er);
    free(ek);
    return acc;
}

/* Direct MLE of X (padded) at (rho, zc), K bits first then N bits. */
static u64 mle_x_direct(const orc_site* s, const u64* rho, int n, const u64* zc, int vc) {
    u64* ek = (u64*)malloc(sizeof(u64) << n);
    u64* ec = (u64*)malloc(sizeof(u64) << vc);
    orc_eq_table(rho, n, ek);
    orc_eq_table(zc, vc, ec);
    u64 acc = 0;
    for (int k = 0; k < s->K; k++)
        for (int j = 0; j < s->N; j++)
            acc = orc_fadd(acc, orc_fmul(orc_fmul(ek[k], ec[j]), orc_fint(s->xt[(u64)j * s->K + k])));
    free(ek);
    free(ec);
    return acc;
}

/* ------------------------------------------------------------------------ */
/* Proof byte buffer: every prover message is appended (u64 LE field        */
/* elements, u32 LE multiplicities) and absorbed under its label.            */
/* ------------------------------------------------------------------------ */

typedef struct {
    uint8_t* p;
    u64 cap, len;
    int overflow;
} pbuf;

static void pb_put(pbuf* b, const void* d, u64 n) {
    if (b->len + n > b->cap) {
        b->overflow = 1;
    } else if (n) {
        memcpy(b->p + b->len, d, n);
    }
    b->len += n;
}

/* send field elements: append and absorb */
static void send_fe(orc_tx* t, pbuf* b, const char* label, const u64* v, u64 n) {
    uint8_t* tmp = (uint8_t*)malloc(8 * (n ? n : 1));
    for (u64 i = 0; i < n; i++) put_le(tmp + 8 * i, v[i], 8);
    pb_put(b, tmp, 8 * n);
    orc_tx_absorb(t, label, tmp, 8 * n);
    free(tmp);
}

/* send a multiplicity table: the raw u32 LE words go into the proof, their
 * tree digest into the transcript. */
static void send_mult(orc_tx* t, pbuf* b, const char* label, const u32* m, u64 n) {
    uint8_t* tmp = (uint8_t*)malloc(4 * n);
    uint8_t dg[32];
    for (u64 i = 0; i < n; i++) put_le(tmp + 4 * i, m[i], 4);
    pb_put(b, tmp, 4 * n);
    orc_tree_digest(tmp, 4 * n, dg);
    orc_tx_absorb(t, label, dg, 32);
    free(tmp);
}

static u64 site_w_bytes(const orc_site* s) {
    return (u64)s->M * (s->w_bits == 4 ? (u64)((s->K + 1) / 2) : (u64)s->K);
}

/* Witness commitment into the transcript: per site, in site order, absorb
 * "site" with D(W) || D(S) || D(X) || D(q) || D(r) || D(y) (D = tree digest of
 * the stored bytes; D(S) of an empty string when there are no scales). */
static void absorb_sites(orc_tx* t, const orc_site* sites, int ns, const orc_wit* wit) {
    for (int s = 0; s < ns; s++) {
        const orc_site* st = &sites[s];
        uint8_t d[192];
        u64 mn = (u64)st->M * st->N;
        orc_tree_digest(st->w, site_w_bytes(st), d);
        orc_tree_digest(st->scales, st->scales ? (u64)st->M * ((st->K + 63) / 64) : 0, d + 32);
        orc_tree_digest(st->xt, (u64)st->N * st->K, d + 64);
        orc_tree_digest(wit[s].q, 4 * mn, d + 96);
        orc_tree_digest(wit[s].r, 4 * mn, d + 128);
        orc_tree_digest(wit[s].y, mn, d + 160);
        orc_tx_absorb(t, "site", d, 192);
    }
}

/* ------------------------------------------------------------------------ */
/* Matmul sum-check with batched claims.                                     */
/* vM = max ceil(log2 M_s), vN = max ceil(log2 N_s), n = max ceil(log2 K_s); */
/* r_row (vM), r_col (vN) squeezed; site s uses their first m_s / nn_s       */
/* coordinates. c_s sent; if more than one site, rho_s squeezed (else 1).    */
/* Round t over padded length-2^n vectors A_s, B_s: g(X) at X = 0, 1, 2 of   */
/* sum_s rho_s sum_b A_s(X, b) B_s(X, b); then r_t and the MSB fold.         */
/* Finally the per-site A_s(rho), B_s(rho).                                  */
/* ------------------------------------------------------------------------ */

static int site_dims(const orc_site* sites, int ns, int* vM, int* vN, int* n) {
    *vM = *vN = *n = 0;
    for (int s = 0; s < ns; s++) {
        int a = orc_log2_ceil((u64)sites[s].M), b = orc_log2_ceil((u64)sites[s].N),
            c = orc_log2_ceil((u64)sites[s].K);
        if (a > *vM) *vM = a;
        if (b > *vN) *vN = b;
        if (c > *n) *n = c;
    }
    return 0;
}

/* The point where the last matmul section (proven or verified) left its sites: the row
 * challenges r_row (vM), the round challenges rho (n) and the final values A_s(rho), B_s(rho).
 * The FFN statement continues from it. (The oracle is single-threaded.) */
#define MM_PT_MAX 64
static struct {
    int vM, n, ns;
    u64 rr[MM_PT_MAX], rho[MM_PT_MAX];
    u64* fin; /* 2 ns values */
} g_mm_pt = {0, 0, 0, {0}, {0}, NULL};

static void mm_pt_record(int vM, const u64* rr, int n, const u64* rho, int ns, const u64* fin) {
    g_mm_pt.vM = vM;
    g_mm_pt.n = n;
    g_mm_pt.ns = ns;
    for (int i = 0; i < vM && i < MM_PT_MAX; i++) g_mm_pt.rr[i] = rr[i];
    for (int i = 0; i < n && i < MM_PT_MAX; i++) g_mm_pt.rho[i] = rho[i];
    free(g_mm_pt.fin);
    g_mm_pt.fin = (u64*)malloc(sizeof(u64) * 2 * (size_t)ns);
    for (int i = 0; i < 2 * ns; i++) g_mm_pt.fin[i] = fin[i];
}

static void mm_prove(orc_tx* t, pbuf* pb, const orc_site* sites, int ns, const orc_wit* wit) {
    int vM, vN, n;
    site_dims(sites, ns, &vM, &vN, &n);
    u64* rr = (u64*)malloc(sizeof(u64) * (vM + 1));
    u64* rc = (u64*)malloc(sizeof(u64) * (vN + 1));
    for (int i = 0; i < vM; i++) rr[i] = orc_tx_squeeze(t, "r_row");
    for (int i = 0; i < vN; i++) rc[i] = orc_tx_squeeze(t, "r_col");

    u64* c = (u64*)malloc(sizeof(u64) * ns);
    for (int s = 0; s < ns; s++) {
        int ms = orc_log2_ceil((u64)sites[s].M), nn = orc_log2_ceil((u64)sites[s].N);
        c[s] = orc_claim(wit[s].q, wit[s].r, sites[s].M, sites[s].N, sites[s].k_shift, rr, ms, rc, nn);
    }
    send_fe(t, pb, "claims", c, (u64)ns);

    u64* rho = (u64*)malloc(sizeof(u64) * ns);
    if (ns == 1)
        rho[0] = 1;
    else
        for (int s = 0; s < ns; s++) rho[s] = orc_tx_squeeze(t, "rho");

    u64 L = (u64)1 << n;
    u64** A = (u64**)malloc(sizeof(u64*) * ns);
    u64** B = (u64**)malloc(sizeof(u64*) * ns);
    for (int s = 0; s < ns; s++) {
        int ms = orc_log2_ceil((u64)sites[s].M), nn = orc_log2_ceil((u64)sites[s].N);
        A[s] = (u64*)calloc(L, sizeof(u64));
        B[s] = (u64*)calloc(L, sizeof(u64));
        orc_partial_w(&sites[s], rr, ms, A[s]);
        orc_partial_x(&sites[s], rc, nn, B[s]);
    }

    u64* chal = (u64*)malloc(sizeof(u64) * (n + 1));
    for (int t_ = 0; t_ < n; t_++) {
        u64 h = L >> 1;
        u64 g[3] = {0, 0, 0};
        for (int s = 0; s < ns; s++) {
            u64 g0 = 0, g1 = 0, g2 = 0;
            for (u64 b = 0; b < h; b++) {
                u64 a0 = A[s][b], a1 = A[s][h + b], b0 = B[s][b], b1 = B[s][h + b];
                u64 a2 = orc_fsub(orc_fmul(2, a1), a0), b2 = orc_fsub(orc_fmul(2, b1), b0);
                g0 = orc_fadd(g0, orc_fmul(a0, b0));
                g1 = orc_fadd(g1, orc_fmul(a1, b1));
                g2 = orc_fadd(g2, orc_fmul(a2, b2));
            }
            g[0] = orc_fadd(g[0], orc_fmul(rho[s], g0));
            g[1] = orc_fadd(g[1], orc_fmul(rho[s], g1));
            g[2] = orc_fadd(g[2], orc_fmul(rho[s], g2));
        }
        send_fe(t, pb, "sc_round", g, 3);
        u64 r = orc_tx_squeeze(t, "sc_chal");
        chal[t_] = r;
        for (int s = 0; s < ns; s++)
            for (u64 b = 0; b < h; b++) {
                A[s][b] = orc_fadd(A[s][b], orc_fmul(r, orc_fsub(A[s][h + b], A[s][b])));
                B[s][b] = orc_fadd(B[s][b], orc_fmul(r, orc_fsub(B[s][h + b], B[s][b])));
            }
        L = h;
    }
    u64* fin = (u64*)malloc(sizeof(u64) * 2 * ns);
    for (int s = 0; s < ns; s++) {
        fin[2 * s] = A[s][0];
        fin[2 * s + 1] = B[s][0];
    }
    send_fe(t, pb, "sc_final", fin, 2 * (u64)ns);
    mm_pt_record(vM, rr, n, chal, ns, fin);
    for (int s = 0; s < ns; s++) {
        free(A[s]);
        free(B[s]);
    }
    free(A); free(B); free(fin); free(rho); free(c); free(rr); free(rc); free(chal);
}

/* ------------------------------------------------------------------------ */
/* LogUp lookups of the rescale remainders and of the clamp pairs.           */
/* Table 0 (remainder range): t_j = j - 2^(k-1), j < 2^k; key = r.           */
/* Table 1 (clamp, also bounds q to 16 bits): t_j = v_j + gamma clamp(v_j),  */
/*   v_j = j - 2^15, j < 2^16; key = q + gamma y.                            */
/* Keys: every site's outputs in storage order, sites concatenated, padded  */
/* to 2^v (v >= 1) with the neutral key 0 (r = 0; q = y = 0).                */
/* Key side as a binary tree of fractions: leaves (1, alpha - f); parent     */
/* (pL qR + pR qL, qL qR) of children 2x, 2x+1. The two trees have the same  */
/* shape and are proven together, layer by layer, in one sum-check whose    */
/* terms are combined with powers of lambda.                                 */
/* ------------------------------------------------------------------------ */

typedef struct {
    u64 nk;       /* real keys */
    int v;        /* tree depth */
    int k;        /* rescale shift */
    /* stored at the witness's own widths (r, q int32, y int8), so the key
     * columns of the largest layer (2^29 keys) take 9 bytes a key */
    int32_t* fr;  /* remainder keys (padded) */
    int32_t* fq;  /* q component (padded) */
    int8_t* fy;   /* y component (padded) */
} orc_keys;

static int keys_build(const orc_site* sites, int ns, const orc_wit* wit, orc_keys* K) {
    u64 nk = 0;
    int k = sites[0].k_shift;
    for (int s = 0; s < ns; s++) {
        nk += (u64)sites[s].M * sites[s].N;
        if (sites[s].k_shift != k) return -1;
    }
    int v = orc_log2_ceil(nk);
    if (v < 1) v = 1;
    u64 L = (u64)1 << v;
    K->nk = nk;
    K->v = v;
    K->k = k;
    K->fr = (int32_t*)calloc(L, sizeof(int32_t));
    K->fq = (int32_t*)calloc(L, sizeof(int32_t));
    K->fy = (int8_t*)calloc(L, sizeof(int8_t));
    u64 o = 0;
    for (int s = 0; s < ns; s++) {
        u64 mn = (u64)sites[s].M * sites[s].N;
        for (u64 e = 0; e < mn; e++, o++) {
            K->fr[o] = wit[s].r[e];
            K->fq[o] = wit[s].q[e];
            K->fy[o] = wit[s].y[e];
        }
    }
    return 0;
}

static void keys_free(orc_keys* K) {
    free(K->fr);
    free(K->fq);
    free(K->fy);
}

/* Multiplicities, counted by the key's table index; a key outside a table's
 * range is counted nowhere (its lookup then fails at the verifier). */
static void mult_rem(const orc_keys* K, u32* m) {
    u64 T = (u64)1 << K->k, L = (u64)1 << K->v;
    int64_t half = (int64_t)1 << (K->k - 1);
    memset(m, 0, T * sizeof(u32));
    for (u64 i = 0; i < L; i++) {
        int64_t j = (int64_t)K->fr[i] + half;
        if (j >= 0 && (u64)j < T) m[j]++;
    }
}

static void mult_clamp(const orc_keys* K, u32* m) {
    u64 L = (u64)1 << K->v;
    memset(m, 0, 65536 * sizeof(u32));
    for (u64 i = 0; i < L; i++) {
        int64_t j = (int64_t)K->fq[i] + 32768;
        if (j >= 0 && j < 65536) m[j]++;
    }
}

static u64 key_field(const orc_keys* K, int tab, u64 i, u64 gamma) {
    if (tab == 0) return orc_fint(K->fr[i]);
    return orc_fadd(orc_fint(K->fq[i]), orc_fmul(gamma, orc_fint(K->fy[i])));
}

/* layers[d] has 2^d nodes; P at [0], Q at [1]. */
typedef struct {
    u64** P;
    u64** Q;
    int v;
} orc_tree;

static void tree_build(const orc_keys* K, int tab, u64 alpha, u64 gamma, orc_tree* T) {
    int v = K->v;
    T->v = v;
    T->P = (u64**)malloc(sizeof(u64*) * (v + 1));
    T->Q = (u64**)malloc(sizeof(u64*) * (v + 1));
    u64 L = (u64)1 << v;
    T->P[v] = (u64*)malloc(L * sizeof(u64));
    T->Q[v] = (u64*)malloc(L * sizeof(u64));
    for (u64 i = 0; i < L; i++) {
        T->P[v][i] = 1;
        T->Q[v][i] = orc_fsub(alpha, key_field(K, tab, i, gamma));
    }
    for (int d = v - 1; d >= 0; d--) {
        u64 n = (u64)1 << d;
        T->P[d] = (u64*)malloc(n * sizeof(u64));
        T->Q[d] = (u64*)malloc(n * sizeof(u64));
        for (u64 x = 0; x < n; x++) {
            u64 pl = T->P[d + 1][2 * x], pr = T->P[d + 1][2 * x + 1];
            u64 ql = T->Q[d + 1][2 * x], qr = T->Q[d + 1][2 * x + 1];
            T->P[d][x] = orc_fadd(orc_fmul(pl, qr), orc_fmul(pr, ql));
            T->Q[d][x] = orc_fmul(ql, qr);
        }
    }
}

static void tree_free(orc_tree* T) {
    for (int d = 0; d <= T->v; d++) {
        free(T->P[d]);
        free(T->Q[d]);
    }
    free(T->P);
    free(T->Q);
}

/* the summand of one layer: sum over tables tau of
 * lambda^(2 tau) (pL qR + pR qL + lambda qL qR) */
static u64 layer_F(const u64 v8[8], u64 lam, u64 lam2) {
    u64 acc = 0, w = 1;
    for (int tau = 0; tau < 2; tau++) {
        const u64* x = v8 + 4 * tau; /* pL, pR, qL, qR */
        u64 f = orc_fadd(orc_fadd(orc_fmul(x[0], x[3]), orc_fmul(x[1], x[2])),
                         orc_fmul(lam, orc_fmul(x[2], x[3])));
        acc = orc_fadd(acc, orc_fmul(w, f));
        w = lam2;
    }
    return acc;
}

static void lu_prove(orc_tx* t, pbuf* pb, const orc_site* sites, int ns, const orc_wit* wit) {
    orc_keys K;
    keys_build(sites, ns, wit, &K);
    int v = K.v;
    u64 Trem = (u64)1 << K.k;
    u32* mr = (u32*)malloc(Trem * sizeof(u32));
    u32* mc = (u32*)malloc(65536 * sizeof(u32));

    mult_rem(&K, mr);
    send_mult(t, pb, "logup_m_rem", mr, Trem);
    u64 gamma = orc_tx_squeeze(t, "logup_gamma");
    mult_clamp(&K, mc);
    send_mult(t, pb, "logup_m_clamp", mc, 65536);
    u64 alpha[2];
    alpha[0] = orc_tx_squeeze(t, "logup_alpha");
    alpha[1] = orc_tx_squeeze(t, "logup_alpha");

    orc_tree T[2];
    tree_build(&K, 0, alpha[0], gamma, &T[0]);
    tree_build(&K, 1, alpha[1], gamma, &T[1]);

    /* layer 1 (two nodes per tree) is sent in the clear */
    u64 l1[8];
    for (int tau = 0; tau < 2; tau++) {
        l1[4 * tau + 0] = T[tau].P[1][0];
        l1[4 * tau + 1] = T[tau].P[1][1];
        l1[4 * tau + 2] = T[tau].Q[1][0];
        l1[4 * tau + 3] = T[tau].Q[1][1];
    }
    send_fe(t, pb, "gkr_l1", l1, 8);
    u64 mu = orc_tx_squeeze(t, "gkr_mu");
    u64* z = (u64*)malloc(sizeof(u64) * (v + 1));
    z[0] = mu;

    for (int d = 1; d < v; d++) {
        u64 lam = orc_tx_squeeze(t, "gkr_lambda");
        u64 lam2 = orc_fmul(lam, lam);
        u64 n = (u64)1 << d;
        /* vectors: for tau: pL, pR, qL, qR (children of layer d in layer d+1), then eq(z, .) */
        u64* V[9];
        for (int tau = 0; tau < 2; tau++) {
            for (int i = 0; i < 4; i++) V[4 * tau + i] = (u64*)malloc(n * sizeof(u64));
            for (u64 x = 0; x < n; x++) {
                V[4 * tau + 0][x] = T[tau].P[d + 1][2 * x];
                V[4 * tau + 1][x] = T[tau].P[d + 1][2 * x + 1];
                V[4 * tau + 2][x] = T[tau].Q[d + 1][2 * x];
                V[4 * tau + 3][x] = T[tau].Q[d + 1][2 * x + 1];
            }
            /* level d + 1 is read by no later layer: release it now, which keeps
             * the prover of the largest layer within a workstation's memory */
            free(T[tau].P[d + 1]);
            free(T[tau].Q[d + 1]);
            T[tau].P[d + 1] = T[tau].Q[d + 1] = NULL;
        }
        V[8] = (u64*)malloc(n * sizeof(u64));
        orc_eq_table(z, d, V[8]);
        u64 L = n;
        u64* rho = (u64*)malloc(sizeof(u64) * d);
        for (int r = 0; r < d; r++) {
            u64 h = L >> 1;
            u64 g[4] = {0, 0, 0, 0};
            for (u64 b = 0; b < h; b++)
                for (u64 X = 0; X < 4; X++) {
                    u64 ev[9];
                    for (int i = 0; i < 9; i++)
                        ev[i] = orc_fadd(V[i][b], orc_fmul(X, orc_fsub(V[i][h + b], V[i][b])));
                    g[X] = orc_fadd(g[X], orc_fmul(ev[8], layer_F(ev, lam, lam2)));
                }
            send_fe(t, pb, "gkr_round", g, 4);
            rho[r] = orc_tx_squeeze(t, "gkr_chal");
            for (int i = 0; i < 9; i++)
                for (u64 b = 0; b < h; b++)
                    V[i][b] = orc_fadd(V[i][b], orc_fmul(rho[r], orc_fsub(V[i][h + b], V[i][b])));
            L = h;
        }
        u64 fin[8];
        for (int i = 0; i < 8; i++) fin[i] = V[i][0];
        send_fe(t, pb, "gkr_final", fin, 8);
        mu = orc_tx_squeeze(t, "gkr_mu");
        for (int r = 0; r < d; r++) z[r] = rho[r];
        z[d] = mu;
        for (int i = 0; i < 9; i++) free(V[i]);
        free(rho);
    }

    /* leaf claims: MLEs of the padded r, q, y key columns at z (v coords) */
    u64 Lk = (u64)1 << v;
    u64* col = (u64*)malloc(Lk * sizeof(u64));
    u64 leaf[3];
    for (u64 i = 0; i < Lk; i++) col[i] = orc_fint(K.fr[i]);
    leaf[0] = orc_mle_eval(col, Lk, z, v);
    for (u64 i = 0; i < Lk; i++) col[i] = orc_fint(K.fq[i]);
    leaf[1] = orc_mle_eval(col, Lk, z, v);
    for (u64 i = 0; i < Lk; i++) col[i] = orc_fint(K.fy[i]);
    leaf[2] = orc_mle_eval(col, Lk, z, v);
    send_fe(t, pb, "leaf", leaf, 3);

    free(col);
    free(z);
    tree_free(&T[0]);
    tree_free(&T[1]);
    free(mr);
    free(mc);
    keys_free(&K);
}

/*
 * Full prover. Writes the proof (matmul section, then lookup section) and the
 * transcript state after each stage (commit, matmul, lookup) into states[96].
 * sec_off[0] = byte length of the matmul section. Returns 0, -1 on bad input,
 * -2 if the proof buffer is too small (*len then holds the size needed).
 */
int orc_prove(u64 seed, const orc_site* sites, int ns, const orc_wit* wit, uint8_t* proof, u64 cap,
              u64* len, uint8_t states[96], u64* sec_off) {
    if (ns < 1) return -1;
    for (int s = 0; s < ns; s++)
        if (sites[s].M < 1 || sites[s].N < 1 || sites[s].K < 1 || sites[s].k_shift < 1 ||
            sites[s].k_shift > 30 || (sites[s].w_bits != 4 && sites[s].w_bits != 8) ||
            sites[s].k_shift != sites[0].k_shift)
            return -1;
    orc_tx t;
    pbuf pb = {proof, cap, 0, 0};
    orc_tx_init(&t, seed);
    absorb_sites(&t, sites, ns, wit);
    memcpy(states, t.st, 32);
    mm_prove(&t, &pb, sites, ns, wit);
    memcpy(states + 32, t.st, 32);
    *sec_off = pb.len;
    lu_prove(&t, &pb, sites, ns, wit);
    memcpy(states + 64, t.st, 32);
    *len = pb.len;
    return pb.overflow ? -2 : 0;
}

/* ------------------------------------------------------------------------ */
/* Verifier. Replays the transcript from the witness it holds (standing in   */
/* for the openings of the committed values and weights) and checks every   */
/* protocol relation. Integer facts of the witness (Y = 2^k q + r, ranges,   */
/* y = clamp(q)) are NOT checked directly: only the protocol may reject.     */
/* Returns 0 on accept or a reason code; detail[0..1] locate the failure.    */
/* ------------------------------------------------------------------------ */

enum {
    REJ_FORMAT = 1,       /* truncated proof, trailing bytes or non-canonical element */
    REJ_CLAIM = 2,        /* c_s differs from the committed output's MLE */
    REJ_MM_ROUND = 3,     /* matmul sum-check round: g(0) + g(1) != claim */
    REJ_MM_FINAL = 4,     /* last matmul claim != sum_s rho_s A_s B_s */
    REJ_MM_A = 5,         /* A_s(rho) != W_s MLE */
    REJ_MM_B = 6,         /* B_s(rho) != X_s MLE */
    REJ_ROOT_REM = 7,     /* remainder lookup: key fraction != table fraction */
    REJ_ROOT_CLAMP = 8,   /* clamp lookup: key fraction != table fraction */
    REJ_GKR_ROUND = 9,    /* layer sum-check round inconsistent */
    REJ_GKR_FINAL = 10,   /* layer end: eq * F != claim */
    REJ_LEAF_P = 11,      /* leaf numerator MLE != 1 */
    REJ_LEAF_Q = 12,      /* leaf denominator != alpha - key MLE */
    REJ_LEAF_OPEN = 13,   /* leaf column claims != committed columns' MLE */
    REJ_ARGS = 14         /* statement malformed */
};

typedef struct {
    const uint8_t* p;
    u64 len, pos;
    int bad;
} prd;

static void rd_fe(orc_tx* t, prd* r, const char* label, u64* out, u64 n) {
    if (r->bad || r->pos + 8 * n > r->len) {
        r->bad = 1;
        for (u64 i = 0; i < n; i++) out[i] = 0;
        return;
    }
    const uint8_t* src = r->p + r->pos;
    for (u64 i = 0; i < n; i++) {
        out[i] = get_le(src + 8 * i, 8);
        if (out[i] >= ORC_P) r->bad = 1;
    }
    orc_tx_absorb(t, label, src, 8 * n);
    r->pos += 8 * n;
}

static void rd_mult(orc_tx* t, prd* r, const char* label, u32* out, u64 n) {
    if (r->bad || r->pos + 4 * n > r->len) {
        r->bad = 1;
        memset(out, 0, 4 * n);
        return;
    }
    const uint8_t* src = r->p + r->pos;
    uint8_t dg[32];
    for (u64 i = 0; i < n; i++) out[i] = (u32)get_le(src + 4 * i, 4);
    orc_tree_digest(src, 4 * n, dg);
    orc_tx_absorb(t, label, dg, 32);
    r->pos += 4 * n;
}

#define FAIL(code, a, b)         \
    do {                         \
        rc = (code);             \
        detail[0] = (a);         \
        detail[1] = (b);         \
        goto done;               \
    } while (0)

/* Verification options for statements too large to check in full: a site
 * whose mask entry is 0 skips the direct recomputation of its claim and of its
 * A/B evaluations (every other check still runs); VERIFY_SKIP_LEAF_OPEN skips
 * recomputing the key columns' MLEs. NULL mask and flags 0 = full verification. */
#define VERIFY_SKIP_LEAF_OPEN 4
static const uint8_t* g_site_mask = NULL;
static int g_verify_flags = 0;
static int site_checked(int s) { return g_site_mask == NULL || g_site_mask[s]; }

static int mm_verify(orc_tx* t, prd* rd, const orc_site* sites, int ns, const orc_wit* wit,
                     int64_t* detail) {
    int rc = 0, vM, vN, n;
    site_dims(sites, ns, &vM, &vN, &n);
    u64* rr = (u64*)malloc(sizeof(u64) * (vM + 1));
    u64* rc_ = (u64*)malloc(sizeof(u64) * (vN + 1));
    u64* c = (u64*)malloc(sizeof(u64) * ns);
    u64* rho = (u64*)malloc(sizeof(u64) * ns);
    u64* pt = (u64*)malloc(sizeof(u64) * (n + 1));
    u64* fin = (u64*)malloc(sizeof(u64) * 2 * ns);
    for (int i = 0; i < vM; i++) rr[i] = orc_tx_squeeze(t, "r_row");
    for (int i = 0; i < vN; i++) rc_[i] = orc_tx_squeeze(t, "r_col");
    rd_fe(t, rd, "claims", c, (u64)ns);
    if (rd->bad) FAIL(REJ_FORMAT, 0, 0);
    for (int s = 0; s < ns; s++) {
        if (!site_checked(s)) continue;
        int ms = orc_log2_ceil((u64)sites[s].M), nn = orc_log2_ceil((u64)sites[s].N);
        u64 want = orc_claim(wit[s].q, wit[s].r, sites[s].M, sites[s].N, sites[s].k_shift, rr, ms, rc_, nn);
        if (want != c[s]) FAIL(REJ_CLAIM, s, 0);
    }
    if (ns == 1)
        rho[0] = 1;
    else
        for (int s = 0; s < ns; s++) rho[s] = orc_tx_squeeze(t, "rho");
    u64 claim = 0;
    for (int s = 0; s < ns; s++) claim = orc_fadd(claim, orc_fmul(rho[s], c[s]));
    for (int r = 0; r < n; r++) {
        u64 g[3];
        rd_fe(t, rd, "sc_round", g, 3);
        if (rd->bad) FAIL(REJ_FORMAT, 1, r);
        if (orc_fadd(g[0], g[1]) != claim) FAIL(REJ_MM_ROUND, r, 0);
        pt[r] = orc_tx_squeeze(t, "sc_chal");
        claim = orc_lagrange(g, 3, pt[r]);
    }
    rd_fe(t, rd, "sc_final", fin, 2 * (u64)ns);
    if (rd->bad) FAIL(REJ_FORMAT, 2, 0);
    mm_pt_record(vM, rr, n, pt, ns, fin);
    {
        u64 acc = 0;
        for (int s = 0; s < ns; s++) acc = orc_fadd(acc, orc_fmul(rho[s], orc_fmul(fin[2 * s], fin[2 * s + 1])));
        if (acc != claim) FAIL(REJ_MM_FINAL, 0, 0);
    }
    for (int s = 0; s < ns; s++) {
        if (!site_checked(s)) continue;
        int ms = orc_log2_ceil((u64)sites[s].M), nn = orc_log2_ceil((u64)sites[s].N);
        if (mle_w_direct(&sites[s], rr, ms, pt, n) != fin[2 * s]) FAIL(REJ_MM_A, s, 0);
        if (mle_x_direct(&sites[s], pt, n, rc_, nn) != fin[2 * s + 1]) FAIL(REJ_MM_B, s, 0);
    }
done:
    free(rr); free(rc_); free(c); free(rho); free(pt); free(fin);
    return rc;
}

/* fraction sum over a table: sum_j m_j / (alpha - t_j), kept as (num, den) */
static void table_fraction(const u32* m, u64 T, int tab, int k, u64 alpha, u64 gamma, u64* num, u64* den) {
    u64 P = 0, Q = 1;
    for (u64 j = 0; j < T; j++) {
        u64 tj;
        if (tab == 0) {
            tj = orc_fint((int64_t)j - ((int64_t)1 << (k - 1)));
        } else {
            int64_t vj = (int64_t)j - 32768;
            int64_t cj = vj < -128 ? -128 : (vj > 127 ? 127 : vj);
            tj = orc_fadd(orc_fint(vj), orc_fmul(gamma, orc_fint(cj)));
        }
        u64 d = orc_fsub(alpha, tj);
        /* P/Q + m/d = (P d + m Q) / (Q d) */
        P = orc_fadd(orc_fmul(P, d), orc_fmul((u64)m[j], Q));
        Q = orc_fmul(Q, d);
    }
    *num = P;
    *den = Q;
}

static int lu_verify(orc_tx* t, prd* rd, const orc_site* sites, int ns, const orc_wit* wit,
                     int64_t* detail) {
    int rc = 0;
    orc_keys K;
    if (keys_build(sites, ns, wit, &K) != 0) {
        detail[0] = detail[1] = 0;
        return REJ_ARGS;
    }
    int v = K.v;
    u64 Trem = (u64)1 << K.k;
    u32* mr = (u32*)malloc(Trem * sizeof(u32));
    u32* mc = (u32*)malloc(65536 * sizeof(u32));
    u64* z = (u64*)malloc(sizeof(u64) * (v + 1));
    u64* rho = (u64*)malloc(sizeof(u64) * (v + 1));
    u64* col = NULL;

    rd_mult(t, rd, "logup_m_rem", mr, Trem);
    u64 gamma = orc_tx_squeeze(t, "logup_gamma");
    rd_mult(t, rd, "logup_m_clamp", mc, 65536);
    if (rd->bad) FAIL(REJ_FORMAT, 3, 0);
    u64 alpha[2];
    alpha[0] = orc_tx_squeeze(t, "logup_alpha");
    alpha[1] = orc_tx_squeeze(t, "logup_alpha");

    u64 l1[8];
    rd_fe(t, rd, "gkr_l1", l1, 8);
    if (rd->bad) FAIL(REJ_FORMAT, 4, 0);
    for (int tau = 0; tau < 2; tau++) {
        const u64* x = l1 + 4 * tau; /* p(0), p(1), q(0), q(1) */
        u64 P0 = orc_fadd(orc_fmul(x[0], x[3]), orc_fmul(x[1], x[2]));
        u64 Q0 = orc_fmul(x[2], x[3]);
        u64 PT, QT;
        table_fraction(tau == 0 ? mr : mc, tau == 0 ? Trem : 65536, tau, K.k, alpha[tau], gamma, &PT, &QT);
        if (Q0 == 0 || orc_fmul(P0, QT) != orc_fmul(Q0, PT)) FAIL(tau == 0 ? REJ_ROOT_REM : REJ_ROOT_CLAMP, 0, 0);
    }
    u64 mu = orc_tx_squeeze(t, "gkr_mu");
    u64 cP[2], cQ[2];
    for (int tau = 0; tau < 2; tau++) {
        const u64* x = l1 + 4 * tau;
        cP[tau] = orc_fadd(x[0], orc_fmul(mu, orc_fsub(x[1], x[0])));
        cQ[tau] = orc_fadd(x[2], orc_fmul(mu, orc_fsub(x[3], x[2])));
    }
    z[0] = mu;
    for (int d = 1; d < v; d++) {
        u64 lam = orc_tx_squeeze(t, "gkr_lambda");
        u64 lam2 = orc_fmul(lam, lam), lam3 = orc_fmul(lam2, lam);
        u64 claim = orc_fadd(orc_fadd(cP[0], orc_fmul(lam, cQ[0])),
                             orc_fadd(orc_fmul(lam2, cP[1]), orc_fmul(lam3, cQ[1])));
        for (int r = 0; r < d; r++) {
            u64 g[4];
            rd_fe(t, rd, "gkr_round", g, 4);
            if (rd->bad) FAIL(REJ_FORMAT, 5, d);
            if (orc_fadd(g[0], g[1]) != claim) FAIL(REJ_GKR_ROUND, d, r);
            rho[r] = orc_tx_squeeze(t, "gkr_chal");
            claim = orc_lagrange(g, 4, rho[r]);
        }
        u64 fin[8];
        rd_fe(t, rd, "gkr_final", fin, 8);
        if (rd->bad) FAIL(REJ_FORMAT, 6, d);
        /* eq(z, rho) in closed form */
        u64 e = 1;
        for (int r = 0; r < d; r++)
            e = orc_fmul(e, orc_fadd(orc_fmul(z[r], rho[r]),
                                     orc_fmul(orc_fsub(1, z[r]), orc_fsub(1, rho[r]))));
        if (orc_fmul(e, layer_F(fin, lam, lam2)) != claim) FAIL(REJ_GKR_FINAL, d, 0);
        mu = orc_tx_squeeze(t, "gkr_mu");
        for (int tau = 0; tau < 2; tau++) {
            const u64* x = fin + 4 * tau;
            cP[tau] = orc_fadd(x[0], orc_fmul(mu, orc_fsub(x[1], x[0])));
            cQ[tau] = orc_fadd(x[2], orc_fmul(mu, orc_fsub(x[3], x[2])));
        }
        for (int r = 0; r < d; r++) z[r] = rho[r];
        z[d] = mu;
    }
    u64 leaf[3];
    rd_fe(t, rd, "leaf", leaf, 3);
    if (rd->bad) FAIL(REJ_FORMAT, 7, 0);
    if (cP[0] != 1 || cP[1] != 1) FAIL(REJ_LEAF_P, 0, 0);
    if (cQ[0] != orc_fsub(alpha[0], leaf[0])) FAIL(REJ_LEAF_Q, 0, 0);
    if (cQ[1] != orc_fsub(alpha[1], orc_fadd(leaf[1], orc_fmul(gamma, leaf[2])))) FAIL(REJ_LEAF_Q, 1, 0);
    if (!(g_verify_flags & VERIFY_SKIP_LEAF_OPEN)) {
        u64 Lk = (u64)1 << v;
        col = (u64*)malloc(Lk * sizeof(u64));
        for (u64 i = 0; i < Lk; i++) col[i] = orc_fint(K.fr[i]);
        if (orc_mle_eval(col, Lk, z, v) != leaf[0]) FAIL(REJ_LEAF_OPEN, 0, 0);
        for (u64 i = 0; i < Lk; i++) col[i] = orc_fint(K.fq[i]);
        if (orc_mle_eval(col, Lk, z, v) != leaf[1]) FAIL(REJ_LEAF_OPEN, 1, 0);
        for (u64 i = 0; i < Lk; i++) col[i] = orc_fint(K.fy[i]);
        if (orc_mle_eval(col, Lk, z, v) != leaf[2]) FAIL(REJ_LEAF_OPEN, 2, 0);
    }
done:
    free(col); free(mr); free(mc); free(z); free(rho);
    keys_free(&K);
    return rc;
}

int orc_verify_opts(u64 seed, const orc_site* sites, int ns, const orc_wit* wit, const uint8_t* proof, u64 len,
                    int64_t detail[2], const uint8_t* site_mask, int flags);

int orc_verify(u64 seed, const orc_site* sites, int ns, const orc_wit* wit, const uint8_t* proof, u64 len,
               int64_t detail[2]) {
    return orc_verify_opts(seed, sites, ns, wit, proof, len, detail, NULL, 0);
}

int orc_verify_opts(u64 seed, const orc_site* sites, int ns, const orc_wit* wit, const uint8_t* proof, u64 len,
                    int64_t detail[2], const uint8_t* site_mask, int flags) {
    g_site_mask = site_mask;
    g_verify_flags = flags;
    detail[0] = detail[1] = 0;
    if (ns < 1) return REJ_ARGS;
    for (int s = 0; s < ns; s++)
        if (sites[s].M < 1 || sites[s].N < 1 || sites[s].K < 1 || sites[s].k_shift < 1 ||
            sites[s].k_shift > 30 || sites[s].k_shift != sites[0].k_shift)
            return REJ_ARGS;
    orc_tx t;
    prd rd = {proof, len, 0, 0};
    orc_tx_init(&t, seed);
    absorb_sites(&t, sites, ns, wit);
    int rc = mm_verify(&t, &rd, sites, ns, wit, detail);
    if (rc) return rc;
    rc = lu_verify(&t, &rd, sites, ns, wit, detail);
    if (rc) return rc;
    if (rd.pos != rd.len) return REJ_FORMAT;
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Gated product h = s (.) u. The pages ("How fast can FlashProve go", 3.1   */
/* Committing intermediate values, the note on the MLP's hidden values) say  */
/* the gated product is a plain product that the sum-check handles without   */
/* committing to it: a claim on h~(z) is reduced to claims on s~(rho) and    */
/* u~(rho), the two committed factors. The textbook product sum-check over   */
/* three multilinear vectors, eq(z, .), s and u, degree 3 per round:         */
/*   absorb "had_site" D(s) || D(u) (the tree digests of the two int8        */
/*     vectors); squeeze z_1..z_v ("had_z"), v = ceil(log2 n);               */
/*   send c = sum_x eq(z, x) s(x) u(x) ("had_claim");                         */
/*   round t = 1..v: send g_t(0), g_t(1), g_t(2), g_t(3) ("had_round"), with  */
/*     g_t(X) = sum_b E(X, b) S(X, b) U(X, b) over the vectors folded by the  */
/*     earlier challenges; squeeze rho_t ("had_chal"); fold E, S and U;       */
/*   send S(rho), U(rho) ("had_final").                                        */
/* The vectors are zero-padded to 2^v; n = 1 gives v = 0 and no rounds.      */
/* ------------------------------------------------------------------------ */

enum {
    REJ_HAD_CLAIM = 15,  /* c != h~(z) recomputed from s and u */
    REJ_HAD_ROUND = 16,  /* g_t(0) + g_t(1) != running claim */
    REJ_HAD_FINAL = 17,  /* eq(z, rho) S U != claim after the last round */
    REJ_HAD_OPEN = 18    /* S or U != the committed vector's MLE at rho */
};

/* The rounds of the textbook product sum-check of E S U over v variables (E,
 * S, U of length 2^v, folded in place): round r sends g(0..3) under lab_round,
 * with g(X) = sum_b E(X, b) S(X, b) U(X, b) on each vector's line through
 * (b, b + h); squeezes rho_r under lab_chal; folds all three. Then sends the
 * final S(rho), U(rho) under lab_final. */
static void prod3_rounds(orc_tx* t, pbuf* pb, u64* E, u64* S, u64* U, int v, const char* lab_round,
                         const char* lab_chal, const char* lab_final) {
    u64 L = (u64)1 << v;
    for (int r = 0; r < v; r++) {
        u64 h = L >> 1;
        u64 g[4] = {0, 0, 0, 0};
        for (u64 b = 0; b < h; b++)
            for (u64 X = 0; X < 4; X++) {
                /* each vector's line through (b, b + h) at X */
                u64 e = orc_fadd(E[b], orc_fmul(X, orc_fsub(E[h + b], E[b])));
                u64 sx = orc_fadd(S[b], orc_fmul(X, orc_fsub(S[h + b], S[b])));
                u64 ux = orc_fadd(U[b], orc_fmul(X, orc_fsub(U[h + b], U[b])));
                g[X] = orc_fadd(g[X], orc_fmul(e, orc_fmul(sx, ux)));
            }
        send_fe(t, pb, lab_round, g, 4);
        u64 rho = orc_tx_squeeze(t, lab_chal);
        for (u64 b = 0; b < h; b++) {
            E[b] = orc_fadd(E[b], orc_fmul(rho, orc_fsub(E[h + b], E[b])));
            S[b] = orc_fadd(S[b], orc_fmul(rho, orc_fsub(S[h + b], S[b])));
            U[b] = orc_fadd(U[b], orc_fmul(rho, orc_fsub(U[h + b], U[b])));
        }
        L = h;
    }
    u64 fin[2] = {S[0], U[0]};
    send_fe(t, pb, lab_final, fin, 2);
}

/* Verifier side of prod3_rounds: each round's g(0) + g(1) against the running
 * claim (starting at *claim), the next claim g(rho) by Lagrange; returns 0 or
 * REJ_FORMAT / bad_round with detail[0] = the round. rho (v entries) and fin
 * (S(rho), U(rho)) are filled in; *claim ends as the last round's g(rho). */
static int prod3_verify(orc_tx* t, prd* rd, int v, u64* claim, u64* rho, u64 fin[2], const char* lab_round,
                        const char* lab_chal, const char* lab_final, int bad_round, int64_t* detail) {
    for (int r = 0; r < v; r++) {
        u64 g[4];
        rd_fe(t, rd, lab_round, g, 4);
        detail[0] = r;
        if (rd->bad) return REJ_FORMAT;
        if (orc_fadd(g[0], g[1]) != *claim) return bad_round;
        rho[r] = orc_tx_squeeze(t, lab_chal);
        *claim = orc_lagrange(g, 4, rho[r]);
    }
    detail[0] = v;
    rd_fe(t, rd, lab_final, fin, 2);
    if (rd->bad) return REJ_FORMAT;
    detail[0] = 0;
    return 0;
}

/* eq(z, rho) in closed form */
static u64 eq_closed(const u64* z, const u64* rho, int v) {
    u64 e = 1;
    for (int i = 0; i < v; i++)
        e = orc_fmul(e, orc_fadd(orc_fmul(z[i], rho[i]), orc_fmul(orc_fsub(1, z[i]), orc_fsub(1, rho[i]))));
    return e;
}

static void had_absorb_site(orc_tx* t, const int8_t* s, const int8_t* u, u64 n) {
    uint8_t d[64];
    orc_tree_digest(s, n, d);
    orc_tree_digest(u, n, d + 32);
    orc_tx_absorb(t, "had_site", d, 64);
}

/* the int8 vector as field elements, zero-padded to 2^v */
static u64* had_lift(const int8_t* a, u64 n, int v) {
    u64 sz = (u64)1 << v;
    u64* out = (u64*)calloc(sz, sizeof(u64));
    for (u64 i = 0; i < n; i++) out[i] = orc_fint(a[i]);
    return out;
}

/* The point z and claim c of the last gated product verified; the FFN statement checks c
 * against the rescaled product it commits. (The oracle is single-threaded.) */
static struct {
    int v;
    u64 z[MM_PT_MAX];
    u64 c;
} g_had_pt;

/* Proof into proof[0..cap); *len = bytes needed. Returns 0, -1 on bad input,
 * -2 if cap is too small. tx is an orc_tx_new handle, advanced in place. */
int orc_had_prove(void* txh, const int8_t* s, const int8_t* u, u64 n, uint8_t* proof, u64 cap, u64* len) {
    if (n < 1) return -1;
    orc_tx* t = (orc_tx*)txh;
    int v = orc_log2_ceil(n);
    u64 sz = (u64)1 << v;
    pbuf pb = {proof, cap, 0, 0};
    had_absorb_site(t, s, u, n);
    u64* z = (u64*)malloc(sizeof(u64) * (v + 1));
    for (int i = 0; i < v; i++) z[i] = orc_tx_squeeze(t, "had_z");
    u64* E = (u64*)malloc(sz * sizeof(u64));
    orc_eq_table(z, v, E);
    u64* S = had_lift(s, n, v);
    u64* U = had_lift(u, n, v);
    u64 c = 0;
    for (u64 x = 0; x < sz; x++) c = orc_fadd(c, orc_fmul(E[x], orc_fmul(S[x], U[x])));
    send_fe(t, &pb, "had_claim", &c, 1);
    prod3_rounds(t, &pb, E, S, U, v, "had_round", "had_chal", "had_final");
    free(z);
    free(E);
    free(S);
    free(U);
    *len = pb.len;
    return pb.overflow ? -2 : 0;
}

/* Verifier: every round's consistency, the end against eq(z, rho) S U in
 * closed form, and (standing in for openings of the committed s and u) the
 * claim c and the final S, U recomputed from the vectors it holds. Returns 0
 * (accept) or a rejection code; detail[0] = the round of a failed round check. */
int orc_had_verify(void* txh, const int8_t* s, const int8_t* u, u64 n, const uint8_t* proof, u64 len,
                   int64_t detail[2]) {
    detail[0] = detail[1] = 0;
    if (n < 1) return REJ_ARGS;
    orc_tx* t = (orc_tx*)txh;
    int v = orc_log2_ceil(n), rc = 0;
    u64 sz = (u64)1 << v;
    prd rd = {proof, len, 0, 0};
    had_absorb_site(t, s, u, n);
    u64* z = (u64*)malloc(sizeof(u64) * (v + 1));
    u64* rho = (u64*)malloc(sizeof(u64) * (v + 1));
    u64* S = had_lift(s, n, v);
    u64* U = had_lift(u, n, v);
    for (int i = 0; i < v; i++) z[i] = orc_tx_squeeze(t, "had_z");
    u64 c, claim;
    rd_fe(t, &rd, "had_claim", &c, 1);
    if (rd.bad) FAIL(REJ_FORMAT, 0, 0);
    g_had_pt.v = v;
    for (int i = 0; i < v && i < MM_PT_MAX; i++) g_had_pt.z[i] = z[i];
    g_had_pt.c = c;
    {
        u64* P = (u64*)malloc(sz * sizeof(u64));
        for (u64 x = 0; x < sz; x++) P[x] = orc_fmul(S[x], U[x]);
        u64 want = orc_mle_eval(P, sz, z, v);
        free(P);
        if (want != c) FAIL(REJ_HAD_CLAIM, 0, 0);
    }
    claim = c;
    u64 fin[2];
    {
        int64_t d0 = 0;
        int r2 = prod3_verify(t, &rd, v, &claim, rho, fin, "had_round", "had_chal", "had_final", REJ_HAD_ROUND, &d0);
        if (r2) FAIL(r2, d0, 0);
    }
    if (orc_fmul(eq_closed(z, rho, v), orc_fmul(fin[0], fin[1])) != claim) FAIL(REJ_HAD_FINAL, 0, 0);
    if (orc_mle_eval(S, sz, rho, v) != fin[0]) FAIL(REJ_HAD_OPEN, 0, 0);
    if (orc_mle_eval(U, sz, rho, v) != fin[1]) FAIL(REJ_HAD_OPEN, 1, 0);
    if (rd.pos != rd.len) FAIL(REJ_FORMAT, -1, 0);
done:
    free(z);
    free(rho);
    free(S);
    free(U);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Per-group scale reduction. A site with per-64-column int8 scales uses     */
/* W_eff[i][k] = S[i][k / 64] w[i][k]; its matmul sum-check ends with a      */
/* claim on W_eff~(z), but only w and S are committed. As for the gated     */
/* product ("How fast can FlashProve go", 3.1: a product that is not        */
/* committed is reduced by sum-check to claims on its committed factors),   */
/* the same degree-3 product sum-check runs over x = (i, k) (row bits       */
/* first; M and K padded to 2^vM and 2^vK) with the factors                 */
/*   Se(i, k) = S[i][k >> 6] (0 past the M x G scales, G = ceil(K / 64)),    */
/*   w(i, k)  (0 past M x K),                                                */
/* at a point z = (z_row, z_col) the caller supplies:                        */
/*   absorb "scl_site" D(W bytes) || D(S bytes);                             */
/*   send a = sum_x eq(z, x) Se(x) w(x) ("scl_claim");                        */
/*   v = vM + vK rounds ("scl_round", "scl_chal"); send Se(rho), w(rho)        */
/*   ("scl_final").                                                           */
/* Se does not depend on the six low column bits, so Se~(rho) is            */
/* S~(rho_row, rho_col_hi), rho_col_hi the first vK - 6 column coordinates  */
/* (none when vK <= 6): a claim on the committed scales.                    */
/* ------------------------------------------------------------------------ */

enum {
    REJ_SCL_CLAIM = 19,  /* a != W_eff~(z) recomputed from w and S */
    REJ_SCL_ROUND = 20,  /* g_t(0) + g_t(1) != running claim */
    REJ_SCL_FINAL = 21,  /* eq(z, rho) Se w != claim after the last round */
    REJ_SCL_OPEN = 22    /* Se(rho) != S~(rho_row, rho_col_hi) or w(rho) != w~(rho) */
};

static int64_t w_raw(const void* w, int bits, int K, u64 i, u64 k) {
    if (bits == 8) return ((const int8_t*)w)[i * (u64)K + k];
    const uint8_t* row = (const uint8_t*)w + i * (u64)((K + 1) / 2);
    int nib = (k & 1) ? (row[k / 2] >> 4) : (row[k / 2] & 15);
    return nib >= 8 ? nib - 16 : nib;
}

/* the two factors over the padded 2^(vM + vK) grid */
static void scl_vectors(const void* w, int bits, const int8_t* sc, int M, int K, int vM, int vK, u64* Se, u64* W) {
    u64 G = (u64)(K + 63) / 64, cols = (u64)1 << vK;
    for (u64 i = 0; i < ((u64)1 << vM); i++)
        for (u64 k = 0; k < cols; k++) {
            u64 x = i * cols + k;
            Se[x] = (i < (u64)M && (k >> 6) < G) ? orc_fint(sc[i * G + (k >> 6)]) : 0;
            W[x] = (i < (u64)M && k < (u64)K) ? orc_fint(w_raw(w, bits, K, i, k)) : 0;
        }
}

static void scl_absorb_site(orc_tx* t, const void* w, int bits, const int8_t* sc, int M, int K) {
    uint8_t d[64];
    orc_tree_digest(w, (u64)M * (bits == 4 ? (u64)((K + 1) / 2) : (u64)K), d);
    orc_tree_digest(sc, (u64)M * (u64)((K + 63) / 64), d + 32);
    orc_tx_absorb(t, "scl_site", d, 64);
}

static int scl_args_ok(int bits, int M, int K) { return (bits == 4 || bits == 8) && M >= 1 && K >= 1; }

int orc_scl_prove(void* txh, const void* w, int bits, const int8_t* sc, int M, int K, const u64* z, uint8_t* proof,
                  u64 cap, u64* len) {
    if (!scl_args_ok(bits, M, K)) return -1;
    orc_tx* t = (orc_tx*)txh;
    int vM = orc_log2_ceil((u64)M), vK = orc_log2_ceil((u64)K), v = vM + vK;
    u64 sz = (u64)1 << v;
    pbuf pb = {proof, cap, 0, 0};
    scl_absorb_site(t, w, bits, sc, M, K);
    u64* E = (u64*)malloc(sz * sizeof(u64));
    u64* Se = (u64*)malloc(sz * sizeof(u64));
    u64* W = (u64*)malloc(sz * sizeof(u64));
    orc_eq_table(z, v, E);
    scl_vectors(w, bits, sc, M, K, vM, vK, Se, W);
    u64 a = 0;
    for (u64 x = 0; x < sz; x++) a = orc_fadd(a, orc_fmul(E[x], orc_fmul(Se[x], W[x])));
    send_fe(t, &pb, "scl_claim", &a, 1);
    prod3_rounds(t, &pb, E, Se, W, v, "scl_round", "scl_chal", "scl_final");
    free(E);
    free(Se);
    free(W);
    *len = pb.len;
    return pb.overflow ? -2 : 0;
}

int orc_scl_verify(void* txh, const void* w, int bits, const int8_t* sc, int M, int K, const u64* z,
                   const uint8_t* proof, u64 len, int64_t detail[2]) {
    detail[0] = detail[1] = 0;
    if (!scl_args_ok(bits, M, K)) return REJ_ARGS;
    orc_tx* t = (orc_tx*)txh;
    int vM = orc_log2_ceil((u64)M), vK = orc_log2_ceil((u64)K), v = vM + vK, rc = 0;
    int vKh = vK > 6 ? vK - 6 : 0;
    u64 sz = (u64)1 << v, G = (u64)(K + 63) / 64;
    prd rd = {proof, len, 0, 0};
    u64* Se = (u64*)malloc(sz * sizeof(u64));
    u64* W = (u64*)malloc(sz * sizeof(u64));
    u64* P = (u64*)malloc(sz * sizeof(u64));
    u64* rho = (u64*)malloc(sizeof(u64) * (v + 1));
    u64* Sp = (u64*)calloc((u64)1 << (vM + vKh), sizeof(u64));
    u64* pt = (u64*)malloc(sizeof(u64) * (vM + vKh + 1));
    scl_absorb_site(t, w, bits, sc, M, K);
    scl_vectors(w, bits, sc, M, K, vM, vK, Se, W);
    u64 a, claim, fin[2];
    rd_fe(t, &rd, "scl_claim", &a, 1);
    if (rd.bad) FAIL(REJ_FORMAT, 0, 0);
    for (u64 x = 0; x < sz; x++) P[x] = orc_fmul(Se[x], W[x]);
    if (orc_mle_eval(P, sz, z, v) != a) FAIL(REJ_SCL_CLAIM, 0, 0);
    claim = a;
    {
        int64_t d0 = 0;
        int r2 = prod3_verify(t, &rd, v, &claim, rho, fin, "scl_round", "scl_chal", "scl_final", REJ_SCL_ROUND, &d0);
        if (r2) FAIL(r2, d0, 0);
    }
    if (orc_fmul(eq_closed(z, rho, v), orc_fmul(fin[0], fin[1])) != claim) FAIL(REJ_SCL_FINAL, 0, 0);
    /* openings: the scales at (rho_row, rho_col_hi), the weights at rho */
    for (u64 i = 0; i < (u64)M; i++)
        for (u64 g = 0; g < G; g++) Sp[(i << vKh) + g] = orc_fint(sc[i * G + g]);
    for (int i = 0; i < vM; i++) pt[i] = rho[i];
    for (int i = 0; i < vKh; i++) pt[vM + i] = rho[vM + i];
    if (orc_mle_eval(Sp, (u64)1 << (vM + vKh), pt, vM + vKh) != fin[0]) FAIL(REJ_SCL_OPEN, 0, 0);
    if (orc_mle_eval(W, sz, rho, v) != fin[1]) FAIL(REJ_SCL_OPEN, 1, 0);
    if (rd.pos != rd.len) FAIL(REJ_FORMAT, -1, 0);
done:
    free(Se);
    free(W);
    free(P);
    free(rho);
    free(Sp);
    free(pt);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* SiLU by lookup. The pages prove non-polynomial steps such as the SiLU by  */
/* committing their outputs and looking them up ("How fast can FlashProve   */
/* go", 2 Background; 3.1: the gate's values are 16-bit and the SiLU's      */
/* output is committed). The table is read over the 16-bit domain           */
/* v in [-2^15, 2^15) as fixed point with 8 fractional bits:                */
/*   silu_q(v) = floor(v sigma(v / 256) + 1/2) = floor(v / (1 + e^(-v/256)) + 1/2), */
/* evaluated in double precision (the table is this formula). One LogUp    */
/* tree over the keys f_i = g_i + gamma s_i, with the steps of the          */
/* remainder / clamp lookup:                                                 */
/*   absorb "silu_site" D(g) || D(s) (int16 little-endian);                  */
/*   squeeze gamma ("silu_gamma"); keys padded to 2^v (v >= 1) with the      */
/*   table's own row (0, silu_q(0)) = (0, 0);                                 */
/*   m_j = #{keys with g = j - 2^15}; send m (2^16 u32, digest absorbed,     */
/*   "silu_m"); squeeze alpha ("silu_alpha");                                 */
/*   tree of leaves (1, alpha - f); send layer one p(0), p(1), q(0), q(1)      */
/*   ("silu_l1"); squeeze mu ("silu_mu");                                     */
/*   layers d = 1..v-1: squeeze lambda ("silu_lambda"); sum-check of          */
/*   eq(z, x)(pL qR + pR qL + lambda qL qR), rounds "silu_round" / "silu_chal";*/
/*   send pL, pR, qL, qR at rho ("silu_final"); squeeze mu; z = (rho, mu);     */
/*   send g~(z), s~(z) ("silu_leaf").                                          */
/* ------------------------------------------------------------------------ */

enum {
    REJ_SILU_ROOT = 23,   /* key fraction != table fraction */
    REJ_SILU_ROUND = 24,  /* layer sum-check round inconsistent */
    REJ_SILU_FINAL = 25,  /* layer end: eq * F != claim */
    REJ_SILU_LEAF = 26,   /* leaf numerator != 1 or denominator != alpha - key */
    REJ_SILU_OPEN = 27    /* g~(z) or s~(z) != the committed column's MLE */
};

int32_t orc_silu_q(int32_t v) { return (int32_t)floor((double)v / (1.0 + exp(-(double)v / 256.0)) + 0.5); }

/* The softmax numerator by lookup (the same pages: the exponential is a lookup table; the
 * integer softmax of "Towards Proving Frontier-Scale LLM Inference", The arithmetic, has a 9-bit
 * numerator). Input v = score - row maximum <= 0 with 8 fractional bits:
 *   exp_q(v) = floor(511 e^(v / 256) + 1/2), and 511 for v > 0 (never reached after the max). */
int32_t orc_exp_q(int32_t v) { return v >= 0 ? 511 : (int32_t)floor(511.0 * exp((double)v / 256.0) + 0.5); }

/* A lookup of a 16-bit function table: the same argument for every table, only the labels and
 * (at the verifier) the table differ. */
typedef struct {
    const char *site, *gamma, *m, *alpha, *l1, *mu, *lambda, *round, *chal, *fin, *leaf;
} lk_labels;
static const lk_labels LK_SILU = {"silu_site", "silu_gamma", "silu_m", "silu_alpha", "silu_l1", "silu_mu",
                                  "silu_lambda", "silu_round", "silu_chal", "silu_final", "silu_leaf"};
static const lk_labels LK_EXP = {"exp_site", "exp_gamma", "exp_m", "exp_alpha", "exp_l1", "exp_mu",
                                 "exp_lambda", "exp_round", "exp_chal", "exp_final", "exp_leaf"};

static void silu_absorb_site(orc_tx* t, const lk_labels* lab, const int16_t* g, const int16_t* s, u64 n) {
    uint8_t d[64];
    uint8_t* b = (uint8_t*)calloc(2 * n, 1);
    for (u64 i = 0; i < n; i++) put_le(b + 2 * i, (u64)(uint16_t)g[i], 2);
    orc_tree_digest(b, 2 * n, d);
    for (u64 i = 0; i < n; i++) put_le(b + 2 * i, (u64)(uint16_t)s[i], 2);
    orc_tree_digest(b, 2 * n, d + 32);
    free(b);
    orc_tx_absorb(t, lab->site, d, 64);
}

static void silu_mult(const int16_t* g, u64 n, u64 L, u32* m) {
    memset(m, 0, 65536 * sizeof(u32));
    for (u64 i = 0; i < L; i++) m[(i < n ? (int64_t)g[i] : 0) + 32768]++;
}

/* layers[d] has 2^d nodes */
/* padding keys are (0, tab(0)): the table's own row for input 0 */
static void silu_tree(const int16_t* g, const int16_t* s, u64 n, int v, u64 alpha, u64 gamma, int32_t pad_s, u64** Pd,
                      u64** Qd) {
    u64 L = (u64)1 << v;
    Pd[v] = (u64*)malloc(L * sizeof(u64));
    Qd[v] = (u64*)malloc(L * sizeof(u64));
    for (u64 i = 0; i < L; i++) {
        u64 f = i < n ? orc_fadd(orc_fint(g[i]), orc_fmul(gamma, orc_fint(s[i]))) : orc_fmul(gamma, orc_fint(pad_s));
        Pd[v][i] = 1;
        Qd[v][i] = orc_fsub(alpha, f);
    }
    for (int d = v - 1; d >= 0; d--) {
        u64 c = (u64)1 << d;
        Pd[d] = (u64*)malloc(c * sizeof(u64));
        Qd[d] = (u64*)malloc(c * sizeof(u64));
        for (u64 x = 0; x < c; x++) {
            Pd[d][x] = orc_fadd(orc_fmul(Pd[d + 1][2 * x], Qd[d + 1][2 * x + 1]),
                                orc_fmul(Pd[d + 1][2 * x + 1], Qd[d + 1][2 * x]));
            Qd[d][x] = orc_fmul(Qd[d + 1][2 * x], Qd[d + 1][2 * x + 1]);
        }
    }
}

static u64 silu_F(const u64 x[4], u64 lam) { /* pL qR + pR qL + lambda qL qR */
    return orc_fadd(orc_fadd(orc_fmul(x[0], x[3]), orc_fmul(x[1], x[2])), orc_fmul(lam, orc_fmul(x[2], x[3])));
}

/* the padded key columns as field elements, and their MLEs at z */
static void silu_leaf_values(const int16_t* g, const int16_t* s, u64 n, int v, const u64* z, int32_t pad_s, u64 out[2]) {
    u64 L = (u64)1 << v;
    u64* col = (u64*)malloc(L * sizeof(u64));
    for (u64 i = 0; i < L; i++) col[i] = i < n ? orc_fint(g[i]) : 0;
    out[0] = orc_mle_eval(col, L, z, v);
    for (u64 i = 0; i < L; i++) col[i] = i < n ? orc_fint(s[i]) : orc_fint(pad_s);
    out[1] = orc_mle_eval(col, L, z, v);
    free(col);
}

static int lookup16_prove(void* txh, const lk_labels* lab, int32_t pad_s, const int16_t* g, const int16_t* s, u64 n,
                          uint8_t* proof, u64 cap, u64* len) {
    if (n < 1) return -1;
    orc_tx* t = (orc_tx*)txh;
    int v = orc_log2_ceil(n);
    if (v < 1) v = 1;
    u64 L = (u64)1 << v;
    pbuf pb = {proof, cap, 0, 0};
    silu_absorb_site(t, lab, g, s, n);
    u64 gamma = orc_tx_squeeze(t, lab->gamma);
    u32* m = (u32*)malloc(65536 * sizeof(u32));
    silu_mult(g, n, L, m);
    send_mult(t, &pb, lab->m, m, 65536);
    u64 alpha = orc_tx_squeeze(t, lab->alpha);
    u64** Pd = (u64**)malloc(sizeof(u64*) * (v + 1));
    u64** Qd = (u64**)malloc(sizeof(u64*) * (v + 1));
    silu_tree(g, s, n, v, alpha, gamma, pad_s, Pd, Qd);
    u64 l1[4] = {Pd[1][0], Pd[1][1], Qd[1][0], Qd[1][1]};
    send_fe(t, &pb, lab->l1, l1, 4);
    u64* z = (u64*)malloc(sizeof(u64) * (v + 1));
    z[0] = orc_tx_squeeze(t, lab->mu);
    for (int d = 1; d < v; d++) {
        u64 lam = orc_tx_squeeze(t, lab->lambda);
        u64 c = (u64)1 << d;
        u64* V[5]; /* pL, pR, qL, qR (children of layer d), eq(z, .) */
        for (int i = 0; i < 5; i++) V[i] = (u64*)malloc(c * sizeof(u64));
        for (u64 x = 0; x < c; x++) {
            V[0][x] = Pd[d + 1][2 * x];
            V[1][x] = Pd[d + 1][2 * x + 1];
            V[2][x] = Qd[d + 1][2 * x];
            V[3][x] = Qd[d + 1][2 * x + 1];
        }
        orc_eq_table(z, d, V[4]);
        u64* rho = (u64*)malloc(sizeof(u64) * d);
        u64 Lr = c;
        for (int r = 0; r < d; r++) {
            u64 h = Lr >> 1;
            u64 gr[4] = {0, 0, 0, 0};
            for (u64 b = 0; b < h; b++)
                for (u64 X = 0; X < 4; X++) {
                    u64 ev[5];
                    for (int i = 0; i < 5; i++) ev[i] = orc_fadd(V[i][b], orc_fmul(X, orc_fsub(V[i][h + b], V[i][b])));
                    gr[X] = orc_fadd(gr[X], orc_fmul(ev[4], silu_F(ev, lam)));
                }
            send_fe(t, &pb, lab->round, gr, 4);
            rho[r] = orc_tx_squeeze(t, lab->chal);
            for (int i = 0; i < 5; i++)
                for (u64 b = 0; b < h; b++) V[i][b] = orc_fadd(V[i][b], orc_fmul(rho[r], orc_fsub(V[i][h + b], V[i][b])));
            Lr = h;
        }
        u64 fin[4] = {V[0][0], V[1][0], V[2][0], V[3][0]};
        send_fe(t, &pb, lab->fin, fin, 4);
        u64 mu = orc_tx_squeeze(t, lab->mu);
        for (int r = 0; r < d; r++) z[r] = rho[r];
        z[d] = mu;
        for (int i = 0; i < 5; i++) free(V[i]);
        free(rho);
    }
    u64 leaf[2];
    silu_leaf_values(g, s, n, v, z, pad_s, leaf);
    send_fe(t, &pb, lab->leaf, leaf, 2);
    for (int d = 0; d <= v; d++) {
        free(Pd[d]);
        free(Qd[d]);
    }
    free(Pd);
    free(Qd);
    free(z);
    free(m);
    *len = pb.len;
    return pb.overflow ? -2 : 0;
}

static int lookup16_verify(void* txh, const lk_labels* lab, int32_t (*tab)(int32_t), const int16_t* g,
                           const int16_t* s, u64 n, const uint8_t* proof, u64 len, int64_t detail[2]) {
    detail[0] = detail[1] = 0;
    if (n < 1) return REJ_ARGS;
    orc_tx* t = (orc_tx*)txh;
    int v = orc_log2_ceil(n), rc = 0;
    if (v < 1) v = 1;
    prd rd = {proof, len, 0, 0};
    u32* m = (u32*)malloc(65536 * sizeof(u32));
    u64* z = (u64*)malloc(sizeof(u64) * (v + 1));
    u64* rho = (u64*)malloc(sizeof(u64) * (v + 1));
    silu_absorb_site(t, lab, g, s, n);
    u64 gamma = orc_tx_squeeze(t, lab->gamma);
    rd_mult(t, &rd, lab->m, m, 65536);
    if (rd.bad) FAIL(REJ_FORMAT, 0, 0);
    u64 alpha = orc_tx_squeeze(t, lab->alpha);
    u64 l1[4];
    rd_fe(t, &rd, lab->l1, l1, 4);
    if (rd.bad) FAIL(REJ_FORMAT, 1, 0);
    {
        /* the table side, sum_j m_j / (alpha - t_j) with t_j = v_j + gamma silu_q(v_j) */
        u64 PT = 0, QT = 1;
        for (u64 j = 0; j < 65536; j++) {
            int32_t vj = (int32_t)j - 32768;
            u64 dj = orc_fsub(alpha, orc_fadd(orc_fint(vj), orc_fmul(gamma, orc_fint(tab(vj)))));
            PT = orc_fadd(orc_fmul(PT, dj), orc_fmul((u64)m[j], QT));
            QT = orc_fmul(QT, dj);
        }
        u64 P0 = orc_fadd(orc_fmul(l1[0], l1[3]), orc_fmul(l1[1], l1[2]));
        u64 Q0 = orc_fmul(l1[2], l1[3]);
        if (Q0 == 0 || orc_fmul(P0, QT) != orc_fmul(Q0, PT)) FAIL(REJ_SILU_ROOT, 0, 0);
    }
    u64 mu = orc_tx_squeeze(t, lab->mu);
    u64 cP = orc_fadd(l1[0], orc_fmul(mu, orc_fsub(l1[1], l1[0])));
    u64 cQ = orc_fadd(l1[2], orc_fmul(mu, orc_fsub(l1[3], l1[2])));
    z[0] = mu;
    for (int d = 1; d < v; d++) {
        u64 lam = orc_tx_squeeze(t, lab->lambda);
        u64 claim = orc_fadd(cP, orc_fmul(lam, cQ));
        for (int r = 0; r < d; r++) {
            u64 gr[4];
            rd_fe(t, &rd, lab->round, gr, 4);
            if (rd.bad) FAIL(REJ_FORMAT, 2, d);
            if (orc_fadd(gr[0], gr[1]) != claim) FAIL(REJ_SILU_ROUND, d, r);
            rho[r] = orc_tx_squeeze(t, lab->chal);
            claim = orc_lagrange(gr, 4, rho[r]);
        }
        u64 fin[4];
        rd_fe(t, &rd, lab->fin, fin, 4);
        if (rd.bad) FAIL(REJ_FORMAT, 3, d);
        if (orc_fmul(eq_closed(z, rho, d), silu_F(fin, lam)) != claim) FAIL(REJ_SILU_FINAL, d, 0);
        mu = orc_tx_squeeze(t, lab->mu);
        cP = orc_fadd(fin[0], orc_fmul(mu, orc_fsub(fin[1], fin[0])));
        cQ = orc_fadd(fin[2], orc_fmul(mu, orc_fsub(fin[3], fin[2])));
        for (int r = 0; r < d; r++) z[r] = rho[r];
        z[d] = mu;
    }
    u64 leaf[2];
    rd_fe(t, &rd, lab->leaf, leaf, 2);
    if (rd.bad) FAIL(REJ_FORMAT, 4, 0);
    if (cP != 1) FAIL(REJ_SILU_LEAF, 0, 0);
    if (cQ != orc_fsub(alpha, orc_fadd(leaf[0], orc_fmul(gamma, leaf[1])))) FAIL(REJ_SILU_LEAF, 1, 0);
    {
        u64 want[2];
        silu_leaf_values(g, s, n, v, z, tab(0), want);
        if (want[0] != leaf[0]) FAIL(REJ_SILU_OPEN, 0, 0);
        if (want[1] != leaf[1]) FAIL(REJ_SILU_OPEN, 1, 0);
    }
    if (rd.pos != rd.len) FAIL(REJ_FORMAT, -1, 0);
done:
    free(m);
    free(z);
    free(rho);
    return rc;
}

int orc_silu_prove(void* txh, const int16_t* g, const int16_t* s, u64 n, uint8_t* proof, u64 cap, u64* len) {
    return lookup16_prove(txh, &LK_SILU, orc_silu_q(0), g, s, n, proof, cap, len);
}
int orc_silu_verify(void* txh, const int16_t* g, const int16_t* s, u64 n, const uint8_t* proof, u64 len,
                    int64_t detail[2]) {
    return lookup16_verify(txh, &LK_SILU, orc_silu_q, g, s, n, proof, len, detail);
}
int orc_exp_prove(void* txh, const int16_t* g, const int16_t* s, u64 n, uint8_t* proof, u64 cap, u64* len) {
    return lookup16_prove(txh, &LK_EXP, orc_exp_q(0), g, s, n, proof, cap, len);
}
int orc_exp_verify(void* txh, const int16_t* g, const int16_t* s, u64 n, const uint8_t* proof, u64 len,
                   int64_t detail[2]) {
    return lookup16_verify(txh, &LK_EXP, orc_exp_q, g, s, n, proof, len, detail);
}

/* ------------------------------------------------------------------------ */
/* The helper-inverse LogUp (the lookup argument of "Towards Proving         */
/* Frontier-Scale LLM Inference", The proof system: LogUp after Haboeck      */
/* 2022), the variant to set against the GKR fraction tree. For the         */
/* remainder table R_k = {j - 2^(k-1)} and a key column r (int32, n keys,   */
/* padded to 2^v, v >= 1, with the key 0):                                  */
/*   absorb "lhi_site" D(r) (int32 little-endian);                          */
/*   m_j = #{keys = j - 2^(k-1)}; send m (2^k u32, digest absorbed, "lhi_m"); */
/*   squeeze alpha ("lhi_alpha"); the helper column h_i = 1 / (alpha - r_i) */
/*   is committed: absorb "lhi_h" D(h as u64 little-endian);                 */
/*   squeeze z_1..z_v ("lhi_z") and beta ("lhi_beta");                       */
/*   send S = sum_i h_i ("lhi_sum");                                         */
/*   sum-check of F(x) = h(x) + beta eq(z, x) (h(x) (alpha - f(x)) - 1) over  */
/*   v variables, claim S: rounds g(0..3) ("lhi_round"), "lhi_chal";         */
/*   send h(rho), f(rho) ("lhi_final").                                       */
/* The verifier checks S against sum_j m_j / (alpha - t_j), every round, the */
/* end against h + beta eq(z, rho) (h (alpha - f) - 1), and h(rho), f(rho)   */
/* against the columns it recomputes (standing in for openings). The        */
/* zero-check part forces h_i (alpha - f_i) = 1 everywhere (with high        */
/* probability over z), so S is the key side of the LogUp identity.         */
/* ------------------------------------------------------------------------ */

enum {
    REJ_LHI_SUM = 28,    /* S != the table side */
    REJ_LHI_ROUND = 29,  /* g(0) + g(1) != running claim */
    REJ_LHI_FINAL = 30,  /* the end does not match F at rho */
    REJ_LHI_OPEN = 31    /* h(rho) or f(rho) != the columns' MLEs */
};

static void lhi_columns(const int32_t* r, u64 n, int v, u64 alpha, u64* f, u64* h) {
    u64 L = (u64)1 << v;
    for (u64 i = 0; i < L; i++) {
        f[i] = i < n ? orc_fint(r[i]) : 0;
        h[i] = orc_finv(orc_fsub(alpha, f[i]));
    }
}

static void lhi_absorb_h(orc_tx* t, const u64* h, u64 L) {
    uint8_t* b = (uint8_t*)malloc(8 * L);
    uint8_t d[32];
    for (u64 i = 0; i < L; i++) put_le(b + 8 * i, h[i], 8);
    orc_tree_digest(b, 8 * L, d);
    free(b);
    orc_tx_absorb(t, "lhi_h", d, 32);
}

static void lhi_absorb_site(orc_tx* t, const int32_t* r, u64 n) {
    uint8_t* b = (uint8_t*)calloc(4 * n, 1);
    uint8_t d[32];
    for (u64 i = 0; i < n; i++) put_le(b + 4 * i, (u64)(u32)r[i], 4);
    orc_tree_digest(b, 4 * n, d);
    free(b);
    orc_tx_absorb(t, "lhi_site", d, 32);
}

static void lhi_mult(const int32_t* r, u64 n, u64 L, int k, u32* m) {
    u64 T = (u64)1 << k;
    int64_t half = (int64_t)1 << (k - 1);
    memset(m, 0, T * sizeof(u32));
    for (u64 i = 0; i < L; i++) {
        int64_t j = (i < n ? (int64_t)r[i] : 0) + half;
        if (j >= 0 && (u64)j < T) m[j]++;
    }
}

/* F at one point of the three lines: h + beta e (h (alpha - f) - 1) */
static u64 lhi_F(u64 h, u64 f, u64 e, u64 alpha, u64 beta) {
    return orc_fadd(h, orc_fmul(beta, orc_fmul(e, orc_fsub(orc_fmul(h, orc_fsub(alpha, f)), 1))));
}

int orc_lhi_prove(void* txh, const int32_t* r, u64 n, int k, uint8_t* proof, u64 cap, u64* len) {
    if (n < 1 || k < 1 || k > 24) return -1;
    orc_tx* t = (orc_tx*)txh;
    int v = orc_log2_ceil(n);
    if (v < 1) v = 1;
    u64 L = (u64)1 << v, T = (u64)1 << k;
    pbuf pb = {proof, cap, 0, 0};
    lhi_absorb_site(t, r, n);
    u32* m = (u32*)malloc(T * sizeof(u32));
    lhi_mult(r, n, L, k, m);
    send_mult(t, &pb, "lhi_m", m, T);
    u64 alpha = orc_tx_squeeze(t, "lhi_alpha");
    u64* f = (u64*)malloc(L * sizeof(u64));
    u64* h = (u64*)malloc(L * sizeof(u64));
    u64* E = (u64*)malloc(L * sizeof(u64));
    u64* z = (u64*)malloc(sizeof(u64) * v);
    lhi_columns(r, n, v, alpha, f, h);
    lhi_absorb_h(t, h, L);
    for (int i = 0; i < v; i++) z[i] = orc_tx_squeeze(t, "lhi_z");
    u64 beta = orc_tx_squeeze(t, "lhi_beta");
    u64 S = 0;
    for (u64 i = 0; i < L; i++) S = orc_fadd(S, h[i]);
    send_fe(t, &pb, "lhi_sum", &S, 1);
    orc_eq_table(z, v, E);
    u64 Lr = L;
    for (int rd = 0; rd < v; rd++) {
        u64 hh = Lr >> 1;
        u64 g[4] = {0, 0, 0, 0};
        for (u64 b = 0; b < hh; b++)
            for (u64 X = 0; X < 4; X++) {
                u64 hx = orc_fadd(h[b], orc_fmul(X, orc_fsub(h[hh + b], h[b])));
                u64 fx = orc_fadd(f[b], orc_fmul(X, orc_fsub(f[hh + b], f[b])));
                u64 ex = orc_fadd(E[b], orc_fmul(X, orc_fsub(E[hh + b], E[b])));
                g[X] = orc_fadd(g[X], lhi_F(hx, fx, ex, alpha, beta));
            }
        send_fe(t, &pb, "lhi_round", g, 4);
        u64 rho = orc_tx_squeeze(t, "lhi_chal");
        for (u64 b = 0; b < hh; b++) {
            h[b] = orc_fadd(h[b], orc_fmul(rho, orc_fsub(h[hh + b], h[b])));
            f[b] = orc_fadd(f[b], orc_fmul(rho, orc_fsub(f[hh + b], f[b])));
            E[b] = orc_fadd(E[b], orc_fmul(rho, orc_fsub(E[hh + b], E[b])));
        }
        Lr = hh;
    }
    u64 fin[2] = {h[0], f[0]};
    send_fe(t, &pb, "lhi_final", fin, 2);
    free(m);
    free(f);
    free(h);
    free(E);
    free(z);
    *len = pb.len;
    return pb.overflow ? -2 : 0;
}

int orc_lhi_verify(void* txh, const int32_t* r, u64 n, int k, const uint8_t* proof, u64 len, int64_t detail[2]) {
    detail[0] = detail[1] = 0;
    if (n < 1 || k < 1 || k > 24) return REJ_ARGS;
    orc_tx* t = (orc_tx*)txh;
    int v = orc_log2_ceil(n), rc = 0;
    if (v < 1) v = 1;
    u64 L = (u64)1 << v, T = (u64)1 << k;
    prd rd = {proof, len, 0, 0};
    u32* m = (u32*)malloc(T * sizeof(u32));
    u64* f = (u64*)malloc(L * sizeof(u64));
    u64* h = (u64*)malloc(L * sizeof(u64));
    u64* z = (u64*)malloc(sizeof(u64) * v);
    u64* rho = (u64*)malloc(sizeof(u64) * v);
    lhi_absorb_site(t, r, n);
    rd_mult(t, &rd, "lhi_m", m, T);
    if (rd.bad) FAIL(REJ_FORMAT, 0, 0);
    u64 alpha = orc_tx_squeeze(t, "lhi_alpha");
    lhi_columns(r, n, v, alpha, f, h); /* the verifier holds the key column, so h too */
    lhi_absorb_h(t, h, L);
    for (int i = 0; i < v; i++) z[i] = orc_tx_squeeze(t, "lhi_z");
    u64 beta = orc_tx_squeeze(t, "lhi_beta");
    u64 S;
    rd_fe(t, &rd, "lhi_sum", &S, 1);
    if (rd.bad) FAIL(REJ_FORMAT, 1, 0);
    {
        /* the table side: sum_j m_j / (alpha - t_j), t_j = j - 2^(k-1) */
        u64 P = 0, Q = 1;
        for (u64 j = 0; j < T; j++) {
            u64 dj = orc_fsub(alpha, orc_fint((int64_t)j - ((int64_t)1 << (k - 1))));
            P = orc_fadd(orc_fmul(P, dj), orc_fmul((u64)m[j], Q));
            Q = orc_fmul(Q, dj);
        }
        if (orc_fmul(S, Q) != P) FAIL(REJ_LHI_SUM, 0, 0);
    }
    u64 claim = S;
    for (int i = 0; i < v; i++) {
        u64 g[4];
        rd_fe(t, &rd, "lhi_round", g, 4);
        if (rd.bad) FAIL(REJ_FORMAT, 2, i);
        if (orc_fadd(g[0], g[1]) != claim) FAIL(REJ_LHI_ROUND, i, 0);
        rho[i] = orc_tx_squeeze(t, "lhi_chal");
        claim = orc_lagrange(g, 4, rho[i]);
    }
    u64 fin[2];
    rd_fe(t, &rd, "lhi_final", fin, 2);
    if (rd.bad) FAIL(REJ_FORMAT, 3, 0);
    if (lhi_F(fin[0], fin[1], eq_closed(z, rho, v), alpha, beta) != claim) FAIL(REJ_LHI_FINAL, 0, 0);
    if (orc_mle_eval(h, L, rho, v) != fin[0]) FAIL(REJ_LHI_OPEN, 0, 0);
    if (orc_mle_eval(f, L, rho, v) != fin[1]) FAIL(REJ_LHI_OPEN, 1, 0);
    if (rd.pos != rd.len) FAIL(REJ_FORMAT, -1, 0);
done:
    free(m);
    free(f);
    free(h);
    free(z);
    free(rho);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* Extension-field challenges (next row f4): "How fast can FlashProve go",   */
/* 4 Tighter Rooflines (a note there): for soundness the challenges live in  */
/* an extension of the Goldilocks field. Here the quadratic extension        */
/* F_p[phi] / (phi^2 - 7) (7 is not a square mod p), an element a + b phi    */
/* stored as (a, b) and sent as 16 bytes (a, then b, u64 little-endian); a   */
/* challenge is two squeezes (a, then b) under its label. First statement:  */
/* the gated-product sum-check of section "Gated product" with every         */
/* challenge, claim, round value and final value in the extension:           */
/*   absorb "had2_site" D(s) || D(u); squeeze z_1..z_v ("had2_z");            */
/*   send c ("had2_claim"); rounds g(0..3) ("had2_round"), "had2_chal";       */
/*   send S(rho), U(rho) ("had2_final").                                      */
/* ------------------------------------------------------------------------ */

typedef struct {
    u64 a, b;
} ext2;

static ext2 e2(u64 a, u64 b) { ext2 r = {a, b}; return r; }
static ext2 e2_add(ext2 x, ext2 y) { return e2(orc_fadd(x.a, y.a), orc_fadd(x.b, y.b)); }
static ext2 e2_sub(ext2 x, ext2 y) { return e2(orc_fsub(x.a, y.a), orc_fsub(x.b, y.b)); }
static ext2 e2_mul(ext2 x, ext2 y) { /* (a + b phi)(c + d phi) = ac + 7 bd + (ad + bc) phi */
    return e2(orc_fadd(orc_fmul(x.a, y.a), orc_fmul(7, orc_fmul(x.b, y.b))),
              orc_fadd(orc_fmul(x.a, y.b), orc_fmul(x.b, y.a)));
}
static ext2 e2_scal(ext2 x, u64 k) { return e2(orc_fmul(x.a, k), orc_fmul(x.b, k)); }

/* ctypes-facing multiplication and inverse (for the pins) */
void orc_e2_mul(const u64 x[2], const u64 y[2], u64 out[2]) {
    ext2 r = e2_mul(e2(x[0], x[1]), e2(y[0], y[1]));
    out[0] = r.a;
    out[1] = r.b;
}
void orc_e2_inv(const u64 x[2], u64 out[2]) { /* 1 / (a + b phi) = (a - b phi) / (a^2 - 7 b^2) */
    u64 n = orc_fsub(orc_fmul(x[0], x[0]), orc_fmul(7, orc_fmul(x[1], x[1])));
    u64 ni = orc_finv(n);
    out[0] = orc_fmul(x[0], ni);
    out[1] = orc_fsub(0, orc_fmul(x[1], ni));
}

static ext2 e2_squeeze(orc_tx* t, const char* label) {
    u64 a = orc_tx_squeeze(t, label);
    u64 b = orc_tx_squeeze(t, label);
    return e2(a, b);
}

static void e2_send(orc_tx* t, pbuf* pb, const char* label, const ext2* v, u64 n) {
    u64* w = (u64*)malloc(sizeof(u64) * 2 * (n ? n : 1));
    for (u64 i = 0; i < n; i++) {
        w[2 * i] = v[i].a;
        w[2 * i + 1] = v[i].b;
    }
    send_fe(t, pb, label, w, 2 * n);
    free(w);
}

static void e2_read(orc_tx* t, prd* rd, const char* label, ext2* v, u64 n) {
    u64* w = (u64*)malloc(sizeof(u64) * 2 * (n ? n : 1));
    rd_fe(t, rd, label, w, 2 * n);
    for (u64 i = 0; i < n; i++) v[i] = e2(w[2 * i], w[2 * i + 1]);
    free(w);
}

/* eq table of an extension point by doubling (z_1 on the most significant bit) */
static void e2_eq_table(const ext2* z, int v, ext2* out) {
    out[0] = e2(1, 0);
    for (int b = 0; b < v; b++) {
        u64 len = (u64)1 << b;
        for (u64 j = len; j-- > 0;) {
            ext2 o = out[j];
            out[2 * j] = e2_mul(o, e2_sub(e2(1, 0), z[b]));
            out[2 * j + 1] = e2_mul(o, z[b]);
        }
    }
}

/* the degree-3 polynomial through (i, g[i]), i = 0..3, at r */
static ext2 e2_lagrange4(const ext2 g[4], ext2 r) {
    ext2 acc = e2(0, 0);
    for (int i = 0; i < 4; i++) {
        ext2 num = e2(1, 0);
        int64_t den = 1;
        for (int j = 0; j < 4; j++) {
            if (j == i) continue;
            num = e2_mul(num, e2_sub(r, e2((u64)j, 0)));
            den *= (int64_t)(i - j);
        }
        acc = e2_add(acc, e2_mul(g[i], e2_scal(num, orc_finv(orc_fint(den)))));
    }
    return acc;
}

int orc_had2_prove(void* txh, const int8_t* s, const int8_t* u, u64 n, uint8_t* proof, u64 cap, u64* len) {
    if (n < 1) return -1;
    orc_tx* t = (orc_tx*)txh;
    int v = orc_log2_ceil(n);
    u64 sz = (u64)1 << v;
    pbuf pb = {proof, cap, 0, 0};
    uint8_t d[64];
    orc_tree_digest(s, n, d);
    orc_tree_digest(u, n, d + 32);
    orc_tx_absorb(t, "had2_site", d, 64);
    ext2* z = (ext2*)malloc(sizeof(ext2) * (v + 1));
    for (int i = 0; i < v; i++) z[i] = e2_squeeze(t, "had2_z");
    ext2* E = (ext2*)malloc(sizeof(ext2) * sz);
    ext2* S = (ext2*)malloc(sizeof(ext2) * sz);
    ext2* U = (ext2*)malloc(sizeof(ext2) * sz);
    e2_eq_table(z, v, E);
    for (u64 x = 0; x < sz; x++) {
        S[x] = e2(x < n ? orc_fint(s[x]) : 0, 0);
        U[x] = e2(x < n ? orc_fint(u[x]) : 0, 0);
    }
    ext2 c = e2(0, 0);
    for (u64 x = 0; x < sz; x++) c = e2_add(c, e2_mul(E[x], e2_mul(S[x], U[x])));
    e2_send(t, &pb, "had2_claim", &c, 1);
    u64 L = sz;
    for (int r = 0; r < v; r++) {
        u64 h = L >> 1;
        ext2 g[4] = {e2(0, 0), e2(0, 0), e2(0, 0), e2(0, 0)};
        for (u64 b = 0; b < h; b++)
            for (u64 X = 0; X < 4; X++) {
                ext2 ex = e2_add(E[b], e2_scal(e2_sub(E[h + b], E[b]), X));
                ext2 sx = e2_add(S[b], e2_scal(e2_sub(S[h + b], S[b]), X));
                ext2 ux = e2_add(U[b], e2_scal(e2_sub(U[h + b], U[b]), X));
                g[X] = e2_add(g[X], e2_mul(ex, e2_mul(sx, ux)));
            }
        e2_send(t, &pb, "had2_round", g, 4);
        ext2 rho = e2_squeeze(t, "had2_chal");
        for (u64 b = 0; b < h; b++) {
            E[b] = e2_add(E[b], e2_mul(rho, e2_sub(E[h + b], E[b])));
            S[b] = e2_add(S[b], e2_mul(rho, e2_sub(S[h + b], S[b])));
            U[b] = e2_add(U[b], e2_mul(rho, e2_sub(U[h + b], U[b])));
        }
        L = h;
    }
    ext2 fin[2] = {S[0], U[0]};
    e2_send(t, &pb, "had2_final", fin, 2);
    free(z);
    free(E);
    free(S);
    free(U);
    *len = pb.len;
    return pb.overflow ? -2 : 0;
}

/* MLE at an extension point of a base-field vector (zero-padded to 2^v) */
static ext2 e2_mle(const int8_t* a, u64 n, const ext2* z, int v) {
    u64 sz = (u64)1 << v;
    ext2* E = (ext2*)malloc(sizeof(ext2) * sz);
    e2_eq_table(z, v, E);
    ext2 acc = e2(0, 0);
    for (u64 x = 0; x < n && x < sz; x++) acc = e2_add(acc, e2_scal(E[x], orc_fint(a[x])));
    free(E);
    return acc;
}

int orc_had2_verify(void* txh, const int8_t* s, const int8_t* u, u64 n, const uint8_t* proof, u64 len,
                    int64_t detail[2]) {
    detail[0] = detail[1] = 0;
    if (n < 1) return REJ_ARGS;
    orc_tx* t = (orc_tx*)txh;
    int v = orc_log2_ceil(n), rc = 0;
    u64 sz = (u64)1 << v;
    prd rd = {proof, len, 0, 0};
    uint8_t d[64];
    orc_tree_digest(s, n, d);
    orc_tree_digest(u, n, d + 32);
    orc_tx_absorb(t, "had2_site", d, 64);
    ext2* z = (ext2*)malloc(sizeof(ext2) * (v + 1));
    ext2* rho = (ext2*)malloc(sizeof(ext2) * (v + 1));
    ext2* E = (ext2*)malloc(sizeof(ext2) * sz);
    for (int i = 0; i < v; i++) z[i] = e2_squeeze(t, "had2_z");
    ext2 c, claim;
    e2_read(t, &rd, "had2_claim", &c, 1);
    if (rd.bad) FAIL(REJ_FORMAT, 0, 0);
    {
        e2_eq_table(z, v, E);
        ext2 want = e2(0, 0);
        for (u64 x = 0; x < n; x++) want = e2_add(want, e2_scal(E[x], orc_fmul(orc_fint(s[x]), orc_fint(u[x]))));
        if (want.a != c.a || want.b != c.b) FAIL(REJ_HAD_CLAIM, 0, 0);
    }
    claim = c;
    for (int r = 0; r < v; r++) {
        ext2 g[4];
        e2_read(t, &rd, "had2_round", g, 4);
        if (rd.bad) FAIL(REJ_FORMAT, r, 0);
        ext2 s01 = e2_add(g[0], g[1]);
        if (s01.a != claim.a || s01.b != claim.b) FAIL(REJ_HAD_ROUND, r, 0);
        rho[r] = e2_squeeze(t, "had2_chal");
        claim = e2_lagrange4(g, rho[r]);
    }
    ext2 fin[2];
    e2_read(t, &rd, "had2_final", fin, 2);
    if (rd.bad) FAIL(REJ_FORMAT, v, 0);
    {
        ext2 e = e2(1, 0);
        for (int i = 0; i < v; i++)
            e = e2_mul(e, e2_add(e2_mul(z[i], rho[i]), e2_mul(e2_sub(e2(1, 0), z[i]), e2_sub(e2(1, 0), rho[i]))));
        ext2 end = e2_mul(e, e2_mul(fin[0], fin[1]));
        if (end.a != claim.a || end.b != claim.b) FAIL(REJ_HAD_FINAL, 0, 0);
    }
    {
        ext2 ws = e2_mle(s, n, rho, v), wu = e2_mle(u, n, rho, v);
        if (ws.a != fin[0].a || ws.b != fin[0].b) FAIL(REJ_HAD_OPEN, 0, 0);
        if (wu.a != fin[1].a || wu.b != fin[1].b) FAIL(REJ_HAD_OPEN, 1, 0);
    }
    if (rd.pos != rd.len) FAIL(REJ_FORMAT, -1, 0);
done:
    free(z);
    free(rho);
    free(E);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* The Freivalds check of a weight matmul (next row f4, the comparison      */
/* statement): "Towards Proving Frontier-Scale LLM Inference", The proof     */
/* system -- instead of recomputing C = A B, check A (B r) = C r for a random */
/* vector r. Here, for one site Y = W_eff X with Y = 2^k q + r standing in    */
/* for the unrounded product (the committed witness):                        */
/*   absorb "frv_site" D(W) || D(S) || D(Xt) || D(q) || D(r);                 */
/*   squeeze rho ("frv_rho"); the vector over tokens is rho^j, j < N;         */
/*   send u = X rho^(.) (K values, "frv_u"): u_k = sum_j X[k][j] rho^j.        */
/* The verifier checks u against X and W_eff u = Y rho^(.) row by row: a     */
/* wrong witness row makes a nonzero polynomial of degree < N in rho vanish, */
/* probability below N / p.                                                   */
/* ------------------------------------------------------------------------ */

enum {
    REJ_FRV_U = 32,   /* u != X rho^(.) */
    REJ_FRV_ROW = 33  /* (W_eff u)_i != (Y rho^(.))_i; detail[0] = i */
};

/* D(W) || D(S) || D(Xt) || D(q) || D(r) of one site */
static void site_digest160(const orc_site* s, const orc_wit* w, uint8_t d[160]) {
    u64 mn = (u64)s->M * s->N;
    uint8_t* qb = (uint8_t*)calloc(4 * mn + 1, 1);
    uint8_t* rb = (uint8_t*)calloc(4 * mn + 1, 1);
    for (u64 i = 0; i < mn; i++) {
        put_le(qb + 4 * i, (u64)(u32)w->q[i], 4);
        put_le(rb + 4 * i, (u64)(u32)w->r[i], 4);
    }
    orc_tree_digest(s->w, site_w_bytes(s), d);
    orc_tree_digest(s->scales, s->scales ? (u64)s->M * ((s->K + 63) / 64) : 0, d + 32);
    orc_tree_digest(s->xt, (u64)s->N * s->K, d + 64);
    orc_tree_digest(qb, 4 * mn, d + 96);
    orc_tree_digest(rb, 4 * mn, d + 128);
    free(qb);
    free(rb);
}

static void frv_absorb(orc_tx* t, const orc_site* s, const orc_wit* w) {
    uint8_t d[160];
    site_digest160(s, w, d);
    orc_tx_absorb(t, "frv_site", d, 160);
}

/* u_k = sum_j X[k][j] rho^j, X[k][j] = xt[j][k] */
static void frv_u(const orc_site* s, u64 rho, u64* u) {
    for (int k = 0; k < s->K; k++) u[k] = 0;
    u64 pw = 1;
    for (int j = 0; j < s->N; j++) {
        for (int k = 0; k < s->K; k++) u[k] = orc_fadd(u[k], orc_fmul(orc_fint(s->xt[(u64)j * s->K + k]), pw));
        pw = orc_fmul(pw, rho);
    }
}

int orc_frv_prove(void* txh, const orc_site* s, const orc_wit* w, uint8_t* proof, u64 cap, u64* len) {
    if (s->M < 1 || s->N < 1 || s->K < 1) return -1;
    orc_tx* t = (orc_tx*)txh;
    pbuf pb = {proof, cap, 0, 0};
    frv_absorb(t, s, w);
    u64 rho = orc_tx_squeeze(t, "frv_rho");
    u64* u = (u64*)malloc(sizeof(u64) * s->K);
    frv_u(s, rho, u);
    send_fe(t, &pb, "frv_u", u, (u64)s->K);
    free(u);
    *len = pb.len;
    return pb.overflow ? -2 : 0;
}

int orc_frv_verify(void* txh, const orc_site* s, const orc_wit* w, const uint8_t* proof, u64 len, int64_t detail[2]) {
    detail[0] = detail[1] = 0;
    if (s->M < 1 || s->N < 1 || s->K < 1) return REJ_ARGS;
    orc_tx* t = (orc_tx*)txh;
    int rc = 0;
    prd rd = {proof, len, 0, 0};
    u64* u = (u64*)malloc(sizeof(u64) * s->K);
    u64* want = (u64*)malloc(sizeof(u64) * s->K);
    frv_absorb(t, s, w);
    u64 rho = orc_tx_squeeze(t, "frv_rho");
    rd_fe(t, &rd, "frv_u", u, (u64)s->K);
    if (rd.bad) FAIL(REJ_FORMAT, 0, 0);
    frv_u(s, rho, want);
    for (int k = 0; k < s->K; k++)
        if (u[k] != want[k]) FAIL(REJ_FRV_U, k, 0);
    for (int i = 0; i < s->M; i++) {
        u64 lhs = 0, rhs = 0, pw = 1;
        for (int k = 0; k < s->K; k++) lhs = orc_fadd(lhs, orc_fmul(orc_fint(w_eff(s, i, k)), u[k]));
        for (int j = 0; j < s->N; j++) {
            /* Y[i][j] = 2^k q + r, witness stored token-major (N x M) */
            u64 y = orc_fadd(orc_fmul(orc_fint((int64_t)1 << s->k_shift), orc_fint(w->q[(u64)j * s->M + i])),
                             orc_fint(w->r[(u64)j * s->M + i]));
            rhs = orc_fadd(rhs, orc_fmul(y, pw));
            pw = orc_fmul(pw, rho);
        }
        if (lhs != rhs) FAIL(REJ_FRV_ROW, i, 0);
    }
    if (rd.pos != rd.len) FAIL(REJ_FORMAT, -1, 0);
done:
    free(u);
    free(want);
    return rc;
}

/* The matmul sum-check of one site with extension-field challenges (next    */
/* row f4): the statement of the matmul section for a single site, every     */
/* challenge and every sent value in F_p[phi] / (phi^2 - 7):                  */
/*   absorb "mm2_site" D(W) || D(S) || D(Xt) || D(q) || D(r);                  */
/*   squeeze r_row (vM coordinates, "mm2_row") and r_col (vN, "mm2_col");      */
/*   send c = Y~(r_row, r_col), Y = 2^k q + r ("mm2_claim");                   */
/*   A[k] = W_eff~(r_row, k), B[k] = X~(k, r_col) over K padded to 2^n;         */
/*   n rounds of g(0), g(1), g(2) of sum_b A(X, b) B(X, b) ("mm2_round"),      */
/*   "mm2_chal"; send A(rho), B(rho) ("mm2_final").                            */

static ext2 e2_lagrange3(const ext2 g[3], ext2 r) {
    ext2 acc = e2(0, 0);
    for (int i = 0; i < 3; i++) {
        ext2 num = e2(1, 0);
        int64_t den = 1;
        for (int j = 0; j < 3; j++) {
            if (j == i) continue;
            num = e2_mul(num, e2_sub(r, e2((u64)j, 0)));
            den *= (int64_t)(i - j);
        }
        acc = e2_add(acc, e2_mul(g[i], e2_scal(num, orc_finv(orc_fint(den)))));
    }
    return acc;
}

/* c, A, B of the site at (r_row, r_col); A, B of length 2^n */
static ext2 mm2_vectors(const orc_site* s, const orc_wit* w, const ext2* zr, int vM, const ext2* zc, int vN, int n,
                        ext2* A, ext2* B) {
    u64 Mp = (u64)1 << vM, Np = (u64)1 << vN, L = (u64)1 << n;
    ext2* er = (ext2*)malloc(sizeof(ext2) * Mp);
    ext2* ec = (ext2*)malloc(sizeof(ext2) * Np);
    e2_eq_table(zr, vM, er);
    e2_eq_table(zc, vN, ec);
    for (u64 k = 0; k < L; k++) A[k] = B[k] = e2(0, 0);
    for (int i = 0; i < s->M; i++)
        for (int k = 0; k < s->K; k++) A[k] = e2_add(A[k], e2_scal(er[i], orc_fint(w_eff(s, i, k))));
    for (int j = 0; j < s->N; j++)
        for (int k = 0; k < s->K; k++) B[k] = e2_add(B[k], e2_scal(ec[j], orc_fint(s->xt[(u64)j * s->K + k])));
    ext2 c = e2(0, 0);
    for (int i = 0; i < s->M; i++)
        for (int j = 0; j < s->N; j++) {
            u64 y = orc_fadd(orc_fmul(orc_fint((int64_t)1 << s->k_shift), orc_fint(w->q[(u64)j * s->M + i])),
                             orc_fint(w->r[(u64)j * s->M + i]));
            c = e2_add(c, e2_scal(e2_mul(er[i], ec[j]), y));
        }
    free(er);
    free(ec);
    return c;
}

int orc_mm2_prove(void* txh, const orc_site* s, const orc_wit* w, uint8_t* proof, u64 cap, u64* len) {
    if (s->M < 1 || s->N < 1 || s->K < 1) return -1;
    orc_tx* t = (orc_tx*)txh;
    int vM = orc_log2_ceil((u64)s->M), vN = orc_log2_ceil((u64)s->N), n = orc_log2_ceil((u64)s->K);
    u64 L = (u64)1 << n;
    pbuf pb = {proof, cap, 0, 0};
    {
        uint8_t d[160];
        site_digest160(s, w, d);
        orc_tx_absorb(t, "mm2_site", d, 160);
    }
    ext2* zr = (ext2*)malloc(sizeof(ext2) * (vM + 1));
    ext2* zc = (ext2*)malloc(sizeof(ext2) * (vN + 1));
    for (int i = 0; i < vM; i++) zr[i] = e2_squeeze(t, "mm2_row");
    for (int i = 0; i < vN; i++) zc[i] = e2_squeeze(t, "mm2_col");
    ext2* A = (ext2*)malloc(sizeof(ext2) * L);
    ext2* B = (ext2*)malloc(sizeof(ext2) * L);
    ext2 c = mm2_vectors(s, w, zr, vM, zc, vN, n, A, B);
    e2_send(t, &pb, "mm2_claim", &c, 1);
    u64 Lr = L;
    for (int r = 0; r < n; r++) {
        u64 h = Lr >> 1;
        ext2 g[3] = {e2(0, 0), e2(0, 0), e2(0, 0)};
        for (u64 b = 0; b < h; b++)
            for (u64 X = 0; X < 3; X++) {
                ext2 ax = e2_add(A[b], e2_scal(e2_sub(A[h + b], A[b]), X));
                ext2 bx = e2_add(B[b], e2_scal(e2_sub(B[h + b], B[b]), X));
                g[X] = e2_add(g[X], e2_mul(ax, bx));
            }
        e2_send(t, &pb, "mm2_round", g, 3);
        ext2 rho = e2_squeeze(t, "mm2_chal");
        for (u64 b = 0; b < h; b++) {
            A[b] = e2_add(A[b], e2_mul(rho, e2_sub(A[h + b], A[b])));
            B[b] = e2_add(B[b], e2_mul(rho, e2_sub(B[h + b], B[b])));
        }
        Lr = h;
    }
    ext2 fin[2] = {A[0], B[0]};
    e2_send(t, &pb, "mm2_final", fin, 2);
    free(zr);
    free(zc);
    free(A);
    free(B);
    *len = pb.len;
    return pb.overflow ? -2 : 0;
}

/* Verifier: the claim against Y, every round (g(0) + g(1) = claim, the next
 * claim g(rho) through the nodes 0, 1, 2), the end A(rho) B(rho) = claim, and
 * A(rho), B(rho) against the MLEs of W_eff and X it recomputes. */
int orc_mm2_verify(void* txh, const orc_site* s, const orc_wit* w, const uint8_t* proof, u64 len, int64_t detail[2]) {
    detail[0] = detail[1] = 0;
    if (s->M < 1 || s->N < 1 || s->K < 1) return REJ_ARGS;
    orc_tx* t = (orc_tx*)txh;
    int vM = orc_log2_ceil((u64)s->M), vN = orc_log2_ceil((u64)s->N), n = orc_log2_ceil((u64)s->K), rc = 0;
    u64 L = (u64)1 << n;
    prd rd = {proof, len, 0, 0};
    {
        uint8_t d[160];
        site_digest160(s, w, d);
        orc_tx_absorb(t, "mm2_site", d, 160);
    }
    ext2* zr = (ext2*)malloc(sizeof(ext2) * (vM + 1));
    ext2* zc = (ext2*)malloc(sizeof(ext2) * (vN + 1));
    ext2* rho = (ext2*)malloc(sizeof(ext2) * (n + 1));
    ext2* A = (ext2*)malloc(sizeof(ext2) * L);
    ext2* B = (ext2*)malloc(sizeof(ext2) * L);
    ext2* E = (ext2*)malloc(sizeof(ext2) * L);
    for (int i = 0; i < vM; i++) zr[i] = e2_squeeze(t, "mm2_row");
    for (int i = 0; i < vN; i++) zc[i] = e2_squeeze(t, "mm2_col");
    ext2 want = mm2_vectors(s, w, zr, vM, zc, vN, n, A, B);
    ext2 c, claim;
    e2_read(t, &rd, "mm2_claim", &c, 1);
    if (rd.bad) FAIL(REJ_FORMAT, 0, 0);
    if (c.a != want.a || c.b != want.b) FAIL(REJ_CLAIM, 0, 0);
    claim = c;
    for (int r = 0; r < n; r++) {
        ext2 g[3];
        e2_read(t, &rd, "mm2_round", g, 3);
        if (rd.bad) FAIL(REJ_FORMAT, 1, r);
        ext2 s01 = e2_add(g[0], g[1]);
        if (s01.a != claim.a || s01.b != claim.b) FAIL(REJ_MM_ROUND, r, 0);
        rho[r] = e2_squeeze(t, "mm2_chal");
        claim = e2_lagrange3(g, rho[r]);
    }
    ext2 fin[2];
    e2_read(t, &rd, "mm2_final", fin, 2);
    if (rd.bad) FAIL(REJ_FORMAT, 2, 0);
    {
        ext2 end = e2_mul(fin[0], fin[1]);
        if (end.a != claim.a || end.b != claim.b) FAIL(REJ_MM_FINAL, 0, 0);
    }
    {
        /* A(rho) = sum_k eq(rho, k) A[k] with A recomputed from W_eff (likewise B from X) */
        e2_eq_table(rho, n, E);
        ext2 a = e2(0, 0), b = e2(0, 0);
        for (u64 k = 0; k < L; k++) {
            a = e2_add(a, e2_mul(E[k], A[k]));
            b = e2_add(b, e2_mul(E[k], B[k]));
        }
        if (a.a != fin[0].a || a.b != fin[0].b) FAIL(REJ_MM_A, 0, 0);
        if (b.a != fin[1].a || b.b != fin[1].b) FAIL(REJ_MM_B, 0, 0);
    }
    if (rd.pos != rd.len) FAIL(REJ_FORMAT, -1, 0);
done:
    free(zr);
    free(zc);
    free(rho);
    free(A);
    free(B);
    free(E);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* MoE routing (next row f3; "How fast can FlashProve go", 2 Background, the */
/* note on MoE layers: they also prove the routing computation and each      */
/* token's choice of expert). Top-1 routing over E experts (E a power of     */
/* two): token t goes to e_t, the first index of the largest of its router   */
/* logits l[t][.] (int8, token-major T x E: the router matmul's rescaled      */
/* outputs). The prover commits the one-hot choice H[t][e] = [e = e_t] (u8)  */
/* and D[t][e] = l[t][e_t] - l[t][e] - [e < e_t] (int32), which lies in      */
/* [0, 256) for every e exactly when e_t is the first maximum. All columns   */
/* are zero-padded from T to 2^vT rows; x = t E + e, the t bits first.       */
/*   absorb "route_site" D(l) || D(H) || D(D as int32 little-endian);        */
/*   squeeze z (vT + vE, "route_z"), w (vT + vE, "route_w"), lambda1 and     */
/*   lambda2 ("route_lambda");                                               */
/*   send D~(z), l~(z) ("route_open");                                       */
/*   sum-check over vT + vE variables of                                    */
/*     F(x) = eq(z_t, t) H(x) (l(x) - G(e)) + lambda1 eq(w, x) H(x) (1 - H(x))*/
/*            + lambda2 eq(w_t, t) H(x),   G(e) = sum_{e' < e} eq(z_e, e'),   */
/*   claim D~(z) + l~(z) + lambda2 sum_{t < T} eq(w_t, t): rounds g(0..3)     */
/*   ("route_round"), "route_chal"; send H~(rho), l~(rho) ("route_final");  */
/*   then the helper-inverse LogUp of the keys D - 128 on R_8 (the statement */
/*   of orc_lhi_prove, T E keys, the same transcript).                       */
/* Why: sum_t eq(z_t, t) (l[t][e_t] - l~(t, z_e) - sum_e eq(z_e, e) [e < e_t])*/
/* is D~(z), and it equals the first sum minus l~(z) because                 */
/* sum_e eq(z_e, e) [e < e'] = G(e'); the second term forces H Boolean and   */
/* the third forces every real row of H to sum to 1 (padded rows to 0), each  */
/* with high probability over w; the range check then makes e_t the first    */
/* argmax.                                                                   */
/* ------------------------------------------------------------------------ */

enum {
    REJ_ROUTE_OPEN = 34,  /* an opened value != the column's MLE; detail[0]: 0 D(z), 1 l(z), 2 H(rho), 3 l(rho) */
    REJ_ROUTE_ROUND = 35, /* g(0) + g(1) != running claim; detail[0] = round */
    REJ_ROUTE_FINAL = 36  /* the end does not match F at rho */
};

/* the honest witness: H and D of the first argmax of every row */
void orc_route_witness(const int8_t* l, u64 T, int E, uint8_t* H, int32_t* D) {
    for (u64 t = 0; t < T; t++) {
        const int8_t* row = l + t * (u64)E;
        int best = 0;
        for (int e = 1; e < E; e++)
            if (row[e] > row[best]) best = e;
        for (int e = 0; e < E; e++) {
            H[t * (u64)E + e] = (uint8_t)(e == best);
            D[t * (u64)E + e] = (int32_t)row[best] - (int32_t)row[e] - (e < best ? 1 : 0);
        }
    }
}

typedef struct {
    int vT, vE, n;
    u64 L;
    u64 *z, *w, lam1, lam2;
    u64 *Hv, *lv, *Dv; /* lifted, zero-padded, length L */
} route_ctx;

static int route_begin(orc_tx* t, const int8_t* l, const uint8_t* H, const int32_t* D, u64 T, int E, route_ctx* c) {
    if (T < 1 || E < 1 || (E & (E - 1)) || E > 4096) return -1;
    c->vT = orc_log2_ceil(T);
    c->vE = orc_log2_ceil((u64)E);
    c->n = c->vT + c->vE;
    c->L = (u64)1 << c->n;
    u64 TE = T * (u64)E;
    uint8_t dg[96];
    uint8_t* db = (uint8_t*)calloc(4 * TE + 1, 1);
    for (u64 i = 0; i < TE; i++) put_le(db + 4 * i, (u64)(u32)D[i], 4);
    orc_tree_digest(l, TE, dg);
    orc_tree_digest(H, TE, dg + 32);
    orc_tree_digest(db, 4 * TE, dg + 64);
    free(db);
    orc_tx_absorb(t, "route_site", dg, 96);
    c->z = (u64*)malloc(sizeof(u64) * (c->n + 1));
    c->w = (u64*)malloc(sizeof(u64) * (c->n + 1));
    for (int i = 0; i < c->n; i++) c->z[i] = orc_tx_squeeze(t, "route_z");
    for (int i = 0; i < c->n; i++) c->w[i] = orc_tx_squeeze(t, "route_w");
    c->lam1 = orc_tx_squeeze(t, "route_lambda");
    c->lam2 = orc_tx_squeeze(t, "route_lambda");
    c->Hv = (u64*)calloc(c->L, sizeof(u64));
    c->lv = (u64*)calloc(c->L, sizeof(u64));
    c->Dv = (u64*)calloc(c->L, sizeof(u64));
    for (u64 i = 0; i < TE; i++) {
        c->Hv[i] = (u64)H[i] % ORC_P;
        c->lv[i] = orc_fint(l[i]);
        c->Dv[i] = orc_fint(D[i]);
    }
    return 0;
}

static void route_end(route_ctx* c) {
    free(c->z);
    free(c->w);
    free(c->Hv);
    free(c->lv);
    free(c->Dv);
}

/* G(e) = sum_{e' < e} eq(z_e, e') for e < E */
static void route_G(const u64* ze, int vE, int E, u64* G) {
    u64* eq = (u64*)malloc(sizeof(u64) * E);
    orc_eq_table(ze, vE, eq);
    u64 acc = 0;
    for (int e = 0; e < E; e++) {
        G[e] = acc;
        acc = orc_fadd(acc, eq[e]);
    }
    free(eq);
}

/* sum_{t < T} eq(w_t, t) */
static u64 route_rowsum(const u64* wt, int vT, u64 T) {
    u64* eq = (u64*)malloc(sizeof(u64) * ((u64)1 << vT));
    orc_eq_table(wt, vT, eq);
    u64 acc = 0;
    for (u64 t = 0; t < T; t++) acc = orc_fadd(acc, eq[t]);
    free(eq);
    return acc;
}

/* the keys D - 128 of the range lookup */
static int32_t* route_keys(const int32_t* D, u64 TE) {
    int32_t* k = (int32_t*)malloc(sizeof(int32_t) * (TE ? TE : 1));
    for (u64 i = 0; i < TE; i++) k[i] = (int32_t)((int64_t)D[i] - 128);
    return k;
}

int orc_route_prove(void* txh, const int8_t* l, const uint8_t* H, const int32_t* D, u64 T, int E, uint8_t* proof,
                    u64 cap, u64* len) {
    orc_tx* t = (orc_tx*)txh;
    route_ctx c;
    if (route_begin(t, l, H, D, T, E, &c)) return -1;
    pbuf pb = {proof, cap, 0, 0};
    u64 open[2] = {orc_mle_eval(c.Dv, c.L, c.z, c.n), orc_mle_eval(c.lv, c.L, c.z, c.n)};
    send_fe(t, &pb, "route_open", open, 2);
    /* the factors as vectors over x: eq(z_t, t), G(e), eq(w, x), eq(w_t, t) */
    u64 L = c.L;
    u64* Et = (u64*)malloc(sizeof(u64) * L);
    u64* Gv = (u64*)malloc(sizeof(u64) * L);
    u64* Ew = (u64*)malloc(sizeof(u64) * L);
    u64* Ewt = (u64*)malloc(sizeof(u64) * L);
    {
        u64* et = (u64*)malloc(sizeof(u64) * ((u64)1 << c.vT));
        u64* ewt = (u64*)malloc(sizeof(u64) * ((u64)1 << c.vT));
        u64* G = (u64*)malloc(sizeof(u64) * E);
        orc_eq_table(c.z, c.vT, et);
        orc_eq_table(c.w, c.vT, ewt);
        orc_eq_table(c.w, c.n, Ew);
        route_G(c.z + c.vT, c.vE, E, G);
        for (u64 x = 0; x < L; x++) {
            Et[x] = et[x >> c.vE];
            Ewt[x] = ewt[x >> c.vE];
            Gv[x] = G[x & (u64)(E - 1)];
        }
        free(et);
        free(ewt);
        free(G);
    }
    u64* V[6] = {Et, c.Hv, c.lv, Gv, Ew, Ewt};
    u64 Lr = L;
    for (int r = 0; r < c.n; r++) {
        u64 h = Lr >> 1;
        u64 g[4] = {0, 0, 0, 0};
        for (u64 b = 0; b < h; b++)
            for (u64 X = 0; X < 4; X++) {
                u64 at[6];
                for (int k = 0; k < 6; k++) at[k] = orc_fadd(V[k][b], orc_fmul(X, orc_fsub(V[k][h + b], V[k][b])));
                u64 Hx = at[1];
                u64 f = orc_fmul(at[0], orc_fmul(Hx, orc_fsub(at[2], at[3])));
                f = orc_fadd(f, orc_fmul(c.lam1, orc_fmul(at[4], orc_fmul(Hx, orc_fsub(1, Hx)))));
                f = orc_fadd(f, orc_fmul(c.lam2, orc_fmul(at[5], Hx)));
                g[X] = orc_fadd(g[X], f);
            }
        send_fe(t, &pb, "route_round", g, 4);
        u64 rho = orc_tx_squeeze(t, "route_chal");
        for (int k = 0; k < 6; k++)
            for (u64 b = 0; b < h; b++) V[k][b] = orc_fadd(V[k][b], orc_fmul(rho, orc_fsub(V[k][h + b], V[k][b])));
        Lr = h;
    }
    u64 fin[2] = {c.Hv[0], c.lv[0]};
    send_fe(t, &pb, "route_final", fin, 2);
    free(Et);
    free(Gv);
    free(Ew);
    free(Ewt);
    /* the range of D: the helper-inverse LogUp on R_8, continuing the transcript */
    u64 TE = T * (u64)E, l2 = 0;
    int32_t* keys = route_keys(D, TE);
    int rc = orc_lhi_prove(txh, keys, TE, 8, pb.overflow || !proof ? NULL : proof + pb.len,
                           pb.overflow || cap < pb.len ? 0 : cap - pb.len, &l2);
    free(keys);
    route_end(&c);
    *len = pb.len + l2;
    if (rc == -2 || pb.overflow) return -2;
    return rc;
}

int orc_route_verify(void* txh, const int8_t* l, const uint8_t* H, const int32_t* D, u64 T, int E,
                     const uint8_t* proof, u64 len, int64_t detail[2]) {
    detail[0] = detail[1] = 0;
    orc_tx* t = (orc_tx*)txh;
    route_ctx c;
    if (route_begin(t, l, H, D, T, E, &c)) return REJ_ARGS;
    int rc = 0;
    u64* rho = (u64*)malloc(sizeof(u64) * (c.n + 1));
    prd rd = {proof, len, 0, 0};
    u64 open[2];
    rd_fe(t, &rd, "route_open", open, 2);
    if (rd.bad) FAIL(REJ_FORMAT, 0, 0);
    if (open[0] != orc_mle_eval(c.Dv, c.L, c.z, c.n)) FAIL(REJ_ROUTE_OPEN, 0, 0);
    if (open[1] != orc_mle_eval(c.lv, c.L, c.z, c.n)) FAIL(REJ_ROUTE_OPEN, 1, 0);
    {
        u64 claim = orc_fadd(orc_fadd(open[0], open[1]), orc_fmul(c.lam2, route_rowsum(c.w, c.vT, T)));
        for (int r = 0; r < c.n; r++) {
            u64 g[4];
            rd_fe(t, &rd, "route_round", g, 4);
            if (rd.bad) FAIL(REJ_FORMAT, 1, r);
            if (orc_fadd(g[0], g[1]) != claim) FAIL(REJ_ROUTE_ROUND, r, 0);
            rho[r] = orc_tx_squeeze(t, "route_chal");
            claim = orc_lagrange(g, 4, rho[r]);
        }
        u64 fin[2];
        rd_fe(t, &rd, "route_final", fin, 2);
        if (rd.bad) FAIL(REJ_FORMAT, 2, 0);
        if (fin[0] != orc_mle_eval(c.Hv, c.L, rho, c.n)) FAIL(REJ_ROUTE_OPEN, 2, 0);
        if (fin[1] != orc_mle_eval(c.lv, c.L, rho, c.n)) FAIL(REJ_ROUTE_OPEN, 3, 0);
        u64* G = (u64*)malloc(sizeof(u64) * E);
        route_G(c.z + c.vT, c.vE, E, G);
        u64 Gr = orc_mle_eval(G, (u64)E, rho + c.vT, c.vE);
        free(G);
        u64 Hr = fin[0], lr = fin[1];
        u64 f = orc_fmul(eq_closed(c.z, rho, c.vT), orc_fmul(Hr, orc_fsub(lr, Gr)));
        f = orc_fadd(f, orc_fmul(c.lam1, orc_fmul(eq_closed(c.w, rho, c.n), orc_fmul(Hr, orc_fsub(1, Hr)))));
        f = orc_fadd(f, orc_fmul(c.lam2, orc_fmul(eq_closed(c.w, rho, c.vT), Hr)));
        if (f != claim) FAIL(REJ_ROUTE_FINAL, 0, 0);
    }
    {
        u64 TE = T * (u64)E;
        int32_t* keys = route_keys(D, TE);
        rc = orc_lhi_verify(txh, keys, TE, 8, proof + rd.pos, len - rd.pos, detail);
        free(keys);
    }
done:
    free(rho);
    route_end(&c);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* The helper-inverse LogUp over the extension (next row f4: challenges in   */
/* F_p[phi] / (phi^2 - 7), "How fast can FlashProve go", 4, the note on      */
/* soundness). The statement of orc_lhi_prove with alpha, z, beta, every     */
/* challenge and every value sent in the extension (16 bytes each); the      */
/* helper column holds extension elements:                                  */
/*   absorb "lhi2_site" D(r); send m (2^k u32, digest absorbed, "lhi2_m");   */
/*   squeeze alpha ("lhi2_alpha"); commit h_i = 1 / (alpha - r_i): absorb    */
/*   "lhi2_h" D(h as (a, b) u64 little-endian pairs); squeeze z_1..z_v       */
/*   ("lhi2_z") and beta ("lhi2_beta"); send S = sum_i h_i ("lhi2_sum");     */
/*   sum-check of h + beta eq(z, x) (h (alpha - f) - 1) over v variables,     */
/*   claim S: rounds g(0..3) ("lhi2_round"), "lhi2_chal"; send h(rho),       */
/*   f(rho) ("lhi2_final").                                                  */
/* The verifier checks as for orc_lhi_verify, in the extension.              */
/* ------------------------------------------------------------------------ */

enum {
    REJ_LHI2_SUM = 37,    /* S != the table side */
    REJ_LHI2_ROUND = 38,  /* g(0) + g(1) != running claim */
    REJ_LHI2_FINAL = 39,  /* the end does not match F at rho */
    REJ_LHI2_OPEN = 40    /* h(rho) or f(rho) != the columns' MLEs */
};

/* 1 / (a + b phi) = (a - b phi) / (a^2 - 7 b^2); 0 for 0 */
static ext2 e2_inv(ext2 x) {
    u64 nrm = orc_fsub(orc_fmul(x.a, x.a), orc_fmul(7, orc_fmul(x.b, x.b)));
    u64 ni = orc_finv(nrm);
    return e2(orc_fmul(x.a, ni), orc_fsub(0, orc_fmul(x.b, ni)));
}

/* eq(z, rho) = prod_i (z_i rho_i + (1 - z_i)(1 - rho_i)) in the extension */
static ext2 e2_eq_closed(const ext2* z, const ext2* rho, int v) {
    ext2 e = e2(1, 0), one = e2(1, 0);
    for (int i = 0; i < v; i++)
        e = e2_mul(e, e2_add(e2_mul(z[i], rho[i]), e2_mul(e2_sub(one, z[i]), e2_sub(one, rho[i]))));
    return e;
}

static void lhi2_columns(const int32_t* r, u64 n, int v, ext2 alpha, ext2* f, ext2* h) {
    u64 L = (u64)1 << v;
    for (u64 i = 0; i < L; i++) {
        f[i] = e2(i < n ? orc_fint(r[i]) : 0, 0);
        h[i] = e2_inv(e2_sub(alpha, f[i]));
    }
}

static void lhi2_absorb_h(orc_tx* t, const ext2* h, u64 L) {
    uint8_t* b = (uint8_t*)malloc(16 * L);
    uint8_t d[32];
    for (u64 i = 0; i < L; i++) {
        put_le(b + 16 * i, h[i].a, 8);
        put_le(b + 16 * i + 8, h[i].b, 8);
    }
    orc_tree_digest(b, 16 * L, d);
    free(b);
    orc_tx_absorb(t, "lhi2_h", d, 32);
}

static void lhi2_absorb_site(orc_tx* t, const int32_t* r, u64 n) {
    uint8_t* b = (uint8_t*)calloc(4 * n, 1);
    uint8_t d[32];
    for (u64 i = 0; i < n; i++) put_le(b + 4 * i, (u64)(u32)r[i], 4);
    orc_tree_digest(b, 4 * n, d);
    free(b);
    orc_tx_absorb(t, "lhi2_site", d, 32);
}

/* F at one point of the three lines: h + beta e (h (alpha - f) - 1) */
static ext2 lhi2_F(ext2 h, ext2 f, ext2 e, ext2 alpha, ext2 beta) {
    return e2_add(h, e2_mul(beta, e2_mul(e, e2_sub(e2_mul(h, e2_sub(alpha, f)), e2(1, 0)))));
}

int orc_lhi2_prove(void* txh, const int32_t* r, u64 n, int k, uint8_t* proof, u64 cap, u64* len) {
    if (n < 1 || k < 1 || k > 24) return -1;
    orc_tx* t = (orc_tx*)txh;
    int v = orc_log2_ceil(n);
    if (v < 1) v = 1;
    u64 L = (u64)1 << v, T = (u64)1 << k;
    pbuf pb = {proof, cap, 0, 0};
    lhi2_absorb_site(t, r, n);
    u32* m = (u32*)malloc(T * sizeof(u32));
    lhi_mult(r, n, L, k, m);
    send_mult(t, &pb, "lhi2_m", m, T);
    ext2 alpha = e2_squeeze(t, "lhi2_alpha");
    ext2* f = (ext2*)malloc(L * sizeof(ext2));
    ext2* h = (ext2*)malloc(L * sizeof(ext2));
    ext2* E = (ext2*)malloc(L * sizeof(ext2));
    ext2* z = (ext2*)malloc(sizeof(ext2) * v);
    lhi2_columns(r, n, v, alpha, f, h);
    lhi2_absorb_h(t, h, L);
    for (int i = 0; i < v; i++) z[i] = e2_squeeze(t, "lhi2_z");
    ext2 beta = e2_squeeze(t, "lhi2_beta");
    ext2 S = e2(0, 0);
    for (u64 i = 0; i < L; i++) S = e2_add(S, h[i]);
    e2_send(t, &pb, "lhi2_sum", &S, 1);
    e2_eq_table(z, v, E);
    u64 Lr = L;
    for (int rd = 0; rd < v; rd++) {
        u64 hh = Lr >> 1;
        ext2 g[4] = {e2(0, 0), e2(0, 0), e2(0, 0), e2(0, 0)};
        for (u64 b = 0; b < hh; b++)
            for (u64 X = 0; X < 4; X++) {
                ext2 hx = e2_add(h[b], e2_scal(e2_sub(h[hh + b], h[b]), X));
                ext2 fx = e2_add(f[b], e2_scal(e2_sub(f[hh + b], f[b]), X));
                ext2 ex = e2_add(E[b], e2_scal(e2_sub(E[hh + b], E[b]), X));
                g[X] = e2_add(g[X], lhi2_F(hx, fx, ex, alpha, beta));
            }
        e2_send(t, &pb, "lhi2_round", g, 4);
        ext2 rho = e2_squeeze(t, "lhi2_chal");
        for (u64 b = 0; b < hh; b++) {
            h[b] = e2_add(h[b], e2_mul(rho, e2_sub(h[hh + b], h[b])));
            f[b] = e2_add(f[b], e2_mul(rho, e2_sub(f[hh + b], f[b])));
            E[b] = e2_add(E[b], e2_mul(rho, e2_sub(E[hh + b], E[b])));
        }
        Lr = hh;
    }
    ext2 fin[2] = {h[0], f[0]};
    e2_send(t, &pb, "lhi2_final", fin, 2);
    free(m);
    free(f);
    free(h);
    free(E);
    free(z);
    *len = pb.len;
    return pb.overflow ? -2 : 0;
}

int orc_lhi2_verify(void* txh, const int32_t* r, u64 n, int k, const uint8_t* proof, u64 len, int64_t detail[2]) {
    detail[0] = detail[1] = 0;
    if (n < 1 || k < 1 || k > 24) return REJ_ARGS;
    orc_tx* t = (orc_tx*)txh;
    int v = orc_log2_ceil(n), rc = 0;
    if (v < 1) v = 1;
    u64 L = (u64)1 << v, T = (u64)1 << k;
    prd rd = {proof, len, 0, 0};
    u32* m = (u32*)malloc(T * sizeof(u32));
    ext2* f = (ext2*)malloc(L * sizeof(ext2));
    ext2* h = (ext2*)malloc(L * sizeof(ext2));
    ext2* E = (ext2*)malloc(L * sizeof(ext2));
    ext2* z = (ext2*)malloc(sizeof(ext2) * v);
    ext2* rho = (ext2*)malloc(sizeof(ext2) * v);
    lhi2_absorb_site(t, r, n);
    rd_mult(t, &rd, "lhi2_m", m, T);
    if (rd.bad) FAIL(REJ_FORMAT, 0, 0);
    ext2 alpha = e2_squeeze(t, "lhi2_alpha");
    lhi2_columns(r, n, v, alpha, f, h); /* the verifier holds the key column, so h too */
    lhi2_absorb_h(t, h, L);
    for (int i = 0; i < v; i++) z[i] = e2_squeeze(t, "lhi2_z");
    ext2 beta = e2_squeeze(t, "lhi2_beta");
    ext2 S;
    e2_read(t, &rd, "lhi2_sum", &S, 1);
    if (rd.bad) FAIL(REJ_FORMAT, 1, 0);
    {
        /* the table side: sum_j m_j / (alpha - t_j) as one fraction P / Q */
        ext2 P = e2(0, 0), Q = e2(1, 0);
        for (u64 j = 0; j < T; j++) {
            ext2 dj = e2_sub(alpha, e2(orc_fint((int64_t)j - ((int64_t)1 << (k - 1))), 0));
            P = e2_add(e2_mul(P, dj), e2_scal(Q, (u64)m[j]));
            Q = e2_mul(Q, dj);
        }
        ext2 lhs = e2_mul(S, Q);
        if (lhs.a != P.a || lhs.b != P.b) FAIL(REJ_LHI2_SUM, 0, 0);
    }
    {
        ext2 claim = S;
        for (int i = 0; i < v; i++) {
            ext2 g[4];
            e2_read(t, &rd, "lhi2_round", g, 4);
            if (rd.bad) FAIL(REJ_FORMAT, 2, i);
            ext2 s01 = e2_add(g[0], g[1]);
            if (s01.a != claim.a || s01.b != claim.b) FAIL(REJ_LHI2_ROUND, i, 0);
            rho[i] = e2_squeeze(t, "lhi2_chal");
            claim = e2_lagrange4(g, rho[i]);
        }
        ext2 fin[2];
        e2_read(t, &rd, "lhi2_final", fin, 2);
        if (rd.bad) FAIL(REJ_FORMAT, 3, 0);
        ext2 want = lhi2_F(fin[0], fin[1], e2_eq_closed(z, rho, v), alpha, beta);
        if (want.a != claim.a || want.b != claim.b) FAIL(REJ_LHI2_FINAL, 0, 0);
        e2_eq_table(rho, v, E);
        ext2 hr = e2(0, 0), fr = e2(0, 0);
        for (u64 x = 0; x < L; x++) {
            hr = e2_add(hr, e2_mul(E[x], h[x]));
            fr = e2_add(fr, e2_mul(E[x], f[x]));
        }
        if (hr.a != fin[0].a || hr.b != fin[0].b) FAIL(REJ_LHI2_OPEN, 0, 0);
        if (fr.a != fin[1].a || fr.b != fin[1].b) FAIL(REJ_LHI2_OPEN, 1, 0);
    }
    if (rd.pos != rd.len) FAIL(REJ_FORMAT, -1, 0);
done:
    free(m);
    free(f);
    free(h);
    free(E);
    free(z);
    free(rho);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* The 16-bit function lookup (the LogUp-GKR tree of lookup16_prove) over    */
/* the extension (next row f4, "How fast can FlashProve go", 4, the note on  */
/* soundness): gamma, alpha, mu, lambda, every round challenge and every     */
/* value sent are extension elements (16 bytes); the tree's fractions live   */
/* in the extension; labels "<fn>2_*" (silu2_site, silu2_gamma, silu2_m,     */
/* silu2_alpha, silu2_l1, silu2_mu, silu2_lambda, silu2_round, silu2_chal,   */
/* silu2_final, silu2_leaf; exp2_* likewise). Keys f = g + gamma s, padded   */
/* with (0, table(0)); the verifier checks the root against the table side   */
/* sum_j m_j / (alpha - v_j - gamma table(v_j)) in the extension.            */
/* ------------------------------------------------------------------------ */

static const lk_labels LK_SILU2 = {"silu2_site", "silu2_gamma", "silu2_m", "silu2_alpha", "silu2_l1", "silu2_mu",
                                   "silu2_lambda", "silu2_round", "silu2_chal", "silu2_final", "silu2_leaf"};
static const lk_labels LK_EXP2 = {"exp2_site", "exp2_gamma", "exp2_m", "exp2_alpha", "exp2_l1", "exp2_mu",
                                  "exp2_lambda", "exp2_round", "exp2_chal", "exp2_final", "exp2_leaf"};

static ext2 x16_F(const ext2 x[4], ext2 lam) { /* pL qR + pR qL + lambda qL qR */
    return e2_add(e2_add(e2_mul(x[0], x[3]), e2_mul(x[1], x[2])), e2_mul(lam, e2_mul(x[2], x[3])));
}

/* MLE at an extension point of a base column given as field elements */
static ext2 x16_mle(const u64* col, u64 L, const ext2* z, int v) {
    ext2* E = (ext2*)malloc(sizeof(ext2) * L);
    e2_eq_table(z, v, E);
    ext2 acc = e2(0, 0);
    for (u64 x = 0; x < L; x++) acc = e2_add(acc, e2_scal(E[x], col[x]));
    free(E);
    return acc;
}

static void x16_leaf_values(const int16_t* g, const int16_t* s, u64 n, int v, const ext2* z, int32_t pad_s,
                            ext2 out[2]) {
    u64 L = (u64)1 << v;
    u64* col = (u64*)malloc(L * sizeof(u64));
    for (u64 i = 0; i < L; i++) col[i] = i < n ? orc_fint(g[i]) : 0;
    out[0] = x16_mle(col, L, z, v);
    for (u64 i = 0; i < L; i++) col[i] = i < n ? orc_fint(s[i]) : orc_fint(pad_s);
    out[1] = x16_mle(col, L, z, v);
    free(col);
}

static int lookup16x_prove(void* txh, const lk_labels* lab, int32_t pad_s, const int16_t* g, const int16_t* s, u64 n,
                           uint8_t* proof, u64 cap, u64* len) {
    if (n < 1) return -1;
    orc_tx* t = (orc_tx*)txh;
    int v = orc_log2_ceil(n);
    if (v < 1) v = 1;
    u64 L = (u64)1 << v;
    pbuf pb = {proof, cap, 0, 0};
    silu_absorb_site(t, lab, g, s, n);
    ext2 gamma = e2_squeeze(t, lab->gamma);
    u32* m = (u32*)malloc(65536 * sizeof(u32));
    silu_mult(g, n, L, m);
    send_mult(t, &pb, lab->m, m, 65536);
    ext2 alpha = e2_squeeze(t, lab->alpha);
    /* the fraction tree: layer d has 2^d nodes */
    ext2** Pd = (ext2**)malloc(sizeof(ext2*) * (v + 1));
    ext2** Qd = (ext2**)malloc(sizeof(ext2*) * (v + 1));
    Pd[v] = (ext2*)malloc(L * sizeof(ext2));
    Qd[v] = (ext2*)malloc(L * sizeof(ext2));
    for (u64 i = 0; i < L; i++) {
        ext2 f = i < n ? e2_add(e2(orc_fint(g[i]), 0), e2_scal(gamma, orc_fint(s[i]))) : e2_scal(gamma, orc_fint(pad_s));
        Pd[v][i] = e2(1, 0);
        Qd[v][i] = e2_sub(alpha, f);
    }
    for (int d = v - 1; d >= 0; d--) {
        u64 c = (u64)1 << d;
        Pd[d] = (ext2*)malloc(c * sizeof(ext2));
        Qd[d] = (ext2*)malloc(c * sizeof(ext2));
        for (u64 x = 0; x < c; x++) {
            Pd[d][x] = e2_add(e2_mul(Pd[d + 1][2 * x], Qd[d + 1][2 * x + 1]), e2_mul(Pd[d + 1][2 * x + 1], Qd[d + 1][2 * x]));
            Qd[d][x] = e2_mul(Qd[d + 1][2 * x], Qd[d + 1][2 * x + 1]);
        }
    }
    ext2 l1[4] = {Pd[1][0], Pd[1][1], Qd[1][0], Qd[1][1]};
    e2_send(t, &pb, lab->l1, l1, 4);
    ext2* z = (ext2*)malloc(sizeof(ext2) * (v + 1));
    z[0] = e2_squeeze(t, lab->mu);
    for (int d = 1; d < v; d++) {
        ext2 lam = e2_squeeze(t, lab->lambda);
        u64 c = (u64)1 << d;
        ext2* V[5]; /* pL, pR, qL, qR (children of layer d), eq(z, .) */
        for (int i = 0; i < 5; i++) V[i] = (ext2*)malloc(c * sizeof(ext2));
        for (u64 x = 0; x < c; x++) {
            V[0][x] = Pd[d + 1][2 * x];
            V[1][x] = Pd[d + 1][2 * x + 1];
            V[2][x] = Qd[d + 1][2 * x];
            V[3][x] = Qd[d + 1][2 * x + 1];
        }
        e2_eq_table(z, d, V[4]);
        ext2* rho = (ext2*)malloc(sizeof(ext2) * d);
        u64 Lr = c;
        for (int r = 0; r < d; r++) {
            u64 h = Lr >> 1;
            ext2 gr[4] = {e2(0, 0), e2(0, 0), e2(0, 0), e2(0, 0)};
            for (u64 b = 0; b < h; b++)
                for (u64 X = 0; X < 4; X++) {
                    ext2 ev[5];
                    for (int i = 0; i < 5; i++) ev[i] = e2_add(V[i][b], e2_scal(e2_sub(V[i][h + b], V[i][b]), X));
                    gr[X] = e2_add(gr[X], e2_mul(ev[4], x16_F(ev, lam)));
                }
            e2_send(t, &pb, lab->round, gr, 4);
            rho[r] = e2_squeeze(t, lab->chal);
            for (int i = 0; i < 5; i++)
                for (u64 b = 0; b < h; b++) V[i][b] = e2_add(V[i][b], e2_mul(rho[r], e2_sub(V[i][h + b], V[i][b])));
            Lr = h;
        }
        ext2 fin[4] = {V[0][0], V[1][0], V[2][0], V[3][0]};
        e2_send(t, &pb, lab->fin, fin, 4);
        ext2 mu = e2_squeeze(t, lab->mu);
        for (int r = 0; r < d; r++) z[r] = rho[r];
        z[d] = mu;
        for (int i = 0; i < 5; i++) free(V[i]);
        free(rho);
    }
    ext2 leaf[2];
    x16_leaf_values(g, s, n, v, z, pad_s, leaf);
    e2_send(t, &pb, lab->leaf, leaf, 2);
    for (int d = 0; d <= v; d++) {
        free(Pd[d]);
        free(Qd[d]);
    }
    free(Pd);
    free(Qd);
    free(z);
    free(m);
    *len = pb.len;
    return pb.overflow ? -2 : 0;
}

static int e2_eqv(ext2 x, ext2 y) { return x.a == y.a && x.b == y.b; }

static int lookup16x_verify(void* txh, const lk_labels* lab, int32_t (*tab)(int32_t), const int16_t* g,
                            const int16_t* s, u64 n, const uint8_t* proof, u64 len, int64_t detail[2]) {
    detail[0] = detail[1] = 0;
    if (n < 1) return REJ_ARGS;
    orc_tx* t = (orc_tx*)txh;
    int v = orc_log2_ceil(n), rc = 0;
    if (v < 1) v = 1;
    prd rd = {proof, len, 0, 0};
    u32* m = (u32*)malloc(65536 * sizeof(u32));
    ext2* z = (ext2*)malloc(sizeof(ext2) * (v + 1));
    ext2* rho = (ext2*)malloc(sizeof(ext2) * (v + 1));
    silu_absorb_site(t, lab, g, s, n);
    ext2 gamma = e2_squeeze(t, lab->gamma);
    rd_mult(t, &rd, lab->m, m, 65536);
    if (rd.bad) FAIL(REJ_FORMAT, 0, 0);
    ext2 alpha = e2_squeeze(t, lab->alpha);
    ext2 l1[4];
    e2_read(t, &rd, lab->l1, l1, 4);
    if (rd.bad) FAIL(REJ_FORMAT, 1, 0);
    {
        /* the table side, sum_j m_j / (alpha - t_j) with t_j = v_j + gamma tab(v_j) */
        ext2 PT = e2(0, 0), QT = e2(1, 0);
        for (u64 j = 0; j < 65536; j++) {
            int32_t vj = (int32_t)j - 32768;
            ext2 dj = e2_sub(alpha, e2_add(e2(orc_fint(vj), 0), e2_scal(gamma, orc_fint(tab(vj)))));
            PT = e2_add(e2_mul(PT, dj), e2_scal(QT, (u64)m[j]));
            QT = e2_mul(QT, dj);
        }
        ext2 P0 = e2_add(e2_mul(l1[0], l1[3]), e2_mul(l1[1], l1[2]));
        ext2 Q0 = e2_mul(l1[2], l1[3]);
        if ((Q0.a == 0 && Q0.b == 0) || !e2_eqv(e2_mul(P0, QT), e2_mul(Q0, PT))) FAIL(REJ_SILU_ROOT, 0, 0);
    }
    ext2 mu = e2_squeeze(t, lab->mu);
    ext2 cP = e2_add(l1[0], e2_mul(mu, e2_sub(l1[1], l1[0])));
    ext2 cQ = e2_add(l1[2], e2_mul(mu, e2_sub(l1[3], l1[2])));
    z[0] = mu;
    for (int d = 1; d < v; d++) {
        ext2 lam = e2_squeeze(t, lab->lambda);
        ext2 claim = e2_add(cP, e2_mul(lam, cQ));
        for (int r = 0; r < d; r++) {
            ext2 gr[4];
            e2_read(t, &rd, lab->round, gr, 4);
            if (rd.bad) FAIL(REJ_FORMAT, 2, d);
            if (!e2_eqv(e2_add(gr[0], gr[1]), claim)) FAIL(REJ_SILU_ROUND, d, r);
            rho[r] = e2_squeeze(t, lab->chal);
            claim = e2_lagrange4(gr, rho[r]);
        }
        ext2 fin[4];
        e2_read(t, &rd, lab->fin, fin, 4);
        if (rd.bad) FAIL(REJ_FORMAT, 3, d);
        if (!e2_eqv(e2_mul(e2_eq_closed(z, rho, d), x16_F(fin, lam)), claim)) FAIL(REJ_SILU_FINAL, d, 0);
        mu = e2_squeeze(t, lab->mu);
        cP = e2_add(fin[0], e2_mul(mu, e2_sub(fin[1], fin[0])));
        cQ = e2_add(fin[2], e2_mul(mu, e2_sub(fin[3], fin[2])));
        for (int r = 0; r < d; r++) z[r] = rho[r];
        z[d] = mu;
    }
    ext2 leaf[2];
    e2_read(t, &rd, lab->leaf, leaf, 2);
    if (rd.bad) FAIL(REJ_FORMAT, 4, 0);
    if (!e2_eqv(cP, e2(1, 0))) FAIL(REJ_SILU_LEAF, 0, 0);
    if (!e2_eqv(cQ, e2_sub(alpha, e2_add(leaf[0], e2_mul(gamma, leaf[1]))))) FAIL(REJ_SILU_LEAF, 1, 0);
    {
        ext2 want[2];
        x16_leaf_values(g, s, n, v, z, tab(0), want);
        if (!e2_eqv(want[0], leaf[0])) FAIL(REJ_SILU_OPEN, 0, 0);
        if (!e2_eqv(want[1], leaf[1])) FAIL(REJ_SILU_OPEN, 1, 0);
    }
    if (rd.pos != rd.len) FAIL(REJ_FORMAT, -1, 0);
done:
    free(m);
    free(z);
    free(rho);
    return rc;
}

int orc_silu2_prove(void* txh, const int16_t* g, const int16_t* s, u64 n, uint8_t* proof, u64 cap, u64* len) {
    return lookup16x_prove(txh, &LK_SILU2, orc_silu_q(0), g, s, n, proof, cap, len);
}
int orc_silu2_verify(void* txh, const int16_t* g, const int16_t* s, u64 n, const uint8_t* proof, u64 len,
                     int64_t detail[2]) {
    return lookup16x_verify(txh, &LK_SILU2, orc_silu_q, g, s, n, proof, len, detail);
}
int orc_exp2_prove(void* txh, const int16_t* g, const int16_t* s, u64 n, uint8_t* proof, u64 cap, u64* len) {
    return lookup16x_prove(txh, &LK_EXP2, orc_exp_q(0), g, s, n, proof, cap, len);
}
int orc_exp2_verify(void* txh, const int16_t* g, const int16_t* s, u64 n, const uint8_t* proof, u64 len,
                    int64_t detail[2]) {
    return lookup16x_verify(txh, &LK_EXP2, orc_exp_q, g, s, n, proof, len, detail);
}

/* ------------------------------------------------------------------------ */
/* The rescale LogUp (the two tables of lu_prove, batched in one GKR) over   */
/* the extension (next row f4, "How fast can FlashProve go", 4, the note on  */
/* soundness), as a statement of its own over the sites' key columns:       */
/*   absorb "lu2_site" D(r) || D(q) (int32 little-endian) || D(y) of the     */
/*   concatenated, unpadded key columns; send m_rem ("lu2_m_rem"); squeeze    */
/*   gamma ("lu2_gamma"); send m_clamp ("lu2_m_clamp"); squeeze alpha_0,      */
/*   alpha_1 ("lu2_alpha"); then lu_prove's layers with every challenge and   */
/*   value in F_p[phi]/(phi^2 - 7): "lu2_l1" (8 values), "lu2_mu",            */
/*   "lu2_lambda", "lu2_round", "lu2_chal", "lu2_final" (8 values), and the  */
/*   leaf claims r~(z), q~(z), y~(z) ("lu2_leaf").                            */
/* ------------------------------------------------------------------------ */

static void lu2_absorb_site(orc_tx* t, const orc_keys* K) {
    u64 nk = K->nk;
    uint8_t* b = (uint8_t*)calloc(4 * nk + 1, 1);
    uint8_t d[96];
    for (u64 i = 0; i < nk; i++) put_le(b + 4 * i, (u64)(u32)(int32_t)K->fr[i], 4);
    orc_tree_digest(b, 4 * nk, d);
    for (u64 i = 0; i < nk; i++) put_le(b + 4 * i, (u64)(u32)(int32_t)K->fq[i], 4);
    orc_tree_digest(b, 4 * nk, d + 32);
    for (u64 i = 0; i < nk; i++) b[i] = (uint8_t)(int8_t)K->fy[i];
    orc_tree_digest(b, nk, d + 64);
    free(b);
    orc_tx_absorb(t, "lu2_site", d, 96);
}

static ext2 lu2_key(const orc_keys* K, int tab, u64 i, ext2 gamma) {
    if (tab == 0) return e2(orc_fint(K->fr[i]), 0);
    return e2_add(e2(orc_fint(K->fq[i]), 0), e2_scal(gamma, orc_fint(K->fy[i])));
}

/* layer summand: sum over tables tau of lambda^(2 tau) (pL qR + pR qL + lambda qL qR) */
static ext2 lu2_F(const ext2 v8[8], ext2 lam, ext2 lam2) {
    ext2 acc = e2(0, 0), w = e2(1, 0);
    for (int tau = 0; tau < 2; tau++) {
        const ext2* x = v8 + 4 * tau;
        ext2 f = e2_add(e2_add(e2_mul(x[0], x[3]), e2_mul(x[1], x[2])), e2_mul(lam, e2_mul(x[2], x[3])));
        acc = e2_add(acc, e2_mul(w, f));
        w = lam2;
    }
    return acc;
}

static ext2 lu2_fold(ext2 a, ext2 b, ext2 r) { return e2_add(a, e2_mul(r, e2_sub(b, a))); }

int orc_lu2_prove(void* txh, const orc_site* sites, int ns, const orc_wit* wit, uint8_t* proof, u64 cap, u64* len) {
    orc_tx* t = (orc_tx*)txh;
    orc_keys K;
    if (ns < 1 || keys_build(sites, ns, wit, &K) != 0) return -1;
    pbuf pb = {proof, cap, 0, 0};
    int v = K.v;
    u64 L = (u64)1 << v, Trem = (u64)1 << K.k;
    lu2_absorb_site(t, &K);
    u32* mr = (u32*)malloc(Trem * sizeof(u32));
    u32* mc = (u32*)malloc(65536 * sizeof(u32));
    mult_rem(&K, mr);
    send_mult(t, &pb, "lu2_m_rem", mr, Trem);
    ext2 gamma = e2_squeeze(t, "lu2_gamma");
    mult_clamp(&K, mc);
    send_mult(t, &pb, "lu2_m_clamp", mc, 65536);
    ext2 alpha[2];
    alpha[0] = e2_squeeze(t, "lu2_alpha");
    alpha[1] = e2_squeeze(t, "lu2_alpha");
    /* the two fraction trees: layer d has 2^d nodes */
    ext2** P[2];
    ext2** Q[2];
    for (int tau = 0; tau < 2; tau++) {
        P[tau] = (ext2**)malloc(sizeof(ext2*) * (v + 1));
        Q[tau] = (ext2**)malloc(sizeof(ext2*) * (v + 1));
        P[tau][v] = (ext2*)malloc(L * sizeof(ext2));
        Q[tau][v] = (ext2*)malloc(L * sizeof(ext2));
        for (u64 i = 0; i < L; i++) {
            P[tau][v][i] = e2(1, 0);
            Q[tau][v][i] = e2_sub(alpha[tau], lu2_key(&K, tau, i, gamma));
        }
        for (int d = v - 1; d >= 0; d--) {
            u64 c = (u64)1 << d;
            P[tau][d] = (ext2*)malloc(c * sizeof(ext2));
            Q[tau][d] = (ext2*)malloc(c * sizeof(ext2));
            for (u64 x = 0; x < c; x++) {
                ext2 pl = P[tau][d + 1][2 * x], pr = P[tau][d + 1][2 * x + 1];
                ext2 ql = Q[tau][d + 1][2 * x], qr = Q[tau][d + 1][2 * x + 1];
                P[tau][d][x] = e2_add(e2_mul(pl, qr), e2_mul(pr, ql));
                Q[tau][d][x] = e2_mul(ql, qr);
            }
        }
    }
    ext2 l1[8];
    for (int tau = 0; tau < 2; tau++) {
        l1[4 * tau + 0] = P[tau][1][0];
        l1[4 * tau + 1] = P[tau][1][1];
        l1[4 * tau + 2] = Q[tau][1][0];
        l1[4 * tau + 3] = Q[tau][1][1];
    }
    e2_send(t, &pb, "lu2_l1", l1, 8);
    ext2* z = (ext2*)malloc(sizeof(ext2) * (v + 1));
    z[0] = e2_squeeze(t, "lu2_mu");
    for (int d = 1; d < v; d++) {
        ext2 lam = e2_squeeze(t, "lu2_lambda");
        ext2 lam2 = e2_mul(lam, lam);
        u64 c = (u64)1 << d;
        ext2* V[9];
        for (int i = 0; i < 9; i++) V[i] = (ext2*)malloc(c * sizeof(ext2));
        for (int tau = 0; tau < 2; tau++)
            for (u64 x = 0; x < c; x++) {
                V[4 * tau + 0][x] = P[tau][d + 1][2 * x];
                V[4 * tau + 1][x] = P[tau][d + 1][2 * x + 1];
                V[4 * tau + 2][x] = Q[tau][d + 1][2 * x];
                V[4 * tau + 3][x] = Q[tau][d + 1][2 * x + 1];
            }
        e2_eq_table(z, d, V[8]);
        ext2* rho = (ext2*)malloc(sizeof(ext2) * d);
        u64 Lr = c;
        for (int r = 0; r < d; r++) {
            u64 h = Lr >> 1;
            ext2 g[4] = {e2(0, 0), e2(0, 0), e2(0, 0), e2(0, 0)};
            for (u64 b = 0; b < h; b++)
                for (u64 X = 0; X < 4; X++) {
                    ext2 ev[9];
                    for (int i = 0; i < 9; i++) ev[i] = e2_add(V[i][b], e2_scal(e2_sub(V[i][h + b], V[i][b]), X));
                    g[X] = e2_add(g[X], e2_mul(ev[8], lu2_F(ev, lam, lam2)));
                }
            e2_send(t, &pb, "lu2_round", g, 4);
            rho[r] = e2_squeeze(t, "lu2_chal");
            for (int i = 0; i < 9; i++)
                for (u64 b = 0; b < h; b++) V[i][b] = lu2_fold(V[i][b], V[i][h + b], rho[r]);
            Lr = h;
        }
        ext2 fin[8];
        for (int i = 0; i < 8; i++) fin[i] = V[i][0];
        e2_send(t, &pb, "lu2_final", fin, 8);
        ext2 mu = e2_squeeze(t, "lu2_mu");
        for (int r = 0; r < d; r++) z[r] = rho[r];
        z[d] = mu;
        for (int i = 0; i < 9; i++) free(V[i]);
        free(rho);
    }
    {
        u64* col = (u64*)malloc(L * sizeof(u64));
        ext2 leaf[3];
        for (u64 i = 0; i < L; i++) col[i] = orc_fint(K.fr[i]);
        leaf[0] = x16_mle(col, L, z, v);
        for (u64 i = 0; i < L; i++) col[i] = orc_fint(K.fq[i]);
        leaf[1] = x16_mle(col, L, z, v);
        for (u64 i = 0; i < L; i++) col[i] = orc_fint(K.fy[i]);
        leaf[2] = x16_mle(col, L, z, v);
        e2_send(t, &pb, "lu2_leaf", leaf, 3);
        free(col);
    }
    for (int tau = 0; tau < 2; tau++) {
        for (int d = 0; d <= v; d++) {
            free(P[tau][d]);
            free(Q[tau][d]);
        }
        free(P[tau]);
        free(Q[tau]);
    }
    free(z);
    free(mr);
    free(mc);
    keys_free(&K);
    *len = pb.len;
    return pb.overflow ? -2 : 0;
}

/* the table side sum_j m_j / (alpha - t_j) as one extension fraction */
static void lu2_table(const u32* m, u64 T, int tab, int k, ext2 alpha, ext2 gamma, ext2* num, ext2* den) {
    ext2 Pn = e2(0, 0), Qd = e2(1, 0);
    for (u64 j = 0; j < T; j++) {
        ext2 tj;
        if (tab == 0) {
            tj = e2(orc_fint((int64_t)j - ((int64_t)1 << (k - 1))), 0);
        } else {
            int64_t vj = (int64_t)j - 32768;
            int64_t cj = vj < -128 ? -128 : (vj > 127 ? 127 : vj);
            tj = e2_add(e2(orc_fint(vj), 0), e2_scal(gamma, orc_fint(cj)));
        }
        ext2 d = e2_sub(alpha, tj);
        Pn = e2_add(e2_mul(Pn, d), e2_scal(Qd, (u64)m[j]));
        Qd = e2_mul(Qd, d);
    }
    *num = Pn;
    *den = Qd;
}

int orc_lu2_verify(void* txh, const orc_site* sites, int ns, const orc_wit* wit, const uint8_t* proof, u64 len,
                   int64_t detail[2]) {
    detail[0] = detail[1] = 0;
    orc_tx* t = (orc_tx*)txh;
    orc_keys K;
    if (ns < 1 || keys_build(sites, ns, wit, &K) != 0) return REJ_ARGS;
    int rc = 0, v = K.v;
    u64 L = (u64)1 << v, Trem = (u64)1 << K.k;
    prd rd = {proof, len, 0, 0};
    u32* mr = (u32*)malloc(Trem * sizeof(u32));
    u32* mc = (u32*)malloc(65536 * sizeof(u32));
    ext2* z = (ext2*)malloc(sizeof(ext2) * (v + 1));
    ext2* rho = (ext2*)malloc(sizeof(ext2) * (v + 1));
    u64* col = NULL;
    lu2_absorb_site(t, &K);
    rd_mult(t, &rd, "lu2_m_rem", mr, Trem);
    ext2 gamma = e2_squeeze(t, "lu2_gamma");
    rd_mult(t, &rd, "lu2_m_clamp", mc, 65536);
    if (rd.bad) FAIL(REJ_FORMAT, 0, 0);
    ext2 alpha[2];
    alpha[0] = e2_squeeze(t, "lu2_alpha");
    alpha[1] = e2_squeeze(t, "lu2_alpha");
    ext2 l1[8];
    e2_read(t, &rd, "lu2_l1", l1, 8);
    if (rd.bad) FAIL(REJ_FORMAT, 1, 0);
    for (int tau = 0; tau < 2; tau++) {
        const ext2* x = l1 + 4 * tau;
        ext2 P0 = e2_add(e2_mul(x[0], x[3]), e2_mul(x[1], x[2])), Q0 = e2_mul(x[2], x[3]), PT, QT;
        lu2_table(tau == 0 ? mr : mc, tau == 0 ? Trem : 65536, tau, K.k, alpha[tau], gamma, &PT, &QT);
        if ((Q0.a == 0 && Q0.b == 0) || !e2_eqv(e2_mul(P0, QT), e2_mul(Q0, PT)))
            FAIL(tau == 0 ? REJ_ROOT_REM : REJ_ROOT_CLAMP, 0, 0);
    }
    ext2 mu = e2_squeeze(t, "lu2_mu"), cP[2], cQ[2];
    for (int tau = 0; tau < 2; tau++) {
        cP[tau] = lu2_fold(l1[4 * tau], l1[4 * tau + 1], mu);
        cQ[tau] = lu2_fold(l1[4 * tau + 2], l1[4 * tau + 3], mu);
    }
    z[0] = mu;
    for (int d = 1; d < v; d++) {
        ext2 lam = e2_squeeze(t, "lu2_lambda");
        ext2 lam2 = e2_mul(lam, lam), lam3 = e2_mul(lam2, lam);
        ext2 claim = e2_add(e2_add(cP[0], e2_mul(lam, cQ[0])), e2_add(e2_mul(lam2, cP[1]), e2_mul(lam3, cQ[1])));
        for (int r = 0; r < d; r++) {
            ext2 g[4];
            e2_read(t, &rd, "lu2_round", g, 4);
            if (rd.bad) FAIL(REJ_FORMAT, 2, d);
            if (!e2_eqv(e2_add(g[0], g[1]), claim)) FAIL(REJ_GKR_ROUND, d, r);
            rho[r] = e2_squeeze(t, "lu2_chal");
            claim = e2_lagrange4(g, rho[r]);
        }
        ext2 fin[8];
        e2_read(t, &rd, "lu2_final", fin, 8);
        if (rd.bad) FAIL(REJ_FORMAT, 3, d);
        if (!e2_eqv(e2_mul(e2_eq_closed(z, rho, d), lu2_F(fin, lam, lam2)), claim)) FAIL(REJ_GKR_FINAL, d, 0);
        mu = e2_squeeze(t, "lu2_mu");
        for (int tau = 0; tau < 2; tau++) {
            cP[tau] = lu2_fold(fin[4 * tau], fin[4 * tau + 1], mu);
            cQ[tau] = lu2_fold(fin[4 * tau + 2], fin[4 * tau + 3], mu);
        }
        for (int r = 0; r < d; r++) z[r] = rho[r];
        z[d] = mu;
    }
    {
        ext2 leaf[3];
        e2_read(t, &rd, "lu2_leaf", leaf, 3);
        if (rd.bad) FAIL(REJ_FORMAT, 4, 0);
        if (!e2_eqv(cP[0], e2(1, 0)) || !e2_eqv(cP[1], e2(1, 0))) FAIL(REJ_LEAF_P, 0, 0);
        if (!e2_eqv(cQ[0], e2_sub(alpha[0], leaf[0]))) FAIL(REJ_LEAF_Q, 0, 0);
        if (!e2_eqv(cQ[1], e2_sub(alpha[1], e2_add(leaf[1], e2_mul(gamma, leaf[2]))))) FAIL(REJ_LEAF_Q, 1, 0);
        col = (u64*)malloc(L * sizeof(u64));
        for (u64 i = 0; i < L; i++) col[i] = orc_fint(K.fr[i]);
        if (!e2_eqv(x16_mle(col, L, z, v), leaf[0])) FAIL(REJ_LEAF_OPEN, 0, 0);
        for (u64 i = 0; i < L; i++) col[i] = orc_fint(K.fq[i]);
        if (!e2_eqv(x16_mle(col, L, z, v), leaf[1])) FAIL(REJ_LEAF_OPEN, 1, 0);
        for (u64 i = 0; i < L; i++) col[i] = orc_fint(K.fy[i]);
        if (!e2_eqv(x16_mle(col, L, z, v), leaf[2])) FAIL(REJ_LEAF_OPEN, 2, 0);
    }
    if (rd.pos != rd.len) FAIL(REJ_FORMAT, -1, 0);
done:
    free(col);
    free(mr);
    free(mc);
    free(z);
    free(rho);
    keys_free(&K);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* The rescale lookups by helper inverses (next row f3: LogUp after Haboeck  */
/* 2022, "Towards Proving Frontier-Scale LLM Inference", The proof system,   */
/* set against the fraction tree of "How fast can FlashProve go", 4 Tighter  */
/* Rooflines). The lookup section of the layer proof with the same keys and  */
/* tables as the GKR form (remainder table R_k, clamp table C16), but with   */
/* the key side as two committed helper columns checked by one sum-check:    */
/*   m_rem (2^k u32, digest absorbed, "lhr_m_rem"); squeeze gamma            */
/*   ("lhr_gamma"); m_clamp (2^16 u32, "lhr_m_clamp"); squeeze alpha0 and    */
/*   alpha1 ("lhr_alpha"); commit h0_i = 1 / (alpha0 - r_i) and              */
/*   h1_i = 1 / (alpha1 - q_i - gamma y_i): absorb "lhr_h" D(h0) || D(h1)    */
/*   (u64 little-endian); squeeze z_1..z_v ("lhr_z") and beta ("lhr_beta");  */
/*   send S0 = sum h0, S1 = sum h1 ("lhr_sum");                              */
/*   sum-check over v variables of                                           */
/*     G = h0 + beta h1 + eq(z, .) (beta^2 (h0 (alpha0 - r) - 1)             */
/*                                  + beta^3 (h1 (alpha1 - q - gamma y) - 1)) */
/*   with claim S0 + beta S1: rounds g(0..3) ("lhr_round"), "lhr_chal";      */
/*   send h0, h1, r, q, y at rho ("lhr_final").                               */
/* The keys are the sites' outputs in storage order, padded to 2^v (v >= 1)  */
/* with the neutral key (r, q, y) = 0, which the multiplicities count. The   */
/* verifier checks S0 and S1 against the table fractions, every round, the  */
/* end against G at rho (eq(z, rho) in closed form), and the five final      */
/* values against the columns it recomputes (standing in for openings). The  */
/* zero-check terms force h0 (alpha0 - r) = 1 and h1 (alpha1 - q - gamma y)  */
/* = 1 on the whole cube (with high probability over z and beta), so S0 and  */
/* S1 are the key sides of the two LogUp identities. v rounds in all,        */
/* against the tree's v (v - 1) / 2, for two committed columns (16 bytes a   */
/* key).                                                                      */
/* ------------------------------------------------------------------------ */

enum {
    REJ_LHR_SUM = 41,    /* S0 or S1 != its table side (detail: the table) */
    REJ_LHR_ROUND = 42,  /* g(0) + g(1) != running claim */
    REJ_LHR_FINAL = 43,  /* the end does not match G at rho */
    REJ_LHR_OPEN = 44    /* a final value != its column's MLE at rho (detail: which) */
};

/* the five columns over the padded keys: r, q, y as field elements, h0, h1 */
static void lhr_columns(const orc_keys* K, u64 a0, u64 a1, u64 gamma, u64* R, u64* Q, u64* Y, u64* H0, u64* H1) {
    u64 L = (u64)1 << K->v;
    for (u64 i = 0; i < L; i++) {
        R[i] = orc_fint(K->fr[i]);
        Q[i] = orc_fint(K->fq[i]);
        Y[i] = orc_fint(K->fy[i]);
        H0[i] = orc_finv(orc_fsub(a0, R[i]));
        H1[i] = orc_finv(orc_fsub(a1, orc_fadd(Q[i], orc_fmul(gamma, Y[i]))));
    }
}

static void lhr_absorb_h(orc_tx* t, const u64* H0, const u64* H1, u64 L) {
    uint8_t* b = (uint8_t*)malloc(8 * L);
    uint8_t d[64];
    for (u64 i = 0; i < L; i++) put_le(b + 8 * i, H0[i], 8);
    orc_tree_digest(b, 8 * L, d);
    for (u64 i = 0; i < L; i++) put_le(b + 8 * i, H1[i], 8);
    orc_tree_digest(b, 8 * L, d + 32);
    free(b);
    orc_tx_absorb(t, "lhr_h", d, 64);
}

/* G at one point, from the five column values and the eq weight there */
static u64 lhr_G(const u64 c[5], u64 e, u64 a0, u64 a1, u64 gamma, u64 beta) {
    u64 b2 = orc_fmul(beta, beta), b3 = orc_fmul(b2, beta);
    u64 t0 = orc_fsub(orc_fmul(c[3], orc_fsub(a0, c[0])), 1);
    u64 t1 = orc_fsub(orc_fmul(c[4], orc_fsub(a1, orc_fadd(c[1], orc_fmul(gamma, c[2])))), 1);
    u64 zc = orc_fadd(orc_fmul(b2, t0), orc_fmul(b3, t1));
    return orc_fadd(orc_fadd(c[3], orc_fmul(beta, c[4])), orc_fmul(e, zc));
}

static void lhr_prove(orc_tx* t, pbuf* pb, const orc_site* sites, int ns, const orc_wit* wit) {
    orc_keys K;
    keys_build(sites, ns, wit, &K);
    int v = K.v;
    u64 L = (u64)1 << v, Trem = (u64)1 << K.k;
    u32* mr = (u32*)malloc(Trem * sizeof(u32));
    u32* mc = (u32*)malloc(65536 * sizeof(u32));
    mult_rem(&K, mr);
    send_mult(t, pb, "lhr_m_rem", mr, Trem);
    u64 gamma = orc_tx_squeeze(t, "lhr_gamma");
    mult_clamp(&K, mc);
    send_mult(t, pb, "lhr_m_clamp", mc, 65536);
    u64 a0 = orc_tx_squeeze(t, "lhr_alpha");
    u64 a1 = orc_tx_squeeze(t, "lhr_alpha");
    /* V[0..4] = r, q, y, h0, h1; V[5] = eq(z, .) */
    u64* V[6];
    for (int i = 0; i < 6; i++) V[i] = (u64*)malloc(L * sizeof(u64));
    lhr_columns(&K, a0, a1, gamma, V[0], V[1], V[2], V[3], V[4]);
    lhr_absorb_h(t, V[3], V[4], L);
    u64* z = (u64*)malloc(sizeof(u64) * v);
    for (int i = 0; i < v; i++) z[i] = orc_tx_squeeze(t, "lhr_z");
    u64 beta = orc_tx_squeeze(t, "lhr_beta");
    u64 S[2] = {0, 0};
    for (u64 i = 0; i < L; i++) {
        S[0] = orc_fadd(S[0], V[3][i]);
        S[1] = orc_fadd(S[1], V[4][i]);
    }
    send_fe(t, pb, "lhr_sum", S, 2);
    orc_eq_table(z, v, V[5]);
    u64 Lr = L;
    for (int rd = 0; rd < v; rd++) {
        u64 hh = Lr >> 1;
        u64 g[4] = {0, 0, 0, 0};
        for (u64 b = 0; b < hh; b++)
            for (u64 X = 0; X < 4; X++) {
                u64 c[6];
                for (int i = 0; i < 6; i++) c[i] = orc_fadd(V[i][b], orc_fmul(X, orc_fsub(V[i][hh + b], V[i][b])));
                g[X] = orc_fadd(g[X], lhr_G(c, c[5], a0, a1, gamma, beta));
            }
        send_fe(t, pb, "lhr_round", g, 4);
        u64 rho = orc_tx_squeeze(t, "lhr_chal");
        for (int i = 0; i < 6; i++)
            for (u64 b = 0; b < hh; b++) V[i][b] = orc_fadd(V[i][b], orc_fmul(rho, orc_fsub(V[i][hh + b], V[i][b])));
        Lr = hh;
    }
    u64 fin[5] = {V[3][0], V[4][0], V[0][0], V[1][0], V[2][0]};
    send_fe(t, pb, "lhr_final", fin, 5);
    for (int i = 0; i < 6; i++) free(V[i]);
    free(z);
    free(mr);
    free(mc);
    keys_free(&K);
}

static int lhr_verify(orc_tx* t, prd* rd, const orc_site* sites, int ns, const orc_wit* wit, int64_t* detail) {
    int rc = 0;
    orc_keys K;
    if (keys_build(sites, ns, wit, &K) != 0) {
        detail[0] = detail[1] = 0;
        return REJ_ARGS;
    }
    int v = K.v;
    u64 L = (u64)1 << v, Trem = (u64)1 << K.k;
    u32* mr = (u32*)malloc(Trem * sizeof(u32));
    u32* mc = (u32*)malloc(65536 * sizeof(u32));
    u64* z = (u64*)malloc(sizeof(u64) * (v + 1));
    u64* rho = (u64*)malloc(sizeof(u64) * (v + 1));
    u64* C[5];
    for (int i = 0; i < 5; i++) C[i] = (u64*)malloc(L * sizeof(u64));
    rd_mult(t, rd, "lhr_m_rem", mr, Trem);
    u64 gamma = orc_tx_squeeze(t, "lhr_gamma");
    rd_mult(t, rd, "lhr_m_clamp", mc, 65536);
    if (rd->bad) FAIL(REJ_FORMAT, 8, 0);
    u64 a0 = orc_tx_squeeze(t, "lhr_alpha");
    u64 a1 = orc_tx_squeeze(t, "lhr_alpha");
    lhr_columns(&K, a0, a1, gamma, C[0], C[1], C[2], C[3], C[4]); /* the verifier holds the keys, so h0, h1 too */
    lhr_absorb_h(t, C[3], C[4], L);
    for (int i = 0; i < v; i++) z[i] = orc_tx_squeeze(t, "lhr_z");
    u64 beta = orc_tx_squeeze(t, "lhr_beta");
    u64 S[2];
    rd_fe(t, rd, "lhr_sum", S, 2);
    if (rd->bad) FAIL(REJ_FORMAT, 9, 0);
    for (int tau = 0; tau < 2; tau++) {
        u64 PT, QT;
        table_fraction(tau == 0 ? mr : mc, tau == 0 ? Trem : 65536, tau, K.k, tau == 0 ? a0 : a1, gamma, &PT, &QT);
        if (orc_fmul(S[tau], QT) != PT) FAIL(REJ_LHR_SUM, tau, 0);
    }
    u64 claim = orc_fadd(S[0], orc_fmul(beta, S[1]));
    for (int i = 0; i < v; i++) {
        u64 g[4];
        rd_fe(t, rd, "lhr_round", g, 4);
        if (rd->bad) FAIL(REJ_FORMAT, 10, i);
        if (orc_fadd(g[0], g[1]) != claim) FAIL(REJ_LHR_ROUND, i, 0);
        rho[i] = orc_tx_squeeze(t, "lhr_chal");
        claim = orc_lagrange(g, 4, rho[i]);
    }
    u64 fin[5];
    rd_fe(t, rd, "lhr_final", fin, 5);
    if (rd->bad) FAIL(REJ_FORMAT, 11, 0);
    {
        /* G at rho from the final values h0, h1, r, q, y */
        u64 c[5] = {fin[2], fin[3], fin[4], fin[0], fin[1]};
        if (lhr_G(c, eq_closed(z, rho, v), a0, a1, gamma, beta) != claim) FAIL(REJ_LHR_FINAL, 0, 0);
    }
    {
        const int col[5] = {3, 4, 0, 1, 2}; /* final value i is column col[i]'s MLE */
        for (int i = 0; i < 5; i++)
            if (orc_mle_eval(C[col[i]], L, rho, v) != fin[i]) FAIL(REJ_LHR_OPEN, i, 0);
    }
done:
    for (int i = 0; i < 5; i++) free(C[i]);
    free(mr);
    free(mc);
    free(z);
    free(rho);
    keys_free(&K);
    return rc;
}

/* The layer proof with the helper-inverse lookup section: the commit and the
 * matmul section of orc_prove, then lhr_prove instead of the fraction tree.
 * Arguments and results as for orc_prove. */
int orc_prove_hi(u64 seed, const orc_site* sites, int ns, const orc_wit* wit, uint8_t* proof, u64 cap, u64* len,
                 uint8_t states[96], u64* sec_off) {
    if (ns < 1) return -1;
    for (int s = 0; s < ns; s++)
        if (sites[s].M < 1 || sites[s].N < 1 || sites[s].K < 1 || sites[s].k_shift < 1 ||
            sites[s].k_shift > 30 || (sites[s].w_bits != 4 && sites[s].w_bits != 8) ||
            sites[s].k_shift != sites[0].k_shift)
            return -1;
    orc_tx t;
    pbuf pb = {proof, cap, 0, 0};
    orc_tx_init(&t, seed);
    absorb_sites(&t, sites, ns, wit);
    memcpy(states, t.st, 32);
    mm_prove(&t, &pb, sites, ns, wit);
    memcpy(states + 32, t.st, 32);
    *sec_off = pb.len;
    lhr_prove(&t, &pb, sites, ns, wit);
    memcpy(states + 64, t.st, 32);
    *len = pb.len;
    return pb.overflow ? -2 : 0;
}

int orc_verify_hi(u64 seed, const orc_site* sites, int ns, const orc_wit* wit, const uint8_t* proof, u64 len,
                  int64_t detail[2]) {
    g_site_mask = NULL;
    g_verify_flags = 0;
    detail[0] = detail[1] = 0;
    if (ns < 1) return REJ_ARGS;
    for (int s = 0; s < ns; s++)
        if (sites[s].M < 1 || sites[s].N < 1 || sites[s].K < 1 || sites[s].k_shift < 1 ||
            sites[s].k_shift > 30 || sites[s].k_shift != sites[0].k_shift)
            return REJ_ARGS;
    orc_tx t;
    prd rd = {proof, len, 0, 0};
    orc_tx_init(&t, seed);
    absorb_sites(&t, sites, ns, wit);
    int rc = mm_verify(&t, &rd, sites, ns, wit, detail);
    if (rc) return rc;
    rc = lhr_verify(&t, &rd, sites, ns, wit, detail);
    if (rc) return rc;
    if (rd.pos != rd.len) return REJ_FORMAT;
    return 0;
}

/* ------------------------------------------------------------------------ */
/* MoE dispatch (next row f3: "prove the routing computation and the choice  */
/* of expert", How fast can FlashProve go, 2 Background, the note on MoE      */
/* layers; the routing proof covers the choice, this statement the moving of */
/* each token's activations to its expert). With T tokens, X the layer input */
/* (T x K int8, token-major), e_t the expert of token t (int32, < E) and D   */
/* the experts' inputs stacked expert by expert (T x K int8: the rows of X    */
/* routed to expert 0 in token order, then expert 1, ...), D = Pi X for the  */
/* permutation that sends token t to position                                */
/*   pos(t) = #{t' : e_t' < e_t} + #{t' < t : e_t' = e_t}.                   */
/* Row bits first, T and K zero-padded to 2^vT, 2^vK:                        */
/*   absorb "dsp_site" D(X) || D(e, int32 little-endian) || D(D);            */
/*   squeeze r_row (vT, "dsp_row") and r_col (vK, "dsp_col");               */
/*   send c = D~(r_row, r_col) ("dsp_claim");                                */
/*   sum-check over t of P(t) B(t), P(t) = eq(r_row, pos(t)) and              */
/*   B(t) = X~(t, r_col) (both 0 on padded t), degree 2: rounds g(0), g(1),  */
/*   g(2) ("dsp_round"), "dsp_chal"; send P(rho), B(rho) ("dsp_final").      */
/* Since D~(r, c) = sum_t eq(r, pos(t)) X~(t, c) exactly when D = Pi X (on   */
/* the cube, hence everywhere), the verifier checks c against D, the rounds, */
/* the end P(rho) B(rho), and P(rho) = sum_t eq(rho, t) eq(r_row, pos(t)),   */
/* B(rho) = X~(rho, r_col) from e and X (standing in for openings).          */
/* ------------------------------------------------------------------------ */

enum {
    REJ_DSP_CLAIM = 45,  /* c != D~(r_row, r_col) */
    REJ_DSP_ROUND = 46,  /* g(0) + g(1) != running claim */
    REJ_DSP_FINAL = 47,  /* the end != P(rho) B(rho) */
    REJ_DSP_OPEN = 48    /* P(rho) or B(rho) != its recomputation (detail: which) */
};

static void dsp_absorb_site(orc_tx* t, const int8_t* X, const int32_t* e, const int8_t* D, u64 T, u64 K) {
    uint8_t d[96];
    orc_tree_digest(X, T * K, d);
    uint8_t* b = (uint8_t*)calloc(4 * T + 1, 1);
    for (u64 i = 0; i < T; i++) put_le(b + 4 * i, (u64)(u32)e[i], 4);
    orc_tree_digest(b, 4 * T, d + 32);
    free(b);
    orc_tree_digest(D, T * K, d + 64);
    orc_tx_absorb(t, "dsp_site", d, 96);
}

/* pos(t) of every token; -1 if some e_t is outside [0, E) */
static int dsp_positions(const int32_t* e, u64 T, int E, u64* pos) {
    u64* before = (u64*)calloc((size_t)E + 1, sizeof(u64));
    for (u64 t = 0; t < T; t++) {
        if (e[t] < 0 || e[t] >= E) {
            free(before);
            return -1;
        }
        before[e[t] + 1]++;
    }
    for (int x = 0; x < E; x++) before[x + 1] += before[x];
    for (u64 t = 0; t < T; t++) pos[t] = before[e[t]]++;
    free(before);
    return 0;
}

/* P (eq(r_row, pos(t)) for t < T) and B (X~(t, r_col)) over 2^vT entries */
static void dsp_vectors(const int8_t* X, const u64* pos, u64 T, u64 K, const u64* rr, int vT, const u64* rc, int vK,
                        u64* P, u64* B) {
    u64 LT = (u64)1 << vT;
    u64* er = (u64*)malloc(sizeof(u64) * LT);
    u64* ec = (u64*)malloc(sizeof(u64) * ((u64)1 << vK));
    orc_eq_table(rr, vT, er);
    orc_eq_table(rc, vK, ec);
    for (u64 t = 0; t < LT; t++) {
        P[t] = 0;
        B[t] = 0;
        if (t >= T) continue;
        P[t] = er[pos[t]];
        for (u64 k = 0; k < K; k++) B[t] = orc_fadd(B[t], orc_fmul(ec[k], orc_fint(X[t * K + k])));
    }
    free(er);
    free(ec);
}

static u64 dsp_claim(const int8_t* D, u64 T, u64 K, const u64* rr, int vT, const u64* rc, int vK) {
    u64* er = (u64*)malloc(sizeof(u64) * ((u64)1 << vT));
    u64* ec = (u64*)malloc(sizeof(u64) * ((u64)1 << vK));
    orc_eq_table(rr, vT, er);
    orc_eq_table(rc, vK, ec);
    u64 c = 0;
    for (u64 p = 0; p < T; p++)
        for (u64 k = 0; k < K; k++) c = orc_fadd(c, orc_fmul(orc_fmul(er[p], ec[k]), orc_fint(D[p * K + k])));
    free(er);
    free(ec);
    return c;
}

int orc_dsp_prove(void* txh, const int8_t* X, const int32_t* e, const int8_t* D, u64 T, u64 K, int E, uint8_t* proof,
                  u64 cap, u64* len) {
    if (T < 1 || K < 1 || E < 1) return -1;
    orc_tx* t = (orc_tx*)txh;
    int vT = orc_log2_ceil(T), vK = orc_log2_ceil(K);
    u64 LT = (u64)1 << vT;
    u64* pos = (u64*)malloc(sizeof(u64) * T);
    if (dsp_positions(e, T, E, pos)) {
        free(pos);
        return -1;
    }
    pbuf pb = {proof, cap, 0, 0};
    dsp_absorb_site(t, X, e, D, T, K);
    u64* rr = (u64*)malloc(sizeof(u64) * (vT + 1));
    u64* rc = (u64*)malloc(sizeof(u64) * (vK + 1));
    for (int i = 0; i < vT; i++) rr[i] = orc_tx_squeeze(t, "dsp_row");
    for (int i = 0; i < vK; i++) rc[i] = orc_tx_squeeze(t, "dsp_col");
    u64 c = dsp_claim(D, T, K, rr, vT, rc, vK);
    send_fe(t, &pb, "dsp_claim", &c, 1);
    u64* P = (u64*)malloc(sizeof(u64) * LT);
    u64* B = (u64*)malloc(sizeof(u64) * LT);
    dsp_vectors(X, pos, T, K, rr, vT, rc, vK, P, B);
    u64 Lr = LT;
    for (int r = 0; r < vT; r++) {
        u64 h = Lr >> 1;
        u64 g[3] = {0, 0, 0};
        for (u64 b = 0; b < h; b++)
            for (u64 X_ = 0; X_ < 3; X_++) {
                u64 p = orc_fadd(P[b], orc_fmul(X_, orc_fsub(P[h + b], P[b])));
                u64 q = orc_fadd(B[b], orc_fmul(X_, orc_fsub(B[h + b], B[b])));
                g[X_] = orc_fadd(g[X_], orc_fmul(p, q));
            }
        send_fe(t, &pb, "dsp_round", g, 3);
        u64 rho = orc_tx_squeeze(t, "dsp_chal");
        for (u64 b = 0; b < h; b++) {
            P[b] = orc_fadd(P[b], orc_fmul(rho, orc_fsub(P[h + b], P[b])));
            B[b] = orc_fadd(B[b], orc_fmul(rho, orc_fsub(B[h + b], B[b])));
        }
        Lr = h;
    }
    u64 fin[2] = {P[0], B[0]};
    send_fe(t, &pb, "dsp_final", fin, 2);
    free(pos);
    free(rr);
    free(rc);
    free(P);
    free(B);
    *len = pb.len;
    return pb.overflow ? -2 : 0;
}

int orc_dsp_verify(void* txh, const int8_t* X, const int32_t* e, const int8_t* D, u64 T, u64 K, int E,
                   const uint8_t* proof, u64 len, int64_t detail[2]) {
    detail[0] = detail[1] = 0;
    if (T < 1 || K < 1 || E < 1) return REJ_ARGS;
    orc_tx* t = (orc_tx*)txh;
    int vT = orc_log2_ceil(T), vK = orc_log2_ceil(K);
    u64 LT = (u64)1 << vT;
    u64* pos = (u64*)malloc(sizeof(u64) * T);
    u64* rr = (u64*)malloc(sizeof(u64) * (vT + 1));
    u64* rcol = (u64*)malloc(sizeof(u64) * (vK + 1));
    u64* rho = (u64*)malloc(sizeof(u64) * (vT + 1));
    u64* P = (u64*)malloc(sizeof(u64) * LT);
    u64* B = (u64*)malloc(sizeof(u64) * LT);
    int rc = 0;
    prd rdd = {proof, len, 0, 0};
    prd* rd = &rdd;
    if (dsp_positions(e, T, E, pos)) FAIL(REJ_ARGS, 0, 0);
    dsp_absorb_site(t, X, e, D, T, K);
    for (int i = 0; i < vT; i++) rr[i] = orc_tx_squeeze(t, "dsp_row");
    for (int i = 0; i < vK; i++) rcol[i] = orc_tx_squeeze(t, "dsp_col");
    u64 c;
    rd_fe(t, rd, "dsp_claim", &c, 1);
    if (rd->bad) FAIL(REJ_FORMAT, 12, 0);
    if (c != dsp_claim(D, T, K, rr, vT, rcol, vK)) FAIL(REJ_DSP_CLAIM, 0, 0);
    u64 claim = c;
    for (int i = 0; i < vT; i++) {
        u64 g[3];
        rd_fe(t, rd, "dsp_round", g, 3);
        if (rd->bad) FAIL(REJ_FORMAT, 13, i);
        if (orc_fadd(g[0], g[1]) != claim) FAIL(REJ_DSP_ROUND, i, 0);
        rho[i] = orc_tx_squeeze(t, "dsp_chal");
        claim = orc_lagrange(g, 3, rho[i]);
    }
    u64 fin[2];
    rd_fe(t, rd, "dsp_final", fin, 2);
    if (rd->bad) FAIL(REJ_FORMAT, 14, 0);
    if (orc_fmul(fin[0], fin[1]) != claim) FAIL(REJ_DSP_FINAL, 0, 0);
    dsp_vectors(X, pos, T, K, rr, vT, rcol, vK, P, B);
    if (orc_mle_eval(P, LT, rho, vT) != fin[0]) FAIL(REJ_DSP_OPEN, 0, 0);
    if (orc_mle_eval(B, LT, rho, vT) != fin[1]) FAIL(REJ_DSP_OPEN, 1, 0);
    if (rd->pos != rd->len) FAIL(REJ_FORMAT, -1, 0);
done:
    free(pos);
    free(rr);
    free(rcol);
    free(rho);
    free(P);
    free(B);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* The FFN layer statement ("How fast can FlashProve go", 3.1: the weights'  */
/* group scales, the SiLU by lookup, the gated product by sum-check): the    */
/* layer proof of orc_prove over the gate, up and down sites, continued on    */
/* the same transcript by                                                    */
/*  - the per-group scale reduction of every site with scales, at the point  */
/*    where the matmul section left W_eff: (r_row's first vM_s coordinates,   */
/*    the last vK_s round challenges); the matmul's A_s(rho) is that value    */
/*    times prod_{j < n - vK_s} (1 - rho_j), since the padded columns of a    */
/*    narrower site are zero;                                                 */
/*  - the hidden activations: h = s u (s the SiLU outputs, u the up          */
/*    projection's outputs) is 16-bit while the down projection reads 8-bit   */
/*    activations, so h is rescaled as a matmul output is (3.1's rescale):    */
/*    q_h = floor((h + 2^(kh-1)) / 2^kh), r_h = h - 2^kh q_h,                 */
/*    y_h = clamp(q_h, -128, 127), and y_h is the down site's X. The          */
/*    statement absorbs "ffn_hidden" D(q_h) || D(r_h) || D(y_h) and runs a    */
/*    second lookup section (the layer proof's, over the keys (r_h, q_h, y_h) */
/*    with remainder table R_kh) proving r_h in R_kh and y_h = clamp(q_h);    */
/*  - the SiLU lookup with g the gate projection's committed outputs y (as    */
/*    16-bit inputs) and s its committed 16-bit outputs;                      */
/*  - the gated product of s (as 8-bit values: SiLU of an 8-bit input lies in */
/*    [-48, 79]) with the up projection's committed outputs, whose claim      */
/*    c = h~(z) the verifier ties to the committed rescale:                   */
/*    c = 2^kh q_h~(z) + r_h~(z). With r_h in R_kh this fixes q_h as the      */
/*    rounded quotient of h, so the down projection's input is the layer's    */
/*    own hidden activation.                                                  */
/* ------------------------------------------------------------------------ */

enum {
    REJ_FFN_LINK = 49,   /* a scale reduction's claim is not the weight value the matmul section left (detail: site) */
    REJ_FFN_HIDDEN = 50, /* the gated product's claim is not 2^kh q_h~(z) + r_h~(z) */
    REJ_FFN_DOWN = 51    /* the down site's committed X is not y_h */
};

static int ffn_args_ok(const orc_site* sites, int ns, int ig, int iu, int idn, int kh) {
    if (ig < 0 || iu < 0 || idn < 0 || ig >= ns || iu >= ns || idn >= ns) return 0;
    if (ig == iu || idn == ig || idn == iu || kh < 1 || kh > 16) return 0;
    return sites[ig].M == sites[iu].M && sites[ig].N == sites[iu].N && sites[idn].K == sites[ig].M &&
           sites[idn].N == sites[ig].N;
}

/* The rescaled hidden activations of n products s_i u_i, by the rounding every site's
 * witness uses. Returns 0, or -1 if kh is outside [1, 16]. */
int orc_ffn_hidden(const int8_t* s, const int8_t* u, u64 n, int kh, int32_t* q, int32_t* r, int8_t* y) {
    if (kh < 1 || kh > 16) return -1;
    for (u64 i = 0; i < n; i++) {
        const int64_t h = (int64_t)s[i] * (int64_t)u[i];
        const int64_t qq = floordiv_pow2(h + ((int64_t)1 << (kh - 1)), kh);
        q[i] = (int32_t)qq;
        r[i] = (int32_t)(h - qq * ((int64_t)1 << kh));
        y[i] = (int8_t)(qq < -128 ? -128 : (qq > 127 ? 127 : qq));
    }
    return 0;
}

/* the scale reduction's point for site s and the factor prod_{j < n - vK} (1 - rho_j) */
static u64 ffn_scl_point(const orc_site* st, u64* z) {
    const int vM = orc_log2_ceil((u64)st->M), vK = orc_log2_ceil((u64)st->K), n = g_mm_pt.n;
    for (int i = 0; i < vM; i++) z[i] = g_mm_pt.rr[i];
    for (int i = 0; i < vK; i++) z[vM + i] = g_mm_pt.rho[n - vK + i];
    u64 f = 1;
    for (int j = 0; j < n - vK; j++) f = orc_fmul(f, orc_fsub(1, g_mm_pt.rho[j]));
    return f;
}

/* s (16-bit SiLU outputs) as the gated product's 8-bit factor; 0 if a value does not fit */
static int8_t* ffn_s8(const int16_t* s, u64 n) {
    int8_t* o = (int8_t*)malloc(n ? n : 1);
    for (u64 i = 0; i < n; i++) {
        if (s[i] < -128 || s[i] > 127) {
            free(o);
            return NULL;
        }
        o[i] = (int8_t)s[i];
    }
    return o;
}

static int16_t* ffn_g16(const int8_t* y, u64 n) {
    int16_t* g = (int16_t*)malloc(sizeof(int16_t) * (n ? n : 1));
    for (u64 i = 0; i < n; i++) g[i] = y[i];
    return g;
}

static void ffn_absorb_hidden(orc_tx* t, const int32_t* qh, const int32_t* rh, const int8_t* yh, u64 n) {
    uint8_t d[96];
    orc_tree_digest(qh, 4 * n, d);
    orc_tree_digest(rh, 4 * n, d + 32);
    orc_tree_digest(yh, n, d + 64);
    orc_tx_absorb(t, "ffn_hidden", d, 96);
}

/* the hidden activations as a lookup section's single site: M x N keys, remainder table R_kh */
static void ffn_hidden_site(const orc_site* gate, int kh, const int32_t* qh, const int32_t* rh, const int8_t* yh,
                            orc_site* ps, orc_wit* pw) {
    memset(ps, 0, sizeof *ps);
    ps->M = gate->M;
    ps->N = gate->N;
    ps->K = 1;
    ps->w_bits = 8;
    ps->k_shift = kh;
    pw->q = (int32_t*)qh;
    pw->r = (int32_t*)rh;
    pw->y = (int8_t*)yh;
}

static int ffn_sites_ok(const orc_site* sites, int ns) {
    for (int s = 0; s < ns; s++)
        if (sites[s].M < 1 || sites[s].N < 1 || sites[s].K < 1 || sites[s].k_shift < 1 ||
            sites[s].k_shift > 30 || (sites[s].w_bits != 4 && sites[s].w_bits != 8) ||
            sites[s].k_shift != sites[0].k_shift)
            return 0;
    return 1;
}

/* Prover. s16: the committed SiLU outputs (gate's M x N entries, token-major like y); qh, rh,
 * yh: the committed rescale of the hidden activations (same layout), rescaled by 2^kh; the
 * down site sites[idn] reads yh as its X. Returns 0, -1 on bad input (including an s that
 * does not fit 8 bits), -2 if the buffer is too small (*len then holds the size needed);
 * state: the transcript after the statement. */
int orc_prove_ffn(u64 seed, const orc_site* sites, int ns, const orc_wit* wit, int ig, int iu, int idn, int kh,
                  const int16_t* s16, const int32_t* qh, const int32_t* rh, const int8_t* yh, uint8_t* proof, u64 cap,
                  u64* len, uint8_t state[32]) {
    if (ns < 1 || !ffn_args_ok(sites, ns, ig, iu, idn, kh) || !ffn_sites_ok(sites, ns)) return -1;
    const u64 n = (u64)sites[ig].M * (u64)sites[ig].N;
    int8_t* s8 = ffn_s8(s16, n);
    if (!s8) return -1;
    orc_tx t;
    pbuf pb = {proof, cap, 0, 0};
    orc_tx_init(&t, seed);
    absorb_sites(&t, sites, ns, wit);
    mm_prove(&t, &pb, sites, ns, wit);
    lu_prove(&t, &pb, sites, ns, wit);
    int rc = 0;
    /* each chained statement writes at the end of the proof so far (a size query once full) */
#define FFN_SUB(call)                                                                  \
    do {                                                                               \
        u64 l_ = 0;                                                                    \
        uint8_t* at_ = pb.overflow ? NULL : pb.p + pb.len;                            \
        u64 room_ = pb.overflow ? 0 : pb.cap - pb.len;                                \
        rc = call;                                                                     \
        if (rc == -2) {                                                                \
            pb.overflow = 1;                                                           \
            rc = 0;                                                                    \
        } else if (rc) {                                                               \
            goto out;                                                                  \
        }                                                                              \
        pb.len += l_;                                                                  \
    } while (0)
    for (int s = 0; s < ns; s++) {
        if (!sites[s].scales) continue;
        u64 z[MM_PT_MAX];
        (void)ffn_scl_point(&sites[s], z);
        FFN_SUB(orc_scl_prove(&t, sites[s].w, sites[s].w_bits, sites[s].scales, sites[s].M, sites[s].K, z, at_, room_,
                              &l_));
    }
    {
        orc_site ps;
        orc_wit pw;
        ffn_hidden_site(&sites[ig], kh, qh, rh, yh, &ps, &pw);
        ffn_absorb_hidden(&t, qh, rh, yh, n);
        lu_prove(&t, &pb, &ps, 1, &pw);
    }
    {
        int16_t* g16 = ffn_g16(wit[ig].y, n);
        FFN_SUB(orc_silu_prove(&t, g16, s16, n, at_, room_, &l_));
        free(g16);
    }
    FFN_SUB(orc_had_prove(&t, s8, wit[iu].y, n, at_, room_, &l_));
#undef FFN_SUB
    memcpy(state, t.st, 32);
    *len = pb.len;
    rc = pb.overflow ? -2 : 0;
out:
    free(s8);
    return rc;
}

/* Verifier of orc_prove_ffn's statement: the layer proof as orc_verify, then each chained
 * statement, with the scale reductions' claims tied to the matmul section's final values,
 * the down site's X to y_h and the gated product's claim to the committed rescale.
 * Returns 0 on accept or a reason code (the sub-statements' own codes for their failures). */
int orc_verify_ffn(u64 seed, const orc_site* sites, int ns, const orc_wit* wit, int ig, int iu, int idn, int kh,
                   const int16_t* s16, const int32_t* qh, const int32_t* rh, const int8_t* yh, const uint8_t* proof,
                   u64 len, int64_t detail[2]) {
    detail[0] = detail[1] = 0;
    g_site_mask = NULL;
    g_verify_flags = 0;
    if (ns < 1 || !ffn_args_ok(sites, ns, ig, iu, idn, kh) || !ffn_sites_ok(sites, ns)) return REJ_ARGS;
    const u64 n = (u64)sites[ig].M * (u64)sites[ig].N;
    int8_t* s8 = ffn_s8(s16, n);
    if (!s8) return REJ_ARGS;
    orc_tx t;
    prd rd = {proof, len, 0, 0};
    orc_tx_init(&t, seed);
    absorb_sites(&t, sites, ns, wit);
    int rc = mm_verify(&t, &rd, sites, ns, wit, detail);
    if (!rc) rc = lu_verify(&t, &rd, sites, ns, wit, detail);
    u64 pos = rd.pos;
    for (int s = 0; s < ns && !rc; s++) {
        if (!sites[s].scales) continue;
        const int v = orc_log2_ceil((u64)sites[s].M) + orc_log2_ceil((u64)sites[s].K);
        const u64 ls = 8 + 32 * (u64)v + 16;
        if (pos + ls > len) {
            rc = REJ_FORMAT;
            break;
        }
        u64 z[MM_PT_MAX];
        const u64 f = ffn_scl_point(&sites[s], z);
        if (orc_fmul(f, get_le(proof + pos, 8)) != g_mm_pt.fin[2 * s]) {
            rc = REJ_FFN_LINK;
            detail[0] = s;
            break;
        }
        rc = orc_scl_verify(&t, sites[s].w, sites[s].w_bits, sites[s].scales, sites[s].M, sites[s].K, z, proof + pos,
                            ls, detail);
        pos += ls;
    }
    if (!rc) {
        /* one committed tensor: the down site's X is the y_h the statement rescales */
        uint8_t dx[32], dy[32];
        orc_tree_digest(sites[idn].xt, n, dx);
        orc_tree_digest(yh, n, dy);
        if (memcmp(dx, dy, 32)) rc = REJ_FFN_DOWN;
    }
    if (!rc) {
        orc_site ps;
        orc_wit pw;
        ffn_hidden_site(&sites[ig], kh, qh, rh, yh, &ps, &pw);
        ffn_absorb_hidden(&t, qh, rh, yh, n);
        prd rh_rd = {proof, len, pos, 0};
        rc = lu_verify(&t, &rh_rd, &ps, 1, &pw, detail);
        pos = rh_rd.pos;
    }
    if (!rc) {
        const int vh = orc_log2_ceil(n);
        const u64 lh = 8 + 32 * (u64)vh + 16;
        if (pos + lh > len) {
            rc = REJ_FORMAT;
        } else {
            const u64 lsilu = len - pos - lh;
            int16_t* g16 = ffn_g16(wit[ig].y, n);
            rc = orc_silu_verify(&t, g16, s16, n, proof + pos, lsilu, detail);
            free(g16);
            if (!rc) rc = orc_had_verify(&t, s8, wit[iu].y, n, proof + pos + lsilu, lh, detail);
        }
        if (!rc) {
            /* c = 2^kh q_h~(z) + r_h~(z) at the gated product's point */
            const u64 sz = (u64)1 << vh;
            u64* Q = (u64*)calloc(sz, sizeof(u64));
            u64* R = (u64*)calloc(sz, sizeof(u64));
            for (u64 i = 0; i < n; i++) {
                Q[i] = orc_fint(qh[i]);
                R[i] = orc_fint(rh[i]);
            }
            const u64 want = orc_fadd(orc_fmul(orc_fint((int64_t)1 << kh), orc_mle_eval(Q, sz, g_had_pt.z, vh)),
                                      orc_mle_eval(R, sz, g_had_pt.z, vh));
            free(Q);
            free(R);
            if (want != g_had_pt.c) rc = REJ_FFN_HIDDEN;
        }
    }
    free(s8);
    return rc;
}
