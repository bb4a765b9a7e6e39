// Host Fiat-Shamir transcript ("How fast can FlashProve go", 2 Background:
// every challenge hashes everything sent so far), SHA-256 based:
//   absorb:  state = SHA256(state || u32le(|label|) || label || u64le(n) || data)
//   squeeze: h = SHA256(state || "sq" || u32le(|label|) || label || u32le(ctr)),
//            the first h (ctr = 0, 1, ...) whose low 8 bytes are < p is kept.
#include <cpuid.h>
#include <immintrin.h>
#include <stdlib.h>
#include <string.h>

#include "fp_internal.h"

// ---- host SHA-256 compression ------------------------------------------------

static void sha_blocks_portable(uint32_t h[8], const uint8_t* p, size_t n) {
    for (; n; n--, p += 64) {
        uint32_t m[16];
        for (int i = 0; i < 16; i++)
            m[i] = ((uint32_t)p[4 * i] << 24) | ((uint32_t)p[4 * i + 1] << 16) | ((uint32_t)p[4 * i + 2] << 8) |
                   (uint32_t)p[4 * i + 3];
        fp_sha_compress(h, m);
    }
}

// SHA-256 with the x86 SHA extensions: sha256rnds2 runs two rounds on the
// state split as {A,B,E,F} / {C,D,G,H}; sha256msg1 / sha256msg2 extend the
// message schedule four words at a time.
__attribute__((target("sha,sse4.1,ssse3"))) static void sha_blocks_shani(uint32_t h[8], const uint8_t* p, size_t n) {
    const __m128i bswap = _mm_set_epi64x(0x0c0d0e0f08090a0bULL, 0x0405060700010203ULL);
    __m128i t = _mm_loadu_si128((const __m128i*)&h[0]);   // D C B A (high to low)
    __m128i s1 = _mm_loadu_si128((const __m128i*)&h[4]);  // H G F E
    t = _mm_shuffle_epi32(t, 0xB1);                       // C D A B
    s1 = _mm_shuffle_epi32(s1, 0x1B);                     // E F G H
    __m128i s0 = _mm_alignr_epi8(t, s1, 8);               // A B E F
    s1 = _mm_blend_epi16(s1, t, 0xF0);                    // C D G H
    for (; n; n--, p += 64) {
        const __m128i save0 = s0, save1 = s1;
        __m128i w[4];
        for (int i = 0; i < 4; i++) w[i] = _mm_shuffle_epi8(_mm_loadu_si128((const __m128i*)(p + 16 * i)), bswap);
        for (int i = 0; i < 16; i++) {
            __m128i msg = _mm_add_epi32(w[i & 3], _mm_loadu_si128((const __m128i*)&kFpShaKHost[4 * i]));
            s1 = _mm_sha256rnds2_epu32(s1, s0, msg);
            msg = _mm_shuffle_epi32(msg, 0x0E);
            s0 = _mm_sha256rnds2_epu32(s0, s1, msg);
            if (i < 12) {
                __m128i x = _mm_sha256msg1_epu32(w[i & 3], w[(i + 1) & 3]);
                x = _mm_add_epi32(x, _mm_alignr_epi8(w[(i + 3) & 3], w[(i + 2) & 3], 4));
                w[i & 3] = _mm_sha256msg2_epu32(x, w[(i + 3) & 3]);
            }
        }
        s0 = _mm_add_epi32(s0, save0);
        s1 = _mm_add_epi32(s1, save1);
    }
    t = _mm_shuffle_epi32(s0, 0x1B);          // F E B A
    s1 = _mm_shuffle_epi32(s1, 0xB1);         // D C H G
    s0 = _mm_blend_epi16(t, s1, 0xF0);        // D C B A
    s1 = _mm_alignr_epi8(s1, t, 8);           // H G F E
    _mm_storeu_si128((__m128i*)&h[0], s0);
    _mm_storeu_si128((__m128i*)&h[4], s1);
}

static bool cpu_has_sha() {
    const char* off = getenv("FP_NO_SHANI");  // forces the portable path (tests)
    if (off && off[0] == '1') return false;
    unsigned a, b, c, d;
    if (!__get_cpuid(1, &a, &b, &c, &d)) return false;
    const bool ssse3 = c & (1u << 9), sse41 = c & (1u << 19);
    if (!__get_cpuid_count(7, 0, &a, &b, &c, &d)) return false;
    return ssse3 && sse41 && (b & (1u << 29));
}

void fp_sha256_host_blocks(uint32_t h[8], const uint8_t* p, size_t n) {
    static const bool shani = cpu_has_sha();
    if (shani)
        sha_blocks_shani(h, p, n);
    else
        sha_blocks_portable(h, p, n);
}

static void put_le(uint8_t* p, uint64_t v, int n) {
    for (int i = 0; i < n; i++) p[i] = (uint8_t)(v >> (8 * i));
}

void fp_tx_absorb_raw(fp_tx* t, const char* label, const void* data, uint64_t n) {
    uint32_t ll = (uint32_t)strlen(label);
    uint8_t l4[4], l8[8];
    put_le(l4, ll, 4);
    put_le(l8, n, 8);
    FpSha256 h;
    h.update(t->st, 32);
    h.update(l4, 4);
    h.update(label, ll);
    h.update(l8, 8);
    if (n) h.update(data, n);
    h.final(t->st);
}

uint64_t fp_tx_squeeze_one(fp_tx* t, const char* label) {
    uint32_t ll = (uint32_t)strlen(label);
    uint8_t l4[4];
    put_le(l4, ll, 4);
    for (uint32_t ctr = 0;; ctr++) {
        uint8_t c4[4], out[32];
        put_le(c4, ctr, 4);
        FpSha256 h;
        h.update(t->st, 32);
        h.update("sq", 2);
        h.update(l4, 4);
        h.update(label, ll);
        h.update(c4, 4);
        h.final(out);
        uint64_t v = 0;
        for (int i = 0; i < 8; i++) v |= (uint64_t)out[i] << (8 * i);
        if (v < 0xFFFFFFFF00000001ull) {
            memcpy(t->st, out, 32);
            return v;
        }
    }
}
