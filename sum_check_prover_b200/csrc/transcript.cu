// Host Fiat-Shamir transcript ("How fast can FlashProve go", 2 Background:
// every challenge hashes everything sent so far), SHA-256 based:
//   absorb:  state = SHA256(state || u32le(|label|) || label || u64le(n) || data)
//   squeeze: h = SHA256(state || "sq" || u32le(|label|) || label || u32le(ctr)),
//            the first h (ctr = 0, 1, ...) whose low 8 bytes are < p is kept.
#include <string.h>

#include "fp_internal.h"

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
