// SHA-256 (FIPS 180-4, sections 4.1.2, 4.2.2, 5.3.3, 6.2.2) for host and device.
//
// One compression function serves the host transcript and the device digest
// kernels. Message words are big-endian; device callers byte-swap 32-bit loads.
#pragma once
#include <stdint.h>
#include <string.h>

#define FP_SHA_K_LIST                                                                          \
    0x428a2f98u, 0x71374491u, 0xb5c0fbcfu, 0xe9b5dba5u, 0x3956c25bu, 0x59f111f1u, 0x923f82a4u, \
        0xab1c5ed5u, 0xd807aa98u, 0x12835b01u, 0x243185beu, 0x550c7dc3u, 0x72be5d74u,          \
        0x80deb1feu, 0x9bdc06a7u, 0xc19bf174u, 0xe49b69c1u, 0xefbe4786u, 0x0fc19dc6u,          \
        0x240ca1ccu, 0x2de92c6fu, 0x4a7484aau, 0x5cb0a9dcu, 0x76f988dau, 0x983e5152u,          \
        0xa831c66du, 0xb00327c8u, 0xbf597fc7u, 0xc6e00bf3u, 0xd5a79147u, 0x06ca6351u,          \
        0x14292967u, 0x27b70a85u, 0x2e1b2138u, 0x4d2c6dfcu, 0x53380d13u, 0x650a7354u,          \
        0x766a0abbu, 0x81c2c92eu, 0x92722c85u, 0xa2bfe8a1u, 0xa81a664bu, 0xc24b8b70u,          \
        0xc76c51a3u, 0xd192e819u, 0xd6990624u, 0xf40e3585u, 0x106aa070u, 0x19a4c116u,          \
        0x1e376c08u, 0x2748774cu, 0x34b0bcb5u, 0x391c0cb3u, 0x4ed8aa4au, 0x5b9cca4fu,          \
        0x682e6ff3u, 0x748f82eeu, 0x78a5636fu, 0x84c87814u, 0x8cc70208u, 0x90befffau,          \
        0xa4506cebu, 0xbef9a3f7u, 0xc67178f2u

#define FP_SHA_H0_LIST \
    0x6a09e667u, 0xbb67ae85u, 0x3c6ef372u, 0xa54ff53au, 0x510e527fu, 0x9b05688cu, 0x1f83d9abu, 0x5be0cd19u

__host__ __device__ __forceinline__ uint32_t fp_rotr(uint32_t x, int n) { return (x >> n) | (x << (32 - n)); }

#ifdef __CUDACC__
static __constant__ uint32_t kFpShaKDev[64] = {FP_SHA_K_LIST};
#endif
static const uint32_t kFpShaKHost[64] = {FP_SHA_K_LIST};

// One compression of the 16 big-endian words m into the state h.
__host__ __device__ __forceinline__ void fp_sha_compress(uint32_t h[8], const uint32_t m[16]) {
#ifdef __CUDA_ARCH__
    const uint32_t* K = kFpShaKDev;
#else
    const uint32_t* K = kFpShaKHost;
#endif
    uint32_t w[16];
#pragma unroll
    for (int t = 0; t < 16; t++) w[t] = m[t];
    uint32_t a = h[0], b = h[1], c = h[2], d = h[3], e = h[4], f = h[5], g = h[6], hh = h[7];
#pragma unroll
    for (int t = 0; t < 64; t++) {
        uint32_t wt;
        if (t < 16) {
            wt = w[t];
        } else {
            // message schedule kept in a 16-word ring
            uint32_t w15 = w[(t + 1) & 15], w2 = w[(t + 14) & 15];
            uint32_t s0 = fp_rotr(w15, 7) ^ fp_rotr(w15, 18) ^ (w15 >> 3);
            uint32_t s1 = fp_rotr(w2, 17) ^ fp_rotr(w2, 19) ^ (w2 >> 10);
            wt = w[t & 15] + s0 + w[(t + 9) & 15] + s1;
            w[t & 15] = wt;
        }
        uint32_t S1 = fp_rotr(e, 6) ^ fp_rotr(e, 11) ^ fp_rotr(e, 25);
        uint32_t ch = (e & f) ^ (~e & g);
        uint32_t T1 = hh + S1 + ch + K[t] + wt;
        uint32_t S0 = fp_rotr(a, 2) ^ fp_rotr(a, 13) ^ fp_rotr(a, 22);
        uint32_t mj = (a & b) ^ (a & c) ^ (b & c);
        hh = g;
        g = f;
        f = e;
        e = d + T1;
        d = c;
        c = b;
        b = a;
        a = T1 + mj + S0;
    }
    h[0] += a; h[1] += b; h[2] += c; h[3] += d;
    h[4] += e; h[5] += f; h[6] += g; h[7] += hh;
}

__host__ __device__ __forceinline__ void fp_sha_init(uint32_t h[8]) {
    const uint32_t h0[8] = {FP_SHA_H0_LIST};
#pragma unroll
    for (int i = 0; i < 8; i++) h[i] = h0[i];
}

// Host compression of n 64-byte blocks; uses the CPU's SHA extensions when it
// has them (defined in transcript.cu).
void fp_sha256_host_blocks(uint32_t h[8], const uint8_t* p, size_t n);

// Host-side incremental hasher (transcript and small host digests).
struct FpSha256 {
    uint32_t h[8];
    uint8_t buf[64];
    uint64_t total = 0;
    uint32_t fill = 0;

    FpSha256() { fp_sha_init(h); }

    void block(const uint8_t* p) { fp_sha256_host_blocks(h, p, 1); }

    void update(const void* data, uint64_t n) {
        const uint8_t* p = (const uint8_t*)data;
        total += n;
        if (fill) {
            uint32_t take = 64 - fill;
            if (take > n) take = (uint32_t)n;
            memcpy(buf + fill, p, take);
            fill += take;
            p += take;
            n -= take;
            if (fill == 64) {
                block(buf);
                fill = 0;
            }
        }
        if (n >= 64) {
            const size_t nb = n / 64;
            fp_sha256_host_blocks(h, p, nb);
            p += 64 * nb;
            n -= 64 * nb;
        }
        if (n) {
            memcpy(buf, p, n);
            fill = (uint32_t)n;
        }
    }

    void final(uint8_t out[32]) {
        uint64_t bits = total * 8u;
        uint8_t pad[72];
        uint32_t padlen = (fill < 56) ? (56 - fill) : (120 - fill);
        memset(pad, 0, sizeof pad);
        pad[0] = 0x80;
        for (int i = 0; i < 8; i++) pad[padlen + i] = (uint8_t)(bits >> (56 - 8 * i));
        update(pad, padlen + 8);
        for (int i = 0; i < 8; i++) {
            out[4 * i] = (uint8_t)(h[i] >> 24);
            out[4 * i + 1] = (uint8_t)(h[i] >> 16);
            out[4 * i + 2] = (uint8_t)(h[i] >> 8);
            out[4 * i + 3] = (uint8_t)h[i];
        }
    }
};
