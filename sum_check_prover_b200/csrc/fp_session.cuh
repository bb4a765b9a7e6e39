// Host <-> device handshake for persistent sum-check kernels.
//
// The transcript lives on the host ("How fast can FlashProve go", 2 Background:
// every challenge is a hash of all the prover sent), so each sum-check round
// needs one exchange: the device publishes the round's values, the host hashes
// them and answers with the challenge. A persistent kernel keeps many rounds in
// one launch; the exchange goes through a mailbox in mapped pinned host memory:
//   device -> host: res[0..n): the host fills these slots with kEmpty (no field
//   element is >= p) before it posts a challenge, and takes the result once all
//   n slots hold field elements; each slot is one atomic 8-byte write, so the
//   device needs no fence or sequence number on this path;
//   host -> device: chal2, then {chal, chal_seq} as one aligned 16-byte store,
//   which the device reads with one 16-byte load (one PCIe read, never torn).
// Only block 0 (thread 0) reads host memory; it forwards the challenge to the
// other blocks through a device-memory relay (FpRelay). Every wait is bounded:
// after a limit of polls the kernel records an error code in the mailbox and
// the relay, and returns; the host sees the code and reports FP_ERR_TIMEOUT.
#pragma once
#include <stdint.h>

#include "fp_field.cuh"

struct alignas(64) FpMailbox {
    volatile uint64_t chal;       // host -> device: {chal, chal_seq} written as one 16-byte unit
    volatile uint64_t chal_seq;
    volatile uint64_t chal2;      // second value of a two-value challenge, written before the unit
    volatile uint64_t pad0;
    volatile uint64_t res_seq;    // unused (results are recognised by their slots)
    volatile uint64_t err;        // device -> host: nonzero = a wait gave up
    volatile uint64_t pad1[2];
    volatile uint64_t res[16];
};

struct FpRelay {
    unsigned int ticket;          // blocks finished with the current round
    unsigned int pad0;
    volatile uint64_t seq;        // latest challenge sequence forwarded by block 0
    volatile uint64_t chal;
    volatile uint64_t chal2;
    volatile uint64_t abort;      // nonzero: block 0 gave up waiting
};

// marker of an empty result slot: not a field element
constexpr uint64_t kEmpty = 0xFFFFFFFFFFFFFFFFull;

// 2^22 polls (each a PCIe read of about a microsecond, or a short sleep): seconds before a wait gives up
constexpr uint32_t kSpinLimit = 1u << 22;

#ifdef __CUDACC__

__device__ __forceinline__ uint64_t ld_volatile_u64(const volatile uint64_t* p) { return *p; }

// one 16-byte volatile load: {chal, chal_seq}
__device__ __forceinline__ void ld_volatile_pair(const volatile uint64_t* p, uint64_t& a, uint64_t& b) {
    asm volatile("ld.volatile.global.v2.u64 {%0, %1}, [%2];" : "=l"(a), "=l"(b) : "l"(p) : "memory");
}

// Wait for challenge `seq`; every thread of the block gets its value(s).
// Returns false if the wait ran out (the block should return).
__device__ __forceinline__ bool session_wait2(FpMailbox* mb, FpRelay* rl, uint64_t seq, uint64_t& chal,
                                              uint64_t& chal2, uint32_t limit = kSpinLimit) {
    __shared__ uint64_t s_chal, s_chal2;
    __shared__ int s_ok;
    if (threadIdx.x == 0) {
        int ok = 0;
        uint64_t v = 0, v2 = 0;
        if (blockIdx.x == 0) {
            for (uint32_t it = 0; it < limit; it++) {
                uint64_t c, sq;
                ld_volatile_pair(&mb->chal, c, sq);
                if (sq >= seq) {
                    v = c;
                    ok = 1;
                    break;
                }
                __nanosleep(64);
            }
            if (ok) {
                v2 = ld_volatile_u64(&mb->chal2);
                if (gridDim.x > 1) {
                    rl->chal = v;
                    rl->chal2 = v2;
                    __threadfence();
                    rl->seq = seq;
                }
            } else {
                mb->err = 1;
                rl->abort = 1;
                __threadfence_system();
            }
        } else {
            for (uint32_t it = 0; it < limit; it++) {
                if (ld_volatile_u64(&rl->seq) >= seq) {
                    ok = 1;
                    break;
                }
                if (ld_volatile_u64(&rl->abort)) break;
                __nanosleep(128);
            }
            if (ok) {
                __threadfence();
                v = ld_volatile_u64(&rl->chal);
                v2 = ld_volatile_u64(&rl->chal2);
            } else {
                mb->err = 2;
                __threadfence_system();
            }
        }
        s_chal = v;
        s_chal2 = v2;
        s_ok = ok;
    }
    __syncthreads();
    chal = s_chal;
    chal2 = s_chal2;
    const bool ok = s_ok != 0;
    __syncthreads();
    return ok;
}

__device__ __forceinline__ bool session_wait(FpMailbox* mb, FpRelay* rl, uint64_t seq, uint64_t& chal,
                                             uint32_t limit = kSpinLimit) {
    uint64_t unused;
    return session_wait2(mb, rl, seq, chal, unused, limit);
}

// Publish n values (one thread calls this); seq is kept for the reader of the code only.
__device__ __forceinline__ void session_publish(FpMailbox* mb, const uint64_t* v, int n, uint64_t seq) {
    (void)seq;
    for (int i = 0; i < n; i++) mb->res[i] = v[i];
}

template <int N>
__device__ __forceinline__ void session_publish(FpMailbox* mb, const uint64_t (&v)[N], uint64_t seq) {
    (void)seq;
#pragma unroll
    for (int i = 0; i < N; i++) mb->res[i] = v[i];
}

#endif
