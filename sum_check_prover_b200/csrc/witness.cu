// Witness of the quantised matrix products ("How fast can FlashProve go", 3.1):
// Y = W_eff . X with exact int32 accumulation on the tensor cores, then the
// rescale q = floor((Y + 2^(k-1)) / 2^k), the committed remainder
// r = Y - 2^k q and the clamp y = clamp(q, -128, 127), fused into the epilogue.
//
// D = Y^T (tokens x output rows) is computed as Xt . W^T so that both
// operands are K-contiguous (token-major activations, row-major weights).
// int4 weights are expanded to int8 in registers while building fragments;
// per-64 group scales multiply each k-tile's partial product (one k-tile is
// one scale group).
//
// Two kernels. Unscaled sites run on tcgen05 (witness_tc_kernel: kind::i8 MMAs
// with the accumulator in tensor memory, 128-token x 128- or 256-row tiles,
// operands in the K-major 128-byte-swizzled layout); sites with scales, and all
// sites when FP_TCGEN05=0, run the mma.sync kernel: tile 128 tokens x 128 rows x
// 64 k, 8 warps (2 x 4), warp tile 64 x 32, m16n8k32 s8.s8.s32, 3-stage
// cp.async pipeline. All sites of a call share one launch per operand variant
// (grouped GEMM over a tile list).
#include <cuda.h>  // CUtensorMap
#include <string.h>

#include <algorithm>
#include <vector>

#include "fp_internal.h"

namespace {

constexpr int BM = 128;  // tokens (rows of D)
constexpr int BN = 128;  // output rows i (columns of D)
constexpr int BK = 64;
constexpr int STAGES = 3;
constexpr int THREADS = 256;
constexpr int A_PITCH = 80;               // bytes per smem row of the Xt tile (64 + 16 pad)
constexpr int B8_PITCH = 80;              // int8 W tile
constexpr int B4_PITCH = 48;              // int4 W tile (32 + 16 pad)
constexpr int A_STAGE = BM * A_PITCH;     // 10240
constexpr int B_STAGE = BN * B8_PITCH;    // 10240 (int4 uses the first BN * 48)

struct SiteDev {
    const uint8_t* w;
    const int8_t* scales;
    const int8_t* xt;
    int32_t* q;
    int32_t* r;
    int8_t* y;
    int32_t M, K, N, k_shift;
    int32_t tiles_i, tiles_j;
    int64_t tile_base;  // first tile index of this site in the launch
};

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem, int src_bytes) {
    uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem), "r"(src_bytes));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

__device__ __forceinline__ void mma_s8(int32_t (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};\n"
        : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// four packed nibbles (k0..k0+3, low nibble first) -> four int8 in one word
__device__ __forceinline__ uint32_t nib4_to_s8x4(uint32_t v16) {
    uint32_t lo = v16 & 0x0F0Fu;
    uint32_t hi = (v16 >> 4) & 0x0F0Fu;
    uint32_t w = __byte_perm(lo, hi, 0x5140);
    return w | ((w & 0x08080808u) * 0x1Eu);  // sign-extend bit 3 of every byte
}

__device__ __forceinline__ int find_site(const SiteDev* sites, int nsites, int64_t t) {
    int lo = 0, hi = nsites - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (sites[mid].tile_base <= t)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

// Load one k-tile of Xt (BM x BK) and W (BN x BK) into a stage.
template <bool W4, bool ALIGNED>
__device__ __forceinline__ void load_tile(const SiteDev& S, int j0, int i0, int k0, uint8_t* sa, uint8_t* sb) {
    const int tid = threadIdx.x;
    if (ALIGNED) {
        // Xt: 128 rows x 4 chunks of 16 bytes
#pragma unroll
        for (int c = tid; c < BM * 4; c += THREADS) {
            int row = c >> 2, ch = c & 3;
            int j = j0 + row, k = k0 + ch * 16;
            bool ok = (j < S.N) && (k < S.K);
            const int8_t* src = ok ? S.xt + (int64_t)j * S.K + k : S.xt;
            cp_async16(sa + row * A_PITCH + ch * 16, src, ok ? 16 : 0);
        }
        if (W4) {
            const int pitch = (S.K + 1) >> 1;
#pragma unroll
            for (int c = tid; c < BN * 2; c += THREADS) {
                int row = c >> 1, ch = c & 1;
                int i = i0 + row, kb = (k0 >> 1) + ch * 16;
                bool ok = (i < S.M) && (kb < pitch);
                const uint8_t* src = ok ? S.w + (int64_t)i * pitch + kb : S.w;
                cp_async16(sb + row * B4_PITCH + ch * 16, src, ok ? 16 : 0);
            }
        } else {
#pragma unroll
            for (int c = tid; c < BN * 4; c += THREADS) {
                int row = c >> 2, ch = c & 3;
                int i = i0 + row, k = k0 + ch * 16;
                bool ok = (i < S.M) && (k < S.K);
                const uint8_t* src = ok ? S.w + (int64_t)i * S.K + k : S.w;
                cp_async16(sb + row * B8_PITCH + ch * 16, src, ok ? 16 : 0);
            }
        }
    } else {
        // generic path: byte loads with full bounds checks
        for (int c = tid; c < BM * BK; c += THREADS) {
            int row = c / BK, kk = c % BK;
            int j = j0 + row, k = k0 + kk;
            sa[row * A_PITCH + kk] = (j < S.N && k < S.K) ? (uint8_t)S.xt[(int64_t)j * S.K + k] : 0;
        }
        if (W4) {
            const int pitch = (S.K + 1) >> 1;
            for (int c = tid; c < BN * (BK / 2); c += THREADS) {
                int row = c / (BK / 2), kb = c % (BK / 2);
                int i = i0 + row, k = k0 + 2 * kb;
                uint8_t v = 0;
                if (i < S.M && k < S.K) {
                    v = S.w[(int64_t)i * pitch + (k >> 1)];
                    if (k + 1 >= S.K) v &= 0x0F;
                }
                sb[row * B4_PITCH + kb] = v;
            }
        } else {
            for (int c = tid; c < BN * BK; c += THREADS) {
                int row = c / BK, kk = c % BK;
                int i = i0 + row, k = k0 + kk;
                sb[row * B8_PITCH + kk] = (i < S.M && k < S.K) ? S.w[(int64_t)i * S.K + k] : 0;
            }
        }
    }
}

template <bool W4, bool SCALED, bool ALIGNED>
__global__ void __launch_bounds__(THREADS, 1)
    witness_gemm_kernel(const SiteDev* __restrict__ sites, int nsites) {
    extern __shared__ __align__(16) uint8_t smem[];
    uint8_t* sA = smem;
    uint8_t* sB = smem + STAGES * A_STAGE;

    const int64_t tile = blockIdx.x;
    const int s = find_site(sites, nsites, tile);
    const SiteDev S = sites[s];
    const int64_t lt = tile - S.tile_base;
    const int j0 = (int)(lt / S.tiles_i) * BM;
    const int i0 = (int)(lt % S.tiles_i) * BN;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int wj = (warp >> 2) * 64;  // warp's token offset in the tile
    const int wi = (warp & 3) * 32;   // warp's row offset in the tile

    int32_t acc[4][4][4];
    int32_t tot[4][4][4];  // scaled running total (dead code without scales)
#pragma unroll
    for (int a = 0; a < 4; a++)
#pragma unroll
        for (int b = 0; b < 4; b++)
#pragma unroll
            for (int e = 0; e < 4; e++) acc[a][b][e] = tot[a][b][e] = 0;

    const int nk = (S.K + BK - 1) / BK;
    const int G = (S.K + 63) / 64;

    if (ALIGNED) {
#pragma unroll
        for (int st = 0; st < STAGES - 1; st++) {
            if (st < nk) load_tile<W4, true>(S, j0, i0, st * BK, sA + st * A_STAGE, sB + st * B_STAGE);
            cp_async_commit();
        }
    }

    for (int kt = 0; kt < nk; kt++) {
        uint8_t* a_st;
        uint8_t* b_st;
        if (ALIGNED) {
            cp_async_wait<STAGES - 2>();
            __syncthreads();
            int nxt = kt + STAGES - 1;
            if (nxt < nk)
                load_tile<W4, true>(S, j0, i0, nxt * BK, sA + (nxt % STAGES) * A_STAGE, sB + (nxt % STAGES) * B_STAGE);
            cp_async_commit();
            a_st = sA + (kt % STAGES) * A_STAGE;
            b_st = sB + (kt % STAGES) * B_STAGE;
        } else {
            __syncthreads();
            load_tile<W4, false>(S, j0, i0, kt * BK, sA, sB);
            __syncthreads();
            a_st = sA;
            b_st = sB;
        }

#pragma unroll
        for (int ks = 0; ks < 2; ks++) {
            uint32_t af[4][4];
            uint32_t bf[4][2];
#pragma unroll
            for (int mt = 0; mt < 4; mt++) {
                const uint8_t* base = a_st + (wj + mt * 16 + g) * A_PITCH + ks * 32 + 4 * t;
                af[mt][0] = *reinterpret_cast<const uint32_t*>(base);
                af[mt][1] = *reinterpret_cast<const uint32_t*>(base + 8 * A_PITCH);
                af[mt][2] = *reinterpret_cast<const uint32_t*>(base + 16);
                af[mt][3] = *reinterpret_cast<const uint32_t*>(base + 8 * A_PITCH + 16);
            }
#pragma unroll
            for (int nt = 0; nt < 4; nt++) {
                const int row = wi + nt * 8 + g;
                if (W4) {
                    const uint8_t* base = b_st + row * B4_PITCH + ks * 16 + 2 * t;
                    bf[nt][0] = nib4_to_s8x4(*reinterpret_cast<const uint16_t*>(base));
                    bf[nt][1] = nib4_to_s8x4(*reinterpret_cast<const uint16_t*>(base + 8));
                } else {
                    const uint8_t* base = b_st + row * B8_PITCH + ks * 32 + 4 * t;
                    bf[nt][0] = *reinterpret_cast<const uint32_t*>(base);
                    bf[nt][1] = *reinterpret_cast<const uint32_t*>(base + 16);
                }
            }
#pragma unroll
            for (int mt = 0; mt < 4; mt++)
#pragma unroll
                for (int nt = 0; nt < 4; nt++) mma_s8(acc[mt][nt], af[mt], bf[nt]);
        }

        if (SCALED) {
            // this k-tile is scale group kt: tot += S[i][kt] * acc, then restart acc
#pragma unroll
            for (int nt = 0; nt < 4; nt++) {
                const int ia = i0 + wi + nt * 8 + 2 * t;
                int32_t s0 = (ia < S.M) ? (int32_t)S.scales[(int64_t)ia * G + kt] : 0;
                int32_t s1 = (ia + 1 < S.M) ? (int32_t)S.scales[(int64_t)(ia + 1) * G + kt] : 0;
#pragma unroll
                for (int mt = 0; mt < 4; mt++) {
                    tot[mt][nt][0] += s0 * acc[mt][nt][0];
                    tot[mt][nt][1] += s1 * acc[mt][nt][1];
                    tot[mt][nt][2] += s0 * acc[mt][nt][2];
                    tot[mt][nt][3] += s1 * acc[mt][nt][3];
                    acc[mt][nt][0] = acc[mt][nt][1] = acc[mt][nt][2] = acc[mt][nt][3] = 0;
                }
            }
        }
    }
    if (ALIGNED) cp_async_wait<0>();

    // epilogue: rescale, remainder, clamp; D[j][i] -> q, r, y at [j * M + i]
    const int k = S.k_shift;
    const int64_t half = (int64_t)1 << (k - 1);
#pragma unroll
    for (int mt = 0; mt < 4; mt++)
#pragma unroll
        for (int nt = 0; nt < 4; nt++)
#pragma unroll
            for (int hh = 0; hh < 2; hh++) {
                const int j = j0 + wj + mt * 16 + g + 8 * hh;
                const int i = i0 + wi + nt * 8 + 2 * t;
                if (j >= S.N) continue;
#pragma unroll
                for (int e = 0; e < 2; e++) {
                    if (i + e >= S.M) continue;
                    int32_t Y = SCALED ? tot[mt][nt][2 * hh + e] : acc[mt][nt][2 * hh + e];
                    int64_t qq = ((int64_t)Y + half) >> k;  // arithmetic shift = floor division
                    int64_t rr = (int64_t)Y - (qq << k);
                    int64_t o = (int64_t)j * S.M + i + e;
                    S.q[o] = (int32_t)qq;
                    S.r[o] = (int32_t)rr;
                    S.y[o] = (int8_t)(qq < -128 ? -128 : (qq > 127 ? 127 : qq));
                }
            }
}


// ---- tensor-core (tcgen05) variant -------------------------------------------------
//
// D = Xt . W^T for unscaled sites on the 5th-generation tensor cores: one CTA per
// 128-token x BN-row tile, the accumulator (128 lanes x BN columns of s32) in
// tensor memory, operands in shared memory in the K-major layout with the
// 128-byte swizzle (a k-tile is 128 bytes deep: row r at (r / 8) * 1024 +
// (r % 8) * 128, its 16-byte chunk c at chunk position c ^ (r % 8)); the four
// K = 32 MMAs of a k-tile start 32 bytes apart inside the swizzle atom. cp.async fills stage kt % S two tiles before use;
// int4 weights land packed in the upper half of their stage and are expanded
// to int8 in place just before the MMAs. One thread issues the four K = 32 MMAs
// of a k-tile and commits them to the stage's mbarrier; a stage is refilled
// once the MMAs two tiles back are done, so the tensor core always has the
// next tile queued. The epilogue reads the accumulator with tcgen05.ld and
// applies the rescale / clamp.
constexpr int TC_BM = 128;   // tokens: MMA M, tensor-memory lanes
constexpr int TC_BK = 128;   // bytes of K per stage
constexpr int TC_THREADS = 256;
constexpr int TC_A_BYTES = TC_BM * TC_BK;  // 16 KB
constexpr uint32_t TC_WAIT_LIMIT = 1u << 24;  // mbarrier polls before the kernel gives up

// Shared-memory plan: a ring of STAGES k-tiles of A (and of B for int8 weights; for int4 weights
// a ring of packed tiles plus a double buffer of expanded int8 B tiles), within 224 KB
template <bool W4, int BN>
struct TcCfg {
    static constexpr int B_BYTES = BN * TC_BK;      // an int8 B tile
    static constexpr int PK_BYTES = BN * TC_BK / 2;  // a packed int4 B tile
    static constexpr int RING = W4 ? TC_A_BYTES + PK_BYTES : TC_A_BYTES + B_BYTES;
    static constexpr int FIXED = W4 ? 2 * B_BYTES : 0;
    static constexpr int STAGES = (224 * 1024 - FIXED) / RING;
    static constexpr int SMEM = STAGES * RING + FIXED + 1024;
    // s32 accumulator, s8 x s8, both K-major, N = BN, M = 128
    static constexpr uint32_t IDESC =
        (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(TC_BM >> 4) << 24);
};

__device__ __forceinline__ uint32_t smem_addr(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

// shared-memory matrix descriptor: K-major with the 128-byte swizzle (8-row x 128-byte atoms,
// 1024 B apart along M / N: the stride byte offset; the leading byte offset is unused), version 1
__device__ __forceinline__ uint64_t tc_desc(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFF) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

__device__ __forceinline__ bool tc_wait(uint32_t mbar, uint32_t parity) {
    for (uint32_t it = 0; it < TC_WAIT_LIMIT; it++) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}\n"
            : "=r"(ok)
            : "r"(mbar), "r"(parity)
            : "memory");
        if (ok) return true;
    }
    return false;
}

// byte offset of 16-byte chunk kk of row `row` in a 128-byte-deep k-tile: row r of 8-row atom
// r / 8 at (r / 8) * 1024 + (r % 8) * 128, chunk kk stored at chunk position kk ^ (r % 8)
__device__ __forceinline__ uint32_t tc_off(int row, int kk) {
    return (row >> 3) * 1024 + (row & 7) * 128 + ((kk ^ (row & 7)) << 4);
}

// cp.async of k-tile k0 into a stage (zero fill outside the matrices)
// 16-byte chunk c of a k-tile -> (row, k chunk): eight consecutive lanes take eight consecutive
// rows of one k chunk, which the swizzle spreads over all 32 banks (global reads stay whole
// 32-byte sectors: four k chunks of a row per warp)
__device__ __forceinline__ void tc_chunk(int c, int& row, int& kk) {
    row = (c & 7) | ((c >> 6) << 3);
    kk = (c >> 3) & 7;
}

// packed int4 staging: row r's 16-byte chunk kq at r * 64 + (kq ^ ((r >> 1) & 3)) * 16, so
// that eight consecutive rows of one chunk hit different banks
__device__ __forceinline__ uint32_t tc_pk_off(int row, int kq) { return row * 64 + ((kq ^ ((row >> 1) & 3)) << 4); }

template <bool W4, int BN>
__device__ __forceinline__ void tc_issue(const SiteDev& S, int j0, int i0, int k0, uint8_t* sa, uint8_t* sb) {
    // sb: the int8 B tile, or (int4) the packed tile
    const int tid = threadIdx.x;
#pragma unroll
    for (int u = 0; u < TC_A_BYTES / 16 / TC_THREADS; u++) {
        int row, kk;
        tc_chunk(tid + TC_THREADS * u, row, kk);
        const int j = j0 + row, k = k0 + kk * 16;
        const bool ok = j < S.N && k < S.K;
        cp_async16(sa + tc_off(row, kk), ok ? S.xt + (int64_t)j * S.K + k : S.xt, ok ? 16 : 0);
    }
    if (W4) {
        // packed rows: 64 bytes of the k-tile each
        const int pitch = S.K >> 1;
        uint8_t* pk = sb;
#pragma unroll
        for (int u = 0; u < BN * 4 / TC_THREADS; u++) {
            const int c = tid + TC_THREADS * u, row = c >> 2, kq = c & 3;
            const int i = i0 + row, k = k0 + kq * 32;
            const bool ok = i < S.M && k < S.K;
            cp_async16(pk + tc_pk_off(row, kq), ok ? S.w + (int64_t)i * pitch + (k >> 1) : S.w, ok ? 16 : 0);
        }
    } else {
#pragma unroll
        for (int u = 0; u < BN * 8 / TC_THREADS; u++) {
            int row, kk;
            tc_chunk(tid + TC_THREADS * u, row, kk);
            const int i = i0 + row, k = k0 + kk * 16;
            const bool ok = i < S.M && k < S.K;
            cp_async16(sb + tc_off(row, kk), ok ? S.w + (int64_t)i * S.K + k : S.w, ok ? 16 : 0);
        }
    }
}

// int4: a packed tile -> the swizzled int8 layout of an expanded B buffer; lane l takes
// row l % 8 of its group, so both the reads and the writes are bank-conflict free
template <int BN>
__device__ __forceinline__ void tc_expand(const uint8_t* pk, uint8_t* sb) {
    const int tid = threadIdx.x;
    uint4 v[BN * 4 / TC_THREADS];
#pragma unroll
    for (int u = 0; u < BN * 4 / TC_THREADS; u++) {
        const int c = tid + TC_THREADS * u, row = (c & 7) | ((c >> 5) << 3), kq = (c >> 3) & 3;
        v[u] = *reinterpret_cast<const uint4*>(pk + tc_pk_off(row, kq));
    }
#pragma unroll
    for (int u = 0; u < BN * 4 / TC_THREADS; u++) {
        const int c = tid + TC_THREADS * u, row = (c & 7) | ((c >> 5) << 3), kq = (c >> 3) & 3;
        // 32 nibbles (low nibble first) -> 32 int8 in two 16-byte chunks
        const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
        uint32_t o[8];
#pragma unroll
        for (int q = 0; q < 4; q++) {
            o[2 * q] = nib4_to_s8x4(w[q] & 0xFFFFu);
            o[2 * q + 1] = nib4_to_s8x4(w[q] >> 16);
        }
        *reinterpret_cast<uint4*>(sb + tc_off(row, 2 * kq)) = make_uint4(o[0], o[1], o[2], o[3]);
        *reinterpret_cast<uint4*>(sb + tc_off(row, 2 * kq + 1)) = make_uint4(o[4], o[5], o[6], o[7]);
    }
}

// q, r, y of 16 consecutive weight rows i..i+15 of token j
__device__ __forceinline__ void tc_store16(const SiteDev& S, int j, int i, const uint32_t (&v)[16]) {
    const int k = S.k_shift;
    const int64_t half = (int64_t)1 << (k - 1);
    int32_t q[16], r[16];
    uint32_t y[4] = {0, 0, 0, 0};
#pragma unroll
    for (int e = 0; e < 16; e++) {
        const int64_t Y = (int32_t)v[e];
        const int64_t qq = (Y + half) >> k;
        q[e] = (int32_t)qq;
        r[e] = (int32_t)(Y - (qq << k));
        const int32_t yc = qq < -128 ? -128 : (qq > 127 ? 127 : (int32_t)qq);
        y[e >> 2] |= ((uint32_t)yc & 0xFFu) << (8 * (e & 3));
    }
    const int64_t o = (int64_t)j * S.M + i;
    const bool vec = i + 16 <= S.M && ((reinterpret_cast<uintptr_t>(S.q + o) | reinterpret_cast<uintptr_t>(S.r + o) |
                                        reinterpret_cast<uintptr_t>(S.y + o)) & 15) == 0;
    if (vec) {
#pragma unroll
        for (int e = 0; e < 16; e += 4) {
            *reinterpret_cast<int4*>(S.q + o + e) = make_int4(q[e], q[e + 1], q[e + 2], q[e + 3]);
            *reinterpret_cast<int4*>(S.r + o + e) = make_int4(r[e], r[e + 1], r[e + 2], r[e + 3]);
        }
        *reinterpret_cast<uint4*>(S.y + o) = make_uint4(y[0], y[1], y[2], y[3]);
    } else {
#pragma unroll
        for (int e = 0; e < 16; e++) {
            if (i + e >= S.M) break;
            S.q[o + e] = q[e];
            S.r[o + e] = r[e];
            S.y[o + e] = (int8_t)(y[e >> 2] >> (8 * (e & 3)));
        }
    }
}

template <bool W4, int BN>
__global__ void __launch_bounds__(TC_THREADS, 1)
    witness_tc_kernel(const SiteDev* __restrict__ sites, int nsites, volatile uint64_t* err) {
    using C = TcCfg<W4, BN>;
    constexpr int ST = C::STAGES;
    constexpr int SBT = W4 ? C::PK_BYTES : C::B_BYTES;  // ring slot of the B side
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = smem_raw + ((1024 - (smem_addr(smem_raw) & 1023)) & 1023);
    uint8_t* sA = smem;
    uint8_t* sB = smem + ST * TC_A_BYTES;  // int8 B tiles, or packed int4 tiles
    uint8_t* sX = sB + ST * SBT;            // int4: two expanded B tiles
    __shared__ __align__(8) uint64_t mbar[ST];
    __shared__ uint32_t tmem_base;
    __shared__ int s_fail;

    const int64_t tile = blockIdx.x;
    const SiteDev S = sites[find_site(sites, nsites, tile)];
    const int64_t lt = tile - S.tile_base;
    const int j0 = (int)(lt / S.tiles_i) * TC_BM;
    const int i0 = (int)(lt % S.tiles_i) * BN;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nk = (S.K + TC_BK - 1) / TC_BK;

    if (tid == 0) {
        s_fail = 0;
#pragma unroll
        for (int st = 0; st < ST; st++) asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(smem_addr(&mbar[st])));
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::);
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_addr(&tmem_base)),
                     "n"(BN));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::);
    }
    // prologue: tiles 0 .. ST-3 in flight (prefetch distance ST - 2)
#pragma unroll
    for (int t = 0; t < ST - 2; t++) {
        if (t < nk) tc_issue<W4, BN>(S, j0, i0, t * TC_BK, sA + t * TC_A_BYTES, sB + t * SBT);
        cp_async_commit();
    }
    asm volatile("tcgen05.fence::before_thread_sync;\n" ::);
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;\n" ::);
    const uint32_t tmem = tmem_base;

    for (int kt = 0; kt < nk; kt++) {
        const int st = kt % ST;
        // refill the stage of tile kt + ST - 2; its previous tile (kt - 2) must be done with it
        // (for int4 this also frees the expanded buffer that tile kt is about to use)
        const int nt = kt + ST - 2, ns = nt % ST;
        const bool late = (W4 || nt < nk) && kt >= 2 && !tc_wait(smem_addr(&mbar[ns]), (uint32_t)(((kt - 2) / ST) & 1));
        if (__syncthreads_or(late)) {
            if (tid == 0) s_fail = 1;
            break;
        }
        if (nt < nk) tc_issue<W4, BN>(S, j0, i0, nt * TC_BK, sA + ns * TC_A_BYTES, sB + ns * SBT);
        cp_async_commit();
        cp_async_wait<ST - 2>();  // tile kt has landed (this thread's copies)
        __syncthreads();
        uint8_t* bt = W4 ? sX + (kt & 1) * C::B_BYTES : sB + st * SBT;  // the B tile the MMAs read
        if (W4) tc_expand<BN>(sB + st * SBT, bt);
        asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");  // generic writes -> tensor-core reads
        asm volatile("tcgen05.fence::before_thread_sync;\n" ::);
        __syncthreads();
        asm volatile("tcgen05.fence::after_thread_sync;\n" ::);
        if (tid == 0) {
            const uint32_t a0 = smem_addr(sA + st * TC_A_BYTES), b0 = smem_addr(bt);
#pragma unroll
            for (int kc = 0; kc < TC_BK / 32; kc++) {
                const uint32_t en = (kt > 0 || kc > 0) ? 1u : 0u;
                asm volatile(
                    "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
                    "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem),
                    "l"(tc_desc(a0 + kc * 32)), "l"(tc_desc(b0 + kc * 32)), "r"(C::IDESC), "r"(en));
            }
            asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
                smem_addr(&mbar[st])));
        }
    }
    cp_async_wait<0>();
    // all MMAs done: the last tile's commit completes after every earlier one
    const int last = nk - 1;
    __syncthreads();
    const bool done = !s_fail && tc_wait(smem_addr(&mbar[last % ST]), (uint32_t)((last / ST) & 1));
    const bool ok = !__syncthreads_or(!done);  // the same answer in every thread (tcgen05.ld is warp-wide)
    asm volatile("tcgen05.fence::after_thread_sync;\n" ::);
    if (ok) {
        // warp w reads lanes 32 (w % 4) .. + 31 (tokens) and the (w / 4)-th half of the columns
        const int j = j0 + 32 * (warp & 3) + lane;
        const int cbase = (BN / 2) * (warp >> 2);
#pragma unroll 1
        for (int c0 = 0; c0 < BN / 2; c0 += 16) {
            uint32_t v[16];
            const uint32_t a = tmem + ((uint32_t)(32 * (warp & 3)) << 16) + (uint32_t)(cbase + c0);
            asm volatile(
                "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
                : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
                  "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
                : "r"(a));
            asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
            const int i = i0 + cbase + c0;
            if (j < S.N && i < S.M) tc_store16(S, j, i, v);
        }
    } else if (tid == 0) {
        *err = 3;  // a tensor-core wait ran out
        __threadfence_system();
    }
    asm volatile("tcgen05.fence::before_thread_sync;\n" ::);
    __syncthreads();
    if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem), "n"(BN));
}

template <bool W4, int BN>
int launch_tc_bn(fp_ctx* c, const std::vector<fp_site>& list, cudaStream_t st) {
    std::vector<SiteDev> h(list.size());
    int64_t tiles = 0;
    double bytes = 0;
    for (size_t s = 0; s < list.size(); s++) {
        const fp_site& t = list[s];
        SiteDev& d = h[s];
        d.w = (const uint8_t*)t.w;
        d.scales = t.scales;
        d.xt = t.xt;
        d.q = t.q;
        d.r = t.r;
        d.y = t.y;
        d.M = t.M;
        d.K = t.K;
        d.N = t.N;
        d.k_shift = t.k_shift;
        d.tiles_i = (t.M + BN - 1) / BN;
        d.tiles_j = (t.N + TC_BM - 1) / TC_BM;
        d.tile_base = tiles;
        tiles += (int64_t)d.tiles_i * d.tiles_j;
        bytes += (double)t.M * (W4 ? t.K / 2 : t.K) + (double)t.N * t.K + 9.0 * t.M * t.N;
    }
    size_t sz = sizeof(SiteDev) * h.size();
    SiteDev* dsites = (SiteDev*)fp_alloc(c->dev, sz);
    char* hst = (char*)fp_alloc(c->host, sz);
    if (!dsites || !hst) return fp_fail(c, FP_ERR_OOM, "witness: scratch exhausted");
    memcpy(hst, h.data(), sz);
    FP_CUDA(c, cudaMemcpyAsync(dsites, hst, sz, cudaMemcpyHostToDevice, st));
    auto kern = witness_tc_kernel<W4, BN>;
    FP_CUDA(c, cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, TcCfg<W4, BN>::SMEM));
    int slot;
    fp_tic(c, st, K_GEMM, bytes, &slot);
    kern<<<(unsigned)tiles, TC_THREADS, TcCfg<W4, BN>::SMEM, st>>>(dsites, (int)h.size(), &c->mb_dev->err);
    fp_toc(c, st, slot);
    FP_CUDA(c, cudaGetLastError());
    return FP_OK;
}

// 256-row tiles when they still give every SM a tile, 128-row tiles otherwise
template <bool W4>
int launch_tc(fp_ctx* c, const std::vector<fp_site>& list, cudaStream_t st) {
    if (list.empty()) return FP_OK;
    int64_t wide = 0;
    for (const fp_site& t : list) wide += (int64_t)((t.M + 255) / 256) * ((t.N + TC_BM - 1) / TC_BM);
    return wide >= c->num_sms ? launch_tc_bn<W4, 256>(c, list, st) : launch_tc_bn<W4, 128>(c, list, st);
}

template <bool W4, bool SCALED, bool ALIGNED>
int launch_variant(fp_ctx* c, const std::vector<fp_site>& list, cudaStream_t st) {
    if (list.empty()) return FP_OK;
    std::vector<SiteDev> h(list.size());
    int64_t tiles = 0;
    double bytes = 0;
    for (size_t s = 0; s < list.size(); s++) {
        const fp_site& t = list[s];
        SiteDev& d = h[s];
        d.w = (const uint8_t*)t.w;
        d.scales = t.scales;
        d.xt = t.xt;
        d.q = t.q;
        d.r = t.r;
        d.y = t.y;
        d.M = t.M;
        d.K = t.K;
        d.N = t.N;
        d.k_shift = t.k_shift;
        d.tiles_i = (t.M + BN - 1) / BN;
        d.tiles_j = (t.N + BM - 1) / BM;
        d.tile_base = tiles;
        tiles += (int64_t)d.tiles_i * d.tiles_j;
        bytes += (double)t.M * (W4 ? (t.K + 1) / 2 : t.K) + (double)t.N * t.K + 9.0 * t.M * t.N;
    }
    size_t sz = sizeof(SiteDev) * h.size();
    SiteDev* dsites = (SiteDev*)fp_alloc(c->dev, sz);
    char* hst = (char*)fp_alloc(c->host, sz);
    if (!dsites || !hst) return fp_fail(c, FP_ERR_OOM, "witness: scratch exhausted");
    memcpy(hst, h.data(), sz);
    FP_CUDA(c, cudaMemcpyAsync(dsites, hst, sz, cudaMemcpyHostToDevice, st));
    const int smem = STAGES * (A_STAGE + B_STAGE);
    auto kern = witness_gemm_kernel<W4, SCALED, ALIGNED>;
    FP_CUDA(c, cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
    int slot;
    fp_tic(c, st, K_GEMM, bytes, &slot);
    kern<<<(unsigned)tiles, THREADS, smem, st>>>(dsites, (int)h.size());
    fp_toc(c, st, slot);
    FP_CUDA(c, cudaGetLastError());
    return FP_OK;
}


// ---- warp-specialised tcgen05 kernel (every site with TMA-readable operands) ---------------
//
// D = Xt . W_eff^T on the 5th-generation tensor cores, for unscaled and scaled sites alike. A
// persistent kernel: one CTA per SM takes tiles of 128 tokens x WS BN weight rows in turn, and
// its warps split the work, handing stages over on mbarriers:
//   warp 0 (one lane)  TMA producer: per k-tile (128 bytes of K) the Xt box (128 tokens x 128
//                      bytes, 128-byte swizzle: the MMA's K-major layout) and the weight box (the
//                      packed int4 rows, the int8 rows, or for unscaled int8 directly in the MMA
//                      layout) into ring stage s, once the MMAs that read its last tile are done.
//   expansion warps    int4 -> int8, or W_eff = s * w split into a high s8 and a low u8 byte limb
//                      (256 hi + lo), from the loaded box into one of two buffers in the MMA layout.
//   warp 1 (one lane)  MMA issue: four K = 32 MMAs per k-tile (and four more on the low limb) into
//                      the tile's tensor-memory accumulator slot; each k-tile commits to the stage
//                      and buffer it read, a tile's last k-tile to the slot's "full" barrier.
//   epilogue warps     tcgen05.ld of a slot (two slots: the next tile's MMAs run meanwhile),
//                      Y = hi 256 + lo for two limbs, the rescale / remainder / clamp, stores.
// Every wait is bounded; a wait that runs out sets the error word and an abort flag that ends the
// other roles' waits, and the kernel drains its copies and MMAs before it frees tensor memory.
#ifndef FP_WS_EPI_WARPS
#define FP_WS_EPI_WARPS 4
#endif
#ifndef FP_WS_SA
#define FP_WS_SA 3
#endif
#ifndef FP_WS_XBUF
#define FP_WS_XBUF 3
#endif
#ifndef FP_WS_EXP_WARPS
#define FP_WS_EXP_WARPS 12
#endif
constexpr int WS_BM = 128;                  // tokens per tile: MMA M, tensor-memory lanes
constexpr int WS_BK = 128;                  // bytes of K per k-tile
constexpr int WS_A_BYTES = WS_BM * WS_BK;   // 16 KB
constexpr uint32_t WS_WAIT_LIMIT = 1u << 24;

template <bool W4, bool SCALED>
struct WsCfg {
    static constexpr bool EXPAND = W4 || SCALED;  // the MMA reads an expanded copy of the weight box
    static constexpr int BN = SCALED ? 128 : 256;  // weight rows per tile: MMA N
    static constexpr int LIMBS = SCALED ? 2 : 1;   // accumulators per tile
    static constexpr int ACC_COLS = LIMBS * BN;    // tensor-memory columns per accumulator slot
    static constexpr int BP_BYTES = BN * (W4 ? WS_BK / 2 : WS_BK);        // the weight box as loaded
    static constexpr int X_BYTES = EXPAND ? LIMBS * BN * WS_BK : 0;       // one expanded buffer
    // Expanded sites: an Xt ring of SA stages (freed by the MMAs that read it), a weight ring of SP
    // stages (freed by the expansion as soon as it has read the box, so the weight stream runs ahead
    // of the MMAs) and SX expanded buffers (the expansion runs up to SX k-tiles ahead of the MMAs).
    // Unscaled int8: one ring of Xt and weight boxes.
    static constexpr int RING = WS_A_BYTES + BP_BYTES;
    static constexpr int BUDGET = 208 * 1024;
    static constexpr int SX = EXPAND ? FP_WS_XBUF : 1;
    static constexpr int SA_RAW = EXPAND ? FP_WS_SA : BUDGET / RING;
    static constexpr int SA = SA_RAW > 6 ? 6 : SA_RAW;
    static constexpr int SP_RAW = EXPAND ? (BUDGET - SX * X_BYTES - SA * WS_A_BYTES) / BP_BYTES : 0;
    static constexpr int SP = SP_RAW > 8 ? 8 : SP_RAW;
    static constexpr int A_STAGE = EXPAND ? WS_A_BYTES : RING;  // bytes of one Xt-ring stage
    static constexpr int EXP_WARPS = EXPAND ? FP_WS_EXP_WARPS : 0;  // the expansion is latency-bound: several per sub-partition
    static constexpr int EPI0 = 3 + EXP_WARPS;     // first epilogue warp
    // epilogue warps: four consecutive ones cover the four lane quarters; eight split the columns in two
    static constexpr int EPI_WARPS = FP_WS_EPI_WARPS;
    static constexpr int THREADS = 32 * (EPI0 + EPI_WARPS);
    static constexpr int SMEM = SA * A_STAGE + SP * BP_BYTES + SX * X_BYTES + 1024;
    // s32 accumulator, A s8, B s8 (or u8 for the low limb), both K-major, N = BN, M = 128
    static constexpr uint32_t IDESC_S8 =
        (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(WS_BM >> 4) << 24);
    static constexpr uint32_t IDESC_U8 =
        (2u << 4) | (1u << 7) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(WS_BM >> 4) << 24);
};

struct alignas(64) SiteWs {
    CUtensorMap tmA;   // Xt: N rows of K bytes, 128 x 128 boxes, 128-byte swizzle
    CUtensorMap tmB;   // W: M rows (packed int4 or int8), boxes of one k-tile x BN rows
    const int8_t* scales;
    int32_t* q;
    int32_t* r;
    int8_t* y;
    int32_t M, K, N, k_shift;
    int32_t G;         // scale groups per row, ceil(K / 64)
    int32_t tiles_i;   // weight-row tiles
    int32_t nk;        // k-tiles
    int32_t pad;
    int64_t tile_base;  // first tile of this site
};

// one bounded wait on an mbarrier phase; false if it ran out (the kernel is then aborting) or
// another role has aborted
__device__ __forceinline__ bool ws_wait(uint32_t mbar, uint32_t parity, volatile int* abort, volatile uint64_t* err) {
    for (uint32_t it = 0; it < WS_WAIT_LIMIT; it++) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}\n"
            : "=r"(ok)
            : "r"(mbar), "r"(parity)
            : "memory");
        if (ok) return true;
        if (*abort) return false;
    }
    *abort = 1;
    *err = 3;  // a tensor-core pipeline wait ran out
    __threadfence_system();
    return false;
}

// ws_wait by every lane of a warp, with one answer for the warp (a warp-collective tcgen05.ld and
// the warp's arrivals stay uniform)
__device__ __forceinline__ bool ws_wait_warp(uint32_t mbar, uint32_t parity, volatile int* abort, volatile uint64_t* err) {
    const bool ok = ws_wait(mbar, parity, abort, err);
    return __all_sync(0xffffffffu, ok);
}

// the same without the abort check: draining the copies and MMAs still in flight
__device__ __forceinline__ void ws_drain(uint32_t mbar, uint32_t parity) {
    for (uint32_t it = 0; it < WS_WAIT_LIMIT; it++) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}\n"
            : "=r"(ok)
            : "r"(mbar), "r"(parity)
            : "memory");
        if (ok) return;
    }
}

__device__ __forceinline__ void ws_arrive(uint32_t mbar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(mbar) : "memory");
}

__device__ __forceinline__ void ws_commit(uint32_t mbar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(mbar) : "memory");
}

__device__ __forceinline__ void ws_mma(uint32_t tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t en) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(en));
}

__device__ __forceinline__ void ws_tma2d(uint32_t dst, const CUtensorMap* tm, int x, int y, uint32_t mbar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
        "[%4];\n" ::"r"(dst),
        "l"(tm), "r"(x), "r"(y), "r"(mbar)
        : "memory");
}

// eight packed nibbles (k0..k7, low nibble first) -> eight sign-extended int8 in two words
__device__ __forceinline__ void nib8_to_s8x8(uint32_t v, uint32_t& o0, uint32_t& o1) {
    uint32_t lo = v & 0x0F0F0F0Fu, hi = (v >> 4) & 0x0F0F0F0Fu;  // k0 k2 k4 k6 / k1 k3 k5 k7
    lo |= (lo & 0x08080808u) * 0x1Eu;                            // sign-extend bit 3 of every byte
    hi |= (hi & 0x08080808u) * 0x1Eu;
    o0 = __byte_perm(lo, hi, 0x5140);
    o1 = __byte_perm(lo, hi, 0x7362);
}

// W_eff = s * w for four signed bytes w (one word): the high s8 limb (W_eff >> 8) and the low u8
// limb (W_eff & 255), so W_eff = 256 hi + lo exactly (|s w| <= 2^14)
__device__ __forceinline__ void ws_limbs4(uint32_t w4, int s, uint32_t& hi, uint32_t& lo) {
    hi = lo = 0;
#pragma unroll
    for (int b = 0; b < 4; b++) {
        const int v = (int)(int8_t)(w4 >> (8 * b)) * s;
        lo |= ((uint32_t)v & 0xFFu) << (8 * b);
        hi |= ((uint32_t)(v >> 8) & 0xFFu) << (8 * b);
    }
}

// The loaded weight box of k-tile kt -> the expanded buffer(s) in the MMA layout (tc_off). et:
// this thread's index among the expansion threads.
template <bool W4, bool SCALED>
__device__ __forceinline__ void ws_expand(const SiteWs& S, const uint8_t* pk, uint8_t* xb, int i0, int kt, int et) {
    using C = WsCfg<W4, SCALED>;
    constexpr int ET = C::EXP_WARPS > 0 ? 32 * C::EXP_WARPS : 32;  // (no expansion warps: never called)
    if (W4) {
        // 16-byte packed chunk c: row c >> 2, k values 32 (c & 3) .. + 31 -> two 16-byte chunks
#pragma unroll
        for (int u = 0; u < (C::BN * 4 + ET - 1) / ET; u++) {
            const int c = et + ET * u, row = c >> 2, kq = c & 3;
            if ((C::BN * 4) % ET != 0 && c >= C::BN * 4) break;
            const uint4 v = *reinterpret_cast<const uint4*>(pk + row * 64 + kq * 16);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
            uint32_t o[8];
#pragma unroll
            for (int q = 0; q < 4; q++) nib8_to_s8x8(w[q], o[2 * q], o[2 * q + 1]);
            if (SCALED) {
                const int i = i0 + row, g = (kt * WS_BK + kq * 32) >> 6;
                const int s = (i < S.M && g < S.G) ? (int)S.scales[(int64_t)i * S.G + g] : 0;
                uint32_t hi[8], lo[8];
#pragma unroll
                for (int q = 0; q < 8; q++) ws_limbs4(o[q], s, hi[q], lo[q]);
                uint8_t* xl = xb + C::BN * WS_BK;
                *reinterpret_cast<uint4*>(xb + tc_off(row, 2 * kq)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
                *reinterpret_cast<uint4*>(xb + tc_off(row, 2 * kq + 1)) = make_uint4(hi[4], hi[5], hi[6], hi[7]);
                *reinterpret_cast<uint4*>(xl + tc_off(row, 2 * kq)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
                *reinterpret_cast<uint4*>(xl + tc_off(row, 2 * kq + 1)) = make_uint4(lo[4], lo[5], lo[6], lo[7]);
            } else {
                *reinterpret_cast<uint4*>(xb + tc_off(row, 2 * kq)) = make_uint4(o[0], o[1], o[2], o[3]);
                *reinterpret_cast<uint4*>(xb + tc_off(row, 2 * kq + 1)) = make_uint4(o[4], o[5], o[6], o[7]);
            }
        }
    } else {
        // scaled int8: 16-byte chunk c: row c >> 3, k values 16 (c & 7) .. + 15
#pragma unroll
        for (int u = 0; u < (C::BN * 8 + ET - 1) / ET; u++) {
            const int c = et + ET * u, row = c >> 3, kc = c & 7;
            if ((C::BN * 8) % ET != 0 && c >= C::BN * 8) break;
            const uint4 v = *reinterpret_cast<const uint4*>(pk + row * 128 + kc * 16);
            const int i = i0 + row, g = (kt * WS_BK + kc * 16) >> 6;
            const int s = (i < S.M && g < S.G) ? (int)S.scales[(int64_t)i * S.G + g] : 0;
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int q = 0; q < 4; q++) ws_limbs4(w[q], s, hi[q], lo[q]);
            *reinterpret_cast<uint4*>(xb + tc_off(row, kc)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
            *reinterpret_cast<uint4*>(xb + C::BN * WS_BK + tc_off(row, kc)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
    }
}

// q, r, y of 16 consecutive weight rows i..i+15 of token j from their accumulator values
__device__ __forceinline__ void ws_store16(const SiteWs& S, int j, int i, const uint32_t (&v)[16]) {
    const int k = S.k_shift;
    const int64_t half = (int64_t)1 << (k - 1);
    int32_t q[16], r[16];
    uint32_t y[4] = {0, 0, 0, 0};
#pragma unroll
    for (int e = 0; e < 16; e++) {
        const int64_t Y = (int32_t)v[e];
        const int64_t qq = (Y + half) >> k;
        q[e] = (int32_t)qq;
        r[e] = (int32_t)(Y - (qq << k));
        const int32_t yc = qq < -128 ? -128 : (qq > 127 ? 127 : (int32_t)qq);
        y[e >> 2] |= ((uint32_t)yc & 0xFFu) << (8 * (e & 3));
    }
    const int64_t o = (int64_t)j * S.M + i;
    const bool vec = i + 16 <= S.M && ((reinterpret_cast<uintptr_t>(S.q + o) | reinterpret_cast<uintptr_t>(S.r + o) |
                                        reinterpret_cast<uintptr_t>(S.y + o)) & 15) == 0;
    if (vec) {
#pragma unroll
        for (int e = 0; e < 16; e += 4) {
            *reinterpret_cast<int4*>(S.q + o + e) = make_int4(q[e], q[e + 1], q[e + 2], q[e + 3]);
            *reinterpret_cast<int4*>(S.r + o + e) = make_int4(r[e], r[e + 1], r[e + 2], r[e + 3]);
        }
        *reinterpret_cast<uint4*>(S.y + o) = make_uint4(y[0], y[1], y[2], y[3]);
    } else {
#pragma unroll
        for (int e = 0; e < 16; e++) {
            if (i + e >= S.M) break;
            S.q[o + e] = q[e];
            S.r[o + e] = r[e];
            S.y[o + e] = (int8_t)(y[e >> 2] >> (8 * (e & 3)));
        }
    }
}

__device__ __forceinline__ void ws_ld16(uint32_t a, uint32_t (&v)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]), "=r"(v[8]),
          "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(a));
}

template <bool W4, bool SCALED>
__global__ void __launch_bounds__(WsCfg<W4, SCALED>::THREADS, 1)
    witness_ws_kernel(const SiteWs* __restrict__ sites, const int4* __restrict__ sched, int64_t ntiles,
                      volatile uint64_t* err) {
    using C = WsCfg<W4, SCALED>;
    constexpr int SA = C::SA, SP = C::SP > 0 ? C::SP : 1;
    extern __shared__ uint8_t ws_smem_raw[];
    uint8_t* smem = ws_smem_raw + ((1024 - (smem_addr(ws_smem_raw) & 1023)) & 1023);
    uint8_t* aring = smem;                          // Xt-ring stage s at s A_STAGE (+ the weight box, unexpanded)
    uint8_t* pring = smem + SA * C::A_STAGE;        // weight-ring stage s at s BP_BYTES (expanded sites)
    uint8_t* xbuf = pring + C::SP * C::BP_BYTES;    // SX expanded buffers (high limb first)
    constexpr int SX = C::SX;
    __shared__ __align__(8) uint64_t afull[SA], aempty[SA], pfull[SP], pempty[SP], xfull[SX], xempty[SX], accfull[2],
        accempty[2], fin;
    __shared__ uint32_t tmem_base;
    __shared__ volatile int s_abort;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
#pragma unroll
        for (int s = 0; s < SA; s++) {
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(smem_addr(&afull[s])));
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(smem_addr(&aempty[s])));
        }
#pragma unroll
        for (int s = 0; s < SP; s++) {
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(smem_addr(&pfull[s])));
            asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_addr(&pempty[s])), "r"(32 * C::EXP_WARPS));
        }
#pragma unroll
        for (int e = 0; e < SX; e++) {
            asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_addr(&xfull[e])), "r"(32 * C::EXP_WARPS));
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(smem_addr(&xempty[e])));
        }
#pragma unroll
        for (int e = 0; e < 2; e++) {
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(smem_addr(&accfull[e])));
            asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_addr(&accempty[e])), "r"(32 * C::EPI_WARPS));
        }
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;\n" ::"r"(smem_addr(&fin)));
        s_abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;\n" ::);
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;\n" ::"r"(smem_addr(&tmem_base)));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::);
    }
    asm volatile("tcgen05.fence::before_thread_sync;\n" ::);
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;\n" ::);
    const uint32_t tmem = tmem_base;

    if (warp == 0 || (warp == 2 && C::EXPAND)) {
        if (lane == 0) {
            // ---- producers: warp 0 the Xt ring (with the weight boxes when nothing is expanded),
            // warp 2 the weight ring of expanded sites ----
            const bool xt = warp == 0;
            const int NS = xt ? SA : SP;
            uint64_t* fullb = xt ? afull : pfull;
            uint64_t* emptyb = xt ? aempty : pempty;
            const uint32_t bytes = xt ? (uint32_t)C::A_STAGE : (uint32_t)C::BP_BYTES;
            uint32_t it = 0;
            const SiteWs* cur = nullptr;
            bool ok = true;
            int4 nx = blockIdx.x < ntiles ? sched[blockIdx.x] : make_int4(0, 0, 0, 0);
            for (int64_t t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
                const int4 e = nx;  // {site, j0, i0, k-tiles}
                if (t + gridDim.x < ntiles) nx = sched[t + gridDim.x];
                const SiteWs* S = &sites[e.x];
                if (S != cur) {
                    asm volatile("fence.proxy.tensormap::generic.acquire.gpu [%0], 128;\n" ::"l"(&S->tmA) : "memory");
                    asm volatile("fence.proxy.tensormap::generic.acquire.gpu [%0], 128;\n" ::"l"(&S->tmB) : "memory");
                    cur = S;
                }
                const int j0 = e.y, i0 = e.z;
                for (int kt = 0; kt < e.w; kt++, it++) {
                    const int s = (int)(it % NS);
                    const uint32_t n = it / NS;
                    if (n > 0 && !ws_wait(smem_addr(&emptyb[s]), (n - 1) & 1u, &s_abort, err)) {
                        ok = false;
                        break;
                    }
                    const uint32_t fb = smem_addr(&fullb[s]);
                    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(fb), "r"(bytes) : "memory");
                    const int kw = kt * (W4 ? WS_BK / 2 : WS_BK);
                    if (xt) {
                        ws_tma2d(smem_addr(aring + s * C::A_STAGE), &S->tmA, kt * WS_BK, j0, fb);
                        if (!C::EXPAND) ws_tma2d(smem_addr(aring + s * C::A_STAGE + WS_A_BYTES), &S->tmB, kw, i0, fb);
                    } else {
                        ws_tma2d(smem_addr(pring + s * C::BP_BYTES), &S->tmB, kw, i0, fb);
                    }
                }
            }
            if (!ok) {
                // let every copy that was issued land before the block ends
                for (int s = 0; s < NS; s++) {
                    if (it <= (uint32_t)s) continue;
                    const uint32_t last = (uint32_t)s + ((it - 1 - (uint32_t)s) / NS) * NS;
                    ws_drain(smem_addr(&fullb[s]), (last / NS) & 1u);
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            // ---- MMA issue ----
            uint32_t it = 0, tc = 0;
            bool ok = true;
            int4 nx = blockIdx.x < ntiles ? sched[blockIdx.x] : make_int4(0, 0, 0, 0);
            for (int64_t t = blockIdx.x; t < ntiles && ok; t += gridDim.x, tc++) {
                const int nk = nx.w;
                if (t + gridDim.x < ntiles) nx = sched[t + gridDim.x];
                const uint32_t a = tc & 1u;
                if (tc >= 2 && !ws_wait(smem_addr(&accempty[a]), ((tc >> 1) - 1) & 1u, &s_abort, err)) break;
                asm volatile("tcgen05.fence::after_thread_sync;\n" ::);
                const uint32_t dst = tmem + a * C::ACC_COLS;
                for (int kt = 0; kt < nk; kt++, it++) {
                    const int s = (int)(it % SA), e = (int)(it % SX);
                    if (!ws_wait(smem_addr(&afull[s]), (it / SA) & 1u, &s_abort, err) ||
                        (C::EXPAND && !ws_wait(smem_addr(&xfull[e]), (it / SX) & 1u, &s_abort, err))) {
                        ok = false;
                        break;
                    }
                    asm volatile("tcgen05.fence::after_thread_sync;\n" ::);
                    const uint32_t a0 = smem_addr(aring + s * C::A_STAGE);
                    const uint32_t b0 = C::EXPAND ? smem_addr(xbuf + e * C::X_BYTES) : a0 + WS_A_BYTES;
#pragma unroll
                    for (int kc = 0; kc < WS_BK / 32; kc++) {
                        const uint32_t en = (kt > 0 || kc > 0) ? 1u : 0u;
                        ws_mma(dst, tc_desc(a0 + kc * 32), tc_desc(b0 + kc * 32), C::IDESC_S8, en);
                        if (SCALED)
                            ws_mma(dst + C::BN, tc_desc(a0 + kc * 32), tc_desc(b0 + C::BN * WS_BK + kc * 32), C::IDESC_U8, en);
                    }
                    ws_commit(smem_addr(&aempty[s]));
                    if (C::EXPAND) ws_commit(smem_addr(&xempty[e]));
                }
                if (ok) ws_commit(smem_addr(&accfull[a]));
            }
            // every MMA issued is complete before the tensor memory is freed
            ws_commit(smem_addr(&fin));
            ws_drain(smem_addr(&fin), 0);
        }
        __syncwarp();
    } else if (warp >= 3 && warp < C::EPI0) {
        // ---- expansion: the weight box of k-tile it from the weight ring into expanded buffer it % SX,
        // the ring stage handed back as soon as it is read ----
        const int et = tid - 96;
        uint32_t it = 0;
        bool ok = true;
        int4 nx = blockIdx.x < ntiles ? sched[blockIdx.x] : make_int4(0, 0, 0, 0);
        for (int64_t t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
            const int4 te = nx;
            if (t + gridDim.x < ntiles) nx = sched[t + gridDim.x];
            const SiteWs* S = &sites[te.x];
            const int i0 = te.z;
            for (int kt = 0; kt < te.w; kt++, it++) {
                const int s = (int)(it % SP), e = (int)(it % SX);
                if (!ws_wait_warp(smem_addr(&pfull[s]), (it / SP) & 1u, &s_abort, err) ||
                    (it >= SX && !ws_wait_warp(smem_addr(&xempty[e]), ((it / SX) - 1) & 1u, &s_abort, err))) {
                    ok = false;
                    break;
                }
                ws_expand<W4, SCALED>(*S, pring + s * C::BP_BYTES, xbuf + e * C::X_BYTES, i0, kt, et);
                asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");  // generic writes -> MMA reads
                ws_arrive(smem_addr(&xfull[e]));
                ws_arrive(smem_addr(&pempty[s]));
            }
        }
    } else if (warp >= C::EPI0) {
        // ---- epilogue: warp w reads tensor-memory lanes 32 (w % 4) .. + 31 (tokens), its share of the
        // columns in chunks of 16, each chunk's load issued before the previous chunk is stored ----
        constexpr int COLS = C::BN / (C::EPI_WARPS / 4), NCH = COLS / 16;
        const int qd = warp & 3, cbase = ((warp - C::EPI0) >> 2) * COLS;
        uint32_t tc = 0;
        int4 nx = blockIdx.x < ntiles ? sched[blockIdx.x] : make_int4(0, 0, 0, 0);
        for (int64_t t = blockIdx.x; t < ntiles; t += gridDim.x, tc++) {
            const int4 te = nx;
            if (t + gridDim.x < ntiles) nx = sched[t + gridDim.x];
            const SiteWs* S = &sites[te.x];
            const int j0 = te.y, i0 = te.z;
            const uint32_t a = tc & 1u;
            if (!ws_wait_warp(smem_addr(&accfull[a]), (tc >> 1) & 1u, &s_abort, err)) break;
            asm volatile("tcgen05.fence::after_thread_sync;\n" ::);
            const int j = j0 + 32 * qd + lane;
            const bool live = j < S->N;
            const uint32_t base = tmem + ((uint32_t)(32 * qd) << 16) + a * C::ACC_COLS + (uint32_t)cbase;
            if (SCALED) {
                // two limbs per chunk: both loads, then Y = 256 hi + lo (no prefetch: the registers of a
                // second chunk would spill)
#pragma unroll 1
                for (int c = 0; c < NCH; c++) {
                    uint32_t v[16], lo[16];
                    ws_ld16(base + (uint32_t)(16 * c), v);
                    ws_ld16(base + (uint32_t)(C::BN + 16 * c), lo);
                    asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
#pragma unroll
                    for (int e = 0; e < 16; e++) v[e] = (uint32_t)(int32_t)(256ll * (int32_t)v[e] + (int32_t)lo[e]);
                    const int i = i0 + cbase + 16 * c;
                    if (live && i < S->M) ws_store16(*S, j, i, v);
                }
            } else {
                uint32_t v[2][16];
                ws_ld16(base, v[0]);
                asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
#pragma unroll
                for (int c = 0; c < NCH; c++) {
                    const int cur = c & 1, nxt = cur ^ 1;
                    if (c + 1 < NCH) ws_ld16(base + (uint32_t)(16 * (c + 1)), v[nxt]);  // lands while chunk c is stored
                    const int i = i0 + cbase + 16 * c;
                    if (live && i < S->M) ws_store16(*S, j, i, v[cur]);
                    asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
                }
            }
            asm volatile("tcgen05.fence::before_thread_sync;\n" ::);
            ws_arrive(smem_addr(&accempty[a]));
        }
    }
    __syncwarp();
    asm volatile("tcgen05.fence::before_thread_sync;\n" ::);
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;\n" ::);
    if (warp == 1) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;\n" ::"r"(tmem));
}

template <bool W4, bool SCALED>
int launch_ws(fp_ctx* c, const std::vector<fp_site>& list, cudaStream_t st) {
    if (list.empty()) return FP_OK;
    using C = WsCfg<W4, SCALED>;
    std::vector<SiteWs> h(list.size());
    int64_t tiles = 0;
    double bytes = 0;
    for (size_t s = 0; s < list.size(); s++) {
        const fp_site& t = list[s];
        SiteWs& d = h[s];
        memset(&d, 0, sizeof d);
        const uint64_t pitch = W4 ? (uint64_t)t.K / 2 : (uint64_t)t.K;
        if (!fp_tmap_u8_2d(&d.tmA, t.xt, (uint64_t)t.K, (uint64_t)t.N, (uint64_t)t.K, WS_BK, WS_BM, true) ||
            !fp_tmap_u8_2d(&d.tmB, t.w, pitch, (uint64_t)t.M, pitch, W4 ? WS_BK / 2 : WS_BK, C::BN, !C::EXPAND))
            return fp_fail(c, FP_ERR_CUDA, "witness: tensor map encoding failed");
        d.scales = t.scales;
        d.q = t.q;
        d.r = t.r;
        d.y = t.y;
        d.M = t.M;
        d.K = t.K;
        d.N = t.N;
        d.k_shift = t.k_shift;
        d.G = (t.K + 63) / 64;
        d.tiles_i = (t.M + C::BN - 1) / C::BN;
        d.nk = (t.K + WS_BK - 1) / WS_BK;
        d.tile_base = tiles;
        tiles += (int64_t)d.tiles_i * ((t.N + WS_BM - 1) / WS_BM);
        bytes += (double)t.M * pitch + (double)t.N * t.K + 9.0 * t.M * t.N + (t.scales ? (double)t.M * d.G : 0.0);
    }
    // the tile schedule, {site, j0, i0, k-tiles} per tile in site order (a site's tiles sweep its
    // weight rows for one token block before the next, so a token block's Xt stays in L2)
    std::vector<int4> sch((size_t)tiles);
    for (size_t s = 0; s < h.size(); s++) {
        const SiteWs& d = h[s];
        const int64_t nt = (int64_t)d.tiles_i * ((d.N + WS_BM - 1) / WS_BM);
        for (int64_t lt = 0; lt < nt; lt++)
            sch[(size_t)(d.tile_base + lt)] =
                make_int4((int)s, (int)(lt / d.tiles_i) * WS_BM, (int)(lt % d.tiles_i) * C::BN, d.nk);
    }
    const size_t sz = sizeof(SiteWs) * h.size(), ssz = sizeof(int4) * sch.size();
    SiteWs* dsites = (SiteWs*)fp_alloc(c->dev, sz);
    int4* dsch = (int4*)fp_alloc(c->dev, ssz);
    char* hst = (char*)fp_alloc(c->host, sz + ssz);
    if (!dsites || !dsch || !hst) return fp_fail(c, FP_ERR_OOM, "witness: scratch exhausted");
    memcpy(hst, h.data(), sz);
    memcpy(hst + sz, sch.data(), ssz);
    FP_CUDA(c, cudaMemcpyAsync(dsites, hst, sz, cudaMemcpyHostToDevice, st));
    FP_CUDA(c, cudaMemcpyAsync(dsch, hst + sz, ssz, cudaMemcpyHostToDevice, st));
    auto kern = witness_ws_kernel<W4, SCALED>;
    FP_CUDA(c, cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM));
    const unsigned grid = (unsigned)std::min<int64_t>(tiles, (int64_t)c->num_sms);
    int slot;
    fp_tic(c, st, K_GEMM, bytes, &slot);
    kern<<<grid, C::THREADS, C::SMEM, st>>>(dsites, dsch, tiles, &c->mb_dev->err);
    fp_toc(c, st, slot);
    FP_CUDA(c, cudaGetLastError());
    return FP_OK;
}

}  // namespace

int fp_launch_witness(fp_ctx* c, const fp_site* sites, int nsites, cudaStream_t st) {
    // group sites by kernel variant: unscaled sites with 16-byte rows go to the tensor-core
    // (tcgen05) kernel, the rest to the mma.sync kernel
    std::vector<fp_site> v[8], tcv[2], wsv[4];
    for (int s = 0; s < nsites; s++) {
        const fp_site& t = sites[s];
        bool w4 = t.w_bits == 4, sc = t.scales != nullptr;
        size_t pitch = w4 ? (size_t)(t.K + 1) / 2 : (size_t)t.K;
        bool al = ((uintptr_t)t.w % 16 == 0) && ((uintptr_t)t.xt % 16 == 0) && (pitch % 16 == 0) &&
                  (t.K % 16 == 0) && (!w4 || t.K % 32 == 0);
        if (al && c->tc_gemm == 2)
            wsv[(w4 ? 2 : 0) + (sc ? 1 : 0)].push_back(t);
        else if (al && !sc && c->tc_gemm == 1)
            tcv[w4 ? 1 : 0].push_back(t);
        else
            v[(w4 ? 4 : 0) + (sc ? 2 : 0) + (al ? 1 : 0)].push_back(t);
    }
    size_t need = 0;
    for (int i = 0; i < 8; i++) need += fp_align_up(sizeof(SiteDev) * v[i].size(), 256) + 256;
    for (int i = 0; i < 2; i++) need += fp_align_up(sizeof(SiteDev) * tcv[i].size(), 256) + 256;
    for (int i = 0; i < 4; i++) {
        size_t tiles = 0;  // the schedule's entries, counted with 128-row tiles (an upper bound)
        for (const fp_site& t : wsv[i]) tiles += (size_t)((t.M + 127) / 128) * (size_t)((t.N + WS_BM - 1) / WS_BM);
        need += fp_align_up(sizeof(SiteWs) * wsv[i].size(), 256) + fp_align_up(sizeof(int4) * tiles, 256) + 512;
    }
    int rc = fp_reserve(c, c->dev, need + (1 << 20));
    if (rc) return rc;
    rc = fp_reserve(c, c->host, need + (1 << 20));
    if (rc) return rc;
    fp_reset(c->dev);
    fp_reset(c->host);
    if ((rc = launch_ws<false, false>(c, wsv[0], st))) return rc;
    if ((rc = launch_ws<false, true>(c, wsv[1], st))) return rc;
    if ((rc = launch_ws<true, false>(c, wsv[2], st))) return rc;
    if ((rc = launch_ws<true, true>(c, wsv[3], st))) return rc;
    if ((rc = launch_tc<false>(c, tcv[0], st))) return rc;
    if ((rc = launch_tc<true>(c, tcv[1], st))) return rc;
    if ((rc = launch_variant<false, false, false>(c, v[0], st))) return rc;
    if ((rc = launch_variant<false, false, true>(c, v[1], st))) return rc;
    if ((rc = launch_variant<false, true, false>(c, v[2], st))) return rc;
    if ((rc = launch_variant<false, true, true>(c, v[3], st))) return rc;
    if ((rc = launch_variant<true, false, false>(c, v[4], st))) return rc;
    if ((rc = launch_variant<true, false, true>(c, v[5], st))) return rc;
    if ((rc = launch_variant<true, true, false>(c, v[6], st))) return rc;
    if ((rc = launch_variant<true, true, true>(c, v[7], st))) return rc;
    return FP_OK;
}
