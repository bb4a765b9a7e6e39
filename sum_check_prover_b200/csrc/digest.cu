// Tree digest of device byte buffers, many buffers per launch.
//
// D(bytes) = SHA256(u64le(len) || T) where T is the root of a 32-ary tree:
// level 0 hashes every 1 KiB chunk (an empty buffer has one empty chunk),
// level l+1 hashes each run of up to 32 consecutive level-l digests.
// The digest binds committed buffers into the Fiat-Shamir transcript
// ("How fast can FlashProve go", 2 Background); the pages' Reed-Solomon and
// Merkle commitment itself is out of scope.
//
// Digests are kept between levels as eight 32-bit words h[0..7], which are
// exactly the big-endian message words of the next level.
#include <string.h>

#include <vector>

#include "fp_internal.h"

namespace {

constexpr uint32_t kChunk = 1024;

struct LevelDesc {
    const uint64_t* prefix;  // njobs + 1 exclusive prefix of node counts at this level
    const uint64_t* child;   // njobs + 1 prefix of node counts one level down (level >= 1)
    uint64_t base;           // word offset of this level in the scratch
    uint64_t child_base;     // word offset of the level below
};

__device__ __forceinline__ uint32_t bswap32(uint32_t x) { return __byte_perm(x, 0, 0x0123); }

__device__ __forceinline__ int find_job(const uint64_t* prefix, int njobs, uint64_t t) {
    int lo = 0, hi = njobs - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (prefix[mid] <= t)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

// SHA-256 of n <= 1024 bytes at p.
__device__ void sha_bytes(const uint8_t* p, uint32_t n, bool aligned16, uint32_t h[8]) {
    fp_sha_init(h);
    uint32_t nfull = n / 64;
    uint32_t m[16];
    if (aligned16 && nfull) {
        // the next block's loads are in flight while this block is compressed
        uint4 nx[4];
#pragma unroll
        for (int i = 0; i < 4; i++) nx[i] = __ldg(reinterpret_cast<const uint4*>(p) + i);
        for (uint32_t b = 0; b < nfull; b++) {
#pragma unroll
            for (int i = 0; i < 4; i++) {
                m[4 * i + 0] = bswap32(nx[i].x);
                m[4 * i + 1] = bswap32(nx[i].y);
                m[4 * i + 2] = bswap32(nx[i].z);
                m[4 * i + 3] = bswap32(nx[i].w);
            }
            if (b + 1 < nfull) {
#pragma unroll
                for (int i = 0; i < 4; i++) nx[i] = __ldg(reinterpret_cast<const uint4*>(p + 64 * (b + 1)) + i);
            }
            fp_sha_compress(h, m);
        }
    }
    for (uint32_t b = 0; b < nfull && !aligned16; b++) {
        const uint8_t* q = p + 64 * b;
        {
#pragma unroll
            for (int i = 0; i < 16; i++)
                m[i] = ((uint32_t)q[4 * i] << 24) | ((uint32_t)q[4 * i + 1] << 16) | ((uint32_t)q[4 * i + 2] << 8) |
                       (uint32_t)q[4 * i + 3];
        }
        fp_sha_compress(h, m);
    }
    // tail with padding: 0x80, zeros, 64-bit big-endian bit length
    uint32_t tail = n - 64 * nfull;
    const uint8_t* q = p + 64 * nfull;
    uint64_t bits = (uint64_t)n * 8;
    for (int pass = 0; pass < 2; pass++) {
#pragma unroll
        for (int i = 0; i < 16; i++) {
            uint32_t w = 0;
#pragma unroll
            for (int j = 0; j < 4; j++) {
                uint32_t idx = 64 * pass + 4 * i + j;
                uint32_t byte = 0;
                if (idx < tail)
                    byte = q[idx];
                else if (idx == tail)
                    byte = 0x80;
                w = (w << 8) | byte;
            }
            m[i] = w;
        }
        bool last = (pass == 0) ? (tail < 56) : true;
        if (last) {
            m[14] = (uint32_t)(bits >> 32);
            m[15] = (uint32_t)bits;
        }
        fp_sha_compress(h, m);
        if (last) break;
    }
}

// SHA-256 of nw (multiple of 8, <= 256) big-endian words.
__device__ void sha_words(const uint32_t* w, uint32_t nw, uint32_t h[8]) {
    fp_sha_init(h);
    uint32_t m[16];
    uint32_t nfull = nw / 16;
    uint32_t nx[16];
    if (nfull) {
#pragma unroll
        for (int i = 0; i < 16; i++) nx[i] = __ldcg(w + i);
    }
    for (uint32_t b = 0; b < nfull; b++) {
#pragma unroll
        for (int i = 0; i < 16; i++) m[i] = nx[i];
        if (b + 1 < nfull) {
#pragma unroll
            for (int i = 0; i < 16; i++) nx[i] = __ldcg(w + 16 * (b + 1) + i);
        }
        fp_sha_compress(h, m);
    }
    uint32_t tail = nw - 16 * nfull;  // 0 or 8
#pragma unroll
    for (int i = 0; i < 16; i++) m[i] = 0;
    for (uint32_t i = 0; i < tail; i++) m[i] = w[16 * nfull + i];
    m[tail] = 0x80000000u;
    uint64_t bits = (uint64_t)nw * 32;
    m[14] = (uint32_t)(bits >> 32);
    m[15] = (uint32_t)bits;
    fp_sha_compress(h, m);
}

__global__ void digest_leaf_kernel(const FpDigestJob* jobs, int njobs, LevelDesc L, uint32_t* scratch,
                                   uint64_t total) {
    uint64_t t = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= total) return;
    int j = find_job(L.prefix, njobs, t);
    uint64_t c = t - L.prefix[j];
    FpDigestJob jb = jobs[j];
    uint64_t off = c * kChunk;
    uint32_t n = 0;
    if (jb.len > off) n = (jb.len - off < kChunk) ? (uint32_t)(jb.len - off) : kChunk;
    const uint8_t* p = jb.ptr + off;
    bool al = ((reinterpret_cast<uintptr_t>(jb.ptr) & 15) == 0);
    uint32_t h[8];
    sha_bytes(p, n, al, h);
    uint32_t* o = scratch + L.base + 8 * t;
#pragma unroll
    for (int i = 0; i < 8; i++) o[i] = h[i];
}

__global__ void digest_node_kernel(int njobs, LevelDesc L, uint32_t* scratch, uint64_t total) {
    uint64_t t = (uint64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= total) return;
    int j = find_job(L.prefix, njobs, t);
    uint64_t node = t - L.prefix[j];
    uint64_t nchild = L.child[j + 1] - L.child[j];
    uint64_t first = 32 * node;
    uint32_t m = (uint32_t)((nchild - first) < 32 ? (nchild - first) : 32);
    const uint32_t* w = scratch + L.child_base + 8 * (L.child[j] + first);
    uint32_t h[8];
    sha_words(w, 8 * m, h);
    uint32_t* o = scratch + L.base + 8 * t;
#pragma unroll
    for (int i = 0; i < 8; i++) o[i] = h[i];
}

__global__ void digest_final_kernel(const FpDigestJob* jobs, int njobs, const uint64_t* top, const uint32_t* scratch,
                                    uint32_t* out) {
    int j = blockIdx.x * blockDim.x + threadIdx.x;
    if (j >= njobs) return;
    uint64_t len = jobs[j].len;
    uint32_t m[16];
    uint32_t b[8];
    for (int i = 0; i < 8; i++) b[i] = (uint32_t)(len >> (8 * i)) & 0xFF;  // u64le bytes
    m[0] = (b[0] << 24) | (b[1] << 16) | (b[2] << 8) | b[3];
    m[1] = (b[4] << 24) | (b[5] << 16) | (b[6] << 8) | b[7];
    const uint32_t* d = scratch + top[j];
    for (int i = 0; i < 8; i++) m[2 + i] = d[i];
    m[10] = 0x80000000u;
    m[11] = m[12] = m[13] = m[14] = 0;
    m[15] = 40 * 8;
    uint32_t h[8];
    fp_sha_init(h);
    fp_sha_compress(h, m);
    for (int i = 0; i < 8; i++) out[8 * j + i] = h[i];
}

}  // namespace

int fp_digest_many(fp_ctx* c, const FpDigestJob* jobs, int njobs, uint8_t* out, cudaStream_t s) {
    if (njobs <= 0) return FP_OK;
    // node counts per level
    std::vector<std::vector<uint64_t>> cnt;
    std::vector<uint64_t> c0(njobs);
    for (int j = 0; j < njobs; j++) c0[j] = jobs[j].len == 0 ? 1 : (jobs[j].len + kChunk - 1) / kChunk;
    cnt.push_back(c0);
    while (true) {
        bool more = false;
        std::vector<uint64_t> nx(njobs, 0);
        for (int j = 0; j < njobs; j++) {
            uint64_t prev = cnt.back()[j];
            if (prev > 1) {
                nx[j] = (prev + 31) / 32;
                more = true;
            }
        }
        if (!more) break;
        cnt.push_back(nx);
    }
    int nlev = (int)cnt.size();
    // prefixes, bases, top offsets
    std::vector<uint64_t> pref((size_t)nlev * (njobs + 1));
    std::vector<uint64_t> base(nlev);
    uint64_t words = 0;
    for (int l = 0; l < nlev; l++) {
        uint64_t acc = 0;
        for (int j = 0; j < njobs; j++) {
            pref[(size_t)l * (njobs + 1) + j] = acc;
            acc += cnt[l][j];
        }
        pref[(size_t)l * (njobs + 1) + njobs] = acc;
        base[l] = words;
        words += 8 * acc;
    }
    std::vector<uint64_t> top(njobs);
    for (int j = 0; j < njobs; j++) {
        int l = 0;
        while (l + 1 < nlev && cnt[l + 1][j] > 0) l++;
        top[j] = base[l] + 8 * pref[(size_t)l * (njobs + 1) + j];
    }
    size_t bytes_jobs = sizeof(FpDigestJob) * njobs;
    size_t bytes_pref = sizeof(uint64_t) * pref.size();
    size_t bytes_top = sizeof(uint64_t) * njobs;
    size_t meta = fp_align_up(bytes_jobs, 256) + fp_align_up(bytes_pref, 256) + fp_align_up(bytes_top, 256);
    size_t need = meta + fp_align_up(4 * words, 256) + fp_align_up(32 * (size_t)njobs, 256) + 4096;
    int rc = fp_reserve(c, c->dig, need);
    if (rc) return rc;
    rc = fp_reserve(c, c->dig_host, meta + 32 * (size_t)njobs + 4096);
    if (rc) return rc;
    fp_reset(c->dig);
    fp_reset(c->dig_host);
    char* dmeta = (char*)fp_alloc(c->dig, meta);
    uint32_t* scratch = (uint32_t*)fp_alloc(c->dig, 4 * words);
    uint32_t* dout = (uint32_t*)fp_alloc(c->dig, 32 * (size_t)njobs);
    // metadata goes through pinned staging; the stream is synchronised below
    // before the staging area can be reused
    char* h = c->dig_host.p;
    memcpy(h, jobs, bytes_jobs);
    memcpy(h + fp_align_up(bytes_jobs, 256), pref.data(), bytes_pref);
    memcpy(h + fp_align_up(bytes_jobs, 256) + fp_align_up(bytes_pref, 256), top.data(), bytes_top);
    FP_CUDA(c, cudaMemcpyAsync(dmeta, h, meta, cudaMemcpyHostToDevice, s));
    const FpDigestJob* djobs = (const FpDigestJob*)dmeta;
    const uint64_t* dpref = (const uint64_t*)(dmeta + fp_align_up(bytes_jobs, 256));
    const uint64_t* dtop = (const uint64_t*)(dmeta + fp_align_up(bytes_jobs, 256) + fp_align_up(bytes_pref, 256));

    for (int l = 0; l < nlev; l++) {
        uint64_t total = pref[(size_t)l * (njobs + 1) + njobs];
        if (total == 0) continue;
        LevelDesc L;
        L.prefix = dpref + (size_t)l * (njobs + 1);
        L.child = l ? dpref + (size_t)(l - 1) * (njobs + 1) : nullptr;
        L.base = base[l];
        L.child_base = l ? base[l - 1] : 0;
        int threads = 128;
        unsigned blocks = (unsigned)((total + threads - 1) / threads);
        int slot;
        if (l == 0) {
            double bytes = 0;
            for (int j = 0; j < njobs; j++) bytes += (double)jobs[j].len;
            fp_tic(c, s, K_DIGEST_LEAF, bytes + 32.0 * total, &slot);
            digest_leaf_kernel<<<blocks, threads, 0, s>>>(djobs, njobs, L, scratch, total);
        } else {
            fp_tic(c, s, K_DIGEST_NODE, 32.0 * (total + pref[(size_t)(l - 1) * (njobs + 1) + njobs]), &slot);
            digest_node_kernel<<<blocks, threads, 0, s>>>(njobs, L, scratch, total);
        }
        fp_toc(c, s, slot);
        FP_CUDA(c, cudaGetLastError());
    }
    int slot;
    fp_tic(c, s, K_DIGEST_FINAL, 64.0 * njobs, &slot);
    digest_final_kernel<<<(njobs + 127) / 128, 128, 0, s>>>(djobs, njobs, dtop, scratch, dout);
    fp_toc(c, s, slot);
    FP_CUDA(c, cudaGetLastError());
    uint32_t* hout = (uint32_t*)(h + meta);
    FP_CUDA(c, cudaMemcpyAsync(hout, dout, 32 * (size_t)njobs, cudaMemcpyDeviceToHost, s));
    FP_CUDA(c, cudaStreamSynchronize(s));
    for (int j = 0; j < njobs; j++)
        for (int i = 0; i < 8; i++) {
            uint32_t w = hout[8 * j + i];
            out[32 * j + 4 * i + 0] = (uint8_t)(w >> 24);
            out[32 * j + 4 * i + 1] = (uint8_t)(w >> 16);
            out[32 * j + 4 * i + 2] = (uint8_t)(w >> 8);
            out[32 * j + 4 * i + 3] = (uint8_t)w;
        }
    return FP_OK;
}
