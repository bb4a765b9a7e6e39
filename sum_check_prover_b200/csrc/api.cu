// Context, errors, scratch arena, timing hooks, statement checks and the small
// entry points (digest, witness commitment, partial evaluation).
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <emmintrin.h>

#include <atomic>
#include <chrono>

#include "fp_internal.h"

int fp_version(void) { return 100; }

int fp_fail(fp_ctx* c, int code, const std::string& msg) {
    if (c) c->err = msg;
    return code;
}

int fp_cuda_check(fp_ctx* c, cudaError_t e, const char* what) {
    return fp_fail(c, FP_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

int fp_log2_ceil(uint64_t n) {
    int v = 0;
    while ((1ull << v) < n) v++;
    return v;
}

// ---------------------------------------------------------------------------
// context
// ---------------------------------------------------------------------------

// True when a kernel-replaying profiler has injected itself into this process
// (its injection libraries are mapped, or CUDA's injection hook is set).
static bool profiler_injected() {
    const char* inj = getenv("CUDA_INJECTION64_PATH");
    if (inj && inj[0]) return true;
    FILE* f = fopen("/proc/self/maps", "r");
    if (!f) return false;
    char line[1024];
    bool found = false;
    while (!found && fgets(line, sizeof line, f))
        found = strstr(line, "InjectionTarget") || strstr(line, "TreeLauncherTarget") || strstr(line, "cuda-injection");
    fclose(f);
    return found;
}

fp_ctx* fp_ctx_create(int device) {
    fp_ctx* c = new fp_ctx();
    c->device = device;
    if (cudaSetDevice(device) != cudaSuccess) {
        delete c;
        return nullptr;
    }
    cudaDeviceProp prop;
    if (cudaGetDeviceProperties(&prop, device) != cudaSuccess) {
        delete c;
        return nullptr;
    }
    c->num_sms = prop.multiProcessorCount;
    c->host.pinned_host = true;
    c->dig_host.pinned_host = true;
    if (cudaMalloc(&c->tickets, 4096) != cudaSuccess || cudaMemset(c->tickets, 0, 4096) != cudaSuccess ||
        cudaMalloc(&c->relay, sizeof(FpRelay)) != cudaSuccess ||
        cudaMemset(c->relay, 0, sizeof(FpRelay)) != cudaSuccess ||
        cudaHostAlloc((void**)&c->mb, sizeof(FpMailbox), cudaHostAllocMapped) != cudaSuccess ||
        cudaHostGetDevicePointer((void**)&c->mb_dev, c->mb, 0) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) {
        cudaGetLastError();
        if (c->tickets) cudaFree(c->tickets);
        if (c->relay) cudaFree(c->relay);
        if (c->mb) cudaFreeHost(c->mb);
        delete c;
        return nullptr;
    }
    memset((void*)c->mb, 0, sizeof(FpMailbox));
    // A profiler that replays kernels holds the host inside the launch call, so
    // a kernel that waits for the host's challenges could never be answered:
    // under an injected profiler (or FP_STEPPED=1) every round is its own launch.
    const char* st = getenv("FP_STEPPED");
    c->stepped_env = profiler_injected() || (st && st[0] == '1');
    c->stepped = c->stepped_env;
    // witness GEMM kernels: "0" the mma.sync kernel for every site, "1" the single-role tcgen05
    // kernel for unscaled sites; otherwise the warp-specialised tcgen05 kernel for every site whose
    // operands TMA can read
    const char* tg = getenv("FP_TCGEN05");
    c->tc_gemm = (tg && tg[0] == '0') ? 0 : (tg && tg[0] == '1') ? 1 : 2;
    return c;
}

void fp_ctx_destroy(fp_ctx* c) {
    if (!c) return;
    cudaSetDevice(c->device);
    cudaDeviceSynchronize();
    for (auto& p : c->ev_live) {
        cudaEventDestroy(p.a);
        cudaEventDestroy(p.b);
    }
    for (auto e : c->ev_free) cudaEventDestroy(e);
    if (c->ev_ref) cudaEventDestroy(c->ev_ref);
    if (c->dev.p) cudaFree(c->dev.p);
    if (c->dig.p) cudaFree(c->dig.p);
    if (c->host.p) cudaFreeHost(c->host.p);
    if (c->dig_host.p) cudaFreeHost(c->dig_host.p);
    if (c->tickets) cudaFree(c->tickets);
    if (c->relay) cudaFree(c->relay);
    if (c->mb) cudaFreeHost(c->mb);
    delete c;
}

// ---------------------------------------------------------------------------
// persistent-kernel handshake (host side)
// ---------------------------------------------------------------------------

uint64_t fp_seq_reserve(fp_ctx* c, uint64_t n) {
    uint64_t base = c->seq;
    c->seq += n;
    return base;
}

// Reset the relay before a persistent launch and clear stale mailbox errors.
int fp_session_begin(fp_ctx* c, cudaStream_t s) {
    c->mb->err = 0;
    c->t_result = -1;
    fp_session_expect(c, 0);
    FP_CUDA(c, cudaMemsetAsync(c->relay, 0, sizeof(FpRelay), s));
    return FP_OK;
}

// a failed wait: record the error, then let whatever is still resident run out
// (fp_session_abandon) so the next session starts from an empty mailbox
static int session_fail(fp_ctx* c, cudaStream_t s, int code, const char* msg) {
    const int rc = fp_fail(c, code, msg);
    fp_session_abandon(c, s);
    return rc;
}

int fp_session_wait(fp_ctx* c, uint64_t seq, cudaStream_t s) {
    (void)seq;
    const volatile FpMailbox* mb = c->mb;
    const int n = c->res_n;
    using clk = std::chrono::steady_clock;
    const auto t0 = clk::now();
    auto next_query = t0 + std::chrono::milliseconds(2);
    c->host_waits++;
    for (uint64_t spin = 0;; spin++) {
        bool full = true;
        for (int i = 0; i < n; i++) full = full && (mb->res[i] != kEmpty);
        if (full) {
            std::atomic_thread_fence(std::memory_order_acquire);
            const auto t1 = clk::now();
            c->host_wait_s += std::chrono::duration<double>(t1 - t0).count();
            c->t_result = std::chrono::duration<double>(t1.time_since_epoch()).count();
            return FP_OK;
        }
        if ((spin & 255) != 255) continue;
        if (mb->err) return session_fail(c, s, FP_ERR_TIMEOUT, "a persistent kernel stopped waiting for the host");
        const auto now = clk::now();
        if (now < next_query) continue;
        // the device may have failed: look at the stream every couple of milliseconds
        next_query = now + std::chrono::milliseconds(2);
        cudaError_t q = cudaStreamQuery(s);
        if (q != cudaErrorNotReady) {
            bool done = true;
            for (int i = 0; i < n; i++) done = done && (mb->res[i] != kEmpty);
            if (done) continue;
            if (q != cudaSuccess) {
                const int rc = fp_cuda_check(c, q, "persistent kernel");
                fp_session_abandon(c, s);
                return rc;
            }
            return session_fail(c, s, FP_ERR_TIMEOUT, "a persistent kernel ended without publishing");
        }
        if (std::chrono::duration<double>(now - t0).count() > 30.0)
            return session_fail(c, s, FP_ERR_TIMEOUT, "no answer from the device within 30 s");
    }
}

// Empty the n result slots the next publish will fill (before posting the challenge that triggers it).
void fp_session_expect(fp_ctx* c, int n) {
    volatile FpMailbox* mb = c->mb;
    for (int i = 0; i < 16; i++) mb->res[i] = kEmpty;
    c->res_n = n;
}

// Waits (bounded) for a challenge that is never posted, then reports it.
__global__ void session_selftest_kernel(FpMailbox* mb, FpRelay* rl, uint64_t seq, uint32_t limit) {
    uint64_t chal;
    if (session_wait(mb, rl, seq, chal, limit) && threadIdx.x == 0) session_publish(mb, &chal, 1, seq);
}

int fp_session_selftest(fp_ctx* c, void* stream) {
    if (!c) return FP_ERR_ARG;
    FP_CUDA(c, cudaSetDevice(c->device));
    cudaStream_t s = (cudaStream_t)stream;
    int rc = fp_session_begin(c, s);
    if (rc) return rc;
    const uint64_t seq = fp_seq_reserve(c, 1) + 1;  // nobody posts this challenge
    fp_session_expect(c, 1);
    // 2^20 polls: about a second before the kernel gives up
    session_selftest_kernel<<<2, 64, 0, s>>>(c->mb_dev, c->relay, seq, 1u << 20);
    FP_CUDA(c, cudaGetLastError());
    rc = fp_session_wait(c, seq, s);
    cudaError_t e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return fp_cuda_check(c, e, "session self-test");
    c->mb->err = 0;
    return rc;
}

// Answer with a challenge: the second value first, then {chal, seq} in one
// aligned 16-byte store, so the device's 16-byte read sees both or neither.
void fp_session_post2(fp_ctx* c, uint64_t seq, uint64_t chal, uint64_t chal2) {
    volatile FpMailbox* mb = c->mb;
    mb->chal2 = chal2;
    std::atomic_signal_fence(std::memory_order_seq_cst);
    _mm_store_si128((__m128i*)(&mb->chal), _mm_set_epi64x((long long)seq, (long long)chal));
    std::atomic_thread_fence(std::memory_order_release);
    if (c->t_result >= 0) {
        const double dt =
            std::chrono::duration<double>(std::chrono::steady_clock::now().time_since_epoch()).count() - c->t_result;
        c->host_turn_s += dt;
        if (dt > c->host_turn_max) c->host_turn_max = dt;
        c->t_result = -1;
    }
}

void fp_session_post(fp_ctx* c, uint64_t seq, uint64_t chal) { fp_session_post2(c, seq, chal, 0); }

// A session the host stops early (it refused a round's values) leaves its resident
// kernel waiting; after its bounded wait the kernel would flag the mailbox under the
// next session. Instead every later wait is answered at once (a sequence number above
// all, the challenge 0) so the kernel runs to its end; its results are ignored. Then the
// stream is drained and the mailbox returned to its empty state.
void fp_session_abandon(fp_ctx* c, cudaStream_t s) {
    if (!c) return;
    fp_session_expect(c, 0);
    fp_session_post2(c, ~0ull - 1, 0, 0);
    cudaStreamSynchronize(s);
    volatile FpMailbox* mb = c->mb;
    _mm_store_si128((__m128i*)(&mb->chal), _mm_set_epi64x(0, 0));  // no kernel runs on the stream now
    mb->chal2 = 0;
    mb->err = 0;
    c->t_result = -1;
}

const char* fp_last_error(const fp_ctx* c) { return c ? c->err.c_str() : "null context"; }

int fp_reserve(fp_ctx* c, FpArena& a, size_t bytes) {
    bytes = fp_align_up(bytes, 1 << 20);
    if (bytes <= a.cap) return FP_OK;
    FP_CUDA(c, cudaDeviceSynchronize());
    if (a.p) {
        if (a.pinned_host)
            cudaFreeHost(a.p);
        else
            cudaFree(a.p);
    }
    a.p = nullptr;
    a.cap = 0;
    a.top = 0;
    cudaError_t e = a.pinned_host ? cudaMallocHost((void**)&a.p, bytes) : cudaMalloc((void**)&a.p, bytes);
    if (e != cudaSuccess) {
        cudaGetLastError();
        a.p = nullptr;
        return fp_fail(c, FP_ERR_OOM, std::string(a.pinned_host ? "pinned host" : "device") +
                                          " scratch allocation of " + std::to_string(bytes) + " bytes failed");
    }
    a.cap = bytes;
    return FP_OK;
}

void* fp_alloc(FpArena& a, size_t bytes) {
    size_t off = fp_align_up(a.top, 256);
    if (off + bytes > a.cap) return nullptr;
    a.top = off + bytes;
    return a.p + off;
}

// ---------------------------------------------------------------------------
// timing hooks
// ---------------------------------------------------------------------------

static cudaEvent_t ev_get(fp_ctx* c) {
    if (!c->ev_free.empty()) {
        cudaEvent_t e = c->ev_free.back();
        c->ev_free.pop_back();
        return e;
    }
    cudaEvent_t e;
    cudaEventCreate(&e);
    return e;
}

void fp_tic(fp_ctx* c, cudaStream_t s, int kernel, double bytes, int* slot) {
    *slot = -1;
    c->launches++;
    if (!c->profiling) return;
    if (!c->ref_set) {
        if (!c->ev_ref) cudaEventCreate(&c->ev_ref);
        cudaEventRecord(c->ev_ref, s);
        c->ref_set = true;
    }
    FpEvPair p;
    p.a = ev_get(c);
    p.b = ev_get(c);
    p.kernel = kernel;
    p.bytes = bytes;
    cudaEventRecord(p.a, s);
    c->ev_live.push_back(p);
    *slot = (int)c->ev_live.size() - 1;
}

void fp_toc(fp_ctx* c, cudaStream_t s, int slot) {
    if (slot < 0) return;
    cudaEventRecord(c->ev_live[slot].b, s);
}

static void stats_resolve(fp_ctx* c) {
    for (auto& p : c->ev_live) {
        cudaEventSynchronize(p.b);
        float ms = 0.f, at = 0.f;
        cudaEventElapsedTime(&ms, p.a, p.b);
        cudaEventElapsedTime(&at, c->ev_ref, p.a);
        c->stats[p.kernel].launches += 1;
        c->stats[p.kernel].ms += ms;
        c->stats[p.kernel].bytes += p.bytes;
        c->log.push_back(fp_launch_rec{p.kernel, 0, (double)ms, p.bytes, (double)at});
        c->ev_free.push_back(p.a);
        c->ev_free.push_back(p.b);
    }
    c->ev_live.clear();
}

void fp_stats_reset(fp_ctx* c) {
    stats_resolve(c);
    for (auto& s : c->stats) s = FpKStat();
    c->log.clear();
}

int fp_ctx_set_profiling(fp_ctx* c, int on) {
    if (!c || on < 0 || on > 2) return FP_ERR_ARG;
    stats_resolve(c);
    // 1: every round is its own launch, timed alone; 2: launches as in production
    // (resident sum-check kernels, whose time then includes the host exchanges)
    c->profiling = on == 1 ? 1 : on == 2 ? 2 : 0;
    c->stepped = c->profiling == 1 || c->stepped_env;
    for (auto& s : c->stats) s = FpKStat();
    c->log.clear();
    c->ref_set = false;
    return FP_OK;
}

int64_t fp_ctx_launches(const fp_ctx* c) { return c ? c->launches : -1; }

int fp_host_stats(const fp_ctx* c, double out[2]) {
    if (!c || !out) return FP_ERR_ARG;
    out[0] = (double)c->host_waits;
    out[1] = c->host_wait_s;
    out[2] = c->host_turn_s;
    out[3] = c->host_turn_max;
    return FP_OK;
}

int fp_kernel_stats(fp_ctx* c, fp_kernel_stat* out, int cap) {
    if (!c || (cap > 0 && !out)) return FP_ERR_ARG;
    stats_resolve(c);
    int n = 0;
    for (int k = 0; k < K_COUNT; k++) {
        if (c->stats[k].launches == 0) continue;
        if (n < cap) {
            out[n].kernel = k;
            out[n].launches = c->stats[k].launches;
            out[n].ms = c->stats[k].ms;
            out[n].bytes = c->stats[k].bytes;
        }
        n++;
    }
    return n;
}

int64_t fp_kernel_log(fp_ctx* c, fp_launch_rec* out, int64_t cap) {
    if (!c || (cap > 0 && !out)) return FP_ERR_ARG;
    stats_resolve(c);
    const int64_t n = (int64_t)c->log.size();
    for (int64_t i = 0; i < n && i < cap; i++) out[i] = c->log[i];
    return n;
}

// the degree-3 polynomial through (i, g[i]), i = 0..3, at r: the next claim of a
// degree-3 sum-check round
uint64_t fp_lagrange4(const uint64_t g[4], uint64_t r) {
    static const uint64_t inv2 = gl_inv(2), inv6 = gl_inv(6);
    const uint64_t r1 = gl_sub(r, 1), r2 = gl_sub(r, 2), r3 = gl_sub(r, 3);
    // L0 = -(r-1)(r-2)(r-3)/6, L1 = r(r-2)(r-3)/2, L2 = -r(r-1)(r-3)/2, L3 = r(r-1)(r-2)/6
    const uint64_t l0 = gl_sub(0, gl_mul(gl_mul(gl_mul(r1, r2), r3), inv6));
    const uint64_t l1 = gl_mul(gl_mul(gl_mul(r, r2), r3), inv2);
    const uint64_t l2 = gl_sub(0, gl_mul(gl_mul(gl_mul(r, r1), r3), inv2));
    const uint64_t l3 = gl_mul(gl_mul(gl_mul(r, r1), r2), inv6);
    return gl_add(gl_add(gl_mul(g[0], l0), gl_mul(g[1], l1)), gl_add(gl_mul(g[2], l2), gl_mul(g[3], l3)));
}

const char* fp_kernel_name(int k) {
    static const char* names[K_COUNT] = {
        "witness_gemm", "digest_leaf", "digest_node", "digest_final", "eq_build", "partial_acc",
        "partial_fin", "claim", "sc_round", "sc_final", "hist", "keys_gather", "tree_leaf",
        "tree_up", "gkr_round", "gkr_final", "leaf_eval", "reduce", "had_claim", "had_round", "had_final",
        "silu_hist", "silu_tree", "silu_round", "silu_leaf", "had2_round", "had2_final",
        "lhi_hist", "lhi_column", "lhi_round", "lhi_final",
        "mm2_eq", "mm2_contract", "mm2_claim", "mm2_round", "mm2_final", "frv_u",
        "route_witness", "route_vectors", "route_open", "route_round", "route_final",
        "lhi2_column", "lhi2_round", "lhi2_final", "silu2_tree", "silu2_round", "silu2_leaf",
        "lu2_hist", "lu2_tree", "lu2_round", "lu2_leaf", "lhr_column", "lhr_round", "lhr_final", "dsp_claim",
        "dsp_vectors", "silu_inputs", "ffn_hidden", "scl_group"};
    return (k >= 0 && k < K_COUNT) ? names[k] : "?";
}

// ---------------------------------------------------------------------------
// statement checks
// ---------------------------------------------------------------------------

int fp_check_sites(fp_ctx* c, const fp_site* sites, int nsites, bool need_witness) {
    int rc = fp_check_shapes(c, sites, nsites);
    if (rc) return rc;
    for (int s = 0; s < nsites; s++) {
        const fp_site& t = sites[s];
        char buf[160];
        if (!t.w || !t.xt) {
            snprintf(buf, sizeof buf, "site %d: null operand", s);
            return fp_fail(c, FP_ERR_ARG, buf);
        }
        if (need_witness && (!t.q || !t.r || !t.y)) {
            snprintf(buf, sizeof buf, "site %d: null witness buffer", s);
            return fp_fail(c, FP_ERR_ARG, buf);
        }
    }
    return FP_OK;
}

int fp_check_shapes(fp_ctx* c, const fp_site* sites, int nsites) {
    if (!sites || nsites < 1) return fp_fail(c, FP_ERR_SHAPE, "need at least one site");
    for (int s = 0; s < nsites; s++) {
        const fp_site& t = sites[s];
        char buf[160];
        if (t.w_bits != 4 && t.w_bits != 8) {
            snprintf(buf, sizeof buf, "site %d: w_bits must be 4 or 8", s);
            return fp_fail(c, FP_ERR_ARG, buf);
        }
        if (t.M < 1 || t.N < 1 || t.K < 1 || t.M > (1 << 24) || t.N > (1 << 24) || t.K > (1 << 20)) {
            snprintf(buf, sizeof buf, "site %d: dims %d x %d x %d outside [1, 2^24] x [1, 2^20] x [1, 2^24]", s,
                     t.M, t.K, t.N);
            return fp_fail(c, FP_ERR_SHAPE, buf);
        }
        if (t.k_shift < 1 || t.k_shift > 20) {
            snprintf(buf, sizeof buf, "site %d: k_shift %d outside [1, 20]", s, t.k_shift);
            return fp_fail(c, FP_ERR_SHAPE, buf);
        }
        // worst-case |Y| < 2^31 keeps the int32 accumulation exact
        double wmax = (t.w_bits == 4 ? 8.0 : 128.0) * (t.scales ? 128.0 : 1.0);
        if (wmax * 128.0 * (double)t.K >= 2147483648.0) {
            snprintf(buf, sizeof buf, "site %d: K = %d can overflow the int32 accumulator", s, t.K);
            return fp_fail(c, FP_ERR_SHAPE, buf);
        }
    }
    return FP_OK;
}

// ---------------------------------------------------------------------------
// transcript entry points
// ---------------------------------------------------------------------------

fp_tx* fp_tx_create(uint64_t seed) {
    fp_tx* t = new fp_tx();
    uint8_t b[15];
    memcpy(b, "FPSC-v1", 7);
    for (int i = 0; i < 8; i++) b[7 + i] = (uint8_t)(seed >> (8 * i));
    FpSha256 h;
    h.update(b, 15);
    h.final(t->st);
    return t;
}

void fp_tx_destroy(fp_tx* t) { delete t; }

int fp_tx_absorb(fp_tx* t, const char* label, const void* data, size_t n) {
    if (!t || !label || (n && !data)) return FP_ERR_ARG;
    fp_tx_absorb_raw(t, label, data, n);
    return FP_OK;
}

int fp_tx_squeeze(fp_tx* t, const char* label, uint64_t* out, size_t n) {
    if (!t || !label || (n && !out)) return FP_ERR_ARG;
    for (size_t i = 0; i < n; i++) out[i] = fp_tx_squeeze_one(t, label);
    return FP_OK;
}

int fp_tx_state(const fp_tx* t, uint8_t out[32]) {
    if (!t || !out) return FP_ERR_ARG;
    memcpy(out, t->st, 32);
    return FP_OK;
}

// ---------------------------------------------------------------------------
// digest, witness, partial evaluation
// ---------------------------------------------------------------------------

int fp_digest(fp_ctx* c, const void* dev, size_t nbytes, uint8_t out[32], void* stream) {
    if (!c || !out || (nbytes && !dev)) return fp_fail(c, FP_ERR_ARG, "fp_digest: null argument");
    FP_CUDA(c, cudaSetDevice(c->device));
    FpDigestJob j{(const uint8_t*)dev, (uint64_t)nbytes};
    return fp_digest_many(c, &j, 1, out, (cudaStream_t)stream);
}

int fp_digests(fp_ctx* c, const void* const* devs, const size_t* nbytes, int n, uint8_t* out, void* stream) {
    if (!c || !devs || !nbytes || !out || n < 1) return fp_fail(c, FP_ERR_ARG, "fp_digests: null argument");
    std::vector<FpDigestJob> jobs((size_t)n);
    for (int i = 0; i < n; i++) {
        if (nbytes[i] && !devs[i]) return fp_fail(c, FP_ERR_ARG, "fp_digests: null buffer");
        jobs[i] = FpDigestJob{(const uint8_t*)devs[i], (uint64_t)nbytes[i]};
    }
    FP_CUDA(c, cudaSetDevice(c->device));
    return fp_digest_many(c, jobs.data(), n, out, (cudaStream_t)stream);
}

namespace {

// the witness and digests of sites[0, nsites): 192-byte site records into rec
int commit_records(fp_ctx* c, const fp_site* sites, int nsites, void* stream, std::vector<uint8_t>& rec) {
    int rc = fp_check_sites(c, sites, nsites, true);
    if (rc) return rc;
    FP_CUDA(c, cudaSetDevice(c->device));
    cudaStream_t s = (cudaStream_t)stream;
    fp_reset(c->dev);
    c->mb->err = 0;
    rc = fp_launch_witness(c, sites, nsites, s);
    if (rc) return rc;
    // digests: W and scales only where no offline digest is given
    std::vector<FpDigestJob> jobs;
    std::vector<int> where;  // job -> (site * 6 + slot)
    for (int i = 0; i < nsites; i++) {
        const fp_site& t = sites[i];
        uint64_t mn = (uint64_t)t.M * t.N;
        uint64_t wb = (uint64_t)t.M * (t.w_bits == 4 ? (uint64_t)((t.K + 1) / 2) : (uint64_t)t.K);
        uint64_t sb = t.scales ? (uint64_t)t.M * ((t.K + 63) / 64) : 0;
        if (!t.w_digest) {
            jobs.push_back({(const uint8_t*)t.w, wb});
            where.push_back(6 * i + 0);
            jobs.push_back({(const uint8_t*)t.scales, sb});
            where.push_back(6 * i + 1);
        }
        jobs.push_back({(const uint8_t*)t.xt, (uint64_t)t.N * t.K});
        where.push_back(6 * i + 2);
        jobs.push_back({(const uint8_t*)t.q, 4 * mn});
        where.push_back(6 * i + 3);
        jobs.push_back({(const uint8_t*)t.r, 4 * mn});
        where.push_back(6 * i + 4);
        jobs.push_back({(const uint8_t*)t.y, mn});
        where.push_back(6 * i + 5);
    }
    std::vector<uint8_t> dg(32 * jobs.size());
    rc = fp_digest_many(c, jobs.data(), (int)jobs.size(), dg.data(), s);
    if (rc) return rc;
    if (c->mb->err)  // the digests synchronised the stream
        return fp_fail(c, FP_ERR_TIMEOUT, "witness GEMM: a tensor-core completion wait ran out");
    rec.assign(192 * (size_t)nsites, 0);
    for (int i = 0; i < nsites; i++)
        if (sites[i].w_digest) memcpy(&rec[192 * i], sites[i].w_digest, 64);
    for (size_t j = 0; j < jobs.size(); j++) memcpy(&rec[32 * where[j]], &dg[32 * j], 32);
    return FP_OK;
}

}  // namespace

int fp_commit_witness(fp_ctx* c, fp_tx* tx, const fp_site* sites, int nsites, void* stream) {
    if (!c || !tx) return fp_fail(c, FP_ERR_ARG, "fp_commit_witness: null context or transcript");
    std::vector<uint8_t> rec;
    int rc = commit_records(c, sites, nsites, stream, rec);
    if (rc) return rc;
    for (int i = 0; i < nsites; i++) fp_tx_absorb_raw(tx, "site", &rec[192 * i], 192);
    return FP_OK;
}

int fp_commit_witness_shard(fp_ctx* c, fp_tx* tx, const fp_site* sites, int nsites, const fp_shard* shard,
                            void* stream) {
    if (!c || !tx || !shard) return fp_fail(c, FP_ERR_ARG, "fp_commit_witness_shard: null argument");
    FpShardView sh;
    int rc = fp_shard_view(c, shard, nsites, sh);
    if (rc) return rc;
    if ((rc = fp_check_shapes(c, sites, nsites))) return rc;
    const int lo = sh.lo[sh.rank], own = sh.lo[sh.rank + 1] - lo;
    std::vector<uint8_t> rec;
    if ((rc = commit_records(c, sites + lo, own, stream, rec))) return rc;
    std::vector<uint64_t> mine(24 * (size_t)own), all(24 * (size_t)nsites);
    memcpy(mine.data(), rec.data(), rec.size());
    if ((rc = fp_shard_gather(sh, mine.data(), 24, all.data())))
        return fp_fail(c, rc, "fp_commit_witness_shard: the all-gather failed");
    const uint8_t* b = (const uint8_t*)all.data();
    for (int i = 0; i < nsites; i++) fp_tx_absorb_raw(tx, "site", b + 192 * (size_t)i, 192);
    return FP_OK;
}

int mle_partial_eval(fp_ctx* c, const void* mat, int bits, const int8_t* scales, int rows, int cols,
                     const uint64_t* point, int npoint, uint64_t* out, void* stream) {
    if (!c || !mat || !out || (npoint && !point)) return fp_fail(c, FP_ERR_ARG, "mle_partial_eval: null argument");
    if (bits != 4 && bits != 8) return fp_fail(c, FP_ERR_ARG, "mle_partial_eval: bits must be 4 or 8");
    if (rows < 1 || cols < 1 || rows > (1 << 24) || cols > (1 << 24))
        return fp_fail(c, FP_ERR_SHAPE, "mle_partial_eval: dims outside [1, 2^24]");
    if (npoint != fp_log2_ceil((uint64_t)rows) || npoint > 32)
        return fp_fail(c, FP_ERR_SHAPE, "mle_partial_eval: npoint must be ceil(log2 rows)");
    for (int i = 0; i < npoint; i++)
        if (point[i] >= 0xFFFFFFFF00000001ull) return fp_fail(c, FP_ERR_ARG, "mle_partial_eval: point not canonical");
    FP_CUDA(c, cudaSetDevice(c->device));
    cudaStream_t s = (cudaStream_t)stream;
    FpPeJob job{mat, bits, scales, rows, cols, point, npoint, out, 1ll << fp_log2_ceil((uint64_t)cols)};
    int rc = fp_reserve(c, c->dev, fp_partial_scratch(c, &job, 1) + (1 << 16));
    if (rc) return rc;
    rc = fp_reserve(c, c->host, fp_partial_host_scratch(&job, 1) + (1 << 16));
    if (rc) return rc;
    fp_reset(c->dev);
    fp_reset(c->host);
    rc = fp_partial_many(c, &job, 1, s);
    if (rc) return rc;
    FP_CUDA(c, cudaStreamSynchronize(s));
    return FP_OK;
}

int fp_proof_size(const fp_site* sites, int nsites, size_t* mm, size_t* lu) {
    if (!sites || nsites < 1 || !mm || !lu) return FP_ERR_ARG;
    int n = 0;
    uint64_t nk = 0;
    for (int s = 0; s < nsites; s++) {
        if (sites[s].K < 1 || sites[s].M < 1 || sites[s].N < 1) return FP_ERR_SHAPE;
        int a = fp_log2_ceil((uint64_t)sites[s].K);
        if (a > n) n = a;
        nk += (uint64_t)sites[s].M * sites[s].N;
    }
    int v = fp_log2_ceil(nk);
    if (v < 1) v = 1;
    *mm = 8 * (size_t)nsites + 24 * (size_t)n + 16 * (size_t)nsites;
    size_t l = 4 * ((size_t)1 << sites[0].k_shift) + 4 * 65536 + 64 + 24;
    for (int d = 1; d < v; d++) l += 32 * (size_t)d + 64;
    *lu = l;
    return FP_OK;
}
