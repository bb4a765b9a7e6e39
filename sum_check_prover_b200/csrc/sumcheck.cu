// Matmul sum-check with claims batched by a random linear combination
// ("How fast can FlashProve go", 2 Background: sum-check reduces each
// polynomial operation to claims on committed values and weights; 2 and 2.1:
// claims are merged into one).
//
// Statement per site s: sum_k A_s[k] B_s[k] = c_s with A_s = W~_s(r_row, .),
// B_s = X~_s(., r_col), c_s = MLE of 2^k q + r at (r_row, r_col) ("How fast
// can FlashProve go", 3.1: 2^k g + r stands in for the unrounded product).
// The batched claim sum_s rho_s c_s is proven in n = max ceil(log2 K_s)
// rounds of the degree-2 polynomial g(X) = sum_s rho_s sum_b A_s(X,b) B_s(X,b).
//
// All rounds run in one resident cooperative launch (the handshake of
// fp_session.cuh): each round folds the previous round's vectors by the
// previous challenge (MSB binding) and evaluates g at 0 and 2 in the same pass
// (the host takes g(1) from the running claim); warp shuffles, a block tree and
// the last block to finish reduce the sums. One pair per thread.
#include <string.h>

#include <algorithm>
#include <map>
#include <vector>

#include "fp_internal.h"
#include "fp_reduce.cuh"
#include "fp_session.cuh"

namespace {

constexpr int SC_THREADS = 256;

struct ScArgs {
    uint64_t* A[2];  // ping-pong vectors; A[0], B[0] hold the partial evaluations (site stride 2^n)
    uint64_t* B[2];
    const uint64_t* rho;
    uint64_t* fin;   // 2 * nsites final values
    int nsites, n;
    int grid, per_block;
    uint64_t seq0;   // round t publishes seq0 + t and waits for challenge seq0 + t
    int t_begin, t_end;  // rounds run by this launch; t_end > n includes the final values
};

// All n rounds of the matmul sum-check, then the final values, in one launch.
// Round t pairs (b, b + half) of every site; from round 2 on the inputs are the
// previous round's vectors (length 4 half per site), folded by the previous
// challenge on the fly, the folded halves going to the other buffer.
template <bool MULTI>
__global__ void __launch_bounds__(SC_THREADS, 3) sc_session_kernel(ScArgs P, FpMailbox* mb, FpRelay* rl, uint64_t* part) {
    uint64_t rprev = 0;
    for (int t = P.t_begin; t <= P.n && t <= P.t_end; t++) {
        if (t > 1 && !session_wait(mb, rl, P.seq0 + t - 1, rprev)) return;
        const int logh = P.n - t;
        const int64_t half = 1ll << logh;
        const int64_t npairs = (int64_t)P.nsites * half;
        int64_t want = (npairs + P.per_block - 1) / P.per_block;
        const unsigned active = (unsigned)(want < 1 ? 1 : (want > P.grid ? P.grid : want));
        if (blockIdx.x >= active) return;
        const bool fold = t > 1;
        // ping-pong by round parity (selects, not a dynamic index into the parameter struct)
        const bool odd = t & 1;
        const uint64_t* Ain = (fold && odd) ? P.A[1] : P.A[0];
        const uint64_t* Bin = (fold && odd) ? P.B[1] : P.B[0];
        uint64_t* Aout = odd ? P.A[0] : P.A[1];
        uint64_t* Bout = odd ? P.B[0] : P.B[1];
        // each block takes a contiguous range of pairs (its threads stride through it, so
        // loads stay coalesced and a thread meets few site boundaries): products are
        // summed exactly per site and weighted by rho_s once per site
        const int64_t chunk = ((npairs + active - 1) / active + blockDim.x - 1) / blockDim.x * blockDim.x;
        const int64_t pbeg = (int64_t)blockIdx.x * chunk;
        const int64_t pend = pbeg + chunk < npairs ? pbeg + chunk : npairs;
        GlAcc s0, s2;               // current site's sums of A(0)B(0) and A(2)B(2)
        GlAcc w0, w2;               // rho-weighted sums over finished sites (MULTI)
        int64_t scur = -1;
        for (int64_t p = pbeg + threadIdx.x; p < pend; p += blockDim.x) {
            const int64_t s = p >> logh, b = p & (half - 1);
            if (MULTI && s != scur) {
                if (scur >= 0) {
                    const uint64_t rs = __ldg(P.rho + scur);
                    w0.mac(s0.value(), rs);
                    w2.mac(s2.value(), rs);
                    s0 = GlAcc();
                    s2 = GlAcc();
                }
                scur = s;
            }
            uint64_t a0, a1, b0, b1;
            if (fold) {
                const int64_t bi = s * 4 * half + b;
                a0 = gl_fold_fast(__ldcg(Ain + bi), __ldcg(Ain + bi + 2 * half), rprev);
                a1 = gl_fold_fast(__ldcg(Ain + bi + half), __ldcg(Ain + bi + 3 * half), rprev);
                b0 = gl_fold_fast(__ldcg(Bin + bi), __ldcg(Bin + bi + 2 * half), rprev);
                b1 = gl_fold_fast(__ldcg(Bin + bi + half), __ldcg(Bin + bi + 3 * half), rprev);
                const int64_t bo = s * 2 * half + b;
                Aout[bo] = a0;
                Aout[bo + half] = a1;
                Bout[bo] = b0;
                Bout[bo + half] = b1;
            } else {
                const int64_t bi = s * 2 * half + b;
                a0 = __ldcg(Ain + bi);
                a1 = __ldcg(Ain + bi + half);
                b0 = __ldcg(Bin + bi);
                b1 = __ldcg(Bin + bi + half);
            }
            // g(0) and g(2); the host takes g(1) from the running claim. The value at 2 only
            // feeds a product, so it may stay weakly reduced.
            const uint64_t a2 = gl_add(gl_sub(a1, a0), a1);
            const uint64_t b2 = gl_add(gl_sub(b1, b0), b1);
            s0.mac(a0, b0);
            s2.mac(a2, b2);
        }
        uint64_t acc[2];
        if (MULTI) {
            if (scur >= 0) {
                const uint64_t rs = __ldg(P.rho + scur);
                w0.mac(s0.value(), rs);
                w2.mac(s2.value(), rs);
            }
            acc[0] = w0.value();
            acc[1] = w2.value();
        } else {
            acc[0] = s0.value();
            acc[1] = s2.value();
        }
        bool last;
        if (active == 1) {
            block_sum_gl<2>(acc);
            last = true;
        } else {
            last = grid_sum_gl_n<2>(acc, part, &rl->ticket, active);
        }
        if (last && threadIdx.x == 0) session_publish(mb, acc, P.seq0 + t);
    }
    if (P.t_end <= P.n || blockIdx.x != 0) return;
    if (!session_wait(mb, rl, P.seq0 + P.n, rprev)) return;
    // the round-n vectors (length 2 per site) sit in A[0] when n == 1, else in the round's output buffer
    const uint64_t* Af = (P.n == 1 || (P.n & 1)) ? P.A[0] : P.A[1];
    const uint64_t* Bf = (P.n == 1 || (P.n & 1)) ? P.B[0] : P.B[1];
    for (int s = threadIdx.x; s < P.nsites; s += blockDim.x) {
        P.fin[2 * s] = gl_fold(__ldcg(Af + 2 * s), __ldcg(Af + 2 * s + 1), rprev);
        P.fin[2 * s + 1] = gl_fold(__ldcg(Bf + 2 * s), __ldcg(Bf + 2 * s + 1), rprev);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const uint64_t done = 0;
        session_publish(mb, &done, 1, P.seq0 + P.n + 1);
    }
}

// A_s(rho), B_s(rho): fold the length-2 vectors by the last challenge (len == 2),
// or copy them (n == 0, len == 1).
__global__ void sc_final_kernel(const uint64_t* A, const uint64_t* B, int nsites, int len, uint64_t r,
                                uint64_t* out) {
    int s = blockIdx.x * blockDim.x + threadIdx.x;
    if (s >= nsites) return;
    if (len == 2) {
        out[2 * s] = gl_fold(A[2 * s], A[2 * s + 1], r);
        out[2 * s + 1] = gl_fold(B[2 * s], B[2 * s + 1], r);
    } else {
        out[2 * s] = A[s];
        out[2 * s + 1] = B[s];
    }
}

}  // namespace

void put_u64s(uint8_t* p, const uint64_t* v, size_t n) {
    for (size_t i = 0; i < n; i++)
        for (int b = 0; b < 8; b++) p[8 * i + b] = (uint8_t)(v[i] >> (8 * b));
}

// ---- the host half ---------------------------------------------------------------
//
// The protocol is written once, over a source of device values, so that the
// one-GPU path, a statement whose sites are shared among several ranks (each
// rank proving its own sites and exchanging its partial sums through the
// caller's all-gather), and the callback driver of the tests run the same
// transcript steps.

namespace {

// Values of this rank's sites.
struct MmSource {
    virtual ~MmSource() {}
    virtual int start(const FpPoint& zr, const FpPoint& zc) = 0;  // eq tables, partial evaluations
    virtual int claims(uint64_t* out) = 0;                        // c_s of this rank's sites
    virtual int rounds(const uint64_t* rho) = 0;                  // this rank's rho_s; the rounds begin
    virtual int round(int t, uint64_t g02[2]) = 0;                // this rank's share of g_t(0), g_t(2)
    virtual int answer(int t, uint64_t r) = 0;                    // round t's challenge
    virtual int finals(uint64_t* out) = 0;                        // A_s(rho), B_s(rho) of this rank's sites
    virtual void abandon() {}
};

}  // namespace

// the ranks' `per` words for each of their own sites, gathered in site order
int fp_shard_gather(const FpShardView& sh, const uint64_t* mine, int per, uint64_t* all) {
    const int own = sh.lo[sh.rank + 1] - sh.lo[sh.rank];
    if (sh.world == 1) {
        memcpy(all, mine, 8 * (size_t)per * own);
        return FP_OK;
    }
    int most = 0;
    for (int r = 0; r < sh.world; r++) most = std::max(most, sh.lo[r + 1] - sh.lo[r]);
    const size_t slot = 8 * (size_t)per * std::max(1, most);
    std::vector<uint8_t> send(slot, 0), recv(slot * sh.world);
    memcpy(send.data(), mine, 8 * (size_t)per * own);
    if (sh.ag(sh.user, send.data(), slot, recv.data()) != 0) return FP_ERR_ARG;
    for (int r = 0; r < sh.world; r++)
        memcpy(all + (size_t)per * sh.lo[r], recv.data() + slot * r, 8 * (size_t)per * (sh.lo[r + 1] - sh.lo[r]));
    return FP_OK;
}

// the ranks' n words added mod p, in place
int fp_shard_sum(const FpShardView& sh, uint64_t* v, int n) {
    if (sh.world == 1) return FP_OK;
    std::vector<uint64_t> recv((size_t)n * sh.world);
    if (sh.ag(sh.user, v, 8 * (size_t)n, recv.data()) != 0) return FP_ERR_ARG;
    for (int i = 0; i < n; i++) {
        uint64_t a = 0;
        for (int r = 0; r < sh.world; r++) a = gl_add(a, recv[(size_t)r * n + i] % GL_P);
        v[i] = a;
    }
    return FP_OK;
}

int fp_shard_view(fp_ctx* c, const fp_shard* shard, int nsites, FpShardView& sh) {
    if (!shard) {
        sh.rank = 0;
        sh.world = 1;
        sh.lo = {0, nsites};
        sh.ag = nullptr;
        sh.user = nullptr;
        return FP_OK;
    }
    if (shard->world < 1 || shard->rank < 0 || shard->rank >= shard->world || !shard->site_lo ||
        (shard->world > 1 && !shard->allgather))
        return fp_fail(c, FP_ERR_ARG, "shard: bad rank, world, site ranges or all-gather");
    sh.rank = shard->rank;
    sh.world = shard->world;
    sh.lo.assign(shard->site_lo, shard->site_lo + shard->world + 1);
    if (sh.lo[0] != 0 || sh.lo[sh.world] != nsites) return fp_fail(c, FP_ERR_ARG, "shard: site ranges must cover the sites");
    for (int r = 0; r < sh.world; r++)
        if (sh.lo[r + 1] <= sh.lo[r]) return fp_fail(c, FP_ERR_ARG, "shard: every rank needs at least one site");
    sh.ag = shard->allgather;
    sh.user = shard->user;
    return FP_OK;
}

namespace {

int mm_protocol(fp_tx* tx, int vM, int vN, int n, int nsites, const FpShardView& sh, MmSource& src, uint8_t* proof,
                size_t* proof_len, FpMmPoint* pt_out = nullptr) {
    int rc;
    const int lo = sh.lo[sh.rank], own = sh.lo[sh.rank + 1] - lo;
    FpPoint zr, zc;
    zr.v = vM;
    zc.v = vN;
    for (int i = 0; i < vM; i++) zr.z[i] = fp_tx_squeeze_one(tx, "r_row");
    for (int i = 0; i < vN; i++) zc.z[i] = fp_tx_squeeze_one(tx, "r_col");
    if ((rc = src.start(zr, zc))) return rc;
    std::vector<uint64_t> chal;

    // claims of every site, in site order
    std::vector<uint64_t> mine(2 * (size_t)std::max(1, own)), all(2 * (size_t)nsites);
    if ((rc = src.claims(mine.data()))) return rc;
    if ((rc = fp_shard_gather(sh, mine.data(), 1, all.data()))) return rc;
    size_t pos = 0;
    put_u64s(proof + pos, all.data(), nsites);
    fp_tx_absorb_raw(tx, "claims", proof + pos, 8 * (size_t)nsites);
    pos += 8 * (size_t)nsites;
    std::vector<uint64_t> rho(nsites, 1);
    if (nsites > 1)
        for (int s = 0; s < nsites; s++) rho[s] = fp_tx_squeeze_one(tx, "rho");
    uint64_t claim = 0;  // sum_s rho_s c_s, then g_t(r_t) after each round
    for (int s = 0; s < nsites; s++) claim = gl_add(claim, gl_mul(rho[s], all[s]));
    if ((rc = src.rounds(rho.data() + lo))) return rc;

    static const uint64_t inv2 = gl_inv(2);
    for (int t = 1; t <= n; t++) {
        uint64_t g02[2];
        if ((rc = src.round(t, g02))) return rc;
        if ((rc = fp_shard_sum(sh, g02, 2))) {
            src.abandon();
            return rc;
        }
        // g(1) = claim - g(0); the next claim is g(r) (Lagrange on the nodes 0, 1, 2)
        uint64_t g[3] = {g02[0], gl_sub(claim, g02[0]), g02[1]};
        put_u64s(proof + pos, g, 3);
        fp_tx_absorb_raw(tx, "sc_round", proof + pos, 24);
        pos += 24;
        const uint64_t r = fp_tx_squeeze_one(tx, "sc_chal");
        chal.push_back(r);
        if ((rc = src.answer(t, r))) return rc;
        const uint64_t r1 = gl_sub(r, 1), r2 = gl_sub(r, 2);
        claim = gl_add(gl_add(gl_mul(g[0], gl_mul(gl_mul(r1, r2), inv2)), gl_sub(0, gl_mul(g[1], gl_mul(r, r2)))),
                       gl_mul(g[2], gl_mul(gl_mul(r, r1), inv2)));
    }
    if ((rc = src.finals(mine.data()))) return rc;
    if ((rc = fp_shard_gather(sh, mine.data(), 2, all.data()))) return rc;
    put_u64s(proof + pos, all.data(), 2 * (size_t)nsites);
    fp_tx_absorb_raw(tx, "sc_final", proof + pos, 16 * (size_t)nsites);
    pos += 16 * (size_t)nsites;
    *proof_len = pos;
    if (pt_out) {
        pt_out->r_row.assign(zr.z, zr.z + vM);
        pt_out->rho = chal;
        pt_out->fin = all;
        pt_out->valid = true;
    }
    return FP_OK;
}

// Device values: eq tables, claims, partial evaluations and the resident round kernel
// over this rank's sites (sites, nsites), with the statement's common n.
struct MmDevice : MmSource {
    fp_ctx* c;
    cudaStream_t st;
    const fp_site* sites;
    int nsites, n;
    int64_t L;
    std::vector<FpPeJob> pe;
    uint64_t *bufA[2], *bufB[2], *dclaims, *drho, *hrho, *hbuf, *part, *dfin;
    ScArgs P;
    const void* kern = nullptr;
    bool session = false;
    bool weighted = false;  // the statement has more than one site: every site's sums carry its rho_s

    int start(const FpPoint& zr, const FpPoint& zc) override {
        std::map<int, uint64_t*> eqr, eqc;  // eq tables by prefix length
        int rc;
        for (int s = 0; s < nsites; s++) {
            eqr[fp_log2_ceil((uint64_t)sites[s].M)] = nullptr;
            eqc[fp_log2_ceil((uint64_t)sites[s].N)] = nullptr;
        }
        for (auto& kv : eqr) {
            kv.second = (uint64_t*)fp_alloc(c->dev, (size_t)8 << kv.first);
            FpPoint p = zr;
            p.v = kv.first;
            if ((rc = fp_eq_table(c, p, kv.second, st))) return rc;
        }
        for (auto& kv : eqc) {
            kv.second = (uint64_t*)fp_alloc(c->dev, (size_t)8 << kv.first);
            FpPoint p = zc;
            p.v = kv.first;
            if ((rc = fp_eq_table(c, p, kv.second, st))) return rc;
        }
        std::vector<const uint64_t*> er(nsites), ec(nsites);
        for (int s = 0; s < nsites; s++) {
            er[s] = eqr[fp_log2_ceil((uint64_t)sites[s].M)];
            ec[s] = eqc[fp_log2_ceil((uint64_t)sites[s].N)];
        }
        dclaims = (uint64_t*)fp_alloc(c->dev, 8 * (size_t)nsites);
        if ((rc = fp_claims(c, sites, nsites, er.data(), ec.data(), dclaims, st))) return rc;
        // A_s = W~_s(r_row, .), B_s = X~_s(., r_col), one launch for all of them
        zrow = zr;
        zcol = zc;
        for (int s = 0; s < nsites; s++) {
            pe[2 * s].z = zrow.z;
            pe[2 * s].out = bufA[0] + (size_t)s * L;
            pe[2 * s + 1].z = zcol.z;
            pe[2 * s + 1].out = bufB[0] + (size_t)s * L;
        }
        return FP_OK;
    }
    FpPoint zrow, zcol;

    int claims(uint64_t* out) override {
        FP_CUDA(c, cudaMemcpyAsync(hbuf, dclaims, 8 * (size_t)nsites, cudaMemcpyDeviceToHost, st));
        FP_CUDA(c, cudaStreamSynchronize(st));
        memcpy(out, hbuf, 8 * (size_t)nsites);
        return FP_OK;
    }

    int rounds(const uint64_t* rho) override {
        memcpy(hrho, rho, 8 * (size_t)nsites);
        FP_CUDA(c, cudaMemcpyAsync(drho, hrho, 8 * (size_t)nsites, cudaMemcpyHostToDevice, st));
        int rc;
        if ((rc = fp_partial_many(c, pe.data(), (int)pe.size(), st))) return rc;
        if (n == 0) return FP_OK;
        int occ = 0;
        // a rank that holds one site of a larger statement still weights it by its rho_s
        kern = weighted ? (const void*)sc_session_kernel<true> : (const void*)sc_session_kernel<false>;
        FP_CUDA(c, cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, SC_THREADS, 0));
        P.A[0] = bufA[0];
        P.A[1] = bufA[1];
        P.B[0] = bufB[0];
        P.B[1] = bufB[1];
        P.rho = drho;
        P.fin = dfin;
        P.nsites = nsites;
        P.n = n;
        P.per_block = SC_THREADS;  // one pair per thread: small rounds spread over more blocks
        const int64_t want = ((int64_t)nsites * (L / 2) + P.per_block - 1) / P.per_block;
        P.grid = (int)std::max<int64_t>(1, std::min<int64_t>(want, (int64_t)std::max(1, occ) * c->num_sms));
        P.seq0 = fp_seq_reserve(c, n + 2);
        if ((rc = fp_session_begin(c, st))) return rc;
        session = true;
        fp_session_expect(c, 2);  // round 1 publishes without a challenge
        if (!c->stepped) {
            P.t_begin = 1;
            P.t_end = n + 1;
            // round 1 reads A, B (16 B per element); each later round reads 4 and writes 2 values of
            // both vectors per pair (96 B), over S L / 2^t pairs: 64 S L bytes in all
            return launch(dim3(P.grid), K_SC_ROUND, 64.0 * nsites * L);
        }
        return FP_OK;
    }

    int launch(dim3 grid, int kernel, double bytes) {
        void* args[] = {&P, &c->mb_dev, &c->relay, &part};
        int slot;
        fp_tic(c, st, kernel, bytes, &slot);
        FP_CUDA(c, cudaLaunchCooperativeKernel(kern, grid, dim3(SC_THREADS), args, 0, st));
        fp_toc(c, st, slot);
        return FP_OK;
    }

    int round(int t, uint64_t g02[2]) override {
        int rc;
        if (c->stepped) {
            P.t_begin = P.t_end = t;
            const double pairs = (double)nsites * (double)(1ll << (n - t));
            if ((rc = launch(dim3(P.grid), K_SC_ROUND, t == 1 ? 32.0 * pairs : 96.0 * pairs))) return rc;
        }
        if ((rc = fp_session_wait(c, P.seq0 + t, st))) return rc;
        g02[0] = c->mb->res[0];
        g02[1] = c->mb->res[1];
        return FP_OK;
    }

    int answer(int t, uint64_t r) override {
        fp_session_expect(c, t < n ? 2 : 1);  // the last challenge triggers the final values
        fp_session_post(c, P.seq0 + t, r);
        return FP_OK;
    }

    int finals(uint64_t* out) override {
        int rc;
        if (n > 0) {
            if (c->stepped) {
                P.t_begin = P.t_end = n + 1;
                if ((rc = launch(dim3(1), K_SC_FINAL, 32.0 * nsites))) return rc;
            }
            if ((rc = fp_session_wait(c, P.seq0 + n + 1, st))) return rc;
            session = false;
        } else {
            int slot;
            fp_tic(c, st, K_SC_FINAL, 32.0 * nsites, &slot);
            sc_final_kernel<<<(nsites + 127) / 128, 128, 0, st>>>(bufA[0], bufB[0], nsites, 1, 0, dfin);
            fp_toc(c, st, slot);
            FP_CUDA(c, cudaGetLastError());
        }
        FP_CUDA(c, cudaMemcpyAsync(hbuf, dfin, 16 * (size_t)nsites, cudaMemcpyDeviceToHost, st));
        FP_CUDA(c, cudaStreamSynchronize(st));
        memcpy(out, hbuf, 16 * (size_t)nsites);
        return FP_OK;
    }

    void abandon() override {
        if (session) fp_session_abandon(c, st);
        session = false;
    }
};

// scratch of this rank's sites and the device source over them
int mm_device_setup(fp_ctx* c, const fp_site* sites, int nsites, int n, cudaStream_t st, MmDevice& d) {
    const int64_t L = 1ll << n;
    std::map<int, int> lens_r, lens_c;
    for (int s = 0; s < nsites; s++) {
        lens_r[fp_log2_ceil((uint64_t)sites[s].M)] = 1;
        lens_c[fp_log2_ceil((uint64_t)sites[s].N)] = 1;
    }
    size_t need = 0;
    for (auto& kv : lens_r) need += fp_align_up((size_t)8 << kv.first, 256);
    for (auto& kv : lens_c) need += fp_align_up((size_t)8 << kv.first, 256);
    need += fp_claims_scratch(sites, nsites);
    const size_t vec = (size_t)8 * nsites * L;
    need += 4 * fp_align_up(vec, 256);
    // partial-evaluation jobs (points filled in once squeezed)
    d.pe.assign(2 * (size_t)nsites, FpPeJob{});
    for (int s = 0; s < nsites; s++) {
        d.pe[2 * s] = FpPeJob{sites[s].w, sites[s].w_bits, sites[s].scales, sites[s].M, sites[s].K, nullptr,
                              fp_log2_ceil((uint64_t)sites[s].M), nullptr, L};
        d.pe[2 * s + 1] = FpPeJob{sites[s].xt, 8, nullptr, sites[s].N, sites[s].K, nullptr,
                                  fp_log2_ceil((uint64_t)sites[s].N), nullptr, L};
    }
    need += fp_partial_scratch(c, d.pe.data(), (int)d.pe.size());
    need += fp_align_up((size_t)8 * 3 * 16 * c->num_sms, 256) + fp_align_up(8 * (size_t)nsites, 256) * 3 + (1 << 16);
    int rc;
    if ((rc = fp_reserve(c, c->dev, need))) return rc;
    if ((rc = fp_reserve(c, c->host, fp_align_up(sizeof(uint64_t) * (4 * (size_t)nsites + 64), 256) + 8192 +
                                         (size_t)160 * nsites + fp_partial_host_scratch(d.pe.data(), (int)d.pe.size()))))
        return rc;
    fp_reset(c->dev);
    fp_reset(c->host);
    d.c = c;
    d.st = st;
    d.sites = sites;
    d.nsites = nsites;
    d.n = n;
    d.L = L;
    memset(&d.P, 0, sizeof d.P);
    d.hbuf = (uint64_t*)fp_alloc(c->host, sizeof(uint64_t) * (4 * (size_t)nsites + 64));
    d.hrho = (uint64_t*)fp_alloc(c->host, 8 * (size_t)nsites);
    d.drho = (uint64_t*)fp_alloc(c->dev, 8 * (size_t)nsites);
    d.bufA[0] = (uint64_t*)fp_alloc(c->dev, vec);
    d.bufA[1] = (uint64_t*)fp_alloc(c->dev, vec);
    d.bufB[0] = (uint64_t*)fp_alloc(c->dev, vec);
    d.bufB[1] = (uint64_t*)fp_alloc(c->dev, vec);
    d.part = (uint64_t*)fp_alloc(c->dev, (size_t)8 * 3 * 16 * c->num_sms);
    d.dfin = (uint64_t*)fp_alloc(c->dev, 16 * (size_t)nsites);
    if (!d.hbuf || !d.hrho || !d.drho || !d.bufA[0] || !d.bufA[1] || !d.bufB[0] || !d.bufB[1] || !d.part || !d.dfin)
        return fp_fail(c, FP_ERR_OOM, "sumcheck: scratch exhausted");
    return FP_OK;
}

// the statement's dimensions over all its sites
void mm_dims(const fp_site* sites, int nsites, int& vM, int& vN, int& n) {
    vM = vN = n = 0;
    for (int s = 0; s < nsites; s++) {
        vM = std::max(vM, fp_log2_ceil((uint64_t)sites[s].M));
        vN = std::max(vN, fp_log2_ceil((uint64_t)sites[s].N));
        n = std::max(n, fp_log2_ceil((uint64_t)sites[s].K));
    }
}

// Values from the caller (the callback driver).
struct MmCallback : MmSource {
    fp_values_fn fn;
    void* user;
    int own, n;
    int start(const FpPoint& zr, const FpPoint& zc) override {
        std::vector<uint64_t> in(zr.v + zc.v + 1);
        for (int i = 0; i < zr.v; i++) in[i] = zr.z[i];
        for (int i = 0; i < zc.v; i++) in[zr.v + i] = zc.z[i];
        return fn(user, FP_VAL_START, zr.v + zc.v, in.data(), nullptr) ? FP_ERR_ARG : FP_OK;
    }
    int claims(uint64_t* out) override { return fn(user, FP_VAL_CLAIM, own, nullptr, out) ? FP_ERR_ARG : FP_OK; }
    int rounds(const uint64_t* rho) override {
        return fn(user, FP_VAL_WEIGHTS, own, rho, nullptr) ? FP_ERR_ARG : FP_OK;
    }
    int round(int t, uint64_t g02[2]) override { return fn(user, FP_VAL_ROUND, t, nullptr, g02) ? FP_ERR_ARG : FP_OK; }
    int answer(int t, uint64_t r) override { return fn(user, FP_VAL_ANSWER, t, &r, nullptr) ? FP_ERR_ARG : FP_OK; }
    int finals(uint64_t* out) override { return fn(user, FP_VAL_FINALS, own, nullptr, out) ? FP_ERR_ARG : FP_OK; }
};

int prove_matmul(fp_ctx* c, fp_tx* tx, const fp_site* sites, int nsites, const fp_shard* shard, uint8_t* proof,
                 size_t* proof_len, void* stream) {
    if (!c || !tx || !proof_len) return fp_fail(c, FP_ERR_ARG, "sumcheck_prove_matmul: null argument");
    FpShardView sh;
    int rc = fp_shard_view(c, shard, nsites, sh);
    if (rc) return rc;
    const int lo = sh.lo[sh.rank], own = sh.lo[sh.rank + 1] - lo;
    if (!sites || nsites < 1) return fp_fail(c, FP_ERR_SHAPE, "need at least one site");
    if ((rc = fp_check_shapes(c, sites, nsites))) return rc;
    if (own > 0 && (rc = fp_check_sites(c, sites + lo, own, true))) return rc;
    size_t mm_bytes, lu_bytes;
    fp_proof_size(sites, nsites, &mm_bytes, &lu_bytes);
    if (!proof || *proof_len < mm_bytes) {
        *proof_len = mm_bytes;
        return fp_fail(c, FP_ERR_ARG, "sumcheck_prove_matmul: proof buffer too small");
    }
    FP_CUDA(c, cudaSetDevice(c->device));
    int vM, vN, n;
    mm_dims(sites, nsites, vM, vN, n);
    MmDevice dev;
    if ((rc = mm_device_setup(c, sites + lo, own, n, (cudaStream_t)stream, dev))) return rc;
    dev.weighted = nsites > 1;
    c->mm_point.valid = false;
    rc = mm_protocol(tx, vM, vN, n, nsites, sh, dev, proof, proof_len, &c->mm_point);
    if (rc) dev.abandon();
    return rc;
}

}  // namespace

int sumcheck_prove_matmul(fp_ctx* c, fp_tx* tx, const fp_site* sites, int nsites, uint8_t* proof, size_t* proof_len,
                          void* stream) {
    return prove_matmul(c, tx, sites, nsites, nullptr, proof, proof_len, stream);
}

size_t fp_two_vector_scratch(const fp_ctx* c, int n) {
    const size_t vec = (size_t)8 << n;
    return 2 * fp_align_up(vec, 256) + fp_align_up((size_t)8 * 3 * 16 * c->num_sms, 256) + 3 * 256 + 4096;
}

size_t fp_two_vector_host_scratch() { return 3 * 256 + 8192; }

int fp_two_vector_sumcheck(fp_ctx* c, fp_tx* tx, uint64_t* A, uint64_t* B, int n, uint64_t claim, const char* lab_round,
                           const char* lab_chal, uint8_t* proof, size_t* pos, uint64_t fin[2], cudaStream_t st) {
    // the matmul rounds' device source with one site and no batching weight; A and B are the
    // site's vectors and are overwritten
    MmDevice d;
    d.c = c;
    d.st = st;
    d.sites = nullptr;
    d.nsites = 1;
    d.n = n;
    d.L = 1ll << n;
    memset(&d.P, 0, sizeof d.P);
    d.bufA[0] = A;
    d.bufB[0] = B;
    d.bufA[1] = (uint64_t*)fp_alloc(c->dev, (size_t)8 << n);
    d.bufB[1] = (uint64_t*)fp_alloc(c->dev, (size_t)8 << n);
    d.part = (uint64_t*)fp_alloc(c->dev, (size_t)8 * 3 * 16 * c->num_sms);
    d.dfin = (uint64_t*)fp_alloc(c->dev, 16);
    d.drho = (uint64_t*)fp_alloc(c->dev, 8);
    d.hrho = (uint64_t*)fp_alloc(c->host, 8);
    d.hbuf = (uint64_t*)fp_alloc(c->host, 8 * 64);
    if (!d.bufA[1] || !d.bufB[1] || !d.part || !d.dfin || !d.drho || !d.hrho || !d.hbuf)
        return fp_fail(c, FP_ERR_OOM, "two-vector sum-check: scratch exhausted");
    const uint64_t one = 1;
    int rc;
    if ((rc = d.rounds(&one))) return rc;
    static const uint64_t inv2 = gl_inv(2);
    for (int t = 1; t <= n; t++) {
        uint64_t g02[2];
        if ((rc = d.round(t, g02))) return rc;
        const uint64_t g[3] = {g02[0], gl_sub(claim, g02[0]), g02[1]};
        put_u64s(proof + *pos, g, 3);
        fp_tx_absorb_raw(tx, lab_round, proof + *pos, 24);
        *pos += 24;
        const uint64_t r = fp_tx_squeeze_one(tx, lab_chal);
        if ((rc = d.answer(t, r))) return rc;
        const uint64_t r1 = gl_sub(r, 1), r2 = gl_sub(r, 2);
        claim = gl_add(gl_add(gl_mul(g[0], gl_mul(gl_mul(r1, r2), inv2)), gl_sub(0, gl_mul(g[1], gl_mul(r, r2)))),
                       gl_mul(g[2], gl_mul(gl_mul(r, r1), inv2)));
    }
    return d.finals(fin);
}

int sumcheck_prove_matmul_shard(fp_ctx* c, fp_tx* tx, const fp_site* sites, int nsites, const fp_shard* shard,
                                uint8_t* proof, size_t* proof_len, void* stream) {
    if (!shard) return fp_fail(c, FP_ERR_ARG, "sumcheck_prove_matmul_shard: null shard");
    return prove_matmul(c, tx, sites, nsites, shard, proof, proof_len, stream);
}

int fp_mm_shard_protocol_drive(fp_tx* tx, const fp_site* sites, int nsites, const fp_shard* shard, fp_values_fn fn,
                               void* user, uint8_t* proof, size_t* proof_len) {
    if (!tx || !fn || !proof_len || !sites || nsites < 1) return FP_ERR_ARG;
    FpShardView sh;
    int rc = fp_shard_view(nullptr, shard, nsites, sh);
    if (rc) return rc;
    if ((rc = fp_check_shapes(nullptr, sites, nsites))) return rc;
    size_t mm_bytes, lu_bytes;
    fp_proof_size(sites, nsites, &mm_bytes, &lu_bytes);
    if (!proof || *proof_len < mm_bytes) {
        *proof_len = mm_bytes;
        return FP_ERR_ARG;
    }
    int vM, vN, n;
    mm_dims(sites, nsites, vM, vN, n);
    MmCallback cb;
    cb.fn = fn;
    cb.user = user;
    cb.own = sh.lo[sh.rank + 1] - sh.lo[sh.rank];
    cb.n = n;
    return mm_protocol(tx, vM, vN, n, nsites, sh, cb, proof, proof_len);
}

int sumcheck_last_point(fp_ctx* c, uint64_t* r_row, int cap_row, int* v_row, uint64_t* rho, int cap_rho, int* n) {
    if (!c || !v_row || !n) return FP_ERR_ARG;
    if (!c->mm_point.valid) return fp_fail(c, FP_ERR_ARG, "sumcheck_last_point: no matmul section proven yet");
    *v_row = (int)c->mm_point.r_row.size();
    *n = (int)c->mm_point.rho.size();
    if ((r_row && cap_row < *v_row) || (rho && cap_rho < *n)) return fp_fail(c, FP_ERR_ARG, "sumcheck_last_point: buffer too small");
    if (r_row) memcpy(r_row, c->mm_point.r_row.data(), 8 * (size_t)*v_row);
    if (rho) memcpy(rho, c->mm_point.rho.data(), 8 * (size_t)*n);
    return FP_OK;
}
