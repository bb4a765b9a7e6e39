// Internal declarations shared by the library's translation units.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include <string>
#include <vector>

#include "../../include/fp.h"
#include "fp_session.cuh"
#include "fp_sha256.cuh"

// ---------------------------------------------------------------------------
// kernels known to the per-kernel timing table
// ---------------------------------------------------------------------------
enum FpKernel {
    K_GEMM = 0,
    K_DIGEST_LEAF,
    K_DIGEST_NODE,
    K_DIGEST_FINAL,
    K_EQ_BUILD,
    K_PARTIAL_ACC,
    K_PARTIAL_FIN,
    K_CLAIM,
    K_SC_ROUND,
    K_SC_FINAL,
    K_HIST,
    K_KEYS_GATHER,
    K_TREE_LEAF,
    K_TREE_UP,
    K_GKR_ROUND,
    K_GKR_FINAL,
    K_LEAF_EVAL,
    K_REDUCE,
    K_HAD_CLAIM,
    K_HAD_ROUND,
    K_HAD_FINAL,
    K_SILU_HIST,
    K_SILU_TREE,
    K_SILU_ROUND,
    K_SILU_LEAF,
    K_HAD2_ROUND,
    K_HAD2_FINAL,
    K_LHI_HIST,
    K_LHI_COLUMN,
    K_LHI_ROUND,
    K_LHI_FINAL,
    K_MM2_EQ,
    K_MM2_CONTRACT,
    K_MM2_CLAIM,
    K_MM2_ROUND,
    K_MM2_FINAL,
    K_FRV_U,
    K_ROUTE_WITNESS,
    K_ROUTE_VECTORS,
    K_ROUTE_OPEN,
    K_ROUTE_ROUND,
    K_ROUTE_FINAL,
    K_LHI2_COLUMN,
    K_LHI2_ROUND,
    K_LHI2_FINAL,
    K_X16_TREE,
    K_X16_ROUND,
    K_X16_LEAF,
    K_LU2_HIST,
    K_LU2_TREE,
    K_LU2_ROUND,
    K_LU2_LEAF,
    K_LHR_COLUMN,
    K_LHR_ROUND,
    K_LHR_FINAL,
    K_DSP_CLAIM,
    K_DSP_VECTORS,
    K_SILU_INPUTS,
    K_FFN_HIDDEN,
    K_SCL_GROUP,
    K_COUNT
};

struct FpKStat {
    int launches = 0;
    double ms = 0.0;
    double bytes = 0.0;
};

// a pair of events around one launch, resolved lazily
struct FpEvPair {
    cudaEvent_t a, b;
    int kernel;
    double bytes;
};

// A growable block carved by a bump allocator. Growing it frees the old block,
// so every entry point reserves what it needs before handing out pointers.
struct FpArena {
    char* p = nullptr;
    size_t cap = 0;
    size_t top = 0;
    bool pinned_host = false;
};

// where the last single-GPU matmul section left its sites: the row challenges, the round
// challenges and the final values A_s(rho), B_s(rho)
struct FpMmPoint {
    bool valid = false;
    std::vector<uint64_t> r_row, rho, fin;
};

struct fp_ctx {
    int device = 0;
    int num_sms = 148;
    std::string err;
    FpArena dev;       // device scratch of the current entry point
    FpArena dig;       // device scratch of the digest kernels (independent of dev)
    FpArena host;      // pinned host staging of the current entry point
    FpArena dig_host;  // pinned host staging of the digest path
    // small persistent device block: reduction tickets (kept zero between launches)
    unsigned int* tickets = nullptr;
    // persistent-kernel handshake: mailbox in mapped pinned host memory, relay on the device
    FpMailbox* mb = nullptr;      // host view
    FpMailbox* mb_dev = nullptr;  // device view of the same memory
    FpRelay* relay = nullptr;
    uint64_t seq = 1;             // next sequence number to hand out (the empty mailbox holds 0)
    int res_n = 0;                // result slots the next publish fills
    // stepped: launch the sum-check kernels once per round instead of once per
    // sum-check (under a kernel-replaying profiler, and while profiling)
    int stepped = 0;
    int stepped_env = 0;
    // witness GEMM kernels: 2 warp-specialised tcgen05 (default), 1 single-role tcgen05 for
    // unscaled sites, 0 mma.sync (FP_TCGEN05 selects 0 or 1)
    int tc_gemm = 2;
    FpMmPoint mm_point;
    // timing
    int profiling = 0;
    int64_t launches = 0;  // every kernel launch of the library on this context
    int64_t host_waits = 0;   // host waits for a device result (sum-check rounds)
    double host_wait_s = 0;   // host seconds spent in those waits
    double host_turn_s = 0;   // host seconds from a result's arrival to the next posted challenge
    double host_turn_max = 0;
    double t_result = -1;     // arrival time of the last result (steady clock seconds), -1: none pending
    std::vector<FpEvPair> ev_live;
    std::vector<cudaEvent_t> ev_free;
    cudaEvent_t ev_ref = nullptr;  // recorded before the first timed launch since profiling was set
    bool ref_set = false;
    FpKStat stats[K_COUNT];
    std::vector<fp_launch_rec> log;  // every timed launch since profiling was switched on
};

struct fp_tx {
    uint8_t st[32];
};

// ---- helpers (api.cu) ------------------------------------------------------
int fp_fail(fp_ctx* c, int code, const std::string& msg);
int fp_cuda_check(fp_ctx* c, cudaError_t e, const char* what);
#define FP_CUDA(c, call)                                  \
    do {                                                  \
        cudaError_t e__ = (call);                         \
        if (e__ != cudaSuccess) return fp_cuda_check(c, e__, #call); \
    } while (0)

// arenas: reserve (may reallocate, contents and pointers lost), then alloc
// 256-byte aligned blocks; reset at the start of every public call.
int fp_reserve(fp_ctx* c, FpArena& a, size_t bytes);
void* fp_alloc(FpArena& a, size_t bytes);
static inline void fp_reset(FpArena& a) { a.top = 0; }

// timing hooks around a launch (no-ops unless profiling)
void fp_tic(fp_ctx* c, cudaStream_t s, int kernel, double bytes, int* slot);
void fp_toc(fp_ctx* c, cudaStream_t s, int slot);
void fp_stats_reset(fp_ctx* c);

// persistent-kernel handshake (api.cu). seq_reserve hands out n consecutive
// sequence numbers and returns the base; wait blocks until the device published
// seq (bounded: FP_ERR_TIMEOUT, FP_ERR_CUDA if the kernel died); post answers
// with a challenge.
uint64_t fp_seq_reserve(fp_ctx* c, uint64_t n);
int fp_session_wait(fp_ctx* c, uint64_t seq, cudaStream_t s);
void fp_session_post(fp_ctx* c, uint64_t seq, uint64_t chal);
void fp_session_expect(fp_ctx* c, int n);
void fp_session_post2(fp_ctx* c, uint64_t seq, uint64_t chal, uint64_t chal2);
int fp_session_begin(fp_ctx* c, cudaStream_t s);
// Let a resident kernel of a session the host stopped early run to its end, and clear the mailbox.
void fp_session_abandon(fp_ctx* c, cudaStream_t s);

// transcript (transcript.cu)
void fp_tx_absorb_raw(fp_tx* t, const char* label, const void* data, uint64_t n);
uint64_t fp_tx_squeeze_one(fp_tx* t, const char* label);

// statement checks shared by the entry points (api.cu)
int fp_check_sites(fp_ctx* c, const fp_site* sites, int nsites, bool need_witness);
int fp_log2_ceil(uint64_t n);

// digests of device buffers (digest.cu): out is host, 32 bytes per job
struct FpDigestJob {
    const uint8_t* ptr;
    uint64_t len;
};
int fp_digest_many(fp_ctx* c, const FpDigestJob* jobs, int njobs, uint8_t* out, cudaStream_t s);
// D(W) || D(S) || D(Xt) || D(q) || D(r) of one site (D(W) || D(S) from w_digest when given;
// matmul_ext.cu); synchronises the stream
int fp_site_digest160(fp_ctx* c, const fp_site& s, uint8_t d[160], cudaStream_t st);

// witness (witness.cu)
int fp_launch_witness(fp_ctx* c, const fp_site* sites, int nsites, cudaStream_t s);

// MLE building blocks (mle.cu)
struct FpPoint {
    uint64_t z[32];
    int v;
};
int fp_eq_table(fp_ctx* c, const FpPoint& z, uint64_t* out, cudaStream_t s);
// out[c] = sum_{i<rows} eq[i] M_eff[i][c]; eq device (rows entries); out device (cols_pad)
// Row contractions out[c] = sum_{i<rows} eq(z, i) M_eff[i][c], many per launch
// (partial.cu). z is host memory (v = ceil(log2 rows) coordinates); out is
// device memory with out_len >= cols entries, the ones past cols zeroed.
// out[c] = sum_i w_i M_eff[i][c]: w_i = eq(z, i) for the point z (v coordinates, host), or, when
// wts is set, w_i = wts[i * wts_stride] (device, canonical; z and v unused)
struct FpPeJob {
    const void* mat;
    int bits;
    const int8_t* scales;
    int rows, cols;
    const uint64_t* z;
    int v;
    uint64_t* out;
    int64_t out_len;
    const uint64_t* wts = nullptr;
    int wts_stride = 1;
};
size_t fp_partial_scratch(const fp_ctx* c, const FpPeJob* jobs, int njobs);
size_t fp_partial_host_scratch(const FpPeJob* jobs, int njobs);
int fp_partial_many(fp_ctx* c, const FpPeJob* jobs, int njobs, cudaStream_t s);
size_t fp_claims_scratch(const fp_site* sites, int nsites);
// per-site output claims into dev_out[s]
// A statement's sites shared among ranks: rank r proves sites [lo[r], lo[r + 1]);
// small values are exchanged through the caller's all-gather.
struct FpShardView {
    int rank = 0, world = 1;
    std::vector<int> lo;
    fp_allgather_fn ag = nullptr;
    void* user = nullptr;
};
int fp_shard_view(fp_ctx* c, const fp_shard* shard, int nsites, FpShardView& sh);  // NULL: one rank
// every rank's `per` words for each of its own sites, in site order (all: nsites * per words)
int fp_shard_gather(const FpShardView& sh, const uint64_t* mine, int per, uint64_t* all);
// the ranks' n words added mod p, in place
int fp_shard_sum(const FpShardView& sh, uint64_t* v, int n);
// The lookup keys: every site's outputs in storage order, concatenated; indices
// in [n, 2^v) are the neutral key (r, q, y) = 0.
// A 2-D byte tensor (rows of `inner` bytes, `pitch` bytes apart) as a TMA tensor map (128 bytes at
// `tmap`, 64-byte aligned): boxes of box_inner x box_rows, zero fill outside, optional 128-byte
// swizzle. False if the driver's encoder is unavailable or rejects the shape.
bool fp_tmap_u8_2d(void* tmap, const void* base, uint64_t inner, uint64_t rows, uint64_t pitch, uint32_t box_inner,
                   uint32_t box_rows, bool swizzle128);

struct FpKeyCols {
    const int32_t* r;
    const int32_t* q;
    const int8_t* y;
    int64_t n;
};
// the key columns (the single site's own buffers, or a copy gathered into c->dev)
size_t fp_lookup_keys_scratch(int nsites, int64_t nk);
int fp_lookup_keys(fp_ctx* c, const fp_site* sites, int nsites, cudaStream_t st, FpKeyCols* K);
// multiplicities of both tables over the keys padded to L (device, c->dev), copied to
// hm (host: 2^k u32, 2^16 u32, the count of keys outside the tables) with their digests
size_t fp_lookup_mults_scratch(int k);
int fp_lookup_mults(fp_ctx* c, const FpKeyCols& K, int k, int64_t L, cudaStream_t st, uint8_t* hm, uint8_t dg_rem[32],
                    uint8_t dg_cl[32]);
// The rounds of sum_b A(b) B(b) over two device vectors of length 2^n (overwritten) from
// the given claim: each round's g(0), g(1), g(2) sent under lab_round at proof + *pos, the
// challenge squeezed under lab_chal; fin = A(rho), B(rho). The matmul sum-check's kernel with
// one site; scratch from the context's arenas (fp_two_vector_scratch, _host_scratch).
size_t fp_two_vector_scratch(const fp_ctx* c, int n);
size_t fp_two_vector_host_scratch();
int fp_two_vector_sumcheck(fp_ctx* c, fp_tx* tx, uint64_t* A, uint64_t* B, int n, uint64_t claim, const char* lab_round,
                           const char* lab_chal, uint8_t* proof, size_t* pos, uint64_t fin[2], cudaStream_t st);
// shapes, rescale exponents and the int32 domain of every site (no pointers looked at)
int fp_check_shapes(fp_ctx* c, const fp_site* sites, int nsites);

int fp_claims(fp_ctx* c, const fp_site* sites, int nsites, const uint64_t* const* eq_rows,
              const uint64_t* const* eq_cols, uint64_t* dev_out, cudaStream_t s);

static inline size_t fp_align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// blocks of 256 threads for a grid-stride loop over `work` items: enough to cover it, at
// most four per SM
static inline unsigned fp_grid256(const fp_ctx* c, int64_t work) {
    const int64_t want = (work + 255) / 256, cap = 4 * (int64_t)c->num_sms;
    return (unsigned)(want < 1 ? 1 : (want > cap ? cap : want));
}

// little-endian u64 words into a proof buffer (sumcheck.cu)
void put_u64s(uint8_t* p, const uint64_t* v, size_t n);

// The helper-inverse LogUp of an int32 key column on R_k (lhi.cu): its proof length, the
// device (and host) scratch of fp_lhi_run, and the run itself from "lhi_site" on, which
// allocates from c->dev and c->host as the caller reserved them (no reset). Returns FP_OK,
// 1 when some key lies outside the table, or an error.
size_t fp_lhi_proof_len(int64_t n, int k);
size_t fp_lhi_scratch(fp_ctx* c, int64_t n, int k, size_t* host_bytes);
int fp_lhi_run(fp_ctx* c, fp_tx* tx, const int32_t* r, int64_t n, int k, uint8_t* proof, size_t* proof_len,
               cudaStream_t st);

// the degree-3 polynomial through (i, g[i]), i = 0..3, at r (api.cu)
uint64_t fp_lagrange4(const uint64_t g[4], uint64_t r);
