/*
 * fp.h -- C ABI of libfp: a sum-check prover for the fixed-point quantised
 * matrix products of a transformer layer, over the Goldilocks field
 * p = 2^64 - 2^32 + 1, with the rescale and clamp of every product proven by
 * LogUp lookups. Hand-written CUDA for sm_100a (NVIDIA B200).
 *
 * What is proven (page "How fast can FlashProve go"):
 *  - 2 Background: the prover commits every intermediate value; sum-check
 *    reduces each polynomial operation (here Y = W.X) to claims on committed
 *    values and weights; non-polynomial steps (rescale, clamp) are proven by
 *    lookups; Fiat-Shamir makes every challenge a hash of all messages so far.
 *  - 3.1 Committing intermediate values: a rescale q = round(Y / 2^k) commits
 *    the remainder r = Y - 2^k q; the matmul sum-check uses 2^k q + r in place
 *    of Y and a lookup shows that r is small. Field: Goldilocks.
 *  - 2 / 2.1 Batching: many claims are merged into one (random linear
 *    combination of the per-matmul claims).
 *  - 4 Tighter Rooflines: a lookup's key side is a binary tree, every level
 *    proven by sum-check. Page "Towards Proving Frontier-Scale LLM Inference",
 *    The proof system: lookups by logarithmic derivatives (LogUp), whose
 *    fractions fill that tree.
 *  - 2 and 3.1 again: products that are never committed (the MLP's gated
 *    product, the per-group scaled weights) are reduced by sum-check to claims
 *    on their committed factors, and the SiLU and the softmax exponential are
 *    proven by lookups into 16-bit function tables.
 * The exact byte-level protocol (transcript encoding, tree digest, message
 * order, bit order, rounding tie) is specified in the repository's design
 * notes and implemented independently by the CPU oracle.
 *
 * Conventions for every entry point:
 *  - Pointers documented "device" are CUDA device pointers on the context's
 *    device (e.g. torch tensors' data_ptr()); "host" pointers are ordinary
 *    host memory. The caller owns every buffer it passes; the library never
 *    frees or retains them past the call.
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *    stream). Kernels run on it; every call returns only after its results
 *    (transcript updates, proof bytes) are on the host.
 *  - Scratch memory comes from a per-context device arena that grows on
 *    demand (cudaMalloc) and is released by fp_ctx_destroy.
 *  - Return value: FP_OK (0), a positive warning, or a negative FP_ERR_*
 *    code; fp_last_error(ctx) describes the last failure. No exception or
 *    signal crosses the ABI. After FP_ERR_CUDA the context should be
 *    destroyed.
 *  - A context or transcript must not be used from two threads at once.
 */
#ifndef FP_H_
#define FP_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FP_OK 0
#define FP_WARN_KEYS_OUTSIDE_TABLE 1 /* proof written; some key lies outside its table (the verifier will reject) */
#define FP_ERR_ARG -1                /* null pointer, bad enum value, buffer too small */
#define FP_ERR_SHAPE -2              /* dimensions out of the accepted domain */
#define FP_ERR_CUDA -3               /* a CUDA call failed */
#define FP_ERR_TIMEOUT -4            /* a bounded wait on the device ran out */
#define FP_ERR_OOM -5                /* device or pinned-host allocation failed */

typedef struct fp_ctx fp_ctx;
typedef struct fp_tx fp_tx;

/*
 * One matrix product Y = W . X ("site").
 *  w       device. W, M x K row-major. w_bits = 8: int8, K bytes per row.
 *          w_bits = 4: two's-complement nibbles packed two per byte along K,
 *          low nibble = even k, ceil(K/2) bytes per row (an odd K leaves the
 *          last high nibble zero).
 *  scales  device, nullable. int8 group scales, M x ceil(K/64) row-major:
 *          W_eff[i][k] = scales[i][k/64] * W[i][k].
 *  xt      device. X stored token-major: X^T as N x K row-major int8.
 *  q, r, y device, N x M row-major (token-major): q, r int32, y int8.
 *          Outputs of fp_commit_witness, inputs of the two provers.
 *  k_shift rescale exponent k, 1 <= k <= 20 (same for all sites of a call to
 *          logup_prove_rescale).
 *  w_digest host, nullable: 64 bytes D(W) || D(scales) computed once offline
 *          with fp_digest (weights committed in advance, page "FlashProve: How
 *          AI Answers Become Provable...", What FlashProve actually proves:
 *          offline commitment). NULL makes fp_commit_witness hash W itself
 *          (operands that are activations, e.g. attention's Q or V).
 * Accepted domain: 1 <= M, N <= 2^24, 1 <= K <= 2^20, and the worst-case
 * |Y| = max|W_eff| * 128 * K must stay below 2^31 (int32 accumulation exact),
 * e.g. K < 16384 for int4 with scales. Violations return FP_ERR_SHAPE.
 */
typedef struct {
    const void* w;
    const int8_t* scales;
    const int8_t* xt;
    int32_t* q;
    int32_t* r;
    int8_t* y;
    int32_t w_bits;
    int32_t M, K, N;
    int32_t k_shift;
    const uint8_t* w_digest;
} fp_site;

/* Library version (major * 10000 + minor * 100 + patch). */
int fp_version(void);

/* Create a context on CUDA device `device`; NULL on failure. */
fp_ctx* fp_ctx_create(int device);
void fp_ctx_destroy(fp_ctx* ctx);
/* Message of the last failure on this context (static storage, valid until the next call). */
const char* fp_last_error(const fp_ctx* ctx);

/*
 * Host Fiat-Shamir transcript ("How fast can FlashProve go", 2 Background:
 * each challenge is a hash of everything the prover has sent; SHA-256 here).
 *   state0 = SHA256("FPSC-v1" || u64le(seed))
 *   absorb:  state = SHA256(state || u32le(|label|) || label || u64le(n) || data)
 *   squeeze: h = SHA256(state || "sq" || u32le(|label|) || label || u32le(ctr)),
 *            ctr = 0, 1, ...; the first h whose low 8 bytes (little-endian)
 *            are < p becomes the state, that value the challenge.
 * fp_tx_squeeze draws n challenges in order into out[0..n).
 */
fp_tx* fp_tx_create(uint64_t seed);
void fp_tx_destroy(fp_tx* tx);
int fp_tx_absorb(fp_tx* tx, const char* label, const void* data, size_t n);
int fp_tx_squeeze(fp_tx* tx, const char* label, uint64_t* out, size_t n);
int fp_tx_state(const fp_tx* tx, uint8_t out[32]);

/*
 * Tree digest of a device byte buffer: SHA-256 of every 1 KiB chunk, then of
 * every run of up to 32 consecutive digests until one is left, finally
 * SHA256(u64le(nbytes) || top). out: host, 32 bytes. dev may be NULL when
 * nbytes == 0.
 */
int fp_digest(fp_ctx* ctx, const void* dev, size_t nbytes, uint8_t out[32], void* stream);

/*
 * fp_digest of n device buffers in one pass (the chunks of all buffers hashed by the same
 * launches): devs[i] (device, NULL allowed when nbytes[i] == 0) and nbytes[i] (host arrays of
 * n entries); out: host, 32 n bytes, digest i at out + 32 i. n >= 1, else FP_ERR_ARG.
 */
int fp_digests(fp_ctx* ctx, const void* const* devs, const size_t* nbytes, int n, uint8_t* out, void* stream);

/*
 * Witness and commitment of `nsites` products ("How fast can FlashProve go",
 * 3.1). For every site: Y = W_eff . X (exact int32 accumulation),
 * q = floor((Y + 2^(k-1)) / 2^k) (round half up), r = Y - 2^k q,
 * y = clamp(q, -128, 127), written to the site's q, r, y. Then, in site order,
 * absorbs "site" with D(W) || D(scales) || D(xt) || D(q) || D(r) || D(y) into tx.
 * Sites whose operands are other sites' outputs are committed by a later call,
 * after the call that produced them.
 */
int fp_commit_witness(fp_ctx* ctx, fp_tx* tx, const fp_site* sites, int nsites, void* stream);

/*
 * Multilinear partial evaluation: contracts the rows of a rows x cols matrix
 * with eq(point, .) ("How fast can FlashProve go", 2 Background and 4: the
 * matmul sum-check's weight decode), out[c] = sum_i eq(point, i) * M_eff[i][c]
 * for c < cols, 0 for cols <= c < 2^ceil(log2 cols).
 *  mat     device; bits = 4 (packed as fp_site.w) or 8 (int8), row-major.
 *  scales  device, nullable: per-64-column int8 scales, rows x ceil(cols/64).
 *  point   host, npoint = ceil(log2 rows) canonical field elements; its first
 *          coordinate binds the most significant row-index bit.
 *  out     device, 2^ceil(log2 cols) canonical u64.
 * W~(r_i, .) is mle_partial_eval(W); X~(., r_j) is mle_partial_eval(xt).
 */
int mle_partial_eval(fp_ctx* ctx, const void* mat, int bits, const int8_t* scales, int rows, int cols,
                     const uint64_t* point, int npoint, uint64_t* out, void* stream);

/*
 * mle_partial_eval without any device allocation. The pages have no
 * counterpart: this entry point exists for callers that must not allocate
 * device memory -- code running inside a host callback or an allocator hook,
 * under a memory pool that forbids out-of-band cudaMalloc, or in a process that
 * has already reserved all device memory. It takes no fp_ctx (creating one
 * allocates) and calls no cudaMalloc, cudaFree or allocating library routine.
 *
 * Same arguments and result as mle_partial_eval; `out` (device) receives
 * 2^ceil(log2 cols) values. Scratch is a fixed 16 MiB device array inside the
 * library (held by each GPU the entry point has run on, until the process
 * exits), which
 * limits the shape: ceil(rows / 1024) * cols must not exceed 2^21, and
 * npoint <= 24. Larger shapes return FP_ERR_SHAPE; bad pointers or bits
 * FP_ERR_ARG; a CUDA failure FP_ERR_CUDA. The kernels are queued on `stream`
 * and the call returns without waiting: the result is ready when the stream
 * reaches that point.
 *
 * Every call looks up the scratch array's device address on the current
 * device (cudaGetSymbolAddress). The CUDA runtime loads the library's modules
 * lazily (the default since CUDA 12), so the first call on each device loads
 * this one and reserves its 16 MiB there: make that first call outside the
 * context that must not allocate, and before any stream capture. Later calls
 * allocate nothing. Every call on a device shares the one scratch
 * array and leaves its contents behind; each call overwrites every entry it
 * reads, so nothing needs clearing, but calls whose kernels overlap on the GPU
 * (different streams of the same device) race on the array and must be
 * ordered by the caller.
 */
int mle_partial_eval_noalloc(const void* mat, int bits, const int8_t* scales, int rows, int cols,
                             const uint64_t* point, int npoint, uint64_t* out, void* stream);

/*
 * Matmul sum-check over all sites with claims batched by a random linear
 * combination ("How fast can FlashProve go", 2 and 2.1). Squeezes r_row, r_col;
 * sends the claims c_s = MLE of 2^k q + r at (r_row, r_col); squeezes rho_s
 * (more than one site); runs n = max ceil(log2 K) degree-2 rounds, each
 * sending g(0), g(1), g(2) and folding by the squeezed challenge; sends
 * A_s(rho), B_s(rho). Proof bytes (u64 little-endian field elements):
 *   nsites claims | n x 3 round values | 2 x nsites final values.
 * proof: host buffer; *proof_len: capacity in, bytes written out. Too small:
 * FP_ERR_ARG with the size needed in *proof_len and tx untouched.
 */
int sumcheck_prove_matmul(fp_ctx* ctx, fp_tx* tx, const fp_site* sites, int nsites, uint8_t* proof,
                          size_t* proof_len, void* stream);

/*
 * One statement proven by several ranks, one process per GPU ("How fast can
 * FlashProve go", 4 Tighter Rooflines: the work spread over the GPUs of one
 * node). The sites are independent until their claims are combined, so rank r
 * proves the sites [site_lo[r], site_lo[r + 1]) -- their witness, digests,
 * claims, partial evaluations and their share of every round -- and the ranks
 * exchange only small values through the caller's all-gather: the 192-byte
 * site records, the claims, each round's partial g(0), g(2) (16 bytes per
 * rank), and the final values. Every rank then absorbs the same values in the
 * same order, so all ranks hold one transcript and write the proof bytes of
 * the one-rank statement.
 *
 * allgather(user, mine, bytes, all): every rank passes `bytes` bytes (the same
 * count on every rank in every call); `all` (host, world * bytes) receives the
 * ranks' bytes in rank order. Returns 0, or nonzero to stop the call with
 * FP_ERR_ARG. Every rank must make the same calls in the same order.
 * site_lo: host, world + 1 entries, site_lo[0] = 0, site_lo[world] = nsites,
 * non-decreasing, every rank owning at least one site.
 */
typedef int (*fp_allgather_fn)(void* user, const void* mine, size_t bytes, void* all);
typedef struct {
    int rank;
    int world;
    const int* site_lo;
    fp_allgather_fn allgather;
    void* user;
} fp_shard;

/*
 * fp_commit_witness for a statement shared among ranks: computes the witness
 * and the digests of this rank's sites only, gathers every rank's 192-byte
 * site records and absorbs all of them in site order. sites: all nsites
 * descriptors; shapes are read for every site, device pointers only for this
 * rank's sites. Errors as for fp_commit_witness; a failed all-gather returns
 * FP_ERR_ARG.
 */
int fp_commit_witness_shard(fp_ctx* ctx, fp_tx* tx, const fp_site* sites, int nsites, const fp_shard* shard,
                            void* stream);

/*
 * sumcheck_prove_matmul for a statement shared among ranks: this rank's claims,
 * partial evaluations and round shares are computed from its own sites; the
 * proof and the transcript are those of the one-rank call, on every rank.
 * sites as for fp_commit_witness_shard. Errors as for sumcheck_prove_matmul.
 */
int sumcheck_prove_matmul_shard(fp_ctx* ctx, fp_tx* tx, const fp_site* sites, int nsites, const fp_shard* shard,
                                uint8_t* proof, size_t* proof_len, void* stream);

/*
 * LogUp proof of every site's rescale remainder and clamp ("How fast can
 * FlashProve go", 3.1 and 4; "Towards Proving Frontier-Scale LLM Inference",
 * The proof system). Keys: all outputs in storage order, sites concatenated,
 * padded to 2^v (v >= 1) with 0. Remainder table t_j = j - 2^(k-1) (2^k rows);
 * clamp table t_j = v_j + gamma clamp(v_j), v_j = j - 2^15 (2^16 rows).
 * Proof bytes: m_rem (2^k u32) | m_clamp (2^16 u32) | layer-one values (8 u64)
 * | for d = 1..v-1: d x 4 round values, 8 final values | 3 leaf values.
 * Returns FP_WARN_KEYS_OUTSIDE_TABLE (proof still written) when some r or q
 * falls outside its table. proof / proof_len as for sumcheck_prove_matmul.
 */
int logup_prove_rescale(fp_ctx* ctx, fp_tx* tx, const fp_site* sites, int nsites, uint8_t* proof,
                        size_t* proof_len, void* stream);

/*
 * The lookup section in the helper-inverse form (LogUp after Haboeck 2022,
 * "Towards Proving Frontier-Scale LLM Inference", The proof system), the
 * alternative to logup_prove_rescale's fraction tree ("How fast can FlashProve
 * go", 4 Tighter Rooflines). Same sites, keys, tables and multiplicities; the
 * key side is two committed helper columns checked by one sum-check of v rounds
 * (the tree takes v (v - 1) / 2):
 *   m_rem, "lhr_m_rem"; gamma; m_clamp, "lhr_m_clamp"; alpha0, alpha1;
 *   absorb "lhr_h" D(h0) || D(h1), h0_i = 1 / (alpha0 - r_i),
 *   h1_i = 1 / (alpha1 - q_i - gamma y_i); z_1..z_v, beta; send S0 = sum h0,
 *   S1 = sum h1; rounds of G = h0 + beta h1 + eq(z, .) (beta^2 (h0 (alpha0 - r)
 *   - 1) + beta^3 (h1 (alpha1 - q - gamma y) - 1)), claim S0 + beta S1; send
 *   h0, h1, r, q, y at rho.
 * Proof bytes: m_rem (2^k u32) | m_clamp (2^16 u32) | S0, S1 | v x 4 round
 * values | 5 final values. Keys up to 2^30. Returns FP_WARN_KEYS_OUTSIDE_TABLE
 * (proof still written) when some r or q lies outside its table; proof and
 * proof_len as for sumcheck_prove_matmul; other errors as logup_prove_rescale.
 */
int logup_prove_rescale_hi(fp_ctx* ctx, fp_tx* tx, const fp_site* sites, int nsites, uint8_t* proof,
                           size_t* proof_len, void* stream);

/*
 * Sum-check of a gated product h = s (.) u that is never committed ("How fast
 * can FlashProve go", 3.1 Committing intermediate values: the MLP's gated
 * product is a plain product, so sum-check handles it without committing to
 * it). s, u: device int8 vectors of n entries each (for an MLP, the SiLU output
 * and the up projection, [tokens, hidden] row-major), caller-owned, read only.
 * Both are zero-padded to 2^v, v = ceil(log2 n). The call continues tx:
 *   absorb "had_site" D(s) || D(u) (tree digests as fp_digest);
 *   squeeze z_1..z_v ("had_z"); send c = sum_x eq(z, x) s(x) u(x) ("had_claim");
 *   round t = 1..v: send g_t(0), g_t(1), g_t(2), g_t(3) ("had_round") with
 *     g_t(X) = sum over the unbound Boolean b of eq(z, (rho_<t, X, b))
 *     s~(rho_<t, X, b) u~(rho_<t, X, b); squeeze rho_t ("had_chal");
 *   send s~(rho), u~(rho) ("had_final").
 * Proof bytes (u64 LE field elements): c | v x 4 round values | 2 final values,
 * 8 + 32 v + 16 bytes. The verifier checks g_t(0) + g_t(1) against the running
 * claim, g_v(rho_v) = eq(z, rho) s~(rho) u~(rho), and the two final values
 * against openings of s and u. 1 <= n <= 2^30, else FP_ERR_SHAPE; null
 * arguments FP_ERR_ARG; proof / proof_len as for sumcheck_prove_matmul.
 */
int sumcheck_prove_hadamard(fp_ctx* ctx, fp_tx* tx, const int8_t* s, const int8_t* u, int64_t n, uint8_t* proof,
                            size_t* proof_len, void* stream);

/*
 * The gated-product sum-check with challenges in the quadratic extension
 * F_p[phi]/(phi^2 - 7) ("How fast can FlashProve go", 4, the note on soundness:
 * challenges from an extension field; 7 is not a square mod p). The statement of
 * sumcheck_prove_hadamard with every challenge, claim, round value and final value
 * an extension element a + b phi, sent as a then b (16 bytes) and squeezed as two
 * base challenges under its label. Same arguments; the call continues tx:
 *   absorb "had2_site" D(s) || D(u); squeeze z_1..z_v ("had2_z");
 *   send c ("had2_claim"); round t = 1..v: send g_t(0..3) ("had2_round"),
 *   squeeze rho_t ("had2_chal"); send s~(rho), u~(rho) ("had2_final").
 * Proof bytes: 16 + 64 v + 32. Errors as for sumcheck_prove_hadamard.
 */
int sumcheck_prove_hadamard_ext2(fp_ctx* ctx, fp_tx* tx, const int8_t* s, const int8_t* u, int64_t n,
                                 uint8_t* proof, size_t* proof_len, void* stream);

/*
 * Protocol drivers (no GPU work). The host half of a statement (the transcript,
 * the round polynomials, the running claim, the proof layout) is separate from
 * the device work that feeds it; a driver runs that host half with its device
 * values supplied by a callback, so the protocol can be checked against values
 * computed elsewhere. The callback gets (user, kind, t, in, out) and returns 0,
 * or nonzero to stop the driver with FP_ERR_ARG. What in and out hold for each
 * kind is given per driver below. Values are canonical field elements.
 */
enum {
    FP_VAL_START = 0,   /* the point is known */
    FP_VAL_SINGLE = 1,  /* a statement without rounds */
    FP_VAL_ROUND = 2,   /* round t's device values */
    FP_VAL_ANSWER = 3,  /* round t's challenge */
    FP_VAL_FINALS = 4,  /* the final values */
    FP_VAL_COLUMN = 5,  /* a committed column is formed: its digest */
    FP_VAL_CLAIM = 6,   /* the claim the rounds start from */
    FP_VAL_WEIGHTS = 7  /* the batching weights of the caller's sites */
};
typedef int (*fp_values_fn)(void* user, int kind, int t, const uint64_t* in, uint64_t* out);

/*
 * The host half of sumcheck_prove_hadamard_ext2 (v variables); tx must have
 * absorbed "had2_site". Callback kinds:
 *   FP_VAL_START: in = z_1..z_v (2 v words, a then b each), t = v;
 *   FP_VAL_SINGLE (v = 0 only): out = c, s(0), u(0) (6 words);
 *   FP_VAL_ROUND: out = h_t(0), h_t(1), h_t(2) (6 words), where
 *     h_t(X) = sum_b eq(z_>t, b) s~(rho_<t, X, b) u~(rho_<t, X, b);
 *   FP_VAL_ANSWER: in = rho_t (2 words);
 *   FP_VAL_FINALS: out = s~(rho), u~(rho) (4 words).
 * The proof and proof_len are as for sumcheck_prove_hadamard_ext2.
 */
int fp_had2_protocol_drive(fp_tx* tx, int v, fp_values_fn fn, void* user, uint8_t* proof, size_t* proof_len);

/*
 * Per-group scale reduction: a claim on W_eff~(z), W_eff[i][k] = S[i][k / 64] w[i][k]
 * (what the matmul sum-check of a site with scales ends with), reduced to claims on
 * the committed weights w and scales S by the same product sum-check as the gated
 * product ("How fast can FlashProve go", 3.1: a product that is not committed is
 * reduced by sum-check to its committed factors). Variables x = (i, k), row bits
 * first, M and K padded to 2^vM, 2^vK; factors Se(i, k) = S[i][k >> 6] (zero past
 * the M x ceil(K/64) scales) and w(i, k) (zero past M x K).
 * w: device, M x K int8 or int4 (two per byte, low nibble = even k, rows of
 * ceil(K/2) bytes); scales: device, M x ceil(K/64) int8; point: host, vM + vK
 * canonical field elements (row coordinates first). The call continues tx:
 *   absorb "scl_site" D(W) || D(S); send a = sum_x eq(z, x) Se(x) w(x) ("scl_claim");
 *   vM + vK rounds of g(0..3) ("scl_round") and challenges ("scl_chal");
 *   send Se~(rho), w~(rho) ("scl_final").
 * Se~(rho) equals S~(rho_row, rho_col_hi), rho_col_hi the first vK - 6 column
 * coordinates (none when vK <= 6). Proof: 8 + 32 (vM + vK) + 16 bytes.
 * w_digest: host, the 64 bytes D(W) || D(S) when the weights were committed in advance
 * (as fp_site.w_digest), or null to digest them here; a wrong value gives a proof the
 * verifier rejects.
 * M, K >= 1 and vM + vK <= 30, else FP_ERR_SHAPE; null or non-canonical
 * arguments FP_ERR_ARG; proof / proof_len as for sumcheck_prove_matmul.
 */
int sumcheck_reduce_scales(fp_ctx* ctx, fp_tx* tx, const void* w, int w_bits, const int8_t* scales, int M, int K,
                           const uint64_t* point, const uint8_t* w_digest, uint8_t* proof, size_t* proof_len,
                           void* stream);

/*
 * SiLU by lookup ("How fast can FlashProve go", 2 Background and 3.1: the SiLU is
 * not a polynomial, so its committed 16-bit outputs are proven by a lookup). The
 * table reads a 16-bit input v with 8 fractional bits and stores
 * silu_q(v) = floor(v / (1 + e^(-v/256)) + 1/2), evaluated in double precision.
 * g, s: device int16 columns of n entries (the SiLU's inputs and its claimed
 * outputs), caller-owned, read only. One LogUp-GKR tree over the keys
 * f = g + gamma s; the call continues tx:
 *   absorb "silu_site" D(g) || D(s) (int16 little-endian); squeeze gamma
 *   ("silu_gamma"); keys padded to 2^v (v = max(1, ceil(log2 n))) with (0, 0);
 *   send m_j = #{keys with g = j - 2^15} (2^16 u32; "silu_m" absorbs their
 *   digest); squeeze alpha ("silu_alpha"); send layer one p(0), p(1), q(0),
 *   q(1) ("silu_l1"); squeeze mu ("silu_mu"); for d = 1..v-1: squeeze lambda
 *   ("silu_lambda"), d rounds of g(0..3) ("silu_round") and challenges
 *   ("silu_chal") of the sum-check of eq(z, x)(pL qR + pR qL + lambda qL qR),
 *   the children pL, pR, qL, qR at rho ("silu_final"), squeeze mu; then
 *   g~(z), s~(z) ("silu_leaf").
 * Proof bytes: 4 * 2^16 + 32 + sum_{d=1}^{v-1} (32 d + 32) + 16. The verifier
 * checks the root against sum_j m_j / (alpha - v_j - gamma silu_q(v_j)), every
 * layer, and the leaf against alpha - (g~ + gamma s~). 1 <= n <= 2^30, else
 * FP_ERR_SHAPE; null arguments FP_ERR_ARG; proof / proof_len as for
 * sumcheck_prove_matmul.
 */
int logup_prove_silu(fp_ctx* ctx, fp_tx* tx, const int16_t* g, const int16_t* s, int64_t n, uint8_t* proof,
                     size_t* proof_len, void* stream);

/*
 * Helper-inverse LogUp on the remainder table R_k = {j - 2^(k-1) : j < 2^k}
 * ("Towards Proving Frontier-Scale LLM Inference", The proof system: LogUp after
 * Haboeck 2022, the key side a committed column of inverses checked by one
 * sum-check; set against the GKR fraction tree of logup_prove_rescale).
 * r: device int32 key column of n entries (caller-owned, read only); keys are
 * padded to 2^v (v = max(1, ceil(log2 n))) with 0. The call continues tx:
 *   absorb "lhi_site" D(r) (int32 little-endian); send m_j = #{keys equal to
 *   j - 2^(k-1)} (2^k u32, keys outside the table not counted; "lhi_m" absorbs
 *   their digest); squeeze alpha ("lhi_alpha"); absorb "lhi_h" D(h) for the
 *   helper column h_i = 1 / (alpha - r_i) (u64 little-endian, 2^v entries);
 *   squeeze z_1..z_v ("lhi_z") and beta ("lhi_beta"); send S = sum_i h_i
 *   ("lhi_sum"); v rounds of g(0..3) ("lhi_round") and challenges ("lhi_chal")
 *   of the sum-check of h(x) + beta eq(z, x) (h(x) (alpha - f(x)) - 1), claim S;
 *   send h~(rho), f~(rho) ("lhi_final").
 * Proof bytes: 4 2^k + 8 + 32 v + 16. Returns FP_OK, or 1 when some key lies
 * outside the table (the proof is still written; it will not verify).
 * 1 <= k <= 24 and null arguments: FP_ERR_ARG; 1 <= n <= 2^30, else
 * FP_ERR_SHAPE; proof / proof_len as for sumcheck_prove_matmul.
 */
int logup_prove_helper_inverse(fp_ctx* ctx, fp_tx* tx, const int32_t* r, int64_t n, int k, uint8_t* proof,
                               size_t* proof_len, void* stream);

/*
 * The matmul sum-check of one site with challenges in the quadratic extension
 * F_p[phi]/(phi^2 - 7) ("How fast can FlashProve go", 2 Background: the matmul
 * Y = W X reduced by sum-check to claims on its operands; 4, the note on
 * soundness: challenges from an extension field). site: one fp_site with its
 * witness (q, r) from fp_commit_witness; device pointers, caller-owned, read
 * only. The call continues tx:
 *   absorb "mm2_site" D(W) || D(S) || D(Xt) || D(q) || D(r) (D(W) || D(S) from
 *   site->w_digest when given); squeeze r_row (ceil(log2 M) extension
 *   coordinates, "mm2_row") and r_col (ceil(log2 N), "mm2_col"); send
 *   c = sum_{i,j} eq(r_row, i) eq(r_col, j) (2^k q[j][i] + r[j][i])
 *   ("mm2_claim"); n = ceil(log2 K) rounds of g(0), g(1), g(2) of
 *   sum_b A(X, b) B(X, b), A = W_eff~(r_row, .), B = X~(., r_col)
 *   ("mm2_round"), challenges ("mm2_chal"); send A(rho), B(rho) ("mm2_final").
 * Proof bytes: 16 + 48 n + 32. Site checks and errors as for
 * sumcheck_prove_matmul.
 */
int sumcheck_prove_matmul_ext2(fp_ctx* ctx, fp_tx* tx, const fp_site* site, uint8_t* proof, size_t* proof_len,
                               void* stream);

/*
 * Freivalds' check of a weight matmul, the prover's side ("Towards Proving
 * Frontier-Scale LLM Inference", The proof system: the weight matmuls are
 * checked by Freivalds' algorithm, A (B r) = C r for a random vector r), the
 * comparison statement for the matmul sum-check. site: one fp_site with its
 * witness; device pointers, caller-owned, read only. The call continues tx:
 *   absorb "frv_site" D(W) || D(S) || D(Xt) || D(q) || D(r) (D(W) || D(S) from
 *   site->w_digest when given); squeeze rho ("frv_rho"); send
 *   u_k = sum_j X[k][j] rho^j for k < K ("frv_u").
 * The verifier checks u against X and sum_k W_eff[i][k] u_k =
 * sum_j (2^k q + r)[j][i] rho^j for every row i. Proof bytes: 8 K. Site checks
 * and errors as for sumcheck_prove_matmul.
 */
int freivalds_prove_matmul(fp_ctx* ctx, fp_tx* tx, const fp_site* site, uint8_t* proof, size_t* proof_len,
                           void* stream);

/*
 * The host half of sumcheck_prove_matmul_ext2 (vM, vN point coordinates, n
 * rounds); tx must have absorbed "mm2_site". Callback kinds:
 *   FP_VAL_START: in = r_row then r_col (2 (vM + vN) words), t = vM + vN;
 *   FP_VAL_CLAIM: out = c (2 words);
 *   FP_VAL_ROUND: out = g_t(0), g_t(1), g_t(2) (6 words);
 *   FP_VAL_ANSWER: in = rho_t (2 words);
 *   FP_VAL_FINALS: out = A(rho), B(rho) (4 words).
 * The proof and proof_len are as for sumcheck_prove_matmul_ext2.
 */
int fp_mm2_protocol_drive(fp_tx* tx, int vM, int vN, int n, fp_values_fn fn, void* user, uint8_t* proof,
                          size_t* proof_len);

/*
 * The host half of sumcheck_prove_matmul_shard (and, with shard NULL, of
 * sumcheck_prove_matmul): tx must have absorbed the site records. sites: all
 * nsites descriptors, only their shapes read. Callback kinds, for this rank's
 * own sites (own = site_lo[rank + 1] - site_lo[rank], all sites with no shard):
 *   FP_VAL_START: in = r_row then r_col (vM + vN words), t = vM + vN;
 *   FP_VAL_CLAIM: out = c_s of the own sites (own words), t = own;
 *   FP_VAL_WEIGHTS: in = rho_s of the own sites (own words), t = own;
 *   FP_VAL_ROUND: out = this rank's share of g_t(0), g_t(2) (2 words): the
 *     sums over its own sites of rho_s sum_b A_s(X, b) B_s(X, b) at X = 0, 2;
 *   FP_VAL_ANSWER: in = r_t (1 word);
 *   FP_VAL_FINALS: out = A_s(rho), B_s(rho) of the own sites (2 own words).
 * The proof and proof_len are as for sumcheck_prove_matmul.
 */
int fp_mm_shard_protocol_drive(fp_tx* tx, const fp_site* sites, int nsites, const fp_shard* shard, fp_values_fn fn,
                               void* user, uint8_t* proof, size_t* proof_len);

/*
 * MoE routing, top-1 ("How fast can FlashProve go", 2 Background, the note on MoE
 * layers: the routing computation and each token's choice of expert are proven).
 * Token t goes to e_t, the first index of its largest router logit. logits:
 * device, T x E int8 token-major (the router matmul's rescaled outputs), read
 * only; E a power of two. H (T x E u8) and D (T x E int32): device, caller-
 * allocated, written by the call: the committed choice H[t][e] = [e = e_t] and
 * D[t][e] = l[t][e_t] - l[t][e] - [e < e_t]. With x = t E + e (token bits first,
 * rows zero-padded to 2^vT, n = vT + log2 E) the call continues tx:
 *   absorb "route_site" D(logits) || D(H) || D(D as int32 little-endian);
 *   squeeze z, w (n each, "route_z", "route_w"), lambda1, lambda2
 *   ("route_lambda"); send D~(z), l~(z) ("route_open"); n rounds of g(0..3)
 *   ("route_round") and challenges ("route_chal") of the sum-check of
 *   eq(z_t, t) H (l - G(e)) + lambda1 eq(w, x) H (1 - H) + lambda2 eq(w_t, t) H,
 *   G(e) = sum_{e' < e} eq(z_e, e'), claim D~(z) + l~(z) + lambda2 sum_{t < T}
 *   eq(w_t, t); send H~(rho), l~(rho) ("route_final"); then the statement of
 *   logup_prove_helper_inverse for the keys D - 128 (T E of them) on R_8.
 * Proof bytes: 16 + 32 n + 16 + the helper-inverse proof (4 * 256 + 8 + 32 v + 16,
 * v = max(1, ceil(log2 (T E)))). E not a power of two in [1, 4096], T < 1 or
 * n > 26: FP_ERR_SHAPE; null arguments FP_ERR_ARG; proof / proof_len as for
 * sumcheck_prove_matmul.
 */
int sumcheck_prove_routing(fp_ctx* ctx, fp_tx* tx, const int8_t* logits, int64_t T, int E, uint8_t* H, int32_t* D,
                           uint8_t* proof, size_t* proof_len, void* stream);

/*
 * MoE dispatch ("How fast can FlashProve go", 2 Background, the note on MoE
 * layers: the routing is proven): the experts' inputs D are the rows of the
 * layer input X moved to their experts. X: device, T x K int8 token-major (the
 * tensor the layer's gate and up sites read); e: device, T int32, the expert
 * of every token (the routing proof's choice), each in [0, E); D: device,
 * T x K int8, the experts' inputs stacked expert by expert, each expert's
 * tokens in token order. The call continues tx:
 *   absorb "dsp_site" D(X) || D(e) || D(D); squeeze r_row ("dsp_row",
 *   ceil(log2 T) coordinates) and r_col ("dsp_col", ceil(log2 K)); send
 *   c = D~(r_row, r_col) ("dsp_claim"); ceil(log2 T) degree-2 rounds of
 *   sum_t eq(r_row, pos(t)) X~(t, r_col), pos(t) = #{t' : e_t' < e_t} +
 *   #{t' < t : e_t' = e_t} ("dsp_round" g(0), g(1), g(2), "dsp_chal"); send
 *   both factors at rho ("dsp_final").
 * The verifier checks c against D, the rounds, the end, and the factors
 * against e and X. Proof bytes: 8 + 24 ceil(log2 T) + 16. 1 <= T, K <= 2^24,
 * 1 <= E <= 2^20, else FP_ERR_SHAPE; an expert index outside [0, E) gives
 * FP_ERR_ARG; proof / proof_len as for sumcheck_prove_matmul.
 */
int sumcheck_prove_dispatch(fp_ctx* ctx, fp_tx* tx, const int8_t* X, const int32_t* e, const int8_t* D, int64_t T,
                            int64_t K, int E, uint8_t* proof, size_t* proof_len, void* stream);

/*
 * The host half of sumcheck_prove_routing up to "route_final" (n variables);
 * tx must have absorbed "route_site". Callback kinds:
 *   FP_VAL_START: in = z_1..z_n, w_1..w_n, lambda1, lambda2 (2 n + 2 words), t = n;
 *   FP_VAL_CLAIM: out = D~(z), l~(z), sum_{t < T} eq(w_t, t) (3 words);
 *   FP_VAL_ROUND: out = g_t(0..3) (4 words);
 *   FP_VAL_ANSWER: in = rho_t (1 word);
 *   FP_VAL_FINALS: out = H~(rho), l~(rho) (2 words).
 * The proof holds 16 + 32 n + 16 bytes.
 */
int fp_route_protocol_drive(fp_tx* tx, int n, fp_values_fn fn, void* user, uint8_t* proof, size_t* proof_len);

/*
 * The helper-inverse LogUp over the quadratic extension F_p[phi]/(phi^2 - 7)
 * ("How fast can FlashProve go", 4, the note on soundness: challenges from an
 * extension field): the statement of logup_prove_helper_inverse with alpha, z,
 * beta, every challenge and every value sent an extension element (16 bytes: a
 * then b), the helper column the extension inverses 1 / (alpha - r_i) committed
 * as 16-byte pairs, and the labels "lhi2_site", "lhi2_m", "lhi2_alpha",
 * "lhi2_h", "lhi2_z", "lhi2_beta", "lhi2_sum", "lhi2_round", "lhi2_chal",
 * "lhi2_final". Proof bytes: 4 2^k + 16 + 64 v + 32. Same arguments, status and
 * errors as logup_prove_helper_inverse.
 */
int logup_prove_helper_inverse_ext2(fp_ctx* ctx, fp_tx* tx, const int32_t* r, int64_t n, int k, uint8_t* proof,
                                    size_t* proof_len, void* stream);

/*
 * The host half of logup_prove_helper_inverse_ext2 from the multiplicities on
 * (as fp_lhi_protocol_drive, every value an extension element of two words):
 *   FP_VAL_COLUMN: in = alpha (2 words); out = D(h) (4 words);
 *   FP_VAL_START: in = z_1..z_v, beta (2 v + 2 words), t = v;
 *   FP_VAL_ROUND: out = H_t(0), H_t(1), Q_t(0), Q_t(1), Q_t(2) (10 words);
 *   FP_VAL_ANSWER: in = rho_t (2 words);
 *   FP_VAL_FINALS: out = h~(rho), f~(rho) (4 words).
 * The proof holds 4 2^k + 16 + 64 v + 32 bytes.
 */
int fp_lhi2_protocol_drive(fp_tx* tx, int v, int k, const uint32_t* m, const uint8_t* m_digest, fp_values_fn fn,
                           void* user, uint8_t* proof, size_t* proof_len);

/*
 * The host half of logup_prove_helper_inverse from the multiplicities on (v >= 1
 * variables, table R_k): m (host, 2^k u32) and m_digest (host, 32 bytes: the
 * digest of m's bytes) are given; tx must have absorbed "lhi_site". Callback
 * kinds (see the protocol drivers above):
 *   FP_VAL_COLUMN: in = alpha (1 word); out = D(h) (32 bytes as 4 little-endian words);
 *   FP_VAL_START: in = z_1..z_v, beta (v + 1 words), t = v;
 *   FP_VAL_ROUND: out = H_t(0), H_t(1), Q_t(0), Q_t(1), Q_t(2) (5 words) with
 *     H_t(X) = sum_b h~(rho_<t, X, b) and
 *     Q_t(X) = sum_b eq(z_>t, b) h~(rho_<t, X, b) (alpha - f~(rho_<t, X, b));
 *   FP_VAL_ANSWER: in = rho_t (1 word);
 *   FP_VAL_FINALS: out = h~(rho), f~(rho) (2 words).
 * The proof and proof_len are as for logup_prove_helper_inverse.
 */
int fp_lhi_protocol_drive(fp_tx* tx, int v, int k, const uint32_t* m, const uint8_t* m_digest, fp_values_fn fn,
                          void* user, uint8_t* proof, size_t* proof_len);

/*
 * The host half of logup_prove_rescale_hi from the multiplicities on (v
 * variables, k the rescale shift); tx must have reached the lookup section.
 * m: host, 2^k u32 of m_rem then 2^16 of m_clamp; m_digests: 64 bytes, their
 * two tree digests. Callback kinds:
 *   FP_VAL_COLUMN: in = alpha0, alpha1, gamma; out = D(h0) || D(h1) (8 words,
 *     little-endian bytes);
 *   FP_VAL_START: in = z_1..z_v, beta (v + 1 words), t = v;
 *   FP_VAL_ROUND: out = A0(0), A0(1), A1(0), A1(1), Q0(0..2), Q1(0..2)
 *     (10 words; A sums of h0 and h1, Q the eq(z_>t)-weighted sums of
 *     h0 (alpha0 - r) and h1 (alpha1 - q - gamma y));
 *   FP_VAL_ANSWER: in = rho_t;
 *   FP_VAL_FINALS: out = h0, h1, r, q, y at rho (5 words).
 * proof and proof_len as for logup_prove_rescale_hi.
 */
int fp_lhr_protocol_drive(fp_tx* tx, int v, int k, const uint32_t* m, const uint8_t* m_digests, fp_values_fn fn,
                          void* user, uint8_t* proof, size_t* proof_len);

/*
 * The SiLU and softmax numerator lookups over the quadratic extension
 * F_p[phi]/(phi^2 - 7) ("How fast can FlashProve go", 4, the note on soundness:
 * challenges from an extension field): the statements of logup_prove_silu and
 * logup_prove_exp with gamma, alpha, mu, lambda, every round challenge and every
 * value sent an extension element (16 bytes: a then b), the tree's fractions in
 * the extension, and the labels "silu2_*" / "exp2_*" (site, gamma, m, alpha, l1,
 * mu, lambda, round, chal, final, leaf). Proof bytes: 4 * 2^16 + 64 + 32 +
 * sum_{d=1}^{v-1} (64 d + 64). Same arguments and errors as logup_prove_silu.
 */
int logup_prove_silu_ext2(fp_ctx* ctx, fp_tx* tx, const int16_t* g, const int16_t* s, int64_t n, uint8_t* proof,
                          size_t* proof_len, void* stream);
int logup_prove_exp_ext2(fp_ctx* ctx, fp_tx* tx, const int16_t* g, const int16_t* s, int64_t n, uint8_t* proof,
                         size_t* proof_len, void* stream);

/*
 * The host half of logup_prove_silu_ext2 (table 0) or logup_prove_exp_ext2
 * (table 1) from the multiplicities on, v >= 1 variables: gamma (2 words, squeezed
 * by the caller after the site), m (host, 2^16 u32) and m_digest (32 bytes) are
 * given. Callback kinds:
 *   FP_VAL_COLUMN: in = gamma, alpha (4 words); out = layer one's P(0), P(1), Q(0),
 *     Q(1) (8 words);
 *   FP_VAL_START: layer d begins; in = z_1..z_d, lambda (2 d + 2 words), t = d;
 *   FP_VAL_ROUND: out = h_t(0), h_t(1), h_t(2) of the current layer (6 words);
 *   FP_VAL_ANSWER: in = rho_t (2 words);
 *   FP_VAL_FINALS: out = pL, pR, qL, qR at rho (8 words);
 *   FP_VAL_CLAIM: in = the leaf point z_1..z_v (2 v words), t = v; out = g~(z), s~(z)
 *     of the padded columns (4 words).
 * The proof and proof_len are as for logup_prove_silu_ext2 with 2^v keys.
 */
int fp_lookup16x_protocol_drive(fp_tx* tx, int table, int v, const uint64_t* gamma, const uint32_t* m,
                                const uint8_t* m_digest, fp_values_fn fn, void* user, uint8_t* proof,
                                size_t* proof_len);

/*
 * The rescale LogUp over the quadratic extension ("How fast can FlashProve go", 4,
 * the note on soundness): the remainder table R_k and the clamp table C16 of
 * logup_prove_rescale batched in one GKR, with every challenge and value an
 * extension element (16 bytes: a then b), as a statement of its own over the
 * sites' key columns (q, r, y of every site, concatenated in site order):
 *   absorb "lu2_site" D(r) || D(q) (int32 little-endian) || D(y); send m_rem
 *   ("lu2_m_rem"); squeeze gamma ("lu2_gamma"); send m_clamp ("lu2_m_clamp");
 *   squeeze alpha_0, alpha_1 ("lu2_alpha"); send layer one of both trees
 *   ("lu2_l1", 8 values); squeeze mu ("lu2_mu"); per layer d = 1..v-1 squeeze
 *   lambda ("lu2_lambda"), d rounds of g(0..3) ("lu2_round", "lu2_chal") of the
 *   sum-check of eq(z, x) sum_tau lambda^(2 tau) (pL qR + pR qL + lambda qL qR),
 *   the eight children at rho ("lu2_final"), squeeze mu; then r~(z), q~(z), y~(z)
 *   ("lu2_leaf").
 * Proof bytes: 4 2^k + 4 2^16 + 128 + sum_{d=1}^{v-1} (64 d + 128) + 48. Returns
 * FP_OK, or 1 when some key lies outside its table (the proof is still written).
 * Site checks and errors as for logup_prove_rescale.
 */
int logup_prove_rescale_ext2(fp_ctx* ctx, fp_tx* tx, const fp_site* sites, int nsites, uint8_t* proof,
                             size_t* proof_len, void* stream);

/*
 * The host half of logup_prove_rescale_ext2 from the multiplicities on (v >= 1
 * variables, remainder table R_k): m_rem (2^k u32), m_clamp (2^16 u32) and their
 * 32-byte digests are given; tx must have absorbed "lu2_site". Callback kinds:
 *   FP_VAL_COLUMN: in = gamma, alpha_0, alpha_1 (6 words); out = layer one of
 *     both trees, P(0), P(1), Q(0), Q(1) per table (16 words);
 *   FP_VAL_START: layer d begins; in = z_1..z_d, lambda (2 d + 2 words), t = d;
 *   FP_VAL_ROUND: out = h_t(0), h_t(1), h_t(2) (6 words);
 *   FP_VAL_ANSWER: in = rho_t (2 words);
 *   FP_VAL_FINALS: out = pL, pR, qL, qR at rho, per table (16 words);
 *   FP_VAL_CLAIM: in = the leaf point (2 v words), t = v; out = r~(z), q~(z), y~(z)
 *     (6 words).
 */
int fp_lu2_protocol_drive(fp_tx* tx, int v, int k, const uint32_t* m_rem, const uint8_t* d_rem, const uint32_t* m_clamp,
                          const uint8_t* d_clamp, fp_values_fn fn, void* user, uint8_t* proof, size_t* proof_len);

/* The SiLU table's 2^16 entries silu_q(v), v = -2^15 .. 2^15 - 1, into host out (no GPU work). */
int fp_silu_table(int32_t* out);

/* The SiLU's inputs and outputs for 8-bit inputs ("How fast can FlashProve go", 3.1: the SiLU
 * output is committed and proven by lookup; here its inputs are the gate projection's committed
 * outputs). For the n device int8 values y (the gate site's y, token-major): g[i] = y[i] (device
 * int16), s[i] = silu_q(y[i]) (device int16) and s8[i] = s[i] (device int8: silu_q maps
 * [-128, 127] into [-48, 79]). All four buffers are the caller's, n entries each, on ctx's
 * device; the kernel runs on `stream` and nothing is allocated. Returns FP_OK or FP_ERR_ARG. */
int fp_silu_inputs(fp_ctx* ctx, const int8_t* y, int64_t n, int16_t* g, int16_t* s, int8_t* s8, void* stream);

/* The FFN's hidden activations, rescaled for the down projection ("How fast can FlashProve go",
 * 3.1: the gated product of the SiLU outputs with the up projection's outputs, brought back to
 * 8 bits as every matmul output is): for the n device int8 SiLU outputs s and up outputs u
 * (same token-major layout), h = s[i] u[i], q[i] = floor((h + 2^(kh-1)) / 2^kh), r[i] = h -
 * 2^kh q[i] (device int32 each) and y[i] = clamp(q[i], -128, 127) (device int8; the down site's
 * activations). kh in [1, 16]. All buffers are the caller's, n entries each, on ctx's device;
 * the kernel runs on `stream` and nothing is allocated. Returns FP_OK or FP_ERR_ARG. */
int fp_ffn_hidden(fp_ctx* ctx, const int8_t* s, const int8_t* u, int64_t n, int kh, int32_t* q, int32_t* r, int8_t* y,
                  void* stream);

/* The point where the last matmul section proven with ctx (sumcheck_prove_matmul) left its
 * sites: the row challenges r_row (v_row of them, into host r_row) and the round challenges
 * rho_1..rho_n (into host rho). A chained statement continues from it: a site's weight value
 * A_s(rho) is W_eff's MLE at (r_row's first ceil(log2 M_s) coordinates, the last ceil(log2 K_s)
 * round challenges) times prod_{j <= n - ceil(log2 K_s)} (1 - rho_j) (the padded columns of a
 * narrower site are zero), the point of the per-group scale reduction (sumcheck_reduce_scales).
 * Null buffers query the sizes. Returns FP_ERR_ARG if no matmul section was proven yet or a
 * buffer is too small. */
int sumcheck_last_point(fp_ctx* ctx, uint64_t* r_row, int cap_row, int* v_row, uint64_t* rho, int cap_rho, int* n);

/*
 * The softmax numerator by lookup ("Towards Proving Frontier-Scale LLM Inference",
 * The arithmetic: the exponential is a lookup table, the integer softmax has a
 * 9-bit numerator): the same argument as logup_prove_silu with the labels
 * "exp_site", "exp_gamma", "exp_m", "exp_alpha", "exp_l1", "exp_mu",
 * "exp_lambda", "exp_round", "exp_chal", "exp_final", "exp_leaf" and the table
 * exp_q(v) = floor(511 e^(v/256) + 1/2) for v = score - row maximum <= 0, 511
 * for v > 0. Keys are padded with the table's row for input 0, (0, 511). Same
 * arguments, proof layout and errors as logup_prove_silu.
 */
int logup_prove_exp(fp_ctx* ctx, fp_tx* tx, const int16_t* g, const int16_t* s, int64_t n, uint8_t* proof,
                    size_t* proof_len, void* stream);

/* The numerator table's 2^16 entries exp_q(v), v = -2^15 .. 2^15 - 1, into host out (no GPU work). */
int fp_exp_table(int32_t* out);

/*
 * Self-test of the bounded device waits. The sum-check kernels stay resident
 * across rounds and wait (a bounded number of polls) for each Fiat-Shamir
 * challenge from the host. This call launches a kernel that waits for a
 * challenge nobody posts: after about a second it gives up and flags the
 * mailbox, and the call returns FP_ERR_TIMEOUT. The context stays usable.
 */
int fp_session_selftest(fp_ctx* ctx, void* stream);

/* Proof section sizes in bytes for a statement (no GPU work). */
int fp_proof_size(const fp_site* sites, int nsites, size_t* matmul_bytes, size_t* logup_bytes);

/*
 * Per-kernel timing: while profiling is on (fp_ctx_set_profiling(ctx, 1) or 2,
 * which also clears the counters), every launch of the library on this context is
 * bracketed by CUDA events on its stream. fp_kernel_stats fills up to `cap`
 * records {kernel id, launches, total device ms, algorithmic bytes moved} and
 * returns the number of kernels seen; names come from fp_kernel_name(id).
 */
typedef struct {
    int32_t kernel;
    int32_t launches;
    double ms;
    double bytes;
} fp_kernel_stat;
int fp_ctx_set_profiling(fp_ctx* ctx, int on);
/* With profiling level 1 (and when the process runs under an injected profiler,
 * or with FP_STEPPED=1 in the environment) every sum-check round is its own
 * kernel launch, so that each launch can be timed; otherwise one resident kernel
 * runs all rounds of a sum-check, and level 2 times those launches as they run
 * (host exchanges included). Both modes produce the same proof bytes. 0 turns
 * timing off; other values are FP_ERR_ARG. */
/* Number of kernels the library has launched on this context since its creation. */
int64_t fp_ctx_launches(const fp_ctx* ctx);
/* Host side of the round exchanges since the context was created:
 * out[0] = waits for a device result, out[1] = seconds spent waiting,
 * out[2] = seconds from a result's arrival to the next challenge posted (the
 * host's own share of a round: hashing and bookkeeping), out[3] = the longest
 * such turnaround in seconds. */
int fp_host_stats(const fp_ctx* ctx, double out[4]);
int fp_kernel_stats(fp_ctx* ctx, fp_kernel_stat* out, int cap);
/* Per-launch records of the same timing, in launch order: {kernel id, 0, device
 * ms of that launch, its algorithmic bytes, the device ms from the first timed launch
 * since fp_ctx_set_profiling to this launch's start (a timeline: the gaps between
 * launches are host work and waits)}. Copies up to `cap` records into `out` (host
 * memory owned by the caller) and returns how many there are; cleared by
 * fp_ctx_set_profiling. */
typedef struct {
    int32_t kernel;
    int32_t reserved;
    double ms;
    double bytes;
    double start_ms;
} fp_launch_rec;
int64_t fp_kernel_log(fp_ctx* ctx, fp_launch_rec* out, int64_t cap);
const char* fp_kernel_name(int kernel);

#ifdef __cplusplus
}
#endif
#endif /* FP_H_ */
