/*
 * smuon.h -- C ABI of the B200 (sm_100a) Sign-Muon optimizer-step library.
 *
 * The method: "SignMuon: Communication-Efficient Distributed Muon
 * Optimization" (technical summary, section 2 "Method": core mechanism 1-3,
 * distributed algorithm flow steps 1-5, communication efficiency; English
 * abstract), with two neighbours from the same family: "CacheMuon" (section
 * "Method": fresh solve, cache reuse, residual trigger) and "LionMuon"
 * (section "Methodology": period-P alternation, shared double-EMA momentum).
 *
 * Conventions shared by every entry point
 *  - Every function returns smuon_status: SMUON_OK (0) or a negative code.
 *  - Arguments are checked on the host before anything is enqueued; on an
 *    error nothing is launched and smuon_last_error() describes the problem.
 *  - Every call is asynchronous on the caller's CUDA stream (passed as
 *    void*, a cudaStream_t; NULL = legacy default stream) and never
 *    synchronises the host.
 *  - The caller owns all device memory: matrices, outputs, device flags and
 *    the workspace, whose size comes from the matching *_workspace_bytes
 *    query. The library allocates no device memory on these paths.
 *  - Matrices are row-major: element (i, j) of an smuon_mat lives at
 *    data + (i * ld + j) * sizeof(dtype). ld >= cols.
 *  - Problems found on the device (NaN/Inf in a norm, a bounded wait that
 *    ran out) are OR-ed into the optional caller-provided int32 *d_status.
 *  - Device code is built for sm_100a only; on another device every call
 *    that would launch returns SMUON_ERR_UNSUPPORTED.
 */
#ifndef SMUON_H
#define SMUON_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t smuon_status;

#define SMUON_OK               0
#define SMUON_ERR_INVALID_ARG (-1)  /* null pointer, bad count, bad flag */
#define SMUON_ERR_SHAPE       (-2)  /* shapes that do not match each other */
#define SMUON_ERR_DTYPE       (-3)  /* dtype not accepted at that argument */
#define SMUON_ERR_UNSUPPORTED (-4)  /* e.g. more than 64 workers, wrong GPU */
#define SMUON_ERR_WORKSPACE   (-5)  /* workspace missing, too small, misaligned */
#define SMUON_ERR_CUDA        (-6)  /* a CUDA runtime call failed */

/* element types */
#define SMUON_F32  0
#define SMUON_BF16 1
#define SMUON_I8   2
#define SMUON_BITS 3  /* the 1-bit message of a sign matrix (SignMuon summary, flow step 3, all-gather
                         variant; communication efficiency: one bit per parameter): data holds uint32
                         words, entry i of the row-major flattening (i = row*cols + col) at bit i % 32
                         of word i / 32, ceil(rows*cols / 128) * 4 words (a 16-byte multiple) with the
                         bits past the last entry zero; ld must equal cols and data be 16-byte aligned.
                         A set bit is the sign +1 (u >= 0), a clear bit -1 */

/* bits OR-ed into *d_status by device code */
#define SMUON_DEV_NONFINITE_NORM 1  /* a Frobenius norm (or a spectral-norm estimate) was NaN or Inf */
#define SMUON_DEV_WAIT_TIMEOUT   2  /* a bounded pipeline wait ran out; results invalid */

/* a row-major matrix in device memory */
typedef struct {
  void*   data;
  int32_t rows, cols;
  int64_t ld;      /* elements between consecutive rows, >= cols */
  int32_t dtype;   /* SMUON_F32 | SMUON_BF16 | SMUON_I8 */
} smuon_mat;

const char* smuon_last_error(void);           /* thread-local message of the last failure */
int32_t     smuon_version(void);              /* (major << 16) | minor */

/* ------------------------------------------------------------------------
 * Launch counting and tracing (diagnostics; not part of the method).
 * smuon_launch_count: kernels launched by this library since it was loaded.
 * smuon_trace_enable(1): from then on every launch is bracketed by two CUDA
 * events on its stream and logged with its work: for the GEMM stages the
 * flops the tensor cores executed (padded tiles, three products in split
 * mode) and the method's nominal 2*M*N*K flops; for the bandwidth-bound
 * kernels the bytes the method must move. smuon_trace_read synchronises on the logged events,
 * copies up to max_recs records (oldest first), clears the log and returns
 * the number copied (with out == NULL: the number logged).
 * ---------------------------------------------------------------------- */
#define SMUON_WORK_FLOPS 0
#define SMUON_WORK_BYTES 1
typedef struct {
  char    name[40];
  int32_t kind;     /* SMUON_WORK_FLOPS | SMUON_WORK_BYTES */
  double  work;     /* flops issued to the tensor (or CUDA) cores, tiles x tile flops; or bytes */
  double  nominal;  /* the method's nominal flops (2*M*N*K per product); equals work for bytes */
  float   ms;       /* event-timed duration, -1 if unavailable */
} smuon_trace_rec;

int64_t smuon_launch_count(void);
void    smuon_trace_enable(int32_t on);
int32_t smuon_trace_read(smuon_trace_rec* out, int32_t max_recs);

/* ------------------------------------------------------------------------
 * smuon_ns -- momentum + Frobenius normalisation + Newton-Schulz polar step.
 *
 * SignMuon summary, section 2 core mechanism 1 and algorithm flow step 1:
 * each worker updates its local momentum and takes its polar factor by a
 * Newton-Schulz iteration; section 4 hyper-parameters: Frobenius scaling.
 * Readings: momentum M <- beta*M + G (heavy ball); X0 = M/(||M||_F + eps);
 * K steps X <- aX + b(XX^T)X + c(XX^T)^2 X on the smaller Gram side (a tall
 * matrix is iterated transposed); CacheMuon method 1 for EMIT_Q.
 *
 *  M_in[n_mats]   momentum matrices (F32; BF16 or I8 accepted when G == NULL).
 *                 Updated in place when G != NULL.
 *  U_out[n_mats]  polar-factor outputs, same shape as M_in[i] (F32 or BF16),
 *                 or I8: then only the entrywise sign of U is written, +1 for
 *                 u >= 0 (-0 included) and -1 otherwise (NaN included), taken on
 *                 the float32 value in the last step's epilogue (SignMuon
 *                 summary, flow step 2: the sign matrix without U in memory),
 *                 or BITS: the same signs as the worker's 1-bit message (flow
 *                 step 3, all-gather variant), written by that epilogue, pad
 *                 words zeroed by the call; needs cols % 32 == 0 and the
 *                 tensor-core modes, not with SMUON_NS_EMIT_Q.
 *  G[n_mats]      nullable gradients (F32 or BF16), same shapes.
 *  beta           momentum coefficient (ignored when G == NULL).
 *  a, b, c        Newton-Schulz coefficients; c == 0 skips the A^2 product.
 *  iters          K >= 1.
 *  eps            added to the Frobenius norm.
 *  flags          SMUON_NS_* below.
 *  Q_out[n_mats]  with SMUON_NS_EMIT_Q: BF16 m x m cached left transforms
 *                 Q = P_{K-1}...P_0, P_k = aI + bA_k + cA_k^2 (m = min side),
 *                 so that Q X0 = X_K. NULL otherwise.
 *  d_skip_if      nullable device int32: when nonzero at run time every
 *                 kernel of this call returns at once (CacheMuon hit).
 *  ws, ws_bytes   workspace, >= smuon_ns_workspace_bytes(), 256-byte aligned.
 *                 Its contents are scratch; it must not be shared with a call
 *                 that may run concurrently.
 *  d_status       nullable device int32 for SMUON_DEV_* bits.
 * Limits: 1 <= rows, cols <= 65536 per matrix; n_mats <= 4096.
 * ---------------------------------------------------------------------- */
#define SMUON_NS_FP32_REF      1u  /* FP32 operands on CUDA cores (reference mode) */
#define SMUON_NS_SPLIT_BF16    2u  /* accurate mode: every GEMM operand split into bf16 hi + lo
                                      parts, three tcgen05 MMAs per product (3x tensor work). X between
                                      steps and A for the b A term are kept as their hi + lo parts alone
                                      (x ~ hi + lo to about 2^-17 relative); the a X and b A terms are
                                      formed in float32 from them */
#define SMUON_NS_NO_NORMALIZE  4u  /* skip the Frobenius normalisation (s = 1) */
#define SMUON_NS_EMIT_Q        8u  /* also write the CacheMuon transform Q */
#define SMUON_NS_SIMT_BF16    16u  /* diagnostic: BF16 operands on CUDA cores instead of tcgen05 */
#define SMUON_NS_SPECTRAL     64u  /* normalise by the spectral norm instead: X_0 = M / (||M||_2 + eps)
                                      (SignMuon summary, section 4: either norm will do); ||M||_2 from a
                                      Lanczos estimate of the largest eigenvalue of the first Gram matrix,
                                      per matrix, on the device: at most 64 steps, each matrix stopped once
                                      the residual of its largest Ritz pair is below 1e-4 of it. Not with
                                      SMUON_NS_NO_NORMALIZE, SMUON_NS_EMIT_Q or SMUON_NS_GRAM_ONLY */
#define SMUON_NS_PLAIN_LEAD(k) ((uint32_t)(k) << 12)  /* with SMUON_NS_SPLIT_BF16: the first k (0..7)
                                      Newton-Schulz steps take plain BF16 operands (one MMA per product, the
                                      lo parts still written for the later steps) -- for matrices whose
                                      smaller side is at least 512; smaller matrices take only their first
                                      step plain. While the normalised singular values are small, the B X
                                      term of a step is small beside the float32 a X term, so its operand
                                      rounding barely reaches the output. On Gaussian momenta this keeps five
                                      quintic steps within the split mode's accuracy for k <= 2; the top
                                      normalised singular value starts near 1/sqrt(m) + 1/sqrt(n). A matrix
                                      with one dominant singular value starts near 1: leave k = 0 there. Not
                                      with SMUON_NS_SPECTRAL (s_max = 1), SMUON_NS_EMIT_Q or
                                      SMUON_NS_GRAM_ONLY */
#define SMUON_NS_PLAIN_LEAD_MASK (7u << 12)
#define SMUON_NS_ONE_SM     0x80u  /* tensor-core stages on single-SM 128 x 256 tiles. Without it, a call
                                      whose matrices all have a smaller side of at least 256 runs them on
                                      pairs of SMs: 256 x 256 tiles, clusters of two CTAs, tcgen05 MMAs over
                                      both SMs. Each output element takes the same products in the same
                                      order in both forms, so U and Q agree bit for bit. (The CacheMuon
                                      probe, which takes no flags, always uses pairs when m >= 256; its
                                      residual sums the same per-warp partials over another tiling.) */
#define SMUON_NS_TEST_WAIT_EXPIRY 0x8000u  /* failure-detection test, not for use: every tensor-core stage's
                                      copy producers issue nothing and its pipeline waits are limited to
                                      65536 SM clocks (about 2 s otherwise), so each stage's first waits run
                                      out; the CTAs then record SMUON_DEV_WAIT_TIMEOUT in d_status, wait (with
                                      the full budget) for anything they issued, free their tensor memory and
                                      return. U is not written */
#define SMUON_NS_GRAM_ONLY    32u  /* CacheMuon fresh solve iterated on the m x m Gram ("Gram
                                      Newton-Schulz", CacheMuon summary, method item 1): A_0 = X_0 X_0^T once,
                                      then per step P_k = aI + bA_k + cA_k^2, Q_{k+1} = P_k Q_k and
                                      A_{k+1} = P_k A_k P_k (= P_k^2 A_k; the P_k commute with A_k), and
                                      finally U = Q_K X_0: 4 m^2 n once plus about 8 m^3 per step,
                                      instead of 4 m^2 n + 4 m^3 per step; fewer flops when m < n. Needs
                                      SMUON_NS_EMIT_Q, one matrix, c != 0 and the tensor-core modes */

smuon_status smuon_ns_workspace_bytes(const smuon_mat* M_in, int32_t n_mats, int32_t iters,
                                      uint32_t flags, size_t* bytes);

smuon_status smuon_ns(const smuon_mat* M_in, const smuon_mat* U_out, int32_t n_mats,
                      const smuon_mat* G, float beta,
                      float a, float b, float c, int32_t iters, float eps, uint32_t flags,
                      const smuon_mat* Q_out, const int32_t* d_skip_if,
                      void* ws, size_t ws_bytes, int32_t* d_status, void* stream);

/* ------------------------------------------------------------------------
 * smuon_ns_static -- smuon_ns without a caller-provided workspace.
 *
 * The paper has no counterpart: this is a deployment convenience. It is for
 * callers that cannot allocate device memory at the point of the call, for
 * example code running under an external memory budget or allocator that
 * forbids foreign allocations, or callers that must not enter the CUDA
 * allocator (which may synchronise the device) in a latency-critical
 * section. It computes exactly what smuon_ns computes, with the same
 * arguments minus ws / ws_bytes; its scratch is a fixed array of
 * SMUON_NS_STATIC_SCRATCH_BYTES in the library's device image, so every GPU
 * that loads the library holds that memory until the process exits.
 *  - Batches whose smuon_ns_workspace_bytes() exceeds the array are rejected
 *    with SMUON_ERR_WORKSPACE before anything is enqueued.
 *  - It calls no cudaMalloc, cudaFree or other allocating routine.
 *  - The first call on a device looks up the array's device address (with
 *    that device current); make that first call before any stream capture.
 *    The address is kept per device and context: a call from a new context
 *    (after cudaDeviceReset, for instance) looks it up again, so make the
 *    first call after such a reset outside stream capture too.
 *  - All calls share the one array and it keeps the last call's contents
 *    (nothing in it needs to start at zero: every call rewrites what it
 *    reads). Calls that may overlap on the GPU (other streams, other host
 *    threads) race on it: serialise them, e.g. on one stream.
 * ---------------------------------------------------------------------- */
#define SMUON_NS_STATIC_SCRATCH_BYTES (32u << 20)

smuon_status smuon_ns_static(const smuon_mat* M_in, const smuon_mat* U_out, int32_t n_mats,
                             const smuon_mat* G, float beta,
                             float a, float b, float c, int32_t iters, float eps, uint32_t flags,
                             const smuon_mat* Q_out, const int32_t* d_skip_if,
                             int32_t* d_status, void* stream);

/* ------------------------------------------------------------------------
 * smuon_sign_pack -- entrywise sign and 1-bit packing of M workers' outputs.
 *
 * SignMuon summary, algorithm flow step 2 (S = sign(U)) and step 3 all-gather
 * variant (one bit per entry); all-reduce variant with int8 signs.
 * Readings: sign(u) = +1 iff u >= 0 (so -0 -> +1, NaN -> -1). Entry i of the
 * row-major flattening (i = row*cols + col, independent of ld) goes to bit
 * i % 32 of word i / 32; each worker's buffer holds words = ceil(N/128)*4
 * uint32 (16-byte multiple), pad bits zero.
 *
 *  U[M]        same-shape matrices (F32 or BF16), one per worker; or I8 sign
 *              matrices (an I8 smuon_ns output), packed by the same rule.
 *  packed      nullable device [M][words] uint32.
 *  signs_i8    nullable device [M][N] int8 (+1/-1), N = rows*cols.
 * At least one output must be given. M in 1..64.
 * ---------------------------------------------------------------------- */
smuon_status smuon_sign_pack(const smuon_mat* U, int32_t M, uint32_t* packed, int8_t* signs_i8,
                             void* stream);

/* ------------------------------------------------------------------------
 * smuon_vote -- majority vote over M workers.
 *
 * SignMuon summary, core mechanism 3 and flow steps 3-4: integer SUM of the
 * signs then sign(sum) (int8 all-reduce variant), or, from the bit-packed
 * buffers, sum = 2*popcount - M then the same threshold (all-gather variant).
 * Ties (even M) give tie_value.
 *
 *  packed      [M][words] as written by smuon_sign_pack, or NULL
 *  signs_i8    [M][N] int8, or NULL (exactly one of the two). The vote is the
 *              sign of the integer sum of the M rows, so a row may also hold a
 *              partial sum of several workers' signs (e.g. the result of an
 *              int8 SUM all-reduce, with M = 1); the per-entry total must stay
 *              within -127..127.
 *  vote        device [N] int8 in {-1, 0, +1}
 * M in 1..64.
 * ---------------------------------------------------------------------- */
smuon_status smuon_vote(const uint32_t* packed, const int8_t* signs_i8, int32_t M, int64_t N,
                        int8_t tie_value, int8_t* vote, void* stream);

/* ------------------------------------------------------------------------
 * smuon_update -- parameter update, batched over layers.
 *
 * SignMuon summary, algorithm flow step 4: W <- W - eta * S_bar, and step 5:
 * the optional local polar step applied to the voted matrix (a dense
 * direction D). Reading: one float32 subtraction W - f32(eta)*v (dense:
 * W - f32(f32(eta)*D)), then one round-to-nearest-even into W's type.
 *
 * Exactly one source per call:
 *  U[n_layers*M]     (worker-minor) -> fused sign / vote / update in one pass;
 *                    F32, BF16, or I8 sign matrices (entry >= 0 counts as +1;
 *                    I8 takes no packed_out: pack with smuon_sign_pack), or
 *                    BITS messages (a set bit counts as +1; the vote reads
 *                    M/8 bytes per entry; no packed_out: they are the message);
 *                    vote_kind SMUON_VOTE_POPCOUNT (bit masks + popcount) or
 *                    SMUON_VOTE_INT8 (integer sum); both give the same vote.
 *                    Optional outputs: packed_out[l] ([M][words] message, the
 *                    all-gather payload), vote_out[l] ([N] int8).
 *  votes[n_layers]   I8 matrices of -1/0/+1 (e.g. from smuon_vote).
 *  dense[n_layers]   F32 or BF16 direction D of W's shape.
 *  W[n_layers]       F32 or BF16, updated in place. With the U source W may be
 *                    NULL when packed_out or vote_out is given: the call then
 *                    only writes the message and the votes (the input of the
 *                    local polar step, step 5; shapes are taken from U).
 * packed_out and vote_out are host arrays of n_layers device pointers
 * (entries may be NULL) or NULL. M in 1..64. d_status: nullable device int32
 * for SMUON_DEV_* bits, as in smuon_ns.
 *
 * The 1-bit vote of a call whose layers all have BF16 W (contiguous, 16-byte
 * aligned, entry counts that are multiples of 8) and M <= 16 runs in its
 * bulk-copy form: a ring of shared-memory slots, filled by the bulk-copy
 * engine, holds W and the messages of 8192 entries per slot. Its pipeline
 * waits are bounded (about 2 s of SM clock); one that runs out ORs
 * SMUON_DEV_WAIT_TIMEOUT into *d_status, and the update is then incomplete.
 * ---------------------------------------------------------------------- */
#define SMUON_VOTE_POPCOUNT 0u
#define SMUON_VOTE_INT8     1u
#define SMUON_VOTE_TEST_WAIT_EXPIRY 0x100u  /* failure-detection test, not for use (OR-ed into vote_kind):
                                      the bulk-copy form of the 1-bit vote issues no copy and its waits
                                      are limited to 65536 SM clocks, so they run out: W is left as it was
                                      and SMUON_DEV_WAIT_TIMEOUT goes to d_status */

smuon_status smuon_update(const smuon_mat* W, int32_t n_layers,
                          const smuon_mat* U, const smuon_mat* votes, const smuon_mat* dense,
                          int32_t M, float eta, int8_t tie_value, uint32_t vote_kind,
                          uint32_t* const* packed_out, int8_t* const* vote_out, int32_t* d_status,
                          void* stream);

/* ------------------------------------------------------------------------
 * Plan handles: the same calls, prepared once and launched many times.
 *
 * smuon_ns_plan_create checks its arguments like smuon_ns, builds the plan
 * and uploads it into ws on `stream`; smuon_ns_execute then enqueues only the
 * kernels (d_skip_if as in smuon_ns). smuon_update_plan_create /
 * smuon_update_execute do the same for smuon_update. Between executions the
 * matrices' contents may change but not their addresses, and ws must hold
 * the plan (do not use it for another call). A handle is a small host object
 * owned by the caller; smuon_plan_destroy frees it (device memory is never
 * allocated). Executing a plan is capturable in a CUDA graph.
 * ---------------------------------------------------------------------- */
typedef struct smuon_plan_s* smuon_plan;

smuon_status smuon_ns_plan_create(const smuon_mat* M_in, const smuon_mat* U_out, int32_t n_mats,
                                  const smuon_mat* G, float beta, float a, float b, float c,
                                  int32_t iters, float eps, uint32_t flags, const smuon_mat* Q_out,
                                  void* ws, size_t ws_bytes, int32_t* d_status, void* stream,
                                  smuon_plan* out);
smuon_status smuon_ns_execute(smuon_plan plan, const int32_t* d_skip_if, void* stream);
smuon_status smuon_update_plan_create(const smuon_mat* W, int32_t n_layers, const smuon_mat* U,
                                      const smuon_mat* votes, const smuon_mat* dense, int32_t M,
                                      float eta, int8_t tie_value, uint32_t vote_kind,
                                      uint32_t* const* packed_out, int8_t* const* vote_out,
                                      int32_t* d_status, smuon_plan* out);
smuon_status smuon_update_execute(smuon_plan plan, void* stream);
void         smuon_plan_destroy(smuon_plan plan);

/* ------------------------------------------------------------------------
 * cachemuon_reuse_probe -- CacheMuon cached-transform reuse and residual
 * trigger, with the decision kept on the device.
 *
 * CacheMuon summary, section "Method" item 2 (D_hat = Q_{a_t} X_t with X_t
 * the normalised momentum) and item 3 (err = ||D_hat D_hat^T - I||_F /
 * ||I||_F; accept iff err <= gamma, else refresh with a fresh solve); section
 * "Significance" (a host-device sync for the check limited the authors'
 * wall-clock; here the check is fused into a device kernel).
 * Readings: I has the smaller side m, ||I||_F = sqrt(m); equality accepts;
 * NaN rejects; Q == NULL means no cache yet (first step): the call writes
 * err = +inf, accept = 0 and counts a miss without launching the GEMMs.
 *
 *  Q          BF16 m x m (as written by smuon_ns with SMUON_NS_EMIT_Q), or NULL
 *  M_t        F32 momentum (r x c); normalised inside, not modified
 *  D_hat      F32 or BF16 r x c output (written even when rejected)
 *  d_err      device float, d_accept device int32, d_counters device struct
 *  Intended use: probe, then smuon_ns(..., U_out = D_hat, SMUON_NS_EMIT_Q,
 *  Q_out = Q, d_skip_if = d_accept) which does nothing on a hit.
 * ---------------------------------------------------------------------- */
typedef struct {
  int64_t hits;
  int64_t misses;
  int64_t probes;      /* probes that ran the GEMMs (hits + misses - first steps) */
  int64_t reserved;
} cachemuon_counters;

smuon_status cachemuon_workspace_bytes(const smuon_mat* M_t, size_t* bytes);

smuon_status cachemuon_reuse_probe(const smuon_mat* Q, const smuon_mat* M_t, const smuon_mat* D_hat,
                                   float gamma, float eps, float* d_err, int32_t* d_accept,
                                   cachemuon_counters* d_counters, void* ws, size_t ws_bytes,
                                   int32_t* d_status, void* stream);

/* ------------------------------------------------------------------------
 * Counter-based gradient streams of the simulated workers (harness: the
 * pages describe no generator; this one makes a worker's gradient a pure
 * function of its coordinates so kernels can draw it instead of reading it).
 *
 * Entry i (row-major, whatever the leading dimension) of worker k's gradient
 * of matrix j at step t is sigma times Gaussian number i % 4 drawn from
 * Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As
 * Easy as 1, 2, 3", SC 2011) at counter (i/4 low word, i/4 high word, t, 0)
 * and key (seed_base + k, matrix_base + j): the counter's four output words
 * give two Box-Muller pairs, evaluated in float32 with every operation
 * rounded on its own (u1 = ((x0 >> 8) + 1) 2^-24, radius sqrt(-2 ln u1),
 * angle (x1 >> 30) pi/2 + ((x1 >> 8) & 0x3fffff) 2^-22 pi/2, ln, sin and cos
 * from fixed series), so any IEEE float32 evaluation of the same steps
 * reproduces the bits.
 * ---------------------------------------------------------------------- */
typedef struct {
  uint32_t seed_base;
  uint32_t matrix_base;
  float    sigma;
  uint32_t reserved;    /* 0 */
} smuon_grad_stream;

/* G[l*workers + k] (F32, rows x cols, any ld >= cols) <- worker k's gradient
 * of matrix matrix_base + l at step `step`. Enqueued on `stream`; errors:
 * SMUON_ERR_INVALID_ARG (NULL G or gs, workers < 1, n_layers < 1),
 * SMUON_ERR_SHAPE, SMUON_ERR_DTYPE (not F32). */
smuon_status smuon_harness_gaussian(const smuon_mat* G, int32_t n_layers, int32_t workers,
                                    const smuon_grad_stream* gs, uint32_t step, void* stream);

/* ------------------------------------------------------------------------
 * lionmuon_step -- one step of the LionMuon period-P schedule.
 *
 * LionMuon summary, section "Methodology" item 1 (a Muon step every P-th
 * iteration, Lion sign steps otherwise), item 2 (one shared double-EMA
 * buffer; G_hat = beta1*M + (1-beta1)*G) and item 4 (special cases), section
 * "Problem" (W - eta*sign(G_hat) and W - eta*msign(G_hat)).
 * Readings: steps are 1-indexed and step t is a Muon step iff P > 0 and
 * t % P == 0 (P = 0 means "never", i.e. P = infinity); with M workers a sign
 * step takes the majority vote of sign(G_hat^(m)) and a Muon step
 * orthogonalises mean_m G_hat^(m) (dense update); then every worker's EMA
 * becomes beta2*M + (1-beta2)*G. G_hat and the EMA are float32:
 * f32(beta*M) + f32(f32(1-beta)*G).
 *
 *  st->W[n_layers]          F32 or BF16 weights, updated in place
 *  st->mom[n_layers*M]      F32 EMA per worker (worker-minor), updated in place
 *  st->t                    steps taken; the call runs step t+1 and increments it
 *  G[n_layers*M]            F32 gradients (worker-minor), or NULL to draw them in-kernel from
 *                           st->grad (see smuon_harness_gaussian; no gradient bytes are read)
 *  ns_flags                 SMUON_NS_* flags of the Muon steps' Newton-Schulz call
 *                           (e.g. SMUON_NS_SPLIT_BF16), plus optionally
 *                           SMUON_LION_MUON_VOTE: the other reading of a Muon step
 *                           with M workers -- every worker orthogonalises its own
 *                           G_hat and the step is a Sign-Muon step, W -= eta *
 *                           vote(sign(NS(G_hat^(m)))) (SignMuon summary, flow
 *                           steps 2-5, applied to G_hat); M x n_layers Newton-Schulz
 *                           problems instead of n_layers, and a larger workspace
 * Workers 1..64.
 * ---------------------------------------------------------------------- */
#define SMUON_LION_MUON_VOTE 0x100u

typedef struct {
  int32_t                  n_layers;
  int32_t                  workers;
  const smuon_mat*         W;
  const smuon_mat*         mom;
  int64_t                  t;
  const smuon_grad_stream* grad;  /* nullable: with G == NULL, worker k's gradient of layer l at step
                                     t + 1 is drawn inside the kernels from stream (k, matrix_base + l) */
} lionmuon_state;

smuon_status lionmuon_workspace_bytes(const lionmuon_state* st, int32_t iters, uint32_t ns_flags,
                                      size_t* bytes);

smuon_status lionmuon_step(lionmuon_state* st, int32_t P, float beta1, float beta2, float eta,
                           float a, float b, float c, int32_t iters, int8_t tie_value,
                           uint32_t ns_flags, const smuon_mat* G, void* ws, size_t ws_bytes,
                           int32_t* d_status, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* SMUON_H */
