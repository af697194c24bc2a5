"""Plain, slow CPU oracle of the Sign-Muon optimizer step and its two neighbours.

TEST INFRASTRUCTURE ONLY: used by ``tests/``, ``__graft_entry__.smoke()`` and
the benchmark's CPU-baseline leg, never by the product path. It shares no code
with the CUDA library and imports nothing from it.

Arithmetic is float64 numpy, one function per step of the method, with numpy's
matmul as the only library primitive. Where the method takes a discrete
decision or stores a rounded state (the update of a float32/bf16 weight, the
LionMuon interpolation whose sign is taken, the EMA stored in float32), the
oracle follows the kernel's precision exactly: float32 operations in the
stated order, and bf16 round-to-nearest-even written out from its definition.

Sources (page title, section):
  [SM]  "SignMuon: Communication-Efficient Distributed Muon Optimization"
        (technical summary page, section 2 "Method": core mechanism items 1-3,
        distributed algorithm flow steps 1-5, communication efficiency; and the
        English abstract).
  [CM]  "CacheMuon" technical summary, section "Method": fresh solve, cache
        reuse, residual-based trigger.
  [LM]  "LionMuon" technical summary, section "Methodology": alternating
        schedule, shared double-EMA momentum, special cases; section "Problem"
        for the two update kinds.

Readings where the pages are silent:
  R1  Sign-Muon momentum is heavy-ball M <- beta*M + G from zero, no Nesterov.
  R2  Newton-Schulz step X <- aX + b(XX^T)X + c(XX^T)^2 X with the coefficients
      given per workload (cubic (1.5,-0.5,0), quintic (3.4445,-4.7750,2.0315)).
  R3  The iteration runs on the smaller Gram side: a tall matrix is
      transposed, iterated, and transposed back.
  R4  Frobenius normalisation X0 = M / (||M||_F + eps), eps = 1e-7 (the spectral
      norm ||M||_2 in its place is the option the same section allows).
  R5  sign(u) = +1 if u >= 0 else -1 (so -0.0 -> +1, NaN -> -1).
  R6  Vote ties (even number of workers) give ``tie_value`` (0 by default).
  R8  Packed bits: entry i of the row-major flattening goes to bit i % 32 of
      32-bit word i // 32 (little-endian words); the buffer is padded with
      zero bits to a multiple of 4 words (16 bytes).
  R9  Update: W_new = round_dtype(f32(W) - f32(eta) * v), one float32
      subtraction, then one round-to-nearest-even to bf16 for bf16 weights.
      The dense form (local polar step, Muon step) is f32(W) - f32(f32(eta)*D).
  R11 LionMuon Muon steps orthogonalise the mean over workers of G_hat.
      Alternative (muon_vote): each worker orthogonalises its own G_hat and
      the Muon step votes on the signs, as a Sign-Muon step.
  R12 LionMuon EMA update M <- beta2*M + (1-beta2)*G after G_hat is formed.
  R13 Steps are 1-indexed; step t is a Muon step iff P > 0 and t % P == 0.
  R14 CacheMuon's cached left transform is Q = P_{K-1} ... P_1 P_0 with
      P_k = aI + bA_k + cA_k^2, so that Q X_0 = X_K.
  R15 Residual err = ||D D^T - I||_F / ||I||_F with I of the smaller side
      (||I||_F = sqrt(m)); accept iff err <= gamma (NaN rejects); no cache on
      the first step.

Parity pins for every function live in tests/test_oracle_pins.py.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "momentum", "frobenius_scale", "spectral_scale", "newton_schulz", "newton_schulz_with_q",
    "sign_extract", "pack_bits", "unpack_bits", "packed_words", "vote_from_signs",
    "vote_from_packed", "bf16_round", "update_with_vote", "update_dense",
    "newton_schulz_gram_only", "sign_muon_step", "cachemuon_probe", "cachemuon_run", "lion_interpolate",
    "lion_ema", "lionmuon_step", "ns_flops", "cachemuon_flops",
]


# --------------------------------------------------------------------------
# [SM] flow step 1: local momentum (reading R1)
# --------------------------------------------------------------------------
def momentum(M: np.ndarray, G: np.ndarray, beta: float) -> np.ndarray:
    """M_{t+1} = beta * M_t + G_t, in float64 ([SM] flow step 1; reading R1)."""
    return np.float64(beta) * np.asarray(M, np.float64) + np.asarray(G, np.float64)


# --------------------------------------------------------------------------
# [SM] core mechanism 1 / flow step 1: polar factor via Newton-Schulz
# --------------------------------------------------------------------------
def frobenius_scale(M: np.ndarray, eps: float) -> float:
    """s = 1 / (||M||_F + eps): the Frobenius normalisation before the iteration
    ([SM] section 4 hyper-parameters name Frobenius scaling; reading R4)."""
    M = np.asarray(M, np.float64)
    return 1.0 / (np.sqrt(np.sum(M * M)) + eps)


def _ns_core(X: np.ndarray, a: float, b: float, c: float, iters: int, track_q: bool):
    """K Newton-Schulz steps on a wide matrix X (rows <= cols).

    Each step forms the Gram A = X X^T, the left multiplier
    P = aI + bA + cA^2, and X <- P X (reading R2). When ``track_q`` is set
    the product Q = P_{K-1} ... P_0 is accumulated as well (reading R14).
    """
    m = X.shape[0]
    I = np.eye(m)
    Q = I.copy() if track_q else None
    for _ in range(iters):
        A = X @ X.T
        B = b * A + c * (A @ A)
        X = a * X + B @ X
        if track_q:
            Q = a * Q + B @ Q
    return X, Q


def spectral_scale(M: np.ndarray, eps: float) -> float:
    """s = 1 / (||M||_2 + eps): the spectral-norm normalisation, the other choice
    [SM] section 4 allows (largest singular value from LAPACK's SVD)."""
    return 1.0 / (np.linalg.norm(np.asarray(M, np.float64), 2) + eps)


def newton_schulz(M: np.ndarray, a: float, b: float, c: float, iters: int,
                  eps: float = 1e-7, normalize: bool = True, spectral: bool = False) -> np.ndarray:
    """Polar-factor approximation U = NS_K(M) in float64, same orientation as M.

    [SM] core mechanism 1 and flow step 1 (each worker orthogonalises its
    momentum with a Newton-Schulz iteration); [CM] problem statement (the
    iteration replaces an SVD). Readings R2, R3, R4 (spectral: the spectral
    norm instead of the Frobenius norm).
    """
    M = np.asarray(M, np.float64)
    tall = M.shape[0] > M.shape[1]
    X = M.T if tall else M
    if normalize:
        X = X * (spectral_scale(M, eps) if spectral else frobenius_scale(M, eps))
    X, _ = _ns_core(X, a, b, c, iters, False)
    return X.T if tall else X


def newton_schulz_with_q(M: np.ndarray, a: float, b: float, c: float, iters: int,
                         eps: float = 1e-7):
    """CacheMuon fresh solve: the direction D = NS_K(M) and the cached left
    transform Q (m x m, m the smaller side) with Q X_0 = X_K ([CM] method 1;
    reading R14). D is returned in M's orientation; Q acts on the wide form."""
    M = np.asarray(M, np.float64)
    tall = M.shape[0] > M.shape[1]
    X = (M.T if tall else M) * frobenius_scale(M, eps)
    X, Q = _ns_core(X, a, b, c, iters, True)
    return (X.T if tall else X), Q


def newton_schulz_gram_only(M: np.ndarray, a: float, b: float, c: float, iters: int,
                            eps: float = 1e-7):
    """The fresh solve iterated on the m x m Gram matrix ("Gram Newton-Schulz",
    [CM] method item 1): A_0 = X_0 X_0^T, then per step P_k = aI + bA_k + cA_k^2,
    Q_{k+1} = P_k Q_k and A_{k+1} = P_k A_k P_k; finally X_K = Q_K X_0. In exact
    arithmetic this is the iteration of newton_schulz_with_q (P_k is a
    polynomial in A_k, so X_{k+1} X_{k+1}^T = P_k A_k P_k). Returns (D, Q) like it."""
    M = np.asarray(M, np.float64)
    tall = M.shape[0] > M.shape[1]
    X0 = (M.T if tall else M) * frobenius_scale(M, eps)
    m = X0.shape[0]
    I = np.eye(m)
    A = X0 @ X0.T
    Q = I.copy()
    for _ in range(iters):
        P = a * I + b * A + c * (A @ A)
        Q = P @ Q
        A = P @ A @ P
    X = Q @ X0
    return (X.T if tall else X), Q


# --------------------------------------------------------------------------
# [SM] core mechanism 2, flow step 2: entrywise sign (reading R5)
# --------------------------------------------------------------------------
def sign_extract(U: np.ndarray) -> np.ndarray:
    """S = sign(U) in {-1, +1} as int8, with U >= 0 -> +1 (so -0.0 -> +1 and
    NaN -> -1) ([SM] flow step 2; reading R5)."""
    U = np.asarray(U)
    return np.where(U >= 0, 1, -1).astype(np.int8)


# --------------------------------------------------------------------------
# [SM] flow step 3, all-gather variant: 1 bit per entry (reading R8)
# --------------------------------------------------------------------------
def packed_words(n: int) -> int:
    """Words in one worker's packed buffer: ceil(n / 128) * 4 (16-byte padding)."""
    return ((n + 127) // 128) * 4


def pack_bits(S: np.ndarray) -> np.ndarray:
    """Packs a sign matrix into uint32 words: bit i % 32 of word i // 32 is 1
    iff entry i (row-major) is +1 ([SM] flow step 3 all-gather variant;
    communication efficiency: one bit per parameter; reading R8)."""
    flat = (np.asarray(S).reshape(-1) > 0).astype(np.uint64)
    nw = packed_words(flat.size)
    bits = np.zeros(nw * 32, np.uint64)
    bits[:flat.size] = flat
    place = np.uint64(1) << np.arange(32, dtype=np.uint64)
    return (bits.reshape(nw, 32) * place).sum(axis=1).astype(np.uint32)


def unpack_bits(words: np.ndarray, n: int) -> np.ndarray:
    """Inverse of ``pack_bits``: int8 signs (+1 for a set bit, -1 otherwise)."""
    w = np.asarray(words, np.uint32).astype(np.uint64)
    i = np.arange(n)
    bit = (w[i // 32] >> (i % 32).astype(np.uint64)) & np.uint64(1)
    return np.where(bit == 1, 1, -1).astype(np.int8)


# --------------------------------------------------------------------------
# [SM] core mechanism 3, flow steps 3-4: majority vote (readings R6, R7)
# --------------------------------------------------------------------------
def _threshold(total: np.ndarray, tie_value: int) -> np.ndarray:
    return np.where(total > 0, 1, np.where(total < 0, -1, tie_value)).astype(np.int8)


def vote_from_signs(signs, tie_value: int = 0) -> np.ndarray:
    """All-reduce variant: integer sum of the workers' signs, then sign(sum)
    with ties -> tie_value ([SM] core mechanism 3; flow step 3 all-reduce
    variant and step 4; reading R6)."""
    total = np.zeros(np.asarray(signs[0]).shape, np.int64)
    for s in signs:
        total += np.asarray(s, np.int64)
    return _threshold(total, tie_value)


def vote_from_packed(packed, workers: int, n: int, tie_value: int = 0) -> np.ndarray:
    """All-gather variant: per entry, the count of set bits over the workers'
    packed buffers gives sum = 2*count - M, then the same threshold
    ([SM] flow step 3 all-gather variant and step 4). Flat result of n int8."""
    count = np.zeros(n, np.int64)
    for w in packed:
        w = np.asarray(w, np.uint32).astype(np.uint64)
        idx = np.arange(n)
        bits = (w[idx // 32] >> (idx % 32).astype(np.uint64)) & np.uint64(1)
        count += bits.astype(np.int64)
    return _threshold(2 * count - workers, tie_value)


# --------------------------------------------------------------------------
# [SM] flow step 4: parameter update (readings R9, R10)
# --------------------------------------------------------------------------
def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even), returned as the
    float32 values bf16 holds. Written from the definition of the format: keep
    the top 16 bits of the float32 pattern, rounding the dropped 16 bits to
    nearest with ties to the even kept pattern; NaN stays a (quiet) NaN."""
    f = np.ascontiguousarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    keep = u >> 16
    dropped = u & 0xFFFF
    round_up = (dropped > 0x8000) | ((dropped == 0x8000) & ((keep & 1) == 1))
    keep = keep + round_up.astype(np.uint64)
    out = (keep.astype(np.uint32) << 16)
    nan = np.isnan(f)
    out = np.where(nan, (u.astype(np.uint32) & 0xFFFF0000) | 0x00400000, out).astype(np.uint32)
    return out.view(np.float32).reshape(f.shape)


def _store(x32: np.ndarray, dtype: str) -> np.ndarray:
    return bf16_round(x32) if dtype == "bf16" else x32.astype(np.float32)


def update_with_vote(W: np.ndarray, vote: np.ndarray, eta: float, dtype: str) -> np.ndarray:
    """W_{t+1} = W_t - eta * vote, computed as one float32 subtraction and stored
    in W's type ([SM] flow step 4; reading R9). eta*vote is exact in float32
    because the vote is -1, 0 or +1."""
    W32 = np.asarray(W, np.float32)
    ev = (np.float32(eta) * np.asarray(vote, np.float32).reshape(W32.shape)).astype(np.float32)
    return _store((W32 - ev).astype(np.float32), dtype)


def update_dense(W: np.ndarray, D: np.ndarray, eta: float, dtype: str) -> np.ndarray:
    """W_{t+1} = W_t - eta * D for a dense direction (the optional local polar
    step, [SM] flow step 5; a Muon step, [LM] problem section): product
    rounded to float32, then one float32 subtraction, then W's type (R9)."""
    W32 = np.asarray(W, np.float32)
    ed = (np.float32(eta) * np.asarray(D, np.float32)).astype(np.float32)
    return _store((W32 - ed).astype(np.float32), dtype)


# --------------------------------------------------------------------------
# whole Sign-Muon step ([SM] flow steps 1-5)
# --------------------------------------------------------------------------
def sign_muon_step(W_layers, M_layers, G_layers, beta, coeffs, iters, eta, w_dtype,
                   tie_value=0, vote_kind="popcount", local_polar=False, eps=1e-7, spectral=False):
    """One distributed Sign-Muon step over a set of layers, with the M workers
    simulated: per layer and worker, momentum -> Newton-Schulz polar factor ->
    sign; then the vote over workers and the update; optionally a local polar
    step on the voted matrix ([SM] flow steps 1-5). spectral: the spectral-norm
    normalisation of reading R4 in every Newton-Schulz call.

    Returns dict(W=[...], M=[[...]], U=[[...]], vote=[...]) (new lists)."""
    a, b, c = coeffs
    W_out, M_out, U_out, V_out = [], [], [], []
    for W, Ms, Gs in zip(W_layers, M_layers, G_layers):
        Ms_new = [momentum(Mm, Gm, beta) for Mm, Gm in zip(Ms, Gs)]
        Us = [newton_schulz(Mm, a, b, c, iters, eps, spectral=spectral) for Mm in Ms_new]
        signs = [sign_extract(U) for U in Us]
        if vote_kind == "int8":
            v = vote_from_signs(signs, tie_value)
        else:
            n = signs[0].size
            v = vote_from_packed([pack_bits(s) for s in signs], len(signs), n,
                                 tie_value).reshape(signs[0].shape)
        if local_polar:
            D = newton_schulz(v.astype(np.float64), a, b, c, iters, eps, spectral=spectral)
            Wn = update_dense(W, D, eta, w_dtype)
        else:
            Wn = update_with_vote(W, v, eta, w_dtype)
        W_out.append(Wn)
        M_out.append(Ms_new)
        U_out.append(Us)
        V_out.append(v)
    return dict(W=W_out, M=M_out, U=U_out, vote=V_out)


# --------------------------------------------------------------------------
# [CM] method: fresh solve, cache reuse, residual trigger (R14, R15)
# --------------------------------------------------------------------------
def cachemuon_probe(Q: np.ndarray, M_t: np.ndarray, eps: float = 1e-7):
    """Candidate D_hat = Q X_t with X_t the normalised momentum (wide form),
    and its orthogonality residual err = ||D D^T - I||_F / ||I||_F
    ([CM] method 2 and 3; reading R15). D_hat is returned in M_t's orientation."""
    M = np.asarray(M_t, np.float64)
    tall = M.shape[0] > M.shape[1]
    X = (M.T if tall else M) * frobenius_scale(M, eps)
    D = np.asarray(Q, np.float64) @ X
    m = D.shape[0]
    R = D @ D.T - np.eye(m)
    err = np.sqrt(np.sum(R * R)) / np.sqrt(m)
    return (D.T if tall else D), float(err)


def cachemuon_run(momenta, gamma, coeffs, iters, eps=1e-7):
    """CacheMuon schedule over a sequence of momenta: no cache on the first
    step; afterwards probe the cached transform, accept iff err <= gamma
    (NaN rejects), else run the fresh solve and refresh Q ([CM] method 1-3).

    Returns per-step (direction, accepted, err) and the final Q."""
    a, b, c = coeffs
    Q = None
    out = []
    for M in momenta:
        if Q is not None:
            D, err = cachemuon_probe(Q, M, eps)
            if err <= gamma:
                out.append((D, True, err))
                continue
        else:
            err = float("inf")
        D, Q = newton_schulz_with_q(M, a, b, c, iters, eps)
        out.append((D, False, err))
    return out, Q


# --------------------------------------------------------------------------
# [LM] methodology: period-P alternation with a shared double EMA
# --------------------------------------------------------------------------
def lion_interpolate(M: np.ndarray, G: np.ndarray, beta1: float) -> np.ndarray:
    """G_hat = beta1 * M + (1 - beta1) * G ([LM] methodology item 2), in the
    kernel's float32: f32(beta1*M) + f32(c1*G) with c1 = f32(1 - beta1),
    because the sign of G_hat is a decision taken in that precision."""
    b1 = np.float32(beta1)
    c1 = np.float32(np.float32(1.0) - b1)
    M = np.asarray(M, np.float32)
    G = np.asarray(G, np.float32)
    return ((b1 * M).astype(np.float32) + (c1 * G).astype(np.float32)).astype(np.float32)


def lion_ema(M: np.ndarray, G: np.ndarray, beta2: float) -> np.ndarray:
    """M <- beta2 * M + (1 - beta2) * G after G_hat is formed ([LM]
    methodology item 2, double EMA; reading R12), stored in float32 with the
    same operation order as ``lion_interpolate``."""
    return lion_interpolate(M, G, beta2)


def lionmuon_step(t, W_layers, M_layers, G_layers, period, beta1, beta2, eta, coeffs,
                  iters, w_dtype, tie_value=0, eps=1e-7, muon_vote=False):
    """Step t (1-indexed) of LionMuon with M simulated workers.

    Muon step iff period > 0 and t % period == 0 ([LM] methodology item 1;
    reading R13): W <- W - eta * NS(mean_m G_hat^(m)) (reading R11, dense
    update). With muon_vote, the alternative reading of R11: every worker
    orthogonalises its own G_hat^(m) and the Muon step is a Sign-Muon step,
    W <- W - eta * vote(sign(NS(G_hat^(m)))) ([SM] flow steps 2-5 applied to
    G_hat). Otherwise a Lion sign step: W <- W - eta * vote(sign(G_hat^(m)))
    ([LM] problem section; the vote follows [SM]). Both kinds then update the
    shared EMA (reading R12). Returns (kind, W list, M lists)."""
    a, b, c = coeffs
    muon = period > 0 and t % period == 0
    W_out, M_out = [], []
    for W, Ms, Gs in zip(W_layers, M_layers, G_layers):
        Gh = [lion_interpolate(Mm, Gm, beta1) for Mm, Gm in zip(Ms, Gs)]
        if muon and muon_vote:
            U = [newton_schulz(g.astype(np.float64), a, b, c, iters, eps) for g in Gh]
            v = vote_from_signs([sign_extract(u) for u in U], tie_value)
            Wn = update_with_vote(W, v, eta, w_dtype)
        elif muon:
            mean = np.mean(np.stack([g.astype(np.float64) for g in Gh]), axis=0)
            D = newton_schulz(mean, a, b, c, iters, eps)
            Wn = update_dense(W, D, eta, w_dtype)
        else:
            v = vote_from_signs([sign_extract(g) for g in Gh], tie_value)
            Wn = update_with_vote(W, v, eta, w_dtype)
        W_out.append(Wn)
        M_out.append([lion_ema(Mm, Gm, beta2) for Mm, Gm in zip(Ms, Gs)])
    return ("muon" if muon else "sign"), W_out, M_out


# --------------------------------------------------------------------------
# work counts (for reports; not part of the method)
# --------------------------------------------------------------------------
def ns_flops(rows: int, cols: int, iters: int, c: float, with_q: bool = False) -> int:
    """Nominal Newton-Schulz flops: per step 2m^2 n (Gram) + 2m^3 (A^2, skipped
    when c == 0) + 2m^2 n (B X), plus 2m^3 per step for accumulating Q."""
    m, n = min(rows, cols), max(rows, cols)
    per = 4 * m * m * n + (2 * m ** 3 if c != 0 else 0) + (2 * m ** 3 if with_q else 0)
    return per * iters


def cachemuon_flops(rows: int, cols: int) -> dict:
    """Reuse D = QX costs 2m^2 n; the probe D D^T costs 2m^2 n."""
    m, n = min(rows, cols), max(rows, cols)
    return dict(reuse=2 * m * m * n, probe=2 * m * m * n)
