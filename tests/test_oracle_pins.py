"""Pins of the CPU oracle against facts that do not come from the oracle itself:
hand-derived worked examples (tests/golden), closed forms via LAPACK's SVD,
invariants stated on the pages, special cases and brute force on tiny inputs.
CPU only."""
import itertools
import json
import os

import numpy as np
import pytest
import torch

import oracle as O
import workloads as WL
from tests.conftest import GOLDEN


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _rel(a, b):
    return np.linalg.norm(np.asarray(a) - np.asarray(b)) / np.linalg.norm(np.asarray(b))


def _poly(s, coeffs, iters):
    a, b, c = coeffs
    for _ in range(iters):
        s = a * s + b * s ** 3 + c * s ** 5
    return s


# ---------------------------------------------------------------- Newton-Schulz
def test_ns_golden_diag():
    g = _golden("ns_diag_2x2.json")
    M = np.array(g["M"])
    for case in g["cases"]:
        U = O.newton_schulz(M, *case["coeffs"], case["iters"], eps=1e-7)
        np.testing.assert_allclose(U, np.array(case["U"]), rtol=g["rtol"], atol=1e-12)


@pytest.mark.parametrize("shape", [(4, 6), (6, 4), (16, 16), (32, 48), (96, 64), (1, 9)])
@pytest.mark.parametrize("coeffs", [WL.CUBIC, WL.QUINTIC])
@pytest.mark.parametrize("iters", [1, 2, 5])
def test_ns_svd_closed_form(shape, coeffs, iters):
    """NS acts on singular values only: NS_K(M) = U diag(f^K(sigma/(||M||_F+eps))) V^T."""
    rng = np.random.default_rng(7)
    M = rng.standard_normal(shape)
    U, S, Vt = np.linalg.svd(M, full_matrices=False)
    s = S / (np.sqrt(np.sum(S ** 2)) + 1e-7)
    expect = (U * _poly(s, coeffs, iters)) @ Vt
    got = O.newton_schulz(M, *coeffs, iters, eps=1e-7)
    assert got.shape == M.shape
    assert _rel(got, expect) < 1e-10


def test_ns_cubic_converges_to_polar_factor():
    """Enough cubic steps on singular values inside (0, sqrt(3)) reach U V^T (the
    exact polar factor the iteration stands in for)."""
    rng = np.random.default_rng(3)
    U, _ = np.linalg.qr(rng.standard_normal((24, 24)))
    V, _ = np.linalg.qr(rng.standard_normal((40, 24)))
    S = np.linspace(0.3, 1.0, 24)
    M = (U * S) @ V.T
    got = O.newton_schulz(M, *WL.CUBIC, 40, normalize=False)
    assert _rel(got, U @ V.T) < 1e-12


def test_orthogonal_input_fixed_point():
    """Orthogonal input maps to itself for the exact polar factor and for the
    cubic core without normalisation (f(1) = 1); the quintic scales it by f(1)."""
    rng = np.random.default_rng(5)
    Q, _ = np.linalg.qr(rng.standard_normal((32, 32)))
    Uq, _, Vq = np.linalg.svd(Q)
    assert _rel(Uq @ Vq, Q) < 1e-13
    assert _rel(O.newton_schulz(Q, *WL.CUBIC, 5, normalize=False), Q) < 1e-13
    f1 = sum(WL.QUINTIC)
    assert _rel(O.newton_schulz(Q, *WL.QUINTIC, 1, normalize=False), f1 * Q) < 1e-13


@pytest.mark.parametrize("shape", [(8, 8), (12, 30), (30, 12)])
def test_spectral_norm_bounds(shape):
    """The normalised input has spectral norm <= ||.||_F = 1 (SignMuon summary,
    theory section: spectral norm of the update at most 1); the cubic keeps it
    <= 1 and the quintic stays under max_{[0,1]} f^K."""
    rng = np.random.default_rng(11)
    M = rng.standard_normal(shape) * 3.0
    assert np.linalg.norm(M * O.frobenius_scale(M, 1e-7), 2) <= 1.0
    grid = np.linspace(0, 1, 200001)
    for coeffs in (WL.CUBIC, WL.QUINTIC):
        for K in (1, 3, 5):
            bound = _poly(grid, coeffs, K).max()
            assert np.linalg.norm(O.newton_schulz(M, *coeffs, K), 2) <= bound + 1e-12
    assert np.linalg.norm(O.newton_schulz(M, *WL.CUBIC, 5), 2) <= 1.0 + 1e-12


def test_momentum_from_zero_and_ema_scalar_multiple():
    rng = np.random.default_rng(2)
    G1, G2 = rng.standard_normal((2, 6, 9))
    M1 = O.momentum(np.zeros((6, 9)), G1, 0.9)
    M2 = O.momentum(M1, G2, 0.9)
    np.testing.assert_allclose(M1, G1, rtol=0, atol=0)
    np.testing.assert_allclose(M2, 0.9 * G1 + G2, rtol=1e-15)
    # EMA form from zero is a scalar multiple, so the normalised NS output agrees
    ema = 0.1 * G1
    np.testing.assert_allclose(O.newton_schulz(ema, *WL.QUINTIC, 2, eps=0.0),
                               O.newton_schulz(M1, *WL.QUINTIC, 2, eps=0.0), rtol=1e-12, atol=1e-14)


# ----------------------------------------------------------------------- signs
def test_sign_convention():
    u = np.array([0.0, -0.0, np.nan, -1e-30, 1e-30, -np.inf, np.inf], np.float32)
    np.testing.assert_array_equal(O.sign_extract(u), [1, 1, -1, -1, 1, -1, 1])


def test_pack_golden():
    g = _golden("pack_bits_example.json")
    S = -np.ones(np.prod(g["shape"]), np.int8)
    S[g["positive_entries"]] = 1
    np.testing.assert_array_equal(O.pack_bits(S.reshape(g["shape"])), np.array(g["words"], np.uint32))


@pytest.mark.parametrize("n", [1, 31, 32, 33, 127, 128, 129, 1000, 4097])
def test_pack_roundtrip_and_padding(n):
    rng = np.random.default_rng(n)
    S = np.where(rng.random(n) < 0.5, 1, -1).astype(np.int8)
    w = O.pack_bits(S)
    assert w.size == O.packed_words(n) and (w.size * 4) % 16 == 0
    np.testing.assert_array_equal(O.unpack_bits(w, n), S)
    # every bit past entry n-1 is zero
    all_bits = np.unpackbits(w.view(np.uint8), bitorder="little")
    assert not all_bits[n:].any()
    # bits set == positives (independent popcount over bytes)
    assert int(all_bits.sum()) == int((S > 0).sum())


def test_payload_bytes():
    """One bit per entry (32x less than float32) or int8 (4x less), SignMuon
    summary, communication efficiency."""
    n = 768 * 2304
    assert O.packed_words(n) * 4 * 32 == n * 4
    assert n * 1 * 4 == n * 4


# ------------------------------------------------------------------------ vote
def test_vote_truth_table_m3():
    g = _golden("vote_m3_truth_table.json")
    for row in g["rows"]:
        signs = [np.array([s], np.int8) for s in row["signs"]]
        assert O.vote_from_signs(signs)[0] == row["vote"]
        packed = [O.pack_bits(s) for s in signs]
        assert O.vote_from_packed(packed, 3, 1)[0] == row["vote"]


@pytest.mark.parametrize("M", range(1, 11))
@pytest.mark.parametrize("tie", [-1, 0, 1])
def test_popcount_vote_equals_int8_vote_exhaustive(M, tie):
    patterns = np.array(list(itertools.product([-1, 1], repeat=M)), np.int8)  # [2^M, M]
    signs = [patterns[:, m].copy() for m in range(M)]
    n = patterns.shape[0]
    v8 = O.vote_from_signs(signs, tie)
    vp = O.vote_from_packed([O.pack_bits(s) for s in signs], M, n, tie)
    np.testing.assert_array_equal(v8, vp)
    # brute force: count the +1s directly
    pos = (patterns > 0).sum(axis=1)
    expect = np.where(2 * pos > M, 1, np.where(2 * pos < M, -1, tie))
    np.testing.assert_array_equal(v8, expect)


@pytest.mark.parametrize("M", [16, 31, 64])
def test_popcount_vote_equals_int8_vote_random(M):
    rng = np.random.default_rng(M)
    n = 3000
    signs = [np.where(rng.random(n) < 0.5, 1, -1).astype(np.int8) for _ in range(M)]
    np.testing.assert_array_equal(O.vote_from_signs(signs),
                                  O.vote_from_packed([O.pack_bits(s) for s in signs], M, n))


@pytest.mark.parametrize("M", [1, 2, 3, 8])
def test_vote_identical_is_identity(M):
    rng = np.random.default_rng(M)
    S = np.where(rng.random((7, 13)) < 0.5, 1, -1).astype(np.int8)
    np.testing.assert_array_equal(O.vote_from_signs([S] * M), S)


def test_vote_symmetry():
    rng = np.random.default_rng(1)
    signs = [np.where(rng.random(500) < 0.5, 1, -1).astype(np.int8) for _ in range(6)]
    v = O.vote_from_signs(signs, 0)
    vn = O.vote_from_signs([-s for s in signs], 0)
    np.testing.assert_array_equal(vn, -v)


# ---------------------------------------------------------------------- update
def test_bf16_golden_bits():
    g = _golden("bf16_rne_bits.json")
    for case in g["cases"]:
        f = np.array([int(case["f32"], 16)], np.uint32).view(np.float32)
        got = O.bf16_round(f).view(np.uint32)[0] >> 16
        assert got == int(case["bf16"], 16), case


def test_bf16_matches_torch_conversion():
    rng = np.random.default_rng(9)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10.0 ** rng.integers(-40, 38, 100000),
                        np.array([0.0, -0.0, np.inf, -np.inf, 3.0e38, -3.4e38, 1e-45, -1e-45], np.float32)]).astype(np.float32)
    mine = O.bf16_round(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    np.testing.assert_array_equal(mine.view(np.uint32), ref.view(np.uint32))
    assert np.isnan(O.bf16_round(np.array([np.nan], np.float32)))[0]


def test_update_golden():
    g = _golden("update_rounding.json")
    for case in g["cases"]:
        W = np.array([case["W"]], np.float32)
        got = O.update_with_vote(W, np.array([case["vote"]]), case["eta"], case["dtype"])
        assert got[0] == np.float32(case["expect"]), case


def test_update_matches_torch_arithmetic():
    rng = np.random.default_rng(4)
    W = O.bf16_round(rng.standard_normal(20000).astype(np.float32) * 0.02)
    v = rng.integers(-1, 2, 20000).astype(np.int8)
    D = rng.standard_normal(20000).astype(np.float32)
    eta = 0.02
    tw = torch.from_numpy(W)
    ref = (tw - torch.tensor(eta, dtype=torch.float32) * torch.from_numpy(v).float()).to(torch.bfloat16).float()
    np.testing.assert_array_equal(O.update_with_vote(W, v, eta, "bf16"), ref.numpy())
    ref_d = (tw - (torch.tensor(eta, dtype=torch.float32) * torch.from_numpy(D))).to(torch.bfloat16).float()
    np.testing.assert_array_equal(O.update_dense(W, D, eta, "bf16"), ref_d.numpy())
    ref32 = tw - torch.tensor(eta, dtype=torch.float32) * torch.from_numpy(v).float()
    np.testing.assert_array_equal(O.update_with_vote(W, v, eta, "f32"), ref32.numpy())


def test_sign_muon_step_vote_kinds_agree():
    """The all-reduce (int8 sum) and all-gather (packed bits) variants give the
    same vote (SignMuon summary, algorithm flow step 3)."""
    rng = np.random.default_rng(8)
    shapes = [(8, 20), (20, 8)]
    W = [rng.standard_normal(s).astype(np.float32) for s in shapes]
    M = [[np.zeros(s) for _ in range(4)] for s in shapes]
    G = [[rng.standard_normal(s) for _ in range(4)] for s in shapes]
    r1 = O.sign_muon_step(W, M, G, 0.9, WL.QUINTIC, 2, 0.01, "f32", vote_kind="int8")
    r2 = O.sign_muon_step(W, M, G, 0.9, WL.QUINTIC, 2, 0.01, "f32", vote_kind="popcount")
    for a, b in zip(r1["vote"], r2["vote"]):
        np.testing.assert_array_equal(a, b)


# ------------------------------------------------------------------- CacheMuon
def test_cachemuon_q_reproduces_fresh_solve():
    """Q X_0 = X_K at the refresh step (reading R14)."""
    rng = np.random.default_rng(12)
    for shape in [(24, 40), (40, 24)]:
        M = rng.standard_normal(shape)
        D, Q = O.newton_schulz_with_q(M, *WL.QUINTIC, 5)
        np.testing.assert_allclose(D, O.newton_schulz(M, *WL.QUINTIC, 5), rtol=0, atol=1e-13)
        Dh, _ = O.cachemuon_probe(Q, M)
        np.testing.assert_allclose(Dh, D, rtol=0, atol=1e-12)


def test_cachemuon_probe_residual_closed_form():
    """With Q from the fresh solve and the same momentum, the residual is
    sqrt(sum_i (f^K(s_i)^2 - 1)^2) / sqrt(m), from the SVD of M."""
    rng = np.random.default_rng(13)
    M = rng.standard_normal((20, 50))
    _, Q = O.newton_schulz_with_q(M, *WL.QUINTIC, 5)
    _, err = O.cachemuon_probe(Q, M)
    S = np.linalg.svd(M, compute_uv=False)
    fk = _poly(S / (np.sqrt(np.sum(S ** 2)) + 1e-7), WL.QUINTIC, 5)
    expect = np.sqrt(np.sum((fk ** 2 - 1) ** 2)) / np.sqrt(20)
    assert abs(err - expect) < 1e-10 * max(1.0, expect)


def test_cachemuon_gamma_limits():
    momenta = list(WL.cachemuon_momenta((16, 24), 6, drift=0.05, seed0=99))
    out, _ = O.cachemuon_run(momenta, np.inf, WL.QUINTIC, 5)
    assert [acc for _, acc, _ in out] == [False] + [True] * 5
    out, _ = O.cachemuon_run(momenta, -1.0, WL.QUINTIC, 5)
    assert [acc for _, acc, _ in out] == [False] * 6
    for (D, _, _), M in zip(out, momenta):
        np.testing.assert_allclose(D, O.newton_schulz(M, *WL.QUINTIC, 5), rtol=0, atol=1e-13)


def test_cachemuon_nan_rejects():
    Q = np.eye(4)
    M = np.ones((4, 6))
    M[0, 0] = np.nan
    _, err = O.cachemuon_probe(Q, M)
    assert np.isnan(err) and not (err <= 15.0)


# ------------------------------------------------------------------- LionMuon
def _lion_inputs(seed=21, shapes=((6, 10), (10, 6)), workers=3, steps=5):
    rng = np.random.default_rng(seed)
    W = [O.bf16_round(rng.standard_normal(s).astype(np.float32) * 0.02) for s in shapes]
    Gs = [[[rng.standard_normal(s).astype(np.float32) for _ in range(workers)] for s in shapes]
          for _ in range(steps)]
    return W, Gs


def test_lionmuon_schedule_reading():
    kinds = []
    W, Gs = _lion_inputs()
    M = [[np.zeros(w.shape, np.float32) for _ in range(3)] for w in W]
    for t in range(1, 6):
        k, W, M = O.lionmuon_step(t, W, M, Gs[t - 1], 2, 0.9, 0.99, 1e-3, WL.QUINTIC, 2, "bf16")
        kinds.append(k)
    assert kinds == ["sign", "muon", "sign", "muon", "sign"]


def test_lionmuon_p1_is_pure_muon():
    """P = 1: every step is a Muon step on the Lion-interpolated momentum
    (LionMuon summary, special cases)."""
    W, Gs = _lion_inputs()
    M = [[np.zeros(w.shape, np.float32) for _ in range(3)] for w in W]
    Wr = [w.copy() for w in W]
    Mr = [[m.copy() for m in ms] for ms in M]
    for t in range(1, 6):
        _, W, M = O.lionmuon_step(t, W, M, Gs[t - 1], 1, 0.9, 0.99, 1e-3, WL.QUINTIC, 2, "bf16")
        # plain Muon with the same momentum rule, written directly
        for i in range(len(Wr)):
            gh = [(np.float32(0.9) * Mr[i][m]).astype(np.float32)
                  + (np.float32(np.float32(1) - np.float32(0.9)) * Gs[t - 1][i][m]).astype(np.float32)
                  for m in range(3)]
            D = O.newton_schulz(np.mean(np.stack(gh).astype(np.float64), 0), *WL.QUINTIC, 2)
            Wr[i] = O.update_dense(Wr[i], D, 1e-3, "bf16")
            Mr[i] = [(np.float32(0.99) * Mr[i][m]).astype(np.float32)
                     + (np.float32(np.float32(1) - np.float32(0.99)) * Gs[t - 1][i][m]).astype(np.float32)
                     for m in range(3)]
    for a, b in zip(W, Wr):
        np.testing.assert_array_equal(a, b)


def test_lion_interpolate_and_ema_golden():
    """Hand-derived float32 cases of the interpolation G_hat = beta1 M + (1-beta1) G
    and of the EMA update (same arithmetic with beta2), bit for bit, including
    two ties to even and the coefficient taken from f32(beta)."""
    g = _golden("lion_f32.json")
    for case in g["cases"]:
        M = np.array([case["M"]], np.float32)
        G = np.array([case["G"]], np.float32)
        want = int(case["expect_bits"], 16)
        for fn in (O.lion_interpolate, O.lion_ema):
            got = fn(M, G, case["beta"])
            assert got.dtype == np.float32
            assert int(got.view(np.uint32)[0]) == want, (fn.__name__, case)


def _bf16_torch(x):
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16).float().numpy()


def test_lionmuon_pinf_equal_betas_is_signum():
    """P = infinity with beta1 = beta2 and the EMA from zero: every step is a sign
    step on the EMA itself, i.e. Signum with a majority vote (LionMuon summary,
    special cases). The reference loop is written here with numpy float32
    arithmetic, a direct count of the positive signs and torch's bf16
    conversion, calling nothing of the oracle."""
    W, Gs = _lion_inputs(seed=22)
    beta, eta, workers = 0.9, 1e-3, 3
    M = [[np.zeros(w.shape, np.float32) for _ in range(workers)] for w in W]
    Ws = [w.copy() for w in W]
    Ms = [[m.copy() for m in ms] for ms in M]
    b32 = np.float32(beta)
    c32 = np.float32(np.float32(1.0) - b32)
    for t in range(1, 6):
        kind, W, M = O.lionmuon_step(t, W, M, Gs[t - 1], 0, beta, beta, eta, WL.QUINTIC, 2, "bf16")
        assert kind == "sign"
        for i in range(len(Ws)):
            new = []
            for m in range(workers):
                prod_m = np.multiply(b32, Ms[i][m], dtype=np.float32)
                prod_g = np.multiply(c32, Gs[t - 1][i][m], dtype=np.float32)
                new.append(np.add(prod_m, prod_g, dtype=np.float32))
            Ms[i] = new
            positives = sum((x >= 0).astype(np.int64) for x in new)
            v = np.where(2 * positives > workers, 1.0, -1.0).astype(np.float32)  # odd count: no ties
            Ws[i] = _bf16_torch(np.subtract(Ws[i], np.float32(eta) * v, dtype=np.float32))
    for a, b in zip(W, Ws):
        np.testing.assert_array_equal(a, b)
    for a, b in zip(M, Ms):
        for x, y in zip(a, b):
            np.testing.assert_array_equal(x, y)


@pytest.mark.parametrize("workers", [1, 2, 3, 4])
@pytest.mark.parametrize("shape", [(6, 10), (10, 6)])
def test_sign_muon_local_polar_identical_workers(workers, shape):
    """The local polar step (SignMuon summary, algorithm flow step 5) with M
    identical workers: the vote is the workers' common sign matrix S itself
    (no ties: the sum is M S), and the direction is the Newton-Schulz map of S,
    written here by its singular-value closed form; with W = 0 the update is
    -f32(f32(eta) D) exactly."""
    rng = np.random.default_rng(40 + workers)
    G = rng.standard_normal(shape)
    W = [np.zeros(shape, np.float32)]
    Ms = [[np.zeros(shape) for _ in range(workers)]]
    Gs = [[G.copy() for _ in range(workers)]]
    eta, iters = 0.02, 3
    out = O.sign_muon_step(W, Ms, Gs, 0.9, WL.QUINTIC, iters, eta, "f32", local_polar=True)
    # every worker orthogonalised the same momentum G: its sign matrix by the closed form
    Ug, Sg, Vgt = np.linalg.svd(G, full_matrices=False)
    Ug_ns = (Ug * _poly(Sg / (np.sqrt(np.sum(Sg ** 2)) + 1e-7), WL.QUINTIC, iters)) @ Vgt
    S = np.where(Ug_ns >= 0, 1.0, -1.0)
    np.testing.assert_array_equal(out["vote"][0], S.astype(np.int8))
    Us, Ss, Vst = np.linalg.svd(S, full_matrices=False)
    D = (Us * _poly(Ss / (np.sqrt(np.sum(Ss ** 2)) + 1e-7), WL.QUINTIC, iters)) @ Vst
    expect = -(np.float32(eta) * D.astype(np.float32)).astype(np.float32)
    np.testing.assert_allclose(out["W"][0], expect, rtol=3e-7, atol=0)
    # the dense step moves W by eta * D, not by eta * vote: they differ
    assert np.abs(out["W"][0] + np.float32(eta) * S.astype(np.float32)).max() > 1e-4


def test_ns_flops_counts():
    assert O.ns_flops(256, 256, 5, 0.0) == 5 * 4 * 256 ** 3
    assert O.ns_flops(4096, 4096, 5, 2.0) == 5 * 6 * 4096 ** 3
    assert O.ns_flops(3072, 768, 1, 2.0) == 4 * 768 ** 2 * 3072 + 2 * 768 ** 3


def test_lionmuon_muon_vote_is_sign_muon_on_g_hat():
    """The vote reading of the Muon step: each worker's G_hat is orthogonalised
    and the signs are voted. Written with the singular-value closed form of
    the iteration and a direct count of the signs, independent of the oracle's
    iteration and vote functions; three workers, odd count, so no ties."""
    W, Gs = _lion_inputs(seed=31)
    M = [[np.zeros(w.shape, np.float32) for _ in range(3)] for w in W]
    kind, Wn, Mn = O.lionmuon_step(1, W, M, Gs[0], 1, 0.9, 0.99, 1e-3, WL.QUINTIC, 2, "f32", muon_vote=True)
    assert kind == "muon"
    for i, w in enumerate(W):
        count = np.zeros(w.shape, np.int64)
        for m in range(3):
            gh = (np.float32(np.float32(1) - np.float32(0.9)) * Gs[0][i][m]).astype(np.float64)  # M = 0
            U, S, Vt = np.linalg.svd(gh, full_matrices=False)
            s = S / (np.sqrt(np.sum(S ** 2)) + 1e-7)
            ns = (U * _poly(s, WL.QUINTIC, 2)) @ Vt
            count += (ns >= 0)
        v = np.where(2 * count > 3, 1, -1)
        expect = (w.astype(np.float32) - np.float32(1e-3) * v.astype(np.float32)).astype(np.float32)
        np.testing.assert_array_equal(Wn[i], expect)
    # the EMA does not depend on the kind of step
    _, _, Md = O.lionmuon_step(1, W, M, Gs[0], 1, 0.9, 0.99, 1e-3, WL.QUINTIC, 2, "f32")
    for a, b in zip(Mn, Md):
        for x, y in zip(a, b):
            np.testing.assert_array_equal(x, y)


@pytest.mark.parametrize("shape", [(8, 40), (40, 8), (24, 24)])
@pytest.mark.parametrize("iters", [1, 3, 5])
def test_gram_only_solve_matches_the_x_iteration(shape, iters):
    """Iterating on the Gram matrix reaches the same X_K and Q as iterating on
    X: both equal the singular-value closed form."""
    rng = np.random.default_rng(11)
    M = rng.standard_normal(shape)
    D1, Q1 = O.newton_schulz_with_q(M, *WL.QUINTIC, iters)
    D2, Q2 = O.newton_schulz_gram_only(M, *WL.QUINTIC, iters)
    U, S, Vt = np.linalg.svd(M, full_matrices=False)
    s = S / (np.sqrt(np.sum(S ** 2)) + 1e-7)
    closed = (U * _poly(s, WL.QUINTIC, iters)) @ Vt
    assert _rel(D2, closed) < 1e-10
    assert _rel(D2, D1) < 1e-10 and _rel(Q2, Q1) < 1e-10
    # Q is a product of commuting symmetric factors: symmetric
    assert _rel(Q2, Q2.T) < 1e-12


@pytest.mark.parametrize("shape", [(6, 10), (10, 6), (12, 12)])
@pytest.mark.parametrize("coeffs,iters", [(WL.QUINTIC, 1), (WL.QUINTIC, 5), (WL.CUBIC, 5)])
def test_ns_spectral_scaling_closed_form(shape, coeffs, iters):
    """Spectral normalisation divides by the largest singular value, so the
    largest scaled singular value is (almost) exactly 1."""
    rng = np.random.default_rng(13)
    M = rng.standard_normal(shape)
    U, S, Vt = np.linalg.svd(M, full_matrices=False)
    s = S / (S.max() + 1e-7)
    assert abs(s.max() - 1.0) < 1e-6
    expect = (U * _poly(s, coeffs, iters)) @ Vt
    assert _rel(O.newton_schulz(M, *coeffs, iters, spectral=True), expect) < 1e-10
    # a rank-one matrix: spectral and Frobenius norms agree
    r1 = np.outer(rng.standard_normal(shape[0]), rng.standard_normal(shape[1]))
    assert _rel(O.newton_schulz(r1, *coeffs, iters, spectral=True), O.newton_schulz(r1, *coeffs, iters)) < 1e-12


def test_sign_muon_step_spectral_passes_the_scaling_through():
    """sign_muon_step(spectral=True) orthogonalises every worker's momentum
    with the spectral scaling: with one quintic step its U is the singular-
    value closed form p(s_i / s_max), a different matrix from the Frobenius
    step's, and the vote and update follow from those signs."""
    rng = np.random.default_rng(31)
    shape, M = (6, 9), 3
    W = [np.zeros(shape)]
    Ms = [[np.zeros(shape) for _ in range(M)]]
    G = [[rng.standard_normal(shape) for _ in range(M)]]
    out = O.sign_muon_step(W, Ms, G, 0.9, WL.QUINTIC, 1, 0.01, "f32", spectral=True)
    plain = O.sign_muon_step(W, Ms, G, 0.9, WL.QUINTIC, 1, 0.01, "f32")
    for k in range(M):
        Uk, S, Vt = np.linalg.svd(G[0][k], full_matrices=False)
        expect = (Uk * _poly(S / (S.max() + 1e-7), WL.QUINTIC, 1)) @ Vt
        assert _rel(out["U"][0][k], expect) < 1e-10
        assert _rel(out["U"][0][k], plain["U"][0][k]) > 1e-3
    v = O.vote_from_packed([O.pack_bits(O.sign_extract(u)) for u in out["U"][0]], M, 54).reshape(shape)
    np.testing.assert_array_equal(out["vote"][0], v)
    np.testing.assert_array_equal(out["W"][0], O.update_with_vote(W[0], v, 0.01, "f32"))


@pytest.mark.parametrize("honest,bad", [(3, 1), (4, 1), (5, 2), (6, 3)])
def test_vote_tolerates_a_minority_of_corrupted_workers(honest, bad):
    """The robustness the SignMuon summary's significance section claims for
    the majority vote, brute force: for every pattern of honest signs and every
    pattern of corrupted ones, an entry whose honest margin |sum| exceeds the
    number of corrupted workers keeps the honest vote."""
    hp = np.array(list(itertools.product([-1, 1], repeat=honest)), np.int8)     # [2^h, h]
    bp = np.array(list(itertools.product([-1, 1], repeat=bad)), np.int8)        # [2^b, b]
    H = np.repeat(hp, len(bp), axis=0)
    B = np.tile(bp, (len(hp), 1))
    signs = [H[:, k] for k in range(honest)] + [B[:, k] for k in range(bad)]
    v = O.vote_from_signs(signs, 0)
    margin = H.astype(np.int64).sum(axis=1)
    safe = np.abs(margin) > bad
    assert safe.any()
    np.testing.assert_array_equal(v[safe], np.sign(margin[safe]))
    # and the bound is tight: at margin == bad some corruption reaches a tie or flips the vote
    edge = np.abs(margin) == bad
    if edge.any():
        assert np.any(v[edge] != np.sign(margin[edge]))
