"""Design check for the Newton-Schulz operand precision, on the CPU: the
tensor-core products restated in float32 torch with their operands rounded to
bf16 (plain: one product of the bf16 operands; split: x = hi + lo with
hi = bf16(x), lo = bf16(x - hi), and the three products hi*hi, hi*lo, lo*hi),
the a X term in float32 as the kernel's epilogue keeps it. Five quintic steps on
Gaussian momenta of the GPT-2 shapes, against the float64 oracle:

* plain BF16 misses the stated criteria (error about 2e-2, sign flips about 3e-3);
* keeping any one kind of product plain in every step misses them too, so no
  per-product precision choice passes;
* the split mode meets them; and with the first two steps plain it still does
  (the normalised singular values start near 1/sqrt(m), so the B X term of an
  early step is small beside a X), while three plain steps do not;
* carrying X between steps as its bf16 hi and lo parts alone (x ~ hi + lo,
  relative error near 2^-17, the operands the split products read anyway)
  instead of a float32 master, and taking the b A term from A's hi and lo
  parts instead of a float32 A, keeps the split mode within the criteria, with
  and without the plain leading steps; the kernels' split mode does both.

The GPU tests check the kernels' modes against the oracle directly."""
import numpy as np
import pytest
import torch

import oracle as O
import workloads as WL


def _bf(x):
    return x.to(torch.bfloat16).to(torch.float32)


def _prod(A, B, split):
    if not split:
        return _bf(A) @ _bf(B)
    Ah, Bh = _bf(A), _bf(B)
    Al, Bl = _bf(A - Ah), _bf(B - Bh)
    return Ah @ Bh + Ah @ Bl + Al @ Bh


def _hilo(x):
    hi = _bf(x)
    return hi + _bf(x - hi)


def _ns(M, modes, hilo_carry=False):
    """modes[k] = (gram, poly, axpy) split flags of step k; hilo_carry: X is kept
    between steps, and A read for the b A term, as bf16 hi + bf16 lo instead of
    float32."""
    a, b, c = WL.QUINTIC
    X = (M / (np.sqrt(np.sum(M.astype(np.float64) ** 2)) + 1e-7)).astype(np.float32)
    X = torch.from_numpy(X)
    for k, (g, p, x) in enumerate(modes):
        A = _prod(X, X.T.contiguous(), g)
        B = b * (_hilo(A) if hilo_carry else A) + c * _prod(A, A, p)
        X = a * X + _prod(B, X, x)
        if hilo_carry and k + 1 < len(modes):
            X = _hilo(X)
    return X.double().numpy()


def _criteria(U, R):
    err = np.linalg.norm(U - R) / np.linalg.norm(R)
    dis = (U >= 0) != (R >= 0)
    worst = np.abs(R[dis]).max() / np.abs(R).max() if dis.any() else 0.0
    return err, dis.mean(), worst


def _passes(U, R):
    err, frac, worst = _criteria(U, R)
    return err <= 1e-2 and frac <= 1e-4 and worst < 1e-3


SPLIT = (True, True, True)
PLAIN = (False, False, False)


@pytest.mark.parametrize("shape", [(768, 2304), (768, 768)])
def test_operand_precision_choices(shape):
    torch.set_num_threads(max(1, min(8, torch.get_num_threads())))
    M = np.random.default_rng(shape[0] * 7 + shape[1]).standard_normal(shape)
    R = O.newton_schulz(M, *WL.QUINTIC, 5)
    assert not _passes(_ns(M, [PLAIN] * 5), R)
    for one_plain in ((False, True, True), (True, False, True), (True, True, False)):
        assert not _passes(_ns(M, [one_plain] * 5), R)
    assert _passes(_ns(M, [SPLIT] * 5), R)
    lead2 = _ns(M, [PLAIN] * 2 + [SPLIT] * 3)
    assert _passes(lead2, R) and _criteria(lead2, R)[0] < 1e-3
    assert not _passes(_ns(M, [PLAIN] * 3 + [SPLIT] * 2), R)
    for lead in (0, 2):
        carried = _ns(M, [PLAIN] * lead + [SPLIT] * (5 - lead), hilo_carry=True)
        assert _passes(carried, R) and _criteria(carried, R)[0] < 1e-3


@pytest.mark.parametrize("shape", [(96, 320), (200, 96)])
def test_plain_leading_steps_on_small_matrices(shape):
    """Small matrices start with larger normalised singular values (near
    1/sqrt(m) + 1/sqrt(n)): one plain leading step still meets the criteria, two
    do not. The library therefore runs later plain steps only where the smaller
    side is at least 512."""
    M = np.random.default_rng(shape[0] * 7 + shape[1]).standard_normal(shape)
    R = O.newton_schulz(M, *WL.QUINTIC, 5)
    assert _passes(_ns(M, [PLAIN] + [SPLIT] * 4), R)
    assert not _passes(_ns(M, [PLAIN] * 2 + [SPLIT] * 3), R)
