"""Helpers for the GPU parity tests: host<->device conversion and the
tolerance checks stated for the path (relative Frobenius error of the
Newton-Schulz output; sign disagreements only near zero)."""
import numpy as np
import torch


def dev(x, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(x)).to(device="cuda", dtype=dtype)


def host(t):
    return t.detach().float().cpu().numpy() if t.dtype != torch.int8 else t.cpu().numpy()


def rel_fro(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.linalg.norm(got - ref) / np.linalg.norm(ref))


def sign_disagreements(U_gpu, U_ref):
    """Entries where sign(U_gpu) != sign(U_ref) with the U >= 0 -> +1 rule;
    returns (fraction, max |U_ref| over those entries / max |U_ref|)."""
    U_gpu = np.asarray(U_gpu, np.float64)
    U_ref = np.asarray(U_ref, np.float64)
    dis = (U_gpu >= 0) != (U_ref >= 0)
    frac = float(dis.mean())
    worst = float(np.abs(U_ref[dis]).max() / np.abs(U_ref).max()) if dis.any() else 0.0
    return frac, worst


def check_ns_outputs(pairs, tol):
    """Acceptance criteria of the path over a set of (U_gpu, U_ref) pairs: the relative
    Frobenius error of each output <= tol; sign disagreements <= 1e-4 of all
    entries, each with |U_ref| < 1e-3 max|U_ref| of its matrix."""
    worst_err, n_dis, n_all, worst_mag = 0.0, 0, 0, 0.0
    for U_gpu, U_ref in pairs:
        e = rel_fro(U_gpu, U_ref)
        assert e <= tol, f"relative Frobenius error {e:.3e} > {tol} (shape {np.shape(U_ref)})"
        frac, worst = sign_disagreements(U_gpu, U_ref)
        worst_err = max(worst_err, e)
        n_dis += int(round(frac * np.size(U_ref)))
        n_all += np.size(U_ref)
        worst_mag = max(worst_mag, worst)
    assert n_dis <= 1e-4 * n_all, f"{n_dis} sign disagreements in {n_all} entries"
    assert worst_mag < 1e-3, f"a sign disagreement at |U|/max|U| = {worst_mag:.2e}"
    return worst_err, n_dis / max(n_all, 1), worst_mag
