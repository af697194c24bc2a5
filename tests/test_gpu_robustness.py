"""Failure handling on the GPU without a GPU fault.

* A corrupted worker, made on the host: one worker's message inverted, zeroed
  or replaced by a copy of another's before the vote (the majority vote is
  what the SignMuon summary's significance section calls robust). The kernels
  must give the oracle's vote of the same corrupted inputs, bit for bit, and
  the honest majority wherever its margin exceeds the corrupted count.
* Out-of-bounds writes: every output of the main kernels sits between canary
  bytes that must come back untouched (a stand-in for a memory checker).
* Checkpoint and resume: a LionMuon run (gradients drawn in-kernel from the
  counter-based streams) and a CacheMuon schedule stopped, saved, restored
  into fresh buffers and continued equal the uninterrupted runs bit for bit.
"""
import os

import numpy as np
import pytest
import torch

import matrix_aware_sign_b200 as S
import oracle as O
import workloads as WL
from matrix_aware_sign_b200 import checkpoint as C
from tests.gpu_util import dev, host

pytestmark = pytest.mark.gpu


# ------------------------------------------------------------------ a corrupted worker
@pytest.mark.parametrize("corruption", ["inverted", "zeroed", "copied"])
@pytest.mark.parametrize("source", ["messages", "packed_vote", "u"])
def test_vote_with_a_corrupted_worker(corruption, source):
    M, bad, shapes = 5, 2, [(64, 147), (96, 128)]
    W = WL.weights(shapes, "normal002", "f32")
    U = [WL.synthetic_polar_outputs(s, M, seed=70 + i, dtype="f32") for i, s in enumerate(shapes)]
    for i, s in enumerate(shapes):
        if corruption == "inverted":
            U[i][bad] = -U[i][bad]
        elif corruption == "zeroed":
            U[i][bad] = np.full(s, -1.0, np.float32)  # every bit clear: all signs -1
        else:
            U[i][bad] = U[i][0].copy()
    signs = [[O.sign_extract(u) for u in layer] for layer in U]
    Wd = [dev(w) for w in W]
    eta = 0.01
    if source == "messages":
        msgs = [[S.Bits(dev(O.pack_bits(sg).view(np.int32), torch.int32), *s) for sg in layer]
                for s, layer in zip(shapes, signs)]
        S.smuon_update(Wd, eta, U=msgs, M=M)
    elif source == "packed_vote":
        votes = []
        for i, (r, c) in enumerate(shapes):
            packed = dev(np.stack([O.pack_bits(sg) for sg in signs[i]]).view(np.int32), torch.int32)
            v = torch.zeros(r * c, dtype=torch.int8, device="cuda")
            S.smuon_vote(M, r * c, v, packed=packed)
            votes.append(v.view(r, c))
        S.smuon_update(Wd, eta, votes=votes)
    else:
        S.smuon_update(Wd, eta, U=[[dev(u) for u in layer] for layer in U], M=M)
    torch.cuda.synchronize()
    for i, s in enumerate(shapes):
        v = O.vote_from_signs(signs[i])
        np.testing.assert_array_equal(host(Wd[i]), O.update_with_vote(W[i], v, eta, "f32"))
        honest = sum(signs[i][k].astype(np.int64) for k in range(M) if k != bad)
        safe = np.abs(honest) > 1  # one corrupted worker cannot overturn a margin of two
        np.testing.assert_array_equal(v[safe], np.sign(honest[safe]))


# ------------------------------------------------------------------ canaries around every output
CANARY = 0xA5


class Padded:
    """A tensor of `shape` and `dtype` placed between 256 canary bytes on each side."""

    def __init__(self, shape, dtype, fill=0):
        n = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
        self.raw = torch.full((n + 512,), CANARY, dtype=torch.uint8, device="cuda")
        self.t = self.raw[256:256 + n].view(dtype).view(shape)
        if fill is not None:
            self.t.fill_(fill)

    def intact(self):
        return bool(torch.all(self.raw[:256] == CANARY)) and bool(torch.all(self.raw[-256:] == CANARY))


def test_outputs_stay_inside_their_buffers():
    shapes, M = [(64, 147), (96, 320), (352, 64), (33, 128)], 3
    rng = np.random.default_rng(2)
    bufs = []
    Mom = [Padded(s, torch.float32) for s in shapes for _ in range(M)]
    G = [dev(rng.standard_normal(s).astype(np.float32)) for s in shapes for _ in range(M)]
    Uf = [Padded(s, torch.float32) for s in shapes for _ in range(M)]
    Ub = [Padded(s, torch.bfloat16) for s in shapes for _ in range(M)]
    Ui = [Padded(s, torch.int8) for s in shapes for _ in range(M)]
    bufs += Mom + Uf + Ub + Ui
    for flags in (0, S.NS_SPLIT_BF16, S.NS_FP32_REF):
        S.smuon_ns([m.t for m in Mom], [u.t for u in Uf], *WL.QUINTIC, 3, G=G, beta=0.9, flags=flags)
    S.smuon_ns([m.t for m in Mom], [u.t for u in Ub], *WL.QUINTIC, 1, G=G, beta=0.9)
    S.smuon_ns([m.t for m in Mom], [u.t for u in Ui], *WL.QUINTIC, 2, G=G, beta=0.9, flags=S.NS_SPLIT_BF16)
    bit_shapes = [s for s in shapes if s[1] % 32 == 0]
    Mb = [dev(rng.standard_normal(s).astype(np.float32)) for s in bit_shapes for _ in range(M)]
    words = [Padded((S.packed_words(r * c),), torch.int32) for r, c in bit_shapes for _ in range(M)]
    bufs += words
    bits = [S.Bits(w.t, r, c) for w, (r, c) in zip(words, [s for s in bit_shapes for _ in range(M)])]
    S.smuon_ns(Mb, bits, *WL.QUINTIC, 5, flags=S.NS_SPLIT_BF16 | S.ns_plain_lead(2))
    L = len(shapes)
    Wd = [Padded(s, torch.bfloat16) for s in shapes]
    packed = [Padded((M, S.packed_words(r * c)), torch.int32) for r, c in shapes]
    votes = [Padded((r * c,), torch.int8) for r, c in shapes]
    signs = [Padded((M, r * c), torch.int8) for r, c in shapes]
    bufs += Wd + packed + votes + signs
    for kind in (S.VOTE_POPCOUNT, S.VOTE_INT8):
        S.smuon_update([w.t for w in Wd], 0.01, U=[[u.t for u in Ub[l * M:(l + 1) * M]] for l in range(L)], M=M,
                       vote_kind=kind, packed_out=[p.t for p in packed], vote_out=[v.t for v in votes])
    S.smuon_update([w.t for w in Wd], 0.01, U=[[u.t for u in Ui[l * M:(l + 1) * M]] for l in range(L)], M=M,
                   vote_kind=S.VOTE_INT8)
    Wb = [Wd[l] for l, s in enumerate(shapes) if s[1] % 32 == 0]
    S.smuon_update([w.t for w in Wb], 0.01, U=[bits[j * M:(j + 1) * M] for j in range(len(Wb))], M=M)
    for l, (r, c) in enumerate(shapes):
        S.smuon_sign_pack([u.t for u in Ub[l * M:(l + 1) * M]], packed=packed[l].t, signs_i8=signs[l].t)
        S.smuon_vote(M, r * c, votes[l].t, packed=packed[l].t)
        S.smuon_vote(M, r * c, votes[l].t, signs_i8=signs[l].t)
    S.smuon_update([w.t for w in Wd], 0.01, votes=[v.t.view(s) for v, s in zip(votes, shapes)])
    S.smuon_update([w.t for w in Wd], 0.01, dense=[u.t for u in Uf[::M]])
    # LionMuon: W and every worker's EMA
    lw = [Padded(s, torch.bfloat16) for s in shapes]
    lm = [[Padded(s, torch.float32) for _ in range(M)] for s in shapes]
    bufs += lw + [m for layer in lm for m in layer]
    opt = S.LionMuon([w.t for w in lw], [[m.t for m in layer] for layer in lm], grad=S.GradStream(3, 0, 1.0, 0))
    for _ in range(4):
        S.lionmuon_step(opt, None, 2, 0.9, 0.99, 1e-3, *WL.QUINTIC, 5, ns_flags=S.NS_SPLIT_BF16)
    # CacheMuon probe outputs
    cm_m = dev(rng.standard_normal((200, 96)).astype(np.float32))
    cm_d = Padded((200, 96), torch.float32)
    bufs.append(cm_d)
    cm = S.CacheMuon(cm_m, cm_d.t, 15.0, WL.QUINTIC, 5)
    for _ in range(3):
        cm.step()
    torch.cuda.synchronize()
    assert all(b.intact() for b in bufs)


# ------------------------------------------------------------------ checkpoint and resume
def test_lionmuon_resumes_bit_for_bit(tmp_path):
    shapes, M, P = [(64, 96), (96, 64), (33, 40)], 4, 3
    W0 = WL.weights(shapes, "normal002", "bf16")

    def fresh():
        Wd = [dev(w, torch.bfloat16) for w in W0]
        mom = [[torch.zeros(s, device="cuda") for _ in range(M)] for s in shapes]
        return S.LionMuon(Wd, mom, grad=S.GradStream(21, 5, 1.0, 0))

    def run(opt, n):
        for _ in range(n):
            S.lionmuon_step(opt, None, P, 0.9, 0.99, 3e-3, *WL.QUINTIC, 5, ns_flags=S.NS_SPLIT_BF16)

    straight = fresh()
    run(straight, 7)
    first = fresh()
    run(first, 4)
    path = os.path.join(tmp_path, "lion.pt")
    C.save(path, first)
    resumed = fresh()
    for w in resumed.W:  # garbage in the new run's buffers: everything must come from the file
        w.fill_(7.0)
    C.load(path, resumed)
    assert resumed.t == 4
    run(resumed, 3)
    torch.cuda.synchronize()
    assert resumed.t == straight.t == 7
    for a, b in zip(resumed.W, straight.W):
        assert torch.equal(a, b)
    for la, lb in zip(resumed.mom, straight.mom):
        for a, b in zip(la, lb):
            assert torch.equal(a, b)


def test_cachemuon_resumes_bit_for_bit(tmp_path):
    shape = (160, 320)
    mom = list(WL.cachemuon_momenta(shape, 6, drift=0.02))

    def run(cm, Md, ts):
        for t in ts:
            Md.copy_(dev(mom[t]))
            cm.step()

    Ma, Da = dev(mom[0]), torch.zeros(shape, device="cuda")
    straight = S.CacheMuon(Ma, Da, 2.0, WL.QUINTIC, 5)
    run(straight, Ma, range(6))
    Mb, Db = dev(mom[0]), torch.zeros(shape, device="cuda")
    first = S.CacheMuon(Mb, Db, 2.0, WL.QUINTIC, 5)
    run(first, Mb, range(3))
    snap = C.snapshot(first)
    Mc, Dc = torch.zeros(shape, device="cuda"), torch.zeros(shape, device="cuda")
    resumed = S.CacheMuon(Mc, Dc, 2.0, WL.QUINTIC, 5)
    C.restore(resumed, snap)
    run(resumed, Mc, range(3, 6))
    torch.cuda.synchronize()
    assert torch.equal(Dc, Da) and torch.equal(resumed.Q, straight.Q)
    assert resumed.counters() == straight.counters()


# ------------------------------------------------------------------ first use inside a CUDA graph capture
def test_first_call_captured_in_a_cuda_graph():
    """A process's first smuon_ns call may be made inside a CUDA graph capture:
    building the plan (SM-pair occupancy query, attribute setting) enqueues
    nothing, the plan upload is a captured kernel, and the replay gives the
    eager result bit for bit. Run in a fresh process, so the call is the first."""
    import subprocess
    import sys
    code = (
        "import sys, torch\n"
        "import matrix_aware_sign_b200 as S, workloads as WL\n"
        "M=[torch.randn(768, 2304, device='cuda')]; U=[torch.empty(768, 2304, device='cuda')]\n"
        "ws=S.workspace(S.smuon_ns_workspace_bytes(M, 5, S.NS_SPLIT_BF16), 'cuda')\n"
        "g=torch.cuda.CUDAGraph(); side=torch.cuda.Stream(); torch.cuda.synchronize()\n"
        "with torch.cuda.stream(side):\n"
        "    with torch.cuda.graph(g, stream=side):\n"
        "        S.smuon_ns(M, U, *WL.QUINTIC, 5, flags=S.NS_SPLIT_BF16, ws=ws)\n"
        "g.replay(); torch.cuda.synchronize()\n"
        "U2=[torch.empty(768, 2304, device='cuda')]\n"
        "S.smuon_ns(M, U2, *WL.QUINTIC, 5, flags=S.NS_SPLIT_BF16); torch.cuda.synchronize()\n"
        "sys.exit(0 if torch.equal(U[0], U2[0]) else 3)\n")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", code], cwd=root, timeout=240, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr[-2000:]
