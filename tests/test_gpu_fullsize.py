"""Full-size workloads on the GPU, checked against the oracle on sampled
outputs (the layers, matrices or entries the oracle can afford) and, where
the oracle cannot follow, against properties that hold at any size.

GPT-2-small set (48 matrices, 8 workers, five quintic steps, popcount vote):
with the local polar step, and with the 1-bit messages written by the
Newton-Schulz epilogue (the bench's form), in the split-BF16 mode. CacheMuon
large matrices: 4096^2, 8192^2 and 4096x16384 fresh solves against the oracle
(the two large ones marked slow), and the schedule by properties. LionMuon on
the GPT-2-Large set (144 matrices, 16 workers, P = 4): sign steps bit-exact on
sampled entries, the Muon step's direction on sampled layers."""
import numpy as np
import pytest
import torch

import matrix_aware_sign_b200 as S
import oracle as O
import workloads as WL
from tests.gpu_util import check_ns_outputs, dev, host, rel_fro

pytestmark = pytest.mark.gpu


def _free_gb():
    free, _ = torch.cuda.mem_get_info()
    return free / 2 ** 30


# ------------------------------------------------------------------ GPT-2 small, one step
def test_gpt2_small_set_one_step_sampled():
    cfg = WL.SIGN_MUON_WORKLOADS["c3_gpt2s"]
    M, shapes = cfg.workers, cfg.shapes
    L = len(shapes)
    W = WL.weights(shapes, cfg.w_init, cfg.w_dtype)
    grads = WL.GradientStreams(shapes, M, cfg.grad_sigma).next_step()
    Md = [torch.zeros(s, device="cuda") for s in shapes for _ in range(M)]
    Ud = [torch.zeros(s, dtype=torch.bfloat16, device="cuda") for s in shapes for _ in range(M)]
    Gd = [dev(g) for layer in grads for g in layer]
    S.smuon_ns(Md, Ud, *cfg.coeffs, cfg.iters, G=Gd, beta=cfg.beta, flags=S.NS_SPLIT_BF16)
    del Gd
    # all-gather variant: packed signs -> popcount vote -> local polar step -> dense update
    Wd = [dev(w, torch.bfloat16) for w in W]
    votes, dirs = [], []
    for l, (r, c) in enumerate(shapes):
        packed = torch.zeros((M, S.packed_words(r * c)), dtype=torch.int32, device="cuda")
        S.smuon_sign_pack(Ud[l * M:(l + 1) * M], packed=packed)
        v = torch.zeros(r * c, dtype=torch.int8, device="cuda")
        S.smuon_vote(M, r * c, v, packed=packed, tie_value=cfg.tie_value)
        votes.append(v.view(r, c))
        dirs.append(torch.zeros((r, c), device="cuda"))
    S.smuon_ns(votes, dirs, *cfg.coeffs, cfg.iters, flags=S.NS_SPLIT_BF16)
    S.smuon_update(Wd, cfg.eta, dense=dirs)
    torch.cuda.synchronize()
    # oracle on one layer of each distinct shape (all 8 workers)
    pairs, n_dis, n_all = [], 0, 0
    for l in (0, 1, 2, 3):
        ref_u = [O.newton_schulz(grads[l][k].astype(np.float64), *cfg.coeffs, cfg.iters) for k in range(M)]
        pairs += [(host(Ud[l * M + k]), ref_u[k]) for k in range(M)]
        signs = [O.sign_extract(u) for u in ref_u]
        v_ref = O.vote_from_packed([O.pack_bits(s) for s in signs], M, signs[0].size).reshape(shapes[l])
        v_gpu = host(votes[l])
        n_dis += int((v_gpu != v_ref).sum())
        n_all += v_ref.size
        D_ref = O.newton_schulz(v_ref.astype(np.float64), *cfg.coeffs, cfg.iters)
        # the two local polar steps start from votes that differ in the few
        # near-zero entries counted above: allow that input difference on top
        # of the Newton-Schulz tolerance
        dv = rel_fro(v_gpu.astype(np.float64), v_ref.astype(np.float64))
        assert rel_fro(host(dirs[l]), D_ref) < 1e-2 + 2 * dv
        W_ref = O.update_dense(W[l], D_ref, cfg.eta, "bf16")
        # bf16 weights: the updated weights agree to well within the update's size
        # (the rounding of each side to bf16 differs where the directions do)
        assert rel_fro(host(Wd[l]), W_ref) < 3e-3  # bf16 rounding noise alone is ~1e-3
        assert rel_fro(host(Wd[l]), W[l]) > 1e-2  # and the update was applied
    check_ns_outputs(pairs, 1e-2)
    assert n_dis <= 1e-4 * n_all


def test_gpt2_small_set_one_step_messages():
    """The GPT-2-small step as the bench runs it: five quintic steps with two
    plain leading steps, the 1-bit messages written by the last epilogue, and
    the fused vote / update from the messages. On one layer of each shape: the
    messages' signs within the sign criterion of the oracle's, and W equal,
    bit for bit, to the oracle's update wherever the vote agrees; the votes
    differ at no more than 1e-4 of the entries."""
    cfg = WL.SIGN_MUON_WORKLOADS["c3_gpt2s"]
    M, shapes = cfg.workers, cfg.shapes
    W = WL.weights(shapes, cfg.w_init, cfg.w_dtype)
    grads = WL.GradientStreams(shapes, M, cfg.grad_sigma).next_step()
    Md = [torch.zeros(s, device="cuda") for s in shapes for _ in range(M)]
    Ub = [S.Bits.empty(*s) for s in shapes for _ in range(M)]
    Gd = [dev(g) for layer in grads for g in layer]
    Wd = [dev(w, torch.bfloat16) for w in W]
    flags = S.NS_SPLIT_BF16 | S.ns_plain_lead(2)
    S.smuon_ns(Md, Ub, *cfg.coeffs, cfg.iters, G=Gd, beta=cfg.beta, flags=flags)
    S.smuon_update(Wd, cfg.eta, U=[Ub[l * M:(l + 1) * M] for l in range(len(shapes))], M=M,
                   tie_value=cfg.tie_value)
    torch.cuda.synchronize()
    del Gd
    n_flip, n_vote, n_all, worst = 0, 0, 0, 0.0
    for l in (0, 1, 2, 3):
        n = shapes[l][0] * shapes[l][1]
        ref_u = [O.newton_schulz(grads[l][k].astype(np.float64), *cfg.coeffs, cfg.iters) for k in range(M)]
        signs = [O.sign_extract(u).reshape(-1) for u in ref_u]
        gpu = [O.unpack_bits(Ub[l * M + k].words.cpu().numpy().view(np.uint32), n) for k in range(M)]
        for k in range(M):
            dis = gpu[k] != signs[k]
            n_flip += int(dis.sum())
            if dis.any():
                worst = max(worst, float(np.abs(ref_u[k].reshape(-1)[dis]).max() / np.abs(ref_u[k]).max()))
        v_ref = O.vote_from_signs(signs, cfg.tie_value)
        v_gpu = O.vote_from_signs(gpu, cfg.tie_value)
        n_vote += int((v_gpu != v_ref).sum())
        n_all += n
        # given its own votes the update is exact: W follows the messages bit for bit
        np.testing.assert_array_equal(host(Wd[l]), O.update_with_vote(W[l], v_gpu.reshape(shapes[l]), cfg.eta, "bf16"))
        agree = (v_gpu == v_ref).reshape(shapes[l])
        W_ref = O.update_with_vote(W[l], v_ref.reshape(shapes[l]), cfg.eta, "bf16")
        np.testing.assert_array_equal(host(Wd[l])[agree], W_ref[agree])
    assert n_flip <= 1e-4 * n_all * M and worst < 1e-3
    assert n_vote <= 1e-4 * n_all


# ------------------------------------------------------------------ CacheMuon
@pytest.mark.slow
@pytest.mark.parametrize("shape", [(8192, 8192), (4096, 16384)])
def test_cachemuon_large_fresh_solve_against_oracle(shape):
    """The two larger shapes of the CacheMuon sweep: the fresh solve's
    direction D (split BF16, five quintic steps) and its cached transform Q
    against the float64 oracle, in full."""
    rng = np.random.default_rng(4242)
    M = rng.standard_normal(shape, dtype=np.float32)
    m = min(shape)
    D = torch.zeros(shape, device="cuda")
    Q = torch.zeros((m, m), dtype=torch.bfloat16, device="cuda")
    S.smuon_ns([dev(M)], [D], *WL.QUINTIC, 5, flags=S.NS_SPLIT_BF16 | S.NS_EMIT_Q, Q_out=[Q])
    torch.cuda.synchronize()
    D_ref, Q_ref = O.newton_schulz_with_q(M.astype(np.float64), *WL.QUINTIC, 5)
    check_ns_outputs([(host(D), D_ref)], 1e-2)
    assert rel_fro(host(Q), Q_ref) < 1e-2


def test_cachemuon_4096sq_against_oracle():
    shape = (4096, 4096)
    mom = list(WL.cachemuon_momenta(shape, 2, drift=0.01))
    Md = dev(mom[0])
    D = torch.zeros(shape, device="cuda")
    cm = S.CacheMuon(Md, D, 15.0, WL.QUINTIC, 5)
    cm.step()
    torch.cuda.synchronize()
    D_ref, Q_ref = O.newton_schulz_with_q(mom[0], *WL.QUINTIC, 5)
    check_ns_outputs([(host(D), D_ref)], 1e-2)
    assert rel_fro(host(cm.Q), Q_ref) < 1e-2
    Md.copy_(dev(mom[1]))
    cm.step()
    torch.cuda.synchronize()
    Dh_ref, err_ref = O.cachemuon_probe(Q_ref, mom[1])
    assert abs(cm.err.item() - err_ref) <= 2e-2 * err_ref + 1e-3
    assert cm.accept.item() == int(err_ref <= 15.0)
    assert rel_fro(host(D), Dh_ref) < 1e-2
    assert cm.counters() == {"hits": 1, "misses": 1, "probes": 1}


@pytest.mark.parametrize("shape,drift,gamma", [((8192, 8192), 0.01, 2.0), ((4096, 16384), 0.01, 2.0),
                                               ((4096, 16384), 1.0, 2.0), ((4096, 16384), 0.01, -1.0)])
def test_cachemuon_large_properties(shape, drift, gamma):
    """Beyond the oracle's reach: the residual the kernel reports is the
    residual of the candidate it returned, the decision follows it, the
    counters follow the decisions, and a rejected step is a fresh solve
    (gamma < 0 rejects every probe, so every step refreshes at full size)."""
    m = min(shape)
    gen = torch.Generator(device="cuda").manual_seed(4242)
    Md = torch.randn(shape, device="cuda", generator=gen)
    D = torch.zeros(shape, device="cuda")
    decisions = []
    cm = S.CacheMuon(Md, D, gamma, WL.QUINTIC, 5)
    for t in range(4):
        if t:
            Md.add_(torch.randn(shape, device="cuda", generator=gen), alpha=drift)
        cm.step()
        torch.cuda.synchronize()
        acc = int(cm.accept.item())
        decisions.append(acc)
        if t:
            Dw = D if shape[0] <= shape[1] else D.T
            R = Dw.double() @ Dw.double().T - torch.eye(m, device="cuda", dtype=torch.float64)
            if acc:  # D is the candidate the probe measured
                err = float(torch.linalg.norm(R) / m ** 0.5)
                assert abs(cm.err.item() - err) <= 5e-3 * err + 1e-3
            else:  # D is the fresh solve of this momentum
                D_fresh = torch.empty_like(D)
                S.smuon_ns([Md], [D_fresh], *WL.QUINTIC, 5, flags=S.NS_SPLIT_BF16)
                torch.cuda.synchronize()
                assert torch.equal(D, D_fresh)
            assert acc == int(cm.err.item() <= gamma)
    c = cm.counters()
    assert decisions[0] == 0 and c["hits"] == sum(decisions) and c["misses"] == 4 - sum(decisions)
    assert c["probes"] == 3
    if gamma < 0:
        assert decisions == [0, 0, 0, 0]


# ------------------------------------------------------------------ LionMuon
def test_lionmuon_gpt2_large_sampled():
    cfg = WL.LION_MUON_WORKLOADS["c5_gpt2l"]
    M, shapes = cfg.workers, cfg.shapes
    n_params = sum(r * c for r, c in shapes)
    need_gb = n_params * M * 4 * 2 / 2 ** 30 + 12
    if _free_gb() < need_gb:
        pytest.skip(f"needs {need_gb:.0f} GiB free")
    gen = torch.Generator(device="cuda").manual_seed(5)
    W0 = [dev(w, torch.bfloat16) for w in WL.weights(shapes, "normal002", "bf16")]
    Wd = [w.clone() for w in W0]
    mom = [[torch.zeros(s, device="cuda") for _ in range(M)] for s in shapes]
    G = [[torch.empty(s, device="cuda") for _ in range(M)] for s in shapes]
    flags = S.NS_SPLIT_BF16 | S.ns_plain_lead(2)  # the bench's configuration
    opt = S.LionMuon(Wd, mom)
    ws = S.workspace(opt.workspace_bytes(cfg.iters, flags))
    rng = np.random.default_rng(0)
    samples = {l: rng.integers(0, shapes[l][0] * shapes[l][1], 2000) for l in (0, 1, 2, 3, 77, 143)}
    W_s = {l: host(W0[l]).reshape(-1)[idx] for l, idx in samples.items()}
    M_s = {l: [np.zeros(len(idx), np.float32) for _ in range(M)] for l, idx in samples.items()}
    Wprev_layer1 = None
    for t in range(1, 5):  # P = 4: three sign steps, then a Muon step
        for layer in G:
            for g in layer:
                g.normal_(generator=gen)
        if t == 4:
            Wprev_layer1 = Wd[1].float().cpu().numpy()
            M_l1 = [m.cpu().numpy() for m in mom[1]]
            G_l1 = [g.cpu().numpy() for g in G[1]]
            M_l3 = [m.cpu().numpy() for m in mom[3]]
            G_l3 = [g.cpu().numpy() for g in G[3]]
        G_s = {l: [G[l][k].view(-1)[torch.from_numpy(idx).cuda()].cpu().numpy() for k in range(M)]
               for l, idx in samples.items()}
        S.lionmuon_step(opt, G, cfg.period, cfg.beta1, cfg.beta2, cfg.eta, *cfg.coeffs, cfg.iters,
                        tie_value=cfg.tie_value, ns_flags=flags, ws=ws)
        torch.cuda.synchronize()
        muon = t % cfg.period == 0
        for l, idx in samples.items():
            if not muon:  # sign steps are elementwise: the oracle follows the sampled entries
                kind, Wn, Mn = O.lionmuon_step(t, [W_s[l]], [M_s[l]], [G_s[l]], cfg.period, cfg.beta1,
                                               cfg.beta2, cfg.eta, cfg.coeffs, cfg.iters, "bf16", cfg.tie_value)
                assert kind == "sign"
                np.testing.assert_array_equal(host(Wd[l]).reshape(-1)[idx], Wn[0])
                M_s[l] = Mn[0]
            else:
                M_s[l] = [O.lion_ema(M_s[l][k], G_s[l][k], cfg.beta2) for k in range(M)]
            for k in range(M):  # the shared EMA is bit-exact at every step
                np.testing.assert_array_equal(mom[l][k].view(-1)[torch.from_numpy(idx).cuda()].cpu().numpy(),
                                              M_s[l][k])
            W_s[l] = host(Wd[l]).reshape(-1)[idx]
    assert opt.t == 4
    # the Muon step's direction on sampled layers (1280 x 1280 and the tall 5120 x 1280): the same step
    # replayed from the same EMA and gradients on a float32 shadow whose weights start at zero, so the
    # shadow holds -f32(f32(eta) D) exactly; D against the oracle's by the Newton-Schulz criteria
    for l, (M_l, G_l) in ((1, (M_l1, G_l1)), (3, (M_l3, G_l3))):
        shadow = [torch.zeros(shapes[l], device="cuda")]
        smom = [[dev(x) for x in M_l]]
        sopt = S.LionMuon(shadow, smom, t=3)
        S.lionmuon_step(sopt, [[dev(g) for g in G_l]], cfg.period, cfg.beta1, cfg.beta2, cfg.eta, *cfg.coeffs,
                        cfg.iters, tie_value=cfg.tie_value, ns_flags=flags)
        torch.cuda.synchronize()
        d_gpu = -host(shadow[0]).astype(np.float64) / np.float32(cfg.eta)
        gh = [O.lion_interpolate(M_l[k], G_l[k], cfg.beta1) for k in range(M)]
        D_ref = O.newton_schulz(np.mean(np.stack([g.astype(np.float64) for g in gh]), 0), *cfg.coeffs, cfg.iters)
        check_ns_outputs([(d_gpu, D_ref)], 1e-2)
        if l == 1:  # the bf16 weights moved by that same step: RN_bf16(W - f32(eta D)) = RN_bf16(W + shadow)
            step = host(shadow[0]).astype(np.float32)
            np.testing.assert_array_equal(host(Wd[1]), O.bf16_round(np.add(Wprev_layer1, step, dtype=np.float32)))


# ------------------------------------------------------------------ LLaMA-style sets
@pytest.mark.parametrize("name", ["llama124m", "llama355m"])
def test_llama_style_set_one_step_sampled(name):
    """The LLaMA-style layer sets (same kernels, other shapes): one Sign-Muon
    step in the accurate split-BF16 mode with the fused popcount vote; the
    oracle follows one matrix of each distinct shape (all workers)."""
    cfg = WL.SIGN_MUON_WORKLOADS[name]
    M, shapes = cfg.workers, cfg.shapes
    n_params = sum(r * c for r, c in shapes)
    if _free_gb() < n_params * M * 4 * 5 / 2 ** 30 + 8:
        pytest.skip("not enough device memory")
    W = WL.weights(shapes, cfg.w_init, cfg.w_dtype)
    gen = torch.Generator(device="cuda").manual_seed(77)
    Gd = [torch.randn(s, device="cuda", generator=gen) for s in shapes for _ in range(M)]
    Md = [torch.zeros(s, device="cuda") for s in shapes for _ in range(M)]
    Ud = [torch.zeros(s, dtype=torch.bfloat16, device="cuda") for s in shapes for _ in range(M)]
    S.smuon_ns(Md, Ud, *cfg.coeffs, cfg.iters, G=Gd, beta=cfg.beta, flags=S.NS_SPLIT_BF16)
    Wd = [dev(w, torch.bfloat16) for w in W]
    packed = [torch.zeros((M, S.packed_words(r * c)), dtype=torch.int32, device="cuda") for r, c in shapes]
    S.smuon_update(Wd, cfg.eta, U=[Ud[l * M:(l + 1) * M] for l in range(len(shapes))], M=M,
                   packed_out=packed)
    torch.cuda.synchronize()
    pairs, n_dis, n_all = [], 0, 0
    for l in (4, 5, 6):  # one matrix of each shape (d x d, h x d, d x h)
        G = [Gd[l * M + k].cpu().numpy() for k in range(M)]
        ref_u = [O.newton_schulz(g.astype(np.float64), *cfg.coeffs, cfg.iters) for g in G]
        pairs += [(host(Ud[l * M + k]), ref_u[k]) for k in range(M)]
        signs = [O.sign_extract(u) for u in ref_u]
        v = O.vote_from_signs(signs, cfg.tie_value)
        agree_w = host(Wd[l]) == O.update_with_vote(W[l], v, cfg.eta, "bf16")
        n_dis += int((~agree_w).sum())
        n_all += agree_w.size
        # the packed message carries the oracle's signs wherever the vote inputs agree
        for k in range(M):
            bits = np.unpackbits(packed[l][k].cpu().numpy().view(np.uint8), bitorder="little")[:signs[k].size]
            assert np.mean(bits.astype(np.int8) * 2 - 1 != signs[k].reshape(-1)) <= 1e-4
    check_ns_outputs(pairs, 1e-2)
    assert n_dis <= 1e-4 * n_all
