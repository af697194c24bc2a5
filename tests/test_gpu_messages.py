"""The 1-bit message on the GPU: written by the last Newton-Schulz epilogue
(a BITS output) and read by the fused vote / update kernel; the plain leading
steps of the split mode; and a bounded pipeline wait made to run out. Called
through the C ABI and checked against the oracle."""
import numpy as np
import pytest
import torch

import matrix_aware_sign_b200 as S
import oracle as O
import workloads as WL
from tests.gpu_util import check_ns_outputs, dev, host

pytestmark = pytest.mark.gpu

# wide and tall, cols a multiple of 32; m = 33 leaves a ragged tile row
SHAPES_BITS = [(96, 320), (352, 64), (256, 256), (200, 96), (33, 128)]


def _words(b):
    return b.words.cpu().numpy().view(np.uint32)


@pytest.mark.parametrize("flags,iters", [(0, 1), (S.NS_SPLIT_BF16, 1), (S.NS_SPLIT_BF16, 5),
                                         (S.NS_SPLIT_BF16 | S.ns_plain_lead(2), 5), (0, 3)])
def test_ns_bits_output_is_the_sign_of_the_f32_output(flags, iters):
    """The message written by the epilogue equals, bit for bit (pad bits zero),
    the packed signs of an F32 output of the same call; both epilogue forms are
    covered (32-column chunks with one step, the shared-memory source ring and
    16-column halves from two steps on), wide and tall."""
    rng = np.random.default_rng(iters * 10 + flags)
    Ms = [rng.standard_normal(s).astype(np.float32) for s in SHAPES_BITS]
    Md = [dev(m) for m in Ms]
    U32 = [torch.zeros(s, device="cuda") for s in SHAPES_BITS]
    bits = [S.Bits(torch.full((S.packed_words(r * c),), -1, dtype=torch.int32, device="cuda"), r, c)
            for r, c in SHAPES_BITS]
    S.smuon_ns(Md, U32, *WL.QUINTIC, iters, flags=flags)
    S.smuon_ns(Md, bits, *WL.QUINTIC, iters, flags=flags)
    torch.cuda.synchronize()
    pairs = []
    for i, s in enumerate(SHAPES_BITS):
        u = host(U32[i])
        np.testing.assert_array_equal(_words(bits[i]), O.pack_bits(O.sign_extract(u)))
        pairs.append((u, O.newton_schulz(Ms[i].astype(np.float64), *WL.QUINTIC, iters)))
    if flags & S.NS_SPLIT_BF16 or iters == 1:  # plain BF16 meets the criteria with one quintic step
        check_ns_outputs(pairs, 1e-2)


@pytest.mark.parametrize("wdtype", ["f32", "bf16"])
@pytest.mark.parametrize("M,tie", [(1, 0), (3, 0), (4, 1), (8, 0), (8, -1), (16, 0), (33, 0), (64, 1)])
def test_fused_vote_update_from_messages(wdtype, M, tie):
    """1-bit messages as the source of smuon_update: the bit-sliced count of the
    M workers' bits, the threshold with ties, and the update, bit-exact against
    the oracle's popcount vote; ragged last words, a strided W (entry-by-entry
    path) and the vote output."""
    shapes = [(64, 147), (7, 13), (256, 256), (1, 1), (130, 300), (37, 50)]
    W = WL.weights(shapes, "normal002", wdtype)
    tw = torch.bfloat16 if wdtype == "bf16" else torch.float32
    Wd = [dev(w, tw) for w in W]
    Wbig = torch.zeros((37, 64), dtype=tw, device="cuda")
    Wbig[:, :50] = Wd[-1]
    Wd[-1] = Wbig[:, :50]
    rng = np.random.default_rng(M * 3 + tie + 7)
    signs = [[np.where(rng.random(s) < 0.5, 1, -1).astype(np.int8) for _ in range(M)] for s in shapes]
    msgs = [[S.Bits(dev(O.pack_bits(sg).view(np.int32), torch.int32), *s) for sg in layer]
            for s, layer in zip(shapes, signs)]
    votes = [torch.full((r * c,), 9, dtype=torch.int8, device="cuda") for r, c in shapes]
    eta = 0.02
    S.smuon_update(Wd, eta, U=msgs, M=M, tie_value=tie, vote_out=votes)
    torch.cuda.synchronize()
    for i, s in enumerate(shapes):
        v = O.vote_from_packed([O.pack_bits(sg) for sg in signs[i]], M, s[0] * s[1], tie).reshape(s)
        np.testing.assert_array_equal(host(votes[i]).reshape(s), v)
        np.testing.assert_array_equal(host(Wd[i]), O.update_with_vote(W[i], v, eta, wdtype))
    assert torch.all(Wbig[:, 50:] == 0)


def _bits_update(shapes, M, tie, seed, wdtype="bf16", with_votes=True, kind=0, status=None):
    """Random signs packed as messages, the fused update through the C ABI, and
    the names of the vote kernels that ran."""
    rng = np.random.default_rng(seed)
    W = WL.weights(shapes, "normal002", wdtype)
    tw = torch.bfloat16 if wdtype == "bf16" else torch.float32
    Wd = [dev(w, tw) for w in W]
    signs = [[np.where(rng.random(s) < 0.5, 1, -1).astype(np.int8) for _ in range(M)] for s in shapes]
    msgs = [[S.Bits(dev(O.pack_bits(sg).view(np.int32), torch.int32), *s) for sg in layer]
            for s, layer in zip(shapes, signs)]
    votes = [torch.full((r * c,), 9, dtype=torch.int8, device="cuda") for r, c in shapes] if with_votes else None
    S.trace_enable(True)
    S.smuon_update(Wd, 0.02, U=msgs, M=M, tie_value=tie, vote_out=votes, vote_kind=kind, status=status)
    torch.cuda.synchronize()
    names = {r["name"] for r in S.trace_read() if r["name"].startswith("k_vote")}
    S.trace_enable(False)
    return W, Wd, signs, votes, names


BULK_SHAPES = [(96, 320), (1024, 1032), (8, 1024), (1, 8), (24, 328), (768, 2304)]


@pytest.mark.parametrize("M,tie", [(1, 0), (2, -1), (2, 1), (7, 0), (8, 0), (8, 1), (15, 0), (16, -1)])
def test_bits_vote_bulk_copy_form(M, tie):
    """Layers of bf16 W whose entry counts are multiples of 8 take the 1-bit vote
    in its bulk-copy form (8192-entry blocks of W and the M message rows in a
    shared-memory ring): W and the votes equal the oracle's bit for bit, on
    layers of one block, of a ragged last block (96 x 320: 3.75 blocks; 24 x
    328: a last word of 8 valid entries), of one 16-byte row (1 x 8) and of many
    blocks, for odd and even M with each tie value."""
    W, Wd, signs, votes, names = _bits_update(BULK_SHAPES, M, tie, seed=M * 10 + tie + 3)
    assert names == {"k_vote_update_bits_tma"}
    for i, s in enumerate(BULK_SHAPES):
        v = O.vote_from_packed([O.pack_bits(sg) for sg in signs[i]], M, s[0] * s[1], tie).reshape(s)
        np.testing.assert_array_equal(host(votes[i]).reshape(s), v)
        np.testing.assert_array_equal(host(Wd[i]), O.update_with_vote(W[i], v, 0.02, "bf16"))


@pytest.mark.parametrize("case", ["m17", "f32", "ragged"])
def test_bits_vote_other_layers_take_the_word_form(case):
    """M = 17, f32 W, or a layer whose entry count is not a multiple of 8 keep
    the whole launch on the word-per-lane kernel; the result is the oracle's."""
    shapes = [(96, 320), (7, 13)] if case == "ragged" else [(96, 320), (64, 64)]
    M = 17 if case == "m17" else 8
    wdtype = "f32" if case == "f32" else "bf16"
    W, Wd, signs, votes, names = _bits_update(shapes, M, 0, seed=len(case), wdtype=wdtype, with_votes=False)
    assert names == {"k_vote_update_bits"}
    for i, s in enumerate(shapes):
        v = O.vote_from_packed([O.pack_bits(sg) for sg in signs[i]], M, s[0] * s[1], 0).reshape(s)
        np.testing.assert_array_equal(host(Wd[i]), O.update_with_vote(W[i], v, 0.02, wdtype))


def test_bits_vote_unaligned_w_takes_the_word_form():
    """A bf16 W that starts 8 bytes past a 16-byte boundary cannot be staged by
    the bulk-copy engine: the launch keeps the word-per-lane kernel and gives
    the oracle's result."""
    shapes, M = [(96, 320)], 8
    W = WL.weights(shapes, "normal002", "bf16")
    base = torch.zeros(96 * 320 + 4, dtype=torch.bfloat16, device="cuda")
    Wv = base[4:].view(96, 320)
    Wv.copy_(dev(W[0], torch.bfloat16))
    rng = np.random.default_rng(17)
    signs = [np.where(rng.random(shapes[0]) < 0.5, 1, -1).astype(np.int8) for _ in range(M)]
    msgs = [[S.Bits(dev(O.pack_bits(sg).view(np.int32), torch.int32), *shapes[0]) for sg in signs]]
    S.trace_enable(True)
    S.smuon_update([Wv], 0.02, U=msgs, M=M)
    torch.cuda.synchronize()
    names = {r["name"] for r in S.trace_read() if r["name"].startswith("k_vote")}
    S.trace_enable(False)
    assert names == {"k_vote_update_bits"}
    v = O.vote_from_packed([O.pack_bits(sg) for sg in signs], M, 96 * 320, 0).reshape(shapes[0])
    np.testing.assert_array_equal(host(Wv), O.update_with_vote(W[0], v, 0.02, "bf16"))


def test_bits_vote_plan_in_a_cuda_graph():
    """A prepared update over 1-bit messages (the bulk-copy form) captured in a
    CUDA graph and replayed twice equals two oracle updates."""
    shapes, M = [(768, 2304), (3072, 768)], 8
    W = WL.weights(shapes, "normal002", "bf16")
    Wd = [dev(w, torch.bfloat16) for w in W]
    rng = np.random.default_rng(23)
    signs = [[np.where(rng.random(s) < 0.5, 1, -1).astype(np.int8) for _ in range(M)] for s in shapes]
    msgs = [[S.Bits(dev(O.pack_bits(sg).view(np.int32), torch.int32), *s) for sg in layer]
            for s, layer in zip(shapes, signs)]
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    plan = S.UpdatePlan(Wd, 0.02, U=msgs, M=M, status=st)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        g.capture_begin()
        plan.run(stream=s)
        g.capture_end()
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    for i, sh in enumerate(shapes):
        v = O.vote_from_packed([O.pack_bits(sg) for sg in signs[i]], M, sh[0] * sh[1], 0).reshape(sh)
        w1 = O.update_with_vote(W[i], v, 0.02, "bf16")
        np.testing.assert_array_equal(host(Wd[i]), O.update_with_vote(w1, v, 0.02, "bf16"))


def test_bits_vote_bounded_wait_expiry():
    """The bulk-copy vote's waits are bounded: with SMUON_VOTE_TEST_WAIT_EXPIRY
    the producer issues no copy, every consumer wait runs out after 65536 SM
    clocks, the call returns with SMUON_DEV_WAIT_TIMEOUT in d_status and W
    untouched; the next call is correct again and leaves its status clear."""
    shapes = [(96, 320), (8, 1024)]
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    W, Wd, signs, votes, names = _bits_update(shapes, 8, 0, seed=99, kind=S.VOTE_TEST_WAIT_EXPIRY, status=st)
    assert names == {"k_vote_update_bits_tma"}
    assert int(st.item()) & S.DEV_WAIT_TIMEOUT
    for i in range(len(shapes)):
        np.testing.assert_array_equal(host(Wd[i]), W[i])
    st.zero_()
    W, Wd, signs, votes, names = _bits_update(shapes, 8, 0, seed=98, status=st)
    assert int(st.item()) == 0
    for i, s in enumerate(shapes):
        v = O.vote_from_packed([O.pack_bits(sg) for sg in signs[i]], 8, s[0] * s[1], 0).reshape(s)
        np.testing.assert_array_equal(host(Wd[i]), O.update_with_vote(W[i], v, 0.02, "bf16"))


def test_fused_vote_update_from_messages_many_layers():
    """More layers than one launch's table holds, W = NULL (votes only) and M = 2
    with ties."""
    M = 2
    rng = np.random.default_rng(5)
    shapes = [(int(rng.integers(1, 40)), int(rng.integers(1, 120))) for _ in range(150)]
    signs = [[np.where(rng.random(s) < 0.5, 1, -1).astype(np.int8) for _ in range(M)] for s in shapes]
    msgs = [[S.Bits(dev(O.pack_bits(sg).view(np.int32), torch.int32), *s) for sg in layer]
            for s, layer in zip(shapes, signs)]
    votes = [torch.full((r * c,), 9, dtype=torch.int8, device="cuda") for r, c in shapes]
    S.smuon_update(None, 0.0, U=msgs, M=M, tie_value=0, vote_out=votes)
    torch.cuda.synchronize()
    for i, s in enumerate(shapes):
        np.testing.assert_array_equal(host(votes[i]), O.vote_from_signs([sg.reshape(-1) for sg in signs[i]]))


def test_sign_muon_step_through_messages_equals_the_f32_path():
    """A whole Sign-Muon step with the messages written by the epilogue and read
    by the vote kernel gives, bit for bit, the step through an F32 U and the
    fused sign / popcount vote of the same Newton-Schulz values; and the
    oracle's update wherever no worker's sign disagrees with the oracle's."""
    shapes, M = [(96, 320), (352, 64), (128, 128)], 8
    rng = np.random.default_rng(11)
    W = WL.weights(shapes, "normal002", "bf16")
    G = [[rng.standard_normal(s).astype(np.float32) for _ in range(M)] for s in shapes]
    flags = S.NS_SPLIT_BF16
    out = {}
    for form in ("bits", "f32"):
        Md = [torch.zeros(s, device="cuda") for s in shapes for _ in range(M)]
        if form == "bits":
            U = [S.Bits.empty(*s) for s in shapes for _ in range(M)]
        else:
            U = [torch.zeros(s, device="cuda") for s in shapes for _ in range(M)]
        Wd = [dev(w, torch.bfloat16) for w in W]
        S.smuon_ns(Md, U, *WL.QUINTIC, 5, G=[dev(g) for layer in G for g in layer], beta=0.95, flags=flags)
        S.smuon_update(Wd, 0.02, U=[U[l * M:(l + 1) * M] for l in range(len(shapes))], M=M)
        torch.cuda.synchronize()
        out[form] = ([host(w) for w in Wd], U)
    for a, b in zip(out["bits"][0], out["f32"][0]):
        np.testing.assert_array_equal(a, b)
    for l, s in enumerate(shapes):
        ref_u = [O.newton_schulz(O.momentum(np.zeros(s), g, 0.95), *WL.QUINTIC, 5) for g in G[l]]
        check_ns_outputs([(host(out["f32"][1][l * M + k]), ref_u[k]) for k in range(M)], 1e-2)
        signs = [O.sign_extract(u) for u in ref_u]
        v = O.vote_from_signs(signs)
        W_ref = O.update_with_vote(W[l], v, 0.02, "bf16")
        gpu_signs = [O.sign_extract(host(out["f32"][1][l * M + k])) for k in range(M)]
        same = np.all([gs == rs for gs, rs in zip(gpu_signs, signs)], axis=0)
        np.testing.assert_array_equal(out["bits"][0][l][same], W_ref[same])


@pytest.mark.parametrize("shape", [(768, 2304), (768, 768), (3072, 768), (1280, 5120), (1280, 1280)])
def test_plain_lead_two_steps_meets_the_criteria(shape):
    """SMUON_NS_PLAIN_LEAD(2) on Gaussian momenta of the GPT-2 layer shapes: the
    two plain leading steps leave five quintic steps within the split mode's
    accuracy (relative error well under 1e-3, the sign criterion met)."""
    rng = np.random.default_rng(shape[0] + shape[1])
    M = rng.standard_normal(shape).astype(np.float32)
    U = torch.zeros(shape, device="cuda")
    S.smuon_ns([dev(M)], [U], *WL.QUINTIC, 5, flags=S.NS_SPLIT_BF16 | S.ns_plain_lead(2))
    torch.cuda.synchronize()
    err, frac, worst = check_ns_outputs([(host(U), O.newton_schulz(M.astype(np.float64), *WL.QUINTIC, 5))], 1e-2)
    assert err < 1e-3


@pytest.mark.parametrize("form", [0, S.NS_ONE_SM])
def test_bounded_wait_runs_out_and_the_context_survives(form):
    """SMUON_NS_TEST_WAIT_EXPIRY: the tensor-core stages' producers issue nothing
    and their waits are limited to 65536 clocks, so every stage's waits run out.
    The call returns, SMUON_DEV_WAIT_TIMEOUT is set, and the next normal call
    still matches the oracle. Both forms: 256 x 640 runs on SM pairs unless
    SMUON_NS_ONE_SM asks for single-SM tiles."""
    rng = np.random.default_rng(3)
    Mx = rng.standard_normal((256, 640)).astype(np.float32)
    Md = dev(Mx)
    U = torch.full((256, 640), 5.0, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for flags in (S.NS_SPLIT_BF16 | S.NS_TEST_WAIT_EXPIRY, S.NS_TEST_WAIT_EXPIRY):
        status.zero_()
        S.smuon_ns([Md], [U], *WL.QUINTIC, 2, flags=flags | form, status=status)
        torch.cuda.synchronize()
        assert int(status.item()) & S.DEV_WAIT_TIMEOUT
    status.zero_()
    S.smuon_ns([Md], [U], *WL.QUINTIC, 2, flags=S.NS_SPLIT_BF16 | form, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    check_ns_outputs([(host(U), O.newton_schulz(Mx.astype(np.float64), *WL.QUINTIC, 2))], 1e-2)
