"""Host-side checks of the C-ABI library (no GPU): it loads, exports every
function that include/smuon.h declares, and rejects bad arguments before it
would touch a device."""
import ctypes
import os
import re

import pytest

from tests.conftest import ROOT

HEADER = os.path.join(ROOT, "include", "smuon.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s+\**([a-z_][a-z0-9_]*)\s*\(", text, re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def L():
    import matrix_aware_sign_b200 as S
    return S.lib()


def test_header_declares_the_boundary():
    names = _declared()
    for want in ["smuon_ns", "smuon_sign_pack", "smuon_vote", "smuon_update", "cachemuon_reuse_probe",
                 "lionmuon_step", "smuon_ns_workspace_bytes", "cachemuon_workspace_bytes",
                 "lionmuon_workspace_bytes", "smuon_last_error", "smuon_version"]:
        assert want in names, want


def test_library_exports_every_declared_symbol(L):
    for name in _declared():
        assert hasattr(L, name), f"libsmuon.so does not export {name}"


def test_version(L):
    assert L.smuon_version() >> 16 == 1


def test_vote_rejects_bad_arguments_before_launch(L):
    import matrix_aware_sign_b200 as S
    # neither source given
    assert L.smuon_vote(None, None, 3, 10, 0, 1234, None) == -1
    assert b"exactly one" in L.smuon_last_error()
    # too many workers
    assert L.smuon_vote(64, None, 65, 10, 0, 1234, None) == -4
    # bad tie value
    assert L.smuon_vote(64, None, 3, 10, 2, 1234, None) == -1


def test_ns_rejects_bad_arguments_before_launch(L):
    import matrix_aware_sign_b200 as S
    m = S.SmuonMat(4096, 8, 8, 8, S.F32)
    arr = (S.SmuonMat * 1)(m)
    bad = (S.SmuonMat * 1)(S.SmuonMat(4096, 8, 8, 4, S.F32))  # ld < cols
    assert L.smuon_ns(arr, arr, 0, None, 0.9, 1.5, -0.5, 0.0, 5, 1e-7, 0, None, None, None, 0, None, None) == -1
    assert L.smuon_ns(arr, arr, 1, None, 0.9, 1.5, -0.5, 0.0, 0, 1e-7, 0, None, None, None, 0, None, None) == -1
    assert L.smuon_ns(bad, arr, 1, None, 0.9, 1.5, -0.5, 0.0, 5, 1e-7, 0, None, None, None, 0, None, None) == -2
    assert L.smuon_ns(arr, arr, 1, None, 0.9, 1.5, -0.5, 0.0, 5, 1e-7, 0x100, None, None, None, 0, None, None) == -1
    assert L.smuon_ns(arr, arr, 1, None, 0.9, 1.5, -0.5, 0.0, 5, 1e-7, S.NS_EMIT_Q, None, None, None, 0, None,
                      None) == -1
    i8 = (S.SmuonMat * 1)(S.SmuonMat(4096, 8, 8, 8, S.I8))
    g = (S.SmuonMat * 1)(m)
    # int8 momentum cannot take a gradient
    assert L.smuon_ns(i8, arr, 1, g, 0.9, 1.5, -0.5, 0.0, 5, 1e-7, 0, None, None, None, 0, None, None) == -3


def test_workspace_query_runs_on_the_host(L):
    import matrix_aware_sign_b200 as S
    arr = (S.SmuonMat * 2)(S.SmuonMat(4096, 64, 147, 147, S.F32), S.SmuonMat(8192, 2048, 512, 512, S.F32))
    out = ctypes.c_size_t(0)
    assert L.smuon_ns_workspace_bytes(arr, 2, 5, 0, ctypes.byref(out)) == 0
    # at least the bf16 X operands and f32 masters of both matrices
    assert out.value > (64 * 256 + 512 * 2048) * (2 + 2 + 4 + 4)
    out2 = ctypes.c_size_t(0)
    assert L.smuon_ns_workspace_bytes(arr, 2, 1, 0, ctypes.byref(out2)) == 0
    assert out2.value < out.value


def test_update_rejects_bad_source_combinations(L):
    import matrix_aware_sign_b200 as S
    W = (S.SmuonMat * 1)(S.SmuonMat(4096, 8, 8, 8, S.F32))
    assert L.smuon_update(W, 1, None, None, None, 1, 0.01, 0, 0, None, None, None, None) == -1
    assert L.smuon_update(W, 1, W, W, None, 1, 0.01, 0, 0, None, None, None, None) == -1
    assert L.smuon_update(W, 1, W, None, None, 1, 0.01, 0, 7, None, None, None, None) == -1
    # no W: only with the U source and an output to write
    assert L.smuon_update(None, 1, W, None, None, 1, 0.01, 0, 0, None, None, None, None) == -1
    assert L.smuon_update(None, 1, None, W, None, 1, 0.01, 0, 0, None, None, None, None) == -1


def test_gradient_streams_reject_bad_arguments_before_launch(L):
    import matrix_aware_sign_b200 as S
    G = (S.SmuonMat * 2)(S.SmuonMat(4096, 8, 8, 8, S.F32), S.SmuonMat(4096, 8, 8, 8, S.BF16))
    gs = S.GradStream(0, 0, 1.0, 0)
    assert L.smuon_harness_gaussian(None, 1, 1, ctypes.byref(gs), 1, None) == -1
    assert L.smuon_harness_gaussian(G, 1, 1, None, 1, None) == -1
    assert L.smuon_harness_gaussian(G, 0, 1, ctypes.byref(gs), 1, None) == -1
    assert L.smuon_harness_gaussian(G, 1, 2, ctypes.byref(gs), 1, None) == -3  # the second is not F32
    # a LionMuon step without gradients needs a stream in its state
    W = (S.SmuonMat * 1)(S.SmuonMat(4096, 8, 8, 8, S.F32))
    mom = (S.SmuonMat * 1)(S.SmuonMat(8192, 8, 8, 8, S.F32))
    st = S.LionMuonState(1, 1, W, mom, 0, None)
    assert L.lionmuon_step(ctypes.byref(st), 4, 0.9, 0.99, 0.01, 1.5, -0.5, 0.0, 5, 0, 0, None, None, 0, None,
                           None) == -1
    assert b"no gradient stream" in L.smuon_last_error()
    assert st.t == 0


def test_gram_only_rejects_unsupported_requests(L):
    import matrix_aware_sign_b200 as S
    m = (S.SmuonMat * 1)(S.SmuonMat(4096, 8, 16, 16, S.F32))
    q = (S.SmuonMat * 1)(S.SmuonMat(8192, 8, 8, 8, S.BF16))
    two = (S.SmuonMat * 2)(S.SmuonMat(4096, 8, 16, 16, S.F32), S.SmuonMat(4096, 8, 16, 16, S.F32))
    q2 = (S.SmuonMat * 2)(S.SmuonMat(8192, 8, 8, 8, S.BF16), S.SmuonMat(8192, 8, 8, 8, S.BF16))
    g = S.NS_GRAM_ONLY
    args = lambda c: (c, 5, 1e-7)
    # needs EMIT_Q
    assert L.smuon_ns(m, m, 1, None, 0.0, 3.4445, -4.775, *args(2.0315), g, q, None, None, 0, None, None) == -1
    # one matrix only, tensor cores only, c != 0
    assert L.smuon_ns(two, two, 2, None, 0.0, 3.4445, -4.775, *args(2.0315), g | S.NS_EMIT_Q, q2, None, None, 0,
                      None, None) == -4
    assert L.smuon_ns(m, m, 1, None, 0.0, 3.4445, -4.775, *args(2.0315), g | S.NS_EMIT_Q | S.NS_FP32_REF, q, None,
                      None, 0, None, None) == -4
    assert L.smuon_ns(m, m, 1, None, 0.0, 1.5, -0.5, *args(0.0), g | S.NS_EMIT_Q, q, None, None, 0, None,
                      None) == -4


def test_spectral_flag_validation_and_workspace(L):
    """SMUON_NS_SPECTRAL excludes NO_NORMALIZE, EMIT_Q and GRAM_ONLY; its
    workspace adds the Lanczos vectors (66 vectors of m floats per matrix, the
    tridiagonal coefficients) and, in split mode (whose plain chain keeps A as
    its hi and lo parts only), the f32 A that the Lanczos run reads."""
    import torch
    import matrix_aware_sign_b200 as S
    m = (S.SmuonMat * 1)(S.SmuonMat(4096, 8, 16, 16, S.F32))
    q = (S.SmuonMat * 1)(S.SmuonMat(8192, 8, 8, 8, S.BF16))
    sp = S.NS_SPECTRAL
    for extra in (S.NS_NO_NORMALIZE, S.NS_EMIT_Q, S.NS_GRAM_ONLY | S.NS_EMIT_Q):
        assert L.smuon_ns(m, m, 1, None, 0.0, 3.4445, -4.775, 2.0315, 5, 1e-7, sp | extra, q, None, None, 0, None,
                          None) == -4
        assert b"SMUON_NS_SPECTRAL" in L.smuon_last_error()
    mats = [torch.zeros(s) for s in [(256, 1024), (64, 147), (300, 200)]]
    for flags in (0, S.NS_SPLIT_BF16, S.NS_FP32_REF):
        base = S.smuon_ns_workspace_bytes(mats, 5, flags)
        spec = S.smuon_ns_workspace_bytes(mats, 5, flags | sp)
        lz = 4 * 66 * (256 + 64 + 200) + 4 * 2 * 64 * 3  # at most 64 Lanczos steps: 65 vectors and w
        # f32 A per group [count][m][ldm], ldm = m rounded up to 128
        af = 4 * (256 * 256 + 64 * 128 + 200 * 256) if flags == S.NS_SPLIT_BF16 else 0
        assert base + lz + af <= spec <= base + lz + af + 4 * 256 * 4 + 3 * 256, (base, spec)


def test_int8_sign_sources_reject_packed_message(L):
    """I8 sign matrices are accepted as the U source of smuon_update, but not
    with packed_out (the message is packed by smuon_sign_pack)."""
    import ctypes
    import matrix_aware_sign_b200 as S
    W = (S.SmuonMat * 1)(S.SmuonMat(4096, 8, 32, 32, S.F32))
    U = (S.SmuonMat * 2)(S.SmuonMat(8192, 8, 32, 32, S.I8), S.SmuonMat(12288, 8, 32, 32, S.I8))
    packed = (ctypes.c_void_p * 1)(16384)
    assert L.smuon_update(W, 1, U, None, None, 2, 0.01, 0, S.VOTE_INT8, packed, None, None, None) == -4
    assert b"packed_out needs F32 or BF16 U" in L.smuon_last_error()


def test_size_limits_are_checked_on_the_host(L):
    """Each side in 1..65536 and at most 4096 matrices per call: the limits
    are rejected (or, at the limit, sized) before anything is enqueued."""
    import ctypes
    import matrix_aware_sign_b200 as S
    out = ctypes.c_size_t(0)
    edge = (S.SmuonMat * 1)(S.SmuonMat(4096, 1, 65536, 65536, S.F32))
    assert L.smuon_ns_workspace_bytes(edge, 1, 1, 0, ctypes.byref(out)) == 0 and out.value > 0
    for rows, cols in [(1, 65537), (65537, 1), (0, 8), (8, 0)]:
        big = (S.SmuonMat * 1)(S.SmuonMat(4096, rows, cols, max(cols, 1), S.F32))
        assert L.smuon_ns(big, big, 1, None, 0.9, 1.5, -0.5, 0.0, 1, 1e-7, 0, None, None, None, 0, None,
                          None) == -2, (rows, cols)
    many = (S.SmuonMat * 4097)(*[S.SmuonMat(4096, 8, 8, 8, S.F32)] * 4097)
    assert L.smuon_ns(many, many, 4097, None, 0.9, 1.5, -0.5, 0.0, 1, 1e-7, 0, None, None, None, 0, None,
                      None) == -1
    assert b"n_mats" in L.smuon_last_error()


def test_plain_lead_and_bits_outputs_are_checked_before_launch(L):
    """SMUON_NS_PLAIN_LEAD needs the split mode and excludes spectral scaling and the
    cached transform; a 1-bit output needs cols % 32 == 0, ld == cols, 16-byte
    alignment and the tensor-core modes (no device is touched on these paths)."""
    import matrix_aware_sign_b200 as S
    args = (None, 0.9, 3.4445, -4.775, 2.0315, 5, 1e-7)
    m = (S.SmuonMat * 1)(S.SmuonMat(4096, 64, 128, 128, S.F32))
    u = (S.SmuonMat * 1)(S.SmuonMat(4096, 64, 128, 128, S.F32))

    def call(M_in, U, flags, Q=None):
        return L.smuon_ns(M_in, U, 1, *args, flags, Q, None, None, 0, None, None)

    assert call(m, u, S.ns_plain_lead(2)) == -1                       # without the split mode
    assert b"SPLIT" in L.smuon_last_error()
    assert call(m, u, S.NS_SPLIT_BF16 | S.ns_plain_lead(2) | S.NS_SPECTRAL) == -4
    assert call(m, u, S.NS_SPLIT_BF16 | S.ns_plain_lead(2) | S.NS_EMIT_Q, u) == -4
    with pytest.raises(ValueError):
        S.ns_plain_lead(8)
    bits = (S.SmuonMat * 1)(S.SmuonMat(4096, 64, 128, 128, S.BITS))
    assert call(m, bits, S.NS_FP32_REF) == -4                          # CUDA-core modes write no bits
    assert call(m, bits, S.NS_SPLIT_BF16 | S.NS_EMIT_Q, u) == -4       # nor with the cached transform
    m100 = (S.SmuonMat * 1)(S.SmuonMat(4096, 64, 100, 100, S.F32))
    bits100 = (S.SmuonMat * 1)(S.SmuonMat(4096, 64, 100, 100, S.BITS))
    assert call(m100, bits100, 0) == -2                                # cols % 32 != 0
    assert b"cols % 32" in L.smuon_last_error()
    strided = (S.SmuonMat * 1)(S.SmuonMat(4096, 64, 128, 160, S.BITS))
    assert call(m, strided, 0) == -2                                   # a message has no row stride
    unaligned = (S.SmuonMat * 1)(S.SmuonMat(4100, 64, 128, 128, S.BITS))
    assert call(m, unaligned, 0) == -1


def test_update_rejects_a_packed_output_for_message_sources(L):
    import matrix_aware_sign_b200 as S
    W = (S.SmuonMat * 1)(S.SmuonMat(4096, 8, 64, 64, S.F32))
    U = (S.SmuonMat * 2)(S.SmuonMat(8192, 8, 64, 64, S.BITS), S.SmuonMat(12288, 8, 64, 64, S.BITS))
    po = (ctypes.c_void_p * 1)(16384)
    assert L.smuon_update(W, 1, U, None, None, 2, 0.01, 0, 0, po, None, None, None) == -1
    assert b"message" in L.smuon_last_error()
    mixed = (S.SmuonMat * 2)(S.SmuonMat(8192, 8, 64, 64, S.BITS), S.SmuonMat(12288, 8, 64, 64, S.I8))
    assert L.smuon_update(W, 1, mixed, None, None, 2, 0.01, 0, 0, None, None, None, None) == -3


def test_bits_wrapper_describes_a_message():
    import torch

    import matrix_aware_sign_b200 as S
    b = S.Bits(torch.zeros(S.packed_words(96 * 40), dtype=torch.int32), 96, 40)
    m = S.mat(b)
    assert (m.rows, m.cols, m.ld, m.dtype) == (96, 40, 40, S.BITS)
    with pytest.raises(ValueError):
        S.Bits(torch.zeros(10, dtype=torch.int32), 96, 40)            # too few words
    with pytest.raises(ValueError):
        S.Bits(torch.zeros(S.packed_words(96 * 40), dtype=torch.int64), 96, 40)


def test_sm_pair_choice_is_a_valid_flag_and_sizes_the_tile_tables(L):
    """SMUON_NS_ONE_SM is a known flag. The SM-pair choice is made from the flags
    and the shapes alone (the host's sizing pass and the device's filling pass
    agree): 256 x 256 pair tiles need fewer schedule entries than 128 x 256
    single-SM tiles, so an eligible batch asks for no more workspace in the pair
    form, and a batch with a matrix below 256 rows asks for the same in both."""
    import matrix_aware_sign_b200 as S

    def ws(shapes, flags):
        arr = (S.SmuonMat * len(shapes))(*[S.SmuonMat(4096, r, c, c, S.F32) for r, c in shapes])
        out = ctypes.c_size_t(0)
        assert L.smuon_ns_workspace_bytes(arr, len(shapes), 5, flags, ctypes.byref(out)) == 0
        return out.value

    big = [(768, 2304), (4096, 4096)]
    for fl in (0, S.NS_SPLIT_BF16, S.NS_SPLIT_BF16 | S.NS_EMIT_Q):
        assert ws(big, fl) <= ws(big, fl | S.NS_ONE_SM)
        small = big + [(64, 147)]
        assert ws(small, fl) == ws(small, fl | S.NS_ONE_SM)
    gram = S.NS_SPLIT_BF16 | S.NS_EMIT_Q | S.NS_GRAM_ONLY  # the CacheMuon stages take pairs too
    assert ws([(768, 2304)], gram) <= ws([(768, 2304)], gram | S.NS_ONE_SM)
    assert ws([(200, 700)], gram) == ws([(200, 700)], gram | S.NS_ONE_SM)
