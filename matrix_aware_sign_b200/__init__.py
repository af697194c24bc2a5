"""Thin Python binding of libsmuon.so (the C ABI in include/smuon.h).

Argument marshalling only: every step of the optimizer runs in the library's
CUDA kernels. PyTorch supplies device memory and the current stream. There is
no fallback: if the shared library is missing, importing a function raises.

Functions keep the C names: smuon_ns, smuon_sign_pack, smuon_vote,
smuon_update, cachemuon_reuse_probe, lionmuon_step (plus the workspace
queries). Matrices are 2-D torch tensors with unit column stride.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_float, c_int8, c_int32, c_int64, c_size_t, c_uint32, c_void_p

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsmuon.so")

F32, BF16, I8, BITS = 0, 1, 2, 3
NS_FP32_REF, NS_SPLIT_BF16, NS_NO_NORMALIZE, NS_EMIT_Q, NS_SIMT_BF16 = 1, 2, 4, 8, 16
NS_GRAM_ONLY = 32  # CacheMuon fresh solve iterated on the m x m Gram (with NS_EMIT_Q, one matrix)
NS_SPECTRAL = 64  # spectral-norm normalisation X_0 = M / (||M||_2 + eps) (Lanczos estimate on the device)
NS_TEST_WAIT_EXPIRY = 0x8000  # failure-detection test: the tensor-core stages' pipeline waits run out
NS_ONE_SM = 0x80  # tensor-core stages on single-SM 128 x 256 tiles instead of SM pairs (256 x 256 tiles)


def ns_plain_lead(k: int) -> int:
    """SMUON_NS_PLAIN_LEAD(k): with NS_SPLIT_BF16, the first k Newton-Schulz steps use plain BF16 operands."""
    if not 0 <= k <= 7:
        raise ValueError("k must be in 0..7")
    return k << 12
VOTE_POPCOUNT, VOTE_INT8 = 0, 1
VOTE_TEST_WAIT_EXPIRY = 0x100  # failure-detection test: the bulk-copy 1-bit vote's waits run out, W unchanged
LION_MUON_VOTE = 0x100  # lionmuon_step ns_flags: Muon steps as Sign-Muon steps (per-worker NS + vote)
DEV_NONFINITE_NORM, DEV_WAIT_TIMEOUT = 1, 2

STATUS_NAMES = {0: "OK", -1: "INVALID_ARG", -2: "SHAPE", -3: "DTYPE", -4: "UNSUPPORTED",
                -5: "WORKSPACE", -6: "CUDA"}


class SmuonError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"smuon status {code} ({STATUS_NAMES.get(code, '?')}): {msg}")
        self.code = code


class SmuonMat(ctypes.Structure):
    _fields_ = [("data", c_void_p), ("rows", c_int32), ("cols", c_int32), ("ld", c_int64),
                ("dtype", c_int32)]


class CacheMuonCounters(ctypes.Structure):
    _fields_ = [("hits", c_int64), ("misses", c_int64), ("probes", c_int64), ("reserved", c_int64)]


class TraceRec(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 40), ("kind", c_int32), ("work", ctypes.c_double),
                ("nominal", ctypes.c_double), ("ms", c_float)]


class GradStream(ctypes.Structure):
    """smuon_grad_stream: worker k's gradient of matrix j is keyed (seed_base + k, matrix_base + j)."""
    _fields_ = [("seed_base", c_uint32), ("matrix_base", c_uint32), ("sigma", c_float), ("reserved", c_uint32)]


class LionMuonState(ctypes.Structure):
    _fields_ = [("n_layers", c_int32), ("workers", c_int32), ("W", POINTER(SmuonMat)),
                ("mom", POINTER(SmuonMat)), ("t", c_int64), ("grad", POINTER(GradStream))]


_lib = None


def lib() -> ctypes.CDLL:
    """Loads libsmuon.so once; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m matrix_aware_sign_b200.build` (there is no fallback)")
        L = ctypes.CDLL(LIB_PATH)
        M = POINTER(SmuonMat)
        sigs = {
            "smuon_last_error": (ctypes.c_char_p, []),
            "smuon_version": (c_int32, []),
            "smuon_launch_count": (c_int64, []),
            "smuon_trace_enable": (None, [c_int32]),
            "smuon_trace_read": (c_int32, [POINTER(TraceRec), c_int32]),
            "smuon_ns_workspace_bytes": (c_int32, [M, c_int32, c_int32, c_uint32, POINTER(c_size_t)]),
            "smuon_ns": (c_int32, [M, M, c_int32, M, c_float, c_float, c_float, c_float, c_int32, c_float,
                                   c_uint32, M, c_void_p, c_void_p, c_size_t, c_void_p, c_void_p]),
            "smuon_sign_pack": (c_int32, [M, c_int32, c_void_p, c_void_p, c_void_p]),
            "smuon_vote": (c_int32, [c_void_p, c_void_p, c_int32, c_int64, c_int8, c_void_p, c_void_p]),
            "smuon_update": (c_int32, [M, c_int32, M, M, M, c_int32, c_float, c_int8, c_uint32,
                                       POINTER(c_void_p), POINTER(c_void_p), c_void_p, c_void_p]),
            "smuon_ns_static": (c_int32, [M, M, c_int32, M, c_float, c_float, c_float, c_float, c_int32, c_float,
                                          c_uint32, M, c_void_p, c_void_p, c_void_p]),
            "smuon_ns_plan_create": (c_int32, [M, M, c_int32, M, c_float, c_float, c_float, c_float, c_int32,
                                               c_float, c_uint32, M, c_void_p, c_size_t, c_void_p, c_void_p,
                                               POINTER(c_void_p)]),
            "smuon_ns_execute": (c_int32, [c_void_p, c_void_p, c_void_p]),
            "smuon_update_plan_create": (c_int32, [M, c_int32, M, M, M, c_int32, c_float, c_int8, c_uint32,
                                                   POINTER(c_void_p), POINTER(c_void_p), c_void_p,
                                                   POINTER(c_void_p)]),
            "smuon_update_execute": (c_int32, [c_void_p, c_void_p]),
            "smuon_plan_destroy": (None, [c_void_p]),
            "cachemuon_workspace_bytes": (c_int32, [M, POINTER(c_size_t)]),
            "cachemuon_reuse_probe": (c_int32, [M, M, M, c_float, c_float, c_void_p, c_void_p, c_void_p,
                                                c_void_p, c_size_t, c_void_p, c_void_p]),
            "smuon_harness_gaussian": (c_int32, [M, c_int32, c_int32, POINTER(GradStream), c_uint32, c_void_p]),
            "lionmuon_workspace_bytes": (c_int32, [POINTER(LionMuonState), c_int32, c_uint32,
                                                   POINTER(c_size_t)]),
            "lionmuon_step": (c_int32, [POINTER(LionMuonState), c_int32, c_float, c_float, c_float, c_float,
                                        c_float, c_float, c_int32, c_int8, c_uint32, M, c_void_p, c_size_t,
                                        c_void_p, c_void_p]),
        }
        for name, (res, args) in sigs.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(code: int) -> None:
    if code != 0:
        raise SmuonError(code, lib().smuon_last_error().decode())


_DT = {torch.float32: F32, torch.bfloat16: BF16, torch.int8: I8}


class Bits:
    """The 1-bit message of a rows x cols sign matrix (SMUON_BITS): `words` is a
    contiguous int32 tensor of packed_words(rows * cols) words, entry i of the
    row-major flattening at bit i % 32 of word i // 32."""

    def __init__(self, words: torch.Tensor, rows: int, cols: int):
        if words.dtype != torch.int32 or not words.is_contiguous() or words.numel() < packed_words(rows * cols):
            raise ValueError("words must be a contiguous int32 tensor of packed_words(rows * cols) words")
        self.words, self.rows, self.cols = words, int(rows), int(cols)

    @property
    def shape(self):
        return (self.rows, self.cols)

    @property
    def device(self):
        return self.words.device

    @staticmethod
    def empty(rows: int, cols: int, device=None) -> "Bits":
        return Bits(torch.zeros(packed_words(rows * cols), dtype=torch.int32, device=device or "cuda"), rows, cols)


def mat(t) -> SmuonMat:
    """Describes a 2-D row-major tensor (unit column stride), or a Bits message."""
    if isinstance(t, Bits):
        return SmuonMat(t.words.data_ptr(), t.rows, t.cols, t.cols, BITS)
    if t.dim() != 2 or (t.stride(1) != 1 and t.shape[1] > 1):
        raise ValueError("matrices must be 2-D with unit column stride")
    if t.dtype not in _DT:
        raise ValueError(f"dtype {t.dtype} is not supported")
    ld = t.stride(0) if t.shape[0] > 1 else t.shape[1]
    return SmuonMat(t.data_ptr(), t.shape[0], t.shape[1], max(ld, t.shape[1]), _DT[t.dtype])


def _mats(ts):
    if ts is None:
        return None
    arr = (SmuonMat * len(ts))(*[mat(t) for t in ts])
    return arr


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream


def workspace(nbytes: int, device=None) -> torch.Tensor:
    """Caller-owned workspace (torch allocation, 512-byte aligned)."""
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device or "cuda")


# ---------------------------------------------------------------- diagnostics
WORK_FLOPS, WORK_BYTES = 0, 1


def launch_count() -> int:
    return lib().smuon_launch_count()


def trace_enable(on: bool = True) -> None:
    lib().smuon_trace_enable(1 if on else 0)


def trace_read() -> list[dict]:
    """Synchronises on the logged launch events and returns and clears them."""
    n = lib().smuon_trace_read(None, 0)
    if n == 0:
        return []
    buf = (TraceRec * n)()
    got = lib().smuon_trace_read(buf, n)
    return [dict(name=r.name.decode(), kind=r.kind, work=r.work, nominal=r.nominal, ms=r.ms) for r in buf[:got]]


# ---------------------------------------------------------------- smuon_ns
def smuon_ns_workspace_bytes(M_in, iters: int, flags: int = 0) -> int:
    arr = _mats(M_in)
    out = c_size_t(0)
    _check(lib().smuon_ns_workspace_bytes(arr, len(M_in), iters, flags, ctypes.byref(out)))
    return out.value


def smuon_ns(M_in, U_out, a, b, c, iters, G=None, beta=0.0, eps=1e-7, flags=0, Q_out=None,
             skip_if=None, ws=None, status=None, stream=None):
    """Momentum (when G is given) + Frobenius normalisation + K Newton-Schulz steps."""
    if ws is None:
        ws = workspace(smuon_ns_workspace_bytes(M_in, iters, flags), M_in[0].device)
    _check(lib().smuon_ns(_mats(M_in), _mats(U_out), len(M_in), _mats(G), beta, a, b, c, iters, eps, flags,
                          _mats(Q_out), _ptr(skip_if), ws.data_ptr(), ws.numel(), _ptr(status),
                          _stream(stream)))
    return ws


NS_STATIC_SCRATCH_BYTES = 32 << 20


def smuon_ns_static(M_in, U_out, a, b, c, iters, G=None, beta=0.0, eps=1e-7, flags=0, Q_out=None,
                    skip_if=None, status=None, stream=None):
    """smuon_ns with the library's fixed device scratch array (no workspace, no allocation)."""
    _check(lib().smuon_ns_static(_mats(M_in), _mats(U_out), len(M_in), _mats(G), beta, a, b, c, iters, eps, flags,
                                 _mats(Q_out), _ptr(skip_if), _ptr(status), _stream(stream)))


class NsPlan:
    """smuon_ns prepared once (plan uploaded into `ws`); run() enqueues only the kernels."""

    def __init__(self, M_in, U_out, a, b, c, iters, G=None, beta=0.0, eps=1e-7, flags=0, Q_out=None, ws=None,
                 status=None, stream=None):
        self.tensors = (list(M_in), list(U_out), G, Q_out, status)  # keep the buffers alive
        if ws is None:
            ws = workspace(smuon_ns_workspace_bytes(M_in, iters, flags), M_in[0].device)
        self.ws = ws
        h = c_void_p()
        _check(lib().smuon_ns_plan_create(_mats(M_in), _mats(U_out), len(M_in), _mats(G), beta, a, b, c, iters, eps,
                                          flags, _mats(Q_out), ws.data_ptr(), ws.numel(), _ptr(status),
                                          _stream(stream), ctypes.byref(h)))
        self.handle = h

    def run(self, skip_if=None, stream=None):
        _check(lib().smuon_ns_execute(self.handle, _ptr(skip_if), _stream(stream)))

    def __del__(self):
        h = getattr(self, "handle", None)
        if h and _lib is not None:
            _lib.smuon_plan_destroy(h)
            self.handle = None


class UpdatePlan:
    """smuon_update prepared once; run() enqueues only the kernels."""

    def __init__(self, W, eta, U=None, votes=None, dense=None, M=1, tie_value=0, vote_kind=VOTE_POPCOUNT,
                 packed_out=None, vote_out=None, status=None):
        Uflat = None if U is None else [u for layer in U for u in layer]
        self.tensors = (None if W is None else list(W), Uflat, votes, dense, packed_out, vote_out, status)
        n = len(U) if W is None else len(W)  # W None: signs, message and votes only
        po = None if packed_out is None else (c_void_p * n)(*[_ptr(p) for p in packed_out])
        vo = None if vote_out is None else (c_void_p * n)(*[_ptr(v) for v in vote_out])
        h = c_void_p()
        _check(lib().smuon_update_plan_create(_mats(W), n, _mats(Uflat), _mats(votes), _mats(dense), M, eta,
                                              tie_value, vote_kind, po, vo, _ptr(status), ctypes.byref(h)))
        self.handle = h

    def run(self, stream=None):
        _check(lib().smuon_update_execute(self.handle, _stream(stream)))

    def __del__(self):
        h = getattr(self, "handle", None)
        if h and _lib is not None:
            _lib.smuon_plan_destroy(h)
            self.handle = None


# ---------------------------------------------------------------- sign / vote / update
def packed_words(n: int) -> int:
    return ((n + 127) // 128) * 4


def smuon_sign_pack(U, packed=None, signs_i8=None, stream=None):
    _check(lib().smuon_sign_pack(_mats(U), len(U), _ptr(packed), _ptr(signs_i8), _stream(stream)))


def smuon_vote(M: int, N: int, vote, packed=None, signs_i8=None, tie_value: int = 0, stream=None):
    _check(lib().smuon_vote(_ptr(packed), _ptr(signs_i8), M, N, tie_value, vote.data_ptr(), _stream(stream)))


def smuon_update(W, eta: float, U=None, votes=None, dense=None, M: int = 1, tie_value: int = 0,
                 vote_kind: int = VOTE_POPCOUNT, packed_out=None, vote_out=None, status=None, stream=None):
    """U is a list over layers of lists over workers (flattened worker-minor).
    W may be None with U and packed_out / vote_out: signs, message and votes only.
    status: optional device int32 tensor for SMUON_DEV_* bits."""
    Uflat = None if U is None else [u for layer in U for u in layer]
    n = len(U) if W is None else len(W)
    po = None if packed_out is None else (c_void_p * n)(*[_ptr(p) for p in packed_out])
    vo = None if vote_out is None else (c_void_p * n)(*[_ptr(v) for v in vote_out])
    _check(lib().smuon_update(_mats(W), n, _mats(Uflat), _mats(votes), _mats(dense), M, eta, tie_value,
                              vote_kind, po, vo, _ptr(status), _stream(stream)))


# ---------------------------------------------------------------- CacheMuon
def cachemuon_workspace_bytes(M_t) -> int:
    out = c_size_t(0)
    _check(lib().cachemuon_workspace_bytes(ctypes.byref(mat(M_t)), ctypes.byref(out)))
    return out.value


def new_counters(device=None) -> torch.Tensor:
    """Device storage for cachemuon_counters (4 x int64)."""
    return torch.zeros(4, dtype=torch.int64, device=device or "cuda")


def cachemuon_reuse_probe(Q, M_t, D_hat, gamma, err, accept, counters=None, eps=1e-7, ws=None, status=None,
                          stream=None):
    if ws is None:
        ws = workspace(cachemuon_workspace_bytes(M_t), M_t.device)
    qm = None if Q is None else ctypes.byref(mat(Q))
    _check(lib().cachemuon_reuse_probe(qm, ctypes.byref(mat(M_t)), ctypes.byref(mat(D_hat)), gamma, eps,
                                       err.data_ptr(), accept.data_ptr(), _ptr(counters), ws.data_ptr(),
                                       ws.numel(), _ptr(status), _stream(stream)))
    return ws


class CacheMuon:
    """CacheMuon schedule for one matrix, kept on the device: every step probes
    the cached transform (reuse D_hat = Q X_t, residual, accept flag) and then
    enqueues the fresh solve, whose kernels return at once when the flag says
    the cached transform was accepted. The host never waits on the GPU; read
    counters() at the end."""

    def __init__(self, M_t, D_out, gamma, coeffs, iters, flags=NS_SPLIT_BF16, eps=1e-7):
        dev = M_t.device
        m = min(M_t.shape)
        self.M, self.D, self.gamma, self.eps = M_t, D_out, float(gamma), eps
        self.Q = torch.zeros((m, m), dtype=torch.bfloat16, device=dev)
        self.err = torch.zeros(1, dtype=torch.float32, device=dev)
        self.accept = torch.zeros(1, dtype=torch.int32, device=dev)
        self.cnt = new_counters(dev)
        self.ws_probe = workspace(cachemuon_workspace_bytes(M_t), dev)
        self.fresh = NsPlan([M_t], [D_out], *coeffs, iters, flags=flags | NS_EMIT_Q, Q_out=[self.Q], eps=eps)
        self.steps = 0

    def probe(self, stream=None):
        """The step's probe: D_hat = Q X_t into D, its residual and the accept flag (no cache on the first step)."""
        cachemuon_reuse_probe(self.Q if self.steps > 0 else None, self.M, self.D, self.gamma, self.err, self.accept,
                              self.cnt, eps=self.eps, ws=self.ws_probe, stream=stream)

    def refresh(self, stream=None):
        """The step's fresh solve (D and Q), whose kernels return at once when the probe accepted."""
        self.fresh.run(skip_if=self.accept, stream=stream)
        self.steps += 1

    def step(self, stream=None):
        self.probe(stream)
        self.refresh(stream)

    def counters(self) -> dict:
        h, mi, pr, _ = self.cnt.tolist()
        return {"hits": h, "misses": mi, "probes": pr}


# ---------------------------------------------------------------- LionMuon
class LionMuon:
    """Holds the C lionmuon_state for lists W[layer] and mom[layer][worker].
    With `grad` (a GradStream), lionmuon_step may be called with G=None: the
    kernels then draw the workers' gradients from the counter-based streams."""

    def __init__(self, W, mom, t: int = 0, grad: GradStream | None = None):
        self.W = list(W)
        self.mom = [list(m) for m in mom]
        self.workers = len(self.mom[0])
        self._w = _mats(self.W)
        self._m = _mats([m for layer in self.mom for m in layer])
        self.grad = grad
        self.state = LionMuonState(len(self.W), self.workers, self._w, self._m, t,
                                   None if grad is None else ctypes.pointer(grad))

    @property
    def t(self) -> int:
        return self.state.t

    def workspace_bytes(self, iters: int, ns_flags: int = 0) -> int:
        out = c_size_t(0)
        _check(lib().lionmuon_workspace_bytes(ctypes.byref(self.state), iters, ns_flags, ctypes.byref(out)))
        return out.value


def lionmuon_step(opt: LionMuon, G, P, beta1, beta2, eta, a, b, c, iters, tie_value=0, ns_flags=0, ws=None,
                  status=None, stream=None):
    """G is a list over layers of lists over workers, or None to draw the
    gradients in-kernel from opt.grad at step t + 1. Returns the workspace used."""
    if ws is None:
        ws = workspace(opt.workspace_bytes(iters, ns_flags), opt.W[0].device)
    Gflat = None if G is None else _mats([g for layer in G for g in layer])
    _check(lib().lionmuon_step(ctypes.byref(opt.state), P, beta1, beta2, eta, a, b, c, iters, tie_value, ns_flags,
                               Gflat, ws.data_ptr(), ws.numel(), _ptr(status), _stream(stream)))
    return ws


def smuon_harness_gaussian(G, workers: int, stream_desc: GradStream, step: int, stream=None):
    """G: flat list [layer * workers + worker] of float32 matrices, filled
    with the counter-based gradient streams at `step`."""
    n = len(G)
    if n % workers:
        raise ValueError("len(G) must be a multiple of workers")
    _check(lib().smuon_harness_gaussian(_mats(G), n // workers, workers, ctypes.byref(stream_desc), step,
                                        _stream(stream)))
