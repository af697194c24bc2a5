"""CPU oracle for the Sign-Muon / CacheMuon / LionMuon optimizer step.

TEST INFRASTRUCTURE ONLY. Nothing in the product path (the CUDA library and
its Python binding) may import, call or execute anything in this package; only
the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of the
benchmark use it. It shares no code, tables or helpers with the CUDA path.

See ``oracle.smuon_oracle`` for the functions and the passages they follow.
"""
from .smuon_oracle import *  # noqa: F401,F403
