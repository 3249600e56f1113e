"""SureLock on B200: the decoding step of a masked diffusion LM run on the
active (unlocked) rows only, plus the KL sure test that locks converged rows.

The compute path is libsurelock.so (hand-written sm_100a CUDA behind the C ABI
in include/surelock.h).  `token_locking_b200.runtime` is its Python binding;
import it explicitly (it needs torch and a built library).
"""
from ._abi import LIB_PATH, SureLockError, lib  # noqa: F401

__all__ = ["LIB_PATH", "SureLockError", "lib"]
