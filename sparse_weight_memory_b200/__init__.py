"""B200-native (sm_100a) Fast-weight Product Key Memory: the chunked
read-then-write memory step behind a C ABI (include/fwpkm.h).

    from sparse_weight_memory_b200 import FwPKMState
    mem = FwPKMState(N=256 * 256, dq=512, dv=512, topk=8, chunk=256)
    mem.set_tables(subkeys, values)
    out = mem.step(Q, Vtarget, gate, eta=1.0)       # torch CUDA tensors
"""
from .fwpkm import FwPKMState, FwpkmError, load_library, LIB_PATH  # noqa: F401

__all__ = ["FwPKMState", "FwpkmError", "load_library", "LIB_PATH"]
