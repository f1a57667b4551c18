"""Measured gather ceilings for the roofline of the sparse attention (libdsaprobe.so).

The attention's dominant traffic is a gather of random 256-byte rows (one KV head of one
selected cache row, for K and for V).  Where those rows come from decides its ceiling:
L2 when the K/V cache fits there, HBM otherwise.  ``gather_peaks`` times the probe kernels
(the same access shape, no arithmetic) on an L2-resident buffer and on one far larger than
L2 and returns the best rate of each, in GB/s.  Measurement support only: the layer never
calls this.
"""
from __future__ import annotations

import ctypes

from . import _build

_lib = None


def _load():
    global _lib
    if _lib is None:
        _build.build_probe()
        L = ctypes.CDLL(_build.PROBE_LIB)
        L.dsa_probe_gather.argtypes = [ctypes.c_void_p, ctypes.c_uint32, ctypes.c_void_p,
                                       ctypes.c_uint32, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_int, ctypes.c_void_p]
        L.dsa_probe_gather.restype = ctypes.c_double
        _lib = L
    return _lib


def gather_rate(buf_bytes: int, variant: int, blocks: int, chunks_per_warp: int = 64,
                reps: int = 5) -> float:
    """GB/s of random 256-byte row reads from a buffer of buf_bytes (a power of two)."""
    import torch

    rows = buf_bytes // 256
    assert rows > 0 and rows & (rows - 1) == 0
    buf = torch.zeros(buf_bytes // 2, dtype=torch.int16, device="cuda")
    # one index per row read, none reused within a launch (a reused row could hit in L2)
    n_idx = 1 << max(22, (blocks * 8 * chunks_per_warp * 32 - 1).bit_length())
    idx = torch.empty(n_idx, dtype=torch.int32, device="cuda")
    sink = torch.empty(blocks * 256 * 4, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    rate = _load().dsa_probe_gather(buf.data_ptr(), rows, idx.data_ptr(), n_idx, variant, blocks,
                                    chunks_per_warp, reps, sink.data_ptr())
    torch.cuda.synchronize()
    del buf, idx, sink
    return rate / 1e9


def gather_peaks(num_sms: int, l2_bytes: int = 64 << 20, hbm_bytes: int = 8 << 30) -> dict:
    """Best measured gather rate (GB/s) from an L2-resident buffer and from HBM, with the
    configurations tried."""
    out = {}
    for name, size in (("l2", l2_bytes), ("hbm", hbm_bytes)):
        tries = {}
        for variant, blocks in ((1, num_sms), (0, num_sms * 8), (3, num_sms), (2, num_sms * 8)):
            kind = "cp.async smem" if variant & 1 else "ld.global regs"
            addr = ", 32-bit index" if variant >= 2 else ""
            tries[f"{kind}{addr} x{blocks} CTAs"] = gather_rate(size, variant, blocks)
        best = max(tries, key=tries.get)
        out[name] = {"gbs": tries[best], "best": best, "tried": tries, "buffer_bytes": size}
    return out
