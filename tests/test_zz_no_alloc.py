"""dsa_decode_noalloc: the decode entry point that allocates nothing.

Some callers cannot allocate device memory at all (a host framework that owns every
byte of the GPU, a decode loop that must not allocate once it is running, a plugin
that receives tensors but no allocator), so this entry point takes no workspace and
runs in the library's own fixed per-device scratch array.  Its results must match the
workspace-based dsa_decode on the same inputs, call after call (the scratch keeps the
previous call's contents, which must not leak into the next result).

This file is collected last on purpose; it must pass alone in a fresh process and
after the rest of the suite.
"""
import numpy as np
import pytest
import torch

import dsa_synth as S
from tests import parity as PT

pytestmark = pytest.mark.gpu


def _decode_case():
    # long histories so the fixed 32 MiB scratch needs more than one pass
    lens = [600000 + 37 * i for i in range(14)] + [5, 3000]
    return S.Workload("decode_noalloc", [1] * len(lens), lens, top_k=2048, n_q_heads=8,
                      n_kv_heads=1, seed=3)


def test_noalloc_decode_matches_workspace_decode_twice():
    import indexer_top_gated_b200 as dsa

    w = _decode_case()
    dev = S.make_device_inputs(w)
    shape = dsa.workload_shape(w)
    rg = dsa.ragged(dev["q_offsets"], dev["kv_offsets"], w.q_lens, w.kv_lens)
    _, rec = dsa.dsa_workspace_size(shape, rg, True)
    ws = torch.empty(rec, dtype=torch.uint8, device="cuda")
    shp = (w.total_q, w.n_q_heads, w.head_dim)
    out_ref = torch.empty(shp, dtype=torch.bfloat16, device="cuda")
    idx_ref = torch.empty((w.total_q, w.top_k), dtype=torch.int32, device="cuda")
    dsa.dsa_decode(shape, rg, dev["q_idx"], dev["k_idx"], dev["w"], dev["q"], dev["k"], dev["v"],
                   dev["gate"], out_ref, idx_out=idx_ref, workspace=ws)
    ref = PT.bf16_tensor_to_f64(out_ref)
    for call in range(2):
        out = torch.full(shp, float("nan"), dtype=torch.bfloat16, device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        # without idx_out the index rows also live in the fixed scratch
        dsa.dsa_decode_noalloc(shape, rg, dev["q_idx"], dev["k_idx"], dev["w"], dev["q"],
                               dev["k"], dev["v"], dev["gate"], out, err_count=err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        PT.assert_close(PT.bf16_tensor_to_f64(out), ref, f"call {call}")
        idx = torch.full((w.total_q, w.top_k), -7, dtype=torch.int32, device="cuda")
        dsa.dsa_decode_noalloc(shape, rg, dev["q_idx"], dev["k_idx"], dev["w"], dev["q"],
                               dev["k"], dev["v"], dev["gate"], out, idx_out=idx)
        torch.cuda.synchronize()
        assert torch.equal(idx, idx_ref)
        PT.assert_close(PT.bf16_tensor_to_f64(out), ref, f"call {call} with idx_out")
    assert dsa.dsa_device_status() == 0


def test_noalloc_rejects_rows_larger_than_its_scratch():
    import indexer_top_gated_b200 as dsa

    shape = dsa.LayerShape(top_k=2048)
    # 9 million positions: one row of scores alone is 36 MB > 32 MiB
    rg = dsa.Ragged(1, 0x1000, 0x2000, 1, 9_000_000, 1, 9_000_000)
    A = 0x10000
    rc = dsa.lib.dsa_decode_noalloc(shape.params(), rg, A, A, A, A, A, A, None, A, None, None, None)
    assert rc == dsa.DSA_ERR_WORKSPACE
    with pytest.raises(dsa.DsaError, match="workspace"):
        dsa.dsa_decode_noalloc(shape, rg, _Fake(A), _Fake(A), _Fake(A), _Fake(A), _Fake(A),
                               _Fake(A), None, _Fake(A))


class _Fake:
    def __init__(self, a):
        self.a = a

    def data_ptr(self):
        return self.a
