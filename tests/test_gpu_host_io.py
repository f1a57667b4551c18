"""GPU checks of dsa_prefill_from_host (host buffers, copies overlapped with compute).

The layer runs on row ranges as their inputs arrive, so its output must equal one
dsa_prefill over device-resident inputs bit for bit, for any number of ranges, ragged
batches with histories and the fused indexer -> Top-K path alike.
"""
import numpy as np
import pytest
import torch

import dsa_synth as S

pytestmark = pytest.mark.gpu

dsa = None


@pytest.fixture(scope="module", autouse=True)
def _lib():
    global dsa
    import indexer_top_gated_b200 as m
    dsa = m
    torch.cuda.init()
    yield
    assert dsa.dsa_device_status(clear=True) == 0


def _tensor(x, pinned):
    if x.dtype == np.uint16:
        t = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16)
    elif x.dtype == np.int64:
        t = torch.from_numpy(x.astype(np.int32))
    else:
        t = torch.from_numpy(np.ascontiguousarray(x))
    return t.pin_memory() if pinned else t.cuda()


def _run(w, plans, small_ws=False):
    host_np = S.make_host_inputs(w)
    host = {k: _tensor(v, True) for k, v in host_np.items()}
    dev = {k: _tensor(v, False) for k, v in host_np.items()}
    shape = dsa.workload_shape(w)
    rg = dsa.ragged(dev["q_offsets"], dev["kv_offsets"], w.q_lens, w.kv_lens)
    mn, rec = dsa.dsa_workspace_size(shape, rg)
    # a minimal workspace cannot hold every row's index row: the layer then runs per range
    ws = torch.empty(mn if small_ws else rec, dtype=torch.uint8, device="cuda")
    ref = torch.empty((w.total_q, w.n_q_heads, 128), dtype=torch.bfloat16, device="cuda")
    dsa.dsa_prefill(shape, rg, dev["q_idx"], dev["k_idx"], dev["w"], dev["q"], dev["k"], dev["v"],
                    dev.get("gate"), ref, workspace=ws)
    torch.cuda.synchronize()
    ref = ref.cpu()
    for n_chunks, order in plans:
        # device buffers start as junk: the call must upload every input it reads
        dev2 = {k: torch.full_like(v, 7) for k, v in dev.items()}
        dev2["out"] = torch.zeros((w.total_q, w.n_q_heads, 128), dtype=torch.bfloat16, device="cuda")
        host["out"] = torch.zeros((w.total_q, w.n_q_heads, 128), dtype=torch.bfloat16).pin_memory()
        rg2 = dsa.ragged(dev2["q_offsets"], dev2["kv_offsets"], w.q_lens, w.kv_lens)
        dsa.dsa_prefill_from_host(shape, rg2, host, dev2, n_chunks, ws, order=order)
        torch.cuda.synchronize()
        assert torch.equal(host["out"], ref), f"{n_chunks} ranges, order {order}"


def test_host_prefill_ragged_histories():
    w = S.Workload("custom", [300, 1, 700, 40], [900, 513, 700, 2000], top_k=64, n_q_heads=32,
                   n_kv_heads=4, qkv_scale=S.INV_SQRT_128, gate=True)
    _run(w, [(1, 1), (3, 1), (7, 2), (5, 2), (0, 0)])


def test_host_prefill_layer_per_range_small_workspace():
    w = S.Workload("custom", [300, 1, 700, 40], [900, 513, 700, 2000], top_k=64, n_q_heads=32,
                   n_kv_heads=4, qkv_scale=S.INV_SQRT_128, gate=True)
    _run(w, [(1, 1), (4, 1), (4, 2), (0, 0)], small_ws=True)


def test_host_prefill_fused_path_and_no_gate():
    w = S.Workload("custom", [12288], [12288], top_k=512, n_q_heads=32, n_kv_heads=4,
                   qkv_scale=S.INV_SQRT_128, gate=False)
    _run(w, [(0, 0), (5, 1), (16, 2)])
