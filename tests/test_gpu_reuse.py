"""Index reuse across layers: one indexer -> Top-K pass serves the sparse attention of
several layers.

[SAE] "5. Abstract Implementation Sketch of Indexer + Top-K" names the reuse of index
results from previous layers, and [HSA] "Engineering and Evaluation Recommendations" the
reuse of the scoring work.  The library's mechanism is its split ABI: dsa_index_topk (or
dsa_index_scores + dsa_topk) writes the index rows once, and any number of
dsa_sparse_attn_gated calls read them with each layer's own q, K/V cache and gate.  This
test runs that call sequence for two layers and checks each against the oracle's attention
over the first layer's selection.
"""
import numpy as np
import pytest
import torch

import dsa_synth as S
import oracle as O
from tests import parity as PT

pytestmark = pytest.mark.gpu


def _dev(host):
    out = {}
    for k, v in host.items():
        if k in ("q_offsets", "kv_offsets"):
            out[k] = torch.from_numpy(v.astype(np.int32)).cuda()
        elif v.dtype == np.uint16:
            out[k] = torch.from_numpy(v.view(np.int16)).cuda().view(torch.bfloat16)
        else:
            out[k] = torch.from_numpy(np.ascontiguousarray(v)).cuda()
    return out


@pytest.mark.parametrize("fused", [True, False])
def test_one_selection_serves_two_layers(fused):
    import indexer_top_gated_b200 as dsa

    q_lens, kv_lens = [2600, 300], [3000, 700]
    w1 = S.Workload("layer1", q_lens, kv_lens, top_k=256, n_q_heads=32, n_kv_heads=4, seed=0)
    w2 = S.Workload("layer2", q_lens, kv_lens, top_k=256, n_q_heads=32, n_kv_heads=4, seed=1)
    h1, h2 = S.make_host_inputs(w1), S.make_host_inputs(w2)
    d1, d2 = _dev(h1), _dev(h2)
    shape = dsa.workload_shape(w1)
    rg = dsa.ragged(d1["q_offsets"], d1["kv_offsets"], q_lens, kv_lens)
    idx = torch.full((w1.total_q, w1.top_k), -7, dtype=torch.int32, device="cuda")
    if fused:
        _, rec = dsa.dsa_index_topk_workspace_size(shape, rg, w1.total_q)
        ws = torch.empty(rec, dtype=torch.uint8, device="cuda")
        dsa.dsa_index_topk(shape, rg, d1["q_idx"], d1["k_idx"], d1["w"], 0, w1.total_q, idx,
                           w1.top_k, None, ws)
    else:
        ld = max(kv_lens)
        sc = torch.empty((w1.total_q, ld), device="cuda")
        dsa.dsa_index_scores(shape, rg, d1["q_idx"], d1["k_idx"], d1["w"], 0, w1.total_q, sc, ld)
        dsa.dsa_topk(shape, rg, sc, ld, 0, w1.total_q, idx, w1.top_k)
    outs = []
    for d in (d1, d2):
        out = torch.zeros((w1.total_q, 32, 128), dtype=torch.bfloat16, device="cuda")
        dsa.dsa_sparse_attn_gated(shape, rg, d["q"], d["k"], d["v"], idx, w1.top_k, 0,
                                  w1.total_q, d["gate"], out)
        outs.append(out)
    torch.cuda.synchronize()
    assert dsa.dsa_device_status(clear=True) == 0

    o1, o2 = O.Oracle.for_workload(w1, h1), O.Oracle.for_workload(w2, h2)
    rows = sorted(set(range(0, w1.total_q, 53)) | {0, 2599, 2600, w1.total_q - 1})
    idx_ref, out1_ref, _ = o1.layer_rows(rows)
    np.testing.assert_array_equal(idx.cpu().numpy()[rows], idx_ref)
    out2_ref = np.stack([o2.sparse_attn_row(r, idx_ref[i])[0] for i, r in enumerate(rows)])
    g1 = PT.bf16_tensor_to_f64(outs[0])[rows]
    g2 = PT.bf16_tensor_to_f64(outs[1])[rows]
    PT.assert_close(g1, out1_ref, "layer 1 over its own selection")
    PT.assert_close(g2, out2_ref, "layer 2 over layer 1's selection")
    # layer 2's own indexer would select differently (its outputs differ too): the second
    # call really ran on the reused rows
    idx_own, out2_own, _ = o2.layer_rows(rows)
    long_rows = [i for i, r in enumerate(rows) if w1.row_position(r) >= w1.top_k]
    assert all(not np.array_equal(idx_own[i], idx_ref[i]) for i in long_rows)
    assert not PT.close_report(g2[long_rows], out2_own[long_rows])["ok"]
