"""GPU parity of every C-ABI entry point against the CPU oracle.

Indexer scores and Top-K index sets are compared bit for bit (dyadic-grid inputs make
every score exact in fp32); gated bf16 outputs are compared within the tolerance in
tests/parity.py.  Sizes span several tiles with ragged tails; the full-size workloads
run in the launch configuration the benchmark uses and are checked on sampled rows.
"""
import numpy as np
import pytest
import torch

import dsa_synth as S
import oracle as O
from tests import parity as PT

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


def _dev(host):
    out = {}
    for k, v in host.items():
        if k in ("q_offsets", "kv_offsets"):
            out[k] = torch.from_numpy(v.astype(np.int32)).cuda()
        elif v.dtype == np.uint16:
            out[k] = torch.from_numpy(v.view(np.int16)).cuda().view(torch.bfloat16)
        else:
            out[k] = torch.from_numpy(v).cuda()
    return out


def _workload(q_lens, kv_lens, K=64, Hq=32, Hkv=4, Hi=4, dtype="bf16", scale=S.INV_SQRT_128,
              gate=True, seed=0):
    return S.Workload("custom", list(q_lens), list(kv_lens), top_k=K, n_q_heads=Hq,
                      n_kv_heads=Hkv, n_idx_heads=Hi, idx_dtype=dtype, qkv_scale=scale, gate=gate,
                      seed=seed)


def _rg(w, dev):
    return dsa.ragged(dev["q_offsets"], dev["kv_offsets"], w.q_lens, w.kv_lens)


def _ld(w):
    return (max(w.kv_lens) + 3) // 4 * 4 + 4


# ----------------------------------------------------------------------------- indexer

INDEXER_CASES = {
    "single_t1000": dict(q_lens=[1000], kv_lens=[1000]),
    "ragged_with_empty": dict(q_lens=[1, 70, 0, 129, 3], kv_lens=[5, 200, 50, 700, 1200]),
    "decode_rows": dict(q_lens=[1] * 20, kv_lens=[1, 2, 127, 128, 129, 300, 1000, 2999] + [777] * 12),
    "fp8_t700": dict(q_lens=[700], kv_lens=[700], dtype="fp8"),
    "fp8_ragged": dict(q_lens=[33, 1, 200], kv_lens=[100, 513, 900], dtype="fp8"),
    "one_head": dict(q_lens=[300], kv_lens=[600], Hi=1),
    "three_heads": dict(q_lens=[65, 130], kv_lens=[65, 400], Hi=3),
}


@pytest.mark.parametrize("case", sorted(INDEXER_CASES))
def test_index_scores_bitexact(case):
    w = _workload(**INDEXER_CASES[case])
    host = S.make_host_inputs(w)
    dev = _dev(host)
    ld = _ld(w)
    scores = torch.full((w.total_q, ld), float("nan"), device="cuda")
    dsa.dsa_index_scores(dsa.workload_shape(w), _rg(w, dev), dev["q_idx"], dev["k_idx"], dev["w"],
                         0, w.total_q, scores, ld)
    got = scores.cpu().numpy()
    orc = O.Oracle.for_workload(w, host)
    for r in range(w.total_q):
        p = w.row_position(r)
        ref = orc.index_scores_row(r)
        np.testing.assert_array_equal(got[r, : p + 1], ref.astype(np.float32), err_msg=f"row {r}")
        assert np.isnan(got[r, p + 1:]).all(), f"row {r} wrote past its causal bound"


def test_index_scores_row_window_and_row_weights():
    """A launch over a window of rows, with per-row head weights."""
    w = _workload([300, 200], [500, 200])
    host = S.make_host_inputs(w)
    rng = np.random.default_rng(0)
    host["w"] = (rng.integers(1, 5, size=(w.total_q, 4)) / 4.0).astype(np.float32)
    dev = _dev(host)
    shape = dsa.workload_shape(w)
    shape.w_row_stride = 4
    ld = _ld(w)
    q0, qn = 250, 180
    scores = torch.full((qn, ld), float("nan"), device="cuda")
    dsa.dsa_index_scores(shape, _rg(w, dev), dev["q_idx"], dev["k_idx"], dev["w"], q0, qn, scores,
                         ld)
    got = scores.cpu().numpy()
    orc = O.Oracle(host, top_k=w.top_k, n_idx_heads=4, idx_dim=64, n_q_heads=w.n_q_heads,
                   n_kv_heads=w.n_kv_heads, head_dim=128, w_row_stride=4)
    for i in range(qn):
        ref = orc.index_scores_row(q0 + i)
        np.testing.assert_array_equal(got[i, : len(ref)], ref.astype(np.float32))


# ----------------------------------------------------------------------------- top-k

def _topk_case(rows, K):
    """rows: list of fp32 arrays; each becomes one sequence with one query at p = n-1."""
    n = [len(x) for x in rows]
    w = _workload([1] * len(rows), n, K=K)
    ld = (max(n) + 3) // 4 * 4
    scores = np.full((len(rows), ld), np.nan, np.float32)
    for i, x in enumerate(rows):
        scores[i, : len(x)] = x
    qo = torch.tensor(w.q_offsets.astype(np.int32), device="cuda")
    ko = torch.tensor(w.kv_offsets.astype(np.int32), device="cuda")
    rg = dsa.ragged(qo, ko, w.q_lens, w.kv_lens)
    st = torch.from_numpy(scores).cuda()
    idx = torch.full((len(rows), K), -7, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(len(rows), dtype=torch.int32, device="cuda")
    dsa.dsa_topk(dsa.workload_shape(w), rg, st, ld, 0, len(rows), idx, K, cnt)
    return idx.cpu().numpy(), cnt.cpu().numpy()


@pytest.mark.parametrize("K", [1, 5, 256, 2048])
def test_topk_bitexact_random_rows(K):
    rng = np.random.default_rng(K)
    rows = []
    for n in (1, K - 1 if K > 1 else 1, K, K + 1, 3 * K + 7, 5000, 33000, 70001):
        for kind in range(5):
            if kind == 0:
                x = rng.integers(0, 4, size=n).astype(np.float32)             # heavy ties
            elif kind == 1:
                x = rng.normal(size=n).astype(np.float32)                      # negatives
            elif kind == 2:
                x = np.zeros(n, np.float32)                                    # all equal
                x[rng.integers(0, n, size=max(1, n // 7))] = -0.0              # -0 == +0
            elif kind == 3:
                x = (rng.integers(0, 64 * 256, size=n) / 256.0).astype(np.float32)  # dyadic
            else:
                x = rng.normal(size=n).astype(np.float32)
                x[rng.integers(0, n, size=n // 3)] = 1.5                       # tie block
            rows.append(x)
    idx, cnt = _topk_case(rows, K)
    for i, x in enumerate(rows):
        ref = O.topk_row(x.astype(np.float64), K)
        np.testing.assert_array_equal(idx[i], ref, err_msg=f"row {i} n={len(x)}")
        assert cnt[i] == min(K, len(x))


def test_topk_on_indexer_scores_matches_oracle_selection():
    w = _workload([1500], [3000], K=256)
    host = S.make_host_inputs(w)
    dev = _dev(host)
    ld = _ld(w)
    rg = _rg(w, dev)
    shape = dsa.workload_shape(w)
    scores = torch.empty((w.total_q, ld), device="cuda")
    dsa.dsa_index_scores(shape, rg, dev["q_idx"], dev["k_idx"], dev["w"], 0, w.total_q, scores, ld)
    idx = torch.empty((w.total_q, 256), dtype=torch.int32, device="cuda")
    dsa.dsa_topk(shape, rg, scores, ld, 0, w.total_q, idx, 256)
    got = idx.cpu().numpy()
    orc = O.Oracle.for_workload(w, host)
    for r in range(0, w.total_q, 7):
        ref = O.topk_row(orc.index_scores_row(r), 256)
        np.testing.assert_array_equal(got[r], ref)


# ----------------------------------------------------------------------------- attention

ATTN_CASES = {
    "gqa8": dict(Hq=32, Hkv=4),
    "mha": dict(Hq=8, Hkv=8),
    "gqa16": dict(Hq=32, Hkv=2),
    "kv16": dict(Hq=32, Hkv=16),
    "one_kv": dict(Hq=8, Hkv=1),
}


def _attn_run(w, dev, idx, lse=True, err=True, gate=True):
    out = torch.zeros((w.total_q, w.n_q_heads, w.head_dim), dtype=torch.bfloat16, device="cuda")
    lse_t = torch.zeros((w.total_q, w.n_q_heads), device="cuda") if lse else None
    err_t = torch.zeros(1, dtype=torch.int32, device="cuda") if err else None
    dsa.dsa_sparse_attn_gated(dsa.workload_shape(w), _rg(w, dev), dev["q"], dev["k"], dev["v"],
                              idx, idx.shape[1], 0, w.total_q, dev.get("gate") if gate else None,
                              out, lse_t, err_t)
    return out, lse_t, err_t


@pytest.mark.parametrize("case", sorted(ATTN_CASES))
def test_sparse_attn_matches_oracle(case):
    cfg = ATTN_CASES[case]
    w = _workload([40, 1, 90], [300, 50, 90], K=96, **cfg)
    host = S.make_host_inputs(w)
    dev = _dev(host)
    orc = O.Oracle.for_workload(w, host)
    idx_ref, out_ref, lse_ref = orc.layer_rows(range(w.total_q))
    out, lse, err = _attn_run(w, dev, torch.from_numpy(idx_ref).cuda())
    PT.assert_close(PT.bf16_tensor_to_f64(out), out_ref, case)
    np.testing.assert_allclose(lse.cpu().numpy(), lse_ref, rtol=1e-5, atol=1e-5)
    assert int(err.item()) == 0


@pytest.mark.parametrize("case", ["gqa8", "mha", "gqa16"])
def test_sparse_attn_gated_mix_matches_oracle(case):
    """The gate mixing in a second branch: sigmoid(g) o + (1 - sigmoid(g)) o2."""
    cfg = ATTN_CASES[case]
    w = _workload([40, 1, 90], [300, 50, 90], K=96, **cfg)
    host = S.make_host_inputs(w)
    dev = _dev(host)
    orc = O.Oracle.for_workload(w, host)
    idx_ref, out_gated, _ = orc.layer_rows(range(w.total_q))
    rng = np.random.default_rng(5)
    o2_bits = S.f32_to_bf16_bits((rng.normal(size=(w.total_q, w.n_q_heads, 128)) * 2e-3)
                                 .astype(np.float32))
    ref = np.stack([orc.sparse_attn_mix_row(r, idx_ref[r], o2_bits[r]) for r in range(w.total_q)])
    o2 = torch.from_numpy(o2_bits.view(np.int16)).cuda().view(torch.bfloat16)
    idx_t = torch.from_numpy(idx_ref).cuda()
    shape = dsa.workload_shape(w)
    out = torch.zeros((w.total_q, w.n_q_heads, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((w.total_q, w.n_q_heads), device="cuda")
    dsa.dsa_sparse_attn_gated_mix(shape, _rg(w, dev), dev["q"], dev["k"], dev["v"], idx_t, w.top_k,
                                  0, w.total_q, dev["gate"], o2, out, lse)
    torch.cuda.synchronize()
    PT.assert_close(PT.bf16_tensor_to_f64(out), ref, case + " mix")
    # the second branch matters: the gated-only reference must fail the same check
    with pytest.raises(AssertionError):
        PT.assert_close(PT.bf16_tensor_to_f64(out), out_gated, case + " mix vs gated")
    # a zero second branch gives dsa_sparse_attn_gated's output bit for bit
    zero = torch.zeros_like(o2)
    out0 = torch.zeros_like(out)
    dsa.dsa_sparse_attn_gated_mix(shape, _rg(w, dev), dev["q"], dev["k"], dev["v"], idx_t, w.top_k,
                                  0, w.total_q, dev["gate"], zero, out0)
    out_g, _, _ = _attn_run(w, dev, idx_t, lse=False, err=False)
    torch.cuda.synchronize()
    assert torch.equal(out0, out_g)


def test_sparse_attn_sharp_softmax_and_no_gate():
    """q, k ~ N(0,1): the softmax is far from uniform; also the ungated path."""
    w = _workload([64], [1000], K=512, scale=1.0, gate=False)
    host = S.make_host_inputs(w)
    dev = _dev(host)
    idx_ref, out_ref, _ = O.Oracle.for_workload(w, host).layer_rows(range(w.total_q))
    out, _, _ = _attn_run(w, dev, torch.from_numpy(idx_ref).cuda(), gate=False)
    PT.assert_close(PT.bf16_tensor_to_f64(out), out_ref, "sharp")


def test_sparse_attn_any_order_padding_and_bad_entries():
    """Indices in any order, padding anywhere, out-of-range entries skipped and counted."""
    w = _workload([3], [200], K=16)
    host = S.make_host_inputs(w)
    dev = _dev(host)
    rows = np.array([
        [5, -1, 199, 0, 17, -1, 3, 100, 150, -1, 42, 7, 8, 9, -1, 1],        # p = 197
        [198, 300, -1, 2, 4000, 6, -1, -1, -1, -1, -1, -1, -1, -1, -1, 11],   # p = 198
        [-1] * 16,                                                         # nothing selected
    ], dtype=np.int32)
    out, lse, err = _attn_run(w, dev, torch.from_numpy(rows).cuda())
    orc = O.Oracle.for_workload(w, host)
    got = PT.bf16_tensor_to_f64(out)
    for r in range(3):
        p = w.row_position(r)
        clean = np.where(rows[r] <= p, rows[r], -1).astype(np.int32)
        ref, lref = orc.sparse_attn_row(r, clean)
        if r < 2:
            PT.assert_close(got[r], ref, f"row {r}")
            np.testing.assert_allclose(lse.cpu().numpy()[r], lref, rtol=1e-5)
        else:
            assert np.all(got[r] == 0) and np.all(np.isneginf(lse.cpu().numpy()[r]))
    bad = sum(int(np.sum(rows[r] > w.row_position(r))) for r in range(3))
    assert bad == 3 and int(err.item()) == bad


def test_tolerance_check_discriminates():
    """One swapped index or a dropped gate must fail the parity check."""
    w = _workload([16], [600], K=64)
    host = S.make_host_inputs(w)
    dev = _dev(host)
    idx_ref, out_ref, _ = O.Oracle.for_workload(w, host).layer_rows(range(w.total_q))
    out, _, _ = _attn_run(w, dev, torch.from_numpy(idx_ref).cuda())
    assert PT.close_report(PT.bf16_tensor_to_f64(out), out_ref)["ok"]
    bad = idx_ref.copy()
    for r in range(len(bad)):
        sel = set(bad[r].tolist())
        bad[r, 0] = next(j for j in range(w.row_position(r) + 1) if j not in sel)
    out2, _, _ = _attn_run(w, dev, torch.from_numpy(bad).cuda())
    assert not PT.close_report(PT.bf16_tensor_to_f64(out2), out_ref)["ok"]
    out3, _, _ = _attn_run(w, dev, torch.from_numpy(idx_ref).cuda(), gate=False)
    assert not PT.close_report(PT.bf16_tensor_to_f64(out3), out_ref)["ok"]


# ----------------------------------------------------------------------------- whole layer

LAYER_CASES = [
    ("prefill_t4096_k256", 8),
    ("prefill_t32768_k2048", 32),
    ("decode_b64_l131072", 64),
    ("prefill_t131072_needles", 64),
    ("mixed_serving", 64),
]


def _run_layer(w, dev, ws_bytes=None):
    shape = dsa.workload_shape(w)
    rg = _rg(w, dev)
    decode = max(w.q_lens) == 1
    mn, rec = dsa.dsa_workspace_size(shape, rg, decode)
    ws_bytes = rec if ws_bytes is None else ws_bytes
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    out = torch.zeros((w.total_q, w.n_q_heads, w.head_dim), dtype=torch.bfloat16, device="cuda")
    idx = torch.full((w.total_q, w.top_k), -7, dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    fn = dsa.dsa_decode if decode else dsa.dsa_prefill
    fn(shape, rg, dev["q_idx"], dev["k_idx"], dev["w"], dev["q"], dev["k"], dev["v"], dev["gate"],
       out, idx_out=idx, err_count=err, workspace=ws, ws_bytes=ws_bytes)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return idx, out


@pytest.mark.parametrize("name,scale", LAYER_CASES)
def test_layer_reduced_sizes_all_rows(name, scale):
    w = S.workload(name, scale_down=scale)
    dev = S.make_device_inputs(w)
    idx, out = _run_layer(w, dev)
    host = S.make_host_inputs(w)
    rows = list(range(w.total_q))
    idx_ref, out_ref, _ = O.Oracle.for_workload(w, host).layer_rows(rows)
    np.testing.assert_array_equal(idx.cpu().numpy(), idx_ref)
    PT.assert_close(PT.bf16_tensor_to_f64(out), out_ref, name)
    for r in w.needle_rows:
        assert set(w.needle_pos) <= set(idx[r].cpu().numpy().tolist())


def test_layer_many_passes_small_workspace():
    """A workspace of a few rows forces many indexer / Top-K / attention passes."""
    w = S.workload("prefill_t32768_k2048", scale_down=64)
    dev = S.make_device_inputs(w)
    shape = dsa.workload_shape(w)
    mn, _ = dsa.dsa_workspace_size(shape, _rg(w, dev))
    idx_a, out_a = _run_layer(w, dev)
    idx_b, out_b = _run_layer(w, dev, ws_bytes=mn * 37 + 5)
    assert torch.equal(idx_a, idx_b)
    assert torch.equal(out_a, out_b)


@pytest.mark.parametrize("name", S.WORKLOADS)
def test_full_size_sampled_rows(name):
    """Full-size workloads in the benchmark's launch configuration, sampled rows."""
    w = S.workload(name)
    free, _ = torch.cuda.mem_get_info()
    if w.device_bytes() * 1.1 > free:
        pytest.skip(f"needs {w.device_bytes() / 2**30:.1f} GiB")
    dev = S.make_device_inputs(w)
    idx, out = _run_layer(w, dev)
    rows = PT.sample_rows(w, 40)
    assert len(rows) >= 40
    for r in rows:
        idx_ref, out_ref, _, _ = PT.oracle_row(w, r)
        np.testing.assert_array_equal(idx[r].cpu().numpy(), idx_ref, err_msg=f"row {r}")
        PT.assert_close(PT.bf16_tensor_to_f64(out[r]), out_ref, f"{name} row {r}")
    for r in w.needle_rows:
        assert set(w.needle_pos) <= set(idx[r].cpu().numpy().tolist())
    del dev, idx, out
    torch.cuda.empty_cache()


def test_full_size_discrimination():
    """At the benchmark's size (T = 32768, K = 2048): one swapped index, or a dropped gate,
    fails the parity check on every sampled row, while the layer's own output passes."""
    w = S.workload("prefill_t32768_k2048")
    dev = S.make_device_inputs(w)
    idx, out = _run_layer(w, dev)
    shape = dsa.workload_shape(w)
    rg = _rg(w, dev)
    rows = [2048, 5000, 17000, 32767]
    for r in rows:
        idx_ref, out_ref, _, _ = PT.oracle_row(w, r)
        np.testing.assert_array_equal(idx[r].cpu().numpy(), idx_ref)
        assert PT.close_report(PT.bf16_tensor_to_f64(out[r]), out_ref)["ok"]
        bad = idx[r: r + 1].clone()
        sel = set(bad[0].cpu().numpy().tolist())
        bad[0, 0] = next(j for j in range(w.row_position(r) + 1) if j not in sel)
        one = torch.zeros_like(out)
        dsa.dsa_sparse_attn_gated(shape, rg, dev["q"], dev["k"], dev["v"], bad, w.top_k, r, 1,
                                  dev["gate"], one)
        nogate = torch.zeros_like(out)
        dsa.dsa_sparse_attn_gated(shape, rg, dev["q"], dev["k"], dev["v"], idx[r: r + 1],
                                  w.top_k, r, 1, None, nogate)
        torch.cuda.synchronize()
        assert not PT.close_report(PT.bf16_tensor_to_f64(one[r]), out_ref)["ok"], r
        assert not PT.close_report(PT.bf16_tensor_to_f64(nogate[r]), out_ref)["ok"], r
    del dev, idx, out
    torch.cuda.empty_cache()


def test_mixed_batch_runs_prefill_chunks_fused_and_decode_rows_materialised():
    """A batch of prefill chunks and single decode queries (the serving layout), with host
    offsets: the chunks' rows take the fused indexer -> Top-K, the decode rows score tiles of
    16 queries, one attention launch covers all; every row matches the oracle."""
    q_lens = [300, 1, 1, 640, 1, 1, 1, 200] + [1] * 9
    kv_lens = [2500, 3000, 5, 4000, 129, 6000, 4097, 900] + [700 + 311 * i for i in range(9)]
    w = _workload(q_lens, kv_lens, K=256)
    host = S.make_host_inputs(w)
    dev = _dev(host)
    dsa.dsa_fused_rows(reset=True)
    idx, out = _run_layer(w, dev)
    fused = dsa.dsa_fused_rows(reset=True)
    assert fused == sum(q for q in q_lens if q >= 128)
    rows = list(range(w.total_q))
    idx_ref, out_ref, _ = O.Oracle.for_workload(w, host).layer_rows(rows)
    np.testing.assert_array_equal(idx.cpu().numpy(), idx_ref)
    PT.assert_close(PT.bf16_tensor_to_f64(out), out_ref, "mixed batch")
