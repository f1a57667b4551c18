"""GPU parity of the fused indexer -> Top-K entry (dsa_index_topk).

On dyadic-grid inputs every score is exact in fp32, so the fused path must give, bit for
bit, the index rows of dsa_index_scores + dsa_topk (which are pinned to the oracle in
test_gpu_parity.py); sampled rows are also checked against the oracle directly.  The
cases cover rows shorter than the candidate slots (every score kept), long rows (sampled
threshold; beyond 2048 samples a CTA per row), ragged batches with history, e4m3 inputs, per-row weights, K = 1 and a K
near the slot limit, rows whose threshold misses (all scores tied: the CUDA-core
fallback), passes forced by a small workspace, and the layer taking the fused path.
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


def _workload(q_lens, kv_lens, K=64, Hi=4, dtype="bf16", seed=0):
    return S.Workload("custom", list(q_lens), list(kv_lens), top_k=K, n_q_heads=8,
                      n_kv_heads=8, n_idx_heads=Hi, idx_dtype=dtype, qkv_scale=S.INV_SQRT_128,
                      gate=True, seed=seed)


def _rg(w, dev):
    return dsa.ragged(dev["q_offsets"], dev["kv_offsets"], w.q_lens, w.kv_lens)


def _materialised(w, shape, rg, dev, q0, qn):
    ld = (max(w.kv_lens) + 3) // 4 * 4
    scores = torch.empty((qn, ld), device="cuda")
    dsa.dsa_index_scores(shape, rg, dev["q_idx"], dev["k_idx"], dev["w"], q0, qn, scores, ld)
    idx = torch.full((qn, w.top_k), -7, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(qn, dtype=torch.int32, device="cuda")
    dsa.dsa_topk(shape, rg, scores, ld, q0, qn, idx, w.top_k, cnt)
    return idx.cpu().numpy(), cnt.cpu().numpy()


def _fused(w, shape, rg, dev, q0, qn, ws_bytes=None, ld_idx=None):
    mn, rec = dsa.dsa_index_topk_workspace_size(shape, rg, qn)
    nbytes = rec if ws_bytes is None else max(mn, ws_bytes)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    ws.fill_(0xFF)  # nothing in the workspace has to start out initialised
    ld_idx = ld_idx or w.top_k
    idx = torch.full((qn, ld_idx), -7, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(qn, dtype=torch.int32, device="cuda")
    dsa.dsa_index_topk(shape, rg, dev["q_idx"], dev["k_idx"], dev["w"], q0, qn, idx, ld_idx, cnt,
                       ws)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), cnt.cpu().numpy()


def _check_oracle_rows(w, host, idx, q0, rows):
    orc = O.Oracle.for_workload(w, host)
    for r in rows:
        ref = O.topk_row(orc.index_scores_row(q0 + r), w.top_k)
        np.testing.assert_array_equal(idx[r, : w.top_k], ref, err_msg=f"row {q0 + r}")


FUSED_CASES = {
    # one long sequence: rows below the slot count keep every score, longer rows go
    # through the sampled threshold
    "prefill_t8192_k512": dict(q_lens=[8192], kv_lens=[8192], K=512),
    # ragged with history (queries are the last rows of their sequence), rows of every
    # length class, a tile straddling sequences
    "ragged_history": dict(q_lens=[700, 1, 2600, 64, 3], kv_lens=[3000, 5000, 2600, 9000, 3],
                           K=256),
    "fp8": dict(q_lens=[3000], kv_lens=[6000], dtype="fp8", K=300),
    "k1": dict(q_lens=[1500], kv_lens=[1500], K=1),
    "k4096": dict(q_lens=[600], kv_lens=[20000], K=4096),
    "one_head": dict(q_lens=[2000], kv_lens=[5000], Hi=1, K=200),
    # a full head pair and a pair of one head (each head's accumulator signalled on its own)
    "three_heads": dict(q_lens=[1800, 700], kv_lens=[6000, 700], Hi=3, K=256),
    # rows of more than 2048 samples (n > 32768): their thresholds come from the one-CTA-per-row
    # kernel
    "long_rows": dict(q_lens=[96], kv_lens=[40000], K=512),
}


@pytest.mark.parametrize("case", sorted(FUSED_CASES))
def test_index_topk_matches_materialised(case):
    w = _workload(**FUSED_CASES[case])
    host = S.make_host_inputs(w)
    dev = _dev(host)
    shape = dsa.workload_shape(w)
    rg = _rg(w, dev)
    ref_idx, ref_cnt = _materialised(w, shape, rg, dev, 0, w.total_q)
    idx, cnt = _fused(w, shape, rg, dev, 0, w.total_q)
    np.testing.assert_array_equal(idx, ref_idx)
    np.testing.assert_array_equal(cnt, ref_cnt)
    rows = PT.sample_rows(w, 12, seed=3)
    _check_oracle_rows(w, host, idx, 0, rows)


def test_index_topk_row_window_row_weights_and_wide_idx():
    w = _workload([2500, 1800], [4000, 1800], K=128)
    host = S.make_host_inputs(w)
    rng = np.random.default_rng(5)
    host["w"] = (rng.integers(1, 5, size=(w.total_q, 4)) / 4.0).astype(np.float32)
    dev = _dev(host)
    shape = dsa.workload_shape(w)
    shape.w_row_stride = 4
    rg = _rg(w, dev)
    q0, qn = 900, 3000
    ref_idx, ref_cnt = _materialised(w, shape, rg, dev, q0, qn)
    idx, cnt = _fused(w, shape, rg, dev, q0, qn, ld_idx=w.top_k + 5)
    np.testing.assert_array_equal(idx[:, : w.top_k], ref_idx)
    assert (idx[:, w.top_k:] == -7).all()  # columns past K are not written
    np.testing.assert_array_equal(cnt, ref_cnt)


@pytest.mark.parametrize("weights", [(1.0, -0.5, 0.25, -1.0), (-0.25, -1.0, -0.5, -0.125)])
def test_index_topk_negative_and_mixed_sign_weights(weights):
    """Head weights of mixed sign, or all negative, give negative scores and thresholds, and
    (all negative) many rows whose best scores are exact zeros: the selection's key range,
    its clamping and the marking pass's float compares must still reproduce the materialised
    path bit for bit."""
    w = _workload([5000], [7000], K=256)
    host = S.make_host_inputs(w)
    host["w"] = np.array(weights, dtype=np.float32)
    dev = _dev(host)
    shape = dsa.workload_shape(w)
    rg = _rg(w, dev)
    ref_idx, ref_cnt = _materialised(w, shape, rg, dev, 0, w.total_q)
    idx, cnt = _fused(w, shape, rg, dev, 0, w.total_q)
    np.testing.assert_array_equal(idx, ref_idx)
    np.testing.assert_array_equal(cnt, ref_cnt)
    _check_oracle_rows(w, host, idx, 0, PT.sample_rows(w, 12, seed=4))


def test_index_topk_threshold_misses_fall_back():
    """Rows whose q_idx is zero have all scores tied at 0: every score passes the sampled
    threshold, the candidates overflow their slots and the row is recomputed on CUDA cores
    and selected exactly (the K lowest positions).  Other rows take the normal path."""
    w = _workload([6000], [6000], K=300)
    host = S.make_host_inputs(w)
    zero_rows = np.arange(0, 6000, 3)
    host["q_idx"][zero_rows] = 0
    dev = _dev(host)
    shape = dsa.workload_shape(w)
    rg = _rg(w, dev)
    ref_idx, ref_cnt = _materialised(w, shape, rg, dev, 0, w.total_q)
    idx, cnt = _fused(w, shape, rg, dev, 0, w.total_q)
    np.testing.assert_array_equal(idx, ref_idx)
    np.testing.assert_array_equal(cnt, ref_cnt)
    for r in zero_rows[zero_rows >= w.top_k][:50]:
        np.testing.assert_array_equal(idx[r], np.arange(w.top_k))


def test_index_topk_fallback_e4m3_and_row_weights():
    """Rows whose threshold comes out too high: their q_idx is all 0.5 and so is the key
    at every 16th position, so every sample holds the row's maximum score and fewer than
    K scores reach the threshold.  The CUDA-core recompute must then decode e4m3 and apply
    per-row weights exactly as the indexer does; the other rows take the normal path."""
    w = _workload([4000], [4000], dtype="fp8", K=300)
    host = S.make_host_inputs(w)
    rng = np.random.default_rng(11)
    host["w"] = (rng.integers(1, 5, size=(w.total_q, 4)) / 4.0).astype(np.float32)
    half_e4m3 = 0x30  # exponent field 6 (2^-1), mantissa 0
    strong_rows = np.arange(1, 4000, 2)
    host["q_idx"][strong_rows] = half_e4m3
    host["k_idx"][0::16] = half_e4m3
    dev = _dev(host)
    shape = dsa.workload_shape(w)
    shape.w_row_stride = 4
    rg = _rg(w, dev)
    ref_idx, ref_cnt = _materialised(w, shape, rg, dev, 0, w.total_q)
    idx, cnt = _fused(w, shape, rg, dev, 0, w.total_q)
    np.testing.assert_array_equal(idx, ref_idx)
    np.testing.assert_array_equal(cnt, ref_cnt)
    # the strong keys are selected by every strong row (they hold its maximum score)
    for r in strong_rows[strong_rows > 2000][:20]:
        assert set(range(0, r + 1, 16)) <= set(idx[r].tolist())


def test_index_topk_passes_from_a_small_workspace():
    w = _workload([5000, 3000], [5000, 7000], K=256)
    host = S.make_host_inputs(w)
    dev = _dev(host)
    shape = dsa.workload_shape(w)
    rg = _rg(w, dev)
    mn, _ = dsa.dsa_index_topk_workspace_size(shape, rg, w.total_q)
    per_row = (dsa.dsa_index_topk_workspace_size(shape, rg, 2)[1] -
               dsa.dsa_index_topk_workspace_size(shape, rg, 1)[1])
    ref_idx, ref_cnt = _materialised(w, shape, rg, dev, 0, w.total_q)
    for extra_rows in (0, 37, 999):
        idx, cnt = _fused(w, shape, rg, dev, 0, w.total_q, ws_bytes=mn + extra_rows * per_row)
        np.testing.assert_array_equal(idx, ref_idx, err_msg=f"extra rows {extra_rows}")
        np.testing.assert_array_equal(cnt, ref_cnt)


def test_index_topk_needles_scaled():
    """The planted-needle workload (scaled down): identical index rows, and every needle
    is selected by every row of the designated block."""
    w = S.workload("prefill_t131072_needles", scale_down=8)
    host = S.make_host_inputs(w)
    dev = _dev(host)
    shape = dsa.workload_shape(w)
    rg = _rg(w, dev)
    ref_idx, _ = _materialised(w, shape, rg, dev, 0, w.total_q)
    idx, _ = _fused(w, shape, rg, dev, 0, w.total_q)
    np.testing.assert_array_equal(idx, ref_idx)
    for r in w.needle_rows:
        assert set(w.needle_pos) <= set(idx[r].tolist()), f"row {r}"


def test_prefill_layer_takes_the_fused_path():
    """A prefill whose score matrix exceeds 256 MiB runs steps 1-2 fused: its index rows
    equal the materialised ones and the output equals attention over them."""
    w = S.Workload("custom", [12288], [12288], top_k=512, n_q_heads=32, n_kv_heads=4,
                   qkv_scale=S.INV_SQRT_128, gate=True)
    host = S.make_host_inputs(w)
    dev = _dev(host)
    shape = dsa.workload_shape(w)
    rg = _rg(w, dev)
    _, rec = dsa.dsa_workspace_size(shape, rg)
    ws = torch.empty(rec, dtype=torch.uint8, device="cuda")
    out = torch.empty((w.total_q, w.n_q_heads, 128), dtype=torch.bfloat16, device="cuda")
    idx_out = torch.empty((w.total_q, w.top_k), dtype=torch.int32, device="cuda")
    n0 = dsa.dsa_launch_count()
    dsa.dsa_prefill(shape, rg, dev["q_idx"], dev["k_idx"], dev["w"], dev["q"], dev["k"], dev["v"],
                    dev["gate"], out, idx_out=idx_out, workspace=ws)
    torch.cuda.synchronize()
    # the fused path: sampled keys, samples, thresholds, candidates, selection, fallback,
    # attention
    assert dsa.dsa_launch_count() - n0 == 7
    ref_idx, _ = _materialised(w, shape, rg, dev, 0, w.total_q)
    np.testing.assert_array_equal(idx_out.cpu().numpy(), ref_idx)
    out2 = torch.empty_like(out)
    ref_t = torch.from_numpy(ref_idx).cuda()
    dsa.dsa_sparse_attn_gated(shape, rg, dev["q"], dev["k"], dev["v"], ref_t, w.top_k, 0,
                              w.total_q, dev["gate"], out2)
    torch.cuda.synchronize()
    assert torch.equal(out, out2)


# ----------------------------------------------------------------------------- block granularity

BLOCK_CASES = {
    "b32_k16": dict(q_lens=[1500], kv_lens=[1500], K=16, B=32),
    "b64_ragged": dict(q_lens=[700, 1, 300, 5], kv_lens=[3000, 4097, 300, 70], K=12, B=64),
    "b128_k40": dict(q_lens=[2000], kv_lens=[6000], K=40, B=128),
    "b32_fp8": dict(q_lens=[900], kv_lens=[2000], K=20, B=32, dtype="fp8"),
}


@pytest.mark.parametrize("case", sorted(BLOCK_CASES))
def test_index_topk_blocks_matches_oracle(case):
    cfg = dict(BLOCK_CASES[case])
    B = cfg.pop("B")
    w = _workload(**cfg)
    host = S.make_host_inputs(w)
    dev = _dev(host)
    shape = dsa.workload_shape(w)
    rg = _rg(w, dev)
    Kb = w.top_k
    ld = Kb * B + 3
    mn, rec = dsa.dsa_index_topk_blocks_workspace_size(shape, rg, B, w.total_q)
    idx = torch.full((w.total_q, ld), -7, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(w.total_q, dtype=torch.int32, device="cuda")
    for ws_bytes in (rec, mn + 5 * (rec - mn) // max(1, w.total_q)):  # one pass, then many
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
        idx.fill_(-7)
        dsa.dsa_index_topk_blocks(shape, rg, dev["q_idx"], dev["k_idx"], dev["w"], B, 0, w.total_q,
                                  idx, ld, cnt, ws)
        torch.cuda.synchronize()
        got = idx.cpu().numpy()
        orc = O.Oracle.for_workload(w, host)
        for r in PT.sample_rows(w, 24, seed=9):
            ref = O.block_topk_row(orc.index_scores_row(r), B, Kb)
            np.testing.assert_array_equal(got[r, : Kb * B], ref, err_msg=f"{case} row {r}")
            assert int(cnt[r]) == int((ref >= 0).sum())
        assert (got[:, Kb * B:] == -7).all()


def test_block_selection_feeds_attention():
    """Attention over a block selection (top_k = Kb * B positions) matches the oracle."""
    B, Kb = 64, 6
    w = _workload([300], [2000], K=Kb)
    host = S.make_host_inputs(w)
    dev = _dev(host)
    shape = dsa.workload_shape(w)
    rg = _rg(w, dev)
    _, rec = dsa.dsa_index_topk_blocks_workspace_size(shape, rg, B, w.total_q)
    ws = torch.empty(rec, dtype=torch.uint8, device="cuda")
    idx = torch.empty((w.total_q, Kb * B), dtype=torch.int32, device="cuda")
    dsa.dsa_index_topk_blocks(shape, rg, dev["q_idx"], dev["k_idx"], dev["w"], B, 0, w.total_q,
                              idx, Kb * B, None, ws)
    shape_a = dsa.workload_shape(w)
    shape_a.top_k = Kb * B
    out = torch.zeros((w.total_q, w.n_q_heads, 128), dtype=torch.bfloat16, device="cuda")
    dsa.dsa_sparse_attn_gated(shape_a, rg, dev["q"], dev["k"], dev["v"], idx, Kb * B, 0,
                              w.total_q, dev["gate"], out)
    torch.cuda.synchronize()
    got_idx = idx.cpu().numpy()
    w_a = _workload([300], [2000], K=Kb * B)
    orc = O.Oracle.for_workload(w_a, host)
    rows = list(range(0, 300, 37))
    ref = np.stack([orc.sparse_attn_row(r, got_idx[r])[0] for r in rows])
    PT.assert_close(PT.bf16_tensor_to_f64(out)[rows], ref, "block attention")
