"""GPU parity with non-default numeric scales: the indexer's dequantisation scales and the
attention's logit scale.

The indexer may run at lower precision ([GSA] "4. The Role of Gating and Engineering
Considerations"): its inputs then carry dequantisation scales, and the score is
sum_h w_h * max(0, c * q_h . k_h) with c = idx_scale_q * idx_scale_k.  The library folds c
into the shared head weights (stride 0) or applies it to each dot (per-row weights); the
oracle applies each scale to each element.
 - Power-of-two scales keep every score exact in fp32 on the dyadic grid, so scores and
   index rows must match the oracle bit for bit (bf16 and e4m3, both weight layouts, the
   materialised and the fused Top-K, the whole layer).
 - A scale that is not a power of two (0.3 * 1.7) rounds: scores must agree to a few fp32
   ulps of the score, and the selected set must be a valid Top-K of the oracle's fp64
   scores up to that rounding.
 - attn_scale = 0.2 replaces 1/sqrt(d) in the softmax ([HSA] step 3, [SAE] section 5 give
   1/sqrt(dim); the ABI lets a caller override it): outputs within the parity tolerance,
   and the default scale must fail against the 0.2 reference.
Each of these fails if either side drops, squares or misplaces a scale.
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
            out[k] = torch.from_numpy(np.ascontiguousarray(v)).cuda()
    return out


def _wl(q_lens, kv_lens, K=64, Hq=32, Hkv=4, dtype="bf16", scale=S.INV_SQRT_128, seed=0):
    return S.Workload("custom", list(q_lens), list(kv_lens), top_k=K, n_q_heads=Hq,
                      n_kv_heads=Hkv, idx_dtype=dtype, qkv_scale=scale, gate=True, seed=seed)


def _shape(w, sq=1.0, sk=1.0, attn_scale=0.0, stride=0):
    s = dsa.workload_shape(w)
    s.idx_scale_q, s.idx_scale_k, s.attn_scale, s.w_row_stride = sq, sk, attn_scale, stride
    return s


def _oracle(w, host, sq=1.0, sk=1.0, attn_scale=0.0, stride=0):
    return O.Oracle(host, top_k=w.top_k, n_idx_heads=w.n_idx_heads, idx_dim=w.idx_dim,
                    n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads, head_dim=w.head_dim,
                    idx_fp8=(w.idx_dtype == "fp8"), idx_scale_q=sq, idx_scale_k=sk,
                    attn_scale=attn_scale, w_row_stride=stride)


def _row_weights(host, w, stride):
    rng = np.random.default_rng(9)
    wt = np.zeros((w.total_q, stride), np.float32)
    wt[:, : w.n_idx_heads] = rng.integers(1, 9, size=(w.total_q, w.n_idx_heads)) / 8.0
    host["w"] = wt


def _scores(w, dev, shape):
    ld = (max(w.kv_lens) + 3) // 4 * 4 + 4
    scores = torch.full((w.total_q, ld), float("nan"), device="cuda")
    rg = dsa.ragged(dev["q_offsets"], dev["kv_offsets"], w.q_lens, w.kv_lens)
    dsa.dsa_index_scores(shape, rg, dev["q_idx"], dev["k_idx"], dev["w"], 0, w.total_q, scores, ld)
    return scores.cpu().numpy()


POW2 = [(0.5, 4.0), (0.25, 0.5)]


@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
@pytest.mark.parametrize("stride", [0, 5])
@pytest.mark.parametrize("sq,sk", POW2)
def test_index_scores_power_of_two_scales_bitexact(dtype, stride, sq, sk):
    w = _wl([300, 1, 129], [300, 700, 1000], dtype=dtype)
    host = S.make_host_inputs(w)
    if stride:
        _row_weights(host, w, stride)
    got = _scores(w, _dev(host), _shape(w, sq, sk, stride=stride))
    orc = _oracle(w, host, sq, sk, stride=stride)
    unscaled = _oracle(w, host, stride=stride)
    for r in range(w.total_q):
        ref = orc.index_scores_row(r)
        np.testing.assert_array_equal(got[r, : len(ref)], ref.astype(np.float32), err_msg=f"row {r}")
        assert np.isnan(got[r, len(ref):]).all()
    # the scale was applied (the unscaled scores differ by the factor sq * sk != 1)
    r = w.total_q - 1
    ref1 = unscaled.index_scores_row(r)
    assert np.any(ref1 > 0)
    np.testing.assert_array_equal(got[r, : len(ref1)], (ref1 * (sq * sk)).astype(np.float32))


@pytest.mark.parametrize("stride", [0, 4])
def test_index_scores_non_dyadic_scale_within_rounding(stride):
    """c = 0.3 * 1.7 rounds in fp32: every term w_h max(0, c x_h) is >= 0, so the score's
    own magnitude bounds the rounding of its few products and fused adds (5 roundings of
    2^-24 relative each at most; 1e-6 relative is checked).  Where the exact score is 0 the
    oracle's fp64 product of scaled operands leaves a residue of ~1e-17: 1e-12 absolute."""
    w = _wl([200, 77], [600, 900])
    host = S.make_host_inputs(w)
    if stride:
        _row_weights(host, w, stride)
    got = _scores(w, _dev(host), _shape(w, 0.3, 1.7, stride=stride))
    orc = _oracle(w, host, 0.3, 1.7, stride=stride)
    worst = 0.0
    for r in range(w.total_q):
        ref = orc.index_scores_row(r)
        err = np.abs(got[r, : len(ref)].astype(np.float64) - ref)
        bad = err > 1e-6 * ref + 1e-12
        assert not np.any(bad), f"row {r}: {err[bad][:4]} at ref {ref[bad][:4]}"
        big = ref > 1e-6
        worst = max(worst, float(np.max(err[big] / ref[big], initial=0.0)))
    # a squared or dropped scale would be off by a factor 0.51 or 1/0.51
    assert worst < 1e-6


def _valid_selection(s, K, idx, rtol):
    """idx holds min(K, n) distinct ascending positions; every selected score is >= every
    unselected one up to rtol of the K-th largest score (ties at fp32 rounding may go
    either way)."""
    n = len(s)
    take = min(K, n)
    sel = idx[:take]
    assert np.all(idx[take:] == -1)
    assert len(np.unique(sel)) == take and np.all(np.diff(sel) > 0)
    assert sel.min() >= 0 and sel.max() < n
    if take == n:
        return
    kth = np.sort(s)[::-1][K - 1]
    mask = np.zeros(n, bool)
    mask[sel] = True
    tol = rtol * abs(kth) + 1e-30
    assert s[mask].min() >= kth - tol
    assert s[~mask].max() <= kth + tol


def _index_topk(w, dev, shape):
    rg = dsa.ragged(dev["q_offsets"], dev["kv_offsets"], w.q_lens, w.kv_lens)
    _, rec = dsa.dsa_index_topk_workspace_size(shape, rg, w.total_q)
    ws = torch.empty(rec, dtype=torch.uint8, device="cuda")
    idx = torch.full((w.total_q, w.top_k), -7, dtype=torch.int32, device="cuda")
    dsa.dsa_index_topk(shape, rg, dev["q_idx"], dev["k_idx"], dev["w"], 0, w.total_q, idx,
                       w.top_k, None, ws)
    return idx.cpu().numpy()


@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
@pytest.mark.parametrize("stride", [0, 4])
def test_index_topk_power_of_two_scales_bitexact(dtype, stride):
    """The fused indexer -> Top-K (sampled threshold, candidates, exact selection) with
    power-of-two scales: index rows equal the oracle's selection bit for bit."""
    w = _wl([2500], [4000], K=300, dtype=dtype)
    host = S.make_host_inputs(w)
    if stride:
        _row_weights(host, w, stride)
    got = _index_topk(w, _dev(host), _shape(w, 0.5, 4.0, stride=stride))
    orc = _oracle(w, host, 0.5, 4.0, stride=stride)
    for r in list(range(0, w.total_q, 23)) + [w.total_q - 1]:
        ref = O.topk_row(orc.index_scores_row(r), w.top_k)
        np.testing.assert_array_equal(got[r], ref, err_msg=f"row {r}")


def test_topk_non_dyadic_scale_is_a_valid_selection():
    """0.3 * 1.7: the materialised and the fused Top-K each select a valid Top-K of the
    oracle's fp64 scores up to fp32 rounding, and both paths agree with each other on the
    GPU's own fp32 scores."""
    w = _wl([2500], [4000], K=300)
    host = S.make_host_inputs(w)
    dev = _dev(host)
    shape = _shape(w, 0.3, 1.7)
    fused = _index_topk(w, dev, shape)
    rg = dsa.ragged(dev["q_offsets"], dev["kv_offsets"], w.q_lens, w.kv_lens)
    ld = (max(w.kv_lens) + 3) // 4 * 4
    sc = torch.empty((w.total_q, ld), device="cuda")
    dsa.dsa_index_scores(shape, rg, dev["q_idx"], dev["k_idx"], dev["w"], 0, w.total_q, sc, ld)
    mat = torch.full((w.total_q, w.top_k), -7, dtype=torch.int32, device="cuda")
    dsa.dsa_topk(shape, rg, sc, ld, 0, w.total_q, mat, w.top_k)
    mat = mat.cpu().numpy()
    scores32 = sc.cpu().numpy()
    orc = _oracle(w, host, 0.3, 1.7)
    for r in list(range(0, w.total_q, 37)) + [w.total_q - 1]:
        s = orc.index_scores_row(r)
        _valid_selection(s, w.top_k, mat[r], 1e-6)
        _valid_selection(s, w.top_k, fused[r], 1e-6)
        # on the GPU's own fp32 scores the selection is exact
        np.testing.assert_array_equal(mat[r], O.topk_row(scores32[r, : len(s)].astype(np.float64),
                                                         w.top_k))
    np.testing.assert_array_equal(fused, mat)


@pytest.mark.parametrize("decode", [False, True])
def test_layer_with_scales_matches_oracle(decode):
    """Whole layer with idx scales (0.5, 4) and attn_scale 0.2 against the oracle with the
    same parameters.  q and k ~ N(0,1) so that the logit scale shapes the softmax (logits
    of standard deviation ~2.3); v and the gate keep the configurations' distributions."""
    if decode:
        w = _wl([1] * 6, [1, 300, 129, 2048, 3000, 777], K=256, Hq=16, Hkv=2)
    else:
        w = _wl([400, 90], [400, 1000], K=128, Hq=16, Hkv=2)
    host = S.make_host_inputs(w)
    host["q"] = S.host_bf16(host["q"].size, S.NORMAL, 7, S.T_Q, 0, 1.0).reshape(host["q"].shape)
    host["k"] = S.host_bf16(host["k"].size, S.NORMAL, 7, S.T_K, 0, 1.0).reshape(host["k"].shape)
    dev = _dev(host)
    shape = _shape(w, 0.5, 4.0, attn_scale=0.2)
    rg = dsa.ragged(dev["q_offsets"], dev["kv_offsets"], w.q_lens, w.kv_lens)
    _, rec = dsa.dsa_workspace_size(shape, rg, decode)
    ws = torch.empty(rec, dtype=torch.uint8, device="cuda")
    out = torch.zeros((w.total_q, w.n_q_heads, 128), dtype=torch.bfloat16, device="cuda")
    idx = torch.full((w.total_q, w.top_k), -7, dtype=torch.int32, device="cuda")
    fn = dsa.dsa_decode if decode else dsa.dsa_prefill
    fn(shape, rg, dev["q_idx"], dev["k_idx"], dev["w"], dev["q"], dev["k"], dev["v"], dev["gate"],
       out, idx_out=idx, workspace=ws)
    torch.cuda.synchronize()
    rows = list(range(w.total_q))
    idx_ref, out_ref, _ = _oracle(w, host, 0.5, 4.0, attn_scale=0.2).layer_rows(rows)
    np.testing.assert_array_equal(idx.cpu().numpy(), idx_ref)
    got = PT.bf16_tensor_to_f64(out)
    PT.assert_close(got, out_ref, "scaled layer")
    # the default logit scale gives a different layer: it must fail the same check
    _, out_default, _ = _oracle(w, host, 0.5, 4.0).layer_rows(rows)
    assert not PT.close_report(got, out_default)["ok"]


def test_attention_scale_override_lse():
    """dsa_sparse_attn_gated with attn_scale 0.2: outputs and the LSE (natural log of the
    0.2-scaled logits' exponential sum) against the oracle."""
    w = _wl([40, 1, 90], [300, 50, 90], K=96, scale=1.0)
    host = S.make_host_inputs(w)
    dev = _dev(host)
    orc = _oracle(w, host, attn_scale=0.2)
    idx_ref, out_ref, lse_ref = orc.layer_rows(range(w.total_q))
    out = torch.zeros((w.total_q, w.n_q_heads, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((w.total_q, w.n_q_heads), device="cuda")
    rg = dsa.ragged(dev["q_offsets"], dev["kv_offsets"], w.q_lens, w.kv_lens)
    dsa.dsa_sparse_attn_gated(_shape(w, attn_scale=0.2), rg, dev["q"], dev["k"], dev["v"],
                              torch.from_numpy(idx_ref).cuda(), w.top_k, 0, w.total_q,
                              dev["gate"], out, lse)
    torch.cuda.synchronize()
    PT.assert_close(PT.bf16_tensor_to_f64(out), out_ref, "attn_scale 0.2")
    np.testing.assert_allclose(lse.cpu().numpy(), lse_ref, rtol=1e-5, atol=1e-5)
