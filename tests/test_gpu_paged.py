"""GPU checks of the paged cache layout (dsa_ragged.block_table).

The same problem is run twice: with contiguous cache rows, and with every sequence's
positions spread over pages in a random physical order (unused pages hold junk).  Paging
only changes where rows are read, so every output (index rows, attention output, LSE)
must be bit-identical to the contiguous run; the paged results are also compared directly
with the oracle run on the logical (contiguous) sequences: index rows bit for bit, outputs
within the parity tolerance.
Covered: the materialised layer (prefill and decode), the fused indexer -> Top-K path
(sampled keys, candidate indexer and the CUDA-core recompute of rows whose threshold
missed), and two sequences sharing the pages of a common prefix.
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


def _to_dev(x):
    if x.dtype == np.uint16:
        return torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def _paged(w, host, page_size, seed=0, extra_pages=3):
    """Physical cache arrays and block table holding host's cache rows in shuffled pages."""
    rng = np.random.default_rng(seed)
    n_pages = [(L + page_size - 1) // page_size for L in w.kv_lens]
    total = sum(n_pages) + extra_pages
    perm = rng.permutation(total)
    max_pages = max(1, max(n_pages))
    table = np.zeros((w.batch, max_pages), dtype=np.int32)
    phys = {}
    for name in ("k_idx", "k", "v"):
        arr = host[name]
        junk = rng.integers(0, 2 ** 15, size=(total * page_size,) + arr.shape[1:])
        phys[name] = junk.astype(arr.dtype) & (0x3F7F if arr.dtype == np.uint16 else 0x3F)
    nxt = 0
    for b, L in enumerate(w.kv_lens):
        ko = int(w.kv_offsets[b])
        for pg in range(n_pages[b]):
            page = int(perm[nxt])
            nxt += 1
            table[b, pg] = page
            n = min(page_size, L - pg * page_size)
            for name in ("k_idx", "k", "v"):
                phys[name][page * page_size: page * page_size + n] = \
                    host[name][ko + pg * page_size: ko + pg * page_size + n]
    return phys, table, total * page_size


def _layer(fn, w, dev, cache, rg, ws_bytes=None):
    shape = dsa.workload_shape(w)
    decode = fn is dsa.dsa_decode
    _, rec = dsa.dsa_workspace_size(shape, rg, decode)
    ws = torch.empty(ws_bytes or rec, dtype=torch.uint8, device="cuda")
    out = torch.empty((w.total_q, w.n_q_heads, 128), dtype=torch.bfloat16, device="cuda")
    idx = torch.full((w.total_q, w.top_k), -7, dtype=torch.int32, device="cuda")
    fn(shape, rg, dev["q_idx"], cache["k_idx"], dev["w"], dev["q"], cache["k"], cache["v"],
       dev.get("gate"), out, idx_out=idx, workspace=ws)
    torch.cuda.synchronize()
    return out, idx


def _both(w, page_size, fn=None, seed=0):
    host = S.make_host_inputs(w)
    dev = {k: _to_dev(v) for k, v in host.items() if k not in ("q_offsets", "kv_offsets")}
    qo = torch.from_numpy(w.q_offsets.astype(np.int32)).cuda()
    ko = torch.from_numpy(w.kv_offsets.astype(np.int32)).cuda()
    rg = dsa.ragged(qo, ko, w.q_lens, w.kv_lens)
    fn = fn or dsa.dsa_prefill
    out_c, idx_c = _layer(fn, w, dev, dev, rg)
    phys, table, rows = _paged(w, host, page_size, seed)
    cache = {k: _to_dev(v) for k, v in phys.items()}
    bt = _to_dev(table)  # the descriptor holds only its address: keep the tensor alive
    rgp = dsa.ragged(qo, ko, w.q_lens, w.kv_lens, block_table=bt, page_size=page_size,
                     cache_rows=rows)
    out_p, idx_p = _layer(fn, w, dev, cache, rgp)
    return (out_c, idx_c), (out_p, idx_p), (host, dev, rg, rgp, cache, bt)


def _wl(q_lens, kv_lens, K, Hq=32, Hkv=4):
    return S.Workload("custom", list(q_lens), list(kv_lens), top_k=K, n_q_heads=Hq,
                      n_kv_heads=Hkv, qkv_scale=S.INV_SQRT_128, gate=True)


@pytest.mark.parametrize("page_size", [128, 512])
def test_paged_prefill_materialised_equals_contiguous(page_size):
    w = _wl([300, 1, 700], [900, 513, 700], K=64)
    (oc, ic), (op, ip), _ = _both(w, page_size)
    assert torch.equal(ic, ip)
    assert torch.equal(oc, op)


def test_paged_decode_equals_contiguous():
    w = _wl([1] * 12, [1, 127, 128, 129, 1000, 4097, 300, 2500, 640, 768, 5000, 33], K=256)
    (oc, ic), (op, ip), _ = _both(w, 256, fn=dsa.dsa_decode)
    assert torch.equal(ic, ip)
    assert torch.equal(oc, op)


def test_paged_fused_prefill_equals_contiguous():
    """Long enough for dsa_prefill to take the fused indexer -> Top-K path."""
    w = _wl([12288], [12288], K=512)
    (oc, ic), (op, ip), _ = _both(w, 256, seed=3)
    assert torch.equal(ic, ip)
    assert torch.equal(oc, op)


def test_paged_index_topk_with_recomputed_rows():
    """Rows with all-tied scores miss their threshold and are recomputed on CUDA cores,
    reading the paged k_idx."""
    w = _wl([3000], [5000], K=300)
    host = S.make_host_inputs(w)
    host["q_idx"][::3] = 0
    dev = {k: _to_dev(v) for k, v in host.items() if k not in ("q_offsets", "kv_offsets")}
    qo = torch.from_numpy(w.q_offsets.astype(np.int32)).cuda()
    ko = torch.from_numpy(w.kv_offsets.astype(np.int32)).cuda()
    shape = dsa.workload_shape(w)

    def run(rg, k_idx):
        _, rec = dsa.dsa_index_topk_workspace_size(shape, rg, w.total_q)
        ws = torch.empty(rec, dtype=torch.uint8, device="cuda")
        idx = torch.full((w.total_q, w.top_k), -7, dtype=torch.int32, device="cuda")
        dsa.dsa_index_topk(shape, rg, dev["q_idx"], k_idx, dev["w"], 0, w.total_q, idx, w.top_k,
                           None, ws)
        torch.cuda.synchronize()
        return idx

    idx_c = run(dsa.ragged(qo, ko, w.q_lens, w.kv_lens), dev["k_idx"])
    phys, table, rows = _paged(w, host, 128, seed=5)
    bt = _to_dev(table)
    rgp = dsa.ragged(qo, ko, w.q_lens, w.kv_lens, block_table=bt, page_size=128,
                     cache_rows=rows)
    idx_p = run(rgp, _to_dev(phys["k_idx"]))
    assert torch.equal(idx_c, idx_p)
    assert (idx_p[::3][: -1, :10].cpu().numpy() == np.arange(10)).all()
    # and against the oracle's selection on the logical sequence (recomputed and regular rows)
    orc = O.Oracle.for_workload(w, host)
    got = idx_p.cpu().numpy()
    for r in list(range(0, w.total_q, 41)) + [w.total_q - 1]:
        np.testing.assert_array_equal(got[r], O.topk_row(orc.index_scores_row(r), w.top_k),
                                      err_msg=f"row {r}")


def test_shared_prefix_pages():
    """Two sequences whose first 512 positions are the same cache rows: sharing those pages
    gives the results of two contiguous copies."""
    ps = 128
    w = _wl([200, 300], [1000, 900], K=128)
    host = S.make_host_inputs(w)
    ko0, ko1 = int(w.kv_offsets[0]), int(w.kv_offsets[1])
    for name in ("k_idx", "k", "v"):  # sequence 1 starts with sequence 0's first 512 rows
        host[name][ko1: ko1 + 512] = host[name][ko0: ko0 + 512]
    dev = {k: _to_dev(v) for k, v in host.items() if k not in ("q_offsets", "kv_offsets")}
    qo = torch.from_numpy(w.q_offsets.astype(np.int32)).cuda()
    ko = torch.from_numpy(w.kv_offsets.astype(np.int32)).cuda()
    out_c, idx_c = _layer(dsa.dsa_prefill, w, dev, dev, dsa.ragged(qo, ko, w.q_lens, w.kv_lens))
    # pages: sequence 0 owns 8 pages (0..7), sequence 1 reuses pages 0..3 then owns 8..11
    pages0 = list(range(8))
    pages1 = [0, 1, 2, 3, 8, 9, 10, 11]
    phys = {}
    for name in ("k_idx", "k", "v"):
        arr = host[name]
        out = np.zeros((12 * ps,) + arr.shape[1:], dtype=arr.dtype)
        out[: 1000] = arr[ko0: ko0 + 1000]
        out[8 * ps: 8 * ps + 900 - 512] = arr[ko1 + 512: ko1 + 900]
        phys[name] = out
    table = np.array([pages0, pages1], dtype=np.int32)
    cache = {k: _to_dev(v) for k, v in phys.items()}
    bt = _to_dev(table)
    rgp = dsa.ragged(qo, ko, w.q_lens, w.kv_lens, block_table=bt, page_size=ps,
                     cache_rows=12 * ps)
    out_p, idx_p = _layer(dsa.dsa_prefill, w, dev, cache, rgp)
    assert torch.equal(idx_c, idx_p)
    assert torch.equal(out_c, out_p)
    _check_oracle(w, host, idx_p, out_p, range(w.total_q), "shared prefix")


def _check_oracle(w, host, idx, out, rows, what):
    """Paged results against the oracle on the logical sequences (host arrays)."""
    rows = list(rows)
    idx_ref, out_ref, _ = O.Oracle.for_workload(w, host).layer_rows(rows)
    got_idx = idx.cpu().numpy()[rows]
    np.testing.assert_array_equal(got_idx, idx_ref, err_msg=what)
    PT.assert_close(PT.bf16_tensor_to_f64(out)[rows], out_ref, what)


PAGED_ORACLE_CASES = {
    "materialised": (dict(q_lens=[300, 1, 700], kv_lens=[900, 513, 700], K=64), 128, "prefill"),
    "fused": (dict(q_lens=[12288], kv_lens=[12288], K=512), 256, "prefill"),
    "decode": (dict(q_lens=[1] * 12, kv_lens=[1, 127, 128, 129, 1000, 4097, 300, 2500, 640, 768,
                                               5000, 33], K=256), 256, "decode"),
}


@pytest.mark.parametrize("case", sorted(PAGED_ORACLE_CASES))
def test_paged_matches_oracle(case):
    """Shuffled, non-identity page assignments (unused pages hold junk), checked row by row
    against the oracle on the logical sequences, not only against the contiguous GPU run."""
    cfg, ps, kind = PAGED_ORACLE_CASES[case]
    w = _wl(cfg["q_lens"], cfg["kv_lens"], K=cfg["K"])
    fn = dsa.dsa_decode if kind == "decode" else dsa.dsa_prefill
    _, (op, ip), (host, _, _, _, _, bt) = _both(w, ps, fn=fn, seed=11)
    table = bt.cpu().numpy()
    # the mapping is not the identity: some logical page lives elsewhere
    ident = np.arange(table.shape[1])[None, :] + np.concatenate(
        [[0], np.cumsum([(L + ps - 1) // ps for L in w.kv_lens])[:-1]])[:, None]
    used = np.arange(table.shape[1])[None, :] < np.array(
        [(L + ps - 1) // ps for L in w.kv_lens])[:, None]
    assert np.any(table[used] != ident[used])
    if w.total_q > 2000:
        rows = sorted(set(range(0, w.total_q, 97)) | {w.total_q - 2, w.total_q - 1})
    else:
        rows = range(w.total_q)
    _check_oracle(w, host, ip, op, rows, f"paged {case}")
