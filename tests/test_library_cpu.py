"""CPU-side checks of the C-ABI library: it builds, loads, exports every declared entry
point, and rejects bad arguments on the host before any CUDA call is made."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    text = open(os.path.join(ROOT, "include", "dsa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dsa_[a-z_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = _declared()
    for required in ("dsa_index_scores", "dsa_topk", "dsa_sparse_attn_gated", "dsa_prefill",
                     "dsa_decode", "dsa_workspace_size", "dsa_status_string"):
        assert required in names


def test_library_exports_every_declared_symbol():
    import indexer_top_gated_b200 as dsa
    lib = ctypes.CDLL(dsa.LIB_PATH)
    for name in _declared():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", dsa.LIB_PATH], capture_output=True,
                         text=True).stdout
    exported = set(re.findall(r"\bT (dsa_\w+)", out))
    assert set(_declared()) <= exported
    assert set(dsa.EXPORTS) == set(_declared())


def test_status_strings_and_version():
    import indexer_top_gated_b200 as dsa
    assert dsa.status_string(0) == "ok"
    assert "workspace" in dsa.status_string(dsa.DSA_ERR_WORKSPACE)
    assert dsa.lib.dsa_version() >= 100


class _FakeTensor:
    """Stands in for a device tensor: only its address is read on the host path."""

    def __init__(self, addr, nbytes=1 << 20):
        self.addr, self.nbytes = addr, nbytes

    def data_ptr(self):
        return self.addr

    def numel(self):
        return self.nbytes

    def element_size(self):
        return 1


def _rg(dsa, batch=1, max_q=8, max_kv=8):
    return dsa.Ragged(batch, 0x1000, 0x2000, max_q, max_kv, max_q * batch, max_kv * batch)


def test_host_validation_rejects_bad_arguments():
    import indexer_top_gated_b200 as dsa
    L = dsa.lib
    good = dsa.LayerShape(top_k=4)
    rg = _rg(dsa)
    P = good.params()
    null = None
    A = 0x10000  # 16-byte aligned fake addresses; never dereferenced on these paths
    # bad K
    bad = dsa.LayerShape(top_k=0).params()
    assert L.dsa_topk(ctypes.byref(bad), ctypes.byref(rg), A, 8, 0, 1, A, 4, null, null) == \
        dsa.DSA_ERR_UNSUPPORTED
    # scores leading dimension not a multiple of 4 / too small
    assert L.dsa_topk(ctypes.byref(P), ctypes.byref(rg), A, 6, 0, 1, A, 4, null, null) == \
        dsa.DSA_ERR_INVALID_ARG
    assert L.dsa_topk(ctypes.byref(P), ctypes.byref(rg), A, 4, 0, 1, A, 4, null, null) == \
        dsa.DSA_ERR_INVALID_ARG
    # row range outside the batch
    assert L.dsa_topk(ctypes.byref(P), ctypes.byref(rg), A, 8, 4, 5, A, 4, null, null) == \
        dsa.DSA_ERR_INVALID_ARG
    # idx leading dimension below K
    assert L.dsa_topk(ctypes.byref(P), ctypes.byref(rg), A, 8, 0, 1, A, 3, null, null) == \
        dsa.DSA_ERR_INVALID_ARG
    # unsupported indexer dim / head dim / GQA layout
    for shape in (dsa.LayerShape(idx_dim=32), dsa.LayerShape(n_idx_heads=5)):
        p = shape.params()
        assert L.dsa_index_scores(ctypes.byref(p), ctypes.byref(rg), A, A, A, 0, 1, A, 8, null) \
            == dsa.DSA_ERR_UNSUPPORTED
    for shape, code in ((dsa.LayerShape(head_dim=64), dsa.DSA_ERR_UNSUPPORTED),
                        (dsa.LayerShape(n_q_heads=30, n_kv_heads=4), dsa.DSA_ERR_INVALID_ARG),
                        (dsa.LayerShape(n_q_heads=64, n_kv_heads=2), dsa.DSA_ERR_UNSUPPORTED),
                        (dsa.LayerShape(n_q_heads=12, n_kv_heads=3), dsa.DSA_ERR_UNSUPPORTED)):
        p = shape.params()
        assert L.dsa_sparse_attn_gated(ctypes.byref(p), ctypes.byref(rg), A, A, A, A, 2048, 0, 1,
                                       null, A, null, null, null) == code
    # misaligned tensors
    p = dsa.LayerShape(top_k=4).params()
    assert L.dsa_sparse_attn_gated(ctypes.byref(p), ctypes.byref(rg), A + 2, A, A, A, 4, 0, 1,
                                   null, A, null, null, null) == dsa.DSA_ERR_INVALID_ARG
    # workspace missing / misaligned / too small
    for ws, nbytes in ((None, 1 << 20), (A + 16, 1 << 20), (A, 8)):
        rc = L.dsa_prefill(ctypes.byref(p), ctypes.byref(rg), A, A, A, A, A, A, null, A, null,
                           null, ws, nbytes, null)
        assert rc == dsa.DSA_ERR_WORKSPACE, (ws, nbytes, rc)
    # decode needs one query per sequence
    rg2 = _rg(dsa, batch=2, max_q=3)
    assert L.dsa_decode(ctypes.byref(p), ctypes.byref(rg2), A, A, A, A, A, A, null, A, null, null,
                        A, 1 << 20, null) == dsa.DSA_ERR_INVALID_ARG
    # the mixing entry needs both the gate logits and the second branch
    for gate_p, other_p in ((None, A), (A, None)):
        assert L.dsa_sparse_attn_gated_mix(ctypes.byref(p), ctypes.byref(rg), A, A, A, A, 4, 0, 1,
                                           gate_p, other_p, A, null, null, null) == \
            dsa.DSA_ERR_INVALID_ARG
    assert L.dsa_sparse_attn_gated_mix(ctypes.byref(p), ctypes.byref(rg), A, A, A, A, 4, 0, 1, A,
                                       A + 8, A, null, null, null) == dsa.DSA_ERR_INVALID_ARG
    # null ragged / params
    assert L.dsa_topk(None, ctypes.byref(rg), A, 8, 0, 1, A, 4, null, null) == dsa.DSA_ERR_INVALID_ARG


def test_paged_cache_descriptor_is_validated():
    import indexer_top_gated_b200 as dsa
    L = dsa.lib
    P = dsa.LayerShape(top_k=4).params()
    A = 0x10000
    base = dict(block_table=A, max_pages=4, page_size=128)
    bad = (dict(page_size=100), dict(page_size=64), dict(page_size=384), dict(max_pages=1),
           dict(total_kv=1000))
    for b in bad:
        rg = dsa.Ragged(1, 0x1000, 0x2000, 8, 500, 8, 1024, None, 0, 0)
        for k, v in dict(base, **b).items():
            setattr(rg, k, v)
        rc = L.dsa_sparse_attn_gated(ctypes.byref(P), ctypes.byref(rg), A, A, A, A, 4, 0, 1,
                                     None, A, None, None, None)
        assert rc == dsa.DSA_ERR_INVALID_ARG, (b, rc)
    # a valid descriptor passes the host checks (workspace sizing is host-only)
    rg = dsa.Ragged(1, 0x1000, 0x2000, 8, 500, 8, 1024, A, 4, 128)
    mn, rec = dsa.dsa_workspace_size(dsa.LayerShape(top_k=4), rg)
    assert 0 < mn <= rec
    assert L.dsa_version() == 102


def test_block_selection_arguments():
    import indexer_top_gated_b200 as dsa
    L = dsa.lib
    rg = dsa.Ragged(1, 0x1000, 0x2000, 64, 4096, 64, 4096, None, 0, 0)
    shape = dsa.LayerShape(top_k=8)
    mn, rec = dsa.dsa_index_topk_blocks_workspace_size(shape, rg, 64, 64)
    assert 0 < mn < rec
    for bad_block in (16, 48, 8192):
        with pytest.raises(RuntimeError, match="invalid"):
            dsa.dsa_index_topk_blocks_workspace_size(shape, rg, bad_block, 64)
    P = shape.params()
    A = 0x10000
    # ld_idx must hold Kb * block positions
    assert L.dsa_index_topk_blocks(ctypes.byref(P), ctypes.byref(rg), A, A, A, 64, 0, 1, A,
                                   8 * 64 - 1, None, A, rec, None) == dsa.DSA_ERR_INVALID_ARG
    assert L.dsa_index_topk_blocks(ctypes.byref(P), ctypes.byref(rg), A, A, A, 64, 0, 1, A,
                                   8 * 64, None, A, mn - 1, None) == dsa.DSA_ERR_WORKSPACE


def test_workspace_size_is_host_only():
    import indexer_top_gated_b200 as dsa
    shape = dsa.LayerShape(top_k=2048)
    rg = dsa.Ragged(1, 0x1000, 0x2000, 32768, 32768, 32768, 32768)
    mn, rec = dsa.dsa_workspace_size(shape, rg, is_decode=True)
    assert mn == 32768 * 4 + 2048 * 4
    assert mn <= rec <= (1 << 30) + mn
    # prefill of one long sequence: one fused pass over all rows, each row holding its
    # candidate slots (8 bytes each, at least 2K of them) and its index row
    mn_p, rec_p = dsa.dsa_workspace_size(shape, rg, is_decode=False)
    assert mn_p == mn
    assert rec_p >= 32768 * (2 * 2048 * 8 + 2048 * 4)
    # a small prefill keeps its scores materialised (they fit in L2)
    rg_small = dsa.Ragged(1, 0x1000, 0x2000, 4096, 4096, 4096, 4096)
    assert dsa.dsa_workspace_size(dsa.LayerShape(top_k=256), rg_small)[1] <= 1 << 30


def test_fused_index_topk_workspace_and_limits():
    import indexer_top_gated_b200 as dsa
    rg = dsa.Ragged(1, 0x1000, 0x2000, 32768, 32768, 32768, 32768)
    mn, rec = dsa.dsa_index_topk_workspace_size(dsa.LayerShape(top_k=2048), rg, 32768)
    assert 0 < mn < rec
    # rec holds every row: per row at least the candidate slots
    assert rec - mn >= 32767 * 2 * 2048 * 8
    # K beyond the candidate slots, or rows beyond the position bitmap: unsupported
    with pytest.raises(RuntimeError, match="unsupported"):
        dsa.dsa_index_topk_workspace_size(dsa.LayerShape(top_k=6000), rg, 1)
    long_rg = dsa.Ragged(1, 0x1000, 0x2000, 1, 400000, 1, 400000)
    with pytest.raises(RuntimeError, match="unsupported"):
        dsa.dsa_index_topk_workspace_size(dsa.LayerShape(top_k=64), long_rg, 1)
    L = dsa.lib
    P = dsa.LayerShape(top_k=2048).params()
    A = 0x10000
    args = lambda ws, nbytes, q0=0, qn=1, ld=2048: (  # noqa: E731
        ctypes.byref(P), ctypes.byref(rg), A, A, A, q0, qn, A, ld, None, ws, nbytes, None)
    assert L.dsa_index_topk(*args(A, mn)[:10], None, mn, None) == dsa.DSA_ERR_WORKSPACE
    assert L.dsa_index_topk(*args(A + 16, mn)) == dsa.DSA_ERR_WORKSPACE
    assert L.dsa_index_topk(*args(A, mn - 1)) == dsa.DSA_ERR_WORKSPACE
    assert L.dsa_index_topk(*args(A, mn, ld=2047)) == dsa.DSA_ERR_INVALID_ARG
    assert L.dsa_index_topk(*args(A, mn, q0=32768)) == dsa.DSA_ERR_INVALID_ARG
    assert L.dsa_index_topk(*args(A, mn, qn=0)) == 0  # nothing to do


def test_mixed_batch_workspace_plan_uses_host_offsets():
    """With host copies of the offsets, a batch mixing prefill chunks and single queries is
    planned per stretch of sequences: the recommended workspace holds every row's index row
    plus the largest stretch's steps 1-2 (host-side sizing only, no device access)."""
    import numpy as np

    import dsa_synth as S
    import indexer_top_gated_b200 as dsa

    w = S.workload("mixed_serving")
    shape = dsa.workload_shape(w)
    qoh = w.q_offsets.astype(np.int32)
    koh = w.kv_offsets.astype(np.int32)
    base = (w.batch, 0x1000, 0x2000, max(w.q_lens), max(w.kv_lens), w.total_q, w.total_kv,
            None, 0, 0)
    plain = dsa.Ragged(*base)
    planned = dsa.Ragged(*base, qoh.ctypes.data, koh.ctypes.data)
    mn0, rec0 = dsa.dsa_workspace_size(shape, plain)
    mn1, rec1 = dsa.dsa_workspace_size(shape, planned)
    assert mn0 == mn1
    assert rec1 != rec0 and rec1 >= w.total_q * w.top_k * 4
    # a batch of one kind is planned as before
    one = S.workload("prefill_t32768_k2048")
    q1 = one.q_offsets.astype(np.int32)
    k1 = one.kv_offsets.astype(np.int32)
    b1 = (1, 0x1000, 0x2000, 32768, 32768, 32768, 32768, None, 0, 0)
    assert dsa.dsa_workspace_size(dsa.workload_shape(one), dsa.Ragged(*b1)) == \
        dsa.dsa_workspace_size(dsa.workload_shape(one), dsa.Ragged(*b1, q1.ctypes.data, k1.ctypes.data))


def test_probe_library_exports_its_declared_entry_point():
    """The benchmark's gather-ceiling probe (libdsaprobe.so) builds for sm_100a and exports
    the function include/dsa_probe.h declares; argument checks return 0 without a launch."""
    import ctypes
    import os
    import re

    from indexer_top_gated_b200 import _build, peaks
    hdr = open(os.path.join(_build.INCLUDE, "dsa_probe.h")).read()
    names = re.findall(r"^\w[\w\s\*]*?\b(dsa_\w+)\(", hdr, re.M)
    assert names == ["dsa_probe_gather"]
    L = peaks._load()
    for n in names:
        assert hasattr(L, n)
    # n_rows not a power of two / null buffers: rejected on the host
    assert L.dsa_probe_gather(0x1000, 3, 0x2000, 64, 0, 1, 1, 1, 0x3000) == 0.0
    assert L.dsa_probe_gather(None, 4, 0x2000, 64, 0, 1, 1, 1, 0x3000) == 0.0
    # unknown variant; a 32-bit index of 16-byte units covers at most 2^28 rows of 256 B
    assert L.dsa_probe_gather(0x1000, 4, 0x2000, 64, 4, 1, 1, 1, 0x3000) == 0.0
    assert L.dsa_probe_gather(0x1000, 1 << 29, 0x2000, 64, 2, 1, 1, 1, 0x3000) == 0.0
