"""Helpers shared by the GPU parity tests: tolerance checks and sampled-row oracle checks.

Tolerance (gated bf16 outputs vs the fp64 oracle):
  max |err| <= 1e-2 and mean |err| <= 1e-3 (the stated bar), plus two checks that keep
  the bar meaningful at these magnitudes (|out| is ~1e-3 for near-uniform softmax, so
  an all-zero output would pass the absolute bar):
  ||err||_2 / ||ref||_2 <= 1e-2, and per element |err| <= 2^-7 |ref| + 2^-6 rms_h, with
  rms_h the root mean square of the reference over the element's (row, head).
Derivation of the per-element bound: the output is rounded to bf16 (relative 2^-9);
the softmax weights enter the P.V product rounded to bf16 (relative 2^-9 each), so an
element's error is sum_j (p^_j - p_j) v_j / l: with the rounding errors of ~2048 weights
independent, its standard deviation is ~2^-9 / sqrt(3) times the spread of sum_j p_j v_j / l
over the head's elements, i.e. ~1.1e-3 rms_h for random V; logits, exponentials and sums
are fp32 (relative ~1e-6).  2^-7 leaves a factor 4 over the output rounding, and 2^-6 rms_h
is ~14 standard deviations of the weight rounding, while one wrong index among K or a
dropped gate moves many elements by far more.
"""
from __future__ import annotations

import math

import numpy as np

import dsa_synth as S
import oracle as O

MAX_ABS = 1e-2
MEAN_ABS = 1e-3
REL_L2 = 1e-2
ELEM_REL = 2.0 ** -7
ELEM_RMS = 2.0 ** -6


def close_report(got: np.ndarray, ref: np.ndarray) -> dict:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(got - ref)
    nref = np.linalg.norm(ref)
    # (row, head) scale: the last axis is the head dimension
    rms_h = np.sqrt(np.mean(ref * ref, axis=-1, keepdims=True)) if ref.ndim else np.abs(ref)
    rep = {
        "max_abs": float(err.max()) if err.size else 0.0,
        "mean_abs": float(err.mean()) if err.size else 0.0,
        "rel_l2": float(np.linalg.norm(got - ref) / nref) if nref > 0 else float(np.linalg.norm(got)),
        "elem_viol": int(np.sum(err > ELEM_REL * np.abs(ref) + ELEM_RMS * rms_h)),
    }
    rep["ok"] = (rep["max_abs"] <= MAX_ABS and rep["mean_abs"] <= MEAN_ABS
                 and rep["rel_l2"] <= REL_L2 and rep["elem_viol"] == 0)
    return rep


def assert_close(got, ref, what=""):
    rep = close_report(got, ref)
    assert rep["ok"], f"{what}: {rep}"
    return rep


def bf16_tensor_to_f64(t) -> np.ndarray:
    import torch
    return t.detach().to("cpu").to(torch.float64).numpy()


def _host_idx_rows(w: S.Workload, tensor: int, start_row: int, nrows: int) -> np.ndarray:
    Hi, Di = w.n_idx_heads, w.idx_dim
    n = nrows * Hi * Di
    if w.idx_dtype == "fp8":
        a = S.host_e4m3_grid(n, w.seed, tensor, start_row * Hi * Di)
    else:
        a = S.host_bf16(n, w.idx_family, w.seed, tensor, start_row * Hi * Di, w.qkv_scale)
    return a.reshape(nrows, Hi, Di)


def oracle_row(w: S.Workload, r: int):
    """Oracle (idx, out, lse) of packed query row r, regenerating only what it reads.

    The indexer sees the sequence's keys 0..p; the attention sees only the selected
    rows, gathered on the host into a compact batch-of-one problem (the oracle's
    attention reads rows through the index list and never needs the rest).
    """
    b = w.row_seq(r)
    p = w.row_position(r)
    kv0 = int(w.kv_offsets[b])
    Hq, Hkv, d, K = w.n_q_heads, w.n_kv_heads, w.head_dim, w.top_k
    q_idx = _host_idx_rows(w, S.T_Q_IDX, r, 1)
    k_idx = _host_idx_rows(w, S.T_K_IDX, kv0, p + 1)
    if w.needle_pos and b == 0:
        u_enc, key_enc = S.needle_arrays(w)
        for j in w.needle_pos:
            if j <= p:
                k_idx[j] = key_enc
        if r in w.needle_rows:
            q_idx[0] = u_enc
    wt = S.host_f32(w.n_idx_heads, w.w_family, w.seed, S.T_W, 0)
    orc = O.Oracle({"q_idx": q_idx, "k_idx": k_idx, "w": wt, "q_offsets": np.array([0, 1]),
                    "kv_offsets": np.array([0, p + 1])}, top_k=K, n_idx_heads=w.n_idx_heads,
                   idx_dim=w.idx_dim, n_q_heads=Hq, n_kv_heads=Hkv, head_dim=d,
                   idx_fp8=(w.idx_dtype == "fp8"))
    scores = orc.index_scores_row(0)
    idx = O.topk_row(scores, K)
    sel = idx[idx >= 0]
    n = len(sel)
    kk = np.empty((max(n, 1), Hkv, d), np.uint16)
    vv = np.empty((max(n, 1), Hkv, d), np.uint16)
    for t, j in enumerate(sel):
        start = (kv0 + int(j)) * Hkv * d
        kk[t] = S.host_bf16(Hkv * d, S.NORMAL, w.seed, S.T_K, start, w.qkv_scale).reshape(Hkv, d)
        vv[t] = S.host_bf16(Hkv * d, S.NORMAL, w.seed, S.T_V, start, w.qkv_scale).reshape(Hkv, d)
    arrays = {"q": S.host_bf16(Hq * d, S.NORMAL, w.seed, S.T_Q, r * Hq * d, w.qkv_scale).reshape(1, Hq, d),
              "k": kk, "v": vv, "q_offsets": np.array([0, 1]), "kv_offsets": np.array([0, max(n, 1)])}
    if w.gate:
        arrays["gate"] = S.host_bf16(Hq * d, S.NORMAL, w.seed, S.T_GATE, r * Hq * d, 1.0).reshape(1, Hq, d)
    orc2 = O.Oracle(arrays, top_k=K, n_idx_heads=w.n_idx_heads, idx_dim=w.idx_dim, n_q_heads=Hq,
                    n_kv_heads=Hkv, head_dim=d)
    compact = np.full(K, -1, np.int32)
    compact[:n] = np.arange(n, dtype=np.int32)
    out, lse = orc2.sparse_attn_row(0, compact)
    return idx, out, lse, scores


def fused_cap(K: int) -> int:
    """Candidate slots per row of the library's fused indexer -> Top-K path (a planning
    constant of that path, restated here to aim rows at its regimes): rows with n <= K
    select everything, rows with n <= cap keep every score as a candidate, longer rows
    use the sampled threshold."""
    e = K / 16.0 + 1.0
    R = math.ceil(e + 5.0 * math.sqrt(e) + 16.0)
    return int(math.ceil(16.0 * (R + 6.0 * math.sqrt(R)) / 256.0) * 256)


def sample_rows(w: S.Workload, count: int, seed: int = 1):
    """Rows to check: the first and last row of every sequence (of the first 16 and the last
    one when there are more), the needle rows, the decode row with the longest history, rows
    on both sides of n = K and n = cap (the fused path's regimes: select all, keep every
    score, sampled threshold), then seeded random rows up to `count`."""
    total = w.total_q
    rows = {0, total - 1}
    qo = w.q_offsets
    seqs = list(range(min(w.batch, 16))) + [w.batch - 1]
    for b in seqs:
        if w.q_lens[b] > 0:
            rows.add(int(qo[b]))
            rows.add(int(qo[b + 1]) - 1)
    if w.needle_rows:
        rows.add(w.needle_rows[0])
        rows.add(w.needle_rows[-1])
    dec = [b for b in range(w.batch) if w.q_lens[b] == 1]
    if dec:
        rows.add(int(qo[max(dec, key=lambda b: w.kv_lens[b])]))
        rows.add(int(qo[min(dec, key=lambda b: w.kv_lens[b])]))
    K, cap = w.top_k, fused_cap(w.top_k)
    for b in range(w.batch):
        if w.q_lens[b] < 2:
            continue
        p0 = w.kv_lens[b] - w.q_lens[b]
        for n in (K, K + 1, cap, cap + 1):
            i = n - 1 - p0  # query index whose position is n - 1
            if 0 <= i < w.q_lens[b]:
                rows.add(int(qo[b]) + i)
    rng = np.random.default_rng(seed)
    while len(rows) < count:
        rows.add(int(rng.integers(0, total)))
    return sorted(r for r in rows if 0 <= r < total)
