#!/usr/bin/env python
"""Benchmark of the B200 gated Indexer + Top-K sparse-attention layer.

One step = one pass of the whole layer (indexer scores, Top-K, gated sparse attention)
over the prefill workload T = 32768, K = 2048, GQA 32 query / 4 KV heads x 128,
indexer 4 heads x 64 (bf16), with inputs resident in HBM.  Prints one JSON line.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun the global batch is `world` copies of the workload, split over ranks by the
data-parallel partitioner (indexer_top_gated_b200.partition: whole sequences by cost); each
rank runs its share with no collective on the data path (weak scaling), and the reported
time is the max over ranks.  Beside the headline the same run measures the gather ceilings
that bound the attention, the decode workload and the K = 2048 workloads whose cache does
not fit in L2.
`--impl reference` times the CPU oracle on bounded samples of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "sparse-attn layer tokens/sec (prefill) & µs/token (decode) at K=2048, % roofline"
WORKLOAD = "prefill_t32768_k2048"
DECODE_WORKLOAD = "decode_b64_l131072"
# measured in the same run beside the headline: the K = 2048 configurations whose K/V cache
# no longer fits in L2
EXTRA_WORKLOADS = ["prefill_t131072_needles", "mixed_serving"]
L2_BYTES = 126e6
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target wall time of the CPU-baseline sample")
    ap.add_argument("--ws-rows", type=int, default=0,
                    help="cap the workspace at this many query rows per pass (profiling)")
    ap.add_argument("--lean", action="store_true",
                    help="only the timed region: no e2e, decode, CPU-baseline, gather-peak or "
                         "extra-workload legs")
    ap.add_argument("--also", default=",".join(EXTRA_WORKLOADS),
                    help="comma-separated workloads also measured (not the headline); '' for none")
    ap.add_argument("--no-peaks", action="store_true", help="skip the live gather-ceiling probe")
    ap.add_argument("--seq-stride", type=int, default=1,
                    help="keep every N-th sequence of the workload: a smaller case with the same "
                         "mix of sequences, for profile captures of workloads whose inputs exceed "
                         "what a capture may hold (not a bench line)")
    a = ap.parse_args()
    if a.lean:
        a.no_e2e = a.no_decode = a.no_cpu_baseline = a.no_peaks = True
        a.also = ""
    return a


# ----------------------------------------------------------------------------- helpers

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def algorithmic(w):
    """Algorithmic work of one pass of the layer over workload w, per stage."""
    K, Hi, Di, Hq, Hkv, d = w.top_k, w.n_idx_heads, w.idx_dim, w.n_q_heads, w.n_kv_heads, w.head_dim
    e_idx = 1 if w.idx_dtype == "fp8" else 2
    n_sum = 0
    sel_sum = 0
    for Q, L in zip(w.q_lens, w.kv_lens):
        p0 = L - Q  # positions of the first query
        n = np.arange(p0 + 1, L + 1, dtype=np.int64)
        n_sum += int(n.sum())
        sel_sum += int(np.minimum(n, K).sum())
    tq, tk = w.total_q, w.total_kv
    return {
        "idx_flops": 2 * Hi * Di * n_sum,
        "idx_bytes": 4 * n_sum + (tq + tk) * Hi * Di * e_idx,
        "topk_bytes": 4 * n_sum + 4 * K * tq,
        # fused path: the selection never sees the score matrix; its floor is reading the
        # K selected (position, score) pairs and writing the index rows
        "topk_bytes_fused": 12 * sel_sum,
        # what the fused path's selection stage moves: each row's bf16 samples (every 16th score),
        # its candidate pairs (about 16 R of them, R = e + 5 sqrt(e) + 16 samples, e = K S / n,
        # or all n when n <= cap) and its index row
        "topk_bytes_fused_moved": fused_moved_bytes(w),
        "attn_bytes": sel_sum * Hkv * d * 2 * 2 + 3 * tq * Hq * d * 2 + 4 * K * tq,
        "attn_flops": 4 * sel_sum * Hq * d,
        "scores": n_sum,
        "selected": sel_sum,
    }


def _sub_workload(w, seqs):
    """Workload w restricted to the sequences seqs (for per-path byte accounting)."""
    import copy
    sw = copy.copy(w)
    sw.q_lens = [w.q_lens[b] for b in seqs]
    sw.kv_lens = [w.kv_lens[b] for b in seqs]
    return sw


def fused_moved_bytes(w) -> int:
    """Bytes the fused selection stage reads and writes for workload w (see algorithmic)."""
    K = w.top_k
    e = K / 16.0 + 1.0
    rr = math.ceil(e + 5.0 * math.sqrt(e) + 16.0)
    cap = int(math.ceil(16.0 * (rr + 6.0 * math.sqrt(rr)) / 256.0) * 256)
    total = 0
    for Q, L in zip(w.q_lens, w.kv_lens):
        n = np.arange(L - Q + 1, L + 1, dtype=np.float64)
        S_ = np.floor((n - 1) / 16.0) + 1
        R = np.minimum(np.ceil(K * S_ / n + 5.0 * np.sqrt(K * S_ / n) + 16.0), S_)
        cand = np.where(n <= K, 0.0, np.where(n <= cap, n, 16.0 * R))
        samples = np.where(n <= cap, 0.0, S_)
        total += float((2.0 * samples + 8.0 * cand + 4.0 * K).sum())  # bf16 samples
    return int(total)


def aggregate_max(ms_local: float, tokens_per_rank: int, world: int, device="cuda"):
    """Whole-job throughput: tokens of all ranks over the slowest rank's time (max over ranks)."""
    import torch
    t = torch.tensor([ms_local], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms_max = float(t.item())
    return ms_max, tokens_per_rank * world / (ms_max / 1e3)


def rank_workload(w, world: int, rank: int):
    """This rank's share of a global batch of `world` copies of workload w (weak scaling):
    the data-parallel partitioner deals whole sequences to ranks by cost; the rank's
    sequences are generated with seed = rank, so ranks hold different data."""
    import copy

    from indexer_top_gated_b200 import partition as PA
    if world == 1:
        return w
    sh = PA.shard(list(w.q_lens) * world, list(w.kv_lens) * world, w.top_k, world, rank,
                  by="sequences")
    rw = copy.copy(w)
    rw.q_lens, rw.kv_lens, rw.seed = list(sh.q_lens), list(sh.kv_lens), rank
    if (rw.q_lens, rw.kv_lens) != (list(w.q_lens), list(w.kv_lens)):
        rw.needle_pos, rw.needle_rows = [], []  # planted rows belong to the workload's own layout
    return rw


def source_sha(paths):
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def l2_note(w):
    """How the timed steps relate to the 126 MB L2 (no flush between steps)."""
    mib = 3 * w.total_q * w.n_q_heads * w.head_dim * 2 / 2**20
    if mib * 2**20 > 126e6:
        return f"inputs larger than L2 (q + gate + out = {mib:.0f} MiB per step); no flush"
    return f"inputs fit in L2 (q + gate + out = {mib:.0f} MiB per step); no flush: L2-warm timing"


def committed_traffic(kernel_file: str, summary: str, key: str = "traffic_bytes_per_full_launch"):
    """DRAM bytes per launch recorded by an ncu capture (a `key: value` line of a summary in
    profiles/), or None if there is none or the kernel's source has changed since."""
    path = os.path.join(ROOT, "profiles", summary)
    if not os.path.exists(path):
        return None
    vals = {}
    for line in open(path):
        if ":" in line:
            k, v = line.split(":", 1)
            vals[k.strip()] = v.strip()
    try:
        if vals.get("source_sha256_16") != source_sha([kernel_file, "indexer_top_gated_b200/csrc/common.cuh"]):
            return None
        return float(vals[key])
    except Exception:
        return None


ATTN_SRC = "indexer_top_gated_b200/csrc/sparse_attn.cuh"


def attn_traffic(workload: str, seq_stride: int = 1):
    # a committed capture is of the full workload (or scaled to it): none for a reduced case
    if seq_stride > 1:
        return None
    return committed_traffic(ATTN_SRC, f"sparse_attn_gated_{workload}.txt")


def kv_cache_bytes(w) -> int:
    return 2 * w.total_kv * w.n_kv_heads * w.head_dim * 2


def stage_report(w, stage_ms, stage_n, peaks, gather, fused_rows=0):
    """Per-stage achieved rates and roofline fractions of one step of workload w.

    - indexer: algorithmic flops (512 per score) against the sustained dense bf16 peak;
    - Top-K: against the HBM copy peak, the bytes the path that ran moves -- materialised:
      4 B per causal score read + 4 B per index written (the scope table's definition, which
      the >= 60 % target is stated against); fused: the sampled scores it reads (4 B per 16
      positions), its candidate pairs (8 B each, the count estimated from the threshold rule)
      and the index rows.  On the fused path the scope table's bytes are also given as an
      equivalent rate (a materialised selection would have to move them; above the HBM peak
      it says the fused path does better than any materialised one could), and so is the
      floor of 12 B per selected position;
    - attention: algorithmic bytes (selected K/V rows, q, gate, out, indices) against the
      measured gather ceiling of random 256-byte rows from L2 (every gathered byte crosses
      L2 -> SM), plus the DRAM bytes of a committed ncu capture against the HBM copy peak.
    """
    # rows whose steps 1-2 ran fused (the library counts them): all, none, or -- in a mixed
    # batch -- the long query groups (Q_b >= 128), the rest materialised
    long_rows = sum(q for q in w.q_lens if q >= 128)
    if fused_rows >= w.total_q:
        fused, alg = True, algorithmic(w)
    elif fused_rows == 0:
        fused, alg = False, algorithmic(w)
    else:
        assert fused_rows == long_rows, (fused_rows, long_rows)
        fused = True
        alg = algorithmic(w)
        lw = _sub_workload(w, [b for b, q in enumerate(w.q_lens) if q >= 128])
        sw = _sub_workload(w, [b for b, q in enumerate(w.q_lens) if q < 128])
        a_l, a_s = algorithmic(lw), algorithmic(sw)
        # the selection stage moved the long groups' fused bytes and the short ones' scores
        alg["topk_bytes_fused_moved"] = a_l["topk_bytes_fused_moved"] + a_s["topk_bytes"]
        alg["topk_bytes_fused"] = a_l["topk_bytes_fused"] + a_s["topk_bytes"]
    sec1 = stage_ms[1] / 1e3
    idx_tf = alg["idx_flops"] / (stage_ms[0] / 1e3) / 1e12 if stage_ms[0] > 0 else None
    tk_s = alg["topk_bytes"] / sec1 / 1e9 if sec1 > 0 else None
    tk_f = alg["topk_bytes_fused"] / sec1 / 1e9 if sec1 > 0 else None
    tk_m = alg["topk_bytes_fused_moved"] / sec1 / 1e9 if sec1 > 0 else None
    tk = tk_m if fused else tk_s
    at = alg["attn_bytes"] / (stage_ms[2] / 1e3) / 1e9 if stage_ms[2] > 0 else None
    traffic = attn_traffic(w.name, getattr(w, "seq_stride", 1))
    l2p = gather.get("l2", {}).get("gbs") if gather else None
    dram_gbs = traffic / stage_n[2] / (stage_ms[2] / stage_n[2] / 1e3) / 1e9 \
        if traffic and stage_ms[2] > 0 else None
    hbm = peaks["hbm_gbs"]
    stages = [
        {"kernel": "idx_scores", "ms_per_step": stage_ms[0], "launches_per_step": stage_n[0],
         "bound": "tensor", "achieved": idx_tf, "unit": "TFLOP/s",
         "peak": peaks["bf16_tflops_sustained"],
         "frac": idx_tf / peaks["bf16_tflops_sustained"] if idx_tf else None,
         "path": "fused: sampled threshold, candidates only" if fused else "materialised scores"},
        {"kernel": "topk_select", "ms_per_step": stage_ms[1], "launches_per_step": stage_n[1],
         "bound": "hbm", "unit": "GB/s", "peak": hbm,
         "achieved": tk, "frac": tk / hbm if tk else None,
         "bytes_definition": ("fused path: sampled scores read + candidate pairs read + index "
                              "rows written" if fused else
                              "4 B per causal score read + 4 B per index written (the "
                              "target's definition)"),
         "scope_equivalent_gbs": tk_s if fused else None,
         "scope_equivalent_frac": tk_s / hbm if (fused and tk_s) else None,
         "scope_definition": "4 B per causal score + 4 B per index (what a materialised "
                             "selection moves; the >= 60 % target is stated on it)",
         "floor_gbs": tk_f if fused else None,
         "floor_frac": tk_f / hbm if (fused and tk_f) else None,
         "floor_definition": "12 B per selected position"},
        {"kernel": "sparse_attn_gated", "ms_per_step": stage_ms[2], "launches_per_step": stage_n[2],
         "bound": "l2", "unit": "GB/s", "achieved": at, "peak": l2p,
         "frac": at / l2p if (at and l2p) else None,
         "peak_definition": "measured gather of random 256-byte rows from an L2-resident buffer",
         "kv_cache_bytes": kv_cache_bytes(w),
         "kv_fits_l2": kv_cache_bytes(w) <= L2_BYTES,
         "dram_traffic_per_launch": traffic / stage_n[2] if traffic else None,
         "dram_gbs": dram_gbs, "dram_frac": dram_gbs / hbm if dram_gbs else None},
    ]
    for st in stages:
        if st["bound"] == "hbm" and st["frac"] is not None:
            assert st["frac"] <= 1.0, f"{st['kernel']}: {st['frac']:.3f} of the HBM peak is not an HBM rate"
    return stages


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.tmp = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.tmp, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        self.tmp.flush()
        rows = []
        with open(self.tmp.name) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.tmp.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if num(r[2]) is not None]
        pw = [num(r[3]) for r in rows if num(r[3]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        busy = [s for s, r in zip(sm, rows) if num(r[3]) and num(r[3]) > 200] or sm
        return {"sm_mhz": statistics.median(busy) if busy else None,
                "sm_max_mhz": max(mx) if mx else None,
                "power_w_max": max(pw) if pw else None,
                "samples": len(rows), "reasons": reasons}


# ----------------------------------------------------------------------------- GPU arm

def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import dsa_synth as S
    import indexer_top_gated_b200 as dsa

    dev_id = local_rank
    torch.cuda.set_device(dev_id)
    w = rank_workload(S.workload(args.workload), world, rank)
    if args.seq_stride > 1:
        w = _sub_workload(w, [b for b in range(w.batch) if b % args.seq_stride == 0])
        w.needle_pos, w.needle_rows = [], []  # planted rows belong to the full layout
        w.seq_stride = args.seq_stride
    inputs = S.make_device_inputs(w)
    shape = dsa.workload_shape(w)
    rg = dsa.ragged(inputs["q_offsets"], inputs["kv_offsets"], w.q_lens, w.kv_lens)
    decode = max(w.q_lens) == 1
    layer = dsa.dsa_decode if decode else dsa.dsa_prefill
    ws_min, ws_bytes = dsa.dsa_workspace_size(shape, rg, decode)
    if args.ws_rows > 0:
        ws_bytes = min(ws_bytes, ws_min * args.ws_rows)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    out = torch.empty((w.total_q, w.n_q_heads, w.head_dim), dtype=torch.bfloat16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()

    def step():
        layer(shape, rg, inputs["q_idx"], inputs["k_idx"], inputs["w"], inputs["q"], inputs["k"],
              inputs["v"], inputs["gate"], out, err_count=err, workspace=ws, ws_bytes=ws_bytes)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    dsa.dsa_stage_times(reset=True)

    # ---- timed region: K steps, inputs resident, events on the launching stream
    launches0 = dsa.dsa_launch_count()
    dsa.dsa_fused_rows(reset=True)
    dsa.dsa_stage_timing(True)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev_id) as clocks:
        barrier()
        torch.cuda.synchronize()
        t0.record(stream)
        for _ in range(args.steps):
            step()
        t1.record(stream)
        torch.cuda.synchronize()
        barrier()
    dsa.dsa_stage_timing(False)
    launches = dsa.dsa_launch_count() - launches0
    fused_rows = dsa.dsa_fused_rows(reset=True) // max(1, args.steps)
    stage_ms, stage_launches = dsa.dsa_stage_times(reset=True)
    ms_total = t0.elapsed_time(t1)
    status = dsa.dsa_device_status()
    assert status == 0, f"device status {status}"
    assert int(err.item()) == 0

    ms_max, value = aggregate_max(ms_total, w.total_q * args.steps, world)

    # ---- end to end through the C ABI with host buffers
    e2e = None
    if not args.no_e2e:
        names = ["q_idx", "k_idx", "w", "q", "k", "v", "gate", "q_offsets", "kv_offsets"]
        host = {k: inputs[k].cpu().pin_memory() for k in names}
        out_host = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        h2d = sum(host[k].numel() * host[k].element_size() for k in names)
        d2h = out.numel() * out.element_size()

        host_io = dict(host, out=out_host)
        dev_io = dict(inputs, out=out)

        if decode:
            def e2e_step():
                for k in names:
                    inputs[k].copy_(host[k], non_blocking=True)
                step()
                out_host.copy_(out, non_blocking=True)
        else:
            def e2e_step():
                # one C-ABI call: uploads overlapped with the computation of earlier row ranges,
                # output rows copied back as they are done
                dsa.dsa_prefill_from_host(shape, rg, host_io, dev_io, 0, ws, ws_bytes)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_e2e = max(3, args.steps // 3)
        e0.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        te_ms, te_val = aggregate_max(e0.elapsed_time(e1), w.total_q * n_e2e, world)
        e2e = {"value": te_val, "unit": "tokens/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "steps": n_e2e, "ms_per_step": te_ms / n_e2e}

    result = {
        "w": w, "value": value, "ms_total": ms_max, "launches": launches,
        "fused_rows": fused_rows,
        "stage_ms": stage_ms, "stage_launches": stage_launches, "clocks": clocks.summary(),
        "e2e": e2e, "ws_bytes": ws_bytes,
    }
    del inputs, ws, out
    torch.cuda.empty_cache()
    return result


def run_decode_side(args):
    """Decode step time on the decode workload (one new token for each of 64 sequences)."""
    import torch

    import dsa_synth as S
    import indexer_top_gated_b200 as dsa

    w = S.workload(DECODE_WORKLOAD)
    free, _ = torch.cuda.mem_get_info()
    if w.device_bytes() * 1.2 > free:
        return None
    inputs = S.make_device_inputs(w)
    shape = dsa.workload_shape(w)
    rg = dsa.ragged(inputs["q_offsets"], inputs["kv_offsets"], w.q_lens, w.kv_lens)
    _, ws_bytes = dsa.dsa_workspace_size(shape, rg, True)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    out = torch.empty((w.total_q, w.n_q_heads, w.head_dim), dtype=torch.bfloat16, device="cuda")

    def step():
        dsa.dsa_decode(shape, rg, inputs["q_idx"], inputs["k_idx"], inputs["w"], inputs["q"],
                       inputs["k"], inputs["v"], inputs["gate"], out, workspace=ws,
                       ws_bytes=ws_bytes)

    for _ in range(5):
        step()
    torch.cuda.synchronize()
    dsa.dsa_stage_times(reset=True)
    dsa.dsa_stage_timing(True)
    n = 50
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(n):
        step()
    e1.record()
    torch.cuda.synchronize()
    dsa.dsa_stage_timing(False)
    stage_ms, _ = dsa.dsa_stage_times(reset=True)
    ms = e0.elapsed_time(e1) / n
    alg = algorithmic(w)
    del inputs, ws, out
    torch.cuda.empty_cache()
    return {"workload": DECODE_WORKLOAD, "batch": w.batch, "context": w.kv_lens[0],
            "us_per_step": ms * 1e3, "us_per_token": ms * 1e3 / w.batch,
            "stage_us_per_step": [x * 1e3 / n for x in stage_ms],
            "k_idx_scan_gbs": (w.total_kv * w.n_idx_heads * w.idx_dim * 2) /
                              (stage_ms[0] / n / 1e3) / 1e9}


def run_extra_workload(name, gather, steps=3, warmup=2):
    """One more workload in the same run (not the headline): tokens/s and the per-stage
    roofline fractions of a few steps of dsa_prefill / dsa_decode, inputs resident."""
    import torch

    import dsa_synth as S
    import indexer_top_gated_b200 as dsa

    w = S.workload(name)
    decode = max(w.q_lens) == 1
    free, _ = torch.cuda.mem_get_info()
    if w.device_bytes() * 1.1 > free:
        return {"workload": name, "skipped": f"needs {w.device_bytes() / 2**30:.1f} GiB"}
    inputs = S.make_device_inputs(w)
    shape = dsa.workload_shape(w)
    rg = dsa.ragged(inputs["q_offsets"], inputs["kv_offsets"], w.q_lens, w.kv_lens)
    _, ws_bytes = dsa.dsa_workspace_size(shape, rg, decode)
    free, _ = torch.cuda.mem_get_info()
    ws_bytes = int(min(ws_bytes, max(free - (4 << 30), 0)))
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    out = torch.empty((w.total_q, w.n_q_heads, w.head_dim), dtype=torch.bfloat16, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    layer = dsa.dsa_decode if decode else dsa.dsa_prefill

    def step():
        layer(shape, rg, inputs["q_idx"], inputs["k_idx"], inputs["w"], inputs["q"], inputs["k"],
              inputs["v"], inputs["gate"], out, err_count=err, workspace=ws, ws_bytes=ws_bytes)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    dsa.dsa_stage_times(reset=True)
    dsa.dsa_fused_rows(reset=True)
    dsa.dsa_stage_timing(True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clocks:
        e0.record()
        for _ in range(steps):
            step()
        e1.record()
        torch.cuda.synchronize()
    dsa.dsa_stage_timing(False)
    stage_ms, stage_launches = dsa.dsa_stage_times(reset=True)
    fused_rows = dsa.dsa_fused_rows(reset=True) // steps
    ms = e0.elapsed_time(e1) / steps
    assert dsa.dsa_device_status() == 0 and int(err.item()) == 0
    peaks, _ = load_peaks()
    sm = [x / steps for x in stage_ms]
    sn = [max(1, n // steps) for n in stage_launches]
    rep = {"workload": name, "batch": w.batch, "total_q": w.total_q, "total_kv": w.total_kv,
           "max_kv_len": max(w.kv_lens), "top_k": w.top_k, "q_heads": w.n_q_heads,
           "kv_heads": w.n_kv_heads, "steps": steps, "warmup": warmup, "ms_per_step": ms,
           "tokens_per_s": w.total_q / (ms / 1e3), "workspace_bytes": ws_bytes,
           "fused_rows": fused_rows,
           "stages": stage_report(w, sm, sn, peaks, gather, fused_rows), "clocks": clocks.summary()}
    del inputs, ws, out
    torch.cuda.empty_cache()
    return rep


# ----------------------------------------------------------------------------- CPU oracle

def cpu_oracle_sample(w, target_seconds: float, rows_per_call=None, offset=0):
    """Time the CPU oracle (as it stands) on evenly spaced query rows of workload w."""
    import concurrent.futures as cf

    import dsa_synth as S
    import oracle as O

    host = _host_inputs_threaded(w)
    orc = O.Oracle.for_workload(w, host)
    threads = O.hardware_threads()
    total = w.total_q

    def rows_for(n, off):
        step = max(1, total // n)
        return [min(total - 1, off % step + i * step) for i in range(n)]

    if rows_per_call is None:  # pilot, then size the sample to the target time
        pilot = rows_for(max(threads, 8), 17)
        t = time.perf_counter()
        orc.layer_rows(pilot, nthreads=threads)
        per_row = (time.perf_counter() - t) / len(pilot)
        n = int(max(threads, min(total, target_seconds / max(per_row, 1e-6))))
    else:
        n = rows_per_call
    rows = rows_for(n, offset)
    t = time.perf_counter()
    orc.layer_rows(rows, nthreads=threads)
    secs = time.perf_counter() - t
    return {"rows": len(rows), "seconds": secs, "threads": threads, "orc": orc,
            "first_rows": rows[:4]}


def _host_inputs_threaded(w):
    """Host copies of the workload (threaded generation; not part of any timing)."""
    import concurrent.futures as cf

    import dsa_synth as S

    Hi, Di, Hq, Hkv, d = w.n_idx_heads, w.idx_dim, w.n_q_heads, w.n_kv_heads, w.head_dim
    tq, tk = w.total_q, w.total_kv
    specs = {
        "q_idx": (tq * Hi * Di, w.idx_family, S.T_Q_IDX, w.qkv_scale, (tq, Hi, Di)),
        "k_idx": (tk * Hi * Di, w.idx_family, S.T_K_IDX, w.qkv_scale, (tk, Hi, Di)),
        "q": (tq * Hq * d, S.NORMAL, S.T_Q, w.qkv_scale, (tq, Hq, d)),
        "k": (tk * Hkv * d, S.NORMAL, S.T_K, w.qkv_scale, (tk, Hkv, d)),
        "v": (tk * Hkv * d, S.NORMAL, S.T_V, w.qkv_scale, (tk, Hkv, d)),
        "gate": (tq * Hq * d, S.NORMAL, S.T_GATE, 1.0, (tq, Hq, d)),
    }
    out = {}
    chunk = 1 << 22
    with cf.ThreadPoolExecutor(max_workers=os.cpu_count() or 4) as ex:
        for name, (n, fam, tid, scale, shp) in specs.items():
            arr = np.empty(n, np.uint16)
            futs = []
            for s in range(0, n, chunk):
                c = min(chunk, n - s)
                futs.append(ex.submit(S.lib().synth_fill_bf16_host, arr[s:].ctypes.data, c, fam,
                                      w.seed, tid, s, scale))
            for f in futs:
                f.result()
            out[name] = arr.reshape(shp)
    out["w"] = S.host_f32(Hi, w.w_family, w.seed, S.T_W, 0)
    out["q_offsets"] = w.q_offsets
    out["kv_offsets"] = w.kv_offsets
    return out


def run_reference(args, rank, world):
    """The reference arm: the CPU oracle on bounded samples of the same workload."""
    if rank != 0:
        return
    import dsa_synth as S
    import oracle as O

    w = S.workload(args.workload)
    host = _host_inputs_threaded(w)
    orc = O.Oracle.for_workload(w, host)
    threads = O.hardware_threads()
    total = w.total_q
    per_step = max(threads, 16)
    stride = max(1, total // per_step)
    for s in range(args.warmup):
        orc.layer_rows([min(total - 1, (s * 7) % stride + i * stride) for i in range(per_step)],
                       nthreads=threads)
    t = time.perf_counter()
    for s in range(args.steps):
        orc.layer_rows([min(total - 1, (s * 13 + 5) % stride + i * stride)
                        for i in range(per_step)], nthreads=threads)
    secs = time.perf_counter() - t
    rows = per_step * args.steps
    value = rows / secs
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs * 1e3 / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "config": {"workload": w.name, "batch": w.batch, "seq_len": w.kv_lens[0],
                   "top_k": w.top_k, "parallelism": "cpu"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": f"{per_step} evenly spaced query rows of {total} per step "
                                   f"(full layer per row: scores, Top-K, gated attention)"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- main

def main():
    args = parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    import datetime

    import torch
    import torch.distributed as dist
    if world > 1:
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    res = run_ours(args, rank, world, local_rank)
    decode = None
    if world == 1 and not args.no_decode:
        decode = run_decode_side(args)
    gather = None
    if rank == 0 and not args.no_peaks:
        from indexer_top_gated_b200 import peaks as P
        gather = P.gather_peaks(torch.cuda.get_device_properties(local_rank).multi_processor_count)
    extra = []
    if world == 1:
        for name in [x for x in args.also.split(",") if x]:
            extra.append(run_extra_workload(name, gather))
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    w = res["w"]
    peaks, peak_src = load_peaks()
    steps = args.steps
    stage_ms = [m / steps for m in res["stage_ms"]]          # per step
    stage_n = [max(1, n // steps) for n in res["stage_launches"]]
    stages = stage_report(w, stage_ms, stage_n, peaks, gather, res["fused_rows"])
    dom = int(np.argmax(stage_ms))
    alg = algorithmic(w)
    roof = {"kernel": stages[dom]["kernel"], "bound": stages[dom]["bound"],
            "achieved": stages[dom]["achieved"], "peak": stages[dom]["peak"],
            "unit": stages[dom]["unit"], "frac": stages[dom]["frac"],
            "traffic": stages[dom].get("dram_traffic_per_launch"),
            "algorithmic_per_launch": (alg["attn_bytes"] if dom == 2 else alg["topk_bytes"]
                                       if dom == 1 else alg["idx_flops"]) / stage_n[dom]}
    if dom == 2:
        roof["peak_source"] = ("measured live in this run: " + gather["l2"]["best"]
                               if gather else "not measured (--no-peaks)")
        roof["dram"] = {"achieved": stages[2]["dram_gbs"], "peak": peaks["hbm_gbs"],
                        "frac": stages[2]["dram_frac"], "unit": "GB/s",
                        "peak_source": f"{peak_src} (hbm_gbs)"}
    else:
        roof["peak_source"] = f"{peak_src} ({'hbm_gbs' if dom else 'bf16_tflops_sustained'})"
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        c = cpu_oracle_sample(w, args.cpu_seconds)
        cpu = {"value": c["rows"] / c["seconds"], "unit": "tokens/s", "cores": c["threads"],
               "kind": "oracle",
               "sample": f"{c['rows']} evenly spaced query rows of {w.total_q} (first {c['first_rows']}), "
                         f"full layer per row (fp64 scores, sort-based Top-K, fp64 gated attention), "
                         f"{c['seconds']:.1f} s wall"}
    line = {
        "metric": METRIC, "value": res["value"], "unit": "tokens/s", "n_gpus": world,
        "steps": steps, "warmup": args.warmup, "ms_per_step": res["ms_total"] / steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "seq_len": w.kv_lens[0],
                   "top_k": w.top_k, "q_heads": w.n_q_heads, "kv_heads": w.n_kv_heads,
                   "head_dim": w.head_dim, "idx_heads": w.n_idx_heads, "idx_dim": w.idx_dim,
                   "idx_dtype": w.idx_dtype,
                   "parallelism": (f"dp{world} (a batch of {world} copies of the workload, "
                                   f"whole sequences dealt to ranks by cost; no collective "
                                   f"on the data path)" if world > 1 else "dp1"),
                   "l2": l2_note(w),
                   "workspace_bytes": res["ws_bytes"],
                   **({"seq_stride": args.seq_stride} if args.seq_stride > 1 else {})},
        "roofline": roof,
        "stages": stages,
        "cpu_baseline": cpu,
        "e2e": res["e2e"],
        "gpu_launches": res["launches"],
        "clocks": res["clocks"],
        "decode": decode,
        "gather_peaks": gather,
        "workloads": extra,
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
