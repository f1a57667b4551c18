"""The attention's general gather addressing -- the form a K or V cache array larger than
64 GiB takes -- gives the same output, bit for bit, as the 32-bit offsets that test-sized
caches use (addressing changes no arithmetic).  The library reads DSA_ATTN_ADDR_ROWS once, so
the general form runs in a child process with the variable set; the parent runs the default
form and also checks the child's output against the oracle.
"""
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import dsa_synth as S
import oracle as O
from tests import parity as PT

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# KV heads per CTA and query-head tiles: (2, 1), (2, 2), (1, 1)
CASES = {"gqa8": dict(Hq=32, Hkv=4), "gqa16": dict(Hq=32, Hkv=2), "one_kv": dict(Hq=8, Hkv=1)}


def run_case(case: str):
    """Attention over the oracle's selection for a small ragged workload; returns the output
    as int16 bits and the oracle's reference."""
    import indexer_top_gated_b200 as dsa
    cfg = CASES[case]
    w = S.Workload("custom", [40, 1, 90], [300, 50, 90], top_k=96, n_q_heads=cfg["Hq"],
                   n_kv_heads=cfg["Hkv"], n_idx_heads=4, idx_dtype="bf16",
                   qkv_scale=S.INV_SQRT_128, gate=True, seed=3)
    host = S.make_host_inputs(w)
    dev = {}
    for k, v in host.items():
        if k in ("q_offsets", "kv_offsets"):
            dev[k] = torch.from_numpy(v.astype(np.int32)).cuda()
        elif v.dtype == np.uint16:
            dev[k] = torch.from_numpy(v.view(np.int16)).cuda().view(torch.bfloat16)
        else:
            dev[k] = torch.from_numpy(v).cuda()
    idx_ref, out_ref, _ = O.Oracle.for_workload(w, host).layer_rows(range(w.total_q))
    out = torch.zeros((w.total_q, w.n_q_heads, w.head_dim), dtype=torch.bfloat16, device="cuda")
    rg = dsa.ragged(dev["q_offsets"], dev["kv_offsets"], w.q_lens, w.kv_lens)
    dsa.dsa_sparse_attn_gated(dsa.workload_shape(w), rg, dev["q"], dev["k"], dev["v"],
                              torch.from_numpy(idx_ref).cuda(), w.top_k, 0, w.total_q,
                              dev["gate"], out)
    torch.cuda.synchronize()
    assert dsa.dsa_device_status(clear=True) == 0
    return out.view(torch.int16).cpu().numpy(), out_ref


CHILD = """
import sys
import numpy as np
sys.path.insert(0, {root!r})
from tests.test_gpu_addr import run_case
np.save({path!r}, run_case({case!r})[0])
"""


@pytest.mark.parametrize("case", sorted(CASES))
def test_general_gather_addressing_matches_32bit_offsets(case, tmp_path):
    path = str(tmp_path / "out.npy")
    env = dict(os.environ, DSA_ATTN_ADDR_ROWS="1")
    r = subprocess.run([sys.executable, "-c", CHILD.format(root=ROOT, path=path, case=case)],
                       env=env, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    general = np.load(path)
    default, ref = run_case(case)
    np.testing.assert_array_equal(general, default)
    got = PT.bf16_tensor_to_f64(torch.from_numpy(general).view(torch.bfloat16))
    PT.assert_close(got, ref, case + " (general addressing)")
