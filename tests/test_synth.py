"""The seeded input generator: determinism, sub-range consistency and value families."""
import numpy as np
import torch

import dsa_synth as S


def test_subrange_fill_matches_whole_fill():
    whole = S.host_bf16(5000, S.NORMAL, 7, S.T_Q, 0, S.INV_SQRT_128)
    part = S.host_bf16(1234, S.NORMAL, 7, S.T_Q, 2000, S.INV_SQRT_128)
    np.testing.assert_array_equal(whole[2000:3234], part)
    g = S.host_bf16(3000, S.GRID, 7, S.T_K_IDX)
    np.testing.assert_array_equal(g[100:200], S.host_bf16(100, S.GRID, 7, S.T_K_IDX, 100))


def test_streams_differ_by_seed_and_tensor():
    a = S.host_bf16(256, S.NORMAL, 0, S.T_Q, 0, 1.0)
    assert not np.array_equal(a, S.host_bf16(256, S.NORMAL, 1, S.T_Q, 0, 1.0))
    assert not np.array_equal(a, S.host_bf16(256, S.NORMAL, 0, S.T_K, 0, 1.0))


def test_grid_values_and_e4m3_codes():
    g = S.bf16_bits_to_f32(S.host_bf16(90000, S.GRID, 3, S.T_Q_IDX))
    vals, counts = np.unique(g, return_counts=True)
    np.testing.assert_array_equal(vals, np.arange(-4, 5) / 8.0)
    assert counts.min() > 9000  # near-uniform over the 9 values
    codes = S.host_e4m3_grid(90000, 3, S.T_Q_IDX)
    dec = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    np.testing.assert_array_equal(dec, g)  # same draws, same values in both encodings


def test_bf16_rounding_matches_torch():
    x = np.random.default_rng(0).normal(size=100000).astype(np.float32) * 3
    ours = S.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)
    # the C generator rounds the same way: its bf16 normal draws equal the rounding of
    # its own fp32 draws
    f32 = S.host_f32(20000, S.NORMAL, 5, S.T_V, 0, S.INV_SQRT_128)
    np.testing.assert_array_equal(S.host_bf16(20000, S.NORMAL, 5, S.T_V, 0, S.INV_SQRT_128),
                                  S.f32_to_bf16_bits(f32))


def test_normal_moments():
    x = S.host_f32(400000, S.NORMAL, 11, S.T_GATE, 0, 1.0).astype(np.float64)
    assert abs(x.mean()) < 0.01
    assert abs(x.var() - 1.0) < 0.01
    assert np.abs(x).max() <= 6.0


def test_weights_family():
    w = S.host_f32(3000, S.WEIGHT, 0, S.T_W)
    assert set(np.unique(w).tolist()) == {0.25, 0.5, 1.0}


def test_workload_shapes():
    w = S.workload("mixed_serving")
    assert w.batch == 264 and w.q_lens[:8] == [8192] * 8 and w.q_lens[8:] == [1] * 256
    assert all(8192 <= L <= 262144 + 8192 for L in w.kv_lens[:8])
    assert all(4096 <= L <= 262144 for L in w.kv_lens[8:])
    c4 = S.workload("prefill_t131072_needles")
    assert len(c4.needle_pos) == 16 and max(c4.needle_pos) < 131072 - 128
    assert c4.needle_rows == list(range(131072 - 128, 131072))
    # needle score 42 * 1/4 = 10.5 per head
    u, key = c4.needle_u(), c4.needle_key_row()
    np.testing.assert_array_equal((u * key).sum(1), [10.5] * 4)
