"""The seeded input generator: determinism, shapes and distributions."""
import numpy as np
import pytest
import torch

from gated_deltanet_recurrent_sigmoid_b200 import workloads as wl


def test_bf16_rounding_matches_torch_round_to_nearest_even():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(10000).astype(np.float32),
                        np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -1 - 2 ** -8, 0.0, -0.0,
                                  3.0e38, 1e-40], dtype=np.float32)])
    ours = wl.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    back = wl.bf16_bits_to_f32(ours)
    assert np.array_equal(back, torch.from_numpy(ours.view(np.int16)).view(torch.bfloat16).float().numpy())


@pytest.mark.parametrize("spec", [wl.TINY, wl.SPEC_B128_T4, wl.sweep_spec(64)], ids=lambda s: s.name)
def test_generate_is_deterministic(spec):
    a, b = wl.generate(spec), wl.generate(spec)
    for f in ("q", "k", "v", "a", "b", "A_log", "dt_bias", "state_pool", "state_indices"):
        assert np.array_equal(getattr(a, f), getattr(b, f)), f


def test_decode_b512_shapes_and_padding():
    w = wl.generate(wl.DECODE_B512)
    assert w.q.shape == (512, 1, 4, 128) and w.v.shape == (512, 1, 8, 128)
    assert w.state_pool.shape == (1024, 8, 128, 128) and w.state_pool.dtype == np.float32
    idx = w.state_indices
    assert (idx == -1).sum() == 25
    live = idx[idx >= 0]
    assert len(np.unique(live)) == len(live) and live.max() < 1024
    assert abs(float(w.state_pool[:64].std()) - 0.1) < 1e-3
    assert np.all((w.A_log >= 0) & (w.A_log <= np.log(16) + 1e-6))
    assert np.all(np.abs(w.dt_bias) <= 1)
    qf = wl.bf16_bits_to_f32(w.q)
    assert abs(qf.mean()) < 0.02 and abs(qf.std() - 1) < 0.02


def test_sweep_lengths_and_cu_seqlens():
    w = wl.generate(wl.sweep_spec(256))
    lens = w.seq_lens
    assert w.cu_seqlens[0] == 0 and np.all(np.diff(w.cu_seqlens) >= 1)
    assert lens.min() >= 1 and lens.max() <= 64 and w.T_tot == lens.sum()
    assert (w.state_indices == -1).sum() == 25
    assert w.state_pool.shape[0] == 512


def test_spec_decode_uniform_stride():
    w = wl.generate(wl.SPEC_B128_T4)
    assert np.array_equal(w.cu_seqlens, np.arange(0, 513, 4, dtype=np.int32))
    assert w.q.shape == (512, 4, 128)


def test_algorithmic_bytes_decode_b512():
    w = wl.generate(wl.DECODE_B512)
    P = int((w.state_indices >= 0).sum())
    assert P == 487
    state = 2 * 487 * 8 * 128 * 128 * 4
    acts = 487 * (2 * 4 * 128 + 8 * 128 + 16) * 2 + 512 * 8 * 128 * 2 + 64 + 2048
    assert wl.algorithmic_bytes(w) == state + acts
