"""The unfused pair (gating kernel; recurrence with precomputed g, beta) and
fp32 activations, through the C ABI, against the oracle.

Tolerances as for the fused path: state max abs 1e-4, output
1e-2 + 1e-2 |o_ref|; gates (fp32 g) within 1e-6 relative of fp64.
"""
import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_recurrent_sigmoid_b200 import binding
from gated_deltanet_recurrent_sigmoid_b200 import workloads as wl
from gpu_helpers import assert_out_close, assert_state_close, bf16_tensor, to_device
from helpers import BF16_NEG_INF, BF16_POS_INF

pytestmark = pytest.mark.gpu

L2 = binding.L2NORM_QK
INTER = binding.WRITE_INTERMEDIATE
TILES = [(8, 8), (16, 16), (32, 16), (32, 32), (64, 16), (64, 32)]


@pytest.fixture(scope="module", autouse=True)
def _lib(gdn_lib):
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return gdn_lib


def fp32_inputs(w, seed):
    """fp32 activations that are NOT bf16 values: the bf16 inputs plus a small
    fp32 perturbation (the same arrays go to both sides)."""
    rng = np.random.default_rng(seed)
    f = {}
    for n in ("q", "k", "v", "a", "b"):
        x = wl.bf16_bits_to_f32(getattr(w, n))
        f[n] = (x + rng.standard_normal(x.shape).astype(np.float32) * np.float32(1e-3)).astype(np.float32)
    return f


def gates_of(w):
    g, beta = oracle.gating(w.a, w.b, w.A_log, w.dt_bias)
    return g.astype(np.float32), beta.astype(np.float32)


def run_recurrent(w, g, beta, acts=None, beta_dtype=torch.float32, flags=L2, tile=(0, 0)):
    d = to_device(w)
    if acts is not None:
        for n in ("q", "k", "v"):
            d[n] = torch.from_numpy(acts[n]).cuda()
        d["out"] = torch.full(w.v.shape, float("nan"), device="cuda")
    lead = d["q"].shape[:-2]
    gt = torch.from_numpy(g).cuda().view(*lead, w.spec.HV)
    bt = torch.from_numpy(beta).cuda().view(*lead, w.spec.HV).to(beta_dtype)
    inter = None
    if flags & INTER:
        inter = torch.full((w.T_tot, w.spec.HV, 128, 128), float("nan"), device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    binding.recurrent_update(d["q"], d["k"], d["v"], gt, bt, d["state_pool"], d["state_indices"], d["cu_seqlens"],
                             d["out"], flags=flags, intermediate_states=inter, device_status=status,
                             tile_v=tile[0], tile_rows=tile[1])
    torch.cuda.synchronize()
    return d, int(status.item()), inter


def compare(w, d, inter, o_ref, s_ref, i_ref, flags):
    assert_out_close(d["out"].float().cpu().numpy(), o_ref)
    live = w.state_indices[(w.state_indices >= 0) & (w.seq_lens > 0)]
    pool = d["state_pool"].cpu().numpy()
    assert_state_close(pool[live], s_ref[live])
    untouched = np.ones(w.spec.num_slots, bool)
    untouched[live] = False
    assert np.array_equal(pool[untouched], w.state_pool[untouched])
    if flags & INTER:
        it = inter.cpu().numpy()
        nan_ref = np.isnan(i_ref)
        assert np.array_equal(np.isnan(it), nan_ref)
        assert_state_close(it[~nan_ref], i_ref[~nan_ref], "intermediate")


SPECS = [wl.TINY, wl.shrink(wl.DECODE_B512, 40), wl.shrink(wl.SPEC_B128_T4, 20), wl.shrink(wl.sweep_spec(64), 10)]


@pytest.mark.parametrize("spec", SPECS, ids=lambda s: s.name)
@pytest.mark.parametrize("tile", [(0, 0)] + TILES, ids=lambda t: f"tile{t[0]}x{t[1]}")
def test_recurrent_update_with_given_gates_matches_oracle(spec, tile):
    w = wl.generate(spec)
    g, beta = gates_of(w)
    flags = L2 | (INTER if spec.intermediate else 0)
    d, status, inter = run_recurrent(w, g, beta, flags=flags, tile=tile)
    ost, o_ref, s_ref, i_ref = oracle.update(w.q, w.k, w.v, None, None, None, None, w.state_pool,
                                             w.state_indices, w.cu_seqlens, flags=flags, g=g, beta=beta)
    assert status == ost == 0
    compare(w, d, inter, o_ref, s_ref, i_ref, flags)


def test_recurrent_update_bf16_beta():
    w = wl.generate(wl.shrink(wl.SPEC_B128_T4, 16))
    g, beta = gates_of(w)
    beta_bf16 = wl.bf16_bits_to_f32(wl.f32_to_bf16_bits(beta))      # what the kernel will read
    d, status, inter = run_recurrent(w, g, beta, beta_dtype=torch.bfloat16, flags=L2 | INTER)
    ost, o_ref, s_ref, i_ref = oracle.update(w.q, w.k, w.v, None, None, None, None, w.state_pool,
                                             w.state_indices, w.cu_seqlens, flags=L2 | INTER, g=g, beta=beta_bf16)
    assert status == ost == 0
    compare(w, d, inter, o_ref, s_ref, i_ref, L2 | INTER)


@pytest.mark.parametrize("spec", SPECS, ids=lambda s: s.name)
@pytest.mark.parametrize("tile", [(0, 0), (16, 16), (64, 32)], ids=lambda t: f"tile{t[0]}x{t[1]}")
def test_fp32_activations_fused_match_oracle(spec, tile):
    w = wl.generate(spec)
    f = fp32_inputs(w, 3)
    flags = L2 | (INTER if spec.intermediate else 0)
    d = to_device(w)
    for n in ("q", "k", "v", "a", "b"):
        d[n] = torch.from_numpy(f[n]).cuda()
    d["out"] = torch.full(w.v.shape, float("nan"), device="cuda")
    inter = torch.full((w.T_tot, spec.HV, 128, 128), float("nan"), device="cuda") if flags & INTER else None
    binding.decode_update(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"], d["dt_bias"], d["state_pool"],
                          d["state_indices"], d["cu_seqlens"], d["out"], flags=flags, intermediate_states=inter,
                          tile_v=tile[0], tile_rows=tile[1])
    torch.cuda.synchronize()
    _, o_ref, s_ref, i_ref = oracle.update(f["q"], f["k"], f["v"], f["a"], f["b"], w.A_log, w.dt_bias,
                                           w.state_pool, w.state_indices, w.cu_seqlens, flags=flags)
    compare(w, d, inter, o_ref, s_ref, i_ref, flags)


def test_fp32_activations_given_gates_match_oracle():
    w = wl.generate(wl.shrink(wl.SPEC_B128_T4, 16))
    f = fp32_inputs(w, 4)
    g, beta = gates_of(w)
    d, status, inter = run_recurrent(w, g, beta, acts=f, flags=L2 | INTER)
    _, o_ref, s_ref, i_ref = oracle.update(f["q"], f["k"], f["v"], None, None, None, None, w.state_pool,
                                           w.state_indices, w.cu_seqlens, flags=L2 | INTER, g=g, beta=beta)
    compare(w, d, inter, o_ref, s_ref, i_ref, L2 | INTER)


@pytest.mark.parametrize("beta_dtype", [torch.float32, torch.bfloat16], ids=["beta_f32", "beta_bf16"])
@pytest.mark.parametrize("ab_f32", [False, True], ids=["ab_bf16", "ab_f32"])
def test_gating_kernel_matches_oracle(beta_dtype, ab_f32):
    w = wl.generate(wl.sweep_spec(64))
    a_np, b_np = w.a.copy(), w.b.copy()
    a_np[:7, 0] = BF16_NEG_INF                                  # softplus(-inf) = 0
    a_np[7:14, 1] = wl.f32_to_bf16_bits(np.full(7, 30.0, np.float32))   # threshold branch
    b_np[:5, 2], b_np[5:10, 3] = BF16_POS_INF, BF16_NEG_INF
    if ab_f32:
        a_in, b_in = wl.bf16_bits_to_f32(a_np), wl.bf16_bits_to_f32(b_np)
        a_t, b_t = torch.from_numpy(a_in).cuda(), torch.from_numpy(b_in).cuda()
    else:
        a_in, b_in = a_np, b_np
        a_t, b_t = bf16_tensor(a_np), bf16_tensor(b_np)
    T, HV = w.T_tot, w.spec.HV
    g_t = torch.full((T, HV), float("nan"), device="cuda")
    beta_t = torch.full((T, HV), float("nan"), device="cuda", dtype=beta_dtype)
    binding.gating(torch.from_numpy(w.A_log).cuda(), a_t, torch.from_numpy(w.dt_bias).cuda(), b_t, g_t, beta_t)
    torch.cuda.synchronize()
    g_ref, beta_ref = oracle.gating(a_in, b_in, w.A_log, w.dt_bias)
    g = g_t.cpu().numpy().astype(np.float64)
    np.testing.assert_allclose(g, g_ref, rtol=2e-6, atol=0)
    bt = beta_t.float().cpu().numpy().astype(np.float64)
    tol = 1e-6 if beta_dtype == torch.float32 else 2 ** -8
    np.testing.assert_allclose(bt, beta_ref, rtol=tol, atol=1e-7)
    assert np.all(g[:7, 0] == 0) and np.all(bt[:5, 2] == 1) and np.all(bt[5:10, 3] == 0)


def test_unfused_pipeline_matches_fused_update():
    """GPU gating then GPU recurrence == the fused GPU update (the pair's g is
    rounded to fp32 in between, so within tolerance rather than bitwise)."""
    spec = wl.shrink(wl.SPEC_B128_T4, 24)
    w = wl.generate(spec)
    fused = to_device(w)
    binding.decode_update(fused["q"], fused["k"], fused["v"], fused["a"], fused["b"], fused["A_log"],
                          fused["dt_bias"], fused["state_pool"], fused["state_indices"], fused["cu_seqlens"],
                          fused["out"])
    d = to_device(w)
    g = torch.empty(w.T_tot, spec.HV, device="cuda")
    beta = torch.empty(w.T_tot, spec.HV, device="cuda")
    binding.gating(d["A_log"], d["a"], d["dt_bias"], d["b"], g, beta)
    binding.recurrent_update(d["q"], d["k"], d["v"], g, beta, d["state_pool"], d["state_indices"], d["cu_seqlens"],
                             d["out"])
    torch.cuda.synchronize()
    assert (d["state_pool"] - fused["state_pool"]).abs().max().item() <= 1e-5
    assert (d["out"].float() - fused["out"].float()).abs().max().item() <= 2e-2


def test_pipelined_schedule_rejects_unbuilt_modes():
    w = wl.generate(wl.TINY)
    d = to_device(w)
    g, beta = gates_of(w)
    gt = torch.from_numpy(g).cuda().view(4, 1, 4)
    bt = torch.from_numpy(beta).cuda().view(4, 1, 4)
    with pytest.raises(binding.GdnError) as e:
        binding.recurrent_update(d["q"], d["k"], d["v"], gt, bt, d["state_pool"], d["state_indices"], None, d["out"],
                                 schedule=binding.SCHEDULE_PIPELINED)
    assert e.value.status == binding.ERR_UNSUPPORTED
