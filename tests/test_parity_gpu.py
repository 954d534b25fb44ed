"""CUDA path (through the C ABI) against the CPU oracle on seeded inputs.

Tolerances, fixed for this path: the fp32 state within max abs 1e-4 of the
fp64 oracle; the bf16 output within 1e-2 + 1e-2 |o_ref|; slot handling,
padding, untouched memory and status bits exact.
"""
import dataclasses
import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_recurrent_sigmoid_b200 import binding
from gated_deltanet_recurrent_sigmoid_b200 import workloads as wl
from gpu_helpers import (assert_out_close, assert_state_close, bf16_tensor, oracle_chain, oracle_on, out_as_f32,
                         run_gpu, run_oracle, sample_subproblem, to_device, workload_arrays)
from helpers import BF16_NEG_INF, BF16_POS_INF, bf16, random_problem

pytestmark = pytest.mark.gpu

L2 = binding.L2NORM_QK
INTER = binding.WRITE_INTERMEDIATE


@pytest.fixture(scope="module", autouse=True)
def _lib(gdn_lib):
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return gdn_lib


PER_TILE = binding.SCHEDULE_PER_TILE
PIPELINED = binding.SCHEDULE_PIPELINED
# (schedule, V-tile width, rows per thread) of every kernel the library can launch
KERNELS = [(PER_TILE, 16, 16), (PER_TILE, 32, 16), (PER_TILE, 32, 32), (PER_TILE, 64, 16), (PER_TILE, 64, 32),
           (PIPELINED, 0, 0), (PER_TILE, 8, 8)]
KERNEL_IDS = ["tile16x16", "tile32x16", "tile32x32", "tile64x16", "tile64x32", "pipelined", "tile8x8"]
# the library's two default tiles and the pipelined schedule
MAIN = [KERNELS[0], KERNELS[4], KERNELS[5]]
MAIN_IDS = ["tile16x16", "tile64x32", "pipelined"]


def kw_of(kernel):
    return dict(schedule=kernel[0], tile_v=kernel[1], tile_rows=kernel[2])


def check_full(w, flags=L2, tile_v=0, scale=None, schedule=binding.SCHEDULE_AUTO, tile_rows=0):
    """Whole-problem comparison: outputs, every pool slot, intermediates."""
    inter = bool(flags & INTER)
    d, status, inter_t = run_gpu(w, flags=flags, inter=inter, tile_v=tile_v, scale=scale, schedule=schedule,
                                 tile_rows=tile_rows)
    ostatus, o_ref, s_ref, i_ref = run_oracle(w, flags=flags, scale=scale)
    assert status == ostatus
    assert_out_close(out_as_f32(d["out"]), o_ref)
    pool = d["state_pool"].cpu().numpy()
    touched = np.zeros(w.spec.num_slots, bool)
    live = w.state_indices[(w.state_indices >= 0) & (w.seq_lens > 0)]
    if not flags & binding.NO_FINAL_WRITEBACK:
        touched[live] = True
    assert np.array_equal(pool[~touched], w.state_pool[~touched]), "untouched slots changed"
    if touched.any():
        assert_state_close(pool[touched], s_ref[touched])
    if inter:
        it = inter_t.cpu().numpy()
        nan_ref = np.isnan(i_ref)
        assert np.array_equal(np.isnan(it), nan_ref), "intermediate rows written differ"
        assert_state_close(it[~nan_ref], i_ref[~nan_ref], "intermediate")
    return d


SMALL = [
    wl.TINY,
    wl.shrink(wl.DECODE_B512, 40),
    wl.shrink(wl.FULLHEAD_B256, 10),
    wl.shrink(wl.SPEC_B128_T4, 24),
    wl.shrink(wl.sweep_spec(64), 12),
]


@pytest.mark.parametrize("spec", SMALL, ids=lambda s: s.name)
@pytest.mark.parametrize("kernel", KERNELS, ids=KERNEL_IDS)
def test_small_configs_match_oracle(spec, kernel):
    w = wl.generate(spec)
    flags = L2 | (INTER if spec.intermediate else 0)
    check_full(w, flags=flags, **kw_of(kernel))


@pytest.mark.parametrize("spec", [wl.TINY, wl.SPEC_B128_T4, wl.sweep_spec(1), wl.sweep_spec(8),
                                  wl.sweep_spec(64)], ids=lambda s: s.name)
@pytest.mark.parametrize("kernel", [(binding.SCHEDULE_AUTO, 0, 0), KERNELS[5]], ids=["default", "pipelined"])
def test_full_size_configs_match_oracle(spec, kernel):
    """Full-size configurations the oracle finishes in seconds, compared whole."""
    w = wl.generate(spec)
    check_full(w, flags=L2 | (INTER if spec.intermediate else 0), **kw_of(kernel))


def sampled_check(spec, n_sample, seed=0, schedule=binding.SCHEDULE_AUTO, tile_v=0, tile_rows=0):
    """Full-size problem in the benchmark's launch configuration; the oracle
    recomputes a sample of sequences (always including padded ones and the
    longest), everything else is checked through properties."""
    w = wl.generate(spec)
    d = to_device(w)
    pool_before = d["state_pool"].clone()
    d, status, _ = run_gpu(w, d=d, schedule=schedule, tile_v=tile_v, tile_rows=tile_rows)
    assert status == 0
    rng = np.random.default_rng(seed)
    N = spec.N
    pads = np.flatnonzero(w.state_indices < 0)
    longest = np.argsort(-w.seq_lens, kind="stable")[:4]
    seqs = np.unique(np.concatenate([rng.choice(N, size=min(n_sample, N), replace=False), pads[:4], longest]))
    arrays, rows, slots = sample_subproblem(w, seqs)
    ostatus, o_ref, s_ref, _ = oracle_on(arrays)
    assert ostatus == 0
    out = d["out"].view(w.T_tot, spec.HV, spec.V)
    assert_out_close(out[torch.from_numpy(rows).cuda()].float().cpu().numpy(), o_ref, "sampled out")
    live = slots >= 0
    got = d["state_pool"][torch.from_numpy(slots[live].astype(np.int64)).cuda()].cpu().numpy()
    assert_state_close(got, s_ref, "sampled state")
    # properties over the whole problem
    assert torch.isfinite(out.float()).all()
    pad_rows = torch.from_numpy(np_token_rows(w, pads)).cuda()
    if len(pads):
        assert (out[pad_rows].float() == 0).all()
    untouched = torch.ones(spec.num_slots, dtype=torch.bool, device="cuda")
    untouched[torch.from_numpy(w.state_indices[w.state_indices >= 0].astype(np.int64)).cuda()] = False
    assert torch.equal(d["state_pool"][untouched], pool_before[untouched])
    assert torch.isfinite(d["state_pool"][~untouched]).all()


def np_token_rows(w, seqs):
    from gpu_helpers import token_rows
    return token_rows(w, seqs)


def test_decode_b512_full_size_sampled():
    sampled_check(wl.DECODE_B512, 96)


def test_decode_b512_full_size_sampled_pipelined():
    sampled_check(wl.DECODE_B512, 48, schedule=PIPELINED)


def test_decode_b512_full_size_sampled_tile16():
    sampled_check(wl.DECODE_B512, 48, schedule=PER_TILE, tile_v=16, tile_rows=16)


def test_fullhead_b256_full_size_sampled():
    sampled_check(wl.FULLHEAD_B256, 48)


@pytest.mark.parametrize("N", [256, 1024])
def test_sweep_full_size_sampled(N):
    sampled_check(wl.sweep_spec(N), 48)


def test_chained_single_token_calls_match_multi_token_call():
    """A T-token call equals T single-token calls that carry the state."""
    w = wl.generate(wl.shrink(wl.SPEC_B128_T4, 16))
    d_all, _, _ = run_gpu(w)
    d = to_device(w)
    T = 4
    cu1 = torch.arange(w.spec.N + 1, dtype=torch.int32, device="cuda")
    outs = []
    for t in range(T):
        rows = torch.arange(w.spec.N, device="cuda") * T + t
        o = torch.empty(w.spec.N, w.spec.HV, w.spec.V, dtype=torch.bfloat16, device="cuda")
        binding.decode_update(d["q"][rows].contiguous(), d["k"][rows].contiguous(), d["v"][rows].contiguous(),
                              d["a"][rows].contiguous(), d["b"][rows].contiguous(), d["A_log"], d["dt_bias"],
                              d["state_pool"], d["state_indices"], cu1, o)
        outs.append(o)
    torch.cuda.synchronize()
    chained = torch.stack(outs, 1).reshape(d_all["out"].shape).float()
    assert (chained - d_all["out"].float()).abs().max().item() <= 2e-2
    assert (d["state_pool"] - d_all["state_pool"]).abs().max().item() <= 1e-5


def test_intermediate_states_equal_prefix_states():
    """inter[bos + t] equals the pool after a call over the first t+1 tokens."""
    w = wl.generate(wl.shrink(wl.SPEC_B128_T4, 8))
    tile = dict(schedule=PER_TILE, tile_v=16, tile_rows=16)       # same kernel for every call
    _, _, inter = run_gpu(w, flags=L2 | INTER, inter=True, **tile)
    T = 4
    for t in range(T):
        d = to_device(w)
        rows = (torch.arange(w.spec.N, device="cuda")[:, None] * T + torch.arange(t + 1, device="cuda")).reshape(-1)
        cu = torch.arange(0, w.spec.N * (t + 1) + 1, t + 1, dtype=torch.int32, device="cuda")
        o = torch.empty(len(rows), w.spec.HV, w.spec.V, dtype=torch.bfloat16, device="cuda")
        binding.decode_update(d["q"][rows].contiguous(), d["k"][rows].contiguous(), d["v"][rows].contiguous(),
                              d["a"][rows].contiguous(), d["b"][rows].contiguous(), d["A_log"], d["dt_bias"],
                              d["state_pool"], d["state_indices"], cu, o, **tile)
        torch.cuda.synchronize()
        idx = torch.from_numpy(w.state_indices.astype(np.int64)).cuda()
        got = inter.view(w.spec.N, T, w.spec.HV, 128, 128)[:, t]
        assert torch.equal(got, d["state_pool"][idx])


def test_kernels_agree():
    w = wl.generate(wl.shrink(wl.sweep_spec(64), 16))
    ref, _, _ = run_gpu(w, **kw_of(KERNELS[0]))
    for kernel in KERNELS[1:]:
        d, _, _ = run_gpu(w, **kw_of(kernel))
        assert (d["state_pool"] - ref["state_pool"]).abs().max().item() <= 1e-5
        assert (d["out"].float() - ref["out"].float()).abs().max().item() <= 2e-2


def test_deterministic():
    w = wl.generate(wl.shrink(wl.SPEC_B128_T4, 16))
    d1, _, i1 = run_gpu(w, flags=L2 | INTER, inter=True)
    d2, _, i2 = run_gpu(w, flags=L2 | INTER, inter=True)
    assert torch.equal(d1["out"], d2["out"]) and torch.equal(d1["state_pool"], d2["state_pool"])
    assert torch.equal(i1, i2)


def test_fixed_length_layout_equals_varlen():
    spec = wl.shrink(wl.SPEC_B128_T4, 12)
    w = wl.generate(spec)
    dv, _, _ = run_gpu(w)
    d = to_device(w)
    N, T = spec.N, 4
    r = lambda x: x.view(N, T, *x.shape[1:])
    binding.decode_update(r(d["q"]), r(d["k"]), r(d["v"]), r(d["a"]), r(d["b"]), d["A_log"], d["dt_bias"],
                          d["state_pool"], d["state_indices"], None, r(d["out"]))
    torch.cuda.synchronize()
    assert torch.equal(d["out"], dv["out"]) and torch.equal(d["state_pool"], dv["state_pool"])


def test_strided_views_of_packed_projections():
    """q, k, v as column slices of one packed projection row and a, b
    interleaved per value head give bit-identical results."""
    spec = wl.shrink(wl.sweep_spec(64), 10)
    w = wl.generate(spec)
    ref, _, _ = run_gpu(w)
    d = to_device(w)
    T, H, HV, K, V = w.T_tot, spec.H, spec.HV, spec.K, spec.V
    width = 2 * H * K + HV * V + 64
    packed = torch.zeros(T, width, dtype=torch.bfloat16, device="cuda")
    packed[:, :H * K] = d["q"].reshape(T, -1)
    packed[:, H * K:2 * H * K] = d["k"].reshape(T, -1)
    packed[:, 2 * H * K:2 * H * K + HV * V] = d["v"].reshape(T, -1)
    q = packed[:, :H * K].view(T, H, K)
    k = packed[:, H * K:2 * H * K].view(T, H, K)
    v = packed[:, 2 * H * K:2 * H * K + HV * V].view(T, HV, V)
    ba = torch.stack([d["b"], d["a"]], dim=-1).contiguous()          # [T, HV, 2]
    b, a = ba[..., 0], ba[..., 1]
    binding.decode_update(q, k, v, a, b, d["A_log"], d["dt_bias"], d["state_pool"], d["state_indices"],
                          d["cu_seqlens"], d["out"])
    torch.cuda.synchronize()
    ost, o_ref, s_ref, _ = run_oracle(w)
    assert ost == 0
    assert_out_close(out_as_f32(d["out"]), o_ref, "strided out")
    live = w.state_indices[w.state_indices >= 0]
    assert_state_close(d["state_pool"].cpu().numpy()[live], s_ref[live], "strided state")
    assert torch.equal(d["out"], ref["out"]) and torch.equal(d["state_pool"], ref["state_pool"])


def test_guard_bands_untouched():
    spec = wl.shrink(wl.SPEC_B128_T4, 8)
    w = wl.generate(spec)
    ref, _, iref = run_gpu(w, flags=L2 | INTER, inter=True)
    d = to_device(w)
    sentinel = -1024.0          # exact in bf16 and fp32
    S, HV = spec.num_slots, spec.HV
    pool_buf = torch.full((S + 2, HV, 128, 128), sentinel, device="cuda")
    pool_buf[1:-1] = d["state_pool"]
    out_buf = torch.full((w.T_tot + 2, HV, 128), sentinel, dtype=torch.bfloat16, device="cuda")
    inter_buf = torch.full((w.T_tot + 2, HV, 128, 128), sentinel, device="cuda")
    binding.decode_update(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"], d["dt_bias"], pool_buf[1:-1],
                          d["state_indices"], d["cu_seqlens"], out_buf[1:-1], intermediate_states=inter_buf[1:-1])
    torch.cuda.synchronize()
    for buf in (pool_buf, out_buf, inter_buf):
        assert (buf[0].float() == sentinel).all() and (buf[-1].float() == sentinel).all()
    assert torch.equal(pool_buf[1:-1], ref["state_pool"]) and torch.equal(out_buf[1:-1], ref["out"])
    assert torch.equal(inter_buf[1:-1], iref)


@pytest.mark.parametrize("kernel", MAIN, ids=MAIN_IDS)
def test_device_status_and_skipped_sequences(kernel):
    rng = np.random.default_rng(5)
    p = random_problem(rng, lens=[2, 1, 3, 2], H=2, HV=4, K=128, V=128, num_slots=8)
    p["state_indices"][1] = 8          # out of range
    p["state_indices"][3] = -7         # below -1
    spec = wl.WorkloadSpec("bad", N=4, H=2, HV=4, num_slots=8, seed=0, T=None)
    w = wl.Workload(spec, p["q"], p["k"], p["v"], p["a"], p["b"], p["A_log"], p["dt_bias"], p["state_pool"],
                    p["state_indices"], p["cu_seqlens"])
    d, status, _ = run_gpu(w, **kw_of(kernel))
    ostatus, o_ref, s_ref, _ = run_oracle(w)
    assert status == ostatus == oracle.BAD_SLOT
    assert_out_close(out_as_f32(d["out"]), o_ref)       # skipped rows stay NaN on both sides
    pool = d["state_pool"].cpu().numpy()
    for i in (0, 2):
        s = p["state_indices"][i]
        assert_state_close(pool[s], s_ref[s])
    # bad cu_seqlens
    p["state_indices"] = rng.permutation(8)[:4].astype(np.int32)
    w2 = wl.Workload(spec, p["q"], p["k"], p["v"], p["a"], p["b"], p["A_log"], p["dt_bias"], p["state_pool"],
                     p["state_indices"], np.array([0, 2, 3, 6, 9], dtype=np.int32))   # last runs past T_tot
    d2, status2, _ = run_gpu(w2, **kw_of(kernel))
    ostatus2, o_ref2, _, _ = run_oracle(w2)
    assert status2 == ostatus2 == oracle.BAD_SEQLENS
    assert_out_close(out_as_f32(d2["out"]), o_ref2)


@pytest.mark.parametrize("kernel", MAIN, ids=MAIN_IDS)
def test_empty_sequences_all_padded_and_no_tokens(kernel):
    rng = np.random.default_rng(6)
    p = random_problem(rng, lens=[0, 3, 0, 1], H=1, HV=2, K=128, V=128, num_slots=6, pad=(3,))
    spec = wl.WorkloadSpec("empties", N=4, H=1, HV=2, num_slots=6, seed=0, T=None)
    w = wl.Workload(spec, p["q"], p["k"], p["v"], p["a"], p["b"], p["A_log"], p["dt_bias"], p["state_pool"],
                    p["state_indices"], p["cu_seqlens"])
    check_full(w, **kw_of(kernel))
    p2 = dict(p, state_indices=np.full(4, -1, dtype=np.int32))
    w2 = wl.Workload(spec, p2["q"], p2["k"], p2["v"], p2["a"], p2["b"], p2["A_log"], p2["dt_bias"],
                     p2["state_pool"], p2["state_indices"], p2["cu_seqlens"])
    check_full(w2, **kw_of(kernel))


@pytest.mark.parametrize("kernel", MAIN, ids=MAIN_IDS)
def test_no_final_writeback_and_l2norm_off(kernel):
    w = wl.generate(wl.shrink(wl.SPEC_B128_T4, 12))
    kw = kw_of(kernel)
    check_full(w, flags=L2 | INTER | binding.NO_FINAL_WRITEBACK, **kw)
    check_full(w, flags=INTER, **kw)
    check_full(w, flags=L2, scale=0.3, **kw)


@pytest.mark.parametrize("kernel", MAIN, ids=MAIN_IDS)
def test_special_gate_values_match_oracle(kernel):
    """Infinite a and b (decay 1, beta 0 or 1), A_log = -inf, softplus above
    its threshold and one-hot q/k: the same special cases that pin the oracle."""
    rng = np.random.default_rng(7)
    N, H, HV = 8, 2, 4
    p = random_problem(rng, N=N, T=1, H=H, HV=HV, K=128, V=128)
    p["a"] = np.where(rng.random((N, HV)) < 0.3, BF16_NEG_INF, bf16(24.0)).astype(np.uint16)
    p["b"] = np.where(rng.random((N, HV)) < 0.5, BF16_NEG_INF, BF16_POS_INF).astype(np.uint16)
    p["A_log"] = np.array([0.0, -np.inf, np.log(2.0), 1.0], dtype=np.float32)
    k = np.zeros((N, H, 128), np.float32)
    k[np.arange(N), 0, rng.integers(0, 128, N)] = 2.0
    r = rng.standard_normal((N, 128))
    k[:, 1] = r / np.linalg.norm(r, axis=1, keepdims=True)      # unit length, so L2-off stays O(1)
    p["k"] = wl.f32_to_bf16_bits(k)
    spec = wl.WorkloadSpec("special", N=N, H=H, HV=HV, num_slots=2 * N, seed=0, T=None)
    w = wl.Workload(spec, p["q"], p["k"], p["v"], p["a"], p["b"], p["A_log"], p["dt_bias"], p["state_pool"],
                    p["state_indices"], p["cu_seqlens"])
    check_full(w, **kw_of(kernel))
    check_full(w, flags=0, **kw_of(kernel))


def test_check_indices_flag_rejects_duplicates():
    w = wl.generate(wl.TINY)
    d = to_device(w)
    flags = L2 | binding.CHECK_INDICES
    binding.decode_update(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"], d["dt_bias"], d["state_pool"],
                          d["state_indices"], None, d["out"], flags=flags)
    dup = d["state_indices"].clone()
    dup[1] = dup[0]
    with pytest.raises(binding.GdnError) as e:
        binding.decode_update(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"], d["dt_bias"], d["state_pool"],
                              dup, None, d["out"], flags=flags)
    assert e.value.status == binding.ERR_INDICES


def test_validation_on_device_tensors():
    w = wl.generate(wl.TINY)
    d = to_device(w)
    args = lambda **kw: [kw.get(n, d[n]) for n in ("q", "k", "v", "a", "b", "A_log", "dt_bias", "state_pool",
                                                     "state_indices", "cu_seqlens", "out")]
    raw = torch.zeros(d["q"].numel() + 8, dtype=torch.bfloat16, device="cuda")
    q_off = raw[4:4 + d["q"].numel()].view(d["q"].shape)                      # 8-byte offset
    for kw, code in [(dict(q=q_off), binding.ERR_ALIGN), (dict(out=d["v"]), binding.ERR_ALIAS),
                     (dict(A_log=d["A_log"].double()), binding.ERR_DTYPE)]:
        with pytest.raises(binding.GdnError) as e:
            binding.decode_update(*args(**kw))
        assert e.value.status == code


@pytest.mark.parametrize("spec", [wl.TINY, wl.shrink(wl.SPEC_B128_T4, 16)], ids=lambda s: s.name)
def test_host_staged_decode_matches_device_call(spec):
    """One packed host-to-device copy, one launch, one copy back: same bits
    as the device-resident call."""
    w = wl.generate(spec)
    ref, _, _ = run_gpu(w)
    d = to_device(w)
    varlen = w.cu_seqlens is not None
    staged = binding.HostStagedDecode(d["q"].shape[:-2], spec.H, spec.HV, spec.K, spec.V, spec.N, d["A_log"],
                                      d["dt_bias"], d["state_pool"], varlen=varlen)
    for name in ("q", "k", "v", "a", "b", "state_indices", "cu_seqlens"):
        if d.get(name) is not None:
            getattr(staged, name).copy_(d[name].cpu())
    out = staged.step()
    torch.cuda.synchronize()
    ost, o_ref, s_ref, _ = run_oracle(w)
    assert ost == 0
    assert_out_close(out.float().numpy(), o_ref, "host-staged out")
    live = w.state_indices[w.state_indices >= 0]
    assert_state_close(d["state_pool"].cpu().numpy()[live], s_ref[live], "host-staged state")
    assert torch.equal(out, ref["out"].cpu())
    assert torch.equal(d["state_pool"], ref["state_pool"])
    assert staged.h2d_bytes >= sum(d[n].numel() * d[n].element_size() for n in ("q", "k", "v", "a", "b"))


@pytest.mark.parametrize("spec", [wl.TINY, wl.shrink(wl.SPEC_B128_T4, 16), wl.shrink(wl.DECODE_B512, 8)],
                         ids=lambda s: s.name)
@pytest.mark.parametrize("depth", [2, 3, 4])
def test_pipelined_host_decode_matches_device_calls(spec, depth):
    """Five host-fed steps with different inputs, copies overlapped across
    steps (2, 3 or 4 slots in flight): every step's host output and the final
    pool match five chained oracle calls (each reading the pool the previous
    one left), and are the bits of the same five steps run as
    device-resident calls, in order."""
    ws = [wl.generate(dataclasses.replace(spec, seed=spec.seed + 100 * n)) for n in range(5)]
    ref = to_device(ws[0])
    ref_outs = []
    for w in ws:                                   # same pool and parameters, successive inputs
        d = to_device(w)
        binding.decode_update(d["q"], d["k"], d["v"], d["a"], d["b"], ref["A_log"], ref["dt_bias"],
                              ref["state_pool"], d["state_indices"], d["cu_seqlens"], d["out"])
        ref_outs.append(d["out"].cpu())
    torch.cuda.synchronize()
    d0 = to_device(ws[0])
    varlen = ws[0].cu_seqlens is not None
    pipe = binding.PipelinedHostDecode(d0["q"].shape[:-2], spec.H, spec.HV, spec.K, spec.V, spec.N, d0["A_log"],
                                       d0["dt_bias"], d0["state_pool"], varlen=varlen, depth=depth)
    outs = []
    for w in ws:
        d = to_device(w)
        slot = pipe.inputs()
        for name in ("q", "k", "v", "a", "b", "state_indices", "cu_seqlens"):
            if d.get(name) is not None:
                getattr(slot, name).copy_(d[name].cpu())
        prev = pipe.step()
        if prev is not None:
            outs.append(prev.clone())
    outs.extend(o.clone() for o in pipe.finish())
    torch.cuda.synchronize()
    assert len(outs) == len(ref_outs)
    steps = [dict(workload_arrays(w), A_log=ws[0].A_log, dt_bias=ws[0].dt_bias) for w in ws]
    o_refs, s_ref = oracle_chain(steps, ws[0].state_pool)
    for n, (got, o_ref) in enumerate(zip(outs, o_refs)):
        assert_out_close(got.float().numpy(), o_ref, f"pipelined step {n} out")
    touched = np.unique(np.concatenate([w.state_indices[w.state_indices >= 0] for w in ws]))
    assert_state_close(d0["state_pool"].cpu().numpy()[touched], s_ref[touched], "pipelined final state")
    for got, exp in zip(outs, ref_outs):
        assert torch.equal(got, exp)
    assert torch.equal(d0["state_pool"], ref["state_pool"])


@pytest.mark.parametrize("kernel", MAIN, ids=MAIN_IDS)
def test_cuda_graph_capture_replays_the_same_update(kernel):
    """The launch is capturable: a graph of two chained updates replays to
    two chained oracle calls, and to the bits of the same two updates run
    eagerly."""
    w = wl.generate(wl.shrink(wl.SPEC_B128_T4, 12))
    kw = kw_of(kernel)
    eager = to_device(w)
    for _ in range(2):
        binding.decode_update(eager["q"], eager["k"], eager["v"], eager["a"], eager["b"], eager["A_log"],
                              eager["dt_bias"], eager["state_pool"], eager["state_indices"], eager["cu_seqlens"],
                              eager["out"], **kw)
    torch.cuda.synchronize()
    d = to_device(w)
    pool0 = d["state_pool"].clone()
    stream = torch.cuda.Stream()
    call = binding.PreparedCall(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"], d["dt_bias"], d["state_pool"],
                                d["state_indices"], d["cu_seqlens"], d["out"], stream=stream, **kw)
    call()                                   # warm-up (one-time per-device setup happens outside capture)
    torch.cuda.synchronize()
    d["state_pool"].copy_(pool0)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        call()
        call()
    d["state_pool"].copy_(pool0)
    torch.cuda.synchronize()
    graph.replay()
    torch.cuda.synchronize()
    o_refs, s_ref = oracle_chain([workload_arrays(w)] * 2, w.state_pool)
    assert_out_close(out_as_f32(d["out"]), o_refs[1], "graph replay out")
    live = w.state_indices[w.state_indices >= 0]
    assert_state_close(d["state_pool"].cpu().numpy()[live], s_ref[live], "graph replay state")
    assert torch.equal(d["out"], eager["out"]) and torch.equal(d["state_pool"], eager["state_pool"])


@pytest.mark.parametrize("kernel", MAIN, ids=MAIN_IDS)
def test_programmatic_dependent_launch_keeps_results(kernel):
    """With GDN_LAUNCH_PDL every launch still waits for the previous kernel
    before reading: a chain of six launches over the same pool (each reads
    the state the previous one wrote) matches six chained oracle calls, step
    by step, and equals the chain without PDL bit for bit."""
    w = wl.generate(wl.shrink(wl.DECODE_B512, 200))
    kw = kw_of(kernel)
    steps = 6
    results = []
    for flags in (L2, L2 | binding.LAUNCH_PDL):
        d = to_device(w)
        outs = [torch.empty_like(d["out"]) for _ in range(steps)]
        for o in outs:
            binding.decode_update(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"], d["dt_bias"],
                                  d["state_pool"], d["state_indices"], d["cu_seqlens"], o, flags=flags, **kw)
        torch.cuda.synchronize()
        results.append(([o.clone() for o in outs], d["state_pool"].clone()))
    o_refs, s_ref = oracle_chain([workload_arrays(w)] * steps, w.state_pool)
    outs, pool = results[1]
    for n in range(steps):
        assert_out_close(out_as_f32(outs[n]), o_refs[n], f"PDL chain step {n} out")
    live = w.state_indices[w.state_indices >= 0]
    assert_state_close(pool.cpu().numpy()[live], s_ref[live], "PDL chain state")
    for a_, b_ in zip(results[0][0], results[1][0]):
        assert torch.equal(a_, b_)
    assert torch.equal(results[0][1], results[1][1])
