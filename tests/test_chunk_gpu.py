"""The chunked (tensor-core) schedule against the oracle.

Same update, same tolerances as the per-token kernels: state max abs 1e-4,
output 1e-2 + 1e-2 |o_ref|, slots and status exact.  Sequences span several
64-token chunks with ragged tails.
"""
import numpy as np
import pytest
import torch

import oracle
from gated_deltanet_recurrent_sigmoid_b200 import binding
from gated_deltanet_recurrent_sigmoid_b200 import workloads as wl
from gpu_helpers import (assert_out_close, assert_state_close, oracle_chain, oracle_on, out_as_f32, run_gpu,
                         run_oracle, sample_subproblem, to_device, workload_arrays)
from helpers import random_problem

pytestmark = pytest.mark.gpu

CHUNKED = binding.SCHEDULE_CHUNKED
SPLIT = binding.SCHEDULE_CHUNKED_SPLIT
L2 = binding.L2NORM_QK


@pytest.fixture(params=[CHUNKED, SPLIT], ids=["single", "split"])
def sched(request):
    """Both chunked schedules: one kernel with every chunk product on chip, or
    the block kernel + state kernel around a workspace."""
    return request.param


@pytest.fixture(scope="module", autouse=True)
def _lib(gdn_lib):
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return gdn_lib


def check(w, sched, flags=L2, scale=None):
    d, status, _ = run_gpu(w, flags=flags, schedule=sched, scale=scale)
    ost, o_ref, s_ref, _ = run_oracle(w, flags=flags, scale=scale)
    assert status == ost
    assert_out_close(out_as_f32(d["out"]), o_ref)
    pool = d["state_pool"].cpu().numpy()
    live = w.state_indices[(w.state_indices >= 0) & (w.seq_lens > 0)] if not flags & binding.NO_FINAL_WRITEBACK \
        else np.zeros(0, np.int64)
    touched = np.zeros(w.spec.num_slots, bool)
    touched[live] = True
    assert np.array_equal(pool[~touched], w.state_pool[~touched])
    if touched.any():
        assert_state_close(pool[touched], s_ref[touched])
    return d


def problem(lens, pad=(), H=4, HV=8, seed=0):
    rng = np.random.default_rng(seed)
    p = random_problem(rng, lens=lens, H=H, HV=HV, K=128, V=128, pad=pad)
    spec = wl.WorkloadSpec("chunk_case", N=len(lens), H=H, HV=HV, num_slots=p["state_pool"].shape[0], seed=seed,
                           T=None)
    return wl.Workload(spec, p["q"], p["k"], p["v"], p["a"], p["b"], p["A_log"], p["dt_bias"], p["state_pool"],
                       p["state_indices"], p["cu_seqlens"])


@pytest.mark.parametrize("lens", [[1], [64], [65], [200, 7, 130], [3, 64, 128, 1, 300]],
                         ids=["1", "64", "65", "ragged3", "ragged5"])
def test_chunked_matches_oracle(lens, sched):
    check(problem(lens, seed=len(lens)), sched)


def test_chunked_padding_empty_and_gqa(sched):
    check(problem([70, 0, 33, 129], pad=(2,), H=2, HV=6, seed=9), sched)


def test_chunked_l2norm_off_and_scale(sched):
    w = problem([90, 40], seed=3)
    # L2 off: unit-length k keeps the state O(1)
    k = wl.bf16_bits_to_f32(w.k)
    w.k = wl.f32_to_bf16_bits(k / np.linalg.norm(k, axis=-1, keepdims=True))
    check(w, sched, flags=0)
    check(problem([90, 40], seed=4), sched, scale=0.2)


def test_chunked_weak_and_mixed_decay(sched):
    """exp(A_log) tiny: the decays stay near 1, so the state's scale never
    leaves its range (no rescaling); mixed heads cover both cases in one
    call."""
    w = problem([150, 3, 70, 200], seed=12)
    w.A_log = np.full_like(w.A_log, -9.0)
    check(w, sched)
    w = problem([150, 3, 70, 200], seed=13)
    w.A_log = w.A_log.copy()
    w.A_log[::2] = -9.0
    check(w, sched)


def test_chunked_no_final_writeback_and_fixed_layout(sched):
    check(problem([77, 12], seed=5), sched, flags=L2 | binding.NO_FINAL_WRITEBACK)
    check(wl.generate(wl.shrink(wl.SPEC_B128_T4, 16)), sched)  # T = 4, one partial chunk each
    check(wl.generate(wl.TINY), sched)                          # fixed [N, 1] layout
    fixed = wl.WorkloadSpec("fixed_t100", N=3, H=4, HV=8, num_slots=6, seed=14, T=100)
    check(wl.generate(fixed), sched)                            # fixed [N, T] layout, blocks across sequences


@pytest.mark.parametrize("spec", [wl.sweep_spec(8), wl.sweep_spec(64)], ids=lambda s: s.name)
def test_chunked_full_size_sweeps(spec, sched):
    check(wl.generate(spec), sched)


def test_chunked_prefill_b64_sampled(sched):
    """Full-size prefill-style batch in the benchmark's launch configuration;
    the oracle recomputes a sample of sequences."""
    w = wl.generate(wl.PREFILL_B64)
    d, status, _ = run_gpu(w, schedule=sched)
    assert status == 0
    rng = np.random.default_rng(0)
    seqs = np.sort(rng.choice(w.spec.N, size=6, replace=False))
    arrays, rows, slots = sample_subproblem(w, seqs)
    _, o_ref, s_ref, _ = oracle_on(arrays)
    out = d["out"].view(w.T_tot, w.spec.HV, w.spec.V)
    assert_out_close(out[torch.from_numpy(rows).cuda()].float().cpu().numpy(), o_ref, "sampled out")
    live = slots >= 0
    got = d["state_pool"][torch.from_numpy(slots[live].astype(np.int64)).cuda()].cpu().numpy()
    assert_state_close(got, s_ref, "sampled state")


def test_chunked_agrees_with_per_token_kernel(sched):
    w = wl.generate(wl.shrink(wl.sweep_spec(64), 24))
    a, _, _ = run_gpu(w, schedule=sched)
    b, _, _ = run_gpu(w, schedule=binding.SCHEDULE_PER_TILE, tile_v=16, tile_rows=16)
    assert (a["state_pool"] - b["state_pool"]).abs().max().item() <= 1e-4
    assert (a["out"].float() - b["out"].float()).abs().max().item() <= 3e-2


def test_chunked_rejects_unbuilt_modes(sched):
    w = wl.generate(wl.shrink(wl.SPEC_B128_T4, 4))
    d = to_device(w)
    inter = torch.empty((w.T_tot, w.spec.HV, 128, 128), device="cuda")
    with pytest.raises(binding.GdnError) as e:
        binding.decode_update(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"], d["dt_bias"], d["state_pool"],
                              d["state_indices"], d["cu_seqlens"], d["out"], intermediate_states=inter,
                              schedule=sched)
    assert e.value.status == binding.ERR_UNSUPPORTED


def test_chunked_device_status(sched):
    w = problem([70, 20, 5], seed=11)
    w.state_indices = w.state_indices.copy()
    w.state_indices[1] = w.spec.num_slots           # out of range
    d, status, _ = run_gpu(w, schedule=sched)
    ost, o_ref, s_ref, _ = run_oracle(w)
    assert status == ost == oracle.BAD_SLOT
    assert_out_close(out_as_f32(d["out"]), o_ref)


def _bits_equal(a, b):
    return torch.equal(a["state_pool"], b["state_pool"]) and torch.equal(a["out"], b["out"])


def test_auto_schedule_picks_by_length_and_pairs():
    """GDN_SCHEDULE_AUTO (bit-identical to asking for the schedule it picks):
    few long sequences run the split kernels when a workspace is given (the
    binding allocates one) and the on-chip chunked kernel without one -- with
    few enough pairs from 80 tokens per sequence on average;
    sequences of a few dozen tokens run the on-chip chunked kernel either
    way; short ones, or a call with per-token states, the per-tile kernel."""
    long_w = problem([200, 150, 300], seed=21)                 # 24 pairs, mean 217
    auto, _, _ = run_gpu(long_w)
    split, _, _ = run_gpu(long_w, schedule=SPLIT)
    assert _bits_equal(auto, split)
    auto_nows, _, _ = run_gpu(long_w, workspace=None)
    chunked, _, _ = run_gpu(long_w, schedule=CHUNKED)
    assert _bits_equal(auto_nows, chunked)
    per_tile, _, _ = run_gpu(long_w, schedule=binding.SCHEDULE_PER_TILE)
    assert not _bits_equal(auto, per_tile) and not _bits_equal(auto, chunked)

    two_cta_w = problem([70, 90, 110], seed=24)               # 24 pairs, mean 90: two state CTAs a pair
    auto, _, _ = run_gpu(two_cta_w)
    split, _, _ = run_gpu(two_cta_w, schedule=SPLIT)
    assert _bits_equal(auto, split)
    below_w = problem([60, 70, 80], seed=25)                  # 24 pairs, mean 70: below the split range
    auto, _, _ = run_gpu(below_w)
    chunked, _, _ = run_gpu(below_w, schedule=CHUNKED)
    assert _bits_equal(auto, chunked)

    mid_w = problem([30, 60, 10, 45], seed=23)                # 32 pairs, mean 36
    auto, _, _ = run_gpu(mid_w)
    chunked, _, _ = run_gpu(mid_w, schedule=CHUNKED)
    assert _bits_equal(auto, chunked)

    short_w = problem([3, 20, 10], seed=22)                   # 24 pairs, mean 11
    auto, _, _ = run_gpu(short_w)
    per_tile, _, _ = run_gpu(short_w, schedule=binding.SCHEDULE_PER_TILE)
    assert _bits_equal(auto, per_tile)

    auto_d, _, auto_i = run_gpu(long_w, inter=True)
    pt_d, _, pt_i = run_gpu(long_w, inter=True, schedule=binding.SCHEDULE_PER_TILE)
    assert _bits_equal(auto_d, pt_d) and torch.equal(auto_i, pt_i)


def test_chunked_strided_views_of_packed_projections(sched):
    """q, k, v as column slices of one packed projection row (token stride
    wider than a head's row) and a, b interleaved per value head: the
    oracle's results, and the same bits as contiguous inputs, on both
    chunked schedules."""
    w = problem([200, 37, 130, 64, 5], seed=61)
    ref, _, _ = run_gpu(w, schedule=sched)
    d = to_device(w)
    T, H, HV, K, V = w.T_tot, w.spec.H, w.spec.HV, w.spec.K, w.spec.V
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
                          d["cu_seqlens"], d["out"], schedule=sched)
    torch.cuda.synchronize()
    ost, o_ref, s_ref, _ = run_oracle(w)
    assert ost == 0
    assert_out_close(out_as_f32(d["out"]), o_ref, "strided out")
    live = w.state_indices[w.state_indices >= 0]
    assert_state_close(d["state_pool"].cpu().numpy()[live], s_ref[live], "strided state")
    assert torch.equal(d["out"], ref["out"]) and torch.equal(d["state_pool"], ref["state_pool"])


@pytest.mark.parametrize("lens", [[200, 37, 130, 64, 5], [200, 37, 130, 64, 5] * 3,
                                  [int(x) for x in np.random.default_rng(71).integers(1, 65, 320)]],
                         ids=["two_cta_form", "full_form", "compact_form"])
def test_split_is_deterministic(lens):
    """Five runs of the split schedule on the same inputs give the same bits
    (no atomics or order-dependent sums in either kernel: a race between the
    kernels' reuse of shared memory or TMEM would show here)."""
    w = problem(lens, seed=72)
    ref, _, _ = run_gpu(w, schedule=SPLIT)
    for _ in range(4):
        d, status, _ = run_gpu(w, schedule=SPLIT)
        assert status == 0
        assert torch.equal(d["out"], ref["out"]) and torch.equal(d["state_pool"], ref["state_pool"])


def test_split_full_width_state_kernel_mid_batch():
    """96 (sequence, head) pairs -- more than one wave of two-CTA pairs on 148
    SMs, fewer than the compact form's 296 -- run the full-width state kernel:
    ragged lengths, an empty and a padded sequence, weak and strong decays,
    compared whole with the oracle."""
    lens = [200, 37, 130, 64, 5, 1, 300, 65, 128, 0, 90, 150]
    w = problem(lens, pad=(4,), seed=73)
    w.A_log = w.A_log.copy()
    w.A_log[::2] = -9.0
    check(w, SPLIT)


def test_split_compact_many_short_sequences():
    """Enough short sequences (320 x 8 heads) that the split schedule runs its
    compact state kernel: empty sequences, padded slots, weak and strong
    decays, all compared whole with the oracle."""
    rng = np.random.default_rng(41)
    lens = [int(x) for x in rng.integers(0, 41, size=320)]
    lens[5] = 0
    lens[17] = 64
    lens[18] = 65
    w = problem(lens, pad=(3, 77, 200), seed=41)
    w.A_log = w.A_log.copy()
    w.A_log[::2] = -9.0
    check(w, SPLIT)


def _args(d):
    return (d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"], d["dt_bias"], d["state_pool"], d["state_indices"],
            d["cu_seqlens"], d["out"])


def test_graph_capture_and_pdl_chain(sched):
    """Both chunked schedules capture in a CUDA graph and chain with
    programmatic dependent launch (the split one as two kernels): two chained
    calls replayed from a graph, and two chained PDL calls, match two chained
    oracle calls and give the bits of two eager calls."""
    w = problem([150, 40, 90], seed=51)
    eager = to_device(w)
    for _ in range(2):
        binding.decode_update(*_args(eager), schedule=sched)
    torch.cuda.synchronize()

    d = to_device(w)
    pool0 = d["state_pool"].clone()
    ws = torch.empty(binding.chunked_workspace_bytes(w.T_tot, w.spec.HV), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.Stream()
    call = binding.PreparedCall(*_args(d), stream=stream, schedule=sched, workspace=ws)
    call()                                   # one-time per-device set-up outside the capture
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
    assert torch.equal(d["out"], eager["out"]) and torch.equal(d["state_pool"], eager["state_pool"])

    p = to_device(w)
    first = torch.empty_like(p["out"])
    binding.decode_update(*_args(p)[:-1], first, schedule=sched, flags=L2 | binding.LAUNCH_PDL)
    binding.decode_update(*_args(p), schedule=sched, flags=L2 | binding.LAUNCH_PDL)
    torch.cuda.synchronize()
    o_refs, s_ref = oracle_chain([workload_arrays(w)] * 2, w.state_pool)
    live = w.state_indices[w.state_indices >= 0]
    for name, got in (("graph", d), ("pdl", p)):
        assert_out_close(out_as_f32(got["out"]), o_refs[1], f"{name} chain out")
        assert_state_close(got["state_pool"].cpu().numpy()[live], s_ref[live], f"{name} chain state")
    assert_out_close(out_as_f32(first), o_refs[0], "pdl chain first out")
    assert torch.equal(p["out"], eager["out"]) and torch.equal(p["state_pool"], eager["state_pool"])


def test_split_writes_nothing_outside_its_workspace():
    """Guard bands around the workspace keep their sentinel bytes; the
    minimal workspace (gdn_chunked_workspace_bytes exactly) is enough."""
    w = problem([70, 3, 130, 64], seed=52)
    d = to_device(w)
    need = binding.chunked_workspace_bytes(w.T_tot, w.spec.HV)
    guard = 4096
    buf = torch.full((need + 2 * guard,), 0xA5, dtype=torch.uint8, device="cuda")
    ws = buf[guard:guard + need]
    assert ws.data_ptr() % 256 == 0
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    binding.decode_update(*_args(d), schedule=SPLIT, workspace=ws, device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert bool((buf[:guard] == 0xA5).all()) and bool((buf[guard + need:] == 0xA5).all())
    ost, o_ref, s_ref, _ = run_oracle(w)
    assert_out_close(out_as_f32(d["out"]), o_ref)
