"""Helpers for the GPU parity tests: move a workload to the device, run the
CUDA path through the C ABI, run the oracle on the same inputs (whole or on a
sample of sequences), and compare with the stated tolerances.

Tolerances (fixed for this path): state max |S_gpu - S_ref| <= 1e-4;
output |o - o_ref| <= 1e-2 + 1e-2 |o_ref|; slots and indices bit-exact.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from gated_deltanet_recurrent_sigmoid_b200 import binding
from gated_deltanet_recurrent_sigmoid_b200.workloads import Workload, bf16_bits_to_f32

STATE_ATOL = 1e-4
OUT_ATOL = 1e-2
OUT_RTOL = 1e-2


def bf16_tensor(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def to_device(w: Workload, device="cuda") -> dict:
    d = dict(q=bf16_tensor(w.q, device), k=bf16_tensor(w.k, device), v=bf16_tensor(w.v, device),
             a=bf16_tensor(w.a, device), b=bf16_tensor(w.b, device),
             A_log=torch.from_numpy(w.A_log).to(device), dt_bias=torch.from_numpy(w.dt_bias).to(device),
             state_pool=torch.from_numpy(w.state_pool).to(device),
             state_indices=torch.from_numpy(w.state_indices).to(device),
             cu_seqlens=None if w.cu_seqlens is None else torch.from_numpy(w.cu_seqlens).to(device))
    d["out"] = torch.full(w.v.shape, float("nan"), dtype=torch.bfloat16, device=device)
    return d


def run_gpu(w: Workload, flags=binding.L2NORM_QK, inter=False, tile_v=0, d=None, scale=None,
            schedule=binding.SCHEDULE_AUTO, tile_rows=0, workspace="auto"):
    """Run the CUDA path once; returns (device dict, status word, inter tensor)."""
    d = d or to_device(w)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    inter_t = None
    if inter:
        inter_t = torch.full((w.T_tot, w.spec.HV, w.spec.K, w.spec.V), float("nan"), device="cuda")
    binding.decode_update(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"], d["dt_bias"], d["state_pool"],
                          d["state_indices"], d["cu_seqlens"], d["out"], scale=scale, flags=flags,
                          intermediate_states=inter_t, device_status=status, tile_v=tile_v, schedule=schedule,
                          tile_rows=tile_rows, workspace=workspace)
    torch.cuda.synchronize()
    return d, int(status.item()), inter_t


def run_oracle(w: Workload, flags=oracle.L2NORM_QK, scale=None):
    return oracle.update(w.q, w.k, w.v, w.a, w.b, w.A_log, w.dt_bias, w.state_pool, w.state_indices,
                         w.cu_seqlens, scale=scale, flags=flags)


def token_rows(w: Workload, seqs) -> np.ndarray:
    lens = w.seq_lens
    starts = np.concatenate([[0], np.cumsum(lens)])
    return np.concatenate([np.arange(starts[i], starts[i] + lens[i]) for i in seqs]).astype(np.int64) \
        if len(seqs) else np.zeros(0, np.int64)


def sample_subproblem(w: Workload, seqs):
    """The oracle's inputs for a subset of sequences (sequences are
    independent, so the subset's results are exactly those of the full call).
    Returns (arrays, token rows in the full problem, slots in the full pool)."""
    seqs = np.asarray(seqs)
    rows = token_rows(w, seqs)
    flat = lambda x, tail: x.reshape((-1,) + x.shape[-tail:])[rows]
    slots = w.state_indices[seqs]
    live = slots >= 0
    sub_pool = w.state_pool[slots[live]]
    new_idx = np.full(len(seqs), -1, dtype=np.int32)
    new_idx[live] = np.arange(live.sum(), dtype=np.int32)
    lens = w.seq_lens[seqs]
    cu = np.zeros(len(seqs) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(lens)
    arrays = dict(q=flat(w.q, 2), k=flat(w.k, 2), v=flat(w.v, 2), a=flat(w.a, 1), b=flat(w.b, 1),
                  A_log=w.A_log, dt_bias=w.dt_bias, state_pool=np.ascontiguousarray(sub_pool),
                  state_indices=new_idx, cu_seqlens=cu)
    return arrays, rows, slots


def oracle_on(arrays, flags=oracle.L2NORM_QK, scale=None):
    return oracle.update(arrays["q"], arrays["k"], arrays["v"], arrays["a"], arrays["b"], arrays["A_log"],
                         arrays["dt_bias"], arrays["state_pool"], arrays["state_indices"], arrays["cu_seqlens"],
                         scale=scale, flags=flags)


def out_as_f32(out: torch.Tensor) -> np.ndarray:
    return out.float().cpu().numpy()


def assert_out_close(o_gpu: np.ndarray, o_ref: np.ndarray, what="out"):
    o_gpu = o_gpu.reshape(o_ref.shape).astype(np.float64)
    nan_ref = np.isnan(o_ref)
    assert np.array_equal(np.isnan(o_gpu), nan_ref), f"{what}: written rows differ"
    err = np.abs(o_gpu - o_ref)[~nan_ref]
    bound = (OUT_ATOL + OUT_RTOL * np.abs(o_ref))[~nan_ref]
    bad = err > bound
    assert not bad.any(), f"{what}: {bad.sum()} elements out of tolerance, worst {err.max():.3e}"


def assert_state_close(s_gpu: np.ndarray, s_ref: np.ndarray, what="state"):
    err = np.abs(s_gpu.astype(np.float64) - s_ref)
    assert np.isfinite(s_gpu).all(), f"{what}: non-finite values"
    assert err.max() <= STATE_ATOL, f"{what}: max abs err {err.max():.3e} > {STATE_ATOL}"


def max_errors(o_gpu: np.ndarray, o_ref: np.ndarray, s_gpu=None, s_ref=None) -> dict:
    """Largest output and state errors of a comparison (for the drift log)."""
    o_gpu = o_gpu.reshape(o_ref.shape).astype(np.float64)
    written = ~np.isnan(o_ref)
    res = {"out": float(np.abs(o_gpu - o_ref)[written].max()) if written.any() else 0.0}
    if s_gpu is not None and s_ref is not None and np.size(s_ref):
        res["state"] = float(np.abs(s_gpu.astype(np.float64) - s_ref).max())
    return res


def log_errors(case: str, **fields) -> None:
    """Append one case's largest errors to the JSON-lines file named by the
    GDN_PARITY_LOG environment variable (nothing when it is unset): the
    record of how far from the tolerances each long-sequence case lands."""
    import json
    import os
    path = os.environ.get("GDN_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"case": case, **fields}) + "\n")


def oracle_chain(steps, pool0: np.ndarray, flags=oracle.L2NORM_QK):
    """The oracle over successive calls that share one fp32 state pool: each
    step's inputs are a dict of oracle arrays (without state_pool); the pool
    after a step is rounded to fp32, as the library stores it, before the
    next step reads it.  Returns (outputs per step, pool after the last step
    in fp64)."""
    pool = np.ascontiguousarray(pool0, dtype=np.float32)
    outs, s_ref = [], pool.astype(np.float64)
    for arrays in steps:
        st, o_ref, s_ref, _ = oracle.update(arrays["q"], arrays["k"], arrays["v"], arrays["a"], arrays["b"],
                                            arrays["A_log"], arrays["dt_bias"], pool, arrays["state_indices"],
                                            arrays.get("cu_seqlens"), flags=flags)
        assert st == 0
        outs.append(o_ref)
        pool = s_ref.astype(np.float32)
    return outs, s_ref


def workload_arrays(w: Workload) -> dict:
    """A workload's inputs as the oracle takes them (pool excluded)."""
    return dict(q=w.q, k=w.k, v=w.v, a=w.a, b=w.b, A_log=w.A_log, dt_bias=w.dt_bias,
                state_indices=w.state_indices, cu_seqlens=w.cu_seqlens)


def random_workload(lens, H, HV, seed, weak_heads=(), pad=()) -> Workload:
    """A random problem with the workloads' distributions and the given
    sequence lengths (K = V = 128); value heads in `weak_heads` get
    A_log = -9 (decay within 1e-4 of 1 per token)."""
    from gated_deltanet_recurrent_sigmoid_b200 import workloads as wl
    from helpers import random_problem
    rng = np.random.default_rng(seed)
    p = random_problem(rng, lens=lens, H=H, HV=HV, K=128, V=128, pad=pad)
    spec = wl.WorkloadSpec(f"random_{len(lens)}x{max(lens)}", N=len(lens), H=H, HV=HV,
                           num_slots=p["state_pool"].shape[0], seed=seed, T=None)
    w = Workload(spec, p["q"], p["k"], p["v"], p["a"], p["b"], p["A_log"], p["dt_bias"], p["state_pool"],
                 p["state_indices"], p["cu_seqlens"])
    w.A_log = w.A_log.copy()
    for h in weak_heads:
        w.A_log[h] = -9.0
    return w
