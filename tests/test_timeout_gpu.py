"""The kernels' bounded waits, made to run out on purpose.

A test-only copy of the library (tests/timeout_probe/) withholds the arrival
that pairs with each kernel's first bulk copy of a sequence's data (its
state, or for the two-CTA split state kernel, which loads the state with
plain loads, the first piece's U / fo / gamma) and limits every wait to
2 ms, so each kernel gives up at its first wait.  For the on-chip chunked
kernel, the three split state kernels (two CTAs per pair -- 12 pairs --,
full-width -- 84 pairs, more than fit one wave of two-CTA pairs on 148 SMs --
and compact) and the pipelined kernel, one call through that copy must

  - return GDN_OK and report GDN_DEV_TIMEOUT in the status word,
  - leave every byte outside its buffers alone (guard bands around the pool,
    the outputs and the workspace keep their sentinels) and the pool itself
    unchanged (nothing was computed, so nothing is written back),
  - leave the device usable with its tensor memory freed: the same call
    through the product library right afterwards, on the same device (whose
    kernels allocate tensor memory on every SM they run on), matches the
    oracle.
No wait here depends on the GPU misbehaving: the arrival is simply never
made, and the waits are bounded by the global timer.
"""
import ctypes
import os

import numpy as np
import pytest
import torch

from gated_deltanet_recurrent_sigmoid_b200 import binding
from gpu_helpers import (assert_out_close, assert_state_close, out_as_f32, random_workload, run_oracle,
                         to_device)

pytestmark = pytest.mark.gpu


def _load_builder():
    """The probe's build module, loaded by path under its own name (both
    probe directories have a build.py)."""
    import importlib.util
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "timeout_probe", "build.py")
    spec = importlib.util.spec_from_file_location("timeout_probe_build", path)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


SENTINEL = -1024.0      # exact in bf16 and fp32
GUARD = 4096            # workspace guard band, bytes


@pytest.fixture(scope="module")
def timeout_lib(gdn_lib):
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    probe_build = _load_builder()
    lib = ctypes.CDLL(probe_build.build())
    P = ctypes.POINTER(binding.GdnTensor)
    lib.gdn_decode_update.restype = ctypes.c_int
    lib.gdn_decode_update.argtypes = [P] * 11 + [ctypes.c_float, ctypes.c_uint32, ctypes.POINTER(binding.GdnExtra)]
    return lib


CASES = {
    # schedule, lengths, heads: each reaches the named kernel's state wait
    "chunked": (binding.SCHEDULE_CHUNKED, [70, 3, 130, 64], 2, 4),
    "split_half": (binding.SCHEDULE_CHUNKED_SPLIT, [150, 40, 90], 2, 4),
    "split_full": (binding.SCHEDULE_CHUNKED_SPLIT, [150, 40, 90] * 7, 2, 4),
    "split_compact": (binding.SCHEDULE_CHUNKED_SPLIT, [int(x) for x in np.random.default_rng(5).integers(1, 65, 40)],
                      4, 8),
    "pipelined": (binding.SCHEDULE_PIPELINED, [1] * 24, 2, 4),
}


def guarded(w):
    """Device tensors of a workload, with the pool and the outputs placed
    inside larger buffers whose first and last rows hold a sentinel."""
    d = to_device(w)
    pool = torch.full((w.spec.num_slots + 2, w.spec.HV, 128, 128), SENTINEL, device="cuda")
    pool[1:-1] = d["state_pool"]
    out = torch.full((w.T_tot + 2, w.spec.HV, 128), SENTINEL, dtype=torch.bfloat16, device="cuda")
    d["pool_buf"], d["out_buf"] = pool, out
    d["state_pool"], d["out"] = pool[1:-1], out[1:-1]
    return d


@pytest.mark.parametrize("case", list(CASES))
def test_bounded_wait_runs_out_and_the_device_stays_usable(timeout_lib, case):
    sched, lens, H, HV = CASES[case]
    w = random_workload(lens, H=H, HV=HV, seed=300 + len(lens))
    d = guarded(w)
    pool_before = d["pool_buf"].clone()
    need = binding.chunked_workspace_bytes(w.T_tot, HV)
    ws_buf = torch.full((need + 2 * GUARD,), 0xA5, dtype=torch.uint8, device="cuda")
    ws = ws_buf[GUARD:GUARD + need]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    descs = [binding.describe(d[n]) for n in ("q", "k", "v", "a", "b", "A_log", "dt_bias", "state_pool",
                                               "state_indices", "cu_seqlens", "out")]
    extra = binding.GdnExtra()
    extra.stream = torch.cuda.current_stream().cuda_stream
    extra.device_status = status.data_ptr()
    extra.schedule = sched
    if sched == binding.SCHEDULE_CHUNKED_SPLIT:
        extra.workspace, extra.workspace_bytes = ws.data_ptr(), need
    out_before = d["out_buf"].clone()
    rc = timeout_lib.gdn_decode_update(*[binding._ref(x) for x in descs], ctypes.c_float(128 ** -0.5),
                                       ctypes.c_uint32(binding.L2NORM_QK), ctypes.byref(extra))
    torch.cuda.synchronize()
    assert rc == binding.OK
    assert int(status.item()) & binding.DEV_TIMEOUT, f"status {int(status.item())}"
    # nothing outside the call's buffers, and nothing in the pool, changed
    assert torch.equal(d["pool_buf"], pool_before)
    assert bool((d["out_buf"][0].float() == SENTINEL).all()) and bool((d["out_buf"][-1].float() == SENTINEL).all())
    assert bool((ws_buf[:GUARD] == 0xA5).all()) and bool((ws_buf[GUARD + need:] == 0xA5).all())
    assert torch.equal(d["out_buf"], out_before)         # no output was written

    # the product library on the same device, same inputs: the oracle's results
    fresh = to_device(w)
    st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
    binding.decode_update(fresh["q"], fresh["k"], fresh["v"], fresh["a"], fresh["b"], fresh["A_log"],
                          fresh["dt_bias"], fresh["state_pool"], fresh["state_indices"], fresh["cu_seqlens"],
                          fresh["out"], device_status=st2, schedule=sched)
    torch.cuda.synchronize()
    ost, o_ref, s_ref, _ = run_oracle(w)
    assert int(st2.item()) == ost == 0
    assert_out_close(out_as_f32(fresh["out"]), o_ref)
    live = w.state_indices[w.state_indices >= 0]
    assert_state_close(fresh["state_pool"].cpu().numpy()[live], s_ref[live])
