"""gdn_decode_update_static_scratch: the entry point for callers that cannot
allocate device memory (a host program owns every allocation, or cudaMalloc
is off limits on their path).  It runs the split chunked update on the
library's built-in scratch array instead of a caller workspace.

Checked through the C ABI against the existing entry point (gdn_decode_update
on the split schedule with a torch-allocated workspace) on the same inputs,
for two calls in a row -- the second call finds the first call's data in the
shared array.  Both run the same deterministic kernels and differ only in the
workspace address, so the results must be the same bits; each is also
compared with the oracle at the tolerances of the other GPU tests.  This file
is collected last so that a run stopping at the first failure has run every
other test; it also passes alone in a fresh process (the first call on the
device looks up the array's address).
"""
import numpy as np
import pytest
import torch

from gated_deltanet_recurrent_sigmoid_b200 import binding
from gated_deltanet_recurrent_sigmoid_b200 import workloads as wl
from gpu_helpers import assert_out_close, assert_state_close, out_as_f32, run_oracle, to_device
from helpers import random_problem

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(gdn_lib):
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return gdn_lib


def problem(lens, H, HV, seed):
    rng = np.random.default_rng(seed)
    p = random_problem(rng, lens=lens, H=H, HV=HV, K=128, V=128, pad=())
    spec = wl.WorkloadSpec("no_alloc_case", N=len(lens), H=H, HV=HV, num_slots=p["state_pool"].shape[0],
                           seed=seed, T=None)
    return wl.Workload(spec, p["q"], p["k"], p["v"], p["a"], p["b"], p["A_log"], p["dt_bias"], p["state_pool"],
                       p["state_indices"], p["cu_seqlens"])


def args(d):
    return (d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"], d["dt_bias"], d["state_pool"], d["state_indices"],
            d["cu_seqlens"], d["out"])


def test_static_scratch_matches_workspace_entry_point_twice():
    cases = [problem([200, 37, 130, 64], H=4, HV=8, seed=31),      # 431 tokens: 7 blocks x 8 heads
             problem([90, 5, 260, 1], H=2, HV=6, seed=32)]         # then other sizes on the same array
    for w in cases:
        ref = to_device(w)
        binding.decode_update(*args(ref), schedule=binding.SCHEDULE_CHUNKED_SPLIT)
        got = to_device(w)
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        binding.decode_update_static_scratch(*args(got), device_status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert torch.equal(got["out"], ref["out"]), "static scratch out differs from the workspace path"
        assert torch.equal(got["state_pool"], ref["state_pool"]), "static scratch state differs"
        ost, o_ref, s_ref, _ = run_oracle(w)
        assert ost == 0
        assert_out_close(out_as_f32(got["out"]), o_ref, "static scratch out")
        live = w.state_indices[w.state_indices >= 0]
        assert_state_close(got["state_pool"].cpu().numpy()[live], s_ref[live], "static scratch state")


def test_static_scratch_rejects_calls_beyond_its_size():
    # 4160 tokens x 8 heads need 65 x 8 = 520 records > 510 that fit in 64 MiB
    T, H, HV = 4160, 4, 8
    assert binding.chunked_workspace_bytes(T, HV) > binding.STATIC_SCRATCH_BYTES
    bf = torch.bfloat16
    d = dict(q=torch.zeros(T, H, 128, dtype=bf, device="cuda"), k=torch.zeros(T, H, 128, dtype=bf, device="cuda"),
             v=torch.zeros(T, HV, 128, dtype=bf, device="cuda"), a=torch.zeros(T, HV, dtype=bf, device="cuda"),
             b=torch.zeros(T, HV, dtype=bf, device="cuda"), A_log=torch.zeros(HV, device="cuda"),
             dt_bias=torch.zeros(HV, device="cuda"), state_pool=torch.zeros(2, HV, 128, 128, device="cuda"),
             state_indices=torch.tensor([0, 1], dtype=torch.int32, device="cuda"),
             cu_seqlens=torch.tensor([0, 2000, T], dtype=torch.int32, device="cuda"),
             out=torch.full((T, HV, 128), 7.0, dtype=bf, device="cuda"))
    with pytest.raises(binding.GdnError) as e:
        binding.decode_update_static_scratch(*args(d))
    assert e.value.status == binding.ERR_SCRATCH
    torch.cuda.synchronize()
    assert bool((d["out"] == 7.0).all())          # rejected before any launch
