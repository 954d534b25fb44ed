"""First calls from several host threads at once.

The chunked, split and pipelined launchers do a one-time set-up per device
(shared-memory opt-ins, the SM count) on their first call there.  In a fresh
process, six threads -- two per schedule -- are released together by a
barrier and each makes its schedule's first call on the same device, on its
own stream and buffers (the ctypes call releases the interpreter lock, so the
calls run in the library at the same time).  Every result is compared with
the oracle.
"""
import os
import subprocess
import sys
import textwrap

import numpy as np
import pytest
import torch

from gated_deltanet_recurrent_sigmoid_b200 import binding
from gpu_helpers import assert_out_close, assert_state_close, random_workload, run_oracle

pytestmark = pytest.mark.gpu

TESTS = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(TESTS)
CASES = [(binding.SCHEDULE_CHUNKED_SPLIT, 201), (binding.SCHEDULE_CHUNKED_SPLIT, 202),
         (binding.SCHEDULE_CHUNKED, 203), (binding.SCHEDULE_CHUNKED, 204),
         (binding.SCHEDULE_PIPELINED, 205), (binding.SCHEDULE_PIPELINED, 206)]
LENS = [70, 3, 130, 64]

CHILD = textwrap.dedent("""
    import sys, threading
    import numpy as np, torch
    sys.path[:0] = [{root!r}, {tests!r}]
    from gated_deltanet_recurrent_sigmoid_b200 import binding
    from gpu_helpers import random_workload, to_device
    cases, lens, out_path = {cases!r}, {lens!r}, {out!r}
    binding.load()
    jobs = []
    for sched, seed in cases:
        w = random_workload(lens, H=2, HV=4, seed=seed)
        d = to_device(w)
        ws = torch.empty(binding.chunked_workspace_bytes(w.T_tot, 4), dtype=torch.uint8, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        jobs.append((sched, d, ws, st, torch.cuda.Stream()))
    torch.cuda.synchronize()
    barrier = threading.Barrier(len(jobs))
    errors = []
    def run(job):
        sched, d, ws, st, stream = job
        try:
            barrier.wait()
            binding.decode_update(d["q"], d["k"], d["v"], d["a"], d["b"], d["A_log"], d["dt_bias"],
                                  d["state_pool"], d["state_indices"], d["cu_seqlens"], d["out"],
                                  device_status=st, stream=stream, schedule=sched,
                                  workspace=ws if sched == binding.SCHEDULE_CHUNKED_SPLIT else None)
            stream.synchronize()
        except Exception as e:
            errors.append(repr(e))
    threads = [threading.Thread(target=run, args=(j,)) for j in jobs]
    for t in threads: t.start()
    for t in threads: t.join()
    assert not errors, errors
    res = {{}}
    for n, (sched, d, ws, st, stream) in enumerate(jobs):
        res[f"out{{n}}"] = d["out"].float().cpu().numpy()
        res[f"pool{{n}}"] = d["state_pool"].cpu().numpy()
        res[f"status{{n}}"] = st.cpu().numpy()
    np.savez(out_path, **res)
""")


def test_first_calls_from_several_threads(tmp_path):
    out = str(tmp_path / "threads.npz")
    script = CHILD.format(root=ROOT, tests=TESTS, cases=CASES, lens=LENS, out=out)
    res = subprocess.run([sys.executable, "-c", script], capture_output=True, text=True, timeout=600)
    assert res.returncode == 0, res.stderr[-3000:]
    got = np.load(out)
    for n, (sched, seed) in enumerate(CASES):
        w = random_workload(LENS, H=2, HV=4, seed=seed)
        ost, o_ref, s_ref, _ = run_oracle(w)
        assert int(got[f"status{n}"][0]) == ost == 0
        assert_out_close(got[f"out{n}"], o_ref, f"thread {n} out")
        live = w.state_indices[w.state_indices >= 0]
        assert_state_close(got[f"pool{n}"][live], s_ref[live], f"thread {n} state")
