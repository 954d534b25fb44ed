"""Benchmark of the fused sigmoid-gating GDN decode update on B200.

One step = one call of the whole hot path (one fused kernel) over one batch
of the Qwen3-Next per-rank decode shape: B = 512 sequences, T = 1, H = 4 key
heads, HV = 8 value heads, K = V = 128, fp32 state pool of 1024 slots, 5 %
padded (-1) slots.  Prints ONE JSON line (rank 0).

    python bench.py [--gpus N --steps K --warmup W] [--impl reference]
    torchrun --nproc-per-node N bench.py --gpus N ...    (one replica per GPU)

value      whole-job state-traffic throughput: algorithmic HBM bytes of all
           ranks' steps / max-over-ranks device time (CUDA events), GB/s.
           Inputs are resident in HBM; consecutive steps rotate over 4 copies
           of the inputs (2.1 GB in all), so no step finds its data in L2.
e2e        the same metric through the public API with pinned HOST buffers:
           every step copies its inputs host -> device, runs the update and
           reads the output back, synchronising on the result.
roofline   the fused kernel against the measured HBM copy bandwidth.
cpu_baseline  the CPU oracle (single thread, fp64) on a bounded sample of
           the same workload (rank 0, N = 1 only).
--impl reference  times the CPU oracle alone (the reference arm).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from gated_deltanet_recurrent_sigmoid_b200 import workloads as wl  # noqa: E402

METRIC = "µs/call and state GB/s (% of B200 HBM peak) at B=512, HV=8, K=V=128"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
ROTATING_COPIES = 4
# the library's GDN_SCHEDULE_AUTO thresholds (mean tokens per sequence, by the
# (sequence, value head) pair count), as documented in include/gdn_decode.h


def split_pays(pairs, mean_tokens, sms=148):
    """Whether AUTO runs the split chunked kernels (the binding passes a workspace)."""
    if 2 * pairs <= sms:
        return mean_tokens >= 80
    if pairs < 128:
        return mean_tokens >= 144
    if pairs < 256:
        return mean_tokens >= 192
    if pairs < 512:
        return mean_tokens >= 512
    return False


def chunked_min_mean_tokens(pairs):
    """The on-chip chunked kernel's threshold."""
    return 20 if pairs < 64 else (14 if pairs < 512 else 13)


# DRAM traffic of one launch of the fused kernel on decode_b512_hv8, from the
# ncu capture summarised in profiles/ (dram__bytes_read.sum +
# dram__bytes_write.sum).  Valid only for the kernel sources it was taken on.
NCU_TRAFFIC = {"kernel_sha256": "56a5bd6fd0f772dbd0de9456b16af0c872fa8c6c4137184b3fa31d1fb1ea9a96",
               "workload": "decode_b512_hv8", "bytes_per_launch": 257377792 + 202355968}


def h2d_link_gbs(nbytes, device, reps=40):
    """Pinned host -> device copy rate (GB/s) for a copy of `nbytes`: a warm-up
    copy, then `reps` copies back to back on one stream, timed with events."""
    import torch
    if nbytes <= 0:
        return None
    host = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    dev = torch.empty(nbytes, dtype=torch.uint8, device=device)
    s = torch.cuda.Stream(device)
    with torch.cuda.stream(s):
        dev.copy_(host, non_blocking=True)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            dev.copy_(host, non_blocking=True)
        e1.record()
    s.synchronize()
    return round(nbytes * reps / (e0.elapsed_time(e1) * 1e-3) / 1e9, 1)


def kernel_source_hash() -> str:
    """Hash of the per-tile kernel's device code (the kernel the traffic figure
    belongs to)."""
    with open(os.path.join(ROOT, "gated_deltanet_recurrent_sigmoid_b200", "csrc", "gdn_decode_kernel.cuh"), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()


# fp32 CUDA-core bound of the per-token arithmetic: 148 SMs x 128 fp32 lanes x
# 2 flops per FMA x the 1965 MHz maximum SM clock (B200 unit counts).
ALU_F32_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------

CLOCK_FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
                "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
                "clocks_event_reasons.sw_power_cap")
REASON_NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")


class ClockSampler:
    """nvidia-smi sampling of this GPU's clocks while the timed region runs."""

    def __init__(self, device_index: int):
        self.proc = None
        try:
            import torch
            ident = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
        except Exception:
            ident = str(device_index)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", ident, f"--query-gpu={CLOCK_FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=10)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], [], set()
        for line in out.splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != 7:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for name, val in zip(REASON_NAMES, parts[3:]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline and the reference arm)
# ---------------------------------------------------------------------------

def oracle_subset_args(w, seqs):
    """The oracle's inputs for a subset of sequences (a compact pool holding
    only their live slots)."""
    lens = w.seq_lens
    starts = np.concatenate([[0], np.cumsum(lens)])
    rows = np.concatenate([np.arange(starts[i], starts[i] + lens[i]) for i in seqs])
    flat = lambda x, tail: x.reshape((-1,) + x.shape[-tail:])[rows]
    slots = w.state_indices[seqs]
    live = slots >= 0
    idx = np.full(len(seqs), -1, np.int32)
    idx[live] = np.arange(live.sum(), dtype=np.int32)
    cu = np.zeros(len(seqs) + 1, np.int32)
    cu[1:] = np.cumsum(lens[seqs])
    args = (flat(w.q, 2), flat(w.k, 2), flat(w.v, 2), flat(w.a, 1), flat(w.b, 1), w.A_log, w.dt_bias,
            np.ascontiguousarray(w.state_pool[slots[live]]), idx, cu)
    return args


def oracle_subset_seconds(w, seqs):
    """Wall time of the oracle on a subset of sequences (its own inputs)."""
    import oracle
    args = oracle_subset_args(w, seqs)
    t0 = time.perf_counter()
    oracle.update(*args)
    return time.perf_counter() - t0


def subset_bytes(w, seqs):
    s = w.spec
    live = w.state_indices[seqs] >= 0
    lens = w.seq_lens[seqs]
    head = s.K * s.V * 4
    nbytes = 2 * int(live.sum()) * s.HV * head
    nbytes += int(lens[live].sum()) * (2 * s.H * s.K + s.HV * s.V + 2 * s.HV) * 2
    nbytes += int(lens.sum()) * s.HV * s.V * 2 + 8 * s.HV + 4 * len(seqs)
    return nbytes


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline(w, budget_s=10.0):
    """The oracle as it stands, single-threaded, over the whole workload
    repeated until about ``budget_s`` seconds of CPU work."""
    seqs = np.arange(w.spec.N)
    oracle_subset_seconds(w, seqs[:1])   # untimed: loads the oracle library
    total_t, reps = 0.0, 0
    while reps == 0 or total_t < budget_s:
        total_t += oracle_subset_seconds(w, seqs)
        reps += 1
    per = total_t / reps
    return {"value": round(wl.algorithmic_bytes(w) / per / 1e9, 4), "unit": "GB/s", "cores": 1,
            "kind": "oracle", "us_per_call": round(per * 1e6, 1), "cpu": cpu_model(),
            "sample": f"whole {w.spec.name} workload ({w.spec.N} sequences), {reps} repetitions, "
                      f"{total_t:.1f} s single-threaded fp64 C loop nest"}


def cpu_baseline_all_cores(w, budget_s=10.0):
    """The same oracle, unchanged, run on all host cores: the sequences are
    split into one contiguous group per core and each group is one oracle
    call on its own thread (the C loop nest runs without the interpreter
    lock)."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    cores = max(1, len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count() or 1)
    groups = [g for g in np.array_split(np.arange(w.spec.N), cores) if len(g)]
    args = [oracle_subset_args(w, g) for g in groups]
    total_t, reps = 0.0, 0
    oracle_subset_seconds(w, groups[0][:1])   # untimed: loads the oracle library
    with ThreadPoolExecutor(len(groups)) as pool:
        while reps == 0 or total_t < budget_s:
            t0 = time.perf_counter()
            list(pool.map(lambda a: oracle.update(*a), args))
            total_t += time.perf_counter() - t0
            reps += 1
    per = total_t / reps
    return {"value": round(wl.algorithmic_bytes(w) / per / 1e9, 4), "unit": "GB/s", "cores": len(groups),
            "kind": "oracle", "us_per_call": round(per * 1e6, 1), "cpu": cpu_model(),
            "sample": f"whole {w.spec.name} workload split into {len(groups)} sequence groups, one thread each, "
                      f"{reps} repetitions, {total_t:.1f} s"}


def parity_sample(w, prepare, torch, device, nseq=8, final_writeback=True):
    """Part of the cpu_baseline leg: one fresh call of the timed kernel on the
    workload's original inputs, and the oracle on a sample of its sequences;
    the largest errors and whether they meet the tolerances (state max abs
    1e-4, output |o - o_ref| <= 1e-2 + 1e-2 |o_ref|).  Without the final
    write-back the pool slots must be bit-identical to the inputs and the
    state after each sequence's last token is read from the per-token states."""
    import oracle
    c = device_copy(w, torch, device)
    prepare(c)()
    torch.cuda.synchronize(device)
    rng = np.random.default_rng(0)
    seqs = np.sort(rng.choice(w.spec.N, size=min(nseq, w.spec.N), replace=False))
    args = oracle_subset_args(w, seqs)
    status, o_ref, s_ref, _ = oracle.update(*args)
    lens = w.seq_lens
    starts = np.concatenate([[0], np.cumsum(lens)])
    rows = np.concatenate([np.arange(starts[i], starts[i] + lens[i]) for i in seqs]).astype(np.int64)
    s = w.spec
    o_gpu = c["out"].reshape(w.T_tot, s.HV, s.V)[torch.from_numpy(rows).to(device)].float().cpu().numpy()
    o_ref = o_ref.reshape(o_gpu.shape)
    written = ~np.isnan(o_ref)
    err_o = np.abs(o_gpu.astype(np.float64) - o_ref)[written]
    ok_o = bool(np.all(err_o <= 1e-2 + 1e-2 * np.abs(o_ref[written])))
    slots = w.state_indices[seqs]
    live = slots >= 0
    pool_slots = torch.from_numpy(slots[live].astype(np.int64)).to(device)
    pool_untouched = None
    if final_writeback:
        s_gpu = c["state_pool"][pool_slots].cpu().numpy()
    else:
        pool_untouched = bool(np.array_equal(c["state_pool"][pool_slots].cpu().numpy(),
                                             w.state_pool[slots[live]]))
        last = [starts[i] + lens[i] - 1 for i in seqs[live]]
        s_gpu = c["inter"][torch.tensor(last, dtype=torch.int64, device=device)].cpu().numpy()
    err_s = float(np.abs(s_gpu.astype(np.float64) - s_ref).max()) if live.any() else 0.0
    del c
    res = {"sequences": int(len(seqs)), "tokens": int(len(rows)), "oracle_status": int(status),
           "max_abs_out_err": round(float(err_o.max()) if err_o.size else 0.0, 6),
           "max_abs_state_err": float(f"{err_s:.3e}"),
           "within_tolerance": ok_o and err_s <= 1e-4 and pool_untouched is not False}
    if pool_untouched is not None:
        res["pool_untouched"] = pool_untouched
    return res


def run_reference(args, w):
    """Reference arm: the CPU oracle on bounded per-step samples."""
    N = w.spec.N
    rng = np.random.default_rng(0)
    oracle_subset_seconds(w, np.arange(1))   # untimed: loads the oracle library
    t1 = oracle_subset_seconds(w, np.arange(min(8, N))) / min(8, N)
    budget = 120.0
    per_step = max(1, min(N, int(budget / max(1, args.steps + args.warmup) / max(t1, 1e-6))))
    for _ in range(args.warmup):
        oracle_subset_seconds(w, rng.choice(N, per_step, replace=False))
    tot_t, tot_b = 0.0, 0
    for _ in range(args.steps):
        seqs = np.sort(rng.choice(N, per_step, replace=False))
        tot_t += oracle_subset_seconds(w, seqs)
        tot_b += subset_bytes(w, seqs)
    value = tot_b / tot_t / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(tot_t / args.steps * 1e3, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(w, 1),
            "cpu_baseline": {"kind": "oracle", "cores": 1, "value": round(value, 4), "unit": "GB/s", "cpu": cpu_model(),
                             "sample": f"{per_step} random sequences of {w.spec.name} per step"},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

def kernel_name(schedule, tile_v, tile_rows, one_token, pairs, mean_tokens=1.0, chunk_ok=False, sms=148):
    """Name of the kernel the library launches for these settings (mirrors
    the library's documented choice, including the split schedule's state
    kernel: two CTAs per (sequence, head) pair while they fit one wave, the
    compact form from 2 pairs per SM at <= 128 tokens per sequence on
    average, else the full-width form)."""
    from gated_deltanet_recurrent_sigmoid_b200 import binding
    if schedule == binding.SCHEDULE_AUTO and not tile_v and not tile_rows and chunk_ok:
        if split_pays(pairs, mean_tokens, sms):
            schedule = binding.SCHEDULE_CHUNKED_SPLIT      # the binding passes a workspace
        elif mean_tokens >= chunked_min_mean_tokens(pairs):
            schedule = binding.SCHEDULE_CHUNKED
    if schedule == binding.SCHEDULE_CHUNKED_SPLIT:
        if 2 * pairs <= sms:
            state = "gdn_chunk_state_half_kernel"
        elif pairs >= 2 * sms and mean_tokens <= 128:
            state = "gdn_chunk_state_compact_kernel"
        else:
            state = "gdn_chunk_state_kernel"
        return f"gdn::split::gdn_chunk_wy_kernel<true> + gdn::split::{state}"
    if schedule == binding.SCHEDULE_PIPELINED:
        return "gdn::pipe::gdn_decode_pipelined_kernel<3>"
    if schedule == binding.SCHEDULE_CHUNKED:
        return "gdn::local::gdn_chunk_local_kernel<true>"
    if tile_v:
        bv, rows = tile_v, tile_rows or 16
    else:
        bv, rows = (64, 32) if one_token else ((32, 32) if pairs >= 2048 else ((8, 8) if pairs <= 64 else (16, 16)))
        rows = tile_rows or rows
    return f"gdn::gdn_decode_kernel<128,128,{bv},{128 // rows}>"


def workload_config(w, world, pdl=False):
    s = w.spec
    return {"workload": s.name, "B": s.N, "T": s.T if s.T is not None else f"U{{{s.min_len}..{s.max_len}}}",
            "H": s.H, "HV": s.HV,
            "K": s.K, "V": s.V, "num_slots": s.num_slots, "padded": int((w.state_indices < 0).sum()),
            "state_dtype": "f32", "activation_dtype": "bf16",
            "l2": f"inputs larger than L2: steps rotate over {ROTATING_COPIES} input copies",
            "launch": "programmatic dependent launch" if pdl else "plain stream order",
            "parallelism": "replicas" if world == 1 else f"dp{world}"}


def device_copy(w, torch, device):
    bf = lambda x: torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).to(device)
    d = dict(q=bf(w.q), k=bf(w.k), v=bf(w.v), a=bf(w.a), b=bf(w.b),
             A_log=torch.from_numpy(w.A_log).to(device), dt_bias=torch.from_numpy(w.dt_bias).to(device),
             state_pool=torch.from_numpy(w.state_pool).to(device),
             state_indices=torch.from_numpy(w.state_indices).to(device),
             cu_seqlens=None if w.cu_seqlens is None else torch.from_numpy(w.cu_seqlens).to(device))
    d["out"] = torch.empty(w.v.shape, dtype=torch.bfloat16, device=device)
    if w.spec.intermediate:
        d["inter"] = torch.empty((w.T_tot, w.spec.HV, w.spec.K, w.spec.V), device=device)
    return d


# the other workload families, timed after the headline one (per_config)
PER_CONFIG = [wl.TINY.name, wl.FULLHEAD_B256.name, wl.SPEC_B128_T4.name] + [wl.sweep_spec(n).name
                                                                             for n in wl.SWEEP_NS]
L2_FLUSH_BYTES = 256 << 20     # twice the B200's 126 MB L2


def oracle_sample_us(w, rng, max_seqs=16):
    """The oracle (single thread, fp64) on a random sample of the workload's
    sequences, scaled to the whole call by its share of the active
    (token, value head) pairs (padded and empty sequences cost nothing);
    returns (us per call, description of the sample)."""
    N = w.spec.N
    seqs = np.sort(rng.choice(N, size=min(max_seqs, N), replace=False))
    oracle_subset_seconds(w, seqs[:1])   # untimed: loads the oracle library
    secs = oracle_subset_seconds(w, seqs)
    live = w.state_indices >= 0
    work_all = int(w.seq_lens[live].sum()) + int(live.sum())
    work_smp = int(w.seq_lens[seqs][live[seqs]].sum()) + int(live[seqs].sum())
    scale = work_all / max(1, work_smp)
    return secs * scale * 1e6, (f"{len(seqs)} random sequences ({int(w.seq_lens[seqs].sum())} tokens) timed, "
                                f"scaled x{scale:.1f} by active tokens + sequences")


def per_config_table(torch, binding, device, stream, flags, peak, sms, launches=50):
    """Every other workload family through the library's default (AUTO) choice:
    one fresh call checked against the oracle on a sample of sequences, then
    `launches` isolated launches, each after an L2 flush (a 256 MB memset
    outside the event pair) and bracketed by CUDA events on the launch stream;
    the median launch against the measured HBM copy bandwidth, on the
    algorithmic bytes.  Multi-token calls that run the per-token kernel also
    report the fraction of the fp32 CUDA-core bound of their algorithmic
    flops."""
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    rng = np.random.default_rng(0)
    rows = []
    for name in PER_CONFIG:
        w = wl.generate(wl.BY_NAME[name])
        s = w.spec
        f = flags | (binding.WRITE_INTERMEDIATE if s.intermediate else 0)
        c = device_copy(w, torch, device)
        call = binding.PreparedCall(c["q"], c["k"], c["v"], c["a"], c["b"], c["A_log"], c["dt_bias"],
                                    c["state_pool"], c["state_indices"], c["cu_seqlens"], c["out"], flags=f,
                                    intermediate_states=c.get("inter"), stream=stream)
        par = parity_sample(w, lambda cc: binding.PreparedCall(
            cc["q"], cc["k"], cc["v"], cc["a"], cc["b"], cc["A_log"], cc["dt_bias"], cc["state_pool"],
            cc["state_indices"], cc["cu_seqlens"], cc["out"], flags=f, intermediate_states=cc.get("inter"),
            stream=stream), torch, device)
        for _ in range(3):
            call()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(launches)]
        with torch.cuda.stream(stream):
            for a_, b_ in ev:
                flush.zero_()
                a_.record(stream)
                call()
                b_.record(stream)
        torch.cuda.synchronize(device)
        us = float(np.median([a_.elapsed_time(b_) * 1e3 for a_, b_ in ev]))
        nbytes = wl.algorithmic_bytes(w)
        one_token = w.T_tot == s.N and not s.intermediate
        kname = kernel_name(binding.SCHEDULE_AUTO, 0, 0, one_token, s.N * s.HV, w.T_tot / max(1, s.N),
                            not s.intermediate, sms)
        o_us, o_how = oracle_sample_us(w, rng)
        row = {"workload": name, "kernel": kname, "us_per_call": round(us, 3),
               "gb_s": round(nbytes / (us * 1e-6) / 1e9, 2), "hbm_frac": round(nbytes / (us * 1e-6) / 1e9 / peak, 4),
               "algorithmic_bytes": nbytes, "oracle_us_per_call_1core": round(o_us, 1), "oracle_sample": o_how,
               "parity": par}
        if not one_token and "gdn_decode_kernel" in kname:
            row["alu_frac"] = round(wl.algorithmic_flops(w) / (us * 1e-6) / 1e12 / ALU_F32_PEAK_TFLOPS, 4)
        rows.append(row)
        del call, c
    del flush
    return {"rows": rows, "how": f"AUTO schedule, PDL flag as the headline; median of {launches} isolated "
                                 "launches, each after a 256 MB L2 flush outside its CUDA-event pair",
            "peak_gbs": peak}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=wl.DECODE_B512.name, choices=sorted(wl.BY_NAME))
    ap.add_argument("--copies", type=int, default=ROTATING_COPIES)
    ap.add_argument("--tile-v", type=int, default=0)
    ap.add_argument("--tile-rows", type=int, default=0)
    ap.add_argument("--schedule", default="auto", choices=["auto", "per_tile", "pipelined", "chunked", "split"])
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--e2e-depth", type=int, default=3,
                    help="host-fed steps in flight in the pipelined e2e loop (staging slots)")
    ap.add_argument("--skip-cpu-baseline", action="store_true")
    ap.add_argument("--skip-e2e", action="store_true")
    ap.add_argument("--skip-per-config", action="store_true",
                    help="omit the table of the other workload families (timed after the headline one)")
    ap.add_argument("--unfused", action="store_true",
                    help="time the two-kernel pair (gating, then the recurrence) instead of the fused update")
    ap.add_argument("--no-final-writeback", dest="final_writeback", action="store_false",
                    help="leave the pool untouched (GDN_NO_FINAL_WRITEBACK): the per-token states are the "
                         "result; requires a workload that writes them")
    ap.add_argument("--no-pdl", dest="pdl", action="store_false",
                    help="launch in plain stream order instead of with programmatic dependent launch")
    args = ap.parse_args()

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    w = wl.generate(wl.BY_NAME[args.workload])
    if not args.final_writeback and not w.spec.intermediate:
        ap.error("--no-final-writeback needs a workload that writes the per-token states")

    if args.impl == "reference":
        if rank == 0:
            run_reference(args, w)
        return

    import torch
    import torch.distributed as dist
    from gated_deltanet_recurrent_sigmoid_b200 import binding, build

    if world > 1:
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", device_id=torch.device("cuda", local_rank),
                                timeout=__import__("datetime").timedelta(seconds=120))
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    if local_rank == 0:
        build.build()
    if world > 1:
        dist.barrier()
    binding.load()

    schedule = {"auto": binding.SCHEDULE_AUTO, "per_tile": binding.SCHEDULE_PER_TILE,
                "pipelined": binding.SCHEDULE_PIPELINED, "chunked": binding.SCHEDULE_CHUNKED,
                "split": binding.SCHEDULE_CHUNKED_SPLIT}[args.schedule]
    stream = torch.cuda.Stream(device)
    copies = [device_copy(w, torch, device) for _ in range(max(1, args.copies))]
    flags = binding.L2NORM_QK | (binding.WRITE_INTERMEDIATE if w.spec.intermediate else 0)
    if not args.final_writeback:
        flags |= binding.NO_FINAL_WRITEBACK
    if args.pdl:
        flags |= binding.LAUNCH_PDL
    def prepare(c):
        if args.unfused:
            # the two-kernel baseline the fused update replaces (gating, then the
            # recurrence reading g and beta back from HBM)
            return binding.PreparedUnfusedCall(c["q"], c["k"], c["v"], c["a"], c["b"], c["A_log"], c["dt_bias"],
                                               c["state_pool"], c["state_indices"], c["cu_seqlens"], c["out"],
                                               flags=flags, intermediate_states=c.get("inter"), stream=stream,
                                               tile_v=args.tile_v, tile_rows=args.tile_rows)
        return binding.PreparedCall(c["q"], c["k"], c["v"], c["a"], c["b"], c["A_log"], c["dt_bias"],
                                    c["state_pool"], c["state_indices"], c["cu_seqlens"], c["out"], flags=flags,
                                    intermediate_states=c.get("inter"), stream=stream, tile_v=args.tile_v,
                                    schedule=schedule, tile_rows=args.tile_rows)

    calls = [prepare(c) for c in copies]
    nbytes = wl.algorithmic_bytes(w, final_writeback=args.final_writeback)
    torch.cuda.synchronize(device)

    # warm-up
    for s in range(args.warmup):
        calls[s % len(calls)]()
    stream.synchronize()

    # timed region: K steps, one fused kernel each, back to back on the launch
    # stream, bracketed by CUDA events on that stream (the region holds only
    # this kernel, so its average launch duration is the region time / K)
    region0 = torch.cuda.Event(enable_timing=True)
    region1 = torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(device)
    sampler = ClockSampler(local_rank)
    time.sleep(0.2)
    torch.cuda.nvtx.range_push(f"timed region: {args.steps} steps of {w.spec.name}")
    region0.record(stream)
    for s in range(args.steps):
        calls[s % len(calls)]()
    region1.record(stream)
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize(device)
    clocks = sampler.stop()
    if world > 1:
        dist.barrier()
    region_ms = region0.elapsed_time(region1)
    avg_kernel_ms = region_ms / args.steps

    t = torch.tensor([region_ms], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    max_region_ms = float(t.item())
    ms_per_step = max_region_ms / args.steps
    value = nbytes * world * args.steps / (max_region_ms * 1e-3) / 1e9

    # per-launch distribution: isolated launches, each bracketed by its own
    # events (so programmatic dependent launch cannot overlap neighbours)
    dist_n = min(args.steps, 300)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(dist_n)]
    for s_, (a_, b_) in enumerate(ev):
        a_.record(stream)
        calls[s_ % len(calls)]()
        b_.record(stream)
    torch.cuda.synchronize(device)
    per_launch = np.array([a_.elapsed_time(b_) * 1e3 for a_, b_ in ev])
    launch_us = {"p10": round(float(np.percentile(per_launch, 10)), 3),
                 "p50": round(float(np.percentile(per_launch, 50)), 3),
                 "p90": round(float(np.percentile(per_launch, 90)), 3), "launches": dist_n,
                 "how": "isolated launches, CUDA events around each, inputs rotating over the copies"}

    # end to end through the public API with pinned host buffers.  Every step
    # copies its inputs host -> device (one packed copy), runs the update and
    # copies its output back; the host receives every step's output.  The
    # pipelined loop (the headline e2e) overlaps a step's copies with the
    # neighbouring steps' kernels (the updates stay in order on one stream);
    # the serial loop synchronises on each step before issuing the next.
    e2e = e2e_serial = None
    if not args.skip_e2e:
        c0 = copies[0]
        s = w.spec
        staged_args = (c0["q"].shape[:-2], s.H, s.HV, s.K, s.V, s.N, c0["A_log"], c0["dt_bias"], c0["state_pool"])
        staged_kw = dict(varlen=c0["cu_seqlens"] is not None, flags=flags, intermediate_states=c0.get("inter"),
                         tile_v=args.tile_v, tile_rows=args.tile_rows, schedule=schedule)

        def fill(slot):
            for name in ("q", "k", "v", "a", "b", "state_indices", "cu_seqlens"):
                if c0.get(name) is not None:
                    getattr(slot, name).copy_(c0[name].cpu())

        def timed(run_steps):
            if world > 1:
                dist.barrier()
            torch.cuda.synchronize(device)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            last_stream = run_steps()
            e1.record(last_stream)
            torch.cuda.synchronize(device)
            te = torch.tensor([e0.elapsed_time(e1)], dtype=torch.float64, device=device)
            if world > 1:
                dist.all_reduce(te, op=dist.ReduceOp.MAX)
            return float(te.item()) / args.e2e_steps

        pipe = binding.PipelinedHostDecode(*staged_args, stream=stream, depth=args.e2e_depth, **staged_kw)
        for slot in pipe.slots:
            fill(slot)
        for _ in range(4):
            pipe.inputs()
            pipe.step()
        pipe.finish()

        def run_pipe():
            for _ in range(args.e2e_steps):
                pipe.inputs()
                pipe.step()
            pipe.finish()
            return pipe.copy_out

        torch.cuda.nvtx.range_push("e2e: pipelined host-fed steps")
        e2e_ms = timed(run_pipe)
        torch.cuda.nvtx.range_pop()
        link = h2d_link_gbs(int(pipe.h2d_bytes), device)
        e2e = {"value": round(nbytes * world / (e2e_ms * 1e-3) / 1e9, 3), "unit": "GB/s",
               "us_per_call": round(e2e_ms * 1e3, 3), "h2d_bytes_per_step": int(pipe.h2d_bytes),
               "d2h_bytes_per_step": int(pipe.d2h_bytes), "api": "binding.PipelinedHostDecode",
               "pipeline_depth": pipe.depth,
               # the host link's pinned host -> device rate, right after the loop:
               # a step cannot take less than h2d_bytes_per_step / this
               "h2d_link_gbs": link,
               "h2d_floor_us": round(pipe.h2d_bytes / (link * 1e3), 3) if link else None,
               "how": "each step: pinned host inputs -> device, update, output -> pinned host; the host "
                      "receives every step's output; copies overlap the neighbouring steps' kernels"}
        del pipe

        staged = binding.HostStagedDecode(*staged_args, stream=stream, **staged_kw)
        fill(staged)
        for _ in range(3):
            staged.step()
            stream.synchronize()

        def run_serial():
            for _ in range(args.e2e_steps):
                staged.step()
                stream.synchronize()      # the step ends when the host holds the output
            return stream

        torch.cuda.nvtx.range_push("e2e: serial host-fed steps")
        es_ms = timed(run_serial)
        torch.cuda.nvtx.range_pop()
        e2e_serial = {"value": round(nbytes * world / (es_ms * 1e-3) / 1e9, 3), "unit": "GB/s",
                      "us_per_call": round(es_ms * 1e3, 3), "api": "binding.HostStagedDecode",
                      "how": "each step synchronised before the next"}
        del staged

    if rank == 0:
        peak, peak_src = hbm_peak()
        achieved = nbytes / (avg_kernel_ms * 1e-3) / 1e9
        nflops = wl.algorithmic_flops(w)
        traffic = None
        if (NCU_TRAFFIC["kernel_sha256"] == kernel_source_hash() and NCU_TRAFFIC["workload"] == w.spec.name
                and not args.unfused and args.schedule in ("auto", "per_tile") and not args.tile_v
                and not args.tile_rows):
            traffic = NCU_TRAFFIC["bytes_per_launch"]
        kname = ("gdn::gdn_gating_kernel + " if args.unfused else "") + kernel_name(
            schedule, args.tile_v, args.tile_rows, w.T_tot == w.spec.N and not w.spec.intermediate,
            w.spec.N * w.spec.HV, w.T_tot / max(1, w.spec.N), not args.unfused and not w.spec.intermediate,
            torch.cuda.get_device_properties(device).multi_processor_count)
        line = {
            "metric": METRIC, "value": round(value, 3), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_per_step, 6), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": workload_config(w, world, args.pdl) | ({} if args.final_writeback else
                                                             {"final_writeback": False}),
            "us_per_call": round(avg_kernel_ms * 1e3, 3),
            "launch_us": launch_us,
            "hbm_frac": {"of_measured": round(achieved / peak, 4), "of_nominal": round(achieved / NOMINAL_HBM_GBS, 4),
                         "peak_source": peak_src},
            # every shape is rated against HBM on its algorithmic bytes; a
            # multi-token call on the per-token kernel also shows the fraction
            # of the fp32 CUDA-core bound of its per-token arithmetic
            "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak, "unit": "GB/s",
                         "frac": round(achieved / peak, 4), "traffic": traffic, "algorithmic_bytes_per_launch": nbytes,
                         "algorithmic_flops_per_launch": nflops, "hbm_peak_source": peak_src, "kernel": kname} | (
                {"alu_frac": round(nflops / (avg_kernel_ms * 1e-3) / 1e12 / ALU_F32_PEAK_TFLOPS, 4),
                 "alu_peak_tflops": round(ALU_F32_PEAK_TFLOPS, 2),
                 "alu_peak_source": "derived: 148 SMs x 128 fp32 lanes x 2 x 1965 MHz"}
                if w.T_tot != w.spec.N and "gdn_decode_kernel" in kname else {}),
            "e2e": e2e,
            "e2e_serial": e2e_serial,
            "gpu_launches": args.steps * (2 if args.unfused or "+" in kname else 1),
            "gpu_launches_note": "launches inside the timed region; the per-launch distribution and e2e run after it",
            "clocks": clocks,
        }
        if world == 1 and not args.skip_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(w)
            line["cpu_baseline_all_cores"] = cpu_baseline_all_cores(w)
            line["parity"] = parity_sample(w, prepare, torch, device, final_writeback=args.final_writeback)
        if world == 1 and not args.skip_per_config and w.spec.name == wl.DECODE_B512.name:
            line["per_config"] = per_config_table(torch, binding, device, stream,
                                                  binding.L2NORM_QK | (binding.LAUNCH_PDL if args.pdl else 0), peak,
                                                  torch.cuda.get_device_properties(device).multi_processor_count)
        print(json.dumps(line), flush=True)

    del calls
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
