"""bench.py's command-line contract, on the CPU.

The reference arm (the oracle on the host cores) prints the one JSON line the
driver parses, with the keys the base contract and the reference arm require;
the kernel-name mirror follows the library's documented choices (the names
are what the bench line reports as the dominant kernel)."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from gated_deltanet_recurrent_sigmoid_b200 import binding  # noqa: E402


def test_reference_arm_prints_the_contract_line():
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "tiny_b4", "--steps", "2",
                        "--warmup", "1"], cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e", "gpu_launches"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] == 1 and d["n_gpus"] == 1
    assert d["config"]["workload"] == "tiny_b4" and d["value"] > 0 and d["higher_is_better"] is True
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert d["gpu_launches"] == 0


@pytest.mark.parametrize("one_token,pairs,mean,expected", [
    (True, 4096, 1.0, "gdn::gdn_decode_kernel<128,128,64,4>"),                  # decode: 64x32
    (False, 4096, 4.0, "gdn::gdn_decode_kernel<128,128,32,4>"),                 # many short chains: 32x32
    (False, 1024, 4.0, "gdn::gdn_decode_kernel<128,128,16,8>"),                 # spec decode: 16x16
    (False, 8, 12.0, "gdn::gdn_decode_kernel<128,128,8,16>"),                   # few short chains: 8x8
    (False, 8, 29.0, "gdn::local::gdn_chunk_local_kernel<true>"),               # sweep_b1
    (False, 8192, 31.8, "gdn::local::gdn_chunk_local_kernel<true>"),            # sweep_b1024
    (False, 64, 1686.0, "gdn::split::gdn_chunk_wy_kernel<true> + gdn::split::gdn_chunk_state_half_kernel"),
    (False, 512, 480.0, "gdn::local::gdn_chunk_local_kernel<true>"),           # prefill_b64_t512
    (False, 256, 600.0, "gdn::split::gdn_chunk_wy_kernel<true> + gdn::split::gdn_chunk_state_kernel"),
    (False, 128, 150.0, "gdn::local::gdn_chunk_local_kernel<true>"),
    (False, 64, 90.0, "gdn::split::gdn_chunk_wy_kernel<true> + gdn::split::gdn_chunk_state_half_kernel"),
    (False, 96, 130.0, "gdn::local::gdn_chunk_local_kernel<true>"),
    (False, 96, 150.0, "gdn::split::gdn_chunk_wy_kernel<true> + gdn::split::gdn_chunk_state_kernel"),
    (False, 1024, 12.0, "gdn::gdn_decode_kernel<128,128,16,8>"),
])
def test_kernel_name_mirrors_the_documented_choice(one_token, pairs, mean, expected):
    assert bench.kernel_name(binding.SCHEDULE_AUTO, 0, 0, one_token, pairs, mean, chunk_ok=not one_token,
                             sms=148) == expected


def test_split_schedule_names_its_state_kernel():
    def name(pairs, mean):
        return bench.kernel_name(binding.SCHEDULE_CHUNKED_SPLIT, 0, 0, False, pairs, mean, sms=148).split("::")[-1]
    assert name(8192, 32.0) == "gdn_chunk_state_compact_kernel"     # many short sequences
    assert name(74, 32.0) == "gdn_chunk_state_half_kernel"          # two CTAs per pair fit one wave
    assert name(75, 2000.0) == "gdn_chunk_state_kernel"
    assert name(296, 129.0) == "gdn_chunk_state_kernel"


def test_auto_thresholds_match_the_header():
    """The thresholds the bench mirrors are the ones the header documents."""
    header = " ".join(open(os.path.join(ROOT, "include", "gdn_decode.h")).read().split())
    assert ("L >= 80 (2 P <= the device's SM count), >= 144 (P < 128), >= 192 (P < 256) or >= 512 (P < 512)"
            in header)
    assert "L >= 20 (P < 64), >= 14 (P < 512) or >= 13" in header
    assert [bench.split_pays(p, m) for p, m in ((74, 80), (74, 79), (75, 144), (75, 143), (127, 144), (127, 143),
                                                (128, 192), (128, 191), (511, 512), (511, 511),
                                                (512, 100000))] == [True, False, True, False, True, False, True,
                                                                    False, True, False, False]
    assert bench.split_pays(64, 100, sms=120) is False and bench.split_pays(64, 100, sms=128) is True
    assert [bench.chunked_min_mean_tokens(p) for p in (8, 63, 64, 511, 512, 8192)] == [20, 20, 14, 14, 13, 13]
