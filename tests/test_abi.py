"""The C-ABI library on the CPU: it loads, exports every declared symbol,
and its host-side validation rejects bad arguments before any CUDA call.

These tests never launch a kernel: every call below either fails a host
check or has nothing to do (N = 0), so no GPU is needed.
"""
import ctypes
import os
import re
import subprocess

import pytest
import torch

from gated_deltanet_recurrent_sigmoid_b200 import binding, build

HEADER = os.path.join(build.INCLUDE, "gdn_decode.h")


def declared_functions():
    text = open(HEADER).read()
    return re.findall(r"GDN_API\s+[\w\s\*]+?\b(gdn_\w+)\s*\(", text)


def test_header_declares_the_abi():
    assert set(declared_functions()) == {"gdn_decode_update", "gdn_recurrent_update", "gdn_gating",
                                         "gdn_status_string", "gdn_version", "gdn_chunked_workspace_bytes",
                                         "gdn_decode_update_static_scratch", "gdn_host_step_issue",
                                         "gdn_static_scratch_bytes"}


def test_library_exports_every_declared_symbol(gdn_lib):
    nm = subprocess.run(["nm", "-D", "--defined-only", build.LIB_PATH], capture_output=True, text=True,
                        check=True).stdout
    exported = {line.split()[-1] for line in nm.splitlines() if " T " in line}
    for name in declared_functions():
        assert name in exported, name
        assert hasattr(gdn_lib, name)
    # nothing else leaks out of the library
    assert {e for e in exported if e.startswith("gdn")} == set(declared_functions())


def test_version_matches_header(gdn_lib):
    m = re.search(r"#define GDN_DECODE_ABI_VERSION (\d+)", open(HEADER).read())
    assert gdn_lib.gdn_version() == int(m.group(1))


def test_status_strings(gdn_lib):
    for code in range(0, -11, -1):
        s = binding.status_string(code)
        assert s and "unknown" not in s
    assert "unknown" in binding.status_string(-100)


def test_header_constants_match_binding():
    text = open(HEADER).read()
    def define(name):
        m = re.search(rf"#define {name}\s+\(?(-?\d+)(u << (\d+))?\)?", text)
        return int(m.group(1)) << int(m.group(3)) if m.group(3) else int(m.group(1))
    assert define("GDN_L2NORM_QK") == binding.L2NORM_QK
    assert define("GDN_WRITE_INTERMEDIATE") == binding.WRITE_INTERMEDIATE
    assert define("GDN_NO_FINAL_WRITEBACK") == binding.NO_FINAL_WRITEBACK
    assert define("GDN_CHECK_INDICES") == binding.CHECK_INDICES
    assert define("GDN_LAUNCH_PDL") == binding.LAUNCH_PDL
    for name in ("AUTO", "PER_TILE", "PIPELINED", "CHUNKED", "CHUNKED_SPLIT"):
        assert define(f"GDN_SCHEDULE_{name}") == getattr(binding, f"SCHEDULE_{name}")
    for name, val in [("GDN_ERR_NULL_ARG", -1), ("GDN_ERR_DTYPE", -2), ("GDN_ERR_SHAPE", -3),
                      ("GDN_ERR_ALIGN", -4), ("GDN_ERR_ALIAS", -5), ("GDN_ERR_UNSUPPORTED", -6),
                      ("GDN_ERR_ARG", -7), ("GDN_ERR_INDICES", -8), ("GDN_ERR_CUDA", -9),
                      ("GDN_ERR_SCRATCH", -10)]:
        assert int(re.search(rf"#define {name}\s+\((-?\d+)\)", text).group(1)) == val
    assert ctypes.sizeof(binding.GdnTensor) == 8 + 4 + 4 + 8 * 4 + 8 * 4
    assert ctypes.sizeof(binding.GdnExtra) == 8 + 8 + 8 + 4 * 4 + 8 + 8
    # 11 descriptors, scale + flags, extra, 2 x (2 pointers + size), 2 streams, 3 events, reused (+ padding)
    assert ctypes.sizeof(binding.GdnHostStep) == 11 * 8 + 8 + 8 + 2 * 24 + 16 + 24 + 8


def make(N=4, T=1, H=2, HV=4, K=128, V=128, slots=8, varlen=True):
    """CPU tensors shaped like a valid call (host pointers are fine for the
    host checks; the library never dereferences them before launching)."""
    bf = torch.bfloat16
    lead = (N * T,) if varlen else (N, T)
    t = dict(q=torch.zeros(*lead, H, K, dtype=bf), k=torch.zeros(*lead, H, K, dtype=bf),
             v=torch.zeros(*lead, HV, V, dtype=bf), a=torch.zeros(*lead, HV, dtype=bf),
             b=torch.zeros(*lead, HV, dtype=bf), A_log=torch.zeros(HV), dt_bias=torch.zeros(HV),
             state_pool=torch.zeros(slots, HV, K, V), state_indices=torch.arange(N, dtype=torch.int32),
             cu_seqlens=torch.arange(0, N * T + 1, T, dtype=torch.int32) if varlen else None,
             out=torch.zeros(*lead, HV, V, dtype=bf))
    return t


def call(t, **kw):
    return binding.decode_update(t["q"], t["k"], t["v"], t["a"], t["b"], t["A_log"], t["dt_bias"],
                                 t["state_pool"], t["state_indices"], t["cu_seqlens"], t["out"],
                                 stream=None, **kw)


def expect(code, t, **kw):
    with pytest.raises(binding.GdnError) as e:
        call(t, **kw)
    assert e.value.status == code, binding.status_string(e.value.status)


def test_empty_batch_is_ok_without_launch(gdn_lib):
    t = make(N=0)
    assert call(t) is t["out"]
    t = make(N=3, T=0, varlen=False)
    call(t)


def test_rejects_bad_dtypes_and_shapes(gdn_lib):
    t = make(); t["q"] = t["q"].float(); expect(binding.ERR_DTYPE, t)
    t = make(); t["state_pool"] = t["state_pool"].double(); expect(binding.ERR_DTYPE, t)
    t = make(); t["state_indices"] = t["state_indices"].long(); expect(binding.ERR_DTYPE, t)
    t = make(); t["v"] = t["v"][:, :3]; expect(binding.ERR_SHAPE, t)            # HV mismatch with out
    t = make(HV=3); expect(binding.ERR_SHAPE, t)                                  # HV % H != 0
    t = make(); t["cu_seqlens"] = t["cu_seqlens"][:-1]; expect(binding.ERR_SHAPE, t)
    t = make(); t["A_log"] = torch.zeros(3); expect(binding.ERR_SHAPE, t)
    t = make(); t["state_pool"] = t["state_pool"].transpose(2, 3); expect(binding.ERR_SHAPE, t)
    t = make(varlen=False, T=2); t["q"] = t["q"][:, :, :, :64]; expect(binding.ERR_SHAPE, t)


def test_rejects_unsupported_head_size(gdn_lib):
    expect(binding.ERR_UNSUPPORTED, make(K=64, V=64))
    expect(binding.ERR_UNSUPPORTED, make(), tile_v=128)
    expect(binding.ERR_UNSUPPORTED, make(), tile_v=16, tile_rows=32)
    expect(binding.ERR_ARG, make(), schedule=7)


def test_rejects_misalignment(gdn_lib):
    t = make()
    raw = torch.zeros(t["q"].numel() + 8, dtype=torch.bfloat16)
    t["q"] = raw[1:1 + t["q"].numel()].view(t["q"].shape)                         # 2-byte offset
    expect(binding.ERR_ALIGN, t)
    t = make()
    raw = torch.zeros(t["state_pool"].numel() + 4)
    t["state_pool"] = raw[1:1 + t["state_pool"].numel()].view(t["state_pool"].shape)
    expect(binding.ERR_ALIGN, t)


def test_rejects_aliasing(gdn_lib):
    t = make(); t["out"] = t["v"]; expect(binding.ERR_ALIAS, t)
    t = make(); t["A_log"] = t["state_pool"].view(-1)[:4]; expect(binding.ERR_ALIAS, t)
    t = make(); buf = torch.zeros(2 * t["out"].numel(), dtype=torch.bfloat16)
    t["out"] = buf[: t["out"].numel()].view(t["out"].shape)
    t["v"] = buf[t["out"].numel() // 2:][: t["v"].numel()].view(t["v"].shape)   # half overlap
    expect(binding.ERR_ALIAS, t)


def test_rejects_bad_scalars_and_flags(gdn_lib):
    expect(binding.ERR_ARG, make(), scale=0.0)
    expect(binding.ERR_ARG, make(), scale=float("nan"))
    expect(binding.ERR_ARG, make(), flags=1 << 7)


def test_intermediate_required_with_flag(gdn_lib):
    expect(binding.ERR_NULL_ARG, make(), flags=binding.L2NORM_QK | binding.WRITE_INTERMEDIATE)


def test_binding_fails_loudly_without_library(monkeypatch):
    monkeypatch.setattr(binding, "_LIB", None)
    monkeypatch.setattr(build, "LIB_PATH", "/nonexistent/libgdn_decode.so")
    with pytest.raises(binding.GdnError):
        binding.load()


def test_chunked_workspace_bytes(gdn_lib):
    """One 131,584-byte record per (64-token block, value head); host-only."""
    rec = 131584
    assert binding.chunked_workspace_bytes(0, 8) == 0
    assert binding.chunked_workspace_bytes(5, 0) == 0
    assert binding.chunked_workspace_bytes(1, 1) == rec
    assert binding.chunked_workspace_bytes(64, 8) == 8 * rec
    assert binding.chunked_workspace_bytes(65, 8) == 16 * rec
    assert binding.chunked_workspace_bytes(13488, 8) == 211 * 8 * rec
    assert rec % 256 == 0


def test_split_schedule_checks_its_workspace(gdn_lib):
    """GDN_SCHEDULE_CHUNKED_SPLIT needs a workspace: missing, too small,
    misaligned or overlapping a tensor of the call is rejected before any
    launch; AUTO ignores one that is too small."""
    split = binding.SCHEDULE_CHUNKED_SPLIT
    t = make(N=2, T=3)
    need = binding.chunked_workspace_bytes(6, 4)
    expect(binding.ERR_NULL_ARG, t, schedule=split, workspace=None)
    raw = torch.empty(need + 512, dtype=torch.uint8)
    off = (-raw.data_ptr()) % 256                                       # 256-byte aligned view
    expect(binding.ERR_ARG, t, schedule=split, workspace=raw[off:off + need - 256])
    expect(binding.ERR_ALIGN, t, schedule=split, workspace=raw[off + 16:off + 16 + need])
    t2 = make(N=2, T=3)
    raw = torch.zeros(need // 4 + t2["state_pool"].numel() + 64, dtype=torch.float32)
    big = raw[((-raw.data_ptr()) % 256) // 4:]                                         # 256-byte aligned
    t2["state_pool"] = big[: t2["state_pool"].numel()].view(t2["state_pool"].shape)   # workspace overlaps the pool
    expect(binding.ERR_ALIAS, t2, schedule=split, workspace=big.view(torch.uint8)[:need])


def test_host_step_rejects_missing_pointers(gdn_lib):
    """gdn_host_step_issue checks its pointers before any CUDA call."""
    assert gdn_lib.gdn_host_step_issue(None) == binding.ERR_NULL_ARG
    st = binding.GdnHostStep()
    assert gdn_lib.gdn_host_step_issue(ctypes.byref(st)) == binding.ERR_NULL_ARG
    extra = binding.GdnExtra()
    st.extra = ctypes.pointer(extra)
    buf = (ctypes.c_char * 64)()
    st.host_in = st.dev_in = st.dev_out = st.host_out = ctypes.addressof(buf)
    st.ev_h2d = st.ev_ran = None
    assert gdn_lib.gdn_host_step_issue(ctypes.byref(st)) == binding.ERR_NULL_ARG


def test_struct_layouts_match_the_c_header(tmp_path):
    """Every field offset and struct size of the ctypes mirrors equals what a
    C compiler makes of include/gdn_decode.h."""
    import shutil
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    structs = {"gdn_tensor": binding.GdnTensor, "gdn_extra": binding.GdnExtra, "gdn_host_step": binding.GdnHostStep}
    lines = ["#include <stdio.h>", "#include <stddef.h>", '#include "gdn_decode.h"', "int main(void) {"]
    for cname, py in structs.items():
        lines.append(f'    printf("{cname} size %zu\\n", sizeof({cname}));')
        for fname, _ in py._fields_:
            lines.append(f'    printf("{cname} {fname} %zu\\n", offsetof({cname}, {fname}));')
    lines += ["    return 0;", "}"]
    src = tmp_path / "layout.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "layout"
    subprocess.run([cc, "-std=c99", "-I", os.path.dirname(HEADER), str(src), "-o", str(exe)], check=True)
    got = {}
    for line in subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.splitlines():
        cname, field, value = line.split()
        got[(cname, field)] = int(value)
    for cname, py in structs.items():
        assert got[(cname, "size")] == ctypes.sizeof(py), cname
        for fname, _ in py._fields_:
            assert got[(cname, fname)] == getattr(py, fname).offset, (cname, fname)


def test_static_scratch_size_matches_binding(gdn_lib):
    """The binding's constant equals the array size the library was built
    with (gdn_static_scratch_bytes) and the header's #define."""
    assert gdn_lib.gdn_static_scratch_bytes() == binding.STATIC_SCRATCH_BYTES
    m = re.search(r"#define GDN_STATIC_SCRATCH_BYTES \((\d+)ull << (\d+)\)", open(HEADER).read())
    assert int(m.group(1)) << int(m.group(2)) == binding.STATIC_SCRATCH_BYTES


def _static_call(gdn_lib, t, extra=None):
    descs = [binding.describe(t[n]) for n in ("q", "k", "v", "a", "b", "A_log", "dt_bias", "state_pool",
                                                "state_indices", "cu_seqlens", "out")]
    return gdn_lib.gdn_decode_update_static_scratch(*[binding._ref(d) for d in descs], ctypes.c_float(0.088),
                                                    ctypes.c_uint32(binding.L2NORM_QK),
                                                    ctypes.byref(extra) if extra is not None else None)


def test_static_scratch_guards_run_before_any_cuda_call(gdn_lib):
    """gdn_decode_update_static_scratch rejects a caller workspace, a nonzero
    workspace size, a schedule other than AUTO / CHUNKED_SPLIT, a call too
    large for its array and hostile shapes -- all before any CUDA call (so
    on this GPU-less host), leaving `out` untouched."""
    for field, value in [("workspace", 256), ("workspace_bytes", 4096),
                         ("schedule", binding.SCHEDULE_PER_TILE), ("schedule", binding.SCHEDULE_CHUNKED),
                         ("schedule", 9)]:
        t = make(N=2, T=3)
        t["out"].fill_(7.0)
        extra = binding.GdnExtra()
        setattr(extra, field, value)
        assert _static_call(gdn_lib, t, extra) == binding.ERR_ARG, (field, value)
        assert bool((t["out"] == 7.0).all())
    # 4160 tokens x 8 heads need 520 records > the 510 that fit in 64 MiB:
    # strides of zero give a large shape with no storage behind it
    T, H, HV = 4160, 4, 8
    assert binding.chunked_workspace_bytes(T, HV) > binding.STATIC_SCRATCH_BYTES
    t = make(N=2, T=3, H=H, HV=HV)
    t["v"] = torch.zeros(1, HV, 128, dtype=torch.bfloat16).expand(T, HV, 128)
    assert _static_call(gdn_lib, t) == binding.ERR_SCRATCH
    # leading dims whose product overflows 64 bits are a shape error, not a
    # wrapped size that slips past the check
    d = binding.describe(torch.zeros(1, 1, HV, 128, dtype=torch.bfloat16))
    for shape in [(1 << 40, 1 << 40), (-1, 4), (1 << 31, 1), (65536, 65536)]:
        d.shape[0], d.shape[1] = shape
        descs = [binding.describe(t[n]) for n in ("q", "k")] + [d] + \
                [binding.describe(t[n]) for n in ("a", "b", "A_log", "dt_bias", "state_pool", "state_indices",
                                                  "cu_seqlens", "out")]
        rc = gdn_lib.gdn_decode_update_static_scratch(*[ctypes.byref(x) for x in descs], ctypes.c_float(0.088),
                                                      ctypes.c_uint32(1), None)
        assert rc == binding.ERR_SHAPE, shape


def test_chunked_workspace_bytes_saturates(gdn_lib):
    assert binding.chunked_workspace_bytes(1 << 62, 1 << 30) == (1 << 64) - 1
    assert binding.chunked_workspace_bytes((1 << 31) - 1, (1 << 31) - 1) == (1 << 64) - 1
