"""Thin ctypes binding of ``libgdn_decode.so`` (C ABI in include/gdn_decode.h).

Argument marshalling only: torch tensors are described to the C ABI by
their device pointer, dtype, shape and strides, and the current CUDA stream
is passed along.  Every step of the update runs in the library's kernel.
The library is loaded on first use; if it is missing this module raises --
there is no fallback path.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import List, Optional

import torch

from . import build as _build

L2NORM_QK = 1 << 0
WRITE_INTERMEDIATE = 1 << 1
NO_FINAL_WRITEBACK = 1 << 2
CHECK_INDICES = 1 << 3
LAUNCH_PDL = 1 << 4

DEV_BAD_SLOT = 1
DEV_BAD_SEQLENS = 2
DEV_TIMEOUT = 4

SCHEDULE_AUTO = 0
SCHEDULE_PER_TILE = 1
SCHEDULE_PIPELINED = 2
SCHEDULE_CHUNKED = 3
SCHEDULE_CHUNKED_SPLIT = 4

OK = 0
ERR_NULL_ARG, ERR_DTYPE, ERR_SHAPE, ERR_ALIGN, ERR_ALIAS = -1, -2, -3, -4, -5
ERR_UNSUPPORTED, ERR_ARG, ERR_INDICES, ERR_CUDA = -6, -7, -8, -9
ERR_SCRATCH = -10
STATIC_SCRATCH_BYTES = 64 << 20     # gdn_decode_update_static_scratch's built-in array (checked
                                    # against the library's gdn_static_scratch_bytes() by the tests)

_DTYPE_CODES = {torch.bfloat16: 1, torch.float32: 2, torch.int32: 3}


class GdnError(RuntimeError):
    """A non-zero status from the C ABI."""

    def __init__(self, status: int, message: str):
        super().__init__(message)
        self.status = status


class GdnTensor(ctypes.Structure):
    _fields_ = [("data", ctypes.c_void_p), ("dtype", ctypes.c_int32), ("ndim", ctypes.c_int32),
                ("shape", ctypes.c_int64 * 4), ("stride", ctypes.c_int64 * 4)]


class GdnExtra(ctypes.Structure):
    _fields_ = [("stream", ctypes.c_void_p), ("intermediate_states", ctypes.POINTER(GdnTensor)),
                ("device_status", ctypes.c_void_p), ("tile_v", ctypes.c_int32),
                ("tile_rows", ctypes.c_int32), ("schedule", ctypes.c_int32), ("reserved", ctypes.c_int32),
                ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_uint64)]


class GdnHostStep(ctypes.Structure):
    _fields_ = ([(n, ctypes.POINTER(GdnTensor)) for n in
                 ("q", "k", "v", "a", "b", "A_log", "dt_bias", "state_pool", "state_indices", "cu_seqlens", "out")] +
                [("scale", ctypes.c_float), ("flags", ctypes.c_uint32), ("extra", ctypes.POINTER(GdnExtra)),
                 ("host_in", ctypes.c_void_p), ("dev_in", ctypes.c_void_p), ("in_bytes", ctypes.c_uint64),
                 ("dev_out", ctypes.c_void_p), ("host_out", ctypes.c_void_p), ("out_bytes", ctypes.c_uint64),
                 ("copy_in_stream", ctypes.c_void_p), ("copy_out_stream", ctypes.c_void_p),
                 ("ev_h2d", ctypes.c_void_p), ("ev_ran", ctypes.c_void_p), ("ev_d2h", ctypes.c_void_p),
                 ("reused", ctypes.c_int32)])


_LIB = None


def library_path() -> str:
    return _build.LIB_PATH


def load() -> ctypes.CDLL:
    """Load the in-tree library; raise if it has not been built."""
    global _LIB
    if _LIB is None:
        path = _build.LIB_PATH
        if not os.path.exists(path):
            raise GdnError(ERR_CUDA, f"{path} is missing: build it with "
                                     "`python -m gated_deltanet_recurrent_sigmoid_b200.build`")
        lib = ctypes.CDLL(path)
        P = ctypes.POINTER(GdnTensor)
        lib.gdn_decode_update.restype = ctypes.c_int
        lib.gdn_decode_update.argtypes = [P] * 11 + [ctypes.c_float, ctypes.c_uint32, ctypes.POINTER(GdnExtra)]
        lib.gdn_recurrent_update.restype = ctypes.c_int
        lib.gdn_recurrent_update.argtypes = [P] * 9 + [ctypes.c_float, ctypes.c_uint32, ctypes.POINTER(GdnExtra)]
        lib.gdn_gating.restype = ctypes.c_int
        lib.gdn_gating.argtypes = [P] * 6 + [ctypes.POINTER(GdnExtra)]
        lib.gdn_status_string.restype = ctypes.c_char_p
        lib.gdn_status_string.argtypes = [ctypes.c_int]
        lib.gdn_version.restype = ctypes.c_int
        lib.gdn_version.argtypes = []
        lib.gdn_chunked_workspace_bytes.restype = ctypes.c_uint64
        lib.gdn_chunked_workspace_bytes.argtypes = [ctypes.c_int64, ctypes.c_int64]
        lib.gdn_host_step_issue.restype = ctypes.c_int
        lib.gdn_host_step_issue.argtypes = [ctypes.POINTER(GdnHostStep)]
        lib.gdn_static_scratch_bytes.restype = ctypes.c_uint64
        lib.gdn_static_scratch_bytes.argtypes = []
        lib.gdn_decode_update_static_scratch.restype = ctypes.c_int
        lib.gdn_decode_update_static_scratch.argtypes = [P] * 11 + [ctypes.c_float, ctypes.c_uint32,
                                                                    ctypes.POINTER(GdnExtra)]
        _LIB = lib
    return _LIB


def status_string(status: int) -> str:
    return load().gdn_status_string(int(status)).decode()


def describe(t: Optional[torch.Tensor]) -> Optional[GdnTensor]:
    """gdn_tensor descriptor of a tensor (None stays None)."""
    if t is None:
        return None
    if t.dim() < 1 or t.dim() > 4:
        raise GdnError(ERR_SHAPE, f"rank {t.dim()} tensor cannot cross the C ABI")
    d = GdnTensor()
    d.data = t.data_ptr()
    d.dtype = _DTYPE_CODES.get(t.dtype, 0)
    d.ndim = t.dim()
    for i, (n, s) in enumerate(zip(t.shape, t.stride())):
        d.shape[i] = n
        d.stride[i] = s
    return d


def _ref(d: Optional[GdnTensor]):
    return None if d is None else ctypes.byref(d)


def chunked_workspace_bytes(T_tot: int, HV: int) -> int:
    """Workspace bytes of GDN_SCHEDULE_CHUNKED_SPLIT (gdn_chunked_workspace_bytes)."""
    return int(load().gdn_chunked_workspace_bytes(int(T_tot), int(HV)))


def _workspace_for(workspace, schedule: int, q: torch.Tensor, v: torch.Tensor, N: int):
    """The workspace to pass: the caller's tensor, or (workspace="auto") one
    allocated here when the split chunked schedule is asked for, or when the
    library may choose it (AUTO with fewer than 512 (sequence, value head)
    pairs and at least 80 tokens per sequence on average -- the library's
    widest range for the split kernels)."""
    if workspace is None or isinstance(workspace, torch.Tensor):
        return workspace
    if workspace != "auto":
        raise ValueError("workspace must be a tensor, None or 'auto'")
    T_tot = v.numel() // (v.shape[-1] * v.shape[-2]) if v.dim() >= 2 else 0
    HV = v.shape[-2] if v.dim() >= 2 else 0
    if not (schedule == SCHEDULE_CHUNKED_SPLIT or (schedule == SCHEDULE_AUTO and N > 0 and N * HV < 512 and T_tot >= 80 * N)):
        return None
    nbytes = chunked_workspace_bytes(T_tot, HV)
    return torch.empty(nbytes, dtype=torch.uint8, device=q.device) if nbytes else None


def _set_workspace(extra: GdnExtra, ws: Optional[torch.Tensor]) -> None:
    extra.workspace = ws.data_ptr() if ws is not None and ws.numel() else None
    extra.workspace_bytes = ws.numel() * ws.element_size() if ws is not None else 0


def decode_update(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, a: torch.Tensor, b: torch.Tensor,
                  A_log: torch.Tensor, dt_bias: torch.Tensor, state_pool: torch.Tensor,
                  state_indices: torch.Tensor, cu_seqlens: Optional[torch.Tensor], out: torch.Tensor,
                  scale: Optional[float] = None, flags: int = L2NORM_QK,
                  intermediate_states: Optional[torch.Tensor] = None,
                  device_status: Optional[torch.Tensor] = None,
                  stream: Optional[torch.cuda.Stream] = None, tile_v: int = 0,
                  schedule: int = SCHEDULE_AUTO, tile_rows: int = 0, workspace="auto") -> torch.Tensor:
    """Fused sigmoid-gating GDN decode update, in place on ``state_pool``.

    Shapes, dtypes and semantics are those of ``gdn_decode_update`` in
    include/gdn_decode.h.  ``scale`` defaults to 1/sqrt(K).  ``flags`` gets
    WRITE_INTERMEDIATE added automatically when ``intermediate_states`` is
    given.  Runs asynchronously on ``stream`` (default: the current torch
    stream).  ``workspace``: a uint8 device tensor for the split chunked
    schedule, None, or "auto" (allocated here with torch when that schedule
    is asked for or may be chosen).  Returns ``out``.  Raises GdnError on a
    non-zero status.
    """
    lib = load()
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    if intermediate_states is not None:
        flags |= WRITE_INTERMEDIATE
    if stream is None:
        stream = torch.cuda.current_stream(q.device) if q.is_cuda else None
    descs = [describe(t) for t in (q, k, v, a, b, A_log, dt_bias, state_pool, state_indices, cu_seqlens, out)]
    inter = describe(intermediate_states)
    extra = GdnExtra()
    extra.stream = stream.cuda_stream if stream is not None else None
    extra.intermediate_states = ctypes.pointer(inter) if inter is not None else None
    extra.device_status = device_status.data_ptr() if device_status is not None else None
    extra.tile_v = int(tile_v)
    extra.tile_rows = int(tile_rows)
    extra.schedule = int(schedule)
    ws = _workspace_for(workspace, schedule, q, v, state_indices.shape[0])
    _set_workspace(extra, ws)
    status = lib.gdn_decode_update(*[_ref(d) for d in descs], ctypes.c_float(scale), ctypes.c_uint32(flags),
                                   ctypes.byref(extra))
    if status != OK:
        raise GdnError(status, status_string(status))
    return out


def decode_update_static_scratch(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, a: torch.Tensor,
                                 b: torch.Tensor, A_log: torch.Tensor, dt_bias: torch.Tensor,
                                 state_pool: torch.Tensor, state_indices: torch.Tensor,
                                 cu_seqlens: Optional[torch.Tensor], out: torch.Tensor,
                                 scale: Optional[float] = None, flags: int = L2NORM_QK,
                                 device_status: Optional[torch.Tensor] = None,
                                 stream: Optional[torch.cuda.Stream] = None) -> torch.Tensor:
    """``gdn_decode_update_static_scratch``: the split chunked update with the
    library's built-in scratch array, for callers that cannot allocate device
    memory.  Nothing is allocated here either.  Calls that may overlap on the
    GPU share the array and must be ordered (e.g. issued on one stream).
    Raises GdnError (ERR_SCRATCH when the call needs more than
    STATIC_SCRATCH_BYTES of scratch)."""
    lib = load()
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    if stream is None:
        stream = torch.cuda.current_stream(q.device) if q.is_cuda else None
    descs = [describe(t) for t in (q, k, v, a, b, A_log, dt_bias, state_pool, state_indices, cu_seqlens, out)]
    extra = GdnExtra()
    extra.stream = stream.cuda_stream if stream is not None else None
    extra.device_status = device_status.data_ptr() if device_status is not None else None
    status = lib.gdn_decode_update_static_scratch(*[_ref(d) for d in descs], ctypes.c_float(scale),
                                                  ctypes.c_uint32(flags), ctypes.byref(extra))
    if status != OK:
        raise GdnError(status, status_string(status))
    return out


def recurrent_update(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor, beta: torch.Tensor,
                     state_pool: torch.Tensor, state_indices: torch.Tensor, cu_seqlens: Optional[torch.Tensor],
                     out: torch.Tensor, scale: Optional[float] = None, flags: int = L2NORM_QK,
                     intermediate_states: Optional[torch.Tensor] = None,
                     device_status: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None,
                     tile_v: int = 0, schedule: int = SCHEDULE_AUTO, tile_rows: int = 0) -> torch.Tensor:
    """The recurrence of the unfused pair with precomputed gates
    (``gdn_recurrent_update``): decay = exp(g), beta given per (token, value
    head).  Arguments otherwise as ``decode_update``."""
    lib = load()
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[-1])
    if intermediate_states is not None:
        flags |= WRITE_INTERMEDIATE
    if stream is None:
        stream = torch.cuda.current_stream(q.device) if q.is_cuda else None
    descs = [describe(t) for t in (q, k, v, g, beta, state_pool, state_indices, cu_seqlens, out)]
    inter = describe(intermediate_states)
    extra = GdnExtra()
    extra.stream = stream.cuda_stream if stream is not None else None
    extra.intermediate_states = ctypes.pointer(inter) if inter is not None else None
    extra.device_status = device_status.data_ptr() if device_status is not None else None
    extra.tile_v = int(tile_v)
    extra.tile_rows = int(tile_rows)
    extra.schedule = int(schedule)
    status = lib.gdn_recurrent_update(*[_ref(d) for d in descs], ctypes.c_float(scale), ctypes.c_uint32(flags),
                                      ctypes.byref(extra))
    if status != OK:
        raise GdnError(status, status_string(status))
    return out


def gating(A_log: torch.Tensor, a: torch.Tensor, dt_bias: torch.Tensor, b: torch.Tensor, g: torch.Tensor,
           beta: torch.Tensor, stream: Optional[torch.cuda.Stream] = None) -> tuple:
    """The gating step alone (``gdn_gating``): g = -exp(A_log) softplus(a +
    dt_bias) (fp32) and beta = sigmoid(b) into the given [T_tot, HV] tensors."""
    lib = load()
    if stream is None:
        stream = torch.cuda.current_stream(a.device) if a.is_cuda else None
    descs = [describe(t) for t in (A_log, a, dt_bias, b, g, beta)]
    extra = GdnExtra()
    extra.stream = stream.cuda_stream if stream is not None else None
    status = lib.gdn_gating(*[_ref(d) for d in descs], ctypes.byref(extra))
    if status != OK:
        raise GdnError(status, status_string(status))
    return g, beta


def decode_update_host(host: dict, device: dict, *, scale: Optional[float] = None, flags: int = L2NORM_QK,
                       stream: Optional[torch.cuda.Stream] = None, tile_v: int = 0,
                       schedule: int = SCHEDULE_AUTO, tile_rows: int = 0) -> None:
    """End-to-end call from pinned host buffers.

    ``host`` holds pinned CPU tensors q, k, v, a, b, state_indices,
    cu_seqlens (optional) and out; ``device`` holds device tensors of the
    same names plus A_log, dt_bias, state_pool (resident) and optionally
    intermediate_states.  The call copies the per-step inputs host -> device,
    runs the update and copies ``out`` device -> host, all on ``stream``
    (asynchronous; synchronise the stream before reading host ``out``).
    """
    if stream is None:
        stream = torch.cuda.current_stream(device["q"].device)
    with torch.cuda.stream(stream):
        for name in ("q", "k", "v", "a", "b", "state_indices", "cu_seqlens"):
            if host.get(name) is not None:
                device[name].copy_(host[name], non_blocking=True)
        decode_update(device["q"], device["k"], device["v"], device["a"], device["b"], device["A_log"],
                      device["dt_bias"], device["state_pool"], device["state_indices"], device.get("cu_seqlens"),
                      device["out"], scale=scale, flags=flags,
                      intermediate_states=device.get("intermediate_states"), stream=stream, tile_v=tile_v,
                      schedule=schedule, tile_rows=tile_rows)
        host["out"].copy_(device["out"], non_blocking=True)


class PreparedCall:
    """A decode update whose descriptors are built once.

    For a serving loop that calls the update on the same buffers every step
    (the state pool, index and activation buffers are reused), this removes
    the per-call descriptor marshalling; each ``__call__`` is one C-ABI call
    that enqueues one kernel on ``stream``.  The tensors must stay alive and
    keep their storage while the object is used.
    """

    def __init__(self, q, k, v, a, b, A_log, dt_bias, state_pool, state_indices, cu_seqlens, out,
                 scale: Optional[float] = None, flags: int = L2NORM_QK, intermediate_states=None,
                 device_status=None, stream: Optional[torch.cuda.Stream] = None, tile_v: int = 0,
                 schedule: int = SCHEDULE_AUTO, tile_rows: int = 0, workspace="auto"):
        self._lib = load()
        self._keep = (q, k, v, a, b, A_log, dt_bias, state_pool, state_indices, cu_seqlens, out,
                      intermediate_states, device_status)
        if scale is None:
            scale = 1.0 / math.sqrt(q.shape[-1])
        if intermediate_states is not None:
            flags |= WRITE_INTERMEDIATE
        self._descs = [describe(t) for t in self._keep[:11]]
        self._inter = describe(intermediate_states)
        self._extra = GdnExtra()
        self.stream = stream if stream is not None else torch.cuda.current_stream(q.device)
        self._extra.stream = self.stream.cuda_stream
        self._extra.intermediate_states = ctypes.pointer(self._inter) if self._inter is not None else None
        self._extra.device_status = device_status.data_ptr() if device_status is not None else None
        self._extra.tile_v = int(tile_v)
        self._extra.tile_rows = int(tile_rows)
        self._extra.schedule = int(schedule)
        self.workspace = _workspace_for(workspace, schedule, q, v, state_indices.shape[0])
        _set_workspace(self._extra, self.workspace)
        self._args = [_ref(d) for d in self._descs] + [ctypes.c_float(scale), ctypes.c_uint32(flags),
                                                       ctypes.byref(self._extra)]
        self._scale, self._flags = float(scale), int(flags)
        self._fn = self._lib.gdn_decode_update

    def __call__(self) -> None:
        status = self._fn(*self._args)
        if status != OK:
            raise GdnError(status, status_string(status))

    def fill_host_step(self, st: "GdnHostStep") -> None:
        """Copy this call's arguments into a gdn_host_step (the transfer
        fields are the caller's)."""
        names = ("q", "k", "v", "a", "b", "A_log", "dt_bias", "state_pool", "state_indices", "cu_seqlens", "out")
        for name, d in zip(names, self._descs):
            setattr(st, name, ctypes.pointer(d) if d is not None else None)
        st.scale = self._scale
        st.flags = self._flags
        st.extra = ctypes.pointer(self._extra)


class HostStagedDecode:
    """A decode step fed from pinned host memory, with the fewest transfers.

    All per-step inputs (q, k, v, a, b, state_indices and cu_seqlens) live in
    ONE pinned host buffer, mirrored by one device buffer; each ``step()`` is
    one host-to-device copy of that buffer, one kernel launch and one
    device-to-host copy of ``out``, all on ``stream`` (asynchronous: sync the
    stream before reading ``out_host``).  Write a step's inputs into the host
    views (``q``, ``k``, ... attributes) before calling ``step()``.  The
    state pool, A_log and dt_bias stay resident on the device.

    Shapes follow ``decode_update``: q, k [T_tot, H, K]; v, out [T_tot, HV, V];
    a, b [T_tot, HV]; state_indices [N]; cu_seqlens [N+1] or None with
    fixed-length [N, T, ...] leading dims given by ``tokens_shape``.
    """

    _ALIGN = 256

    def __init__(self, tokens_shape, H, HV, K, V, N, A_log, dt_bias, state_pool, varlen=True,
                 scale: Optional[float] = None, flags: int = L2NORM_QK, intermediate_states=None,
                 stream: Optional[torch.cuda.Stream] = None, tile_v: int = 0, tile_rows: int = 0,
                 schedule: int = SCHEDULE_AUTO):
        dev = state_pool.device
        tokens_shape = tuple(tokens_shape)
        layout = [("q", tokens_shape + (H, K), torch.bfloat16), ("k", tokens_shape + (H, K), torch.bfloat16),
                  ("v", tokens_shape + (HV, V), torch.bfloat16), ("a", tokens_shape + (HV,), torch.bfloat16),
                  ("b", tokens_shape + (HV,), torch.bfloat16), ("state_indices", (N,), torch.int32)]
        if varlen:
            layout.append(("cu_seqlens", (N + 1,), torch.int32))
        offsets, off = {}, 0
        for name, shape, dt in layout:
            nbytes = math.prod(shape) * torch.tensor([], dtype=dt).element_size()
            offsets[name] = (off, nbytes, shape, dt)
            off += -(-nbytes // self._ALIGN) * self._ALIGN
        self.host_buffer = torch.empty(off, dtype=torch.uint8).pin_memory()
        self.device_buffer = torch.empty(off, dtype=torch.uint8, device=dev)
        views = {}
        for name, (o, n, shape, dt) in offsets.items():
            setattr(self, name, self.host_buffer[o:o + n].view(dt).view(shape))
            views[name] = self.device_buffer[o:o + n].view(dt).view(shape)
        if not varlen:
            self.cu_seqlens = None
        self.out_device = torch.empty(tokens_shape + (HV, V), dtype=torch.bfloat16, device=dev)
        self.out_host = torch.empty(self.out_device.shape, dtype=torch.bfloat16).pin_memory()
        self.stream = stream if stream is not None else torch.cuda.current_stream(dev)
        self._call = PreparedCall(views["q"], views["k"], views["v"], views["a"], views["b"], A_log, dt_bias,
                                  state_pool, views["state_indices"], views.get("cu_seqlens"), self.out_device,
                                  scale=scale, flags=flags, intermediate_states=intermediate_states,
                                  stream=self.stream, tile_v=tile_v, tile_rows=tile_rows, schedule=schedule)
        self.h2d_bytes = off
        self.d2h_bytes = self.out_host.numel() * self.out_host.element_size()

    def step(self) -> torch.Tensor:
        with torch.cuda.stream(self.stream):
            self.device_buffer.copy_(self.host_buffer, non_blocking=True)
            self._call()
            self.out_host.copy_(self.out_device, non_blocking=True)
        return self.out_host


class PipelinedHostDecode:
    """Host-fed decode steps with the transfers overlapped across steps.

    ``depth`` ``HostStagedDecode`` slots are used in turn.  Step k copies its
    inputs in on a copy stream, runs the update on the compute stream (steps
    stay in order there, so each step sees the previous step's state) and
    copies its output back on a third stream; meanwhile later steps' input
    copies and earlier steps' output copies run beside step k's kernel.
    ``inputs()`` returns the host views to fill for the next step (waiting, if
    needed, until that slot's previous input copy has read them); ``step()``
    issues the step and returns the host output of the step issued
    ``depth - 1`` calls before it (waiting for it), or None while the pipeline
    fills; ``finish()`` returns the host outputs of the steps still pending,
    in order.  A returned output stays valid until the next ``step()`` call.
    With depth 3 the host waits for an output one step after its kernel has
    ended, so it keeps issuing ahead of the GPU.  Other arguments are those of
    ``HostStagedDecode``.
    """

    def __init__(self, *args, stream: Optional[torch.cuda.Stream] = None, depth: int = 3, **kw):
        if depth < 2:
            raise ValueError("depth must be at least 2")
        dev = args[8].device if len(args) > 8 else kw["state_pool"].device
        self.depth = int(depth)
        self.compute = stream if stream is not None else torch.cuda.Stream(dev)
        self.copy_in = torch.cuda.Stream(dev)
        self.copy_out = torch.cuda.Stream(dev)
        self.slots = [HostStagedDecode(*args, stream=self.compute, **kw) for _ in range(self.depth)]
        self._h2d = [torch.cuda.Event() for _ in range(self.depth)]
        self._ran = [torch.cuda.Event() for _ in range(self.depth)]
        self._d2h = [torch.cuda.Event() for _ in range(self.depth)]
        self.h2d_bytes = self.slots[0].h2d_bytes
        self.d2h_bytes = self.slots[0].d2h_bytes
        self.k = 0          # steps issued
        self.done = 0       # steps whose output has been returned
        # one gdn_host_step per slot: the whole step is one C call.  torch
        # creates an event's CUDA handle at its first record; record each once.
        for e in self._h2d + self._ran + self._d2h:
            e.record(self.compute)
        self._issue = load().gdn_host_step_issue
        self._steps = []
        for b, sl in enumerate(self.slots):
            st = GdnHostStep()
            sl._call.fill_host_step(st)
            st.host_in, st.dev_in, st.in_bytes = sl.host_buffer.data_ptr(), sl.device_buffer.data_ptr(), sl.h2d_bytes
            st.dev_out, st.host_out, st.out_bytes = sl.out_device.data_ptr(), sl.out_host.data_ptr(), sl.d2h_bytes
            st.copy_in_stream, st.copy_out_stream = self.copy_in.cuda_stream, self.copy_out.cuda_stream
            st.ev_h2d, st.ev_ran, st.ev_d2h = (self._h2d[b].cuda_event, self._ran[b].cuda_event,
                                                self._d2h[b].cuda_event)
            self._steps.append((st, ctypes.byref(st)))

    def inputs(self) -> "HostStagedDecode":
        """The slot whose host views (``q``, ``k``, ...) the next step reads."""
        b = self.k % self.depth
        if self.k >= self.depth:
            self._h2d[b].synchronize()
        return self.slots[b]

    def _output(self) -> torch.Tensor:
        b = self.done % self.depth
        self._d2h[b].synchronize()
        self.done += 1
        return self.slots[b].out_host

    def step(self) -> Optional[torch.Tensor]:
        # gdn_host_step_issue: copy in (after step k - depth's update has read
        # slot b), update (after step k - depth's output has left slot b),
        # copy out, each ordered by the slot's events
        st, ref = self._steps[self.k % self.depth]
        st.reused = 1 if self.k >= self.depth else 0
        status = self._issue(ref)
        if status != OK:
            raise GdnError(status, status_string(status))
        self.k += 1
        return self._output() if self.k - self.done >= self.depth else None

    def finish(self) -> List[torch.Tensor]:
        return [self._output() for _ in range(self.k - self.done)]


class PreparedUnfusedCall:
    """The unfused pair as one prepared step: the gating kernel writes g and
    beta (fp32, [T_tot, HV], owned here) and the recurrence reads them --
    two launches and one round trip of the gates through HBM, which is what
    the fused update saves.  Arguments as ``PreparedCall``."""

    def __init__(self, q, k, v, a, b, A_log, dt_bias, state_pool, state_indices, cu_seqlens, out,
                 scale: Optional[float] = None, flags: int = L2NORM_QK, intermediate_states=None,
                 device_status=None, stream: Optional[torch.cuda.Stream] = None, tile_v: int = 0,
                 tile_rows: int = 0):
        lib = load()
        lead = q.shape[:-2]
        HV = v.shape[-2]
        self.g = torch.empty(math.prod(lead), HV, dtype=torch.float32, device=q.device)
        self.beta = torch.empty_like(self.g)
        a2, b2 = a.reshape(-1, HV), b.reshape(-1, HV)
        self.stream = stream if stream is not None else torch.cuda.current_stream(q.device)
        if scale is None:
            scale = 1.0 / math.sqrt(q.shape[-1])
        if intermediate_states is not None:
            flags |= WRITE_INTERMEDIATE
        self._keep = (q, k, v, a2, b2, A_log, dt_bias, state_pool, state_indices, cu_seqlens, out,
                      intermediate_states, device_status)
        self._gd = [describe(t) for t in (A_log, a2, dt_bias, b2, self.g, self.beta)]
        g_view, beta_view = self.g.view(*lead, HV), self.beta.view(*lead, HV)
        self._keep2 = (g_view, beta_view)
        self._rd = [describe(t) for t in (q, k, v, g_view, beta_view, state_pool, state_indices, cu_seqlens, out)]
        self._inter = describe(intermediate_states)
        self._gx = GdnExtra()
        self._gx.stream = self.stream.cuda_stream
        self._rx = GdnExtra()
        self._rx.stream = self.stream.cuda_stream
        self._rx.intermediate_states = ctypes.pointer(self._inter) if self._inter is not None else None
        self._rx.device_status = device_status.data_ptr() if device_status is not None else None
        self._rx.tile_v = int(tile_v)
        self._rx.tile_rows = int(tile_rows)
        self._gargs = [_ref(d) for d in self._gd] + [ctypes.byref(self._gx)]
        self._rargs = [_ref(d) for d in self._rd] + [ctypes.c_float(scale), ctypes.c_uint32(flags),
                                                     ctypes.byref(self._rx)]
        self._gating = lib.gdn_gating
        self._recurrent = lib.gdn_recurrent_update

    def __call__(self) -> None:
        status = self._gating(*self._gargs)
        if status == OK:
            status = self._recurrent(*self._rargs)
        if status != OK:
            raise GdnError(status, status_string(status))
