"""Seeded synthetic inputs shaped like Qwen3-Next decode workloads.

This module draws random inputs and nothing else: it holds no step of the
decode update's arithmetic, so that the CUDA path and the CPU oracle can both
be fed from it without sharing any of the method.  The workloads follow the
pages' serving setup ("[Qwen3Next] Optimize
fused_sigmoid_gating_delta_rule_update_kernel", Benchmarking and Profiling:
TP4, batch 512 on B200, i.e. 8 value heads per rank with K = V = 128).

Recipe, per workload (all draws from one numpy ``PCG64`` stream per seed, in
this order): sequence lengths (varlen only), q, k, v, a, b ~ N(0, 1) rounded
to bf16 with round-to-nearest-even; A_log = ln U(1, 16) (fp32);
dt_bias ~ U(-1, 1) (fp32); the whole state pool ~ N(0, 0.1^2) (fp32); slot
indices = the first N entries of a random permutation of the pool; then
floor(pad_frac * N) positions, chosen by a second permutation, set to -1.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

HEAD_DIM = 128


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (nearest, ties to even); returns uint16 patterns."""
    x = np.asarray(x, dtype=np.float32)
    u = np.ascontiguousarray(x).view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16).reshape(x.shape)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 patterns to the fp32 values they encode (exact)."""
    bits = np.asarray(bits, dtype=np.uint16)
    wide = np.ascontiguousarray(bits).astype(np.uint32) << 16
    return wide.view(np.float32).reshape(bits.shape)


@dataclasses.dataclass(frozen=True)
class WorkloadSpec:
    """Sizes and distribution knobs of one synthetic decode workload."""
    name: str
    N: int                      # sequences in the batch
    H: int                      # key heads
    HV: int                     # value heads (GQA: HV % H == 0)
    num_slots: int              # state-pool slots
    seed: int
    T: Optional[int] = 1        # fixed tokens per sequence, or None for varlen
    max_len: int = 64           # varlen: lengths drawn U{min_len..max_len}
    min_len: int = 1
    pad_frac: float = 0.0       # fraction of state_indices set to -1
    varlen: bool = False        # pass cu_seqlens (also used for uniform T)
    intermediate: bool = False  # write per-token states
    K: int = HEAD_DIM
    V: int = HEAD_DIM


@dataclasses.dataclass
class Workload:
    """Host arrays of one workload (bf16 tensors as uint16 patterns)."""
    spec: WorkloadSpec
    q: np.ndarray               # [T_tot, H, K] uint16 (or [N, T, H, K] when not varlen)
    k: np.ndarray
    v: np.ndarray               # [T_tot, HV, V] uint16
    a: np.ndarray               # [T_tot, HV] uint16
    b: np.ndarray
    A_log: np.ndarray           # [HV] float32
    dt_bias: np.ndarray         # [HV] float32
    state_pool: np.ndarray      # [num_slots, HV, K, V] float32
    state_indices: np.ndarray   # [N] int32
    cu_seqlens: Optional[np.ndarray]  # [N+1] int32 or None

    @property
    def T_tot(self) -> int:
        return int(np.prod(self.q.shape[:-2]))

    @property
    def seq_lens(self) -> np.ndarray:
        if self.cu_seqlens is not None:
            return np.diff(self.cu_seqlens).astype(np.int64)
        return np.full(self.spec.N, self.q.shape[1], dtype=np.int64)


def _bf16_normal(rng: np.random.Generator, shape) -> np.ndarray:
    return f32_to_bf16_bits(rng.standard_normal(shape, dtype=np.float32))


def generate(spec: WorkloadSpec) -> Workload:
    """Draw the arrays of ``spec`` from its seed (bit-identical on every host)."""
    rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([spec.seed, spec.N])))
    N, H, HV, K, V = spec.N, spec.H, spec.HV, spec.K, spec.V
    if spec.T is None:
        lens = rng.integers(spec.min_len, spec.max_len + 1, size=N).astype(np.int32)
    else:
        lens = np.full(N, spec.T, dtype=np.int32)
    T_tot = int(lens.sum())
    varlen = spec.varlen or spec.T is None
    lead = (T_tot,) if varlen else (N, int(spec.T))

    q = _bf16_normal(rng, lead + (H, K))
    k = _bf16_normal(rng, lead + (H, K))
    v = _bf16_normal(rng, lead + (HV, V))
    a = _bf16_normal(rng, lead + (HV,))
    b = _bf16_normal(rng, lead + (HV,))
    A_log = np.log(rng.uniform(1.0, 16.0, size=HV)).astype(np.float32)
    dt_bias = rng.uniform(-1.0, 1.0, size=HV).astype(np.float32)
    state = rng.standard_normal((spec.num_slots, HV, K, V), dtype=np.float32)
    state *= np.float32(0.1)
    if N > spec.num_slots:
        raise ValueError("pool smaller than the batch")
    indices = rng.permutation(spec.num_slots)[:N].astype(np.int32)
    n_pad = int(np.floor(spec.pad_frac * N))
    if n_pad:
        indices[rng.permutation(N)[:n_pad]] = -1
    cu = None
    if varlen:
        cu = np.zeros(N + 1, dtype=np.int32)
        np.cumsum(lens, out=cu[1:])
    return Workload(spec, q, k, v, a, b, A_log, dt_bias, state, indices, cu)


# The five workload families (seed = family index; sweep seeds mix in N).
TINY = WorkloadSpec("tiny_b4", N=4, H=2, HV=4, num_slots=8, seed=0)
DECODE_B512 = WorkloadSpec("decode_b512_hv8", N=512, H=4, HV=8, num_slots=1024,
                           seed=1, pad_frac=0.05)
FULLHEAD_B256 = WorkloadSpec("fullhead_b256_hv32", N=256, H=16, HV=32, num_slots=512, seed=2)
SPEC_B128_T4 = WorkloadSpec("spec_b128_t4", N=128, H=4, HV=8, num_slots=256, seed=3,
                            T=4, varlen=True, intermediate=True)
SWEEP_NS = (1, 8, 64, 256, 1024)


def sweep_spec(N: int) -> WorkloadSpec:
    return WorkloadSpec(f"sweep_b{N}", N=N, H=4, HV=8, num_slots=2 * N, seed=4,
                        T=None, max_len=64, pad_frac=0.10)


# Prefill-style: few sequences, long and ragged (the chunked schedule's workload).
PREFILL_B8 = WorkloadSpec("prefill_b8_t2k", N=8, H=4, HV=8, num_slots=16, seed=5, T=None, min_len=1024,
                          max_len=2048)
PREFILL_B64 = WorkloadSpec("prefill_b64_t512", N=64, H=4, HV=8, num_slots=128, seed=6, T=None, min_len=256,
                           max_len=768)

ALL_SPECS = [TINY, DECODE_B512, FULLHEAD_B256, SPEC_B128_T4] + [sweep_spec(n) for n in SWEEP_NS] + [PREFILL_B8,
                                                                                                   PREFILL_B64]
BY_NAME = {s.name: s for s in ALL_SPECS}


def shrink(spec: WorkloadSpec, N: int, num_slots: Optional[int] = None, name: Optional[str] = None) -> WorkloadSpec:
    """The same family at a smaller batch (for checks the oracle runs in seconds)."""
    return dataclasses.replace(spec, name=name or f"{spec.name}_n{N}", N=N,
                               num_slots=num_slots or max(N, min(spec.num_slots, 2 * N)))


def algorithmic_bytes(w: Workload, write_intermediate: Optional[bool] = None,
                      final_writeback: bool = True) -> int:
    """HBM bytes one call must move: state read + write for every non-padded
    sequence, the optional per-token states, and the activations.

    state:  (1 + final_writeback) * P * HV * K * V * 4, P = non-padded sequences
    inter:  T_active * HV * K * V * 4
    acts:   active tokens * (2*H*K + HV*V + 2*HV) * 2  (q, k, v, a, b)
            + T_tot * HV * V * 2 (out) + 8 * HV (A_log, dt_bias)
            + 4 * N (state_indices) + 4 * (N + 1) (cu_seqlens, when given)
    """
    s = w.spec
    inter = s.intermediate if write_intermediate is None else write_intermediate
    active = w.state_indices >= 0
    lens = w.seq_lens
    P = int(active.sum())
    T_act = int(lens[active].sum())
    head = s.K * s.V * 4
    nbytes = (1 + int(final_writeback)) * P * s.HV * head
    if inter:
        nbytes += T_act * s.HV * head
    nbytes += T_act * (2 * s.H * s.K + s.HV * s.V + 2 * s.HV) * 2
    nbytes += w.T_tot * s.HV * s.V * 2
    nbytes += 8 * s.HV + 4 * s.N
    if w.cu_seqlens is not None:
        nbytes += 4 * (s.N + 1)
    return nbytes


def algorithmic_flops(w: Workload) -> int:
    """About 7 K V flops per active (token, value head): decay, two dot
    products over K, the rank-1 update and the output contraction."""
    s = w.spec
    active = w.state_indices >= 0
    T_act = int(w.seq_lens[active].sum())
    return 7 * s.K * s.V * T_act * s.HV
