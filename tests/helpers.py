"""Shared test helpers: input marshalling only (no step of the update)."""
from __future__ import annotations

import json
import os

import numpy as np

from gated_deltanet_recurrent_sigmoid_b200.workloads import (
    bf16_bits_to_f32, f32_to_bf16_bits)

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")

BF16_POS_INF = np.uint16(0x7F80)
BF16_NEG_INF = np.uint16(0xFF80)


def bf16(x) -> np.ndarray:
    """bf16 patterns of values that must be exact in bf16 (asserted)."""
    x = np.asarray(x, dtype=np.float32)
    bits = f32_to_bf16_bits(x)
    back = bf16_bits_to_f32(bits)
    assert np.array_equal(back, x, equal_nan=True), "value not exact in bf16"
    return bits


def load_golden(name: str) -> dict:
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _f32_scalar(x) -> np.float32:
    if x == "ln2_f32":
        return np.float32(np.log(2.0))
    if x == "-inf":
        return np.float32(-np.inf)
    return np.float32(x)


def golden_arrays(case: dict) -> dict:
    """One sequence of len(tokens) tokens, fixed-length layout [N=1, T, ...]."""
    K, V, H, HV = case["K"], case["V"], case["H"], case["HV"]
    toks = case["tokens"]
    T = len(toks)
    q = bf16([[t["q"]] for t in toks]).reshape(1, T, H, K)
    k = bf16([[t["k"]] for t in toks]).reshape(1, T, H, K)
    v = bf16([[t["v"]] for t in toks]).reshape(1, T, HV, V)
    a = bf16([[t["a"]] for t in toks]).reshape(1, T, HV)
    b = bf16([[t["b"]] for t in toks]).reshape(1, T, HV)
    A_log = np.array([_f32_scalar(x) for x in case["A_log"]], dtype=np.float32)
    dt_bias = np.array(case["dt_bias"], dtype=np.float32)
    state = np.array(case["state_in"], dtype=np.float32).reshape(1, HV, K, V)
    return dict(q=q, k=k, v=v, a=a, b=b, A_log=A_log, dt_bias=dt_bias,
                state_pool=state, state_indices=np.array([0], dtype=np.int32),
                cu_seqlens=None)


def random_problem(rng, N=3, T=None, lens=None, H=2, HV=4, K=8, V=8, num_slots=None,
                   pad=(), state_scale=0.1):
    """Small random problem in the varlen layout (cu_seqlens given)."""
    if lens is None:
        lens = np.full(N, T if T is not None else 1)
    lens = np.asarray(lens, dtype=np.int32)
    N = len(lens)
    T_tot = int(lens.sum())
    num_slots = num_slots or 2 * N
    q = f32_to_bf16_bits(rng.standard_normal((T_tot, H, K), dtype=np.float32))
    k = f32_to_bf16_bits(rng.standard_normal((T_tot, H, K), dtype=np.float32))
    v = f32_to_bf16_bits(rng.standard_normal((T_tot, HV, V), dtype=np.float32))
    a = f32_to_bf16_bits(rng.standard_normal((T_tot, HV), dtype=np.float32))
    b = f32_to_bf16_bits(rng.standard_normal((T_tot, HV), dtype=np.float32))
    A_log = np.log(rng.uniform(1, 16, HV)).astype(np.float32)
    dt_bias = rng.uniform(-1, 1, HV).astype(np.float32)
    state = (rng.standard_normal((num_slots, HV, K, V), dtype=np.float32) * np.float32(state_scale))
    idx = rng.permutation(num_slots)[:N].astype(np.int32)
    for p in pad:
        idx[p] = -1
    cu = np.zeros(N + 1, dtype=np.int32)
    cu[1:] = np.cumsum(lens)
    return dict(q=q, k=k, v=v, a=a, b=b, A_log=A_log, dt_bias=dt_bias,
                state_pool=state, state_indices=idx, cu_seqlens=cu)
