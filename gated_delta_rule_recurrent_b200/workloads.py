"""Seeded synthetic inputs for the recurrent gated-delta-rule decode step.

This module is the one piece shared by the CUDA path's tests and benchmark and
by the CPU oracle's tests: it draws inputs and holds none of the method's
arithmetic. Every tensor is drawn on the CPU with a seeded
``torch.Generator`` in float32 and then narrowed to the dtype the op takes
(bfloat16 for query/key/value/beta/state/a/b, float32 for g/gk/dt_bias/
decay_scale, int32 for lengths and indices), following the argument table of
"lite_boost.ops.recurrent_gated_delta_rule" (section "参数") and the input
table of "com.microsoft.LinearAttentionGate" (section "Inputs").

Distributions (identical for every workload unless its entry says otherwise):

* query, key: N(0, 1), then L2-normalised over D_k in float32 (the op expects
  unit-norm heads and does not normalise them itself), then bfloat16.
* value: N(0, 1), bfloat16.
* beta: the logistic function of N(0, 1) draws, bfloat16 (values in (0, 1)).
* g: minus the softplus of N(0, 1) draws, float32 [B, H_v, T] (negative).
* gk: minus 0.1 times the softplus of N(0, 1) draws, float32 [B, H_v, T, D_k].
* state pool: 0.1 * N(0, 1), bfloat16 [pool, H_v, D_k, D_v], drawn slot by slot.
* gate inputs: a, b ~ N(0, 1) bfloat16 [B, T, H_v]; dt_bias ~ U(0, 1) float32
  [H_v]; decay_scale = -exp(U(-1, 1)) float32 [H_v] (the gated-DeltaNet form
  -exp(A_log) with A_log ~ U(-1, 1)).

Padded token positions (t >= actual_seq_lengths[b]) can be filled with NaN in
every per-token input (``poison_padding=True``) to show that they are not read.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional, Sequence

import torch

__all__ = ["Workload", "WORKLOADS", "PREFILL_WORKLOADS", "make_inputs", "workload"]


@dataclasses.dataclass(frozen=True)
class Workload:
    """Sizes and structure of one synthetic decode workload."""

    name: str
    B: int
    H_qk: int
    H_v: int
    T: int
    D_k: int
    D_v: int
    pool: int
    scale_value: float
    gated: bool
    lengths: str  # "full", "fixed" (see fixed_lengths), "uniform" (U{1..T}) or "upper" (U{T/2..T})
    indices: str  # "fixed" (see fixed_indices), "subset" (random B of pool) or "perm"
    fixed_lengths: Optional[Sequence[int]] = None
    fixed_indices: Optional[Sequence[int]] = None
    seed: int = 1000

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS: Dict[int, Workload] = {
    # Tiny case the oracle checks in milliseconds.
    0: Workload("tiny_B2_H4_T2_64x64", B=2, H_qk=4, H_v=4, T=2, D_k=64, D_v=64, pool=2,
                scale_value=1.0 / 8.0, gated=False, lengths="fixed", indices="fixed",
                fixed_lengths=(2, 1), fixed_indices=(1, 0), seed=1000),
    # Single sequence at the API page's example shape (section "样例").
    1: Workload("single_seq_B1_H64_T1_64x512", B=1, H_qk=64, H_v=64, T=1, D_k=64, D_v=512,
                pool=1, scale_value=1.0 / math.sqrt(64), gated=False, lengths="full",
                indices="fixed", fixed_indices=(0,), seed=1001),
    # Batched decode with grouped heads: value head h reads q/k head h // 2.
    2: Workload("gqa_B64_Hqk16_Hv32_T1_128x128", B=64, H_qk=16, H_v=32, T=1, D_k=128,
                D_v=128, pool=256, scale_value=1.0 / math.sqrt(128), gated=False,
                lengths="full", indices="subset", seed=1002),
    # Speculative multi-token decode, T = 8 padded, lengths U{1..8}.
    3: Workload("spec_B128_H32_T8_128x128", B=128, H_qk=32, H_v=32, T=8, D_k=128, D_v=128,
                pool=128, scale_value=1.0 / math.sqrt(128), gated=False, lengths="uniform",
                indices="perm", seed=1003),
    # Large-batch decode with the fused gate prologue (2 GiB bfloat16 pool).
    4: Workload("gated_B512_H64_T1_64x512", B=512, H_qk=64, H_v=64, T=1, D_k=64, D_v=512,
                pool=512, scale_value=1.0 / math.sqrt(64), gated=True, lengths="full",
                indices="perm", seed=1004),
}


# Long-prompt (prefill) workloads: the grouped-head, 128 x 128 shape of the
# decode workloads over a prompt of up to T tokens, lengths U{T/2..T}, with
# the fused gate.
PREFILL_WORKLOADS: Dict[str, Workload] = {
    "prefill": Workload("prefill_B8_Hqk16_Hv32_T2048_128x128", B=8, H_qk=16, H_v=32, T=2048,
                        D_k=128, D_v=128, pool=16, scale_value=1.0 / math.sqrt(128),
                        gated=True, lengths="upper", indices="subset", seed=1005),
}


def workload(key) -> Workload:
    """Look a workload up by number or by name."""
    if isinstance(key, Workload):
        return key
    if isinstance(key, int):
        return WORKLOADS[key]
    if key in PREFILL_WORKLOADS:
        return PREFILL_WORKLOADS[key]
    for w in list(WORKLOADS.values()) + list(PREFILL_WORKLOADS.values()):
        if w.name == key:
            return w
    raise KeyError(f"unknown workload {key!r}")


def _unit_rows(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-30)


def make_inputs(w, *, seed: Optional[int] = None, poison_padding: bool = False,
                with_state: bool = True) -> Dict[str, object]:
    """Draw every input of one call of workload ``w`` on the CPU.

    Returns a dict with the op's argument names: query, key, value, beta,
    state_pool, actual_seq_lengths, ssm_state_indices, g, gk,
    num_accepted_tokens, scale_value, and the gate inputs a, b, dt_bias,
    decay_scale (both the plain and the gated argument sets are drawn, in a
    fixed order, so either entry point can be fed from one draw).
    """
    w = workload(w)
    gen = torch.Generator(device="cpu")
    gen.manual_seed(w.seed if seed is None else seed)
    B, Hq, Hv, T, Dk, Dv, P = w.B, w.H_qk, w.H_v, w.T, w.D_k, w.D_v, w.pool

    def randn(*shape):
        return torch.randn(*shape, generator=gen, dtype=torch.float32)

    def rand(*shape):
        return torch.rand(*shape, generator=gen, dtype=torch.float32)

    # Lengths and slot indices.
    if w.lengths == "fixed":
        lengths = torch.tensor(list(w.fixed_lengths), dtype=torch.int32)
    elif w.lengths == "full":
        lengths = torch.full((B,), T, dtype=torch.int32)
    elif w.lengths == "uniform":
        lengths = torch.randint(1, T + 1, (B,), generator=gen, dtype=torch.int32)
    elif w.lengths == "upper":
        lengths = torch.randint((T + 1) // 2, T + 1, (B,), generator=gen, dtype=torch.int32)
    else:
        raise ValueError(w.lengths)
    if w.indices == "fixed":
        indices = torch.tensor(list(w.fixed_indices), dtype=torch.int32)
    elif w.indices in ("subset", "perm"):
        indices = torch.randperm(P, generator=gen)[:B].to(torch.int32)
    else:
        raise ValueError(w.indices)

    query = _unit_rows(randn(B, Hq, T, Dk)).to(torch.bfloat16)
    key = _unit_rows(randn(B, Hq, T, Dk)).to(torch.bfloat16)
    value = randn(B, Hv, T, Dv).to(torch.bfloat16)
    beta = torch.sigmoid(randn(B, Hv, T)).to(torch.bfloat16)
    g = -torch.nn.functional.softplus(randn(B, Hv, T))
    gk = -0.1 * torch.nn.functional.softplus(randn(B, Hv, T, Dk))
    a = randn(B, T, Hv).to(torch.bfloat16)
    b = randn(B, T, Hv).to(torch.bfloat16)
    dt_bias = rand(Hv)
    decay_scale = -torch.exp(rand(Hv) * 2.0 - 1.0)

    state_pool = None
    if with_state:
        state_pool = torch.empty(P, Hv, Dk, Dv, dtype=torch.bfloat16)
        for s in range(P):
            state_pool[s] = (0.1 * randn(Hv, Dk, Dv)).to(torch.bfloat16)

    if poison_padding:
        nan = float("nan")
        for bi in range(B):
            L = int(lengths[bi])
            if L < T:
                for t_ in (query, key):
                    t_[bi, :, L:, :] = nan
                value[bi, :, L:, :] = nan
                beta[bi, :, L:] = nan
                g[bi, :, L:] = nan
                gk[bi, :, L:, :] = nan
                a[bi, L:, :] = nan
                b[bi, L:, :] = nan

    return {
        "query": query.contiguous(),
        "key": key.contiguous(),
        "value": value.contiguous(),
        "beta": beta.contiguous(),
        "state_pool": state_pool,
        "actual_seq_lengths": lengths.contiguous(),
        "ssm_state_indices": indices.contiguous(),
        "g": g.contiguous(),
        "gk": gk.contiguous(),
        "num_accepted_tokens": lengths.clone(),
        "scale_value": float(w.scale_value),
        "a": a.contiguous(),
        "b": b.contiguous(),
        "dt_bias": dt_bias.contiguous(),
        "decay_scale": decay_scale.contiguous(),
    }


def make_gate_inputs(shape, dtype=torch.bfloat16, *, seed: int = 2024):
    """Inputs of the standalone gate op with the gate workload's distributions:
    a, b ~ N(0, 1) of ``shape`` (heads on the last axis) narrowed to ``dtype``;
    dt_bias ~ U(0, 1) and decay_scale = -exp(U(-1, 1)), float32 [H]."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    H = shape[-1]
    a = torch.randn(*shape, generator=gen, dtype=torch.float32).to(dtype)
    b = torch.randn(*shape, generator=gen, dtype=torch.float32).to(dtype)
    dt_bias = torch.rand(H, generator=gen, dtype=torch.float32)
    decay_scale = -torch.exp(torch.rand(H, generator=gen, dtype=torch.float32) * 2.0 - 1.0)
    return {"a": a, "b": b, "dt_bias": dt_bias, "decay_scale": decay_scale}
