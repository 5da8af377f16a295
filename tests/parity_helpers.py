"""Shared helpers of the GPU parity tests: run the CUDA path and the oracle on the
same seeded inputs and compare element by element.

Tolerance for floating-point results (out, touched state slots):
    |gpu - oracle| <= 2**-7 * |oracle| + 1e-3
i.e. about two bfloat16 ulps: both sides round to bfloat16 once from a wider
type (fp32 on the GPU, fp64 in the oracle), so they differ by at most one ulp
of the final rounding plus the fp32 accumulation error, which is orders of
magnitude below the absolute floor here. Results that involve no arithmetic
must match bit for bit: padded output positions are +0.0 and pool slots no
item touches keep their bits.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle.gdr_oracle import recurrent_gated_delta_rule, recurrent_gated_delta_rule_gated

RTOL = 2.0**-7
ATOL = 1e-3

PER_TOKEN = ("query", "key", "value", "beta", "g", "gk", "a", "b")


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").to(torch.float64).numpy()


def run_oracle(x: dict, gated: bool, items=None):
    """Oracle on the whole call, or on the batch items ``items`` with a compacted pool.

    Returns (out [B', H_v, T, D_v], pool-like array, slots) where ``slots`` maps
    row r of the returned pool to the slot of the full pool it stands for.
    """
    idx = x["ssm_state_indices"].to(torch.int64).numpy()
    asl = x["actual_seq_lengths"].to(torch.int64).numpy()
    pool = x["state_pool"]
    if items is None:
        items = np.arange(idx.shape[0])
        slots = np.arange(pool.shape[0])
        pool_np = f64(pool)
        idx_sub = idx
    else:
        items = np.asarray(items)
        sel = idx[items]
        valid = (sel >= 0) & (sel < pool.shape[0])
        slots = np.unique(sel[valid])
        pool_np = f64(pool[torch.from_numpy(slots)]) if slots.size else \
            np.zeros((1,) + tuple(pool.shape[1:]))
        remap = {int(s): i for i, s in enumerate(slots)}
        idx_sub = np.array([remap.get(int(s), -1) for s in sel])
    sub = {k: (f64(x[k][torch.from_numpy(items)]) if k in PER_TOKEN else None)
           for k in PER_TOKEN}
    nat_all = x.get("num_accepted_tokens")
    nat = None if nat_all is None else nat_all.to(torch.int64).numpy()[items]
    if gated:
        out, st = recurrent_gated_delta_rule_gated(
            sub["query"], sub["key"], sub["value"], sub["a"], sub["b"], f64(x["dt_bias"]),
            f64(x["decay_scale"]), pool_np, asl[items], idx_sub, sub["gk"], nat,
            x["scale_value"])
    else:
        out, st = recurrent_gated_delta_rule(
            sub["query"], sub["key"], sub["value"], sub["beta"], pool_np, asl[items], idx_sub,
            sub["g"], sub["gk"], nat, x["scale_value"])
    return out, st, slots


def to_device(x: dict, device="cuda") -> dict:
    return {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}


def run_gpu(xd: dict, gated: bool, out=None, state_layout="kv"):
    """One call of the CUDA path on device tensors (the pool is updated in place).
    With state_layout "vk" the pool in ``xd`` is [pool, H_v, D_v, D_k]."""
    from gated_delta_rule_recurrent_b200 import decode, decode_gated

    if gated:
        return decode_gated(xd["query"], xd["key"], xd["value"], xd["a"], xd["b"], xd["dt_bias"],
                            xd["decay_scale"], xd["state_pool"], xd["actual_seq_lengths"],
                            xd["ssm_state_indices"], xd["gk"], xd["num_accepted_tokens"],
                            xd["scale_value"], out=out, state_layout=state_layout)
    return decode(xd["query"], xd["key"], xd["value"], xd["beta"], xd["state_pool"],
                  xd["actual_seq_lengths"], xd["ssm_state_indices"], xd["g"], xd["gk"],
                  xd["num_accepted_tokens"], xd["scale_value"], out=out,
                  state_layout=state_layout)


def to_vk(pool: torch.Tensor) -> torch.Tensor:
    """A [pool, H_v, D_k, D_v] state pool as [pool, H_v, D_v, D_k] (and back)."""
    return pool.transpose(2, 3).contiguous()


def assert_close(got: np.ndarray, ref: np.ndarray, what: str) -> None:
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    err = np.abs(got - ref)
    bound = RTOL * np.abs(ref) + ATOL
    bad = ~(err <= bound)  # NaN counts as bad
    if bad.any():
        i = tuple(np.argwhere(bad)[0])
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {bad.size} elements out of tolerance; first at {i}: "
            f"gpu={got[i]!r} oracle={ref[i]!r} (max err {np.nanmax(err):.3g})")


def bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy()


def check_call(x: dict, out_gpu: torch.Tensor, pool_before: torch.Tensor,
               pool_after: torch.Tensor, gated: bool, items=None) -> None:
    """Compare one GPU call with the oracle on all items (or on ``items``)."""
    out_ref, st_ref, slots = run_oracle(x, gated, items)
    asl = x["actual_seq_lengths"].to(torch.int64).numpy()
    idx = x["ssm_state_indices"].to(torch.int64).numpy()
    B, T = x["query"].shape[0], x["query"].shape[2]
    P = pool_before.shape[0]
    sel = np.arange(B) if items is None else np.asarray(items)
    out_sel = out_gpu.detach().cpu()[torch.from_numpy(sel)]
    assert_close(f64(out_sel), out_ref, "out")
    # padded positions and skipped items: exactly +0.0
    ob = bits(out_sel)
    for r, bi in enumerate(sel):
        L = int(min(max(asl[bi], 0), T))
        if not 0 <= idx[bi] < P:
            L = 0
        assert np.all(ob[r, :, L:, :] == 0), f"item {bi}: padded out not +0.0"
    # touched slots: tolerance; every other slot: identical bits
    touched = {int(idx[bi]) for bi in range(B)
               if 0 <= idx[bi] < P and min(max(asl[bi], 0), T) > 0}
    for r, s in enumerate(slots):
        if int(s) in touched:
            assert_close(f64(pool_after[int(s)]), st_ref[r], f"state slot {int(s)}")
    untouched = sorted(set(range(P)) - touched)
    if untouched:
        ut = torch.tensor(untouched)
        assert np.array_equal(bits(pool_after[ut]), bits(pool_before[ut])), \
            "an untouched pool slot changed"
