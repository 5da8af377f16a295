"""Algorithmic traffic and work of one decode call, for roofline reporting.

Algorithmic bytes count what the method must move between HBM and the SMs,
each tensor element once:

* state: read and written once per touched (item, value head): 2 * 2 * D_k * D_v
  bytes (bfloat16), for items with length > 0 and a slot inside the pool;
* per valid token of an item: query and key, 2 bytes per element, once per
  query/key head (2 * H_qk * D_k * 2); per value head, value (2 * D_v),
  gk (4 * D_k) and either g and beta (4 + 2) or the gate inputs a and b (2 + 2);
* out: written for every (item, value head, token), padding included
  (2 * B * H_v * T * D_v);
* per item, the int32 length, slot index and accepted-token count (12 bytes);
  with the fused gate, the two float32 [H_v] vectors once (8 * H_v).

Padded tokens' inputs are not counted: the kernel does not read them.
"""
from __future__ import annotations

from typing import Iterable, Optional


def algorithmic_bytes(B: int, H_qk: int, H_v: int, T: int, D_k: int, D_v: int,
                      lengths: Iterable[int], gated: bool,
                      touched_items: Optional[int] = None) -> int:
    lengths = [min(max(int(x), 0), T) for x in lengths]
    if touched_items is None:
        touched_items = sum(1 for x in lengths if x > 0)
    state = 2 * 2 * D_k * D_v * H_v * touched_items
    per_token = 2 * H_qk * D_k * 2 + H_v * (2 * D_v + 4 * D_k + (2 + 2 if gated else 4 + 2))
    tokens = sum(lengths) * per_token
    out = 2 * B * H_v * T * D_v
    scalars = 12 * B + (8 * H_v if gated else 0)
    return state + tokens + out + scalars


def flops(H_v: int, D_k: int, D_v: int, lengths: Iterable[int], T: int) -> int:
    """Floating-point operations of the four steps as written: per (item, value head,
    valid token) and state element, decay 1 + memory read 2 + update 2 + output 2."""
    n_tok = sum(min(max(int(x), 0), T) for x in lengths)
    return 7 * D_k * D_v * H_v * n_tok
