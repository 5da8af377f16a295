"""A bounded wait that runs out, on the GPU, with nothing in flight (test build).

The kernels' failure protocol (gdr_ptx.cuh): a wait on another role's signal
gives up after a budget, flags the device error word, and tells the rest of
the CTA to give up too; whoever saw a wait fail stops signalling, so the
kernel ends, frees its tensor memory, and commits no state for a tile whose
inputs were not seen to land. Copies already started are drained first.

The shipped library's budget is about 2 s and no call ever reaches it. These
tests load the second build, ``libgdr_testhooks.so`` (compiled with
-DGDR_TEST_HOOKS; the shipped library has no hooks). There the budget is a
device variable and the producer can hold one tile back: it starts no copy
for it and never signals it ready, and stops issuing. So every copy that was
started lands, and only waits for signals that will never come run out.

For each kernel family, one call with a held-back tile must
* return promptly (a short budget, abandoned waits elsewhere in the CTA);
* flag a wait bit in the device error word, and never the drain bit;
* leave the held tile's state block bit-identical, and every other state
  element either bit-identical or equal to the oracle within the parity
  tolerance (no stale or partial data);
and a normal call right after, on the same device, must pass parity with a
clear error word (the CTA really ended and freed its resources).
"""
import ctypes
import time

import numpy as np
import pytest
import torch

from gated_delta_rule_recurrent_b200 import workloads
from parity_helpers import ATOL, RTOL, bits, check_call, f64, run_oracle

pytestmark = pytest.mark.gpu

ERR_CONSUMER, ERR_PRODUCER, ERR_DRAIN = 1, 2, 4
SHORT_BUDGET = 4_000_000  # cycles, about 2 ms


@pytest.fixture(scope="module")
def hooks():
    from gated_delta_rule_recurrent_b200 import binding, build

    path = build.ensure_built(test_hooks=True)
    L = ctypes.CDLL(path)
    L.gdr_decode.argtypes = binding._DECODE_ARGTYPES
    L.gdr_decode.restype = ctypes.c_int
    L.gdr_prefill.argtypes = binding._DECODE_ARGTYPES
    L.gdr_prefill.restype = ctypes.c_int
    L.gdr_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint32), ctypes.c_int]
    L.gdr_device_error.restype = ctypes.c_int
    L.gdr_last_launch.argtypes = [ctypes.POINTER(binding.LaunchInfo)]
    L.gdr_last_launch.restype = ctypes.c_int
    L.gdr_last_error.restype = ctypes.c_char_p
    L.gdrtest_set_hooks.argtypes = [ctypes.c_longlong, ctypes.c_int]
    L.gdrtest_set_hooks.restype = ctypes.c_int
    yield L
    assert L.gdrtest_set_hooks(0, -1) == 0


def _decode(L, xd, state_layout="kv", prefill=False):
    """gdr_decode (or gdr_prefill) of the test build, with the binding's
    argument checks."""
    from gated_delta_rule_recurrent_b200 import binding

    _, dims, out, stream = binding._common(
        xd["query"], xd["key"], xd["value"], xd["state_pool"], xd["actual_seq_lengths"],
        xd["ssm_state_indices"], xd["gk"], xd["num_accepted_tokens"], None, state_layout)
    P = binding._ptr
    entry = L.gdr_prefill if prefill else L.gdr_decode
    rc = entry(ctypes.byref(dims), P(xd["query"]), P(xd["key"]), P(xd["value"]),
               P(xd["beta"]), P(xd["state_pool"]), P(xd["actual_seq_lengths"]),
               P(xd["ssm_state_indices"]), P(xd["g"]), P(xd["gk"]),
               P(xd["num_accepted_tokens"]), float(xd["scale_value"]), P(out), stream)
    assert rc == 0, L.gdr_last_error().decode()
    return out


def _error_word(L):
    flags = ctypes.c_uint32(0)
    assert L.gdr_device_error(ctypes.byref(flags), 1) == 0
    return int(flags.value)


def _grid(L):
    from gated_delta_rule_recurrent_b200 import binding

    info = binding.LaunchInfo()
    assert L.gdr_last_launch(ctypes.byref(info)) == 0
    return info.as_dict()


# (what, D_k, D_v, H, B, T): one shape per kernel family, with more tiles than
# SMs so that CTA 0 has a tile before the held one. In the prefill kernel the
# held tile is the first one of CTA 0's second consumer group, whose first
# group keeps working beside it.
FAMILIES = [
    ("single_token", 64, 512, 4, 40, 1),
    ("chunked", 64, 512, 4, 6, 3),
    ("tensor_core", 128, 128, 4, 40, 3),
    ("tensor_core", 128, 128, 4, 40, 8),  # the instance built for T = 8
    ("tensor_core_one", 128, 128, 4, 40, 1),
    ("prefill", 128, 128, 4, 40, 20),
]


@pytest.mark.parametrize("what,D_k,D_v,H,B,T", FAMILIES,
                         ids=[f"{f[0]}-T{f[5]}" for f in FAMILIES])
def test_held_tile_times_out_cleanly(hooks, what, D_k, D_v, H, B, T):
    L = hooks
    pf = what == "prefill"
    w = workloads.WORKLOADS[0].replace(name=f"hold_{what}", B=B, H_qk=H, H_v=H, T=T, D_k=D_k,
                                       D_v=D_v, pool=B + 2, lengths="full", indices="subset",
                                       scale_value=D_k**-0.5, seed=77 + D_k + T)
    x = workloads.make_inputs(w)
    pool0 = x["state_pool"].clone()

    # a normal call first: its launch shape says which tile is CTA 0's second
    assert L.gdrtest_set_hooks(0, -1) == 0
    _error_word(L)
    xd = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    _decode(L, xd, prefill=pf)
    torch.cuda.synchronize()
    launch = _grid(L)
    assert launch["kernel"] == what, launch
    grid = launch["grid"]
    n_slices = D_v // launch["tile_cols"]
    n_tiles = B * H * n_slices
    assert n_tiles > grid, "CTA 0 must have a second tile"
    held = grid  # CTA 0's second tile
    assert _error_word(L) == 0

    # the call with the held tile
    xd = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    assert L.gdrtest_set_hooks(SHORT_BUDGET, held) == 0
    t0 = time.perf_counter()
    _decode(L, xd, prefill=pf)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    assert L.gdrtest_set_hooks(0, -1) == 0
    err = _error_word(L)
    assert err & (ERR_CONSUMER | ERR_PRODUCER), f"no wait was flagged (word {err})"
    assert not err & ERR_DRAIN, f"a started copy was not seen to land (word {err})"
    if what != "chunked":  # there the finalisers wait for the same tile too
        assert err & ERR_CONSUMER, f"word {err}"
    assert elapsed < 5.0, f"the call took {elapsed:.1f} s"

    # the held tile's block is untouched; everything else is old or right
    pool = xd["state_pool"].cpu()
    b_h, s_h = held // n_slices, held % n_slices
    item, head = b_h // H, b_h % H
    slot = int(x["ssm_state_indices"][item])
    cols = slice(s_h * launch["tile_cols"], (s_h + 1) * launch["tile_cols"])
    assert np.array_equal(bits(pool[slot, head, :, cols]), bits(pool0[slot, head, :, cols])), \
        "the held tile's state block changed"
    _, st_ref, slots = run_oracle(x, False)
    new, old = f64(pool), f64(pool0)
    for r, s in enumerate(slots):
        same = bits(pool[int(s)]) == bits(pool0[int(s)])
        close = np.abs(new[int(s)] - st_ref[r]) <= RTOL * np.abs(st_ref[r]) + ATOL
        assert np.all(same | close), f"slot {int(s)} holds values that are neither old nor right"
    # CTA 0's first tile (item 0, head 0, first column slice) did commit
    slot0 = int(x["ssm_state_indices"][0])
    assert not np.array_equal(bits(pool[slot0]), bits(pool0[slot0])), \
        "CTA 0's first tile was not committed"

    # the device is healthy: a normal call right after passes parity
    xd = {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    out = _decode(L, xd, prefill=pf)
    torch.cuda.synchronize()
    check_call(x, out, pool0, xd["state_pool"].cpu(), False)
    assert _error_word(L) == 0
