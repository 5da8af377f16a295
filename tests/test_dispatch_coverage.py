"""Every kernel form the entry points can launch is run, checked against the
oracle, and watched for stray writes.

The library lists its kernel forms (``gdr_kernel_form``: kernel family,
D_k, tile width, gate, pool layout). ``CASES`` below names one call shape per
form. A CPU test requires the two sets to be equal, so a new table entry in
the dispatcher cannot ship without a case that reaches it. The GPU test runs
each case, asks the library which kernel it launched (``gdr_last_launch``)
and requires the case's form, then compares the call with the oracle of
"lite_boost.ops.recurrent_gated_delta_rule" (section 算法流程, steps 1-4) as
the other parity tests do.

Every tensor of a GPU case sits inside a larger allocation with 4 KiB guard
bands of a fixed byte pattern on both sides. After the call, each guard byte
must be unchanged and every input must keep its bits: no kernel writes outside
``out`` and the pool slots its items name. This is the test of stray writes
that compute-sanitizer would otherwise give.

Tile widths are chosen by the number of tiles per SM, so the batch size that
reaches a width is computed from the device's SM count with the dispatcher's
rule (the widest width that divides D_v and gives every SM at least 16 tiles,
else the narrowest).
"""
import math

import numpy as np
import pytest
import torch

from gated_delta_rule_recurrent_b200 import workloads

MIN_TILES_PER_SM = 16
GUARD = 4096
PATTERN = 0xA5

# (kernel, D_k, tile_cols, layout, T, D_v, H): one call shape per kernel form,
# and one more where a form has a separate instance for some token count (the
# tensor-core kernel at T = 8); each runs with and without the fused gate. B
# is derived at run time.
CASES = [
    ("prefill", 128, 128, "kv", 21, 256, 4),
    ("tensor_core_one", 128, 128, "kv", 1, 256, 4),
    ("tensor_core", 128, 128, "kv", 5, 256, 4),
    ("tensor_core", 128, 128, "kv", 8, 256, 4),  # the instance built for T = 8
    ("tensor_core_one", 128, 128, "vk", 1, 256, 4),
    ("tensor_core", 128, 128, "vk", 5, 256, 4),
    ("tensor_core", 128, 128, "vk", 8, 256, 4),
    ("rows", 64, 64, "vk", 1, 512, 64),
    ("rows", 64, 16, "vk", 1, 512, 64),
    ("rows", 128, 64, "vk", 1, 192, 64),
    ("rows", 128, 16, "vk", 1, 192, 4),
    ("single_token", 64, 512, "kv", 1, 512, 64),
    ("single_token", 64, 256, "kv", 1, 512, 64),
    ("single_token", 64, 128, "kv", 1, 512, 64),
    ("single_token", 64, 64, "kv", 1, 512, 64),
    ("chunked", 64, 128, "kv", 4, 512, 64),
    ("chunked", 64, 64, "kv", 4, 512, 64),
    ("chunked", 64, 128, "vk", 3, 512, 64),
    ("chunked", 64, 64, "vk", 2, 512, 64),
    ("single_token", 128, 64, "kv", 1, 192, 4),
    ("chunked", 128, 64, "kv", 6, 192, 4),
    ("chunked", 128, 64, "vk", 2, 192, 4),
]

# tile widths of the width-chosen tables, widest first
WIDTHS = {("single_token", 64, "kv"): (512, 256, 128, 64), ("chunked", 64, "kv"): (128, 64),
          ("chunked", 64, "vk"): (128, 64), ("rows", 64, "vk"): (64, 16),
          ("rows", 128, "vk"): (64, 16)}


def case_key(case, gated):
    kernel, D_k, vs, layout = case[:4]
    return (kernel, D_k, vs, bool(gated), layout)


def batch_for(case, sms):
    """Smallest batch whose call the dispatcher sends to this case's tile width."""
    kernel, D_k, vs, layout, T, D_v, H = case
    widths = WIDTHS.get((kernel, D_k, layout))
    if widths is None or vs == widths[-1]:
        return 3  # fixed-width forms, and the narrowest width: a few items
    need = MIN_TILES_PER_SM * sms
    B = math.ceil(need / (H * D_v // vs))
    wider = widths[widths.index(vs) - 1] if widths.index(vs) > 0 else None
    assert wider is None or B * H * D_v // wider < need
    return B


def test_every_kernel_form_has_a_case(built_library):
    from gated_delta_rule_recurrent_b200 import kernel_forms

    forms = {(f["kernel"], f["D_k"], f["tile_cols"], f["gated"], f["layout"])
             for f in kernel_forms()}
    cases = {case_key(c, g) for c in CASES for g in (False, True)}
    assert len(forms) == len(kernel_forms()), "a kernel form is listed twice"
    assert forms == cases, (f"forms without a case: {sorted(forms - cases)}; "
                            f"cases of no form: {sorted(cases - forms)}")


# --------------------------------------------------------------------------- GPU


def guarded(t: torch.Tensor):
    """A device copy of ``t`` placed inside a byte buffer with guard bands."""
    n = t.numel() * t.element_size()
    buf = torch.full((n + 2 * GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
    view = buf[GUARD:GUARD + n].view(t.dtype).view(t.shape)
    view.copy_(t)
    return view, buf


def guards_intact(buf) -> bool:
    return bool((buf[:GUARD] == PATTERN).all()) and bool((buf[-GUARD:] == PATTERN).all())


@pytest.mark.gpu
@pytest.mark.parametrize("gated", [False, True])
@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[0]}-Dk{c[1]}-w{c[2]}-{c[3]}-T{c[4]}")
def test_kernel_form(built_library, case, gated):
    from gated_delta_rule_recurrent_b200 import (decode, decode_gated, last_launch, prefill,
                                                 prefill_gated)
    from parity_helpers import bits, check_call, to_vk

    kernel, D_k, vs, layout, T, D_v, H = case
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    B = batch_for(case, sms)
    w = workloads.WORKLOADS[0].replace(
        name="form", B=B, H_qk=H, H_v=H, T=T, D_k=D_k, D_v=D_v, pool=B + 3,
        lengths="uniform" if T > 1 else "full", indices="subset", scale_value=D_k**-0.5,
        seed=31 * B + 7 * T + D_v + D_k + vs)
    x = workloads.make_inputs(w, poison_padding=T > 1)
    pool_before = x["state_pool"].clone()

    names = ["query", "key", "value", "gk", "actual_seq_lengths", "ssm_state_indices",
             "num_accepted_tokens"] + (["a", "b", "dt_bias", "decay_scale"] if gated
                                       else ["beta", "g"])
    dev, bufs = {}, {}
    for n in names:
        dev[n], bufs[n] = guarded(x[n])
    pool_src = to_vk(x["state_pool"]) if layout == "vk" else x["state_pool"]
    dev["state_pool"], bufs["state_pool"] = guarded(pool_src)
    out0 = torch.zeros(B, H, T, D_v, dtype=torch.bfloat16)
    dev["out"], bufs["out"] = guarded(out0)
    inputs_before = {n: bits(x[n]) for n in names}

    args = (dev["query"], dev["key"], dev["value"])
    if kernel == "prefill":
        if gated:
            prefill_gated(*args, dev["a"], dev["b"], dev["dt_bias"], dev["decay_scale"],
                          dev["state_pool"], dev["actual_seq_lengths"],
                          dev["ssm_state_indices"], dev["gk"], dev["num_accepted_tokens"],
                          x["scale_value"], out=dev["out"])
        else:
            prefill(*args, dev["beta"], dev["state_pool"], dev["actual_seq_lengths"],
                    dev["ssm_state_indices"], dev["g"], dev["gk"], dev["num_accepted_tokens"],
                    x["scale_value"], out=dev["out"])
    elif gated:
        decode_gated(*args, dev["a"], dev["b"], dev["dt_bias"], dev["decay_scale"],
                     dev["state_pool"], dev["actual_seq_lengths"], dev["ssm_state_indices"],
                     dev["gk"], dev["num_accepted_tokens"], x["scale_value"], out=dev["out"],
                     state_layout=layout)
    else:
        decode(*args, dev["beta"], dev["state_pool"], dev["actual_seq_lengths"],
               dev["ssm_state_indices"], dev["g"], dev["gk"], dev["num_accepted_tokens"],
               x["scale_value"], out=dev["out"], state_layout=layout)
    launched = last_launch()
    torch.cuda.synchronize()

    got = (launched["kernel"], launched["D_k"], launched["tile_cols"], launched["gated"],
           launched["layout"])
    assert got == case_key(case, gated), f"dispatched {launched}"
    for n, buf in bufs.items():
        assert guards_intact(buf), f"a guard band around {n} changed"
    for n in names:
        assert np.array_equal(bits(dev[n].cpu()), inputs_before[n]), f"input {n} changed"
    pool_after = dev["state_pool"].cpu()
    if layout == "vk":
        pool_after = to_vk(pool_after)
    check_call(x, dev["out"].cpu(), pool_before, pool_after, gated)
