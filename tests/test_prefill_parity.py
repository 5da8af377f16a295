"""Prefill (gdr_prefill / gdr_prefill_gated) against the CPU oracle (GPU).

The oracle is the same token-by-token recurrence of
"lite_boost.ops.recurrent_gated_delta_rule" (section 算法流程, steps 1-4)
used for decode calls; it loops over any number of tokens. The prefill
kernel computes it chunk by chunk with the state in fp32 tensor memory, so
these cases span many chunks, ragged lengths that end inside a chunk,
committed counts that split a chunk, NaN-poisoned padding, empty and skipped
items, several column slices and grouped heads, and decay regimes where the
running products vanish or are exactly one. The bar is the decode parity
bar: out and touched slots within 2^-7 |oracle| + 1e-3, padded outputs +0.0
and untouched slots bit for bit.
"""
import numpy as np
import pytest
import torch

from gated_delta_rule_recurrent_b200 import workloads
from parity_helpers import bits, check_call, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(built_library):
    return built_library


def run_prefill(xd, gated, out=None):
    from gated_delta_rule_recurrent_b200 import prefill, prefill_gated

    if gated:
        return prefill_gated(xd["query"], xd["key"], xd["value"], xd["a"], xd["b"],
                             xd["dt_bias"], xd["decay_scale"], xd["state_pool"],
                             xd["actual_seq_lengths"], xd["ssm_state_indices"], xd["gk"],
                             xd["num_accepted_tokens"], xd["scale_value"], out=out)
    return prefill(xd["query"], xd["key"], xd["value"], xd["beta"], xd["state_pool"],
                   xd["actual_seq_lengths"], xd["ssm_state_indices"], xd["g"], xd["gk"],
                   xd["num_accepted_tokens"], xd["scale_value"], out=out)


def _roundtrip(x, gated):
    from gated_delta_rule_recurrent_b200 import last_launch

    xd = to_device(x)
    pool_before = x["state_pool"].clone()
    out, pool = run_prefill(xd, gated)
    launched = last_launch()
    torch.cuda.synchronize()
    assert launched["kernel"] == "prefill" and launched["gated"] == gated, launched
    check_call(x, out, pool_before, pool.cpu(), gated)
    return out, pool


def _prompt(T, B=3, H_qk=2, H_v=4, D_v=128, seed=0, lengths="uniform", pool=None):
    w = workloads.WORKLOADS[0].replace(name=f"prompt_T{T}", B=B, H_qk=H_qk, H_v=H_v, T=T,
                                       D_k=128, D_v=D_v, pool=pool or B + 2, lengths=lengths,
                                       indices="subset", scale_value=128**-0.5,
                                       seed=900 + T + seed)
    return workloads.make_inputs(w, poison_padding=True)


@pytest.mark.parametrize("T", [9, 64, 200, 1024])
@pytest.mark.parametrize("gated", [False, True])
def test_prompt_lengths(T, gated):
    """Ragged lengths in [1, T] (the last chunk of an item usually partial)."""
    _roundtrip(_prompt(T), gated)


@pytest.mark.parametrize("gated", [False, True])
def test_two_slices_grouped_heads(gated):
    """D_v = 256 (two 128-column tiles per head), four value heads per q/k head."""
    _roundtrip(_prompt(77, B=2, H_qk=1, H_v=4, D_v=256, seed=1), gated)


@pytest.mark.parametrize("gated", [False, True])
def test_committed_counts_split_chunks(gated):
    """n < L: the slot gets the state after n tokens (reading E) while outputs
    run on to L; n = 0 leaves the slot's bits; n inside a chunk splits it."""
    x = _prompt(100, B=6, seed=2, lengths="full")
    x["actual_seq_lengths"] = torch.tensor([100, 100, 57, 100, 33, 90], dtype=torch.int32)
    x["num_accepted_tokens"] = torch.tensor([0, 100, 13, 8, 1, 90], dtype=torch.int32)
    _roundtrip(x, gated)


@pytest.mark.parametrize("gated", [False, True])
def test_empty_skipped_and_clamped_items(gated):
    x = _prompt(40, B=6, seed=3, lengths="full", pool=10)
    x["actual_seq_lengths"] = torch.tensor([0, -5, 99, 17, 40, 3], dtype=torch.int32)
    x["ssm_state_indices"] = torch.tensor([0, 1, 2, 3, 10, -1], dtype=torch.int32)
    x["num_accepted_tokens"] = x["actual_seq_lengths"].clamp(0, 40)
    for name in ("query", "key", "value", "gk"):
        x[name][0] = float("nan")
    out, _ = _roundtrip(x, gated)
    ob = bits(out.cpu())
    for bi in (0, 1, 4, 5):
        assert np.all(ob[bi] == 0)


@pytest.mark.parametrize("gated", [False, True])
def test_long_prompt_past_the_bench_length(gated):
    """T = 4096 (512 chunks per tile), one full-length item beside a ragged
    one, two value heads sharing a q/k head."""
    x = _prompt(4096, B=2, H_qk=1, H_v=2, seed=10, lengths="full")
    x["actual_seq_lengths"] = torch.tensor([4096, 2999], dtype=torch.int32)
    x["num_accepted_tokens"] = x["actual_seq_lengths"].clone()
    _roundtrip(x, gated)


@pytest.mark.parametrize("gated", [False, True])
def test_long_prompt_committed_mid_prompt(gated):
    """n far inside a long prompt: the slot gets the state after n tokens
    while outputs run on to L (reading E), with n on and off a chunk
    boundary."""
    x = _prompt(1000, B=3, seed=11, lengths="full")
    x["actual_seq_lengths"] = torch.tensor([1000, 977, 640], dtype=torch.int32)
    x["num_accepted_tokens"] = torch.tensor([500, 333, 640], dtype=torch.int32)
    _roundtrip(x, gated)


def test_one_token_prompt():
    _roundtrip(_prompt(1, B=4, seed=4, lengths="full"), False)


@pytest.mark.parametrize("regime", ["vanishing", "none", "mixed"])
def test_decay_regimes(regime):
    """As for multi-token decode: products that fall below the fp32 range
    within a chunk, no decay with beta near 1, and alternating decays."""
    x = _prompt(64, seed=5, lengths="full")
    if regime == "vanishing":
        x["g"][:] = -30.0
        x["gk"][:] = -5.0
    elif regime == "none":
        x["g"][:] = 0.0
        x["gk"][:] = 0.0
        x["beta"][:] = 0.99609375
    else:
        x["g"][:, :, 0::2] = -12.0
        x["g"][:, :, 1::2] = -0.01
        x["gk"][..., 0::3] = -8.0
    _roundtrip(x, False)


def test_prefill_then_decode_continues_the_state():
    """The pool a prefill leaves is the state a decode call continues from:
    prefill of 50 tokens, then one decode token, against the oracle of both
    calls in sequence."""
    from parity_helpers import run_gpu

    x = _prompt(50, B=3, seed=6, lengths="full")
    xd = to_device(x)
    pool0 = x["state_pool"].clone()
    out_p, pool_p = run_prefill(xd, False)
    torch.cuda.synchronize()
    check_call(x, out_p, pool0, pool_p.cpu(), False)
    w1 = workloads.WORKLOADS[0].replace(name="next", B=3, H_qk=2, H_v=4, T=1, D_k=128,
                                        D_v=128, pool=5, lengths="full", indices="subset",
                                        scale_value=128**-0.5, seed=950)
    y = workloads.make_inputs(w1, with_state=False)
    y["ssm_state_indices"] = x["ssm_state_indices"].clone()
    y["state_pool"] = pool_p.cpu()
    yd = to_device(y)
    yd["state_pool"] = pool_p
    pool_mid = y["state_pool"].clone()
    out_d, pool_d = run_gpu(yd, False)
    torch.cuda.synchronize()
    check_call(y, out_d, pool_mid, pool_d.cpu(), False)


def test_deterministic_and_error_word_clear():
    from gated_delta_rule_recurrent_b200 import device_error

    x = _prompt(130, seed=7)
    device_error(reset=True)
    a_out, a_pool = run_prefill(to_device(x), True)
    b_out, b_pool = run_prefill(to_device(x), True)
    torch.cuda.synchronize()
    assert np.array_equal(bits(a_out.cpu()), bits(b_out.cpu()))
    assert np.array_equal(bits(a_pool.cpu()), bits(b_pool.cpu()))
    assert device_error(reset=True) == 0


def test_unsupported_sizes_are_refused():
    from gated_delta_rule_recurrent_b200 import GdrError

    w = workloads.WORKLOADS[0].replace(name="dk64", B=2, T=20, lengths="full", indices="subset",
                                       pool=3, seed=8)
    x = to_device(workloads.make_inputs(w))  # D_k = 64
    with pytest.raises(GdrError, match="GDR_ERR_UNSUPPORTED"):
        run_prefill(x, False)
