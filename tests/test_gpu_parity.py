"""CUDA path against the CPU oracle, element by element, through the C ABI (GPU).

Covers the five seeded workloads (the full-size gated workload on sampled
batch items, in the exact launch configuration the benchmark times), ragged
shapes that span several tiles, every token count 1..8, grouped heads, and the
edge cases of the op: zero-length items, padded tokens with NaN inputs, slot
indices outside the pool, lengths outside [0, T], untouched slots, an empty
batch, chained calls, and a non-default stream.
"""
import numpy as np
import pytest
import torch

from gated_delta_rule_recurrent_b200 import workloads
from parity_helpers import bits, check_call, run_gpu, to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(built_library):
    return built_library


def _roundtrip(x, gated, items=None):
    xd = to_device(x)
    pool_before = x["state_pool"].clone()
    out, pool = run_gpu(xd, gated)
    torch.cuda.synchronize()
    check_call(x, out, pool_before, pool.cpu(), gated, items)
    return out, pool


@pytest.mark.parametrize("cfg", [0, 1, 2])
@pytest.mark.parametrize("gated", [False, True])
def test_workloads_small(cfg, gated):
    _roundtrip(workloads.make_inputs(cfg), gated)


@pytest.mark.parametrize("gated", [False, True])
def test_speculative_multi_token_with_nan_padding(gated):
    x = workloads.make_inputs(3, poison_padding=True)
    assert (x["actual_seq_lengths"] < 8).any() and (x["actual_seq_lengths"] == 8).any()
    _roundtrip(x, gated)


def test_large_batch_gated_full_size_sampled():
    """The 512 x 64-head x 64x512 gated workload, as the benchmark launches it;
    the oracle checks a spread of batch items one by one."""
    x = workloads.make_inputs(4)
    items = [0, 1, 77, 255, 256, 400, 510, 511]
    _roundtrip(x, True, items)


@pytest.mark.slow
def test_large_batch_gated_full_size_all_items():
    """The same call with every one of the 512 items checked against the oracle
    (about 40 s of oracle time)."""
    _roundtrip(workloads.make_inputs(4), True)


@pytest.mark.parametrize("D_k,D_v,H_qk,H_v,T", [
    (64, 192, 3, 6, 3),     # three column slices, grouped heads
    (128, 320, 2, 8, 5),    # five slices, 4 value heads per q/k head
    (64, 64, 1, 5, 8),      # multi-query, all 8 tokens
    (128, 64, 7, 7, 1),
    (128, 128, 2, 2, 2),
    (64, 512, 4, 4, 6),
    (128, 256, 2, 4, 8),    # two 128-column slices, all 8 tokens
    (128, 512, 1, 3, 3),    # four slices, multi-query
])
@pytest.mark.parametrize("gated", [False, True])
def test_ragged_shapes(D_k, D_v, H_qk, H_v, T, gated):
    w = workloads.WORKLOADS[0].replace(name="ragged", B=5, H_qk=H_qk, H_v=H_v, T=T, D_k=D_k,
                                       D_v=D_v, pool=9, lengths="uniform", indices="subset",
                                       scale_value=D_k**-0.5, seed=7 + D_k + D_v + T)
    _roundtrip(workloads.make_inputs(w, poison_padding=True), gated)


@pytest.mark.parametrize("gated", [False, True])
def test_many_tiles_with_empty_items(gated):
    """Thousands of tiles per call, so every CTA reuses its stages many times,
    with runs of zero-length items and slots outside the pool between stored tiles."""
    w = workloads.WORKLOADS[3].replace(name="sparse", B=96, pool=128, seed=4242)
    x = workloads.make_inputs(w, poison_padding=True)
    L = x["actual_seq_lengths"]
    L[1::3] = 0
    L[2::7] = -1
    x["ssm_state_indices"][5::11] = 1000
    x["num_accepted_tokens"] = L.clamp(0, 8)
    for name in ("query", "key", "value", "gk"):
        x[name][L <= 0] = float("nan")
    _roundtrip(x, gated)


@pytest.mark.parametrize("T", list(range(1, 9)))
def test_every_token_count(T):
    w = workloads.WORKLOADS[0].replace(name=f"T{T}", B=3, T=T, pool=4, lengths="full",
                                       indices="subset", seed=50 + T)
    _roundtrip(workloads.make_inputs(w), False)


@pytest.mark.parametrize("regime", ["vanishing", "none", "mixed"])
def test_decay_regimes_multi_token(regime):
    """Multi-token calls regroup the recurrence around running products of the
    per-token decays. "vanishing": g = -30 and gk = -5, so the products fall
    below the fp32 range within a few tokens (the state forgets, nothing may
    overflow or turn NaN); "none": g = gk = 0 with beta near 1 (the pure delta
    rule, where the regrouped sums cancel the most); "mixed": alternating
    strong and weak decay per token and per row."""
    w = workloads.WORKLOADS[3].replace(name=f"decay_{regime}", B=12, pool=16, seed=321)
    x = workloads.make_inputs(w)
    if regime == "vanishing":
        x["g"][:] = -30.0
        x["gk"][:] = -5.0
    elif regime == "none":
        x["g"][:] = 0.0
        x["gk"][:] = 0.0
        x["beta"][:] = 0.99609375  # bf16 just below 1
    else:
        x["g"][:, :, 0::2] = -12.0
        x["g"][:, :, 1::2] = -0.01
        x["gk"][..., 0::3] = -8.0
    _roundtrip(x, False)


@pytest.mark.parametrize("gated", [False, True])
def test_edge_lengths_and_slots(gated):
    w = workloads.WORKLOADS[0].replace(name="edges", B=8, H_qk=2, H_v=4, T=4, D_k=128,
                                       D_v=128, pool=10, lengths="full", indices="subset",
                                       seed=99)
    x = workloads.make_inputs(w)
    # lengths: 0, negative, beyond T, partial; slots: outside the pool both ways
    x["actual_seq_lengths"] = torch.tensor([0, -3, 9, 2, 4, 1, 3, 4], dtype=torch.int32)
    x["ssm_state_indices"] = torch.tensor([0, 1, 2, 3, -1, 10, 6, 9], dtype=torch.int32)
    x["num_accepted_tokens"] = x["actual_seq_lengths"].clamp(0, 4)
    for name in ("query", "key", "value", "gk"):
        x[name][3, :, 2:] = float("nan")
        x[name][0] = float("nan")
    x["beta"][0] = float("nan")
    x["g"][0] = float("nan")
    x["a"][0] = float("nan")
    x["b"][0] = float("nan")
    out, _ = _roundtrip(x, gated)
    ob = bits(out.cpu())
    for bi in (0, 1, 4, 5):
        assert np.all(ob[bi] == 0)


def test_empty_batch():
    x = to_device(workloads.make_inputs(0))
    xd = {k: (v[:0] if isinstance(v, torch.Tensor) and k not in
              ("state_pool", "dt_bias", "decay_scale") else v) for k, v in x.items()}
    before = bits(x["state_pool"])
    out, pool = run_gpu(xd, False)
    torch.cuda.synchronize()
    assert out.shape[0] == 0
    assert np.array_equal(bits(pool), before)


def test_chained_calls_match_chained_oracle():
    """The pool written by one call feeds the next (the page's state_out -> state)."""
    x = workloads.make_inputs(2)
    xd = to_device(x)
    for step in range(3):
        pool_before = xd["state_pool"].cpu()
        x["state_pool"] = pool_before
        out, pool = run_gpu(xd, False)
        torch.cuda.synchronize()
        check_call(x, out, pool_before, pool.cpu(), False)
        # next token: fresh per-token inputs, same pool
        nxt = workloads.make_inputs(2, seed=2000 + step, with_state=False)
        for k in ("query", "key", "value", "beta", "g", "gk"):
            xd[k] = nxt[k].cuda()
            x[k] = nxt[k]


def test_side_stream_and_determinism():
    x = workloads.make_inputs(3)
    xd1 = to_device(x)
    xd2 = to_device(x)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        out1, pool1 = run_gpu(xd1, False)
    s.synchronize()
    out2, pool2 = run_gpu(xd2, False)
    torch.cuda.synchronize()
    assert np.array_equal(bits(out1), bits(out2))
    assert np.array_equal(bits(pool1), bits(pool2))


def test_device_error_word_stays_clear():
    from gated_delta_rule_recurrent_b200 import device_error

    device_error(reset=True)
    for cfg in (0, 2, 3):
        _roundtrip(workloads.make_inputs(cfg), cfg == 2)
    assert device_error(reset=True) == 0


def test_device_errors_reported_without_launch():
    from gated_delta_rule_recurrent_b200 import GdrError

    x = to_device(workloads.make_inputs(0))
    before = bits(x["state_pool"])
    bad = dict(x)
    bad["query"] = torch.zeros(2, 3, 2, 64, dtype=torch.bfloat16, device="cuda")
    bad["key"] = bad["query"].clone()
    with pytest.raises(GdrError, match="GDR_ERR_DIMS"):
        run_gpu(bad, False)  # H_v = 4 is not a multiple of H_qk = 3
    # a misaligned view of otherwise valid storage
    big = torch.zeros(x["value"].numel() + 1, dtype=torch.bfloat16, device="cuda")
    bad = dict(x)
    bad["value"] = big[1:].view(x["value"].shape)
    with pytest.raises(GdrError, match="GDR_ERR_ALIGN"):
        run_gpu(bad, False)
    torch.cuda.synchronize()
    assert np.array_equal(bits(x["state_pool"]), before)


@pytest.mark.parametrize("T", [1, 2, 5, 8])
@pytest.mark.parametrize("gated", [False, True])
def test_committed_token_counts(T, gated):
    """num_accepted_tokens = n in [0, L] per item: outputs of all L tokens,
    the slot left with the state after n tokens (untouched when n = 0)."""
    w = workloads.WORKLOADS[0].replace(name=f"commit{T}", B=24, H_qk=2, H_v=4, T=T, D_k=128,
                                       D_v=128, pool=32, lengths="uniform", indices="subset",
                                       seed=600 + T)
    x = workloads.make_inputs(w)
    L = x["actual_seq_lengths"]
    gen = torch.Generator().manual_seed(T)
    n = (torch.rand(L.shape, generator=gen) * (L + 1).float()).floor().to(torch.int32)
    n[0], n[1] = 0, L[1]  # nothing committed; everything committed
    n[2] = 99             # clamped to L
    x["num_accepted_tokens"] = n
    _roundtrip(x, gated)


def test_committed_counts_absent_means_all():
    x = workloads.make_inputs(3)
    x["num_accepted_tokens"] = None
    xd = to_device(x)
    pool_before = x["state_pool"].clone()
    out, pool = run_gpu(xd, False)
    torch.cuda.synchronize()
    x2 = dict(x)
    x2["num_accepted_tokens"] = x["actual_seq_lengths"].clone()
    check_call(x2, out, pool_before, pool.cpu(), False)


def test_cuda_graph_capture_and_replay():
    """A decode call captured in a CUDA graph replays with the same results as
    a direct call: the library queues only kernels on the caller's stream
    (configuration and tensor maps are host work done at capture time)."""
    from gated_delta_rule_recurrent_b200 import decode

    x = workloads.make_inputs(3)
    direct = to_device(x)
    out_ref, pool_ref = run_gpu(direct, False)
    torch.cuda.synchronize()
    xd = to_device(x)
    pool0 = xd["state_pool"].clone()
    out = torch.empty_like(out_ref)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):  # warm-up outside the graph (first-call setup)
        run_gpu(xd, False, out=out)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    xd["state_pool"].copy_(pool0)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        decode(xd["query"], xd["key"], xd["value"], xd["beta"], xd["state_pool"],
               xd["actual_seq_lengths"], xd["ssm_state_indices"], xd["g"], xd["gk"],
               xd["num_accepted_tokens"], xd["scale_value"], out=out)
    xd["state_pool"].copy_(pool0)
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert np.array_equal(bits(out.cpu()), bits(out_ref.cpu()))
    assert np.array_equal(bits(xd["state_pool"].cpu()), bits(pool_ref.cpu()))
    # a second replay continues from the pool the first one left
    g.replay()
    torch.cuda.synchronize()
    assert not np.array_equal(bits(xd["state_pool"].cpu()), bits(pool_ref.cpu()))
