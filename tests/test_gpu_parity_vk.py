"""The k-contiguous state layout [pool, H_v, D_v, D_k] (GPU).

The same op with the state pool stored per head as the transpose of the
page's [D_k, D_v] tile, the layout the NPU operator keeps internally
("lite_boost.ops.recurrent_gated_delta_rule", section 注). Each call runs on
the transposed pool; the pool it leaves is transposed back and checked
against the oracle (which keeps the page's layout) exactly as for the default
layout: out and touched slots within the tolerance, padded outputs +0.0 and
untouched slots bit for bit.
"""
import numpy as np
import pytest
import torch

from gated_delta_rule_recurrent_b200 import workloads
from parity_helpers import bits, check_call, run_gpu, to_device, to_vk

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(built_library):
    return built_library


def _roundtrip_vk(x, gated, items=None):
    xd = to_device(x)
    pool_before = x["state_pool"].clone()
    xd["state_pool"] = to_vk(xd["state_pool"])
    out, pool_vk = run_gpu(xd, gated, state_layout="vk")
    torch.cuda.synchronize()
    check_call(x, out, pool_before, to_vk(pool_vk).cpu(), gated, items)
    return out, pool_vk


@pytest.mark.parametrize("cfg", [0, 1, 2, 3])
@pytest.mark.parametrize("gated", [False, True])
def test_workloads(cfg, gated):
    _roundtrip_vk(workloads.make_inputs(cfg, poison_padding=(cfg == 3)), gated)


def test_large_batch_gated_full_size_sampled():
    x = workloads.make_inputs(4)
    _roundtrip_vk(x, True, [0, 1, 100, 255, 256, 511])


@pytest.mark.parametrize("T", list(range(1, 9)))
def test_every_token_count(T):
    w = workloads.WORKLOADS[0].replace(name=f"vkT{T}", B=3, T=T, D_k=128, D_v=128, pool=4,
                                       lengths="full", indices="subset", seed=150 + T)
    _roundtrip_vk(workloads.make_inputs(w), False)


@pytest.mark.parametrize("D_k,D_v,H_qk,H_v,T", [
    (64, 192, 3, 6, 3),
    (128, 320, 2, 8, 5),
    (64, 64, 1, 5, 8),
    (128, 64, 7, 7, 1),
    (64, 512, 4, 4, 2),
    (128, 128, 2, 4, 1),    # one token on the tensor-core path
    (128, 256, 2, 4, 8),    # two 128-column slices, all 8 tokens
    (128, 512, 1, 3, 3),    # four slices, multi-query
])
@pytest.mark.parametrize("gated", [False, True])
def test_ragged_shapes(D_k, D_v, H_qk, H_v, T, gated):
    w = workloads.WORKLOADS[0].replace(name="vkragged", B=5, H_qk=H_qk, H_v=H_v, T=T, D_k=D_k,
                                       D_v=D_v, pool=9, lengths="uniform", indices="subset",
                                       scale_value=D_k**-0.5, seed=17 + D_k + D_v + T)
    _roundtrip_vk(workloads.make_inputs(w, poison_padding=True), gated)


def test_edge_lengths_and_slots():
    w = workloads.WORKLOADS[0].replace(name="vkedges", B=8, H_qk=2, H_v=4, T=4, D_k=128,
                                       D_v=128, pool=10, lengths="full", indices="subset",
                                       seed=199)
    x = workloads.make_inputs(w)
    x["actual_seq_lengths"] = torch.tensor([0, -3, 9, 2, 4, 1, 3, 4], dtype=torch.int32)
    x["ssm_state_indices"] = torch.tensor([0, 1, 2, 3, -1, 10, 6, 9], dtype=torch.int32)
    x["num_accepted_tokens"] = x["actual_seq_lengths"].clamp(0, 4)
    for name in ("query", "key", "value", "gk"):
        x[name][3, :, 2:] = float("nan")
        x[name][0] = float("nan")
    out, _ = _roundtrip_vk(x, False)
    ob = bits(out.cpu())
    for bi in (0, 1, 4, 5):
        assert np.all(ob[bi] == 0)


def test_same_results_as_the_default_layout():
    """Both layouts compute the same sums in the same order up to the tile
    split; outputs agree within the tolerance and are each deterministic."""
    x = workloads.make_inputs(3)
    xd_kv = to_device(x)
    out_kv, pool_kv = run_gpu(xd_kv, False)
    xd_vk = to_device(x)
    xd_vk["state_pool"] = to_vk(xd_vk["state_pool"])
    out_vk, pool_vk = run_gpu(xd_vk, False, state_layout="vk")
    xd_vk2 = to_device(x)
    xd_vk2["state_pool"] = to_vk(xd_vk2["state_pool"])
    out_vk2, _ = run_gpu(xd_vk2, False, state_layout="vk")
    torch.cuda.synchronize()
    assert np.array_equal(bits(out_vk.cpu()), bits(out_vk2.cpu()))
    d = (out_kv.float() - out_vk.float()).abs()
    assert float(d.max()) <= 2 * (2.0**-7 * float(out_kv.float().abs().max()) + 1e-3)
    assert pool_kv.shape == to_vk(pool_vk).shape


@pytest.mark.parametrize("T", [1, 4, 8])
def test_committed_token_counts(T):
    w = workloads.WORKLOADS[0].replace(name=f"vkcommit{T}", B=16, T=T, D_k=128, D_v=128,
                                       pool=20, lengths="uniform", indices="subset",
                                       seed=700 + T)
    x = workloads.make_inputs(w)
    L = x["actual_seq_lengths"]
    gen = torch.Generator().manual_seed(100 + T)
    x["num_accepted_tokens"] = (torch.rand(L.shape, generator=gen) * (L + 1).float()).floor().to(torch.int32)
    x["num_accepted_tokens"][0] = 0
    _roundtrip_vk(x, False)
