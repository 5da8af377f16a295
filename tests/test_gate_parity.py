"""The standalone LinearAttentionGate op (CUDA) against the CPU oracle (GPU).

"com.microsoft.LinearAttentionGate", sections Description, Inputs, Outputs and
Type constraints: decay = decay_scale * softplus(a + dt_bias) and beta =
sigmoid(b), computed in float32 and narrowed to the tensor type on store. The
oracle computes in float64; both sides narrow once, so an element may differ
by one unit in the last place of the narrow type (fp16, bf16) or by a few fp32
ulps from the fp32 exponential and logarithm.
"""
import numpy as np
import pytest
import torch

from gated_delta_rule_recurrent_b200 import workloads
from oracle import gdr_oracle as O

pytestmark = pytest.mark.gpu

DTYPES = {torch.float32: (4e-6, 1e-37), torch.float16: (2.0 ** -10, 2.0 ** -24),
          torch.bfloat16: (2.0 ** -7, 1e-37)}


@pytest.fixture(scope="module", autouse=True)
def _lib(built_library):
    return built_library


def narrow(x64, dtype):
    """The oracle's float64 values rounded to nearest even in `dtype`."""
    if dtype == torch.float32:
        return x64.astype(np.float32).astype(np.float64)
    if dtype == torch.float16:
        return x64.astype(np.float16).astype(np.float64)
    return O.bf16_round(x64)


def check(got, ref64, dtype):
    rtol, atol = DTYPES[dtype]
    g = got.float().cpu().numpy().astype(np.float64)
    with np.errstate(over="ignore", invalid="ignore"):  # inf/NaN inputs are intended
        r = narrow(ref64, dtype)
    both_nan = np.isnan(g) & np.isnan(r)
    same_inf = np.isinf(g) & np.isinf(r) & (np.sign(g) == np.sign(r))
    with np.errstate(invalid="ignore"):
        ok = both_nan | same_inf | (np.abs(g - r) <= rtol * np.abs(r) + atol)
    assert ok.all(), (f"{(~ok).sum()} of {ok.size} elements off; first: got "
                      f"{g[~ok][:4]}, want {r[~ok][:4]}")


def run(x, want_beta, dtype):
    from gated_delta_rule_recurrent_b200 import linear_attention_gate

    xd = {k: v.cuda() for k, v in x.items()}
    decay, beta = linear_attention_gate(xd["a"], xd["dt_bias"], xd["decay_scale"],
                                        b=xd["b"], want_beta=want_beta)
    torch.cuda.synchronize()
    ref_decay, ref_beta = O.linear_attention_gate(x["a"].double().numpy(),
                                                  x["dt_bias"].double().numpy(),
                                                  x["decay_scale"].double().numpy(),
                                                  x["b"].double().numpy() if want_beta else None)
    check(decay, ref_decay, dtype)
    if want_beta:
        check(beta, ref_beta, dtype)
    else:
        assert beta is None
    return decay, beta


@pytest.mark.parametrize("dtype", list(DTYPES))
@pytest.mark.parametrize("shape", [(64,), (2, 3, 64), (5, 1, 7), (512, 1, 64), (3, 5, 2, 33)])
@pytest.mark.parametrize("want_beta", [True, False])
def test_shapes_and_types(dtype, shape, want_beta):
    run(workloads.make_gate_inputs(shape, dtype, seed=len(shape) * 100 + shape[-1]), want_beta,
        dtype)


@pytest.mark.parametrize("dtype", list(DTYPES))
def test_large_tensor(dtype):
    """32768 rows x 8 tokens x 64 heads: many vectors per thread."""
    run(workloads.make_gate_inputs((32768, 8, 64), dtype, seed=5), True, dtype)


@pytest.mark.parametrize("dtype", list(DTYPES))
def test_misaligned_views_take_the_scalar_path(dtype):
    """Tensors that start off a 16-byte boundary (views one element in)."""
    from gated_delta_rule_recurrent_b200 import linear_attention_gate

    x = workloads.make_gate_inputs((9, 2, 13), dtype, seed=77)
    n = x["a"].numel()
    big_a = torch.zeros(n + 1, dtype=dtype, device="cuda")
    big_b = torch.zeros(n + 1, dtype=dtype, device="cuda")
    big_a[1:] = x["a"].reshape(-1).cuda()
    big_b[1:] = x["b"].reshape(-1).cuda()
    a = big_a[1:].view(x["a"].shape)
    b = big_b[1:].view(x["b"].shape)
    out_d = torch.empty(n + 1, dtype=dtype, device="cuda")[1:].view(x["a"].shape)
    out_b = torch.empty(n + 1, dtype=dtype, device="cuda")[1:].view(x["a"].shape)
    assert a.data_ptr() % 16 != 0
    decay, beta = linear_attention_gate(a, x["dt_bias"].cuda(), x["decay_scale"].cuda(), b=b,
                                        decay=out_d, beta=out_b)
    torch.cuda.synchronize()
    ref_decay, ref_beta = O.linear_attention_gate(x["a"].double().numpy(),
                                                  x["dt_bias"].double().numpy(),
                                                  x["decay_scale"].double().numpy(),
                                                  x["b"].double().numpy())
    check(decay, ref_decay, dtype)
    check(beta, ref_beta, dtype)


@pytest.mark.parametrize("dtype", list(DTYPES))
def test_per_head_vectors_off_a_16_byte_boundary(dtype):
    """H a multiple of 8 with dt_bias and decay_scale one float into their
    buffers: the vector path then reads them element by element."""
    from gated_delta_rule_recurrent_b200 import last_launch, linear_attention_gate

    x = workloads.make_gate_inputs((300, 4, 64), dtype, seed=78)
    H = x["a"].shape[-1]
    dtb = torch.zeros(H + 1, dtype=torch.float32, device="cuda")
    dsc = torch.zeros(H + 1, dtype=torch.float32, device="cuda")
    dtb[1:] = x["dt_bias"].cuda()
    dsc[1:] = x["decay_scale"].cuda()
    assert dtb[1:].data_ptr() % 16 != 0
    decay, beta = linear_attention_gate(x["a"].cuda(), dtb[1:], dsc[1:], b=x["b"].cuda(),
                                        want_beta=True)
    torch.cuda.synchronize()
    assert last_launch()["kernel"] == "gate"
    ref_decay, ref_beta = O.linear_attention_gate(x["a"].double().numpy(),
                                                  x["dt_bias"].double().numpy(),
                                                  x["decay_scale"].double().numpy(),
                                                  x["b"].double().numpy())
    check(decay, ref_decay, dtype)
    check(beta, ref_beta, dtype)


@pytest.mark.parametrize("dtype", list(DTYPES))
def test_special_values(dtype):
    """Saturation, infinities and NaN: softplus(-inf) = 0 (decay = -0.0 for a
    negative scale), softplus(+inf) = inf, sigmoid(+-inf) = 1, 0; NaN propagates."""
    x = workloads.make_gate_inputs((4, 16), dtype, seed=3)
    specials = torch.tensor([0.0, -0.0, 80.0, -80.0, 1e4, -1e4, float("inf"), float("-inf"),
                             float("nan"), 20.0, -20.0, 1e-30, 3.0, -3.0, 15.0, -15.0])
    x["a"][0] = specials.to(dtype)
    x["b"][1] = specials.to(dtype)
    x["a"][2] = -specials.to(dtype)
    x["b"][3] = -specials.to(dtype)
    run(x, True, dtype)


def test_b_given_but_beta_not_requested_is_not_read():
    x = workloads.make_gate_inputs((6, 32), torch.bfloat16, seed=11)
    x["b"][:] = float("nan")
    decay, beta = run(x, False, torch.bfloat16)
    assert beta is None and torch.isfinite(decay.float()).all()


def test_beta_without_b_is_rejected():
    from gated_delta_rule_recurrent_b200 import linear_attention_gate

    x = {k: v.cuda() for k, v in workloads.make_gate_inputs((2, 8), torch.float32).items()}
    with pytest.raises(RuntimeError):
        linear_attention_gate(x["a"], x["dt_bias"], x["decay_scale"], b=None, want_beta=True)
