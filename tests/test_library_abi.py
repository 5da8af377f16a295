"""The C-ABI library loads, exports every symbol include/gdr.h declares, and its
host-side checks reject bad arguments before anything is queued (CPU only).

The argument-check cases pass placeholder pointers that must never reach a
kernel, so they run only on a machine without a CUDA device; the GPU tests
repeat the interesting cases with real device buffers.
"""
import ctypes
import os
import re

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdr.h")

GDR_OK, GDR_ERR_NULL, GDR_ERR_DIMS, GDR_ERR_ALIGN, GDR_ERR_UNSUPPORTED, GDR_ERR_CUDA = range(6)


def declared_symbols():
    with open(HEADER) as f:
        text = f.read()
    return re.findall(r"GDR_API\s+[\w\s\*]+?\b(gdr_\w+)\s*\(", text)


def test_header_declares_the_entry_points():
    names = declared_symbols()
    for want in ("gdr_decode", "gdr_gate_fused", "gdr_linear_attention_gate",
                 "gdr_status_string", "gdr_last_error", "gdr_abi_version"):
        assert want in names
    assert len(names) == len(set(names))


def test_library_exports_every_declared_symbol(built_library):
    lib = ctypes.CDLL(built_library)
    for name in declared_symbols():
        assert hasattr(lib, name), f"{name} declared in gdr.h but not exported"


def test_internal_symbols_are_hidden(built_library):
    nm = os.popen(f"nm -D --defined-only {built_library}").read()
    exported = {line.split()[-1] for line in nm.splitlines() if " T " in line}
    gdr_exported = {s for s in exported if s.startswith("gdr_")}
    assert gdr_exported == set(declared_symbols())


def test_status_strings_and_version(built_library):
    from gated_delta_rule_recurrent_b200 import binding

    L = binding.lib()
    assert L.gdr_abi_version() == 6
    for code, name in binding.STATUS_NAMES.items():
        assert L.gdr_status_string(code).decode() == name
    assert L.gdr_status_string(99).decode() == "unknown status"


no_device = pytest.mark.skipif(torch.cuda.is_available(),
                               reason="placeholder pointers are for a machine without a GPU")


def _call_decode(lib, dims, ptr=16, misalign=0, nulls=()):
    from gated_delta_rule_recurrent_b200.binding import Dims

    d = Dims(*dims)
    args = []
    for i in range(10):
        args.append(None if i in nulls else ctypes.c_void_p(ptr + misalign))
    q, k, v, beta, pool, asl, idx, g, gk, nat = args
    return lib.gdr_decode(ctypes.byref(d), q, k, v, beta, pool, asl, idx, g, gk, nat,
                          ctypes.c_float(1.0), ctypes.c_void_p(ptr + misalign), None)


GOOD = (2, 2, 4, 4, 64, 64, 2)  # B, T, H_qk, H_v, D_k, D_v, pool (layout 0)


@no_device
@pytest.mark.parametrize("dims,status", [
    ((2, 0, 4, 4, 64, 64, 2), GDR_ERR_DIMS),      # T < 1
    ((2, 9, 4, 4, 64, 64, 2), GDR_ERR_DIMS),      # T > 8: decode only
    ((2, 2, 3, 4, 64, 64, 2), GDR_ERR_DIMS),      # H_v not a multiple of H_qk
    ((2, 2, 0, 4, 64, 64, 2), GDR_ERR_DIMS),
    ((2, 2, 4, 4, 64, 64, 0), GDR_ERR_DIMS),      # empty pool
    ((-1, 2, 4, 4, 64, 64, 2), GDR_ERR_DIMS),
    ((2, 2, 4, 4, 96, 64, 2), GDR_ERR_UNSUPPORTED),  # D_k not 64/128
    ((2, 2, 4, 4, 64, 96, 2), GDR_ERR_UNSUPPORTED),  # D_v not a multiple of 64
    ((2**30, 1, 1, 64, 64, 512, 2), GDR_ERR_DIMS),    # grid overflow
    ((2, 2, 4, 4, 64, 64, 2, 2), GDR_ERR_DIMS),      # unknown state layout
    ((2, 2, 4, 4, 64, 64, 2, -1), GDR_ERR_DIMS),
])
def test_bad_sizes_rejected(built_library, dims, status):
    from gated_delta_rule_recurrent_b200 import binding

    L = binding.lib()
    assert _call_decode(L, dims) == status
    assert L.gdr_last_error().decode() != ""


@no_device
def test_null_and_misaligned_rejected(built_library):
    from gated_delta_rule_recurrent_b200 import binding

    L = binding.lib()
    assert L.gdr_decode(None, *([None] * 10), ctypes.c_float(1.0), None, None) == GDR_ERR_NULL
    for i in range(9):  # every tensor argument except num_accepted_tokens is required
        assert _call_decode(L, GOOD, nulls=(i,)) == GDR_ERR_NULL, i
    assert _call_decode(L, GOOD, misalign=8) == GDR_ERR_ALIGN
    assert "aligned" in L.gdr_last_error().decode()


@no_device
def test_empty_batch_is_a_no_op(built_library):
    from gated_delta_rule_recurrent_b200 import binding

    L = binding.lib()
    assert _call_decode(L, (0, 2, 4, 4, 64, 64, 2), ptr=0, nulls=tuple(range(10))) == GDR_OK


@no_device
def test_gate_fused_checks(built_library):
    from gated_delta_rule_recurrent_b200.binding import Dims, lib

    L = lib()
    d = Dims(*GOOD)
    p = ctypes.c_void_p(16)
    # a missing gate input
    rc = L.gdr_gate_fused(ctypes.byref(d), p, p, p, None, p, p, p, p, p, p, p, None,
                          ctypes.c_float(1.0), p, None)
    assert rc == GDR_ERR_NULL
    bad = Dims(2, 9, 4, 4, 64, 64, 2)
    rc = L.gdr_gate_fused(ctypes.byref(bad), p, p, p, p, p, p, p, p, p, p, p, None,
                          ctypes.c_float(1.0), p, None)
    assert rc == GDR_ERR_DIMS


def test_binding_refuses_cpu_tensors(built_library):
    from gated_delta_rule_recurrent_b200 import decode, workloads

    x = workloads.make_inputs(0)
    with pytest.raises(RuntimeError, match="CUDA"):
        decode(x["query"], x["key"], x["value"], x["beta"], x["state_pool"],
               x["actual_seq_lengths"], x["ssm_state_indices"], x["g"], x["gk"],
               x["num_accepted_tokens"], x["scale_value"])


@no_device
@pytest.mark.parametrize("args,status", [
    (dict(a=None), GDR_ERR_NULL),
    (dict(dt_bias=None), GDR_ERR_NULL),
    (dict(decay_scale=None), GDR_ERR_NULL),
    (dict(decay=None), GDR_ERR_NULL),
    (dict(b=None), GDR_ERR_NULL),            # beta requested without b (the gate page's rule)
    (dict(rows=-1), GDR_ERR_DIMS),
    (dict(H=0), GDR_ERR_DIMS),
    (dict(rows=1 << 60, H=8), GDR_ERR_DIMS),  # rows * H >= 2^62
    (dict(dtype=3), GDR_ERR_UNSUPPORTED),
    (dict(rows=0), GDR_OK),                  # nothing queued
])
def test_gate_host_checks(built_library, args, status):
    """The standalone gate's argument checks, with placeholder pointers."""
    from gated_delta_rule_recurrent_b200 import binding

    L = binding.lib()
    P = ctypes.c_void_p
    kw = dict(a=P(16), b=P(16), dt_bias=P(16), decay_scale=P(16), decay=P(16), beta=P(16),
              rows=4, H=8, dtype=2)
    kw.update(args)
    rc = L.gdr_linear_attention_gate(kw["a"], kw["b"], kw["dt_bias"], kw["decay_scale"],
                                     kw["decay"], kw["beta"], kw["rows"], kw["H"], kw["dtype"],
                                     None)
    assert rc == status, L.gdr_last_error().decode()


@no_device
def test_gate_without_beta_accepts_missing_b(built_library):
    """b may be absent when beta is not requested (checked without a device:
    rows = 0 queues nothing)."""
    from gated_delta_rule_recurrent_b200 import binding

    L = binding.lib()
    P = ctypes.c_void_p
    assert L.gdr_linear_attention_gate(P(16), None, P(16), P(16), P(16), None, 0, 8, 0, None) == 0
