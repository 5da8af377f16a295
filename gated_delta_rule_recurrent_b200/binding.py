"""ctypes binding of libgdr: torch tensors in, C-ABI calls out.

Only argument marshalling happens here: shape/dtype/device checks (raising
RuntimeError as the op's page specifies in section 异常 of
"lite_boost.ops.recurrent_gated_delta_rule"), the sizes struct, raw device
pointers and the current CUDA stream. Every step of the computation runs in
the library's kernels. Loading fails loudly when libgdr.so is missing; there
is no fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

__all__ = ["decode", "decode_gated", "prefill", "prefill_gated", "linear_attention_gate",
           "device_error", "GdrError", "lib",
           "library_path", "last_launch", "kernel_forms", "KERNEL_NAMES",
           "STATUS_NAMES", "Dims", "LaunchInfo"]

_PKG_DIR = os.path.dirname(os.path.abspath(__file__))

STATUS_NAMES = {0: "GDR_OK", 1: "GDR_ERR_NULL", 2: "GDR_ERR_DIMS", 3: "GDR_ERR_ALIGN",
                4: "GDR_ERR_UNSUPPORTED", 5: "GDR_ERR_CUDA"}


class GdrError(RuntimeError):
    """A libgdr entry point returned a nonzero status."""

    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class Dims(ctypes.Structure):
    """gdr_dims; ``layout`` is 0 (GDR_LAYOUT_KV) unless given."""
    _fields_ = [(n, ctypes.c_int32)
                for n in ("B", "T", "H_qk", "H_v", "D_k", "D_v", "pool_size", "layout")]


class LaunchInfo(ctypes.Structure):
    """gdr_launch_info: one kernel launch (or one kernel form of the dispatcher)."""
    _fields_ = [(n, ctypes.c_int32) for n in ("kernel", "D_k", "tile_cols", "gated", "layout",
                                              "grid", "threads", "smem_bytes", "stages")]

    def as_dict(self) -> dict:
        d = {n: int(getattr(self, n)) for n, _ in self._fields_}
        d["kernel"] = KERNEL_NAMES.get(d["kernel"], d["kernel"])
        d["layout"] = "vk" if d["layout"] == 1 else "kv"
        d["gated"] = bool(d["gated"])
        return d


# gdr_kernel values of include/gdr.h
KERNEL_NAMES = {0: "none", 1: "single_token", 2: "chunked", 3: "tensor_core",
                4: "tensor_core_one", 5: "gate", 6: "prefill", 7: "rows"}

_P = ctypes.c_void_p
_DECODE_ARGTYPES = [ctypes.POINTER(Dims), _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                    ctypes.c_float, _P, _P]
_GATED_ARGTYPES = [ctypes.POINTER(Dims), _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                   ctypes.c_float, _P, _P]

_lib = None


def library_path() -> str:
    return os.environ.get("GDR_LIBRARY", os.path.join(_PKG_DIR, "libgdr.so"))


def lib() -> ctypes.CDLL:
    """The loaded libgdr.so (loaded once; raises if it is missing)."""
    global _lib
    if _lib is None:
        path = library_path()
        if not os.path.exists(path):
            raise RuntimeError(
                f"libgdr.so not found at {path}; build it with "
                "`python -m gated_delta_rule_recurrent_b200.build`")
        L = ctypes.CDLL(path)
        L.gdr_decode.argtypes = _DECODE_ARGTYPES
        L.gdr_decode.restype = ctypes.c_int
        L.gdr_gate_fused.argtypes = _GATED_ARGTYPES
        L.gdr_gate_fused.restype = ctypes.c_int
        L.gdr_prefill.argtypes = _DECODE_ARGTYPES
        L.gdr_prefill.restype = ctypes.c_int
        L.gdr_prefill_gated.argtypes = _GATED_ARGTYPES
        L.gdr_prefill_gated.restype = ctypes.c_int
        L.gdr_status_string.argtypes = [ctypes.c_int]
        L.gdr_status_string.restype = ctypes.c_char_p
        L.gdr_last_error.argtypes = []
        L.gdr_last_error.restype = ctypes.c_char_p
        L.gdr_abi_version.argtypes = []
        L.gdr_abi_version.restype = ctypes.c_int
        L.gdr_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint32), ctypes.c_int]
        L.gdr_device_error.restype = ctypes.c_int
        P = ctypes.c_void_p
        L.gdr_linear_attention_gate.argtypes = [P, P, P, P, P, P, ctypes.c_int64, ctypes.c_int32,
                                                ctypes.c_int, P]
        L.gdr_linear_attention_gate.restype = ctypes.c_int
        L.gdr_last_launch.argtypes = [ctypes.POINTER(LaunchInfo)]
        L.gdr_last_launch.restype = ctypes.c_int
        L.gdr_kernel_form_count.argtypes = []
        L.gdr_kernel_form_count.restype = ctypes.c_int
        L.gdr_kernel_form.argtypes = [ctypes.c_int, ctypes.POINTER(LaunchInfo)]
        L.gdr_kernel_form.restype = ctypes.c_int
        _lib = L
    return _lib


def _check(rc: int) -> None:
    if rc != 0:
        raise GdrError(rc, lib().gdr_last_error().decode())


def device_error(reset: bool = True, device=None) -> int:
    """The device error word of ``device`` (bit 0: a consumer wait ran out of time,
    bit 1: a producer wait, bit 2: the final drain). Synchronises the device."""
    flags = ctypes.c_uint32(0)
    with torch.cuda.device(device if device is not None else torch.cuda.current_device()):
        rc = lib().gdr_device_error(ctypes.byref(flags), int(bool(reset)))
    _check(rc)
    return int(flags.value)


def last_launch() -> dict:
    """The calling thread's most recent kernel launch through the library
    (``gdr_last_launch``): kernel family, D_k, tile columns, gate, layout and
    the launch shape. ``kernel`` is "none" after a call that queued nothing."""
    info = LaunchInfo()
    _check(lib().gdr_last_launch(ctypes.byref(info)))
    return info.as_dict()


def kernel_forms() -> list:
    """Every decode kernel form the dispatcher can choose (``gdr_kernel_form``),
    as dicts with kernel, D_k, tile_cols, gated and layout. Needs no GPU."""
    L = lib()
    forms = []
    for i in range(L.gdr_kernel_form_count()):
        info = LaunchInfo()
        _check(L.gdr_kernel_form(i, ctypes.byref(info)))
        d = info.as_dict()
        forms.append({k: d[k] for k in ("kernel", "D_k", "tile_cols", "gated", "layout")})
    return forms


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, shape, device) -> None:
    if not isinstance(t, torch.Tensor):
        raise RuntimeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise RuntimeError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise RuntimeError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if t.device != device:
        raise RuntimeError(f"{name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise RuntimeError(f"{name} must be contiguous")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


# gdr_state_layout values of include/gdr.h
_LAYOUTS = {"kv": 0, "vk": 1}


def _common(query, key, value, state_pool, actual_seq_lengths, ssm_state_indices, gk,
            num_accepted_tokens, out, state_layout="kv"):
    if not isinstance(query, torch.Tensor) or query.dim() != 4:
        raise RuntimeError("query must be a 4-D tensor [B, H_qk, T, D_k]")
    device = query.device
    if device.type != "cuda":
        raise RuntimeError("all tensors must be on a CUDA device")
    B, H_qk, T, D_k = query.shape
    if not isinstance(value, torch.Tensor) or value.dim() != 4:
        raise RuntimeError("value must be a 4-D tensor [B, H_v, T, D_v]")
    H_v, D_v = value.shape[1], value.shape[3]
    if state_layout not in _LAYOUTS:
        raise RuntimeError('state_layout must be "kv" ([pool, H_v, D_k, D_v]) or "vk" '
                           '([pool, H_v, D_v, D_k])')
    if not isinstance(state_pool, torch.Tensor) or state_pool.dim() != 4:
        raise RuntimeError("state_pool must be a 4-D tensor [pool, H_v, D_k, D_v] "
                           "(or [pool, H_v, D_v, D_k] for state_layout='vk')")
    P = state_pool.shape[0]
    bf16, f32, i32 = torch.bfloat16, torch.float32, torch.int32
    _need(query, "query", bf16, (B, H_qk, T, D_k), device)
    _need(key, "key", bf16, (B, H_qk, T, D_k), device)
    _need(value, "value", bf16, (B, H_v, T, D_v), device)
    _need(state_pool, "state_pool", bf16,
          (P, H_v, D_k, D_v) if state_layout == "kv" else (P, H_v, D_v, D_k), device)
    _need(actual_seq_lengths, "actual_seq_lengths", i32, (B,), device)
    _need(ssm_state_indices, "ssm_state_indices", i32, (B,), device)
    _need(gk, "gk", f32, (B, H_v, T, D_k), device)
    if num_accepted_tokens is not None:
        _need(num_accepted_tokens, "num_accepted_tokens", i32, (B,), device)
    if out is None:
        out = torch.empty((B, H_v, T, D_v), dtype=bf16, device=device)
    else:
        _need(out, "out", bf16, (B, H_v, T, D_v), device)
    dims = Dims(B, T, H_qk, H_v, D_k, D_v, P, _LAYOUTS[state_layout])
    stream = ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)
    return device, dims, out, stream


def decode(query: torch.Tensor, key: torch.Tensor, value: torch.Tensor, beta: torch.Tensor,
           state_pool: torch.Tensor, actual_seq_lengths: torch.Tensor,
           ssm_state_indices: torch.Tensor, g: torch.Tensor, gk: torch.Tensor,
           num_accepted_tokens: Optional[torch.Tensor] = None, scale_value: float = 1.0, *,
           out: Optional[torch.Tensor] = None,
           state_layout: str = "kv") -> Tuple[torch.Tensor, torch.Tensor]:
    """recurrent_gated_delta_rule decode step through ``gdr_decode``.

    Argument order and defaults follow the op's page. ``state_pool`` is
    updated in place and returned as the second result (the page's
    ``state_out``). ``num_accepted_tokens`` (optional, [B] int32) is the
    number of leading tokens whose state update is committed: outputs of all
    valid tokens are computed, the slot keeps the state after the first n
    (unchanged for n = 0); None commits them all. ``state_layout`` "vk" takes
    the pool as [pool, H_v, D_v, D_k] (k contiguous) instead of the page's
    [pool, H_v, D_k, D_v]. Queued on the current CUDA stream; no
    synchronisation.
    """
    device, dims, out, stream = _common(query, key, value, state_pool, actual_seq_lengths,
                                        ssm_state_indices, gk, num_accepted_tokens, out,
                                        state_layout)
    B, H_v, T = dims.B, dims.H_v, dims.T
    _need(beta, "beta", torch.bfloat16, (B, H_v, T), device)
    _need(g, "g", torch.float32, (B, H_v, T), device)
    with torch.cuda.device(device):
        rc = lib().gdr_decode(ctypes.byref(dims), _ptr(query), _ptr(key), _ptr(value),
                              _ptr(beta), _ptr(state_pool), _ptr(actual_seq_lengths),
                              _ptr(ssm_state_indices), _ptr(g), _ptr(gk),
                              _ptr(num_accepted_tokens), float(scale_value), _ptr(out), stream)
    _check(rc)
    return out, state_pool


def decode_gated(query: torch.Tensor, key: torch.Tensor, value: torch.Tensor, a: torch.Tensor,
                 b: torch.Tensor, dt_bias: torch.Tensor, decay_scale: torch.Tensor,
                 state_pool: torch.Tensor, actual_seq_lengths: torch.Tensor,
                 ssm_state_indices: torch.Tensor, gk: torch.Tensor,
                 num_accepted_tokens: Optional[torch.Tensor] = None, scale_value: float = 1.0,
                 *, out: Optional[torch.Tensor] = None,
                 state_layout: str = "kv") -> Tuple[torch.Tensor, torch.Tensor]:
    """Decode step with the LinearAttentionGate prologue fused, through ``gdr_gate_fused``.

    ``a`` and ``b`` are [B, T, H_v] bf16; ``dt_bias`` and ``decay_scale`` are
    [H_v] fp32. g and beta are computed inside the kernel. ``state_layout`` as
    for ``decode``.
    """
    device, dims, out, stream = _common(query, key, value, state_pool, actual_seq_lengths,
                                        ssm_state_indices, gk, num_accepted_tokens, out,
                                        state_layout)
    B, H_v, T = dims.B, dims.H_v, dims.T
    _need(a, "a", torch.bfloat16, (B, T, H_v), device)
    _need(b, "b", torch.bfloat16, (B, T, H_v), device)
    _need(dt_bias, "dt_bias", torch.float32, (H_v,), device)
    _need(decay_scale, "decay_scale", torch.float32, (H_v,), device)
    with torch.cuda.device(device):
        rc = lib().gdr_gate_fused(ctypes.byref(dims), _ptr(query), _ptr(key), _ptr(value),
                                  _ptr(a), _ptr(b), _ptr(dt_bias), _ptr(decay_scale),
                                  _ptr(state_pool), _ptr(actual_seq_lengths),
                                  _ptr(ssm_state_indices), _ptr(gk),
                                  _ptr(num_accepted_tokens), float(scale_value), _ptr(out),
                                  stream)
    _check(rc)
    return out, state_pool


def prefill(query: torch.Tensor, key: torch.Tensor, value: torch.Tensor, beta: torch.Tensor,
            state_pool: torch.Tensor, actual_seq_lengths: torch.Tensor,
            ssm_state_indices: torch.Tensor, g: torch.Tensor, gk: torch.Tensor,
            num_accepted_tokens: Optional[torch.Tensor] = None, scale_value: float = 1.0, *,
            out: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """The recurrence over a long prompt through ``gdr_prefill``: the arguments
    and results of ``decode`` for any token count T (D_k = 128, D_v a multiple
    of 128, the [pool, H_v, D_k, D_v] pool)."""
    device, dims, out, stream = _common(query, key, value, state_pool, actual_seq_lengths,
                                        ssm_state_indices, gk, num_accepted_tokens, out, "kv")
    B, H_v, T = dims.B, dims.H_v, dims.T
    _need(beta, "beta", torch.bfloat16, (B, H_v, T), device)
    _need(g, "g", torch.float32, (B, H_v, T), device)
    with torch.cuda.device(device):
        rc = lib().gdr_prefill(ctypes.byref(dims), _ptr(query), _ptr(key), _ptr(value),
                               _ptr(beta), _ptr(state_pool), _ptr(actual_seq_lengths),
                               _ptr(ssm_state_indices), _ptr(g), _ptr(gk),
                               _ptr(num_accepted_tokens), float(scale_value), _ptr(out), stream)
    _check(rc)
    return out, state_pool


def prefill_gated(query: torch.Tensor, key: torch.Tensor, value: torch.Tensor, a: torch.Tensor,
                  b: torch.Tensor, dt_bias: torch.Tensor, decay_scale: torch.Tensor,
                  state_pool: torch.Tensor, actual_seq_lengths: torch.Tensor,
                  ssm_state_indices: torch.Tensor, gk: torch.Tensor,
                  num_accepted_tokens: Optional[torch.Tensor] = None, scale_value: float = 1.0,
                  *, out: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """``prefill`` with the LinearAttentionGate fused, through ``gdr_prefill_gated``
    (the gate arguments of ``decode_gated``)."""
    device, dims, out, stream = _common(query, key, value, state_pool, actual_seq_lengths,
                                        ssm_state_indices, gk, num_accepted_tokens, out, "kv")
    B, H_v, T = dims.B, dims.H_v, dims.T
    _need(a, "a", torch.bfloat16, (B, T, H_v), device)
    _need(b, "b", torch.bfloat16, (B, T, H_v), device)
    _need(dt_bias, "dt_bias", torch.float32, (H_v,), device)
    _need(decay_scale, "decay_scale", torch.float32, (H_v,), device)
    with torch.cuda.device(device):
        rc = lib().gdr_prefill_gated(ctypes.byref(dims), _ptr(query), _ptr(key), _ptr(value),
                                     _ptr(a), _ptr(b), _ptr(dt_bias), _ptr(decay_scale),
                                     _ptr(state_pool), _ptr(actual_seq_lengths),
                                     _ptr(ssm_state_indices), _ptr(gk),
                                     _ptr(num_accepted_tokens), float(scale_value), _ptr(out),
                                     stream)
    _check(rc)
    return out, state_pool


# gdr_dtype values of include/gdr.h
_GATE_DTYPES = {torch.float32: 0, torch.float16: 1, torch.bfloat16: 2}


def linear_attention_gate(a: torch.Tensor, dt_bias: torch.Tensor, decay_scale: torch.Tensor,
                          b: Optional[torch.Tensor] = None, want_beta: Optional[bool] = None,
                          decay: Optional[torch.Tensor] = None,
                          beta: Optional[torch.Tensor] = None):
    """The LinearAttentionGate op on its own ("com.microsoft.LinearAttentionGate").

    decay = decay_scale * softplus(a + dt_bias) and, when requested, beta =
    sigmoid(b), computed in float32 and narrowed to a's dtype (float32, float16
    or bfloat16). The head axis is the last axis of ``a``; dt_bias and
    decay_scale are float32 [H]. ``want_beta`` defaults to ``b is not None``;
    requesting beta without b is an error (the page's rule), while a b given
    with want_beta=False is accepted and not read. Returns (decay, beta or None).
    """
    if not isinstance(a, torch.Tensor) or a.dim() < 1:
        raise RuntimeError("a must be a tensor of rank >= 1 (heads on the last axis)")
    device = a.device
    if device.type != "cuda":
        raise RuntimeError("all tensors must be on a CUDA device")
    if a.dtype not in _GATE_DTYPES:
        raise RuntimeError(f"a must be float32, float16 or bfloat16, got {a.dtype}")
    if want_beta is None:
        want_beta = b is not None
    if want_beta and b is None:
        raise RuntimeError("beta was requested but b is None")
    H = a.shape[-1]
    _need(a, "a", a.dtype, a.shape, device)
    _need(dt_bias, "dt_bias", torch.float32, (H,), device)
    _need(decay_scale, "decay_scale", torch.float32, (H,), device)
    if b is not None:
        _need(b, "b", a.dtype, a.shape, device)
    if decay is None:
        decay = torch.empty_like(a)
    _need(decay, "decay", a.dtype, a.shape, device)
    if want_beta:
        if beta is None:
            beta = torch.empty_like(a)
        _need(beta, "beta", a.dtype, a.shape, device)
    else:
        beta = None
    rows = a.numel() // H if H > 0 else 0
    stream = torch.cuda.current_stream(device).cuda_stream
    with torch.cuda.device(device):
        rc = lib().gdr_linear_attention_gate(
            _ptr(a), _ptr(b if want_beta else None), _ptr(dt_bias), _ptr(decay_scale),
            _ptr(decay), _ptr(beta), rows, H, _GATE_DTYPES[a.dtype], ctypes.c_void_p(stream))
    _check(rc)
    return decay, beta
