"""Python binding of libswitchlayer.so, the sm_100a Switch-layer forward pass.

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  PyTorch supplies device memory (tensors) and the current stream.
There is no fallback: if the shared library is missing or cannot be loaded,
every call raises.

The C entry points are exposed under their C names (``switch_layer_forward``,
``switch_layer_capacity`` ...); ``forward`` is a convenience wrapper that
allocates the outputs and the workspace with torch and calls
``switch_layer_forward``.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# SWL_LIBRARY=checked loads the range-checked build (see build.py)
LIB_PATH = os.path.join(_HERE, "libswitchlayer_checked.so"
                        if os.environ.get("SWL_LIBRARY", "") == "checked"
                        else "libswitchlayer.so")

SWL_F32, SWL_BF16 = 0, 1
SWL_WS_HOST_IO = 1
SWL_WS_TOP2 = 2
SWL_WS_NTLB = 4
SWL_NUM_STAGES = 5
STATUS = {0: "SWL_OK", 1: "SWL_ERR_INVALID_ARG", 2: "SWL_ERR_UNSUPPORTED",
          3: "SWL_ERR_WORKSPACE", 4: "SWL_ERR_CUDA", 5: "SWL_ERR_DEVICE"}

# Every symbol declared in include/switch_layer.h.
EXPORTS = ("switch_layer_capacity", "switch_layer_workspace_size", "switch_layer_forward",
           "switch_layer_forward_timed", "switch_layer_forward_host_io",
           "switch_layer_device_status", "switch_layer_status_string",
           "switch_layer_stage_name", "switch_layer_launch_count",
           "switch_layer_forward_noalloc", "switch_layer_set_router_mode",
           "switch_layer_router_mode", "switch_layer_describe_plan",
           "switch_layer_noalloc_status", "switch_layer_shard_record_bytes",
           "switch_layer_forward_shard_begin", "switch_layer_forward_shard_end",
           "switch_layer_set_wait_limit_ns", "switch_layer_set_stall_test",
           "switch_layer_forward_top2", "switch_layer_forward_ntlb", "switch_layer_ep_max_recv_rows",
           "switch_layer_ep_workspace_size", "switch_layer_ep_counts",
           "switch_layer_ep_dispatch", "switch_layer_ep_experts", "switch_layer_ep_combine",
           "switch_layer_variant_workspace_size", "switch_layer_forward_variant",
           "switch_layer_backward_workspace_size", "switch_layer_backward")
SWL_ACT_RELU, SWL_ACT_GEGLU = 0, 1


class Variant(ctypes.Structure):
    """struct swl_variant of include/switch_layer.h."""
    _fields_ = [("top_k", ctypes.c_int), ("normalize", ctypes.c_int),
                ("activation", ctypes.c_int), ("router_noise", ctypes.c_void_p)]
SWL_ROUTER_TENSOR = 0
SWL_ROUTER_FFMA = 1
SWL_NOALLOC_MAX_BYTES = 64 << 20


class SwitchLayerError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__("%s (%s)%s" % (STATUS.get(status, "status %d" % status),
                                        _status_string(status),
                                        (": " + what) if what else ""))


_lib: Optional[ctypes.CDLL] = None

_i64, _i32, _dbl, _vp, _sz = (ctypes.c_int64, ctypes.c_int, ctypes.c_double, ctypes.c_void_p,
                              ctypes.c_size_t)
_FWD_ARGS = [_i64, _i64, _i64, _i64, _i32,            # T, d, d_ff, N, dtype
             _vp, _vp, _vp, _vp, _vp, _vp, _dbl,       # x, W_r, W1, b1, W2, b2, cf
             _vp, _vp, _vp, _vp, _vp,                  # out, expert_idx, gate, pos, aux
             _vp, _vp, _sz, _vp]                       # b_r, workspace, bytes, stream


def lib() -> ctypes.CDLL:
    """Load libswitchlayer.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError("%s is missing: build it with "
                           "`python -m sparse_mixture_experts_argmax_b200.build`"
                           % os.path.basename(LIB_PATH))
    L = ctypes.CDLL(LIB_PATH)
    L.switch_layer_capacity.restype = _i64
    L.switch_layer_capacity.argtypes = [_i64, _i64, _dbl]
    L.switch_layer_workspace_size.restype = _i32
    L.switch_layer_workspace_size.argtypes = [_i64, _i64, _i64, _i64, _i32, _dbl, _i32,
                                              ctypes.POINTER(_sz)]
    L.switch_layer_forward.restype = _i32
    L.switch_layer_forward.argtypes = _FWD_ARGS
    L.switch_layer_forward_timed.restype = _i32
    L.switch_layer_forward_timed.argtypes = _FWD_ARGS + [ctypes.POINTER(_vp)]
    L.switch_layer_forward_host_io.restype = _i32
    L.switch_layer_forward_host_io.argtypes = _FWD_ARGS
    L.switch_layer_device_status.restype = _i32
    L.switch_layer_device_status.argtypes = [_vp, _vp]
    L.switch_layer_status_string.restype = ctypes.c_char_p
    L.switch_layer_status_string.argtypes = [_i32]
    L.switch_layer_stage_name.restype = ctypes.c_char_p
    L.switch_layer_stage_name.argtypes = [_i32]
    L.switch_layer_launch_count.restype = ctypes.c_uint64
    L.switch_layer_launch_count.argtypes = []
    L.switch_layer_set_router_mode.restype = ctypes.c_int
    L.switch_layer_set_router_mode.argtypes = [_i32]
    L.switch_layer_router_mode.restype = ctypes.c_int
    L.switch_layer_router_mode.argtypes = []
    L.switch_layer_describe_plan.restype = _i32
    L.switch_layer_describe_plan.argtypes = [_i64, _i64, _i64, _i64, _i32, _dbl, _i32,
                                             ctypes.c_char_p, _sz]
    L.switch_layer_forward_noalloc.restype = _i32
    L.switch_layer_forward_noalloc.argtypes = _FWD_ARGS[:17] + [_vp, _vp]
    L.switch_layer_noalloc_status.restype = _i32
    L.switch_layer_noalloc_status.argtypes = [_vp]
    L.switch_layer_ep_max_recv_rows.restype = _i64
    L.switch_layer_ep_max_recv_rows.argtypes = [_i64, _i32, _i64, _dbl]
    L.switch_layer_ep_workspace_size.restype = _i32
    L.switch_layer_ep_workspace_size.argtypes = [_i64, _i64, _i64, _i64, _i32, _i32, _i64, _dbl,
                                                 ctypes.POINTER(_sz)]
    L.switch_layer_ep_counts.restype = _i32
    L.switch_layer_ep_counts.argtypes = [_i64, _i32, _i32, _i64, _dbl, _vp,
                                         ctypes.POINTER(_i64), ctypes.POINTER(_i64)]
    L.switch_layer_ep_dispatch.restype = _i32
    L.switch_layer_ep_dispatch.argtypes = [_i64, _i64, _i64, _i64, _i32, _i32, _i32, _i64, _dbl,
                                           _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
    L.switch_layer_ep_experts.restype = _i32
    L.switch_layer_ep_experts.argtypes = [_i64, _i64, _i64, _i64, _i32, _i32, _i32, _i64, _dbl,
                                          _vp, _vp, _i64, _vp, _vp, _vp, _vp, _vp, _vp, _sz,
                                          _vp]
    L.switch_layer_ep_combine.restype = _i32
    L.switch_layer_ep_combine.argtypes = [_i64, _i64, _i64, _i64, _i32, _i32, _i32, _i64, _dbl,
                                          _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
    L.switch_layer_backward_workspace_size.restype = _i32
    L.switch_layer_backward_workspace_size.argtypes = [_i64, _i64, _i64, _i64, _i32, _dbl,
                                                       ctypes.POINTER(_sz)]
    L.switch_layer_backward.restype = _i32
    L.switch_layer_backward.argtypes = ([_i64, _i64, _i64, _i64, _i32] + [_vp] * 7 + [_dbl] +
                                        [_vp] * 5 + [_sz, _vp, ctypes.c_float] + [_vp] * 8 +
                                        [_sz, _vp])
    L.switch_layer_variant_workspace_size.restype = _i32
    L.switch_layer_variant_workspace_size.argtypes = [_i64, _i64, _i64, _i64, _i32, _dbl,
                                                      ctypes.POINTER(Variant),
                                                      ctypes.POINTER(_sz)]
    L.switch_layer_forward_variant.restype = _i32
    L.switch_layer_forward_variant.argtypes = (_FWD_ARGS[:18] + [ctypes.POINTER(Variant)] +
                                               _FWD_ARGS[18:])
    L.switch_layer_forward_top2.restype = _i32
    L.switch_layer_forward_top2.argtypes = _FWD_ARGS[:12] + [_i32] + _FWD_ARGS[12:]
    L.switch_layer_forward_ntlb.restype = _i32
    L.switch_layer_forward_ntlb.argtypes = _FWD_ARGS
    L.switch_layer_set_wait_limit_ns.restype = _i32
    L.switch_layer_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    L.switch_layer_set_stall_test.restype = _i32
    L.switch_layer_set_stall_test.argtypes = [_i32]
    L.switch_layer_shard_record_bytes.restype = _sz
    L.switch_layer_shard_record_bytes.argtypes = [_i64]
    L.switch_layer_forward_shard_begin.restype = _i32
    L.switch_layer_forward_shard_begin.argtypes = [_i64, _i64, _i64, _i64, _i32, _i64,
                                                   _vp, _vp, _vp, _dbl, _vp, _vp, _vp, _vp,
                                                   _vp, _sz, _vp]
    L.switch_layer_forward_shard_end.restype = _i32
    L.switch_layer_forward_shard_end.argtypes = [_i64, _i64, _i64, _i64, _i32, _i64, _i32,
                                                 _i32, _vp, _vp, _vp, _vp, _vp, _vp, _dbl,
                                                 _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]
    _lib = L
    return L


def _status_string(status: int) -> str:
    try:
        return lib().switch_layer_status_string(status).decode()
    except Exception:  # pragma: no cover - only while reporting another failure
        return "?"


def _check(status: int, what: str = "") -> None:
    if status != 0:
        raise SwitchLayerError(status, what)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream_handle(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def dtype_code(dt: torch.dtype) -> int:
    if dt == torch.float32:
        return SWL_F32
    if dt == torch.bfloat16:
        return SWL_BF16
    raise TypeError("activation dtype must be float32 or bfloat16, got %s" % dt)


# ---------------------------------------------------------------------------
# C entry points, same names
# ---------------------------------------------------------------------------
def switch_layer_capacity(T: int, N: int, capacity_factor: float) -> int:
    return int(lib().switch_layer_capacity(T, N, capacity_factor))


def switch_layer_workspace_size(T, d, d_ff, N, dtype: int, capacity_factor: float,
                                flags: int = 0) -> int:
    n = _sz(0)
    _check(lib().switch_layer_workspace_size(T, d, d_ff, N, dtype, capacity_factor, flags,
                                             ctypes.byref(n)), "workspace_size")
    return int(n.value)


def _shape_of(x, W1, W_r):
    T, d = x.shape
    N, d_ff, d2 = W1.shape
    if d2 != d or tuple(W_r.shape) != (N, d):
        raise ValueError("shape mismatch: x %s, W_r %s, W1 %s" % (tuple(x.shape),
                                                                  tuple(W_r.shape),
                                                                  tuple(W1.shape)))
    return T, d, d_ff, N


def _require(t: torch.Tensor, name: str, dtype=None, device="cuda"):
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch.Tensor" % name)
    if device == "cuda" and not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if device == "cpu" and t.is_cuda:
        raise ValueError("%s must be a host tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if dtype is not None and t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))


def switch_layer_forward(x, W_r, W1, b1, W2, b2, capacity_factor, out, expert_idx, gate,
                         pos_in_expert, aux_loss, b_r=None, workspace=None, stream=None,
                         stage_events: Optional[Sequence] = None) -> None:
    """Enqueue one forward pass (all tensors on the GPU; see include/switch_layer.h)."""
    T, d, d_ff, N = _shape_of(x, W1, W_r)
    act = x.dtype
    for t, n in ((x, "x"), (W1, "W1"), (b1, "b1"), (W2, "W2"), (b2, "b2"), (out, "out")):
        _require(t, n, act)
    _require(W_r, "W_r", torch.float32)
    if b_r is not None:
        _require(b_r, "b_r", torch.float32)
    _require(expert_idx, "expert_idx", torch.int32)
    _require(pos_in_expert, "pos_in_expert", torch.int32)
    _require(gate, "gate", torch.float32)
    _require(aux_loss, "aux_loss", torch.float32)
    _require(workspace, "workspace", torch.uint8)
    args = (T, d, d_ff, N, dtype_code(act), _ptr(x), _ptr(W_r), _ptr(W1), _ptr(b1), _ptr(W2),
            _ptr(b2), float(capacity_factor), _ptr(out), _ptr(expert_idx), _ptr(gate),
            _ptr(pos_in_expert), _ptr(aux_loss), _ptr(b_r), _ptr(workspace),
            workspace.numel(), _stream_handle(stream))
    if stage_events is None:
        _check(lib().switch_layer_forward(*args), "forward")
    else:
        if len(stage_events) != SWL_NUM_STAGES + 1:
            raise ValueError("need %d stage events" % (SWL_NUM_STAGES + 1))
        for e in stage_events:          # torch creates the CUDA event on first record
            if not e.cuda_event:
                e.record()
        evs = (_vp * (SWL_NUM_STAGES + 1))(*[ctypes.c_void_p(int(e.cuda_event))
                                             for e in stage_events])
        _check(lib().switch_layer_forward_timed(*args, evs), "forward_timed")


def switch_layer_forward_top2(x, W_r, W1, b1, W2, b2, capacity_factor, normalize, out,
                              expert_idx, gate, pos_in_expert, aux_loss, b_r=None,
                              workspace=None, stream=None) -> None:
    """Enqueue one forward pass of the top-2 variant (expert_idx, gate,
    pos_in_expert are [T, 2]; workspace sized with SWL_WS_TOP2)."""
    T, d, d_ff, N = _shape_of(x, W1, W_r)
    act = x.dtype
    for t, n in ((x, "x"), (W1, "W1"), (b1, "b1"), (W2, "W2"), (b2, "b2"), (out, "out")):
        _require(t, n, act)
    _require(W_r, "W_r", torch.float32)
    if b_r is not None:
        _require(b_r, "b_r", torch.float32)
    for t, n, dt in ((expert_idx, "expert_idx", torch.int32), (gate, "gate", torch.float32),
                     (pos_in_expert, "pos_in_expert", torch.int32)):
        _require(t, n, dt)
        if t.numel() != 2 * T:
            raise ValueError("%s must hold [T, 2] values" % n)
    _require(aux_loss, "aux_loss", torch.float32)
    _require(workspace, "workspace", torch.uint8)
    _check(lib().switch_layer_forward_top2(
        T, d, d_ff, N, dtype_code(act), _ptr(x), _ptr(W_r), _ptr(W1), _ptr(b1), _ptr(W2),
        _ptr(b2), float(capacity_factor), 1 if normalize else 0, _ptr(out), _ptr(expert_idx),
        _ptr(gate), _ptr(pos_in_expert), _ptr(aux_loss), _ptr(b_r), _ptr(workspace),
        workspace.numel(), _stream_handle(stream)), "forward_top2")


def switch_layer_forward_ntlb(x, W_r, W1, b1, W2, b2, capacity_factor, out, expert_idx, gate,
                              pos_in_expert, aux_loss, b_r=None, workspace=None,
                              stream=None) -> None:
    """Enqueue one forward pass of the No-Token-Left-Behind variant (expert_idx,
    gate, pos_in_expert are [T, 2]; workspace sized with SWL_WS_NTLB)."""
    T, d, d_ff, N = _shape_of(x, W1, W_r)
    act = x.dtype
    for t, n in ((x, "x"), (W1, "W1"), (b1, "b1"), (W2, "W2"), (b2, "b2"), (out, "out")):
        _require(t, n, act)
    _require(W_r, "W_r", torch.float32)
    if b_r is not None:
        _require(b_r, "b_r", torch.float32)
    for t, n, dt in ((expert_idx, "expert_idx", torch.int32), (gate, "gate", torch.float32),
                     (pos_in_expert, "pos_in_expert", torch.int32)):
        _require(t, n, dt)
        if t.numel() != 2 * T:
            raise ValueError("%s must hold [T, 2] values" % n)
    _require(aux_loss, "aux_loss", torch.float32)
    _require(workspace, "workspace", torch.uint8)
    _check(lib().switch_layer_forward_ntlb(
        T, d, d_ff, N, dtype_code(act), _ptr(x), _ptr(W_r), _ptr(W1), _ptr(b1), _ptr(W2),
        _ptr(b2), float(capacity_factor), _ptr(out), _ptr(expert_idx), _ptr(gate),
        _ptr(pos_in_expert), _ptr(aux_loss), _ptr(b_r), _ptr(workspace), workspace.numel(),
        _stream_handle(stream)), "forward_ntlb")


def switch_layer_forward_host_io(x_host, W_r, W1, b1, W2, b2, capacity_factor, out_host,
                                 expert_idx_host, gate_host, pos_host, aux_host, b_r=None,
                                 workspace=None, stream=None) -> None:
    """Enqueue H2D(x) -> forward -> D2H(outputs); host tensors should be pinned."""
    T, d, d_ff, N = _shape_of(x_host, W1, W_r)
    act = x_host.dtype
    _require(x_host, "x_host", act, device="cpu")
    _require(out_host, "out_host", act, device="cpu")
    for t, n in ((W1, "W1"), (b1, "b1"), (W2, "W2"), (b2, "b2")):
        _require(t, n, act)
    _require(W_r, "W_r", torch.float32)
    _require(expert_idx_host, "expert_idx_host", torch.int32, device="cpu")
    _require(pos_host, "pos_host", torch.int32, device="cpu")
    _require(gate_host, "gate_host", torch.float32, device="cpu")
    _require(aux_host, "aux_host", torch.float32, device="cpu")
    _require(workspace, "workspace", torch.uint8)
    _check(lib().switch_layer_forward_host_io(
        T, d, d_ff, N, dtype_code(act), _ptr(x_host), _ptr(W_r), _ptr(W1), _ptr(b1), _ptr(W2),
        _ptr(b2), float(capacity_factor), _ptr(out_host), _ptr(expert_idx_host),
        _ptr(gate_host), _ptr(pos_host), _ptr(aux_host), _ptr(b_r), _ptr(workspace),
        workspace.numel(), _stream_handle(stream)), "forward_host_io")


def switch_layer_device_status(workspace: torch.Tensor, stream=None) -> int:
    return int(lib().switch_layer_device_status(_ptr(workspace), _stream_handle(stream)))


def switch_layer_status_string(status: int) -> str:
    return _status_string(status)


def switch_layer_stage_name(k: int) -> Optional[str]:
    r = lib().switch_layer_stage_name(k)
    return None if r is None else r.decode()


def switch_layer_launch_count() -> int:
    return int(lib().switch_layer_launch_count())


def switch_layer_set_router_mode(mode: int) -> None:
    """SWL_ROUTER_TENSOR (default) or SWL_ROUTER_FFMA for bf16 layers (process-wide)."""
    _check(lib().switch_layer_set_router_mode(int(mode)), "switch_layer_set_router_mode")


def switch_layer_router_mode() -> int:
    return int(lib().switch_layer_router_mode())


def switch_layer_describe_plan(T, d, d_ff, N, dtype: int, capacity_factor: float,
                               num_sms: int = 148) -> dict:
    """The kernels a forward call of this shape would launch (host-only), as a dict
    of the C entry point's key=value pairs (integers converted)."""
    buf = ctypes.create_string_buffer(256)
    _check(lib().switch_layer_describe_plan(T, d, d_ff, N, dtype, capacity_factor, num_sms,
                                            buf, len(buf)), "describe_plan")
    out = {}
    for kv in buf.value.decode().split(","):
        k, v = kv.split("=", 1)
        out[k] = int(v) if v.lstrip("-").isdigit() else v
    return out


def switch_layer_set_wait_limit_ns(ns: int) -> None:
    """Failure-path test hook: bound of every wait inside the kernels (0: 2 s)."""
    _check(lib().switch_layer_set_wait_limit_ns(int(ns)), "set_wait_limit_ns")


def switch_layer_set_stall_test(on: bool) -> None:
    """Failure-path test hook: make the expert FFN's first GEMM2 wait run out."""
    _check(lib().switch_layer_set_stall_test(1 if on else 0), "set_stall_test")


def switch_layer_ep_max_recv_rows(N, world, T_total, capacity_factor) -> int:
    return int(lib().switch_layer_ep_max_recv_rows(N, world, T_total, capacity_factor))


def switch_layer_ep_workspace_size(T, d, d_ff, N, dtype, world, T_total, capacity_factor) -> int:
    n = _sz(0)
    _check(lib().switch_layer_ep_workspace_size(T, d, d_ff, N, dtype, world, T_total,
                                                capacity_factor, ctypes.byref(n)),
           "ep_workspace_size")
    return int(n.value)


def switch_layer_ep_counts(N, world, rank, T_total, capacity_factor, gathered_host):
    """(send rows per peer, receive rows per peer) from a host copy of the records."""
    _require(gathered_host, "gathered_host", torch.uint8, device="cpu")
    send = (_i64 * world)()
    recv = (_i64 * world)()
    _check(lib().switch_layer_ep_counts(N, world, rank, int(T_total), float(capacity_factor),
                                        _ptr(gathered_host), send, recv), "ep_counts")
    return [int(v) for v in send], [int(v) for v in recv]


def switch_layer_ep_dispatch(x, d_ff, N, world, rank, T_total, capacity_factor, gathered,
                             expert_idx, pos_in_expert, aux_loss, send_rows, workspace,
                             stream=None) -> None:
    T, d = x.shape
    _check(lib().switch_layer_ep_dispatch(
        T, d, d_ff, N, dtype_code(x.dtype), world, rank, int(T_total), float(capacity_factor),
        _ptr(gathered), _ptr(x), _ptr(expert_idx), _ptr(pos_in_expert), _ptr(aux_loss),
        _ptr(send_rows), _ptr(workspace), workspace.numel(), _stream_handle(stream)),
        "ep_dispatch")


def switch_layer_ep_experts(T, d, d_ff, N, act_dtype, world, rank, T_total, capacity_factor,
                            gathered, recv_rows, W1_local, b1_local, W2_local, b2_local, ret_rows,
                            workspace, stream=None) -> None:
    for t, n in ((W1_local, "W1_local"), (b1_local, "b1_local"), (W2_local, "W2_local"),
                 (b2_local, "b2_local")):
        _require(t, n, act_dtype)
    _check(lib().switch_layer_ep_experts(
        T, d, d_ff, N, dtype_code(act_dtype), world, rank, int(T_total), float(capacity_factor),
        _ptr(gathered), _ptr(recv_rows), recv_rows.shape[0], _ptr(W1_local), _ptr(b1_local),
        _ptr(W2_local), _ptr(b2_local), _ptr(ret_rows), _ptr(workspace), workspace.numel(),
        _stream_handle(stream)), "ep_experts")


def switch_layer_ep_combine(T, d, d_ff, N, act_dtype, world, rank, T_total, capacity_factor,
                            back_rows, expert_idx, gate, pos_in_expert, out, workspace,
                            stream=None) -> None:
    _check(lib().switch_layer_ep_combine(
        T, d, d_ff, N, dtype_code(act_dtype), world, rank, int(T_total), float(capacity_factor),
        _ptr(back_rows), _ptr(expert_idx), _ptr(gate), _ptr(pos_in_expert), _ptr(out),
        _ptr(workspace), workspace.numel(), _stream_handle(stream)), "ep_combine")


def switch_layer_shard_record_bytes(N: int) -> int:
    return int(lib().switch_layer_shard_record_bytes(N))


def switch_layer_forward_shard_begin(x, W_r, capacity_factor, T_total, expert_idx, gate,
                                     pos_in_expert, record, d_ff, b_r=None, workspace=None,
                                     stream=None) -> None:
    """Step 1 of a forward over one rank's token range of a global batch."""
    T, d = x.shape
    N = W_r.shape[0]
    _require(x, "x")
    _require(W_r, "W_r", torch.float32)
    if b_r is not None:
        _require(b_r, "b_r", torch.float32)
    _require(record, "record", torch.uint8)
    _require(workspace, "workspace", torch.uint8)
    if record.numel() != switch_layer_shard_record_bytes(N):
        raise ValueError("record must hold %d bytes" % switch_layer_shard_record_bytes(N))
    _check(lib().switch_layer_forward_shard_begin(
        T, d, d_ff, N, dtype_code(x.dtype), int(T_total), _ptr(x), _ptr(W_r), _ptr(b_r),
        float(capacity_factor), _ptr(expert_idx), _ptr(gate), _ptr(pos_in_expert),
        _ptr(record), _ptr(workspace), workspace.numel(), _stream_handle(stream)),
        "forward_shard_begin")


def switch_layer_forward_shard_end(x, W1, b1, W2, b2, capacity_factor, T_total, rank, world,
                                   gathered, out, expert_idx, gate, pos_in_expert, aux_loss,
                                   workspace=None, stream=None) -> None:
    """Step 3 of a forward over one rank's token range of a global batch."""
    T, d = x.shape
    N, d_ff, _ = W1.shape
    act = x.dtype
    for t, n in ((x, "x"), (W1, "W1"), (b1, "b1"), (W2, "W2"), (b2, "b2"), (out, "out")):
        _require(t, n, act)
    _require(gathered, "gathered", torch.uint8)
    _require(workspace, "workspace", torch.uint8)
    if gathered.numel() != world * switch_layer_shard_record_bytes(N):
        raise ValueError("gathered must hold world * record bytes")
    _check(lib().switch_layer_forward_shard_end(
        T, d, d_ff, N, dtype_code(act), int(T_total), int(rank), int(world), _ptr(gathered),
        _ptr(x), _ptr(W1), _ptr(b1), _ptr(W2), _ptr(b2), float(capacity_factor), _ptr(out),
        _ptr(expert_idx), _ptr(gate), _ptr(pos_in_expert), _ptr(aux_loss), _ptr(workspace),
        workspace.numel(), _stream_handle(stream)), "forward_shard_end")


# ---------------------------------------------------------------------------
# convenience: allocate outputs + workspace with torch and run
# ---------------------------------------------------------------------------
def alloc_workspace(T, d, d_ff, N, act_dtype: torch.dtype, capacity_factor: float,
                    host_io: bool = False, device="cuda", top2: bool = False,
                    ntlb: bool = False) -> torch.Tensor:
    n = switch_layer_workspace_size(T, d, d_ff, N, dtype_code(act_dtype), capacity_factor,
                                    (SWL_WS_HOST_IO if host_io else 0) |
                                    (SWL_WS_TOP2 if top2 else 0) |
                                    (SWL_WS_NTLB if ntlb else 0))
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device)


def alloc_outputs(T, d, act_dtype, device="cuda") -> dict:
    return {
        "out": torch.empty((T, d), dtype=act_dtype, device=device),
        "expert_idx": torch.empty(T, dtype=torch.int32, device=device),
        "gate": torch.empty(T, dtype=torch.float32, device=device),
        "pos_in_expert": torch.empty(T, dtype=torch.int32, device=device),
        "aux_loss": torch.empty(1, dtype=torch.float32, device=device),
    }


def forward(inputs: dict, capacity_factor: float, workspace: Optional[torch.Tensor] = None,
            outputs: Optional[dict] = None, stream=None, check: bool = True) -> dict:
    """Run the layer on ``inputs`` (keys x, W_r, b_r, W1, b1, W2, b2; CUDA tensors)."""
    x, W1 = inputs["x"], inputs["W1"]
    T, d = x.shape
    N, d_ff, _ = W1.shape
    if workspace is None:
        workspace = alloc_workspace(T, d, d_ff, N, x.dtype, capacity_factor, device=x.device)
    if outputs is None:
        outputs = alloc_outputs(T, d, x.dtype, device=x.device)
    switch_layer_forward(x, inputs["W_r"], W1, inputs["b1"], inputs["W2"], inputs["b2"],
                         capacity_factor, outputs["out"], outputs["expert_idx"], outputs["gate"],
                         outputs["pos_in_expert"], outputs["aux_loss"], b_r=inputs.get("b_r"),
                         workspace=workspace, stream=stream)
    if check:
        _check(switch_layer_device_status(workspace, stream), "device status")
    return outputs


def forward_shard(inputs: dict, capacity_factor: float, T_total: int, rank: int, world: int,
                  exchange, workspace: Optional[torch.Tensor] = None,
                  outputs: Optional[dict] = None, stream=None, check: bool = True) -> dict:
    """One rank's part of a forward over a global batch: ``inputs`` holds this
    rank's token range (x) and the full weights; ``exchange(record)`` returns
    the records of all ranks in rank order (an all-gather)."""
    x, W1 = inputs["x"], inputs["W1"]
    T, d = x.shape
    N, d_ff, _ = W1.shape
    if workspace is None:
        workspace = alloc_workspace(max(T, 1), d, d_ff, N, x.dtype, capacity_factor,
                                    device=W1.device)
    if outputs is None:
        outputs = alloc_outputs(T, d, x.dtype, device=W1.device)
    record = torch.empty(switch_layer_shard_record_bytes(N), dtype=torch.uint8,
                         device=W1.device)
    switch_layer_forward_shard_begin(x, inputs["W_r"], capacity_factor, T_total,
                                     outputs["expert_idx"], outputs["gate"],
                                     outputs["pos_in_expert"], record, d_ff,
                                     b_r=inputs.get("b_r"), workspace=workspace, stream=stream)
    gathered = exchange(record)
    switch_layer_forward_shard_end(x, W1, inputs["b1"], inputs["W2"], inputs["b2"],
                                   capacity_factor, T_total, rank, world, gathered,
                                   outputs["out"], outputs["expert_idx"], outputs["gate"],
                                   outputs["pos_in_expert"], outputs["aux_loss"],
                                   workspace=workspace, stream=stream)
    if check:
        _check(switch_layer_device_status(workspace, stream), "device status")
    return outputs


def forward_top2(inputs: dict, capacity_factor: float, normalize: bool = True,
                 workspace: Optional[torch.Tensor] = None, stream=None,
                 check: bool = True) -> dict:
    """Run the top-2 variant on ``inputs`` (CUDA tensors); [T, 2] routing outputs."""
    x, W1 = inputs["x"], inputs["W1"]
    T, d = x.shape
    N, d_ff, _ = W1.shape
    if workspace is None:
        workspace = alloc_workspace(T, d, d_ff, N, x.dtype, capacity_factor, device=x.device,
                                    top2=True)
    o = {"out": torch.empty((T, d), dtype=x.dtype, device=x.device),
         "expert_idx": torch.empty((T, 2), dtype=torch.int32, device=x.device),
         "gate": torch.empty((T, 2), dtype=torch.float32, device=x.device),
         "pos_in_expert": torch.empty((T, 2), dtype=torch.int32, device=x.device),
         "aux_loss": torch.empty(1, dtype=torch.float32, device=x.device)}
    switch_layer_forward_top2(x, inputs["W_r"], W1, inputs["b1"], inputs["W2"], inputs["b2"],
                              capacity_factor, normalize, o["out"], o["expert_idx"], o["gate"],
                              o["pos_in_expert"], o["aux_loss"], b_r=inputs.get("b_r"),
                              workspace=workspace, stream=stream)
    if check:
        _check(switch_layer_device_status(workspace, stream), "device status")
    return o


def forward_ntlb(inputs: dict, capacity_factor: float,
                 workspace: Optional[torch.Tensor] = None, stream=None,
                 check: bool = True) -> dict:
    """Run the No-Token-Left-Behind variant on ``inputs`` (CUDA tensors); [T, 2]
    routing outputs."""
    x, W1 = inputs["x"], inputs["W1"]
    T, d = x.shape
    N, d_ff, _ = W1.shape
    if workspace is None:
        workspace = alloc_workspace(T, d, d_ff, N, x.dtype, capacity_factor, device=x.device,
                                    ntlb=True)
    o = {"out": torch.empty((T, d), dtype=x.dtype, device=x.device),
         "expert_idx": torch.empty((T, 2), dtype=torch.int32, device=x.device),
         "gate": torch.empty((T, 2), dtype=torch.float32, device=x.device),
         "pos_in_expert": torch.empty((T, 2), dtype=torch.int32, device=x.device),
         "aux_loss": torch.empty(1, dtype=torch.float32, device=x.device)}
    switch_layer_forward_ntlb(x, inputs["W_r"], W1, inputs["b1"], inputs["W2"], inputs["b2"],
                              capacity_factor, o["out"], o["expert_idx"], o["gate"],
                              o["pos_in_expert"], o["aux_loss"], b_r=inputs.get("b_r"),
                              workspace=workspace, stream=stream)
    if check:
        _check(switch_layer_device_status(workspace, stream), "device status")
    return o


def forward_ep(inputs: dict, capacity_factor: float, N: int, T_total: int, rank: int,
               world: int, allgather, alltoall, stream=None, check: bool = True) -> dict:
    """One rank's part of an expert-parallel forward pass.  ``inputs``: this
    rank's token range x, the full W_r (and b_r), and the weights of this
    rank's experts W1/b1/W2/b2 ([N / world, ...]).  ``allgather(record)``
    returns every rank's record in rank order (device); ``alltoall(rows,
    send_counts, recv_counts)`` exchanges row blocks between ranks (rows [sum
    send, d] -> [sum recv, d])."""
    x, W1 = inputs["x"], inputs["W1"]
    T, d = x.shape
    d_ff = W1.shape[1]
    dev = W1.device
    ws = torch.empty(switch_layer_ep_workspace_size(T, d, d_ff, N, dtype_code(x.dtype), world,
                                                    T_total, capacity_factor),
                     dtype=torch.uint8, device=dev)
    o = alloc_outputs(T, d, x.dtype, device=dev)
    record = torch.empty(switch_layer_shard_record_bytes(N), dtype=torch.uint8, device=dev)
    switch_layer_forward_shard_begin(x, inputs["W_r"], capacity_factor, T_total, o["expert_idx"],
                                     o["gate"], o["pos_in_expert"], record, d_ff,
                                     b_r=inputs.get("b_r"), workspace=ws, stream=stream)
    gathered = allgather(record)
    send_c, recv_c = switch_layer_ep_counts(N, world, rank, T_total, capacity_factor,
                                            gathered.cpu())
    send = torch.empty((sum(send_c), d), dtype=x.dtype, device=dev)
    switch_layer_ep_dispatch(x, d_ff, N, world, rank, T_total, capacity_factor, gathered,
                             o["expert_idx"], o["pos_in_expert"], o["aux_loss"], send, ws,
                             stream)
    recv = alltoall(send, send_c, recv_c)
    ret = torch.empty_like(recv)
    switch_layer_ep_experts(T, d, d_ff, N, x.dtype, world, rank, T_total, capacity_factor,
                            gathered, recv, W1, inputs["b1"], inputs["W2"], inputs["b2"], ret, ws,
                            stream)
    back = alltoall(ret, recv_c, send_c)
    switch_layer_ep_combine(T, d, d_ff, N, x.dtype, world, rank, T_total, capacity_factor, back,
                            o["expert_idx"], o["gate"], o["pos_in_expert"], o["out"], ws, stream)
    if check:
        _check(switch_layer_device_status(ws, stream), "device status")
    return o


def make_variant(top_k: int = 1, normalize: bool = True, activation: str = "relu",
                 router_noise: Optional[torch.Tensor] = None) -> Variant:
    if router_noise is not None:
        _require(router_noise, "router_noise", torch.float32)
    return Variant(int(top_k), 1 if normalize else 0,
                   {"relu": SWL_ACT_RELU, "geglu": SWL_ACT_GEGLU}[activation],
                   None if router_noise is None else router_noise.data_ptr())


def switch_layer_variant_workspace_size(T, d, d_ff, N, dtype, capacity_factor,
                                        variant: Variant) -> int:
    n = _sz(0)
    _check(lib().switch_layer_variant_workspace_size(T, d, d_ff, N, dtype, capacity_factor,
                                                     ctypes.byref(variant), ctypes.byref(n)),
           "variant_workspace_size")
    return int(n.value)


def forward_variant(inputs: dict, capacity_factor: float, top_k: int = 1, normalize: bool = True,
                    activation: str = "relu", router_noise: Optional[torch.Tensor] = None,
                    workspace: Optional[torch.Tensor] = None, stream=None,
                    check: bool = True) -> dict:
    """Run a layer variant (top-2 routing, GEGLU experts, router input jitter)."""
    x, W1 = inputs["x"], inputs["W1"]
    T, d = x.shape
    N = W1.shape[0]
    d_ff = W1.shape[1] // (2 if activation == "geglu" else 1)
    v = make_variant(top_k, normalize, activation, router_noise)
    if workspace is None:
        workspace = torch.empty(max(256, switch_layer_variant_workspace_size(
            T, d, d_ff, N, dtype_code(x.dtype), capacity_factor, v)), dtype=torch.uint8,
            device=x.device)
    shape_k = (T, top_k) if top_k == 2 else (T,)
    o = {"out": torch.empty((T, d), dtype=x.dtype, device=x.device),
         "expert_idx": torch.empty(shape_k, dtype=torch.int32, device=x.device),
         "gate": torch.empty(shape_k, dtype=torch.float32, device=x.device),
         "pos_in_expert": torch.empty(shape_k, dtype=torch.int32, device=x.device),
         "aux_loss": torch.empty(1, dtype=torch.float32, device=x.device)}
    for t, n in ((x, "x"), (W1, "W1"), (inputs["b1"], "b1"), (inputs["W2"], "W2"),
                 (inputs["b2"], "b2")):
        _require(t, n, x.dtype)
    _require(inputs["W_r"], "W_r", torch.float32)
    _check(lib().switch_layer_forward_variant(
        T, d, d_ff, N, dtype_code(x.dtype), _ptr(x), _ptr(inputs["W_r"]), _ptr(W1),
        _ptr(inputs["b1"]), _ptr(inputs["W2"]), _ptr(inputs["b2"]), float(capacity_factor),
        _ptr(o["out"]), _ptr(o["expert_idx"]), _ptr(o["gate"]), _ptr(o["pos_in_expert"]),
        _ptr(o["aux_loss"]), _ptr(inputs.get("b_r")), ctypes.byref(v), _ptr(workspace),
        workspace.numel(), _stream_handle(stream)), "forward_variant")
    if check:
        _check(switch_layer_device_status(workspace, stream), "device status")
    return o


def backward(inputs: dict, capacity_factor: float, fwd: dict, fwd_workspace: torch.Tensor,
             dout: torch.Tensor, daux: float = 0.0, stream=None, check: bool = True) -> dict:
    """Gradients of sum(dout * out) + daux * aux for a forward call made with
    ``fwd_workspace`` (its outputs ``fwd``): dx, dW_r, db_r, dW1, db1, dW2, db2."""
    x, W1 = inputs["x"], inputs["W1"]
    T, d = x.shape
    N, d_ff, _ = W1.shape
    dev = x.device
    n = _sz(0)
    _check(lib().switch_layer_backward_workspace_size(T, d, d_ff, N, dtype_code(x.dtype),
                                                      float(capacity_factor), ctypes.byref(n)),
           "backward_workspace_size")
    bws = torch.empty(max(256, int(n.value)), dtype=torch.uint8, device=dev)
    g = {"dx": torch.empty_like(x), "dW_r": torch.empty_like(inputs["W_r"]),
         "db_r": torch.empty(N, dtype=torch.float32, device=dev),
         "dW1": torch.empty_like(W1), "db1": torch.empty_like(inputs["b1"]),
         "dW2": torch.empty_like(inputs["W2"]), "db2": torch.empty_like(inputs["b2"])}
    _require(dout, "dout", x.dtype)
    _check(lib().switch_layer_backward(
        T, d, d_ff, N, dtype_code(x.dtype), _ptr(x), _ptr(inputs["W_r"]), _ptr(inputs.get("b_r")),
        _ptr(W1), _ptr(inputs["b1"]), _ptr(inputs["W2"]), _ptr(inputs["b2"]),
        float(capacity_factor), _ptr(fwd["out"]), _ptr(fwd["expert_idx"]), _ptr(fwd["gate"]),
        _ptr(fwd["pos_in_expert"]), _ptr(fwd_workspace), fwd_workspace.numel(), _ptr(dout),
        float(daux), _ptr(g["dx"]), _ptr(g["dW_r"]), _ptr(g["db_r"]), _ptr(g["dW1"]),
        _ptr(g["db1"]), _ptr(g["dW2"]), _ptr(g["db2"]), _ptr(bws), bws.numel(),
        _stream_handle(stream)), "backward")
    if check:
        _check(switch_layer_device_status(fwd_workspace, stream), "device status")
    return g
