"""Batch-invariant token logprobs and the REINFORCE Zero loss/gradient on B200.

Thin Python binding over librz.so (include/rz.h).  Every step of the path runs in the
library's CUDA kernels; this module only marshals torch tensors (device memory, streams)
into the C calls, which keep their C names.  There is no CPU or PyTorch fallback: if
librz.so is missing or no CUDA device is present, the calls raise.
"""
from __future__ import annotations

import ctypes
import functools
import os

from .build import LIB as _LIB_PATH

__all__ = [
    "RZ_OK", "RZError", "lib", "rz_status_string", "rz_workspace_bytes_logprobs", "rz_workspace_bytes_loss",
    "rz_workspace_bytes_segment_loss", "rz_token_logprobs", "rz_loss_fwd_bwd", "rz_segment_loss",
    "rz_read_device_status", "rz_num_launches_loss", "rz_loss_fwd_bwd_timed", "rz_loss_fwd_bwd_ex",
    "rz_loss_fwd_bwd_streamed", "rz_loss_fwd_bwd_host_io", "rz_segment_loss_ex", "rz_ratio_stats", "rz_grad_norms", "rz_quantize_rows_e4m3",
    "rz_token_logprobs_fp8", "rz_sum_shards_f32", "rz_selftest_wait_timeout", "rz_token_logprobs_noalloc",
    "rz_mxfp4_scale_bytes", "rz_quantize_rows_mxfp4", "rz_token_logprobs_mxfp4",
    "rz_workspace_bytes_ratio_stats", "rz_workspace_bytes_grad_norms", "rz_selftest_forward_after_timeout",
    "rz_loss_options", "loss_options",
    "EXPORTED_SYMBOLS", "STAT_NAMES", "KERNEL_KINDS",
]

RZ_OK = 0
STATUS_NAMES = {
    0: "RZ_OK", 1: "RZ_ERR_INVALID_ARG", 2: "RZ_ERR_UNSUPPORTED_SHAPE", 3: "RZ_ERR_WORKSPACE_TOO_SMALL",
    4: "RZ_ERR_CUDA", 5: "RZ_ERR_DEVICE_CHECK", 6: "RZ_ERR_DEVICE_TIMEOUT",
}
EXPORTED_SYMBOLS = (
    "rz_status_string", "rz_workspace_bytes_logprobs", "rz_workspace_bytes_loss", "rz_workspace_bytes_segment_loss",
    "rz_token_logprobs", "rz_loss_fwd_bwd", "rz_segment_loss", "rz_read_device_status", "rz_num_launches_loss",
    "rz_loss_fwd_bwd_timed", "rz_token_logprobs_noalloc", "rz_loss_fwd_bwd_ex", "rz_loss_fwd_bwd_streamed",
    "rz_loss_fwd_bwd_host_io",
    "rz_segment_loss_ex",
    "rz_workspace_bytes_ratio_stats", "rz_ratio_stats", "rz_workspace_bytes_grad_norms", "rz_grad_norms",
    "rz_quantize_rows_e4m3", "rz_token_logprobs_fp8", "rz_sum_shards_f32", "rz_selftest_wait_timeout",
    "rz_selftest_forward_after_timeout", "rz_mxfp4_scale_bytes", "rz_quantize_rows_mxfp4", "rz_token_logprobs_mxfp4",
)
RZ_LOSS_CLIP_IS, RZ_LOSS_SEQ_GATE, RZ_LOSS_TOKEN_MASK = 1, 2, 4
STAT_NAMES = ("k1", "k2", "k3", "w_min", "w_max", "dev_max", "dev_median", "dev_peak_over_median", "count")


class rz_loss_options(ctypes.Structure):
    """Mirror of the C struct rz_loss_options (include/rz.h)."""
    _fields_ = [("flags", ctypes.c_int32), ("clip_max", ctypes.c_float), ("gate_lo", ctypes.c_double),
                ("gate_hi", ctypes.c_double), ("token_mask", ctypes.c_void_p), ("n_resp_total", ctypes.c_int32)]


def loss_options(clip_max=None, gate=None, token_mask=None, n_resp_total=0):
    """Build rz_loss_options: clip_max (float), gate ((lo, hi)), token_mask (contiguous uint8 CUDA
    tensor [n_tok], kept alive by the returned struct; its length is checked at each call)."""
    if token_mask is not None:
        _need(token_mask, _torch().uint8, "token_mask")
    o = rz_loss_options()
    o.flags, o.clip_max, o.gate_lo, o.gate_hi, o.token_mask = 0, 0.0, 0.0, 0.0, None
    if clip_max is not None:
        o.flags |= RZ_LOSS_CLIP_IS
        o.clip_max = float(clip_max)
    if gate is not None:
        o.flags |= RZ_LOSS_SEQ_GATE
        o.gate_lo, o.gate_hi = float(gate[0]), float(gate[1])
    if token_mask is not None:
        o.flags |= RZ_LOSS_TOKEN_MASK
        o.token_mask = token_mask.data_ptr()
    o._token_mask = token_mask
    o.n_resp_total = int(n_resp_total)
    return o


KERNEL_KINDS = ("lmhead_lse", "merge_lse", "response_coef", "token_kappa", "loss_final", "dz", "dh", "dw",
                "block_first")

_lib = None


class RZError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {STATUS_NAMES.get(code, code)}")
        self.code = code


def lib() -> ctypes.CDLL:
    """The loaded librz.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise ImportError(f"librz.so not built at {_LIB_PATH}; run invariant_logprobs_reinforce_b200.build.build()")
        L = ctypes.CDLL(_LIB_PATH)
        P, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
        L.rz_status_string.argtypes = [ctypes.c_int]
        L.rz_status_string.restype = ctypes.c_char_p
        L.rz_workspace_bytes_logprobs.argtypes = [i64, i32, i32]
        L.rz_workspace_bytes_logprobs.restype = sz
        L.rz_workspace_bytes_loss.argtypes = [i64, i32, i32, i32, i32]
        L.rz_workspace_bytes_loss.restype = sz
        L.rz_workspace_bytes_segment_loss.argtypes = [i64, i32, i32]
        L.rz_workspace_bytes_segment_loss.restype = sz
        L.rz_token_logprobs.argtypes = [P, P, P, i64, i32, i32, P, P, P, sz, P]
        L.rz_token_logprobs.restype = ctypes.c_int
        L.rz_loss_fwd_bwd.argtypes = [P, P, P, P, P, P, P, i64, i32, i32, i32, i32, P, P, P, P, P, P, sz, P]
        L.rz_loss_fwd_bwd.restype = ctypes.c_int
        L.rz_segment_loss.argtypes = [P, P, P, P, P, i64, i32, i32, P, P, P, P, sz, P]
        L.rz_segment_loss.restype = ctypes.c_int
        L.rz_loss_fwd_bwd_timed.argtypes = [P, P, P, P, P, P, P, i64, i32, i32, i32, i32, P, P, P, P, P, P, sz, P,
                                             P, P, i32, ctypes.POINTER(ctypes.c_int32)]
        L.rz_loss_fwd_bwd_timed.restype = ctypes.c_int
        L.rz_num_launches_loss.argtypes = [i64]
        L.rz_num_launches_loss.restype = i32
        L.rz_token_logprobs_noalloc.argtypes = [P, P, P, i64, i32, i32, P, P, P]
        L.rz_token_logprobs_noalloc.restype = ctypes.c_int
        L.rz_loss_fwd_bwd_ex.argtypes = [P, P, P, P, P, P, P, i64, i32, i32, i32, i32, ctypes.POINTER(rz_loss_options),
                                          P, P, P, P, P, P, sz, P]
        L.rz_loss_fwd_bwd_ex.restype = ctypes.c_int
        L.rz_loss_fwd_bwd_streamed.argtypes = [P, P, P, P, P, P, P, P, i64, i32, i32, i32, i32,
                                                ctypes.POINTER(rz_loss_options), P, P, P, P, P, P, sz, P]
        L.rz_loss_fwd_bwd_streamed.restype = ctypes.c_int
        L.rz_loss_fwd_bwd_host_io.argtypes = [P, P, P, P, P, P, P, P, i64, i32, i32, i32, i32,
                                               ctypes.POINTER(rz_loss_options), P, P, P, P, P, P, P, P, sz, P]
        L.rz_loss_fwd_bwd_host_io.restype = ctypes.c_int
        L.rz_segment_loss_ex.argtypes = [P, P, P, P, P, i64, i32, i32, ctypes.POINTER(rz_loss_options), P, P, P, P,
                                          sz, P]
        L.rz_segment_loss_ex.restype = ctypes.c_int
        L.rz_workspace_bytes_ratio_stats.argtypes = [i64, i32]
        L.rz_workspace_bytes_ratio_stats.restype = sz
        L.rz_ratio_stats.argtypes = [P, P, P, i64, i32, P, P, P, P, sz, P]
        L.rz_ratio_stats.restype = ctypes.c_int
        L.rz_workspace_bytes_grad_norms.argtypes = []
        L.rz_workspace_bytes_grad_norms.restype = sz
        L.rz_grad_norms.argtypes = [P, P, i64, i32, i32, P, P, sz, P]
        L.rz_grad_norms.restype = ctypes.c_int
        L.rz_quantize_rows_e4m3.argtypes = [P, i64, i32, P, P, P]
        L.rz_quantize_rows_e4m3.restype = ctypes.c_int
        L.rz_token_logprobs_fp8.argtypes = [P, P, P, P, P, i64, i32, i32, P, P, P, sz, P]
        L.rz_token_logprobs_fp8.restype = ctypes.c_int
        L.rz_mxfp4_scale_bytes.argtypes = [i64, i32]
        L.rz_mxfp4_scale_bytes.restype = sz
        L.rz_quantize_rows_mxfp4.argtypes = [P, i64, i32, P, P, P]
        L.rz_quantize_rows_mxfp4.restype = ctypes.c_int
        L.rz_token_logprobs_mxfp4.argtypes = [P, P, P, P, P, i64, i32, i32, P, P, P, sz, P]
        L.rz_token_logprobs_mxfp4.restype = ctypes.c_int
        L.rz_sum_shards_f32.argtypes = [P, i32, i64, P, P]
        L.rz_sum_shards_f32.restype = ctypes.c_int
        L.rz_selftest_wait_timeout.argtypes = [ctypes.c_uint64, P, sz, ctypes.POINTER(ctypes.c_uint64), P]
        L.rz_selftest_wait_timeout.restype = ctypes.c_int
        L.rz_selftest_forward_after_timeout.argtypes = [i32, P, P, P, i64, i32, i32, P, P, P, sz, P]
        L.rz_selftest_forward_after_timeout.restype = ctypes.c_int
        L.rz_read_device_status.argtypes = [P, P, ctypes.POINTER(ctypes.c_int32)]
        L.rz_read_device_status.restype = ctypes.c_int
        _lib = L
    return _lib


def rz_status_string(code: int) -> str:
    return lib().rz_status_string(code).decode()


def rz_workspace_bytes_logprobs(n_tok: int, d: int, V: int) -> int:
    return int(lib().rz_workspace_bytes_logprobs(n_tok, d, V))


def rz_workspace_bytes_loss(n_tok: int, n_resp: int, n_groups: int, d: int, V: int) -> int:
    return int(lib().rz_workspace_bytes_loss(n_tok, n_resp, n_groups, d, V))


def rz_workspace_bytes_segment_loss(n_tok: int, n_resp: int, n_groups: int) -> int:
    return int(lib().rz_workspace_bytes_segment_loss(n_tok, n_resp, n_groups))


def rz_workspace_bytes_ratio_stats(n_tok: int, n_resp: int) -> int:
    return int(lib().rz_workspace_bytes_ratio_stats(n_tok, n_resp))


def rz_workspace_bytes_grad_norms() -> int:
    return int(lib().rz_workspace_bytes_grad_norms())


# ----------------------------------------------------------------------------- helpers

def _torch():
    import torch
    return torch


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream):
    """The stream to enqueue on: `stream`, else the current stream of the current device
    (the entry points make the tensors' device current first, see _on_tensor_device)."""
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    elif stream.device != torch.device("cuda", torch.cuda.current_device()):
        raise ValueError(f"stream is on {stream.device}, the tensors on cuda:{torch.cuda.current_device()}")
    return ctypes.c_void_p(stream.cuda_stream)


def _on_tensor_device(fn):
    """Run an entry point with the device of its first CUDA tensor argument current: the
    library launches on the current device, which must be the one that holds the data."""
    @functools.wraps(fn)
    def wrapper(*args, **kwargs):
        torch = _torch()
        for a in (*args, *kwargs.values()):
            if isinstance(a, torch.Tensor) and a.is_cuda:
                with torch.cuda.device(a.device):
                    return fn(*args, **kwargs)
        return fn(*args, **kwargs)
    return wrapper


def _need(t, dtype, name, device=None):
    torch = _torch()
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be on a CUDA device")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _shape(t, shape, name):
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    return t


def _need_shaped(t, dtype, name, device, shape):
    """_need plus an exact shape; None passes through (an omitted optional argument)."""
    if t is None:
        return None
    return _shape(_need(t, dtype, name, device), shape, name)


def _matrix(t, dtype, name, device=None):
    _need(t, dtype, name, device)
    if t.dim() != 2:
        raise ValueError(f"{name} must be 2-D, got shape {tuple(t.shape)}")
    return t.shape


def _segments(lp_rollout, rewards, seg_offsets, group_ids, n, dev):
    """Checks the per-token rollout logprobs and the response / group description; returns R."""
    torch = _torch()
    _need_shaped(lp_rollout, torch.float32, "lp_rollout", dev, (n,))
    _need(rewards, torch.float32, "rewards", dev)
    if rewards.dim() != 1:
        raise ValueError("rewards must be 1-D [n_resp]")
    R = rewards.shape[0]
    _need_shaped(seg_offsets, torch.int64, "seg_offsets", dev, (R + 1,))
    _need_shaped(group_ids, torch.int32, "group_ids", dev, (R,))
    return R


def _token_vector(t, name):
    """A per-token fp32 vector on a CUDA device; returns (n, device)."""
    _need(t, _torch().float32, name)
    if t.dim() != 1:
        raise ValueError(f"{name} must be 1-D [n_tok]")
    return t.shape[0], t.device


def _loss_inputs(H, W_head, token_ids, lp_rollout, rewards, seg_offsets, group_ids, H_name="H"):
    """Checks the loss entry points' device inputs; returns (device, n, d, V, R)."""
    torch = _torch()
    n, d = _matrix(H, torch.bfloat16, H_name)
    dev = H.device
    V, dw = _matrix(W_head, torch.bfloat16, "W_head", dev)
    if dw != d:
        raise ValueError(f"W_head has d = {dw}, H has d = {d}")
    _need_shaped(token_ids, torch.int32, "token_ids", dev, (n,))
    R = _segments(lp_rollout, rewards, seg_offsets, group_ids, n, dev)
    return dev, n, d, V, R


def _loss_outputs(dev, n, d, V, loss=None, dH=None, dW=None, lp=None, kappa=None):
    torch = _torch()
    _need_shaped(loss, torch.float32, "loss", dev, (1,))
    _need_shaped(dH, torch.bfloat16, "dH", dev, (n, d))
    _need_shaped(dW, torch.float32, "dW", dev, (V, d))
    _need_shaped(lp, torch.float32, "lp_out", dev, (n,))
    _need_shaped(kappa, torch.float32, "kappa_out", dev, (n,))


def _options_ref(options, n, dev):
    """ctypes reference to rz_loss_options after checking its token mask against this call."""
    if options is None:
        return None
    if not isinstance(options, rz_loss_options):
        raise TypeError("options must be an rz_loss_options (see loss_options)")
    if options.flags & RZ_LOSS_TOKEN_MASK:
        m = getattr(options, "_token_mask", None)
        if m is None or m.data_ptr() != (options.token_mask or 0):
            raise ValueError("options carry a token mask without its tensor; build them with loss_options()")
        _need_shaped(m, _torch().uint8, "token_mask", dev, (n,))
    return ctypes.byref(options)


def _workspace(nbytes, workspace, device):
    torch = _torch()
    if workspace is None:
        return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
    _need(workspace, torch.uint8, "workspace", device)
    return workspace


def _check(code, what):
    if code != RZ_OK:
        raise RZError(code, what)


# ----------------------------------------------------------------------------- entry points

@_on_tensor_device
def rz_token_logprobs(H, W_head, token_ids, lp_out=None, lse_out=None, workspace=None, stream=None,
                      want_lse=True):
    """Token logprobs of the sampled tokens (bf16 H [n,d], bf16 W [V,d], int32 ids [n]).

    Returns (lp, lse) as fp32 CUDA tensors (lse is None when want_lse is False and no
    lse_out is given).
    """
    torch = _torch()
    n, d = _matrix(H, torch.bfloat16, "H")
    dev = H.device
    V, dw = _matrix(W_head, torch.bfloat16, "W_head", dev)
    if dw != d:
        raise ValueError(f"W_head has d = {dw}, H has d = {d}")
    _need_shaped(token_ids, torch.int32, "token_ids", dev, (n,))
    _need_shaped(lp_out, torch.float32, "lp_out", dev, (n,))
    _need_shaped(lse_out, torch.float32, "lse_out", dev, (n,))
    lp = lp_out if lp_out is not None else torch.empty(n, dtype=torch.float32, device=dev)
    lse = lse_out if lse_out is not None else (torch.empty(n, dtype=torch.float32, device=dev) if want_lse else None)
    ws_bytes = rz_workspace_bytes_logprobs(n, d, V)
    ws = _workspace(ws_bytes, workspace, dev)
    code = lib().rz_token_logprobs(_ptr(H), _ptr(W_head), _ptr(token_ids), n, d, V, _ptr(lp), _ptr(lse), _ptr(ws),
                                   ws.numel(), _stream_handle(stream))
    _check(code, "rz_token_logprobs")
    return lp, lse


@_on_tensor_device
def rz_token_logprobs_noalloc(H, W_head, token_ids, lp_out, lse_out=None, stream=None):
    """rz_token_logprobs from the library's fixed scratch instead of a workspace: the caller
    passes every output buffer, and neither this wrapper nor the library allocates.  Calls
    that may overlap on the GPU must be serialised by the caller (they share the scratch).
    Returns (lp_out, lse_out)."""
    torch = _torch()
    n, d = _matrix(H, torch.bfloat16, "H")
    dev = H.device
    V, dw = _matrix(W_head, torch.bfloat16, "W_head", dev)
    if dw != d:
        raise ValueError(f"W_head has d = {dw}, H has d = {d}")
    _need_shaped(token_ids, torch.int32, "token_ids", dev, (n,))
    if lp_out is None:
        raise ValueError("lp_out is required (this entry point allocates nothing)")
    _need_shaped(lp_out, torch.float32, "lp_out", dev, (n,))
    _need_shaped(lse_out, torch.float32, "lse_out", dev, (n,))
    _check(lib().rz_token_logprobs_noalloc(_ptr(H), _ptr(W_head), _ptr(token_ids), n, d, V, _ptr(lp_out),
                                           _ptr(lse_out), _stream_handle(stream)), "rz_token_logprobs_noalloc")
    return lp_out, lse_out


@_on_tensor_device
def rz_loss_fwd_bwd(H, W_head, token_ids, lp_rollout, rewards, seg_offsets, group_ids, n_groups, loss=None,
                    dH=None, dW=None, lp_out=None, kappa_out=None, workspace=None, stream=None, want_lp=True,
                    want_kappa=True):
    """Forward + REINFORCE Zero loss + backward.  Returns dict(loss, dH, dW, lp, kappa, workspace)."""
    torch = _torch()
    dev, n, d, V, R = _loss_inputs(H, W_head, token_ids, lp_rollout, rewards, seg_offsets, group_ids)
    _loss_outputs(dev, n, d, V, loss, dH, dW, lp_out, kappa_out)
    loss = loss if loss is not None else torch.empty(1, dtype=torch.float32, device=dev)
    dH = dH if dH is not None else torch.empty((n, d), dtype=torch.bfloat16, device=dev)
    dW = dW if dW is not None else torch.empty((V, d), dtype=torch.float32, device=dev)
    if lp_out is None and want_lp:
        lp_out = torch.empty(n, dtype=torch.float32, device=dev)
    if kappa_out is None and want_kappa:
        kappa_out = torch.empty(n, dtype=torch.float32, device=dev)
    ws_bytes = rz_workspace_bytes_loss(n, R, n_groups, d, V)
    ws = _workspace(ws_bytes, workspace, dev)
    code = lib().rz_loss_fwd_bwd(_ptr(H), _ptr(W_head), _ptr(token_ids), _ptr(lp_rollout), _ptr(rewards),
                                 _ptr(seg_offsets), _ptr(group_ids), n, R, n_groups, d, V, _ptr(loss), _ptr(dH),
                                 _ptr(dW), _ptr(lp_out), _ptr(kappa_out), _ptr(ws), ws.numel(),
                                 _stream_handle(stream))
    _check(code, "rz_loss_fwd_bwd")
    return dict(loss=loss, dH=dH, dW=dW, lp=lp_out, kappa=kappa_out, workspace=ws)


def rz_num_launches_loss(n_tok: int) -> int:
    return int(lib().rz_num_launches_loss(n_tok))


@_on_tensor_device
def rz_loss_fwd_bwd_timed(events, H, W_head, token_ids, lp_rollout, rewards, seg_offsets, group_ids, n_groups,
                          loss, dH, dW, lp_out, kappa_out, workspace, stream=None):
    """rz_loss_fwd_bwd recording a CUDA event pair around every kernel launch.

    ``events`` is a list of 2*capacity torch.cuda.Event(enable_timing=True) objects that
    have been recorded once (so their handles exist).  Returns the kernel kind of each
    recorded launch (indices into KERNEL_KINDS).
    """
    dev, n, d, V, R = _loss_inputs(H, W_head, token_ids, lp_rollout, rewards, seg_offsets, group_ids)
    _loss_outputs(dev, n, d, V, loss, dH, dW, lp_out, kappa_out)
    for name, t in (("loss", loss), ("dH", dH), ("dW", dW)):
        if t is None:
            raise ValueError(f"{name} is required")
    _need(workspace, _torch().uint8, "workspace", dev)
    cap = len(events) // 2
    handles = (ctypes.c_void_p * (2 * cap))(*[ctypes.c_void_p(e.cuda_event) for e in events[:2 * cap]])
    kinds = (ctypes.c_int32 * max(cap, 1))()
    count = ctypes.c_int32(0)
    code = lib().rz_loss_fwd_bwd_timed(_ptr(H), _ptr(W_head), _ptr(token_ids), _ptr(lp_rollout), _ptr(rewards),
                                       _ptr(seg_offsets), _ptr(group_ids), n, R, n_groups, d, V, _ptr(loss), _ptr(dH),
                                       _ptr(dW), _ptr(lp_out), _ptr(kappa_out), _ptr(workspace), workspace.numel(),
                                       _stream_handle(stream), handles, kinds, cap, ctypes.byref(count))
    _check(code, "rz_loss_fwd_bwd_timed")
    return [int(kinds[i]) for i in range(count.value)]


@_on_tensor_device
def rz_segment_loss(lp, lp_rollout, rewards, seg_offsets, group_ids, n_groups, loss=None, kappa_out=None,
                    w_out=None, want_w=False, workspace=None, stream=None):
    """The loss stage alone from given logprobs.  Returns dict(loss, kappa, w, workspace)."""
    torch = _torch()
    n, dev = _token_vector(lp, "lp")
    R = _segments(lp_rollout, rewards, seg_offsets, group_ids, n, dev)
    _need_shaped(loss, torch.float32, "loss", dev, (1,))
    _need_shaped(kappa_out, torch.float32, "kappa_out", dev, (n,))
    _need_shaped(w_out, torch.float32, "w_out", dev, (n,))
    loss = loss if loss is not None else torch.empty(1, dtype=torch.float32, device=dev)
    kappa_out = kappa_out if kappa_out is not None else torch.empty(n, dtype=torch.float32, device=dev)
    if w_out is None and want_w:
        w_out = torch.empty(n, dtype=torch.float32, device=dev)
    ws = _workspace(rz_workspace_bytes_segment_loss(n, R, n_groups), workspace, dev)
    code = lib().rz_segment_loss(_ptr(lp), _ptr(lp_rollout), _ptr(rewards), _ptr(seg_offsets), _ptr(group_ids), n,
                                 R, n_groups, _ptr(loss), _ptr(kappa_out), _ptr(w_out), _ptr(ws), ws.numel(),
                                 _stream_handle(stream))
    _check(code, "rz_segment_loss")
    return dict(loss=loss, kappa=kappa_out, w=w_out, workspace=ws)


@_on_tensor_device
def rz_read_device_status(workspace, stream=None):
    """Synchronise the stream and return (status code, raw RZ_DEV_* bits) of a workspace."""
    bits = ctypes.c_int32(0)
    code = lib().rz_read_device_status(_ptr(workspace), _stream_handle(stream), ctypes.byref(bits))
    return int(code), int(bits.value)


@_on_tensor_device
def rz_loss_fwd_bwd_ex(H, W_head, token_ids, lp_rollout, rewards, seg_offsets, group_ids, n_groups, options,
                       workspace=None, stream=None):
    """rz_loss_fwd_bwd with rz_loss_options (see loss_options).  Returns the same dict."""
    torch = _torch()
    dev, n, d, V, R = _loss_inputs(H, W_head, token_ids, lp_rollout, rewards, seg_offsets, group_ids)
    opt = _options_ref(options, n, dev)
    out = dict(loss=torch.empty(1, dtype=torch.float32, device=dev),
               dH=torch.empty((n, d), dtype=torch.bfloat16, device=dev),
               dW=torch.empty((V, d), dtype=torch.float32, device=dev),
               lp=torch.empty(n, dtype=torch.float32, device=dev),
               kappa=torch.empty(n, dtype=torch.float32, device=dev))
    ws = _workspace(rz_workspace_bytes_loss(n, R, n_groups, d, V), workspace, dev)
    code = lib().rz_loss_fwd_bwd_ex(_ptr(H), _ptr(W_head), _ptr(token_ids), _ptr(lp_rollout), _ptr(rewards),
                                    _ptr(seg_offsets), _ptr(group_ids), n, R, n_groups, d, V, opt, _ptr(out["loss"]),
                                    _ptr(out["dH"]), _ptr(out["dW"]), _ptr(out["lp"]), _ptr(out["kappa"]), _ptr(ws),
                                    ws.numel(), _stream_handle(stream))
    _check(code, "rz_loss_fwd_bwd_ex")
    out["workspace"] = ws
    return out


@_on_tensor_device
def rz_loss_fwd_bwd_streamed(H_host, H_dev, W_head, token_ids, lp_rollout, rewards, seg_offsets, group_ids, n_groups,
                             options=None, out=None, workspace=None, stream=None):
    """rz_loss_fwd_bwd_ex with H read from host memory (H_host: CPU bf16 tensor, pinned for the copies to
    overlap the compute) into the device buffer H_dev, chunk by chunk.  `out` (the dict this returns) may be
    passed back in to reuse its buffers.  H_host must stay unchanged until the work on the stream is done."""
    torch = _torch()
    dev, n, d, V, R = _loss_inputs(H_dev, W_head, token_ids, lp_rollout, rewards, seg_offsets, group_ids, "H_dev")
    if not isinstance(H_host, torch.Tensor) or H_host.dtype != torch.bfloat16:
        raise TypeError("H_host must be a bf16 torch.Tensor")
    if H_host.device.type != "cpu" or not H_host.is_contiguous():
        raise ValueError("H_host must be a contiguous CPU tensor")
    if tuple(H_host.shape) != tuple(H_dev.shape):
        raise ValueError("H_host and H_dev must have the same shape")
    opt = _options_ref(options, n, dev)
    if out is not None:
        _loss_outputs(dev, n, d, V, out["loss"], out["dH"], out["dW"], out.get("lp"), out.get("kappa"))
    else:
        out = dict(loss=torch.empty(1, dtype=torch.float32, device=dev),
                   dH=torch.empty((n, d), dtype=torch.bfloat16, device=dev),
                   dW=torch.empty((V, d), dtype=torch.float32, device=dev),
                   lp=torch.empty(n, dtype=torch.float32, device=dev),
                   kappa=torch.empty(n, dtype=torch.float32, device=dev))
    ws = _workspace(rz_workspace_bytes_loss(n, R, n_groups, d, V), workspace, dev)
    code = lib().rz_loss_fwd_bwd_streamed(_ptr(H_host), _ptr(H_dev), _ptr(W_head), _ptr(token_ids), _ptr(lp_rollout),
                                          _ptr(rewards), _ptr(seg_offsets), _ptr(group_ids), n, R, n_groups, d, V, opt,
                                          _ptr(out["loss"]),
                                          _ptr(out["dH"]), _ptr(out["dW"]), _ptr(out.get("lp")), _ptr(out.get("kappa")),
                                          _ptr(ws), ws.numel(), _stream_handle(stream))
    _check(code, "rz_loss_fwd_bwd_streamed")
    out["workspace"] = ws
    return out


@_on_tensor_device
def rz_loss_fwd_bwd_host_io(H_host, H_dev, W_head, token_ids, lp_rollout, rewards, seg_offsets, group_ids, n_groups,
                            dH_host=None, dW_host=None, options=None, out=None, workspace=None, stream=None):
    """rz_loss_fwd_bwd_streamed that also copies the gradients to host memory: dH_host (CPU bf16 [n, d]) chunk by
    chunk as each chunk's dH is produced, dW_host (CPU fp32 [V, d]) after the last chunk; either may be None.
    Pin them (and H_host) for the copies to overlap the compute.  Returns the same dict as the streamed call, plus
    dH_host and dW_host; the host buffers hold the results once the stream's work is done."""
    torch = _torch()
    dev, n, d, V, R = _loss_inputs(H_dev, W_head, token_ids, lp_rollout, rewards, seg_offsets, group_ids, "H_dev")
    if not isinstance(H_host, torch.Tensor) or H_host.dtype != torch.bfloat16:
        raise TypeError("H_host must be a bf16 torch.Tensor")
    if H_host.device.type != "cpu" or not H_host.is_contiguous():
        raise ValueError("H_host must be a contiguous CPU tensor")
    if tuple(H_host.shape) != tuple(H_dev.shape):
        raise ValueError("H_host and H_dev must have the same shape")
    for name, t, dt, shape in (("dH_host", dH_host, torch.bfloat16, (n, d)), ("dW_host", dW_host, torch.float32, (V, d))):
        if t is None:
            continue
        if not isinstance(t, torch.Tensor) or t.dtype != dt:
            raise TypeError(f"{name} must be a {dt} torch.Tensor")
        if t.device.type != "cpu" or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CPU tensor")
        _shape(t, shape, name)
    opt = _options_ref(options, n, dev)
    if out is not None:
        _loss_outputs(dev, n, d, V, out["loss"], out["dH"], out["dW"], out.get("lp"), out.get("kappa"))
    else:
        out = dict(loss=torch.empty(1, dtype=torch.float32, device=dev),
                   dH=torch.empty((n, d), dtype=torch.bfloat16, device=dev),
                   dW=torch.empty((V, d), dtype=torch.float32, device=dev),
                   lp=torch.empty(n, dtype=torch.float32, device=dev),
                   kappa=torch.empty(n, dtype=torch.float32, device=dev))
    ws = _workspace(rz_workspace_bytes_loss(n, R, n_groups, d, V), workspace, dev)
    code = lib().rz_loss_fwd_bwd_host_io(_ptr(H_host), _ptr(H_dev), _ptr(W_head), _ptr(token_ids), _ptr(lp_rollout),
                                         _ptr(rewards), _ptr(seg_offsets), _ptr(group_ids), n, R, n_groups, d, V, opt,
                                         _ptr(out["loss"]), _ptr(out["dH"]), _ptr(out["dW"]), _ptr(out.get("lp")),
                                         _ptr(out.get("kappa")), _ptr(dH_host), _ptr(dW_host), _ptr(ws), ws.numel(),
                                         _stream_handle(stream))
    _check(code, "rz_loss_fwd_bwd_host_io")
    out["workspace"] = ws
    out["dH_host"], out["dW_host"] = dH_host, dW_host
    return out


@_on_tensor_device
def rz_segment_loss_ex(lp, lp_rollout, rewards, seg_offsets, group_ids, n_groups, options, want_w=False,
                       workspace=None, stream=None):
    """rz_segment_loss with rz_loss_options.  Returns dict(loss, kappa, w, workspace)."""
    torch = _torch()
    n, dev = _token_vector(lp, "lp")
    R = _segments(lp_rollout, rewards, seg_offsets, group_ids, n, dev)
    opt = _options_ref(options, n, dev)
    loss = torch.empty(1, dtype=torch.float32, device=dev)
    kappa = torch.empty(n, dtype=torch.float32, device=dev)
    w = torch.empty(n, dtype=torch.float32, device=dev) if want_w else None
    ws = _workspace(rz_workspace_bytes_segment_loss(n, R, n_groups), workspace, dev)
    code = lib().rz_segment_loss_ex(_ptr(lp), _ptr(lp_rollout), _ptr(rewards), _ptr(seg_offsets), _ptr(group_ids), n,
                                    R, n_groups, opt, _ptr(loss),
                                    _ptr(kappa), _ptr(w), _ptr(ws), ws.numel(), _stream_handle(stream))
    _check(code, "rz_segment_loss_ex")
    return dict(loss=loss, kappa=kappa, w=w, workspace=ws)


@_on_tensor_device
def rz_ratio_stats(lp, lp_rollout, seg_offsets, token_mask=None, want_resp_mean=True, workspace=None, stream=None):
    """Ratio diagnostics.  Returns (stats tensor [9] fp64 on device, per-response mean ratio or None)."""
    torch = _torch()
    n, dev = _token_vector(lp, "lp")
    _need_shaped(lp_rollout, torch.float32, "lp_rollout", dev, (n,))
    _need(seg_offsets, torch.int64, "seg_offsets", dev)
    if seg_offsets.dim() != 1 or seg_offsets.shape[0] < 1:
        raise ValueError("seg_offsets must be 1-D [n_resp + 1]")
    _need_shaped(token_mask, torch.uint8, "token_mask", dev, (n,))
    R = seg_offsets.shape[0] - 1
    stats = torch.empty(9, dtype=torch.float64, device=dev)
    rm = torch.empty(R, dtype=torch.float32, device=dev) if want_resp_mean else None
    ws = _workspace(rz_workspace_bytes_ratio_stats(n, R), workspace, dev)
    code = lib().rz_ratio_stats(_ptr(lp), _ptr(lp_rollout), _ptr(seg_offsets), n, R, _ptr(token_mask), _ptr(stats),
                                _ptr(rm), _ptr(ws), ws.numel(), _stream_handle(stream))
    _check(code, "rz_ratio_stats")
    return stats, rm


@_on_tensor_device
def rz_grad_norms(dH, dW, workspace=None, stream=None):
    """(||dH||, ||dW||) as an fp64 device tensor [2]."""
    torch = _torch()
    n, d = _matrix(dH, torch.bfloat16, "dH")
    dev = dH.device
    V, dw = _matrix(dW, torch.float32, "dW", dev)
    if dw != d:
        raise ValueError(f"dW has d = {dw}, dH has d = {d}")
    out = torch.empty(2, dtype=torch.float64, device=dev)
    ws = _workspace(rz_workspace_bytes_grad_norms(), workspace, dev)
    code = lib().rz_grad_norms(_ptr(dH), _ptr(dW), n, d, V, _ptr(out), _ptr(ws), ws.numel(), _stream_handle(stream))
    _check(code, "rz_grad_norms")
    return out


@_on_tensor_device
def rz_quantize_rows_e4m3(X, stream=None):
    """bf16 [rows, d] -> (e4m3 codes as uint8 [rows, d], fp32 per-row scales [rows])."""
    torch = _torch()
    rows, d = _matrix(X, torch.bfloat16, "X")
    q = torch.empty((rows, d), dtype=torch.uint8, device=X.device)
    sc = torch.empty(rows, dtype=torch.float32, device=X.device)
    _check(lib().rz_quantize_rows_e4m3(_ptr(X), rows, d, _ptr(q), _ptr(sc), _stream_handle(stream)),
           "rz_quantize_rows_e4m3")
    return q, sc


@_on_tensor_device
def rz_token_logprobs_fp8(H8, h_scale, W8, w_scale, token_ids, lp_out=None, lse_out=None, workspace=None,
                          stream=None, want_lse=True):
    """Token logprobs from e4m3 operands with per-row scales.  Returns (lp, lse)."""
    torch = _torch()
    n, d = _matrix(H8, torch.uint8, "H8")
    dev = H8.device
    V, dw = _matrix(W8, torch.uint8, "W8", dev)
    if dw != d:
        raise ValueError(f"W8 has d = {dw}, H8 has d = {d}")
    _need_shaped(h_scale, torch.float32, "h_scale", dev, (n,))
    _need_shaped(w_scale, torch.float32, "w_scale", dev, (V,))
    _need_shaped(token_ids, torch.int32, "token_ids", dev, (n,))
    _need_shaped(lp_out, torch.float32, "lp_out", dev, (n,))
    _need_shaped(lse_out, torch.float32, "lse_out", dev, (n,))
    lp = lp_out if lp_out is not None else torch.empty(n, dtype=torch.float32, device=dev)
    lse = lse_out if lse_out is not None else (torch.empty(n, dtype=torch.float32, device=dev) if want_lse else None)
    ws = _workspace(rz_workspace_bytes_logprobs(n, d, V), workspace, dev)
    code = lib().rz_token_logprobs_fp8(_ptr(H8), _ptr(h_scale), _ptr(W8), _ptr(w_scale), _ptr(token_ids), n, d, V,
                                       _ptr(lp), _ptr(lse), _ptr(ws), ws.numel(), _stream_handle(stream))
    _check(code, "rz_token_logprobs_fp8")
    return lp, lse


def rz_mxfp4_scale_bytes(rows: int, d: int) -> int:
    return int(lib().rz_mxfp4_scale_bytes(rows, d))


@_on_tensor_device
def rz_quantize_rows_mxfp4(X, stream=None):
    """bf16 [rows, d] -> (packed E2M1 codes uint8 [rows, d/2], tiled UE8M0 scales uint8
    [rz_mxfp4_scale_bytes(rows, d)]); the layouts are those of include/rz.h."""
    torch = _torch()
    rows, d = _matrix(X, torch.bfloat16, "X")
    nbytes = rz_mxfp4_scale_bytes(rows, d)
    if nbytes == 0 and rows > 0:
        raise ValueError(f"d = {d} is not supported (a multiple of 256 up to 32768)")
    q = torch.empty((rows, d // 2), dtype=torch.uint8, device=X.device)
    sc = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=X.device)
    _check(lib().rz_quantize_rows_mxfp4(_ptr(X), rows, d, _ptr(q), _ptr(sc), _stream_handle(stream)),
           "rz_quantize_rows_mxfp4")
    return q, sc


@_on_tensor_device
def rz_token_logprobs_mxfp4(H4, h_scales, W4, w_scales, token_ids, lp_out=None, lse_out=None, workspace=None,
                            stream=None, want_lse=True):
    """Token logprobs from MXFP4 operands (codes [rows, d/2] and tiled scales from
    rz_quantize_rows_mxfp4).  Returns (lp, lse)."""
    torch = _torch()
    n, half = _matrix(H4, torch.uint8, "H4")
    dev = H4.device
    V, half_w = _matrix(W4, torch.uint8, "W4", dev)
    if half_w != half:
        raise ValueError(f"W4 has {half_w} bytes per row, H4 has {half}")
    d = 2 * half
    for name, t, rows in (("h_scales", h_scales, n), ("w_scales", w_scales, V)):
        _need(t, torch.uint8, name, dev)
        if t.dim() != 1 or t.numel() < rz_mxfp4_scale_bytes(rows, d):
            raise ValueError(f"{name} must be 1-D with at least rz_mxfp4_scale_bytes({rows}, {d}) bytes")
    _need_shaped(token_ids, torch.int32, "token_ids", dev, (n,))
    _need_shaped(lp_out, torch.float32, "lp_out", dev, (n,))
    _need_shaped(lse_out, torch.float32, "lse_out", dev, (n,))
    lp = lp_out if lp_out is not None else torch.empty(n, dtype=torch.float32, device=dev)
    lse = lse_out if lse_out is not None else (torch.empty(n, dtype=torch.float32, device=dev) if want_lse else None)
    ws = _workspace(rz_workspace_bytes_logprobs(n, d, V), workspace, dev)
    code = lib().rz_token_logprobs_mxfp4(_ptr(H4), _ptr(h_scales), _ptr(W4), _ptr(w_scales), _ptr(token_ids), n, d,
                                         V, _ptr(lp), _ptr(lse), _ptr(ws), ws.numel(), _stream_handle(stream))
    _check(code, "rz_token_logprobs_mxfp4")
    return lp, lse


@_on_tensor_device
def rz_sum_shards_f32(stacked, out=None, stream=None):
    """Rank-order sum of the rows of a [nshards, count] fp32 CUDA tensor (fp64 accumulation)."""
    torch = _torch()
    nshards, count = _matrix(stacked, torch.float32, "stacked")
    _need_shaped(out, torch.float32, "out", stacked.device, (count,))
    out = out if out is not None else torch.empty(count, dtype=torch.float32, device=stacked.device)
    _check(lib().rz_sum_shards_f32(_ptr(stacked), nshards, count, _ptr(out), _stream_handle(stream)),
           "rz_sum_shards_f32")
    return out


def rz_selftest_wait_timeout(limit_ns: int, stream=None):
    """Run the bounded-wait self-test; returns (status code, status bits, waited ns)."""
    torch = _torch()
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    waited = ctypes.c_uint64(0)
    _check(lib().rz_selftest_wait_timeout(limit_ns, _ptr(ws), ws.numel(), ctypes.byref(waited),
                                          _stream_handle(stream)), "rz_selftest_wait_timeout")
    code, bits = rz_read_device_status(ws, stream)
    return code, bits, int(waited.value)


@_on_tensor_device
def rz_selftest_forward_after_timeout(H, W_head, token_ids, use_noalloc_scratch=False, stream=None):
    """Run the forward (with a workspace, or from the allocation-free scratch) with one wait
    that gives up enqueued before its kernels.  Returns (lp, lse, status code, status bits);
    the status is that of the workspace (0, 0 for the scratch, whose status is internal)."""
    torch = _torch()
    n, d = _matrix(H, torch.bfloat16, "H")
    dev = H.device
    V, dw = _matrix(W_head, torch.bfloat16, "W_head", dev)
    if dw != d:
        raise ValueError(f"W_head has d = {dw}, H has d = {d}")
    _need_shaped(token_ids, torch.int32, "token_ids", dev, (n,))
    lp = torch.empty(n, dtype=torch.float32, device=dev)
    lse = torch.empty(n, dtype=torch.float32, device=dev)
    ws = None if use_noalloc_scratch else _workspace(rz_workspace_bytes_logprobs(n, d, V), None, dev)
    code = lib().rz_selftest_forward_after_timeout(1 if use_noalloc_scratch else 0, _ptr(H), _ptr(W_head),
                                                   _ptr(token_ids), n, d, V, _ptr(lp), _ptr(lse), _ptr(ws),
                                                   0 if ws is None else ws.numel(), _stream_handle(stream))
    _check(code, "rz_selftest_forward_after_timeout")
    status = (0, 0) if ws is None else rz_read_device_status(ws, stream)
    return lp, lse, status[0], status[1]
