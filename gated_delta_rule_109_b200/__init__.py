"""Python binding of libkda, the B200 Kimi Delta Attention forward library.

Argument marshalling only: every step of the computation runs in libkda's CUDA
kernels (``csrc/``), reached through its C ABI (``include/kda.h``).  PyTorch
supplies device memory and the current stream.  There is no fallback: if the
library is not built, every call raises.

    import gated_delta_rule_109_b200 as kda
    out, final_state = kda.forward(q, k, v, log_alpha, beta, initial_state)
    out = kda.decode_step(q, k, v, log_alpha, beta, state)   # state updated in place
    # scalar-gate variants: Gated DeltaNet (log_alpha [B,T,H]) and DeltaNet (None)
    out, final_state = kda.gdn_forward(q, k, v, g, beta, initial_state)
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libkda.so")

KDA_OK, KDA_ERR_INVALID_ARG, KDA_ERR_UNSUPPORTED, KDA_ERR_MISALIGNED, KDA_ERR_CUDA, KDA_ERR_TIMEOUT = range(6)
KDA_BF16, KDA_F32 = 0, 1
KDA_PREP_LOGSIGMOID_GATE, KDA_PREP_L2NORM_QK = 1, 2

# every symbol include/kda.h declares
EXPORTS = ("kda_forward", "kda_forward_ws", "kda_forward_workspace_bytes",
           "kda_forward_workspace_min_bytes", "kda_segment_workspace_bytes", "kda_forward_raw", "kda_segment_local",
           "kda_segment_start_state", "kda_segment_correct", "kda_forward_noalloc",
           "kda_forward_noalloc_scratch_bytes", "kda_workspace_pool_bytes", "kda_workspace_pool_trim",
           "kda_forward_host", "kda_forward_host_workspace_bytes",
           "kda_backward", "kda_backward_workspace_bytes",
           "kda_decode_step", "kda_gdn_forward", "kda_gdn_forward_ws", "kda_gdn_decode_step",
           "kda_status_string", "kda_check_status", "kda_selftest_timeout", "kda_last_cuda_error",
           "kda_launch_count",
           "kda_version")

_lib = None


class KDAError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str = ""):
        self.status = status
        msg = "%s returned %s" % (where, status_string(status) if _lib else str(status))
        if detail:
            msg += " (%s)" % detail
        super().__init__(msg)


def load(path: Optional[str] = None) -> ctypes.CDLL:
    """Load libkda.so (built in-tree by ``gated_delta_rule_109_b200.build``)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise RuntimeError("libkda.so is not built (%s); run `python -m gated_delta_rule_109_b200.build`" % p)
    lib = ctypes.CDLL(p)
    vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.kda_forward.restype = i
    lib.kda_forward.argtypes = [vp] * 8 + [i] * 6 + [f, vp]
    lib.kda_decode_step.restype = i
    lib.kda_decode_step.argtypes = [vp] * 7 + [i] * 5 + [f, vp]
    lib.kda_forward_ws.restype = i
    lib.kda_forward_ws.argtypes = [vp] * 8 + [i] * 6 + [f, vp, ctypes.c_size_t, vp]
    lib.kda_gdn_forward_ws.restype = i
    lib.kda_gdn_forward_ws.argtypes = [vp] * 8 + [i] * 6 + [f, vp, ctypes.c_size_t, vp]
    for name in ("kda_forward_workspace_bytes", "kda_forward_workspace_min_bytes", "kda_segment_workspace_bytes"):
        getattr(lib, name).restype = ctypes.c_size_t
        getattr(lib, name).argtypes = [i] * 6
    lib.kda_forward_raw.restype = i
    lib.kda_forward_raw.argtypes = [vp] * 8 + [i] * 6 + [f, ctypes.c_uint, vp, ctypes.c_size_t, vp]
    lib.kda_segment_local.restype = i
    lib.kda_segment_local.argtypes = [vp] * 9 + [i] * 6 + [f, vp, ctypes.c_size_t, vp]
    lib.kda_segment_start_state.restype = i
    lib.kda_segment_start_state.argtypes = [vp, vp, i, vp, i, i, i, i, vp]
    lib.kda_segment_correct.restype = i
    lib.kda_segment_correct.argtypes = [vp] * 4 + [i] * 5 + [vp, ctypes.c_size_t, vp]
    lib.kda_forward_noalloc.restype = i
    lib.kda_forward_noalloc.argtypes = [vp] * 8 + [i] * 6 + [f, vp]
    lib.kda_forward_noalloc_scratch_bytes.restype = ctypes.c_size_t
    lib.kda_forward_host.restype = i
    lib.kda_forward_host.argtypes = [vp] * 8 + [i] * 6 + [f, i, vp, ctypes.c_size_t, vp]
    lib.kda_forward_host_workspace_bytes.restype = ctypes.c_size_t
    lib.kda_forward_host_workspace_bytes.argtypes = [i] * 7
    lib.kda_backward.restype = i
    lib.kda_backward.argtypes = [vp] * 14 + [i] * 6 + [f, vp, ctypes.c_size_t, vp]
    lib.kda_backward_workspace_bytes.restype = ctypes.c_size_t
    lib.kda_backward_workspace_bytes.argtypes = [i] * 5
    lib.kda_forward_noalloc_scratch_bytes.argtypes = []
    lib.kda_workspace_pool_bytes.restype = ctypes.c_size_t
    lib.kda_workspace_pool_bytes.argtypes = []
    lib.kda_workspace_pool_trim.restype = i
    lib.kda_workspace_pool_trim.argtypes = [vp]
    lib.kda_gdn_forward.restype = i
    lib.kda_gdn_forward.argtypes = [vp] * 8 + [i] * 6 + [f, vp]
    lib.kda_gdn_decode_step.restype = i
    lib.kda_gdn_decode_step.argtypes = [vp] * 7 + [i] * 5 + [f, vp]
    lib.kda_status_string.restype = ctypes.c_char_p
    lib.kda_status_string.argtypes = [i]
    lib.kda_check_status.restype = i
    lib.kda_check_status.argtypes = [vp]
    lib.kda_selftest_timeout.restype = i
    lib.kda_selftest_timeout.argtypes = [ctypes.c_uint, vp]
    lib.kda_last_cuda_error.restype = ctypes.c_char_p
    lib.kda_last_cuda_error.argtypes = []
    lib.kda_launch_count.restype = ctypes.c_ulonglong
    lib.kda_launch_count.argtypes = []
    lib.kda_version.restype = i
    lib.kda_version.argtypes = []
    if path is None:
        _lib = lib
    return lib


def status_string(status: int) -> str:
    return load().kda_status_string(int(status)).decode()


def _check(status: int, where: str):
    if status != KDA_OK:
        detail = load().kda_last_cuda_error().decode() if status == KDA_ERR_CUDA else ""
        raise KDAError(status, where, detail)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return KDA_BF16
    if t.dtype == torch.float32:
        return KDA_F32
    raise TypeError("q, k, v must be bfloat16 or float32, got %s" % t.dtype)


def _need(t: torch.Tensor, name: str, shape, dtype=None, device=None):
    if tuple(t.shape) != tuple(shape):
        raise ValueError("%s has shape %s, expected %s" % (name, tuple(t.shape), tuple(shape)))
    if dtype is not None and t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if device is not None and t.device != device:
        raise ValueError("%s is on %s, expected %s" % (name, t.device, device))


def _on_cuda(dev: torch.device, where: str):
    """The kernels take device memory only: a host tensor is refused here, before
    its address could reach a kernel."""
    if dev.type != "cuda":
        raise ValueError("%s takes CUDA tensors, got tensors on %s" % (where, dev))


def _need_workspace(workspace, dev: torch.device, where: str):
    """A caller's workspace: a contiguous CUDA tensor on the device the call runs on."""
    if not isinstance(workspace, torch.Tensor):
        raise TypeError("%s: workspace must be a torch.Tensor" % where)
    if workspace.device.type != "cuda" or not workspace.is_contiguous():
        raise ValueError("%s: workspace must be a contiguous CUDA tensor, got one on %s" % (where, workspace.device))
    want = dev.index if dev.index is not None else torch.cuda.current_device()
    if workspace.device.index != want:
        raise ValueError("%s: workspace is on %s, the call runs on cuda:%d" % (where, workspace.device, want))


def _forward(entry, gate_shape, q, k, v, log_alpha, beta, initial_state, out, final_state,
             return_final_state, scale, workspace=None, one_kernel=False):
    lib = load()
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    _on_cuda(dev, entry)
    code = _dtype_code(q)
    _need(q, "q", (B, T, H, dk), q.dtype, dev)
    _need(k, "k", (B, T, H, dk), q.dtype, dev)
    _need(v, "v", (B, T, H, dv), q.dtype, dev)
    if log_alpha is not None or gate_shape is not None:
        _need(log_alpha, "log_alpha", gate_shape(B, T, H, dk), torch.float32, dev)
    _need(beta, "beta", (B, T, H), torch.float32, dev)
    if initial_state is not None:
        _need(initial_state, "initial_state", (B, H, dk, dv), torch.float32, dev)
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=torch.float32, device=dev)
    _need(out, "out", (B, T, H, dv), torch.float32, dev)
    if final_state is None and return_final_state:
        final_state = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    if final_state is not None:
        _need(final_state, "final_state", (B, H, dk, dv), torch.float32, dev)
    if workspace is not None and one_kernel:
        raise ValueError("%s: one_kernel takes no workspace" % entry)
    if workspace is not None or one_kernel:
        if workspace is not None:
            _need_workspace(workspace, dev, entry)
        entry = entry + "_ws"
        st = getattr(lib, entry)(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
                                 _ptr(initial_state), _ptr(out), _ptr(final_state),
                                 B, T, H, dk, dv, code, float(scale), _ptr(workspace),
                                 0 if workspace is None else workspace.numel() * workspace.element_size(),
                                 _stream(dev))
    else:
        fn = getattr(lib, entry)
        st = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
                _ptr(initial_state), _ptr(out), _ptr(final_state),
                B, T, H, dk, dv, code, float(scale), _stream(dev))
    _check(st, entry)
    return out, final_state


def _decode(entry, gate_shape, q, k, v, log_alpha, beta, state, out, scale):
    lib = load()
    B, H, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    _on_cuda(dev, entry)
    code = _dtype_code(q)
    _need(q, "q", (B, H, dk), q.dtype, dev)
    _need(k, "k", (B, H, dk), q.dtype, dev)
    _need(v, "v", (B, H, dv), q.dtype, dev)
    if log_alpha is not None or gate_shape is not None:
        _need(log_alpha, "log_alpha", gate_shape(B, H, dk), torch.float32, dev)
    _need(beta, "beta", (B, H), torch.float32, dev)
    _need(state, "state", (B, H, dk, dv), torch.float32, dev)
    if out is None:
        out = torch.empty((B, H, dv), dtype=torch.float32, device=dev)
    _need(out, "out", (B, H, dv), torch.float32, dev)
    fn = getattr(lib, entry)
    st = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta),
            _ptr(state), _ptr(out), B, H, dk, dv, code, float(scale), _stream(dev))
    _check(st, entry)
    return out


def forward(q, k, v, log_alpha, beta, initial_state=None, *, out=None, final_state=None,
            return_final_state=True, scale: float = 0.0, workspace=None, one_kernel=False):
    """Chunked KDA prefill (``kda_forward``, or ``kda_forward_ws`` with a workspace).

    q, k ``[B,T,H,dk]`` and v ``[B,T,H,dv]`` (bf16 or fp32, one dtype);
    log_alpha ``[B,T,H,dk]`` fp32; beta ``[B,T,H]`` fp32; initial_state
    ``[B,H,dk,dv]`` fp32 or None.  Returns ``(out [B,T,H,dv] fp32,
    final_state [B,H,dk,dv] fp32 or None)``.  ``final_state`` may be passed as
    the same tensor as ``initial_state`` to carry the state in place.
    ``scale`` 0 means 1/sqrt(dk).  ``workspace``: a contiguous device tensor
    (see :func:`workspace_bytes` / :func:`make_workspace`) for the two-kernel
    prefill (bf16 inputs, dk = dv = 128); without one, ``kda_forward`` takes it
    from the library's pool.  ``one_kernel``: ``kda_forward_ws`` with no
    workspace, the one-kernel prefill that needs no memory beyond its arguments.
    """
    return _forward("kda_forward", lambda B, T, H, dk: (B, T, H, dk), q, k, v, log_alpha, beta,
                    initial_state, out, final_state, return_final_state, scale, workspace, one_kernel)


def forward_raw(q, k, v, gate, beta, initial_state=None, *, workspace, logsigmoid_gate=True,
                normalize_qk=True, out=None, final_state=None, return_final_state=True, scale: float = 0.0):
    """Prefill on raw activations (``kda_forward_raw``): with ``logsigmoid_gate``
    the gate ``[B,T,H,dk]`` holds pre-activations x and log alpha = log sigmoid(x);
    with ``normalize_qk`` q and k rows are L2-normalised.  Both run inside the
    two-kernel prefill (bf16, dk = dv = 128), which needs ``workspace``."""
    lib = load()
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    _on_cuda(dev, "kda_forward_raw")
    code = _dtype_code(q)
    _need(q, "q", (B, T, H, dk), q.dtype, dev)
    _need(k, "k", (B, T, H, dk), q.dtype, dev)
    _need(v, "v", (B, T, H, dv), q.dtype, dev)
    _need(gate, "gate", (B, T, H, dk), torch.float32, dev)
    _need(beta, "beta", (B, T, H), torch.float32, dev)
    if initial_state is not None:
        _need(initial_state, "initial_state", (B, H, dk, dv), torch.float32, dev)
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=torch.float32, device=dev)
    _need(out, "out", (B, T, H, dv), torch.float32, dev)
    if final_state is None and return_final_state:
        final_state = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    if final_state is not None:
        _need(final_state, "final_state", (B, H, dk, dv), torch.float32, dev)
    if workspace is None:
        raise ValueError("kda_forward_raw needs a workspace")
    _need_workspace(workspace, dev, "kda_forward_raw")
    prep = (KDA_PREP_LOGSIGMOID_GATE if logsigmoid_gate else 0) | (KDA_PREP_L2NORM_QK if normalize_qk else 0)
    st = lib.kda_forward_raw(_ptr(q), _ptr(k), _ptr(v), _ptr(gate), _ptr(beta), _ptr(initial_state), _ptr(out),
                             _ptr(final_state), B, T, H, dk, dv, code, float(scale), prep, _ptr(workspace),
                             workspace.numel() * workspace.element_size(), _stream(dev))
    _check(st, "kda_forward_raw")
    return out, final_state


def segment_local(q, k, v, log_alpha, beta, initial_state=None, *, workspace, scale: float = 0.0):
    """Phase 1 of a time-axis split (``kda_segment_local``): returns
    ``(out, local_final, transfer)`` of one contiguous segment of a sequence."""
    lib = load()
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    _on_cuda(dev, "kda_segment_local")
    _need_workspace(workspace, dev, "kda_segment_local")
    code = _dtype_code(q)
    for t, n, shp in ((q, "q", (B, T, H, dk)), (k, "k", (B, T, H, dk)), (v, "v", (B, T, H, dv))):
        _need(t, n, shp, q.dtype, dev)
    _need(log_alpha, "log_alpha", (B, T, H, dk), torch.float32, dev)
    _need(beta, "beta", (B, T, H), torch.float32, dev)
    if initial_state is not None:
        _need(initial_state, "initial_state", (B, H, dk, dv), torch.float32, dev)
    out = torch.empty((B, T, H, dv), dtype=torch.float32, device=dev)
    local_final = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    transfer = torch.empty((B, H, dk, dk), dtype=torch.float32, device=dev)
    st = lib.kda_segment_local(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(initial_state),
                               _ptr(out), _ptr(local_final), _ptr(transfer), B, T, H, dk, dv, code, float(scale),
                               _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(dev))
    _check(st, "kda_segment_local")
    return out, local_final, transfer


def segment_start_state(transfers, local_finals):
    """The state entering the next segment (``kda_segment_start_state``) from the
    stacked ``[R, B, H, dk, dk]`` transfers and ``[R, B, H, dk, dv]`` local finals
    of the earlier segments."""
    R, B, H, dk, _ = transfers.shape
    dv = local_finals.shape[-1]
    dev = transfers.device
    _on_cuda(dev, "kda_segment_start_state")
    _need(transfers, "transfers", (R, B, H, dk, dk), torch.float32, dev)
    _need(local_finals, "local_finals", (R, B, H, dk, dv), torch.float32, dev)
    start = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    st = load().kda_segment_start_state(_ptr(transfers), _ptr(local_finals), R, _ptr(start), B, H, dk, dv,
                                        _stream(dev))
    _check(st, "kda_segment_start_state")
    return start


def segment_correct(start, local_final, out, *, workspace, final_state=None):
    """Phase 3 (``kda_segment_correct``): ``out`` += the start state's outputs;
    returns ``final_state`` (= local_final + the propagated start)."""
    B, T, H, dv = out.shape
    dk = start.shape[-2]
    dev = out.device
    _on_cuda(dev, "kda_segment_correct")
    _need_workspace(workspace, dev, "kda_segment_correct")
    _need(start, "start", (B, H, dk, dv), torch.float32, dev)
    _need(local_final, "local_final", (B, H, dk, dv), torch.float32, dev)
    _need(out, "out", (B, T, H, dv), torch.float32, dev)
    if final_state is None:
        final_state = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    st = load().kda_segment_correct(_ptr(start), _ptr(local_final), _ptr(out), _ptr(final_state), B, T, H, dk, dv,
                                    _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(dev))
    _check(st, "kda_segment_correct")
    return final_state


def forward_host_workspace_bytes(B, T, H, dk, dv, dtype=torch.bfloat16, block_tokens: int = 0) -> int:
    """Bytes of the device workspace ``kda_forward_host`` needs."""
    code = KDA_BF16 if dtype == torch.bfloat16 else KDA_F32
    return int(load().kda_forward_host_workspace_bytes(B, T, H, dk, dv, code, int(block_tokens)))


def forward_host(q, k, v, log_alpha, beta, initial_state=None, *, out=None, final_state=None,
                 return_final_state=True, block_tokens: int = 0, workspace=None, device=None,
                 scale: float = 0.0, synchronize: bool = True):
    """Prefill with host tensors in and out (``kda_forward_host``): copies and
    kernels overlap block by block.  ``q, k, v, log_alpha, beta`` (and
    ``initial_state``) are CPU tensors in the usual layouts (pinned memory for
    asynchronous copies); ``out`` / ``final_state`` (CPU, fp32) are allocated
    pinned when None.  ``workspace``: a uint8 tensor on ``device`` of at least
    :func:`forward_host_workspace_bytes` bytes (allocated when None).  With
    ``synchronize`` the call waits for the device stream before returning."""
    lib = load()
    dev = torch.device("cuda") if device is None else torch.device(device)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    cpu = torch.device("cpu")
    for t, n, shp, dt in ((q, "q", (B, T, H, dk), q.dtype), (k, "k", (B, T, H, dk), q.dtype),
                          (v, "v", (B, T, H, dv), q.dtype), (log_alpha, "log_alpha", (B, T, H, dk), torch.float32),
                          (beta, "beta", (B, T, H), torch.float32)):
        _need(t, n, shp, dt, cpu)
    if initial_state is not None:
        _need(initial_state, "initial_state", (B, H, dk, dv), torch.float32, cpu)
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=torch.float32, pin_memory=True)
    _need(out, "out", (B, T, H, dv), torch.float32, cpu)
    if final_state is None and return_final_state:
        final_state = torch.empty((B, H, dk, dv), dtype=torch.float32, pin_memory=True)
    if final_state is not None:
        _need(final_state, "final_state", (B, H, dk, dv), torch.float32, cpu)
    _on_cuda(dev, "kda_forward_host")
    nbytes = forward_host_workspace_bytes(B, T, H, dk, dv, q.dtype, block_tokens)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=dev)
    _need_workspace(workspace, dev, "kda_forward_host")
    st = lib.kda_forward_host(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(initial_state),
                              _ptr(out), _ptr(final_state), B, T, H, dk, dv, _dtype_code(q), float(scale),
                              int(block_tokens), _ptr(workspace), workspace.numel() * workspace.element_size(),
                              _stream(dev))
    _check(st, "kda_forward_host")
    if synchronize:
        torch.cuda.current_stream(dev).synchronize()
    return out, final_state


def backward_workspace_bytes(B: int, T: int, H: int, dk: int, dv: int) -> int:
    """Bytes of the workspace ``kda_backward`` needs (0: unsupported shape)."""
    return int(load().kda_backward_workspace_bytes(B, T, H, dk, dv))


def backward(q, k, v, log_alpha, beta, grad_out, initial_state=None, grad_final_state=None, *,
             workspace=None, scale: float = 0.0, initial_state_grad: bool = True):
    """Gradients of :func:`forward` (``kda_backward``).

    ``grad_out`` [B,T,H,dv] and ``grad_final_state`` [B,H,dk,dv] (None: zero) are
    the cotangents of the outputs and of the final state.  Returns a dict of fp32
    tensors ``dq, dk, dv, dlog_alpha, dbeta`` and ``dinitial_state`` (None unless
    ``initial_state_grad``).  ``workspace``: a uint8 device tensor of at least
    :func:`backward_workspace_bytes` bytes (allocated here when None).
    """
    lib = load()
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    _on_cuda(dev, "kda_backward")
    for t, n, shp in ((q, "q", (B, T, H, dk)), (k, "k", (B, T, H, dk)), (v, "v", (B, T, H, dv))):
        _need(t, n, shp, q.dtype, dev)
    _need(log_alpha, "log_alpha", (B, T, H, dk), torch.float32, dev)
    _need(beta, "beta", (B, T, H), torch.float32, dev)
    _need(grad_out, "grad_out", (B, T, H, dv), torch.float32, dev)
    if initial_state is not None:
        _need(initial_state, "initial_state", (B, H, dk, dv), torch.float32, dev)
    if grad_final_state is not None:
        _need(grad_final_state, "grad_final_state", (B, H, dk, dv), torch.float32, dev)
    nbytes = backward_workspace_bytes(B, T, H, dk, dv)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=dev)
    _need_workspace(workspace, dev, "kda_backward")
    f32 = dict(dtype=torch.float32, device=dev)
    g = dict(dq=torch.empty((B, T, H, dk), **f32), dk=torch.empty((B, T, H, dk), **f32),
             dv=torch.empty((B, T, H, dv), **f32), dlog_alpha=torch.empty((B, T, H, dk), **f32),
             dbeta=torch.empty((B, T, H), **f32),
             dinitial_state=torch.empty((B, H, dk, dv), **f32) if initial_state_grad else None)
    st = lib.kda_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(beta), _ptr(initial_state),
                          _ptr(grad_out), _ptr(grad_final_state), _ptr(g["dq"]), _ptr(g["dk"]), _ptr(g["dv"]),
                          _ptr(g["dlog_alpha"]), _ptr(g["dbeta"]), _ptr(g["dinitial_state"]),
                          B, T, H, dk, dv, _dtype_code(q), float(scale), _ptr(workspace),
                          workspace.numel() * workspace.element_size(), _stream(dev))
    _check(st, "kda_backward")
    return g


class KDAFunction(torch.autograd.Function):
    """``out, final_state = KDAFunction.apply(q, k, v, log_alpha, beta, initial_state)``
    with ``kda_forward`` forward and ``kda_backward`` backward (gradients in fp32,
    cast to each input's dtype)."""

    @staticmethod
    def forward(ctx, q, k, v, log_alpha, beta, initial_state):
        out, final_state = forward(q, k, v, log_alpha, beta, initial_state)
        ctx.save_for_backward(q, k, v, log_alpha, beta, initial_state)
        return out, final_state

    @staticmethod
    def backward(ctx, grad_out, grad_final_state):
        q, k, v, log_alpha, beta, initial_state = ctx.saved_tensors
        g = backward(q, k, v, log_alpha, beta, grad_out.contiguous().float(),
                     initial_state, None if grad_final_state is None else grad_final_state.contiguous().float(),
                     initial_state_grad=initial_state is not None)
        return (g["dq"].to(q.dtype), g["dk"].to(k.dtype), g["dv"].to(v.dtype), g["dlog_alpha"], g["dbeta"],
                g["dinitial_state"])


def forward_noalloc(q, k, v, log_alpha, beta, initial_state=None, *, out=None, final_state=None,
                    return_final_state=True, scale: float = 0.0):
    """:func:`forward` through ``kda_forward_noalloc``: the two-kernel prefill on
    scratch owned by the library (no workspace argument, nothing allocated)."""
    return _forward("kda_forward_noalloc", lambda B, T, H, dk: (B, T, H, dk), q, k, v, log_alpha, beta,
                    initial_state, out, final_state, return_final_state, scale)


def noalloc_scratch_bytes() -> int:
    return int(load().kda_forward_noalloc_scratch_bytes())


def workspace_pool_bytes(device=None) -> int:
    """Device memory held by the workspace pool of ``kda_forward`` on ``device``
    (``kda_workspace_pool_bytes``)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    _on_cuda(dev, "kda_workspace_pool_bytes")
    with torch.cuda.device(dev):
        return int(load().kda_workspace_pool_bytes())


def workspace_pool_trim(device=None):
    """Return the pool's unused memory to the device (``kda_workspace_pool_trim``),
    after the work enqueued on the current stream."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    _on_cuda(dev, "kda_workspace_pool_trim")
    with torch.cuda.device(dev):
        _check(load().kda_workspace_pool_trim(_stream(dev)), "kda_workspace_pool_trim")


def workspace_bytes(B, T, H, dk, dv, dtype=torch.bfloat16, minimum=False, segment=False) -> int:
    """Workspace size for :func:`forward` (``kda_forward_workspace_bytes`` /
    ``..._min_bytes``), or with ``segment`` for :func:`segment_local` and
    :func:`segment_correct` (``kda_segment_workspace_bytes``); 0 when the
    two-kernel prefill does not apply."""
    code = KDA_BF16 if dtype == torch.bfloat16 else KDA_F32
    lib = load()
    fn = (lib.kda_segment_workspace_bytes if segment else
          lib.kda_forward_workspace_min_bytes if minimum else lib.kda_forward_workspace_bytes)
    return int(fn(int(B), int(T), int(H), int(dk), int(dv), code))


def make_workspace(B, T, H, dk, dv, dtype=torch.bfloat16, device="cuda", nbytes=None, segment=False):
    """A workspace tensor of ``workspace_bytes(...)`` bytes (or ``nbytes``), or None if not needed."""
    n = workspace_bytes(B, T, H, dk, dv, dtype, segment=segment) if nbytes is None else int(nbytes)
    if n == 0:
        return None
    return torch.empty(n, dtype=torch.uint8, device=device)


def decode_step(q, k, v, log_alpha, beta, state, *, out=None, scale: float = 0.0):
    """One KDA decode step (``kda_decode_step``); ``state`` is updated in place.

    q, k ``[B,H,dk]``, v ``[B,H,dv]`` (bf16 or fp32); log_alpha ``[B,H,dk]``
    fp32; beta ``[B,H]`` fp32; state ``[B,H,dk,dv]`` fp32.  Returns
    ``out [B,H,dv]`` fp32.
    """
    return _decode("kda_decode_step", lambda B, H, dk: (B, H, dk), q, k, v, log_alpha, beta, state,
                   out, scale)


def gdn_forward(q, k, v, log_alpha, beta, initial_state=None, *, out=None, final_state=None,
                return_final_state=True, scale: float = 0.0, workspace=None, one_kernel=False):
    """Chunked prefill of Gated DeltaNet / DeltaNet (``kda_gdn_forward``, or
    ``kda_gdn_forward_ws`` with a workspace).

    As :func:`forward`, with one decay per token and head: log_alpha
    ``[B,T,H]`` fp32 (<= 0), or None for DeltaNet (no decay).
    """
    shape = None if log_alpha is None else (lambda B, T, H, dk: (B, T, H))
    return _forward("kda_gdn_forward", shape, q, k, v, log_alpha, beta, initial_state, out,
                    final_state, return_final_state, scale, workspace, one_kernel)


def gdn_decode_step(q, k, v, log_alpha, beta, state, *, out=None, scale: float = 0.0):
    """One Gated DeltaNet / DeltaNet decode step (``kda_gdn_decode_step``).

    As :func:`decode_step`, with log_alpha ``[B,H]`` fp32 or None.
    """
    shape = None if log_alpha is None else (lambda B, H, dk: (B, H))
    return _decode("kda_gdn_decode_step", shape, q, k, v, log_alpha, beta, state, out, scale)


def check_status(device=None):
    """Synchronise the current stream and raise on a recorded device-side failure."""
    dev = torch.device("cuda") if device is None else torch.device(device)
    _check(load().kda_check_status(_stream(dev)), "kda_check_status")


def selftest_timeout(wait_ms: int = 50, device=None):
    """Enqueue the failure-path self-test (``kda_selftest_timeout``): a bounded
    device-side wait that gives up after ~wait_ms; the next :func:`check_status`
    raises KDAError with KDA_ERR_TIMEOUT."""
    dev = torch.device("cuda") if device is None else torch.device(device)
    _check(load().kda_selftest_timeout(int(wait_ms), _stream(dev)), "kda_selftest_timeout")


def launch_count() -> int:
    """Kernels enqueued through libkda by this process so far."""
    return int(load().kda_launch_count())


def version() -> int:
    return int(load().kda_version())
