"""Bounded-decay gated delta rule (the Kimi Delta Attention scan) on B200.

A thin ctypes binding over ``libkda.so``, whose C ABI is declared in
``include/kda.h``. Every step of the computation runs in the library's CUDA
kernels; this module only allocates outputs with torch, reads strides and
passes pointers and the current CUDA stream. There is no CPU fallback: the
functions raise if the library is missing or a tensor is not on a CUDA device.

* :func:`bounded_decay` -- ``alpha = exp(g_min * sigmoid(exp(A) * z))``
  ("Kimi K3: Bounded Decay and Delta Memory", eq. 5).
* :func:`prefill` -- the scan over whole sequences, returning ``(o, final_state)``
  (same page, eq. 1; chunkwise form of the "KDA cheat sheet", eqs. 3-4).
* :func:`decode_step` -- one token against a kept state, updated in place.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

__all__ = ["bounded_decay", "softplus_decay", "prefill", "prefill_logits", "prefill_noalloc", "scan_backward", "scan_backward_chunked", "chunked_backward_workspace_bytes", "bounded_decay_backward", "decode_step", "decode_step_logits", "prefill_workspace_bytes", "device_status", "KDAError",
           "library_path", "load_library"]

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libkda.so")

KDA_F32, KDA_BF16 = 0, 1
KDA_GATE_ALPHA, KDA_GATE_LOG = 0, 1
KDA_QK_L2NORM, KDA_BETA_LOGITS, KDA_STATE_VK, KDA_GATE_SOFTPLUS = 1, 2, 4, 8
_STATUS = {0: "KDA_OK", 1: "KDA_ERR_INVALID_ARG", 2: "KDA_ERR_UNSUPPORTED", 3: "KDA_ERR_CUDA"}


class KDAError(RuntimeError):
    """A libkda call returned a non-zero status."""

    def __init__(self, fn: str, status: int, detail: str):
        self.status = status
        super().__init__(f"{fn} failed with {_STATUS.get(status, status)}: {detail}")


class Strides(ctypes.Structure):
    _fields_ = [("b", ctypes.c_int64), ("t", ctypes.c_int64), ("h", ctypes.c_int64)]


class Layout(ctypes.Structure):
    _fields_ = [(n, Strides) for n in ("q", "k", "v", "gate", "beta", "o")]


_lib = None


def library_path() -> str:
    return _LIB_PATH


def load_library(path: Optional[str] = None) -> ctypes.CDLL:
    """Load ``libkda.so`` (built by ``python -m gated_delta_rule_bounded_b200.build``)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or _LIB_PATH
    if not os.path.exists(p):
        raise ImportError(f"{p} is missing; build it with `python -m gated_delta_rule_bounded_b200.build`")
    lib = ctypes.CDLL(p)
    vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    sp = ctypes.POINTER(Strides)
    lp = ctypes.POINTER(Layout)
    lib.kda_bounded_decay.argtypes = [vp, sp, i32, vp, ctypes.c_float, i64, i64, i64, i64, vp, sp, i32, vp]
    lib.kda_softplus_decay.argtypes = [vp, sp, i32, vp, i64, i64, i64, i64, vp, sp, i32, vp]
    lib.kda_prefill_workspace_bytes.argtypes = [i64, i64, i64, i64, i64, i64, i32, ctypes.POINTER(ctypes.c_size_t)]
    lib.kda_prefill.argtypes = [vp, vp, vp, i32, vp, i32, vp, vp, vp, vp, i64,
                                i64, i64, i64, i64, i64, lp, vp, vp, ctypes.c_size_t, vp]
    lib.kda_prefill_noalloc.argtypes = [vp, vp, vp, i32, vp, i32, vp, vp, vp, vp, i64,
                                        i64, i64, i64, i64, i64, lp, vp, vp]
    lib.kda_decode_step.argtypes = [vp, vp, vp, i32, vp, i32, vp, vp, i64, i64, i64, i64, lp, vp, vp]
    u32 = ctypes.c_uint
    lib.kda_prefill_logits.argtypes = [vp, vp, vp, i32, vp, vp, vp, ctypes.c_float, vp, u32, vp, vp, vp, i64,
                                       i64, i64, i64, i64, i64, lp, vp, vp, ctypes.c_size_t, vp]
    lib.kda_decode_step_logits.argtypes = [vp, vp, vp, i32, vp, vp, vp, ctypes.c_float, vp, u32, vp, i64, i64, i64,
                                           i64, lp, vp, vp]
    lib.kda_scan_backward_workspace_bytes.argtypes = [i64, i64, i64, i64, i64, i64, ctypes.POINTER(ctypes.c_size_t)]
    lib.kda_scan_backward.argtypes = [vp, vp, vp, i32, vp, i32, vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, i64, lp,
                                      vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
    lib.kda_bounded_decay_backward.argtypes = [vp, vp, ctypes.c_float, vp, i64, i64, i64, i64, vp, vp, vp]
    lib.kda_scan_backward_chunked_workspace_bytes.argtypes = [i64, i64, i64, i64, i64, i64,
                                                              ctypes.POINTER(ctypes.c_size_t)]
    lib.kda_scan_backward_chunked.argtypes = [vp, vp, vp, i32, vp, i32, vp, vp, vp, vp, vp, i64, i64, i64, i64, i64,
                                              i64, lp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
    lib.kda_selftest_wait_expiry.argtypes = [vp]
    for fn in ("kda_scan_backward_workspace_bytes", "kda_scan_backward", "kda_bounded_decay_backward",
               "kda_selftest_wait_expiry", "kda_scan_backward_chunked_workspace_bytes", "kda_scan_backward_chunked"):
        getattr(lib, fn).restype = ctypes.c_int
    for fn in ("kda_bounded_decay", "kda_softplus_decay", "kda_prefill_workspace_bytes", "kda_prefill", "kda_prefill_noalloc",
               "kda_decode_step", "kda_prefill_logits", "kda_decode_step_logits"):
        getattr(lib, fn).restype = ctypes.c_int
    lib.kda_last_error.restype = ctypes.c_char_p
    lib.kda_last_error.argtypes = []
    lib.kda_version.restype = ctypes.c_char_p
    lib.kda_version.argtypes = []
    lib.kda_device_status.argtypes = [ctypes.POINTER(ctypes.c_int), ctypes.c_int]
    lib.kda_device_status.restype = ctypes.c_int
    if path is None:
        _lib = lib
    return lib


def _check(fn: str, status: int):
    if status != 0:
        raise KDAError(fn, status, load_library().kda_last_error().decode())


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.float32:
        return KDA_F32
    if dt == torch.bfloat16:
        return KDA_BF16
    raise TypeError(f"unsupported dtype {dt}; use torch.bfloat16 or torch.float32")


def _cuda(t: torch.Tensor, name: str):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")


def _rowwise(t: torch.Tensor) -> torch.Tensor:
    """The innermost dim must be contiguous and rows 16-byte aligned; copy otherwise."""
    if t.dim() == 0:
        return t
    if t.stride(-1) != 1 and t.shape[-1] > 1:
        return t.contiguous()
    es = t.element_size()
    aligned = t.data_ptr() % 16 == 0 and all(
        (s * es) % 16 == 0 or n <= 1 for s, n in zip(t.stride()[:-1], t.shape[:-1]))
    return t if aligned else t.contiguous()


def _strides4(t: torch.Tensor) -> Strides:
    """B, T, H strides of a [B,T,H,D] tensor."""
    return Strides(t.stride(0), t.stride(1), t.stride(2))


def _strides3(t: torch.Tensor) -> Strides:
    """B, T, H strides of a [B,T,H] tensor."""
    return Strides(t.stride(0), t.stride(1), t.stride(2))


def _stream(device: torch.device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def bounded_decay(logits: torch.Tensor, A_log: torch.Tensor, g_min: float = -5.0, *,
                  log_decay: bool = False, out: Optional[torch.Tensor] = None,
                  _softplus: bool = False) -> torch.Tensor:
    """Retention factors (or log-decays with ``log_decay=True``) for ``logits [B,T,H,K]``."""
    _cuda(logits, "logits")
    if logits.dim() == 3:  # decode-shaped [B,H,K]
        res = bounded_decay(logits.unsqueeze(1), A_log, g_min, log_decay=log_decay,
                            out=None if out is None else out.unsqueeze(1), _softplus=_softplus)
        return res[:, 0]
    if logits.dim() != 4:
        raise ValueError("logits must be [B,T,H,K] or [B,H,K]")
    B, T, H, K = logits.shape
    logits = _rowwise(logits)
    A_log = A_log.to(device=logits.device, dtype=torch.float32).contiguous()
    if A_log.shape != (H,):
        raise ValueError("A_log must be [H]")
    if out is None:
        out = torch.empty_like(logits, memory_format=torch.contiguous_format)
    _cuda(out, "out")
    zs, os_ = _strides4(logits), _strides4(out)
    lib = load_library()
    kind = KDA_GATE_LOG if log_decay else KDA_GATE_ALPHA
    if _softplus:
        _check("kda_softplus_decay", lib.kda_softplus_decay(
            logits.data_ptr(), ctypes.byref(zs), _dtype_code(logits.dtype), A_log.data_ptr(),
            B, T, H, K, out.data_ptr(), ctypes.byref(os_), kind, _stream(logits.device)))
    else:
        _check("kda_bounded_decay", lib.kda_bounded_decay(
            logits.data_ptr(), ctypes.byref(zs), _dtype_code(logits.dtype), A_log.data_ptr(),
            float(g_min), B, T, H, K, out.data_ptr(), ctypes.byref(os_), kind, _stream(logits.device)))
    return out


def softplus_decay(logits: torch.Tensor, A_log: torch.Tensor, *, log_decay: bool = False,
                   out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Kimi Linear's unbounded gate (``kda_softplus_decay``): ``g = -exp(A_log[h]) * softplus(logits)``,
    retention factors ``exp(g)`` (or ``g`` with ``log_decay=True``); shapes as in ``bounded_decay``."""
    return bounded_decay(logits, A_log, log_decay=log_decay, out=out, _softplus=True)


def prefill_workspace_bytes(B: int, T: int, H: int, K: int, V: int, n_seq: int = 0,
                            dtype: torch.dtype = torch.bfloat16) -> int:
    n = ctypes.c_size_t(0)
    _check("kda_prefill_workspace_bytes", load_library().kda_prefill_workspace_bytes(
        B, T, H, K, V, n_seq, _dtype_code(dtype), ctypes.byref(n)))
    return int(n.value)


def _prefill(q, k, v, gate, beta, initial_state, cu_seqlens, gate_is_log, output_final_state, out, final_state,
             workspace, use_workspace, logits=None, gate_name="gate"):
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (gate, "gate"), (beta, "beta")):
        _cuda(t, n)
    if q.dim() != 4 or k.shape != q.shape or v.dim() != 4 or v.shape[:3] != q.shape[:3]:
        raise ValueError("q, k must be [B,T,H,K] and v [B,T,H,V]")
    if q.dtype != k.dtype or q.dtype != v.dtype:
        raise TypeError("q, k and v must share one dtype")
    if gate.shape != q.shape or gate.dtype != torch.float32:
        raise ValueError(f"{gate_name} must be fp32 [B,T,H,K]")
    if beta.shape != q.shape[:3] or beta.dtype != torch.float32:
        raise ValueError("beta must be fp32 [B,T,H]")
    B, T, H, K = q.shape
    V = v.shape[3]
    q, k, v, gate = map(_rowwise, (q, k, v, gate))
    dev = q.device
    cu_ptr, n_seq, N = None, 0, B
    if cu_seqlens is not None:
        _cuda(cu_seqlens, "cu_seqlens")
        if cu_seqlens.dtype != torch.int32:
            raise TypeError("cu_seqlens must be int32")
        cu_seqlens = cu_seqlens.contiguous()
        n_seq = cu_seqlens.numel() - 1
        N = n_seq
        cu_ptr = cu_seqlens.data_ptr()
    s0_ptr = None
    sshape = (N, H, V, K) if (logits is not None and logits[2] & KDA_STATE_VK) else (N, H, K, V)
    if initial_state is not None:
        _cuda(initial_state, "initial_state")
        if initial_state.shape != sshape or initial_state.dtype != torch.float32 \
                or not initial_state.is_contiguous():
            raise ValueError(f"initial_state must be a contiguous fp32 {list(sshape)} tensor")
        s0_ptr = initial_state.data_ptr()
    if output_final_state and final_state is None:
        final_state = torch.empty(sshape, device=dev, dtype=torch.float32)
    sf_ptr = None
    if final_state is not None:
        if final_state.shape != sshape or final_state.dtype != torch.float32 \
                or not final_state.is_contiguous():
            raise ValueError(f"final_state must be a contiguous fp32 {list(sshape)} tensor")
        sf_ptr = final_state.data_ptr()
    if out is None:
        out = torch.empty((B, T, H, V), device=dev, dtype=q.dtype)
    ws_need = prefill_workspace_bytes(B, T, H, K, V, n_seq, q.dtype)
    if workspace is None and ws_need > 0 and use_workspace:
        workspace = torch.empty(ws_need, device=dev, dtype=torch.uint8)
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    layout = Layout(_strides4(q), _strides4(k), _strides4(v), _strides4(gate), _strides3(beta), _strides4(out))
    lib = load_library()
    if logits is None:
        _check("kda_prefill", lib.kda_prefill(
            q.data_ptr(), k.data_ptr(), v.data_ptr(), _dtype_code(q.dtype), gate.data_ptr(),
            KDA_GATE_LOG if gate_is_log else KDA_GATE_ALPHA, beta.data_ptr(), s0_ptr, sf_ptr,
            cu_ptr, n_seq, B, T, H, K, V, ctypes.byref(layout), out.data_ptr(), ws_ptr, ws_bytes,
            _stream(dev)))
    else:
        A_log, g_min, flags, dt_bias = logits
        _check("kda_prefill_logits", lib.kda_prefill_logits(
            q.data_ptr(), k.data_ptr(), v.data_ptr(), _dtype_code(q.dtype), gate.data_ptr(),
            A_log.data_ptr(), None if dt_bias is None else dt_bias.data_ptr(), g_min, beta.data_ptr(), flags,
            s0_ptr, sf_ptr,
            cu_ptr, n_seq, B, T, H, K, V, ctypes.byref(layout), out.data_ptr(), ws_ptr, ws_bytes,
            _stream(dev)))
    return out, final_state


def prefill(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, gate: torch.Tensor, beta: torch.Tensor,
            initial_state: Optional[torch.Tensor] = None, cu_seqlens: Optional[torch.Tensor] = None, *,
            gate_is_log: bool = False, output_final_state: bool = True,
            out: Optional[torch.Tensor] = None, final_state: Optional[torch.Tensor] = None,
            workspace: Optional[torch.Tensor] = None,
            use_workspace: bool = True) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Scan whole sequences. Returns ``(o [B,T,H,V], final_state [N,H,K,V] fp32 or None)``.

    q, k ``[B,T,H,K]`` and v ``[B,T,H,V]`` share a dtype (bf16 or fp32); gate ``[B,T,H,K]`` fp32
    holds alpha (or g = log alpha when ``gate_is_log``); beta ``[B,T,H]`` fp32. With ``cu_seqlens``
    (int32 ``[N+1]`` on the device) B must be 1 and the states have N rows.
    ``final_state`` may be ``initial_state`` itself to resume in place. ``workspace`` (uint8, on the
    device) enables the two-kernel path when large enough; when it is None and ``use_workspace`` is
    true, one of ``prefill_workspace_bytes`` bytes is allocated; ``use_workspace=False`` runs the
    single fused kernel.
    """
    return _prefill(q, k, v, gate, beta, initial_state, cu_seqlens, gate_is_log, output_final_state, out,
                    final_state, workspace, use_workspace)


def _gate_flag(gate: str) -> int:
    if gate not in ("bounded", "softplus"):
        raise ValueError('gate must be "bounded" (g_min sigmoid) or "softplus" (Kimi Linear)')
    return KDA_GATE_SOFTPLUS if gate == "softplus" else 0


def _layout_flag(state_layout: str) -> int:
    if state_layout not in ("kv", "vk"):
        raise ValueError('state_layout must be "kv" ([N,H,K,V]) or "vk" ([N,H,V,K])')
    return KDA_STATE_VK if state_layout == "vk" else 0


def prefill_logits(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, z: torch.Tensor, A_log: torch.Tensor,
                   g_min: float, beta: torch.Tensor, initial_state: Optional[torch.Tensor] = None,
                   cu_seqlens: Optional[torch.Tensor] = None, *, qk_l2norm: bool = False,
                   beta_logits: bool = False, state_layout: str = "kv", gate: str = "bounded",
                   dt_bias: Optional[torch.Tensor] = None, output_final_state: bool = True,
                   out: Optional[torch.Tensor] = None, final_state: Optional[torch.Tensor] = None,
                   workspace: Optional[torch.Tensor] = None,
                   use_workspace: bool = True) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """``prefill`` fed with the decay logits ``z [B,T,H,K]`` (fp32) instead of alpha: the scan kernels
    evaluate ``g = g_min * sigmoid(exp(A_log[h]) * z)`` themselves (``kda_prefill_logits``).
    ``A_log [H]`` fp32 on the device; ``g_min < 0``. ``qk_l2norm``: the kernels L2-normalise q and k over
    K per (token, head); ``beta_logits``: ``beta`` holds logits and the kernels apply the sigmoid;
    ``state_layout="vk"``: the states are ``[N,H,V,K]`` (value-by-key) instead of ``[N,H,K,V]``;
    ``gate="softplus"``: the logits feed Kimi Linear's unbounded gate ``g = -exp(A_log) softplus(z)``
    (``g_min`` unused). ``dt_bias [H,K]`` fp32 (optional) is added to ``z`` before either gate. Other
    arguments as in ``prefill``."""
    _cuda(A_log, "A_log")
    if A_log.shape != (q.shape[2],) or A_log.dtype != torch.float32:
        raise ValueError("A_log must be fp32 [H]")
    flags = ((KDA_QK_L2NORM if qk_l2norm else 0) | (KDA_BETA_LOGITS if beta_logits else 0)
             | _layout_flag(state_layout) | _gate_flag(gate))
    bias = _bias(dt_bias, q.shape[2], q.shape[3])
    return _prefill(q, k, v, z, beta, initial_state, cu_seqlens, False, output_final_state, out, final_state,
                    workspace, use_workspace, logits=(A_log.contiguous(), float(g_min), flags, bias), gate_name="z")


def _bias(dt_bias: Optional[torch.Tensor], H: int, K: int) -> Optional[torch.Tensor]:
    if dt_bias is None:
        return None
    _cuda(dt_bias, "dt_bias")
    if dt_bias.shape != (H, K) or dt_bias.dtype != torch.float32:
        raise ValueError("dt_bias must be fp32 [H,K]")
    return dt_bias.contiguous()


NOALLOC_SCRATCH_BYTES = 128 << 20  # the library's static scratch (KDA_NOALLOC_SCRATCH_BYTES)


def prefill_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, gate: torch.Tensor, beta: torch.Tensor,
                    out: torch.Tensor, initial_state: Optional[torch.Tensor] = None,
                    final_state: Optional[torch.Tensor] = None, cu_seqlens: Optional[torch.Tensor] = None, *,
                    gate_is_log: bool = False) -> None:
    """``kda_prefill_noalloc``: the prefill with the library's static scratch as its workspace.

    For callers that must not allocate device memory between steps (cudaMalloc / cudaFree
    synchronise the device): neither this wrapper nor the call allocates anything, so every
    tensor, ``out [B,T,H,V]`` and the optional ``final_state [N,H,K,V]`` included, comes from the
    caller, contiguous in its innermost dim with 16-byte aligned rows. The first call on a device
    looks up the scratch address (make it before any stream capture); calls that may overlap on
    the GPU share the scratch and race on it. Sizes needing more than ``NOALLOC_SCRATCH_BYTES``
    of workspace raise ``KDAError`` (KDA_ERR_UNSUPPORTED).
    """
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (gate, "gate"), (beta, "beta"), (out, "out")):
        _cuda(t, n)
    if q.dim() != 4 or k.shape != q.shape or v.dim() != 4 or v.shape[:3] != q.shape[:3] or out.shape != v.shape:
        raise ValueError("q, k must be [B,T,H,K]; v and out [B,T,H,V]")
    if not (q.dtype == k.dtype == v.dtype == out.dtype):
        raise TypeError("q, k, v and out must share one dtype")
    if gate.shape != q.shape or gate.dtype != torch.float32:
        raise ValueError("gate must be fp32 [B,T,H,K]")
    if beta.shape != q.shape[:3] or beta.dtype != torch.float32:
        raise ValueError("beta must be fp32 [B,T,H]")
    B, T, H, K = q.shape
    V = v.shape[3]
    n_seq, N = 0, B
    if cu_seqlens is not None:
        _cuda(cu_seqlens, "cu_seqlens")
        if cu_seqlens.dtype != torch.int32 or not cu_seqlens.is_contiguous():
            raise TypeError("cu_seqlens must be a contiguous int32 tensor")
        n_seq = N = cu_seqlens.numel() - 1
    for t, n in ((initial_state, "initial_state"), (final_state, "final_state")):
        if t is not None:
            _cuda(t, n)
            if t.shape != (N, H, K, V) or t.dtype != torch.float32 or not t.is_contiguous():
                raise ValueError(f"{n} must be a contiguous fp32 [{N},{H},{K},{V}] tensor")
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (gate, "gate"), (out, "out")):
        if _rowwise(t) is not t:
            raise ValueError(f"{n}: innermost dim must be contiguous with 16-byte aligned rows")
    layout = Layout(_strides4(q), _strides4(k), _strides4(v), _strides4(gate), _strides3(beta), _strides4(out))
    ptr = lambda t: t.data_ptr() if t is not None else None
    _check("kda_prefill_noalloc", load_library().kda_prefill_noalloc(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), _dtype_code(q.dtype), gate.data_ptr(),
        KDA_GATE_LOG if gate_is_log else KDA_GATE_ALPHA, beta.data_ptr(), ptr(initial_state), ptr(final_state),
        ptr(cu_seqlens), n_seq, B, T, H, K, V, ctypes.byref(layout), out.data_ptr(), _stream(q.device)))


def decode_step(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, gate: torch.Tensor, beta: torch.Tensor,
                state: torch.Tensor, *, gate_is_log: bool = False,
                out: Optional[torch.Tensor] = None, logits=None) -> torch.Tensor:
    """One token against the kept ``state [B,H,K,V]`` (fp32, updated in place). Returns ``o [B,H,V]``.

    q, k ``[B,H,K]`` (or ``[B,1,H,K]``), v ``[B,H,V]``, gate ``[B,H,K]`` fp32, beta ``[B,H]`` fp32.
    ``logits=(A_log, g_min, flags, dt_bias)`` is the internal form of ``decode_step_logits``.
    """
    q, k, v, gate = (x[:, 0] if x.dim() == 4 else x for x in (q, k, v, gate))
    if beta.dim() == 3:
        beta = beta[:, 0]
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (gate, "gate"), (beta, "beta"), (state, "state")):
        _cuda(t, n)
    B, H, K = q.shape
    V = v.shape[2]
    if k.shape != q.shape or v.shape[:2] != (B, H) or gate.shape != q.shape or beta.shape != (B, H):
        raise ValueError("decode shapes: q, k, gate [B,H,K]; v [B,H,V]; beta [B,H]")
    if q.dtype != k.dtype or q.dtype != v.dtype:
        raise TypeError("q, k and v must share one dtype")
    if gate.dtype != torch.float32 or beta.dtype != torch.float32:
        raise TypeError("gate and beta must be fp32")
    sshape = (B, H, V, K) if (logits is not None and logits[2] & KDA_STATE_VK) else (B, H, K, V)
    if state.shape != sshape or state.dtype != torch.float32 or not state.is_contiguous():
        raise ValueError(f"state must be a contiguous fp32 {list(sshape)} tensor")
    q, k, v, gate = map(_rowwise, (q, k, v, gate))
    if out is None:
        out = torch.empty((B, H, V), device=q.device, dtype=q.dtype)
    s3 = lambda x: Strides(x.stride(0), 0, x.stride(1))  # noqa: E731
    layout = Layout(s3(q), s3(k), s3(v), s3(gate), Strides(beta.stride(0), 0, beta.stride(1)), s3(out))
    lib = load_library()
    if logits is None:
        _check("kda_decode_step", lib.kda_decode_step(
            q.data_ptr(), k.data_ptr(), v.data_ptr(), _dtype_code(q.dtype), gate.data_ptr(),
            KDA_GATE_LOG if gate_is_log else KDA_GATE_ALPHA, beta.data_ptr(), state.data_ptr(),
            B, H, K, V, ctypes.byref(layout), out.data_ptr(), _stream(q.device)))
    else:
        A_log, g_min, flags, dt_bias = logits
        _check("kda_decode_step_logits", lib.kda_decode_step_logits(
            q.data_ptr(), k.data_ptr(), v.data_ptr(), _dtype_code(q.dtype), gate.data_ptr(),
            A_log.data_ptr(), None if dt_bias is None else dt_bias.data_ptr(), g_min, beta.data_ptr(), flags,
            state.data_ptr(),
            B, H, K, V, ctypes.byref(layout), out.data_ptr(), _stream(q.device)))
    return out


def decode_step_logits(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, z: torch.Tensor, A_log: torch.Tensor,
                       g_min: float, beta: torch.Tensor, state: torch.Tensor, *, qk_l2norm: bool = False,
                       beta_logits: bool = False, state_layout: str = "kv", gate: str = "bounded",
                       dt_bias: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """``decode_step`` fed with the decay logits ``z [B,H,K]`` (fp32): the step evaluates the bounded gate
    itself (``kda_decode_step_logits``). ``A_log [H]`` fp32 on the device; ``g_min < 0``; ``qk_l2norm``,
    ``beta_logits``, ``state_layout`` (``state`` is ``[B,H,V,K]`` for ``"vk"``), ``gate`` and ``dt_bias`` as
    in ``prefill_logits``."""
    _cuda(A_log, "A_log")
    if A_log.shape != (q.shape[-2],) or A_log.dtype != torch.float32:
        raise ValueError("A_log must be fp32 [H]")
    flags = ((KDA_QK_L2NORM if qk_l2norm else 0) | (KDA_BETA_LOGITS if beta_logits else 0)
             | _layout_flag(state_layout) | _gate_flag(gate))
    bias = _bias(dt_bias, q.shape[-2], q.shape[-1])
    return decode_step(q, k, v, z, beta, state, out=out, logits=(A_log.contiguous(), float(g_min), flags, bias))


def scan_backward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, gate: torch.Tensor, beta: torch.Tensor,
                  initial_state: Optional[torch.Tensor], d_o: torch.Tensor, d_final_state: Optional[torch.Tensor] = None,
                  cu_seqlens: Optional[torch.Tensor] = None, *, gate_is_log: bool = False) -> dict:
    """Gradients of the scan (``kda_scan_backward``): returns fp32 ``dq, dk [B,T,H,K]``, ``dv [B,T,H,V]``,
    ``dgate`` (dL/dalpha, or dL/dg with ``gate_is_log``), ``dbeta [B,T,H]`` and ``d_initial_state [N,H,K,V]``
    for ``L = <o, d_o> + <S_T, d_final_state>``. Inputs as for ``prefill``: with ``cu_seqlens`` (int32
    ``[N+1]``, B = 1) the states are per sequence (N = number of sequences, else N = B) and the gradients
    of tokens outside every sequence are zero."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (gate, "gate"), (beta, "beta"), (d_o, "d_o")):
        _cuda(t, n)
    if q.dim() != 4 or k.shape != q.shape or v.dim() != 4 or v.shape[:3] != q.shape[:3]:
        raise ValueError("q, k must be [B,T,H,K] and v [B,T,H,V]")
    if gate.shape != q.shape or gate.dtype != torch.float32 or beta.shape != q.shape[:3] or beta.dtype != torch.float32:
        raise ValueError("gate must be fp32 [B,T,H,K] and beta fp32 [B,T,H]")
    B, T, H, K = q.shape
    V = v.shape[3]
    dev = q.device
    q, k, v, gate = map(_rowwise, (q, k, v, gate))
    d_o = d_o.to(torch.float32).contiguous()
    if d_o.shape != (B, T, H, V):
        raise ValueError("d_o must be [B,T,H,V]")
    N, n_seq, cu_ptr = B, 0, None
    if cu_seqlens is not None:
        _cuda(cu_seqlens, "cu_seqlens")
        if cu_seqlens.dtype != torch.int32:
            raise TypeError("cu_seqlens must be int32")
        if B != 1:
            raise ValueError("cu_seqlens requires B == 1")
        cu_seqlens = cu_seqlens.contiguous()
        N = n_seq = cu_seqlens.numel() - 1
        cu_ptr = cu_seqlens.data_ptr()
    f32 = lambda t: None if t is None else t.to(device=dev, dtype=torch.float32).contiguous()  # noqa: E731
    initial_state, d_final_state = f32(initial_state), f32(d_final_state)
    for t, n in ((initial_state, "initial_state"), (d_final_state, "d_final_state")):
        if t is not None and t.shape != (N, H, K, V):
            raise ValueError(f"{n} must be [{N},{H},{K},{V}]")
    new = torch.zeros if cu_seqlens is not None else torch.empty
    out = {"dq": new(B, T, H, K, device=dev), "dk": new(B, T, H, K, device=dev),
           "dv": new(B, T, H, V, device=dev), "dgate": new(B, T, H, K, device=dev),
           "dbeta": new(B, T, H, device=dev), "d_initial_state": torch.empty(N, H, K, V, device=dev)}
    lib = load_library()
    n = ctypes.c_size_t(0)
    _check("kda_scan_backward_workspace_bytes",
           lib.kda_scan_backward_workspace_bytes(B, T, H, K, V, n_seq, ctypes.byref(n)))
    ws = torch.empty(max(int(n.value), 16), device=dev, dtype=torch.uint8)
    layout = Layout(_strides4(q), _strides4(k), _strides4(v), _strides4(gate), _strides3(beta), Strides(0, 0, 0))
    ptr = lambda t: t.data_ptr() if t is not None else None  # noqa: E731
    _check("kda_scan_backward", lib.kda_scan_backward(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), _dtype_code(q.dtype), gate.data_ptr(),
        KDA_GATE_LOG if gate_is_log else KDA_GATE_ALPHA, beta.data_ptr(), ptr(initial_state), d_o.data_ptr(),
        ptr(d_final_state), cu_ptr, n_seq, B, T, H, K, V, ctypes.byref(layout), out["dq"].data_ptr(), out["dk"].data_ptr(),
        out["dv"].data_ptr(), out["dgate"].data_ptr(), out["dbeta"].data_ptr(), out["d_initial_state"].data_ptr(),
        ws.data_ptr(), ws.numel(), _stream(dev)))
    return out


def scan_backward_chunked(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, gate: torch.Tensor, beta: torch.Tensor,
                          initial_state: Optional[torch.Tensor], d_o: torch.Tensor,
                          d_final_state: Optional[torch.Tensor] = None, cu_seqlens: Optional[torch.Tensor] = None, *,
                          gate_is_log: bool = False, workspace: Optional[torch.Tensor] = None) -> dict:
    """The gradients of ``scan_backward`` through the chunkwise form in parallel over 64-token chunks
    (``kda_scan_backward_chunked``): bf16 ``q, k, v`` with K = V = 128; dense batch rows or packed sequences
    (``cu_seqlens`` int32 ``[N+1]``, B = 1, states per sequence). Same outputs as ``scan_backward``.
    ``workspace``: optional uint8 device tensor of at least ``chunked_backward_workspace_bytes`` bytes."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (gate, "gate"), (beta, "beta"), (d_o, "d_o")):
        _cuda(t, n)
    if q.dim() != 4 or k.shape != q.shape or v.dim() != 4 or v.shape[:3] != q.shape[:3]:
        raise ValueError("q, k must be [B,T,H,K] and v [B,T,H,V]")
    if gate.shape != q.shape or gate.dtype != torch.float32 or beta.shape != q.shape[:3] or beta.dtype != torch.float32:
        raise ValueError("gate must be fp32 [B,T,H,K] and beta fp32 [B,T,H]")
    B, T, H, K = q.shape
    V = v.shape[3]
    dev = q.device
    q, k, v, gate = map(_rowwise, (q, k, v, gate))
    d_o = d_o.to(torch.float32).contiguous()
    if d_o.shape != (B, T, H, V):
        raise ValueError("d_o must be [B,T,H,V]")
    N, n_seq, cu_ptr = B, 0, None
    if cu_seqlens is not None:
        _cuda(cu_seqlens, "cu_seqlens")
        if cu_seqlens.dtype != torch.int32:
            raise TypeError("cu_seqlens must be int32")
        if B != 1:
            raise ValueError("cu_seqlens requires B == 1")
        cu_seqlens = cu_seqlens.contiguous()
        N = n_seq = cu_seqlens.numel() - 1
        cu_ptr = cu_seqlens.data_ptr()
    f32 = lambda t: None if t is None else t.to(device=dev, dtype=torch.float32).contiguous()  # noqa: E731
    initial_state, d_final_state = f32(initial_state), f32(d_final_state)
    for t, n in ((initial_state, "initial_state"), (d_final_state, "d_final_state")):
        if t is not None and t.shape != (N, H, K, V):
            raise ValueError(f"{n} must be [{N},{H},{K},{V}]")
    new = torch.zeros if cu_seqlens is not None else torch.empty  # tokens outside every sequence: zero
    out = {"dq": new(B, T, H, K, device=dev), "dk": new(B, T, H, K, device=dev),
           "dv": new(B, T, H, V, device=dev), "dgate": new(B, T, H, K, device=dev),
           "dbeta": new(B, T, H, device=dev), "d_initial_state": torch.empty(N, H, K, V, device=dev)}
    lib = load_library()
    need = chunked_backward_workspace_bytes(B, T, H, K, V, n_seq)
    if workspace is None:
        workspace = torch.empty(max(need, 16), device=dev, dtype=torch.uint8)
    layout = Layout(_strides4(q), _strides4(k), _strides4(v), _strides4(gate), _strides3(beta), Strides(0, 0, 0))
    ptr = lambda t: t.data_ptr() if t is not None else None  # noqa: E731
    _check("kda_scan_backward_chunked", lib.kda_scan_backward_chunked(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), _dtype_code(q.dtype), gate.data_ptr(),
        KDA_GATE_LOG if gate_is_log else KDA_GATE_ALPHA, beta.data_ptr(), ptr(initial_state), d_o.data_ptr(),
        ptr(d_final_state), cu_ptr, n_seq, B, T, H, K, V, ctypes.byref(layout), out["dq"].data_ptr(),
        out["dk"].data_ptr(), out["dv"].data_ptr(), out["dgate"].data_ptr(), out["dbeta"].data_ptr(),
        out["d_initial_state"].data_ptr(), workspace.data_ptr(), workspace.numel(), _stream(dev)))
    return out


def chunked_backward_workspace_bytes(B: int, T: int, H: int, K: int = 128, V: int = 128, n_seq: int = 0) -> int:
    """Workspace bytes of ``scan_backward_chunked`` (``kda_scan_backward_chunked_workspace_bytes``; ``n_seq``:
    the number of packed sequences, 0 without ``cu_seqlens``)."""
    n = ctypes.c_size_t(0)
    _check("kda_scan_backward_chunked_workspace_bytes",
           load_library().kda_scan_backward_chunked_workspace_bytes(B, T, H, K, V, n_seq, ctypes.byref(n)))
    return int(n.value)


def bounded_decay_backward(logits: torch.Tensor, A_log: torch.Tensor, g_min: float,
                           d_log_decay: torch.Tensor) -> Tuple[torch.Tensor, torch.Tensor]:
    """``kda_bounded_decay_backward``: ``(dL/dlogits [B,T,H,K], dL/dA_log [H])`` given ``dL/dg`` (all fp32)."""
    _cuda(logits, "logits")
    B, T, H, K = logits.shape
    z = logits.to(torch.float32).contiguous()
    dg = d_log_decay.to(device=z.device, dtype=torch.float32).contiguous()
    A = A_log.to(device=z.device, dtype=torch.float32).contiguous()
    dz, dA = torch.empty_like(z), torch.empty(H, device=z.device)
    _check("kda_bounded_decay_backward", load_library().kda_bounded_decay_backward(
        z.data_ptr(), A.data_ptr(), float(g_min), dg.data_ptr(), B, T, H, K, dz.data_ptr(), dA.data_ptr(),
        _stream(z.device)))
    return dz, dA


def selftest_wait_expiry(device=None) -> None:
    """``kda_selftest_wait_expiry``: one kernel whose bounded wait runs out (about a second); the next
    ``device_status()`` then reports True."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    _check("kda_selftest_wait_expiry", load_library().kda_selftest_wait_expiry(_stream(dev)))


def device_status(reset: bool = True) -> bool:
    """Synchronises the device; True if a kernel's bounded wait expired since the last reset."""
    flag = ctypes.c_int(0)
    _check("kda_device_status", load_library().kda_device_status(ctypes.byref(flag), int(reset)))
    return bool(flag.value)
