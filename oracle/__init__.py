"""fp64 CPU oracle for the bounded-decay gated delta rule.

TEST INFRASTRUCTURE ONLY. The test suite, the smoke check and the benchmark's
CPU-baseline leg are the only callers. The CUDA library and its Python binding
never import this package, and the two share no code: inputs reach both sides
from the seeded generators in ``workloads.py`` and nothing else.

The arithmetic lives in ``kda_oracle.c`` (plain C, double precision, the
token-by-token recurrence written in the order of the defining equations).
This module only converts arrays to contiguous fp64 (an exact widening for
bf16 and fp32 inputs) and calls it.

Functions and the passages they follow:

* :func:`bounded_decay` -- "Kimi K3: Bounded Decay and Delta Memory",
  Formula and conventions, eq. 5: ``g = g_min * sigmoid(exp(A) * z)``,
  ``alpha = exp(g)``. An optional per-(head, channel) bias is added to the
  logits first, in fp64 ("KDA cheat sheet", How the inputs are produced:
  ``z = W_up W_down x + b``; the chunked kernel call on the "Kept memory" page
  names it ``dt_bias``).
* :func:`scan_backward`, :func:`bounded_decay_backward` -- gradients of the
  scan and of the gate: eq. 1 and eq. 5 restated with plain fp64 PyTorch ops
  (:func:`scan_torch`) and differentiated by autograd. Pinned by the C
  oracle's forward values and by finite differences (gradcheck).
* :func:`softplus_decay` -- Kimi Linear's unbounded gate, the contrast drawn in
  Figure 3(a) of the same page: ``g = -exp(A) * softplus(z)`` (with the same
  optional bias on z).
* :func:`l2norm`, :func:`sigmoid` -- the input preparation the surrounding
  model applies ("KDA cheat sheet", How the inputs are produced: q, k =
  L2Norm(...), beta = Sigmoid(W_beta x)); they check the scan entry points that
  do this preparation inside their kernels. L2Norm is read as the unit
  normalisation of the key axis, guarded by an epsilon of 1e-6 under the root.
* :func:`scan` -- same page, eq. 1 (fade, correct, then read the updated
  state), with the contract table of that page: q, k ``[B,T,H,K]``, v
  ``[B,T,H,V]``, alpha ``[B,T,H,K]``, beta ``[B,T,H]``, state ``[B,H,K,V]``
  (key-by-value), omitted initial state means zeros, T = 0 returns the input
  state. Packed variable-length sequences follow the ``cu_seqlens`` argument
  of the production kernel call excerpted on the "Kept memory" page.

Parity status: both functions are pinned by the ``-m "not gpu"`` tests in
``tests/test_oracle_pins.py`` (printed toy outputs, closed forms, the
independent product form of the "KDA cheat sheet", exact rational brute force
and the chunkwise form of the same cheat sheet).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        i64 = ctypes.c_int64
        lib.kda_oracle_bounded_decay.argtypes = [dp, dp, ctypes.c_double, i64, i64, i64, i64, dp, dp]
        lib.kda_oracle_bounded_decay.restype = None
        lib.kda_oracle_scan.argtypes = [dp, dp, dp, dp, dp, dp, ctypes.POINTER(i64), i64,
                                        i64, i64, i64, i64, i64, dp, dp, ctypes.c_int]
        lib.kda_oracle_scan.restype = ctypes.c_int
        lib.kda_oracle_max_threads.argtypes = []
        lib.kda_oracle_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    """Contiguous fp64 copy of a numpy array or a (CPU or CUDA) torch tensor."""
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor: widen in torch (bf16 -> fp64 is exact)
        import torch
        x = x.detach().to(device="cpu", dtype=torch.float64).contiguous().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double)) if a is not None else None


def max_threads() -> int:
    """OpenMP threads the oracle uses by default (``OMP_NUM_THREADS`` or all cores)."""
    return int(_load().kda_oracle_max_threads())


def l2norm(x, eps: float = 1e-6) -> np.ndarray:
    """Unit normalisation over the last axis (the key channels of each token and head), in fp64:
    ``x / sqrt(sum(x^2) + eps)``."""
    x = _f64(x)
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)


def sigmoid(x) -> np.ndarray:
    """The logistic function in fp64, evaluated without overflow for either sign."""
    x = _f64(x)
    e = np.exp(-np.abs(x))
    return np.where(x >= 0, 1.0 / (1.0 + e), e / (1.0 + e))


def _biased(z, dt_bias):
    """The gate's input: the logits z ``[B,T,H,K]`` plus the bias ``[H,K]`` (when given), in fp64."""
    z = _f64(z)
    if dt_bias is None:
        return z
    b = _f64(dt_bias)
    if b.shape != (z.shape[2], z.shape[3]):
        raise ValueError("dt_bias must be [H,K]")
    return z + b[None, None]


def softplus_decay(z, A_log, return_log: bool = False, dt_bias=None):
    """Kimi Linear's unbounded gate in fp64 ("Kimi K3: Bounded Decay and Delta Memory", Figure 3(a)
    contrast; "KDA cheat sheet", g_min table): ``g = -exp(A_log[h]) * softplus(z + dt_bias)`` with
    ``softplus(x) = max(x, 0) + log(1 + exp(-|x|))``; ``alpha = exp(g)``. z ``[B,T,H,K]``."""
    z = _biased(z, dt_bias)
    sc = np.exp(_f64(A_log))[None, None, :, None]
    g = -sc * (np.maximum(z, 0.0) + np.log1p(np.exp(-np.abs(z))))
    alpha = np.exp(g)
    return (alpha, g) if return_log else alpha


def bounded_decay(z, A_log, g_min: float = -5.0, return_log: bool = False, dt_bias=None):
    """alpha (and optionally g) for logits ``z [B,T,H,K]``, per-head ``A_log [H]`` and the optional bias
    ``dt_bias [H,K]`` added to z: ``g = g_min * sigmoid(exp(A_log[h]) * (z + dt_bias[h]))``."""
    lib = _load()
    z = _biased(z, dt_bias)
    A = _f64(A_log)
    if z.ndim != 4 or A.shape != (z.shape[2],):
        raise ValueError("z must be [B,T,H,K] and A_log [H]")
    B, T, H, K = z.shape
    alpha = np.empty_like(z)
    g = np.empty_like(z)
    lib.kda_oracle_bounded_decay(_ptr(z), _ptr(A), float(g_min), B, T, H, K, _ptr(alpha), _ptr(g))
    return (alpha, g) if return_log else alpha


def scan(q, k, v, alpha, beta, initial_state=None, cu_seqlens=None, n_threads: int = 0):
    """Token-by-token scan. Returns ``(o [B,T,H,V], final_state [N,H,K,V])`` in fp64.

    ``N`` is ``B``, or the number of packed sequences when ``cu_seqlens`` (int
    offsets, length ``N+1``) is given, in which case ``B`` must be 1.
    """
    lib = _load()
    q, k, v, alpha, beta = map(_f64, (q, k, v, alpha, beta))
    if q.ndim != 4 or k.shape != q.shape or alpha.shape != q.shape:
        raise ValueError("q, k, alpha must share the shape [B,T,H,K]")
    B, T, H, K = q.shape
    if v.ndim != 4 or v.shape[:3] != (B, T, H):
        raise ValueError("v must be [B,T,H,V]")
    V = v.shape[3]
    if beta.shape != (B, T, H):
        raise ValueError("beta must be [B,T,H]")
    cu = None
    N = B
    if cu_seqlens is not None:
        cu = np.ascontiguousarray(np.asarray(
            cu_seqlens.cpu() if hasattr(cu_seqlens, "cpu") else cu_seqlens, dtype=np.int64))
        N = cu.shape[0] - 1
    s0 = None
    if initial_state is not None:
        s0 = _f64(initial_state)
        if s0.shape != (N, H, K, V):
            raise ValueError(f"initial_state must be [{N},{H},{K},{V}]")
    o = np.zeros((B, T, H, V), dtype=np.float64)
    sf = np.zeros((N, H, K, V), dtype=np.float64)
    cu_ptr = cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)) if cu is not None else None
    rc = lib.kda_oracle_scan(_ptr(q), _ptr(k), _ptr(v), _ptr(alpha), _ptr(beta), _ptr(s0),
                             cu_ptr, N if cu is not None else 0, B, T, H, K, V,
                             _ptr(o), _ptr(sf), int(n_threads))
    if rc != 0:
        raise ValueError("oracle scan rejected its arguments")
    return o, sf


def scan_torch(q, k, v, alpha, beta, initial_state=None):
    """Eq. 1 token by token with fp64 torch tensors (differentiable): fade, correct, then read.
    Returns ``(o [B,T,H,V], final_state [B,H,K,V])``."""
    import torch
    B, T, H, K = q.shape
    V = v.shape[-1]
    S = initial_state if initial_state is not None else torch.zeros(B, H, K, V, dtype=torch.float64)
    outs = []
    for t in range(T):
        Sb = alpha[:, t][..., None] * S                                    # Diag(alpha) S
        delta = v[:, t] - torch.einsum("bhk,bhkv->bhv", k[:, t], Sb)      # v - Sbar^T k
        S = Sb + beta[:, t][..., None, None] * k[:, t][..., None] * delta[..., None, :]
        outs.append(torch.einsum("bhk,bhkv->bhv", q[:, t], S))             # S^T q
    return torch.stack(outs, dim=1), S


def scan_backward(q, k, v, alpha, beta, initial_state, d_o, d_final_state=None):
    """Gradients of ``L = <o, d_o> + <S_T, d_final_state>`` with respect to q, k, v, alpha, beta and the
    initial state, in fp64 (numpy arrays; ``initial_state`` may be None = zeros)."""
    import torch
    t64 = lambda x: torch.tensor(_f64(x), requires_grad=True)  # noqa: E731
    Q, Kk, Vv, A, Bt = (t64(x) for x in (q, k, v, alpha, beta))
    S0 = t64(initial_state) if initial_state is not None else torch.zeros(
        Q.shape[0], Q.shape[2], Q.shape[3], Vv.shape[3], dtype=torch.float64, requires_grad=True)
    o, sf = scan_torch(Q, Kk, Vv, A, Bt, S0)
    L = (o * torch.tensor(_f64(d_o))).sum()
    if d_final_state is not None:
        L = L + (sf * torch.tensor(_f64(d_final_state))).sum()
    L.backward()
    return {n: x.grad.numpy() for n, x in (("q", Q), ("k", Kk), ("v", Vv), ("alpha", A), ("beta", Bt),
                                              ("initial_state", S0))}


def bounded_decay_backward(z, A_log, g_min, d_log_decay):
    """dL/dz and dL/dA_log of eq. 5's log-decay ``g = g_min * sigmoid(exp(A_log) * z)`` given dL/dg."""
    import torch
    Z = torch.tensor(_f64(z), requires_grad=True)
    Al = torch.tensor(_f64(A_log), requires_grad=True)
    g = g_min * torch.sigmoid(torch.exp(Al)[None, None, :, None] * Z)
    (g * torch.tensor(_f64(d_log_decay))).sum().backward()
    return Z.grad.numpy(), Al.grad.numpy()
