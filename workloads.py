"""Seeded synthetic inputs for the KDA scan workloads.

This module is the only code that both the CUDA path's callers and the fp64
oracle's callers use. It draws random tensors and nothing else: it holds none
of the method's arithmetic (no gate, no decay, no scan). The decay logits ``z``
leave here as logits; each side turns them into retention factors with its
own gate.

Distributions follow the workload descriptions the benchmark and the tests
reproduce (all draws on the CPU from ``torch.Generator().manual_seed(seed)``,
in this fixed order: varlen lengths, q, k, v, z, A_log, beta logits, initial
state):

* q, k: fp32 N(0,1), L2-normalised over the key dimension per (token, head)
  (the surrounding model's L2Norm on q and k, "KDA cheat sheet", How the
  inputs are produced), then cast to the workload dtype;
* v: N(0,1) in the workload dtype;
* z (decay logits): N(0, z_std) fp32; A_log: N(0, 0.5) fp32 per head;
* beta: sigmoid of N(0,1), fp32 (the model's write-strength preparation);
* initial state: zeros, or N(0, init_std) fp32, shape [N,H,K,V];
* varlen lengths: uniform integers in [len_lo, len_hi].

"N(0, s)" is read as a normal with standard deviation s.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch

DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16}


@dataclasses.dataclass(frozen=True)
class ScanWorkload:
    """Sizes and distributions of one prefill-scan workload."""
    name: str
    B: int
    T: int
    H: int
    K: int
    V: int
    dtype: str = "bf16"
    z_std: float = 1.0
    init_std: Optional[float] = None   # None: zero initial state
    n_seq: Optional[int] = None        # packed varlen sequences (B must be 1)
    len_lo: int = 0
    len_hi: int = 0
    g_min: float = -5.0
    seed: int = 0


@dataclasses.dataclass(frozen=True)
class DecodeWorkload:
    """Sizes and distributions of the kept-memory decode workload."""
    name: str
    B: int
    H: int
    K: int
    V: int
    steps: int
    dtype: str = "bf16"
    z_std: float = 1.0
    init_std: float = 0.1
    g_min: float = -5.0
    seed: int = 0


# The five workloads: a tiny fp32 scan, the kept-memory decode step, a single
# 4096-token prefill, 16 packed variable-length sequences, and a long K != V
# prefill (the last is checked by splitting at T = 8192 and resuming).
TINY_FP32 = ScanWorkload("tiny_fp32_B1_T256_H4_K32_V32", 1, 256, 4, 32, 32, dtype="f32", z_std=1.0)
DECODE = DecodeWorkload("decode_B64_H96_K128_V128", 64, 96, 128, 128, steps=1000, z_std=1.0, init_std=0.1)
PREFILL = ScanWorkload("prefill_B1_T4096_H96_K128_V128", 1, 4096, 96, 128, 128, z_std=2.0)
VARLEN = ScanWorkload("varlen_N16_L512to8192_H96_K128_V128", 1, 0, 96, 128, 128, z_std=2.0,
                      init_std=0.1, n_seq=16, len_lo=512, len_hi=8192)
LONG_KV = ScanWorkload("long_B4_T16384_H32_K128_V256", 4, 16384, 32, 128, 256, z_std=2.0, init_std=0.1)


def _gen(seed: int) -> torch.Generator:
    return torch.Generator(device="cpu").manual_seed(int(seed))


def _unit_rows(x: torch.Tensor) -> torch.Tensor:
    return torch.nn.functional.normalize(x, p=2.0, dim=-1)


def make_scan_inputs(w: ScanWorkload, T: Optional[int] = None, H: Optional[int] = None) -> dict:
    """CPU tensors for one scan workload (``T``/``H`` override the sizes for scaled-down cases).

    Returns a dict with q, k, v ``[B,T,H,*]`` (workload dtype), z ``[B,T,H,K]`` fp32,
    A_log ``[H]`` fp32, beta ``[B,T,H]`` fp32, initial_state ``[N,H,K,V]`` fp32 or None,
    cu_seqlens int32 ``[N+1]`` or None, and g_min.
    """
    g = _gen(w.seed)
    H = w.H if H is None else H
    dt = DTYPES[w.dtype]
    cu = None
    if w.n_seq is not None:
        lengths = torch.randint(w.len_lo, w.len_hi + 1, (w.n_seq,), generator=g)
        cu = torch.zeros(w.n_seq + 1, dtype=torch.int32)
        cu[1:] = torch.cumsum(lengths, 0).to(torch.int32)
        B, TT = 1, int(cu[-1])
    else:
        B, TT = w.B, (w.T if T is None else T)
    K, V = w.K, w.V
    q = _unit_rows(torch.randn(B, TT, H, K, generator=g)).to(dt)
    k = _unit_rows(torch.randn(B, TT, H, K, generator=g)).to(dt)
    v = torch.randn(B, TT, H, V, generator=g).to(dt)
    z = torch.randn(B, TT, H, K, generator=g) * w.z_std
    A_log = torch.randn(H, generator=g) * 0.5
    beta = torch.sigmoid(torch.randn(B, TT, H, generator=g))
    N = B if cu is None else w.n_seq
    s0 = None
    if w.init_std is not None:
        s0 = torch.randn(N, H, K, V, generator=g) * w.init_std
    return dict(q=q, k=k, v=v, z=z, A_log=A_log, beta=beta, initial_state=s0,
                cu_seqlens=cu, g_min=w.g_min)


def make_output_grad(w: ScanWorkload, T: Optional[int] = None, H: Optional[int] = None) -> torch.Tensor:
    """dL/do ``[B,T,H,V]`` fp32 N(0,1) for the gradient workloads (its own seed, so the scan inputs of
    the same workload are unchanged)."""
    g = _gen(w.seed + 1)
    return torch.randn(w.B, w.T if T is None else T, w.H if H is None else H, w.V, generator=g)


def make_decode_params(w: DecodeWorkload) -> dict:
    """Per-head log-scale ``A_log [H]`` and the initial kept state ``[B,H,K,V]`` fp32."""
    g = _gen(w.seed)
    A_log = torch.randn(w.H, generator=g) * 0.5
    state = torch.randn(w.B, w.H, w.K, w.V, generator=g) * w.init_std
    return dict(A_log=A_log, state=state, g_min=w.g_min)


def make_decode_step(w: DecodeWorkload, step: int) -> dict:
    """Inputs of decode step ``step``: q, k ``[B,H,K]``, v ``[B,H,V]``, z ``[B,H,K]``, beta ``[B,H]``.

    Each step draws from its own generator (seeded from the workload seed and
    the step index), so any step can be regenerated without the others.
    """
    g = _gen(w.seed * 1_000_003 + 7919 * (step + 1))
    dt = DTYPES[w.dtype]
    q = _unit_rows(torch.randn(w.B, w.H, w.K, generator=g)).to(dt)
    k = _unit_rows(torch.randn(w.B, w.H, w.K, generator=g)).to(dt)
    v = torch.randn(w.B, w.H, w.V, generator=g).to(dt)
    z = torch.randn(w.B, w.H, w.K, generator=g) * w.z_std
    beta = torch.sigmoid(torch.randn(w.B, w.H, generator=g))
    return dict(q=q, k=k, v=v, z=z, beta=beta)


def random_scan_case(B: int, T: int, H: int, K: int, V: int, seed: int, dtype: str = "f32",
                     z_std: float = 1.0, init_std: Optional[float] = 0.1, n_seq: Optional[int] = None,
                     len_lo: int = 0, len_hi: int = 0, raw_inputs: bool = False) -> dict:
    """A scan case of arbitrary small sizes with the standard distributions.

    With ``raw_inputs`` the case holds what the model has *before* its preparation: q and k are
    N(0, 2) draws that are not L2-normalised, and ``beta`` holds the N(0,1) logits instead of their
    sigmoid (for the entry points that prepare q, k and beta inside their kernels)."""
    w = ScanWorkload(f"case_{B}_{T}_{H}_{K}_{V}_{seed}", B, T, H, K, V, dtype=dtype, z_std=z_std,
                     init_std=init_std, n_seq=n_seq, len_lo=len_lo, len_hi=len_hi, seed=seed)
    d = make_scan_inputs(w)
    if raw_inputs:
        g = _gen(seed + 7919)
        dt = DTYPES[dtype]
        d["q"] = (torch.randn(d["q"].shape, generator=g) * 2.0).to(dt)
        d["k"] = (torch.randn(d["k"].shape, generator=g) * 2.0).to(dt)
        d["beta"] = torch.randn(d["beta"].shape, generator=g)
    return d
