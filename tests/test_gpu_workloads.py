"""Full-size parity of the call the benchmark times, kda_prefill_logits, on the three prefill
workloads: the single 4096-token sequence (H = 96, K = V = 128, zero initial state), the 16 packed
sequences of 512..8192 tokens with their own initial states, and the long K != V case (B = 4,
T = 16384, H = 32, V = 256) run whole and split at T = 8192 and resumed from the final state.

The GPU computes every head with the same launch configuration as the benchmark (the two-kernel
path, the gate evaluated from the logits inside the kernels); the fp64 oracle runs on a sample of
heads and the two are compared there with the tolerances of ``tests/parity.py`` (for the packed
sequences, per sequence as well).
"""
import pytest
import torch

import oracle
import workloads as W
from tests.parity import DEV, check, to_dev

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module")
def kda():
    from gated_delta_rule_bounded_b200 import build
    build.build()
    import gated_delta_rule_bounded_b200 as m
    m.load_library()
    return m


def oracle_heads(d, heads, cut=None):
    z, q, k, v, beta = (d[n][:, :, heads] for n in ("z", "q", "k", "v", "beta"))
    s0 = d["initial_state"][:, heads] if d["initial_state"] is not None else None
    alpha = oracle.bounded_decay(z, d["A_log"][heads], d["g_min"])
    return oracle.scan(q, k, v, alpha, beta, s0, d["cu_seqlens"])


def logits_call(kda, g, a=None, b=None, s0=None, final_state=None):
    sl = slice(a, b)
    return kda.prefill_logits(g["q"][:, sl], g["k"][:, sl], g["v"][:, sl], g["z"][:, sl], g["A_log"], g["g_min"],
                              g["beta"][:, sl], g["initial_state"] if s0 is None else s0, g["cu_seqlens"],
                              final_state=final_state)


def test_prefill_workload_logits_sampled_heads(kda):
    d = W.make_scan_inputs(W.PREFILL)
    g = to_dev(d)
    o, sf = logits_call(kda, g)
    torch.cuda.synchronize()
    assert not kda.device_status()
    heads = [0, 13, 47, 95]
    ro, rs = oracle_heads(d, heads)
    check(o[:, :, heads], ro, "bf16", "o")
    check(sf[:, heads], rs, "bf16", "final_state")


def test_varlen_workload_logits_sampled_heads(kda):
    d = W.make_scan_inputs(W.VARLEN)
    g = to_dev(d)
    g["cu_seqlens"] = g["cu_seqlens"].contiguous()
    o, sf = logits_call(kda, g)
    torch.cuda.synchronize()
    assert not kda.device_status()
    heads = [3, 60]
    ro, rs = oracle_heads(d, heads)
    check(o[:, :, heads], ro, "bf16", "o")
    check(sf[:, heads], rs, "bf16", "final_state")
    cu = d["cu_seqlens"].tolist()
    for n in range(len(cu) - 1):
        s, e = cu[n], cu[n + 1]
        check(o[:, s:e][:, :, heads], ro[:, s:e], "bf16", f"o seq {n}")
        check(sf[n, heads], rs[n], "bf16", f"final_state seq {n}")


def test_long_kv_workload_logits_split_resume_sampled(kda):
    d = W.make_scan_inputs(W.LONG_KV)
    g = to_dev(d)
    o, sf = logits_call(kda, g)
    half = W.LONG_KV.T // 2
    st = g["initial_state"].clone()
    o1, _ = logits_call(kda, g, 0, half, s0=st, final_state=st)
    o2, _ = logits_call(kda, g, half, None, s0=st, final_state=st)
    torch.cuda.synchronize()
    assert not kda.device_status()
    heads = [5, 30]
    ro, rs = oracle_heads(d, heads)
    check(o[:, :, heads], ro, "bf16", "o")
    check(sf[:, heads], rs, "bf16", "final_state")
    check(torch.cat([o1, o2], 1)[:, :, heads], ro, "bf16", "o (split)")
    check(st[:, heads], rs, "bf16", "final_state (split)")
