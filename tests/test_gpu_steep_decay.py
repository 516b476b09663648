"""GPU parity where the decay is steeper than the block-boundary factorisation can hold.

The chunked kernels factor each decay ratio exp(G_t - G_i) across 16-token blocks; the factor of a
diagonal block is the reciprocal of the block's whole decay, which stays in range for a per-token
log-decay g >= -5 ("KDA cheat sheet", Lower-bounded decay: the g_min trick) but not for the bounded
gate at a lower g_min ("Kimi K3: Bounded Decay and Delta Memory", Formula and conventions, eq. 5
fixes g_min only as a parameter < 0), for alpha near or equal to 0, or for Kimi Linear's unbounded
gate. Blocks whose decay leaves the range on some channel take their diagonal tiles pair by pair.
Each case here mixes such blocks with ordinary ones and is checked against the fp64 oracle on the
two-kernel (workspace) and the single-kernel paths, with the tolerances of ``tests/parity.py``.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests.parity import DEV, check, to_dev

pytestmark = pytest.mark.gpu

PATHS = pytest.mark.parametrize("use_workspace", [True, False], ids=["split", "fused"])
SAFE_LOG2 = -120.0  # a block's log2-decay sum below this takes the pairwise diagonal path


@pytest.fixture(scope="module")
def kda():
    from gated_delta_rule_bounded_b200 import build
    build.build()
    import gated_delta_rule_bounded_b200 as m
    m.load_library()
    return m


def block_sums_log2(log_decay: np.ndarray) -> np.ndarray:
    """Per 16-token block (counted from the start of the sequence), per (b, h, channel): the log2-decay
    sum; [B, T // 16, H, K]."""
    B, T, H, K = log_decay.shape
    n = T // 16
    return log_decay[:, :16 * n].reshape(B, n, 16, H, K).sum(axis=2) / np.log(2.0)


def steep_case(g_min: float, seed: int, T: int = 203):
    d = W.random_scan_case(2, T, 3, 128, 128, seed=seed, dtype="bf16", z_std=2.0, init_std=0.1)
    d["g_min"] = g_min
    d["A_log"] = torch.tensor([0.0, 1.0, -0.5])
    # one block of one head saturates the gate on a few channels (g = g_min on 16 tokens)
    d["z"][0, 16:32, 0, :8] = 30.0
    return d


@pytest.mark.parametrize("g_min", [-6.0, -8.0, -12.0])
@PATHS
def test_prefill_logits_below_the_factorisation_range(kda, g_min, use_workspace):
    d = steep_case(g_min, seed=71)
    g = to_dev(d)
    o, sf = kda.prefill_logits(g["q"], g["k"], g["v"], g["z"], g["A_log"], g_min, g["beta"], g["initial_state"],
                               use_workspace=use_workspace)
    torch.cuda.synchronize()
    assert not kda.device_status()
    alpha, lg = oracle.bounded_decay(d["z"], d["A_log"], g_min, return_log=True)
    sums = block_sums_log2(lg)
    assert (sums < SAFE_LOG2).any(), "the case must reach the pairwise path"
    if g_min > -7:
        assert (sums.min(axis=3) >= SAFE_LOG2).any(), "and keep ordinary blocks too"
    ro, rs = oracle.scan(d["q"], d["k"], d["v"], alpha, d["beta"], d["initial_state"])
    check(o, ro, "bf16", "o")
    check(sf, rs, "bf16", "final_state")


@pytest.mark.parametrize("gate_is_log", [False, True], ids=["alpha", "log-decay"])
@PATHS
def test_prefill_alpha_with_exact_zeros(kda, gate_is_log, use_workspace):
    # alpha = 0 (g = -inf) erases a channel's past entirely; the kernels take it as 2^-126 (g = -87.3),
    # whose remainder is far below what fp32 resolves next to the fresh write.
    d = W.random_scan_case(1, 150, 2, 128, 128, seed=73, dtype="bf16", z_std=2.0, init_std=0.1)
    gen = torch.Generator().manual_seed(74)
    g_ref = d["g_min"] * torch.sigmoid(torch.exp(d["A_log"])[None, None, :, None] * d["z"])
    alpha = torch.exp(g_ref).float()
    alpha[torch.rand(alpha.shape, generator=gen) < 0.05] = 0.0    # scattered zeros
    alpha[0, 40, 1, :] = 0.0                                       # a whole token of head 1
    alpha[0, 64:80, 0, 5] = 0.0                                    # a whole block on one channel
    alpha[0, 100:110] = 1.0                                        # and retention 1
    gate = torch.log(alpha) if gate_is_log else alpha
    assert (alpha == 0).sum() > 100
    g = to_dev(d)
    o, sf = kda.prefill(g["q"], g["k"], g["v"], gate.to(DEV), g["beta"], g["initial_state"], gate_is_log=gate_is_log,
                        use_workspace=use_workspace)
    torch.cuda.synchronize()
    assert not kda.device_status()
    ro, rs = oracle.scan(d["q"], d["k"], d["v"], alpha.double().numpy(), d["beta"], d["initial_state"])
    check(o, ro, "bf16", "o")
    check(sf, rs, "bf16", "final_state")


@PATHS
def test_prefill_steep_gate_varlen_split_resume(kda, use_workspace):
    # packed sequences with their own initial states, in-kernel L2Norm and beta sigmoid, g_min = -9;
    # then the first two sequences again, split mid-chunk and resumed from the final state in place.
    lens = [70, 0, 129, 1, 64, 200]
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    T, H = int(cu[-1]), 2
    d = W.random_scan_case(1, T, H, 128, 128, seed=75, dtype="bf16", z_std=2.0, init_std=None, raw_inputs=True)
    d["cu_seqlens"] = cu
    d["g_min"] = -9.0
    d["initial_state"] = torch.randn(len(lens), H, 128, 128, generator=torch.Generator().manual_seed(76)) * 0.1
    g = to_dev(d)
    kw = dict(qk_l2norm=True, beta_logits=True, use_workspace=use_workspace)
    o, sf = kda.prefill_logits(g["q"], g["k"], g["v"], g["z"], g["A_log"], -9.0, g["beta"], g["initial_state"],
                               g["cu_seqlens"], **kw)
    # sequence 0 (70 tokens) as two calls of 37 and 33 tokens, resuming in place
    st = g["initial_state"][:1].clone()
    parts = []
    for a, b in ((0, 37), (37, 70)):
        oo, _ = kda.prefill_logits(g["q"][:, a:b], g["k"][:, a:b], g["v"][:, a:b], g["z"][:, a:b], g["A_log"], -9.0,
                                   g["beta"][:, a:b], st, final_state=st, **kw)
        parts.append(oo)
    torch.cuda.synchronize()
    assert not kda.device_status()
    alpha, lg = oracle.bounded_decay(d["z"], d["A_log"], -9.0, return_log=True)
    assert (block_sums_log2(lg) < SAFE_LOG2).any()
    q, k, beta = oracle.l2norm(d["q"]), oracle.l2norm(d["k"]), oracle.sigmoid(d["beta"])
    ro, rs = oracle.scan(q, k, d["v"], alpha, beta, d["initial_state"], d["cu_seqlens"])
    check(o, ro, "bf16", "o")
    check(sf, rs, "bf16", "final_state")
    check(torch.cat(parts, 1), ro[:, :70], "bf16", "o (sequence 0, split)")
    check(st, rs[:1], "bf16", "final_state (sequence 0, split)")


@PATHS
def test_prefill_logits_softplus_both_paths(kda, use_workspace):
    # Kimi Linear's unbounded gate, now chunked with or without a workspace.
    d = W.random_scan_case(2, 150, 3, 128, 128, seed=77, dtype="bf16", z_std=2.0, init_std=0.1)
    d["A_log"] = torch.tensor([-1.0, 1.0, 2.5])
    g = to_dev(d)
    o, sf = kda.prefill_logits(g["q"], g["k"], g["v"], g["z"], g["A_log"], g["g_min"], g["beta"], g["initial_state"],
                               gate="softplus", use_workspace=use_workspace)
    torch.cuda.synchronize()
    assert not kda.device_status()
    alpha, lg = oracle.softplus_decay(d["z"], d["A_log"], return_log=True)
    assert (block_sums_log2(lg) < SAFE_LOG2).any()
    ro, rs = oracle.scan(d["q"], d["k"], d["v"], alpha, d["beta"], d["initial_state"])
    check(o, ro, "bf16", "o")
    check(sf, rs, "bf16", "final_state")


@PATHS
def test_prefill_logits_every_option_together(kda, use_workspace):
    # packed ragged sequences with initial states, dt_bias, in-kernel L2Norm and beta sigmoid, value-by-key
    # states and a bounded gate steep enough (g_min = -7) to put some blocks out of range
    lens = [64, 1, 0, 150, 77]
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    T, H = int(cu[-1]), 3
    d = W.random_scan_case(1, T, H, 128, 128, seed=81, dtype="bf16", z_std=2.0, init_std=None, raw_inputs=True)
    d["cu_seqlens"] = cu
    d["A_log"] = torch.tensor([0.8, -0.3, 0.2])
    s0 = torch.randn(len(lens), H, 128, 128, generator=torch.Generator().manual_seed(82)) * 0.1
    b = torch.randn(H, 128, generator=torch.Generator().manual_seed(83))
    g = to_dev(d)
    o, sf = kda.prefill_logits(g["q"], g["k"], g["v"], g["z"], g["A_log"], -7.0, g["beta"],
                               s0.transpose(-1, -2).contiguous().to(DEV), g["cu_seqlens"], qk_l2norm=True,
                               beta_logits=True, state_layout="vk", dt_bias=b.to(DEV), use_workspace=use_workspace)
    torch.cuda.synchronize()
    assert not kda.device_status()
    alpha, lg = oracle.bounded_decay(d["z"], d["A_log"], -7.0, return_log=True, dt_bias=b)
    assert (block_sums_log2(lg) < SAFE_LOG2).any()
    ro, rs = oracle.scan(oracle.l2norm(d["q"]), oracle.l2norm(d["k"]), d["v"], alpha, oracle.sigmoid(d["beta"]),
                         s0, d["cu_seqlens"])
    check(o, ro, "bf16", "o")
    check(sf.transpose(-1, -2), rs, "bf16", "final_state")


@pytest.mark.slow
def test_softplus_prefill_workload_sampled_heads(kda):
    # the bench's unbounded-gate leg: the 4096 x 96 prefill through Kimi Linear's gate on the two-kernel path
    d = W.make_scan_inputs(W.PREFILL)
    g = to_dev(d)
    o, sf = kda.prefill_logits(g["q"], g["k"], g["v"], g["z"], g["A_log"], g["g_min"], g["beta"], None,
                               gate="softplus")
    torch.cuda.synchronize()
    assert not kda.device_status()
    heads = [0, 13, 47, 95]
    alpha, lg = oracle.softplus_decay(d["z"][:, :, heads], d["A_log"][heads], return_log=True)
    assert (block_sums_log2(lg) < SAFE_LOG2).any()
    ro, rs = oracle.scan(d["q"][:, :, heads], d["k"][:, :, heads], d["v"][:, :, heads], alpha, d["beta"][:, :, heads])
    check(o[:, :, heads], ro, "bf16", "o")
    check(sf[:, heads], rs, "bf16", "final_state")
