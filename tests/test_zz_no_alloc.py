"""kda_prefill_noalloc, the prefill that takes its workspace from the library's static scratch.

Collected last (the file name sorts after every other test file) so that it also runs after the
rest of the GPU suite has used the device; it must pass alone in a fresh process too.

Each case calls the allocation-free entry point through the C ABI twice in a row, on different
inputs (and, in the varlen case, a different slot layout), and checks both results against
kda_prefill given a caller-allocated workspace (the existing entry point), with the bf16
tolerance of the GPU parity suite: rms(err) <= 2e-2 rms(ref) plus the elementwise guard
|err| <= 0.05 (|ref| + rms(ref)); fp32: max |err| <= 1e-4. One head of each call is also checked
against the fp64 oracle with the same tolerance.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W

pytestmark = pytest.mark.gpu

DEV = "cuda"
BF16_REL_RMS = 2e-2
GUARD = 0.05
FP32_ATOL = 1e-4


@pytest.fixture(scope="module")
def kda():
    from gated_delta_rule_bounded_b200 import build
    build.build()
    import gated_delta_rule_bounded_b200 as m
    m.load_library()
    return m


def check(got, ref, dtype, what):
    got = got.detach().double().cpu().numpy() if isinstance(got, torch.Tensor) else np.asarray(got, np.float64)
    ref = ref.detach().double().cpu().numpy() if isinstance(ref, torch.Tensor) else np.asarray(ref, np.float64)
    assert got.shape == ref.shape, f"{what}: shape {got.shape} != {ref.shape}"
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    err = np.abs(got - ref)
    if dtype == "f32":
        assert float(err.max()) <= FP32_ATOL, f"{what}: max abs err {float(err.max()):.3e}"
        return
    rms = float(np.sqrt(np.mean(ref ** 2)))
    ratio = float(np.sqrt(np.mean(err ** 2))) / rms
    assert ratio <= BF16_REL_RMS, f"{what}: rms error / rms {ratio:.3e} > {BF16_REL_RMS}"
    worst = float((err / (np.abs(ref) + rms)).max())
    assert worst <= GUARD, f"{what}: elementwise error {worst:.3e} of (|ref| + rms) > {GUARD}"


def inputs(kda, d):
    g = {k: (v.to(DEV) if isinstance(v, torch.Tensor) else v) for k, v in d.items()}
    g["alpha"] = kda.bounded_decay(g["z"], g["A_log"], g["g_min"])
    if g["cu_seqlens"] is not None:
        g["cu_seqlens"] = g["cu_seqlens"].contiguous()
    return g


def run_noalloc(kda, g):
    """The allocation-free call, through the C ABI, into caller-owned out / final_state."""
    B, T, H, _ = g["q"].shape
    V = g["v"].shape[3]
    N = B if g["cu_seqlens"] is None else g["cu_seqlens"].numel() - 1
    out = torch.full((B, T, H, V), float("nan"), device=DEV, dtype=g["q"].dtype)
    sf = torch.full((N, H, g["q"].shape[3], V), float("nan"), device=DEV)
    kda.prefill_noalloc(g["q"], g["k"], g["v"], g["alpha"], g["beta"], out, g["initial_state"], sf,
                        g["cu_seqlens"])
    return out, sf


def compare_one(kda, d, dtype):
    g = inputs(kda, d)
    o_na, sf_na = run_noalloc(kda, g)
    o_ref, sf_ref = kda.prefill(g["q"], g["k"], g["v"], g["alpha"], g["beta"], g["initial_state"],
                                g["cu_seqlens"])
    torch.cuda.synchronize()
    assert not kda.device_status(), "a kernel's bounded wait expired"
    check(o_na, o_ref, dtype, "o vs kda_prefill")
    check(sf_na, sf_ref, dtype, "final_state vs kda_prefill")
    # One head against the fp64 oracle.
    h = [d["q"].shape[2] - 1]
    s0 = d["initial_state"][:, h] if d["initial_state"] is not None else None
    alpha = oracle.bounded_decay(d["z"][:, :, h], d["A_log"][h], d["g_min"])
    ro, rs = oracle.scan(d["q"][:, :, h], d["k"][:, :, h], d["v"][:, :, h], alpha, d["beta"][:, :, h], s0,
                         d["cu_seqlens"])
    check(o_na[:, :, h], ro, dtype, "o vs oracle")
    check(sf_na[:, h], rs, dtype, "final_state vs oracle")


def test_noalloc_two_calls_in_a_row_bf16(kda):
    # First call: 2 x 300 tokens (5 chunks each, ragged tail), 4 heads, V = 256, initial state.
    d1 = W.random_scan_case(2, 300, 4, 128, 256, seed=101, dtype="bf16", z_std=2.0, init_std=0.1)
    need1 = kda.prefill_workspace_bytes(2, 300, 4, 128, 256)
    assert 0 < need1 <= kda.NOALLOC_SCRATCH_BYTES
    compare_one(kda, d1, "bf16")
    # Second call right after, on other values and a smaller shape: the scratch still holds the
    # first call's blocks, which must not leak into this one.
    d2 = W.random_scan_case(1, 190, 3, 128, 128, seed=202, dtype="bf16", z_std=2.0, init_std=None)
    compare_one(kda, d2, "bf16")


def test_noalloc_two_calls_in_a_row_varlen(kda):
    for seed, lens in ((7, [70, 0, 129, 1, 64, 200]), (8, [1, 300, 0, 63])):
        cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
        d = W.random_scan_case(1, int(cu[-1]), 2, 128, 128, seed=seed, dtype="bf16", z_std=2.0, init_std=None)
        d["cu_seqlens"] = cu
        d["initial_state"] = torch.randn(len(lens), 2, 128, 128, generator=torch.Generator().manual_seed(seed)) * 0.1
        compare_one(kda, d, "bf16")


def test_noalloc_fp32_needs_no_scratch(kda):
    assert kda.prefill_workspace_bytes(1, 150, 2, 64, 64, dtype=torch.float32) == 0
    for seed in (3, 4):
        d = W.random_scan_case(1, 150, 2, 64, 64, seed=seed, dtype="f32", z_std=1.0, init_std=0.1)
        compare_one(kda, d, "f32")


def test_noalloc_rejects_sizes_beyond_the_scratch(kda):
    # 4096 tokens x 96 heads need 64 x 96 x 66,048 bytes of workspace, beyond 128 MiB.
    q = torch.zeros(1, 4096, 96, 128, device=DEV, dtype=torch.bfloat16)
    gate = torch.ones(1, 4096, 96, 128, device=DEV)
    beta = torch.zeros(1, 4096, 96, device=DEV)
    out = torch.empty_like(q)
    assert kda.prefill_workspace_bytes(1, 4096, 96, 128, 128) > kda.NOALLOC_SCRATCH_BYTES
    with pytest.raises(kda.KDAError) as e:
        kda.prefill_noalloc(q, q, q, gate, beta, out)
    assert e.value.status == 2 and "static scratch" in str(e.value)
