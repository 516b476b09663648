"""GPU parity: the CUDA path against the fp64 oracle on the same seeded inputs.

Both sides start from the same raw inputs (q, k, v, decay logits z, A_log,
beta, initial state) drawn by ``workloads.py``. The GPU side runs its own gate
kernel and scan kernels through the C ABI; the oracle side runs its own fp64
gate and token-by-token scan. The scan tolerances are those of ``tests/parity.py``
(fp32: max-abs 1e-4; bf16: relative RMS 2e-2 with an elementwise guard, and
max-abs 2e-2 of the RMS on the fp32 final state). The gate's:
|g - g_ref| <= |g_ref| 2^-22 (1 + |e^A z|) for fp32 output (the fp32 rounding of
the sigmoid's argument carried through), within one bf16 rounding (2^-8
relative) for bf16 output.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests.parity import DEV, check, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def kda():
    from gated_delta_rule_bounded_b200 import build
    build.build()
    import gated_delta_rule_bounded_b200 as m
    m.load_library()
    return m


def gpu_pipeline(kda, d, **kw):
    """z -> alpha (gate kernel) -> scan (prefill kernels), all through the C ABI."""
    g = to_dev(d)
    alpha = kda.bounded_decay(g["z"], g["A_log"], g["g_min"])
    o, sf = kda.prefill(g["q"], g["k"], g["v"], alpha, g["beta"], g["initial_state"], g["cu_seqlens"], **kw)
    torch.cuda.synchronize()
    assert not kda.device_status(), "a kernel's bounded wait expired"
    return o, sf


# bf16 prefill runs either as two kernels (state-independent chunk operands for all chunks in
# parallel through a workspace, then the recurrence) or as one fused kernel (no workspace).
PATHS = pytest.mark.parametrize("use_workspace", [True, False], ids=["split", "fused"])


def oracle_pipeline(d, heads=None):
    """Oracle gate and scan, optionally on a subset of heads."""
    sel = (lambda x: x) if heads is None else (lambda x: x[:, :, heads])
    z, q, k, v, beta = (sel(d[n]) for n in ("z", "q", "k", "v", "beta"))
    A = d["A_log"] if heads is None else d["A_log"][heads]
    s0 = d["initial_state"]
    if s0 is not None and heads is not None:
        s0 = s0[:, heads]
    alpha = oracle.bounded_decay(z, A, d["g_min"])
    return oracle.scan(q, k, v, alpha, beta, s0, d["cu_seqlens"])


# ---------------------------------------------------------------------------------------------
# Gate
# ---------------------------------------------------------------------------------------------

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", [(1, 256, 4, 32), (2, 37, 3, 128), (1, 5, 96, 128)])
def test_gate_matches_oracle(kda, dtype, shape):
    g = torch.Generator().manual_seed(sum(shape))
    z = (torch.randn(*shape, generator=g) * 4).to(W.DTYPES[dtype])
    A = torch.randn(shape[2], generator=g) * 0.5
    for g_min in (-5.0, -1.5):
        alpha = kda.bounded_decay(z.to(DEV), A.to(DEV), g_min).double().cpu().numpy()
        lg = kda.bounded_decay(z.to(DEV), A.to(DEV), g_min, log_decay=True).double().cpu().numpy()
        ra, rg = oracle.bounded_decay(z, A, g_min, return_log=True)
        if dtype == "f32":
            # fp32 evaluation: x = e^A z is itself rounded (relative 2^-24), and sigmoid carries
            # that into g with a factor of at most |x|, so |dg| <= |g| 2^-22 (1 + |x|).
            x = np.abs(np.exp(A.double().numpy())[None, None, :, None] * z.double().numpy())
            tol_g = np.abs(rg) * 2.0 ** -22 * (1 + x)
            assert np.all(np.abs(lg - rg) <= tol_g), "log-decay outside the fp32 evaluation bound"
            assert np.all(np.abs(alpha - ra) <= ra * (tol_g + 2.0 ** -22)), "alpha outside the fp32 bound"
        else:
            np.testing.assert_allclose(alpha, ra, rtol=2.0 ** -8, atol=0)
            np.testing.assert_allclose(lg, rg, rtol=2.0 ** -8, atol=1e-30)
        lo = np.exp(g_min) * (1 - (2.0 ** -8 if dtype == "bf16" else 1e-6))  # one rounding of the output
        assert np.all(alpha >= lo) and np.all(alpha <= 1.0)


def test_gate_strided_logits(kda):
    g = torch.Generator().manual_seed(3)
    big = torch.randn(2, 9, 3, 192, generator=g)
    z = big[..., 32:160]                       # a non-contiguous view, rows 16-byte aligned
    A = torch.randn(3, generator=g)
    got = kda.bounded_decay(z.to(DEV), A.to(DEV), -5.0).double().cpu().numpy()
    np.testing.assert_allclose(got, oracle.bounded_decay(z, A, -5.0), rtol=2e-6)


# ---------------------------------------------------------------------------------------------
# Prefill, small cases that span several chunks and a ragged tail
# ---------------------------------------------------------------------------------------------

def test_tiny_fp32_workload(kda):
    """B=1, T=256, H=4, K=V=32, fp32, zero initial state: max-abs <= 1e-4."""
    d = W.make_scan_inputs(W.TINY_FP32)
    o, sf = gpu_pipeline(kda, d)
    ro, rs = oracle_pipeline(d)
    check(o, ro, "f32", "o")
    check(sf, rs, "f32", "final_state")


@pytest.mark.parametrize("B,T,H,K,V,init", [
    (1, 200, 3, 128, 128, False),
    (2, 131, 2, 128, 128, True),
    (1, 64, 2, 128, 256, True),
    (2, 77, 2, 128, 64, True),
    (1, 300, 1, 64, 128, True),
    (1, 1, 2, 128, 128, True),
    (3, 16, 2, 32, 48, True),
])
@PATHS
def test_prefill_bf16_matches_oracle(kda, B, T, H, K, V, init, use_workspace):
    d = W.random_scan_case(B, T, H, K, V, seed=T + H + K, dtype="bf16", z_std=2.0,
                           init_std=0.1 if init else None)
    o, sf = gpu_pipeline(kda, d, use_workspace=use_workspace)
    ro, rs = oracle_pipeline(d)
    check(o, ro, "bf16", "o")
    check(sf, rs, "bf16", "final_state")


@pytest.mark.parametrize("B,T,H,K,V", [(1, 150, 2, 32, 32), (2, 70, 3, 64, 16), (1, 40, 1, 128, 256)])
def test_prefill_fp32_matches_oracle(kda, B, T, H, K, V):
    d = W.random_scan_case(B, T, H, K, V, seed=5 + T, dtype="f32", z_std=1.0, init_std=0.1)
    o, sf = gpu_pipeline(kda, d)
    ro, rs = oracle_pipeline(d)
    check(o, ro, "f32", "o")
    check(sf, rs, "f32", "final_state")


@pytest.mark.parametrize("dtype,use_workspace", [("bf16", True), ("bf16", False), ("f32", True)],
                         ids=["bf16-split", "bf16-fused", "f32"])
def test_prefill_varlen_with_empty_segments(kda, dtype, use_workspace):
    lens = [70, 0, 129, 1, 0, 64, 200]
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    d = W.random_scan_case(1, int(cu[-1]), 2, 128, 128, seed=17, dtype=dtype, z_std=2.0, init_std=None)
    d["cu_seqlens"] = cu
    d["initial_state"] = torch.randn(len(lens), 2, 128, 128, generator=torch.Generator().manual_seed(1)) * 0.1
    o, sf = gpu_pipeline(kda, d, use_workspace=use_workspace)
    ro, rs = oracle_pipeline(d)
    check(o, ro, dtype, "o")
    check(sf, rs, dtype, "final_state")
    # Zero-length sequences return their initial state exactly.
    for n, L in enumerate(lens):
        if L == 0:
            assert torch.equal(sf[n].cpu(), d["initial_state"][n])


@pytest.mark.parametrize("with_init", [True, False])
def test_prefill_empty_sequence(kda, with_init):
    B, H, K, V = 2, 3, 128, 64
    s0 = torch.randn(B, H, K, V) if with_init else None
    z = torch.zeros(B, 0, H, K, device=DEV)
    q = torch.zeros(B, 0, H, K, device=DEV, dtype=torch.bfloat16)
    v = torch.zeros(B, 0, H, V, device=DEV, dtype=torch.bfloat16)
    o, sf = kda.prefill(q, q, v, z, torch.zeros(B, 0, H, device=DEV),
                        None if s0 is None else s0.to(DEV))
    torch.cuda.synchronize()
    assert o.shape == (B, 0, H, V)
    assert torch.equal(sf.cpu(), s0 if with_init else torch.zeros(B, H, K, V))


@PATHS
def test_prefill_strided_views(kda, use_workspace):
    """q, k, v as slices of one fused projection tensor; gate and o as views too."""
    B, T, H, K, V = 2, 97, 3, 128, 128
    g = torch.Generator().manual_seed(8)
    fused = torch.randn(B, T, H, 2 * K + V, generator=g)
    q = torch.nn.functional.normalize(fused[..., :K], dim=-1).bfloat16()
    k = torch.nn.functional.normalize(fused[..., K:2 * K], dim=-1).bfloat16()
    qkv = torch.cat([q, k, fused[..., 2 * K:].bfloat16()], dim=-1).to(DEV)
    zbig = (torch.randn(B, T, H, K + 64, generator=g) * 2)
    A = torch.randn(H, generator=g) * 0.5
    beta_big = torch.sigmoid(torch.randn(B, T, H, 2, generator=g))
    s0 = torch.randn(B, H, K, V, generator=g) * 0.1
    qd, kd, vd = qkv[..., :K], qkv[..., K:2 * K], qkv[..., 2 * K:]
    assert not qd.is_contiguous()
    alpha = kda.bounded_decay(zbig[..., 32:32 + K].to(DEV), A.to(DEV), -5.0)
    o_big = torch.zeros(B, T, H, 2 * V, device=DEV, dtype=torch.bfloat16)
    o, sf = kda.prefill(qd, kd, vd, alpha, beta_big[..., 0].to(DEV), s0.to(DEV), out=o_big[..., V:],
                        use_workspace=use_workspace)
    torch.cuda.synchronize()
    assert o.data_ptr() == o_big[..., V:].data_ptr()
    ra = oracle.bounded_decay(zbig[..., 32:32 + K], A, -5.0)
    ro, rs = oracle.scan(q, k, fused[..., 2 * K:].bfloat16(), ra, beta_big[..., 0], s0)
    check(o, ro, "bf16", "o")
    check(sf, rs, "bf16", "final_state")
    assert torch.count_nonzero(o_big[..., :V]) == 0


def test_prefill_log_gate_and_inputs_untouched(kda):
    d = W.random_scan_case(1, 130, 2, 128, 128, seed=23, dtype="bf16", z_std=2.0, init_std=0.1)
    g = to_dev(d)
    lg = kda.bounded_decay(g["z"], g["A_log"], -5.0, log_decay=True)
    copies = {n: g[n].clone() for n in ("q", "k", "v", "beta", "initial_state")}
    lg_copy = lg.clone()
    o, sf = kda.prefill(g["q"], g["k"], g["v"], lg, g["beta"], g["initial_state"], gate_is_log=True)
    torch.cuda.synchronize()
    for n, c in copies.items():
        assert torch.equal(g[n], c), f"{n} was modified"
    assert torch.equal(lg, lg_copy)
    ro, rs = oracle_pipeline(d)
    check(o, ro, "bf16", "o")
    check(sf, rs, "bf16", "final_state")


@PATHS
def test_prefill_resume_in_place(kda, use_workspace):
    """final_state may alias initial_state; splitting and resuming equals one pass."""
    d = W.random_scan_case(2, 200, 2, 128, 128, seed=31, dtype="bf16", z_std=2.0, init_std=0.1)
    g = to_dev(d)
    alpha = kda.bounded_decay(g["z"], g["A_log"], -5.0)
    kw = dict(use_workspace=use_workspace)
    o_full, s_full = kda.prefill(g["q"], g["k"], g["v"], alpha, g["beta"], g["initial_state"], **kw)
    st = g["initial_state"].clone()
    cut = 77
    o1, _ = kda.prefill(g["q"][:, :cut], g["k"][:, :cut], g["v"][:, :cut], alpha[:, :cut], g["beta"][:, :cut],
                        st, final_state=st, **kw)
    o2, _ = kda.prefill(g["q"][:, cut:], g["k"][:, cut:], g["v"][:, cut:], alpha[:, cut:], g["beta"][:, cut:],
                        st, final_state=st, **kw)
    torch.cuda.synchronize()
    ro, rs = oracle_pipeline(d)
    check(torch.cat([o1, o2], 1), ro, "bf16", "o (split)")
    check(st, rs, "bf16", "final_state (split)")
    check(o_full, ro, "bf16", "o")
    check(s_full, rs, "bf16", "final_state")


# ---------------------------------------------------------------------------------------------
# Decode
# ---------------------------------------------------------------------------------------------

def decode_run(kda, w, steps, heads_sample):
    """Runs `steps` decode steps on the GPU; returns GPU outputs and final state on sampled
    heads plus the oracle's (the oracle scans the sampled heads' steps as one sequence)."""
    prm = W.make_decode_params(w)
    state = prm["state"].to(DEV)
    A = prm["A_log"].to(DEV)
    bsel, hsel = heads_sample
    outs, ins = [], {n: [] for n in ("q", "k", "v", "z", "beta")}
    for s in range(steps):
        st = W.make_decode_step(w, s)
        gd = to_dev(st)
        alpha = kda.bounded_decay(gd["z"], A, w.g_min)
        o = kda.decode_step(gd["q"], gd["k"], gd["v"], alpha, gd["beta"], state)
        outs.append(o[bsel][:, hsel].cpu())
        for n in ins:
            ins[n].append(st[n][bsel][:, hsel])
    torch.cuda.synchronize()
    got_o = torch.stack(outs, 1)                        # [b, steps, h, V]
    got_s = state[bsel][:, hsel].cpu()
    seq = {n: torch.stack(x, 1) for n, x in ins.items()}  # [b, steps, h, *]
    alpha = oracle.bounded_decay(seq["z"], prm["A_log"][hsel], w.g_min)
    ro, rs = oracle.scan(seq["q"], seq["k"], seq["v"], alpha, seq["beta"], prm["state"][bsel][:, hsel])
    return got_o, got_s, ro, rs


def test_decode_small_matches_oracle(kda):
    w = W.DecodeWorkload("decode_small", 3, 4, 128, 128, steps=40)
    got_o, got_s, ro, rs = decode_run(kda, w, 40, (torch.arange(3), torch.arange(4)))
    check(got_o, ro, "bf16", "o")
    check(got_s, rs, "bf16", "state")


def test_decode_more_heads_than_sms(kda):
    """B*H = 600 heads > SM count: each persistent CTA walks several heads through its ring."""
    w = W.DecodeWorkload("decode_many", 5, 120, 128, 128, steps=6)
    got_o, got_s, ro, rs = decode_run(kda, w, 6, (torch.tensor([0, 4]), torch.tensor([0, 59, 119])))
    check(got_o, ro, "bf16", "o")
    check(got_s, rs, "bf16", "state")
    assert not kda.device_status()


@pytest.mark.parametrize("K,V", [(32, 32), (64, 128), (128, 128), (128, 256), (48, 80)])
def test_decode_shapes_fp32(kda, K, V):
    w = W.DecodeWorkload("decode_fp32", 2, 3, K, V, steps=25, dtype="f32")
    got_o, got_s, ro, rs = decode_run(kda, w, 25, (torch.arange(2), torch.arange(3)))
    check(got_o, ro, "f32", "o")
    check(got_s, rs, "f32", "state")


def test_decode_alpha_zero_and_one(kda):
    """Gate end points: alpha = 0 wipes the faded state, alpha = 1 with beta = 0 keeps it."""
    B, H, K, V = 2, 2, 128, 128
    g = torch.Generator().manual_seed(2)
    state = (torch.randn(B, H, K, V, generator=g) * 0.1)
    q = torch.nn.functional.normalize(torch.randn(B, H, K, generator=g), dim=-1).bfloat16()
    k = torch.nn.functional.normalize(torch.randn(B, H, K, generator=g), dim=-1).bfloat16()
    v = torch.randn(B, H, V, generator=g).bfloat16()
    for a_val, b_val in ((0.0, 0.7), (1.0, 0.0)):
        alpha = torch.full((B, H, K), a_val)
        beta = torch.full((B, H), b_val)
        sd = state.clone().to(DEV)
        o = kda.decode_step(q.to(DEV), k.to(DEV), v.to(DEV), alpha.to(DEV), beta.to(DEV), sd)
        torch.cuda.synchronize()
        ro, rs = oracle.scan(q[:, None], k[:, None], v[:, None], alpha[:, None], beta[:, None], state)
        check(o, ro[:, 0], "bf16", "o")
        check(sd, rs, "bf16", "state")


@pytest.mark.slow
def test_decode_workload_1000_steps_sampled(kda):
    """The kept-memory decode workload (B=64, H=96, K=V=128, 1000 steps), every head on the
    GPU, the oracle on a sample of (batch, head) pairs."""
    w = W.DECODE
    bsel = torch.tensor([0, 17, 63])
    hsel = torch.tensor([0, 41, 95])
    got_o, got_s, ro, rs = decode_run(kda, w, w.steps, (bsel, hsel))
    check(got_o, ro, "bf16", "o")
    check(got_s, rs, "bf16", "state")


# ---------------------------------------------------------------------------------------------
# Full-size prefill workloads, sampled heads
# ---------------------------------------------------------------------------------------------

@pytest.mark.slow
@PATHS
def test_prefill_workload_4096_sampled_heads(kda, use_workspace):
    d = W.make_scan_inputs(W.PREFILL)
    o, sf = gpu_pipeline(kda, d, use_workspace=use_workspace)
    heads = [0, 13, 47, 95]
    ro, rs = oracle_pipeline(d, heads)
    check(o[:, :, heads], ro, "bf16", "o")
    check(sf[:, heads], rs, "bf16", "final_state")


@pytest.mark.slow
@PATHS
def test_varlen_workload_sampled_heads(kda, use_workspace):
    d = W.make_scan_inputs(W.VARLEN)
    o, sf = gpu_pipeline(kda, d, use_workspace=use_workspace)
    heads = [3, 60]
    ro, rs = oracle_pipeline(d, heads)
    check(o[:, :, heads], ro, "bf16", "o")
    check(sf[:, heads], rs, "bf16", "final_state")
    cu = d["cu_seqlens"].numpy()
    for n in range(len(cu) - 1):  # per-sequence bound as well
        s, e = cu[n], cu[n + 1]
        check(o[:, s:e][:, :, heads], ro[:, s:e], "bf16", f"o seq {n}")


@pytest.mark.slow
def test_long_kv_workload_split_resume_sampled(kda):
    """B=4, T=16384, H=32, K=128, V=256: one pass, and a split at 8192 resumed from the
    final state, both against the oracle on sampled heads."""
    d = W.make_scan_inputs(W.LONG_KV)
    g = to_dev(d)
    alpha = kda.bounded_decay(g["z"], g["A_log"], -5.0)
    o, sf = kda.prefill(g["q"], g["k"], g["v"], alpha, g["beta"], g["initial_state"])
    half = 8192
    o1, s1 = kda.prefill(g["q"][:, :half], g["k"][:, :half], g["v"][:, :half], alpha[:, :half],
                         g["beta"][:, :half], g["initial_state"])
    o2, s2 = kda.prefill(g["q"][:, half:], g["k"][:, half:], g["v"][:, half:], alpha[:, half:],
                         g["beta"][:, half:], s1)
    torch.cuda.synchronize()
    heads = [5, 30]
    ro, rs = oracle_pipeline(d, heads)
    check(o[:, :, heads], ro, "bf16", "o")
    check(sf[:, heads], rs, "bf16", "final_state")
    check(torch.cat([o1, o2], 1)[:, :, heads], ro, "bf16", "o (split)")
    check(s2[:, heads], rs, "bf16", "final_state (split)")


# ---------------------------------------------------------------------------------------------
# Gate inside the scan (kda_prefill_logits / kda_decode_step_logits)
# ---------------------------------------------------------------------------------------------
# Both evaluate eq. 5 with the gate kernel's own device function, so a scan fed with the logits
# must equal, bit for bit, the gate kernel followed by the scan on its output (log-decay for the
# chunked bf16 kernels, which take log2 of it; alpha for the token-by-token kernel).

@pytest.mark.parametrize("dtype,use_workspace,cu", [("bf16", True, False), ("bf16", False, False),
                                                    ("bf16", True, True), ("f32", True, False)],
                         ids=["bf16-split", "bf16-fused", "bf16-varlen", "f32"])
def test_prefill_logits_equals_gate_then_scan(kda, dtype, use_workspace, cu):
    B, T, H = (1, 333, 3) if cu else (2, 200, 3)
    d = W.random_scan_case(B, T, H, 128, 128, seed=41, dtype=dtype, z_std=2.0, init_std=0.1)
    if cu:
        lens = [100, 0, 64, 169]
        d["cu_seqlens"] = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
        d["initial_state"] = torch.randn(len(lens), H, 128, 128, generator=torch.Generator().manual_seed(2)) * 0.1
    g = to_dev(d)
    use_log = dtype == "bf16"
    gate = kda.bounded_decay(g["z"], g["A_log"], g["g_min"], log_decay=use_log)
    o_ref, s_ref = kda.prefill(g["q"], g["k"], g["v"], gate, g["beta"], g["initial_state"], g["cu_seqlens"],
                               gate_is_log=use_log, use_workspace=use_workspace)
    o, sf = kda.prefill_logits(g["q"], g["k"], g["v"], g["z"], g["A_log"], g["g_min"], g["beta"],
                               g["initial_state"], g["cu_seqlens"], use_workspace=use_workspace)
    torch.cuda.synchronize()
    assert not kda.device_status()
    assert torch.equal(o, o_ref) and torch.equal(sf, s_ref)
    ro, rs = oracle_pipeline(d)
    check(o, ro, dtype, "o")
    check(sf, rs, dtype, "final_state")


@pytest.mark.parametrize("K,V,dtype", [(128, 128, "bf16"), (64, 32, "f32")], ids=["bulk", "token-kernel"])
def test_decode_logits_equals_gate_then_step(kda, K, V, dtype):
    B, H = 3, 5
    gen = torch.Generator().manual_seed(9)
    dt = W.DTYPES[dtype]
    q = torch.nn.functional.normalize(torch.randn(B, H, K, generator=gen), dim=-1).to(dt).to(DEV)
    k = torch.nn.functional.normalize(torch.randn(B, H, K, generator=gen), dim=-1).to(dt).to(DEV)
    v = torch.randn(B, H, V, generator=gen).to(dt).to(DEV)
    z = (torch.randn(B, H, K, generator=gen) * 2).to(DEV)
    A_log = (torch.randn(H, generator=gen) * 0.5).to(DEV)
    beta = torch.sigmoid(torch.randn(B, H, generator=gen)).to(DEV)
    s0 = (torch.randn(B, H, K, V, generator=gen) * 0.1).to(DEV)
    s_ref, s_new = s0.clone(), s0.clone()
    for _ in range(3):
        alpha = kda.bounded_decay(z, A_log, -5.0)
        o_ref = kda.decode_step(q, k, v, alpha, beta, s_ref)
        o = kda.decode_step_logits(q, k, v, z, A_log, -5.0, beta, s_new)
    torch.cuda.synchronize()
    assert not kda.device_status()
    assert torch.equal(o, o_ref) and torch.equal(s_new, s_ref)


# ---------------------------------------------------------------------------------------------
# The logits' bias (dt_bias [H,K], "KDA cheat sheet", How the inputs are produced: z = W_up W_down x + b)
# ---------------------------------------------------------------------------------------------
# The kernels add the bias to z in fp32 before the gate, so a call with the bias must equal, bit for
# bit, the same call without it on z + dt_bias summed by the caller in fp32; the oracle adds the bias
# in fp64 before its own gate.

def bias_for(H, K, seed):
    return torch.randn(H, K, generator=torch.Generator().manual_seed(seed)) * 1.5


@pytest.mark.parametrize("dtype,use_workspace,gate", [("bf16", True, "bounded"), ("bf16", False, "bounded"),
                                                      ("bf16", True, "softplus"), ("f32", True, "bounded")],
                         ids=["bf16-split", "bf16-fused", "bf16-softplus", "f32"])
def test_prefill_logits_with_dt_bias(kda, dtype, use_workspace, gate):
    B, T, H = 2, 150, 3
    d = W.random_scan_case(B, T, H, 128, 128, seed=51, dtype=dtype, z_std=2.0, init_std=0.1)
    b = bias_for(H, 128, 52)
    g = to_dev(d)
    kw = dict(gate=gate, use_workspace=use_workspace)
    o, sf = kda.prefill_logits(g["q"], g["k"], g["v"], g["z"], g["A_log"], g["g_min"], g["beta"], g["initial_state"],
                               dt_bias=b.to(DEV), **kw)
    zb = (d["z"] + b[None, None]).to(DEV)
    o2, s2 = kda.prefill_logits(g["q"], g["k"], g["v"], zb, g["A_log"], g["g_min"], g["beta"], g["initial_state"], **kw)
    torch.cuda.synchronize()
    assert not kda.device_status()
    assert torch.equal(o, o2) and torch.equal(sf, s2)
    if gate == "softplus":
        alpha = oracle.softplus_decay(d["z"], d["A_log"], dt_bias=b)
    else:
        alpha = oracle.bounded_decay(d["z"], d["A_log"], d["g_min"], dt_bias=b)
    ro, rs = oracle.scan(d["q"], d["k"], d["v"], alpha, d["beta"], d["initial_state"])
    check(o, ro, dtype, "o")
    check(sf, rs, dtype, "final_state")


@pytest.mark.parametrize("K,V,dtype", [(128, 128, "bf16"), (64, 32, "f32")], ids=["bulk", "token-kernel"])
def test_decode_logits_with_dt_bias(kda, K, V, dtype):
    B, T, H = 3, 4, 5
    d = W.random_scan_case(B, T, H, K, V, seed=53, dtype=dtype, z_std=2.0, init_std=0.1)
    b = bias_for(H, K, 54)
    g = to_dev(d)
    st, st2 = g["initial_state"].clone(), g["initial_state"].clone()
    outs, outs2 = [], []
    for t in range(T):
        outs.append(kda.decode_step_logits(g["q"][:, t], g["k"][:, t], g["v"][:, t], g["z"][:, t], g["A_log"],
                                           g["g_min"], g["beta"][:, t], st, dt_bias=b.to(DEV)))
        zb = (d["z"][:, t] + b[None]).to(DEV)
        outs2.append(kda.decode_step_logits(g["q"][:, t], g["k"][:, t], g["v"][:, t], zb, g["A_log"], g["g_min"],
                                            g["beta"][:, t], st2))
    torch.cuda.synchronize()
    assert not kda.device_status()
    o = torch.stack(outs, 1)
    assert torch.equal(o, torch.stack(outs2, 1)) and torch.equal(st, st2)
    alpha = oracle.bounded_decay(d["z"], d["A_log"], d["g_min"], dt_bias=b)
    ro, rs = oracle.scan(d["q"], d["k"], d["v"], alpha, d["beta"], d["initial_state"])
    check(o, ro, dtype, "o")
    check(st, rs, dtype, "state")


# ---------------------------------------------------------------------------------------------
# Input preparation inside the kernels (KDA_QK_L2NORM, KDA_BETA_LOGITS)
# ---------------------------------------------------------------------------------------------
# The oracle prepares the raw inputs itself (fp64 L2Norm of q and k over K, sigmoid of the beta
# logits) and scans; the GPU gets the raw q, k and beta logits. Tolerances as everywhere else.

def oracle_prepared(d, heads=None):
    sel = (lambda x: x) if heads is None else (lambda x: x[:, :, heads])
    z, q, k, v, b = (sel(d[n]) for n in ("z", "q", "k", "v", "beta"))
    A = d["A_log"] if heads is None else d["A_log"][heads]
    s0 = d["initial_state"]
    if s0 is not None and heads is not None:
        s0 = s0[:, heads]
    alpha = oracle.bounded_decay(z, A, d["g_min"])
    return oracle.scan(oracle.l2norm(q), oracle.l2norm(k), v, alpha, oracle.sigmoid(b), s0, d["cu_seqlens"])


@pytest.mark.parametrize("dtype,use_workspace,cu", [("bf16", True, False), ("bf16", False, False),
                                                    ("bf16", True, True), ("f32", True, False)],
                         ids=["bf16-split", "bf16-fused", "bf16-varlen", "f32"])
def test_prefill_logits_prepares_q_k_beta(kda, dtype, use_workspace, cu):
    B, T, H, K = (1, 333, 3, 128) if cu else ((2, 200, 3, 128) if dtype == "bf16" else (2, 90, 2, 64))
    d = W.random_scan_case(B, T, H, K, 128, seed=77, dtype=dtype, z_std=2.0, init_std=0.1, raw_inputs=True)
    if cu:
        lens = [100, 0, 64, 169]
        d["cu_seqlens"] = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
        d["initial_state"] = torch.randn(len(lens), H, K, 128, generator=torch.Generator().manual_seed(5)) * 0.1
    g = to_dev(d)
    o, sf = kda.prefill_logits(g["q"], g["k"], g["v"], g["z"], g["A_log"], g["g_min"], g["beta"],
                               g["initial_state"], g["cu_seqlens"], qk_l2norm=True, beta_logits=True,
                               use_workspace=use_workspace)
    torch.cuda.synchronize()
    assert not kda.device_status()
    ro, rs = oracle_prepared(d)
    check(o, ro, dtype, "o")
    check(sf, rs, dtype, "final_state")


@pytest.mark.parametrize("K,V,dtype", [(128, 128, "bf16"), (64, 32, "f32")], ids=["bulk", "token-kernel"])
def test_decode_logits_prepares_q_k_beta(kda, K, V, dtype):
    d = W.random_scan_case(4, 3, 5, K, V, seed=19, dtype=dtype, z_std=1.0, init_std=0.1, raw_inputs=True)
    g = to_dev(d)
    state = g["initial_state"].clone()
    outs = []
    for t in range(3):
        outs.append(kda.decode_step_logits(g["q"][:, t], g["k"][:, t], g["v"][:, t], g["z"][:, t], g["A_log"],
                                           g["g_min"], g["beta"][:, t], state, qk_l2norm=True, beta_logits=True))
    torch.cuda.synchronize()
    assert not kda.device_status()
    ro, rs = oracle_prepared(d)
    check(torch.stack(outs, dim=1), ro, dtype, "o")
    check(state, rs, dtype, "state")


# ---------------------------------------------------------------------------------------------
# Value-by-key state layout (KDA_STATE_VK): states [N,H,V,K]
# ---------------------------------------------------------------------------------------------

@pytest.mark.parametrize("dtype,use_workspace,K,V", [("bf16", True, 128, 256), ("bf16", False, 128, 128),
                                                      ("f32", True, 64, 32)],
                         ids=["bf16-split-V256", "bf16-fused", "f32"])
def test_prefill_logits_value_by_key_states(kda, dtype, use_workspace, K, V):
    d = W.random_scan_case(2, 150, 3, K, V, seed=23, dtype=dtype, z_std=2.0, init_std=0.1)
    g = to_dev(d)
    s0_vk = g["initial_state"].transpose(-1, -2).contiguous()
    o, sf_vk = kda.prefill_logits(g["q"], g["k"], g["v"], g["z"], g["A_log"], g["g_min"], g["beta"], s0_vk,
                                  state_layout="vk", use_workspace=use_workspace)
    torch.cuda.synchronize()
    assert not kda.device_status()
    assert sf_vk.shape == (2, 3, V, K)
    ro, rs = oracle_pipeline(d)
    check(o, ro, dtype, "o")
    check(sf_vk.transpose(-1, -2), rs, dtype, "final_state")


@pytest.mark.parametrize("K,V,dtype", [(128, 128, "bf16"), (128, 128, "f32"), (64, 32, "f32")],
                         ids=["bulk-bf16", "bulk-f32", "token-kernel"])
def test_decode_logits_value_by_key_state(kda, K, V, dtype):
    d = W.random_scan_case(4, 3, 5, K, V, seed=31, dtype=dtype, z_std=1.0, init_std=0.1, raw_inputs=True)
    g = to_dev(d)
    state_vk = g["initial_state"].transpose(-1, -2).contiguous()
    outs = []
    for t in range(3):
        outs.append(kda.decode_step_logits(g["q"][:, t], g["k"][:, t], g["v"][:, t], g["z"][:, t], g["A_log"],
                                           g["g_min"], g["beta"][:, t], state_vk, qk_l2norm=True, beta_logits=True,
                                           state_layout="vk"))
    torch.cuda.synchronize()
    assert not kda.device_status()
    ro, rs = oracle_prepared(d)
    check(torch.stack(outs, dim=1), ro, dtype, "o")
    check(state_vk.transpose(-1, -2), rs, dtype, "state")


# ---------------------------------------------------------------------------------------------
# Kimi Linear's unbounded gate (KDA_GATE_SOFTPLUS, kda_softplus_decay)
# ---------------------------------------------------------------------------------------------
# fp32 gate: |g - g_ref| <= |g_ref| 2^-20 (expf, log1pf and the e^A product, each a few ulp; no argument
# rounding enters since softplus reads z directly). The scans use the tolerances above.

def oracle_softplus_pipeline(d):
    alpha = oracle.softplus_decay(d["z"], d["A_log"])
    return oracle.scan(d["q"], d["k"], d["v"], alpha, d["beta"], d["initial_state"], d["cu_seqlens"])


def test_softplus_gate_matches_oracle(kda):
    d = W.random_scan_case(2, 300, 3, 128, 32, seed=13, dtype="f32", z_std=4.0, init_std=None)
    g = kda.softplus_decay(d["z"].to(DEV), d["A_log"].to(DEV), log_decay=True)
    torch.cuda.synchronize()
    _, ref = oracle.softplus_decay(d["z"], d["A_log"], return_log=True)
    err = np.abs(g.double().cpu().numpy() - ref)
    assert np.all(err <= np.abs(ref) * 2.0 ** -20), float((err / np.abs(ref)).max())
    assert ref.min() < -20.0  # the decay is far below what a bounded gate allows


@pytest.mark.parametrize("dtype,use_workspace", [("bf16", True), ("bf16", False), ("f32", True)],
                         ids=["bf16-split", "bf16-fused", "f32"])
def test_prefill_logits_softplus_gate(kda, dtype, use_workspace):
    d = W.random_scan_case(2, 150, 3, 128, 128, seed=43, dtype=dtype, z_std=2.0, init_std=0.1)
    g = to_dev(d)
    o, sf = kda.prefill_logits(g["q"], g["k"], g["v"], g["z"], g["A_log"], g["g_min"], g["beta"],
                               g["initial_state"], gate="softplus", use_workspace=use_workspace)
    torch.cuda.synchronize()
    assert not kda.device_status()
    ro, rs = oracle_softplus_pipeline(d)
    check(o, ro, dtype, "o")
    check(sf, rs, dtype, "final_state")


def test_prefill_logits_softplus_chunked_extreme_decay(kda):
    # The chunked path of the unbounded gate, with heads whose decay within one 16-token block is far past
    # what the block-boundary factorisation can hold (exp of thousands), packed ragged sequences with their
    # own initial states, and q, k, beta prepared inside the kernels; against the fp64 oracle.
    lens = [70, 0, 129, 1, 64, 200]
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32)
    T, H, K, V = int(cu[-1]), 4, 128, 128
    d = W.random_scan_case(1, T, H, K, V, seed=61, dtype="bf16", z_std=4.0, init_std=None, raw_inputs=True)
    d["A_log"] = torch.tensor([-1.0, 0.5, 2.0, 4.0])
    d["cu_seqlens"] = cu
    d["initial_state"] = torch.randn(len(lens), H, K, V, generator=torch.Generator().manual_seed(62)) * 0.1
    g = to_dev(d)
    o, sf = kda.prefill_logits(g["q"], g["k"], g["v"], g["z"], g["A_log"], g["g_min"], g["beta"], g["initial_state"],
                               g["cu_seqlens"], qk_l2norm=True, beta_logits=True, gate="softplus")
    torch.cuda.synchronize()
    assert not kda.device_status()
    alpha, lg = oracle.softplus_decay(d["z"], d["A_log"], return_log=True)
    # the last heads' decay over some 16-token block is beyond the fp32 range of its reciprocal
    assert float(lg[0, :16, 3].sum(axis=0).min()) < -200.0
    ro, rs = oracle.scan(oracle.l2norm(d["q"]), oracle.l2norm(d["k"]), d["v"], alpha, oracle.sigmoid(d["beta"]),
                         d["initial_state"], d["cu_seqlens"])
    check(o, ro, "bf16", "o")
    check(sf, rs, "bf16", "final_state")


def test_decode_logits_softplus_gate(kda):
    d = W.random_scan_case(4, 3, 5, 128, 128, seed=47, dtype="bf16", z_std=2.0, init_std=0.1)
    g = to_dev(d)
    state = g["initial_state"].clone()
    outs = [kda.decode_step_logits(g["q"][:, t], g["k"][:, t], g["v"][:, t], g["z"][:, t], g["A_log"], g["g_min"],
                                   g["beta"][:, t], state, gate="softplus") for t in range(3)]
    torch.cuda.synchronize()
    assert not kda.device_status()
    ro, rs = oracle_softplus_pipeline(d)
    check(torch.stack(outs, dim=1), ro, "bf16", "o")
    check(state, rs, "bf16", "state")


# ---------------------------------------------------------------------------------------------
# Gradients: kda_scan_backward, kda_bounded_decay_backward against the fp64 autograd oracle
# ---------------------------------------------------------------------------------------------
# The backward kernel works in fp32 for either input dtype (bf16 inputs are exact fp32 values), so one
# bound serves both: |grad - ref| <= 3e-4 (|ref| + rms(ref)) elementwise, per gradient. A single fp32
# rounding per operation over a few hundred dependent steps stays far inside it; a wrong term or index
# does not.

def check_grad(got, ref, what):
    got = got.detach().double().cpu().numpy()
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, f"{what}: shape {got.shape} != {ref.shape}"
    rms = float(np.sqrt(np.mean(ref ** 2))) + 1e-30
    worst = float((np.abs(got - ref) / (np.abs(ref) + rms)).max())
    assert worst <= 3e-4, f"{what}: elementwise error {worst:.3e} of (|ref| + rms)"


@pytest.mark.parametrize("B,T,H,K,V,dtype,log_gate", [(2, 100, 2, 64, 64, "f32", False),
                                                       (1, 70, 2, 128, 128, "bf16", True),
                                                       (2, 33, 3, 32, 16, "f32", True)])
def test_scan_backward_matches_autograd_oracle(kda, B, T, H, K, V, dtype, log_gate):
    d = W.random_scan_case(B, T, H, K, V, seed=T + K, dtype=dtype, z_std=2.0, init_std=0.1)
    gen = torch.Generator().manual_seed(T)
    do = torch.randn(B, T, H, V, generator=gen)
    dsf = torch.randn(B, H, K, V, generator=gen) * 0.1
    alpha, lg = oracle.bounded_decay(d["z"], d["A_log"], d["g_min"], return_log=True)
    gate = torch.tensor(lg if log_gate else alpha, dtype=torch.float32)
    gd = to_dev(d)
    out = kda.scan_backward(gd["q"], gd["k"], gd["v"], gate.to(DEV), gd["beta"], gd["initial_state"], do.to(DEV),
                            dsf.to(DEV), gate_is_log=log_gate)
    torch.cuda.synchronize()
    # the oracle sees exactly the gate values the GPU read
    a_used = np.exp(gate.double().numpy()) if log_gate else gate.double().numpy()
    ref = oracle.scan_backward(d["q"], d["k"], d["v"], a_used, d["beta"], d["initial_state"], do, dsf)
    for n, key in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("beta", "dbeta"), ("initial_state", "d_initial_state")):
        check_grad(out[key], ref[n], key)
    check_grad(out["dgate"], ref["alpha"] * a_used if log_gate else ref["alpha"], "dgate")


@pytest.mark.parametrize("dtype,K,V", [("bf16", 128, 128), ("f32", 64, 32)])
def test_scan_backward_varlen_matches_oracle_per_sequence(kda, dtype, K, V):
    # Packed sequences of ragged lengths (one empty, one of a single token, several crossing the 32-token
    # checkpoint segments), each with its own initial state and dL/dS_T; every sequence must get the
    # gradients of its own scan, and an empty one dL/dS_0 = dL/dS_T.
    lens = [70, 0, 129, 1, 64, 33]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    N, T, H = len(lens), int(cu[-1]), 2
    d = W.random_scan_case(1, T, H, K, V, seed=41, dtype=dtype, z_std=2.0, init_std=None)
    gen = torch.Generator().manual_seed(42)
    s0 = torch.randn(N, H, K, V, generator=gen) * 0.1
    dsf = torch.randn(N, H, K, V, generator=gen) * 0.1
    do = torch.randn(1, T, H, V, generator=gen)
    _, lg = oracle.bounded_decay(d["z"], d["A_log"], d["g_min"], return_log=True)
    gate = torch.tensor(lg, dtype=torch.float32)
    gd = to_dev(d)
    out = kda.scan_backward(gd["q"], gd["k"], gd["v"], gate.to(DEV), gd["beta"], s0.to(DEV), do.to(DEV), dsf.to(DEV),
                            cu_seqlens=torch.tensor(cu).to(DEV), gate_is_log=True)
    torch.cuda.synchronize()
    a_used = np.exp(gate.double().numpy())
    for n in range(N):
        a, b = int(cu[n]), int(cu[n + 1])
        if a == b:
            np.testing.assert_array_equal(out["d_initial_state"][n].cpu().numpy(), dsf[n].numpy())
            continue
        sl = lambda x: x[:, a:b]  # noqa: E731
        ref = oracle.scan_backward(sl(d["q"]), sl(d["k"]), sl(d["v"]), a_used[:, a:b], sl(d["beta"]), s0[n:n + 1],
                                   do[:, a:b], dsf[n:n + 1])
        for name, key in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("beta", "dbeta")):
            check_grad(out[key][:, a:b], ref[name], f"{key} of sequence {n}")
        check_grad(out["dgate"][:, a:b], ref["alpha"] * a_used[:, a:b], f"dgate of sequence {n}")
        check_grad(out["d_initial_state"][n:n + 1], ref["initial_state"], f"d_initial_state of sequence {n}")


@pytest.mark.parametrize("B,T,H,K", [(1, 37, 2, 6), (2, 300, 3, 128)])
def test_gate_backward_paths(kda, B, T, H, K):
    # K = 6: the scalar path (rows are not whole float4s); 2 x 300 x 3 x 128: many row blocks per head, whose
    # partial sums of dL/dA_log meet in one atomic each.
    gen = torch.Generator().manual_seed(K + T)
    z = torch.randn(B, T, H, K, generator=gen) * 2.0
    A_log = torch.randn(H, generator=gen) * 0.5
    dg = torch.randn(B, T, H, K, generator=gen)
    dz, dA = kda.bounded_decay_backward(z.to(DEV), A_log.to(DEV), -5.0, dg.to(DEV))
    torch.cuda.synchronize()
    rz, rA = oracle.bounded_decay_backward(z, A_log, -5.0, dg)
    check_grad(dz, rz, "dz")
    np.testing.assert_allclose(dA.double().cpu().numpy(), rA, rtol=1e-4, atol=1e-4 * float(np.abs(rA).max()))


def test_gate_backward_matches_autograd_oracle(kda):
    d = W.random_scan_case(2, 50, 3, 64, 16, seed=3, dtype="f32", z_std=2.0, init_std=None)
    dg = torch.randn(2, 50, 3, 64, generator=torch.Generator().manual_seed(4))
    dz, dA = kda.bounded_decay_backward(d["z"].to(DEV), d["A_log"].to(DEV), d["g_min"], dg.to(DEV))
    torch.cuda.synchronize()
    rz, rA = oracle.bounded_decay_backward(d["z"], d["A_log"], d["g_min"], dg)
    check_grad(dz, rz, "dz")
    np.testing.assert_allclose(dA.double().cpu().numpy(), rA, rtol=1e-4, atol=1e-4)


def test_usage_example_calls(kda):
    # A short tour of the Python API at a small size: every call must accept what is passed (views
    # included) and return finite values of the documented shapes.
    B, T, H, K, V = 1, 130, 4, 128, 128
    gen = torch.Generator().manual_seed(11)
    q, k = (torch.randn(B, T, H, K, generator=gen).to(DEV, torch.bfloat16) for _ in range(2))
    v = torch.randn(B, T, H, V, generator=gen).to(DEV, torch.bfloat16)
    z = torch.randn(B, T, H, K, generator=gen).to(DEV)
    A_log = torch.zeros(H, device=DEV)
    beta = torch.rand(B, T, H, generator=gen).to(DEV)
    o, S = kda.prefill_logits(q, k, v, z, A_log, -5.0, beta, qk_l2norm=True)
    assert o.shape == (B, T, H, V) and S.shape == (B, H, K, V)
    o1 = kda.decode_step_logits(q[:, 0], k[:, 0], v[:, 0], z[:, 0], A_log, -5.0, beta[:, 0], S)
    assert o1.shape == (B, H, V)
    g = kda.bounded_decay(z, A_log, -5.0, log_decay=True)
    grads = kda.scan_backward(q, k, v, g, beta, None, torch.randn_like(o, dtype=torch.float32), gate_is_log=True)
    dz, dA_log = kda.bounded_decay_backward(z, A_log, -5.0, grads["dgate"])
    torch.cuda.synchronize()
    assert not kda.device_status()
    for t in (o, S, o1, dz, dA_log, *grads.values()):
        assert torch.isfinite(t.float()).all()
