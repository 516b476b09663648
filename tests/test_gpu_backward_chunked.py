"""kda_scan_backward_chunked (gradients through the chunkwise form, parallel over chunks) against the fp64
autograd oracle.

Tolerance (reading of the pages' bf16 bound for gradients computed from bf16 tensor-core states): per
gradient, relative RMS error rms(gpu - oracle) <= 2e-3 rms(oracle) and the elementwise guard
|gpu - oracle| <= 0.05 (|oracle| + rms(oracle)). The chunk-start states come from the bf16 forward; every
other step is fp32 (the batched products on TF32 tensor cores). Measured: relative RMS 1e-5 to 5e-4, guard
at most 1.3e-2 on these cases.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda"
RMS, GUARD = 2e-3, 0.05


def check(got, ref, what):
    got = got.detach().double().cpu().numpy()
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape and np.all(np.isfinite(got)), what
    rms = float(np.sqrt(np.mean(ref ** 2))) + 1e-30
    err = np.abs(got - ref)
    ratio = float(np.sqrt(np.mean(err ** 2))) / rms
    guard = float((err / (np.abs(ref) + rms)).max())
    assert ratio <= RMS and guard <= GUARD, f"{what}: rms ratio {ratio:.2e} (<= {RMS}), guard {guard:.2e} (<= {GUARD})"


@pytest.fixture(scope="module")
def kda():
    import gated_delta_rule_bounded_b200 as k
    k.load_library()
    return k


@pytest.mark.parametrize("B,T,H,seed,log_gate,init,dsf,g_min", [
    (1, 70, 2, 3, True, False, False, None),     # ragged last chunk, zero states
    (2, 200, 3, 5, True, True, True, None),      # batch rows, initial state, dL/dS_T
    (1, 129, 2, 7, False, True, True, None),     # alpha given (dL/dalpha), one token in the last chunk
    (1, 96, 2, 9, True, True, True, -12.0),      # steep decay: 16-token blocks far below e^-80
    (1, 64, 1, 11, True, True, True, None),      # exactly one chunk
])
def test_chunked_backward_matches_autograd_oracle(kda, B, T, H, seed, log_gate, init, dsf, g_min):
    d = W.random_scan_case(B, T, H, 128, 128, seed=seed, dtype="bf16", z_std=2.0, init_std=0.1 if init else None)
    if g_min is not None:
        d["g_min"] = g_min
    gen = torch.Generator().manual_seed(seed + 1)
    do = torch.randn(B, T, H, 128, generator=gen)
    d_sf = torch.randn(B, H, 128, 128, generator=gen) * 0.1 if dsf else None
    alpha, lg = oracle.bounded_decay(d["z"], d["A_log"], d["g_min"], return_log=True)
    gate = torch.tensor(lg if log_gate else alpha, dtype=torch.float32)
    s0 = d["initial_state"]
    out = kda.scan_backward_chunked(d["q"].to(DEV), d["k"].to(DEV), d["v"].to(DEV), gate.to(DEV), d["beta"].to(DEV),
                                    None if s0 is None else s0.to(DEV), do.to(DEV),
                                    None if d_sf is None else d_sf.to(DEV), gate_is_log=log_gate)
    torch.cuda.synchronize()
    assert not kda.device_status()
    a_used = np.exp(gate.double().numpy()) if log_gate else gate.double().numpy()
    ref = oracle.scan_backward(d["q"], d["k"], d["v"], a_used, d["beta"], s0, do, d_sf)
    for n, key in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("beta", "dbeta"), ("initial_state", "d_initial_state")):
        check(out[key], ref[n], key)
    check(out["dgate"], ref["alpha"] * a_used if log_gate else ref["alpha"], "dgate")


def test_chunked_backward_empty_and_errors(kda):
    q = torch.zeros(1, 0, 2, 128, device=DEV, dtype=torch.bfloat16)
    v = torch.zeros(1, 0, 2, 128, device=DEV, dtype=torch.bfloat16)
    g = torch.zeros(1, 0, 2, 128, device=DEV)
    b = torch.zeros(1, 0, 2, device=DEV)
    dsf = torch.randn(1, 2, 128, 128, device=DEV)
    out = kda.scan_backward_chunked(q, q, v, g, b, None, torch.zeros(1, 0, 2, 128, device=DEV), dsf, gate_is_log=True)
    torch.cuda.synchronize()
    assert torch.equal(out["d_initial_state"], dsf)  # T = 0: dL/dS_0 = dL/dS_T
    d = W.random_scan_case(1, 70, 2, 128, 128, seed=3, dtype="bf16", z_std=2.0, init_std=None)
    _, lg = oracle.bounded_decay(d["z"], d["A_log"], d["g_min"], return_log=True)
    small = torch.empty(16, device=DEV, dtype=torch.uint8)
    with pytest.raises(kda.KDAError):
        kda.scan_backward_chunked(d["q"].to(DEV), d["k"].to(DEV), d["v"].to(DEV), torch.tensor(lg).float().to(DEV),
                                  d["beta"].to(DEV), None, torch.zeros(1, 70, 2, 128, device=DEV), None,
                                  gate_is_log=True, workspace=small)


def test_chunked_backward_packed_sequences_match_oracle_per_sequence(kda):
    # Packed sequences of ragged lengths starting anywhere inside a 64-token chunk (one empty, one of a single
    # token, one exactly a chunk long, several crossing chunk boundaries), each with its own initial state and
    # dL/dS_T; tokens before the first and after the last sequence belong to none. Every sequence must get the
    # gradients of its own scan, an empty one dL/dS_0 = dL/dS_T, and the tokens outside every sequence zero.
    lens = [70, 0, 129, 1, 64, 33, 200]
    cu = np.concatenate([[3], 3 + np.cumsum(lens)]).astype(np.int32)
    N, T, H = len(lens), int(cu[-1]) + 5, 2
    d = W.random_scan_case(1, T, H, 128, 128, seed=43, dtype="bf16", z_std=2.0, init_std=None)
    gen = torch.Generator().manual_seed(44)
    s0 = torch.randn(N, H, 128, 128, generator=gen) * 0.1
    dsf = torch.randn(N, H, 128, 128, generator=gen) * 0.1
    do = torch.randn(1, T, H, 128, generator=gen)
    _, lg = oracle.bounded_decay(d["z"], d["A_log"], d["g_min"], return_log=True)
    gate = torch.tensor(lg, dtype=torch.float32)
    out = kda.scan_backward_chunked(d["q"].to(DEV), d["k"].to(DEV), d["v"].to(DEV), gate.to(DEV), d["beta"].to(DEV),
                                    s0.to(DEV), do.to(DEV), dsf.to(DEV), cu_seqlens=torch.tensor(cu).to(DEV),
                                    gate_is_log=True)
    torch.cuda.synchronize()
    assert not kda.device_status()
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
            check(out[key][:, a:b], ref[name], f"{key} of sequence {n}")
        check(out["dgate"][:, a:b], ref["alpha"] * a_used[:, a:b], f"dgate of sequence {n}")
        check(out["d_initial_state"][n:n + 1], ref["initial_state"], f"d_initial_state of sequence {n}")
    outside = torch.cat([torch.arange(0, int(cu[0])), torch.arange(int(cu[-1]), T)])
    for key in ("dq", "dk", "dv", "dgate", "dbeta"):
        assert torch.count_nonzero(out[key][:, outside]) == 0, key
