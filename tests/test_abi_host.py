"""Host-side checks of the C ABI (no GPU needed).

The library must load and export every function that ``include/kda.h``
declares, and every argument error must be reported with its status code
before anything is launched, so these calls never touch a device.
"""
import ctypes
import os
import re
import subprocess

import pytest

import gated_delta_rule_bounded_b200 as kda
from gated_delta_rule_bounded_b200 import Layout, Strides

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kda.h")

OK, INVALID, UNSUPPORTED = 0, 1, 2
FAKE = 1 << 20  # a non-null, 16-byte aligned address that is never dereferenced


@pytest.fixture(scope="module")
def lib():
    from gated_delta_rule_bounded_b200 import build
    build.build()
    return kda.load_library()


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:int|const char\*)\s+(kda_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for fn in ("kda_bounded_decay", "kda_prefill", "kda_prefill_workspace_bytes", "kda_decode_step",
               "kda_last_error", "kda_version"):
        assert fn in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", kda.library_path()], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT\s+(\w+)$", out, flags=re.M))
    for fn in declared_functions():
        assert fn in exported, f"{fn} declared in kda.h but not exported"
        assert hasattr(lib, fn)


def test_header_compiles_as_c(tmp_path):
    c = tmp_path / "t.c"
    c.write_text('#include "kda.h"\nint main(void){return (int)sizeof(kda_layout) == 144 ? 0 : 1;}\n')
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.dirname(HEADER), str(c),
                    "-o", str(tmp_path / "t")], check=True)
    assert subprocess.run([str(tmp_path / "t")]).returncode == 0


def _prefill(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, dtype=1, gate=FAKE, gk=0, beta=FAKE, s0=None, sf=None, cu=None,
             n_seq=0, B=1, T=64, H=2, K=128, V=128, layout=None, o=FAKE, ws=None, wsb=0, stream=None)
    a.update(kw)
    rc = lib.kda_prefill(a["q"], a["k"], a["v"], a["dtype"], a["gate"], a["gk"], a["beta"], a["s0"], a["sf"],
                         a["cu"], a["n_seq"], a["B"], a["T"], a["H"], a["K"], a["V"], a["layout"], a["o"],
                         a["ws"], a["wsb"], a["stream"])
    return rc, lib.kda_last_error().decode()


def _decode(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, dtype=1, gate=FAKE, gk=0, beta=FAKE, state=FAKE, B=2, H=2, K=128, V=128,
             layout=None, o=FAKE, stream=None)
    a.update(kw)
    rc = lib.kda_decode_step(a["q"], a["k"], a["v"], a["dtype"], a["gate"], a["gk"], a["beta"], a["state"],
                             a["B"], a["H"], a["K"], a["V"], a["layout"], a["o"], a["stream"])
    return rc, lib.kda_last_error().decode()


def _gate(lib, **kw):
    a = dict(z=FAKE, zs=None, dtype=0, A=FAKE, g_min=-5.0, B=1, T=4, H=2, K=32, out=FAKE, os=None, kind=0,
             stream=None)
    a.update(kw)
    rc = lib.kda_bounded_decay(a["z"], a["zs"], a["dtype"], a["A"], a["g_min"], a["B"], a["T"], a["H"], a["K"],
                               a["out"], a["os"], a["kind"], a["stream"])
    return rc, lib.kda_last_error().decode()


@pytest.mark.parametrize("kw,code,msg", [
    (dict(B=-1), INVALID, "negative"),
    (dict(dtype=7), INVALID, "dtype"),
    (dict(gk=5), INVALID, "gate kind"),
    (dict(K=24), UNSUPPORTED, "multiples of 16"),
    (dict(V=272), UNSUPPORTED, "multiples of 16"),
    (dict(K=0), UNSUPPORTED, "multiples of 16"),
    (dict(H=0), INVALID, "H must be positive"),
    (dict(q=None), INVALID, "null"),
    (dict(o=None), INVALID, "null"),
    (dict(cu=FAKE, n_seq=3, B=2), INVALID, "B == 1"),
    (dict(q=FAKE + 8), UNSUPPORTED, "16-byte"),
    (dict(s0=FAKE, sf=FAKE + 64), INVALID, "overlap"),
    (dict(s0=FAKE + 4), UNSUPPORTED, "16-byte"),
])
def test_prefill_rejects_bad_arguments(lib, kw, code, msg):
    rc, err = _prefill(lib, **kw)
    assert rc == code and msg in err


def test_prefill_rejects_misaligned_strides(lib):
    lay = Layout(*[Strides(64 * 2 * 128, 2 * 128, 128) for _ in range(6)])
    lay.q = Strides(64 * 2 * 132, 2 * 132, 132)   # bf16 rows of 132 elements: 264 bytes, not a 16-byte multiple
    rc, err = _prefill(lib, layout=ctypes.byref(lay))
    assert rc == UNSUPPORTED and "16-byte" in err
    lay.q = Strides(-1, 256, 128)
    rc, err = _prefill(lib, layout=ctypes.byref(lay))
    assert rc == INVALID and "negative stride" in err


@pytest.mark.parametrize("kw,code,msg", [
    (dict(B=-2), INVALID, "negative"),
    (dict(K=8), UNSUPPORTED, "multiples of 16"),
    (dict(state=None), INVALID, "null"),
    (dict(gk=3), INVALID, "gate kind"),
    (dict(state=FAKE + 4), UNSUPPORTED, "16-byte"),
])
def test_decode_rejects_bad_arguments(lib, kw, code, msg):
    rc, err = _decode(lib, **kw)
    assert rc == code and msg in err


@pytest.mark.parametrize("kw,code,msg", [
    (dict(g_min=0.0), INVALID, "g_min"),
    (dict(g_min=1.0), INVALID, "g_min"),
    (dict(g_min=float("nan")), INVALID, "g_min"),
    (dict(g_min=float("-inf")), INVALID, "g_min"),
    (dict(kind=9), INVALID, "out_kind"),
    (dict(dtype=4), INVALID, "dtype"),
    (dict(z=None), INVALID, "null"),
    (dict(K=6), UNSUPPORTED, "multiple of 4"),
    (dict(T=-1), INVALID, "negative"),
])
def test_gate_rejects_bad_arguments(lib, kw, code, msg):
    rc, err = _gate(lib, **kw)
    assert rc == code and msg in err


def test_empty_calls_succeed_without_launch(lib):
    assert _gate(lib, T=0, z=None, out=None)[0] == OK
    assert _decode(lib, B=0, q=None)[0] == OK
    # T = 0 with no final state requested has nothing to do.
    assert _prefill(lib, T=0, q=None, k=None, v=None)[0] == OK


def test_workspace_query(lib):
    n = ctypes.c_size_t(123)
    assert lib.kda_prefill_workspace_bytes(1, 4096, 96, 128, 128, 0, 1, ctypes.byref(n)) == OK
    assert n.value >= 0
    assert lib.kda_prefill_workspace_bytes(1, -1, 96, 128, 128, 0, 1, ctypes.byref(n)) == INVALID
    assert lib.kda_prefill_workspace_bytes(1, 1, 1, 128, 128, 0, 1, None) == INVALID


def _backward(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, dtype=1, gate=FAKE, gk=1, beta=FAKE, s0=None, do=FAKE, dsf=None, cu=None,
             n_seq=0, B=1, T=64, H=2, K=128, V=128, layout=None, dq=FAKE, dk=FAKE, dv=FAKE, dg=FAKE, db=FAKE,
             ds0=None, ws=FAKE, wsb=0, stream=None)
    a.update(kw)
    rc = lib.kda_scan_backward(a["q"], a["k"], a["v"], a["dtype"], a["gate"], a["gk"], a["beta"], a["s0"], a["do"],
                               a["dsf"], a["cu"], a["n_seq"], a["B"], a["T"], a["H"], a["K"], a["V"], a["layout"],
                               a["dq"], a["dk"], a["dv"], a["dg"], a["db"], a["ds0"], a["ws"], a["wsb"], a["stream"])
    return rc, lib.kda_last_error().decode()


@pytest.mark.parametrize("kw,code,msg", [
    (dict(B=-1), INVALID, "negative"),
    (dict(n_seq=-1), INVALID, "negative"),
    (dict(cu=FAKE, n_seq=3, B=2), INVALID, "B == 1"),
    (dict(gk=3), INVALID, "gate kind"),
    (dict(K=48), UNSUPPORTED, "K and V"),
    (dict(dq=None), INVALID, "null"),
    (dict(wsb=1024), INVALID, "workspace"),
    (dict(cu=FAKE, n_seq=4, wsb=1024), INVALID, "workspace"),
])
def test_scan_backward_rejects_bad_arguments(lib, kw, code, msg):
    rc, err = _backward(lib, **kw)
    assert rc == code and msg in err, (rc, err)


def test_scan_backward_workspace_query(lib):
    def ws(B, T, H, K, V, n_seq):
        n = ctypes.c_size_t(0)
        assert lib.kda_scan_backward_workspace_bytes(B, T, H, K, V, n_seq, ctypes.byref(n)) == OK
        return n.value
    slice_ = 128 * 128 * 4
    # one sequence per batch row: (ceil(T/32) + 1) checkpoints and 32 scratch states per (row, head)
    assert ws(2, 100, 3, 128, 128, 0) == 2 * 3 * (4 + 1 + 32) * slice_
    # packed sequences: floor(T/32) + 2N + 1 checkpoint slots per head, 32 scratch states per (sequence, head)
    assert ws(1, 100, 3, 128, 128, 5) == 3 * (3 + 10 + 1) * slice_ + 5 * 3 * 32 * slice_
    n = ctypes.c_size_t(0)
    assert lib.kda_scan_backward_workspace_bytes(1, 10, 1, 128, 128, -1, ctypes.byref(n)) == INVALID


def test_last_error_cleared_on_success(lib):
    _gate(lib, g_min=0.0)
    assert lib.kda_last_error().decode() != ""
    assert _gate(lib, T=0)[0] == OK
    assert lib.kda_last_error().decode() == ""


def test_python_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(1, 2, 1, 16)
    with pytest.raises(ValueError, match="CUDA"):
        kda.bounded_decay(x, torch.zeros(1))
    with pytest.raises(ValueError, match="CUDA"):
        kda.prefill(x, x, x, x, torch.zeros(1, 2, 1))


def test_noalloc_scratch_limit_matches_binding():
    m = re.search(r"#define\s+KDA_NOALLOC_SCRATCH_BYTES\s+\(\(size_t\)(\d+)\s*<<\s*(\d+)\)", open(HEADER).read())
    assert m, "KDA_NOALLOC_SCRATCH_BYTES not found in kda.h"
    assert int(m.group(1)) << int(m.group(2)) == kda.NOALLOC_SCRATCH_BYTES


def test_noalloc_rejects_oversize_before_any_device_call(lib):
    # 4096 tokens x 96 heads need 64 x 96 x 66,048 bytes of workspace, beyond the static scratch;
    # the call must refuse on the host (the fake pointers are never dereferenced).
    layout = Layout(*[Strides(4096 * 96 * 128, 96 * 128, 128)] * 3, Strides(4096 * 96 * 128, 96 * 128, 128),
                    Strides(4096 * 96, 96, 1), Strides(4096 * 96 * 128, 96 * 128, 128))
    rc = lib.kda_prefill_noalloc(FAKE, FAKE, FAKE, 1, FAKE, 0, FAKE, None, None, None, 0,
                                 1, 4096, 96, 128, 128, ctypes.byref(layout), FAKE, None)
    assert rc == UNSUPPORTED
    msg = lib.kda_last_error().decode()
    assert "static scratch" in msg and str(64 * 96 * 66048) in msg
    # Bad sizes are reported by the workspace query it shares with kda_prefill.
    rc = lib.kda_prefill_noalloc(FAKE, FAKE, FAKE, 1, FAKE, 0, FAKE, None, None, None, 0,
                                 1, -1, 96, 128, 128, None, FAKE, None)
    assert rc == INVALID


def test_logits_entry_points_reject_bad_gate_arguments(lib):
    layout = Layout(*[Strides(0, 128, 128)] * 4, Strides(0, 1, 1), Strides(0, 128, 128))
    for g_min in (0.0, 1.0, float("nan"), float("inf")):
        rc = lib.kda_prefill_logits(FAKE, FAKE, FAKE, 1, FAKE, FAKE, None, g_min, FAKE, 0, None, None, None, 0,
                                    1, 4, 1, 128, 128, ctypes.byref(layout), FAKE, None, 0, None)
        assert rc == INVALID and "g_min" in lib.kda_last_error().decode()
        rc = lib.kda_decode_step_logits(FAKE, FAKE, FAKE, 1, FAKE, FAKE, None, g_min, FAKE, 0, FAKE, 1, 1, 128, 128,
                                        ctypes.byref(layout), FAKE, None)
        assert rc == INVALID and "g_min" in lib.kda_last_error().decode()
    rc = lib.kda_prefill_logits(FAKE, FAKE, FAKE, 1, FAKE, None, None, -5.0, FAKE, 0, None, None, None, 0,
                                1, 4, 1, 128, 128, ctypes.byref(layout), FAKE, None, 0, None)
    assert rc == INVALID and "null" in lib.kda_last_error().decode()
    rc = lib.kda_decode_step_logits(FAKE, FAKE, FAKE, 1, FAKE, None, None, -5.0, FAKE, 0, FAKE, 1, 1, 128, 128,
                                    ctypes.byref(layout), FAKE, None)
    assert rc == INVALID and "null" in lib.kda_last_error().decode()


def test_logits_entry_points_reject_unknown_flags(lib):
    layout = Layout(*[Strides(0, 128, 128)] * 4, Strides(0, 1, 1), Strides(0, 128, 128))
    rc = lib.kda_prefill_logits(FAKE, FAKE, FAKE, 1, FAKE, FAKE, None, -5.0, FAKE, 16, None, None, None, 0,
                                1, 4, 1, 128, 128, ctypes.byref(layout), FAKE, None, 0, None)
    assert rc == INVALID and "flags" in lib.kda_last_error().decode()
    rc = lib.kda_decode_step_logits(FAKE, FAKE, FAKE, 1, FAKE, FAKE, None, -5.0, FAKE, 32, FAKE, 1, 1, 128, 128,
                                    ctypes.byref(layout), FAKE, None)
    assert rc == INVALID and "flags" in lib.kda_last_error().decode()


def test_logits_entry_points_reject_a_misaligned_bias(lib):
    layout = Layout(*[Strides(0, 128, 128)] * 4, Strides(0, 1, 1), Strides(0, 128, 128))
    rc = lib.kda_prefill_logits(FAKE, FAKE, FAKE, 1, FAKE, FAKE, FAKE + 4, -5.0, FAKE, 0, None, None, None, 0,
                                1, 4, 1, 128, 128, ctypes.byref(layout), FAKE, None, 0, None)
    assert rc == UNSUPPORTED and "dt_bias" in lib.kda_last_error().decode()
    rc = lib.kda_decode_step_logits(FAKE, FAKE, FAKE, 1, FAKE, FAKE, FAKE + 8, -5.0, FAKE, 0, FAKE, 1, 1, 128, 128,
                                    ctypes.byref(layout), FAKE, None)
    assert rc == UNSUPPORTED and "dt_bias" in lib.kda_last_error().decode()


def test_prefill_rejects_more_heads_than_a_grid_dimension_holds(lib):
    # the operand kernel runs one grid row per head; more than 65535 heads are refused up front
    H = 65536
    layout = Layout(*[Strides(0, H * 128, 128)] * 4, Strides(0, H, 1), Strides(0, H * 128, 128))
    rc = lib.kda_prefill(FAKE, FAKE, FAKE, 1, FAKE, 0, FAKE, None, None, None, 0,
                         1, 4, H, 128, 128, ctypes.byref(layout), FAKE, None, 0, None)
    assert rc == UNSUPPORTED and "65535" in lib.kda_last_error().decode()


def _backward_chunked(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, dtype=1, gate=FAKE, gk=1, beta=FAKE, s0=None, do=FAKE, dsf=None, cu=None,
             n_seq=0, B=1, T=64, H=2, K=128, V=128, layout=None, dq=FAKE, dk=FAKE, dv=FAKE, dg=FAKE, db=FAKE,
             ds0=None, ws=FAKE, wsb=0, stream=None)
    a.update(kw)
    f = lib.kda_scan_backward_chunked
    f.restype = ctypes.c_int
    vp, i64 = ctypes.c_void_p, ctypes.c_int64
    f.argtypes = [vp, vp, vp, ctypes.c_int, vp, ctypes.c_int, vp, vp, vp, vp, vp, i64, i64, i64, i64, i64, i64, vp,
                  vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
    rc = f(a["q"], a["k"], a["v"], a["dtype"], a["gate"], a["gk"], a["beta"], a["s0"], a["do"], a["dsf"], a["cu"],
           a["n_seq"], a["B"], a["T"], a["H"], a["K"], a["V"], a["layout"], a["dq"], a["dk"], a["dv"], a["dg"], a["db"],
           a["ds0"], a["ws"], a["wsb"], a["stream"])
    return rc, lib.kda_last_error().decode()


@pytest.mark.parametrize("kw,code,msg", [
    (dict(B=-1), INVALID, "negative"),
    (dict(gk=3), INVALID, "gate kind"),
    (dict(K=64), UNSUPPORTED, "K = V = 128"),
    (dict(dtype=0), UNSUPPORTED, "bf16"),
    (dict(dq=None), INVALID, "null"),
    (dict(wsb=1024), INVALID, "workspace"),
    (dict(cu=FAKE, n_seq=2, B=2), INVALID, "B == 1"),
    (dict(n_seq=-1), INVALID, "negative"),
    (dict(cu=FAKE, n_seq=3, wsb=1 << 20), INVALID, "workspace"),
])
def test_scan_backward_chunked_rejects_bad_arguments(lib, kw, code, msg):
    # every check runs on the host before any launch
    rc, err = _backward_chunked(lib, **kw)
    assert rc == code and msg in err, (rc, err)


def test_scan_backward_chunked_workspace_query(lib):
    f = lib.kda_scan_backward_chunked_workspace_bytes
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_int64] * 6 + [ctypes.POINTER(ctypes.c_size_t)]
    n = ctypes.c_size_t(0)
    assert f(1, 4096, 96, 128, 128, 0, ctypes.byref(n)) == OK
    dense = n.value
    per_chunk_head = dense / (64 * 96)
    assert 800e3 < per_chunk_head < 1000e3  # the chunk buffers (~880 KB per chunk and head) plus fixed parts
    # packed sequences: the forward's slots, T / 64 + n_seq + 1 chunks per head
    assert f(1, 4096, 96, 128, 128, 16, ctypes.byref(n)) == OK
    assert 16 * 96 * 800e3 < n.value - dense < 18 * 96 * 1000e3
    assert f(1, 4096, 96, 64, 128, 0, ctypes.byref(n)) == UNSUPPORTED
    assert f(0, 4096, 96, 128, 128, 0, ctypes.byref(n)) == OK and n.value == 0
    assert f(1, 0, 96, 128, 128, 4, ctypes.byref(n)) == OK and n.value == 0
    assert f(1, 64, 2, 128, 128, -1, ctypes.byref(n)) == INVALID
