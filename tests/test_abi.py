"""The C ABI library (CPU-side checks: no kernel runs here).

The library loads, exports every entry point include/falcon.h declares, and
rejects bad arguments on the host before touching the device. On a machine
without a GPU a well-formed call fails loudly with FALCON_ERR_CUDA: there is no
CPU fallback anywhere in the product path.
"""
import ctypes
import os
import re

import pytest

from delta_rule_linear_falcon_b200 import build as B
from delta_rule_linear_falcon_b200 import falcon as F

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    B.build()
    return F.lib()


def declared_functions():
    txt = open(os.path.join(ROOT, "include", "falcon.h")).read()
    return re.findall(r"FALCON_API\s+[\w\s\*]+?\b(falcon_\w+)\s*\(", txt)


def test_header_declares_the_entry_points():
    names = set(declared_functions())
    assert {"falcon_fwd_chunk", "falcon_fwd_recurrent", "falcon_decode_step",
            "falcon_workspace_size", "falcon_status_string", "falcon_check_device_errors"} <= names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name
        assert ctypes.cast(getattr(L, name), ctypes.c_void_p).value


@pytest.mark.parametrize("mirror,ctype", [(F.FalconArgs, "falcon_args_t"), (F.FalconGrads, "falcon_grads_t")])
def test_struct_layout_matches_header(tmp_path, mirror, ctype):
    """The binding's struct mirrors have the C compiler's offsets for every field of the
    header's structs (a small C program compiled against include/falcon.h prints them)."""
    import subprocess
    fields = [name for name, _ in mirror._fields_]
    src = tmp_path / "layout.c"
    src.write_text("#include <stdio.h>\n#include <stddef.h>\n#include \"falcon.h\"\nint main(void) {\n"
                   + "".join(f'  printf("{f} %zu\\n", offsetof({ctype}, {f}));\n' for f in fields)
                   + f'  printf("sizeof %zu\\n", sizeof({ctype}));\n  return 0;\n}}\n')
    exe = tmp_path / "layout"
    inc = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")
    subprocess.run(["gcc", "-std=c99", "-I", inc, "-o", str(exe), str(src)], check=True)
    got = dict(line.split() for line in subprocess.run([str(exe)], capture_output=True, text=True,
                                                        check=True).stdout.splitlines())
    for f in fields:
        assert getattr(mirror, f).offset == int(got[f]), f
    assert ctypes.sizeof(mirror) == int(got["sizeof"])


def test_status_strings(L):
    for code in range(6):
        s = F.falcon_status_string(code)
        assert isinstance(s, str) and s
    assert F.falcon_status_string(99) == "unknown status"
    assert F.falcon_version() >= 100


def _args(**kw):
    base = dict(rule=1, io_dtype=1, B=2, H=3, T=10, dk=128, dv=128, q=0x1000, k=0x2000, v=0x3000,
                alpha=0x4000, eta=0x5000, eps=1e-6, window=1, chunk=64, S0=None, k_prev=None,
                o=0x6000, S_out=None, k_last=None)
    base.update(kw)
    return F.FalconArgs(**base)


@pytest.mark.parametrize("kw,expect", [
    (dict(rule=0), F.FALCON_ERR_INVALID_ARG),
    (dict(rule=7), F.FALCON_ERR_INVALID_ARG),
    (dict(io_dtype=5), F.FALCON_ERR_INVALID_ARG),
    (dict(B=-1), F.FALCON_ERR_INVALID_ARG),
    (dict(dk=0), F.FALCON_ERR_INVALID_ARG),
    (dict(eps=-1.0), F.FALCON_ERR_INVALID_ARG),
    (dict(eps=float("nan")), F.FALCON_ERR_INVALID_ARG),
    (dict(q=None), F.FALCON_ERR_INVALID_ARG),
    (dict(o=None), F.FALCON_ERR_INVALID_ARG),
    (dict(k=0x2004), F.FALCON_ERR_INVALID_ARG),            # misaligned
    (dict(alpha=0x4002), F.FALCON_ERR_INVALID_ARG),
    (dict(S0=0x7008), F.FALCON_ERR_INVALID_ARG),
    (dict(rule=3, window=0), F.FALCON_ERR_INVALID_ARG),
    (dict(dk=96), F.FALCON_ERR_UNSUPPORTED),
    (dict(dv=48), F.FALCON_ERR_UNSUPPORTED),
    (dict(io_dtype=0), F.FALCON_ERR_UNSUPPORTED),   # fp32 inputs: the recurrent form serves them
    (dict(rule=5), F.FALCON_ERR_UNSUPPORTED),       # Falcon-2/2A run on the recurrent form
    (dict(rule=6 | 0x100), F.FALCON_ERR_UNSUPPORTED),
    (dict(chunk=128), F.FALCON_ERR_UNSUPPORTED),
    (dict(chunk=8), F.FALCON_ERR_UNSUPPORTED),
    (dict(rule=3, window=65), F.FALCON_ERR_UNSUPPORTED),
])
def test_chunk_rejects_bad_arguments_on_host(L, kw, expect):
    a = _args(**kw)
    assert L.falcon_fwd_chunk(ctypes.byref(a), None, 0, None) == expect


def test_null_args_struct(L):
    assert L.falcon_fwd_chunk(None, None, 0, None) == F.FALCON_ERR_INVALID_ARG
    assert L.falcon_fwd_recurrent(None, None) == F.FALCON_ERR_INVALID_ARG
    assert L.falcon_workspace_size(None) == 0


@pytest.mark.parametrize("kw,expect", [
    (dict(dk=129), F.FALCON_ERR_UNSUPPORTED),
    (dict(dv=200), F.FALCON_ERR_UNSUPPORTED),
    (dict(rule=3, window=65), F.FALCON_ERR_UNSUPPORTED),
    (dict(v=None), F.FALCON_ERR_INVALID_ARG),
])
def test_recurrent_rejects_bad_arguments_on_host(L, kw, expect):
    assert L.falcon_fwd_recurrent(ctypes.byref(_args(**kw)), None) == expect


def _dec(L, **kw):
    a = dict(rule=1, io_dtype=1, N=4, H=2, dk=128, dv=128, S=0x1000, k_prev=0x2000, q=0x3000,
             k=0x4000, v=0x5000, alpha=0x6000, eta=0x7000, eps=1e-6, o=0x8000, stream=None)
    a.update(kw)
    return L.falcon_decode_step(a["rule"], a["io_dtype"], a["N"], a["H"], a["dk"], a["dv"], a["S"],
                                a["k_prev"], a["q"], a["k"], a["v"], a["alpha"], a["eta"],
                                a["eps"], a["o"], a["stream"])


@pytest.mark.parametrize("kw,expect", [
    (dict(rule=3), F.FALCON_ERR_UNSUPPORTED),
    (dict(rule=4), F.FALCON_ERR_UNSUPPORTED),
    (dict(rule=9), F.FALCON_ERR_INVALID_ARG),
    (dict(dk=96), F.FALCON_ERR_UNSUPPORTED),
    (dict(dv=300), F.FALCON_ERR_UNSUPPORTED),
    (dict(S=None), F.FALCON_ERR_INVALID_ARG),
    (dict(S=0x1004), F.FALCON_ERR_INVALID_ARG),
    (dict(N=-2), F.FALCON_ERR_INVALID_ARG),
    (dict(N=0), F.FALCON_OK),
])
def test_decode_rejects_bad_arguments_on_host(L, kw, expect):
    assert _dec(L, **kw) == expect


def _grads(**kw):
    base = dict(dO=0x10000, dS_T=None, dq=0x11000, dk=0x12000, dv=0x13000, dalpha=0x14000,
                deta=0x15000, dS0=None, dk_prev=None)
    base.update(kw)
    return F.FalconGrads(**base)


@pytest.mark.parametrize("akw,gkw,ws,expect", [
    (dict(rule=5), {}, 1 << 30, F.FALCON_ERR_UNSUPPORTED),       # Falcon-2/2A: forward only
    (dict(rule=6 | 0x100), {}, 1 << 30, F.FALCON_ERR_UNSUPPORTED),
    (dict(dk=129), {}, 1 << 30, F.FALCON_ERR_UNSUPPORTED),
    (dict(dv=256), {}, 1 << 30, F.FALCON_ERR_UNSUPPORTED),
    (dict(rule=3, window=16), {}, 1 << 30, F.FALCON_ERR_UNSUPPORTED),   # more pairs than the step inputs hold
    (dict(rule=3, window=9, dk=16, dv=16), {}, 1 << 30, F.FALCON_ERR_UNSUPPORTED),   # above 8 pairs
    (dict(rule=3, window=0), {}, 1 << 30, F.FALCON_ERR_INVALID_ARG),
    (dict(q=None), {}, 1 << 30, F.FALCON_ERR_INVALID_ARG),
    (dict(eps=-1.0), {}, 1 << 30, F.FALCON_ERR_INVALID_ARG),
    ({}, dict(dO=None), 1 << 30, F.FALCON_ERR_INVALID_ARG),
    ({}, dict(deta=None), 1 << 30, F.FALCON_ERR_INVALID_ARG),
    ({}, dict(dq=0x11002), 1 << 30, F.FALCON_ERR_INVALID_ARG),        # misaligned
    ({}, {}, 0, F.FALCON_ERR_WORKSPACE),
    ({}, {}, 1024, F.FALCON_ERR_WORKSPACE),
    (dict(B=0), {}, 0, F.FALCON_OK),
    (dict(T=0), {}, 0, F.FALCON_OK),
])
def test_backward_rejects_bad_arguments_on_host(L, akw, gkw, ws, expect):
    a = _args(**{"o": None, **akw})
    g = _grads(**gkw)
    ws_ptr = 0x100000 if ws else None
    assert L.falcon_bwd_recurrent(ctypes.byref(a), ctypes.byref(g), ws_ptr, ws, None) == expect
    assert L.falcon_bwd_recurrent(None, ctypes.byref(g), ws_ptr, ws, None) == F.FALCON_ERR_INVALID_ARG
    assert L.falcon_bwd_recurrent(ctypes.byref(_args(o=None)), None, ws_ptr, ws, None) in (
        F.FALCON_ERR_INVALID_ARG, F.FALCON_OK)


def test_backward_workspace_size(L):
    """Checkpoints every C = ceil(sqrt(T)) steps plus one segment of C + 1 recomputed states, fp32,
    per slice of 8 value rows (the last slice of a head padded to 8 rows)."""
    import math
    for T, dk, dv in ((256, 32, 32), (100, 128, 64), (1, 16, 8), (4096, 128, 128), (50, 24, 48)):
        a = _args(T=T, dk=dk, dv=dv, o=None)
        C = math.ceil(math.sqrt(T))
        nseg = -(-T // C)
        rows = 8 * -(-dv // 8)
        assert L.falcon_bwd_workspace_size(ctypes.byref(a)) == 2 * 3 * (nseg + C + 1) * rows * dk * 4
    assert L.falcon_bwd_workspace_size(ctypes.byref(_args(T=0))) == 0
    assert L.falcon_bwd_workspace_size(ctypes.byref(_args(rule=5))) == 0
    assert L.falcon_bwd_workspace_size(None) == 0


def test_empty_problems_launch_nothing(L):
    assert L.falcon_fwd_chunk(ctypes.byref(_args(B=0)), None, 0, None) == F.FALCON_OK
    assert L.falcon_fwd_recurrent(ctypes.byref(_args(H=0)), None) == F.FALCON_OK


def test_no_cpu_fallback_without_gpu(L):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    # well-formed call: the host checks pass, then the device query fails loudly
    assert L.falcon_fwd_chunk(ctypes.byref(_args()), None, 0, None) == F.FALCON_ERR_CUDA
    assert L.falcon_fwd_recurrent(ctypes.byref(_args(dk=32, dv=32)), None) == F.FALCON_ERR_CUDA
    assert _dec(L) == F.FALCON_ERR_CUDA
    assert L.falcon_bwd_recurrent(ctypes.byref(_args(o=None)), ctypes.byref(_grads()), 0x100000, 1 << 30,
                                  None) == F.FALCON_ERR_CUDA


def test_binding_raises_when_library_missing(monkeypatch, tmp_path):
    monkeypatch.setattr(F, "_lib", None)
    monkeypatch.setattr(F, "LIB_PATH", str(tmp_path / "libfalcon.so"))
    with pytest.raises(RuntimeError, match="missing"):
        F.lib()


def test_product_package_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "delta_rule_linear_falcon_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, fn)).read()
                assert "import oracle" not in txt and "from oracle" not in txt, fn
                assert "falcon_oracle" not in txt, fn


@pytest.mark.parametrize("block,budget,expect", [
    (-1, 10 ** 6, F.FALCON_ERR_INVALID_ARG),
    (0, 100, F.FALCON_ERR_INVALID_ARG),
    (0, 1 << 40, F.FALCON_ERR_INVALID_ARG),
    (3, 10 ** 6, F.FALCON_OK),
])
def test_debug_stall_hook_checks_its_arguments(L, block, budget, expect):
    """The failure-path test hook validates on the host; arming it launches nothing, and an
    armed stall is consumed by the next chunk call of the thread (here one with no GPU, which
    returns FALCON_ERR_CUDA after the host checks)."""
    assert F.falcon_debug_stall_next_call(block, budget) == expect
    if expect == F.FALCON_OK:
        a = _args()
        assert L.falcon_fwd_chunk(ctypes.byref(a), None, 0, None) in (F.FALCON_ERR_CUDA, F.FALCON_OK)
