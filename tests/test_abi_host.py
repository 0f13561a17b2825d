"""Host-side checks of the C ABI (no GPU needed):
  - libhc_b200.so builds for sm_100a, loads, and exports every entry point
    declared in include/*.h with the binding's signatures;
  - argument validation refuses bad calls with the documented status before
    anything is launched.
The validation calls use fake device addresses, so they run in a child process
with CUDA_VISIBLE_DEVICES="" -- even a validation bug could not launch a kernel.
"""
from __future__ import annotations

import ctypes as C
import glob
import os
import re
import subprocess
import sys
import textwrap

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _built_lib():
    from hyper_connections_stream_b200 import build
    return build.build()


def _declared_entry_points():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        names |= set(re.findall(r"HC_API\s+[\w\s\*]+?\b(hc_\w+)\s*\(", src))
    return names


def test_library_exports_every_declared_entry_point():
    path = _built_lib()
    lib = C.CDLL(path)
    declared = _declared_entry_points()
    assert {"hc_sinkhorn", "hc_read_rmsnorm", "hc_write_mix", "hc_write_then_read",
            "hc_status_string", "hc_last_error", "hc_version", "hc_set_path", "hc_get_path",
            "hc_device_fault", "hc_selftest_bounded_wait"} <= declared
    for name in declared:
        assert hasattr(lib, name), name
    from hyper_connections_stream_b200 import _lib
    assert declared <= set(_lib.SIGNATURES), declared - set(_lib.SIGNATURES)
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\sT\s(hc_\w+)", out))
    assert exported == declared, exported ^ declared


def test_library_is_built_for_sm100a():
    """Every object is compiled for sm_100a only (the architecture-specific
    target: tcgen05, TMA) and linked by the same command."""
    from hyper_connections_stream_b200 import build
    assert build.GENCODE == ["-gencode", "arch=compute_100a,code=sm_100a"]
    assert all(build.GENCODE[i] in build.COMMON for i in range(2))
    assert os.path.exists(_built_lib())


def test_status_and_stream_types_as_documented():
    """The boundary's deviations from the planned interface, as recorded in
    the design notes: status 6 is HC_ERR_DEVICE (a kernel's bounded wait ran
    out; there is no index-checking build), and the stream argument is the
    opaque hc_stream (a cudaStream_t passed as void *, so the header needs no
    CUDA header)."""
    src = open(os.path.join(ROOT, "include", "hc_api.h")).read()
    enum = dict((k, int(v)) for k, v in re.findall(r"\b(HC_(?:OK|ERR_\w+))\s*=\s*(\d+)", src))
    assert enum == {"HC_OK": 0, "HC_ERR_INVALID_ARG": 1, "HC_ERR_UNSUPPORTED": 2,
                    "HC_ERR_MISALIGNED": 3, "HC_ERR_ALIAS": 4, "HC_ERR_CUDA": 5,
                    "HC_ERR_DEVICE": 6}
    assert re.search(r"typedef\s+void\s*\*\s*hc_stream\s*;", src)
    assert "cudaStream_t" not in re.sub(r"/\*.*?\*/", "", src, flags=re.S)


_CHILD = textwrap.dedent(r"""
    import ctypes as C, json, math
    from hyper_connections_stream_b200 import _lib as B
    L = B.lib()
    A16 = 0x10000          # fake, 16-byte aligned device addresses (never dereferenced)
    def buf(i): return A16 * (i + 1) * 4096
    res = {}
    def call(tag, fn, *args):
        res[tag] = (getattr(L, fn)(*args), L.hc_last_error().decode())
    T, n, d = 8, 4, 1024
    H, y, Ho, x, A, b, a, g = (buf(i) for i in range(8))
    bf = B.HC_BF16
    call("ok_T0", "hc_write_then_read", None, None, None, None, bf, 0, n, d, 0, None, 0, 0,
         None, 0, 0, None, 0, None, 1e-6, None)
    call("T_neg", "hc_write_mix", H, y, Ho, bf, -1, n, d, 0, A, 0, 0, b, 0, None)
    call("n0", "hc_write_mix", H, y, Ho, bf, T, 0, d, 0, A, 0, 0, b, 0, None)
    call("n9", "hc_write_mix", H, y, Ho, bf, T, 9, d, 0, A, 0, 0, b, 0, None)
    call("d_ragged", "hc_write_mix", H, y, Ho, bf, T, n, 12, 0, A, 0, 0, b, 0, None)
    call("d_f32_ok_but_null", "hc_write_mix", None, y, Ho, B.HC_F32, T, n, 12, 0, A, 0, 0, b, 0, None)
    call("d_too_big", "hc_read_rmsnorm", H, x, bf, T, n, 32768 + 8, 0, a, 0, None, 1e-6, None)
    call("dtype", "hc_write_mix", H, y, Ho, 7, T, n, d, 0, A, 0, 0, b, 0, None)
    call("mixmode", "hc_write_mix", H, y, Ho, bf, T, n, d, 5, A, 0, 0, b, 0, None)
    call("readmode", "hc_read_rmsnorm", H, x, bf, T, n, d, 3, a, 0, None, 1e-6, None)
    call("K0", "hc_write_mix", H, y, Ho, bf, T, n, d, 1, A, 0, 0, b, 0, None)
    call("K_huge", "hc_write_mix", H, y, Ho, bf, T, n, d, 1, A, 0, 1 << 20, b, 0, None)
    call("stride_neg", "hc_write_mix", H, y, Ho, bf, T, n, d, 0, A, -16, 0, b, 0, None)
    call("eps_neg", "hc_read_rmsnorm", H, x, bf, T, n, d, 0, a, 0, None, -1.0, None)
    call("eps_nan", "hc_read_rmsnorm", H, x, bf, T, n, d, 0, a, 0, None, float("nan"), None)
    call("eps_inf", "hc_read_rmsnorm", H, x, bf, T, n, d, 0, a, 0, None, float("inf"), None)
    call("null_H", "hc_write_mix", None, y, Ho, bf, T, n, d, 0, A, 0, 0, b, 0, None)
    call("null_A", "hc_write_mix", H, y, Ho, bf, T, n, d, 0, None, 0, 0, b, 0, None)
    call("null_b", "hc_write_then_read", H, y, Ho, x, bf, T, n, d, 0, A, 0, 0, None, 0, 0, a, 0, None, 1e-6, None)
    call("mis_H", "hc_write_mix", H + 8, y, Ho, bf, T, n, d, 0, A, 0, 0, b, 0, None)
    call("mis_x", "hc_read_rmsnorm", H, x + 4, bf, T, n, d, 0, a, 0, None, 1e-6, None)
    call("mis_g", "hc_read_rmsnorm", H, x, bf, T, n, d, 0, a, 0, g + 4, 1e-6, None)
    call("mis_A", "hc_write_mix", H, y, Ho, bf, T, n, d, 0, A + 2, 0, 0, b, 0, None)
    hb = T * n * d * 2
    call("alias_partial", "hc_write_mix", H, y, H + 16, bf, T, n, d, 0, A, 0, 0, b, 0, None)
    call("alias_y", "hc_write_mix", H, y, y - hb + 16, bf, T, n, d, 0, A, 0, 0, b, 0, None)
    call("alias_x_H", "hc_write_then_read", H, y, Ho, H + hb - 16, bf, T, n, d, 0, A, 0, 0, b, 0, 0, a, 0, None, 1e-6, None)
    call("alias_x_read", "hc_read_rmsnorm", H, H + 32, bf, T, n, d, 0, a, 0, None, 1e-6, None)
    call("sk_n0", "hc_sinkhorn", A, A, T, 0, 20, None)
    call("sk_K0", "hc_sinkhorn", A, A, T, 4, 0, None)
    call("sk_null", "hc_sinkhorn", None, A, T, 4, 20, None)
    call("sk_alias", "hc_sinkhorn", A, A + 4, T, 4, 20, None)
    call("sk_T0", "hc_sinkhorn", None, None, 0, 4, 20, None)
    call("st_lo", "hc_selftest_bounded_wait", 0, None)
    call("st_hi", "hc_selftest_bounded_wait", 1000000, None)
    call("path_bad", "hc_set_path", 7)
    pout = C.c_int(0)
    call("sp_null", "hc_step_path", bf, 2, T, n, d, None)
    call("sp_op", "hc_step_path", bf, 3, T, n, d, C.byref(pout))
    call("sp_T0", "hc_step_path", bf, 2, 0, n, d, C.byref(pout))
    call("sp_n9", "hc_step_path", bf, 2, T, 9, d, C.byref(pout))
    call("sp_d_ragged", "hc_step_path", bf, 0, T, n, 12, C.byref(pout))
    call("sp_dtype", "hc_step_path", 7, 1, T, n, d, C.byref(pout))
    xb = T * d * 2
    call("ex_T0", "hc_expand", None, None, bf, 0, n, d, None)
    call("ex_n9", "hc_expand", x, H, bf, T, 9, d, None)
    call("ex_null", "hc_expand", None, H, bf, T, n, d, None)
    call("ex_mis", "hc_expand", x + 8, H, bf, T, n, d, None)
    call("ex_alias", "hc_expand", H + hb - 16, H, bf, T, n, d, None)
    call("er_readmode", "hc_expand_then_read", x, H, y, bf, T, n, d, 4, a, 0, None, 1e-6, None)
    call("er_null_a", "hc_expand_then_read", x, H, y, bf, T, n, d, 0, None, 0, None, 1e-6, None)
    call("er_eps", "hc_expand_then_read", x, H, y, bf, T, n, d, 0, a, 0, None, -2.0, None)
    call("er_alias_xr_H", "hc_expand_then_read", x, H, H + 64, bf, T, n, d, 0, a, 0, None, 1e-6, None)
    call("er_alias_xr_x", "hc_expand_then_read", x, H, x + 32, bf, T, n, d, 0, a, 0, None, 1e-6, None)
    call("er_d_too_big", "hc_expand_then_read", x, H, y, bf, T, n, 32768 + 8, 0, a, 0, None, 1e-6, None)
    call("co_null_w", "hc_collapse", H, x, bf, T, n, d, 0, None, 0, None)
    call("co_stride", "hc_collapse", H, x, bf, T, n, d, 0, a, -4, None)
    call("co_alias", "hc_collapse", H, H + hb - xb + 16, bf, T, n, d, 0, a, 0, None)
    call("co_mis_w", "hc_collapse", H, x, bf, T, n, d, 0, a + 1, 0, None)
    Xl, Wl = buf(20), buf(40)
    call("lw_f32", "hc_linear_then_write", Xl, Wl, H, Ho, None, B.HC_F32, T, n, d, 64, A, 0, b, 0, None)
    call("lw_k_ragged", "hc_linear_then_write", Xl, Wl, H, Ho, None, bf, T, n, d, 60, A, 0, b, 0, None)
    call("lw_k0", "hc_linear_then_write", Xl, Wl, H, Ho, None, bf, T, n, d, 0, A, 0, b, 0, None)
    call("lw_T0", "hc_linear_then_write", None, None, None, None, None, bf, 0, n, d, 64, None, 0, None, 0, None)
    call("lw_mis_X", "hc_linear_then_write", Xl + 8, Wl, H, Ho, None, bf, T, n, d, 64, A, 0, b, 0, None)
    call("lw_null_A", "hc_linear_then_write", Xl, Wl, H, Ho, None, bf, T, n, d, 64, None, 0, b, 0, None)
    call("lw_alias_y", "hc_linear_then_write", Xl, Wl, H, Ho, Ho + 64, bf, T, n, d, 64, A, 0, b, 0, None)
    call("lw_alias_X", "hc_linear_then_write", Xl, Wl, H, Xl + 32, None, bf, T, n, d, 64, A, 0, b, 0, None)
    P0, P1, P2 = buf(60), buf(61), buf(62)
    def parts(*ps):
        arr = (C.c_void_p * len(ps))(*ps)
        parts.keep.append(arr)  # the host array must outlive the call
        return C.cast(arr, C.c_void_p)
    parts.keep = []
    ok3 = parts(P0, P1, P2)
    def rw(tag, pp, R, Hh=H, Hout=Ho, xx=x, yo=None, d_=d, T_=T, dt=bf):
        call(tag, "hc_reduce_write_then_read", pp, R, Hh, Hout, xx, yo, dt, T_, n, d_, 0, A, 0, 0,
             b, 0, 0, a, 0, None, 1e-6, None)
    rw("rw_T0", ok3, 3, Hh=None, Hout=None, xx=None, T_=0)
    rw("rw_R0", ok3, 0)
    rw("rw_R9", parts(*([P0] * 9)), 9)
    rw("rw_parts_null", None, 3)
    rw("rw_part_null", parts(P0, None, P2), 3)
    rw("rw_part_mis", parts(P0, P1 + 8, P2), 3)
    rw("rw_alias_x_part", ok3, 3, xx=P1 + 32)
    rw("rw_alias_Hout_part", ok3, 3, Hout=P2 - hb + 64)
    rw("rw_alias_yout_H", ok3, 3, yo=H + 64)
    rw("rw_mis_yout", ok3, 3, yo=buf(70) + 8)
    rw("rw_d_too_big", ok3, 3, d_=32768 + 8)
    X0, X1 = buf(80), buf(81)
    okx = parts(X0, X1)
    ok2 = parts(P0, P1)
    def rs(tag, pp, xx, R, rank, T_=T, Hh=H, Hout=Ho):
        call(tag, "hc_reduce_scatter_write_then_read", pp, R, rank, T_, Hh, Hout, xx, None, bf, n,
             d, 0, A, 0, 0, b, 0, 0, a, 0, None, 1e-6, None)
    rs("rs_T0", ok2, okx, 2, 1, T_=0, Hh=None, Hout=None)
    rs("rs_empty_shard", ok2, okx, 2, 1, T_=1, Hh=None, Hout=None)
    rs("rs_rank_neg", ok2, okx, 2, -1)
    rs("rs_rank_big", ok2, okx, 2, 2)
    rs("rs_R9", parts(*([P0] * 9)), parts(*([X0] * 9)), 9, 0)
    rs("rs_x_null", ok2, None, 2, 0)
    rs("rs_x_entry_null", ok2, parts(X0, None), 2, 0)
    rs("rs_x_mis", ok2, parts(X0, X1 + 8), 2, 0)
    rs("rs_x_dup", ok2, parts(X0, X0), 2, 0)
    rs("rs_x_is_part", ok2, parts(X0, P1), 2, 0)
    rs("rs_x_over_H", ok2, parts(X0, H + 64), 2, 0)
    call("ipc_export_null", "hc_ipc_export", None, None, None)
    call("ipc_open_null", "hc_ipc_open", None, None)
    call("ipc_close_null", "hc_ipc_close", None)
    print(json.dumps(res))
""")


def test_argument_validation_statuses():
    _built_lib()
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", PYTHONPATH=ROOT)
    out = subprocess.run([sys.executable, "-c", _CHILD], capture_output=True, text=True, env=env,
                         cwd=ROOT, timeout=300)
    assert out.returncode == 0, out.stderr
    import json
    res = json.loads(out.stdout.strip().splitlines()[-1])
    OK, INV, UNS, MIS, ALI = 0, 1, 2, 3, 4
    want = {
        "ok_T0": OK, "T_neg": INV, "n0": INV, "n9": UNS, "d_ragged": UNS,
        "d_f32_ok_but_null": INV, "d_too_big": UNS, "dtype": INV, "mixmode": INV,
        "readmode": INV, "K0": INV, "K_huge": UNS, "stride_neg": INV, "eps_neg": INV,
        "eps_nan": INV, "eps_inf": INV, "null_H": INV, "null_A": INV, "null_b": INV,
        "mis_H": MIS, "mis_x": MIS, "mis_g": MIS, "mis_A": MIS, "alias_partial": ALI,
        "alias_y": ALI, "alias_x_H": ALI, "alias_x_read": ALI, "sk_n0": INV, "sk_K0": INV,
        "sk_null": INV, "sk_alias": ALI, "sk_T0": OK, "st_lo": INV, "st_hi": INV, "path_bad": INV,
        "sp_null": INV, "sp_op": INV, "sp_T0": INV, "sp_n9": UNS, "sp_d_ragged": UNS, "sp_dtype": INV,
        "ex_T0": OK, "ex_n9": UNS, "ex_null": INV, "ex_mis": MIS, "ex_alias": ALI,
        "er_readmode": INV, "er_null_a": INV, "er_eps": INV, "er_alias_xr_H": ALI,
        "er_alias_xr_x": ALI, "er_d_too_big": UNS, "co_null_w": INV, "co_stride": INV,
        "co_alias": ALI, "co_mis_w": MIS,
        "lw_f32": UNS, "lw_k_ragged": UNS, "lw_k0": INV, "lw_T0": OK, "lw_mis_X": MIS,
        "lw_null_A": INV, "lw_alias_y": ALI, "lw_alias_X": ALI,
        "rw_T0": OK, "rw_R0": INV, "rw_R9": UNS, "rw_parts_null": INV, "rw_part_null": INV,
        "rw_part_mis": MIS, "rw_alias_x_part": ALI, "rw_alias_Hout_part": ALI,
        "rw_alias_yout_H": ALI, "rw_mis_yout": MIS, "rw_d_too_big": UNS,
        "ipc_export_null": INV, "ipc_open_null": INV, "ipc_close_null": INV,
        "rs_T0": OK, "rs_empty_shard": OK, "rs_rank_neg": INV, "rs_rank_big": INV, "rs_R9": UNS,
        "rs_x_null": INV, "rs_x_entry_null": INV, "rs_x_mis": MIS, "rs_x_dup": ALI,
        "rs_x_is_part": ALI, "rs_x_over_H": ALI,
    }
    for tag, code in want.items():
        got, msg = res[tag]
        assert got == code, (tag, got, code, msg)
        if code != OK:
            assert msg, tag  # a reason is recorded for every refusal


def test_status_strings_and_version():
    from hyper_connections_stream_b200 import _lib
    L = _lib.lib()
    for st in range(7):
        assert L.hc_status_string(st).decode() not in ("", "unknown status")
    assert L.hc_status_string(99).decode() == "unknown status"
    assert L.hc_version() >= 100


def test_binding_refuses_cpu_tensors():
    """The binding has no CPU path: host tensors are refused, not computed."""
    import pytest
    import torch
    from hyper_connections_stream_b200 import _lib
    H = torch.zeros((2, 4, 16), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        _lib.read_rmsnorm(H, torch.ones(4))


def test_public_header_compiles_standalone_as_c_and_cpp(tmp_path):
    """include/hc_api.h is a C ABI: it must compile on its own (no CUDA headers)
    as C99 and as C++."""
    src = tmp_path / "use_header.c"
    src.write_text('#include "hc_api.h"\nint main(void) { return hc_version() < 0; }\n')
    inc = os.path.join(ROOT, "include")
    for cmd in (["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror"],
                ["g++", "-std=c++17", "-Wall", "-Wextra", "-Werror", "-x", "c++"]):
        out = subprocess.run([*cmd, "-I", inc, "-c", str(src), "-o", str(tmp_path / "o.o")],
                             capture_output=True, text=True)
        assert out.returncode == 0, (cmd[0], out.stderr)


def test_parameter_layouts():
    """Token strides the binding passes for shared and per-token parameters,
    including no tokens at all (a rank of the reduce-scatter form may own
    none) and a strided view of a wider per-token array."""
    import pytest
    import torch
    from hyper_connections_stream_b200._lib import _tok_layout
    n = 4
    assert _tok_layout("A", torch.zeros(n, n), 7, (n, n)) == 0
    assert _tok_layout("A", torch.zeros(0, n, n), 0, (n, n)) == n * n
    assert _tok_layout("a", torch.zeros(0, n), 0, (n,)) == n
    assert _tok_layout("A", torch.zeros(1, n, n), 1, (n, n)) == n * n
    assert _tok_layout("A", torch.zeros(5, n, n), 5, (n, n)) == n * n
    z = torch.zeros(5, 24)
    assert _tok_layout("a", z[:, 16:20], 5, (n,)) == 24
    with pytest.raises(ValueError):
        _tok_layout("A", torch.zeros(n, n).t(), 3, (n, n))       # shared but transposed
    with pytest.raises(ValueError):
        _tok_layout("A", torch.zeros(5, n, n).transpose(1, 2), 5, (n, n))
    with pytest.raises(ValueError):
        _tok_layout("A", torch.zeros(4, n, n), 5, (n, n))
