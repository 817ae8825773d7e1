"""The C-ABI library: loads without a GPU, exports every entry point the header
declares, and rejects bad arguments on the host before any CUDA call. CPU only."""

import ctypes
import os
import re
import subprocess

import pytest

import jagged_pointwise_attention_b200 as hstu
from jagged_pointwise_attention_b200 import _native
from jagged_pointwise_attention_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hstu.h")


@pytest.fixture(scope="module")
def lib():
    build()
    return _native.load()


def header_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(hstu_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_expected_entry_points():
    names = header_functions()
    for must in ("hstu_attn_fwd", "hstu_attn_plan", "hstu_attn_run", "hstu_layer_fwd",
                 "hstu_linear_fwd", "hstu_layernorm_gate_fwd", "hstu_device_status"):
        assert must in names


def test_every_header_symbol_is_exported(lib):
    out = subprocess.check_output(["nm", "-D", "--defined-only", _native.LIB_PATH], text=True)
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    missing = [n for n in header_functions() if n not in exported]
    assert not missing, missing
    # the binding declares exactly the header's functions
    assert sorted(_native.SIGNATURES) == header_functions()


def test_library_loads_without_gpu(lib):
    assert lib.hstu_abi_version() == 2
    assert lib.hstu_status_string(0) == b"ok"
    assert lib.hstu_status_string(4).startswith(b"device pipeline wait")


def test_workspace_queries(lib):
    # the plan's part: header + one int4 per (sequence, query tile), bounded by
    # T/128 + B + 1 and rounded up to 256 bytes, and as much again for the
    # per-unit sequence-start masks of packed tiles; then the run's bias
    # tables: 3968 bytes per head and distinct diagonal offset of the
    # position window, 576 bytes per unit of key summary
    units = min(90000 // 128 + 16 + 1, 16 * 64)
    plan = 256 + 2 * ((16 * units + 255) // 256 * 256)
    # 8192 positions: offsets 0 .. ceil((8192 + 126) / 128) = 65, capped at 64 tiles
    assert lib.hstu_attn_workspace_bytes(16, 90000, 8192, 4, 8192) == \
        plan + 4 * 64 * 3968 + 576 * units
    # 200 positions: offsets 0 .. ceil(326 / 128) = 3
    assert lib.hstu_attn_workspace_bytes(16, 90000, 8192, 2, 200) == \
        plan + 2 * 4 * 3968 + 576 * units
    assert lib.hstu_attn_workspace_bytes(-1, 10, 10, 1, 1) == 0
    assert lib.hstu_attn_workspace_bytes(1, 10, 0, 1, 1) == 0
    assert lib.hstu_attn_workspace_bytes(1, 10, 131073, 1, 1) == 0
    assert lib.hstu_attn_workspace_bytes(1, 10, 10, 0, 1) == 0
    lw = lib.hstu_layer_workspace_bytes(1000, 4, 512, 4, 128, 512)
    assert lw >= 1000 * 512 * 2 * 7          # U|V|Q|K, A, Y, LayerNorm(x)


def _attn(lib, **kw):
    a = dict(dtype=1, q=16, qs=512, k=16, ks=512, v=16, vs=512, off=16, B=2, T=10, H=4, dqk=128,
             dv=128, ts=None, pos=None, P=0, tb=None, NB=0, N=8, out=16, os=512, ws=16,
             wsb=1 << 20, stream=None)
    a.update(kw)
    return lib.hstu_attn_fwd(a["dtype"], a["q"], a["qs"], a["k"], a["ks"], a["v"], a["vs"],
                             a["off"], a["B"], a["T"], a["H"], a["dqk"], a["dv"], a["ts"],
                             a["pos"], a["P"], a["tb"], a["NB"], a["N"], a["out"], a["os"],
                             a["ws"], a["wsb"], a["stream"])


def test_attention_argument_validation(lib):
    INV, UNS = _native.HSTU_ERR_INVALID_ARG, _native.HSTU_ERR_UNSUPPORTED
    assert _attn(lib, dtype=7) == INV
    assert _attn(lib, q=None) == INV
    assert _attn(lib, off=None) == INV
    assert _attn(lib, N=0) == INV
    assert _attn(lib, N=131073) == INV
    assert _attn(lib, B=-1) == INV
    assert _attn(lib, qs=100) == INV                      # stride below H*d
    assert _attn(lib, qs=520, ks=520, vs=520, os=516) == INV   # not a multiple of 8
    assert _attn(lib, q=24) == INV                        # misaligned base
    assert _attn(lib, dqk=96, dv=96, qs=384, ks=384, vs=384, os=384) == UNS
    assert _attn(lib, dv=64, vs=256, os=256) == UNS       # d_qk != d_v on bf16
    # bf16 takes d in {32, 64, 128}: d = 32 gets past the head-dimension check
    # (and fails later, on the workspace), d = 48 does not
    d32 = dict(dqk=32, dv=32, qs=128, ks=128, vs=128, os=128)
    assert _attn(lib, wsb=64, **d32) == INV
    assert _attn(lib, dqk=48, dv=48, qs=192, ks=192, vs=192, os=192, wsb=64) == UNS
    assert _attn(lib, ws=None) == INV
    assert _attn(lib, wsb=64) == INV                      # workspace too small
    assert _attn(lib, tb=16, NB=0) == INV
    assert _attn(lib, tb=16, NB=1025) == INV
    assert _attn(lib, pos=16, P=0) == INV
    assert _attn(lib, dtype=0, dqk=129, dv=129, qs=1032, ks=1032, vs=1032, os=1032) == UNS
    # empty batches launch nothing and succeed without a GPU
    assert _attn(lib, B=0, T=0) == _native.HSTU_OK
    assert _attn(lib, T=0) == _native.HSTU_OK


def test_linear_and_ln_validation(lib):
    INV, UNS = _native.HSTU_ERR_INVALID_ARG, _native.HSTU_ERR_UNSUPPORTED
    # K % 64, N % 128
    assert lib.hstu_linear_fwd(16, 96, 10, 96, 16, 96, 128, None, 0, None, 0, 16, 128, None) == UNS
    assert lib.hstu_linear_fwd(16, 64, 10, 64, 16, 64, 100, None, 0, None, 0, 16, 100, None) == UNS
    assert lib.hstu_linear_fwd(16, 64, 10, 64, 16, 64, 128, None, 2, None, 0, 16, 128, None) == INV
    assert lib.hstu_linear_fwd(16, 64, 10, 64, 16, 64, 128, None, 9, None, 0, 16, 128, None) == INV
    assert lib.hstu_linear_fwd(16, 64, 0, 64, 16, 64, 128, None, 0, None, 0, 16, 128, None) == 0
    assert lib.hstu_layernorm_gate_fwd(16, 512, 16, 512, 4, 500, None, None,
                                       ctypes.c_float(1e-5), 16, 512, None) == UNS
    assert lib.hstu_layernorm_gate_fwd(None, 512, 16, 512, 4, 512, None, None,
                                       ctypes.c_float(1e-5), 16, 512, None) == INV
    assert lib.hstu_debug_wait_timeout(0, None) == INV


def test_fp8_validation(lib):
    INV, UNS = _native.HSTU_ERR_INVALID_ARG, _native.HSTU_ERR_UNSUPPORTED
    # quantization: K % 16, code row stride % 16, null scales, empty
    assert lib.hstu_quant_rows_e4m3(16, 104, 4, 100, 16, 112, 16, None) == UNS
    assert lib.hstu_quant_rows_e4m3(16, 128, 4, 128, 16, 136, 16, None) == INV
    assert lib.hstu_quant_rows_e4m3(16, 128, 4, 128, 16, 128, None, None) == INV
    assert lib.hstu_quant_rows_e4m3(16, 128, 0, 128, 16, 128, 16, None) == 0
    # FP8 linear: K % 128, missing scales, code strides % 16
    assert lib.hstu_linear_fp8_fwd(16, 64, 16, 10, 64, 16, 64, 16, 128, None, 0, None, 0, 16, 128,
                                   None) == UNS
    assert lib.hstu_linear_fp8_fwd(16, 128, None, 10, 128, 16, 128, 16, 128, None, 0, None, 0, 16,
                                   128, None) == INV
    assert lib.hstu_linear_fp8_fwd(16, 136, 16, 10, 128, 16, 128, 16, 128, None, 0, None, 0, 16,
                                   128, None) == INV
    # fused LayerNorm gate quantization: code stride % 16
    assert lib.hstu_layernorm_gate_fp8_fwd(16, 512, 16, 512, 4, 512, None, None,
                                           ctypes.c_float(1e-5), 16, 520, 16, None) == INV
    assert lib.hstu_layer_fp8_workspace_bytes(1000, 4, 512, 4, 128, 512) > 1000 * 512 * 2 * 5
    # LayerNorm (input norm) and its fused quantization: F % 256, strides
    assert lib.hstu_layernorm_fwd(16, 512, 4, 384, None, None, ctypes.c_float(1e-5), 16, 512,
                                  None) == UNS
    assert lib.hstu_layernorm_fwd(16, 500, 4, 512, None, None, ctypes.c_float(1e-5), 16, 512,
                                  None) == INV
    assert lib.hstu_layernorm_fp8_fwd(16, 512, 4, 512, None, None, ctypes.c_float(1e-5), 16, 520,
                                      16, None) == INV
    assert lib.hstu_layernorm_fwd(16, 512, 0, 512, None, None, ctypes.c_float(1e-5), 16, 512,
                                  None) == 0


def test_backward_validation(lib):
    INV, UNS = _native.HSTU_ERR_INVALID_ARG, _native.HSTU_ERR_UNSUPPORTED

    def bwd(**kw):
        a = dict(q=16, k=16, v=16, dout=16, off=16, B=2, T=10, H=2, dqk=32, dv=32, ts=None,
                 pos=None, P=0, tb=None, NB=0, N=8, dq=16, dk=16, dvv=16, dpos=None, dtime=None)
        a.update(kw)
        return lib.hstu_attn_bwd_f32(a["q"], a["k"], a["v"], a["dout"], a["off"], a["B"], a["T"],
                                     a["H"], a["dqk"], a["dv"], a["ts"], a["pos"], a["P"],
                                     a["tb"], a["NB"], a["N"], a["dq"], a["dk"], a["dvv"],
                                     a["dpos"], a["dtime"], None)
    assert bwd(dqk=129) == UNS
    assert bwd(H=0) == INV
    assert bwd(pos=16, P=8) == INV                       # dpos missing
    assert bwd(ts=16, tb=16, NB=8) == INV                # dtime missing
    assert bwd(ts=16, tb=16, NB=2000, dtime=16) == INV   # bucket count
    assert bwd(pos=16, P=13000, dpos=16) == UNS          # table partials exceed shared memory
    assert bwd(q=None) == INV
    assert bwd(B=0, T=0) == 0


def test_tc_backward_validation(lib):
    INV, UNS = _native.HSTU_ERR_INVALID_ARG, _native.HSTU_ERR_UNSUPPORTED
    BF16, F32 = _native.HSTU_DTYPE_BF16, _native.HSTU_DTYPE_F32

    def bwd(**kw):
        a = dict(dt=BF16, q=16, qs=256, k=16, ks=256, v=16, vs=256, dout=16, dos=256, off=16, B=2,
                 T=10, H=2, d=128, ts=None, pos=None, P=0, tb=None, NB=0, N=8, dq=16, dk=16,
                 dvv=16, dpos=None, dtime=None, ws=16, wsb=1 << 20)
        a.update(kw)
        return lib.hstu_attn_bwd(a["dt"], a["q"], a["qs"], a["k"], a["ks"], a["v"], a["vs"],
                                 a["dout"], a["dos"], a["off"], a["B"], a["T"], a["H"], a["d"],
                                 a["ts"], a["pos"], a["P"], a["tb"], a["NB"], a["N"], a["dq"],
                                 a["dk"], a["dvv"], a["dpos"], a["dtime"], a["ws"], a["wsb"], None)
    assert bwd(d=32) == UNS
    assert bwd(d=96) == UNS
    assert bwd(dt=F32) == UNS                           # the fp32 path is hstu_attn_bwd_f32
    assert bwd(dt=7) == INV
    assert bwd(H=0) == INV
    assert bwd(pos=16, P=8) == INV                      # dpos missing
    assert bwd(ts=16, tb=16, NB=8) == INV               # dtime missing
    assert bwd(ts=16, tb=16, NB=2000, dtime=16) == INV  # bucket count
    assert bwd(q=None) == INV
    assert bwd(ws=None) == INV
    assert bwd(qs=255) == INV                           # stride below H * d
    assert bwd(ks=264 + 4) == INV                       # stride not a multiple of 8
    assert bwd(dq=20) == INV                            # fp32 outputs 16-byte aligned
    assert bwd(wsb=8) == INV                            # workspace below the plan's size
    assert bwd(B=0, T=0) == 0
    assert lib.hstu_attn_bwd_workspace_bytes(4, 1000, 512) >= 256
    assert lib.hstu_attn_bwd_workspace_bytes(-1, 1000, 512) == 0


def test_binding_fails_loudly_without_library(tmp_path):
    with pytest.raises(ImportError):
        _native.load(str(tmp_path / "missing.so"))


def test_binding_rejects_cpu_tensors():
    import torch
    x = torch.zeros(4, 2, 64, dtype=torch.bfloat16)
    off = torch.tensor([0, 4])
    with pytest.raises(ValueError):
        hstu.hstu_attn_fwd(x, x, x, off, None, None, None, 4)
