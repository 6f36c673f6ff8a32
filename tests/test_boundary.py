"""The C ABI boundary without a GPU: the library loads, exports every symbol that
include/wush.h declares, and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re

import pytest

import blockwise_adaptive_transforms_b200 as W
from blockwise_adaptive_transforms_b200 import _build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "wush.h")

OK, INVALID, UNSUPPORTED, MISALIGNED = 0, 1, 2, 3


@pytest.fixture(scope="module")
def lib():
    _build.build()
    return W.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(wush_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_documented_entry_points():
    names = declared_functions()
    for required in ("wush_quant_act", "wush_quant_weight", "wush_status_string"):
        assert required in names
    assert set(names) == set(W.EXPORTED_SYMBOLS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    # and they are C symbols (no C++ mangling)
    nm = os.popen(f"nm -D --defined-only {W.LIB_PATH}").read()
    for name in declared_functions():
        assert re.search(rf"\bT {name}$", nm, re.M), name


def test_status_strings_and_version(lib):
    assert W.wush_status_string(0) == "WUSH_OK"
    for s in range(1, 6):
        assert W.wush_status_string(s).startswith(W.STATUS[s])
    assert "unknown" in W.wush_status_string(99)
    assert W.wush_version() == 100


# fake, never-dereferenced addresses: every call below returns before touching CUDA
A16 = 0x10000
A4 = 0x20004
A1 = 0x30001


def call_act(lib, x=A16, T=A16, n=128, d=256, G=32, fmt=0, codes=A16, scales=A16, ts=None):
    return lib.wush_quant_act(x, T, n, d, G, fmt, codes, scales, ts, None)


def test_null_pointers_rejected(lib):
    assert call_act(lib, x=None) == INVALID
    assert call_act(lib, T=None) == INVALID
    assert call_act(lib, codes=None) == INVALID
    assert call_act(lib, scales=None) == INVALID
    assert call_act(lib, fmt=1, G=16, ts=None) == INVALID            # NVFP4 needs tensor_scale
    assert lib.wush_quant_weight(None, A16, 8, 64, 32, 0, A16, A16, None, None) == INVALID
    assert lib.wush_quant_act_debug(A16, A16, 8, 64, 32, 0, A16, A16, None, None, None) == INVALID


def test_sizes_rejected(lib):
    assert call_act(lib, n=-1) == INVALID
    assert call_act(lib, d=0) == INVALID
    assert call_act(lib, d=-32) == INVALID
    assert call_act(lib, d=48) == INVALID                # not a multiple of G = 32
    assert call_act(lib, d=40, G=16, fmt=2) == INVALID
    assert call_act(lib, n=2 ** 31) == INVALID
    assert call_act(lib, d=2 ** 31 + 32) == INVALID


def test_unsupported_format_and_group(lib):
    assert call_act(lib, fmt=3) == UNSUPPORTED
    assert call_act(lib, fmt=-1) == UNSUPPORTED
    assert call_act(lib, fmt=0, G=16) == UNSUPPORTED     # MXFP4 groups are 32
    assert call_act(lib, fmt=1, G=32, ts=A16) == UNSUPPORTED  # NVFP4 groups are 16
    assert call_act(lib, fmt=2, G=64) == UNSUPPORTED
    assert call_act(lib, fmt=2, G=8) == UNSUPPORTED


def test_misaligned_pointers(lib):
    assert call_act(lib, x=A16 + 2) == MISALIGNED
    assert call_act(lib, T=A4) == MISALIGNED
    assert call_act(lib, codes=A16 + 8) == MISALIGNED
    assert call_act(lib, fmt=2, scales=A1) == MISALIGNED       # INT4 scales are fp32
    assert call_act(lib, fmt=0, scales=A1, n=0) == OK          # byte scales need no alignment
    assert call_act(lib, fmt=1, G=16, ts=A1) == MISALIGNED
    assert lib.wush_quant_act_debug(A16, A16, 8, 64, 32, 0, A16, A16, None, A4, None) == MISALIGNED


def test_empty_batch_is_ok_without_launch(lib):
    assert call_act(lib, n=0) == OK
    assert call_act(lib, n=0, x=None, codes=None, scales=None) == OK   # empty tensors have no storage
    assert call_act(lib, n=0, fmt=0, G=16) == UNSUPPORTED
    assert lib.wush_quant_weight(A16, A16, 0, 64, 32, 0, A16, A16, None, None) == OK
    assert call_act(lib, n=0, fmt=1, G=16, ts=A16) == OK


def test_wait_limit_setter(lib):
    assert lib.wush_set_wait_limit_ns(0) == OK
    assert lib.wush_set_wait_limit_ns(5_000_000_000) == OK
    assert lib.wush_set_wait_limit_ns(0) == OK


def test_python_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(4, 64, dtype=torch.bfloat16)
    T = torch.zeros(2, 32, 32)
    with pytest.raises(TypeError):
        W.wush_quant_act(x, T, 32, "mxfp4")


def test_build_flags_target_sm100a_only():
    assert _build.ARCH_FLAGS == ["-gencode", "arch=compute_100a,code=sm_100a"]


def test_builder_argument_checks(lib):
    b = lib.wush_build_transforms
    assert b(A16, A16, 64, 64, 256, 8, 0.01, 1, A16, A16, None, None, None, None) == UNSUPPORTED
    assert b(A16, A16, 0, 64, 256, 32, 0.01, 1, A16, A16, None, None, None, None) == INVALID
    assert b(A16, A16, 64, 0, 256, 32, 0.01, 1, A16, A16, None, None, None, None) == INVALID
    assert b(A16, A16, 64, 64, 250, 32, 0.01, 1, A16, A16, None, None, None, None) == INVALID
    assert b(A16, A16, 64, 64, 256, 32, -1.0, 1, A16, A16, None, None, None, None) == INVALID
    assert b(A16, A16, 64, 64, 256, 32, float("nan"), 1, A16, A16, None, None, None, None) == INVALID
    assert b(None, A16, 64, 64, 256, 32, 0.01, 1, A16, A16, None, None, None, None) == INVALID
    assert b(A16, A16, 64, 64, 256, 32, 0.01, 1, None, A16, None, None, None, None) == INVALID
    assert b(A16 + 2, A16, 64, 64, 256, 32, 0.01, 1, A16, A16, None, None, None, None) == MISALIGNED
    assert b(A16, A1, 64, 64, 256, 32, 0.01, 1, A16, A16, None, None, None, None) == MISALIGNED
    assert b(A16, A16, 64, 64, 256, 32, 0.01, 1, A16, A16, A4, None, None, None) == MISALIGNED


def test_error_detail_buffer_contract(lib):
    # nothing has failed on this (fresh) thread yet
    import threading
    out = {}

    def fresh():
        out["n"] = lib.wush_last_error_detail(None, 0)
        buf = ctypes.create_string_buffer(8)
        out["short"] = (lib.wush_last_error_detail(buf, len(buf)), buf.value)

    t = threading.Thread(target=fresh)
    t.start()
    t.join()
    assert out["n"] == len("no CUDA failure recorded on this thread")
    n, text = out["short"]
    assert n == out["n"] and text == b"no CUDA"        # truncated to len - 1, NUL-terminated


@pytest.mark.skipif(__import__("torch").cuda.is_available(), reason="needs a machine without a GPU")
def test_cuda_failure_names_the_failing_call(lib):
    # without a device the status query's stream synchronisation fails in the runtime
    bits = ctypes.c_uint32(0)
    assert lib.wush_device_status(None, ctypes.byref(bits)) == 4
    detail = W.wush_last_error_detail()
    assert detail.startswith("cudaStreamSynchronize(") and "failed: cudaError" in detail, detail
    e = W.WushError(4, "wush_device_status")
    assert e.detail == detail and detail in str(e)


def test_binding_rejects_host_tensors_before_any_cuda_call():
    # the binding's type checks come before it looks for a stream or a device
    import torch
    x = torch.zeros((4, 32), dtype=torch.bfloat16)
    T = torch.zeros((1, 32, 32), dtype=torch.float32)
    with pytest.raises(TypeError):
        W.wush_quant_act(x, T, 32, "mxfp4")
    with pytest.raises(TypeError):
        W.wush_quant_act_mx_atoms(x, T)
    with pytest.raises(TypeError):
        W.nvfp4_workspace("cpu")
    with pytest.raises(TypeError):
        W._launch_stream(None, torch.device("cpu"))
    x16 = torch.zeros((4, 32), dtype=torch.bfloat16)
    T16 = torch.zeros((2, 16, 16), dtype=torch.float32)
    ws = torch.zeros(4, dtype=torch.int32)
    for call in (lambda: W.wush_quant_act_nvfp4_onepass(x16, T16, ws),
                 lambda: W.wush_quant_act_nv_atoms_onepass(x16, T16, ws),
                 lambda: W.wush_quant_act_nvfp4_onepass_noalloc(x16, T16)):
        with pytest.raises(TypeError):
            call()


def test_hadamard_argument_checks(lib):
    assert lib.wush_hadamard(3, 1, A16, None) == UNSUPPORTED          # not a power of two
    assert lib.wush_hadamard(0, 1, A16, None) == UNSUPPORTED
    assert lib.wush_hadamard(512, 1, A16, None) == UNSUPPORTED        # above 256
    assert lib.wush_hadamard(32, -1, A16, None) == INVALID
    assert lib.wush_hadamard(32, 2 ** 40, A16, None) == INVALID       # more than 2^40 entries
    assert lib.wush_hadamard(32, 1, None, None) == INVALID
    assert lib.wush_hadamard(32, 1, A1, None) == MISALIGNED
    assert lib.wush_hadamard(32, 0, None, None) == OK                 # nothing to write


def test_noalloc_checks_arguments_before_any_cuda_call(lib):
    f = lib.wush_quant_act_nvfp4_onepass_noalloc
    assert f(None, A16, 8, 64, A16, A16, A4, None) == INVALID
    assert f(A16, A16, 8, 64, A16, A16, None, None) == INVALID        # tensor_scale is an output
    assert f(A16, A16, -1, 64, A16, A16, A4, None) == INVALID
    assert f(A16, A16, 8, 40, A16, A16, A4, None) == INVALID          # d_in % 16
    assert f(A1, A16, 8, 64, A16, A16, A4, None) == MISALIGNED
    assert f(A16, A16, 8, 64, A16, A16, A1, None) == MISALIGNED
    assert f(A16, A16, 0, 64, None, None, None, None) == OK           # empty batch
    g = lib.wush_quant_act_nvfp4_onepass
    assert g(A16, A16, 8, 64, A16, A16, A4, None, None) == INVALID    # workspace required
    assert g(A16, A16, 8, 64, A16, A16, A4, A4, None) == MISALIGNED
    h = lib.wush_quant_act_nv_atoms_onepass
    assert h(A16, A16, 8, 64, A16, A16, A4, None, None) == INVALID    # workspace required
    assert h(A16, A16, 8, 64, A16, A16, A4, A4, None) == MISALIGNED   # workspace alignment
    assert h(A16, A16, 8, 64, A16, A4, A4, A16, None) == MISALIGNED   # scale atoms alignment
    assert h(A16, A16, 8, 40, A16, A16, A4, A16, None) == INVALID     # d_in % 16
    assert h(A16, A16, 0, 64, None, None, None, None, None) == OK     # empty batch
