"""B200-native fused WUSH blockwise transform + 4-bit quantisation.

Thin Python binding of the C ABI in ``include/wush.h`` (``libwush.so``, built in-tree
for sm_100a).  The functions carry the C names; they only marshal arguments: torch
tensors supply device memory and the current CUDA stream, every step of the
computation runs in the library's kernels.  There is no CPU fallback: if the library
is missing or cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

from ._build import LIB_PATH, build as build_library  # noqa: F401

__all__ = ["FMT", "WushError", "wush_quant_act", "wush_quant_weight", "wush_quant_act_debug",
           "wush_quant_weight_debug", "wush_quant_act_shared", "wush_quant_act_shared_debug",
           "wush_build_transforms", "wush_device_status", "wush_set_wait_limit_ns",
           "wush_selftest_wait_timeout", "wush_status_string", "wush_version", "load_library",
           "EXPORTED_SYMBOLS", "output_shapes", "wush_hadamard", "wush_dequant", "wush_gemm_mxfp4",
           "wush_mx_scales_to_atoms", "atom_bytes", "wush_quant_act_mx_atoms", "wush_quant_weight_mx_atoms",
           "wush_quant_act_shared_mx_atoms", "wush_gemm_nvfp4", "wush_quant_act_nv_atoms",
           "wush_quant_weight_nv_atoms", "wush_quant_act_nvfp4_amax", "wush_nvfp4_scale_from_amax",
           "wush_quant_act_nvfp4_with_scale", "wush_set_small_batch_rows", "wush_quant_act_nvfp4_onepass",
           "nvfp4_workspace", "wush_quant_act_nvfp4_onepass_noalloc", "wush_set_gemm_cta_pairs",
           "wush_quant_act_nv_atoms_onepass",
           "wush_last_error_detail"]

FMT = {"mxfp4": 0, "nvfp4": 1, "int4": 2}
STATUS = {0: "WUSH_OK", 1: "WUSH_ERR_INVALID_ARG", 2: "WUSH_ERR_UNSUPPORTED", 3: "WUSH_ERR_MISALIGNED",
          4: "WUSH_ERR_CUDA", 5: "WUSH_ERR_DEVICE_TIMEOUT"}
EXPORTED_SYMBOLS = ("wush_quant_act", "wush_quant_weight", "wush_quant_act_debug",
                    "wush_quant_weight_debug", "wush_quant_act_shared", "wush_quant_act_shared_debug",
                    "wush_dequant", "wush_gemm_mxfp4", "wush_mx_scales_to_atoms", "wush_quant_act_mx_atoms",
                    "wush_quant_weight_mx_atoms", "wush_quant_act_shared_mx_atoms",
                    "wush_gemm_nvfp4", "wush_quant_act_nv_atoms", "wush_quant_weight_nv_atoms",
                    "wush_quant_act_nvfp4_amax", "wush_nvfp4_scale_from_amax", "wush_quant_act_nvfp4_with_scale",
                    "wush_set_small_batch_rows", "wush_quant_act_nvfp4_onepass",
                    "wush_quant_act_nvfp4_onepass_noalloc", "wush_set_gemm_cta_pairs",
                    "wush_quant_act_nv_atoms_onepass",
                    "wush_build_transforms", "wush_hadamard", "wush_device_status",
                    "wush_set_wait_limit_ns",
                    "wush_selftest_wait_timeout", "wush_status_string", "wush_last_error_detail",
                    "wush_version")


class WushError(RuntimeError):
    """A non-zero wush_status; for WUSH_ERR_CUDA `detail` names the failing CUDA call.

    Raised on the thread that made the call, so the library's per-thread record of the
    failure is still the one for this call."""

    def __init__(self, status: int, where: str):
        self.status = status
        self.detail = wush_last_error_detail() if status == 4 else ""
        extra = f" [{self.detail}]" if self.detail else ""
        super().__init__(f"{where}: {wush_status_string(status)} (status {status}){extra}")


_LIB = None
_P, _I64, _I32, _U64 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_uint64


def load_library(path: str | None = None) -> ctypes.CDLL:
    """Load libwush.so (once) and declare the C signatures."""
    global _LIB
    if _LIB is not None and path is None:
        return _LIB
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise OSError(f"{p} is missing: build it with `python -m blockwise_adaptive_transforms_b200._build`")
    lib = ctypes.CDLL(p)
    quant = [_P, _P, _I64, _I64, _I32, _I32, _P, _P, _P, _P]
    lib.wush_quant_act.argtypes = quant
    lib.wush_quant_weight.argtypes = quant
    lib.wush_quant_act_shared.argtypes = quant
    dbg = [_P, _P, _I64, _I64, _I32, _I32, _P, _P, _P, _P, _P]
    lib.wush_quant_act_debug.argtypes = dbg
    lib.wush_quant_weight_debug.argtypes = dbg
    lib.wush_quant_act_shared_debug.argtypes = dbg
    for f in ("wush_quant_act", "wush_quant_weight", "wush_quant_act_debug", "wush_quant_weight_debug",
              "wush_quant_act_shared", "wush_quant_act_shared_debug"):
        getattr(lib, f).restype = ctypes.c_int
    lib.wush_dequant.argtypes = [_P, _P, _P, _I64, _I64, _I32, _I32, _P, _P]
    lib.wush_dequant.restype = ctypes.c_int
    for f in ("wush_quant_act_mx_atoms", "wush_quant_weight_mx_atoms", "wush_quant_act_shared_mx_atoms"):
        getattr(lib, f).argtypes = [_P, _P, _I64, _I64, _P, _P, _P]
        getattr(lib, f).restype = ctypes.c_int
    for f in ("wush_quant_act_nv_atoms", "wush_quant_weight_nv_atoms"):
        getattr(lib, f).argtypes = [_P, _P, _I64, _I64, _P, _P, _P, _P]
        getattr(lib, f).restype = ctypes.c_int
    lib.wush_gemm_mxfp4.argtypes = [_P, _P, _P, _P, _I64, _I64, _I64, _P, _P]
    lib.wush_gemm_mxfp4.restype = ctypes.c_int
    lib.wush_gemm_nvfp4.argtypes = [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _P, _P]
    lib.wush_gemm_nvfp4.restype = ctypes.c_int
    lib.wush_quant_act_nvfp4_amax.argtypes = [_P, _P, _I64, _I64, _P, _P]
    lib.wush_quant_act_nvfp4_amax.restype = ctypes.c_int
    lib.wush_nvfp4_scale_from_amax.argtypes = [_P, _P]
    lib.wush_nvfp4_scale_from_amax.restype = ctypes.c_int
    lib.wush_quant_act_nvfp4_with_scale.argtypes = [_P, _P, _I64, _I64, _P, _P, _P, _P]
    lib.wush_quant_act_nvfp4_with_scale.restype = ctypes.c_int
    lib.wush_mx_scales_to_atoms.argtypes = [_P, _I64, _I64, _P, _P]
    lib.wush_mx_scales_to_atoms.restype = ctypes.c_int
    lib.wush_build_transforms.argtypes = [_P, _P, _I64, _I64, _I64, _I32, ctypes.c_double, _I32,
                                          _P, _P, _P, _P, _P, _P]
    lib.wush_build_transforms.restype = ctypes.c_int
    lib.wush_hadamard.argtypes = [_I32, _I64, _P, _P]
    lib.wush_hadamard.restype = ctypes.c_int
    lib.wush_device_status.argtypes = [_P, ctypes.POINTER(ctypes.c_uint32)]
    lib.wush_device_status.restype = ctypes.c_int
    lib.wush_quant_act_nvfp4_onepass.argtypes = [_P, _P, _I64, _I64, _P, _P, _P, _P, _P]
    lib.wush_quant_act_nvfp4_onepass.restype = ctypes.c_int
    lib.wush_quant_act_nv_atoms_onepass.argtypes = [_P, _P, _I64, _I64, _P, _P, _P, _P, _P]
    lib.wush_quant_act_nv_atoms_onepass.restype = ctypes.c_int
    lib.wush_quant_act_nvfp4_onepass_noalloc.argtypes = [_P, _P, _I64, _I64, _P, _P, _P, _P]
    lib.wush_quant_act_nvfp4_onepass_noalloc.restype = ctypes.c_int
    lib.wush_set_gemm_cta_pairs.argtypes = [_I32]
    lib.wush_set_gemm_cta_pairs.restype = ctypes.c_int
    lib.wush_set_small_batch_rows.argtypes = [_I64]
    lib.wush_set_small_batch_rows.restype = ctypes.c_int
    lib.wush_set_wait_limit_ns.argtypes = [_U64]
    lib.wush_set_wait_limit_ns.restype = ctypes.c_int
    lib.wush_selftest_wait_timeout.argtypes = [_U64, _P, ctypes.POINTER(ctypes.c_uint32)]
    lib.wush_selftest_wait_timeout.restype = ctypes.c_int
    lib.wush_status_string.argtypes = [ctypes.c_int]
    lib.wush_status_string.restype = ctypes.c_char_p
    lib.wush_last_error_detail.argtypes = [ctypes.c_char_p, ctypes.c_size_t]
    lib.wush_last_error_detail.restype = ctypes.c_int
    lib.wush_version.argtypes = []
    lib.wush_version.restype = ctypes.c_int
    if path is None:
        _LIB = lib
    return lib


def wush_status_string(status: int) -> str:
    return load_library().wush_status_string(int(status)).decode()


def wush_last_error_detail() -> str:
    """The failing CUDA call behind this thread's last WUSH_ERR_CUDA (empty text if none)."""
    lib = load_library()
    buf = ctypes.create_string_buffer(512)
    lib.wush_last_error_detail(buf, len(buf))
    return buf.value.decode(errors="replace")


def wush_version() -> int:
    return int(load_library().wush_version())


def _stream_handle(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _launch_stream(stream, device) -> torch.cuda.Stream:
    """The stream a call launches on: ``stream`` (a torch stream or a raw handle), else the
    current stream of the input's device."""
    if torch.device(device).type != "cuda":
        raise TypeError("inputs must be CUDA tensors")
    if stream is None:
        return torch.cuda.current_stream(device)
    if isinstance(stream, torch.cuda.Stream):
        return stream
    return torch.cuda.ExternalStream(int(stream), device=device)


def _empty(shape, dtype, s, zero=False):
    """An output buffer allocated (and, if asked, zero-filled) on the launch stream s, so
    that torch's caching allocator orders its reuse after the launch and no fill on
    another stream races the kernel."""
    with torch.cuda.stream(s):
        return (torch.zeros if zero else torch.empty)(shape, dtype=dtype, device=s.device)


def _fmt_code(fmt) -> int:
    return FMT[fmt] if isinstance(fmt, str) else int(fmt)


def output_shapes(rows: int, d_in: int, G: int, fmt):
    """(codes shape, scales shape, scales dtype) of a call."""
    f = _fmt_code(fmt)
    return (rows, d_in // 2), (rows, d_in // G), (torch.float32 if f == FMT["int4"] else torch.uint8)


def _check_dev(t: torch.Tensor, name: str, dtype=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _alloc_outputs(s, rows: int, d_in: int, G: int, fmt, codes, scales, tensor_scale):
    cs, ss, sdt = output_shapes(rows, d_in, G, fmt)
    if codes is None:
        codes = _empty(cs, torch.uint8, s)
    if scales is None:
        scales = _empty(ss, sdt, s)
    if tensor_scale is None and _fmt_code(fmt) == FMT["nvfp4"]:
        tensor_scale = _empty(1, torch.float32, s)
    _check_dev(codes, "codes", torch.uint8)
    _check_dev(scales, "scales", sdt)
    if tuple(codes.shape) != cs or tuple(scales.shape) != ss:
        raise ValueError(f"output shapes must be codes {cs} and scales {ss}")
    if tensor_scale is not None:
        _check_dev(tensor_scale, "tensor_scale", torch.float32)
    return codes, scales, tensor_scale


def _ptr(t):
    return None if t is None else t.data_ptr()


def _call(fn_name, inp, in_dtype, T, G, fmt, codes, scales, tensor_scale, y, stream, shared=False):
    lib = load_library()
    _check_dev(inp, "input", in_dtype)
    _check_dev(T, "T", torch.float32)
    if inp.dim() != 2:
        raise ValueError("input must be 2-D [rows][d_in]")
    rows, d_in = int(inp.shape[0]), int(inp.shape[1])
    if d_in % G:
        raise ValueError("d_in must be a multiple of G")
    t_shape = (G, G) if shared else (d_in // G, G, G)
    if tuple(T.shape) != t_shape:
        raise ValueError(f"T must have shape {t_shape}")
    s = _launch_stream(stream, inp.device)
    codes, scales, tensor_scale = _alloc_outputs(s, rows, d_in, G, fmt, codes, scales, tensor_scale)
    args = [_ptr(inp), _ptr(T), rows, d_in, int(G), _fmt_code(fmt), _ptr(codes), _ptr(scales),
            _ptr(tensor_scale)]
    if y is not None:
        args.append(_ptr(y))
    args.append(s.cuda_stream)
    with torch.cuda.device(inp.device):
        st = getattr(lib, fn_name)(*args)
    if st != 0:
        raise WushError(st, fn_name)
    return codes, scales, tensor_scale


def wush_quant_act(x, T, G, fmt, codes=None, scales=None, tensor_scale=None, stream=None):
    """Activations x (bf16 [n_tok][d_in]) -> (codes u8 [n_tok][d_in/2], scales, tensor_scale)."""
    return _call("wush_quant_act", x, torch.bfloat16, T, G, fmt, codes, scales, tensor_scale, None, stream)


def wush_quant_weight(w, T, G, fmt, codes=None, scales=None, tensor_scale=None, stream=None):
    """Weights w (fp32 [d_out][d_in]) -> (codes, scales, tensor_scale)."""
    return _call("wush_quant_weight", w, torch.float32, T, G, fmt, codes, scales, tensor_scale, None, stream)


def _y_buffer(inp, y, stream):
    if y is None:
        y = _empty(inp.shape, torch.float32, _launch_stream(stream, inp.device))
    _check_dev(y, "y_out", torch.float32)
    if tuple(y.shape) != tuple(inp.shape):
        raise ValueError("y_out must have the input's shape")
    return y


def wush_quant_act_debug(x, T, G, fmt, y_out=None, stream=None):
    """As wush_quant_act, also returning the fp32 transformed values y the kernel quantised."""
    y = _y_buffer(x, y_out, stream)
    c, s, ts = _call("wush_quant_act_debug", x, torch.bfloat16, T, G, fmt, None, None, None, y, stream)
    return c, s, ts, y


def wush_quant_weight_debug(w, T, G, fmt, y_out=None, stream=None):
    y = _y_buffer(w, y_out, stream)
    c, s, ts = _call("wush_quant_weight_debug", w, torch.float32, T, G, fmt, None, None, None, y, stream)
    return c, s, ts, y


def wush_quant_act_shared(x, T, G, fmt, codes=None, scales=None, tensor_scale=None, stream=None):
    """H+Quant comparator: every block uses the one fp32 [G][G] matrix T (e.g. Hadamard)."""
    return _call("wush_quant_act_shared", x, torch.bfloat16, T, G, fmt, codes, scales, tensor_scale, None, stream,
                 shared=True)


def wush_quant_act_shared_debug(x, T, G, fmt, y_out=None, stream=None):
    y = _y_buffer(x, y_out, stream)
    c, s, ts = _call("wush_quant_act_shared_debug", x, torch.bfloat16, T, G, fmt, None, None, None, y, stream,
                     shared=True)
    return c, s, ts, y


def wush_dequant(codes, scales, tensor_scale, G, fmt, out=None, stream=None):
    """fp32 values [rows][d_in] represented by codes (u8 [rows][d_in/2]) and scales."""
    lib = load_library()
    _check_dev(codes, "codes", torch.uint8)
    if codes.dim() != 2:
        raise ValueError("codes must be 2-D [rows][d_in/2]")
    rows, d_in = int(codes.shape[0]), 2 * int(codes.shape[1])
    cs, ss, sdt = output_shapes(rows, d_in, G, fmt)
    _check_dev(scales, "scales", sdt)
    if tuple(scales.shape) != ss:
        raise ValueError(f"scales must have shape {ss}")
    if tensor_scale is not None:
        _check_dev(tensor_scale, "tensor_scale", torch.float32)
    s = _launch_stream(stream, codes.device)
    if out is None:
        out = _empty((rows, d_in), torch.float32, s)
    _check_dev(out, "out", torch.float32)
    if tuple(out.shape) != (rows, d_in):
        raise ValueError("out must be [rows][d_in]")
    with torch.cuda.device(codes.device):
        st = lib.wush_dequant(_ptr(codes), _ptr(scales), _ptr(tensor_scale), rows, d_in, int(G), _fmt_code(fmt),
                              _ptr(out), s.cuda_stream)
    if st != 0:
        raise WushError(st, "wush_dequant")
    return out


def atom_bytes(rows: int, C: int) -> int:
    """Size of the scale-atom buffer for [rows][C] scales (rows padded to 128, C to 4)."""
    return ((rows + 127) // 128 * 128) * ((C + 3) // 4 * 4)


def wush_mx_scales_to_atoms(scales, out=None, stream=None):
    """Row-major E8M0 scales u8 [rows][C] -> the tcgen05 scale-atom layout (u8, flat)."""
    lib = load_library()
    _check_dev(scales, "scales", torch.uint8)
    rows, C = int(scales.shape[0]), int(scales.shape[1])
    s = _launch_stream(stream, scales.device)
    if out is None:
        out = _empty(atom_bytes(rows, C), torch.uint8, s)
    _check_dev(out, "atoms", torch.uint8)
    if out.numel() < atom_bytes(rows, C):
        raise ValueError("atoms buffer too small")
    with torch.cuda.device(scales.device):
        st = lib.wush_mx_scales_to_atoms(_ptr(scales), rows, C, _ptr(out), s.cuda_stream)
    if st != 0:
        raise WushError(st, "wush_mx_scales_to_atoms")
    return out


def _quant_atoms(fn_name, inp, in_dtype, T, codes, atoms, stream, shared=False, G=32, tensor_scale=None):
    lib = load_library()
    _check_dev(inp, "input", in_dtype)
    _check_dev(T, "T", torch.float32)
    rows, d_in = int(inp.shape[0]), int(inp.shape[1])
    if d_in % G:
        raise ValueError(f"d_in must be a multiple of {G}")
    t_shape = (G, G) if shared else (d_in // G, G, G)
    if tuple(T.shape) != t_shape:
        raise ValueError(f"T must have shape {t_shape}")
    s = _launch_stream(stream, inp.device)
    if codes is None:
        codes = _empty((rows, d_in // 2), torch.uint8, s)
    if atoms is None:
        atoms = _empty(atom_bytes(rows, d_in // G), torch.uint8, s, zero=True)
    _check_dev(codes, "codes", torch.uint8)
    _check_dev(atoms, "scale atoms", torch.uint8)
    if tuple(codes.shape) != (rows, d_in // 2) or atoms.numel() < atom_bytes(rows, d_in // G):
        raise ValueError("output buffers have the wrong size")
    args = [_ptr(inp), _ptr(T), rows, d_in, _ptr(codes), _ptr(atoms)]
    if G == 16:
        if tensor_scale is None:
            tensor_scale = _empty(1, torch.float32, s)
        _check_dev(tensor_scale, "tensor_scale", torch.float32)
        args.append(_ptr(tensor_scale))
    with torch.cuda.device(inp.device):
        st = getattr(lib, fn_name)(*args, s.cuda_stream)
    if st != 0:
        raise WushError(st, fn_name)
    return (codes, atoms) if G == 32 else (codes, atoms, tensor_scale)


def wush_quant_act_mx_atoms(x, T, codes=None, atoms=None, stream=None):
    """MXFP4 activations with the scales written in the scale-atom layout: (codes, atoms)."""
    return _quant_atoms("wush_quant_act_mx_atoms", x, torch.bfloat16, T, codes, atoms, stream)


def wush_quant_weight_mx_atoms(w, T, codes=None, atoms=None, stream=None):
    return _quant_atoms("wush_quant_weight_mx_atoms", w, torch.float32, T, codes, atoms, stream)


def wush_quant_act_shared_mx_atoms(x, T, codes=None, atoms=None, stream=None):
    return _quant_atoms("wush_quant_act_shared_mx_atoms", x, torch.bfloat16, T, codes, atoms, stream, shared=True)


def wush_quant_act_nv_atoms(x, T, codes=None, atoms=None, tensor_scale=None, stream=None):
    """NVFP4 activations with the E4M3 scales in the scale-atom layout:
    (codes, atoms, tensor_scale)."""
    return _quant_atoms("wush_quant_act_nv_atoms", x, torch.bfloat16, T, codes, atoms, stream, G=16,
                        tensor_scale=tensor_scale)


def wush_quant_weight_nv_atoms(w, T, codes=None, atoms=None, tensor_scale=None, stream=None):
    return _quant_atoms("wush_quant_weight_nv_atoms", w, torch.float32, T, codes, atoms, stream, G=16,
                        tensor_scale=tensor_scale)


def _nv_stage_input(x, T):
    _check_dev(x, "x", torch.bfloat16)
    _check_dev(T, "T", torch.float32)
    n, d = int(x.shape[0]), int(x.shape[1])
    if d % 16 or tuple(T.shape) != (d // 16, 16, 16):
        raise ValueError("NVFP4 needs d_in % 16 == 0 and T of shape [d_in/16][16][16]")
    return n, d


def wush_quant_act_nvfp4_amax(x, T, amax=None, stream=None):
    """max |y| of this batch's G = 16 WUSH transform as a device fp32 tensor of one element
    (the first NVFP4 stage; reduce it across ranks before fixing the scale)."""
    lib = load_library()
    n, d = _nv_stage_input(x, T)
    s = _launch_stream(stream, x.device)
    if amax is None:
        amax = _empty(1, torch.float32, s)
    _check_dev(amax, "amax", torch.float32)
    with torch.cuda.device(x.device):
        st = lib.wush_quant_act_nvfp4_amax(_ptr(x), _ptr(T), n, d, _ptr(amax), s.cuda_stream)
    if st != 0:
        raise WushError(st, "wush_quant_act_nvfp4_amax")
    return amax


def wush_nvfp4_scale_from_amax(amax, stream=None):
    """In place: amax -> the tensor scale amax / 2688."""
    lib = load_library()
    _check_dev(amax, "amax", torch.float32)
    s = _launch_stream(stream, amax.device)
    with torch.cuda.device(amax.device):
        st = lib.wush_nvfp4_scale_from_amax(_ptr(amax), s.cuda_stream)
    if st != 0:
        raise WushError(st, "wush_nvfp4_scale_from_amax")
    return amax


def wush_quant_act_nvfp4_with_scale(x, T, tensor_scale, codes=None, scales=None, stream=None):
    """NVFP4 codes and E4M3 scales of x under a given device tensor scale: (codes, scales)."""
    lib = load_library()
    n, d = _nv_stage_input(x, T)
    _check_dev(tensor_scale, "tensor_scale", torch.float32)
    s = _launch_stream(stream, x.device)
    if codes is None:
        codes = _empty((n, d // 2), torch.uint8, s)
    if scales is None:
        scales = _empty((n, d // 16), torch.uint8, s)
    _check_dev(codes, "codes", torch.uint8)
    _check_dev(scales, "scales", torch.uint8)
    if tuple(codes.shape) != (n, d // 2) or tuple(scales.shape) != (n, d // 16):
        raise ValueError("output buffers have the wrong size")
    with torch.cuda.device(x.device):
        st = lib.wush_quant_act_nvfp4_with_scale(_ptr(x), _ptr(T), n, d, _ptr(codes), _ptr(scales),
                                                 _ptr(tensor_scale), s.cuda_stream)
    if st != 0:
        raise WushError(st, "wush_quant_act_nvfp4_with_scale")
    return codes, scales


def nvfp4_workspace(device=None, stream=None):
    """A zeroed workspace for wush_quant_act_nvfp4_onepass (16 bytes of device memory),
    allocated and zeroed on ``stream`` (default: the device's current stream)."""
    dev = torch.device(device if device is not None else "cuda")
    if dev.type == "cuda" and dev.index is None:
        dev = torch.device("cuda", torch.cuda.current_device())
    return _empty(4, torch.int32, _launch_stream(stream, dev), zero=True)


def wush_quant_act_nvfp4_onepass(x, T, workspace, codes=None, scales=None, tensor_scale=None, stream=None):
    """NVFP4 activations in one launch: (codes, scales, tensor_scale).  Decode-sized batches
    on CUDA cores, larger ones on the tensor-core kernel (one cooperative launch).
    ``workspace``: from nvfp4_workspace(); zero before the first call, left zero by each."""
    lib = load_library()
    n, d = _nv_stage_input(x, T)
    _check_dev(workspace, "workspace", torch.int32)
    s = _launch_stream(stream, x.device)
    if codes is None:
        codes = _empty((n, d // 2), torch.uint8, s)
    if scales is None:
        scales = _empty((n, d // 16), torch.uint8, s)
    if tensor_scale is None:
        tensor_scale = _empty(1, torch.float32, s)
    for t, name, dt in ((codes, "codes", torch.uint8), (scales, "scales", torch.uint8),
                        (tensor_scale, "tensor_scale", torch.float32)):
        _check_dev(t, name, dt)
    if tuple(codes.shape) != (n, d // 2) or tuple(scales.shape) != (n, d // 16) or workspace.numel() < 4:
        raise ValueError("output or workspace buffers have the wrong size")
    with torch.cuda.device(x.device):
        st = lib.wush_quant_act_nvfp4_onepass(_ptr(x), _ptr(T), n, d, _ptr(codes), _ptr(scales), _ptr(tensor_scale),
                                              _ptr(workspace), s.cuda_stream)
    if st != 0:
        raise WushError(st, "wush_quant_act_nvfp4_onepass")
    return codes, scales, tensor_scale


def wush_quant_act_nv_atoms_onepass(x, T, workspace, codes=None, atoms=None, tensor_scale=None, stream=None):
    """NVFP4 activations in one launch of the tensor-core kernel with the E4M3 scales in the
    scale-atom layout: (codes, atoms, tensor_scale).  ``workspace``: from nvfp4_workspace()."""
    lib = load_library()
    n, d = _nv_stage_input(x, T)
    _check_dev(workspace, "workspace", torch.int32)
    s = _launch_stream(stream, x.device)
    if codes is None:
        codes = _empty((n, d // 2), torch.uint8, s)
    if atoms is None:
        atoms = _empty(atom_bytes(n, d // 16), torch.uint8, s, zero=True)
    if tensor_scale is None:
        tensor_scale = _empty(1, torch.float32, s)
    for t, name, dt in ((codes, "codes", torch.uint8), (atoms, "scale atoms", torch.uint8),
                        (tensor_scale, "tensor_scale", torch.float32)):
        _check_dev(t, name, dt)
    if tuple(codes.shape) != (n, d // 2) or atoms.numel() < atom_bytes(n, d // 16) or workspace.numel() < 4:
        raise ValueError("output or workspace buffers have the wrong size")
    with torch.cuda.device(x.device):
        st = lib.wush_quant_act_nv_atoms_onepass(_ptr(x), _ptr(T), n, d, _ptr(codes), _ptr(atoms), _ptr(tensor_scale),
                                                 _ptr(workspace), s.cuda_stream)
    if st != 0:
        raise WushError(st, "wush_quant_act_nv_atoms_onepass")
    return codes, atoms, tensor_scale


def wush_quant_act_nvfp4_onepass_noalloc(x, T, codes=None, scales=None, tensor_scale=None, stream=None):
    """As wush_quant_act_nvfp4_onepass on the library's own static scratch (no workspace;
    calls that may overlap race).  Returns (codes, scales, tensor_scale)."""
    lib = load_library()
    n, d = _nv_stage_input(x, T)
    s = _launch_stream(stream, x.device)
    if codes is None:
        codes = _empty((n, d // 2), torch.uint8, s)
    if scales is None:
        scales = _empty((n, d // 16), torch.uint8, s)
    if tensor_scale is None:
        tensor_scale = _empty(1, torch.float32, s)
    for t, name, dt in ((codes, "codes", torch.uint8), (scales, "scales", torch.uint8),
                        (tensor_scale, "tensor_scale", torch.float32)):
        _check_dev(t, name, dt)
    if tuple(codes.shape) != (n, d // 2) or tuple(scales.shape) != (n, d // 16):
        raise ValueError("output buffers have the wrong size")
    with torch.cuda.device(x.device):
        st = lib.wush_quant_act_nvfp4_onepass_noalloc(_ptr(x), _ptr(T), n, d, _ptr(codes), _ptr(scales),
                                                      _ptr(tensor_scale), s.cuda_stream)
    if st != 0:
        raise WushError(st, "wush_quant_act_nvfp4_onepass_noalloc")
    return codes, scales, tensor_scale


def _gemm_args(a_codes, a_atoms, b_codes, b_atoms, out, vs, s):
    for t, n in ((a_codes, "a_codes"), (b_codes, "b_codes"), (a_atoms, "a_atoms"), (b_atoms, "b_atoms")):
        _check_dev(t, n, torch.uint8)
    M, K2 = int(a_codes.shape[0]), int(a_codes.shape[1])
    N = int(b_codes.shape[0])
    if int(b_codes.shape[1]) != K2:
        raise ValueError("A and B must share K")
    K = 2 * K2
    if a_atoms.numel() < atom_bytes(M, K // vs) or b_atoms.numel() < atom_bytes(N, K // vs):
        raise ValueError("scale atom buffers too small")
    if out is None:
        out = _empty((M, N), torch.bfloat16, s)
    _check_dev(out, "out", torch.bfloat16)
    if tuple(out.shape) != (M, N):
        raise ValueError("out must be [M][N]")
    return M, N, K, out


def wush_gemm_mxfp4(a_codes, a_atoms, b_codes, b_atoms, out=None, stream=None):
    """bf16 [M][N] = A B^T from MXFP4 codes ([M][K/2], [N][K/2]) and scale atoms."""
    lib = load_library()
    s = _launch_stream(stream, a_codes.device)
    M, N, K, out = _gemm_args(a_codes, a_atoms, b_codes, b_atoms, out, 32, s)
    with torch.cuda.device(a_codes.device):
        st = lib.wush_gemm_mxfp4(_ptr(a_codes), _ptr(a_atoms), _ptr(b_codes), _ptr(b_atoms), M, N, K, _ptr(out),
                                 s.cuda_stream)
    if st != 0:
        raise WushError(st, "wush_gemm_mxfp4")
    return out


def wush_gemm_nvfp4(a_codes, a_atoms, a_tensor_scale, b_codes, b_atoms, b_tensor_scale, out=None, stream=None):
    """bf16 [M][N] = s_A s_B A B^T from NVFP4 codes, E4M3 scale atoms and the two fp32
    tensor scales (device tensors of one element)."""
    lib = load_library()
    s = _launch_stream(stream, a_codes.device)
    M, N, K, out = _gemm_args(a_codes, a_atoms, b_codes, b_atoms, out, 16, s)
    _check_dev(a_tensor_scale, "a_tensor_scale", torch.float32)
    _check_dev(b_tensor_scale, "b_tensor_scale", torch.float32)
    with torch.cuda.device(a_codes.device):
        st = lib.wush_gemm_nvfp4(_ptr(a_codes), _ptr(a_atoms), _ptr(a_tensor_scale), _ptr(b_codes), _ptr(b_atoms),
                                 _ptr(b_tensor_scale), M, N, K, _ptr(out), s.cuda_stream)
    if st != 0:
        raise WushError(st, "wush_gemm_nvfp4")
    return out


def wush_hadamard(G, copies=None, device=None, stream=None):
    """The normalised Sylvester Hadamard matrix of order G, written on the device by the
    library: fp32 [G][G], or [copies][G][G] when ``copies`` is given (the per-block form of
    the Hadamard-only transform).  One copy is the shared matrix of the H+Quant comparator."""
    lib = load_library()
    dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
    if dev.type != "cuda":
        raise TypeError("wush_hadamard writes device memory; give a CUDA device")
    n = 1 if copies is None else int(copies)
    s = _launch_stream(stream, dev)
    out = _empty((n, G, G) if copies is not None else (G, G), torch.float32, s)
    with torch.cuda.device(dev):
        st = lib.wush_hadamard(int(G), n, _ptr(out), s.cuda_stream)
    if st != 0:
        raise WushError(st, "wush_hadamard")
    return out


def wush_build_transforms(w, xcal, G, lam=0.01, use_hadamard=True, want_f64=False, stream=None):
    """Per-block WUSH transforms of one layer, built on the device in fp64.

    w: fp32 [d_out][d_in] weights; xcal: bf16 [n_cal][d_in] calibration activations.
    Returns (T_wush, T_xvsh) as fp32 [C][G][G]; with ``want_f64`` also the fp64
    transforms and the singular values: (T_wush, T_xvsh, T_wush64, T_xvsh64, s64)."""
    lib = load_library()
    _check_dev(w, "w", torch.float32)
    _check_dev(xcal, "xcal", torch.bfloat16)
    if w.dim() != 2 or xcal.dim() != 2 or w.shape[1] != xcal.shape[1]:
        raise ValueError("w [d_out][d_in] and xcal [n_cal][d_in] must share d_in")
    d_out, d_in = int(w.shape[0]), int(w.shape[1])
    n_cal = int(xcal.shape[0])
    if d_in % G:
        raise ValueError("d_in must be a multiple of G")
    C = d_in // G
    dev = w.device
    s = _launch_stream(stream, dev)
    Tw = _empty((C, G, G), torch.float32, s)
    Tx = _empty((C, G, G), torch.float32, s)
    Tw64 = Tx64 = s64 = None
    if want_f64:
        Tw64 = _empty((C, G, G), torch.float64, s)
        Tx64 = _empty((C, G, G), torch.float64, s)
        s64 = _empty((C, G), torch.float64, s)
    with torch.cuda.device(dev):
        st = lib.wush_build_transforms(_ptr(w), _ptr(xcal), d_out, n_cal, d_in, int(G), float(lam),
                                       1 if use_hadamard else 0, _ptr(Tw), _ptr(Tx), _ptr(Tw64),
                                       _ptr(Tx64), _ptr(s64), s.cuda_stream)
    if st != 0:
        raise WushError(st, "wush_build_transforms")
    return (Tw, Tx, Tw64, Tx64, s64) if want_f64 else (Tw, Tx)


def wush_device_status(stream=None):
    """Synchronise the stream, read and clear the device error word: (status, bits)."""
    bits = ctypes.c_uint32(0)
    st = load_library().wush_device_status(_stream_handle(stream), ctypes.byref(bits))
    return int(st), int(bits.value)


def wush_set_gemm_cta_pairs(enable: bool) -> None:
    """FP4 GEMMs with M % 256 == 0 on CTA pairs, or (default) always on single CTAs."""
    load_library().wush_set_gemm_cta_pairs(1 if enable else 0)


def wush_set_small_batch_rows(rows: int) -> None:
    """Activation batches of at most `rows` rows use the CUDA-core path (0: never; < 0: default)."""
    st = load_library().wush_set_small_batch_rows(int(rows))
    if st != 0:
        raise WushError(st, "wush_set_small_batch_rows")


def wush_set_wait_limit_ns(ns: int) -> None:
    load_library().wush_set_wait_limit_ns(int(ns))


def wush_selftest_wait_timeout(limit_ns: int, stream=None):
    bits = ctypes.c_uint32(0)
    st = load_library().wush_selftest_wait_timeout(int(limit_ns), _stream_handle(stream), ctypes.byref(bits))
    return int(st), int(bits.value)
