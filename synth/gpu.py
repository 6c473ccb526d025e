"""Device-side generation of the large synthetic caches (same bytes as the
NumPy generator in ``synth``; checked by tests/test_gpu_synth.py)."""
from __future__ import annotations

import ctypes as C
import os
import shutil
import subprocess

import torch

import synth

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth_kernels.cu")
_LIB = os.path.join(_HERE, "_build", "libcsa2synth.so")
_lib = None


def build(force=False):
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        os.makedirs(os.path.dirname(_LIB), exist_ok=True)
        nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-Xcompiler", "-fPIC",
                               "-shared", _SRC, "-o", tmp])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(build())
        _lib.synth_mxfp4_rows.restype = C.c_int
        _lib.synth_mxfp4_rows.argtypes = [C.c_void_p, C.c_void_p, C.c_uint64, C.c_uint64, C.c_uint64, C.c_int,
                                          C.c_int64, C.c_int64, C.c_int, C.c_void_p]
        _lib.synth_e4m3_rows.restype = C.c_int
        _lib.synth_e4m3_rows.argtypes = [C.c_void_p, C.c_uint64, C.c_int64, C.c_int64, C.c_int, C.c_void_p]
        _lib.synth_normal_bf16.restype = C.c_int
        _lib.synth_normal_bf16.argtypes = [C.c_void_p, C.c_uint64, C.c_int64, C.c_int64, C.c_void_p]
    return _lib


def _stream():
    return C.c_void_p(torch.cuda.current_stream().cuda_stream)


def mxfp4_rows_into(codes, scales, seed, t_codes, t_scales, seq, layer, r0, nrows, n, lognormal=False):
    """Fill device tensors codes [nrows, n/2] / scales [nrows, n/32] (views)."""
    assert codes.is_cuda and codes.is_contiguous() and scales.is_contiguous()
    kc = int(synth.stream_key(seed, t_codes, seq, layer))
    ks = int(synth.stream_key(seed, t_scales, seq, layer))
    kn = int(synth.stream_key(seed, synth.T_ROWNORM, seq, 0))
    rc = lib().synth_mxfp4_rows(codes.data_ptr(), scales.data_ptr(), kc, ks, kn, int(lognormal), r0, nrows, n,
                                _stream())
    if rc != 0:
        raise RuntimeError(f"synth_mxfp4_rows failed: cuda error {rc}")


def e4m3_rows_into(out, seed, tensor, seq, layer, r0, nrows, n=512):
    assert out.is_cuda and out.is_contiguous()
    key = int(synth.stream_key(seed, tensor, seq, layer))
    rc = lib().synth_e4m3_rows(out.data_ptr(), key, r0, nrows, n, _stream())
    if rc != 0:
        raise RuntimeError(f"synth_e4m3_rows failed: cuda error {rc}")


def normal_bf16_into(out, seed, tensor, seq, layer):
    """Fill a device uint16 tensor with synth.normal_bf16(seed, tensor, seq, layer, out.numel())."""
    assert out.is_cuda and out.is_contiguous() and out.dtype in (torch.bfloat16, torch.int16, torch.uint16)
    key = int(synth.stream_key(seed, tensor, seq, layer))
    rc = lib().synth_normal_bf16(out.data_ptr(), key, 0, out.numel(), _stream())
    if rc != 0:
        raise RuntimeError(f"synth_normal_bf16 failed: cuda error {rc}")
