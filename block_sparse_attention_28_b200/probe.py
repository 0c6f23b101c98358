"""Python binding of libsta_probe (include/sta_probe.h): measurement probes
of the TMA load stream and of the tcgen05 MMA rate that the attention kernel
of libsta is read against. Argument marshalling only; not part of the method.
"""
import ctypes
import os

import torch

from . import Grid, StaError, _ptr, _stream  # noqa: F401

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsta_probe.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python block_sparse_attention_28_b200/build.py`")

_lib = ctypes.CDLL(LIB_PATH)
_vp, _i32, _sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
_lib.sta_probe_tma_stream.argtypes = [_vp, _sz, _i32, _i32, _i32, _vp]
_lib.sta_probe_tma_stream.restype = ctypes.c_int
_lib.sta_probe_mma_rate.argtypes = [_i32, _i32, _i32, _vp, _vp]
_lib.sta_probe_mma_rate.restype = ctypes.c_int
_lib.sta_probe_get_device_error.argtypes = [_vp]
_lib.sta_probe_get_device_error.restype = ctypes.c_int


def _check(status, what):
    if status != 0:
        raise StaError(status, what)


def sta_probe_tma_stream(buf, ctas_per_sm, slots, iters, stream=None):
    _check(_lib.sta_probe_tma_stream(_ptr(buf), buf.numel() * buf.element_size(), int(ctas_per_sm),
                                     int(slots), int(iters), _stream(stream)),
           "sta_probe_tma_stream")


def sta_probe_mma_rate(n, a_in_tmem, iters, stream=None):
    """SM cycles of `iters` back-to-back M=128, K=16 bf16 MMAs of width n on
    every SM (one CTA each); returns a CPU int64 tensor, one entry per SM."""
    dev = torch.device("cuda", torch.cuda.current_device())
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    cycles = torch.full((sms,), -2, dtype=torch.int64, device=dev)
    _check(_lib.sta_probe_mma_rate(int(n), 1 if a_in_tmem else 0, int(iters), _ptr(cycles), _stream(stream)),
           "sta_probe_mma_rate")
    return cycles.cpu()


def sta_probe_get_device_error(stream=None):
    return int(_lib.sta_probe_get_device_error(_stream(stream)))
