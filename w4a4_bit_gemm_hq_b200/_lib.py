"""Thin Python binding of the libhq C ABI (``include/hq.h``).

Argument marshalling only: every step of the layer runs in the CUDA kernels of
``libhq.so``.  Device tensors are PyTorch CUDA tensors (PyTorch provides the
memory and the stream); calls are enqueued on the current CUDA stream.  There
is no CPU fallback: if the library cannot be loaded, importing this module
raises.
"""
import ctypes as ct
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhq.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        "libhq.so is missing: build it with `python w4a4_bit_gemm_hq_b200/build_lib.py` "
        "(or __graft_entry__.build()); there is no CPU fallback")

lib = ct.CDLL(LIB_PATH)

HQ_OK, HQ_ERR_ARG, HQ_ERR_ALIGN, HQ_ERR_UNSUPPORTED, HQ_ERR_CUDA, HQ_ERR_TIMEOUT = range(6)
HQ_F16, HQ_BF16, HQ_F32 = 0, 1, 2

_P = ct.c_void_p
_I64 = ct.c_int64
_I32 = ct.c_int32
_ST = ct.c_int  # hq_status

# name -> (argtypes, restype); the same list is checked against the header by the tests
SIGNATURES = {
    "hq_status_str": ([_ST], ct.c_char_p),
    "hq_device_sm_count": ([], ct.c_int),
    "hq_packed_weight_bytes": ([_I64, _I64], ct.c_size_t),
    "hq_rotate_quant": ([_P, ct.c_int, _I64, _I64, _I64, _I32, _P, _P, _P, _P], _ST),
    "hq_rotate": ([_P, ct.c_int, _I64, _I64, _I32, _P, _P, _P], _ST),
    "hq_channel_sqnorm": ([_P, ct.c_int, _I64, _I64, _I32, _P, _P, _P], _ST),
    "hq_select_salient": ([_P, _I64, _I32, _P], _ST),
    "w4_pack": ([_P, ct.c_int, _I64, _I64, _I32, _P, _P, _P, _P], _ST),
    "serq_prepare": ([_P, _I64, _I64, _P, _P, _P, _I32, _P, _I32, _P, _P, _P], _ST),
    "hq_linear_workspace_size": ([_I64, _I64, _I64, _I32], ct.c_size_t),
    "w4a4_linear": ([_P, _P, _I64, _I64, _P, _P, _P, _I64, _I32, _P, _P, _P, _I32, _P, ct.c_int, _P,
                     ct.c_size_t, _P], _ST),
    "w4a4_linear_noalloc": ([_P, _P, _I64, _I64, _P, _P, _P, _I64, _I32, _P, _P, _P, _I32, _P, ct.c_int, _P], _ST),
    "hq_debug_accum": ([_P, _I64, _I64, _P, _P, _I64, _I32, _P, _P, _I32, _P, _P, _I32, _P, ct.c_size_t, _P],
                       _ST),
    "hq_rotate_quant8": ([_P, ct.c_int, _I64, _I64, _I64, _I32, _P, _P, _P, _P], _ST),
    "hq_rotate_quant_asym": ([_P, ct.c_int, _I64, _I64, _I64, _I32, _P, _P, _P, _P, _P], _ST),
    "w4a4_linear_asym": ([_P, _P, _P, _I64, _I64, _P, _P, _P, _I64, _I32, _P, _P, _P, _I32, _P, ct.c_int, _P], _ST),
    "hq_debug_accum_asym": ([_P, _P, _I64, _I64, _P, _P, _I64, _I32, _P, _P], _ST),
    "w4a8_linear": ([_P, _P, _I64, _I64, _P, _P, _P, _I64, _I32, _P, _P, _P, _I32, _P, ct.c_int, _P,
                     ct.c_size_t, _P], _ST),
    "hq_debug_accum8": ([_P, _I64, _I64, _P, _P, _I64, _I32, _P, _P, _I32, _P, _P, _I32, _P, ct.c_size_t, _P],
                        _ST),
    "hq_calib_extreme_tokens": ([_P, ct.c_int, _I64, _I64, _I64, _I64, _P, _P, _P], _ST),
    "hq_calib_pca_max_elems": ([], ct.c_size_t),
    "hq_calib_top1_pca": ([_P, _I64, _I64, _I32, _P, _P, _P], _ST),
    "hq_calib_householder": ([_P, ct.c_int, _I64, _I64, _I64, _P, _P, _P], _ST),
    "hq_calib_channel_absmax": ([_P, ct.c_int, _I64, _I64, _I64, _P, _P], _ST),
    "hq_calib_sorted_perm": ([_P, _I64, _P, _P], _ST),
    "hq_calib_flatten_scales": ([_P, _P, _I64, ct.c_float, _P, _P], _ST),
    "hq_permute_channels": ([_P, ct.c_int, _I64, _I64, _I64, _P, _P, _I32, _P, _P], _ST),
    "hq_quant_mxfp4": ([_P, ct.c_int, _I64, _I64, _I64, _P, _P, _P], _ST),
    "hq_mxfp4_linear": ([_P, _P, _I64, _I64, _P, _P, _I64, _P, _I32, _P], _ST),
    "hq_last_device_status": ([_P], _ST),
    "hq_debug_wait_probe": ([ct.c_uint64, _P], _ST),
}

for _name, (_args, _res) in SIGNATURES.items():
    _f = getattr(lib, _name)
    _f.argtypes = _args
    _f.restype = _res


class HQError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__("%s: %s" % (where, lib.hq_status_str(status).decode()))


def check(status, where):
    if status != HQ_OK:
        raise HQError(status, where)


def dtype_code(dt):
    if dt == torch.float16:
        return HQ_F16
    if dt == torch.bfloat16:
        return HQ_BF16
    if dt == torch.float32:
        return HQ_F32
    raise TypeError("unsupported dtype %s" % dt)


def ptr(t):
    return None if t is None else ct.c_void_p(t.data_ptr())


def stream_handle(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ct.c_void_p(s.cuda_stream)
