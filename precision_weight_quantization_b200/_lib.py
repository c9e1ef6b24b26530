"""ctypes loader for libpwq.so (the C ABI in include/pwq.h).

The library is built in-tree by ``precision_weight_quantization_b200/build.py``
(``__graft_entry__.build()`` runs it).  There is no fallback: if the shared
library is missing or cannot be loaded, importing the package raises.
"""
import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libpwq.so")

# pwq_status values (include/pwq.h)
PWQ_OK = 0
PWQ_ERR_NULL = 1
PWQ_ERR_ALIGN = 2
PWQ_ERR_SHAPE = 3
PWQ_ERR_STRIDE = 4
PWQ_ERR_OVERLAP = 5
PWQ_ERR_WORKSPACE = 6
PWQ_ERR_CUDA = 7
PWQ_ERR_ARG = 8
PWQ_MAX_SIBLINGS = 8


class PwqTensor(ctypes.Structure):
    """struct pwq_tensor"""
    _fields_ = [("ptr", ctypes.c_void_p), ("batch", ctypes.c_int64), ("rows", ctypes.c_int64),
                ("cols", ctypes.c_int64), ("batch_stride", ctypes.c_int64),
                ("row_stride", ctypes.c_int64)]


class PwqError(RuntimeError):
    def __init__(self, status: int, func: str, detail: str):
        self.status = status
        super().__init__("%s failed: %s (%s)" % (func, status_string(status), detail))


_P = ctypes.c_void_p
_T = ctypes.POINTER(PwqTensor)
_S = ctypes.c_int
_PP = ctypes.POINTER(ctypes.c_void_p)
_IP = ctypes.POINTER(ctypes.c_int)
_SIG = {
    "fp8_block_quant": (_S, [_T, _T, _P, _P]),
    "fp8_block_dequant": (_S, [_T, _P, _T, _P]),
    "mxfp8_quant": (_S, [_T, _T, _P, _P]),
    "mxfp8_dequant": (_S, [_T, _P, _T, _P]),
    "nvfp4_workspace_size": (ctypes.c_size_t, [ctypes.c_int, _T]),
    "nvfp4_group_amax": (_S, [_T, ctypes.c_int, _P, _P]),
    "nvfp4_quant": (_S, [_T, ctypes.c_int, _T, ctypes.POINTER(ctypes.c_void_p), _P, _P, _P,
                         ctypes.c_size_t, _P]),
    "nvfp4_dequant": (_S, [_T, _P, _P, _T, _P]),
    "nvfp4_fake_quant": (_S, [_T, _T, ctypes.c_int, _P, _P, _P, ctypes.c_size_t, _P]),
    "nvfp4_4over6_workspace_size": (ctypes.c_size_t, [ctypes.c_int, _T]),
    "nvfp4_4over6_quant": (_S, [_T, ctypes.c_int, _T, ctypes.POINTER(ctypes.c_void_p), _P, _P, ctypes.c_int, _P,
                                ctypes.c_size_t, _P]),
    "nvfp4_4over6_fake_quant": (_S, [_T, _T, ctypes.c_int, _P, _P, ctypes.c_int, _P, ctypes.c_size_t, _P]),
    "nvfp4_4over6_workspace_size_grouped": (ctypes.c_size_t, [ctypes.c_int, _IP, _T]),
    "nvfp4_4over6_quant_grouped": (_S, [ctypes.c_int, _IP, _T, _T, _PP, _PP, ctypes.c_int, _P, ctypes.c_size_t,
                                        _P]),
    "nvfp4_4over6_fake_quant_grouped": (_S, [ctypes.c_int, _IP, _T, _T, _PP, ctypes.c_int, _P, ctypes.c_size_t,
                                             _P]),
    "fp8_block_quant_grouped": (_S, [ctypes.c_int, _T, _T, _PP, _P]),
    "fp8_block_dequant_grouped": (_S, [ctypes.c_int, _T, _PP, _T, _P]),
    "mxfp8_quant_grouped": (_S, [ctypes.c_int, _T, _T, _PP, _P]),
    "mxfp8_dequant_grouped": (_S, [ctypes.c_int, _T, _PP, _T, _P]),
    "nvfp4_dequant_grouped": (_S, [ctypes.c_int, _T, _PP, _PP, _T, _P]),
    "nvfp4_workspace_size_grouped": (ctypes.c_size_t, [ctypes.c_int, _IP, _T]),
    "nvfp4_quant_grouped": (_S, [ctypes.c_int, _IP, _T, _T, _PP, _PP, _P, ctypes.c_size_t, _P]),
    "nvfp4_fake_quant_grouped": (_S, [ctypes.c_int, _IP, _T, _T, _PP, _P, ctypes.c_size_t, _P]),
    "fp8_block_requant": (_S, [_T, _P, _T, _P, _P]),
    "fp8_block_requant_mxfp8": (_S, [_T, _P, _T, _P, _P]),
    "fp8_block_requant_grouped": (_S, [ctypes.c_int, _T, _PP, _T, _PP, _P]),
    "fp8_block_requant_mxfp8_grouped": (_S, [ctypes.c_int, _T, _PP, _T, _PP, _P]),
    "fp8_block_requant_nvfp4_workspace_size": (ctypes.c_size_t, [ctypes.c_int, _T]),
    "fp8_block_requant_nvfp4": (_S, [_T, _PP, ctypes.c_int, _T, _PP, _P, _P, _P, ctypes.c_size_t, _P]),
    "fp8_block_requant_nvfp4_workspace_size_grouped": (ctypes.c_size_t, [ctypes.c_int, _IP, _T]),
    "fp8_block_requant_nvfp4_grouped": (_S, [ctypes.c_int, _IP, _T, _PP, _T, _PP, _PP, _P, ctypes.c_size_t, _P]),
    "nvfp4_observe_workspace_size": (ctypes.c_size_t, []),
    "nvfp4_activation_observe": (_S, [_T, ctypes.c_int, ctypes.c_float, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "pwq_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "pwq_last_error_detail": (ctypes.c_char_p, []),
    "pwq_build_info": (ctypes.c_char_p, []),
    "pwq_device_error": (_S, [ctypes.POINTER(ctypes.c_uint32)]),
    "pwq_selftest_division": (_S, [ctypes.c_int, _P, _P]),
    "pwq_selftest_codecs": (_S, [ctypes.c_uint32, ctypes.c_uint32, _P, _P, _P, _P]),
    "pwq_selftest_flow_timeout_workspace_size": (ctypes.c_size_t, [_T]),
    "pwq_selftest_flow_timeout": (_S, [_T, _T, ctypes.c_uint64, _P, ctypes.c_size_t, _P]),
    "nvfp4_fake_quant_noalloc": (_S, [_T, _T, ctypes.c_int, _P, _P, _P]),
    "pwq_mma_scale_bytes": (ctypes.c_size_t, [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64]),
    "pwq_scales_to_mma": (_S, [_P, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, _P, _P]),
    "pwq_scales_from_mma": (_S, [_P, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, _P, _P]),
    "mxfp8_quant_grouped_mma": (_S, [ctypes.c_int, _T, _T, _PP, _P]),
    "nvfp4_quant_grouped_mma": (_S, [ctypes.c_int, _IP, _T, _T, _PP, _PP, _P, ctypes.c_size_t, _P]),
}


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError("libpwq.so is not built (%s); run `python "
                          "precision_weight_quantization_b200/build.py`" % LIB_PATH)
    L = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in _SIG.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    return L


lib = _load()


def status_string(status: int) -> str:
    return lib.pwq_status_string(status).decode()


def check(status: int, func: str):
    if status != PWQ_OK:
        raise PwqError(status, func, lib.pwq_last_error_detail().decode())
