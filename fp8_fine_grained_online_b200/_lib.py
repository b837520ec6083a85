"""ctypes binding of the C ABI in ``include/fp8fg.h`` (libfp8fg.so).

Argument marshalling only: every step of the computation runs in the CUDA
library.  Importing this module raises if the library has not been built;
there is no fallback implementation.
"""
import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libfp8fg.so")

STATUS_NAMES = {
    0: "FP8_OK", 1: "FP8_ERR_NULL", 2: "FP8_ERR_SHAPE", 3: "FP8_ERR_ALIGN",
    4: "FP8_ERR_LAYOUT", 5: "FP8_ERR_DTYPE", 6: "FP8_ERR_DEVICE", 7: "FP8_ERR_CUDA",
    8: "FP8_ERR_UNIMPLEMENTED", 9: "FP8_ERR_DEVICE_TIMEOUT",
}
FP8_OK = 0
FP8_IN_BF16, FP8_IN_FP32 = 0, 1
FP8_OUT_FP32, FP8_OUT_BF16 = 0, 1

# Entry points and their C signatures (restype, argtypes).
_i64, _int, _vp = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
SIGNATURES = {
    "fp8_quantize_act_1x128": (_int, [_vp, _int, _i64, _i64, _i64, _vp, _i64, _vp, _i64, _i64,
                                      _vp]),
    "fp8_quantize_act_1x128_gather": (_int, [_vp, _int, _i64, _i64, _i64, _vp, _i64, _vp, _i64,
                                             _vp, _i64, _i64, _vp]),
    "fp8_quantize_act_1x128_scatter": (_int, [_vp, _int, _i64, _i64, _i64, _vp, _i64, _vp,
                                              _i64, _i64, _vp, _i64, _i64, _vp]),
    "fp8_quantize_weight_128x128": (_int, [_vp, _int, _i64, _i64, _i64, _vp, _int, _i64, _vp,
                                           _i64, _i64, _vp]),
    "fp8_blockscaled_gemm": (_int, [_vp, _i64, _vp, _i64, _i64, _vp, _i64, _int, _vp, _i64, _i64,
                                    _vp, _int, _i64, _i64, _i64, _i64, _vp]),
    "fp8_blockscaled_gemm_quant": (_int, [_vp, _i64, _vp, _i64, _i64, _vp, _i64, _vp, _i64, _i64,
                                          _vp, _i64, _vp, _i64, _i64, _vp, _i64, _i64, _i64,
                                          _i64, _vp]),
    "fp8_quantize_act_128x1": (_int, [_vp, _int, _i64, _i64, _i64, _vp, _i64, _vp, _i64, _i64,
                                      _vp]),
    "fp8_blockscaled_gemm_colscale": (_int, [_vp, _i64, _vp, _i64, _i64, _vp, _i64, _vp, _i64,
                                             _vp, _int, _i64, _i64, _i64, _i64, _vp]),
    "fp8_grouped_gemm": (_int, [_vp, _i64, _vp, _i64, _i64, _vp, _i64, _vp, _i64, _i64, _i64,
                                _vp, _int, _i64, _vp, _int, _i64, _i64, _i64, _vp]),
    "fp8_dequantize": (_int, [_vp, _i64, _i64, _i64, _vp, _i64, _i64, _int, _vp, _int, _i64,
                              _vp]),
    "fp8_status_string": (ctypes.c_char_p, [_int]),
    "fp8_get_device_error": (_int, [_vp, ctypes.POINTER(_int)]),
    "fp8_set_wait_limit": (_int, [_i64]),
}


class Fp8Error(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        name = STATUS_NAMES.get(status, str(status))
        super().__init__("%s returned %s" % (where, name))


def load(path=LIB_PATH):
    if not os.path.exists(path):
        raise ImportError(
            "the CUDA library %s is not built (run __graft_entry__.build() or "
            "python fp8_fine_grained_online_b200/build.py); there is no fallback" % path)
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = load()


def check(status, where):
    if status != FP8_OK:
        raise Fp8Error(status, where)
