"""ctypes loading of libhca.so and its C signatures (argument marshalling only)."""
import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libhca.so")

HCA_OK = 0
HCA_ERR_INVALID_ARG = 1
HCA_ERR_UNSUPPORTED = 2
HCA_ERR_CUDA = 3
HCA_ERR_TIMEOUT = 4
HCA_ERR_DEVICE_INPUT = 5
HCA_ERR_INTERNAL = 6

HCA_QK_NORM = 1
HCA_OUT_GATE = 2
HCA_PAGED = 4
HCA_WRITE_LSE = 8
HCA_OUT_F32 = 16
HCA_WINDOW_RING = 32

# Names of every entry point declared in include/hca.h.
EXPORTS = ("hca_compress", "hca_prefill", "hca_decode_workspace_size", "hca_decode", "hca_decode_vha",
           "hca_decode_noalloc",
           "hca_vha", "hca_append_state_size", "hca_append", "hca_status_string", "hca_get_device_error",
           "hca_debug_set_wait_limit", "hca_debug_set_drop_slab", "hca_debug_wait_probe", "hca_gate_logits",
           "hca_prefill_backward_workspace_size", "hca_prefill_backward", "hca_debug_set_backward_segment",
           "hca_debug_set_dsa_rows_limit",
           "hca_dsa_index", "hca_dsa_topk", "hca_dsa_attend")

_lib = None

_vp = ctypes.c_void_p
_i = ctypes.c_int
_f = ctypes.c_float
_u = ctypes.c_uint
_sz = ctypes.c_size_t


def load():
    """Load the in-tree libhca.so; raises if it has not been built (there is no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError("libhca.so is not built (run compressed_long_context_b200/build.py); "
                           "there is no CPU or PyTorch fallback")
    lib = ctypes.CDLL(LIB_PATH)
    lib.hca_status_string.restype = ctypes.c_char_p
    lib.hca_status_string.argtypes = [_i]
    lib.hca_get_device_error.restype = _i
    lib.hca_get_device_error.argtypes = [_vp]
    lib.hca_compress.restype = _i
    lib.hca_compress.argtypes = [_vp, _vp, _vp, _vp, _vp] + [_i] * 6 + [_vp]
    lib.hca_prefill.restype = _i
    lib.hca_prefill.argtypes = [_vp] * 7 + [_i] * 8 + [_f, _u, _vp]
    lib.hca_decode_workspace_size.restype = _sz
    lib.hca_decode_workspace_size.argtypes = [_i] * 4
    lib.hca_decode.restype = _i
    lib.hca_decode.argtypes = ([_vp, _vp, _vp, _vp, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _f, _vp, _vp, _vp, _sz]
                               + [_i] * 8 + [_f, _u, _vp])
    lib.hca_decode_vha.restype = _i
    lib.hca_decode_vha.argtypes = ([_vp, _vp, _vp, _vp, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _f, _vp, _vp, _vp, _i, _vp,
                                    _vp, _sz] + [_i] * 8 + [_f, _u, _vp])
    lib.hca_decode_noalloc.restype = _i
    lib.hca_decode_noalloc.argtypes = ([_vp, _vp, _vp, _vp, _i, _i, _i, _vp, _vp, _vp, _vp, _vp, _f, _vp, _vp]
                                       + [_i] * 8 + [_f, _u, _vp])
    lib.hca_vha.restype = _i
    lib.hca_vha.argtypes = [_vp, _vp, _vp, ctypes.c_longlong, _i, _i, _i, _u, _vp]
    lib.hca_append_state_size.restype = _sz
    lib.hca_append_state_size.argtypes = [_i] * 4
    lib.hca_append.restype = _i
    lib.hca_append.argtypes = [_vp] * 9 + [_i] * 3 + [_vp] + [_i] * 7 + [_u, _vp]
    lib.hca_gate_logits.restype = _i
    lib.hca_gate_logits.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, _vp]
    lib.hca_prefill_backward_workspace_size.restype = _sz
    lib.hca_prefill_backward_workspace_size.argtypes = [_i] * 7
    lib.hca_prefill_backward.restype = _i
    lib.hca_prefill_backward.argtypes = [_vp] * 13 + [_vp, _sz] + [_i] * 8 + [_f, _u, _vp]
    lib.hca_dsa_index.restype = _i
    lib.hca_dsa_index.argtypes = [_vp] * 5 + [_i] * 4 + [_vp]
    lib.hca_dsa_topk.restype = _i
    lib.hca_dsa_topk.argtypes = [_vp] * 3 + [_i] * 3 + [_vp]
    lib.hca_dsa_attend.restype = _i
    lib.hca_dsa_attend.argtypes = [_vp] * 6 + [_i] * 5 + [_f, _vp]
    lib.hca_debug_set_backward_segment.restype = _i
    lib.hca_debug_set_backward_segment.argtypes = [_i]
    lib.hca_debug_set_dsa_rows_limit.restype = _i
    lib.hca_debug_set_dsa_rows_limit.argtypes = [ctypes.c_longlong]
    lib.hca_debug_set_wait_limit.restype = _i
    lib.hca_debug_set_wait_limit.argtypes = [ctypes.c_ulonglong, _vp]
    lib.hca_debug_set_drop_slab.restype = _i
    lib.hca_debug_set_drop_slab.argtypes = [_i, _vp]
    lib.hca_debug_wait_probe.restype = _i
    lib.hca_debug_wait_probe.argtypes = [_vp]
    _lib = lib
    return lib
