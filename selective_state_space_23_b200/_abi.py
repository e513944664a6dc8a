"""ctypes loader for libssm_b200.so (the C ABI in include/ssm_scan.h).

Loading fails loudly: there is no fallback implementation of any entry point.
"""
import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libssm_b200.so")

SSM_F32, SSM_BF16 = 0, 1
SSM_OK, SSM_EINVAL, SSM_EUNSUPPORTED, SSM_ECUDA, SSM_EWORKSPACE = 0, 1, 2, 3, 4
CKPT_STEPS = 16
MAX_DSTATE = 16
NOALLOC_SCRATCH_BYTES = 8 << 20
SSM_SCALAR_A, SSM_REVERSE, SSM_ZOH, SSM_CHANNELS_LAST = 1, 2, 4, 8

_vp = ctypes.c_void_p
_i = ctypes.c_int
_sz = ctypes.c_size_t
_ll3 = ctypes.c_longlong * 3
_ll4 = ctypes.c_longlong * 4
_ll2 = ctypes.c_longlong * 2


class Strides(ctypes.Structure):
    """ssm_strides: element strides of every io tensor of a strided scan call."""
    _fields_ = [(n, _ll3) for n in ("u", "delta", "z", "out", "dout", "du", "ddelta", "dz")] + \
               [(n, _ll4) for n in ("B", "C", "dB", "dC")]


class DecodeStrides(ctypes.Structure):
    """ssm_decode_strides: element strides of the tensors of a strided decode step."""
    _fields_ = [("state", _ll3)] + [(n, _ll2) for n in ("x", "dt", "z", "out")] + \
               [(n, _ll3) for n in ("B", "C")]

# name -> (restype, argtypes)
SIGNATURES = {
    "ssm_status_string": (ctypes.c_char_p, [_i]),
    "ssm_last_error": (ctypes.c_char_p, []),
    "ssm_version": (ctypes.c_char_p, []),
    "ssm_scan_fwd_workspace_size": (_sz, [_i, _i, _i, _i, _i]),
    "ssm_scan_fwd": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _vp, _vp, _vp, _vp, _vp, _sz,
                          _i, _i, _i, _i, _i, _vp]),
    "ssm_scan_bwd_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i]),
    "ssm_scan_bwd": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _vp, _vp, _vp, _vp,
                          _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz,
                          _i, _i, _i, _i, _i, _vp]),
    "ssm_scan_fwd_scalar_a_workspace_size": (_sz, [_i, _i, _i, _i, _i]),
    "ssm_scan_fwd_scalar_a": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _vp, _vp, _vp, _vp,
                                   _vp, _sz, _i, _i, _i, _i, _i, _vp]),
    "ssm_scan_bwd_scalar_a_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i]),
    "ssm_scan_bwd_scalar_a": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _vp, _vp, _vp, _vp,
                                   _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz,
                                   _i, _i, _i, _i, _i, _vp]),
    "ssm_scan_fwd_ex_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i, _i]),
    "ssm_scan_fwd_ex": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _vp, _vp, _vp, _vp,
                             _vp, _sz, _i, _i, _i, _i, _i, _i, _i, _vp]),
    "ssm_scan_bwd_ex_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i, _i, _i]),
    "ssm_scan_bwd_ex": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _vp, _vp, _vp, _vp,
                             _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz,
                             _i, _i, _i, _i, _i, _i, _i, _vp]),
    "ssm_scan_fwd_host_workspace_size": (_sz, [_i, _i, _i, _i, _i]),
    "ssm_scan_fwd_host": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _vp, _vp, _vp, _vp, _sz,
                               _i, _i, _i, _i, _i, _vp]),
    "ssm_scan_fwd_noalloc": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _vp, _vp, _vp, _vp,
                                  _i, _i, _i, _i, _i, _vp]),
    "ssm_state_update": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _vp,
                              _i, _i, _i, _i, _vp]),
    "ssm_state_update_ex": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _vp,
                                 _i, _i, _i, _i, _i, _i, _vp]),
    "ssm_wait_timeouts": (_i, [ctypes.POINTER(ctypes.c_uint)]),
    "ssm_scan_fwd_strided_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i, _i]),
    "ssm_scan_fwd_strided": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _vp, _vp, _vp, _vp,
                                  _vp, _sz, _i, _i, _i, _i, _i, _i, _i, ctypes.POINTER(Strides),
                                  _vp]),
    "ssm_scan_bwd_strided_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i, _i, _i]),
    "ssm_scan_bwd_strided": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _vp, _vp, _vp, _vp,
                                  _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz,
                                  _i, _i, _i, _i, _i, _i, _i, ctypes.POINTER(Strides), _vp]),
    "ssm_scan_fwd_summary_workspace_size": (_sz, [_i, _i, _i, _i, _i, _i, _i]),
    "ssm_scan_fwd_summary": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _vp, _vp, _vp, _sz,
                                  _i, _i, _i, _i, _i, _i, _i, _vp]),
    "ssm_scan_chain": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp]),
    "ssm_state_update_strided_workspace_size": (_sz, [_i, _i, _i, _i, _i]),
    "ssm_state_update_strided": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _vp, _vp,
                                      _sz, _i, _i, _i, _i, _i, _i,
                                      ctypes.POINTER(DecodeStrides), _vp]),
}

_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library (raises RuntimeError if it is missing or incomplete)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m selective_state_space_23_b200.build` "
                "(nvcc, sm_100a). There is no CPU or fallback implementation.")
        l = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(l, name)  # AttributeError if the symbol is not exported
            f.restype = res
            f.argtypes = args
        _lib = l
    return _lib


def last_error() -> str:
    return lib().ssm_last_error().decode()


def wait_timeouts() -> int:
    """Bounded waits that ran out in the library's kernels on the current device (0 = none)."""
    n = ctypes.c_uint(0)
    check(lib().ssm_wait_timeouts(ctypes.byref(n)), "ssm_wait_timeouts")
    return int(n.value)


def check(rc: int, what: str) -> None:
    if rc != SSM_OK:
        msg = lib().ssm_status_string(rc).decode()
        raise RuntimeError(f"{what} failed: {msg} ({rc}): {last_error()}")
