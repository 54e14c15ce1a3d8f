"""ctypes loader for libcgtp.so: symbol signatures and status handling.

Argument marshalling only.  Importing this module does not touch the GPU;
``lib()`` loads the in-tree library and raises if it is missing, so the
product path can never run without the CUDA kernels.
"""
import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcgtp.so")

_p = ctypes.c_void_p
_i = ctypes.c_int
_f = ctypes.c_float
_sz = ctypes.c_size_t

# name -> (restype, argtypes), mirroring include/cgtp.h
SIGNATURES = {
    "cgtp_status_string": (ctypes.c_char_p, [_i]),
    "cgtp_last_cuda_error": (_i, []),
    "cgtp_plan_create": (_i, [_i, _i, _i, _i, _i, ctypes.POINTER(_p)]),
    "cgtp_plan_destroy": (_i, [_p]),
    "cgtp_supported": (_i, [_i, _i, _i, _i]),
    "cgtp_plan_set_checked": (_i, [_p, _i]),
    "cgtp_plan_check": (_i, [_p, ctypes.POINTER(_i)]),
    "cgtp_plan_info": (_i, [_p, ctypes.POINTER(_i), _p, ctypes.POINTER(_i)]),
    "cgtp_cg_block": (_i, [_i, _i, _i, _p]),
    "cgtp_graph_build": (_i, [_p, _i, _f, _f, _p, _i, _p, _p, _p, _p, _p, _p, _i, _p, _p]),
    "cgtp_csr_transpose": (_i, [_i, _i, _p, _p, _p, _p, _p, _p, _sz, _p]),
    "cgtp_graph_check": (_i, [_i, _i, _p, _p, _p, _p, _p]),
    "cgtp_spherical_harmonics": (_i, [_i, _i, _p, _p, _p, _p]),
    "cgtp_conv_forward": (_i, [_p, _i, _i, _p, _p, _p, _p, _p, _p, _p]),
    "cgtp_conv_backward_workspace_size": (_i, [_p, _i, ctypes.POINTER(_sz)]),
    "cgtp_conv_backward": (_i, [_p, _i, _i, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _sz, _p]),
    "cgtp_conv_double_backward_workspace_size": (_i, [_p, _i, ctypes.POINTER(_sz)]),
    "cgtp_conv_double_backward": (_i, [_p, _i, _i, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p,
                                       _p, _p, _p, _p, _p, _sz, _p]),
    "cgtp_uvw_forward_workspace_size": (_i, [_p, _i, _i, ctypes.POINTER(_sz)]),
    "cgtp_uvw_forward": (_i, [_p, _i, _i, _p, _p, _p, _p, _p, _p, _i, _p, _p, _sz, _p]),
    "cgtp_uvw_backward_workspace_size": (_i, [_p, _i, _i, _i, ctypes.POINTER(_sz)]),
    "cgtp_uvw_backward": (_i, [_p, _i, _i, _p, _p, _p, _p, _p, _p, _p, _p, _p, _i, _p, _p, _p, _p, _p, _p,
                               _sz, _p]),
    "cgtp_forces": (_i, [_i, _i, _p, _p, _p, _p, _p, _p]),
    "cgtp_gather_rows": (_i, [_i, _i, _p, _p, _p, _p]),
    "cgtp_scatter_add_rows": (_i, [_i, _i, _p, _p, _p, _p]),
    "cgtp_radial_forward": (_i, [_p, _i, _p, _f, _p, _p, _p, _p]),
    "cgtp_radial_backward": (_i, [_p, _i, _p, _f, _p, _p, _p, _p, _p]),
    "cgtp_tp_forward": (_i, [_p, _i, _p, _p, _p, _p, _p]),
    "cgtp_tp_backward_workspace_size": (_i, [_p, _i, ctypes.POINTER(_sz)]),
    "cgtp_tp_backward": (_i, [_p, _i, _p, _p, _p, _p, _p, _p, _p, _p, _sz, _p]),
    "cgtp_tp_backward_noalloc": (_i, [_p, _i, _p, _p, _p, _p, _p, _p, _p, _p]),
    "cgtp_cp_forward": (_i, [_p, _i, _i, _p, _p, _p, _p, _p, _p, _p]),
    "cgtp_cp_backward_workspace_size": (_i, [_p, _i, _i, ctypes.POINTER(_sz)]),
    "cgtp_cp_backward": (_i, [_p, _i, _i, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _sz, _p]),
}

STATUS = {0: "CGTP_OK", 1: "CGTP_ERR_INVALID_ARG", 2: "CGTP_ERR_UNSUPPORTED", 3: "CGTP_ERR_BAD_GRAPH",
          4: "CGTP_ERR_OOM", 5: "CGTP_ERR_CUDA", 6: "CGTP_ERR_TABLE", 7: "CGTP_ERR_WORKSPACE"}


class CGTPError(RuntimeError):
    def __init__(self, fn, status, cuda_error=0):
        self.status = status
        self.cuda_error = cuda_error
        msg = f"{fn} failed: {STATUS.get(status, status)}"
        if status == 5:
            msg += f" (cudaError {cuda_error})"
        super().__init__(msg)


_LIB = None


def lib():
    """The loaded library (raises OSError if libcgtp.so has not been built)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise OSError(f"libcgtp.so not found at {LIB_PATH}; run __graft_entry__.build() "
                          "or python -m equivariant_mlip_tensor_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = L
    return _LIB


def call(name, *args):
    """Call an entry point and raise CGTPError on a non-zero status."""
    st = getattr(lib(), name)(*args)
    if st != 0:
        raise CGTPError(name, st, lib().cgtp_last_cuda_error())
    return st
