"""ctypes view of libgqa_attn.so (the C ABI in include/gqa_attn.h).

Argument marshalling only: every entry point forwards plain pointers and sizes
to the library.  Loading fails loudly if the library has not been built.
"""
from __future__ import annotations

import ctypes
import pathlib

LIB_PATH = pathlib.Path(__file__).resolve().parent / "libgqa_attn.so"

# every symbol include/gqa_attn.h declares
EXPORTS = (
    "gqa_attn_fwd",
    "gqa_attn_fwd_f32",
    "gqa_attn_fwd_host",
    "gqa_attn_fwd_host_varlen",
    "gqa_attn_workspace_bytes",
    "gqa_attn_set_workspace",
    "gqa_attn_plan",
    "gqa_attn_get_device_error",
    "gqa_attn_strerror",
    "gqa_attn_decode_noalloc",
    "gqa_attn_fwd_blocksparse",
    "gqa_attn_bwd_workspace_bytes",
    "gqa_attn_bwd",
    "gqa_attn_fwd_blocksparse_varlen",
    "gqa_attn_fwd_fp8",
    "gqa_attn_sparse_varlen_schedule",
    "gqa_attn_decode_kvcache",
    "gqa_attn_decode_paged",
    "gqa_attn_decode_fp8",
    "gqa_attn_selftest_timeout",
    "gqa_attn_fwd_window",
)

STATUS = {
    0: "GQA_OK",
    -1: "GQA_ERR_NULL",
    -2: "GQA_ERR_SHAPE",
    -3: "GQA_ERR_HEADDIM",
    -4: "GQA_ERR_ALIGN",
    -5: "GQA_ERR_SPLITS",
    -6: "GQA_ERR_WORKSPACE",
    -7: "GQA_ERR_SCALE",
    -8: "GQA_ERR_CUDA",
    -9: "GQA_ERR_UNSUPPORTED",
}
STATUS_CODE = {v: k for k, v in STATUS.items()}

_lib = None


def load() -> ctypes.CDLL:
    global _lib
    if _lib is not None:
        return _lib
    if not LIB_PATH.exists():
        raise ImportError(f"{LIB_PATH.name} is not built; run "
                          "`python -m exact_attention_gqa_b200.build`")
    lib = ctypes.CDLL(str(LIB_PATH))
    P, I, F, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    fwd_args = [P, P, P, P, P, I, I, I, I, I, I, F, I, I, I, P, P]
    for name in ("gqa_attn_fwd", "gqa_attn_fwd_f32"):
        fn = getattr(lib, name)
        fn.argtypes = fwd_args
        fn.restype = I
    lib.gqa_attn_fwd_host.argtypes = [P, P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, F, I, I, I,
                                      I, P]
    lib.gqa_attn_fwd_host.restype = I
    lib.gqa_attn_fwd_host_varlen.argtypes = [P, P, P, P, P, P, P, P, P, P, P, P, I, I, I, I, I,
                                             I, F, I, I, I, P]
    lib.gqa_attn_fwd_host_varlen.restype = I
    lib.gqa_attn_workspace_bytes.argtypes = [I, I, I, I, I]
    lib.gqa_attn_workspace_bytes.restype = Z
    lib.gqa_attn_set_workspace.argtypes = [P, Z]
    lib.gqa_attn_set_workspace.restype = I
    IP = ctypes.POINTER(ctypes.c_int)
    lib.gqa_attn_plan.argtypes = [I, I, I, I, I, I, F, I, I, I, I, IP, IP, IP]
    lib.gqa_attn_plan.restype = I
    lib.gqa_attn_get_device_error.argtypes = [IP, P]
    lib.gqa_attn_get_device_error.restype = I
    lib.gqa_attn_bwd_workspace_bytes.argtypes = [I, I, I]
    lib.gqa_attn_bwd_workspace_bytes.restype = Z
    lib.gqa_attn_bwd.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, F, I, P]
    lib.gqa_attn_bwd.restype = I
    lib.gqa_attn_fwd_blocksparse.argtypes = [P, P, P, P, P, I, I, I, I, I, I, F, I, P, P, P]
    lib.gqa_attn_fwd_blocksparse.restype = I
    lib.gqa_attn_fwd_blocksparse_varlen.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, F,
                                                    I, P, P, P, I, I, P]
    lib.gqa_attn_fwd_blocksparse_varlen.restype = I
    lib.gqa_attn_sparse_varlen_schedule.argtypes = [P, P, I, I, I, I, I, P, P, I, IP, IP]
    lib.gqa_attn_sparse_varlen_schedule.restype = I
    lib.gqa_attn_fwd_fp8.argtypes = [P, P, P, P, P, I, I, I, I, I, I, F, F, F, F, I, P, P]
    lib.gqa_attn_fwd_fp8.restype = I
    lib.gqa_attn_fwd_window.argtypes = [P, P, P, P, P, I, I, I, I, I, I, F, I, I, P, P]
    lib.gqa_attn_fwd_window.restype = I
    lib.gqa_attn_decode_kvcache.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, F, I, I, I, P]
    lib.gqa_attn_decode_kvcache.restype = I
    lib.gqa_attn_decode_paged.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, F, I, I,
                                          I, P]
    lib.gqa_attn_decode_paged.restype = I
    lib.gqa_attn_decode_fp8.argtypes = [P, P, P, F, F, P, P, P, P, I, I, I, I, I, I, I, I, I, F,
                                        I, I, I, P]
    lib.gqa_attn_decode_fp8.restype = I
    lib.gqa_attn_selftest_timeout.argtypes = [I, P]
    lib.gqa_attn_selftest_timeout.restype = I
    lib.gqa_attn_strerror.argtypes = [I]
    lib.gqa_attn_strerror.restype = ctypes.c_char_p
    _lib = lib
    return lib


def strerror(code: int) -> str:
    return load().gqa_attn_strerror(int(code)).decode()


class GqaError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} returned {STATUS.get(code, code)}: {strerror(code)}")
        self.code = code
