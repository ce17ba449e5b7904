"""ctypes loader for libdsa_b200.so (the C ABI declared in include/dsa.h).

There is no fallback: if the shared library is missing or fails to load, importing the
binding raises, and every call goes to the CUDA kernels of that library.
"""
import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libdsa_b200.so")

c_int, c_i64, c_f32, c_size, c_vp = ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t, ctypes.c_void_p

# name -> (restype, argtypes), in the order of include/dsa.h
SIGNATURES = {
    "dsa_status_string": (ctypes.c_char_p, [c_int]),
    "dsa_version": (c_int, []),
    "dsa_last_cuda_error": (c_int, [ctypes.POINTER(ctypes.c_char_p)]),
    "dsa_get_device_status": (c_int, [ctypes.POINTER(c_int), ctypes.POINTER(c_int)]),
    "dsa_selftest_bounded_wait": (c_int, [ctypes.c_uint64, c_vp]),
    "dsa_index": (c_int, [c_vp, c_vp, c_vp, c_vp, c_vp, c_int, c_i64, c_i64, c_int, c_int, c_int, c_int,
                          c_i64, c_i64, c_vp, c_i64, c_vp]),
    "dsa_topk_workspace_size": (c_size, [c_i64, c_i64, c_int]),
    "dsa_topk": (c_int, [c_vp, c_i64, c_vp, c_vp, c_int, c_i64, c_i64, c_int, c_vp, c_vp, c_size, c_vp]),
    "dsa_index_topk_workspace_size": (c_size, [c_i64, c_int]),
    "dsa_index_topk": (c_int, [c_vp, c_vp, c_vp, c_vp, c_vp, c_int, c_i64, c_i64, c_int, c_int, c_int, c_int, c_int,
                               c_i64, c_i64, c_i64, c_int, c_vp, c_vp, c_size, c_vp]),
    "dsa_sparse_attn_prefill": (c_int, [c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_int, c_i64, c_int, c_int, c_int,
                                        c_int, c_f32, c_vp, c_vp, c_vp]),
    "dsa_sparse_attn_prefill_tc": (c_int, [c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_int, c_i64, c_int, c_int, c_int,
                                           c_int, c_f32, c_vp, c_vp, c_vp]),
    "dsa_sparse_attn_prefill_reuse_workspace_size": (c_size, [c_i64, c_int, c_int, c_int]),
    "dsa_sparse_attn_prefill_reuse": (c_int, [c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_int, c_i64, c_i64, c_int, c_int,
                                              c_int, c_int, c_int, c_f32, c_vp, c_vp, c_vp, c_vp, c_size, c_vp]),
    "dsa_sparse_attn_decode_workspace_size": (c_size, [c_int, c_int, c_int, c_int]),
    "dsa_sparse_attn_decode": (c_int, [c_vp, c_vp, c_vp, c_vp, c_vp, c_int, c_int, c_int, c_int, c_int, c_f32,
                                       c_vp, c_vp, c_vp, c_size, c_vp]),
    "dsa_sparse_attn_decode_noalloc": (c_int, [c_vp, c_vp, c_vp, c_vp, c_vp, c_int, c_int, c_int, c_int, c_int,
                                               c_f32, c_vp, c_vp, c_vp]),
    "dsa_prefill_workspace_size": (c_size, [c_i64, c_int]),
    "dsa_prefill": (c_int, [c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_int, c_i64, c_i64, c_int, c_int,
                            c_int, c_int, c_int, c_int, c_int, c_int, c_f32, c_i64, c_vp, c_vp, c_vp, c_vp,
                            c_size, c_vp]),
    "dsa_prefill_host_workspace_size": (c_size, [c_int, c_i64, c_i64, c_int, c_int, c_int, c_int, c_int, c_int, c_int,
                                                 c_i64]),
    "dsa_prefill_host": (c_int, [c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_int, c_i64, c_i64, c_int, c_int,
                                 c_int, c_int, c_int, c_int, c_int, c_int, c_f32, c_i64, c_vp, c_vp, c_size, c_vp]),
    "dsa_decode_workspace_size": (c_size, [c_int, c_int, c_int, c_int, c_int]),
    "dsa_decode": (c_int, [c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_int, c_i64, c_int, c_int, c_int, c_int,
                           c_int, c_int, c_int, c_f32, c_vp, c_vp, c_vp, c_vp, c_size, c_vp]),
    "dsa_sparse_attn_bwd_workspace_size": (c_size, [c_i64, c_i64, c_int, c_int, c_int, c_int]),
    "dsa_sparse_attn_prefill_bwd": (c_int, [c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_int, c_i64,
                                            c_i64, c_int, c_int, c_int, c_int, c_int, c_f32, c_vp, c_vp, c_vp,
                                            c_vp, c_size, c_vp]),
    "dsa_indexer_kl_loss_workspace_size": (c_size, [c_i64, c_i64, c_int, c_int, c_int, c_int, c_i64, c_int]),
    "dsa_indexer_kl_loss": (c_int, [c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_int, c_i64, c_i64, c_int, c_int,
                                    c_int, c_int, c_int, c_int, c_int, c_f32, c_i64, c_vp, c_vp, c_vp, c_vp, c_vp,
                                    c_vp, c_size, c_vp]),
    "dsa_indexer_kl_loss_sparse_workspace_size": (c_size, [c_i64, c_i64, c_int, c_int, c_int, c_int, c_i64, c_int]),
    "dsa_indexer_kl_loss_sparse": (c_int, [c_vp, c_vp, c_vp, c_vp, c_vp, c_vp, c_int, c_vp, c_vp, c_int, c_i64, c_i64,
                                           c_int, c_int, c_int, c_int, c_int, c_int, c_int, c_f32, c_i64, c_vp, c_vp,
                                           c_vp, c_vp, c_vp, c_vp, c_size, c_vp]),
}

_lib = None


def load() -> ctypes.CDLL:
    """Loads libdsa_b200.so once and attaches the C signatures.  Raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with lightning_indexer_b200.build.build()")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


class DSAError(RuntimeError):
    def __init__(self, name: str, status: int):
        msg = load().dsa_status_string(status).decode()
        if status == -4:
            text = ctypes.c_char_p()
            code = load().dsa_last_cuda_error(ctypes.byref(text))
            msg += f" [cuda error {code}: {text.value.decode() if text.value else ''}]"
        super().__init__(f"{name} failed: {msg} ({status})")
        self.status = status


def call(name: str, *args) -> int:
    """Calls a status-returning entry point and raises DSAError on a non-zero status."""
    st = getattr(load(), name)(*args)
    if st != 0:
        raise DSAError(name, st)
    return st
