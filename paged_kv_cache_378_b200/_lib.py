"""ctypes loader for ``libpagedkv.so`` (the C ABI in ``include/pagedkv.h``)."""

import ctypes
import os
import threading

from . import build as _build

_lock = threading.Lock()
_lib = None


class PkvCache(ctypes.Structure):
    _fields_ = [
        ("k_pool", ctypes.c_void_p),
        ("v_pool", ctypes.c_void_p),
        ("num_layers", ctypes.c_int32),
        ("num_blocks", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("block_size", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
    ]


class PkvBlockState(ctypes.Structure):
    _fields_ = [
        ("block_tables", ctypes.c_void_p),
        ("seq_lens", ctypes.c_void_p),
        ("refcount", ctypes.c_void_p),
        ("free_ring", ctypes.c_void_p),
        ("free_state", ctypes.c_void_p),
    ]


# name -> (restype, argtypes); mirrors include/pagedkv.h
SIGNATURES = {
    "pkv_kv_append": (ctypes.c_int, [ctypes.POINTER(PkvCache), ctypes.c_int, ctypes.c_void_p,
                                     ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]),
    "pkv_block_copy": (ctypes.c_int, [ctypes.POINTER(PkvCache), ctypes.c_void_p, ctypes.c_int,
                                      ctypes.c_void_p]),
    "pkv_block_copy_device_count": (ctypes.c_int, [ctypes.POINTER(PkvCache), ctypes.c_void_p,
                                                   ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]),
    "pkv_swap_blocks": (ctypes.c_int, [ctypes.POINTER(PkvCache), ctypes.POINTER(PkvCache),
                                       ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_void_p]),
    "pkv_prefix_block_hashes": (ctypes.c_int, [
        ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
        ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]),
    "pkv_block_manager_step": (ctypes.c_int, [
        ctypes.POINTER(PkvBlockState), ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
        ctypes.c_void_p]),
    "pkv_block_manager_release": (ctypes.c_int, [
        ctypes.POINTER(PkvBlockState), ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
        ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]),
    "pkv_attention_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int] * 7),
    "pkv_partition_tokens": (ctypes.c_int, [ctypes.c_int] * 6),
    "pkv_workspace_init": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "pkv_paged_decode_attention": (ctypes.c_int, [
        ctypes.POINTER(PkvCache), ctypes.c_int, ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
        ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_float, ctypes.c_void_p,
        ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_void_p]),
    "pkv_append_paged_decode_attention": (ctypes.c_int, [
        ctypes.POINTER(PkvCache), ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
        ctypes.c_void_p,
        ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_float,
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_void_p]),
    "pkv_paged_decode_attention_noalloc": (ctypes.c_int, [
        ctypes.POINTER(PkvCache), ctypes.c_int, ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
        ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_float, ctypes.c_void_p,
        ctypes.c_int, ctypes.c_void_p]),
    "pkv_get_device_status": (ctypes.c_int, [ctypes.POINTER(ctypes.c_uint), ctypes.c_int]),
    "pkv_set_wait_limit_ns": (ctypes.c_int, [ctypes.c_ulonglong]),
    "pkv_strerror": (ctypes.c_char_p, [ctypes.c_int]),
    "pkv_abi_version": (ctypes.c_int, []),
    "pkv_build_hash": (ctypes.c_char_p, []),
}


def lib_path():
    return _build.LIB_PATH


def load():
    """Load the CUDA library, building it in-tree first if it is missing or
    was built from sources other than the checkout's (its embedded source
    hash differs).

    There is no fallback: if the library cannot be built or loaded, this raises.
    """
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        path = lib_path()
        if _build.needs_build(path):
            _build.build()
        lib = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        want = _build.source_hash()
        got = lib.pkv_build_hash().decode()
        if got != want:
            raise RuntimeError(f"{path} was built from other sources (hash {got}, checkout {want})")
        _lib = lib
        return lib


def exported_symbols():
    return list(SIGNATURES)


def loaded_path():
    return lib_path() if _lib is not None else None


if os.environ.get("PKV_EAGER_LOAD") == "1":   # pragma: no cover
    load()
