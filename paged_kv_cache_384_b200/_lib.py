"""ctypes loader for the in-tree ``libpagedattn.so`` (argument types only, no logic).

There is no fallback: if the library is missing or fails to load, importing the package
raises, and every entry point is a call into the CUDA library.
"""
import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpagedattn.so")

c_int, c_int32, c_int64, c_float, c_double, c_size_t, c_void_p, c_uint32 = (
    ctypes.c_int, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_double,
    ctypes.c_size_t, ctypes.c_void_p, ctypes.c_uint32)
P = ctypes.POINTER

# name -> (restype, argtypes); mirrors include/pagedattn.h
SIGNATURES = {
    "pa_last_error": (ctypes.c_char_p, []),
    "pa_version": (ctypes.c_char_p, []),
    "pa_device_error": (c_int, [P(c_uint32), c_int]),
    "pa_decode_workspace_bytes": (c_size_t, [c_int, c_int, c_int]),
    "paged_attention_decode": (c_int, [
        c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
        c_int, c_int, c_int, c_int, c_int, c_int, c_float, c_int, c_int, c_int,
        c_void_p, c_size_t, c_void_p]),
    "paged_attention_decode_gqa": (c_int, [
        c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
        c_int, c_int, c_int, c_int, c_int, c_int, c_int, c_float, c_int, c_int, c_int,
        c_void_p, c_size_t, c_void_p]),
    "paged_attention_decode_static_scratch": (c_int, [
        c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
        c_int, c_int, c_int, c_int, c_int, c_int, c_float, c_int, c_int, c_int, c_void_p]),
    "paged_attention_prefill": (c_int, [
        c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_int,
        c_int, c_int, c_int, c_int, c_int, c_float, c_int, c_int, c_void_p]),
    "paged_attention_prefill_quant": (c_int, [
        c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_int,
        c_int, c_int, c_int, c_int, c_int, c_int, c_int, c_float, c_int, c_int, c_int, c_void_p]),
    "reshape_and_cache": (c_int, [
        c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_int,
        c_int64, c_int64, c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p]),
    "reshape_and_cache_quant": (c_int, [
        c_void_p, c_void_p, c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_void_p, c_int, c_int,
        c_int, c_int, c_int, c_int64, c_int64, c_void_p]),
    "copy_blocks": (c_int, [
        c_void_p, c_void_p, c_void_p, c_int, c_int, c_size_t, c_void_p, c_void_p, c_size_t, c_void_p]),
    "swap_blocks": (c_int, [
        c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_size_t,
        c_void_p, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "pa_bm_create": (c_void_p, [c_int, c_int, c_void_p]),
    "pa_bm_destroy": (None, [c_void_p]),
    "pa_bm_allocate": (c_int, [c_void_p, c_int, c_void_p]),
    "pa_bm_free": (c_int, [c_void_p, c_void_p, c_int]),
    "pa_bm_share": (c_int, [c_void_p, c_void_p, c_int]),
    "pa_bm_copy_on_write": (c_int, [c_void_p, c_int32, P(c_int32)]),
    "pa_bm_num_free": (c_int, [c_void_p]),
    "pa_bm_ref_count": (c_int, [c_void_p, c_int32]),
    "pa_bm_usage_ratio": (c_double, [c_void_p]),
    "pa_bm_free_list": (c_int, [c_void_p, c_void_p, c_int, P(c_int)]),
    "pa_slot_mapping_host": (c_int, [c_void_p, c_int, c_int, c_int, c_void_p, c_void_p, c_int, c_void_p]),
    "pa_profile_enable": (c_int, [c_int]),
    "pa_decode_use_tensor_cores": (c_int, [c_int]),
    "pa_profile_read": (c_int, [P(c_double), P(c_double), P(c_int), c_int]),
}


def load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python paged_kv_cache_384_b200/build.py` "
            "(there is no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib
