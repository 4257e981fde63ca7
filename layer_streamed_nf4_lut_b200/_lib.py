"""ctypes binding of libsoup.so (the C-ABI in include/soup.h).  Argument marshalling only.

Importing this module loads the in-tree libsoup.so and fails loudly if it is missing: there
is no fallback implementation of any kernel.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import (POINTER, Structure, c_char_p, c_float, c_int, c_int32, c_longlong, c_size_t, c_void_p,
                    CFUNCTYPE)

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libsoup.so")

SOUP_OK = 0
STATUS = {0: "SOUP_OK", -1: "SOUP_ERR_INVALID_ARG", -2: "SOUP_ERR_STATE", -3: "SOUP_ERR_OOM", -4: "SOUP_ERR_CUDA",
          -5: "SOUP_ERR_TIMEOUT", -6: "SOUP_ERR_DEVICE_CHECK", -7: "SOUP_ERR_UNSUPPORTED", -8: "SOUP_ERR_IO"}
SOUP_RESIDENT, SOUP_STREAMED = 0, 1
SOUP_SOURCE_RAM, SOUP_SOURCE_FILE, SOUP_SOURCE_AUTO = 0, 1, 2
SOUP_LOSS_SFT, SOUP_LOSS_DPO, SOUP_LOSS_KTO, SOUP_LOSS_ORPO, SOUP_LOSS_SIMPO = 0, 1, 2, 3, 4
LOSS_KINDS = {"sft": 0, "dpo": 1, "kto": 2, "orpo": 3, "simpo": 4}
PROJ = ("q", "k", "v", "o", "gate", "up", "down")


class SoupError(RuntimeError):
    def __init__(self, status: int, msg: str = ""):
        self.status = status
        super().__init__(f"{STATUS.get(status, status)}: {msg}")


class ModelConfig(Structure):
    _fields_ = [("n_layers", c_int), ("hidden", c_int), ("n_heads", c_int), ("n_kv_heads", c_int),
                ("head_dim", c_int), ("intermediate", c_int), ("vocab", c_int), ("rms_eps", c_float),
                ("rope_theta", c_float), ("lora_r", c_int), ("lora_alpha", c_float), ("mode", c_int),
                ("n_layer_buffers", c_int), ("max_tokens", c_int), ("device", c_int), ("stream_source", c_int),
                ("stack_path", ctypes.c_char_p)]


ALLOC_FN = CFUNCTYPE(c_void_p, c_size_t, c_void_p)
FREE_FN = CFUNCTYPE(None, c_void_p, c_void_p)


class Allocator(Structure):
    _fields_ = [("alloc", ALLOC_FN), ("free", FREE_FN), ("user", c_void_p)]


class Stats(Structure):
    _fields_ = [("layer_loads", c_longlong), ("bytes_h2d", c_longlong), ("layer_reuses", c_longlong),
                ("kernel_launches", c_longlong), ("device_bytes", c_longlong), ("pinned_bytes", c_longlong),
                ("steps", c_longlong), ("file_bytes_read", c_longlong), ("file_read_ms", ctypes.c_double),
                ("stream_source", c_int)]


class ProfileEntry(Structure):
    _fields_ = [("name", ctypes.c_char * 32), ("launches", c_longlong), ("total_ms", ctypes.c_double),
                ("flops", ctypes.c_double), ("bytes", ctypes.c_double)]


class GemmPlanInfo(Structure):
    _fields_ = [("mt", c_int), ("bn", c_int), ("splits", c_int), ("fused_reduce", c_int), ("stream_k_ctas", c_int),
                ("stream_k_tiles", c_int), ("stream_k_tiles_m", c_int), ("stream_k_kblocks", c_int)]


class Batch(Structure):
    _fields_ = [("ids", c_void_p), ("loss_mask", c_void_p), ("B", c_int), ("S", c_int), ("ids_on_host", c_int),
                ("n_pairs", c_int), ("prefix_len", c_int), ("beta", c_float), ("lr", c_float),
                ("apply_optimizer", c_int), ("dpo_shared_load", c_int), ("labels", c_void_p), ("gamma", c_float),
                ("lambda_or", c_float), ("lambda_d", c_float), ("lambda_u", c_float), ("share_prefix", c_int)]


# name -> (restype, argtypes); every function returns soup_status unless stated
SIGNATURES = {
    "soup_model_create": [POINTER(ModelConfig), POINTER(Allocator), POINTER(c_void_p)],
    "soup_model_destroy": [c_void_p],
    "soup_layer_blob_bytes": [POINTER(ModelConfig), POINTER(c_size_t)],
    "soup_layer_blob_part": [POINTER(ModelConfig), c_int, c_int, POINTER(c_size_t), POINTER(c_size_t)],
    "soup_model_quantize_layer": [c_void_p, c_int, POINTER(c_void_p), c_void_p, c_void_p, c_void_p],
    "soup_model_load_layer": [c_void_p, c_int, POINTER(c_void_p), c_void_p, c_void_p],
    "soup_model_load_layer_nf4": [c_void_p, c_int, c_void_p, c_size_t],
    "soup_model_read_layer_nf4": [c_void_p, c_int, c_void_p, c_size_t],
    "soup_model_set_head": [c_void_p, c_void_p, c_void_p, c_void_p],
    "soup_lora_numel": [POINTER(ModelConfig), POINTER(c_size_t)],
    "soup_lora_offset": [POINTER(ModelConfig), c_int, c_int, c_int, POINTER(c_size_t), POINTER(c_int), POINTER(c_int)],
    "soup_model_set_lora": [c_void_p, c_void_p, c_void_p, c_void_p, c_void_p],
    "soup_set_lora_enabled": [c_void_p, c_int],
    "soup_model_set_lora_proj": [c_void_p, c_int, c_int, c_void_p, c_void_p, c_void_p],
    "soup_model_refresh_lora": [c_void_p, c_void_p],
    "soup_model_merge_lora": [c_void_p, c_int, c_int, c_void_p, c_void_p],
    "soup_layer_fwd": [c_void_p, c_int, c_void_p, c_void_p, c_int, c_int, c_void_p],
    "soup_layer_bwd": [c_void_p, c_int, c_void_p, c_void_p, c_int, c_int, c_void_p],
    "soup_step": [c_void_p, c_int, POINTER(Batch), POINTER(c_float), c_void_p],
    "soup_optimizer_step": [c_void_p, c_float, c_void_p],
    "soup_last_logps": [c_void_p, POINTER(c_float), POINTER(c_float), c_int],
    "soup_nf4_quantize": [c_void_p, c_longlong, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p],
    "soup_nf4_quantize_static": [c_void_p, c_longlong, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p],
    "soup_nf4_quantize_host": [c_void_p, c_longlong, c_void_p, c_void_p, c_void_p, c_void_p, c_int],
    "soup_nf4_dequantize": [c_void_p, c_void_p, c_void_p, c_void_p, c_longlong, c_void_p, c_void_p],
    "soup_nf4_matmul": [c_void_p, c_int, c_int, c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_void_p,
                        c_void_p, c_void_p],
    "soup_nf4_codebook": [POINTER(c_float)],
    "soup_get_stats": [c_void_p, POINTER(Stats)],
    "soup_reset_stats": [c_void_p],
    "soup_check_device": [c_void_p, c_void_p],
    "soup_selftest_bounded_wait": [c_void_p, c_int, c_void_p],
    "soup_set_profiling": [c_void_p, c_int],
    "soup_h2d_probe": [c_void_p, c_int, POINTER(ctypes.c_double)],
    "soup_get_profile": [c_void_p, POINTER(ProfileEntry), c_int, POINTER(c_int), c_int],
    "soup_set_timed_category": [c_void_p, ctypes.c_char_p],
    "soup_get_timed_category": [c_void_p, POINTER(ProfileEntry), c_int],
    "soup_get_timed_profile": [c_void_p, POINTER(ProfileEntry), c_int, POINTER(c_int), c_int],
    "soup_gemm_plan": [c_int, c_int, c_int, c_int, c_int, c_int, POINTER(GemmPlanInfo)],
    "soup_gemm_stream_k_pieces": [ctypes.c_longlong, c_int, c_int, c_int, c_int, POINTER(c_int), POINTER(c_int),
                                  POINTER(c_int), POINTER(c_int), POINTER(c_int)],
    "soup_gemm_stream_k_shares": [ctypes.c_longlong, c_int, c_int, c_int, c_int, POINTER(c_int), POINTER(c_int),
                                  POINTER(c_int)],
}
STRING_FUNCS = {"soup_status_string": [c_int32], "soup_last_error": [c_void_p]}


def load(path: str = LIB_PATH):
    if not os.path.exists(path):
        raise ImportError(f"libsoup.so not found at {path}: build it with `python -m layer_streamed_nf4_lut_b200.build`"
                          " (there is no non-CUDA fallback)")
    lib = ctypes.CDLL(path)
    for name, args in SIGNATURES.items():
        f = getattr(lib, name)
        f.restype = c_int32
        f.argtypes = args
    for name, args in STRING_FUNCS.items():
        f = getattr(lib, name)
        f.restype = c_char_p
        f.argtypes = args
    return lib


lib = load()


def check(status: int, model_handle=None):
    if status != SOUP_OK:
        msg = ""
        if model_handle:
            msg = (lib.soup_last_error(model_handle) or b"").decode(errors="replace")
        raise SoupError(status, msg or lib.soup_status_string(status).decode())
