"""ctypes binding of libnf4ls.so: the C-ABI calls under the same names.

Argument marshalling only.  Every step of the training path runs in the library's
CUDA kernels; torch supplies device memory, pinned host memory and streams.  The
library must be built (``python -m nf4_layer_streamed_b200.build``); loading fails
loudly when it is missing -- there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libnf4ls.so")

OK = 0
STATUS = {0: "OK", -1: "INVALID_ARG", -2: "SHAPE", -3: "ALIGN", -4: "CODEBOOK_MISMATCH",
          -5: "FINGERPRINT_MISMATCH", -6: "BUFFER_BUSY", -7: "TIMEOUT", -8: "CUDA", -9: "DEVICE_FAULT",
          -10: "SOURCE_REFUSED", -11: "IO"}


class NF4LSError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS.get(status, status)}: {msg}")
        self.status = status


class LayerCfg(ctypes.Structure):
    _fields_ = [("hidden", ctypes.c_int32), ("inter", ctypes.c_int32), ("n_q", ctypes.c_int32),
                ("n_kv", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("batch", ctypes.c_int32),
                ("seq", ctypes.c_int32), ("rope_theta", ctypes.c_float), ("rms_eps", ctypes.c_float),
                ("lora_r", ctypes.c_int32), ("lora_alpha", ctypes.c_float)]


class Lora(ctypes.Structure):
    _fields_ = [("A_q", ctypes.c_void_p), ("B_q", ctypes.c_void_p), ("A_v", ctypes.c_void_p),
                ("B_v", ctypes.c_void_p)]


class LoraGrads(ctypes.Structure):
    _fields_ = [("dA_q", ctypes.c_void_p), ("dB_q", ctypes.c_void_p), ("dA_v", ctypes.c_void_p),
                ("dB_v", ctypes.c_void_p)]


class ModelCfg(ctypes.Structure):
    _fields_ = [("layer", LayerCfg), ("n_layers", ctypes.c_int32), ("vocab", ctypes.c_int32),
                ("tied", ctypes.c_int32), ("lr", ctypes.c_float), ("beta1", ctypes.c_float),
                ("beta2", ctypes.c_float), ("adam_eps", ctypes.c_float), ("weight_decay", ctypes.c_float),
                ("head_chunk_rows", ctypes.c_int32)]


class Model(ctypes.Structure):
    _fields_ = [("embed_dev", ctypes.c_void_p), ("lm_head_dev", ctypes.c_void_p),
                ("norm_final_dev", ctypes.c_void_p), ("lora_dev", ctypes.c_void_p),
                ("grads_dev", ctypes.c_void_p), ("adam_m_dev", ctypes.c_void_p),
                ("adam_v_dev", ctypes.c_void_p), ("pool", ctypes.c_void_p),
                ("shards_dev", ctypes.c_void_p), ("ws_dev", ctypes.c_void_p), ("ws_bytes", ctypes.c_size_t),
                ("head_pool", ctypes.c_void_p), ("embed_host", ctypes.c_void_p)]


class PoolStats(ctypes.Structure):
    _fields_ = [("bytes_copied", ctypes.c_uint64), ("copies", ctypes.c_uint64), ("hits", ctypes.c_uint64),
                ("acquisitions", ctypes.c_uint64), ("peer_bytes", ctypes.c_uint64)]


class PlanStep(ctypes.Structure):
    _fields_ = [("slot", ctypes.c_int32), ("hit", ctypes.c_int32), ("fill", ctypes.c_int32),
                ("after_release", ctypes.c_int32), ("owner", ctypes.c_int32), ("host_read", ctypes.c_int32),
                ("broadcast", ctypes.c_int32)]


class DiskInfo(ctypes.Structure):
    _fields_ = [("read_gbs", ctypes.c_double), ("block_device", ctypes.c_int32), ("nvme", ctypes.c_int32),
                ("rotational", ctypes.c_int32), ("direct_io", ctypes.c_int32)]


P = ctypes.c_void_p
I32 = ctypes.c_int32
SZ = ctypes.c_size_t
U64 = ctypes.c_uint64

# name -> (restype, argtypes): every symbol that include/nf4ls.h declares.
SIGNATURES = {
    "nf4ls_last_error": (ctypes.c_char_p, []),
    "nf4ls_version": (ctypes.c_int, []),
    "nf4ls_device_error": (ctypes.c_int, [P]),
    "nf4ls_wait_probe": (ctypes.c_int, [ctypes.c_int32, P, P]),
    "nf4ls_launch_count": (U64, []),
    "nf4ls_profile": (ctypes.c_int, [ctypes.c_int]),
    "nf4ls_profile_read": (ctypes.c_int, [ctypes.c_int, P]),
    "nf4ls_profile_reset": (ctypes.c_int, []),
    "nf4ls_codebooks": (ctypes.c_int, [P, P, ctypes.POINTER(U64)]),
    "nf4ls_quantize_scratch_bytes": (SZ, [SZ]),
    "nf4_quantize_tensor": (ctypes.c_int, [P, SZ, P, P, P, P, P, SZ, P]),
    "nf4_dequantize_tensor": (ctypes.c_int, [P, P, P, P, SZ, P, P]),
    "nf4ls_quantize_noalloc_max_elems": (SZ, []),
    "nf4_quantize_tensor_noalloc": (ctypes.c_int, [P, SZ, P, P, P, P, P]),
    "nf4ls_shard_bytes": (SZ, [ctypes.POINTER(LayerCfg)]),
    "nf4ls_shard_quantized_bytes": (SZ, [ctypes.POINTER(LayerCfg)]),
    "nf4ls_shard_scratch_bytes": (SZ, [ctypes.POINTER(LayerCfg)]),
    "nf4_quantize_shard": (ctypes.c_int, [ctypes.POINTER(LayerCfg), P, U64, P, SZ, ctypes.POINTER(SZ), P, SZ, P]),
    "nf4ls_shard_check": (ctypes.c_int, [P, ctypes.POINTER(LayerCfg), U64]),
    "nf4ls_workspace_bytes": (SZ, [ctypes.POINTER(LayerCfg)]),
    "layer_forward": (ctypes.c_int, [ctypes.POINTER(LayerCfg), P, ctypes.POINTER(Lora), P, P, P, SZ, P]),
    "layer_backward": (ctypes.c_int, [ctypes.POINTER(LayerCfg), P, ctypes.POINTER(Lora), P, P, P,
                                      ctypes.POINTER(LoraGrads), P, SZ, P]),
    "nf4ls_set_gemm_path": (ctypes.c_int, [ctypes.c_int]),
    "nf4ls_set_gemm_pair": (ctypes.c_int, [ctypes.c_int]),
    "nf4ls_set_gemm_half": (ctypes.c_int, [ctypes.c_int]),
    "nf4ls_set_attention_path": (ctypes.c_int, [ctypes.c_int]),
    "nf4ls_pool_create": (ctypes.c_int, [P, P, P, ctypes.c_int, ctypes.c_int, P, SZ, ctypes.POINTER(P)]),
    "nf4ls_pool_prefetch": (ctypes.c_int, [P, ctypes.c_int]),
    "stream_prefetch": (ctypes.c_int, [P, ctypes.c_int, P, ctypes.POINTER(P)]),
    "nf4ls_pool_release": (ctypes.c_int, [P, ctypes.c_int, P]),
    "nf4ls_wait": (ctypes.c_int, [P, ctypes.c_int, ctypes.c_int]),
    "nf4ls_pool_set_poison": (ctypes.c_int, [P, ctypes.c_int]),
    "nf4ls_pool_get_stats": (ctypes.c_int, [P, ctypes.POINTER(PoolStats)]),
    "nf4ls_pool_synchronize": (ctypes.c_int, [P]),
    "nf4ls_pool_destroy": (ctypes.c_int, [P]),
    "nf4ls_nccl_unique_id": (ctypes.c_int, [P]),
    "nf4ls_pool_share": (ctypes.c_int, [P, ctypes.c_int, ctypes.c_int, P]),
    "nf4ls_plan_create": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, ctypes.POINTER(P)]),
    "nf4ls_plan_share": (ctypes.c_int, [P, ctypes.c_int, ctypes.c_int]),
    "nf4ls_plan_prefetch": (ctypes.c_int, [P, ctypes.c_int, ctypes.POINTER(PlanStep)]),
    "nf4ls_plan_acquire": (ctypes.c_int, [P, ctypes.c_int, ctypes.POINTER(PlanStep)]),
    "nf4ls_plan_release": (ctypes.c_int, [P, ctypes.c_int]),
    "nf4ls_plan_destroy": (ctypes.c_int, [P]),
    "nf4ls_step_pass_ops": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, P, P, ctypes.c_int, ctypes.POINTER(I32)]),
    "nf4ls_disk_probe": (ctypes.c_int, [ctypes.c_char_p, SZ, ctypes.POINTER(DiskInfo)]),
    "nf4ls_disk_accept": (ctypes.c_int, [ctypes.POINTER(DiskInfo), ctypes.c_double]),
    "nf4ls_choose_source": (ctypes.c_int, [SZ, SZ, ctypes.POINTER(ctypes.c_int32)]),
    "nf4ls_pool_file_staging_bytes": (SZ, [P, ctypes.c_int]),
    "nf4ls_pool_create_file": (ctypes.c_int, [ctypes.c_char_p, P, P, ctypes.c_int, ctypes.c_int, P, SZ, P, SZ,
                                              ctypes.POINTER(P)]),
    "nf4ls_lora_stride": (SZ, [ctypes.POINTER(LayerCfg)]),
    "nf4ls_model_workspace_bytes": (SZ, [ctypes.POINTER(ModelCfg)]),
    "nf4ls_train_step": (ctypes.c_int, [ctypes.POINTER(ModelCfg), ctypes.POINTER(Model), P, I32, P, P]),
    "nf4ls_forward_loss": (ctypes.c_int, [ctypes.POINTER(ModelCfg), ctypes.POINTER(Model), P, I32, P, P]),
    "nf4ls_forward_backward": (ctypes.c_int, [ctypes.POINTER(ModelCfg), ctypes.POINTER(Model), P, P, P]),
    "nf4ls_adamw_step": (ctypes.c_int, [ctypes.POINTER(ModelCfg), ctypes.POINTER(Model), I32, P]),
    "nf4ls_adapter_file_bytes": (SZ, [ctypes.POINTER(ModelCfg)]),
    "nf4ls_adapter_save": (ctypes.c_int, [ctypes.c_char_p, ctypes.POINTER(ModelCfg), ctypes.POINTER(Model), I32, P]),
    "nf4ls_adapter_load": (ctypes.c_int, [ctypes.c_char_p, ctypes.POINTER(ModelCfg), ctypes.POINTER(Model),
                                          ctypes.POINTER(ctypes.c_int32), P]),
    "nf4ls_mse_loss": (ctypes.c_int, [P, SZ, P, P, P, ctypes.c_int, P]),
    "nf4ls_gemm_bf16": (ctypes.c_int, [P, P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                       ctypes.c_int, P]),
    "nf4ls_gemm_nf4": (ctypes.c_int, [P, ctypes.c_int, ctypes.c_int, P, P, P, P, ctypes.c_int, ctypes.c_int,
                                      ctypes.c_int, P, ctypes.c_int, P]),
    "nf4ls_attention_fwd": (ctypes.c_int, [ctypes.POINTER(LayerCfg), P, P, P, ctypes.c_int, ctypes.c_int, P, P, P]),
    "nf4ls_attention_bwd": (ctypes.c_int, [ctypes.POINTER(LayerCfg), P, P, P, ctypes.c_int, ctypes.c_int, P, P, P, P,
                                           P, P, P, P]),
}

_LIB = None


def lib() -> ctypes.CDLL:
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m nf4_layer_streamed_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _LIB = L
    return _LIB


def check(status: int) -> None:
    if status != OK:
        raise NF4LSError(status, lib().nf4ls_last_error().decode(errors="replace"))


def last_error() -> str:
    return lib().nf4ls_last_error().decode(errors="replace")


def call(name: str, *args):
    """Calls a status-returning entry point and raises NF4LSError on failure."""
    st = getattr(lib(), name)(*args)
    check(st)
    return st


def call_status(name: str, *args) -> int:
    """Calls a status-returning entry point and returns the status."""
    return getattr(lib(), name)(*args)
