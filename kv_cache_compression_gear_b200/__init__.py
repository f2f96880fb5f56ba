"""GEAR KV-cache codec for NVIDIA B200: CUDA kernels behind a C ABI (libgear.so)
with a thin ctypes binding. See include/gear.h for the ABI."""
from .gear import (GEAR_BF16, GEAR_F16, GEAR_F32, GEAR_OK, Cache, GearCacheStruct, GearError, GearParams,
                   PagedCache, append_buffer, append_rows, decode_attn, device_status, encode_batch, lib,
                   make_params, status_string)

__all__ = ["Cache", "GearCacheStruct", "GearError", "GearParams", "PagedCache", "append_buffer", "append_rows",
           "decode_attn", "device_status", "encode_batch",
           "lib", "make_params", "status_string", "GEAR_F16", "GEAR_BF16", "GEAR_F32", "GEAR_OK"]
