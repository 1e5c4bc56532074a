"""Helpers shared by the GPU tests: moving raw bits between numpy and the
device, and calling the library through its binding."""
from __future__ import annotations

import numpy as np
import torch

from fp32_weight_compression_b200 import wc


def to_device(bits: np.ndarray, fp8=torch.float8_e4m3fn) -> torch.Tensor:
    """uint16 bits -> bf16 tensor, float16 values -> fp16 tensor, uint8 bits
    -> fp8 tensor (e4m3 unless fp8=torch.float8_e5m2), uint32 bits -> fp32
    tensor, on cuda:0."""
    bits = np.ascontiguousarray(bits)
    if bits.dtype == np.uint16:
        t = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)
    elif bits.dtype == np.float16:
        t = torch.from_numpy(bits.view(np.int16)).view(torch.float16)
    elif bits.dtype == np.uint8:
        t = torch.from_numpy(bits.copy()).view(fp8)
    elif bits.dtype == np.uint32:
        t = torch.from_numpy(bits.view(np.int32)).view(torch.float32)
    else:
        raise TypeError(bits.dtype)
    return t.to("cuda")


def to_bits(t: torch.Tensor) -> np.ndarray:
    t = t.detach().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    if t.dtype == torch.float16:
        return t.view(torch.int16).cpu().numpy().view(np.float16)
    if t.dtype in (torch.float8_e4m3fn, torch.float8_e5m2):
        return t.view(torch.uint8).cpu().numpy()
    if t.dtype == torch.float32:
        return t.view(torch.int32).cpu().numpy().view(np.uint32)
    raise TypeError(t.dtype)


def gpu_encode(bits: np.ndarray) -> np.ndarray:
    return wc.encode(to_device(bits)).cpu().numpy()


def gpu_roundtrip(bits: np.ndarray, fp8=torch.float8_e4m3fn):
    """(container bytes, decoded bits) through wc_encode / wc_decode."""
    t = to_device(bits, fp8)
    cont = wc.encode(t)
    out = wc.decode(cont, shape=(bits.size,), dtype=t.dtype)
    torch.cuda.synchronize()
    return cont.cpu().numpy(), to_bits(out)


def cont_device(cont_np: np.ndarray, pad: int = 0) -> torch.Tensor:
    """Container bytes on the device (16-byte aligned, optional tail room)."""
    buf = torch.zeros(cont_np.size + pad, dtype=torch.uint8, device="cuda")
    buf[: cont_np.size] = torch.from_numpy(np.ascontiguousarray(cont_np))
    return buf[: cont_np.size]
