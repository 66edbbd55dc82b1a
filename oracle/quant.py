"""Blockwise NF4 with double-quantised absmax (oracle; test infrastructure only).

What is computed follows "Soup 层流式 NF4 训练实测：在 4 GB 显存上以位级一致标准完成 8B 模型 LoRA 微调" (m.mzlw.cn)
§2.1 (offline per-tensor quantisation into packed bytes plus absmax, nested
absmax and offset sidecars) and §2.4 (per-weight streamed bytes: N/2 packed +
N/64 absmax + N/4096 nested absmax + 4 bytes offset, about 0.516 B/param;
16-entry and 256-entry fp32 code tables).  All arithmetic is fp32, as the
pages fix it.  Readings taken where the pages are silent:

* blocks of 64 consecutive elements of the row-major [out, in] tensor;
  nested groups of 256 consecutive blocks, the last one possibly partial;
* u = x / absmax as one IEEE fp32 division; nearest table entry by the
  midpoint rule of ``codebooks``;
* a block whose absmax is 0 (or a group whose nested absmax is 0) gets the
  index of the table's exact 0;
* element 2j goes to the high nibble of byte j, element 2j+1 to the low one;
* offset = fp32(sequential float64 sum of the fp32 absmax values, in block
  order, divided by the block count in float64);
* dequantisation: s = fp32(fp32(code8[q] * nested) + offset), then
  w = bf16_rne(fp32(nf4[c] * s)); no fused multiply-add anywhere.
"""
from __future__ import annotations

import numpy as np

from . import bf16, codebooks

BLOCK = 64
NESTED = 256


def quantize(w) -> dict:
    """Quantise a flat array of bf16 values (given as fp32) to the NF4-DQ format."""
    x = np.asarray(w, dtype=np.float32).reshape(-1)
    n = x.size
    if n % BLOCK:
        raise ValueError("element count must be a multiple of 64")
    nf4 = codebooks.nf4_table()
    code8 = codebooks.code8_table()
    xb = x.reshape(-1, BLOCK)
    absmax = np.max(np.abs(xb), axis=1).astype(np.float32)
    with np.errstate(invalid="ignore", divide="ignore"):
        u = (xb / absmax[:, None]).astype(np.float32)
    codes = codebooks.nearest_index(u, nf4)
    codes[absmax == 0.0] = codebooks.zero_index(nf4)
    flat = codes.reshape(-1)
    packed = ((flat[0::2] << 4) | flat[1::2]).astype(np.uint8)

    nb = absmax.size
    offset = np.float32(np.cumsum(absmax.astype(np.float64))[-1] / np.float64(nb))
    c = (absmax - offset).astype(np.float32)
    ng = (nb + NESTED - 1) // NESTED
    pad = np.zeros(ng * NESTED, dtype=np.float32)
    pad[:nb] = np.abs(c)
    nested = np.max(pad.reshape(ng, NESTED), axis=1).astype(np.float32)
    gidx = np.arange(nb) // NESTED
    with np.errstate(invalid="ignore", divide="ignore"):
        uu = (c / nested[gidx]).astype(np.float32)
    q8 = codebooks.nearest_index(uu, code8)
    q8[nested[gidx] == 0.0] = codebooks.zero_index(code8)
    return {
        "packed": packed,
        "q8": q8.astype(np.uint8),
        "nested": nested,
        "offset": np.float32(offset),
        "n": n,
    }


def block_scales(q: dict) -> np.ndarray:
    """fp32 dequantised absmax per block: fp32(fp32(code8[q8] * nested) + offset)."""
    code8 = codebooks.code8_table()
    gidx = np.arange(q["q8"].size) // NESTED
    prod = (code8[q["q8"].astype(np.int64)] * q["nested"][gidx]).astype(np.float32)
    return (prod + np.float32(q["offset"])).astype(np.float32)


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8).astype(np.int64)
    out = np.empty(p.size * 2, dtype=np.int64)
    out[0::2] = p >> 4
    out[1::2] = p & 0xF
    return out


def dequantize_bits(q: dict) -> np.ndarray:
    """bf16 bit patterns (uint16) of the dequantised weights, flat."""
    nf4 = codebooks.nf4_table()
    codes = unpack_codes(q["packed"])
    s = block_scales(q)
    prod = (nf4[codes].reshape(-1, BLOCK) * s[:, None]).astype(np.float32)
    return bf16.f32_to_bf16_bits(prod.reshape(-1))


def dequantize(q: dict) -> np.ndarray:
    """Dequantised weights as float64 values (each exactly a bf16 value)."""
    return bf16.bf16_bits_to_f32(dequantize_bits(q)).astype(np.float64)


def tensor_bytes(n: int) -> dict:
    """Streamed bytes of one quantised tensor of n elements (the per-weight identity)."""
    nb = n // BLOCK
    ng = (nb + NESTED - 1) // NESTED
    return {"packed": n // 2, "q8": nb, "nested": 4 * ng, "offset": 4,
            "total": n // 2 + nb + 4 * ng + 4}
