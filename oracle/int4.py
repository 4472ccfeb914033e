"""Asymmetric 4-bit KV quantisation: fp32 mirror of the encoder, exact decoder.

Test infrastructure only (see ``oracle/__init__.py``).

Pages: "DuoAttention: Efficient Long-Context LLM Inference with Retrieval and
Streaming Heads" (hotpaper.ai), abstract (combined with quantisation, 3.3M-token
Llama-3-8B decoding on one A100) and section "기술적 접근법" (compatible with
8-bit weights plus a 4-bit KV cache).  The pages give no scheme; the reading
used here is one group per (token, KV head) of d channels, K and V separately,
asymmetric, with fp16 scale and zero:

    mn = min x,  mx = max x                      (exact)
    sc = fp16_rn( fp32(mx - mn) / 15 )           (two fp32 roundings, then fp16)
    zp = fp16_rn(mn)
    u  = clamp(rint_even( fp32( fp32(x - zp) / sc ) ), 0, 15);  u = 0 if sc == 0
    x_hat = sc * u + zp                          (exact in fp64)

Every encoder step is one IEEE single-precision operation, so an independent
implementation that performs the same correctly rounded operations produces the
same codes and scales bit for bit.  Nibble order: the low nibble of byte i holds
channel 2i, the high nibble channel 2i+1.
"""

import numpy as np

__all__ = ["quantize_int4", "pack_nibbles", "unpack_nibbles", "dequantize_int4"]


def quantize_int4(x):
    """x: float32 [..., d] -> (codes uint8 [..., d] in 0..15, sc fp16 [...], zp fp16 [...])."""
    x = np.asarray(x, dtype=np.float32)
    mn = x.min(axis=-1)
    mx = x.max(axis=-1)
    span = np.subtract(mx, mn, dtype=np.float32)
    sc32 = np.divide(span, np.float32(15.0), dtype=np.float32)
    sc = sc32.astype(np.float16)
    zp = mn.astype(np.float16)
    scf = sc.astype(np.float32)[..., None]
    zpf = zp.astype(np.float32)[..., None]
    with np.errstate(divide="ignore", invalid="ignore"):
        t = np.divide(np.subtract(x, zpf, dtype=np.float32), scf,
                      dtype=np.float32)
    u = np.rint(t)
    u = np.where(scf == 0, np.float32(0), u)
    u = np.clip(u, 0, 15)
    return u.astype(np.uint8), sc, zp


def pack_nibbles(codes):
    """uint8 codes [..., d] (0..15) -> bytes [..., d/2], low nibble = even channel."""
    codes = np.asarray(codes, dtype=np.uint8)
    lo = codes[..., 0::2]
    hi = codes[..., 1::2]
    return (lo | (hi << 4)).astype(np.uint8)


def unpack_nibbles(packed):
    """Inverse of :func:`pack_nibbles`."""
    packed = np.asarray(packed, dtype=np.uint8)
    out = np.empty(packed.shape[:-1] + (packed.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = packed & 0xF
    out[..., 1::2] = packed >> 4
    return out


def dequantize_int4(codes, sc, zp):
    """x_hat = sc * u + zp in float64 (exact: fp16 values times 0..15)."""
    return (np.asarray(sc, dtype=np.float64)[..., None] * codes.astype(np.float64)
            + np.asarray(zp, dtype=np.float64)[..., None])
