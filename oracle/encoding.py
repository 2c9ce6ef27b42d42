"""Decoders from stored bit patterns to float64 (oracle; test infrastructure only).

The pages fix the storage types only by name: bfloat16 for the lightning-indexer
case and float32 for the sampling case (DeepSelect hub page, use-case
paragraphs).  The decoders below follow the IEEE-754 binary32 layout (1 sign
bit, 8 exponent bits with bias 127, 23 fraction bits) and the bfloat16 layout,
which is the upper half of a binary32 (1 sign, 8 exponent, 7 fraction bits).
They are written from those layouts, not from a library conversion, and the
tests check them against a library conversion over every bfloat16 pattern.
"""

import numpy as np

NEG_INF_BF16 = 0xFF80      # bfloat16 bit pattern of -inf (padding value)
NEG_INF_F32 = 0xFF800000   # binary32 bit pattern of -inf (padding value)


def _decode(bits, frac_bits):
    """Decode unsigned integer bit patterns with an 8-bit exponent field."""
    bits = np.asarray(bits).astype(np.int64)
    total = 1 + 8 + frac_bits
    sign = (bits >> (total - 1)) & 1
    expo = (bits >> frac_bits) & 0xFF
    frac = bits & ((1 << frac_bits) - 1)
    mag = np.empty(bits.shape, dtype=np.float64)
    normal = (expo > 0) & (expo < 255)
    # normal numbers: (1 + frac / 2^frac_bits) * 2^(expo - 127)
    mag[normal] = np.ldexp(1.0 + frac[normal] / float(1 << frac_bits),
                           (expo[normal] - 127).astype(np.int32))
    # zero and subnormals: frac / 2^frac_bits * 2^(-126)
    sub = expo == 0
    mag[sub] = np.ldexp(frac[sub].astype(np.float64),
                        np.full(int(sub.sum()), -126 - frac_bits, dtype=np.int32))
    special = expo == 255
    mag[special & (frac == 0)] = np.inf
    mag[special & (frac != 0)] = np.nan
    return np.where(sign == 1, -mag, mag)


def decode_bf16(bits):
    """bfloat16 bit patterns (any integer dtype, low 16 bits used) -> float64."""
    return _decode(np.asarray(bits).astype(np.int64) & 0xFFFF, 7)


def decode_f32(bits):
    """binary32 values or bit patterns -> float64.

    A float32 array is reinterpreted as its bit patterns first, so the decoder
    sees exactly the stored bits.
    """
    a = np.asarray(bits)
    if a.dtype == np.float32:
        a = a.view(np.uint32)
    return _decode(a.astype(np.int64) & 0xFFFFFFFF, 23)
