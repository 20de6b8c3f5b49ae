"""NVFP4 expert weights for the oracle (test infrastructure only): element and
scale decoding, dequantisation and a reference quantiser, in exact fp64.

Only tests/ may import this module; it shares nothing with the CUDA package.

The pages name the format without defining it: TensorFold #593 ("Checkpoint
formats on that family") uses NVIDIA's NVFP4 checkpoint in its stored form,
with 4-bit weights and 16-bit activations, and issue #310 counts its inputs in
groups of 16.  This module takes NVIDIA's public NVFP4 definition for the
rest:

- an element is FP4 E2M1: a sign bit, two exponent bits (bias 1) and one
  mantissa bit, so the magnitudes are 0, 0.5, 1, 1.5, 2, 3, 4 and 6;
- every run of 16 consecutive elements of a row (along the reduction
  dimension) shares one block scale in FP8 E4M3: a sign bit, four exponent
  bits (bias 7) and three mantissa bits, no infinities, S.1111.111 = NaN,
  largest finite value 448;
- each tensor carries one fp32 scale, and an element's value is
  tensor scale x block scale x element.

Storage:

- codes two per byte, element 2i in the low nibble and element 2i + 1 in the
  high nibble, [rows][cols / 2];
- block scales one byte each, [rows][cols / 16].

The quantiser here produces test data and is not NVIDIA's calibration.  Its
tensor scale is a power of two, at least amax / (6 x 448).  So every block
scale fits E4M3, and every dequantised weight (at most 2 x 4 significant bits
times a power of two) is exact in bf16.  The bf16 oracle then takes the
dequantised weights unchanged.
"""
import numpy as np

BLOCK = 16            # elements per block scale
E2M1_MAX = 6.0
E4M3_MAX = 448.0


# ------------------------------------------------------------------ FP4 E2M1
def e2m1_decode(codes):
    """Value of each 4-bit code (0..15), from its sign / exponent / mantissa bits."""
    c = np.asarray(codes, dtype=np.int64)
    if np.any((c < 0) | (c > 15)):
        raise ValueError("E2M1 codes are 4-bit")
    sign = np.where(c & 8, -1.0, 1.0)
    e = (c >> 1) & 3
    m = c & 1
    mag = np.where(e == 0, 0.5 * m, np.ldexp(1.0 + 0.5 * m, e - 1))
    return sign * mag


def e2m1_encode(x):
    """Round each value to the nearest E2M1 value, ties to the even code;
    magnitudes above 6 saturate to 6.  -0.0 and +0.0 both give code 0."""
    x = np.asarray(x, dtype=np.float64)
    if np.any(np.isnan(x)):
        raise ValueError("NaN has no E2M1 code")
    a = np.minimum(np.abs(x), E2M1_MAX)
    # grid spacing of the binade: 0.5 below 2, 1 in [2, 4), 2 from 4 on; an
    # even multiple of the spacing is an even code in each binade
    step = np.where(a < 2.0, 0.5, np.where(a < 4.0, 1.0, 2.0))
    q = np.minimum(np.rint(a / step) * step, E2M1_MAX)
    # magnitude -> code: 0, 0.5, 1, 1.5 are 0..3 (steps of 0.5), 2, 3 are 4, 5,
    # 4, 6 are 6, 7
    mag_code = np.where(q < 2.0, q / 0.5, np.where(q < 4.0, q + 2.0, q / 2.0 + 4.0))
    code = mag_code.astype(np.int64)
    neg = (x < 0) & (code != 0)
    return (code | np.where(neg, 8, 0)).astype(np.uint8)


# ------------------------------------------------------------------ FP8 E4M3
def e4m3_decode(codes):
    """Value of each byte as FP8 E4M3 (NaN for S.1111.111)."""
    c = np.asarray(codes, dtype=np.int64)
    if np.any((c < 0) | (c > 255)):
        raise ValueError("E4M3 codes are 8-bit")
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 15
    m = c & 7
    mag = np.where(e == 0, np.ldexp(m / 8.0, -6), np.ldexp(1.0 + m / 8.0, e - 7))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag


def e4m3_encode(x):
    """Round each non-negative value to the nearest E4M3 value, ties to the
    even code; values above 448 saturate to 448."""
    x = np.asarray(x, dtype=np.float64)
    if np.any(np.isnan(x)) or np.any(x < 0):
        raise ValueError("block scales are finite and non-negative")
    a = np.minimum(x, E4M3_MAX)
    # spacing: 2^-9 below the smallest normal 2^-6, else 2^(floor(log2 a) - 3)
    _, ex = np.frexp(np.maximum(a, np.ldexp(1.0, -6)))  # a = f 2^ex, f in [0.5, 1)
    step = np.ldexp(1.0, ex - 1 - 3)
    q = np.minimum(np.rint(a / step) * step, E4M3_MAX)
    # value -> code
    _, qe = np.frexp(np.maximum(q, np.ldexp(1.0, -6)))
    e_field = np.where(q < np.ldexp(1.0, -6), 0, qe - 1 + 7)
    m_field = np.where(e_field == 0, np.rint(q / np.ldexp(1.0, -9)),
                       np.rint((q / np.ldexp(1.0, qe - 1) - 1.0) * 8.0))
    return ((e_field.astype(np.int64) << 3) | m_field.astype(np.int64)).astype(np.uint8)


# ------------------------------------------------------------------ storage
def pack_nibbles(codes):
    """[rows, cols] codes (cols even) -> [rows, cols / 2] bytes, element 2i low."""
    c = np.asarray(codes, dtype=np.uint8)
    if c.ndim != 2 or c.shape[1] % 2:
        raise ValueError("codes must be [rows, even cols]")
    return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)


def unpack_nibbles(packed):
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty((p.shape[0], 2 * p.shape[1]), dtype=np.uint8)
    out[:, 0::2] = p & 15
    out[:, 1::2] = p >> 4
    return out


# ------------------------------------------------------------ dequantise
def nvfp4_dequantize(packed, scales, tensor_scale):
    """fp64 [rows, cols] weights: tensor_scale x block scale x element."""
    codes = unpack_nibbles(packed)
    rows, cols = codes.shape
    s = np.asarray(scales, dtype=np.uint8)
    if cols % BLOCK or s.shape != (rows, cols // BLOCK):
        raise ValueError("scales must be [rows, cols / 16]")
    block = np.repeat(e4m3_decode(s), BLOCK, axis=1)
    return float(tensor_scale) * block * e2m1_decode(codes)


# ------------------------------------------------------------- quantise
def nvfp4_tensor_scale(w):
    """The smallest power of two at least amax / (6 x 448) (1.0 for an all-zero tensor)."""
    amax = float(np.max(np.abs(w))) if np.size(w) else 0.0
    if amax == 0.0:
        return 1.0
    return float(np.ldexp(1.0, int(np.ceil(np.log2(amax / (E2M1_MAX * E4M3_MAX))))))


def nvfp4_quantize(w, tensor_scale=None):
    """fp64 [rows, cols] (cols a multiple of 16) -> (packed codes, block
    scales, tensor scale): each block's scale is its amax / (6 x tensor
    scale) rounded to E4M3, and each element its value / (tensor scale x
    block scale) rounded to E2M1 (a block whose scale rounds to 0 is all 0)."""
    w = np.asarray(w, dtype=np.float64)
    if w.ndim != 2 or w.shape[1] % BLOCK:
        raise ValueError("weights must be [rows, cols], cols a multiple of 16")
    st = nvfp4_tensor_scale(w) if tensor_scale is None else float(tensor_scale)
    rows, cols = w.shape
    blocks = w.reshape(rows, cols // BLOCK, BLOCK)
    amax = np.max(np.abs(blocks), axis=2)
    scales = e4m3_encode(amax / (E2M1_MAX * st))
    sb = e4m3_decode(scales)
    denom = st * sb[:, :, None]
    x = np.divide(blocks, denom, out=np.zeros_like(blocks), where=denom > 0)
    codes = e2m1_encode(x).reshape(rows, cols)
    return pack_nibbles(codes), scales, st


def nvfp4_to_bf16_bits(packed, scales, tensor_scale):
    """The dequantised weights as bf16 bit patterns (uint16), for the bf16
    oracle.  Every value must be exact in bf16 (true for a power-of-two tensor
    scale); anything else raises, since the bf16 oracle would then see other
    weights than the format holds."""
    w = nvfp4_dequantize(packed, scales, tensor_scale)
    bits32 = w.astype(np.float32).view(np.uint32)
    if not np.array_equal(w.astype(np.float32).astype(np.float64), w) or np.any(bits32 & 0xFFFF):
        raise ValueError("dequantised weights are not exact in bf16")
    return (bits32 >> 16).astype(np.uint16)

