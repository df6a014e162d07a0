"""FP8 (e4m3) quantisation of the softmax branch's q, k, v: a plain CPU
reference.

TEST INFRASTRUCTURE ONLY (see the package docstring).

The pages state only that the fastest configuration runs the model in FP8
(README "Your first render": the tuned fp8 inference script; "Performance
Results": branch-specific Ulysses sequence parallelism and FP8 give 1.4 s
per step on 8 B200). They give no format or scaling. Readings used here:

* Format: e4m3 as defined by the OCP 8-bit floating point specification:
  1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits; exponent field 0
  holds subnormals m * 2^-9; no infinities; the largest finite magnitude is
  1.75 * 2^8 = 448; code 0x7F / 0xFF is NaN.
* Conversion: round to nearest, ties to even, saturating to +-448 (values
  beyond the range become +-448, never NaN).
* Scaling: one fp32 scale per (batch, head) and tensor, scale = amax / 448
  (1 when amax = 0), computed in fp32; the stored code is the conversion of
  the fp32 quotient x / scale, and x is represented by code * scale.

Everything is written from that definition with integer arithmetic on the
exponent and mantissa, so that it shares nothing with the GPU conversion
instructions it is compared against.
"""
import numpy as np

__all__ = ["E4M3_MAX", "e4m3_decode", "e4m3_encode", "quantize_e4m3", "dequantize_e4m3"]

E4M3_MAX = 448.0


def e4m3_decode(codes):
    """Value of each e4m3 code (float64); NaN for 0x7F and 0xFF."""
    c = np.asarray(codes, dtype=np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * 2.0 ** (e - 7))
    val = np.where((c & 0x7F) == 0x7F, np.nan, val)
    return sign * val


def _encode_one(x):
    """e4m3 code of one finite float (round to nearest even, saturating)."""
    sign = 0x80 if (x < 0 or (x == 0 and np.signbit(x))) else 0
    a = abs(float(x))
    if a >= E4M3_MAX:
        return sign | 0x7E
    if a == 0.0:
        return sign
    # exact binary decomposition a = frac * 2^exp, frac in [0.5, 1)
    frac, exp = np.frexp(a)
    # normal numbers of e4m3 have exponent field E in 1..15: a in [2^(E-7), 2^(E-6))
    E = exp - 1 + 7
    if E >= 1:
        # scaled mantissa with 3 fraction bits: a / 2^(E-7) = 1.mmm..., times 8
        t = a / 2.0 ** (E - 7) * 8.0          # exact (power-of-two scaling), in [8, 16)
    else:
        # subnormal: steps of 2^-9
        E = 0
        t = a / 2.0 ** -9                      # exact, in [0, 8)
    q = int(np.floor(t))
    rem = t - q
    if rem > 0.5 or (rem == 0.5 and (q & 1)):
        q += 1
    if E >= 1:
        if q == 16:                             # mantissa overflow: next binade
            q = 8
            E += 1
        m = q - 8
    else:
        if q == 8:                              # rounds up to the smallest normal
            E, m = 1, 0
        else:
            m = q
    if E > 15 or (E == 15 and m == 7):          # beyond 448 (0x7F is NaN): saturate
        return sign | 0x7E
    return sign | (E << 3) | m


def e4m3_encode(x):
    """e4m3 codes (uint8) of an array of finite floats."""
    x = np.asarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint8)
    flat = x.reshape(-1)
    of = out.reshape(-1)
    for i in range(flat.size):
        of[i] = _encode_one(flat[i])
    return out


def quantize_e4m3(x):
    """Per-(b, h) quantisation of x [B, H, L, w] (float32 values, e.g. the
    stored bf16 inputs): returns (codes uint8 [B, H, L, w], scale float32
    [B, H]). The quotient x / scale is formed in float32, as the definition
    above fixes."""
    x = np.asarray(x, dtype=np.float32)
    B, H = x.shape[:2]
    codes = np.empty(x.shape, dtype=np.uint8)
    scale = np.empty((B, H), dtype=np.float32)
    for b in range(B):
        for h in range(H):
            amax = np.float32(np.abs(x[b, h]).max()) if x[b, h].size else np.float32(0)
            s = np.float32(amax / np.float32(E4M3_MAX)) if amax > 0 else np.float32(1.0)
            scale[b, h] = s
            codes[b, h] = e4m3_encode((x[b, h] / s).astype(np.float32))
    return codes, scale


def dequantize_e4m3(codes, scale):
    """float64 values code * scale, scale per (b, h)."""
    return e4m3_decode(codes) * np.asarray(scale, dtype=np.float64)[:, :, None, None]
