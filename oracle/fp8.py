"""FP8 (e4m3) oracle -- TEST INFRASTRUCTURE ONLY (numpy, float64).

The pages run Flide with FP8 weights and activations where the hardware has
them (techfi24.com, "Exact State Forking": the kernel uses FP8 when
available; "Performances": a 35B model quantised to FP8).  They name no FP8
encoding or scaling scheme.  Reading used here: the e4m3 format of the OCP
8-bit floating point specification (1 sign, 4 exponent bits with bias 7, 3
mantissa bits, no infinities, S.1111.111 is NaN, largest finite value 448),
one scale per tensor (its absolute maximum maps to 448), round to nearest
even with saturation to +-448; attention then runs on the decoded values.

Functions:
  decode_e4m3(codes)          e4m3 code -> exact value (float64)
  encode_e4m3(y)              exact value -> nearest e4m3 code (RNE, saturating)
  quantize_e4m3(x, amax=None) per-tensor quantisation in the float32 steps
                              inv = 448 / amax, y = x * inv, code = e4m3(y);
                              descale = amax / 448 (amax 0: inv = descale = 1)
  gdn_fp8(...)                Gated DeltaNet fork scan over decoded fp8 q, k, v
                              (sq Q, sk K, sv V) with the given gates and
                              states; the delta rule is not linear in k, so the
                              decoded values times the descale factors are
                              formed in float32 (exact for power-of-two
                              factors, as the tests use) and handed to the
                              fp64 GDN oracle
  attention_fp8(...)          fork attention over decoded fp8 inputs: with
                              q = sq Q, k = sk K, v = sv V (Q, K, V the decoded
                              codes) the attention of (q, k, v) at softmax
                              scale c equals sv times the attention of
                              (Q, K, V) at scale c sq sk -- exact linearity, so
                              the fp64 attention oracle is reused unchanged.

Pins: ``tests/test_fp8_oracle.py``.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0


def decode_e4m3(codes) -> np.ndarray:
    """Values of e4m3 codes (uint8) as float64; NaN for the two NaN codes."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c >> 7, -1.0, 1.0)
    e = (c >> 3) & 15
    m = (c & 7).astype(np.float64)
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & ((c & 7) == 7), np.nan, mag)
    return sign * mag


def encode_e4m3(y) -> np.ndarray:
    """Nearest e4m3 code of each value (round half to even, magnitudes above
    448 saturate to 448, NaN -> 0x7F with the sign bit)."""
    y = np.asarray(y, dtype=np.float64)
    neg = np.signbit(y)
    a = np.abs(y)
    out = np.zeros(y.shape, np.int64)
    sub = a < 2.0 ** -6
    # subnormals (and zero): multiples of 2^-9; a rounded value of 8 is the
    # smallest normal 2^-6, whose code is also 8
    out[sub] = np.rint(a[sub] * 2.0 ** 9).astype(np.int64)
    nrm = ~sub & ~np.isnan(a)
    if nrm.any():
        an = np.minimum(a[nrm], 2.0 ** 10)  # keep exponents bounded; saturated below
        _, ex = np.frexp(an)                # an = f 2^ex, f in [0.5, 1)
        e = ex - 1                          # an in [2^e, 2^(e+1))
        m = np.rint(an * np.exp2(3.0 - e)).astype(np.int64)  # in [8, 16]
        carry = m == 16
        e = np.where(carry, e + 1, e)
        m = np.where(carry, 8, m)
        code = ((e + 7) << 3) | (m - 8)
        out[nrm] = np.where((e > 8) | ((e == 8) & (m == 15)), 0x7E, code)
    out[np.isnan(a)] = 0x7F
    out = np.where(neg, out | 0x80, out)
    return out.astype(np.uint8)


def quantize_e4m3(x, amax=None):
    """Per-tensor e4m3 quantisation of x (float32 or bf16-valued array).

    amax: the absolute maximum the scale is taken from (default: of x itself;
    a larger value lets several tensors share one scale).  The scaling steps
    are float32 operations, so a device implementation that rounds the same
    way gives the same codes.  Returns (codes uint8, descale float32)."""
    x = np.asarray(x, dtype=np.float32)
    a = np.float32(np.max(np.abs(x))) if amax is None else np.float32(amax)
    if a == 0:
        inv = np.float32(1.0)
        descale = np.float32(1.0)
    else:
        inv = np.float32(E4M3_MAX) / a
        descale = a / np.float32(E4M3_MAX)
    y = (x * inv).astype(np.float32)
    return encode_e4m3(y.astype(np.float64)), np.float32(descale)


def attention_fp8(tree, q8, k8, v8, pk8, pv8, descale, scale, rows=None):
    """Fork attention over e4m3 inputs with per-tensor descale factors
    (sq, sk, sv); past K/V rows use sk and sv.  Returns float64 [T, Hq, d]
    (or [n, d] for the (token, head) pairs in ``rows``)."""
    from . import attention_all, attention_rows
    sq, sk, sv = (float(s) for s in descale)
    dec = lambda a: None if a is None else decode_e4m3(a).astype(np.float32)  # exact
    Q, K, V, PK, PV = dec(q8), dec(k8), dec(v8), dec(pk8), dec(pv8)
    c = float(scale) * sq * sk
    if rows is None:
        return sv * attention_all(tree, Q, K, V, PK, PV, c)
    return sv * attention_rows(tree, Q, K, V, PK, PV, c, rows)


def gdn_fp8(tree, q8, k8, v8, g, beta, descale, state_in=None, pairs=None):
    """Gated DeltaNet fork scan over e4m3 q, k, v with descale factors
    (sq, sk, sv): float64 [T, H, dv] (zeros outside ``pairs``)."""
    from . import gdn
    sq, sk, sv = (np.float32(s) for s in descale)
    dq = lambda a, s: (decode_e4m3(a).astype(np.float32) * s).astype(np.float32)
    return gdn(tree, dq(q8, sq), dq(k8, sk), dq(v8, sv), np.asarray(g, np.float32),
               np.asarray(beta, np.float32), state_in=state_in, pairs=pairs)
