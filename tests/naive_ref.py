"""A second, naive reference for the oracle's pins (test helper).

Written independently of ``oracle/moeact_oracle.c``: every rounding is done
with exact rational arithmetic (``fractions.Fraction``) against an explicit
list of representable values, the sigmoid with ``decimal`` at 60 digits, and
the E8M0 search over exact thresholds.  It is slow (pure Python loops) and is
only used on tiny grids and scalar sweeps.
"""
from __future__ import annotations

import decimal
import functools
import math
import struct
from fractions import Fraction

# ------------------------------------------------------------ fp32 / bf16
F32_MIN_SUB = Fraction(1, 2 ** 149)
F32_MAX = Fraction(2 ** 24 - 1, 2 ** 24) * 2 ** 128


def f32_bits(x: float) -> int:
    return struct.unpack("<I", struct.pack("<f", x))[0]


def f32_from_bits(u: int) -> float:
    return struct.unpack("<f", struct.pack("<I", u & 0xFFFFFFFF))[0]


def bf16_value(b: int) -> float:
    return f32_from_bits((b & 0xFFFF) << 16)


def _round_to_grid(q: Fraction, mant_bits: int, emin: int, max_val: Fraction,
                   overflow_value):
    """Round |q| (exact, >= 0) to the binary format with `mant_bits` stored
    mantissa bits and minimum normal exponent emin; ties to even.
    Returns a Fraction, or `overflow_value` if it rounds past max_val."""
    if q == 0:
        return Fraction(0)
    # exponent of the binade containing q (not below emin: subnormal spacing)
    e = q.numerator.bit_length() - q.denominator.bit_length()
    if Fraction(2) ** e > q:
        e -= 1
    e = max(e, emin)
    ulp = Fraction(2) ** (e - mant_bits)
    k = q / ulp
    fl = math.floor(k)
    rem = k - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    v = fl * ulp
    if v > max_val:
        return overflow_value
    return v


def round_f32(q: Fraction):
    """Exact rational -> nearest fp32 (ties even) as a Python float; +-inf on overflow."""
    sign = -1 if q < 0 else 1
    # IEEE overflow: round with unbounded exponent, then inf if beyond max
    v = _round_to_grid(abs(q), 23, -126, F32_MAX, None)
    if v is None:
        return sign * math.inf
    return sign * float(v) if v != 0 else math.copysign(0.0, sign)


BF16_MAX = Fraction(2 ** 8 - 1, 2 ** 8) * 2 ** 128


def round_bf16_value(x: float) -> float:
    """fp32 value -> nearest bf16 value (ties even), as a Python float."""
    if math.isnan(x):
        return math.nan
    if math.isinf(x):
        return x
    q = Fraction(x)
    sign = -1.0 if math.copysign(1.0, x) < 0 else 1.0
    v = _round_to_grid(abs(q), 7, -126, BF16_MAX, None)
    if v is None:
        return sign * math.inf
    return sign * float(v)


def fmul(a: float, b: float) -> float:
    """fp32 product of two fp32 values (IEEE, RNE)."""
    if math.isnan(a) or math.isnan(b):
        return math.nan
    if math.isinf(a) or math.isinf(b):
        return a * b  # inf*0 -> nan, else +-inf (Python float semantics agree)
    r = round_f32(Fraction(a) * Fraction(b))
    if r == 0:
        return math.copysign(0.0, math.copysign(1.0, a) * math.copysign(1.0, b))
    return r


def fsub(a: float, b: float) -> float:
    if math.isnan(a) or math.isnan(b) or math.isinf(a) or math.isinf(b):
        return a - b
    r = round_f32(Fraction(a) - Fraction(b))
    return r


def ffma(a: float, b: float, c: float) -> float:
    """fp32 fused multiply-add: one rounding of a*b+c."""
    if any(math.isnan(t) or math.isinf(t) for t in (a, b, c)):
        return a * b + c
    r = round_f32(Fraction(a) * Fraction(b) + Fraction(c))
    if r == 0:
        prod_neg = (math.copysign(1.0, a) * math.copysign(1.0, b)) < 0
        if prod_neg and math.copysign(1.0, c) < 0:
            return -0.0
        return 0.0
    return r


# ------------------------------------------------------------ sigmoid
@functools.lru_cache(maxsize=None)
def sigmoid_f32(b: int) -> float:
    """Correctly rounded fp32 sigma of the bf16 value with bit pattern b."""
    g = bf16_value(b)
    if math.isnan(g):
        return math.nan
    if math.isinf(g):
        return 1.0 if g > 0 else 0.0
    # |g| > 200: sigma < e^g < 2^-288 (rounds to +0) or 1 - sigma < e^-g
    # (rounds to 1); decimal's exponent range cannot hold exp(3e38).
    if g < -200:
        return 0.0
    if g > 200:
        return 1.0
    ctx = decimal.Context(prec=60)
    e = ctx.exp(ctx.minus(decimal.Decimal(g)))
    sig = ctx.divide(decimal.Decimal(1), ctx.add(decimal.Decimal(1), e))
    q = Fraction(sig)
    return round_f32(q)


# ------------------------------------------------------------ E4M3 / E8M0
def _e4m3_values():
    vals = []
    for c in range(0x7F):  # non-negative codes, 0x7F is NaN
        e, m = c >> 3, c & 7
        v = Fraction(m, 8) * Fraction(1, 64) if e == 0 else (1 + Fraction(m, 8)) * Fraction(2) ** (e - 7)
        vals.append((v, c))
    return vals


E4M3_VALUES = _e4m3_values()


def e4m3_encode(x) -> int:
    """Nearest E4M3 (ties to the even code), saturate to 448, NaN -> 0x7F.
    x: float or Fraction (exact)."""
    if isinstance(x, float):
        if math.isnan(x):
            return 0x7F
        neg = math.copysign(1.0, x) < 0
        if math.isinf(x):
            return 0xFE if neg else 0x7E
        q = abs(Fraction(x))
    else:
        neg = x < 0
        q = abs(x)
    best = None
    for v, c in E4M3_VALUES:
        d = abs(v - q)
        if best is None or d < best[0] or (d == best[0] and c % 2 == 0):
            best = (d, c)
    return best[1] | (0x80 if neg else 0)


def e8m0(amax: float) -> int:
    if math.isnan(amax):
        return 255
    a = Fraction(abs(amax)) if not math.isinf(amax) else None
    for e in range(-127, 128):
        if a is not None and a <= 448 * Fraction(2) ** e:
            return e + 127
    return 254


def quantize_block(vals):
    """(scale byte, [codes]) of one MXFP8 block of fp32 values."""
    amax = 0.0
    for v in vals:
        if math.isnan(v):
            amax = math.nan
            break
        amax = max(amax, abs(v))
    b = e8m0(amax)
    if b == 255:
        return b, [0x7F] * len(vals)
    mul = Fraction(2) ** (127 - b)
    codes = []
    for v in vals:
        if math.isinf(v):
            codes.append(0xFE if v < 0 else 0x7E)
        else:
            q = Fraction(v) * mul
            c = e4m3_encode(q)
            if q == 0 and math.copysign(1.0, v) < 0:
                c = 0x80
            codes.append(c)
    return b, codes


def mxfp8(y, dirs):
    """y: list of rows (fp32 floats), width W.  Returns dict of nested lists."""
    M = len(y)
    W = len(y[0]) if M else 0
    out = {}
    if dirs & 1:
        rq = [[0] * W for _ in range(M)]
        rs = [[0] * (W // 32) for _ in range(M)]
        for i in range(M):
            for jb in range(W // 32):
                b, cs = quantize_block(y[i][32 * jb:32 * jb + 32])
                rs[i][jb] = b
                rq[i][32 * jb:32 * jb + 32] = cs
        out["row_codes"], out["row_scales"] = rq, rs
    if dirs & 2:
        nb = (M + 31) // 32
        cq = [[0] * W for _ in range(M)]
        cs_ = [[0] * W for _ in range(nb)]
        for ib in range(nb):
            rows = range(32 * ib, min(M, 32 * ib + 32))
            for j in range(W):
                b, cs = quantize_block([y[i][j] for i in rows])
                cs_[ib][j] = b
                for k, i in enumerate(rows):
                    cq[i][j] = cs[k]
        out["col_codes"], out["col_scales"] = cq, cs_
    return out


# ------------------------------------------------------------ the method
def fwd_values(xb, s, N, act="swiglu", staged=False):
    """xb: rows of bf16 bit patterns; s: list of fp32.  Returns fp32 y rows."""
    y = []
    for i, row in enumerate(xb):
        yr = []
        for j in range(N):
            if act == "swiglu":
                g = bf16_value(row[j])
                u = bf16_value(row[N + j])
                silu = fmul(g, sigmoid_f32(row[j]))
                if staged:
                    h = round_bf16_value(fmul(round_bf16_value(silu), u))
                else:
                    h = fmul(silu, u)
            else:
                x = bf16_value(row[j])
                r = x if (x > 0 or math.isnan(x)) else 0.0
                h = fmul(r, r)
            yr.append(fmul(h, s[i]))
        y.append(yr)
    return y


def bwd_values(dyb, xb, s, N, act="swiglu"):
    """Returns (dx rows as bf16-rounded floats, dscale list as fp32)."""
    dx, dsc = [], []
    for i, row in enumerate(xb):
        W = 2 * N if act == "swiglu" else N
        d = [0.0] * W
        acc = Fraction(0)
        nan = False
        for j in range(N):
            gy = bf16_value(dyb[i][j])
            p = fmul(gy, s[i])
            if act == "swiglu":
                g = bf16_value(row[j])
                u = bf16_value(row[N + j])
                sig = sigmoid_f32(row[j])
                silu = fmul(g, sig)
                dsilu = ffma(silu, fsub(1.0, sig), sig)
                d[j] = round_bf16_value(fmul(fmul(p, u), dsilu))
                d[N + j] = round_bf16_value(fmul(p, silu))
                h = fmul(silu, u)
            else:
                x = bf16_value(row[j])
                r = x if (x > 0 or math.isnan(x)) else 0.0
                d[j] = round_bf16_value(fmul(p, fmul(2.0, r)))
                h = fmul(r, r)
            if math.isnan(gy) or math.isnan(h) or math.isinf(gy) or math.isinf(h):
                nan = True
            else:
                acc += Fraction(gy) * Fraction(h)
        dx.append(d)
        dsc.append(math.nan if nan else float(acc))
    return dx, dsc


# ------------------------------------------------------------ ClampedSwiGLU
def fadd(a: float, b: float) -> float:
    return fsub(a, -b)


@functools.lru_cache(maxsize=None)
def sigmoid_of(z: float) -> float:
    """Correctly rounded fp32 sigma of an fp32 value z (decimal, 60 digits)."""
    if math.isnan(z):
        return math.nan
    if math.isinf(z):
        return 1.0 if z > 0 else 0.0
    if z < -200:
        return 0.0
    if z > 200:
        return 1.0
    ctx = decimal.Context(prec=60)
    e = ctx.exp(ctx.minus(decimal.Decimal(z)))
    return round_f32(Fraction(ctx.divide(decimal.Decimal(1), ctx.add(decimal.Decimal(1), e))))


def _clamped_parts(gb, ub, alpha, L):
    g, u = bf16_value(gb), bf16_value(ub)
    gc = L if g > L else g
    uc = L if u > L else (-L if u < -L else u)
    z = fmul(alpha, gc)
    sig = sigmoid_of(z)
    silu = fmul(gc, sig)
    v = fadd(uc, 1.0)
    return g, u, sig, silu, v, fmul(silu, v)


def clamped_fwd_values(xb, s, N, alpha, L):
    return [[fmul(_clamped_parts(row[j], row[N + j], alpha, L)[5], s[i]) for j in range(N)]
            for i, row in enumerate(xb)]


def clamped_bwd_values(dyb, xb, s, N, alpha, L):
    dx, dsc = [], []
    for i, row in enumerate(xb):
        d = [0.0] * (2 * N)
        acc, bad = Fraction(0), False
        for j in range(N):
            g, u, sig, silu, v, h = _clamped_parts(row[j], row[N + j], alpha, L)
            gy = bf16_value(dyb[i][j])
            p = fmul(gy, s[i])
            if not g > L:
                dsilu = ffma(fmul(alpha, silu), fsub(1.0, sig), sig)
                d[j] = round_bf16_value(fmul(fmul(p, v), dsilu))
            if not (u > L or u < -L):
                d[N + j] = round_bf16_value(fmul(p, silu))
            if any(math.isnan(t) or math.isinf(t) for t in (gy, h)):
                bad = True
            else:
                acc += Fraction(gy) * Fraction(h)
        dx.append(d)
        dsc.append(math.nan if bad else float(acc))
    return dx, dsc
