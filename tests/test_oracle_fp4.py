"""Pins of the oracle's FP4 (e2m1) indexer-key storage.

* The e2m1 values come out of a generic sign/exponent/mantissa decoder that is
  first checked against two independent implementations of other formats of
  the same family (numpy's float16 for all 65536 codes, torch's float8 e4m3
  for all 256 codes).
* Rounding is checked against a brute-force nearest search over the grid with
  the tie rule (the code whose mantissa bit is 0) and saturation at 6.
* The quantiser is checked through the properties its reading fixes: the
  smallest power-of-two block scale with no saturation, the 8-binade span of a
  row, the all-zero cases, the packing order, and the error bound.
"""
import numpy as np
import pytest
import torch

import oracle


def minifloat(code: int, ebits: int, mbits: int, bias: int, ieee_specials: bool,
              e4m3_nan: bool = False) -> float:
    """Value of a sign / exponent / mantissa code, generic in the widths."""
    s = (code >> (ebits + mbits)) & 1
    e = (code >> mbits) & ((1 << ebits) - 1)
    f = code & ((1 << mbits) - 1)
    emax = (1 << ebits) - 1
    if ieee_specials and e == emax:
        v = float("inf") if f == 0 else float("nan")
    elif e4m3_nan and e == emax and f == (1 << mbits) - 1:
        v = float("nan")
    elif e == 0:
        v = f / (1 << mbits) * 2.0 ** (1 - bias)
    else:
        v = (1 + f / (1 << mbits)) * 2.0 ** (e - bias)
    return -v if s else v


def same(a, b):
    return (np.isnan(a) and np.isnan(b)) or a == b


def test_generic_decoder_matches_float16_and_e4m3():
    codes = np.arange(65536, dtype=np.uint16)
    f16 = codes.view(np.float16).astype(np.float64)
    for c in range(0, 65536, 7):
        assert same(minifloat(c, 5, 10, 15, True), f16[c]), c
    e4 = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64)
    for c in range(256):
        assert same(minifloat(c, 4, 3, 7, False, e4m3_nan=True), float(e4[c])), c


def test_e2m1_values():
    for c in range(16):
        assert oracle.e2m1_value(c) == minifloat(c, 2, 1, 1, False), c
    mags = [oracle.e2m1_value(c) for c in range(8)]
    assert mags == sorted(mags) and len(set(mags)) == 8


def brute_code(x: float) -> int:
    mags = np.array([minifloat(c, 2, 1, 1, False) for c in range(8)])
    a = abs(x)
    d = np.abs(mags - a)
    best = np.nonzero(d == d.min())[0]
    code = int(best[0]) if len(best) == 1 else int([b for b in best if b % 2 == 0][0])
    sign = 8 if (x < 0 or (x == 0 and np.signbit(x))) else 0
    return sign | code


def test_e2m1_rounding_against_brute_force():
    g = np.random.default_rng(1)
    xs = list(g.uniform(-7.5, 7.5, size=3000))
    mags = [minifloat(c, 2, 1, 1, False) for c in range(8)]
    mids = [(mags[i] + mags[i + 1]) / 2 for i in range(7)]     # exact ties
    xs += mids + [-m for m in mids] + [0.0, -0.0, 6.0, 6.5, 100.0, -100.0, 0.25, 0.2500001]
    for x in xs:
        assert oracle.e2m1_code(x) == brute_code(min(max(x, -6.0), 6.0)), x


def _rows(seed):
    g = np.random.default_rng(seed)
    x = g.normal(0.0, 1.0, size=(40, 128))
    x[1] *= 1e3                                   # large
    x[2] *= 1e-5                                  # small
    x[3, 32:64] = 0.0                             # a zero block
    x[4] = 0.0                                    # a zero row
    x[5, 64:96] *= 1e-4                           # a block far below the row's max
    x[6, :32] = 6.0                               # amax exactly 6 * 2^0
    x[7, :32] = 6.0000001                         # just above
    return x


def test_quantize_e2m1_properties():
    x = _rows(2)
    packed, exps = oracle.quantize_e2m1(x)
    assert packed.shape == (40, 64) and exps.shape == (40, 4)
    xf = x.astype(np.float32).astype(np.float64)
    E = exps.astype(np.int64) - 127
    for r in range(x.shape[0]):
        amaxes = np.abs(xf[r].reshape(4, 32)).max(1)
        if (amaxes == 0).all():
            assert (E[r] == 0).all() and (packed[r] == 0).all()
            continue
        top = max(int(np.ceil(np.log2(a / 6.0))) - 1 for a in amaxes if a > 0)
        natural = []
        for b in range(4):
            a = amaxes[b]
            if a == 0:
                natural.append(None)
                continue
            e = E[r, b]
            # the smallest power of two with no saturation ...
            nat = e
            while 6.0 * 2.0 ** (nat - 1) >= a:
                nat -= 1
            while 6.0 * 2.0 ** nat < a:
                nat += 1
            natural.append(nat)
        emax = max(n for n in natural if n is not None)
        assert top <= emax
        for b in range(4):
            want = emax - 8 if natural[b] is None else max(natural[b], emax - 8)
            assert E[r, b] == want, (r, b, E[r, b], want)
        assert E[r].max() - E[r].min() <= 8
        # every code is the brute-force nearest of x / 2^E
        for j in range(128):
            byte = packed[r, j // 2]
            q = (byte >> 4) if j % 2 else (byte & 15)
            y = float(np.float32(xf[r, j]) * np.float32(2.0 ** -E[r, j // 32]))
            assert q == brute_code(min(max(y, -6.0), 6.0)), (r, j)


def test_quantize_e2m1_error_bound_and_packing():
    x = _rows(3)
    packed, exps = oracle.quantize_e2m1(x)
    deq = oracle.dequantize_e2m1(packed, exps)
    E = (exps.astype(np.int64) - 127).repeat(32, axis=1)
    # the widest gap of the grid is 2 (between 4 and 6): half of it at most
    assert (np.abs(deq - x) <= 2.0 ** E * (1.0 + 1e-6)).all()
    # packing: a row of distinct grid values, channel j at a known code
    codes = np.arange(128) % 16
    row = np.array([oracle.e2m1_value(int(c)) for c in codes])[None]
    row[0, 0] = 6.0                                          # every block reaches 6
    row[0, 32] = row[0, 64] = row[0, 96] = 6.0
    p, e = oracle.quantize_e2m1(row)
    assert (e == 127).all()
    d = oracle.dequantize_e2m1(p, e)
    np.testing.assert_array_equal(d, row)
    assert p[0, 1] == (int(codes[3]) << 4) | int(codes[2])
