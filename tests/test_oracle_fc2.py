"""Pins of the oracle's activation -> MXFP8 -> FC2 GEMM path (oracle.grouped_fc2).

TransformerEngine PR #3238 (Greptile summary, sequence diagram): the grouped
activation hands its quantized grouped tensor to the grouped linear after it
(ForwardScaledActivationGroupedLinear).  The oracle takes the rowwise MXFP8 of
the scaled SwiGLU (pinned elsewhere) and multiplies its exact values with each
expert's MXFP8 weight.  Pinned here against things other than itself:

* an exact brute force on a tiny grid: every product summed as a Fraction,
  with E4M3 values taken from the format definition (tests/naive_ref.py) and
  the MXFP8 of the activation computed by the naive reference;
* special cases with closed forms: identity weights give back the dequantized
  activation, raising every weight scale by one doubles every output, and
  each expert's rows see only that expert's weight;
* the dequantization of the 256 E4M3 codes against the format definition.
"""
from fractions import Fraction

import numpy as np

import naive_ref as nr
import oracle
from moe_gated_activation_b200.workloads import bf16_bits, random_case


def _weights(E, H, N, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    codes = np.zeros((E, H, N), np.uint8)
    scales = np.zeros((E, H, N // 32), np.uint8)
    for e in range(E):
        w = (rng.standard_normal((H, N)) * scale).astype(np.float32)
        q = oracle.mxfp8_quantize(w, oracle.ROWWISE)
        codes[e], scales[e] = q["row_codes"], q["row_scales"]
    return codes, scales


def test_e4m3_values_match_the_format_definition():
    v = oracle.e4m3_values()
    table = {c: val for val, c in nr.E4M3_VALUES}
    for c in range(256):
        mag = c & 0x7F
        if mag == 0x7F:
            assert np.isnan(v[c])
            continue
        want = float(table[mag]) * (-1.0 if c & 0x80 else 1.0)
        assert v[c] == want and np.signbit(v[c]) == bool(c & 0x80), hex(c)


def test_fc2_equals_an_exact_brute_force_on_a_tiny_grid():
    M, N, H = 5, 64, 3
    case = random_case(M, N, 21, std=1.5)
    xb = bf16_bits(case["x"])
    s = case["s"].numpy()
    row_offs = np.array([0, 2, 5], np.int64)            # two experts: rows 0-1, 2-4
    wc, ws = _weights(2, H, N, 5)
    got = oracle.grouped_fc2(xb, s, N, row_offs, wc, ws)
    # naive reference: the activation and its MXFP8 from naive_ref, then
    # every product as an exact Fraction
    y = nr.fwd_values([list(map(int, r)) for r in xb], list(map(float, s)), N)
    mx = nr.mxfp8(y, 1)
    val = {c: v for v, c in nr.E4M3_VALUES}

    def code_value(c):
        v = val[c & 0x7F]
        return -v if c & 0x80 else v

    for i in range(M):
        e = 0 if i < 2 else 1
        for h in range(H):
            acc = Fraction(0)
            for k in range(N):
                a = code_value(mx["row_codes"][i][k]) * Fraction(2) ** (mx["row_scales"][i][k // 32] - 127)
                w = code_value(int(wc[e, h, k])) * Fraction(2) ** (int(ws[e, h, k // 32]) - 127)
                acc += a * w
            ref = float(acc)
            assert abs(got[i, h] - ref) <= 1e-12 * max(1.0, abs(ref)), (i, h, got[i, h], ref)


def test_identity_weights_give_the_dequantized_activation():
    M, N = 64, 128
    case = random_case(M, N, 22)
    xb, s = bf16_bits(case["x"]), case["s"].numpy()
    eye = np.where(np.eye(N, dtype=bool), 0x38, 0).astype(np.uint8)[None]   # 1.0 on the diagonal
    ws = np.full((1, N, N // 32), 127, np.uint8)
    got = oracle.grouped_fc2(xb, s, N, np.array([0, M], np.int64), eye, ws)
    a = oracle.act_fwd(xb, s, N, oracle.ROWWISE)
    codes, scales = a["row_codes"], a["row_scales"]
    for i in range(0, M, 7):
        for k in range(0, N, 5):
            c = int(codes[i, k])
            v = float(dict((cc, vv) for vv, cc in nr.E4M3_VALUES)[c & 0x7F])
            v = -v if c & 0x80 else v
            assert got[i, k] == v * 2.0 ** (int(scales[i, k // 32]) - 127)


def test_weight_scale_plus_one_doubles_the_output():
    M, N, H = 96, 96, 40
    case = random_case(M, N, 23)
    xb, s = bf16_bits(case["x"]), case["s"].numpy()
    ro = np.array([0, 32, 32, 96], np.int64)          # an empty expert in the middle
    wc, ws = _weights(3, H, N, 7)
    a = oracle.grouped_fc2(xb, s, N, ro, wc, ws)
    b = oracle.grouped_fc2(xb, s, N, ro, wc, ws + 1)
    assert np.array_equal(b, 2 * a)


def test_each_expert_uses_its_own_weight():
    M, N = 64, 64
    case = random_case(M, N, 24)
    xb, s = bf16_bits(case["x"]), case["s"].numpy()
    ro = np.array([0, 16, 48, 64], np.int64)
    eye = np.where(np.eye(N, dtype=bool), 0x38, 0).astype(np.uint8)
    wc = np.stack([eye] * 3)
    ws = np.stack([np.full((N, N // 32), 127 + e, np.uint8) for e in range(3)])   # expert e: 2^e I
    got = oracle.grouped_fc2(xb, s, N, ro, wc, ws)
    a = oracle.mxfp8_dequantize_rows(*(lambda q: (q["row_codes"], q["row_scales"]))(
        oracle.act_fwd(xb, s, N, oracle.ROWWISE)))
    for e in range(3):
        r0, r1 = ro[e], ro[e + 1]
        assert np.array_equal(got[r0:r1], a[r0:r1] * 2.0 ** e)
