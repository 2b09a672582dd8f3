"""The golden fixtures of tests/golden/ against the oracle and independent decoders.

page1_identity_constants.txt holds the constants page 1 prints for the exact
E2M1 -> E4M3 conversion; e2m1_identity.txt and tiny_w4a4_y_x1024.txt were written
by tests/golden/make_golden.py from the oracle alone, and are checked here
against what does not come from the oracle (torch's float8 decoder, the OCP E2M1
field formula, integer arithmetic)."""
import hashlib
import os

import numpy as np
import torch

import oracle
from block_scaled_precision_nvfp4_b200 import workloads as wl

GOLD = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _kv(name):
    out = {}
    for ln in open(os.path.join(GOLD, name)):
        if ln.strip() and not ln.startswith("#"):
            k, v = ln.split()
            out[k] = int(v, 0)
    return out


def _e2m1_field(c):
    """OCP E2M1 from its fields: sign, 2-bit exponent (bias 1), 1-bit mantissa."""
    s, e, m = c >> 3, (c >> 1) & 3, c & 1
    mag = 0.5 * m if e == 0 else 2.0 ** (e - 1) * (1 + m / 2)
    return -mag if s else mag


def _e4m3_torch(b):
    return float(torch.tensor([b], dtype=torch.uint8).view(torch.float8_e4m3fn).float())


def test_page1_constants_give_value_times_2_to_the_exponent_for_all_codes():
    k = _kv("page1_identity_constants.txt")
    assert k["codes"] == 16
    for c in range(16):
        q = (c << 4) * 0x01010101                         # the code in all four high nibbles
        r = (q & k["sign_mask"]) | ((q & k["field_mask"]) >> k["field_shift"])
        for j in range(4):
            b = (r >> (8 * j)) & 0xFF
            assert _e4m3_torch(b) == _e2m1_field(c) * 2.0 ** k["value_exponent"]
        assert oracle.e2m1_to_e4m3_word(q) == r            # the oracle applies exactly that


def test_identity_table_fixture():
    rows = [ln.split() for ln in open(os.path.join(GOLD, "e2m1_identity.txt")) if not ln.startswith("#")]
    assert len(rows) == 16
    for c, (code, byte, v2, v4) in enumerate(rows):
        assert int(code) == c
        b = int(byte, 16)
        assert float(v2) == _e2m1_field(c) and float(v4) == _e4m3_torch(b)
        assert float(v4) == float(v2) * 2.0 ** -6


def test_tiny_workload_fixture():
    lines = [ln.split() for ln in open(os.path.join(GOLD, "tiny_w4a4_y_x1024.txt")) if not ln.startswith("#")]
    digest = lines[0][1]
    t = wl.tiny_w4a4(0)
    Y = oracle.gemm_w4a4(t.A.codes, t.A.scales, 1.0, t.W.codes, t.W.scales, 1.0, t.M, t.N, t.K)
    Yi = Y * 1024.0
    assert np.array_equal(Yi, np.round(Yi))
    Yi = Yi.astype(np.int64)
    assert hashlib.sha256(np.ascontiguousarray(Yi).tobytes()).hexdigest() == digest
    # the sampled entries by plain integer arithmetic on the decoded codes and scale exponents
    codes_a = wl.unpack_codes(t.A.codes).astype(np.int64)
    codes_w = wl.unpack_codes(t.W.codes).astype(np.int64)
    twice = np.array([int(2 * _e2m1_field(c)) for c in range(16)], dtype=np.int64)   # 2*value
    ka = (t.A.scales.astype(np.int64) >> 3) - 7                                     # 2^k scales
    kw = (t.W.scales.astype(np.int64) >> 3) - 7
    for r, c, v in ((int(a), int(b), int(x)) for a, b, x in lines[1:]):
        tot = 0
        for g in range(t.K // 16):
            s = int(np.sum(twice[codes_a[r, 16 * g:16 * g + 16]] * twice[codes_w[c, 16 * g:16 * g + 16]]))
            tot += s << (ka[r, g] + kw[c, g] + 8)       # (a*w)*4 * 2^(ka+kw) * 2^10 / 4
        assert tot == v
