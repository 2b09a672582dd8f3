"""Comparison rule shared by the GPU parity tests.

Tolerance (from the matmul's specification): against the FP64 oracle value
(not its BF16 rounding), relative Frobenius error <= 2e-3 and per-element
|err| <= 1e-2 * max|ref|.  BF16 output rounding alone contributes ~1.5e-3 of
relative Frobenius error; FP32 accumulation adds ~1e-6.  Guards against
vacuous passes: the reference must be non-empty, finite and non-zero, the
result finite, and both the same size.
"""
import numpy as np

REL_FRO_TOL = 2e-3
MAX_ABS_REL_TOL = 1e-2


def bf16_to_f64(t) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def check(y, ref, what=""):
    y = np.asarray(y, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert y.shape == ref.shape, f"{what}: shape {y.shape} != {ref.shape}"
    assert ref.size > 0, f"{what}: empty comparison"
    assert np.all(np.isfinite(ref)), f"{what}: non-finite reference"
    assert np.all(np.isfinite(y)), f"{what}: non-finite result ({np.sum(~np.isfinite(y))} values)"
    nref = np.linalg.norm(ref)
    assert nref > 0, f"{what}: all-zero reference"
    rel = np.linalg.norm(y - ref) / nref
    mx = np.max(np.abs(y - ref)) / np.max(np.abs(ref))
    assert rel <= REL_FRO_TOL, f"{what}: relative Frobenius error {rel:.3e} > {REL_FRO_TOL}"
    assert mx <= MAX_ABS_REL_TOL, f"{what}: max |err|/max|ref| {mx:.3e} > {MAX_ABS_REL_TOL}"
    return rel, mx


def packed_reference(s, K):
    """The MMA scale layout restated: packed[rb][ks][i][j][t] = s[rb*128 + 32j + i][4ks + t],
    zero rows past the end (numpy reshapes only)."""
    rows = s.shape[0]
    rb_n = (rows + 127) // 128
    pad = np.zeros((rb_n * 128, K // 16), np.uint8)
    pad[:rows] = s
    v = pad.reshape(rb_n, 4, 32, K // 64, 4)          # [rb][j][i][ks][t]
    return np.ascontiguousarray(v.transpose(0, 3, 2, 1, 4)).ravel()  # [rb][ks][i][j][t]


class Accum:
    """check() for a result compared in pieces: the same tolerances, on the whole.

    add(y, ref) takes one piece; finish(count) asserts that exactly `count` elements
    were compared and that the relative Frobenius error and max |err| / max |ref| of
    the whole result are within REL_FRO_TOL and MAX_ABS_REL_TOL."""

    def __init__(self, what=""):
        self.what = what
        self.n = 0
        self.err2 = 0.0
        self.ref2 = 0.0
        self.max_err = 0.0
        self.max_ref = 0.0

    def add(self, y, ref):
        y = np.asarray(y, dtype=np.float64)
        ref = np.asarray(ref, dtype=np.float64)
        assert y.shape == ref.shape, f"{self.what}: shape {y.shape} != {ref.shape}"
        assert np.all(np.isfinite(ref)), f"{self.what}: non-finite reference"
        assert np.all(np.isfinite(y)), f"{self.what}: non-finite result"
        d = y - ref
        self.n += y.size
        self.err2 += float(np.sum(d * d))
        self.ref2 += float(np.sum(ref * ref))
        if y.size:
            self.max_err = max(self.max_err, float(np.max(np.abs(d))))
            self.max_ref = max(self.max_ref, float(np.max(np.abs(ref))))

    def finish(self, count):
        assert self.n == count, f"{self.what}: compared {self.n} elements, expected {count}"
        assert self.n > 0 and self.ref2 > 0, f"{self.what}: empty or all-zero reference"
        rel = np.sqrt(self.err2 / self.ref2)
        mx = self.max_err / self.max_ref
        assert rel <= REL_FRO_TOL, f"{self.what}: relative Frobenius error {rel:.3e} > {REL_FRO_TOL}"
        assert mx <= MAX_ABS_REL_TOL, f"{self.what}: max |err|/max|ref| {mx:.3e} > {MAX_ABS_REL_TOL}"
        return rel, mx
