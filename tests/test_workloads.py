"""The seeded input generators: encoding positions and rounding (CPU only)."""
import numpy as np
import torch

from block_scaled_precision_nvfp4_b200 import workloads as wl


def test_e2m1_rne_ties_and_saturation():
    t = np.array([0.0, 0.25, 0.26, 0.75, 1.25, 1.3, 1.75, 2.5, 2.6, 3.5, 5.0, 5.1, 100.0,
                  -0.5, -6.0, -0.1], dtype=np.float32)
    expect = [0, 0, 1, 2, 2, 3, 4, 4, 5, 6, 6, 7, 7, 8 | 1, 8 | 7, 0]
    assert wl.e2m1_rne(t).tolist() == expect


def test_quantiser_positions_even_k_low_nibble():
    x = np.zeros((2, 32), dtype=np.float32)
    x[0, 0] = 6.0      # k=0 -> low nibble of byte 0
    x[1, 17] = -6.0    # k=17 -> high nibble of byte 8, group 1
    q = wl.quantize_nvfp4(x)
    assert q.g == np.float32(6.0 / (6 * 448))
    assert q.codes[0, 0] == 0x07 and q.codes[0, 1:].sum() == 0
    assert q.codes[1, 8] == 0xF0 and q.codes[1, :8].sum() == 0
    assert q.scales[0, 0] == 0x7E and q.scales[0, 1] == 0   # 448, then an all-zero group
    assert q.scales[1, 1] == 0x7E and q.scales[1, 0] == 0


def test_quantiser_reconstruction_error_is_small():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((64, 256), dtype=np.float32)
    q = wl.quantize_nvfp4(x)
    tab = np.array([0, .5, 1, 1.5, 2, 3, 4, 6, -0., -.5, -1, -1.5, -2, -3, -4, -6])
    s = torch.from_numpy(q.scales).view(torch.float8_e4m3fn).double().numpy()
    xr = tab[wl.unpack_codes(q.codes)] * s.repeat(16, axis=1) * q.g
    rel = np.linalg.norm(xr - x) / np.linalg.norm(x)
    assert 0.05 < rel < 0.15   # NVFP4 on Gaussian data: ~10% relative error


def test_chunked_quantiser_matches_whole():
    rng = np.random.Generator(np.random.PCG64(3))
    state = rng.bit_generator.state
    q1 = wl.quantize_nvfp4_chunked(rng, 100, 64, 0.02, chunk_rows=7)
    rng.bit_generator.state = state
    x = rng.standard_normal((100, 64), dtype=np.float32) * np.float32(0.02)
    q2 = wl.quantize_nvfp4(x)
    assert np.array_equal(q1.codes, q2.codes) and np.array_equal(q1.scales, q2.scales)
    assert q1.g == q2.g


def test_tiny_workload_recipe():
    t = wl.tiny_w4a4(0)
    assert t.A.codes.shape == (128, 128) and t.W.codes.shape == (256, 128)
    k = (t.A.scales.astype(int) >> 3) - 7
    assert k.min() == -4 and k.max() == 4 and np.all(t.A.scales & 7 == 0)


def test_zipf_routing_counts():
    ids = wl.zipf_routing(8192, 8, 1.1, 2)
    c = np.bincount(ids, minlength=8)
    assert c.sum() == 8192 and np.all(np.diff(c) <= 60) and c[0] > 2 * c[1] * 0.9
    assert c.min() >= 128
