"""Pins of the oracle's MXFP8 / NVFP4 decoders and quantisers against the
format definitions (OCP Microscaling E4M3 / E8M0 / E2M1)."""
import numpy as np
import pytest

from oracle import quant as q

rng = np.random.default_rng(7)


def test_e4m3_spec_values():
    cases = {0x00: 0.0, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6,
             0x38: 1.0, 0x3C: 1.5, 0x40: 2.0, 0x7E: 448.0, 0xFE: -448.0,
             0xB8: -1.0, 0x80: -0.0}
    for c, v in cases.items():
        assert q.e4m3_decode(c) == v, hex(c)
    assert np.isnan(q.e4m3_decode(0x7F)) and np.isnan(q.e4m3_decode(0xFF))
    finite = q.e4m3_decode(np.arange(0x7F))
    assert np.all(np.diff(finite) > 0)                    # monotone codes


def test_e8m0_and_e2m1_spec_values():
    assert q.e8m0_decode(0x7F) == 1.0
    assert q.e8m0_decode(0x80) == 2.0 and q.e8m0_decode(0x7E) == 0.5
    assert q.e8m0_decode(0) == 2.0 ** -127 and np.isnan(q.e8m0_decode(0xFF))
    assert list(q.e2m1_decode(np.arange(8))) == [0, 0.5, 1, 1.5, 2, 3, 4, 6]
    assert list(q.e2m1_decode(np.arange(8, 16))) == [-0.0, -0.5, -1, -1.5,
                                                    -2, -3, -4, -6]


def test_rounding_exact_ties_and_saturation():
    vals = q.e4m3_decode(np.arange(0x7F))
    assert np.array_equal(q.e4m3_decode(q.round_e4m3(vals)), vals)
    # 1.0625 lies halfway between 1.0 (0x38, even) and 1.125 (0x39)
    assert q.round_e4m3(1.0625) == 0x38
    assert q.round_e4m3(1.1875) == 0x3A                   # tie -> even 1.25
    assert q.round_e4m3(1000.0) == 0x7E and q.round_e4m3(-1e6) == 0xFE
    assert q.round_e2m1(2.5) == 0x4 and q.round_e2m1(5.0) == 0x6   # ties even
    assert q.round_e2m1(0.25) == 0x0 and q.round_e2m1(7.5) == 0x7
    assert q.round_e2m1(-0.8) == 0x8 | 0x2


def test_mxfp8_roundtrip_and_error_bound():
    w = rng.standard_normal((6, 64))
    codes, e = q.quant_mxfp8(w)
    wd = q.dequant_mxfp8(codes, e)
    assert np.array_equal(q.dequant_mxfp8(*q.quant_mxfp8(wd)), wd)
    # E4M3 RNE: error <= half a unit in the last place (top binade [256, 448]
    # has ulp 32, so <= 16 * 2^e); magnitudes above 448 * 2^e clip to 448 * 2^e
    sc = q.e8m0_decode(e)[..., None]
    err = np.abs(wd - w).reshape(6, 2, 32)
    a = np.abs(w).reshape(6, 2, 32)
    inside = a <= 448 * sc
    assert np.all(err[inside] <= np.broadcast_to(16 * sc, a.shape)[inside])
    assert np.all(err[~inside] <= (a - 448 * sc)[~inside] + 1e-15)
    # largest element lands in [256, 448] * 2^e  (max scaling)
    top = (codes & 0x7F).reshape(6, 2, 32).max(-1)
    assert np.all(q.e4m3_decode(top) >= 256)
    assert np.all(q.e8m0_decode(q.quant_mxfp8(np.zeros((1, 32)))[1]) == 2.0 ** -127)


def test_nvfp4_roundtrip_and_packing():
    w = rng.standard_normal((4, 64)) * 0.03
    packed, sb, S = q.quant_nvfp4(w)
    assert packed.shape == (4, 32) and sb.shape == (4, 4)
    codes = q.unpack_nvfp4(packed)
    assert np.array_equal(codes[:, 0], packed[:, 0] & 0xF)
    assert np.array_equal(codes[:, 1], packed[:, 0] >> 4)
    wd = q.dequant_nvfp4(packed, sb, S)
    blk = np.abs(w).reshape(4, 4, 16).max(-1)
    # worst-case E2M1 step is 2 (between 4 and 6); half of it relative to 6
    assert np.all(np.abs(wd - w).reshape(4, 4, 16)
                  <= blk[..., None] * (1.0 / 6.0) * 1.0 + 1e-12)
    p2, sb2, S2 = q.quant_nvfp4(wd)
    assert np.allclose(q.dequant_nvfp4(p2, sb2, S2), wd, rtol=0, atol=1e-12)


@pytest.mark.parametrize("fmt", ["mxfp8", "nvfp4"])
def test_decoded_products_exact_in_bf16(fmt):
    """e4m3*2^e and e2m1*e4m3 have <= 8 significant bits: exact in BF16."""
    w = rng.standard_normal((8, 64)) * 0.05
    if fmt == "mxfp8":
        wd = q.dequant_mxfp8(*q.quant_mxfp8(w))
    else:
        p, sb, _ = q.quant_nvfp4(w)
        wd = q.dequant_nvfp4(p, sb)
    f = wd.astype(np.float32)
    assert np.array_equal(f.astype(np.float64), wd)
    assert np.all((f.view(np.uint32) & 0xFFFF) == 0)


def test_nvfp4_mse_scales_never_worse_than_max_scaling():
    """Per block, the MSE-selected scale's squared error is at most that of
    the max-scaling scale (which is among the candidates), and strictly
    smaller somewhere on Gaussian weights."""
    w = rng.standard_normal((16, 128)) * 0.04
    pm, sm, Sm = q.quant_nvfp4(w)
    pe, se, Se = q.quant_nvfp4_mse(w)
    assert Sm == Se
    em = ((q.dequant_nvfp4(pm, sm, Sm) - w) ** 2).reshape(16, 8, 16).sum(-1)
    ee = ((q.dequant_nvfp4(pe, se, Se) - w) ** 2).reshape(16, 8, 16).sum(-1)
    assert np.all(ee <= em + 1e-18)
    assert np.any(ee < em * 0.99)


def test_nvfp4_mse_matches_scalar_search():
    """Brute force, one block at a time in scalar Python: try every code of
    the window around the max-scaling code, decode, keep the smallest sum of
    squared errors (first found among codes taken from high to low)."""
    w = rng.standard_normal((3, 48)) * 0.05
    _, sb, S = q.quant_nvfp4_mse(w)
    S = float(S)
    e2 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    for r in range(3):
        for b in range(3):
            blk = [float(v) for v in w[r, 16 * b:16 * b + 16]]
            c_max = int(q.round_e4m3(max(abs(v) for v in blk) / (6 * S)))
            best, best_err = None, None
            for c in range(min(126, c_max + 1), max(1, c_max - 8) - 1, -1):
                sc = float(q.e4m3_decode(c)) * S
                err = 0.0
                for v in blk:
                    y = abs(v) / sc
                    # nearest E2M1 magnitude, ties to the even code
                    d = [abs(y - m) for m in e2]
                    k = min(range(8), key=lambda i: (d[i], i % 2))
                    if y >= 6.0:
                        k = 7
                    err += (abs(v) - e2[k] * sc) ** 2
                if best_err is None or err < best_err:
                    best, best_err = c, err
            assert sb[r, b] == best, (r, b, sb[r, b], best)


def test_nvfp4_mse_exact_block_has_zero_error():
    """A block of E2M1 values (largest magnitude 6) times the scale of code
    0x30 (0.5) and the tensor scale S = 2^-10 (fixed by a tensor maximum of
    6 * 448 * 2^-10 in the other block) is reproduced exactly: the search
    keeps the max-scaling code 0x30, whose error is 0."""
    vals = np.array([0.5, -1.0, 1.5, 2.0, -3.0, 4.0, 0.0, 6.0] * 2)
    S0 = 2.0 ** -10
    w = np.zeros((1, 32))
    w[0, :16] = vals * 0.5 * S0
    w[0, 16] = 6.0 * 448.0 * S0
    p, sb, S = q.quant_nvfp4_mse(w)
    assert float(S) == S0 and sb[0, 0] == 0x30
    assert np.array_equal(q.dequant_nvfp4(p, sb, S)[0, :16], w[0, :16])
