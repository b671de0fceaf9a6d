"""Pins of the oracle's quantizer and packing: hand-worked bytes, grid inputs
that must round-trip exactly, the half-step error bound, degenerate blocks,
identity-gauge reduction and the bits/value closed form."""
import os

import numpy as np
import pytest

from oracle import codec as oc
from oracle import gauge as og
from oracle import quant as oq
from oracle.fpround import fl16, fl32, fl_bf16
from oracle.metrics import bits_per_value

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "packing.txt")


def _golden_rows():
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        b, codes, hexbytes = [p.strip() for p in line.split(";")]
        yield int(b), [int(c) for c in codes.split()], bytes.fromhex(hexbytes.replace(" ", ""))


@pytest.mark.parametrize("bits,codes,want", list(_golden_rows()))
def test_packing_golden(bits, codes, want):
    got = oq.pack_codes(np.array(codes), bits)
    assert bytes(got.tolist()) == want
    assert oq.unpack_codes(got, bits, len(codes)).tolist() == codes


@pytest.mark.parametrize("bits", [2, 3, 4, 6, 8])
def test_pack_unpack_round_trip(bits):
    q = np.random.default_rng(bits).integers(0, 2 ** bits, (5, 7, 256))
    p = oq.pack_codes(q, bits)
    assert p.shape == (5, 7, 256 * bits // 8)
    assert np.array_equal(oq.unpack_codes(p, bits, 256), q)


@pytest.mark.parametrize("bits", [3, 4, 6])
def test_grid_inputs_round_trip_exactly(bits):
    # y = z + k s with z, s exact in fp16 and k in [0, 2^b - 1] covering both ends:
    # the block min is z and the range is s (2^b - 1), so the step is exactly s.
    rng = np.random.default_rng(bits)
    qmax = 2 ** bits - 1
    checked = 0
    for _ in range(50):
        z = float(fl16(rng.normal(0, 4)))
        s = float(fl16(abs(rng.normal(0, 0.5)) + 1e-3))
        k = rng.integers(0, qmax + 1, 256)
        k[0], k[1] = 0, qmax
        y = z + k * s
        assert np.array_equal(fl32(y), y)          # exactly representable
        q, zz, ss = oq.quantize_ranges(y[None], bits)
        if fl32(fl32(y.max() - y.min()) / qmax) != s:
            continue                                # s itself not recovered exactly: skip
        assert zz[0] == z and ss[0] == s
        assert np.array_equal(q[0], k)
        assert np.array_equal(oq.dequantize(q[0], z, s), y)
        checked += 1
    assert checked >= 25


@pytest.mark.parametrize("bits", [3, 4, 6])
def test_error_within_half_step(bits):
    y = fl32(np.random.default_rng(9).standard_normal((400, 256)) * 3)
    q, z, s = oq.quantize_ranges(y, bits)
    err = np.abs(oq.dequantize(q, z[:, None], s[:, None]) - y)
    # half a step, plus what the fp16 rounding of z and s can push out of range
    qmax = 2 ** bits - 1
    slack = np.abs(y.min(-1) - z) + qmax * np.abs(fl32((y.max(-1) - y.min(-1)) / qmax) - s)
    assert np.all(err <= (s / 2 * (1 + 1e-6) + slack)[:, None] + 1e-12)
    assert q.min() == 0 and q.max() == qmax


def test_constant_and_tiny_blocks():
    y = np.full((1, 256), 1.2345678, dtype=np.float64)
    y = fl32(y)
    q, z, s = oq.quantize_ranges(y, 4)
    assert s[0] == 0 and np.all(q == 0) and z[0] == fl16(y[0, 0])
    y2 = fl32(np.linspace(0, 2.0 ** -26, 256))[None]  # range so small that s rounds to 0 in fp16
    q2, z2, s2 = oq.quantize_ranges(y2, 4)
    assert s2[0] == 0 and np.all(q2 == 0)


def test_rne_ties_go_to_even():
    # z = 0, s = 1: t = y exactly; 0.5 -> 0, 1.5 -> 2, 2.5 -> 2
    y = np.array([[0.0, 0.5, 1.5, 2.5, 15.0]])
    q = oq.quantize(y, 0.0, 1.0, 4)
    assert q.tolist() == [[0, 0, 2, 2, 15]]


def test_identity_gauge_is_plain_quantizer():
    rng = np.random.default_rng(5)
    x = fl_bf16(rng.standard_normal((1, 2, 1, 2, 64, 32)) * 2)
    G = np.broadcast_to(np.eye(16), (1, 2, 2, 2, 16, 16))
    enc = oc.encode_block_uniform(x, G, 4, tb=16, w=16)
    q, z, s = oq.quantize_ranges(oq.block_uniform_view(x, 16, 16), 4)
    assert np.array_equal(enc["q"], q) and np.array_equal(enc["z"], z) and np.array_equal(enc["s"], s)


def test_block_view_orders_tokens_major():
    y = np.arange(32 * 32, dtype=np.float64).reshape(32, 32)
    v = oq.block_uniform_view(y, 16, 16)
    assert v.shape == (2, 2, 256)
    assert v[1, 0, 0] == y[16, 0] and v[1, 0, 1] == y[16, 1] and v[1, 0, 16] == y[17, 0]
    assert v[0, 1, 0] == y[0, 16]
    assert np.array_equal(oq.block_uniform_unview(v, 16, 16), y)
    k = oq.kivi_key_view(y, 16)
    assert k.shape == (2, 32, 16) and k[1, 3, 2] == y[18, 3]
    vv = oq.kivi_value_view(y, 16)
    assert vv.shape == (32, 2, 16) and vv[5, 1, 2] == y[5, 18]


@pytest.mark.parametrize("bits,w", [(3, 16), (4, 16), (6, 16), (4, 128), (3, 128)])
def test_bits_per_value_closed_form(bits, w):
    L, B, H, T, d = 2, 1, 2, 64, 128
    cb, sc = oc.sizes(L, B, H, T, d, bits, tb=16, w=w)
    n = L * 2 * B * H * T * d
    assert bits_per_value(cb, sc, n) == pytest.approx(bits + 32.0 / (16 * w), rel=1e-15)
    x = fl_bf16(np.random.default_rng(0).standard_normal((L, 2, B, H, T, d)))
    G = np.broadcast_to(np.eye(16), (L, 2, H, d // 16, 16, 16))
    enc = oc.encode_block_uniform(x, G, bits, tb=16, w=w)
    assert enc["codes"].size == cb and enc["z"].size == sc


def test_kivi_sizes_and_round_trip_error():
    rng = np.random.default_rng(6)
    x = fl_bf16(rng.standard_normal((1, 2, 1, 2, 64, 64)))
    G = og.gauge_from_A(rng.normal(0, 0.1, (1, 2, 2, 4, 16, 16)))
    G32 = fl32(G)
    enc = oc.encode_kivi(x, G32, 3)
    cb, sc = oc.sizes(1, 1, 2, 64, 64, 3, mode="kivi")
    assert enc["key"]["codes"].size + enc["value"]["codes"].size == cb
    assert enc["key"]["z"].size + enc["value"]["z"].size == sc
    xr = oc.decode_kivi(enc, G32, 3)
    rel = np.sqrt(((xr - x) ** 2).sum() / (x ** 2).sum())
    assert 0.01 < rel < 0.2


def test_zero_extremes_are_positive_zero():
    """-0 and +0 are one real number: a block whose minimum (or whole range) is
    zero stores the fp16 +0 as its zero point and step, whichever zero the
    values carry and in whatever order they come."""
    for blk in ([-0.0, 0.0, 1.0], [0.0, -0.0, 1.0], [-0.0, 2.0], [-0.0, -0.0], [0.0, -0.0]):
        q, z, s = oq.quantize_ranges(np.array([blk]), 4)
        assert np.signbit(z).sum() == 0 and np.signbit(s).sum() == 0, blk
        assert np.asarray(z, np.float16).view(np.uint16)[0] == 0
    # a negative minimum keeps its sign, and a non-zero block is unchanged
    q, z, s = oq.quantize_ranges(np.array([[-0.5, 1.0]]), 4)
    assert z[0] == -0.5 and s[0] == fl16(fl32(1.5 / 15))


def test_saturation_at_fp16_range():
    """Ranges beyond fp16: the zero point clamps to -65504 (fp16's largest finite
    magnitude), the step to 65504, and the codes then saturate.  Worked by hand at
    4 bits (qmax 15): block [-1e6, 1e6] has fl32(2e6 / 15) = 133333.33 > 65504, so
    z = -65504, s = 65504, inv = fl32(1 / 65504); -1e6 gives t < 0 -> 0, 1e6 gives
    t = (1e6 + 65504) / 65504 = 16.27 -> 15, and 0 gives t = 1.0 -> 1."""
    q, z, s = oq.quantize_ranges(np.array([[-1e6, 1e6, 0.0]]), 4)
    assert z[0] == -65504.0 and s[0] == 65504.0
    assert list(q[0]) == [0, 15, 1]
    # a minimum below the range, a step inside it: z clamps, s does not
    q, z, s = oq.quantize_ranges(np.array([[-70000.0, -69970.0]]), 4)
    assert z[0] == -65504.0 and s[0] == fl16(fl32(30.0 / 15.0)) == 2.0
    assert list(q[0]) == [0, 0]  # both below z: t < 0
    # the largest step that is not clamped: (mx - mn) / 15 exactly 65504
    q, z, s = oq.quantize_ranges(np.array([[0.0, 65504.0 * 15]]), 4)
    assert z[0] == 0.0 and s[0] == 65504.0 and list(q[0]) == [0, 15]


def test_metrics_hand_values():
    """nrmse = ||x - xhat|| / ||x||, mse = mean squared error, max_abs, and bits/value
    = 8 (code bytes + 4 bytes of fp16 step and zero per range) / values, on values
    worked by hand."""
    from oracle import metrics as om
    x, xh = np.array([3.0, 4.0]), np.array([3.0, 0.0])
    assert om.nrmse(x, xh) == 0.8          # sqrt(16) / sqrt(25)
    assert om.mse(x, xh) == 8.0            # (0 + 16) / 2
    assert om.max_abs(x, xh) == 4.0
    assert om.nrmse(np.zeros(3), np.ones(3)) == 0.0  # zero reference: defined as 0
    # 4 bits, 16 x 16 ranges: 128 code bytes and one range per 256 values -> 4.125
    assert om.bits_per_value(128, 1, 256) == 4.125


def test_kivi_views_by_index():
    """kivi_key_view puts token 32 g + i of channel c at [g, c, i]; kivi_value_view puts
    channel 32 g + i of token t at [t, g, i]; both unviews invert them exactly
    (values that encode their own (t, c) index)."""
    T, d = 64, 64
    t = np.arange(T)[:, None]
    c = np.arange(d)[None, :]
    y = (1000 * t + c).astype(np.float64)[None]      # [1, T, d]
    kv = oq.kivi_key_view(y, 32)                       # [1, T/32, d, 32]
    assert kv.shape == (1, 2, 64, 32)
    assert kv[0, 1, 5, 7] == 1000 * (32 + 7) + 5
    assert kv[0, 0, 63, 31] == 1000 * 31 + 63
    vv = oq.kivi_value_view(y, 32)                     # [1, T, d/32, 32]
    assert vv.shape == (1, 64, 2, 32)
    assert vv[0, 10, 1, 3] == 1000 * 10 + 32 + 3
    assert np.array_equal(oq.kivi_key_unview(kv), y) and np.array_equal(oq.kivi_value_unview(vv), y)


def test_kivi_exact_grid_encode_decode():
    """An identity gauge on inputs whose ranges are exact grids: every key channel's 32
    tokens take the values 0..7 (3 bits: z = 0, s = 1), every value token's 32 channels
    too; the codes are then the values themselves, packed as the layout states, and the
    decode returns the input exactly."""
    L, B, H, T, d, bits = 1, 1, 1, 32, 32, 3
    t = np.arange(T)[:, None]
    c = np.arange(d)[None, :]
    keys = ((t + c) % 8).astype(np.float64)            # each channel: 0..7 over its 32 tokens
    vals = ((3 * c + t) % 8).astype(np.float64)        # each token: 0..7 over its 32 channels
    x = np.stack([keys, vals])[None, :, None, None]    # [1, 2, 1, 1, T, d]
    G = np.broadcast_to(np.eye(16), (L, 2, H, d // 16, 16, 16)).copy()
    enc = oc.encode_kivi(x, G, bits)
    assert np.all(enc["key"]["z"] == 0) and np.all(enc["key"]["s"] == 1)
    assert np.all(enc["value"]["z"] == 0) and np.all(enc["value"]["s"] == 1)
    assert np.array_equal(enc["key"]["q"][0, 0, 0, 0], keys.T)           # [channel][token]
    assert np.array_equal(enc["value"]["q"][0, 0, 0, :, 0], vals)        # [token][channel]
    # channel 0's key record: tokens 0..31 hold 0,1,..,7,0,.. -> 3-bit stream 0b..010001000
    rec = enc["key"]["codes"][0, 0, 0, 0, 0]
    assert rec.size == 12 and int.from_bytes(bytes(rec[:3]), "little") == sum(k << (3 * k) for k in range(8))
    xr = oc.decode_kivi(enc, G, bits)
    assert np.array_equal(xr, x)
