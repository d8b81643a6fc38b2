"""Pins of the oracle's group-scaled signed INT4 format (ExpertMesh README: signed
INT4 weights with group scales in an [expert, output, packed_input] layout).

Reading of the format, stated where the page leaves it open: one bf16 scale
per 128 consecutive inputs of an output row, s = bf16(max|w|/7),
q = clamp(rint(w/s), -8, 7), two nibbles per byte with the even input index in
the low nibble, two's complement.
"""

import numpy as np

from oracle import moe_oracle as O


def test_bf16_round_ties_to_even():
    one = 1.0
    vals = np.array([one + 2 ** -8, one + 3 * 2 ** -8, one + 2 ** -9, -(one + 3 * 2 ** -8), 3.0e38], np.float32)
    want = [1.0, 1.0 + 2 ** -6, 1.0, -(1.0 + 2 ** -6)]
    got = O.bf16_round(vals)
    assert got[:4].tolist() == want
    assert (got.view(np.uint32) & 0xFFFF == 0).all()


def test_pack_unpack_is_a_bijection_on_bytes():
    b = np.arange(256, dtype=np.uint8)[None, :]
    q = O.unpack_int4(b)
    assert q.min() == -8 and q.max() == 7
    assert (O.pack_int4(q) == b).all()


def test_nibble_order_low_nibble_is_even_index():
    assert O.pack_int4(np.array([1, -1], np.int8)).tolist() == [0xF1]
    assert O.pack_int4(np.array([-8, 7], np.int8)).tolist() == [0x78]


def test_hand_group_with_max_seven():
    # max |w| = 7 -> s = 1 exactly, q = rint(w) (ties to even)
    w = np.zeros((1, 128), np.float32)
    w[0, :6] = [7.0, 0.5, 1.5, 2.5, -0.5, -7.0]
    q, s = O.quantize_int4_g128(w)
    assert s.tolist() == [[1.0]]
    assert q[0, :6].tolist() == [7, 0, 2, 2, 0, -7]
    np.testing.assert_array_equal(O.dequantize_int4_g128(O.pack_int4(q), s), O.quantize_int4_g128(w)[0].astype(float))


def test_zero_group_has_zero_scale_and_codes():
    w = np.zeros((2, 256), np.float32)
    w[1, 128:] = 1.0
    q, s = O.quantize_int4_g128(w)
    assert s.tolist() == [[0.0, 0.0], [0.0, O.bf16_round(np.float32(1.0) / np.float32(7.0)).item()]]
    assert (q[0] == 0).all() and (q[1, :128] == 0).all() and (q[1, 128:] == 7).all()


def test_round_trip_error_within_half_a_step():
    rng = np.random.default_rng(0)
    w = (rng.standard_normal((3, 16, 512)) / np.sqrt(512)).astype(np.float32)
    q, s = O.quantize_int4_g128(w)
    assert q.min() >= -7 and q.max() <= 7
    assert (np.abs(q).reshape(3, 16, 4, 128).max(-1) == 7).all()      # the max of each group maps to +-7
    dq = O.dequantize_int4_g128(O.pack_int4(q), s)
    step = np.repeat(s.astype(np.float64), 128, axis=-1)
    assert (np.abs(dq - w) <= step / 2 * (1 + 1e-6)).all()
    # the scale is a bf16 value within one bf16 rounding of max|w|/7
    amax = np.abs(w.reshape(3, 16, 4, 128)).max(-1).astype(np.float64)
    assert (np.abs(s - amax / 7) <= 2 ** -8 * amax / 7).all()
