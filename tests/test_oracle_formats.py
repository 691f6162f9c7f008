"""Pins for the oracle's number formats and weight formats (CPU only).

Every check compares the oracle with something other than itself: a library
cast (torch), brute force over all values of a format, the worked examples in
tests/golden (derived by hand from the pages' definitions), or the gguf
package's independent Q4_0 implementation.
"""
import numpy as np
import pytest
import torch

import qg_synth
from oracle import qg_oracle as O
from tests.conftest import golden


# ---------------------------------------------------------------- bf16 ----

def _torch_bf16(v32):
    return torch.from_numpy(v32).to(torch.bfloat16).to(torch.float64).numpy()


def test_round_bf16_matches_torch_cast_on_f32_inputs():
    g = np.random.default_rng(1)
    v = np.concatenate([
        g.standard_normal(20000) * 10.0 ** g.integers(-30, 30, 20000),
        # exact halfway points between neighbouring bf16 values (ties-to-even)
        (np.arange(1, 2000, dtype=np.float64) * 2 + 1) * 2.0 ** -9,
        # bf16 subnormal range
        g.standard_normal(2000) * 2.0 ** -130,
        [0.0, -0.0, 3.3895313892515355e38, 1e-45],
    ]).astype(np.float32)
    np.testing.assert_array_equal(O.round_bf16(v.astype(np.float64)), _torch_bf16(v))


def test_directed_bf16_rounding_brute_force():
    # every positive finite bf16 value, sorted
    bits = np.arange(0x0001, 0x7F80, dtype=np.uint16)
    grid = (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    g = np.random.default_rng(2)
    v = np.abs(g.standard_normal(5000)) * 10.0 ** g.integers(-20, 20, 5000)
    v = np.concatenate([v, grid[::997]])          # exact grid points too
    i = np.searchsorted(grid, v, side="right") - 1  # largest grid value <= v
    down = grid[i]
    j = np.searchsorted(grid, v, side="left")       # smallest grid value >= v
    up = grid[j]
    np.testing.assert_array_equal(O.round_bf16_down(v), down)
    np.testing.assert_array_equal(O.round_bf16_up(v), up)
    np.testing.assert_array_equal(O.round_bf16_down(-v), -up)


def test_bf16_bits_roundtrip_against_torch():
    bits = np.arange(0, 0x10000, dtype=np.uint32).astype(np.uint16)
    t = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    v = O.bf16_bits_to_f64(bits)
    fin = np.isfinite(t)
    np.testing.assert_array_equal(v[fin], t[fin])
    np.testing.assert_array_equal(O.bf16_value_to_bits(v[fin]), bits[fin])


# -------------------------------------------------------- affine-INT8 ----

def test_pack_unpack_all_byte_values_all_lanes():
    q = np.zeros((256, 4 * 256), dtype=np.uint8)
    for lane in range(4):
        q[:, lane::4] = np.arange(256, dtype=np.uint8)[:, None]
    q[:, 1::4] = 255 - q[:, 1::4]
    np.testing.assert_array_equal(O.affine8_unpack(O.affine8_pack(q)), q)


def test_pack_is_little_endian_byte_per_column():
    q = np.array([[0x01, 0x02, 0x03, 0x04, 0xAA, 0xBB, 0xCC, 0xDD]], dtype=np.uint8)
    w = O.affine8_pack(q)
    assert w.tolist() == [[0x04030201, 0xDDCCBBAA]]
    # same as reinterpreting the row's bytes as little-endian u32 words
    np.testing.assert_array_equal(w, q.view("<u4"))


def test_affine8_dequant_fixture_constants():
    gd = golden("affine8_fixture_dequant.txt")
    s_bits = int(gd["scale_bits"][0][0], 16)
    b_bits = int(gd["bias_bits"][0][0], 16)
    # the page's constants, cast by torch, give the golden bit patterns
    assert qg_synth.f32_to_bf16_bits(np.array([0.004], np.float32))[0] == s_bits
    assert qg_synth.f32_to_bf16_bits(np.array([-0.508], np.float32))[0] == b_bits
    assert O.bf16_bits_to_f64(np.uint16(s_bits)) == float(gd["scale_bf16"][0][0])
    assert O.bf16_bits_to_f64(np.uint16(b_bits)) == float(gd["bias_bf16"][0][0])
    codes = [int(r[0]) for r in gd["q"]]
    want = [float(r[1]) for r in gd["q"]]
    q = np.zeros((1, 64), dtype=np.uint8)
    q[0, :len(codes)] = codes
    w = O.affine8_dequant_exact(O.affine8_pack(q), np.array([[s_bits]], np.uint16),
                                np.array([[b_bits]], np.uint16))
    np.testing.assert_array_equal(w[0, :len(codes)], want)
    # the float32 dequant is that exact value, which float32 holds exactly here
    np.testing.assert_array_equal(
        O.affine8_dequant_f32(O.affine8_pack(q), np.array([[s_bits]], np.uint16),
                              np.array([[b_bits]], np.uint16))[0, :len(codes)],
        np.array(want, np.float32))


def test_affine8_quantize_roundtrip_bound():
    w = qg_synth.gaussian((64, 512), 0.02, seed=3)
    words, s, b = O.affine8_quantize(w)
    wh = O.affine8_dequant_exact(words, s, b)
    sc = np.repeat(O.bf16_bits_to_f64(s), 64, axis=1)
    bi = np.repeat(O.bf16_bits_to_f64(b), 64, axis=1)
    assert np.all(np.abs(w - wh) <= sc / 2 * (1 + 1e-12))
    # the f32 dequant adds at most one float32 rounding
    wf = O.affine8_dequant_f32(words, s, b).astype(np.float64)
    assert np.all(np.abs(w - wf) <= sc / 2 + np.spacing(np.abs(wf).astype(np.float32)))
    # directed roundings bracket every group
    g = w.reshape(64, 8, 64)
    assert np.all(O.bf16_bits_to_f64(b) <= g.min(axis=2))
    assert np.all(O.bf16_bits_to_f64(b) + 255 * O.bf16_bits_to_f64(s) >= g.max(axis=2))
    assert np.all(bi <= w)


def test_affine8_quantize_constant_group():
    w = np.full((2, 64), 0.25, dtype=np.float32)
    words, s, b = O.affine8_quantize(w)
    np.testing.assert_array_equal(O.affine8_dequant_exact(words, s, b), w)


# --------------------------------------------------------------- Q4_0 ----

def _hexbytes(tokens):
    return np.array([int(t, 16) for t in tokens], dtype=np.uint8)


def _q4_worked_blocks():
    A = np.arange(32, dtype=np.float32) - 16
    B = np.zeros(32, np.float32)
    B[0] = 8
    C = np.zeros(32, np.float32)
    return {"A": A, "B": B, "C": C}


@pytest.mark.parametrize("name", ["A", "B", "C"])
def test_q4_0_worked_example(name):
    gd = golden("q4_0_worked_example.txt")
    x = _q4_worked_blocks()[name]
    got = O.q4_0_quantize(x[None])
    np.testing.assert_array_equal(got[0], _hexbytes(gd[f"{name}_bytes"][0]))
    deq = O.q4_0_dequant_exact(got, 32)[0]
    want = np.array([float(t) for t in gd[f"{name}_dequant"][0]])
    np.testing.assert_array_equal(deq, want)
    np.testing.assert_array_equal(np.signbit(deq), np.signbit(want))   # -0.0 where d < 0, n = 8


def test_q4_0_closed_form_of_block_A():
    # n_j = ceil(j/2) clamped to 15, derived from the rule (see the golden file)
    got = O.q4_0_quantize((np.arange(32, dtype=np.float32) - 16)[None])
    _, n = O.q4_0_unpack(got, 32)
    want = np.minimum(15, (np.arange(32) + 1) // 2)
    np.testing.assert_array_equal(n[0], want)


def test_q4_0_against_gguf_package():
    gq = pytest.importorskip("gguf.quants")
    from gguf import GGMLQuantizationType as T
    x = qg_synth.gaussian((37, 256), 0.02, seed=4)
    x[3, 5] = 0.0
    x[4, :32] = 0.0                      # all-zero block
    x[5, 32:64] = x[5, 32]               # constant block
    ours = O.q4_0_quantize(x)
    theirs = gq.quantize(x, T.Q4_0)
    np.testing.assert_array_equal(ours, theirs)
    np.testing.assert_array_equal(O.q4_0_dequant_exact(ours, 256),
                                  gq.dequantize(theirs, T.Q4_0).astype(np.float64))


def test_q4_0_roundtrip_bound():
    x = qg_synth.gaussian((16, 1024), 0.02, seed=5).astype(np.float64)
    blocks = O.q4_0_quantize(x)
    d16, n = O.q4_0_unpack(blocks, 1024)
    xb = x.reshape(16, 32, 32)
    m = np.take_along_axis(xb, np.argmax(np.abs(xb), axis=2)[:, :, None], axis=2)[:, :, 0]
    d = m / -8.0                                        # unrounded scale
    err = np.abs(x - O.q4_0_dequant_exact(blocks, 1024)).reshape(16, 32, 32)
    slack = 8 * np.abs(d - d16)[:, :, None] + 1e-12     # fp16 storage of d
    nn = n.reshape(16, 32, 32)
    unclamped = nn < 15
    assert np.all((err <= np.abs(d)[:, :, None] / 2 + slack)[unclamped])
    assert np.all(err <= np.abs(d)[:, :, None] + slack)


def test_q4_0_unpack_nibble_order():
    blk = np.zeros((1, 18), np.uint8)
    blk[0, 0:2] = np.array([1.0], np.float16).view(np.uint8)
    blk[0, 2:] = np.arange(16, dtype=np.uint8) | (np.uint8(15) - np.arange(16, dtype=np.uint8)) << 4
    d, n = O.q4_0_unpack(blk, 32)
    assert d[0, 0] == 1.0
    np.testing.assert_array_equal(n[0, :16], np.arange(16))
    np.testing.assert_array_equal(n[0, 16:], 15 - np.arange(16))
