"""Pins of the oracle's Whisper encoder layer (fuel-transformers 0.19.1,
src/models/lazy_quantized_whisper.rs, encoder_layer / multi_head_attn /
layer_norm_affine / q_linear) against library routines, closed forms and
special cases: torch's layer_norm, gelu(approximate="tanh") and
scaled_dot_product_attention in float64; the identity layer; and the whole
layer recomposed from torch ops on the oracle-independent Q4_0 reader."""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import qg_synth
from oracle import qg_oracle as O


def test_layer_norm_against_torch_and_closed_forms():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((7, 96)) * 3 + 1
    g, b = rng.standard_normal(96), rng.standard_normal(96)
    want = F.layer_norm(torch.from_numpy(x), (96,), torch.from_numpy(g), torch.from_numpy(b),
                        eps=1e-5).numpy()
    np.testing.assert_allclose(O.layer_norm(x, g, b, 1e-5), want, rtol=1e-12, atol=1e-12)
    # a constant row normalises to zero: the output is beta exactly
    np.testing.assert_array_equal(O.layer_norm(np.full((2, 96), 4.25), g, b, 1e-5), np.stack([b, b]))
    # two-valued row +-a: normalised values are +-a / sqrt(a^2 + eps)
    a = 0.5
    row = np.tile([a, -a], 48)
    np.testing.assert_allclose(O.layer_norm(row, np.ones(96), np.zeros(96), 1e-5),
                               row / math.sqrt(a * a + 1e-5), rtol=1e-14)


def test_gelu_tanh_against_torch():
    x = np.linspace(-12, 12, 2001)
    want = F.gelu(torch.from_numpy(x), approximate="tanh").numpy()
    np.testing.assert_allclose(O.gelu_tanh(x), want, rtol=1e-13, atol=1e-15)
    assert O.gelu_tanh(np.array([0.0]))[0] == 0.0
    np.testing.assert_allclose(O.gelu_tanh(np.array([40.0])), [40.0], rtol=1e-15)


@pytest.mark.parametrize("causal", [False, True])
def test_mha_rows_against_sdpa(causal):
    rng = np.random.default_rng(2)
    T, H, D = 9, 3, 16
    q, k, v = (rng.standard_normal((T, H * D)) for _ in range(3))
    got = O.mha_rows(q, k, v, H, causal=causal)
    tq = torch.from_numpy(q).view(T, H, D).transpose(0, 1)
    tk = torch.from_numpy(k).view(T, H, D).transpose(0, 1)
    tv = torch.from_numpy(v).view(T, H, D).transpose(0, 1)
    want = F.scaled_dot_product_attention(tq, tk, tv, is_causal=causal).transpose(0, 1).reshape(T, -1)
    np.testing.assert_allclose(got, want.numpy(), rtol=1e-12, atol=1e-12)


def test_mha_rows_prefix_and_gqa():
    """Causal rows after a cached prefix (S > T: row i sits at position
    S - T + i) against an explicit mask; grouped KV heads against the
    repeat_kv expansion."""
    rng = np.random.default_rng(3)
    T, S, H, Hkv, D = 4, 10, 4, 2, 8
    q = rng.standard_normal((T, H * D))
    k, v = rng.standard_normal((S, Hkv * D)), rng.standard_normal((S, Hkv * D))
    got = O.mha_rows(q, k, v, H, causal=True, kv_heads=Hkv)
    rep = lambda a: np.repeat(a.reshape(S, Hkv, D), H // Hkv, axis=1).reshape(S, H * D)
    mask = np.arange(S)[None, :] <= (S - T + np.arange(T))[:, None]
    tq = torch.from_numpy(q).view(T, H, D).transpose(0, 1)
    tk = torch.from_numpy(rep(k)).view(S, H, D).transpose(0, 1)
    tv = torch.from_numpy(rep(v)).view(S, H, D).transpose(0, 1)
    want = F.scaled_dot_product_attention(tq, tk, tv, attn_mask=torch.from_numpy(mask))
    np.testing.assert_allclose(got, want.transpose(0, 1).reshape(T, -1).numpy(), rtol=1e-12,
                               atol=1e-12)


def _tiny_layer(seed, d=64, ffn=128, zero=False):
    rng = np.random.default_rng(seed)
    def q4(N, K):
        w = np.zeros((N, K), np.float32) if zero else rng.standard_normal((N, K)).astype(np.float32) * 0.05
        return O.q4_0_quantize(w)
    def vec(n, s=0.1):
        return np.zeros(n) if zero else (rng.standard_normal(n) * s).astype(np.float32).astype(np.float64)
    return {"ln1_g": 1 + vec(d), "ln1_b": vec(d), "q": q4(d, d), "q_b": vec(d), "k": q4(d, d),
            "v": q4(d, d), "v_b": vec(d), "o": q4(d, d), "o_b": vec(d), "ln2_g": 1 + vec(d),
            "ln2_b": vec(d), "fc1": q4(ffn, d), "fc1_b": vec(ffn), "fc2": q4(d, ffn),
            "fc2_b": vec(d)}


def test_encoder_layer_with_zero_weights_is_the_identity():
    lw = _tiny_layer(4, zero=True)
    x = np.random.default_rng(5).standard_normal((6, 64))
    np.testing.assert_array_equal(O.whisper_encoder_layer(x, lw, 2), x)


def test_encoder_layer_against_torch_composition():
    """The layer rebuilt from torch ops (layer_norm, linear, SDPA, gelu) on
    weights read by the test's own Q4_0 decoder, with bf16 roundings at the
    same points."""
    d, H, ffn, T = 64, 2, 128, 7
    lw = _tiny_layer(6, d, ffn)
    x = np.random.default_rng(7).standard_normal((T, d))

    def w_of(blocks, K):   # independent Q4_0 reader: fp16 d then 16 nibble bytes per block
        b = blocks.reshape(blocks.shape[0], K // 32, 18)
        dd = b[:, :, :2].copy().view(np.float16)[:, :, 0].astype(np.float64)
        lo, hi = (b[:, :, 2:] & 15).astype(np.float64), (b[:, :, 2:] >> 4).astype(np.float64)
        n = np.concatenate([lo, hi], axis=2)
        return torch.from_numpy((dd[:, :, None] * (n - 8)).reshape(blocks.shape[0], K))
    bf = lambda t: t.to(torch.bfloat16).double()
    t = lambda a: torch.from_numpy(np.asarray(a, np.float64))
    lin = lambda a, blk, K, bias=None: F.linear(bf(a), bf(w_of(blk, K)),
                                                None if bias is None else t(bias))
    X = t(x)
    xl = bf(F.layer_norm(X, (d,), t(lw["ln1_g"]), t(lw["ln1_b"]), eps=1e-5))
    q, k, v = bf(lin(xl, lw["q"], d, lw["q_b"])), bf(lin(xl, lw["k"], d)), bf(lin(xl, lw["v"], d, lw["v_b"]))
    split = lambda a: a.view(T, H, d // H).transpose(0, 1)
    ctx = bf(F.scaled_dot_product_attention(split(q), split(k), split(v)).transpose(0, 1).reshape(T, d))
    xa = X + lin(ctx, lw["o"], d, lw["o_b"])
    xl2 = bf(F.layer_norm(xa, (d,), t(lw["ln2_g"]), t(lw["ln2_b"]), eps=1e-5))
    mid = bf(F.gelu(lin(xl2, lw["fc1"], d, lw["fc1_b"]), approximate="tanh"))
    want = xa + lin(mid, lw["fc2"], ffn, lw["fc2_b"])
    det = {}
    got = O.whisper_encoder_layer(x, lw, H, details=det)
    np.testing.assert_allclose(got, want.numpy(), rtol=1e-9, atol=1e-9)
    np.testing.assert_allclose(det["ctx"], ctx.numpy(), rtol=0, atol=2 ** -8 * np.abs(ctx.numpy()).max())
