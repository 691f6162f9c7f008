"""Pins for the oracle's arithmetic (CPU only).

GEMVs against pure-Python brute force (bytes pulled out of the words with
shifts, one multiply-add at a time), identity and one-hot matrices; norms,
SiLU and attention against torch's own routines in float64; RoPE against a
complex-number formulation and its group law; the decode step against a
whole-prefix causal forward and a zero-weight closed form.
"""
import cmath
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import qg_synth
from oracle import qg_oracle as O


def _bf16(bits):
    return torch.from_numpy(np.asarray(bits, np.uint16).view(np.int16)).view(torch.bfloat16).double().numpy()


# ---------------------------------------------------------------- GEMV ----

def _brute_gemv_affine8(words, scales, biases, x):
    N, W = words.shape
    K = 4 * W
    B = x.shape[0]
    s = _bf16(scales)
    b = _bf16(biases)
    y = [[0.0] * N for _ in range(B)]
    for bb in range(B):
        for r in range(N):
            acc = 0.0
            for c in range(K):
                q = (int(words[r, c // 4]) >> (8 * (c % 4))) & 0xFF
                acc += (q * s[r, c // 64] + b[r, c // 64]) * float(x[bb, c])
            y[bb][r] = acc
    return np.array(y)


def test_gemv_affine8_brute_force():
    words, s, b = qg_synth.affine8_packed(5, 128, seed=11)
    x = _bf16(qg_synth.gaussian_bf16_bits((3, 128), 1.0, seed=12))
    np.testing.assert_allclose(O.gemv_affine8(words, s, b, x),
                               _brute_gemv_affine8(words, s, b, x), rtol=1e-12, atol=1e-14)


def test_gemv_affine8_identity_and_one_hot():
    K = 128
    q = np.eye(K, dtype=np.uint8)
    one = qg_synth.f32_to_bf16_bits(np.ones((K, K // 64), np.float32))
    zero = np.zeros((K, K // 64), np.uint16)
    x = _bf16(qg_synth.gaussian_bf16_bits((2, K), 1.0, seed=13))
    np.testing.assert_array_equal(O.gemv_affine8(O.affine8_pack(q), one, zero, x), x)
    words, s, b = qg_synth.affine8_packed(7, K, seed=14)
    e = np.zeros((1, K))
    e[0, 77] = 1.0
    np.testing.assert_array_equal(O.gemv_affine8(words, s, b, e)[0],
                                  O.affine8_dequant_exact(words, s, b)[:, 77])


def test_gemv_affine8_factorisation():
    # sum_g s_g * (sum_c q_c x_c) + beta_g * (sum_c x_c) equals the plain sum
    words, s, b = qg_synth.affine8_packed(9, 256, seed=15)
    x = _bf16(qg_synth.gaussian_bf16_bits((2, 256), 1.0, seed=16))
    q = O.affine8_unpack(words).astype(np.float64).reshape(9, 4, 64)
    xs = x.reshape(2, 4, 64)
    y = np.einsum("rg,brg->br", _bf16(s), np.einsum("rgc,bgc->brg", q, xs)) \
        + np.einsum("rg,bg->br", _bf16(b), xs.sum(axis=2))
    np.testing.assert_allclose(O.gemv_affine8(words, s, b, x), y, rtol=1e-12)


def test_gemv_affine8_residual():
    words, s, b = qg_synth.affine8_packed(6, 64, seed=17)
    x = np.ones((1, 64))
    r = np.arange(6.0)[None]
    np.testing.assert_allclose(O.gemv_affine8(words, s, b, x, residual=r),
                               O.gemv_affine8(words, s, b, x) + r, rtol=0, atol=0)


def _brute_gemv_q4_0(blocks, x, bias):
    N = blocks.shape[0]
    K = x.shape[1]
    y = np.zeros((x.shape[0], N))
    for bb in range(x.shape[0]):
        for r in range(N):
            acc = 0.0
            for blk in range(K // 32):
                base = blk * 18
                d = float(np.frombuffer(bytes(blocks[r, base:base + 2]), dtype="<f2")[0])
                for j in range(32):
                    byte = int(blocks[r, base + 2 + (j % 16)])
                    n = (byte & 0xF) if j < 16 else (byte >> 4)
                    acc += d * (n - 8) * float(x[bb, blk * 32 + j])
            y[bb, r] = acc + (bias[r] if bias is not None else 0.0)
    return y


def test_gemv_q4_0_brute_force():
    blocks = qg_synth.q4_0_packed(4, 96, seed=18)
    x = qg_synth.gaussian((2, 96), 1.0, seed=19).astype(np.float64)
    bias = qg_synth.gaussian((4,), 1.0, seed=20).astype(np.float64)
    np.testing.assert_allclose(O.gemv_q4_0(blocks, x, bias), _brute_gemv_q4_0(blocks, x, bias),
                               rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(O.gemv_q4_0(blocks, x), _brute_gemv_q4_0(blocks, x, None),
                               rtol=1e-12, atol=1e-14)


def test_gemv_q4_0_identity():
    K = 64
    blk = np.zeros((K, K // 32, 18), np.uint8)
    blk[:, :, 0:2] = np.array([1.0], np.float16).view(np.uint8)
    n = np.full((K, K), 8, np.uint8)
    n[np.arange(K), np.arange(K)] = 9
    n = n.reshape(K, K // 32, 32)
    blk[:, :, 2:] = n[:, :, :16] | (n[:, :, 16:] << 4)
    x = qg_synth.gaussian((3, K), 1.0, seed=21).astype(np.float64)
    np.testing.assert_array_equal(O.gemv_q4_0(blk.reshape(K, -1), x), x)


def test_gemm_q4_0_bf16_contract_brute_force():
    blocks = qg_synth.q4_0_packed(4, 64, seed=22)
    A = qg_synth.gaussian((3, 64), 1.0, seed=23)
    bias = qg_synth.gaussian((4,), 1.0, seed=24)
    Ab = torch.from_numpy(A).to(torch.bfloat16).double()
    # dequantize with the brute-force reader (identity x), cast with torch
    W = _brute_gemv_q4_0(blocks, np.eye(64), None).T
    Wb = torch.from_numpy(W.astype(np.float32)).to(torch.bfloat16).double()
    want = (Ab @ Wb.T).numpy() + bias
    np.testing.assert_allclose(O.gemm_q4_0_bf16(blocks, A, bias), want, rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------- elementwise --

def test_rmsnorm_closed_form_and_torch():
    w = qg_synth.f32_to_bf16_bits(np.linspace(0.5, 1.5, 64).astype(np.float32))
    c, eps = 0.3, 1e-6
    np.testing.assert_allclose(O.rmsnorm(np.full(64, c), w, eps), c / math.sqrt(c * c + eps) * _bf16(w),
                               rtol=1e-14)
    x = qg_synth.gaussian((5, 64), 3.0, seed=25).astype(np.float64)
    want = F.rms_norm(torch.from_numpy(x), (64,), torch.from_numpy(_bf16(w)), eps=eps).numpy()
    np.testing.assert_allclose(O.rmsnorm(x, w, eps), want, rtol=1e-13)
    # scale invariance with eps = 0
    np.testing.assert_allclose(O.rmsnorm(7.0 * x, w, 0.0), O.rmsnorm(x, w, 0.0), rtol=1e-13)


def test_rmsnorm_perhead_is_rmsnorm_per_slice():
    D = 32
    w = qg_synth.f32_to_bf16_bits((1 + 0.1 * qg_synth.gaussian((D,), 1.0, seed=26)).astype(np.float32))
    x = qg_synth.gaussian((3, 4 * D), 2.0, seed=27).astype(np.float64)
    want = F.rms_norm(torch.from_numpy(x).reshape(3, 4, D), (D,), torch.from_numpy(_bf16(w)),
                      eps=1e-5).reshape(3, 4 * D).numpy()
    np.testing.assert_allclose(O.rmsnorm_perhead(x, w, 1e-5, D), want, rtol=1e-13)


def test_rope_complex_form():
    # NeoX pairs (i, i+half) rotate like the complex number x_i + 1j*x_{i+half}
    D, theta, pos = 8, 10000.0, 37
    x = qg_synth.gaussian((3 * D,), 1.0, seed=28).astype(np.float64)
    got = O.rope_neox(x, pos, theta, D).reshape(3, D)
    xh = x.reshape(3, D)
    for h in range(3):
        for i in range(D // 2):
            z = complex(xh[h, i], xh[h, i + D // 2]) * cmath.exp(1j * pos * theta ** (-2 * i / D))
            assert abs(got[h, i] - z.real) < 1e-12 and abs(got[h, i + D // 2] - z.imag) < 1e-12


def test_rope_invariants():
    D = 128
    x = qg_synth.gaussian((4 * D,), 1.0, seed=29).astype(np.float64)
    np.testing.assert_array_equal(O.rope_neox(x, 0, 1e6, D), x)
    y = O.rope_neox(x, 511, 1e6, D).reshape(4, 2, D // 2)
    xr = x.reshape(4, 2, D // 2)
    np.testing.assert_allclose((y ** 2).sum(axis=1), (xr ** 2).sum(axis=1), rtol=1e-12)
    np.testing.assert_allclose(O.rope_neox(O.rope_neox(x, 200, 1e6, D), 311, 1e6, D),
                               O.rope_neox(x, 511, 1e6, D), rtol=1e-9, atol=1e-12)


def test_rope_partial_rotary_dim_passes_tail_through():
    D, rd = 64, 32
    x = qg_synth.gaussian((2 * D,), 1.0, seed=30).astype(np.float64)
    y = O.rope_neox(x, 9, 1e4, D, rotary_dim=rd).reshape(2, D)
    np.testing.assert_array_equal(y[:, rd:], x.reshape(2, D)[:, rd:])
    np.testing.assert_allclose(y[:, :rd], O.rope_neox(x.reshape(2, D)[:, :rd].reshape(-1), 9, 1e4, rd).reshape(2, rd))


def test_silu_mul_against_torch():
    g = qg_synth.gaussian((1000,), 4.0, seed=31).astype(np.float64)
    u = qg_synth.gaussian((1000,), 1.0, seed=32).astype(np.float64)
    want = (F.silu(torch.from_numpy(g)) * torch.from_numpy(u)).numpy()
    np.testing.assert_allclose(O.silu_mul(g, u), want, rtol=1e-14)


# ------------------------------------------------------------ attention --

def _cache(Hkv, L, D, seed):
    return (_bf16(qg_synth.gaussian_bf16_bits((Hkv, L, D), 1.0, seed)),
            _bf16(qg_synth.gaussian_bf16_bits((Hkv, L, D), 1.0, seed + 1)))


def test_attention_matches_torch_sdpa_with_repeat_kv():
    H, Hkv, D, L = 16, 8, 128, 77
    k, v = _cache(Hkv, 100, D, 33)
    q = qg_synth.gaussian((H * D,), 1.0, seed=35).astype(np.float64)
    got = O.decode_attention(q, k, v, L, H, Hkv, D)
    kk = torch.from_numpy(k[:, :L]).repeat_interleave(H // Hkv, dim=0)   # explicit repeat_kv
    vv = torch.from_numpy(v[:, :L]).repeat_interleave(H // Hkv, dim=0)
    want = F.scaled_dot_product_attention(torch.from_numpy(q).reshape(H, 1, D), kk, vv).reshape(-1).numpy()
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-13)


def test_attention_special_cases():
    H, Hkv, D = 4, 2, 16
    k, v = _cache(Hkv, 8, D, 36)
    q = qg_synth.gaussian((H * D,), 1.0, seed=38).astype(np.float64)
    # L = 1: the only value row comes back exactly
    out = O.decode_attention(q, k, v, 1, H, Hkv, D).reshape(H, D)
    for h in range(H):
        np.testing.assert_array_equal(out[h], v[h // 2, 0])
    # identical keys: the mean of the values
    k2 = np.repeat(k[:, :1], 8, axis=1)
    out = O.decode_attention(q, k2, v, 8, H, Hkv, D).reshape(H, D)
    for h in range(H):
        np.testing.assert_allclose(out[h], v[h // 2].mean(axis=0), rtol=1e-12, atol=1e-14)
    # one dominant key: its value row
    k3 = np.zeros_like(k)
    qh = q.reshape(H, D)
    for h in range(H):
        k3[h // 2, 5] += 200.0 * qh[h] / np.linalg.norm(qh[h])
    out = O.decode_attention(q, k3, v, 8, H, Hkv, D).reshape(H, D)
    for h in range(H):
        np.testing.assert_allclose(out[h], v[h // 2, 5], rtol=1e-9, atol=1e-12)


def test_argmax_first_strict_max_skips_nan():
    assert O.argmax_first([1.0, 3.0, 3.0, 2.0]) == 1
    assert O.argmax_first([float("nan"), 0.5, float("nan"), 0.7, 0.7]) == 3
    assert O.argmax_first([float("-inf")] * 3) == 0
    x = qg_synth.gaussian((5000,), 1.0, seed=39)
    assert O.argmax_first(x) == int(np.argmax(x))


# --------------------------------------------------------- decode step ---

def _tiny(seed, fixture=True):
    cfg = dict(qg_synth.QWEN3_TINY)
    return cfg, qg_synth.qwen3_weights(cfg, seed, fixture=fixture)


@pytest.mark.parametrize("fixture", [True, False])
def test_decode_step_matches_causal_prefix_forward(fixture):
    cfg, w = _tiny(3, fixture)
    toks = [5, 200, 17, 17, 260, 0]
    kc, vc = O.new_kv_cache(cfg, 16)
    for p, t in enumerate(toks):
        logits = O.decode_step(cfg, w, kc, vc, t, p)
    full = O.prefix_forward(cfg, w, toks)
    np.testing.assert_allclose(logits, full[-1], rtol=1e-9, atol=1e-9 * np.abs(full[-1]).max())
    assert np.isfinite(logits).all()


def test_decode_step_zero_weights_closed_form():
    # With every linear zero, attention and MLP add nothing: the logits are
    # the LM head applied to the normed embedding row.
    cfg, w = _tiny(4, fixture=False)
    for lw in w["layers"]:
        for name in qg_synth.LINEARS:
            words, s, b = lw[name]
            lw[name] = (np.zeros_like(words), s, np.zeros_like(b))
    ew, es, eb = w["embed"]
    t = 42
    kc, vc = O.new_kv_cache(cfg, 4)
    logits = O.decode_step(cfg, w, kc, vc, t, 0)
    e = O.affine8_dequant_exact(ew, es, eb)
    row = e[t].astype(np.float32).astype(np.float64)
    xn = torch.from_numpy(row / np.sqrt(np.mean(row ** 2) + cfg["eps"])).to(torch.bfloat16).double().numpy()
    np.testing.assert_allclose(logits, e @ xn, rtol=1e-12, atol=1e-12)


def test_bf16_alternative_marks_only_near_midpoint_values():
    # 1 and 1 + 2^-7 are neighbouring bf16 values; 1 + 2^-8 is their midpoint
    mid = 1.0 + 2.0 ** -8
    v = np.array([mid, mid * (1 + 2.0 ** -20), mid * (1 - 2.0 ** -20), 1.0 + 2.0 ** -10,
                  -mid, 3.0, 0.0])
    alt = O.bf16_alternative(v, 2.0 ** -18)
    # the midpoint rounds to even (1.0); the other neighbour is 1 + 2^-7
    assert alt[0] == 1.0 + 2.0 ** -7
    assert alt[1] == 1.0 and alt[2] == 1.0 + 2.0 ** -7   # just above / below: the other side
    assert np.isnan(alt[3]) and np.isnan(alt[5]) and np.isnan(alt[6])
    assert alt[4] == -(1.0 + 2.0 ** -7)
    # with rel = 0 only exact midpoints count
    assert np.isnan(O.bf16_alternative(v[1:2], 0.0)[0])
    # the alternative is always a bf16 value adjacent to round_bf16(v)
    r = O.round_bf16(v[:3])
    assert np.all(np.abs(alt[:3] - r) == 2.0 ** -7)


def test_bf16_rounding_ok_is_the_set_of_roundings_within_the_error_bound():
    mid = 1.0 + 2.0 ** -8                        # midpoint of 1 and 1 + 2^-7
    up, down = 1.0 + 2.0 ** -7, 1.0
    near = mid * (1 + 2.0 ** -20)
    # within the bound of a midpoint both neighbours are roundings of a value
    # in [v - eps, v + eps]
    assert O.bf16_rounding_ok([near], [up])[0] and O.bf16_rounding_ok([near], [down])[0]
    # far from it only the nearest one
    far = 1.0 + 2.0 ** -10
    assert O.bf16_rounding_ok([far], [down])[0] and not O.bf16_rounding_ok([far], [up])[0]
    # a value on the grid rounds to itself; two steps away is never right
    assert O.bf16_rounding_ok([1.0], [1.0])[0] and not O.bf16_rounding_ok([1.0], [up])[0]
    assert not O.bf16_rounding_ok([near], [1.0 + 2.0 ** -6])[0]
    assert O.bf16_rounding_ok([np.nan], [np.nan])[0]
    # an absolute bound well above a tiny value's own bf16 step admits every
    # rounding inside it, and nothing outside
    t = 3.6e-6
    step = 2.0 ** -26                            # bf16 step at 2^-19 .. 2^-18
    cand = O.round_bf16(t) + step * np.arange(-4, 5)
    ok = O.bf16_rounding_ok(np.full(cand.shape, t), cand, abs_tol=2.5 * step)
    want = [bool(np.any(O.round_bf16(np.linspace(t - 2.5 * step, t + 2.5 * step, 4001)) == c))
            for c in cand]
    assert list(ok) == want and 5 <= sum(want) <= 6
    # brute force: r is accepted exactly when some value within eps rounds to it
    g = np.random.default_rng(7)
    v = g.normal(size=400)
    eps = 2.0 ** -9 * np.abs(v)
    below = lambda a: float(O.round_bf16_down(np.nextafter(a, -np.inf)))   # next bf16 down
    above = lambda a: float(O.round_bf16_up(np.nextafter(a, np.inf)))      # next bf16 up
    for vi, ei in zip(v, eps):
        grid = np.linspace(vi - ei, vi + ei, 2001)
        reach = set(O.round_bf16(grid).tolist())
        lo, hi = min(reach), max(reach)
        for r in (lo, hi, below(lo), above(hi)):
            assert bool(O.bf16_rounding_ok([vi], [r], rel=2.0 ** -9)[0]) == (r in reach), (vi, r)


def _small_layer():
    cfg = dict(hidden=512, layers=1, heads=4, kv_heads=2, head_dim=128, ffn=1024, vocab=300,
               eps=1e-6, theta=1e6)
    w = qg_synth.qwen3_weights(cfg, 9, norm_jitter=0.1)
    x = O.embed_rows(*w["embed"], [17])[0]
    kc, vc = O.new_kv_cache(cfg, 16)
    kc[:] = O.bf16_bits_to_f64(qg_synth.gaussian_bf16_bits(kc.shape, 1.0, 3))
    vc[:] = O.bf16_bits_to_f64(qg_synth.gaussian_bf16_bits(vc.shape, 1.0, 4))
    return cfg, w["layers"][0], x, kc[0], vc[0]


# ---- float32 emulation of one decoder layer (test code): the same ops as the
# oracle's layer in numpy float32, in orders of its own (sequential sums,
# an online softmax over row batches), for the bound pins below.

F32 = np.float32


def _f32_rmsnorm(x, w_bits, eps):
    x = np.asarray(x, F32)
    ss = F32(0)
    for v in x:                        # sequential: the longest chain
        ss = F32(ss + F32(v * v))
    inv = F32(1) / F32(np.sqrt(F32(F32(ss / F32(x.size)) + F32(eps))))
    return F32(x * inv) * F32(O.bf16_bits_to_f64(w_bits))


def _f32_norm_rope(x, w_bits, eps, pos, theta, D):
    h = np.asarray(x, F32).reshape(-1, D)
    out = np.empty_like(h)
    a = pos * O.rope_inv_freq(theta, D)
    c, s = F32(np.cos(a)), F32(np.sin(a))
    for i in range(h.shape[0]):
        n = _f32_rmsnorm(h[i], w_bits, eps)
        x1, x2 = n[:D // 2], n[D // 2:]
        out[i, :D // 2] = F32(x1 * c) - F32(x2 * s)
        out[i, D // 2:] = F32(x2 * c) + F32(x1 * s)
    return out.ravel()


def _f32_attention(q, kc, vc, L, H, Hkv, D, batch=24, round_q=False, round_p=False):
    """Online softmax over batches of rows, float32, like the kernels; with
    round_q / round_p the query / the weights are rounded to bf16 first (the
    multi-row kernel's tensor-core operands)."""
    if round_q:
        q = O.round_bf16(np.asarray(q, F32))
    q = np.asarray(q, F32).reshape(H, D) * F32(F32(1) / F32(np.sqrt(F32(D))))
    out = np.zeros((H, D), F32)
    g = H // Hkv
    for h in range(H):
        K_, V_ = kc[h // g, :L].astype(F32), vc[h // g, :L].astype(F32)
        m, l, o = F32(-np.inf), F32(0), np.zeros(D, F32)
        for t0 in range(0, L, batch):
            sc = (K_[t0:t0 + batch] @ q[h]).astype(F32)
            mx = F32(max(m, sc.max()))
            a = F32(np.exp(F32(m - mx)))
            l, o = F32(l * a), (o * a).astype(F32)
            for t in range(sc.size):
                p = F32(np.exp(F32(sc[t] - mx)))
                if round_p:
                    p = F32(O.round_bf16(p))
                l = F32(l + p)
                o = (o + p * V_[t0 + t]).astype(F32)
            m = mx
        out[h] = o / l
    return out.ravel()


def _f32_gemv(lw_m, x):
    w = O.affine8_dequant_f32(*lw_m)
    return (w @ np.asarray(x, F32)).astype(F32)


def _f32_silu_mul(gate, up):
    z = np.asarray(gate, F32)
    return (F32(z / F32(F32(1) + np.exp(-z).astype(F32))) * np.asarray(up, F32)).astype(F32)


def _f32_layer(cfg, lw, x, kc, vc, pos):
    """One layer in float32 with bf16 stores at the rounding points: the
    values another implementation would hand to decode_layer_forced."""
    H, Hkv, D, eps, th = cfg["heads"], cfg["kv_heads"], cfg["head_dim"], cfg["eps"], cfg["theta"]
    r = {}
    r["xn"] = O.round_bf16(_f32_rmsnorm(x, lw["input_norm"], eps))
    r["q_proj"] = _f32_gemv(lw["q"], r["xn"])
    r["k_proj"] = _f32_gemv(lw["k"], r["xn"])
    r["v_proj"] = _f32_gemv(lw["v"], r["xn"])
    r["k"] = O.round_bf16(_f32_norm_rope(r["k_proj"], lw["k_norm"], eps, pos, th, D))
    r["v"] = O.round_bf16(r["v_proj"])
    k1, v1 = kc.copy(), vc.copy()
    k1[:, pos, :] = r["k"].reshape(Hkv, D)
    v1[:, pos, :] = r["v"].reshape(Hkv, D)
    qp = _f32_norm_rope(r["q_proj"], lw["q_norm"], eps, pos, th, D)
    r["att"] = O.round_bf16(_f32_attention(qp, k1, v1, pos + 1, H, Hkv, D))
    r["x_attn"] = (np.asarray(x, F32) + _f32_gemv(lw["o"], r["att"])).astype(F32)
    r["xn2"] = O.round_bf16(_f32_rmsnorm(r["x_attn"], lw["post_norm"], eps))
    r["gate"] = _f32_gemv(lw["gate"], r["xn2"])
    r["up"] = _f32_gemv(lw["up"], r["xn2"])
    r["h"] = O.round_bf16(_f32_silu_mul(r["gate"], r["up"]))
    y = (r["x_attn"] + _f32_gemv(lw["down"], r["h"])).astype(F32)
    return {k: np.asarray(v, np.float64) for k, v in r.items()}, y.astype(np.float64)


def test_float32_op_chains_stay_within_their_derived_bounds():
    """Each bound holds for a float32 evaluation of its chain (sequential
    sums, batched online softmax), and is not vacuous: far below half a bf16
    step relative to the values it bounds."""
    rng = np.random.default_rng(5)
    cfg, lw, x, kc, vc = _small_layer()
    eps, th, D = cfg["eps"], cfg["theta"], cfg["head_dim"]
    xf = rng.standard_normal(512).astype(F32) * F32(3)
    v = O.rmsnorm(xf, lw["input_norm"], eps)
    err = np.abs(_f32_rmsnorm(xf, lw["input_norm"], eps) - v)
    rel = O.rmsnorm_rel_bound(512)
    assert np.all(err <= rel * np.abs(v)) and rel < 2.0 ** -17
    kp = rng.standard_normal(2 * D).astype(F32)
    kr, kb = O.norm_rope_bound(kp, lw["k_norm"], eps, 9, th, D)
    assert np.all(np.abs(_f32_norm_rope(kp, lw["k_norm"], eps, 9, th, D) - kr) <= kb)
    assert np.max(kb) < 2.0 ** -16 * np.sqrt(np.mean(kr ** 2)) * 8
    H, Hkv = cfg["heads"], cfg["kv_heads"]
    qp = rng.standard_normal(H * D).astype(F32)
    att, ab = O.attention_bound(qp, np.zeros(H * D), kc, vc, 10, H, Hkv, D)
    np.testing.assert_allclose(att, O.decode_attention(qp, kc, vc, 10, H, Hkv, D), atol=1e-12)
    assert np.all(np.abs(_f32_attention(qp, kc, vc, 10, H, Hkv, D) - att) <= ab)
    assert np.max(ab) < 2.0 ** -14 * np.max(np.abs(vc))
    # bf16 query and weights (the multi-row kernel): within the widened bound
    _, abr = O.attention_bound(qp, np.zeros(H * D), kc, vc, 10, H, Hkv, D, 2.0 ** -8, 2.0 ** -8)
    f32r = _f32_attention(qp, kc, vc, 10, H, Hkv, D, round_q=True, round_p=True)
    assert np.all(np.abs(f32r - att) <= abr) and np.any(np.abs(f32r - att) > ab)
    # a query known only within dq widens the bound by about the score error
    _, ab2 = O.attention_bound(qp, np.full(H * D, 1e-3), kc, vc, 10, H, Hkv, D)
    assert np.all(ab2 > ab)
    g, u = rng.standard_normal(1000).astype(F32) * F32(4), rng.standard_normal(1000).astype(F32)
    hm = O.silu_mul(g, u)
    assert np.all(np.abs(_f32_silu_mul(g, u) - hm) <= O.silu_mul_rel_bound() * np.abs(hm))


def test_decode_layer_forced_accepts_a_float32_layer_and_follows_it():
    """A float32 layer with bf16 stores passes every rounding check; its GEMV
    outputs meet the float32-accumulation tolerance against the references;
    and the returned output follows the forced values."""
    cfg, lw, x, kc, vc = _small_layer()
    forced, y32 = _f32_layer(cfg, lw, x, kc, vc, 9)
    k2, v2 = kc.copy(), vc.copy()
    refs, bad = O.decode_layer_forced(cfg, lw, x, k2, v2, 9, forced)
    assert set(bad) == set(O.LAYER_BF16_POINTS)
    assert all(b.size == 0 for b in bad.values()), {k: b[:5] for k, b in bad.items()}
    for name in O.LAYER_FP32_POINTS:
        np.testing.assert_allclose(forced[name], refs[name], rtol=1e-3, atol=2e-3)
    np.testing.assert_allclose(y32, refs["y"], rtol=1e-3, atol=2e-3)
    np.testing.assert_array_equal(k2[:, 9, :].ravel(), forced["k"])
    # with its own rounded values forced, the float64 layer is reproduced
    # up to the float32 GEMV outputs it is then fed
    y64 = O.decode_layer(cfg, lw, x, kc.copy(), vc.copy(), 9)
    np.testing.assert_allclose(refs["y"], y64, rtol=1e-3, atol=2e-3)


def test_decode_layer_forced_flags_planted_mistakes():
    """Mistakes a kernel could make are flagged at their rounding point: a
    value two bf16 steps off, gate and up swapped in the SiLU-mul, the RoPE
    sign flipped, a K/V head taken from the wrong head, an attention output
    row of another head; a missing or misnamed point is an error."""
    cfg, lw, x, kc, vc = _small_layer()
    H, Hkv, D = cfg["heads"], cfg["kv_heads"], cfg["head_dim"]
    forced, _ = _f32_layer(cfg, lw, x, kc, vc, 9)

    def bad_of(**change):
        f = dict(forced, **change)
        return O.decode_layer_forced(cfg, lw, x, kc.copy(), vc.copy(), 9, f)[1]

    two = forced["xn"].copy()
    two[5] = O.round_bf16_up(O.round_bf16_up(two[5] * (1 + 2.0 ** -7)) * (1 + 2.0 ** -7))
    assert list(bad_of(xn=two)["xn"]) == [5]
    swapped = O.round_bf16(O.silu_mul(forced["up"], forced["gate"]))
    assert bad_of(h=swapped)["h"].size > 0.5 * swapped.size
    kp = O.rmsnorm_perhead(forced["k_proj"], lw["k_norm"], cfg["eps"], D)
    wrong_sign = O.round_bf16(O.rope_neox(kp, -9, cfg["theta"], D))
    assert bad_of(k=wrong_sign)["k"].size > 0.5 * wrong_sign.size
    v_heads = forced["v"].reshape(Hkv, D)[::-1].ravel()
    assert bad_of(v=v_heads)["v"].size > 0.5 * v_heads.size
    att_rows = forced["att"].reshape(H, D)[[1, 0] + list(range(2, H))].ravel()
    assert bad_of(att=att_rows)["att"].size > 0.5 * D
    with pytest.raises(KeyError):
        O.decode_layer_forced(cfg, lw, x, kc.copy(), vc.copy(), 9,
                              {k: v for k, v in forced.items() if k != "h"})
    f = dict(forced)
    f["attn"] = f.pop("att")
    with pytest.raises(KeyError):
        O.decode_layer_forced(cfg, lw, x, kc.copy(), vc.copy(), 9, f)


def test_lm_head_tie_bound_is_the_exact_linear_effect_of_each_tie():
    cfg = dict(hidden=256, layers=0, heads=2, kv_heads=1, head_dim=128, ffn=256, vocab=500,
               eps=1e-6, theta=1e6)
    w = qg_synth.qwen3_weights(cfg, 4, norm_jitter=0.2)
    x = qg_synth.gaussian((256,), 1.0, 5).astype(np.float64)
    logits, ex0 = O.lm_head_tie_bound(cfg, w, x, rel=0.0)
    np.testing.assert_array_equal(logits, O.lm_head(cfg, w, x))
    assert np.all(ex0 == 0)
    rel = 2.0 ** -9   # a quarter of the values count as ties
    _, ex = O.lm_head_tie_bound(cfg, w, x, rel=rel)
    v = O.rmsnorm(x, w["final_norm"], cfg["eps"])
    xn = O.round_bf16(v)
    alt = O.bf16_alternative(v, rel)
    ties = np.flatnonzero(~np.isnan(alt))
    assert ties.size > 0
    brute = np.zeros_like(logits)
    for j in ties:   # one tie at a time through the full head
        xa = xn.copy()
        xa[j] = alt[j]
        brute += np.abs(O.gemv_affine8(*w["embed"], xa[None])[0] - logits)
    np.testing.assert_allclose(ex, brute, rtol=1e-9, atol=1e-12)


def test_code_predict_chain_indices_and_concat_order():
    """A code predictor built by hand (no layers, hidden = vocab = 64, 4 code
    groups): input_proj = [0 | I] passes the code embedding through and drops
    the LM hidden state; table j maps code t to a one-hot at (t + j) mod 64;
    head g maps a one-hot at c to the logit row (c + 10 g) mod 64. So group
    g's code is (previous + (g - 1) + 10 g) mod 64: from 5 the chain is 15,
    36, 4. Using table g or head g - 1, or the concatenation in the other
    order, gives another chain."""
    h = V = 64
    G = 4
    cfg = dict(hidden=h, layers=0, heads=1, kv_heads=1, head_dim=64, ffn=64, vocab=V,
               eps=1e-6, theta=1e6)
    eye = np.eye(h)
    ip = np.concatenate([np.zeros((h, h)), eye], axis=1)
    tables = [np.roll(eye, j, axis=1) for j in range(G)]       # row t: one-hot at t + j
    heads = [np.roll(eye, 10 * g, axis=0) for g in range(G)]   # column c -> row c + 10 g
    w = {"input_proj": O.affine8_quantize(ip),
         "code_embed": [O.affine8_quantize(t) for t in tables],
         "heads": [O.affine8_quantize(m) for m in heads],
         "layers": [], "final_norm": np.full(h, 0x3F80, dtype=np.uint16)}
    lm_hidden = qg_synth.gaussian((h,), 1.0, 3)
    codes, logits = O.code_predict(cfg, w, lm_hidden, 5)
    assert codes == [5, 15, 36, 4]
    assert len(logits) == G - 1 and all(lg.shape == (V,) for lg in logits)
    # group 1's logits directly: one nonzero logit, at 15
    lg = O.code_predict_group(cfg, w, lm_hidden, 5, 1)
    assert np.count_nonzero(lg > 1.0) == 1 and int(np.argmax(lg)) == 15


def _golden_penalty():
    path = os.path.join(os.path.dirname(__file__), "golden", "repetition_penalty_example.txt")
    d = {}
    for line in open(path):
        if line.strip() and not line.startswith("#"):
            k, *v = line.split()
            d[k] = v
    return d


def test_repetition_penalty_worked_example_and_order():
    d = _golden_penalty()
    got = O.apply_repetition_penalty([float(v) for v in d["logits"]], [int(v) for v in d["past"]],
                                     float(d["penalty"][0]))
    np.testing.assert_allclose(got, [float(v) for v in d["expected"]], rtol=1e-6)
    # negative scores are multiplied; every occurrence counts, in float32;
    # tokens outside the vocabulary are skipped
    got = O.apply_repetition_penalty([-1.0, 2.0, 0.5], [0, 0, 1, -1, 3], 1.2)
    p = np.float32(1.2)
    assert got[0] == np.float32(np.float32(-1.0) * p) * p
    assert got[1] == np.float32(2.0) / p and got[2] == np.float32(0.5)


def test_sample_token_distribution_ties_nan_and_greedy():
    lg = np.log(np.array([1.0, 2.0, 3.0], dtype=np.float32))   # probabilities 1/6, 2/6, 3/6
    # descending order 2, 1, 0 with running sums 1/2, 5/6, 1
    assert O.sample_token(lg, [], 1.0, 1.0, 3, 0.4) == 2
    assert O.sample_token(lg, [], 1.0, 1.0, 3, 0.6) == 1
    assert O.sample_token(lg, [], 1.0, 1.0, 3, 0.95) == 0
    rs = (np.arange(1000) + 0.5) / 1000
    counts = np.bincount([O.sample_token(lg, [], 1.0, 1.0, 3, r) for r in rs], minlength=3)
    np.testing.assert_allclose(counts / 1000, [1 / 6, 2 / 6, 3 / 6], atol=2e-3)
    # top_k = 1 and r = 0 give the maximum; top_k = 2 drops index 0
    assert O.sample_token(lg, [], 1.0, 1.0, 1, 0.99) == 2
    assert O.sample_token(lg, [], 1.0, 1.0, 3, 0.0) == 2
    assert all(O.sample_token(lg, [], 1.0, 1.0, 2, r) in (1, 2) for r in rs)
    # equal values keep index order (a stable sort)
    eq = np.array([5.0, 5.0, 1.0], dtype=np.float32)
    assert O.sample_token(eq, [], 1.0, 1.0, 2, 0.3) == 0
    assert O.sample_token(eq, [], 1.0, 1.0, 2, 0.7) == 1
    # a NaN score is never drawn; temperature 0 or top_k 0 is greedy after
    # the penalty (which here moves the maximum from 2 to 1)
    nanl = np.array([np.nan, 1.0, 2.0], dtype=np.float32)
    assert all(O.sample_token(nanl, [], 1.0, 1.0, 3, r) in (1, 2) for r in rs)
    pen = np.array([0.0, 1.9, 2.0], dtype=np.float32)
    assert O.sample_token(pen, [2], 1.2, 0.0, 5, 0.5) == 1
    assert O.sample_token(pen, [2], 1.2, 1.0, 0, 0.5) == 1
    # a lower temperature sharpens: at T = 0.1 the probabilities are in the
    # ratio 1 : 2^10 : 3^10
    counts = np.bincount([O.sample_token(lg, [], 1.0, 0.1, 3, r) for r in rs], minlength=3)
    tot = 1 + 2 ** 10 + 3 ** 10
    np.testing.assert_allclose(counts / 1000, [1 / tot, 2 ** 10 / tot, 3 ** 10 / tot], atol=2e-3)


def test_token_logprob_closed_forms_and_library_logsumexp():
    from scipy.special import logsumexp
    V = 1000
    assert O.token_logprob(np.zeros(V), 17) == pytest.approx(-math.log(V), abs=1e-12)
    x = qg_synth.gaussian((V,), 3.0, 8).astype(np.float64)
    for t in (0, 17, int(np.argmax(x))):
        assert O.token_logprob(x, t) == pytest.approx(x[t] - logsumexp(x), abs=1e-12)
        assert O.token_logprob(x + 1e4, t) == pytest.approx(O.token_logprob(x, t), abs=1e-9)
    one_hot = np.full(V, -1e4)
    one_hot[3] = 0.0
    assert O.token_logprob(one_hot, 3) == pytest.approx(0.0, abs=1e-12)
    assert math.isnan(O.token_logprob(x, V)) and math.isnan(O.token_logprob(x, -1))
    x[5] = np.nan
    assert math.isnan(O.token_logprob(x, 0))
