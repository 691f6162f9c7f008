"""GPU parity of the single-op kernels against the oracle (through the C ABI).

Unpack and dequant are compared bit for bit; fp32-accumulated outputs within
|gpu - ref| <= 2e-3 + 1e-3 |ref| (plus half a bf16 ulp for bf16 stores).
Shapes span several tiles with ragged tails, the degenerate sizes (one row,
one group, batch 1 and 32) and the full model shapes (sampled rows where the
oracle would be too slow for all of them).
"""
import math

import numpy as np
import pytest
import torch

import qg_synth
from oracle import qg_oracle as O
from tests.gpu_util import assert_parity, bf16_dev, dev, host64

pytestmark = pytest.mark.gpu

qg = pytest.importorskip("weight_only_quantized_03_b200")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _affine8(N, K, seed, quantized):
    if quantized:
        return O.affine8_quantize(qg_synth.gaussian((N, K), 0.02, seed))
    return qg_synth.affine8_packed(N, K, seed)


# ----------------------------------------------------------- bit-exact -----

@pytest.mark.parametrize("N,K,kind", [(3, 64, "fixture"), (33, 192, "quantized"),
                                      (2048, 1024, "random")])
def test_unpack_and_dequant_affine8_bit_exact(N, K, kind):
    if kind == "fixture":
        w, s, b = qg_synth.affine8_fixture(N, K, 0x5EED12340001)
    else:
        w, s, b = _affine8(N, K, 7, kind == "quantized")
    out = torch.empty((N, K), dtype=torch.float32, device="cuda")
    qg.qg_unpack_affine8(dev(w), out)
    np.testing.assert_array_equal(out.cpu().numpy(), O.affine8_unpack(w).astype(np.float32))
    qg.qg_dequant_affine8_g64(dev(w), dev(s), dev(b), out)
    np.testing.assert_array_equal(out.cpu().numpy().view(np.uint32),
                                  O.affine8_dequant_f32(w, s, b).view(np.uint32))


@pytest.mark.parametrize("N,K,kind", [(17, 96, "quantized"), (1280, 1280, "random"),
                                      (5, 5120, "random")])
def test_dequant_q4_0_bit_exact(N, K, kind):
    blocks = (O.q4_0_quantize(qg_synth.gaussian((N, K), 0.02, 8)) if kind == "quantized"
              else qg_synth.q4_0_packed(N, K, 9))
    out = torch.empty((N, K), dtype=torch.float32, device="cuda")
    qg.qg_dequant_q4_0(dev(blocks), out)
    got = out.cpu().numpy()
    want = O.q4_0_dequant_exact(blocks, K).astype(np.float32)
    np.testing.assert_array_equal(got, want)                       # -0.0 == +0.0 here
    np.testing.assert_array_equal(np.signbit(got), np.signbit(want))


# ------------------------------------------------------- affine8 GEMV ------

GEMV_CASES = [
    # N, K, B, x_dtype, y_dtype, residual, quantized weights
    (1, 64, 1, "bf16", "f32", False, True),
    (7, 128, 3, "bf16", "f32", True, True),
    (1000, 1024, 1, "bf16", "f32", False, False),
    (1024, 1024, 1, "bf16", "bf16", False, True),
    (2048, 1024, 4, "bf16", "f32", False, False),
    (3072, 1024, 16, "bf16", "f32", False, False),
    (1024, 3072, 1, "bf16", "f32", True, False),
    (1024, 2048, 2, "f32", "f32", True, False),
    (33, 192, 32, "bf16", "bf16", False, True),
    (4100, 64, 9, "f32", "f32", False, False),
    (300, 6144, 5, "bf16", "f32", False, False),
    (9473, 256, 1, "bf16", "f32", False, False),
    (40000, 128, 2, "bf16", "f32", False, False),
    # the tensor-core streaming path (bf16 x, K % 512 == 0, B <= 32): ragged
    # rows, one or two n-tiles, batch tiles of 8 past B = 8, column splits over 2, 4 and 8 warps
    # (uneven when K / 512 is not a multiple), residual, bf16 output
    (1001, 512, 8, "bf16", "bf16", True, True),
    (1001, 512, 32, "bf16", "bf16", True, True),
    (2050, 2048, 8, "bf16", "f32", True, False),
    (17, 1024, 3, "bf16", "f32", False, True),
    (5000, 3072, 5, "bf16", "f32", False, False),
    (64, 3072, 1, "bf16", "f32", True, False),
    (3, 1536, 6, "bf16", "bf16", False, False),
    (16, 4096, 1, "bf16", "bf16", False, False),
    (200, 8192, 2, "bf16", "f32", False, False),
    (2050, 2048, 9, "bf16", "f32", True, False),    # two batch tiles, the second of 1 row
    (1024, 3072, 24, "bf16", "bf16", True, False),  # three batch tiles
]


@pytest.mark.parametrize("N,K,B,xd,yd,res,quant", GEMV_CASES)
def test_gemv_affine8(N, K, B, xd, yd, res, quant):
    w, s, b = _affine8(N, K, 100 + N + K + B, quant)
    xbits = qg_synth.gaussian_bf16_bits((B, K), 1.0, 200 + B)
    if xd == "bf16":
        x_d = bf16_dev(xbits)
        x64 = O.bf16_bits_to_f64(xbits)
    else:
        xf = qg_synth.gaussian((B, K), 1.0, 201 + B)
        x_d = dev(xf)
        x64 = xf.astype(np.float64)
    r = qg_synth.gaussian((B, N), 1.0, 300) if res else None
    y = torch.empty((B, N), dtype=torch.float32 if yd == "f32" else torch.bfloat16, device="cuda")
    if res and yd == "f32":
        y.copy_(dev(r))            # in place: y = W x + y
        rr = y
    else:
        rr = dev(r) if res else None
    qg.qg_gemv_affine8_g64(dev(w), dev(s), dev(b), x_d, y, residual=rr)
    ref = O.gemv_affine8(w, s, b, x64, residual=r)
    assert_parity(host64(y), ref, bf16_out=(yd == "bf16"), what=f"gemv {N}x{K} B={B}")


@pytest.mark.parametrize("B,K", [(2, 1024), (8, 2048)])
def test_gemv_affine8_large_activations_prescaled(B, K):
    # |x| far beyond fp16's range: the tensor-core path prescales x by a
    # power of two, so the products stay exact and nothing overflows (B x K
    # = 8 x 2048 takes the bulk copy of x into shared memory)
    N = 300
    w, s, b = qg_synth.affine8_packed(N, K, 77)
    xf = (qg_synth.gaussian((B, K), 1.0, 78) * 2.0 ** 20).astype(np.float32)
    xbits = qg_synth.f32_to_bf16_bits(xf)
    y = torch.empty((B, N), dtype=torch.float32, device="cuda")
    qg.qg_gemv_affine8_g64(dev(w), dev(s), dev(b), bf16_dev(xbits), y)
    ref = O.gemv_affine8(w, s, b, O.bf16_bits_to_f64(xbits))
    assert_parity(host64(y), ref, what="prescaled x")


def test_gemv_affine8_lm_head_full_size_sampled_rows():
    # the tied LM head of the 0.6B shape: 151936 x 1024, batch 1 and 4 (the
    # tensor-core GEMV) and 5, 16, 32 (the tensor-core matmul, which takes
    # batches past 4 for matrices of a wave of 128-row tiles or more)
    N, K = 151936, 1024
    w, s, b = qg_synth.affine8_packed(N, K, 4242)
    for B in (1, 4, 5, 16, 32):
        xbits = qg_synth.gaussian_bf16_bits((B, K), 1.0, 4243 + B)
        y = torch.empty((B, N), dtype=torch.float32, device="cuda")
        qg.qg_gemv_affine8_g64(dev(w), dev(s), dev(b), bf16_dev(xbits), y)
        rows = np.sort(np.random.default_rng(B).choice(N, 3000, replace=False))
        rows = np.concatenate([[0, N - 1], rows])
        ref = O.gemv_affine8(w[rows], s[rows], b[rows], O.bf16_bits_to_f64(xbits))
        assert_parity(host64(y)[:, rows], ref, what=f"lm head B={B}")


# ---------------------------------------------------------- Q4_0 GEMV ------

Q4_CASES = [
    (1280, 1280, 1, True, False), (5120, 1280, 1, True, False), (1280, 5120, 1, True, False),
    (1280, 1280, 1, False, True), (7, 32, 3, True, True), (100, 96, 32, False, False),
    (64, 256, 8, True, False), (333, 2048, 5, False, False),
]


@pytest.mark.parametrize("N,K,B,bias,quant", Q4_CASES)
def test_gemv_q4_0(N, K, B, bias, quant):
    blocks = (O.q4_0_quantize(qg_synth.gaussian((N, K), 0.02, 11)) if quant
              else qg_synth.q4_0_packed(N, K, 12))
    x = qg_synth.gaussian((B, K), 1.0, 13)
    bv = qg_synth.gaussian((N,), 1.0, 14) if bias else None
    y = torch.empty((B, N), dtype=torch.float32, device="cuda")
    qg.qg_gemv_q4_0(dev(blocks), dev(x), y, bias=dev(bv) if bias else None)
    ref = O.gemv_q4_0(blocks, x.astype(np.float64), None if bv is None else bv.astype(np.float64))
    assert_parity(host64(y), ref, what=f"q4_0 gemv {N}x{K} B={B}")


# ---------------------------------------------------- Q4_0 GEMM (tcgen05) -

GEMM_CASES = [
    # M, N, K, bias, quantized weights
    (1, 128, 64, False, True),
    (130, 256, 128, True, True),       # ragged M, one 256-column tile
    (200, 384, 192, True, False),      # 128-column tiles, three K stages
    (257, 512, 1280, False, False),    # K ring wraps (20 stages over 4)
    (5, 128, 256, True, True),         # one raw chunk of W (K = 256), a 5-row A tile
    # the Whisper-large-v3 encoder projections at M = 1500 frames
    (1500, 1280, 1280, True, False),
    (1500, 5120, 1280, True, False),
    (1500, 1280, 5120, True, False),
    # two 128-row A sub-tiles per CTA, the last CTA's second one wholly past M
    (1300, 5120, 128, True, False),
]


@pytest.mark.parametrize("M,N,K,bias,quant", GEMM_CASES)
def test_gemm_q4_0(M, N, K, bias, quant):
    blocks = (O.q4_0_quantize(qg_synth.gaussian((N, K), 0.02, 21)) if quant
              else qg_synth.q4_0_packed(N, K, 22))
    A = qg_synth.gaussian((M, K), 1.0, 23)
    bv = qg_synth.gaussian((N,), 1.0, 24) if bias else None
    C = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.empty(qg.qg_gemm_q4_0_workspace_size(M, N, K), dtype=torch.uint8, device="cuda")
    qg.qg_gemm_q4_0(dev(blocks), dev(A), C, bias=dev(bv) if bias else None, ws=ws)
    assert qg.qg_gemm_q4_0_error(M, K, ws) == (0, 0)
    ref = O.gemm_q4_0_bf16(blocks, A, None if bv is None else bv.astype(np.float64))
    assert_parity(host64(C), ref, what=f"q4_0 gemm {M}x{N}x{K}")


def test_gemm_q4_0_two_byte_aligned_blocks():
    # blocks only 2-byte aligned: W bytes are read 16 bits at a time
    M, N, K = 300, 512, 256
    blocks = qg_synth.q4_0_packed(N, K, 31)
    buf = torch.zeros(blocks.size + 2, dtype=torch.uint8, device="cuda")
    buf[2:].copy_(dev(blocks).view(-1))
    bl = buf[2:].view(N, -1)
    A = qg_synth.gaussian((M, K), 1.0, 32)
    C = torch.empty((M, N), dtype=torch.float32, device="cuda")
    ws = torch.empty(qg.qg_gemm_q4_0_workspace_size(M, N, K), dtype=torch.uint8, device="cuda")
    qg.qg_gemm_q4_0(bl, dev(A), C, ws=ws)
    assert qg.qg_gemm_q4_0_error(M, K, ws) == (0, 0)
    assert_parity(host64(C), O.gemm_q4_0_bf16(blocks, A), what="q4_0 gemm, 2-byte aligned blocks")


# -------------------------------------------------------- elementwise ------

@pytest.mark.parametrize("rows,dim,eps,yd", [(1, 1024, 1e-6, "bf16"), (10, 1024, 1e-6, "f32"),
                                             (3, 64, 1e-5, "bf16"), (2, 2048, 1e-6, "bf16"),
                                             (5, 4, 1e-6, "f32")])
def test_rmsnorm(rows, dim, eps, yd):
    x = qg_synth.gaussian((rows, dim), 3.0, 20)
    w = qg_synth.f32_to_bf16_bits((1 + 0.2 * qg_synth.gaussian((dim,), 1.0, 21)).astype(np.float32))
    y = torch.empty((rows, dim), dtype=torch.float32 if yd == "f32" else torch.bfloat16,
                    device="cuda")
    qg.qg_rmsnorm(dev(x), dev(w), eps, y)
    assert_parity(host64(y), O.rmsnorm(x, w, eps), bf16_out=(yd == "bf16"), what="rmsnorm")


@pytest.mark.parametrize("xd,yd,D", [("f32", "f32", 128), ("bf16", "bf16", 128),
                                     ("f32", "bf16", 64), ("f32", "f32", 256)])
def test_rmsnorm_perhead(xd, yd, D):
    rows, heads = 3, 16
    xf = qg_synth.gaussian((rows, heads * D), 2.0, 22)
    w = qg_synth.f32_to_bf16_bits((1 + 0.2 * qg_synth.gaussian((D,), 1.0, 23)).astype(np.float32))
    if xd == "bf16":
        bits = qg_synth.f32_to_bf16_bits(xf)
        x_d, x64 = bf16_dev(bits), O.bf16_bits_to_f64(bits)
    else:
        x_d, x64 = dev(xf), xf.astype(np.float64)
    y = torch.empty((rows, heads * D), dtype=torch.float32 if yd == "f32" else torch.bfloat16,
                    device="cuda")
    qg.qg_rmsnorm_perhead(x_d, dev(w), 1e-6, y, heads)
    assert_parity(host64(y), O.rmsnorm_perhead(x64, w, 1e-6, D), bf16_out=(yd == "bf16"),
                  what="perhead")


@pytest.mark.parametrize("dt,rd,theta", [("f32", 128, 1e6), ("bf16", 128, 1e6), ("f32", 64, 1e4)])
def test_rope_neox(dt, rd, theta):
    D, heads = 128, 8
    pos = np.array([0, 1, 511, 2047, 32767], dtype=np.int32)
    xf = qg_synth.gaussian((len(pos), heads * D), 1.0, 24)
    if dt == "bf16":
        bits = qg_synth.f32_to_bf16_bits(xf)
        x_d, x64 = bf16_dev(bits), O.bf16_bits_to_f64(bits)
    else:
        x_d, x64 = dev(xf), xf.astype(np.float64)
    qg.qg_rope_neox(x_d, dev(pos), theta, heads, rotary_dim=rd)
    ref = np.stack([O.rope_neox(x64[i], int(p), theta, D, rd) for i, p in enumerate(pos)])
    assert_parity(host64(x_d), ref, bf16_out=(dt == "bf16"), what="rope")


@pytest.mark.parametrize("n,od", [(3072, "bf16"), (30720, "f32"), (1, "bf16")])
def test_silu_mul(n, od):
    g = qg_synth.gaussian((n,), 4.0, 25)
    u = qg_synth.gaussian((n,), 1.0, 26)
    out = torch.empty(n, dtype=torch.float32 if od == "f32" else torch.bfloat16, device="cuda")
    qg.qg_silu_mul(dev(g), dev(u), out)
    assert_parity(host64(out), O.silu_mul(g, u), bf16_out=(od == "bf16"), what="silu_mul")


def test_residual_add():
    x = qg_synth.gaussian((5000,), 1.0, 27)
    d = qg_synth.gaussian((5000,), 1.0, 28)
    xd = dev(x)
    qg.qg_residual_add(xd, dev(d))
    assert_parity(host64(xd), x.astype(np.float64) + d, what="residual")


def test_embed_rows_bit_exact_and_bad_token():
    V, Hd = 261, 64
    w, s, b = qg_synth.affine8_fixture(V, Hd, 0x5EED12340001)
    toks = np.array([0, 260, 17, -1, 261], dtype=np.int32)
    x = torch.empty((len(toks), Hd), dtype=torch.float32, device="cuda")
    qg.qg_embed_affine8_g64(dev(w), dev(s), dev(b), dev(toks), x)
    got = x.cpu().numpy()
    np.testing.assert_array_equal(got[:3], O.embed_rows(w, s, b, toks[:3]).astype(np.float32))
    assert np.isnan(got[3:]).all()


# ---------------------------------------------------------- attention ------

ATTN_CASES = [
    # B, H, Hkv, D, cap, kv_len per sequence
    (1, 16, 8, 128, 513, [512]),
    (1, 16, 8, 128, 513, [1]),
    (2, 16, 8, 128, 600, [33, 600]),
    (3, 2, 1, 64, 70, [31, 32, 64]),
    (1, 4, 4, 256, 40, [40]),
    (10, 16, 8, 128, 513, [512, 1, 100, 511, 256, 2, 3, 400, 512, 77]),
    (1, 16, 8, 128, 2048, [2048]),
    (1, 16, 8, 128, 2049, [1500]),     # clusters of 16 (chunks of 129 rows), the last ones empty
    (2, 8, 1, 32, 5, [0, 6]),          # invalid lengths -> zero rows
    (4, 16, 4, 128, 300, [300, 1, 150, 299]),   # 4 query heads per kv head
    (2, 6, 2, 64, 100, [100, 37]),              # 3 query heads per kv head
    (1, 4, 2, 96, 50, [50]),                    # head_dim 96: the split kernel
    (32, 16, 8, 128, 16, [16, 1, 2, 15] * 8),   # many sequences, one-CTA clusters
    (1, 2, 2, 32, 1000, [999]),                 # head_dim 32, long chunks
    (2, 16, 16, 64, 1, [1, 1]),                 # MHA, head_dim 64, one row (code predictor)
    (1, 16, 16, 64, 300, [300]),                # MHA, head_dim 64
    # the tensor-core kernel (B * Hkv * cap >= 2^16): one CTA per pair,
    # clusters of 4 and of 8, 8 query heads per KV head, ragged last blocks
    (32, 16, 8, 128, 2048, [2048, 1, 2047, 64, 65, 1000, 0, 2048] * 4),
    (8, 16, 8, 128, 2048, [2048, 1, 2047, 63, 513, 1000, 2049, 1536]),
    (4, 16, 2, 64, 8192, [8192, 1, 5000, 129]),
    (1, 8, 1, 128, 65536, [65536]),
]


@pytest.mark.parametrize("B,H,Hkv,D,cap,lens", ATTN_CASES)
def test_decode_attention(B, H, Hkv, D, cap, lens):
    kbits = qg_synth.gaussian_bf16_bits((B, Hkv, cap, D), 1.0, 30)
    vbits = qg_synth.gaussian_bf16_bits((B, Hkv, cap, D), 1.0, 31)
    q = qg_synth.gaussian((B, H * D), 1.0, 32)
    kv_len = np.array(lens, dtype=np.int32)
    ws = torch.empty(qg.qg_decode_attention_workspace_size(B, H, Hkv, D, cap), dtype=torch.uint8,
                     device="cuda")
    for od in ("f32", "bf16"):
        out = torch.empty((B, H * D), dtype=torch.float32 if od == "f32" else torch.bfloat16,
                          device="cuda")
        qg.qg_decode_attention(dev(q), bf16_dev(kbits), bf16_dev(vbits), dev(kv_len), out, H, Hkv,
                               1.0 / math.sqrt(D), ws)
        got = host64(out)
        for b in range(B):
            L = int(kv_len[b])
            if 1 <= L <= cap:
                k64 = O.bf16_bits_to_f64(kbits[b, :, :L])
                v64 = O.bf16_bits_to_f64(vbits[b, :, :L])
                ref = O.decode_attention(q[b], k64, v64, L, H, Hkv, D)
                assert_parity(got[b], ref, bf16_out=(od == "bf16"), what=f"attn b={b} L={L}")
            else:
                assert np.all(got[b] == 0.0)


# ---------------------------------------------------------- argmax -------

@pytest.mark.parametrize("B,V", [(1, 1), (3, 7), (1, 151936), (4, 2048), (32, 151936), (2, 5000)])
def test_argmax_first_strict_max_bit_exact(B, V):
    """Index of the first strict maximum per row, NaNs skipped, 0 when no
    value beats -inf: equal to the oracle's fold on every row, including
    rows with repeated maxima (ties across chunks), NaNs, -0/+0 ties, +inf,
    and rows of only -inf or only NaN."""
    rng = np.random.default_rng(7 * B + V)
    x = rng.standard_normal((B, V)).astype(np.float32)
    for b in range(B):
        kind = b % 6
        if kind == 1 and V > 3:      # the maximum repeated, last copy in another chunk
            m = x[b].max() + 1.0
            x[b, [V // 3, V - 1, 2 * V // 3]] = m
        elif kind == 2:              # NaNs everywhere but a few values
            x[b, ::2] = np.nan
        elif kind == 3:              # -0 and +0 as the maximum
            x[b] = -1.0
            x[b, V // 2:] = 0.0
            x[b, V // 4] = -0.0
        elif kind == 4:              # nothing beats -inf
            x[b] = -np.inf if b % 12 == 4 else np.nan
        elif kind == 5 and V > 1:    # +inf after a larger finite run
            x[b, V - 1] = np.inf
    out = torch.empty(B, dtype=torch.int32, device="cuda")
    ws = torch.empty(qg.qg_argmax_workspace_size(B, V), dtype=torch.uint8, device="cuda")
    qg.qg_argmax_f32(dev(x), out, ws)
    got = out.cpu().numpy()
    want = np.array([O.argmax_first(x[b]) for b in range(B)], dtype=np.int32)
    np.testing.assert_array_equal(got, want)


# ---------------------------------------------------------- sampling -----

def _allowed_draws(logits, past, penalty, temperature, top_k, r, slack=1e-6):
    """The indices the oracle's draw can give when its running sums move by
    `slack` (the fp32 exp of two libraries may differ in the last bit)."""
    s = O.apply_repetition_penalty(logits, past, penalty)
    t = s / np.float32(temperature)
    order = [i for i in np.argsort(-t, kind="stable") if not np.isnan(t[i])][:min(top_k, len(t))]
    e = np.exp((t[order] - t[order[0]]).astype(np.float32))
    cum = np.cumsum(e / e.sum(dtype=np.float32), dtype=np.float32)
    ok = {order[j] for j in range(len(order))
          if cum[j] >= r - slack and (j == 0 or cum[j - 1] < r + slack)}
    if cum[-1] < r + slack:
        ok.add(order[0])
    return ok


@pytest.mark.parametrize("B,V,top_k,temperature", [(3, 2048, 50, 0.8), (2, 151936, 64, 1.0),
                                                   (4, 2048, 1, 0.7), (2, 5000, 8, 1.3),
                                                   (3, 2048, 0, 1.0), (2, 151936, 20, 0.0)])
def test_sample_matches_the_oracle(B, V, top_k, temperature):
    """Repetition penalty over past tokens (duplicates, -1 and out-of-range
    entries), then greedy (top_k 0 or temperature 0: bit-exact against the
    oracle) or a top-k draw with given uniform numbers (the oracle's index,
    up to the last-bit freedom of fp32 exp at a running-sum boundary)."""
    rng = np.random.default_rng(100 * B + top_k)
    logits = (3.0 * rng.standard_normal((B, V))).astype(np.float32)
    P = 40
    past = rng.integers(0, min(V, 300), size=(B, P)).astype(np.int32)
    past[:, 5] = past[:, 4]          # a repeated token
    past[:, -3:] = [-1, V, V + 7]    # empty slot and out-of-range entries
    logits[:, past[0, 0]] = -2.5     # a negative score that is penalized
    r = rng.random(B).astype(np.float32)
    out = torch.empty(B, dtype=torch.int32, device="cuda")
    ws = torch.empty(qg.qg_sample_workspace_size(B, V, top_k), dtype=torch.uint8, device="cuda")
    qg.qg_sample(dev(logits), out, ws, past=dev(past), penalty=1.2, temperature=temperature,
                 top_k=top_k, r=dev(r))
    got = out.cpu().numpy()
    for b in range(B):
        want = O.sample_token(logits[b], past[b], 1.2, temperature, top_k, r[b])
        if top_k == 0 or temperature == 0.0:
            assert got[b] == want
        else:
            assert got[b] == want or got[b] in _allowed_draws(
                logits[b], past[b], 1.2, temperature, top_k, r[b]), (b, got[b], want)


@pytest.mark.parametrize("B,V", [(3, 2048), (2, 151936), (1, 7)])
def test_token_logprob_matches_the_oracle(B, V):
    """Log-softmax at the selected token (the greedy one, another, an
    out-of-range one -> NaN) against the float64 oracle."""
    rng = np.random.default_rng(V + B)
    x = (4.0 * rng.standard_normal((B, V))).astype(np.float32)
    toks = np.array([int(np.argmax(x[b])) if b % 3 == 0 else (b * 37) % V for b in range(B)],
                    dtype=np.int32)
    if B > 2:
        toks[2] = V
    out = torch.empty(B, dtype=torch.float32, device="cuda")
    ws = torch.empty(qg.lib.qg_token_logprob_workspace_size(B, V), dtype=torch.uint8,
                     device="cuda")
    qg.qg_token_logprob(dev(x), dev(toks), out, ws)
    got = out.cpu().numpy().astype(np.float64)
    for b in range(B):
        ref = O.token_logprob(x[b].astype(np.float64), int(toks[b]))
        if math.isnan(ref):
            assert math.isnan(got[b])
        else:
            assert abs(got[b] - ref) <= 2e-3 + 1e-3 * abs(ref), (b, got[b], ref)
