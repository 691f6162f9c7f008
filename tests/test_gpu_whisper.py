"""GPU parity of the Whisper encoder layer row (fuel-transformers 0.19.1,
src/models/lazy_quantized_whisper.rs, encoder_layer): LayerNorm, the Q4_0
tensor-core matmul's epilogues (bf16 A in, bias, residual, gelu_tanh, bf16
out), multi-row softmax attention, and the whole layer at the
Whisper-large-v3 shape (M = 1500 frames, d_model 1280, 20 heads of 64, FFN
5120), checked stage by stage: each stage of the oracle runs from the GPU's
own inputs of that stage.

Tolerances: fp32-accumulated outputs |gpu - ref| <= 2e-3 + 1e-3 |ref|; bf16
outputs add half a bf16 ulp. The attention rounds its softmax weights to
bf16 for the weighted sum of V (and sums the rounded weights): a relative
change of at most 2^-8 (bf16's unit roundoff) per weight, which moves an
output by at most e^(2^-7) 2^-8 sum_s p_s |v_s - o| <= 1.02 * 2^-8
(sum_s p_s |v_s| + |o|), added to the bound (``extra``). A GELU output adds the fp32 bound times the largest
slope of gelu_tanh minus one (0.13).
"""
import numpy as np
import pytest
import torch

import qg_synth
from oracle import qg_oracle as O
from tests.gpu_util import assert_parity, dev, host64

pytestmark = pytest.mark.gpu

qg = pytest.importorskip("weight_only_quantized_03_b200")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


P_ROUND_BOUND = 1.02 * 2.0 ** -8


def _bf16(a):
    return dev(qg_synth.f32_to_bf16_bits(np.asarray(a, np.float32))).view(torch.bfloat16)


@pytest.mark.parametrize("rows,dim", [(1500, 1280), (37, 768), (5, 2048)])
def test_layernorm(rows, dim):
    x = qg_synth.gaussian((rows, dim), 2.0, 1) + 0.5
    g = qg_synth.gaussian((dim,), 0.1, 2) + 1.0
    b = qg_synth.gaussian((dim,), 0.1, 3)
    ref = O.layer_norm(x, g, b, 1e-5)
    for dt in (torch.float32, torch.bfloat16):
        y = torch.empty((rows, dim), dtype=dt, device="cuda")
        qg.qg_layernorm(dev(x), dev(g), dev(b), 1e-5, y)
        torch.cuda.synchronize()
        assert_parity(host64(y), ref, bf16_out=dt == torch.bfloat16, what=f"LN {dt}")


ATT_CASES = [
    # B, T, S, H, Hkv, D, causal
    (1, 1500, 1500, 20, 20, 64, False),   # Whisper-large-v3 encoder self-attention
    (2, 256, 256, 16, 8, 128, True),      # a 256-row prompt, GQA
    (1, 77, 77, 3, 3, 64, False),         # ragged tiles
    (2, 50, 130, 4, 2, 128, True),        # 50 rows after an 80-row prefix
    (1, 9, 0, 2, 2, 64, False),           # no keys: zero rows
]


@pytest.mark.parametrize("B,T,S,H,Hkv,D,causal", ATT_CASES)
def test_attention_rows(B, T, S, H, Hkv, D, causal):
    qb = qg_synth.gaussian_bf16_bits((B, T, H * D), 1.0, 10)
    kb = qg_synth.gaussian_bf16_bits((B, S, Hkv * D), 1.0, 11)
    vb = qg_synth.gaussian_bf16_bits((B, S, Hkv * D), 1.0, 12)
    out = torch.full((B, T, H * D), float("nan"), dtype=torch.bfloat16, device="cuda")
    qg.qg_attention_rows(dev(qb).view(torch.bfloat16), dev(kb).view(torch.bfloat16),
                         dev(vb).view(torch.bfloat16), out, H, Hkv, causal=causal)
    torch.cuda.synchronize()
    got = host64(out)
    for b in range(B):
        q, k, v = (O.bf16_bits_to_f64(a[b]) for a in (qb, kb, vb))
        if S == 0:
            np.testing.assert_array_equal(got[b], 0.0)
            continue
        ref, aw = O.mha_rows(q, k, v, H, causal=causal, kv_heads=Hkv, abs_weighted=True)
        assert_parity(got[b], ref, bf16_out=True, extra=P_ROUND_BOUND * (aw + np.abs(ref)),
                      what=f"attention b={b}")


@pytest.mark.parametrize("M,N,K", [(300, 256, 128), (1500, 1280, 1280), (1500, 5120, 1280)])
def test_gemm_q4_0_epilogues(M, N, K):
    """bf16 A in; bias; bias + residual into fp32; bias + gelu_tanh into
    bf16; against the oracle's bf16-operand matmul."""
    blocks = qg_synth.q4_0_packed(N, K, 30)
    A = O.round_bf16(qg_synth.gaussian((M, K), 1.0, 31))
    bias = qg_synth.gaussian((N,), 0.1, 32)
    res = qg_synth.gaussian((M, N), 1.0, 33)
    ref = O.gemm_q4_0_bf16(blocks, A, bias)
    Ad, bd = _bf16(A), dev(bias)
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    c16 = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    qg.qg_gemm_q4_0_ex(dev(blocks), Ad, c16, bias=bd, ws=ws)
    c32 = dev(res)
    qg.qg_gemm_q4_0_ex(dev(blocks), Ad, c32, bias=bd, residual=c32, ws=ws)
    cg = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    qg.qg_gemm_q4_0_ex(dev(blocks), Ad, cg, bias=bd, gelu=True, ws=ws)
    torch.cuda.synchronize()
    assert qg.qg_gemm_q4_0_error(0, 0, ws)[1] == 0
    assert_parity(host64(c16), ref, bf16_out=True, what="bf16 out")
    assert_parity(host64(c32), ref + res, what="residual")
    tol = 0.13 * (2e-3 + 1e-3 * np.abs(ref))
    assert_parity(host64(cg), O.gelu_tanh(ref), bf16_out=True, extra=tol, what="gelu")


SMALL_W = dict(d_model=256, heads=4, ffn=512, eps=1e-5)


@pytest.mark.parametrize("shape,M", [("large_v3", 1500), ("small", 200), ("small", 1)])
def test_whisper_encoder_layer_stagewise(shape, M):
    cfg = dict(qg_synth.WHISPER_LARGE_V3) if shape == "large_v3" else dict(SMALL_W)
    w = qg_synth.whisper_layer_weights(cfg, 500)
    layer = qg.WhisperEncoderLayer(cfg, w)
    x = qg_synth.gaussian((M, cfg["d_model"]), 1.0, 501)
    xd = dev(x)
    ws = layer.workspace(M)
    layer.qg_whisper_encoder_layer(xd, ws)
    torch.cuda.synchronize()
    it = {k: v.clone() for k, v in layer.intermediates(ws, M).items()}
    assert torch.count_nonzero(it.pop("err")) == 0
    g = {k: host64(v) for k, v in it.items()}
    y = host64(xd)
    H, eps = cfg["heads"], cfg["eps"]
    assert_parity(g["xl"], O.layer_norm(x, w["ln1_g"], w["ln1_b"], eps), bf16_out=True, what="LN1")
    for name, bias in (("q", w["q_b"]), ("k", None), ("v", w["v_b"])):
        assert_parity(g[name], O.gemm_q4_0_bf16(w[name], g["xl"], bias), bf16_out=True, what=name)
    ref, aw = O.mha_rows(g["q"], g["k"], g["v"], H, abs_weighted=True)
    assert_parity(g["ctx"], ref, bf16_out=True, extra=P_ROUND_BOUND * (aw + np.abs(ref)),
                  what="attention")
    assert_parity(g["xa"], x + O.gemm_q4_0_bf16(w["o"], g["ctx"], w["o_b"]), what="out + residual")
    assert_parity(g["xl2"], O.layer_norm(g["xa"], w["ln2_g"], w["ln2_b"], eps), bf16_out=True,
                  what="LN2")
    pre = O.gemm_q4_0_bf16(w["fc1"], g["xl2"], w["fc1_b"])
    assert_parity(g["mid"], O.gelu_tanh(pre), bf16_out=True,
                  extra=0.13 * (2e-3 + 1e-3 * np.abs(pre)), what="fc1 + gelu")
    assert_parity(y, g["xa"] + O.gemm_q4_0_bf16(w["fc2"], g["mid"], w["fc2_b"]),
                  what="fc2 + residual")
    # and the whole layer against the oracle's, as a cascade check
    ref_y = O.whisper_encoder_layer(x, w, H, eps)
    rel = np.sqrt(np.mean((y - ref_y) ** 2) / np.mean(ref_y ** 2))
    assert rel < 1e-2, rel


def test_gemm_timeout_path_reports_and_the_context_stays_usable():
    """The matmul's bounded waits: with every load withheld
    (qg_gemm_q4_0_stall_test), the MMA issuer's first wait runs out after
    about 1 ms with nothing in flight; the call's error word reads nonzero
    (QG_ERR_TIMEOUT), C is untouched, and a normal call right after is
    correct."""
    M, N, K = 256, 256, 128
    blocks = qg_synth.q4_0_packed(N, K, 40)
    A = O.round_bf16(qg_synth.gaussian((M, K), 1.0, 41))
    Ad = _bf16(A)
    C = torch.zeros((M, N), dtype=torch.float32, device="cuda")
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    st = qg.lib.qg_gemm_q4_0_stall_test(qg._p(dev(blocks)), qg._p(Ad), qg._p(C), M, N, K,
                                        qg._p(ws), 256, qg._stream(None))
    assert st == qg.QG_OK
    status, code = qg.qg_gemm_q4_0_error(0, 0, ws)
    assert status == qg.QG_ERR_TIMEOUT and code != 0
    assert torch.count_nonzero(C) == 0
    qg.qg_gemm_q4_0_ex(dev(blocks), Ad, C, ws=ws)
    torch.cuda.synchronize()
    assert qg.qg_gemm_q4_0_error(0, 0, ws)[1] == 0
    assert_parity(host64(C), O.gemm_q4_0_bf16(blocks, A), what="after the timeout")
