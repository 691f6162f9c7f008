"""GPU parity of the batched prefill row (qg_prefill) and its tensor-core
affine8 matmul (qg_gemm_affine8_g64).

The matmul is compared element by element with the oracle's exact GEMV
(|gpu - ref| <= 2e-3 + 1e-3 |ref|) at prompt, batch and ragged shapes.

The prefill is checked layer by layer and row by row, teacher-forced: the
GPU's run cut to l layers gives the residual rows entering layer l; the run
with l + 1 layers gives that layer's values for every row (the inspection
buffers) and its K/V rows in the cache. Row t of the prompt is a decode step
at position p0 + t over the cache rows before it (the rows the GPU wrote),
so each row goes through the oracle's op-by-op layer check
(``decode_layer_forced``): every fp32 GEMV output against the oracle's from
the GPU's inputs, every bf16 rounding point within its derived float32
bound, widened for the two roundings the multi-row attention adds (the
roped query and the softmax weights are rounded to bf16 for the tensor-core
products: 2^-8 relative each). The last row's logits are checked from the
GPU's final residual.
"""
import numpy as np
import pytest
import torch

import qg_synth
from oracle import qg_oracle as O
from tests.gpu_util import assert_parity, dev, host64
from tests.test_gpu_decode_step import _prefill

pytestmark = pytest.mark.gpu

qg = pytest.importorskip("weight_only_quantized_03_b200")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


@pytest.mark.parametrize("T,N,K,res,bf16", [(256, 2048, 2048, False, False),
                                            (256, 1024, 6144, True, False),
                                            (5, 300, 128, True, False),
                                            (17, 384, 1024, False, True),
                                            (1, 1024, 3072, False, False),
                                            (32, 3072, 1024, True, False),
                                            (16, 1000, 2048, True, False),
                                            (1, 300, 64, False, True)])
def test_gemm_affine8(T, N, K, res, bf16):
    w, s, b = qg_synth.affine8_packed(N, K, 60)
    xb = qg_synth.gaussian_bf16_bits((T, K), 1.0, 61)
    r = qg_synth.gaussian((T, N), 1.0, 62) if res else None
    ref = O.gemv_affine8(w, s, b, O.bf16_bits_to_f64(xb), None if r is None else r)
    y = (dev(r) if res else
         torch.full((T, N), float("nan"), dtype=torch.bfloat16 if bf16 else torch.float32,
                    device="cuda"))
    ws = torch.zeros(1, dtype=torch.int32, device="cuda")
    qg.qg_gemm_affine8_g64(dev(w), dev(s), dev(b), dev(xb).view(torch.bfloat16), y,
                           residual=y if res else None, ws=ws)
    torch.cuda.synchronize()
    assert int(ws.item()) == 0
    assert_parity(host64(y), ref, bf16_out=bf16, what=f"T={T} N={N} K={K}")


SMALL = dict(hidden=512, layers=3, heads=4, kv_heads=2, head_dim=128, ffn=1024, vocab=1000,
             eps=1e-6, theta=1e6)

FP32 = ("q_proj", "k_proj", "v_proj", "x_attn", "gate", "up")


def _check_prefill(cfg, w, T, p0, cap, rows=None, seed=80):
    model = qg.Qwen3Model(cfg, w)
    st = model.new_state(1, cap)
    Lr, Hkv, D = cfg["layers"], cfg["kv_heads"], cfg["head_dim"]
    kbits = _prefill((Lr, 1, Hkv, cap, D), seed)
    vbits = _prefill((Lr, 1, Hkv, cap, D), seed + 1)
    toks = dev(qg_synth.tokens(T, cfg["vocab"], seed + 2))
    ws = model.prefill_workspace(T)
    logits = torch.empty(cfg["vocab"], dtype=torch.float32, device="cuda")
    xs, inter = [], []
    for l in range(Lr + 1):
        st["k_cache"].copy_(dev(kbits).view(torch.bfloat16))
        st["v_cache"].copy_(dev(vbits).view(torch.bfloat16))
        model.qg_prefill(st, toks, p0, ws, logits=logits, layers=l)
        it = model.prefill_intermediates(ws, T)
        xs.append(host64(it["x"]))
        if l >= 1:
            inter.append({k: host64(v) for k, v in it.items() if k != "x"})
    torch.cuda.synchronize()
    kg, vg = host64(st["k_cache"])[:, 0], host64(st["v_cache"])[:, 0]
    ew, es, eb = w["embed"]
    np.testing.assert_array_equal(xs[0], O.embed_rows(ew, es, eb, host64(toks).astype(int)))
    for l in range(Lr):
        for t in (range(T) if rows is None else rows):
            pos = p0 + t
            what = f"layer {l} row {t} (position {pos})"
            it = inter[l]
            forced = {k: it[k][t] for k in FP32}
            forced.update(xn=it["xn"][t], xn2=it["xn2"][t], h=it["h"][t], att=it["att"][t],
                          k=kg[l, :, pos, :].ravel(), v=vg[l, :, pos, :].ravel())
            det = {}
            refs, bad = O.decode_layer_forced(cfg, w["layers"][l], xs[l][t], kg[l].copy(),
                                              vg[l].copy(), pos, forced, details=det,
                                              q_round=2.0 ** -8, p_round=2.0 ** -8)
            for name, idx in bad.items():
                assert idx.size == 0, f"{what}: {name} is not a correct bf16 rounding: {det.get(name)}"
            for name in FP32:
                assert_parity(forced[name], refs[name], what=f"{what} {name}")
            assert_parity(xs[l + 1][t], refs["y"], what=f"{what} residual")
        # cache rows outside the prompt are untouched
        keep = np.ones(cap, bool)
        keep[p0:p0 + T] = False
        np.testing.assert_array_equal(kg[l][:, keep], O.bf16_bits_to_f64(kbits[l, 0])[:, keep])
    ref, tie = O.lm_head_tie_bound(cfg, w, xs[Lr][T - 1])
    assert_parity(host64(logits), ref, extra=tie, what="last row LM head")


@pytest.mark.parametrize("T,p0", [(40, 0), (33, 7)])
def test_prefill_small_decoder_every_row(T, p0):
    cfg = dict(SMALL)
    w = qg_synth.qwen3_weights(cfg, 21, norm_jitter=0.1)
    _check_prefill(cfg, w, T, p0, cap=48)


def test_prefill_qwen3_1_7b_shape_256_rows():
    """The 1.7B layer shapes (hidden 2048, FFN 6144, 16/8 heads of 128), the
    256-row prompt at positions 0..255, two layers; the rows checked span
    the attention's 64-row tiles and the matmul's token tiles."""
    cfg = dict(qg_synth.QWEN3_1_7B, layers=2)
    w = qg_synth.qwen3_weights(cfg, 17)
    _check_prefill(cfg, w, 256, 0, cap=2049, rows=[0, 1, 63, 64, 130, 255])


def test_prefill_bad_token_writes_no_cache_row():
    cfg = dict(SMALL, layers=1)
    w = qg_synth.qwen3_weights(cfg, 22)
    model = qg.Qwen3Model(cfg, w)
    st = model.new_state(1, 16)
    toks = dev(np.array([3, cfg["vocab"], 5], np.int32))
    ws = model.prefill_workspace(3)
    model.qg_prefill(st, toks, 2, ws)
    torch.cuda.synchronize()
    k = host64(st["k_cache"])[0, 0]
    assert np.all(k[:, 3] == 0) and np.any(k[:, 2] != 0) and np.any(k[:, 4] != 0)
    assert np.isnan(host64(model.prefill_intermediates(ws, 3)["x"])[1]).all()
