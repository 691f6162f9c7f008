"""GPU parity of the code predictor (qg_code_predict) against the oracle.

Each group's logits are compared with the oracle's logits for that group
computed from the GPU's previous code (teacher-forced on the code chain, so
one near-tie argmax does not send the two sides down different chains), and
each chosen code is the oracle's greedy code wherever the oracle's top two
logits are further apart than the logits' error.

Without decoder layers the logits meet the element-wise bound everywhere
(measured: about 1e-7 relative at the full shape), which pins the input
construction, input_proj, the final norm, the heads and the code chain.
Through the layers a bf16 rounding point can legitimately round to the
other neighbour where its value lies within fp32 noise of a midpoint, and
the flip carries into later layers and groups (the same cascade as in the
whole-depth decode-step test; seen here at 2 and 5 layers): there the
logits are held to a relative-RMS bound of 1e-2. The layers themselves, at
the predictor's shapes, are checked per rounding point by the teacher-forced
decode-step test below.
"""
import numpy as np
import pytest
import torch

import qg_synth
from oracle import qg_oracle as O
from tests.gpu_util import ATOL, assert_parity, dev, host64

pytestmark = pytest.mark.gpu

qg = pytest.importorskip("weight_only_quantized_03_b200")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


SMALL_CP = dict(hidden=512, layers=2, heads=8, kv_heads=8, head_dim=64, ffn=1024, vocab=512,
                eps=1e-6, theta=1e6)


def _check(cfg, w, lm_hidden, code0, codes, logits, elementwise):
    B = lm_hidden.shape[0]
    G = len(w["heads"])
    np.testing.assert_array_equal(codes[0], code0)
    for b in range(B):
        for g in range(1, G):
            ref = O.code_predict_group(cfg, w, lm_hidden[b], int(codes[g - 1][b]), g)
            got = logits[g][b]
            err = np.abs(got - ref)
            if elementwise:
                assert_parity(got, ref, what=f"b={b} group {g} logits")
            rel_rms = np.sqrt(np.mean(err ** 2)) / np.sqrt(np.mean(ref ** 2))
            assert rel_rms <= 1e-2, f"b={b} group {g}: relative RMS error {rel_rms:.3e}"
            top = np.sort(ref)[-2:]
            if top[1] - top[0] > 2 * err.max() + ATOL:
                want = O.argmax_first(ref)
                assert int(codes[g][b]) == want, f"b={b} group {g}: code {codes[g][b]} != {want}"


@pytest.mark.parametrize("shape,B,G,layers", [("full", 1, 16, 0), ("full", 2, 4, 0),
                                               ("small", 1, 5, None), ("small", 3, 4, None),
                                               ("full", 1, 16, None)])
def test_code_predict_matches_oracle(shape, B, G, layers):
    """The makima code predictor shape ("full": hidden 1024, 5 layers, 16
    heads without GQA, head_dim 64, FFN 3072, 16 groups of 2048 codes), also
    without layers (element-wise), and a small one (2 layers) at batch 1 and
    3."""
    cfg = dict(qg_synth.CODE_PREDICTOR) if shape == "full" else dict(SMALL_CP)
    if layers is not None:
        cfg["layers"] = layers
    w = qg_synth.code_predictor_weights(cfg, G, 41, norm_jitter=0.1)
    model = qg.CodePredictor(cfg, w)
    lm_hidden = qg_synth.gaussian((B, cfg["hidden"]), 1.0, 42).astype(np.float32)
    code0 = qg_synth.tokens(B, cfg["vocab"], 43).astype(np.int32)
    codes = torch.empty((G, B), dtype=torch.int32, device="cuda")
    logits = torch.zeros((G, B, cfg["vocab"]), dtype=torch.float32, device="cuda")
    ws = model.workspace(B)
    model.qg_code_predict(dev(lm_hidden), dev(code0), codes, ws, logits=logits)
    torch.cuda.synchronize()
    got_codes = codes.cpu().numpy()
    assert np.all((got_codes >= 0) & (got_codes < cfg["vocab"]))
    _check(cfg, w, lm_hidden.astype(np.float64), code0, got_codes, host64(logits),
           elementwise=cfg["layers"] == 0)


def test_code_predict_graph_replay_and_bad_code():
    """On a non-default stream the call is recorded once and replayed:
    bit-identical codes and logits to the eager launches; a new code0 gives
    the new chain. A group-0 code outside the codebook gives NaN logits for
    group 1 (the embedding half of its input is NaN)."""
    cfg = dict(SMALL_CP)
    G, B = 4, 2
    w = qg_synth.code_predictor_weights(cfg, G, 44)
    model = qg.CodePredictor(cfg, w)
    lm = dev(qg_synth.gaussian((B, cfg["hidden"]), 1.0, 45).astype(np.float32))
    code0 = dev(np.array([3, 400], np.int32))
    ws = model.workspace(B)
    s = torch.cuda.Stream()
    res = {}
    for mode in ("graph", "eager"):
        qg.lib.qg_step_graphs_enable(1 if mode == "graph" else 0)
        qg.lib.qg_step_graphs_clear()
        outs = []
        for c0 in ([3, 400], [9, 1]):
            codes = torch.empty((G, B), dtype=torch.int32, device="cuda")
            logits = torch.empty((G, B, cfg["vocab"]), dtype=torch.float32, device="cuda")
            with torch.cuda.stream(s):
                code0.copy_(torch.tensor(c0, dtype=torch.int32))
                model.qg_code_predict(lm, code0, codes, ws, logits=logits, stream=s)
            s.synchronize()
            outs.append((codes.clone(), logits[1:].clone()))
        res[mode] = outs
    qg.lib.qg_step_graphs_enable(1)
    qg.lib.qg_step_graphs_clear()
    for (cg, lg), (ce, le) in zip(res["graph"], res["eager"]):
        assert torch.equal(cg, ce) and torch.equal(lg, le)
    assert not torch.equal(res["graph"][0][1], res["graph"][1][1])
    codes = torch.empty((G, B), dtype=torch.int32, device="cuda")
    logits = torch.empty((G, B, cfg["vocab"]), dtype=torch.float32, device="cuda")
    model.qg_code_predict(lm, dev(np.array([5, cfg["vocab"]], np.int32)), codes, ws, logits=logits)
    lg = logits.cpu().numpy()
    assert np.isfinite(lg[1, 0]).all() and np.isnan(lg[1, 1]).all()


def test_code_predictor_layers_teacher_forced():
    """The decoder layers at the code predictor's shapes (MHA 16/16,
    head_dim 64, FFN 3072, hidden 1024), run as decode steps at positions 0
    (the predictor's fresh cache) and 6, checked per layer and per bf16
    rounding point by the decode-step tests' teacher forcing."""
    from tests.test_gpu_decode_step import _step_checked
    cfg = dict(qg_synth.CODE_PREDICTOR)
    cfg["layers"] = 2
    w = qg_synth.qwen3_weights(cfg, 46, norm_jitter=0.1)
    model = qg.Qwen3Model(cfg, w)
    cap = 8
    st = model.new_state(2, cap)
    caches = [O.new_kv_cache(cfg, cap) for _ in range(2)]
    toks = [11, 1500]
    for p in range(7):
        logits = _step_checked(model, st, cfg, w, caches, toks, p)
        toks = [int(np.argmax(logits[b])) for b in range(2)]



def _slot(trace, B, cfg, offs, base, kv_bytes):
    """The values of one trace slot as float64 numpy arrays: the residual
    ``x``, the layer's values under the oracle's point names, and the K/V
    rows it wrote."""
    (o_xn, o_att, o_xn2, o_h), (o_q, o_k, o_v, o_xa, o_g, o_u) = offs
    HD, KD = cfg["heads"] * cfg["head_dim"], cfg["kv_heads"] * cfg["head_dim"]
    hid, F = cfg["hidden"], cfg["ffn"]

    def get(o, n, dt):
        size = 2 if dt == torch.bfloat16 else 4
        t = trace[base + o: base + o + size * B * n].view(dt).view(B, n)
        return host64(t)
    bf, f32 = torch.bfloat16, torch.float32
    v = {"x": get(0, hid, f32), "xn": get(o_xn, hid, bf), "att": get(o_att, HD, bf),
         "xn2": get(o_xn2, hid, bf), "h": get(o_h, F, bf), "q_proj": get(o_q, HD, f32),
         "k_proj": get(o_k, KD, f32), "v_proj": get(o_v, KD, f32), "x_attn": get(o_xa, hid, f32),
         "gate": get(o_g, F, f32), "up": get(o_u, F, f32)}
    snap = kv_bytes[0]
    v["k"] = get(snap, KD, bf)
    v["v"] = get(snap + kv_bytes[1], KD, bf)
    return v


@pytest.mark.parametrize("B,G", [(1, 16), (2, 3)])
def test_code_predict_layers_checked_op_by_op_per_group(B, G):
    """qg_code_predict's own layer chain at the makima code predictor shape
    (hidden 1024, 5 layers, MHA 16/16, head_dim 64, FFN 3072, 2048 codes),
    traced group by group (qg_code_predict_traced): every group's bf16
    input is the concatenation of the LM hidden state and the previous
    code's embedding (bit-exact), input_proj meets the fp32 bound, every
    layer is checked op by op against the oracle (each fp32 GEMV output
    from the GPU's inputs, each bf16 rounding point a correct rounding
    within its derived float32 bound, with a fresh one-row cache at
    position 0), the head's logits meet the bound from the GPU's final
    residual (plus the exact effect of final-norm ties), and each code is
    the first maximum of the GPU's own logits. The traced results equal
    the untraced call's bit for bit."""
    from tests.test_gpu_decode_step import _forced_layer
    cfg = dict(qg_synth.CODE_PREDICTOR)
    w = qg_synth.code_predictor_weights(cfg, G, 47, norm_jitter=0.1)
    model = qg.CodePredictor(cfg, w)
    lm_hidden = qg_synth.gaussian((B, cfg["hidden"]), 1.0, 48).astype(np.float32)
    code0 = qg_synth.tokens(B, cfg["vocab"], 49).astype(np.int32)
    total, per_group, slot0, per_slot = model.trace_layout(B)
    trace = torch.zeros(total, dtype=torch.uint8, device="cuda")
    codes = torch.empty((G, B), dtype=torch.int32, device="cuda")
    logits = torch.zeros((G, B, cfg["vocab"]), dtype=torch.float32, device="cuda")
    ws = model.workspace(B)
    model.qg_code_predict_traced(dev(lm_hidden), dev(code0), codes, ws, trace, logits=logits)
    codes2 = torch.empty_like(codes)
    logits2 = torch.zeros_like(logits)
    model.qg_code_predict(dev(lm_hidden), dev(code0), codes2, ws, logits=logits2)
    torch.cuda.synchronize()
    assert torch.equal(codes, codes2) and torch.equal(logits[1:], logits2[1:])
    got_codes = codes.cpu().numpy()
    lg = host64(logits)
    offs = model.step_offsets(B)
    Hkv, D = cfg["kv_heads"], cfg["head_dim"]
    kv_row = B * Hkv * D * 2
    kv_bytes = ((per_slot - 2 * ((kv_row + 255) // 256 * 256)), (kv_row + 255) // 256 * 256)
    np.testing.assert_array_equal(got_codes[0], code0)
    for g in range(1, G):
        gb = (g - 1) * per_group
        comb = host64(trace[gb: gb + B * 2 * cfg["hidden"] * 2].view(torch.bfloat16)
                      .view(B, 2 * cfg["hidden"]))
        slots = [_slot(trace, B, cfg, offs, gb + slot0 + s * per_slot, kv_bytes)
                 for s in range(cfg["layers"] + 1)]
        for b in range(B):
            what = f"b={b} group {g}"
            emb = O.embed_rows(*w["code_embed"][g - 1], [int(got_codes[g - 1][b])])[0]
            ref_comb = O.round_bf16(np.concatenate([lm_hidden[b].astype(np.float64), emb]))
            np.testing.assert_array_equal(comb[b], ref_comb, err_msg=f"{what} input")
            x0 = O.gemv_affine8(*w["input_proj"], comb[b][None])[0]
            assert_parity(slots[0]["x"][b], x0, what=f"{what} input_proj")
            for l in range(cfg["layers"]):
                s_in, s_out = slots[l], slots[l + 1]
                inter = {k: s_out[k][b] for k in ("xn", "xn2", "h", "q_proj", "k_proj", "v_proj",
                                                 "x_attn", "gate", "up")}
                inter["attn"] = s_out["att"][b]
                kc, vc = np.zeros((Hkv, 1, D)), np.zeros((Hkv, 1, D))
                _forced_layer(cfg, w["layers"][l], s_in["x"][b], kc, vc, 0, inter,
                              s_out["k"][b], s_out["v"][b], s_out["x"][b], f"{what} layer {l}")
            head = {"embed": w["heads"][g], "final_norm": w["final_norm"]}
            ref, tie = O.lm_head_tie_bound(cfg, head, slots[-1]["x"][b])
            assert_parity(lg[g][b], ref, extra=tie, what=f"{what} head")
            assert int(got_codes[g][b]) == O.argmax_first(lg[g][b]), what
