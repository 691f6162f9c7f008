"""GPU parity of the whole decode step (qg_decode_step) against the oracle.

1. The tiny synthetic decoder of the turbospark parity gate (hidden 64, 2
   layers, 2 heads / 1 KV head, head_dim 64, vocab 261, eps 1e-5, theta 1e4,
   LCG code bytes with constant scale/bias): 32 greedy steps with tokens and
   appended cache rows teacher-forced (each step starts both sides from the
   same state); logits within tolerance at every step and the same greedy
   token wherever the oracle's top two logits are not within tolerance.
2. A small decoder (hidden 512, 3 layers, 4/2 heads, head_dim 128, FFN
   1024, vocab 1000), B up to 4, 40 greedy steps.
3. The Qwen3-0.6B shape (28 layers, hidden 1024, 16/8 heads, head_dim 128,
   FFN 3072, vocab 151936, eps 1e-6, theta 1e6) with random packed weights,
   the KV cache prefilled with seeded N(0,1) bf16 rows, stepped at position
   511 (attends 512 rows): logits and the appended K/V rows.
4. Invalid tokens/positions give NaN logits and leave the cache untouched.
5. One step is 5 launches per layer plus the embedding and the LM head.

Why stage by stage: the bf16 stores (norm outputs, K/V rows, attention and
SiLU-mul outputs) make the two sides take different roundings wherever a
value sits within fp32 noise of a bf16 midpoint; such a one-ulp difference in
one layer is amplified by the layers after it, so whole-step logits can miss
the per-element bound although every stage meets it. Each stage is
therefore compared from identical inputs; the whole-depth comparison has its
own, looser bound (test_qwen3_0_6b_step_whole_depth_bf16_cascade_bound).
"""
import numpy as np
import pytest
import torch

import qg_synth
from oracle import qg_oracle as O
from tests.gpu_util import ATOL, RTOL, assert_parity, dev, host64

pytestmark = pytest.mark.gpu

qg = pytest.importorskip("weight_only_quantized_03_b200")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def _greedy_ok(gpu_logits, ref_logits):
    g = int(np.argmax(gpu_logits))
    r = O.argmax_first(ref_logits)
    if g == r:
        return True
    top = np.sort(ref_logits)[-2:]
    return abs(top[1] - top[0]) <= 2 * (ATOL + RTOL * abs(top[1]))


def _forced_layer(cfg, lw, x, kc_l, vc_l, p, inter_b, k_row, v_row, x_out, what):
    """One layer of the oracle checked op by op against the GPU's values of
    that layer (``decode_layer_forced``): each fp32 GEMV output of the GPU
    (q/k/v, the residual after o_proj, gate, up, and ``x_out``, the residual
    after the layer) against the oracle's from the GPU's own inputs, under
    the fp32-accumulation bound; each bf16 value at a rounding point as a
    correct rounding of the oracle's value of its op chain within that
    chain's derived float32 error bound."""
    forced = dict(inter_b, k=k_row.ravel(), v=v_row.ravel())
    forced["att"] = forced.pop("attn")  # the oracle's name for the attention output
    det = {}
    refs, bad = O.decode_layer_forced(cfg, lw, x, kc_l, vc_l, p, forced, details=det)
    for name, idx in bad.items():
        assert idx.size == 0, f"{what}: {name} is not a correct bf16 rounding: {det.get(name)}"
    for name in O.LAYER_FP32_POINTS:
        assert_parity(forced[name], refs[name], what=f"{what} {name}")
    assert_parity(x_out, refs["y"], what=f"{what} residual")


def _intermediates(model, st):
    return {k: host64(t) for k, t in model.intermediates(st).items()}


def _step_checked(model, st, cfg, w, caches, toks, p):
    """One decode step at position p for every sequence, checked stage by
    stage from identical inputs: the GPU prefix runs (the same step cut to l
    layers) give the residual stream entering each layer; the oracle runs
    that one layer from the GPU's input, teacher-forced at the layer's bf16
    rounding points with the GPU's own values (after checking each is a
    correct rounding). The LM head is checked from the GPU's final residual
    stream. Returns the GPU logits."""
    B = len(toks)
    t, pos = dev(np.array(toks, np.int32)), dev(np.full(B, p, np.int32))
    xs, inter = [], []
    for l in range(cfg["layers"] + 1):
        model.qg_decode_step(st, t, pos, layers=l)
        xs.append(host64(model.residual(st)))
        if l >= 1:
            inter.append(_intermediates(model, st))
    logits = host64(st["logits"])
    kg, vg = host64(st["k_cache"]), host64(st["v_cache"])
    ew, es, eb = w["embed"]
    np.testing.assert_array_equal(xs[0], O.embed_rows(ew, es, eb, toks))
    for b in range(B):
        kc, vc = caches[b]
        for l in range(cfg["layers"]):
            what = f"b={b} p={p} layer {l}"
            _forced_layer(cfg, w["layers"][l], xs[l][b], kc[l], vc[l], p,
                          {k: a[b] for k, a in inter[l].items()},
                          kg[l, b, :, p, :], vg[l, b, :, p, :], xs[l + 1][b], what)
            kc[l, :, p, :] = kg[l, b, :, p, :]
            vc[l, :, p, :] = vg[l, b, :, p, :]
        ref, tie = O.lm_head_tie_bound(cfg, w, xs[-1][b])
        assert_parity(logits[b], ref, extra=tie, what=f"b={b} p={p} LM head")
    return logits


@pytest.mark.parametrize("fixture", [True, False])
def test_tiny_decoder_stagewise_greedy(fixture):
    cfg = dict(qg_synth.QWEN3_TINY)
    w = qg_synth.qwen3_weights(cfg, 5, fixture=fixture, norm_jitter=0.0 if fixture else 0.1)
    model = qg.Qwen3Model(cfg, w)
    cap = 40
    st = model.new_state(1, cap)
    caches = [O.new_kv_cache(cfg, cap)]
    tok = 259
    for p in range(32):
        logits = _step_checked(model, st, cfg, w, caches, [tok], p)
        tok = int(np.argmax(logits[0]))


def _prefill(shape, seed):
    return qg_synth.gaussian_bf16_bits(shape, 1.0, seed)


SMALL = dict(hidden=512, layers=3, heads=4, kv_heads=2, head_dim=128, ffn=1024, vocab=1000,
             eps=1e-6, theta=1e6)


@pytest.mark.parametrize("B", [1, 3, 4])
def test_small_decoder_stagewise_greedy(B):
    """A decoder small enough for a 40-step oracle run. Positions 0..39
    cross the 32-row attention chunks; B sequences start from different
    tokens and follow the GPU's greedy tokens; every step is checked stage
    by stage (_step_checked)."""
    cfg = dict(SMALL)
    w = qg_synth.qwen3_weights(cfg, 21, norm_jitter=0.1)
    model = qg.Qwen3Model(cfg, w)
    cap = 48
    st = model.new_state(B, cap)
    caches = [O.new_kv_cache(cfg, cap) for _ in range(B)]
    toks = [7, 500, 999, 123][:B]
    for p in range(40):
        logits = _step_checked(model, st, cfg, w, caches, toks, p)
        toks = [int(np.argmax(logits[b])) for b in range(B)]


@pytest.mark.parametrize("B", [1, 2])
def test_qwen3_0_6b_step_layer_by_layer_at_position_511(B):
    """Teacher-forced per layer: layer l of the oracle starts from the GPU's
    residual stream after l-1 layers, so each comparison covers the bf16
    rounding points of one layer only. The GPU prefix runs are the same step
    with the layer count cut to l (the weights of the first l layers)."""
    cfg = dict(qg_synth.QWEN3_0_6B)
    w = qg_synth.qwen3_weights(cfg, 11)
    model = qg.Qwen3Model(cfg, w)
    cap = 520
    st = model.new_state(B, cap)
    Lr, Hkv, D = cfg["layers"], cfg["kv_heads"], cfg["head_dim"]
    kbits = _prefill((Lr, B, Hkv, cap, D), 70)
    vbits = _prefill((Lr, B, Hkv, cap, D), 71)
    st["k_cache"].copy_(dev(kbits).view(torch.bfloat16))
    st["v_cache"].copy_(dev(vbits).view(torch.bfloat16))
    toks = dev(qg_synth.tokens(B, cfg["vocab"], 72))
    pos_np = np.array([511, 300][:B], dtype=np.int32)
    pos = dev(pos_np)
    xs, inter = [], []
    for l in range(Lr + 1):
        model.qg_decode_step(st, toks, pos, layers=l)
        xs.append(host64(model.residual(st)))
        if l >= 1:
            inter.append(_intermediates(model, st))
    logits = host64(st["logits"])
    kg, vg = host64(st["k_cache"]), host64(st["v_cache"])
    ew, es, eb = w["embed"]
    np.testing.assert_array_equal(xs[0], O.embed_rows(ew, es, eb, host64(toks).astype(int)))
    for b in range(B):
        p = int(pos_np[b])
        kc = O.bf16_bits_to_f64(kbits[:, b])
        vc = O.bf16_bits_to_f64(vbits[:, b])
        for l in range(Lr):
            what = f"b={b} layer {l}"
            _forced_layer(cfg, w["layers"][l], xs[l][b], kc[l], vc[l], p,
                          {k: a[b] for k, a in inter[l].items()},
                          kg[l, b, :, p, :], vg[l, b, :, p, :], xs[l + 1][b], what)
            np.testing.assert_array_equal(kg[l, b, :, p + 1, :], kc[l, :, p + 1, :])
        ref, tie = O.lm_head_tie_bound(cfg, w, xs[Lr][b])
        assert_parity(logits[b], ref, extra=tie, what=f"b={b} LM head")


@pytest.mark.parametrize("B,layers", [(2, 3), (12, 2)])
def test_qwen3_1_7b_shaped_layers_at_position_2047(B, layers):
    """The 1.7B layer shapes (hidden 2048, FFN 6144, K/V cache of 2049 rows)
    with a few layers, teacher-forced per layer at positions up to 2047.
    B = 2 takes the cluster attention kernel; B = 12 (12 x 8 x 2049 cached
    rows) the tensor-core attention kernel with the step's fused q/k norm,
    RoPE and K/V append, and the tensor-core GEMV in batch tiles of 8."""
    cfg = dict(qg_synth.QWEN3_1_7B, layers=layers)
    w = qg_synth.qwen3_weights(cfg, 17)
    model = qg.Qwen3Model(cfg, w)
    cap = 2049
    st = model.new_state(B, cap)
    Lr, Hkv, D = cfg["layers"], cfg["kv_heads"], cfg["head_dim"]
    kbits = _prefill((Lr, B, Hkv, cap, D), 80)
    vbits = _prefill((Lr, B, Hkv, cap, D), 81)
    st["k_cache"].copy_(dev(kbits).view(torch.bfloat16))
    st["v_cache"].copy_(dev(vbits).view(torch.bfloat16))
    toks = dev(qg_synth.tokens(B, cfg["vocab"], 82))
    pos_np = np.array([2047, 1000, 5, 2048, 0, 777, 1500, 31, 32, 33, 1999, 64][:B], dtype=np.int32)
    pos = dev(pos_np)
    xs, inter = [], []
    for l in range(Lr + 1):
        model.qg_decode_step(st, toks, pos, layers=l)
        xs.append(host64(model.residual(st)))
        if l >= 1:
            inter.append(_intermediates(model, st))
    logits = host64(st["logits"])
    kg, vg = host64(st["k_cache"]), host64(st["v_cache"])
    for b in range(B):
        p = int(pos_np[b])
        kc = O.bf16_bits_to_f64(kbits[:, b])
        vc = O.bf16_bits_to_f64(vbits[:, b])
        for l in range(Lr):
            what = f"b={b} p={p} layer {l}"
            _forced_layer(cfg, w["layers"][l], xs[l][b], kc[l], vc[l], p,
                          {k: a[b] for k, a in inter[l].items()},
                          kg[l, b, :, p, :], vg[l, b, :, p, :], xs[l + 1][b], what)
        if b < 2:  # the LM head oracle (151936 x 2048 in f64) for two rows
            ref, tie = O.lm_head_tie_bound(cfg, w, xs[Lr][b])
            assert_parity(logits[b], ref, extra=tie, what=f"b={b} LM head")


def test_qwen3_0_6b_step_whole_depth_bf16_cascade_bound():
    """Untethered 28-layer step against the oracle. The bf16 stores make
    the two sides take different roundings where a value sits within fp32
    noise of a bf16 midpoint, and those one-ulp differences compound from
    layer to layer, so the per-element bound (2e-3 + 1e-3 |ref|) applies per layer
    (test above); across the whole depth the logits must agree to a relative
    RMS error of 2e-2 (a few bf16 ulps, 2^-8 = 3.9e-3 each)."""
    cfg = dict(qg_synth.QWEN3_0_6B)
    w = qg_synth.qwen3_weights(cfg, 11)
    model = qg.Qwen3Model(cfg, w)
    cap = 520
    st = model.new_state(1, cap)
    Lr, Hkv, D = cfg["layers"], cfg["kv_heads"], cfg["head_dim"]
    kbits = _prefill((Lr, 1, Hkv, cap, D), 70)
    vbits = _prefill((Lr, 1, Hkv, cap, D), 71)
    st["k_cache"].copy_(dev(kbits).view(torch.bfloat16))
    st["v_cache"].copy_(dev(vbits).view(torch.bfloat16))
    tok = int(qg_synth.tokens(1, cfg["vocab"], 72)[0])
    model.qg_decode_step(st, dev(np.array([tok], np.int32)), dev(np.array([511], np.int32)))
    got = host64(st["logits"])[0]
    ref = O.decode_step(cfg, w, O.bf16_bits_to_f64(kbits[:, 0]), O.bf16_bits_to_f64(vbits[:, 0]),
                        tok, 511)
    rel_rms = np.sqrt(np.mean((got - ref) ** 2) / np.mean(ref ** 2))
    assert rel_rms <= 2e-2, rel_rms


def test_invalid_token_or_position_gives_nan_and_leaves_cache():
    cfg = dict(qg_synth.QWEN3_TINY)
    w = qg_synth.qwen3_weights(cfg, 6, fixture=True)
    model = qg.Qwen3Model(cfg, w)
    cap = 8
    st = model.new_state(3, cap)
    model.qg_decode_step(st, dev(np.array([1, 2, 3], np.int32)), dev(np.array([0, 0, 0], np.int32)))
    before = st["k_cache"].clone()
    toks = np.array([5, 261, 7], np.int32)       # token 261 is out of range
    pos = np.array([1, 1, cap], np.int32)         # position cap is out of range
    model.qg_decode_step(st, dev(toks), dev(pos))
    lg = host64(st["logits"])
    assert np.isfinite(lg[0]).all()
    assert np.isnan(lg[1]).all() and np.isnan(lg[2]).all()
    after = st["k_cache"]
    assert torch.equal(after[:, 1], before[:, 1])
    assert torch.equal(after[:, 2], before[:, 2])
    assert not torch.equal(after[:, 0], before[:, 0])


@pytest.mark.parametrize("shape,B,cap,per_layer", [("small", 1, 16, 5), ("0.6b", 4, 16, 6),
                                                   ("0.6b", 1, 520, 5), ("0.6b", 8, 520, 6)])
def test_step_launch_count(shape, B, cap, per_layer):
    """One step is the embedding, the LM head and per layer: 5 launches
    (the fused stages; no separate norm or SiLU-mul kernels where the
    tensor-core GEMV takes the shapes and B x K <= 8192); past that, here the
    down projection's B x 3072 at B = 4 and 8, the SiLU-mul is a launch of
    its own (6 a layer). Past 4 sequences the LM head is a norm plus a
    tensor-core matmul (one launch more)."""
    cfg = dict(SMALL) if shape == "small" else dict(qg_synth.QWEN3_0_6B)
    cfg["layers"] = min(cfg["layers"], 2)
    model = qg.Qwen3Model(cfg, qg_synth.qwen3_weights(cfg, 23))
    st = model.new_state(B, cap)
    t, p = dev(np.arange(1, B + 1, dtype=np.int32)), dev(np.full(B, 3, np.int32))
    n0 = qg.lib.qg_kernel_launch_count()
    model.qg_decode_step(st, t, p)
    head = 3 if B >= 5 else 2
    assert qg.lib.qg_kernel_launch_count() - n0 == per_layer * cfg["layers"] + head


def test_step_graph_replay_equals_eager_launches():
    """On a non-default stream qg_decode_step records its launches into a
    CUDA graph once and replays it: the replay reads tokens and positions at
    run time (a new token gives new logits), enqueues no kernel launches of
    its own, and gives bit-identical logits and cache rows to the eager
    launches of the same steps."""
    cfg = dict(SMALL)
    w = qg_synth.qwen3_weights(cfg, 24)
    model = qg.Qwen3Model(cfg, w)
    s = torch.cuda.Stream()
    outs = {}
    for mode in ("graph", "eager"):
        qg.lib.qg_step_graphs_enable(1 if mode == "graph" else 0)
        qg.lib.qg_step_graphs_clear()
        st = model.new_state(2, 16)
        t = dev(np.array([5, 900], np.int32))
        pos = dev(np.array([0, 0], np.int32))
        res, launches = [], []
        for p, toks in enumerate(([5, 900], [17, 3], [17, 3], [999, 0])):
            with torch.cuda.stream(s):
                t.copy_(torch.tensor(toks, dtype=torch.int32))
                pos.fill_(p)
                n0 = qg.lib.qg_kernel_launch_count()
                model.qg_decode_step(st, t, pos, stream=s)
                launches.append(qg.lib.qg_kernel_launch_count() - n0)
            s.synchronize()
            res.append((st["logits"].clone(), st["k_cache"].clone()))
        outs[mode] = (res, launches)
    qg.lib.qg_step_graphs_enable(1)
    qg.lib.qg_step_graphs_clear()
    per_step = 5 * cfg["layers"] + 2
    assert outs["eager"][1] == [per_step] * 4
    assert outs["graph"][1] == [per_step, 0, 0, 0]  # recorded once, then replayed
    for (lg, kg), (le, ke) in zip(outs["graph"][0], outs["eager"][0]):
        assert torch.equal(lg, le) and torch.equal(kg, ke)
    assert not torch.equal(outs["graph"][0][0][0], outs["graph"][0][1][0])
