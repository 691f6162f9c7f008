#!/usr/bin/env python
"""Benchmark of the weight-only-quantized decode path on B200.

One step = one decode step of a random-init Qwen3-0.6B-shaped text decoder
(28 layers, hidden 1024, 16 Q / 8 KV heads, head_dim 128, FFN 3072, tied
vocab 151936; affine-INT8 group-64 packed weights) for B sequences at KV
length 512 (position 511, attending 512 cached rows): every hot-path stage
(embedding dequant, RMSNorms, q/k/v, q/k norm + RoPE + KV append, split-KV
attention, o-proj + residual, gate/up + SiLU-mul, down + residual, final norm
and the tied LM head). The step is captured once into a CUDA graph and
replayed. Inputs are seeded synthetic data; the weights of one step total
~692 MB, larger than L2 (126 MB), so nothing survives in L2 between steps.

Multi-GPU: replicas only -- every rank decodes its own sequences with its own
weight copy; no data-path collective. ``value`` is the total steps/s of all
ranks (weak scaling), timed as the max over ranks.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--batch B]
       python bench.py --impl reference   (the CPU oracle on the host cores)
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import qg_synth  # noqa: E402

METRIC = "quantized GEMV HBM GB/s & % of peak; decode steps/s (Qwen3-0.6B shape, b=1)"
FALLBACK_HBM_GBS = 6650.0
KV_LEN = 512


# ------------------------------------------------------------ byte model ----

def affine8_bytes(N, K, B, x_bytes=2, y_bytes=4):
    """Algorithmic bytes of one affine-INT8 g64 GEMV: codes, bf16 scales and
    biases, the activations read and the outputs written."""
    return N * K + N * (K // 64) * 4 + B * K * x_bytes + B * N * y_bytes


def step_bytes(cfg, B, L):
    """Algorithmic bytes of one decode step: every packed weight byte once,
    the norm weights, the embedding row, the K/V rows attended (L per layer
    and sequence, read) and appended (one per layer and sequence)."""
    h, H, Hk, D, F, V = (cfg["hidden"], cfg["heads"], cfg["kv_heads"], cfg["head_dim"],
                         cfg["ffn"], cfg["vocab"])
    sh = qg_synth.linear_shapes(cfg)
    w = sum(affine8_bytes(n, k, 0) for n, k in sh.values()) * cfg["layers"]
    head = affine8_bytes(V, h, 0)
    norms = cfg["layers"] * (2 * h + 2 * D) * 2 + h * 2
    emb = B * (h + (h // 64) * 4)
    kv_read = B * cfg["layers"] * 2 * L * Hk * D * 2
    kv_write = B * cfg["layers"] * 2 * Hk * D * 2
    acts = B * V * 4
    return w + head + norms + emb + kv_read + kv_write + acts


# ------------------------------------------------------------- plumbing -----

def graph_time_ms(fns, stream, n, warm=3):
    """Mean device time of one launch: n launches (fns[i % len(fns)], so
    inputs rotate over several copies) captured back to back in one CUDA graph
    and bracketed by CUDA events on `stream`, the stream they run on; host
    launch overhead is not in the figure."""
    import torch
    with torch.cuda.stream(stream):
        for i in range(warm):
            fns[i % len(fns)]()
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(n):
            fns[i % len(fns)]()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        g.replay()
        e0.record(stream)
        g.replay()
        e1.record(stream)
    stream.synchronize()
    del g
    return e0.elapsed_time(e1) / n


L2_BYTES = 126 << 20


def _tob(a):
    """numpy -> torch on the device (uint16/uint32 travel as int16/int32)."""
    import torch
    return torch.from_numpy(a.view({1: np.uint8, 2: np.int16, 4: np.int32}[a.dtype.itemsize])).cuda()


def _hbm_entry(nbytes, ms, peak, **extra):
    gbs = nbytes / (ms / 1000.0) / 1e9
    d = {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
         "algorithmic_bytes": nbytes, "launch_us": ms * 1000.0}
    d.update(extra)
    return d


def affine8_chain(qg, stream, N, K, B, seed, n_min, hbm_peak):
    """One affine8 GEMV N x K at batch B, timed per launch as a chain of
    launches back to back in a CUDA graph over rotated copies of the matrix
    that together exceed L2 three times (so every launch streams from HBM)."""
    import torch
    wnp, snp, bnp = qg_synth.affine8_packed(N, K, seed)
    per = wnp.nbytes + snp.nbytes + bnp.nbytes
    copies = max(1, -(-3 * L2_BYTES // per))
    mats = [(_tob(wnp), _tob(snp), _tob(bnp)) for _ in range(copies)]
    x = torch.from_numpy(qg_synth.gaussian_bf16_bits((B, K), 1.0, seed + 1).view(np.int16)) \
        .cuda().view(torch.bfloat16)
    y = torch.empty((B, N), dtype=torch.float32, device="cuda")
    fns = [(lambda m=m: qg.qg_gemv_affine8_g64(*m, x, y, stream=stream)) for m in mats]
    ms = graph_time_ms(fns, stream, max(n_min, 2 * copies))
    del mats
    return _hbm_entry(affine8_bytes(N, K, B), ms, hbm_peak,
                      note=f"chain in a CUDA graph over {copies} copies (> 3x L2)")


def c1_c2_gemvs(qg, stream, hbm_peak):
    """C1: the 1024 x 1024 GEMV at B = 1 as a chain of 512 launches. C2: the
    Qwen3-0.6B layer set (q, k, v, o, gate, up, down) and the tied LM head
    151936 x 1024 at B = 1, 4 and 16."""
    out = {"gemv_affine8_1024x1024_b1_chain": affine8_chain(qg, stream, 1024, 1024, 1, 31, 512,
                                                           hbm_peak)}
    cfg = qg_synth.QWEN3_0_6B
    sh = dict(qg_synth.linear_shapes(cfg))
    sh["lm_head"] = (cfg["vocab"], cfg["hidden"])
    c2 = {}
    for B in (1, 4, 16):
        for i, (name, (N, K)) in enumerate(sh.items()):
            c2[f"{name}_b{B}"] = affine8_chain(qg, stream, N, K, B, 40 + i, 64, hbm_peak)
    tot = {B: sum(c2[f"{n}_b{B}"]["algorithmic_bytes"] for n in sh) for B in (1, 4, 16)}
    us = {B: sum(c2[f"{n}_b{B}"]["launch_us"] for n in sh) for B in (1, 4, 16)}
    out["c2_qwen3_0.6b_layer_set"] = {
        "workload": "Qwen3-0.6B layer GEMVs q 2048x1024, k/v 1024x1024, o 1024x2048, gate/up "
                    "3072x1024, down 1024x3072 and the tied LM head 151936x1024, affine8 g64",
        "per_matrix": c2,
        "set_gbs": {f"b{B}": tot[B] / (us[B] / 1e6) / 1e9 for B in (1, 4, 16)},
        "set_frac": {f"b{B}": tot[B] / (us[B] / 1e6) / 1e9 / hbm_peak for B in (1, 4, 16)},
        "note": "each matrix timed alone per launch (chained launches in a CUDA graph, "
                "inputs rotated over > 3x L2); set figures = total bytes / summed launch times"}
    return out


def c4_whisper(qg, stream, hbm_peak):
    """C4: the Whisper-large-v3 encoder's Q4_0 matmuls at M = 1500 on the
    tensor cores (Q/K/V/O 1280x1280, FC1 5120x1280, FC2 1280x5120) and the
    same matrices as batch-1 Q4_0 GEMVs."""
    import torch
    M = 1500
    tf_peak, tf_kind = measured_tensor_peak()
    gemm = {}
    for name, (N, K) in (("qkvo_1280x1280", (1280, 1280)), ("fc1_5120x1280", (5120, 1280)),
                         ("fc2_1280x5120", (1280, 5120))):
        blocks = _tob(qg_synth.q4_0_packed(N, K, 22))
        A = torch.from_numpy(qg_synth.gaussian((M, K), 1.0, 23).astype(np.float32)).cuda()
        bias = torch.from_numpy(qg_synth.gaussian((N,), 0.1, 24).astype(np.float32)).cuda()
        C = torch.empty((M, N), dtype=torch.float32, device="cuda")
        ws = torch.empty(qg.qg_gemm_q4_0_workspace_size(M, N, K), dtype=torch.uint8, device="cuda")
        ms = graph_time_ms([lambda: qg.qg_gemm_q4_0(blocks, A, C, bias=bias, ws=ws, stream=stream)],
                           stream, 50)
        tf = 2.0 * M * N * K / (ms / 1000.0) / 1e12
        gemm[name] = {"shape": [M, N, K], "bound": "tensor", "achieved": tf, "peak": tf_peak,
                      "unit": "TFLOP/s", "frac": tf / tf_peak, "launch_us": ms * 1000.0,
                      "peak_kind": tf_kind}
    gemv = {}
    for name, (N, K) in (("1280x1280", (1280, 1280)), ("5120x1280", (5120, 1280)),
                         ("1280x5120", (1280, 5120))):
        bnp = qg_synth.q4_0_packed(N, K, 25)
        copies = -(-3 * L2_BYTES // bnp.nbytes)
        mats = [_tob(bnp) for _ in range(copies)]
        x = torch.from_numpy(qg_synth.gaussian((1, K), 1.0, 13).astype(np.float32)).cuda()
        bias = torch.from_numpy(qg_synth.gaussian((N,), 0.1, 26).astype(np.float32)).cuda()
        y = torch.empty((1, N), dtype=torch.float32, device="cuda")
        fns = [(lambda m=m: qg.qg_gemv_q4_0(m, x, y, bias=bias, stream=stream)) for m in mats]
        ms = graph_time_ms(fns, stream, max(100, 2 * copies))
        vbytes = N * (K // 32) * 18 + K * 4 + N * 4 + N * 4
        gemv[name] = _hbm_entry(vbytes, ms, hbm_peak,
                                note=f"chain in a CUDA graph over {copies} copies (> 3x L2)")
        del mats
    # the whole encoder layer (LN, q/k/v, attention, out + residual, LN, fc1 +
    # GELU, fc2 + residual): nine launches per call; x is restored from a
    # pristine copy before each call and that copy's own time is subtracted
    try:
        layer_entry = whisper_layer_entry(qg, stream, M, tf_peak)
    except Exception as e:  # noqa: BLE001
        stream.synchronize()
        layer_entry = {"error": f"{type(e).__name__}: {e}"[:300]}
    return {"c4_whisper_q4_0": {
        "workload": "Whisper-large-v3 encoder projections as Q4_0 blk32, M = 1500 frames "
                    "(GEMM, f32 activations rounded to bf16) and batch 1 (GEMV)",
        "gemm": gemm, "gemv_b1": gemv, "encoder_layer": layer_entry,
        "note": "GEMM FLOPs 2*M*N*K (dequant work not counted), includes the A fp32->bf16 pass"}}


def whisper_layer_entry(qg, stream, M, tf_peak):
    """The Whisper-large-v3 encoder layer at M frames, timed per call."""
    import torch
    wcfg = dict(qg_synth.WHISPER_LARGE_V3)
    layer = qg.WhisperEncoderLayer(wcfg, qg_synth.whisper_layer_weights(wcfg, 500))
    d, F, H = wcfg["d_model"], wcfg["ffn"], wcfg["heads"]
    x0 = torch.from_numpy(qg_synth.gaussian((M, d), 1.0, 501)).cuda()
    x = x0.clone()
    lws = layer.workspace(M)
    ms_all = graph_time_ms([lambda: (x.copy_(x0), layer.qg_whisper_encoder_layer(x, lws,
                                                                              stream=stream))],
                           stream, 20)
    ms_cp = graph_time_ms([lambda: x.copy_(x0)], stream, 20)
    ms_l = ms_all - ms_cp
    flops = 2.0 * M * (4 * d * d + 2 * d * F) + 4.0 * M * M * d
    tf = flops / (ms_l / 1000.0) / 1e12
    return {"workload": "Whisper-large-v3 encoder layer, M = 1500, Q4_0 weights",
            "us_per_layer": ms_l * 1000.0, "flops": flops, "achieved": tf,
            "peak": tf_peak, "unit": "TFLOP/s", "frac": tf / tf_peak,
            "launches": 9, "note": "FLOPs: the six matmuls 2*M*N*K and the attention "
                                   "4*M^2*d (softmax and LayerNorms not counted)"}


def step_graph(model, st, toks, pos, stream):
    """One decode step captured into a CUDA graph (after two eager steps)."""
    import torch
    with torch.cuda.stream(stream):
        for _ in range(2):
            model.qg_decode_step(st, toks, pos, stream=stream)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        model.qg_decode_step(st, toks, pos, stream=stream)
    return g


def time_replays(g, stream, n, warm=3):
    import torch
    with torch.cuda.stream(stream):
        for _ in range(warm):
            g.replay()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(n):
            g.replay()
        e1.record(stream)
    stream.synchronize()
    return e0.elapsed_time(e1) / n


def c3_batch10(qg, stream, hbm_peak, model, cfg):
    """C3 at batch 10: the 0.6B step at KV 512 for 10 sequences."""
    import torch
    B = 10
    st = model.new_state(B, KV_LEN + 1)
    st["k_cache"].normal_()
    st["v_cache"].normal_()
    toks = torch.from_numpy(qg_synth.tokens(B, cfg["vocab"], 73)).cuda()
    pos = torch.full((B,), KV_LEN - 1, dtype=torch.int32, device="cuda")
    g = step_graph(model, st, toks, pos, stream)
    ms = time_replays(g, stream, 100)
    del g, st
    sb = step_bytes(cfg, B, KV_LEN)
    return {"c3_qwen3_0.6b_step_b10_kv512": {
        "steps_per_s": 1000.0 / ms, "tokens_per_s": B * 1000.0 / ms, "us_per_step": ms * 1000.0,
        "algorithmic_bytes": sb, "achieved": sb / (ms / 1000.0) / 1e9, "peak": hbm_peak,
        "unit": "GB/s", "frac": sb / (ms / 1000.0) / 1e9 / hbm_peak}}


def c5_1_7b(qg, stream, hbm_peak):
    """C5: the Qwen3-1.7B-shaped decode (hidden 2048, FFN 6144, 28 layers,
    vocab 151936) at KV 2048 (position 2047) for batch 1, 8 and 32, and the
    256-row prefill (as decode steps at positions 0..255, batch 1)."""
    import torch
    import weight_only_quantized_03_b200 as qgm
    cfg = dict(qg_synth.QWEN3_1_7B)
    model = qgm.Qwen3Model(cfg, qg_synth.qwen3_weights(cfg, 19))
    cap = 2049
    out = {"workload": "Qwen3-1.7B-shaped affine-INT8 g64 decode, KV 2048", "points": {}}
    for B in (1, 8, 32):
        st = model.new_state(B, cap)
        st["k_cache"].normal_()
        st["v_cache"].normal_()
        toks = torch.from_numpy(qg_synth.tokens(B, cfg["vocab"], 92)).cuda()
        pos = torch.full((B,), 2047, dtype=torch.int32, device="cuda")
        g = step_graph(model, st, toks, pos, stream)
        ms = time_replays(g, stream, 30)
        sb = step_bytes(cfg, B, 2048)
        out["points"][f"b{B}"] = {"us_per_step": ms * 1000.0, "tokens_per_s": B * 1000.0 / ms,
                                  "algorithmic_bytes": sb, "achieved": sb / (ms / 1000.0) / 1e9,
                                  "frac": sb / (ms / 1000.0) / 1e9 / hbm_peak}
        del g, st
        torch.cuda.empty_cache()
    out["prefill_256_rows"] = prefill_rows(qg, model, cfg, stream)
    out["peak"] = hbm_peak
    out["unit"] = "GB/s"
    return {"c5_qwen3_1.7b": out}


def prefill_rows(qg, model, cfg, stream):
    """256 prompt rows of one sequence at positions 0..255: the batched
    prefill (qg_prefill: every layer's linears as tensor-core matmuls over
    all rows, causal multi-row attention; the call's launches timed with CUDA
    events, host launch time included) and, for comparison, the same rows
    run one at a time as decode steps (graph replays)."""
    import torch
    T = 256
    st = model.new_state(1, 2049)
    toks = torch.from_numpy(qg_synth.tokens(T, cfg["vocab"], 91)).cuda()
    ws = model.prefill_workspace(T)
    logits = torch.empty(cfg["vocab"], dtype=torch.float32, device="cuda")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        for _ in range(2):
            model.qg_prefill(st, toks, 0, ws, logits=logits, stream=stream)
        reps = 5
        e0.record(stream)
        for _ in range(reps):
            model.qg_prefill(st, toks, 0, ws, logits=logits, stream=stream)
        e1.record(stream)
    stream.synchronize()
    ms_b = e0.elapsed_time(e1) / reps
    pos = torch.zeros(1, dtype=torch.int32, device="cuda")
    tok1 = toks[:1].clone()
    g = step_graph(model, st, tok1, pos, stream)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for r in range(T):
            pos.fill_(r)
            tok1.copy_(toks[r:r + 1])
            g.replay()
        e1.record(stream)
    stream.synchronize()
    ms_r = e0.elapsed_time(e1)
    del g, st
    return {"batched": {"ms": ms_b, "rows_per_s": T / (ms_b / 1000.0),
                        "method": "qg_prefill: all rows per layer on the tensor cores"},
            "row_at_a_time": {"ms": ms_r, "rows_per_s": T / (ms_r / 1000.0),
                              "method": "one decode step (graph replay) per row"},
            "speedup": ms_r / ms_b}


def code_predictor_frame(qg, stream, hbm_peak, n):
    """One frame of the makima Qwen3-TTS code predictor (hidden 1024, 5
    layers, 16 heads, head_dim 64, FFN 3072, 16 groups of 2048 codes; random
    packed weights), batch 1: the 15 sequential groups of one
    qg_code_predict call, timed with CUDA events over n back-to-back calls
    (each call replays the recorded graph of the whole frame)."""
    import torch
    import weight_only_quantized_03_b200 as qgm
    cfg, G = dict(qg_synth.CODE_PREDICTOR), qg_synth.CODE_GROUPS
    model = qgm.CodePredictor(cfg, qg_synth.code_predictor_weights(cfg, G, 51))
    lm = torch.from_numpy(qg_synth.gaussian((1, cfg["hidden"]), 1.0, 52).astype(np.float32)).cuda()
    code0 = torch.tensor([7], dtype=torch.int32, device="cuda")
    codes = torch.empty((G, 1), dtype=torch.int32, device="cuda")
    ws = model.workspace(1)
    n0 = qg.lib.qg_kernel_launch_count()  # the first call records the frame's launches
    with torch.cuda.stream(stream):
        for _ in range(3):
            model.qg_code_predict(lm, code0, codes, ws, stream=stream)
    stream.synchronize()
    launches = qg.lib.qg_kernel_launch_count() - n0
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(n):
            model.qg_code_predict(lm, code0, codes, ws, stream=stream)
        e1.record(stream)
    stream.synchronize()
    ms = e0.elapsed_time(e1) / n
    h, F, V = cfg["hidden"], cfg["ffn"], cfg["vocab"]
    HD = cfg["heads"] * cfg["head_dim"]
    layer = sum(affine8_bytes(N, K, 1) for N, K in
                ((HD, h), (HD, h), (HD, h), (h, HD), (F, h), (F, h), (h, F)))
    group = cfg["layers"] * layer + affine8_bytes(h, 2 * h, 1) + affine8_bytes(V, h, 1)
    fbytes = (G - 1) * group
    return {"workload": "Qwen3-TTS code predictor frame (makima CodePredictorConfig), batch 1",
            "frames_per_s": 1000.0 / ms, "ms_per_frame": ms, "groups": G - 1,
            "launches_per_frame": launches, "algorithmic_bytes": fbytes,
            "achieved": fbytes / (ms / 1000.0) / 1e9, "peak": hbm_peak, "unit": "GB/s",
            "note": "weights are read once per group (15 per frame); the 5 layers' 72 MB "
                    "can stay in L2 between groups, so achieved may pass the HBM peak"}


def measured_tensor_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["bf16_tflops"]), "measured (bf16 burst)"
    except Exception:
        return 1590.0, "fallback"


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def source_sha256(paths):
    """sha256 over the given source files, concatenated in order."""
    h = hashlib.sha256()
    for p in paths:
        h.update(open(p, "rb").read())
    return h.hexdigest()


GEMV_SOURCES = [os.path.join(ROOT, "weight_only_quantized_03_b200", "csrc", f)
                for f in ("gemv_affine8_tc.cu", "gemv_tc.cuh", "qg_internal.cuh")]
LM_HEAD_SOURCES = GEMV_SOURCES
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")


def traffic_from_profile(kernel_files, key="gemv_affine8_lm_head_151936x1024_b1",
                         field="dram_bytes_per_launch"):
    """DRAM bytes (read + written) of a kernel from one ncu capture, kept in
    profiles/traffic.json, or None when the entry is missing or was taken on
    a different version of the kernel sources (their sha256 must match)."""
    try:
        with open(TRAFFIC_FILE) as f:
            d = json.load(f)[key]
    except (OSError, KeyError, ValueError):
        return None
    if d.get("kernel_source_sha256") != source_sha256(kernel_files):
        return None
    return d.get(field)


def step_gemv_traffic(B):
    """DRAM bytes per step of the step's layer GEMV launches (batch 1 only)."""
    if B != 1:
        return None
    return traffic_from_profile(GEMV_SOURCES, "step_layer_gemvs_qwen3_0.6b_b1_kv512",
                                "dram_bytes_per_step")


class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons while running."""
    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.rows = []
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) == 6:
                self.rows.append(parts)

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm = [float(r[0]) for r in self.rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in self.rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in self.rows for i in range(4) if r[2 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(self.rows)}


def cpu_cores():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("user_api") == "blas"]
        if n and n[0]:
            return int(n[0])
    except Exception:
        pass
    return os.cpu_count()


# ------------------------------------------------------ oracle (CPU) legs ---

def oracle_sample(cfg, weights, budget_steps=None, layers_only=None):
    """Time the CPU oracle on a bounded sample of the decode step: whole
    steps (28 layers + LM head) or, with ``layers_only``, that many single
    layers plus one LM head, scaled to a whole step. Returns (steps/s,
    description)."""
    from oracle import qg_oracle as O
    Hk, D = cfg["kv_heads"], cfg["head_dim"]
    cap = KV_LEN + 1
    kc = O.bf16_bits_to_f64(qg_synth.gaussian_bf16_bits((cfg["layers"], Hk, cap, D), 1.0, 70))
    vc = O.bf16_bits_to_f64(qg_synth.gaussian_bf16_bits((cfg["layers"], Hk, cap, D), 1.0, 71))
    tok = int(qg_synth.tokens(1, cfg["vocab"], 72)[0])
    if layers_only is None:
        t0 = time.perf_counter()
        for _ in range(budget_steps):
            O.decode_step(cfg, weights, kc, vc, tok, KV_LEN - 1)
        dt = (time.perf_counter() - t0) / budget_steps
        return 1.0 / dt, f"{budget_steps} full decode step(s) at position {KV_LEN - 1}, batch 1"
    ew, es, eb = weights["embed"]
    x = O.embed_rows(ew, es, eb, [tok])[0]
    t0 = time.perf_counter()
    for i in range(layers_only):
        l = i % cfg["layers"]
        x = O.decode_layer(cfg, weights["layers"][l], x, kc[l], vc[l], KV_LEN - 1)
    t_layer = (time.perf_counter() - t0) / layers_only
    t0 = time.perf_counter()
    O.lm_head(cfg, weights, x)
    t_head = time.perf_counter() - t0
    return 1.0 / (cfg["layers"] * t_layer + t_head), (
        f"{layers_only} single decoder layers at position {KV_LEN - 1} plus one LM head, "
        f"scaled to 28 layers + head, batch 1")


def run_reference(args):
    """The oracle on the host cores, as it stands. Each of the W + K steps is
    a bounded sample of the workload: one decoder layer of the 0.6B step at
    position 511 (a full step is 28 layers and the LM head). The LM head is
    timed once after the timed samples. ``ms_per_step`` is the measured time
    of one sample; ``value`` is the full-step rate those times give
    (1 / (28 x mean layer time + LM head time)), marked as extrapolated."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from oracle import qg_oracle as O
    cfg = dict(qg_synth.QWEN3_0_6B)
    weights = qg_synth.qwen3_weights(cfg, 11)
    Hk, D = cfg["kv_heads"], cfg["head_dim"]
    cap = KV_LEN + 1
    kc = O.bf16_bits_to_f64(qg_synth.gaussian_bf16_bits((cfg["layers"], Hk, cap, D), 1.0, 70))
    vc = O.bf16_bits_to_f64(qg_synth.gaussian_bf16_bits((cfg["layers"], Hk, cap, D), 1.0, 71))
    tok = int(qg_synth.tokens(1, cfg["vocab"], 72)[0])
    x = O.embed_rows(*weights["embed"], [tok])[0]
    for i in range(args.warmup):
        O.decode_layer(cfg, weights["layers"][i % cfg["layers"]], x, kc[0], vc[0], KV_LEN - 1)
    t0 = time.perf_counter()
    for i in range(args.steps):
        l = i % cfg["layers"]
        x = O.decode_layer(cfg, weights["layers"][l], x, kc[l], vc[l], KV_LEN - 1)
    t_layers = time.perf_counter() - t0
    t0 = time.perf_counter()
    O.lm_head(cfg, weights, x)
    t_head = time.perf_counter() - t0
    t_layer = t_layers / args.steps
    v = 1.0 / (cfg["layers"] * t_layer + t_head)
    cores = cpu_cores()
    desc = (f"each timed step: one decoder layer of the 28 at position {KV_LEN - 1}, batch 1 "
            f"({args.steps} timed, layers in order); the LM head timed once ({t_head:.3f} s)")
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "steps/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * t_layer, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"Qwen3-0.6B-shaped affine-INT8 g64 decode step, batch 1, KV {KV_LEN}"},
        "sample": {"timed_step": "one decoder layer (1/28 of the layers of a decode step)",
                   "ms_per_step_is": "measured time of one sample (one layer)",
                   "value_is": "extrapolated full-step rate: 1 / (28 x mean layer time + LM head time)",
                   "full_step_s": 1.0 / v, "lm_head_s": t_head},
        "cpu_baseline": {"value": v, "unit": "steps/s", "cores": cores, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": v, "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------ ranks ---------

def max_over_ranks(ms, world, dist=None, device="cpu"):
    """The slowest rank's time: every rank contributes its own device time
    and all get the maximum (an all-reduce, the same collective on every
    rank); with one rank, the time itself."""
    if world <= 1:
        return ms
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_value(world, units_per_rank, max_ms):
    """Whole-job throughput of independent replicas: the units all ranks
    processed over the slowest rank's time."""
    return world * units_per_rank / (max_ms / 1000.0)


# ------------------------------------------------------------ GPU arm -------

TIMELINE_NAMES = {1: "embed", 2: "qkv", 3: "attn", 4: "o", 5: "gate_up", 6: "down", 7: "head",
                  8: "other"}
GEMV_KINDS = ("qkv", "o", "gate_up", "down")


def run_timeline(args):
    """The timeline leg (run by the main arm as a subprocess on the
    diagnostic build, QG_LIBRARY=libqg_timeline.so): one step of the bench
    workload captured into a CUDA graph with per-launch %globaltimer records,
    replayed 5 times with L2 flushed before each; per launch kind, the median
    over replays of the summed step share (each launch's exit minus the
    previous launch's exit, i.e. its part of the critical path). Prints one
    JSON line."""
    import ctypes
    import torch
    import weight_only_quantized_03_b200 as qg
    if not qg.lib.qg_timeline_available():
        print(json.dumps({"unavailable": "library built without QG_TIMELINE"}))
        return 0
    cfg = dict(qg_synth.QWEN3_0_6B)
    B = args.batch
    model = qg.Qwen3Model(cfg, qg_synth.qwen3_weights(cfg, 11))
    st = model.new_state(B, KV_LEN + 1)
    st["k_cache"].normal_()
    st["v_cache"].normal_()
    toks = torch.from_numpy(qg_synth.tokens(B, cfg["vocab"], 72)).cuda()
    pos = torch.full((B,), KV_LEN - 1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        for _ in range(3):
            model.qg_decode_step(st, toks, pos, stream=stream)
    stream.synchronize()
    nrec = 1024
    rec = torch.zeros(nrec * 4, dtype=torch.int64, device="cuda")
    flush = torch.empty(L2_BYTES * 2, dtype=torch.uint8, device="cuda")
    assert qg.lib.qg_timeline_begin(ctypes.c_void_p(rec.data_ptr()), nrec) == 0
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        model.qg_decode_step(st, toks, pos, stream=stream)
    kinds = (ctypes.c_int * nrec)()
    n = qg.lib.qg_timeline_end(kinds, nrec)
    shares, spans = [], []
    for rep in range(6):
        with torch.cuda.stream(stream):
            flush.fill_(rep & 0xFF)
            rec.zero_()
            g.replay()
        stream.synchronize()
        if rep == 0:
            continue
        r = rec.view(nrec, 4).cpu().numpy().astype(np.uint64)[:n]
        entry = (~r[:, 0]).astype(np.int64)
        ex = r[:, 2].astype(np.int64)
        prev = np.concatenate([[entry[0]], ex[:-1]])
        d = {}
        for i in range(n):
            k = TIMELINE_NAMES.get(kinds[i], "other")
            d[k] = d.get(k, 0.0) + (ex[i] - prev[i]) / 1e3
        shares.append(d)
        spans.append((ex[-1] - entry[0]) / 1e3)
    del g
    med = {k: statistics.median(d[k] for d in shares) for k in shares[0]}
    counts = {}
    for i in range(n):
        k = TIMELINE_NAMES.get(kinds[i], "other")
        counts[k] = counts.get(k, 0) + 1
    print(json.dumps({"launches": n, "span_us": statistics.median(spans), "share_us": med,
                      "count": counts}), flush=True)
    return 0


def timeline_leg(batch):
    """Runs the timeline leg in a subprocess (the diagnostic build is a
    separate library); None when it is missing or fails."""
    lib = os.path.join(ROOT, "weight_only_quantized_03_b200", "libqg_timeline.so")
    if not os.path.exists(lib):
        return None
    env = dict(os.environ, QG_LIBRARY="libqg_timeline.so")
    try:
        r = subprocess.run([sys.executable, os.path.abspath(__file__), "--timeline-leg",
                            "--batch", str(batch)], env=env, capture_output=True, text=True,
                           timeout=600)
        line = [l for l in r.stdout.splitlines() if l.startswith("{")][-1]
        d = json.loads(line)
        return None if "unavailable" in d else d
    except Exception:
        return None


def gemv_class_bytes(cfg, B):
    """Algorithmic bytes per step of the layer GEMV launches (q/k/v, o,
    gate/up, down of every layer): codes, scales, biases, the bf16 inputs
    and the fp32 outputs (and residual reads of o and down)."""
    h, F = cfg["hidden"], cfg["ffn"]
    HD, KD = cfg["heads"] * cfg["head_dim"], cfg["kv_heads"] * cfg["head_dim"]
    per_layer = (affine8_bytes(HD + 2 * KD, h, B) + affine8_bytes(h, HD, B) + B * h * 4
                 + affine8_bytes(2 * F, h, B) + affine8_bytes(h, F, B) + B * h * 4)
    return cfg["layers"] * per_layer


def run_ours(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    import weight_only_quantized_03_b200 as qg

    def barrier():
        if world > 1:
            dist.barrier()

    cfg = dict(qg_synth.QWEN3_0_6B)
    B = args.batch
    weights = qg_synth.qwen3_weights(cfg, 11)
    model = qg.Qwen3Model(cfg, weights, device=f"cuda:{local}")
    cap = KV_LEN + 1
    st = model.new_state(B, cap)
    kshape = (cfg["layers"], B, cfg["kv_heads"], cap, cfg["head_dim"])
    st["k_cache"].copy_(torch.from_numpy(qg_synth.gaussian_bf16_bits(kshape, 1.0, 70).view(np.int16))
                        .view(torch.bfloat16))
    st["v_cache"].copy_(torch.from_numpy(qg_synth.gaussian_bf16_bits(kshape, 1.0, 71).view(np.int16))
                        .view(torch.bfloat16))
    toks_np = qg_synth.tokens(B, cfg["vocab"], 72 + rank)
    pos_np = np.full(B, KV_LEN - 1, dtype=np.int32)
    toks = torch.from_numpy(toks_np).cuda()
    pos = torch.from_numpy(pos_np).cuda()
    stream = torch.cuda.Stream()
    hbm_peak, peak_kind = measured_peaks()

    # the clock sampler runs from the warm-up to the end of the measurements
    clk = ClockSampler(local).__enter__()
    # ---- capture one step into a CUDA graph
    with torch.cuda.stream(stream):
        for _ in range(3):
            model.qg_decode_step(st, toks, pos)
    stream.synchronize()
    graph = torch.cuda.CUDAGraph()
    n0 = qg.lib.qg_kernel_launch_count()
    with torch.cuda.graph(graph, stream=stream):
        model.qg_decode_step(st, toks, pos)
    launches_per_step = qg.lib.qg_kernel_launch_count() - n0

    # ---- warm-up, then K timed replays
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            graph.replay()
    stream.synchronize()
    barrier()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    barrier()
    with torch.cuda.stream(stream):
        ev0.record(stream)
        for _ in range(args.steps):
            graph.replay()
        ev1.record(stream)
    stream.synchronize()
    torch.cuda.synchronize()
    barrier()
    ms = max_over_ranks(ev0.elapsed_time(ev1), world, dist, "cuda")
    ms_per_step = ms / args.steps
    value = aggregate_value(world, args.steps, ms)

    # ---- the tied LM-head GEMV (151936 x 1024) alone, timed per launch
    V, h = cfg["vocab"], cfg["hidden"]
    ew, es, eb = [torch.from_numpy(a.view({2: np.int16, 4: np.int32}[a.dtype.itemsize])).cuda()
                  for a in weights["embed"]]
    xb = torch.from_numpy(qg_synth.gaussian_bf16_bits((B, h), 1.0, 5).view(np.int16)).cuda() \
        .view(torch.bfloat16)
    yl = torch.empty((B, V), dtype=torch.float32, device="cuda")
    nlaunch = max(20, min(200, args.steps))
    # back to back in a CUDA graph; the 166 MB table exceeds L2 on its own
    lm_ms = graph_time_ms([lambda: qg.qg_gemv_affine8_g64(ew, es, eb, xb, yl, stream=stream)],
                          stream, nlaunch)
    lm_bytes = affine8_bytes(V, h, B)
    kernels = {"gemv_affine8_lm_head_151936x1024": _hbm_entry(
        lm_bytes, lm_ms, hbm_peak, batch=B, traffic=traffic_from_profile(LM_HEAD_SOURCES)
        if B == 1 else None, note="back-to-back launches in a CUDA graph")}

    # ---- e2e through the public API with host buffers: token and position
    # in from pinned host memory, then either the greedy token (argmax on the
    # device, 4 bytes a sequence) or the whole logits back to the host
    h_tok = torch.from_numpy(toks_np).pin_memory()
    h_pos = torch.from_numpy(pos_np).pin_memory()
    h_logits = torch.empty((B, V), dtype=torch.float32).pin_memory()
    h_next = torch.empty(B, dtype=torch.int32).pin_memory()
    next_tok = torch.empty(B, dtype=torch.int32, device="cuda")
    am_ws = torch.empty(qg.qg_argmax_workspace_size(B, V), dtype=torch.uint8, device="cuda")
    e2e_steps = max(10, min(args.steps, 200))

    def e2e_run(on_device_argmax):
        def one():
            toks.copy_(h_tok, non_blocking=True)
            pos.copy_(h_pos, non_blocking=True)
            model.qg_decode_step(st, toks, pos, stream=stream)
            if on_device_argmax:
                qg.qg_argmax_f32(st["logits"], next_tok, am_ws, stream=stream)
                h_next.copy_(next_tok, non_blocking=True)
            else:
                h_logits.copy_(st["logits"], non_blocking=True)
        with torch.cuda.stream(stream):
            for _ in range(3):
                one()
        stream.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(e2e_steps):
                one()
            e1.record(stream)
        stream.synchronize()
        ms = max_over_ranks(e0.elapsed_time(e1), world, dist, "cuda")
        return aggregate_value(world, e2e_steps, ms)

    e2e_value = e2e_run(True)
    e2e_logits_value = e2e_run(False)
    # the same step both times: the device's greedy token is the host's
    e2e_token_ok = all(int(h_next[b]) == int(torch.argmax(h_logits[b])) for b in range(B))
    del graph

    # ---- the other configurations, each timed per launch on its stream; a
    # leg that fails is reported in its own entry, the line still printed
    def leg(name, fn):
        try:
            kernels.update(fn())
        except Exception as e:  # noqa: BLE001
            stream.synchronize()
            kernels[name] = {"error": f"{type(e).__name__}: {e}"[:300]}

    if not args.quick:
        leg("c1_c2", lambda: c1_c2_gemvs(qg, stream, hbm_peak))
        leg("c3_qwen3_0.6b_step_b10_kv512", lambda: c3_batch10(qg, stream, hbm_peak, model, cfg))
        leg("c4_whisper_q4_0", lambda: c4_whisper(qg, stream, hbm_peak))
        leg("c5_qwen3_1.7b", lambda: c5_1_7b(qg, stream, hbm_peak))
        leg("code_predictor_frame", lambda: {"code_predictor_frame": code_predictor_frame(
            qg, stream, hbm_peak, max(10, min(50, args.steps)))})
    clk.__exit__(None, None, None)

    # ---- the step's dominant kernel class: its layer GEMV launches, from the
    # in-graph timeline of the same step (diagnostic build, subprocess)
    tl = timeline_leg(B) if rank == 0 and world == 1 and not args.no_timeline else None
    sb = step_bytes(cfg, B, KV_LEN)
    gb = gemv_class_bytes(cfg, B)
    if tl:
        gemv_us = sum(tl["share_us"].get(k, 0.0) for k in GEMV_KINDS)
        roof = {"bound": "hbm", "kernel": "gemv_tc_kernel: the step's layer GEMV launches "
                f"(q/k/v, o, gate/up, down; {sum(tl['count'].get(k, 0) for k in GEMV_KINDS)} "
                "per step)",
                "achieved": gb / (gemv_us / 1e6) / 1e9, "peak": hbm_peak, "unit": "GB/s",
                "frac": gb / (gemv_us / 1e6) / 1e9 / hbm_peak,
                "traffic": step_gemv_traffic(B), "algorithmic_bytes": gb,
                "in_graph_us_per_step": gemv_us, "peak_kind": peak_kind,
                "timing": "in-graph %globaltimer timeline of the bench step (diagnostic build): "
                          "each launch's exit minus the previous launch's exit, summed",
                "timeline": tl}
    else:
        lm = kernels["gemv_affine8_lm_head_151936x1024"]
        roof = dict(lm, kernel="gemv_affine8 (LM head 151936x1024)", peak_kind=peak_kind,
                    note="timeline build unavailable: the LM-head launch alone")
    line = {
        "metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded random packed weights, N(0,1) bf16 KV cache)",
        "config": {
            "workload": f"Qwen3-0.6B-shaped affine-INT8 g64 decode step, batch {B}, KV {KV_LEN}",
            "batch": B, "kv_len": KV_LEN, "layers": cfg["layers"], "hidden": cfg["hidden"],
            "vocab": cfg["vocab"], "parallelism": f"replicas x{world}",
            "l2": f"inputs larger than L2 ({sb / 1e6:.0f} MB per step)", "graph": "CUDA graph + PDL",
        },
        "roofline": roof,
        "step_roofline": {"algorithmic_bytes": sb, "achieved": sb / (ms_per_step / 1000.0) / 1e9,
                          "peak": hbm_peak, "unit": "GB/s",
                          "frac": sb / (ms_per_step / 1000.0) / 1e9 / hbm_peak},
        "e2e": {"value": e2e_value, "unit": "steps/s", "h2d_bytes_per_step": 2 * 4 * B,
                "d2h_bytes_per_step": 4 * B, "result": "greedy token (argmax on the device)",
                "token_matches_host_argmax": e2e_token_ok},
        "e2e_logits": {"value": e2e_logits_value, "unit": "steps/s",
                       "h2d_bytes_per_step": 2 * 4 * B, "d2h_bytes_per_step": 4 * B * V},
        "kernels": kernels,
        "gpu_launches": int(launches_per_step * args.steps),
        "clocks": clk.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, desc = oracle_sample(cfg, weights, budget_steps=1)
        line["cpu_baseline"] = {"value": v, "unit": "steps/s", "cores": cpu_cores(),
                                "kind": "oracle", "sample": desc}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_ncu_case(args):
    """One kernel alone, warm-up then ``--steps`` launches, for an ncu capture
    (no timing, no JSON line): ``step`` is the bench's whole decode step
    (launched eagerly, no step graph); ``lm_head`` is the tied LM-head GEMV of the
    0.6B shape at ``--batch``; ``gemm`` the Whisper FC1 Q4_0 GEMM
    (1500 x 5120 x 1280); ``attn`` the decode attention at the 1.7B shape,
    batch 32, KV 2048."""
    import torch
    import weight_only_quantized_03_b200 as qg
    to = lambda a: torch.from_numpy(a.view({1: np.uint8, 2: np.int16, 4: np.int32}[a.dtype.itemsize])).cuda()
    if args.ncu_case == "step":
        # the bench's decode step (0.6B shape, KV 512) launched eagerly: 5
        # launches per layer plus the embedding and the LM head per step
        cfg = dict(qg_synth.QWEN3_0_6B)
        model = qg.Qwen3Model(cfg, qg_synth.qwen3_weights(cfg, 11))
        B = args.batch
        st = model.new_state(B, KV_LEN + 1)
        st["k_cache"].normal_()
        st["v_cache"].normal_()
        toks = torch.from_numpy(qg_synth.tokens(B, cfg["vocab"], 72)).cuda()
        pos = torch.full((B,), KV_LEN - 1, dtype=torch.int32, device="cuda")
        qg.lib.qg_step_graphs_enable(0)
        run = lambda: model.qg_decode_step(st, toks, pos)
    elif args.ncu_case == "lm_head":
        cfg = qg_synth.QWEN3_0_6B
        V, h = cfg["vocab"], cfg["hidden"]
        w, s, b = (to(a) for a in qg_synth.affine8_packed(V, h, 4242))
        x = to(qg_synth.gaussian_bf16_bits((args.batch, h), 1.0, 5)).view(torch.bfloat16)
        y = torch.empty((args.batch, V), dtype=torch.float32, device="cuda")
        run = lambda: qg.qg_gemv_affine8_g64(w, s, b, x, y)
    elif args.ncu_case == "attn":
        # the 1.7B attention shape at batch 32 and KV 2048: 268 MB of K/V
        B, H, Hkv, D, L = 32, 16, 8, 128, 2048
        q = to(qg_synth.gaussian((B, H * D), 1.0, 30).astype(np.float32)).view(torch.float32)
        kc = to(qg_synth.gaussian_bf16_bits((B, Hkv, L, D), 1.0, 31)).view(torch.bfloat16)
        vc = to(qg_synth.gaussian_bf16_bits((B, Hkv, L, D), 1.0, 32)).view(torch.bfloat16)
        kv_len = torch.full((B,), L, dtype=torch.int32, device="cuda")
        out = torch.empty((B, H * D), dtype=torch.bfloat16, device="cuda")
        ws = torch.empty(qg.qg_decode_attention_workspace_size(B, H, Hkv, D, L),
                         dtype=torch.uint8, device="cuda")
        run = lambda: qg.qg_decode_attention(q, kc, vc, kv_len, out, H, Hkv, D ** -0.5, ws)
    else:
        M, N, K = 1500, 5120, 1280
        blocks = to(qg_synth.q4_0_packed(N, K, 22))
        A = to(qg_synth.gaussian((M, K), 1.0, 23).astype(np.float32)).view(torch.float32)
        C = torch.empty((M, N), dtype=torch.float32, device="cuda")
        ws = torch.empty(qg.qg_gemm_q4_0_workspace_size(M, N, K), dtype=torch.uint8, device="cuda")
        run = lambda: qg.qg_gemm_q4_0(blocks, A, C, ws=ws)
    for _ in range(args.warmup + args.steps):
        run()
    torch.cuda.synchronize()
    print(f"ncu case {args.ncu_case}: {args.warmup} + {args.steps} launches done", flush=True)
    return 0


def run_sweep(args):
    """The Qwen3-1.7B-shaped decode (28 layers, hidden 2048, FFN 6144, vocab
    151936, affine-INT8 g64): a 256-row prefill (batched, and row at a time
    for comparison) at positions 0..255 (batch 1), then decode steps at KV lengths 512,
    1024 and 2048 for batch 1, 2, 4, 8, 16 and 32, each a CUDA-graph replay
    timed with CUDA events. Prints one JSON line (not the bench contract's
    line)."""
    import torch
    import weight_only_quantized_03_b200 as qg
    cfg = dict(qg_synth.QWEN3_1_7B)
    weights = qg_synth.qwen3_weights(cfg, 19)
    model = qg.Qwen3Model(cfg, weights)
    cap = 2049
    stream = torch.cuda.Stream()
    gen = torch.Generator(device="cuda").manual_seed(90)
    out = {"metric": "decode steps/s and tokens/s (Qwen3-1.7B shape, affine-INT8 g64)",
           "data": "synthetic (seeded random packed weights; K/V cache N(0,1) bf16 drawn on device)",
           "points": []}

    def graph_step(st, toks, pos):
        with torch.cuda.stream(stream):
            for _ in range(2):
                model.qg_decode_step(st, toks, pos, stream=stream)
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            model.qg_decode_step(st, toks, pos, stream=stream)
        return g

    # prefill: 256 rows, batched (and row at a time for comparison)
    out["prefill_256_rows"] = prefill_rows(qg, model, cfg, stream)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    for B in (1, 2, 4, 8, 16, 32):
        st = model.new_state(B, cap)
        st["k_cache"].normal_(generator=gen)
        st["v_cache"].normal_(generator=gen)
        toks = torch.from_numpy(qg_synth.tokens(B, cfg["vocab"], 92)).cuda()
        pos = torch.zeros(B, dtype=torch.int32, device="cuda")
        per = {}
        for L in (512, 1024, 2048):
            pos.fill_(L - 1)
            g = graph_step(st, toks, pos)
            n = max(5, args.steps)
            with torch.cuda.stream(stream):
                for _ in range(args.warmup):
                    g.replay()
                e0.record(stream)
                for _ in range(n):
                    g.replay()
                e1.record(stream)
            stream.synchronize()
            us = e0.elapsed_time(e1) / n * 1000.0
            per[str(L)] = {"us_per_step": us, "steps_per_s": 1e6 / us, "tokens_per_s": B * 1e6 / us}
            del g
        out["points"].append({"batch": B, "kv_len": per})
        del st
        torch.cuda.empty_cache()
    print(json.dumps(out), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ncu-case", choices=["step", "lm_head", "gemm", "attn"], default=None,
                    help="launch one kernel only (for an ncu capture); prints no JSON line")
    ap.add_argument("--sweep", action="store_true",
                    help="the Qwen3-1.7B-shaped prefill and batch sweep (its own JSON line)")
    ap.add_argument("--quick", action="store_true",
                    help="the decode step, e2e and LM head only (skip the other configurations)")
    ap.add_argument("--timeline-leg", action="store_true", help=argparse.SUPPRESS)
    ap.add_argument("--no-timeline", action="store_true",
                    help="skip the in-graph timeline leg (roofline then reports the LM head)")
    args = ap.parse_args()
    if args.timeline_leg:
        return run_timeline(args)
    if args.ncu_case:
        return run_ncu_case(args)
    if args.sweep:
        if args.warmup < 3:
            args.warmup = 3
        return run_sweep(args)
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
