"""CPU oracle for the weight-only-quantized decode path.

TEST INFRASTRUCTURE ONLY. Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module. It shares no code
with the CUDA library and never imports it; the product path never calls it.

Everything is plain numpy in float64, written from the definitions on the
source pages, one step after another in the order the pages run them. Library
primitives (a dot product, a matmul) stand in for single steps only. Where
the GPU stores a value in bf16, the oracle rounds the float64 value to bf16
(round to nearest even) at the same point; everything else stays float64.

Sources (cited per function):
  [TS] turbospark-runtime 0.3.0, src/qwen3_asr_metal.rs -- resident packed
       affine-INT8 (group 64) Qwen3 text decoder.
  [FT] fuel-transformers 0.19.1, src/models/lazy_quantized_whisper.rs --
       GGUF Q4_0 Whisper (Q4_0 bake and forward).
  [MK] makima commit eabd130 "Add Qwen3-TTS streaming endpoint",
       src/tts/qwen3/model.rs and src/tts/qwen3/config.rs -- unquantized
       candle Qwen3 decoder (RoPE, attention, MLP, layer order, defaults).

Every function is pinned by a ``-m "not gpu"`` test in tests/test_oracle_*.py
against something other than itself (closed forms, a worked example, a
library routine, brute force, invariants). No function here is parity
unpinned.
"""
from __future__ import annotations

import math

import numpy as np

GROUP = 64
QK4_0 = 32
Q4_0_BLOCK_BYTES = 18

# ---------------------------------------------------------------------------
# Number formats
# ---------------------------------------------------------------------------

_BF16_MIN_EXP = -125      # frexp exponent of the smallest normal bf16 (2**-126)
_BF16_SIG_BITS = 8        # significant bits of bf16 (7 stored + 1 implicit)


def _bf16_quantize(v, how):
    """Round float64 values onto the bf16 grid with the integer rounding
    function ``how`` (np.rint = nearest-even, np.floor, np.ceil)."""
    v = np.asarray(v, dtype=np.float64)
    out = v.copy()
    fin = np.isfinite(v) & (v != 0)
    _, e = np.frexp(v[fin])                       # v = m * 2**e, 0.5 <= |m| < 1
    e = np.maximum(e, _BF16_MIN_EXP)              # fixed quantum below the normal range
    r = np.ldexp(how(np.ldexp(v[fin], _BF16_SIG_BITS - e)), e - _BF16_SIG_BITS)
    r = np.where(np.abs(r) >= 2.0 ** 128, np.copysign(np.inf, r), r)
    out[fin] = r
    return out


def round_bf16(v):
    """float64 -> nearest bf16 value (ties to even), returned as float64."""
    return _bf16_quantize(v, np.rint)


def round_bf16_down(v):
    """float64 -> largest bf16 value <= v."""
    return _bf16_quantize(v, np.floor)


def round_bf16_up(v):
    """float64 -> smallest bf16 value >= v."""
    return _bf16_quantize(v, np.ceil)


def bf16_bits_to_f64(bits):
    """bf16 bit patterns (uint16) -> float64 values (exact)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    with np.errstate(invalid="ignore"):
        return b.view(np.float32).astype(np.float64)


def bf16_value_to_bits(v):
    """bf16-representable float64 values -> uint16 bit patterns."""
    f = np.asarray(v, dtype=np.float64).astype(np.float32)
    return (f.view(np.uint32) >> 16).astype(np.uint16)


def f16_bits_to_f64(bits):
    """IEEE binary16 bit patterns -> float64 (exact)."""
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


# ---------------------------------------------------------------------------
# Affine-INT8, group 64  [TS: PackedLinear, load_packed_linear, embed_row_bytes]
# ---------------------------------------------------------------------------

def affine8_quantize(w):
    """Quantize float weights ``w [N, K]`` to the affine-INT8 g64 format.

    The pages only read checkpoints that arrive already packed ([TS]
    ``open`` checks ``quantization_config {bits 8, group_size 64, mode
    affine}``), so the quantizer is this library's reading: per group of 64,
    bias = bf16 rounded down from the group minimum, scale = bf16 rounded up
    from (max - bias) / 255, code = nearest integer of (w - bias) / scale
    clamped to [0, 255]. The directed roundings keep every weight inside
    [bias, bias + 255 * scale], so |w - dequant| <= scale / 2.

    Returns (words uint32 [N, K/4], scales uint16 [N, K/64], biases uint16).
    """
    w = np.asarray(w, dtype=np.float64)
    N, K = w.shape
    assert K % GROUP == 0
    g = w.reshape(N, K // GROUP, GROUP)
    lo = g.min(axis=2)
    hi = g.max(axis=2)
    bias = round_bf16_down(lo)
    scale = round_bf16_up((hi - bias) / 255.0)
    scale = np.where(scale > 0, scale, 2.0 ** -126)
    q = np.rint((g - bias[:, :, None]) / scale[:, :, None])
    q = np.clip(q, 0, 255).astype(np.uint8).reshape(N, K)
    return affine8_pack(q), bf16_value_to_bits(scale), bf16_value_to_bits(bias)


def affine8_pack(q):
    """Pack byte codes ``q [N, K]`` into u32 words ``[N, K/4]``: column
    ``4*j + i`` is byte ``i`` (bits 8i..8i+7) of word ``j`` -- the U32
    ``[rows, cols/4]`` tensor holding ``rows * cols`` bytes of [TS]
    ``load_packed_linear``, read byte-per-column by ``embed_row_bytes``."""
    q = np.asarray(q, dtype=np.uint8)
    N, K = q.shape
    words = np.zeros((N, K // 4), dtype=np.uint64)
    for i in range(4):
        words |= q[:, i::4].astype(np.uint64) << np.uint64(8 * i)
    return words.astype(np.uint32)


def affine8_unpack(words):
    """Inverse of ``affine8_pack``: u32 words ``[N, K/4]`` -> byte codes ``[N, K]``."""
    words = np.asarray(words, dtype=np.uint32).astype(np.uint64)
    N, W = words.shape
    q = np.zeros((N, 4 * W), dtype=np.uint8)
    for i in range(4):
        q[:, i::4] = ((words >> np.uint64(8 * i)) & np.uint64(0xFF)).astype(np.uint8)
    return q


def affine8_dequant_exact(words, scales, biases):
    """Exact dequantized weights in float64: ``w = q * scale + bias`` with
    the group of column c being c // 64 ([TS] ``embed_row_bytes``). The
    product and sum are exact in float64 (8-bit code times 8-bit bf16
    significand, then one add)."""
    q = affine8_unpack(words).astype(np.float64)
    N, K = q.shape
    s = np.repeat(bf16_bits_to_f64(scales), GROUP, axis=1)
    b = np.repeat(bf16_bits_to_f64(biases), GROUP, axis=1)
    assert s.shape == (N, K)
    return q * s + b


def affine8_dequant_f32(words, scales, biases):
    """Dequantized weights as float32 values: the exact value rounded once
    to float32 (what a float32 ``q * s + b`` gives, since ``q * s`` is
    exact in float32)."""
    return affine8_dequant_exact(words, scales, biases).astype(np.float32)


def gemv_affine8(words, scales, biases, x, residual=None):
    """``y[b, r] = sum_c (q[r,c] * s[r, c//64] + beta[r, c//64]) * x[b, c]``
    (+ ``residual[b, r]``). The GEMV of [TS] ``step`` (every packed linear,
    no linear bias), accumulated in float64. ``x`` is ``[B, K]`` float64."""
    w = affine8_dequant_exact(words, scales, biases)
    y = np.asarray(x, dtype=np.float64) @ w.T
    if residual is not None:
        y = y + np.asarray(residual, dtype=np.float64)
    return y


def embed_rows(words, scales, biases, token_ids):
    """Tied-embedding lookup: dequantize one packed row per token ([TS]
    ``embed_row_bytes``; the same table is the LM head). Returns the float32
    residual-stream rows as float64 values."""
    ids = np.asarray(token_ids, dtype=np.int64)
    return affine8_dequant_f32(words[ids], scales[ids], biases[ids]).astype(np.float64)


# ---------------------------------------------------------------------------
# GGUF Q4_0  [FT: quantize_in_out_to_q4_0, q_linear]
# ---------------------------------------------------------------------------

def q4_0_quantize(x):
    """Quantize float32 rows ``x [N, K]`` into Q4_0 blocks as ggml's
    ``BlockQ4_0::from_float`` does (named by [FT]
    ``quantize_in_out_to_q4_0``): per block of 32, ``m`` = the element of
    largest magnitude (first one on ties, sign kept), ``d = m / -8``,
    ``id = 1/d`` (0 when d == 0), code ``n = min(15, trunc(x * id + 8.5))``;
    stored as fp16 ``d`` followed by 16 bytes, byte j holding code j in its
    low nibble and code j+16 in its high nibble. All arithmetic in float32
    as ggml runs it. Returns uint8 ``[N, (K/32) * 18]``."""
    x = np.asarray(x, dtype=np.float32)
    N, K = x.shape
    assert K % QK4_0 == 0
    blk = x.reshape(N, K // QK4_0, QK4_0)
    idx = np.argmax(np.abs(blk), axis=2)                     # first index of max |x|
    m = np.take_along_axis(blk, idx[:, :, None], axis=2)[:, :, 0]
    m = np.where(np.abs(m) > 0, m, np.float32(0.0))   # the running max starts at +0
    d = (m / np.float32(-8.0)).astype(np.float32)
    with np.errstate(divide="ignore"):
        inv = np.where(d != 0, np.float32(1.0) / d, np.float32(0.0)).astype(np.float32)
    v = (blk * inv[:, :, None]).astype(np.float32) + np.float32(8.5)
    n = np.minimum(15, np.trunc(v.astype(np.float32))).astype(np.uint8)
    out = np.empty((N, K // QK4_0, Q4_0_BLOCK_BYTES), dtype=np.uint8)
    out[:, :, 0:2] = d.astype(np.float16).view(np.uint8).reshape(N, K // QK4_0, 2)
    out[:, :, 2:] = n[:, :, :16] | (n[:, :, 16:] << 4)
    return out.reshape(N, (K // QK4_0) * Q4_0_BLOCK_BYTES)


def q4_0_unpack(blocks, K):
    """Q4_0 bytes ``[N, (K/32)*18]`` -> (fp16 ``d`` as float64 ``[N, K/32]``,
    codes ``n`` uint8 ``[N, K]``), codes in column order."""
    b = np.asarray(blocks, dtype=np.uint8)
    N = b.shape[0]
    nb = K // QK4_0
    b = b.reshape(N, nb, Q4_0_BLOCK_BYTES)
    d = f16_bits_to_f64(b[:, :, 0:2].copy().view(np.uint16)[:, :, 0])
    lo = b[:, :, 2:] & 0x0F
    hi = b[:, :, 2:] >> 4
    n = np.concatenate([lo, hi], axis=2).reshape(N, K)
    return d, n


def q4_0_dequant_exact(blocks, K):
    """``w = d * (n - 8)`` (exact in float64 and in float32)."""
    d, n = q4_0_unpack(blocks, K)
    return np.repeat(d, QK4_0, axis=1) * (n.astype(np.float64) - 8.0)


def gemv_q4_0(blocks, x, bias=None):
    """Q4_0 linear of [FT] ``q_linear``: ``y = x @ W^T (+ bias)``, float64
    accumulation. ``x`` is ``[B, K]``."""
    x = np.asarray(x, dtype=np.float64)
    w = q4_0_dequant_exact(blocks, x.shape[1])
    y = x @ w.T
    if bias is not None:
        y = y + np.asarray(bias, dtype=np.float64)[None, :]
    return y


def gemm_q4_0_bf16(blocks, A, bias=None):
    """The M-row Q4_0 matmul of the Whisper encoder ([FT] ``encoder_layer``
    -> ``q_linear``) under this library's tensor-core operand contract: the
    float32 activations and the dequantized weights are each rounded to bf16
    (nearest even) before the product; accumulation is float64."""
    A = round_bf16(np.asarray(A, dtype=np.float64))
    w = round_bf16(q4_0_dequant_exact(blocks, A.shape[1]))
    C = A @ w.T
    if bias is not None:
        C = C + np.asarray(bias, dtype=np.float64)[None, :]
    return C


# ---------------------------------------------------------------------------
# Elementwise pieces  [TS: step; MK: model.rs]
# ---------------------------------------------------------------------------

def rmsnorm(x, w_bits, eps):
    """``y = x / sqrt(mean(x^2) + eps) * w`` over the last axis; ``w`` bf16
    ([TS] ``encode_rms_norm_bf16w`` calls; [MK] ``rms_norm`` layers)."""
    x = np.asarray(x, dtype=np.float64)
    w = bf16_bits_to_f64(w_bits)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * w


def rmsnorm_perhead(x, w_bits, eps, D):
    """Per-head RMSNorm (Qwen3 q_norm / k_norm): the norm of ``rmsnorm``
    applied to every ``D``-wide head slice with one shared ``[D]`` weight
    ([TS] ``encode_rms_norm_bf16w_perhead``; [MK] ``apply_head_norm``)."""
    x = np.asarray(x, dtype=np.float64)
    shp = x.shape
    return rmsnorm(x.reshape(shp[:-1] + (shp[-1] // D, D)), w_bits, eps).reshape(shp)


def rope_inv_freq(theta, rotary_dim):
    """``inv_freq_i = theta^(-2i / rotary_dim)`` for ``i < rotary_dim/2``
    ([MK] ``RotaryEmbedding::new``)."""
    i = np.arange(rotary_dim // 2, dtype=np.float64)
    return theta ** (-2.0 * i / rotary_dim)


def rope_neox(x, pos, theta, D, rotary_dim=None):
    """NeoX (rotate-half) RoPE on each ``D``-wide head of ``x [..., heads*D]``
    at integer position ``pos`` ([MK] ``RotaryEmbedding::apply`` /
    ``rotate_half``; [TS] ``encode_rope_neox_subdim`` with rotary_dim =
    head_dim). With angle ``a_i = pos * inv_freq_i`` and half = rotary_dim/2:
    ``out_i = x_i cos a_i - x_{i+half} sin a_i`` and
    ``out_{i+half} = x_{i+half} cos a_i + x_i sin a_i``; dims at or beyond
    ``rotary_dim`` pass through."""
    rd = D if rotary_dim is None else rotary_dim
    x = np.asarray(x, dtype=np.float64)
    shp = x.shape
    h = x.reshape(shp[:-1] + (shp[-1] // D, D)).copy()
    half = rd // 2
    a = float(pos) * rope_inv_freq(theta, rd)
    c, s = np.cos(a), np.sin(a)
    x1 = h[..., :half].copy()
    x2 = h[..., half:rd].copy()
    h[..., :half] = x1 * c - x2 * s
    h[..., half:rd] = x2 * c + x1 * s
    return h.reshape(shp)


def silu_mul(gate, up):
    """``silu(gate) * up`` with ``silu(z) = z / (1 + exp(-z))`` ([TS]
    ``encode_silu_mul``; [MK] ``Qwen3Mlp::forward``)."""
    g = np.asarray(gate, dtype=np.float64)
    return g / (1.0 + np.exp(-g)) * np.asarray(up, dtype=np.float64)


def decode_attention(q, k_cache, v_cache, kv_len, H, Hkv, D, scale=None):
    """Decode attention of one query row per sequence over the first
    ``kv_len`` cached rows ([TS] ``encode_attention_decode`` with
    ``kv_start = 0``; [MK] ``Qwen3Attention::forward``). Query head h reads
    KV head ``h // (H / Hkv)`` ([MK] ``repeat_kv``); scores are
    ``q . k_t * scale`` with ``scale = 1/sqrt(D)``; softmax over all
    ``kv_len`` scores in float64 (no splitting).

    q ``[H*D]``; k_cache, v_cache ``[Hkv, >= kv_len, D]`` float64 values.
    Returns ``[H*D]``.
    """
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    q = np.asarray(q, dtype=np.float64).reshape(H, D)
    g = H // Hkv
    out = np.zeros((H, D))
    for h in range(H):
        kh = h // g
        K_ = k_cache[kh, :kv_len, :]
        V_ = v_cache[kh, :kv_len, :]
        s = (K_ @ q[h]) * scale
        p = np.exp(s - s.max())
        p = p / p.sum()
        out[h] = p @ V_
    return out.reshape(H * D)


def argmax_first(logits):
    """Index of the first strict maximum, NaNs skipped (fold from -inf,
    replace only on ``>``) -- [TS] ``argmax``. 0 when nothing beats -inf."""
    best_i, best_v = 0, -math.inf
    for i, v in enumerate(np.asarray(logits, dtype=np.float64).tolist()):
        if v > best_v:
            best_i, best_v = i, v
    return best_i


def token_logprob(logits, token):
    """The log-probability of ``token`` under the softmax of ``logits``
    ([TS] ``compute_selected_logprob`` of the greedy token, whose body the
    page does not print: read as the log-softmax), float64 with the maximum
    subtracted: x[t] - (m + log sum exp(x - m)). NaN for a NaN logit or a
    token outside the row."""
    x = np.asarray(logits, dtype=np.float64)
    if not 0 <= int(token) < x.shape[0] or np.isnan(x).any():
        return math.nan
    m = x.max()
    return float(x[int(token)] - (m + math.log(np.exp(x - m).sum())))


def apply_repetition_penalty(logits, past, penalty):
    """[MK] ``apply_repetition_penalty``: for every past token in order (each
    occurrence counts; tokens outside the vocabulary are skipped), a negative
    score is multiplied by the penalty and any other divided by it, in
    float32 as on the page. Returns a new float32 array."""
    s = np.array(logits, dtype=np.float32)
    p = np.float32(penalty)
    for t in past:
        t = int(t)
        if 0 <= t < s.shape[0]:
            s[t] = s[t] * p if s[t] < 0 else s[t] / p
    return s


def sample_token(logits, past, penalty, temperature, top_k, r):
    """[MK] ``sample_token`` in float32, step by step as on the page:
    repetition penalty; greedy when top_k == 0 or temperature == 0 (the
    first strict maximum, ``argmax_first``: this library's greedy rule);
    otherwise divide by the temperature, sort descending (stable: equal
    values by index), keep the first k = min(top_k, V), exp(t - t_0) summed
    in order, and return the first index whose running sum of probabilities
    reaches ``r`` (the first of the k if none does). NaN scores are left out
    of the sort (the page's comparison leaves their place unspecified)."""
    s = apply_repetition_penalty(logits, past, penalty) if penalty != 1.0 else \
        np.array(logits, dtype=np.float32)
    if top_k == 0 or temperature == 0.0:
        return argmax_first(s)
    t = s / np.float32(temperature)
    order = [i for i in np.argsort(-t, kind="stable") if not np.isnan(t[i])]
    top = order[:min(top_k, len(t))]
    if not top:
        return 0
    t0 = t[top[0]]
    total = np.float32(0.0)
    for i in top:
        total = np.float32(total + np.exp(np.float32(t[i] - t0)))
    cum = np.float32(0.0)
    for i in top:
        cum = np.float32(cum + np.float32(np.exp(np.float32(t[i] - t0)) / total))
        if cum >= np.float32(r):
            return int(i)
    return int(top[0])


# ---------------------------------------------------------------------------
# The decode step  [TS: step]
# ---------------------------------------------------------------------------

def decode_layer(cfg, lw, x, k_cache_l, v_cache_l, pos):
    """One decoder layer of [TS] ``step`` on the residual stream ``x``
    (``[hidden]``, float64): input norm -> q, k, v GEMVs -> per-head q/k norm
    -> NeoX RoPE on q and on k -> K/V written at cache row ``pos`` ->
    attention over rows ``[0, pos]`` -> o_proj -> residual add ->
    post-attention norm -> gate, up -> SiLU-mul -> down -> residual add.

    Precision points (where the GPU stores bf16, rounded here as well): norm
    outputs feeding a GEMV, K and V written to the cache, the attention
    output and the SiLU-mul output. The residual stream and q/k/v and
    gate/up outputs stay float64 (float32 on the GPU).

    ``k_cache_l``/``v_cache_l`` are ``[Hkv, cap, D]`` float64 arrays of bf16
    values; row ``pos`` is overwritten. Returns the new residual stream."""
    H, Hkv, D = cfg["heads"], cfg["kv_heads"], cfg["head_dim"]
    eps, theta = cfg["eps"], cfg["theta"]
    xn = round_bf16(rmsnorm(x, lw["input_norm"], eps))
    q = gemv_affine8(*lw["q"], xn[None])[0]
    k = gemv_affine8(*lw["k"], xn[None])[0]
    v = gemv_affine8(*lw["v"], xn[None])[0]
    q = rope_neox(rmsnorm_perhead(q, lw["q_norm"], eps, D), pos, theta, D)
    k = rope_neox(rmsnorm_perhead(k, lw["k_norm"], eps, D), pos, theta, D)
    k_cache_l[:, pos, :] = round_bf16(k).reshape(Hkv, D)
    v_cache_l[:, pos, :] = round_bf16(v).reshape(Hkv, D)
    att = round_bf16(decode_attention(q, k_cache_l, v_cache_l, pos + 1, H, Hkv, D))
    x = x + gemv_affine8(*lw["o"], att[None])[0]
    xn = round_bf16(rmsnorm(x, lw["post_norm"], eps))
    gate = gemv_affine8(*lw["gate"], xn[None])[0]
    up = gemv_affine8(*lw["up"], xn[None])[0]
    hmid = round_bf16(silu_mul(gate, up))
    return x + gemv_affine8(*lw["down"], hmid[None])[0]


def bf16_alternative(v, rel):
    """The other bf16 rounding of each value that lies within ``rel * |v|`` of
    a bf16 rounding midpoint, NaN elsewhere.

    A value computed in lower precision (float32 on the GPU) can land on
    either side of such a midpoint, so both bf16 neighbours are correct
    results there; this is the one ``round_bf16`` does not pick."""
    v = np.asarray(v, dtype=np.float64)
    r = round_bf16(v)
    lo, hi = round_bf16_down(v), round_bf16_up(v)
    near = (lo != hi) & (np.abs(v - (lo + hi) / 2.0) <= rel * np.abs(v))
    return np.where(near, np.where(r == lo, hi, lo), np.nan)


def bf16_rounding_ok(v, r, rel=2.0 ** -16, abs_tol=0.0):
    """Whether each ``r`` is the bf16 rounding (to nearest even) of some
    value within ``eps = rel * |v| + abs_tol`` of the float64 value ``v``
    (``abs_tol`` a scalar or an array shaped like ``v``).

    This is the set of results that an implementation computing ``v`` with an
    error of at most ``eps`` (float32 arithmetic, another summation order)
    can store. ``round_bf16`` is monotonic, so the set is every bf16 value
    from ``round_bf16(v - eps)`` to ``round_bf16(v + eps)``. Away from a
    rounding midpoint and for ``eps`` below half a bf16 step, that is
    ``round_bf16(v)`` alone. NaN matches NaN."""
    v = np.asarray(v, dtype=np.float64)
    r = np.asarray(r, dtype=np.float64)
    eps = rel * np.abs(v) + abs_tol
    ok = (r >= round_bf16(v - eps)) & (r <= round_bf16(v + eps))
    return ok | (np.isnan(v) & np.isnan(r))


# ---------------------------------------------------------------------------
# float32 error bounds of the short op chains between a GEMV output and the
# next bf16 rounding point. They decide which bf16 values the teacher-forced
# check accepts at a rounding point: every value that rounds from within the
# bound of the exact result. Standard forward error analysis with the unit
# roundoff u = 2^-24 of float32 (round to nearest): a chain of n roundings
# has relative error at most gamma_n = n u / (1 - n u); a sum of n terms
# evaluated along a tree of depth n is within gamma_n * sum|terms| of exact.
# The depths below bound those of any summation order this library's kernels
# use (the kernel sources state theirs); expf is taken to be within 2 ulp
# (4u relative), sqrtf and division correctly rounded.
# ---------------------------------------------------------------------------

U32 = 2.0 ** -24
EXPF_REL = 4.0 * U32


def gamma(n):
    """Relative error bound of a chain of n float32 roundings."""
    return n * U32 / (1.0 - n * U32)


def sumsq_depth(n):
    """Longest chain of roundings in the float32 sum of squares of an
    n-vector (a norm's statistic): n/32 + 32 covers per-thread partial sums
    over a strided slice, a warp reduction and a sum over warps."""
    return n // 32 + 32


def rmsnorm_rel_bound(n):
    """Relative error bound of each output of an RMSNorm of an exact float32
    n-vector computed in float32: the sum of squares (all terms positive, so
    relative ``gamma(sumsq_depth(n))``), the division by n and the add of
    eps (2), the square root (halves the relative error, +1), the reciprocal
    (+1), then x * inv * w (+2)."""
    return 1.01 * (0.5 * gamma(sumsq_depth(n) + 3) + gamma(4))


def norm_rope_bound(x, w_bits, eps, pos, theta, D):
    """(value, bound) of NeoX RoPE applied to the per-head RMSNorm of an
    exact float32 vector ``x [heads*D]``: the value in float64 and, per
    element, the float32 error bound. Each rotated element is a*c - b*s (or
    b*c + a*s) of two normed elements a, b (relative error
    ``rmsnorm_rel_bound(D)`` each) and the float32 cos/sin of the angle
    (computed in double and rounded once: relative u); the two products and
    the difference add 3 roundings: bound (rho + 3u) (|a c| + |b s|)."""
    n = rmsnorm_perhead(x, w_bits, eps, D)
    v = rope_neox(n, pos, theta, D)
    hn = np.abs(n).reshape(-1, D)
    half = D // 2
    a = pos * rope_inv_freq(theta, D)
    c, sn = np.abs(np.cos(a)), np.abs(np.sin(a))
    mag = np.empty_like(hn)
    mag[:, :half] = hn[:, :half] * c + hn[:, half:] * sn
    mag[:, half:] = hn[:, half:] * c + hn[:, :half] * sn
    rho = rmsnorm_rel_bound(D) + gamma(4)
    return v, 1.01 * rho * mag.reshape(v.shape)


def attention_depths(L, D):
    """(dot, rescale, accumulate) depths of the decode attention kernels: a
    score is a float32 dot of D products (per-lane partial sums over D/32 to
    D/8 columns and a shuffle tree: D/8 + 8); along any cached row's path the
    running softmax state is rescaled by a computed exp at most L/32 + 16
    times (once per batch of rows, then the merges of warps, CTAs and
    splits); the weighted sums of V and of the weights take at most
    L/4 + 96 roundings."""
    return D // 8 + 8, L // 32 + 16, L // 4 + 96


def attention_bound(qp, dqp, k_cache, v_cache, kv_len, H, Hkv, D, q_round=0.0, p_round=0.0):
    """(value, bound) of ``decode_attention`` computed in float32 from a
    query ``qp [H*D]`` known within ``dqp`` (per element) and exact bf16
    cache rows.

    Score t: s_t = scale * sum_d q_d k_td with scale = 1/sqrt(D) as a float32
    (2 roundings) times q (1): its error is within
    scale * (sum_d dq_d |k_td| + (3u + gamma(dot)) sum_d |q_d k_td|).
    Softmax: a perturbation e_t of the log-weight of row t moves the output
    by sum_t p_t (e^{e_t} - 1) (v_t - o) / sum_t p_t e^{e_t}, at most
    e^{2 max e} sum_t p_t |e_t| |v_t - o|. The log-weight of row t is off by
    its score's error, the rounding of s_t - m (u |s_t - m|), its exp (4u)
    and each computed rescale on its path (4u, plus u |m_old - m_new|,
    which summed along the path is at most the score range). The weighted
    sums add gamma(accumulate) (sum_t p_t |v_t| + |o|) and the final division
    u |o|. A kernel that rounds the query to bf16 before the scores
    (``q_round`` = 2^-8, the bf16 unit roundoff) widens ``dqp`` by
    q_round |q|; one that rounds the weights p_t to bf16 for the weighted
    sum and its denominator (``p_round`` = 2^-8) reweights each row by at
    most that much: log(1 + p_round) more on every log-weight."""
    q = np.asarray(qp, dtype=np.float64).reshape(H, D)
    dq = np.asarray(dqp, dtype=np.float64).reshape(H, D) + q_round * np.abs(q)
    g = H // Hkv
    scale = 1.0 / math.sqrt(D)
    n_dot, n_res, n_acc = attention_depths(kv_len, D)
    out = np.zeros((H, D))
    err = np.zeros((H, D))
    for h in range(H):
        K_ = k_cache[h // g, :kv_len, :]
        V_ = v_cache[h // g, :kv_len, :]
        s = (K_ @ q[h]) * scale
        ds = scale * (np.abs(K_) @ dq[h] + (3 * U32 + gamma(n_dot)) * (np.abs(K_) @ np.abs(q[h])))
        m = s.max()
        p = np.exp(s - m)
        p = p / p.sum()
        o = p @ V_
        rng = m - s.min()
        e = ds + U32 * (m - s) + EXPF_REL * (n_res + 2) + U32 * rng + math.log1p(p_round)
        out[h] = o
        err[h] = (np.exp(2 * e.max()) * (p * e) @ np.abs(V_ - o[None, :])
                  + gamma(n_acc) * (p @ np.abs(V_) + np.abs(o)) + U32 * np.abs(o))
    return out.reshape(H * D), 1.01 * err.reshape(H * D)


def silu_mul_rel_bound():
    """Relative error bound of silu(z) * up from exact float32 z and up:
    expf (4u) on 1 + e^{-z} gives at most 4u relative there, the add, the
    division and the product one rounding each."""
    return 1.01 * (EXPF_REL + gamma(3))


LAYER_FP32_POINTS = ("q_proj", "k_proj", "v_proj", "x_attn", "gate", "up")
LAYER_BF16_POINTS = ("xn", "k", "v", "att", "xn2", "h")


def decode_layer_forced(cfg, lw, x, k_cache_l, v_cache_l, pos, forced, details=None,
                        q_round=0.0, p_round=0.0):
    """``decode_layer`` checked op by op against another implementation's
    values of one layer (teacher-forced).

    ``forced`` holds that implementation's values: its float32 GEMV outputs
    ``q_proj`` [H*D], ``k_proj``, ``v_proj`` [Hkv*D] (before the per-head
    norm), ``x_attn`` (the residual stream after o_proj and its residual
    add) [hidden], ``gate``, ``up`` [ffn]; and its bf16 values at the
    layer's rounding points ``xn`` (input norm) [hidden], ``k`` and ``v``
    (the cache rows written at ``pos``) [Hkv*D], ``att`` (attention output)
    [H*D], ``xn2`` (post-attention norm) [hidden], ``h`` (SiLU-mul) [ffn].

    Every step is computed in float64 from the forced values before it, so
    each comparison covers one op chain:
      * the GEMV outputs are returned as references (``refs``), to be held
        to the float32-accumulation tolerance by the caller: q/k/v_proj =
        W xn, x_attn = x + W_o att, gate/up = W xn2, and ``y`` = x_attn +
        W_down h (the layer's output);
      * each rounding point is checked to be a correct bf16 rounding of the
        float64 value of its op chain within that chain's float32 error
        bound (``bf16_rounding_ok`` with the bounds above): xn from x, k from
        k_proj (norm and RoPE), v from v_proj (exact), att from q_proj and
        the cache (norm, RoPE, attention), xn2 from x_attn, h from gate and
        up.
    ``q_round`` and ``p_round`` pass to ``attention_bound`` for a kernel
    that rounds the query or the softmax weights to bf16 (the multi-row
    attention of a batched prefill does both).
    Returns ``(refs, bad)``: ``bad`` maps each rounding point to the indices
    whose forced value is not a correct rounding (with ``details``, a dict,
    filled per point with their values, the forced values and the bounds).
    Rows ``pos`` of the caches receive the forced K and V rows."""
    H, Hkv, D, hid = cfg["heads"], cfg["kv_heads"], cfg["head_dim"], cfg["hidden"]
    eps, theta = cfg["eps"], cfg["theta"]
    names = set(LAYER_FP32_POINTS) | set(LAYER_BF16_POINTS)
    if set(forced) != names:  # a misnamed or missing point would go unchecked
        raise KeyError("decode_layer_forced: points must be exactly "
                       f"{sorted(names)}, got {sorted(forced)}")
    f = {k: np.asarray(v, dtype=np.float64).ravel() for k, v in forced.items()}
    bad = {}

    def check(name, val, bound):
        bad[name] = np.flatnonzero(~bf16_rounding_ok(val, f[name], 0.0, bound))
        if details is not None and bad[name].size:
            i = bad[name]
            b = np.broadcast_to(bound, val.shape)[i]
            details[name] = {"index": i, "value": val[i], "forced": f[name][i], "bound": b}

    x = np.asarray(x, dtype=np.float64)
    v = rmsnorm(x, lw["input_norm"], eps)
    check("xn", v, rmsnorm_rel_bound(hid) * np.abs(v))
    refs = {"q_proj": gemv_affine8(*lw["q"], f["xn"][None])[0],
            "k_proj": gemv_affine8(*lw["k"], f["xn"][None])[0],
            "v_proj": gemv_affine8(*lw["v"], f["xn"][None])[0]}
    kr, kb = norm_rope_bound(f["k_proj"], lw["k_norm"], eps, pos, theta, D)
    check("k", kr, kb)
    check("v", f["v_proj"], 0.0)
    k_cache_l[:, pos, :] = f["k"].reshape(Hkv, D)
    v_cache_l[:, pos, :] = f["v"].reshape(Hkv, D)
    qr, qb = norm_rope_bound(f["q_proj"], lw["q_norm"], eps, pos, theta, D)
    att, ab = attention_bound(qr, qb, k_cache_l, v_cache_l, pos + 1, H, Hkv, D, q_round, p_round)
    check("att", att, ab)
    refs["x_attn"] = x + gemv_affine8(*lw["o"], f["att"][None])[0]
    v2 = rmsnorm(f["x_attn"], lw["post_norm"], eps)
    check("xn2", v2, rmsnorm_rel_bound(hid) * np.abs(v2))
    refs["gate"] = gemv_affine8(*lw["gate"], f["xn2"][None])[0]
    refs["up"] = gemv_affine8(*lw["up"], f["xn2"][None])[0]
    hm = silu_mul(f["gate"], f["up"])
    check("h", hm, silu_mul_rel_bound() * np.abs(hm))
    refs["y"] = f["x_attn"] + gemv_affine8(*lw["down"], f["h"][None])[0]
    return refs, bad


def lm_head(cfg, weights, x):
    """Final RMSNorm (bf16 output) and the tied LM head of [TS] ``step``."""
    ew, es, eb = weights["embed"]
    xn = round_bf16(rmsnorm(x, weights["final_norm"], cfg["eps"]))
    return gemv_affine8(ew, es, eb, xn[None])[0]


def lm_head_tie_bound(cfg, weights, x, rel=None):
    """``lm_head`` of an exact float32 residual ``x`` plus the bound on the
    effect of bf16 rounding ties of the final norm: an element within the
    norm's float32 error bound (``rmsnorm_rel_bound``) of a rounding
    midpoint may round either way, and the head is linear in the normed
    vector, so such a tie at element j moves logit r by
    ``|w[r][j]| * |alt_j - round_j|`` exactly. Returns ``(logits, extra)``."""
    if rel is None:
        rel = rmsnorm_rel_bound(cfg["hidden"])
    ew, es, eb = weights["embed"]
    v = rmsnorm(x, weights["final_norm"], cfg["eps"])
    xn = round_bf16(v)
    logits = gemv_affine8(ew, es, eb, xn[None])[0]
    alt = bf16_alternative(v, rel)
    extra = np.zeros_like(logits)
    codes = affine8_unpack(ew)
    sc, bi = bf16_bits_to_f64(es), bf16_bits_to_f64(eb)
    for j in np.flatnonzero(~np.isnan(alt)):
        col = codes[:, j] * sc[:, j // GROUP] + bi[:, j // GROUP]
        extra += np.abs(col) * abs(alt[j] - xn[j])
    return logits, extra


def decode_step(cfg, weights, k_cache, v_cache, token, pos):
    """One token of one sequence through every layer ([TS] ``step``): the
    dequantized embedding row of [TS] ``embed_row_bytes``, ``decode_layer``
    for each layer, then ``lm_head``. ``k_cache``/``v_cache`` are float64
    ``[layers, Hkv, cap, D]``; row ``pos`` of every layer is overwritten.
    Returns the logits ``[vocab]`` (float64)."""
    ew, es, eb = weights["embed"]
    x = embed_rows(ew, es, eb, [token])[0]
    for l, lw in enumerate(weights["layers"]):
        x = decode_layer(cfg, lw, x, k_cache[l], v_cache[l], pos)
    return lm_head(cfg, weights, x)


def new_kv_cache(cfg, cap):
    return (np.zeros((cfg["layers"], cfg["kv_heads"], cap, cfg["head_dim"])),
            np.zeros((cfg["layers"], cfg["kv_heads"], cap, cfg["head_dim"])))


# ---------------------------------------------------------------------------
# The Whisper encoder layer  [FT: encoder_layer, multi_head_attn,
# layer_norm_affine, q_linear]
# ---------------------------------------------------------------------------

def layer_norm(x, gamma, beta, eps):
    """LayerNorm over the last axis with an affine f32 gamma and beta ([FT]
    ``layer_norm_affine``: ``layer_norm_last_dim`` then ``* g + b``): the
    mean and the biased variance of the row, ``(x - mean) / sqrt(var + eps)
    * gamma + beta``."""
    x = np.asarray(x, dtype=np.float64)
    mu = x.mean(axis=-1, keepdims=True)
    var = np.mean((x - mu) ** 2, axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps) * np.asarray(gamma, np.float64) + np.asarray(beta, np.float64)


def gelu_tanh(x):
    """The tanh form of GELU named by [FT] (``gelu_tanh``):
    ``0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3)))``."""
    x = np.asarray(x, dtype=np.float64)
    return 0.5 * x * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (x + 0.044715 * x ** 3)))


def mha_rows(q, k, v, n_heads, causal=False, kv_heads=None, abs_weighted=False):
    """Multi-head softmax attention of [FT] ``multi_head_attn`` for all rows
    at once: q ``[T, H*D]``, k and v ``[S, Hkv*D]``, per head
    ``softmax(q_h k_h^T / sqrt(D)) v_h`` over all S rows, or with
    ``causal`` over rows ``j <= i`` (the mask of [FT] and of [MK]
    ``causal_mask``). With ``kv_heads`` < heads, query head h reads KV head
    ``h // (H / Hkv)`` ([MK] ``repeat_kv``). float64; returns ``[T, H*D]``,
    and with ``abs_weighted`` also ``sum_s p_s |v_s|`` per output (what a
    relative change of each weight moves the output by, at most)."""
    q = np.asarray(q, np.float64)
    k = np.asarray(k, np.float64)
    v = np.asarray(v, np.float64)
    T = q.shape[0]
    S = k.shape[0]
    Hkv = n_heads if kv_heads is None else kv_heads
    D = q.shape[1] // n_heads
    g = n_heads // Hkv
    out = np.zeros((T, n_heads * D))
    aw = np.zeros((T, n_heads * D))
    for h in range(n_heads):
        kh = h // g
        s = q[:, h * D:(h + 1) * D] @ k[:, kh * D:(kh + 1) * D].T / math.sqrt(D)
        if causal:
            s = s + np.triu(np.full((T, S), -np.inf), k=1 + S - T)
        p = np.exp(s - s.max(axis=1, keepdims=True))
        p = p / p.sum(axis=1, keepdims=True)
        out[:, h * D:(h + 1) * D] = p @ v[:, kh * D:(kh + 1) * D]
        if abs_weighted:
            aw[:, h * D:(h + 1) * D] = p @ np.abs(v[:, kh * D:(kh + 1) * D])
    return (out, aw) if abs_weighted else out


def whisper_encoder_layer(x, lw, n_heads, eps=1e-5, details=None):
    """One Whisper encoder layer ([FT] ``encoder_layer``), pre-LayerNorm:
    ``x + out(attn(LN1(x)))`` then ``+ fc2(gelu_tanh(fc1(LN2(.))))``, with
    ``q_linear`` as the Q4_0 matmul under this library's tensor-core operand
    contract (``gemm_q4_0_bf16``: operands rounded to bf16). k_proj has no
    bias; q, v, out, fc1 and fc2 have f32 biases.

    Precision points (where the GPU stores bf16; rounded here as well): the
    LayerNorm outputs, q, k and v (the attention operands), the attention
    output (the out projection's input) and the GELU output (fc2's input).
    The residual stream stays float64 (float32 on the GPU).

    ``x`` ``[T, d]``; ``lw`` holds ``ln1_g, ln1_b, q, q_b, k, v, v_b, o, o_b,
    ln2_g, ln2_b, fc1, fc1_b, fc2, fc2_b`` (Q4_0 blocks and f32 vectors).
    With ``details`` (a dict) the intermediate values are stored in it."""
    x = np.asarray(x, np.float64)
    xl = round_bf16(layer_norm(x, lw["ln1_g"], lw["ln1_b"], eps))
    q = round_bf16(gemm_q4_0_bf16(lw["q"], xl, lw["q_b"]))
    k = round_bf16(gemm_q4_0_bf16(lw["k"], xl))
    v = round_bf16(gemm_q4_0_bf16(lw["v"], xl, lw["v_b"]))
    ctx = round_bf16(mha_rows(q, k, v, n_heads))
    xa = x + gemm_q4_0_bf16(lw["o"], ctx, lw["o_b"])
    xl2 = round_bf16(layer_norm(xa, lw["ln2_g"], lw["ln2_b"], eps))
    mid = round_bf16(gelu_tanh(gemm_q4_0_bf16(lw["fc1"], xl2, lw["fc1_b"])))
    y = xa + gemm_q4_0_bf16(lw["fc2"], mid, lw["fc2_b"])
    if details is not None:
        details.update(xl=xl, q=q, k=k, v=v, ctx=ctx, xa=xa, xl2=xl2, mid=mid, y=y)
    return y


# ---------------------------------------------------------------------------
# The code predictor  [MK: src/tts/qwen3/code_predictor.rs]
# ---------------------------------------------------------------------------

def code_predict_group(cfg, w, lm_hidden, prev_code, g):
    """Logits of code group ``g`` (>= 1) of [MK] ``CodePredictor::predict``
    given the previous group's code: embed ``prev_code`` with table g-1,
    concatenate it after ``lm_hidden``, project with ``input_proj``, run every
    layer with a fresh KV cache (so each attends to its own row at position
    0), final RMSNorm, head g. The concatenation feeds a GEMV and is rounded
    to bf16 like every GEMV input here (reading: the page runs the whole
    predictor in one dtype; this library's activations into a GEMV are
    bf16)."""
    emb = embed_rows(*w["code_embed"][g - 1], [prev_code])[0]
    comb = round_bf16(np.concatenate([np.asarray(lm_hidden, dtype=np.float64), emb]))
    x = gemv_affine8(*w["input_proj"], comb[None])[0]
    Hkv, D = cfg["kv_heads"], cfg["head_dim"]
    for lw in w["layers"]:
        kc, vc = np.zeros((Hkv, 1, D)), np.zeros((Hkv, 1, D))
        x = decode_layer(cfg, lw, x, kc, vc, 0)
    xn = round_bf16(rmsnorm(x, w["final_norm"], cfg["eps"]))
    return gemv_affine8(*w["heads"][g], xn[None])[0]


def code_predict(cfg, w, lm_hidden, code0):
    """[MK] ``CodePredictor::predict`` for one sequence: codes of groups
    1..groups-1 chosen greedily one after another (``argmax_first``), each
    from the previous one. Returns ``(codes, logits)``: the ``groups`` codes
    starting with ``code0`` and the logits of groups 1.. (a list)."""
    codes, logits = [int(code0)], []
    for g in range(1, len(w["heads"])):
        lg = code_predict_group(cfg, w, lm_hidden, codes[-1], g)
        logits.append(lg)
        codes.append(argmax_first(lg))
    return codes, logits


def prefix_forward(cfg, weights, token_ids):
    """Whole-prefix forward with a causal mask ([MK] ``Qwen3Model::forward``
    with the mask of ``causal_mask`` and ``Qwen3Attention::forward``): all
    rows at once, no cache, the same precision points as ``decode_step``.
    Returns logits ``[T, vocab]``. Used to pin ``decode_step``: the
    incremental cache must give the same last-row logits."""
    H, Hkv, D = cfg["heads"], cfg["kv_heads"], cfg["head_dim"]
    eps, theta = cfg["eps"], cfg["theta"]
    T = len(token_ids)
    ew, es, eb = weights["embed"]
    x = embed_rows(ew, es, eb, token_ids)
    mask = np.triu(np.full((T, T), -np.inf), k=1)
    g = H // Hkv
    for lw in weights["layers"]:
        xn = round_bf16(rmsnorm(x, lw["input_norm"], eps))
        q = gemv_affine8(*lw["q"], xn)
        k = gemv_affine8(*lw["k"], xn)
        v = gemv_affine8(*lw["v"], xn)
        q = np.stack([rope_neox(rmsnorm_perhead(q[t], lw["q_norm"], eps, D), t, theta, D) for t in range(T)])
        k = np.stack([rope_neox(rmsnorm_perhead(k[t], lw["k_norm"], eps, D), t, theta, D) for t in range(T)])
        k = round_bf16(k).reshape(T, Hkv, D)
        v = round_bf16(v).reshape(T, Hkv, D)
        q = q.reshape(T, H, D)
        att = np.zeros((T, H, D))
        for h in range(H):
            s = q[:, h, :] @ k[:, h // g, :].T / math.sqrt(D) + mask
            p = np.exp(s - s.max(axis=1, keepdims=True))
            p = p / p.sum(axis=1, keepdims=True)
            att[:, h, :] = p @ v[:, h // g, :]
        att = round_bf16(att.reshape(T, H * D))
        x = x + gemv_affine8(*lw["o"], att)
        xn = round_bf16(rmsnorm(x, lw["post_norm"], eps))
        hmid = round_bf16(silu_mul(gemv_affine8(*lw["gate"], xn), gemv_affine8(*lw["up"], xn)))
        x = x + gemv_affine8(*lw["down"], hmid)
    xn = round_bf16(rmsnorm(x, weights["final_norm"], eps))
    return gemv_affine8(ew, es, eb, xn)
