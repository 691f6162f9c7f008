"""Seeded synthetic inputs shared by the oracle tests, the GPU tests and the bench.

This module draws random numbers and lays them out in the byte formats the
library consumes. It holds none of the method's arithmetic: it never
quantizes, dequantizes, multiplies or normalises anything. Packed weights are
drawn directly as codes plus per-group constants (the way the synthetic
checkpoint of turbospark-runtime 0.3.0, src/qwen3_asr_metal.rs, test
`packed_linear`, draws every weight byte at random), so the GPU leg of the
bench never needs a quantizer.

Every generator takes an explicit integer seed and uses numpy's PCG64, so the
same seed gives the same bytes on every machine.
"""
from __future__ import annotations

import numpy as np
import torch

GROUP = 64      # affine-INT8 group width (columns per scale/bias pair)
QK4_0 = 32      # Q4_0 block width
Q4_0_BLOCK_BYTES = 18


def _rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(int(seed)))


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Cast float32 values to bf16 bit patterns (torch's round-to-nearest-even cast)."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def gaussian(shape, std: float, seed: int) -> np.ndarray:
    """float32 N(0, std^2) array."""
    return (_rng(seed).standard_normal(size=shape) * std).astype(np.float32)


def gaussian_bf16_bits(shape, std: float, seed: int) -> np.ndarray:
    """bf16 bit patterns of N(0, std^2) draws (activations, KV-cache rows)."""
    return f32_to_bf16_bits(gaussian(shape, std, seed))


def tokens(n: int, vocab: int, seed: int) -> np.ndarray:
    return _rng(seed).integers(0, vocab, size=n, dtype=np.int64).astype(np.int32)


def affine8_packed(N: int, K: int, seed: int, std: float = 0.02):
    """Packed affine-INT8 g64 matrix drawn directly in its storage format.

    Codes are uniform bytes. Each group of 64 columns gets a bf16 scale near
    ``std / 73.9`` (73.9 is the standard deviation of a uniform byte) and a
    bf16 bias near ``-127.5 * scale``, both jittered per group so that a
    wrong group index shows up in a parity test. Returns
    ``(words uint32 [N, K/4], scales uint16 bf16 bits [N, K/64],
    biases uint16 bf16 bits [N, K/64])``.
    """
    assert K % GROUP == 0
    g = _rng(seed)
    q = g.integers(0, 256, size=(N, K), dtype=np.int64).astype(np.uint8)
    s0 = std / 73.9
    G = K // GROUP
    scale = (s0 * (0.75 + 0.5 * g.random(size=(N, G)))).astype(np.float32)
    bias = (-127.5 * scale * (1.0 + 0.1 * g.standard_normal(size=(N, G)))).astype(np.float32)
    words = np.ascontiguousarray(q).view(np.uint32).reshape(N, K // 4)  # little-endian byte order
    return words.copy(), f32_to_bf16_bits(scale), f32_to_bf16_bits(bias)


def affine8_fixture(N: int, K: int, seed: int):
    """The turbospark synthetic-checkpoint pattern: random code bytes from the
    pages' LCG with constant bf16(0.004) scales and bf16(-0.508) biases."""
    assert K % GROUP == 0
    q = lcg_bytes(seed, N * K).reshape(N, K)
    words = np.ascontiguousarray(q).view(np.uint32).reshape(N, K // 4).copy()
    G = K // GROUP
    s = f32_to_bf16_bits(np.full((N, G), 0.004, np.float32))
    b = f32_to_bf16_bits(np.full((N, G), -0.508, np.float32))
    return words, s, b


def q4_0_packed(N: int, K: int, seed: int, std: float = 0.02) -> np.ndarray:
    """Q4_0 matrix drawn directly as blocks: per block an fp16 ``d`` of random
    sign and magnitude near ``2.5 * std / 8``, and 16 random nibble bytes.
    Returns uint8 ``[N, (K/32) * 18]`` (row-major blocks, fp16 little-endian
    first, as a GGUF file stores them)."""
    assert K % QK4_0 == 0
    g = _rng(seed)
    nb = K // QK4_0
    d = (2.5 * std / 8.0) * (0.75 + 0.5 * g.random(size=(N, nb)))
    d = np.where(g.random(size=(N, nb)) < 0.5, -d, d).astype(np.float16)
    out = np.empty((N, nb, Q4_0_BLOCK_BYTES), dtype=np.uint8)
    out[:, :, 0:2] = d.view(np.uint8).reshape(N, nb, 2)
    out[:, :, 2:] = g.integers(0, 256, size=(N, nb, 16), dtype=np.int64).astype(np.uint8)
    return out.reshape(N, nb * Q4_0_BLOCK_BYTES)


def lcg_bytes(seed: int, n: int) -> np.ndarray:
    """Bytes from the 64-bit LCG of the turbospark synthetic checkpoint
    (multiplier 6364136223846793005, increment 1442695040888963407, the byte
    is bits 33..40 of the new state). Vectorised by jumping the LCG ahead."""
    M = 6364136223846793005
    C = 1442695040888963407
    mask = (1 << 64) - 1
    out = np.empty(n, dtype=np.uint8)
    # Advance in blocks of 4096 states: state_{i+j} = A_j * state_i + C_j.
    J = 4096
    A = np.empty(J, dtype=object)
    Cs = np.empty(J, dtype=object)
    a, c = 1, 0
    for j in range(J):
        a, c = (a * M) & mask, (c * M + C) & mask
        A[j], Cs[j] = a, c
    A64 = np.array([int(v) for v in A], dtype=np.uint64)
    C64 = np.array([int(v) for v in Cs], dtype=np.uint64)
    state = np.uint64(seed & mask)
    with np.errstate(over="ignore"):
        for start in range(0, n, J):
            m = min(J, n - start)
            states = A64[:m] * state + C64[:m]
            out[start:start + m] = ((states >> np.uint64(33)) & np.uint64(0xFF)).astype(np.uint8)
            state = states[m - 1]
    return out


# ---------------------------------------------------------------------------
# Model-shaped weight sets
# ---------------------------------------------------------------------------

QWEN3_0_6B = dict(hidden=1024, layers=28, heads=16, kv_heads=8, head_dim=128,
                  ffn=3072, vocab=151936, eps=1e-6, theta=1e6)
QWEN3_1_7B = dict(hidden=2048, layers=28, heads=16, kv_heads=8, head_dim=128,
                  ffn=6144, vocab=151936, eps=1e-6, theta=1e6)
# The code predictor of makima's Qwen3-TTS (CodePredictorConfig defaults:
# hidden 1024, 5 layers, 16 heads without GQA, head_dim 64, FFN 3 x hidden,
# 16 code groups of 2048 codes, eps 1e-6; RoPE base of the main model).
CODE_PREDICTOR = dict(hidden=1024, layers=5, heads=16, kv_heads=16, head_dim=64,
                      ffn=3072, vocab=2048, eps=1e-6, theta=1e6)
CODE_GROUPS = 16
# The synthetic text decoder of the turbospark parity gate.
QWEN3_TINY = dict(hidden=64, layers=2, heads=2, kv_heads=1, head_dim=64,
                  ffn=128, vocab=261, eps=1e-5, theta=1e4)

LINEARS = ("q", "k", "v", "o", "gate", "up", "down")


def linear_shapes(cfg: dict) -> dict:
    h, H, Hk, D, F = cfg["hidden"], cfg["heads"], cfg["kv_heads"], cfg["head_dim"], cfg["ffn"]
    return {"q": (H * D, h), "k": (Hk * D, h), "v": (Hk * D, h), "o": (h, H * D),
            "gate": (F, h), "up": (F, h), "down": (h, F)}


def qwen3_weights(cfg: dict, seed: int, fixture: bool = False, norm_jitter: float = 0.0):
    """Random-init packed weights for a Qwen3-shaped decoder.

    Returns a dict with ``embed`` (tied embedding / LM-head affine8 triple),
    ``final_norm`` (bf16 bits) and ``layers``: a list of dicts holding the
    seven affine8 triples and four bf16 norm-weight vectors. Norm weights are
    1.0 (as in the turbospark synthetic checkpoint) unless ``norm_jitter`` > 0.
    """
    gen = affine8_fixture if fixture else affine8_packed
    shapes = linear_shapes(cfg)
    h, D = cfg["hidden"], cfg["head_dim"]
    sd = seed * 1000

    def norm(n, s):
        v = np.ones(n, np.float32)
        if norm_jitter:
            v = v + norm_jitter * gaussian((n,), 1.0, s)
        return f32_to_bf16_bits(v)

    out = {"embed": gen(cfg["vocab"], h, sd + 1), "final_norm": norm(h, sd + 2), "layers": []}
    for l in range(cfg["layers"]):
        base = sd + 10 + 20 * l
        lw = {name: gen(*shapes[name], base + i) for i, name in enumerate(LINEARS)}
        lw["input_norm"] = norm(h, base + 10)
        lw["post_norm"] = norm(h, base + 11)
        lw["q_norm"] = norm(D, base + 12)
        lw["k_norm"] = norm(D, base + 13)
        out["layers"].append(lw)
    return out


def code_predictor_weights(cfg: dict, groups: int, seed: int, norm_jitter: float = 0.0):
    """Random-init packed weights for a code predictor: the decoder layers
    and final norm of ``qwen3_weights`` (its embedding table unused), plus
    ``input_proj`` [hidden][2 hidden] and ``groups`` code-embedding tables
    and output heads [vocab][hidden] (affine8 triples)."""
    base = qwen3_weights(cfg, seed, norm_jitter=norm_jitter)
    h, V = cfg["hidden"], cfg["vocab"]
    sd = seed * 1000 + 900
    return {"input_proj": affine8_packed(h, 2 * h, sd),
            "code_embed": [affine8_packed(V, h, sd + 1 + g) for g in range(groups)],
            "heads": [affine8_packed(V, h, sd + 101 + g) for g in range(groups)],
            "layers": base["layers"], "final_norm": base["final_norm"]}


# Whisper-large-v3 encoder layer shape (d_model 1280, 20 heads of 64, FFN
# 5120, LayerNorm eps 1e-5; fuel-transformers lazy_quantized_whisper.rs).
WHISPER_LARGE_V3 = dict(d_model=1280, heads=20, ffn=5120, eps=1e-5)


def whisper_layer_weights(cfg: dict, seed: int) -> dict:
    """Random-init weights of one Whisper encoder layer: the six projections
    as Q4_0 blocks (``q4_0_packed``; k_proj has no bias) and float32
    LayerNorm vectors (gamma near 1, beta near 0) and biases N(0, 0.1^2)."""
    d, F = cfg["d_model"], cfg["ffn"]
    shapes = {"q": (d, d), "k": (d, d), "v": (d, d), "o": (d, d), "fc1": (F, d), "fc2": (d, F)}
    w = {n: q4_0_packed(N, K, seed + i) for i, (n, (N, K)) in enumerate(shapes.items())}
    vecs = {"ln1_g": d, "ln1_b": d, "q_b": d, "v_b": d, "o_b": d, "ln2_g": d, "ln2_b": d,
            "fc1_b": F, "fc2_b": d}
    for i, (n, size) in enumerate(vecs.items()):
        v = gaussian((size,), 0.1, seed + 100 + i)
        w[n] = (v + 1.0).astype(np.float32) if n.endswith("_g") else v
    return w
