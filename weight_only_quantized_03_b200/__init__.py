"""Python binding of libqg, weight-only-quantized decode kernels for B200.

Argument marshalling only: every function here forwards torch tensors' device
pointers, shapes and the current CUDA stream to the C ABI of the same name
(include/qg.h) and raises QGError when it returns a non-zero status. No
computation happens in Python and there is no fallback: importing this module
fails if libqg.so is missing.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# QG_LIBRARY may name the diagnostic build next to it (libqg_timeline.so)
_NAME = os.environ.get("QG_LIBRARY", "libqg.so")
if _NAME not in ("libqg.so", "libqg_timeline.so"):
    raise ImportError(f"QG_LIBRARY={_NAME!r}: expected libqg.so or libqg_timeline.so")
LIB_PATH = os.path.join(_HERE, _NAME)

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python weight_only_quantized_03_b200/build.py`"
    )
lib = ctypes.CDLL(LIB_PATH)

QG_OK = 0
QG_ERR_INVALID_ARGUMENT = 1
QG_ERR_UNSUPPORTED_SHAPE = 2
QG_ERR_MISALIGNED = 3
QG_ERR_WORKSPACE_TOO_SMALL = 4
QG_ERR_CUDA = 5
QG_ERR_TIMEOUT = 6
QG_F32 = 0
QG_BF16 = 1

_vp = ctypes.c_void_p
_i = ctypes.c_int
_f = ctypes.c_float
_d = ctypes.c_double
_sz = ctypes.c_size_t


class QGError(RuntimeError):
    def __init__(self, name, status, msg):
        super().__init__(f"{name} returned {status}: {msg}")
        self.status = status


class qg_affine8_matrix(ctypes.Structure):
    _fields_ = [("w", _vp), ("scales", _vp), ("biases", _vp)]


class qg_qwen3_layer(ctypes.Structure):
    _fields_ = [("input_norm", _vp), ("post_norm", _vp), ("q_norm", _vp), ("k_norm", _vp)] + [
        (n, qg_affine8_matrix) for n in ("q", "k", "v", "o", "gate", "up", "down")]


class qg_qwen3_config(ctypes.Structure):
    _fields_ = [("hidden", _i), ("layers", _i), ("heads", _i), ("kv_heads", _i),
                ("head_dim", _i), ("ffn", _i), ("vocab", _i), ("eps", _f), ("theta", _d)]


class qg_qwen3_weights(ctypes.Structure):
    _fields_ = [("embed", qg_affine8_matrix), ("final_norm", _vp),
                ("layers", ctypes.POINTER(qg_qwen3_layer))]


class qg_whisper_config(ctypes.Structure):
    _fields_ = [("d_model", ctypes.c_int), ("heads", ctypes.c_int), ("ffn", ctypes.c_int),
                ("eps", ctypes.c_float)]


class qg_whisper_layer(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("ln1_g", "ln1_b", "q", "q_b", "k", "v", "v_b", "o", "o_b", "ln2_g", "ln2_b",
                 "fc1", "fc1_b", "fc2", "fc2_b")]


class qg_code_predictor_weights(ctypes.Structure):
    _fields_ = [("input_proj", qg_affine8_matrix),
                ("code_embed", ctypes.POINTER(qg_affine8_matrix)),
                ("heads", ctypes.POINTER(qg_affine8_matrix)),
                ("layers", ctypes.POINTER(qg_qwen3_layer)), ("final_norm", _vp), ("groups", _i)]


_SIGS = {
    "qg_last_error": (ctypes.c_char_p, []),
    "qg_abi_version": (_i, []),
    "qg_kernel_launch_count": (ctypes.c_ulonglong, []),
    "qg_gemv_affine8_g64": (_i, [_vp, _vp, _vp, _vp, _i, _vp, _i, _vp, _i, _i, _i, _vp]),
    "qg_gemv_q4_0": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _vp]),
    "qg_gemm_q4_0_workspace_size": (_sz, [_i, _i, _i]),
    "qg_gemm_q4_0": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _vp, _sz, _vp]),
    "qg_gemm_q4_0_error": (_i, [_i, _i, _vp, ctypes.POINTER(ctypes.c_uint), _vp]),
    "qg_rmsnorm": (_i, [_vp, _vp, _f, _vp, _i, _i, _i, _vp]),
    "qg_rmsnorm_perhead": (_i, [_vp, _i, _vp, _f, _vp, _i, _i, _i, _i, _vp]),
    "qg_rope_neox": (_i, [_vp, _i, _vp, _d, _i, _i, _i, _i, _vp]),
    "qg_silu_mul": (_i, [_vp, _vp, _vp, _i, _i, _vp]),
    "qg_residual_add": (_i, [_vp, _vp, _i, _vp]),
    "qg_embed_affine8_g64": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _vp]),
    "qg_decode_attention_workspace_size": (_sz, [_i, _i, _i, _i, _i]),
    "qg_decode_attention": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _vp, _sz,
                                 _vp]),
    "qg_decode_attention_static_scratch_capacity": (_sz, []),
    "qg_decode_attention_static_scratch": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i,
                                                _f, _vp]),
    "qg_decode_step_workspace_size": (_sz, [ctypes.POINTER(qg_qwen3_config), _i, _i]),
    "qg_decode_step": (_i, [ctypes.POINTER(qg_qwen3_config), ctypes.POINTER(qg_qwen3_weights),
                            _vp, _vp, _i, _vp, _vp, _vp, _i, _vp, _sz, _vp]),
    "qg_decode_step_inspect": (_i, [ctypes.POINTER(qg_qwen3_config), _i, _i,
                                    ctypes.POINTER(ctypes.c_size_t)]),
    "qg_decode_step_inspect_f32": (_i, [ctypes.POINTER(qg_qwen3_config), _i, _i,
                                        ctypes.POINTER(ctypes.c_size_t)]),
    "qg_code_predict_workspace_size": (_sz, [ctypes.POINTER(qg_qwen3_config), _i]),
    "qg_gemm_q4_0_ex": (_i, [_vp, _vp, _i, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp, _sz, _vp]),
    "qg_gemm_q4_0_stall_test": (_i, [_vp, _vp, _vp, _i, _i, _i, _vp, _sz, _vp]),
    "qg_gemm_affine8_g64": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _vp, _i, _i, _i, _vp, _sz, _vp]),
    "qg_prefill_workspace_size": (_sz, [ctypes.POINTER(qg_qwen3_config), _i]),
    "qg_prefill": (_i, [ctypes.POINTER(qg_qwen3_config), ctypes.POINTER(qg_qwen3_weights), _vp,
                        _vp, _i, _vp, _i, _i, _vp, _vp, _sz, _vp]),
    "qg_prefill_inspect": (_i, [ctypes.POINTER(qg_qwen3_config), _i,
                                ctypes.POINTER(ctypes.c_size_t)]),
    "qg_layernorm": (_i, [_vp, _vp, _vp, _f, _vp, _i, _i, _i, _vp]),
    "qg_attention_rows": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp]),
    "qg_whisper_encoder_layer_workspace_size": (_sz, [ctypes.POINTER(qg_whisper_config), _i]),
    "qg_whisper_encoder_layer": (_i, [ctypes.POINTER(qg_whisper_config),
                                      ctypes.POINTER(qg_whisper_layer), _vp, _i, _vp, _sz, _vp]),
    "qg_whisper_encoder_layer_inspect": (_i, [ctypes.POINTER(qg_whisper_config), _i,
                                              ctypes.POINTER(ctypes.c_size_t)]),
    "qg_timeline_available": (_i, []),
    "qg_timeline_begin": (_i, [_vp, _i]),
    "qg_timeline_end": (_i, [ctypes.POINTER(ctypes.c_int), _i]),
    "qg_code_predict_trace_layout": (_i, [ctypes.POINTER(qg_qwen3_config), _i, _i,
                                          ctypes.POINTER(ctypes.c_size_t)]),
    "qg_code_predict_traced": (_i, [ctypes.POINTER(qg_qwen3_config),
                                    ctypes.POINTER(qg_code_predictor_weights), _vp, _vp, _vp,
                                    _vp, _i, _vp, _sz, _vp, _sz, _vp]),
    "qg_code_predict": (_i, [ctypes.POINTER(qg_qwen3_config),
                             ctypes.POINTER(qg_code_predictor_weights), _vp, _vp, _vp, _vp, _i,
                             _vp, _sz, _vp]),
    "qg_token_logprob_workspace_size": (_sz, [_i, _i]),
    "qg_token_logprob": (_i, [_vp, _i, _i, _vp, _vp, _vp, _sz, _vp]),
    "qg_sample_workspace_size": (_sz, [_i, _i, _i]),
    "qg_sample": (_i, [_vp, _i, _i, _vp, _i, _f, _f, _i, _vp, _vp, _vp, _sz, _vp]),
    "qg_step_graphs_enable": (None, [_i]),
    "qg_step_graphs_clear": (None, []),
    "qg_argmax_workspace_size": (_sz, [_i, _i]),
    "qg_argmax_f32": (_i, [_vp, _i, _i, _vp, _vp, _sz, _vp]),
    "qg_unpack_affine8": (_i, [_vp, _vp, _i, _i, _vp]),
    "qg_dequant_affine8_g64": (_i, [_vp, _vp, _vp, _vp, _i, _i, _vp]),
    "qg_dequant_q4_0": (_i, [_vp, _vp, _i, _i, _vp]),
}

for _name, (_res, _args) in _SIGS.items():
    _fn = getattr(lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


def last_error() -> str:
    return lib.qg_last_error().decode()


def _call(name, *args):
    st = getattr(lib, name)(*args)
    if st != QG_OK:
        raise QGError(name, st, last_error())


def _p(t):
    return None if t is None else t.data_ptr()


def _stream(stream=None):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else stream


def _dt(t):
    if t.dtype == torch.float32:
        return QG_F32
    if t.dtype == torch.bfloat16:
        return QG_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


# ------------------------------------------------------------------ ops ----

def qg_gemv_affine8_g64(w, scales, biases, x, y, residual=None, stream=None):
    """y[B,N] = dequant(w, scales, biases)[N,K] @ x[B,K] (+ residual). w is
    int32/uint32-viewed [N, K/4]; scales/biases int16/bf16 bits [N, K/64]."""
    N, K = w.shape[0], w.shape[1] * 4
    B = x.shape[0] if x.dim() == 2 else 1
    _call("qg_gemv_affine8_g64", _p(w), _p(scales), _p(biases), _p(x), _dt(x), _p(y), _dt(y),
          _p(residual), N, K, B, _stream(stream))


def qg_gemv_q4_0(blocks, x, y, bias=None, stream=None):
    N = blocks.shape[0]
    K = blocks.shape[1] // 18 * 32
    B = x.shape[0] if x.dim() == 2 else 1
    _call("qg_gemv_q4_0", _p(blocks), _p(x), _p(bias), _p(y), N, K, B, _stream(stream))


def qg_gemm_q4_0_workspace_size(M, N, K):
    return int(lib.qg_gemm_q4_0_workspace_size(M, N, K))


def qg_gemm_q4_0(blocks, A, C, bias=None, ws=None, stream=None):
    N = blocks.shape[0]
    K = blocks.shape[1] // 18 * 32
    M = A.shape[0]
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _call("qg_gemm_q4_0", _p(blocks), _p(A), _p(bias), _p(C), M, N, K, _p(ws), nbytes,
          _stream(stream))


def qg_gemm_q4_0_ex(blocks, A, C, bias=None, residual=None, gelu=False, ws=None, stream=None):
    """C = epilogue(bf16(A) @ bf16(W)^T + bias (+ residual)), A fp32 or bf16
    [M, K], C fp32 or bf16 [M, N]; gelu applies gelu_tanh."""
    N = blocks.shape[0]
    K = blocks.shape[1] // 18 * 32
    M = A.shape[0]
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _call("qg_gemm_q4_0_ex", _p(blocks), _p(A), _dt(A), _p(bias), _p(residual), _p(C), _dt(C),
          1 if gelu else 0, M, N, K, _p(ws), nbytes, _stream(stream))


def qg_gemm_affine8_g64(w, scales, biases, x, y, residual=None, ws=None, stream=None):
    """y[T, N] = x[T, K] (bf16) @ dequant(w)[N, K]^T (+ residual) on the
    tensor cores; ws holds the 4-byte error word."""
    N, K = w.shape[0], w.shape[1] * 4
    T = x.shape[0]
    nbytes = 0 if ws is None else ws.numel() * ws.element_size()
    _call("qg_gemm_affine8_g64", _p(w), _p(scales), _p(biases), _p(x), _p(y), _dt(y),
          _p(residual), N, K, T, _p(ws), nbytes, _stream(stream))


def qg_layernorm(x, gamma, beta, eps, y, stream=None):
    _call("qg_layernorm", _p(x), _p(gamma), _p(beta), eps, _p(y), _dt(y), x.shape[0],
          x.shape[1], _stream(stream))


def qg_attention_rows(q, k, v, out, H, Hkv, causal=False, stream=None):
    """q, out bf16 [B, T, H*D]; k, v bf16 [B, S, Hkv*D] (a leading batch
    dimension may be omitted)."""
    if q.dim() == 2:
        q, k, v, out = q[None], k[None], v[None], out[None]
    B, T = q.shape[0], q.shape[1]
    S = k.shape[1]
    D = q.shape[2] // H
    _call("qg_attention_rows", _p(q), _p(k), _p(v), _p(out), B, T, S, H, Hkv, D,
          1 if causal else 0, _stream(stream))


def qg_gemm_q4_0_error(M, K, ws, stream=None):
    """(status, code) of the device error word of the last GEMM on ``ws``."""
    code = ctypes.c_uint(0)
    st = lib.qg_gemm_q4_0_error(M, K, _p(ws), ctypes.byref(code), _stream(stream))
    return st, code.value


def qg_rmsnorm(x, w, eps, y, stream=None):
    rows, dim = x.shape
    _call("qg_rmsnorm", _p(x), _p(w), float(eps), _p(y), _dt(y), rows, dim, _stream(stream))


def qg_rmsnorm_perhead(x, w, eps, y, heads, stream=None):
    rows = x.shape[0]
    D = x.shape[1] // heads
    _call("qg_rmsnorm_perhead", _p(x), _dt(x), _p(w), float(eps), _p(y), _dt(y), rows, heads, D,
          _stream(stream))


def qg_rope_neox(x, pos, theta, heads, rotary_dim=None, stream=None):
    rows = x.shape[0]
    D = x.shape[1] // heads
    _call("qg_rope_neox", _p(x), _dt(x), _p(pos), float(theta), rows, heads, D,
          D if rotary_dim is None else rotary_dim, _stream(stream))


def qg_silu_mul(gate, up, out, stream=None):
    _call("qg_silu_mul", _p(gate), _p(up), _p(out), _dt(out), gate.numel(), _stream(stream))


def qg_residual_add(x, delta, stream=None):
    _call("qg_residual_add", _p(x), _p(delta), x.numel(), _stream(stream))


def qg_embed_affine8_g64(w, scales, biases, tokens, x, stream=None):
    _call("qg_embed_affine8_g64", _p(w), _p(scales), _p(biases), _p(tokens), _p(x), w.shape[0],
          w.shape[1] * 4, tokens.numel(), _stream(stream))


def qg_decode_attention_workspace_size(B, H, Hkv, D, cap):
    return int(lib.qg_decode_attention_workspace_size(B, H, Hkv, D, cap))


def qg_decode_attention(q, k_cache, v_cache, kv_len, out, H, Hkv, scale, ws, stream=None):
    """q [B, H*D] fp32; caches [B, Hkv, cap, D] bf16; kv_len int32 [B]."""
    B, _, cap, D = k_cache.shape
    _call("qg_decode_attention", _p(q), _p(k_cache), _p(v_cache), _p(kv_len), _p(out), _dt(out),
          B, H, Hkv, D, cap, float(scale), _p(ws), ws.numel() * ws.element_size(),
          _stream(stream))


def qg_argmax_workspace_size(B, V):
    return int(lib.qg_argmax_workspace_size(B, V))


def qg_argmax_f32(logits, out, ws, stream=None):
    """out[b] (int32, device) = first strict maximum of logits[b] (fp32
    [B, V]), NaNs skipped, 0 when nothing beats -inf."""
    B, V = logits.shape
    _call("qg_argmax_f32", _p(logits), B, V, _p(out), _p(ws), ws.numel() * ws.element_size(),
          _stream(stream))


def qg_token_logprob(logits, tokens, out, ws, stream=None):
    """out[b] (fp32, device) = log-softmax of logits[b] (fp32 [B, V]) at
    tokens[b] (int32, device)."""
    B, V = logits.shape
    _call("qg_token_logprob", _p(logits), B, V, _p(tokens), _p(out), _p(ws),
          ws.numel() * ws.element_size(), _stream(stream))


def qg_sample_workspace_size(B, V, top_k):
    return int(lib.qg_sample_workspace_size(B, V, top_k))


def qg_sample(logits, out, ws, past=None, penalty=1.0, temperature=1.0, top_k=0, r=None,
              stream=None):
    """out[b] (int32, device): repetition penalty over past[b] (int32 [B, P],
    -1 = empty), then greedy (top_k 0 or temperature 0) or a top-k draw with
    the uniform numbers r (fp32 [B]) from the temperature softmax."""
    B, V = logits.shape
    P = 0 if past is None else past.shape[1]
    _call("qg_sample", _p(logits), B, V, _p(past), P, float(penalty), float(temperature),
          int(top_k), _p(r), _p(out), _p(ws), ws.numel() * ws.element_size(), _stream(stream))


def qg_decode_attention_static_scratch_capacity():
    return int(lib.qg_decode_attention_static_scratch_capacity())


def qg_decode_attention_static_scratch(q, k_cache, v_cache, kv_len, out, H, Hkv, scale,
                                       stream=None):
    """qg_decode_attention with the library's fixed scratch (no workspace)."""
    B, _, cap, D = k_cache.shape
    _call("qg_decode_attention_static_scratch", _p(q), _p(k_cache), _p(v_cache), _p(kv_len),
          _p(out), _dt(out), B, H, Hkv, D, cap, float(scale), _stream(stream))


def qg_unpack_affine8(w, out, stream=None):
    _call("qg_unpack_affine8", _p(w), _p(out), w.shape[0], w.shape[1] * 4, _stream(stream))


def qg_dequant_affine8_g64(w, scales, biases, out, stream=None):
    _call("qg_dequant_affine8_g64", _p(w), _p(scales), _p(biases), _p(out), w.shape[0],
          w.shape[1] * 4, _stream(stream))


def qg_dequant_q4_0(blocks, out, stream=None):
    _call("qg_dequant_q4_0", _p(blocks), _p(out), blocks.shape[0], blocks.shape[1] // 18 * 32,
          _stream(stream))


# ---------------------------------------------------------- decode step ----

class Qwen3Model:
    """Device-resident packed Qwen3 weights plus the C structs that point at
    them. ``weights`` is the host dict layout of ``qg_synth.qwen3_weights``
    (numpy arrays); everything is uploaded once to ``device``."""

    def __init__(self, cfg: dict, weights: dict, device="cuda"):
        self.cfg = dict(cfg)
        self._keep = []

        def up(a):
            t = torch.from_numpy(a.view({2: "int16", 4: "int32"}[a.dtype.itemsize])).to(device)
            self._keep.append(t)
            return t.data_ptr()

        def mat(triple):
            w, s, b = triple
            return qg_affine8_matrix(up(w), up(s), up(b))

        self.c_cfg = qg_qwen3_config(cfg["hidden"], cfg["layers"], cfg["heads"], cfg["kv_heads"],
                                     cfg["head_dim"], cfg["ffn"], cfg["vocab"], cfg["eps"],
                                     cfg["theta"])
        L = cfg["layers"]
        self.c_layers = (qg_qwen3_layer * max(L, 1))()
        for i, lw in enumerate(weights["layers"]):
            cl = self.c_layers[i]
            cl.input_norm = up(lw["input_norm"])
            cl.post_norm = up(lw["post_norm"])
            cl.q_norm = up(lw["q_norm"])
            cl.k_norm = up(lw["k_norm"])
            for n in ("q", "k", "v", "o", "gate", "up", "down"):
                setattr(cl, n, mat(lw[n]))
        self.c_weights = qg_qwen3_weights(mat(weights["embed"]), up(weights["final_norm"]),
                                          ctypes.cast(self.c_layers, ctypes.POINTER(qg_qwen3_layer)))
        self.device = device

    def workspace_size(self, B, cap):
        return int(lib.qg_decode_step_workspace_size(ctypes.byref(self.c_cfg), B, cap))

    def new_state(self, B, cap):
        """Zeroed KV caches [layers, B, kv_heads, cap, head_dim] bf16, a
        workspace and a logits
        buffer for batch B."""
        c = self.cfg
        shape = (c["layers"], B, c["kv_heads"], cap, c["head_dim"])
        return dict(
            k_cache=torch.zeros(shape, dtype=torch.bfloat16, device=self.device),
            v_cache=torch.zeros(shape, dtype=torch.bfloat16, device=self.device),
            ws=torch.zeros(self.workspace_size(B, cap), dtype=torch.uint8, device=self.device),
            logits=torch.empty((B, c["vocab"]), dtype=torch.float32, device=self.device),
            B=B, cap=cap)

    def residual(self, state):
        """The fp32 residual stream [B, hidden] after the last layer of the
        latest step (the head of the step workspace, per include/qg.h)."""
        n = state["B"] * self.cfg["hidden"]
        return state["ws"][: 4 * n].view(torch.float32).view(state["B"], self.cfg["hidden"])

    def intermediates(self, state):
        """The last decoder layer's values after a step
        (``qg_decode_step_inspect`` and ``_inspect_f32``): dict of torch views
        into the workspace -- bf16 ``xn`` [B, hidden], ``attn``
        [B, heads*head_dim], ``xn2`` [B, hidden], ``h`` [B, ffn]; fp32
        ``q_proj`` [B, heads*head_dim], ``k_proj``, ``v_proj``
        [B, kv_heads*head_dim], ``x_attn`` [B, hidden], ``gate``, ``up``
        [B, ffn]."""
        c, B = self.cfg, state["B"]
        ws = state["ws"]
        off = (ctypes.c_size_t * 4)()
        _call("qg_decode_step_inspect", ctypes.byref(self.c_cfg), B, state["cap"], off)
        off32 = (ctypes.c_size_t * 6)()
        _call("qg_decode_step_inspect_f32", ctypes.byref(self.c_cfg), B, state["cap"], off32)

        def view(o, n, dt=torch.bfloat16):
            size = 2 if dt == torch.bfloat16 else 4
            return ws[o:o + size * B * n].view(dt).view(B, n)
        HD, KD, h, F = c["heads"] * c["head_dim"], c["kv_heads"] * c["head_dim"], c["hidden"], c["ffn"]
        f32 = torch.float32
        return {"xn": view(off[0], h), "attn": view(off[1], HD), "xn2": view(off[2], h),
                "h": view(off[3], F), "q_proj": view(off32[0], HD, f32),
                "k_proj": view(off32[1], KD, f32), "v_proj": view(off32[2], KD, f32),
                "x_attn": view(off32[3], h, f32), "gate": view(off32[4], F, f32),
                "up": view(off32[5], F, f32)}

    def prefill_workspace(self, T):
        n = int(lib.qg_prefill_workspace_size(ctypes.byref(self.c_cfg), T))
        return torch.empty(n, dtype=torch.uint8, device=self.device)

    def qg_prefill(self, state, tokens, p0, ws, logits=None, stream=None, layers=None):
        """The prompt rows ``tokens`` (device int32 [T]) of sequence 0 of
        ``state`` at positions p0 .. p0+T-1; the last row's logits into
        ``logits`` ([vocab]) when given. ``layers`` runs only the first that
        many layers."""
        cfg = self.c_cfg
        if layers is not None:
            cfg = qg_qwen3_config.from_buffer_copy(self.c_cfg)
            cfg.layers = layers
        _call("qg_prefill", ctypes.byref(cfg), ctypes.byref(self.c_weights),
              _p(state["k_cache"]), _p(state["v_cache"]), state["cap"], _p(tokens),
              tokens.shape[0], p0, _p(logits), _p(ws), ws.numel(), _stream(stream))

    def prefill_intermediates(self, ws, T):
        """The last layer's values after qg_prefill (qg_prefill_inspect)."""
        off = (ctypes.c_size_t * 12)()
        _call("qg_prefill_inspect", ctypes.byref(self.c_cfg), T, off)
        c = self.cfg
        HD, KD, h, F = c["heads"] * c["head_dim"], c["kv_heads"] * c["head_dim"], c["hidden"], c["ffn"]
        bf, f32 = torch.bfloat16, torch.float32
        spec = [("x", h, f32), ("xn", h, bf), ("q_proj", HD, f32), ("k_proj", KD, f32),
                ("v_proj", KD, f32), ("q_rope", HD, bf), ("att", HD, bf), ("x_attn", h, f32),
                ("xn2", h, bf), ("gate", F, f32), ("up", F, f32), ("h", F, bf)]
        out = {}
        for i, (name, n, dt) in enumerate(spec):
            size = 2 if dt == bf else 4
            out[name] = ws[off[i]:off[i] + size * T * n].view(dt).view(T, n)
        return out

    def qg_decode_step(self, state, tokens, positions, stream=None, layers=None):
        """tokens, positions: device int32 [B]. Writes state['logits'].
        ``layers`` runs only the first that many layers (then the head)."""
        cfg = self.c_cfg
        if layers is not None:
            cfg = qg_qwen3_config.from_buffer_copy(self.c_cfg)
            cfg.layers = layers
        _call("qg_decode_step", ctypes.byref(cfg), ctypes.byref(self.c_weights),
              _p(state["k_cache"]), _p(state["v_cache"]), state["cap"], _p(tokens),
              _p(positions), _p(state["logits"]), state["B"], _p(state["ws"]),
              state["ws"].numel(), _stream(stream))


class CodePredictor:
    """Device-resident packed code-predictor weights (the host dict layout of
    ``qg_synth.code_predictor_weights``) and ``qg_code_predict``."""

    def __init__(self, cfg: dict, weights: dict, device="cuda"):
        self.cfg = dict(cfg)
        self._keep = []

        def up(a):
            t = torch.from_numpy(a.view({2: "int16", 4: "int32"}[a.dtype.itemsize])).to(device)
            self._keep.append(t)
            return t.data_ptr()

        def mat(triple):
            w, s, b = triple
            return qg_affine8_matrix(up(w), up(s), up(b))

        self.c_cfg = qg_qwen3_config(cfg["hidden"], cfg["layers"], cfg["heads"], cfg["kv_heads"],
                                     cfg["head_dim"], cfg["ffn"], cfg["vocab"], cfg["eps"],
                                     cfg["theta"])
        G = len(weights["heads"])
        self.groups = G
        self.c_embed = (qg_affine8_matrix * G)(*[mat(t) for t in weights["code_embed"]])
        self.c_heads = (qg_affine8_matrix * G)(*[mat(t) for t in weights["heads"]])
        L = cfg["layers"]
        self.c_layers = (qg_qwen3_layer * max(L, 1))()
        for i, lw in enumerate(weights["layers"]):
            cl = self.c_layers[i]
            cl.input_norm = up(lw["input_norm"])
            cl.post_norm = up(lw["post_norm"])
            cl.q_norm = up(lw["q_norm"])
            cl.k_norm = up(lw["k_norm"])
            for n in ("q", "k", "v", "o", "gate", "up", "down"):
                setattr(cl, n, mat(lw[n]))
        self.c_weights = qg_code_predictor_weights(
            mat(weights["input_proj"]), ctypes.cast(self.c_embed, ctypes.POINTER(qg_affine8_matrix)),
            ctypes.cast(self.c_heads, ctypes.POINTER(qg_affine8_matrix)),
            ctypes.cast(self.c_layers, ctypes.POINTER(qg_qwen3_layer)), up(weights["final_norm"]), G)
        self.device = device

    def workspace(self, B):
        n = int(lib.qg_code_predict_workspace_size(ctypes.byref(self.c_cfg), B))
        return torch.empty(n, dtype=torch.uint8, device=self.device)

    def qg_code_predict(self, lm_hidden, code0, codes, ws, logits=None, stream=None):
        """lm_hidden fp32 [B, hidden], code0 int32 [B] (device) -> codes int32
        [groups, B]; logits fp32 [groups, B, vocab] when given."""
        B = lm_hidden.shape[0]
        _call("qg_code_predict", ctypes.byref(self.c_cfg), ctypes.byref(self.c_weights),
              _p(lm_hidden), _p(code0), _p(codes), _p(logits), B, _p(ws),
              ws.numel(), _stream(stream))

    def trace_layout(self, B):
        """(total bytes, bytes per group, offset of slot 0 in a group, bytes
        per slot) of the trace of ``qg_code_predict_traced``."""
        out = (ctypes.c_size_t * 4)()
        _call("qg_code_predict_trace_layout", ctypes.byref(self.c_cfg), B, self.groups, out)
        return tuple(int(v) for v in out)

    def step_offsets(self, B):
        """Offsets of the step buffers inside a trace slot (the workspace
        head, cap 1): ``qg_decode_step_inspect`` and ``_inspect_f32``."""
        off = (ctypes.c_size_t * 4)()
        _call("qg_decode_step_inspect", ctypes.byref(self.c_cfg), B, 1, off)
        off32 = (ctypes.c_size_t * 6)()
        _call("qg_decode_step_inspect_f32", ctypes.byref(self.c_cfg), B, 1, off32)
        return list(off), list(off32)

    def qg_code_predict_traced(self, lm_hidden, code0, codes, ws, trace, logits=None,
                               stream=None):
        """qg_code_predict that also fills ``trace`` (uint8, trace_layout()[0]
        bytes) with every group's layer values."""
        B = lm_hidden.shape[0]
        _call("qg_code_predict_traced", ctypes.byref(self.c_cfg), ctypes.byref(self.c_weights),
              _p(lm_hidden), _p(code0), _p(codes), _p(logits), B, _p(ws), ws.numel(),
              _p(trace), trace.numel(), _stream(stream))


class WhisperEncoderLayer:
    """Device-resident weights of one Whisper encoder layer (the host dict of
    ``qg_synth.whisper_layer_weights``) and ``qg_whisper_encoder_layer``."""

    NAMES = ("ln1_g", "ln1_b", "q", "q_b", "k", "v", "v_b", "o", "o_b", "ln2_g", "ln2_b", "fc1",
             "fc1_b", "fc2", "fc2_b")

    def __init__(self, cfg: dict, weights: dict, device="cuda"):
        self.cfg = dict(cfg)
        self._keep = {}
        for n in self.NAMES:
            a = weights[n]
            t = torch.from_numpy(a if a.dtype == "uint8" else a.astype("float32")).to(device)
            self._keep[n] = t
        self.c_cfg = qg_whisper_config(cfg["d_model"], cfg["heads"], cfg["ffn"], cfg["eps"])
        self.c_w = qg_whisper_layer(*[self._keep[n].data_ptr() for n in self.NAMES])
        self.device = device

    def tensor(self, name):
        return self._keep[name]

    def workspace(self, M):
        n = int(lib.qg_whisper_encoder_layer_workspace_size(ctypes.byref(self.c_cfg), M))
        return torch.empty(n, dtype=torch.uint8, device=self.device)

    def qg_whisper_encoder_layer(self, x, ws, stream=None):
        """x fp32 [M, d_model] in place."""
        _call("qg_whisper_encoder_layer", ctypes.byref(self.c_cfg), ctypes.byref(self.c_w), _p(x),
              x.shape[0], _p(ws), ws.numel(), _stream(stream))

    def intermediates(self, ws, M):
        """Views into the workspace after a call: bf16 ``xl``, ``q``, ``k``,
        ``v``, ``ctx``, ``xl2`` [M, d], ``mid`` [M, ffn]; fp32 ``xa`` [M, d];
        and the six matmuls' error words (``err``, int32)."""
        off = (ctypes.c_size_t * 9)()
        _call("qg_whisper_encoder_layer_inspect", ctypes.byref(self.c_cfg), M, off)
        d, F = self.cfg["d_model"], self.cfg["ffn"]

        def view(o, n, dt=torch.bfloat16):
            size = 2 if dt == torch.bfloat16 else 4
            return ws[o:o + size * M * n].view(dt).view(M, n)
        out = {name: view(off[i], d) for i, name in enumerate(("xl", "q", "k", "v", "ctx"))}
        out["xa"] = view(off[5], d, torch.float32)
        out["xl2"] = view(off[6], d)
        out["mid"] = view(off[7], F)
        out["err"] = ws[off[8]:off[8] + 6 * 256].view(torch.int32).view(6, 64)[:, 0]
        return out
