"""C-ABI checks that need no GPU: the library loads, exports every entry
point include/qg.h declares, and refuses bad arguments before any launch with
a message that names the argument (the refusal pattern of turbospark-runtime
0.3.0, src/qwen3_asr_metal.rs, `open` / `load_packed_linear` and its
`open_rejects_undersized_norm_tensors` test)."""
import ctypes
import os
import re

import pytest

import weight_only_quantized_03_b200 as qg

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = 0x7F0000000000  # a 256-byte aligned address that is never dereferenced


def declared_functions():
    with open(os.path.join(ROOT, "include", "qg.h")) as f:
        text = f.read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(qg_\w+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for must in ["qg_gemv_affine8_g64", "qg_gemv_q4_0", "qg_gemm_q4_0", "qg_rmsnorm",
                 "qg_rmsnorm_perhead", "qg_rope_neox", "qg_silu_mul", "qg_residual_add",
                 "qg_decode_attention", "qg_decode_step", "qg_last_error"]:
        assert must in names


def test_library_exports_every_declared_symbol():
    for name in declared_functions():
        assert hasattr(qg.lib, name), name
    assert qg.lib.qg_abi_version() >= 1


def _status(name, *args):
    st = getattr(qg.lib, name)(*args)
    return st, qg.last_error()


def test_gemv_rejects_bad_k_batch_and_pointers():
    st, msg = _status("qg_gemv_affine8_g64", FAKE, FAKE, FAKE, FAKE, qg.QG_BF16, FAKE, qg.QG_F32,
                      None, 128, 100, 1, None)
    assert st == qg.QG_ERR_UNSUPPORTED_SHAPE and "K=100" in msg
    st, msg = _status("qg_gemv_affine8_g64", FAKE, FAKE, FAKE, FAKE, qg.QG_BF16, FAKE, qg.QG_F32,
                      None, 128, 128, 33, None)
    assert st == qg.QG_ERR_UNSUPPORTED_SHAPE and "B=33" in msg
    st, msg = _status("qg_gemv_affine8_g64", None, FAKE, FAKE, FAKE, qg.QG_BF16, FAKE, qg.QG_F32,
                      None, 128, 128, 1, None)
    assert st == qg.QG_ERR_INVALID_ARGUMENT and "w=" in msg
    st, msg = _status("qg_gemv_affine8_g64", FAKE + 4, FAKE, FAKE, FAKE, qg.QG_BF16, FAKE,
                      qg.QG_F32, None, 128, 128, 1, None)
    assert st == qg.QG_ERR_MISALIGNED and "w is not 16-byte aligned" in msg
    st, msg = _status("qg_gemv_affine8_g64", FAKE, FAKE, FAKE, FAKE, 7, FAKE, qg.QG_F32, None,
                      128, 128, 1, None)
    assert st == qg.QG_ERR_INVALID_ARGUMENT and "x_dtype" in msg
    # empty work is a valid no-op that launches nothing
    st, msg = _status("qg_gemv_affine8_g64", None, None, None, None, qg.QG_BF16, None, qg.QG_F32,
                      None, 0, 128, 1, None)
    assert st == qg.QG_OK and msg == ""


def test_q4_0_rejects_bad_k():
    st, msg = _status("qg_gemv_q4_0", FAKE, FAKE, None, FAKE, 16, 48, 1, None)
    assert st == qg.QG_ERR_UNSUPPORTED_SHAPE and "K=48" in msg


def test_attention_rejects_bad_group_and_small_workspace():
    st, msg = _status("qg_decode_attention", FAKE, FAKE, FAKE, FAKE, FAKE, qg.QG_BF16, 1, 12, 8,
                      128, 64, 1.0, FAKE, 1 << 20, None)
    assert st == qg.QG_ERR_UNSUPPORTED_SHAPE and "Hkv=8" in msg
    need = qg.lib.qg_decode_attention_workspace_size(1, 16, 8, 128, 513)
    assert need > 0
    st, msg = _status("qg_decode_attention", FAKE, FAKE, FAKE, FAKE, FAKE, qg.QG_BF16, 1, 16, 8,
                      128, 513, 1.0, FAKE, need - 1, None)
    assert st == qg.QG_ERR_WORKSPACE_TOO_SMALL and str(need) in msg


def test_attention_static_scratch_refuses_shapes_beyond_its_capacity():
    """The fixed scratch limits only the shapes that take the split kernel
    (here head_dim 96); cluster and tensor-core shapes use no scratch."""
    cap_bytes = qg.lib.qg_decode_attention_static_scratch_capacity()
    assert cap_bytes == 4 << 20
    need = qg.lib.qg_decode_attention_workspace_size(32, 16, 2, 96, 32768)
    assert need > cap_bytes
    st, msg = _status("qg_decode_attention_static_scratch", FAKE, FAKE, FAKE, FAKE, FAKE,
                      qg.QG_BF16, 32, 16, 2, 96, 32768, 1.0, None)
    assert st == qg.QG_ERR_WORKSPACE_TOO_SMALL and str(need) in msg and str(cap_bytes) in msg
    import torch
    if not torch.cuda.is_available():
        # shapes whose nominal split workspace exceeds the array but that take
        # the cluster kernel (2 query heads per KV head) or the tensor-core
        # kernel (8 per KV head, long cache) are not refused for capacity
        # (with no device they stop at the address lookup, before any launch)
        for Hkv in (8, 2):
            assert qg.lib.qg_decode_attention_workspace_size(32, 16, Hkv, 128, 32768) > cap_bytes
            st, msg = _status("qg_decode_attention_static_scratch", FAKE, FAKE, FAKE, FAKE, FAKE,
                              qg.QG_BF16, 32, 16, Hkv, 128, 32768, 1.0, None)
            assert st == qg.QG_ERR_CUDA and "address lookup" in msg


def test_elementwise_reject_bad_shapes():
    assert _status("qg_rmsnorm", FAKE, FAKE, 1e-6, FAKE, qg.QG_BF16, 1, 6, None)[0] == \
        qg.QG_ERR_UNSUPPORTED_SHAPE
    st, msg = _status("qg_rope_neox", FAKE, qg.QG_F32, FAKE, 1e6, 1, 2, 128, 130, None)
    assert st == qg.QG_ERR_UNSUPPORTED_SHAPE and "rotary_dim=130" in msg
    assert _status("qg_rmsnorm_perhead", FAKE, qg.QG_F32, FAKE, 1e-6, FAKE, qg.QG_F32, 1, 2, 48,
                   None)[0] == qg.QG_ERR_UNSUPPORTED_SHAPE


def _tiny_model_structs(layers=2):
    cfg = qg.qg_qwen3_config(64, layers, 2, 1, 64, 128, 261, 1e-5, 1e4)
    mat = qg.qg_affine8_matrix(FAKE, FAKE, FAKE)
    arr = (qg.qg_qwen3_layer * layers)()
    for i in range(layers):
        arr[i].input_norm = arr[i].post_norm = arr[i].q_norm = arr[i].k_norm = FAKE
        for n in ("q", "k", "v", "o", "gate", "up", "down"):
            setattr(arr[i], n, mat)
    w = qg.qg_qwen3_weights(mat, FAKE, ctypes.cast(arr, ctypes.POINTER(qg.qg_qwen3_layer)))
    return cfg, w, arr


def test_decode_step_names_the_bad_tensor():
    cfg, w, arr = _tiny_model_structs()
    arr[1].down.w = None          # a missing matrix in layer 1
    need = qg.lib.qg_decode_step_workspace_size(ctypes.byref(cfg), 1, 16)
    st, msg = _status("qg_decode_step", ctypes.byref(cfg), ctypes.byref(w), FAKE, FAKE, 16, FAKE,
                      FAKE, FAKE, 1, FAKE, need, None)
    assert st == qg.QG_ERR_INVALID_ARGUMENT and "layer 1" in msg and "down" in msg
    arr[1].down.w = FAKE
    arr[0].k_norm = None          # a missing norm weight
    st, msg = _status("qg_decode_step", ctypes.byref(cfg), ctypes.byref(w), FAKE, FAKE, 16, FAKE,
                      FAKE, FAKE, 1, FAKE, need, None)
    assert st == qg.QG_ERR_INVALID_ARGUMENT and "layer 0" in msg and "norm" in msg
    arr[0].k_norm = FAKE
    st, msg = _status("qg_decode_step", ctypes.byref(cfg), ctypes.byref(w), FAKE, FAKE, 16, FAKE,
                      FAKE, FAKE, 1, FAKE, need - 256, None)
    assert st == qg.QG_ERR_WORKSPACE_TOO_SMALL
    bad = qg.qg_qwen3_config(64, 2, 3, 2, 64, 128, 261, 1e-5, 1e4)
    st, msg = _status("qg_decode_step", ctypes.byref(bad), ctypes.byref(w), FAKE, FAKE, 16, FAKE,
                      FAKE, FAKE, 1, FAKE, need, None)
    assert st == qg.QG_ERR_UNSUPPORTED_SHAPE and "kv_heads=2" in msg


def test_argmax_rejects_bad_arguments():
    need = qg.lib.qg_argmax_workspace_size(2, 1000)
    assert need >= 2 * 8
    st, msg = _status("qg_argmax_f32", FAKE, 2, 0, FAKE, FAKE, need, None)
    assert st == qg.QG_ERR_UNSUPPORTED_SHAPE and "V=0" in msg
    st, msg = _status("qg_argmax_f32", None, 2, 1000, FAKE, FAKE, need, None)
    assert st == qg.QG_ERR_INVALID_ARGUMENT and "logits" in msg
    st, msg = _status("qg_argmax_f32", FAKE + 2, 2, 1000, FAKE, FAKE, need, None)
    assert st == qg.QG_ERR_MISALIGNED
    st, msg = _status("qg_argmax_f32", FAKE, 2, 1000, FAKE, FAKE, need - 8, None)
    assert st == qg.QG_ERR_WORKSPACE_TOO_SMALL and str(need) in msg
    assert _status("qg_argmax_f32", None, 0, 1000, None, None, 0, None)[0] == qg.QG_OK


def test_code_predict_names_the_bad_table():
    cfg, _, arr = _tiny_model_structs()
    G = 3
    mats = lambda: (qg.qg_affine8_matrix * G)(*[qg.qg_affine8_matrix(FAKE, FAKE, FAKE)
                                                for _ in range(G)])
    emb, heads = mats(), mats()
    w = qg.qg_code_predictor_weights(
        qg.qg_affine8_matrix(FAKE, FAKE, FAKE),
        ctypes.cast(emb, ctypes.POINTER(qg.qg_affine8_matrix)),
        ctypes.cast(heads, ctypes.POINTER(qg.qg_affine8_matrix)),
        ctypes.cast(arr, ctypes.POINTER(qg.qg_qwen3_layer)), FAKE, G)
    need = qg.lib.qg_code_predict_workspace_size(ctypes.byref(cfg), 1)
    assert need > qg.lib.qg_decode_step_workspace_size(ctypes.byref(cfg), 1, 1)

    def call(ws_bytes=need, codes=FAKE):
        return _status("qg_code_predict", ctypes.byref(cfg), ctypes.byref(w), FAKE, FAKE, codes,
                       None, 1, FAKE, ws_bytes, None)

    heads[2].w = None
    st, msg = call()
    assert st == qg.QG_ERR_INVALID_ARGUMENT and "heads" in msg
    heads[2].w = FAKE
    emb[0].scales = None
    st, msg = call()
    assert st == qg.QG_ERR_INVALID_ARGUMENT and "code_embed" in msg
    emb[0].scales = FAKE
    st, msg = call(codes=None)
    assert st == qg.QG_ERR_INVALID_ARGUMENT and "codes" in msg
    st, msg = call(ws_bytes=need - 256)
    assert st == qg.QG_ERR_WORKSPACE_TOO_SMALL and str(need) in msg
    w.groups = 1
    st, msg = call()
    assert st == qg.QG_ERR_UNSUPPORTED_SHAPE and "groups=1" in msg


def test_sample_rejects_bad_arguments():
    need = qg.lib.qg_sample_workspace_size(2, 151936, 50)
    args = lambda **kw: [kw.get("logits", FAKE), 2, kw.get("V", 151936), FAKE, 4,
                         ctypes.c_float(kw.get("penalty", 1.2)), ctypes.c_float(1.0),
                         kw.get("top_k", 50), kw.get("r", FAKE), FAKE, FAKE, kw.get("ws", need), None]
    st, msg = _status("qg_sample", *args(top_k=65))
    assert st == qg.QG_ERR_UNSUPPORTED_SHAPE and "top_k=65" in msg
    st, msg = _status("qg_sample", *args(penalty=0.0))
    assert st == qg.QG_ERR_INVALID_ARGUMENT and "penalty" in msg
    st, msg = _status("qg_sample", *args(r=None))
    assert st == qg.QG_ERR_INVALID_ARGUMENT
    st, msg = _status("qg_sample", *args(V=8192 * 2048 // 50 + 4096))
    assert st == qg.QG_ERR_UNSUPPORTED_SHAPE and "candidates" in msg
    st, msg = _status("qg_sample", *args(ws=need - 256))
    assert st == qg.QG_ERR_WORKSPACE_TOO_SMALL and str(need) in msg


def test_new_row_entry_points_refuse_bad_shapes():
    """The multi-row attention, the extended Q4_0 matmul, the affine8
    matmul, LayerNorm, the Whisper layer and the prefill refuse bad shapes
    before any launch, naming the argument."""
    st, msg = _status("qg_attention_rows", FAKE, FAKE, FAKE, FAKE, 1, 4, 4, 2, 2, 96, 0, None)
    assert st == qg.QG_ERR_UNSUPPORTED_SHAPE and "D=96" in msg
    st, msg = _status("qg_attention_rows", FAKE, FAKE, FAKE, FAKE, 1, 8, 4, 2, 2, 64, 1, None)
    assert st == qg.QG_ERR_UNSUPPORTED_SHAPE and "causal" in msg
    st, msg = _status("qg_gemm_q4_0_ex", FAKE, FAKE, qg.QG_BF16, None, FAKE, FAKE, qg.QG_BF16, 0,
                      128, 128, 128, FAKE, 256, None)
    assert st == qg.QG_ERR_INVALID_ARGUMENT and "residual" in msg
    st, msg = _status("qg_gemm_affine8_g64", FAKE, FAKE, FAKE, FAKE, FAKE, qg.QG_F32, None, 128,
                      96, 4, FAKE, 4, None)
    assert st == qg.QG_ERR_UNSUPPORTED_SHAPE and "K=96" in msg
    st, msg = _status("qg_layernorm", FAKE, FAKE, FAKE, 1e-5, FAKE, qg.QG_BF16, 4, 4096, None)
    assert st == qg.QG_ERR_UNSUPPORTED_SHAPE and "dim=4096" in msg
    wc = qg.qg_whisper_config(1280, 16, 5120, 1e-5)   # head size 80
    st, msg = _status("qg_whisper_encoder_layer", ctypes.byref(wc), None, FAKE, 10, FAKE, 1 << 30,
                      None)
    assert st == qg.QG_ERR_UNSUPPORTED_SHAPE and "heads=16" in msg
    cfg = qg.qg_qwen3_config(512, 1, 4, 2, 128, 1024, 1000, 1e-6, 1e6)
    st, msg = _status("qg_prefill", ctypes.byref(cfg), None, FAKE, FAKE, 16, FAKE, 10, 8, FAKE,
                      FAKE, 1 << 30, None)
    assert st == qg.QG_ERR_UNSUPPORTED_SHAPE and "cap=16" in msg
