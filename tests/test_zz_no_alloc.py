"""qg_decode_attention_static_scratch: the attention entry point that takes no
workspace (its scratch is a fixed device array inside libqg).

Collected last on purpose (file name): it must give the same results as the
workspace entry point whether it runs alone or after every other GPU test,
and on two calls in a row (the second reuses the scratch the first left).
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


# Calls in a row with different shapes. The first two take the cluster
# kernel (head_dim 128, 2 query heads per KV head), which merges through
# distributed shared memory and leaves the scratch untouched. The others take
# the split kernel, whose partials and ticket counters live in the static
# scratch: 8 query heads per KV head, then head_dim 96, then the first split
# shape again with other lengths, so each call starts from the scratch the
# previous call left (other split plans, counters left at zero or not).
CALLS = [
    (1, 16, 8, 128, 513, [512], 60, "f32"),
    (3, 16, 8, 128, 600, [33, 600, 1], 70, "bf16"),
    (2, 16, 2, 128, 700, [700, 350], 80, "f32"),
    (3, 12, 4, 96, 300, [257, 1, 300], 90, "bf16"),
    (2, 16, 2, 128, 700, [513, 64], 100, "f32"),
]


def _takes_split_kernel(B, H, Hkv, D, cap):
    """The library's rule: the tensor-core kernel serves head_dim 64/128 with
    at most 8 query heads per KV head when B * Hkv * cap >= 2^16, the cluster
    kernel head_dim 32/64/128/256 with at most 4; every other shape merges
    its splits through the scratch."""
    g = H // Hkv
    mma = D in (64, 128) and g <= 8 and B * Hkv * cap >= 1 << 16
    return not mma and not (D in (32, 64, 128, 256) and g <= 4)


def _inputs(B, H, Hkv, D, cap, lens, seed):
    kbits = qg_synth.gaussian_bf16_bits((B, Hkv, cap, D), 1.0, seed)
    vbits = qg_synth.gaussian_bf16_bits((B, Hkv, cap, D), 1.0, seed + 1)
    q = qg_synth.gaussian((B, H * D), 1.0, seed + 2)
    return kbits, vbits, q, np.array(lens, dtype=np.int32)


def test_static_scratch_matches_workspace_entry_point_on_consecutive_calls():
    assert qg.qg_decode_attention_static_scratch_capacity() == 4 << 20
    assert sum(_takes_split_kernel(c[0], c[1], c[2], c[3], c[4]) for c in CALLS) == 3
    for B, H, Hkv, D, cap, lens, seed, od in CALLS:
        kbits, vbits, q, kv_len = _inputs(B, H, Hkv, D, cap, lens, seed)
        qd, kd, vd, ld = dev(q), bf16_dev(kbits), bf16_dev(vbits), dev(kv_len)
        dt = torch.float32 if od == "f32" else torch.bfloat16
        scale = 1.0 / math.sqrt(D)
        ws = torch.empty(qg.qg_decode_attention_workspace_size(B, H, Hkv, D, cap),
                         dtype=torch.uint8, device="cuda")
        assert ws.numel() <= qg.qg_decode_attention_static_scratch_capacity()
        ref = torch.empty((B, H * D), dtype=dt, device="cuda")
        qg.qg_decode_attention(qd, kd, vd, ld, ref, H, Hkv, scale, ws)
        got = torch.full((B, H * D), float("nan"), dtype=dt, device="cuda")
        qg.qg_decode_attention_static_scratch(qd, kd, vd, ld, got, H, Hkv, scale)
        torch.cuda.synchronize()
        g, r = host64(got), host64(ref)
        assert_parity(g, r, bf16_out=(od == "bf16"), what=f"static vs workspace B={B} cap={cap}")
        # and both against the oracle
        k64, v64 = O.bf16_bits_to_f64(kbits), O.bf16_bits_to_f64(vbits)
        for b in range(B):
            oref = O.decode_attention(q[b], k64[b], v64[b], int(kv_len[b]), H, Hkv, D)
            assert_parity(g[b], oref, bf16_out=(od == "bf16"), what=f"static vs oracle b={b}")
