"""The kernels at band sizes other than the pages' (sink 64, recent 256, window
512), against the float64 oracle: the degenerate ones (recent 1, where a
streaming query reads the sink and itself; window 1, the query alone; no
sink), sizes that end inside a 128-key tile, and the largest the library
accepts (sink + recent = 8192, window = 8192).  For each: the append (caches
byte for byte), the one-token decode after it, the prefill, and the verify
block.  Tolerances as the other parity tests.

Rows that attend one or two keys (window 1 with a sink logit; sink 1 +
recent 1) have |O| close to |v|, up to about 5, where the output's own bf16
rounding is already half an ulp (0.0156); the prefill adds the same
bf16-rounded probabilities to the row sum that the PV product uses, so that
no second rounding error stacks on top.  They are held to the same bar."""
import numpy as np
import pytest
import torch

import oracle
import kv_cache_reduction_b200 as duo
from kv_cache_reduction_b200 import inputs

from gpu_helpers import assert_close, host_cache, layers, random_cache

pytestmark = pytest.mark.gpu

MASK = (1, 0, 0, 1, 0, 1, 1, 0)
# (sink, recent, window): window > 0 makes a sliding-window layer (with sink logits)
SIZES = [(0, 1, 0), (1, 1, 0), (5, 37, 0), (0, 300, 0), (64, 8128, 0),
         (0, 0, 1), (0, 0, 100), (0, 0, 8192)]
IDS = [f"sink{s}-recent{r}" if not w else f"window{w}" for s, r, w in SIZES]


def _layer(B, sink, recent, window):
    if window:
        sig = inputs.randn_f32((48,), 7000 + window)
        return layers(B, window=window, sink_logit=sig)
    return layers(B, full_mask=MASK, sink=sink, recent=recent)


def _span(sink, recent, window):
    return window if window else sink + recent


@pytest.mark.parametrize("sink,recent,window", SIZES, ids=IDS)
def test_append_then_decode(cuda_device, sink, recent, window):
    B = 2
    span = _span(sink, recent, window)
    p, o = _layer(B, sink, recent, window)
    total = span + 300
    cache = random_cache(p, total, [0] * B, [0] * B, seed=11)
    ref = host_cache(o, cache)
    # chunks that stop one short of the band, on it, one past it, then past it by far
    chunks = [c for c in (span - 1, 1, 1, 298) if c > 0]
    for step, n in enumerate(chunks):
        k = inputs.randn_bf16((B, n, 8, 128), 100 + 2 * step, "cuda")
        v = inputs.randn_bf16((B, n, 8, 128), 101 + 2 * step, "cuda")
        duo.duo_kv_append(p, cache, k, v)
        oracle.kv_append(o, ref, inputs.bits(k), inputs.bits(v))
        torch.cuda.synchronize()
        assert duo.duo_get_device_status() == duo.DUO_OK
        got = host_cache(o, cache)
        for name in ("full_k", "full_v", "strm_k", "strm_v", "seq_len", "ring_head"):
            assert np.array_equal(getattr(got, name), getattr(ref, name)), (name, step)
        n_now = int(cache.seq_len.max().item())
        q = inputs.randn_bf16((B, 48, 128), 200 + step, "cuda")
        out = torch.full((B, 48, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.full((B, 48), float("nan"), dtype=torch.float32, device="cuda")
        duo.duo_attn_decode(p, cache, q, n_now, out, lse, duo.workspace_for(p, n_now))
        torch.cuda.synchronize()
        assert duo.duo_get_device_status() == duo.DUO_OK
        ro, rl = oracle.attn_decode(o, ref, inputs.bits(q))
        assert_close(out, ro.reshape(B, 48, 128), lse, rl.reshape(B, 48), f"decode n={n_now}")


@pytest.mark.parametrize("sink,recent,window", SIZES, ids=IDS)
def test_prefill(cuda_device, sink, recent, window):
    B, L = 1, 600                                     # five tiles, the last one ragged
    p, o = _layer(B, sink, recent, window)
    q = inputs.randn_bf16((B, L, 48, 128), 300, "cuda")
    k = inputs.randn_bf16((B, L, 8, 128), 301, "cuda")
    v = inputs.randn_bf16((B, L, 8, 128), 302, "cuda")
    out = torch.full((B, L, 48, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B, 48, L), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.zeros(duo.duo_prefill_workspace_bytes(), dtype=torch.uint8, device="cuda")
    duo.duo_attn_prefill(p, q, k, v, out, lse, workspace=ws)
    torch.cuda.synchronize()
    assert duo.duo_get_device_status() == duo.DUO_OK
    ro, rl = oracle.attn_prefill(o, inputs.bits(q), inputs.bits(k), inputs.bits(v))
    got = out.permute(0, 2, 1, 3).reshape(-1, 128)
    assert_close(got, ro, lse.reshape(-1), rl, "prefill")


@pytest.mark.parametrize("sink,recent,window", SIZES, ids=IDS)
@pytest.mark.parametrize("q_len", [3, 8])
def test_verify_block(cuda_device, sink, recent, window, q_len):
    span = _span(sink, recent, window)
    seq = [0, 1, span - 1 if span > 1 else 2, span, span + 77]
    B = len(seq)
    p, o = _layer(B, sink, recent, window)
    ring = window if window else recent
    rh = [0, 0, 0, 0, 77 % ring]
    cache = random_cache(p, span + 77, seq, rh, seed=400 + q_len)
    n_max = max(seq)
    qb = inputs.randn_bf16((B, q_len, 48, 128), 410, "cuda")
    kb = inputs.randn_bf16((B, q_len, 8, 128), 411, "cuda")
    vb = inputs.randn_bf16((B, q_len, 8, 128), 412, "cuda")
    out = torch.full((B, q_len, 48, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B, q_len, 48), float("nan"), dtype=torch.float32, device="cuda")
    nbytes = max(duo.duo_decode_block_workspace_bytes(p, q_len, n_max), 256)
    ws = torch.zeros((nbytes + 255) // 256 * 256, dtype=torch.uint8, device="cuda")
    snap = host_cache(o, cache)
    duo.duo_attn_decode_block(p, cache, qb, kb, vb, n_max, out, lse, ws)
    torch.cuda.synchronize()
    assert duo.duo_get_device_status() == duo.DUO_OK
    ro, rl = oracle.attn_decode_block(o, snap, inputs.bits(qb), inputs.bits(kb), inputs.bits(vb))
    assert_close(out, ro.reshape(B, q_len, 48, 128), lse, rl.reshape(B, q_len, 48), f"block q_len={q_len}")
