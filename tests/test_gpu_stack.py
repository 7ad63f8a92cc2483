"""The 40-layer decode stack (DuoAttention layers 3, 7, ..., 39 with 2 of 8
heads full; sliding-window layers of 512 with sink logits elsewhere).

* full size (B=16, context 131072) for two layers of each kind, six
  sequences of each against the oracle: sliding layers 0 and 38 (38 with every
  ring pointer one slot before the wrap) and DuoAttention layers 3 and 39,
  each with its own seeded head mask;
* the whole 40-layer step captured in one CUDA graph gives the same bytes as
  the same 40 calls made eagerly (smaller context)."""
import numpy as np
import pytest
import torch

import oracle
import kv_cache_reduction_b200 as duo
from kv_cache_reduction_b200 import inputs

from gpu_helpers import assert_close, layers, random_cache

pytestmark = pytest.mark.gpu


def layer_of(w, li, batch):
    mask = inputs.stack_layer_masks(w)[li]
    if mask is None:
        sig = inputs.randn_f32((48,), w.seed * 100 + li)
        return layers(batch, window=inputs.WINDOW, sink_logit=sig)
    return layers(batch, full_mask=mask)


@pytest.mark.slow
@pytest.mark.parametrize("li", [0, 3, 38, 39])
def test_stack40_layer_full_size_sampled(cuda_device, li):
    w = inputs.workload("stack40")
    B, n = w.batch, w.seq_len
    p, o = layer_of(w, li, B)
    rng = np.random.default_rng(w.seed + li)
    ring = p.ring_slots - p.sink if p.window == 0 else p.window
    if li == 38:
        rh = [ring - 1] * B             # the next ring write wraps to slot 0
    else:
        rh = rng.integers(0, ring, size=B).tolist()
    cache = random_cache(p, n, [n] * B, rh, seed=w.seed * 100 + li)
    q = inputs.randn_bf16((B, 48, 128), w.seed * 100 + li + 50, "cuda")
    out = torch.empty((B, 48, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, 48), dtype=torch.float32, device="cuda")
    duo.duo_attn_decode(p, cache, q, n, out, lse, duo.workspace_for(p, n))
    torch.cuda.synchronize()
    assert duo.duo_get_device_status() == duo.DUO_OK
    o1 = oracle.Layer(1, 48, 8, 128, o.sink, o.recent, o.window, o.softmax_scale, o.full_mask,
                      o.sink_logit)
    for b in (0, 3, 6, 9, 12, 15):
        hc = oracle.Cache(o1, n if o1.n_full else 1)
        if o1.n_full:
            hc.full_k = inputs.bits(cache.full_k[b:b + 1])
            hc.full_v = inputs.bits(cache.full_v[b:b + 1])
        hc.strm_k = inputs.bits(cache.strm_k[b:b + 1])
        hc.strm_v = inputs.bits(cache.strm_v[b:b + 1])
        hc.seq_len = cache.seq_len[b:b + 1].cpu().numpy().astype(np.int32)
        hc.ring_head = cache.ring_head[b:b + 1].cpu().numpy().astype(np.int32)
        ro, rl = oracle.attn_decode(o1, hc, inputs.bits(q[b:b + 1]))
        assert_close(out[b:b + 1], ro.reshape(1, 48, 128), lse[b:b + 1], rl.reshape(1, 48),
                     f"layer {li} sequence {b}")


def test_stack40_graph_replay_matches_eager(cuda_device):
    w = inputs.workload("stack40")
    B, n = 2, 4096
    state = []
    max_ws = 0
    for li in range(w.layers):
        p, _ = layer_of(w, li, B)
        cache = random_cache(p, n, [n, n - 7], [3, 100], seed=900 + li)
        q = inputs.randn_bf16((B, 48, 128), 950 + li, "cuda")
        state.append((p, cache, q, torch.empty((B, 48, 128), dtype=torch.bfloat16, device="cuda"),
                      torch.empty((B, 48), dtype=torch.float32, device="cuda")))
        max_ws = max(max_ws, duo.duo_decode_workspace_bytes(p, n))
    ws = torch.zeros(max_ws, dtype=torch.uint8, device="cuda")

    def step():
        for p, cache, q, out, lse in state:
            duo.duo_attn_decode(p, cache, q, n, out, lse, ws)

    step()
    torch.cuda.synchronize()
    eager = [(s[3].clone(), s[4].clone()) for s in state]
    for s in state:
        s[3].zero_()
        s[4].zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        step()
    g.replay()
    torch.cuda.synchronize()
    assert duo.duo_get_device_status() == duo.DUO_OK
    for (o_e, l_e), s in zip(eager, state):
        assert torch.equal(o_e, s[3]) and torch.equal(l_e, s[4])
