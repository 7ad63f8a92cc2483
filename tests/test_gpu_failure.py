"""Failure detection without a GPU fault: every wait inside the pipelined
kernels is bounded.  The failure-injection hook (include/duo_attn_testing.h)
makes CTA 0's tile producer of one kernel stop issuing copies, so the waits of
its consumers run out; the kernel records DUO_ERR_TIMEOUT and returns, the
status reads it once, and the next call on the same context computes the right
result again (checked against the oracle)."""
import contextlib

import pytest
import torch

import oracle
import kv_cache_reduction_b200 as duo
from kv_cache_reduction_b200 import inputs

from gpu_helpers import assert_close, host_cache, layers, random_cache

pytestmark = pytest.mark.gpu


@contextlib.contextmanager
def withheld(kernel, tile):
    duo.duo_testing_withhold_tile(kernel, tile)
    try:
        yield
    finally:
        duo.duo_testing_withhold_tile(kernel, -1)


# (batch, context, tile): CTA 0 stops at its first tile, or inside its first
# item (40 sequences at 4096 give items of about 11 tiles)
@pytest.mark.parametrize("B,n,tile", [(1, 700, 0), (40, 4096, 5)])
def test_decode_expired_wait(cuda_device, B, n, tile):
    p, o = layers(B, full_mask=(1, 0, 0, 0, 0, 0, 0, 0))
    cache = random_cache(p, n, [n] * B, [b % 256 for b in range(B)], seed=80)
    q = inputs.randn_bf16((B, 48, 128), 81, "cuda")
    out = torch.empty((B, 48, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, 48), dtype=torch.float32, device="cuda")
    ws = duo.workspace_for(p, n)
    assert duo.duo_get_device_status() == duo.DUO_OK
    with withheld(duo.DUO_TESTING_DECODE, tile):
        duo.duo_attn_decode(p, cache, q, n, out, lse, ws)
        assert duo.duo_get_device_status() == duo.DUO_ERR_TIMEOUT
    assert duo.duo_get_device_status() == duo.DUO_OK          # read once, then cleared
    duo.duo_attn_decode(p, cache, q, n, out, lse, ws)
    assert duo.duo_get_device_status() == duo.DUO_OK
    ro, rl = oracle.attn_decode(o, host_cache(o, cache), inputs.bits(q))
    assert_close(out, ro.reshape(B, 48, 128), lse, rl.reshape(B, 48), "decode after a timeout")


@pytest.mark.parametrize("tile", [0, 3])
def test_prefill_expired_wait(cuda_device, tile):
    B, L = 1, 400
    p, o = layers(B, full_mask=(1, 0, 0, 1, 0, 0, 0, 0))
    q = inputs.randn_bf16((B, L, 48, 128), 82, "cuda")
    k = inputs.randn_bf16((B, L, 8, 128), 83, "cuda")
    v = inputs.randn_bf16((B, L, 8, 128), 84, "cuda")
    out = torch.empty((B, L, 48, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, 48, L), dtype=torch.float32, device="cuda")
    ws = torch.empty(duo.duo_prefill_workspace_bytes(), dtype=torch.uint8, device="cuda")
    with withheld(duo.DUO_TESTING_PREFILL, tile):
        duo.duo_attn_prefill(p, q, k, v, out, lse, workspace=ws)
        assert duo.duo_get_device_status() == duo.DUO_ERR_TIMEOUT
    duo.duo_attn_prefill(p, q, k, v, out, lse, workspace=ws)
    assert duo.duo_get_device_status() == duo.DUO_OK
    ro, rl = oracle.attn_prefill(o, inputs.bits(q), inputs.bits(k), inputs.bits(v))
    assert_close(out.permute(0, 2, 1, 3).reshape(-1, 128), ro, lse.reshape(-1), rl,
                 "prefill after a timeout")


@pytest.mark.parametrize("tile", [0])
def test_decode_block_expired_wait(cuda_device, tile):
    B, q_len, n = 2, 4, 600
    p, o = layers(B, full_mask=(0, 1, 0, 0, 0, 0, 1, 0))
    cache = random_cache(p, n, [n, n - 100], [3, 200], seed=85)
    qb = inputs.randn_bf16((B, q_len, 48, 128), 86, "cuda")
    kb = inputs.randn_bf16((B, q_len, 8, 128), 87, "cuda")
    vb = inputs.randn_bf16((B, q_len, 8, 128), 88, "cuda")
    out = torch.empty((B, q_len, 48, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, q_len, 48), dtype=torch.float32, device="cuda")
    nbytes = duo.duo_decode_block_workspace_bytes(p, q_len, n)
    ws = torch.empty((nbytes + 255) // 256 * 256, dtype=torch.uint8, device="cuda")
    with withheld(duo.DUO_TESTING_DECODE_BLOCK, tile):
        duo.duo_attn_decode_block(p, cache, qb, kb, vb, n, out, lse, ws)
        assert duo.duo_get_device_status() == duo.DUO_ERR_TIMEOUT
    duo.duo_attn_decode_block(p, cache, qb, kb, vb, n, out, lse, ws)
    assert duo.duo_get_device_status() == duo.DUO_OK
    ro, rl = oracle.attn_decode_block(o, host_cache(o, cache), inputs.bits(qb), inputs.bits(kb),
                                      inputs.bits(vb))
    assert_close(out, ro.reshape(B, q_len, 48, 128), lse, rl.reshape(B, q_len, 48),
                 "block decode after a timeout")
