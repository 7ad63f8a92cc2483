"""duo_attn_decode_static: decode without a caller workspace.

Some callers cannot allocate device memory when they decode (an engine plugin
that must not allocate inside its execute hook, a server working within a
fixed memory budget, a latency-critical loop that cannot afford cudaMalloc's
device-wide synchronisation).  This entry point keeps its split partials in a
fixed 16 MiB array inside the library instead.  Here it must give the same
output as duo_attn_decode with a workspace, on two calls in a row (the array
keeps the previous call's contents), and it must refuse a layer whose
partials do not fit without launching anything.

This file is collected last so that a failure here cannot hide the others.
"""
import ctypes

import pytest
import torch

import kv_cache_reduction_b200 as duo
from kv_cache_reduction_b200 import inputs

from gpu_helpers import LSE_ABS, MAX_ABS, MEAN_ABS, layers, random_cache

pytestmark = pytest.mark.gpu


def _close(a, b, la, lb):
    err = (a.float() - b.float()).abs()
    assert err.max().item() <= MAX_ABS and err.mean().item() <= MEAN_ABS
    fin = torch.isfinite(lb)
    assert torch.equal(torch.isfinite(la), fin)
    assert (la[fin] - lb[fin]).abs().max().item() <= LSE_ABS


def test_static_scratch_decode_matches_workspace_decode(cuda_device):
    B = 4
    p, _ = layers(B, full_mask=inputs.seeded_full_mask(2002, 2))
    seq = [5000, 1, 321, 4000]
    cache = random_cache(p, 5000, seq, [0, 0, 17, 255], seed=70)
    q = inputs.randn_bf16((B, 48, 128), 71, "cuda")
    out_ref = torch.empty((B, 48, 128), dtype=torch.bfloat16, device="cuda")
    lse_ref = torch.empty((B, 48), dtype=torch.float32, device="cuda")
    duo.duo_attn_decode(p, cache, q, 5000, out_ref, lse_ref, duo.workspace_for(p, 5000))
    torch.cuda.synchronize()
    for call in range(2):
        out = torch.full((B, 48, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.full((B, 48), float("nan"), dtype=torch.float32, device="cuda")
        duo.duo_attn_decode_static(p, cache, q, 5000, out, lse)
        torch.cuda.synchronize()
        assert duo.duo_get_device_status() == duo.DUO_OK
        _close(out, out_ref, lse, lse_ref)


def test_static_scratch_decode_sliding_layer_twice(cuda_device):
    B = 3
    sig = inputs.randn_f32((48,), 72)
    p, _ = layers(B, window=512, sink_logit=sig)
    cache = random_cache(p, 1, [900, 40, 512], [100, 40, 0], seed=73)
    out_ref = torch.empty((B, 48, 128), dtype=torch.bfloat16, device="cuda")
    lse_ref = torch.empty((B, 48), dtype=torch.float32, device="cuda")
    for call in range(2):
        q = inputs.randn_bf16((B, 48, 128), 74 + call, "cuda")
        duo.duo_attn_decode(p, cache, q, 900, out_ref, lse_ref, duo.workspace_for(p, 900))
        out = torch.empty_like(out_ref)
        lse = torch.empty_like(lse_ref)
        duo.duo_attn_decode_static(p, cache, q, 900, out, lse)
        torch.cuda.synchronize()
        _close(out, out_ref, lse, lse_ref)


def test_static_scratch_rejects_layers_that_do_not_fit(cuda_device):
    """A batch whose partials need more than 16 MiB is refused on the host;
    the cache pointers are never touched because nothing is launched."""
    p = duo.DuoParams(1024, full_mask=(1,) * 8)
    need = duo.duo_decode_workspace_bytes(p, 4096)
    assert need > 16 << 20
    fake = duo._Cache(0x10000, 0x10000, 4096, None, None, 0x10000, 0x10000)
    lib = duo.load_library()
    pc = p.as_c()
    rc = lib.duo_attn_decode_static(ctypes.byref(pc), ctypes.byref(fake), 0x10000, 4096, 0x10000,
                                    None, None, None)
    assert rc == duo.DUO_ERR_WORKSPACE
    assert str(need) in duo.duo_last_error()
