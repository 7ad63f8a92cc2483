"""Failure detection without a GPU fault: every wait inside the kernels is
bounded.  A test hook (DUO_TEST_WITHHOLD_TILE) makes the first decode CTA's
producer stop issuing copies, so its consumers' waits run out; the kernel
records DUO_ERR_TIMEOUT, returns, and the context stays usable."""
import os

import pytest
import torch

import kv_cache_reduction_b200 as duo
from kv_cache_reduction_b200 import inputs

from gpu_helpers import layers, random_cache

pytestmark = pytest.mark.gpu


def test_expired_wait_reports_timeout_and_context_survives(cuda_device, monkeypatch):
    p, _ = layers(1, full_mask=(1, 0, 0, 0, 0, 0, 0, 0))
    cache = random_cache(p, 300, [300], [0], seed=80)
    q = inputs.randn_bf16((1, 48, 128), 81, "cuda")
    out = torch.empty((1, 48, 128), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((1, 48), dtype=torch.float32, device="cuda")
    ws = duo.workspace_for(p, 300)
    assert duo.duo_get_device_status() == duo.DUO_OK
    monkeypatch.setenv("DUO_TEST_WITHHOLD_TILE", "0")
    duo.duo_attn_decode(p, cache, q, 300, out, lse, ws)
    assert duo.duo_get_device_status() == duo.DUO_ERR_TIMEOUT
    monkeypatch.delenv("DUO_TEST_WITHHOLD_TILE")
    # the next call on the same context runs normally (a timed-out call may
    # leave the workspace's split counters non-zero: zero it again)
    ws.zero_()
    ref = torch.empty_like(out)
    duo.duo_attn_decode(p, cache, q, 300, ref, lse, ws)
    assert duo.duo_get_device_status() == duo.DUO_OK
    assert torch.isfinite(ref.float()).all()
