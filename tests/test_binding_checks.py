"""The binding's checks of what plain pointers cannot carry (dtype, shape,
contiguity, device), on CPU: each call below is rejected with ValueError
before it reaches the library, so no kernel runs and nothing is launched.
The dtype and shape rules are tested with the device rule stubbed out (host
tensors stand in for device ones) and a fake library that fails if reached;
the device rule is tested on its own."""
import pytest
import torch

import kv_cache_reduction_b200 as duo

BF = torch.bfloat16


class _Reached(Exception):
    pass


class _FakeLib:
    def __getattr__(self, name):
        def call(*args):
            raise _Reached(name)
        return call


@pytest.fixture
def host_as_device(monkeypatch):
    def contiguous_only(t, name):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    monkeypatch.setattr(duo, "_on_device", contiguous_only)
    monkeypatch.setattr(duo, "load_library", lambda *a, **k: _FakeLib())


def _layer(B=2):
    return duo.DuoParams(B, full_mask=(1, 0, 0, 1, 0, 1, 1, 0))


def _cache(p, cap=64, device="cpu"):
    return duo.DuoCache.allocate(p, cap, device=device)


def test_host_tensors_are_rejected_before_the_library():
    p = _layer()
    q = torch.zeros((2, 16, 48, 128), dtype=BF)
    k = torch.zeros((2, 16, 8, 128), dtype=BF)
    with pytest.raises(ValueError, match="CUDA tensor"):
        duo.duo_attn_prefill(p, q, k, k, torch.zeros_like(q), None)
    with pytest.raises(ValueError, match="CUDA tensor"):
        duo.duo_kv_append(p, _cache(p), k, k)


@pytest.mark.parametrize("case", ["q dtype", "k heads", "out length", "lse layout", "v batch"])
def test_prefill_shapes_and_dtypes(host_as_device, case):
    p = _layer()
    q = torch.zeros((2, 16, 48, 128), dtype=BF)
    k = torch.zeros((2, 16, 8, 128), dtype=BF)
    v = torch.zeros((2, 16, 8, 128), dtype=BF)
    out = torch.zeros_like(q)
    lse = torch.zeros((2, 48, 16))
    if case == "q dtype":
        q = q.float()
    elif case == "k heads":
        k = torch.zeros((2, 16, 6, 128), dtype=BF)
    elif case == "out length":
        out = torch.zeros((2, 15, 48, 128), dtype=BF)
    elif case == "lse layout":
        lse = torch.zeros((2, 16, 48))
    elif case == "v batch":
        v = torch.zeros((1, 16, 8, 128), dtype=BF)
    with pytest.raises(ValueError):
        duo.duo_attn_prefill(p, q, k, v, out, lse)


def test_prefill_well_formed_arguments_reach_the_library(host_as_device):
    p = _layer()
    q = torch.zeros((2, 16, 48, 128), dtype=BF)
    k = torch.zeros((2, 16, 8, 128), dtype=BF)
    with pytest.raises(_Reached, match="duo_attn_prefill"):
        duo.duo_attn_prefill(p, q, k, k, torch.zeros_like(q), torch.zeros((2, 48, 16)),
                             workspace=torch.zeros(16, dtype=torch.uint8),
                             gate=torch.zeros((2, 16, 48), dtype=BF), stream=0)
    with pytest.raises(_Reached):               # an empty prompt passes seq_len 0
        duo.duo_attn_prefill(p, q, k, k, torch.zeros_like(q), None, seq_len=0, stream=0)


def test_prefill_seq_len_must_be_q_length_or_zero(host_as_device):
    p = _layer()
    q = torch.zeros((2, 16, 48, 128), dtype=BF)
    k = torch.zeros((2, 16, 8, 128), dtype=BF)
    with pytest.raises(ValueError, match="seq_len"):
        duo.duo_attn_prefill(p, q, k, k, torch.zeros_like(q), None, seq_len=8)


def test_non_contiguous_tensors_are_rejected(host_as_device):
    p = _layer()
    q = torch.zeros((2, 48, 16, 128), dtype=BF).transpose(1, 2)      # [2][16][48][128], strided
    k = torch.zeros((2, 16, 8, 128), dtype=BF)
    with pytest.raises(ValueError, match="contiguous"):
        duo.duo_attn_prefill(p, q, k, k, torch.zeros((2, 16, 48, 128), dtype=BF), None)


def test_append_shapes(host_as_device):
    p = _layer()
    cache = _cache(p)
    k = torch.zeros((2, 4, 8, 128), dtype=BF)
    with pytest.raises(ValueError, match="shape"):
        duo.duo_kv_append(p, cache, k, k, n_new=3)          # the rows must be exactly n_new
    with pytest.raises(ValueError, match="shape"):
        duo.duo_kv_append(p, cache, k, torch.zeros((2, 4, 8, 64), dtype=BF))
    with pytest.raises(_Reached, match="duo_kv_append"):
        duo.duo_kv_append(p, cache, k, k, stream=0)


def test_cache_geometry_is_checked_against_the_layer(host_as_device):
    p = _layer()
    cache = _cache(p)
    cache.seq_len = torch.zeros((3,), dtype=torch.int32)              # wrong batch
    with pytest.raises(ValueError, match="seq_len"):
        cache.as_c(p)
    cache = _cache(p)
    cache.strm_k = torch.zeros((2, 4, 64, 128), dtype=BF)            # 64 slots, not sink + recent
    with pytest.raises(ValueError, match="strm_k"):
        cache.as_c(p)
    cache = _cache(p)
    cache.full_v = cache.full_v.float()
    with pytest.raises(ValueError, match="full_v"):
        cache.as_c(p)


def test_decode_accepts_both_one_token_layouts_and_checks_them(host_as_device):
    p = _layer()
    for q in (torch.zeros((2, 48, 128), dtype=BF), torch.zeros((2, 1, 48, 128), dtype=BF)):
        lse = torch.zeros(q.shape[:-1])
        with pytest.raises(_Reached, match="duo_attn_decode"):
            duo.duo_attn_decode(p, _cache(p), q, 10, torch.zeros_like(q), lse,
                                torch.zeros(256, dtype=torch.uint8), stream=0)
        with pytest.raises(_Reached, match="duo_attn_decode_static"):
            duo.duo_attn_decode_static(p, _cache(p), q, 10, torch.zeros_like(q), lse, stream=0)
    with pytest.raises(ValueError, match="shape"):
        duo.duo_attn_decode(p, _cache(p), torch.zeros((2, 2, 48, 128), dtype=BF), 10,
                            torch.zeros((2, 2, 48, 128), dtype=BF), None, torch.zeros(256, dtype=torch.uint8))


def test_block_decode_shapes(host_as_device):
    p = _layer()
    q = torch.zeros((2, 4, 48, 128), dtype=BF)
    kv = torch.zeros((2, 3, 8, 128), dtype=BF)                      # block of 3 keys for 4 queries
    with pytest.raises(ValueError, match="k_new"):
        duo.duo_attn_decode_block(p, _cache(p), q, kv, kv, 10, torch.zeros_like(q), None,
                                  torch.zeros(256, dtype=torch.uint8))
    kv = torch.zeros((2, 4, 8, 128), dtype=BF)
    with pytest.raises(_Reached, match="duo_attn_decode_block"):
        duo.duo_attn_decode_block(p, _cache(p), q, kv, kv, 10, torch.zeros_like(q),
                                  torch.zeros((2, 4, 48)), torch.zeros(256, dtype=torch.uint8), stream=0)


def test_sink_logit_and_norm_weights(host_as_device):
    p = duo.DuoParams(1, window=512, sink_logit=torch.zeros((47,)))
    with pytest.raises(ValueError, match="sink_logit"):
        p.as_c()
    with pytest.raises(ValueError, match="q_norm_weight"):
        duo.DuoQKPrep(q_norm_weight=torch.zeros((128,))).as_c()       # fp32, not bf16


def test_prep_defaults_are_the_page_rope_parameters():
    import json
    import os
    rope = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_constants.json")))[
        "rope_full_attention"]["value"]
    d = duo.DuoQKPrep()
    assert (d.rope_theta, d.rope_factor, d.original_max_position, d.beta_fast, d.beta_slow,
            d.attention_factor) == (rope["rope_theta"], rope["factor"],
                                    rope["original_max_position_embeddings"], rope["beta_fast"],
                                    rope["beta_slow"], rope["attention_factor"])
