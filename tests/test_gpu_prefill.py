"""duo_attn_prefill (tcgen05 kernel) on the GPU against the float64 oracle.

Outputs: max-abs 2e-2, mean-abs 2e-3; LSE 1e-3.  Small sequences compare
every row; the full-size workloads compare a seeded sample of rows that
includes every tile edge and band boundary.  The attended key set of every
row is checked exactly with uniform attention over one-hot value rows.
"""
import numpy as np
import pytest
import torch

import oracle
import kv_cache_reduction_b200 as duo
from kv_cache_reduction_b200 import inputs

from gpu_helpers import LSE_ABS, assert_close, layers

pytestmark = pytest.mark.gpu


def prefill_gpu(params, q, k, v, dynamic=True):
    """dynamic: CTAs claim work tiles from a counter in a workspace (the path
    the benchmark times); else the static stride over the work list."""
    B, L, Hq, D = q.shape
    out = torch.full((B, L, Hq, D), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((B, Hq, L), float("nan"), dtype=torch.float32, device="cuda")
    ws = None
    if dynamic:
        # stale contents: the call must zero the counter itself
        ws = torch.full((duo.duo_prefill_workspace_bytes(),), 0x7f, dtype=torch.uint8, device="cuda")
    duo.duo_attn_prefill(params, q, k, v, out, lse, workspace=ws)
    torch.cuda.synchronize()
    assert duo.duo_get_device_status() == duo.DUO_OK
    return out, lse


def make_qkv(B, L, seed, hkv=8, rmsnorm=False):
    q = inputs.randn_bf16((B, L, 6 * hkv, 128), seed, "cuda")
    k = inputs.randn_bf16((B, L, hkv, 128), seed + 1, "cuda")
    v = inputs.randn_bf16((B, L, hkv, 128), seed + 2, "cuda")
    if rmsnorm:
        q, k = inputs.rmsnorm_bf16(q), inputs.rmsnorm_bf16(k)
    return q, k, v


def sample_rows(B, Hq, L, n_random, seed):
    """Row ids (b*Hq + h)*L + i over every head, for positions at tile edges,
    band boundaries and a seeded random set."""
    edges = {0, 1, 2, 63, 64, 65, 127, 128, 129, 255, 256, 257, 319, 320, 321, 383, 384, 511, 512,
             513, 639, 640, L // 2, L - 129, L - 128, L - 2, L - 1}
    rng = np.random.default_rng(seed)
    pos = sorted({p for p in edges if 0 <= p < L} | set(rng.integers(0, L, size=n_random).tolist()))
    rows = [(b * Hq + h) * L + i for b in range(B) for h in range(Hq) for i in pos]
    return np.asarray(rows, dtype=np.int64), pos


def compare_rows(out, lse, ref_o, ref_l, rows, B, Hq, L, what):
    r = torch.as_tensor(rows)
    i, h, b = r % L, (r // L) % Hq, r // L // Hq
    got_o = out[b, i, h].float().cpu().numpy()
    got_l = lse[b, h, i].cpu().numpy()
    return assert_close(torch.from_numpy(got_o), ref_o, torch.from_numpy(got_l), ref_l, what)


@pytest.mark.parametrize("dynamic", [True, False])
@pytest.mark.parametrize("L", [1, 5, 127, 128, 129, 300, 321, 600])
def test_prefill_duo_layer_all_rows(cuda_device, L, dynamic):
    B = 2
    p, o = layers(B, full_mask=(1, 0, 0, 1, 0, 1, 1, 0))
    q, k, v = make_qkv(B, L, 40)
    out, lse = prefill_gpu(p, q, k, v, dynamic)
    ref_o, ref_l = oracle.attn_prefill(o, inputs.bits(q), inputs.bits(k), inputs.bits(v))
    got_o = out.permute(0, 2, 1, 3).reshape(-1, 128)
    assert_close(got_o, ref_o, lse.reshape(-1), ref_l, f"L={L}")


@pytest.mark.parametrize("L", [7, 512, 513, 700, 1100])
def test_prefill_sliding_layer_with_sink_all_rows(cuda_device, L):
    B = 2
    sig = inputs.randn_f32((48,), 41)
    p, o = layers(B, window=512, sink_logit=sig)
    q, k, v = make_qkv(B, L, 42, rmsnorm=True)
    out, lse = prefill_gpu(p, q, k, v)
    ref_o, ref_l = oracle.attn_prefill(o, inputs.bits(q), inputs.bits(k), inputs.bits(v))
    assert_close(out.permute(0, 2, 1, 3).reshape(-1, 128), ref_o, lse.reshape(-1), ref_l, f"L={L}")


@pytest.mark.parametrize("cfg", [dict(sink=0, recent=100), dict(sink=200, recent=50),
                                 dict(sink=64, recent=256, window=0), dict(window=64),
                                 dict(window=1000), dict(sink=5, recent=1)])
def test_prefill_other_band_shapes(cuda_device, cfg):
    B, L = 1, 777
    kw = dict(sink=cfg.get("sink", 64), recent=cfg.get("recent", 256), window=cfg.get("window", 0))
    p, o = layers(B, full_mask=(0, 1, 0, 0, 0, 0, 0, 0), **kw)
    q, k, v = make_qkv(B, L, 43)
    out, lse = prefill_gpu(p, q, k, v)
    ref_o, ref_l = oracle.attn_prefill(o, inputs.bits(q), inputs.bits(k), inputs.bits(v))
    assert_close(out.permute(0, 2, 1, 3).reshape(-1, 128), ref_o, lse.reshape(-1), ref_l, str(cfg))


def test_prefill_attended_sets_exact(cuda_device):
    """q = 0: every attended key weighs 1/|S|.  V rows carry one-hot codes of
    their position within a 128-key chunk (zero outside the chunk), so
    O[i, d] * |S_i| is 1 exactly when key chunk*128 + d is attended by row i."""
    B, L = 1, 700
    for kw in (dict(full_mask=(1, 0, 0, 0, 0, 0, 0, 0)), dict(window=512)):
        p, o = layers(B, **kw)
        q = torch.zeros((B, L, 48, 128), dtype=torch.bfloat16, device="cuda")
        k = inputs.randn_bf16((B, L, 8, 128), 44, "cuda")
        for chunk in range((L + 127) // 128):
            pos = torch.arange(L, device="cuda")
            code = torch.zeros((L, 128), device="cuda")
            sel = (pos // 128) == chunk
            code[sel, pos[sel] % 128] = 1.0
            v = code.to(torch.bfloat16)[None, :, None, :].expand(B, L, 8, 128).contiguous()
            out, lse = prefill_gpu(p, q, k, v)
            ref_o, ref_l = oracle.attn_prefill(o, inputs.bits(q), inputs.bits(k), inputs.bits(v))
            size = np.exp(ref_l)                                   # |S| per row
            got = out.permute(0, 2, 1, 3).reshape(-1, 128).float().cpu().numpy() * size[:, None]
            want = ref_o * size[:, None]
            assert np.all(np.isin(np.round(want), [0.0, 1.0]))
            assert np.array_equal(np.round(got), np.round(want)), f"{kw} chunk {chunk}"
            assert np.abs(lse.reshape(-1).cpu().numpy() - ref_l).max() <= LSE_ABS


def test_prefill_schedules_give_identical_bytes(cuda_device):
    """A work tile's result does not depend on which CTA computes it, so the
    static and the dynamic schedule (and repeated dynamic runs) agree bit for
    bit; 4000 tokens give 32 query tiles x 48 pairs, several per CTA."""
    B, L = 2, 4000
    p, _ = layers(B, full_mask=(0, 0, 1, 0, 0, 1, 0, 0))
    q, k, v = make_qkv(B, L, 46)
    o_s, l_s = prefill_gpu(p, q, k, v, dynamic=False)
    for _ in range(2):
        o_d, l_d = prefill_gpu(p, q, k, v, dynamic=True)
        assert torch.equal(o_s, o_d) and torch.equal(l_s, l_d)


def test_prefill_workspace_too_small_is_refused(cuda_device):
    p, _ = layers(1, full_mask=(1,) * 8)
    q, k, v = make_qkv(1, 64, 47)
    out = torch.zeros_like(q)
    small = torch.zeros(duo.duo_prefill_workspace_bytes() - 1, dtype=torch.uint8, device="cuda")
    with pytest.raises(duo.DuoError) as e:
        duo.duo_attn_prefill(p, q, k, v, out, None, workspace=small)
    assert e.value.code == duo.DUO_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.all(out == 0)


def test_prefill_zero_length_is_noop(cuda_device):
    p, _ = layers(1, full_mask=(1,) * 8)
    q, k, v = make_qkv(1, 4, 45)
    out = torch.zeros((1, 4, 48, 128), dtype=torch.bfloat16, device="cuda")
    duo.duo_attn_prefill(p, q, k, v, out, None, seq_len=0)
    torch.cuda.synchronize()
    assert torch.all(out == 0)


@pytest.mark.slow
def test_prefill_16k_workload_sampled(cuda_device):
    w = inputs.workload("prefill_16k")
    p, o = layers(w.batch, full_mask=w.full_mask)
    q, k, v = make_qkv(w.batch, w.seq_len, w.seed)
    out, lse = prefill_gpu(p, q, k, v)
    rows, _ = sample_rows(w.batch, 48, w.seq_len, 40, w.seed)
    ref_o, ref_l = oracle.attn_prefill(o, inputs.bits(q), inputs.bits(k), inputs.bits(v), rows=rows)
    compare_rows(out, lse, ref_o, ref_l, rows, w.batch, 48, w.seq_len, "prefill_16k")
    # every row finite
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()


@pytest.mark.slow
def test_sliding_32k_workload_sampled(cuda_device):
    w = inputs.workload("sliding_32k")
    sig = inputs.randn_f32((48,), w.seed + 9)
    p, o = layers(w.batch, window=w.window, sink_logit=sig)
    q, k, v = make_qkv(w.batch, w.seq_len, w.seed, rmsnorm=True)
    out, lse = prefill_gpu(p, q, k, v)
    rows, _ = sample_rows(w.batch, 48, w.seq_len, 200, w.seed)
    ref_o, ref_l = oracle.attn_prefill(o, inputs.bits(q), inputs.bits(k), inputs.bits(v), rows=rows)
    compare_rows(out, lse, ref_o, ref_l, rows, w.batch, 48, w.seq_len, "sliding_32k")
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()


@pytest.mark.parametrize("mode", ["per_element", "per_head"])
@pytest.mark.parametrize("L", [129, 300])
def test_prefill_output_gate(cuda_device, mode, L):
    """out * sigmoid(g) fused into the epilogue, against the oracle's gate."""
    B = 2
    p, o = layers(B, full_mask=(1, 0, 0, 1, 0, 1, 1, 0))
    q, k, v = make_qkv(B, L, 48)
    shape = (B, L, 48, 128) if mode == "per_element" else (B, L, 48)
    g = (inputs.randn_f32(shape, 49) * 2.5).to("cuda", torch.bfloat16)
    out = torch.full((B, L, 48, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, 48, L), dtype=torch.float32, device="cuda")
    ws = torch.empty(duo.duo_prefill_workspace_bytes(), dtype=torch.uint8, device="cuda")
    duo.duo_attn_prefill(p, q, k, v, out, lse, workspace=ws, gate=g)
    torch.cuda.synchronize()
    assert duo.duo_get_device_status() == duo.DUO_OK
    ref_o, ref_l = oracle.attn_prefill(o, inputs.bits(q), inputs.bits(k), inputs.bits(v))
    gm = oracle.GATE_PER_ELEMENT if mode == "per_element" else oracle.GATE_PER_HEAD
    ref_g = oracle.gate_prefill(ref_o, inputs.bits(g), gm, L, 48)
    assert_close(out.permute(0, 2, 1, 3).reshape(-1, 128), ref_g, lse.reshape(-1), ref_l, mode)
