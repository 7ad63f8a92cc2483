"""The roofline numerators bench.py reports, pinned to the oracle's attended-set
rule: prefill FLOPs count 4 * 128 per attended (query, key) pair and query head,
decode bytes count each attended K/V row once per KV head.  The pair counts come
from the oracle (brute force over its per-pair rule for small L, its cumulative
count for large L), never from the closed form under test."""
import pytest

import bench
import oracle
from kv_cache_reduction_b200 import inputs


def _layer(kind: str) -> oracle.Layer:
    if kind == "full":
        return oracle.Layer(1, 6, 1, 128, inputs.SINK, inputs.RECENT, 0, full_mask=(1,))
    if kind == "streaming":
        return oracle.Layer(1, 6, 1, 128, inputs.SINK, inputs.RECENT, 0, full_mask=(0,))
    return oracle.Layer(1, 6, 1, 128, 0, 0, inputs.WINDOW, full_mask=(0,))


def _span(kind: str):
    return {"full": None, "streaming": inputs.SINK + inputs.RECENT, "sliding": inputs.WINDOW}[kind]


@pytest.mark.parametrize("kind", ["full", "streaming", "sliding"])
@pytest.mark.parametrize("L", [1, 2, 63, 64, 65, 255, 256, 319, 320, 321, 511, 512, 513, 700])
def test_pair_count_matches_brute_force_over_the_oracle_rule(kind, L):
    layer = _layer(kind)
    if L <= 321:
        brute = sum(oracle.attended(layer, 0, i, j) for i in range(L) for j in range(L))
    else:
        brute = oracle.count_pairs(layer, 0, L)
    assert bench.attended_pairs(L, _span(kind)) == brute


@pytest.mark.parametrize("kind", ["full", "streaming", "sliding"])
@pytest.mark.parametrize("L", [16384, 32768])
def test_pair_count_matches_the_oracle_at_workload_lengths(kind, L):
    assert bench.attended_pairs(L, _span(kind)) == oracle.count_pairs(_layer(kind), 0, L)


def test_prefill_flops_of_the_two_prefill_workloads():
    # prefill_16k: 12 query heads on full KV heads, 36 on streaming ones, B=1
    w = inputs.workload("prefill_16k")
    assert sum(w.full_mask) == 2
    full = oracle.count_pairs(_layer("full"), 0, w.seq_len)
    strm = oracle.count_pairs(_layer("streaming"), 0, w.seq_len)
    assert bench.prefill_flops(w) == 4 * 128 * (12 * full + 36 * strm) * w.batch
    assert bench.prefill_flops(w) == pytest.approx(920.38e9, rel=1e-5)
    # sliding_32k: all 48 query heads on the 512-key band, B=2
    w = inputs.workload("sliding_32k")
    band = oracle.count_pairs(_layer("sliding"), 0, w.seq_len)
    assert bench.prefill_flops(w) == 4 * 128 * 48 * band * w.batch
    assert bench.prefill_flops(w) == pytest.approx(818.20e9, rel=1e-5)


@pytest.mark.parametrize("n", [1, 63, 64, 320, 321, 1000, 32768])
def test_decode_bytes_count_the_last_rows_attended_keys(n):
    # keys the decode query (position n - 1) attends: the oracle's cumulative
    # pair count at n minus the one at n - 1
    def last_row(kind):
        layer = _layer(kind)
        return oracle.count_pairs(layer, 0, n) - (oracle.count_pairs(layer, 0, n - 1) if n > 1 else 0)

    B, n_full, n_ring = 3, 2, 6
    rows = B * (n_full * last_row("full") + n_ring * last_row("streaming"))
    q_out = 2 * B * 48 * 128 * 2
    assert bench.decode_bytes(B, n, n_full, n_ring) == rows * 512 + q_out


def test_decode_bytes_of_the_main_workload():
    w = inputs.workload("decode_b32")
    assert sum(w.full_mask) == 2
    assert bench.decode_bytes(w.batch, w.seq_len, 2, 6) == 1_105_985_536


@pytest.mark.parametrize("L", range(1, 14))
@pytest.mark.parametrize("sink,recent,window", [(2, 3, 0), (0, 1, 0), (3, 1, 0), (0, 0, 4), (0, 0, 1)])
def test_pair_count_matches_brute_force_with_small_spans(L, sink, recent, window):
    # every band edge is crossed within L <= 13
    layer = oracle.Layer(1, 6, 1, 128, sink, recent, window, full_mask=(0,))
    brute = sum(oracle.attended(layer, 0, i, j) for i in range(L) for j in range(L))
    span = window if window else sink + recent
    assert bench.attended_pairs(L, span) == brute


def _block_union(layer: oracle.Layer, n: int, q_len: int) -> int:
    """Keys that any query of a block at positions n .. n + q_len - 1 attends,
    by brute force over the oracle's per-pair rule."""
    keys = set()
    for t in range(q_len):
        i = n + t
        keys.update(j for j in range(i + 1) if oracle.attended(layer, 0, i, j))
    return len(keys)


@pytest.mark.parametrize("n", [1, 2, 3, 5, 7, 9, 12, 20])
@pytest.mark.parametrize("q_len", [1, 3, 8])
@pytest.mark.parametrize("sink,recent", [(2, 3), (0, 4), (3, 1), (0, 1)])
def test_verify_ring_rows_match_the_union_of_the_blocks_bands(n, q_len, sink, recent):
    layer = oracle.Layer(1, 6, 1, 128, sink, recent, 0, full_mask=(0,))
    # the union holds the cached keys plus all q_len keys of the block itself
    assert bench.block_ring_rows(n, sink, recent) + q_len == _block_union(layer, n, q_len)


def test_verify_bytes_of_the_verify_workload():
    w = inputs.workload("decode_b32")
    n, q_len = w.seq_len, 8
    ring = _block_union(_layer("streaming"), n, q_len) - q_len
    assert ring == inputs.SINK + inputs.RECENT - 1
    rows = w.batch * (2 * n + 6 * ring) + w.batch * 8 * q_len
    assert bench.verify_bytes(w.batch, n, q_len, 2, 6) == rows * 512 + 2 * w.batch * q_len * 48 * 128 * 2


def test_stack_bytes_of_the_forty_layer_step():
    w = inputs.workload("stack40")
    n = w.seq_len

    def last_row(kind):          # keys the query at position n - 1 attends
        layer = _layer(kind)
        return sum(oracle.attended(layer, 0, n - 1, j) for j in range(n))

    per_full_layer = w.batch * (2 * last_row("full") + 6 * last_row("streaming")) * 512
    per_sliding_layer = w.batch * 8 * last_row("sliding") * 512
    q_out = 2 * w.batch * 48 * 128 * 2
    masks = inputs.stack_layer_masks(w)
    assert sum(m is None for m in masks) == 30 and all(sum(m) == 2 for m in masks if m is not None)
    want = 10 * per_full_layer + 30 * per_sliding_layer + 40 * q_out
    assert bench.stack_bytes(w) == want
    assert want == pytest.approx(22.65e9, rel=1e-3)


def test_timed_sample_cycles_until_the_budget():
    import time
    ran = []

    def run(u):
        ran.append(u)
        time.sleep(0.002)

    units = ["a", "b", "c"]
    done, t, used = bench.timed_sample(units, run, lambda u: 10, 0.025)
    assert t >= 0.025 and used == len(ran) and done == 10 * used
    assert used > len(units)                                   # cycled past one pass
    assert ran[:6] == ["a", "b", "c", "a", "b", "c"]
    # a budget below one unit still runs one unit; the pass limit caps the rest
    assert bench.timed_sample(units, lambda u: None, lambda u: 1, 0.0)[2] == 1
    assert bench.timed_sample(units, lambda u: None, lambda u: 1, 1e9, max_passes=2)[2] == 6


def test_decode_cpu_baseline_leg_runs_on_host_tensors():
    """The bench's CPU-baseline leg of the main line, driven on small host
    tensors (the leg reads the caches back to the host, so it needs no GPU):
    it runs the oracle over whole decode steps (every row of the batch per
    call) until its budget and reports bytes per second."""
    import types
    import torch
    import kv_cache_reduction_b200 as duo

    wl = object.__new__(bench.DecodeB32)
    n = 700
    wl.w = types.SimpleNamespace(seq_len=n)
    wl.params = duo.DuoParams(2, full_mask=(0, 0, 0, 0, 0, 1, 0, 1))
    wl.cache = duo.DuoCache.allocate(wl.params, n, device="cpu")
    for i, t in enumerate((wl.cache.full_k, wl.cache.full_v, wl.cache.strm_k, wl.cache.strm_v)):
        t.copy_(inputs.randn_bf16(tuple(t.shape), 50 + i, "cpu"))
    wl.cache.seq_len.fill_(n)
    wl.cache.ring_head.copy_(torch.tensor([3, 200], dtype=torch.int32))
    wl.q = inputs.randn_bf16((2, 48, 128), 60, "cpu")
    r = wl.oracle_sample(0.3)
    assert r["kind"] == "oracle" and r["unit"] == "GB/s" and r["value"] > 0
    assert "whole decode steps (96 rows per call" in r["sample"]
    used = int(r["sample"].split()[0])
    assert used >= 1
    assert r["threads_busy"] == min(r["cores"], 2 * 2 * 6)


def test_decode_small_cpu_baseline_leg_runs_on_host_tensors():
    """The config-1 line's CPU leg on small host tensors: the oracle's prefill
    of the prompt, then append + decode steps, timed per step."""
    import torch
    import kv_cache_reduction_b200 as duo

    wl = object.__new__(bench.DecodeSmall)
    wl.STEPS = 3
    L = 40
    wl.params = duo.DuoParams(1, full_mask=(1, 0, 0, 1, 0, 1, 1, 0))
    wl.cap = L + wl.STEPS
    wl.qp = inputs.randn_bf16((1, L, 48, 128), 70, "cpu")
    wl.kp = inputs.randn_bf16((1, L, 8, 128), 71, "cpu")
    wl.vp = inputs.randn_bf16((1, L, 8, 128), 72, "cpu")
    wl.k1 = inputs.randn_bf16((wl.STEPS, 1, 1, 8, 128), 73, "cpu")
    wl.v1 = inputs.randn_bf16((wl.STEPS, 1, 1, 8, 128), 74, "cpu")
    wl.q1 = inputs.randn_bf16((wl.STEPS, 1, 48, 128), 75, "cpu")
    r = wl.oracle_sample(0.05)
    assert r["kind"] == "oracle" and r["unit"] == "us/step" and r["value"] > 0 and r["prefill_us"] > 0
    assert r["sample"].split()[0].isdigit()
