"""The C ABI library loads, exports every declared symbol, and rejects bad
arguments on the host before touching a device (CPU only, no kernel runs)."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

import kv_cache_reduction_b200 as duo
from kv_cache_reduction_b200 import build as duo_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include"))
           if f.endswith(".h")]


@pytest.fixture(scope="module")
def lib():
    duo_build.build()
    return duo.load_library()


def declared_functions():
    names = []
    for h in HEADERS:
        text = open(h).read()
        names += re.findall(r"DUO_API\s+[\w\s\*]+?\b(duo_\w+)\s*\(", text)
    return names


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("duo_kv_append", "duo_attn_prefill", "duo_attn_decode", "duo_decode_workspace_bytes",
              "duo_get_device_status", "duo_status_string", "duo_last_error"):
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(duo.EXPORTED) <= set(declared_functions())


def test_library_exports_nothing_else(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", duo.LIBRARY_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    ours = {n for n in exported if n.startswith("duo_")}
    assert ours == set(declared_functions())


def test_library_has_no_gpu_driver_dependency(lib):
    out = subprocess.run(["ldd", duo.LIBRARY_PATH], capture_output=True, text=True).stdout
    assert "libcuda.so" not in out and "libtorch" not in out


def test_status_strings(lib):
    for code in range(0, -8, -1):
        assert duo.duo_status_string(code) not in ("", "unknown status")
    assert duo.duo_status_string(-99) == "unknown status"


def test_testing_hook_checks_its_arguments(lib):
    """The failure-injection hook (include/duo_attn_testing.h) takes the three
    pipelined kernels and a tile >= -1, and is off again after tile -1."""
    for kernel in (0, 4, -1):
        with pytest.raises(duo.DuoError) as e:
            duo.duo_testing_withhold_tile(kernel, 0)
        assert e.value.code == duo.DUO_ERR_INVALID_ARG
    with pytest.raises(duo.DuoError):
        duo.duo_testing_withhold_tile(duo.DUO_TESTING_PREFILL, -2)
    for kernel in (duo.DUO_TESTING_DECODE, duo.DUO_TESTING_PREFILL, duo.DUO_TESTING_DECODE_BLOCK):
        duo.duo_testing_withhold_tile(kernel, 3)
        duo.duo_testing_withhold_tile(kernel, -1)


def _params(**kw):
    base = dict(batch=2, full_mask=(1, 0, 0, 1, 0, 0, 0, 0))
    base.update(kw)
    return duo.DuoParams(**base)


def _call_append(p, cache=None):
    lib = duo.load_library()
    pc = p.as_c()
    c = cache or duo._Cache(0x1000, 0x1000, 64, 0x1000, 0x1000, 0x1000, 0x1000)
    return lib.duo_kv_append(ctypes.byref(pc), ctypes.byref(c), 0x1000, 0x1000, 1, None)


@pytest.mark.parametrize("kw,code", [
    (dict(head_dim=64), duo.DUO_ERR_UNSUPPORTED),
    (dict(num_q_heads=40), duo.DUO_ERR_UNSUPPORTED),
    (dict(num_kv_heads=65, num_q_heads=390), duo.DUO_ERR_UNSUPPORTED),
    (dict(batch=0), duo.DUO_ERR_INVALID_ARG),
    (dict(softmax_scale=0.0), duo.DUO_ERR_INVALID_ARG),
    (dict(softmax_scale=float("inf")), duo.DUO_ERR_INVALID_ARG),
    (dict(recent=0), duo.DUO_ERR_INVALID_ARG),
    (dict(sink=-1), duo.DUO_ERR_INVALID_ARG),
    (dict(sink=8000, recent=500), duo.DUO_ERR_INVALID_ARG),
    (dict(window=-3), duo.DUO_ERR_INVALID_ARG),
    (dict(window=9000), duo.DUO_ERR_INVALID_ARG),
    (dict(full_mask=(2, 0, 0, 0, 0, 0, 0, 0)), duo.DUO_ERR_INVALID_ARG),
])
def test_bad_params_are_rejected_before_any_launch(lib, kw, code):
    assert _call_append(_params(**kw)) == code
    assert duo.duo_last_error() != ""


def test_bad_pointers_are_rejected(lib):
    p = _params()
    pc = p.as_c()
    ok = dict(full_k=0x1000, full_v=0x1000, capacity=64, strm_k=0x1000, strm_v=0x1000,
              seq_len=0x1000, ring_head=0x1000)
    for key, bad in [("full_k", 0), ("strm_v", 0), ("seq_len", 0), ("full_k", 0x1008),
                     ("capacity", 0), ("ring_head", 0x1002)]:
        c = duo._Cache(**{**ok, key: bad})
        assert lib.duo_kv_append(ctypes.byref(pc), ctypes.byref(c), 0x1000, 0x1000, 1, None) == \
            duo.DUO_ERR_INVALID_ARG, key
    c = duo._Cache(**ok)
    assert lib.duo_kv_append(ctypes.byref(pc), ctypes.byref(c), 0, 0x1000, 1, None) == duo.DUO_ERR_INVALID_ARG
    assert lib.duo_kv_append(ctypes.byref(pc), ctypes.byref(c), 0x1004, 0x1000, 1, None) == duo.DUO_ERR_INVALID_ARG
    assert lib.duo_kv_append(ctypes.byref(pc), ctypes.byref(c), 0x1000, 0x1000, -1, None) == duo.DUO_ERR_INVALID_ARG
    # n_new == 0 is a no-op that touches nothing
    assert lib.duo_kv_append(ctypes.byref(pc), ctypes.byref(c), 0, 0, 0, None) == duo.DUO_OK
    # a null params pointer
    assert lib.duo_kv_append(None, ctypes.byref(c), 0x1000, 0x1000, 1, None) == duo.DUO_ERR_INVALID_ARG


def test_sliding_layer_needs_no_mask_or_full_cache(lib):
    p = duo.DuoParams(batch=1, window=512, full_mask=())
    pc = p.as_c()
    pc.full_mask = None
    c = duo._Cache(None, None, 0, 0x1000, 0x1000, 0x1000, 0x1000)
    rc = lib.duo_kv_append(ctypes.byref(pc), ctypes.byref(c), 0x1000, 0x1000, 1, None)
    # passes every host check; without a GPU the device check then fails
    assert rc in (duo.DUO_ERR_CUDA, duo.DUO_ERR_DEVICE, duo.DUO_OK)
    assert rc != duo.DUO_ERR_INVALID_ARG


def test_decode_argument_checks(lib):
    p = _params()
    pc = p.as_c()
    c = duo._Cache(0x1000, 0x1000, 64, 0x1000, 0x1000, 0x1000, 0x1000)
    call = lambda msl, q=0x1000, out=0x1000, ws=0x1000, wsb=1 << 30: lib.duo_attn_decode(
        ctypes.byref(pc), ctypes.byref(c), q, msl, out, None, ws, wsb, None, None)
    assert call(65) == duo.DUO_ERR_INVALID_ARG      # longer than the capacity
    assert call(-1) == duo.DUO_ERR_INVALID_ARG
    assert call(10, q=0) == duo.DUO_ERR_INVALID_ARG
    assert call(10, out=0x1001) == duo.DUO_ERR_INVALID_ARG


def test_prefill_argument_checks(lib):
    p = _params()
    pc = p.as_c()
    f = lib.duo_attn_prefill
    a = 0x1000
    assert f(ctypes.byref(pc), a, a, a, -5, a, None, None, 0, None, None) == duo.DUO_ERR_INVALID_ARG
    assert f(ctypes.byref(pc), a, 0, a, 16, a, None, None, 0, None, None) == duo.DUO_ERR_INVALID_ARG
    assert f(ctypes.byref(pc), a, a, a, 16, a, 0x1004, None, 0, None, None) == duo.DUO_ERR_INVALID_ARG
    assert f(ctypes.byref(pc), 0, 0, 0, 0, 0, None, None, 0, None, None) == duo.DUO_OK   # empty prefill
    need = duo.duo_prefill_workspace_bytes()
    assert need >= 4
    # a workspace that is too small or misaligned is refused before anything runs
    assert f(ctypes.byref(pc), a, a, a, 16, a, None, 0x2000, need - 1, None, None) == duo.DUO_ERR_WORKSPACE
    assert f(ctypes.byref(pc), a, a, a, 16, a, None, 0x2008, need, None, None) == duo.DUO_ERR_WORKSPACE


def test_gate_argument_checks(lib):
    """A bad output gate is refused on the host before anything runs."""
    p = _params()
    pc = p.as_c()
    a = 0x1000
    f = lib.duo_attn_prefill
    for mode, values in ((3, a), (-1, a), (duo.DUO_GATE_PER_ELEMENT, None),
                         (duo.DUO_GATE_PER_HEAD, 0x1008)):
        g = duo._Gate(mode, values)
        assert f(ctypes.byref(pc), a, a, a, 16, a, None, None, 0, ctypes.byref(g), None) == \
            duo.DUO_ERR_INVALID_ARG, (mode, values)
        c = duo._Cache(a, a, 64, a, a, a, a)
        assert lib.duo_attn_decode(ctypes.byref(pc), ctypes.byref(c), a, 10, a, None, a, 1 << 30,
                                   ctypes.byref(g), None) == duo.DUO_ERR_INVALID_ARG
    # mode NONE ignores the values pointer: the empty prefill still succeeds
    g = duo._Gate(duo.DUO_GATE_NONE, None)
    assert f(ctypes.byref(pc), 0, 0, 0, 0, 0, None, None, 0, ctypes.byref(g), None) == duo.DUO_OK


def test_workspace_size_is_host_arithmetic(lib):
    p = _params(batch=32)
    n = duo.duo_decode_workspace_bytes(p, 32768)
    assert n > 0 and n % 4 == 0
    assert duo.duo_decode_workspace_bytes(p, 64) <= n
    assert duo.duo_decode_workspace_bytes(_params(head_dim=64), 128) == 0


def test_gate_shape_picks_the_mode():
    """The binding reads the gate mode from the gate's shape: out's shape is one
    gate per channel, out's shape without the channel dimension one per head."""
    out = torch.zeros((2, 3, 48, 128), dtype=torch.bfloat16)
    g = duo._gate(torch.zeros_like(out), out)
    assert g._obj.mode == duo.DUO_GATE_PER_ELEMENT
    g = duo._gate(torch.zeros((2, 3, 48), dtype=torch.bfloat16), out)
    assert g._obj.mode == duo.DUO_GATE_PER_HEAD
    assert duo._gate(None, out) is None
    with pytest.raises(ValueError):
        duo._gate(torch.zeros((2, 3, 48, 64), dtype=torch.bfloat16), out)
    with pytest.raises(ValueError):
        duo._gate(torch.zeros((2, 3, 48), dtype=torch.float32), out)
