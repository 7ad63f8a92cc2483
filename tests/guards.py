"""Guard regions around device buffers, the out-of-bounds write check the GPU
parity tests use in place of a memory checker.

Every buffer handed out is a view into a larger byte allocation with GUARD
bytes of a fixed pattern on each side.  After a call, check() asserts that
both sides still hold the pattern, so a kernel that wrote one element past the
end of its output, cache or workspace (or before its start) fails the test.
The view starts GUARD bytes into the allocation, which keeps the 256-byte
alignment the library asks of workspaces."""
from __future__ import annotations

import math

import torch

import kv_cache_reduction_b200 as duo

GUARD = 4096
PATTERN = 0xA5


class Guarded:
    def __init__(self, device="cuda"):
        self.device = device
        self.bufs = []

    def empty(self, shape, dtype, name: str, fill=None) -> torch.Tensor:
        elem = torch.empty((), dtype=dtype).element_size()
        nbytes = math.prod(shape) * elem
        raw = torch.full((GUARD + nbytes + GUARD,), PATTERN, dtype=torch.uint8, device=self.device)
        view = raw[GUARD:GUARD + nbytes].view(dtype).view(tuple(shape))
        if fill is not None:
            view.fill_(fill)
        self.bufs.append((name, raw, nbytes))
        return view

    def like(self, t: torch.Tensor, name: str) -> torch.Tensor:
        """A guarded copy of t."""
        g = self.empty(t.shape, t.dtype, name)
        g.copy_(t)
        return g

    def cache(self, params: duo.DuoParams, capacity: int, name: str = "cache") -> duo.DuoCache:
        """A duo.DuoCache whose every tensor is guarded (zeroed state)."""
        B, D, bf = params.batch, params.head_dim, torch.bfloat16
        fk = fv = sk = sv = None
        if params.n_full:
            fk = self.empty((B, params.n_full, capacity, D), bf, f"{name}.full_k", 0)
            fv = self.empty((B, params.n_full, capacity, D), bf, f"{name}.full_v", 0)
        if params.n_ring:
            sk = self.empty((B, params.n_ring, params.ring_slots, D), bf, f"{name}.strm_k", 0)
            sv = self.empty((B, params.n_ring, params.ring_slots, D), bf, f"{name}.strm_v", 0)
        return duo.DuoCache(fk, fv, capacity, sk, sv,
                            self.empty((B,), torch.int32, f"{name}.seq_len", 0),
                            self.empty((B,), torch.int32, f"{name}.ring_head", 0))

    def check(self):
        torch.cuda.synchronize()
        for name, raw, nbytes in self.bufs:
            head = raw[:GUARD]
            tail = raw[GUARD + nbytes:]
            assert bool((head == PATTERN).all()), f"{name}: written before its start"
            assert bool((tail == PATTERN).all()), f"{name}: written past its end"
