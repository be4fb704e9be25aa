"""sata_decode_step_static, the decode step that allocates no device memory.

It exists for callers that must not call cudaMalloc (a serving runtime that
owns all device memory through its own arena, a plugin inside another
application's allocator, a process under a memory budget).  Its partial sums
live in a static device array, so it must give the same result as the ordinary
sata_decode_step, call after call.  This file is collected last so that a run
stopping at the first failure has already run every other test; it also runs
on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

from symmetric_taylor_self_b200 import workloads as wl
from tests.parity import TOL, token_rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sata():
    from symmetric_taylor_self_b200 import build as b
    b.build()
    import symmetric_taylor_self_b200 as s
    s.load()
    assert torch.cuda.is_available()
    return s


def _state_pair(sata, B, H, d, seed):
    """Two identical states built by an ordinary prefill."""
    q, k, v = wl.random_inputs(B, H, 200, d, d, seed=seed)
    st_a = sata.State(B, H, d, d, 4)
    sata.prefill(q.cuda(), k.cuda(), v.cuda(), P=4, state=st_a)
    st_b = sata.State(B, H, d, d, 4)
    st_b.S.copy_(st_a.S)
    st_b.Z.copy_(st_a.Z)
    st_b.st.tokens = st_a.st.tokens
    torch.cuda.synchronize()
    return st_a, st_b


@pytest.mark.parametrize("B,H,d", [(4, 8, 32), (1, 8, 64), (2, 3, 16)])
def test_static_decode_matches_ordinary_decode_twice(sata, B, H, d):
    st_a, st_b = _state_pair(sata, B, H, d, seed=4000 + d)
    steps = wl.random_inputs(B, H, 2, d, d, seed=5000 + d)
    for t in range(2):                                   # two calls in a row
        q, k, v = (x[:, :, t].contiguous().cuda() for x in steps)
        ya = sata.decode_step(st_a, q, k, v)
        yb = torch.empty_like(ya)
        sata.sata_decode_step_static(st_b.st, q, k, v, yb)
        torch.cuda.synchronize()
        err, _, _ = token_rel_err(yb.cpu().numpy().reshape(-1, d), ya.cpu().numpy().reshape(-1, d))
        assert err <= TOL, f"call {t}: {err:.3e}"
        for X, Y in ((st_a.S, st_b.S), (st_a.Z, st_b.Z)):
            rel = (X - Y).abs().max().item() / X.abs().max().item()
            assert rel <= TOL
    assert st_b.tokens == st_a.tokens
