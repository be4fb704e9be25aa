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


@pytest.mark.parametrize("d_K,d_V,P", [(32, 4, 4), (16, 8, 4), (64, 128, 4), (32, 64, 3), (17, 16, 2),
                                       (9, 32, 1), (128, 16, 3), (33, 8, 4), (64, 32, 2)])
def test_static_decode_against_oracle(sata, d_K, d_V, P):
    """The allocation-free decode step checked against the oracle itself, over
    the value widths, d_K != d_V, odd d_K and P = 1..4 it accepts: a prefill of
    N tokens into the state, then three static decode steps, whose outputs must
    match the oracle's recurrence at tokens N, N+1, N+2."""
    import oracle
    B, H, N, steps = 2, 2, 90, 3
    q, k, v = wl.random_inputs(B, H, N + steps, d_K, d_V, seed=7000 + 10 * d_K + d_V + P)
    st = sata.State(B, H, d_K, d_V, P)
    sata.prefill(q[:, :, :N].contiguous().cuda(), k[:, :, :N].contiguous().cuda(),
                 v[:, :, :N].contiguous().cuda(), P=P, state=st)
    ys = []
    for i in range(steps):
        y = torch.empty((B, H, d_V), dtype=torch.float32, device="cuda")
        sata.sata_decode_step_static(st.st, q[:, :, N + i].contiguous().cuda(), k[:, :, N + i].contiguous().cuda(),
                                     v[:, :, N + i].contiguous().cuda(), y)
        ys.append(y)
    torch.cuda.synchronize()
    assert sata.sata_sync_status() == 0
    assert st.tokens == N + steps
    got = torch.stack(ys, dim=2).double().cpu().numpy()           # [B, H, steps, d_V]
    ref = oracle.prefill(q, k, v, P)
    for (b, h), (yr, _, _, _) in ref.items():
        err, excl, _ = token_rel_err(got[b, h], yr[N:N + steps])
        assert err <= TOL, f"head {(b, h)}: {err:.3e}"
        assert excl == 0


def test_static_decode_scratch_limit(sata):
    """A shape whose partial sums exceed the static array is refused before any
    launch (about 4500 heads fit at d_K = d_V = 32, P = 4: 7 groups x 33 values
    per head), and the state is left untouched."""
    B, H, d = 1, 4600, 32
    st = sata.State(B, H, d, d, 4)
    before = st.S[0, :4].clone()
    x = torch.zeros((B, H, d), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((B, H, d), dtype=torch.float32, device="cuda")
    with pytest.raises(sata.SataError) as e:
        sata.sata_decode_step_static(st.st, x, x, x, out)
    assert e.value.status == sata.SATA_ENOMEM
    torch.cuda.synchronize()
    assert torch.equal(st.S[0, :4], before)
    assert st.tokens == 0
