"""GPU parity: libsata (through the C ABI) against the float64 oracle.

Every case feeds both sides the same seeded bf16 inputs (the oracle widens
them to float64) and gates the per-token normwise error at parity.TOL.
Small cases cover every token and span several feature tiles, several chunks
and a ragged tail; the full-size workloads are checked on the heads and
token ranges the oracle can finish in seconds.
"""
import math

import numpy as np
import pytest
import torch

from symmetric_taylor_self_b200 import workloads as wl
from tests.parity import TOL, tensor_rel_err, token_rel_err

pytestmark = pytest.mark.gpu

PATHS = {"cuda_core": 1, "auto": 0}     # auto: tensor cores for the shapes below with P <= 4
TC_SHAPES = {(16, 16), (16, 32), (16, 64), (32, 16), (32, 32), (32, 64), (64, 16), (64, 32), (64, 64),
             (64, 128), (128, 64), (128, 128)}


def _on_tc(path, d_K, d_V, P):
    return path == "auto" and (d_K, d_V) in TC_SHAPES and P <= 4


@pytest.fixture(scope="module")
def sata():
    from symmetric_taylor_self_b200 import build as b
    b.build()
    import symmetric_taylor_self_b200 as s
    s.load()
    assert torch.cuda.is_available()
    yield s
    s.sata_set_option(s.SATA_OPT_PREFILL_PATH, 0)


def _set_path(sata, path):
    sata.sata_set_option(sata.SATA_OPT_PREFILL_PATH, PATHS[path])


def _oracle_heads(oracle_mod, q, k, v, P, heads, T=None):
    return oracle_mod.prefill(q, k, v, P, heads=heads, T=T)


def _check_heads(y_gpu, ref, T=None, what=""):
    for (b, h), (y, den, S, Z) in ref.items():
        yy = y_gpu[b, h, : (T or y.shape[0])].double().cpu().numpy()
        err, excl, tens = token_rel_err(yy, y)
        assert err <= TOL, f"{what} head {(b, h)}: max per-token rel err {err:.3e} > {TOL}"
        assert excl == 0


@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("d,N", [(8, 1), (8, 33), (8, 300), (16, 127), (16, 129), (32, 1),
                                 (32, 257), (64, 31), (64, 129)])
def test_prefill_small_ragged(sata, oracle_mod, path, d, N):
    _set_path(sata, path)
    q, k, v = wl.random_inputs(1, 2, N, d, d, seed=1000 + d * 7 + N)
    y = sata.prefill(q.cuda(), k.cuda(), v.cuda(), P=4)
    torch.cuda.synchronize()
    assert sata.sata_sync_status() == 0
    ref = _oracle_heads(oracle_mod, q, k, v, 4, [(0, 0), (0, 1)])
    _check_heads(y, ref, what=f"d={d} N={N}")


@pytest.mark.parametrize("P", [1, 2, 3])
def test_prefill_lower_P(sata, oracle_mod, P):
    _set_path(sata, "auto")
    q, k, v = wl.random_inputs(1, 1, 100, 16, 16, seed=50 + P)
    y = sata.prefill(q.cuda(), k.cuda(), v.cuda(), P=P)
    ref = _oracle_heads(oracle_mod, q, k, v, P, [(0, 0)])
    _check_heads(y, ref, what=f"P={P}")


@pytest.mark.parametrize("d,P,N", [(4, 5, 200), (8, 6, 150), (4, 8, 130), (8, 8, 40)])
def test_prefill_and_decode_higher_P(sata, oracle_mod, d, P, N):
    """P > 4 (seven-index features): CUDA-core prefill over N tokens, then three
    decode steps, against the oracle's recurrence over all N + 3 tokens."""
    _set_path(sata, "auto")
    B, H, steps = 1, 2, 3
    q, k, v = wl.random_inputs(B, H, N + steps, d, d, seed=900 + 10 * d + P)
    st = sata.State(B, H, d, d, P)
    y = sata.prefill(q[:, :, :N].contiguous().cuda(), k[:, :, :N].contiguous().cuda(),
                     v[:, :, :N].contiguous().cuda(), P=P, state=st)
    ys = [sata.decode_step(st, q[:, :, N + i].contiguous().cuda(), k[:, :, N + i].contiguous().cuda(),
                           v[:, :, N + i].contiguous().cuda()) for i in range(steps)]
    torch.cuda.synchronize()
    assert sata.sata_sync_status() == 0
    yall = torch.cat([y, torch.stack(ys, dim=2)], dim=2)
    _check_heads(yall, _oracle_heads(oracle_mod, q, k, v, P, [(0, 0), (0, 1)]), what=f"d={d} P={P}")


@pytest.mark.parametrize("d_K,d_V,N,tc", [(32, 64, 150, True), (64, 16, 140, True), (128, 128, 20, True),
                                          (128, 128, 300, True), (64, 128, 200, True), (128, 64, 260, True),
                                          (16, 64, 140, True), (12, 8, 90, False)])
def test_prefill_and_decode_other_head_sizes(sata, oracle_mod, d_K, d_V, N, tc):
    """d_K != d_V and d = 128 run on the tensor-core prefill (d_K, d_V in
    {16, 32, 64, 128}); odd or small head sizes on the CUDA-core prefill.
    Prefill plus two decode steps against the oracle."""
    _set_path(sata, "auto")
    sata.sata_reset_kernel_stats()
    B, H, steps = 1, 1, 2
    q, k, v = wl.random_inputs(B, H, N + steps, d_K, d_V, seed=1300 + d_K + d_V)
    st = sata.State(B, H, d_K, d_V, 4)
    y = sata.prefill(q[:, :, :N].contiguous().cuda(), k[:, :, :N].contiguous().cuda(),
                     v[:, :, :N].contiguous().cuda(), P=4, state=st)
    ys = [sata.decode_step(st, q[:, :, N + i].contiguous().cuda(), k[:, :, N + i].contiguous().cuda(),
                           v[:, :, N + i].contiguous().cuda()) for i in range(steps)]
    torch.cuda.synchronize()
    assert sata.sata_sync_status() == 0
    yall = torch.cat([y, torch.stack(ys, dim=2)], dim=2)
    assert ("tc_scan" in sata.sata_kernel_stats()) == tc
    _check_heads(yall, _oracle_heads(oracle_mod, q, k, v, 4, [(0, 0)]), what=f"d_K={d_K} d_V={d_V}")


def test_prefill_f32_tiny_workload(sata, oracle_mod):
    """The tiny configuration as specified: fp32 q, k, v ~ N(0, 1), used as drawn
    (sata_prefill_f32, CUDA-core path), every token against the oracle on the same
    fp32 values; the bf16 entry point on the rounded draws differs from it by the
    input rounding alone."""
    w = wl.WORKLOADS["tiny_d8"]
    (q, k, v), _ = wl.make_inputs(w, dtype=torch.float32)
    sata.sata_reset_kernel_stats()
    y = sata.prefill_f32(q.cuda(), k.cuda(), v.cuda(), P=w.P)
    torch.cuda.synchronize()
    assert sata.sata_sync_status() == 0
    assert "simt_scan" in sata.sata_kernel_stats() and "tc_scan" not in sata.sata_kernel_stats()
    ref = _oracle_heads(oracle_mod, q, k, v, w.P, [(0, 0)])
    _check_heads(y, ref, what="tiny_d8, fp32 inputs")
    # the rounded draws change the result by more than the float32 path's own error
    yb = sata.prefill(q.to(torch.bfloat16).cuda(), k.to(torch.bfloat16).cuda(), v.to(torch.bfloat16).cuda(), P=w.P)
    d = (yb - y).abs().max().item() / y.abs().max().item()
    e = (y[0, 0].double().cpu() - torch.from_numpy(ref[(0, 0)][0])).abs().max().item() / y.abs().max().item()
    assert d > 10 * e


@pytest.mark.parametrize("d_K,d_V,N", [(64, 64, 300), (16, 32, 150), (5, 4, 70)])
def test_prefill_f32_other_shapes(sata, oracle_mod, d_K, d_V, N):
    """fp32 inputs on shapes the bf16 entry point serves on tensor cores, and an
    odd d_K, in two calls through a state: every token of both heads, and the
    final state, against the oracle."""
    B, H, m = 1, 2, N // 3
    q, k, v = wl.random_inputs(B, H, N, d_K, d_V, seed=5600 + d_K + d_V, dtype=torch.float32)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    st = sata.State(B, H, d_K, d_V, 4)
    ya = sata.prefill_f32(qc[:, :, :m].contiguous(), kc[:, :, :m].contiguous(), vc[:, :, :m].contiguous(), 4, st)
    yb = sata.prefill_f32(qc[:, :, m:].contiguous(), kc[:, :, m:].contiguous(), vc[:, :, m:].contiguous(), 4, st)
    torch.cuda.synchronize()
    assert sata.sata_sync_status() == 0 and st.tokens == N
    ref = _oracle_heads(oracle_mod, q, k, v, 4, [(0, 0), (0, 1)])
    _check_heads(torch.cat([ya, yb], dim=2), ref, what=f"fp32 d_K={d_K} d_V={d_V}")
    for (b, h), (_, _, S, Z) in ref.items():
        assert np.abs(st.S[b, h].double().cpu().numpy() - S).max() / np.abs(S).max() <= TOL
        assert np.abs(st.Z[b, h].double().cpu().numpy() - Z).max() / np.abs(Z).max() <= TOL


@pytest.mark.parametrize("name", ["tiny_d8", "prefill_d16"])
def test_prefill_workload_all_heads(sata, oracle_mod, name):
    _set_path(sata, "auto")
    w = wl.WORKLOADS[name]
    (q, k, v), _ = wl.make_inputs(w)
    y = sata.prefill(q.cuda(), k.cuda(), v.cuda(), P=w.P)
    ref = _oracle_heads(oracle_mod, q, k, v, w.P, list(w.oracle_heads))
    _check_heads(y, ref, what=name)


def test_prefill_workload_d32(sata, oracle_mod):
    _set_path(sata, "auto")
    w = wl.WORKLOADS["prefill_d32"]
    (q, k, v), _ = wl.make_inputs(w)
    y = sata.prefill(q.cuda(), k.cuda(), v.cuda(), P=w.P)
    ref = _oracle_heads(oracle_mod, q, k, v, w.P, list(w.oracle_heads))
    _check_heads(y, ref, what="prefill_d32 full heads")
    allh = [(b, h) for b in range(w.B) for h in range(w.H)]
    ref = _oracle_heads(oracle_mod, q, k, v, w.P, allh, T=1024)
    _check_heads(y, ref, T=1024, what="prefill_d32 all heads t<1024")


def test_prefill_workload_d64(sata, oracle_mod):
    """The headline workload at full size (B=1, H=8, N=65536, d = 64) in the
    benchmark's launch configuration: every token of head 0 up to 2048, and on
    every head a sample of tokens out to the end of the sequence (where the
    readout operand's scale 2^-sigma_c has grown the most), each checked with the
    oracle's direct form at that token."""
    _set_path(sata, "auto")
    w = wl.WORKLOADS["prefill_d64"]
    (q, k, v), _ = wl.make_inputs(w)
    y = sata.prefill(q.cuda(), k.cuda(), v.cuda(), P=w.P)
    torch.cuda.synchronize()
    assert sata.sata_sync_status() == 0
    ref = _oracle_heads(oracle_mod, q, k, v, w.P, list(w.oracle_heads), T=w.oracle_tokens)
    _check_heads(y, ref, T=w.oracle_tokens, what="prefill_d64 head 0, first 2048 tokens")
    rng = np.random.default_rng(64)
    ts = sorted({2047, 2048, 16383, 16384, 32767, 32768, 49151, 65535,
                 *rng.integers(2048, w.N, 8).tolist()})
    yc = y.cpu()
    for h in range(w.H):
        yr, _, kappa = oracle_mod.direct_at(q[0, h], k[0, h], v[0, h], w.P, ts)
        err, excl, _ = token_rel_err(yc[0, h, ts].double().numpy(), yr, kappa)
        assert err <= TOL, f"prefill_d64 head {h}, tokens {ts}: {err:.3e}"
        assert excl <= 2


@pytest.mark.parametrize("name", ["prefill_d128", "prefill_d64_dv32", "prefill_d16_p6"])
def test_prefill_workload_other_shapes(sata, oracle_mod, name):
    """The benchmark's other prefill workloads (d = 128, d_K != d_V, P = 6) at
    full size, in its launch configuration: the first tokens of head 0 against
    the oracle's recurrence, and on every head a sample of tokens out to the end
    of the sequence against the direct form."""
    _set_path(sata, "auto")
    w = wl.WORKLOADS[name]
    (q, k, v), _ = wl.make_inputs(w)
    sata.sata_reset_kernel_stats()
    y = sata.prefill(q.cuda(), k.cuda(), v.cuda(), P=w.P)
    torch.cuda.synchronize()
    assert sata.sata_sync_status() == 0
    assert ("tc_scan" in sata.sata_kernel_stats()) == (w.P <= 4)
    ref = _oracle_heads(oracle_mod, q, k, v, w.P, list(w.oracle_heads), T=w.oracle_tokens)
    _check_heads(y, ref, T=w.oracle_tokens, what=f"{name} head 0, first {w.oracle_tokens} tokens")
    rng = np.random.default_rng(w.seed)
    ts = sorted({w.oracle_tokens, w.N // 2 - 1, w.N // 2, w.N - 1,
                 *rng.integers(w.oracle_tokens, w.N, 6).tolist()})
    yc = y.cpu()
    for h in range(w.H):
        yr, _, kappa = oracle_mod.direct_at(q[0, h], k[0, h], v[0, h], w.P, ts)
        err, excl, _ = token_rel_err(yc[0, h, ts].double().numpy(), yr, kappa)
        assert err <= TOL, f"{name} head {h}, tokens {ts}: {err:.3e}"
        assert excl <= 2


@pytest.mark.parametrize("mode", ["deterministic", "atomic", "host"])
def test_prefill_d64_internal_segments(sata, oracle_mod, mode):
    """d = 64, P = 4 with 64 heads: in the fixed-order mode the partial buffer
    bound splits the 3000 tokens into two segments inside one call (the state is
    stored and reloaded between them); the host-buffer entry point splits it
    into four.  Two heads are checked on every token, with their final S and Z."""
    _set_path(sata, "auto")
    B, H, N, d = 1, 64, 3000, 64
    q, k, v = wl.random_inputs(B, H, N, d, d, seed=6400)
    st = sata.State(B, H, d, d, 4)
    if mode == "host":
        stream = torch.cuda.Stream()
        st.set_stream(stream)
        yh = torch.empty((B, H, N, d), dtype=torch.float32).pin_memory()
        sata.sata_prefill_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), yh, B, H, N, d, d, 4, st.st, stream)
        stream.synchronize()
        y = yh
    else:
        sata.sata_set_option(sata.SATA_OPT_DETERMINISTIC, 1 if mode == "deterministic" else 0)
        try:
            sata.sata_reset_kernel_stats()
            y = sata.prefill(q.cuda(), k.cuda(), v.cuda(), P=4, state=st)
            torch.cuda.synchronize()
            n_scan = sata.sata_kernel_stats()["tc_scan"][0]
        finally:
            sata.sata_set_option(sata.SATA_OPT_DETERMINISTIC, 0)
        assert (n_scan >= 2) if mode == "deterministic" else (n_scan == 1)
    torch.cuda.synchronize()
    assert sata.sata_sync_status() == 0
    heads = [(0, 5), (0, 63)]
    ref = _oracle_heads(oracle_mod, q, k, v, 4, heads)
    _check_heads(y, ref, what=f"{mode} d=64 N={N}")
    for (b, h), (_, _, S, Z) in ref.items():
        Sg, Zg = st.S[b, h].double().cpu().numpy(), st.Z[b, h].double().cpu().numpy()
        assert np.abs(Sg - S).max() / np.abs(S).max() <= TOL
        assert np.abs(Zg - Z).max() / np.abs(Z).max() <= TOL


def test_prefill_host_profiled_segments(sata, oracle_mod):
    """The host-buffer entry point over 65 chunks splits the sequence into four
    unequal segments (10 %, 20 %, 55 %, 15 % of the chunks: 6, 13, 36 and 10
    here), carrying the state between them: every token of two heads and their
    final state against the oracle, and the output against the device-buffer
    call within the tolerance (the segments prescale their rows separately)."""
    _set_path(sata, "auto")
    B, H, N, d = 1, 2, 8300, 32
    q, k, v = wl.random_inputs(B, H, N, d, d, seed=6500)
    st = sata.State(B, H, d, d, 4)
    stream = torch.cuda.Stream()
    st.set_stream(stream)
    yh = torch.empty((B, H, N, d), dtype=torch.float32).pin_memory()
    sata.sata_reset_kernel_stats()
    sata.sata_prefill_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), yh, B, H, N, d, d, 4, st.st, stream)
    stream.synchronize()
    assert sata.sata_sync_status(stream) == 0
    assert sata.sata_kernel_stats()["tc_scan"][0] == 4
    ref = _oracle_heads(oracle_mod, q, k, v, 4, [(0, 0), (0, 1)])
    _check_heads(yh, ref, what=f"host segments d={d} N={N}")
    for (b, h), (_, _, S, Z) in ref.items():
        Sg, Zg = st.S[b, h].double().cpu().numpy(), st.Z[b, h].double().cpu().numpy()
        assert np.abs(Sg - S).max() / np.abs(S).max() <= TOL
        assert np.abs(Zg - Z).max() / np.abs(Z).max() <= TOL
    yd = sata.prefill(q.cuda(), k.cuda(), v.cuda(), P=4).cpu()
    err, _, _ = token_rel_err(yh.double().numpy().reshape(-1, d), yd.double().numpy().reshape(-1, d))
    assert err <= TOL


@pytest.mark.parametrize("d_K,d_V,N", [(64, 32, 700), (128, 128, 300), (32, 64, 520)])
def test_prefill_host_other_shapes(sata, oracle_mod, d_K, d_V, N):
    """The host-buffer entry point on the other tensor-core shapes (three token
    segments at these lengths, the state carried between them): every token of
    both heads against the oracle."""
    _set_path(sata, "auto")
    B, H = 1, 2
    q, k, v = wl.random_inputs(B, H, N, d_K, d_V, seed=6600 + d_K + d_V)
    stream = torch.cuda.Stream()
    yh = torch.empty((B, H, N, d_V), dtype=torch.float32).pin_memory()
    sata.sata_reset_kernel_stats()
    sata.sata_prefill_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), yh, B, H, N, d_K, d_V, 4, None, stream)
    stream.synchronize()
    assert sata.sata_sync_status(stream) == 0
    assert sata.sata_kernel_stats()["tc_scan"][0] == 3
    ref = _oracle_heads(oracle_mod, q, k, v, 4, [(0, 0), (0, 1)])
    _check_heads(yh, ref, what=f"host d_K={d_K} d_V={d_V} N={N}")


def test_prefill_host_back_to_back_calls(sata):
    """Two host-buffer calls on one stream with different inputs and no sync
    between them (four segments each): each output equals the device-buffer
    prefill of its own inputs. The second call's input copies may not start
    before the first call's kernels have read the shared device copies."""
    _set_path(sata, "auto")
    B, H, N, d = 1, 8, 16384, 64
    x1 = wl.random_inputs(B, H, N, d, d, seed=5900)
    x2 = wl.random_inputs(B, H, N, d, d, seed=5901)
    stream = torch.cuda.Stream()
    ys = [torch.empty((B, H, N, d), dtype=torch.float32).pin_memory() for _ in range(2)]
    pinned = [[t.pin_memory() for t in x] for x in (x1, x2)]
    for (q, k, v), y in zip(pinned, ys):
        sata.sata_prefill_host(q, k, v, y, B, H, N, d, d, 4, None, stream)
    stream.synchronize()
    assert sata.sata_sync_status(stream) == 0
    for (q, k, v), y in zip((x1, x2), ys):
        ref = sata.prefill(q.cuda(), k.cuda(), v.cuda(), P=4).cpu()
        assert ((y - ref).abs().max() / ref.abs().max()).item() <= 1e-5


def test_prefill_d64_long_head(sata, oracle_mod):
    """One d = 64 head over 8192 tokens against the oracle's recurrence: every
    token and the final state."""
    _set_path(sata, "auto")
    q, k, v = wl.random_inputs(1, 1, 8192, 64, 64, seed=6401)
    st = sata.State(1, 1, 64, 64, 4)
    y = sata.prefill(q.cuda(), k.cuda(), v.cuda(), P=4, state=st)
    torch.cuda.synchronize()
    ref = _oracle_heads(oracle_mod, q, k, v, 4, [(0, 0)])
    _check_heads(y, ref, what="d=64 N=8192")
    (_, _, S, Z), = ref.values()
    assert np.abs(st.S[0, 0].double().cpu().numpy() - S).max() / np.abs(S).max() <= TOL
    assert np.abs(st.Z[0, 0].double().cpu().numpy() - Z).max() / np.abs(Z).max() <= TOL


def test_decode_workload(sata, oracle_mod):
    """8192-token prefill into a state, then 1024 decode steps; four heads are
    followed by the oracle through all 9216 tokens."""
    _set_path(sata, "auto")
    w = wl.WORKLOADS["decode_d32"]
    (q, k, v), (qs, ks, vs) = wl.make_inputs(w)
    st = sata.State(w.B, w.H, w.d_K, w.d_V, w.P)
    y = sata.prefill(q.cuda(), k.cuda(), v.cuda(), P=w.P, state=st)
    qs, ks, vs = qs.cuda(), ks.cuda(), vs.cuda()
    outs = torch.empty((w.steps, w.B, w.H, w.d_V), dtype=torch.float32, device="cuda")
    for i in range(w.steps):
        sata.decode_step(st, qs[i], ks[i], vs[i], out=outs[i])
    torch.cuda.synchronize()
    assert st.tokens == w.N + w.steps
    heads = list(w.oracle_heads)
    qf = torch.cat([q, qs.cpu().permute(1, 2, 0, 3)], dim=2)
    kf = torch.cat([k, ks.cpu().permute(1, 2, 0, 3)], dim=2)
    vf = torch.cat([v, vs.cpu().permute(1, 2, 0, 3)], dim=2)
    ref = oracle_mod.prefill(qf, kf, vf, w.P, heads=heads)
    for (b, h), (yr, den, S, Z) in ref.items():
        err, _, _ = token_rel_err(y[b, h].cpu().numpy(), yr[: w.N])
        assert err <= TOL, f"prefill part of head {(b, h)}: {err:.3e}"
        err, _, _ = token_rel_err(outs[:, b, h].cpu().numpy(), yr[w.N:])
        assert err <= TOL, f"decode part of head {(b, h)}: {err:.3e}"
        Sg = st.S[b, h].double().cpu().numpy()
        Zg = st.Z[b, h].double().cpu().numpy()
        assert np.abs(Sg - S).max() / np.abs(S).max() <= TOL
        assert np.abs(Zg - Z).max() / np.abs(Z).max() <= TOL


@pytest.mark.parametrize("path", list(PATHS))
def test_state_output_and_continuation(sata, oracle_mod, path):
    """prefill(N) == prefill(N - m) then prefill(m) from the state == prefill(N - m)
    then m decode steps; the final state matches the oracle's."""
    _set_path(sata, path)
    B, H, N, d, m = 2, 3, 200, 16, 37
    q, k, v = wl.random_inputs(B, H, N, d, d, seed=77)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    y_full = sata.prefill(qc, kc, vc, P=4)
    st = sata.State(B, H, d, d, 4)
    y_a = sata.prefill(qc[:, :, : N - m].contiguous(), kc[:, :, : N - m].contiguous(),
                       vc[:, :, : N - m].contiguous(), P=4, state=st)
    st2 = sata.State(B, H, d, d, 4)
    st2.S.copy_(st.S)
    st2.Z.copy_(st.Z)
    st2.st.tokens = st.tokens
    y_b = sata.prefill(qc[:, :, N - m:].contiguous(), kc[:, :, N - m:].contiguous(),
                       vc[:, :, N - m:].contiguous(), P=4, state=st)
    dec = [sata.decode_step(st2, qc[:, :, t].contiguous(), kc[:, :, t].contiguous(),
                            vc[:, :, t].contiguous()) for t in range(N - m, N)]
    torch.cuda.synchronize()
    y_seg = torch.cat([y_a, y_b], dim=2)
    y_dec = torch.cat([y_a, torch.stack(dec, dim=2)], dim=2)
    ref = oracle_mod.prefill(q, k, v, 4)
    for (b, h), (yr, den, S, Z) in ref.items():
        for name, yy in (("one call", y_full), ("two calls", y_seg), ("decode", y_dec)):
            err, _, _ = token_rel_err(yy[b, h].cpu().numpy(), yr)
            assert err <= TOL, f"{name} head {(b, h)}: {err:.3e}"
        for stt in (st, st2):
            Sg, Zg = stt.S[b, h].double().cpu().numpy(), stt.Z[b, h].double().cpu().numpy()
            assert np.abs(Sg - S).max() / np.abs(S).max() <= TOL
            assert np.abs(Zg - Z).max() / np.abs(Z).max() <= TOL
    assert st.tokens == N and st2.tokens == N


@pytest.mark.parametrize("d_K", [64, 128])
def test_value_halves_state_continuation(sata, oracle_mod, d_K):
    """d_V = 128 on device buffers runs as two d_V = 64 prefills over the column
    halves of v, out and S, both producing Z. Two calls carrying the state (the
    second half must find the incoming Z, not the first half's result): outputs
    of both calls and the final S and Z against the oracle; the fixed-order mode
    repeats bit for bit; the host-buffer path (whole rows) agrees."""
    _set_path(sata, "auto")
    B, H, N, m, d_V = 1, 2, 260, 110, 128
    q, k, v = wl.random_inputs(B, H, N, d_K, d_V, seed=5500 + d_K)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    st = sata.State(B, H, d_K, d_V, 4)
    sata.sata_reset_kernel_stats()
    y_a = sata.prefill(qc[:, :, : N - m].contiguous(), kc[:, :, : N - m].contiguous(),
                       vc[:, :, : N - m].contiguous(), P=4, state=st)
    # the second call in a caller workspace of exactly the queried size (which covers a
    # carried state's copy of Z)
    ws = torch.empty(sata.sata_workspace_bytes(B, H, m, d_K, d_V, 4), dtype=torch.uint8, device="cuda")
    y_b = sata.prefill(qc[:, :, N - m:].contiguous(), kc[:, :, N - m:].contiguous(),
                       vc[:, :, N - m:].contiguous(), P=4, state=st, workspace=ws)
    torch.cuda.synchronize()
    assert sata.sata_sync_status() == 0
    assert sata.sata_kernel_stats()["tc_scan"][0] == 4   # two calls x two halves
    y = torch.cat([y_a, y_b], dim=2)
    ref = oracle_mod.prefill(q, k, v, 4, heads=[(0, 1)])
    yr, _, S, Z = ref[(0, 1)]
    err, _, _ = token_rel_err(y[0, 1].cpu().numpy(), yr)
    assert err <= TOL, f"two calls: {err:.3e}"
    Sg, Zg = st.S[0, 1].double().cpu().numpy(), st.Z[0, 1].double().cpu().numpy()
    assert np.abs(Sg - S).max() / np.abs(S).max() <= TOL
    assert np.abs(Zg - Z).max() / np.abs(Z).max() <= TOL
    sata.sata_set_option(sata.SATA_OPT_DETERMINISTIC, 1)
    try:
        y1 = sata.prefill(qc, kc, vc, P=4)
        y2 = sata.prefill(qc, kc, vc, P=4)
    finally:
        sata.sata_set_option(sata.SATA_OPT_DETERMINISTIC, 0)
    assert torch.equal(y1, y2)
    stream = torch.cuda.Stream()
    yh = torch.empty((B, H, N, d_V), dtype=torch.float32).pin_memory()
    sata.sata_prefill_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), yh, B, H, N, d_K, d_V, 4, None, stream)
    stream.synchronize()
    assert sata.sata_sync_status(stream) == 0
    assert tensor_rel_err(yh[0, 1].double().numpy(), yr) <= TOL
    assert tensor_rel_err(y1[0, 1].double().cpu().numpy(), yr) <= TOL


@pytest.mark.parametrize("d_K,P", [(64, 1), (64, 3), (128, 2), (128, 3)])
def test_value_halves_lower_P(sata, oracle_mod, d_K, P):
    """The d_V = 128 halves at P < 4 (other unit plans for the (d_K, 64) instance):
    every token of both heads against the oracle."""
    _set_path(sata, "auto")
    sata.sata_reset_kernel_stats()
    q, k, v = wl.random_inputs(1, 2, 170, d_K, 128, seed=5800 + d_K + P)
    y = sata.prefill(q.cuda(), k.cuda(), v.cuda(), P=P)
    torch.cuda.synchronize()
    assert sata.sata_sync_status() == 0
    assert sata.sata_kernel_stats()["tc_scan"][0] == 2
    _check_heads(y, _oracle_heads(oracle_mod, q, k, v, P, [(0, 0), (0, 1)]), what=f"halves d_K={d_K} P={P}")


@pytest.mark.parametrize("path", list(PATHS))
def test_deterministic(sata, path):
    """With SATA_OPT_DETERMINISTIC = 1 every path is bitwise reproducible."""
    _set_path(sata, path)
    sata.sata_set_option(sata.SATA_OPT_DETERMINISTIC, 1)
    try:
        q, k, v = wl.random_inputs(1, 4, 333, 32, 32, seed=5)
        qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
        a = sata.prefill(qc, kc, vc, P=4)
        b = sata.prefill(qc, kc, vc, P=4)
        assert torch.equal(a, b)
    finally:
        sata.sata_set_option(sata.SATA_OPT_DETERMINISTIC, 0)


@pytest.mark.parametrize("d", [16, 32, 64])
def test_atomic_partials_match_fixed_order(sata, d):
    """The default tensor-core prefill (partial sums added in L2) agrees with
    the fixed-order reduction to fp32 rounding, and runs no tc_reduce."""
    _set_path(sata, "auto")
    q, k, v = (x.cuda() for x in wl.random_inputs(1, 3, 700, d, d, seed=77 + d))
    sata.sata_set_option(sata.SATA_OPT_DETERMINISTIC, 1)
    try:
        ref = sata.prefill(q, k, v, P=4)
    finally:
        sata.sata_set_option(sata.SATA_OPT_DETERMINISTIC, 0)
    sata.sata_reset_kernel_stats()
    y = sata.prefill(q, k, v, P=4)
    torch.cuda.synchronize()
    stats = sata.sata_kernel_stats()
    assert "tc_scan" in stats and "tc_reduce" not in stats
    assert (y - ref).abs().max().item() <= 1e-5 * ref.abs().max().item()


def test_empty_inputs_are_noops(sata):
    x = torch.empty((1, 2, 0, 16), dtype=torch.bfloat16, device="cuda")
    y = sata.prefill(x, x, x, P=4)
    assert y.shape == (1, 2, 0, 16)
    x = torch.empty((0, 2, 5, 16), dtype=torch.bfloat16, device="cuda")
    assert sata.prefill(x, x, x, P=4).shape == (0, 2, 5, 16)
    assert sata.sata_sync_status() == 0


def test_decode_small_against_oracle(sata, oracle_mod):
    """Decode from an empty state for every supported d_V, all heads."""
    for d in (4, 8, 16, 64, 128):
        B, H, T = 1, 2, 5
        q, k, v = wl.random_inputs(B, H, T, d, d, seed=900 + d)
        st = sata.State(B, H, d, d, 4)
        outs = [sata.decode_step(st, q[:, :, t].contiguous().cuda(), k[:, :, t].contiguous().cuda(),
                                 v[:, :, t].contiguous().cuda()) for t in range(T)]
        torch.cuda.synchronize()
        yg = torch.stack(outs, dim=2).cpu().numpy()
        for (b, h), (yr, _, _, _) in oracle_mod.prefill(q, k, v, 4).items():
            err, _, _ = token_rel_err(yg[b, h], yr)
            assert err <= TOL, f"d={d}: {err:.3e}"


@pytest.mark.parametrize("d", [16, 32, 64])
def test_tensor_core_path_selected_and_multi_segment_state(sata, oracle_mod, d):
    """The tensor-core path serves d in {16, 32, 64}; a state carried in from a
    previous call is honoured."""
    sata.sata_set_option(sata.SATA_OPT_PREFILL_PATH, 2)
    B, H, N = 1, 2, 300
    q, k, v = wl.random_inputs(B, H, N, d, d, seed=31 + d)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    sata.sata_reset_kernel_stats()
    st = sata.State(B, H, d, d, 4)
    y1 = sata.prefill(qc[:, :, :170].contiguous(), kc[:, :, :170].contiguous(), vc[:, :, :170].contiguous(),
                      P=4, state=st)
    y2 = sata.prefill(qc[:, :, 170:].contiguous(), kc[:, :, 170:].contiguous(), vc[:, :, 170:].contiguous(),
                      P=4, state=st)
    torch.cuda.synchronize()
    assert sata.sata_sync_status() == 0
    stats = sata.sata_kernel_stats()
    assert stats.get("tc_scan", (0, 0))[0] >= 2
    y = torch.cat([y1, y2], dim=2)
    for (b, h), (yr, _, S, Z) in oracle_mod.prefill(q, k, v, 4).items():
        err, _, _ = token_rel_err(y[b, h].cpu().numpy(), yr)
        assert err <= TOL, f"d={d} head {h}: {err:.3e}"
        assert np.abs(st.S[b, h].double().cpu().numpy() - S).max() / np.abs(S).max() <= TOL
    sata.sata_set_option(sata.SATA_OPT_PREFILL_PATH, 0)


@pytest.mark.parametrize("path,d,N", [("auto", 64, 1000), ("auto", 32, 300), ("auto", 16, 129),
                                      ("cuda_core", 8, 300)])
def test_prefill_host_matches_device_and_oracle(sata, oracle_mod, path, d, N):
    """sata_prefill_host (host buffers, copies pipelined by token segment) gives
    the device entry point's result and passes the oracle."""
    _set_path(sata, path)
    B, H = 1, 2
    q, k, v = wl.random_inputs(B, H, N, d, d, seed=700 + d + N)
    y_dev = sata.prefill(q.cuda(), k.cuda(), v.cuda(), P=4)
    qh, kh, vh = q.pin_memory(), k.pin_memory(), v.pin_memory()
    yh = torch.full((B, H, N, d), float("nan"), dtype=torch.float32).pin_memory()
    stream = torch.cuda.Stream()
    sata.sata_prefill_host(qh, kh, vh, yh, B, H, N, d, d, 4, None, stream)
    stream.synchronize()
    torch.cuda.synchronize()
    assert sata.sata_sync_status() == 0
    assert torch.isfinite(yh).all()
    scale = y_dev.abs().max().item()
    # The host path runs the sequence as token segments, each with its own power-of-two
    # operand prescale (from that segment's maxima), so the fp16 roundings of tiny operands
    # differ from the one-segment device call: agreement to 1e-4, both within the oracle bar.
    assert (yh - y_dev.cpu()).abs().max().item() <= 1e-4 * scale
    _check_heads(yh, _oracle_heads(oracle_mod, q, k, v, 4, [(0, 1)]), what=f"host d={d} N={N}")


def test_prefill_host_carries_state(sata, oracle_mod):
    """Two host-buffer calls on one state equal one call over the whole sequence."""
    _set_path(sata, "auto")
    B, H, N, d = 1, 2, 700, 64
    q, k, v = wl.random_inputs(B, H, N, d, d, seed=77)
    st = sata.State(B, H, d, d, 4)
    stream = torch.cuda.Stream()
    st.set_stream(stream)
    parts = []
    for a, b in ((0, 300), (300, N)):
        yh = torch.empty((B, H, b - a, d), dtype=torch.float32).pin_memory()
        sata.sata_prefill_host(q[:, :, a:b].contiguous().pin_memory(), k[:, :, a:b].contiguous().pin_memory(),
                               v[:, :, a:b].contiguous().pin_memory(), yh, B, H, b - a, d, d, 4, st.st, stream)
        stream.synchronize()
        parts.append(yh)
    assert sata.sata_sync_status(stream) == 0
    assert st.tokens == N
    y = torch.cat(parts, dim=2)
    for (b, h), (yr, _, S, Z) in oracle_mod.prefill(q, k, v, 4).items():
        err, _, _ = token_rel_err(y[b, h].double().numpy(), yr)
        assert err <= TOL, f"head {h}: {err:.3e}"
        assert np.abs(st.S[b, h].double().cpu().numpy() - S).max() / np.abs(S).max() <= TOL


def test_bounded_wait_reports_timeout(sata):
    """A producer signal withheld on purpose: every wait gives up after the
    limit, the kernel exits cleanly, and the status comes back as SATA_ETIMEOUT;
    the next call runs normally."""
    sata.sata_set_option(sata.SATA_OPT_PREFILL_PATH, 2)
    sata.sata_set_option(sata.SATA_OPT_WAIT_LIMIT, 50_000_000)      # 50 ms
    q, k, v = wl.random_inputs(1, 1, 512, 16, 16, seed=8)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    assert sata.sata_sync_status() == 0
    sata.sata_set_option(sata.SATA_OPT_TEST_STALL, 1)
    sata.prefill(qc, kc, vc, P=4)
    assert sata.sata_sync_status() == sata.SATA_ETIMEOUT
    assert sata.sata_get_option(sata.SATA_OPT_TEST_STALL) == 0
    sata.sata_set_option(sata.SATA_OPT_WAIT_LIMIT, 0)
    a = sata.prefill(qc, kc, vc, P=4)
    assert sata.sata_sync_status() == 0
    b = sata.prefill(qc, kc, vc, P=4)
    # equal up to the order of the L2 partial-sum additions (SATA_OPT_DETERMINISTIC = 0)
    assert (a - b).abs().max().item() <= 1e-6 * a.abs().max().item()
    sata.sata_set_option(sata.SATA_OPT_PREFILL_PATH, 0)


@pytest.mark.parametrize("d_K,d_V,scale,vscale", [(32, 32, 100.0, 1.0), (32, 32, 1e-3, 1.0), (64, 64, 30.0, 1e4),
                                                (16, 16, 1.0, 1e-4), (64, 64, 1e-2, 300.0)])
def test_tensor_core_path_any_input_range(sata, oracle_mod, d_K, d_V, scale, vscale):
    """The pages put no bound on q, k, v and the accuracy depends on the input
    statistics ([CC-TAYLOR] "Precision vs efficiency"): the tensor-core path
    prescales each head's q/c, k and v by powers of two, so inputs far from
    N(0, 1) keep their accuracy.  Gated per token on the well-conditioned
    tokens (kappa <= 8, as everywhere), against the oracle's direct form."""
    sata.sata_set_option(sata.SATA_OPT_PREFILL_PATH, 2)
    try:
        N = 300
        q, k, v = wl.random_inputs(1, 2, N, d_K, d_V, seed=9 + d_K, scale=scale, vscale=vscale)
        y = sata.prefill(q.cuda(), k.cuda(), v.cuda(), P=4)
        torch.cuda.synchronize()
        assert sata.sata_sync_status() == 0
        for h in range(2):
            yr, den, kappa = oracle_mod.direct(q[0, h], k[0, h], v[0, h], 4)
            err, excl, _ = token_rel_err(y[0, h].double().cpu().numpy(), yr, kappa)
            assert err <= TOL, f"scale {scale}/{vscale} head {h}: {err:.3e}"
            assert excl < N // 2
    finally:
        sata.sata_set_option(sata.SATA_OPT_PREFILL_PATH, 0)


def test_non_finite_inputs_are_reported(sata):
    """An infinite input cannot be represented: the call reports SATA_ERANGE at
    sync and the affected head's outputs are not finite (never silent); the other
    head and the next call are unaffected."""
    sata.sata_set_option(sata.SATA_OPT_PREFILL_PATH, 2)
    try:
        q, k, v = wl.random_inputs(1, 2, 200, 32, 32, seed=19)
        k[0, 1, 50, 3] = float("inf")
        y = sata.prefill(q.cuda(), k.cuda(), v.cuda(), P=4)
        assert sata.sata_sync_status() == sata.SATA_ERANGE
        assert not torch.isfinite(y[0, 1]).all()
        assert torch.isfinite(y[0, 0]).all()
        k[0, 1, 50, 3] = 0.0
        sata.prefill(q.cuda(), k.cuda(), v.cuda(), P=4)
        assert sata.sata_sync_status() == 0
    finally:
        sata.sata_set_option(sata.SATA_OPT_PREFILL_PATH, 0)


# ------------------------------------------------------------ backward ----
# sata_prefill_backward against the oracle's chain-rule gradient of the direct
# form, on every token of the checked heads.  Gate: tensor-wise max error over
# max |reference| <= TOL for each of dq, dk, dv.

def _check_grads(sata, oracle_mod, B, H, N, d_K, d_V, P, seed, heads=None):
    q, k, v = wl.random_inputs(B, H, N, d_K, d_V, seed=seed)
    dy = wl.random_cotangent(B, H, N, d_V, seed=seed + 1)
    dq, dk, dv = sata.prefill_backward(q.cuda(), k.cuda(), v.cuda(), dy.cuda(), P)
    torch.cuda.synchronize()
    heads = heads or [(b, h) for b in range(B) for h in range(H)]
    ref = oracle_mod.grad_heads(q, k, v, dy, P, heads=heads)
    for (b, h), (rq, rk, rv) in ref.items():
        for name, g, r in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
            err = tensor_rel_err(g[b, h].double().cpu().numpy(), r)
            assert err <= TOL, f"{name} head {(b, h)} d_K={d_K} d_V={d_V} P={P} N={N}: {err:.3e}"
    return dq, dk, dv


@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("d_K,d_V,P,N", [(16, 16, 4, 100), (8, 8, 4, 77), (32, 32, 4, 70),
                                         (64, 64, 4, 130), (16, 32, 3, 65), (12, 8, 2, 50),
                                         (8, 8, 5, 40), (4, 4, 1, 33), (128, 128, 2, 37),
                                         (6, 8, 7, 29), (32, 4, 4, 140), (128, 128, 2, 100),
                                         (64, 128, 2, 70), (64, 16, 4, 300), (128, 64, 3, 260),
                                         (32, 64, 4, 290), (64, 32, 1, 200), (16, 16, 2, 400),
                                         (128, 128, 4, 160), (128, 64, 4, 140)])
def test_backward_matches_oracle(sata, oracle_mod, path, d_K, d_V, P, N):
    """auto: the forward and the three gradient scans run on tensor cores for the
    tensor-core shapes with P <= 4; cuda_core: everything on CUDA cores."""
    _set_path(sata, path)
    sata.sata_reset_kernel_stats()
    _check_grads(sata, oracle_mod, 1, 2, N, d_K, d_V, P, seed=5000 + d_K + P * 3 + N)
    stats = sata.sata_kernel_stats()
    assert ("bwd_tc_finish" in stats) == _on_tc(path, d_K, d_V, P)
    assert ("bwd_tc_scan" in stats) == _on_tc(path, d_K, d_V, P)
    _set_path(sata, "auto")


_T4_ROOT = -1.5960716379833215   # the real root of 1 + x + x^2/2 + x^3/6


@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("d_K,d_V", [(128, 64), (128, 128), (64, 64), (32, 32)])
def test_backward_near_root_denominator(sata, oracle_mod, path, d_K, d_V):
    """Head 1's first token has q_0 . k_0 / c just above the real root of the
    P = 4 series, so its denominator T_4(x) is about 0.01 and its cotangent
    dy / den is ~100x every other token's: the gradients of the other tokens
    must keep their accuracy beside it."""
    _set_path(sata, path)
    N, P = 600, 4
    q, k, v = wl.random_inputs(1, 2, N, d_K, d_V, seed=5400 + d_K + d_V)
    dy = wl.random_cotangent(1, 2, N, d_V, seed=5401)
    k0 = k[0, 1, 0].double()
    alpha = (_T4_ROOT + 0.015) * math.sqrt(d_K) / float(k0 @ k0)
    q[0, 1, 0] = (alpha * k0).to(q.dtype)
    x = float(q[0, 1, 0].double() @ k0) / math.sqrt(d_K)
    den0 = 1 + x + x * x / 2 + x ** 3 / 6
    assert 2e-3 < den0 < 3e-2
    dq, dk, dv = sata.prefill_backward(q.cuda(), k.cuda(), v.cuda(), dy.cuda(), P)
    torch.cuda.synchronize()
    assert sata.sata_sync_status() == 0
    ref = oracle_mod.grad_heads(q, k, v, dy, P, heads=[(0, 0), (0, 1)])
    for (b, h), (rq, rk, rv) in ref.items():
        for name, g, r in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
            err = tensor_rel_err(g[b, h].double().cpu().numpy(), r)
            assert err <= TOL, f"{name} head {(b, h)} d_K={d_K} d_V={d_V}: {err:.3e}"
    _set_path(sata, "auto")


@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("d_K,d_V,t0", [(64, 64, 317), (128, 64, 128), (32, 32, 599)])
def test_backward_cotangent_outlier(sata, oracle_mod, path, d_K, d_V, t0):
    """One token's dy is 10^4 times the others' (t0 mid-sequence, on a chunk
    boundary, or last): in the reversed gradient scans the outlier's chunk comes
    in the middle, at the start or at the end, and the chunks on either side of
    it must keep their accuracy."""
    _set_path(sata, path)
    N, P = 600, 4
    q, k, v = wl.random_inputs(1, 2, N, d_K, d_V, seed=5700 + d_K + t0)
    dy = wl.random_cotangent(1, 2, N, d_V, seed=5701)
    dy[0, 1, t0] *= 1e4
    dq, dk, dv = sata.prefill_backward(q.cuda(), k.cuda(), v.cuda(), dy.cuda(), P)
    torch.cuda.synchronize()
    assert sata.sata_sync_status() == 0
    ref = oracle_mod.grad_heads(q, k, v, dy, P, heads=[(0, 0), (0, 1)])
    for (b, h), (rq, rk, rv) in ref.items():
        for name, g, r in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
            err = tensor_rel_err(g[b, h].double().cpu().numpy(), r)
            assert err <= TOL, f"{name} head {(b, h)} d_K={d_K} t0={t0}: {err:.3e}"
    _set_path(sata, "auto")


def test_backward_single_token(sata):
    """N = 1: y_0 = v_0 whatever q and k are, so dv = dy and dq = dk = 0 (up to
    rounding: dw = g.v - g.y cancels)."""
    q, k, v = (x.cuda() for x in wl.random_inputs(1, 2, 1, 8, 16, seed=5050))
    dy = wl.random_cotangent(1, 2, 1, 16, seed=5051).cuda()
    dq, dk, dv = sata.prefill_backward(q, k, v, dy, 4)
    torch.cuda.synchronize()
    assert torch.allclose(dv, dy, rtol=1e-6, atol=1e-6)
    assert dq.abs().max().item() <= 1e-5 and dk.abs().max().item() <= 1e-5


def test_backward_several_segments(sata, oracle_mod):
    """d = 64, P = 4 with 8 heads: the partial buffer holds about 1400 tokens,
    so 3000 tokens run as three segments (S carried forward, G backward)."""
    _check_grads(sata, oracle_mod, 2, 4, 3000, 64, 64, 4, seed=5100, heads=[(0, 0), (1, 3)])


@pytest.mark.parametrize("path", list(PATHS))
def test_backward_is_deterministic_and_linear_in_dy(sata, path):
    """Bitwise repeatable with SATA_OPT_DETERMINISTIC = 1 (the recomputed
    forward may run on tensor cores, the gradient scans then run on CUDA cores),
    and linear in dy: to fp32 rounding on CUDA cores; on the tensor-core gradient
    scans (fp16 operands, r rounded after a per-head power-of-two scale that
    depends on dy) to about their stated accuracy."""
    _set_path(sata, path)
    q, k, v = (x.cuda() for x in wl.random_inputs(1, 2, 200, 16, 16, seed=5200))
    dy1 = wl.random_cotangent(1, 2, 200, 16, seed=5201).cuda()
    dy2 = wl.random_cotangent(1, 2, 200, 16, seed=5202).cuda()
    sata.sata_set_option(sata.SATA_OPT_DETERMINISTIC, 1)
    try:
        a = sata.prefill_backward(q, k, v, dy1, 4)
        b = sata.prefill_backward(q, k, v, dy1, 4)
    finally:
        sata.sata_set_option(sata.SATA_OPT_DETERMINISTIC, 0)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    c = sata.prefill_backward(q, k, v, dy2, 4)
    s = sata.prefill_backward(q, k, v, dy1 + 2.0 * dy2, 4)
    for x, y, z in zip(a, c, s):
        tol = 1e-4 if path == "cuda_core" else 1e-3
        assert torch.allclose(z, x + 2.0 * y, rtol=tol, atol=tol * z.abs().max().item())


def test_attention_autograd(sata, oracle_mod):
    """attention() as a torch autograd op: y matches prefill, and .backward()
    gives the oracle's gradients (cast to the inputs' bf16)."""
    q, k, v = wl.random_inputs(1, 1, 90, 16, 16, seed=5300)
    dy = wl.random_cotangent(1, 1, 90, 16, seed=5301)
    qc, kc, vc = (x.cuda().requires_grad_() for x in (q, k, v))
    y = sata.attention(qc, kc, vc, 4)
    y.backward(dy.cuda())
    rq, rk, rv = oracle_mod.direct_grad(q[0, 0], k[0, 0], v[0, 0], dy[0, 0], 4)
    for g, r in ((qc.grad, rq), (kc.grad, rk), (vc.grad, rv)):
        assert g.dtype == torch.bfloat16
        assert tensor_rel_err(g[0, 0].double().cpu().numpy(), r) <= 1e-2   # bf16 rounding of the gradient


@pytest.mark.parametrize("name", ["backward_d64", "backward_d16"])
def test_backward_workload_full_size(sata, oracle_mod, name):
    """The benchmark's backward workloads at full size, in the benchmark's
    launch configuration (all heads, library workspace); the oracle checks
    every token of the listed heads."""
    w = wl.WORKLOADS[name]
    (q, k, v), _ = wl.make_inputs(w)
    dy = wl.cotangent(w)
    sata.sata_reset_kernel_stats()
    dq, dk, dv = sata.prefill_backward(q.cuda(), k.cuda(), v.cuda(), dy.cuda(), w.P)
    torch.cuda.synchronize()
    assert sata.sata_sync_status() == 0
    assert "bwd_tc_scan" in sata.sata_kernel_stats()
    ref = oracle_mod.grad_heads(q, k, v, dy, w.P, heads=list(w.oracle_heads))
    for (b, h), (rq, rk, rv) in ref.items():
        for nm, g, r in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
            err = tensor_rel_err(g[b, h].double().cpu().numpy(), r)
            assert err <= TOL, f"{name} {nm} head {(b, h)}: {err:.3e}"


# ------------------------------------------------ sequence split (row f4) ----

@pytest.mark.parametrize("d,lens,P", [(32, (300, 212), 4), (64, (128, 257, 100), 4), (16, (64, 64, 64, 65), 4),
                                     (8, (50, 1, 77), 5)])
def test_sequence_split_emulated_ranks(sata, oracle_mod, d, lens, P):
    """The product steps of the sequence split on one GPU, its ranks run one
    after another in this process (no kernel waits on another rank): segment
    states, the exclusive prefix in rank order (sata_state_accumulate), then
    each segment's prefill from its prefix.  The concatenated outputs match the
    oracle over the whole sequence and one prefill on one GPU; the last rank's
    state matches the whole sequence's state."""
    from symmetric_taylor_self_b200 import seqsplit
    _set_path(sata, "auto")
    N = sum(lens)
    q, k, v = wl.random_inputs(1, 2, N, d, d, seed=900 + d)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    bounds = np.cumsum((0,) + lens)
    segs = [(qc[:, :, a:b].contiguous(), kc[:, :, a:b].contiguous(), vc[:, :, a:b].contiguous())
            for a, b in zip(bounds[:-1], bounds[1:])]
    impl = seqsplit.LibraryImpl()
    gathered = [impl.tensors(impl.segment_state(*sg, P)) for sg in segs]
    ys, st = [], None
    for r, sg in enumerate(segs):
        st = seqsplit.exclusive_prefix(impl, (1, 2, d, d, P), gathered, r, list(lens), qc.device)
        assert st.tokens == bounds[r]
        ys.append(impl.prefill(*sg, P, st))
    y = torch.cat(ys, dim=2)
    torch.cuda.synchronize()
    assert sata.sata_sync_status() == 0
    ref = _oracle_heads(oracle_mod, q, k, v, P, [(0, 0), (0, 1)])
    _check_heads(y, ref, what=f"split d={d} {lens}")
    whole = sata.State(1, 2, d, d, P)
    y1 = sata.prefill(qc, kc, vc, P=P, state=whole)
    torch.cuda.synchronize()
    assert (y - y1).abs().max().item() <= 1e-3 * y1.abs().max().item()
    assert st.tokens == N
    for got, want in ((st.S, whole.S), (st.Z, whole.Z)):
        assert (got - want).abs().max().item() <= 1e-4 * want.abs().max().item()


def test_state_accumulate_adds_and_counts(sata):
    """sata_state_accumulate: S += dS, Z += dZ elementwise, tokens += n."""
    st = sata.State(2, 3, 8, 16, 4)
    dS = torch.randn_like(st.S)
    dZ = torch.randn_like(st.Z)
    sata.sata_state_accumulate(st.st, dS, dZ, 7)
    sata.sata_state_accumulate(st.st, dS, dZ, 5)
    torch.cuda.synchronize()
    assert st.tokens == 12
    assert torch.allclose(st.S, 2 * dS, rtol=0, atol=1e-6) and torch.allclose(st.Z, 2 * dZ, rtol=0, atol=1e-6)
