"""Host-side checks of libsata: it builds, loads, exports every symbol the
header declares, and its host-only calls (basis tables, sizes, argument
validation) behave, all without a GPU."""
import ctypes
import itertools
import math
import os
import re
from collections import Counter

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from symmetric_taylor_self_b200 import build as b
    b.build()
    from symmetric_taylor_self_b200 import binding
    return binding.load()


def header_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"SATA_API\s+[\w\s\*]*?\b(sata_\w+)\s*\(", src))
    return names


def test_every_declared_symbol_is_exported(lib):
    names = header_symbols()
    assert len(names) >= 16
    for n in names:
        assert hasattr(lib, n), n
    from symmetric_taylor_self_b200.binding import EXPORTED
    assert set(EXPORTED) == names


def test_exported_symbols_via_nm(lib):
    import subprocess
    from symmetric_taylor_self_b200.binding import LIB_PATH
    out = subprocess.run(["nm", "-D", "--defined-only", LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (sata_\w+)", out))
    assert header_symbols() <= exported


def test_library_is_built_for_sm100a():
    import subprocess
    from symmetric_taylor_self_b200.build import NVCC_FLAGS
    assert "arch=compute_100a,code=sm_100a" in NVCC_FLAGS


def test_status_strings(lib):
    for code in range(0, -8, -1):
        s = lib.sata_status_string(code).decode()
        assert s.startswith("SATA_")
    assert lib.sata_version() >= 10000


@pytest.mark.parametrize("d,P", [(1, 1), (1, 4), (2, 3), (8, 4), (16, 4), (32, 4), (64, 4), (128, 4), (5, 6),
                                 (8, 8), (16, 6)])
def test_num_features(lib, d, P):
    from symmetric_taylor_self_b200 import sata_num_features
    assert sata_num_features(d, P) == math.comb(d + P - 1, P - 1)


@pytest.mark.parametrize("d,P", [(1, 4), (2, 2), (3, 4), (8, 4), (16, 4), (32, 4), (64, 4), (7, 5), (4, 8),
                                 (8, 6)])
def test_basis_matches_oracle_bit_exact(lib, oracle_mod, d, P):
    from symmetric_taylor_self_b200 import sata_build_basis
    M, C, off = sata_build_basis(d, P)
    deg, Mo, Co, offo = oracle_mod.basis(d, P)
    assert off.numpy().tolist() == offo.tolist()
    Mn = M.numpy().astype(np.int64)
    Mn[Mn == 255] = -1
    assert np.array_equal(Mn, Mo.astype(np.int64))
    assert np.array_equal(np.asarray(C.numpy(), dtype=np.int64), Co)


@pytest.mark.parametrize("d,p", [(2, 3), (3, 3), (4, 2), (5, 3)])
def test_basis_matches_brute_force(lib, d, p):
    from symmetric_taylor_self_b200 import sata_build_basis
    M, C, off = sata_build_basis(d, p + 1)
    counts = Counter(tuple(sorted(t)) for t in itertools.product(range(d), repeat=p))
    rows = [tuple(int(i) for i in M[r, :p]) for r in range(int(off[p]), int(off[p + 1]))]
    assert rows == sorted(counts)
    assert [int(c) for c in np.asarray(C.numpy(), dtype=np.int64)[int(off[p]):int(off[p + 1])]] == \
        [counts[t] for t in sorted(counts)]


def test_size_queries(lib):
    from symmetric_taylor_self_b200 import sata_state_bytes, sata_workspace_bytes
    S, Z = sata_state_bytes(1, 8, 64, 64, 4)
    assert S == 8 * 47905 * 64 * 4 and Z == 8 * 47905 * 4
    assert (S + Z) // 8 // 4 == 3113825           # (d_V + 1) binom(67, 3) per head
    ws = sata_workspace_bytes(1, 8, 65536, 64, 64, 4)
    # prefill_d64 in the default mode: the prescaled fp16 rows (201 MB) and the L2-resident
    # readout sums of one segment (143 MB); no per-unit partial buffer
    rows = 8 * 65536 * (64 + 64 + 64) * 2
    sums = 8 * 512 * 17 * 128 * 16
    assert rows + sums <= ws < rows + sums + (1 << 20)
    assert ws < 0.6e9
    from symmetric_taylor_self_b200 import sata_backward_workspace_bytes as bwb
    small, big = bwb(1, 1, 1000, 16, 16, 4), bwb(1, 1, 100000, 16, 16, 4)
    # y, den and r are kept for every token: at least (2 d_V + 2) fp32 values per token
    assert big - small >= (100000 - 1000) * (2 * 16 + 2) * 4


def test_argument_validation_needs_no_gpu(lib):
    from symmetric_taylor_self_b200 import binding as bd
    vp = ctypes.c_void_p
    fake = vp(0x10000)           # never dereferenced: checks fail before any launch
    # unsupported shapes
    assert lib.sata_prefill_ex(fake, fake, fake, fake, 1, 1, 8, 8, 12, 4, None, None, 0, None) == bd.SATA_EUNSUPPORTED
    assert lib.sata_prefill_ex(fake, fake, fake, fake, 1, 1, 8, 8, 8, 9, None, None, 0, None) == bd.SATA_EUNSUPPORTED
    assert lib.sata_prefill_ex(fake, fake, fake, fake, 1, 1, 8, 256, 8, 4, None, None, 0, None) == bd.SATA_EUNSUPPORTED
    # invalid values
    assert lib.sata_prefill_ex(fake, fake, fake, fake, -1, 1, 8, 8, 8, 4, None, None, 0, None) == bd.SATA_EINVAL
    assert lib.sata_prefill_ex(fake, fake, fake, fake, 1, 1, -3, 8, 8, 4, None, None, 0, None) == bd.SATA_EINVAL
    assert lib.sata_prefill_ex(fake, fake, fake, fake, 1, 1, 8, 0, 8, 4, None, None, 0, None) == bd.SATA_EINVAL
    assert lib.sata_prefill_ex(None, fake, fake, fake, 1, 1, 8, 8, 8, 4, None, None, 0, None) == bd.SATA_EINVAL
    # misaligned pointer
    assert lib.sata_prefill_ex(vp(0x10002), fake, fake, fake, 1, 1, 8, 8, 8, 4, None, None, 0, None) == bd.SATA_EALIGN
    # empty problems are no-ops
    assert lib.sata_prefill_ex(None, None, None, None, 1, 1, 0, 8, 8, 4, None, None, 0, None) == bd.SATA_OK
    assert lib.sata_prefill_ex(None, None, None, None, 0, 4, 16, 8, 8, 4, None, None, 0, None) == bd.SATA_OK
    # state mismatch
    st = bd.sata_state(B=1, H=1, d_K=8, d_V=8, P=3, F=120, S=0x10000, Z=0x10000, stream=None, tokens=0)
    assert lib.sata_prefill_ex(fake, fake, fake, fake, 1, 1, 8, 8, 8, 4, ctypes.byref(st), None, 0, None) == bd.SATA_EINVAL
    # host-buffer prefill: the same shape checks, host pointers required
    assert lib.sata_prefill_host(fake, fake, fake, fake, 1, 1, 8, 8, 12, 4, None, None) == bd.SATA_EUNSUPPORTED
    assert lib.sata_prefill_host(None, fake, fake, fake, 1, 1, 8, 8, 8, 4, None, None) == bd.SATA_EINVAL
    assert lib.sata_prefill_host(None, None, None, None, 1, 1, 0, 8, 8, 4, None, None) == bd.SATA_OK
    # fp32-input prefill: the same checks
    f32 = lib.sata_prefill_f32
    assert f32(fake, fake, fake, fake, 1, 1, 8, 8, 12, 4, None, None) == bd.SATA_EUNSUPPORTED
    assert f32(fake, fake, fake, fake, 1, 1, 8, 8, 8, 9, None, None) == bd.SATA_EUNSUPPORTED
    assert f32(fake, fake, fake, fake, 1, 1, -3, 8, 8, 4, None, None) == bd.SATA_EINVAL
    assert f32(fake, None, fake, fake, 1, 1, 8, 8, 8, 4, None, None) == bd.SATA_EINVAL
    assert f32(fake, fake, vp(0x10004), fake, 1, 1, 8, 8, 8, 4, None, None) == bd.SATA_EALIGN
    assert f32(None, None, None, None, 1, 1, 0, 8, 8, 4, None, None) == bd.SATA_OK
    st = bd.sata_state(B=1, H=1, d_K=8, d_V=8, P=3, F=120, S=0x10000, Z=0x10000, stream=None, tokens=0)
    assert f32(fake, fake, fake, fake, 1, 1, 8, 8, 8, 4, ctypes.byref(st), None) == bd.SATA_EINVAL
    # backward
    bw = lambda *a: lib.sata_prefill_backward(*a, None, 0, None)
    assert bw(fake, fake, fake, fake, fake, fake, fake, 1, 1, 8, 8, 12, 4) == bd.SATA_EUNSUPPORTED
    assert bw(fake, fake, fake, fake, fake, fake, fake, 1, 1, 8, 8, 8, 9) == bd.SATA_EUNSUPPORTED
    assert bw(fake, fake, fake, None, fake, fake, fake, 1, 1, 8, 8, 8, 4) == bd.SATA_EINVAL
    assert bw(fake, fake, fake, fake, fake, fake, fake, 1, -1, 8, 8, 8, 4) == bd.SATA_EINVAL
    assert bw(fake, fake, fake, fake, fake, vp(0x10004), fake, 1, 1, 8, 8, 8, 4) == bd.SATA_EALIGN
    assert bw(None, None, None, None, None, None, None, 1, 1, 0, 8, 8, 4) == bd.SATA_OK
    # state accumulation
    st = bd.sata_state(B=1, H=1, d_K=8, d_V=8, P=4, F=165, S=0x10000, Z=0x10000, stream=None, tokens=0)
    assert lib.sata_state_accumulate(None, fake, fake, 1) == bd.SATA_EINVAL
    assert lib.sata_state_accumulate(ctypes.byref(st), None, fake, 1) == bd.SATA_EINVAL
    assert lib.sata_state_accumulate(ctypes.byref(st), fake, fake, -1) == bd.SATA_EINVAL
    assert lib.sata_state_accumulate(ctypes.byref(st), vp(0x10008), fake, 1) == bd.SATA_EALIGN
    st.F = 999
    assert lib.sata_state_accumulate(ctypes.byref(st), fake, fake, 1) == bd.SATA_EINVAL
    # decode
    assert lib.sata_decode_step(None, fake, fake, fake, fake) == bd.SATA_EINVAL
    st = bd.sata_state(B=1, H=1, d_K=8, d_V=8, P=4, F=999, S=0x10000, Z=0x10000, stream=None, tokens=0)
    assert lib.sata_decode_step(ctypes.byref(st), fake, fake, fake, fake) == bd.SATA_EINVAL
    # options
    assert lib.sata_set_option(bd.SATA_OPT_PREFILL_PATH, 7) == bd.SATA_EINVAL
    assert lib.sata_set_option(999, 0) == bd.SATA_EINVAL
    v = ctypes.c_int64(-1)
    assert lib.sata_get_option(bd.SATA_OPT_PREFILL_PATH, ctypes.byref(v)) == bd.SATA_OK and v.value == 0


def test_binding_refuses_without_library(tmp_path):
    from symmetric_taylor_self_b200 import binding
    saved = binding._lib
    try:
        binding._lib = None
        with pytest.raises(ImportError):
            binding.load(str(tmp_path / "missing.so"))
    finally:
        binding._lib = saved


def test_product_path_does_not_touch_oracle():
    """The package never imports, links or executes anything under oracle/."""
    pkg = os.path.join(ROOT, "symmetric_taylor_self_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cpp", ".h", ".cuh")):
                src = open(os.path.join(dirpath, fn)).read()
                assert "import oracle" not in src and "from oracle" not in src, fn
                assert "sata_oracle" not in src and "liboracle" not in src, fn


def test_static_decode_rejects_oversized_requests_before_any_cuda_call(lib):
    """The no-allocation decode step rejects shapes whose partial sums exceed its
    static scratch, before touching the GPU.  Run on the CPU suite only: the
    pointers below are placeholders that must never reach a kernel."""
    from symmetric_taylor_self_b200 import binding as bd
    B, H, d = 64, 64, 64
    F = math.comb(d + 3, 3)
    G = (F + 1023) // 1024
    assert B * H * G * (d + 1) > 2 ** 20          # oversized by construction
    fake = ctypes.c_void_p(0x10000)
    st = bd.sata_state(B=B, H=H, d_K=d, d_V=d, P=4, F=F, S=0x10000, Z=0x10000, stream=None, tokens=0)
    assert lib.sata_decode_step_static(ctypes.byref(st), fake, fake, fake, fake) == bd.SATA_ENOMEM
    assert st.tokens == 0
    # the allocation-free step derives its basis for P <= 4 only
    st5 = bd.sata_state(B=1, H=1, d_K=8, d_V=8, P=5, F=math.comb(12, 4), S=0x10000, Z=0x10000, stream=None, tokens=0)
    assert lib.sata_decode_step_static(ctypes.byref(st5), fake, fake, fake, fake) == bd.SATA_EUNSUPPORTED
    # invalid arguments are rejected the same way as by sata_decode_step
    assert lib.sata_decode_step_static(None, fake, fake, fake, fake) == bd.SATA_EINVAL
    st.F = 7
    assert lib.sata_decode_step_static(ctypes.byref(st), fake, fake, fake, fake) == bd.SATA_EINVAL
