"""The C-ABI library loads, exports every declared symbol, and rejects bad
arguments on the host (no GPU needed: nothing here reaches a CUDA call)."""

import ctypes
import os
import re

import pytest

import combine_ep_route_02_b200 as ep
from combine_ep_route_02_b200 import _binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    text = "".join(open(os.path.join(ROOT, "include", h)).read()
                   for h in sorted(os.listdir(os.path.join(ROOT, "include"))) if h.endswith(".h"))
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ep_[a-z_]+)\s*\(", text)))


# Every call below must fail its host checks.  They pass fake device
# addresses, so this module only runs where no GPU is visible: a check that
# went missing must never turn into a launch on real memory.
pytestmark = pytest.mark.skipif(
    __import__("torch").cuda.is_available(),
    reason="host-check tests pass fake device pointers; run them where no GPU is visible")


@pytest.fixture(scope="module")
def lib():
    from combine_ep_route_02_b200 import build
    build.build()
    return B.lib()


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert set(names) == set(B.EXPORTS)
    for n in names:
        assert hasattr(lib, n), n
    out = os.popen(f"nm -D --defined-only {B.LIB}").read()
    for n in names:
        assert re.search(rf"\bT {n}\b", out), n


def test_status_strings(lib):
    for s in range(5):
        assert lib.ep_status_string(s).startswith(b"EP_")


def test_workspace_size(lib):
    # NT tiles of max(64, ceil(T/64)) tokens; [NT][P] + [NT][R] + [NT] int32,
    # each rounded up to 256 bytes
    # (+ 256 bytes for the fused small-batch kernel's completion counter)
    assert ep.ep_workspace_size(8192, 8, 256, 8) == 64 * 256 * 4 + 2048 + 256 + 256
    assert ep.ep_workspace_size(1, 8, 288, 32) == 1280 + 256 + 256 + 256
    assert ep.ep_workspace_size(16384, 8, 288, 32) == 64 * 288 * 4 + 64 * 32 * 4 + 256 + 256
    assert ep.ep_workspace_size(0, 8, 256, 8) > 0
    assert ep.ep_workspace_size(-1, 8, 256, 8) == 0
    assert ep.ep_workspace_size(10, 0, 256, 8) == 0


FAKE = 0x100000  # never dereferenced: every call below fails its host checks
MIS = FAKE + 2   # misaligned


def route(lib, T=4, E=16, G=1, Kg=1, k=2, logits=FAKE):
    cfg = B.RouteCfg(E, G, Kg, k, 1.0, 1)
    return lib.ep_route(logits, None, T, cfg, FAKE, FAKE, None)


@pytest.mark.parametrize("kw", [
    dict(T=-1), dict(E=0), dict(E=16, G=3), dict(E=16, G=4, Kg=5), dict(k=0),
    dict(E=16, G=4, Kg=1, k=5),          # k > (E/G) * topk_group
    dict(E=16, G=16, Kg=2, k=2),         # groups of one expert
    dict(logits=MIS),
])
def test_route_rejects_invalid(lib, kw):
    assert route(lib, **kw) == B.EP_ERR_INVALID


@pytest.mark.parametrize("kw", [dict(E=2048, k=2), dict(E=64, G=64, Kg=1, k=1), dict(E=64, k=33)])
def test_route_rejects_unsupported(lib, kw):
    st = route(lib, **kw)
    assert st in (B.EP_ERR_UNSUPPORTED, B.EP_ERR_INVALID) and st != B.EP_OK


def layout(lib, T=4, k=2, E=16, P=16, R=4, phys=None, nrep=None, ws=FAKE, max_rep=0, align=1):
    return lib.ep_dispatch_layout(FAKE, T, k, E, P, R, phys, nrep, max_rep, align, FAKE, FAKE,
                                  FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, ws, None, None)


@pytest.mark.parametrize("kw", [
    dict(P=16, R=3), dict(P=20), dict(phys=FAKE), dict(phys=FAKE, nrep=FAKE, max_rep=0),
    dict(ws=FAKE + 16), dict(T=-2), dict(k=0), dict(align=0), dict(align=-4),
])
def test_layout_rejects_invalid(lib, kw):
    assert layout(lib, **kw) == B.EP_ERR_INVALID


def test_layout_rejects_too_many_experts(lib):
    assert layout(lib, E=5000, P=5000, R=8) == B.EP_ERR_UNSUPPORTED


def test_layout_rejects_unsupported_alignment(lib):
    assert layout(lib, align=2048) == B.EP_ERR_UNSUPPORTED
    # T*k + P*(A-1) rows must stay below 2^31
    T = (1 << 31) // 16 - 100                    # T*k fits, the padding does not
    assert layout(lib, T=T, k=16, E=4096, P=4096, R=8, align=1024) == B.EP_ERR_UNSUPPORTED


@pytest.mark.parametrize("args", [
    (FAKE, 4, 100, 2, 0, FAKE, 1, FAKE, FAKE),    # fp8 needs H % 128 == 0
    (FAKE, 4, 100, 2, 0, FAKE, 0, FAKE, None),    # bf16 needs H % 8 == 0
    (MIS, 4, 256, 2, 0, FAKE, 1, FAKE, FAKE),     # x not 16-byte aligned
    (FAKE, 4, 256, 2, 0, FAKE, 1, MIS, FAKE),     # recv_x not 16-byte aligned
    (FAKE, 4, 256, 2, 0, FAKE, 1, FAKE, None),    # fp8 without a scale buffer
    (FAKE, 4, 256, 0, 0, FAKE, 1, FAKE, FAKE),
])
def test_dispatch_rejects_invalid(lib, args):
    assert lib.ep_dispatch(*args, 0, None, None) == B.EP_ERR_INVALID


@pytest.mark.parametrize("args", [
    (FAKE, FAKE, FAKE, 4, 100, 2, 0, FAKE),
    (MIS, FAKE, FAKE, 4, 256, 2, 0, FAKE),
    (FAKE, FAKE, FAKE, 4, 256, 2, 0, MIS),
    (FAKE, FAKE, FAKE, -1, 256, 2, 0, FAKE),
])
def test_combine_rejects_invalid(lib, args):
    assert lib.ep_combine(*args, 0, None, None) == B.EP_ERR_INVALID


@pytest.mark.parametrize("args", [
    (FAKE, 4, 100, None, None, 0, 1, FAKE, FAKE),     # I % 128 != 0
    (FAKE, 4, 256, FAKE, None, 16, 1, FAKE, FAKE),    # offsets without counts
    (FAKE, 4, 256, FAKE, FAKE, 0, 1, FAKE, FAKE),     # counts for no experts
    (MIS, 4, 256, None, None, 0, 1, FAKE, FAKE),      # gate_up misaligned
    (FAKE, 4, 256, None, None, 0, 1, MIS, FAKE),      # act misaligned
    (FAKE, 4, 256, None, None, 0, 1, FAKE, None),     # fp8 without scales
    (FAKE, -1, 256, None, None, 0, 1, FAKE, FAKE),
])
def test_silu_mul_rejects_invalid(lib, args):
    assert lib.ep_silu_mul(*args, 0, None) == B.EP_ERR_INVALID


def test_silu_mul_rejects_too_many_experts(lib):
    assert lib.ep_silu_mul(FAKE, 4, 256, FAKE, FAKE, 5000, 1, FAKE, FAKE, 0,
                           None) == B.EP_ERR_UNSUPPORTED


def test_binding_raises(lib):
    with pytest.raises(ep.EpError) as ei:
        B._check("ep_route", B.EP_ERR_INVALID)
    assert ei.value.status == B.EP_ERR_INVALID


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(B, "_lib", None)
    monkeypatch.setattr(B, "LIB", str(tmp_path / "missing.so"))
    with pytest.raises(ImportError):
        B.lib()


def test_exchange_entry_points_reject_bad_arguments(lib):
    """the NCCL exchange calls check their arguments before touching the
    communicator (no GPU, no NCCL communicator needed)"""
    import numpy as np
    c = np.zeros(4, np.int32)
    assert lib.ep_exchange_counts(None, FAKE, FAKE, 256, FAKE, FAKE, None) in (
        B.EP_ERR_INVALID, B.EP_ERR_UNSUPPORTED)
    assert lib.ep_exchange_counts(FAKE, FAKE, FAKE, 0, FAKE, FAKE, None) in (
        B.EP_ERR_INVALID, B.EP_ERR_UNSUPPORTED)
    assert lib.ep_dispatch_exchange(None, FAKE, c.ctypes.data, c.ctypes.data, 16, FAKE,
                                    None) == B.EP_ERR_INVALID
    assert lib.ep_combine_exchange(None, FAKE, c.ctypes.data, c.ctypes.data, 16, FAKE,
                                   None) == B.EP_ERR_INVALID


def test_route_dispatch_rejects_invalid(lib):
    cfg = B.RouteCfg(256, 8, 4, 8, 2.5, 1)
    args = [FAKE, None, 16, cfg, 256, 8, None, None, 0, 1, FAKE, 7168, 1, 0, FAKE, FAKE,
            FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, MIS, 0, None, None]
    assert lib.ep_route_dispatch(*args) == B.EP_ERR_INVALID          # workspace misaligned
    args[26] = FAKE
    bad_h = list(args)
    bad_h[11] = 7000                                                  # fp8 needs H % 128 == 0
    assert lib.ep_route_dispatch(*bad_h) == B.EP_ERR_INVALID
    bad_x = list(args)
    bad_x[10] = MIS                                                   # x not 16-byte aligned
    assert lib.ep_route_dispatch(*bad_x) == B.EP_ERR_INVALID


def test_testing_knob_range(lib):
    assert lib.ep_testing_set_wait_limit(1 << 33) == B.EP_ERR_INVALID
    assert lib.ep_testing_set_wait_limit(-1) == B.EP_OK
