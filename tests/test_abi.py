"""C ABI checks that need no GPU: the library loads, exports every entry
point that include/*.h declares, and rejects bad arguments on the host with
the documented status codes before touching the device."""
import ctypes
import glob
import os
import re

import pytest

import speculative_decoding_verification_88_b200 as sv
from speculative_decoding_verification_88_b200 import build as svbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
OK, INVALID, MISALIGNED, WORKSPACE = 0, 1, 2, 3


@pytest.fixture(scope="module")
def lib():
    svbuild.build()
    return sv.load_library()


def declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names |= set(re.findall(r"\b(spec_verify_\w+)\s*\(", text))
    return sorted(names)


def test_header_declares_the_entry_points():
    names = declared_functions()
    assert set(names) == set(sv.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_launch_counter_needs_no_device(lib):
    n = lib.spec_verify_kernel_launches()
    assert n >= 0 and lib.spec_verify_kernel_launches() == n  # nothing launched between


def test_status_strings(lib):
    for code in range(6):
        assert sv.status_string(code).startswith("SV_")
    assert "unknown" in sv.status_string(99)


def test_workspace_size_limits(lib):
    assert sv.workspace_size(256, 1, 8, 128256) > 0
    assert sv.workspace_size(0, 1, 4, 10) > 0
    assert sv.workspace_size(1, 1, 33, 10) == 0
    assert sv.workspace_size(1, 1, -1, 10) == 0
    assert sv.workspace_size(1, 1, 4, 0) == 0
    assert sv.workspace_size(1, 65, 4, 10) == 0
    assert sv.workspace_size(-1, 1, 4, 10) == 0
    assert sv.workspace_size(64, 1, 4, 128256) % 256 == 0
    assert sv.workspace_size(128, 1, 8, 128256) >= sv.workspace_size(64, 1, 8, 128256)


# Host pointers stand in for device pointers: every call below fails
# validation before any CUDA call, so nothing is dereferenced.
BUF = (ctypes.c_uint8 * 4096)()
A = ctypes.addressof(BUF)  # 16-byte aligned in practice; checked below
A16 = (A + 15) // 16 * 16


def stoch(lib, **kw):
    args = dict(target=A16, t_dtype=1, t_sb=40, t_sp=8, draft=A16, d_dtype=1, d_sb=32, d_sp=8,
                tokens=A16, B=4, k=4, V=8, T=1.0, seed=1, off=0, acc=A16, out=A16, probs=None,
                ws=A16, ws_bytes=1 << 20, stream=None)
    args.update(kw)
    return lib.spec_verify_stochastic(*args.values())


def test_stochastic_validation(lib):
    assert stoch(lib, B=0, target=None) == OK
    assert stoch(lib, k=33) == INVALID
    assert stoch(lib, k=-1) == INVALID
    assert stoch(lib, V=0) == INVALID
    assert stoch(lib, target=None) == INVALID
    assert stoch(lib, draft=None) == INVALID
    assert stoch(lib, tokens=None) == INVALID
    assert stoch(lib, acc=None) == INVALID
    assert stoch(lib, ws=None) == INVALID
    assert stoch(lib, t_dtype=2) == INVALID
    assert stoch(lib, d_dtype=-1) == INVALID
    for T in (0.0, -1.0, float("inf"), float("nan"), 1e-40):
        assert stoch(lib, T=T) == INVALID, T
    assert stoch(lib, t_sb=-8) == INVALID
    assert stoch(lib, target=A16 + 1) == MISALIGNED
    assert stoch(lib, t_dtype=0, target=A16 + 2) == MISALIGNED
    assert stoch(lib, tokens=A16 + 2) == MISALIGNED
    assert stoch(lib, out=A16 + 1) == MISALIGNED
    assert stoch(lib, probs=A16 + 2) == MISALIGNED
    assert stoch(lib, ws=A16 + 8) == MISALIGNED
    assert stoch(lib, ws_bytes=16) == WORKSPACE


def test_greedy_and_multi_validation(lib):
    def g(**kw):
        a = dict(target=A16, t=1, sb=40, sp=8, tok=A16, B=2, k=4, V=8, acc=A16, out=A16,
                 ws=A16, wb=1 << 20, st=None)
        a.update(kw)
        return lib.spec_verify_greedy(*a.values())

    assert g(B=0, target=None) == OK
    assert g(k=40) == INVALID
    assert g(tok=None) == INVALID
    assert g(t=5) == INVALID
    assert g(sp=-1) == INVALID
    assert g(acc=A16 + 1) == MISALIGNED
    assert g(wb=8) == WORKSPACE

    def m(**kw):
        a = dict(target=A16, t=1, sb=80, sg=40, sp=8, tok=A16, B=2, G=2, k=4, V=8, best=A16,
                 acc=A16, out=A16, ws=A16, wb=1 << 20, st=None)
        a.update(kw)
        return lib.spec_verify_multi_candidate(*a.values())

    assert m(G=0) == INVALID
    assert m(G=65) == INVALID
    assert m(best=None) == INVALID
    assert m(best=A16 + 2) == MISALIGNED
    assert m(wb=64) == WORKSPACE


def test_multi_rows_validation(lib):
    def r(**kw):
        a = dict(rows=A16, t=1, sb=80, sr=8, rmap=A16, tok=A16, B=2, G=2, k=4, R=3, V=8,
                 best=A16, acc=A16, out=A16, ws=A16, wb=1 << 20, st=None)
        a.update(kw)
        return lib.spec_verify_multi_candidate_rows(*a.values())

    assert r(B=0, rows=None, rmap=None) == OK
    assert r(R=0) == INVALID
    assert r(R=2 * 5 + 1) == INVALID  # more rows than G * (k + 1)
    assert r(rmap=None) == INVALID
    assert r(best=None) == INVALID
    assert r(rmap=A16 + 2) == MISALIGNED
    assert r(wb=64) == WORKSPACE


def test_threshold_validation(lib):
    def t(**kw):
        a = dict(x=A16, dt=1, sb=40, sp=8, tok=A16, B=2, k=4, V=8, T=1.0, tau=0.1, acc=A16,
                 out=A16, ws=A16, wb=1 << 20, st=None)
        a.update(kw)
        return lib.spec_verify_threshold(*a.values())

    assert t(B=0, x=None) == OK
    for T in (0.0, -1.0, float("inf"), float("nan"), 1e-40):
        assert t(T=T) == INVALID, T
    for tau in (0.0, -0.5, 1.5, float("nan")):
        assert t(tau=tau) == INVALID, tau
    assert t(k=33) == INVALID
    assert t(tok=None) == INVALID
    assert t(acc=A16 + 1) == MISALIGNED
    assert t(wb=64) == WORKSPACE


def test_tree_validation(lib):
    assert sv.tree_workspace_size(4, 26, 128256) > 0
    assert sv.tree_workspace_size(4, 0, 10) == 0
    assert sv.tree_workspace_size(4, 65, 10) == 0
    assert sv.tree_workspace_size(-1, 4, 10) == 0

    def t(**kw):
        a = dict(x=A16, dt=1, sb=80, sn=8, par=A16, tok=A16, B=2, N=10, V=8, acc=A16,
                 path=A16, out=A16, ws=A16, wb=1 << 20, st=None)
        a.update(kw)
        return lib.spec_verify_tree_greedy(*a.values())

    assert t(B=0, x=None, par=None, tok=None) == OK
    assert t(N=0) == INVALID
    assert t(N=65) == INVALID
    assert t(par=None) == INVALID
    assert t(tok=None) == INVALID
    assert t(path=None) == INVALID
    assert t(dt=3) == INVALID
    assert t(par=A16 + 2) == MISALIGNED
    assert t(path=A16 + 1) == MISALIGNED
    assert t(wb=64) == WORKSPACE


def test_tree_stochastic_validation(lib):
    assert sv.tree_stochastic_workspace_size(64, 26, 128256) > 0
    assert sv.tree_stochastic_workspace_size(4, 0, 10) == 0
    assert sv.tree_stochastic_workspace_size(4, 65, 10) == 0
    assert sv.tree_stochastic_workspace_size(-1, 4, 10) == 0
    assert sv.tree_stochastic_workspace_size(8, 26, 128256) >= \
        sv.tree_stochastic_workspace_size(4, 26, 128256)

    def t(**kw):
        a = dict(x=A16, dt=1, sb=80, sn=8, par=A16, tok=A16, B=2, N=10, V=8, T=1.0, seed=3,
                 off=0, acc=A16, path=A16, out=A16, ws=A16, wb=1 << 20, st=None)
        a.update(kw)
        return lib.spec_verify_tree_stochastic(*a.values())

    assert t(B=0, x=None, par=None, tok=None) == OK
    for T in (0.0, -1.0, float("inf"), float("nan"), 1e-40):
        assert t(T=T) == INVALID, T
    assert t(N=0) == INVALID
    assert t(N=65) == INVALID
    assert t(B=-1) == INVALID
    assert t(sn=-8) == INVALID
    assert t(par=None) == INVALID
    assert t(tok=None) == INVALID
    assert t(path=None) == INVALID
    assert t(ws=None) == INVALID
    assert t(dt=3) == INVALID
    assert t(x=A16 + 1) == MISALIGNED
    assert t(par=A16 + 2) == MISALIGNED
    assert t(out=A16 + 1) == MISALIGNED
    assert t(ws=A16 + 8) == MISALIGNED
    assert t(wb=64) == WORKSPACE


def test_commit_validation(lib):
    def c(**kw):
        a = dict(acc=A16, out=A16, B=2, k=4, lens=A16, buf=A16, stride=16, cap=16, nxt=A16,
                 ws=None, st=None)
        a.update(kw)
        return lib.spec_verify_commit(*a.values())

    assert c(B=0, acc=None, out=None, lens=None, buf=None) == OK
    assert c(B=-1) == INVALID
    assert c(k=33) == INVALID
    assert c(cap=-1) == INVALID
    assert c(stride=8) == INVALID  # row stride below the capacity
    assert c(acc=None) == INVALID
    assert c(lens=None) == INVALID
    assert c(buf=None) == INVALID
    assert c(out=A16 + 2) == MISALIGNED
    assert c(nxt=A16 + 1) == MISALIGNED
    assert c(ws=A16 + 4) == MISALIGNED


def test_philox_and_workspace_validation(lib):
    assert lib.spec_verify_philox4x32_10(None, 0, 0, None, None) == OK
    assert lib.spec_verify_philox4x32_10(None, 4, 0, A16, None) == INVALID
    assert lib.spec_verify_philox4x32_10(A16 + 4, 4, 0, A16, None) == MISALIGNED
    assert lib.spec_verify_workspace_init(None, 16, None) == INVALID
    assert lib.spec_verify_workspace_init(A16 + 4, 16, None) == MISALIGNED
    flags = ctypes.c_uint32()
    assert lib.spec_verify_read_device_status(None, ctypes.byref(flags), 0, None) == INVALID


def test_binding_refuses_cpu_tensors():
    import torch

    t = torch.zeros(1, 2, 8)
    with pytest.raises(TypeError):
        sv.greedy(t, torch.zeros(1, 1, dtype=torch.int32))
