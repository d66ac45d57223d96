"""C-ABI library: loads, exports every declared symbol, rejects bad arguments on the host.

No GPU is needed: every call below fails validation before any CUDA call is made.
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from adaptive_block_sparse_b200 import build as b
    b.build()
    import adaptive_block_sparse_b200 as nb
    return nb.load_library()


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "nabla.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(nabla_[a-z_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = _declared_functions()
    for n in ("nabla_reorder", "nabla_build_mask", "nabla_attn_fwd", "nabla_attn_bwd"):
        assert n in names
    assert len(names) >= 10


def test_library_exports_every_declared_symbol(lib):
    import adaptive_block_sparse_b200 as nb
    for name in _declared_functions():
        assert hasattr(lib, name), name
    assert set(nb.EXPORTED) == set(_declared_functions())


def test_library_is_built_for_sm100a():
    from adaptive_block_sparse_b200 import build as b
    assert "arch=compute_100a,code=sm_100a" in " ".join(b.ARCH)


def _shape(nb, **kw):
    base = dict(B=1, H=2, T=2, Hg=16, W=16, D=64, P=8)
    base.update(kw)
    return nb._Shape(*[base[k] for k in ("B", "H", "T", "Hg", "W", "D", "P")])


def test_host_validation_rejects_bad_arguments(lib):
    import adaptive_block_sparse_b200 as nb
    A = ctypes.c_void_p(0x10000)       # fake, aligned, never dereferenced
    Bp = ctypes.c_void_p(0x20000000)
    mis = ctypes.c_void_p(0x10008)     # not 16-byte aligned
    st = ctypes.c_void_p(0)
    good = _shape(nb)
    INV, UNS, WS = nb.NABLA_ERR_INVALID_ARG, nb.NABLA_ERR_UNSUPPORTED, nb.NABLA_ERR_WORKSPACE
    # shapes
    BF, F32, F16 = nb.NABLA_BF16, nb.NABLA_F32, nb.NABLA_F16

    def ro(src=A, sd=BF, dst=Bp, dd=BF, pool=None, shape=good, inv=0):
        return lib.nabla_reorder(src, sd, dst, dd, pool, shape, inv, st)
    assert ro(shape=_shape(nb, Hg=12)) == INV
    assert ro(shape=_shape(nb, D=96)) == UNS
    assert ro(shape=_shape(nb, P=4)) == UNS
    assert ro(shape=_shape(nb, B=0)) == INV
    # pointers and dtypes
    assert ro(src=None) == INV
    assert ro(src=mis) == INV
    assert ro(dst=A) == INV                                               # overlap
    assert ro(pool=A, inv=1) == INV                                       # pool with inverse
    assert ro(dst=None) == INV                                            # no dst and no pool
    assert ro(dst=None, pool=ctypes.c_void_p(0x20000004)) == INV          # misaligned pool
    assert ro(dst=None, inv=1, pool=None) == INV                          # inverse needs dst
    assert ro(sd=F16) == INV                                              # forward needs bf16 source
    assert ro(dd=F32) == INV                                              # no f32 forward output
    assert ro(sd=F32, dd=BF, inv=1) == INV                                # inverse keeps the dtype
    assert ro(inv=3) == INV                                               # unknown direction
    assert ro(inv=-1) == INV
    assert ro(inv=2, dd=F32) == INV                                       # keep-order: bf16 or fp16 out
    assert ro(inv=2, dst=None, pool=A) == INV                             # keep-order needs dst
    win = nb._Window(0, 0, 0)
    ws_need = lib.nabla_mask_workspace_bytes(good)
    assert ws_need > 256

    def bm(thr=0.5, window=win, scale=0.125, bits=A, ridx=None, rcnt=None, ws=Bp, wsb=ws_need, layout=0):
        return lib.nabla_build_mask(A, A, None, None, good, thr, window, scale, bits, ridx, rcnt,
                                    None, None, layout, ws, wsb, st)
    assert bm(thr=1.5) == INV
    assert bm(thr=-0.1) == INV
    assert bm(thr=float("nan")) == INV
    assert bm(window=nb._Window(2, 3, 3)) == INV                          # even window
    assert bm(window=nb._Window(3, 0, 3)) == INV
    assert bm(scale=0.0) == INV
    assert bm(bits=None) == INV
    assert bm(ridx=A, rcnt=None) == INV                                   # list without count
    assert bm(wsb=ws_need - 1) == WS
    assert bm(ws=None) == WS
    assert bm(ws=ctypes.c_void_p(0x20000010)) == WS                       # misaligned workspace
    assert bm(layout=2) == INV                                            # unknown layout
    thr3 = (ctypes.c_double * 3)(0.5, 0.8, 0.95)

    def sw(thrs=thr3, n=3, window=win, bits=A, ws=Bp, wsb=ws_need, qp=A):
        return lib.nabla_build_mask_sweep(None, None, qp, qp, good, ctypes.cast(thrs, ctypes.c_void_p)
                                          if thrs is not None else None, n, window, 0.125, bits, None,
                                          ws, wsb, st)
    assert sw(n=0) == INV
    assert sw(n=65) == INV
    assert sw(thrs=None) == INV
    assert sw(thrs=(ctypes.c_double * 3)(0.5, 1.5, 0.8)) == INV              # thr out of range
    assert sw(thrs=(ctypes.c_double * 3)(0.5, float("nan"), 0.8)) == INV
    assert sw(window=nb._Window(2, 3, 3)) == INV
    assert sw(bits=None) == INV
    assert sw(qp=None) == INV                                                  # no Q, K, nor pools
    assert sw(wsb=ws_need - 1) == WS
    fws = lib.nabla_fwd_workspace_bytes(good)

    def fwd(q=A, o=Bp, scale=0.125, odt=0, ws=Bp, wsb=fws, ridx=A, vdt=0, layout=0):
        return lib.nabla_attn_fwd(q, A, A, vdt, ridx, good, scale, o, odt, None, layout, ws, wsb, st)
    assert fwd(q=None) == INV
    assert fwd(q=mis) == INV
    assert fwd(ridx=None) == INV
    assert fwd(scale=-1.0) == INV
    assert fwd(odt=7) == INV
    assert fwd(odt=2) == INV
    assert fwd(vdt=1) == INV
    assert fwd(wsb=fws - 1) == WS
    assert fwd(layout=2) == INV                                            # unknown layout
    bws = lib.nabla_bwd_workspace_bytes(good)
    assert bws > 256

    def bwd(q=A, lse=A, vdt=0, odt=0, cidx=A, scale=0.125, dq=Bp, layout=0, ws=Bp, wsb=bws):
        return lib.nabla_attn_bwd(q, A, A, vdt, A, odt, A, lse, A, A, cidx, A, good, scale, dq, Bp,
                                  Bp, layout, ws, wsb, st)
    assert bwd(q=None) == INV
    assert bwd(q=mis) == INV
    assert bwd(lse=None) == INV
    assert bwd(cidx=None) == INV
    assert bwd(cidx=ctypes.c_void_p(0x10002)) == INV                      # lists need 4-byte alignment
    assert bwd(vdt=1) == INV                                              # V is bf16 or fp16
    assert bwd(odt=2) == INV                                              # O is bf16 or f32
    assert bwd(scale=float("inf")) == INV
    assert bwd(dq=None) == INV
    assert bwd(layout=2) == INV                                           # unknown layout
    assert bwd(wsb=bws - 1) == WS
    assert bwd(ws=ctypes.c_void_p(0x20000010)) == WS                      # misaligned workspace
    assert lib.nabla_fwd_workspace_bytes(_shape(nb, D=96)) == 0
    assert lib.nabla_status_string(3) == b"NABLA_ERR_WORKSPACE"
    assert lib.nabla_selftest_bounded_wait(None, 256, st) == WS
    assert lib.nabla_selftest_bounded_wait(Bp, 255, st) == WS
    assert lib.nabla_selftest_bounded_wait(ctypes.c_void_p(0x20000010), 256, st) == WS   # misaligned
