"""CPU-side checks of the C-ABI boundary: the library loads, exports every
symbol include/lserve.h declares, and host-side validation rejects bad
arguments with the documented status codes before touching the GPU."""
import ctypes
import os
import re

import pytest

import block_sparse_attention_page_b200 as lserve

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    with open(os.path.join(ROOT, "include", "lserve.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"\b(lserve_[a-z_]+)\s*\(", text)))


def test_header_declares_the_four_hot_path_calls():
    names = _declared()
    for n in ["lserve_page_stats", "lserve_page_select", "lserve_sparse_decode_attn",
              "lserve_blocksparse_prefill"]:
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(lserve.library_path())
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing
    assert set(_declared()) <= set(lserve.EXPORTED)


def test_status_strings():
    for s in range(7):
        assert lserve.status_string(s)
    assert lserve.status_string(0) == "ok"


def _desc(**kw):
    d = dict(B=1, H_q=4, H_kv=2, D=64, N_L=16, N_P=64, max_pages=32, num_pool_pages=32)
    d.update(kw)
    return lserve.paged_desc(d["B"], d["H_q"], d["H_kv"], d["D"], d["N_L"], d["N_P"],
                             d["max_pages"], d["num_pool_pages"])


FAKE = ctypes.c_void_p(1 << 20)        # aligned, never dereferenced on failing paths
MISALIGNED = ctypes.c_void_p((1 << 20) + 2)


def _stats(desc, k=FAKE, first=0):
    return lserve.lib.lserve_page_stats(ctypes.byref(desc), k, FAKE, FAKE, FAKE, FAKE, first, None)


def _select(desc, top_k=8, q=FAKE, ws=None, ws_bytes=0):
    return lserve.lib.lserve_page_select(ctypes.byref(desc), q, FAKE, FAKE, FAKE, FAKE, top_k, FAKE,
                                         FAKE, None, ws, ws_bytes, None)


def _decode(desc, top_k=8, sink=64, local=256, scale=0.125, out=FAKE, ws=None, ws_bytes=0):
    return lserve.lib.lserve_sparse_decode_attn(ctypes.byref(desc), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                                FAKE, FAKE, top_k, sink, local, scale, out, None, ws,
                                                ws_bytes, None)


@pytest.mark.parametrize("bad", [dict(B=0), dict(H_kv=0), dict(H_q=3), dict(N_P=40), dict(N_L=0),
                                 dict(max_pages=0), dict(num_pool_pages=0)])
def test_invalid_shapes_are_rejected(bad):
    d = _desc(**bad)
    assert _stats(d) == lserve.ERR_INVALID_ARG
    assert _select(d) == lserve.ERR_INVALID_ARG
    assert _decode(d) == lserve.ERR_INVALID_ARG


@pytest.mark.parametrize("bad", [dict(D=96), dict(D=256), dict(H_q=6, H_kv=2), dict(N_L=4, N_P=64),
                                 dict(N_P=48, N_L=16)])
def test_unsupported_shapes(bad):
    d = _desc(**bad)
    assert _stats(d) == lserve.ERR_UNSUPPORTED
    assert _decode(d) == lserve.ERR_UNSUPPORTED


def test_null_and_misaligned_pointers():
    d = _desc()
    assert lserve.lib.lserve_page_stats(None, FAKE, FAKE, FAKE, FAKE, FAKE, 0, None) == \
        lserve.ERR_INVALID_ARG
    assert _stats(d, k=None) == lserve.ERR_INVALID_ARG
    assert _stats(d, k=MISALIGNED) == lserve.ERR_INVALID_ARG
    assert _stats(d, first=-1) == lserve.ERR_INVALID_ARG
    assert _select(d, q=MISALIGNED) == lserve.ERR_INVALID_ARG
    assert _decode(d, out=None) == lserve.ERR_INVALID_ARG
    assert _decode(d, out=MISALIGNED) == lserve.ERR_INVALID_ARG


def test_bad_scalars():
    d = _desc()
    assert _select(d, top_k=0) == lserve.ERR_INVALID_ARG
    assert _select(d, top_k=33) == lserve.ERR_INVALID_ARG
    assert _decode(d, top_k=0) == lserve.ERR_INVALID_ARG
    assert _decode(d, sink=-1) == lserve.ERR_INVALID_ARG
    assert _decode(d, local=-5) == lserve.ERR_INVALID_ARG
    assert _decode(d, scale=float("nan")) == lserve.ERR_INVALID_ARG


def test_missing_workspace_is_reported():
    # select without phys_scores needs a workspace; the check precedes any launch
    assert _select(_desc()) == lserve.ERR_WORKSPACE
    assert _select(_desc(), ws=FAKE, ws_bytes=16) == lserve.ERR_WORKSPACE


def test_prefill_rejects_bad_descriptors():
    hk = (ctypes.c_uint8 * 2)(0, 1)
    for bad in [lserve.prefill_desc(0, 4, 2, 64, 64, 1, 4), lserve.prefill_desc(128, 4, 3, 64, 64, 1, 4)]:
        st = lserve.lib.lserve_blocksparse_prefill(ctypes.byref(bad), FAKE, FAKE, FAKE,
                                                   ctypes.cast(hk, ctypes.c_void_p), 0.125, FAKE,
                                                   None, None, 0, None)
        assert st in (lserve.ERR_INVALID_ARG, lserve.ERR_UNSUPPORTED)


def test_prefill_paged_rejects_bad_arguments():
    # every check precedes a launch: bad paged descriptors, mismatched heads /
    # head_dim, a table too short for the sequence, null or misaligned pools
    hk = (ctypes.c_uint8 * 2)(0, 1)
    d = lserve.prefill_desc(1000, 4, 2, 64, 64, 1, 4)
    good = lserve.paged_desc(1, 4, 2, 64, 16, 64, 16, 32)

    def call(pd, bt=FAKE, kp=FAKE, vp=FAKE, sp=FAKE, desc=d):
        return lserve.lib.lserve_blocksparse_prefill_paged(
            ctypes.byref(desc), ctypes.byref(pd), FAKE, FAKE, FAKE, ctypes.cast(hk, ctypes.c_void_p),
            0.125, FAKE, None, bt, kp, vp, sp, None, 0, None)

    assert call(lserve.paged_desc(1, 4, 2, 64, 16, 40, 16, 32)) == lserve.ERR_INVALID_ARG  # N_P % N_L
    assert call(lserve.paged_desc(1, 4, 2, 128, 16, 64, 16, 32)) == lserve.ERR_INVALID_ARG  # head_dim
    assert call(lserve.paged_desc(1, 4, 4, 64, 16, 64, 16, 32)) == lserve.ERR_INVALID_ARG  # H_kv
    assert call(lserve.paged_desc(1, 4, 2, 64, 16, 64, 15, 32)) == lserve.ERR_INVALID_ARG  # 15 pages < 1000
    assert call(lserve.paged_desc(1, 4, 2, 64, 24, 96, 16, 32)) == lserve.ERR_UNSUPPORTED  # N_L = 24
    assert call(good, bt=None) == lserve.ERR_INVALID_ARG
    assert call(good, kp=None) == lserve.ERR_INVALID_ARG
    assert call(good, sp=ctypes.c_void_p(FAKE.value + 8)) == lserve.ERR_INVALID_ARG
    assert call(good, bt=ctypes.c_void_p(FAKE.value + 2)) == lserve.ERR_INVALID_ARG
    bad = lserve.prefill_desc(0, 4, 2, 64, 64, 1, 4)
    assert call(good, desc=bad) in (lserve.ERR_INVALID_ARG, lserve.ERR_UNSUPPORTED)


def test_workspace_size_of_select():
    d = _desc()
    assert lserve.workspace_size(lserve.OP_SELECT, d) >= 1 * 2 * 32 * 4
    assert lserve.workspace_size(99, d) == 0


def test_decode_ex_rejects_unknown_flags():
    d = _desc()
    for flags in (8, 16, 0x80000000):
        st = lserve.lib.lserve_sparse_decode_attn_ex(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE,
                                                     FAKE, FAKE, FAKE, 8, 64, 256, 0.125, FAKE, None,
                                                     flags, None, 0, None)
        assert st == lserve.ERR_INVALID_ARG
    # a known flag passes the flag check and fails later: on the missing
    # workspace (GPU present) or on the device query (no GPU here)
    st = lserve.lib.lserve_sparse_decode_attn_ex(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                                 FAKE, FAKE, 8, 64, 256, 0.125, FAKE, None,
                                                 lserve.DECODE_OVERLAP_PROLOGUE, None, 0, None)
    assert st in (lserve.ERR_WORKSPACE, lserve.ERR_CUDA)


def _quant(desc, k=FAKE, k8=FAKE, scale=FAKE):
    return lserve.lib.lserve_quantize_pages_kv8(ctypes.byref(desc), k, FAKE, FAKE, FAKE, k8, FAKE, scale,
                                                FAKE, None)


def _decode8(desc, top_k=8, k8=FAKE, scale=FAKE, flags=0, out=FAKE):
    return lserve.lib.lserve_sparse_decode_attn_kv8(ctypes.byref(desc), FAKE, k8, FAKE, scale, FAKE, FAKE,
                                                    FAKE, FAKE, FAKE, FAKE, top_k, 64, 256, 0.125, out,
                                                    None, flags, None, 0, None)


@pytest.mark.parametrize("bad", [dict(B=0), dict(H_kv=0), dict(H_q=3), dict(N_P=40), dict(N_L=0),
                                 dict(max_pages=0), dict(num_pool_pages=0)])
def test_kv8_calls_reject_invalid_shapes(bad):
    d = _desc(**bad)
    assert _quant(d) == lserve.ERR_INVALID_ARG
    assert _decode8(d) == lserve.ERR_INVALID_ARG


@pytest.mark.parametrize("bad", [dict(D=96), dict(H_q=6, H_kv=2), dict(N_P=48, N_L=16)])
def test_kv8_calls_reject_unsupported_shapes(bad):
    d = _desc(**bad)
    assert _quant(d) == lserve.ERR_UNSUPPORTED
    assert _decode8(d) == lserve.ERR_UNSUPPORTED


def test_kv8_calls_reject_null_misaligned_and_bad_scalars():
    d = _desc()
    assert _quant(d, k=None) == lserve.ERR_INVALID_ARG
    assert _quant(d, k8=MISALIGNED) == lserve.ERR_INVALID_ARG
    assert _quant(d, scale=None) == lserve.ERR_INVALID_ARG
    assert _decode8(d, k8=None) == lserve.ERR_INVALID_ARG
    assert _decode8(d, k8=MISALIGNED) == lserve.ERR_INVALID_ARG
    assert _decode8(d, scale=MISALIGNED) == lserve.ERR_INVALID_ARG
    assert _decode8(d, out=None) == lserve.ERR_INVALID_ARG
    assert _decode8(d, top_k=0) == lserve.ERR_INVALID_ARG
    assert _decode8(d, top_k=33) == lserve.ERR_INVALID_ARG
    assert _decode8(d, flags=8) == lserve.ERR_INVALID_ARG
