"""The C-ABI library on a host without a GPU: it builds, loads, exports every symbol that
include/ra.h declares, and rejects invalid arguments with status codes before touching
the device (no compute call is made here)."""

import ctypes
import os
import re

import pytest

from sequence_softmax_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ra.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.load()


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ra_[a-z_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for name in ("ra_partial", "ra_merge", "ra_ring_forward", "ra_status_string", "ra_get_device_error"):
        assert name in syms


def test_every_declared_symbol_is_exported(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
    assert set(declared_symbols()) == set(binding.SIGNATURES)


def test_abi_version_and_status_strings(lib):
    assert lib.ra_abi_version() == 4
    from sequence_softmax_b200 import binding
    assert binding.ABI_VERSION == lib.ra_abi_version()
    assert binding.load().ra_abi_version() == binding.ABI_VERSION
    for code in range(6):
        s = binding.status_string(code)
        assert s.startswith("RA_")
    assert binding.status_string(99) == "RA_UNKNOWN_STATUS"


FAKE = ctypes.c_void_p(0x10000)  # never dereferenced: every call below fails validation first
FAKE_2 = ctypes.c_void_p(0x10002)  # 2-byte aligned only
FAKE_8 = ctypes.c_void_p(0x10008)  # 8-byte aligned only


def _ring(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, dt=1, B=1, H=1, N=256, d=128, scale=0.1, n_chunks=2, causal=1,
             layout=0, o=FAKE, lse=None, stream=None)
    a.update(kw)
    return lib.ra_ring_forward(*a.values())


@pytest.mark.parametrize("kw,code", [
    (dict(n_chunks=0), binding.RA_ERR_INVALID_ARG),
    (dict(N=250, n_chunks=4), binding.RA_ERR_INVALID_ARG),            # N % P != 0
    (dict(N=256, n_chunks=3, layout=2), binding.RA_ERR_INVALID_ARG),  # zig-zag needs N % 2P == 0
    (dict(layout=7), binding.RA_ERR_INVALID_ARG),
    (dict(scale=0.0), binding.RA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), binding.RA_ERR_INVALID_ARG),
    (dict(causal=2), binding.RA_ERR_INVALID_ARG),
    (dict(dt=5), binding.RA_ERR_INVALID_ARG),
    (dict(d=96), binding.RA_ERR_UNSUPPORTED),                         # bf16 needs d in {64, 128}
    (dict(dt=0, d=160), binding.RA_ERR_UNSUPPORTED),                  # fp32 needs d <= 128
    (dict(B=-1), binding.RA_ERR_INVALID_ARG),
    (dict(q=ctypes.c_void_p(0x10008)), binding.RA_ERR_INVALID_ARG),  # 8-byte aligned only
    (dict(o=None), binding.RA_ERR_INVALID_ARG),
])
def test_ring_forward_rejects(lib, kw, code):
    assert _ring(lib, **kw) == code


Q_, K_, V_ = (ctypes.c_void_p(a) for a in (0x1000000, 0x2000000, 0x3000000))  # 64 KB tensors, 16 MB apart


@pytest.mark.parametrize("o,lse", [
    (ctypes.c_void_p(0x1008000), None),          # o inside q
    (ctypes.c_void_p(0x2FFFF00), None),          # o runs into k
    (V_, None),                                  # o is v
    (ctypes.c_void_p(0x5000000), ctypes.c_void_p(0x3000400)),  # lse inside v
    (ctypes.c_void_p(0x5000000), ctypes.c_void_p(0x5008000)),  # lse inside o
])
def test_ring_forward_rejects_overlapping_outputs(lib, o, lse):
    """o and lse are written, and hold key-norm values before the attention kernel runs, so
    neither may share memory with q, k, v or the other."""
    assert _ring(lib, q=Q_, k=K_, v=V_, o=o, lse=lse) == binding.RA_ERR_INVALID_ARG


def test_ring_forward_empty_is_noop(lib):
    assert _ring(lib, N=0) == binding.RA_OK
    assert _ring(lib, B=0) == binding.RA_OK
    assert _ring(lib, H=0) == binding.RA_OK


def _partial(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, dt=1, B=1, H=1, Lq=128, Lk=128, d=64, scale=0.1, causal=0,
             q_tok0=0, q_ts=1, k_tok0=0, k_ts=1, o=FAKE, lse=FAKE, stream=None)
    a.update(kw)
    return lib.ra_partial(*a.values())


@pytest.mark.parametrize("kw,code", [
    (dict(Lq=-1), binding.RA_ERR_INVALID_ARG),
    (dict(q_ts=0), binding.RA_ERR_INVALID_ARG),
    (dict(k_ts=-2), binding.RA_ERR_INVALID_ARG),
    (dict(d=32), binding.RA_ERR_UNSUPPORTED),
    (dict(lse=None), binding.RA_ERR_INVALID_ARG),
    (dict(scale=-1.0), binding.RA_ERR_INVALID_ARG),
])
def test_partial_rejects(lib, kw, code):
    assert _partial(lib, **kw) == code


def test_partial_empty_is_noop(lib):
    assert _partial(lib, Lq=0) == binding.RA_OK


def _partial_fold(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, dt=1, B=1, H=1, Lq=128, Lk=128, d=64, scale=0.1, causal=0,
             q_tok0=0, q_ts=1, k_tok0=0, k_ts=1, o=FAKE, lse=FAKE, kmax=None, stream=None)
    a.update(kw)
    return lib.ra_partial_fold(*a.values())


@pytest.mark.parametrize("kw,code", [
    (dict(Lq=-1), binding.RA_ERR_INVALID_ARG),
    (dict(q_ts=0), binding.RA_ERR_INVALID_ARG),
    (dict(d=32), binding.RA_ERR_UNSUPPORTED),
    (dict(lse=None), binding.RA_ERR_INVALID_ARG),
    (dict(o=None), binding.RA_ERR_INVALID_ARG),
    (dict(causal=2), binding.RA_ERR_INVALID_ARG),
    (dict(kmax=FAKE_2), binding.RA_ERR_INVALID_ARG),  # a k_norm_max not 4-byte aligned
])
def test_partial_fold_rejects(lib, kw, code):
    assert _partial_fold(lib, **kw) == code


def test_partial_fold_empty_chunk_leaves_the_state(lib):
    """Lq == 0 and Lk == 0 launch nothing (the state is never touched: FAKE is not a real pointer)."""
    assert _partial_fold(lib, Lq=0) == binding.RA_OK
    assert _partial_fold(lib, Lk=0) == binding.RA_OK


def _key_norm_max(lib, **kw):
    a = dict(k=FAKE, dt=1, B=1, H=2, Lk=128, d=128, out=FAKE, stream=None)
    a.update(kw)
    return lib.ra_key_norm_max(*a.values())


@pytest.mark.parametrize("kw,code", [
    (dict(Lk=-1), binding.RA_ERR_INVALID_ARG),
    (dict(B=-1), binding.RA_ERR_INVALID_ARG),
    (dict(dt=0), binding.RA_ERR_UNSUPPORTED),  # fp32 keys: the fp32 kernel takes every row max
    (dict(d=32), binding.RA_ERR_UNSUPPORTED),
    (dict(B=65536, H=65536), binding.RA_ERR_UNSUPPORTED),  # B * H beyond 2^31 - 1
    (dict(out=None), binding.RA_ERR_INVALID_ARG),
    (dict(out=FAKE_2), binding.RA_ERR_INVALID_ARG),
    (dict(k=None), binding.RA_ERR_INVALID_ARG),
    (dict(k=FAKE_8), binding.RA_ERR_INVALID_ARG),  # keys not 16-byte aligned
    (dict(out=ctypes.c_void_p(0x10100)), binding.RA_ERR_INVALID_ARG),  # inside the keys
])
def test_key_norm_max_rejects(lib, kw, code):
    assert _key_norm_max(lib, **kw) == code


def test_key_norm_max_no_heads_is_noop(lib):
    assert _key_norm_max(lib, B=0) == binding.RA_OK


def _merge(lib, **kw):
    a = dict(o=FAKE, lse=FAKE, n=2, rows=16, d=128, out=FAKE, out_dt=1, lse_out=None, stream=None)
    a.update(kw)
    return lib.ra_merge(*a.values())


@pytest.mark.parametrize("kw,code", [
    (dict(n=0), binding.RA_ERR_INVALID_ARG),
    (dict(d=6), binding.RA_ERR_INVALID_ARG),       # d % 4 != 0
    (dict(out_dt=3), binding.RA_ERR_INVALID_ARG),
    (dict(n=65), binding.RA_ERR_UNSUPPORTED),
    (dict(rows=-1), binding.RA_ERR_INVALID_ARG),
    (dict(out=None), binding.RA_ERR_INVALID_ARG),
])
def test_merge_rejects(lib, kw, code):
    assert _merge(lib, **kw) == code


def test_merge_empty_is_noop(lib):
    assert _merge(lib, rows=0) == binding.RA_OK


def _ring_bwd(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, d_o=FAKE, lse=FAKE, dt=1, B=1, H=2, N=256, d=128, scale=0.1,
             n_chunks=2, causal=1, layout=2, dq=FAKE, dk=FAKE, dv=FAKE, ws=FAKE, ws_bytes=1 << 30, stream=None)
    a.update(kw)
    return lib.ra_ring_backward(*a.values())


@pytest.mark.parametrize("kw,code", [
    (dict(n_chunks=0), binding.RA_ERR_INVALID_ARG),
    (dict(N=256, n_chunks=3), binding.RA_ERR_INVALID_ARG),           # zig-zag needs N % 2P == 0
    (dict(layout=9), binding.RA_ERR_INVALID_ARG),
    (dict(scale=0.0), binding.RA_ERR_INVALID_ARG),
    (dict(d=96), binding.RA_ERR_UNSUPPORTED),
    (dict(ws_bytes=1000), binding.RA_ERR_INVALID_ARG),               # workspace too small (needs 2048)
    (dict(ws=None), binding.RA_ERR_INVALID_ARG),
    (dict(lse=ctypes.c_void_p(0x10002)), binding.RA_ERR_INVALID_ARG),
    (dict(dk=ctypes.c_void_p(0x10004)), binding.RA_ERR_INVALID_ARG),
])
def test_ring_backward_rejects(lib, kw, code):
    assert _ring_bwd(lib, **kw) == code


def test_ring_backward_workspace_size(lib):
    f = lib.ra_ring_backward_workspace_bytes
    assert f(1, 1, 2, 256, 128) == 2 * 256 * 4            # D, one fp32 per query row
    assert f(0, 1, 2, 256, 16) == 2 * 256 * 4
    assert f(1, -1, 2, 256, 128) == -1
    assert _ring_bwd(lib, ws_bytes=f(1, 1, 2, 256, 128) - 1) == binding.RA_ERR_INVALID_ARG
    assert _ring_bwd(lib, N=0) == binding.RA_OK


def _partial_bwd(lib, **kw):
    a = dict(q=FAKE, k=FAKE, v=FAKE, d_o=FAKE, lse=FAKE, delta=FAKE, dt=1, B=1, H=1, Lq=128, Lk=128, d=64,
             scale=0.1, causal=1, q_tok0=0, q_ts=1, k_tok0=0, k_ts=1, dq=FAKE, dk=FAKE, dv=FAKE, stream=None)
    a.update(kw)
    return lib.ra_partial_backward(*a.values())


@pytest.mark.parametrize("kw,code", [
    (dict(Lk=-1), binding.RA_ERR_INVALID_ARG),
    (dict(q_ts=0), binding.RA_ERR_INVALID_ARG),
    (dict(d=32), binding.RA_ERR_UNSUPPORTED),
    (dict(delta=None), binding.RA_ERR_INVALID_ARG),
    (dict(dq=ctypes.c_void_p(0x10008)), binding.RA_ERR_INVALID_ARG),
    (dict(causal=3), binding.RA_ERR_INVALID_ARG),
])
def test_partial_backward_rejects(lib, kw, code):
    assert _partial_bwd(lib, **kw) == code


def test_partial_backward_empty_is_noop(lib):
    assert _partial_bwd(lib, Lq=0) == binding.RA_OK
    assert _partial_bwd(lib, Lk=0) == binding.RA_OK


@pytest.mark.parametrize("kw,code", [
    (dict(rows=-1), binding.RA_ERR_INVALID_ARG),
    (dict(d=96), binding.RA_ERR_UNSUPPORTED),
    (dict(delta=None), binding.RA_ERR_INVALID_ARG),
    (dict(rows=0), binding.RA_OK),
])
def test_backward_delta_rejects(lib, kw, code):
    a = dict(o=FAKE, d_o=FAKE, dt=1, rows=16, d=128, delta=FAKE, stream=None)
    a.update(kw)
    assert lib.ra_backward_delta(*a.values()) == code


def test_product_path_does_not_reach_the_oracle():
    """The CUDA path's sources never import or link the CPU oracle."""
    pkg = os.path.join(ROOT, "sequence_softmax_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f


def test_host_pipeline_groups_cover_every_row_once():
    """The host-buffer forward's head groups: contiguous, non-empty, covering [0, BH), with
    the first and last groups no larger than the middle ones (their copies are not hidden)."""
    from sequence_softmax_b200.binding import _pipeline_bounds
    for BH in range(1, 70):
        for G in range(1, min(BH, 6) + 1):
            b = _pipeline_bounds(BH, G)
            assert b[0] == 0 and b[-1] == BH and len(b) == G + 1
            sizes = [b[i + 1] - b[i] for i in range(G)]
            assert all(s >= 1 for s in sizes), (BH, G, b)
            if G >= 3:
                assert max(sizes[0], sizes[-1]) <= min(sizes[1:-1]) + 1, (BH, G, sizes)
    assert _pipeline_bounds(8, 4) == [0, 1, 4, 7, 8]
