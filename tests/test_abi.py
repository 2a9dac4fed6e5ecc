"""Host-only checks of the C ABI: the library loads, exports every entry point
that include/qattn.h declares, and refuses invalid arguments by name before
touching the GPU (so these run without a device)."""
import ctypes
import os
import re

import pytest

import quantized_exact_attention_qattn_b200 as qa
from quantized_exact_attention_qattn_b200 import _lib
from quantized_exact_attention_qattn_b200 import build as qbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qattn.h")


@pytest.fixture(scope="module")
def lib():
    qbuild.build()
    return qa.load()


PROBE_HEADER = os.path.join(ROOT, "include", "qattn_probe.h")


def declared_functions(path=HEADER):
    src = open(path).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(qattn_\w+)\s*\(", src)))


def test_header_declares_the_expected_entry_points():
    names = declared_functions()
    assert set(names) == set(_lib.EXPORTED), names
    assert set(declared_functions(PROBE_HEADER)) == set(_lib.EXPORTED_PROBE)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions() + declared_functions(PROBE_HEADER):
        assert hasattr(lib, name), name
    assert lib.qattn_version().decode().startswith("qattn-b200")


def _view(ptr=0x1000, strides=(1 << 20, 512, 128, 1)):
    v = _lib.BNHD()
    v.ptr = ptr
    for i, s in enumerate(strides):
        v.stride[i] = s
    return v


FAKE = 0x7f0000001000        # never dereferenced: every call below is refused first


def test_fwd_refusals(lib):
    args = dict(B=1, Nq=128, Nkv=128, Hq=2, Hkv=2, D=128)

    def call(**kw):
        a = dict(args, **kw)
        return lib.qattn_fwd(a["B"], a["Nq"], a["Nkv"], a["Hq"], a["Hkv"], a["D"], kw.get("q8", FAKE),
                             FAKE, FAKE, FAKE, kw.get("mode", 0), FAKE, FAKE,
                             kw.get("sm_scale", 0.0), kw.get("out", FAKE), kw.get("err", FAKE), None)
    assert call(D=96) == 4
    assert call(Hq=3) == 4
    assert call(Nq=0) == 2
    assert call(B=-1) == 2
    assert call(mode=3) == 4
    assert call(mode=-1) == 4
    assert call(sm_scale=-1.0) == 4
    assert call(sm_scale=float("nan")) == 4
    assert call(q8=None) == 1
    assert call(err=None) == 1
    assert call(out=FAKE + 2) == 3
    assert "16-byte" in lib.qattn_last_error().decode()


def test_prep_refusals(lib):
    def call(rot=96, q=None, D=128, eps=1e-5, theta=10000.0):
        return lib.qattn_prep(1, 8, 2, 2, D, q or _view(), _view(), FAKE, FAKE, eps, rot, theta, 0,
                              FAKE, FAKE, None)
    assert call(rot=95) == 4
    assert call(rot=8) == 4              # not a multiple of 16
    assert call(rot=144) == 4            # larger than D
    assert call(theta=0.0) == 4
    assert call(eps=-1.0) == 4
    assert call(D=100) == 4
    assert call(q=_view(strides=(1 << 20, 512, 128, 2))) == 3
    assert call(q=_view(strides=(1 << 20, 516, 128, 1))) == 3
    assert call(q=_view(ptr=FAKE + 8)) == 3
    assert call(q=_view(ptr=0)) == 1


def test_quant_refusals_and_workspace_query(lib):
    need = lib.qattn_quant_workspace_bytes(1, 37810, 56, 128)
    nk = (37810 + 63) // 64
    assert need >= nk * 56 * 128 * (8 + 4) + 56 * 128 * 4
    assert lib.qattn_quant_workspace_bytes(1, 0, 56, 128) == 0
    assert lib.qattn_quant_workspace_bytes(1, 10, 56, 96) == 0

    def call(ws=FAKE, nbytes=None, v=None, k_mean=FAKE):
        return lib.qattn_quant(1, 37810, 37810, 56, 56, 128, _view(), _view(), v or _view(),
                               FAKE, FAKE, FAKE, FAKE, k_mean, FAKE, FAKE, ws,
                               need if nbytes is None else nbytes, None)
    assert call(nbytes=need - 1) == 5
    assert call(ws=None) == 5
    assert call(k_mean=None) == 1
    assert call(v=_view(strides=(1 << 20, 512, 100, 1))) == 3
    assert "workspace" in (lib.qattn_quant(1, 64, 64, 1, 1, 128, _view(), _view(), _view(), FAKE,
                                           FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, None) and
                           lib.qattn_last_error().decode())


def test_hadamard_needs_power_of_four_head_dim(lib):
    need = lib.qattn_quant_workspace_bytes(1, 64, 1, 128)
    st = lib.qattn_quant_hadamard(1, 64, 64, 1, 1, 128, _view(), _view(), _view(), FAKE, FAKE,
                                  FAKE, FAKE, FAKE, FAKE, FAKE, need, None)
    assert st == 4 and "Hadamard" in lib.qattn_last_error().decode()


def test_scores_refusals(lib):
    def call(tiles=FAKE, n=4, s_out=FAKE, D=128, mode=0, out=FAKE):
        return lib.qattn_scores(1, 128, 128, 2, 2, D, FAKE, FAKE, FAKE, FAKE, mode, FAKE, FAKE, 0.0,
                                tiles, n, s_out, out, FAKE, None)
    assert call(n=0) == 2
    assert call(n=65537) == 2
    assert call(tiles=None) == 1
    assert call(s_out=None) == 1
    assert call(tiles=FAKE + 4) == 3
    assert call(D=96) == 4                 # then the qattn_fwd checks
    assert call(mode=3) == 4
    assert call(out=None) == 1
    assert lib.qattn_check(None, None) == 1


def test_stall_hook_refuses_negative_tiles_and_resets(lib):
    assert lib.qattn_debug_stall_kv_tile(-2) == 2          # QATTN_ERR_SHAPE
    assert "kv_tile" in lib.qattn_last_error().decode() or "tile" in lib.qattn_last_error().decode()
    assert lib.qattn_debug_stall_kv_tile(-1) == 0          # off (the initial state)


def test_host_pipeline_workspace_query_and_refusals(lib):
    ws = lib.qattn_host_workspace_bytes
    one = ws(1, 37810, 37810, 56, 56, 128, 7)
    # two buffer sets, each at least the chunk's BF16 Q/K/V and output
    assert one >= 2 * 4 * 37810 * 7 * 128 * 2
    assert ws(1, 37810, 37810, 56, 56, 128, 56) == ws(1, 37810, 37810, 56, 56, 128, 500)
    assert ws(1, 37810, 37810, 56, 56, 128, 8) > one
    assert ws(1, 100, 100, 4, 3, 128, 1) == 0        # Hq % Hkv
    assert ws(1, 100, 100, 4, 4, 96, 1) == 0         # head dim
    assert ws(1, 100, 100, 4, 4, 128, 0) == 0        # chunk
    need = ws(1, 256, 256, 2, 2, 128, 1)
    ALIGNED = 0x7f0000010000

    def call(q=None, k=None, v=None, Nq=256, hadamard=0, chunk=1, out=FAKE, ws_ptr=ALIGNED,
             nbytes=need, err=FAKE):
        view = _view(strides=(256 * 2 * 128, 2 * 128, 128, 1))
        return lib.qattn_attention_host(1, Nq, 256, 2, 2, 128, q or view, k or view, v or view,
                                        None, None, 1e-5, 0, 10000.0, hadamard, 0.0, out, chunk,
                                        ws_ptr, nbytes, err, None, None, None, None)
    assert call(chunk=0) == 2
    assert call(hadamard=2) == 4
    assert call(Nq=128) == 4 and "Nq == Nkv" in lib.qattn_last_error().decode()
    assert call(q=_view(ptr=0)) == 1
    assert call(k=_view(strides=(256 * 4 * 128, 4 * 128, 256, 1))) == 3   # heads not back to back
    assert call(out=None) == 1
    assert call(err=None) == 1
    assert call(out=FAKE + 8) == 3
    assert call(nbytes=need - 1) == 5
    assert call(ws_ptr=ALIGNED + 16) == 5


def test_default_host_chunk_rule():
    f = qa.default_kv_heads_per_chunk
    assert f(1, 37810, 37810, 56, 56, 128) == 4        # 1.63 GB of input: ~14 chunks
    assert f(1, 1024, 32768, 16, 4, 256) == 2          # 143 MB, GQA: two heads per chunk
    assert f(32, 729, 729, 16, 16, 64) == 4            # 143 MB: four chunks
    assert f(1, 256, 256, 2, 2, 128) == 1              # two KV heads: one per chunk
    assert f(1, 256, 256, 1, 1, 128) == 1
    for args in [(1, 37810, 37810, 56, 56, 128), (2, 5000, 5000, 8, 2, 128), (1, 9000, 9000, 3, 3, 64)]:
        c = f(*args)
        assert 1 <= c <= args[4]


def test_tc_probe_refusals(lib):
    assert lib.qattn_tc_probe(2, 100, 148, FAKE, FAKE, None) == 2
    assert lib.qattn_tc_probe(0, 0, 148, FAKE, FAKE, None) == 2
    assert lib.qattn_tc_probe(0, (1 << 20) + 1, 148, FAKE, FAKE, None) == 2
    assert lib.qattn_tc_probe(1, 100, 0, FAKE, FAKE, None) == 2
    assert lib.qattn_tc_probe(1, 100, 148, None, FAKE, None) == 1
    assert lib.qattn_tc_probe(1, 100, 148, FAKE, None, None) == 1


def test_fp16_pv_refusals(lib):
    def fwd(Nkv=128, cap=128, mode=1, v=FAKE):
        return lib.qattn_fwd_pv16(1, 128, Nkv, 2, 2, 128, FAKE, FAKE, FAKE, FAKE, mode, v, cap, 0.0,
                                  FAKE, FAKE, None)
    assert fwd(cap=120) == 2                 # below Nkv
    assert fwd(mode=3) == 4
    assert fwd(v=None) == 1
    assert fwd(v=FAKE + 8) == 3

    def v16(N=100, cap=104, out=FAKE):
        return lib.qattn_quant_v16(1, N, 2, 128, _view(), out, cap, None)
    assert v16(cap=96) == 2
    assert v16(cap=102) == 2
    assert v16(out=None) == 1
    assert v16(out=FAKE + 4) == 3
    assert v16(N=0) == 2


def test_quant_k32_refuses_like_quant(lib):
    need = lib.qattn_quant_workspace_bytes(1, 64, 1, 128)
    assert lib.qattn_quant_k32(1, 64, 64, 1, 1, 128, _view(), _view(), _view(), FAKE, FAKE, FAKE,
                               FAKE, FAKE, FAKE, FAKE, FAKE, need - 1, None) == 5
    assert lib.qattn_quant_k32(1, 64, 64, 1, 1, 96, _view(), _view(), _view(), FAKE, FAKE, FAKE,
                               FAKE, FAKE, FAKE, FAKE, FAKE, need, None) == 4


def test_int8v_refusals(lib):
    assert lib.qattn_fwd_int8v(1, 128, 128, 2, 2, 128, FAKE, FAKE, FAKE, FAKE, 0, FAKE, FAKE, 0.0,
                               FAKE, FAKE, None) == 4          # D must be 256
    assert lib.qattn_quant_v_rotated(1, 128, 2, 128, _view(), FAKE, FAKE, FAKE, 1 << 20, None) == 4
    assert lib.qattn_quant_v_rotated(1, 128, 2, 256, _view(), None, FAKE, FAKE, 1 << 20, None) == 1
    assert lib.qattn_quant_v_rotated(1, 128, 2, 256, _view(), FAKE, FAKE, FAKE, 16, None) == 5
