"""The C-ABI library loads, exports every declared entry point, and rejects bad
arguments on the host before touching any device memory (CPU only)."""
import ctypes
import os
import re

import pytest

from long_context_decode_lr_b200 import build as lrbuild
from long_context_decode_lr_b200 import lowram as lr

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    lrbuild.build()
    return lr.library()


def declared_functions():
    names = set()
    for hdr in os.listdir(os.path.join(ROOT, "include")):
        if hdr.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", hdr)).read()
            txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
            names |= set(re.findall(r"\b(lr_[a-z0-9_]+)\s*\(", txt))
    return sorted(names)


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert "lr_decode_attn" in names and "lr_pack_prefill" in names
    for n in names:
        assert hasattr(lib, n), n


def test_version_and_strings(lib):
    assert lib.lr_abi_version() == 2
    assert lib.lr_status_string(lr.LR_ERR_WORKSPACE) == b"workspace too small"


FAKE = 0x10000  # a 256-byte-aligned address that is never dereferenced


def _shape(**kw):
    d = dict(batch=1, T=1000, n_layers=2, n_kv_heads=2, head_dim=128, rank=128, hidden=256, dtype=lr.LR_BF16)
    d.update(kw)
    return lr.lr_cache_shape(*[d[f] for f, _ in lr.lr_cache_shape._fields_])


def _pred(**kw):
    d = dict(W_lin=FAKE, W1=FAKE, b1=FAKE, W2=FAKE, b2=None, per_sequence=1)
    d.update(kw)
    return lr.lr_predictor(*[d[f] for f, _ in lr.lr_predictor._fields_])


def _decode(lib, shape=None, layer=0, hq=8, q=FAKE, res_idx=FAKE, res_val=FAKE, k=10, blocks=None, n_sel=0,
            pred=None, ws=FAKE, ws_bytes=1 << 40, o=FAKE):
    shape = _shape() if shape is None else shape
    pred = _pred() if pred is None else pred
    return lib.lr_decode_attn(ctypes.byref(shape), layer, hq, q, FAKE, FAKE, ctypes.byref(pred), res_idx,
                              res_val, None, k, blocks, n_sel, 0.0, o, ws, ws_bytes, None)


@pytest.mark.parametrize("kw,status", [
    (dict(layer=2), lr.LR_ERR_INVALID_ARG),
    (dict(layer=-1), lr.LR_ERR_INVALID_ARG),
    (dict(hq=7), lr.LR_ERR_INVALID_ARG),
    (dict(hq=2 * 16), lr.LR_ERR_UNSUPPORTED),
    (dict(k=1001), lr.LR_ERR_INVALID_ARG),
    (dict(k=-1), lr.LR_ERR_INVALID_ARG),
    (dict(q=None), lr.LR_ERR_INVALID_ARG),
    (dict(q=FAKE + 4), lr.LR_ERR_INVALID_ARG),
    (dict(res_idx=None), lr.LR_ERR_INVALID_ARG),
    (dict(o=None), lr.LR_ERR_INVALID_ARG),
    (dict(blocks=FAKE, n_sel=17), lr.LR_ERR_INVALID_ARG),
    (dict(ws=None), lr.LR_ERR_INVALID_ARG),
    (dict(ws=FAKE + 16), lr.LR_ERR_INVALID_ARG),
    (dict(ws_bytes=100), lr.LR_ERR_WORKSPACE),
    (dict(shape=_shape(head_dim=100)), lr.LR_ERR_UNSUPPORTED),
    (dict(shape=_shape(hidden=1024)), lr.LR_ERR_UNSUPPORTED),
    (dict(shape=_shape(rank=0)), lr.LR_ERR_INVALID_ARG),
    (dict(shape=_shape(T=-5)), lr.LR_ERR_INVALID_ARG),
    (dict(shape=_shape(dtype=7)), lr.LR_ERR_INVALID_ARG),
    (dict(pred=_pred(W1=None)), lr.LR_ERR_INVALID_ARG),
    (dict(pred=_pred(per_sequence=2)), lr.LR_ERR_INVALID_ARG),
])
def test_decode_rejects_bad_arguments(lib, kw, status):
    assert _decode(lib, **kw) == status
    assert lib.lr_last_error()


def test_null_shape_and_pack_checks(lib):
    assert lib.lr_decode_attn(None, 0, 8, FAKE, FAKE, FAKE, None, None, None, None, 0, None, 0, 0.0, FAKE,
                              FAKE, 1 << 40, None) == lr.LR_ERR_INVALID_ARG
    shape, pred = _shape(), _pred()
    args = [ctypes.byref(shape), FAKE, FAKE, FAKE, ctypes.byref(pred), 10, FAKE, FAKE, FAKE, None, None, FAKE]
    assert lib.lr_pack_prefill(*args, 16, None) == lr.LR_ERR_WORKSPACE
    bad = list(args)
    bad[5] = 2000
    assert lib.lr_pack_prefill(*bad, 1 << 40, None) == lr.LR_ERR_INVALID_ARG
    bad = list(args)
    bad[1] = None
    assert lib.lr_pack_prefill(*bad, 1 << 40, None) == lr.LR_ERR_INVALID_ARG
    assert lib.lr_topk_tokens(FAKE, 4, 100, 101, FAKE, FAKE, 256, None) == lr.LR_ERR_INVALID_ARG
    assert lib.lr_topk_tokens(FAKE, 4, 100, 10, FAKE, FAKE, 16, None) == lr.LR_ERR_WORKSPACE
    assert lib.lr_residual_block_ptr(FAKE, 4, 10, 100, None, None) == lr.LR_ERR_INVALID_ARG


def test_workspace_sizes_grow_with_work(lib):
    s1, s2 = _shape(T=1000), _shape(T=100000)
    assert 0 < lib.lr_pack_workspace_bytes(ctypes.byref(s1), 10) < lib.lr_pack_workspace_bytes(ctypes.byref(s2), 10)
    assert lib.lr_decode_workspace_bytes(ctypes.byref(s1), 8, 0) >= 256
    assert lib.lr_decode_workspace_bytes(ctypes.byref(_shape(head_dim=12)), 8, 0) == 0


def _decode_tail(lib, tail_K=FAKE, tail_V=FAKE, n_tail=16, ws_bytes=1 << 40):
    shape, pred = _shape(), _pred()
    return lib.lr_decode_attn_tail(ctypes.byref(shape), 0, 8, FAKE, FAKE, FAKE, ctypes.byref(pred), FAKE, FAKE,
                                   None, 10, None, 0, tail_K, tail_V, n_tail, 0.0, FAKE, FAKE, ws_bytes, None)


@pytest.mark.parametrize("kw,status", [
    (dict(n_tail=-1), lr.LR_ERR_INVALID_ARG),
    (dict(n_tail=lr.LR_MAX_TAIL + 1), lr.LR_ERR_INVALID_ARG),
    (dict(tail_K=None), lr.LR_ERR_INVALID_ARG),
    (dict(tail_V=None), lr.LR_ERR_INVALID_ARG),
    (dict(tail_V=FAKE + 8), lr.LR_ERR_INVALID_ARG),
    (dict(ws_bytes=100), lr.LR_ERR_WORKSPACE),
    (dict(tail_K=None, tail_V=None, n_tail=0, ws_bytes=100), lr.LR_ERR_WORKSPACE),  # no tail: NULL is fine
])
def test_decode_tail_rejects_bad_arguments(lib, kw, status):
    """The tail arguments are checked on the host, before any launch."""
    assert _decode_tail(lib, **kw) == status
    assert lib.lr_last_error()


def _select(lib, shape=None, layer=0, hq=8, n_sel=4, ws=FAKE, ws_bytes=1 << 40, blocks=FAKE, abar=FAKE,
            scores=None):
    shape = _shape() if shape is None else shape
    return lib.lr_select_blocks(ctypes.byref(shape), layer, hq, FAKE, abar, FAKE, n_sel, 0.0, blocks, scores,
                                ws, ws_bytes, None)


@pytest.mark.parametrize("kw,status", [
    (dict(layer=2), lr.LR_ERR_INVALID_ARG),
    (dict(hq=7), lr.LR_ERR_INVALID_ARG),
    (dict(hq=2 * 16), lr.LR_ERR_UNSUPPORTED),
    (dict(n_sel=-1), lr.LR_ERR_INVALID_ARG),
    (dict(n_sel=17), lr.LR_ERR_INVALID_ARG),          # T = 1000 has 16 blocks
    (dict(blocks=None), lr.LR_ERR_INVALID_ARG),
    (dict(ws=None), lr.LR_ERR_INVALID_ARG),
    (dict(ws_bytes=100), lr.LR_ERR_WORKSPACE),
    (dict(abar=None), lr.LR_ERR_INVALID_ARG),
    (dict(n_sel=0, abar=None, scores=FAKE), lr.LR_ERR_INVALID_ARG),   # scores asked: Abar needed
    (dict(scores=FAKE + 4), lr.LR_ERR_INVALID_ARG),                     # misaligned scores_out
])
def test_select_blocks_rejects_bad_arguments(lib, kw, status):
    assert _select(lib, **kw) == status
    assert lib.lr_last_error()


def test_select_workspace_counts_queries_and_blocks(lib):
    small, big = _shape(T=1000), _shape(T=64000)
    assert lib.lr_select_workspace_bytes(ctypes.byref(small), 8) < lib.lr_select_workspace_bytes(ctypes.byref(big), 8)
    assert lib.lr_select_workspace_bytes(ctypes.byref(small), 8) >= 256 + 8 * 128 * 4 + 2 * 16 * 4


def test_decode_path_override_changes_the_plan(lib, monkeypatch):
    """bf16 / head_dim 128 caches plan the CTA-pair kernel; LOWRAM_DECODE_PATH=general forces
    the CUDA-core plan instead (it has its own workspace layout)."""
    shape = _shape(T=32768, n_layers=4, n_kv_heads=8, rank=1024)
    sizes = {}
    for path in ("pair", "general"):
        monkeypatch.setenv("LOWRAM_DECODE_PATH", path)
        sizes[path] = lib.lr_decode_workspace_bytes(ctypes.byref(shape), 32, 0)
    monkeypatch.delenv("LOWRAM_DECODE_PATH")
    default = lib.lr_decode_workspace_bytes(ctypes.byref(shape), 32, 0)
    assert default == sizes["pair"]
    assert len(set(sizes.values())) == 2 and min(sizes.values()) > 0
    f32 = _shape(T=32768, n_layers=4, n_kv_heads=8, rank=1024, dtype=lr.LR_F32)
    monkeypatch.setenv("LOWRAM_DECODE_PATH", "pair")  # not available for fp32: the general plan
    a = lib.lr_decode_workspace_bytes(ctypes.byref(f32), 32, 0)
    monkeypatch.setenv("LOWRAM_DECODE_PATH", "general")
    assert a == lib.lr_decode_workspace_bytes(ctypes.byref(f32), 32, 0)


def test_block_means_rejects_bad_arguments(lib):
    shape = _shape()
    assert lib.lr_block_means(ctypes.byref(shape), None, FAKE, None) == lr.LR_ERR_INVALID_ARG
    assert lib.lr_block_means(ctypes.byref(shape), FAKE, FAKE + 8, None) == lr.LR_ERR_INVALID_ARG
    assert lib.lr_block_means(ctypes.byref(_shape(head_dim=12)), FAKE, FAKE, None) == lr.LR_ERR_UNSUPPORTED
    assert lib.lr_block_means(ctypes.byref(_shape(T=0)), None, None, None) == lr.LR_OK  # nothing to do


def test_pack_path_override_changes_the_plan(lib, monkeypatch):
    """bf16 / head_dim 128 caches plan the tensor-core packer (rebuilt-key buffer, fp16
    weights); LOWRAM_PACK_PATH=general forces the CUDA-core plan (a residual row per token)."""
    shape = _shape(T=4096, n_layers=4, n_kv_heads=8, rank=1024)
    monkeypatch.setenv("LOWRAM_PACK_PATH", "general")
    general = lib.lr_pack_workspace_bytes(ctypes.byref(shape), 409)
    monkeypatch.delenv("LOWRAM_PACK_PATH")
    tensor = lib.lr_pack_workspace_bytes(ctypes.byref(shape), 409)
    D = 4 * 8 * 128
    assert tensor >= 4096 * D * 2 and general >= 4 * 8 * 4096 * 128 * 2 and tensor != general
    hd64 = _shape(T=4096, head_dim=64, rank=128)
    monkeypatch.setenv("LOWRAM_PACK_PATH", "pair")
    a = lib.lr_pack_workspace_bytes(ctypes.byref(hd64), 409)
    monkeypatch.setenv("LOWRAM_PACK_PATH", "general")
    assert a == lib.lr_pack_workspace_bytes(ctypes.byref(hd64), 409)


def test_quantize_and_q2_decode_reject_bad_arguments(lib):
    shape = _shape()
    q = lib.lr_quantize_residuals
    assert q(ctypes.byref(shape), -1, FAKE, FAKE, FAKE, FAKE, None) == lr.LR_ERR_INVALID_ARG
    assert q(ctypes.byref(shape), 10, None, FAKE, FAKE, FAKE, None) == lr.LR_ERR_INVALID_ARG
    assert q(ctypes.byref(shape), 10, FAKE, FAKE, None, FAKE, None) == lr.LR_ERR_INVALID_ARG
    assert q(ctypes.byref(shape), 0, None, None, None, None, None) == lr.LR_OK
    pred = _pred()
    d = lib.lr_decode_attn_q2
    args = lambda codes, lo: (ctypes.byref(shape), 0, 8, FAKE, FAKE, FAKE, ctypes.byref(pred), FAKE, codes, lo, FAKE,
                              None, 10, None, 0, 0.0, FAKE, FAKE, 1 << 40, None)
    assert d(*args(None, FAKE)) == lr.LR_ERR_INVALID_ARG
    assert d(*args(FAKE, None)) == lr.LR_ERR_INVALID_ARG


def test_fit_predictor_rejects_bad_arguments(lib):
    shape = _shape()
    ws_bytes = lib.lr_fit_workspace_bytes(ctypes.byref(shape), 1)
    assert ws_bytes > 1000 * 2 * 2 * 128 * 2                       # at least the rebuilt keys
    assert lib.lr_fit_workspace_bytes(ctypes.byref(_shape(head_dim=64)), 1) == 0   # unsupported shape
    f = lib.lr_fit_predictor

    def call(shape=shape, n_steps=3, step=0.1, b2=None, out=None, ws=FAKE, ws_bytes=ws_bytes, A=FAKE, per_seq=1):
        p = lr.lr_predictor_f32(FAKE, FAKE, FAKE, FAKE, b2, per_seq)
        return f(ctypes.byref(shape), A, FAKE, FAKE, ctypes.byref(p), n_steps, step,
                 None if out is None else ctypes.byref(out), ws, ws_bytes, None)

    assert call(n_steps=-1) == lr.LR_ERR_INVALID_ARG
    assert call(step=-0.5) == lr.LR_ERR_INVALID_ARG
    assert call(step=float("nan")) == lr.LR_ERR_INVALID_ARG
    assert call(A=None) == lr.LR_ERR_INVALID_ARG
    assert call(per_seq=2) == lr.LR_ERR_INVALID_ARG
    assert call(ws_bytes=ws_bytes - 1) == lr.LR_ERR_WORKSPACE
    assert call(shape=_shape(head_dim=64)) == lr.LR_ERR_UNSUPPORTED
    assert call(shape=_shape(dtype=lr.LR_F32)) == lr.LR_ERR_UNSUPPORTED
    assert call(out=lr.lr_predictor_out(FAKE, FAKE, FAKE, FAKE, FAKE)) == lr.LR_ERR_INVALID_ARG  # out.b2 w/o b2
