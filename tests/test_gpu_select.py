"""GPU parity of lr_block_means and lr_select_blocks against the oracle.

The block means are compared with the oracle's block_means (fp32 sums of storage values).
The block scores are fp32 on the GPU and fp64 in the oracle, so the selection follows the
rule for integer results decided in floating point: the GPU's list must be exactly the
top-n_sel of the GPU's own scores (ties to the lower block id, ascending; checked with the
oracle's selection function applied to those scores), the scores must match the oracle's,
and the list may differ from the oracle's top-n_sel only in blocks whose oracle score lies
within a small band of the n_sel-th largest score. A planted block (its keys aligned with a
query) must be selected and drives a selective decode step that matches the oracle decode
over the same list; selecting every block returns them all.
"""
import dataclasses

import numpy as np
import pytest
import torch

from long_context_decode_lr_b200 import lowram as lr
from long_context_decode_lr_b200 import synth
from oracle import lowram_oracle as orc

import helpers as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from long_context_decode_lr_b200 import build
    build.build()
    lr.library()


def _gpu_means(p):
    w = p.w
    abar = torch.empty((w.batch, w.nblk, w.rank), dtype=torch.float32, device="cuda")
    lr.lr_block_means(H.shape_of(w), p.st["A"], abar)
    return abar


def _gpu_select(p, layer, q_st, n_sel, abar=None):
    w = p.w
    shape = H.shape_of(w)
    abar = _gpu_means(p) if abar is None else abar
    ws = lr.workspace(lr.lr_select_workspace_bytes(shape, w.n_q_heads))
    out = torch.full((w.batch, w.n_kv_heads, max(n_sel, 1)), -7, dtype=torch.int32, device="cuda")
    scores = torch.empty((w.batch, w.n_kv_heads, w.nblk), dtype=torch.float32, device="cuda")
    lr.lr_select_blocks(shape, layer, w.n_q_heads, q_st, abar, p.st["Bt"], n_sel, 0.0, out, ws, scores_out=scores)
    torch.cuda.synchronize()
    return out.cpu().numpy()[..., :n_sel], scores.cpu().numpy().astype(np.float64)


def _oracle_scores(p, layer, q_ref):
    w = p.w
    sc = orc.default_scale(w.head_dim, 0.0)
    return np.stack([orc.block_scores(q_ref[b], p.ref["A"][b], p.ref["Bt"][b], layer, w.n_kv_heads, w.head_dim, sc)
                     for b in range(w.batch)])


def _check(got, gpu_scores, scores, n_sel):
    B, Hkv, nblk = scores.shape
    scale = np.abs(scores).max()
    np.testing.assert_allclose(gpu_scores, scores, rtol=0, atol=1e-4 * scale + 1e-6)
    band = 1e-4 * scale + 1e-6
    for b in range(B):
        # exact: the list is the top-n_sel of the GPU's own scores, ties to the lower id
        np.testing.assert_array_equal(got[b], orc.select_blocks(gpu_scores[b], n_sel))
        want = orc.select_blocks(scores[b], n_sel)
        for h in range(Hkv):
            g = got[b, h]
            assert np.all(np.diff(g) > 0) and g.min(initial=0) >= 0 and g.max(initial=0) < nblk
            diff = set(g.tolist()) ^ set(want[h].tolist())
            if diff:
                thr = np.sort(scores[b, h])[::-1][n_sel - 1]
                assert all(abs(scores[b, h, j] - thr) <= band for j in diff), (b, h, diff)


@pytest.mark.parametrize("w", [dict(T=1000), dict(T=700, batch=2), dict(T=65, rank=64, head_dim=64, hidden=128),
                               synth.WORKLOADS["tiny_1k"]])
def test_block_means(w):
    wl = w if isinstance(w, synth.Workload) else H.small(**w)
    p = H.packed_problem(wl)
    got = _gpu_means(p).double().cpu().numpy()
    want = np.stack([orc.block_means(p.ref["A"][b]) for b in range(wl.batch)])
    np.testing.assert_allclose(got, want, rtol=1e-5, atol=1e-6 * np.abs(want).max())


@pytest.mark.parametrize("case", [
    dict(w=dict(T=1000), n_sel=5),
    dict(w=dict(T=1000), n_sel=1),
    dict(w=dict(T=1000), n_sel=16),
    dict(w=dict(T=700, batch=2), n_sel=3),
    dict(w=dict(q_per_kv=8, T=900), n_sel=6),
    dict(w=dict(q_per_kv=3, n_kv_heads=12, T=900, d_model=1536), n_sel=4),   # 36 query heads: two passes
])
def test_select_small(case):
    p = H.packed_problem(H.small(**case["w"]))
    q_st, q_ref = H.queries(p, 1)
    got, gsc = _gpu_select(p, 1, q_st, case["n_sel"])
    _check(got, gsc, _oracle_scores(p, 1, q_ref), case["n_sel"])
    if case["n_sel"] == p.w.nblk:
        assert np.all(got == np.arange(p.w.nblk))


def test_scores_only_and_no_selection():
    p = H.packed_problem(H.small(T=1000))
    q_st, q_ref = H.queries(p, 0)
    got, gsc = _gpu_select(p, 0, q_st, 0)
    assert got.size == 0
    np.testing.assert_allclose(gsc, _oracle_scores(p, 0, q_ref), atol=1e-4 * np.abs(gsc).max())


def _planted(p, layer, h, j, q_ref):
    w = p.w
    Bh = orc.key_slice(p.ref["Bt"][0], layer, h, w.n_kv_heads, w.head_dim)
    A = p.ref["A"][0].copy()
    A[j * 64:(j + 1) * 64] += 40.0 * (np.linalg.pinv(Bh) @ q_ref[0, h * w.q_per_kv])
    A_dev, A_ref = synth.to_storage(A[None], w.dtype)
    st, ref = dict(p.st), dict(p.ref)
    st["A"], ref["A"] = A_dev.cuda(), A_ref
    return dataclasses.replace(p, st=st, ref=ref)


def test_planted_block_is_selected_and_drives_decode():
    """A block whose keys point along a query head wins the selection for that head, and
    the selective decode over the GPU's list matches the oracle decode over the same list.
    The planted keys make the output large (|o| of order 1e3): the attention tolerance's
    max-abs bound scales with max(1, |o|) there (bf16 output resolution)."""
    p0 = H.packed_problem(H.small(T=1000))
    layer, h, j = 0, 1, 9
    q_st, q_ref = H.queries(p0, layer)
    p = _planted(p0, layer, h, j, q_ref)
    got, gsc = _gpu_select(p, layer, q_st, 1)
    assert got[0, h, 0] == j
    blocks, gsc = _gpu_select(p, layer, q_st, 4)
    _check(blocks, gsc, _oracle_scores(p, layer, q_ref), 4)
    out, code = H.gpu_decode(p, layer, q_st, blocks=blocks.astype(np.int32))
    assert code == 0
    ref = H.oracle_decode(p, layer, q_ref, blocks=blocks)
    assert np.abs(ref).max() > 100.0
    H.assert_attention_close(out, ref)


def test_selected_blocks_drive_decode():
    """The selected list is the block_list of a selective decode step, which matches the
    oracle decode over the same list."""
    p = H.packed_problem(H.small(T=1000))
    q_st, q_ref = H.queries(p, 0)
    blocks, gsc = _gpu_select(p, 0, q_st, 4)
    _check(blocks, gsc, _oracle_scores(p, 0, q_ref), 4)
    out, code = H.gpu_decode(p, 0, q_st, blocks=blocks.astype(np.int32))
    assert code == 0
    H.assert_attention_close(out, H.oracle_decode(p, 0, q_ref, blocks=blocks))


def test_select_fp32():
    p = H.packed_problem(synth.WORKLOADS["tiny_1k"])
    q_st, q_ref = H.queries(p, 0)
    got, gsc = _gpu_select(p, 0, q_st, 4)
    _check(got, gsc, _oracle_scores(p, 0, q_ref), 4)


@pytest.mark.slow
@pytest.mark.parametrize("name,div", [("mistral_group_32k", 8), ("llama_262k_sel16", 16)])
def test_select_full_size(name, div):
    w = synth.WORKLOADS[name]
    p = H.direct_problem(w)
    layer = 2
    q_st, q_ref = H.queries(p, layer)
    got, gsc = _gpu_select(p, layer, q_st, w.nblk // div)
    _check(got, gsc, _oracle_scores(p, layer, q_ref), w.nblk // div)
