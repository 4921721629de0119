"""GPU parity of lr_select_blocks against the oracle's block scores and selection.

The scores are fp32 on the GPU and fp64 in the oracle, so the check follows the rule for
decisions taken in floating point: the GPU's list must be sorted, distinct and in range,
and it may differ from the oracle's top-n_sel only in blocks whose oracle score lies
within a small band of the n_sel-th largest score. A planted block (its keys aligned with
a query) must be selected; selecting every block returns them all; a selected list drives
a decode step that matches the oracle decode over the same list.
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


def _gpu_select(p, layer, q_st, n_sel):
    w = p.w
    shape = H.shape_of(w)
    ws = lr.workspace(lr.lr_select_workspace_bytes(shape, w.n_q_heads))
    out = torch.full((w.batch, w.n_kv_heads, max(n_sel, 1)), -7, dtype=torch.int32, device="cuda")
    lr.lr_select_blocks(shape, layer, w.n_q_heads, q_st, p.st["A"], p.st["Bt"], n_sel, 0.0, out, ws)
    torch.cuda.synchronize()
    return out.cpu().numpy()[..., :n_sel]


def _oracle_scores(p, layer, q_ref):
    w = p.w
    sc = orc.default_scale(w.head_dim, 0.0)
    return np.stack([orc.block_scores(q_ref[b], p.ref["A"][b], p.ref["Bt"][b], layer, w.n_kv_heads, w.head_dim, sc)
                     for b in range(w.batch)])


def _check(got, scores, n_sel):
    B, Hkv, nblk = scores.shape
    band = 1e-4 * np.abs(scores).max() + 1e-6
    for b in range(B):
        want = orc.select_blocks(scores[b], n_sel)
        for h in range(Hkv):
            g = got[b, h]
            assert np.all(np.diff(g) > 0) and g.min(initial=0) >= 0 and g.max(initial=0) < nblk
            diff = set(g.tolist()) ^ set(want[h].tolist())
            if diff:
                thr = np.sort(scores[b, h])[::-1][n_sel - 1]
                assert all(abs(scores[b, h, j] - thr) <= band for j in diff), (b, h, diff)


@pytest.mark.parametrize("case", [
    dict(w=dict(T=1000), n_sel=5),
    dict(w=dict(T=1000), n_sel=1),
    dict(w=dict(T=1000), n_sel=16),
    dict(w=dict(T=700, batch=2), n_sel=3),
    dict(w=dict(q_per_kv=8, T=900), n_sel=6),
])
def test_select_small(case):
    p = H.packed_problem(H.small(**case["w"]))
    q_st, q_ref = H.queries(p, 1)
    got = _gpu_select(p, 1, q_st, case["n_sel"])
    _check(got, _oracle_scores(p, 1, q_ref), case["n_sel"])
    if case["n_sel"] == p.w.nblk:
        assert np.all(got == np.arange(p.w.nblk))


def test_planted_block_is_selected():
    p = H.packed_problem(H.small(T=1000))
    w, layer, h, j = p.w, 0, 1, 9
    q_st, q_ref = H.queries(p, layer)
    Bh = orc.key_slice(p.ref["Bt"][0], layer, h, w.n_kv_heads, w.head_dim)
    A = p.ref["A"][0].copy()
    A[j * 64:(j + 1) * 64] += 40.0 * (np.linalg.pinv(Bh) @ q_ref[0, h * w.q_per_kv])
    A_dev, A_ref = synth.to_storage(A[None], w.dtype)
    st, ref = dict(p.st), dict(p.ref)
    st["A"], ref["A"] = A_dev.cuda(), A_ref
    p2 = dataclasses.replace(p, st=st, ref=ref)
    got = _gpu_select(p2, layer, q_st, 1)
    assert got[0, h, 0] == j
    _check(_gpu_select(p2, layer, q_st, 4), _oracle_scores(p2, layer, q_ref), 4)


def test_selected_blocks_drive_decode():
    """The selected list is the block_list of a selective decode step, which matches the
    oracle decode over the same list."""
    p = H.packed_problem(H.small(T=1000))
    q_st, q_ref = H.queries(p, 0)
    blocks = _gpu_select(p, 0, q_st, 4).astype(np.int32)
    _check(blocks, _oracle_scores(p, 0, q_ref), 4)
    out, code = H.gpu_decode(p, 0, q_st, blocks=blocks)
    assert code == 0
    H.assert_attention_close(out, H.oracle_decode(p, 0, q_ref, blocks=blocks))


def test_select_fp32():
    p = H.packed_problem(synth.WORKLOADS["tiny_1k"])
    q_st, q_ref = H.queries(p, 0)
    got = _gpu_select(p, 0, q_st, 4)
    _check(got, _oracle_scores(p, 0, q_ref), 4)


def test_select_32k_one_eighth():
    w = synth.WORKLOADS["mistral_group_32k"]
    p = H.direct_problem(w)
    q_st, q_ref = H.queries(p, 2)
    got = _gpu_select(p, 2, q_st, w.nblk // 8)
    _check(got, _oracle_scores(p, 2, q_ref), w.nblk // 8)
