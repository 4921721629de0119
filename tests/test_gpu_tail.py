"""GPU parity of lr_decode_attn_tail: the compressed cache plus an exact tail of newly
generated tokens in one softmax, against the fp64 oracle on the same inputs.

Cases: a tail next to full and selective reconstruction, a tail with nothing selected
(the tail alone), a one-token tail alone (the output is that token's value), an empty
context (T = 0), batch 2, a long tail, the fp32 path, the forced CUDA-core path, and the
262K-token workload (full and 1/16 selective) with a 256-token tail.
"""
import numpy as np
import pytest
import torch

from long_context_decode_lr_b200 import lowram as lr
from long_context_decode_lr_b200 import synth

import helpers as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from long_context_decode_lr_b200 import build
    build.build()
    lr.library()


def _tail(p, layer, n_tail):
    K, V = synth.tail_tokens(p.w, synth.model_weights(p.w), layer, n_tail)
    Kd, Kr = synth.to_storage(K, p.w.dtype)
    Vd, Vr = synth.to_storage(V, p.w.dtype)
    return (Kd.cuda().contiguous(), Vd.cuda().contiguous()), (Kr, Vr)


def _check(p, n_tail, layer=0, blocks=None, rel_l2=H.REL_L2, max_abs=H.MAX_ABS):
    q_st, q_ref = H.queries(p, layer)
    t_dev, t_ref = _tail(p, layer, n_tail)
    got, code = H.gpu_decode(p, layer, q_st, blocks=blocks, tail=t_dev)
    ref = H.oracle_decode(p, layer, q_ref, blocks=blocks, tail=t_ref)
    assert code == 0
    H.assert_attention_close(got, ref, rel_l2=rel_l2, max_abs=max_abs)
    return got, ref, t_ref


CASES = {
    "full_tail5": dict(w=dict(T=1000), sel=None, n_tail=5),
    "sel_tail17": dict(w=dict(T=1000), sel=4, n_tail=17),
    "batch2_tail64": dict(w=dict(T=700, batch=2), sel=None, n_tail=64),
    "gqa8_tail300": dict(w=dict(q_per_kv=8, T=400), sel=None, n_tail=300),
}


@pytest.mark.parametrize("name", list(CASES))
def test_tail_bf16(name):
    c = CASES[name]
    p = H.packed_problem(H.small(**c["w"]), sel=c["sel"])
    _check(p, c["n_tail"])


def test_tail_alone_and_single_token():
    p = H.packed_problem(H.small(T=600), sel=3)
    empty = np.zeros((p.w.batch, p.w.n_kv_heads, 0), dtype=np.int32)
    _check(p, 9, blocks=empty)
    got, _, (Kr, Vr) = _check(p, 1, blocks=empty)
    G = p.w.q_per_kv
    want = np.repeat(Vr[:, :, 0, :], G, axis=1)  # softmax over one token: its value, exactly
    np.testing.assert_array_equal(got, want)


def test_tail_with_empty_context():
    """T = 0: nothing is cached yet, the tail alone is attended."""
    from oracle import lowram_oracle as orc
    p = H.packed_problem(H.small(T=640), sel=2)
    w0 = H.small(T=0, res_pct=0)
    shape = H.shape_of(w0)
    q_st, q_ref = H.queries(p, 0)
    t_dev, (Kr, Vr) = _tail(p, 0, 12)
    o = torch.full((1, w0.n_q_heads, w0.head_dim), 7.0, dtype=torch.bfloat16, device="cuda")
    ws = lr.workspace(lr.lr_decode_workspace_bytes(shape, w0.n_q_heads, 0))
    one = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    pred = lr.Predictor(p.st["W_lin"], p.st["W1"], p.st["b1"], p.st["W2"])
    lr.lr_decode_attn_tail(shape, 0, w0.n_q_heads, q_st, one, p.st["Bt"], pred, None, None, None, 0, None, 0,
                           t_dev[0], t_dev[1], 12, 0.0, o, ws)
    assert lr.lr_get_device_error(ws) == 0
    r = p.ref
    L, Hkv, hd = w0.n_layers, w0.n_kv_heads, w0.head_dim
    ref = orc.decode_sequence(q_ref[0], np.zeros((0, w0.rank)), r["Bt"][0], r["W_lin"][0], r["W1"][0], r["b1"][0],
                              r["W2"][0], None, 0, np.zeros((L, Hkv, 0), np.int64), np.zeros((L, Hkv, 0, hd)),
                              None, orc.default_scale(hd, 0.0), Hkv, hd, Kr[0], Vr[0])
    H.assert_attention_close(o.double().cpu().numpy()[0], ref)


def test_tail_fp32_general_path():
    w = synth.WORKLOADS["tiny_1k"]
    p = H.packed_problem(w)
    _check(p, 33, rel_l2=1e-4, max_abs=1e-4)


@pytest.mark.parametrize("path", ["general"])
def test_tail_fallback_paths(path, monkeypatch):
    monkeypatch.setenv("LOWRAM_DECODE_PATH", path)
    p = H.packed_problem(H.small(T=900, batch=2), sel=5)
    _check(p, 21)


@pytest.mark.slow
@pytest.mark.parametrize("name,sel", [("llama_262k_full", None), ("llama_262k_sel16", "list")])
def test_tail_full_size(name, sel):
    w = synth.WORKLOADS[name]
    p = H.direct_problem(w, sel=w.n_sel if sel else None)
    _check(p, 256, layer=w.n_layers - 1, blocks=p.blocks)
