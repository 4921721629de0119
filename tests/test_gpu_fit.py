"""GPU parity of lr_fit_predictor (test-time fitting) against the oracle's fit_predictor.

Inputs come from the seeded generator and the oracle's packer (A rounded to bf16); the same
fp32 starting parameters go to both sides. The fitted parameters are compared through their
updates theta_n - theta_0, per parameter tensor, relative L2 <= 2e-2. The bound comes from
the arithmetic: the GPU reads rebuilt keys, residuals, GELU outputs and GELU' products in fp16
(relative 2^-11 each), uses the tanh-form GELU (within 2.71e-4 of x Phi(x)) and accumulates in
fp32, so one step's update carries a relative error of about 1e-3, and a few steps compound
it. The fitted predictor must also lower the oracle's loss, n_steps = 0 must leave the
parameters unchanged, and the rounded copies must equal the fp32 parameters rounded.
"""
import numpy as np
import pytest
import torch

from long_context_decode_lr_b200 import lowram as lr
from long_context_decode_lr_b200 import synth
from oracle import lowram_oracle as orc

import helpers as H

pytestmark = pytest.mark.gpu

NAMES = ("W_lin", "W1", "b1", "W2", "b2")
UPDATE_TOL = 2e-2


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from long_context_decode_lr_b200 import build
    build.build()
    lr.library()


def _params(w, with_b2=True, per_sequence=True):
    mw = synth.model_weights(w)
    pred = H.predictor_arrays(w, mw, with_b2=True)
    # the fp32 starting point: the stored (bf16) values of the pinv-initialised predictor
    p = {n: synth.to_storage(getattr(pred, n), w.dtype)[1] for n in NAMES}
    if not per_sequence:
        p = {n: a[:1] for n, a in p.items()}
    if not with_b2:
        p["b2"] = None
    return p


def _gpu_fit(p, params, n_steps, step, per_sequence=True, out=False):
    w = p.w
    shape = H.shape_of(w)
    dev = [None if params[n] is None else torch.from_numpy(np.ascontiguousarray(params[n], np.float32)).cuda()
           for n in NAMES]
    outs = None
    if out:
        outs = [None if t is None else torch.empty(t.shape, dtype=torch.bfloat16, device="cuda") for t in dev]
    ws = lr.workspace(lr.lr_fit_workspace_bytes(shape, per_sequence))
    lr.lr_fit_predictor(shape, p.st["A"], p.st["Bt"], p.st["V"], dev, n_steps, step, ws, out=outs,
                        per_sequence=per_sequence)
    assert lr.lr_get_device_error(ws) == 0
    got = {n: None if t is None else t.double().cpu().numpy() for n, t in zip(NAMES, dev)}
    if out:
        return got, {n: None if t is None else t.double().cpu().numpy() for n, t in zip(NAMES, outs)}
    return got


def _oracle_fit(p, params, n_steps, step, per_sequence=True):
    w, r = p.w, p.ref
    out = {n: None if a is None else np.array(a, copy=True) for n, a in params.items()}
    for l in range(w.n_layers):
        for h in range(w.n_kv_heads):
            seqs = range(w.batch) if per_sequence else [None]
            for b in seqs:
                bs = [b] if b is not None else list(range(w.batch))
                kt = np.concatenate([orc.reconstruct_keys(r["A"][x], orc.key_slice(r["Bt"][x], l, h, w.n_kv_heads,
                                                                                   w.head_dim)) for x in bs])
                v = np.concatenate([r["V"][x][l, :, h, :] for x in bs])
                pi = 0 if b is None else b
                start = {n: None if a is None else a[pi, l, h] for n, a in params.items()}
                fitted = orc.fit_predictor(kt, v, start, n_steps, step)
                for n in NAMES:
                    if out[n] is not None:
                        out[n][pi, l, h] = fitted[n]
    return out


def _compare(got, want, start):
    for n in NAMES:
        if start[n] is None:
            continue
        d_got, d_want = got[n] - start[n], want[n] - start[n]
        rel = np.linalg.norm(d_got - d_want) / max(np.linalg.norm(d_want), 1e-30)
        print(f"[fit parity] {n}: update rel L2 {rel:.3e} (|update| {np.linalg.norm(d_want):.3e})")
        assert rel <= UPDATE_TOL, (n, rel)


def _loss(p, params, l, h, b=0):
    w, r = p.w, p.ref
    kt = orc.reconstruct_keys(r["A"][b], orc.key_slice(r["Bt"][b], l, h, w.n_kv_heads, w.head_dim))
    return orc.predictor_loss(kt, r["V"][b][l, :, h, :], {n: None if a is None else a[b, l, h] for n, a in params.items()})


CASES = {
    "ragged_h256_b2": dict(w=dict(T=1000), b2=True),
    "h128_no_b2": dict(w=dict(T=777, hidden=128), b2=False),
    "batch2": dict(w=dict(T=513, batch=2), b2=True),
}


@pytest.mark.parametrize("name", list(CASES))
def test_fit_small(name):
    c = CASES[name]
    w = H.small(**c["w"])
    p = H.packed_problem(w, k=0)
    start = _params(w, with_b2=c["b2"])
    got = _gpu_fit(p, start, 4, 0.5)
    want = _oracle_fit(p, start, 4, 0.5)
    _compare(got, want, start)
    for l in range(w.n_layers):
        for h in range(w.n_kv_heads):
            assert _loss(p, got, l, h) < _loss(p, start, l, h)


def test_fit_shared_predictor_over_two_sequences():
    w = H.small(T=600, batch=2)
    p = H.packed_problem(w, k=0)
    start = _params(w, per_sequence=False)
    got = _gpu_fit(p, start, 3, 0.5, per_sequence=False)
    want = _oracle_fit(p, start, 3, 0.5, per_sequence=False)
    _compare(got, want, start)


def test_fit_zero_steps_and_rounded_copies():
    w = H.small(T=300)
    p = H.packed_problem(w, k=0)
    start = _params(w)
    got, rounded = _gpu_fit(p, start, 0, 0.5, out=True)
    for n in NAMES:
        np.testing.assert_array_equal(got[n], start[n])
        np.testing.assert_array_equal(rounded[n], orc.round_bf16(start[n]))
    got, rounded = _gpu_fit(p, start, 2, 0.5, out=True)
    for n in NAMES:
        np.testing.assert_array_equal(rounded[n], orc.round_bf16(got[n]))


@pytest.mark.slow
def test_fit_full_size_two_steps():
    """The 131,072-token Mistral-shaped group, two steps (the pages' setting for a
    meta-learned start); per (layer, KV head) updates compared with the oracle on a sample of
    heads (every update tensor of those heads)."""
    w = synth.WORKLOADS["pack_131k_r10"]
    p = H.packed_problem(w, k=0, oracle=False)
    # A from the oracle's projection of the same keys (rounded to bf16)
    A = orc.round_storage(orc.project_keys(p.ref["K"][0], p.ref["Bt"][0]), w.dtype)
    p.ref["A"] = A[None]
    p.st["A"] = torch.from_numpy(A[None]).to(torch.bfloat16).cuda()
    start = _params(w)
    got = _gpu_fit(p, start, 2, 0.5)
    for l, h in [(0, 0), (1, 5), (3, 7)]:
        kt = orc.reconstruct_keys(A, orc.key_slice(p.ref["Bt"][0], l, h, w.n_kv_heads, w.head_dim))
        s = {n: start[n][0, l, h] for n in NAMES}
        want = orc.fit_predictor(kt, p.ref["V"][0][l, :, h, :], s, 2, 0.5)
        _compare({n: got[n][0, l, h] for n in NAMES}, want, s)
