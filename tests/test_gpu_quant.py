"""2-bit residual rows on the GPU.

lr_quantize_residuals decides integer codes in fp32, the same precision the oracle's
quantiser uses, so its codes, row minima and steps must equal the oracle's bit for bit on
the same stored rows (packed-cache rows, wide-range random rows, rows with exact ties and
constant rows, head_dim 64, fp32 storage). lr_decode_attn_q2 takes codes made by the
oracle's quantiser from the oracle's packed residual rows and must match the oracle decode
over the dequantised rows (lo + code * step) within the attention tolerance, on the pair
kernel and on the forced CUDA-core path, full and selective, at small and full size.
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


def _gpu_quantize(rows_dev, shape):
    n, hd = rows_dev.shape
    codes = torch.empty((n, hd // 4), dtype=torch.uint8, device="cuda")
    lo = torch.empty(n, dtype=torch.float32, device="cuda")
    step = torch.empty(n, dtype=torch.float32, device="cuda")
    lr.lr_quantize_residuals(shape, n, rows_dev, codes, lo, step)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), lo.cpu().numpy(), step.cpu().numpy()


def _check_exact(rows_ref, rows_dev, shape):
    codes, lo, step = _gpu_quantize(rows_dev, shape)
    c_ref, lo_ref, st_ref = orc.quantize_residual_rows(rows_ref)
    np.testing.assert_array_equal(codes, orc.pack_2bit(c_ref))
    np.testing.assert_array_equal(lo, lo_ref)
    np.testing.assert_array_equal(step, st_ref)


def test_quantize_packed_rows_exact():
    p = H.packed_problem(H.small(T=1000))
    rows = p.ref["val"].reshape(-1, p.w.head_dim)
    _check_exact(rows, p.st["val"].reshape(-1, p.w.head_dim).contiguous(), H.shape_of(p.w))


@pytest.mark.parametrize("dtype,hd", [("bf16", 128), ("bf16", 64), ("f32", 128), ("bf16", 256)])
def test_quantize_random_and_special_rows_exact(dtype, hd):
    g = np.random.default_rng(7)
    rows = g.standard_normal((3000, hd)) * np.exp(g.uniform(-6, 6, (3000, 1)))
    rows[0] = 2.5                                              # constant row
    rows[1, :] = 0.0
    rows[1, :8] = [0.0, 0.5, 1.5, 2.5, 3.0, 1.0, 2.0, 3.0]     # exact ties at x.5 steps
    rows[2, :] = -1.0
    rows[2, 1] = 5.0                                           # one outlier
    dev, ref = synth.to_storage(rows, dtype)
    shape = lr.cache_shape(1, 16, 1, 1, hd, 64, 128, H.TORCH_DT[dtype])
    _check_exact(ref, dev.cuda().contiguous(), shape)


def _q2_problem(p):
    """The oracle's 2-bit codes of the oracle's packed rows, as GPU inputs and as the
    dequantised rows the oracle decode adds."""
    w = p.w
    rows = p.ref["val"].reshape(-1, w.head_dim)
    c, lo, st = orc.quantize_residual_rows(rows)
    deq = orc.dequantize_residual_rows(c, lo, st).reshape(p.ref["val"].shape)
    shp = p.ref["val"].shape[:-1]
    dev = {"codes": torch.from_numpy(orc.pack_2bit(c).reshape(*shp, w.head_dim // 4)).cuda(),
           "lo": torch.from_numpy(lo.reshape(shp)).cuda(), "step": torch.from_numpy(st.reshape(shp)).cuda()}
    return dataclasses.replace(p, ref=dict(p.ref, val=deq)), dev


def _decode_q2(p, dev, layer, q_st, blocks=None, use_ptr=True):
    w = p.w
    shape = H.shape_of(w)
    bl, n_sel = None, 0
    if blocks is not None:
        bl = torch.from_numpy(np.ascontiguousarray(blocks, dtype=np.int32).reshape(-1)).cuda()
        n_sel = blocks.shape[-1]
    ws = lr.workspace(lr.lr_decode_workspace_bytes(shape, w.n_q_heads, n_sel))
    o = torch.empty((w.batch, w.n_q_heads, w.head_dim), dtype=H.TORCH_DT[w.dtype], device="cuda")
    lr.lr_decode_attn_q2(shape, layer, w.n_q_heads, q_st, p.st["A"], p.st["Bt"], H.gpu_predictor(p), p.st["idx"],
                         dev["codes"], dev["lo"], dev["step"], p.st["ptr"] if use_ptr else None, p.k, bl, n_sel,
                         0.0, o, ws)
    return o.double().cpu().numpy(), lr.lr_get_device_error(ws)


CASES = {
    "full": dict(w=dict(T=1000), sel=None),
    "sel4_noptr": dict(w=dict(T=1000), sel=4, ptr=False),
    "batch2_gqa8": dict(w=dict(T=700, batch=2, q_per_kv=8), sel=None),
    "every_token": dict(w=dict(T=300, res_pct=100), sel=None),
}


@pytest.mark.parametrize("path", ["pair", "general"])
@pytest.mark.parametrize("name", list(CASES))
def test_decode_q2_small(name, path, monkeypatch):
    monkeypatch.setenv("LOWRAM_DECODE_PATH", path)
    c = CASES[name]
    p, dev = _q2_problem(H.packed_problem(H.small(**c["w"]), sel=c["sel"]))
    layer = 1
    q_st, q_ref = H.queries(p, layer)
    got, code = _decode_q2(p, dev, layer, q_st, blocks=p.blocks, use_ptr=c.get("ptr", True))
    assert code == 0
    H.assert_attention_close(got, H.oracle_decode(p, layer, q_ref))


def test_decode_q2_fp32_general():
    p, dev = _q2_problem(H.packed_problem(synth.WORKLOADS["tiny_1k"]))
    q_st, q_ref = H.queries(p, 0)
    got, code = _decode_q2(p, dev, 0, q_st)
    assert code == 0
    H.assert_attention_close(got, H.oracle_decode(p, 0, q_ref), rel_l2=1e-4, max_abs=1e-4)


@pytest.mark.slow
@pytest.mark.parametrize("name,sel", [("llama_262k_full", None), ("mistral_group_131k_b4_sel8", "list")])
def test_decode_q2_full_size(name, sel):
    w = synth.WORKLOADS[name]
    p, dev = _q2_problem(H.direct_problem(w, sel=w.n_sel if sel else None))
    layer = w.n_layers - 1
    q_st, q_ref = H.queries(p, layer)
    got, code = _decode_q2(p, dev, layer, q_st, blocks=p.blocks)
    assert code == 0
    H.assert_attention_close(got, H.oracle_decode(p, layer, q_ref))
