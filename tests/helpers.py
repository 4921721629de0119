"""Problem builders and comparison helpers shared by the GPU parity tests.

Inputs come from the seeded generator (long_context_decode_lr_b200.synth), are
rounded once to the storage type, and the same values go to the oracle (as fp64)
and to the CUDA library (as device tensors). Expected values come only from the
oracle.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch

from long_context_decode_lr_b200 import lowram as lr
from long_context_decode_lr_b200 import synth
from oracle import lowram_oracle as orc

TORCH_DT = {"bf16": torch.bfloat16, "f32": torch.float32}

# Attention-output tolerance against the fp64 oracle (bf16 storage, fp32 accumulation):
# relative L2 <= 1e-2 and max-abs <= 2e-2 * max(1, max|ref|). The absolute bound is stated
# for outputs of unit scale. Every floating result carries a relative error, and a bf16
# output alone is rounded to 8 significant bits (at |o| >= 8 half a bf16 step already
# exceeds 2e-2), so beyond |o| = 1 the max-abs bound grows with the output's magnitude.
REL_L2 = 1e-2
MAX_ABS = 2e-2


def small(base="mistral_group_32k", **kw) -> synth.Workload:
    """A reduced Mistral-shaped group: d_model 512, 2 layers, 2 KV heads, hd 128, r 128."""
    d = dict(d_model=512, n_layers=2, n_kv_heads=2, rank=128, T=1000, dz=48)
    d.update(kw)
    return synth.small_workload(base, **d)


@dataclasses.dataclass
class Problem:
    w: synth.Workload
    st: dict           # name -> storage tensor on the GPU
    ref: dict          # name -> float64 numpy values of the same tensors
    k: int
    blocks: Optional[np.ndarray]
    has_b2: bool


def _store(arr, dtype, device="cuda"):
    t, v = synth.to_storage(arr, dtype)
    return t.to(device), v


def predictor_arrays(w, mw, with_b2=False, batch=None):
    p = synth.predictor_init(w, mw, batch=batch)
    if with_b2:
        g = np.random.default_rng(w.seed + 77)
        p.b1 = g.standard_normal(p.b1.shape).astype(np.float32) * 0.3
        p.b2 = g.standard_normal(p.b2.shape).astype(np.float32) * 0.3
    return p


def packed_problem(w: synth.Workload, k: Optional[int] = None, with_b2=False, sel=None,
                   dup_rows: int = 0, oracle: bool = True) -> Problem:
    """Inputs of a decode step whose cache is packed by the oracle from generated K, V."""
    mw = synth.model_weights(w)
    pred = predictor_arrays(w, mw, with_b2)
    k = w.k if k is None else k
    st, ref = {}, {}
    for name in ("W_lin", "W1", "b1", "W2", "b2"):
        st[name], ref[name] = _store(getattr(pred, name), w.dtype)
    K_all, V_all, Bt_all = [], [], []
    for b in range(w.batch):
        K, V = synth.keys_values(w, mw, b)
        if dup_rows:
            # copy rows so that some tokens have bit-identical keys and values
            src = np.arange(dup_rows) * 3 + 5
            K[src + 1] = K[src]
            V[:, src + 1] = V[:, src]
        Bt = synth.key_basis_from_keys(K, w.rank)
        K_all.append(K), V_all.append(V), Bt_all.append(Bt)
    st["K"], ref["K"] = _store(np.stack(K_all), w.dtype)
    st["V"], ref["V"] = _store(np.stack(V_all), w.dtype)
    st["Bt"], ref["Bt"] = _store(np.stack(Bt_all), w.dtype)
    if not oracle:
        return Problem(w=w, st=st, ref=ref, k=k, blocks=_blocks(w, sel), has_b2=with_b2)
    A, idx, val, ptr, err = [], [], [], [], []
    for b in range(w.batch):
        p = orc.pack_sequence(ref["K"][b], ref["V"][b], ref["Bt"][b], ref["W_lin"][b], ref["W1"][b],
                              ref["b1"][b], ref["W2"][b], ref["b2"][b] if with_b2 else None, k, w.dtype,
                              w.n_kv_heads, w.head_dim)
        A.append(p["A"]), idx.append(p["idx"]), val.append(p["val"]), ptr.append(p["ptr"]), err.append(p["err"])
    ref["A"], ref["idx"], ref["val"] = np.stack(A), np.stack(idx), np.stack(val)
    ref["ptr"], ref["err"] = np.stack(ptr), np.stack(err)
    st["A"] = torch.from_numpy(ref["A"]).to(TORCH_DT[w.dtype]).cuda()
    st["val"] = torch.from_numpy(ref["val"]).to(TORCH_DT[w.dtype]).cuda()
    st["idx"] = torch.from_numpy(ref["idx"].astype(np.int32)).cuda()
    st["ptr"] = torch.from_numpy(ref["ptr"].astype(np.int32)).cuda()
    blocks = _blocks(w, sel)
    return Problem(w=w, st=st, ref=ref, k=k, blocks=blocks, has_b2=with_b2)


def direct_problem(w: synth.Workload, sel=None) -> Problem:
    """Inputs of a decode step whose cache is drawn directly (long contexts)."""
    mw = synth.model_weights(w)
    pred = predictor_arrays(w, mw)
    st, ref = {}, {}
    for name in ("W_lin", "W1", "b1", "W2", "b2"):
        st[name], ref[name] = _store(getattr(pred, name), w.dtype)
    c = synth.decode_cache(w, mw)
    st["A"], ref["A"] = _store(c.A, w.dtype)
    st["Bt"], ref["Bt"] = _store(c.Bt, w.dtype)
    st["val"], ref["val"] = _store(c.res_val, w.dtype)
    ref["idx"] = c.res_idx.astype(np.int64)
    st["idx"] = torch.from_numpy(c.res_idx).cuda()
    n_seg = w.batch * w.n_layers * w.n_kv_heads
    st["ptr"] = torch.empty((w.batch, w.n_layers, w.n_kv_heads, w.nblk + 1), dtype=torch.int32, device="cuda")
    lr.lr_residual_block_ptr(st["idx"], n_seg, w.k, w.T, st["ptr"])
    return Problem(w=w, st=st, ref=ref, k=w.k, blocks=_blocks(w, sel), has_b2=False)


def _blocks(w, sel):
    if sel is None:
        return None
    if sel == "all":
        return np.broadcast_to(np.arange(w.nblk, dtype=np.int32), (w.batch, w.n_kv_heads, w.nblk)).copy()
    return synth.block_lists(w, n_sel=sel)


def queries(p: Problem, layer: int):
    mw = synth.model_weights(p.w)
    q = synth.queries(p.w, mw, layer)
    return _store(q, p.w.dtype)


def shape_of(w: synth.Workload, T=None, batch=None):
    return lr.cache_shape(w.batch if batch is None else batch, w.T if T is None else T, w.n_layers,
                          w.n_kv_heads, w.head_dim, w.rank, w.hidden, TORCH_DT[w.dtype])


def gpu_predictor(p: Problem) -> lr.Predictor:
    s = p.st
    return lr.Predictor(s["W_lin"], s["W1"], s["b1"], s["W2"], s["b2"] if p.has_b2 else None, True)


def gpu_decode(p: Problem, layer: int, q_st, use_ptr=True, scale=0.0, blocks=None, n_sel=None, tail=None):
    w = p.w
    shape = shape_of(w)
    blocks = p.blocks if blocks is None else blocks
    bl = None
    if blocks is not None:
        flat = np.ascontiguousarray(blocks, dtype=np.int32).reshape(-1)
        # an empty selection still passes a (non-null) list with n_sel = 0
        bl = torch.from_numpy(flat if flat.size else np.zeros(4, np.int32)).cuda()
    n_sel = 0 if blocks is None else (blocks.shape[-1] if n_sel is None else n_sel)
    ws = lr.workspace(lr.lr_decode_workspace_bytes(shape, w.n_q_heads, n_sel))
    o = torch.empty((w.batch, w.n_q_heads, w.head_dim), dtype=TORCH_DT[w.dtype], device="cuda")
    pred = gpu_predictor(p)
    if tail is None:
        lr.lr_decode_attn(shape, layer, w.n_q_heads, q_st, p.st["A"], p.st["Bt"], pred,
                          p.st["idx"] if p.k else None, p.st["val"] if p.k else None,
                          p.st["ptr"] if (use_ptr and p.k) else None, p.k, bl, n_sel, scale, o, ws)
    else:  # tail = (K, V) device tensors [B, Hkv, n_tail, hd] in the cache dtype
        lr.lr_decode_attn_tail(shape, layer, w.n_q_heads, q_st, p.st["A"], p.st["Bt"], pred,
                               p.st["idx"] if p.k else None, p.st["val"] if p.k else None,
                               p.st["ptr"] if (use_ptr and p.k) else None, p.k, bl, n_sel,
                               tail[0], tail[1], tail[0].shape[2], scale, o, ws)
    code = lr.lr_get_device_error(ws)
    return o.to(torch.float64).cpu().numpy(), code


def oracle_decode(p: Problem, layer: int, q_ref, scale=0.0, blocks=None, heads=None, tail=None):
    w = p.w
    blocks = p.blocks if blocks is None else blocks
    sc = orc.default_scale(w.head_dim, scale)
    out = np.zeros((w.batch, w.n_q_heads, w.head_dim))
    for b in range(w.batch):
        r = p.ref
        out[b] = orc.decode_sequence(q_ref[b], r["A"][b], r["Bt"][b], r["W_lin"][b], r["W1"][b], r["b1"][b],
                                     r["W2"][b], r["b2"][b] if p.has_b2 else None, layer, r["idx"][b],
                                     r["val"][b], None if blocks is None else blocks[b], sc,
                                     w.n_kv_heads, w.head_dim,
                                     None if tail is None else tail[0][b], None if tail is None else tail[1][b])
    return out


def assert_attention_close(got, ref, rel_l2=REL_L2, max_abs=MAX_ABS):
    diff = got - ref
    nref = np.linalg.norm(ref)
    rel = np.linalg.norm(diff) / max(nref, 1e-30)
    mab = np.abs(diff).max() if diff.size else 0.0
    bound = max_abs * max(1.0, float(np.abs(ref).max()) if ref.size else 1.0)
    assert np.all(np.isfinite(got)), "non-finite output"
    print(f"[attention parity] rel_l2={rel:.3e} max_abs={mab:.3e} (bound {bound:.3e})")
    assert rel <= rel_l2 and mab <= bound, f"rel_l2={rel:.3e} max_abs={mab:.3e} bound={bound:.3e}"
    return rel, mab


def rel_l2(got, ref):
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30))
