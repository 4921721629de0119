"""Seeded synthetic inputs for the LowRAM compressed-cache path.

The tests, the benchmark and the oracle's checks all draw their inputs from
here. The module holds no step of the compressed-cache arithmetic (projection,
reconstruction, prediction, error ranking, attention). It draws what a real
prefill would hand to the packer and what a real decode step would hand to the
attention call:

* hidden states ``x = z·M + 0.05·eps`` with a seeded 2 % subset of outlier
  tokens that get an extra ``N(0, I)`` term, and the per-layer projections
  ``W_K, W_V, W_Q ~ N(0, 1/d_model)`` (the workload recipe of each config);
* the group keys ``K_group = x·[W_K^1 .. W_K^L]`` and values ``x·W_V^l``;
* the key basis: the top-``r`` eigenvectors of the key Gram matrix, i.e. the
  right singular vectors of a truncated SVD of ``K_group`` (the xKV basis of
  the LowRAM project page, Figure 3);
* the predictor's starting point: the pseudoinverse linear map
  ``pinv(W_K^h)·W_V^h`` plus a random two-layer branch (LowRAM explainer
  "Predicting the value cache from keys", paragraph on why a key can predict
  a value);
* for decode-only workloads whose context is too long to materialise ``x`` on
  the host, a compressed cache drawn from the same distribution: ``A`` is
  ``x·(W_K·B^T)``, sampled exactly through the Cholesky factor of the
  projected covariance, and the residual rows are drawn as ``N(0, 1)`` at a
  seeded token subset.

Random draws use numpy's PCG64 with a ``SeedSequence`` built from the
workload seed and a stream label, so every array is reproducible on any host.
Arrays come back as float32 (or int32); rounding to the storage type is done
by :func:`to_storage`.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional

import numpy as np

BLOCK = 64  # tokens per selectable key block


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: model shape, cache shape and residual budget."""

    name: str
    description: str
    d_model: int
    n_layers: int      # L_g: adjacent layers that share one key factor A
    n_kv_heads: int    # Hkv
    q_per_kv: int      # G: query heads per KV head
    head_dim: int      # hd
    rank: int          # r: key rank of the layer group
    hidden: int        # H: predictor hidden width
    batch: int         # B
    T: int             # context tokens per sequence
    dz: int            # latent dimension of the hidden-state model
    res_pct: int       # residual budget, integer percent of tokens
    sel_div: int       # 0: full reconstruction; n: keep nblk//n blocks per (b, h)
    dtype: str         # storage type: "f32" or "bf16"
    seed: int

    @property
    def n_q_heads(self) -> int:
        return self.n_kv_heads * self.q_per_kv

    @property
    def D(self) -> int:
        return self.n_layers * self.n_kv_heads * self.head_dim

    @property
    def nblk(self) -> int:
        return (self.T + BLOCK - 1) // BLOCK

    @property
    def k(self) -> int:
        return residual_count(self.T, self.res_pct)

    @property
    def n_sel(self) -> int:
        return self.nblk // self.sel_div if self.sel_div else 0

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


def residual_count(T: int, pct: int) -> int:
    """Residual rows per (sequence, layer, KV head): floor(T * pct / 100)."""
    return (T * pct) // 100


def _mistral(name, desc, batch, T, res_pct, sel_div, seed) -> Workload:
    return Workload(name=name, description=desc, d_model=4096, n_layers=4,
                    n_kv_heads=8, q_per_kv=4, head_dim=128, rank=1024, hidden=256,
                    batch=batch, T=T, dz=96, res_pct=res_pct, sel_div=sel_div,
                    dtype="bf16", seed=seed)


WORKLOADS: Dict[str, Workload] = {}


def _add(w: Workload) -> None:
    WORKLOADS[w.name] = w


_add(Workload(name="tiny_1k", description="1 layer, d_model 256, 2 KV heads x GQA 2, head_dim 64, "
              "full-rank keys (r=128), hidden 64, T=1024, 25% residuals, fp32",
              d_model=256, n_layers=1, n_kv_heads=2, q_per_kv=2, head_dim=64, rank=128,
              hidden=64, batch=1, T=1024, dz=48, res_pct=25, sel_div=0, dtype="f32",
              seed=1000))
_add(_mistral("mistral_group_32k", "Mistral-7B-shaped 4-layer group, r=1024, B=1, T=32768, "
              "full reconstruction, 10% residuals, bf16", 1, 32768, 10, 0, 1001))
_add(_mistral("mistral_group_131k_b4_sel8", "Mistral-7B-shaped 4-layer group, B=4, T=131072, "
              "1/8 of 64-token blocks selected, 10% residuals, bf16", 4, 131072, 10, 8, 1002))
_add(_mistral("llama_262k_full", "Llama-3.1-8B-shaped 4-layer group, B=1, T=262144, full "
              "reconstruction, 5% residuals, bf16", 1, 262144, 5, 0, 1003))
_add(_mistral("llama_262k_sel16", "Llama-3.1-8B-shaped 4-layer group, B=1, T=262144, 1/16 of "
              "blocks selected, 5% residuals, bf16", 1, 262144, 5, 16, 1003))
for _pct in (5, 10, 25):
    _add(_mistral(f"pack_131k_r{_pct}", f"Mistral-7B-shaped 4-layer group pack, B=1, T=131072, "
                  f"{_pct}% residuals, bf16", 1, 131072, _pct, 0, 1004))
# a smaller pack of the same shape (inputs still larger than L2), for kernel profiles
_add(_mistral("pack_32k_r10", "Mistral-7B-shaped 4-layer group pack, B=1, T=32768, 10% residuals, bf16",
              1, 32768, 10, 0, 1005))
for _b in (1, 2, 4, 8):
    for _t, _tn in ((32768, "32k"), (131072, "131k")):
        _add(_mistral(f"sweep_b{_b}_{_tn}", f"decode sweep: B={_b}, T={_t}, full reconstruction, "
                      f"10% residuals, bf16", _b, _t, 10, 0, 1004))


# ----------------------------------------------------------------------------- RNG

def _rng(seed: int, *stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, *stream])))


_STREAM_MODEL, _STREAM_SEQ, _STREAM_MLP, _STREAM_QUERY, _STREAM_BLOCKS, _STREAM_CACHE, _STREAM_TAIL = range(7)
_CHUNK = 4096  # tokens drawn per RNG call; fixed so that draws do not depend on memory limits


@dataclasses.dataclass
class ModelWeights:
    M: np.ndarray      # [dz, d_model]
    W_K: np.ndarray    # [L, d_model, Hkv*hd]
    W_V: np.ndarray    # [L, d_model, Hkv*hd]
    W_Q: np.ndarray    # [L, d_model, Hq*hd]


def model_weights(w: Workload) -> ModelWeights:
    """The frozen model's pieces that shape the cache: M and the K/V/Q projections."""
    g = _rng(w.seed, _STREAM_MODEL)
    d = w.d_model
    M = g.standard_normal((w.dz, d), dtype=np.float32) * np.float32(1.0 / np.sqrt(w.dz))
    s = np.float32(1.0 / np.sqrt(d))
    W_K = np.stack([g.standard_normal((d, w.n_kv_heads * w.head_dim), dtype=np.float32) * s
                    for _ in range(w.n_layers)])
    W_V = np.stack([g.standard_normal((d, w.n_kv_heads * w.head_dim), dtype=np.float32) * s
                    for _ in range(w.n_layers)])
    W_Q = np.stack([g.standard_normal((d, w.n_q_heads * w.head_dim), dtype=np.float32) * s
                    for _ in range(w.n_layers)])
    return ModelWeights(M=M, W_K=W_K, W_V=W_V, W_Q=W_Q)


def _outlier_tokens(g: np.random.Generator, T: int) -> np.ndarray:
    n_out = T // 50
    mask = np.zeros(T, dtype=bool)
    if n_out:
        mask[g.choice(T, size=n_out, replace=False)] = True
    return mask


def hidden_chunks(w: Workload, mw: ModelWeights, b: int, T: Optional[int] = None):
    """Yield (t0, x[t0:t0+c]) for sequence b: x = z M + 0.05 eps (+ eps' on outliers)."""
    T = w.T if T is None else T
    g = _rng(w.seed, _STREAM_SEQ, b)
    out = _outlier_tokens(g, T)
    for t0 in range(0, T, _CHUNK):
        c = min(_CHUNK, T - t0)
        z = g.standard_normal((c, w.dz), dtype=np.float32)
        eps = g.standard_normal((c, w.d_model), dtype=np.float32)
        x = z @ mw.M + np.float32(0.05) * eps
        o = out[t0:t0 + c]
        if o.any():
            x[o] += g.standard_normal((int(o.sum()), w.d_model), dtype=np.float32)
        yield t0, x


def keys_values(w: Workload, mw: ModelWeights, b: int, T: Optional[int] = None,
                want_values: bool = True):
    """K_group [T, D] and V [L, T, Hkv, hd] (float32) of sequence b."""
    T = w.T if T is None else T
    L, Hkv, hd = w.n_layers, w.n_kv_heads, w.head_dim
    WK = np.concatenate(list(mw.W_K), axis=1)            # [d, D], layer-major columns
    WV = np.concatenate(list(mw.W_V), axis=1)
    K = np.empty((T, w.D), dtype=np.float32)
    V = np.empty((L, T, Hkv, hd), dtype=np.float32) if want_values else None
    for t0, x in hidden_chunks(w, mw, b, T):
        c = x.shape[0]
        K[t0:t0 + c] = x @ WK
        if want_values:
            V[:, t0:t0 + c] = (x @ WV).reshape(c, L, Hkv, hd).transpose(1, 0, 2, 3)
    return K, V


def _top_eigvecs(G: np.ndarray, r: int) -> np.ndarray:
    """Top-r eigenvectors (columns, descending eigenvalue) of a symmetric PSD matrix."""
    import scipy.linalg
    n = G.shape[0]
    vals, vecs = scipy.linalg.eigh(G, subset_by_index=[n - r, n - 1])
    return vecs[:, ::-1].copy()


def key_basis_from_keys(K: np.ndarray, r: int) -> np.ndarray:
    """Bt [D, r]: the top-r right singular vectors of K (truncated SVD), as columns."""
    G = np.zeros((K.shape[1], K.shape[1]), dtype=np.float64)
    for t0 in range(0, K.shape[0], _CHUNK):
        c = K[t0:t0 + _CHUNK].astype(np.float64)
        G += c.T @ c
    return _top_eigvecs(G, r).astype(np.float32)


def key_basis_population(w: Workload, mw: ModelWeights) -> np.ndarray:
    """Bt [D, r] from the keys' population covariance W^T (M^T M + s I) W."""
    WK = np.concatenate(list(mw.W_K), axis=1).astype(np.float64)
    M = mw.M.astype(np.float64)
    s = 0.05 ** 2 + 1.0 / 50.0
    G = WK.T @ (M.T @ M) @ WK + s * (WK.T @ WK)
    return _top_eigvecs(G, w.rank).astype(np.float32)


@dataclasses.dataclass
class Predictor:
    """Per (sequence, layer, KV head) predictor in nn.Linear layout (out x in)."""

    W_lin: np.ndarray  # [B, L, Hkv, hd, hd]
    W1: np.ndarray     # [B, L, Hkv, H, hd]
    b1: np.ndarray     # [B, L, Hkv, H]
    W2: np.ndarray     # [B, L, Hkv, hd, H]
    b2: np.ndarray     # [B, L, Hkv, hd]


def predictor_init(w: Workload, mw: ModelWeights, batch: Optional[int] = None) -> Predictor:
    """W_lin = (pinv(W_K^h) W_V^h)^T; W1, W2 ~ N(0, 0.02) per sequence; b1 = b2 = 0."""
    B = w.batch if batch is None else batch
    L, Hkv, hd, H = w.n_layers, w.n_kv_heads, w.head_dim, w.hidden
    lin = np.empty((L, Hkv, hd, hd), dtype=np.float32)
    for l in range(L):
        for h in range(Hkv):
            wk = mw.W_K[l][:, h * hd:(h + 1) * hd].astype(np.float64)
            wv = mw.W_V[l][:, h * hd:(h + 1) * hd].astype(np.float64)
            lin[l, h] = (np.linalg.pinv(wk) @ wv).T.astype(np.float32)
    W_lin = np.broadcast_to(lin, (B, L, Hkv, hd, hd)).copy()
    W1 = np.empty((B, L, Hkv, H, hd), dtype=np.float32)
    W2 = np.empty((B, L, Hkv, hd, H), dtype=np.float32)
    sd = np.float32(np.sqrt(0.02))
    for b in range(B):
        g = _rng(w.seed, _STREAM_MLP, b)
        W1[b] = g.standard_normal((L, Hkv, H, hd), dtype=np.float32) * sd
        W2[b] = g.standard_normal((L, Hkv, hd, H), dtype=np.float32) * sd
    return Predictor(W_lin=W_lin, W1=W1, b1=np.zeros((B, L, Hkv, H), np.float32),
                     W2=W2, b2=np.zeros((B, L, Hkv, hd), np.float32))


def queries(w: Workload, mw: ModelWeights, layer: int, batch: Optional[int] = None) -> np.ndarray:
    """q [B, Hq, hd]: one fresh (non-outlier) token per sequence through W_Q of the layer."""
    B = w.batch if batch is None else batch
    q = np.empty((B, w.n_q_heads, w.head_dim), dtype=np.float32)
    for b in range(B):
        g = _rng(w.seed, _STREAM_QUERY, b, layer)
        z = g.standard_normal((1, w.dz), dtype=np.float32)
        x = z @ mw.M + np.float32(0.05) * g.standard_normal((1, w.d_model), dtype=np.float32)
        q[b] = (x @ mw.W_Q[layer]).reshape(w.n_q_heads, w.head_dim)
    return q


def tail_tokens(w: Workload, mw: ModelWeights, layer: int, n_tail: int, batch: Optional[int] = None):
    """Keys and values [B, Hkv, n_tail, hd] of n_tail tokens generated after the cache was
    packed: fresh hidden states of the workload's process through W_K, W_V of the layer."""
    B = w.batch if batch is None else batch
    K = np.empty((B, w.n_kv_heads, n_tail, w.head_dim), dtype=np.float32)
    V = np.empty_like(K)
    for b in range(B):
        g = _rng(w.seed, _STREAM_TAIL, b, layer)
        z = g.standard_normal((n_tail, w.dz), dtype=np.float32)
        x = z @ mw.M + np.float32(0.05) * g.standard_normal((n_tail, w.d_model), dtype=np.float32)
        K[b] = (x @ mw.W_K[layer]).reshape(n_tail, w.n_kv_heads, w.head_dim).transpose(1, 0, 2)
        V[b] = (x @ mw.W_V[layer]).reshape(n_tail, w.n_kv_heads, w.head_dim).transpose(1, 0, 2)
    return K, V


def block_lists(w: Workload, batch: Optional[int] = None, n_sel: Optional[int] = None) -> np.ndarray:
    """[B, Hkv, n_sel] sorted 64-token block ids: first and last 4 always, the rest drawn."""
    B = w.batch if batch is None else batch
    nblk = w.nblk
    n_sel = w.n_sel if n_sel is None else n_sel
    out = np.empty((B, w.n_kv_heads, n_sel), dtype=np.int32)
    for b in range(B):
        for h in range(w.n_kv_heads):
            g = _rng(w.seed, _STREAM_BLOCKS, b, h)
            edge = min(4, nblk // 2)
            fixed = sorted(set(range(edge)) | set(range(nblk - edge, nblk)))
            fixed = fixed[:n_sel]
            middle = np.arange(edge, nblk - edge)
            extra = g.choice(middle, size=max(0, n_sel - len(fixed)), replace=False) \
                if n_sel > len(fixed) else np.empty(0, np.int64)
            out[b, h] = np.sort(np.concatenate([np.asarray(fixed, np.int64), extra]))
    return out


@dataclasses.dataclass
class DecodeCache:
    """A compressed cache drawn directly (decode-only workloads)."""

    A: np.ndarray        # [B, T, r]
    Bt: np.ndarray       # [B, D, r]
    res_idx: np.ndarray  # [B, L, Hkv, k] int32, ascending
    res_val: np.ndarray  # [B, L, Hkv, k, hd]


def decode_cache(w: Workload, mw: ModelWeights, batch: Optional[int] = None,
                 T: Optional[int] = None, Bt: Optional[np.ndarray] = None) -> DecodeCache:
    """A = x (W_K_all Bt) drawn exactly: z (M C) + noise with covariance C^T C (C = W_K_all Bt)."""
    B = w.batch if batch is None else batch
    T = w.T if T is None else T
    if Bt is None:
        Bt = key_basis_population(w, mw)
    WK = np.concatenate(list(mw.W_K), axis=1)
    C = (WK.astype(np.float64) @ Bt.astype(np.float64))          # [d, r]
    Lc = np.linalg.cholesky(C.T @ C + 1e-12 * np.eye(C.shape[1])).T.astype(np.float32)  # row-vector form
    MC = (mw.M.astype(np.float64) @ C).astype(np.float32)        # [dz, r]
    k = residual_count(T, w.res_pct)
    A = np.empty((B, T, w.rank), dtype=np.float32)
    idx = np.empty((B, w.n_layers, w.n_kv_heads, k), dtype=np.int32)
    val = np.empty((B, w.n_layers, w.n_kv_heads, k, w.head_dim), dtype=np.float32)
    for b in range(B):
        g = _rng(w.seed, _STREAM_CACHE, b)
        out = _outlier_tokens(g, T)
        for t0 in range(0, T, _CHUNK):
            c = min(_CHUNK, T - t0)
            z = g.standard_normal((c, w.dz), dtype=np.float32)
            eta = g.standard_normal((c, w.rank), dtype=np.float32)
            a = z @ MC + np.float32(0.05) * (eta @ Lc)
            o = out[t0:t0 + c]
            if o.any():
                a[o] += g.standard_normal((int(o.sum()), w.rank), dtype=np.float32) @ Lc
            A[b, t0:t0 + c] = a
        for l in range(w.n_layers):
            for h in range(w.n_kv_heads):
                idx[b, l, h] = np.sort(g.choice(T, size=k, replace=False)).astype(np.int32)
                val[b, l, h] = g.standard_normal((k, w.head_dim), dtype=np.float32)
    return DecodeCache(A=A, Bt=np.broadcast_to(Bt, (B,) + Bt.shape).copy(), res_idx=idx, res_val=val)


def error_vectors(seed: int, n_segments: int, T: int, ties: bool = False) -> np.ndarray:
    """Seeded per-token error vectors [S, T] float32 (>= 0) for the top-k step alone.

    ``ties=True`` draws from a handful of values so that many errors are equal.
    """
    g = _rng(seed, 99)
    if ties:
        return g.integers(0, 5, size=(n_segments, T)).astype(np.float32) * np.float32(0.25)
    return (g.standard_normal((n_segments, T), dtype=np.float32) ** 2) * np.float32(3.0)


def to_storage(a: np.ndarray, dtype: str):
    """(torch tensor in the storage type, float64 numpy copy of exactly those values)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    if dtype == "bf16":
        t = t.to(torch.bfloat16)
    elif dtype != "f32":
        raise ValueError(dtype)
    return t, t.to(torch.float64).numpy()


def small_workload(base: str = "mistral_group_32k", **kw) -> Workload:
    """A reduced copy of a workload (for parity cases the oracle finishes in seconds)."""
    return WORKLOADS[base].replace(**kw)


def names() -> List[str]:
    return list(WORKLOADS)
