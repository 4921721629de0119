"""Oracle: the plain, slow fp64 reference of LowRAM's compressed-cache path.

TEST INFRASTRUCTURE. Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this module. The product path (the
CUDA library and its Python binding) never calls it, and this module imports
nothing from the product. The two share only the seeded input generator.

Every function is the plain definition of one step, written in fp64 numpy with
library primitives (matmul, erf, a stable sort) and no blocking, fusion or
reordering. Inputs are taken as the exact values of the storage type (bf16 or
fp32 values held in float64). Sources, by page and section:

* "LowRAM" project page, Figure 3 ("Store the pattern, keep the exceptions"):
  the keys of a group of adjacent layers share one per-token factor A and each
  layer keeps its own smaller factor, K ~= A.B.
* "LowRAM KV cache compression -- Predicting the value cache from keys"
  (explainer), paragraph 2: values are rebuilt as the predictor's output plus
  an exact residual where one is stored, then used by ordinary attention;
  paragraph 3: the predictor starts from the pseudoinverse linear map and adds a
  small nonlinear branch; paragraph 4: residuals go to the tokens ranked worst
  by reconstruction error, one predictor per head; the "Where the memory
  actually goes" paragraph: the per-head storage budget.
* arXiv 2611.07025 abstract page: only a selected subset of the cached pairs
  is rebuilt at each decoding step (selective reconstruction); the predictor is
  fitted at test time.
* explainer, paragraph on prefill cost: the predictor is fitted to each context
  with gradient steps (150 steps, a full fit of 300, 2 from a meta-learned start).
* explainer, comparison table: LowRAM combined with quantisation keeps its
  residuals at 2 bits per number.

Readings where the pages are silent (each also listed in the design notes):
the predictor sees the reconstructed key; a residual is the difference
``v - v_hat``; the error is the squared L2 norm over the head's entries; ties
in the error ranking go to the lower token index; GELU is the exact erf form;
the softmax scale is ``1/sqrt(head_dim)``; an empty attention set gives a zero
output; the stored factor A and residual rows are rounded to the storage type
with round-to-nearest-even.

Parity pins: every function here is checked by ``tests/test_oracle_pins.py``
against facts the pages or mathematics fix (Slim-Attention exactness, 100 %
residual budget, full-rank keys, brute-force top-k, tabulated normal CDF
values, a hand-computed predictor, the worked memory example, column sums and
the rank-space identity for block means, hand-computed 2-bit codes and the
nearest-level property, finite-difference gradients and the least-squares limit
of the fitting steps).
"""
from __future__ import annotations

import math
from typing import Dict, Optional, Sequence

import numpy as np
from scipy.special import erf

BLOCK = 64


# --------------------------------------------------------------------------- storage rounding

def round_bf16(x) -> np.ndarray:
    """Round fp64 values to the nearest bfloat16 (ties to even), returned as fp64.

    bfloat16 keeps 8 significant bits and the fp32 exponent range: a normal
    value in [2^e, 2^(e+1)) is rounded to a multiple of 2^(e-7); below 2^-126
    the spacing stays 2^-133. Overflow past the largest finite value gives inf.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.array(x, dtype=np.float64, copy=True)
    fin = np.isfinite(x) & (x != 0)
    xf = x[fin]
    _, e = np.frexp(np.abs(xf))          # |x| = m * 2^e, m in [0.5, 1): |x| in [2^(e-1), 2^e)
    q = np.ldexp(1.0, np.maximum(e - 1 - 7, -133))   # spacing of bf16 values in that binade
    r = np.round(xf / q) * q             # np.round: half to even; xf/q is exact (power of two)
    big = np.abs(r) >= 2.0 ** 128
    r[big] = np.copysign(np.inf, r[big])
    out[fin] = r
    return out


def round_storage(x, dtype: str) -> np.ndarray:
    """Round to the storage type named by dtype ('f64' keeps values, 'f32', 'bf16')."""
    x = np.asarray(x, dtype=np.float64)
    if dtype == "f64":
        return x.copy()
    if dtype == "f32":
        return x.astype(np.float32).astype(np.float64)
    if dtype == "bf16":
        return round_bf16(x)
    raise ValueError(dtype)


# --------------------------------------------------------------------------- method steps

def gelu(x) -> np.ndarray:
    """GELU, exact form: x * Phi(x) = 0.5 x (1 + erf(x / sqrt 2))."""
    x = np.asarray(x, dtype=np.float64)
    return 0.5 * x * (1.0 + erf(x / math.sqrt(2.0)))


def project_keys(K_group: np.ndarray, Bt: np.ndarray) -> np.ndarray:
    """Shared factor A = K_group . B^T for one sequence (project page, Figure 3).

    K_group [T, D] holds the concatenated keys of the layer group; Bt [D, r]
    holds the basis B^T whose columns are orthonormal (a truncated SVD's right
    singular vectors), so A is the least-squares coefficient matrix of K on B.
    """
    return np.asarray(K_group, np.float64) @ np.asarray(Bt, np.float64)


def key_slice(Bt: np.ndarray, layer: int, head: int, n_kv_heads: int, head_dim: int) -> np.ndarray:
    """B_l^h as rows of Bt: [hd, r], the basis rows belonging to (layer, KV head)."""
    c0 = (layer * n_kv_heads + head) * head_dim
    return np.asarray(Bt, np.float64)[c0:c0 + head_dim, :]


def reconstruct_keys(A: np.ndarray, Bt_lh: np.ndarray) -> np.ndarray:
    """k~_t = A[t] . B_l^h for every row of A (project page, Figure 3)."""
    return np.asarray(A, np.float64) @ np.asarray(Bt_lh, np.float64).T


def predict_values(kt, W_lin, W1, b1, W2, b2=None) -> np.ndarray:
    """v_hat = k~ W_lin^T + GELU(k~ W1^T + b1) W2^T + b2 (explainer, paragraphs 2-3).

    Weights are in nn.Linear layout (out x in): W_lin [hd, hd], W1 [H, hd],
    b1 [H], W2 [hd, H], b2 [hd] (None means zero).
    """
    kt = np.asarray(kt, np.float64)
    u = kt @ np.asarray(W1, np.float64).T + np.asarray(b1, np.float64)
    v = kt @ np.asarray(W_lin, np.float64).T + gelu(u) @ np.asarray(W2, np.float64).T
    if b2 is not None:
        v = v + np.asarray(b2, np.float64)
    return v


def token_errors(v, v_hat) -> np.ndarray:
    """e_t = sum_j (v_t[j] - v_hat_t[j])^2: squared L2 error per token (explainer, paragraph 4)."""
    d = np.asarray(v, np.float64) - np.asarray(v_hat, np.float64)
    return np.sum(d * d, axis=-1)


def topk_residual_tokens(e, k: int) -> np.ndarray:
    """The k tokens with the largest error, ties to the lower index, returned ascending.

    Orders tokens by (error descending, index ascending), keeps the first k and
    sorts those indices (explainer, paragraph 4: residuals go to the worst tokens).
    """
    e = np.asarray(e, np.float64)
    T = e.shape[0]
    if not 0 <= k <= T:
        raise ValueError("k out of range")
    order = np.lexsort((np.arange(T), -e))
    return np.sort(order[:k]).astype(np.int64)


def block_ptr(idx, T: int, block: int = BLOCK) -> np.ndarray:
    """ptr[j] = number of residual indices below block * j, for j = 0 .. ceil(T/block)."""
    idx = np.asarray(idx, np.int64)
    nblk = (T + block - 1) // block
    return np.array([int(np.count_nonzero(idx < block * j)) for j in range(nblk + 1)], dtype=np.int64)


def pack_sequence(K_group, V, Bt, W_lin, W1, b1, W2, b2, k: int, dtype: str,
                  n_kv_heads: int, head_dim: int) -> Dict[str, np.ndarray]:
    """The prefill-side packer for one sequence, step by step.

    K_group [T, D]; V [L, T, Hkv, hd]; Bt [D, r]; predictor arrays indexed
    [L, Hkv, ...]. Returns A (rounded to dtype), idx [L, Hkv, k] ascending,
    val [L, Hkv, k, hd] (rounded), ptr [L, Hkv, nblk+1] and err [L, Hkv, T].
    """
    A = round_storage(project_keys(K_group, Bt), dtype)
    L, T = V.shape[0], V.shape[1]
    nblk = (T + BLOCK - 1) // BLOCK
    idx = np.zeros((L, n_kv_heads, k), np.int64)
    val = np.zeros((L, n_kv_heads, k, head_dim), np.float64)
    ptr = np.zeros((L, n_kv_heads, nblk + 1), np.int64)
    err = np.zeros((L, n_kv_heads, T), np.float64)
    for l in range(L):
        for h in range(n_kv_heads):
            kt = reconstruct_keys(A, key_slice(Bt, l, h, n_kv_heads, head_dim))
            vh = predict_values(kt, W_lin[l, h], W1[l, h], b1[l, h], W2[l, h],
                                None if b2 is None else b2[l, h])
            v = np.asarray(V[l, :, h, :], np.float64)
            e = token_errors(v, vh)
            sel = topk_residual_tokens(e, k)
            err[l, h] = e
            idx[l, h] = sel
            val[l, h] = round_storage(v[sel] - vh[sel], dtype)
            ptr[l, h] = block_ptr(sel, T)
    return {"A": A, "idx": idx, "val": val, "ptr": ptr, "err": err}


def selected_tokens(T: int, blocks: Optional[Sequence[int]], block: int = BLOCK) -> np.ndarray:
    """Token indices attended: all of [0, T) (blocks None), else the union of the blocks' ranges."""
    if blocks is None:
        return np.arange(T, dtype=np.int64)
    parts = [np.arange(block * j, min(block * j + block, T), dtype=np.int64) for j in blocks]
    if not parts:
        return np.zeros(0, np.int64)
    return np.unique(np.concatenate(parts))


def decode_sequence(q, A, Bt, W_lin, W1, b1, W2, b2, layer: int, res_idx, res_val,
                    blocks, scale: float, n_kv_heads: int, head_dim: int,
                    tail_K=None, tail_V=None) -> np.ndarray:
    """One decode step of one layer for one sequence: o [Hq, hd].

    For KV head h: gather the attended tokens (all, or the selected blocks:
    arXiv abstract, selective reconstruction), rebuild their keys A.B_l^h,
    rebuild their values as prediction + residual where one is stored
    (explainer, paragraph 2), and run softmax attention for the query heads
    h*G .. h*G+G-1 with max-subtracted exponentials. Predictor arrays are
    indexed [L, Hkv, ...]; res_idx [L, Hkv, k]; res_val [L, Hkv, k, hd];
    blocks is None (all tokens) or a per-KV-head sequence of block ids.

    tail_K, tail_V [Hkv, n_tail, hd] (optional): tokens generated after the cache was
    packed, kept exactly (explainer, paragraph on prefill and decode costs: newly
    generated tokens are stored exactly). They join the same softmax with their own
    keys and values, whatever the block selection.
    """
    q = np.asarray(q, np.float64)
    Hq = q.shape[0]
    G = Hq // n_kv_heads
    T = A.shape[0]
    n_tail = 0 if tail_K is None else np.asarray(tail_K).shape[1]
    o = np.zeros((Hq, head_dim), np.float64)
    for h in range(n_kv_heads):
        S = selected_tokens(T, None if blocks is None else blocks[h])
        kt = np.zeros((0, head_dim), np.float64)
        v = np.zeros((0, head_dim), np.float64)
        if S.size:
            kt = reconstruct_keys(np.asarray(A, np.float64)[S], key_slice(Bt, layer, h, n_kv_heads, head_dim))
            v = predict_values(kt, W_lin[layer, h], W1[layer, h], b1[layer, h], W2[layer, h],
                               None if b2 is None else b2[layer, h])
            r_full = np.zeros((T, head_dim), np.float64)
            r_full[np.asarray(res_idx[layer, h], np.int64)] = np.asarray(res_val[layer, h], np.float64)
            v = v + r_full[S]
        if n_tail:
            kt = np.concatenate([kt, np.asarray(tail_K[h], np.float64)])
            v = np.concatenate([v, np.asarray(tail_V[h], np.float64)])
        if kt.shape[0] == 0:
            continue
        for g in range(G):
            hq = h * G + g
            s = (kt @ q[hq]) * scale
            w = np.exp(s - s.max())
            o[hq] = (w @ v) / w.sum()
    return o


def block_scores(q, A, Bt, layer: int, n_kv_heads: int, head_dim: int, scale: float,
                 block: int = BLOCK) -> np.ndarray:
    """Relevance of every 64-token block to the current query, per KV head: [Hkv, nblk].

    The pages rebuild only the chunks the current query selects (explainer, paragraph on
    prefill and decode costs; arXiv abstract) but their trained selector is not available.
    Here a block's key is the mean of its reconstructed keys (the last block clipped at
    T), and its score for KV head h is the largest scaled dot product with that mean over
    the query heads h*G .. h*G+G-1 that read head h.
    """
    q = np.asarray(q, np.float64)
    A = np.asarray(A, np.float64)
    T = A.shape[0]
    G = q.shape[0] // n_kv_heads
    nblk = (T + block - 1) // block
    out = np.empty((n_kv_heads, nblk), np.float64)
    for h in range(n_kv_heads):
        kt = reconstruct_keys(A, key_slice(Bt, layer, h, n_kv_heads, head_dim))
        for j in range(nblk):
            kbar = kt[j * block:min(T, (j + 1) * block)].mean(axis=0)
            out[h, j] = max(float(q[h * G + g] @ kbar) * scale for g in range(G))
    return out


def select_blocks(scores, n_sel: int) -> np.ndarray:
    """The n_sel blocks of highest score per KV head, ties to the lower block id, returned
    in ascending order: [Hkv, n_sel] (the block-list layout lr_decode_attn reads)."""
    scores = np.asarray(scores, np.float64)
    out = np.empty((scores.shape[0], n_sel), np.int64)
    for h in range(scores.shape[0]):
        order = np.lexsort((np.arange(scores.shape[1]), -scores[h]))
        out[h] = np.sort(order[:n_sel])
    return out


def block_means(A, block: int = BLOCK) -> np.ndarray:
    """Mean of the A rows of every 64-token block, the last block clipped at T: [nblk, r].

    The rebuilt key is linear in A, so the mean rebuilt key of block j for KV head h is
    block_means(A)[j] . B_l^h (the block key that block_scores ranks): the block means
    are query-independent and can be formed once, when the cache is packed.
    """
    A = np.asarray(A, np.float64)
    T = A.shape[0]
    nblk = (T + block - 1) // block
    out = np.zeros((nblk, A.shape[1]), np.float64)
    for j in range(nblk):
        out[j] = A[j * block:min(T, (j + 1) * block)].mean(axis=0)
    return out


def default_scale(head_dim: int, scale: float) -> float:
    """The softmax scale: the given one when positive, else 1/sqrt(head_dim)."""
    return scale if scale > 0 else 1.0 / math.sqrt(head_dim)


def dense_attention(q, K, V, scale: float) -> np.ndarray:
    """Textbook single-query attention: softmax(q K^T * scale) V, for q [hd], K, V [T, hd]."""
    s = (np.asarray(K, np.float64) @ np.asarray(q, np.float64)) * scale
    w = np.exp(s - s.max())
    return (w @ np.asarray(V, np.float64)) / w.sum()


# --------------------------------------------------------------------------- accounting

def predictor_numbers(head_dim: int, hidden: int) -> int:
    """Stored numbers of one head's predictor: W_lin, W1, W2 and the two bias vectors."""
    return head_dim * head_dim + 2 * head_dim * hidden + hidden + head_dim


def residual_budget(T: int, head_dim: int, ratio: float, hidden: int) -> float:
    """Residual rows one head can afford at a target value-cache compression ratio.

    Follows the explainer's "Where the memory actually goes" paragraph: the
    head's value cache holds T*hd numbers, the target keeps T*hd/ratio of them,
    the predictor is a fixed cost, and each residual costs hd numbers plus an
    index counted as two numbers.
    """
    return (T * head_dim / ratio - predictor_numbers(head_dim, hidden)) / (head_dim + 2)


def dense_cache_bytes_per_token(n_layers: int, n_kv_heads: int, head_dim: int, elem_bytes: int) -> int:
    """Bytes one token adds to an uncompressed K+V cache."""
    return n_layers * n_kv_heads * head_dim * 2 * elem_bytes


# --------------------------------------------------------------------------- 2-bit residual rows

def quantize_residual_rows(rows):
    """2-bit codes of residual rows (explainer, comparison table: LowRAM + quantisation
    stores its residuals with 2 bits per number). The pages name no quantiser; the reading
    taken is the plain uniform one per row: four levels lo + c * step, c in {0, 1, 2, 3},
    from the row's minimum lo to its maximum hi, step = (hi - lo) / 3, and each entry gets
    the nearest level (ties to the even code). The code of an entry is an integer decided
    in floating point, so it is taken in fp32, the precision of the kernel that packs the
    rows: hi - lo, the step, x - lo and the quotient are each one correctly rounded fp32
    operation; a row with step 0 (all entries equal) gets code 0 everywhere.

    rows [n, hd] (exact values of the storage type) -> codes [n, hd] uint8, lo [n] fp32,
    step [n] fp32.
    """
    x = np.asarray(rows, np.float64).astype(np.float32)
    n = x.shape[0]
    codes = np.zeros(x.shape, np.uint8)
    lo = np.zeros(n, np.float32)
    step = np.zeros(n, np.float32)
    for i in range(n):
        row = x[i]
        if row.size == 0:
            continue
        l, h = np.float32(row.min()), np.float32(row.max())
        st = np.float32(np.float32(h - l) / np.float32(3.0))
        lo[i], step[i] = l, st
        if st > 0:
            t = (row - l).astype(np.float32) / st
            codes[i] = np.clip(np.rint(t.astype(np.float32)), 0, 3).astype(np.uint8)
    return codes, lo, step


def dequantize_residual_rows(codes, lo, step) -> np.ndarray:
    """The residual rows a decode step adds: lo + code * step per entry, [n, hd] fp64."""
    return (np.asarray(lo, np.float64)[:, None]
            + np.asarray(codes, np.float64) * np.asarray(step, np.float64)[:, None])


def pack_2bit(codes) -> np.ndarray:
    """Byte layout of the codes: entry 4i + s of a row sits in bits 2s..2s+1 of byte i."""
    c = np.asarray(codes, np.uint8)
    n, hd = c.shape
    c4 = c.reshape(n, hd // 4, 4).astype(np.uint32)
    return (c4[..., 0] | (c4[..., 1] << 2) | (c4[..., 2] << 4) | (c4[..., 3] << 6)).astype(np.uint8)


def unpack_2bit(packed, hd: int) -> np.ndarray:
    """Inverse of pack_2bit: [n, hd / 4] bytes -> [n, hd] codes."""
    p = np.asarray(packed, np.uint8).astype(np.uint32)
    out = np.stack([(p >> (2 * s)) & 3 for s in range(4)], axis=-1)
    return out.reshape(p.shape[0], hd).astype(np.uint8)


# --------------------------------------------------------------------------- test-time fitting

def gelu_grad(x) -> np.ndarray:
    """Derivative of the erf-form GELU: Phi(x) + x phi(x)."""
    x = np.asarray(x, np.float64)
    Phi = 0.5 * (1.0 + erf(x / math.sqrt(2.0)))
    phi = np.exp(-0.5 * x * x) / math.sqrt(2.0 * math.pi)
    return Phi + x * phi


def predictor_loss(kt, v, params) -> float:
    """Mean squared value error of the predictor over the context's tokens and the head's
    entries: mean_{t, j} (v_hat_t[j] - v_t[j])^2. The explainer (paragraph 2 and the
    paragraph on prefill cost) fits the per-head network to this context with gradient
    steps; it does not name the loss, and the mean squared error is the plainest reading
    (the same per-token error that ranks the residuals, averaged)."""
    vh = predict_values(kt, params["W_lin"], params["W1"], params["b1"], params["W2"], params.get("b2"))
    d = vh - np.asarray(v, np.float64)
    return float(np.mean(d * d))


def predictor_grads(kt, v, params):
    """Gradients of predictor_loss with respect to every predictor parameter (W_lin, W1,
    b1, W2 and b2 when the predictor has one), by the chain rule through
    v_hat = k W_lin^T + GELU(k W1^T + b1) W2^T + b2."""
    kt = np.asarray(kt, np.float64)
    v = np.asarray(v, np.float64)
    W_lin, W1, b1, W2 = (np.asarray(params[n], np.float64) for n in ("W_lin", "W1", "b1", "W2"))
    b2 = params.get("b2")
    u = kt @ W1.T + b1
    g = gelu(u)
    vh = kt @ W_lin.T + g @ W2.T
    if b2 is not None:
        vh = vh + np.asarray(b2, np.float64)
    dv = 2.0 * (vh - v) / v.size          # d loss / d v_hat
    du = (dv @ W2) * gelu_grad(u)         # d loss / d u
    out = {"W_lin": dv.T @ kt, "W1": du.T @ kt, "b1": du.sum(axis=0), "W2": dv.T @ g}
    if b2 is not None:
        out["b2"] = dv.sum(axis=0)
    return out


def fit_predictor(kt, v, params, n_steps: int, lr: float):
    """Test-time fitting of one head's predictor to the context's own (reconstructed key,
    value) pairs: n_steps of full-batch gradient descent on predictor_loss from the given
    start (the pseudoinverse initialisation, or a previous fit). Explainer, paragraph on
    prefill cost: 150 gradient steps per context, a full fit of 300, two steps from a
    meta-learned start; the pages name neither the optimiser nor the step size, so the
    plainest reading is taken: theta <- theta - lr * grad, with lr given by the caller."""
    p = {n: (None if a is None else np.array(a, np.float64, copy=True)) for n, a in params.items()}
    for _ in range(n_steps):
        gr = predictor_grads(kt, v, p)
        for n, d in gr.items():
            p[n] = p[n] - lr * d
    return p
