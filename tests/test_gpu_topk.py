"""GPU top-k residual selection and block pointers: bit-exact against the oracle
on the same seeded error vectors (random, tie-heavy, special values)."""
import numpy as np
import pytest
import torch

from long_context_decode_lr_b200 import lowram as lr
from long_context_decode_lr_b200 import synth
from oracle import lowram_oracle as orc

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from long_context_decode_lr_b200 import build
    build.build()
    lr.library()


def _gpu_topk(e: np.ndarray, k: int) -> np.ndarray:
    S, T = e.shape
    err = torch.from_numpy(np.ascontiguousarray(e, dtype=np.float32)).cuda()
    out = torch.full((S, max(k, 1)), -1, dtype=torch.int32, device="cuda")
    ws = lr.workspace(lr.lr_topk_workspace_bytes(S, T, k))
    lr.lr_topk_tokens(err, S, T, k, out, ws)
    torch.cuda.synchronize()
    return out[:, :k].cpu().numpy()


def _check(e, k):
    got = _gpu_topk(e, k)
    for s in range(e.shape[0]):
        ref = orc.topk_residual_tokens(e[s].astype(np.float64), k)
        np.testing.assert_array_equal(got[s], ref)


@pytest.mark.parametrize("T", [1, 2, 63, 64, 65, 1000, 2048, 3001, 4096, 4097])
@pytest.mark.parametrize("ties", [False, True])
def test_topk_small(T, ties):
    e = synth.error_vectors(T * 7 + ties, 3, T, ties=ties)
    for k in sorted({0, 1, T // 3, T // 2, max(T - 1, 0), T}):
        _check(e, k)


def test_topk_special_values():
    T = 300
    e = synth.error_vectors(5, 2, T)
    e[0, ::7] = 0.0
    e[0, 3::11] = -0.0
    e[1, ::5] = np.nan
    e[1, 2::9] = np.inf
    e[1, 4::13] = -1.0
    for k in (1, 50, 150, 299):
        _check(e, k)


def test_topk_all_equal_takes_lowest_indices():
    e = np.full((2, 5000), 0.5, np.float32)
    got = _gpu_topk(e, 777)
    np.testing.assert_array_equal(got[0], np.arange(777))


@pytest.mark.parametrize("T,k", [(131072, 6553), (131072, 13107), (131072, 32768), (262144, 13107)])
def test_topk_full_size(T, k):
    e = synth.error_vectors(T + k, 4, T)
    e[:, 1000:1400] = e[:, 2000:2400]  # exact ties across the selection boundary region
    _check(e, k)


@pytest.mark.parametrize("T,k", [(1, 0), (1, 1), (64, 64), (1000, 100), (4097, 4000), (131072, 13107)])
def test_block_ptr_exact(T, k):
    rng = np.random.default_rng(T + k)
    S = 3
    idx = np.stack([np.sort(rng.choice(T, k, replace=False)) for _ in range(S)]).astype(np.int32)
    nblk = (T + 63) // 64
    out = torch.empty((S, nblk + 1), dtype=torch.int32, device="cuda")
    lr.lr_residual_block_ptr(torch.from_numpy(idx).cuda() if k else None, S, k, T, out)
    got = out.cpu().numpy()
    for s in range(S):
        np.testing.assert_array_equal(got[s], orc.block_ptr(idx[s], T))
