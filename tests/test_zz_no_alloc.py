"""lr_decode_attn_noalloc: the decode entry point for callers that cannot allocate device
memory (allocator callbacks, runtimes that own every allocation, paths where an allocation
may block or fail). It runs on a scratch area compiled into the library instead of a
caller workspace. This file runs last so that a failure here comes after every other test.

Two calls in a row (different layers, queries and modes) must match the fp64 oracle and the
regular entry point, which uses its own workspace, within the attention tolerance, and leave
a clean device error word (read through lr_get_device_error with no workspace); a shape
whose scratch need exceeds the static area is rejected on the host.
"""
import ctypes
import dataclasses

import numpy as np
import pytest
import torch

from long_context_decode_lr_b200 import lowram as lr

import helpers as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from long_context_decode_lr_b200 import build
    build.build()
    lr.library()


def _both(p, layer, blocks):
    w = p.w
    q_st, q_ref = H.queries(p, layer)
    shape = H.shape_of(w)
    pred = H.gpu_predictor(p)
    bl = None if blocks is None else torch.from_numpy(np.ascontiguousarray(blocks, dtype=np.int32)).cuda()
    n_sel = 0 if blocks is None else blocks.shape[-1]
    ref = torch.empty((w.batch, w.n_q_heads, w.head_dim), dtype=torch.bfloat16, device="cuda")
    ws = lr.workspace(lr.lr_decode_workspace_bytes(shape, w.n_q_heads, n_sel))
    lr.lr_decode_attn(shape, layer, w.n_q_heads, q_st, p.st["A"], p.st["Bt"], pred, p.st["idx"], p.st["val"],
                      p.st["ptr"], p.k, bl, n_sel, 0.0, ref, ws)
    got = torch.full_like(ref, float("nan"))
    lr.lr_decode_attn_noalloc(shape, layer, w.n_q_heads, q_st, p.st["A"], p.st["Bt"], pred, p.st["idx"],
                              p.st["val"], p.st["ptr"], p.k, bl, n_sel, 0.0, got)
    torch.cuda.synchronize()
    assert lr.lr_get_device_error(None) == 0
    # the oracle call names the attended blocks itself (None there means "the problem's list")
    want = H.oracle_decode(dataclasses.replace(p, blocks=blocks), layer, q_ref)
    return got.double().cpu().numpy(), ref.double().cpu().numpy(), want


def test_noalloc_matches_oracle_and_regular_entry_on_consecutive_calls():
    w = H.small(T=1000, batch=2)
    p = H.packed_problem(w, sel=5)
    got1, ref1, want1 = _both(p, 1, None)          # full reconstruction
    got2, ref2, want2 = _both(p, 0, p.blocks)      # selective, the next call on the same scratch
    H.assert_attention_close(got1, want1)
    H.assert_attention_close(got2, want2)
    H.assert_attention_close(got1, ref1)
    H.assert_attention_close(got2, ref2)
    assert not np.array_equal(got1, got2)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    lib = lr.library()
    shape = lr.cache_shape(512, 131072, 4, 8, 128, 1024, 256, torch.bfloat16)
    assert lr.lr_decode_workspace_bytes(shape, 32, 0) > 16 << 20
    fake = 0x10000
    pred = lr.lr_predictor(fake, fake, fake, fake, None, 1)
    st = lib.lr_decode_attn_noalloc(ctypes.byref(shape), 0, 32, fake, fake, fake, ctypes.byref(pred), fake, fake,
                                    None, 10, None, 0, 0.0, fake, None)
    assert st == lr.LR_ERR_WORKSPACE
    assert b"16 MiB" in lib.lr_last_error()
