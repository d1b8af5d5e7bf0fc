"""The workspace-free decode entry point (paged_attn_decode_static).

It exists for callers that cannot allocate device memory for a workspace (a
serving process whose KV pool already holds all free GPU memory, or a caller
behind a plugin / foreign-function layer without a device allocator). It must
give the same outputs as paged_attn_decode with a caller workspace, call after
call, since every call reuses the library's one built-in scratch array.

This file is collected last so that a run stopping at its first failure has
already run every other test; it also passes on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

import workloads as W
from gpu_support import TOL, build_pool, compare, device_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module")
def pkv():
    import paged_kv_cache_440_b200 as p
    return p


def _both(pkv, wl, num_ctas):
    pool = build_pool(pkv, wl, DEV)
    tables, lens = device_inputs(wl, DEV)
    max_ctx = int(wl.context_lens.max())
    pkv.kv_append(pool, 0, wl.k_new, wl.v_new, torch.from_numpy(wl.slot_new).to(DEV))
    ref = pkv.paged_attn_decode(pool, 0, wl.q, tables, lens, max_ctx, wl.scale,
                                num_ctas=num_ctas)
    outs = []
    for _ in range(2):                           # two calls in a row share the scratch
        out = torch.full_like(wl.q, float("nan"))
        pkv.paged_attn_decode_static(pool, 0, wl.q, tables, lens, max_ctx, wl.scale, out=out,
                                     num_ctas=num_ctas)
        outs.append(out)
    torch.cuda.synchronize()
    assert pool.status() == 0
    return ref, outs


@pytest.mark.parametrize("make,num_ctas", [(lambda: W.tiny(DEV), 13),
                                           (lambda: W.gqa70b(DEV), 0)])
def test_static_scratch_matches_caller_workspace(pkv, make, num_ctas):
    wl = make()
    ref, outs = _both(pkv, wl, num_ctas)
    ref_np = ref.float().cpu().numpy().astype(np.float64)
    for out in outs:
        compare(out, ref_np, tol=TOL, what="static scratch vs caller workspace")


def test_static_scratch_rejects_oversized_requests(pkv):
    wl = W.tiny(DEV)
    pool = build_pool(pkv, wl, DEV)
    tables, lens = device_inputs(wl, DEV)
    with pytest.raises(pkv.PagedKVError) as e:
        pkv.paged_attn_decode_static(pool, 0, wl.q, tables, lens, 250, wl.scale, num_ctas=65535)
    assert "built-in scratch" in str(e.value)
