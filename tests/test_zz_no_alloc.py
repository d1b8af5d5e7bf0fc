"""The workspace-free decode entry point (paged_attn_decode_static).

It exists for callers that cannot allocate device memory for a workspace (a
serving process whose KV pool already holds all free GPU memory, or a caller
behind a plugin / foreign-function layer without a device allocator). It must
give exactly the outputs of paged_attn_decode with a caller workspace, call
after call, since every call reuses the library's one built-in scratch array.

This file is collected last so that a run stopping at its first failure has
already run every other test; it also passes on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

import workloads as W
from gpu_support import build_pool, device_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module")
def pkv():
    import paged_kv_cache_440_b200 as p
    return p


def _calls(pkv, wl, specs):
    """For each (q, lengths, num_ctas) in turn: the workspace-free call and, as
    its reference, paged_attn_decode with a caller workspace on the same inputs.
    The calls run back to back, so each static call starts from the scratch the
    previous one left behind."""
    pool = build_pool(pkv, wl, DEV)
    tables, _ = device_inputs(wl, DEV)
    pkv.kv_append(pool, 0, wl.k_new, wl.v_new, torch.from_numpy(wl.slot_new).to(DEV))
    max_ctx = int(wl.context_lens.max())
    pairs = []
    for q, lens, num_ctas in specs:
        out = torch.full_like(q, float("nan"))
        pkv.paged_attn_decode_static(pool, 0, q, tables, lens, max_ctx, wl.scale, out=out,
                                     num_ctas=num_ctas)
        ref = pkv.paged_attn_decode(pool, 0, q, tables, lens, max_ctx, wl.scale,
                                    num_ctas=num_ctas)
        pairs.append((out, ref))
    torch.cuda.synchronize()
    assert pool.status() == 0
    return pairs


@pytest.mark.parametrize("make,ctas", [(lambda: W.tiny(DEV), (13, 7)),
                                       (lambda: W.gqa70b(DEV), (0, 61))])
def test_static_scratch_matches_caller_workspace(pkv, make, ctas):
    """Two calls in a row with different queries, lengths and CTA counts (the
    second with shorter lengths, so its split differs from the first one's)
    give exactly the bits of the workspace entry point on the same inputs."""
    wl = make()
    _, lens = device_inputs(wl, DEV)
    g = torch.Generator(device=DEV).manual_seed(7)
    q2 = torch.randn(wl.q.shape, generator=g, device=DEV).to(wl.q.dtype)
    lens2 = torch.clamp(lens - 9, min=1)
    for out, ref in _calls(pkv, wl, [(wl.q, lens, ctas[0]), (q2, lens2, ctas[1])]):
        assert torch.equal(out, ref), "static scratch vs caller workspace"


def test_static_scratch_rejects_oversized_requests(pkv):
    wl = W.tiny(DEV)
    pool = build_pool(pkv, wl, DEV)
    tables, lens = device_inputs(wl, DEV)
    with pytest.raises(pkv.PagedKVError) as e:
        pkv.paged_attn_decode_static(pool, 0, wl.q, tables, lens, 250, wl.scale, num_ctas=65535)
    assert "built-in scratch" in str(e.value)
