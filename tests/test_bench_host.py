"""The bench's output check, on the CPU: the oracle leg keeps each sampled
sequence's outputs, and the JSON line reports the step's GPU outputs against
them. Here a host tensor stands in for the GPU's output."""
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import workloads as W  # noqa: E402
from oracle import attention, cache_ops  # noqa: E402


def _sample(wl):
    value, secs, n, threads, outs = bench.oracle_sample(wl, budget_s=60.0)
    assert n == wl.batch and sorted(outs) == list(range(wl.batch))
    assert value > 0 and threads >= 1
    return outs


def test_oracle_leg_outputs_are_the_decode_step():
    """The oracle leg's outputs are the step itself: each sequence's new row
    appended at position L - 1, then every query head attending over L tokens."""
    wl = W.tiny("cpu")
    outs = _sample(wl)
    kc = bench._host_f32(wl.k_fill)
    vc = bench._host_f32(wl.v_fill)
    cache_ops.append(kc, vc, bench._host_f32(wl.k_new), bench._host_f32(wl.v_new),
                     wl.slot_new, wl.block_size)
    ref = attention.paged_decode(bench._host_f32(wl.q).astype(np.float64), kc, vc,
                                 wl.block_tables, wl.context_lens, wl.scale)
    for b in range(wl.batch):
        np.testing.assert_allclose(outs[b], ref[b], rtol=1e-12, atol=1e-14)


def test_output_check_accepts_the_oracle_and_flags_an_error():
    wl = W.tiny("cpu")
    outs = _sample(wl)
    good = torch.from_numpy(np.stack([outs[b] for b in range(wl.batch)]).astype(np.float32))
    good = good.to(torch.bfloat16)        # the output dtype rounds each value once
    c = bench.output_check(good, outs)
    assert c["ok"] and c["sequences"] == 4
    assert c["max_abs"] <= 1e-2 and c["max_rel"] <= 1e-2
    bad = good.clone()
    bad[2, 5, 7] += 0.25
    c = bench.output_check(bad, outs)
    assert not c["ok"] and c["max_abs"] > 0.2


def test_output_check_covers_a_quantized_cache():
    """INT8 cache: the oracle leg quantizes the history itself, so its outputs
    are those of the dequantized codes; a zero output is far outside tolerance."""
    wl = W.make_decode_workload("q", 3, 8, 2, 64, 32, "bf16", "int8", [40, 70, 33], seed=3)
    outs = _sample(wl)
    assert all(o.shape == (8, 64) and np.isfinite(o).all() for o in outs.values())
    good = torch.from_numpy(np.stack([outs[b] for b in range(3)]).astype(np.float32))
    assert bench.output_check(good.to(torch.bfloat16), outs)["ok"]
    assert not bench.output_check(torch.zeros_like(good).to(torch.bfloat16), outs)["ok"]


def test_prefill_output_check_rows_are_the_oracle_prefill():
    """The prefill line's oracle rows are those of the chunked-prefill oracle
    (new token i of sequence b at position L_b - c_b + i), and a wrong row is
    flagged."""
    pw = W.make_prefill_workload("p", 8, 2, 64, 16, "bf16", [90, 120], [80, 41], seed=5)
    v, secs, rows, outs, threads = bench.prefill_oracle_sample(pw, budget_s=60.0)
    assert rows == len(outs) and sorted(outs) == [0, 37, 74, 80, 117]
    wl = pw.cache
    q = bench._host_f32(pw.q).astype(np.float64)
    ref = attention.paged_prefill(q, pw.cu_q, bench._host_f32(wl.k_fill),
                                  bench._host_f32(wl.v_fill), wl.block_tables, wl.context_lens,
                                  wl.scale)
    for r, o in outs.items():
        np.testing.assert_allclose(o, ref[r], rtol=1e-12, atol=1e-14)
    gpu = torch.from_numpy(ref.astype(np.float32)).to(torch.bfloat16)
    assert bench.output_check(gpu, outs)["ok"]
    gpu[74, 3, 0] += 0.5
    assert not bench.output_check(gpu, outs)["ok"]
