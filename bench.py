"""Benchmark of one paged decode step on the LLaMA-70B-shaped GQA layer.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload gqa70b|mha13b|quant_a_int8|...] [--ctas G]

A step is the whole hot path for one batch: the append of each sequence's new
K/V token into the paged cache and the paged decode attention over the cache
including it, through the library's C ABI: paged_attn_decode_append (the
append folded into the persistent attention kernel) and its split-K merge
kernel; with --separate-append, kv_append + paged_attn_decode instead.

Workload (default): batch 32, 64 query / 8 KV heads, head_dim 128, bf16,
16-token blocks, context lengths uniform on [512, 4096] (seed 0), pool 1.2x
the blocks needed, shuffled placement, q/K/V ~ N(0, 1). The cache (287 MB of
K/V) exceeds L2, and L2 is also flushed before every timed step, outside the
timed events, by reading a 256 MiB buffer (which leaves L2 holding clean
lines, as the previous layer's step would).

Metric: KV HBM GB/s = algorithmic bytes per step / step time, where the
bytes are K+V of every cached token read once, q read, output written, plus
the append's reads and writes. Also reported: % of 8 TB/s, decode tokens/s
(sequences per second per layer), the partition kernel's roofline fraction
against the measured copy bandwidth, an end-to-end figure with host buffers,
and the CPU oracle on a bounded sample.

Multi-GPU (torchrun): replicas only. Each rank runs the same workload on its
own GPU with no data-path collective; the step time is the max over ranks and
the value the sum of all ranks' bytes over it.
"""
import argparse
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "paged decode attention: KV HBM GB/s (% of 8 TB/s), decode tokens/s"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")

WORKLOADS = {
    "gqa70b": ("LLaMA-70B-shaped GQA layer: 64 q / 8 kv heads, head_dim 128, bf16, block 16, "
               "batch 32, context U[512,4096], pool 1.2x, shuffled placement",
               lambda dev: W.gqa70b(dev)),
    "mha13b": ("13B-shaped MHA layer: 40/40 heads, head_dim 128, fp16, block 16, batch 32 x 2048",
               lambda dev: W.mha13b(dev)),
    "quant_a_int8": ("INT8 per-token-head KV: 64/8 heads, head_dim 128, block 32, 64 x 4096",
                     lambda dev: W.quant_long("int8", "a", dev)),
    "quant_a_e5m2": ("FP8-E5M2 per-token-head KV: 64/8 heads, head_dim 128, block 32, 64 x 4096",
                     lambda dev: W.quant_long("e5m2", "a", dev)),
    "quant_b_int8": ("INT8 per-token-head KV: 64/8 heads, head_dim 128, block 32, 8 x 32768",
                     lambda dev: W.quant_long("int8", "b", dev)),
    "quant_b_e5m2": ("FP8-E5M2 per-token-head KV: 64/8 heads, head_dim 128, block 32, 8 x 32768",
                     lambda dev: W.quant_long("e5m2", "b", dev)),
    "quant_a_int4": ("INT4 per-token-head KV (two codes per byte): 64/8 heads, head_dim 128, "
                     "block 32, 64 x 4096", lambda dev: W.quant_long("int4", "a", dev)),
    "quant_a_e5m2_cast": ("FP8-E5M2 KV cast with no scale: 64/8 heads, head_dim 128, block 32, "
                          "64 x 4096", lambda dev: W.quant_long("e5m2_cast", "a", dev)),
    "quant_a_int8_kchan": ("INT8 KV, keys with fixed per-channel scales, values per token-head: "
                           "64/8 heads, head_dim 128, block 32, 64 x 4096",
                           lambda dev: W.quant_long("int8_kchan", "a", dev)),
    "shared_prefix": ("Shared prompt: 200 requests, 1500-token prefix in 94 shared blocks (the last "
                      "copied on write per request), suffixes U[1,512], 64/8 heads, D 128, bf16, "
                      "block 16; GB/s counts logical bytes (the shared prefix is read from L2)",
                      lambda dev: SharedPrefixStep(dev)),
    "shared_prefix_cascade": ("Shared prompt as above through the cascade step: the 93 blocks all "
                              "200 requests still share once for all of them on the tensor cores, "
                              "each request's remaining positions through the decode kernel, then "
                              "the merge; GB/s counts the same logical bytes",
                              lambda dev: SharedPrefixStep(dev, cascade=True)),
}


def measured_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def elt_bytes(cache):
    return 2 if cache in ("bf16", "fp16") else 0.5 if cache == "int4" else 1


def max_over_ranks(values, world, device):
    """Per-rank times -> the slowest rank's (every rank gets the same list)."""
    if world == 1:
        return list(values)
    t = torch.tensor(values, device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return [float(x) for x in t]


def job_throughput(bytes_per_step, world, step_s):
    """Whole-job GB/s: every rank (replica) moves bytes_per_step per step; the
    job's step takes the slowest rank's time."""
    return bytes_per_step * world / step_s / 1e9


def step_bytes(wl):
    """Algorithmic bytes of one step: (decode kernel bytes, append bytes)."""
    e = elt_bytes(wl.cache_dtype)
    tokens = int(wl.context_lens.sum())
    kv = tokens * wl.kv_heads * wl.head_dim * 2 * e
    if wl.cache_dtype in ("int8", "e5m2", "int4"):
        kv += tokens * wl.kv_heads * 2 * 4                   # per-token-head scales
    elif wl.cache_dtype == "int8_kchan":
        kv += tokens * wl.kv_heads * 4 + wl.kv_heads * wl.head_dim * 4   # V rows + K channels
    q_out = 2 * wl.batch * wl.q_heads * wl.head_dim * 2
    rows = wl.batch * wl.kv_heads
    append = rows * wl.head_dim * 2 * 2 + wl.batch * 8        # read new K, V and slots
    append += rows * wl.head_dim * 2 * e + \
        (rows * 2 * 4 if wl.cache_dtype in ("int8", "e5m2", "int4") else
         rows * 4 if wl.cache_dtype == "int8_kchan" else 0)                  # write rows
    return int(kv + q_out), int(append)


def cascade_hbm_bytes(wl):
    """Bytes a cascade step must read or write in HBM: the shared blocks' K/V
    once, the K/V of every position past them, q, out and the new rows."""
    bs, row = wl.block_size, wl.kv_heads * wl.head_dim * 2 * 2      # K + V of one position
    shared = wl.cascade_blocks * bs
    later = int((wl.context_lens - shared).sum())
    q_out = 2 * wl.batch * wl.q_heads * wl.head_dim * 2
    return (shared + later) * row + q_out + step_bytes(wl)[1]


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index, period=0.002):
        self.index, self.period = index, period
        self.samples = []
        self.ok = False
        self._stop = threading.Event()
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:    # no NVML: report it, do not guess
            self.err = str(e)

    def _reasons(self):
        try:
            return self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            return self.nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append((time.time(),
                                     self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM),
                                     self._reasons()))
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def stop(self):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self, t0, t1):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        s = [x for x in self.samples if t0 <= x[0] <= t1] or self.samples[-3:]
        mhz = [x[1] for x in s]
        bits = 0
        for x in s:
            bits |= x[2]
        reasons = [n for b, n in self.REASONS.items() if bits & b and n != "gpu_idle"]
        return {"sm_mhz": float(np.median(mhz)) if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(s)}


def hold_gpu(seconds):
    """Queue a GPU spin of about `seconds` so that the host can enqueue every
    timed step while the GPU is busy: the device-timed region then holds no
    gaps where the GPU waits for the host to launch the next kernel."""
    torch.cuda._sleep(int(max(seconds, 1e-4) * 2.0e9))   # cycles at ~2 GHz


# ------------------------------------------------------------------ oracle arm

def _host_f32(t):
    """Exact float32 host copy of a bf16 / fp16 tensor (through its bits)."""
    u = t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    if t.dtype == torch.bfloat16:
        return (u.astype(np.uint32) << 16).view(np.float32)
    return u.view(np.float16).astype(np.float32)


class OracleStep:
    """The fp64 CPU oracle, as it stands, on one sequence of the workload at a
    time: that sequence's append (quantized for a 1-byte or 4-bit cache) and its
    decode attention for every query head. Quantized caches hold the oracle's
    own codes of the whole history, made once before timing; the shared-prompt
    workload holds the oracle's own copy-on-write cache. For a quantized cache a
    sequence's history is quantized into it by prepare(b), outside the timing,
    just before the sequence is first timed."""

    def __init__(self, wl):
        from oracle import cache_ops, quant
        self.wl = wl
        self.q = _host_f32(wl.q).astype(np.float64)
        kind = wl.cache_dtype
        self.kind = kind
        if getattr(wl, "sp", None) is not None:          # shared prompt
            self._init_shared(wl)
        elif kind in ("bf16", "fp16"):
            dt = np.float16 if kind == "fp16" else np.float32
            self.kc, self.vc = _host_f32(wl.k_fill).astype(dt), _host_f32(wl.v_fill).astype(dt)
            self.kn, self.vn = _host_f32(wl.k_new).astype(dt), _host_f32(wl.v_new).astype(dt)
            self.tables = wl.block_tables
        else:
            H, bs, D = wl.kv_heads, wl.block_size, wl.head_dim
            row = D // 2 if kind == "int4" else D
            shape = (wl.num_blocks, H, bs, row)
            cdt = np.int8 if kind in ("int8", "int8_kchan") else np.uint8
            self.kc, self.vc = np.zeros(shape, cdt), np.zeros(shape, cdt)
            self.ks = np.zeros(shape[:3], np.float32) if kind != "int8_kchan" else wl.k_chan
            self.vs = np.zeros(shape[:3], np.float32)
            self.kh, self.vh = _host_f32(wl.k_hist), _host_f32(wl.v_hist)
            self.starts = np.concatenate([[0], np.cumsum(np.maximum(wl.context_lens - 1, 0))])
            self.kn, self.vn = _host_f32(wl.k_new), _host_f32(wl.v_new)
            self.tables = wl.block_tables
        self.ready = set()
        self.outs = {}          # sequence -> the oracle's outputs of all its heads

    def prepare(self, b):
        """Untimed: sequence b's cached history in the oracle's cache."""
        from oracle import cache_ops
        wl, kind = self.wl, self.kind
        if b in self.ready or kind in ("bf16", "fp16") or getattr(wl, "sp", None) is not None:
            return
        sl = slice(int(self.starts[b]), int(self.starts[b + 1]))
        if kind == "int8_kchan":
            cache_ops.append_quantized_kchan(self.kc, self.vc, self.vs, self.kh[sl], self.vh[sl],
                                             wl.slot_hist[sl], wl.block_size, wl.k_chan)
        else:
            cache_ops.append_quantized(self.kc, self.vc, self.ks, self.vs, self.kh[sl],
                                       self.vh[sl], wl.slot_hist[sl], wl.block_size, kind)
        self.ready.add(b)

    def _init_shared(self, wl):
        from oracle import allocator, cache_ops
        sp = wl.sp
        bs, H, D, P = sp.block_size, sp.kv_heads, sp.head_dim, sp.prefix_len
        m = allocator.PoolModel(sp.num_blocks)
        kc = np.zeros((sp.num_blocks, H, bs, D), np.float32)
        vc = np.zeros_like(kc)
        pre = m.alloc(-(-P // bs))
        cache_ops.append(kc, vc, _host_f32(sp.prefix_k), _host_f32(sp.prefix_v),
                         np.array([pre[t // bs] * bs + t % bs for t in range(P)]), bs)
        sk, sv = _host_f32(sp.suffix_k), _host_f32(sp.suffix_v)
        tables, off = [], 0
        rows, slots = [], []
        for b in range(sp.batch):
            t = list(pre)
            fresh = m.alloc(1)[0]
            cache_ops.block_copy([kc, vc], [(t[-1], fresh)])
            t[-1] = fresh
            L = P + int(sp.suffix_lens[b])
            t += m.alloc(-(-L // bs) - len(t))
            for p_ in range(P, L - 1):                    # the history; the last is the step's
                rows.append(off + p_ - P)
                slots.append(t[p_ // bs] * bs + p_ % bs)
            off += int(sp.suffix_lens[b])
            tables.append(t)
        cache_ops.append(kc, vc, sk[rows], sv[rows], np.array(slots), bs)
        mb = max(len(t) for t in tables)
        self.tables = np.full((sp.batch, mb), -1, np.int64)
        for b, t in enumerate(tables):
            self.tables[b, :len(t)] = t
        self.kc, self.vc = kc, vc
        self.kn, self.vn = _host_f32(wl.k_new), _host_f32(wl.v_new)
        L = wl.context_lens
        self.slot_new = np.array([tables[b][(L[b] - 1) // bs] * bs + (L[b] - 1) % bs
                                  for b in range(sp.batch)], np.int64)

    def run(self, b):
        """Append and decode of sequence b; returns the metric's bytes for it."""
        from oracle import attention, cache_ops, quant
        wl, kind = self.wl, self.kind
        slot = (self.slot_new if hasattr(self, "slot_new") else wl.slot_new)[b:b + 1]
        if kind in ("bf16", "fp16"):
            cache_ops.append(self.kc, self.vc, self.kn[b:b + 1], self.vn[b:b + 1], slot,
                             wl.block_size)
            kd, vd = self.kc, self.vc
            nblk = -(-int(wl.context_lens[b]) // wl.block_size)
            ids = self.tables[b, :nblk]
            tab = self.tables
        else:
            if kind == "int8_kchan":
                cache_ops.append_quantized_kchan(self.kc, self.vc, self.vs, self.kn[b:b + 1],
                                                 self.vn[b:b + 1], slot, wl.block_size, wl.k_chan)
            else:
                cache_ops.append_quantized(self.kc, self.vc, self.ks, self.vs, self.kn[b:b + 1],
                                           self.vn[b:b + 1], slot, wl.block_size, kind)
            # dequantize the sequence's blocks (the oracle attends over values)
            nblk = -(-int(wl.context_lens[b]) // wl.block_size)
            ids = self.tables[b, :nblk]
            unpack = quant.unpack_int4 if kind == "int4" else (lambda c: c)
            if kind == "int8_kchan":
                kd = quant.dequantize_k_channels(self.kc[ids].transpose(0, 2, 1, 3), wl.k_chan) \
                    .transpose(0, 2, 1, 3)
                vd = quant.dequantize(self.vc[ids], self.vs[ids], "int8")
            else:
                kd = quant.dequantize(unpack(self.kc[ids]), self.ks[ids], kind)
                vd = quant.dequantize(unpack(self.vc[ids]), self.vs[ids], kind)
            tab = np.full_like(self.tables, -1)
            tab[b, :nblk] = np.arange(nblk)
        self.outs[b] = np.stack([attention.decode_one(self.q, kd, vd, tab, wl.context_lens,
                                                      wl.scale, b, h) for h in range(wl.q_heads)])
        e = elt_bytes(kind)
        nb = int(wl.context_lens[b]) * wl.kv_heads * wl.head_dim * 2 * e \
            + 2 * wl.q_heads * wl.head_dim * 2 + wl.kv_heads * wl.head_dim * 2 * 2 * (1 + e)
        if kind in ("int8", "e5m2", "int4", "int8_kchan"):
            nb += int(wl.context_lens[b]) * wl.kv_heads * 8
        return nb


def oracle_sample(wl, budget_s=15.0, threads=None):
    """Time the CPU oracle (as it stands) on a bounded sample of the step: the
    append and decode of whole sequences, taken in order until ~budget_s of
    CPU work. threads: BLAS threads for the run (None: as configured).
    Returns (GB/s in the metric's bytes, seconds, sequences, threads used,
    {sequence: the oracle's outputs [Hq, D]})."""
    from threadpoolctl import threadpool_info, threadpool_limits
    ost = OracleStep(wl)
    with threadpool_limits(limits=threads):
        used = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
        done, nbytes, t_total, t_setup = 0, 0, 0.0, 0.0
        for b in range(wl.batch):
            t0 = time.perf_counter()
            ost.prepare(b)                         # untimed: the cache before the step
            t1 = time.perf_counter()
            nbytes += ost.run(b)
            t_total += time.perf_counter() - t1
            t_setup += t1 - t0
            done += 1
            if t_total >= budget_s or t_setup >= 2 * budget_s:
                break
    return nbytes / t_total / 1e9, t_total, done, used, ost.outs


def output_check(gpu_out, oracle_outs, tol=1e-2):
    """The step's GPU outputs against the oracle's on the sampled sequences
    (decode: the first ones of the batch, in order) or new-token rows
    (prefill): how many, max abs and max rel (floor 1e-2 on |oracle|) error,
    both within tol. gpu_out's first index is the sample's key."""
    g = _host_f32(gpu_out).astype(np.float64)
    ea = er = 0.0
    for b, o in oracle_outs.items():
        err = np.abs(g[b] - o)
        ea = max(ea, float(err.max()))
        er = max(er, float((err / np.maximum(np.abs(o), 1e-2)).max()))
    return {"sequences": len(oracle_outs), "max_abs": ea, "max_rel": er,
            "tolerance": tol, "ok": bool(ea <= tol and er <= tol)}


# ------------------------------------------------------------------ shared prefix

class SharedPrefixStep:
    """The shared-prompt workload as a decode step: 200 requests share a
    1500-token prompt (94 blocks of 16, the last holding 12 tokens). Setup goes
    through the library's allocator: each request shares the prompt blocks,
    copies the partial one on write, and appends its suffix except the last
    token, which is the step's append."""

    def __init__(self, device, cascade=False):
        self.sp = sp = W.shared_prefix(device)
        # cascade step: the prompt's full blocks, shared by every request
        self.cascade_blocks = sp.prefix_len // sp.block_size if cascade else 0
        self.batch, self.q_heads, self.kv_heads = sp.batch, sp.q_heads, sp.kv_heads
        self.head_dim, self.block_size, self.cache_dtype = sp.head_dim, sp.block_size, "bf16"
        self.group = sp.q_heads // sp.kv_heads
        self.scale, self.q, self.num_blocks = sp.scale, sp.q, sp.num_blocks
        self.k_fill = None
        self.context_lens = (sp.prefix_len + sp.suffix_lens).astype(np.int32)
        ends = np.cumsum(sp.suffix_lens) - 1          # each request's last suffix row
        idx = torch.from_numpy(ends.astype(np.int64)).to(sp.suffix_k.device)
        self.k_new = sp.suffix_k.index_select(0, idx).contiguous()
        self.v_new = sp.suffix_v.index_select(0, idx).contiguous()

    def setup(self, pool, pkv):
        sp, bs = self.sp, self.block_size
        dev = sp.q.device
        P = sp.prefix_len
        nprefix = -(-P // bs)
        prefix_ids = pool.alloc(nprefix)
        slots = torch.tensor([prefix_ids[t // bs] * bs + t % bs for t in range(P)],
                             dtype=torch.int64, device=dev)
        pkv.kv_append(pool, 0, sp.prefix_k, sp.prefix_v, slots)
        tables, pairs = [], []
        for _ in range(self.batch):
            pool.share(prefix_ids)
            tables.append(list(prefix_ids))
        for t in tables:                      # copy-on-write of the partial block
            new = pool.cow_prepare(t[-1])
            pairs.append((t[-1], new))
            t[-1] = new
        pkv.kv_block_copy(pool, pairs)
        sl, rows, off = [], [], 0
        for b, t in enumerate(tables):
            L = int(self.context_lens[b])
            t += pool.alloc(-(-L // bs) - len(t))
            sl += [t[p // bs] * bs + p % bs for p in range(P, L - 1)]
            rows += list(range(off, off + int(sp.suffix_lens[b]) - 1))
            off += int(sp.suffix_lens[b])
        if sl:
            ri = torch.tensor(rows, dtype=torch.int64, device=dev)
            pkv.kv_append(pool, 0, sp.suffix_k.index_select(0, ri).contiguous(),
                          sp.suffix_v.index_select(0, ri).contiguous(),
                          torch.tensor(sl, dtype=torch.int64, device=dev))
        mb = max(len(t) for t in tables)
        self.block_tables = np.full((self.batch, mb), -1, np.int32)
        for b, t in enumerate(tables):
            self.block_tables[b, :len(t)] = t
        L = self.context_lens
        self.slot_new = np.array([tables[b][(L[b] - 1) // bs] * bs + (L[b] - 1) % bs
                                  for b in range(self.batch)], np.int64)


# ------------------------------------------------------------------ prefill

PREFILL_WORKLOADS = {
    "prefill70b": ("LLaMA-70B-shaped GQA layer (64/8 heads, D 128, bf16, block 16): 8 requests "
                   "each prefilling 512 new tokens behind a 1536-token cached prefix",
                   lambda dev: W.prefill70b(dev)),
}


def prefill_flops(pw):
    """Algorithmic FLOPs: each new token at position p and each query head does
    q.K over p + 1 positions and P.V over them (2 FLOPs per multiply-add)."""
    wl = pw.cache
    tot = 0
    for b in range(wl.batch):
        L, c = int(wl.context_lens[b]), int(pw.chunk_lens[b])
        tot += sum(L - c + i + 1 for i in range(c))
    return 4 * wl.head_dim * wl.q_heads * tot


def run_prefill(args, rank, world, device):
    import paged_kv_cache_440_b200 as pkv
    desc, make = PREFILL_WORKLOADS[args.workload]
    pw = make(device)
    wl = pw.cache
    pool = pkv.KVPool(1, wl.num_blocks, wl.block_size, wl.kv_heads, wl.head_dim,
                      wl.cache_dtype, device)
    K, V, _, _ = pool.layer_views(0)
    K.copy_(wl.k_fill)
    V.copy_(wl.v_fill)
    tables = torch.from_numpy(wl.block_tables).to(device)
    lens = torch.from_numpy(wl.context_lens.astype(np.int32)).to(device)
    cu = torch.from_numpy(pw.cu_q).to(device)
    max_q, max_ctx = int(pw.chunk_lens.max()), int(wl.context_lens.max())
    out = torch.empty_like(pw.q)
    flush = torch.ones(64 << 20, dtype=torch.float32, device=device)
    sink = torch.empty((), dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)

    def step(q=pw.q, tb=tables, ln=lens, c=cu, o=out):
        pkv.paged_attn_prefill(pool, 0, q, c, max_q, tb, ln, max_ctx, wl.scale, out=o)

    for _ in range(args.warmup):
        torch.sum(flush, 0, out=sink)
        step()
    torch.cuda.synchronize(device)
    pool.status_clear()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    sampler = ClockSampler(device.index if device.index is not None else 0).start()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(device)
    t0 = time.time()
    hold_gpu(1e-3 + 150e-6 * args.steps)
    for i in range(args.steps):
        torch.sum(flush, 0, out=sink)
        evs[i][0].record(stream)
        step()
        evs[i][1].record(stream)
    torch.cuda.synchronize(device)
    t1 = time.time()
    sampler.stop()
    out_timed = out.clone()        # the last timed step's outputs, for the output check
    step_s = float(np.mean([a.elapsed_time(b_) for a, b_ in evs])) / 1e3
    step_s, = max_over_ranks([step_s], world, device)
    e2e = None
    if not args.no_e2e:
        h_q = pw.q.cpu().pin_memory()
        h_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        d_q = torch.empty_like(pw.q)
        times = []
        for i in range(args.warmup + max(10, args.steps // 10)):
            torch.sum(flush, 0, out=sink)
            torch.cuda.synchronize(device)
            a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            d_q.copy_(h_q, non_blocking=True)
            step(q=d_q)
            h_out.copy_(out, non_blocking=True)
            b_.record(stream)
            b_.synchronize()
            if i >= args.warmup:
                times.append(a.elapsed_time(b_) / 1e3)
        e2e_s, = max_over_ranks([float(np.mean(times))], world, device)
        e2e = (e2e_s, h_q.numel() * 2, h_out.numel() * 2)
    return {"pw": pw, "desc": desc, "step_s": step_s, "out": out_timed,
            "clocks": sampler.summary(t0, t1),
            "status": pool.status(), "e2e": e2e, "launches": args.steps}


def prefill_oracle_sample(pw, budget_s, threads=None):
    """TFLOP/s of the fp64 oracle on a bounded sample of the prefill rows:
    (TFLOP/s, seconds, rows, {new-token row: its outputs [Hq, D]}, threads)."""
    from threadpoolctl import threadpool_info, threadpool_limits
    with threadpool_limits(limits=threads):
        used = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
        return _prefill_oracle_sample(pw, budget_s) + (used,)


def _prefill_oracle_sample(pw, budget_s):
    from oracle import attention
    wl = pw.cache
    k = wl.k_fill.float().cpu().numpy()
    v = wl.v_fill.float().cpu().numpy()
    q = pw.q.float().cpu().numpy().astype(np.float64)
    G = wl.q_heads // wl.kv_heads
    flops, t, rows, outs = 0, 0.0, 0, {}
    for b in range(wl.batch):
        L, c = int(wl.context_lens[b]), int(pw.chunk_lens[b])
        for i in range(0, c, 37):                     # a spread of positions
            pos = L - c + i
            r = int(pw.cu_q[b]) + i
            t0 = time.perf_counter()
            outs[r] = np.stack([attention.prefill_one(q[r, h], k, v, wl.block_tables[b], pos,
                                                      h // G, wl.scale)
                                for h in range(wl.q_heads)])
            t += time.perf_counter() - t0
            flops += 4 * wl.head_dim * wl.q_heads * (pos + 1)
            rows += 1
            if t >= budget_s:
                return flops / t / 1e12, t, rows, outs
    return flops / t / 1e12, t, rows, outs


def prefill_main(args, rank, world, device):
    r = run_prefill(args, rank, world, device)
    pw = r["pw"]
    wl = pw.cache
    flops = prefill_flops(pw) * world
    tflops = flops / r["step_s"] / 1e12
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            peak, kind = float(json.load(f)["bf16_tflops"]), "measured (MEASURED_PEAKS.json bf16_tflops, cuBLAS burst)"
    except Exception:
        peak, kind = 1590.0, "fallback 1590 TFLOP/s"
    traffic = None
    try:
        with open(TRAFFIC_FILE) as f:
            tr = json.load(f).get(args.workload)
        if tr and tr.get("kernel_source_hash") == kernel_hash("attn_prefill.cu"):
            traffic = tr["bytes_per_launch"]
    except (OSError, ValueError):
        pass
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, secs, rows, oouts, threads = prefill_oracle_sample(pw, args.cpu_budget)
        v1, secs1, rows1, _, _ = prefill_oracle_sample(pw, args.cpu_budget / 3, threads=1)
        cpu = {"value": round(v, 6), "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
               "sample": "%d new-token rows (all 64 heads each), %.1f s of fp64 numpy" % (rows, secs),
               "one_thread": {"value": round(v1, 6), "unit": "TFLOP/s",
                              "sample": "%d rows, %.1f s" % (rows1, secs1)},
               # the timed step's outputs of the sampled rows against the oracle's
               "output_check": output_check(r["out"], oouts)}
    if rank == 0:
        line = {
            "metric": "chunked prefill attention TFLOP/s", "value": round(tflops, 2),
            "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(r["step_s"] * 1e3, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": wl.cache_dtype, "data": "synthetic",
            "config": {"workload": r["desc"], "batch": wl.batch, "new_tokens": int(pw.cu_q[-1]),
                       "cached_tokens": int(wl.context_lens.sum()), "q_heads": wl.q_heads,
                       "kv_heads": wl.kv_heads, "head_dim": wl.head_dim,
                       "block_size": wl.block_size,
                       "parallelism": "replicas" if world > 1 else "1 gpu",
                       "l2": "L2 flushed before each timed step by reading 256 MiB"},
            "roofline": {"bound": "tensor", "achieved": round(tflops / world, 2), "peak": peak,
                         "unit": "TFLOP/s", "frac": round(tflops / world / peak, 4),
                         "traffic": traffic, "kernel": "attn_prefill_kernel", "peak_source": kind,
                         "kernel_ms": round(r["step_s"] * 1e3, 5)},
            "cpu_baseline": cpu,
            "e2e": None if r["e2e"] is None else {
                "value": round(flops / r["e2e"][0] / 1e12, 2), "unit": "TFLOP/s",
                "h2d_bytes_per_step": r["e2e"][1], "d2h_bytes_per_step": r["e2e"][2]},
            "gpu_launches": r["launches"], "clocks": r["clocks"], "device_status": r["status"],
        }
        print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ ours

def run_ours(args, rank, world, device):
    import paged_kv_cache_440_b200 as pkv
    desc, make = WORKLOADS[args.workload]
    wl = make(device)
    pool = pkv.KVPool(1, wl.num_blocks, wl.block_size, wl.kv_heads, wl.head_dim,
                      wl.cache_dtype, device)
    K, V, KS, _ = pool.layer_views(0)
    if getattr(wl, "k_chan", None) is not None:
        KS.copy_(torch.from_numpy(wl.k_chan).to(device))   # the layer's key channel scales
    if getattr(wl, "setup", None) is not None:
        wl.setup(pool, pkv)        # builds the cache through the allocator and CoW
    elif wl.k_fill is not None:
        K.copy_(wl.k_fill)
        V.copy_(wl.v_fill)
    else:
        slots = torch.from_numpy(wl.slot_hist).to(device)
        for s in range(0, wl.k_hist.shape[0], 65536):
            pkv.kv_append(pool, 0, wl.k_hist[s:s + 65536].contiguous(),
                          wl.v_hist[s:s + 65536].contiguous(), slots[s:s + 65536].contiguous())
    tables = torch.from_numpy(wl.block_tables).to(device)
    lens = torch.from_numpy(wl.context_lens.astype(np.int32)).to(device)
    slot_new = torch.from_numpy(wl.slot_new).to(device)
    max_ctx = int(wl.context_lens.max())
    G = args.ctas or pkv.default_ctas(pool)
    casc = getattr(wl, "cascade_blocks", 0)
    ws = (pkv.make_cascade_workspace if casc else pkv.make_workspace)(pool, wl.batch,
                                                                       wl.q_heads, G)
    out = torch.empty_like(wl.q)
    flush = torch.ones(64 << 20, dtype=torch.float32, device=device)   # 256 MiB
    flush_sink = torch.empty((), dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)

    def flush_l2():
        torch.sum(flush, 0, out=flush_sink)

    fused = not args.separate_append and wl.group <= 8

    def one_step():
        if casc:    # shared prefix once for all requests, then per request, then the merge
            pkv.paged_attn_decode_cascade(pool, 0, wl.q, tables, lens, max_ctx, casc, wl.scale,
                                          k_new=wl.k_new, v_new=wl.v_new, out=out, num_ctas=G,
                                          workspace=ws)
        elif fused:   # append folded into the attention kernel, then the merge
            pkv.paged_attn_decode_append(pool, 0, wl.q, wl.k_new, wl.v_new, tables, lens,
                                         max_ctx, wl.scale, out=out, num_ctas=G, workspace=ws)
        else:
            pkv.kv_append(pool, 0, wl.k_new, wl.v_new, slot_new)
            pkv.paged_attn_decode(pool, 0, wl.q, tables, lens, max_ctx, wl.scale, out=out,
                                  num_ctas=G, workspace=ws)

    for _ in range(args.warmup):
        flush_l2()
        one_step()
    torch.cuda.synchronize(device)
    pool.status_clear()

    # Timed region: K steps, each bracketed by events; the L2 flush before each
    # step is outside the events. A GPU spin queued first lets the host enqueue
    # every step before the GPU reaches it, so no step waits on the host.
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    sampler = ClockSampler(device.index if device.index is not None else 0).start()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(device)
    t0 = time.time()
    hold_gpu(1e-3 + 150e-6 * args.steps)
    for i in range(args.steps):
        flush_l2()
        evs[i][0].record(stream)
        one_step()
        evs[i][1].record(stream)
    torch.cuda.synchronize(device)
    t1 = time.time()
    out_timed = out.clone()        # the last timed step's outputs, for the output check
    if world > 1:
        torch.distributed.barrier()
    # The attention kernel alone, same conditions (L2 flushed before each launch),
    # for its roofline fraction.
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    hold_gpu(1e-3 + 150e-6 * args.steps)
    for i in range(args.steps if not casc else 0):   # (cascade: the step is the figure)
        flush_l2()
        kev[i][0].record(stream)
        if fused:
            pkv.paged_attn_partition_append(pool, 0, wl.q, wl.k_new, wl.v_new, tables, lens,
                                            max_ctx, wl.scale, out, ws, num_ctas=G)
        else:
            pkv.paged_attn_partition(pool, 0, wl.q, tables, lens, max_ctx, wl.scale, out, ws,
                                     num_ctas=G)
        kev[i][1].record(stream)
    torch.cuda.synchronize(device)
    t2 = time.time()
    sampler.stop()
    status = pool.status()
    step_ms = np.array([a.elapsed_time(b) for a, b in evs])
    step_s = float(step_ms.mean()) / 1e3
    part_s = float(np.mean([a.elapsed_time(b) for a, b in kev])) / 1e3 if not casc else \
        float(step_ms.mean()) / 1e3
    step_s, part_s = max_over_ranks([step_s, part_s], world, device)
    clocks = sampler.summary(t0, t2)

    # ---------------------------------------------------------- end to end
    e2e = None
    if not args.no_e2e:
        # The step's inputs travel in one pinned host buffer and one copy: q,
        # the new K/V rows, block tables, lengths (and slots when the append is
        # a separate kernel), each at a 256-byte offset.
        parts = [wl.q, wl.k_new, wl.v_new, tables, lens] + ([] if fused else [slot_new])
        offs, n = [], 0
        for t in parts:
            offs.append(n)
            n += -(-t.numel() * t.element_size() // 256) * 256
        h_in = torch.empty(n, dtype=torch.uint8).pin_memory()
        d_in = torch.empty(n, dtype=torch.uint8, device=device)
        views = []
        for t, o in zip(parts, offs):
            nb = t.numel() * t.element_size()
            h_in[o:o + nb].copy_(t.contiguous().view(torch.uint8).reshape(-1).cpu())
            views.append(d_in[o:o + nb].view(t.dtype).view(t.shape))
        d_q, d_kn, d_vn, d_tab, d_len = views[:5]
        d_slot = None if fused else views[5]
        h_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        d_out = torch.empty_like(out)
        h2d = sum(t.numel() * t.element_size() for t in parts)
        d2h = h_out.numel() * h_out.element_size()
        n_e2e = max(10, args.steps // 10)
        times = []
        for i in range(args.warmup + n_e2e):
            flush_l2()
            torch.cuda.synchronize(device)
            a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            d_in.copy_(h_in, non_blocking=True)
            if casc:
                pkv.paged_attn_decode_cascade(pool, 0, d_q, d_tab, d_len, max_ctx, casc, wl.scale,
                                              k_new=d_kn, v_new=d_vn, out=d_out, num_ctas=G,
                                              workspace=ws)
            elif fused:
                pkv.paged_attn_decode_append(pool, 0, d_q, d_kn, d_vn, d_tab, d_len, max_ctx,
                                             wl.scale, out=d_out, num_ctas=G, workspace=ws)
            else:
                pkv.kv_append(pool, 0, d_kn, d_vn, d_slot)
                pkv.paged_attn_decode(pool, 0, d_q, d_tab, d_len, max_ctx, wl.scale, out=d_out,
                                      num_ctas=G, workspace=ws)
            h_out.copy_(d_out, non_blocking=True)
            b_.record(stream)
            b_.synchronize()
            if i >= args.warmup:
                times.append(a.elapsed_time(b_) / 1e3)
        e2e_s = float(np.mean(times))
        e2e_s, = max_over_ranks([e2e_s], world, device)
        e2e = (e2e_s, h2d, d2h)

    dec_bytes, app_bytes = step_bytes(wl)
    res = {"wl": wl, "desc": desc, "G": G, "step_s": step_s, "part_s": part_s, "out": out_timed,
           "dec_bytes": dec_bytes, "app_bytes": app_bytes, "clocks": clocks, "fused": fused,
           "status": status, "e2e": e2e,
           "launches": args.steps * (2 if fused and not casc else 3), "cascade": casc,
           "wall": t1 - t0, "step_ms_median": float(np.median(step_ms))}
    return res


CACHE_OPS = ("Cache ops of a LLaMA-70B-shaped model (80 layers, 8 kv heads, head_dim 128, "
             "block 16): bf16 append of one decode step (32 tokens) and of 4096-token chunks "
             "(one launch alone, and 16 chunks into 16 layers back to back), INT8 append of a "
             "chunk, INT8 quantize of 32768 rows, copy-on-write copy of 200 blocks in every "
             "layer (K and V) and in one layer")
CACHE_LAYERS = 80


def cache_ops_main(args, device):
    """Time kv_append, kv_quantize and kv_block_copy (CUDA events; L2 flushed
    before each timed region) and report their algorithmic GB/s. A single
    launch's region also holds the launch itself (an empty kernel measures
    about 6 us under this protocol), so the chunk appends are also timed as
    a stream of 16 launches on distinct data."""
    import paged_kv_cache_440_b200 as pkv
    g = torch.Generator(device=device).manual_seed(0)
    NB, bs, H, D, T, NC = 5504, 16, 8, 128, 4096, 16
    layers = max(1, args.cache_layers)
    pool = pkv.KVPool(layers, NB, bs, H, D, "bf16", device)
    qpool = pkv.KVPool(1, NB, bs, H, D, "int8", device)
    pool1 = pkv.KVPool(1, NB, bs, H, D, "bf16", device)
    for pl in (qpool, pool1):
        for t in pl.layer_views(0):
            if t is not None:
                t.zero_()
    ks = [torch.randn(T, H, D, generator=g, device=device).to(torch.bfloat16) for _ in range(NC)]
    vs = [torch.randn(T, H, D, generator=g, device=device).to(torch.bfloat16) for _ in range(NC)]
    perm = torch.randperm(NB * bs, generator=g, device=device)
    slots = [perm[i * T:(i + 1) * T].to(torch.int64).contiguous() for i in range(NC)]
    x = torch.randn(T * H, D, generator=g, device=device).to(torch.bfloat16)
    codes = torch.empty(T * H, D, dtype=torch.int8, device=device)
    scales = torch.empty(T * H, dtype=torch.float32, device=device)
    ids = torch.randperm(NB, generator=torch.Generator().manual_seed(1))[:400].tolist()
    pairs = list(zip(ids[:200], ids[200:]))
    flush = torch.ones(64 << 20, dtype=torch.float32, device=device)   # 256 MiB
    sink = torch.empty((), dtype=torch.float32, device=device)
    row = H * D * 2
    chunk = T * (4 * row + 8)
    blk = 2 * 2 * H * bs * D * 2                  # K and V of one block, read and written
    # name, launch i of the timed region, launches per region, bytes per launch
    ops = [
        ("append_step_bf16", lambda i: pkv.kv_append(pool1, 0, ks[0][:32], vs[0][:32], slots[0][:32]),
         1, 32 * (4 * row + 8)),
        ("append_chunk_bf16", lambda i: pkv.kv_append(pool1, 0, ks[0], vs[0], slots[0]), 1, chunk),
        ("append_chunk_bf16_stream", lambda i: pkv.kv_append(pool, i % layers, ks[i], vs[i], slots[i]),
         NC, chunk),
        ("append_chunk_int8", lambda i: pkv.kv_append(qpool, 0, ks[0], vs[0], slots[0]), 1,
         T * (2 * row + 2 * H * D + 2 * H * 4 + 8)),
        ("quantize_int8", lambda i: pkv.kv_quantize(x, "int8", codes=codes, scales=scales), 1,
         T * H * (D * 2 + D + 4)),
        ("block_copy_200_one_layer", lambda i: pkv.kv_block_copy(pool1, pairs), 1, 200 * blk),
        ("block_copy_200_all_layers", lambda i: pkv.kv_block_copy(pool, pairs), 1,
         200 * layers * blk),
    ]
    steps = max(1, min(args.steps, 200))
    peak, peak_kind = measured_peak()
    parts = {}
    sampler = ClockSampler(device.index if device.index is not None else 0).start()
    t0 = time.time()
    for name, fn, inner, nbytes in ops:
        n = steps if inner == 1 and nbytes < (1 << 30) else max(1, min(steps, 20))
        for _ in range(args.warmup):
            torch.sum(flush, 0, out=sink)
            for i in range(inner):
                fn(i)
        torch.cuda.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(n)]
        hold_gpu(1e-3 + (300e-6 * inner + nbytes / 4e12) * n)   # every launch queued first
        for a, b_ in evs:
            torch.sum(flush, 0, out=sink)
            a.record()
            for i in range(inner):
                fn(i)
            b_.record()
        torch.cuda.synchronize()
        sec = sum(a.elapsed_time(b_) for a, b_ in evs) / n / inner / 1e3
        parts[name] = {"us": round(sec * 1e6, 2), "bytes": int(nbytes), "launches": inner,
                       "regions": n,
                       "GB/s": round(nbytes / sec / 1e9, 1),
                       "frac": round(nbytes / sec / 1e9 / peak, 4)}
    t1 = time.time()
    sampler.stop()
    big = parts["append_chunk_bf16_stream"]
    print(json.dumps({
        "metric": "KV cache ops GB/s (append, quantize, copy-on-write copy)",
        "value": big["GB/s"], "unit": "GB/s", "n_gpus": 1, "steps": steps,
        "warmup": args.warmup, "ms_per_step": round(big["us"] * big["launches"] / 1e3, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": CACHE_OPS, "layers": layers,
                   "l2": "L2 flushed before each timed region by reading "
                   "256 MiB; a stream's 16 chunks are distinct (537 MB, above the L2)"},
        "roofline": {"bound": "hbm", "achieved": big["GB/s"], "peak": peak, "unit": "GB/s",
                     "frac": big["frac"], "traffic": None, "kernel": "append16_kernel",
                     "peak_source": peak_kind},
        "parts": parts, "clocks": sampler.summary(t0, t1),
        "gpu_launches": sum(p["regions"] * p["launches"] for p in parts.values()),
        "device_status": pool.status() | pool1.status() | qpool.status()}),
        flush=True)


def reference_arm(args, world):
    """The reference arm's JSON line: the CPU oracle timed over exactly
    args.steps bounded steps after args.warmup untimed ones."""
    from threadpoolctl import threadpool_info
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    if args.workload in PREFILL_WORKLOADS:
        from oracle import attention
        desc, make = PREFILL_WORKLOADS[args.workload]
        pw = make("cpu")
        wl = pw.cache
        k, v = wl.k_fill.float().numpy(), wl.v_fill.float().numpy()
        q = pw.q.float().numpy().astype(np.float64)
        G = wl.q_heads // wl.kv_heads
        rows = [(b, i) for b in range(wl.batch) for i in range(0, int(pw.chunk_lens[b]), 37)]

        def one(n):
            b, i = rows[n % len(rows)]
            pos = int(wl.context_lens[b]) - int(pw.chunk_lens[b]) + i
            for h in range(wl.q_heads):
                attention.prefill_one(q[pw.cu_q[b] + i, h], k, v, wl.block_tables[b], pos,
                                      h // G, wl.scale)
            return 4 * wl.head_dim * wl.q_heads * (pos + 1)
        metric, unit, what = ("chunked prefill attention TFLOP/s", "TFLOP/s",
                              "one new-token row (all %d heads)" % wl.q_heads)
        scale_out = 1e12
    elif args.workload == "cache_ops":
        from oracle import cache_ops
        NB, bs, H, D, T = 5504, 16, 8, 128, 4096
        rng = np.random.default_rng(0)
        kc = np.zeros((NB, H, bs, D), dtype=np.uint16)
        vc = np.zeros_like(kc)
        kn = rng.integers(0, 1 << 16, (T, H, D), dtype=np.uint16)
        vn = rng.integers(0, 1 << 16, (T, H, D), dtype=np.uint16)
        slots = rng.permutation(NB * bs)[:T].astype(np.int64)

        def one(n):
            cache_ops.append(kc, vc, kn, vn, slots, bs)
            return T * (4 * H * D * 2 + 8)
        desc = CACHE_OPS
        wl = type("CacheOps", (), {"batch": T})
        metric, unit, what = ("KV cache ops GB/s (append, quantize, copy-on-write copy)", "GB/s",
                              "one 4096-token bf16 chunk appended at random rows")
        scale_out = 1e9
    else:
        desc, make = WORKLOADS[args.workload]
        wl = make("cpu")
        ost = OracleStep(wl)

        def one(n):
            b = n % wl.batch
            ost.prepare(b)        # untimed below: the cache state before the step
            return b
        metric, unit, what = (METRIC, "GB/s",
                              "one sequence's append and decode (all %d heads)" % wl.q_heads)
        scale_out = 1e9
    times, work = [], 0
    for n in range(args.warmup + args.steps):
        if args.workload in PREFILL_WORKLOADS or args.workload == "cache_ops":
            t0 = time.perf_counter()
            w = one(n)
            dt = time.perf_counter() - t0
        else:
            b = one(n)
            t0 = time.perf_counter()
            w = ost.run(b)
            dt = time.perf_counter() - t0
        if n >= args.warmup:
            times.append(dt)
            work += w
    secs = float(np.sum(times))
    value = work / secs / scale_out
    sample = "each step %s, in order; %d timed steps, %.2f s" % (what, args.steps, secs)
    return {
        "impl": "reference", "metric": metric, "value": round(value, 6), "unit": unit,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(secs / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "u16" if args.workload == "cache_ops" else "f64", "data": "synthetic",
        "config": {"workload": desc, "batch": wl.batch},
        "cpu_baseline": {"value": round(value, 6), "unit": unit, "cores": threads,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 6), "unit": unit, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS) + sorted(PREFILL_WORKLOADS) +
                    ["cache_ops"], default="gqa70b")
    ap.add_argument("--ctas", type=int, default=0, help="CTAs of the attention kernel (0 = one per SM)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--separate-append", action="store_true",
                    help="kv_append + paged_attn_decode instead of paged_attn_decode_append")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--cache-layers", type=int, default=CACHE_LAYERS,
                    help="cache_ops: layers of the pool (the copy-on-write copy covers all of them)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))

    if args.impl == "reference":
        # The oracle as it stands, on the host cores: W untimed and K timed steps,
        # each a bounded sample of the workload (one sequence's append and decode,
        # or one new-token row of a prefill), taken in order. Rank 0 alone.
        if rank == 0:
            print(json.dumps(reference_arm(args, world)), flush=True)
        if world > 1:
            torch.distributed.destroy_process_group()
        return

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if args.workload == "cache_ops":
        if rank == 0:
            cache_ops_main(args, device)
        if world > 1:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()
        return
    if args.workload in PREFILL_WORKLOADS:
        prefill_main(args, rank, world, device)
        if world > 1:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()
        return
    r = run_ours(args, rank, world, device)
    wl = r["wl"]
    total_bytes = (r["dec_bytes"] + r["app_bytes"]) * world
    gbs = job_throughput(r["dec_bytes"] + r["app_bytes"], world, r["step_s"])
    peak, peak_kind = measured_peak()
    # the timed kernel's algorithmic bytes: the KV stream, q and out, plus the
    # new rows when the append is folded into it
    kern_bytes = r["dec_bytes"] + (r["app_bytes"] if r.get("fused") else 0)
    achieved = kern_bytes / r["part_s"] / 1e9
    traffic = None
    try:
        with open(TRAFFIC_FILE) as f:
            tr = json.load(f).get(args.workload)
        if tr and tr.get("kernel_source_hash") == kernel_hash():
            traffic = tr["bytes_per_launch"]
    except Exception:
        pass
    bound_note = None
    if args.workload == "shared_prefix":
        # the shared prompt is read from L2, so logical bytes over time is no
        # HBM fraction: the HBM figure is the DRAM bytes ncu counted per launch
        achieved = traffic / r["part_s"] / 1e9 if traffic else None
        bound_note = ("achieved = ncu DRAM bytes per launch / kernel time (the shared prompt is "
                      "served from L2)" if traffic else
                      "no DRAM capture of the current kernel source: HBM fraction not reported")
    elif r.get("cascade"):
        # the step's three kernels as one: the bytes HBM must deliver are the
        # shared blocks' K/V once, every position past them, q, out and the new
        # rows; the timed figure is the whole step
        achieved = cascade_hbm_bytes(wl) / r["step_s"] / 1e9
        bound_note = ("whole step (prefix pass, attention, merge): achieved = the shared blocks' "
                      "K/V once + every later position's K/V + q + out + new rows, / step time")
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        g_cpu, secs, nseq, threads, oouts = oracle_sample(wl, args.cpu_budget)
        g_one, secs1, nseq1, _, _ = oracle_sample(wl, args.cpu_budget / 3, threads=1)
        cpu = {"value": round(g_cpu, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
               "sample": "%d of %d sequences (append + all %d heads each), %.1f s of fp64 numpy"
                         % (nseq, wl.batch, wl.q_heads, secs),
               "one_thread": {"value": round(g_one, 4), "unit": "GB/s",
                              "sample": "%d sequences, %.1f s" % (nseq1, secs1)},
               # the timed step's outputs of the sampled sequences against the oracle's
               "output_check": output_check(r["out"], oouts)}
    if rank == 0:
        line = {
            "metric": METRIC, "value": round(gbs, 2), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(r["step_s"] * 1e3, 5), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": wl.cache_dtype if wl.cache_dtype != "e5m2" else "fp8_e5m2",
            "data": "synthetic",
            "config": {"workload": r["desc"], "batch": wl.batch, "q_heads": wl.q_heads,
                       "kv_heads": wl.kv_heads, "head_dim": wl.head_dim,
                       "block_size": wl.block_size, "cached_tokens": int(wl.context_lens.sum()),
                       "num_ctas": r["G"], "parallelism": "replicas" if world > 1 else "1 gpu",
                       "l2": "K/V %.1fx L2 (126 MB); L2 flushed before each timed step by "
                             "reading 256 MiB" % (r["dec_bytes"] / 126e6),
                       "bytes_per_step": r["dec_bytes"] + r["app_bytes"]},
            # the shared prompt's value counts logical bytes (read from L2): no HBM percentage
            "pct_of_8tbs": None if args.workload.startswith("shared_prefix")
            else round(100 * gbs / world / NOMINAL_HBM_GBS, 2),
            "decode_tokens_per_s": round(wl.batch * world / r["step_s"], 1),
            "roofline": {"bound": "hbm",
                         "achieved": None if achieved is None else round(achieved, 2),
                         "peak": peak, "unit": "GB/s",
                         "frac": None if achieved is None else round(achieved / peak, 4),
                         "traffic": traffic, "note": bound_note,
                         "kernel": "cascade step: attn_prefill_kernel (prefix pass) + "
                                   "attn_partition_kernel + attn_merge_kernel" if r.get("cascade")
                         else "attn_partition_kernel" + (" (append fused)" if r.get("fused")
                                                         else ""),
                         "peak_source": peak_kind + " (MEASURED_PEAKS.json hbm_gbs)"
                         if peak_kind == "measured" else "fallback 6650 GB/s",
                         "kernel_ms": round(r["part_s"] * 1e3, 5)},
            "cpu_baseline": cpu,
            "e2e": None if r["e2e"] is None else {
                "value": round(total_bytes / r["e2e"][0] / 1e9, 2), "unit": "GB/s",
                "h2d_bytes_per_step": r["e2e"][1], "d2h_bytes_per_step": r["e2e"][2]},
            "gpu_launches": r["launches"],
            "clocks": r["clocks"],
            "step_ms_median": round(r["step_ms_median"], 5),
            "device_status": r["status"],
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


def kernel_hash(src="attn_decode.cu"):
    """Hash of a kernel's source file; ncu traffic figures apply only to it."""
    import hashlib
    with open(os.path.join(ROOT, "paged_kv_cache_440_b200", "csrc", src), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


if __name__ == "__main__":
    main()
