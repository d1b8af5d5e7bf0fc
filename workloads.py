"""Seeded synthetic inputs for the paged decode path.

Shared by the tests (which feed both the CUDA path and the CPU oracle) and by
``bench.py``. This module only draws random numbers and lays out block tables;
it holds none of the path's arithmetic (no attention, quantization, append or
copy). Every draw comes from one ``torch.Generator`` per workload, in a fixed
order: lengths -> placement -> q -> K -> V -> new tokens.

The shapes follow the workloads the pages describe (a 70B-class GQA layer with
8 KV heads of dim 128 in bf16, a 13B-class MHA layer with 40 heads in fp16, a
1500-token prompt shared by 200 requests, block sizes 16 and 32, per-token-head
INT8 / FP8-E5M2 KV); the values are N(0, 1) (times 0.5 for the MHA layer).
"""
from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch

_TORCH_DT = {"bf16": torch.bfloat16, "fp16": torch.float16}


@dataclass
class DecodeWorkload:
    """One decode step over a paged cache: inputs only, no results."""
    name: str
    batch: int
    q_heads: int
    kv_heads: int
    head_dim: int
    block_size: int
    q_dtype: str                 # "bf16" | "fp16"
    cache_dtype: str             # "bf16" | "fp16" | "int8" | "e5m2"
    num_blocks: int
    scale: float
    context_lens: np.ndarray     # int32 [B], includes the token appended this step
    block_tables: np.ndarray     # int32 [B, max_blocks]; -1 past the last used entry
    q: torch.Tensor              # [B, Hq, D] q_dtype
    k_new: torch.Tensor          # [B, Hkv, D] q_dtype: the step's new token
    v_new: torch.Tensor
    slot_new: np.ndarray         # int64 [B]: slot of position context_lens[b] - 1
    value_std: float = 1.0
    seed: int = 0
    # 16-bit caches: random content for every pool row, [NB, Hkv, bs, D]
    k_fill: Optional[torch.Tensor] = None
    v_fill: Optional[torch.Tensor] = None
    # 1-byte caches: the history as tokens, [T, Hkv, D] q_dtype, and their slots
    k_hist: Optional[torch.Tensor] = None
    v_hist: Optional[torch.Tensor] = None
    slot_hist: Optional[np.ndarray] = None
    # "int8_kchan" caches: the layer's fixed key channel scales, float32 [Hkv, D]
    k_chan: Optional[np.ndarray] = None
    extra: dict = field(default_factory=dict)

    @property
    def group(self):
        return self.q_heads // self.kv_heads

    @property
    def max_blocks(self):
        return self.block_tables.shape[1]

    @property
    def total_tokens(self):
        return int(np.sum(self.context_lens))


def _blocks_for(n, bs):
    return -(-int(n) // int(bs))


def _place(gen, lens, bs, num_blocks):
    """Random distinct physical blocks for every sequence, in sequence order."""
    need = [_blocks_for(n, bs) for n in lens]
    perm = torch.randperm(num_blocks, generator=gen).numpy().astype(np.int32)
    mb = max(1, max(need))
    tables = np.full((len(lens), mb), -1, dtype=np.int32)
    pos = 0
    for b, k in enumerate(need):
        tables[b, :k] = perm[pos:pos + k]
        pos += k
    return tables


def _slots(tables, lens, bs, positions):
    """slot = physical block * bs + row, for the given position of each sequence."""
    out = np.empty(len(lens), dtype=np.int64)
    for b, t in enumerate(positions):
        out[b] = int(tables[b, t // bs]) * bs + (t % bs)
    return out


def make_decode_workload(name, batch, q_heads, kv_heads, head_dim, block_size,
                         q_dtype, cache_dtype, lens, num_blocks=None, scale=None,
                         value_std=1.0, seed=0, device="cpu", slack=1.2,
                         placement=None):
    """Draw one decode step's inputs.

    lens: context lengths including the token appended this step (one per
    sequence). num_blocks defaults to ceil(slack * blocks needed).
    placement: optional explicit block tables (int32 [B, >= max blocks]).
    """
    gen = torch.Generator().manual_seed(seed)
    lens = np.asarray(lens, dtype=np.int32)
    need = sum(_blocks_for(n, block_size) for n in lens)
    if num_blocks is None:
        num_blocks = max(1, int(np.ceil(slack * need)))
    if placement is None:
        tables = _place(gen, lens, block_size, num_blocks)
    else:
        tables = np.asarray(placement, dtype=np.int32)
    if scale is None:
        scale = 1.0 / np.sqrt(head_dim)
    dt = _TORCH_DT[q_dtype]
    # Large draws go to the target device through a generator seeded from the
    # CPU stream, so the whole workload is a function of `seed` and `device`.
    dev_seed = int(torch.randint(0, 2**62, (1,), generator=gen).item())
    dgen = torch.Generator(device=device).manual_seed(dev_seed)

    def randn(*shape):
        return (torch.randn(*shape, generator=dgen, device=device, dtype=torch.float32)
                * value_std).to(dt)

    q = randn(batch, q_heads, head_dim)
    wl = DecodeWorkload(
        name=name, batch=batch, q_heads=q_heads, kv_heads=kv_heads,
        head_dim=head_dim, block_size=block_size, q_dtype=q_dtype,
        cache_dtype=cache_dtype, num_blocks=num_blocks, scale=float(scale),
        context_lens=lens, block_tables=tables, q=q,
        k_new=None, v_new=None, slot_new=None, value_std=value_std, seed=seed)
    if cache_dtype in ("bf16", "fp16"):
        wl.k_fill = randn(num_blocks, kv_heads, block_size, head_dim)
        wl.v_fill = randn(num_blocks, kv_heads, block_size, head_dim)
    else:
        hist = [int(n) - 1 for n in lens]
        T = int(sum(max(h, 0) for h in hist))
        wl.k_hist = randn(T, kv_heads, head_dim)
        wl.v_hist = randn(T, kv_heads, head_dim)
        slots = np.empty(T, dtype=np.int64)
        pos = 0
        for b, h in enumerate(hist):
            for t in range(max(h, 0)):
                slots[pos] = int(tables[b, t // block_size]) * block_size + t % block_size
                pos += 1
        wl.slot_hist = slots
    wl.k_new = randn(batch, kv_heads, head_dim)
    wl.v_new = randn(batch, kv_heads, head_dim)
    if cache_dtype == "int8_kchan":
        # keys whose channels differ in spread (sigma in [0.25, 4] per head and
        # channel), with calibrated-style channel scales 4 sigma / 127: values
        # beyond 4 sigma saturate
        sigma = torch.empty(kv_heads, head_dim).uniform_(0.25, 4.0, generator=gen)
        sig_d = sigma.to(device)
        wl.k_hist = (wl.k_hist.float() * sig_d).to(dt)
        wl.k_new = (wl.k_new.float() * sig_d).to(dt)
        wl.k_chan = (sigma * 4.0 / 127.0).numpy().astype(np.float32)
    wl.slot_new = np.where(lens > 0, _slots(tables, lens, block_size,
                                            [max(int(n) - 1, 0) for n in lens]), -1)
    return wl


# ---------------------------------------------------------------------------
# The five workloads (sizes as the pages describe them; seed 0 throughout).
# ---------------------------------------------------------------------------

def tiny(device="cpu", seed=0):
    """4 sequences of 17/33/100/250 tokens, 8 q / 2 kv heads, D 64, bs 16,
    64-block pool, tables = the first 28 blocks of a random permutation."""
    gen = torch.Generator().manual_seed(seed)
    lens = [17, 33, 100, 250]
    perm = torch.randperm(64, generator=gen).numpy().astype(np.int32)
    tables = np.full((4, 16), -1, dtype=np.int32)
    pos = 0
    for b, n in enumerate(lens):
        k = _blocks_for(n, 16)
        tables[b, :k] = perm[pos:pos + k]
        pos += k
    return make_decode_workload("tiny", 4, 8, 2, 64, 16, "bf16", "bf16", lens,
                                num_blocks=64, scale=0.125, seed=seed,
                                device=device, placement=tables)


def gqa70b(device="cpu", seed=0, batch=32, lo=512, hi=4096):
    """LLaMA-70B-shaped GQA layer: 64 q / 8 kv heads, D 128, bf16, bs 16,
    batch 32, context lengths uniform on [512, 4096], pool 1.2x the blocks needed."""
    gen = torch.Generator().manual_seed(seed)
    lens = torch.randint(lo, hi + 1, (batch,), generator=gen).numpy()
    return make_decode_workload("gqa70b", batch, 64, 8, 128, 16, "bf16", "bf16",
                                lens, seed=seed + 1, device=device)


def mha13b(device="cpu", seed=0, batch=32, ctx=2048):
    """13B-shaped MHA layer: 40 q / 40 kv heads, D 128, fp16, bs 16, batch 32,
    every context 2048 tokens, random placement, values N(0,1) * 0.5."""
    return make_decode_workload("mha13b", batch, 40, 40, 128, 16, "fp16", "fp16",
                                [ctx] * batch, value_std=0.5, seed=seed,
                                device=device)


def quant_long(kind, variant="a", device="cpu", seed=0):
    """Quantized KV: 64 q / 8 kv heads, D 128, bs 32, bf16 q; (a) 64 x 4096,
    (b) 8 x 32768 tokens; K/V ~ N(0,1) stored as INT8 or FP8-E5M2 (and the
    other 1-byte and 4-bit kinds; "int8_kchan" keys spread per channel)."""
    batch, ctx = (64, 4096) if variant == "a" else (8, 32768)
    return make_decode_workload("quant_%s_%s" % (variant, kind), batch, 64, 8, 128,
                                32, "bf16", kind, [ctx] * batch, seed=seed,
                                device=device)


@dataclass
class SharedPrefixWorkload:
    """200 requests sharing a 1500-token prompt, each with a private suffix."""
    batch: int
    prefix_len: int
    suffix_lens: np.ndarray      # int32 [B], uniform on [1, 512]
    q_heads: int
    kv_heads: int
    head_dim: int
    block_size: int
    dtype: str
    scale: float
    prefix_k: torch.Tensor       # [prefix_len, Hkv, D]
    prefix_v: torch.Tensor
    suffix_k: torch.Tensor       # [sum(suffix_lens), Hkv, D], sequence-major
    suffix_v: torch.Tensor
    q: torch.Tensor              # [B, Hq, D]
    num_blocks: int


def shared_prefix(device="cpu", seed=0, batch=200, prefix_len=1500, max_suffix=512):
    gen = torch.Generator().manual_seed(seed)
    suffix = torch.randint(1, max_suffix + 1, (batch,), generator=gen).numpy().astype(np.int32)
    bs = 16
    prefix_blocks = _blocks_for(prefix_len, bs)
    # each request: its own copy of the partial prefix block plus its suffix blocks
    per_seq = [_blocks_for(prefix_len + int(u), bs) - prefix_blocks + 1 for u in suffix]
    num_blocks = int(np.ceil(1.2 * (prefix_blocks + sum(per_seq))))
    dev_seed = int(torch.randint(0, 2**62, (1,), generator=gen).item())
    dgen = torch.Generator(device=device).manual_seed(dev_seed)

    def randn(*shape):
        return torch.randn(*shape, generator=dgen, device=device,
                           dtype=torch.float32).to(torch.bfloat16)

    q = randn(batch, 64, 128)
    pk = randn(prefix_len, 8, 128)
    pv = randn(prefix_len, 8, 128)
    total = int(suffix.sum())
    sk = randn(total, 8, 128)
    sv = randn(total, 8, 128)
    return SharedPrefixWorkload(batch, prefix_len, suffix, 64, 8, 128, bs, "bf16",
                                1.0 / np.sqrt(128), pk, pv, sk, sv, q, num_blocks)


CONFIGS = {
    "tiny": tiny,
    "gqa70b": gqa70b,
    "mha13b": mha13b,
}


# ---------------------------------------------------------------------------
# Chunked prefill: a decode-shaped 16-bit cache whose last c_b positions of
# each sequence are that step's new tokens, plus their queries.
# ---------------------------------------------------------------------------

@dataclass
class PrefillWorkload:
    cache: DecodeWorkload        # k_fill / v_fill hold every position (new tokens included)
    chunk_lens: np.ndarray       # int32 [B]: new tokens per sequence (<= context length)
    cu_q: np.ndarray             # int32 [B + 1]
    q: torch.Tensor              # [sum(chunk_lens), Hq, D], sequence-major


def make_prefill_workload(name, q_heads, kv_heads, head_dim, block_size, dtype, lens, chunks,
                          seed=0, device="cpu"):
    cache = make_decode_workload(name, len(lens), q_heads, kv_heads, head_dim, block_size,
                                 dtype, dtype, lens, seed=seed, device=device)
    chunks = np.asarray(chunks, dtype=np.int32)
    cu = np.concatenate([[0], np.cumsum(chunks)]).astype(np.int32)
    gen = torch.Generator(device=device).manual_seed(seed + 7919)
    q = torch.randn(int(cu[-1]), q_heads, head_dim, generator=gen, device=device,
                    dtype=torch.float32).to(_TORCH_DT[dtype])
    return PrefillWorkload(cache, chunks, cu, q)


def prefill70b(device="cpu", seed=0, batch=8, prefix=1536, chunk=512):
    """LLaMA-70B-shaped GQA layer (64/8 heads, D 128, bf16, bs 16): `batch`
    requests each prefilling a `chunk`-token piece of the prompt behind a
    `prefix`-token cached prefix (chunked prefill after a prefix-cache hit)."""
    lens = [prefix + chunk] * batch
    return make_prefill_workload("prefill70b", 64, 8, 128, 16, "bf16", lens, [chunk] * batch,
                                 seed=seed, device=device)
