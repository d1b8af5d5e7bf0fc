"""KV memory arithmetic from the pages.

Test infrastructure only (see ``oracle/__init__``).

* One layer's KV cache = 2 x kv_heads x seq_len x head_dim x dtype_bytes, the 2 for
  K and V; the whole model = that x num_layers
  [KV Cache 原理与 PagedAttention, §一 "显存占用公式";
  bjdmk.com.cn/news/6246348, §2.2 gives the same per-token product].
* Paging cuts the cache into fixed-size blocks (16 tokens by default, 16-32
  typical) [KV Cache 原理与 PagedAttention, §三 "工作方式" 1;
  aiworkagent.org q17, "Block Size"]; a sequence then wastes only the unused
  tail of its last block, under one block (at most 15 tokens for 16)
  [KV Cache 原理与 PagedAttention, §三 收益 table, 内部碎片 row;
  bjdmk.com.cn/news/6246348, §3.1].
"""


def kv_cache_bytes(num_layers, kv_heads, head_dim, dtype_bytes, seq_len):
    """2 * layers * kv_heads * head_dim * bytes * seq_len."""
    return 2 * num_layers * kv_heads * head_dim * dtype_bytes * seq_len


def blocks_for(seq_len, block_size):
    """Number of fixed-size blocks a sequence of seq_len tokens occupies."""
    return -(-int(seq_len) // int(block_size))


def internal_waste_tokens(seq_len, block_size):
    """Unused token slots in the sequence's last block."""
    return blocks_for(seq_len, block_size) * block_size - int(seq_len)


def scale_bytes(num_layers, kv_heads, dtype_scale_bytes, seq_len):
    """Per-token-head scales of a quantized cache: one fp32 each for K and V."""
    return 2 * num_layers * kv_heads * dtype_scale_bytes * seq_len
