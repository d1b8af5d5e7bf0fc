"""ctypes binding of libpagedkv.so (the C ABI declared in include/pagedkv.h).

Argument marshalling only: every computation runs in the library's CUDA
kernels. torch supplies device memory and the current stream. Importing this
module raises ImportError when the compiled library is missing; there is no
fallback path.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpagedkv.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        "libpagedkv.so is not built (expected at %s); run "
        "`python -m paged_kv_cache_440_b200.build`" % LIB_PATH)

lib = ctypes.CDLL(LIB_PATH)

# ----------------------------------------------------------------- constants
KV_OK, KV_ERR_INVALID, KV_ERR_OOM, KV_ERR_CUDA, KV_ERR_UNSUPPORTED = 0, 1, 2, 3, 4
KV_BF16, KV_FP16, KV_FP8_E5M2, KV_INT8, KV_FP8_E5M2_CAST, KV_INT4 = 0, 1, 2, 3, 4, 5
KV_INT8_KCHAN = 6
KV_DEVERR_BLOCK_ID, KV_DEVERR_CONTEXT, KV_DEVERR_SLOT, KV_DEVERR_TIMEOUT = 1, 2, 4, 8

DTYPE_CODES = {"bf16": KV_BF16, "fp16": KV_FP16, "e5m2": KV_FP8_E5M2, "int8": KV_INT8,
               "e5m2_cast": KV_FP8_E5M2_CAST, "int4": KV_INT4, "int8_kchan": KV_INT8_KCHAN}
TORCH_CODES = {torch.bfloat16: KV_BF16, torch.float16: KV_FP16}
CACHE_TORCH = {"bf16": torch.bfloat16, "fp16": torch.float16, "e5m2": torch.uint8,
               "int8": torch.int8, "e5m2_cast": torch.uint8, "int4": torch.uint8,
               "int8_kchan": torch.int8}


def code_row(kind, head_dim):
    """Stored elements of one (token, head) row: INT4 packs two codes per byte."""
    return head_dim // 2 if kind == "int4" else head_dim


class PoolDesc(ctypes.Structure):
    _fields_ = [("num_layers", ctypes.c_int32), ("num_blocks", ctypes.c_int32),
                ("block_size", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("cache_dtype", ctypes.c_int32)]


_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_I64 = ctypes.c_int64
_U64 = ctypes.c_uint64
_PI32 = ctypes.POINTER(ctypes.c_int32)
_PU64 = ctypes.POINTER(ctypes.c_uint64)
_F = ctypes.c_float

class PrefixCacheStats(ctypes.Structure):
    _fields_ = [("nodes", ctypes.c_int64), ("cached_blocks", ctypes.c_int64),
                ("lookups", ctypes.c_int64), ("hits", ctypes.c_int64),
                ("hit_tokens", ctypes.c_int64)]


_PI32 = ctypes.POINTER(ctypes.c_int32)

_SIGS = {
    "paged_attn_prefill": [_P, _I32, _P, _I32, _I32, _I32, _P, _I32, _I32, _P, _I32, _P, _I32,
                           _F, _P, _P],
    "kv_prefix_cache_create": [_P, ctypes.POINTER(_P)],
    "kv_prefix_cache_destroy": [_P],
    "kv_prefix_match": [_P, _PI32, _I32, _I32, _PI32, _PI32, _PI32],
    "kv_prefix_insert": [_P, _PI32, _I32, _PI32, _I32, _PI32],
    "kv_prefix_evict": [_P, _I32, _PI32, _PI32],
    "kv_prefix_clear": [_P],
    "kv_prefix_stats": [_P, ctypes.POINTER(PrefixCacheStats)],
    "kv_pool_required_bytes": [ctypes.POINTER(PoolDesc), _PU64],
    "kv_pool_create": [ctypes.POINTER(PoolDesc), _P, _U64, ctypes.POINTER(_P)],
    "kv_pool_destroy": [_P],
    "kv_pool_layer_ptrs": [_P, _I32, ctypes.POINTER(_P), ctypes.POINTER(_P),
                           ctypes.POINTER(_P), ctypes.POINTER(_P)],
    "kv_pool_status_ptr": [_P, ctypes.POINTER(_P)],
    "kv_pool_status_clear": [_P, _P],
    "kv_pool_status": [_P, _P, _PI32],
    "kv_alloc_blocks": [_P, _I32, _PI32],
    "kv_free_blocks": [_P, _I32, _PI32],
    "kv_share_blocks": [_P, _I32, _PI32],
    "kv_cow_prepare": [_P, _I32, _PI32],
    "kv_block_refcount": [_P, _I32, _PI32],
    "kv_pool_stats": [_P, _PI32, _PI32, _PI32],
    "kv_append": [_P, _I32, _P, _P, _I32, _P, _I32, _P],
    "kv_quantize": [_P, _I32, _I64, _I32, _I32, _P, _P, _P],
    "kv_block_copy": [_P, _PI32, _I32, _P],
    "paged_attn_workspace_bytes": [_P, _I32, _I32, _I32, _PU64],
    "paged_attn_default_ctas": [_P, _PI32],
    "paged_attn_decode": [_P, _I32, _P, _I32, _I32, _I32, _P, _I32, _P, _I32, _F, _P, _I32,
                          _P, _U64, _P],
    "paged_attn_partition": [_P, _I32, _P, _I32, _I32, _I32, _P, _I32, _P, _I32, _F, _P,
                             _I32, _P, _U64, _P],
    "paged_attn_decode_append": [_P, _I32, _P, _P, _P, _I32, _I32, _I32, _P, _I32, _P, _I32, _F,
                                 _P, _I32, _P, _U64, _P],
    "paged_attn_partition_append": [_P, _I32, _P, _P, _P, _I32, _I32, _I32, _P, _I32, _P, _I32,
                                    _F, _P, _I32, _P, _U64, _P],
    "paged_attn_merge": [_P, _I32, _I32, _P, _I32, _I32, _I32, _I32, _P, _P, _U64, _P],
    "paged_attn_decode_cascade": [_P, _I32, _P, _P, _P, _I32, _I32, _I32, _P, _I32, _P, _I32,
                                  _I32, _F, _P, _I32, _P, _U64, _P],
    "paged_attn_cascade_workspace_bytes": [_P, _I32, _I32, _I32, _PU64],
    "kv_selftest_wait_timeout": [_P, ctypes.c_uint32, _P],
    "paged_attn_decode_static": [_P, _I32, _P, _I32, _I32, _I32, _P, _I32, _P, _I32, _F, _P,
                                 _I32, _P],
}
for _name, _args in _SIGS.items():
    _fn = getattr(lib, _name)
    _fn.argtypes = _args
    _fn.restype = ctypes.c_int
lib.kv_last_error.argtypes = []
lib.kv_last_error.restype = ctypes.c_char_p
lib.kv_version.argtypes = []
lib.kv_version.restype = ctypes.c_char_p


class PagedKVError(RuntimeError):
    def __init__(self, status, message):
        super().__init__("pagedkv status %d: %s" % (status, message))
        self.status = status


def check(status):
    if status != KV_OK:
        raise PagedKVError(status, lib.kv_last_error().decode(errors="replace"))


def _stream(stream=None, device=None):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _need(t, name, dtype=None, device=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch.Tensor" % name)
    if not t.is_cuda:
        raise ValueError("%s must be on a CUDA device" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if dtype is not None and t.dtype not in (dtype if isinstance(dtype, tuple) else (dtype,)):
        raise ValueError("%s has dtype %s, expected %s" % (name, t.dtype, dtype))
    if device is not None and t.device != device:
        raise ValueError("%s is on %s, expected %s" % (name, t.device, device))


def required_bytes(num_layers, num_blocks, block_size, num_kv_heads, head_dim, cache_dtype):
    d = PoolDesc(num_layers, num_blocks, block_size, num_kv_heads, head_dim,
                 DTYPE_CODES[cache_dtype])
    n = ctypes.c_uint64()
    check(lib.kv_pool_required_bytes(ctypes.byref(d), ctypes.byref(n)))
    return n.value


class KVPool:
    """A block pool over one torch-allocated device buffer (held by this object)."""

    def __init__(self, num_layers, num_blocks, block_size, num_kv_heads, head_dim,
                 cache_dtype="bf16", device="cuda"):
        self.desc = PoolDesc(num_layers, num_blocks, block_size, num_kv_heads, head_dim,
                             DTYPE_CODES[cache_dtype])
        self.cache_dtype = cache_dtype
        self.device = torch.device(device)
        nbytes = required_bytes(num_layers, num_blocks, block_size, num_kv_heads, head_dim,
                                cache_dtype)
        self.buffer = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
        h = ctypes.c_void_p()
        check(lib.kv_pool_create(ctypes.byref(self.desc), _ptr(self.buffer), nbytes,
                                 ctypes.byref(h)))
        self.handle = h
        self.status_clear()

    # geometry
    num_layers = property(lambda s: s.desc.num_layers)
    num_blocks = property(lambda s: s.desc.num_blocks)
    block_size = property(lambda s: s.desc.block_size)
    num_kv_heads = property(lambda s: s.desc.num_kv_heads)
    head_dim = property(lambda s: s.desc.head_dim)
    quantized = property(lambda s: s.cache_dtype in ("int8", "e5m2", "e5m2_cast", "int4",
                                                     "int8_kchan"))

    def close(self):
        if getattr(self, "handle", None):
            lib.kv_pool_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def layer_ptrs(self, layer):
        k, v, ks, vs = (ctypes.c_void_p() for _ in range(4))
        check(lib.kv_pool_layer_ptrs(self.handle, layer, ctypes.byref(k), ctypes.byref(v),
                                     ctypes.byref(ks), ctypes.byref(vs)))
        return k.value, v.value, ks.value, vs.value

    def _view(self, addr, nbytes, dtype, shape):
        off = addr - self.buffer.data_ptr()
        return self.buffer[off:off + nbytes].view(dtype).view(shape)

    def layer_views(self, layer):
        """(K, V, K_scale, V_scale) torch views of one layer's regions.

        For "int8_kchan" pools K_scale is the layer's [kv_heads, head_dim]
        channel-scale array, which the caller fills before appending."""
        k, v, ks, vs = self.layer_ptrs(layer)
        row = code_row(self.cache_dtype, self.head_dim)   # elements per (token, head) row
        shape = (self.num_blocks, self.num_kv_heads, self.block_size, row)
        dt = CACHE_TORCH[self.cache_dtype]
        elt = 2 if self.cache_dtype in ("bf16", "fp16") else 1
        n = self.num_blocks * self.num_kv_heads * self.block_size
        K = self._view(k, n * row * elt, dt, shape)
        V = self._view(v, n * row * elt, dt, shape)
        if ks is None:
            return K, V, None, None
        sshape = shape[:3]
        if self.cache_dtype == "int8_kchan":
            KS = self._view(ks, self.num_kv_heads * self.head_dim * 4, torch.float32,
                            (self.num_kv_heads, self.head_dim))
        else:
            KS = self._view(ks, n * 4, torch.float32, sshape)
        return K, V, KS, self._view(vs, n * 4, torch.float32, sshape)

    # status word
    def status_clear(self, stream=None):
        check(lib.kv_pool_status_clear(self.handle, _stream(stream, self.device)))

    def status(self, stream=None):
        v = ctypes.c_int32()
        check(lib.kv_pool_status(self.handle, _stream(stream, self.device), ctypes.byref(v)))
        return v.value

    # allocator
    def alloc(self, n):
        ids = (ctypes.c_int32 * max(n, 1))()
        check(lib.kv_alloc_blocks(self.handle, n, ids))
        return list(ids[:n])

    def free(self, ids):
        arr = (ctypes.c_int32 * max(len(ids), 1))(*ids)
        check(lib.kv_free_blocks(self.handle, len(ids), arr))

    def share(self, ids):
        arr = (ctypes.c_int32 * max(len(ids), 1))(*ids)
        check(lib.kv_share_blocks(self.handle, len(ids), arr))

    def cow_prepare(self, block):
        out = ctypes.c_int32()
        check(lib.kv_cow_prepare(self.handle, block, ctypes.byref(out)))
        return out.value

    def refcount(self, block):
        out = ctypes.c_int32()
        check(lib.kv_block_refcount(self.handle, block, ctypes.byref(out)))
        return out.value

    def stats(self):
        u, f, s = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
        check(lib.kv_pool_stats(self.handle, ctypes.byref(u), ctypes.byref(f), ctypes.byref(s)))
        return {"used": u.value, "free": f.value, "shared": s.value}


class PrefixCache:
    """Host-side prefix cache over a pool's blocks (C ABI kv_prefix_*): a radix
    tree of token sequences with longest-prefix match and LRU leaf eviction."""

    def __init__(self, pool):
        self.pool = pool
        h = ctypes.c_void_p()
        check(lib.kv_prefix_cache_create(pool.handle, ctypes.byref(h)))
        self.handle = h

    @staticmethod
    def _arr(xs):
        xs = list(xs)
        return (ctypes.c_int32 * max(len(xs), 1))(*xs), len(xs)

    def match(self, tokens):
        """(block ids, matched tokens); the caller owns one reference per id."""
        arr, n = self._arr(tokens)
        cap = max(-(-n // self.pool.block_size), 1)
        out = (ctypes.c_int32 * cap)()
        nb, mt = ctypes.c_int32(), ctypes.c_int32()
        check(lib.kv_prefix_match(self.handle, arr, n, cap, out, ctypes.byref(nb),
                                  ctypes.byref(mt)))
        return list(out[:nb.value]), mt.value

    def insert(self, tokens, block_ids):
        arr, n = self._arr(tokens)
        ids, nb = self._arr(block_ids)
        new = ctypes.c_int32()
        check(lib.kv_prefix_insert(self.handle, arr, n, ids, nb, ctypes.byref(new)))
        return new.value

    def evict(self, want):
        out = (ctypes.c_int32 * max(want, 1))()
        k = ctypes.c_int32()
        check(lib.kv_prefix_evict(self.handle, want, out, ctypes.byref(k)))
        return list(out[:k.value])

    def clear(self):
        check(lib.kv_prefix_clear(self.handle))

    def stats(self):
        st = PrefixCacheStats()
        check(lib.kv_prefix_stats(self.handle, ctypes.byref(st)))
        return {f: getattr(st, f) for f, _ in PrefixCacheStats._fields_}

    def close(self):
        if getattr(self, "handle", None):
            lib.kv_prefix_cache_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


# ------------------------------------------------------------------ ops

def kv_append(pool, layer, k_new, v_new, slot_mapping, stream=None):
    """Write k_new/v_new [T, Hkv, D] rows to their slots (int64 [T])."""
    _need(k_new, "k_new", (torch.bfloat16, torch.float16), pool.device)
    _need(v_new, "v_new", k_new.dtype, pool.device)
    _need(slot_mapping, "slot_mapping", torch.int64, pool.device)
    T = k_new.shape[0]
    if tuple(k_new.shape) != (T, pool.num_kv_heads, pool.head_dim) or v_new.shape != k_new.shape \
            or slot_mapping.shape != (T,):
        raise ValueError("k_new, v_new must be [T, kv_heads, head_dim], slot_mapping [T]")
    check(lib.kv_append(pool.handle, layer, _ptr(k_new), _ptr(v_new), TORCH_CODES[k_new.dtype],
                        _ptr(slot_mapping), T, _stream(stream, pool.device)))


def kv_quantize(x, kind, codes=None, scales=None, stream=None):
    """Per-row absmax quantization of x [..., D] -> (codes [..., D], fp32 scales [...])."""
    _need(x, "x", (torch.bfloat16, torch.float16))
    D = x.shape[-1]
    rows = x.numel() // D if D else 0
    if codes is None:
        codes = torch.empty(x.shape[:-1] + (code_row(kind, D),), dtype=CACHE_TORCH[kind],
                            device=x.device)
    if scales is None:
        scales = torch.empty(x.shape[:-1], dtype=torch.float32, device=x.device)
    _need(codes, "codes", CACHE_TORCH[kind], x.device)
    _need(scales, "scales", torch.float32, x.device)
    check(lib.kv_quantize(_ptr(x), TORCH_CODES[x.dtype], rows, D, DTYPE_CODES[kind],
                          _ptr(codes), _ptr(scales), _stream(stream, x.device)))
    return codes, scales


def kv_block_copy(pool, pairs, stream=None):
    """Copy whole blocks src -> dst (all layers). pairs: iterable of (src, dst)."""
    flat = [int(v) for pr in pairs for v in pr]
    n = len(flat) // 2
    arr = (ctypes.c_int32 * max(len(flat), 1))(*flat)
    check(lib.kv_block_copy(pool.handle, arr, n, _stream(stream, pool.device)))


def workspace_bytes(pool, num_seqs, num_q_heads, num_ctas=0):
    n = ctypes.c_uint64()
    check(lib.paged_attn_workspace_bytes(pool.handle, num_seqs, num_q_heads, num_ctas,
                                         ctypes.byref(n)))
    return n.value


def default_ctas(pool):
    n = ctypes.c_int32()
    check(lib.paged_attn_default_ctas(pool.handle, ctypes.byref(n)))
    return n.value


def make_workspace(pool, num_seqs, num_q_heads, num_ctas=0):
    n = workspace_bytes(pool, num_seqs, num_q_heads, num_ctas)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=pool.device)


def _attn_args(pool, q, block_tables, context_lens, out):
    _need(q, "q", (torch.bfloat16, torch.float16), pool.device)
    _need(block_tables, "block_tables", torch.int32, pool.device)
    _need(context_lens, "context_lens", torch.int32, pool.device)
    B, Hq, D = q.shape
    if D != pool.head_dim or block_tables.dim() != 2 or block_tables.shape[0] != B \
            or context_lens.shape != (B,):
        raise ValueError("q [B, Hq, D], block_tables [B, max_blocks], context_lens [B]")
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", q.dtype, pool.device)
    if out.shape != q.shape:
        raise ValueError("out must have q's shape")
    return B, Hq, out


def paged_attn_decode(pool, layer, q, block_tables, context_lens, max_context, scale,
                      out=None, num_ctas=0, workspace=None, stream=None):
    """Decode attention of q [B, Hq, D] over the paged cache; returns out."""
    B, Hq, out = _attn_args(pool, q, block_tables, context_lens, out)
    if workspace is None:
        workspace = make_workspace(pool, B, Hq, num_ctas)
    check(lib.paged_attn_decode(pool.handle, layer, _ptr(q), TORCH_CODES[q.dtype], B, Hq,
                                _ptr(block_tables), block_tables.shape[1], _ptr(context_lens),
                                max_context, float(scale), _ptr(out), num_ctas,
                                _ptr(workspace), workspace.numel(), _stream(stream, pool.device)))
    return out


def paged_attn_decode_static(pool, layer, q, block_tables, context_lens, max_context, scale,
                             out=None, num_ctas=0, stream=None):
    """paged_attn_decode without a workspace argument: the library's built-in
    16 MiB scratch is used instead (see include/pagedkv.h). For callers that
    cannot allocate device memory; calls must not overlap on the GPU."""
    B, Hq, out = _attn_args(pool, q, block_tables, context_lens, out)
    check(lib.paged_attn_decode_static(pool.handle, layer, _ptr(q), TORCH_CODES[q.dtype], B, Hq,
                                       _ptr(block_tables), block_tables.shape[1],
                                       _ptr(context_lens), max_context, float(scale), _ptr(out),
                                       num_ctas, _stream(stream, pool.device)))
    return out


def paged_attn_decode_append(pool, layer, q, k_new, v_new, block_tables, context_lens,
                             max_context, scale, out=None, num_ctas=0, workspace=None,
                             stream=None):
    """Write each sequence's new token (k_new, v_new [B, Hkv, D]) at position
    L - 1 and attend q over the cache including it, in one attention kernel."""
    B, Hq, out = _attn_args(pool, q, block_tables, context_lens, out)
    _need(k_new, "k_new", q.dtype, pool.device)
    _need(v_new, "v_new", q.dtype, pool.device)
    if tuple(k_new.shape) != (B, pool.num_kv_heads, pool.head_dim) or v_new.shape != k_new.shape:
        raise ValueError("k_new, v_new must be [B, kv_heads, head_dim]")
    if workspace is None:
        workspace = make_workspace(pool, B, Hq, num_ctas)
    check(lib.paged_attn_decode_append(pool.handle, layer, _ptr(q), _ptr(k_new), _ptr(v_new),
                                       TORCH_CODES[q.dtype], B, Hq, _ptr(block_tables),
                                       block_tables.shape[1], _ptr(context_lens), max_context,
                                       float(scale), _ptr(out), num_ctas, _ptr(workspace),
                                       workspace.numel(), _stream(stream, pool.device)))
    return out


def cascade_workspace_bytes(pool, num_seqs, num_q_heads, num_ctas=0):
    n = ctypes.c_uint64()
    check(lib.paged_attn_cascade_workspace_bytes(pool.handle, num_seqs, num_q_heads, num_ctas,
                                                 ctypes.byref(n)))
    return n.value


def make_cascade_workspace(pool, num_seqs, num_q_heads, num_ctas=0):
    n = cascade_workspace_bytes(pool, num_seqs, num_q_heads, num_ctas)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=pool.device)


def paged_attn_decode_cascade(pool, layer, q, block_tables, context_lens, max_context,
                              prefix_blocks, scale, k_new=None, v_new=None, out=None,
                              num_ctas=0, workspace=None, stream=None):
    """Decode step for sequences whose block tables begin with the same
    prefix_blocks shared blocks: the prefix once for all of them on the tensor
    cores, each sequence's remaining positions (with the new token's append
    when k_new, v_new [B, Hkv, D] are given) through the decode kernel, then
    the merge. Returns out."""
    B, Hq, out = _attn_args(pool, q, block_tables, context_lens, out)
    if (k_new is None) != (v_new is None):
        raise ValueError("k_new and v_new go together")
    if k_new is not None:
        _need(k_new, "k_new", q.dtype, pool.device)
        _need(v_new, "v_new", q.dtype, pool.device)
        if tuple(k_new.shape) != (B, pool.num_kv_heads, pool.head_dim) or v_new.shape != k_new.shape:
            raise ValueError("k_new, v_new must be [B, kv_heads, head_dim]")
    if workspace is None:
        workspace = make_cascade_workspace(pool, B, Hq, num_ctas)
    kn = None if k_new is None else _ptr(k_new)
    vn = None if v_new is None else _ptr(v_new)
    check(lib.paged_attn_decode_cascade(pool.handle, layer, _ptr(q), kn, vn,
                                        TORCH_CODES[q.dtype], B, Hq, _ptr(block_tables),
                                        block_tables.shape[1], _ptr(context_lens), max_context,
                                        prefix_blocks, float(scale), _ptr(out), num_ctas,
                                        _ptr(workspace), workspace.numel(),
                                        _stream(stream, pool.device)))
    return out


def paged_attn_partition(pool, layer, q, block_tables, context_lens, max_context, scale,
                         out, workspace, num_ctas=0, stream=None):
    B, Hq, out = _attn_args(pool, q, block_tables, context_lens, out)
    check(lib.paged_attn_partition(pool.handle, layer, _ptr(q), TORCH_CODES[q.dtype], B, Hq,
                                   _ptr(block_tables), block_tables.shape[1],
                                   _ptr(context_lens), max_context, float(scale), _ptr(out),
                                   num_ctas, _ptr(workspace), workspace.numel(),
                                   _stream(stream, pool.device)))
    return out


def paged_attn_prefill(pool, layer, q, cu_q_lens, max_q_len, block_tables, context_lens,
                       max_context, scale, out=None, stream=None):
    """Chunked prefill: q [T, Hq, D] (sequence-major rows, cu_q_lens [B+1]
    int32 on the device); each new token attends to the positions up to its
    own. The new tokens' K/V must already be in the pool."""
    _need(q, "q", (torch.bfloat16, torch.float16), pool.device)
    _need(cu_q_lens, "cu_q_lens", torch.int32, pool.device)
    _need(block_tables, "block_tables", torch.int32, pool.device)
    _need(context_lens, "context_lens", torch.int32, pool.device)
    T, Hq, D = q.shape
    B = context_lens.shape[0]
    if cu_q_lens.shape[0] != B + 1 or block_tables.shape[0] != B:
        raise ValueError("cu_q_lens must be [B+1] and block_tables [B, max_blocks]")
    if out is None:
        out = torch.empty_like(q)
    check(lib.paged_attn_prefill(pool.handle, layer, _ptr(q), TORCH_CODES[q.dtype], B, Hq,
                                 _ptr(cu_q_lens), T, max_q_len, _ptr(block_tables),
                                 block_tables.shape[1], _ptr(context_lens), max_context,
                                 float(scale), _ptr(out), _stream(stream, pool.device)))
    return out


def paged_attn_partition_append(pool, layer, q, k_new, v_new, block_tables, context_lens,
                                max_context, scale, out, workspace, num_ctas=0, stream=None):
    B, Hq, out = _attn_args(pool, q, block_tables, context_lens, out)
    _need(k_new, "k_new", q.dtype, pool.device)
    _need(v_new, "v_new", q.dtype, pool.device)
    if tuple(k_new.shape) != (B, pool.num_kv_heads, pool.head_dim) or v_new.shape != k_new.shape:
        raise ValueError("k_new, v_new must be [B, kv_heads, head_dim]")
    check(lib.paged_attn_partition_append(pool.handle, layer, _ptr(q), _ptr(k_new), _ptr(v_new),
                                          TORCH_CODES[q.dtype], B, Hq, _ptr(block_tables),
                                          block_tables.shape[1], _ptr(context_lens), max_context,
                                          float(scale), _ptr(out), num_ctas, _ptr(workspace),
                                          workspace.numel(), _stream(stream, pool.device)))
    return out


def paged_attn_merge(pool, context_lens, max_blocks_per_seq, max_context, out, workspace,
                     num_ctas=0, stream=None):
    _need(out, "out", (torch.bfloat16, torch.float16), pool.device)
    _need(context_lens, "context_lens", torch.int32, pool.device)
    B, Hq, _ = out.shape
    check(lib.paged_attn_merge(pool.handle, B, Hq, _ptr(context_lens), max_blocks_per_seq,
                               max_context, num_ctas, TORCH_CODES[out.dtype], _ptr(out),
                               _ptr(workspace), workspace.numel(),
                               _stream(stream, pool.device)))
    return out


def selftest_wait_timeout(status, limit_us=1000, stream=None):
    """Run the bounded-wait self-test; status is a device int32 tensor [1]."""
    _need(status, "status", torch.int32)
    check(lib.kv_selftest_wait_timeout(_ptr(status), limit_us, _stream(stream, status.device)))


def version():
    return lib.kv_version().decode()
