"""Paged KV-cache decode attention for NVIDIA B200 (sm_100a).

Python binding of libpagedkv.so.  The functions keep the C ABI's names
(``pa_decode``, ``pa_cache_write``, ``pa_copy_blocks``, ``pa_bm_*``) and only
marshal arguments: they take torch tensors for device memory and streams,
check dtypes / devices / contiguity, and pass raw pointers to the library.
All computation happens in the library's CUDA kernels and C++ block manager;
if the library is missing, every call raises.

Layouts (see include/pagedkv.h for the full contract):
  q, out            [num_seqs, num_q_heads, head_dim]            fp16 / bf16
                    (out may be float32: the value before the final rounding)
  k_cache, v_cache  [num_blocks, num_kv_heads, block_size, head_dim]
  block_tables      [num_seqs, max_blocks_per_seq] int32
  context_lens      [num_seqs] int32
  k, v (new tokens) [num_tokens, num_kv_heads, head_dim]
  slot_mapping      [num_tokens] int64
  pairs             [num_pairs, 2] int32
"""
from __future__ import annotations

import ctypes

from . import _lib
from ._lib import (PA_BF16, PA_F16, PA_KERNEL_AUTO, PA_KERNEL_MMA,
                   PA_KERNEL_SIMT, PagedKVError, NoFreeBlocksError,
                   pa_decode_desc)

__all__ = [
    "pa_decode", "pa_decode_noalloc", "pa_prefill", "pa_prefill_workspace_bytes",
    "pa_cache_write",
    "pa_copy_blocks",
    "pa_decode_workspace_bytes", "pa_decode_partition_size", "make_desc",
    "BlockManager", "PagedKVError", "NoFreeBlocksError", "library_path",
    "pa_launch_count", "pa_read_probe", "pa_wait_probe",
    "PA_KERNEL_AUTO", "PA_KERNEL_MMA", "PA_KERNEL_SIMT",
]

_KERNELS = {"auto": PA_KERNEL_AUTO, "mma": PA_KERNEL_MMA,
            "simt": PA_KERNEL_SIMT}
_REDUCES = {"auto": _lib.PA_REDUCE_AUTO, "kernel": _lib.PA_REDUCE_KERNEL}
_PREFILL_KERNELS = {"auto": _lib.PA_PREFILL_AUTO, "tile": _lib.PA_PREFILL_TILE}
_PREFILL_PV = {"auto": _lib.PA_PV_AUTO, "split": _lib.PA_PV_SPLIT,
               "single": _lib.PA_PV_SINGLE}


def library_path() -> str:
    return _lib.LIB_PATH


def pa_read_probe(buf, sink, stream=None):
    """Read the whole CUDA tensor ``buf`` once with streaming loads (a
    bandwidth measurement helper); ``sink`` is an int32 CUDA tensor."""
    import torch
    st = _lib.load().pa_read_probe(
        _dev(buf, "buf"), buf.numel() * buf.element_size(),
        _dev(sink, "sink", torch.int32), _stream(stream))
    _lib.check(st, "pa_read_probe")


def pa_wait_probe(dev_err, stream=None):
    """Make one bounded device wait run out (about 1 s of device time): the
    kernel sets ``dev_err`` (an int32 CUDA tensor) to PA_ERR_DEVICE_TIMEOUT,
    frees its tensor memory and returns, as the attention kernels do when a
    copy never lands."""
    import torch
    if dev_err is None:
        raise ValueError("pa_wait_probe needs a dev_err tensor")
    st = _lib.load().pa_wait_probe(_dev(dev_err, "dev_err", torch.int32),
                                   _stream(stream))
    _lib.check(st, "pa_wait_probe")


def pa_launch_count() -> int:
    """Kernel launches libpagedkv has issued in this process."""
    return int(_lib.load().pa_launch_count())


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.float16:
        return PA_F16
    if t.dtype == torch.bfloat16:
        return PA_BF16
    raise TypeError(f"expected float16 or bfloat16, got {t.dtype}")


def _dev(t, name: str, dtype=None):
    """Pointer of a contiguous CUDA tensor (None -> NULL)."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return t.data_ptr()


def _stream(stream) -> int:
    import torch
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def make_desc(q, k_cache, block_tables, *, partition_size: int = 0,
              max_context_len: int = 0, kernel: str = "auto",
              reduce: str = "auto") -> pa_decode_desc:
    """Decode descriptor from tensor shapes."""
    num_seqs, num_q_heads, head_dim = q.shape
    num_blocks, num_kv_heads, block_size, hd2 = k_cache.shape
    if hd2 != head_dim:
        raise ValueError("q and k_cache disagree on head_dim")
    if block_tables.shape[0] != num_seqs:
        raise ValueError("block_tables rows != num_seqs")
    return pa_decode_desc(
        num_seqs=num_seqs, num_q_heads=num_q_heads, num_kv_heads=num_kv_heads,
        head_dim=head_dim, block_size=block_size,
        max_blocks_per_seq=block_tables.shape[1], num_blocks=num_blocks,
        dtype=_dtype_code(q), partition_size=partition_size,
        max_context_len=max_context_len, kernel=_KERNELS[kernel],
        reduce=_REDUCES[reduce])


def _out_mode(desc, out, dt):
    """``out`` in q's dtype, or float32: the value before the final rounding
    (desc.out_fp32 follows the tensor)."""
    import torch
    if out.dtype == dt:
        desc.out_fp32 = 0
    elif out.dtype == torch.float32:
        desc.out_fp32 = 1
    else:
        raise TypeError(f"out dtype {out.dtype} is neither q's dtype {dt} "
                        "nor float32")


def pa_decode_workspace_bytes(desc: pa_decode_desc) -> int:
    return int(_lib.load().pa_decode_workspace_bytes(ctypes.byref(desc)))


def pa_decode_partition_size(desc: pa_decode_desc) -> int:
    ps = _lib.load().pa_decode_partition_size(ctypes.byref(desc))
    if ps < 0:
        _lib.check(_lib.PA_ERR_INVALID_ARG, "pa_decode_partition_size")
    return ps


def pa_decode(out, q, k_cache, v_cache, block_tables, context_lens,
              scale: float, *, partition_size: int = 0,
              max_context_len: int = 0, kernel: str = "auto",
              reduce: str = "auto", workspace=None, dev_err=None,
              stream=None, desc: pa_decode_desc | None = None):
    """out[b, h] = softmax(scale * K_b q[b, h]) V_b over each sequence's
    paged K/V.  ``workspace`` (uint8 CUDA tensor) is allocated with torch when
    the call needs one and none is given.  Returns ``out``."""
    import torch
    lib = _lib.load()
    if desc is None:
        desc = make_desc(q, k_cache, block_tables,
                         partition_size=partition_size,
                         max_context_len=max_context_len, kernel=kernel,
                         reduce=reduce)
    dt = q.dtype
    for name, t in (("k_cache", k_cache), ("v_cache", v_cache)):
        if t.dtype != dt:
            raise TypeError(f"{name} dtype {t.dtype} != q dtype {dt}")
    _out_mode(desc, out, dt)
    need = int(lib.pa_decode_workspace_bytes(ctypes.byref(desc)))
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr = _dev(workspace, "workspace") if workspace is not None else None
    ws_bytes = workspace.numel() * workspace.element_size() \
        if workspace is not None else 0
    st = lib.pa_decode(
        _dev(out, "out"), _dev(q, "q"), _dev(k_cache, "k_cache"),
        _dev(v_cache, "v_cache"),
        _dev(block_tables, "block_tables", torch.int32),
        _dev(context_lens, "context_lens", torch.int32),
        ctypes.c_float(scale), ctypes.byref(desc), ws_ptr, ws_bytes,
        _dev(dev_err, "dev_err", torch.int32), _stream(stream))
    _lib.check(st, "pa_decode")
    return out


def pa_decode_noalloc(out, q, k_cache, v_cache, block_tables, context_lens,
                      scale: float, *, partition_size: int = 0,
                      max_context_len: int = 0, kernel: str = "auto",
                      reduce: str = "auto", dev_err=None, stream=None,
                      desc: pa_decode_desc | None = None):
    """pa_decode for callers that cannot allocate device memory: the
    workspace is the library's built-in scratch area
    (PA_NOALLOC_SCRATCH_BYTES per device), so this wrapper allocates nothing
    either.  Calls that overlap on one device race on that area.  Returns
    ``out``."""
    import torch
    lib = _lib.load()
    if desc is None:
        desc = make_desc(q, k_cache, block_tables,
                         partition_size=partition_size,
                         max_context_len=max_context_len, kernel=kernel,
                         reduce=reduce)
    for name, t in (("k_cache", k_cache), ("v_cache", v_cache)):
        if t.dtype != q.dtype:
            raise TypeError(f"{name} dtype {t.dtype} != q dtype {q.dtype}")
    _out_mode(desc, out, q.dtype)
    st = lib.pa_decode_noalloc(
        _dev(out, "out"), _dev(q, "q"), _dev(k_cache, "k_cache"),
        _dev(v_cache, "v_cache"),
        _dev(block_tables, "block_tables", torch.int32),
        _dev(context_lens, "context_lens", torch.int32),
        ctypes.c_float(scale), ctypes.byref(desc),
        _dev(dev_err, "dev_err", torch.int32), _stream(stream))
    _lib.check(st, "pa_decode_noalloc")
    return out


def _prefill_desc(q, k_cache, block_tables, max_q_len, max_context_len,
                  kernel="auto", pv="auto"):
    total_q, num_q_heads, head_dim = q.shape
    num_blocks, num_kv_heads, block_size, hd2 = k_cache.shape
    if hd2 != head_dim:
        raise ValueError("q and the caches disagree on head_dim")
    return _lib.pa_prefill_desc(
        num_seqs=block_tables.shape[0], num_q_heads=num_q_heads,
        num_kv_heads=num_kv_heads, head_dim=head_dim, block_size=block_size,
        max_blocks_per_seq=block_tables.shape[1], num_blocks=num_blocks,
        dtype=_dtype_code(q), total_q=total_q, max_q_len=max_q_len,
        max_context_len=max_context_len, kernel=_PREFILL_KERNELS[kernel],
        pv=_PREFILL_PV[pv])


def pa_prefill_workspace_bytes(q, k_cache, block_tables, *,
                               max_q_len: int | None = None) -> int:
    """Bytes of device workspace ``pa_prefill`` needs for these tensors and
    ``max_q_len`` (default: every row of ``q``): the sequence order and the
    tile map (``pa_prefill_workspace_bytes`` of the C ABI)."""
    if max_q_len is None:
        max_q_len = q.shape[0]
    desc = _prefill_desc(q, k_cache, block_tables, max_q_len, 0)
    return int(_lib.load().pa_prefill_workspace_bytes(ctypes.byref(desc)))


def pa_prefill(out, q, k_cache, v_cache, block_tables, context_lens,
               query_start, scale: float, *, max_q_len: int,
               max_context_len: int = 0, kernel: str = "auto",
               pv: str = "auto", workspace=None, dev_err=None, stream=None):
    """Causal attention of each sequence's new tokens (rows
    query_start[b] .. query_start[b+1]-1 of ``q``) over its paged K/V, the
    new tokens being the last ones of the context.  ``max_q_len`` bounds
    every sequence's new-token count (it picks the layout; a sequence above
    it is flagged and left unwritten).  ``kernel``: "auto" or "tile" (the
    same kernel).  ``pv``: precision of P in P . V -- "auto" (P's residual
    added in the tiles that need it), "split" (in every tile) or "single"
    (one rounding of P).  ``workspace`` (a uint8 device tensor of
    ``pa_prefill_workspace_bytes`` bytes) is allocated per call when not
    given.  Returns ``out``."""
    import torch
    lib = _lib.load()
    if out.shape != q.shape:
        raise ValueError("q and out disagree on shape")
    for name, t in (("k_cache", k_cache), ("v_cache", v_cache)):
        if t.dtype != q.dtype:
            raise TypeError(f"{name} dtype {t.dtype} != q dtype {q.dtype}")
    desc = _prefill_desc(q, k_cache, block_tables, max_q_len, max_context_len,
                         kernel, pv)
    _out_mode(desc, out, q.dtype)
    need = lib.pa_prefill_workspace_bytes(ctypes.byref(desc))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8,
                                device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    st = lib.pa_prefill(
        _dev(out, "out"), _dev(q, "q"), _dev(k_cache, "k_cache"),
        _dev(v_cache, "v_cache"),
        _dev(block_tables, "block_tables", torch.int32),
        _dev(context_lens, "context_lens", torch.int32),
        _dev(query_start, "query_start", torch.int32),
        ctypes.c_float(scale), ctypes.byref(desc),
        _dev(workspace, "workspace"), ctypes.c_size_t(ws_bytes),
        _dev(dev_err, "dev_err", torch.int32), _stream(stream))
    _lib.check(st, "pa_prefill")
    return out


def _reachable(t, name: str, dtype=None):
    """Pointer of a contiguous CUDA tensor or pinned (page-locked) CPU
    tensor; the library checks that the device can reach it."""
    if not (t.is_cuda or t.is_pinned()):
        raise ValueError(f"{name} must be a CUDA tensor or pinned CPU memory")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    return t.data_ptr()


def pa_swap_blocks(dst_k, dst_v, src_k, src_v, pairs, *, dev_err=None,
                   stream=None):
    """Copy block pairs[i, 0] of (src_k, src_v) to block pairs[i, 1] of
    (dst_k, dst_v); any of the pools (and ``pairs``) may be pinned CPU
    tensors, e.g. a host pool for swapped-out sequences."""
    import torch
    lib = _lib.load()
    ns, hkv, bs, d = src_k.shape
    nd = dst_k.shape[0]
    for name, t, n in (("dst_k", dst_k, nd), ("dst_v", dst_v, nd),
                       ("src_v", src_v, ns)):
        if t.shape != (n, hkv, bs, d):
            raise ValueError(f"{name} shape {tuple(t.shape)} does not match")
        if t.dtype != src_k.dtype:
            raise TypeError(f"{name} dtype differs from src_k")
    if pairs.ndim != 2 or pairs.shape[1] != 2:
        raise ValueError("pairs must be [n, 2]")
    st = lib.pa_swap_blocks(
        _reachable(dst_k, "dst_k"), _reachable(dst_v, "dst_v"),
        _reachable(src_k, "src_k"), _reachable(src_v, "src_v"),
        _reachable(pairs, "pairs", torch.int32), pairs.shape[0], hkv, d, bs,
        ns, nd, _dtype_code(src_k), _dev(dev_err, "dev_err", torch.int32),
        _stream(stream))
    _lib.check(st, "pa_swap_blocks")


def pa_pool_blocks(nbytes: int, num_layers: int, num_kv_heads: int,
                   head_dim: int, block_size: int, dtype) -> int:
    """Blocks of block_size tokens (K and V of every layer) that fit in
    ``nbytes``; ``dtype`` is torch.float16 or torch.bfloat16."""
    import torch
    code = {torch.float16: PA_F16, torch.bfloat16: PA_BF16}.get(dtype)
    if code is None:
        raise TypeError(f"expected float16 or bfloat16, got {dtype}")
    n = _lib.load().pa_pool_blocks(int(nbytes), num_layers, num_kv_heads,
                                   head_dim, block_size, code)
    if n < 0:
        _lib.check(_lib.PA_ERR_INVALID_ARG, "pa_pool_blocks")
    return n


def pa_cache_write(k_cache, v_cache, k, v, slot_mapping, *, dev_err=None,
                   stream=None):
    """Copy each new token's K and V rows into cache slot slot_mapping[t]
    (negative slots are skipped)."""
    import torch
    lib = _lib.load()
    num_blocks, num_kv_heads, block_size, head_dim = k_cache.shape
    num_tokens = k.shape[0]
    if k.shape != (num_tokens, num_kv_heads, head_dim) or v.shape != k.shape:
        raise ValueError("k, v must be [num_tokens, num_kv_heads, head_dim]")
    if slot_mapping.shape != (num_tokens,):
        raise ValueError("slot_mapping must be [num_tokens]")
    for name, t in (("v_cache", v_cache), ("k", k), ("v", v)):
        if t.dtype != k_cache.dtype:
            raise TypeError(f"{name} dtype {t.dtype} != k_cache dtype")
    st = lib.pa_cache_write(
        _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"), _dev(k, "k"),
        _dev(v, "v"), _dev(slot_mapping, "slot_mapping", torch.int64),
        num_tokens, num_kv_heads, head_dim, block_size, num_blocks,
        _dtype_code(k_cache), _dev(dev_err, "dev_err", torch.int32),
        _stream(stream))
    _lib.check(st, "pa_cache_write")


def pa_copy_blocks(k_cache, v_cache, pairs, *, dev_err=None, stream=None):
    """k_cache[dst] = k_cache[src] and v_cache[dst] = v_cache[src] for every
    (src, dst) row of ``pairs`` (int32 [n, 2] on the device)."""
    import torch
    lib = _lib.load()
    num_blocks, num_kv_heads, block_size, head_dim = k_cache.shape
    if pairs.dim() != 2 or pairs.shape[1] != 2:
        raise ValueError("pairs must be [num_pairs, 2]")
    if v_cache.dtype != k_cache.dtype:
        raise TypeError("k_cache and v_cache dtypes differ")
    st = lib.pa_copy_blocks(
        _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"),
        _dev(pairs, "pairs", torch.int32), pairs.shape[0], num_kv_heads,
        head_dim, block_size, num_blocks, _dtype_code(k_cache),
        _dev(dev_err, "dev_err", torch.int32), _stream(stream))
    _lib.check(st, "pa_copy_blocks")


class BlockManager:
    """Host block manager of libpagedkv (pa_bm_* calls).

    Free pool, per-sequence block tables, reference counts, fork and
    copy-on-write.  Not thread-safe.
    """

    def __init__(self, num_blocks: int, block_size: int, free_order=None):
        self._lib = _lib.load()
        self.num_blocks = num_blocks
        self.block_size = block_size
        handle = ctypes.c_void_p()
        order = None
        if free_order is not None:
            import numpy as np
            arr = np.ascontiguousarray(free_order, dtype=np.int32)
            if arr.shape != (num_blocks,):
                raise ValueError("free_order must have num_blocks entries")
            order = arr.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
        _lib.check(self._lib.pa_bm_create(num_blocks, block_size, order,
                                          ctypes.byref(handle)),
                   "pa_bm_create")
        self._h = handle

    def close(self):
        if self._h:
            self._lib.pa_bm_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def add_seq(self, seq_id: int):
        _lib.check(self._lib.pa_bm_add_seq(self._h, seq_id), "pa_bm_add_seq")

    def fork(self, parent: int, child: int):
        _lib.check(self._lib.pa_bm_fork(self._h, parent, child), "pa_bm_fork")

    def append(self, seq_id: int, n_tokens: int):
        """Returns (slots int64 ndarray [n_tokens], cow_pairs int32 [k, 2])."""
        import numpy as np
        slots = np.empty(max(n_tokens, 0), dtype=np.int64)
        pairs = np.empty(2, dtype=np.int32)
        ncow = ctypes.c_int(0)
        st = self._lib.pa_bm_append(
            self._h, seq_id, n_tokens,
            slots.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
            pairs.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), 1,
            ctypes.byref(ncow))
        _lib.check(st, "pa_bm_append")
        return slots, pairs[: 2 * ncow.value].reshape(-1, 2).copy()

    def append_batch(self, seq_ids, n_tokens, slots_out=None):
        """One call for a whole decode step: appends n_tokens[i] tokens to
        seq_ids[i].  Returns (slots int64 [sum], cow_pairs int32 [k, 2]).
        ``slots_out`` (optional int64 ndarray, e.g. a view of pinned memory)
        receives the slots.  Raises NoFreeBlocksError (with .num_done) if the
        pool runs out."""
        import numpy as np
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        nt = np.ascontiguousarray(n_tokens, dtype=np.int32)
        if nt.shape != ids.shape:
            raise ValueError("seq_ids and n_tokens differ in length")
        total = int(nt.sum())
        if slots_out is not None:
            if (slots_out.dtype != np.int64 or slots_out.shape != (total,)
                    or not slots_out.flags.c_contiguous):
                raise ValueError("slots_out must be contiguous int64 [sum]")
            slots = slots_out
        else:
            slots = np.empty(total, dtype=np.int64)
        pairs = np.empty(2 * max(len(ids), 1), dtype=np.int32)
        ncow, ndone = ctypes.c_int(0), ctypes.c_int(0)
        st = self._lib.pa_bm_append_batch(
            self._h, ids.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
            nt.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), len(ids),
            slots.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
            pairs.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), len(ids),
            ctypes.byref(ncow), ctypes.byref(ndone))
        try:
            _lib.check(st, "pa_bm_append_batch")
        except PagedKVError as e:
            e.num_done = ndone.value
            raise
        return slots, pairs[: 2 * ncow.value].reshape(-1, 2).copy()

    def free_seq(self, seq_id: int):
        _lib.check(self._lib.pa_bm_free_seq(self._h, seq_id), "pa_bm_free_seq")

    def truncate(self, seq_id: int, new_len: int):
        _lib.check(self._lib.pa_bm_truncate(self._h, seq_id, new_len),
                   "pa_bm_truncate")

    def block_table(self, seq_ids, max_blocks: int, table_out=None,
                    lens_out=None):
        """Returns (table int32 [n, max_blocks] padded with -1, lens int32).
        Optional contiguous int32 ``table_out`` / ``lens_out`` arrays receive
        the result in place."""
        import numpy as np
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        table = table_out if table_out is not None else \
            np.empty((len(ids), max_blocks), dtype=np.int32)
        lens = lens_out if lens_out is not None else \
            np.empty(len(ids), dtype=np.int32)
        for arr, shp in ((table, (len(ids), max_blocks)), (lens, (len(ids),))):
            if (arr.dtype != np.int32 or arr.shape != shp
                    or not arr.flags.c_contiguous):
                raise ValueError("block_table outputs: wrong dtype/shape")
        st = self._lib.pa_bm_block_table(
            self._h, ids.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
            len(ids), max_blocks,
            table.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
            lens.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)))
        _lib.check(st, "pa_bm_block_table")
        return table, lens

    def num_free(self) -> int:
        return self._lib.pa_bm_num_free(self._h)

    def num_used(self) -> int:
        return self._lib.pa_bm_num_used(self._h)

    def refcount(self, block: int) -> int:
        return self._lib.pa_bm_refcount(self._h, block)

    def seq_len(self, seq_id: int) -> int:
        return self._lib.pa_bm_seq_len(self._h, seq_id)

    def num_seq_blocks(self, seq_id: int) -> int:
        return self._lib.pa_bm_num_seq_blocks(self._h, seq_id)

    # -- prefix cache -------------------------------------------------------
    def match_prefix(self, seq_id: int, tokens) -> int:
        """Attach the longest cached run of full blocks that starts
        ``tokens`` to the new, empty ``seq_id``; returns the tokens matched
        (only the rest needs a prefill)."""
        import numpy as np
        t = np.ascontiguousarray(tokens, dtype=np.int32)
        out = ctypes.c_int64(0)
        _lib.check(self._lib.pa_bm_match_prefix(
            self._h, seq_id, t.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
            len(t), ctypes.byref(out)), "pa_bm_match_prefix")
        return out.value

    def cache_insert(self, seq_id: int, tokens):
        """Cache the full blocks of the first len(tokens) tokens of
        ``seq_id`` (call once their K/V are written)."""
        import numpy as np
        t = np.ascontiguousarray(tokens, dtype=np.int32)
        _lib.check(self._lib.pa_bm_cache_insert(
            self._h, seq_id, t.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
            len(t)), "pa_bm_cache_insert")

    def cache_evict(self, max_blocks: int) -> int:
        out = ctypes.c_int(0)
        _lib.check(self._lib.pa_bm_cache_evict(self._h, max_blocks,
                                               ctypes.byref(out)),
                   "pa_bm_cache_evict")
        return out.value

    def num_cached(self) -> int:
        return self._lib.pa_bm_num_cached(self._h)

    def cache_nodes(self):
        """The cached tree as (parent_index int32 [n], block int32 [n],
        tokens int32 [n, block_size]), parents before children."""
        import numpy as np
        n = max(self.num_cached(), 0)
        parent = np.empty(max(n, 1), dtype=np.int32)
        block = np.empty(max(n, 1), dtype=np.int32)
        toks = np.empty((max(n, 1), self.block_size), dtype=np.int32)
        got = ctypes.c_int(0)
        p32 = ctypes.POINTER(ctypes.c_int32)
        _lib.check(self._lib.pa_bm_cache_nodes(
            self._h, n, parent.ctypes.data_as(p32), block.ctypes.data_as(p32),
            toks.ctypes.data_as(p32), ctypes.byref(got)), "pa_bm_cache_nodes")
        k = got.value
        return parent[:k], block[:k], toks[:k]

    def cached_paths(self):
        """Every cached block as the tuple of its token keys from the root
        (the same form as the oracle model's ``cached_paths``)."""
        parent, _, toks = self.cache_nodes()
        paths = []
        for i in range(len(parent)):
            key = tuple(int(t) for t in toks[i])
            paths.append((key,) if parent[i] < 0 else paths[parent[i]] + (key,))
        return set(paths)

    # -- swapping to a host pool ------------------------------------------------
    def set_host_blocks(self, num_host_blocks: int):
        _lib.check(self._lib.pa_bm_set_host_blocks(self._h, num_host_blocks),
                   "pa_bm_set_host_blocks")
        self.num_host_blocks = num_host_blocks

    def _swap(self, fn, name, seq_ids, pairs_out):
        import numpy as np
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        cap = sum(max(self.num_seq_blocks(int(s)), 0) for s in ids)
        if pairs_out is None:
            pairs = np.empty((max(cap, 1), 2), dtype=np.int32)
        else:
            if (pairs_out.dtype != np.int32 or pairs_out.ndim != 2
                    or pairs_out.shape[1] != 2
                    or not pairs_out.flags.c_contiguous):
                raise ValueError("pairs_out must be contiguous int32 [k, 2]")
            pairs, cap = pairs_out, pairs_out.shape[0]
        n = ctypes.c_int(0)
        _lib.check(fn(self._h, ids.ctypes.data_as(ctypes.POINTER(
            ctypes.c_int64)), len(ids), pairs.ctypes.data_as(
                ctypes.POINTER(ctypes.c_int32)), cap, ctypes.byref(n)), name)
        return pairs[:n.value]

    def swap_out(self, seq_ids, pairs_out=None):
        """Swap the group out; returns (device, host) block pairs int32
        [k, 2] (a view of ``pairs_out`` if given, e.g. pinned memory)."""
        return self._swap(self._lib.pa_bm_swap_out, "pa_bm_swap_out",
                          seq_ids, pairs_out)

    def swap_in(self, seq_ids, pairs_out=None):
        """Swap the group back in; returns (host, device) block pairs."""
        return self._swap(self._lib.pa_bm_swap_in, "pa_bm_swap_in", seq_ids,
                          pairs_out)

    def num_free_host(self) -> int:
        return self._lib.pa_bm_num_free_host(self._h)

    def host_refcount(self, block: int) -> int:
        return self._lib.pa_bm_host_refcount(self._h, block)

    def is_swapped(self, seq_id: int) -> bool:
        r = self._lib.pa_bm_is_swapped(self._h, seq_id)
        if r < 0:
            raise KeyError(seq_id)
        return bool(r)

    def seq_blocks(self, seq_id: int):
        """Table entries in logical order (host ids while swapped out)."""
        import numpy as np
        n = max(self.num_seq_blocks(seq_id), 0)
        out = np.empty(max(n, 1), dtype=np.int32)
        got = ctypes.c_int(0)
        _lib.check(self._lib.pa_bm_seq_blocks(
            self._h, seq_id, out.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
            n, ctypes.byref(got)), "pa_bm_seq_blocks")
        return out[:got.value]
