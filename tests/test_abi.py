"""The C ABI: the library loads, exports every symbol include/pagedkv.h
declares, and rejects bad arguments on the host (no GPU needed: argument
checks run before any CUDA call)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    text = open(os.path.join(ROOT, "include", "pagedkv.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_\w+)\s*\(", text)))


def test_every_declared_symbol_is_exported(pkv):
    from paged_kv_cache_383_b200 import _lib
    names = declared_functions()
    assert len(names) >= 20
    raw = ctypes.CDLL(_lib.LIB_PATH)
    for n in names:
        assert hasattr(raw, n), n
    assert set(names) == set(_lib.SIGNATURES), \
        set(names) ^ set(_lib.SIGNATURES)


def test_version_and_status_strings(pkv):
    from paged_kv_cache_383_b200 import _lib
    lib = _lib.load()
    assert b"sm_100a" in lib.pa_version()
    assert lib.pa_status_string(_lib.PA_ERR_NO_FREE_BLOCKS) == b"no free blocks"


def _desc(**kw):
    from paged_kv_cache_383_b200 import pa_decode_desc
    base = dict(num_seqs=2, num_q_heads=8, num_kv_heads=2, head_dim=128,
                block_size=16, max_blocks_per_seq=4, num_blocks=16, dtype=1,
                partition_size=0, max_context_len=0, kernel=0)
    base.update(kw)
    return pa_decode_desc(**base)


@pytest.mark.parametrize("kw,status", [
    (dict(head_dim=96), 2),
    (dict(block_size=8), 2),
    (dict(num_q_heads=7), 1),
    (dict(num_q_heads=32, num_kv_heads=2), 2),
    (dict(partition_size=24), 1),
    (dict(dtype=5), 1),
    (dict(kernel=9), 1),
    (dict(reduce=4), 1),
    (dict(num_seqs=-1), 1),
])
def test_decode_rejects_bad_descriptors(pkv, kw, status):
    from paged_kv_cache_383_b200 import _lib
    lib = _lib.load()
    d = _desc(**kw)
    st = lib.pa_decode(None, None, None, None, None, None, ctypes.c_float(1.0),
                       ctypes.byref(d), None, 0, None, None)
    assert st == status
    assert lib.pa_last_error()


def test_decode_rejects_null_and_misaligned(pkv):
    from paged_kv_cache_383_b200 import _lib
    lib = _lib.load()
    d = _desc()
    st = lib.pa_decode(None, None, None, None, None, None, ctypes.c_float(1.0),
                       ctypes.byref(d), None, 0, None, None)
    assert st == _lib.PA_ERR_INVALID_ARG
    fake = 0x1000
    st = lib.pa_decode(fake + 2, fake, fake, fake, fake, fake,
                       ctypes.c_float(1.0), ctypes.byref(d), None, 0, None,
                       None)
    assert st == _lib.PA_ERR_INVALID_ARG
    assert b"aligned" in lib.pa_last_error()
    st = lib.pa_decode(fake, fake, fake, fake, fake, fake,
                       ctypes.c_float(float("nan")), ctypes.byref(d), None, 0,
                       None, None)
    assert st == _lib.PA_ERR_INVALID_ARG


def test_decode_needs_workspace_for_split(pkv):
    from paged_kv_cache_383_b200 import _lib
    lib = _lib.load()
    d = _desc(partition_size=16, max_blocks_per_seq=8)
    need = lib.pa_decode_workspace_bytes(ctypes.byref(d))
    # o: 2 seqs x 8 q heads x 8 partitions x 128 floats; (m, l): x 2 floats;
    # 2 seqs x 2 kv heads int32 counters; 2 seqs x 8 partitions int32 of
    # unit order; 2 int32 of sequence order; each piece rounded up to 16
    # bytes
    assert need == 2 * 8 * 8 * 128 * 4 + 2 * 8 * 8 * 2 * 4 + 16 + 64 + 16
    fake = 0x1000
    st = lib.pa_decode(fake, fake, fake, fake, fake, fake,
                       ctypes.c_float(1.0), ctypes.byref(d), None, 0, None,
                       None)
    assert st == _lib.PA_ERR_WORKSPACE
    d1 = _desc(partition_size=64)
    # one partition: only the sequence order (2 int32, rounded to 16 bytes)
    assert lib.pa_decode_workspace_bytes(ctypes.byref(d1)) == 16
    assert lib.pa_decode_partition_size(ctypes.byref(d1)) == 64


def test_zero_sized_calls_are_noops(pkv):
    from paged_kv_cache_383_b200 import _lib
    lib = _lib.load()
    d = _desc(num_seqs=0)
    assert lib.pa_decode(None, None, None, None, None, None,
                         ctypes.c_float(1.0), ctypes.byref(d), None, 0, None,
                         None) == 0
    assert lib.pa_cache_write(None, None, None, None, None, 0, 8, 128, 16, 4,
                              1, None, None) == 0
    assert lib.pa_copy_blocks(None, None, None, 0, 8, 128, 16, 4, 1, None,
                              None) == 0
    assert lib.pa_cache_write(None, None, None, None, None, 3, 8, 128, 16, 4,
                              1, None, None) == _lib.PA_ERR_INVALID_ARG


@pytest.mark.parametrize("seqs,hq,hkv,total_q,max_q", [
    (8, 64, 8, 33166, 8192),    # whole prompts: T = 16, bound by total_q
    (16, 64, 8, 8192, 512),     # 512-token chunks: 32 tiles each, exact
    (256, 64, 8, 1024, 4),      # 4 drafts: one tile per sequence
    (3, 8, 8, 1000, 700),       # G = 1: T = 128
    (5, 32, 8, 7, 7),           # fewer rows than tiles' worth
])
def test_prefill_workspace_formula(pkv, seqs, hq, hkv, total_q, max_q):
    """pa_prefill_workspace_bytes is the header's formula: the order
    (num_seqs int32) rounded up to 16, a 16-byte work counter, and 8 bytes
    per tile-map entry for min(total_q // T + num_seqs,
    num_seqs * ceil(max_q_len / T)) entries of T = 128 / G new tokens,
    rounded up to 16."""
    from paged_kv_cache_383_b200 import _lib
    lib = _lib.load()
    d = _lib.pa_prefill_desc(num_seqs=seqs, num_q_heads=hq, num_kv_heads=hkv,
                             head_dim=128, block_size=16,
                             max_blocks_per_seq=512, num_blocks=4096, dtype=1,
                             total_q=total_q, max_q_len=max_q,
                             max_context_len=8192)
    t = 128 // (hq // hkv)
    cap = min(total_q // t + seqs, seqs * -(-max_q // t))
    up16 = lambda n: (n + 15) // 16 * 16
    assert (lib.pa_prefill_workspace_bytes(ctypes.byref(d)) ==
            up16(4 * seqs) + 16 + up16(8 * cap))


def test_prefill_needs_its_order_workspace(pkv):
    from paged_kv_cache_383_b200 import _lib
    lib = _lib.load()
    d = _lib.pa_prefill_desc(num_seqs=5, num_q_heads=8, num_kv_heads=2,
                             head_dim=128, block_size=16,
                             max_blocks_per_seq=4, num_blocks=16, dtype=1,
                             total_q=20, max_q_len=4, max_context_len=64)
    # the sequence order (5 int32 -> 32 bytes), the work counter (16) and
    # the tile map: G = 4, so 32 new tokens per tile, room for
    # min(20 // 32 + 5, 5 * 1) = 5 tiles of 8 bytes (-> 48)
    assert lib.pa_prefill_workspace_bytes(ctypes.byref(d)) == 96
    fake = 0x1000
    args = [fake] * 7 + [ctypes.c_float(1.0), ctypes.byref(d)]
    for ws, nbytes in ((None, 96), (fake, 80), (fake + 4, 96)):
        st = lib.pa_prefill(*args, ws, nbytes, None, None)
        assert st == _lib.PA_ERR_WORKSPACE, (ws, nbytes)
        assert b"workspace" in lib.pa_last_error()
    d0 = _lib.pa_prefill_desc(num_seqs=0, num_q_heads=8, num_kv_heads=2,
                              head_dim=128, block_size=16,
                              max_blocks_per_seq=4, num_blocks=16, dtype=1)
    assert lib.pa_prefill(*([None] * 7), ctypes.c_float(1.0),
                          ctypes.byref(d0), None, 0, None, None) == 0


def test_prefill_refuses_more_query_tiles_than_the_grid_holds(pkv):
    from paged_kv_cache_383_b200 import _lib
    lib = _lib.load()
    # G = 1: 128 new tokens per tile; one CTA per (tile, KV head) in a
    # one-dimensional grid of at most 2^31 - 1: (2^31 - 1) // 128 + 1 tiles
    # x 256 KV heads is over
    d = _lib.pa_prefill_desc(num_seqs=1, num_q_heads=256, num_kv_heads=256,
                             head_dim=128, block_size=16,
                             max_blocks_per_seq=1 << 20, num_blocks=1 << 20,
                             dtype=1, total_q=(1 << 31) - 1,
                             max_q_len=(1 << 31) - 1)
    fake = 0x1000
    st = lib.pa_prefill(*([fake] * 7), ctypes.c_float(1.0), ctypes.byref(d),
                        fake, 16, None, None)
    assert st == _lib.PA_ERR_UNSUPPORTED
    assert b"query tiles" in lib.pa_last_error()


def test_wait_probe_needs_an_error_word(pkv):
    from paged_kv_cache_383_b200 import _lib
    lib = _lib.load()
    assert lib.pa_wait_probe(None, None) == _lib.PA_ERR_INVALID_ARG
    assert b"error word" in lib.pa_last_error()


def test_prefill_kernel_choice_is_checked(pkv):
    from paged_kv_cache_383_b200 import _lib
    lib = _lib.load()
    fake = 0x1000

    def call(**kw):
        base = dict(num_seqs=2, num_q_heads=32, num_kv_heads=8, head_dim=128,
                    block_size=16, max_blocks_per_seq=4, num_blocks=16,
                    dtype=1, total_q=20, max_q_len=10, max_context_len=64)
        base.update(kw)
        d = _lib.pa_prefill_desc(**base)
        return lib.pa_prefill(*([fake] * 7), ctypes.c_float(1.0),
                              ctypes.byref(d), None, 0, None, None)

    for kernel in (7, 2, -1):
        assert call(kernel=kernel) == _lib.PA_ERR_INVALID_ARG
        assert b"kernel" in lib.pa_last_error()
    # a valid choice gets as far as the workspace check
    assert call(kernel=_lib.PA_PREFILL_AUTO) == _lib.PA_ERR_WORKSPACE
    assert call(kernel=_lib.PA_PREFILL_TILE) == _lib.PA_ERR_WORKSPACE
    # precision of P in P . V: auto, split or single; nothing else
    for pv in (-1, 3):
        assert call(pv=pv) == _lib.PA_ERR_INVALID_ARG
        assert b"pv" in lib.pa_last_error()
    for pv in (_lib.PA_PV_AUTO, _lib.PA_PV_SPLIT, _lib.PA_PV_SINGLE):
        assert call(pv=pv) == _lib.PA_ERR_WORKSPACE


def test_out_fp32_flag_is_checked(pkv):
    from paged_kv_cache_383_b200 import _lib
    lib = _lib.load()
    fake = 0x1000
    d = _desc(out_fp32=2)
    assert lib.pa_decode(fake, fake, fake, fake, fake, fake,
                         ctypes.c_float(1.0), ctypes.byref(d), None, 0, None,
                         None) == _lib.PA_ERR_INVALID_ARG
    assert b"out_fp32" in lib.pa_last_error()
    p = _lib.pa_prefill_desc(num_seqs=2, num_q_heads=8, num_kv_heads=2,
                             head_dim=128, block_size=16,
                             max_blocks_per_seq=4, num_blocks=16, dtype=1,
                             total_q=8, max_q_len=4, max_context_len=64,
                             out_fp32=3)
    assert lib.pa_prefill(*([fake] * 7), ctypes.c_float(1.0),
                          ctypes.byref(p), None, 0, None,
                          None) == _lib.PA_ERR_INVALID_ARG
