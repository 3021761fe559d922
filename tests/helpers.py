"""Shared helpers of the GPU parity tests: oracle calls on sampled sequences
and the decode tolerance.

Tolerance (decode output against the unrounded fp64 oracle): every element
within 2e-3 absolute, and every element with |ref| >= 0.2 within 1e-2
relative.  One carve-out, the output-rounding floor: where half a unit in the
last place of the output dtype at |ref| is itself >= 2e-3 (|ref| >= 1 for
bf16, >= 8 for fp16), no correctly rounded output can meet 2e-3, so such
elements are held to the relative bound and to half an ulp + 2e-3.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import attention as oa

ATOL = 2e-3
RTOL = 1e-2
REL_FLOOR = 0.2
MANTISSA = {torch.bfloat16: 8, torch.float16: 11}   # incl. implicit bit


def half_ulp(ref: np.ndarray, dtype) -> np.ndarray:
    p = MANTISSA[dtype]
    e = np.floor(np.log2(np.maximum(np.abs(ref), 1e-30)))
    return 2.0 ** (e - p)          # ulp = 2^(e - p + 1)


def check_decode(out, ref, dtype, what=""):
    """Assert the tolerance; returns (max_abs, max_rel over |ref|>=0.2)."""
    out = np.asarray(out, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert out.shape == ref.shape
    assert np.isfinite(out).all(), f"{what}: non-finite output"
    err = np.abs(out - ref)
    hu = half_ulp(ref, dtype)
    floor = hu >= ATOL
    bad_abs = (~floor) & (err > ATOL)
    bad_floor = floor & (err > hu + ATOL)
    big = np.abs(ref) >= REL_FLOOR
    rel = np.where(big, err / np.maximum(np.abs(ref), 1e-30), 0.0)
    bad_rel = rel > RTOL
    max_abs = float(err.max()) if err.size else 0.0
    max_rel = float(rel.max()) if rel.size else 0.0
    assert not bad_abs.any(), (
        f"{what}: {int(bad_abs.sum())} elements over abs {ATOL}; "
        f"max abs err {float(err[~floor].max()):.3e}")
    assert not bad_floor.any(), f"{what}: rounding-floor elements too far"
    assert not bad_rel.any(), f"{what}: max rel err {max_rel:.3e}"
    return max_abs, max_rel


def to_np(t) -> np.ndarray:
    return t.detach().float().cpu().numpy()


def oracle_paged_sample(q, k_cache, v_cache, tables, lengths, scale, seqs):
    """fp64 oracle for the listed sequences; the sequences' own blocks are
    copied to the host (a relabelled sub-pool: the oracle's result does not
    depend on block ids) so full-size pools need not leave the device."""
    out = {}
    for b in seqs:
        L = int(lengths[b])
        nblk = -(-L // k_cache.shape[2])
        ids = np.asarray(tables[b][:nblk], dtype=np.int64)
        if nblk:
            idx = torch.from_numpy(ids).to(k_cache.device)
            kc = to_np(k_cache.index_select(0, idx))
            vc = to_np(v_cache.index_select(0, idx))
        else:
            shp = (1,) + tuple(k_cache.shape[1:])
            kc = vc = np.zeros(shp)
        sub = np.arange(max(nblk, 1))[None, :]
        out[b] = oa.paged_decode(to_np(q[b:b + 1]), kc, vc, sub,
                                 np.array([L]), scale)[0]
    return out


def sample_seqs(lengths, k=6, seed=0):
    """The shortest and longest sequences plus a few random ones."""
    lengths = np.asarray(lengths)
    order = np.argsort(lengths, kind="stable")
    rng = np.random.default_rng(seed)
    pick = {int(order[0]), int(order[-1])}
    extra = rng.choice(len(lengths), size=min(k, len(lengths)), replace=False)
    for b in extra:
        if len(pick) >= k:
            break
        pick.add(int(b))
    return sorted(pick)


def poison_unwritten(inp) -> None:
    """Fill every cache slot no sequence has written (the tail of each last
    block and every block no table references) with NaN, in place.  Keys
    past a context are masked, so the result must not change."""
    bs = inp.workload.block_size
    used = np.zeros(inp.num_blocks, dtype=bool)
    for b, L in enumerate(inp.lengths):
        n = (int(L) + bs - 1) // bs
        used[inp.block_tables[b, :n]] = True
        if L % bs:
            last = int(inp.block_tables[b, n - 1])
            inp.k_cache[last, :, L % bs:] = float("nan")
            inp.v_cache[last, :, L % bs:] = float("nan")
    free = torch.from_numpy(np.flatnonzero(~used)).to(inp.k_cache.device)
    inp.k_cache[free] = float("nan")
    inp.v_cache[free] = float("nan")


def check_strict(out32, ref, what=""):
    """The tolerance with no carve-out, for float32 outputs (the kernel's
    value before the final rounding): every element within 2e-3 absolute,
    every element with |ref| >= 0.2 within 1e-2 relative."""
    out32 = np.asarray(out32, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert out32.shape == ref.shape
    assert np.isfinite(out32).all(), f"{what}: non-finite output"
    err = np.abs(out32 - ref)
    big = np.abs(ref) >= REL_FLOOR
    rel = np.where(big, err / np.maximum(np.abs(ref), 1e-30), 0.0)
    assert err.max() <= ATOL, f"{what}: max abs err {err.max():.3e}"
    assert rel.max() <= RTOL, f"{what}: max rel err {rel.max():.3e}"
    return float(err.max()), float(rel.max())


def prefill_both(pkv, out, *args, **kw):
    """pa_prefill into ``out`` (the input dtype) and, on the same inputs,
    into a float32 tensor (the kernel's value before the output rounding);
    returns the float32 tensor."""
    import torch
    out32 = torch.full(out.shape, float("nan"), dtype=torch.float32,
                       device=out.device)
    pkv.pa_prefill(out32, *args, **kw)
    pkv.pa_prefill(out, *args, **kw)
    return out32


def check_prefill(out, out32, ref, what="", rows=None):
    """The tolerance for a prefill output, with the output-rounding floor
    handled as its reading prescribes: the float32 value (before the output
    rounding) must meet the tolerance with no carve-out -- every element
    within 2e-3, every element with |ref| >= 0.2 within 1e-2 relative -- and
    the dtype output must be exactly its round-to-nearest-even.  So the only
    error past 2e-3 in the dtype output is that rounding itself: up to half
    an ulp, 2^-9 |ref| in bf16, which at |ref| >= 0.5 leaves a rounded output
    as little as 5e-5 of room under a flat 2e-3.  ``rows`` selects the rows
    compared (all if None)."""
    import torch
    assert out32.dtype == torch.float32
    if rows is not None:
        idx = torch.as_tensor(np.asarray(rows), device=out.device)
        out, out32 = out.index_select(0, idx), out32.index_select(0, idx)
    assert torch.equal(out, out32.to(out.dtype)), (
        f"{what}: dtype output is not the rounding of the float32 value")
    return check_strict(to_np(out32), ref, what)
