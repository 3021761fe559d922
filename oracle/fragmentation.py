"""Block counts, internal-fragmentation waste and prefix-sharing arithmetic.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Sources:

* [KV-cache chapter] "Internal fragmentation: the cost of guessing wrong on
  purpose" -- the contiguous scheme reserves ``max_seq_len`` slots per request.
* [KV-cache chapter] "Worked Example 1: how much memory fragmentation actually
  costs" -- under paging each request takes ``ceil(len / block_size)`` blocks;
  waste is the slots reserved minus the tokens stored, as a percentage of the
  slots reserved; the reduction factor is contiguous slots over paged slots.
* [Taming the Tail] "Why This Crushes Tail Latency" -- only the last block of
  a sequence can be partly empty, so per-sequence waste is below one block.
* [KV-cache chapter] "Worked Example 2: what a shared system prompt is
  actually worth" and answers A3/A5 of "Active recall" -- block counts with and
  without a shared prompt, and how many prompt blocks are whole (shareable).

Reading (the two sharing counts).  Worked Example 2 stores the prompt once as
``ceil(prompt / block_size)`` blocks and each request's question as
``ceil(question / block_size)`` blocks; answer A3 counts only whole prompt
blocks, ``floor(prompt / block_size)``, as shareable.  For a 380-token prompt
at block size 16 these differ (24 vs 23): 380 is not a multiple of 16, although
Worked Example 2 says the boundary is aligned.  ``sharing_blocks`` restates
Worked Example 2's own count; ``shareable_prompt_blocks`` restates A3's.  The
block manager's real count for that case (23 shared whole blocks plus one
shared partial block that each writer copies) is what the block-manager tests
check.
"""
from __future__ import annotations

from dataclasses import dataclass


def blocks_for(length: int, block_size: int) -> int:
    """Blocks a sequence of ``length`` tokens occupies: ``ceil(len / bs)``."""
    if length < 0 or block_size <= 0:
        raise ValueError("length must be >= 0 and block_size > 0")
    return (length + block_size - 1) // block_size


def waste_slots(length: int, block_size: int) -> int:
    """Empty token slots in a sequence's last block."""
    return blocks_for(length, block_size) * block_size - length


@dataclass(frozen=True)
class FragmentationReport:
    """Paged vs contiguous reservation for one batch of finished requests."""
    blocks_per_seq: tuple
    waste_per_seq: tuple
    total_blocks: int
    actual_tokens: int
    paged_slots: int
    contiguous_slots: int
    paged_waste_pct: float        # unrounded percentages
    contiguous_waste_pct: float
    reduction_factor: float

    def rounded(self, ndigits: int = 2) -> dict:
        """The report with the three ratios rounded as the worked examples
        print them."""
        return {
            "total_blocks": self.total_blocks,
            "actual_tokens": self.actual_tokens,
            "paged_slots": self.paged_slots,
            "contiguous_slots": self.contiguous_slots,
            "paged_waste_pct": round(self.paged_waste_pct, ndigits),
            "contiguous_waste_pct": round(self.contiguous_waste_pct, ndigits),
            "reduction_factor": round(self.reduction_factor, ndigits),
        }


def fragmentation(lengths, block_size: int,
                  max_seq_len: int) -> FragmentationReport:
    """Compare paged allocation against per-request max-length reservation.

    Paged: each request holds ``ceil(len / block_size)`` blocks; the slots it
    reserves are blocks times block size.  Contiguous: each request reserves
    ``max_seq_len`` slots up front.  Waste is reserved minus stored tokens, as
    a percentage of what was reserved; the reduction factor is contiguous over
    paged slots.
    """
    lengths = [int(x) for x in lengths]
    if any(x > max_seq_len for x in lengths):
        raise ValueError("a request is longer than max_seq_len")
    per_blocks = tuple(blocks_for(x, block_size) for x in lengths)
    per_waste = tuple(waste_slots(x, block_size) for x in lengths)
    total_blocks = sum(per_blocks)
    actual = sum(lengths)
    paged = total_blocks * block_size
    contiguous = max_seq_len * len(lengths)
    return FragmentationReport(
        blocks_per_seq=per_blocks,
        waste_per_seq=per_waste,
        total_blocks=total_blocks,
        actual_tokens=actual,
        paged_slots=paged,
        contiguous_slots=contiguous,
        paged_waste_pct=100.0 * (paged - actual) / paged,
        contiguous_waste_pct=100.0 * (contiguous - actual) / contiguous,
        reduction_factor=contiguous / paged,
    )


def sharing_blocks(prompt_len: int, suffix_len: int, num_requests: int,
                   block_size: int) -> dict:
    """Blocks for ``num_requests`` requests with and without a shared prompt,
    counted as Worked Example 2 and answer A5 count them: the prompt takes
    ``ceil(prompt / bs)`` blocks and each request's own part
    ``ceil(suffix / bs)``; without sharing every request holds both, with
    sharing the prompt blocks are held once."""
    p = blocks_for(prompt_len, block_size)
    s = blocks_for(suffix_len, block_size)
    without = num_requests * (p + s)
    with_sharing = p + num_requests * s
    return {"prompt_blocks": p, "suffix_blocks": s,
            "without_sharing": without, "with_sharing": with_sharing,
            "reduction_factor": without / with_sharing}


def shareable_prompt_blocks(prompt_len: int, block_size: int) -> dict:
    """Whole prompt blocks (no private token inside) and the prompt tokens
    they hold, as answer A3 counts them: ``floor(prompt / bs)`` blocks."""
    whole = prompt_len // block_size
    return {"blocks": whole, "tokens": whole * block_size,
            "fraction": whole * block_size / prompt_len}
