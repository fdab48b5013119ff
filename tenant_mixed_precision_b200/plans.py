"""Rank plans: how many singular vectors each bit width keeps.

Delta-CoMe fills 8/3/2-bit groups of singular vectors in descending singular-value order and drops
the rest (0 bit), at the size of a 1-bit delta ("Delta-CoMe: Training-Free Delta-Compression with
Mixed-Precision for Large Language Models", sections "Approach" and "Limitations": a greedy
search chose the group sizes).  Here the group sizes are given and the last group takes whatever
the code-bit budget ratio*16*d_out*d_in still allows (scales, zeros and S are not charged).
"""
from __future__ import annotations


def budget_plan(d_out: int, d_in: int, ratio: float, widths) -> list[tuple[int, int]]:
    """widths: [(bits, count or None), ...]; None = as many as the remaining budget allows."""
    cap = min(d_out, d_in)
    budget = ratio * 16.0 * d_out * d_in
    per = d_out + d_in
    used, taken, plan = 0, 0, []
    for bits, count in widths:
        if bits <= 0:
            continue
        if count is None:
            count = int((budget - used) // (bits * per))
        count = max(0, min(int(count), cap - taken))
        plan.append((int(bits), count))
        used += bits * count * per
        taken += count
    return plan


# The allocations of the benchmark workloads (1/16 mixed, 1/32 mixed, single-precision 3-bit).
MIXED_1_16 = [(8, 2), (3, 32), (2, None)]
MIXED_1_32 = [(8, 1), (3, 16), (2, None)]
ALL_3BIT = [(3, None)]
