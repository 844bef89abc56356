"""Segments of one head class in original positions, as lists of (start, end)
runs ("4.1.2 · LongLoRA: 用S²-Attn完成长上下文微调" §1: strict shifted heads have a
short head group [0, s), full groups [s + kG, s + kG + G) and a short tail
[N - s, N); rolled shifted heads have the wrap group [N - s, N) then [0, s)).
Test helper; checked against the oracle's adjacency matrices in
tests/test_oracle_pins.py."""
from __future__ import annotations


def segments(N: int, G: int, variant: int, cls: int) -> list[list[tuple[int, int]]]:
    s = G // 2
    if variant == 2:
        return [[(0, N)]]
    if cls == 0:
        return [[(a, a + G)] for a in range(0, N, G)]
    if variant == 0:
        return [[(0, s)]] + [[(a, a + G)] for a in range(s, N - s, G)] + [[(N - s, N)]]
    return [[(a, a + G)] for a in range(s, N - s, G)] + [[(N - s, N), (0, s)]]
