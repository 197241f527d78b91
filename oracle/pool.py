"""Model of the page allocator's free-list policy (host logic).

The pages keep the KV cache and its gradients in non-contiguous pages, so that
appending needs no reallocation or copy and memory does not fragment ([pt] §2B
"Gerenciamento de KV Cache Paginado"; [it] §2B).  They do not say which free
page is handed out next.  Reading: a free list used as a stack (LIFO on free),
initially holding ids 0..n-1 so that they are handed out ascending, or, with a
non-zero seed, in the order of a Fisher-Yates shuffle driven by SplitMix64.

SplitMix64 (Steele, Lea and Flood, "Fast Splittable Pseudorandom Number
Generators", OOPSLA 2014): state += 0x9E3779B97F4A7C15, then the output is the
state passed through two xor-shift-multiply rounds and a final xor-shift.
Fisher-Yates (Durstenfeld's form): for i = n-1 down to 1, j = r mod (i+1) with
r the next generator output, swap a[i] and a[j].
"""
from __future__ import annotations

_MASK = (1 << 64) - 1


class SplitMix64:
    def __init__(self, seed: int):
        self.state = seed & _MASK

    def next(self) -> int:
        self.state = (self.state + 0x9E3779B97F4A7C15) & _MASK
        z = self.state
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK
        return z ^ (z >> 31)


def initial_order(num_pages: int, seed: int) -> list[int]:
    """Order in which a fresh pool hands out its pages."""
    order = list(range(num_pages))
    if seed:
        rng = SplitMix64(seed)
        for i in range(num_pages - 1, 0, -1):
            j = rng.next() % (i + 1)
            order[i], order[j] = order[j], order[i]
    return order


class PoolModel:
    """alloc / free over the free-list stack; errors mirror the library's."""

    def __init__(self, num_pages: int, seed: int = 0):
        self.num_pages = num_pages
        self.stack = list(reversed(initial_order(num_pages, seed)))
        self.used = [False] * num_pages

    def alloc(self):
        if not self.stack:
            return None  # out of pages
        p = self.stack.pop()
        self.used[p] = True
        return p

    def free(self, p: int) -> bool:
        if not (0 <= p < self.num_pages) or not self.used[p]:
            return False  # bad page (out of range or double free)
        self.used[p] = False
        self.stack.append(p)
        return True
