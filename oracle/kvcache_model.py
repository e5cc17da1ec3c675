"""Plain Python model of the BlockKVCache contract.

TEST INFRASTRUCTURE ONLY.  Written from "Core 注意力" (WorldFoundry docs),
section "Block KV cache 的调用顺序":

* every chunk follows before_update -> update -> cached_k/cached_v -> after_update;
* repeating the current chunk index overwrites the same logical chunk;
* the index plus one appends, or rolls the local window once it is full;
* skipping an index is an error;
* sink_size is a prefix that is never evicted, window_size is the rolling
  region, their sum is the cache's sequence length and is divisible by
  chunk_size.

Readings taken where the page is silent (each one is exercised by a test):

* the first chunk index is 0; a phase out of order is an error that leaves
  the state unchanged;
* sink_size is itself a multiple of chunk_size (otherwise one chunk would
  straddle the sink and the window) and the window holds at least one chunk;
* update takes exactly chunk_size tokens;
* logical chunk c lives in physical slot c while c < sink/chunk, after that in
  sink/chunk + (c - sink/chunk) mod (window/chunk);
* the visible tokens after writing chunk i are the physical prefix of
  min(i + 1, slots) slots; in logical order they are the sink chunks followed
  by the last window/chunk chunks up to i.

The model keeps per-slot contents as Python objects, so a test can state the
expected buffer bit for bit.
"""
from __future__ import annotations


class OrderError(Exception):
    """A call out of the documented order (the page says this raises)."""


class BlockKVCacheModel:
    IDLE, BEFORE, UPDATED, CACHED = 0, 1, 2, 3

    def __init__(self, cache_len: int, chunk_size: int, window_size: int, sink_size: int = 0):
        if chunk_size <= 0 or window_size < 0 or sink_size < 0:
            raise ValueError("sizes must be positive")
        if sink_size + window_size != cache_len:
            raise ValueError("sink_size + window_size must equal the cache length")
        if cache_len % chunk_size != 0:
            raise ValueError("cache length must be divisible by chunk_size")
        if sink_size % chunk_size != 0:
            raise ValueError("sink_size must be a multiple of chunk_size")
        if window_size < chunk_size:
            raise ValueError("the window must hold at least one chunk")
        self.chunk = chunk_size
        self.n_sink = sink_size // chunk_size
        self.n_window = window_size // chunk_size
        self.n_slots = self.n_sink + self.n_window
        self.slots = [None] * self.n_slots        # physical slot -> (chunk index, payload)
        self.committed = -1                      # last index passed to after_update
        self.current = -1                        # index of the cycle in progress
        self.phase = self.IDLE

    # --- slot arithmetic ---------------------------------------------------
    def slot_of(self, c: int) -> int:
        if c < self.n_sink:
            return c
        return self.n_sink + (c - self.n_sink) % self.n_window

    def visible_len(self, c: int) -> int:
        return self.chunk * min(c + 1, self.n_slots)

    def logical_chunks(self, c: int) -> list[int]:
        sink = list(range(min(c + 1, self.n_sink)))
        first = max(self.n_sink, c - self.n_window + 1)
        return sink + list(range(first, c + 1))

    # --- the four calls ----------------------------------------------------
    def before_update(self, idx: int) -> None:
        if self.phase != self.IDLE:
            raise OrderError("before_update while a chunk is in progress")
        if self.committed < 0:
            ok = idx == 0
        else:
            ok = idx in (self.committed, self.committed + 1)
        if not ok:
            raise OrderError(f"chunk index {idx} after {self.committed}")
        self.current = idx
        self.phase = self.BEFORE

    def update(self, payload, n_tokens: int) -> int:
        if self.phase != self.BEFORE:
            raise OrderError("update without before_update")
        if n_tokens != self.chunk:
            raise ValueError("update takes exactly chunk_size tokens")
        s = self.slot_of(self.current)
        self.slots[s] = (self.current, payload)
        self.phase = self.UPDATED
        return s

    def cached(self) -> tuple[int, list]:
        """Visible length and the physical slots' payloads, in physical order."""
        if self.phase not in (self.UPDATED, self.CACHED):
            raise OrderError("cached before update")
        self.phase = self.CACHED
        n = min(self.current + 1, self.n_slots)
        return self.visible_len(self.current), [self.slots[s][1] for s in range(n)]

    def cached_logical(self) -> list:
        """Visible payloads in logical (chunk index) order."""
        if self.phase not in (self.UPDATED, self.CACHED):
            raise OrderError("cached before update")
        by_idx = {c: p for c, p in (x for x in self.slots if x is not None)}
        return [by_idx[c] for c in self.logical_chunks(self.current)]

    def after_update(self, idx: int) -> None:
        if self.phase != self.CACHED:
            raise OrderError("after_update before cached")
        if idx != self.current:
            raise OrderError("after_update with a different chunk index")
        self.committed = idx
        self.phase = self.IDLE

    def state(self) -> tuple[int, int, int, int, int]:
        """(current, committed, write slot, visible length, phase)."""
        cur = self.current
        slot = self.slot_of(cur) if cur >= 0 else -1
        vis = self.visible_len(cur) if self.phase in (self.UPDATED, self.CACHED) else (
            self.visible_len(self.committed) if self.committed >= 0 else 0)
        return cur, self.committed, slot, vis, self.phase
