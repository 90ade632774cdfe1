"""CPU oracle for the sketch cache and the width adapter (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and bench.py's CPU legs may import
this module; it shares no code with the CUDA library.  Plain Python and numpy
(float64).

Source: the reading notes "SequenceO1：用可缓存的低秩草图实现端到端十万级用户历史建模".

* Section 2.4 "Local KVCache": the cache stores only the user-side sketch; its
  key holds the user id, the model version, the history timestamp and the
  sketch configuration; request-specific suffixes and candidate features are
  not cached.  Entries live for a time-to-live (three hours in training, one
  in serving) and capacity eviction bounds memory.  A miss runs FlashSA once
  and its result serves every target of the group (section 2.3, Figure 2:
  hit -> the fixed-size sketch; miss -> one compression).
* Section 2.3: a linear width adapter W_A in R^{d x D} maps the sketch to the
  ranking width (D = 1024 in the final configuration); the adapted sketch
  keeps k rows.  Its result is shared within a group but not persisted
  (section 2.4), so it is not cached.

Readings where the page is silent:
  C1  an entry is fresh while now - t_insert < ttl (strictly); an expired
      entry is a miss and is dropped when found;
  C2  a lookup that hits refreshes the entry's last-use time; capacity
      eviction takes a free slot (the smallest index) if there is one, else
      the expired entry inserted earliest, else the least recently used one
      (ties: the smaller slot index);
  C3  inserting a key that is present replaces its sketch and resets its
      insertion time; within one batch, a key that appears twice keeps the
      later sketch;
  C4  the adapter has no bias: Y = X~ W_A (reading R2: no bias anywhere).
"""

from __future__ import annotations

from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

F64 = np.float64


class SketchCacheModel:
    """Reference model of the cache's decisions (readings C1-C3).  Slots are
    numbered 0..capacity-1 and taken in increasing order while free."""

    def __init__(self, k: int, d: int, capacity: int, ttl: float):
        self.k, self.d, self.capacity, self.ttl = k, d, capacity, float(ttl)
        self.index: Dict[Tuple, int] = {}            # key -> slot
        self.slot_key: List[Optional[Tuple]] = [None] * capacity
        self.t_insert = [0.0] * capacity
        self.t_use = [0.0] * capacity
        self.xt = np.zeros((capacity, k, d), F64)
        self.m = np.zeros((capacity, k), F64)
        self.hits = self.misses = self.evictions = 0

    def _fresh(self, s: int, now: float) -> bool:
        return now - self.t_insert[s] < self.ttl

    def _drop(self, s: int) -> None:
        del self.index[self.slot_key[s]]
        self.slot_key[s] = None

    def lookup(self, keys: Sequence[Tuple], now: float) -> List[int]:
        """Slot of every key, or -1 on a miss (absent or expired)."""
        out = []
        for key in keys:
            s = self.index.get(tuple(key), -1)
            if s >= 0 and not self._fresh(s, now):
                self._drop(s)
                s = -1
            if s >= 0:
                self.t_use[s] = now
                self.hits += 1
            else:
                self.misses += 1
            out.append(s)
        return out

    def _victim(self, now: float) -> int:
        for s in range(self.capacity):
            if self.slot_key[s] is None:
                return s
        expired = [s for s in range(self.capacity) if not self._fresh(s, now)]
        if expired:
            s = min(expired, key=lambda i: (self.t_insert[i], i))
        else:
            s = min(range(self.capacity), key=lambda i: (self.t_use[i], i))
        self._drop(s)
        self.evictions += 1
        return s

    def insert(self, keys: Sequence[Tuple], now: float, xt: np.ndarray, m: np.ndarray) -> List[int]:
        """Stores xt[b], m[b] under keys[b]; returns the slot of each."""
        out = []
        for b, key in enumerate(keys):
            key = tuple(key)
            s = self.index.get(key, -1)
            if s < 0:
                s = self._victim(now)
                self.index[key] = s
                self.slot_key[s] = key
            self.t_insert[s] = now
            self.t_use[s] = now
            self.xt[s] = xt[b]
            self.m[s] = m[b]
            out.append(s)
        return out


def width_adapter(Xt: np.ndarray, W_A: np.ndarray) -> np.ndarray:
    """Y = X~ W_A over the last axis (section 2.3; reading C4)."""
    return np.asarray(Xt, F64) @ np.asarray(W_A, F64)
