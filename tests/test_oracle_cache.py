"""Pins for the sketch-cache model and the width adapter (oracle/sa_cache.py).

The cache's decisions are fixed by the notes' section 2.4 (key = user,
model version, history timestamp, sketch config; a time-to-live; capacity
eviction) and readings C1-C3.  Each pin is a hand-worked scenario with its
expected outcome written out: freshness at and just before the TTL, least
recently used eviction with a hit refreshing an entry, expired entries
evicted before live ones, replacement of a present key, every key field
taking part, the counters.  The adapter (section 2.3, reading C4) is pinned
by the identity, a selector matrix and pure-Python loops.

Planted mistakes (each trips a pin): a TTL test that keeps an entry at
exactly ttl, first-in-first-out eviction, a hit that does not refresh the
entry, eviction that ignores expiry, a key that drops the model version, an
adapter reading W_A's rows in reverse order.
"""

import numpy as np
import pytest

from oracle.sa_cache import SketchCacheModel, width_adapter


def _sk(v, k=2, d=3):
    return np.full((1, k, d), float(v)), np.full((1, k), float(v))


def _key(uid, ver=1, ts=100, cfg=7):
    return (uid, ver, ts, cfg)


def pin_ttl(model=SketchCacheModel):
    c = model(2, 3, 4, ttl=10.0)
    c.insert([_key(1)], 0.0, *_sk(5))
    assert c.lookup([_key(1)], 9.999) != [-1]
    assert c.lookup([_key(1)], 10.0) == [-1]      # C1: fresh only while age < ttl
    assert c.lookup([_key(1)], 1.0) == [-1]       # an expired entry was dropped


def pin_lru(model=SketchCacheModel):
    c = model(2, 3, 2, ttl=100.0)
    c.insert([_key(1)], 0.0, *_sk(1))
    c.insert([_key(2)], 1.0, *_sk(2))
    assert c.lookup([_key(1)], 2.0)[0] >= 0       # refreshes key 1
    c.insert([_key(3)], 3.0, *_sk(3))             # evicts key 2, the least recently used
    got = c.lookup([_key(1), _key(2), _key(3)], 4.0)
    assert got[0] >= 0 and got[1] == -1 and got[2] >= 0
    assert c.evictions == 1


def pin_expired_first(model=SketchCacheModel):
    c = model(2, 3, 2, ttl=8.0)
    c.insert([_key(1)], 0.0, *_sk(1))
    c.insert([_key(2)], 5.0, *_sk(2))
    c.lookup([_key(1)], 6.0)                      # key 1 used last, but inserted at 0
    c.insert([_key(3)], 9.0, *_sk(3))             # key 1 has expired (9 - 0 >= 8): it goes
    got = c.lookup([_key(2), _key(3)], 9.5)
    assert got[0] >= 0 and got[1] >= 0


def pin_replace_and_round_trip(model=SketchCacheModel):
    c = model(2, 3, 3, ttl=50.0)
    s = c.insert([_key(1)], 0.0, *_sk(1))[0]
    x2, m2 = _sk(2)
    assert c.insert([_key(1)], 1.0, x2, m2)[0] == s      # C3: same slot, new sketch
    xs = np.stack([_sk(3)[0][0], _sk(4)[0][0]])
    ms = np.stack([_sk(3)[1][0], _sk(4)[1][0]])
    c.insert([_key(9), _key(9)], 2.0, xs, ms)           # the later one wins
    a, b = c.lookup([_key(1), _key(9)], 3.0)
    assert np.all(c.xt[a] == 2.0) and np.all(c.m[a] == 2.0)
    assert np.all(c.xt[b] == 4.0) and np.all(c.m[b] == 4.0)
    assert c.lookup([_key(1)], 50.9) != [-1]            # the replacement reset the TTL at 1
    assert c.lookup([_key(1)], 51.0) == [-1]


def pin_expired_oldest_first(model=SketchCacheModel):
    c = model(2, 3, 3, ttl=10.0)
    c.insert([_key(1)], 2.0, *_sk(1))             # slot 0, inserted at 2
    c.insert([_key(2)], 0.0, *_sk(2))             # slot 1, inserted at 0
    c.insert([_key(3)], 5.0, *_sk(3))             # slot 2
    c.insert([_key(4)], 13.0, *_sk(4))            # keys 1 and 2 expired: key 2 (inserted first) goes
    got = c.lookup([_key(1), _key(2)], 13.5)
    assert got[1] == -1
    assert c.evictions == 1


def pin_key_fields(model=SketchCacheModel):
    c = model(2, 3, 8, ttl=50.0)
    c.insert([_key(1)], 0.0, *_sk(1))
    got = c.lookup([_key(2), _key(1, ver=2), _key(1, ts=101), _key(1, cfg=8), _key(1)], 1.0)
    assert got[:4] == [-1, -1, -1, -1] and got[4] >= 0
    assert (c.hits, c.misses) == (1, 4)


def pin_adapter(adapter=width_adapter):
    rng = np.random.default_rng(3)
    X = rng.standard_normal((2, 5, 4))
    assert np.max(np.abs(adapter(X, np.eye(4)) - X)) == 0.0
    sel = np.zeros((4, 6))
    sel[2, 5] = 1.0
    Y = adapter(X, sel)
    assert np.all(Y[..., 5] == X[..., 2]) and not np.any(Y[..., :5])
    W = rng.standard_normal((4, 3))
    want = [[[sum(X[b, j, i] * W[i, c] for i in range(4)) for c in range(3)] for j in range(5)]
            for b in range(2)]
    assert np.max(np.abs(adapter(X, W) - np.array(want))) < 1e-13


CACHE_PINS = [pin_ttl, pin_lru, pin_expired_first, pin_expired_oldest_first,
              pin_replace_and_round_trip, pin_key_fields]


@pytest.mark.parametrize("pin", CACHE_PINS + [pin_adapter], ids=lambda p: p.__name__)
def test_cache_oracle_satisfies_pin(pin):
    pin()


class _TtlInclusive(SketchCacheModel):
    def _fresh(self, s, now):
        return now - self.t_insert[s] <= self.ttl


class _Fifo(SketchCacheModel):
    def _victim(self, now):
        for s in range(self.capacity):
            if self.slot_key[s] is None:
                return s
        s = min(range(self.capacity), key=lambda i: (self.t_insert[i], i))
        self._drop(s)
        self.evictions += 1
        return s


class _NoRefresh(SketchCacheModel):
    def lookup(self, keys, now):
        saved = list(self.t_use)
        out = super().lookup(keys, now)
        self.t_use = saved
        return out


class _IgnoreExpiry(SketchCacheModel):
    def _victim(self, now):
        for s in range(self.capacity):
            if self.slot_key[s] is None:
                return s
        s = min(range(self.capacity), key=lambda i: (self.t_use[i], i))
        self._drop(s)
        self.evictions += 1
        return s


class _NoVersion(SketchCacheModel):
    def lookup(self, keys, now):
        return super().lookup([(k[0], 1, k[2], k[3]) for k in keys], now)


MUTANTS = {"TTL keeps an entry at exactly ttl": _TtlInclusive, "FIFO eviction": _Fifo,
           "a hit does not refresh": _NoRefresh, "eviction ignores expiry": _IgnoreExpiry,
           "key without the model version": _NoVersion}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_cache_mutant_is_caught(name):
    caught = []
    for pin in CACHE_PINS:
        try:
            pin(model=MUTANTS[name])
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"mutant {name!r} passed every pin"


def test_adapter_mutant_is_caught():
    # W_A read with its rows in reverse order (a layout mistake)
    with pytest.raises(AssertionError):
        pin_adapter(adapter=lambda X, W: np.asarray(X) @ np.asarray(W)[::-1])
