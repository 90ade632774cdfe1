"""GPU parity of the sketch cache and the width adapter (sections 2.3 and 2.4
of the SequenceO1 reading notes) against the oracle (oracle/sa_cache.py),
through the C ABI.

* Cache decisions: a seeded stream of lookups and inserts (a small key
  universe, so that hits, expiry, replacement, duplicate keys and capacity
  eviction all occur) runs on the library and on SketchCacheModel; the hit
  masks, the counters and every sketch a lookup returns must be identical
  (the cache only moves fp32 data: bit-exact).
* Cached forward: a first call misses every user and must match the SA
  oracle; a second call with some of the same keys returns exactly the
  sketches the first call stored for them and computes the others (three
  runs of consecutive misses, each compressed in place over its rows).
* Adapter: Y = X~ W_A against the oracle on the bf16-rounded operands
  (ragged row tails, d = 64 and 128, D = 256 and 1024): the only rounding
  left is fp32 accumulation and the bf16 output, |err| <= 2^-8 |Y| + 1e-6
  sum |x||w|.
"""

import numpy as np
import pytest

from gpu_util import assert_user_close
from oracle import sa_batch
from oracle.sa_cache import SketchCacheModel, width_adapter
from synthetic.workloads import make_inputs, round_to_bf16

pytestmark = pytest.mark.gpu


def _sketches(rng, n, k, d):
    return (rng.standard_normal((n, k, d)).astype(np.float32),
            rng.uniform(0.0, 100.0, (n, k)).astype(np.float32))


@pytest.mark.parametrize("capacity,ttl", [(8, 5.0), (3, 1e9), (32, 2.0)])
def test_cache_decisions_and_round_trip_match_the_model(capacity, ttl):
    import torch
    from sketch_attention_compression_b200 import SketchCache
    k, d = 4, 8
    rng = np.random.default_rng(capacity * 31 + int(ttl))
    cache = SketchCache(k, d, capacity, ttl)
    model = SketchCacheModel(k, d, capacity, ttl)
    now = 0.0
    universe = [(u, v, 100 + u % 3, 7) for u in range(12) for v in (1, 2)]
    for step in range(120):
        now += float(rng.choice([0.0, 0.25, 0.5, 1.0, 3.0]))
        keys = [universe[i] for i in rng.integers(0, len(universe), int(rng.integers(1, 7)))]
        if step % 2 == 0:
            xt, m = _sketches(rng, len(keys), k, d)
            cache.insert(keys, now, torch.from_numpy(xt).cuda(), torch.from_numpy(m).cuda())
            model.insert(keys, now, xt, m)
        else:
            out_x = torch.full((len(keys), k, d), -7.0, device="cuda")
            out_m = torch.full((len(keys), k), -7.0, device="cuda")
            hit = cache.lookup(keys, now, out_x, out_m)
            slots = model.lookup(keys, now)
            assert list(hit) == [s >= 0 for s in slots], f"step {step}"
            got_x, got_m = out_x.cpu().numpy(), out_m.cpu().numpy()
            for b, s in enumerate(slots):
                if s >= 0:
                    assert np.array_equal(got_x[b], model.xt[s].astype(np.float32)), f"step {step}"
                    assert np.array_equal(got_m[b], model.m[s].astype(np.float32)), f"step {step}"
                else:  # a miss leaves the output row as it was
                    assert np.all(got_x[b] == -7.0) and np.all(got_m[b] == -7.0)
    st = cache.stats()
    assert (st["hits"], st["misses"], st["evictions"]) == (model.hits, model.misses,
                                                           model.evictions)
    assert st["entries"] == len(model.index)
    assert model.hits > 0
    if capacity < len(universe):
        assert model.evictions > 0
    cache.close()


def _query(inp):
    import torch
    from sketch_attention_compression_b200 import SketchQuery
    t = {key: torch.from_numpy(inp[key]).cuda().to(torch.bfloat16) for key in ("P", "W_Q", "W_K")}
    return SketchQuery(t["P"], t["W_Q"], t["W_K"], inp["scale"])


@pytest.mark.parametrize("k", [64, 300])
def test_cached_forward_serves_hits_and_computes_misses(k):
    import torch
    from sketch_attention_compression_b200 import SketchCache, read_device_status
    lengths = [700, 0, 129, 3000, 1, 255, 4100, 96]
    inp = make_inputs(lengths, 128, k, "bf16", seed=k)
    q = _query(inp)
    X = torch.from_numpy(inp["X"]).cuda().to(torch.bfloat16)
    cache = SketchCache(k, 128, capacity=16, ttl=60.0)
    keys = [(100 + b, 3, 555, 9) for b in range(len(lengths))]
    Xt1, m1, hit1, ws = cache.forward(q, keys, 0.0, X, inp["offsets"])
    assert not hit1.any()
    assert read_device_status(ws) == 0
    Xo, mo = sa_batch(inp["X"], inp["offsets"], inp["P"], inp["W_Q"], inp["W_K"], inp["scale"])
    g1x, g1m = Xt1.double().cpu().numpy(), m1.double().cpu().numpy()
    for b in range(len(lengths)):
        assert_user_close(g1x[b], g1m[b], Xo[b], mo[b], "bf16", f"user {b}")
    # Second call: users 0, 3, 6 keep their keys (hits); the others are new
    # (history timestamp moved), so they are recomputed from the rows.
    keys2 = [key if b in (0, 3, 6) else (key[0], key[1], 556, key[3]) for b, key in enumerate(keys)]
    Xt2, m2, hit2, _ = cache.forward(q, keys2, 10.0, X, inp["offsets"], workspace=ws)
    assert list(hit2) == [b in (0, 3, 6) for b in range(len(lengths))]
    g2x, g2m = Xt2.double().cpu().numpy(), m2.double().cpu().numpy()
    for b in range(len(lengths)):
        if hit2[b]:
            assert np.array_equal(g2x[b], g1x[b]) and np.array_equal(g2m[b], g1m[b])
        else:
            assert_user_close(g2x[b], g2m[b], Xo[b], mo[b], "bf16", f"user {b} (second call)")
    assert read_device_status(ws) == 0
    st = cache.stats()
    assert (st["hits"], st["misses"], st["entries"]) == (3, 13, 13)
    # An all-hit call runs no SA pass and returns the stored sketches.
    Xt3, m3, hit3, _ = cache.forward(q, keys2, 20.0, X, inp["offsets"], workspace=ws)
    assert hit3.all()
    assert torch.equal(Xt3, Xt2) and torch.equal(m3, m2)
    cache.close()
    q.close()


def test_cached_forward_full_size():
    # The benchmark's 16 x 100K workload through the cache: the first call
    # computes every user; the second keeps ten of the sixteen keys, serves
    # them from the pool bit for bit and recomputes the other six in place;
    # sampled users of both calls against the oracle.
    import torch
    from gpu_util import assert_total_mass
    from sketch_attention_compression_b200 import SketchCache, read_device_status
    from synthetic import generate
    inp = generate("batch16_n100k_d128_k128_mixture_bf16")
    q = _query(inp)
    X = torch.from_numpy(inp["X"]).cuda().to(torch.bfloat16)
    cache = SketchCache(128, 128, capacity=32, ttl=60.0)
    keys = [(1000 + b, 1, 7, 0) for b in range(16)]
    Xt1, m1, hit1, ws = cache.forward(q, keys, 0.0, X, inp["offsets"])
    assert not hit1.any() and read_device_status(ws) == 0
    g1x, g1m = Xt1.double().cpu().numpy(), m1.double().cpu().numpy()
    keys2 = keys[:10] + [(2000 + b, 1, 7, 0) for b in range(10, 16)]
    Xt2, m2, hit2, _ = cache.forward(q, keys2, 1.0, X, inp["offsets"], workspace=ws)
    assert list(hit2) == [b < 10 for b in range(16)]
    assert read_device_status(ws) == 0
    g2x, g2m = Xt2.double().cpu().numpy(), m2.double().cpu().numpy()
    assert np.array_equal(g2x[:10], g1x[:10]) and np.array_equal(g2m[:10], g1m[:10])
    users = [0, 9, 10, 15]
    Xo, mo = sa_batch(inp["X"], inp["offsets"], inp["P"], inp["W_Q"], inp["W_K"], inp["scale"],
                      users=users)
    for b in users:
        assert_user_close(g1x[b], g1m[b], Xo[b], mo[b], "bf16", f"user {b} (first call)")
        assert_user_close(g2x[b], g2m[b], Xo[b], mo[b], "bf16", f"user {b} (second call)")
    assert_total_mass(g2m, inp["offsets"], "bf16")
    cache.close()
    q.close()


def test_cached_forward_rejects_bad_host_offsets():
    import torch
    from sketch_attention_compression_b200 import SAError, SketchCache
    inp = make_inputs([10, 20], 128, 64, "bf16", seed=1)
    q = _query(inp)
    X = torch.from_numpy(inp["X"]).cuda().to(torch.bfloat16)
    cache = SketchCache(64, 128, capacity=4, ttl=60.0)
    keys = [(1, 1, 1, 1), (2, 1, 1, 1)]
    for bad in ([0, 25, 20], [1, 10, 30], [0, 10, 31]):
        with pytest.raises(SAError):
            cache.forward(q, keys, 0.0, X, np.array(bad, dtype=np.int64))
    assert cache.stats()["misses"] == 0  # rejected before any lookup
    # a time that is not finite would break the index's ordering
    offs = np.array([0, 10, 30], dtype=np.int64)
    Xt = torch.zeros((2, 64, 128), dtype=torch.float32, device="cuda")
    m = torch.zeros((2, 64), dtype=torch.float32, device="cuda")
    for now in (float("nan"), float("inf")):
        with pytest.raises(SAError):
            cache.forward(q, keys, now, X, offs)
        with pytest.raises(SAError):
            cache.lookup(keys, now, Xt, m)
        with pytest.raises(SAError):
            cache.insert(keys, now, Xt, m)
    assert cache.stats() == {"entries": 0, "hits": 0, "misses": 0, "evictions": 0}
    cache.close()
    q.close()


@pytest.mark.parametrize("d,D,rows", [(128, 1024, 2 * 300), (64, 256, 129), (128, 256, 1),
                                      (64, 1024, 1000)])
def test_width_adapter_matches_oracle(d, D, rows):
    import torch
    from sketch_attention_compression_b200 import WidthAdapter
    rng = np.random.default_rng(d + D + rows)
    Xt = (rng.standard_normal((rows, d)) * 3.0).astype(np.float32)
    W = (rng.standard_normal((d, D)) / np.sqrt(d)).astype(np.float32)
    ad = WidthAdapter(torch.from_numpy(W).cuda())
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    Y = ad.forward(torch.from_numpy(Xt).cuda(), device_flags=flags)
    torch.cuda.synchronize()
    assert flags.item() == 0
    assert Y.shape == (rows, D) and Y.dtype == torch.bfloat16
    Xb, Wb = round_to_bf16(Xt).astype(np.float64), round_to_bf16(W).astype(np.float64)
    want = width_adapter(Xb, Wb)
    bound = np.abs(Xb) @ np.abs(Wb)
    err = np.abs(Y.double().cpu().numpy() - want)
    assert np.all(err <= 2.0 ** -8 * np.abs(want) + 1e-6 * bound), float(err.max())
    ad.close()
