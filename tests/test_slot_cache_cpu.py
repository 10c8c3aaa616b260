"""mlora_slot_cache through the C ABI (host only, no GPU): which adapter each slot
holds, pins of in-flight batches, least-recently-used eviction among unpinned slots."""
import random
import threading

import pytest

import segmented_rank_gemm_02_b200 as mlora


def test_hits_misses_and_fresh_slots_first():
    c = mlora.SlotCache(3)
    assert c.acquire(100) == (0, True, None)
    assert c.acquire(200) == (1, True, None)
    assert c.acquire(100) == (0, False, None)          # hit: pinned twice now
    assert c.lookup(200) == 1 and c.lookup(999) == -1
    assert c.stats() == (1, 2, 0)


def test_lru_among_unpinned_slots():
    c = mlora.SlotCache(3)
    for a in (1, 2, 3):
        c.acquire(a)
    c.release(1)                                        # released: slot 1, slot 2, slot 0
    c.release(2)
    c.release(0)
    # least recently released first: slot 1 (adapter 2), then slot 2 (adapter 3)
    assert c.acquire(4) == (1, True, 2)
    assert c.acquire(5) == (2, True, 3)
    assert c.acquire(1) == (0, False, None)             # adapter 1 was never evicted
    assert c.lookup(2) == -1 and c.lookup(3) == -1
    assert c.stats()[2] == 2


def test_pinned_slots_are_never_evicted():
    c = mlora.SlotCache(2)
    c.acquire(10)
    c.acquire(20)
    with pytest.raises(mlora.MloraError) as e:
        c.acquire(30)
    assert e.value.status == mlora.ERR_NO_SLOT
    c.release(1)
    assert c.acquire(30) == (1, True, 20)
    assert c.lookup(10) == 0


def test_release_errors_and_invalidate():
    c = mlora.SlotCache(2)
    with pytest.raises(mlora.MloraError):
        c.release(0)                                    # not pinned
    with pytest.raises(mlora.MloraError):
        c.release(5)                                    # out of range
    s, load, _ = c.acquire(7)
    c.invalidate(s)                                     # e.g. its load failed
    assert c.lookup(7) == -1
    assert c.acquire(7)[1] is True                      # a new miss, in a fresh slot
    c.release(s)
    # an emptied unpinned slot is reused before a slot holding an adapter
    other = 1 - s
    c.release(other)
    assert c.acquire(8)[0] == s


def test_against_a_reference_model():
    """Random acquire / release sequences agree with a plain Python model."""
    rng = random.Random(3)
    n = 5
    c = mlora.SlotCache(n)
    holder = [None] * n            # adapter per slot
    pins = [0] * n
    order = []                     # unpinned used slots, least recent first
    fresh = list(range(n))
    for _ in range(2000):
        if rng.random() < 0.55:
            a = rng.randrange(12)
            if a in holder:
                s = holder.index(a)
                if s in order:
                    order.remove(s)
                pins[s] += 1
                assert c.acquire(a) == (s, False, None)
            elif fresh or order:
                s = fresh.pop(0) if fresh else order.pop(0)
                ev = holder[s]
                holder[s] = a
                pins[s] = 1
                assert c.acquire(a) == (s, True, ev)
            else:
                with pytest.raises(mlora.MloraError):
                    c.acquire(a)
        else:
            pinned = [s for s in range(n) if pins[s] > 0]
            if not pinned:
                continue
            s = rng.choice(pinned)
            pins[s] -= 1
            if pins[s] == 0:
                order.append(s)
            c.release(s)


def test_threads_share_one_cache():
    c = mlora.SlotCache(8)
    errors = []

    def worker(seed):
        rng = random.Random(seed)
        try:
            for _ in range(500):
                try:
                    s, _, _ = c.acquire(rng.randrange(20))
                except mlora.MloraError as e:
                    assert e.status == mlora.ERR_NO_SLOT
                    continue
                c.release(s)
        except Exception as e:  # pragma: no cover
            errors.append(e)

    ts = [threading.Thread(target=worker, args=(i,)) for i in range(6)]
    for t in ts:
        t.start()
    for t in ts:
        t.join()
    assert not errors
    hits, misses, evictions = c.stats()
    assert hits + misses > 0 and evictions <= misses
