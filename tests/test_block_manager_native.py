"""The native host block manager (include/block_manager.h, C++ in the library)
against the oracle (oracle/block_manager.py): identical results, call by call,
on seeded random call sequences, plus the pages' scenarios and thread safety.
Host code only: runs without a GPU."""

import random
import threading

import pytest

from oracle.block_manager import BlockManager as Oracle
from oracle.block_manager import BlockManagerError, OutOfBlocks
from paged_kv_cache_463_b200 import binding as b


def _native(nb, bs):
    return b.BlockManager(nb, bs)


def _apply(o, n, op, args):
    """Run one call on both; return both outcomes (value or error class)."""
    def run(fn):
        try:
            return ("ok", fn())
        except OutOfBlocks as e:
            return ("oob", (e.done, e.slots, [tuple(c) for c in e.copies]) if op in ("append", "append_batch") else None)
        except BlockManagerError:
            return ("err", None)
        except b.PagedAttnError as e:
            return ("oob" if e.status == b.PA_ERR_OUT_OF_BLOCKS else "err", None)

    if op == "add":
        return run(lambda: o.add_sequence(*args)), run(lambda: n.add_sequence(*args))
    if op == "free":
        return run(lambda: o.free_sequence(*args)), run(lambda: n.free_sequence(*args))
    if op == "ensure":
        return run(lambda: o.ensure_capacity(*args)), run(lambda: n.ensure_capacity(*args))
    if op == "fork":
        return run(lambda: o.fork(*args)), run(lambda: n.fork(*args))
    if op == "prefix":
        return run(lambda: o.allocate_with_prefix(*args)), run(lambda: n.allocate_with_prefix(*args))
    if op == "evict":
        return run(lambda: o.evict_lru_sequence(*args)), run(lambda: n.evict_lru_sequence(*args))
    if op == "table":
        return run(lambda: o.block_table(*args)), run(lambda: n.block_table(*args))
    if op == "len":
        return run(lambda: o.seq_len(*args)), run(lambda: n.seq_len(*args))
    if op == "batch":
        def nat():
            t, l = n.build_batch(*args)
            return t.tolist(), l.tolist()
        return run(lambda: o.build_batch(*args)), run(nat)
    if op == "append_batch":
        def orc():
            slots, copies = [], []
            for k, sid in enumerate(args[0]):
                try:
                    sl, cp = o.append_tokens(sid, 1)
                except OutOfBlocks:
                    raise OutOfBlocks("oob", k, slots, copies)
                slots += sl
                copies += cp
            return slots, [tuple(c) for c in copies]
        ro = run(orc)
        st, slots, pairs = n.append_batch(args[0])
        sl, pr = slots.tolist(), [tuple(x) for x in pairs.tolist()]
        rn = ("ok", (sl, pr)) if st == b.PA_OK else ("oob", (len(sl), sl, pr))
        return ro, rn
    if op == "append":
        ro = run(lambda: o.append_tokens(*args))
        try:
            st, slots, copies = n.append_tokens(*args)
            rn = ("ok", (slots, copies)) if st == b.PA_OK else ("oob", (len(slots), slots, copies))
        except b.PagedAttnError:
            rn = ("err", None)
        if ro[0] == "ok":
            ro = ("ok", (ro[1][0], [tuple(c) for c in ro[1][1]]))
        return ro, rn
    raise AssertionError(op)


@pytest.mark.parametrize("seed", range(6))
def test_random_calls_match_the_oracle(seed):
    rnd = random.Random(100 + seed)
    nb, bs = rnd.choice([(24, 16), (64, 16), (40, 8)])
    o, n = Oracle(nb, bs), _native(nb, bs)
    live, nxt = [], 0
    for step in range(1500):
        r = rnd.random()
        if r < 0.12 or not live:
            op, args = "add", (nxt,)
        elif r < 0.40:
            op, args = "append", (rnd.choice(live), rnd.randint(1, 3 * bs))
        elif r < 0.48:
            op, args = "fork", (rnd.choice(live), nxt)
        elif r < 0.56:
            op, args = "free", (rnd.choice(live),)
        elif r < 0.62:
            op, args = "ensure", (rnd.choice(live), rnd.randint(0, 5 * bs))
        elif r < 0.74:
            toks = [rnd.randrange(3) for _ in range(rnd.randint(1, 4 * bs))]
            op, args = "prefix", (nxt, toks)
        elif r < 0.78:
            op, args = "evict", (rnd.choice(live + [None]),)
        elif r < 0.84:
            op, args = "table", (rnd.choice(live),)
        elif r < 0.88:
            op, args = "len", (rnd.choice(live + [10 ** 6]),)
        elif r < 0.91:
            k = rnd.randint(1, min(6, len(live)))
            op, args = "batch", (rnd.sample(live, k), rnd.choice([4, 8, 16]))
        elif r < 0.94:
            op, args = "append_batch", (rnd.sample(live, rnd.randint(1, len(live))),)
        else:
            op, args = "add", (rnd.choice(live),)  # duplicate id: an error on both sides
        ro, rn = _apply(o, n, op, args)
        assert ro == rn, (step, op, args, ro, rn)
        if op in ("add", "fork", "prefix") and ro[0] == "ok":
            live.append(nxt)
            nxt += 1
        elif op in ("add", "fork", "prefix"):
            nxt += 1
        if op == "free" and ro[0] == "ok":
            live.remove(args[0])
        if op == "evict" and ro[0] == "ok":
            live.remove(ro[1])
        # native state equals the oracle's (ref counts, free list length, cache size)
        assert n.num_free() == o.num_free()
        assert n.cached_blocks() == o.cached_blocks()
        assert [n.ref_count(x) for x in range(nb)] == o.ref_counts
    n.close()


def test_pages_scenarios_natively():
    """Fork + copy-on-write (Q18) and prefix sharing (Q20) through the C ABI."""
    n = _native(8, 16)
    n.add_sequence(0)
    st, slots, copies = n.append_tokens(0, 40)
    assert st == b.PA_OK and copies == [] and len(slots) == 40
    parent = n.block_table(0)
    n.fork(0, 1)
    assert [n.ref_count(x) for x in parent] == [2, 2, 2]
    st, slots, copies = n.append_tokens(1, 1)
    child = n.block_table(1)
    assert copies == [(parent[2], child[2])] and slots == [child[2] * 16 + 8]
    tables, lens = n.build_batch([0, 1], 4)
    assert tables.tolist() == [parent + [-1], child + [-1]] and lens.tolist() == [40, 41]
    n2 = _native(16, 16)
    m, slots = n2.allocate_with_prefix(5, list(range(40)))
    assert m == 0 and n2.cached_blocks() == 2
    m, slots = n2.allocate_with_prefix(6, list(range(32)) + [9] * 3)
    assert m == 32 and len(slots) == 3 and n2.block_table(6)[:2] == n2.block_table(5)[:2]


def test_errors_natively():
    with pytest.raises(b.PagedAttnError) as e:
        b.BlockManager(0, 16)
    assert e.value.status == b.PA_ERR_INVALID_ARG
    n = _native(2, 16)
    n.add_sequence(1)
    with pytest.raises(b.PagedAttnError) as e:
        n.add_sequence(1)
    assert e.value.status == b.PA_ERR_INVALID_ARG
    with pytest.raises(b.PagedAttnError) as e:
        n.ensure_capacity(1, 48)
    assert e.value.status == b.PA_ERR_OUT_OF_BLOCKS
    assert len(n.block_table(1)) == 2  # blocks allocated before the failure stay
    st, slots, copies = n.append_tokens(1, 40)
    assert st == b.PA_ERR_OUT_OF_BLOCKS and len(slots) == 32
    with pytest.raises(b.PagedAttnError) as e:
        n.seq_len(99)
    assert e.value.status == b.PA_ERR_INVALID_ARG
    with pytest.raises(b.PagedAttnError) as e:
        n.build_batch([1], 1)  # table longer than bt_stride
    assert e.value.status == b.PA_ERR_INVALID_ARG


def test_thread_safety():
    """Threads appending to their own sequences concurrently: every block is
    handed out once and the counts add up afterwards."""
    n = _native(4096, 16)
    errors = []

    def worker(t):
        try:
            for k in range(40):
                sid = t * 1000 + k
                n.add_sequence(sid)
                st, slots, _ = n.append_tokens(sid, 33)
                assert st == b.PA_OK and len(slots) == 33
                if k % 3 == 0:
                    n.free_sequence(sid)
        except Exception as e:  # pragma: no cover - reported below
            errors.append(e)

    threads = [threading.Thread(target=worker, args=(t,)) for t in range(8)]
    for th in threads:
        th.start()
    for th in threads:
        th.join()
    assert not errors
    held = set()
    live = [t * 1000 + k for t in range(8) for k in range(40) if k % 3 != 0]
    for sid in live:
        tb = n.block_table(sid)
        assert len(tb) == 3 and not (set(tb) & held)
        held |= set(tb)
    assert n.num_free() == 4096 - len(held)
