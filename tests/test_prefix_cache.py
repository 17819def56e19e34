"""Prefix-reuse directory (host C++ in libkda): chained 512-token block hashes, longest cached prefix,
resume at the deepest checkpointed block end, sparse checkpoint plan, LRU slot and block eviction."""
import numpy as np
import pytest

import kda_linear_attention_02_b200 as kda
from kda_linear_attention_02_b200 import build as kbuild

B = kda.KDA_PREFIX_BLOCK


@pytest.fixture(scope="module", autouse=True)
def _lib():
    kbuild.build()


def _fnv1a64(data: bytes) -> int:
    # 64-bit FNV-1a from its published definition: offset basis, then per byte xor and multiply by the prime
    h = 0xCBF29CE484222325
    for b in data:
        h ^= b
        h = (h * 0x100000001B3) & 0xFFFFFFFFFFFFFFFF
    return h


def _chained(tokens, seed):
    out, prev = [], seed
    for b in range(len(tokens) // B):
        blk = np.asarray(tokens[b * B:(b + 1) * B], dtype="<i4").tobytes()
        prev = _fnv1a64(prev.to_bytes(8, "little") + blk)
        out.append(prev)
    return out


def _tokens(n, seed):
    return np.random.default_rng(seed).integers(0, 200_000, size=n, dtype=np.int32)


def test_block_hashes_match_fnv1a_definition():
    t = _tokens(3 * B + 100, 0)
    for seed in (0, 12345, 2 ** 63 + 7):
        assert kda.kda_prefix_block_hashes(t, seed).tolist() == _chained(t, seed)


def test_block_hashes_are_prefix_hashes():
    a = _tokens(6 * B, 1)
    b = a.copy()
    b[3 * B + 17] += 1                                  # change one token of block 3
    ha, hb = kda.kda_prefix_block_hashes(a), kda.kda_prefix_block_hashes(b)
    assert ha[:3].tolist() == hb[:3].tolist()           # blocks before the change agree
    assert all(x != y for x, y in zip(ha[3:], hb[3:]))  # every later block differs (chained)
    assert kda.kda_prefix_block_hashes(a[:4 * B + 511]).tolist() == ha[:4].tolist()   # partial tail ignored
    assert len(kda.kda_prefix_block_hashes(a[:B - 1])) == 0


def test_plan_unit_boundaries_and_last_block():
    c = kda.kda_prefix_cache_create(1000, 8, 4)       # unit = 4 blocks = 2048 tokens
    try:
        assert kda.kda_prefix_cache_plan(c, 10, 0) == [4, 8, 10]
        assert kda.kda_prefix_cache_plan(c, 8, 0) == [4, 8]
        assert kda.kda_prefix_cache_plan(c, 12, 8) == [12]
        assert kda.kda_prefix_cache_plan(c, 13, 5) == [8, 12, 13]
        assert kda.kda_prefix_cache_plan(c, 5, 5) == []
        assert kda.kda_prefix_cache_plan(c, 3, 0) == [3]
    finally:
        kda.kda_prefix_cache_destroy(c)


def _insert_commit(c, h, ends):
    slots = kda.kda_prefix_cache_insert(c, h, ends)
    kda.kda_prefix_cache_commit(c, slots)              # the states have been copied into the slots
    return slots


def _lookup(c, h):
    """A lookup whose pin is released right away (the caller's read of the slot is done)."""
    r = kda.kda_prefix_cache_lookup(c, h)
    kda.kda_prefix_cache_release(c, r[2])
    return r


def test_lookup_resumes_at_deepest_checkpoint_of_shared_prefix():
    c = kda.kda_prefix_cache_create(1000, 8, 4)
    try:
        a = _tokens(10 * B, 2)
        ha = kda.kda_prefix_block_hashes(a)
        assert _lookup(c, ha) == (0, 0, -1)
        ends = kda.kda_prefix_cache_plan(c, 10, 0)
        slots = _insert_commit(c, ha, ends)
        assert ends == [4, 8, 10] and sorted(slots) == [0, 1, 2]
        assert kda.kda_prefix_cache_stats(c) == (10, 3)
        # the same prompt again: everything matches, resume at its end
        assert _lookup(c, ha) == (10, 10, slots[2])
        # shares 9.5 blocks, then diverges: 9 blocks match, the deepest checkpoint inside is block 8
        b = np.concatenate([a[:9 * B + 256], _tokens(3 * B, 3)])
        hb = kda.kda_prefix_block_hashes(b)
        assert _lookup(c, hb) == (9, 8, slots[1])
        ends_b = kda.kda_prefix_cache_plan(c, len(hb), 8)
        assert ends_b == [len(hb)]
        slots_b = _insert_commit(c, hb, ends_b)
        assert slots_b == [3]
        assert _lookup(c, hb) == (len(hb), len(hb), 3)
        # the first prompt again: its ends are stored already, nothing to copy
        assert kda.kda_prefix_cache_insert(c, ha, ends) == [kda.KDA_PREFIX_STORED] * 3
        # an unrelated prompt matches nothing
        assert _lookup(c, kda.kda_prefix_block_hashes(_tokens(4 * B, 4))) == (0, 0, -1)
    finally:
        kda.kda_prefix_cache_destroy(c)


def test_slot_eviction_is_least_recently_used():
    c = kda.kda_prefix_cache_create(1000, 2, 2)        # two slots
    try:
        r = [kda.kda_prefix_block_hashes(_tokens(2 * B, 10 + i)) for i in range(3)]
        assert _insert_commit(c, r[0], [2]) == [0]
        assert _insert_commit(c, r[1], [2]) == [1]
        _lookup(c, r[0])                               # r[0] becomes the most recently used
        assert _insert_commit(c, r[2], [2]) == [1]     # takes r[1]'s slot
        assert _lookup(c, r[1]) == (2, 0, -1)          # hashes kept, checkpoint gone
        assert _lookup(c, r[0]) == (2, 2, 0)
        assert kda.kda_prefix_cache_stats(c) == (6, 2)
    finally:
        kda.kda_prefix_cache_destroy(c)


def test_block_eviction_takes_the_slot_along():
    c = kda.kda_prefix_cache_create(4, 4, 2)           # at most 4 block hashes
    try:
        r0 = kda.kda_prefix_block_hashes(_tokens(2 * B, 20))
        r1 = kda.kda_prefix_block_hashes(_tokens(4 * B, 21))
        assert _insert_commit(c, r0, [2]) == [0]
        # r1's last two blocks evict r0's two (least recently used); r0's slot 0 is freed and handed out first
        assert _insert_commit(c, r1, [2, 4]) == [0, 1]
        assert _lookup(c, r0) == (0, 0, -1)
        assert kda.kda_prefix_cache_stats(c) == (4, 2)
        assert _lookup(c, r1) == (4, 4, 1)
    finally:
        kda.kda_prefix_cache_destroy(c)


def test_pending_slots_are_not_resume_points():
    c = kda.kda_prefix_cache_create(1000, 4, 2)
    try:
        h = kda.kda_prefix_block_hashes(_tokens(6 * B, 40))
        s1 = _insert_commit(c, h[:2], [2])             # block end 2 committed
        slots = kda.kda_prefix_cache_insert(c, h, [2, 4, 6])
        assert slots[0] == kda.KDA_PREFIX_STORED and slots[1] >= 0 and slots[2] >= 0
        # before the copies are committed, the deepest usable checkpoint is the committed one
        assert _lookup(c, h) == (6, 2, s1[0])
        kda.kda_prefix_cache_commit(c, slots[1:2])
        assert _lookup(c, h) == (6, 4, slots[1])
        kda.kda_prefix_cache_abort(c, slots)           # block end 6's copy will not happen
        assert _lookup(c, h) == (6, 4, slots[1])
        assert kda.kda_prefix_cache_stats(c) == (6, 2)
    finally:
        kda.kda_prefix_cache_destroy(c)


def test_pinned_and_pending_slots_are_never_reused():
    c = kda.kda_prefix_cache_create(1000, 2, 2)        # two slots
    try:
        r = [kda.kda_prefix_block_hashes(_tokens(2 * B, 50 + i)) for i in range(4)]
        assert _insert_commit(c, r[0], [2]) == [0]
        m = kda.kda_prefix_cache_lookup(c, r[0])        # slot 0 pinned: a request resumes from it
        assert m == (2, 2, 0)
        assert kda.kda_prefix_cache_insert(c, r[1], [2]) == [1]   # slot 1 pending (not committed)
        # neither the pinned nor the pending slot may be handed to a third request
        assert kda.kda_prefix_cache_insert(c, r[2], [2]) == [kda.KDA_PREFIX_NO_SLOT]
        kda.kda_prefix_cache_release(c, 0)
        # slot 0 is now the least recently used committed, unpinned slot; slot 1 is still pending
        assert kda.kda_prefix_cache_insert(c, r[3], [2]) == [0]
        assert _lookup(c, r[0]) == (2, 0, -1)
        with pytest.raises(kda.KDAError):
            kda.kda_prefix_cache_release(c, 0)        # no pin left to release
    finally:
        kda.kda_prefix_cache_destroy(c)


def test_prefix_cache_argument_errors():
    with pytest.raises(kda.KDAError):
        kda.kda_prefix_cache_create(10, 4, 1)          # unit below 1024 tokens
    with pytest.raises(kda.KDAError):
        kda.kda_prefix_cache_create(10, 4, 13)         # unit above 6144 tokens
    with pytest.raises(kda.KDAError):
        kda.kda_prefix_cache_create(0, 4, 2)
    c = kda.kda_prefix_cache_create(10, 4, 2)
    try:
        h = kda.kda_prefix_block_hashes(_tokens(2 * B, 30))
        with pytest.raises(kda.KDAError):
            kda.kda_prefix_cache_insert(c, h, [3])     # an end past the request
        with pytest.raises(kda.KDAError):
            kda.kda_prefix_cache_plan(c, 2, 3)         # resume past the request
        with pytest.raises(kda.KDAError):
            kda.kda_prefix_cache_commit(c, [4])        # no such slot
        with pytest.raises(kda.KDAError):
            kda.kda_prefix_cache_release(c, 9)
    finally:
        kda.kda_prefix_cache_destroy(c)
