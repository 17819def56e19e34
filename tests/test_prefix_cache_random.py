"""Randomised request streams through the prefix-reuse directory (host C++), checked against invariants
that its contract fixes rather than against a second implementation of it:
  * a lookup's resume point lies inside its matched prefix, and the slot it names is the one that the
    latest insert handed to that block end and whose copy has been committed (never a pending slot);
  * an insert never hands out a slot that an unreleased lookup has pinned or that another request's
    uncommitted copy holds (a slot is never shared by two live entries);
  * a plan's ends are increasing, lie past the resume point and end at the request's last block;
  * a request no longer than the directory is found whole right after it is inserted when no other
    request is in flight (an insert evicts only entries that the same request has not touched yet, and
    never one whose slot is pending or pinned);
  * the directory never holds more hashes or slots than it was created with.
Requests are drawn as branches of a few shared base token streams, so prefixes overlap.  Several
requests are in flight at once: each one looks up (pinning its resume slot), inserts (its new slots
pending), and finishes later -- committing or abandoning its copies and releasing its pin -- in an
order drawn with the stream, so lookups and inserts of other requests fall between insert and commit."""
import numpy as np
import pytest
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import kda_linear_attention_02_b200 as kda
from kda_linear_attention_02_b200 import build as kbuild

B = kda.KDA_PREFIX_BLOCK
BASES = [np.random.default_rng(100 + i).integers(0, 200_000, size=12 * B, dtype=np.int32) for i in range(3)]


@pytest.fixture(scope="module", autouse=True)
def _lib():
    kbuild.build()


request = st.tuples(st.integers(0, len(BASES) - 1),     # base stream
                    st.integers(0, 12),                   # blocks shared with it
                    st.integers(0, 4),                    # own blocks after the branch point
                    st.integers(0, 2 ** 31 - 1),          # seed of the own blocks
                    st.integers(0, 3),                    # requests to finish before this one starts
                    st.booleans())                        # commit (True) or abandon its copies


@settings(max_examples=200, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(max_blocks=st.integers(1, 24), n_slots=st.integers(0, 6), unit=st.integers(2, 12),
       stream=st.lists(request, min_size=1, max_size=25))
def test_random_request_streams_keep_the_invariants(max_blocks, n_slots, unit, stream):
    c = kda.kda_prefix_cache_create(max_blocks, n_slots, unit)
    owner = {}        # slot -> hash of the block end its committed copy belongs to
    flight = []       # requests in flight: (pinned slot, [(slot, hash) pending], commit?)
    pending = {}      # slot -> hash, for slots whose copies are in flight

    def finish(req):
        pin, mine, commit = req
        slots = [s for s, _ in mine]
        for s, h in mine:
            del pending[s]
        if commit:
            kda.kda_prefix_cache_commit(c, slots)
            for s, h in mine:
                owner[s] = h
        else:
            kda.kda_prefix_cache_abort(c, slots)
            for s in slots:
                owner.pop(s, None)
        kda.kda_prefix_cache_release(c, pin)

    try:
        for base, shared, own, seed, n_finish, commit in stream:
            for _ in range(min(n_finish, len(flight))):
                finish(flight.pop(0))
            toks = np.concatenate([BASES[base][:shared * B],
                                   np.random.default_rng(seed).integers(0, 200_000, size=own * B, dtype=np.int32)])
            h = kda.kda_prefix_block_hashes(toks)
            n = len(h)
            m, r, slot = kda.kda_prefix_cache_lookup(c, h)
            assert 0 <= r <= m <= n
            if r > 0:
                assert 0 <= slot < n_slots and slot not in pending and owner.get(slot) == int(h[r - 1])
            else:
                assert slot == -1
            ends = kda.kda_prefix_cache_plan(c, n, r)
            assert all(a < b for a, b in zip(ends, ends[1:]))
            assert all(r < e <= n for e in ends)
            assert (ends[-1] == n) if n > r else ends == []
            assert all(e % unit == 0 for e in ends[:-1])
            pinned = {p for p, _, _ in flight if p >= 0} | ({slot} if slot >= 0 else set())
            slots = kda.kda_prefix_cache_insert(c, h, ends)
            assert len(slots) == len(ends)
            got = [s for s in slots if s >= 0]
            assert len(set(got)) == len(got) and all(0 <= s < n_slots for s in got)
            assert not (set(got) & pinned) and not (set(got) & set(pending))
            assert all(s in (kda.KDA_PREFIX_NO_SLOT, kda.KDA_PREFIX_STORED) for s in slots if s < 0)
            mine = [(s, int(h[e - 1])) for e, s in zip(ends, slots) if s >= 0]
            for s, hh in mine:
                owner.pop(s, None)                   # the slot's old checkpoint is gone
                pending[s] = hh
            flight.append((slot, mine, commit))
            nb, ns = kda.kda_prefix_cache_stats(c)
            assert nb <= max_blocks and 0 <= ns <= n_slots
            if 0 < n <= max_blocks and len(flight) == 1:   # no other request holds busy slots
                m2, r2, s2 = kda.kda_prefix_cache_lookup(c, h)
                assert m2 == n
                assert r2 == 0 or (s2 not in pending and owner.get(s2) == int(h[r2 - 1]))
                kda.kda_prefix_cache_release(c, s2)
        while flight:
            finish(flight.pop(0))
        # every pin released and every copy settled: each slot in use holds a committed copy
        nb, ns = kda.kda_prefix_cache_stats(c)
        assert ns <= len(owner)
    finally:
        kda.kda_prefix_cache_destroy(c)
