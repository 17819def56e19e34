"""Randomised request streams through the prefix-reuse directory (host C++), checked against invariants
that its contract fixes rather than against a second implementation of it:
  * a lookup's resume point lies inside its matched prefix, and the slot it names is the one that the
    latest insert handed to that block end (a slot is never shared by two live entries);
  * a plan's ends are increasing, lie past the resume point and end at the request's last block;
  * a request no longer than the directory is found whole right after it is inserted (an insert evicts
    only entries that the same request has not touched yet);
  * the directory never holds more hashes or slots than it was created with.
Requests are drawn as branches of a few shared base token streams, so prefixes overlap."""
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
                    st.integers(0, 2 ** 31 - 1))          # seed of the own blocks


@settings(max_examples=150, deadline=None, suppress_health_check=[HealthCheck.too_slow])
@given(max_blocks=st.integers(1, 24), n_slots=st.integers(0, 6), unit=st.integers(2, 12),
       stream=st.lists(request, min_size=1, max_size=25))
def test_random_request_streams_keep_the_invariants(max_blocks, n_slots, unit, stream):
    c = kda.kda_prefix_cache_create(max_blocks, n_slots, unit)
    owner = {}   # slot -> hash of the block end it was last handed to
    try:
        for base, shared, own, seed in stream:
            toks = np.concatenate([BASES[base][:shared * B],
                                   np.random.default_rng(seed).integers(0, 200_000, size=own * B, dtype=np.int32)])
            h = kda.kda_prefix_block_hashes(toks)
            n = len(h)
            m, r, slot = kda.kda_prefix_cache_lookup(c, h)
            assert 0 <= r <= m <= n
            if r > 0:
                assert 0 <= slot < n_slots and owner.get(slot) == int(h[r - 1])
            else:
                assert slot == -1
            ends = kda.kda_prefix_cache_plan(c, n, r)
            assert all(a < b for a, b in zip(ends, ends[1:]))
            assert all(r < e <= n for e in ends)
            assert (ends[-1] == n) if n > r else ends == []
            assert all(e % unit == 0 for e in ends[:-1])
            slots = kda.kda_prefix_cache_insert(c, h, ends)
            assert len(slots) == len(ends)
            got = [s for s in slots if s >= 0]
            assert len(set(got)) == len(got) and all(0 <= s < n_slots for s in got)
            for e, s in zip(ends, slots):
                if s >= 0:
                    owner[s] = int(h[e - 1])
            nb, ns = kda.kda_prefix_cache_stats(c)
            assert nb <= max_blocks and 0 <= ns <= n_slots
            if 0 < n <= max_blocks:
                m2, r2, s2 = kda.kda_prefix_cache_lookup(c, h)
                assert m2 == n
                assert r2 == 0 or owner.get(s2) == int(h[r2 - 1])
    finally:
        kda.kda_prefix_cache_destroy(c)
