"""Stateful property test of the host block manager against the oracle
(hypothesis): random sequences of reservations, prompts with prefix reuse,
registrations, forks, releases, matches and host state checkpoints (the
state image saved and loaded into a fresh pool, which carries on) -- edge
cases included (empty prompts, zero-token registrations, full pools) -- with
every status and the whole pool state compared bit-exact after each step.
No GPU."""
import hypothesis.strategies as st
import pytest
from hypothesis import HealthCheck, settings
from hypothesis.stateful import RuleBasedStateMachine, initialize, invariant, rule

import pagedattention_decode_03_b200 as pa
from oracle import Status

from test_host_prefix import Both

SEQS = st.integers(0, 7)
TOKENS = st.lists(st.integers(0, 2), min_size=0, max_size=80)


class PoolMachine(RuleBasedStateMachine):
    @initialize(nb=st.integers(4, 24), B=st.sampled_from([16, 32]))
    def setup(self, nb, B):
        self.x = Both(nb, B, max_seqs=8, mbps=8)
        self.hist = {}

    @rule(s=SEQS, toks=TOKENS)
    def prompt(self, s, toks):
        st_, _ = self.x.reserve_prefix(s, toks)
        if st_ == Status.OK:
            self.hist[s] = list(toks)

    @rule(s=SEQS, k=st.integers(0, 80))
    def register(self, s, k):
        toks = self.hist.get(s, [])[:k]
        self.x.register(s, toks)

    @rule(s=SEQS, toks=st.lists(st.integers(0, 2), min_size=1, max_size=40))
    def grow(self, s, toks):
        cur = self.x.o.lens.get(s, 0)
        if self.x.reserve(s, cur + len(toks)) == Status.OK:
            self.hist[s] = self.hist.get(s, [])[:cur] + list(toks)

    @rule(s=SEQS)
    def reserve_same_length(self, s):
        self.x.reserve(s, self.x.o.lens.get(s, 0))
        self.hist.setdefault(s, [])

    @rule(a=SEQS, b=SEQS)
    def fork(self, a, b):
        if self.x.fork(a, b) == Status.OK:
            self.hist[b] = list(self.hist.get(a, []))

    @rule(s=SEQS)
    def release(self, s):
        if self.x.release(s) == Status.OK:
            self.hist.pop(s, None)

    @rule(toks=TOKENS)
    def match(self, toks):
        self.x.match(toks)

    @rule()
    def checkpoint(self):
        """Carry on in a fresh pool restored from the state image."""
        p = self.x.p
        image = pa.pa_state_save(p)
        fresh = pa.pa_pool_create(num_layers=1, num_kv_heads=1, block_size=p.block_size,
                                  num_blocks=p.num_blocks, max_seqs=p.max_seqs,
                                  max_blocks_per_seq=p.max_blocks_per_seq, host_only=True)
        pa.pa_state_load(fresh, image)
        self.x.p = fresh

    @invariant()
    def same(self):
        if hasattr(self, "x"):
            self.x.same()


@pytest.fixture(scope="module", autouse=True)
def built():
    from pagedattention_decode_03_b200 import build
    build.build()


TestPool = PoolMachine.TestCase
TestPool.settings = settings(max_examples=150, stateful_step_count=40, deadline=None,
                             suppress_health_check=[HealthCheck.too_slow], derandomize=True)
