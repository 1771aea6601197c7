"""Host-side checks of the sibling-set planner (pa_plan_siblings): which forked
sequences the decode reads together, from the host block tables alone.  No GPU.

Forked sequences hold their prompt's blocks by reference count ("Managing the
KV Cache", Block Tables and Sharing; "kv-cache-pagedattention-serving", The
bonus: sharing via copy-on-write), so a set's members must start with the same
physical blocks.  The planner is an implementation choice; these tests pin its
stated rules against the tables themselves.
"""
import numpy as np
import pytest

import pagedattention_decode_03_b200 as pa


def host_pool(nb, max_seqs, mbps):
    return pa.pa_pool_create(num_layers=1, num_kv_heads=1, block_size=16, num_blocks=nb,
                             max_seqs=max_seqs, max_blocks_per_seq=mbps, host_only=True)


def tables(pool, seqs):
    return {s: pa.pa_get_seq(pool, s) for s in seqs}   # s -> (len, table)


def check_rules(pool, seqs, group):
    """The planner's stated rules, checked against the tables."""
    set_of, set_cp = pa.pa_plan_siblings(pool, seqs, group)
    t = tables(pool, seqs)
    members = {}
    for i, k in enumerate(set_of):
        if k >= 0:
            members.setdefault(k, []).append(i)
    assert sorted(members) == list(range(len(set_cp)))
    for k, items in members.items():
        cp = set_cp[k]
        assert 2 <= len(items) <= 8 // group
        assert cp >= 2
        first = t[seqs[items[0]]][1]
        for i in items:
            n, tab = t[seqs[i]]
            nb = -(-n // 16)
            assert cp <= nb - 1                       # the last block stays private
            assert tab[:cp] == first[:cp]             # a common run of full blocks
        # the run is as long as the rules allow: it stops where the tables differ
        # or at a member's last block
        caps = [-(-t[seqs[i]][0] // 16) - 1 for i in items]
        if cp < min(caps):
            assert len({tuple(t[seqs[i]][1][: cp + 1]) for i in items}) > 1
    return set_of, set_cp


def parallel_sampling(prompts, samples, plen, grow):
    """`prompts` prompts of `plen` tokens, each forked into `samples` sequences
    that then grow by `grow` tokens (copy-on-write of the shared tail)."""
    n = prompts * samples
    nb_need = prompts * (-(-plen // 16)) + n * (-(-grow // 16) + 2)
    pool = host_pool(nb_need + 8, n, -(-(plen + grow) // 16) + 1)
    for p in range(prompts):
        pa.pa_alloc_blocks(pool, p * samples, plen)
        for c in range(1, samples):
            pa.pa_fork_cow(pool, p * samples, p * samples + c)
    for g in range(grow):
        for s in range(n):
            pa.pa_alloc_blocks(pool, s, plen + g + 1)
    return pool, list(range(n))


def test_parallel_sampling_sets_per_prompt():
    """4 prompts x 8 samples of 2,050 tokens after one step: one set per prompt
    reading the 128 full prompt blocks once (G = 1); pairs for G = 4; none for G = 8."""
    pool, seqs = parallel_sampling(4, 8, 2050, 1)
    set_of, set_cp = check_rules(pool, seqs, 1)
    assert set_cp == [128] * 4
    for p in range(4):
        assert len({set_of[8 * p + c] for c in range(8)}) == 1
    set_of, set_cp = check_rules(pool, seqs, 4)
    assert len(set_cp) == 16 and set(set_cp) == {128}
    assert pa.pa_plan_siblings(pool, seqs, 8) == ([-1] * 32, [])


def test_large_family_splits_into_sets_of_eight():
    pool, seqs = parallel_sampling(1, 12, 300, 5)
    set_of, set_cp = check_rules(pool, seqs, 1)
    sizes = sorted(np.bincount([k for k in set_of if k >= 0]).tolist())
    assert sizes == [4, 8]


def test_before_any_append_the_shared_tail_is_not_read_once():
    """Right after the forks every block is shared, the partial tail too; the
    tail stays per sequence (it is each member's last block)."""
    pool, seqs = parallel_sampling(2, 4, 100, 0)
    set_of, set_cp = check_rules(pool, seqs, 2)
    assert set_cp == [6, 6]                            # 100 tokens = 6 full blocks + 4


def test_short_or_no_common_prefix_forms_no_set():
    pool, seqs = parallel_sampling(1, 3, 20, 30)      # one full shared block only
    assert pa.pa_plan_siblings(pool, seqs, 1) == ([-1, -1, -1], [])
    pool = host_pool(64, 4, 16)
    for s, n in enumerate([200, 200, 33, 1]):          # unrelated sequences
        pa.pa_alloc_blocks(pool, s, n)
    assert pa.pa_plan_siblings(pool, [0, 1, 2, 3], 1) == ([-1] * 4, [])


@pytest.mark.parametrize("seed", range(20))
def test_random_fork_trees_follow_the_rules(seed):
    g = np.random.default_rng([seed, 61])
    max_seqs = 40
    pool = host_pool(2000, max_seqs, 120)
    live = []
    nxt = 0
    for _ in range(int(g.integers(1, 4))):
        pa.pa_alloc_blocks(pool, nxt, int(g.integers(1, 400)))
        live.append(nxt)
        nxt += 1
    for _ in range(int(g.integers(5, 30))):
        op = g.random()
        if op < 0.4 and nxt < max_seqs:
            parent = int(g.choice(live))
            pa.pa_fork_cow(pool, parent, nxt)
            live.append(nxt)
            nxt += 1
        else:
            s = int(g.choice(live))
            n, _ = pa.pa_get_seq(pool, s)
            pa.pa_alloc_blocks(pool, s, n + int(g.integers(1, 40)))
    order = [int(x) for x in g.permutation(live)]
    for group in (1, 2, 4, 8):
        check_rules(pool, order, group)


def test_argument_errors():
    pool, seqs = parallel_sampling(1, 2, 40, 0)
    with pytest.raises(pa.PAError) as e:
        pa.pa_plan_siblings(pool, seqs, 3)
    assert e.value.status == pa.PA_ERR_INVALID_ARG
    with pytest.raises(pa.PAError) as e:
        pa.pa_plan_siblings(pool, [0, 5], 1)
    assert e.value.status in (pa.PA_ERR_NO_SEQ, pa.PA_ERR_INVALID_ARG)
