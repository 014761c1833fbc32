"""CPU tests of the host page bookkeeping (include/gqa_pager.h): each call's effect,
all-or-nothing failures, and a long random run against a plain Python model plus the
invariants that hold for any allocation policy (every page owned once; a slot's pages
cover exactly ceil(len / page_size) blocks)."""
import random

import pytest
import torch

import gqa_decode_attention_04_b200 as gq

OUT_OF_PAGES, INVALID = -6, -1


def _state(p: gq.Pager):
    bt, lens = p.gather(list(range(p.max_seqs)))
    return bt.clone(), lens.clone(), p.free_pages


def _check_invariants(p: gq.Pager):
    bt, lens, free = _state(p)
    owned = []
    for s in range(p.max_seqs):
        nb = -(-int(lens[s]) // p.page_size)
        row = bt[s].tolist()
        assert all(x >= 0 for x in row[:nb]) and all(x == -1 for x in row[nb:]), (s, row, int(lens[s]))
        owned += row[:nb]
    assert len(owned) == len(set(owned)), "a page owned twice"
    assert all(0 <= x < p.num_pages for x in owned)
    assert len(owned) + free == p.num_pages


def test_fresh_pager_is_empty():
    p = gq.Pager(num_pages=10, page_size=16, max_seqs=3, max_blocks_per_seq=4)
    bt, lens = p.gather([2, 0])
    assert bt.shape == (2, 4) and (bt == -1).all() and (lens == 0).all()
    assert p.free_pages == 10 and p.seq_len(1) == 0
    _check_invariants(p)


def test_extend_takes_pages_in_order_and_only_when_a_block_starts():
    p = gq.Pager(num_pages=8, page_size=16, max_seqs=2, max_blocks_per_seq=4)
    p.extend(0, 17)                 # blocks 0, 1
    p.extend(1, 16)                 # block 0 exactly full
    p.extend(0, 15)                 # 32 tokens: still 2 blocks
    bt, lens = p.gather([0, 1])
    assert bt[0].tolist() == [0, 1, -1, -1] and bt[1].tolist() == [2, -1, -1, -1]
    assert lens.tolist() == [32, 16] and p.free_pages == 5
    p.extend(1, 0)                  # no-op
    assert p.free_pages == 5
    _check_invariants(p)


def test_step_reports_positions_and_lengths():
    p = gq.Pager(num_pages=8, page_size=4, max_seqs=3, max_blocks_per_seq=4)
    p.extend(0, 4)
    p.extend(2, 2)
    pos, lens = p.step([2, 0, 1])
    assert pos.tolist() == [2, 4, 0] and lens.tolist() == [3, 5, 1]
    bt, _ = p.gather([0, 1, 2])
    # slot 0 crossed into block 1, slot 1 started block 0, slot 2 stayed in its block
    assert bt[0].tolist()[:2] == [0, 2] and bt[1].tolist()[0] == 3 and bt[2].tolist()[:2] == [1, -1]
    assert p.free_pages == 4
    _check_invariants(p)


def test_failed_calls_change_nothing():
    p = gq.Pager(num_pages=3, page_size=4, max_seqs=3, max_blocks_per_seq=2)
    p.extend(0, 4)
    p.extend(1, 4)
    p.extend(2, 3)
    before = _state(p)
    cases = [
        (lambda: p.step([0, 1]), OUT_OF_PAGES),     # needs 2 pages, 0 free
        (lambda: p.step([2, 2]), INVALID),          # slot listed twice
        (lambda: p.step([2, 5]), INVALID),          # slot out of range
        (lambda: p.extend(0, 5), INVALID),          # 9 tokens > 2 blocks of 4
        (lambda: p.extend(2, 2), OUT_OF_PAGES),
        (lambda: p.extend(1, -1), INVALID),
        (lambda: p.truncate(2, 4), INVALID),        # longer than the slot
        (lambda: p.gather([0, 3]), INVALID),
    ]
    for call, status in cases:
        with pytest.raises(gq.GQAError) as e:
            call()
        assert e.value.status == status, e.value
        now = _state(p)
        assert torch.equal(now[0], before[0]) and torch.equal(now[1], before[1]) and now[2] == before[2]
    # the step that failed on a duplicate left no mark behind: the same slot steps fine now
    p.truncate(0, 0)
    pos, lens = p.step([2])
    assert pos.tolist() == [3] and lens.tolist() == [4]


def test_truncate_frees_whole_blocks_and_pages_are_reused_last_freed_first():
    p = gq.Pager(num_pages=6, page_size=4, max_seqs=2, max_blocks_per_seq=3)
    p.extend(0, 12)                 # pages 0, 1, 2
    p.truncate(0, 5)                # keeps blocks 0, 1; frees page 2
    assert p.free_pages == 4 and p.gather([0])[0][0].tolist() == [0, 1, -1]
    p.release(0)                    # frees 1, then 0 (0 ends on top)
    assert p.free_pages == 6 and p.seq_len(0) == 0
    p.extend(1, 9)
    assert p.gather([1])[0][0].tolist() == [0, 1, 2]
    _check_invariants(p)


def test_zero_slots_and_zero_pages():
    p = gq.Pager(num_pages=0, page_size=16, max_seqs=1, max_blocks_per_seq=1)
    with pytest.raises(gq.GQAError) as e:
        p.extend(0, 1)
    assert e.value.status == OUT_OF_PAGES
    pos, lens = p.step([])
    assert pos.numel() == 0 and lens.numel() == 0
    with pytest.raises(gq.GQAError):
        gq.Pager(num_pages=4, page_size=0, max_seqs=1, max_blocks_per_seq=1)
    with pytest.raises(gq.GQAError):
        gq.Pager(num_pages=4, page_size=16, max_seqs=1, max_blocks_per_seq=0)


class _Model:
    """The header's allocation policy written out in Python: a stack of free pages (page 0
    on top at the start; pages freed in reverse block order) and per-slot page lists."""

    def __init__(self, num_pages, ps, max_seqs, mb):
        self.free = list(range(num_pages - 1, -1, -1))
        self.ps, self.mb = ps, mb
        self.pages = [[] for _ in range(max_seqs)]
        self.lens = [0] * max_seqs

    def _need(self, s, new_len):
        nb = -(-new_len // self.ps)
        return None if nb > self.mb else nb - len(self.pages[s])

    def extend(self, s, n):
        need = self._need(s, self.lens[s] + n)
        if need is None:
            return INVALID
        if need > len(self.free):
            return OUT_OF_PAGES
        for _ in range(need):
            self.pages[s].append(self.free.pop())
        self.lens[s] += n
        return 0

    def step(self, seqs):
        if len(set(seqs)) != len(seqs):
            return INVALID, None
        needs = [self._need(s, self.lens[s] + 1) for s in seqs]
        if any(n is None for n in needs):
            return INVALID, None
        if sum(needs) > len(self.free):
            return OUT_OF_PAGES, None
        pos = []
        for s in seqs:
            pos.append(self.lens[s])
            self.extend(s, 1)
        return 0, pos

    def truncate(self, s, new_len):
        nb = -(-new_len // self.ps)
        while len(self.pages[s]) > nb:
            self.free.append(self.pages[s].pop())
        self.lens[s] = new_len
        return 0


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_random_operations_match_the_model(seed):
    rng = random.Random(seed)
    P, ps, S, MB = 40, rng.choice([1, 4, 16]), 6, 12
    p, m = gq.Pager(P, ps, S, MB), _Model(P, ps, S, MB)
    for it in range(600):
        op = rng.random()
        if op < 0.35:
            seqs = rng.sample(range(S), rng.randint(0, S))
            if rng.random() < 0.1 and seqs:
                seqs.append(seqs[0])
            st, pos = m.step(seqs)
            try:
                got_pos, got_lens = p.step(seqs)
                assert st == 0 and got_pos.tolist() == pos
                assert got_lens.tolist() == [x + 1 for x in pos]
            except gq.GQAError as e:
                assert e.status == st and st != 0
        elif op < 0.65:
            s, n = rng.randrange(S), rng.randint(0, 3 * ps)
            st = m.extend(s, n)
            try:
                p.extend(s, n)
                assert st == 0
            except gq.GQAError as e:
                assert e.status == st and st != 0
        else:
            s = rng.randrange(S)
            new_len = rng.randint(0, m.lens[s])
            m.truncate(s, new_len)
            p.truncate(s, new_len)
        bt, lens, free = _state(p)
        assert lens.tolist() == m.lens and free == len(m.free)
        for s in range(S):
            assert bt[s].tolist() == m.pages[s] + [-1] * (MB - len(m.pages[s]))
        if it % 50 == 0:
            _check_invariants(p)
