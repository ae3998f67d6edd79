"""The host block manager (pa_block_manager.h) against the pages and the plain-Python model.

CPU only.  Three kinds of checks:
  * pins from the pages: a 47-token request takes 3 blocks of 16 ("PagedAttention"
    digest, "PagedAttention in one picture"); the block-size-4 page map of the
    "LLM Inference Visualizer" ("How paging grows") comes out of one allocation
    history; a fork shares blocks and a write into a shared block clones it first
    (digest, "Copy-on-write: when two requests share a prefix");
  * operation by operation, the C++ manager equals oracle/block_model.py on seeded
    random workloads (slots, copy pairs, swap pairs, free counts, references,
    tables), with requests evicted to a host pool and brought back;
  * a data-level invariant that holds for any correct manager: with every token
    written to its slot and every copy applied, each request reads back exactly its
    own token history through its block table -- its prefix as it was at the fork,
    then its own tokens -- whatever the other requests wrote, and after a round
    trip through the host pool.
"""

import json
import os

import numpy as np
import pytest

from oracle.block_model import BlockModel, NoBlocks

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _pa():
    import paged_kv_cache_362_b200 as pa

    return pa


def test_47_tokens_take_three_blocks():
    g = json.load(open(os.path.join(GOLDEN, "p2_block_rounding.json")))
    pa = _pa()
    for bm in (pa.BlockManager(10, g["block_size"]), BlockModel(10, g["block_size"])):
        slots = bm.add_sequence(7, g["tokens"])
        free = bm.num_free_blocks if isinstance(bm, pa.BlockManager) else len(bm.free)
        assert 10 - free == g["blocks"]
        assert list(slots) == list(range(g["tokens"]))            # a fresh pool: blocks 0, 1, 2 in order
        assert g["blocks"] * g["block_size"] - g["tokens"] <= g["max_waste_tokens"]


def test_visualizer_page_map_from_one_history():
    """Requests A, B, C and a request D that later finishes, growing in turn, reproduce the
    diagram's page map (the history is this test's construction; the pages show the end state)."""
    g = json.load(open(os.path.join(GOLDEN, "p3_block_size4.json")))
    bs = g["block_size"]
    ids = {"A": 1, "B": 2, "C": 3, "D": 4}
    # block allocations in page order 0..11: A B D A C D B A D C B D
    order = "ABDACDBADCBD"
    pa = _pa()
    bm = pa.BlockManager(12, bs)
    model = BlockModel(12, bs)
    for r, sid in ids.items():
        bm.add_sequence(sid, 0)
        model.add_sequence(sid, 0)
    length = {r: 0 for r in ids}
    for r in order:
        # grow the request until it needs its next block, then take one token in it
        while length[r] % bs != 0:
            bm.append_tokens([ids[r]])
            model.append_tokens([ids[r]])
            length[r] += 1
        bm.append_tokens([ids[r]])
        model.append_tokens([ids[r]])
        length[r] += 1
    # A holds 9 tokens in the diagram: 8 full slots and 1 in its third block
    assert length["A"] == len(g["tokens"])
    bm.free_sequence(ids["D"])
    model.free_sequence(ids["D"])
    bt, cl = bm.block_tables([ids["A"], ids["B"], ids["C"]], 3)
    pages = {}
    for r, row in zip("ABC", bt):
        for j, b in enumerate(row):
            if b >= 0:
                pages[str(int(b))] = f"{r}{j}"
    expect = {k: v for k, v in g["physical_pages"].items() if v is not None}
    assert pages == expect
    assert [g["logical_to_physical"][f"A{j}"] for j in range(3)] == list(bt[0])
    assert 3 * bs - int(cl[0]) == g["empty_slots_in_last_block"]
    assert bm.num_free_blocks == 4 and sorted(model.free) == [2, 5, 8, 11]


def test_fork_shares_and_copy_on_write_clones():
    pa = _pa()
    bm = pa.BlockManager(16, 16)
    bm.add_sequence(1, 40)                        # blocks 0, 1, 2 (2 holds 8 tokens)
    bm.fork(1, 2)
    assert [bm.ref_count(b) for b in range(3)] == [2, 2, 2]
    slots, pairs = bm.append_tokens([2])          # the child writes into the shared partial block
    assert pairs.tolist() == [[2, 3]]             # cloned first: block 3 is the child's copy
    assert slots.tolist() == [3 * 16 + 8]
    assert [bm.ref_count(b) for b in range(4)] == [2, 2, 1, 1]
    slots, pairs = bm.append_tokens([1])          # the parent now owns block 2 alone: written in place
    assert pairs.size == 0 and slots.tolist() == [2 * 16 + 8]
    # a fork at a block boundary needs no copy: the next token opens a fresh block
    bm.add_sequence(5, 32)                        # blocks 4, 5 (full)
    bm.fork(5, 6)
    slots, pairs = bm.append_tokens([6, 5])
    assert pairs.size == 0 and slots.tolist() == [6 * 16, 7 * 16]
    assert bm.ref_count(4) == 2 and bm.ref_count(5) == 2


def test_no_blocks_changes_nothing():
    pa = _pa()
    bm = pa.BlockManager(4, 16)
    bm.add_sequence(1, 48)                        # blocks 0..2
    bm.fork(1, 2)
    bm.fork(1, 3)
    before = [bm.ref_count(b) for b in range(4)], bm.num_free_blocks
    # three sequences each open a fresh block: three needed, one free
    with pytest.raises(pa.PagedAttentionError) as e:
        bm.append_tokens([1, 2, 3])
    assert e.value.code == pa.PA_ERR_NO_BLOCKS
    assert ([bm.ref_count(b) for b in range(4)], bm.num_free_blocks) == before
    assert bm.sequence_length(1) == 48 and bm.sequence_blocks(2) == 3
    with pytest.raises(pa.PagedAttentionError):
        bm.add_sequence(9, 33)                    # 3 blocks, 1 free
    assert bm.num_sequences == 3


def test_exact_accounting_when_sharers_append_together():
    """Two sequences share a partial block and both append: one copy, the other writes in place."""
    pa = _pa()
    bm = pa.BlockManager(2, 16)
    bm.add_sequence(1, 8)                         # block 0
    bm.fork(1, 2)
    slots, pairs = bm.append_tokens([1, 2])       # one free block is enough
    assert pairs.tolist() == [[0, 1]]
    assert slots.tolist() == [1 * 16 + 8, 0 * 16 + 8]


def test_swap_moves_private_blocks_and_keeps_shared_ones():
    """Eviction moves only what the request alone holds; its shared prefix stays on the device."""
    pa = _pa()
    bm = pa.BlockManager(16, 16, 8)
    bm.add_sequence(1, 40)                        # blocks 0, 1, 2
    bm.fork(1, 2)
    bm.append_tokens([2])                         # 2 copies block 2 -> 3; shares 0 and 1
    out = bm.swap_out(2)
    assert out.tolist() == [[3, 0]]               # only the private block, to host block 0
    assert bm.is_swapped(2) and bm.ref_count(0) == 2 and bm.ref_count(3) == 0
    with pytest.raises(pa.PagedAttentionError):
        bm.append_tokens([2])                     # no appends while evicted
    with pytest.raises(pa.PagedAttentionError):
        bm.block_tables([2], 4)
    back = bm.swap_in(2)
    assert back.tolist() == [[0, 3]]              # the freed block 3 is handed out again
    bt, cl = bm.block_tables([2], 4)
    assert bt.tolist() == [[0, 1, 3, -1]] and cl.tolist() == [41]
    assert bm.num_free_host_blocks == 8
    bm2 = pa.BlockManager(4, 16, 0)               # no host pool: nothing can be evicted
    bm2.add_sequence(1, 5)
    with pytest.raises(pa.PagedAttentionError) as e:
        bm2.swap_out(1)
    assert e.value.code == pa.PA_ERR_NO_BLOCKS


def test_argument_errors():
    pa = _pa()
    bm = pa.BlockManager(8, 16)
    bm.add_sequence(1, 3)
    for call in (lambda: bm.add_sequence(1, 3), lambda: bm.fork(9, 10), lambda: bm.fork(1, 1),
                 lambda: bm.append_tokens([42]), lambda: bm.free_sequence(42),
                 lambda: bm.block_tables([1], 0)):
        with pytest.raises(pa.PagedAttentionError) as e:
            call()
        assert e.value.code == pa.PA_ERR_INVALID_ARG
    with pytest.raises(pa.PagedAttentionError):
        pa.BlockManager(0, 16)


def _random_ops(rng, steps):
    """A seeded serving-like history: prompts, forks (shared prefixes), decode steps, finishes."""
    live, next_id = [], 0
    for _ in range(steps):
        r = rng.random()
        if r < 0.2 or not live:
            yield ("add", next_id, int(rng.integers(0, 70)))
            live.append(next_id)
            next_id += 1
        elif r < 0.35:
            parent = int(rng.choice(live))
            yield ("fork", parent, next_id)
            live.append(next_id)
            next_id += 1
        elif r < 0.78:
            k = int(rng.integers(1, min(len(live), 12) + 1))
            yield ("append", [int(x) for x in rng.choice(live, size=k, replace=True)])
        elif r < 0.85:
            yield ("swap", int(rng.choice(live)))
        else:
            sid = int(rng.choice(live))
            live.remove(sid)
            yield ("free", sid)


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
@pytest.mark.parametrize("block_size", [16, 4])
def test_matches_model_and_keeps_every_history(seed, block_size):
    pa = _pa()
    nb, nh = 48, 24
    bm, model = pa.BlockManager(nb, block_size, nh), BlockModel(nb, block_size, nh)
    rng = np.random.default_rng(seed)
    pool = np.full(nb * block_size, -1, dtype=np.int64)     # token written in each slot
    host = np.full(nh * block_size, -1, dtype=np.int64)     # the host pool, for swapped-out blocks
    history: dict[int, list[int]] = {}
    swapped: set[int] = set()

    def move(src, dst, pairs):
        for a, b in pairs:
            dst[b * block_size:(b + 1) * block_size] = src[a * block_size:(a + 1) * block_size]

    token = 0
    for op in _random_ops(rng, 400):
        if op[0] == "add":
            _, sid, n = op
            try:
                exp = model.add_sequence(sid, n)
            except NoBlocks:
                with pytest.raises(pa.PagedAttentionError) as e:
                    bm.add_sequence(sid, n)
                assert e.value.code == pa.PA_ERR_NO_BLOCKS
                continue
            got = bm.add_sequence(sid, n)
            assert got.tolist() == exp
            toks = list(range(token, token + n))
            token += n
            pool[got] = toks
            history[sid] = toks
        elif op[0] == "swap":
            _, sid = op
            if sid not in history:
                continue
            if sid in swapped:
                try:
                    exp = model.swap_in(sid)
                except NoBlocks:
                    with pytest.raises(pa.PagedAttentionError) as e:
                        bm.swap_in(sid)
                    assert e.value.code == pa.PA_ERR_NO_BLOCKS
                    continue
                got = bm.swap_in(sid)
                assert [tuple(p) for p in got.tolist()] == exp
                move(host, pool, got)
                swapped.discard(sid)
            else:
                try:
                    exp = model.swap_out(sid)
                except NoBlocks:
                    with pytest.raises(pa.PagedAttentionError) as e:
                        bm.swap_out(sid)
                    assert e.value.code == pa.PA_ERR_NO_BLOCKS
                    continue
                got = bm.swap_out(sid)
                assert [tuple(p) for p in got.tolist()] == exp
                move(pool, host, got)
                # the freed device blocks are written by others from now on
                for d, _ in got.tolist():
                    pool[d * block_size:(d + 1) * block_size] = -7
                swapped.add(sid)
            assert bm.is_swapped(sid) == (sid in swapped)
        elif op[0] == "fork":
            _, parent, child = op
            if parent not in history or parent in swapped:
                continue
            model.fork(parent, child)
            bm.fork(parent, child)
            history[child] = list(history[parent])
        elif op[0] == "append":
            sids = [s for s in op[1] if s in history and s not in swapped]
            if not sids:
                continue
            try:
                exp_slots, exp_pairs = model.append_tokens(sids)
            except NoBlocks:
                with pytest.raises(pa.PagedAttentionError) as e:
                    bm.append_tokens(sids)
                assert e.value.code == pa.PA_ERR_NO_BLOCKS
                continue
            slots, pairs = bm.append_tokens(sids)
            assert slots.tolist() == exp_slots
            assert [tuple(p) for p in pairs.tolist()] == exp_pairs
            # copies first (what pa_copy_blocks does), then the new tokens (pa_reshape_and_cache)
            for src, dst in pairs.tolist():
                pool[dst * block_size:(dst + 1) * block_size] = pool[src * block_size:(src + 1) * block_size]
            for s, sl in zip(sids, slots.tolist()):
                pool[sl] = token
                history[s].append(token)
                token += 1
        else:
            _, sid = op
            if sid not in history:
                continue
            model.free_sequence(sid)
            bm.free_sequence(sid)
            del history[sid]
            swapped.discard(sid)
        # state equal after every operation
        assert bm.num_free_blocks == len(model.free)
        assert bm.num_free_host_blocks == len(model.host_free)
        assert [bm.ref_count(b) for b in range(nb)] == model.refs
        resident = [s_ for s_ in history if s_ not in swapped]
        if resident:
            sids = sorted(resident)
            mb = max(len(model.tables[s]) for s in sids) or 1
            bt, cl = bm.block_tables(sids, mb)
            exp_bt, exp_cl = model.block_tables(sids, mb)
            assert bt.tolist() == exp_bt and cl.tolist() == exp_cl
            # every request reads back exactly its own history through its table
            for row, n, s in zip(bt, cl, sids):
                idx = [int(row[i // block_size]) * block_size + i % block_size for i in range(int(n))]
                assert pool[idx].tolist() == history[s]
    assert token > 300, "the history should have written many tokens"


class _NoCopyModel(BlockModel):
    """A planted mistake: writes into shared blocks without cloning them."""

    def append_tokens(self, sids):
        slots = []
        for sid in sids:
            table, n = self.tables[sid], self.lengths[sid]
            if n % self.block_size == 0:
                table.append(self._take())
            slots.append(self.slot(table[-1], n % self.block_size))
            self.lengths[sid] = n + 1
        return slots, []


def test_history_check_catches_a_missing_copy():
    """The data-level invariant is a pin in its own right: a model that skips copy-on-write fails it."""
    m = _NoCopyModel(8, 4)
    pool = np.full(32, -1)
    slots = m.add_sequence(1, 6)
    pool[slots] = range(6)
    m.fork(1, 2)
    (s1,), _ = m.append_tokens([1])
    (s2,), _ = m.append_tokens([2])
    pool[s1], pool[s2] = 100, 200
    row = m.tables[1]
    seq1 = [pool[row[i // 4] * 4 + i % 4] for i in range(7)]
    assert seq1 != [0, 1, 2, 3, 4, 5, 100]        # the child's token overwrote the parent's
