"""The host block manager (C, via the C ABI; no GPU needed): refcounted pages,
fork with shared pages, copy-on-write on append, release deletes the entry.

An independent Python model of the same rules is driven by random operation
sequences and compared with the library after every step; the leak check
(every page back in the pool after every sequence is freed) is the fix the
page "Flash Attention与Paged KV Cache优化大模型计算效率" §5.2 describes."""
import numpy as np
import pytest

from paged_kv_cache_380_b200 import build, ops


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    ops.load()


class Model:
    """Plain Python statement of the allocator rules."""

    def __init__(self, P, ps, mp):
        self.P, self.ps, self.mp = P, ps, mp
        self.ref = [0] * P
        self.free = list(range(P - 1, -1, -1))
        self.seqs = {}
        self.next = 0

    def take(self):
        p = self.free.pop()
        self.ref[p] = 1
        return p

    def drop(self, p):
        self.ref[p] -= 1
        if self.ref[p] == 0:
            self.free.append(p)

    def add(self):
        i = self.next
        self.next += 1
        self.seqs[i] = ([], 0)
        return i

    def fork(self, parent):
        pages, n = self.seqs[parent]
        for p in pages:
            self.ref[p] += 1
        i = self.next
        self.next += 1
        self.seqs[i] = (list(pages), n)
        return i

    def append(self, s, k):
        pages, n = self.seqs[s]
        need = -(-(n + k) // self.ps)
        if need > self.mp:
            return "invalid"
        cow = k > 0 and n % self.ps != 0 and self.ref[pages[-1]] > 1
        if need - len(pages) + cow > len(self.free):
            return "oom"
        copies = []
        pages = list(pages)
        if cow:
            old = pages[-1]
            new = self.take()
            self.drop(old)
            pages[-1] = new
            copies = [(old, new)]
        while len(pages) < need:
            pages.append(self.take())
        slots = [pages[(n + i) // self.ps] * self.ps + (n + i) % self.ps for i in range(k)]
        self.seqs[s] = (pages, n + k)
        return slots, copies

    def release(self, s):
        pages, _ = self.seqs.pop(s)
        for p in pages:
            self.drop(p)


def test_random_operations_match_the_model():
    rng = np.random.default_rng(0)
    for trial in range(20):
        P, ps, mp = int(rng.integers(4, 40)), int(rng.choice([1, 2, 4, 16])), int(rng.integers(2, 12))
        bm, m = ops.BlockManager(P, ps, mp), Model(P, ps, mp)
        for step in range(200):
            live = list(m.seqs)
            op = rng.integers(0, 4) if live else 0
            if op == 0:
                assert bm.add_sequence() == m.add()
            elif op == 1:
                s = int(rng.choice(live))
                assert bm.fork(s) == m.fork(s)
            elif op == 2:
                s, k = int(rng.choice(live)), int(rng.integers(0, 2 * ps + 2))
                want = m.append(s, k)
                if want == "oom":
                    with pytest.raises(ops.PagedKVError) as e:
                        bm.append(s, k)
                    assert e.value.code == -7
                elif want == "invalid":
                    with pytest.raises(ops.PagedKVError):
                        bm.append(s, k)
                else:
                    slots, copies = bm.append(s, k)
                    assert slots.tolist() == want[0] and copies == want[1]
            else:
                s = int(rng.choice(live))
                bm.free(s)
                m.release(s)
            assert bm.num_free_pages() == len(m.free)
            assert [bm.refcount(p) for p in range(P)] == m.ref
            assert bm.num_sequences() == len(m.seqs)
            if m.seqs:
                ids = sorted(m.seqs)
                table, lens = bm.block_tables(ids)
                for row, i in zip(range(len(ids)), ids):
                    pages, n = m.seqs[i]
                    assert table[row, :len(pages)].tolist() == pages and (table[row, len(pages):] == -1).all()
                    assert lens[row] == n
        for s in list(m.seqs):                       # leak check
            bm.free(s)
        assert bm.num_free_pages() == P and all(bm.refcount(p) == 0 for p in range(P))
        assert bm.num_sequences() == 0


def test_live_sequences_never_write_the_same_slot():
    bm = ops.BlockManager(64, 4, 16)
    root = bm.add_sequence()
    bm.append(root, 10)                              # 2.5 pages: last page shared after forks
    kids = [bm.fork(root) for _ in range(4)]
    written = {}
    for s in kids + [root]:
        slots, copies = bm.append(s, 3)
        for x in slots.tolist():
            assert x not in written, "two sequences got the same slot"
            written[x] = s


def test_double_free_and_unknown_ids_are_errors():
    bm = ops.BlockManager(8, 4, 4)
    s = bm.add_sequence()
    bm.append(s, 5)
    bm.free(s)
    with pytest.raises(ops.PagedKVError):
        bm.free(s)
    with pytest.raises(ops.PagedKVError):
        bm.append(12345, 1)
    with pytest.raises(ops.PagedKVError):
        bm.fork(s)
    assert bm.num_free_pages() == 8


def test_out_of_pages_leaves_state_unchanged():
    bm = ops.BlockManager(3, 4, 8)
    a = bm.add_sequence()
    bm.append(a, 8)
    with pytest.raises(ops.PagedKVError) as e:
        bm.append(a, 9)                              # needs 3 more pages, 1 free
    assert e.value.code == -7
    table, lens = bm.block_tables([a])
    assert lens.tolist() == [8] and bm.num_free_pages() == 1
