"""Reference model of the block manager (pure Python).

TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT.  Only the tests, the smoke check
in ``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` may use it.

Rules, from "The KV Cache and PagedAttention":
  * a text's cache is cut into equal blocks; its logical blocks map to
    physical blocks anywhere in the pool (§Like Pages of Memory);
  * the block table records, per logical block, its physical block and its
    filled places; a text receives a further block only once its current
    blocks are full (§The Block Table);
  * a finished text returns its blocks to the pool (§The Block Table);
  * parallel samples of one prompt point at the same physical blocks, each
    block counting the texts that use it; a text that must change a shared
    block copies it, changes the copy, and the original's count falls by one
    (§Shared, Copied on Write);
  * a text either has every block it needs or none (§When Memory Runs Out):
    an operation that cannot get every block it needs changes nothing.

Free-list policy (the pages leave it open): blocks are taken from the front of
the free list and returned to its back; the initial order is given.  The
"places filled" field is kept as the text's token count (filled places of
block j = min(B, n - j*B)).

Prefix reuse ("The KV Cache and PagedAttention", §What Came After): a full
block is identified by a hash of its tokens chained with the hash of all
tokens before it; a text that begins like an earlier one takes over the
earlier text's blocks.  ``add_seq_tokens`` takes over cached blocks up to the
first miss and caches the prompt's new full blocks; a cached block with count
zero keeps its hash while it waits in the free list, a hit takes it back out,
and handing it out again from the free list drops the hash.  The chained hash
is SplitMix64's output mix applied token by token (defined below).  A hash is
how a block is looked up, not proof that it holds the same text: a cached
block is taken over only if the whole prefix it was cached for (every token
up to its end) equals the new prompt's, compared here token by token.
``key_bits`` keeps only the low bits of the hash as the lookup key, so that
tests can make different prefixes meet on one key; a key already held stays
with its block.

Pinned by tests/golden/cow_two_answers.json (the pages' two-answer example)
and by invariants checked in tests/test_block_manager.py; prefix reuse by the
hand-worked sessions in tests/test_prefix_reuse.py.
"""
from __future__ import annotations

from collections import deque
from typing import Dict, List, Optional, Sequence, Tuple

_M64 = (1 << 64) - 1


def _mix64(z: int) -> int:
    """SplitMix64's output mix (Steele, Lea, Flood, OOPSLA 2014)."""
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _M64
    return z ^ (z >> 31)


def block_hash(prev: int, tokens: Sequence[int]) -> int:
    """Hash of one full block: the hash of everything before it (0 for the
    first block), then each token id taken as an unsigned 32-bit number."""
    h = prev
    for t in tokens:
        h = _mix64(h ^ (((int(t) & 0xFFFFFFFF) + 0x9E3779B97F4A7C15) & _M64))
    return h


class BlockManagerError(Exception):
    def __init__(self, kind: str, msg: str = ""):
        super().__init__(f"{kind}: {msg}")
        self.kind = kind


class BlockManagerModel:
    def __init__(self, num_blocks: int, block_size: int,
                 initial_order: Optional[Sequence[int]] = None, key_bits: int = 64):
        if num_blocks <= 0 or block_size <= 0:
            raise BlockManagerError("invalid", "num_blocks and block_size must be > 0")
        self.num_blocks = num_blocks
        self.block_size = block_size
        order = list(range(num_blocks)) if initial_order is None else [int(b) for b in initial_order]
        if sorted(order) != list(range(num_blocks)):
            raise BlockManagerError("invalid", "initial order is not a permutation")
        self.free: deque = deque(order)
        self.ref: List[int] = [0] * num_blocks
        self.tables: Dict[int, List[int]] = {}
        self.tokens: Dict[int, int] = {}
        self.cache: Dict[int, int] = {}        # lookup key -> block
        self.cached: Dict[int, int] = {}       # block -> its key
        self.prefix_of: Dict[int, tuple] = {}  # block -> every token up to its end
        self.key_mask = (1 << key_bits) - 1

    # -- helpers -----------------------------------------------------------
    def _take(self) -> int:
        b = self.free.popleft()
        h = self.cached.pop(b, None)
        self.prefix_of.pop(b, None)
        if h is not None and self.cache.get(h) == b:
            del self.cache[h]
        self.ref[b] = 1
        return b

    def _need(self, n: int) -> None:
        if len(self.free) < n:
            raise BlockManagerError("out_of_blocks", f"need {n}, have {len(self.free)}")

    # -- operations --------------------------------------------------------
    def add_seq(self, seq_id: int, num_tokens: int) -> None:
        """A new text whose first ``num_tokens`` tokens (its prompt) are
        stored at once: ceil(n / B) fresh blocks."""
        if seq_id in self.tables:
            raise BlockManagerError("exists", str(seq_id))
        if num_tokens < 0:
            raise BlockManagerError("invalid", "negative token count")
        n_blocks = -(-num_tokens // self.block_size)
        self._need(n_blocks)
        self.tables[seq_id] = [self._take() for _ in range(n_blocks)]
        self.tokens[seq_id] = num_tokens

    def add_seq_tokens(self, seq_id: int, tokens: Sequence[int]) -> int:
        """A new text from its prompt's token ids.  Its leading full blocks
        whose chained hashes are cached (up to the first miss) are taken over;
        the rest are fresh.  Returns the number of tokens taken over."""
        if seq_id in self.tables:
            raise BlockManagerError("exists", str(seq_id))
        B = self.block_size
        n = len(tokens)
        full = n // B
        hashes, hits, prev, run = [], [], 0, True
        for j in range(full):
            prev = block_hash(prev, tokens[j * B:(j + 1) * B])
            key = prev & self.key_mask
            hashes.append(key)
            prefix = tuple(int(t) for t in tokens[:(j + 1) * B])
            if run and key in self.cache and self.prefix_of[self.cache[key]] == prefix:
                hits.append(self.cache[key])
            else:
                run = False
        n_blocks = -(-n // B)
        waiting = sum(1 for b in hits if self.ref[b] == 0)
        if len(self.free) - waiting < n_blocks - len(hits):
            raise BlockManagerError("out_of_blocks", f"need {n_blocks - len(hits)}")
        table = []
        for b in hits:
            if self.ref[b] == 0:
                self.free.remove(b)
            self.ref[b] += 1
            table.append(b)
        for j in range(len(hits), n_blocks):
            b = self._take()
            table.append(b)
            if j < full and hashes[j] not in self.cache:
                self.cache[hashes[j]] = b
                self.cached[b] = hashes[j]
                self.prefix_of[b] = tuple(int(t) for t in tokens[:(j + 1) * B])
        self.tables[seq_id] = table
        self.tokens[seq_id] = n
        return len(hits) * B

    def num_cached_blocks(self) -> int:
        return len(self.cache)

    def fork(self, parent: int, child: int) -> None:
        """The child shares every block of the parent; each count goes up by one."""
        if parent not in self.tables:
            raise BlockManagerError("no_seq", str(parent))
        if child in self.tables:
            raise BlockManagerError("exists", str(child))
        self.tables[child] = list(self.tables[parent])
        self.tokens[child] = self.tokens[parent]
        for b in self.tables[child]:
            self.ref[b] += 1

    def append_slot(self, seq_id: int) -> Tuple[int, int, int]:
        """Room for the text's next token.  Returns (slot, cow_src, cow_dst);
        the copy pair is (-1, -1) when no copy is needed.  The caller copies
        block cow_src to cow_dst before writing the token."""
        if seq_id not in self.tables:
            raise BlockManagerError("no_seq", str(seq_id))
        table = self.tables[seq_id]
        n = self.tokens[seq_id]
        place = n % self.block_size
        src = dst = -1
        if place == 0:
            self._need(1)
            table.append(self._take())
        else:
            last = table[-1]
            if self.ref[last] > 1:
                self._need(1)
                dst = self._take()
                self.ref[last] -= 1
                table[-1] = dst
                src = last
        self.tokens[seq_id] = n + 1
        return table[-1] * self.block_size + place, src, dst

    def free_seq(self, seq_id: int) -> None:
        """The text is done: every block's count drops by one; blocks that
        reach zero go back to the pool, in table order."""
        if seq_id not in self.tables:
            raise BlockManagerError("no_seq", str(seq_id))
        for b in self.tables.pop(seq_id):
            if self.ref[b] <= 0:
                raise BlockManagerError("corrupt", f"count of block {b} below zero")
            self.ref[b] -= 1
            if self.ref[b] == 0:
                self.free.append(b)
        del self.tokens[seq_id]

    # -- queries -----------------------------------------------------------
    def num_free(self) -> int:
        return len(self.free)

    def refcount(self, block: int) -> int:
        return self.ref[block]

    def export(self, seq_ids: Sequence[int], max_blocks_per_seq: int):
        """Block tables (``-1`` past each text's last block) and token counts."""
        tables, lens = [], []
        for s in seq_ids:
            if s not in self.tables:
                raise BlockManagerError("no_seq", str(s))
            t = self.tables[s]
            if len(t) > max_blocks_per_seq:
                raise BlockManagerError("table_full", f"{len(t)} > {max_blocks_per_seq}")
            tables.append(t + [-1] * (max_blocks_per_seq - len(t)))
            lens.append(self.tokens[s])
        return tables, lens
