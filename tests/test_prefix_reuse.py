"""Prefix reuse in the block manager ("The KV Cache and PagedAttention",
section "What Came After": every full block is identified by a hash of its
tokens chained with the hash of all tokens before it, and a text that begins
like an earlier one takes over the earlier text's blocks).

The oracle's model is pinned by hand-worked sessions and planted mistakes;
the C++ manager must match the model exactly on seeded random sessions
(CPU only)."""
import random

import pytest

from oracle import BlockManagerError, BlockManagerModel


class Cpp:
    """The C++ manager through the binding, with the model's interface."""

    def __init__(self, n, b, key_bits=64):
        import paged_kv_cache_326_b200 as P
        self.P = P
        P.pa_set_option(P.PA_OPT_PREFIX_KEY_BITS, key_bits)
        try:
            self.bm = P.BlockManager(n, b)
        finally:
            P.pa_set_option(P.PA_OPT_PREFIX_KEY_BITS, 64)
        self.block_size = b

    def _run(self, fn, *a):
        try:
            return fn(*a)
        except self.P.PagedAttnError as e:
            kind = {-3: "out_of_blocks", -4: "no_seq", -5: "exists", -6: "table_full",
                    -1: "invalid"}.get(e.code, str(e.code))
            raise BlockManagerError(kind) from None

    def add_seq_tokens(self, s, toks):
        return self._run(self.bm.add_seq_tokens, s, toks)

    def add_seq(self, s, n):
        return self._run(self.bm.add_seq, s, n)

    def fork(self, p, c):
        return self._run(self.bm.fork, p, c)

    def append_slot(self, s):
        return self._run(self.bm.append_slot, s)

    def free_seq(self, s):
        return self._run(self.bm.free_seq, s)

    def num_free(self):
        return self.bm.num_free()

    def num_cached_blocks(self):
        return self.bm.num_cached_blocks()

    def refcount(self, b):
        return self.bm.refcount(b)

    def export(self, ids, mb):
        t, l = self.bm.export(ids, mb)
        return t.tolist(), l.tolist()


@pytest.fixture(scope="module", autouse=True)
def built():
    from paged_kv_cache_326_b200 import build
    build.build()


# ---------------------------------------------------------------------------
# pins of the rules (hand-worked sessions, blocks of 4, free list in order)
# ---------------------------------------------------------------------------

def pin_same_beginning_takes_over_full_blocks(make):
    bm = make(16, 4)
    assert bm.add_seq_tokens(1, list(range(1, 11))) == 0        # blocks 0, 1 full, 2 partial
    assert bm.num_cached_blocks() == 2
    assert bm.add_seq_tokens(2, list(range(1, 9)) + [99, 98]) == 8
    tables, lens = bm.export([1, 2], 4)
    assert tables == [[0, 1, 2, -1], [0, 1, 3, -1]] and lens == [10, 10]
    assert [bm.refcount(b) for b in range(4)] == [2, 2, 1, 1]
    assert bm.num_free() == 12


def pin_partial_last_block_is_never_shared(make):
    bm = make(16, 4)
    toks = list(range(1, 11))
    bm.add_seq_tokens(1, toks)
    assert bm.add_seq_tokens(2, toks) == 8                       # identical prompts
    tables, _ = bm.export([1, 2], 4)
    assert tables[0][:2] == tables[1][:2] and tables[0][2] != tables[1][2]


def pin_hash_covers_everything_before(make):
    """Equal second blocks after different first blocks share nothing."""
    bm = make(16, 4)
    bm.add_seq_tokens(1, [1, 2, 3, 4, 5, 6, 7, 8])
    assert bm.add_seq_tokens(2, [0, 2, 3, 4, 5, 6, 7, 8]) == 0
    tables, _ = bm.export([1, 2], 2)
    assert set(tables[0]).isdisjoint(tables[1])
    assert bm.num_cached_blocks() == 4


def pin_waiting_blocks_are_taken_back(make):
    """A finished text's cached blocks wait in the free list; a text that
    begins the same way takes them back out."""
    bm = make(8, 4)
    bm.add_seq_tokens(1, list(range(12)))
    bm.free_seq(1)
    assert bm.num_free() == 8 and bm.num_cached_blocks() == 3
    assert bm.add_seq_tokens(2, list(range(12)) + [5]) == 12
    tables, _ = bm.export([2], 4)
    assert tables == [[0, 1, 2, 3]]
    assert bm.num_free() == 4 and [bm.refcount(b) for b in range(4)] == [1, 1, 1, 1]


def pin_handing_out_evicts_and_reuse_stops_at_the_first_miss(make):
    """Blocks 0, 1 (cached, waiting) sit at the back of the free list after
    blocks 2..5; taking five fresh blocks hands out block 0 again, which
    drops its hash.  The same prompt then misses at its first block and takes
    over nothing, although its second block's hash is still cached."""
    bm = make(6, 4)
    bm.add_seq_tokens(1, list(range(8)))                          # blocks 0, 1
    bm.free_seq(1)                                                # free list: 2 3 4 5 0 1
    bm.add_seq(2, 20)                                             # takes 2 3 4 5 0
    assert bm.num_cached_blocks() == 1                            # block 1 keeps its hash
    bm.free_seq(2)                                                # free list: 1 2 3 4 5 0
    assert bm.add_seq_tokens(3, list(range(8))) == 0
    tables, _ = bm.export([3], 2)
    # fresh blocks from the front: block 1 is handed out (its old hash goes),
    # and both new full blocks are cached under the prompt's hashes
    assert tables == [[1, 2]]
    assert [bm.refcount(b) for b in range(3)] == [0, 1, 1]
    assert bm.num_cached_blocks() == 2
    assert bm.add_seq_tokens(4, list(range(8))) == 8              # now a full takeover


def pin_out_of_blocks_changes_nothing(make):
    bm = make(4, 4)
    bm.add_seq_tokens(1, list(range(8)))
    before = (bm.export([1], 2), bm.num_free(), bm.num_cached_blocks())
    with pytest.raises(BlockManagerError) as e:
        bm.add_seq_tokens(2, list(range(8)) + list(range(100, 112)))   # 2 reused + 3 fresh > 2
    assert e.value.kind == "out_of_blocks"
    assert (bm.export([1], 2), bm.num_free(), bm.num_cached_blocks()) == before
    assert bm.add_seq_tokens(2, list(range(8)) + [1, 2]) == 8            # 1 fresh fits


def _key(tokens, B, bits):
    """Lookup key of the last full block of `tokens` with `bits` key bits
    (test set-up only: used to find prompts whose keys meet)."""
    from oracle.block_manager import block_hash
    h = 0
    for j in range(len(tokens) // B):
        h = block_hash(h, tokens[j * B:(j + 1) * B])
    return h & ((1 << bits) - 1)


def pin_equal_keys_of_different_blocks_share_nothing(make):
    """With 4 key bits, two different one-block prompts whose keys meet: the
    second takes over nothing, and its block is not cached (the key stays
    with the first block)."""
    bits, B = 4, 4
    a = [1, 2, 3, 4]
    b = next([5, 6, 7, t] for t in range(1000) if _key([5, 6, 7, t], B, bits) == _key(a, B, bits))
    bm = make(8, B, key_bits=bits)
    assert bm.add_seq_tokens(1, a) == 0
    assert bm.add_seq_tokens(2, b) == 0
    tables, _ = bm.export([1, 2], 1)
    assert tables[0] != tables[1]
    assert bm.num_cached_blocks() == 1
    assert bm.add_seq_tokens(3, a + [9]) == 4                      # the first still hits


def pin_equal_last_blocks_after_different_prefixes_share_nothing(make):
    """With 4 key bits: text 1 is [P, X], text 2 is [Q] alone (so Q's block is
    cached), text 3 is [Q, X] where the keys of [P, X] and [Q, X] meet.  Text 3
    takes over Q's block, but not text 1's X block, although the key and X's
    own token ids agree: the whole prefix before X differs."""
    bits, B = 4, 4
    P_, X = [1, 2, 3, 4], [7, 7, 7, 7]
    Q = next([9, 9, 9, t] for t in range(1000)
             if _key([9, 9, 9, t], B, bits) not in (_key(P_, B, bits), _key(P_ + X, B, bits))
             and _key([9, 9, 9, t] + X, B, bits) == _key(P_ + X, B, bits))
    bm = make(8, B, key_bits=bits)
    assert bm.add_seq_tokens(1, P_ + X) == 0
    assert bm.add_seq_tokens(2, Q) == 0
    assert bm.add_seq_tokens(3, Q + X) == 4
    tables, _ = bm.export([1, 2, 3], 2)
    assert tables[2][0] == tables[1][0] and tables[2][1] != tables[0][1]


PINS = [pin_same_beginning_takes_over_full_blocks, pin_partial_last_block_is_never_shared,
        pin_hash_covers_everything_before, pin_waiting_blocks_are_taken_back,
        pin_handing_out_evicts_and_reuse_stops_at_the_first_miss,
        pin_out_of_blocks_changes_nothing, pin_equal_keys_of_different_blocks_share_nothing,
        pin_equal_last_blocks_after_different_prefixes_share_nothing]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_model_pin(pin):
    pin(BlockManagerModel)


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_cpp_pin(pin):
    pin(Cpp)


# ---------------------------------------------------------------------------
# planted mistakes in copies of the model
# ---------------------------------------------------------------------------

class NoChain(BlockManagerModel):
    """Planted mistake: each block hashed on its own tokens only."""

    def add_seq_tokens(self, seq_id, tokens):
        import oracle.block_manager as M
        real = M.block_hash
        M.block_hash = lambda prev, toks: real(0, toks)
        try:
            return super().add_seq_tokens(seq_id, tokens)
        finally:
            M.block_hash = real


class CachesPartial(BlockManagerModel):
    """Planted mistake: the partial last block is cached and shared too."""

    def add_seq_tokens(self, seq_id, tokens):
        B = self.block_size
        pad = (-len(tokens)) % B
        got = super().add_seq_tokens(seq_id, list(tokens) + [-1] * pad)
        self.tokens[seq_id] = len(tokens)
        return min(got, len(tokens))


class NoEviction(BlockManagerModel):
    """Planted mistake: handing a block out again keeps its hash."""

    def _take(self):
        b = self.free.popleft()
        self.ref[b] = 1
        return b


class KeyOnly(BlockManagerModel):
    """Planted mistake: a key match is taken as a hit, with no check of the
    cached block's prefix."""

    def add_seq_tokens(self, seq_id, tokens):
        self.prefix_of = _Anything()
        return super().add_seq_tokens(seq_id, tokens)


class _Anything(dict):
    def __getitem__(self, k):
        return _Equal()


class _Equal:
    def __eq__(self, other):
        return True


class LastBlockOnly(BlockManagerModel):
    """Planted mistake: only the cached block's own token ids are compared,
    not the prefix before it."""

    def add_seq_tokens(self, seq_id, tokens):
        B = self.block_size
        real = self.prefix_of
        self.prefix_of = {b: _Tail(p, B) for b, p in real.items()}
        try:
            return super().add_seq_tokens(seq_id, tokens)
        finally:
            merged = {b: (p.full if isinstance(p, _Tail) else p) for b, p in self.prefix_of.items()}
            self.prefix_of = merged


class _Tail:
    def __init__(self, full, B):
        self.full, self.B = full, B

    def __eq__(self, other):
        return tuple(self.full[-self.B:]) == tuple(other[-self.B:])


@pytest.mark.parametrize("cls", [NoChain, CachesPartial, NoEviction, KeyOnly, LastBlockOnly],
                         ids=lambda c: c.__name__)
def test_planted_prefix_mistake_is_caught(cls):
    failed = 0
    for pin in PINS:
        try:
            pin(cls)
        except (AssertionError, BlockManagerError, ValueError, KeyError):
            failed += 1
    assert failed, cls.__name__


# ---------------------------------------------------------------------------
# the C++ manager against the model
# ---------------------------------------------------------------------------

def _session(make, seed):
    """Random operations over prompts from a few shared beginnings (so blocks
    are taken over, wait in the free list, are taken back and evicted); every
    result and the full state after each operation are logged."""
    rnd = random.Random(seed)
    B = rnd.choice([2, 4, 8])
    bm = make(48, B)
    stems = [[rnd.randrange(50) for _ in range(rnd.randrange(0, 5 * B))] for _ in range(4)]
    live, next_id, log = [], 0, []
    for _ in range(300):
        op = rnd.random()
        try:
            if op < 0.35 or not live:
                toks = list(rnd.choice(stems))[:rnd.randrange(0, 5 * B + 1)]
                toks += [rnd.randrange(50) for _ in range(rnd.randrange(0, B + 2))]
                log.append(("tok", bm.add_seq_tokens(next_id, toks)))
                live.append(next_id)
                next_id += 1
            elif op < 0.45:
                bm.add_seq(next_id, rnd.randrange(0, 3 * B))
                live.append(next_id)
                next_id += 1
                log.append(("add",))
            elif op < 0.55:
                p = rnd.choice(live)
                bm.fork(p, next_id)
                live.append(next_id)
                next_id += 1
                log.append(("fork",))
            elif op < 0.8:
                log.append(("app", tuple(bm.append_slot(rnd.choice(live)))))
            else:
                s = rnd.choice(live)
                bm.free_seq(s)
                live.remove(s)
                log.append(("free",))
        except BlockManagerError as e:
            log.append(("err", e.kind))
            if e.kind == "out_of_blocks" and live:
                s = live.pop(0)
                bm.free_seq(s)
        tables, lens = bm.export(live, 64) if live else ([], [])
        log.append((tuple(map(tuple, tables)), tuple(lens), bm.num_free(),
                    bm.num_cached_blocks(), tuple(bm.refcount(b) for b in range(48))))
    return log


@pytest.mark.parametrize("seed", range(8))
def test_cpp_matches_model_exactly(seed):
    assert _session(Cpp, seed) == _session(BlockManagerModel, seed)


@pytest.mark.parametrize("seed", range(6))
def test_cpp_matches_model_when_keys_collide(seed):
    """3 key bits: prompts meet on keys all the time; the C++ manager (token
    ids plus a check hash) still shares exactly what the model (whole
    prefixes compared) shares."""
    import functools
    cpp = functools.partial(Cpp, key_bits=3)
    model = functools.partial(BlockManagerModel, key_bits=3)
    assert _session(cpp, 100 + seed) == _session(model, 100 + seed)


def test_sessions_do_reuse_and_evict():
    """The sessions exercise what they are meant to: takeovers happen."""
    log = _session(BlockManagerModel, 3)
    assert any(e[0] == "tok" and e[1] > 0 for e in log if isinstance(e[0], str))


def test_taken_over_blocks_attend_like_private_ones():
    """Two prompts begin with the same 8 tokens (blocks of 4).  The second
    text takes over the first's two full blocks and stores only its own
    remaining tokens (negative slots for the taken-over ones).  Its decode
    through the oracle then equals torch's fp64 attention on its contiguous
    keys and values, i.e. the shared blocks hold exactly its prefix."""
    import numpy as np
    import torch

    import oracle
    from tests.oracle_pins import f64, sdpa_contiguous

    B, H, D, N = 4, 2, 8, 16
    bm = Cpp(N, B)
    g = torch.Generator().manual_seed(7)
    prefix = [5, 6, 7, 8, 9, 10, 11, 12]
    prompts = [prefix + [1, 2], prefix + [3, 4, 13, 14, 15]]
    # a token's key and value depend only on the token and its position here,
    # as in a model whose prefix is the same
    table_k = torch.randn(64, 32, H, D, generator=g).half()   # [token id][position]
    table_v = torch.randn(64, 32, H, D, generator=g).half()
    kc = torch.full((N, H, B, D), float("nan"), dtype=torch.float16)
    vc = torch.full((N, H, B, D), float("nan"), dtype=torch.float16)
    reused = []
    for sid, toks in enumerate(prompts):
        cached = bm.add_seq_tokens(sid, toks)
        reused.append(cached)
        tables, _ = bm.export([sid], 8)
        ks = torch.stack([table_k[t, p] for p, t in enumerate(toks)])
        vs = torch.stack([table_v[t, p] for p, t in enumerate(toks)])
        slots = np.array([tables[0][p // B] * B + p % B if p >= cached else -1
                          for p in range(len(toks))])
        kc_new, vc_new = oracle.cache_write(f64(kc), f64(vc), f64(ks), f64(vs), slots, B)
        kc, vc = torch.from_numpy(kc_new).half(), torch.from_numpy(vc_new).half()
    assert reused == [0, 8]
    tables, lens = bm.export([0, 1], 8)
    q = torch.randn(2, H, D, generator=g).half()
    got = oracle.paged_decode(f64(q), f64(kc), f64(vc), np.array(tables), lens, 0.3, B)
    K = [torch.stack([table_k[t, p] for p, t in enumerate(toks)]) for toks in prompts]
    V = [torch.stack([table_v[t, p] for p, t in enumerate(toks)]) for toks in prompts]
    ref = sdpa_contiguous(q, K, V, 0.3)
    assert np.abs(got - ref).max() <= 1e-12


def test_many_takebacks_keep_the_free_list_order():
    """Thousands of take-backs of waiting blocks (each leaves a stale entry
    behind in the C++ free list, compacted from time to time) give the same
    tables as the model."""
    def run(make):
        bm = make(64, 4)
        out = []
        for i in range(3000):
            toks = list(range(i % 5, i % 5 + 8)) + [i % 3]
            out.append(bm.add_seq_tokens(i, toks))
            out.append(tuple(bm.export([i], 4)[0][0]))
            bm.free_seq(i)
            out.append((bm.num_free(), bm.num_cached_blocks()))
        return out
    assert run(Cpp) == run(BlockManagerModel)


def test_reuse_across_requests_feeds_the_shared_prefix_split():
    """Four requests that begin with the same 12-token system prompt (blocks
    of 4) take over its three blocks; the host splitter then finds those
    blocks as the group's prefix, and the oracle's shared-prefix form over
    the split equals its plain decode over the tables bit for bit."""
    import numpy as np
    import torch

    import oracle
    import paged_kv_cache_326_b200 as P

    B, H, D, N = 4, 2, 8, 32
    bm = Cpp(N, B)
    system = list(range(100, 112))
    asks = [[1, 2], [3, 4, 5, 6, 7], [8], [9, 10, 11, 12]]
    got = [bm.add_seq_tokens(i, system + a) for i, a in enumerate(asks)]
    assert got == [0, 12, 12, 12]
    tables, lens = bm.export(list(range(4)), 8)
    pt, pl, tt, tl = P.split_shared_prefix(torch.tensor(tables, dtype=torch.int32),
                                           torch.tensor(lens, dtype=torch.int32), B, 4)
    assert pl.tolist() == [12] and pt.tolist()[0][:3] == tables[0][:3]
    assert tl.tolist() == [len(a) for a in asks]
    g = torch.Generator().manual_seed(3)
    kc = torch.randn(N, H, B, D, generator=g).double().numpy()
    vc = torch.randn(N, H, B, D, generator=g).double().numpy()
    q = torch.randn(4, H, D, generator=g).double().numpy()
    plain = oracle.paged_decode(q, kc, vc, np.array(tables), lens, 0.3, B)
    prows = [[b for b in r if b >= 0] for r in pt.tolist()]
    trows = [[b for b in r if b >= 0] for r in tt.tolist()]
    shared = oracle.paged_decode_shared(q, kc, vc, prows, pl.tolist(), trows, tl.tolist(), 4,
                                        0.3, B)
    assert np.array_equal(plain, shared)
