"""CPU oracle: paged decode attention and the KV-cache write, in fp64.

TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT.  Only the tests, the smoke check
in ``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` may import it.
It shares no code with the CUDA path and imports nothing from the package.

What it computes is the plain definition.  Paging changes where the keys and
values live, not what attention computes ("The KV Cache and PagedAttention",
§Like Pages of Memory: logical blocks are contiguous to the text, physical
blocks sit anywhere; §The Block Table: the kernel finds each logical block's
physical block in the table and reads it there).  So the oracle

  1. writes the new token's key and value into its slot ("KV cache", §How it
     works: each generated token's key and value join the cache; "The KV
     Cache and PagedAttention", §One Token at a Time: a step computes keys
     and values for the new token alone and keeps the older ones);
  2. gathers each text's tokens through its block table into one contiguous
     fp64 buffer (token t sits in logical block t // B at place t % B);
  3. runs textbook attention for the one new query: weights
     softmax(scale * q . k_t) over every stored key including the new one
     ("KV cache", §How it works), output sum_t w_t v_t.

Readings where the pages are silent (each also listed in the design notes):
  * pool layout ``[num_blocks][num_heads][block_size][head_dim]`` for K and V;
  * the context length counts the token written in this step (write, then
    attend);
  * ``scale`` is a parameter (the workloads use 1/sqrt(head_dim) in fp32);
  * a text with no tokens gets a zero output;
  * a negative slot marks a padding token that is not written;
  * table entries past the text's last block are never read.

Precision: inputs are the exact fp16/bf16 values widened to fp64; every step
is fp64; softmax subtracts the maximum before exponentiating (an identity, so
the result is the same number up to rounding).

Prompt phase (``prefill``): causal attention of a prompt's tokens over the
prompt itself, whose keys and values are then stored in the cache (the
write is ``cache_write``).

Shared prefixes (``split_shared_prefix``, ``paged_decode_shared``): texts
in groups that share the leading blocks of one prompt attend over the group's
prefix followed by their own tail, which is the same token sequence as their
joined table.

Block copies (``copy_blocks``): whole blocks copied from a source pool to a
destination pool ("The KV Cache and PagedAttention", §Shared, Copied on
Write: a text that must change a block it shares first receives a duplicate
of it; §When Memory Runs Out: blocks are moved out of the pool to CPU
memory and back).

Pinned by tests/test_oracle.py against: torch's fp64 attention on unpaged
contiguous tensors, scalar brute force with ``math.fsum`` on tiny inputs,
closed forms (one token gives its value; equal scores give the mean of the
values; one dominant score gives its value), bit-identity under a relabelling
of physical blocks, under a change of block size, and for texts that share
prefix blocks, and a hand-worked cache write; grouped-query attention against
the same pool with key/value heads replicated per query head, torch's fp64
attention on repeated heads, and brute force for one shared head; block
copies against the worked copy-on-write example of the pages (each answer
reads the prompt plus its own token and nothing of the other's), torch's
index_copy_ on raw bit patterns, and a copy out and back that restores every
block; shared prefixes against ``paged_decode`` on the joined tables (bit for
bit), a prefix and tail written out by hand for a forked prompt, scalar brute
force, and the order of prefix and tail swapped (softmax ignores order).
"""
from __future__ import annotations

from typing import Iterable, Optional, Sequence, Tuple

import numpy as np


def cache_write(k_cache: np.ndarray, v_cache: np.ndarray, k: np.ndarray, v: np.ndarray,
                slot_mapping: Sequence[int], block_size: int) -> Tuple[np.ndarray, np.ndarray]:
    """Return copies of the caches with token t's key/value placed at slot
    ``slot_mapping[t]``: physical block ``slot // block_size``, place
    ``slot % block_size``.  Negative slots are skipped.

    A pure copy of values, so it works on any dtype, including raw uint16
    bit patterns; the result is exact.  Caches are ``[N][H][B][D]``; k and v
    are ``[T][H][D]``."""
    kc = k_cache.copy()
    vc = v_cache.copy()
    for t, slot in enumerate(slot_mapping):
        slot = int(slot)
        if slot < 0:
            continue
        block, place = divmod(slot, block_size)
        kc[block, :, place, :] = k[t]
        vc[block, :, place, :] = v[t]
    return kc, vc


def copy_blocks(src_k: np.ndarray, src_v: np.ndarray, dst_k: np.ndarray, dst_v: np.ndarray,
                pairs: Sequence[Tuple[int, int]]) -> Tuple[np.ndarray, np.ndarray]:
    """Return copies of the destination pools in which, for every pair
    (src, dst), block dst holds block src of the source pools: every head,
    every place, every bit.  Every pair reads the source pools as they were
    before the call (the source arrays are never written, even when they are
    the destination arrays too).  Pools are ``[N][H][B][D]`` of any dtype."""
    kd = dst_k.copy()
    vd = dst_v.copy()
    for src, dst in pairs:
        kd[int(dst)] = src_k[int(src)]
        vd[int(dst)] = src_v[int(src)]
    return kd, vd


def gather_context(cache: np.ndarray, block_table: Sequence[int], context_len: int,
                   block_size: int) -> np.ndarray:
    """Contiguous fp64 ``[L][H][D]`` copy of one text's keys (or values):
    token t comes from physical block ``block_table[t // block_size]``, place
    ``t % block_size``."""
    L = int(context_len)
    H, D = cache.shape[1], cache.shape[3]
    out = np.empty((L, H, D), dtype=np.float64)
    for t in range(L):
        phys = int(block_table[t // block_size])
        out[t] = cache[phys, :, t % block_size, :]
    return out


def attend(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float) -> np.ndarray:
    """Attention of one query per head over L stored keys/values, fp64.

    q ``[H][D]``, K and V ``[L][H][D]``; returns ``[H][D]``.
    z_t = scale * sum_d q[d] K[t, d];  w = softmax(z);  out = sum_t w_t V[t].
    With L == 0 the output is zero."""
    q = np.asarray(q, dtype=np.float64)
    H, D = q.shape
    L = K.shape[0]
    out = np.zeros((H, D), dtype=np.float64)
    if L == 0:
        return out
    for h in range(H):
        z = float(scale) * (K[:, h, :] @ q[h])
        e = np.exp(z - z.max())
        w = e / e.sum()
        out[h] = w @ V[:, h, :]
    return out


def kv_head_of(num_heads: int, num_kv_heads: int) -> np.ndarray:
    """Query head h reads key/value head h // (num_heads / num_kv_heads):
    consecutive query heads use common keys and values ("The KV Cache
    and PagedAttention", §What Came After; num_kv_heads == num_heads is plain
    multi-head attention, num_kv_heads == 1 one set for all heads)."""
    if num_kv_heads <= 0 or num_heads % num_kv_heads:
        raise ValueError("num_heads must be a multiple of num_kv_heads")
    return np.arange(num_heads) // (num_heads // num_kv_heads)


def paged_decode(q: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray,
                 block_tables: np.ndarray, context_lens: Sequence[int], scale: float,
                 block_size: int,
                 pairs: Optional[Iterable[Tuple[int, int]]] = None) -> np.ndarray:
    """Decode attention over paged caches, fp64 ``[S][H][D]``.

    The caches may hold fewer heads than q (grouped-query attention): query
    head h then reads key/value head ``kv_head_of(H, H_kv)[h]``.

    With ``pairs`` (a list of (seq, head)), only those outputs are computed
    (the rest stay zero); this is how large workloads are checked one output
    at a time."""
    S, H, D = q.shape
    kvh = kv_head_of(H, k_cache.shape[1])
    out = np.zeros((S, H, D), dtype=np.float64)
    if pairs is None:
        for s in range(S):
            K = gather_context(k_cache, block_tables[s], context_lens[s], block_size)
            V = gather_context(v_cache, block_tables[s], context_lens[s], block_size)
            out[s] = attend(q[s], K[:, kvh, :], V[:, kvh, :], scale)
        return out
    by_seq = {}
    for s, h in pairs:
        by_seq.setdefault(int(s), []).append(int(h))
    for s, heads in by_seq.items():
        K = gather_context(k_cache, block_tables[s], context_lens[s], block_size)
        V = gather_context(v_cache, block_tables[s], context_lens[s], block_size)
        sel = kvh[heads]
        full = attend(q[s][heads], K[:, sel, :], V[:, sel, :], scale)
        for i, h in enumerate(heads):
            out[s, h] = full[i]
    return out


def split_shared_prefix(block_tables: np.ndarray, context_lens: Sequence[int], block_size: int,
                        group_size: int):
    """Cut the tables of groups of ``group_size`` consecutive texts into a
    shared prefix per group and a private tail per text ("The KV Cache and
    PagedAttention", §Shared, Copied on Write: the samples of one prompt point
    at the same physical blocks).  A group's prefix is the longest run of
    leading table entries that every text of the group holds at the same
    index and has filled completely.  Returns (prefix_tables as a list of
    lists, prefix_lens, tail_tables, tail_lens)."""
    S = len(context_lens)
    if group_size < 1 or S % group_size:
        raise ValueError("the number of texts must be a multiple of group_size")
    prefix_tables, prefix_lens, tail_tables, tail_lens = [], [], [], []
    for g in range(S // group_size):
        members = range(g * group_size, (g + 1) * group_size)
        first = block_tables[g * group_size]
        p = 0
        while p < len(first) and all(
                int(block_tables[s][p]) == int(first[p]) and (p + 1) * block_size <= int(context_lens[s])
                for s in members):
            p += 1
        prefix_tables.append([int(b) for b in first[:p]])
        prefix_lens.append(p * block_size)
        for s in members:
            tail = int(context_lens[s]) - p * block_size
            nb = -(-tail // block_size)
            tail_tables.append([int(b) for b in block_tables[s][p:p + nb]])
            tail_lens.append(tail)
    return prefix_tables, prefix_lens, tail_tables, tail_lens


def paged_decode_shared(q: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray,
                        prefix_tables, prefix_lens: Sequence[int], tail_tables,
                        tail_lens: Sequence[int], group_size: int, scale: float,
                        block_size: int,
                        pairs: Optional[Iterable[Tuple[int, int]]] = None) -> np.ndarray:
    """Decode attention for texts that share a prefix, fp64 ``[S][H][D]``:
    text t (group t // group_size) attends over its group's prefix tokens
    followed by its own tail tokens, i.e. the tokens of the joined table, with
    the plain definition of ``attend``.  The pools may hold fewer heads than q
    (grouped-query attention): query head h then reads key/value head
    ``kv_head_of(H, H_kv)[h]``, as in ``paged_decode``.  ``pairs`` as in
    ``paged_decode``."""
    S, H, D = q.shape
    kvh = kv_head_of(H, k_cache.shape[1])
    out = np.zeros((S, H, D), dtype=np.float64)
    wanted = None
    if pairs is not None:
        wanted = {}
        for s, h in pairs:
            wanted.setdefault(int(s), []).append(int(h))
    for t in range(S):
        if wanted is not None and t not in wanted:
            continue
        g = t // group_size
        K = np.concatenate([gather_context(k_cache, prefix_tables[g], prefix_lens[g], block_size),
                            gather_context(k_cache, tail_tables[t], tail_lens[t], block_size)])
        V = np.concatenate([gather_context(v_cache, prefix_tables[g], prefix_lens[g], block_size),
                            gather_context(v_cache, tail_tables[t], tail_lens[t], block_size)])
        heads = list(range(H)) if wanted is None else wanted[t]
        full = attend(q[t][heads], K[:, kvh[heads], :], V[:, kvh[heads], :], scale)
        for i, h in enumerate(heads):
            out[t, h] = full[i]
    return out


def prefill(q: np.ndarray, k: np.ndarray, v: np.ndarray, cu_seqlens: Sequence[int],
            scale: float) -> np.ndarray:
    """Prompt phase, fp64: every prompt's tokens attend causally over the
    prompt's own keys and values ("The KV Cache and PagedAttention", §One Token
    at a Time: the prompt is processed all at once, and its keys and values
    are what later steps reuse; "KV cache", §How it works: position t attends
    over positions 0..t).  Tokens of all prompts are packed: prompt s holds
    rows cu_seqlens[s] .. cu_seqlens[s+1]-1 of q ``[T][H][D]`` and of k, v
    ``[T][H_kv][D]`` (query head h reads key/value head ``kv_head_of``).

    For prompt s, head h and position t:
        z_u = scale * q[t] . k[u] for u <= t,  out[t] = softmax(z) . v[0..t]."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    T, H, D = q.shape
    kvh = kv_head_of(H, k.shape[1])
    out = np.zeros((T, H, D), dtype=np.float64)
    for s in range(len(cu_seqlens) - 1):
        a, b = int(cu_seqlens[s]), int(cu_seqlens[s + 1])
        L = b - a
        if L == 0:
            continue
        causal = np.tril(np.ones((L, L), dtype=bool))
        for h in range(H):
            z = float(scale) * (q[a:b, h, :] @ k[a:b, kvh[h], :].T)     # [L][L]
            z = np.where(causal, z, -np.inf)
            e = np.exp(z - z.max(axis=1, keepdims=True))
            w = e / e.sum(axis=1, keepdims=True)
            out[a:b, h, :] = w @ v[a:b, kvh[h], :]
    return out


def prefill_with_prefix(q: np.ndarray, k: np.ndarray, v: np.ndarray, cu_seqlens: Sequence[int],
                        k_cache: np.ndarray, v_cache: np.ndarray, block_tables: np.ndarray,
                        cached_lens: Sequence[int], scale: float,
                        block_size: int) -> np.ndarray:
    """Prompt phase of prompts whose first tokens are already in the paged
    cache, fp64 ("The KV Cache and PagedAttention", §What Came After: a prompt
    that begins like an earlier one reuses the earlier one's blocks, which
    saves the time spent on the prompt).

    Prompt s has ``cached_lens[s]`` tokens in the caches, found through
    ``block_tables[s]`` as in decode; its other tokens are rows
    cu_seqlens[s] .. cu_seqlens[s+1]-1 of q ``[T][H][D]`` and k, v
    ``[T][H_kv][D]``, at positions cached_lens[s] + i.  With K the cached keys
    followed by k[a:b] (V likewise), row a + i (position P = cached_lens[s] + i)
    is
        z_u = scale * q[a+i] . K[u] for u <= P,  out[a+i] = softmax(z) . V[0..P],
    i.e. the rows of the ordinary prompt phase over the whole prompt that
    belong to the new tokens."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    T, H, D = q.shape
    kvh = kv_head_of(H, k.shape[1])
    out = np.zeros((T, H, D), dtype=np.float64)
    for s in range(len(cu_seqlens) - 1):
        a, b = int(cu_seqlens[s]), int(cu_seqlens[s + 1])
        n = b - a
        if n == 0:
            continue
        c = int(cached_lens[s])
        K = np.concatenate([gather_context(k_cache, block_tables[s], c, block_size), k[a:b]])
        V = np.concatenate([gather_context(v_cache, block_tables[s], c, block_size), v[a:b]])
        allowed = np.arange(c + n)[None, :] <= (c + np.arange(n))[:, None]   # [n][c + n]
        for h in range(H):
            z = float(scale) * (q[a:b, h, :] @ K[:, kvh[h], :].T)
            z = np.where(allowed, z, -np.inf)
            e = np.exp(z - z.max(axis=1, keepdims=True))
            w = e / e.sum(axis=1, keepdims=True)
            out[a:b, h, :] = w @ V[:, kvh[h], :]
    return out


def decode_step(q, k, v, k_cache, v_cache, slot_mapping, block_tables, context_lens,
                scale, block_size, pairs=None):
    """One decode step of one layer: write the new tokens, then attend.
    Returns (out fp64, k_cache', v_cache')."""
    kc, vc = cache_write(k_cache, v_cache, k, v, slot_mapping, block_size)
    out = paged_decode(q, kc, vc, block_tables, context_lens, scale, block_size, pairs)
    return out, kc, vc
