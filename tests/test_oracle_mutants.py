"""Each copy of the oracle below has one planted mistake of the kind a
careless implementation makes; the pins must catch every one (CPU only)."""
import numpy as np
import pytest

import oracle
from tests import oracle_pins as P


def _decode_with(attend_fn=None, gather_fn=None, len_fn=None):
    attend_fn = attend_fn or oracle.attend
    gather_fn = gather_fn or oracle.gather_context
    len_fn = len_fn or (lambda L: L)

    def fn(q, k_cache, v_cache, block_tables, context_lens, scale, block_size):
        S, H, D = q.shape
        out = np.zeros((S, H, D))
        for s in range(S):
            L = len_fn(int(context_lens[s]))
            K = gather_fn(k_cache, block_tables[s], L, block_size)
            V = gather_fn(v_cache, block_tables[s], L, block_size)
            out[s] = attend_fn(q[s], K, V, scale)
        return out
    return fn


def gather_swapped_index(cache, table, L, B):
    H, D = cache.shape[1], cache.shape[3]
    out = np.empty((L, H, D))
    for t in range(L):
        out[t] = cache[int(table[t % B]) if t % B < len(table) else 0, :, min(t // B, B - 1), :]
    return out


def gather_off_by_one_place(cache, table, L, B):
    H, D = cache.shape[1], cache.shape[3]
    out = np.empty((L, H, D))
    for t in range(L):
        out[t] = cache[int(table[t // B]), :, (t + 1) % B, :]
    return out


def attend_no_scale(q, K, V, scale):
    return oracle.attend(q, K, V, 1.0)


def attend_k_v_swapped(q, K, V, scale):
    return oracle.attend(q, V, K, scale)


def attend_unnormalised(q, K, V, scale):
    H, D = q.shape
    out = np.zeros((H, D))
    for h in range(H):
        z = scale * (K[:, h, :] @ q[h])
        out[h] = np.exp(z - z.max()) @ V[:, h, :]
    return out


def attend_wrong_head(q, K, V, scale):
    H = q.shape[0]
    return oracle.attend(q, K[:, [(h + 1) % H for h in range(H)], :], V, scale)


def attend_mean_of_keys(q, K, V, scale):
    H, D = q.shape
    out = np.zeros((H, D))
    for h in range(H):
        z = scale * (K[:, h, :] @ q[h])
        w = np.exp(z - z.max())
        out[h] = (w / w.sum()) @ K[:, h, :]
    return out


def attend_weights_transposed_sign(q, K, V, scale):
    return oracle.attend(-q, K, V, scale)


MUTANTS = {
    "block/place swapped": _decode_with(gather_fn=gather_swapped_index),
    "place off by one": _decode_with(gather_fn=gather_off_by_one_place),
    "scale dropped": _decode_with(attend_fn=attend_no_scale),
    "K and V swapped": _decode_with(attend_fn=attend_k_v_swapped),
    "softmax not normalised": _decode_with(attend_fn=attend_unnormalised),
    "wrong head's keys": _decode_with(attend_fn=attend_wrong_head),
    "keys mixed instead of values": _decode_with(attend_fn=attend_mean_of_keys),
    "score sign flipped": _decode_with(attend_fn=attend_weights_transposed_sign),
    "new token left out": _decode_with(len_fn=lambda L: max(L - 1, 0)),
}


def _fails_some_pin(fn):
    failed = []
    for pin in P.ATTENTION_PINS:
        try:
            pin(fn)
        except (AssertionError, IndexError, ValueError):
            failed.append(pin.__name__)
    return failed


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_attention_mistake_is_caught(name):
    assert _fails_some_pin(MUTANTS[name]), f"no pin catches: {name}"


def test_unmodified_oracle_passes_all_pins():
    assert _fails_some_pin(oracle.paged_decode) == []


def write_block_place_swapped(kc, vc, k, v, slots, B):
    kc, vc = kc.copy(), vc.copy()
    for t, s in enumerate(slots):
        if s < 0:
            continue
        place, block = divmod(int(s), B)
        if place < kc.shape[2] and block < kc.shape[0]:
            kc[block, :, place, :] = k[t]
            vc[block, :, place, :] = v[t]
    return kc, vc


def write_ignores_negative_check(kc, vc, k, v, slots, B):
    kc, vc = kc.copy(), vc.copy()
    for t, s in enumerate(slots):
        block, place = divmod(int(s), B)
        kc[block, :, place, :] = k[t]
        vc[block, :, place, :] = v[t]
    return kc, vc


def write_k_into_v(kc, vc, k, v, slots, B):
    return oracle.cache_write(kc, vc, v, k, slots, B)


@pytest.mark.parametrize("fn", [write_block_place_swapped, write_ignores_negative_check,
                                write_k_into_v], ids=lambda f: f.__name__)
def test_planted_write_mistake_is_caught(fn):
    failed = 0
    for pin in P.WRITE_PINS:
        try:
            pin(fn)
        except (AssertionError, IndexError):
            failed += 1
    assert failed, fn.__name__


def decode_gqa_heads_by_modulo(q, k_cache, v_cache, block_tables, context_lens, scale, B):
    """Planted mistake: query head h reads key/value head h % H_kv."""
    S, H, D = q.shape
    kvh = np.arange(H) % k_cache.shape[1]
    out = np.zeros((S, H, D))
    for s in range(S):
        K = oracle.gather_context(k_cache, block_tables[s], context_lens[s], B)
        V = oracle.gather_context(v_cache, block_tables[s], context_lens[s], B)
        out[s] = oracle.attend(q[s], K[:, kvh, :], V[:, kvh, :], scale)
    return out


def test_planted_gqa_head_mapping_mistake_is_caught():
    failed = []
    for pin in P.GQA_PINS:
        try:
            pin(decode_gqa_heads_by_modulo)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed


def test_unmodified_oracle_passes_gqa_pins():
    for pin in P.GQA_PINS:
        pin(oracle.paged_decode)


# --- block copies: planted mistakes -------------------------------------------

def copy_swaps_src_and_dst(sk, sv, dk, dv, pairs):
    return oracle.copy_blocks(sk, sv, dk, dv, [(d, s) for s, d in pairs])


def copy_k_into_v(sk, sv, dk, dv, pairs):
    return oracle.copy_blocks(sk, sk, dk, dv, pairs)


def copy_first_head_only(sk, sv, dk, dv, pairs):
    kd, vd = dk.copy(), dv.copy()
    for s, d in pairs:
        kd[d, 0] = sk[s, 0]
        vd[d, 0] = sv[s, 0]
    return kd, vd


def copy_misses_last_place(sk, sv, dk, dv, pairs):
    kd, vd = dk.copy(), dv.copy()
    for s, d in pairs:
        kd[d, :, :-1] = sk[s, :, :-1]
        vd[d, :, :-1] = sv[s, :, :-1]
    return kd, vd


def copy_in_place_sequentially(sk, sv, dk, dv, pairs):
    """Writes into the source arrays themselves (a later pair may then read
    an earlier pair's result)."""
    for s, d in pairs:
        dk[d] = sk[s]
        dv[d] = sv[s]
    return dk, dv


@pytest.mark.parametrize("fn", [copy_swaps_src_and_dst, copy_k_into_v, copy_first_head_only,
                                copy_misses_last_place, copy_in_place_sequentially],
                         ids=lambda f: f.__name__)
def test_planted_copy_mistake_is_caught(fn):
    failed = 0
    for pin in P.COPY_PINS:
        try:
            pin(fn)
        except (AssertionError, IndexError):
            failed += 1
    assert failed, fn.__name__


def test_unmodified_oracle_passes_copy_pins():
    for pin in P.COPY_PINS:
        pin(oracle.copy_blocks)



# --- 8-bit cache: planted mistakes --------------------------------------------

def _encode_variant(x, ties_even=True, saturate=True, keep_sign=True):
    """The E4M3 rounding with one rule changed (a planted mistake)."""
    vals = np.array([oracle.e4m3_value(c) for c in range(0x7F)])
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros(x.shape, dtype=np.uint8)
    for i, v in np.ndenumerate(x):
        if np.isnan(v):
            out[i] = 0x7F
            continue
        a = abs(v)
        if a > 448.0 and not saturate:
            out[i] = 0x7F
            continue
        a = min(a, 448.0)
        hi = int(np.searchsorted(vals, a))
        lo = max(hi - 1, 0)
        if vals[hi] == a:
            c = hi
        elif a - vals[lo] < vals[hi] - a:
            c = lo
        elif a - vals[lo] > vals[hi] - a:
            c = hi
        else:
            c = (lo if lo % 2 == 0 else hi) if ties_even else hi
        out[i] = (0x80 if (np.signbit(v) and keep_sign) else 0) | c
    return out


def encode_ties_away(x):
    return _encode_variant(x, ties_even=False)


def encode_without_saturation(x):
    return _encode_variant(x, saturate=False)


def encode_drops_sign(x):
    return _encode_variant(x, keep_sign=False)


def test_planted_e4m3_encoding_mistakes_are_caught():
    for fn in (encode_ties_away, encode_without_saturation, encode_drops_sign):
        failed = 0
        for pin in (P.pin_e4m3_every_fp16_vs_torch,
                    lambda e: P.pin_e4m3_closed_forms(e, oracle.e4m3_decode)):
            try:
                pin(fn)
            except AssertionError:
                failed += 1
        assert failed, fn.__name__


def decode_with_bias_8(codes):
    return oracle.e4m3_decode(codes) / 2.0


def test_planted_e4m3_decoding_mistake_is_caught():
    with pytest.raises(AssertionError):
        P.pin_e4m3_closed_forms(oracle.e4m3_encode, decode_with_bias_8)


def quantize_multiplying(x, scale):
    return oracle.e4m3_encode(np.asarray(x, dtype=np.float32) * np.float32(scale))


def test_planted_scale_mistake_is_caught():
    with pytest.raises(AssertionError):
        P.pin_fp8_attention_on_representable_values(oracle.paged_decode_fp8, quantize_multiplying)


# --- prompt phase: planted mistakes -------------------------------------------

def prefill_not_causal(q, k, v, cu, scale):
    """Planted mistake: every position sees the whole prompt."""
    out = np.zeros(q.shape)
    for s in range(len(cu) - 1):
        a, b = cu[s], cu[s + 1]
        for t in range(a, b):
            out[t] = oracle.attend(q[t], k[a:b], v[a:b], scale)
    return out


def prefill_excludes_self(q, k, v, cu, scale):
    """Planted mistake: position t sees 0..t-1 only (the first sees nothing)."""
    out = np.zeros(q.shape)
    for s in range(len(cu) - 1):
        a, b = cu[s], cu[s + 1]
        for t in range(a, b):
            out[t] = oracle.attend(q[t], k[a:t], v[a:t], scale)
    return out


def prefill_crosses_prompts(q, k, v, cu, scale):
    """Planted mistake: the prompts are treated as one long prompt."""
    return oracle.prefill(q, k, v, [0, cu[-1]], scale)


@pytest.mark.parametrize("fn", [prefill_not_causal, prefill_excludes_self,
                                prefill_crosses_prompts], ids=lambda f: f.__name__)
def test_planted_prefill_mistake_is_caught(fn):
    failed = 0
    for pin in P.PREFILL_PINS:
        try:
            pin(fn)
        except (AssertionError, ValueError, IndexError):
            failed += 1
    assert failed, fn.__name__


# --- prompt phase over a stored prefix: planted mistakes ---------------------

def prefix_ignored(q, k, v, cu, kc, vc, tables, cached, scale, B):
    """Planted mistake: the stored prefix is left out."""
    return oracle.prefill(q, k, v, cu, scale)


def prefix_offset_dropped(q, k, v, cu, kc, vc, tables, cached, scale, B):
    """Planted mistake: new row i sees keys 0..i of the joined list, as if it
    sat at position i instead of cached + i."""
    out = np.zeros(q.shape)
    for s in range(len(cu) - 1):
        a, b, c = int(cu[s]), int(cu[s + 1]), int(cached[s])
        K = np.concatenate([oracle.gather_context(kc, tables[s], c, B), k[a:b]])
        V = np.concatenate([oracle.gather_context(vc, tables[s], c, B), v[a:b]])
        kvh = oracle.kv_head_of(q.shape[1], k.shape[1])
        for i in range(b - a):
            out[a + i] = oracle.attend(q[a + i], K[:i + 1][:, kvh], V[:i + 1][:, kvh], scale)
    return out


def prefix_sees_the_future(q, k, v, cu, kc, vc, tables, cached, scale, B):
    """Planted mistake: new rows see every new token, not just the earlier ones."""
    out = np.zeros(q.shape)
    for s in range(len(cu) - 1):
        a, b, c = int(cu[s]), int(cu[s + 1]), int(cached[s])
        K = np.concatenate([oracle.gather_context(kc, tables[s], c, B), k[a:b]])
        V = np.concatenate([oracle.gather_context(vc, tables[s], c, B), v[a:b]])
        kvh = oracle.kv_head_of(q.shape[1], k.shape[1])
        for i in range(b - a):
            out[a + i] = oracle.attend(q[a + i], K[:, kvh], V[:, kvh], scale)
    return out


def prefix_gathered_block_major(q, k, v, cu, kc, vc, tables, cached, scale, B):
    """Planted mistake: a stored token's row is taken as place t // B of
    block table[t % B] (the block and place indices swapped)."""
    def gather(cache, table, c):
        out = np.empty((c, cache.shape[1], cache.shape[3]))
        for t in range(c):
            out[t] = cache[int(table[min(t % B, len(table) - 1)]), :, min(t // B, B - 1), :]
        return out
    out = np.zeros(q.shape)
    kvh = oracle.kv_head_of(q.shape[1], k.shape[1])
    for s in range(len(cu) - 1):
        a, b, c = int(cu[s]), int(cu[s + 1]), int(cached[s])
        K = np.concatenate([gather(kc, tables[s], c), k[a:b]])
        V = np.concatenate([gather(vc, tables[s], c), v[a:b]])
        for i in range(b - a):
            out[a + i] = oracle.attend(q[a + i], K[:c + i + 1][:, kvh], V[:c + i + 1][:, kvh],
                                       scale)
    return out


@pytest.mark.parametrize("fn", [prefix_ignored, prefix_offset_dropped, prefix_sees_the_future,
                                prefix_gathered_block_major], ids=lambda f: f.__name__)
def test_planted_prefix_prefill_mistake_is_caught(fn):
    failed = 0
    for pin in P.PREFIX_PINS:
        try:
            pin(fn)
        except (AssertionError, ValueError, IndexError):
            failed += 1
    assert failed, fn.__name__


# --- shared prefixes: planted mistakes ----------------------------------------

def _shared_with(group_of=None, use_prefix=True, use_tail=True):
    def fn(q, kc, vc, pt, pl, tt, tl, gs, scale, B):
        S, H, D = q.shape
        out = np.zeros((S, H, D))
        G = len(pl)
        for t in range(S):
            g = group_of(t, gs, G) if group_of else t // gs
            parts_k, parts_v = [], []
            if use_prefix:
                parts_k.append(oracle.gather_context(kc, pt[g], pl[g], B))
                parts_v.append(oracle.gather_context(vc, pt[g], pl[g], B))
            if use_tail:
                parts_k.append(oracle.gather_context(kc, tt[t], tl[t], B))
                parts_v.append(oracle.gather_context(vc, tt[t], tl[t], B))
            K = np.concatenate(parts_k) if parts_k else np.zeros((0, H, D))
            V = np.concatenate(parts_v) if parts_v else np.zeros((0, H, D))
            out[t] = oracle.attend(q[t], K, V, scale)
        return out
    return fn


def _shared_head_map_mod():
    """Grouped-query mistake: query head h reads key/value head h % H_kv
    instead of h // (H / H_kv)."""
    def fn(q, kc, vc, pt, pl, tt, tl, gs, scale, B):
        S, H, D = q.shape
        Hkv = kc.shape[1]
        out = np.zeros((S, H, D))
        for t in range(S):
            g = t // gs
            K = np.concatenate([oracle.gather_context(kc, pt[g], pl[g], B),
                                oracle.gather_context(kc, tt[t], tl[t], B)])
            V = np.concatenate([oracle.gather_context(vc, pt[g], pl[g], B),
                                oracle.gather_context(vc, tt[t], tl[t], B)])
            heads = np.arange(H) % Hkv
            out[t] = oracle.attend(q[t], K[:, heads, :], V[:, heads, :], scale)
        return out
    return fn


SHARED_MUTANTS = {
    "prefix_of_wrong_group": _shared_with(group_of=lambda t, gs, G: t % G),
    "prefix_dropped": _shared_with(use_prefix=False),
    "tail_dropped": _shared_with(use_tail=False),
    "grouped_query_head_map_mod": _shared_head_map_mod(),
}


@pytest.mark.parametrize("name", sorted(SHARED_MUTANTS))
def test_planted_shared_prefix_mistake_is_caught(name):
    failed = 0
    for pin in P.SHARED_PINS:
        try:
            pin(SHARED_MUTANTS[name])
        except (AssertionError, ValueError, IndexError):
            failed += 1
    assert failed, name


def split_ignores_fill(bt, lens, B, gs):
    """Planted mistake: a shared block counts even when partly filled."""
    S = len(lens)
    pt, pl, tt, tl = [], [], [], []
    for g in range(S // gs):
        first = bt[g * gs]
        p = 0
        while p < len(first) and first[p] >= 0 and all(bt[s][p] == first[p]
                                                       for s in range(g * gs, (g + 1) * gs)):
            p += 1
        pt.append([int(b) for b in first[:p]])
        pl.append(min(p * B, min(lens[g * gs:(g + 1) * gs])))
        for s in range(g * gs, (g + 1) * gs):
            rest = lens[s] - pl[-1]
            tt.append([int(b) for b in bt[s][p:p + -(-rest // B)]])
            tl.append(rest)
    return pt, pl, tt, tl


def split_first_member_only(bt, lens, B, gs):
    """Planted mistake: the prefix is read off the group's first table only."""
    S = len(lens)
    pt, pl, tt, tl = [], [], [], []
    for g in range(S // gs):
        first = bt[g * gs]
        p = 0
        while p < len(first) and (p + 1) * B <= lens[g * gs]:
            p += 1
        pt.append([int(b) for b in first[:p]])
        pl.append(p * B)
        for s in range(g * gs, (g + 1) * gs):
            rest = lens[s] - p * B
            tt.append([int(b) for b in bt[s][p:p + -(-rest // B)]])
            tl.append(rest)
    return pt, pl, tt, tl


@pytest.mark.parametrize("fn", [split_ignores_fill, split_first_member_only],
                         ids=lambda f: f.__name__)
def test_planted_split_mistake_is_caught(fn):
    failed = 0
    for pin in P.SPLIT_PINS:
        try:
            pin(fn)
        except (AssertionError, ValueError, IndexError):
            failed += 1
    assert failed, fn.__name__


def test_unmodified_oracle_passes_shared_pins():
    for pin in P.SHARED_PINS:
        pin(oracle.paged_decode_shared)
    for pin in P.SPLIT_PINS:
        pin(oracle.split_shared_prefix)
