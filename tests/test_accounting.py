"""The byte accounting used by the bench against the pages' worked numbers."""
from paged_kv_cache_326_b200.accounting import decode_kv_bytes, kv_bytes_per_token, tokens_that_fit
from tests.oracle_pins import load_golden


def test_opt13b_token_bytes():
    g = load_golden("kv_bytes.json")["opt13b"]
    b = kv_bytes_per_token(g["kv_heads"], g["head_dim"], g["layers"], g["elem_bytes"])
    assert b == g["bytes_per_token"]
    assert round(2048 * b / 1e9, 1) in (1.6, 1.7) and abs(2048 * b / 2**30 - 1.5625) < 1e-9
    n = tokens_that_fit(12 * 2**30, g["kv_heads"], g["head_dim"], g["layers"], g["elem_bytes"])
    assert n == g["tokens_in_12_gib"]
    assert n // 2048 == g["texts_of_2048_in_12_gib"]


def test_shared_kv_sets():
    for name in ("llama2_70b", "falcon_7b"):
        g = load_golden("kv_bytes.json")[name]
        b = kv_bytes_per_token(g["kv_heads"], g["head_dim"], g["layers"], g["elem_bytes"])
        assert b == g["bytes_per_token_kib"] * 1024


def test_decode_bytes_counts_every_stored_token():
    assert decode_kv_bytes([5, 9, 16, 23], 8, 64, 2) == 53 * 2 * 8 * 64 * 2
