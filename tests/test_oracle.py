"""The oracle against its pins (CPU only)."""
import numpy as np
import pytest
import torch

import oracle
from tests import oracle_pins as P


@pytest.mark.parametrize("pin", P.ATTENTION_PINS, ids=lambda f: f.__name__)
def test_attention_pin(pin):
    pin(oracle.paged_decode)


@pytest.mark.parametrize("pin", P.WRITE_PINS, ids=lambda f: f.__name__)
def test_write_pin(pin):
    pin(oracle.cache_write)


@pytest.mark.parametrize("pin", P.COPY_PINS, ids=lambda f: f.__name__)
def test_copy_pin(pin):
    pin(oracle.copy_blocks)


def test_step_writes_before_attending():
    """The token written in this step is one of the keys the query attends to
    ("KV cache", How it works: the cached keys and the new token's own)."""
    H, D, B = 2, 8, 4
    q, K, V = P.random_texts([7], H, D, 111)
    kc, vc, tables = P.scatter_to_pool([K[0][:6]], [V[0][:6]], B, 4, 111)
    slot = int(tables[0, 6 // B]) * B + 6 % B
    out, kc2, vc2 = oracle.decode_step(P.f64(q), P.f64(K[0][6:7]), P.f64(V[0][6:7]), P.f64(kc),
                                       P.f64(vc), [slot], tables, [7], 0.3, B)
    ref = P.sdpa_contiguous(q, K, V, 0.3)
    assert np.abs(out - ref).max() <= 1e-12


def test_pairs_subset_matches_full():
    H, D, B = 3, 8, 4
    lens = [5, 9, 16]
    q, K, V = P.random_texts(lens, H, D, 121)
    kc, vc, tables = P.scatter_to_pool(K, V, B, 16, 121)
    full = oracle.paged_decode(P.f64(q), P.f64(kc), P.f64(vc), tables, lens, 0.3, B)
    pairs = [(0, 2), (2, 0), (2, 1), (1, 1)]
    part = oracle.paged_decode(P.f64(q), P.f64(kc), P.f64(vc), tables, lens, 0.3, B, pairs=pairs)
    for s, h in pairs:
        assert np.array_equal(full[s, h], part[s, h])


def test_tiny_workload_runs_and_is_finite():
    """The tiny workload end to end through the oracle: NaN poison in unused
    rows never reaches the output."""
    from paged_kv_cache_326_b200 import workloads as W
    w = W.tiny(device="cpu")
    out, kc, vc = oracle.decode_step(
        P.f64(w.q), P.f64(w.k), P.f64(w.v), P.f64(w.k_cache), P.f64(w.v_cache),
        w.slot_mapping.numpy(), w.block_tables.numpy(), w.context_lens.numpy(), w.scale,
        w.block_size)
    assert out.shape == (4, 8, 64) and np.isfinite(out).all()


@pytest.mark.parametrize("pin", P.GQA_PINS, ids=lambda f: f.__name__)
def test_gqa_pin(pin):
    pin(oracle.paged_decode)


def test_kv_head_of_rejects_uneven_groups():
    with pytest.raises(ValueError):
        oracle.kv_head_of(6, 4)
    assert list(oracle.kv_head_of(8, 2)) == [0, 0, 0, 0, 1, 1, 1, 1]


def test_e4m3_codes_match_torch_on_every_fp16_value():
    P.pin_e4m3_every_fp16_vs_torch(oracle.e4m3_encode)


def test_e4m3_codes_match_torch_on_random_fp32():
    P.pin_e4m3_random_fp32_vs_torch(oracle.e4m3_encode)


def test_e4m3_closed_forms():
    P.pin_e4m3_closed_forms(oracle.e4m3_encode, oracle.e4m3_decode)


def test_fp8_attention_on_representable_values():
    P.pin_fp8_attention_on_representable_values(oracle.paged_decode_fp8, oracle.quantize)


def test_fp8_cache_write_matches_hand_worked_golden():
    """The 8-bit write against codes worked out by hand from the E4M3 format
    (tests/golden/cache_write_fp8_tiny.json): division by the scale, ties to
    the even mantissa, saturation at 448, subnormals, negative zero, the
    slot's block and place, a skipped padding token, untouched rows."""
    import json
    import os
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                    "cache_write_fp8_tiny.json")))
    shape = (g["num_blocks"], g["num_heads"], g["block_size"], g["head_dim"])
    kc = np.full(shape, g["fill"], dtype=np.uint8)
    vc = np.full(shape, g["fill"], dtype=np.uint8)
    k = np.array(g["k"], dtype=np.float32)
    v = np.array(g["v"], dtype=np.float32)
    k2, v2 = oracle.cache_write_fp8(kc, vc, k, v, g["slot_mapping"], g["block_size"],
                                    g["k_scale"], g["v_scale"])
    assert k2.tolist() == g["expected_k_cache"]
    assert v2.tolist() == g["expected_v_cache"]


@pytest.mark.parametrize("pin", P.PREFILL_PINS, ids=lambda f: f.__name__)
def test_prefill_pin(pin):
    pin(oracle.prefill)


@pytest.mark.parametrize("pin", P.PREFIX_PINS, ids=lambda f: f.__name__)
def test_prefill_with_prefix_pin(pin):
    pin(oracle.prefill_with_prefix)


@pytest.mark.parametrize("pin", P.SHARED_PINS, ids=lambda f: f.__name__)
def test_shared_prefix_oracle_pin(pin):
    pin(oracle.paged_decode_shared)


@pytest.mark.parametrize("pin", P.SPLIT_PINS, ids=lambda f: f.__name__)
def test_split_oracle_pin(pin):
    pin(oracle.split_shared_prefix)


def test_split_then_shared_is_paged_decode():
    P.pin_split_then_shared_is_decode(oracle.split_shared_prefix, oracle.paged_decode_shared)
