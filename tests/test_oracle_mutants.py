"""Each planted mistake in the oracle must make at least one pin fail (CPU only).

The variants are compiled from the oracle's own source with -DORACLE_MUTANT=k:
 1 GQA head mapping h % Hkv instead of h / G
 2 causal mask drops the diagonal key
 3 softmax scale dropped
 4 offset inside a block shifted by one
 5 causal mask aligned top-left (ignores the cached prefix)
 6 block size hard-wired to 256 in the page index
 7 slot -1 written to slot 0 instead of skipped
 8 bf16 output truncated instead of rounded to nearest-even
 9 softmax normalisation (division by the sum) dropped
10 split-KV merge without the exp(m_c - M) rescaling
11 rotary embedding pairs adjacent elements instead of the two halves
12 rotary table holds -sin (rotation by the negative angle)
13 rotary frequency exponent -i/D instead of -2i/D
14 fused rotary store writes the key unrotated
15 rotary embedding reads the table row of position + 1
"""
import pytest

from oracle import oracle as O
import test_oracle_pins as P
import test_oracle_rope as R

PINS = [
    (P.test_page_table_worked_example, {}),
    (P.test_store_then_gather_round_trip, {}),
    (P.test_store_skips_minus_one_and_touches_nothing_else, {}),
    (P.test_bf16_rounding_matches_torch, {}),
    (P.test_decode_matches_torch_sdpa, dict(lens=[5, 33, 64, 1, 100], hq=8, hkv=2, d=128, bs=16)),
    (P.test_decode_matches_torch_sdpa, dict(lens=[1, 17, 256, 300], hq=4, hkv=2, d=64, bs=256)),
    (P.test_decode_equal_keys_give_mean_value, {}),
    (P.test_decode_single_key_returns_value_row, {}),
    (P.test_split_merge_identity, dict(chunk=16)),
    (P.test_prefill_matches_torch_sdpa, dict(prefix=32, sfx=[5, 17, 1], causal=True, hq=4, hkv=2, d=64, bs=16)),
    (P.test_prefill_shared_vs_duplicated_prefix, {}),
    (R.test_rope_table_worked_example, {}),
    (R.test_rope_table_frequencies_are_geometric, dict(d=64, base=1e4)),
    (R.test_rope_is_complex_rotation_of_the_halves, dict(d=64)),
    (R.test_rope_position_zero_is_identity, {}),
    (R.test_rope_store_writes_rotated_key_and_raw_value, {}),
]


@pytest.mark.parametrize("mutant", list(range(1, 16)))
def test_planted_mistake_is_caught(mutant):
    bad = O.Oracle(mutant)
    caught = []
    for fn, kw in PINS:
        try:
            fn(bad, **kw)
        except (AssertionError, ValueError):
            caught.append(fn.__name__)
    assert caught, f"planted mistake {mutant} passed every pin"
