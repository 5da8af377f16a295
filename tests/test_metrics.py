"""The algorithmic bytes behind every roofline fraction (CPU).

Each figure is the sum written out by hand from its terms: the bf16 state read
and written once per touched (item, value head), the per-token inputs (q and
k once per query/key head, v, gk and g/beta or a/b per value head), the bf16
output for every (item, head, token) including padding, and the per-item
int32 scalars (plus the per-head gate vectors when the gate is fused).
"""
from gated_delta_rule_recurrent_b200.metrics import algorithmic_bytes, flops


def test_large_batch_gated_step():
    # B = 512 items, 64 q/k and value heads, T = 1, 64 x 512 state, fused gate
    state = 2 * 2 * 64 * 512 * (512 * 64)
    per_token = 2 * 64 * 64 * 2 + 64 * (2 * 512 + 4 * 64 + 2 + 2)
    out = 2 * 512 * 64 * 1 * 512
    scalars = 12 * 512 + 8 * 64
    assert state + 512 * per_token + out + scalars == 4_378_991_104
    assert algorithmic_bytes(512, 64, 64, 1, 64, 512, [1] * 512, True) == 4_378_991_104


def test_grouped_heads_plain_step():
    # B = 64, 16 q/k heads, 32 value heads, T = 1, 128 x 128, g and beta given
    state = 2 * 2 * 128 * 128 * (64 * 32)
    per_token = 2 * 16 * 128 * 2 + 32 * (2 * 128 + 4 * 128 + 4 + 2)
    out = 2 * 64 * 32 * 128
    assert state + 64 * per_token + out + 12 * 64 == 136_852_224
    assert algorithmic_bytes(64, 16, 32, 1, 128, 128, [1] * 64, False) == 136_852_224


def test_padding_and_empty_items():
    # padded tokens' inputs are not read, but their outputs are written; an
    # item with no valid token touches no state
    base = algorithmic_bytes(2, 1, 1, 4, 8, 8, [4, 4], False)
    ragged = algorithmic_bytes(2, 1, 1, 4, 8, 8, [4, 0], False)
    per_token = 2 * 1 * 8 * 2 + 1 * (2 * 8 + 4 * 8 + 4 + 2)
    state_one = 2 * 2 * 8 * 8
    assert base - ragged == 4 * per_token + state_one
    # lengths are clamped to [0, T]
    assert algorithmic_bytes(2, 1, 1, 4, 8, 8, [9, -3], False) == ragged


def test_flops_per_state_element():
    assert flops(4, 8, 16, [3, 1, 0], 4) == 7 * 8 * 16 * 4 * 4
