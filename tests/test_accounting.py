"""The byte counts behind every bandwidth figure (CPU).

The decode's algorithmic bytes per sequence of L tokens are the K and V of
its valid tokens once per KV head (2*L*Hkv*D*sz), q in and o out
(2*Hq*D*sz), and its table entries and length (4*ceil(L/B) + 4); empty
reserved slots are not counted (page "PagedAttention Analysis", section 2:
the waste paging avoids is at most the unfilled part of a last block).
"""

from pkv_inputs import make_case
from pkv_inputs.accounting import decode_algorithmic_bytes


def test_hand_computed_example():
    # Llama-8B heads (32 q / 8 kv, d128, bf16), block 16, lengths 1, 16, 17:
    #   L=1:  2*1*8*128*2 = 4096   + q/o 16384 + table 4*1+4 = 8   -> 20488
    #   L=16: 2*16*8*128*2 = 65536 + 16384     + 8                  -> 81928
    #   L=17: 2*17*8*128*2 = 69632 + 16384     + 4*2+4 = 12         -> 86028
    assert decode_algorithmic_bytes([1, 16, 17], 32, 8, 128, 16, 2) == 20488 + 81928 + 86028


def test_partial_last_block_counts_only_its_valid_tokens():
    full = decode_algorithmic_bytes([32], 4, 4, 64, 16, 2)
    part = decode_algorithmic_bytes([31], 4, 4, 64, 16, 2)
    assert full - part == 2 * 4 * 64 * 2  # one token's K and V, nothing for the empty slot


def test_batch256_workload_bytes_are_the_recorded_ones():
    # the seeded lognormal recipe gives 222,307 tokens and 914,820,836 bytes,
    # the figures the profiles' traffic ratios are taken against
    c = make_case("llama8b_gqa_b256", with_append=False)
    lens = c.context_lens.tolist()
    assert len(lens) == 256 and sum(lens) == 222307
    assert min(lens) >= 1 and max(lens) <= 4096
    assert decode_algorithmic_bytes(lens, 32, 8, 128, 16, 2) == 914820836


def test_unique_bytes_count_a_shared_block_once():
    from pkv_inputs.accounting import unique_kv_bytes
    per_tok = 2 * 2 * 64 * 2  # Hkv 2, d64, 16-bit, K and V
    # two sequences share blocks 7 and 3 (32 tokens), then own blocks 5 and 9
    bt = [[7, 3, 5], [7, 3, 9]]
    assert unique_kv_bytes(bt, [40, 35], 16, 2, 64, 2) == (32 + 8 + 3) * per_tok
    # a block shared with different fill levels counts its fullest reader
    assert unique_kv_bytes([[4], [4]], [5, 11], 16, 2, 64, 2) == 11 * per_tok
    # no sharing: the unique bytes are the per-sequence K/V bytes
    lens = [1, 16, 17]
    bt = [[0], [1], [2, 3]]
    kv = sum(2 * L * 2 * 64 * 2 for L in lens)
    assert unique_kv_bytes(bt, lens, 16, 2, 64, 2) == kv


def test_shared_prefix_workload_unique_bytes():
    """16 prompts of 1000 tokens: 62 full blocks shared by 6 samples, and each
    sample's own 8 prompt tokens plus 64 decoded ones (fp16, 40 KV heads)."""
    from pkv_inputs import make_shared_prefix_case
    from pkv_inputs.accounting import unique_kv_bytes
    sp = make_shared_prefix_case(num_heads=4, num_kv_heads=4, head_dim=16)
    st = sp.steps[-1]
    got = unique_kv_bytes(st["block_tables"].tolist(), st["context_lens"].tolist(), 16, 4, 16, 2)
    per_tok = 2 * 4 * 16 * 2
    assert got == (16 * 992 + 96 * 72) * per_tok
