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
