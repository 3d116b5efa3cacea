"""Seeded synthetic inputs for paged decode attention, shared by both sides.

This package builds the inputs that the CUDA path and the CPU oracle both
consume: query vectors, the physical K/V pools, block tables, context lengths,
slot mappings and copy-on-write pairs. It holds none of the attention
arithmetic. Every value comes from a seeded generator (``numpy`` for lengths
and placements, ``torch`` for the normal q/K/V draws), so both sides see the
same bytes.

Modules:

* ``workloads`` - the five decode workloads and a generic random case builder.
* ``block_manager`` - the host-side refcounted block allocator with
  copy-on-write, used only to decide block placement and CoW copies for test
  inputs.
* ``accounting`` - byte counts used for the bandwidth figures.
"""

from .block_manager import (  # noqa: F401
    BeamSearch, BlockAllocator, BlockMove, CowCopy, PrefixCache, SeqState, SwapSpace)
from .workloads import (  # noqa: F401
    make_beam_search_case, make_prefix_cache_case,
    DecodeCase,
    POOL_LAYOUT,
    WORKLOADS,
    make_case,
    make_random_case,
    make_sharing_case,
    make_shared_prefix_case,
    nan_fill_value,
)
from .accounting import (  # noqa: F401
    decode_algorithmic_bytes,
    kv_bytes_per_token,
    unique_kv_bytes,
)
