"""Float64 CPU oracle for the IndexCache decode path. TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The product (the C-ABI library and its
Python binding under ``lightning_indexer_cross_b200``) never imports, calls or
links it, and it shares no code with the CUDA path: it reads the same seeded
input tensors and nothing else.

Every function is a plain, slow, obviously-correct restatement of what the
pages describe; see ``indexcache_oracle`` for the per-function citations and
the readings taken where the pages are silent.
"""
from .indexcache_oracle import (  # noqa: F401
    decode_e4m3,
    indexer_scores,
    topk_indices,
    sparse_mla,
    dense_sink_attention,
    layer_stack,
    validate_schedule,
    governing_full_layer,
    index_overlap,
    reuse_overlap,
)
from .cache_append_oracle import (  # noqa: F401
    layernorm_bias,
    encode_e4m3,
    rope_interleaved,
    quantize_key_e4m3,
    cache_append,
    rope_query,
)
from .gate_oracle import decompress, decompressed_gate  # noqa: F401
