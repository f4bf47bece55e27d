"""CPU oracle for tile-routed FP16/INT8 causal prefill attention (TileMix).

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import, call,
link or run anything in this package.  The library's product path never does:
it fails loudly when its CUDA extension is missing instead of falling back here.

The oracle is plain and slow on purpose: numpy for block quantisation
(``quant.py``, INT8 and INT4 codes), pure Python for the routing templates (``routing.py``, with its
own splitmix64), and plain C in fp64 / int64 for the attention rows
(``attention_oracle.c``, OpenMP over rows, no blocking); the decode step
(``decode.py``) composes those; ``adaptive.py`` restates the pooled-score
(content-aware) routing policy in fp32 in its stated order; ``mass.py`` is the
fp64 importance-mass exposure probe; ``fp8.py`` the e4m3 codec and block
quantiser of the FP8 low path (the C attention oracle reads those codes when
asked to).  It shares no code,
header, table or constant generator with the CUDA path.

Pages followed: "TileMix: Tile-Centric Mixed-Precision Attention for LLM
Inference Acceleration" (agihunt.info summary, method paragraphs), "Precision
Has a Map: TileMix Routes INT8 Inside Dense Attention" (cognaptus.com, sections
"Dense attention does not require uniform precision" and "The routing mechanism
is designed to stay inside the hot loop"), and the 59188saintaubert.com
explainer (steps one to three).

Pins: every function here is checked by ``tests/test_oracle_pins.py`` against
brute force, closed forms, hand-derived words and invariants the pages fix.
The attention outputs are pinned by an independent whole-matrix fp64 brute
force (``tests/bruteforce.py``: plain softmax attention for all-FP16 words, the
routed scores key by key for mixed and all-INT8 words) on small batches.  The
pages print no worked numeric example of an output, so no stored expected
output value comes from the pages.
"""
from . import adaptive, fp8, mass
from .attention import all_rows, attention_rows, build, half_to_double, int_scores
from .decode import decode_rows, quantize_rows
from .quant import quantize_blocks, quantize_k, quantize_k_int4, quantize_q, quantize_q_int4
from .routing import (BLOCK_M, BLOCK_N, MAX_GROUPS, TEMPLATES, auto_g, build_routing,
                      fp16_groups, int8_target, last_legal_tile, legal_groups, n_ktiles,
                      n_qtiles, tile_offsets)

__all__ = [
    "adaptive", "fp8", "mass", "BLOCK_M", "BLOCK_N", "MAX_GROUPS", "TEMPLATES", "all_rows", "attention_rows", "auto_g",
    "build", "build_routing", "decode_rows", "fp16_groups", "half_to_double", "int8_target",
    "int_scores",
    "last_legal_tile", "legal_groups", "n_ktiles", "n_qtiles", "quantize_blocks",
    "quantize_k", "quantize_k_int4", "quantize_q", "quantize_q_int4", "tile_offsets",
]
