"""Plain, slow, fp64 CPU oracle for the dictionary-coded KV cache.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It
shares no code with the CUDA path (no kernels, headers, helpers or
constants) and imports nothing from the product package.

Method source: "LLM Inference in a Flash!" (Zhao, Kim, Hooper, Manolache,
Mahoney, Shao, Keutzer, Gholami), as described by the authors' abstract
(readsearch.ai listing) and by the evolve.pub review of the paper (sections
"Summary", "Key claims under review" and the FAQ entry on the 15x KV cache
compression).

Modules
-------
encode   greedy pursuit (the projection-based replacement for OMP), the
         fp16 coefficient storage rule and the 32-bit code word format.
decode   decode attention with query-aware hierarchical sparsity, written
         as the plain definition over decoded key/value vectors; optional
         integer softmax (token-wise INT16 logits, integer exponential).
certify  replay of someone else's codes in fp64: checks every greedy pick.
omp      orthogonal matching pursuit (least-squares refit at every step), the
         encoder the pages replace; only for measuring what the greedy
         pursuit gives up (``python -m oracle.compare_omp``).

Pins: every function here is checked in ``tests/test_oracle_*.py`` against
facts fixed by the pages or by mathematics (brute force on tiny inputs,
exact recovery, the energy identity, dense attention as a special case).
One quantity is "parity unpinned": the pages' 15x dynamic-KV compression
figure, whose code bit widths the pages do not give.
"""

from .encode import (FP16_MAX, greedy_pursuit, encode_ref, store_coef_fp16,
                     pack_words, unpack_words)
from .decode import (topk_count, select_top, decode_attn_ref,
                     decode_head_ref, decode_vectors, integer_softmax)
from .certify import certify_codes, certify_codes_batched
from .omp import omp, omp_ref

__all__ = [
    "FP16_MAX", "greedy_pursuit", "encode_ref", "store_coef_fp16",
    "pack_words", "unpack_words", "topk_count", "select_top",
    "decode_attn_ref", "decode_head_ref", "decode_vectors", "certify_codes", "certify_codes_batched",
    "omp", "omp_ref", "integer_softmax",
]
