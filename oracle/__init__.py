"""fp64 CPU oracle of the NSA forward pass (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports, links or calls anything here, and this
package never imports the product package.  Inputs arrive as numpy arrays
(bf16 bit patterns as uint16, fp32 gates and weights).

Every function follows the definition written out in ``nsa_oracle.c``; the
header of that file cites the pages and lists the readings taken where the
pages are silent.  ``backward.py`` (``from oracle import backward``) holds the
fp64 gradients of that forward with the block selection held fixed, in plain
numpy; its header states the readings it takes.
"""
from .oracle import (OracleParams, build, compress, nsa_rows, nsa_query, select_f32,
                     num_cmp_blocks, prefill_reference, decode_reference, bf16_round_f64,
                     block_means, block_select_rows, block_select_reference,
                     block_select_query, block_select_decode_reference, dsa_rows, backward_c)

__all__ = ["OracleParams", "build", "compress", "nsa_rows", "nsa_query", "select_f32",
           "num_cmp_blocks", "prefill_reference", "decode_reference", "bf16_round_f64",
           "block_means", "block_select_rows", "block_select_reference",
           "block_select_query", "block_select_decode_reference", "dsa_rows", "backward_c"]
