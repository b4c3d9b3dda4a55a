"""CPU oracle for packed mixed-precision KV-cache decode attention.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the CPU
baseline / reference arm of ``bench.py`` may import it; the library never does.
Functions without an independent pin are marked "parity unpinned" in their
docstrings (none at present).
"""
from .kvq_oracle import (  # noqa: F401
    MAX_RETAINED, OracleCache, attention, buffer_bytes, dequantize, max_rel_error,
    minmax_quantize, pack_codes, quantize_keys, quantize_values, quantized_prefix,
    retained_positions, unpack_codes,
)
