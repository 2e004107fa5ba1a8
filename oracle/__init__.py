"""CPU oracle of the KIVI cache and decode attention.

TEST INFRASTRUCTURE ONLY.  ``tests/``, the package's ``smoke()`` check and the
benchmark's CPU-baseline leg may import it; the library path never does, and
nothing here imports the CUDA library.  The arithmetic lives in the plain C file
``kivi_oracle.c`` (built on demand with gcc); this package holds its ctypes
wrapper, the cache state machine and the pages' byte arithmetic.
"""
from .oracle import (  # noqa: F401
    G,
    R,
    OracleCache,
    attend_one,
    attention_bf16,
    cache_bytes,
    dequant_record,
    f16_bits_to_double,
    fake_quant_keys,
    f32_to_f16_bits,
    make_record,
    prefill_attention,
    num_groups,
    quantize_group,
    record_bytes,
)
