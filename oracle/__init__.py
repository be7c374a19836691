"""fp64 CPU oracle for exact attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, the smoke check and the benchmark's CPU-baseline legs may
import this package.  The product (the CUDA library and its Python binding)
never imports it and has no CPU fallback.
"""
from .attention import (ROW_CHUNK, as_f64, attention_backward,  # noqa: F401
                        attention_forward, attention_probs,
                        online_softmax_forward, printed_block_sum_forward,
                        scores, softmax_rows)
