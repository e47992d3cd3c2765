"""fp64 CPU oracle for exact attention (test infrastructure, never on the product path).

Only tests, the smoke check and the bench's CPU-baseline leg import this
package.  It shares no code with the CUDA library.
"""

from .attention import (attention, attention_bwd, attention_fp8, decode_paged, decode_paged_gqa, decode_paged_mtp,
                        e4m3_decode, gather_pages)

__all__ = ["attention", "attention_bwd", "attention_fp8", "decode_paged", "decode_paged_gqa", "decode_paged_mtp",
           "e4m3_decode", "gather_pages"]
