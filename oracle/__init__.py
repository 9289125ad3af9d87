"""CPU fp64 oracle (test infrastructure only; never imported by the library)."""
from .attn import (allowed_mask, attn_probs, attn_fwd, attn_rows, attn_bwd, attn_decode,
                   attn_decode_paged, attn_decode_append, paged_rows,
                   merge_partials, fwd_flops, allowed_pairs, score_matrix_elements)
