"""B200 (sm_100a) TurboQuant inner-product quantizer: encode vectors to
(b-1)-bit Lloyd-Max indices + 1 QJL sign bit per coordinate after a random
rotation, and estimate inner products / top-k directly from the packed codes;
also the MSE-only variant, decode attention over quantized keys and values,
and the merge step of a search sharded across ranks.

The compute lives in libtq.so (include/tq.h); this package is its binding.
"""
from . import _binding as binding  # noqa: F401  (raises if libtq.so is missing)
from ._binding import (  # noqa: F401
    TQError, tq_attention_decode, tq_build_codebook, tq_build_codebook_mse,
    tq_build_codebook_split, tq_decode, tq_encode,
    tq_exact_topk, tq_logits_fp32, tq_score, tq_score_topk, tq_status_str, tq_topk, tq_topk_merge,
    tq_topk_noalloc, tq_workspace_bytes)
from .quantizer import Codes, TurboQuant, Workspace, exact_topk, logits_fp32  # noqa: F401
from . import sharded  # noqa: F401  (search over a database sharded across ranks)
