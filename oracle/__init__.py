"""Plain CPU oracle for the CONF-KV decode step (test infrastructure only).

This package is the independent reference that the CUDA path is checked
against. It is slow and literal on purpose: fp64 two-pass softmax attention,
a full sort for eviction, a scalar round-half-even quantiser, and the cache
kept as a position-sorted list of tokens. It shares no code, header, table or
constant generator with the CUDA library, and the CUDA library never imports
it. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline /
reference legs of ``bench.py`` may import it.

Sources restated here (cited by page title and section):

* "CONF-KV: Confidence-Aware KV-Cache Eviction with Mixed-Precision Storage
  for Long-Horizon LLMs", chatpaper.ai summary, abstract ("CONF-KV abstract").
* "Conf-KV: confidence-aware KV-cache eviction with mixed ..." rcap.io post
  ("CONF-KV post"): the method paragraphs and the decode-loop pseudo-code.
* "KVpop: KV-cache compression with online predictive pruning", gist.science
  technical summary ("KVpop summary"), sections 2.1 and 2.4.

Parity status per function is listed in the header of each module.
"""
from .confidence import confidence, confidence_batch, choose_budget, layer_budgets
from .quant import quantize_row, dequantize_rows
from .attention import attend
from .policy import ema_update, recency, composite_score, select_victims
from .segment import Params, Segment, prefill_segment, OracleCache

__all__ = [
    "confidence", "confidence_batch", "choose_budget", "layer_budgets",
    "quantize_row", "dequantize_rows", "attend",
    "ema_update", "recency", "composite_score", "select_victims",
    "Params", "Segment", "prefill_segment", "OracleCache",
]
