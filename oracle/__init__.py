"""CPU oracle for predicted-query token-level sparse decoding (test infrastructure).

This package is the slow, plain float64 statement of what the CUDA path
computes.  It exists to check that path and to time a CPU baseline: only
``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its CPU-baseline and
reference arms) may import it.  It shares no code with the CUDA library and
imports nothing from it.

Sources (the method's pages print no equation, so each step is a reading of
their prose; every reading is named where it is made):

* "Reproduction: AsyncSpade -- Efficient Test-Time Scaling with Asynchronous
  Sparse Decoding" (Hugging Face dataset card
  debajyotidasgupta/asyncspade-repro-artifacts), cited as *repro card* with
  its section: the claims table "What reproduces (and what does not)" (C1-C5),
  "Layout", "Key finding worth flagging for the next agent".
* "AsyncSpade: Efficient Test-Time Scaling with Asynchronous Sparse Decoding"
  research-map summary (atlas.scime.ai), cited as *summary* with its section
  ("Problem", "Approach", "Key results").
* The paper's abstract (arXiv 2510.07486), cited as *abstract*.

Parity status per function is listed in each module's header.
"""
from .predict import ridge_coefficients, normalise_coefficients, window_prediction, predict_query  # noqa: F401
from .scan import gather_sequence, score_row, score_keys, select_row, select_topk  # noqa: F401
from .attend import attend_set, sparse_attend  # noqa: F401
from .quest import quest_meta, quest_page_scores, quest_select_row, quest_select  # noqa: F401
from .flops import decode_flops, QWEN3_8B, QWEN3_32B  # noqa: F401
from .pipeline import decode_step  # noqa: F401
from .readings import (score_row_mean, score_row_mass, select_per_head, pooled_features,  # noqa: F401
                       pooled_prediction, predict_query_pooled, set_overlap, recent_window_overlap)
