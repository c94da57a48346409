"""CPU oracle for one EAGLE tree-verification step.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this package:
only the tests, the smoke check in ``__graft_entry__`` and the CPU-baseline leg
of ``bench.py`` call it.  It shares no code, header, table or helper with the
CUDA library and imports nothing from it.

Everything is plain numpy in fp64, written step by step from the pages:

* ``tree``      EAGLE-2 dynamic draft tree: confidence = softmax of the draft
                logits, global acceptance V = product of confidences along the
                root path, per-level top-k expansion, rerank to the best m
                ("s1mplewind eagle" notes, EAGLE-2: "Well-Calibrated Draft Model",
                "Expansion of tree", "Reranking Nodes").
* ``static_tree`` EAGLE-1's fixed tree: a template of parents and sibling
                ranks filled from each parent's top tokens ("EAGLE" notes,
                "1. EAGLE pipeline / Draft Model").
* ``mask``      tree attention mask: a node sees the shared prefix, its
                ancestors and itself ("Технический анализ EAGLE-4", section
                "Деревья проверки EAGLE-4 и утилита управления").
* ``attention`` tree-masked softmax attention with an explicit dense mask
                (same section; "Tree Attention" in the EAGLE notes, "3.Verify").
* ``accept``    greedy longest-accepted-path walk and stochastic acceptance
                with probability min(1, p_target/p_draft) plus residual
                resampling (EAGLE-2 "Well-Calibrated Draft Model" formula;
                aivaro.ru EAGLE-3 answer, section 4 steps 3-4; EAGLE-4
                write-up, same section as the mask).
* ``paged``     the prefix cache as pages of a shared pool named by a block
                table: gather, and compaction into pages.
* ``sizing``    cost-aware tree sizing: a measured latency table, each
                level's gain in cumulative probability over its marginal cost
                against a threshold (EAGLE-4 write-up, same section).
* ``kv``        after acceptance: the accepted path's keys and values are
                appended to the prefix cache, the rejected ones dropped (EAGLE-4
                write-up, same section).

Pins (tests/test_oracle_*.py) tie each function to something other than
itself: hand-worked fixtures, closed forms, library routines on special cases,
brute force on tiny inputs and a chi-square test of distribution preservation.
Attention values have no printed example on the pages; they are pinned only
through special cases that reduce to library attention (causal, decode, MHA).
"""
from .common import decode_logits, logsumexp, softmax, near_tie  # noqa: F401
from .tree import build_tree, build_trees  # noqa: F401
from .static_tree import build_static_tree, template_rows  # noqa: F401
from .mask import ancestor_mask, pack_mask, positions  # noqa: F401
from .attention import tree_attention, tree_attention_rows  # noqa: F401
from .accept import accept_greedy, accept_stochastic, inverse_cdf, inverse_cdf_band  # noqa: F401
from .kv import compact_kv  # noqa: F401
from .paged import compact_kv_paged, gather_pages  # noqa: F401
from .sizing import cost_at, keep_level, level_ratio, level_width, levels_kept  # noqa: F401
