"""Plain, slow, fp64 CPU oracle for block-sparse INT8 video attention.

TEST INFRASTRUCTURE ONLY. Nothing on the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may call it. It shares no code with
the CUDA library; the only module both sides use is ``workloads`` (seeded
inputs, no method arithmetic).

What it computes, step by step, and where the source pages describe it:

* ``quant``     per-block symmetric INT8 of Q (128-row blocks) and K (64-row
                blocks), scale = amax/127, round half to even; int32 sum-pools.
                "Configure Sol Sparse Attention", *How it works* (proxy scores
                run on the same prequantized INT8 Q/K as the exact path).
* ``route``     proxy score per (128-query block, 64-key block) pair from the
                pooled INT8 sums; Sol rule keep-iff score >= mean + tau*std over
                the query block's row; dense prefix protection.
                "Configure Sol Sparse Attention", *How it works* and *The inputs
                that matter* (routing_threshold, prefix_policy manual).
                Fixed-sparsity top-k selection over the same scores, prefix
                dense ("Ref2VA VSA", *2-stage attention patch*).
* ``attention`` softmax attention over the kept blocks exactly plus one
                centroid term per skipped 64-token block (1x64) or two 32-token
                centroids (2x32); and the explicit logical-block-mask entry
                (LCSA, "FlashVSR Sparge Attention", intro and *How it works*);
                the residual virtual K/V mode, physical keys exact and each
                added virtual slice as centroid terms ("Configure H3 Static
                Virtual KV").

Every function is pinned by ``tests/test_oracle_*.py`` against something
other than itself (brute force, closed forms, dense softmax attention through
torch, exact-arithmetic statistics). The one quantity left unpinned is the
approximation quality of the centroid terms against dense attention
("parity unpinned" for that comparison only: the pages give no error figure).
"""
from .quant import quantize_blocks, dequantize_blocks, q_pools, k_half_pools, block_rows
from .route import proxy_scores, sol_route, route_head, topk_keep_count, topk_route
from .attention import (centroid_groups, centroid_table, sol_attention_head,
                        masked_attention_head, physical_allowed, lcsa_mask,
                        resolve_scale, virtual_kv_residual_head)

__all__ = [
    "quantize_blocks", "dequantize_blocks", "q_pools", "k_half_pools", "block_rows",
    "proxy_scores", "sol_route", "route_head", "topk_keep_count", "topk_route",
    "centroid_groups", "centroid_table", "sol_attention_head", "lcsa_mask",
    "masked_attention_head", "physical_allowed", "resolve_scale", "virtual_kv_residual_head",
]
