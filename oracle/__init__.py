"""CPU oracle for Top-p block routing and block-sparse attention (fp64, NumPy).

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or link this
package: only the test suite, the smoke check and the benchmark's CPU-baseline leg use it.
It shares no code, constants or helpers with the CUDA library; the two meet only through
the seeded inputs of the `workloads` module.

Everything is plain and slow on purpose: each function follows one passage of the pages
and computes in float64 on the exact input values (bf16/fp32 upcast), with library
primitives (sort, cumsum, matmul, exp) as the only building blocks.

Sources (page title, section):
  * FVAttn blog summary "腾讯+中山大学新作：视频生成提速2.11×，靠的是RLB和SASA",
    section "AI视频生成的阿喀琉斯之踵…": Top-p routing keeps, per query, the smallest
    descending-importance set of key blocks whose cumulative importance reaches p;
    section "RLB…": per-head load = number of blocks each head must compute, heaviest first;
    section "SASA…": fill a unit's slack with the best blocks routing left out, within a budget.
  * Video-generation acceleration notes (wzjinhao.cn) §5.2 "块稀疏注意力的教学实现":
    block representatives are token means, block score = mean(Q_blk)·mean(K_blk)/sqrt(d),
    a forced local band, then masked softmax attention; §5.3: full coverage equals dense.
  * vLLM-Omni Sol-Attn article §2.1/§2.2 and §5.2: frame-level top-k on mean-pooled
    frames, unioned with neighbouring frames and the first frame.

Parity pins: every function here is checked by tests/test_oracle_pins.py against closed
forms, brute force on tiny inputs, hand-computed golden cases (tests/golden/) and library
routines (torch scaled_dot_product_attention). No function is unpinned.
"""
from .route import (RouteCfg, pool_blocks, pool_frames, block_scores, row_softmax,
                    topp_row, topk_row, forced_blocks, frame_topk_select, route, near_tie_rows,
                    valid_near_tie_set, sasa_tile_augment, sasa_near_tie_rows, valid_sasa_row, frame_sets,
                    block_forced, frame_token_mask, frame_entry_code)
from .attention import attention_sets, attention_token_mask, attention_rows, selected_flops, attention_dense_mask
from .schedule import csr_from_mask, head_loads, tile_costs, lpt_order
from .rlb import imbalance, rlb_plan

__all__ = [
    "RouteCfg", "pool_blocks", "pool_frames", "block_scores", "row_softmax", "topp_row", "topk_row",
    "forced_blocks", "frame_topk_select", "route", "near_tie_rows", "valid_near_tie_set",
    "sasa_tile_augment", "sasa_near_tie_rows", "valid_sasa_row", "frame_sets", "block_forced",
    "frame_token_mask", "frame_entry_code", "attention_dense_mask",
    "attention_sets", "attention_token_mask", "attention_rows", "selected_flops",
    "csr_from_mask", "head_loads", "tile_costs", "lpt_order", "imbalance", "rlb_plan",
]
