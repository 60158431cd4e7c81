"""Independent fp64 CPU oracle for the token-choice Mixture-of-Experts layer.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may
import or run anything in this package.  The CUDA library never calls it and
shares no code, constant or helper with it.

The oracle follows the definitions on the pages:

* "How do Mixture of Expert Models Work?", section "The Math Behind MoEs":
  y = sum_i G(x)_i E_i(x), G(x) = Softmax(TopK(x . W_g)), Mixtral's
  Softmax(Top2(x . W_g)) . SwiGLU_i(x).
* "[Paper Club] Upcycling Large Language Models into Mixture of Experts",
  the walk-through of the MoE layer (route -> permute with capacity ->
  expert FFN -> un-permute scaled by the router probability).
* Same page, "Expert Capacity" tactic: at most C tokens per expert,
  overflow dropped.
* "Take a Closer Look at the MoE LLM Routing", "Drop-towards-the-End":
  when capacity is set, tokens later in the sequence are dropped first.
"""

from .moe_oracle import (  # noqa: F401
    router_logits,
    top_k,
    gating_softmax,
    gating_softmax_all,
    capacity,
    assign_capacity,
    assign_capacity_shard,
    priority_order,
    silu,
    gelu,
    expert_ffn,
    moe_forward,
    moe_forward_tokens,
    expert_choice_scores,
    expert_choice_select,
    moe_forward_expert_choice,
)
