"""fp64 CPU oracle (test infrastructure only; see gla_oracle.py)."""

from .gla_backward_oracle import (gla_backward, gla_backward_head, gla_backward_head_manual,
                                  gla_forward_torch_head)
from .gla_oracle import gla_bruteforce_head, gla_forward, gla_head, relu, sigmoid
from .gla_gdn_oracle import gla_gdn_forward, gla_gdn_head
from .gla_softmax_oracle import anchor_key_ranges, softmax_anchor_forward, softmax_anchor_head
from .gla_rope_oracle import (gla_rope_bruteforce_head, gla_rope_forward, gla_rope_head,
                              rope_pair_angles, rope_rotate)

__all__ = ["gla_bruteforce_head", "gla_forward", "gla_head", "relu", "sigmoid", "gla_backward",
           "gla_backward_head", "gla_backward_head_manual", "gla_forward_torch_head",
           "gla_rope_bruteforce_head", "gla_rope_forward", "gla_rope_head", "rope_pair_angles",
           "rope_rotate", "gla_gdn_forward", "gla_gdn_head", "anchor_key_ranges",
           "softmax_anchor_forward", "softmax_anchor_head"]
