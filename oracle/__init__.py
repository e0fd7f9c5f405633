"""CPU oracle (test infrastructure only): see ``oracle.moe_oracle``."""
from .moe_oracle import *  # noqa: F401,F403
from .moe_oracle import (PER_PICK, DEDUP, TWO_HOP, round_to, ulp, softmax, route_topk,  # noqa: F401
                         demand_hist, replica_assign, optimal_max_active, token_balanced_active,
                         build_layout, own_rank_share, pack, combine, combine_two_hop)
