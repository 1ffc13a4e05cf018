"""CPU oracle for the HGA hot path (test infrastructure only; see hga_oracle)."""
from .hga_oracle import (BLOCK, GROUP, QBLOCK, TIE_REL, attn_bwd, attn_fwd,  # noqa: F401
                         build_summaries, decode_attn, decode_route, keyset,
                         prepare_segment, query_summaries, rope, round_bf16, route,
                         route_causal, routed_keys,
                         segment_step, tier_stage)
