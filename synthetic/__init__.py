"""Seeded synthetic inputs for the Sketch Attention (SA) compression step.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic.  Both the CPU oracle (``oracle/``) and the CUDA path's
tests and benchmark take their inputs from here, so that the two sides see
bit-identical data.

Shapes and value distributions follow the workloads that the SequenceO1 page
describes (user histories of 10K-100K behaviour embeddings, "SequenceO1:
End-to-End Ultra-Long (100K) Sequence Modeling in Recommendation with
Low-Rank Caching", sections 1 and 2.1; long-term interests that recur far
apart in time, section 3.3).  Douyin's production histories are not
available, so these seeded draws stand in for them.

Conventions (the notation of section 2.1 of that page):
  X        (N, d)   behaviour embeddings of all users, concatenated row-wise
  offsets  (B+1,)   int64, user b owns rows [offsets[b], offsets[b+1])
  P        (k, d)   shared prototypes P^(0)
  W_Q, W_K (d, d)   projections, used as  S = (P W_Q)(X W_K)^T * scale
  queries  (B, k, d) per-user query matrices of a refinement layer's SA step
                     (section 2.2), in place of P
"""

from .workloads import (  # noqa: F401
    WORKLOADS,
    Workload,
    action_params,
    action_types,
    bf16_bits,
    bf16_from_bits,
    generate,
    round_to_bf16,
    ragged_lengths,
    refine_params,
    upstream_gradients,
    user_queries,
    workload_lengths,
)
