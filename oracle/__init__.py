"""CPU oracle for the MSA hot path: test infrastructure only (see msa_oracle)."""
from .msa_oracle import *  # noqa: F401,F403
from .msa_oracle import EPS, bf16_to_f64, chunk_layout, rope, rope_theta, encode_memory  # noqa: F401
from .msa_oracle import router_query, cosine, chunk_scores, doc_scores, topk, route_topk  # noqa: F401
from .msa_oracle import sparse_context, attention, sparse_attend, sparse_attend_tokens  # noqa: F401
from .msa_oracle import aux_loss  # noqa: F401
