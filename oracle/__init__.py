"""CPU oracle for the RTPurbo sparse decode step -- test infrastructure only.

Imported by tests/, __graft_entry__.smoke() and bench.py's CPU-baseline and
reference legs; never by the product path (dynamic_top_sparse_b200).
"""
from .rtpurbo import *  # noqa: F401,F403
from .rtpurbo import (HEAD_LOCAL, HEAD_RETRIEVAL, Selection, StepResult,  # noqa: F401
                      append_index_keys, attend, decode_step, default_scale,
                      dense_decode, descending_order, prefill_attention, index_logits, local_rows,
                      project_index_key, query_index, round_to, round_to_bf16,
                      round_to_f32, softmax_mass, topk_select, topp_select)
