"""CPU oracle for the GQE attention forward pass (test infrastructure only).

Imported only by the tests, the smoke check and bench.py's CPU-baseline legs. It shares
no code with the CUDA path and imports nothing from it.
"""
from .gqe_oracle import (  # noqa: F401
    VARIANTS, Layer, Routing, Result, default_head_dim, router_logits, group_softmax,
    top_k_per_group, route, kv_projection, routed_queries, shared_query, stream_kv_head,
    attention_rows, attention, combine, output_projection, aux_loss, forward, forward_rows,
    DecodeResult, decode, Grads, attention_rows_backward, slot_weights_backward,
    aux_loss_grad_p, group_softmax_backward, backward, backward_x_rows,
)
