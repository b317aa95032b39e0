"""CPU fp64 oracle for the column->row tensor-parallel transformer block.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import or call anything in this package.
The library's product path never does: it runs on the CUDA kernels alone and
fails loudly when they are missing.  The oracle shares no code with the CUDA
path (no kernels, headers, helpers or constants); only the seeded input
generator module feeds both.

Everything here is plain numpy in float64 on inputs converted exactly from
their bf16 (or fp32) bits, with no intermediate rounding.  Matrix products use
numpy's matmul and erf comes from ``scipy.special``; no blocking, fusion or
reordering is added beyond what the definitions state.

The backward pass of the FFN block (gradients of the forward block by the
chain rule, with the sum over shards of the column layer's input gradient as
its one reduction) is pinned the same way: a normal-table check of GeLU',
central finite differences, float64 autograd and sharding invariance; so is
the attention sub-layer's backward pass (finite differences of the forward
oracle, float64 autograd of torch's attention, head-group sharding and
permutation, closed forms for one-token sequences and a constant V).

Source of the method: the page "Tensor Parallelism > Combining Column and Row
Parallelism" (mbrenndoerfer.com), cited below as [TP-CR] with its numbered
steps (1 column-parallel W1, 2 row-parallel W2, 3 all-reduce) and its
paragraphs (on the nonlinearity, on feature reductions, on multi-head
attention, on head independence, on the QKV split, and on the two reductions
per layer with residual adds between the sub-layers).

Parity pins: every function here is pinned by the ``-m "not gpu"`` tests
(closed forms, library special cases, brute force on tiny inputs and the
invariants the page fixes); none is "parity unpinned".
"""
from .tp_block import (  # noqa: F401
    gelu,
    relu,
    ffn_forward,
    ffn_forward_sharded,
    layernorm,
    attention_heads,
    attn_forward,
    attn_forward_sharded,
    layer_forward,
    reduce_partials,
    gelu_grad,
    relu_grad,
    ffn_backward,
    ffn_backward_sharded,
    attention_heads_backward,
    attn_backward,
    attn_backward_sharded,
)
