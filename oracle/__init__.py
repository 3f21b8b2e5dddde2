"""CPU oracle for ring attention with emulated context-parallel ranks.

TEST INFRASTRUCTURE ONLY. Nothing in the product path imports, links or runs
anything in this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.

Everything here is plain numpy in float64, written from the definitions on the
source pages, with no blocking, fusion or reordering beyond what a definition
states (query rows are evaluated in independent row blocks only to bound
memory; every row's result is computed from its own full key range).
It shares no code, constants or helpers with the CUDA library.

Sources (cited by page title and section):
  * Ultralytics glossary, "Context Parallelism" -- section "How context
    parallelism works" (ring attention: partial attention per arriving KV
    block, pass the block on, repeat; result equals full-sequence attention).
  * Blog "Context Parallelism v.s. Sequence Parallelism (Megatron-LM)" --
    section "Symmetric chunk assignment" (2*cp chunks, rank r holds chunks r
    and 2*cp-1-r, global position ids carried, pad to a multiple of 2*cp).
  * aiunderstanding.org, "Sequence parallelism and ring attention" --
    sections "Deep dive" and "Technical insight" (online softmax: running max
    and running normaliser, earlier partial sums rescaled; exact result).
  * RoPE at carried global positions (``rotary.py``): the same Megatron blog
    section says rotary embeddings must use the global positions of the
    chunks a rank holds; the rotation is the published RoFormer definition.

Parity status: every function here is pinned by ``tests/test_oracle_*.py``
(brute force, closed forms, library special cases, invariants, the page's
rank/chunk table). No function is "parity unpinned".
"""
from .layout import (CONTIGUOUS, HEAD_TAIL, STRIPED, padded_len, perm_index, permute, unpermute, rank_chunks,
                     varlen_index, varlen_permute, varlen_unpermute)
from .attn import (attention, merge, ring_emulate, blockwise_attention,
                        attention_bwd, attention_bwd_block, visible_mask, causal_pairs_per_rank, gqa_expand,
                   gqa_reduce)
from .rotary import HALF as ROPE_HALF, INTERLEAVED as ROPE_INTERLEAVED, rope, rope_grad

__all__ = [
    "CONTIGUOUS", "HEAD_TAIL", "STRIPED", "padded_len", "perm_index", "permute", "unpermute", "rank_chunks",
    "varlen_index", "varlen_permute", "varlen_unpermute",
    "attention", "merge", "ring_emulate", "blockwise_attention", "attention_bwd", "attention_bwd_block", "visible_mask",
    "causal_pairs_per_rank", "gqa_expand", "gqa_reduce", "ROPE_HALF", "ROPE_INTERLEAVED", "rope", "rope_grad",
]
