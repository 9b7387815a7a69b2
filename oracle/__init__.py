"""Oracle for the context-parallel attention hot path -- TEST INFRASTRUCTURE ONLY.

A plain, slow, obviously-correct CPU restatement (NumPy fp64 and pure-Python loops)
of what the per-rank context-parallel attention path computes:

* non-causal scaled dot-product attention with its log-sum-exp (``ref.attention``),
* the exact merge of two partial (O, LSE) results over disjoint key sets, which is
  the Ring Attention step (``ref.merge``),
* the DeepSpeed-Ulysses sequence<->head re-partition run over P virtual ranks
  (``ref.seq2head`` / ``ref.head2seq``),
* the attention_mdtrt sample's RMSNorm of the Q and K head rows, in the float32 the
  page fixes (``ref.rmsnorm_heads``).

Sources (the pages print prose and figures only, no formula; each function states
the reading it takes):

* "Scaling AI Inference Across Multiple GPUs Using NVIDIA TensorRT with Multi-Device
  Inference Support" (NVIDIA developer blog), sections 上下文并行 / Context
  parallelism, AllGather KV (Fig. 2), 环形注意力 / Ring Attention (Fig. 3) and
  DeepSpeed Ulysses (Fig. 4).
* "Simplifying Model Serving Across Multiple GPUs with NVIDIA TensorRT Multi-Device
  Integration in NVIDIA Dynamo-Triton", section 使用 Ulysses 上下文并行性分发 Cosmos 3
  (44160 video tokens, 5520 per rank at CP8, text path replicated).
* "TensorRT 多设备注意力推理实战" (guide to the attention_mdtrt sample), section
  模型的核心结构 (QK^T -> Softmax -> Attn*V per head).

Who may use it: only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU
baseline / reference arm.  The product package ``context_long_sequence_non_b200``
never imports this package and this package never imports the product; the two
share no code.  Only the seeded input generators (a separate module holding none of
the method's arithmetic) feed both.

Pins: every function here is pinned in ``tests/test_oracle.py`` against closed forms,
hand-derived worked examples (``tests/golden/``), invariants, library routines
(``scipy.special.softmax`` / ``logsumexp``) and a loop-only brute force; planted
mistakes in the oracle are shown to fail those pins.
"""

from .ref import (  # noqa: F401
    attention,
    attention_rows,
    merge,
    merge_chunks,
    seq2head,
    head2seq,
    ring_attention,
    ulysses_attention,
    set_threads,
    threads,
)
