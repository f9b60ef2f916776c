"""CPU reference (the oracle) for paged attention over a block-table KV cache.

TEST INFRASTRUCTURE ONLY.  Nothing in the product package imports, calls or
links anything here; only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may use it.

It is the plain definition, written for a reader to check by eye against the
source pages, in float64 with numpy:

* ``block_pool``  - the Block / BlockTable bookkeeping of the page
  "Nano-vLLM-Ascend: lightweight LLM inference framework for Ascend NPU",
  section 2.1 (PageAttention memory management): fixed 16-token blocks, a
  logical-to-physical block map per sequence, a reference count per block;
  and the free-list allocator role of BlockAllocator from the page "Ascend NPU
  LLM inference optimisation: the vLLM-Ascend approach", section 2.1.
* ``kv_write``    - writing new tokens' K/V into their slots, as bytes.
* ``attention``   - gather through the block table, then softmax(q K^T * scale) V
  per query head (Nano-vLLM-Ascend page, section 2.2.1, the unfused attention;
  section 4.2 names the 1/sqrt(d) scale), with the softmax done in fp64 (the
  vLLM-Ascend page, section 3.1, moves softmax out of fp16 for accuracy); causal
  chunked prefill over the paged context (vllm-ascend page, section 1.1, PCP).
* ``brute``       - a scalar pure-Python twin of ``attention`` for tiny cases.
* ``kv_quant``    - INT8 KV cache (Nano-vLLM-Ascend page, section 4.3; vLLM-Ascend
  page, section 5): per-(token, KV head) symmetric absmax codes with an fp32
  scale, written on append and dequantised for attention.
* ``context_split`` - decode with each sequence's context split across devices
  (vllm-ascend page, sections 1.1 and 3.1, DCP: every device attends over the
  part of the KV cache it holds, the intermediate results are gathered and
  combined): the block-interleaved split, each part's output and log-sum-exp,
  and the log-sum-exp merge.
* ``rope``        - rotary position embedding of new tokens' queries and keys
  fused with the KV write (Nano-vLLM-Ascend page, sections 3.1 and 5.1: the
  rotary multiply by per-position cos/sin tables, inverted by negating sin).

Parity pins (tests/test_oracle_pins.py, tests/test_oracle_rope.py,
tests/test_oracle_kv_quant.py): the pages' worked block arithmetic
(tests/golden/), closed forms, torch's float64 scaled_dot_product_attention on
dense inputs, the scalar twin, and invariants (block permutation, prefix
sharing, prefill row i == decode of the first prefix+i+1 tokens); for the
rotary step, rotation closed forms, the page's inverse rule, angle addition,
the relative-position property and torch complex multiplication; for the
INT8 cache, the absmax code, the half-step error bound, exact grid rows and
torch's int8 quantiser; for the context split, the shards partition every
sequence (the page's 1000-token example over three ranks), torch's logsumexp
and SDPA, and the merge against full attention (tests/test_oracle_context_split.py).
No function
here is "parity unpinned".
"""

from . import attention, block_pool, brute, context_split, kv_quant, kv_write, rope  # noqa: F401
from .attention import decode_attention, gather_kv, prefill_attention, split_partials  # noqa: F401
from .block_pool import OraclePool, replay  # noqa: F401
from .kv_write import write_kv  # noqa: F401
from .rope import rope_tokens, rope_write_kv, rotary  # noqa: F401
