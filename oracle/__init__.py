"""CPU oracle for paged MLA decode attention -- TEST INFRASTRUCTURE ONLY.

This package is the slow, obviously-correct reference that the CUDA path is
checked against.  It is not part of the product: only ``tests/``,
``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import
it.  It shares no code, constants or helpers with the CUDA path under
``mla_decode_attention_16_b200/`` and never imports it.

Contents
--------
mla_ref.mla_decode_ref
    fp64 gather of the paged latent cache through the block table followed by a
    naive two-pass softmax (max pass, then exp/sum pass) and the PV product.
mla_ref.mla_partial_ref / mla_ref.merge_partials_ref
    the split-KV rewrite: per-chunk (o, lse) pairs and their log-sum-exp merge.
sched_ref.tile_schedule_ref
    the tile scheduler (per-partition quota + greedy in-order walk), pure Python
    integers.
append_ref.append_kv_ref / append_ref.decode_with_append_ref
    the new tokens' rows written into their page slots (the step before a
    decode), and "append, then decode".
fp8_ref.mla_decode_fp8_ref / fp8_ref.append_kv_fp8_ref
    the FP8 (e5m2) cache variant: the query cast to e5m2, the cache's e5m2
    values as K and V, the plain decode on those values; the append that casts
    the new rows to e5m2 (``e5m2_quantize`` / ``e5m2_encode`` / ``e5m2_decode``:
    the format and its round-to-nearest-even cast).

Sources (pages, by title and section)
-------------------------------------
* "FlashMLA 在 Hopper GPU 上的 MHA 内核调度优化解析" (blog.hotdry.top), sections
  计算边界特性与优化方向抉择 (d_k = 576 / d_v = 512 shapes, cost model),
  跷跷板调度的数学重构 (online rescaling must equal the plain softmax exactly),
  辅助优化：可编程依赖启动与瓦片调度 (splitkv + combine kernels, tile scheduler).
* "FlashMLA: 高性能GPU注意力机制计算库" walk-through (hanhandi.cn doc-0479),
  sections 项目主要功能 (paged cache, block size 64, BF16/FP16),
  4. Softmax数值稳定性优化 (subtract the running max before exponentiating),
  6. SM资源调度优化 (quota = ceil(total_blocks / num_sm_parts) + fixed overhead).
* "DeepSeek开源FlashMLA全解析" (ruibaoantu.com), section 2.1 item 4
  结果融合 (merge the chunk outputs with dynamic weights).
* "FlashAttention终极指南" (cnnetsun.cn): ``cache_seqlens`` / ``causal`` /
  ``return_softmax_lse`` conventions of a KV-cache attention call.
* "云上AI推理新突破：FlashMLA赋能DeepSeek-V2-Lite提速16%", section 3. 动态精度缩放,
  and "DeepSeek开源FlashMLA全解析", section 1.2 计算模式创新: Q.K^T from float8_e5m2
  operands, softmax and P.V back at FP16 precision.

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
(``tests/append_pins.py`` for the append, ``tests/fp8_pins.py`` for the FP8 variant)
(closed forms, invariants, brute force, an independent library special case)
and ``tests/test_oracle_mutants.py`` (planted mistakes must fail a pin).
"""

from .mla_ref import (  # noqa: F401
    D_K,
    D_V,
    PAGE,
    mla_decode_ref,
    mla_partial_ref,
    merge_partials_ref,
    visible_key_count,
)
from .sched_ref import FIXED_OVERHEAD_BLOCKS, tile_schedule_ref  # noqa: F401
from .append_ref import append_kv_ref, decode_with_append_ref  # noqa: F401
from .fp8_ref import (  # noqa: F401
    append_kv_fp8_ref,
    e5m2_decode,
    e5m2_encode,
    e5m2_quantize,
    mla_decode_fp8_ref,
)
