"""Plain, slow, CPU fp64 oracle for the paged decode-attention path.

TEST INFRASTRUCTURE ONLY.  This package is the independent definition the
CUDA path is checked against.  Only ``tests/``, ``__graft_entry__.smoke()``
and ``bench.py``'s ``cpu_baseline`` / ``--impl reference`` legs may import it;
the product package (``paged_kv_cache_378_b200``) never imports, links or
calls anything here, and this package never imports the product.

Sources (cited by page title and section throughout):

* [ITHOME]  ithelp.ithome.com.tw article 10405755 on PagedAttention
  (sections "PagedAttention 的核心想法", "手動畫一次 block table",
  "不是完全沒有代價").
* [PU]      "Infra: PagedAttention" by Fanyi Pu (sections
  "KV Cache 为什么会浪费显存", "按 Block 分配",
  "共享前缀，分叉时 Copy-on-write", "Continuous Batching").
* [AKIRA]   "只用了 8 格，為什麼占了 12 格？" (akira.ipas-ai.com
  paged-attention-story; section "阿頁的辦法：不必連號，我有一張對照表").

Modules:

* ``bf16``      exact widening of bf16 bit patterns to float64.
* ``paging``    block arithmetic and the host block manager (allocation on
                demand, fork with reference counts, copy-on-write, release).
* ``attention`` kv_append, block_copy, per-partition partials, the
                max-rescaled merge, and dense paged decode attention.

Every function here is pinned by ``tests/test_oracle_pins.py`` against values
the pages print, closed forms, library routines or brute force; none is
marked "parity unpinned".
"""

from . import bf16, paging, attention  # noqa: F401

__all__ = ["bf16", "paging", "attention"]
