"""StateKV per-frame streaming prefill on B200 (sm_100a).

The compute path is the C-ABI library ``libstatekv.so`` (kernels in ``csrc/``);
``kv_cache_selection_b200.statekv`` is its thin Python binding and
``kv_cache_selection_b200.synthetic`` draws seeded inputs.
"""

__version__ = "0.1.0"
