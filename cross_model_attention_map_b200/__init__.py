"""Cross-model attention-map reuse on NVIDIA B200 (sm_100a).

The compute lives in ``libiamap.so`` (hand-written CUDA behind a C ABI, ``include/iamap.h``);
``iamap`` is its ctypes binding. Import ``cross_model_attention_map_b200.iamap`` to use it (the
import fails loudly when the library has not been built).
"""

__all__ = ["iamap", "build"]
