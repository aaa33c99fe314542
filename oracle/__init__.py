"""fp64 CPU oracle for exact attention (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package; the CUDA path never does.
"""

from .attention import (attention_backward, attention_forward, default_scale,
                        online_softmax_forward)

__all__ = ["attention_forward", "attention_backward", "online_softmax_forward", "default_scale"]
