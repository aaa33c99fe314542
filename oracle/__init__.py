"""fp64 CPU oracle for exact attention (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package; the CUDA path never does.
"""

from .attention import (attention_backward, attention_backward_dropout, attention_backward_varlen,
                        attention_forward, attention_forward_dropout, attention_forward_kvcache,
                        attention_forward_varlen, default_scale, dropout_keep, dropout_threshold,
                        online_softmax_forward)
from .philox import philox4x32_10

__all__ = ["attention_forward", "attention_backward", "online_softmax_forward", "default_scale",
           "attention_forward_varlen", "attention_backward_varlen", "attention_forward_kvcache",
           "attention_forward_dropout", "attention_backward_dropout", "dropout_keep", "dropout_threshold",
           "philox4x32_10"]
