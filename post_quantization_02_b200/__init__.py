"""KronQ per-layer quantization path on B200 (sm_100a).

The compute lives in libkronq.so (C ABI: include/kronq.h), built in-tree by
``post_quantization_02_b200.build``.  ``abi`` binds each entry point under its
C name; ``pipeline`` chains them for one sublayer; ``alloc`` is the host-side
mixed-precision bit allocation.
"""

from . import abi  # noqa: F401
from .abi import (  # noqa: F401
    KronqError,
    kronq_abi_version,
    kronq_biip_rotate,
    kronq_cholesky_inv,
    kronq_covariance,
    kronq_layer_loss,
    kronq_pack,
    kronq_quantize_layer,
    kronq_sensitivity,
    kronq_status_string,
    kronq_unpack,
    kronq_workspace_size,
)
