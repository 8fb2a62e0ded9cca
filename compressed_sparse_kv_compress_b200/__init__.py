"""cskv: the DeepSeek V4 hybrid CSA/HCA decode attention path on B200 (sm_100a).

The computation lives in ``libcskv.so`` (hand-written CUDA, C ABI in
``include/cskv.h``); this package only marshals torch tensors into it.
"""

from . import api  # noqa: F401
from ._lib import LIB_PATH, CskvError, load  # noqa: F401
from .api import (  # noqa: F401
    csa_compress,
    hca_compress,
    hybrid_decode_attn,
    lindex_score_topk,
    lindex_topk_from_scores,
)
from .step import DecodeStep  # noqa: F401
