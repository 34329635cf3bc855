"""Gist Sparse Attention (GSA) hot path for NVIDIA B200 (sm_100a).

The computation lives in libgsa.so (CUDA kernels behind the C ABI declared
in include/gsa.h).  This package holds the thin ctypes binding (``_abi``,
re-exported here under the C names), the in-tree build (``build``) and the
seeded synthetic workloads (``workloads``).
"""
from ._abi import (  # noqa: F401
    EXPORTS, GSA_BF16, GSA_DEVERR_BAD_INDEX, GSA_DEVERR_CAPACITY, GSA_DEVERR_TIMEOUT, GSA_ERR_CUDA,
    GSA_ERR_INVALID_ARG, GSA_ERR_TIMEOUT, GSA_ERR_UNSUPPORTED, GSA_ERR_WORKSPACE, GSA_F32, GSA_OK, GSA_OP_DECODE,
    GSA_OP_GIST_STEP, GSA_OP_HGSA, GSA_OP_HGSA2, GSA_OP_MULTIQUERY, GSA_OP_PREFILL, GSA_PRIOR_GISTS, GSA_PRIOR_HGSA, GSA_PRIOR_HGSA2,
    GSA_PRIOR_NONE, GsaError, gsa_decode, gsa_decode_backward, gsa_decode_noalloc, gsa_desc, gsa_gist_step,
    gsa_noalloc_status, gsa_score_select,
    gsa_h2desc, gsa_hdesc, gsa_multiquery_select, gsa_prefill, gsa_prefill_attend, gsa_prefill_score, gsa_score_gists, gsa_status_string,
    gsa_topk_select, gsa_topp_select, gsa_unfold_attend, gsa_version, gsa_workspace_bytes, gsa_workspace_init,
    gsa_workspace_status,
    hgsa2_decode, hgsa2_select, hgsa_decode, hgsa_select, load, make_desc, make_h2desc, make_hdesc,
)
