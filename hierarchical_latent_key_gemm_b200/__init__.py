"""B200-native Latent Sparse Attention (LSA) hot path.

liblsa.so (CUDA, sm_100a) holds every kernel; ``lsa`` is its Python binding
and ``workloads`` draws the seeded synthetic inputs.
"""
from . import lsa, workloads  # noqa: F401
from .lsa import (  # noqa: F401
    Index, LsaError, lsa_append, lsa_build_index, lsa_build_index_from_tree, lsa_check,
    lsa_fullscan_select, lsa_kmeans, lsa_project_pool, lsa_query_latent, lsa_select,
    lsa_sparse_attn, make_build_params, make_select_params,
)
