"""CPU oracle for the LSA hot path (test infrastructure; see lsa_oracle.py)."""
from .lsa_oracle import *  # noqa: F401,F403
from .lsa_oracle import Tree, KMeansResult  # noqa: F401
