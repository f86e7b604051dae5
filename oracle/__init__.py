"""Oracle package -- test infrastructure only (tests, smoke check, bench CPU arm).

The library under ``mot_flow_matching_b200`` never imports this package.
"""
from .mot_attn_oracle import *  # noqa: F401,F403
