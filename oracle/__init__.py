"""CPU fp64 oracle of the WUSH-KV runtime hot path.

TEST INFRASTRUCTURE: imported only by the tests, the graft smoke check and the
benchmark's CPU-baseline / reference legs; never by the product path.
"""
from .wushkv_oracle import *  # noqa: F401,F403
