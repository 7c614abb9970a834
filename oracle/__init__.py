"""CPU oracle of the MoE expert layer -- test infrastructure, not product.

Importable only from tests/, __graft_entry__.smoke() and bench.py's CPU
baseline legs.  It shares no code with the CUDA path.
"""
from . import moe_ref, mxfp8_ref  # noqa: F401
