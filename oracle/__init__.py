"""CPU oracle of the HiFA4-style 4-bit attention forward -- TEST INFRASTRUCTURE ONLY.

Only tests/, __graft_entry__.smoke() and bench.py's CPU baseline / reference leg may
import this package.  The product path (bit_flashattention_b200) never does, and this
package never imports the product.  See hifa4_oracle.c for the arithmetic and its
citations; this module only marshals numpy arrays through ctypes.
"""
from .oracle import *  # noqa: F401,F403
