"""`python -m block_scaled_precision_act_b200` builds libbsp.so in-tree."""
from .build import build

print(build())
