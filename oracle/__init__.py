"""fp64 CPU oracle of the SparseLoRA hot path. Test infrastructure only: the product
path never imports it."""
from .sparselora_oracle import *  # noqa: F401,F403
