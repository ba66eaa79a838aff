"""fp64 CPU oracle for the LoRA adapter branch (test infrastructure only).

Only tests, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline and
reference legs may use this package.  The product library never imports it.
"""
from . import lora_oracle  # noqa: F401
