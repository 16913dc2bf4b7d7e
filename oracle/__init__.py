"""fp64 CPU oracle for the DyRA approximated linear layer.

TEST INFRASTRUCTURE ONLY. Nothing in the product (the CUDA library and its
Python binding) imports, calls or links anything here. Only tests/, the
smoke check in __graft_entry__.py and the CPU-baseline leg of bench.py use it.

oracle.monarch holds the Monarch static part (DyRA App. B) and DyRA on top of it.
"""

from .dyra_oracle import (  # noqa: F401
    Factors,
    als_half_steps,
    als_updates,
    als_inference,
    dense,
    error_report,
    inference,
    inference_rows,
    offline_prepare,
    offline_prepare_from_svd,
    rel_fro,
    round_to,
    weight_only,
)
