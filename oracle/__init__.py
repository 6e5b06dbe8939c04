"""fp64 CPU oracle for the batched Muon update.

Test infrastructure only: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``.  The CUDA library never imports,
links or calls anything here, and nothing here imports the CUDA library.
"""
from .muon_oracle import (  # noqa: F401
    NORM_EPS,
    NS_A,
    NS_B,
    adamw_step,
    clip_coefficient,
    clip_grad_norm_buckets,
    frobenius_normalize,
    lr_scale_factor,
    momentum_update,
    muon_step,
    muon_weight_update,
    nesterov_input,
    newton_schulz,
    ns_flops,
    ns_iteration,
    rank_mean,
    orthogonality_error,
    relative_frobenius,
    round_to_bf16,
)
