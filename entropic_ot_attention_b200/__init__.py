"""B200-native blockwise band Sinkhorn attention (C-ABI library libeot + thin binding).

Method: "Blockwise Differentiable Sinkhorn Attention", technical summary (gist.science
2605.08123).  See include/eot.h for the C ABI.  Importing this package requires the built
library (``python -m entropic_ot_attention_b200.build``); there is no fallback path.
"""
from . import _abi
from .api import (SinkhornAttentionFn, band_half_step, band_output, make_problem, resolved_impl, sinkhorn_attention,
                  sinkhorn_bwd, sinkhorn_fwd, workspace)
from .certificate import bias_certificate, choose_tail_depth, contraction_certificate
from .host_pipeline import HostStep

__all__ = ["sinkhorn_attention", "sinkhorn_fwd", "sinkhorn_bwd", "band_half_step", "band_output", "SinkhornAttentionFn", "make_problem",
           "workspace", "resolved_impl", "HostStep", "bias_certificate", "choose_tail_depth", "contraction_certificate", "_abi"]
