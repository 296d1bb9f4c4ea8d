"""CPU oracle for the NVFP4 W4A4 group-limited MoE layer.  TEST INFRASTRUCTURE ONLY.

This package is the slow, plain reference that the CUDA library is checked
against.  Only the tests, ``__graft_entry__.smoke()`` and the ``cpu_baseline``
leg of ``bench.py`` may import it; the library never does, and it imports
nothing from the library.  Everything is NumPy: FP64 for the layer math on
dequantised values, and one NumPy float32 operation per step where the
quantisation rule is stated in FP32.

Sources followed (page titles of the pages describing the method):

* "NVFP4 quantization" (Reflection developer docs), section "Quantization
  scheme": the format (E2M1 codes, an E4M3 scale for every 16-value block and
  an FP32 scale for the whole tensor) and which tensors carry it (the routed
  experts' gate, up and down projections and their input activations).
* "Reflection releases Beam, a 501B-parameter MoE model ..." (bpdata news),
  section "Mixture-of-Experts details": sigmoid scores over 256 experts,
  8 groups of 32, keep 4 groups by the sum of each group's top two scores,
  top 8 experts inside them, outputs combined with normalised router weights
  scaled by 2.5; section "Residual stream and numerical decisions": the router
  and the SwiGLU product are computed in FP32; the residual stream adds the sublayer
  output of step k with weight 1/sqrt(k) and keeps the stream with sqrt((k-1)/k), and
  norms are computed in FP32 (``residual.py``).
* "FP8 quantization", sections "Quantization scheme" and "Quantization method": the FP8 W8A8
  variant, per-output-channel weight scales and per-token activation scales (``fp8.py``).
* "NVFP4 quantization", section "Quantization method": the post-training block-scale search
  that minimises the Hessian-weighted error (``local_hessian.py``).
* "Beam-1.0 auf 4x NVIDIA RTX PRO 6000 ..." (eurokommerz), section "Drei
  Checkpoints und was sie speichern": experts in blocks of 16 values, an
  expert is about 22 MB = 39.3M parameters x 0.5625 bytes.

Readings where the pages leave a step open (the global/block scale rule,
rounding modes, the static intermediate scale, tie-breaks, output dtype) are
stated in the module that implements each step.

Parity pins (``tests/test_oracle_*.py``) tie every function here to something
other than itself: library routines (``torch.float8_e4m3fn`` casts,
``np.argsort``), brute force over tiny inputs, closed forms and invariants,
and the size figures printed on the pages.
"""
from .formats import (  # noqa: F401
    E2M1_VALUES, e4m3_table, e2m1_decode, e4m3_decode, e4m3_encode, e2m1_encode,
    global_scale, quantize, dequantize, swizzle_scales, unswizzle_scales,
    swizzled_scale_bytes, nvfp4_tensor_bytes,
)
from .router import route, RouteResult  # noqa: F401
from .moe import permutation, expert_mlp, moe_forward, QuantTensor, quantize_tensor  # noqa: F401
from .residual import rmsnorm, rmsnorm_scale, residual_weights, residual_add  # noqa: F401
from .local_hessian import quantize_local_hessian, hessian_blocks, candidate_offsets  # noqa: F401
from . import fp8  # noqa: F401
