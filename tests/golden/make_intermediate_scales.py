"""Write the static per-expert global scales g_h of the SwiGLU intermediate.

The down projection's input h = silu(gate) * up is NVFP4 like every expert input
("NVFP4 quantization", section "Quantization scheme"), and post-training
quantisation ("Quantization method") fixes its scale offline.  Reading used for
the synthetic layers: run the oracle on a calibration batch of 256 tokens
(activations seed 1, same distribution as the layer input), take each expert's
FP64 amax A_e of h over the tokens routed to it, and set g_h[e] = fp32(A_e / 2688)
(the global-scale rule of the quantiser).  An expert that receives no
calibration token takes the largest A_e of the other experts.

Only the oracle and the seeded input generators are used.  Run from the repo
root:  python tests/golden/make_intermediate_scales.py [tiny|beam]
"""
import os
import sys
import types

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from workloads import TINY, BEAM, activations, router_weight, expert_weight  # noqa: E402

CALIB_TOKENS = 256
CALIB_SEED = 1


def calibrate(shape):
    cfg = types.SimpleNamespace(E=shape.E, n_groups=shape.n_groups, topk_groups=shape.topk_groups,
                                topk=shape.topk, routed_scale=shape.routed_scale)
    x = activations(CALIB_TOKENS, shape, seed=CALIB_SEED).float().numpy()
    r = oracle.route(x, router_weight(shape).numpy(), cfg)
    xc, xs, gx = oracle.quantize(x)
    amax = np.zeros(shape.E)
    for e in range(shape.E):
        toks = np.flatnonzero((r.idx == e).any(axis=1))
        if len(toks) == 0:
            continue
        xhat = oracle.dequantize(xc[toks], xs[toks], gx)
        gq = oracle.quantize_tensor(expert_weight(shape, e, "gate").float().numpy())
        uq = oracle.quantize_tensor(expert_weight(shape, e, "up").float().numpy())
        gv = xhat @ gq.dequant().T
        uv = xhat @ uq.dequant().T
        h = gv / (1.0 + np.exp(-gv)) * uv
        amax[e] = np.abs(h).max()
        print(f"expert {e}: {len(toks)} tokens, amax {amax[e]:.6g}", flush=True)
    amax[amax == 0] = amax.max()
    return np.array([oracle.global_scale(a) for a in amax], dtype=np.float32)


def main():
    which = sys.argv[1:] or ["tiny", "beam"]
    for name in which:
        shape = {"tiny": TINY, "beam": BEAM}[name]
        g_h = calibrate(shape)
        path = os.path.join(ROOT, "tests", "golden", f"intermediate_scales_{name}.txt")
        with open(path, "w") as f:
            f.write(f"# Static global scale g_h[e] of the SwiGLU intermediate, {name} layer "
                    f"(H={shape.H}, I={shape.I}, E={shape.E}).\n")
            f.write("# Written by tests/golden/make_intermediate_scales.py from the oracle on a "
                    f"{CALIB_TOKENS}-token calibration batch (seed {CALIB_SEED}); "
                    "g_h = fp32(amax_e(h) / 2688).\n")
            f.write("# expert g_h(float32 hex) g_h(decimal)\n")
            for e, g in enumerate(g_h):
                f.write(f"{e} {np.float32(g).view(np.uint32):08x} {float(g):.9g}\n")
        print("wrote", path)


if __name__ == "__main__":
    main()
