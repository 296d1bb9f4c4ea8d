"""Counter-based synthetic inputs that come out bit-identical on the CPU and on a GPU.

Every random number is a pure function of (seed, stream, element index): a
32-bit counter goes through two rounds of the MurmurHash3 ``fmix32`` finaliser
(Appleby's published 32-bit avalanche mix).  Eight hashed bytes are summed
(an Irwin-Hall sum, mean 1020, standard deviation sqrt(8 * (256**2 - 1) / 12))
to give an approximately normal integer; one float32 multiply turns it into the
requested standard deviation and one round-to-nearest-even cast gives BF16.
Integer work is exact and a single IEEE float32 multiply rounds the same way on
every device, so ``approx_normal(..., device="cuda")`` equals the CPU result bit
for bit.  The tails are bounded at about 4.9 standard deviations.

Workload shapes follow the Beam layer as the architecture summary describes it
(hidden 5120, 256 experts of intermediate 2560 in 8 groups of 32, top-4 groups,
top-8 experts, routed scale 2.5) and a tiny layer with the same structure.
"""
from __future__ import annotations

import concurrent.futures
import dataclasses
import math
import os

import numpy as np
import torch

_MASK32 = 0xFFFFFFFF
_IH_MEAN = 8 * 255 / 2.0                       # mean of the sum of 8 uniform bytes
_IH_STD = math.sqrt(8 * (256 ** 2 - 1) / 12.0)  # its standard deviation
_CHUNK = 1 << 24                               # elements generated per pass
_THREADS = max(1, min(32, len(os.sched_getaffinity(0))))


def _fmix32_int(h: int) -> int:
    """MurmurHash3 fmix32 on a Python int (used for keys)."""
    h &= _MASK32
    h ^= h >> 16
    h = (h * 0x85EBCA6B) & _MASK32
    h ^= h >> 13
    h = (h * 0xC2B2AE35) & _MASK32
    h ^= h >> 16
    return h


def _mul32(h: torch.Tensor, c: int) -> torch.Tensor:
    """(h * c) mod 2**32 for 0 <= h < 2**32 held in int64, without int64 overflow."""
    lo = c & 0xFFFF
    hi = c >> 16
    return (h * lo + (((h * hi) & 0xFFFF) << 16)) & _MASK32


def _fmix32(h: torch.Tensor) -> torch.Tensor:
    h = h ^ (h >> 16)
    h = _mul32(h, 0x85EBCA6B)
    h = h ^ (h >> 13)
    h = _mul32(h, 0xC2B2AE35)
    h = h ^ (h >> 16)
    return h


def _keys(seed: int, stream: int) -> tuple[int, int]:
    k1 = _fmix32_int(seed * 0x9E3779B9 + 0x632BE5AB)
    k2 = _fmix32_int(k1 ^ _fmix32_int(stream * 0x85EBCA77 + 0x27D4EB2F))
    return k1, k2


def _ih_sum(idx: torch.Tensor, k1: int, k2: int) -> torch.Tensor:
    """Sum of the 8 bytes of two hashed words per element index (int64, 0..2040)."""
    total = torch.zeros_like(idx)
    for j in range(2):
        h = _fmix32(((idx * 2 + j) & _MASK32) ^ k1)
        h = _fmix32(h ^ k2)
        total += (h & 0xFF) + ((h >> 8) & 0xFF) + ((h >> 16) & 0xFF) + ((h >> 24) & 0xFF)
    return total


def _ih_sum_np(idx: np.ndarray, k1: int, k2: int) -> np.ndarray:
    """NumPy twin of ``_ih_sum``: uint32 arithmetic wraps modulo 2**32 natively."""
    total = np.zeros(idx.shape, dtype=np.uint32)
    m8 = np.uint32(0x00FF00FF)
    for j in range(2):
        h = idx * np.uint32(2)
        h += np.uint32(j)
        h ^= np.uint32(k1)
        for rnd in range(2):
            if rnd:
                h ^= np.uint32(k2)
            h ^= h >> np.uint32(16)
            h *= np.uint32(0x85EBCA6B)
            h ^= h >> np.uint32(13)
            h *= np.uint32(0xC2B2AE35)
            h ^= h >> np.uint32(16)
        pair = (h & m8) + ((h >> np.uint32(8)) & m8)      # two 16-bit byte-pair sums
        total += (pair & np.uint32(0xFFFF)) + (pair >> np.uint32(16))
    return total.astype(np.int64)


def _ih_sum_np_threaded(lo: int, hi: int, k1: int, k2: int) -> np.ndarray:
    out = np.empty(hi - lo, dtype=np.int64)
    step = 1 << 20
    def work(a):
        b = min(hi, a + step)
        out[a - lo:b - lo] = _ih_sum_np(np.arange(a, b, dtype=np.uint32), k1, k2)
    with concurrent.futures.ThreadPoolExecutor(max_workers=_THREADS) as ex:
        list(ex.map(work, range(lo, hi, step)))
    return out


def approx_normal(shape, seed: int, stream: int, std: float = 1.0, device="cpu",
                  dtype=torch.bfloat16, start: int = 0, backend: str = "auto") -> torch.Tensor:
    """Approximately N(0, std**2) values, deterministic and device-independent.

    ``start`` offsets the element counter, so a slice of a larger tensor can be
    regenerated on its own: ``approx_normal((n,), s, k, start=a)`` equals
    elements ``a .. a+n-1`` of the flattened larger tensor.  On the CPU the hash
    runs in NumPy uint32 arithmetic, on a GPU in torch int64 arithmetic; both
    compute the same integers (``backend`` forces one of "numpy" / "torch").
    """
    shape = tuple(int(d) for d in shape)
    n = int(np.prod(shape)) if shape else 1
    if start + n >= (1 << 31):
        raise ValueError("tensor too large for the 32-bit element counter")
    k1, k2 = _keys(seed, stream)
    use_np = backend == "numpy" or (backend == "auto" and torch.device(device).type == "cpu")
    scale = torch.tensor(std / _IH_STD, dtype=torch.float32)
    out = torch.empty(n, dtype=dtype, device=device)
    for a in range(0, n, _CHUNK):
        b = min(n, a + _CHUNK)
        if use_np:
            s = torch.from_numpy(_ih_sum_np_threaded(start + a, start + b, k1, k2)).to(device)
        else:
            idx = torch.arange(start + a, start + b, dtype=torch.int64, device=device)
            s = _ih_sum(idx, k1, k2)
        z = (s - 1020).to(torch.float32)
        out[a:b] = (z * scale.to(device)).to(dtype)
    return out.reshape(shape)


@dataclasses.dataclass(frozen=True)
class LayerShape:
    """Shape of one routed-expert layer."""
    H: int            # hidden size
    I: int            # expert intermediate size
    E: int            # routed experts
    n_groups: int     # expert groups (contiguous: expert e is in group e // (E // n_groups))
    topk_groups: int  # groups kept per token
    topk: int         # experts kept per token
    routed_scale: float
    wr_std: float     # router weight standard deviation
    w_std: float      # expert weight standard deviation (BF16, before quantisation)


# Tiny layer: 256 hidden, 32 experts of 128 in 8 groups of 4; router N(0, 1/256) (a variance).
TINY = LayerShape(H=256, I=128, E=32, n_groups=8, topk_groups=4, topk=8, routed_scale=2.5,
                  wr_std=1.0 / 16.0, w_std=0.02)
# Beam layer: hidden 5120, 256 experts of 2560 in 8 groups of 32; router N(0, 1/5120) (a variance).
BEAM = LayerShape(H=5120, I=2560, E=256, n_groups=8, topk_groups=4, topk=8, routed_scale=2.5,
                  wr_std=5120 ** -0.5, w_std=0.02)

# Streams of the counter generator.
_S_X, _S_WR = 1, 2


def _expert_stream(e: int, which: str) -> int:
    return 16 + 3 * e + {"gate": 0, "up": 1, "down": 2}[which]


def activations(T: int, shape: LayerShape, seed: int = 0, rms_rows: bool = False,
                device="cpu") -> torch.Tensor:
    """Layer input x as BF16 [T, H], N(0, 1); optionally each row rescaled to RMS 1."""
    x = approx_normal((T, shape.H), seed, _S_X, 1.0, device=device, dtype=torch.float32)
    if rms_rows:
        x64 = x.to("cpu", torch.float64)
        x64 = x64 / torch.sqrt((x64 * x64).mean(dim=1, keepdim=True))
        x = x64.to(torch.float32).to(device)
    return x.to(torch.bfloat16)


def router_weight(shape: LayerShape, seed: int = 0, device="cpu") -> torch.Tensor:
    """Router weight W_r as FP32 [E, H]."""
    return approx_normal((shape.E, shape.H), seed, _S_WR, shape.wr_std, device=device,
                         dtype=torch.float32)


def expert_weight(shape: LayerShape, e: int, which: str, seed: int = 0,
                  device="cpu") -> torch.Tensor:
    """BF16 weight of expert e before quantisation: gate/up [I, H], down [H, I]."""
    rows, cols = (shape.I, shape.H) if which in ("gate", "up") else (shape.H, shape.I)
    return approx_normal((rows, cols), seed, _expert_stream(e, which), shape.w_std,
                         device=device, dtype=torch.bfloat16)


def zipf_bias(E: int, s: float = 1.1, seed: int = 0) -> torch.Tensor:
    """Per-expert router-logit bias 0.5 * ln p(rank), p(r) proportional to r**-s.

    Ranks 1..E come from a seeded permutation of the experts (the counter hash
    of each expert index, ties by index).  Returned as FP32 [E].
    """
    k1, k2 = _keys(seed, 7)
    keys = [_fmix32_int(_fmix32_int(e ^ k1) ^ k2) for e in range(E)]
    order = sorted(range(E), key=lambda e: (keys[e], e))
    rank = np.empty(E, dtype=np.int64)
    for r, e in enumerate(order):
        rank[e] = r + 1
    p = np.arange(1, E + 1, dtype=np.float64) ** (-s)
    p /= p.sum()
    return torch.from_numpy((0.5 * np.log(p[rank - 1])).astype(np.float32))


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    shape: LayerShape
    T: int
    seed: int = 0
    rms_rows: bool = False
    zipf: bool = False

    def describe(self) -> str:
        s = self.shape
        return (f"{self.name}: T={self.T}, H={s.H}, I={s.I}, E={s.E} in {s.n_groups} groups, "
                f"top-{s.topk_groups} groups, top-{s.topk}, x{s.routed_scale}"
                + (", rows RMS 1" if self.rms_rows else "")
                + (", Zipf(1.1) logit bias" if self.zipf else ""))


WORKLOADS = {
    "tiny": Workload("tiny", TINY, 64),
    "decode": Workload("decode", BEAM, 16, rms_rows=True),
    "prefill": Workload("prefill", BEAM, 4096),
    "skewed": Workload("skewed", BEAM, 16384, zipf=True),
}
for _t in (1, 8, 64, 512, 4096, 32768):
    WORKLOADS[f"sweep{_t}"] = Workload(f"sweep{_t}", BEAM, _t)


def workload(name: str) -> Workload:
    return WORKLOADS[name]
