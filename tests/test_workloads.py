"""The seeded input generators: deterministic, slice-consistent, same integers from the
NumPy and torch backends, and the requested mean/spread (CPU only)."""
import numpy as np
import torch

from workloads import BEAM, TINY, activations, approx_normal, expert_weight, router_weight, zipf_bias


def test_backends_agree_bit_for_bit():
    a = approx_normal((777, 129), 5, 11, 0.3, backend="numpy", dtype=torch.float32)
    b = approx_normal((777, 129), 5, 11, 0.3, backend="torch", dtype=torch.float32)
    assert torch.equal(a, b)
    a = approx_normal((4096,), 1, 2, backend="numpy", start=(1 << 31) - 5000)
    b = approx_normal((4096,), 1, 2, backend="torch", start=(1 << 31) - 5000)
    assert torch.equal(a, b)


def test_slices_regenerate():
    full = approx_normal((10, 64), 0, 3)
    part = approx_normal((3, 64), 0, 3, start=4 * 64)
    assert torch.equal(full[4:7], part)


def test_distribution_and_independence():
    x = approx_normal((1 << 20,), 0, 1, dtype=torch.float32).double()
    assert abs(x.mean().item()) < 5e-3 and abs(x.std().item() - 1) < 5e-3
    y = approx_normal((1 << 20,), 0, 2, dtype=torch.float32).double()
    assert abs(torch.corrcoef(torch.stack([x, y]))[0, 1].item()) < 5e-3
    assert x.abs().max().item() < 5.0


def test_layer_inputs_shapes_and_scales():
    x = activations(16, BEAM, rms_rows=True).double()
    assert x.shape == (16, 5120)
    np.testing.assert_allclose(x.pow(2).mean(dim=1).sqrt().numpy(), 1.0, atol=1e-2)
    wr = router_weight(TINY)
    assert wr.dtype == torch.float32 and abs(wr.std().item() - 1 / 16) < 3e-3
    w = expert_weight(TINY, 3, "down")
    assert w.shape == (256, 128) and w.dtype == torch.bfloat16 and abs(w.float().std().item() - 0.02) < 1e-3
    assert not torch.equal(expert_weight(TINY, 3, "gate"), expert_weight(TINY, 4, "gate"))


def test_zipf_bias_range():
    b = zipf_bias(256).double()
    assert torch.unique(b).numel() == 256
    p = np.arange(1, 257) ** -1.1
    p /= p.sum()
    assert abs(b.max().item() - 0.5 * np.log(p[0])) < 1e-6 and abs(b.min().item() - 0.5 * np.log(p[-1])) < 1e-6


def test_hash_follows_the_published_fmix32():
    """Both backends' hash is MurmurHash3's 32-bit finaliser: the torch one (int64 with emulated
    32-bit products) equals the plain Python-integer statement of it on edge and random words;
    fmix32(1) = 0x514E28B7 and fmix32(0) = 0, values the finaliser is commonly checked with."""
    from workloads.synthetic import _fmix32, _fmix32_int
    assert _fmix32_int(0) == 0 and _fmix32_int(1) == 0x514E28B7
    words = [0, 1, 2, 0x7FFFFFFF, 0x80000000, 0xFFFFFFFF, 0xDEADBEEF]
    words += np.random.default_rng(0).integers(0, 1 << 32, 2000, dtype=np.uint64).tolist()
    got = _fmix32(torch.tensor(words, dtype=torch.int64)).tolist()
    assert got == [_fmix32_int(w) for w in words]
