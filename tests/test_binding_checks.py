"""The Python binding rejects tensors of the wrong dtype, shape, layout or device before any
pointer reaches the library.  CPU only: every call here fails a host-side check, and a call
whose CPU tensors pass all the others fails the device check, which comes last."""
import types

import pytest
import torch

import nvfp4_quantized_moe_group_b200 as moe


@pytest.fixture(scope="module")
def cfg():
    return moe.make_cfg(32, 8, 4, 8, 256, 128)


@pytest.fixture(scope="module")
def handle(cfg):
    # the layer calls read only .cfg before their checks pass; .handle is never used here
    return types.SimpleNamespace(cfg=cfg, handle=None)


def _x(T=4, H=256, dtype=torch.bfloat16):
    return torch.zeros((T, H), dtype=dtype)


def _raises(match, fn, *args, **kw):
    with pytest.raises(TypeError, match=match):
        fn(*args, **kw)


@pytest.mark.parametrize("fn", ["forward", "forward_fp8", "forward_partial"])
def test_layer_inputs(cfg, handle, fn):
    f = getattr(moe, fn)
    wr = torch.zeros((32, 256))
    _raises("x must be torch.bfloat16", f, handle, _x(dtype=torch.float32), wr)
    _raises(r"x must have shape \(4, 256\)", f, handle, _x(H=128), wr)
    _raises("x must be a 2-D tensor", f, handle, torch.zeros(256, dtype=torch.bfloat16), wr)
    _raises("x must be a 2-D tensor", f, handle, _x(T=0), wr)
    _raises("x must be contiguous", f, handle, _x(H=512)[:, ::2], wr)
    _raises("w_router must be torch.float32", f, handle, _x(), wr.to(torch.bfloat16))
    _raises(r"w_router must have shape \(32, 256\)", f, handle, _x(), wr.t().contiguous()[:32])
    _raises("w_router must be contiguous", f, handle, _x(), torch.zeros((256, 32)).t())
    _raises("bias must be torch.float32", f, handle, _x(), wr, torch.zeros(32, dtype=torch.float64))
    _raises(r"bias must have shape \(32,\)", f, handle, _x(), wr, torch.zeros(31))
    _raises("ws must be torch.uint8", f, handle, _x(), wr, ws=torch.zeros(1 << 20))
    _raises("must be a CUDA tensor", f, handle, _x(), wr)


def test_layer_outputs(cfg, handle):
    wr = torch.zeros((32, 256))
    _raises("out must be torch.bfloat16", moe.forward, handle, _x(), wr, out=_x(dtype=torch.float32))
    _raises(r"out must have shape \(4, 256\)", moe.forward, handle, _x(), wr, out=_x(T=5))
    _raises(r"out must have shape \(4, 256\)", moe.forward_fp8, handle, _x(), wr, out=_x(T=3))
    _raises("acc_out must be torch.float32", moe.forward_partial, handle, _x(), wr, acc_out=_x())
    _raises(r"acc_out must have shape", moe.forward_partial, handle, _x(), wr,
            acc_out=torch.zeros((4, 128)))


def test_residual_inputs(cfg, handle):
    wr = torch.zeros((32, 256))
    g = torch.ones(256)
    f = moe.forward_residual
    _raises("h must be torch.bfloat16", f, handle, _x(dtype=torch.float32), g, 1e-6, 2, wr)
    _raises(r"gamma must have shape \(256,\)", f, handle, _x(), torch.ones(128), 1e-6, 2, wr)
    _raises("gamma must be torch.float32", f, handle, _x(), g.to(torch.bfloat16), 1e-6, 2, wr)
    _raises(r"out must have shape \(4, 256\)", f, handle, _x(), g, 1e-6, 2, wr, out=_x(T=2))
    _raises("must be a CUDA tensor", f, handle, _x(), g, 1e-6, 2, wr)


def test_route_inputs(cfg):
    wr = torch.zeros((32, 256))
    _raises("w_router must be torch.float32", moe.route, cfg, _x(), wr.double())
    _raises(r"x must have shape \(0, 256\)", moe.route, cfg, _x(T=0, H=128), wr)
    _raises("must be a CUDA tensor", moe.route, cfg, _x(T=0), wr)
    _raises("must be a CUDA tensor", moe.route, cfg, _x(), wr)


def test_quantize_inputs():
    x = _x(T=3, H=64)
    _raises("x must be torch.bfloat16", moe.quantize, x.float())
    _raises("x must be a 2-D tensor", moe.quantize, torch.zeros(64, dtype=torch.bfloat16))
    _raises("g must be torch.float32", moe.quantize, x, g=torch.ones(1, dtype=torch.float64))
    _raises(r"g must have shape \(1,\)", moe.quantize, x, g=torch.ones(2))
    out = (torch.zeros((3, 32), dtype=torch.uint8), torch.zeros((3, 4), dtype=torch.uint8), torch.zeros(1))
    _raises(r"codes must have shape \(3, 32\)", moe.quantize, x, out=(torch.zeros((3, 64), dtype=torch.uint8),) + out[1:])
    _raises(r"scales must have shape \(512,\)", moe.quantize, x, swizzled=True, out=out)
    _raises("g_out must be torch.float32", moe.quantize, x, out=out[:2] + (torch.zeros(1, dtype=torch.int32),))
    _raises("must be a CUDA tensor", moe.quantize, x, out=out)
    _raises("x must be torch.bfloat16", moe.quantize_fp8, x.half())
    _raises("must be a CUDA tensor", moe.quantize_fp8, x)
    _raises(r"hess_blocks must have shape \(4, 16, 16\)", moe.quantize_weights_lh, x, torch.zeros((3, 16, 16)))
    _raises("hess_blocks must be torch.float32", moe.quantize_weights_lh, x, torch.zeros((4, 16, 16)).double())
    _raises("must be a CUDA tensor", moe.quantize_weights_lh, x, torch.zeros((4, 16, 16)))


def test_expert_tensors(cfg):
    H, I = cfg.H, cfg.I
    ex = types.SimpleNamespace(cfg=cfg)
    u8 = lambda r, c: torch.zeros((r, c), dtype=torch.uint8)     # noqa: E731
    gate = (u8(I, H // 2), u8(I, H // 16), 1.0)
    down = (u8(H, I // 2), u8(H, I // 16), 1.0)
    _raises(r"down codes must have shape \(256, 64\)", moe.Experts.set, ex, 0, gate, gate, gate, 1.0)
    _raises(r"gate scales must have shape \(128, 16\)", moe.Experts.set, ex, 0, (gate[0], u8(I, H // 32), 1.0),
            gate, down, 1.0)
    _raises("up codes must be torch.uint8", moe.Experts.set, ex, 0, gate, (gate[0].char(), gate[1], 1.0), down, 1.0)
    _raises("must be a CUDA tensor", moe.Experts.set, ex, 0, gate, gate, down, 1.0)
    f32 = lambda n: torch.zeros(n)                                # noqa: E731
    g8 = (u8(I, H), f32(I))
    d8 = (u8(H, I), f32(H))
    _raises(r"down scales must have shape \(256,\)", moe.Fp8Experts.set, ex, 0, g8, g8, (d8[0], f32(I)))
    _raises("gate scales must be torch.float32", moe.Fp8Experts.set, ex, 0, (g8[0], g8[1].half()), g8, d8)
    _raises("must be a CUDA tensor", moe.Fp8Experts.set, ex, 0, g8, g8, d8)


def test_finalize_inputs():
    acc = torch.zeros((4, 256))
    _raises("acc must be torch.float32", moe.finalize, acc.double())
    _raises(r"out must have shape \(4, 256\)", moe.finalize, acc, out=_x(T=3))
    _raises("must be a CUDA tensor", moe.finalize, acc)


def test_route_noalloc_inputs(cfg):
    wr = torch.zeros((32, 256))
    _raises(r"w_router must have shape \(32, 256\)", moe.route_noalloc, cfg, _x(), torch.zeros((32, 128)))
    _raises("x must be torch.bfloat16", moe.route_noalloc, cfg, _x(dtype=torch.float16), wr)
    _raises("must be a CUDA tensor", moe.route_noalloc, cfg, _x(), wr)


def test_every_declared_call_is_bound():
    from nvfp4_quantized_moe_group_b200 import _lib
    assert set(_lib.declared_symbols()) == set(_lib._SIGS)


def test_missing_library_fails_loudly(monkeypatch):
    """No CPU fallback: without the built library every call raises instead of computing."""
    from nvfp4_quantized_moe_group_b200 import _lib
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", "/nonexistent/libnvfp4moe.so")
    with pytest.raises(ImportError, match="is missing"):
        _lib.lib()
    with pytest.raises(ImportError):
        _lib.cfg_default()


class _OnCuda1(torch.Tensor):
    """A CPU tensor that reports itself as memory of cuda:1 (the device check reads only
    these two attributes)."""

    @property
    def is_cuda(self):
        return True

    @property
    def device(self):
        return torch.device("cuda", 1)


def test_tensors_of_another_device_than_the_current_one(monkeypatch):
    """The library launches on the current device, so tensors of another device are refused
    before any pointer reaches it."""
    from nvfp4_quantized_moe_group_b200 import _lib
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    x = torch.zeros((4, 256), dtype=torch.bfloat16).as_subclass(_OnCuda1)
    with pytest.raises(TypeError, match=r"on cuda:1 but the current device is cuda:0"):
        _lib._require((x, "x", torch.bfloat16, (4, 256)))
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 1)
    _lib._require((x, "x", torch.bfloat16, (4, 256)))
