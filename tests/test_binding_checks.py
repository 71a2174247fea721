"""The Python binding refuses, before anything is enqueued, tensor arguments that the
kernels would read or write out of bounds: host tensors, strided views, wrong element
types, shapes that disagree with the plan.  Checked on the CPU with stand-in tensors
(the attributes the binding looks at), so no device is needed."""
import pytest
import torch

import mixture_experts_fp32_b200 as moe


class FakeCuda:
    """Just enough of a CUDA tensor for the binding's checks."""

    def __init__(self, shape, dtype=torch.bfloat16, contiguous=True, addr=0x10000):
        self.shape = torch.Size(shape)
        self.dtype = dtype
        self.is_cuda = True
        self._contig = contiguous
        self._addr = addr

    def is_contiguous(self):
        return self._contig

    def dim(self):
        return len(self.shape)

    def numel(self):
        n = 1
        for s in self.shape:
            n *= s
        return n

    def data_ptr(self):
        return self._addr


def test_addresses():
    assert moe._addr(None) is None
    assert moe._addr(0x1234) == 0x1234
    assert moe._addr(FakeCuda((4, 8)), "x", moe._BF16) == 0x10000
    assert moe._addr(FakeCuda((4,), torch.bool), "valid", moe._MASK) == 0x10000
    assert moe._addr(FakeCuda((4, 8), torch.float8_e4m3fn), "w", moe._WEIGHT) == 0x10000
    with pytest.raises(ValueError, match="CUDA tensor"):
        moe._addr(torch.zeros(4, 8, dtype=torch.bfloat16), "hidden", moe._BF16)
    with pytest.raises(ValueError, match="contiguous"):
        moe._addr(FakeCuda((4, 8), contiguous=False), "hidden", moe._BF16)
    with pytest.raises(ValueError, match="element type"):
        moe._addr(FakeCuda((4, 8), torch.float16), "hidden", moe._BF16)
    with pytest.raises(ValueError, match="element type"):
        moe._addr(FakeCuda((4,), torch.int64), "perm", moe._I32)


def test_host_tensor_never_reaches_the_library():
    h = torch.zeros(4, 256, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="hidden"):
        moe.moe_forward(0, moe.moe_weights(), h, None, 4, 2, FakeCuda((4, 256)),
                        FakeCuda((1024,), torch.uint8), 1024, stream=0)
    with pytest.raises(ValueError, match="router_w"):
        moe.make_weights(torch.zeros(8, 256))


class _ShapeOnlyPlan(moe.Plan):
    """A Plan without a library plan or GPU: only the host-side shape checks of
    ``weights`` run (no router split is made)."""

    def weights(self, *a, **kw):
        return super().weights(*a, split_router=False, **kw)

    def close(self):
        pass


def _plan(wtype=moe.MOE_W_BF16, S=1):
    p = _ShapeOnlyPlan.__new__(_ShapeOnlyPlan)
    p.cfg = moe.moe_config(64, 256, 8, 2, 128, S, 128 if S else 0, 1, wtype)
    return p


def test_weight_shapes_against_the_plan():
    E, H, I, Is = 8, 256, 128, 128
    bf = dict(router_w=FakeCuda((E, H), torch.float32), w_gate_up=FakeCuda((E, 2 * I, H)),
              w_down=FakeCuda((E, H, I)), ws_gate_up=FakeCuda((2 * Is, H)),
              ws_down=FakeCuda((H, Is)))
    w = _plan().weights(**bf)
    assert w.router_w == 0x10000 and w.router_b is None
    with pytest.raises(ValueError, match="w_down"):
        _plan().weights(**{**bf, "w_down": FakeCuda((E, I, H))})        # transposed
    with pytest.raises(ValueError, match="ws_gate_up is required"):
        _plan().weights(**{**bf, "ws_gate_up": None})
    with pytest.raises(ValueError, match="router_b"):
        _plan().weights(**bf, router_b=FakeCuda((E + 1,), torch.float32))
    no_shared = {k: v for k, v in bf.items() if not k.startswith("ws_")}
    _plan(S=0).weights(**no_shared)
    u8 = torch.uint8
    f8 = dict(router_w=bf["router_w"], w_gate_up=FakeCuda((E, 2 * I, H), u8),
              w_down=FakeCuda((E, H, I), u8),
              s_gate_up=FakeCuda((E, 2 * I // 128, H // 128), torch.float32),
              s_down=FakeCuda((E, H // 128, I // 128), torch.float32),
              ws_gate_up=FakeCuda((2 * Is, H), u8), ws_down=FakeCuda((H, Is), u8),
              ss_gate_up=FakeCuda((2 * Is // 128, H // 128), torch.float32),
              ss_down=FakeCuda((H // 128, Is // 128), torch.float32))
    _plan(moe.MOE_W_FP8_E4M3_B128).weights(**f8)
    with pytest.raises(ValueError, match="s_down"):
        _plan(moe.MOE_W_FP8_E4M3_B128).weights(
            **{**f8, "s_down": FakeCuda((E, I // 128, H // 128), torch.float32)})
    with pytest.raises(ValueError, match="s_gate_up is required"):
        _plan(moe.MOE_W_FP8_E4M3_B128).weights(**{**f8, "s_gate_up": None})


def test_row_and_slab_shapes():
    p = _plan()
    assert p._rows(FakeCuda((64, 256)), FakeCuda((64,), torch.uint8), FakeCuda((64, 256))) == 64
    assert p._rows(FakeCuda((0, 256)), None) == 0
    with pytest.raises(ValueError, match="hidden"):
        p._rows(FakeCuda((64, 128)), None)
    with pytest.raises(ValueError, match="valid"):
        p._rows(FakeCuda((64, 256)), FakeCuda((63,), torch.uint8))
    with pytest.raises(ValueError, match="out"):
        p._rows(FakeCuda((64, 256)), None, FakeCuda((64, 255)))
    p._slabs([FakeCuda((2, 32, 256), torch.float32)] * 2, 32)
    p._slabs([0x1000, 0x2000], 32)                                      # raw addresses
    with pytest.raises(ValueError, match="slab"):
        p._slabs([FakeCuda((1, 32, 256), torch.float32)] * 2, 32)
