"""Host-side behaviour of the binding's layer object on the CPU (the library calls are
replaced by fakes): argument checks before any launch, and the workspace pool."""
import pytest
import torch

from nvfp4_mixture_experts_w4a4_b200 import _lib as C
from nvfp4_mixture_experts_w4a4_b200 import ops


class _Experts:
    E, I, H = 8, 128, 256
    w13_codes = torch.empty(0, dtype=torch.uint8)


class _FakeLib:
    def __init__(self):
        self.forward_calls = 0

    def moe_ffn_forward(self, *a):
        self.forward_calls += 1
        return 0


@pytest.fixture
def layer(monkeypatch):
    fake = _FakeLib()
    monkeypatch.setattr(ops, "_need_cuda", lambda *t: None)
    monkeypatch.setattr(ops, "_s", lambda s=None: None)
    monkeypatch.setattr(ops, "lib", lambda: fake)
    lay = ops.MoeFFN(_Experts(), 2, None)
    sizes = {}

    class _L:
        def __init__(self, total):
            self.total = total

    def layout(T):
        sizes[T] = sizes.get(T, 0) + 1
        return _L(1000 * T + 5000)  # grows with T
    monkeypatch.setattr(lay, "layout", layout)
    monkeypatch.setattr(lay, "desc", lambda *a, **k: C.MoeFfnDesc())
    lay.fake, lay.layout_calls = fake, sizes
    return lay


def test_workspaces_are_pooled_by_size_class(layer):
    a = layer.workspace(1)
    assert a.numel() == 1 << 20                     # the 1 MiB floor
    assert layer.workspace(500).data_ptr() == a.data_ptr()   # 505,000 bytes: same class
    b = layer.workspace(2000)                       # 2,005,000 bytes -> 2 MiB class
    assert b.numel() == 1 << 21 and b.data_ptr() != a.data_ptr()
    assert layer.workspace(1500).data_ptr() == b.data_ptr()  # 1,505,000 bytes -> 2 MiB
    assert len(layer._ws) == 2
    layer.workspace(1)
    assert layer.layout_calls[1] == 1               # the need of a batch size is asked once


def test_forward_checks_its_arguments_before_any_launch(layer):
    E, H = _Experts.E, _Experts.H
    x, logits = torch.zeros(4, H, dtype=torch.bfloat16), torch.zeros(4, E)
    bad = [dict(x=x.float(), logits=logits), dict(x=x[:, :128], logits=logits),
           dict(x=x, logits=torch.zeros(4, E + 1)), dict(x=x, logits=torch.zeros(3, E)),
           dict(x=x, logits=logits, out=torch.zeros(4, H)),
           dict(x=x, logits=logits, out=torch.zeros(H, 4, dtype=torch.bfloat16).t()),
           dict(x=x, logits=logits, h_amax=torch.zeros(E + 1)),
           dict(x=x, logits=logits, h_amax=torch.zeros(E, dtype=torch.float64))]
    for kw in bad:
        with pytest.raises(ValueError):
            layer.forward(**kw)
    assert layer.fake.forward_calls == 0
    out = layer.forward(x, logits, h_amax=torch.zeros(E))
    assert layer.fake.forward_calls == 1 and out.shape == (4, H) and out.dtype == torch.bfloat16
