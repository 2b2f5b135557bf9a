"""Empty problems through the Python API on the GPU: zero-size tensors (whose
data pointers may be null) are accepted and nothing is launched."""
import pytest
import torch

pytestmark = pytest.mark.gpu

fa = pytest.importorskip("exact_io_aware_55_b200")


@pytest.mark.parametrize("shape", [(1, 1, 0, 64), (0, 4, 128, 128), (2, 0, 64, 64)])
@pytest.mark.parametrize("causal", [False, True])
def test_empty_forward_backward_standard(shape, causal):
    q = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    o, lse = fa.attention_forward(q, q, q, causal=causal)
    assert o.shape == shape and lse.shape == shape[:3]
    dq, dk, dv = fa.attention_backward(q, q, q, o, q, lse, causal=causal)
    assert dq.shape == dk.shape == dv.shape == shape
    o2, lse2 = fa.attention_forward_standard(q, q, q, causal=causal)
    assert o2.shape == shape
    torch.cuda.synchronize()
    assert fa.fa_device_status() == (0, 0)


def test_empty_decode():
    q = torch.empty((2, 3, 0, 128), dtype=torch.bfloat16, device="cuda")
    k = torch.randn((2, 3, 64, 128), device="cuda").to(torch.bfloat16)
    o, lse = fa.attention_decode(q, k, k)
    assert o.shape == (2, 3, 0, 128) and lse.shape == (2, 3, 0)
    torch.cuda.synchronize()
    assert fa.fa_device_status() == (0, 0)
