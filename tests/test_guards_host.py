"""The guard bands of the GPU tests (parity_util.Guarded) on the host: a write
just past either end of the tensor is reported, writes inside are not."""
import pytest
import torch

from tests.parity_util import Guarded


@pytest.mark.parametrize("dtype,shape", [(torch.uint8, (3, 5)), (torch.int32, (7,)), (torch.bfloat16, (2, 3, 8)),
                                         (torch.float32, (1000,))])
def test_guard_bands_catch_writes_outside_the_tensor(dtype, shape):
    g = Guarded(shape, dtype, fill=1, device="cpu")
    assert g.t.shape == shape and g.t.dtype == dtype
    assert g.t.data_ptr() % 1024 == g.raw.data_ptr() % 1024  # the tensor keeps the allocation's alignment
    g.t.fill_(3)  # every element written: fine
    g.check("inside")
    for off in (g.GUARD - 1, g.GUARD + g.nbytes, g.raw.numel() - 1):
        h = Guarded(shape, dtype, device="cpu")
        h.raw[off] = 0  # one byte just before the tensor, just after it, at the far end
        with pytest.raises(AssertionError):
            h.check(f"byte {off}")
