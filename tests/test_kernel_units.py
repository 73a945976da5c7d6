"""GPU checks of building blocks of the tensor-core kernels."""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

moda = pytest.importorskip("depth_kv_attention_b200")


def test_fma_pipe_exp2_within_bound():
    """The polynomial exp2 that takes part of the softmax exponentials off the
    MUFU unit: relative error <= 1e-4 against float64 2^x over the range the
    softmax feeds it, and compared with CUDA's exp2f."""
    x = np.concatenate([np.linspace(-125.0, 16.0, 400001), [0.0, -0.5, 0.5, 1.0, -1.0, 8.0]])
    x32 = torch.tensor(x, dtype=torch.float32, device="cuda")
    y = moda.moda_debug_exp2_poly(x32)
    ref_cuda = torch.exp2(x32)
    torch.cuda.synchronize()
    xe = x32.double().cpu().numpy()
    got = y.double().cpu().numpy()
    rel = np.abs(got / np.exp2(xe) - 1.0)
    assert rel.max() <= 1e-4, rel.max()
    relc = np.abs(got / ref_cuda.double().cpu().numpy() - 1.0)
    assert relc.max() <= 1.1e-4, relc.max()
    # masked logits (-inf) and values below the clamp stay negligible
    z = moda.moda_debug_exp2_poly(torch.tensor([-np.inf, -1000.0, -126.0], device="cuda"))
    assert float(z.max()) < 1e-37
