"""The FMA-pipe exponential of the tensor-core Softmax kernel, element by
element against the exact 2^x (float64) and against CUDA's exp2f (through
torch.exp2 on the GPU), over its whole input range [-125, 64] and the clamp
below it."""
import numpy as np
import pytest
import torch

import softmax_attention_video_chunk_b200 as vdn

pytestmark = pytest.mark.gpu

REL_BOUND = 3e-6  # the polynomial's own fit error is 2.7e-6


def test_exp2_poly_relative_error_over_its_range(cuda_ok):
    g = torch.Generator().manual_seed(99)
    grid = torch.linspace(-125.0, 64.0, 4_000_001, dtype=torch.float32)
    # around the integers (the split x = n + f switches n there) and the
    # half-integers (|f| = 1/2, the ends of the polynomial's interval)
    ints = torch.arange(-125, 65, dtype=torch.float32)
    near = torch.cat([ints, ints + 0.5, ints - 0.5, torch.nextafter(ints + 0.5, ints),
                      torch.nextafter(ints + 0.5, ints + 1)])
    rand = (torch.rand(2_000_000, generator=g) * 189.0 - 125.0)
    x = torch.cat([grid, near.clamp(-125.0, 64.0), rand]).cuda()
    y = vdn.selftest_exp2(x)
    y_mufu = torch.exp2(x)
    torch.cuda.synchronize()
    xd = x.double().cpu().numpy()
    exact = np.exp2(xd)
    rel = np.abs(y.double().cpu().numpy() / exact - 1.0)
    rel_mufu = np.abs(y_mufu.double().cpu().numpy() / exact - 1.0)
    print(f"exp2 poly: max rel {rel.max():.3e}; exp2f: {rel_mufu.max():.3e}")
    assert np.all(np.isfinite(y.cpu().numpy()))
    assert rel.max() <= REL_BOUND
    # the two exponentials agree to within both errors
    assert np.max(np.abs(y.double().cpu().numpy() / y_mufu.double().cpu().numpy() - 1)) <= \
        REL_BOUND + rel_mufu.max()


def test_exp2_poly_clamps_below_minus_125(cuda_ok):
    x = torch.tensor([-125.0, -125.5, -126.0, -140.0, -1e4, -3.0e38, -float("inf")],
                     dtype=torch.float32, device="cuda")
    y = vdn.selftest_exp2(x).double().cpu().numpy()
    assert abs(y[0] / 2.0 ** -125 - 1) <= REL_BOUND
    assert np.all(y[1:] == y[0])  # clamped to 2^-125 ...
    assert np.all(torch.tensor(y).half().numpy() == 0)  # ... which is 0 as an fp16 P value


def test_exp2_poly_odd_length_and_in_place(cuda_ok):
    x = torch.linspace(-3, 3, 7, dtype=torch.float32, device="cuda")
    want = np.exp2(x.double().cpu().numpy())
    y = vdn.selftest_exp2(x)
    assert np.max(np.abs(y.double().cpu().numpy() / want - 1)) <= REL_BOUND
    rc = vdn.lib().vdn_selftest_exp2(x.data_ptr(), x.data_ptr(), x.numel(), None)
    torch.cuda.synchronize()
    assert rc == 0
    assert np.max(np.abs(x.double().cpu().numpy() / want - 1)) <= REL_BOUND
