"""Dense projections through the C ABI (sfm_linear) against the oracle's
matmul in fp64: tcgen05 tiles with ragged M tails, every N-tile width (128,
192, 256: the width follows from M and N), single CTAs and CTA pairs, every
epilogue; fp32 mode on the CUDA cores."""
import numpy as np
import pytest
import torch

from oracle import sfm_oracle as O
from tests._gpu_util import rel_l2

pytestmark = pytest.mark.gpu

# 924 x 9216 / 12288 run on CTA pairs (256-row tiles); 800 x 12288 leaves the odd CTA
# of the last pair without rows
SHAPES = [(1, 128, 64), (130, 256, 128), (300, 384, 192), (924, 3072, 3072), (924, 9216, 3072),
          (924, 3072, 12288), (1848, 1024, 512), (800, 12288, 256)]


def _inputs(M, N, K, dtype, seed):
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    x = torch.randn(M, K, generator=g).to(dtype)
    w = (0.02 * torch.randn(N, K, generator=g)).to(dtype)
    return x, w


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_linear_bf16_f32_out(cuda_device, M, N, K):
    from streaming_flow_matching_b200 import linear
    x, w = _inputs(M, N, K, torch.bfloat16, M + N + K)
    y = linear(x.cuda(), w.cuda(), epilogue="f32")
    torch.cuda.synchronize()
    ref = O.linear(x, w)
    e = rel_l2(y.cpu().numpy(), ref)
    # bf16 products are exact in fp32; the fp32 sums over K carry ~ c sqrt(K) 2^-24
    # relative error (c <= 4): 2.6e-5 at K = 12288
    assert e <= 5e-5, e


@pytest.mark.parametrize("M,N,K", [(130, 256, 128), (300, 384, 192), (924, 3072, 3072),
                                   (924, 12288, 3072)])
def test_linear_bf16_epilogues(cuda_device, M, N, K):
    from streaming_flow_matching_b200 import linear
    x, w = _inputs(M, N, K, torch.bfloat16, 7 * M + N)
    xc, wc = x.cuda(), w.cuda()
    ref = O.linear(x, w)
    y = linear(xc, wc, epilogue="out")
    torch.cuda.synchronize()
    assert rel_l2(y.float().cpu().numpy(), ref) <= 5e-3
    y = linear(xc, wc, epilogue="gelu")
    torch.cuda.synchronize()
    assert rel_l2(y.float().cpu().numpy(), O.gelu_tanh(ref)) <= 5e-3
    base = torch.randn(M, N, generator=torch.Generator().manual_seed(5))
    y = base.clone().cuda()
    linear(xc, wc, y, epilogue="resid")
    torch.cuda.synchronize()
    # fp32 sum over K plus one fp32 add to the residual
    assert rel_l2(y.cpu().numpy(), O.f64(base) + ref) <= 2e-5


def test_linear_fp32(cuda_device):
    from streaming_flow_matching_b200 import linear
    x, w = _inputs(68, 768, 256, torch.float32, 3)
    y = linear(x.cuda(), w.cuda(), epilogue="f32")
    torch.cuda.synchronize()
    assert rel_l2(y.cpu().numpy(), O.linear(x, w)) <= 1e-6
