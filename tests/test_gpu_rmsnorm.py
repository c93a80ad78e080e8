"""GPU parity of the RMSNorm that emits the quantizer's amax, and of the
prefill linear fed by it: the normalised rows against the oracle's binary64
RMSNorm (two BF16 steps at most, nearly all identical), the NVFP4 codes of the
GPU's rows bit-exact, the GEMM within tolerance."""
import numpy as np
import pytest
import torch

import oracle
from mqtest import assert_close, bf16_from_u16, ensure_built, oracle_prefill_rows, u16
from nvfp4_quantized_prefill_b200 import binding as mq
from nvfp4_quantized_prefill_b200 import workloads

pytestmark = pytest.mark.gpu
EPS = 1e-5


@pytest.fixture(scope="module", autouse=True)
def _built():
    ensure_built()


def check_rows(y_gpu_u16: np.ndarray, y_ref_u16: np.ndarray, what: str):
    """Identical almost everywhere, and never more than two BF16 steps apart.
    The binary32 reciprocal root r can differ from the binary64 one by an ulp,
    which moves t = bf16(x r) by at most one step (|t| 2^-7); y = bf16(g t)
    then moves by |g| |t| 2^-7 ~ |y| 2^-7 plus its own rounding step, hence
    two steps of |y| 2^-7."""
    yg = torch.from_numpy(y_gpu_u16.view(np.int16)).view(torch.bfloat16).double()
    yr = torch.from_numpy(y_ref_u16.view(np.int16)).view(torch.bfloat16).double()
    step = torch.where(yr == 0, torch.full_like(yr, 2.0 ** -133), yr.abs() * 2.0 ** -7)
    assert ((yg - yr).abs() <= 2.0 * step * 1.0001).all(), what
    assert (y_gpu_u16 == y_ref_u16).mean() > 0.999, what


# K <= 4096 and K <= 8192: the CTA-per-row kernel's two forms; K = 16384: the
# warp-per-row kernel
@pytest.mark.parametrize("M,K,ldx", [(1, 64, 64), (37, 320, 328), (300, 4096, 4096),
                                     (8, 8192, 8192), (5, 8, 8), (1000, 2048, 2056),
                                     (20, 16384, 16384), (700, 6144, 6144)])
def test_rmsnorm_amax(M, K, ldx):
    x = workloads.activation("channel_gain", M, ldx, 21, M)
    g = workloads.rmsnorm_gain(K, 21, 1)
    xd = x.cuda()
    y = torch.empty(M, K, dtype=torch.bfloat16, device="cuda")
    part = torch.empty(mq.MQ_AMAX_PARTIALS_MAX, dtype=torch.float32, device="cuda")
    n = mq.mq_rmsnorm_amax(xd, g.cuda(), EPS, M, K, ldx, y, part)
    torch.cuda.synchronize()
    yu = u16(y.cpu())
    ref = oracle.rmsnorm(x[:, :K].contiguous(), g, EPS)
    check_rows(yu, ref, f"rmsnorm {M}x{K}")
    # the partial maxima are exactly the maximum |y| of what was written
    amax = float(part[:n].max().cpu())
    assert amax == float(y.float().abs().max().cpu())
    assert mq.mq_check() == 0


@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (300, 520, 512), (1000, 1024, 4096)])
def test_prefill_linear_rmsnorm(M, N, K):
    r = workloads.activation("channel_gain", M, K, 22, 0)
    g = workloads.rmsnorm_gain(K, 22, 1)
    w = workloads.weight(N, K, 0.02, 22, 2)
    W = mq.Weight(w.cuda())
    xn = torch.empty(M, K, dtype=torch.bfloat16, device="cuda")
    y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    nb = mq.mq_workspace_bytes(M, K)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    mq.mq_prefill_linear_rmsnorm_nvfp4(W.handle, r.cuda(), g.cuda(), EPS, M, xn, y, ws, nb)
    torch.cuda.synchronize()
    xn_u = u16(xn.cpu())
    check_rows(xn_u, oracle.rmsnorm(r, g, EPS), "rmsnorm in the linear")
    # the quantizer saw the GPU's rows: codes bit-exact against the oracle on them
    xn_cpu = bf16_from_u16(xn_u)
    s = oracle.tensor_scale(oracle.tensor_amax(xn_cpu))
    xc, _ = oracle.quantize(xn_cpu, s)
    codes = ws[: M * K // 2].view(M, K // 2).cpu().numpy()
    assert np.array_equal(codes, xc)
    yr, pr = oracle_prefill_rows(xn_cpu, w, np.arange(M))
    assert_close(y.cpu(), yr, pr, f"rmsnorm prefill {M}x{N}x{K}")
    W.free()
    assert mq.mq_check() == 0
