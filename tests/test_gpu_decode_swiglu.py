"""GPU parity of the BF16 decode linear (against the oracle's binary64 dot
products) and of the fused SwiGLU epilogue / SwiGLU MLP prefill."""
import numpy as np
import pytest
import torch

import oracle
from mqtest import (assert_close, bf16_from_u16, check_h_from_gu, ensure_built, gpu_quantize,
                    oracle_prefill_rows,
                    sample_rows, u16)
from nvfp4_quantized_prefill_b200 import binding as mq
from nvfp4_quantized_prefill_b200 import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    ensure_built()


def gpu_decode(x_cpu, W):
    M = x_cpu.shape[0]
    y = torch.empty(M, W.N, dtype=torch.bfloat16, device="cuda")
    mq.mq_decode_linear_bf16(W.handle, x_cpu.cuda(), M, y)
    torch.cuda.synchronize()
    return y.cpu()


@pytest.mark.parametrize("M,N,K", [(1, 256, 256), (8, 300, 320), (3, 17, 64), (13, 1024, 4096),
                                   (1, 1, 128), (8, 4096, 14336), (2, 6150, 4096), (1, 33, 8192)])
def test_decode_small(M, N, K):
    x = workloads.activation("outlier", M, K, 2, M)
    w = workloads.weight(N, K, 0.02, 2, N)
    W = mq.Weight(w.cuda())
    y = gpu_decode(x, W)
    yr, pr = oracle.decode_linear(x, w)
    assert_close(y, yr, pr, f"decode {M}x{N}x{K}")
    W.free()
    assert mq.mq_check() == 0


def test_decode_deterministic_and_reusable():
    """Groups shared by several warps are summed in a fixed order: repeated
    calls give the same bits, and the per-weight counters are left ready for
    calls with another M on the same handle."""
    N, K = 6144, 4096
    w = workloads.weight(N, K, 0.02, 3, 0)
    W = mq.Weight(w.cuda())
    x = workloads.activation("outlier", 8, K, 3, 1)
    first = gpu_decode(x, W)
    for M in (1, 8, 3, 8):
        y = gpu_decode(x[:M], W)
        assert torch.equal(u16_t(y), u16_t(first[:M])), M
    yr, pr = oracle.decode_linear(x, w)
    assert_close(first, yr, pr, "decode 8x6144x4096")
    W.free()
    assert mq.mq_check() == 0


def u16_t(y):
    return y.view(torch.int16)


def test_decode_phase_switch_llama8b_mlp_weights():
    """Decode at M = 1 and M = 8 on the same handles the prefill uses."""
    wl = workloads.WORKLOADS["llama3_8b_mlp"]
    for i, w in enumerate(workloads.layer_weights(wl)):
        W = mq.Weight(w.cuda())
        for M in wl.decode_M:
            x = workloads.activation("outlier", M, w.shape[1], 20 + M, i)
            y = gpu_decode(x, W)
            yr, pr = oracle.decode_linear(x, w)
            assert_close(y, yr, pr, f"decode {wl.linears[i].name} M={M}")
        W.free()


def _swiglu_case(M, K, I, seed):
    x = workloads.activation("outlier", M, K, seed, 0)
    wgu = workloads.weight(2 * I, K, 0.02, seed, 1)
    Wgu = mq.Weight(wgu.cuda())
    codes, sf, s = gpu_quantize(x.cuda())
    c = torch.from_numpy(codes).cuda()
    f = torch.from_numpy(sf).cuda()
    sd = torch.tensor([s], dtype=torch.float32, device="cuda")
    # plain GEMM gives g | u ...
    y = torch.empty(M, 2 * I, dtype=torch.bfloat16, device="cuda")
    mq.mq_gemm_nvfp4(c, f, sd, M, Wgu.handle, y, 2 * I)
    # ... the fused epilogue gives h and its max
    h = torch.empty(M, I, dtype=torch.bfloat16, device="cuda")
    part = torch.empty(mq.MQ_AMAX_PARTIALS_MAX, dtype=torch.float32, device="cuda")
    n = mq.mq_gemm_nvfp4_swiglu(c, f, sd, M, Wgu.handle, h, part)
    torch.cuda.synchronize()
    return x, wgu, Wgu, y.cpu(), h.cpu(), float(part[:n].max())


@pytest.mark.parametrize("M,K,I", [(200, 256, 256), (128, 512, 384), (1, 64, 128)])
def test_swiglu_epilogue_small(M, K, I):
    x, wgu, Wgu, y, h, hmax = _swiglu_case(M, K, I, 3)
    yr, pr = oracle_prefill_rows(x, wgu, np.arange(M))
    assert_close(y, yr, pr, "gate/up")
    check_h_from_gu(y, h, I, "swiglu")
    assert hmax == float(h.float().abs().max())
    Wgu.free()
    assert mq.mq_check() == 0


def test_mlp_prefill_small_end_to_end():
    M, K, I = 300, 256, 256
    x = workloads.activation("outlier", M, K, 5, 0)
    wgu = workloads.weight(2 * I, K, 0.02, 5, 1)
    wd = workloads.weight(320, I, 0.02, 5, 2)
    Wgu, Wd = mq.Weight(wgu.cuda()), mq.Weight(wd.cuda())
    y = torch.empty(M, 320, dtype=torch.bfloat16, device="cuda")
    h = torch.empty(M, I, dtype=torch.bfloat16, device="cuda")
    nb = mq.mq_mlp_workspace_bytes(M, K, I)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    mq.mq_prefill_mlp_swiglu_nvfp4(Wgu.handle, Wd.handle, x.cuda(), M, y, h, ws, nb)
    torch.cuda.synchronize()
    # h: as from the separately computed gate/up GEMM
    _, _, _, yg, h2, _ = _swiglu_case(M, K, I, 5)
    assert torch.equal(h.cpu().view(torch.int16), h2.view(torch.int16))
    # quantization of h (amax from the epilogue) is bit-exact vs the oracle's
    hq_codes, hq_sf, hs = gpu_quantize(h)
    rc, rsf, rs, _ = oracle.quantize_tensor(h.cpu())
    assert hs == rs and np.array_equal(hq_codes, rc)
    assert np.array_equal(hq_sf, oracle.sf_swizzle(rsf))
    # down projection of the GPU's h against the oracle
    yr, pr = oracle_prefill_rows(h.cpu(), wd, np.arange(M))
    assert_close(y.cpu(), yr, pr, "mlp down")
    Wgu.free()
    Wd.free()


def test_mlp_prefill_llama8b_sampled_rows():
    wl = workloads.WORKLOADS["llama3_8b_mlp"]
    wgu, wd = workloads.layer_weights(wl)
    M, K, I = wl.M, wgu.shape[1], wgu.shape[0] // 2
    x = workloads.layer_activation(wl, K, 0)
    Wgu, Wd = mq.Weight(wgu.cuda()), mq.Weight(wd.cuda())
    y = torch.empty(M, wd.shape[0], dtype=torch.bfloat16, device="cuda")
    h = torch.empty(M, I, dtype=torch.bfloat16, device="cuda")
    nb = mq.mq_mlp_workspace_bytes(M, K, I)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    mq.mq_prefill_mlp_swiglu_nvfp4(Wgu.handle, Wd.handle, x.cuda(), M, y, h, ws, nb)
    torch.cuda.synchronize()
    rows = sample_rows(M, 4, 7)
    # gate/up rows by the oracle -> SwiGLU -> compare h (through the BF16 g, u
    # the GPU computes: g, u within the GEMM bound, h within an ulp of SwiGLU(g, u))
    gu = torch.empty(M, 2 * I, dtype=torch.bfloat16, device="cuda")
    codes, sf, s = gpu_quantize(x.cuda())
    mq.mq_gemm_nvfp4(torch.from_numpy(codes).cuda(), torch.from_numpy(sf).cuda(),
                     torch.tensor([s], device="cuda"), M, Wgu.handle, gu, 2 * I)
    torch.cuda.synchronize()
    r = torch.from_numpy(rows)
    gur, gpr = oracle_prefill_rows(x, wgu, rows)
    assert_close(gu[r].cpu(), gur, gpr, "llama8b gate/up")
    check_h_from_gu(gu[r].cpu(), h[r].cpu(), I, "llama8b swiglu")
    # down projection: oracle on the GPU's h (its full-tensor scale)
    hc = h.cpu()
    yr, pr = oracle_prefill_rows(hc, wd, rows)
    assert_close(y[r].cpu(), yr, pr, "llama8b down")
    Wgu.free()
    Wd.free()
    assert mq.mq_check() == 0
