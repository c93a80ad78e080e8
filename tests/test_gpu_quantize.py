"""GPU parity of NVFP4 quantization (mq_tensor_amax, mq_quantize_nvfp4,
mq_weight_pack) against the CPU oracle: codes, swizzled scales (padding
included) and the tensor scale must match bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from mqtest import ensure_built, fetch_device, gpu_quantize, u16
from nvfp4_quantized_prefill_b200 import binding as mq
from nvfp4_quantized_prefill_b200 import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    ensure_built()


def check_quant(x_cpu: torch.Tensor, what: str):
    codes, sf, s = gpu_quantize(x_cpu.cuda())
    rc, rsf, rs, _ = oracle.quantize_tensor(x_cpu)
    assert np.float32(s) == np.float32(rs), (what, s, rs)
    assert np.array_equal(codes, rc), f"{what}: {(codes != rc).sum()} code bytes differ"
    rswz = oracle.sf_swizzle(rsf)
    assert sf.size == rswz.size
    assert np.array_equal(sf, rswz), f"{what}: {(sf != rswz).sum()} scale bytes differ"


@pytest.mark.parametrize("M,K", [(128, 256), (200, 320), (1, 64), (129, 1024), (37, 448),
                                 (256, 4096)])
@pytest.mark.parametrize("kind", workloads.ACT_KINDS)
def test_quantize_small_bitexact(M, K, kind):
    check_quant(workloads.activation(kind, M, K, 7, M + K), f"{kind} {M}x{K}")


def _tie_matrix():
    """Blocks whose scale makes x * f exact, holding every E2M1 and E4M3
    rounding tie (both signs), plus zero / negative-zero blocks."""
    ties = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    rows = []
    for e in [0, -3, -8, 2]:            # block max 6 * 2^e -> scale 2^e exactly (s_enc = 1)
        blk = [6.0] + ties + [-t for t in ties] + [-0.0]
        rows.append([v * 2.0 ** e for v in blk])
    rows.append([6.375] + [1.0] * 15)   # scale 1.0625: E4M3 tie -> 1.0
    rows.append([7.125] + [1.0] * 15)   # scale 1.1875: E4M3 tie -> 1.25
    rows.append([0.0] * 16)
    rows.append([-0.0] * 16)
    rows.append([2688.0] + [0.1 * i for i in range(15)])   # tensor amax -> s_enc = 1
    v = np.array(rows, dtype=np.float64)
    x = np.zeros((128, 64), dtype=np.float64)
    x[: v.shape[0], :16] = v
    x[: v.shape[0], 16:32] = -v
    x[: v.shape[0], 32:48] = v[:, ::-1]
    return torch.tensor(x, dtype=torch.float32).to(torch.bfloat16)


def test_quantize_ties_bitexact():
    x = _tie_matrix()
    assert oracle.tensor_scale(oracle.tensor_amax(x)) == 1.0
    check_quant(x, "ties")


def test_quantize_zero_tensor():
    x = torch.zeros(130, 128, dtype=torch.bfloat16)
    x[3, 5] = -0.0
    check_quant(x, "zeros")
    codes, sf, s = gpu_quantize(x.cuda())
    assert s == 1.0 and (sf == 0).all()


def test_quantize_full_llama8b_activation_bitexact():
    for kind in ("outlier", "channel_gain"):
        check_quant(workloads.activation(kind, 8192, 4096, 1, 0), f"{kind} 8192x4096")


def test_quantize_strided_rows_and_external_amax():
    M, K, ld = 300, 512, 640
    full = workloads.activation("outlier", M, ld, 3, 0)
    x_cpu = full[:, :K].contiguous()
    xg = full.cuda()
    codes = torch.empty(M, K // 2, dtype=torch.uint8, device="cuda")
    sf = torch.empty(mq.mq_sf_bytes(M, K), dtype=torch.uint8, device="cuda")
    s = torch.empty(1, dtype=torch.float32, device="cuda")
    part = torch.empty(mq.MQ_AMAX_PARTIALS_MAX, dtype=torch.float32, device="cuda")
    n = mq.mq_tensor_amax(xg, M, K, ld, part)
    assert 1 <= n <= mq.MQ_AMAX_PARTIALS_MAX
    torch.cuda.synchronize()
    assert float(part[:n].max()) == oracle.tensor_amax(x_cpu)
    mq.mq_quantize_nvfp4(xg, M, K, ld, codes, sf, s, amax_partials=part, n_partials=n)
    torch.cuda.synchronize()
    rc, rsf, rs, _ = oracle.quantize_tensor(x_cpu)
    assert float(s.item()) == rs
    assert np.array_equal(codes.cpu().numpy(), rc)
    assert np.array_equal(sf.cpu().numpy(), oracle.sf_swizzle(rsf))
    assert mq.mq_check() == 0


def test_quantize_amax_inside_strided_and_workspace_reuse():
    """Amax taken inside mq_quantize_nvfp4 (partial maxima in the workspace):
    strided rows, and a workspace reused across calls -- the second call (a
    much smaller amax) must not see the first call's partial maxima."""
    ws = torch.empty(mq.MQ_AMAX_PARTIALS_MAX, dtype=torch.float32, device="cuda")
    for M, K, ld, gain in ((3000, 4096, 4160, 30.0), (3000, 4096, 4160, 0.01), (17, 448, 448, 1.0)):
        full = (workloads.activation("outlier", M, ld, 4, 1).float() * gain).to(torch.bfloat16)
        x_cpu = full[:, :K].contiguous()
        codes = torch.empty(M, K // 2, dtype=torch.uint8, device="cuda")
        sf = torch.empty(mq.mq_sf_bytes(M, K), dtype=torch.uint8, device="cuda")
        s = torch.empty(1, dtype=torch.float32, device="cuda")
        mq.mq_quantize_nvfp4(full.cuda(), M, K, ld, codes, sf, s, workspace=ws,
                             ws_bytes=ws.numel() * 4)
        torch.cuda.synchronize()
        rc, rsf, rs, _ = oracle.quantize_tensor(x_cpu)
        assert float(s.item()) == rs, (M, K, gain)
        assert np.array_equal(codes.cpu().numpy(), rc), (M, K, gain)
        assert np.array_equal(sf.cpu().numpy(), oracle.sf_swizzle(rsf)), (M, K, gain)
    assert mq.mq_check() == 0


@pytest.mark.parametrize("N,K", [(520, 320), (256, 256), (6144, 4096)])
def test_weight_pack_views_bitexact(N, K):
    w = workloads.weight(N, K, 0.02, 5, N)
    W = mq.Weight(w.cuda())
    v = W.views()
    assert v["N"] == N and v["K"] == K
    torch.cuda.synchronize()
    nbytes_sf = mq.mq_sf_bytes(N, K)

    bf = fetch_device(v["bf16"], N * K * 2).view(np.uint16).reshape(N, K)
    assert np.array_equal(bf, u16(w))
    codes = fetch_device(v["codes"], N * K // 2).reshape(N, K // 2)
    sf = fetch_device(v["sf"], nbytes_sf)
    s = fetch_device(v["s_enc"], 4).view(np.float32)[0]
    rc, rsf, rs, _ = oracle.quantize_tensor(w)
    assert np.float32(s) == np.float32(rs)
    assert np.array_equal(codes, rc)
    assert np.array_equal(sf, oracle.sf_swizzle(rsf))
    W.free()
    assert mq.mq_check() == 0


def _dynamic_range_matrix(M=256, K=512, seed=4):
    """Blocks whose magnitudes span 2^-60 .. 2^40: some block scales land in
    E4M3's subnormal range or underflow to zero relative to the tensor scale,
    one block holds the tensor maximum, signs and zeros mixed in."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K))
    exps = rng.integers(-60, 41, size=(M, K // 16))
    x *= np.repeat(2.0 ** exps, 16, axis=1)
    x[rng.random((M, K)) < 0.05] = 0.0
    x[0, :16] = 3.0e12   # a constant block near the top of the range
    return torch.tensor(x, dtype=torch.float32).to(torch.bfloat16)


def test_quantize_dynamic_range_bitexact():
    x = _dynamic_range_matrix()
    check_quant(x, "dynamic range")
    codes, sf, s = gpu_quantize(x.cuda())
    # blocks far below the maximum quantize to zero scales and zero codes
    assert (sf == 0).any() and (sf != 0).any()


def test_prefill_dynamic_range_within_tolerance():
    from mqtest import assert_close, oracle_prefill_rows
    x = _dynamic_range_matrix(128, 512, 5)
    w = workloads.weight(384, 512, 0.02, 5, 1)
    W = mq.Weight(w.cuda())
    y = torch.empty(128, 384, dtype=torch.bfloat16, device="cuda")
    nb = mq.mq_workspace_bytes(128, 512)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    mq.mq_prefill_linear_nvfp4(W.handle, x.cuda(), 128, y, ws, nb)
    torch.cuda.synchronize()
    yr, pr = oracle_prefill_rows(x, w, np.arange(128))
    assert_close(y.cpu(), yr, pr, "dynamic-range prefill")
    W.free()
