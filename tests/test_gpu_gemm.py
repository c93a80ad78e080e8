"""GPU parity of the block-scaled NVFP4 GEMM (mq_prefill_linear_nvfp4,
mq_gemm_nvfp4) against the oracle's exact sum: every output element within
|gpu - ref| <= 2^-8 |ref| + 1e-5 * sum|products|."""
import numpy as np
import pytest
import torch

import oracle
from mqtest import (assert_close, check_h_from_gu, ensure_built, gpu_quantize, oracle_prefill_rows,
                    sample_rows)
from nvfp4_quantized_prefill_b200 import binding as mq
from nvfp4_quantized_prefill_b200 import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    ensure_built()


def gpu_prefill(x_cpu: torch.Tensor, W: "mq.Weight") -> torch.Tensor:
    M, K = x_cpu.shape
    x = x_cpu.cuda()
    y = torch.empty(M, W.N, dtype=torch.bfloat16, device="cuda")
    nb = mq.mq_workspace_bytes(M, K)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    mq.mq_prefill_linear_nvfp4(W.handle, x, M, y, ws, nb)
    torch.cuda.synchronize()
    return y


# (M, N, K): one tile; several tiles with ragged M / N tails; partial last
# K-tile (K % 256 != 0); N not a multiple of 8 (scalar store path); K = 64.
SMALL = [(128, 256, 256), (300, 520, 512), (1, 256, 64), (257, 768, 320), (130, 100, 448),
         (512, 1024, 1024), (64, 264, 128), (1000, 4096, 256)]


@pytest.mark.parametrize("M,N,K", SMALL)
def test_prefill_small_all_elements(M, N, K):
    x = workloads.activation("outlier", M, K, 0, M)
    w = workloads.weight(N, K, 0.02, 0, N)
    W = mq.Weight(w.cuda())
    y = gpu_prefill(x, W)
    yr, pr = oracle_prefill_rows(x, w, np.arange(M))
    assert_close(y.cpu(), yr, pr, f"prefill {M}x{N}x{K}")
    W.free()
    assert mq.mq_check() == 0


def test_tiny_config_matches_oracle():
    """Tiny layer: X [128, 256] outlier recipe, W [256, 256], seed 0."""
    wl = workloads.WORKLOADS["tiny"]
    w = workloads.layer_weights(wl)[0]
    x = workloads.layer_activation(wl, 256, 0)
    W = mq.Weight(w.cuda())
    y = gpu_prefill(x, W)
    yr, pr = oracle_prefill_rows(x, w, np.arange(128))
    assert_close(y.cpu(), yr, pr, "tiny")
    W.free()


def test_gemm_entry_with_leading_dimension():
    M, N, K, ld = 200, 384, 512, 400
    x = workloads.activation("student_t3", M, K, 4, 0)
    w = workloads.weight(N, K, 0.02, 4, 1)
    W = mq.Weight(w.cuda())
    codes, sf, s = gpu_quantize(x.cuda())
    y = torch.full((M, ld), 7.0, dtype=torch.bfloat16, device="cuda")
    c = torch.from_numpy(codes).cuda()
    f = torch.from_numpy(sf).cuda()
    sd = torch.tensor([s], dtype=torch.float32, device="cuda")
    mq.mq_gemm_nvfp4(c, f, sd, M, W.handle, y, ld)
    torch.cuda.synchronize()
    yr, pr = oracle_prefill_rows(x, w, np.arange(M))
    assert_close(y[:, :N].cpu(), yr, pr, "gemm ldy")
    assert (y[:, N:] == 7.0).all()          # nothing written past N
    W.free()


def _lossless(rows, K, seed, k_lo, k_hi):
    rng = np.random.default_rng(seed)
    mags = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    v = mags[rng.integers(0, 8, size=(rows, K))] * rng.choice([-1.0, 1.0], size=(rows, K))
    kb = rng.integers(k_lo, k_hi + 1, size=(rows, K // 16))
    kb[0, 0] = k_hi
    v = v.reshape(rows, K // 16, 16)
    v[:, :, 0] = 6.0 * rng.choice([-1.0, 1.0], size=(rows, K // 16))
    v = (v * (2.0 ** kb)[:, :, None]).reshape(rows, K)
    v[0, 0] = abs(v[0, 0])
    return torch.tensor(v, dtype=torch.float32).to(torch.bfloat16), v


def test_prefill_lossless_inputs_give_rounded_exact_product():
    """Inputs NVFP4 represents exactly: Y is the exact product rounded to BF16."""
    x, xv = _lossless(256, 512, 1, -3, 1)
    w, wv = _lossless(512, 512, 2, -5, -1)
    W = mq.Weight(w.cuda())
    y = gpu_prefill(x, W).float().cpu().double().numpy()
    exact = xv @ wv.T
    ref = torch.tensor(exact).to(torch.bfloat16).double().numpy()
    # FP32 accumulation of exact dyadic terms: at most a few ulps before rounding
    assert (np.abs(y - ref) <= 2.0 ** -8 * np.abs(exact) + 1e-6).all()
    W.free()


def test_prefill_llama8b_qkv_o_sampled_rows():
    wl = workloads.WORKLOADS["llama3_8b_qkv_o"]
    ws = workloads.layer_weights(wl)
    for i, w in enumerate(ws):
        x = workloads.layer_activation(wl, w.shape[1], i)
        W = mq.Weight(w.cuda())
        y = gpu_prefill(x, W)
        rows = sample_rows(wl.M, 12, i)
        yr, pr = oracle_prefill_rows(x, w, rows)
        assert_close(y[torch.from_numpy(rows)].cpu(), yr, pr, f"llama8b {wl.linears[i].name}")
        W.free()
    assert mq.mq_check() == 0


def test_prefill_chunk_16384_tokens_sampled():
    """One 16384-token chunk (Student-t activations) through the O-shaped and
    the 14336-wide projections, each chunk quantized with its own scale."""
    wl = workloads.WORKLOADS["chunked_131k"]
    x = workloads.layer_activation(wl, 4096, 0)
    for i, w in enumerate(workloads.layer_weights(wl)):
        W = mq.Weight(w.cuda())
        y = gpu_prefill(x, W)
        rows = sample_rows(wl.M, 6, 10 + i)
        cols = np.sort(np.random.default_rng(i).choice(w.shape[0], 1024, replace=False))
        yr, pr = oracle_prefill_rows(x, w, rows, wrows=cols)
        ys = y[torch.from_numpy(rows)][:, torch.from_numpy(cols)].cpu()
        assert_close(ys, yr, pr, f"chunk {wl.linears[i].name}")
        W.free()


# Llama-3-70B-shaped layer at 16384 tokens: the deepest K (down, K = 28672:
# 112 K steps of 256 per tile) and the widest N (gate+up, N = 57344) the
# library runs.  The inputs are drawn with the workload's recipes on the GPU's
# generator (same distributions, so the 470M-element tensors take seconds) and
# copied to the host for the oracle; sampled rows x sampled columns keep the
# oracle's exact sum to seconds.
_L70 = workloads.WORKLOADS["llama3_70b_layer"]


def _gpu_inputs_70b(i: int, K: int):
    lin = _L70.linears[i]
    w = workloads.weight(lin.N, lin.K, lin.std, _L70.seed, 100 + i, device="cuda")
    x = workloads.activation(_L70.act, _L70.M, K, _L70.seed, i, device="cuda")
    return x, w


def _prefill_dev(x: torch.Tensor, W: "mq.Weight") -> torch.Tensor:
    M, K = x.shape
    y = torch.empty(M, W.N, dtype=torch.bfloat16, device="cuda")
    nb = mq.mq_workspace_bytes(M, K)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    mq.mq_prefill_linear_nvfp4(W.handle, x, M, y, ws, nb)
    torch.cuda.synchronize()
    del ws
    return y


@pytest.mark.parametrize("i", [0, 1, 2, 3], ids=["qkv", "o", "gate_up", "down"])
def test_prefill_llama70b_shapes_sampled(i):
    lin = _L70.linears[i]
    x, w = _gpu_inputs_70b(i, lin.K)
    W = mq.Weight(w)
    y = _prefill_dev(x, W)
    rows = sample_rows(_L70.M, 5, 20 + i)
    cols = np.sort(np.random.default_rng(30 + i).choice(lin.N, 768, replace=False))
    cols = np.unique(np.concatenate([cols, [0, 255, 256, lin.N - 1]]))
    ys = y[torch.from_numpy(rows)][:, torch.from_numpy(cols)].cpu()
    del y
    x_cpu, w_cpu = x.cpu(), w.cpu()
    del x
    W.free()
    del w
    torch.cuda.empty_cache()
    yr, pr = oracle_prefill_rows(x_cpu, w_cpu, rows, wrows=cols)
    assert_close(ys, yr, pr, f"llama70b {lin.name} {_L70.M}x{lin.N}x{lin.K}")
    assert mq.mq_check() == 0


def test_swiglu_llama70b_gate_up_sampled():
    """The 70B gate+up weight (N = 57344) through the fused SwiGLU epilogue:
    h on sampled rows within one BF16 ulp of SiLU(g) * u of the GPU's g, u,
    whose sampled columns are within the GEMM bound of the oracle, and the
    epilogue's partial maxima equal to max |h|."""
    lin = _L70.linears[2]
    M, K, I = _L70.M, lin.K, lin.N // 2
    x, w = _gpu_inputs_70b(2, K)
    W = mq.Weight(w)
    codes, sf, s = gpu_quantize(x)
    c, f = torch.from_numpy(codes).cuda(), torch.from_numpy(sf).cuda()
    sd = torch.tensor([s], dtype=torch.float32, device="cuda")
    gu = torch.empty(M, 2 * I, dtype=torch.bfloat16, device="cuda")
    mq.mq_gemm_nvfp4(c, f, sd, M, W.handle, gu, 2 * I)
    h = torch.empty(M, I, dtype=torch.bfloat16, device="cuda")
    part = torch.empty(mq.MQ_AMAX_PARTIALS_MAX, dtype=torch.float32, device="cuda")
    n = mq.mq_gemm_nvfp4_swiglu(c, f, sd, M, W.handle, h, part)
    torch.cuda.synchronize()
    assert float(part[:n].max()) == float(h.float().abs().max())
    rows = torch.from_numpy(sample_rows(M, 4, 40))
    gur, hr = gu[rows].cpu(), h[rows].cpu()
    check_h_from_gu(gur, hr, I, "llama70b swiglu")
    cols = np.sort(np.random.default_rng(41).choice(2 * I, 768, replace=False))
    x_cpu, w_cpu = x.cpu(), w.cpu()
    del gu, h, x
    W.free()
    del w
    torch.cuda.empty_cache()
    yr, pr = oracle_prefill_rows(x_cpu, w_cpu, rows.numpy(), wrows=cols)
    assert_close(gur[:, torch.from_numpy(cols)], yr, pr, "llama70b gate/up")
    assert mq.mq_check() == 0
