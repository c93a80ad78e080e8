"""The prefill layer's attention block end to end, then a decode step on the
same weights and the cache the prefill built -- Mix-Quant's phase hand-off:
NVFP4 projections in prefill, BF16 in decode, a BF16 KV cache between them.

Prefill: RMSNorm (emitting the quantizer's amax) -> NVFP4 QKV projection ->
attention (writing the cache and the amax of its output) -> NVFP4 O
projection quantized with that amax (no amax pass).  Decode: BF16 QKV
projection of a new token -> attention over the cache (appending it) -> BF16
O projection.  Each stage is compared with the oracle on the GPU's own input
to that stage (the chain convention used for SwiGLU's h): codes bit-exact,
linear outputs within the GEMM / decode bound, attention within its bound."""
import numpy as np
import pytest
import torch

import oracle
from mqtest import assert_close, ensure_built, oracle_prefill_rows, u16
from nvfp4_quantized_prefill_b200 import binding as mq
from nvfp4_quantized_prefill_b200 import workloads
from test_gpu_attention import assert_attn_close

pytestmark = pytest.mark.gpu
D = 128
EPS = 1e-5


@pytest.fixture(scope="module", autouse=True)
def _built():
    ensure_built()


@pytest.mark.parametrize("M,H,Hkv", [(300, 4, 2), (256, 8, 8)])
def test_prefill_attention_block_then_decode_step(M, H, Hkv):
    E = H * D                      # model width = query heads x head dim
    Nqkv = (H + 2 * Hkv) * D
    S_max = M + 4
    x = workloads.activation("outlier", M + 1, E, 40 + M, 0)      # M prefill rows + 1 decode token
    gamma = workloads.rmsnorm_gain(E, 40, 1)
    w_qkv = workloads.weight(Nqkv, E, 0.02, 40, 2)
    w_o = workloads.weight(E, E, 0.02, 40, 3)
    Wqkv, Wo = mq.Weight(w_qkv.cuda()), mq.Weight(w_o.cuda())

    # ---- prefill (NVFP4 projections)
    xd = x[:M].cuda().contiguous()
    xn = torch.empty(M, E, dtype=torch.bfloat16, device="cuda")
    qkv = torch.empty(M, Nqkv, dtype=torch.bfloat16, device="cuda")
    nb = mq.mq_workspace_bytes(M, E)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    mq.mq_prefill_linear_rmsnorm_nvfp4(Wqkv.handle, xd, gamma.cuda(), EPS, M, xn, qkv, ws, nb)
    kc = torch.zeros(Hkv, S_max, D, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    o = torch.empty(M, E, dtype=torch.bfloat16, device="cuda")
    part = torch.empty(mq.MQ_AMAX_PARTIALS_MAX, dtype=torch.float32, device="cuda")
    n = mq.mq_attention_prefill_bf16(qkv, M, H, Hkv, D, kc, vc, S_max, o, part)
    codes = torch.empty(M, E // 2, dtype=torch.uint8, device="cuda")
    sf = torch.empty(mq.mq_sf_bytes(M, E), dtype=torch.uint8, device="cuda")
    s = torch.empty(1, dtype=torch.float32, device="cuda")
    mq.mq_quantize_nvfp4(o, M, E, E, codes, sf, s, amax_partials=part, n_partials=n)
    y = torch.empty(M, E, dtype=torch.bfloat16, device="cuda")
    mq.mq_gemm_nvfp4(codes, sf, s, M, Wo.handle, y, E)
    torch.cuda.synchronize()

    # QKV projection of the GPU's normalised rows
    yr, pr = oracle_prefill_rows(xn.cpu(), w_qkv, np.arange(M))
    assert_close(qkv.cpu(), yr, pr, "layer qkv")
    # attention of the GPU's qkv
    qkv_c = qkv.cpu()
    qh, kh, vh = qkv_c[:, :E], qkv_c[:, E:E + Hkv * D], qkv_c[:, E + Hkv * D:]
    ar, aa = oracle.attention(qh, kh, vh, H, Hkv, D)
    assert_attn_close(o, ar, aa, "layer attention")
    # the O projection's quantization used the attention's amax: bit-exact
    rc, rsf, rs, _ = oracle.quantize_tensor(o.cpu())
    assert float(s.item()) == rs
    assert np.array_equal(codes.cpu().numpy(), rc)
    assert np.array_equal(sf.cpu().numpy(), oracle.sf_swizzle(rsf))
    yr, pr = oracle_prefill_rows(o.cpu(), w_o, np.arange(M))
    assert_close(y.cpu(), yr, pr, "layer o projection")

    # ---- decode step (BF16 projections) on the same handles and the cache
    xt = x[M:M + 1].cuda().contiguous()
    qkv_t = torch.empty(1, Nqkv, dtype=torch.bfloat16, device="cuda")
    mq.mq_decode_linear_bf16(Wqkv.handle, xt, 1, qkv_t)
    o_t = torch.empty(1, E, dtype=torch.bfloat16, device="cuda")
    nbd = mq.mq_attention_decode_workspace_bytes(1, M, H, Hkv, D)
    wsd = torch.empty(nbd, dtype=torch.uint8, device="cuda")
    mq.mq_attention_decode_bf16(qkv_t, 1, M, H, Hkv, D, kc, vc, S_max, o_t, wsd, nbd)
    y_t = torch.empty(1, E, dtype=torch.bfloat16, device="cuda")
    mq.mq_decode_linear_bf16(Wo.handle, o_t, 1, y_t)
    torch.cuda.synchronize()
    yr, pr = oracle.decode_linear(x[M:M + 1], w_qkv)
    assert_close(qkv_t.cpu(), yr, pr, "decode qkv")
    # the new token attends over the prefill's cached keys / values and its own
    qt_c = qkv_t.cpu()
    k_all = torch.cat([kh, qt_c[:, E:E + Hkv * D]])
    v_all = torch.cat([vh, qt_c[:, E + Hkv * D:]])
    ar, aa = oracle.attention(qt_c[:, :E], k_all, v_all, H, Hkv, D, pos0=M)
    assert_attn_close(o_t, ar, aa, "decode attention")
    yr, pr = oracle.decode_linear(o_t.cpu(), w_o)
    assert_close(y_t.cpu(), yr, pr, "decode o projection")
    Wqkv.free()
    Wo.free()
    assert mq.mq_check() == 0
