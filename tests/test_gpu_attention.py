"""GPU parity of the prefill layer's attention (tcgen05 tensor cores, writing
the BF16 KV cache and the O projection's amax partials) and of the decode
step's attention over that cache, against the oracle's binary64 attention.

Tolerance, per output element:
    |gpu - ref| <= 2^-8 (a + |ref|),  a = sum_j w_j |v_j| / sum_j w_j
(the oracle's softmax-weighted |v|).  The kernels round each weight to BF16
before the P.V product (2^-9 relative; the prefill divides by the sum of the
same rounded weights) and round o to BF16 (2^-9 |o|); FP32 accumulation of
128-term dot products and 2^x evaluation add far less.  The cache rows are
copies of the BF16 inputs and are compared bit for bit; the amax partials
must equal max |o| of the GPU's own o exactly."""
import numpy as np
import pytest
import torch

import oracle
from mqtest import ensure_built, sample_rows
from nvfp4_quantized_prefill_b200 import binding as mq

pytestmark = pytest.mark.gpu
D = 128


@pytest.fixture(scope="module", autouse=True)
def _built():
    ensure_built()


def _qkv(n, H, Hkv, seed, q_gain=1.0, device="cpu"):
    g = torch.Generator(device=device).manual_seed(seed)
    x = torch.randn(n, (H + 2 * Hkv) * D, generator=g, device=device)
    x[:, : H * D] *= q_gain
    return x.to(torch.bfloat16)


def _split(qkv, H, Hkv):
    return qkv[:, : H * D], qkv[:, H * D:(H + Hkv) * D], qkv[:, (H + Hkv) * D:]


def assert_attn_close(o_gpu, ref, a, what):
    og = o_gpu.float().double().cpu().numpy().reshape(ref.shape)
    bound = 2.0 ** -8 * (a + np.abs(ref))
    err = np.abs(og - ref)
    bad = err > bound
    if bad.any():
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(f"{what}: {int(bad.sum())}/{bad.size} outside the bound; worst at {i}: "
                             f"gpu {og[i]!r} ref {ref[i]!r} a {a[i]!r}")
    assert np.isfinite(og).all()


def _prefill(qkv_d, M, H, Hkv, S_max):
    kc = torch.zeros(Hkv, S_max, D, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    o = torch.empty(M, H * D, dtype=torch.bfloat16, device="cuda")
    part = torch.zeros(mq.MQ_AMAX_PARTIALS_MAX, dtype=torch.float32, device="cuda")
    n = mq.mq_attention_prefill_bf16(qkv_d, M, H, Hkv, D, kc, vc, S_max, o, part)
    torch.cuda.synchronize()
    return o, kc, vc, part, n


@pytest.mark.parametrize("M,H,Hkv,q_gain", [(1, 1, 1, 1.0), (77, 4, 2, 1.0), (128, 2, 1, 1.0),
                                             (300, 4, 2, 4.0), (513, 8, 2, 1.0), (640, 4, 4, 8.0)])
def test_prefill_attention_all_rows(M, H, Hkv, q_gain):
    """Ragged and whole 128-row tiles, grouped and ungrouped KV heads; larger
    query gains make the running maximum grow during a row (rescaled O)."""
    qkv = _qkv(M, H, Hkv, M + H, q_gain)
    S_max = M + 67
    o, kc, vc, part, n = _prefill(qkv.cuda(), M, H, Hkv, S_max)
    q, k, v = _split(qkv, H, Hkv)
    ref, a = oracle.attention(q, k, v, H, Hkv, D)
    assert_attn_close(o, ref, a, f"prefill attention M={M} H={H} Hkv={Hkv}")
    # the KV cache holds the keys / values of positions 0 .. M-1, bit for bit
    kh = k.view(M, Hkv, D).transpose(0, 1)
    vh = v.view(M, Hkv, D).transpose(0, 1)
    assert torch.equal(kc[:, :M].cpu().view(torch.int16), kh.contiguous().view(torch.int16))
    assert torch.equal(vc[:, :M].cpu().view(torch.int16), vh.contiguous().view(torch.int16))
    # the partial maxima: max |o| of the GPU's o, for the O projection's quantizer
    assert float(part[:n].max()) == float(o.float().abs().max())
    assert mq.mq_check() == 0


def test_prefill_attention_llama8b_shape_sampled_rows():
    """Llama-3-8B attention shape at 8192 tokens: 32 query heads over 8 KV
    heads, 64 query tiles; sampled rows (tile edges, the last row) against
    the oracle, every head."""
    M, H, Hkv = 8192, 32, 8
    qkv_d = _qkv(M, H, Hkv, 11, device="cuda")
    o, kc, vc, part, n = _prefill(qkv_d, M, H, Hkv, M)
    rows = sample_rows(M, 4, 12)
    qkv = qkv_d.cpu()
    q, k, v = _split(qkv, H, Hkv)
    ref, a = oracle.attention(q, k, v, H, Hkv, D, rows=rows)
    assert_attn_close(o[torch.from_numpy(rows)], ref, a, "llama8b prefill attention")
    assert torch.equal(kc[3].cpu(), k[:, 3 * D:4 * D])
    assert float(part[:n].max()) == float(o.float().abs().max())
    assert mq.mq_check() == 0


@pytest.mark.parametrize("S,m,H,Hkv", [(300, 1, 8, 2), (300, 4, 8, 2), (129, 8, 4, 1), (1, 16, 4, 4),
                                       (1000, 9, 8, 2), (200, 16, 8, 2), (4032, 64, 2, 2), (6000, 3, 16, 4)])
def test_decode_attention_after_prefill(S, m, H, Hkv):
    """Prefill S tokens into the cache, then decode m new tokens: each new
    token attends over the cached positions and the new ones up to itself --
    the prefill rows S .. S+m-1 of the whole sequence.  Query rows per KV
    head (group x m) from 1 to 64 (one to eight 8-row tiles of the decode
    kernel), caches ending inside a 64-key block and on its boundary
    (4032 + 64 = 4096), and spans of several blocks (6000 positions)."""
    S_max = S + m + 5
    qkv_all = _qkv(S + m, H, Hkv, 7 * S + m)
    _, kc, vc, _, _ = _prefill(qkv_all[:S].cuda().contiguous(), S, H, Hkv, S_max)
    qkv_t = qkv_all[S:].contiguous()
    o = torch.empty(m, H * D, dtype=torch.bfloat16, device="cuda")
    nb = mq.mq_attention_decode_workspace_bytes(m, S, H, Hkv, D)
    ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
    mq.mq_attention_decode_bf16(qkv_t.cuda(), m, S, H, Hkv, D, kc, vc, S_max, o, ws, nb)
    torch.cuda.synchronize()
    q, k, v = _split(qkv_all, H, Hkv)
    ref, a = oracle.attention(q[S:], k, v, H, Hkv, D, pos0=S)
    assert_attn_close(o, ref, a, f"decode attention S={S} m={m}")
    # the new tokens were appended to the cache
    kh = k.view(S + m, Hkv, D).transpose(0, 1)
    assert torch.equal(kc[:, :S + m].cpu().view(torch.int16), kh.contiguous().view(torch.int16))
    assert mq.mq_check() == 0


def test_decode_attention_llama8b_cache():
    """Decode after an 8192-token prefill at the Llama-3-8B attention shape:
    one token, then eight more, each step reading the cache the previous
    calls left."""
    S, H, Hkv = 8192, 32, 8
    S_max = S + 16
    qkv_all = _qkv(S + 9, H, Hkv, 21, device="cuda")
    _, kc, vc, _, _ = _prefill(qkv_all[:S].contiguous(), S, H, Hkv, S_max)
    outs = []
    for pos0, m in ((S, 1), (S + 1, 8)):
        o = torch.empty(m, H * D, dtype=torch.bfloat16, device="cuda")
        nb = mq.mq_attention_decode_workspace_bytes(m, pos0, H, Hkv, D)
        ws = torch.empty(nb, dtype=torch.uint8, device="cuda")
        mq.mq_attention_decode_bf16(qkv_all[pos0:pos0 + m].contiguous(), m, pos0, H, Hkv, D, kc, vc,
                                    S_max, o, ws, nb)
        outs.append(o)
    torch.cuda.synchronize()
    q, k, v = _split(qkv_all.cpu(), H, Hkv)
    ref, a = oracle.attention(q[S:], k, v, H, Hkv, D, pos0=S)
    assert_attn_close(torch.cat(outs), ref, a, "llama8b decode attention")
    assert mq.mq_check() == 0


def test_attention_arguments_rejected_on_the_host():
    x = torch.zeros(16, 6 * D, dtype=torch.bfloat16, device="cuda")
    o = torch.empty(16, 4 * D, dtype=torch.bfloat16, device="cuda")
    part = torch.empty(mq.MQ_AMAX_PARTIALS_MAX, dtype=torch.float32, device="cuda")
    with pytest.raises(mq.MqError) as e:
        mq.mq_attention_prefill_bf16(x, 16, 4, 1, 64, None, None, 0, o, part)   # D != 128
    assert e.value.code == 2
    with pytest.raises(mq.MqError) as e:
        mq.mq_attention_prefill_bf16(x, 16, 4, 3, D, None, None, 0, o, part)    # H % Hkv
    assert e.value.code == 2
    kc = torch.zeros(1, 8, D, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(mq.MqError) as e:
        mq.mq_attention_prefill_bf16(x, 16, 4, 1, D, kc, kc, 8, o, part)        # M > S_max
    assert e.value.code == 2
    assert mq.mq_check() == 0
