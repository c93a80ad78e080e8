"""Pins for the CPU oracle: each test checks the oracle against something other
than itself -- the closed-form values of the number formats, torch's own
(independent) float8 / bf16 conversions, the round-to-nearest-even tie points,
invariants the NVFP4 definition implies, special cases where quantization is
lossless, and brute force on tiny shapes.  CPU only.
"""
import math
import os

import numpy as np
import pytest
import torch

from nvfp4_quantized_prefill_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def dequantize(oracle_mod, codes: np.ndarray, sf: np.ndarray, s_enc: float) -> np.ndarray:
    """Real-valued NVFP4 matrix e2m1(code) * dec(scale) / s_enc in binary64,
    from the oracle's own decode tables (a test-side helper for the pins'
    brute-force references and error bounds)."""
    lut2 = np.array([oracle_mod.e2m1_decode(c) for c in range(16)], dtype=np.float64)
    lut8 = np.array([oracle_mod.e4m3_decode(b) for b in range(256)], dtype=np.float64)
    vals = np.empty((codes.shape[0], codes.shape[1] * 2), dtype=np.float64)
    vals[:, 0::2] = lut2[codes & 15]
    vals[:, 1::2] = lut2[codes >> 4]
    return vals * np.repeat(lut8[sf], 16, axis=1) / float(s_enc)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


# ---------------------------------------------------------------------------
# number formats
# ---------------------------------------------------------------------------

def test_e2m1_decode_all_16_codes(oracle_mod):
    # The eight E2M1 magnitudes are 0, 0.5, 1, 1.5, 2, 3, 4, 6 (codes 0..7);
    # bit 3 is the sign.
    mags = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    for c in range(16):
        v = oracle_mod.e2m1_decode(c)
        want = -mags[c & 7] if c & 8 else mags[c & 7]
        assert v == want and math.copysign(1.0, v) == (-1.0 if c & 8 else 1.0), c


def test_e4m3_decode_matches_torch_all_256(oracle_mod):
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64)
    for b in range(256):
        v = oracle_mod.e4m3_decode(b)
        r = float(ref[b])
        if math.isnan(r):
            assert math.isnan(v), b
        else:
            assert v == r and math.copysign(1, v) == math.copysign(1, r), b
    assert oracle_mod.e4m3_decode(0x7E) == 448.0
    assert oracle_mod.e4m3_decode(0x01) == 2.0 ** -9       # smallest subnormal
    assert oracle_mod.e4m3_decode(0x08) == 2.0 ** -6       # smallest normal
    assert math.isnan(oracle_mod.e4m3_decode(0x7F)) and math.isnan(oracle_mod.e4m3_decode(0xFF))


def test_bf16_conversions_match_torch(oracle_mod):
    g = torch.Generator().manual_seed(5)
    f = torch.randn(4000, generator=g) * torch.exp(torch.randn(4000, generator=g) * 8)
    # exact ties: a bf16 value plus half an ulp
    base = torch.randn(500, generator=g).to(torch.bfloat16)
    bits = base.view(torch.int16).to(torch.int32) & 0xFFFF
    tie = ((bits << 16) | 0x8000).to(torch.int32).view(torch.float32)
    f = torch.cat([f, tie, torch.tensor([0.0, -0.0, 1e-40, -3e38])])
    want = bf16_bits(f.to(torch.bfloat16))
    for i in range(f.numel()):
        assert oracle_mod.float_to_bf16(float(f[i])) == int(want[i]), float(f[i])
    for b in [0, 0x8000, 0x3F80, 0xBF80, 0x7F7F, 0x0001, 0x4049]:
        t = torch.tensor([b], dtype=torch.int32).to(torch.int16).view(torch.bfloat16)
        assert oracle_mod.bf16_to_float(b) == float(t.float())


def test_e4m3_encode_roundtrip_and_torch_rne(oracle_mod):
    for b in range(0x7F):
        assert oracle_mod.e4m3_encode(oracle_mod.e4m3_decode(b)) == b, b
    # torch's cast is an independent RNE implementation (it overflows to NaN
    # beyond 464, so only in-range values are compared against it)
    g = torch.Generator().manual_seed(1)
    vals = [float(v) for v in torch.rand(3000, generator=g) * 460.0]
    vals += [float(v) for v in torch.exp(torch.rand(3000, generator=g) * -18.0) * 2.0]
    for b in range(0x7E):                              # exact midpoints
        lo, hi = oracle_mod.e4m3_decode(b), oracle_mod.e4m3_decode(b + 1)
        vals.append((lo + hi) / 2)
    vals += [2.0 ** -10, 2.0 ** -10 * (1 + 2 ** -20), 0.0]
    ref = torch.tensor(vals, dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8)
    for v, r in zip(vals, ref.tolist()):
        assert oracle_mod.e4m3_encode(v) == r, v


def test_e4m3_encode_saturates(oracle_mod):
    for v in [448.0, 449.0, 463.9, 464.0, 480.0, 1000.0, 1e30, 3.4e38]:
        assert oracle_mod.e4m3_encode(v) == 0x7E, v
    assert oracle_mod.e4m3_encode(2.0 ** -10) == 0x00        # tie to even (0)
    assert oracle_mod.e4m3_encode(3 * 2.0 ** -10) == 0x02    # tie 1.5 ulp -> even 2


def test_e2m1_encode_ties_and_saturation(oracle_mod):
    mags = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    for c, m in enumerate(mags):
        assert oracle_mod.e2m1_encode(m) == c
        if m:
            assert oracle_mod.e2m1_encode(-m) == 8 | c
    # midpoints round to the even code
    ties = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6}
    for v, c in ties.items():
        assert oracle_mod.e2m1_encode(v) == c, v
        assert oracle_mod.e2m1_encode(-v) == 8 | c, -v
        up = float(np.nextafter(np.float32(v), np.float32(10)))
        dn = float(np.nextafter(np.float32(v), np.float32(0)))
        mid_hi = [m for m in mags if m > v][0]
        mid_lo = [m for m in mags if m < v][-1]
        assert oracle_mod.e2m1_encode(up) == mags.index(mid_hi), up
        assert oracle_mod.e2m1_encode(dn) == mags.index(mid_lo), dn
    for v in [6.0001, 7.0, 100.0, 3e38]:
        assert oracle_mod.e2m1_encode(v) == 7
        assert oracle_mod.e2m1_encode(-v) == 15
    assert oracle_mod.e2m1_encode(-0.0) == 8     # signed zero keeps its sign
    assert oracle_mod.e2m1_encode(-0.1) == 8
    assert oracle_mod.e2m1_encode(0.1) == 0


# ---------------------------------------------------------------------------
# tensor scale and quantization
# ---------------------------------------------------------------------------

def test_tensor_scale(oracle_mod):
    assert oracle_mod.tensor_scale(2688.0) == 1.0
    assert oracle_mod.tensor_scale(6.0) == 448.0
    assert oracle_mod.tensor_scale(0.0) == 1.0
    assert oracle_mod.tensor_scale(1e-45) == 1.0          # quotient overflows
    assert oracle_mod.tensor_scale(3.0) == np.float32(2688.0) / np.float32(3.0)


def _quant_case(oracle_mod, M, K, seed, kind="outlier"):
    x = workloads.activation(kind, M, K, seed, 0)
    codes, sf, s, amax = oracle_mod.quantize_tensor(x)
    return x, codes, sf, s, amax


def test_tensor_amax_is_max_abs(oracle_mod):
    x = workloads.activation("outlier", 37, 96, 3, 0)
    assert oracle_mod.tensor_amax(x) == float(x.float().abs().max())


@pytest.mark.parametrize("kind", workloads.ACT_KINDS)
def test_quantize_invariants(oracle_mod, kind):
    M, K = 64, 256
    x, codes, sf, s, amax = _quant_case(oracle_mod, M, K, 11, kind)
    xf = x.float().numpy().astype(np.float64)
    xb = np.abs(xf).reshape(M, K // 16, 16)
    # (1) the block holding the tensor amax gets the largest block scale
    r, c = np.unravel_index(np.argmax(np.abs(xf)), xf.shape)
    assert sf[r, c // 16] == 0x7E
    # (2) in blocks with a normal scale the max-|x| element maps to |code| 7
    nib = np.empty((M, K), dtype=np.int64)
    nib[:, 0::2] = codes & 15
    nib[:, 1::2] = codes >> 4
    for rr in range(M):
        for b in range(K // 16):
            if sf[rr, b] >= 0x08:
                j = b * 16 + int(np.argmax(xb[rr, b]))
                assert nib[rr, j] & 7 == 7, (rr, b)
    # (3) sign bit of every code is the sign bit of x
    sign_x = np.signbit(xf)
    assert np.array_equal((nib >> 3).astype(bool), sign_x)
    # (4) round-to-nearest: dequantization error <= half the local E2M1 spacing
    deq = dequantize(oracle_mod, codes, sf, s)
    lut8 = np.array([oracle_mod.e4m3_decode(b) for b in range(256)])
    unit = np.repeat(lut8[sf], 16, axis=1) / s           # dec(sb) / s_enc
    mag = np.abs(deq) / np.where(unit > 0, unit, 1)
    half = np.where(mag < 2, 0.25, np.where(mag < 4, 0.5, 1.0))
    sat = (np.abs(deq) > 0) & (mag >= 6) & (np.abs(xf) > np.abs(deq))
    err = np.abs(xf - deq)
    ok = (err <= half * unit * (1 + 1e-5)) | sat | (unit == 0)
    assert ok.all()


def test_quantize_scale_invariance(oracle_mod):
    # multiplying the whole tensor by 2^k (exact in bf16) changes nothing
    x = workloads.activation("outlier", 32, 128, 4, 0)
    c0, s0, _, _ = oracle_mod.quantize_tensor(x)
    for k in (-3, 5):
        c1, s1, _, _ = oracle_mod.quantize_tensor((x.float() * 2.0 ** k).to(torch.bfloat16))
        assert np.array_equal(c0, c1) and np.array_equal(s0, s1)


def test_quantize_rows_and_blocks_independent(oracle_mod):
    # with a fixed tensor scale, each 16-block depends only on its own values
    x = workloads.activation("outlier", 24, 128, 6, 0)
    s = oracle_mod.tensor_scale(oracle_mod.tensor_amax(x))
    c0, f0 = oracle_mod.quantize(x, s)
    perm = torch.randperm(24, generator=torch.Generator().manual_seed(0))
    c1, f1 = oracle_mod.quantize(x[perm].contiguous(), s)
    assert np.array_equal(c1, c0[perm.numpy()]) and np.array_equal(f1, f0[perm.numpy()])
    x2 = x.clone()
    x2[5, 32:48] = x2[5, 32:48] * 3
    c2, f2 = oracle_mod.quantize(x2, s)
    diff_c = np.argwhere(c2 != c0)
    diff_f = np.argwhere(f2 != f0)
    assert all(r == 5 and 16 <= col < 24 for r, col in diff_c)
    assert all(r == 5 and col == 2 for r, col in diff_f)


def _lossless_matrix(rows, K, seed, k_lo=-4, k_hi=2):
    """BF16 matrix whose 16-blocks hold e2m1 * 2^kb with block max 6 * 2^kb and
    whose tensor max is 6 * 2^k_hi: NVFP4 quantization is exact for it."""
    rng = np.random.default_rng(seed)
    mags = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    v = mags[rng.integers(0, 8, size=(rows, K))] * rng.choice([-1.0, 1.0], size=(rows, K))
    kb = rng.integers(k_lo, k_hi + 1, size=(rows, K // 16))
    kb[0, 0] = k_hi                    # the block that holds the tensor max
    v = v.reshape(rows, K // 16, 16)
    v[:, :, 0] = 6.0 * rng.choice([-1.0, 1.0], size=(rows, K // 16))
    v = v * (2.0 ** kb)[:, :, None]
    v = v.reshape(rows, K)
    v[0, 0] = abs(v[0, 0])
    return torch.tensor(v, dtype=torch.float32).to(torch.bfloat16), v


def test_quantize_lossless_special_case(oracle_mod):
    x, v = _lossless_matrix(16, 128, 2)
    codes, sf, s, amax = oracle_mod.quantize_tensor(x)
    assert amax == 24.0 and s == np.float32(112.0)
    deq = dequantize(oracle_mod, codes, sf, s)
    assert np.array_equal(deq, v)


# ---------------------------------------------------------------------------
# scale-factor layout
# ---------------------------------------------------------------------------

def test_sf_layout_golden_offsets(oracle_mod):
    with open(os.path.join(GOLDEN, "sf_layout_offsets.txt")) as fh:
        rows = [l.split() for l in fh if l.strip() and not l.startswith("#")]
    assert len(rows) >= 10
    for rr, kb, r, c, off in rows:
        assert oracle_mod.sf_swizzled_offset(int(r), int(c), int(kb)) == int(off), (r, c, kb)


@pytest.mark.parametrize("rows,kb", [(128, 4), (200, 12), (1, 1), (300, 17)])
def test_sf_swizzle_is_padded_permutation(oracle_mod, rows, kb):
    rng = np.random.default_rng(rows + kb)
    sf = rng.integers(1, 256, size=(rows, kb), dtype=np.uint8)
    swz = oracle_mod.sf_swizzle(sf)
    assert swz.size == ((rows + 127) // 128 * 128) * ((kb + 3) // 4 * 4)
    assert np.array_equal(oracle_mod.sf_unswizzle(swz, rows, kb), sf)
    # every real scale lands on a distinct byte; all other bytes are padding 0
    offs = {oracle_mod.sf_swizzled_offset(r, c, kb) for r in range(rows) for c in range(kb)}
    assert len(offs) == rows * kb
    pad = np.ones(swz.size, dtype=bool)
    pad[list(offs)] = False
    assert (swz[pad] == 0).all()


# ---------------------------------------------------------------------------
# GEMM, decode, SwiGLU
# ---------------------------------------------------------------------------

def test_gemm_bruteforce_tiny(oracle_mod):
    for (M, N, K, seed) in [(3, 5, 32, 0), (8, 8, 64, 1), (1, 7, 16, 2), (6, 2, 48, 3)]:
        a = workloads.activation("outlier", M, K, seed, 0)
        b = workloads.weight(N, K, 0.02, seed, 1)
        ac, af, asn, _ = oracle_mod.quantize_tensor(a)
        bc, bf, bsn, _ = oracle_mod.quantize_tensor(b)
        y, p = oracle_mod.gemm_nvfp4(ac, af, asn, bc, bf, bsn)
        # naive binary64 sum of the dequantized values, term by term
        lut2 = [oracle_mod.e2m1_decode(c) for c in range(16)]
        lut8 = [oracle_mod.e4m3_decode(q) for q in range(256)]
        for m in range(M):
            for n in range(N):
                s = 0.0
                sa = 0.0
                for k in range(K):
                    qa = (ac[m, k // 2] >> (4 * (k & 1))) & 15
                    qb = (bc[n, k // 2] >> (4 * (k & 1))) & 15
                    t = lut2[qa] * lut8[af[m, k // 16]] * lut2[qb] * lut8[bf[n, k // 16]]
                    s += t
                    sa += abs(t)
                alpha = 1.0 / (float(np.float32(asn)) * float(np.float32(bsn)))
                assert y[m, n] == alpha * s, (m, n)
                assert p[m, n] == alpha * sa


def test_gemm_lossless_equals_exact_matmul(oracle_mod):
    a, av = _lossless_matrix(9, 256, 10)
    b, bv = _lossless_matrix(20, 256, 11, k_lo=-6, k_hi=0)
    ac, af, asn, _ = oracle_mod.quantize_tensor(a)
    bc, bf, bsn, _ = oracle_mod.quantize_tensor(b)
    y, p = oracle_mod.gemm_nvfp4(ac, af, asn, bc, bf, bsn)
    exact = av @ bv.T          # every term is a small dyadic rational: exact
    # the oracle rounds twice in binary64 (alpha = 1/(s_a*s_b), then alpha*S);
    # the smallest term here is ~2^-12, far above that rounding
    assert (np.abs(y - exact) <= 2.0 ** -51 * np.abs(exact)).all()
    pe = np.abs(av) @ np.abs(bv).T
    assert (np.abs(p - pe) <= 2.0 ** -51 * pe).all()


def test_gemm_operand_swap_and_row_sampling(oracle_mod):
    a = workloads.activation("outlier", 12, 128, 21, 0)
    b = workloads.weight(10, 128, 0.02, 21, 1)
    ac, af, asn, _ = oracle_mod.quantize_tensor(a)
    bc, bf, bsn, _ = oracle_mod.quantize_tensor(b)
    y, _ = oracle_mod.gemm_nvfp4(ac, af, asn, bc, bf, bsn)
    yt, _ = oracle_mod.gemm_nvfp4(bc, bf, bsn, ac, af, asn)
    assert np.array_equal(y, yt.T)
    rows = np.array([11, 0, 5], dtype=np.int64)
    ys, _ = oracle_mod.gemm_nvfp4(ac, af, asn, bc, bf, bsn, rows=rows)
    assert np.array_equal(ys, y[rows])


def test_gemm_close_to_bf16_matmul(oracle_mod):
    # sanity: NVFP4 W4A4 approximates the real product (relative Frobenius
    # error of a few percent for Gaussian data)
    a = workloads.activation("outlier", 32, 512, 7, 0)
    b = workloads.weight(48, 512, 0.02, 7, 1)
    ac, af, asn, _ = oracle_mod.quantize_tensor(a)
    bc, bf, bsn, _ = oracle_mod.quantize_tensor(b)
    y, p = oracle_mod.gemm_nvfp4(ac, af, asn, bc, bf, bsn)
    ref = a.double().numpy() @ b.double().numpy().T
    rel = np.linalg.norm(y - ref) / np.linalg.norm(ref)
    assert 0.01 < rel < 0.25, rel
    assert (p >= np.abs(y)).all()


def test_decode_linear_matches_numpy(oracle_mod):
    x = workloads.activation("outlier", 3, 320, 8, 0)
    w = workloads.weight(17, 320, 0.02, 8, 1)
    y, p = oracle_mod.decode_linear(x, w)
    ref = x.double().numpy() @ w.double().numpy().T
    assert np.allclose(y, ref, rtol=1e-13, atol=1e-15)
    assert np.allclose(p, np.abs(x.double().numpy()) @ np.abs(w.double().numpy()).T, rtol=1e-13)


def test_swiglu_against_torch_silu(oracle_mod):
    g = workloads.activation("outlier", 64, 64, 9, 0)
    u = workloads.activation("outlier", 64, 64, 9, 1)
    h = oracle_mod.swiglu(g, u)
    ref = bf16_bits((torch.nn.functional.silu(g.float()) * u.float()).to(torch.bfloat16))
    # torch computes SiLU its own way: allow at most one bf16 ulp
    hb = torch.from_numpy(h.view(np.int16)).view(torch.bfloat16).float()
    rb = torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16).float()
    ulp = torch.where(rb == 0, torch.full_like(rb, 1e-38), rb.abs() * 2.0 ** -7)
    assert ((hb - rb).abs() <= ulp).all()
    assert (h == ref).mean() > 0.99
    # special cases
    z = torch.zeros(1, 8, dtype=torch.bfloat16)
    one = torch.ones(1, 8, dtype=torch.bfloat16)
    assert (oracle_mod.swiglu(z, one) == 0).all()
    big = torch.full((1, 8), 30.0, dtype=torch.bfloat16)
    assert (oracle_mod.swiglu(big, one) == bf16_bits(big)).all()   # SiLU(30) ~ 30


# ---- RMSNorm in front of a prefill linear (reading: Llama-family RMSNorm) ----

def test_double_to_bf16_matches_torch(oracle_mod):
    rng = np.random.default_rng(11)
    vals = np.concatenate([rng.standard_normal(2000) * 10.0 ** rng.integers(-30, 30, 2000),
                           [0.0, -0.0, 1.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -9, 2.0 ** -133,
                            2.0 ** -134 * 3, 3.0e38, -1.5e-40]])
    got = np.array([oracle_mod.double_to_bf16(v) for v in vals], dtype=np.uint16)
    ref = bf16_bits(torch.tensor(vals, dtype=torch.float64).to(torch.bfloat16))
    assert (got == ref).all()


def test_rmsnorm_closed_forms(oracle_mod):
    K = 64
    # constant rows: x / |x| exactly (eps = 0), with gain 1
    cs = [3.0, -0.75, 1e-3, -250.0, 2.0 ** -20]
    x = torch.tensor([[c] * K for c in cs], dtype=torch.bfloat16)
    one = torch.ones(K, dtype=torch.bfloat16)
    y = oracle_mod.rmsnorm(x, one, 0.0)
    exp = bf16_bits(torch.tensor([[math.copysign(1.0, c)] * K for c in cs], dtype=torch.bfloat16))
    assert (y == exp).all()
    # one-hot rows of length 4: x_j / sqrt(x_j^2 / 4) = 2 sign(x_j); gain scales it
    x4 = torch.zeros(3, 4, dtype=torch.bfloat16)
    x4[0, 1] = 5.0
    x4[1, 3] = -0.125
    x4[2, 0] = 77.0
    g4 = torch.tensor([0.5, -1.5, 3.0, 0.25], dtype=torch.bfloat16)
    y4 = torch.from_numpy(oracle_mod.rmsnorm(x4, g4, 0.0).view(np.int16)).view(torch.bfloat16).float()
    exp4 = torch.zeros(3, 4)
    exp4[0, 1] = 2.0 * -1.5
    exp4[1, 3] = -2.0 * 0.25
    exp4[2, 0] = 2.0 * 0.5
    assert torch.equal(y4, exp4)
    # an all-zero row stays zero
    z = oracle_mod.rmsnorm(torch.zeros(1, K, dtype=torch.bfloat16), one, 1e-5)
    assert (z & 0x7FFF == 0).all()


def test_rmsnorm_scale_invariance(oracle_mod):
    x = workloads.activation("channel_gain", 16, 256, 12, 0)
    g = workloads.activation("outlier", 1, 256, 12, 1)[0]
    y = oracle_mod.rmsnorm(x, g, 0.0)
    for k in (-3, 5):
        assert (oracle_mod.rmsnorm((x.float() * 2.0 ** k).to(torch.bfloat16), g, 0.0) == y).all()


def test_rmsnorm_matches_torch_library(oracle_mod):
    """Unit gain: the normalised row is torch's binary64 rms_norm rounded to BF16."""
    x = workloads.activation("student_t3", 32, 512, 13, 0)
    one = torch.ones(512, dtype=torch.bfloat16)
    y = oracle_mod.rmsnorm(x, one, 1e-5)
    ref = torch.nn.functional.rms_norm(x.double(), (512,), eps=1e-5).to(torch.bfloat16)
    assert (y == bf16_bits(ref)).all()


# ---------------------------------------------------------------------------
# attention (prefill layer and decode step)
# ---------------------------------------------------------------------------

def _qkv(n, H, Hkv, D, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(n, H * D, generator=g).to(torch.bfloat16)
    k = torch.randn(n, Hkv * D, generator=g).to(torch.bfloat16)
    v = torch.randn(n, Hkv * D, generator=g).to(torch.bfloat16)
    return q, k, v


def test_attention_first_query_sees_only_the_first_key(oracle_mod):
    q, k, v = _qkv(6, 4, 2, 16, 1)
    o, a = oracle_mod.attention(q, k, v, 4, 2, 16)
    vv = v.double().numpy().reshape(6, 2, 16)
    for h in range(4):
        assert np.array_equal(o[0, h], vv[0, h // 2])       # one visible key: exactly v_0
        assert np.array_equal(a[0, h], np.abs(vv[0, h // 2]))


def test_attention_zero_queries_give_running_means(oracle_mod):
    """q = 0: every visible key weighs the same, o_i = mean(v_0 .. v_i)."""
    n, H, Hkv, D = 9, 4, 2, 8
    _, k, v = _qkv(n, H, Hkv, D, 2)
    q = torch.zeros(n, H * D, dtype=torch.bfloat16)
    o, _ = oracle_mod.attention(q, k, v, H, Hkv, D)
    vv = v.double().numpy().reshape(n, Hkv, D)
    mean = np.cumsum(vv, axis=0) / np.arange(1, n + 1)[:, None, None]
    for h in range(H):
        assert np.allclose(o[:, h], mean[:, h // 2], rtol=0, atol=1e-14)


def test_attention_dominant_key_selects_its_value(oracle_mod):
    """k_j = c e_j and q_i = c e_t: key t out-scores every other by c^2/sqrt(D)
    (= 64 here), so o_i = v_t up to e^-64."""
    n, D, c = 8, 16, 16.0
    k = torch.zeros(n, D)
    for j in range(n):
        k[j, j] = c
    q = torch.zeros(n, D)
    t = 3
    q[:, t] = c
    v = torch.randn(n, D, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
    o, _ = oracle_mod.attention(q.to(torch.bfloat16), k.to(torch.bfloat16), v, 1, 1, D)
    vv = v.double().numpy()
    for i in range(t, n):
        assert np.allclose(o[i, 0], vv[t], rtol=0, atol=1e-20 + 1e-25)
    # before key t is visible the queries score 0 against every key: uniform
    for i in range(t):
        assert np.allclose(o[i, 0], vv[: i + 1].mean(axis=0), rtol=0, atol=1e-14)


def test_attention_query_heads_read_their_groups_kv_head(oracle_mod):
    """H = 4 query heads over Hkv = 2 KV heads: heads 0-1 read KV head 0 and
    heads 2-3 KV head 1 (a mapping like h % Hkv would mix them)."""
    n, H, Hkv, D = 5, 4, 2, 8
    q, k, _ = _qkv(n, H, Hkv, D, 4)
    v = torch.cat([torch.full((n, D), 1.0), torch.full((n, D), 2.0)], dim=1).to(torch.bfloat16)
    o, a = oracle_mod.attention(q, k, v, H, Hkv, D)
    assert np.all(o[:, 0:2] == 1.0) and np.all(o[:, 2:4] == 2.0)
    assert np.array_equal(a, o)                 # v >= 0: the weighted |v| is o itself


def test_attention_matches_torch_sdpa_in_binary64(oracle_mod):
    n, H, Hkv, D = 37, 8, 2, 32
    q, k, v = _qkv(n, H, Hkv, D, 5)
    o, a = oracle_mod.attention(q, k, v, H, Hkv, D)
    qt = q.double().view(n, H, D).transpose(0, 1)
    kt = k.double().view(n, Hkv, D).transpose(0, 1).repeat_interleave(H // Hkv, dim=0)
    vt = v.double().view(n, Hkv, D).transpose(0, 1).repeat_interleave(H // Hkv, dim=0)
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True)
    ref = ref.transpose(0, 1).numpy()
    assert np.allclose(o, ref, rtol=1e-12, atol=1e-14)
    assert np.all(a >= np.abs(o) - 1e-15)


def test_attention_decode_rows_equal_prefill_rows(oracle_mod):
    """New queries at positions S.. over a cache holding keys 0..S+t are the
    prefill's rows S.. of the concatenated sequence (the phase hand-off)."""
    n, S, H, Hkv, D = 20, 15, 4, 1, 16
    q, k, v = _qkv(n, H, Hkv, D, 6)
    full, _ = oracle_mod.attention(q, k, v, H, Hkv, D)
    dec, _ = oracle_mod.attention(q[S:], k, v, H, Hkv, D, pos0=S)
    assert np.array_equal(dec, full[S:])
    some, _ = oracle_mod.attention(q, k, v, H, Hkv, D, rows=[0, 7, 19])
    assert np.array_equal(some, full[[0, 7, 19]])
