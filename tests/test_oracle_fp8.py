"""Pins of the oracle's FP8 (E4M3 and E5M2) KV-cache arithmetic against facts
fixed outside it: the formats' definitions (E4M3: bias 7, 3 fraction bits,
NaN code, largest finite 448; E5M2: bias 15, 2 fraction bits, infinities
and NaNs, largest finite 57344), torch's own float8_e4m3fn / float8_e5m2
conversions (library routines), round-to-nearest-even at exact midpoints,
and exact identities of attention under a per-tensor scale.

The 8-bit cache stores one code per K/V element and one binary32 scale for
all of K and one for all of V ("fp8_e4m3" KV cache of the serving
configurations in "上下文窗口优化实战：如何用PagedAttention+FlashInfer将Llama3-70B的
128K上下文吞吐提升3.8倍？" section 4.1); element value = code value * scale.
"""
import numpy as np
import pytest
import torch

import oracle
from paged_kv_cache_479_b200 import workloads as wl

from test_oracle_pins import sdpa_reference, to_bits, widen

E4M3_MAX = 448.0


E5M2_MAX = 57344.0
TORCH_FP8 = {"e4m3": torch.float8_e4m3fn, "e5m2": torch.float8_e5m2}


def torch_values(codes, fmt="e4m3"):
    return torch.from_numpy(np.asarray(codes, np.uint8)).view(TORCH_FP8[fmt]).double().numpy()


def torch_encode(x, fmt="e4m3"):
    return torch.from_numpy(np.asarray(x, np.float32)).to(TORCH_FP8[fmt]).view(torch.uint8).numpy()


def test_code_values_from_the_format_definition():
    v = oracle.e4m3_values(np.arange(256, dtype=np.uint8))
    # hand-derived values
    assert v[0x00] == 0.0 and not np.signbit(v[0x00])
    assert v[0x80] == 0.0 and np.signbit(v[0x80])
    assert v[0x01] == 2.0 ** -9                 # smallest subnormal
    assert v[0x07] == 7 * 2.0 ** -9             # largest subnormal
    assert v[0x08] == 2.0 ** -6                 # smallest normal
    assert v[0x38] == 1.0                       # exponent field 7 = bias
    assert v[0x3c] == 1.5
    assert v[0x40] == 2.0
    assert v[0x7e] == E4M3_MAX                  # 1.75 * 2^8
    assert v[0xfe] == -E4M3_MAX
    assert v[0x77] == 240.0 and v[0x78] == 256.0
    assert np.isnan(v[0x7f]) and np.isnan(v[0xff])
    assert np.isfinite(v).sum() == 254          # no infinities
    # sign symmetry and monotone magnitudes
    np.testing.assert_array_equal(v[0x80:0xff], -v[0x00:0x7f])
    assert np.all(np.diff(v[0x00:0x7f]) > 0)
    # the library's reading of every code
    t = torch_values(np.arange(256))
    same = (v == t) | (np.isnan(v) & np.isnan(t))
    assert same.all()


def test_encode_matches_torch_round_to_nearest_even():
    rng = np.random.default_rng(11)
    n = 60000
    x = (rng.standard_normal(n) * np.exp(rng.uniform(-13, 6.5, n))).astype(np.float32)
    x = x[np.abs(x) < 464]                       # torch gives NaN from 480 up
    np.testing.assert_array_equal(oracle.e4m3_encode(x), torch_encode(x))
    # every exact midpoint between neighbouring finite codes: ties go to the even code
    v = oracle.e4m3_values(np.arange(0x7f, dtype=np.uint8))
    mids = ((v[:-1] + v[1:]) / 2).astype(np.float32)
    assert np.array_equal(mids.astype(np.float64), (v[:-1] + v[1:]) / 2)   # exact in binary32
    got = oracle.e4m3_encode(mids)
    lo = np.arange(0x7e, dtype=np.uint8)
    expect = np.where(lo % 2 == 0, lo, lo + 1).astype(np.uint8)
    np.testing.assert_array_equal(got, expect)
    np.testing.assert_array_equal(oracle.e4m3_encode(-mids), expect | 0x80)
    np.testing.assert_array_equal(got, torch_encode(mids))
    # every finite code round-trips
    np.testing.assert_array_equal(oracle.e4m3_encode(v.astype(np.float32)), np.arange(0x7f))


def test_e5m2_code_values_from_the_format_definition():
    v = oracle.fp8_values(np.arange(256, dtype=np.uint8), "e5m2")
    assert v[0x00] == 0.0 and np.signbit(v[0x80])
    assert v[0x01] == 2.0 ** -16 and v[0x03] == 3 * 2.0 ** -16   # subnormals
    assert v[0x04] == 2.0 ** -14                                  # smallest normal
    assert v[0x3c] == 1.0 and v[0x3e] == 1.5 and v[0x40] == 2.0   # exponent field 15 = bias
    assert v[0x7b] == E5M2_MAX and v[0xfb] == -E5M2_MAX
    assert v[0x7c] == np.inf and v[0xfc] == -np.inf
    assert np.isnan(v[[0x7d, 0x7e, 0x7f, 0xfd, 0xfe, 0xff]]).all()
    np.testing.assert_array_equal(v[0x80:0xfc], -v[0x00:0x7c])
    assert np.all(np.diff(v[0x00:0x7d]) > 0)
    # the top byte of an IEEE half: widening is a shift
    half = torch.from_numpy((np.arange(256, dtype=np.int32) << 8).astype(np.int16)).view(torch.float16)
    same = (v == half.double().numpy()) | (np.isnan(v) & torch.isnan(half).numpy())
    assert same.all()
    t = torch_values(np.arange(256), "e5m2")
    assert ((v == t) | (np.isnan(v) & np.isnan(t))).all()


def test_e5m2_encode_matches_torch_and_saturates():
    rng = np.random.default_rng(13)
    n = 60000
    x = (rng.standard_normal(n) * np.exp(rng.uniform(-18, 11, n))).astype(np.float32)
    x = x[np.abs(x) < E5M2_MAX]                  # torch overflows to inf past 61440
    np.testing.assert_array_equal(oracle.fp8_encode(x, 1.0, "e5m2"), torch_encode(x, "e5m2"))
    v = oracle.fp8_values(np.arange(0x7c, dtype=np.uint8), "e5m2")
    mids = ((v[:-1] + v[1:]) / 2).astype(np.float32)
    lo = np.arange(0x7b, dtype=np.uint8)
    expect = np.where(lo % 2 == 0, lo, lo + 1).astype(np.uint8)
    np.testing.assert_array_equal(oracle.fp8_encode(mids, 1.0, "e5m2"), expect)
    np.testing.assert_array_equal(oracle.fp8_encode(v.astype(np.float32), 1.0, "e5m2"),
                                  np.arange(0x7c))
    big = np.array([57344, 61439, 61440, 1e9, np.inf, -7e4, -np.inf, np.nan], np.float32)
    np.testing.assert_array_equal(oracle.fp8_encode(big, 1.0, "e5m2"),
                                  [0x7b, 0x7b, 0x7b, 0x7b, 0x7b, 0xfb, 0xfb, 0x7f])
    s32 = np.float32(0.37)
    np.testing.assert_array_equal(oracle.fp8_encode(x[:5000], s32, "e5m2"),
                                  oracle.fp8_encode((x[:5000] / s32).astype(np.float32), 1.0, "e5m2"))


def test_encode_saturates_and_keeps_nan():
    x = np.array([448, 463.9, 464, 480, 1e6, np.inf, -500, -np.inf, np.nan], np.float32)
    c = oracle.e4m3_encode(x)
    np.testing.assert_array_equal(c[:6], 0x7e)
    np.testing.assert_array_equal(c[6:8], 0xfe)
    assert c[8] == 0x7f
    # below the smallest subnormal's half: zero with the sign kept
    tiny = np.array([2.0 ** -11, -2.0 ** -11, 2.0 ** -10, 2.0 ** -10 * 1.01], np.float32)
    np.testing.assert_array_equal(oracle.e4m3_encode(tiny), [0x00, 0x80, 0x00, 0x01])


def test_encode_divides_by_the_scale_in_binary32():
    rng = np.random.default_rng(12)
    x = rng.standard_normal(5000).astype(np.float32) * 3
    for s in (0.5, 2.0, 0.0234375, 1 / 3):
        s32 = np.float32(s)
        q = (x / s32).astype(np.float32)
        np.testing.assert_array_equal(oracle.e4m3_encode(x, s32), oracle.e4m3_encode(q))
        keep = np.abs(q) < 464                   # torch gives NaN from 480 up
        np.testing.assert_array_equal(oracle.e4m3_encode(x, s32)[keep], torch_encode(q[keep]))
    with pytest.raises(oracle.OracleError):
        oracle.e4m3_encode(x, 0.0)
    with pytest.raises(oracle.OracleError):
        oracle.e4m3_encode(x, -1.0)


# ---------------------------------------------------------------------------
# attention over an 8-bit pool
# ---------------------------------------------------------------------------

def fp8_case(lens, hq, hkv, ps, seed, q_dtype="bf16", pool_factor=1.5, fmt="e4m3"):
    w = wl.make_workload("fp8pin", lens, num_qo_heads=hq, num_kv_heads=hkv, page_size=ps,
                         dtype=q_dtype, seed=seed, pool_factor=pool_factor, head_dim=128)
    rng = np.random.default_rng(seed)
    # finite codes only (NaN / inf codes excluded), roughly normal magnitudes
    top = 0x7f if fmt == "e4m3" else 0x7c
    finite = np.concatenate([np.arange(0x00, top), np.arange(0x80, 0x80 + top)]).astype(np.uint8)
    vals = oracle.fp8_values(finite, fmt)
    weight = np.exp(-0.5 * (vals / 2.0) ** 2)
    weight /= weight.sum()
    pool = np.full((w.num_pages, 2, hkv, ps, 128), 0x7f, np.uint8)   # NaN canaries
    k_dense, v_dense = [], []
    for b in range(w.batch):
        L = int(w.kv_lens[b])
        kc = rng.choice(finite, size=(L, hkv, 128), p=weight)
        vc = rng.choice(finite, size=(L, hkv, 128), p=weight)
        pages = w.pages_of(b)
        for t in range(L):
            pool[pages[t // ps], 0, :, t % ps] = kc[t]
            pool[pages[t // ps], 1, :, t % ps] = vc[t]
        k_dense.append(kc)
        v_dense.append(vc)
    gen = torch.Generator().manual_seed(seed)
    q_bits = to_bits(torch.randn((w.batch, hq, 128), generator=gen), q_dtype)
    return w, q_bits, pool, k_dense, v_dense


def dense_sdpa_fp8(w, q_bits, k_codes, v_codes, k_scale, v_scale, scale, fmt="e4m3"):
    """SDPA in float64 on the dequantised dense K/V (code value * scale)."""
    q = widen(q_bits, w.dtype)
    outs, lses = [], []
    for b in range(w.batch):
        k = torch.from_numpy(torch_values(k_codes[b], fmt) * np.float64(k_scale)).permute(1, 0, 2)[None]
        v = torch.from_numpy(torch_values(v_codes[b], fmt) * np.float64(v_scale)).permute(1, 0, 2)[None]
        o = torch.nn.functional.scaled_dot_product_attention(q[b][None, :, None, :], k, v,
                                                             scale=scale, enable_gqa=True)
        outs.append(o[0, :, 0, :])
        kk = k[0].repeat_interleave(w.group, dim=0)
        lses.append(torch.logsumexp(torch.einsum("hd,hld->hl", q[b], kk) * scale, dim=-1))
    return torch.stack(outs).numpy(), torch.stack(lses).numpy()


FP8_CASES = [
    # (lens, hq, hkv, ps, q dtype, k_scale, v_scale, format)
    ([17, 64, 130, 1], 8, 2, 16, "bf16", 0.0625, 0.03125, "e4m3"),
    ([200, 33], 32, 8, 16, "f16", 0.1, 0.7, "e4m3"),
    ([65, 3, 100], 8, 1, 64, "bf16", 1.0, 1.0, "e4m3"),
    ([90, 300], 16, 4, 16, "bf16", 0.03, 0.11, "e5m2"),
]


@pytest.mark.parametrize("case", range(len(FP8_CASES)))
def test_fp8_decode_matches_dense_sdpa_on_dequantised_values(case):
    lens, hq, hkv, ps, qd, ks, vs, fmt = FP8_CASES[case]
    w, q_bits, pool, kd, vd = fp8_case(lens, hq, hkv, ps, 300 + case, qd, fmt=fmt)
    odt = oracle.BF16 if qd == "bf16" else oracle.F16
    out, lse = oracle.decode_fp8(q_bits, odt, pool, ks, vs, w.page_indptr, w.page_indices,
                                 w.last_page_len, w.sm_scale, fmt)
    ro, rl = dense_sdpa_fp8(w, q_bits, kd, vd, np.float32(ks), np.float32(vs), w.sm_scale, fmt)
    assert np.isfinite(out).all()               # NaN canaries never read
    np.testing.assert_allclose(out, ro, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, rl, rtol=0, atol=1e-12)


def test_fp8_scales_act_as_exact_factors():
    # K scaled by c is the softmax scale multiplied by c; V scaled by c scales
    # the output by c and leaves the lse alone (powers of two keep it exact)
    w, q_bits, pool, _, _ = fp8_case([40, 77], 8, 2, 16, 321)
    base_o, base_l = oracle.decode_fp8(q_bits, oracle.BF16, pool, 1.0, 1.0, w.page_indptr,
                                       w.page_indices, w.last_page_len, w.sm_scale)
    o, l = oracle.decode_fp8(q_bits, oracle.BF16, pool, 4.0, 0.25, w.page_indptr,
                             w.page_indices, w.last_page_len, w.sm_scale / 4)
    np.testing.assert_array_equal(o, base_o * 0.25)
    np.testing.assert_array_equal(l, base_l)


def test_fp8_pool_equals_16bit_pool_of_the_same_values():
    # every E4M3 value is exact in bf16, so the 8-bit pool with unit scales must
    # give exactly the 16-bit decode of the widened pool
    w, q_bits, pool, _, _ = fp8_case([90, 5, 31], 16, 4, 16, 322)
    finite = np.isfinite(oracle.e4m3_values(pool))
    pool16 = to_bits(torch.from_numpy(np.where(finite, oracle.e4m3_values(pool), 0.0)), "bf16")
    o8, l8 = oracle.decode_fp8(q_bits, oracle.BF16, pool, 1.0, 1.0, w.page_indptr,
                               w.page_indices, w.last_page_len, w.sm_scale)
    o16, l16 = oracle.decode(q_bits, pool16, oracle.BF16, w.page_indptr, w.page_indices,
                             w.last_page_len, w.sm_scale)
    np.testing.assert_array_equal(o8, o16)
    np.testing.assert_array_equal(l8, l16)


@pytest.mark.parametrize("fmt", ["e4m3", "e5m2"])
def test_fp8_append_positions_and_codes(fmt):
    # page_size 4: request 0 owns pages [3, 1] and holds 6 tokens after
    # appending 3 -> positions 3, 4, 5 = page 3 slot 3, page 1 slots 0, 1
    P, ps, hkv, D = 4, 4, 2, 16
    pool = np.full((P, 2, hkv, ps, D), 0x55, np.uint8)
    indptr = np.array([0, 2], np.int32)
    indices = np.array([3, 1], np.int32)
    last = np.array([2], np.int32)
    app = np.array([0, 3], np.int32)
    gen = torch.Generator().manual_seed(5)
    k = torch.randn((3, hkv, D), generator=gen) * 20
    v = torch.randn((3, hkv, D), generator=gen) * 300     # some saturate at scale 0.5
    if fmt == "e4m3":
        ks, vs, top, sat = np.float32(0.125), np.float32(0.5), 448.0, 0x7e
    else:
        ks, vs, top, sat = np.float32(0.001), np.float32(0.004), E5M2_MAX, 0x7b
    for dt, odt in (("bf16", oracle.BF16), ("f16", oracle.F16)):
        kb, vb = to_bits(k, dt), to_bits(v, dt)
        out = oracle.append_fp8(pool, ks, vs, indptr, indices, last, kb, vb, odt, app, fmt)
        expect = pool.copy()
        kq = widen(kb, dt).float().numpy() / ks
        vq = widen(vb, dt).float().numpy() / vs

        def enc(x):
            return np.where(np.abs(x) >= top, np.where(x < 0, 0x80 | sat, sat),
                            torch_encode(np.clip(x, -top, top), fmt))
        kc, vc = enc(kq), enc(vq)
        for row, (page, slot) in enumerate([(3, 3), (1, 0), (1, 1)]):
            expect[page, 0, :, slot, :] = kc[row]
            expect[page, 1, :, slot, :] = vc[row]
        np.testing.assert_array_equal(out, expect)
        assert (np.abs(vq) >= top).any()


def test_fp8_append_rejects_bad_scales():
    pool = np.zeros((2, 2, 1, 4, 16), np.uint8)
    args = (np.array([0, 1], np.int32), np.array([0], np.int32), np.array([1], np.int32),
            np.zeros((1, 1, 16), np.uint16), np.zeros((1, 1, 16), np.uint16), oracle.BF16,
            np.array([0, 1], np.int32))
    for ks, vs in ((0.0, 1.0), (1.0, -2.0), (np.inf, 1.0), (1.0, np.nan)):
        with pytest.raises(oracle.OracleError):
            oracle.append_fp8(pool, ks, vs, *args)
