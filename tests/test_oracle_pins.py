"""Pins for the CPU oracle: every check here compares the oracle with something other than itself —
library routines (numpy's IEEE half conversion, scipy's Sylvester Hadamard matrix, torch's
scaled-dot-product attention), closed forms, hand-worked fixtures under ``tests/golden``, invariants
the method fixes (codes in range, error within half a step, streaming == bulk) and brute force.

Passages: per-channel keys / per-token values and the min/max grid (KVQuant review, Method and
Problem; KV cache quantization wiki page, KIVI notes), FP16 recent window (Asymmetric KV Cache
Compression framework page, In practice), grouped/residual split and token-axis append (wiki page,
KIVI notes), Hadamard rotation shared by keys and query (framework page, Method; Dual-QK abstract).
"""
import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import scipy.linalg
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------------------------------------
# fp16 conversion
# --------------------------------------------------------------------------------------------------
def test_f16_to_f32_exhaustive(oracle_mod):
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    mine = oracle_mod.f16_to_f32(h)
    ref = h.view(np.float16).astype(np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(mine), nan)
    assert np.array_equal(mine[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_f32_to_f16_exhaustive_vs_compiler(oracle_mod):
    # Every binary32 bit pattern against the compiler's _Float16 conversion (round to nearest even).
    n = 1 << 32
    chunks = 64
    step = n // chunks
    with ThreadPoolExecutor(max_workers=os.cpu_count() or 4) as ex:
        bad = sum(ex.map(lambda i: oracle_mod.check_f32_to_f16_range(i * step, (i + 1) * step), range(chunks)))
    assert bad == 0


def test_f32_to_f16_sample_vs_numpy(oracle_mod):
    rng = np.random.default_rng(0)
    bits = rng.integers(0, 1 << 32, size=1 << 20, dtype=np.uint64).astype(np.uint32)
    f = bits.view(np.float32)
    f = f[~np.isnan(f)]
    # ties and the subnormal / overflow edges explicitly
    edges = np.array([65504, 65519.996, 65520, 2.0 ** -24, 2.0 ** -25, 1.5 * 2.0 ** -25, 2.0 ** -14,
                      (1 - 2.0 ** -11) * 2.0 ** -14, 1 + 2.0 ** -11, 1 + 3 * 2.0 ** -11, -0.0, 0.0],
                     np.float32)
    f = np.concatenate([f, edges, -edges])
    with np.errstate(over="ignore"):
        ref = f.astype(np.float16).view(np.uint16)
    assert np.array_equal(oracle_mod.f32_to_f16(f), ref)


# --------------------------------------------------------------------------------------------------
# Walsh-Hadamard rotation (framework page, Method / In practice; Dual-QK abstract)
# --------------------------------------------------------------------------------------------------
def test_wht_f64_columns_match_sylvester_hadamard(oracle_mod):
    H = scipy.linalg.hadamard(128).astype(np.float64) / math.sqrt(128.0)
    for i in range(128):
        e = np.zeros(128)
        e[i] = 1.0
        np.testing.assert_allclose(oracle_mod.wht128_f64(e), H[:, i], rtol=0, atol=1e-15)


def test_wht_is_orthogonal_and_preserves_dot(oracle_mod):
    rng = np.random.default_rng(1)
    q, k = rng.standard_normal(128), rng.standard_normal(128)
    Hq, Hk = oracle_mod.wht128_f64(q), oracle_mod.wht128_f64(k)
    assert abs(Hq @ Hk - q @ k) < 1e-12 * (np.abs(q) @ np.abs(k))
    # applying it twice gives the identity (H symmetric and orthonormal after scaling)
    np.testing.assert_allclose(oracle_mod.wht128_f64(Hq), q, atol=1e-13)


def test_wht_f32_scale_constant_and_accuracy(oracle_mod):
    e0 = np.zeros(128, np.float32)
    e0[0] = 1.0
    y = oracle_mod.wht128_f32(e0)
    want = np.float32(1.0 / math.sqrt(128.0))
    assert want.view(np.uint32) == 0x3DB504F3
    assert np.all(y.view(np.uint32) == 0x3DB504F3)
    H = scipy.linalg.hadamard(128).astype(np.float64) / math.sqrt(128.0)
    rng = np.random.default_rng(2)
    for _ in range(50):
        x = (rng.standard_normal(128) * rng.choice([1, 20], 128)).astype(np.float16).astype(np.float32)
        exact = H @ x.astype(np.float64)
        got = oracle_mod.wht128_f32(x).astype(np.float64)
        # 7 rounded adds on partial sums bounded by sum|x|, then one rounded multiply
        bound = 8 * 2.0 ** -24 * np.abs(x).sum() / math.sqrt(128.0) + 1e-30
        assert np.max(np.abs(got - exact)) <= bound


# --------------------------------------------------------------------------------------------------
# min/max quantizer of one group (KVQuant review, Problem; wiki page, KIVI notes)
# --------------------------------------------------------------------------------------------------
def _random_groups(rng, n_groups, G):
    out = []
    for i in range(n_groups):
        kind = i % 5
        if kind == 0:
            x = rng.standard_normal(G)
        elif kind == 1:
            x = rng.standard_normal(G) * 20
        elif kind == 2:
            x = rng.standard_normal(G) * 1e-3 + 3.0
        elif kind == 3:
            x = rng.uniform(-60000, 60000, G)
        else:
            x = rng.standard_normal(G) * 1e-6  # subnormal-scale ranges
        out.append(x.astype(np.float16))
    return out


@pytest.mark.parametrize("bits", [2, 4])
@pytest.mark.parametrize("G", [16, 32, 64, 128])
def test_quantizer_invariants(oracle_mod, bits, G):
    rng = np.random.default_rng(bits * 1000 + G)
    top = (1 << bits) - 1
    for x in _random_groups(rng, 200, G):
        codes, s16, z16 = oracle_mod.quantize_group(x, bits)
        xf = x.astype(np.float64)
        # the zero point is the group minimum, the scale is the step of a uniform grid over [min, max]
        assert np.float16(np.uint16(z16).view(np.float16)) == x.min()
        s = float(np.uint16(s16).view(np.float16))
        z = float(np.uint16(z16).view(np.float16))
        exact_step = (float(x.max()) - float(x.min())) / top
        # fp32 subtraction + division (2 roundings) then fp16 rounding (half an fp16 ulp, 2^-25 abs floor)
        assert abs(s - exact_step) <= 2.0 ** -11 * exact_step + 2.0 ** -25 + 4 * 2.0 ** -24 * exact_step
        assert codes.min() >= 0 and codes.max() <= top
        xh = codes.astype(np.float64) * s + z
        err = np.abs(xf - xh)
        if s == 0.0:
            assert np.all(codes == 0)
            assert np.all(err <= float(x.max()) - float(x.min()))
            continue
        bound = s / 2 + top * abs(exact_step - s) + 2.0 ** -20 * np.abs(xf) + 2.0 ** -20 * s
        assert np.all(err <= bound)
        # brute force: the chosen level is the nearest one (up to fp32 rounding of (x - z) / s)
        levels = np.arange(top + 1)[None, :] * s + z
        d = np.abs(xf[:, None] - levels)
        best = d.min(axis=1)
        chosen = d[np.arange(G), codes]
        assert np.all(chosen <= best + 2.0 ** -20 * (np.abs(xf) + s))


def test_quantizer_constant_group(oracle_mod):
    for val in [0.0, 1.5, -3.25, 65504.0, 2.0 ** -24]:
        x = np.full(32, val, np.float16)
        codes, s16, z16 = oracle_mod.quantize_group(x, 2)
        assert s16 == 0 and np.all(codes == 0)
        assert np.uint16(z16).view(np.float16) == np.float16(val)


def test_quantizer_signed_zero_minimum(oracle_mod):
    # IEEE minimum/maximum order -0 below +0: a group of +0 and -0 has zero = -0 and max = +0.
    x = np.array([0.0, -0.0] * 16, np.float16)
    codes, s16, z16 = oracle_mod.quantize_group(x, 2)
    assert z16 == 0x8000 and s16 == 0 and np.all(codes == 0)
    x = np.array([0.0, 1.5, -0.0] + [0.5] * 29, np.float16)
    codes, s16, z16 = oracle_mod.quantize_group(x, 2)
    assert z16 == 0x8000 and np.uint16(s16).view(np.float16) == np.float16(0.5)
    assert list(codes[:3]) == [0, 3, 0]


@pytest.mark.parametrize("bits", [2, 4])
def test_quantizer_two_valued_and_grid_round_trip(oracle_mod, bits):
    top = (1 << bits) - 1
    rng = np.random.default_rng(3)
    # {min, max} only, with a step that fp16 represents exactly: codes are 0 and top, exact recon
    x = np.where(rng.random(32) < 0.5, -1.0, -1.0 + top * 0.25).astype(np.float16)
    x[0], x[1] = -1.0, -1.0 + top * 0.25
    codes, s16, z16 = oracle_mod.quantize_group(x, bits)
    assert set(codes.tolist()) == {0, top}
    s, z = float(np.uint16(s16).view(np.float16)), float(np.uint16(z16).view(np.float16))
    np.testing.assert_array_equal(codes * s + z, x.astype(np.float64))
    # inputs on a power-of-two grid round-trip exactly
    c = rng.integers(0, top + 1, 64)
    c[0], c[1] = 0, top
    x = (c * 0.125 - 1.5).astype(np.float16)
    codes, s16, z16 = oracle_mod.quantize_group(x, bits)
    np.testing.assert_array_equal(codes, c)


def test_quantizer_half_way_ties_go_to_even(oracle_mod):
    # min 0, max 3 -> step 1; x = 0.5, 1.5, 2.5 sit exactly half-way and round to the even level.
    x = np.array([0.0, 3.0, 0.5, 1.5, 2.5] + [1.0] * 27, np.float16)
    codes, s16, z16 = oracle_mod.quantize_group(x, 2)
    assert np.uint16(s16).view(np.float16) == np.float16(1.0)
    assert list(codes[:5]) == [0, 3, 0, 2, 2]


# --------------------------------------------------------------------------------------------------
# packed layout (hand-worked fixture)
# --------------------------------------------------------------------------------------------------
def _golden_layout():
    rows = []
    with open(os.path.join(GOLDEN, "layout_examples.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


def test_layout_matches_hand_worked_examples(oracle_mod):
    rows = _golden_layout()
    assert len(rows) > 20
    kinds = set()
    for r in rows:
        kinds.add(r[0])
        if r[0] == "kparam":
            assert oracle_mod.key_param_pos(int(r[1])) == int(r[2]), r
            continue
        kind, bits, i, c, word, bit = r[0], int(r[1]), int(r[2]), int(r[3]), int(r[4]), int(r[5])
        fn = {"key": oracle_mod.key_word_bit, "value": oracle_mod.value_word_bit,
              "key_v2": oracle_mod.key_word_bit_v2, "value_v2": oracle_mod.value_word_bit_v2}[kind]
        assert fn(i, c, bits) == (word, bit), r
    assert kinds == {"key", "value", "kparam", "key_v2", "value_v2"}


@pytest.mark.parametrize("kind", ["key", "value"])
@pytest.mark.parametrize("bits", [2, 4])
def test_layout_is_a_bijection_onto_the_tile(oracle_mod, kind, bits):
    fn = oracle_mod.key_word_bit if kind == "key" else oracle_mod.value_word_bit
    used = np.zeros(64 * bits * 32, np.int32)  # one counter per bit of the tile
    for i in range(16):
        for c in range(128):
            w, b = fn(i, c, bits)
            assert 0 <= w < 64 * bits and b % bits == 0 and b + bits <= 32
            used[w * 32 + b: w * 32 + b + bits] += 1
    assert np.all(used == 1)
    pos = sorted(oracle_mod.key_param_pos(c) for c in range(128))
    assert pos == list(range(128))


@pytest.mark.parametrize("kind", ["key", "value"])
@pytest.mark.parametrize("bits", [2, 4])
def test_layout_v2_is_a_bijection_onto_rows(oracle_mod, kind, bits):
    # one 128-token block of one unit: every code bit is used exactly once
    fn = oracle_mod.key_word_bit_v2 if kind == "key" else oracle_mod.value_word_bit_v2
    used = np.zeros(128 * 4 * bits * 32, np.int32)
    for t in range(128):
        for c in range(128):
            w, b = fn(t, c, bits)
            assert 0 <= w < 128 * 4 * bits and b % bits == 0 and b + bits <= 32
            used[w * 32 + b: w * 32 + b + bits] += 1
    assert np.all(used == 1)


# --------------------------------------------------------------------------------------------------
# whole-cache behaviour
# --------------------------------------------------------------------------------------------------
def _cfg(oracle_mod, B=2, Hq=4, Hkv=2, kb=2, vb=2, G=32, R=32, had=0, cap=512, layout=1, sink=0, rope=0.0):
    return oracle_mod.Config(B, Hq, Hkv, kb, vb, G, R, had, cap, layout=layout, sink=sink, rope_theta=rope)


def _inputs(B, T, Hkv, Hq, seed, outliers=True):
    g = torch.Generator().manual_seed(seed)
    k = torch.randn(B, T, Hkv, 128, generator=g)
    if outliers:
        k[..., 5] *= 20
        k[..., 77] *= 15
    v = torch.randn(B, T, Hkv, 128, generator=g)
    q = torch.randn(B, Hq, 128, generator=g)
    return k.half().numpy(), v.half().numpy(), q.half().numpy()


def _key_code(oracle_mod, cfg, cache, b, h, t, c):
    if cfg.layout == 2:
        w, bit = oracle_mod.key_word_bit_v2(t, c, cfg.key_bits)
        word = cache.k_codes[b, h].reshape(-1)[w]
    else:
        w, bit = oracle_mod.key_word_bit(t % 16, c, cfg.key_bits)
        word = cache.k_codes[b, h, t // 16][w]
    return (int(word) >> bit) & ((1 << cfg.key_bits) - 1)


def _value_code(oracle_mod, cfg, cache, b, h, t, c):
    if cfg.layout == 2:
        w, bit = oracle_mod.value_word_bit_v2(t, c, cfg.value_bits)
        word = cache.v_codes[b, h].reshape(-1)[w]
    else:
        w, bit = oracle_mod.value_word_bit(t % 16, c, cfg.value_bits)
        word = cache.v_codes[b, h, t // 16][w]
    return (int(word) >> bit) & ((1 << cfg.value_bits) - 1)


def _unpack_key(oracle_mod, cfg, cache, b, h, t):
    """Dequantize key (b, h, t) from the cache by reading the layout positions the fixture pins."""
    G = cfg.group_size
    s = cache.k_scale[b, h, t // G].view(np.float16).astype(np.float64)
    z = cache.k_zero[b, h, t // G].view(np.float16).astype(np.float64)
    out = np.empty(128)
    for c in range(128):
        p = oracle_mod.key_param_pos(c) if cfg.layout == 1 else c
        out[c] = _key_code(oracle_mod, cfg, cache, b, h, t, c) * s[p] + z[p]
    return out


def _unpack_value(oracle_mod, cfg, cache, b, h, t):
    G = cfg.group_size
    s = cache.v_scale[b, h, t].view(np.float16).astype(np.float64)
    z = cache.v_zero[b, h, t].view(np.float16).astype(np.float64)
    out = np.empty(128)
    for c in range(128):
        out[c] = _value_code(oracle_mod, cfg, cache, b, h, t, c) * s[c // G] + z[c // G]
    return out


def _sdpa(q, k, v, scale):
    """torch's scaled-dot-product attention in fp64. q [B][Hq][D], k/v [B][Hkv][T][D] -> [B][Hq][D]."""
    Hq, Hkv = q.shape[1], k.shape[1]
    kk = torch.from_numpy(k).repeat_interleave(Hq // Hkv, dim=1)
    vv = torch.from_numpy(v).repeat_interleave(Hq // Hkv, dim=1)
    qq = torch.from_numpy(q)[:, :, None, :]
    o = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv, scale=scale)
    return o[:, :, 0, :].numpy()


def test_no_quantization_equals_library_attention(oracle_mod):
    # With R >= T nothing is quantized: the oracle must equal plain softmax attention (GQA 2:1).
    B, T, Hkv, Hq = 2, 200, 2, 4
    cfg = _cfg(oracle_mod, B, Hq, Hkv, R=256, cap=512)
    k, v, q = _inputs(B, T, Hkv, Hq, 11)
    cache = oracle_mod.Cache(cfg)
    oracle_mod.quantize_prefill(cfg, cache, k, v, [T, T - 57])
    out = oracle_mod.decode(cfg, cache, q, 1 / math.sqrt(128))
    for b, Tb in enumerate([T, T - 57]):
        kb = k[b, :Tb].astype(np.float64).transpose(1, 0, 2)[None]
        vb = v[b, :Tb].astype(np.float64).transpose(1, 0, 2)[None]
        ref = _sdpa(q[b:b + 1].astype(np.float64), kb, vb, 1 / math.sqrt(128))
        np.testing.assert_allclose(out[b], ref[0], rtol=1e-12, atol=1e-13)


def test_hadamard_no_quantization_equals_rotated_attention(oracle_mod):
    # Keys are stored rotated (and rounded to fp16); the query is rotated by the same orthonormal H.
    B, T, Hkv, Hq = 1, 96, 1, 2
    cfg = _cfg(oracle_mod, B, Hq, Hkv, R=128, had=1, cap=256)
    k, v, q = _inputs(B, T, Hkv, Hq, 12)
    cache = oracle_mod.Cache(cfg)
    oracle_mod.quantize_prefill(cfg, cache, k, v, [T])
    out = oracle_mod.decode(cfg, cache, q, 0.1)
    H = scipy.linalg.hadamard(128).astype(np.float64) / math.sqrt(128.0)
    ring = cfg.residual + cfg.group_size
    krot = np.stack([cache.k_res[0, 0, t % ring].view(np.float16).astype(np.float64) for t in range(T)])
    # the stored keys are the fp16 rounding of H k (within one fp16 rounding of the exact rotation)
    exact = k[0, :, 0].astype(np.float64) @ H.T
    assert np.all(np.abs(krot - exact) <= np.abs(exact) * 2.0 ** -10 + 2.0 ** -23)
    qrot = q.astype(np.float64) @ H.T
    ref = _sdpa(qrot, krot[None, None], v[0, :, 0].astype(np.float64)[None, None], 0.1)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-13)
    # and q.k is preserved by the rotation: attention on unrotated keys differs only by fp16 rounding
    ref_unrot = _sdpa(q.astype(np.float64), k[0, :, 0].astype(np.float64)[None, None],
                      v[0, :, 0].astype(np.float64)[None, None], 0.1)
    np.testing.assert_allclose(out, ref_unrot, atol=2e-3)


@pytest.mark.parametrize("layout", [1, 2])
@pytest.mark.parametrize("kb,vb,G,R,had", [(2, 2, 32, 32, 0), (4, 2, 32, 0, 1), (2, 4, 64, 100, 0), (4, 4, 16, 16, 1)])
def test_quantized_attention_equals_library_attention_on_dequantized_cache(oracle_mod, kb, vb, G, R, had, layout):
    B, Hkv, Hq = 2, 2, 4
    lens = [301, 160]
    cfg = _cfg(oracle_mod, B, Hq, Hkv, kb, vb, G, R, had, cap=320, layout=layout)
    k, v, q = _inputs(B, max(lens), Hkv, Hq, 13 + kb + G)
    cache = oracle_mod.Cache(cfg)
    oracle_mod.quantize_prefill(cfg, cache, k, v, lens)
    out = oracle_mod.decode(cfg, cache, q, 1 / math.sqrt(128))
    H = scipy.linalg.hadamard(128).astype(np.float64) / math.sqrt(128.0)
    ring = R + G
    for b, T in enumerate(lens):
        Q = max(T - R, 0) // G * G
        assert oracle_mod.quantized_len(T, R, G) == Q
        assert T - Q <= R + G - 1 and (T < R or T - Q >= R)
        K = np.zeros((Hkv, T, 128))
        V = np.zeros((Hkv, T, 128))
        for h in range(Hkv):
            for t in range(T):
                if t < Q:
                    K[h, t] = _unpack_key(oracle_mod, cfg, cache, b, h, t)
                    V[h, t] = _unpack_value(oracle_mod, cfg, cache, b, h, t)
                else:
                    K[h, t] = cache.k_res[b, h, t % ring].view(np.float16)
                    V[h, t] = cache.v_res[b, h, t % ring].view(np.float16)
        # dequantized keys stay close to the (rotated) inputs: error bounded by the group's step
        kin = k[b, :T].astype(np.float64).transpose(1, 0, 2)
        if had:
            kin = kin @ H.T
        # (per channel over each key group: at most half a step of that group's grid, plus roundings)
        for g0 in range(0, Q, G):
            blk = kin[:, g0:g0 + G]
            step = (blk.max(axis=1) - blk.min(axis=1)) / ((1 << kb) - 1)
            err = np.abs(K[:, g0:g0 + G] - blk).max(axis=1)
            assert np.all(err <= step * (0.5 + 2.0 ** -9) + 2.0 ** -9 * np.abs(blk).max(axis=1))
        qq = q[b:b + 1].astype(np.float64)
        if had:
            qq = qq @ H.T
        ref = _sdpa(qq, K[None], V[None], 1 / math.sqrt(128))
        np.testing.assert_allclose(out[b], ref[0], rtol=1e-11, atol=1e-12)


def test_single_token_returns_its_value(oracle_mod):
    cfg = _cfg(oracle_mod, 1, 2, 1, R=4, cap=64)
    k, v, q = _inputs(1, 1, 1, 2, 14)
    cache = oracle_mod.Cache(cfg)
    oracle_mod.quantize_prefill(cfg, cache, k, v, [1])
    out = oracle_mod.decode(cfg, cache, q, 0.3)
    for h in range(2):
        np.testing.assert_array_equal(out[0, h], v[0, 0, 0].astype(np.float64))


def test_tiny_case_against_long_double_brute_force(oracle_mod):
    # T = 8 tokens, all quantized (R = 0, G = 16 over a 16-token capacity is not reached: use T=16).
    cfg = _cfg(oracle_mod, 1, 1, 1, 2, 2, 16, 0, 0, cap=16)
    k, v, q = _inputs(1, 16, 1, 1, 15)
    cache = oracle_mod.Cache(cfg)
    oracle_mod.quantize_prefill(cfg, cache, k, v, [16])
    out = oracle_mod.decode(cfg, cache, q, 1 / math.sqrt(128))
    K = np.array([_unpack_key(oracle_mod, cfg, cache, 0, 0, t) for t in range(16)], np.longdouble)
    V = np.array([_unpack_value(oracle_mod, cfg, cache, 0, 0, t) for t in range(16)], np.longdouble)
    qq = q[0, 0].astype(np.longdouble)
    s = (K @ qq) / np.sqrt(np.longdouble(128))
    p = np.exp(s - s.max())
    ref = (p[:, None] * V).sum(0) / p.sum()
    np.testing.assert_allclose(out[0, 0], ref.astype(np.float64), rtol=1e-13, atol=1e-14)


@pytest.mark.parametrize("layout", [1, 2])
@pytest.mark.parametrize("kb,vb,G,R,had", [(2, 2, 32, 32, 0), (4, 2, 32, 0, 1), (2, 2, 64, 128, 0), (4, 4, 16, 5, 0)])
def test_streaming_append_equals_bulk_prefill(oracle_mod, kb, vb, G, R, had, layout):
    B, Hkv, Hq = 2, 2, 2
    T0, n = 150, 3 * G + 7
    cap = ((T0 + n + G - 1) // G) * G
    cfg = _cfg(oracle_mod, B, Hq, Hkv, kb, vb, G, R, had, cap=cap, layout=layout)
    k, v, _ = _inputs(B, T0 + n, Hkv, Hq, 16 + G)
    stream = oracle_mod.Cache(cfg)
    oracle_mod.quantize_prefill(cfg, stream, k[:, :T0], v[:, :T0], [T0, T0])
    for t in range(T0, T0 + n):
        oracle_mod.append_token(cfg, stream, k[:, t], v[:, t])
    bulk = oracle_mod.Cache(cfg)
    oracle_mod.quantize_prefill(cfg, bulk, k, v, [T0 + n, T0 + n])
    T = T0 + n
    Q = max(T - R, 0) // G * G
    assert np.array_equal(stream.seq_len, bulk.seq_len)
    if layout == 1:
        np.testing.assert_array_equal(stream.k_codes[:, :, : Q // 16], bulk.k_codes[:, :, : Q // 16])
        np.testing.assert_array_equal(stream.v_codes[:, :, : Q // 16], bulk.v_codes[:, :, : Q // 16])
    else:
        np.testing.assert_array_equal(stream.k_codes[:, :, :Q], bulk.k_codes[:, :, :Q])
        per_word = 32 // vb  # tokens covered by one value word
        for t0 in range(0, Q, 128):
            nw = (min(Q, t0 + 128) - t0) // per_word
            np.testing.assert_array_equal(stream.v_codes[:, :, t0 // 128, :, :nw], bulk.v_codes[:, :, t0 // 128, :, :nw])
    np.testing.assert_array_equal(stream.k_scale[:, :, : Q // G], bulk.k_scale[:, :, : Q // G])
    np.testing.assert_array_equal(stream.k_zero[:, :, : Q // G], bulk.k_zero[:, :, : Q // G])
    np.testing.assert_array_equal(stream.v_scale[:, :, :Q], bulk.v_scale[:, :, :Q])
    np.testing.assert_array_equal(stream.v_zero[:, :, :Q], bulk.v_zero[:, :, :Q])
    ring = R + G
    live = [t % ring for t in range(Q, T)]
    np.testing.assert_array_equal(stream.k_res[:, :, live], bulk.k_res[:, :, live])
    np.testing.assert_array_equal(stream.v_res[:, :, live], bulk.v_res[:, :, live])


def test_append_rejects_capacity_overflow(oracle_mod):
    cfg = _cfg(oracle_mod, 1, 1, 1, G=16, R=0, cap=16)
    k, v, _ = _inputs(1, 17, 1, 1, 17)
    cache = oracle_mod.Cache(cfg)
    oracle_mod.quantize_prefill(cfg, cache, k[:, :16], v[:, :16], [16])
    with pytest.raises(ValueError):
        oracle_mod.append_token(cfg, cache, k[:, 16], v[:, 16])


@pytest.mark.parametrize("bits,G", [(2, 32), (2, 64), (2, 128), (4, 32)])
def test_average_bits_closed_form(oracle_mod, bits, G):
    # Buffer sizes give b + 32/G bits per cached element (fp16 scale + zero shared by G elements);
    # 2 bits at G = 32 is 3.0 bits, the size class of the KIVI-2 setting the KVQuant review quotes.
    cfg = _cfg(oracle_mod, 1, 1, 1, bits, bits, G, 0, 0, cap=1024)
    c = oracle_mod.Cache(cfg)
    total_bits = 8 * (c.k_codes.nbytes + c.v_codes.nbytes + c.k_scale.nbytes + c.k_zero.nbytes
                      + c.v_scale.nbytes + c.v_zero.nbytes)
    per_elem = total_bits / (2 * 1024 * 128)
    assert per_elem == bits + 32 / G


# ---- fp16 first token (attention sink): KVQuant review, Method; wiki page, verification notes ------

@pytest.mark.parametrize("layout", [1, 2])
def test_sink_first_token_left_out_of_group_zero(oracle_mod, layout):
    # Token 0 is made the unique minimum of every channel of key group 0: with the sink on, group 0's
    # zero-point must be the minimum over tokens 1..G-1 (brute force here), not token 0's value, and
    # token 0's own codes and value scale / zero must be 0.
    B, Hkv, Hq, G, T = 1, 1, 1, 32, 160
    k, v, _ = _inputs(B, T, Hkv, Hq, 41)
    k[0, 0, 0, :] = np.float16(-1000.0)
    v[0, 0, 0, :] = np.float16(-1000.0)
    for sink in (0, 1):
        cfg = _cfg(oracle_mod, B, Hq, Hkv, G=G, R=0, cap=T, layout=layout, sink=sink)
        cache = oracle_mod.Cache(cfg)
        oracle_mod.quantize_prefill(cfg, cache, k, v, [T])
        zero = cache.k_zero[0, 0, 0].view(np.float16).astype(np.float64)
        want = k[0, 1:G, 0, :].astype(np.float64).min(axis=0) if sink else np.full(128, -1000.0)
        for c in range(128):
            pos = oracle_mod.key_param_pos(c) if layout == 1 else c
            assert zero[pos] == want[c], (sink, c)
        if sink:
            assert all(_key_code(oracle_mod, cfg, cache, 0, 0, 0, c) == 0 for c in range(128))
            assert all(_value_code(oracle_mod, cfg, cache, 0, 0, 0, c) == 0 for c in range(128))
            assert not cache.v_scale[0, 0, 0].any() and not cache.v_zero[0, 0, 0].any()
            np.testing.assert_array_equal(cache.k_res[0, 0, G], k[0, 0, 0].view(np.uint16))  # row R + G
            np.testing.assert_array_equal(cache.v_res[0, 0, G], v[0, 0, 0].view(np.uint16))


@pytest.mark.parametrize("layout", [1, 2])
def test_sink_dominant_first_token_returns_its_fp16_value(oracle_mod, layout):
    # The query points along token 0's key with a margin of e^-60 over every other token, so the
    # softmax is token 0 to within 1e-20: with the sink on the output is token 0's fp16 value exactly
    # (to fp64 rounding); without it, token 0 is read back through its 2-bit codes and misses by the
    # quantization error.
    B, Hkv, Hq, G, T = 1, 1, 1, 32, 300
    k, v, _ = _inputs(B, T, Hkv, Hq, 43, outliers=False)
    k[0, 0, 0, :] = np.float16(16.0)
    q = np.full((1, 1, 128), np.float16(0.5), np.float16)
    scale = 1.0 / math.sqrt(128)
    base = (k[0, :, 0, :].astype(np.float64) @ q[0, 0].astype(np.float64)) * scale
    assert base[0] - base[1:].max() > 60.0
    outs = {}
    for sink in (0, 1):
        cfg = _cfg(oracle_mod, B, Hq, Hkv, G=G, R=32, cap=320, layout=layout, sink=sink)
        cache = oracle_mod.Cache(cfg)
        oracle_mod.quantize_prefill(cfg, cache, k, v, [T])
        outs[sink] = oracle_mod.decode(cfg, cache, q, scale)[0, 0]
    np.testing.assert_allclose(outs[1], v[0, 0, 0].astype(np.float64), rtol=0, atol=1e-13)
    assert np.abs(outs[0] - v[0, 0, 0].astype(np.float64)).max() > 1e-2


def test_sink_without_quantization_equals_library_attention(oracle_mod):
    # R >= T: nothing is quantized, and the fp16 first-token row holds the same bits as the window did,
    # so the result is plain softmax attention (GQA 2:1).
    B, T, Hkv, Hq = 2, 200, 2, 4
    cfg = _cfg(oracle_mod, B, Hq, Hkv, R=256, cap=512, sink=1)
    k, v, q = _inputs(B, T, Hkv, Hq, 47)
    cache = oracle_mod.Cache(cfg)
    oracle_mod.quantize_prefill(cfg, cache, k, v, [T, T - 57])
    out = oracle_mod.decode(cfg, cache, q, 1 / math.sqrt(128))
    for b, Tb in enumerate([T, T - 57]):
        kb = k[b, :Tb].astype(np.float64).transpose(1, 0, 2)[None]
        vb = v[b, :Tb].astype(np.float64).transpose(1, 0, 2)[None]
        ref = _sdpa(q[b:b + 1].astype(np.float64), kb, vb, 1 / math.sqrt(128))
        np.testing.assert_allclose(out[b], ref[0], rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("layout", [1, 2])
@pytest.mark.parametrize("had", [0, 1])
def test_sink_streaming_from_empty_equals_bulk(oracle_mod, layout, had):
    # Starting from an empty cache, the first append writes the fp16 first-token row and the first
    # flush leaves token 0 out of group 0; the result must match a bulk prefill bit for bit.
    B, Hkv, Hq, G, R = 2, 2, 2, 32, 16
    n = 4 * G + 9
    cap = ((n + G - 1) // G) * G
    cfg = _cfg(oracle_mod, B, Hq, Hkv, 2, 2, G, R, had, cap=cap, layout=layout, sink=1)
    k, v, _ = _inputs(B, n, Hkv, Hq, 53)
    stream = oracle_mod.Cache(cfg)
    oracle_mod.quantize_prefill(cfg, stream, k[:, :0], v[:, :0], [0, 0])
    for t in range(n):
        oracle_mod.append_token(cfg, stream, k[:, t], v[:, t])
    bulk = oracle_mod.Cache(cfg)
    oracle_mod.quantize_prefill(cfg, bulk, k, v, [n, n])
    Q = (n - R) // G * G
    if layout == 1:
        np.testing.assert_array_equal(stream.k_codes[:, :, : Q // 16], bulk.k_codes[:, :, : Q // 16])
        np.testing.assert_array_equal(stream.v_codes[:, :, : Q // 16], bulk.v_codes[:, :, : Q // 16])
    else:
        np.testing.assert_array_equal(stream.k_codes[:, :, :Q], bulk.k_codes[:, :, :Q])
        np.testing.assert_array_equal(stream.v_codes[:, :, 0, :, : Q * 2 // 32], bulk.v_codes[:, :, 0, :, : Q * 2 // 32])
    for key in ("k_scale", "k_zero"):
        np.testing.assert_array_equal(getattr(stream, key)[:, :, : Q // G], getattr(bulk, key)[:, :, : Q // G])
    for key in ("v_scale", "v_zero"):
        np.testing.assert_array_equal(getattr(stream, key)[:, :, :Q], getattr(bulk, key)[:, :, :Q])
    np.testing.assert_array_equal(stream.k_res[:, :, R + G], bulk.k_res[:, :, R + G])
    np.testing.assert_array_equal(stream.v_res[:, :, R + G], bulk.v_res[:, :, R + G])



# ---- pre-RoPE keys (KVQuant review, Method and Key idea: quantize keys before RoPE, apply RoPE after
# dequantization) ------------------------------------------------------------------------------------
def _rope_complex(K, theta):
    """RoPE written as complex multiplication: channel pair (i, i + 64) is the complex number
    k[i] + j k[i + 64], turned by exp(j t theta^(-i/64)) at position t. K: [..., T, 128] float64."""
    T = K.shape[-2]
    z = K[..., :64] + 1j * K[..., 64:]
    ang = np.arange(T, dtype=np.float64)[:, None] * theta ** (-np.arange(64, dtype=np.float64) / 64.0)[None, :]
    z = z * np.exp(1j * ang)
    return np.concatenate([z.real, z.imag], axis=-1)


@pytest.mark.parametrize("theta", [10000.0, 500000.0])
def test_rope_without_quantization_equals_library_attention_on_rotated_keys(oracle_mod, theta):
    # R >= T: nothing is quantized; the cache keeps the keys without RoPE, and decode rotates each one
    # at its own position, so the result is plain softmax attention over the rotated keys (GQA 2:1).
    B, T, Hkv, Hq = 2, 300, 2, 4
    cfg = _cfg(oracle_mod, B, Hq, Hkv, R=512, cap=512, rope=theta)
    k, v, q = _inputs(B, T, Hkv, Hq, 61)
    cache = oracle_mod.Cache(cfg)
    oracle_mod.quantize_prefill(cfg, cache, k, v, [T, T - 99])
    # the window holds the keys exactly as given (no RoPE in the cache)
    ring = cfg.residual + cfg.group_size
    assert np.array_equal(cache.k_res[0, 1, 7 % ring], k[0, 7, 1].view(np.uint16))
    out = oracle_mod.decode(cfg, cache, q, 1 / math.sqrt(128))
    for b, Tb in enumerate([T, T - 99]):
        kb = _rope_complex(k[b, :Tb].astype(np.float64).transpose(1, 0, 2), theta)[None]
        vb = v[b, :Tb].astype(np.float64).transpose(1, 0, 2)[None]
        ref = _sdpa(q[b:b + 1].astype(np.float64), kb, vb, 1 / math.sqrt(128))
        np.testing.assert_allclose(out[b], ref[0], rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("layout", [1, 2])
def test_rope_quantized_equals_library_attention_on_dequantized_rotated_keys(oracle_mod, layout):
    # Keys are quantized before RoPE: the dequantized cache rotated at each position, then plain
    # attention, gives the oracle's output; and the stored codes equal those of the same cache
    # without RoPE (quantization does not see the rotation).
    B, Hkv, Hq, G, R = 1, 2, 4, 32, 32
    lens = [301]
    theta = 10000.0
    cfg = _cfg(oracle_mod, B, Hq, Hkv, 2, 2, G, R, 0, cap=384, layout=layout, rope=theta)
    k, v, q = _inputs(B, max(lens), Hkv, Hq, 62)
    cache = oracle_mod.Cache(cfg)
    oracle_mod.quantize_prefill(cfg, cache, k, v, lens)
    pcfg = _cfg(oracle_mod, B, Hq, Hkv, 2, 2, G, R, 0, cap=384, layout=layout)
    plain = oracle_mod.Cache(pcfg)
    oracle_mod.quantize_prefill(pcfg, plain, k, v, lens)
    for name in ("k_codes", "k_scale", "k_zero", "v_codes", "k_res"):
        assert np.array_equal(getattr(cache, name), getattr(plain, name)), name
    out = oracle_mod.decode(cfg, cache, q, 1 / math.sqrt(128))
    T = lens[0]
    Q = max(T - R, 0) // G * G
    ring = R + G
    K = np.zeros((Hkv, T, 128))
    V = np.zeros((Hkv, T, 128))
    for h in range(Hkv):
        for t in range(T):
            if t < Q:
                K[h, t] = _unpack_key(oracle_mod, cfg, cache, 0, h, t)
                V[h, t] = _unpack_value(oracle_mod, cfg, cache, 0, h, t)
            else:
                K[h, t] = cache.k_res[0, h, t % ring].view(np.float16)
                V[h, t] = cache.v_res[0, h, t % ring].view(np.float16)
    ref = _sdpa(q.astype(np.float64), _rope_complex(K, theta)[None], V[None], 1 / math.sqrt(128))
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)


def test_rope_relative_position(oracle_mod):
    # RoPE makes q.k depend on positions only through their difference: a query turned by m positions
    # against keys at positions t scores like the unturned query against keys at t - m. With a single
    # key repeated at every position, turning the query by m therefore moves the attention pattern by m.
    T, theta = 64, 10000.0
    cfg = _cfg(oracle_mod, 1, 1, 1, R=128, cap=128, rope=theta)
    rng = np.random.default_rng(63)
    k1 = rng.standard_normal(128).astype(np.float16)
    k = np.tile(k1, (1, T, 1, 1)).reshape(1, T, 1, 128)
    v = np.zeros((1, T, 1, 128), np.float16)
    v[0, :, 0, 0] = np.arange(T) / 8.0        # channel 0 of the output: the mean attended position / 8
    v[0, :, 0, 1] = (np.arange(T) % 2) * 1.0
    q0 = (2.0 * k1.astype(np.float64))
    cache = oracle_mod.Cache(cfg)
    oracle_mod.quantize_prefill(cfg, cache, k.astype(np.float16), v, [T])
    m = 20
    z = q0[:64] + 1j * q0[64:]
    z = z * np.exp(1j * m * theta ** (-np.arange(64) / 64.0))
    qm = np.concatenate([z.real, z.imag]).astype(np.float16)[None, None]
    out_m = oracle_mod.decode(cfg, cache, qm, 0.5)
    # reference: scores of the turned query equal those of q0 against keys rotated by (t - m)
    qm64 = qm.astype(np.float64)[0, 0]
    K = _rope_complex(np.tile(k1.astype(np.float64), (T, 1)), theta)
    s = 0.5 * K @ qm64
    p = np.exp(s - s.max())
    p /= p.sum()
    assert abs(out_m[0, 0, 0] - p @ (np.arange(T) / 8.0)) < 1e-9
    # the attention peaks at position m, where the key is turned exactly like the query
    assert int(np.argmax(s)) == m


# ---- dense-and-sparse outliers (KVQuant review, Method: per-vector thresholds keep about 1% of the
# entries in an fp16 sparse store; reading R12) ----------------------------------------------------------
def _total_order_key(h):
    """IEEE total order of binary16 bit patterns (-0 < +0), as signed integers; numpy only."""
    h = h.astype(np.int32)
    return np.where(h & 0x8000, -(h & 0x7FFF) - 1, h)


@pytest.mark.parametrize("layout", [1, 2])
def test_outliers_are_each_tokens_largest_entry_kept_in_fp16(oracle_mod, layout):
    B, T, Hkv, Hq, G, R = 1, 300, 2, 2, 32, 32
    cfg = _cfg(oracle_mod, B, Hq, Hkv, 2, 2, G, R, 0, cap=384, layout=layout)
    cfg.outliers = 1
    k, v, q = _inputs(B, T, Hkv, Hq, 81)
    k[0, 17, 1, 40] = -k[0, 17, 1, 40:41].max() - 100.0   # a tie-free negative outlier
    v[0, 20, 0, 3] = v[0, 20, 0, 9] = 50.0                 # a tie: the lower channel wins
    cache = oracle_mod.Cache(cfg)
    oracle_mod.quantize_prefill(cfg, cache, k, v, [T])
    Q = (T - R) // G * G
    for h in range(Hkv):
        for name, x in (("k", k), ("v", v)):
            mag = x[0, :Q, h].view(np.uint16) & 0x7FFF
            want = mag.argmax(axis=1)  # numpy's argmax takes the first of equal maxima
            ch = getattr(cache, f"{name}_out_ch")[0, h, :Q]
            val = getattr(cache, f"{name}_out_val")[0, h, :Q]
            assert np.array_equal(ch, want)
            assert np.array_equal(val, x[0, np.arange(Q), h, want].view(np.uint16))
            assert np.all(getattr(cache, f"{name}_out_ch")[0, h, Q:] == 0xFFFF)  # window tokens: none
    assert cache.k_out_ch[0, 1, 17] == 40 and cache.v_out_ch[0, 0, 20] == 3


def test_outliers_are_chosen_on_the_rotated_keys(oracle_mod):
    # with the Hadamard option the cache holds rotated keys (reading R2), so a key's outlier is the
    # largest entry of the rotated fp16 key: rotate each input key with the pinned fp32 transform,
    # round to fp16, and take the first largest magnitude; values are not rotated
    B, T, Hkv, Hq, G, R = 1, 200, 1, 2, 32, 32
    cfg = _cfg(oracle_mod, B, Hq, Hkv, 2, 2, G, R, 1, cap=224)
    cfg.outliers = 1
    k, v, q = _inputs(B, T, Hkv, Hq, 85)
    cache = oracle_mod.Cache(cfg)
    oracle_mod.quantize_prefill(cfg, cache, k, v, [T])
    Q = (T - R) // G * G
    rot = np.stack([oracle_mod.f32_to_f16(oracle_mod.wht128_f32(oracle_mod.f16_to_f32(k[0, t, 0]))) for t in range(Q)])
    want = (rot & 0x7FFF).argmax(axis=1)
    assert np.array_equal(cache.k_out_ch[0, 0, :Q], want)
    assert np.array_equal(cache.k_out_val[0, 0, :Q], rot[np.arange(Q), want])
    raw = (k[0, :Q, 0].view(np.uint16) & 0x7FFF).argmax(axis=1)
    assert not np.array_equal(want, raw)  # the rotation moves the outliers (channels 5 and 77 are spread)
    assert np.array_equal(cache.v_out_ch[0, 0, :Q], (v[0, :Q, 0].view(np.uint16) & 0x7FFF).argmax(axis=1))


@pytest.mark.parametrize("layout", [1, 2])
def test_outliers_left_out_of_group_statistics(oracle_mod, layout):
    # every key group's per-channel min / max and every value group's per-token min / max run over
    # the non-outlier entries only; a key channel whose entries are all outliers has scale and zero 0
    B, T, Hkv, Hq, G, R, kb, vb = 1, 200, 1, 1, 32, 8, 2, 4
    cfg = _cfg(oracle_mod, B, Hq, Hkv, kb, vb, G, R, 0, cap=256, layout=layout)
    cfg.outliers = 1
    k, v, q = _inputs(B, T, Hkv, Hq, 82)
    k[0, :64, 0, 5] = 1000.0  # channel 5 is every token's outlier in the first two groups
    cache = oracle_mod.Cache(cfg)
    oracle_mod.quantize_prefill(cfg, cache, k, v, [T])
    Q = (T - R) // G * G
    kb16 = k[0, :Q, 0].view(np.uint16)
    kout = np.zeros((Q, 128), bool)
    kout[np.arange(Q), cache.k_out_ch[0, 0, :Q]] = True
    for g in range(Q // G):
        for c in range(128):
            keep = ~kout[g * G:(g + 1) * G, c]
            pos = oracle_mod.key_param_pos(c) if layout == 1 else c
            s16, z16 = cache.k_scale[0, 0, g, pos], cache.k_zero[0, 0, g, pos]
            if not keep.any():
                assert s16 == 0 and z16 == 0
                continue
            col = kb16[g * G:(g + 1) * G, c][keep]
            mn, mx = col[np.argmin(_total_order_key(col))], col[np.argmax(_total_order_key(col))]
            assert z16 == mn
            s32 = np.float32((np.float32(mx.view(np.float16)) - np.float32(mn.view(np.float16))) / np.float32(3))
            assert s16 == np.float16(s32).view(np.uint16)
    assert np.all(cache.k_scale[0, 0, :2, 5 if layout == 2 else oracle_mod.key_param_pos(5)] == 0)
    vb16 = v[0, :Q, 0].view(np.uint16)
    for t in range(Q):
        for j in range(128 // G):
            row = vb16[t, j * G:(j + 1) * G]
            keep = np.arange(j * G, (j + 1) * G) != cache.v_out_ch[0, 0, t]
            col = row[keep]
            assert cache.v_zero[0, 0, t, j] == col[np.argmin(_total_order_key(col))]


def test_outliers_dequantized_attention_equals_library_attention(oracle_mod):
    # the dense codes dequantized, each token's outlier put back, then plain attention = the oracle
    B, Hkv, Hq, G, R = 1, 2, 4, 32, 32
    T = 301
    cfg = _cfg(oracle_mod, B, Hq, Hkv, 2, 2, G, R, 0, cap=320)
    cfg.outliers = 1
    k, v, q = _inputs(B, T, Hkv, Hq, 83)
    cache = oracle_mod.Cache(cfg)
    oracle_mod.quantize_prefill(cfg, cache, k, v, [T])
    out = oracle_mod.decode(cfg, cache, q, 1 / math.sqrt(128))
    Q = (T - R) // G * G
    ring = R + G
    K = np.zeros((Hkv, T, 128))
    V = np.zeros((Hkv, T, 128))
    for h in range(Hkv):
        for t in range(T):
            if t < Q:
                K[h, t] = _unpack_key(oracle_mod, cfg, cache, 0, h, t)
                V[h, t] = _unpack_value(oracle_mod, cfg, cache, 0, h, t)
                K[h, t, cache.k_out_ch[0, h, t]] = cache.k_out_val[0, h, t].view(np.float16)
                V[h, t, cache.v_out_ch[0, h, t]] = cache.v_out_val[0, h, t].view(np.float16)
            else:
                K[h, t] = cache.k_res[0, h, t % ring].view(np.float16)
                V[h, t] = cache.v_res[0, h, t % ring].view(np.float16)
    ref = _sdpa(q.astype(np.float64), K[None], V[None], 1 / math.sqrt(128))
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)
    # and the outliers are exact: the largest entries of the inputs come back bit for bit
    assert np.array_equal(K[0, np.arange(Q), cache.k_out_ch[0, 0, :Q]].astype(np.float16),
                          k[0, np.arange(Q), 0, cache.k_out_ch[0, 0, :Q]])


@pytest.mark.parametrize("layout", [1, 2])
def test_outliers_streaming_equals_bulk(oracle_mod, layout):
    B, Hkv, Hq, G, R = 1, 1, 2, 32, 32
    T0, n = 70, 3 * 32 + 5
    cfg = _cfg(oracle_mod, B, Hq, Hkv, 2, 2, G, R, 0, cap=256, layout=layout)
    cfg.outliers = 1
    k, v, q = _inputs(B, T0 + n, Hkv, Hq, 84)
    bulk = oracle_mod.Cache(cfg)
    oracle_mod.quantize_prefill(cfg, bulk, k, v, [T0 + n])
    stream = oracle_mod.Cache(cfg)
    oracle_mod.quantize_prefill(cfg, stream, k[:, :T0], v[:, :T0], [T0])
    for s in range(n):
        oracle_mod.append_token(cfg, stream, k[:, T0 + s], v[:, T0 + s])
    for name in ("k_codes", "k_scale", "k_zero", "v_scale", "v_zero", "k_out_ch", "k_out_val", "v_out_ch", "v_out_val"):
        assert np.array_equal(getattr(stream, name), getattr(bulk, name)), name


# ---- R13: paged storage --------------------------------------------------------------------------
# KVQuant review (Limitations, Future work, Sparks): blocked allocation instead of copying the
# previous tokens' data on every update. Paging moves where a token's codes and parameters live, never
# what they are: every pin below compares against the contiguous cache of the same inputs.

_PAGED_ARRAYS = ("k_codes", "v_codes", "k_scale", "k_zero", "v_scale", "v_zero", "k_out_ch", "k_out_val",
                 "v_out_ch", "v_out_val")


def _page_slice(cfg, name, j):
    """Index range of logical page j along the token-derived axis of array `name` (contiguous layout)."""
    P, G = cfg.page_tokens, cfg.group_size
    per = {"k_scale": P // G, "k_zero": P // G}.get(name)
    if per is None:
        if name in ("k_codes", "v_codes") and cfg.layout == 1:
            per = P // 16
        elif name == "v_codes":  # rows v2: 128-token value blocks
            per = P // 128
        else:  # rows v2 key rows, value parameters, outliers: one entry per token
            per = P
    return slice(j * per, (j + 1) * per)


def _paged_pair(oracle_mod, layout, outliers, sink, table_fn, lens, appends=0, seed=91):
    B, Hkv, Hq, G, R, P, cap = 2, 2, 4, 32, 32, 128, 512
    M = cap // P
    extra = 3  # spare pool pages nobody uses
    kw = dict(layout=layout, sink=sink)
    contig = _cfg(oracle_mod, B, Hq, Hkv, 2, 2, G, R, 0, cap=cap, **kw)
    contig.outliers = outliers
    paged = _cfg(oracle_mod, B, Hq, Hkv, 2, 2, G, R, 0, cap=cap, **kw)
    paged.outliers = outliers
    paged.page_tokens, paged.num_pages = P, B * Hkv * M + extra
    T = max(lens) + appends
    k, v, q = _inputs(B, T, Hkv, Hq, seed)
    table = table_fn(B, Hkv, M, paged.num_pages)
    cc, pc = oracle_mod.Cache(contig), oracle_mod.Cache(paged, page_table=table)
    for cfg, cache in ((contig, cc), (paged, pc)):
        oracle_mod.quantize_prefill(cfg, cache, k[:, : max(lens)], v[:, : max(lens)], lens)
        for s in range(appends):
            t = max(lens) + s
            oracle_mod.append_token(cfg, cache, k[:, t], v[:, t])
    return contig, cc, paged, pc, q


def _identity_table(B, H, M, n):
    return np.arange(B * H * M, dtype=np.int32).reshape(B, H, M)


def _shuffled_table(B, H, M, n):
    perm = np.random.default_rng(7).permutation(n).astype(np.int32)
    return perm[: B * H * M].reshape(B, H, M)


@pytest.mark.parametrize("layout", [1, 2])
@pytest.mark.parametrize("outliers,sink", [(0, 0), (1, 1)])
def test_paged_identity_table_is_the_contiguous_cache(oracle_mod, layout, outliers, sink):
    # with unit u's page j at pool page u * M + j, the pool is the contiguous cache byte for byte:
    # the layout repeats every P tokens, so paging is an address map and nothing else
    contig, cc, paged, pc, q = _paged_pair(oracle_mod, layout, outliers, sink, _identity_table, [500, 300], appends=9)
    for name in _PAGED_ARRAYS:
        a, b = getattr(cc, name), getattr(pc, name)
        used = a.reshape(-1).size
        assert np.array_equal(b.reshape(-1)[:used], a.reshape(-1)), name
    for name in ("k_res", "v_res", "seq_len"):
        assert np.array_equal(getattr(cc, name), getattr(pc, name)), name
    out_c = oracle_mod.decode(contig, cc, q, 1 / math.sqrt(128))
    out_p = oracle_mod.decode(paged, pc, q, 1 / math.sqrt(128))
    assert np.array_equal(out_c, out_p)


@pytest.mark.parametrize("layout", [1, 2])
@pytest.mark.parametrize("outliers", [0, 1])
def test_paged_shuffled_pool_gathers_to_the_contiguous_cache(oracle_mod, layout, outliers):
    # pages scattered over a pool with spare pages: gathering each unit's pages through the table
    # gives the contiguous arrays, the spare pages stay untouched, and decode is bit-identical
    contig, cc, paged, pc, q = _paged_pair(oracle_mod, layout, outliers, 0, _shuffled_table, [500, 300], appends=12)
    table = pc.page_table
    used = set(table.reshape(-1).tolist())
    for name in _PAGED_ARRAYS:
        a, b = getattr(cc, name), getattr(pc, name)
        for bb in range(table.shape[0]):
            for h in range(table.shape[1]):
                for j in range(table.shape[2]):
                    np.testing.assert_array_equal(b[table[bb, h, j]], a[bb, h][_page_slice(paged, name, j)],
                                                  err_msg=f"{name} unit {bb},{h} page {j}")
        blank = 0xFFFF if name.endswith("_ch") else 0
        for p in set(range(paged.num_pages)) - used:
            assert (b[p] == blank).all(), f"{name}: spare page {p} was written"
    out_c = oracle_mod.decode(contig, cc, q, 1 / math.sqrt(128))
    out_p = oracle_mod.decode(paged, pc, q, 1 / math.sqrt(128))
    assert np.array_equal(out_c, out_p)


@pytest.mark.parametrize("outliers,sink", [(0, 0), (1, 1)])
@pytest.mark.parametrize("layout", [1, 2])
def test_paged_streaming_with_pages_allocated_on_demand(oracle_mod, layout, outliers, sink):
    # the caller hands out a page only when the quantized part first reaches it; streaming then
    # equals a bulk prefill into the same pages (outlier words and the sink row included), and a
    # missing page is an argument error
    B, Hkv, Hq, G, R, P, cap = 1, 2, 2, 32, 32, 128, 512
    cfg = _cfg(oracle_mod, B, Hq, Hkv, 2, 2, G, R, 0, cap=cap, layout=layout, sink=sink)
    cfg.outliers = outliers
    cfg.page_tokens, cfg.num_pages = P, 16
    T0, n = 100, 300
    k, v, q = _inputs(B, T0 + n, Hkv, Hq, 92)
    table = np.full((B, Hkv, cap // P), -1, np.int32)
    free = list(np.random.default_rng(3).permutation(cfg.num_pages))
    stream = oracle_mod.Cache(cfg, page_table=table)

    def need(T):  # allocate the pages the quantized part of length T reaches
        Q = oracle_mod.quantized_len(T, R, G)
        for h in range(Hkv):
            for j in range(-(-Q // P)):
                if stream.page_table[0, h, j] < 0:
                    stream.page_table[0, h, j] = free.pop()

    need(T0)
    oracle_mod.quantize_prefill(cfg, stream, k[:, :T0], v[:, :T0], [T0])
    for s in range(n):
        t = T0 + s
        if oracle_mod.quantized_len(t + 1, R, G) > oracle_mod.quantized_len(t, R, G) and \
                (oracle_mod.quantized_len(t + 1, R, G) - 1) // P != (oracle_mod.quantized_len(t, R, G) - 1) // P:
            with pytest.raises(ValueError):  # the flush reaches a page the caller has not handed out
                oracle_mod.append_token(cfg, stream, k[:, t], v[:, t])
            need(t + 1)
        oracle_mod.append_token(cfg, stream, k[:, t], v[:, t])
    bulk = oracle_mod.Cache(cfg, page_table=stream.page_table.copy())
    oracle_mod.quantize_prefill(cfg, bulk, k, v, [T0 + n])
    for name in _PAGED_ARRAYS + ("seq_len",):
        assert np.array_equal(getattr(stream, name), getattr(bulk, name)), name
    T, Q = T0 + n, oracle_mod.quantized_len(T0 + n, R, G)
    live = [t % (R + G) for t in range(Q, T)]  # ring slots that hold window tokens
    if sink:
        live.append(R + G)  # the first token's fp16 row
    for name in ("k_res", "v_res"):
        assert np.array_equal(getattr(stream, name)[:, :, live], getattr(bulk, name)[:, :, live]), name
    assert np.array_equal(oracle_mod.decode(cfg, stream, q, 0.1), oracle_mod.decode(cfg, bulk, q, 0.1))


def test_paged_config_and_table_validation(oracle_mod):
    base = dict(B=1, Hq=2, Hkv=1, kb=2, vb=2, G=32, R=32, had=0, cap=512)
    k, v, q = _inputs(1, 300, 1, 2, 93)
    for P in (64, 96, 384):  # not a multiple of 128, or not dividing the capacity
        cfg = _cfg(oracle_mod, **base)
        cfg.page_tokens, cfg.num_pages = P, 8
        with pytest.raises(ValueError):
            oracle_mod.quantize_prefill(cfg, oracle_mod.Cache(cfg, page_table=np.zeros((1, 1, 512 // P), np.int32)),
                                        k, v, [300])
    cfg = _cfg(oracle_mod, **base)
    cfg.page_tokens, cfg.num_pages = 128, 4
    for bad in (-1, 4):  # a page the quantized part (256 tokens: pages 0 and 1) needs, outside the pool
        table = np.array([[[0, bad, -1, -1]]], np.int32)
        with pytest.raises(ValueError):
            oracle_mod.quantize_prefill(cfg, oracle_mod.Cache(cfg, page_table=table), k, v, [300])
    # pages past the quantized part may stay unassigned
    oracle_mod.quantize_prefill(cfg, oracle_mod.Cache(cfg, page_table=np.array([[[2, 0, -1, -1]]], np.int32)),
                                k, v, [300])
