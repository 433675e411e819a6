"""Pins for the CPU oracle's building blocks: closed forms, invariants and
library routines that the decoder definition reduces to in special cases.

None of these retypes the oracle's own formula: each expected value comes
from mathematics (a rotation of a unit vector, the softmax of one key, a
constant vector's norm) or from an independent library (torch)."""
import math

import numpy as np
import pytest
import torch

import oracle


def bf(x) -> np.ndarray:
    """fp values -> bf16 bits through torch (library rounding)."""
    t = torch.as_tensor(np.array(x, dtype=np.float64)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def f(bits) -> np.ndarray:
    return oracle.bf16_to_f32(np.asarray(bits, dtype=np.uint16)).astype(np.float64)


# ---------------------------------------------------------------- bf16 rounding

def test_bf16_rounding_matches_torch_everywhere():
    rng = np.random.default_rng(0)
    vals = np.concatenate([
        rng.standard_normal(100000).astype(np.float32) * 10.0 ** rng.integers(-40, 38, 100000),
        np.array([0.0, -0.0, np.inf, -np.inf, 1e-45, 3.4e38, -3.4e38, 1.17e-38], np.float32),
        # exact ties: 1 + 2^-8 (-> 1), 1 + 3*2^-8 (-> 1 + 2^-6): round half to even
        np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 2 + 2 ** -7], np.float32),
    ]).astype(np.float32)
    got = oracle.round_bf16(vals)
    ref = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)
    assert f(oracle.round_bf16(np.array([1 + 2 ** -8], np.float32)))[0] == 1.0
    assert f(oracle.round_bf16(np.array([1 + 3 * 2 ** -8], np.float32)))[0] == 1 + 2 ** -6
    nan = oracle.round_bf16(np.array([np.nan], np.float32))
    assert np.isnan(f(nan)[0])


def test_bf16_roundtrip_exact():
    b = np.arange(0, 65536, dtype=np.uint32).astype(np.uint16)
    fin = (b & 0x7F80) != 0x7F80  # exponent not all ones: neither inf nor NaN
    assert np.array_equal(oracle.round_bf16(oracle.bf16_to_f32(b))[fin], b[fin])


# ---------------------------------------------------------------- RMSNorm

F32_EPS = 2.0 ** -23


@pytest.mark.parametrize("c", [0.5, 3.0, -1.25, 0.0078125])
@pytest.mark.parametrize("n", [2, 512, 2048])
def test_rmsnorm_constant_vector_closed_form(c, n):
    """x = c*1  ->  y = c / sqrt(c^2 + eps) * w (mean of c^2 over any n is c^2)."""
    eps = 1e-5
    x = np.full(n, c, np.float32)
    rng = np.random.default_rng(n)
    w = bf(1 + 0.1 * rng.standard_normal(n))
    got = oracle.rmsnorm(x, w, eps).astype(np.float64)
    expect = c / math.sqrt(c * c + eps) * f(w)
    # fp32 sum of n equal squares, a root, a division and two products
    assert np.all(np.abs(got - expect) <= np.abs(expect) * (n + 8) * F32_EPS)


def test_rmsnorm_two_element_closed_form():
    # x = (3, 4): mean square 12.5
    got = oracle.rmsnorm(np.array([3.0, 4.0], np.float32), bf([1.0, 1.0]), 0.0).astype(np.float64)
    r = 1.0 / math.sqrt(12.5)
    assert np.allclose(got, [3 * r, 4 * r], rtol=4 * F32_EPS, atol=0)


def test_rmsnorm_power_of_two_scale_invariance():
    """With eps = 0, rms(4x) == rms(x) bit for bit (scaling by 4 is exact at every step)."""
    rng = np.random.default_rng(1)
    x = rng.standard_normal(2048).astype(np.float32)
    w = bf(1 + 0.1 * rng.standard_normal(2048))
    assert np.array_equal(oracle.rmsnorm(x, w, 0.0), oracle.rmsnorm(x * np.float32(4.0), w, 0.0))


def test_rmsnorm_against_torch_fp64():
    rng = np.random.default_rng(2)
    x = (rng.standard_normal(2048) * 0.3).astype(np.float32)
    w = bf(1 + 0.1 * rng.standard_normal(2048))
    xt = torch.from_numpy(x.astype(np.float64))
    ref = (xt * torch.rsqrt(xt.pow(2).mean() + 1e-5) * torch.from_numpy(f(w))).numpy()
    got = oracle.rmsnorm(x, w, 1e-5).astype(np.float64)
    assert np.max(np.abs(got - ref) / (np.abs(ref) + 1e-12)) <= 1e-5


# ---------------------------------------------------------------- RoPE

def test_rope_identity_at_position_zero():
    v = np.random.default_rng(3).standard_normal(64).astype(np.float32)
    assert np.array_equal(oracle.rope(v, 0, 500000.0), v)


@pytest.mark.parametrize("pos", [1, 7, 128, 8191])
def test_rope_unit_vector_closed_form(pos):
    """e_i rotates in the plane (i, i + d/2) by pos * theta^(-2i/d)."""
    d, theta = 64, 500000.0
    for i in (0, 5, 31):
        e = np.zeros(d, np.float32)
        e[i] = 1.0
        out = oracle.rope(e, pos, theta)
        ang = pos * theta ** (-2.0 * i / d)
        expect = np.zeros(d)
        expect[i], expect[i + d // 2] = math.cos(ang), math.sin(ang)
        assert np.allclose(out, expect, atol=1e-6)
        # the partner dimension rotates the other way round
        e2 = np.zeros(d, np.float32)
        e2[i + d // 2] = 1.0
        out2 = oracle.rope(e2, pos, theta)
        expect2 = np.zeros(d)
        expect2[i], expect2[i + d // 2] = -math.sin(ang), math.cos(ang)
        assert np.allclose(out2, expect2, atol=1e-6)


def test_rope_preserves_pair_norms_and_relative_positions():
    rng = np.random.default_rng(4)
    d, theta = 128, 500000.0
    q = rng.standard_normal(d).astype(np.float32)
    k = rng.standard_normal(d).astype(np.float32)
    for pos in (3, 100, 4000):
        r = oracle.rope(q, pos, theta)
        pairs_in = q[: d // 2] ** 2 + q[d // 2:] ** 2
        pairs_out = r[: d // 2] ** 2 + r[d // 2:] ** 2
        assert np.allclose(pairs_in, pairs_out, rtol=1e-5)
    # <R_m q, R_n k> depends only on m - n
    a = np.dot(oracle.rope(q, 10, theta), oracle.rope(k, 3, theta))
    b = np.dot(oracle.rope(q, 110, theta), oracle.rope(k, 103, theta))
    assert abs(a - b) <= 1e-4 * np.linalg.norm(q) * np.linalg.norm(k)


def test_rope_matches_transformers_rotate_half():
    """Library reduction: HF Llama's apply_rotary_pos_emb with the plain frequency form."""
    from transformers.models.llama.modeling_llama import apply_rotary_pos_emb
    d, theta, pos = 64, 500000.0, 37
    rng = np.random.default_rng(5)
    q = rng.standard_normal((1, 2, 1, d))
    inv = 1.0 / theta ** (np.arange(0, d, 2) / d)
    emb = np.concatenate([pos * inv, pos * inv])
    cos = torch.from_numpy(np.cos(emb))[None, None]
    sin = torch.from_numpy(np.sin(emb))[None, None]
    qt = torch.from_numpy(q)
    ref, _ = apply_rotary_pos_emb(qt, qt, cos, sin)
    for h in range(2):
        got = oracle.rope(q[0, h, 0].astype(np.float32), pos, theta)
        assert np.allclose(got, ref[0, h, 0].numpy(), atol=2e-6)


# ---------------------------------------------------------------- attention

def _rand_bf(rng, shape, scale=1.0):
    return bf(rng.standard_normal(shape) * scale)


def _rand_q(rng, shape, scale=1.0):
    return (rng.standard_normal(shape) * scale).astype(np.float32)


def test_attention_single_key_returns_v_exactly():
    rng = np.random.default_rng(6)
    q = _rand_q(rng, (8, 64))
    K = _rand_bf(rng, (2, 16, 64))
    V = _rand_bf(rng, (2, 16, 64))
    out = oracle.attention(q, K, V, n_keys=1)
    for h in range(8):
        assert np.array_equal(out[h].astype(np.float64), f(V[h // 4, 0]))


def test_attention_equal_keys_average_values():
    rng = np.random.default_rng(7)
    q = _rand_q(rng, (4, 64))
    K = np.repeat(_rand_bf(rng, (1, 1, 64)), 5, axis=1)
    V = _rand_bf(rng, (1, 5, 64))
    out = oracle.attention(q, K, V, n_keys=5).astype(np.float64)
    mean = f(V)[0].mean(axis=0)
    assert np.all(np.abs(out - mean) <= 16 * F32_EPS * (np.abs(f(V)[0]).max(axis=0) + 1e-30))


def test_attention_weights_sum_to_one():
    rng = np.random.default_rng(8)
    q = _rand_q(rng, (8, 64), 2.0)
    K = _rand_bf(rng, (2, 40, 64), 2.0)
    V = bf(np.ones((2, 40, 64)))
    out = oracle.attention(q, K, V, n_keys=37).astype(np.float64)
    assert np.all(np.abs(out - 1.0) <= 64 * F32_EPS)


def test_attention_two_keys_sigmoid_closed_form():
    """V rows (1,..) and (0,..): output = sigmoid(s1 - s2) with s = q.k / sqrt(d)."""
    d = 64
    q = np.zeros((1, d), np.float32)
    q[0, 0] = 2.0
    K = np.zeros((1, 2, d))
    K[0, 0, 0], K[0, 1, 0] = 3.0, -1.0          # q.k = 6 and -2
    V = np.zeros((1, 2, d))
    V[0, 0, :] = 1.0
    out = oracle.attention(q, bf(K), bf(V), 2).astype(np.float64)
    expect = 1.0 / (1.0 + math.exp(-(6.0 - (-2.0)) / math.sqrt(d)))
    assert np.allclose(out[0], expect, rtol=16 * F32_EPS, atol=0)


def test_attention_gqa_head_mapping():
    """KV head g's values constant c_g: query head h must return c_{h // group}."""
    rng = np.random.default_rng(9)
    nq, nkv = 32, 8
    q = _rand_q(rng, (nq, 64))
    K = _rand_bf(rng, (nkv, 20, 64))
    consts = np.arange(1, nkv + 1) * 0.25
    V = bf(np.broadcast_to(consts[:, None, None], (nkv, 20, 64)))
    out = oracle.attention(q, K, V, n_keys=20).astype(np.float64)
    for h in range(nq):
        assert np.all(np.abs(out[h] - consts[h // (nq // nkv)]) <= 32 * F32_EPS * consts[-1])


def test_attention_against_torch_sdpa_fp64():
    rng = np.random.default_rng(10)
    nq, nkv, d, n = 8, 2, 64, 57
    q = _rand_q(rng, (nq, d))
    K = _rand_bf(rng, (nkv, 64, d))
    V = _rand_bf(rng, (nkv, 64, d))
    got = oracle.attention(q, K, V, n_keys=n).astype(np.float64)
    qt = torch.from_numpy(q.astype(np.float64))[None, :, None, :]
    kt = torch.from_numpy(f(K)[:, :n])[None]
    vt = torch.from_numpy(f(V)[:, :n])[None]
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, enable_gqa=True)
    ref = ref[0, :, 0, :].numpy()
    assert np.max(np.abs(got - ref)) <= 1e-5 * np.max(np.abs(ref))


# ---------------------------------------------------------------- SiLU-gated product

def test_silu_mul_special_values():
    g = np.array([0.0, 30.0, -30.0, 1.0, -1.0], np.float32)
    u = np.array([5.0, 2.0, 7.0, 1.0, 1.0], np.float32)
    out = oracle.silu_mul(g, u).astype(np.float64)
    assert out[0] == 0.0
    assert out[1] == 60.0                       # 1 + e^-30 rounds to 1 in fp32
    assert abs(out[2]) < 1e-10
    assert abs(out[3] - 1.0 / (1.0 + math.exp(-1.0))) <= 4 * F32_EPS
    assert abs(out[4] + 1.0 / (1.0 + math.exp(1.0))) <= 4 * F32_EPS


def test_silu_mul_against_torch():
    rng = np.random.default_rng(11)
    g = (rng.standard_normal(4096) * 3).astype(np.float32)
    u = rng.standard_normal(4096).astype(np.float32)
    ref = (torch.nn.functional.silu(torch.from_numpy(g).double()) * torch.from_numpy(u).double()).numpy()
    got = oracle.silu_mul(g, u).astype(np.float64)
    assert np.all(np.abs(got - ref) <= np.abs(ref) * 8 * F32_EPS + 1e-30)


# ---------------------------------------------------------------- matvec

def test_matvec_within_fp32_bound_of_fp64():
    rng = np.random.default_rng(12)
    W = _rand_bf(rng, (300, 2048), 0.02)
    x = rng.standard_normal(2048).astype(np.float32)
    got = oracle.matvec(W, x).astype(np.float64)
    Wf, xf = f(W), x.astype(np.float64)
    ref = Wf @ xf
    bound = 2048 * 2.0 ** -24 * (np.abs(Wf) @ np.abs(xf)) * 1.01
    assert np.all(np.abs(got - ref) <= bound)
    # threads change nothing: rows are independent
    assert np.array_equal(oracle.matvec(W, x, threads=4), got.astype(np.float32))


def test_matvec_orientation():
    """A single 1 at W[r][c] picks x[c] into y[r] (catches a transposed operand)."""
    W = np.zeros((3, 5))
    W[2, 4] = 1.0
    x = np.array([1.0, 2.0, 3.0, 4.0, 5.0], np.float32)
    y = oracle.matvec(bf(W), x)
    assert list(y) == [0.0, 0.0, 5.0]


def test_argmax_lowest_index_on_ties():
    assert oracle.argmax(np.array([1.0, 3.0, 3.0, 2.0], np.float32)) == 1
    assert oracle.argmax(np.array([-5.0], np.float32)) == 0
