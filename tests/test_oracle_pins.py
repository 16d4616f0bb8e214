"""Pins of the float64 oracle against facts fixed by the pages and by mathematics.

None of these re-type the oracle's own formula: each compares it with a value the
pages print, a closed form, a different formulation (dense matrices, complex
numbers, numpy.convolve, brute-force loops), or an invariant.
"""
import math

import numpy as np
import pytest
import torch

import kva_inputs as KI
from oracle import kva_ref as R
from tests.conftest import read_golden

RNG = np.random.default_rng(12345)


# ---------------------------------------------------------------- geometry
def test_param_counts_match_model_card():
    """Printed millions = bias-free linear counts rounded up to 1M (all six)."""
    for variant, part, printed in read_golden("param_counts.txt"):
        geom = KI.GEOMETRIES[variant]
        pc = geom.param_counts()
        if part == "total":
            # the printed r3 total counts the drafter heads, r2 has none
            n = pc["total"]
        else:
            n = pc[part]
        assert math.ceil(n / 1e6) == int(printed), (variant, part, n)
    # the opening paragraph's '1.24B' for r3
    assert round(KI.R3.param_counts()["total"] / 1e9, 2) == 1.24


def test_param_counts_reject_other_shapes():
    """The pin discriminates: extra matrices or another FFN width break it."""
    g = KI.R3
    bad = KI.with_changes(g, ffn=g.ffn + 256)
    assert math.ceil(bad.param_counts()["trunk"] / 1e6) != 363
    # an attention block with separate q/k/v of width 2d (not d) breaks it too
    d, H, F = g.d_model, g.hidden, g.ffn
    wrong = H * d + 3 * (6 * d * d + 3 * d * F)
    assert math.ceil(wrong / 1e6) != 363


def test_mixer_widths_match_model_card():
    gw = dict((k, int(v)) for k, v in read_golden("mixer_widths.txt"))
    for geom in (KI.R2, KI.R3):
        assert 2 * geom.gdn_n_k * geom.gdn_d_k + geom.gdn_n_v * geom.gdn_d_v == gw["gdn_qkv"]
        assert geom.gdn_n_v == gw["gdn_a"] == gw["gdn_b"]
        assert geom.attn_n_kv * geom.attn_d_h == gw["attn_k"] == gw["attn_v"]
        assert geom.n_gdn == gw["late_gdn_layers"]
        assert geom.n_attn == gw["late_attn_layers"]
        assert geom.n_mix == 24 * (10240 + 96) + 8 * 2048


# ---------------------------------------------------------------- RoPE
def test_rope_low_frequency_angles_match_mla_card():
    """theta = 1e7 and omega_i = theta^(-2i/64) reproduce 3.4 / 2.1 / 1.2 degrees."""
    inv = R.rope_inv_freq(64, 1.0e7)
    for pair, deg in read_golden("rope_low_freq_angles.txt"):
        got = math.degrees(inv[int(pair)] * 131072)
        assert abs(got - float(deg)) < 0.05, (pair, got, deg)
        got2 = math.degrees(inv[int(pair)] * 131000)
        assert abs(got2 - float(deg)) < 0.05
    # other common bases do not fit the printed values
    for theta in (1.0e6, 5.0e6, 1.0e4):
        inv = R.rope_inv_freq(64, theta)
        assert abs(math.degrees(inv[31] * 131072) - 1.2) > 0.1


def test_rope_equals_complex_rotation():
    """Each pair (i, i+r/2) as a complex number is multiplied by e^{i p w_i}."""
    T, n, d, r, theta = 7, 3, 256, 64, 1.0e7
    x = RNG.standard_normal((T, n, d))
    pos = np.array([0, 1, 5, 1023, 4096, 32767, 131071])
    y = R.rope_apply(x, pos, r, theta)
    w = theta ** (-np.arange(r // 2) * 2.0 / r)
    z = x[:, :, : r // 2] + 1j * x[:, :, r // 2 : r]
    zr = z * np.exp(1j * pos[:, None, None] * w[None, None, :])
    np.testing.assert_allclose(y[:, :, : r // 2], zr.real, atol=1e-12)
    np.testing.assert_allclose(y[:, :, r // 2 : r], zr.imag, atol=1e-12)
    np.testing.assert_array_equal(y[:, :, r:], x[:, :, r:])


def test_rope_dot_product_depends_on_relative_position_only():
    d, r, theta = 256, 64, 1.0e7
    q = RNG.standard_normal((1, 1, d))
    k = RNG.standard_normal((1, 1, d))
    vals = []
    for m, nn in [(10, 3), (1010, 1003), (32767, 32760)]:
        qm = R.rope_apply(q, np.array([m]), r, theta)
        kn = R.rope_apply(k, np.array([nn]), r, theta)
        vals.append(float(np.sum(qm * kn)))
    np.testing.assert_allclose(vals, vals[0], rtol=1e-10)
    # and it does depend on the offset
    qm = R.rope_apply(q, np.array([10]), r, theta)
    kn = R.rope_apply(k, np.array([9]), r, theta)
    assert abs(float(np.sum(qm * kn)) - vals[0]) > 1e-6


# ---------------------------------------------------------------- norms, gates
def test_rmsnorm_closed_forms():
    x = RNG.standard_normal((5, 512)) * 30
    y = R.rmsnorm(x, np.ones(512))
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), math.sqrt(512), rtol=1e-8)
    np.testing.assert_allclose(R.rmsnorm(3.5 * x, np.ones(512)), y, rtol=1e-8)
    g = RNG.uniform(0.5, 1.5, 512)
    np.testing.assert_allclose(R.rmsnorm(x, g), y * g, rtol=1e-12)
    # eps sits inside the root: a zero row stays zero, a tiny row is damped
    assert np.all(R.rmsnorm(np.zeros((1, 8)), np.ones(8)) == 0)
    small = np.full((1, 4), 1e-3)
    np.testing.assert_allclose(R.rmsnorm(small, np.ones(4)), 1e-3 / math.sqrt(1e-6 + 1e-6))


def test_l2norm_unit_rows():
    x = RNG.standard_normal((9, 4 * 64)) * 7
    y = R.l2norm_heads(x, 4, 64)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), 1.0, rtol=1e-9)
    xs = x.reshape(9, 4, 64)
    np.testing.assert_allclose(y * np.linalg.norm(xs, axis=-1, keepdims=True), xs, rtol=1e-8)


def test_gates_special_values():
    A_log = np.array([0.0, 1.0, 2.7])
    dt = np.array([0.3, -0.2, 0.0])
    a = -dt[None, :]                          # a + dt_bias = 0 -> softplus = ln 2
    b = np.zeros((1, 3))
    g, beta = R.gdn_gates(a, b, A_log, dt)
    np.testing.assert_allclose(g[0], -np.exp(A_log) * math.log(2.0), rtol=1e-14)
    np.testing.assert_allclose(beta[0], 0.5)
    big = np.array([[50.0, -50.0, 700.0]])
    g2, beta2 = R.gdn_gates(big, big, A_log, np.zeros(3))
    np.testing.assert_allclose(g2[0, 0], -50.0, rtol=1e-14)          # softplus(x) -> x
    np.testing.assert_allclose(g2[0, 1], -math.exp(1.0) * math.exp(-50.0), rtol=1e-10)
    assert np.all(np.isfinite(g2)) and np.all(g2 <= 0)
    np.testing.assert_allclose(beta2[0], [1.0, math.exp(-50.0), 1.0], rtol=1e-12)


# ---------------------------------------------------------------- conv
def test_conv_matches_numpy_convolve_per_channel():
    T, C, K = 37, 6, 4
    X = RNG.standard_normal((T, C))
    tail = RNG.standard_normal((K - 1, C))
    w = RNG.standard_normal((C, K))
    Z, new_tail = R.causal_conv_silu(X, tail, w)
    for c in range(C):
        ext = np.concatenate([tail[:, c], X[:, c]])
        # np.convolve flips its kernel: tap K-1 must meet the current token
        full = np.convolve(ext, w[c, ::-1], mode="valid")
        np.testing.assert_allclose(Z[:, c], full / (1 + np.exp(-full)), rtol=1e-12)
    np.testing.assert_array_equal(new_tail, X[-(K - 1):])


def test_conv_delta_weights_are_shifts():
    T, C, K = 10, 3, 4
    X = RNG.standard_normal((T, C))
    tail = RNG.standard_normal((K - 1, C))
    ext = np.concatenate([tail, X])
    for lag in range(K):
        w = np.zeros((C, K))
        w[:, K - 1 - lag] = 1.0                         # picks the token `lag` steps back
        Z, _ = R.causal_conv_silu(X, tail, w)
        pre = ext[K - 1 - lag:K - 1 - lag + T]
        np.testing.assert_allclose(Z, pre / (1 + np.exp(-pre)), rtol=1e-12)


def test_conv_tail_carry_equals_one_long_sequence():
    T1, T2, C, K = 2, 9, 5, 4                          # T1 < K-1: tail mixes old and new
    X = RNG.standard_normal((T1 + T2, C))
    tail = RNG.standard_normal((K - 1, C))
    w = RNG.standard_normal((C, K))
    Z, t_end = R.causal_conv_silu(X, tail, w)
    Za, ta = R.causal_conv_silu(X[:T1], tail, w)
    Zb, tb = R.causal_conv_silu(X[T1:], ta, w)
    np.testing.assert_allclose(np.concatenate([Za, Zb]), Z, rtol=1e-13)
    np.testing.assert_array_equal(tb, t_end)
    np.testing.assert_array_equal(ta, np.concatenate([tail[T1:], X[:T1]]))


# ---------------------------------------------------------------- scan
def _rand_scan(T, n_k, n_v, d_k, d_v, seed=0, beta_lo=0.0):
    r = np.random.default_rng(seed)
    k = r.standard_normal((T, n_k, d_k))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = r.standard_normal((T, n_v, d_v))
    g = -r.uniform(0.0, 2.0, (T, n_v))
    beta = r.uniform(beta_lo, 1.0, (T, n_v))
    S0 = r.standard_normal((n_v, d_v, d_k)) * 0.3
    return S0, k, v, g, beta


def test_scan_matches_dense_matrix_brute_force():
    """The stated recurrence with explicit d_k x d_k matrices, GQA map h // 2."""
    S0, k, v, g, beta = _rand_scan(11, 2, 4, 5, 3, seed=1)
    got = R.delta_scan_sequential(S0, k, v, g, beta)
    for h in range(4):
        S = S0[h].copy()
        kh = h // 2
        for t in range(11):
            kt = k[t, kh][:, None]
            A = math.exp(g[t, h]) * (np.eye(5) - beta[t, h] * (kt @ kt.T))
            S = S @ A + beta[t, h] * (v[t, h][:, None] @ kt.T)
        np.testing.assert_allclose(got[h], S, rtol=1e-12, atol=1e-12)


def test_scan_beta_zero_is_pure_decay_and_identity():
    S0, k, v, g, beta = _rand_scan(13, 2, 4, 6, 6, seed=2)
    z = np.zeros_like(beta)
    got = R.delta_scan_sequential(S0, k, v, g, z)
    np.testing.assert_allclose(got, np.exp(g.sum(0))[:, None, None] * S0, rtol=1e-12)
    got0 = R.delta_scan_sequential(S0, k, v, np.zeros_like(g), z)
    np.testing.assert_array_equal(got0, S0)
    for fn in (R.delta_scan_chunked,):
        np.testing.assert_allclose(fn(S0, k, v, g, z, chunk=4),
                                   np.exp(g.sum(0))[:, None, None] * S0, rtol=1e-12)
        np.testing.assert_allclose(fn(S0, k, v, np.zeros_like(g), z, chunk=4), S0,
                                   rtol=1e-13, atol=1e-15)


def test_scan_delta_rule_write_property():
    """beta = 1, unit k, no decay: the new state maps k_t exactly to v_t."""
    S0, k, v, g, beta = _rand_scan(6, 1, 2, 8, 4, seed=3)
    for t in range(1, 7):
        S = R.delta_scan_sequential(S0, k[:t], v[:t], np.zeros((t, 2)), np.ones((t, 2)))
        for h in range(2):
            np.testing.assert_allclose(S[h] @ k[t - 1, 0], v[t - 1, h], atol=1e-12)


def test_scan_orthonormal_keys_closed_form():
    """Orthonormal keys, beta = 1, g = 0: S_T = S0 (I - sum k k^T) + sum v k^T."""
    d = 8
    Qm, _ = np.linalg.qr(RNG.standard_normal((d, d)))
    T = 5
    k = Qm[:, :T].T[:, None, :]                       # [T, 1, d]
    v = RNG.standard_normal((T, 1, 3))
    S0 = RNG.standard_normal((1, 3, d))
    got = R.delta_scan_sequential(S0, k, v, np.zeros((T, 1)), np.ones((T, 1)))
    P = sum(np.outer(k[t, 0], k[t, 0]) for t in range(T))
    want = S0[0] @ (np.eye(d) - P) + sum(np.outer(v[t, 0], k[t, 0]) for t in range(T))
    np.testing.assert_allclose(got[0], want, atol=1e-12)


@pytest.mark.parametrize("T,chunk", [(1, 64), (63, 64), (64, 64), (150, 64), (130, 16)])
def test_scan_chunked_equals_sequential(T, chunk):
    S0, k, v, g, beta = _rand_scan(T, 2, 6, 16, 8, seed=T)
    g[: T // 3] *= 20.0                              # strong decay, e^(sum g) underflows
    a = R.delta_scan_sequential(S0, k, v, g, beta)
    b = R.delta_scan_chunked(S0, k, v, g, beta, chunk=chunk)
    np.testing.assert_allclose(b, a, rtol=1e-11, atol=1e-12)


# ---------------------------------------------------------------- attention
def test_attention_equal_keys_gives_prefix_mean():
    T, n, d = 12, 2, 16
    Q = RNG.standard_normal((T, n, d))
    K = np.broadcast_to(RNG.standard_normal((1, n, d)), (T, n, d)).copy()
    V = RNG.standard_normal((T, n, d))
    O = R.block_causal_attention(Q, K, V, 0)
    want = np.cumsum(V, axis=0) / np.arange(1, T + 1)[:, None, None]
    np.testing.assert_allclose(O, want, rtol=1e-12)
    O4 = R.block_causal_attention(Q, K, V, 4)        # blocks of 4: mean restarts
    for t in range(T):
        b0 = (t // 4) * 4
        np.testing.assert_allclose(O4[t], V[b0:t + 1].mean(0), rtol=1e-12)


def test_attention_brute_force_loops():
    T, n, d = 9, 2, 8
    Q, K, V = (RNG.standard_normal((T, n, d)) for _ in range(3))
    O = R.block_causal_attention(Q, K, V, 4)
    for h in range(n):
        for i in range(T):
            js = [j for j in range(T) if j <= i and j // 4 == i // 4]
            s = [sum(Q[i, h, e] * K[j, h, e] for e in range(d)) / math.sqrt(d) for j in js]
            m = max(s)
            p = [math.exp(x - m) for x in s]
            tot = sum(p)
            o = [sum(p[a] * V[js[a], h, e] for a in range(len(js))) / tot for e in range(d)]
            np.testing.assert_allclose(O[i, h], o, rtol=1e-10)


def test_block_causal_equals_causal_within_window():
    T, n, d = 40, 2, 8
    Q, K, V = (RNG.standard_normal((T, n, d)) for _ in range(3))
    np.testing.assert_allclose(R.block_causal_attention(Q, K, V, 64),
                               R.block_causal_attention(Q, K, V, 0), rtol=1e-13)
    np.testing.assert_allclose(R.block_causal_attention(Q, K, V, 40),
                               R.block_causal_attention(Q, K, V, 0), rtol=1e-13)
    # blocks do not see each other: block 2 alone gives the same rows
    Ob = R.block_causal_attention(Q, K, V, 16)
    np.testing.assert_allclose(Ob[16:32], R.block_causal_attention(Q[16:32], K[16:32], V[16:32], 0),
                               rtol=1e-13)


# ---------------------------------------------------------------- projector
def _tiny_f64(seed=7, random_gains=True):
    geom = KI.TINY
    W = R.weights_to_f64(KI.make_projector_weights(geom, seed, random_gains=random_gains))
    return geom, W


def test_projector_with_zero_output_projections_is_linear_chain():
    geom, W = _tiny_f64()
    for b in W["blocks"]:
        b["Wo"] = np.zeros_like(b["Wo"])
        b["Wd"] = np.zeros_like(b["Wd"])
    res = RNG.standard_normal((16, geom.hidden))
    Y = R.projector(res, W, geom)
    h = R.rmsnorm(res, W["g_in"]) @ W["W_in"].T
    np.testing.assert_allclose(Y, R.rmsnorm(h, W["g_out"]) @ W["W_heads"].T, rtol=1e-10)


def test_projector_block_single_token_attends_to_itself():
    # one token: the softmax over a single key is 1, so attention returns V whatever Q and K
    # are, and the block is x + Wo Wv u + Wd (silu(Wg u') * Wu u') written per vector
    geom, W = _tiny_f64()
    blk = W["blocks"][1]
    x = RNG.standard_normal(geom.d_model) * 3
    u = x / math.sqrt(np.mean(x * x) + R.EPS) * blk["g_attn"]
    x1 = x + blk["Wo"] @ (blk["Wv"] @ u)
    u2 = x1 / math.sqrt(np.mean(x1 * x1) + R.EPS) * blk["g_ffn"]
    gate, up = blk["Wg"] @ u2, blk["Wu"] @ u2
    want = x1 + blk["Wd"] @ (gate / (1.0 + np.exp(-gate)) * up)
    got = R.projector_block(x[None], blk, geom.n_heads, geom.head_dim, geom.window)[0]
    np.testing.assert_allclose(got, want, rtol=1e-10, atol=1e-12)
    other = dict(blk, Wq=blk["Wq"] * -7.0, Wk=RNG.standard_normal(blk["Wk"].shape))
    got2 = R.projector_block(x[None], other, geom.n_heads, geom.head_dim, geom.window)[0]
    np.testing.assert_allclose(got2, want, rtol=1e-10, atol=1e-12)


def _block_on_one_token(x, blk):
    # a block on a single token, written per vector: the lone key gets softmax weight 1,
    # so attention returns Wv u; then the SwiGLU FFN on the renormalised stream
    u = x / math.sqrt(np.mean(x * x) + R.EPS) * blk["g_attn"]
    x1 = x + blk["Wo"] @ (blk["Wv"] @ u)
    u2 = x1 / math.sqrt(np.mean(x1 * x1) + R.EPS) * blk["g_ffn"]
    gate, up = blk["Wg"] @ u2, blk["Wu"] @ u2
    return x1 + blk["Wd"] @ (gate / (1.0 + np.exp(-gate)) * up)


def test_projector_chains_its_distinct_blocks_in_order_on_one_token():
    # [KVA] architecture: RMSNorm -> Linear{H -> d} -> block 0 -> block 1 -> block 2 -> RMSNorm
    # -> heads.  On one token every block has the closed form above; the blocks are drawn
    # independently, so repeating one block or running them in another order changes z.
    geom, W = _tiny_f64()
    assert len(W["blocks"]) == 3
    for i in range(3):
        for j in range(i + 1, 3):
            assert np.abs(W["blocks"][i]["Wd"] - W["blocks"][j]["Wd"]).max() > 1e-3
    r = RNG.standard_normal(geom.hidden) * 2
    x = W["W_in"] @ (r / math.sqrt(np.mean(r * r) + R.EPS) * W["g_in"])
    for blk in W["blocks"]:
        x = _block_on_one_token(x, blk)
    z = x / math.sqrt(np.mean(x * x) + R.EPS) * W["g_out"]
    got_z = R.projector_trunk(r[None], W, geom)[0]
    np.testing.assert_allclose(got_z, z, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(R.projector(r[None], W, geom)[0], W["W_heads"] @ z,
                               rtol=1e-10, atol=1e-12)
    # the order matters at this scale: reversed blocks give a different z
    xr = W["W_in"] @ (r / math.sqrt(np.mean(r * r) + R.EPS) * W["g_in"])
    for blk in W["blocks"][::-1]:
        xr = _block_on_one_token(xr, blk)
    zr = xr / math.sqrt(np.mean(xr * xr) + R.EPS) * W["g_out"]
    assert np.abs(zr - z).max() > 1e-6


def test_projector_is_causal_and_position_free():
    geom, W = _tiny_f64()
    res = RNG.standard_normal((20, geom.hidden))
    Y = R.projector(res, W, geom)
    res2 = res.copy()
    res2[12:] = RNG.standard_normal((8, geom.hidden))
    Y2 = R.projector(res2, W, geom)
    np.testing.assert_allclose(Y2[:12], Y[:12], rtol=1e-12)
    assert np.abs(Y2[12:] - Y[12:]).max() > 1e-3
    # ubatch-local: the first k tokens alone give the same rows
    np.testing.assert_allclose(R.projector(res[:7], W, geom), Y[:7], rtol=1e-12)


def test_concatenated_heads_equal_per_layer_heads():
    geom, W = _tiny_f64()
    z = RNG.standard_normal((5, geom.d_model))
    Y = R.projector_heads(z, W["W_heads"])
    for li, off in enumerate(geom.layer_offsets):
        w = geom.layer_width(li)
        Wl = W["W_heads"][off:off + w]
        np.testing.assert_allclose(Y[:, off:off + w],
                                   np.einsum("td,nd->tn", z, Wl), rtol=1e-12, atol=1e-13)


# ---------------------------------------------------------------- cache, carry
def test_paged_slots_are_a_bijection_through_the_page_table():
    pt = KI.make_page_table(1, 8, seed=3).numpy()[0]
    s = R.kv_slots(0, 8 * 16, pt, 16)
    assert sorted(s.tolist()) == list(range(8 * 16))
    for p in (0, 15, 16, 100, 127):
        assert s[p] == pt[p // 16] * 16 + p % 16


def test_update_states_two_ubatches_equal_one():
    geom = KI.TINY
    P = {k: v.double().numpy() for k, v in KI.make_layer_params(geom, 5, random_k_gain=True).items()}
    st = KI.make_states(geom, 1, 6, std=0.1)
    S0 = st["state"][0].double().numpy()
    tail0 = st["conv_tail"][0].double().numpy()
    T = 50
    Y = RNG.standard_normal((T, geom.n_mix))
    mk = lambda: ([np.full((geom.attn_n_kv, 64, geom.attn_d_h), -7.0)],
                  [np.full((geom.attn_n_kv, 64, geom.attn_d_h), -7.0)])
    k1, v1 = mk()
    S1, t1 = R.update_states(Y, geom, P, S0, tail0, k1, v1, 3)
    k2, v2 = mk()
    Sa, ta = R.update_states(Y[:2], geom, P, S0, tail0, k2, v2, 3)
    Sb, tb = R.update_states(Y[2:], geom, P, Sa, ta, k2, v2, 5, scan="chunked")
    np.testing.assert_allclose(Sb, S1, rtol=1e-10, atol=1e-12)
    np.testing.assert_array_equal(tb, t1)
    np.testing.assert_allclose(k2[0], k1[0], rtol=1e-12)
    np.testing.assert_allclose(v2[0], v1[0], rtol=1e-12)
    # rows outside 3..52 untouched
    assert np.all(k1[0][:, :3] == -7.0) and np.all(k1[0][:, 53:] == -7.0)
    # rotation keeps the k-norm of each head: |k| = sqrt(d) * gain-weighted rms
    K = k1[0][:, 3:53].transpose(1, 0, 2)
    Yk = Y[:, geom.layer_offsets[2]:geom.layer_offsets[2] + geom.attn_n_kv * geom.attn_d_h]
    kn = R.rmsnorm(Yk.reshape(T, geom.attn_n_kv, geom.attn_d_h), P["k_norm_g"][0])
    np.testing.assert_allclose(np.linalg.norm(K, axis=-1), np.linalg.norm(kn, axis=-1), rtol=1e-12)
    np.testing.assert_array_equal(K[:, :, geom.rope_dims:], kn[:, :, geom.rope_dims:])


# ------------------------------------------------------------------ q8_0 cache with rotation
@pytest.mark.parametrize("n", [1, 2, 8, 128, 256])
def test_hadamard_rotation_is_the_normalised_sylvester_matrix(n):
    # scipy's hadamard(n) is the Sylvester-ordered matrix of +-1 entries
    from scipy.linalg import hadamard
    x = RNG.standard_normal((5, n))
    np.testing.assert_allclose(R.hadamard_rotate(x), x @ hadamard(n).T / math.sqrt(n), rtol=0,
                               atol=1e-12)


def test_hadamard_rotation_keeps_dot_products_and_undoes_itself():
    # attention scores are unchanged when both q and k are rotated; H / sqrt(n) is its own inverse
    q, k = RNG.standard_normal((7, 256)), RNG.standard_normal((7, 256))
    Hq, Hk = R.hadamard_rotate(q), R.hadamard_rotate(k)
    np.testing.assert_allclose((Hq * Hk).sum(-1), (q * k).sum(-1), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(R.hadamard_rotate(Hq), q, rtol=0, atol=1e-12)


def test_q8_0_closed_form_block():
    # amax 127 -> d = 1 exactly, codes are the nearest integers (x_j = j - 16 + 1/4 -> j - 16)
    x = np.arange(32, dtype=np.float64) - 16 + 0.25
    x[31] = 127.0
    want = np.concatenate([np.arange(31) - 16, [127]]).astype(np.int8)
    d, c = R.q8_0_quantize(x[None])
    assert d.dtype == np.float16 and float(d[0, 0]) == 1.0
    np.testing.assert_array_equal(c[0], want)
    # a power-of-two scale moves d only
    d2, c2 = R.q8_0_quantize(x[None] * 2.0 ** -5)
    assert float(d2[0, 0]) == 2.0 ** -5
    np.testing.assert_array_equal(c2, c)
    np.testing.assert_array_equal(R.q8_0_dequantize(d2, c2)[0], want * 2.0 ** -5)
    # an all-zero block: zero scale, zero codes
    dz, cz = R.q8_0_quantize(np.zeros((1, 64)))
    assert np.all(dz == 0) and np.all(cz == 0)


def test_q8_0_error_bound_and_full_scale_code():
    x = RNG.standard_normal((50, 256)) * np.exp(RNG.standard_normal((50, 1)))
    d, c = R.q8_0_quantize(x)
    xf = x.astype(np.float32).astype(np.float64).reshape(50, 8, 32)
    d32 = np.max(np.abs(xf), axis=-1) / 127.0
    back = R.q8_0_dequantize(d, c).reshape(50, 8, 32)
    # half a step of the float32 scale plus the fp16 storage of the scale for the largest code
    bound = d32 / 2 * (1 + 1e-6) + 127 * np.abs(d32 - d.astype(np.float64))
    assert np.all(np.abs(back - xf) <= bound[..., None])
    # every non-zero block uses the full code range at its largest element
    assert np.all(np.max(np.abs(c.reshape(50, 8, 32).astype(np.int32)), axis=-1) == 127)


def test_q8_0_rounds_half_away_from_zero_exactly():
    # d = 1: codes of values just below / at / above a half (float32 ties and near-ties)
    below = np.nextafter(np.float32(0.5), np.float32(0))
    x = np.zeros(32, dtype=np.float32)
    x[:6] = [below, 0.5, 1.5, -0.5, -below, 2.5]
    x[31] = 127.0
    _, c = R.q8_0_quantize(x[None])
    np.testing.assert_array_equal(c[0, :6], [0, 1, 2, -1, 0, 3])


# ------------------------------------------------------------------ q4_0 projector weights
def test_q4_0_closed_form_blocks():
    # values j - 8 then 7 - j: the first value of largest magnitude is -8, so d = -8 / -8 = 1
    # and every value is its own code minus 8; byte j packs code j (low) and 15 - j (high)
    x = np.concatenate([np.arange(16) - 8.0, 7.0 - np.arange(16)])
    d, c = R.q4_0_quantize(x[None])
    assert d.dtype == np.float16 and float(d[0, 0]) == 1.0
    np.testing.assert_array_equal(c[0], np.concatenate([np.arange(16), 15 - np.arange(16)]))
    packed = R.q4_0_pack(c)
    np.testing.assert_array_equal(packed[0], 240 - 15 * np.arange(16))
    np.testing.assert_array_equal(R.q4_0_unpack(packed), c)
    np.testing.assert_array_equal(R.q4_0_dequantize(d, c)[0], x)
    # times -1/4: the first largest value is now +2, so d = -1/4 and the codes stay
    d2, c2 = R.q4_0_quantize(x[None] * -0.25)
    assert float(d2[0, 0]) == -0.25
    np.testing.assert_array_equal(c2, c)
    np.testing.assert_array_equal(R.q4_0_dequantize(d2, c2)[0], x * -0.25)
    # the opposite extreme is clamped to code 15 (7 d), halves round up (x / d + 8.5, floor)
    y = np.zeros(32)
    y[:7] = [-8.0, 8.0, 0.5, -0.5, 1.5, -1.5, 2.25]
    y[7] = -2.75
    d3, c3 = R.q4_0_quantize(y[None])
    assert float(d3[0, 0]) == 1.0
    np.testing.assert_array_equal(c3[0, :9], [0, 15, 9, 8, 10, 7, 10, 5, 8])
    np.testing.assert_array_equal(R.q4_0_dequantize(d3, c3)[0, :3], [-8.0, 7.0, 1.0])
    np.testing.assert_array_equal(R.q4_0_pack(c3)[0, :3], [0x80, 0x8F, 0x89])
    # a tie in magnitude: the first one (+4) sets d = -1/2; the later -4 clamps to 7 d
    z = np.zeros(32)
    z[3], z[10], z[20] = 4.0, -4.0, 1.0
    d4, c4 = R.q4_0_quantize(z[None])
    assert float(d4[0, 0]) == -0.5
    np.testing.assert_array_equal(R.q4_0_dequantize(d4, c4)[0, [3, 10, 20]], [4.0, -3.5, 1.0])
    # an all-zero block: zero scale, code 8 (value 0)
    dz, cz = R.q4_0_quantize(np.zeros((1, 64)))
    assert np.all(dz == 0) and np.all(cz == 8)


def test_q4_0_error_bound_and_range():
    x = RNG.standard_normal((40, 256)) * np.exp(RNG.standard_normal((40, 1)))
    d, c = R.q4_0_quantize(x)
    assert c.dtype == np.uint8 and c.max() <= 15
    xf = x.astype(np.float32).astype(np.float64).reshape(40, 8, 32)
    first = np.argmax(np.abs(xf), axis=-1)[..., None]
    m = np.take_along_axis(xf, first, axis=-1)[..., 0]
    d32 = m / -8.0
    back = R.q4_0_dequantize(d, c).reshape(40, 8, 32)
    ratio = xf / d32[..., None]                      # in [-8, 8]
    store = 8 * np.abs(d32 - d.astype(np.float64))   # the fp16 scale, at most 8 steps away
    step = np.abs(d32)[..., None]
    # half a step inside the code range, up to a full step where code 15 is clamped
    bound = np.where(ratio <= 7.5, step / 2, step) * (1 + 1e-5) + store[..., None]
    assert np.all(np.abs(back - xf) <= bound)
    # the value that sets the scale comes back up to the scale's fp16 rounding
    mb = np.take_along_axis(back, first, axis=-1)[..., 0]
    assert np.all(np.abs(mb - m) <= store * (1 + 1e-9))
    np.testing.assert_array_equal(R.q4_0_unpack(R.q4_0_pack(c)), c)


# ---------------------------------------------------------------- exact last-token pass
def test_gdn_readout_returns_values_written_at_orthonormal_keys():
    # a state holding rank-1 writes v_j k_j^T at orthonormal keys returns v_j when read with
    # k_j; v head h belongs to key head h // (n_v / n_k)
    n_k, n_v, d = 2, 4, 8
    rng = np.random.default_rng(5)
    Q = [np.linalg.qr(rng.standard_normal((d, d)))[0] for _ in range(n_k)]   # columns: keys
    vals = rng.standard_normal((n_v, d, d))                                   # vals[h, j]: v_j
    S = np.stack([sum(np.outer(vals[h, j], Q[h // 2][:, j]) for j in range(d)) for h in range(n_v)])
    for j in range(d):
        q = np.stack([Q[kh][:, j] for kh in range(n_k)])
        np.testing.assert_allclose(R.gdn_readout(S, q), vals[:, j], rtol=1e-10, atol=1e-12)


def test_gated_rmsnorm_closed_form():
    o = np.array([[3.0, 4.0, 0.0, 0.0], [1.0, 1.0, 1.0, 1.0]])
    z = np.array([[0.0, 2.0, -1.0, 40.0], [1.0, -3.0, 0.5, 0.0]])
    w = np.array([1.0, 0.5, 2.0, 1.5])
    rms0 = math.sqrt(25.0 / 4.0 + R.EPS)
    rms1 = math.sqrt(1.0 + R.EPS)
    sil = lambda t: t / (1.0 + math.exp(-t))
    want = np.array([[3 / rms0 * 1.0 * sil(0.0), 4 / rms0 * 0.5 * sil(2.0), 0.0, 0.0],
                     [1 / rms1 * 1.0 * sil(1.0), 1 / rms1 * 0.5 * sil(-3.0), 1 / rms1 * 2.0 * sil(0.5), 0.0]])
    np.testing.assert_allclose(R.gated_rmsnorm(o, z, w), want, rtol=1e-12, atol=1e-15)


def _tiny_decode_layer(seed=3):
    geom = KI.TINY
    P = {k: v.double().numpy() for k, v in KI.make_layer_params(geom, seed).items()}
    L = {k: v.double().numpy() for k, v in KI.make_last_token_params(geom, seed + 1, random_gains=True).items()}
    st = KI.make_states(geom, 1, seed + 2, std=0.3)
    return geom, P, L, st["state"][0].double().numpy(), st["conv_tail"][0].double().numpy()


def test_gdn_decode_state_and_tail_equal_a_one_token_ubatch():
    # the decode's state update is the prefill's own update on a ubatch of one token
    geom, P, L, S0, tail0 = _tiny_decode_layer()
    x = RNG.standard_normal(geom.last_width(0))
    gw = geom.gdn_width
    o, S1, t1 = R.gdn_decode(x[:gw], x[gw:], tail0[0], S0[0], P["conv_w"][0], P["A_log"][0],
                             P["dt_bias"][0], L["gdn_norm_w"][0], geom)
    one = KI.with_changes(geom, layer_types=(KI.GDN,))
    Pone = {"conv_w": P["conv_w"][:1], "A_log": P["A_log"][:1], "dt_bias": P["dt_bias"][:1],
            "k_norm_g": np.zeros((0, geom.attn_d_h))}
    S_u, t_u = R.update_states(x[None, :gw], one, Pone, S0[:1], tail0[:1], [], [], 0)
    np.testing.assert_allclose(S1, S_u[0], rtol=1e-12, atol=1e-14)
    np.testing.assert_array_equal(t1, t_u[0])
    assert o.shape == (geom.gdn_n_v * geom.gdn_d_v,)


def test_gdn_decode_reads_the_value_it_just_wrote():
    # q = k (same inputs, tail rows and conv taps on the q and k channels), beta -> 1 and
    # g -> 0: the delta rule writes v at k, so the read returns the token's own v after conv
    # and SiLU, and the output is the gated RMSNorm of that v
    geom, P, L, S0, tail0 = _tiny_decode_layer(seed=9)
    nk = geom.gdn_n_k * geom.gdn_d_k
    nv, dv = geom.gdn_n_v, geom.gdn_d_v
    C = geom.gdn_conv_ch
    x = RNG.standard_normal(geom.last_width(0))
    x[:nk] = x[nk:2 * nk]                                  # q inputs = k inputs
    x[C + nv:C + 2 * nv] = 60.0                            # b: beta = sigmoid(60) = 1 - 9e-27
    A_log = np.full(nv, -80.0)                             # g = -exp(-80) softplus(.) ~ -2e-35
    tail = tail0[0].copy()
    tail[:, :nk] = tail[:, nk:2 * nk]
    w = P["conv_w"][0].copy()
    w[:nk] = w[nk:2 * nk]
    gw = geom.gdn_width
    o, S1, _ = R.gdn_decode(x[:gw], x[gw:], tail, S0[0], w, A_log, P["dt_bias"][0],
                            L["gdn_norm_w"][0], geom)
    ext = np.concatenate([tail, x[None, :C]], axis=0)
    conv = sum(ext[j] * w[:, j] for j in range(4))
    act = conv / (1.0 + np.exp(-conv))
    v = act[2 * nk:].reshape(nv, dv)
    k = act[nk:2 * nk].reshape(geom.gdn_n_k, -1)
    k = k / np.sqrt(np.sum(k * k, axis=1, keepdims=True) + R.EPS)
    # with q = k, beta = 1, g = 0 the read is S1 k = (1 - n) S0 k + n v, n = |k|^2 (1 up to
    # the eps inside the L2 norm)
    kv = k[np.arange(nv) // (nv // geom.gdn_n_k)]
    n = np.sum(kv * kv, axis=1, keepdims=True)
    v = (1.0 - n) * np.einsum("hij,hj->hi", S0[0], kv) + n * v
    z = x[gw:].reshape(nv, dv)
    want = v / np.sqrt(np.mean(v * v, axis=1, keepdims=True) + R.EPS) * L["gdn_norm_w"][0] \
        * (z / (1.0 + np.exp(-z)))
    np.testing.assert_allclose(o.reshape(nv, dv), want, rtol=1e-9, atol=1e-12)


def _attn_setup(seed, pos, n_q=6, n_kv=2, d=32, rope=16):
    geom = KI.with_changes(KI.TINY, attn_n_kv=n_kv, attn_d_h=d, rope_dims=rope, attn_n_q=n_q)
    rng = np.random.default_rng(seed)
    kc = rng.standard_normal((n_kv, pos + 4, d))
    vc = rng.standard_normal((n_kv, pos + 4, d))
    x = rng.standard_normal(geom.last_width(2))
    kg = rng.uniform(0.5, 1.5, d)
    qg = rng.uniform(0.5, 1.5, d)
    return geom, kc, vc, x, kg, qg


def test_attn_decode_first_token_returns_its_value_times_the_gate():
    geom, kc, vc, x, kg, qg = _attn_setup(1, 0)
    o = R.attn_decode(x, kg, qg, kc, vc, 0, geom).reshape(6, 32)
    w = geom.attn_width
    v = x[w // 2:w].reshape(2, 32)
    gate = x[w + 6 * 32:].reshape(6, 32)
    for h in range(6):
        np.testing.assert_allclose(o[h], v[h // 3] / (1.0 + np.exp(-gate[h])), rtol=1e-12)


def test_attn_decode_brute_force_loops():
    # explicit loops: 2 x 2 rotations of the pairs (i, i + r/2), softmax over rows 0..pos,
    # query head h on KV head h // 3
    pos = 9
    geom, kc, vc, x, kg, qg = _attn_setup(2, pos)
    kc0, vc0 = kc.copy(), vc.copy()
    o = R.attn_decode(x, kg, qg, kc, vc, pos, geom).reshape(6, 32)
    d, r, w = 32, 16, geom.attn_width

    def norm_rot(vec, g, p):
        y = vec / math.sqrt(sum(t * t for t in vec) / d + R.EPS) * g
        out = y.copy()
        for i in range(r // 2):
            a = p * geom.rope_theta ** (-2.0 * i / r)
            out[i] = y[i] * math.cos(a) - y[i + r // 2] * math.sin(a)
            out[i + r // 2] = y[i + r // 2] * math.cos(a) + y[i] * math.sin(a)
        return out

    knew = [norm_rot(x[hh * d:(hh + 1) * d], kg, pos) for hh in range(2)]
    vnew = [x[w // 2 + hh * d:w // 2 + (hh + 1) * d] for hh in range(2)]
    for hh in range(2):
        np.testing.assert_allclose(kc[hh, pos], knew[hh], rtol=1e-12)      # written in place
        np.testing.assert_array_equal(vc[hh, pos], vnew[hh])
        np.testing.assert_array_equal(kc[hh, :pos], kc0[hh, :pos])         # nothing else moved
    for h in range(6):
        q = norm_rot(x[w + h * d:w + (h + 1) * d], qg, pos)
        hh = h // 3
        scores = [sum(q[i] * (knew[hh][i] if j == pos else kc0[hh, j, i]) for i in range(d)) / math.sqrt(d)
                  for j in range(pos + 1)]
        m = max(scores)
        e = [math.exp(s - m) for s in scores]
        want = sum(e[j] / sum(e) * (vnew[hh] if j == pos else vc0[hh, j]) for j in range(pos + 1))
        gate = x[w + 6 * d + h * d:w + 6 * d + (h + 1) * d]
        np.testing.assert_allclose(o[h], want / (1.0 + np.exp(-gate)), rtol=1e-10, atol=1e-12)


def test_attn_decode_depends_on_relative_positions_only():
    # cache rows written by the prefill's own k path at positions j = 0..pos-1; the score of
    # row j is <R_pos q, R_j k_j> = Re sum_i conj(q_i) k_i e^{i (j - pos) w_i} over the
    # rotated pairs (as complex numbers q_i + i q_(i+r/2)) plus the plain dot product of the
    # other dims: only j - pos enters
    pos = 7
    geom, _, _, x, kg, qg = _attn_setup(3, pos)
    d, r, w = 32, 16, geom.attn_width
    raw = np.random.default_rng(4).standard_normal((pos, w))
    kc = np.zeros((2, pos + 2, d))
    vc = np.zeros_like(kc)
    Kx, Vx = R.attn_kv(raw, kg, 0, geom)
    kc[:, :pos] = Kx.transpose(1, 0, 2)
    vc[:, :pos] = Vx.transpose(1, 0, 2)
    o = R.attn_decode(x, kg, qg, kc, vc, pos, geom).reshape(6, d)
    omega = geom.rope_theta ** (-2.0 * np.arange(r // 2) / r)
    rows = np.concatenate([raw, x[None, :w]], axis=0)                # unrotated k of rows 0..pos
    kn = rows[:, :w // 2].reshape(pos + 1, 2, d)
    kn = kn / np.sqrt(np.mean(kn * kn, axis=-1, keepdims=True) + R.EPS) * kg
    vv = rows[:, w // 2:].reshape(pos + 1, 2, d)
    for h in range(6):
        q = x[w + h * d:w + (h + 1) * d]
        q = q / math.sqrt(np.mean(q * q) + R.EPS) * qg
        qc = q[:r // 2] + 1j * q[r // 2:r]
        kk = kn[:, h // 3]
        kcx = kk[:, :r // 2] + 1j * kk[:, r // 2:r]
        rel = np.arange(pos + 1)[:, None] - pos
        sc = (np.real(np.sum(np.conj(qc)[None] * kcx * np.exp(1j * rel * omega[None]), axis=1))
              + kk[:, r:] @ q[r:]) / math.sqrt(d)
        p = np.exp(sc - sc.max())
        want = (p / p.sum()) @ vv[:, h // 3]
        gate = x[w + 6 * d + h * d:w + 6 * d + (h + 1) * d]
        np.testing.assert_allclose(o[h], want / (1.0 + np.exp(-gate)), rtol=1e-9, atol=1e-12)


def test_attn_decode_paged_equals_contiguous():
    pos, ps = 20, 8
    geom, kc, vc, x, kg, qg = _attn_setup(5, pos)
    n_pages = 6
    pt = np.array([4, 0, 5])                               # rows 0..23 on pages 4, 0, 5
    kp = np.random.default_rng(6).standard_normal((n_pages, 2, ps, 32))
    vp = np.random.default_rng(7).standard_normal((n_pages, 2, ps, 32))
    for j in range(pos):
        kp[pt[j // ps], :, j % ps] = kc[:, j]
        vp[pt[j // ps], :, j % ps] = vc[:, j]
    o_c = R.attn_decode(x, kg, qg, kc, vc, pos, geom)
    o_p = R.attn_decode(x, kg, qg, kp, vp, pos, geom, page_table=pt, page_size=ps)
    np.testing.assert_allclose(o_p, o_c, rtol=1e-12)
    np.testing.assert_allclose(kp[pt[pos // ps], :, pos % ps], kc[:, pos], rtol=1e-12)
