"""Plant plausible mistakes in the oracle (on the CPU) and check a pin catches each.

Every mutant replaces one oracle function with a subtly wrong variant (a dropped
term, a wrong sign, a wrong index or orientation); the named pin tests must then
fail.  This shows the pins constrain the oracle rather than restate it.
"""
import math

import numpy as np
import pytest

from oracle import kva_ref as R
from tests import test_oracle_pins as P


def _rope_wrong_sign(x, positions, rope_dims, theta):
    return R_orig["rope_apply"](x, -np.asarray(positions), rope_dims, theta)


def _rope_interleaved(x, positions, rope_dims, theta):
    # rotates adjacent pairs (2i, 2i+1) instead of the half split
    x = np.array(x, dtype=np.float64, copy=True)
    ang = np.asarray(positions, dtype=np.float64)[:, None] * R.rope_inv_freq(rope_dims, theta)[None, :]
    c, s = np.cos(ang)[:, None, :], np.sin(ang)[:, None, :]
    xi, xj = x[:, :, 0:rope_dims:2].copy(), x[:, :, 1:rope_dims:2].copy()
    x[:, :, 0:rope_dims:2] = xi * c - xj * s
    x[:, :, 1:rope_dims:2] = xj * c + xi * s
    return x


def _inv_freq_wrong_theta(rope_dims, theta):
    return R_orig["rope_inv_freq"](rope_dims, 1.0e6)


def _conv_flipped(X, tail, w):
    return R_orig["causal_conv_silu"](X, tail, w[:, ::-1])


def _scan_decay_outside(S0, k, v, g, beta):
    # decay also applied to the write term: e^g (S(I - b k k^T) + b v k^T)
    S = np.array(S0, dtype=np.float64, copy=True)
    grp = S.shape[0] // k.shape[1]
    kmap = np.arange(S.shape[0]) // grp
    for t in range(k.shape[0]):
        kt = k[t, kmap]
        Sk = np.einsum("hij,hj->hi", S, kt)
        bt = beta[t][:, None, None]
        S = np.exp(g[t])[:, None, None] * (S - bt * Sk[:, :, None] * kt[:, None, :]
                                           + bt * v[t][:, :, None] * kt[:, None, :])
    return S


def _scan_gqa_modulo(S0, k, v, g, beta):
    # v head h reads k head h % n_k instead of h // (n_v / n_k)
    n_v, n_k = S0.shape[0], k.shape[1]
    perm = np.arange(n_v) % n_k
    kk = k[:, perm]                                   # expand to one k per v head
    return R_orig["delta_scan_sequential"](S0, kk, v, g, beta)


def _scan_variant_no_beta(S0, k, v, g, beta):
    S = np.array(S0, dtype=np.float64, copy=True)
    grp = S.shape[0] // k.shape[1]
    kmap = np.arange(S.shape[0]) // grp
    for t in range(k.shape[0]):
        kt = k[t, kmap]
        Sk = np.einsum("hij,hj->hi", S, kt)
        bt = beta[t][:, None, None]
        S = np.exp(g[t])[:, None, None] * (S - Sk[:, :, None] * kt[:, None, :]) \
            + bt * v[t][:, :, None] * kt[:, None, :]
    return S


def _attn_no_scale(Q, K, V, window):
    return R_orig["block_causal_attention"](Q * math.sqrt(Q.shape[-1]), K, V, window)


def _attn_mask_off_by_one(Q, K, V, window):
    T = Q.shape[0]
    S = np.einsum("thd,shd->hts", Q, K) / math.sqrt(Q.shape[-1])
    i, j = np.arange(T)[:, None], np.arange(T)[None, :]
    m = (j < i) | (i == 0) & (j == 0)
    S = np.where(m[None], S, -np.inf)
    S = S - S.max(-1, keepdims=True)
    Pm = np.exp(S)
    Pm /= Pm.sum(-1, keepdims=True)
    return np.einsum("hts,shd->thd", Pm, V)


def _rms_eps_outside(x, g, eps=R.EPS):
    x = np.asarray(x, dtype=np.float64)
    return x / (np.sqrt(np.mean(x * x, axis=-1, keepdims=True)) + eps) * g


def _gates_exp_not_softplus(a, b, A_log, dt_bias):
    return -np.exp(A_log)[None, :] * np.exp(a + dt_bias[None, :]), R.sigmoid(b)


def _chunked_no_decay_mask(S0, k, v, g, beta, chunk=64):
    # forgets the per-pair decay inside the chunk (uses e^gam_t only)
    S = np.array(S0, dtype=np.float64, copy=True)
    grp = S.shape[0] // k.shape[1]
    kmap = np.arange(S.shape[0]) // grp
    T = k.shape[0]
    for c0 in range(0, T, chunk):
        c1 = min(T, c0 + chunk)
        C = c1 - c0
        for h in range(S.shape[0]):
            K, V = k[c0:c1, kmap[h]], v[c0:c1, h]
            gam, bt = np.cumsum(g[c0:c1, h]), beta[c0:c1, h]
            L = np.tril(bt[:, None] * (K @ K.T), -1)
            rhs = bt[:, None] * V - (bt * np.exp(gam))[:, None] * (K @ S[h].T)
            U = np.linalg.solve(np.eye(C) + L, rhs)
            S[h] = np.exp(gam[-1]) * S[h] + (U * np.exp(gam[-1] - gam)[:, None]).T @ K
    return S


R_orig = {name: getattr(R, name) for name in (
    "rope_apply", "rope_inv_freq", "causal_conv_silu", "delta_scan_sequential",
    "block_causal_attention", "rmsnorm", "gdn_gates", "delta_scan_chunked", "hadamard_rotate",
    "q8_0_quantize", "projector_block", "projector_trunk", "gdn_readout", "gated_rmsnorm",
    "gdn_decode", "gqa_decode_attention", "attn_decode", "rope_apply")}

def _hadamard_unnormalised(x):
    # the +-1 Walsh-Hadamard matrix without the 1/sqrt(n) that makes it orthonormal
    return R_orig["hadamard_rotate"](x) * math.sqrt(np.asarray(x).shape[-1])


def _q8_0_truncating(x):
    # codes truncated toward zero instead of rounded
    d, _ = R_orig["q8_0_quantize"](x)
    x = np.asarray(x, dtype=np.float32)
    blk = x.reshape(*x.shape[:-1], x.shape[-1] // 32, 32)
    dd = d.astype(np.float32)[..., None]
    c = np.trunc(np.where(dd > 0, blk / np.where(dd > 0, dd, 1), 0)).astype(np.int8)
    return d, c.reshape(x.shape)


def _q4_0_pack_halves_swapped(codes):
    # value j in the high nibble and value j + 16 in the low one
    c = np.asarray(codes, dtype=np.uint8)
    blk = c.reshape(*c.shape[:-1], c.shape[-1] // 32, 2, 16)
    return ((blk[..., 0, :] << 4) | blk[..., 1, :]).reshape(*c.shape[:-1], c.shape[-1] // 2)


def _q4_0_positive_scale(x):
    # d = max|x| / 8 with the sign dropped: the codes of negative blocks flip
    x = np.asarray(x, dtype=np.float32)
    blk = x.reshape(*x.shape[:-1], x.shape[-1] // 32, 32)
    d = (np.max(np.abs(blk), axis=-1) / np.float32(8.0)).astype(np.float32)
    inv = np.where(d != 0, np.float32(1.0) / np.where(d != 0, d, np.float32(1.0)), np.float32(0.0))
    c = np.minimum(np.floor(blk * inv[..., None] + np.float32(8.5)), 15.0)
    return d.astype(np.float16), c.astype(np.uint8).reshape(x.shape)


def _block_gate_up_swapped(x, blk, n_heads, head_dim, window):
    # the SiLU applied to the up projection instead of the gate
    sw = dict(blk, Wg=blk["Wu"], Wu=blk["Wg"])
    return R_orig["projector_block"](x, sw, n_heads, head_dim, window)


def _block_values_from_keys(x, blk, n_heads, head_dim, window):
    # attention values taken from the key projection
    return R_orig["projector_block"](x, dict(blk, Wv=blk["Wk"]), n_heads, head_dim, window)


def _trunk_block0_repeated(residual, W, geom):
    # runs the first block as often as there are blocks
    return R_orig["projector_trunk"](residual, dict(W, blocks=[W["blocks"][0]] * len(W["blocks"])),
                                     geom)


def _trunk_blocks_reversed(residual, W, geom):
    # runs the blocks last to first
    return R_orig["projector_trunk"](residual, dict(W, blocks=list(W["blocks"])[::-1]), geom)


def _readout_gqa_modulo(S, q):
    # v head h reads query head h % n_k
    n_v = S.shape[0]
    return np.einsum("hij,hj->hi", S, q[np.arange(n_v) % q.shape[0]])


def _gated_norm_sigmoid(o, z, w, eps=R.EPS):
    # sigmoid(z) as the gate instead of silu(z)
    return R_orig["rmsnorm"](o, w, eps) * R.sigmoid(z)


def _decode_reads_old_state(x, z, tail, S, conv_w, A_log, dt_bias, norm_w, geom):
    # the readout taken from the state before the token's own write
    o_new, S1, t1 = R_orig["gdn_decode"](x, z, tail, S, conv_w, A_log, dt_bias, norm_w, geom)
    pr = R.gdn_prepare(np.asarray(x, dtype=np.float64)[None], tail, conv_w, A_log, dt_bias, geom)
    o = R_orig["gdn_readout"](np.asarray(S, dtype=np.float64), pr["q"][0])
    nv, dv = geom.gdn_n_v, geom.gdn_d_v
    return R_orig["gated_rmsnorm"](o, np.asarray(z).reshape(nv, dv), norm_w).reshape(-1), S1, t1


def _gqa_decode_modulo(q, Kc, Vc):
    # query head h reads KV head h % n_kv
    n_q = q.shape[0]
    perm = np.arange(n_q) % Kc.shape[1]
    out = np.empty_like(q)
    for h in range(n_q):
        s = Kc[:, perm[h]] @ q[h] / math.sqrt(q.shape[1])
        p = np.exp(s - s.max())
        out[h] = (p / p.sum()) @ Vc[:, perm[h]]
    return out


def _gqa_decode_no_scale(q, Kc, Vc):
    return R_orig["gqa_decode_attention"](q * math.sqrt(q.shape[1]), Kc, Vc)


def _attn_decode_gate_silu(x, k_gain, q_gain, kcache, vcache, pos, geom, page_table=None, page_size=0):
    # silu(gate) instead of sigmoid(gate): undo the sigmoid and apply silu
    o = R_orig["attn_decode"](x, k_gain, q_gain, kcache, vcache, pos, geom, page_table, page_size)
    w, nqd = geom.attn_width, geom.attn_n_q * geom.attn_d_h
    gate = np.asarray(x, dtype=np.float64)[w + nqd:w + 2 * nqd]
    return o * gate


def _attn_decode_q_unrotated(x, k_gain, q_gain, kcache, vcache, pos, geom, page_table=None, page_size=0):
    # RoPE applied to k only: rope_apply leaves the one-row q (the call with a single
    # position equal to pos and n_q heads) unrotated
    real = R_orig["rope_apply"]

    def rope_k_only(t, positions, rope_dims, theta):
        t = np.asarray(t)
        if t.shape[0] == 1 and t.shape[1] == geom.attn_n_q and geom.attn_n_q != geom.attn_n_kv:
            return np.array(t, dtype=np.float64, copy=True)
        return real(t, positions, rope_dims, theta)

    R.rope_apply = rope_k_only
    try:
        return R_orig["attn_decode"](x, k_gain, q_gain, kcache, vcache, pos, geom, page_table, page_size)
    finally:
        R.rope_apply = real


MUTANTS = [
    ("rope_apply", _rope_wrong_sign, [P.test_rope_equals_complex_rotation]),
    ("rope_apply", _rope_interleaved, [P.test_rope_equals_complex_rotation]),
    ("rope_inv_freq", _inv_freq_wrong_theta, [P.test_rope_low_frequency_angles_match_mla_card]),
    ("causal_conv_silu", _conv_flipped, [P.test_conv_matches_numpy_convolve_per_channel]),
    ("delta_scan_sequential", _scan_decay_outside, [P.test_scan_matches_dense_matrix_brute_force]),
    ("delta_scan_sequential", _scan_gqa_modulo, [P.test_scan_matches_dense_matrix_brute_force]),
    ("delta_scan_sequential", _scan_variant_no_beta, [P.test_scan_matches_dense_matrix_brute_force]),
    ("block_causal_attention", _attn_no_scale, [P.test_attention_brute_force_loops]),
    ("block_causal_attention", _attn_mask_off_by_one, [P.test_attention_equal_keys_gives_prefix_mean]),
    ("rmsnorm", _rms_eps_outside, [P.test_rmsnorm_closed_forms]),
    ("gdn_gates", _gates_exp_not_softplus, [P.test_gates_special_values]),
    ("delta_scan_chunked", _chunked_no_decay_mask, [lambda: P.test_scan_chunked_equals_sequential(150, 64)]),
    ("hadamard_rotate", _hadamard_unnormalised,
     [P.test_hadamard_rotation_keeps_dot_products_and_undoes_itself]),
    ("q8_0_quantize", _q8_0_truncating, [P.test_q8_0_closed_form_block]),
    ("q4_0_pack", _q4_0_pack_halves_swapped, [P.test_q4_0_closed_form_blocks]),
    ("projector_block", _block_gate_up_swapped, [P.test_projector_block_single_token_attends_to_itself]),
    ("projector_block", _block_values_from_keys, [P.test_projector_block_single_token_attends_to_itself]),
    ("q4_0_quantize", _q4_0_positive_scale, [P.test_q4_0_closed_form_blocks]),
    ("projector_trunk", _trunk_block0_repeated,
     [P.test_projector_chains_its_distinct_blocks_in_order_on_one_token]),
    ("projector_trunk", _trunk_blocks_reversed,
     [P.test_projector_chains_its_distinct_blocks_in_order_on_one_token]),
    ("gdn_readout", _readout_gqa_modulo, [P.test_gdn_readout_returns_values_written_at_orthonormal_keys]),
    ("gated_rmsnorm", _gated_norm_sigmoid, [P.test_gated_rmsnorm_closed_form]),
    ("gdn_decode", _decode_reads_old_state, [P.test_gdn_decode_reads_the_value_it_just_wrote]),
    ("gqa_decode_attention", _gqa_decode_modulo, [P.test_attn_decode_brute_force_loops]),
    ("gqa_decode_attention", _gqa_decode_no_scale, [P.test_attn_decode_brute_force_loops]),
    ("attn_decode", _attn_decode_gate_silu, [P.test_attn_decode_first_token_returns_its_value_times_the_gate]),
    ("attn_decode", _attn_decode_q_unrotated, [P.test_attn_decode_depends_on_relative_positions_only]),
]


@pytest.mark.parametrize("idx", range(len(MUTANTS)))
def test_planted_mistake_is_caught(idx, monkeypatch):
    name, bad, pins = MUTANTS[idx]
    monkeypatch.setattr(R, name, bad)
    caught = False
    for pin in pins:
        try:
            pin()
        except AssertionError:
            caught = True
    assert caught, f"no pin caught the mutant of {name} ({bad.__name__})"


def test_unmutated_oracle_passes_the_same_pins():
    for _, _, pins in MUTANTS:
        for pin in pins:
            pin()
