"""Plain float64 CPU oracle of the KVA prefill path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports this module:
only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its CPU-baseline
leg and ``--impl reference``) may call it.  It shares no code with the CUDA
library; the only common import is ``kva_inputs`` (seeded random inputs and
shape bookkeeping, no arithmetic of the method).

Every value is widened to float64 from the exact bf16 / fp32 inputs and all
arithmetic stays in float64.  The functions follow the pages in their order;
citations name the page and the section / table:

  [KVA]  "Qwen3.8-27B-KVA: late-layer KV approximation" model card
         (alimpfard/qwen3.8-27b-kv-approximation).
  [MLA]  "Qwen3.8-27B-MLA" model card (TelperionAI/Qwen3.8-27B-MLA).
  [GDR]  the gated delta rule as stated with the method:
         S_t = exp(g_t) S_{t-1} (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
         g = -exp(A_log) * softplus(a + dt_bias), beta = sigmoid(b),
         causal depthwise conv1d of kernel 4 + SiLU, L2-norm of q and k.

Readings where the pages are silent (each also stated where it is used):
  R1  RMSNorm: x / sqrt(mean(x^2) + 1e-6) * g, gain taken as given (effective).
  R2  projector blocks are pre-norm: x += Wo Attn(rms(x)); x += Wd(silu(Wg u) * Wu u),
      u = rms(x); no biases, no positional encoding, no QK-norm; scale 1/sqrt(128).
  R3  block-causal mask: key j visible to query i iff j <= i and
      floor(i / W) == floor(j / W), indices local to the ubatch; W = 0 means
      plain causal over the ubatch.
  R4  mixer columns per gated-DeltaNet layer: [q (n_k*d_k) | k (n_k*d_k) |
      v (n_v*d_v) | a (n_v) | b (n_v)], heads contiguous; per attention layer:
      [k (n_kv*d_h) | v (n_kv*d_h)].  Late layers are concatenated in layer
      order, drafter heads after them.
  R5  conv: no bias; tap conv_k-1 multiplies the current token; the carried
      tail holds the last conv_k-1 raw (pre-conv) rows, oldest first.
  R6  L2-norm: x / sqrt(sum(x^2) + 1e-6) per head.
  R7  v head h reads k head h // (n_v / n_k).
  R8  state layout [n_v, d_v, d_k] (S as written, v k^T).
  R9  RoPE on the first rope_dims dims of each KV head, NeoX half split:
      pair (i, i + rope_dims/2) rotated by (pos + t) * theta^(-2i/rope_dims).
  R10 attention-layer V is stored as predicted (no norm, no rotation).
  R11 the scan covers every token of the ubatch.
  R15 quantized KV cache ([KVA] "Other notes": with q8_0 caches the approximated
      K/V rows are rotated by the Hadamard transform the exact layers use): every
      d_h-dim K row (after k RMSNorm + RoPE) and V row is multiplied by the
      orthonormal Walsh-Hadamard matrix H_{d_h} / sqrt(d_h) (Sylvester order:
      H_1 = [1], H_2n = [[H_n, H_n], [H_n, -H_n]]), then stored as q8_0 blocks of 32
      consecutive values: scale d = max|x| / 127 kept in fp16, codes round(x / d)
      (half away from zero) as int8; a value reads back as fp16(d) * code.
  R16 q8_0 projector weights ([KVA] "Projector quantization"): each projector matrix
      W [N, K] as q8_0 blocks (R15's block rule) of 32 consecutive input values of a
      row; a weight is fp16(d) * code.
  R18 exact last-token pass ([KVA] "What the hell?"): when it follows, the approximated
      path covers tokens 0..T-2 of the ubatch (the projector is causal, so its predictions
      for them do not depend on token T-1) and the last token enters each late layer's
      state / cache through that layer's exact inputs, one layer at a time (each layer's
      inputs come from the base model's projections of the previous layer's output).
  R19 attention decode: q RMSNorm per head (gain q_norm) and RoPE at the token's
      position like k; scale 1/sqrt(d_h); the output multiplied by sigmoid(gate).
  R20 gated-DeltaNet decode readout: o_h = S_h q_hat (no extra scale; the gated RMSNorm
      that follows makes a constant factor irrelevant), then RMSNorm(o_h) * w * silu(z_h).
  R21 grouped queries: query head h reads KV head h // (n_q / n_kv) (24 over 4 in the
      base model, [MLA] "What this is").
  R17 q4_0 projector weights (the same section's q4_0 row): blocks of 32 consecutive
      input values of a row; m = the block's value of largest magnitude (the first one
      on a tie), d = m / -8 (so m itself is code 0), code q = min(15, floor(x / d + 8.5))
      decided in float32 (8 when d = 0); a weight is fp16(d) * (q - 8).  Stored as the
      fp16 scale and 16 bytes per block, byte j holding the code of value j in its low
      nibble and that of value j + 16 in its high nibble.

Pins: the building blocks here are checked in tests/test_oracle_pins.py against printed
values, closed forms, brute force or invariants; composed steps (gdn_prepare,
update_states) through their parts and the two-ubatches-equal-one invariant; the
projector as a whole (projector_trunk, projector) on one token, where every block has a
per-vector closed form, chained over three independently drawn blocks in order, and by
causality and ubatch locality at longer T; prefill_ubatch is projector followed by
update_states.  tests/test_oracle_mutants.py plants plausible mistakes that those pins
catch (among them a trunk that repeats its first block or runs the blocks in reverse).
The pages print no activations and no trained weights, so no pin compares against a
value of a trained projector.
"""
from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence

import numpy as np

EPS = 1.0e-6


# ---------------------------------------------------------------------------
# elementwise pieces
# ---------------------------------------------------------------------------
def rmsnorm(x: np.ndarray, g: np.ndarray, eps: float = EPS) -> np.ndarray:
    """RMSNorm over the last axis ([KVA] architecture: 'RMSNorm -> Linear'; R1)."""
    x = np.asarray(x, dtype=np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * np.asarray(g, dtype=np.float64)


def silu(x: np.ndarray) -> np.ndarray:
    """x * sigmoid(x)."""
    return x * sigmoid(x)


def sigmoid(x: np.ndarray) -> np.ndarray:
    """1 / (1 + e^-x), evaluated without overflow on either side."""
    x = np.asarray(x, dtype=np.float64)
    out = np.empty_like(x)
    pos = x >= 0
    out[pos] = 1.0 / (1.0 + np.exp(-x[pos]))
    ex = np.exp(x[~pos])
    out[~pos] = ex / (1.0 + ex)
    return out


def softplus(x: np.ndarray) -> np.ndarray:
    """log(1 + e^x), exact in float64 (log-add-exp form)."""
    return np.logaddexp(0.0, np.asarray(x, dtype=np.float64))


# ---------------------------------------------------------------------------
# projector ([KVA] architecture paragraph and table)
# ---------------------------------------------------------------------------
def attention_mask(T: int, window: int) -> np.ndarray:
    """Boolean [T, T] visibility: causal within `window`-token blocks (R3)."""
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    W = window if window > 0 else max(T, 1)
    return (j <= i) & ((i // W) == (j // W))


def block_causal_attention(Q: np.ndarray, K: np.ndarray, V: np.ndarray,
                           window: int) -> np.ndarray:
    """Softmax attention per head with the block-causal mask.

    [KVA] architecture table, attention row: r3 has 24 heads of 128 dims with
    the causal mask cut into 1024-token blocks, r2 20 heads of 128 dims with a
    plain causal mask.  Q, K, V: [T, n_h, dh].
    """
    T, n_h, dh = Q.shape
    mask = attention_mask(T, window)
    S = np.einsum("thd,shd->hts", Q, K) / math.sqrt(dh)
    S = np.where(mask[None], S, -np.inf)
    S = S - S.max(axis=-1, keepdims=True)
    P = np.exp(S)
    P = P / P.sum(axis=-1, keepdims=True)
    return np.einsum("hts,shd->thd", P, V)


def projector_block(x: np.ndarray, blk: Dict[str, np.ndarray], n_heads: int,
                    head_dim: int, window: int) -> np.ndarray:
    """One causal transformer block ([KVA] '3x[causal transformer block]'; R2)."""
    T = x.shape[0]
    u = rmsnorm(x, blk["g_attn"])
    Q = (u @ blk["Wq"].T).reshape(T, n_heads, head_dim)
    K = (u @ blk["Wk"].T).reshape(T, n_heads, head_dim)
    V = (u @ blk["Wv"].T).reshape(T, n_heads, head_dim)
    O = block_causal_attention(Q, K, V, window).reshape(T, n_heads * head_dim)
    x = x + O @ blk["Wo"].T
    u = rmsnorm(x, blk["g_ffn"])
    x = x + (silu(u @ blk["Wg"].T) * (u @ blk["Wu"].T)) @ blk["Wd"].T
    return x


def projector_trunk(residual: np.ndarray, W: Dict, geom) -> np.ndarray:
    """RMSNorm -> Linear{H -> d} -> blocks -> RMSNorm ([KVA] architecture).

    Returns z [T, d], the normalised input of the per-layer heads.
    """
    x = rmsnorm(residual, W["g_in"]) @ W["W_in"].T
    for blk in W["blocks"]:
        x = projector_block(x, blk, geom.n_heads, geom.head_dim, geom.window)
    return rmsnorm(x, W["g_out"])


def projector_heads(z: np.ndarray, W_heads: np.ndarray,
                    rows: Optional[slice] = None) -> np.ndarray:
    """A linear head for each late layer ([KVA] architecture), all concatenated
    along the output rows; rows selects a head block."""
    Wh = W_heads if rows is None else W_heads[rows]
    return z @ Wh.T


def projector(residual: np.ndarray, W: Dict, geom) -> np.ndarray:
    """Full projector: mixer inputs of every late layer (+ drafter) [T, n_total]."""
    return projector_heads(projector_trunk(residual, W, geom), W["W_heads"])


# ---------------------------------------------------------------------------
# gated-DeltaNet state update ([KVA] 'cheap state updates'; [GDR])
# ---------------------------------------------------------------------------
def split_gdn(Yl: np.ndarray, geom):
    """Split one layer's mixer columns into raw conv input X, a and b (R4)."""
    C = geom.gdn_conv_ch
    n_v = geom.gdn_n_v
    return Yl[:, :C], Yl[:, C:C + n_v], Yl[:, C + n_v:C + 2 * n_v]


def causal_conv_silu(X: np.ndarray, tail: np.ndarray, w: np.ndarray):
    """Causal depthwise conv1d + SiLU with a carried tail (R5).

    X [T, C] raw inputs, tail [K-1, C] previous raw rows (oldest first),
    w [C, K].  conv[t, c] = sum_j w[c, j] * Ext[t + j, c] with Ext = [tail; X].
    Returns (silu(conv) [T, C], new tail [K-1, C]).
    """
    K = w.shape[1]
    T = X.shape[0]
    ext = np.concatenate([tail, X], axis=0)
    conv = np.zeros_like(X, dtype=np.float64)
    for j in range(K):
        conv += ext[j:j + T] * w[:, j][None, :]
    return silu(conv), ext[ext.shape[0] - (K - 1):].copy()


def l2norm_heads(x: np.ndarray, n: int, d: int, eps: float = EPS) -> np.ndarray:
    """Per-head L2 normalisation (R6): [T, n*d] -> [T, n, d]."""
    x = x.reshape(x.shape[0], n, d)
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)


def gdn_gates(a: np.ndarray, b: np.ndarray, A_log: np.ndarray, dt_bias: np.ndarray):
    """g = -exp(A_log) * softplus(a + dt_bias), beta = sigmoid(b) ([GDR])."""
    g = -np.exp(A_log)[None, :] * softplus(a + dt_bias[None, :])
    return g, sigmoid(b)


def gdn_prepare(Yl: np.ndarray, tail: np.ndarray, conv_w: np.ndarray,
                A_log: np.ndarray, dt_bias: np.ndarray, geom):
    """conv + SiLU, L2 of q and k, gates for one gated-DeltaNet layer.

    Returns dict(q, k [T, n_k, d_k] unit rows; v [T, n_v, d_v]; g, beta [T, n_v];
    tail new conv tail).
    """
    X, a, b = split_gdn(Yl, geom)
    Z, new_tail = causal_conv_silu(X, tail, conv_w)
    nk, dk, nv, dv = geom.gdn_n_k, geom.gdn_d_k, geom.gdn_n_v, geom.gdn_d_v
    q = l2norm_heads(Z[:, :nk * dk], nk, dk)
    k = l2norm_heads(Z[:, nk * dk:2 * nk * dk], nk, dk)
    v = Z[:, 2 * nk * dk:].reshape(-1, nv, dv)
    g, beta = gdn_gates(a, b, A_log, dt_bias)
    return {"q": q, "k": k, "v": v, "g": g, "beta": beta, "tail": new_tail}


def delta_scan_sequential(S0: np.ndarray, k: np.ndarray, v: np.ndarray,
                          g: np.ndarray, beta: np.ndarray) -> np.ndarray:
    """Token-by-token gated delta rule ([GDR]) in its rank-1 form.

    S0 [n_v, d_v, d_k]; k [T, n_k, d_k]; v [T, n_v, d_v]; g, beta [T, n_v].
    Per token: S <- e^g (S - beta (S k) k^T) + beta v k^T, which equals
    e^g S (I - beta k k^T) + beta v k^T.  v head h reads k head h // (n_v/n_k) (R7).
    """
    S = np.array(S0, dtype=np.float64, copy=True)
    n_v = S.shape[0]
    grp = n_v // k.shape[1]
    kmap = np.arange(n_v) // grp
    for t in range(k.shape[0]):
        kt = k[t, kmap]                                   # [n_v, d_k]
        Sk = np.einsum("hij,hj->hi", S, kt)               # [n_v, d_v]
        bt = beta[t][:, None, None]
        S = np.exp(g[t])[:, None, None] * (S - bt * Sk[:, :, None] * kt[:, None, :]) \
            + bt * v[t][:, :, None] * kt[:, None, :]
    return S


def delta_scan_chunked(S0: np.ndarray, k: np.ndarray, v: np.ndarray,
                       g: np.ndarray, beta: np.ndarray, chunk: int = 64) -> np.ndarray:
    """The same recurrence in chunked (WY / UT-transform) form, float64.

    Within a chunk with local cumulative decay gam_t = sum_{s<=t} g_s:
        (I + L) U = diag(beta) V - diag(beta e^gam) K S0^T,
        L[t, s] = beta_t e^(gam_t - gam_s) k_t.k_s   for s < t (0 otherwise),
        S_end = e^gam_last S0 + sum_s e^(gam_last - gam_s) u_s k_s^T.
    Exponents are masked to s < t before exponentiation, so they are <= 0.
    Only the final state is produced (the path emits no per-token output).
    """
    S = np.array(S0, dtype=np.float64, copy=True)
    n_v = S.shape[0]
    grp = n_v // k.shape[1]
    kmap = np.arange(n_v) // grp
    T = k.shape[0]
    for c0 in range(0, T, chunk):
        c1 = min(T, c0 + chunk)
        C = c1 - c0
        for h in range(n_v):
            K = k[c0:c1, kmap[h]]                 # [C, d_k]
            V = v[c0:c1, h]                       # [C, d_v]
            gam = np.cumsum(g[c0:c1, h])          # [C]
            bt = beta[c0:c1, h]
            tri = np.tril(np.ones((C, C), dtype=bool), -1)
            diff = np.where(tri, gam[:, None] - gam[None, :], 0.0)
            L = np.where(tri, bt[:, None] * np.exp(diff) * (K @ K.T), 0.0)
            rhs = bt[:, None] * V - (bt * np.exp(gam))[:, None] * (K @ S[h].T)
            U = np.linalg.solve(np.eye(C) + L, rhs)      # [C, d_v]
            dec = np.exp(gam[-1] - gam)                   # [C]
            S[h] = np.exp(gam[-1]) * S[h] + (U * dec[:, None]).T @ K
    return S


# ---------------------------------------------------------------------------
# full-attention layers: k_norm + partial RoPE + KV cache ([KVA] table; [MLA])
# ---------------------------------------------------------------------------
def rope_inv_freq(rope_dims: int, theta: float) -> np.ndarray:
    """omega_i = theta^(-2i / rope_dims), i < rope_dims / 2 (R9; [MLA] 'What this is')."""
    i = np.arange(rope_dims // 2, dtype=np.float64)
    return theta ** (-2.0 * i / rope_dims)


def rope_apply(x: np.ndarray, positions: np.ndarray, rope_dims: int,
               theta: float) -> np.ndarray:
    """Rotate pairs (i, i + rope_dims/2) of x [T, n, d] by positions * omega_i.

    (x_i, x_j) -> (x_i cos - x_j sin, x_j cos + x_i sin); dims >= rope_dims kept.
    """
    x = np.array(x, dtype=np.float64, copy=True)
    half = rope_dims // 2
    ang = np.asarray(positions, dtype=np.float64)[:, None] * rope_inv_freq(rope_dims, theta)[None, :]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    xi = x[:, :, :half].copy()
    xj = x[:, :, half:rope_dims].copy()
    x[:, :, :half] = xi * c - xj * s
    x[:, :, half:rope_dims] = xj * c + xi * s
    return x


def attn_kv(Yl: np.ndarray, k_gain: np.ndarray, pos0: int, geom):
    """k RMSNorm per head + RoPE; v unchanged (R10).  Returns K, V [T, n_kv, d_h]."""
    T = Yl.shape[0]
    n, d = geom.attn_n_kv, geom.attn_d_h
    k = Yl[:, :n * d].reshape(T, n, d)
    v = Yl[:, n * d:2 * n * d].reshape(T, n, d)
    k = rmsnorm(k, k_gain)
    k = rope_apply(k, pos0 + np.arange(T), geom.rope_dims, geom.rope_theta)
    return k, v


def hadamard_rotate(x: np.ndarray) -> np.ndarray:
    """x [..., n] times the orthonormal Walsh-Hadamard matrix H_n / sqrt(n), n a power
    of two, Sylvester order (R15).  Written as the recursion that defines H_n: the
    transform of the two halves, then their sum and difference."""
    x = np.asarray(x, dtype=np.float64)
    n = x.shape[-1]
    assert n >= 1 and n & (n - 1) == 0

    def h(v):
        m = v.shape[-1]
        if m == 1:
            return v
        a, b = h(v[..., :m // 2]), h(v[..., m // 2:])
        return np.concatenate([a + b, a - b], axis=-1)

    return h(x) / math.sqrt(n)


def q8_0_quantize(x: np.ndarray):
    """q8_0 blocks of the last axis (a multiple of 32), decided in float32 (R15).

    Returns (d float16 [..., n/32], codes int8 [..., n]).  The rounding decision is
    taken in float32 on float32 inputs, the precision the cache writer computes in."""
    x = np.asarray(x, dtype=np.float32)
    blk = x.reshape(*x.shape[:-1], x.shape[-1] // 32, 32)
    amax = np.max(np.abs(blk), axis=-1)
    d = (amax / np.float32(127.0)).astype(np.float32)
    inv = np.where(d > 0, np.float32(1.0) / np.where(d > 0, d, np.float32(1.0)), np.float32(0.0))
    y = (blk * inv[..., None]).astype(np.float32)
    # half away from zero, decided exactly: y - trunc(y) has no rounding error in float32
    t = np.trunc(y)
    codes = t + np.sign(y) * (np.abs(y - t) >= np.float32(0.5))
    return d.astype(np.float16), codes.astype(np.int8).reshape(x.shape)


def q8_0_dequantize(d: np.ndarray, codes: np.ndarray) -> np.ndarray:
    """fp16(d) * code per block of 32, in float64 (R15)."""
    c = np.asarray(codes, dtype=np.float64)
    blk = c.reshape(*c.shape[:-1], c.shape[-1] // 32, 32)
    return (blk * np.asarray(d, dtype=np.float64)[..., None]).reshape(c.shape)


def q4_0_quantize(x: np.ndarray):
    """q4_0 blocks of the last axis (a multiple of 32), decided in float32 (R17).

    Returns (d float16 [..., n/32], codes uint8 [..., n] in 0..15, one per value)."""
    x = np.asarray(x, dtype=np.float32)
    blk = x.reshape(*x.shape[:-1], x.shape[-1] // 32, 32)
    first = np.argmax(np.abs(blk), axis=-1)[..., None]  # argmax keeps the first maximum
    m = np.take_along_axis(blk, first, axis=-1)[..., 0]
    d = (m / np.float32(-8.0)).astype(np.float32)
    inv = np.where(d != 0, np.float32(1.0) / np.where(d != 0, d, np.float32(1.0)), np.float32(0.0))
    y = (blk * inv[..., None] + np.float32(8.5)).astype(np.float32)
    codes = np.minimum(np.floor(y), 15.0)
    return d.astype(np.float16), codes.astype(np.uint8).reshape(x.shape)


def q4_0_dequantize(d: np.ndarray, codes: np.ndarray) -> np.ndarray:
    """fp16(d) * (code - 8) per block of 32, in float64 (R17); codes one per value."""
    c = np.asarray(codes, dtype=np.float64) - 8.0
    blk = c.reshape(*c.shape[:-1], c.shape[-1] // 32, 32)
    return (blk * np.asarray(d, dtype=np.float64)[..., None]).reshape(c.shape)


def q4_0_pack(codes: np.ndarray) -> np.ndarray:
    """Codes [..., n] (0..15) -> bytes [..., n/2]: per block of 32, byte j = code j in the
    low nibble, code j + 16 in the high nibble (R17)."""
    c = np.asarray(codes, dtype=np.uint8)
    blk = c.reshape(*c.shape[:-1], c.shape[-1] // 32, 2, 16)
    return (blk[..., 0, :] | (blk[..., 1, :] << 4)).reshape(*c.shape[:-1], c.shape[-1] // 2)


def q4_0_unpack(packed: np.ndarray) -> np.ndarray:
    """Bytes [..., n/2] -> codes [..., n], the inverse of q4_0_pack."""
    b = np.asarray(packed, dtype=np.uint8)
    blk = b.reshape(*b.shape[:-1], b.shape[-1] // 16, 16)
    out = np.stack([blk & 0x0F, blk >> 4], axis=-2)
    return out.reshape(*b.shape[:-1], b.shape[-1] * 2)


def kv_slots(pos0: int, T: int, page_table: Optional[np.ndarray] = None,
             page_size: int = 0) -> np.ndarray:
    """Cache row of each token: pos itself (contiguous) or page*page_size + offset."""
    p = pos0 + np.arange(T, dtype=np.int64)
    if page_table is None:
        return p
    return page_table[p // page_size].astype(np.int64) * page_size + p % page_size


# ---------------------------------------------------------------------------
# the whole path for one sequence
# ---------------------------------------------------------------------------
def update_states(Y: np.ndarray, geom, params: Dict[str, np.ndarray],
                  state: np.ndarray, tail: np.ndarray, kcache: List[np.ndarray],
                  vcache: List[np.ndarray], pos0: int,
                  page_table: Optional[np.ndarray] = None, page_size: int = 0,
                  scan: str = "sequential", debug: Optional[Dict] = None,
                  kv_rotate: bool = False):
    """Cheap state updates for one ubatch of one sequence ([KVA] 'Afterwards ...').

    Y [T, >= n_mix] mixer inputs.  state [n_gdn, n_v, d_v, d_k], tail
    [n_gdn, K-1, C] are returned updated (new arrays).  Caches are written in
    place: contiguous kcache[l] [n_kv, max_pos, d_h]; paged kcache[l]
    [n_pages, n_kv, page_size, d_h] addressed through page_table[pages].
    kv_rotate: the caches hold the Hadamard-rotated rows of a q8_0 cache (R15),
    before quantization (q8_0_quantize gives the stored form).
    """
    T = Y.shape[0]
    offs = geom.layer_offsets
    state = np.array(state, dtype=np.float64, copy=True)
    tail = np.array(tail, dtype=np.float64, copy=True)
    scan_fn = delta_scan_sequential if scan == "sequential" else delta_scan_chunked
    for gi, li in enumerate(geom.gdn_layers()):
        Yl = Y[:, offs[li]:offs[li] + geom.gdn_width]
        pr = gdn_prepare(Yl, tail[gi], params["conv_w"][gi], params["A_log"][gi],
                         params["dt_bias"][gi], geom)
        tail[gi] = pr["tail"]
        state[gi] = scan_fn(state[gi], pr["k"], pr["v"], pr["g"], pr["beta"])
        if debug is not None:
            debug.setdefault("gdn", []).append(pr)
    slots = kv_slots(pos0, T, page_table, page_size)
    for ai, li in enumerate(geom.attn_layers()):
        Yl = Y[:, offs[li]:offs[li] + geom.attn_width]
        K, V = attn_kv(Yl, params["k_norm_g"][ai], pos0, geom)
        if kv_rotate:
            K, V = hadamard_rotate(K), hadamard_rotate(V)
        if page_table is None:
            kcache[ai][:, slots, :] = K.transpose(1, 0, 2)
            vcache[ai][:, slots, :] = V.transpose(1, 0, 2)
        else:
            pg, off = slots // page_size, slots % page_size
            kcache[ai][pg, :, off, :] = K
            vcache[ai][pg, :, off, :] = V
        if debug is not None:
            debug.setdefault("attn", []).append((K, V))
    return state, tail


def prefill_ubatch(residual: np.ndarray, W: Dict, geom, params: Dict, state, tail,
                   kcache, vcache, pos0: int, scan: str = "sequential",
                   debug: Optional[Dict] = None, kv_rotate: bool = False):
    """Projector + state updates for one ubatch ([KVA] 'What the hell?').

    Returns (Y [T, n_total] mixer + drafter outputs, new state, new tail).
    """
    Y = projector(residual, W, geom)
    state, tail = update_states(Y, geom, params, state, tail, kcache, vcache, pos0,
                                scan=scan, debug=debug, kv_rotate=kv_rotate)
    return Y, state, tail


# ---------------------------------------------------------------------------
# exact last-token pass ([KVA] "What the hell?": after the cheap state updates the engine
# runs the last token of each ubatch through the late layers exactly, on top of the
# approximated context).  One late layer's token mixer, given that layer's exact inputs
# for the token (R18-R21); the projections around it belong to the base model.
# ---------------------------------------------------------------------------
def gdn_readout(S: np.ndarray, q: np.ndarray) -> np.ndarray:
    """o_h = S_h q_(h // (n_v / n_k)) per v head (R20): S [n_v, d_v, d_k], q [n_k, d_k]
    -> [n_v, d_v].  The state read with a query, as the rank-1 writes v k^T store v at k."""
    n_v = S.shape[0]
    kmap = np.arange(n_v) // (n_v // q.shape[0])
    return np.einsum("hij,hj->hi", S, q[kmap])


def gated_rmsnorm(o: np.ndarray, z: np.ndarray, w: np.ndarray, eps: float = EPS) -> np.ndarray:
    """Output gate of a gated-DeltaNet layer (R20): per v head RMSNorm(o_h) * w * silu(z_h).
    o, z [n_v, d_v], w [d_v]."""
    return rmsnorm(o, w, eps) * silu(np.asarray(z, dtype=np.float64))


def gdn_decode(x: np.ndarray, z: np.ndarray, tail: np.ndarray, S: np.ndarray,
               conv_w: np.ndarray, A_log: np.ndarray, dt_bias: np.ndarray,
               norm_w: np.ndarray, geom):
    """One token through a gated-DeltaNet layer's mixer (R18, R20).

    x [gdn_width] the token's exact [q | k | v | a | b] (R4), z [n_v * d_v] its output gate
    input.  The conv, norms, gates and state update are the prefill's own steps on a
    one-token ubatch; then the state is read with q and the gated RMSNorm applied.
    Returns (o [n_v * d_v], new state [n_v, d_v, d_k], new tail [K-1, C])."""
    pr = gdn_prepare(np.asarray(x, dtype=np.float64)[None], tail, conv_w, A_log, dt_bias, geom)
    S1 = delta_scan_sequential(S, pr["k"], pr["v"], pr["g"], pr["beta"])
    o = gdn_readout(S1, pr["q"][0])
    nv, dv = geom.gdn_n_v, geom.gdn_d_v
    return gated_rmsnorm(o, np.asarray(z, dtype=np.float64).reshape(nv, dv), norm_w).reshape(-1), \
        S1, pr["tail"]


def gqa_decode_attention(q: np.ndarray, Kc: np.ndarray, Vc: np.ndarray) -> np.ndarray:
    """Softmax attention of one query per head over n keys with grouped KV heads (R21):
    q [n_q, d], Kc, Vc [n, n_kv, d]; query head h reads KV head h // (n_q / n_kv); scale
    1/sqrt(d).  Returns [n_q, d]."""
    n_q, d = q.shape
    kmap = np.arange(n_q) // (n_q // Kc.shape[1])
    out = np.empty((n_q, d))
    for h in range(n_q):
        s = Kc[:, kmap[h]] @ q[h] / math.sqrt(d)
        p = np.exp(s - s.max())
        out[h] = (p / p.sum()) @ Vc[:, kmap[h]]
    return out


def attn_decode(x: np.ndarray, k_gain: np.ndarray, q_gain: np.ndarray, kcache: np.ndarray,
                vcache: np.ndarray, pos: int, geom, page_table: Optional[np.ndarray] = None,
                page_size: int = 0) -> np.ndarray:
    """One token at position pos through a full-attention layer's mixer (R18, R19, R21).

    x [last_width] the token's exact [k | v | q | gate]: k and v as in the mixer (k RMSNorm
    + RoPE, v as is) are written to the cache at pos (in place, like update_states); q gets
    its own RMSNorm (gain q_gain) and the same RoPE at pos; the query attends to the
    sequence's cache rows 0..pos (those the approximated path wrote and its own); the
    result is multiplied by sigmoid(gate).  Returns o [n_q * d_h]."""
    x = np.asarray(x, dtype=np.float64)
    n_kv, d, n_q = geom.attn_n_kv, geom.attn_d_h, geom.attn_n_q
    w = geom.attn_width
    Kn, Vn = attn_kv(x[None, :w], k_gain, pos, geom)
    slots = kv_slots(0, pos + 1, page_table, page_size)
    if page_table is None:
        kcache[:, pos, :] = Kn[0]
        vcache[:, pos, :] = Vn[0]
        Kc = kcache[:, slots, :].transpose(1, 0, 2)
        Vc = vcache[:, slots, :].transpose(1, 0, 2)
    else:
        kcache[slots[-1] // page_size, :, slots[-1] % page_size, :] = Kn[0]
        vcache[slots[-1] // page_size, :, slots[-1] % page_size, :] = Vn[0]
        Kc = kcache[slots // page_size, :, slots % page_size, :]
        Vc = vcache[slots // page_size, :, slots % page_size, :]
    q = rmsnorm(x[w:w + n_q * d].reshape(n_q, d), q_gain)
    q = rope_apply(q[None], np.array([pos]), geom.rope_dims, geom.rope_theta)[0]
    gate = x[w + n_q * d:w + 2 * n_q * d].reshape(n_q, d)
    return (gqa_decode_attention(q, Kc, Vc) * sigmoid(gate)).reshape(-1)


def weights_to_f64(W) -> Dict:
    """Widen a weight dict of torch tensors (bf16 / fp32) to float64 numpy."""
    def cv(t):
        return t.detach().to("cpu").double().numpy()
    out = {k: cv(v) for k, v in W.items() if k != "blocks"}
    out["blocks"] = [{k: cv(v) for k, v in b.items()} for b in W["blocks"]]
    return out
