"""The exact last-token pass (kva_last_token_layer) against the float64 oracle.

One token of each sequence goes through one late layer's token mixer with that layer's
exact inputs: a gated-DeltaNet layer updates its state and conv tail with the token and
returns the gated-RMSNorm readout; an attention layer writes the token's K and V rows at
its position and returns the gated grouped-query attention over rows 0..pos.

Bit-exact: the conv tail (the old rows 1, 2 and the token's raw inputs), the V row (a copy
of the token's v in the cache format), every cache row other than the token's.
Within tolerance: the outputs (max |err| <= 2e-2 x RMS), the states (relative Frobenius
<= 1e-2), the K row (plus the storage rounding of the 16-bit cache).
"""
import numpy as np
import pytest
import torch

import kva_inputs as KI
from oracle import kva_ref as R
from tests.parity import BF16_ELEM, assert_rms_close, assert_state_close, f64

pytestmark = pytest.mark.gpu
SENT = -7.0


@pytest.fixture(scope="module")
def K():
    import hybrid_deltanet_attention_kva_b200 as K
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return K


def _stack(base, types):
    return KI.with_changes(base, layer_types=types, n_draft=0)


# a small r3-shaped stack: two gated-DeltaNet layers around an attention layer, so the
# layer's slice of the state, tail and parameters is exercised
R3S = _stack(KI.R3, (KI.GDN, KI.ATTN, KI.GDN))
TINYS = _stack(KI.TINY, (KI.GDN, KI.ATTN, KI.GDN))


@pytest.mark.parametrize("geom,dt,layer", [(TINYS, torch.bfloat16, 2), (R3S, torch.float16, 2),
                                           (R3S, torch.bfloat16, 0), (TINYS, torch.float16, 0)])
def test_gdn_layer_matches_oracle(K, geom, dt, layer):
    n_seq = 3
    P = KI.make_layer_params(geom, 31)
    L = KI.make_last_token_params(geom, 32, random_gains=True)
    st = KI.make_states(geom, n_seq, 33, std=0.1)
    x = KI.make_last_token_inputs(geom, layer, n_seq, 34).to(dt)
    S = st["state"].cuda()
    tail = st["conv_tail"].to(dt).cuda()
    nvdv = geom.gdn_n_v * geom.gdn_d_v
    out = torch.empty(n_seq, nvdv, device="cuda")
    h = K.kva_init(K.make_dims(geom, 16, n_seq, dtype=dt))
    try:
        Wt = K.Weights(layer={k: v.cuda() for k, v in P.items()})
        lp = K.LastParams(geom.attn_n_q, L["gdn_norm_w"].cuda(), L["q_norm_g"].cuda())
        K.kva_last_token_layer(h, layer, x.cuda(), [10, 200, 3000], Wt, lp, S, tail, None, out)
        torch.cuda.synchronize()
        assert K.kva_get_device_status(h) == 0
    finally:
        K.kva_free(h)
    gi = geom.gdn_layers().index(layer)
    gw = geom.gdn_width
    tail0 = st["conv_tail"].to(dt)
    for s in range(n_seq):
        xs = f64(x[s])
        o, S1, t1 = R.gdn_decode(xs[:gw], xs[gw:], f64(tail0[s, gi]), f64(st["state"][s, gi]),
                                 f64(P["conv_w"][gi]), f64(P["A_log"][gi]), f64(P["dt_bias"][gi]),
                                 f64(L["gdn_norm_w"][gi]), geom)
        assert_rms_close(out[s], o, what=f"output seq {s}")
        assert_state_close(S[s, gi], S1, what=f"state seq {s}")
        np.testing.assert_array_equal(f64(tail[s, gi]), t1)
        # the other gated-DeltaNet layer is untouched
        other = 1 - gi
        assert torch.equal(S[s, other].cpu(), st["state"][s, other])
        assert torch.equal(tail[s, other].cpu(), tail0[s, other])


def _filled_cache(K, geom, n_seq, max_pos, paged, seed, page_size=64):
    rng = torch.Generator().manual_seed(seed)
    nkv, dh = geom.attn_n_kv, geom.attn_d_h
    if paged:
        pps = (max_pos + page_size - 1) // page_size
        n_pages = n_seq * pps + 2
        pt = KI.make_page_table(n_seq, pps, seed + 1, n_pages=n_pages)
        shape = (n_pages, nkv, page_size, dh)
    else:
        pt = None
        shape = (n_seq, nkv, max_pos, dh)
    kc = [torch.randn(shape, generator=rng).to(torch.bfloat16) for _ in range(geom.n_attn)]
    vc = [torch.randn(shape, generator=rng).to(torch.bfloat16) for _ in range(geom.n_attn)]
    dk = [k.cuda() for k in kc]
    dv = [v.cuda() for v in vc]
    if paged:
        c = K.KvCache(dk, dv, page_table=pt.cuda(), page_size=page_size, n_pages=n_pages)
    else:
        c = K.KvCache(dk, dv, max_pos=max_pos)
    return c, kc, vc, dk, dv, pt


@pytest.mark.parametrize("geom,dt,paged,positions", [
    (TINYS, torch.bfloat16, False, [0, 77, 700]),
    (R3S, torch.float16, False, [0, 1, 5000]),
    (R3S, torch.bfloat16, True, [63, 64, 2100]),
    (TINYS, torch.float16, True, [5, 500, 129])])
def test_attention_layer_matches_oracle(K, geom, dt, paged, positions):
    n_seq, layer = len(positions), 1
    max_pos = max(positions) + 70
    P = KI.make_layer_params(geom, 41, random_k_gain=True)
    L = KI.make_last_token_params(geom, 42, random_gains=True)
    x = KI.make_last_token_inputs(geom, layer, n_seq, 43).to(dt)
    c, kc, vc, dk, dv, pt = _filled_cache(K, geom, n_seq, max_pos, paged, 44)
    nqd = geom.attn_n_q * geom.attn_d_h
    out = torch.empty(n_seq, nqd, dtype=dt, device="cuda")
    h = K.kva_init(K.make_dims(geom, 16, n_seq, dtype=dt))
    try:
        Wt = K.Weights(layer={k: v.cuda() for k, v in P.items()})
        lp = K.LastParams(geom.attn_n_q, L["gdn_norm_w"].cuda(), L["q_norm_g"].cuda())
        K.kva_last_token_layer(h, layer, x.cuda(), positions, Wt, lp, None, None, c, out)
        torch.cuda.synchronize()
        assert K.kva_get_device_status(h) == 0
    finally:
        K.kva_free(h)
    ok = f64(kc[0])
    ov = f64(vc[0])
    dh, nkv = geom.attn_d_h, geom.attn_n_kv
    for s, p in enumerate(positions):
        if paged:
            o = R.attn_decode(f64(x[s]), f64(P["k_norm_g"][0]), f64(L["q_norm_g"][0]), ok, ov, p, geom,
                              page_table=pt.numpy()[s], page_size=64)
        else:
            o = R.attn_decode(f64(x[s]), f64(P["k_norm_g"][0]), f64(L["q_norm_g"][0]), ok[s], ov[s], p,
                              geom)
        # the output of 16-bit attention: the storage rounding of q, K, V and P allowed as a
        # relative term (like the prefill attention's tests)
        assert_rms_close(out[s], o, what=f"output seq {s} pos {p}", elem=BF16_ELEM)
    gk, gv = f64(dk[0]), f64(dv[0])
    written = np.zeros(gk.shape, dtype=bool)
    for s, p in enumerate(positions):
        if paged:
            pg, r = pt[s, p // 64].item(), p % 64
            written[pg, :, r] = True
        else:
            written[s, :, p] = True
    # the token's rows: K within tolerance of the oracle's, V bit for bit the token's v
    assert_rms_close(gk[written], ok[written], what="K rows", elem=BF16_ELEM)
    for s, p in enumerate(positions):
        xv = f64(x[s, nkv * dh:2 * nkv * dh].to(torch.bfloat16)).reshape(nkv, dh)
        row = gv[pt[s, p // 64].item(), :, p % 64] if paged else gv[s, :, p]
        np.testing.assert_array_equal(row, xv)
    # nothing else moved
    np.testing.assert_array_equal(gk[~written], f64(kc[0])[~written])
    np.testing.assert_array_equal(gv[~written], f64(vc[0])[~written])


def test_attention_layer_at_32k_positions(K):
    """The longest cache of the long-prompt workload: the token at position 32767 reads 32768
    rows per KV head (many splits), r3 heads (24 query heads over 4 KV heads of 256)."""
    geom = _stack(KI.R3, (KI.ATTN,))
    positions = [32767]
    P = KI.make_layer_params(geom, 51)
    L = KI.make_last_token_params(geom, 52, random_gains=True)
    x = KI.make_last_token_inputs(geom, 0, 1, 53).to(torch.float16)
    c, kc, vc, dk, dv, _ = _filled_cache(K, geom, 1, 32768, False, 54)
    out = torch.empty(1, geom.attn_n_q * geom.attn_d_h, device="cuda")
    h = K.kva_init(K.make_dims(geom, 16, 1, dtype=torch.float16))
    try:
        Wt = K.Weights(layer={k: v.cuda() for k, v in P.items()})
        lp = K.LastParams(geom.attn_n_q, None, L["q_norm_g"].cuda())
        K.kva_last_token_layer(h, 0, x.cuda(), positions, Wt, lp, None, None, c, out)
        torch.cuda.synchronize()
        assert K.kva_get_device_status(h) == 0
    finally:
        K.kva_free(h)
    o = R.attn_decode(f64(x[0]), f64(P["k_norm_g"][0]), f64(L["q_norm_g"][0]), f64(kc[0][0]),
                      f64(vc[0][0]), 32767, geom)
    assert_rms_close(out[0], o, what="output at 32767", elem=BF16_ELEM)


def test_prefill_then_last_token_through_every_layer(K):
    """The pass as the engine runs it: kva_prefill_ubatch on tokens 0..T-2 of a ubatch, then
    the last token through every late layer in order, each with its exact inputs; states,
    conv tails, caches and every layer's output against the oracle doing the same."""
    geom = KI.TINY
    T = 100
    dt = torch.float16
    W = KI.make_projector_weights(geom, 61)
    W = {k: (v if k.startswith("g_") or k == "blocks" else v.to(dt)) for k, v in W.items()}
    W["blocks"] = [{k: (v if k.startswith("g_") else v.to(dt)) for k, v in b.items()} for b in W["blocks"]]
    P = KI.make_layer_params(geom, 62, random_k_gain=True)
    L = KI.make_last_token_params(geom, 63, random_gains=True)
    st = KI.make_states(geom, 1, 64, std=0.1)
    res = KI.make_residual(geom, T - 1, 65, dtype=torch.float32, n_outliers=0)
    xs = [KI.make_last_token_inputs(geom, li, 1, 66 + li).to(dt) for li in range(geom.n_late)]
    kc = [torch.full((1, geom.attn_n_kv, T, geom.attn_d_h), SENT, dtype=torch.bfloat16, device="cuda")]
    vc = [torch.full_like(kc[0], SENT)]
    S = st["state"][0].cuda()
    tail = st["conv_tail"][0].to(dt).cuda()
    outs = []
    h = K.kva_init(K.make_dims(geom, T, 1, dtype=dt))
    try:
        Wg = K.Weights(proj={"g_in": W["g_in"].cuda(), "W_in": W["W_in"].cuda(), "g_out": W["g_out"].cuda(),
                             "W_heads": W["W_heads"].cuda(),
                             "blocks": [{k: v.cuda() for k, v in b.items()} for b in W["blocks"]]},
                       layer={k: v.cuda() for k, v in P.items()})
        lp = K.LastParams(geom.attn_n_q, L["gdn_norm_w"].cuda(), L["q_norm_g"].cuda())
        cache = K.KvCache(kc, vc, max_pos=T)
        K.kva_prefill_ubatch(h, res.cuda(), Wg, S, tail, cache, 0)
        for li in range(geom.n_late):
            w = (geom.gdn_n_v * geom.gdn_d_v if geom.layer_types[li] == KI.GDN
                 else geom.attn_n_q * geom.attn_d_h)
            o = torch.empty(1, w, device="cuda")
            K.kva_last_token_layer(h, li, xs[li].cuda(), [T - 1], Wg, lp, S, tail, cache, o)
            outs.append(o)
        torch.cuda.synchronize()
        assert K.kva_get_device_status(h) == 0
    finally:
        K.kva_free(h)
    Wn = R.weights_to_f64(W)
    Pn = {k: f64(v) for k, v in P.items()}
    Ln = {k: f64(v) for k, v in L.items()}
    ko = [np.full((geom.attn_n_kv, T, geom.attn_d_h), SENT)]
    vo = [np.full_like(ko[0], SENT)]
    _, S_o, tail_o = R.prefill_ubatch(f64(res), Wn, geom, Pn, f64(st["state"][0]),
                                      f64(st["conv_tail"][0].to(dt)), ko, vo, 0)
    gw = geom.gdn_width
    gi = ai = 0
    for li in range(geom.n_late):
        x = f64(xs[li][0])
        if geom.layer_types[li] == KI.GDN:
            o, S_o[gi], tail_o[gi] = R.gdn_decode(x[:gw], x[gw:], tail_o[gi], S_o[gi], Pn["conv_w"][gi],
                                                  Pn["A_log"][gi], Pn["dt_bias"][gi], Ln["gdn_norm_w"][gi], geom)
            gi += 1
        else:
            o = R.attn_decode(x, Pn["k_norm_g"][ai], Ln["q_norm_g"][ai], ko[ai], vo[ai], T - 1, geom)
            ai += 1
        assert_rms_close(outs[li][0], o, what=f"layer {li} output", elem=BF16_ELEM)
    assert_state_close(S, S_o)
    assert_rms_close(tail, tail_o, what="conv tails")
    written = ko[0] != SENT
    gk = f64(kc[0][0])
    np.testing.assert_array_equal(gk == SENT, ~written)
    assert written[:, T - 1].all()
    assert_rms_close(gk[written], ko[0][written], what="K cache", elem=BF16_ELEM)
    assert_rms_close(f64(vc[0][0])[written], vo[0][written], what="V cache", elem=BF16_ELEM)


def test_last_token_rejects_bad_arguments(K):
    geom = TINYS
    h = K.kva_init(K.make_dims(geom, 16, 2, dtype=torch.bfloat16))
    try:
        P = KI.make_layer_params(geom, 1)
        Wt = K.Weights(layer={k: v.cuda() for k, v in P.items()})
        x = KI.make_last_token_inputs(geom, 1, 1, 2).cuda()
        out = torch.empty(1, geom.attn_n_q * geom.attn_d_h, dtype=torch.bfloat16, device="cuda")
        c, *_ = _filled_cache(K, geom, 1, 64, False, 3)
        L = KI.make_last_token_params(geom, 4)
        with pytest.raises(K.KvaError) as ei:      # 9 query heads on one KV head: more than 8
            K.kva_last_token_layer(h, 1, x, [5], Wt, K.LastParams(9, None, L["q_norm_g"].cuda()),
                                   None, None, c, out)
        assert ei.value.status == K.KVA_ERR_UNSUPPORTED
        with pytest.raises(K.KvaError) as ei:      # the token's row lies past the cache
            K.kva_last_token_layer(h, 1, x, [64], Wt, K.LastParams(geom.attn_n_q, None, L["q_norm_g"].cuda()),
                                   None, None, c, out)
        assert ei.value.status == K.KVA_ERR_TOO_LARGE
        with pytest.raises(K.KvaError) as ei:      # layer index out of range
            K.kva_last_token_layer(h, 3, x, [5], Wt, K.LastParams(geom.attn_n_q, None, L["q_norm_g"].cuda()),
                                   None, None, c, out)
        assert ei.value.status == K.KVA_ERR_INVALID_ARG
    finally:
        K.kva_free(h)
