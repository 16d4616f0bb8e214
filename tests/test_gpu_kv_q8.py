"""q8_0 KV cache with the Hadamard rotation (the model card's note on quantized KV caches):
GPU cache rows against the float64 oracle.

The oracle's update_states(kv_rotate=True) gives every written row rotated by the
orthonormal Walsh-Hadamard matrix; the GPU stores the same rows as q8_0 blocks.  A stored
value reads back as fp16(d) * code with |code| <= 127 and code = round(x / d), so it lies
within d / 2 + 127 |fp16(d) - d| <= 0.57 d of the value that was quantized (d the block's
scale).  The tests check every written row against that bound (plus, after a projector
pass, the path's stated tolerance for the rows' own error), that every non-zero block uses
the full code range, and that unwritten rows keep their sentinel bytes.
"""
import numpy as np
import pytest
import torch

import kva_inputs as KI
from oracle import kva_ref as R
from tests.parity import f64

pytestmark = pytest.mark.gpu

SENT_BYTE = 0xA5
STEP = 0.57          # the bound above, in units of the block scale
TOL = 2e-2           # the path's max |err| / RMS bar (prefill: the rows' own error)


@pytest.fixture(scope="module")
def K():
    import hybrid_deltanet_attention_kva_b200 as K
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return K


def dequant_rows(raw: np.ndarray, d_h: int):
    """uint8 [..., d_h * 34 / 32] -> (values float64 [..., d_h], scales float64 [..., d_h/32],
    codes int [..., d_h])."""
    nb = d_h // 32
    blk = raw.reshape(*raw.shape[:-1], nb, 34)
    d = blk[..., :2].copy().view(np.float16)[..., 0].astype(np.float64)
    codes = blk[..., 2:].copy().view(np.int8).astype(np.int64)
    vals = (codes * d[..., None]).reshape(*raw.shape[:-1], d_h)
    return vals, d, codes.reshape(*raw.shape[:-1], d_h)


class Q8Caches:
    """q8_0 caches on the device (sentinel bytes) and float64 oracle twins (NaN = unwritten)."""

    def __init__(self, K, geom, n_seq, max_pos, paged=False, page_size=64, seed=77):
        self.geom, self.paged, self.page_size = geom, paged, page_size
        na, nkv, dh = geom.n_attn, geom.attn_n_kv, geom.attn_d_h
        rb = dh * 34 // 32
        if paged:
            pps = (max_pos + page_size - 1) // page_size
            self.n_pages = n_seq * pps + 3
            self.pt = KI.make_page_table(n_seq, pps, seed, n_pages=self.n_pages)
            lead = (self.n_pages, nkv, page_size)
        else:
            lead = (n_seq, nkv, max_pos)
        self.k = [torch.full(lead + (rb,), SENT_BYTE, dtype=torch.uint8, device="cuda") for _ in range(na)]
        self.v = [torch.full(lead + (rb,), SENT_BYTE, dtype=torch.uint8, device="cuda") for _ in range(na)]
        self.ok = [np.full(lead + (dh,), np.nan) for _ in range(na)]
        self.ov = [np.full(lead + (dh,), np.nan) for _ in range(na)]
        if paged:
            self.c = K.KvCache(self.k, self.v, page_table=self.pt.cuda(), page_size=page_size,
                               n_pages=self.n_pages)
        else:
            self.c = K.KvCache(self.k, self.v, max_pos=max_pos)

    def oracle_views(self, s):
        if self.paged:
            return self.ok, self.ov, self.pt.numpy()[s], self.page_size
        return [k[s] for k in self.ok], [v[s] for v in self.ov], None, 0

    def check(self, tol=0.0):
        """Every written row within STEP * d (+ tol * RMS) of the oracle; full-range codes;
        sentinel bytes elsewhere.  Returns the worst excess over the quantization step / RMS."""
        dh = self.geom.attn_d_h
        worst = 0.0
        for name, gl, ol in (("K", self.k, self.ok), ("V", self.v, self.ov)):
            for a in range(len(gl)):
                raw = gl[a].cpu().numpy()
                ref = ol[a]
                written = ~np.isnan(ref[..., 0])
                assert written.any()
                # unwritten rows untouched, written rows fully overwritten
                assert np.all(raw[~written] == SENT_BYTE)
                vals, d, codes = dequant_rows(raw[written], dh)
                want = ref[written]
                rms = float(np.sqrt(np.mean(want * want)))
                err = np.abs(vals - want)
                step = STEP * np.repeat(d, 32, axis=-1)
                excess = float((err - step).max() / rms)
                assert excess <= tol + 1e-4, (name, a, excess)
                worst = max(worst, excess)
                cb = np.abs(codes).reshape(*codes.shape[:-1], dh // 32, 32).max(-1)
                assert np.all((cb == 127) | (d == 0)), (name, a)
        return worst


@pytest.mark.parametrize("geom_name,n_seq,T,paged,dt", [
    ("tiny", 2, 100, False, torch.bfloat16), ("tiny", 3, 2, True, torch.float16),
    ("r3", 2, 200, True, torch.float16), ("r3", 1, 130, False, torch.bfloat16)])
def test_update_states_q8_0_cache(K, geom_name, n_seq, T, paged, dt):
    geom = KI.GEOMETRIES[geom_name]
    if geom_name == "r3":
        geom = KI.with_changes(geom, n_draft=0)
    P = KI.make_layer_params(geom, 21, random_k_gain=True)
    st = KI.make_states(geom, n_seq, 22, std=0.1)
    st["conv_tail"] = st["conv_tail"].to(dt)
    mix = KI.make_mixer_inputs(geom, n_seq, T, 23).to(dt)
    pos = [3 + 257 * s for s in range(n_seq)]
    max_pos = max(pos) + T + 5
    caches = Q8Caches(K, geom, n_seq, max_pos, paged=paged)
    h = K.kva_init(K.make_dims(geom, max(T, 16), n_seq, dtype=dt))
    try:
        S = st["state"].cuda()
        tail = st["conv_tail"].cuda()
        Wt = K.Weights(layer={k: v.cuda() for k, v in P.items()})
        K.kva_update_states(h, mix.cuda(), pos, Wt, S, tail, caches.c)
        assert K.kva_get_device_status(h) == 0
    finally:
        K.kva_free(h)
    Pn = {k: f64(v) for k, v in P.items()}
    for s in range(n_seq):
        kc, vc, pt, ps = caches.oracle_views(s)
        R.update_states(f64(mix[s]), geom, Pn, f64(st["state"][s]), f64(st["conv_tail"][s]), kc, vc,
                        pos[s], page_table=pt, page_size=ps, scan="chunked", kv_rotate=True)
    # the oracle read the GPU's own 16-bit mixer: only the quantization step separates them
    caches.check(tol=0.0)


TINY128 = KI.with_changes(KI.TINY, name="tiny128", gdn_d_k=128, gdn_d_v=128, attn_d_h=256,
                          rope_dims=64, n_draft=1)


@pytest.mark.parametrize("geom,fused", [(TINY128, True), (KI.TINY, False)])
def test_prefill_q8_0_cache_ragged_and_carry(K, geom, fused):
    dt = torch.float16
    splits = [300, 2, 130]
    W = KI.make_projector_weights(geom, 4100)
    W = {k: (v if k.startswith("g_") or k == "blocks" else v.to(dt)) for k, v in W.items()}
    W["blocks"] = [{k: (v if k.startswith("g_") else v.to(dt)) for k, v in b.items()} for b in W["blocks"]]
    P = KI.make_layer_params(geom, 4101)
    st = KI.make_states(geom, 1, 4102)
    res = KI.make_residual(geom, sum(splits), 4103, dtype=torch.float32, n_outliers=0)
    caches = Q8Caches(K, geom, 1, sum(splits) + 16)
    h = K.kva_init(K.make_dims(geom, max(splits), 1, dtype=dt))
    try:
        assert K.kva_heads_fused(h) is fused
        Wg = K.Weights(proj={k: (v.cuda() if k != "blocks" else [{a: b.cuda() for a, b in blk.items()}
                                                                  for blk in v]) for k, v in W.items()},
                       layer={k: v.cuda() for k, v in P.items()})
        S = st["state"][0].cuda()
        tail = st["conv_tail"][0].to(dt).cuda()
        pos = 0
        for T in splits:
            K.kva_prefill_ubatch(h, res[pos:pos + T].cuda(), Wg, S, tail, caches.c, pos)
            pos += T
        torch.cuda.synchronize()
        assert K.kva_get_device_status(h) == 0
    finally:
        K.kva_free(h)
    Wn = R.weights_to_f64(W)
    Pn = {k: f64(v) for k, v in P.items()}
    kc, vc, _, _ = caches.oracle_views(0)
    S_o, tail_o = f64(st["state"][0]), f64(st["conv_tail"][0].to(dt))
    pos = 0
    for T in splits:
        _, S_o, tail_o = R.prefill_ubatch(f64(res[pos:pos + T]), Wn, geom, Pn, S_o, tail_o, kc, vc, pos,
                                          kv_rotate=True)
        pos += T
    caches.check(tol=TOL)
