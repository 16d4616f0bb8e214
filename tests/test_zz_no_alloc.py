"""kva_gdn_layer_update_noalloc: the layer update for callers that may not allocate.

Callers such as an engine that has reserved almost all device memory for its own
cache pool (or a plugin whose host program owns device memory) cannot create a
kva_handle, because that calls cudaMalloc.  The allocation-free entry point keeps
its scratch in a fixed array inside the library instead.  This test checks that it
produces what the handle-based kva_update_states produces for the same layer, on
two calls in a row (the second continues from the first call's state and conv tail).
Both run the same kernels on the same bf16 inputs with deterministic reductions, so the
states and conv tails must be bitwise equal: a tolerance could hide a wrong offset into
the shared scratch.  T = 256 is the largest ubatch the fixed scratch holds, and the r3
layer (n_k * d = 2048, n_v * d = 6144) fills the key and value regions to their limits.
The device status word of the entry point must stay clean after every call.  It sits in
a file collected last so a run that stops at the first failure has already run every
other test.
"""
import numpy as np
import pytest
import torch

import kva_inputs as KI

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def K():
    import hybrid_deltanet_attention_kva_b200 as K
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return K


@pytest.mark.parametrize("geom_name,T", [("r3", 200), ("r3", 256), ("tiny", 97), ("tiny", 256)])
def test_noalloc_matches_handle_path_two_calls(K, geom_name, T):
    base = KI.GEOMETRIES[geom_name]
    # a stack with one gated-DeltaNet layer, so the handle path updates exactly that layer
    geom = KI.with_changes(base, layer_types=(KI.GDN,), n_draft=0)
    P = KI.make_layer_params(geom, 21)
    st = KI.make_states(geom, 1, 22, std=0.1)
    mix = [KI.make_mixer_inputs(geom, 1, T, 23 + i).cuda() for i in range(2)]
    conv_w, A_log, dt_bias = (P[n][0].cuda().contiguous() for n in ("conv_w", "A_log", "dt_bias"))

    # handle-based path
    S_h = st["state"].cuda()
    tail_h = st["conv_tail"].cuda()
    # allocation-free path
    S_n = st["state"][0, 0].cuda().contiguous()
    tail_n = st["conv_tail"][0, 0].cuda().contiguous()

    h = K.kva_init(K.make_dims(geom, T, 1, dtype=torch.bfloat16))
    try:
        Wt = K.Weights(layer={k: v.cuda() for k, v in P.items()})
        for call in range(2):
            K.kva_update_states(h, mix[call], [call * T], Wt, S_h, tail_h, None)
            K.kva_gdn_layer_update_noalloc(mix[call][0], geom.gdn_n_k, geom.gdn_n_v, geom.gdn_d_k,
                                           conv_w, A_log, dt_bias, S_n, tail_n, geom.norm_eps)
            torch.cuda.synchronize()
            assert K.kva_get_device_status(h) == 0
            assert K.kva_gdn_layer_update_noalloc_status() == 0
            assert torch.equal(S_n, S_h[0, 0]), (
                f"state differs after call {call}: max |diff| {(S_n - S_h[0, 0]).abs().max().item()}")
            assert torch.equal(tail_n, tail_h[0, 0]), f"conv tail differs after call {call}"
    finally:
        K.kva_free(h)


def test_noalloc_refuses_sizes_beyond_its_scratch(K):
    geom = KI.with_changes(KI.R3, layer_types=(KI.GDN,), n_draft=0)
    T = 257                                                     # one past the fixed maximum
    mix = torch.zeros(T, geom.gdn_width, dtype=torch.bfloat16, device="cuda")
    P = KI.make_layer_params(geom, 1)
    S = torch.zeros(geom.gdn_n_v, 128, 128, device="cuda")
    tail = torch.zeros(3, geom.gdn_conv_ch, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(K.KvaError) as ei:
        K.kva_gdn_layer_update_noalloc(mix, geom.gdn_n_k, geom.gdn_n_v, 128, P["conv_w"][0].cuda(),
                                       P["A_log"][0].cuda(), P["dt_bias"][0].cuda(), S, tail)
    assert ei.value.status == K.KVA_ERR_TOO_LARGE
    assert bool((S == 0).all())                                 # nothing was launched


def test_noalloc_binding_refuses_formats_it_would_misread(K):
    geom = KI.with_changes(KI.TINY, layer_types=(KI.GDN,), n_draft=0)
    P = KI.make_layer_params(geom, 1)
    args = [P["conv_w"][0].cuda(), P["A_log"][0].cuda(), P["dt_bias"][0].cuda()]
    d, n_k, n_v = geom.gdn_d_k, geom.gdn_n_k, geom.gdn_n_v
    mix = torch.zeros(8, geom.gdn_width, dtype=torch.bfloat16, device="cuda")
    S = torch.zeros(n_v, d, d, device="cuda")
    tail = torch.zeros(3, geom.gdn_conv_ch, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):                             # an fp16 mixer would be read as bf16
        K.kva_gdn_layer_update_noalloc(mix.half(), n_k, n_v, d, *args, S, tail)
    with pytest.raises(ValueError):                             # a state one head short
        K.kva_gdn_layer_update_noalloc(mix, n_k, n_v, d, *args, S[1:].contiguous(), tail)
    with pytest.raises(ValueError):                             # a conv tail of 2 rows
        K.kva_gdn_layer_update_noalloc(mix, n_k, n_v, d, *args, S, tail[:2].contiguous())
    assert bool((S == 0).all())
