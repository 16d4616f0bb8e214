"""Per-kernel parity on the GPU: each step called through the C ABI against the oracle.

Sizes span several tiles and a ragged tail; inputs are seeded; the oracle sees
exactly the bf16 / fp32 values the device reads.
"""
import math

import numpy as np
import pytest
import torch

from oracle import kva_ref as R
from tests.parity import BF16_ELEM, assert_rms_close, assert_state_close, bf16_round, f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def K():
    import hybrid_deltanet_attention_kva_b200 as K
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return K


def _gen(seed):
    g = torch.Generator().manual_seed(seed)
    return g


# ------------------------------------------------------------------ RMSNorm
@pytest.mark.parametrize("dtype,rows,n", [(torch.float32, 37, 512), (torch.bfloat16, 129, 5120),
                                          (torch.float32, 1024, 3072), (torch.float16, 64, 256)])
@pytest.mark.parametrize("odt", [torch.bfloat16, torch.float16])
def test_rmsnorm(K, dtype, rows, n, odt):
    g = _gen(rows)
    x = (torch.randn(rows, n, generator=g) * 3).to(dtype)
    gain = torch.rand(n, generator=g) + 0.5
    out = torch.empty(rows, n, dtype=odt, device="cuda")
    K.kva_op_rmsnorm(x.cuda(), gain.cuda(), out)
    torch.cuda.synchronize()
    want = R.rmsnorm(f64(x), f64(gain))
    assert_rms_close(out, want, what="rmsnorm", elem=BF16_ELEM)


# ------------------------------------------------------------------ GEMM
@pytest.mark.parametrize("M,N,K_,bn", [(128, 256, 64, 256), (200, 1296, 520, 0), (1024, 3072, 3072, 128),
                                       (77, 512, 256, 256), (1024, 2560, 5120, 0), (600, 1040, 704, 512),
                                       (1024, 3072, 3072, 256), (1024, 3072, 8448, 512),
                                       (1000, 3072, 5120, 512)])
@pytest.mark.parametrize("epi", [0, 1, 2])
@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float16])
def test_gemm_epilogues(K, M, N, K_, bn, epi, dt):
    g = _gen(M * 7 + N + epi)
    A = torch.randn(M, K_, generator=g).to(dt)
    B = (torch.randn(N, K_, generator=g) * 0.05).to(dt)
    want = R.projector_heads(f64(A), f64(B))
    if epi == K.EPI_STORE_BF16:
        D = torch.full((M, N), float("nan"), dtype=dt, device="cuda")
    else:
        D = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    D0 = None
    if epi == K.EPI_ADD_F32:
        D0 = torch.randn(M, N, generator=g)
        D.copy_(D0)
        want = want + f64(D0)
    K.kva_op_gemm(A.cuda(), [B.cuda()], D, N=N, epilogue=epi, block_n=bn)
    torch.cuda.synchronize()
    assert_rms_close(D, want, what=f"gemm epi={epi}", elem=BF16_ELEM if epi == 0 else 0.0)


@pytest.mark.parametrize("M,F,K_", [(128, 704, 256), (1000, 1024, 512), (1024, 8448, 3072)])
@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float16])
def test_gemm_swiglu_paired(K, M, F, K_, dt):
    g = _gen(F)
    A = torch.randn(M, K_, generator=g).to(dt)
    Bg = (torch.randn(F, K_, generator=g) * 0.05).to(dt)
    Bu = (torch.randn(F, K_, generator=g) * 0.05).to(dt)
    D = torch.full((M, F), float("nan"), dtype=dt, device="cuda")
    K.kva_op_gemm(A.cuda(), [Bg.cuda(), Bu.cuda()], D, N=F, epilogue=K.EPI_SWIGLU_BF16,
                  b_mode=K.B_PAIRED)
    torch.cuda.synchronize()
    a = f64(A)
    want = R.silu(a @ f64(Bg).T) * (a @ f64(Bu).T)
    assert_rms_close(D, want, what="swiglu", elem=BF16_ELEM)


@pytest.mark.parametrize("M,d", [(300, 256), (1024, 3072)])
@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("bn", [128, 512])
def test_gemm_qkv_segments(K, M, d, dt, bn):
    g = _gen(d)
    A = torch.randn(M, d, generator=g).to(dt)
    Ws = [(torch.randn(d, d, generator=g) * 0.05).to(dt) for _ in range(3)]
    D = torch.full((M, 3 * d), float("nan"), dtype=dt, device="cuda")
    K.kva_op_gemm(A.cuda(), [w.cuda() for w in Ws], D, N=3 * d, b_mode=K.B_SEGMENTS,
                  seg_rows=d, block_n=bn)
    torch.cuda.synchronize()
    want = np.concatenate([f64(A) @ f64(w).T for w in Ws], axis=1)
    assert_rms_close(D, want, what="qkv", elem=BF16_ELEM)


def test_gemm_split_output(K):
    M, N1, N2, K_ = 130, 1024, 512, 256
    g = _gen(5)
    A = torch.randn(M, K_, generator=g).to(torch.bfloat16)
    B = (torch.randn(N1 + N2, K_, generator=g) * 0.05).to(torch.bfloat16)
    D = torch.zeros(M, N1, dtype=torch.bfloat16, device="cuda")
    D1 = torch.zeros(M, N2, dtype=torch.bfloat16, device="cuda")
    K.kva_op_gemm(A.cuda(), [B.cuda()], D, N=N1 + N2, D1=D1, n_split=N1)
    torch.cuda.synchronize()
    want = f64(A) @ f64(B).T
    assert_rms_close(D, want[:, :N1], what="split D", elem=BF16_ELEM)
    assert_rms_close(D1, want[:, N1:], what="split D1", elem=BF16_ELEM)


def test_gemm_rejects_misaligned(K):
    A = torch.zeros(64, 72, dtype=torch.bfloat16, device="cuda")[:, :68]
    with pytest.raises(ValueError):
        K.kva_op_gemm(A, [torch.zeros(64, 68, dtype=torch.bfloat16, device="cuda")],
                      torch.zeros(64, 64, dtype=torch.bfloat16, device="cuda"), N=64)
    A = torch.zeros(64, 68, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(K.KvaError) as ei:
        K.kva_op_gemm(A, [torch.zeros(64, 68, dtype=torch.bfloat16, device="cuda")],
                      torch.zeros(64, 64, dtype=torch.bfloat16, device="cuda"), N=64)
    assert ei.value.status == K.KVA_ERR_ALIGNMENT


# ------------------------------------------------------------------ attention
@pytest.mark.parametrize("T,heads,window", [(128, 2, 0), (300, 3, 0), (1024, 4, 1024), (1024, 2, 256),
                                            (700, 2, 200), (1, 1, 0)])
@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float16])
def test_attention(K, T, heads, window, dt):
    g = _gen(T + heads)
    d = heads * 128
    qkv = torch.randn(T, 3 * d, generator=g).to(dt)
    out = torch.full((T, d), float("nan"), dtype=dt, device="cuda")
    K.kva_op_attention(qkv.cuda(), out, heads, window)
    torch.cuda.synchronize()
    q = f64(qkv)
    Q = q[:, :d].reshape(T, heads, 128)
    Kk = q[:, d:2 * d].reshape(T, heads, 128)
    V = q[:, 2 * d:].reshape(T, heads, 128)
    want = R.block_causal_attention(Q, Kk, V, window).reshape(T, d)
    # the softmax weights are rounded to bf16 before P V: each output element may move
    # by 2^-8 of the weighted sum of |v| it averages (the oracle's attention over |V|)
    scale = R.block_causal_attention(Q, Kk, np.abs(V), window).reshape(T, d)
    assert_rms_close(out, want, what="attention", elem=BF16_ELEM, scale=scale)


@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float16])
def test_attention_rising_scores(K, dt):
    # scores grow along the keys (a shared direction u in q and, with a ramp, in k), so the
    # running row max moves by far more than 2^8 from one 128-key tile to the next and the
    # accumulated output is rescaled on most tiles
    T, heads = 700, 2
    d = heads * 128
    g = _gen(9701)
    u = torch.randn(128, generator=g, dtype=torch.float64)
    u = u / u.norm()
    q = torch.randn(T, heads, 128, generator=g, dtype=torch.float64) + 4.0 * u
    k = torch.randn(T, heads, 128, generator=g, dtype=torch.float64) + \
        (torch.arange(T, dtype=torch.float64) / 8.0)[:, None, None] * u
    v = torch.randn(T, heads, 128, generator=g, dtype=torch.float64)
    qkv = torch.cat([q.reshape(T, d), k.reshape(T, d), v.reshape(T, d)], 1).to(dt)
    out = torch.full((T, d), float("nan"), dtype=dt, device="cuda")
    K.kva_op_attention(qkv.cuda(), out, heads, 0)
    torch.cuda.synchronize()
    x = f64(qkv)
    Q, Kk, V = (x[:, i * d:(i + 1) * d].reshape(T, heads, 128) for i in range(3))
    want = R.block_causal_attention(Q, Kk, V, 0).reshape(T, d)
    scale = R.block_causal_attention(Q, Kk, np.abs(V), 0).reshape(T, d)
    assert_rms_close(out, want, what="attention, rising scores", elem=BF16_ELEM, scale=scale)


# ------------------------------------------------------------------ scan
def _scan_inputs(seed, n_layers, T, n_k, n_v, d, g_scale=1.0, beta=None, gzero=False):
    g = _gen(seed)
    k = torch.randn(n_layers, T, n_k, d, generator=g, dtype=torch.float64)
    k = k / k.norm(dim=-1, keepdim=True)
    k = k.to(torch.float16)
    v = torch.randn(n_layers, T, n_v, d, generator=g).to(torch.float16)
    gg = -torch.rand(n_layers, n_v, T, generator=g) * g_scale
    if gzero:
        gg.zero_()
    bb = torch.rand(n_layers, n_v, T, generator=g) if beta is None else torch.full((n_layers, n_v, T), beta)
    S0 = torch.randn(n_layers, n_v, d, d, generator=g) * 0.1
    gb = torch.stack([gg, bb], dim=1).contiguous()   # [L, 2, n_v, T]
    return k, v, gb, S0


@pytest.mark.parametrize("T,n_k,n_v,d", [(64, 1, 1, 128), (150, 2, 6, 128), (1, 2, 4, 64),
                                         (200, 2, 4, 64), (1024, 16, 48, 128)])
def test_scan_matches_sequential_oracle(K, T, n_k, n_v, d):
    L = 2 if T < 1024 else 1
    k, v, gb, S0 = _scan_inputs(T + d, L, T, n_k, n_v, d)
    st = S0.clone().cuda()
    K.kva_op_gdn_scan(k.reshape(L, T, n_k * d).cuda(), v.reshape(L, T, n_v * d).cuda(), gb.cuda(),
                      st, 1, L, n_k, n_v, d)
    torch.cuda.synchronize()
    for l in range(L):
        want = (R.delta_scan_sequential if T <= 256 else R.delta_scan_chunked)(
            f64(S0[l]), f64(k[l]), f64(v[l]), f64(gb[l, 0].T), f64(gb[l, 1].T))
        assert_state_close(st[l], want)


def test_scan_beta_zero_pure_decay_and_identity(K):
    T, n_k, n_v, d = 130, 1, 2, 128
    k, v, gb, S0 = _scan_inputs(3, 1, T, n_k, n_v, d, g_scale=0.01, beta=0.0)
    st = S0.clone().cuda()
    K.kva_op_gdn_scan(k.reshape(1, T, -1).cuda(), v.reshape(1, T, -1).cuda(), gb.cuda(), st, 1, 1,
                      n_k, n_v, d)
    torch.cuda.synchronize()
    want = np.exp(f64(gb[0, 0]).sum(-1))[:, None, None] * f64(S0[0])
    assert_state_close(st[0], want, tol=1e-5)
    k, v, gb, S0 = _scan_inputs(4, 1, T, n_k, n_v, d, beta=0.0, gzero=True)
    st = S0.clone().cuda()
    K.kva_op_gdn_scan(k.reshape(1, T, -1).cuda(), v.reshape(1, T, -1).cuda(), gb.cuda(), st, 1, 1,
                      n_k, n_v, d)
    torch.cuda.synchronize()
    assert torch.equal(st.cpu(), S0)


def test_scan_strong_decay_no_overflow(K):
    T, n_k, n_v, d = 256, 2, 4, 128
    k, v, gb, S0 = _scan_inputs(5, 1, T, n_k, n_v, d, g_scale=45.0)
    st = S0.clone().cuda()
    K.kva_op_gdn_scan(k.reshape(1, T, -1).cuda(), v.reshape(1, T, -1).cuda(), gb.cuda(), st, 1, 1,
                      n_k, n_v, d)
    torch.cuda.synchronize()
    want = R.delta_scan_sequential(f64(S0[0]), f64(k[0]), f64(v[0]), f64(gb[0, 0].T), f64(gb[0, 1].T))
    assert_state_close(st[0], want)


# ------------------------------------------------------------------ GEMM with q8_0 weights
# The kernel rounds every dequantized weight once to the operand format: harmless for fp16
# (2^-11), but bf16 keeps 8 significant bits, the same input rounding that puts the bf16 path
# under its stated 4e-2 x RMS bar instead of 2e-2.
Q8_TOL = {torch.float16: 2e-2, torch.bfloat16: 4e-2}


def _q8_weights(g, rows, K, scale=0.05):
    """Random weights as q8_0 (codes int8 [rows, K], scales fp16 [K/32, rows]) and their
    dequantized float64 values (the oracle's quantizer and dequantizer)."""
    W = (torch.randn(rows, K, generator=g, dtype=torch.float64) * scale).numpy()
    d, codes = R.q8_0_quantize(W)
    Wd = R.q8_0_dequantize(d, codes)
    return torch.from_numpy(codes), torch.from_numpy(np.ascontiguousarray(d.T)), Wd


@pytest.mark.parametrize("M,N,K_,epi", [(1024, 3072, 3072, 0), (600, 1040, 704, 0), (77, 256, 128, 0),
                                        (1024, 3072, 8448, 2), (1000, 2048, 1024, 2)])
@pytest.mark.parametrize("dt", [torch.float16, torch.bfloat16])
def test_gemm_q8_0_weights(K, M, N, K_, epi, dt):
    g = _gen(M * 3 + N + K_ + epi)
    A = torch.randn(M, K_, generator=g).to(dt)
    Bq, Bs, Wd = _q8_weights(g, N, K_)
    want = R.projector_heads(f64(A), Wd)
    if epi == K.EPI_STORE_BF16:
        D = torch.full((M, N), float("nan"), dtype=dt, device="cuda")
    else:
        D0 = torch.randn(M, N, generator=g)
        D = D0.cuda()
        want = want + f64(D0)
    K.kva_op_gemm_q8_0(A.cuda(), [Bq.cuda()], [Bs.cuda()], D, N=N, epilogue=epi)
    torch.cuda.synchronize()
    # the GPU rounds every dequantized weight once to the operand format
    assert_rms_close(D, want, tol=Q8_TOL[dt], what=f"q8_0 gemm epi={epi}",
                     elem=BF16_ELEM if epi == 0 else 0.0)


def _q4_weights(g, rows, K, scale=0.05):
    """Random weights as q4_0 (packed codes uint8 [rows, K/2], scales fp16 [K/32, rows]) and
    their dequantized float64 values (the oracle's quantizer, packer and dequantizer)."""
    W = (torch.randn(rows, K, generator=g, dtype=torch.float64) * scale).numpy()
    d, codes = R.q4_0_quantize(W)
    Wd = R.q4_0_dequantize(d, codes)
    return (torch.from_numpy(R.q4_0_pack(codes)), torch.from_numpy(np.ascontiguousarray(d.T)), Wd)


@pytest.mark.parametrize("M,N,K_,epi", [(1024, 3072, 3072, 0), (600, 1040, 704, 0), (77, 256, 128, 0),
                                        (1000, 2048, 1024, 2)])
@pytest.mark.parametrize("dt", [torch.float16, torch.bfloat16])
def test_gemm_q4_0_weights(K, M, N, K_, epi, dt):
    g = _gen(M * 5 + N + K_ + epi)
    A = torch.randn(M, K_, generator=g).to(dt)
    Bq, Bs, Wd = _q4_weights(g, N, K_)
    want = R.projector_heads(f64(A), Wd)
    if epi == K.EPI_STORE_BF16:
        D = torch.full((M, N), float("nan"), dtype=dt, device="cuda")
    else:
        D0 = torch.randn(M, N, generator=g)
        D = D0.cuda()
        want = want + f64(D0)
    K.kva_op_gemm_q4_0(A.cuda(), [Bq.cuda()], [Bs.cuda()], D, N=N, epilogue=epi)
    torch.cuda.synchronize()
    # d (c - 8) has at most 15 significant bits: one rounding to the operand format
    assert_rms_close(D, want, tol=Q8_TOL[dt], what=f"q4_0 gemm epi={epi}",
                     elem=BF16_ELEM if epi == 0 else 0.0)


def test_gemm_q4_0_swiglu_and_segments(K):
    g = _gen(4343)
    dt = torch.float16
    M, F, Kd = 1000, 1024, 512
    A = torch.randn(M, Kd, generator=g).to(dt)
    Gq, Gs, Gd = _q4_weights(g, F, Kd)
    Uq, Us, Ud = _q4_weights(g, F, Kd)
    D = torch.empty(M, F, dtype=dt, device="cuda")
    K.kva_op_gemm_q4_0(A.cuda(), [Gq.cuda(), Uq.cuda()], [Gs.cuda(), Us.cuda()], D, N=F,
                       epilogue=K.EPI_SWIGLU_BF16, b_mode=K.B_PAIRED)
    a = f64(A)
    gate, up = a @ Gd.T, a @ Ud.T
    assert_rms_close(D, gate / (1.0 + np.exp(-gate)) * up, tol=Q8_TOL[dt], what="q4_0 swiglu",
                     elem=BF16_ELEM)
    seg = 512
    parts = [_q4_weights(g, seg, Kd) for _ in range(3)]
    D2 = torch.empty(M, 3 * seg, dtype=dt, device="cuda")
    K.kva_op_gemm_q4_0(A.cuda(), [p[0].cuda() for p in parts], [p[1].cuda() for p in parts], D2,
                       N=3 * seg, b_mode=K.B_SEGMENTS, seg_rows=seg)
    want2 = a @ np.concatenate([p[2] for p in parts]).T
    assert_rms_close(D2, want2, tol=Q8_TOL[dt], what="q4_0 segments", elem=BF16_ELEM)


@pytest.mark.parametrize("dt", [torch.float16, torch.bfloat16])
def test_gemm_q8_0_swiglu_and_segments(K, dt):
    g = _gen(4242)
    M, F, Kd = 1000, 1024, 512
    A = torch.randn(M, Kd, generator=g).to(dt)
    Gq, Gs, Gd = _q8_weights(g, F, Kd)
    Uq, Us, Ud = _q8_weights(g, F, Kd)
    D = torch.empty(M, F, dtype=dt, device="cuda")
    K.kva_op_gemm_q8_0(A.cuda(), [Gq.cuda(), Uq.cuda()], [Gs.cuda(), Us.cuda()], D, N=F,
                       epilogue=K.EPI_SWIGLU_BF16, b_mode=K.B_PAIRED)
    a = f64(A)
    gate, up = a @ Gd.T, a @ Ud.T
    want = gate / (1.0 + np.exp(-gate)) * up
    assert_rms_close(D, want, tol=Q8_TOL[dt], what="q8_0 swiglu", elem=BF16_ELEM)
    # q | k | v from three q8_0 matrices of 512 rows each
    seg = 512
    parts = [_q8_weights(g, seg, Kd) for _ in range(3)]
    D2 = torch.empty(M, 3 * seg, dtype=dt, device="cuda")
    K.kva_op_gemm_q8_0(A.cuda(), [p[0].cuda() for p in parts], [p[1].cuda() for p in parts], D2,
                       N=3 * seg, b_mode=K.B_SEGMENTS, seg_rows=seg)
    want2 = a @ np.concatenate([p[2] for p in parts]).T
    assert_rms_close(D2, want2, tol=Q8_TOL[dt], what="q8_0 segments", elem=BF16_ELEM)


def test_pipeline_wait_that_runs_out_is_reported_and_the_next_call_is_clean(K):
    """Failure detection without a GPU fault: the CTA-pair GEMM's MMA issuer waits on a barrier
    that nothing arrives on; the wait gives up after about a millisecond, the kernel drains its
    own copies and MMAs and returns with KVA_DEV_WAIT_TIMEOUT in its status word.  The context
    stays usable: the same GEMM right after is correct and reports nothing."""
    torch.manual_seed(3)
    M, N, Kd = 256, 256, 256
    A = (torch.randn(M, Kd, device="cuda") * 0.5).half()
    B = (torch.randn(N, Kd, device="cuda") * 0.05).half()
    D = torch.zeros(M, N, dtype=torch.half, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    K.kva_test_gemm_wait_timeout(A, B, D, err)
    torch.cuda.synchronize()
    assert int(err.item()) & K.KVA_DEV_WAIT_TIMEOUT
    err.zero_()
    K.kva_op_gemm(A, [B], D, N=N, epilogue=K.EPI_STORE_BF16, block_n=512, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    want = (A.float() @ B.float().T)
    assert torch.allclose(D.float(), want, rtol=2e-3, atol=2e-3)
