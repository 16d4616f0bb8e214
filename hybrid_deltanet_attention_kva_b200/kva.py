"""ctypes binding of libkva (include/kva.h, include/kva_ops.h).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  The functions keep the C names.  Tensors are torch CUDA tensors (the
caller owns them); streams default to torch's current stream.
"""
from __future__ import annotations

import ctypes as C
import os
from typing import Dict, Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkva.so")

MAX_LATE = 64
MAX_BLOCKS = 8

KVA_OK = 0
KVA_ERR_INVALID_ARG = -1
KVA_ERR_UNSUPPORTED = -2
KVA_ERR_TOO_LARGE = -3
KVA_ERR_ALIGNMENT = -4
KVA_ERR_CUDA = -5
KVA_ERR_NO_MEMORY = -6
KVA_ERR_DEVICE = -7
KVA_DEV_PAGE_OOB = 0x1
KVA_DEV_WAIT_TIMEOUT = 0x2

KVA_LAYER_GDN, KVA_LAYER_ATTN = 0, 1
KVA_BF16, KVA_F32, KVA_F16, KVA_Q8_0 = 0, 1, 2, 3
_DT = {torch.bfloat16: KVA_BF16, torch.float32: KVA_F32, torch.float16: KVA_F16}
KVA_KV_CONTIGUOUS, KVA_KV_PAGED = 0, 1
EPI_STORE_BF16, EPI_STORE_F32, EPI_ADD_F32, EPI_SWIGLU_BF16 = 0, 1, 2, 3
B_SINGLE, B_SEGMENTS, B_PAIRED = 0, 1, 2


class KvaDims(C.Structure):
    _fields_ = [
        ("hidden", C.c_int32), ("d_model", C.c_int32), ("n_heads", C.c_int32),
        ("head_dim", C.c_int32), ("ffn", C.c_int32), ("n_blocks", C.c_int32),
        ("attn_window", C.c_int32), ("n_late", C.c_int32),
        ("layer_type", C.c_int32 * MAX_LATE),
        ("gdn_n_k", C.c_int32), ("gdn_n_v", C.c_int32), ("gdn_d_k", C.c_int32),
        ("gdn_d_v", C.c_int32), ("conv_k", C.c_int32), ("attn_n_kv", C.c_int32),
        ("attn_d_h", C.c_int32), ("rope_dims", C.c_int32), ("rope_theta", C.c_double),
        ("norm_eps", C.c_float), ("n_draft_cols", C.c_int32), ("max_T", C.c_int32),
        ("max_seq", C.c_int32), ("compute_dtype", C.c_int32),
    ]


class KvaBlockWeights(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in
                ("g_attn", "Wq", "Wk", "Wv", "Wo", "g_ffn", "Wg", "Wu", "Wd")]


class KvaWeights(C.Structure):
    _fields_ = [("g_in", C.c_void_p), ("W_in", C.c_void_p),
                ("blocks", KvaBlockWeights * MAX_BLOCKS), ("g_out", C.c_void_p),
                ("W_heads", C.c_void_p), ("conv_w", C.c_void_p), ("A_log", C.c_void_p),
                ("dt_bias", C.c_void_p), ("k_norm_g", C.c_void_p), ("weight_format", C.c_int32),
                ("W_in_scale", C.c_void_p), ("W_heads_scale", C.c_void_p),
                ("block_scale", (C.c_void_p * 7) * MAX_BLOCKS)]


KVA_W_16, KVA_W_Q8_0, KVA_W_Q4_0 = 0, 1, 2
Q8_MATRICES = ("Wq", "Wk", "Wv", "Wo", "Wg", "Wu", "Wd")


class KvaKvCache(C.Structure):
    _fields_ = [("layout", C.c_int32), ("n_layers", C.c_int32),
                ("k", C.c_void_p * MAX_LATE), ("v", C.c_void_p * MAX_LATE),
                ("max_pos", C.c_int64), ("page_size", C.c_int32), ("n_pages", C.c_int32),
                ("pages_per_seq", C.c_int32), ("page_table", C.c_void_p), ("dtype", C.c_int32)]


class KvaLastParams(C.Structure):
    _fields_ = [("attn_n_q", C.c_int32), ("gdn_norm_w", C.c_void_p), ("q_norm_g", C.c_void_p)]


ST_NAMES = ("rmsnorm", "gemm_trunk", "attention", "gemm_heads", "gdn_prepare", "gdn_tail",
            "gdn_scan", "kv_write", "last_token")
ST_COUNT = len(ST_NAMES)


class KvaProfile(C.Structure):
    _fields_ = [("ms", C.c_float * ST_COUNT), ("timed", C.c_int32 * ST_COUNT),
                ("launches", C.c_int64 * ST_COUNT)]


class KvaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {kva_strerror(status)} ({status})")


def _load() -> C.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"libkva.so not found at {LIB_PATH}; build it with "
            "`python -m hybrid_deltanet_attention_kva_b200.build` (there is no fallback)")
    lib = C.CDLL(LIB_PATH)
    P, I32, I64, F32, SZ = C.c_void_p, C.c_int32, C.c_int64, C.c_float, C.c_size_t
    sig = {
        "kva_init": (I32, [C.POINTER(KvaDims), C.POINTER(P)]),
        "kva_workspace_bytes": (SZ, [C.POINTER(KvaDims)]),
        "kva_prefill_ubatch": (I32, [P, P, I32, I32, C.POINTER(KvaWeights), P, P,
                                     C.POINTER(KvaKvCache), I64, P, P, P]),
        "kva_update_states": (I32, [P, P, I64, I32, I32, C.POINTER(I64), C.POINTER(KvaWeights),
                                    P, P, C.POINTER(KvaKvCache), P, P, P]),
        "kva_last_token_layer": (I32, [P, I32, I32, P, I64, C.POINTER(I64), C.POINTER(KvaWeights),
                                       C.POINTER(KvaLastParams), P, P, C.POINTER(KvaKvCache), P, I32,
                                       I64, P]),
        "kva_get_device_status": (I32, [P, C.POINTER(I32)]),
        "kva_stats": (I32, [P, C.POINTER(I64)]),
        "kva_heads_fused": (I32, [P, C.POINTER(I32)]),
        "kva_free": (None, [P]),
        "kva_profile_enable": (I32, [P, I32]),
        "kva_profile_read": (I32, [P, C.POINTER(KvaProfile)]),
        "kva_strerror": (C.c_char_p, [I32]),
        "kva_op_rmsnorm": (I32, [P, I32, I64, P, P, I32, I64, I32, I32, F32, P]),
        "kva_op_gemm": (I32, [I32, P, I64, C.POINTER(P), I32, I64, I64, P, I64, P, I64, I64, I32,
                              I32, I32, I32, I32, P, P]),
        "kva_op_gemm_q8_0": (I32, [I32, P, I64, C.POINTER(P), C.POINTER(P), I32, I64, P, I64, I32, I32,
                                   I32, I32, P, P]),
        "kva_op_gemm_q4_0": (I32, [I32, P, I64, C.POINTER(P), C.POINTER(P), I32, I64, P, I64, I32, I32,
                                   I32, I32, P, P]),
        "kva_op_attention": (I32, [I32, P, I64, P, I64, I32, I32, I32, P]),
        "kva_op_gdn_scan": (I32, [P, P, P, P, I32, I32, I32, I32, I32, I32, P]),
        "kva_gdn_layer_update_noalloc": (I32, [P, I64, I32, I32, I32, I32, P, P, P, P, P, F32, P]),
        "kva_test_gemm_wait_timeout": (I32, [I32, P, P, P, I32, I32, I32, P, P]),
        "kva_gdn_layer_update_noalloc_status": (I32, [P, C.POINTER(I32)]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()
EXPORTED = ("kva_init", "kva_workspace_bytes", "kva_prefill_ubatch", "kva_update_states",
            "kva_last_token_layer",
            "kva_get_device_status", "kva_stats", "kva_heads_fused", "kva_free", "kva_strerror",
            "kva_profile_enable", "kva_profile_read",
            "kva_op_rmsnorm", "kva_op_gemm", "kva_op_gemm_q8_0", "kva_op_gemm_q4_0", "kva_op_attention",
            "kva_op_gdn_scan",
            "kva_gdn_layer_update_noalloc", "kva_gdn_layer_update_noalloc_status",
            "kva_test_gemm_wait_timeout")


def lib() -> C.CDLL:
    return _lib


def kva_strerror(status: int) -> str:
    return _lib.kva_strerror(int(status)).decode()


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libkva takes CUDA tensors")
    if not t.is_contiguous():
        raise ValueError("libkva takes contiguous tensors")
    return t.data_ptr()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check(status: int, what: str) -> None:
    if status != KVA_OK:
        raise KvaError(status, what)


# ----------------------------------------------------------------- structs
def make_dims(geom, max_T: int, max_seq: int = 1, dtype=torch.float16) -> KvaDims:
    """kva_dims from any object carrying the geometry attributes; dtype is the
    16-bit operand format of the projector (torch.float16 or torch.bfloat16)."""
    d = KvaDims()
    d.hidden, d.d_model, d.n_heads = geom.hidden, geom.d_model, geom.n_heads
    d.head_dim, d.ffn, d.n_blocks = geom.head_dim, geom.ffn, geom.n_blocks
    d.attn_window = geom.window
    d.n_late = len(geom.layer_types)
    for i, t in enumerate(geom.layer_types):
        d.layer_type[i] = int(t)
    d.gdn_n_k, d.gdn_n_v, d.gdn_d_k, d.gdn_d_v = geom.gdn_n_k, geom.gdn_n_v, geom.gdn_d_k, geom.gdn_d_v
    d.conv_k = geom.conv_k
    d.attn_n_kv, d.attn_d_h, d.rope_dims = geom.attn_n_kv, geom.attn_d_h, geom.rope_dims
    d.rope_theta = geom.rope_theta
    d.norm_eps = geom.norm_eps
    d.n_draft_cols = geom.n_draft * geom.hidden
    d.max_T, d.max_seq = max_T, max_seq
    d.compute_dtype = _DT[dtype]
    return d


class Weights:
    """kva_weights over torch tensors (kept alive by this object).

    proj: g_in, W_in, blocks (g_attn, Wq, Wk, Wv, Wo, g_ffn, Wg, Wu, Wd each), g_out, W_heads.
    16-bit matrices give KVA_W_16.  Quantized matrices come with a "<name>_scale" tensor
    each (fp16 [K/32, N]): int8 codes [N, K] are q8_0, uint8 packed codes [N, K/2] q4_0.
    layer: conv_w, A_log, dt_bias, k_norm_g of the late layers."""

    def __init__(self, proj: Optional[Dict] = None, layer: Optional[Dict] = None):
        self._keep = []
        self.c = KvaWeights()
        if proj is not None:
            self.c.g_in = self._p(proj["g_in"])
            self.c.W_in = self._p(proj["W_in"])
            for i, b in enumerate(proj["blocks"]):
                cb = self.c.blocks[i]
                for name in ("g_attn", "Wq", "Wk", "Wv", "Wo", "g_ffn", "Wg", "Wu", "Wd"):
                    setattr(cb, name, self._p(b[name]))
            self.c.g_out = self._p(proj["g_out"])
            self.c.W_heads = self._p(proj["W_heads"])
            if "W_heads_scale" in proj:  # codes above (int8: q8_0, packed uint8: q4_0), fp16
                # scales [K/32, N] here
                fmt = {torch.uint8: KVA_W_Q4_0, torch.int8: KVA_W_Q8_0}.get(proj["W_heads"].dtype)
                if fmt is None:
                    raise ValueError("quantized W_heads must be int8 (q8_0) or uint8 (q4_0) codes")
                self.c.weight_format = fmt
                self.c.W_in_scale = self._p(proj["W_in_scale"])
                self.c.W_heads_scale = self._p(proj["W_heads_scale"])
                for i, b in enumerate(proj["blocks"]):
                    for j, name in enumerate(Q8_MATRICES):
                        self.c.block_scale[i][j] = self._p(b[name + "_scale"])
        if layer is not None:
            for name in ("conv_w", "A_log", "dt_bias", "k_norm_g"):
                setattr(self.c, name, self._p(layer[name]))

    def _p(self, t):
        self._keep.append(t)
        return _ptr(t)


class KvCache:
    """kva_kv_cache over lists of per-layer K and V tensors: bf16 / fp16 rows of d_h values,
    or uint8 rows of d_h * 34 / 32 bytes for the Hadamard-rotated q8_0 format."""

    def __init__(self, k: Sequence[torch.Tensor], v: Sequence[torch.Tensor], *,
                 max_pos: int = 0, page_table: Optional[torch.Tensor] = None,
                 page_size: int = 0, n_pages: int = 0):
        self._keep = list(k) + list(v)
        self.c = KvaKvCache()
        if len(k) and k[0].dtype == torch.uint8:
            self.c.dtype = KVA_Q8_0
        else:
            self.c.dtype = _DT[k[0].dtype] if len(k) else KVA_BF16
        self.c.n_layers = len(k)
        for i, (kk, vv) in enumerate(zip(k, v)):
            self.c.k[i] = _ptr(kk)
            self.c.v[i] = _ptr(vv)
        if page_table is None:
            self.c.layout = KVA_KV_CONTIGUOUS
            self.c.max_pos = max_pos
        else:
            self._keep.append(page_table)
            self.c.layout = KVA_KV_PAGED
            self.c.page_size = page_size
            self.c.n_pages = n_pages
            self.c.pages_per_seq = page_table.shape[-1]
            self.c.page_table = _ptr(page_table)


# ----------------------------------------------------------------- entry points
def kva_workspace_bytes(dims: KvaDims) -> int:
    return int(_lib.kva_workspace_bytes(C.byref(dims)))


def kva_init(dims: KvaDims) -> int:
    h = C.c_void_p()
    _check(_lib.kva_init(C.byref(dims), C.byref(h)), "kva_init")
    return h.value


def kva_free(handle: int) -> None:
    _lib.kva_free(handle)


def kva_prefill_ubatch(handle: int, residual: torch.Tensor, weights: Weights,
                       deltanet_state: torch.Tensor, conv_state: torch.Tensor,
                       kv: Optional[KvCache], pos: int, draft_out: Optional[torch.Tensor] = None,
                       mixer_out: Optional[torch.Tensor] = None, stream=None) -> None:
    dt = _DT[residual.dtype]
    _check(_lib.kva_prefill_ubatch(
        handle, _ptr(residual), dt, residual.shape[0], C.byref(weights.c), _ptr(deltanet_state),
        _ptr(conv_state), C.byref(kv.c) if kv is not None else None, int(pos), _ptr(draft_out),
        _ptr(mixer_out), _stream(stream)), "kva_prefill_ubatch")


def kva_update_states(handle: int, mixer_in: torch.Tensor, pos: Sequence[int], weights: Weights,
                      state: torch.Tensor, conv_state: torch.Tensor, kv: Optional[KvCache],
                      debug_qkv: Optional[torch.Tensor] = None,
                      debug_gb: Optional[torch.Tensor] = None, stream=None) -> None:
    n_seq, T, ld = mixer_in.shape
    pos_arr = (C.c_int64 * n_seq)(*[int(p) for p in pos])
    _check(_lib.kva_update_states(
        handle, _ptr(mixer_in), ld, n_seq, T, pos_arr, C.byref(weights.c), _ptr(state),
        _ptr(conv_state), C.byref(kv.c) if kv is not None else None, _ptr(debug_qkv),
        _ptr(debug_gb), _stream(stream)), "kva_update_states")


class LastParams:
    """kva_last_params: query heads of an attention layer, the gated RMSNorm weights of the
    gated-DeltaNet layers [n_gdn, d_v] and the q RMSNorm gains of the attention layers
    [n_attn, d_h] (fp32 device tensors)."""

    def __init__(self, attn_n_q: int, gdn_norm_w: Optional[torch.Tensor] = None,
                 q_norm_g: Optional[torch.Tensor] = None):
        self._keep = [t for t in (gdn_norm_w, q_norm_g) if t is not None]
        self.c = KvaLastParams()
        self.c.attn_n_q = attn_n_q
        self.c.gdn_norm_w = _ptr(gdn_norm_w)
        self.c.q_norm_g = _ptr(q_norm_g)


def kva_last_token_layer(handle: int, layer: int, x: torch.Tensor, pos: Sequence[int],
                         weights: Weights, last: LastParams, state: Optional[torch.Tensor],
                         conv_state: Optional[torch.Tensor], kv: Optional[KvCache], out: torch.Tensor,
                         stream=None) -> None:
    """The exact last-token pass through late layer `layer` for x.shape[0] sequences (see
    include/kva.h): x [n_seq, >= layer's input width] in the handle's compute dtype, out
    [n_seq, >= output width] fp32 or the compute dtype."""
    n_seq = x.shape[0]
    if x.stride(1) != 1 or out.stride(1) != 1:
        raise ValueError("x and out must be row-major")
    pos_arr = (C.c_int64 * max(1, n_seq))(*[int(p) for p in pos])
    _check(_lib.kva_last_token_layer(
        handle, layer, n_seq, _ptr(x), x.stride(0), pos_arr, C.byref(weights.c), C.byref(last.c),
        _ptr(state), _ptr(conv_state), C.byref(kv.c) if kv is not None else None, _ptr(out),
        _DT[out.dtype], out.stride(0), _stream(stream)), "kva_last_token_layer")


def kva_get_device_status(handle: int) -> int:
    s = C.c_int32()
    r = _lib.kva_get_device_status(handle, C.byref(s))
    if r not in (KVA_OK, KVA_ERR_DEVICE):
        _check(r, "kva_get_device_status")
    return s.value


def kva_stats(handle: int) -> int:
    n = C.c_int64()
    _check(_lib.kva_stats(handle, C.byref(n)), "kva_stats")
    return n.value


def kva_heads_fused(handle: int) -> bool:
    """True when kva_prefill_ubatch runs the state updates in the heads GEMM's epilogue."""
    f = C.c_int32()
    _check(_lib.kva_heads_fused(handle, C.byref(f)), "kva_heads_fused")
    return bool(f.value)


def kva_profile_enable(handle: int, capacity: int) -> None:
    _check(_lib.kva_profile_enable(handle, int(capacity)), "kva_profile_enable")


def kva_profile_read(handle: int) -> Dict[str, Dict[str, float]]:
    """Per stage: summed device ms, timed launches and enqueued launches since the last read."""
    p = KvaProfile()
    _check(_lib.kva_profile_read(handle, C.byref(p)), "kva_profile_read")
    return {n: {"ms": p.ms[i], "timed": p.timed[i], "launches": p.launches[i]}
            for i, n in enumerate(ST_NAMES)}


def kva_op_rmsnorm(x: torch.Tensor, g: torch.Tensor, out: torch.Tensor, eps: float = 1e-6,
                   stream=None) -> None:
    rows, n = x.shape
    _check(_lib.kva_op_rmsnorm(_ptr(x), _DT[x.dtype], n, _ptr(g), _ptr(out), _DT[out.dtype],
                               out.shape[1], rows, n, float(eps), _stream(stream)),
           "kva_op_rmsnorm")


def kva_op_gemm(A: torch.Tensor, B: Sequence[torch.Tensor], D: torch.Tensor, *, N: int,
                epilogue: int = EPI_STORE_BF16, b_mode: int = B_SINGLE, seg_rows: int = 0,
                D1: Optional[torch.Tensor] = None, n_split: int = 0, block_n: int = 0,
                err: Optional[torch.Tensor] = None, stream=None) -> None:
    M, K = A.shape
    arr = (C.c_void_p * 3)(*([_ptr(b) for b in B] + [None] * (3 - len(B))))
    _check(_lib.kva_op_gemm(
        _DT[A.dtype], _ptr(A), K, arr, b_mode, B[0].shape[1], seg_rows, _ptr(D), D.shape[1], _ptr(D1),
        D1.shape[1] if D1 is not None else 0, n_split, M, N, K, epilogue, block_n, _ptr(err),
        _stream(stream)), "kva_op_gemm")


def kva_op_gemm_q8_0(A: torch.Tensor, Bq: Sequence[torch.Tensor], Bs: Sequence[torch.Tensor],
                     D: torch.Tensor, *, N: int, epilogue: int = EPI_STORE_BF16, b_mode: int = B_SINGLE,
                     seg_rows: int = 0, err: Optional[torch.Tensor] = None, stream=None) -> None:
    """D = A dequant(B)^T with q8_0 weights: Bq[i] int8 [rows, K] codes, Bs[i] fp16 [K/32, rows]
    scales (see include/kva_ops.h)."""
    M, K = A.shape
    q = (C.c_void_p * 3)(*([_ptr(b) for b in Bq] + [None] * (3 - len(Bq))))
    sc = (C.c_void_p * 3)(*([_ptr(b) for b in Bs] + [None] * (3 - len(Bs))))
    _check(_lib.kva_op_gemm_q8_0(_DT[A.dtype], _ptr(A), K, q, sc, b_mode, seg_rows, _ptr(D), D.shape[1],
                                 M, N, K, epilogue, _ptr(err), _stream(stream)), "kva_op_gemm_q8_0")


def kva_op_gemm_q4_0(A: torch.Tensor, Bq: Sequence[torch.Tensor], Bs: Sequence[torch.Tensor],
                     D: torch.Tensor, *, N: int, epilogue: int = EPI_STORE_BF16, b_mode: int = B_SINGLE,
                     seg_rows: int = 0, err: Optional[torch.Tensor] = None, stream=None) -> None:
    """D = A dequant(B)^T with q4_0 weights: Bq[i] uint8 [rows, K/2] packed codes, Bs[i] fp16
    [K/32, rows] scales (see include/kva_ops.h)."""
    M, K = A.shape
    q = (C.c_void_p * 3)(*([_ptr(b) for b in Bq] + [None] * (3 - len(Bq))))
    sc = (C.c_void_p * 3)(*([_ptr(b) for b in Bs] + [None] * (3 - len(Bs))))
    _check(_lib.kva_op_gemm_q4_0(_DT[A.dtype], _ptr(A), K, q, sc, b_mode, seg_rows, _ptr(D), D.shape[1],
                                 M, N, K, epilogue, _ptr(err), _stream(stream)), "kva_op_gemm_q4_0")


def kva_op_attention(qkv: torch.Tensor, out: torch.Tensor, n_heads: int, window: int,
                     stream=None) -> None:
    T = qkv.shape[0]
    _check(_lib.kva_op_attention(_DT[qkv.dtype], _ptr(qkv), qkv.shape[1], _ptr(out), out.shape[1],
                                 T, n_heads, window, _stream(stream)), "kva_op_attention")


def kva_op_gdn_scan(k: torch.Tensor, v: torch.Tensor, gb: torch.Tensor, state: torch.Tensor,
                    n_seq: int, n_layers: int, n_k: int, n_v: int, d: int, stream=None) -> None:
    T = k.shape[-2]
    _check(_lib.kva_op_gdn_scan(_ptr(k), _ptr(v), _ptr(gb), _ptr(state), n_seq, n_layers, T, n_k,
                                n_v, d, _stream(stream)), "kva_op_gdn_scan")


def kva_gdn_layer_update_noalloc(mixer_in: torch.Tensor, n_k: int, n_v: int, d: int,
                                 conv_w: torch.Tensor, A_log: torch.Tensor, dt_bias: torch.Tensor,
                                 state: torch.Tensor, conv_state: torch.Tensor, eps: float = 1e-6,
                                 stream=None) -> None:
    """One gated-DeltaNet layer's state update without any device allocation (see
    include/kva_ops.h): for callers that may not allocate device memory.

    The entry point reads mixer_in and conv_state as bf16 and state as fp32, so other
    formats or sizes are refused here before anything reaches the device."""
    T, ld = mixer_in.shape
    C = 2 * n_k * d + n_v * d
    if mixer_in.dtype != torch.bfloat16 or conv_state.dtype != torch.bfloat16:
        raise ValueError("mixer_in and conv_state must be bf16")
    if state.dtype != torch.float32 or any(t.dtype != torch.float32 for t in (conv_w, A_log, dt_bias)):
        raise ValueError("state, conv_w, A_log and dt_bias must be fp32")
    if mixer_in.stride(1) != 1 or ld < C + 2 * n_v:
        raise ValueError(f"mixer_in must be row-major with at least {C + 2 * n_v} columns")
    ld = mixer_in.stride(0)
    for t, n, what in ((state, n_v * d * d, "state"), (conv_state, 3 * C, "conv_state"),
                       (conv_w, 4 * C, "conv_w"), (A_log, n_v, "A_log"), (dt_bias, n_v, "dt_bias")):
        if t.numel() != n or not t.is_contiguous():
            raise ValueError(f"{what} must be a contiguous tensor of {n} values, got {tuple(t.shape)}")
    _check(_lib.kva_gdn_layer_update_noalloc(
        _ptr(mixer_in), ld, T, n_k, n_v, d, _ptr(conv_w), _ptr(A_log), _ptr(dt_bias), _ptr(state),
        _ptr(conv_state), float(eps), _stream(stream)), "kva_gdn_layer_update_noalloc")


def kva_gdn_layer_update_noalloc_status(stream=None) -> int:
    """Device status bits of kva_gdn_layer_update_noalloc calls since the last read (0 =
    clean); synchronises the stream and clears the bits."""
    st = C.c_int32(0)
    rc = _lib.kva_gdn_layer_update_noalloc_status(_stream(stream), C.byref(st))
    if rc not in (KVA_OK, KVA_ERR_DEVICE):
        _check(rc, "kva_gdn_layer_update_noalloc_status")
    return st.value


def kva_test_gemm_wait_timeout(A: torch.Tensor, B: torch.Tensor, D: torch.Tensor, err: torch.Tensor,
                               stream=None) -> None:
    """The CTA-pair GEMM with one pipeline wait made to run out (see include/kva_ops.h): the
    kernel must come back with KVA_DEV_WAIT_TIMEOUT in the device int `err`."""
    M, K = A.shape
    N = B.shape[0]
    _check(_lib.kva_test_gemm_wait_timeout(_DT[A.dtype], _ptr(A), _ptr(B), _ptr(D), M, N, K, _ptr(err),
                                           _stream(stream)), "kva_test_gemm_wait_timeout")
