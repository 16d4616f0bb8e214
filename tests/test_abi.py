"""The C ABI library loads and exports every symbol the headers declare; host-side
validation rejects bad arguments before touching the GPU (no compute calls here)."""
import ctypes as C
import os
import re
import subprocess

import pytest

import kva_inputs as KI

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for h in ("kva.h", "kva_ops.h"):
        with open(os.path.join(ROOT, "include", h)) as f:
            txt = f.read()
        names |= set(re.findall(r"^\s*(?:int|void|size_t|const char\*)\s+(kva_\w+)\s*\(", txt, re.M))
    return names


def test_headers_declare_the_boundary():
    names = _declared()
    for n in ("kva_init", "kva_prefill_ubatch", "kva_update_states", "kva_free",
              "kva_get_device_status", "kva_strerror", "kva_stats", "kva_workspace_bytes",
              "kva_op_gemm", "kva_op_attention", "kva_op_rmsnorm", "kva_op_gdn_scan"):
        assert n in names


def test_library_exports_every_declared_symbol():
    import hybrid_deltanet_attention_kva_b200 as K
    out = subprocess.run(["nm", "-D", "--defined-only", K.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(kva_\w+)$", out, re.M))
    missing = _declared() - exported
    assert not missing, missing
    assert set(K.EXPORTED) <= exported


def test_binding_names_match_c_names():
    import hybrid_deltanet_attention_kva_b200 as K
    for n in _declared():
        assert hasattr(K, n), n


def test_struct_layouts_match_the_c_compiler(tmp_path):
    """sizeof / offsetof of every ABI struct, from gcc compiling the header, equal ctypes'."""
    import hybrid_deltanet_attention_kva_b200 as K
    fields = {"kva_dims": (K.KvaDims, ["rope_theta", "norm_eps", "max_seq", "layer_type"]),
              "kva_weights": (K.KvaWeights, ["blocks", "W_heads", "k_norm_g", "weight_format",
                                             "W_in_scale", "W_heads_scale", "block_scale"]),
              "kva_block_weights": (K.KvaBlockWeights, ["Wd"]),
              "kva_kv_cache": (K.KvaKvCache, ["v", "max_pos", "page_table"])}
    src = ["#include <stdio.h>", "#include <stddef.h>", '#include "kva.h"', "int main(void){"]
    for st, (_, fs) in fields.items():
        src.append(f'printf("{st} %zu\\n", sizeof({st}));')
        for f in fs:
            src.append(f'printf("{st}.{f} %zu\\n", offsetof({st}, {f}));')
    src.append("return 0;}")
    c = tmp_path / "layout.c"
    c.write_text("\n".join(src))
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(c), "-o", str(exe)], check=True)
    got = dict(line.split() for line in subprocess.run([str(exe)], capture_output=True, text=True,
                                                        check=True).stdout.splitlines())
    for st, (cls, fs) in fields.items():
        assert int(got[st]) == C.sizeof(cls), st
        for f in fs:
            assert int(got[f"{st}.{f}"]) == getattr(cls, f).offset, (st, f)


def test_workspace_and_strerror_without_gpu():
    import hybrid_deltanet_attention_kva_b200 as K
    for g in (KI.TINY, KI.R2, KI.R3):
        assert K.kva_workspace_bytes(K.make_dims(g, 1024, 1)) > 0
    bad = K.make_dims(KI.R3, 1024, 1)
    bad.head_dim = 64
    assert K.kva_workspace_bytes(bad) == 0
    bad = K.make_dims(KI.R3, 1024, 1)
    bad.conv_k = 3
    assert K.kva_workspace_bytes(bad) == 0
    bad = K.make_dims(KI.R3, 1024, 1)
    bad.layer_type[0] = 7
    assert K.kva_workspace_bytes(bad) == 0
    bad = K.make_dims(KI.R3, 1024, 1)
    bad.compute_dtype = K.KVA_F32                     # operands must be 16-bit
    assert K.kva_workspace_bytes(bad) == 0
    assert K.kva_strerror(K.KVA_ERR_TOO_LARGE).startswith("size beyond")
    assert K.kva_strerror(12345) == "unknown status"


def test_host_validation_rejects_before_any_launch():
    import hybrid_deltanet_attention_kva_b200 as K
    L = K.lib()
    h = C.c_void_p()
    assert L.kva_init(None, C.byref(h)) == K.KVA_ERR_INVALID_ARG
    d = K.make_dims(KI.R3, 1024, 1)
    d.n_late = 0
    assert L.kva_init(C.byref(d), C.byref(h)) == K.KVA_ERR_INVALID_ARG
    assert h.value is None
    # entry points refuse a null handle
    assert L.kva_prefill_ubatch(None, None, 0, 1, None, None, None, None, 0, None, None, None) \
        == K.KVA_ERR_INVALID_ARG
    assert L.kva_update_states(None, None, 0, 1, 1, None, None, None, None, None, None, None,
                               None) == K.KVA_ERR_INVALID_ARG
    n = C.c_int64()
    assert L.kva_stats(None, C.byref(n)) == K.KVA_ERR_INVALID_ARG
    f = C.c_int32()
    assert L.kva_heads_fused(None, C.byref(f)) == K.KVA_ERR_INVALID_ARG
    s = C.c_int32()
    assert L.kva_get_device_status(None, C.byref(s)) == K.KVA_ERR_INVALID_ARG
    # per-step ops: misaligned / invalid shapes are refused on the host
    assert L.kva_op_rmsnorm(C.c_void_p(16), 1, 6, C.c_void_p(16), C.c_void_p(16), 0, 6, 2, 6,
                            1e-6, None) == K.KVA_ERR_ALIGNMENT
    assert L.kva_op_rmsnorm(C.c_void_p(16), 1, 8, C.c_void_p(16), C.c_void_p(16), 1, 8, 2, 8,
                            1e-6, None) == K.KVA_ERR_INVALID_ARG          # fp32 out: refused
    arr = (C.c_void_p * 3)(16, None, None)
    assert L.kva_op_gemm(0, C.c_void_p(16), 12, arr, 0, 12, 0, C.c_void_p(16), 64, None, 0, 0,
                         64, 64, 12, 0, 0, None, None) == K.KVA_ERR_ALIGNMENT
    assert L.kva_op_gemm(0, C.c_void_p(16), 64, arr, 5, 64, 0, C.c_void_p(16), 64, None, 0, 0,
                         64, 64, 64, 0, 0, None, None) == K.KVA_ERR_INVALID_ARG
    assert L.kva_op_gemm(1, C.c_void_p(16), 64, arr, 0, 64, 0, C.c_void_p(16), 64, None, 0, 0,
                         64, 64, 64, 0, 0, None, None) == K.KVA_ERR_INVALID_ARG  # fp32 operands
    # quantized-weight GEMMs: K a multiple of 64, scales present and aligned, rows of 8
    one = (C.c_void_p * 3)(16, None, None)
    no_scale = (C.c_void_p * 3)(None, None, None)
    odd_scale = (C.c_void_p * 3)(8, None, None)
    for op in (L.kva_op_gemm_q8_0, L.kva_op_gemm_q4_0):
        assert op(0, C.c_void_p(16), 96, one, one, 0, 0, C.c_void_p(16), 64, 64, 64, 96, 0, None,
                  None) == K.KVA_ERR_UNSUPPORTED                        # K = 96
        assert op(0, C.c_void_p(16), 128, one, no_scale, 0, 0, C.c_void_p(16), 64, 64, 64, 128, 0,
                  None, None) == K.KVA_ERR_INVALID_ARG                  # no scales
        assert op(0, C.c_void_p(16), 128, one, odd_scale, 0, 0, C.c_void_p(16), 64, 64, 64, 128, 0,
                  None, None) == K.KVA_ERR_INVALID_ARG                  # misaligned scales
        assert op(0, C.c_void_p(16), 128, one, one, 0, 0, C.c_void_p(16), 64, 64, 60, 128, 0, None,
                  None) == K.KVA_ERR_ALIGNMENT                          # 60 scale rows
        assert op(0, C.c_void_p(16), 128, one, one, 3, 0, C.c_void_p(16), 64, 64, 64, 128, 0, None,
                  None) == K.KVA_ERR_INVALID_ARG                        # b_mode
        assert op(0, C.c_void_p(16), 128, None, one, 0, 0, C.c_void_p(16), 64, 64, 64, 128, 0, None,
                  None) == K.KVA_ERR_INVALID_ARG                        # no codes
        assert op(1, C.c_void_p(16), 128, one, one, 0, 0, C.c_void_p(16), 64, 64, 64, 128, 0, None,
                  None) == K.KVA_ERR_INVALID_ARG                        # fp32 operands
    assert L.kva_op_attention(0, C.c_void_p(16), 384, C.c_void_p(16), 128, 16, 1, -1, None) \
        == K.KVA_ERR_INVALID_ARG
    assert L.kva_op_gdn_scan(C.c_void_p(16), C.c_void_p(16), C.c_void_p(16), C.c_void_p(16), 1,
                             1, 8, 1, 1, 96, None) == K.KVA_ERR_UNSUPPORTED


def test_binding_constants_match_the_headers(tmp_path):
    """Every enumerator and status bit of the headers has the binding's value (compiled by gcc)."""
    import hybrid_deltanet_attention_kva_b200 as K
    names = set()
    for h in ("kva.h", "kva_ops.h"):
        with open(os.path.join(ROOT, "include", h)) as f:
            txt = f.read()
        for body in re.findall(r"typedef enum \w+ \{(.*?)\}", txt, re.S):
            names |= set(re.findall(r"\b(KVA_\w+)\s*=", body))
        names |= set(re.findall(r"^#define (KVA_DEV_\w+)", txt, re.M))
    assert {"KVA_W_Q4_0", "KVA_Q8_0", "KVA_EPI_SWIGLU_BF16", "KVA_DEV_WAIT_TIMEOUT"} <= names
    src = ["#include <stdio.h>", '#include "kva.h"', '#include "kva_ops.h"', "int main(void){"]
    src += [f'printf("{n} %d\\n", (int)({n}));' for n in sorted(names)]
    src.append("return 0;}")
    c = tmp_path / "consts.c"
    c.write_text("\n".join(src))
    exe = tmp_path / "consts"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(c), "-o", str(exe)], check=True)
    got = {a: int(b) for a, b in (line.split() for line in subprocess.run(
        [str(exe)], capture_output=True, text=True, check=True).stdout.splitlines())}
    for n, v in got.items():
        if n.startswith("KVA_ST_") and n != "KVA_ST_COUNT":  # stages: by name, in order
            assert K.ST_NAMES[v] == n[len("KVA_ST_"):].lower(), n
            continue
        # the binding drops the KVA_ prefix of the epilogue, B-mode and stage enumerators
        short = n[4:] if n.startswith(("KVA_EPI_", "KVA_B_", "KVA_ST_")) else n
        assert hasattr(K, short), n
        assert getattr(K, short) == v, (n, getattr(K, short), v)


def test_weight_format_follows_the_code_dtype(monkeypatch):
    """q8_0 for int8 codes, q4_0 for packed uint8 codes, an error for anything else (pointers
    faked: no device memory is touched)."""
    import torch
    import hybrid_deltanet_attention_kva_b200 as K
    from hybrid_deltanet_attention_kva_b200 import kva as kmod
    monkeypatch.setattr(kmod, "_ptr", lambda t: None if t is None else 16)
    names = ("Wq", "Wk", "Wv", "Wo", "Wg", "Wu", "Wd")

    def proj(codes_dtype, quant=True):
        z = torch.zeros(2, dtype=codes_dtype)
        blk = {"g_attn": z, "g_ffn": z, **{n: z for n in names}}
        p = {"g_in": z, "W_in": z, "g_out": z, "W_heads": z, "blocks": [blk]}
        if quant:
            p["W_in_scale"] = p["W_heads_scale"] = z
            blk.update({n + "_scale": z for n in names})
        return p

    assert K.Weights(proj=proj(torch.float16, quant=False)).c.weight_format == K.KVA_W_16
    assert K.Weights(proj=proj(torch.int8)).c.weight_format == K.KVA_W_Q8_0
    w4 = K.Weights(proj=proj(torch.uint8))
    assert w4.c.weight_format == K.KVA_W_Q4_0
    assert w4.c.W_heads_scale == 16 and w4.c.block_scale[0][6] == 16
    with pytest.raises(ValueError):
        K.Weights(proj=proj(torch.int16))
