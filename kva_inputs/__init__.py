"""Seeded synthetic inputs for the KVA prefill path.

This module is the one piece shared by the CPU oracle (``oracle/``) and the
CUDA path (``hybrid_deltanet_attention_kva_b200``): it draws random tensors of
the right shapes, dtypes and distributions and describes the geometries.  It
holds none of the method's arithmetic (no norm, no projection, no scan, no
rotary table): only random draws, shape bookkeeping and dtype casts.

Geometry facts, each from the pages:
  * projector widths and FFN sizes r2 / r3 -- "Qwen3.8-27B-KVA" model card,
    architecture table (width d, heads @ 128, SwiGLU FFN, trunk/heads/total).
  * per-late-layer mixer widths (10240 + 48 + 48 per gated-DeltaNet layer,
    1024 + 1024 per full-attention layer) -- same card, the late-layer table of
    "What the hell?".
  * 48 gated-DeltaNet + 16 full-attention layers in 64, late half 32..63 --
    same card, "What the hell?" section.
  * 4 KV heads of dim 256 and 64 rotary dims per KV head -- "Qwen3.8-27B-MLA"
    model card, "What this is" section.
  * drafter heads kva.res.34 / 48 / 62 and kva.final, 5120 wide each -- KVA
    card, architecture table row "drafter heads".

Readings taken where the pages are silent:
  * late-layer order: full attention at every 4th layer (35, 39, ..., 63);
  * the q/k/v split inside the 10240 is [q | k | v], head-major;
  * synthetic distributions follow the workload descriptions of the five
    configurations (residual N(0,1) with 8 outlier channels x20, weights
    N(0, 0.02) in bf16, conv weights N(0, 0.5), A_log U(0, 2.7),
    dt_bias N(0, 0.5), unit norm gains), as listed per workload below.

Random draws use ``torch.Generator`` seeded per tensor (CPU by default, so the
values are identical on every machine with this torch build; ``device='cuda'``
draws on the GPU for large benchmark weights, where only the distribution
matters).
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass, field
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np
import torch

GDN = 0
ATTN = 1


@dataclass(frozen=True)
class Geometry:
    """Shapes of one projector + late-layer stack."""

    name: str
    hidden: int            # H: width of the layer-31 residual (5120)
    d_model: int           # d: projector width
    n_heads: int           # projector attention heads
    ffn: int               # SwiGLU hidden width
    layer_types: Tuple[int, ...]  # GDN / ATTN per late layer, in layer order
    gdn_n_k: int           # q/k heads per gated-DeltaNet layer
    gdn_n_v: int           # v heads per gated-DeltaNet layer
    gdn_d_k: int           # q/k head dim
    gdn_d_v: int           # v head dim
    attn_n_kv: int         # KV heads per attention layer
    attn_d_h: int          # KV head dim
    rope_dims: int         # rotary dims at the start of each KV head
    window: int = 0        # projector block-causal window (0: causal over the ubatch)
    n_draft: int = 0       # drafter heads (each `hidden` wide)
    head_dim: int = 128    # projector head dim
    n_blocks: int = 3
    conv_k: int = 4
    rope_theta: float = 1.0e7
    norm_eps: float = 1.0e-6
    attn_n_q: int = 24     # query heads of an attention layer (exact last-token pass only)

    # ---- derived sizes (bookkeeping only) ----
    @property
    def gdn_conv_ch(self) -> int:
        return 2 * self.gdn_n_k * self.gdn_d_k + self.gdn_n_v * self.gdn_d_v

    @property
    def gdn_width(self) -> int:
        return self.gdn_conv_ch + 2 * self.gdn_n_v

    @property
    def attn_width(self) -> int:
        return 2 * self.attn_n_kv * self.attn_d_h

    @property
    def n_late(self) -> int:
        return len(self.layer_types)

    @property
    def n_gdn(self) -> int:
        return sum(1 for t in self.layer_types if t == GDN)

    @property
    def n_attn(self) -> int:
        return sum(1 for t in self.layer_types if t == ATTN)

    def layer_width(self, i: int) -> int:
        return self.gdn_width if self.layer_types[i] == GDN else self.attn_width

    @property
    def layer_offsets(self) -> List[int]:
        offs, o = [], 0
        for i in range(self.n_late):
            offs.append(o)
            o += self.layer_width(i)
        return offs

    @property
    def n_mix(self) -> int:
        return sum(self.layer_width(i) for i in range(self.n_late))

    @property
    def n_draft_cols(self) -> int:
        return self.n_draft * self.hidden

    @property
    def n_total(self) -> int:
        return self.n_mix + self.n_draft_cols

    def last_width(self, i: int) -> int:
        """Columns of layer i's exact last-token inputs: the mixer columns of the layer, then
        the output gate z (n_v * d_v) of a gated-DeltaNet layer, or q and its gate
        (2 * n_q * d_h) of an attention layer."""
        if self.layer_types[i] == GDN:
            return self.gdn_width + self.gdn_n_v * self.gdn_d_v
        return self.attn_width + 2 * self.attn_n_q * self.attn_d_h

    def gdn_layers(self) -> List[int]:
        return [i for i, t in enumerate(self.layer_types) if t == GDN]

    def attn_layers(self) -> List[int]:
        return [i for i, t in enumerate(self.layer_types) if t == ATTN]

    def param_counts(self) -> Dict[str, int]:
        """Linear-weight parameter counts (norm gains listed separately)."""
        d, H, F = self.d_model, self.hidden, self.ffn
        trunk_lin = H * d + self.n_blocks * (4 * d * d + 3 * d * F)
        trunk_gain = H + self.n_blocks * 2 * d + d
        return {
            "trunk": trunk_lin + trunk_gain,
            "heads": self.n_mix * d,
            "drafter": self.n_draft_cols * d,
            "total": trunk_lin + trunk_gain + self.n_total * d,
        }


def late_layer_types_every4(n_late: int = 32, first_layer: int = 32) -> Tuple[int, ...]:
    """Full attention at every 4th layer of the 64-layer stack (35, 39, ... 63)."""
    return tuple(ATTN if (first_layer + i + 1) % 4 == 0 else GDN for i in range(n_late))


R2 = Geometry(name="r2", hidden=5120, d_model=2560, n_heads=20, ffn=7040,
              layer_types=late_layer_types_every4(), gdn_n_k=16, gdn_n_v=48,
              gdn_d_k=128, gdn_d_v=128, attn_n_kv=4, attn_d_h=256, rope_dims=64,
              window=0, n_draft=0)
R3 = Geometry(name="r3", hidden=5120, d_model=3072, n_heads=24, ffn=8448,
              layer_types=late_layer_types_every4(), gdn_n_k=16, gdn_n_v=48,
              gdn_d_k=128, gdn_d_v=128, attn_n_kv=4, attn_d_h=256, rope_dims=64,
              window=1024, n_draft=4)
TINY = Geometry(name="tiny", hidden=512, d_model=256, n_heads=2, ffn=704,
                layer_types=(GDN, GDN, ATTN), gdn_n_k=2, gdn_n_v=4, gdn_d_k=64,
                gdn_d_v=64, attn_n_kv=1, attn_d_h=128, rope_dims=32, window=0,
                n_draft=0, attn_n_q=2)

GEOMETRIES = {"tiny": TINY, "r2": R2, "r3": R3}


def with_changes(geom: Geometry, **kw) -> Geometry:
    return dataclasses.replace(geom, **kw)


# --------------------------------------------------------------------------
# random draws
# --------------------------------------------------------------------------
class Draw:
    """Sequence of seeded tensors: tensor number i is drawn from seed*65537+i."""

    def __init__(self, seed: int, device: str = "cpu"):
        self.seed = int(seed)
        self.i = 0
        self.device = device

    def _gen(self) -> torch.Generator:
        g = torch.Generator(device=self.device)
        g.manual_seed(self.seed * 65537 + self.i)
        self.i += 1
        return g

    def normal(self, shape, std=1.0, mean=0.0, dtype=torch.float32) -> torch.Tensor:
        x = torch.randn(tuple(shape), generator=self._gen(), device=self.device,
                        dtype=torch.float32)
        if std != 1.0:
            x.mul_(std)
        if mean != 0.0:
            x.add_(mean)
        return x.to(dtype)

    def uniform(self, shape, lo, hi, dtype=torch.float32) -> torch.Tensor:
        x = torch.rand(tuple(shape), generator=self._gen(), device=self.device,
                       dtype=torch.float32)
        return (x * (hi - lo) + lo).to(dtype)

    def permutation(self, n: int) -> torch.Tensor:
        return torch.randperm(n, generator=self._gen(), device=self.device)


def make_residual(geom: Geometry, T: int, seed: int, dtype=torch.bfloat16,
                  n_outliers: int = 8, outlier_scale: float = 20.0,
                  device: str = "cpu") -> torch.Tensor:
    """Layer-31 residual stand-in [T, H]: N(0,1), a seeded set of channels x scale."""
    dr = Draw(seed, device)
    x = dr.normal((T, geom.hidden))
    if n_outliers:
        ch = dr.permutation(geom.hidden)[:n_outliers]
        x[:, ch] *= outlier_scale
    return x.to(dtype)


def make_projector_weights(geom: Geometry, seed: int, std: float = 0.02,
                           random_gains: bool = False,
                           device: str = "cpu") -> Dict[str, object]:
    """Projector weights, row-major [out, in] bf16; RMSNorm gains fp32."""
    dr = Draw(seed, device)
    d, H, F = geom.d_model, geom.hidden, geom.ffn
    bf = torch.bfloat16

    def gain(n):
        if random_gains:
            return dr.uniform((n,), 0.5, 1.5)
        return torch.ones(n, dtype=torch.float32, device=device)

    w: Dict[str, object] = {}
    w["g_in"] = gain(H)
    w["W_in"] = dr.normal((d, H), std, dtype=bf)
    blocks = []
    for _ in range(geom.n_blocks):
        b = {}
        b["g_attn"] = gain(d)
        for name in ("Wq", "Wk", "Wv", "Wo"):
            b[name] = dr.normal((d, d), std, dtype=bf)
        b["g_ffn"] = gain(d)
        b["Wg"] = dr.normal((F, d), std, dtype=bf)
        b["Wu"] = dr.normal((F, d), std, dtype=bf)
        b["Wd"] = dr.normal((d, F), std, dtype=bf)
        blocks.append(b)
    w["blocks"] = blocks
    w["g_out"] = gain(d)
    w["W_heads"] = dr.normal((geom.n_total, d), std, dtype=bf)
    return w


def make_layer_params(geom: Geometry, seed: int, random_k_gain: bool = False,
                      device: str = "cpu") -> Dict[str, torch.Tensor]:
    """Base-model parameters the state updates need, per late layer."""
    dr = Draw(seed, device)
    p = {
        "conv_w": dr.normal((geom.n_gdn, geom.gdn_conv_ch, geom.conv_k), 0.5),
        "A_log": dr.uniform((geom.n_gdn, geom.gdn_n_v), 0.0, 2.7),
        "dt_bias": dr.normal((geom.n_gdn, geom.gdn_n_v), 0.5),
    }
    if random_k_gain:
        p["k_norm_g"] = dr.uniform((geom.n_attn, geom.attn_d_h), 0.5, 1.5)
    else:
        p["k_norm_g"] = torch.ones(geom.n_attn, geom.attn_d_h, dtype=torch.float32,
                                   device=device)
    return p


def make_states(geom: Geometry, n_seq: int, seed: int, std: float = 0.0,
                device: str = "cpu") -> Dict[str, torch.Tensor]:
    """Initial recurrent state fp32 [n_seq, n_gdn, n_v, d_v, d_k] and conv tail
    bf16 [n_seq, n_gdn, conv_k-1, C] (zero unless std > 0)."""
    dr = Draw(seed, device)
    shp = (n_seq, geom.n_gdn, geom.gdn_n_v, geom.gdn_d_v, geom.gdn_d_k)
    tshp = (n_seq, geom.n_gdn, geom.conv_k - 1, geom.gdn_conv_ch)
    if std > 0:
        S = dr.normal(shp, std)
        tail = dr.normal(tshp, 1.0, dtype=torch.bfloat16)
    else:
        S = torch.zeros(shp, dtype=torch.float32, device=device)
        tail = torch.zeros(tshp, dtype=torch.bfloat16, device=device)
    return {"state": S, "conv_tail": tail}


def make_mixer_inputs(geom: Geometry, n_seq: int, T: int, seed: int,
                      device: str = "cpu") -> torch.Tensor:
    """Precomputed mixer inputs bf16 [n_seq, T, n_mix], N(0,1)."""
    dr = Draw(seed, device)
    return dr.normal((n_seq, T, geom.n_mix), 1.0, dtype=torch.bfloat16)


def make_last_token_inputs(geom: Geometry, layer: int, n_seq: int, seed: int,
                           device: str = "cpu") -> torch.Tensor:
    """Exact inputs of one late layer for the last token of n_seq sequences, bf16
    [n_seq, last_width(layer)], N(0,1)."""
    dr = Draw(seed, device)
    return dr.normal((n_seq, geom.last_width(layer)), 1.0, dtype=torch.bfloat16)


def make_last_token_params(geom: Geometry, seed: int, random_gains: bool = False,
                           device: str = "cpu") -> Dict[str, torch.Tensor]:
    """Gains of the exact last-token pass: the gated RMSNorm weight of each gated-DeltaNet
    layer [n_gdn, d_v] and the q RMSNorm gain of each attention layer [n_attn, d_h]; 1, or
    U(0.5, 1.5) with random_gains."""
    dr = Draw(seed, device)
    shapes = {"gdn_norm_w": (geom.n_gdn, geom.gdn_d_v), "q_norm_g": (geom.n_attn, geom.attn_d_h)}
    if random_gains:
        return {k: dr.uniform(v, 0.5, 1.5) for k, v in shapes.items()}
    return {k: torch.ones(v, dtype=torch.float32, device=device) for k, v in shapes.items()}


def make_page_table(n_seq: int, pages_per_seq: int, seed: int,
                    n_pages: Optional[int] = None) -> torch.Tensor:
    """Shuffled page table int32 [n_seq, pages_per_seq] over a pool of n_pages."""
    n_pages = n_pages or n_seq * pages_per_seq
    dr = Draw(seed)
    perm = dr.permutation(n_pages)[: n_seq * pages_per_seq]
    return perm.reshape(n_seq, pages_per_seq).to(torch.int32)


# --------------------------------------------------------------------------
# the five workloads
# --------------------------------------------------------------------------
@dataclass
class Workload:
    name: str
    geom: Geometry
    ubatches: List[int]            # token counts per ubatch, in order
    residual_dtype: torch.dtype
    seed: int
    n_seq: int = 1
    state_std: float = 0.0
    paged: bool = False
    page_size: int = 256
    max_pos: int = 0
    n_outliers: int = 8
    projector: bool = True
    notes: str = ""

    @property
    def total_tokens(self) -> int:
        return self.n_seq * sum(self.ubatches)


def workload(idx: int) -> Workload:
    """Standard workload idx in 1..5: tiny T=128, r2 T=1024, r3 1024+512,
    r3 32x1024 long prompt, state-only 8 sequences x 4096 tokens."""
    seed = 1000 + idx
    if idx == 1:
        return Workload("tiny T=128", TINY, [128], torch.float32, seed, max_pos=128,
                        n_outliers=0)
    if idx == 2:
        return Workload("r2 T=1024", R2, [1024], torch.bfloat16, seed, max_pos=1024)
    if idx == 3:
        return Workload("r3 1024+512", R3, [1024, 512], torch.bfloat16, seed,
                        max_pos=1536)
    if idx == 4:
        return Workload("r3 32x1024", R3, [1024] * 32, torch.bfloat16, seed,
                        max_pos=32768)
    if idx == 5:
        return Workload("state-only 8x4096", with_changes(R3, n_draft=0), [1024] * 4,
                        torch.bfloat16, seed, n_seq=8, state_std=0.1, paged=True,
                        page_size=256, max_pos=4096, projector=False)
    raise ValueError(idx)


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact widening of a (bf16 / fp32) tensor to a float64 numpy array."""
    return t.detach().to("cpu").to(torch.float64).numpy()
