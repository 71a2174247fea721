"""The MoE-layer workloads and their seeded inputs.

Shapes follow the layer the pages describe: Step3's 3-of-48 expert selection
with inter_dim 5120 and a fused shared expert (Step3 推論最適化 (MI308X vs H20),
§背景 and §最適化技術), the DP-attention all_gather that pads seven decode
ranks to the one prefill rank (DP Attention and TBO for DeepSeek-V4 on MI355X,
§PrefillDelayer), and the even 8192/8192 micro-batch split (same page, §TBOの
マイクロバッチ分割改善).  The DeepSeek-style and FP8 block-scale shapes come from
the same pages' DeepSeek and blockscale-GEMM mentions.  All values are drawn
from ``synth`` (Philox4x32-10), seed 0 unless stated.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import numpy as np

from . import (STREAM_ROUTER_B, STREAM_ROUTER_W, STREAM_W_DOWN, STREAM_W_GATE_UP,
               STREAM_WS_DOWN, STREAM_WS_GATE_UP, STREAM_X, STREAM_ZIPF_RANK,
               normal_bf16, normal_e4m3_blockscaled, normal_fp32_tensor, uniform_f64)


@dataclass(frozen=True)
class Workload:
    name: str
    T: int                      # rows of hidden states (valid + padding)
    H: int                      # hidden size
    E: int                      # routed experts
    k: int                      # experts per token
    I: int                      # routed expert intermediate size
    S: int = 0                  # shared experts (0 or 1)
    Is: int = 0                 # shared expert intermediate size
    wtype: str = "bf16"         # "bf16" or "fp8" (e4m3 + 128x128 fp32 scales)
    x_sigma: float = 1.0
    w_sigma: float = 0.02
    router_sigma: float | None = None   # None: 1/sqrt(H), i.e. logits ~ N(0, 1)
    bias: str = "none"          # "none" | "normal" (b_e ~ N(0,1)) | "zipf"
    zipf_s: float = 1.1
    mask: str = "all"           # "all" | "dp_padded"
    dp_rows: tuple = field(default=())   # valid rows per DP rank (dp_padded only)
    seed: int = 0

    @property
    def rsigma(self) -> float:
        return self.router_sigma if self.router_sigma is not None else 1.0 / math.sqrt(self.H)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    # T=16, hidden 256, 8 experts top-2, inter 128, no shared expert.
    "tiny": Workload("tiny", T=16, H=256, E=8, k=2, I=128, router_sigma=0.02),
    # Step3-like decode step: 3-of-48, inter 5120, one shared expert of inter 5120.
    "step3_decode": Workload("step3_decode", T=256, H=7168, E=48, k=3, I=5120, S=1, Is=5120),
    # DeepSeek-style decode step: 8-of-256, inter 2048, shared expert, skewed load
    # from a per-expert logit bias b_e ~ N(0, 1).
    "deepseek_decode": Workload("deepseek_decode", T=128, H=7168, E=256, k=8, I=2048, S=1,
                                Is=2048, bias="normal"),
    # DP-attention padded gather: 8 ranks x 1024 rows; rank 4 holds 1024 valid
    # rows (prefill), the other seven 16 each (decode); the rest is padding.
    "dp_padded": Workload("dp_padded", T=8192, H=7168, E=48, k=3, I=5120, mask="dp_padded",
                          dp_rows=(16, 16, 16, 16, 1024, 16, 16, 16)),
    # FP8 block-scale prefill micro-batch: 8192 tokens, 8-of-256, inter 2048,
    # shared expert, Zipf(1.1) expert popularity.
    "fp8_prefill": Workload("fp8_prefill", T=8192, H=7168, E=256, k=8, I=2048, S=1, Is=2048,
                            wtype="fp8", bias="zipf"),
}


def valid_mask(w: Workload) -> np.ndarray:
    """uint8 [T]: 1 for a real token, 0 for a padding row."""
    if w.mask == "all":
        return np.ones(w.T, dtype=np.uint8)
    if w.mask == "dp_padded":
        ranks = len(w.dp_rows)
        assert w.T % ranks == 0
        per = w.T // ranks
        m = np.zeros(w.T, dtype=np.uint8)
        for r, n in enumerate(w.dp_rows):
            m[r * per:r * per + n] = 1      # valid rows are the first n of a rank's block
        return m
    raise ValueError(w.mask)


def router_bias(w: Workload):
    import torch
    if w.bias == "none":
        return None
    if w.bias == "normal":
        return normal_fp32_tensor(w.seed, STREAM_ROUTER_B, (w.E,), 1.0)
    if w.bias == "zipf":
        # Zipf(s) popularity: expert e gets unnormalised mass r_e^-s, r a seeded
        # permutation of the ranks 1..E; as a logit bias that is -s ln r_e.
        u = uniform_f64(w.seed, STREAM_ZIPF_RANK, w.E)
        rank = np.empty(w.E, dtype=np.float64)
        rank[np.argsort(u, kind="stable")] = np.arange(1, w.E + 1)
        return torch.from_numpy((-w.zipf_s * np.log(rank)).astype(np.float32))
    raise ValueError(w.bias)


def make_inputs(w: Workload, masked_fill: str = "normal", with_weights: bool = True) -> dict:
    """All inputs of one forward pass as CPU tensors.

    x bf16 [T,H]; valid u8 [T]; router_w f32 [E,H]; router_b f32 [E] or None;
    bf16: w_gate_up [E,2I,H] (rows 0..I-1 gate, I..2I-1 up), w_down [E,H,I],
          ws_gate_up [2Is,H], ws_down [H,Is] (shared; None when S=0);
    fp8:  the same as uint8 e4m3 codes plus s_* f32 scales per 128x128 block.
    masked_fill: "normal" keeps the drawn values in padding rows, "nan" overwrites
    them with NaN (their contents must not matter).
    """
    import torch
    valid = valid_mask(w)
    x = normal_bf16(w.seed, STREAM_X, (w.T, w.H), w.x_sigma)
    if masked_fill == "nan":
        x[torch.from_numpy(valid == 0)] = float("nan")
    out = {"workload": w, "x": x, "valid": torch.from_numpy(valid),
           "router_w": normal_fp32_tensor(w.seed, STREAM_ROUTER_W, (w.E, w.H), w.rsigma),
           "router_b": router_bias(w)}
    if not with_weights:
        return out
    if w.wtype == "bf16":
        out["w_gate_up"] = normal_bf16(w.seed, STREAM_W_GATE_UP, (w.E, 2 * w.I, w.H), w.w_sigma)
        out["w_down"] = normal_bf16(w.seed, STREAM_W_DOWN, (w.E, w.H, w.I), w.w_sigma)
        if w.S:
            out["ws_gate_up"] = normal_bf16(w.seed, STREAM_WS_GATE_UP, (2 * w.Is, w.H), w.w_sigma)
            out["ws_down"] = normal_bf16(w.seed, STREAM_WS_DOWN, (w.H, w.Is), w.w_sigma)
        else:
            out["ws_gate_up"] = out["ws_down"] = None
    elif w.wtype == "fp8":
        q, s = normal_e4m3_blockscaled(w.seed, STREAM_W_GATE_UP, w.E, 2 * w.I, w.H, w.w_sigma)
        out["w_gate_up"], out["s_gate_up"] = q, s
        q, s = normal_e4m3_blockscaled(w.seed, STREAM_W_DOWN, w.E, w.H, w.I, w.w_sigma)
        out["w_down"], out["s_down"] = q, s
        if w.S:
            q, s = normal_e4m3_blockscaled(w.seed, STREAM_WS_GATE_UP, 1, 2 * w.Is, w.H, w.w_sigma)
            out["ws_gate_up"], out["ss_gate_up"] = q[0], s[0]
            q, s = normal_e4m3_blockscaled(w.seed, STREAM_WS_DOWN, 1, w.H, w.Is, w.w_sigma)
            out["ws_down"], out["ss_down"] = q[0], s[0]
        else:
            out["ws_gate_up"] = out["ws_down"] = out["ss_gate_up"] = out["ss_down"] = None
    else:
        raise ValueError(w.wtype)
    return out
