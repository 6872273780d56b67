"""Seeded synthetic inputs for the MoE layer workloads.

This module only draws random numbers and builds input tensors.  It holds none
of the layer's arithmetic, so both the fp64 oracle (test side) and the CUDA
path use it without sharing any computation.

Recipe (same for every workload):
  * one ``torch.Generator`` per workload, seeded ``1000 + workload number``;
  * draw order: x, then W_g, then W1 (GELU) / W_gu (SwiGLU) expert by expert,
    then W2 / W_down expert by expert, then (only when asked) b1 and b2;
  * x ~ N(0, 1); weight matrices ~ N(0, w_std); expert biases 0 unless
    ``random_bias`` is set (then N(0, 0.02));
  * bf16 tensors are drawn in fp32 and rounded to bf16 (round to nearest even);
  * the skewed workloads add a per-expert router bias b_g[e] = -s ln(e + 1)
    (Zipf-like, s = 1), so expert 0 is the most loaded;
  * a shared expert (when the workload has one) is drawn last, after all of
    the above: S1 (H or 2H rows) then S2, N(0, w_std), then its biases like
    the experts' (GELU with biases);
  * a selection-only bias (when the workload has one) is b_sel[e] =
    sel_s ln(e + 1): with sel_s = s it cancels the Zipf skew for the choice of
    experts (the balanced state DeepSeek-V3's bias adjustment aims at) while
    the gate weights keep the skewed scores.

Layouts: x [T, D]; W_g [D, N]; W1 [N, H, D] or W_gu [N, 2H, D] (gate rows first,
then up rows); W2 / W_down [N, D, H]; b_g [N], b1 [N, H], b2 [N, D] in fp32.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import torch

ACT_GELU, ACT_SWIGLU = 0, 1


@dataclass(frozen=True)
class Workload:
    name: str
    number: int           # 1-based workload number; the seed is 1000 + number
    T: int
    D: int
    H: int
    N: int
    K: int
    act: int              # ACT_GELU / ACT_SWIGLU
    dtype: torch.dtype    # x, weight matrices and the hidden activations
    has_bias: bool        # expert biases b1 / b2 present
    w_std: float
    zipf_s: float = 0.0   # router bias strength; 0 = no router bias
    random_bias: bool = False
    n_shared: int = 0     # 1: a shared expert every token passes through
    sel_s: float = 0.0    # selection-only bias strength; 0 = none
    capacity_factor: float = 0.0   # per-expert capacity ceil(cf T K / N); 0 = no limit
    overflow: int = 0     # with a capacity: 0 drop, 1 reroute to the next candidate

    @property
    def seed(self) -> int:
        return 1000 + self.number

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    # tiny fp32 layer, GELU experts with (zero) biases, no router bias
    "tiny": Workload("tiny", 1, 512, 64, 256, 8, 2, ACT_GELU, torch.float32, True, 0.02),
    # GPT-2-small width, 6 experts, top-2, GELU with biases, bf16
    "gpt2": Workload("gpt2", 2, 8192, 768, 3072, 6, 2, ACT_GELU, torch.bfloat16, True, 0.02),
    # Mixtral-8x7B shape, SwiGLU, Zipf-skewed router
    "mixtral": Workload("mixtral", 3, 4096, 4096, 14336, 8, 2, ACT_SWIGLU, torch.bfloat16, False, 0.02, 1.0),
    # DeepSeek-V3 shape, 256 fine-grained experts, top-8, uniform router
    "deepseek": Workload("deepseek", 4, 16384, 7168, 2048, 256, 8, ACT_SWIGLU, torch.bfloat16, False, 0.006),
    # same, Zipf-skewed router
    "deepseek_zipf": Workload("deepseek_zipf", 4, 16384, 7168, 2048, 256, 8, ACT_SWIGLU, torch.bfloat16,
                              False, 0.006, 1.0),
    # DeepSeek-V3 shape with its shared expert and a selection-only bias that cancels the Zipf skew
    "deepseek_shared": Workload("deepseek_shared", 6, 16384, 7168, 2048, 256, 8, ACT_SWIGLU, torch.bfloat16,
                                False, 0.006, 1.0, n_shared=1, sel_s=1.0),
    # gpt-oss-20b decode shape (T = 1, 8 or 64)
    "decode1": Workload("decode1", 5, 1, 2880, 2880, 32, 4, ACT_SWIGLU, torch.bfloat16, False, 0.02),
    "decode8": Workload("decode8", 5, 8, 2880, 2880, 32, 4, ACT_SWIGLU, torch.bfloat16, False, 0.02),
    "decode64": Workload("decode64", 5, 64, 2880, 2880, 32, 4, ACT_SWIGLU, torch.bfloat16, False, 0.02),
}


def _randn(shape, g, device, std=1.0):
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32) * std


def make_inputs(wl: Workload, device="cpu", T: int | None = None, seed: int | None = None):
    """Draw one workload's inputs. Returns a dict of tensors on ``device``.

    ``T`` overrides the token count (x is drawn first, so weights do not depend
    on T only when T is unchanged; callers that need the same weights at two
    token counts draw the larger T and slice).
    """
    T = wl.T if T is None else T
    g = torch.Generator(device=device)
    g.manual_seed(wl.seed if seed is None else seed)
    D, H, N = wl.D, wl.H, wl.N
    rows1 = H if wl.act == ACT_GELU else 2 * H
    out = {}
    out["x"] = _randn((T, D), g, device).to(wl.dtype)
    out["W_g"] = _randn((D, N), g, device, wl.w_std).to(wl.dtype)
    W1 = torch.empty((N, rows1, D), dtype=wl.dtype, device=device)
    for e in range(N):
        W1[e] = _randn((rows1, D), g, device, wl.w_std).to(wl.dtype)
    W2 = torch.empty((N, D, H), dtype=wl.dtype, device=device)
    for e in range(N):
        W2[e] = _randn((D, H), g, device, wl.w_std).to(wl.dtype)
    out["W1"], out["W2"] = W1, W2
    if wl.has_bias:
        if wl.random_bias:
            out["b1"] = _randn((N, H), g, device, 0.02)
            out["b2"] = _randn((N, D), g, device, 0.02)
        else:
            out["b1"] = torch.zeros((N, H), dtype=torch.float32, device=device)
            out["b2"] = torch.zeros((N, D), dtype=torch.float32, device=device)
    else:
        out["b1"] = out["b2"] = None
    if wl.zipf_s:
        out["b_g"] = torch.tensor([-wl.zipf_s * math.log(e + 1) for e in range(N)], dtype=torch.float32,
                                  device=device)
    else:
        out["b_g"] = None
    out["S1"] = out["S2"] = out["sb1"] = out["sb2"] = None
    if wl.n_shared:
        out["S1"] = _randn((rows1, D), g, device, wl.w_std).to(wl.dtype)
        out["S2"] = _randn((D, H), g, device, wl.w_std).to(wl.dtype)
        if wl.has_bias:
            if wl.random_bias:
                out["sb1"] = _randn((H,), g, device, 0.02)
                out["sb2"] = _randn((D,), g, device, 0.02)
            else:
                out["sb1"] = torch.zeros((H,), dtype=torch.float32, device=device)
                out["sb2"] = torch.zeros((D,), dtype=torch.float32, device=device)
    out["b_sel"] = (torch.tensor([wl.sel_s * math.log(e + 1) for e in range(N)], dtype=torch.float32, device=device)
                    if wl.sel_s else None)
    return out


def bf16_bits(t: torch.Tensor):
    """Host numpy view of a tensor's storage: float32 as is, bf16 as uint16 bit patterns."""
    t = t.detach().contiguous().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view("uint16")
    return t.numpy()
