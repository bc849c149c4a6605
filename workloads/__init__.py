"""Seeded synthetic inputs for the five attention workloads.

This module is the only code shared by the CUDA path's tests/bench and the CPU
oracle.  It draws random tensors and rounds them to bf16; it holds none of the
attention arithmetic.

Recipe (the same for every consumer):

* One ``torch.Generator`` on the requested device, seeded with
  ``1000 + workload index`` unless a seed is given.  CPU and CUDA generators
  produce different streams for the same seed; both sides of a comparison are
  always handed the *same* tensors, so that never matters for parity.
* Prefill: Q, K, V, dO drawn in that order as fp32 i.i.d. N(0,1) in
  [B, T, H, d] layout, then rounded to bf16 (round-to-nearest-even).
* Outlier keys (the long-context GQA workload): after dO, one ``randperm`` of
  the T token positions per (b, kv head); the first round(0.01 * T) positions
  have all d entries of K multiplied by 4 (exact in bf16).
* E4M3 prefill (the FP8 forward): the same Q, K, V draws as prefill (outlier
  keys included), each tensor then quantised with one factor
  descale = amax(|x|) / 448 as code = E4M3(x / descale), rounded to nearest
  by torch's float8_e4m3fn conversion.  The codes and the three factors are
  the inputs; both sides read the same codes.
* Decode: seqlens ~ integer-uniform on [1024, 32768] inclusive, then q
  [B, Hq, d], then per sequence b the K and V cache rows [Tk_max, Hkv, d], all
  fp32 N(0,1) rounded to bf16.  Only the first seqlens[b] rows are read.

The page workloads these mirror: the GPT-2-medium layer timed in the memory-
bound section ("Efficient attention: memory-bound", opening figure), the
Llama-style 32-head d=128 layer at T=8192 of the same page, the 32k-token fine-
tuning example of the "FlashAttention" interview page, and FlashDecoding.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import numpy as np
import torch

__all__ = ["Workload", "WORKLOADS", "prefill_inputs", "prefill_inputs_e4m3", "decode_inputs", "to_f64"]


@dataclass(frozen=True)
class Workload:
    index: int
    name: str
    B: int
    Hq: int
    Hkv: int
    T: int            # Tq == Tk for prefill; Tk_max for decode
    d: int
    causal: bool
    decode: bool = False
    outlier_frac: float = 0.0
    outlier_scale: float = 1.0
    tk_lo: int = 0
    tk_hi: int = 0
    chunk: int = 256
    window: int = 0   # > 0: sliding window of that many keys (implies causal)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def seed(self) -> int:
        return 1000 + self.index

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    1: Workload(1, "selfattn_b1_h1_t128_d64", B=1, Hq=1, Hkv=1, T=128, d=64, causal=False),
    2: Workload(2, "gpt2medium_b64_h16_t1024_d64", B=64, Hq=16, Hkv=16, T=1024, d=64, causal=False),
    3: Workload(3, "causal_b4_h32_t8192_d128", B=4, Hq=32, Hkv=32, T=8192, d=128, causal=True),
    4: Workload(4, "gqa_causal_b1_hq32_hkv8_t32768_d128_outliers", B=1, Hq=32, Hkv=8, T=32768,
                d=128, causal=True, outlier_frac=0.01, outlier_scale=4.0),
    5: Workload(5, "decode_splitkv_b64_hq32_hkv8_d128", B=64, Hq=32, Hkv=8, T=32768, d=128,
                causal=False, decode=True, tk_lo=1024, tk_hi=32768, chunk=256),
}


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _normal_bf16(shape, g, device):
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32).to(torch.bfloat16)


def prefill_inputs(w: Workload, device="cpu", seed=None, Tq=None, Tk=None):
    """Q, K, V, dO (bf16, BTHD) for a prefill workload.  ``Tq``/``Tk`` override
    the lengths for edge cases (Tq != Tk)."""
    Tq = w.T if Tq is None else Tq
    Tk = w.T if Tk is None else Tk
    g = _gen(device, w.seed if seed is None else seed)
    q = torch.randn((w.B, Tq, w.Hq, w.d), generator=g, device=device)
    k = torch.randn((w.B, Tk, w.Hkv, w.d), generator=g, device=device)
    v = torch.randn((w.B, Tk, w.Hkv, w.d), generator=g, device=device)
    do = torch.randn((w.B, Tq, w.Hq, w.d), generator=g, device=device)
    outliers = None
    if w.outlier_frac > 0 and Tk > 0:
        n_out = int(round(w.outlier_frac * Tk))
        outliers = torch.empty((w.B, w.Hkv, n_out), dtype=torch.int64, device=device)
        for b in range(w.B):
            for h in range(w.Hkv):
                idx = torch.randperm(Tk, generator=g, device=device)[:n_out]
                outliers[b, h] = idx
                k[b, idx, h, :] *= w.outlier_scale
    out = {n: t.to(torch.bfloat16).contiguous() for n, t in
           (("q", q), ("k", k), ("v", v), ("do", do))}
    out["outlier_rows"] = outliers
    return out


def prefill_inputs_e4m3(w: Workload, device="cpu", seed=None, Tq=None, Tk=None):
    """E4M3 codes of Q, K, V (torch.float8_e4m3fn, BTHD) and their descale
    factors, from the fp32 draws of ``prefill_inputs`` (same seed, same
    outlier keys) quantised per tensor with amax / 448."""
    Tq = w.T if Tq is None else Tq
    Tk = w.T if Tk is None else Tk
    g = _gen(device, w.seed if seed is None else seed)
    q = torch.randn((w.B, Tq, w.Hq, w.d), generator=g, device=device)
    k = torch.randn((w.B, Tk, w.Hkv, w.d), generator=g, device=device)
    v = torch.randn((w.B, Tk, w.Hkv, w.d), generator=g, device=device)
    if w.outlier_frac > 0 and Tk > 0:
        torch.randn((w.B, Tq, w.Hq, w.d), generator=g, device=device)   # dO's draw, to keep the stream aligned
        n_out = int(round(w.outlier_frac * Tk))
        for b in range(w.B):
            for h in range(w.Hkv):
                idx = torch.randperm(Tk, generator=g, device=device)[:n_out]
                k[b, idx, h, :] *= w.outlier_scale
    out = {}
    for n, t in (("q", q), ("k", k), ("v", v)):
        amax = float(t.abs().max()) if t.numel() else 1.0
        descale = amax / 448.0 if amax > 0 else 1.0
        out[n] = (t / descale).to(torch.float8_e4m3fn).contiguous()
        out[n + "_descale"] = descale
    return out


def decode_inputs(w: Workload, device="cpu", seed=None, B=None, Tk_max=None, seqlens=None):
    """q [B,Hq,d], k/v cache [B,Tk_max,Hkv,d] (bf16) and seqlens int32 [B]."""
    B = w.B if B is None else B
    Tk_max = w.T if Tk_max is None else Tk_max
    g = _gen(device, w.seed if seed is None else seed)
    if seqlens is None:
        hi = min(w.tk_hi, Tk_max)
        lo = min(w.tk_lo, hi)
        seqlens = torch.randint(lo, hi + 1, (B,), generator=g, device=device)
    seqlens = torch.as_tensor(seqlens, device=device).to(torch.int32)
    q = _normal_bf16((B, w.Hq, w.d), g, device)
    kc = torch.empty((B, Tk_max, w.Hkv, w.d), dtype=torch.bfloat16, device=device)
    vc = torch.empty_like(kc)
    for b in range(B):
        kc[b] = _normal_bf16((Tk_max, w.Hkv, w.d), g, device)
        vc[b] = _normal_bf16((Tk_max, w.Hkv, w.d), g, device)
    return {"q": q, "k_cache": kc, "v_cache": vc, "seqlens": seqlens}


def to_f64(t: torch.Tensor) -> np.ndarray:
    """Widen a (bf16) tensor to a float64 numpy array, exactly."""
    return t.detach().to("cpu", torch.float64).numpy()

