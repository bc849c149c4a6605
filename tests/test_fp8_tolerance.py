"""The E4M3 forward's per-element bound (``fp8_o_tolerance``) checked on the
CPU against a model of the kernel's one coarse rounding: exact attention with
P = e^(S - m') rounded to E4M3 before P V (torch's round-to-nearest
float8_e4m3fn conversion), for reference offsets m - m' of 0, 3.3 and 7.9 in
log2 units (the kernel moves its reference lazily, by at most 8), and O rounded
to bf16.  The modelled kernel must stay inside the bound and inside the mean
bound; a modelled kernel that drops one 128-key tile must not."""

import math

import numpy as np
import pytest
import torch

import oracle
from workloads import WORKLOADS, prefill_inputs_e4m3
from _parity import FP8_O_MEAN_ABS, fp8_o_tolerance


def _model(q, k, v, scale, causal, shift_log2, drop_tile=False):
    Tq, Tk = q.shape[0], k.shape[0]
    S = scale * (q @ k.T)
    if causal:
        S = np.where(np.arange(Tk)[None, :] <= np.arange(Tq)[:, None] + (Tk - Tq), S, -np.inf)
    m = np.max(S, axis=1, keepdims=True)
    m = np.where(np.isfinite(m), m, 0.0) - shift_log2 * math.log(2.0)
    x = np.exp(S - m)
    l = x.sum(axis=1, keepdims=True)
    xq = torch.from_numpy(x).to(torch.float8_e4m3fn).double().numpy()
    if drop_tile:
        xq[:, 128:256] = 0.0
    O = xq @ v / np.where(l > 0, l, 1.0)
    return torch.from_numpy(O).to(torch.bfloat16).double().numpy(), S


@pytest.mark.parametrize("Tq,Tk,causal", [(300, 300, True), (450, 200, True), (512, 512, False)])
def test_bound_holds_for_modelled_kernel_and_catches_a_dropped_tile(Tq, Tk, causal):
    w = WORKLOADS[3].with_(B=1, Hq=2, Hkv=2, causal=causal)
    inp = prefill_inputs_e4m3(w, seed=17 + Tq + 5 * Tk + 2, Tq=Tq, Tk=Tk)
    for h in range(2):
        dec = {n: oracle.e4m3_decode(inp[n][0, :, h].view(torch.uint8).numpy()) * inp[n + "_descale"]
               for n in ("q", "k", "v")}
        O, _ = oracle.head_forward(dec["q"], dec["k"], dec["v"], w.scale, causal)
        for shift in (0.0, 3.3, 7.9):
            Om, S = _model(dec["q"], dec["k"], dec["v"], w.scale, causal, shift)
            tol = fp8_o_tolerance(S, dec["v"], O)
            assert (np.abs(Om - O) <= tol).all()
            assert np.abs(Om - O).mean() <= FP8_O_MEAN_ABS
        if Tk > 256:
            Ob, S = _model(dec["q"], dec["k"], dec["v"], w.scale, causal, 0.0, drop_tile=True)
            tol = fp8_o_tolerance(S, dec["v"], O)
            assert (np.abs(Ob - O) > tol).any()
            assert np.abs(Ob - O).mean() > FP8_O_MEAN_ABS
