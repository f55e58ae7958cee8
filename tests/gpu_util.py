"""Helpers shared by the GPU parity tests (no decoder arithmetic here)."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from synth import qwen3 as sq

LOGITS_TOL = 2e-2   # rel-L2 per (request, step) under teacher forcing
HIDDEN_TOL = 1e-2   # rel-L2 per layer of the residual stream


def rel_l2(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def to_cuda(weights):
    return {k: v.cuda() for k, v in weights.items()}


def _steps(step0, R):
    """step0 as one position for every request or one per request."""
    a = np.asarray(step0, dtype=np.int32)
    return np.full(R, int(a), np.int32) if a.ndim == 0 else a.astype(np.int32).copy()


def gpu_teacher_forced(dec, tokens_cpu: torch.Tensor, iters, step0=0):
    """Run one persistent launch per iteration with capture on; returns the
    per-iteration (logits [R,V], hidden [L+1,R,H]) as float64 numpy arrays.
    step0: the first position, shared or per request."""
    s = dec.shape
    R = tokens_cpu.shape[0]
    tok = tokens_cpu.cuda()
    step = torch.from_numpy(_steps(step0, R)).cuda()
    out = []
    for it in range(iters):
        lg = torch.full((R, s.vocab), float("nan"), device="cuda")
        hd = torch.full((s.layers + 1, R, s.hidden), float("nan"), device="cuda")
        dec.kernel.set_capture(0, lg, hd)
        end = (step + 1).to(torch.int32)
        dec.run(step, tok, end)
        torch.cuda.synchronize()
        dec.kernel.check_status()
        out.append((lg.double().cpu().numpy(), hd.double().cpu().numpy()))
    dec.kernel.set_capture(-1, None, None)
    return out, tok.cpu(), step.cpu()


def oracle_teacher_forced(shape, w_cpu, tokens_cpu: torch.Tensor, iters, kc=None, vc=None, step0=0,
                          round_mode=oracle.ROUND_NONE):
    ref = oracle.Decoder(shape, w_cpu)
    toks = tokens_cpu.numpy().copy()
    R, S = toks.shape
    if kc is None:
        kc, vc = ref.new_cache(R, S)
    step = _steps(step0, R)
    out = []
    for _ in range(iters):
        lg = np.full((R, shape.vocab), np.nan)
        hd = np.full((shape.layers + 1, R, shape.hidden), np.nan)
        ref.iteration(kc, vc, step, toks, None, round_mode, lg, hd)
        out.append((lg, hd))
    return out, toks, kc, vc


def compare_captures(gpu, ref, logits_tol=LOGITS_TOL, hidden_tol=HIDDEN_TOL):
    worst_l, worst_h = 0.0, 0.0
    for it, ((gl, gh), (rl, rh)) in enumerate(zip(gpu, ref)):
        for r in range(gl.shape[0]):
            e = rel_l2(gl[r], rl[r])
            worst_l = max(worst_l, e)
            assert e <= logits_tol, f"iteration {it} request {r}: logits rel-L2 {e:.3e}"
            for l in range(gh.shape[0]):
                e = rel_l2(gh[l, r], rh[l, r])
                worst_h = max(worst_h, e)
                assert e <= hidden_tol, f"iteration {it} request {r} layer slot {l}: hidden rel-L2 {e:.3e}"
    return worst_l, worst_h


def bf16_u16(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def u16_to_f64(a: np.ndarray) -> np.ndarray:
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
