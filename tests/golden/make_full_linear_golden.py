"""Writes the expected outputs of the 313,344-token, 3072-wide bidirectional
TTT-Linear layer (seed 0, both gates at 0.1) for sampled heads and token
windows, from the fp64 oracle alone.

    python tests/golden/make_full_linear_golden.py [--out PATH]

As for the MLP layer (make_full_layer_golden.py, whose windows and input
digest this reuses): the reverse pass runs on X' = X + tanh(alpha_f) z_f and
theta mixes every channel of X', so the oracle first runs the forward pass of
all 48 heads (in groups, each projecting only its own rows of theta), forms
X' in fp64, then runs the reverse pass of the sampled heads.  A few minutes
on eight cores; the GPU test only reads the file.

Stored (npz): the sampled heads, the windows, Z_f and Z_r of the sampled
heads on those windows (fp32), both directions' final states W of the
sampled heads (fp32), and a SHA-256 of the inputs (including W_0).  Nothing
here comes from the CUDA path.
"""
from __future__ import annotations

import argparse
import hashlib
import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from oracle import ttt_oracle as O  # noqa: E402
from test_rnn_layer_b200 import synth as S  # noqa: E402

OUT = os.path.join(HERE, "full_linear_T313344_seed0.npz")
HEADS = (3, 17, 30)
WINDOW = 128
N_WINDOWS = 6
GROUP = 8


def windows(T: int) -> list[int]:
    """Starts of N_WINDOWS windows of WINDOW tokens from the first token to the last, aligned down to 64."""
    return [min(T - WINDOW, (k * (T - WINDOW) // (N_WINDOWS - 1)) // 64 * 64) for k in range(N_WINDOWS)]


def input_digest(inp: dict) -> str:
    """SHA-256 over the raw bytes of X, theta_q/k/v, W_0, alpha_f, alpha_r."""
    import torch
    h = hashlib.sha256()
    for k in ("X", "theta_q", "theta_k", "theta_v", "W_0", "alpha_f", "alpha_r"):
        t = inp[k].detach().cpu().contiguous()
        if t.dtype == torch.bfloat16:
            t = t.view(torch.int16)
        h.update(t.numpy().tobytes())
    return h.hexdigest()


def heads_direction(X, th, W0, eta, b, heads, reverse):
    """Z [T, len(heads) d] and the final states of the listed heads for one direction on X."""
    d = W0.shape[2]
    rows = np.concatenate([np.arange(h * d, (h + 1) * d) for h in heads])
    U = [O._heads_from_full(O.project_full(X, t[rows]), len(heads), d) for t in th]
    Zh, WT = O.linear_scan_heads(U[0], U[1], U[2], W0[list(heads)], eta, b, reverse)
    return O._full_from_heads(Zh), WT


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--out", default=OUT)
    args = ap.parse_args()
    w = S.FULL63S
    inp = S.make_linear_inputs(w, seed=0, device="cpu")
    digest = input_digest(inp)
    T, H, d = w.T, w.H, w.d
    X = inp["X"].float().numpy()
    th = [inp[k].float().numpy() for k in ("theta_q", "theta_k", "theta_v")]
    W0 = inp["W_0"].double().numpy()
    af = inp["alpha_f"].double().numpy()
    eta = w.eta_eff
    t0 = time.time()

    Zf = np.empty((T, H * d))
    Wf = np.empty((len(HEADS), d, d))
    for g0 in range(0, H, GROUP):
        heads = list(range(g0, min(H, g0 + GROUP)))
        Zg, Wg = heads_direction(X, th, W0, eta, w.b, heads, False)
        Zf[:, g0 * d:(g0 + len(heads)) * d] = Zg
        for i, h in enumerate(HEADS):
            if h in heads:
                Wf[i] = Wg[heads.index(h)]
        print(f"forward heads {heads[0]}-{heads[-1]} done at {time.time() - t0:.0f} s", flush=True)

    Xp = O.gate(X, Zf, af)
    Zr, Wr = heads_direction(Xp, th, W0, eta, w.b, list(HEADS), True)
    print(f"reverse heads {HEADS} done at {time.time() - t0:.0f} s", flush=True)

    starts = windows(T)
    rows = np.concatenate([np.arange(s, s + WINDOW) for s in starts])
    cols = np.concatenate([np.arange(h * d, (h + 1) * d) for h in HEADS])
    np.savez(args.out, heads=np.array(HEADS), starts=np.array(starts), window=np.array(WINDOW),
             T=np.array(T), digest=np.array(digest), eta=np.array(eta), b=np.array(w.b),
             Z_f=Zf[rows][:, cols].astype(np.float32), Z_r=Zr[rows].astype(np.float32),
             W_f=Wf.astype(np.float32), W_r=Wr.astype(np.float32))
    print("wrote", args.out, f"({time.time() - t0:.0f} s)")


if __name__ == "__main__":
    main()
