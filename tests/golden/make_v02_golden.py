"""Writes v02_28layer_solve.npz from the oracle alone (run from the repo root).

The 640x368 unit at full depth: 28 layers, d = 3072, 24 heads x 128, F = 12288,
920 video + 4 audio tokens, a full cache of 48 units x 1200 tokens (57,600 valid,
p0 = 57,600), and the 4-step uniform Euler solve from eps at tau = 1.  The fp64
oracle needs tens of minutes for it, so the expected values are stored here and
the GPU test compares against them.  Stored: the velocity of the first step, z
after the first step, z after the whole solve, and a fingerprint of the seeded
inputs (the test recomputes it from its own draws and refuses a mismatch).

Inputs: weights seed 1 (sfm_synth.make_weights), cache layer l drawn by
sfm_synth.make_kv_layer (seed 1000 * 2 + l), eps seed 4.
"""
import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import sfm_synth as S                      # noqa: E402
from oracle import sfm_oracle as O         # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "v02_28layer_solve.npz")


def _sum(t):
    return float(O.f64(t).sum())


def fingerprint_head(weights, eps):
    """Float64 sums over the seeded weights and noise (exact on any machine with the
    same draws)."""
    f = [_sum(eps), _sum(weights["w_in"]), _sum(weights["e_mod"]), _sum(weights["w_out"])]
    for lw in (weights["layers"][0], weights["layers"][-1]):
        f += [_sum(lw["w_qkv"][:64]), _sum(lw["w_o"][:64]), _sum(lw["w_1"][:64]),
              _sum(lw["w_2"][:64])]
    return f


def fingerprint_layer(k, v):
    """Float64 sums over a few rows of one layer's cached K and V."""
    return [_sum(k[:8]), _sum(v[-8:])]


def fingerprint(weights, k_layers, v_layers, eps):
    f = fingerprint_head(weights, eps)
    for kl, vl in zip(k_layers, v_layers):
        f += fingerprint_layer(kl, vl)
    return np.array(f)


def inputs():
    w = S.V02
    weights = S.make_weights(w)
    k_layers, v_layers = [], []
    for layer in range(w.n_layers):
        k, v = S.make_kv_layer(w, w.cache_units, layer)
        k_layers.append(k)
        v_layers.append(v)
    _, eps = S.make_latents(w)
    return w, weights, k_layers, v_layers, eps[0]


def main():
    w, weights, k_layers, v_layers, eps = inputs()
    cfg = O.Config(w.n_layers, w.d_model, w.n_heads, w.head_dim, w.d_mlp, w.c_lat, w.n_video,
                   w.n_audio, w.unit_kv_tokens, w.rope_theta, w.rms_eps)
    valid = w.cache_units * w.unit_kv_tokens
    taus = S.uniform_taus(w.n_steps)
    z = O.f64(eps)
    out = {"taus": np.array(taus), "fingerprint": fingerprint(weights, k_layers, v_layers, eps)}
    for i in range(w.n_steps):
        t0 = time.time()
        vel = O.f_theta(cfg, z, taus[i], weights, k_layers, v_layers, valid, valid)
        z = O.euler_step(z, vel, taus[i], taus[i + 1])
        print(f"step {i}: {time.time() - t0:.0f} s", flush=True)
        if i == 0:
            out["v_step0"] = vel
            out["z_step1"] = z
    out["z_solve"] = z
    np.savez(OUT, **out)
    print("wrote", OUT)


if __name__ == "__main__":
    main()
