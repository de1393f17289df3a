"""Writes oracle_tiny_regression.json from the oracle alone (run from the repo root)."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import sfm_synth as S                      # noqa: E402
from oracle import sfm_oracle as O         # noqa: E402


GUIDED_SCALE = 3.5


def tiny_case():
    w = S.TINY
    cfg = O.Config(w.n_layers, w.d_model, w.n_heads, w.head_dim, w.d_mlp, w.c_lat,
                   w.n_video, w.n_audio, w.unit_kv_tokens)
    weights = S.make_weights(w)
    k, v = S.make_kv_slices(w, w.cache_units)
    cache = O.KVCache(w.n_layers, w.cache_units, w.unit_kv_tokens, w.n_heads, w.head_dim)
    cache.append(O.f64(k), O.f64(v))
    z0, eps = S.make_latents(w)
    return w, cfg, weights, cache, eps[0]


def main():
    w, cfg, weights, cache, eps = tiny_case()
    taus = S.uniform_taus(w.n_steps)
    vel = O.f_theta(cfg, eps, 1.0, weights, cache.k, cache.v, cache.valid_tokens,
                    cache.tokens_appended)
    z = O.denoise_solve(cfg, eps, taus, weights, cache.k, cache.v, cache.valid_tokens,
                        cache.tokens_appended)
    # classifier-free guidance against an empty unconditional context
    empty = [O.f64(cache.k[0][:0])] * w.n_layers
    zg = O.denoise_solve_cfg(cfg, eps, taus, weights,
                             (cache.k, cache.v, cache.valid_tokens, cache.tokens_appended),
                             (empty, empty, 0, 0), GUIDED_SCALE)
    out = {"workload": w.name, "taus": taus,
           "guided_scale": GUIDED_SCALE, "guided_solve_rows0to3": zg[:4].tolist(),
           "velocity_tau1_rows0to3": vel[:4].tolist(),
           "solve_rows0to3": z[:4].tolist(),
           "velocity_tau1_l2": float((vel ** 2).sum() ** 0.5),
           "solve_l2": float((z ** 2).sum() ** 0.5)}
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_tiny_regression.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print("wrote", path)


if __name__ == "__main__":
    main()
