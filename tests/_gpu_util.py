"""Shared helpers of the GPU parity tests: workloads, oracle calls, error norms."""
import numpy as np
import torch

import sfm_synth as S
from oracle import sfm_oracle as O

BF16_TOL = 2e-2     # relative L2 on bf16 velocities and latents (stated tolerance)
FP32_TOL = 1e-5     # relative L2 in the fp32 mode

# small bf16 case the oracle finishes in well under a second: several query
# tiles with a ragged tail (204 = 3 x 64 + 12), ragged key tiles (500 + 204 keys)
SMALL_BF16 = S.Workload("small-bf16", 2, 512, 4, 128, 2048, 16, 200, 4, 100, 5, 4, "bf16")
# d_model above 4096 (RMSNorm rows of 528 threads, 33 head-kernel column groups per thread)
WIDE_BF16 = S.Workload("wide-bf16", 1, 4224, 2, 128, 256, 16, 24, 4, 32, 3, 2, "bf16")


def ocfg(w):
    return O.Config(w.n_layers, w.d_model, w.n_heads, w.head_dim, w.d_mlp, w.c_lat, w.n_video,
                    w.n_audio, w.unit_kv_tokens, w.rope_theta, w.rms_eps, mlp=w.mlp,
                    rope_mode=w.rope, grid_w=w.grid_w)


def rel_l2(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))


def to_cuda(weights):
    return {k: ([{n: t.cuda() for n, t in lw.items()} for lw in v] if k == "layers" else v.cuda())
            for k, v in weights.items()}


def oracle_cache_layers(k_slice, v_slice, n_units, unit_tokens, cache_units):
    """Per-layer cache contents the oracle sees after n_units appends (ring order)."""
    if n_units <= cache_units:
        return ([k_slice[l] for l in range(k_slice.shape[0])],
                [v_slice[l] for l in range(v_slice.shape[0])])
    c = O.KVCache(k_slice.shape[0], cache_units, unit_tokens, k_slice.shape[2], k_slice.shape[3])
    c.append(O.f64(k_slice), O.f64(v_slice))
    return list(c.k), list(c.v)


def tol(w):
    return FP32_TOL if w.dtype == "fp32" else BF16_TOL
