"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

This module holds no arithmetic of the method: it only draws the inputs the
performer step consumes (weights of a randomly initialised velocity network,
the thinker's K/V slices, clean latents and noise) and names the workloads.
Both the CUDA path and the oracle receive exactly the tensors made here.

Recipe (fixed seeds):
  weights      seed 1   every matrix and the modality table ~ N(0, 0.02); norm gains 1
  cache K/V    seed 2   ~ N(0, 1)
  z0           seed 3   ~ N(0, 1)
  eps          seed 4   ~ N(0, 1)
  sessions     seed 5   cache lengths ~ U[8K, 64K] tokens, rounded to whole units
Values are drawn in fp32 with torch's Philox/mt19937 generators and rounded
(round-to-nearest-even) to bf16 where the workload stores bf16.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass

import torch

SEED_WEIGHTS, SEED_CACHE, SEED_Z0, SEED_EPS, SEED_SESSIONS = 1, 2, 3, 4, 5
WEIGHT_STD = 0.02


@dataclass(frozen=True)
class Workload:
    """One configuration of the performer step."""
    name: str
    n_layers: int
    d_model: int
    n_heads: int
    head_dim: int
    d_mlp: int
    c_lat: int
    n_video: int
    n_audio: int
    unit_kv_tokens: int      # T_u: K/V tokens per cached unit
    cache_units: int         # valid cached units before the timed append
    n_steps: int             # Euler steps of the solve
    dtype: str               # "bf16" | "fp32"
    rope_theta: float = 10000.0
    rms_eps: float = 1e-6
    mlp: str = "gelu"        # "gelu" | "swiglu": W_1 [F][d] or [2F][d] (interleaved gate/up)
    rope: str = "1d"         # "1d" | "3d": positions p0 + j or (t, y, x)
    grid_w: int = 0          # 3-D RoPE: video raster width in tokens

    @property
    def n_tokens(self):
        return self.n_video + self.n_audio

    @property
    def hd(self):
        return self.n_heads * self.head_dim

    def replace(self, **kw):
        return dataclasses.replace(self, **kw)


# tiny fp32 case: 8x8 video + 4 audio tokens, 2 layers, cache of 4 units x 96 tokens
TINY = Workload("tiny-fp32", 2, 256, 4, 64, 1024, 16, 64, 4, 96, 4, 2, "fp32")
# 192x336 unit: 12x21 = 252 video + 4 audio tokens; 64 cached units x 512 tokens
V01 = Workload("v0.1-192x336", 28, 1536, 12, 128, 6144, 16, 252, 4, 512, 64, 4, "bf16")
# 640x368 unit: 40x23 = 920 video + 4 audio tokens; 48 cached units x 1200 tokens
V02 = Workload("v0.2-640x368", 28, 3072, 24, 128, 12288, 16, 920, 4, 1200, 48, 4, "bf16")

# 8 independent sessions at the 640x368 unit shape, ragged caches (see session_cache_units)
V02X8 = V02.replace(name="v0.2x8-ragged")

WORKLOADS = {w.name: w for w in (TINY, V01, V02, V02X8)}

# isolated attention sweep: cache lengths 4K/16K/64K/128K rounded up to whole 1200-token units
ATTN_SWEEP_TOKENS = [4800, 16800, 66000, 132000]


def torch_dtype(name):
    return {"bf16": torch.bfloat16, "fp32": torch.float32}[name]


def _normal(gen, shape, std, dtype, device):
    t = torch.randn(*shape, generator=gen, dtype=torch.float32, device=device)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def _gen(seed, device):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def make_weights(w: Workload, device="cpu", seed=SEED_WEIGHTS):
    """Random-init weights of the velocity network, matrices stored [out][in]."""
    dt = torch_dtype(w.dtype)
    g = _gen(seed, device)
    ones = lambda n: torch.ones(n, dtype=dt, device=device)
    out = {
        "w_in": _normal(g, (w.d_model, w.c_lat), WEIGHT_STD, dt, device),
        "e_mod": _normal(g, (2, w.d_model), WEIGHT_STD, dt, device),
        "g_final": ones(w.d_model),
        "w_out": _normal(g, (w.c_lat, w.d_model), WEIGHT_STD, dt, device),
        "layers": [],
    }
    for _ in range(w.n_layers):
        out["layers"].append({
            "g_attn": ones(w.d_model),
            "w_qkv": _normal(g, (3 * w.hd, w.d_model), WEIGHT_STD, dt, device),
            "w_o": _normal(g, (w.d_model, w.hd), WEIGHT_STD, dt, device),
            "g_mlp": ones(w.d_model),
            "w_1": _normal(g, ((2 if w.mlp == "swiglu" else 1) * w.d_mlp, w.d_model), WEIGHT_STD,
                           dt, device),
            "w_2": _normal(g, (w.d_model, w.d_mlp), WEIGHT_STD, dt, device),
        })
    return out


def make_kv_slices(w: Workload, n_units, device="cpu", seed=SEED_CACHE):
    """The thinker's K/V slices for n_units units: K, V each [L][n_units*T_u][H][D]."""
    dt = torch_dtype(w.dtype)
    g = _gen(seed, device)
    shape = (w.n_layers, n_units * w.unit_kv_tokens, w.n_heads, w.head_dim)
    return _normal(g, shape, 1.0, dt, device), _normal(g, shape, 1.0, dt, device)


def make_kv_layer(w: Workload, n_units, layer, device="cpu", seed=SEED_CACHE):
    """One layer of the thinker's K/V slices, drawn from its own generator (seed
    1000 * seed + layer), so a 28-layer cache can be built one layer at a time
    without holding every layer's fp32 draw: K, V each [n_units*T_u][H][D]."""
    dt = torch_dtype(w.dtype)
    g = _gen(1000 * seed + layer, device)
    shape = (n_units * w.unit_kv_tokens, w.n_heads, w.head_dim)
    return _normal(g, shape, 1.0, dt, device), _normal(g, shape, 1.0, dt, device)


def make_latents(w: Workload, device="cpu", n_sessions=1):
    """Clean latents z0 (seed 3) and noise eps (seed 4), fp32 [S][N][C]."""
    shape = (n_sessions, w.n_tokens, w.c_lat)
    z0 = _normal(_gen(SEED_Z0, device), shape, 1.0, torch.float32, device)
    eps = _normal(_gen(SEED_EPS, device), shape, 1.0, torch.float32, device)
    return z0, eps


def make_qkv(n_q, n_kv, n_heads, head_dim, dtype="bf16", device="cpu", seed=SEED_CACHE):
    """Isolated attention inputs: Q [n_q][H][D], K, V [n_kv][H][D] ~ N(0, 1)."""
    dt = torch_dtype(dtype)
    g = _gen(seed, device)
    q = _normal(g, (n_q, n_heads, head_dim), 1.0, dt, device)
    k = _normal(g, (n_kv, n_heads, head_dim), 1.0, dt, device)
    v = _normal(g, (n_kv, n_heads, head_dim), 1.0, dt, device)
    return q, k, v


def session_cache_units(n_sessions=8, lo_tokens=8192, hi_tokens=65536, unit_tokens=1200,
                        seed=SEED_SESSIONS):
    """Ragged per-session cache lengths ~ U[lo, hi] tokens, rounded up to whole units."""
    g = _gen(seed, "cpu")
    u = torch.rand(n_sessions, generator=g, dtype=torch.float64)
    toks = lo_tokens + u * (hi_tokens - lo_tokens)
    return [int(-(-int(t) // unit_tokens)) for t in toks]


def uniform_taus(n_steps):
    """The uniform schedule 1 -> 0 as a list of floats (input, not arithmetic of f_theta)."""
    return [1.0 - i / n_steps for i in range(n_steps + 1)]
