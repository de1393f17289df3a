"""fp64 CPU oracle for the performer's next-unit flow-matching denoising step.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import or run
this module.  The product path (``streaming_flow_matching_b200``) never calls
it, and this module imports nothing from the product: the two share no code.

Plain, slow, obviously correct: numpy float64 throughout, one function per step
of the method, written in the order the pages give it.  A library matmul is the
only primitive used; there is no blocking, fusion or reordering.  bf16 inputs are
upcast exactly to float64; no intermediate bf16 rounding is emulated.

Sources (the pages are web write-ups of Wan-Streamer; none prints code):
  [v0.1]  "Wan-Streamer" blog (gongshangzheng.github.io): §3.1 streaming
          formulation, §3.3 block-causal Transformer, §3.4 conditional flow
          matching, Fig. 2 thinker/performer timeline.
  [dig]   "Wan-Streamer v0.2: Higher Resolution, Same Latency" digest
          (nanless.github.io): "method overview and architecture" (performer
          path, pre-sharded K/V cache, audio unsharded), "details" (step count,
          noise schedule undisclosed).
  [blog]  "Wan-Streamer v0.2" blog (zhao9797.github.io): "Infra" section.
  [abs]   "Wan-Streamer v0.2" abstract (chatpaper.ai).

Readings taken where the pages are silent:
  * rectified-flow path z_tau = (1 - tau) z0 + tau eps, velocity eps - z0
    (the path formula of [v0.1] §3.4 was lost in extraction; the symbol glosses
    survive); Euler solve from tau = 1 to tau = 0, z <- z + (tau_next - tau) v.
  * uniform step schedule (the count is undisclosed, [dig] "details").
  * tau enters f_theta through a parameter-free sinusoidal embedding added to
    every token at the input.
  * pre-norm blocks: RMSNorm -> QKV -> 1-D rotate-half RoPE -> softmax
    attention -> O-proj + residual; RMSNorm -> W1 -> tanh-GELU -> W2 + residual;
    final RMSNorm -> velocity head.  No biases.
  * cached K is stored post-RoPE (the thinker builds it), so it is never rotated
    here; current-unit tokens sit at absolute positions P0 + j, P0 = tokens ever
    appended to the session.
  * token order inside the current unit: video raster first, then audio.
  * ring cache: unit u lands in slot u mod n_slots.

Parity status: every step is pinned by tests in ``tests/test_oracle_pins.py``
(closed forms, invariants, brute force at tiny sizes, library routines).  The
composed velocity network f_theta has no published values to pin against; it is
pinned by a scalar-loop brute-force re-derivation at tiny size, by the
block-causal consistency check (performer form == masked full-sequence form),
and by invariants.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

VIDEO, AUDIO = 0, 1


def f64(a):
    """Upcast an array-like (numpy, or a CPU torch tensor of any dtype) to float64."""
    if hasattr(a, "detach"):
        return a.detach().to("cpu").double().numpy()
    return np.asarray(a, dtype=np.float64)


@dataclass
class Config:
    """Shapes of f_theta and of one streaming unit."""
    n_layers: int
    d_model: int
    n_heads: int
    head_dim: int
    d_mlp: int
    c_lat: int
    n_video: int
    n_audio: int
    unit_kv_tokens: int
    rope_theta: float = 10000.0
    rms_eps: float = 1e-6
    mlp: str = "gelu"          # "gelu" | "swiglu" (open reading, see swiglu_mlp)
    rope_mode: str = "1d"      # "1d" | "3d" (open reading, see rope_3d)
    grid_w: int = 0            # 3-D RoPE: video raster width in tokens

    @property
    def n_tokens(self) -> int:
        return self.n_video + self.n_audio

    @property
    def hd(self) -> int:
        return self.n_heads * self.head_dim


# ---------------------------------------------------------------------------
# elementwise pieces
# ---------------------------------------------------------------------------

def rmsnorm(x, g, eps):
    """RMSNorm over the last axis: x / sqrt(mean(x^2) + eps) * g (pre-norm block)."""
    x = f64(x)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * f64(g)


def gelu_tanh(x):
    """tanh approximation of GELU: 0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3)))."""
    x = f64(x)
    return 0.5 * x * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (x + 0.044715 * x ** 3)))


def rope_freqs(head_dim, theta):
    """omega_i = theta^(-2 i / head_dim) for i < head_dim / 2."""
    i = np.arange(head_dim // 2, dtype=np.float64)
    return theta ** (-2.0 * i / head_dim)


def rope(x, pos, theta):
    """1-D rotary embedding, rotate-half pairing (i, i + D/2).

    x: [N][H][D]; pos: [N] absolute positions.  Pair (a, b) = (x_i, x_{i+D/2})
    rotated by angle pos * omega_i:  a' = a cos - b sin,  b' = b cos + a sin.
    """
    x = f64(x)
    d = x.shape[-1]
    half = d // 2
    ang = np.asarray(pos, dtype=np.float64)[:, None] * rope_freqs(d, theta)[None, :]
    c = np.cos(ang)[:, None, :]
    s = np.sin(ang)[:, None, :]
    a = x[..., :half]
    b = x[..., half:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=-1)


def rope_3d_bands(head_dim):
    """Pair bands of the 3-D rotary embedding: (pairs of t, pairs of y, pairs of x).

    Each spatial axis takes head_dim // 6 of the head_dim / 2 rotate-half pairs and time
    takes the rest (128 dims: 22 + 21 + 21 pairs), the split of the Wan video models."""
    half = head_dim // 2
    ns = head_dim // 6
    return half - 2 * ns, ns, ns


def rope_3d(x, pos3, theta):
    """3-D rotary embedding over (t, y, x), rotate-half pairing (i, i + D/2).

    x: [N][H][D]; pos3: [N][3] integer positions (t, y, x).  Pair i of band b (time,
    rows, columns) with n_b pairs, k = i - start_b, rotates by pos3[:, b] * theta^(-k / n_b):
    the 1-D frequency ladder restarted per axis over the band's own width.
    """
    x = f64(x)
    d = x.shape[-1]
    half = d // 2
    nt, ny, nx = rope_3d_bands(d)
    pos3 = np.asarray(pos3, dtype=np.float64)
    axis = np.concatenate([np.zeros(nt, int), np.ones(ny, int), np.full(nx, 2)])
    k = np.concatenate([np.arange(nt), np.arange(ny), np.arange(nx)]).astype(np.float64)
    nb = np.concatenate([np.full(nt, nt), np.full(ny, ny), np.full(nx, nx)]).astype(np.float64)
    w = theta ** (-k / nb)
    ang = pos3[:, axis] * w[None, :]                  # [N][half]
    c = np.cos(ang)[:, None, :]
    sn = np.sin(ang)[:, None, :]
    a = x[..., :half]
    b = x[..., half:]
    return np.concatenate([a * c - b * sn, b * c + a * sn], axis=-1)


def token_positions(cfg, p0, n_units=1):
    """Positions of n_units consecutive units starting at token position p0 (1-D: p0 + i)
    or, for 3-D RoPE, (t, y, x) per token: t = the unit's index on the timeline
    (p0 // unit_kv_tokens + u), (y, x) the video token's raster cell, (0, 0) for audio."""
    n = cfg.n_tokens
    if cfg.rope_mode == "1d":
        return p0 + np.arange(n_units * n)
    j = np.arange(n)
    y = np.where(j < cfg.n_video, j // max(cfg.grid_w, 1), 0)
    x = np.where(j < cfg.n_video, j % max(cfg.grid_w, 1), 0)
    t0 = p0 // cfg.unit_kv_tokens
    return np.concatenate([np.stack([np.full(n, t0 + u), y, x], axis=1) for u in range(n_units)])


def apply_rope(cfg, x, pos):
    """The rotary embedding of the configuration: 1-D over positions, or 3-D over (t, y, x)."""
    if cfg.rope_mode == "3d":
        return rope_3d(x, pos, cfg.rope_theta)
    return rope(x, pos, cfg.rope_theta)


def silu(x):
    """SiLU: x * sigmoid(x) = x / (1 + exp(-x))."""
    x = f64(x)
    return x / (1.0 + np.exp(-x))


def swiglu_gate_up(cfg, w1):
    """Gate and up matrices [F][d] of a SwiGLU W_1 stored [2F][d] in interleaved blocks of
    64 rows: rows 128 b + [0, 64) are gate rows 64 b + [0, 64), rows 128 b + [64, 128) the
    matching up rows (the layout the library reads)."""
    w1 = f64(w1)
    blocks = w1.reshape(-1, 2, 64, w1.shape[-1])
    return blocks[:, 0].reshape(-1, w1.shape[-1]), blocks[:, 1].reshape(-1, w1.shape[-1])


def mlp_forward(cfg, h, lw):
    """The block's MLP on normalised rows h: tanh-GELU (W_1 [F][d]) or SwiGLU
    (silu(h W_g^T) * (h W_u^T), W_1 [2F][d] as in swiglu_gate_up), then W_2."""
    if cfg.mlp == "swiglu":
        wg, wu = swiglu_gate_up(cfg, lw["w_1"])
        return linear(silu(linear(h, wg)) * linear(h, wu), lw["w_2"])
    return linear(gelu_tanh(linear(h, lw["w_1"])), lw["w_2"])


def tau_embedding(tau, d):
    """Parameter-free sinusoidal embedding of the flow time tau.

    e_i = sin(1000 tau w_i) for i < d/2 and e_i = cos(1000 tau w_{i-d/2}) for
    i >= d/2, with w_i = 10000^(-2 i / d).
    """
    half = d // 2
    w = 10000.0 ** (-2.0 * np.arange(half, dtype=np.float64) / d)
    ang = 1000.0 * float(tau) * w
    return np.concatenate([np.sin(ang), np.cos(ang)])


def modality_of_tokens(cfg: Config):
    """Modality id per current-unit token: video raster tokens, then audio tokens."""
    m = np.full(cfg.n_tokens, VIDEO, dtype=np.int64)
    m[cfg.n_video:] = AUDIO
    return m


def linear(x, w):
    """y = x W^T with W stored [out][in] (no bias)."""
    return f64(x) @ f64(w).T


# ---------------------------------------------------------------------------
# attention
# ---------------------------------------------------------------------------

def attention(q, k, v, visible=None):
    """Softmax attention per head, fp64, with max subtraction.

    q: [N][H][D], k, v: [S][H][D]; visible: optional bool [N][S] (True = may
    attend).  Scale 1/sqrt(D).  Returns [N][H][D].
    """
    q, k, v = f64(q), f64(k), f64(v)
    n, h, d = q.shape
    out = np.empty((n, h, d))
    for hh in range(h):
        logits = (q[:, hh, :] @ k[:, hh, :].T) / math.sqrt(d)
        if visible is not None:
            logits = np.where(visible, logits, -np.inf)
        logits = logits - logits.max(axis=1, keepdims=True)
        p = np.exp(logits)
        p = p / p.sum(axis=1, keepdims=True)
        out[:, hh, :] = p @ v[:, hh, :]
    return out


def block_causal_visible(q_units, k_units):
    """Block-causal mask: a query in unit j sees every key whose unit is <= j
    (bidirectional inside a unit) -- [v0.1] §3.3, [dig] "method overview"."""
    return np.asarray(k_units)[None, :] <= np.asarray(q_units)[:, None]


# ---------------------------------------------------------------------------
# K/V cache (pre-allocated, ring of unit slots)
# ---------------------------------------------------------------------------

class KVCache:
    """Pre-allocated per-layer K/V cache of n_slots unit slots of T_u tokens.

    The thinker's K/V slice for unit u is written verbatim into slot
    u mod n_slots ([dig] "performer path": each rank writes the broadcast slice
    into its pre-allocated local cache).  Valid rows are the first
    min(units, n_slots) * T_u rows.  With ring=False a full cache refuses the
    append and stays unchanged.
    """

    def __init__(self, n_layers, n_slots, unit_tokens, n_heads, head_dim, ring=True, dtype=np.float64):
        self.n_slots = n_slots
        self.unit_tokens = unit_tokens
        self.ring = ring
        shape = (n_layers, n_slots * unit_tokens, n_heads, head_dim)
        self.k = np.zeros(shape, dtype=dtype)
        self.v = np.zeros(shape, dtype=dtype)
        self.units = 0          # units ever appended (evicted ones included)

    @property
    def tokens_appended(self):
        return self.units * self.unit_tokens

    @property
    def valid_tokens(self):
        return min(self.units, self.n_slots) * self.unit_tokens

    def append(self, k_slice, v_slice):
        """k_slice, v_slice: [L][n_units * T_u][H][D].  Returns False (and changes
        nothing) when the cache is full and ring is off."""
        t = self.unit_tokens
        n_tok = k_slice.shape[1]
        if n_tok % t != 0:
            raise ValueError("slice length must be a whole number of units")
        n_units = n_tok // t
        if not self.ring and self.units + n_units > self.n_slots:
            return False
        for i in range(n_units):
            slot = (self.units + i) % self.n_slots
            self.k[:, slot * t:(slot + 1) * t] = k_slice[:, i * t:(i + 1) * t]
            self.v[:, slot * t:(slot + 1) * t] = v_slice[:, i * t:(i + 1) * t]
        self.units += n_units
        return True


# ---------------------------------------------------------------------------
# the velocity network f_theta (performer form)
# ---------------------------------------------------------------------------

def embed(cfg: Config, z, tau, w, modality=None):
    """x_j = W_in z_j + e_mod[m(j)] + temb(tau).  Audio and video noisy latents
    enter together ([v0.1] §3.4 cross-modal conditioning)."""
    if modality is None:
        modality = modality_of_tokens(cfg)
    x = linear(z, w["w_in"])
    x = x + f64(w["e_mod"])[modality]
    x = x + tau_embedding(tau, cfg.d_model)[None, :]
    return x


def layer_forward(cfg: Config, x, lw, k_ctx, v_ctx, pos, visible=None, return_kv=False):
    """One pre-norm block.  k_ctx/v_ctx: clean context keys/values [S][H][D]
    (already rotated); the current tokens' own k, v are appended after them."""
    n = x.shape[0]
    h = rmsnorm(x, lw["g_attn"], cfg.rms_eps)
    qkv = linear(h, lw["w_qkv"])
    hd = cfg.hd
    q = qkv[:, :hd].reshape(n, cfg.n_heads, cfg.head_dim)
    k = qkv[:, hd:2 * hd].reshape(n, cfg.n_heads, cfg.head_dim)
    v = qkv[:, 2 * hd:].reshape(n, cfg.n_heads, cfg.head_dim)
    q = apply_rope(cfg, q, pos)
    k = apply_rope(cfg, k, pos)
    K = np.concatenate([f64(k_ctx), k], axis=0)
    V = np.concatenate([f64(v_ctx), v], axis=0)
    a = attention(q, K, V, visible)
    x = x + linear(a.reshape(n, hd), lw["w_o"])
    h2 = rmsnorm(x, lw["g_mlp"], cfg.rms_eps)
    x = x + mlp_forward(cfg, h2, lw)
    if return_kv:
        return x, k, v
    return x


def head(cfg: Config, x, w):
    """Velocity head: v = RMSNorm(x; g_f) W_out^T, one C-vector per token."""
    return linear(rmsnorm(x, w["g_final"], cfg.rms_eps), w["w_out"])


def f_theta(cfg: Config, z, tau, w, cache_k, cache_v, valid_tokens, p0, pos=None, modality=None):
    """Velocity of the current unit's noisy latents z [N][C] at flow time tau.

    Performer form: every current-unit query sees every valid cached token
    (all cached units precede the current one) and every current-unit token
    (bidirectional inside the unit) -- [v0.1] §3.3 block-causal attention,
    clean context c_k of §3.4.  cache_k/cache_v: per-layer [rows][H][D]; only
    the first valid_tokens rows are context.  pos/modality override the
    default token positions (p0 + j) and modality ids (video, then audio).
    """
    x = embed(cfg, z, tau, w, modality)
    if pos is None:
        pos = token_positions(cfg, p0)
    for li, lw in enumerate(w["layers"]):
        kc = f64(cache_k[li][:valid_tokens])
        vc = f64(cache_v[li][:valid_tokens])
        x = layer_forward(cfg, x, lw, kc, vc, pos)
    return head(cfg, x, w)


def euler_step(z, v, tau_from, tau_to):
    """One Euler step along the flow: z <- z + (tau_to - tau_from) v."""
    return f64(z) + (float(tau_to) - float(tau_from)) * f64(v)


def fm_solve(z, taus, velocity):
    """Integrate dz/dtau = velocity(z, tau) from taus[0] (= 1, pure noise) to
    taus[-1] (= 0, clean latent) with explicit Euler steps ([v0.1] §3.4: the
    linear path has a constant velocity field, so few steps suffice)."""
    z = f64(z)
    for i in range(len(taus) - 1):
        z = euler_step(z, velocity(z, taus[i]), taus[i], taus[i + 1])
    return z


def uniform_taus(n_steps):
    """Uniform schedule 1 -> 0 in n_steps steps."""
    return [1.0 - i / n_steps for i in range(n_steps + 1)]


def rf_path(z0, eps, tau):
    """Rectified-flow linear path z_tau = (1 - tau) z0 + tau eps."""
    return (1.0 - tau) * f64(z0) + tau * f64(eps)


def rf_velocity(z0, eps):
    """Constant velocity of the linear path: d z_tau / d tau = eps - z0."""
    return f64(eps) - f64(z0)


def denoise_solve(cfg: Config, eps, taus, w, cache_k, cache_v, valid_tokens, p0):
    """The performer's solve for one unit: Euler over f_theta from eps at tau=1."""
    return fm_solve(eps, taus,
                    lambda z, t: f_theta(cfg, z, t, w, cache_k, cache_v, valid_tokens, p0))


# ---------------------------------------------------------------------------
# classifier-free guidance (the distillation teacher's sampler)
# ---------------------------------------------------------------------------

def guided_velocity(v_cond, v_uncond, scale):
    """Classifier-free guidance: start from the unconditional velocity and move
    `scale` times the conditional-minus-unconditional difference.

    [v0.1] training, Stage 3 (low-latency distillation): the teacher samples with
    classifier-free guidance and more solver steps; the pages give no formula.
    Reading: the usual form of Ho & Salimans (2022), v_u + s (v_c - v_u), so
    s = 1 is the conditional model and s = 0 the unconditional one.
    """
    v_u = f64(v_uncond)
    return v_u + float(scale) * (f64(v_cond) - v_u)


def denoise_solve_cfg(cfg: Config, eps, taus, w, cond, uncond, scale):
    """Guided solve of one unit: at every Euler step f_theta is evaluated twice at
    the same z and tau, once on the conditional context and once on the
    unconditional one, and the step follows their guided velocity.

    cond / uncond: (cache_k, cache_v, valid_tokens, p0) of the two contexts.  The
    performer's only condition is the thinker's K/V in its cache ([abs]: the
    thinker reaches the performer only as K/V conditioning), so the
    unconditional context is a cache holding a null condition; an empty cache
    (valid_tokens = 0: the unit attends to itself alone) is the plainest one.
    """
    def velocity(z, t):
        v_c = f_theta(cfg, z, t, w, *cond)
        v_u = f_theta(cfg, z, t, w, *uncond)
        return guided_velocity(v_c, v_u, scale)
    return fm_solve(eps, taus, velocity)


# ---------------------------------------------------------------------------
# block-causal full-sequence form (prefill / invariant checks)
# ---------------------------------------------------------------------------

def f_theta_sequence(cfg: Config, zs, taus, w, return_kv=False):
    """Masked block-causal forward over several units at once.

    zs: list of per-unit latents [N][C]; taus: per-unit flow times.  Token j of
    unit u is at absolute position u * N + j and sees every token of units <= u.
    Returns the per-unit velocities, and optionally every layer's rotated K/V
    per unit (what a cache built from these units would hold).
    """
    n = cfg.n_tokens
    n_units = len(zs)
    x = np.concatenate([embed(cfg, zs[u], taus[u], w) for u in range(n_units)], axis=0)
    units = np.repeat(np.arange(n_units), n)
    pos = token_positions(cfg, 0, n_units)
    visible = block_causal_visible(units, units)
    kv = []
    empty = np.zeros((0, cfg.n_heads, cfg.head_dim))
    for lw in w["layers"]:
        x, k, v = layer_forward(cfg, x, lw, empty, empty, pos, visible, return_kv=True)
        kv.append((k, v))
    vel = head(cfg, x, w)
    out = [vel[u * n:(u + 1) * n] for u in range(n_units)]
    if return_kv:
        return out, kv
    return out


def f_theta_units(cfg: Config, zs, taus, w, cache_k, cache_v, valid_tokens, p0, return_kv=False):
    """Several consecutive units after a clean cached prefix, in one masked pass.

    [v0.1] §3.3: a unit sees itself bidirectionally and every earlier unit, never a
    later one; the cached prefix (the clean context of §3.4) counts as earlier than
    every unit of the pass.  Unit u's tokens sit at positions p0 + u * N + j (the
    units follow the cache on the timeline).  zs, taus: per-unit latents [N][C] and
    flow times.  cache_k / cache_v: per-layer [rows][H][D], first valid_tokens rows
    valid (already rotated).  Returns the per-unit velocities and, optionally,
    every layer's rotated K/V of the pass's own tokens.  One unit is f_theta; an
    empty prefix with p0 = 0 is f_theta_sequence.
    """
    n = cfg.n_tokens
    n_units = len(zs)
    x = np.concatenate([embed(cfg, zs[u], taus[u], w) for u in range(n_units)], axis=0)
    units = np.repeat(np.arange(n_units), n)
    pos = token_positions(cfg, p0, n_units)
    key_units = np.concatenate([np.full(valid_tokens, -1), units])   # prefix = unit -1
    visible = block_causal_visible(units, key_units)
    kv = []
    for li, lw in enumerate(w["layers"]):
        kc = f64(cache_k[li][:valid_tokens])
        vc = f64(cache_v[li][:valid_tokens])
        x, k, v = layer_forward(cfg, x, lw, kc, vc, pos, visible, return_kv=True)
        kv.append((k, v))
    vel = head(cfg, x, w)
    out = [vel[u * n:(u + 1) * n] for u in range(n_units)]
    if return_kv:
        return out, kv
    return out


# ---------------------------------------------------------------------------
# work counts (for the timed CPU baseline)
# ---------------------------------------------------------------------------

def step_flops(cfg: Config, valid_tokens):
    """Dense FLOPs of one f_theta evaluation: 2MKN per matmul, 4 N S H D for attention."""
    n, d, hd, f = cfg.n_tokens, cfg.d_model, cfg.hd, cfg.d_mlp
    gemm = 2 * n * d * (3 * hd) + 2 * n * hd * d + 2 * n * d * f + 2 * n * f * d
    attn = 4 * n * (valid_tokens + n) * hd
    return cfg.n_layers * (gemm + attn) + 2 * n * cfg.c_lat * d * 2
