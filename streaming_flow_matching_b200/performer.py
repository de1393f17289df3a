"""Thin Python binding over libsfm for torch tensors: argument marshalling only.

Every computation runs in libsfm's CUDA kernels; this module only turns
torch tensors into device pointers, passes the current CUDA stream, and turns
status codes into exceptions.
"""
from __future__ import annotations

import ctypes as C

import torch

from . import _lib as L

_DT = {torch.bfloat16: L.SFM_DTYPE_BF16, torch.float32: L.SFM_DTYPE_FP32}


def _stream():
    return C.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t):
    return C.c_void_p(t.data_ptr()) if t is not None else C.c_void_p(0)


def _need(t, dtype, name, shape=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


class Performer:
    """One libsfm handle: the weights of f_theta, the K/V pool and its sessions."""

    def __init__(self, *, n_layers, d_model, n_heads, head_dim, d_mlp, c_lat, n_video, n_audio,
                 unit_kv_tokens, pool_tokens, max_sessions=1, dtype=torch.bfloat16, ring=True,
                 rope_theta=10000.0, rms_eps=1e-6, weights=None, mlp="gelu", rope="1d", grid_w=0):
        self.dtype = dtype
        self.cfg = L.sfm_config(n_layers, d_model, n_heads, head_dim, d_mlp, c_lat, n_video,
                                n_audio, unit_kv_tokens, max_sessions, pool_tokens, _DT[dtype],
                                int(ring), rope_theta, rms_eps,
                                {"gelu": L.SFM_MLP_GELU, "swiglu": L.SFM_MLP_SWIGLU}[mlp],
                                {"1d": L.SFM_ROPE_1D, "3d": L.SFM_ROPE_3D}[rope], grid_w)
        self.n_tok = n_video + n_audio
        self.shape = dict(n_layers=n_layers, n_heads=n_heads, head_dim=head_dim, c_lat=c_lat)
        self._weights = weights           # keeps the borrowed device memory alive
        self._h = C.c_void_p()
        wp = None
        if weights is not None:
            wp = self._weights_struct(weights)
        L.check(L.lib.sfm_create(C.byref(self.cfg), C.byref(wp) if wp is not None else None,
                                 C.byref(self._h)), "sfm_create")

    @classmethod
    def from_workload(cls, w, weights, pool_tokens=None, max_sessions=1, ring=True):
        if pool_tokens is None:
            pool_tokens = max_sessions * (w.cache_units * w.unit_kv_tokens + w.n_tokens)
        return cls(n_layers=w.n_layers, d_model=w.d_model, n_heads=w.n_heads,
                   head_dim=w.head_dim, d_mlp=w.d_mlp, c_lat=w.c_lat, n_video=w.n_video,
                   n_audio=w.n_audio, unit_kv_tokens=w.unit_kv_tokens, pool_tokens=pool_tokens,
                   max_sessions=max_sessions,
                   dtype=torch.bfloat16 if w.dtype == "bf16" else torch.float32, ring=ring,
                   rope_theta=w.rope_theta, rms_eps=w.rms_eps, weights=weights, mlp=w.mlp,
                   rope=w.rope, grid_w=w.grid_w)

    def _weights_struct(self, w):
        n = self.cfg.n_layers
        for name in ("w_in", "e_mod", "g_final", "w_out"):
            _need(w[name], self.dtype, name)
        arrs = {}
        for name in ("g_attn", "w_qkv", "w_o", "g_mlp", "w_1", "w_2"):
            ts = [lw[name] for lw in w["layers"]]
            if len(ts) != n:
                raise ValueError(f"weights need {n} layers")
            for t in ts:
                _need(t, self.dtype, name)
            arrs[name] = (C.c_void_p * n)(*[t.data_ptr() for t in ts])
        self._ptr_arrays = arrs
        return L.sfm_weights(w["w_in"].data_ptr(), w["e_mod"].data_ptr(), w["g_final"].data_ptr(),
                             w["w_out"].data_ptr(),
                             *[C.cast(arrs[k], C.POINTER(C.c_void_p))
                               for k in ("g_attn", "w_qkv", "w_o", "g_mlp", "w_1", "w_2")])

    # -- sessions -------------------------------------------------------------
    def open_session(self, cache_units):
        s = C.c_int()
        L.check(L.lib.sfm_session_open(self._h, cache_units, C.byref(s)), "sfm_session_open")
        return s.value

    def reset_session(self, session):
        L.check(L.lib.sfm_session_reset(self._h, session), "sfm_session_reset")

    def session_info(self, session):
        info = L.sfm_session_info()
        L.check(L.lib.sfm_session_get_info(self._h, session, C.byref(info)), "sfm_session_get_info")
        return {f: getattr(info, f) for f, _ in L.sfm_session_info._fields_}

    # -- hot path ---------------------------------------------------------------
    def kvcache_append(self, session, k, v):
        _need(k, self.dtype, "k")
        _need(v, self.dtype, "v", k.shape)
        n_tok = k.shape[1]
        L.check(L.lib.sfm_kvcache_append(self._h, session, _ptr(k), _ptr(v), n_tok, _stream()),
                "sfm_kvcache_append")

    def kvcache_append_heads(self, session, k, v, head0):
        """Appends heads [head0, head0 + n_heads) of a slice whose rows hold more heads
        (one rank's share of a head-sharded cache)."""
        _need(k, self.dtype, "k")
        _need(v, self.dtype, "v", k.shape)
        L.check(L.lib.sfm_kvcache_append_heads(self._h, session, _ptr(k), _ptr(v), k.shape[1],
                                               k.shape[2], head0, _stream()),
                "sfm_kvcache_append_heads")

    def kvcache_read(self, session, layer, row0, n_rows):
        shp = (n_rows, self.shape["n_heads"], self.shape["head_dim"])
        k = torch.empty(shp, dtype=self.dtype, device="cuda")
        v = torch.empty(shp, dtype=self.dtype, device="cuda")
        L.check(L.lib.sfm_kvcache_read(self._h, session, layer, row0, n_rows, _ptr(k), _ptr(v),
                                       _stream()), "sfm_kvcache_read")
        return k, v

    def denoise_step(self, session, z, tau_from, tau_to, v_out=None):
        _need(z, torch.float32, "z", (self.n_tok, self.shape["c_lat"]))
        if v_out is not None:
            _need(v_out, torch.float32, "v_out", z.shape)
        L.check(L.lib.sfm_denoise_step(self._h, session, _ptr(z), tau_from, tau_to, _ptr(v_out),
                                       _stream()), "sfm_denoise_step")

    def fm_solve(self, session, z, taus):
        _need(z, torch.float32, "z", (self.n_tok, self.shape["c_lat"]))
        t = (C.c_float * len(taus))(*taus)
        L.check(L.lib.sfm_fm_solve(self._h, session, _ptr(z), t, len(taus), _stream()),
                "sfm_fm_solve")

    def fm_solve_batched(self, sessions, zs, taus):
        for z in zs:
            _need(z, torch.float32, "z", (self.n_tok, self.shape["c_lat"]))
        n = len(sessions)
        s = (C.c_int * n)(*sessions)
        zp = (C.c_void_p * n)(*[z.data_ptr() for z in zs])
        t = (C.c_float * len(taus))(*taus)
        L.check(L.lib.sfm_fm_solve_batched(self._h, n, s, zp, t, len(taus), _stream()),
                "sfm_fm_solve_batched")

    def fm_solve_guided(self, session, uncond_session, z, taus, scale):
        """Classifier-free-guided solve: v = v_u + scale (v_c - v_u) at every step."""
        _need(z, torch.float32, "z", (self.n_tok, self.shape["c_lat"]))
        t = (C.c_float * len(taus))(*taus)
        L.check(L.lib.sfm_fm_solve_guided(self._h, session, uncond_session, _ptr(z), t, len(taus),
                                          scale, _stream()), "sfm_fm_solve_guided")

    def fm_solve_guided_batched(self, sessions, uncond_sessions, zs, taus, scale, v_outs=None):
        """Guided solves of len(sessions) pairs in one batch; v_outs (optional) receive
        the last step's guided velocities."""
        n = len(sessions)
        if len(uncond_sessions) != n or len(zs) != n:
            raise ValueError("sessions, uncond_sessions and zs differ in length")
        for z in zs:
            _need(z, torch.float32, "z", (self.n_tok, self.shape["c_lat"]))
        vp = None
        if v_outs is not None:
            if len(v_outs) != n:
                raise ValueError("v_outs and sessions differ in length")
            for v in v_outs:
                if v is not None:
                    _need(v, torch.float32, "v_out", (self.n_tok, self.shape["c_lat"]))
            vp = (C.c_void_p * n)(*[_ptr(v) for v in v_outs])
        s = (C.c_int * n)(*sessions)
        u = (C.c_int * n)(*uncond_sessions)
        zp = (C.c_void_p * n)(*[z.data_ptr() for z in zs])
        t = (C.c_float * len(taus))(*taus)
        L.check(L.lib.sfm_fm_solve_guided_batched(self._h, n, s, u, zp, t, len(taus), scale, vp,
                                                  _stream()), "sfm_fm_solve_guided_batched")

    def velocity_units(self, session, zs, taus, v_outs=None, commit=False):
        """Velocities of len(zs) consecutive units after the session's cache in one
        block-causal pass (unit u sees the cache and units <= u); commit appends the
        units' own K/V to the cache.  Returns the velocity tensors."""
        n = len(zs)
        if len(taus) != n:
            raise ValueError("zs and taus differ in length")
        for z in zs:
            _need(z, torch.float32, "z", (self.n_tok, self.shape["c_lat"]))
        if v_outs is None:
            v_outs = [torch.empty_like(z) for z in zs]
        for v in v_outs:
            _need(v, torch.float32, "v_out", (self.n_tok, self.shape["c_lat"]))
        zp = (C.c_void_p * n)(*[z.data_ptr() for z in zs])
        vp = (C.c_void_p * n)(*[v.data_ptr() for v in v_outs])
        t = (C.c_float * n)(*taus)
        L.check(L.lib.sfm_velocity_units(self._h, session, n, zp, t, vp, 1 if commit else 0,
                                         _stream()), "sfm_velocity_units")
        return v_outs

    def plan(self):
        """The projections' launch plan fixed at create (QKV, O, MLP-up, MLP-down)."""
        p = L.sfm_plan()
        L.check(L.lib.sfm_get_plan(self._h, C.byref(p)), "sfm_get_plan")
        return {"block_n": list(p.block_n), "pair": list(p.pair), "k_splits": list(p.k_splits),
                "fused_norm": p.fused_norm}

    def test_fault(self, faults, wait_ns=0):
        """Test-only: fault bits and wait bound of this handle's kernels (0, 0 = normal)."""
        L.check(L.lib.sfm_test_fault(self._h, faults, wait_ns), "sfm_test_fault")

    def clear_device_error(self):
        L.check(L.lib.sfm_clear_device_error(self._h), "sfm_clear_device_error")

    def fm_solve_exact_velocity(self, z0, z, taus):
        """Test-only: the Euler solve with the exact rectified-flow velocity (z - z0) / tau
        in place of f_theta; from z = eps it ends at z0 for any schedule."""
        _need(z0, torch.float32, "z0", (self.n_tok, self.shape["c_lat"]))
        _need(z, torch.float32, "z", z0.shape)
        t = (C.c_float * len(taus))(*taus)
        L.check(L.lib.sfm_fm_solve_exact_velocity(self._h, _ptr(z0), _ptr(z), t, len(taus), _stream()),
                "sfm_fm_solve_exact_velocity")

    def set_graph_mode(self, enabled):
        """Solves as one captured CUDA graph (True, the default) or direct launches."""
        L.check(L.lib.sfm_set_graph_mode(self._h, 1 if enabled else 0), "sfm_set_graph_mode")

    def check_device_error(self):
        """Synchronises and returns the handle's device error word (0 = no kernel problem)."""
        code = C.c_int()
        L.check(L.lib.sfm_check_device_error(self._h, C.byref(code)), "sfm_check_device_error")
        return code.value

    def close(self):
        if self._h:
            L.lib.sfm_destroy(self._h)
            self._h = C.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def attention(q, k, v, out=None, workspace=None, unit_tokens=None):
    """O = softmax(Q K^T / sqrt(D)) V per head; q [n_q][H][D], k/v [n_kv][H][D].

    unit_tokens None: every key visible.  Otherwise block-causal: the queries are
    units of unit_tokens tokens whose own keys are the last n_q keys, the first
    n_kv - n_q keys are a prefix all of them see, and a query sees the keys of
    its own and earlier units only.
    """
    dt = _DT[q.dtype]
    _need(q, q.dtype, "q")
    _need(k, q.dtype, "k")
    _need(v, q.dtype, "v", k.shape)
    n_q, H, D = q.shape
    n_kv = k.shape[0]
    if out is None:
        out = torch.empty_like(q)
    need = L.lib.sfm_attention_workspace_bytes(n_q, n_kv, H, D, dt)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    if unit_tokens is None:
        L.check(L.lib.sfm_attention(_ptr(q), _ptr(k), _ptr(v), _ptr(out), n_q, n_kv, H, D, dt,
                                    _ptr(workspace), ws_bytes, _stream()), "sfm_attention")
    else:
        L.check(L.lib.sfm_attention_block_causal(_ptr(q), _ptr(k), _ptr(v), _ptr(out), n_q, n_kv,
                                                 unit_tokens, H, D, dt, _ptr(workspace), ws_bytes,
                                                 _stream()), "sfm_attention_block_causal")
    return out


def attention_workspace_bytes(n_q, n_kv, n_heads, head_dim, dtype=torch.bfloat16):
    return L.lib.sfm_attention_workspace_bytes(n_q, n_kv, n_heads, head_dim, _DT[dtype])


_LINEAR = {"f32": L.SFM_LINEAR_F32, "out": L.SFM_LINEAR_OUT, "gelu": L.SFM_LINEAR_GELU,
           "resid": L.SFM_LINEAR_RESID}


def linear(x, w, y=None, epilogue="f32"):
    """y = x W^T (w stored [out][in]); epilogue f32 | out | gelu | resid (y += x W^T, fp32 y)."""
    dt = _DT[x.dtype]
    _need(x, x.dtype, "x")
    _need(w, x.dtype, "w")
    M, K = x.shape
    N = w.shape[0]
    if y is None:
        odt = x.dtype if epilogue in ("out", "gelu") else torch.float32
        y = torch.zeros(M, N, dtype=odt, device=x.device)
    _need(y, y.dtype, "y", (M, N))
    L.check(L.lib.sfm_linear(_ptr(x), _ptr(w), _ptr(y), M, N, K, _LINEAR[epilogue], dt, _stream()),
            "sfm_linear")
    return y


def euler_update(z, v, dtau):
    _need(z, torch.float32, "z")
    _need(v, torch.float32, "v", z.shape)
    L.check(L.lib.sfm_euler_update(_ptr(z), _ptr(v), dtau, z.numel(), _stream()),
            "sfm_euler_update")
