"""Scalar-loop re-derivation of the velocity network for tiny sizes.

Written independently of the oracle (plain Python floats, nested loops, the
math module), straight from the definition of each step, so that a transposed
operand, a dropped term or a wrong index in the vectorised oracle shows up as a
mismatch.  Only usable at toy sizes.
"""
import math


def _mat(a):
    """Nested Python lists of floats from an array-like."""
    if hasattr(a, "detach"):
        a = a.detach().double().tolist()
    elif hasattr(a, "tolist"):
        a = a.tolist()
    return a


def matvec_out_in(w, x):
    """y[o] = sum_i w[o][i] x[i] for w stored [out][in]."""
    return [sum(w[o][i] * x[i] for i in range(len(x))) for o in range(len(w))]


def rms(xs, g, eps):
    s = 0.0
    for t in xs:
        s += t * t
    r = 1.0 / math.sqrt(s / len(xs) + eps)
    return [xs[i] * r * g[i] for i in range(len(xs))]


def gelu(t):
    c = math.sqrt(2.0 / math.pi)
    return 0.5 * t * (1.0 + math.tanh(c * (t + 0.044715 * t * t * t)))


def rotate(vec, p, theta):
    d = len(vec)
    half = d // 2
    out = [0.0] * d
    for i in range(half):
        ang = p * theta ** (-2.0 * i / d)
        a, b = vec[i], vec[i + half]
        out[i] = a * math.cos(ang) - b * math.sin(ang)
        out[i + half] = b * math.cos(ang) + a * math.sin(ang)
    return out


def temb(tau, d):
    half = d // 2
    out = [0.0] * d
    for i in range(half):
        w = 10000.0 ** (-2.0 * i / d)
        out[i] = math.sin(1000.0 * tau * w)
        out[i + half] = math.cos(1000.0 * tau * w)
    return out


def attend(qv, keys, vals):
    """One query vector against lists of key/value vectors."""
    d = len(qv)
    logits = [sum(qv[i] * k[i] for i in range(d)) / math.sqrt(d) for k in keys]
    m = max(logits)
    e = [math.exp(l - m) for l in logits]
    s = sum(e)
    return [sum(e[j] * vals[j][i] for j in range(len(keys))) / s for i in range(d)]


def velocity(cfg, z, tau, w, cache_k, cache_v, valid, p0):
    """Velocity per current-unit token, by loops over tokens, heads and features."""
    n, d, H, D = cfg.n_tokens, cfg.d_model, cfg.n_heads, cfg.head_dim
    z = _mat(z)
    w_in = _mat(w["w_in"])
    e_mod = _mat(w["e_mod"])
    te = temb(tau, d)
    x = []
    for j in range(n):
        m = 0 if j < cfg.n_video else 1
        e = matvec_out_in(w_in, z[j])
        x.append([e[i] + e_mod[m][i] + te[i] for i in range(d)])
    for li, lw in enumerate(w["layers"]):
        ck = _mat(cache_k[li])[:valid]
        cv = _mat(cache_v[li])[:valid]
        wq = _mat(lw["w_qkv"])
        qs, ks, vs = [], [], []
        for j in range(n):
            hvec = rms(x[j], _mat(lw["g_attn"]), cfg.rms_eps)
            qkv = matvec_out_in(wq, hvec)
            qh, kh, vh = [], [], []
            for h in range(H):
                qh.append(rotate(qkv[h * D:(h + 1) * D], p0 + j, cfg.rope_theta))
                kh.append(rotate(qkv[H * D + h * D:H * D + (h + 1) * D], p0 + j, cfg.rope_theta))
                vh.append(qkv[2 * H * D + h * D:2 * H * D + (h + 1) * D])
            qs.append(qh)
            ks.append(kh)
            vs.append(vh)
        wo = _mat(lw["w_o"])
        w1 = _mat(lw["w_1"])
        w2 = _mat(lw["w_2"])
        new_x = []
        for j in range(n):
            cat = []
            for h in range(H):
                keys = [ck[t][h] for t in range(valid)] + [ks[t][h] for t in range(n)]
                vals = [cv[t][h] for t in range(valid)] + [vs[t][h] for t in range(n)]
                cat.extend(attend(qs[j][h], keys, vals))
            o = matvec_out_in(wo, cat)
            new_x.append([x[j][i] + o[i] for i in range(d)])
        x = new_x
        for j in range(n):
            h2 = rms(x[j], _mat(lw["g_mlp"]), cfg.rms_eps)
            u = [gelu(t) for t in matvec_out_in(w1, h2)]
            dn = matvec_out_in(w2, u)
            x[j] = [x[j][i] + dn[i] for i in range(d)]
    w_out = _mat(w["w_out"])
    g_f = _mat(w["g_final"])
    return [matvec_out_in(w_out, rms(x[j], g_f, cfg.rms_eps)) for j in range(n)]
