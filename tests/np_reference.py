"""An independent float64 evaluation of the layer with numpy's library
routines (matmul, exp), used only to cross-check the C oracle on small cases.
It shares no code with the oracle or the CUDA path."""
import numpy as np


def _widen(a):
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def _norm(x, gamma, eps):
    r = np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    g = 1.0 if gamma is None else np.asarray(gamma, np.float64)
    return x / r * g


def _softmax(z):
    z = z - z.max(axis=-1, keepdims=True)
    e = np.exp(z)
    return e / e.sum(axis=-1, keepdims=True)


def rope(v, pos, base):
    """Rotary embedding written as complex multiplication: the pair
    (v[e], v[e + d/2]) is the complex number v[e] + i v[e + d/2], multiplied
    by exp(i * pos * base^(-2e/d)).  v [..., d]; pos broadcasts against
    v[..., 0]."""
    v = np.asarray(v, np.float64)
    d = v.shape[-1]
    half = d // 2
    z = v[..., :half] + 1j * v[..., half:]
    theta = base ** (-2.0 * np.arange(half) / d)
    z = z * np.exp(1j * np.asarray(pos, np.float64)[..., None] * theta)
    return np.concatenate([z.real, z.imag], axis=-1)


def decode_layer(H, nq, nkv, d, F, eps, norm, residual, w, x, kc, vc, S, rope_base=None):
    W = {k: _widen(w[k]) for k in ("wq", "wk", "wv", "wo", "wg", "wu", "wd")}
    x = np.asarray(x, np.float64)
    B = x.shape[0]
    g = nq // nkv
    a = _norm(x, w.get("gamma_attn"), eps) if norm else x
    q = a @ W["wq"].T
    k = a @ W["wk"].T
    v = a @ W["wv"].T
    if rope_base is not None:
        q = rope(q.reshape(B, nq, d), S, rope_base).reshape(B, nq * d)
        k = rope(k.reshape(B, nkv, d), S, rope_base).reshape(B, nkv * d)
    Kc = _widen(kc)[:, :, :S, :]
    Vc = _widen(vc)[:, :, :S, :]
    o = np.zeros((B, nq * d))
    for b in range(B):
        for h in range(nq):
            j = h // g
            keys = np.concatenate([Kc[b, j], k[b, j * d:(j + 1) * d][None]], axis=0)
            vals = np.concatenate([Vc[b, j], v[b, j * d:(j + 1) * d][None]], axis=0)
            p = _softmax(keys @ q[b, h * d:(h + 1) * d] / np.sqrt(d))
            o[b, h * d:(h + 1) * d] = p @ vals
    hh = o @ W["wo"].T
    if residual:
        hh = x + hh
    m = _norm(hh, w.get("gamma_mlp"), eps) if norm else hh
    gg = m @ W["wg"].T
    uu = m @ W["wu"].T
    act = gg / (1.0 + np.exp(-gg)) * uu
    y = act @ W["wd"].T
    if residual:
        y = hh + y
    return y, {"q": q, "k_new": k, "v_new": v, "attn": o, "h": hh, "act": act}


def prefill_layer(H, nq, nkv, d, F, eps, norm, residual, w, x, P0=0, kc=None, vc=None, rope_base=None):
    """A chunk of T tokens at positions P0..P0+T-1; kc/vc bf16 bits
    [n_kv][S_cap][d] hold the P0 earlier tokens' keys and values."""
    W = {k: _widen(w[k]) for k in ("wq", "wk", "wv", "wo", "wg", "wu", "wd")}
    x = np.asarray(x, np.float64)
    T = x.shape[0]
    g = nq // nkv
    a = _norm(x, w.get("gamma_attn"), eps) if norm else x
    q = a @ W["wq"].T
    k = a @ W["wk"].T
    v = a @ W["wv"].T
    if rope_base is not None:
        pos = P0 + np.arange(T)[:, None]
        q = rope(q.reshape(T, nq, d), pos, rope_base).reshape(T, nq * d)
        k = rope(k.reshape(T, nkv, d), pos, rope_base).reshape(T, nkv * d)
    o = np.zeros((T, nq * d))
    # key p (0..P0+T-1) is visible to token i when p <= P0 + i
    mask = np.arange(P0 + T)[None, :] <= (P0 + np.arange(T))[:, None]
    for h in range(nq):
        j = h // g
        keys = k[:, j * d:(j + 1) * d]
        vals = v[:, j * d:(j + 1) * d]
        if P0:
            keys = np.concatenate([_widen(kc)[j, :P0], keys], axis=0)
            vals = np.concatenate([_widen(vc)[j, :P0], vals], axis=0)
        s = q[:, h * d:(h + 1) * d] @ keys.T / np.sqrt(d)
        s = np.where(mask, s, -np.inf)
        o[:, h * d:(h + 1) * d] = _softmax(s) @ vals
    hh = o @ W["wo"].T
    if residual:
        hh = x + hh
    m = _norm(hh, w.get("gamma_mlp"), eps) if norm else hh
    gg = m @ W["wg"].T
    uu = m @ W["wu"].T
    act = gg / (1.0 + np.exp(-gg)) * uu
    y = act @ W["wd"].T
    if residual:
        y = hh + y
    return y, k, v
