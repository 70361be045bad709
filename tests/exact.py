"""Exact-arithmetic helpers for the oracle's pins: correctly rounded binary32 results of exact
rationals, and an independent exact re-derivation of one compressed step for tiny inputs.

Nothing here calls the oracle. The re-derivation takes each fp32 operation as the exact
rational result rounded once to binary32 (round to nearest, ties to even), sums norms exactly,
and rounds square roots correctly, so it follows a different arithmetic route from the C oracle
(which sums in fp64 and converts through doubles).
"""
from __future__ import annotations

import math
from fractions import Fraction as F

import numpy as np

F32_MAX = F(2 ** 128 - 2 ** 104)


def _floor_log2(a: F) -> int:
    """floor(log2(a)) for a > 0."""
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if F(2) ** e > a:
        e -= 1
    elif F(2) ** (e + 1) <= a:
        e += 1
    return e


def _round_half_even(q: F) -> int:
    n = q.numerator // q.denominator
    r = q - n
    if r > F(1, 2) or (r == F(1, 2) and n % 2 == 1):
        n += 1
    return n


def r32(q) -> np.float32:
    """Correct rounding of an exact rational to binary32 (a zero result is +0)."""
    q = F(q)
    if q == 0:
        return np.float32(0.0)
    sign = -1 if q < 0 else 1
    a = abs(q)
    e = max(_floor_log2(a), -126)
    quantum = F(2) ** (e - 23)
    val = _round_half_even(a / quantum) * quantum
    if val > F32_MAX:
        return np.float32(sign * np.inf)
    return np.float32(sign * float(val))


def r32_sqrt(a) -> np.float32:
    """Correctly rounded binary32 square root of an exact non-negative rational."""
    a = F(a)
    assert a >= 0
    if a == 0:
        return np.float32(0.0)
    f = np.float32(math.sqrt(float(a)))
    while True:
        lo = np.nextafter(f, np.float32(0.0), dtype=np.float32)
        hi = np.nextafter(f, np.float32(np.inf), dtype=np.float32)
        mid_lo = (F(float(lo)) + F(float(f))) / 2
        mid_hi = (F(float(f)) + F(float(hi))) / 2
        if a < mid_lo * mid_lo or (a == mid_lo * mid_lo and _odd(f)):
            f = lo
        elif a > mid_hi * mid_hi or (a == mid_hi * mid_hi and _odd(f)):
            f = hi
        else:
            return f


def _odd(f: np.float32) -> bool:
    return bool(np.array(f, dtype=np.float32).view(np.uint32) & 1)


def ulp32(x) -> float:
    x = abs(np.float32(x))
    return float(np.nextafter(x, np.float32(np.inf), dtype=np.float32) - x)


def fr(x) -> F:
    return F(float(np.float32(x)))


def exact_compressed_step(x, m, v, e_w, e_s, g, C, beta1, eps, lr):
    """Exact re-derivation of one compressed step (tiny inputs only).

    g is float32 [W][d]. Returns a dict of numpy results; does not modify its inputs."""
    g = np.asarray(g, dtype=np.float32)
    W, d = g.shape
    nch = (d + C - 1) // C
    b1 = fr(beta1)
    omb1 = fr(r32(1 - b1))
    xw = np.zeros((W, d), dtype=np.float32)
    for w in range(W):
        for i in range(d):
            mw = r32(fr(r32(b1 * fr(m[i]))) + fr(r32(omb1 * fr(g[w, i]))))
            xw[w, i] = r32(fr(mw) + fr(e_w[w, i]))
    s = np.zeros((W, nch), dtype=np.float32)
    bits = xw >= 0
    new_ew = np.zeros((W, d), dtype=np.float32)
    for w in range(W):
        for k in range(nch):
            lo, hi = k * C, min(d, (k + 1) * C)
            ss = sum((fr(xw[w, i]) ** 2 for i in range(lo, hi)), F(0))
            s[w, k] = r32_sqrt(ss / (hi - lo))
            for i in range(lo, hi):
                q = fr(s[w, k]) if bits[w, i] else -fr(s[w, k])
                new_ew[w, i] = r32(fr(xw[w, i]) - q)
    z = np.zeros(d, dtype=np.float32)
    y = np.zeros(d, dtype=np.float32)
    S = np.zeros(nch, dtype=np.float32)
    new_es = np.zeros(d, dtype=np.float32)
    for k in range(nch):
        lo, hi = k * C, min(d, (k + 1) * C)
        for i in range(lo, hi):
            acc = sum(((fr(s[w, k]) if bits[w, i] else -fr(s[w, k])) for w in range(W)), F(0))
            y[i] = r32(acc / W)
            z[i] = r32(fr(y[i]) + fr(e_s[i]))
        ss = sum((fr(z[i]) ** 2 for i in range(lo, hi)), F(0))
        S[k] = r32_sqrt(ss / (hi - lo))
        for i in range(lo, hi):
            new_es[i] = r32(fr(z[i]) - (fr(S[k]) if z[i] >= 0 else -fr(S[k])))
    new_m = np.zeros(d, dtype=np.float32)
    new_x = np.zeros(d, dtype=np.float32)
    for i in range(d):
        k = i // C
        new_m[i] = S[k] if z[i] >= 0 else -S[k]
        den = r32(fr(r32_sqrt(fr(v[i]))) + fr(eps))
        qv = r32(fr(new_m[i]) / fr(den))
        upd = r32(fr(lr) * fr(qv))
        new_x[i] = r32(fr(x[i]) - fr(upd))
    return {"xw": xw, "s": s, "bits_w": bits, "e_w": new_ew, "y": y, "z": z, "S": S,
            "bits_s": z >= 0, "e_s": new_es, "m": new_m, "x": new_x}


def exact_zero_one_run(x, m, v, g_list, lr_list, C, H, K, beta1, beta2, eps):
    """Exact re-derivation of the 0/1 Adam variant's compression phase (tiny inputs only): from
    the state at the freeze (x, shared m, v; residuals zero) through the steps of g_list
    ([W][d] float32 each) with learning rates lr_list; a synchronisation after every H-th step,
    a variance refresh at every K-th synchronisation (K = 0: never). Every fp32 operation is the
    exact rational result rounded once to binary32 and norms are summed exactly.

    Returns the final x, v, m_w, u_w, e_w, e_s and the list of each synchronisation's
    messages (s, bits_w, S, bits_s, mbar)."""
    g0 = np.asarray(g_list[0], dtype=np.float32)
    W, d = g0.shape
    nch = (d + C - 1) // C
    b1, b2 = fr(beta1), fr(beta2)
    omb1, omb2 = fr(r32(1 - b1)), fr(r32(1 - b2))
    x = np.array(x, dtype=np.float32)
    v = np.array(v, dtype=np.float32)
    m_w = np.array(np.broadcast_to(np.asarray(m, dtype=np.float32), (W, d)), dtype=np.float32)
    u_w = np.zeros((W, d), dtype=np.float32)
    e_w = np.zeros((W, d), dtype=np.float32)
    e_s = np.zeros(d, dtype=np.float32)
    gamma = np.float32(0.0)
    syncs = []
    for t, (g, lr) in enumerate(zip(g_list, lr_list), start=1):
        g = np.asarray(g, dtype=np.float32)
        lrf = fr(lr)
        for w in range(W):
            for i in range(d):
                m_w[w, i] = r32(fr(r32(b1 * fr(m_w[w, i]))) + fr(r32(omb1 * fr(g[w, i]))))
                u_w[w, i] = r32(fr(u_w[w, i]) + fr(r32(lrf * fr(m_w[w, i]))))
        gamma = r32(fr(gamma) + lrf)
        if t % H:
            continue
        xw = np.zeros((W, d), dtype=np.float32)
        for w in range(W):
            for i in range(d):
                xw[w, i] = r32(fr(u_w[w, i]) + fr(e_w[w, i]))
        bits = xw >= 0
        s = np.zeros((W, nch), dtype=np.float32)
        for w in range(W):
            for k in range(nch):
                lo, hi = k * C, min(d, (k + 1) * C)
                ss = sum((fr(xw[w, i]) ** 2 for i in range(lo, hi)), F(0))
                s[w, k] = r32_sqrt(ss / (hi - lo))
                for i in range(lo, hi):
                    q = fr(s[w, k]) if bits[w, i] else -fr(s[w, k])
                    e_w[w, i] = r32(fr(xw[w, i]) - q)
        z = np.zeros(d, dtype=np.float32)
        S = np.zeros(nch, dtype=np.float32)
        for k in range(nch):
            lo, hi = k * C, min(d, (k + 1) * C)
            for i in range(lo, hi):
                acc = sum(((fr(s[w, k]) if bits[w, i] else -fr(s[w, k])) for w in range(W)),
                          F(0))
                y = r32(acc / W)
                z[i] = r32(fr(y) + fr(e_s[i]))
            ss = sum((fr(z[i]) ** 2 for i in range(lo, hi)), F(0))
            S[k] = r32_sqrt(ss / (hi - lo))
            for i in range(lo, hi):
                e_s[i] = r32(fr(z[i]) - (fr(S[k]) if z[i] >= 0 else -fr(S[k])))
        refresh = K > 0 and (len(syncs) + 1) % K == 0
        mbar = np.zeros(d, dtype=np.float32)
        for i in range(d):
            k = i // C
            ubar = fr(S[k]) if z[i] >= 0 else -fr(S[k])
            den = r32(fr(r32_sqrt(fr(v[i]))) + fr(eps))
            x[i] = r32(fr(x[i]) - fr(r32(ubar / fr(den))))
            mbar[i] = r32(ubar / fr(gamma))
            if refresh:
                v[i] = r32(fr(r32(b2 * fr(v[i]))) + fr(r32(omb2 * fr(r32(fr(mbar[i]) ** 2)))))
        m_w[:] = mbar
        u_w[:] = 0.0
        gamma = np.float32(0.0)
        syncs.append({"s": s, "bits_w": bits, "S": S, "bits_s": z >= 0, "mbar": mbar,
                      "refresh": refresh})
    return {"x": x, "v": v, "m_w": m_w, "u_w": u_w, "e_w": e_w, "e_s": e_s, "syncs": syncs}
