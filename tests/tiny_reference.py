"""A second, independent implementation of the whole denoise loop for tiny
shapes (test-only): plain Python loops and direct formulas, f32 storage, no
code shared with oracle/. Token draws use numpy's own Philox-4x64 generator.

It follows the same readings of the pages as the oracle (one layer; f32
rounding after the Q/K/V projections, after attention and after the residual
sum; one softmax over prompt + canvas keys per request; entropy in nats of the
softmax of the logits; freeze the k_t = ceil(U / (T - t)) unfrozen positions
smallest by (entropy, position) to their argmax, the rest frozen to their argmax
at the last step or on an adaptive stop, every other open position redrawn from
(seed, step + 1, position, canvas))."""
import math
import struct

import numpy as np

_M64 = (1 << 64) - 1


def f32(x):
    return struct.unpack("f", struct.pack("f", x))[0]


def draw(seed, step, pos, canvas, V):
    """Word 0 of Philox-4x64-10 at counter (pos, step, canvas, 0), key (seed, 0),
    mapped to [0, V) by the high 32 bits times V, shifted down 32."""
    c = (pos | (step << 64) | (canvas << 128)) - 1
    bg = np.random.Philox(key=int(seed))
    st = bg.state
    st["state"]["counter"] = np.array([(c >> (64 * i)) & _M64 for i in range(4)], dtype=np.uint64)
    st["buffer_pos"] = 4
    bg.state = st
    x0 = int(bg.random_raw(1)[0])
    return ((x0 >> 32) * V) >> 32


def _rows(a):
    return [[float(v) for v in r] for r in np.asarray(a, dtype=np.float64).reshape(np.asarray(a).shape[0], -1)]


def forward_canvas(w, Kp, Vp, tok, Hq, Hk, h):
    """Entropy and argmax of every position of one canvas. w = (E, layers, Wl)
    with layers a list of (Wq, Wk, Wv, Wo); Kp, Vp: per layer, the prompt
    keys / values (lists of rows)."""
    E, layers, Wl = w
    d = len(E[0])
    X = [E[t] for t in tok]
    proj = lambda W, x: [f32(sum(x[k] * W[j][k] for k in range(d))) for j in range(len(W))]
    for (Wq, Wk, Wv, Wo), kp, vp in zip(layers, Kp, Vp):
        Q = [proj(Wq, x) for x in X]
        K = kp + [proj(Wk, x) for x in X]
        Vv = vp + [proj(Wv, x) for x in X]
        O = []
        for q in Q:
            o = []
            for hq in range(Hq):
                g = hq // (Hq // Hk)
                s = [sum(q[hq * h + i] * k[g * h + i] for i in range(h)) / math.sqrt(h) for k in K]
                m = max(s)
                e = [math.exp(v - m) for v in s]
                z = sum(e)
                o += [f32(sum(e[j] / z * Vv[j][g * h + i] for j in range(len(K)))) for i in range(h)]
            O.append(o)
        X = [[f32(x[k] + sum(o[j] * Wo[k][j] for j in range(len(o)))) for k in range(d)] for x, o in zip(X, O)]
    ents, ams = [], []
    for hs in X:
        lg = [sum(hs[k] * wl[k] for k in range(d)) for wl in Wl]
        m = max(lg)
        e = [math.exp(v - m) for v in lg]
        z = sum(e)
        ents.append(-sum((v / z) * math.log(v / z) for v in e if v > 0.0))
        ams.append(min(i for i, v in enumerate(lg) if v == m))
    return ents, ams


def decode(weights, prefix, seeds, C, V, Hq, Hk, h, T, stop_entropy, adaptive, init_tok=None):
    """Whole decode of every canvas; returns (tokens [B][C], steps [B],
    entropies [B][steps][C])."""
    stacked = np.asarray(weights["wq"]).ndim == 3  # [L][out][in] per layer
    L = np.asarray(weights["wq"]).shape[0] if stacked else 1
    per_layer = lambda k: [weights[k][l] for l in range(L)] if stacked else [weights[k]]
    layers = list(zip(*[[_rows(m) for m in per_layer(k)] for k in ("wq", "wk", "wv", "wo")]))
    w = (_rows(weights["embed"]), layers, _rows(weights["lm_head"]))
    out_tok, out_steps, out_ent = [], [], []
    for b, seed in enumerate(seeds):
        rows = lambda a: [[list(map(float, np.asarray(r, np.float64).reshape(-1))) for r in lay]
                          for lay in (np.asarray(a).reshape(L, -1, Hk, h))]
        Kp, Vp = rows(prefix[b][0]), rows(prefix[b][1])
        tok = [draw(seed, 0, p, b, V) for p in range(C)] if init_tok is None else list(init_tok[b])
        frozen = [False] * C
        t = 0
        trace = []
        while True:
            ents, ams = forward_canvas(w, Kp, Vp, tok, Hq, Hk, h)
            trace.append(ents)
            open_ = [p for p in range(C) if not frozen[p]]
            U = len(open_)
            k = U if T - t <= 1 else (U + (T - t) - 1) // (T - t)
            chosen = sorted(open_, key=lambda p: (ents[p], p))[:k]
            for p in chosen:
                tok[p], frozen[p] = ams[p], True
            rest = [p for p in range(C) if not frozen[p]]
            stop = not rest or (adaptive and min(ents[p] for p in rest) < stop_entropy)
            t += 1
            if stop:
                for p in rest:
                    tok[p], frozen[p] = ams[p], True
                break
            for p in rest:
                tok[p] = draw(seed, t, p, b, V)
        out_tok.append(tok)
        out_steps.append(t)
        out_ent.append(trace)
    return out_tok, out_steps, out_ent
