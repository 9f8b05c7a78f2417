"""Plain fp64 CPU oracle of one DiffusionGemma-style canvas denoise step and of
the whole block decode.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py). It shares no code with the
CUDA library: it is written in numpy from the pages, and only the seeded input
generators feed both sides.

What the pages fix, and where (page title, section):
  * the canvas is 256 positions refined together, each starting as a random
    token rather than [MASK] -- "DiffusionGemma解析" 整片并行去噪; "DiffusionGemma
    深度拆解" 架构解剖 4 (统一状态扩散); "谷歌DiffusionGemma" 工作原理.
  * every canvas position attends to every other one, no causal mask --
    "DiffusionGemma解析" 整片并行去噪 (last paragraph); "DiffusionGemma深度拆解"
    架构解剖 2 (双向注意力); the decoder reads the encoder's prompt KV cache --
    架构解剖, overall diagram.
  * the model gives a distribution per position; lower entropy means more
    confident; positions are sorted by entropy ascending, the most certain are
    frozen, the rest get fresh noise -- "DiffusionGemma解析" 整片并行去噪.
  * the frozen token is the one the model is most sure of; unsure positions
    are re-randomised; the block converges once enough positions are stable --
    "谷歌DiffusionGemma" 工作原理.
  * at most 48 steps with an adaptive stop -- "DiffusionGemma解析" 自适应停步机制.
  * MoE FFN: 128 fine-grained experts plus one shared expert, top-8 routing --
    "DiffusionGemma深度拆解" 架构解剖 3.

Readings where the pages are silent: single
layer, embed -> attention -> Wo + residual (-> MoE + residual) -> LM head, no
norm and no positional encoding; KV head g = q // (Hq/Hk); softmax scale
1/sqrt(h); freeze count k_t = ceil(U_t / (T - t)); freeze set = the k_t
unfrozen positions smallest by (entropy, position); frozen token = that step's
argmax (lowest vocab index on ties); every other unfrozen position is redrawn;
stop when nothing is unfrozen or (adaptive) when the smallest entropy among the
still-unfrozen positions is below the threshold, in which case they take their
argmax; entropy uses logits times a per-position inverse temperature, the argmax
uses the unscaled logits; GELU is the exact erf form; the shared expert has gate
weight 1.

Every matmul is computed in fp64 by numpy. Values are rounded to the storage
dtype (bf16 or f32) exactly where the GPU path stores them: Q, canvas K/V, O,
Hs, the expert intermediate and the post-MoE Hs.
"""
import math

import numpy as np

from .numerics import e4m3_to_f64, quantize_rows_e4m3, round_storage, widen
from .philox import canvas_draw

LM_CHUNK = 8192  # vocab rows widened to fp64 at a time (memory only)


# --------------------------------------------------------------------------
# model description helpers
# --------------------------------------------------------------------------
def dims(model):
    return (model["d"], model["Hq"], model["Hk"], model["h"], model["V"])


def prewiden(model, keys=("wq", "wk", "wv", "wo", "lm_head")):
    """A copy of the model dict whose `keys` hold fp64 values instead of stored
    bits (same numbers; saves re-widening them on every call)."""
    m = dict(model)
    for k in keys:
        m[k] = widen(model[k], model["dtype"])
    return m


def n_layers(model):
    """Number of attention layers. A model dict with "n_layers" holds its
    layer weights stacked layer-major (wq, wk, wv, wo as [L][out][in]) and its
    prompt caches as [L][S][Hk][h] per request; without it the model has one
    layer and unstacked arrays."""
    return int(model.get("n_layers", 1))


def layer(model, l):
    """The one-layer view of layer l: its own wq, wk, wv, wo."""
    if "n_layers" not in model:
        assert l == 0
        return model
    m = dict(model)
    for k in ("wq", "wk", "wv", "wo"):
        m[k] = model[k][l]
    return m


def layer_prefix(model, prefix, l):
    """Each request's prompt K/V of layer l."""
    if "n_layers" not in model:
        assert l == 0
        return prefix
    _, _, Hk, h, _ = dims(model)
    return [(np.asarray(k).reshape(n_layers(model), -1, Hk, h)[l], np.asarray(v).reshape(n_layers(model), -1, Hk, h)[l])
            for k, v in prefix]


def kv_head_of(q, Hq, Hk):
    """Consecutive query heads share one KV head."""
    return q // (Hq // Hk)


# --------------------------------------------------------------------------
# forward stages
# --------------------------------------------------------------------------
def embed(model, tok):
    """X[b*C+p, :] = E[tok[b,p], :] (exact, the table is already in storage dtype)."""
    E = model["embed"]
    rows = np.asarray(tok, dtype=np.int64).reshape(-1)
    return widen(E[rows], model["dtype"])


def project_qkv(model, X):
    """Q = X Wq^T, K_c = X Wk^T, V_c = X Wv^T, each rounded to storage dtype."""
    d, Hq, Hk, h, _ = dims(model)
    dt = model["dtype"]
    Q = round_storage(X @ widen(model["wq"], dt).T, dt).reshape(-1, Hq, h)
    Kc = round_storage(X @ widen(model["wk"], dt).T, dt).reshape(-1, Hk, h)
    Vc = round_storage(X @ widen(model["wv"], dt).T, dt).reshape(-1, Hk, h)
    return Q, Kc, Vc


def block_kv(model, tok):
    """K and V of committed canvases, as stored: the next block attends to them
    after the request's prompt ("DiffusionGemma深度拆解" 架构解剖 1: blocks in
    sequence, parallel inside a block; the committed block's K/V come from the
    causal encoder pass). With one layer and no positional encoding a token's
    K/V depend only on its own embedding, so that pass is the K/V projection of
    the committed tokens. tok: [B][C]; returns K, V as [B][C][Hk][h] (fp64
    values rounded to the storage dtype)."""
    assert n_layers(model) == 1, "block K/V are defined for the single-layer model"
    B, C = np.asarray(tok).shape
    _, Kc, Vc = project_qkv(model, embed(model, tok))
    _, _, Hk, h, _ = dims(model)
    return Kc.reshape(B, C, Hk, h), Vc.reshape(B, C, Hk, h)


def append_block(model, prefix, K, V):
    """Each request's prompt K/V followed by its committed block's K/V (fp64)."""
    _, _, Hk, h, _ = dims(model)
    dt = model["dtype"]
    out = []
    for b, (pk, pv) in enumerate(prefix):
        pk = widen(pk, dt).reshape(-1, Hk, h)
        pv = widen(pv, dt).reshape(-1, Hk, h)
        out.append((np.concatenate([pk, K[b]]), np.concatenate([pv, V[b]])))
    return out


def softmax_rows(s):
    m = np.max(s, axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / np.sum(e, axis=-1, keepdims=True)


def attention(model, Q, Kc, Vc, prefix, B, C):
    """Bidirectional GQA attention of each canvas query over [prefix K/V ; canvas K/V].

    Q: [B*C, Hq, h]; Kc, Vc: [B*C, Hk, h]; prefix: list of (K_pre, V_pre) per
    request, each [S_b, Hk, h] (stored dtype). No mask: every query sees all
    S_b + C keys of its own request. Returns O [B*C, Hq*h] rounded to storage.
    """
    d, Hq, Hk, h, _ = dims(model)
    dt = model["dtype"]
    scale = 1.0 / math.sqrt(h)
    O = np.zeros((B * C, Hq, h), dtype=np.float64)
    for b in range(B):
        Kp, Vp = prefix[b]
        Kp = widen(Kp, dt).reshape(-1, Hk, h)
        Vp = widen(Vp, dt).reshape(-1, Hk, h)
        Kall = np.concatenate([Kp, Kc[b * C:(b + 1) * C]], axis=0)
        Vall = np.concatenate([Vp, Vc[b * C:(b + 1) * C]], axis=0)
        for q in range(Hq):
            g = kv_head_of(q, Hq, Hk)
            s = (Q[b * C:(b + 1) * C, q, :] @ Kall[:, g, :].T) * scale
            P = softmax_rows(s)
            O[b * C:(b + 1) * C, q, :] = P @ Vall[:, g, :]
    return round_storage(O.reshape(B * C, Hq * h), dt)


def out_proj_residual(model, X, O):
    """Hs = X + O Wo^T, rounded to storage dtype."""
    dt = model["dtype"]
    return round_storage(X + O @ widen(model["wo"], dt).T, dt)


def gelu_exact(x):
    from scipy.special import erf
    return 0.5 * x * (1.0 + erf(x / math.sqrt(2.0)))


def moe_route(model, Hs, choice=None):
    """Router logits, softmax, top-k by probability (lower expert index first on
    ties), gates renormalised over the chosen experts. Returns (logits, idx, gates).

    choice: optional [rows, k] expert indices used instead of the top-k (to
    evaluate another valid choice where the k-th and (k+1)-th probabilities of
    a row are tied within the comparison tolerance); the gates are still the
    softmax probabilities of the chosen experts renormalised over them."""
    dt = model["dtype"]
    r = Hs @ widen(model["w_router"], dt).T
    p = softmax_rows(r)
    k = model["top_k"]
    E = p.shape[1]
    if choice is None:
        # stable sort on -p keeps the lower index first among equal probabilities
        order = np.argsort(-p, axis=1, kind="stable")[:, :k]
    else:
        order = np.asarray(choice, dtype=np.int64).reshape(p.shape[0], k)
    gp = np.take_along_axis(p, order, axis=1)
    gates = gp / np.sum(gp, axis=1, keepdims=True)
    assert E == model["n_experts"]
    return r, order, gates


def dequant_rows_e4m3(codes, scales):
    """e4m3 codes times their power-of-two row scales (exact)."""
    return e4m3_to_f64(codes) * np.asarray(scales, dtype=np.float64)[..., None]


def fp8_matmul_rows(x, w_codes, w_scales):
    """x W^T with W stored as e4m3 codes and row scales, x quantized per row to
    e4m3 with its own power-of-two scale (as the FP8 LM head); both sides are
    dequantized exactly, so the fp64 product is the exact FP8 product."""
    qx, ex = quantize_rows_e4m3(x)
    return dequant_rows_e4m3(qx, np.exp2(ex.astype(np.float64))) @ dequant_rows_e4m3(w_codes, w_scales).T


def expert_ffn(model, e, x):
    """FFN_e(x) = W_down (GELU(W_gate x) * (W_up x)); intermediate rounded to storage.

    With e4m3 expert weights (model["w_gate_scale"] present: w_gate, w_up and
    w_down hold e4m3 codes with power-of-two scales per output row) each of
    the three products is an FP8 one: the token rows are quantized per row for
    the gate and up projections, and the intermediate (after its rounding to
    the storage dtype) per row for the down projection."""
    dt = model["dtype"]
    if "w_gate_scale" in model:
        g = fp8_matmul_rows(x, model["w_gate"][e], model["w_gate_scale"][e])
        u = fp8_matmul_rows(x, model["w_up"][e], model["w_up_scale"][e])
        a = round_storage(gelu_exact(g) * u, dt)
        return fp8_matmul_rows(a, model["w_down"][e], model["w_down_scale"][e])
    g = x @ widen(model["w_gate"][e], dt).T
    u = x @ widen(model["w_up"][e], dt).T
    a = round_storage(gelu_exact(g) * u, dt)
    return a @ widen(model["w_down"][e], dt).T


def moe_block(model, Hs, choice=None):
    """Hs + sum_e gate_e FFN_e(Hs) + sum_shared FFN_shared(Hs), rounded to storage.
    choice: optional expert indices per row (see moe_route)."""
    dt = model["dtype"]
    r, idx, gates = moe_route(model, Hs, choice)
    E = model["n_experts"]
    out = np.zeros_like(Hs)
    for e in range(E):
        rows, slot = np.nonzero(idx == e)
        if rows.size == 0:
            continue
        y = expert_ffn(model, e, Hs[rows])
        out[rows] += gates[rows, slot][:, None] * y
    for s in range(model["n_shared"]):
        out += expert_ffn(model, E + s, Hs)
    return round_storage(Hs + out, dt), (r, idx, gates)


def lm_head_logits(model, Hs_rows):
    """Unscaled logits Hs W_lm^T in fp64 for the given rows: [rows, V].

    With FP8 LM-head weights (model["lm_head_e4m3"]: e4m3 codes [V][d] with
    power-of-two row scales s_v = model["lm_head_scale"][v]) the product is the
    FP8 one: each row of Hs is quantized to e4m3 with its own power-of-two
    scale 2^e_r, and x[r][v] = 2^e_r s_v sum_k q_r[k] q_v[k]. Every e4m3 value is
    an integer multiple of 2^-9 of magnitude below 2^9, so each product has at
    most 8 significant bits and a sum over d <= 2^20 terms stays an exact
    multiple of 2^-18 below 2^38: the fp64 dot product is exact."""
    if model.get("lm_head_e4m3") is not None:
        return lm_head_logits_e4m3(model, Hs_rows)
    dt = model["dtype"]
    W = model["lm_head"]
    V = W.shape[0]
    out = np.empty((Hs_rows.shape[0], V), dtype=np.float64)
    for v0 in range(0, V, LM_CHUNK):
        v1 = min(V, v0 + LM_CHUNK)
        out[:, v0:v1] = Hs_rows @ widen(W[v0:v1], dt).T
    return out


def lm_head_logits_e4m3(model, Hs_rows):
    """The FP8 LM head (see lm_head_logits)."""
    qa, ea = quantize_rows_e4m3(Hs_rows)
    a = e4m3_to_f64(qa)
    W = model["lm_head_e4m3"]
    sw = np.asarray(model["lm_head_scale"], dtype=np.float64)
    V = W.shape[0]
    out = np.empty((Hs_rows.shape[0], V), dtype=np.float64)
    for v0 in range(0, V, LM_CHUNK):
        v1 = min(V, v0 + LM_CHUNK)
        dot = a @ e4m3_to_f64(W[v0:v1]).T
        out[:, v0:v1] = dot * np.exp2(ea.astype(np.float64))[:, None] * sw[None, v0:v1]
    return out


def entropy_of_logits(l):
    """H = -sum_i p_i ln p_i with p = softmax(l) along the last axis (0 ln 0 = 0)."""
    p = softmax_rows(l)
    with np.errstate(divide="ignore", invalid="ignore"):
        t = np.where(p > 0.0, p * np.log(np.where(p > 0.0, p, 1.0)), 0.0)
    return -np.sum(t, axis=-1)


def argmax_lowest(l):
    """Argmax along the last axis; np.argmax returns the first (lowest) index on ties."""
    return np.argmax(l, axis=-1)


def top2_gap(l):
    """top-1 minus top-2 logit per row (0 when the maximum is tied)."""
    part = np.partition(l, -2, axis=-1)
    return part[..., -1] - part[..., -2]


def entropy_argmax(logits, inv_temp_rows):
    """Per-row entropy of softmax(logits * invT) and argmax of the unscaled logits."""
    ent = entropy_of_logits(logits * inv_temp_rows[:, None])
    am = argmax_lowest(logits)
    return ent, am, top2_gap(logits)


# --------------------------------------------------------------------------
# freeze schedule and selection
# --------------------------------------------------------------------------
def freeze_count(U, t, T):
    """k_t = ceil(U_t / (T - t)); everything left is frozen at the last step."""
    if U <= 0:
        return 0
    if T - t <= 1:
        return U
    return -(-U // (T - t))


def select_freeze(ent_row, frozen_row, k):
    """The k unfrozen positions smallest by the key (entropy, position)."""
    cand = [p for p in range(len(ent_row)) if not frozen_row[p]]
    cand.sort(key=lambda p: (float(ent_row[p]), p))
    mask = np.zeros(len(ent_row), dtype=bool)
    for p in cand[:k]:
        mask[p] = True
    return mask


# --------------------------------------------------------------------------
# state, step, decode
# --------------------------------------------------------------------------
def init_state(seeds, C, V):
    """Canvas b, position p starts at draw(seed_b, step 0, p, b); nothing frozen."""
    B = len(seeds)
    tok = np.array([[canvas_draw(int(seeds[b]), 0, p, b, V) for p in range(C)]
                    for b in range(B)], dtype=np.int64)
    return {
        "tok": tok,
        "frozen": np.zeros((B, C), dtype=bool),
        "step": np.zeros(B, dtype=np.int64),
        "done": np.zeros(B, dtype=bool),
        "seed": np.array([int(s) for s in seeds], dtype=np.uint64),
    }


def init_state_fixed(seeds, C, V, fixed_mask, fixed_tok):
    """A block with some positions given in advance: infilling between a given
    prefix and suffix, or a puzzle's given cells ("DiffusionGemma深度拆解" 为什么值得
    重视 2, fill-in-the-middle, constraints propagating from every direction;
    "谷歌DiffusionGemma" 工作原理, constrained generation). Positions with
    fixed_mask take fixed_tok and start frozen, so they keep their tokens and
    only the open positions count as unfrozen in the freeze schedule; every
    other position starts at its step-0 draw, as in init_state."""
    st = init_state(seeds, C, V)
    mask = np.asarray(fixed_mask, dtype=bool).reshape(st["tok"].shape)
    tok = np.asarray(fixed_tok, dtype=np.int64).reshape(st["tok"].shape)
    st["tok"] = np.where(mask, tok, st["tok"])
    st["frozen"] = mask.copy()
    return st


def copy_state(st):
    return {k: v.copy() for k, v in st.items()}


def attention_layer(model, prefix, X, B, C, l):
    """Layer l: Q/K/V of its input X, attention over the layer's prompt K/V
    and the canvas, Wo + residual. Returns (Q, Kc, Vc, O, output)."""
    ml, pl = layer(model, l), layer_prefix(model, prefix, l)
    Q, Kc, Vc = project_qkv(ml, X)
    O = attention(ml, Q, Kc, Vc, pl, B, C)
    return Q, Kc, Vc, O, out_proj_residual(ml, X, O)


def forward(model, prefix, tok, inv_temp):
    """One forward pass over all canvases: returns (ent, am, gap, extras).

    Layers in sequence, each fed the previous one's output (the residual
    stream); the LM head reads the last layer's output. extras holds the
    embedding X, the last layer's Q, canvas K/V and attention output O, every
    layer's output ("layers") and Hs_attn (the last one)."""
    B, C = tok.shape
    X = embed(model, tok)
    extras = {"X": X, "layers": []}
    Hs = X
    for l in range(n_layers(model)):
        Q, Kc, Vc, O, Hs = attention_layer(model, prefix, Hs, B, C, l)
        extras["layers"].append(Hs)
    extras.update({"Q": Q, "Kc": Kc, "Vc": Vc, "O": O, "Hs_attn": Hs})
    if model.get("n_experts", 0):
        assert n_layers(model) == 1, "the MoE block is defined for the single-layer model"
        Hs, route = moe_block(model, Hs)
        extras["route"] = route
    extras["Hs"] = Hs
    invT = np.ones(B * C) if inv_temp is None else np.asarray(inv_temp, np.float64).reshape(-1)
    logits = lm_head_logits(model, Hs)
    ent, am, gap = entropy_argmax(logits, invT)
    return ent.reshape(B, C), am.reshape(B, C), gap.reshape(B, C), extras


def apply_selection(state, ent, am, sched, V):
    """Freeze, stop test and re-noise for every canvas that is not done.

    Returns the new state and a per-canvas record of the decisions taken."""
    T = sched["max_steps"]
    thr = sched["stop_entropy"]
    adaptive = sched["adaptive_stop"]
    st = copy_state(state)
    B, C = st["tok"].shape
    recs = []
    for b in range(B):
        if st["done"][b]:
            recs.append(None)
            continue
        t = int(st["step"][b])
        frozen = st["frozen"][b]
        U = int(np.count_nonzero(~frozen))
        k = freeze_count(U, t, T)
        F = select_freeze(ent[b], frozen, k)
        st["tok"][b, F] = am[b, F]
        st["frozen"][b] |= F
        rest = ~st["frozen"][b]
        min_rest = float(np.min(ent[b][rest])) if rest.any() else math.inf
        stop = (not rest.any()) or (adaptive and min_rest < thr)
        if stop:
            st["tok"][b, rest] = am[b, rest]
            st["frozen"][b, :] = True
            st["done"][b] = True
        else:
            seed = int(st["seed"][b])
            for p in np.nonzero(rest)[0]:
                st["tok"][b, p] = canvas_draw(seed, t + 1, int(p), b, V)
        st["step"][b] = t + 1
        recs.append({"t": t, "U": U, "k": k, "freeze": F, "stop": stop,
                     "min_rest": min_rest})
    return st, recs


def denoise_step(model, prefix, state, sched, inv_temp=None):
    """One denoise step of every canvas. Returns (new_state, record)."""
    ent, am, gap, extras = forward(model, prefix, state["tok"], inv_temp)
    new_state, recs = apply_selection(state, ent, am, sched, model["V"])
    return new_state, {"ent": ent, "am": am, "gap": gap, "canvas": recs,
                       "extras": extras}


def decode(model, prefix, state, sched, inv_temp=None, keep_extras=False):
    """Run denoise steps until every canvas is done (at most max_steps each).

    Returns (final_state, list of per-step records)."""
    records = []
    st = state
    while not bool(np.all(st["done"])):
        st_before = st
        st, rec = denoise_step(model, prefix, st, sched, inv_temp)
        if not keep_extras:
            rec.pop("extras")
        rec["state_before"] = st_before
        records.append(rec)
        if len(records) > sched["max_steps"]:
            raise RuntimeError("decode did not stop within max_steps")
    return st, records
