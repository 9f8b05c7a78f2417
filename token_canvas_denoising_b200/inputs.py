"""Seeded synthetic inputs for the canvas denoise path.

This module only draws numbers: weights, prompt-prefix K/V, per-position
inverse temperatures and canvas seeds. It holds none of the method's
arithmetic, so both the CUDA path (tests, bench, smoke) and the fp64 oracle can
be fed from it without sharing computation.

Workloads follow the five synthetic configurations of the method's hot path
(no trained weights or prompts exist here, so these stand in for them):

  tiny       B1 C16  S32     d64   Hq2/Hk1  h32  V512     f32   T=8
  canvas256  B1 C256 S1024   d2048 Hq16/Hk8 h128 V32768   bf16  T=48
  vocab262k  B1 C256 S4096   d2816 Hq16/Hk8 h128 V262144  bf16  T=48, invT log-uniform [1/5, 1/0.05]
  longctx    B4 C256 S32768  d2816 Hq16/Hk8 h128 V262144  bf16  T=48, prefix scale U[0.5, 2] per (request, head)
  moe        vocab262k + MoE 128 experts + 1 shared, top-8, GeGLU intermediate 704
  *_fp8      vocab262k / longctx with the LM head stored as e4m3 codes and
             power-of-two row scales (the FP8 deployment the pages report);
             moe_fp8 also stores the expert weights that way

Weights are N(0, std) with std = 1/sqrt(fan_in), fan_in being the contraction
dimension of the matrix; the embedding table uses std 1 (a one-hot lookup reads
one input). Prefix K/V are N(0, 1). Every tensor has its own Philox stream
(numpy's Philox-4x64 keyed on (weight seed, tensor id)); bf16 tensors are drawn
in float32 and rounded once to bf16 (round to nearest even) and are returned as
uint16 bit patterns.
"""
from dataclasses import dataclass, field, replace
import math

import numpy as np

# tensor ids of the per-tensor Philox streams
_TID = {"embed": 1, "wq": 2, "wk": 3, "wv": 4, "wo": 5, "lm_head": 6,
        "prefix_scale": 100, "inv_temp": 101, "w_router": 200}


@dataclass(frozen=True)
class Config:
    name: str
    B: int
    C: int
    S: tuple            # prefix length per request
    d: int
    Hq: int
    Hk: int
    h: int
    V: int
    dtype: str          # "f32" or "bf16"
    max_steps: int
    weight_seed: int
    canvas_seeds: tuple
    inv_temp: str = "one"          # "one" or "loguniform"
    prefix_scale: bool = False     # per (request, kv head) scale U[0.5, 2]
    n_experts: int = 0
    top_k: int = 0
    moe_inter: int = 0
    n_shared: int = 0
    stop_entropy: float = 0.05
    lm_fp8: bool = False           # LM head stored as e4m3 codes with power-of-two row scales
    n_layers: int = 0              # 0: one layer, unstacked arrays; L >= 1: L layers stacked [L][...]
    moe_fp8: bool = False          # expert weights stored as e4m3 codes with power-of-two row scales

    @property
    def M(self):
        return self.B * self.C


def _seeds(n, B):
    return tuple(n * 100 + b for b in range(B))


CONFIGS = {
    "tiny": Config("tiny", 1, 16, (32,), 64, 2, 1, 32, 512, "f32", 8, 1001, (0,)),
    "canvas256": Config("canvas256", 1, 256, (1024,), 2048, 16, 8, 128, 32768, "bf16",
                        48, 1002, _seeds(2, 1)),
    "vocab262k": Config("vocab262k", 1, 256, (4096,), 2816, 16, 8, 128, 262144, "bf16",
                        48, 1003, _seeds(3, 1), inv_temp="loguniform"),
    "longctx": Config("longctx", 4, 256, (32768,) * 4, 2816, 16, 8, 128, 262144, "bf16",
                      48, 1004, _seeds(4, 4), prefix_scale=True),
    "moe": Config("moe", 1, 256, (4096,), 2816, 16, 8, 128, 262144, "bf16", 48, 1005,
                  _seeds(5, 1), inv_temp="loguniform", n_experts=128, top_k=8,
                  moe_inter=704, n_shared=1),
}
CONFIGS["vocab262k_fp8"] = replace(CONFIGS["vocab262k"], name="vocab262k_fp8", lm_fp8=True)
CONFIGS["longctx_fp8"] = replace(CONFIGS["longctx"], name="longctx_fp8", lm_fp8=True)
CONFIGS["moe_fp8"] = replace(CONFIGS["moe"], name="moe_fp8", lm_fp8=True, moe_fp8=True)
CONFIG_ORDER = ["tiny", "canvas256", "vocab262k", "longctx", "moe"]


def derive(cfg, **over):
    """A copy of a configuration with some fields changed (smaller test cases)."""
    if "B" in over and "canvas_seeds" not in over:
        base = cfg.canvas_seeds[0] if cfg.canvas_seeds else 0
        over["canvas_seeds"] = tuple(base + b for b in range(over["B"]))
    if "B" in over and "S" not in over:
        over["S"] = tuple(cfg.S[0] for _ in range(over["B"]))
    return replace(cfg, **over)


def _rng(seed, tid):
    # one 128-bit integer key: numpy reads a list key through float64
    return np.random.Generator(np.random.Philox(key=int(seed) | (int(tid) << 64)))


def f32_to_bf16_bits(x):
    """float32 -> bf16 bit patterns, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    return ((u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)).astype(np.uint16)


def e4m3_rows(w):
    """Rows of a float32 matrix as e4m3 byte codes times power-of-two row
    scales: the scale of a row is 2^ceil(log2(max|row| / 448)) (doubled if
    rounding left it too small), the codes are torch's float8_e4m3fn cast of
    row / scale. Returns (codes uint8, scales float32)."""
    import torch
    amax = np.max(np.abs(w), axis=1).astype(np.float64)
    e = np.where(amax > 0, np.ceil(np.log2(np.maximum(amax, 1e-300) / 448.0)), 0.0)
    e = np.where(amax * np.exp2(-e) > 448.0, e + 1, e)
    scaled = w.astype(np.float64) * np.exp2(-e)[:, None]
    codes = torch.from_numpy(scaled).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    return codes, np.exp2(e).astype(np.float32)


def bf16_bits_to_f32(b):
    return (np.asarray(b, np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal(seed, tid, shape, std, dtype, chunk_rows=8192):
    """N(0, std) tensor of the given shape in storage dtype (uint16 bf16 bits or f32).

    Drawn row-chunk by row-chunk from one Philox stream to bound host memory."""
    rng = _rng(seed, tid)
    shape = tuple(int(s) for s in shape)
    rows = shape[0]
    inner = int(np.prod(shape[1:])) if len(shape) > 1 else 1
    out = np.empty((rows, inner), dtype=np.uint16 if dtype == "bf16" else np.float32)
    for r0 in range(0, rows, chunk_rows):
        r1 = min(rows, r0 + chunk_rows)
        x = rng.standard_normal((r1 - r0, inner), dtype=np.float32)
        x *= np.float32(std)
        out[r0:r1] = f32_to_bf16_bits(x) if dtype == "bf16" else x
    return out.reshape(shape)


@dataclass
class Workload:
    cfg: Config
    weights: dict                  # name -> numpy array (uint16 bf16 bits or float32)
    prefix_k: list                 # per request [S_b, Hk, h]
    prefix_v: list
    inv_temp: np.ndarray           # float32 [B*C]
    seeds: np.ndarray              # uint64 [B]
    extra: dict = field(default_factory=dict)


def make_workload(cfg, weight_overrides=None):
    """Draw every input of a configuration. weight_overrides maps a tensor name
    to an array that replaces the drawn one (used to inject known values)."""
    c = cfg
    dt = c.dtype
    w = {}
    ov = dict(weight_overrides or {})

    def draw(name, shape, std, tid=None):
        if name in ov:
            w[name] = ov.pop(name)
        else:
            w[name] = normal(c.weight_seed, _TID[name] if tid is None else tid, shape, std, dt)

    draw("embed", (c.V, c.d), 1.0)
    layer_shapes = (("wq", (c.Hq * c.h, c.d), 1.0 / math.sqrt(c.d)), ("wk", (c.Hk * c.h, c.d), 1.0 / math.sqrt(c.d)),
                    ("wv", (c.Hk * c.h, c.d), 1.0 / math.sqrt(c.d)),
                    ("wo", (c.d, c.Hq * c.h), 1.0 / math.sqrt(c.Hq * c.h)))
    if c.n_layers:  # layer l > 0 draws from its own streams (tensor id + 1000 l)
        for name, shape, std in layer_shapes:
            if name in ov:
                w[name] = ov.pop(name)
                continue
            w[name] = np.stack([normal(c.weight_seed, _TID[name] + 1000 * l, shape, std, dt)
                                for l in range(c.n_layers)])
    else:
        for name, shape, std in layer_shapes:
            draw(name, shape, std)
    if c.lm_fp8 and "lm_head" not in ov:
        # the same draw as the storage-dtype LM head, stored as e4m3
        w["lm_head"], w["lm_head_scale"] = e4m3_rows(
            normal(c.weight_seed, _TID["lm_head"], (c.V, c.d), 1.0 / math.sqrt(c.d), "f32"))
    else:
        draw("lm_head", (c.V, c.d), 1.0 / math.sqrt(c.d))
    if c.n_experts:
        ne = c.n_experts + c.n_shared
        draw("w_router", (c.n_experts, c.d), 1.0 / math.sqrt(c.d))
        for name, shape, std, base in (
                ("w_gate", (c.moe_inter, c.d), 1.0 / math.sqrt(c.d), 1000),
                ("w_up", (c.moe_inter, c.d), 1.0 / math.sqrt(c.d), 2000),
                ("w_down", (c.d, c.moe_inter), 1.0 / math.sqrt(c.moe_inter), 3000)):
            if name in ov:
                w[name] = ov.pop(name)
                continue
            if c.moe_fp8:  # the same draws, stored as e4m3 codes with row scales
                codes = np.empty((ne,) + shape, dtype=np.uint8)
                sc = np.empty((ne, shape[0]), dtype=np.float32)
                for e in range(ne):
                    codes[e], sc[e] = e4m3_rows(normal(c.weight_seed, base + e, shape, std, "f32"))
                w[name], w[name + "_scale"] = codes, sc
                continue
            arr = np.empty((ne,) + shape, dtype=np.uint16 if dt == "bf16" else np.float32)
            for e in range(ne):
                arr[e] = normal(c.weight_seed, base + e, shape, std, dt)
            w[name] = arr
    if ov:
        raise KeyError(f"unknown weight overrides: {sorted(ov)}")

    scales = None
    if c.prefix_scale:
        scales = _rng(c.weight_seed, _TID["prefix_scale"]).uniform(
            0.5, 2.0, size=(c.B, c.Hk)).astype(np.float32)
    pk, pv = [], []
    for b in range(c.B):
        S = c.S[b]
        for lst, tid in ((pk, 10 + 2 * b), (pv, 11 + 2 * b)):
            per_layer = []
            for l in range(max(1, c.n_layers)):  # [L][S][Hk][h] per request with n_layers
                rng = _rng(c.weight_seed, tid + 1000 * l)
                x = rng.standard_normal((S, c.Hk, c.h), dtype=np.float32)
                if scales is not None:
                    x *= scales[b][None, :, None]
                per_layer.append(f32_to_bf16_bits(x) if dt == "bf16" else x)
            lst.append(np.stack(per_layer) if c.n_layers else per_layer[0])

    if c.inv_temp == "loguniform":
        T = np.exp(_rng(c.weight_seed, _TID["inv_temp"]).uniform(
            math.log(0.05), math.log(5.0), size=c.B * c.C))
        inv_temp = (1.0 / T).astype(np.float32)
    else:
        inv_temp = np.ones(c.B * c.C, dtype=np.float32)
    seeds = np.array(c.canvas_seeds, dtype=np.uint64)
    return Workload(c, w, pk, pv, inv_temp, seeds,
                    {"prefix_scale": scales})
