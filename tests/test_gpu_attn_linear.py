"""Kernel-level parity of the tcgen05 attention (dg_attention) and projection
GEMM (dg_linear) against the fp64 oracle on the same seeded bf16 inputs.

Attention cases: ragged canvas lengths (partial 128-query and 128-key tiles),
ragged and empty prompt prefixes, more than 8 requests (several launches),
split-KV (few work items) and unsplit (many work items), a 32K prefix.
Tolerance: |gpu - ref| <= 1e-2 + 2e-2 |ref| element-wise."""
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from oracle import model as om
from oracle import numerics as on
from token_canvas_denoising_b200 import inputs as fx
from tests.parity import close

pytestmark = pytest.mark.gpu


def _dev(bits):
    from token_canvas_denoising_b200.canvas import to_device
    return to_device(bits, "bf16", "cuda")


def _bf(x):
    return on.bf16_bits_to_f64(x)


@pytest.mark.parametrize("B,C,S,Hq,Hk", [
    (1, 256, (1024,), 16, 8),           # canvas256 shape (split-KV)
    (2, 200, (300, 0), 4, 2),           # ragged canvas, empty prefix
    (3, 77, (1, 129, 256), 2, 1),       # ragged everything, MQA
    (9, 128, tuple(64 * (i + 1) for i in range(9)), 2, 2),  # > 8 requests, MHA
    (2, 256, (32768, 5000), 4, 2),      # long prefix
])
def test_attention_matches_oracle(B, C, S, Hq, Hk):
    from token_canvas_denoising_b200 import ops
    h = 128
    seed = 100 + B * 7 + C
    q = fx.normal(seed, 1, (B * C, Hq * h), 1.0, "bf16")
    kc = fx.normal(seed, 2, (B * C, Hk * h), 1.0, "bf16")
    vc = fx.normal(seed, 3, (B * C, Hk * h), 1.0, "bf16")
    pk = [fx.normal(seed, 10 + b, (S[b], Hk, h), 1.0, "bf16") for b in range(B)]
    pv = [fx.normal(seed, 30 + b, (S[b], Hk, h), 1.0, "bf16") for b in range(B)]
    o = ops.attention(_dev(q), _dev(kc), _dev(vc), [_dev(x) for x in pk], [_dev(x) for x in pv],
                      B, C, Hq, Hk, h)
    o = o.float().cpu().numpy().astype(np.float64)
    model = {"dtype": "bf16", "d": Hq * h, "Hq": Hq, "Hk": Hk, "h": h, "V": 2}
    ref = om.attention(model, _bf(q).reshape(-1, Hq, h), _bf(kc).reshape(-1, Hk, h),
                       _bf(vc).reshape(-1, Hk, h), list(zip(pk, pv)), B, C)
    n, mx = close(o, ref)
    assert n == 0, f"{n} elements out of tolerance, max abs diff {mx:.3g}"


@pytest.mark.parametrize("B,C,S,Hq,Hk,growth", [
    (1, 128, (1024,), 2, 1, 0.6),    # one work item per head: long walk over growing tiles
    (4, 256, (2048,) * 4, 16, 8, 0.3),
])
def test_attention_growing_scores_rescale(B, C, S, Hq, Hk, growth):
    """Prefix keys scaled by 1 + growth * (tile index): the scores grow along
    the sequence, so the running maximum is raised in the middle of the walk,
    in some query rows of a warp and not in others (the lazy rescale of O)."""
    from token_canvas_denoising_b200 import ops
    h = 128
    seed = 300 + B + C
    q = fx.normal(seed, 1, (B * C, Hq * h), 1.0, "bf16")
    kc = fx.normal(seed, 2, (B * C, Hk * h), 1.0, "bf16")
    vc = fx.normal(seed, 3, (B * C, Hk * h), 1.0, "bf16")
    pk, pv = [], []
    for b in range(B):
        k0 = _bf(fx.normal(seed, 10 + b, (S[b], Hk, h), 1.0, "bf16"))
        scale = 1.0 + growth * (np.arange(S[b]) // 128)
        pk.append(fx.f32_to_bf16_bits((k0 * scale[:, None, None]).astype(np.float32)))
        pv.append(fx.normal(seed, 30 + b, (S[b], Hk, h), 1.0, "bf16"))
    o = ops.attention(_dev(q), _dev(kc), _dev(vc), [_dev(x) for x in pk], [_dev(x) for x in pv],
                      B, C, Hq, Hk, h)
    o = o.float().cpu().numpy().astype(np.float64)
    model = {"dtype": "bf16", "d": Hq * h, "Hq": Hq, "Hk": Hk, "h": h, "V": 2}
    ref = om.attention(model, _bf(q).reshape(-1, Hq, h), _bf(kc).reshape(-1, Hk, h),
                       _bf(vc).reshape(-1, Hk, h), list(zip(pk, pv)), B, C)
    n, mx = close(o, ref)
    assert n == 0, f"{n} elements out of tolerance, max abs diff {mx:.3g}"


def test_attention_zero_queries_average_values():
    """Q = 0 makes every score 0: each output row is the mean of all S + C value rows."""
    from token_canvas_denoising_b200 import ops
    B, C, S, Hq, Hk, h = 1, 130, (500,), 2, 1, 128
    q = np.zeros((B * C, Hq * h), np.uint16)
    kc = fx.normal(5, 2, (B * C, Hk * h), 1.0, "bf16")
    vc = fx.normal(5, 3, (B * C, Hk * h), 1.0, "bf16")
    pk = [fx.normal(5, 4, (S[0], Hk, h), 1.0, "bf16")]
    pv = [fx.normal(5, 5, (S[0], Hk, h), 1.0, "bf16")]
    o = ops.attention(_dev(q), _dev(kc), _dev(vc), [_dev(pk[0])], [_dev(pv[0])], B, C, Hq, Hk, h)
    o = o.float().cpu().numpy().reshape(C, Hq, h)
    mean = np.concatenate([_bf(pv[0]).reshape(-1, h), _bf(vc)]).mean(axis=0)
    for qh in range(Hq):
        assert np.allclose(o[:, qh], mean[None, :], rtol=2e-2, atol=1e-2)


@pytest.mark.parametrize("M,N,K,res", [(1, 64, 64, False), (200, 192, 256, True), (256, 4096, 2048, False),
                                       (300, 128, 2816, True), (1024, 256, 128, True)])
def test_linear_matches_oracle(M, N, K, res):
    from token_canvas_denoising_b200 import ops
    a = fx.normal(M + N, 1, (M, K), 1.0, "bf16")
    w = fx.normal(M + N, 2, (N, K), 1.0 / math.sqrt(K), "bf16")
    r = fx.normal(M + N, 3, (M, N), 1.0, "bf16") if res else None
    out = ops.linear(_dev(a), _dev(w), _dev(r) if res else None).float().cpu().numpy()
    ref = _bf(a) @ _bf(w).T + (_bf(r) if res else 0.0)
    ref = on.round_to_bf16(ref)
    n, mx = close(out, ref)
    assert n == 0, f"{n} elements out of tolerance, max abs diff {mx:.3g}"
    # f32 accumulation differs from fp64 only in rounding: almost every element
    # rounds to the same bf16 value
    assert np.mean(out == ref) > 0.99
