"""GPU parity of the whole denoise path against the fp64 oracle, through the C ABI.

Small cases run the full decode in free-running mode (bit-exact until the
first ambiguous decision, lock-step after it). Shapes span several tiles of
every kernel and ragged tails (prefix lengths and canvas lengths that are not
tile multiples).
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from oracle import model as om
from token_canvas_denoising_b200 import inputs as fx
from tests.oracle_adapter import oracle_model, oracle_prefix, oracle_sched
from tests.parity import run_lockstep

pytestmark = pytest.mark.gpu


def _canvas(wl):
    from token_canvas_denoising_b200.canvas import from_workload
    return from_workload(wl)


def _run(cfg, adaptive=True, n_steps=None, free_running=True, check_tensors=True, wl=None):
    from token_canvas_denoising_b200.canvas import schedule
    wl = wl or fx.make_workload(cfg)
    cv, keep = _canvas(wl)
    try:
        invT = None if cfg.inv_temp == "one" else wl.inv_temp.astype(np.float64)
        rep, steps = run_lockstep(cfg, cv, oracle_model(wl), oracle_prefix(wl),
                                  oracle_sched(cfg, adaptive=adaptive),
                                  schedule(cfg.max_steps, cfg.stop_entropy, adaptive), invT,
                                  n_steps=n_steps, free_running=free_running,
                                  check_tensors=check_tensors)
    finally:
        cv.close()
    print(f"{cfg.name}: {steps} steps; {rep.summary()}")
    assert not rep.errors, "\n".join(rep.errors[:20])
    return rep, steps


@pytest.mark.parametrize("adaptive", [True, False])
def test_tiny_f32_full_decode(adaptive):
    rep, steps = _run(fx.CONFIGS["tiny"], adaptive=adaptive)
    assert 1 <= steps <= 8


def test_f32_ragged_multi_request():
    cfg = fx.Config("f32_ragged", B=3, C=37, S=(0, 45, 130), d=96, Hq=4, Hk=2, h=64, V=1000,
                    dtype="f32", max_steps=6, weight_seed=9, canvas_seeds=(5, 6, 7))
    _run(cfg)


def test_bf16_small_multi_tile():
    cfg = fx.Config("bf16_small", B=2, C=200, S=(300, 77), d=256, Hq=4, Hk=2, h=128, V=4096,
                    dtype="bf16", max_steps=12, weight_seed=13, canvas_seeds=(21, 22))
    _run(cfg, n_steps=4)


def test_bf16_canvas256_first_steps_lockstep():
    """The canvas256 workload (B1 C256 S1024 d2048 16/8 heads, V32768): the
    first steps in lock-step (the GPU restarts every step from the oracle's
    state) against the oracle."""
    _run(fx.CONFIGS["canvas256"], n_steps=3, free_running=False)


@pytest.mark.parametrize("dtype,B,C", [("bf16", 2, 512), ("bf16", 1, 1000), ("f32", 1, 1024)])
def test_long_canvas_full_decode(dtype, B, C):
    """Canvases longer than the pages' 256 positions (512 and 1024 are the
    lengths raised as an open question: "DiffusionGemma深度拆解", 局限 2): the
    selection sorts up to 1024 keys per canvas; full free-running decode,
    ragged (1000 = 7 tiles of 128 + 104) and exact tile multiples."""
    if dtype == "bf16":
        cfg = fx.Config(f"long_canvas_{C}", B=B, C=C, S=tuple([200, 0][:B]), d=128, Hq=2, Hk=1, h=128, V=2048,
                        dtype="bf16", max_steps=16, weight_seed=51, canvas_seeds=tuple(8 + b for b in range(B)))
    else:
        cfg = fx.Config(f"long_canvas_f32_{C}", B=B, C=C, S=(40,), d=64, Hq=2, Hk=1, h=32, V=512, dtype="f32",
                        max_steps=12, weight_seed=52, canvas_seeds=(3,))
    _, steps = _run(cfg)
    assert 1 <= steps <= cfg.max_steps


@pytest.mark.parametrize("dtype,L", [("bf16", 3), ("f32", 2)])
def test_layer_stack_full_decode(dtype, L):
    """A stack of attention layers, each over its own prompt K/V
    ("DiffusionGemma深度拆解", 局限 2 and 架构解剖 1): every inner layer's output and
    the last layer's stages against the oracle fed the GPU's inputs, full
    free-running decode."""
    if dtype == "bf16":
        cfg = fx.Config("layers_bf16", B=2, C=150, S=(100, 40), d=128, Hq=2, Hk=1, h=128, V=2048, dtype="bf16",
                        max_steps=10, weight_seed=81, canvas_seeds=(4, 5), n_layers=L)
    else:
        cfg = fx.Config("layers_f32", B=2, C=24, S=(10, 33), d=64, Hq=2, Hk=1, h=32, V=300, dtype="f32",
                        max_steps=7, weight_seed=82, canvas_seeds=(1, 2), n_layers=L)
    _, steps = _run(cfg)
    assert 1 <= steps <= cfg.max_steps


def test_block_kv_needs_the_single_layer_model():
    from token_canvas_denoising_b200 import _lib as L
    cfg = fx.Config("layers_kv", B=1, C=16, S=(8,), d=64, Hq=2, Hk=1, h=32, V=64, dtype="f32", max_steps=4,
                    weight_seed=83, canvas_seeds=(1,), n_layers=2)
    cv, keep = _canvas(fx.make_workload(cfg))
    try:
        with pytest.raises(L.DgError) as e:
            cv.block_kv()
        assert e.value.status == L.DG_ERR_UNSUPPORTED
    finally:
        cv.close()


def test_bf16_moe_small_full_decode():
    """MoE FFN path (router, top-k routing, GeGLU experts, shared expert,
    combine) on a small model, full decode."""
    cfg = fx.Config("moe_small", B=1, C=96, S=(150,), d=256, Hq=2, Hk=1, h=128, V=2048, dtype="bf16",
                    max_steps=8, weight_seed=17, canvas_seeds=(5,), n_experts=32, top_k=4, moe_inter=128,
                    n_shared=1)
    _run(cfg)


def test_bf16_moe_uneven_experts():
    """Many experts per token and few tokens: several experts get no token,
    others several tiles of tokens; I not a multiple of 128."""
    cfg = fx.Config("moe_uneven", B=2, C=40, S=(64, 0), d=192, Hq=2, Hk=2, h=128, V=1024, dtype="bf16",
                    max_steps=6, weight_seed=23, canvas_seeds=(1, 2), n_experts=64, top_k=8, moe_inter=192,
                    n_shared=1)
    _run(cfg, n_steps=3)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_fixed_positions_full_decode(dtype):
    """Infilling: a given prefix and suffix of each canvas (and one given cell
    in the middle of the second) stay fixed while the rest is decoded; full
    decode against the oracle started from the same given positions."""
    from token_canvas_denoising_b200.canvas import schedule
    if dtype == "f32":
        cfg = fx.Config("fixed_f32", B=2, C=24, S=(10, 33), d=64, Hq=2, Hk=1, h=32, V=300, dtype="f32",
                        max_steps=7, weight_seed=3, canvas_seeds=(1, 2))
    else:
        cfg = fx.Config("fixed_bf16", B=2, C=130, S=(100, 40), d=128, Hq=2, Hk=1, h=128, V=1024,
                        dtype="bf16", max_steps=12, weight_seed=31, canvas_seeds=(4, 5))
    wl = fx.make_workload(cfg)
    mask = np.zeros((cfg.B, cfg.C), bool)
    mask[:, :cfg.C // 5] = True
    mask[:, cfg.C - cfg.C // 6:] = True
    mask[1, cfg.C // 2] = True
    toks = np.random.default_rng(7).integers(0, cfg.V, size=(cfg.B, cfg.C))
    cv, keep = _canvas(wl)
    try:
        cv.reset(fixed_mask=mask, fixed_tokens=toks)
        ost = om.init_state_fixed(wl.seeds, cfg.C, cfg.V, mask, toks)
        rep, steps = run_lockstep(cfg, cv, oracle_model(wl), oracle_prefix(wl), oracle_sched(cfg, adaptive=True),
                                  schedule(cfg.max_steps, cfg.stop_entropy, True), None, init=ost)
        final = cv.get_state()
    finally:
        cv.close()
    assert not rep.errors, "\n".join(rep.errors[:20])
    assert np.array_equal(final["tokens"].reshape(cfg.B, cfg.C)[mask], toks[mask])
    assert np.all(final["done"])


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_two_blocks_in_sequence(dtype):
    """Block-autoregressive decoding: block 1 is decoded and committed, its K/V
    (dg_canvas_block_kv, checked against the oracle) are appended to each
    request's prompt cache (dg_canvas_set_prefix), and block 2 is decoded over
    prompt + block 1 against the oracle doing the same."""
    from token_canvas_denoising_b200.canvas import schedule
    from tests.parity import close, oracle_state_to_abi
    if dtype == "f32":
        cfg = fx.Config("blocks_f32", B=2, C=24, S=(10, 33), d=64, Hq=2, Hk=1, h=32, V=300, dtype="f32",
                        max_steps=7, weight_seed=3, canvas_seeds=(1, 2))
    else:
        cfg = fx.Config("blocks_bf16", B=2, C=130, S=(100, 0), d=128, Hq=2, Hk=1, h=128, V=1024,
                        dtype="bf16", max_steps=8, weight_seed=37, canvas_seeds=(6, 7))
    wl = fx.make_workload(cfg)
    m, pre = oracle_model(wl), oracle_prefix(wl)
    sched, osched = schedule(cfg.max_steps, cfg.stop_entropy, True), oracle_sched(cfg, adaptive=True)
    cv, keep = _canvas(wl)
    try:
        rep1, _ = run_lockstep(cfg, cv, m, pre, osched, sched, None)
        assert not rep1.errors, "\n".join(rep1.errors[:20])
        ost = rep1.final_state
        cv.set_state(oracle_state_to_abi(ost))  # both sides commit the same tokens
        K, V = cv.block_kv()
        Ko, Vo = om.block_kv(m, ost["tok"])
        for g, o in ((K, Ko), (V, Vo)):
            n, mx = close(g.float().cpu().numpy(), o.reshape(cfg.B * cfg.C, -1))
            assert n == 0, f"block K/V: {n} elements out of tolerance (max abs diff {mx:.3g})"
        kv = (cfg.Hk, cfg.h)
        new_pk = [torch.cat([keep["prefix_k"][b].reshape(-1, *kv),
                             K[b * cfg.C:(b + 1) * cfg.C].reshape(cfg.C, *kv)]).contiguous() for b in range(cfg.B)]
        new_pv = [torch.cat([keep["prefix_v"][b].reshape(-1, *kv),
                             V[b * cfg.C:(b + 1) * cfg.C].reshape(cfg.C, *kv)]).contiguous() for b in range(cfg.B)]
        cv.set_prefix(new_pk, new_pv)
        seeds2 = tuple(s + 100 for s in cfg.canvas_seeds)
        cv.reset(seeds=seeds2)
        cfg2 = fx.derive(cfg, canvas_seeds=seeds2, S=tuple(s + cfg.C for s in cfg.S))
        rep2, steps2 = run_lockstep(cfg2, cv, m, om.append_block(m, pre, Ko, Vo), osched, sched, None)
        assert not rep2.errors, "\n".join(rep2.errors[:20])
        assert 1 <= steps2 <= cfg.max_steps
    finally:
        cv.close()


def test_decode_block_matches_stepping():
    """dg_decode_block (device loop) ends in the same state as single steps."""
    from token_canvas_denoising_b200.canvas import from_workload, schedule
    cfg = fx.Config("loop", B=2, C=24, S=(10, 33), d=64, Hq=2, Hk=1, h=32, V=300, dtype="f32",
                    max_steps=7, weight_seed=3, canvas_seeds=(1, 2))
    wl = fx.make_workload(cfg)
    s = schedule(cfg.max_steps, cfg.stop_entropy, True)
    a, _ = from_workload(wl)
    b, _ = from_workload(wl)
    try:
        toks, steps = a.decode(s)
        while not np.all(b.get_state()["done"]):
            b.step(s)
        sb = b.get_state()
        assert np.array_equal(toks.numpy(), sb["tokens"])
        assert steps == sb["step"].tolist()
        assert all(1 <= x <= cfg.max_steps for x in steps)
    finally:
        a.close()
        b.close()


def test_state_roundtrip_resumes_bit_exactly():
    from token_canvas_denoising_b200.canvas import from_workload, schedule
    cfg = fx.Config("resume", B=1, C=40, S=(20,), d=64, Hq=2, Hk=1, h=32, V=256, dtype="f32",
                    max_steps=8, weight_seed=4, canvas_seeds=(11,))
    wl = fx.make_workload(cfg)
    s = schedule(cfg.max_steps, cfg.stop_entropy, False)
    a, _ = from_workload(wl)
    b, _ = from_workload(wl)
    try:
        for _ in range(3):
            a.step(s)
        mid = a.get_state()
        b.set_state(mid)
        for _ in range(2):
            a.step(s)
            b.step(s)
        sa, sb = a.get_state(), b.get_state()
        for k in sa:
            assert np.array_equal(sa[k], sb[k]), k
    finally:
        a.close()
        b.close()
