"""Pins of the fp64 oracle against what the pages and mathematics fix.

Each test checks the oracle against something other than itself: a library
routine (numpy's Philox, torch's bf16 cast and SDPA, scipy's entropy and erf),
a closed form, an invariant, or brute force on tiny inputs. The planted-mistake
tests at the end change one detail of the oracle (on the CPU) and check that a
pin catches it.
"""
import itertools
import math

import numpy as np
import pytest
import torch

from oracle import model as om
from oracle import numerics as on
from oracle import philox as op
from token_canvas_denoising_b200 import inputs as fx
from tests.oracle_adapter import oracle_init, oracle_model, oracle_prefix, oracle_sched

GOLDEN = __import__("os").path.join(__import__("os").path.dirname(__file__), "golden")


# ---------------------------------------------------------------- Philox
def _numpy_philox_block(counter, key):
    """numpy's Philox increments its 256-bit counter before each block, so set it
    to counter - 1 and read one block of four raw words."""
    c = sum(int(x) << (64 * i) for i, x in enumerate(counter))
    c = (c - 1) % (1 << 256)
    words = [(c >> (64 * i)) & op.MASK64 for i in range(4)]
    bg = np.random.Philox(key=int(key[0]) | (int(key[1]) << 64))
    st = bg.state
    st["state"]["counter"] = np.array(words, dtype=np.uint64)
    st["buffer_pos"] = 4
    bg.state = st
    return [int(x) for x in bg.random_raw(4)]


@pytest.mark.parametrize("counter,key", [
    ((0, 0, 0, 0), (0, 0)),
    ((1, 0, 0, 0), (5, 7)),
    ((255, 47, 3, 0), (1004 * 100 + 3, 0)),
    ((2**64 - 1, 2**63 + 5, 17, 0), (0xDEADBEEFCAFEF00D, 0)),
    ((12345, 1, 0, 0), (2**64 - 1, 2**64 - 1)),
])
def test_philox_matches_numpy(counter, key):
    assert list(op.philox4x64_10(counter, key)) == _numpy_philox_block(counter, key)


def test_canvas_draw_range_and_uniformity():
    V = 16
    n = 16000
    counts = np.zeros(V)
    for p in range(n):
        t = op.canvas_draw(seed=7, step=p // 256, position=p % 256, canvas=0, vocab=V)
        assert 0 <= t < V
        counts[t] += 1
    chi2 = float(np.sum((counts - n / V) ** 2 / (n / V)))
    assert chi2 < 40.0  # 15 dof; p ~ 5e-4 tail


def test_token_from_word_multiply_shift():
    # exact for powers of two: the id is the top log2(V) bits of the word
    for V in (2, 512, 32768, 262144):
        bits = int(math.log2(V))
        for w in (0, 2**64 - 1, 0x8000000000000000, 0x123456789ABCDEF0):
            assert op.token_from_word(w, V) == w >> (64 - bits)


# ---------------------------------------------------------------- bf16 rounding
def test_bf16_rounding_matches_torch_on_f32_values():
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(100000) * np.exp(rng.uniform(-20, 20, 100000))).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    got = on.round_to_bf16(x.astype(np.float64))
    assert np.array_equal(ref, got)


def test_bf16_rounding_ties_and_no_double_rounding():
    one = 1.0
    u = 2.0 ** -7  # bf16 ulp at 1
    assert on.round_to_bf16(np.array([one + u / 2]))[0] == one            # tie -> even
    assert on.round_to_bf16(np.array([one + 3 * u / 2]))[0] == one + 2 * u  # tie -> even
    assert on.round_to_bf16(np.array([-(one + 3 * u / 2)]))[0] == -(one + 2 * u)
    # just above the tie: an fp32 detour would land on the tie and go down
    x = one + u / 2 + 2.0 ** -40
    assert on.round_to_bf16(np.array([x]))[0] == one + u


# ---------------------------------------------------------------- entropy / argmax
def test_entropy_one_hot_is_zero():
    l = np.full((1, 1000), -1000.0)
    l[0, 17] = 0.0
    assert om.entropy_of_logits(l)[0] == 0.0


@pytest.mark.parametrize("V", [2, 7, 512, 32768])
def test_entropy_uniform_is_ln_v(V):
    l = np.full((3, V), 0.25)
    assert np.allclose(om.entropy_of_logits(l), math.log(V), rtol=0, atol=1e-12)


def test_entropy_two_way_closed_form():
    for x in np.linspace(-8, 8, 33):
        s = 1.0 / (1.0 + math.exp(-x))
        expect = -(s * math.log(s) + (1 - s) * math.log(1 - s))
        got = om.entropy_of_logits(np.array([[x, 0.0]]))[0]
        assert abs(got - expect) < 1e-12


def test_entropy_matches_scipy_with_temperature():
    from scipy.stats import entropy
    rng = np.random.default_rng(1)
    l = rng.standard_normal((6, 4096))
    invT = np.array([1 / 0.05, 1 / 5.0, 1.0, 2.0, 0.5, 7.0])
    ent, am, gap = om.entropy_argmax(l, invT)
    for i in range(6):
        z = l[i] * invT[i]
        p = np.exp(z - z.max())
        p /= p.sum()
        assert abs(ent[i] - entropy(p)) < 1e-10
        assert am[i] == int(np.argmax(l[i]))
    # argmax ignores the temperature and takes the lowest index on ties
    t = np.zeros((1, 10))
    t[0, [3, 6]] = 2.0
    assert om.entropy_argmax(t, np.array([3.0]))[1][0] == 3


# ---------------------------------------------------------------- attention
def _tiny_cfg(**kw):
    base = dict(name="t", B=2, C=6, S=(5, 3), d=16, Hq=4, Hk=2, h=8, V=32, dtype="f32",
                max_steps=6, weight_seed=77, canvas_seeds=(3, 4))
    base.update(kw)
    return fx.Config(**base)


def _sdpa_reference(Q, Kall, Vall, Hq, Hk):
    """torch SDPA (fp64, non-causal) with KV heads expanded for GQA."""
    q = torch.from_numpy(Q).permute(1, 0, 2)[None]            # [1, Hq, C, h]
    k = torch.from_numpy(Kall).permute(1, 0, 2)[None]
    v = torch.from_numpy(Vall).permute(1, 0, 2)[None]
    rep = Hq // Hk
    k = k.repeat_interleave(rep, dim=1)
    v = v.repeat_interleave(rep, dim=1)
    o = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=False)
    return o[0].permute(1, 0, 2).numpy()


@pytest.mark.parametrize("Hq,Hk", [(4, 2), (4, 4), (4, 1)])  # GQA, MHA, MQA
def test_attention_matches_torch_sdpa(Hq, Hk):
    cfg = _tiny_cfg(Hq=Hq, Hk=Hk)
    wl = fx.make_workload(cfg)
    m = oracle_model(wl)
    rng = np.random.default_rng(2)
    M = cfg.B * cfg.C
    Q = rng.standard_normal((M, Hq, cfg.h))
    Kc = rng.standard_normal((M, Hk, cfg.h))
    Vc = rng.standard_normal((M, Hk, cfg.h))
    m32 = dict(m, dtype="f32")
    O = om.attention(m32, Q, Kc, Vc, oracle_prefix(wl), cfg.B, cfg.C).reshape(M, Hq, cfg.h)
    for b in range(cfg.B):
        Kall = np.concatenate([wl.prefix_k[b].astype(np.float64), Kc[b * cfg.C:(b + 1) * cfg.C]])
        Vall = np.concatenate([wl.prefix_v[b].astype(np.float64), Vc[b * cfg.C:(b + 1) * cfg.C]])
        ref = _sdpa_reference(Q[b * cfg.C:(b + 1) * cfg.C], Kall, Vall, Hq, Hk)
        # oracle rounds O to f32 storage; compare at f32 resolution
        assert np.allclose(O[b * cfg.C:(b + 1) * cfg.C], ref, rtol=1e-6, atol=1e-7)


def test_attention_zero_query_is_mean_of_values():
    cfg = _tiny_cfg()
    wl = fx.make_workload(cfg)
    m = oracle_model(wl)
    M = cfg.B * cfg.C
    rng = np.random.default_rng(3)
    Q = np.zeros((M, cfg.Hq, cfg.h))
    Kc = rng.standard_normal((M, cfg.Hk, cfg.h))
    Vc = rng.standard_normal((M, cfg.Hk, cfg.h))
    O = om.attention(m, Q, Kc, Vc, oracle_prefix(wl), cfg.B, cfg.C).reshape(M, cfg.Hq, cfg.h)
    for b in range(cfg.B):
        Vall = np.concatenate([wl.prefix_v[b].astype(np.float64), Vc[b * cfg.C:(b + 1) * cfg.C]])
        for q in range(cfg.Hq):
            g = q // (cfg.Hq // cfg.Hk)
            mean = Vall[:, g, :].mean(axis=0)
            assert np.allclose(O[b * cfg.C:(b + 1) * cfg.C, q], mean, rtol=1e-6, atol=1e-7)


def test_attention_dominant_key_returns_its_value():
    cfg = _tiny_cfg(B=1, S=(5,), canvas_seeds=(1,))
    wl = fx.make_workload(cfg)
    m = oracle_model(wl)
    M = cfg.C
    rng = np.random.default_rng(4)
    u = rng.standard_normal(cfg.h)
    Q = np.tile(u, (M, cfg.Hq, 1))
    Kc = rng.standard_normal((M, cfg.Hk, cfg.h)) * 0.01
    Vc = rng.standard_normal((M, cfg.Hk, cfg.h))
    j = 2  # canvas key 2 of every kv head dominates
    Kc[j] = 100.0 * u
    O = om.attention(m, Q, Kc, Vc, [(np.zeros_like(wl.prefix_k[0]), wl.prefix_v[0])], 1, cfg.C)
    O = O.reshape(M, cfg.Hq, cfg.h)
    for q in range(cfg.Hq):
        g = q // (cfg.Hq // cfg.Hk)
        assert np.allclose(O[:, q], np.tile(Vc[j, g], (M, 1)), rtol=1e-6, atol=1e-6)


def test_forward_permutation_equivariance():
    cfg = _tiny_cfg(B=1, S=(5,), canvas_seeds=(1,), C=7)
    wl = fx.make_workload(cfg)
    m = oracle_model(wl)
    tok = np.array([[3, 9, 1, 30, 9, 0, 12]])
    perm = np.array([4, 0, 6, 2, 1, 5, 3])
    e1, a1, _, x1 = om.forward(m, oracle_prefix(wl), tok, None)
    e2, a2, _, x2 = om.forward(m, oracle_prefix(wl), tok[:, perm], None)
    assert np.allclose(e2[0], e1[0, perm], rtol=0, atol=1e-12)
    assert np.array_equal(a2[0], a1[0, perm])
    assert np.allclose(x2["O"], x1["O"][perm], rtol=0, atol=1e-6)
    assert np.allclose(x2["Hs"], x1["Hs"][perm], rtol=0, atol=1e-6)


# ---------------------------------------------------------------- freeze selection
def test_select_freeze_brute_force():
    rng = np.random.default_rng(5)
    for trial in range(200):
        C = int(rng.integers(1, 9))
        ent = rng.choice([0.1, 0.2, 0.3, 0.7], size=C)  # many exact ties
        frozen = rng.random(C) < 0.3
        unfrozen = [p for p in range(C) if not frozen[p]]
        for k in range(0, len(unfrozen) + 1):
            got = set(np.nonzero(om.select_freeze(ent, frozen, k))[0].tolist())
            # brute force: the unique k-subset whose keys are all below the rest's
            sols = []
            for sub in itertools.combinations(unfrozen, k):
                rest = [p for p in unfrozen if p not in sub]
                if all((ent[a], a) < (ent[b], b) for a in sub for b in rest):
                    sols.append(set(sub))
            assert len(sols) == 1 and got == sols[0]


def test_freeze_schedule_golden():
    """C=256, T=48: 6 per step for 16 steps then 5 per step for 32 (golden file);
    C=16, T=8: 2 per step. Canvas size 256 and the 48-step cap are the pages'."""
    with open(f"{GOLDEN}/freeze_schedule.txt") as f:
        lines = [l.split("#")[0].strip() for l in f]
    rows = [l for l in lines if l]
    for row in rows:
        C, T, counts = row.split(":")
        C, T = int(C), int(T)
        want = [int(x) for x in counts.split(",")]
        got, U = [], C
        for t in range(T):
            k = om.freeze_count(U, t, T)
            got.append(k)
            U -= k
        assert got == want and U == 0


# ---------------------------------------------------------------- whole loop
def _tiny_loop_cfg(V=2, C=4):
    return fx.Config(name="loop", B=1, C=C, S=(3,), d=8, Hq=2, Hk=1, h=4, V=V, dtype="f32",
                     max_steps=3, weight_seed=11, canvas_seeds=(9,))


def _check_trajectory(cfg, st0, final, recs, adaptive):
    T = cfg.max_steps
    assert 1 <= len(recs) <= T
    prev = st0
    for i, rec in enumerate(recs):
        before = rec["state_before"]
        assert np.array_equal(before["tok"], prev["tok"])
        after = recs[i + 1]["state_before"] if i + 1 < len(recs) else final
        r = rec["canvas"][0]
        # frozen positions keep their token and stay frozen
        fb = before["frozen"][0]
        assert np.all(after["frozen"][0][fb])
        assert np.array_equal(after["tok"][0][fb], before["tok"][0][fb])
        # exactly k_t positions freeze, chosen by the (entropy, position) key, with argmax
        assert r["k"] == om.freeze_count(int((~fb).sum()), i, T)
        F = r["freeze"]
        assert F.sum() == r["k"] and not np.any(F & fb)
        assert np.array_equal(after["tok"][0][F], rec["am"][0][F])
        if r["stop"]:
            assert np.all(after["frozen"][0])
            rest = ~(fb | F)
            assert np.array_equal(after["tok"][0][rest], rec["am"][0][rest])
            if rest.any():
                assert adaptive and r["min_rest"] < cfg.stop_entropy
        else:
            for p in np.nonzero(~(fb | F))[0]:
                assert after["tok"][0][p] == op.canvas_draw(int(cfg.canvas_seeds[0]), i + 1,
                                                            int(p), 0, cfg.V)
        prev = after
    assert np.all(final["done"]) and int(final["step"][0]) == len(recs)


@pytest.mark.parametrize("adaptive", [False, True])
def test_whole_loop_all_initial_canvases_v2_c4(adaptive):
    cfg = _tiny_loop_cfg()
    wl = fx.make_workload(cfg)
    m = oracle_model(wl)
    sched = oracle_sched(cfg, adaptive=adaptive)
    for init in itertools.product(range(cfg.V), repeat=cfg.C):
        st0 = oracle_init(wl)
        st0["tok"][0] = np.array(init)
        final, recs = om.decode(m, oracle_prefix(wl), st0, sched)
        _check_trajectory(cfg, st0, final, recs, adaptive)
        if not adaptive:
            assert len(recs) == cfg.max_steps or np.all(final["frozen"])


@pytest.mark.parametrize("V,C", [(4, 5), (8, 6)])
def test_whole_loop_small_vocab(V, C):
    cfg = _tiny_loop_cfg(V=V, C=C)
    wl = fx.make_workload(cfg)
    st0 = oracle_init(wl)
    for b in range(cfg.B):
        for p in range(C):
            assert st0["tok"][b, p] == op.canvas_draw(int(cfg.canvas_seeds[b]), 0, p, b, V)
    final, recs = om.decode(oracle_model(wl), oracle_prefix(wl), st0, oracle_sched(cfg, False))
    _check_trajectory(cfg, st0, final, recs, False)
    assert len(recs) == cfg.max_steps


def test_adaptive_stop_uses_threshold():
    """A near one-hot LM head row drives every entropy far below 0.05, so the
    adaptive stop must end the decode after the first step."""
    cfg = _tiny_loop_cfg(V=8, C=6)
    wl = fx.make_workload(cfg)
    m = oracle_model(wl)
    lm = np.zeros((cfg.V, cfg.d), np.float32)
    lm[5, :] = 1000.0  # logit of token 5 = 1000 * sum(Hs); make sum(Hs) > 0 below
    m["lm_head"] = lm
    m["wo"] = np.zeros_like(m["wo"])
    m["embed"] = np.abs(m["embed"]) + 0.1
    final, recs = om.decode(m, oracle_prefix(wl), oracle_init(wl),
                            oracle_sched(cfg, adaptive=True, max_steps=48))
    assert len(recs) == 1 and np.all(final["tok"] == 5)


# ---------------------------------------------------------------- fixed positions
def test_fixed_positions_empty_mask_is_the_plain_block():
    cfg = _tiny_loop_cfg(V=8, C=6)
    wl = fx.make_workload(cfg)
    a = oracle_init(wl)
    b = om.init_state_fixed(wl.seeds, cfg.C, cfg.V, np.zeros((1, cfg.C), bool), np.zeros((1, cfg.C), int))
    assert np.array_equal(a["tok"], b["tok"]) and not b["frozen"].any()


def test_fixed_positions_keep_tokens_and_only_open_positions_are_scheduled():
    """C = 16, T = 8, 6 positions given: the schedule runs over the 10 open ones,
    k_t = ceil(U / (T - t)) with U = 10, 8, 6, 5, 4, 3, 2, 1 (worked by hand)."""
    cfg = fx.Config(name="fixed", B=1, C=16, S=(3,), d=8, Hq=2, Hk=1, h=4, V=8, dtype="f32",
                    max_steps=8, weight_seed=11, canvas_seeds=(9,))
    wl = fx.make_workload(cfg)
    mask = np.zeros((1, 16), bool)
    mask[0, [0, 1, 2, 13, 14, 15]] = True  # a given prefix and suffix; the middle is filled
    given = np.zeros((1, 16), int)
    given[0, [0, 1, 2, 13, 14, 15]] = [3, 1, 4, 1, 5, 7]
    st0 = om.init_state_fixed(wl.seeds, cfg.C, cfg.V, mask, given)
    final, recs = om.decode(oracle_model(wl), oracle_prefix(wl), st0, oracle_sched(cfg, False))
    _check_trajectory(cfg, st0, final, recs, False)
    assert [int(r["canvas"][0]["freeze"].sum()) for r in recs] == [2, 2, 1, 1, 1, 1, 1, 1]
    assert np.array_equal(final["tok"][mask], given[mask])
    # the open positions were drawn like any other block
    for p in np.nonzero(~mask[0])[0]:
        assert st0["tok"][0, p] == op.canvas_draw(int(cfg.canvas_seeds[0]), 0, int(p), 0, cfg.V)


def test_all_positions_fixed_ends_after_one_step():
    cfg = _tiny_loop_cfg(V=8, C=6)
    wl = fx.make_workload(cfg)
    given = np.array([[7, 6, 5, 4, 3, 2]])
    st0 = om.init_state_fixed(wl.seeds, cfg.C, cfg.V, np.ones((1, cfg.C), bool), given)
    final, recs = om.decode(oracle_model(wl), oracle_prefix(wl), st0, oracle_sched(cfg, False))
    assert len(recs) == 1 and np.array_equal(final["tok"], given) and final["done"].all()


@pytest.mark.parametrize("adaptive", [False, True])
def test_one_fixed_position_all_canvases_v2_c4(adaptive):
    """Every initial canvas of V = 2, C = 4 with position 1 given as either
    token: the trajectory invariants hold and the given token survives."""
    cfg = _tiny_loop_cfg()
    wl = fx.make_workload(cfg)
    m = oracle_model(wl)
    sched = oracle_sched(cfg, adaptive=adaptive)
    mask = np.array([[False, True, False, False]])
    for init in itertools.product(range(cfg.V), repeat=cfg.C):
        st0 = om.init_state_fixed(wl.seeds, cfg.C, cfg.V, mask, np.array([init]))
        st0["tok"][0] = np.array(init)
        final, recs = om.decode(m, oracle_prefix(wl), st0, sched)
        _check_trajectory(cfg, st0, final, recs, adaptive)
        assert final["tok"][0, 1] == init[1]


# ---------------------------------------------------------------- blocks in sequence
def _blk_cfg(dtype="bf16"):
    return fx.Config(name="blk", B=2, C=5, S=(3, 0), d=16, Hq=2, Hk=1, h=8, V=32, dtype=dtype,
                     max_steps=4, weight_seed=2, canvas_seeds=(3, 4))


def test_block_kv_is_the_steps_canvas_kv():
    cfg = _blk_cfg()
    wl = fx.make_workload(cfg)
    m = oracle_model(wl)
    tok = oracle_init(wl)["tok"]
    K, V = om.block_kv(m, tok)
    _, _, _, ex = om.forward(m, oracle_prefix(wl), tok, None)
    assert np.array_equal(K.reshape(ex["Kc"].shape), ex["Kc"])
    assert np.array_equal(V.reshape(ex["Vc"].shape), ex["Vc"])


def test_next_block_attends_to_prompt_then_committed_block():
    """With Wq = 0 every score is 0, so block 2's attention output is the plain
    mean of the request's prompt V rows, its committed block's V rows and its
    own canvas V rows (a wrong tensor, request or order in the append fails)."""
    cfg = _blk_cfg()
    wl = fx.make_workload(cfg)
    m = oracle_model(wl)
    m["wq"] = np.zeros_like(m["wq"])
    st1 = oracle_init(wl)
    K1, V1 = om.block_kv(m, st1["tok"])
    pre2 = om.append_block(m, oracle_prefix(wl), K1, V1)
    tok2 = om.init_state(np.array([7, 8], dtype=np.uint64), cfg.C, cfg.V)["tok"]
    _, _, _, ex = om.forward(m, pre2, tok2, None)
    O = ex["O"].reshape(cfg.B, cfg.C, cfg.Hq, cfg.h)
    _, V2 = om.block_kv(m, tok2)
    for b in range(cfg.B):
        rows = [om.widen(wl.prefix_v[b], cfg.dtype).reshape(-1, cfg.Hk, cfg.h), V1[b], V2[b]]
        mean = np.concatenate(rows).mean(axis=0)[0]
        want = on.round_to_bf16(np.broadcast_to(mean, (cfg.C, cfg.h)))
        for q in range(cfg.Hq):
            assert np.array_equal(O[b, :, q], want)
        assert pre2[b][0].shape[0] == cfg.S[b] + cfg.C


def test_two_blocks_in_sequence_keep_the_invariants():
    cfg = fx.Config(name="two", B=1, C=4, S=(3,), d=8, Hq=2, Hk=1, h=4, V=8, dtype="f32",
                    max_steps=3, weight_seed=11, canvas_seeds=(9,))
    wl = fx.make_workload(cfg)
    m = oracle_model(wl)
    sched = oracle_sched(cfg, False)
    st1 = oracle_init(wl)
    fin1, recs1 = om.decode(m, oracle_prefix(wl), st1, sched)
    _check_trajectory(cfg, st1, fin1, recs1, False)
    K1, V1 = om.block_kv(m, fin1["tok"])
    pre2 = om.append_block(m, oracle_prefix(wl), K1, V1)
    cfg2 = fx.derive(cfg, canvas_seeds=(10,))
    st2 = om.init_state(np.array([10], dtype=np.uint64), cfg.C, cfg.V)
    fin2, recs2 = om.decode(m, pre2, st2, sched)
    _check_trajectory(cfg2, st2, fin2, recs2, False)
    assert pre2[0][0].shape[0] == cfg.S[0] + cfg.C


# ---------------------------------------------------------------- MoE
def _moe_cfg():
    return fx.Config(name="moe_t", B=1, C=5, S=(3,), d=12, Hq=2, Hk=1, h=4, V=16, dtype="f32",
                     max_steps=4, weight_seed=21, canvas_seeds=(1,), n_experts=10, top_k=3,
                     moe_inter=6, n_shared=1)


def test_moe_topk_and_gates():
    cfg = _moe_cfg()
    m = oracle_model(fx.make_workload(cfg))
    Hs = np.eye(5, cfg.d)
    # router rows constructed so token i prefers experts in a known order
    Wr = np.zeros((cfg.n_experts, cfg.d), np.float32)
    order = [7, 2, 9, 0, 5, 1, 3, 4, 6, 8]
    for rank, e in enumerate(order):
        Wr[e, :] = 10.0 - rank
    m["w_router"] = Wr
    r, idx, gates = om.moe_route(m, Hs)
    for i in range(5):
        assert idx[i].tolist() == order[:3]
        assert abs(gates[i].sum() - 1.0) < 1e-15
        e = np.exp(np.array([10.0, 9.0, 8.0]))
        assert np.allclose(gates[i], e / e.sum(), atol=1e-15)
    # ties go to the lower expert index
    m["w_router"] = np.ones((cfg.n_experts, cfg.d), np.float32)
    _, idx, gates = om.moe_route(m, Hs)
    assert idx[0].tolist() == [0, 1, 2] and np.allclose(gates[0], 1 / 3)


def test_moe_identical_experts_reduce_to_single_ffn():
    cfg = _moe_cfg()
    wl = fx.make_workload(cfg)
    m = oracle_model(wl)
    for k in ("w_gate", "w_up", "w_down"):
        arr = m[k].copy()
        arr[:] = arr[0]
        m[k] = arr
    Hs = np.random.default_rng(6).standard_normal((5, cfg.d))
    out, _ = om.moe_block(m, Hs)
    g = Hs @ m["w_gate"][0].astype(np.float64).T
    u = Hs @ m["w_up"][0].astype(np.float64).T
    a = on.round_to_f32(torch.nn.functional.gelu(torch.from_numpy(g)).numpy() * u)
    y = a @ m["w_down"][0].astype(np.float64).T
    assert np.allclose(out, on.round_to_f32(Hs + 2.0 * y), rtol=1e-6, atol=1e-6)


def _gate_pairing_model(router_logits):
    """Three routed experts, top-2, no shared expert, d = 4, I = 1, f32 storage.
    The token is the unit vector e_0, so the router logits are column 0 of
    W_router. Every expert has the same gate and up rows (the same scalar
    activation a), and expert e writes only coordinate e + 1, scaled by
    c_e = e + 1: FFN_e(e_0) = a c_e e_{e+1}."""
    E, d = 3, 4
    m = {"dtype": "f32", "d": d, "n_experts": E, "top_k": 2, "moe_inter": 1, "n_shared": 0}
    wr = np.zeros((E, d), np.float32)
    wr[:, 0] = router_logits
    m["w_router"] = wr
    m["w_gate"] = np.zeros((E, 1, d), np.float32)
    m["w_gate"][:, 0, 0] = 1.5
    m["w_up"] = np.zeros((E, 1, d), np.float32)
    m["w_up"][:, 0, 0] = 1.0
    m["w_down"] = np.zeros((E, d, 1), np.float32)
    for e in range(E):
        m["w_down"][e, e + 1, 0] = e + 1.0
    return m


@pytest.mark.parametrize("logits,chosen", [((2.0, 1.0, 0.0), (0, 1)), ((0.0, 1.0, 2.0), (2, 1)),
                                           ((1.0, -3.0, 2.0), (2, 0))])
def test_moe_gate_pairing_with_distinct_experts(logits, chosen):
    """Each expert's output is weighted by its own gate. With router logits
    r_i > r_j for the two chosen experts, the renormalised gates are
    e^(r_i) / (e^(r_i) + e^(r_j)) and e^(r_j) / (...), so the contributions on
    the experts' own coordinates, divided by c_e, stand in the ratio
    e^(r_i - r_j) (for logits 2 and 1: exactly e), sum to the shared activation
    a, and the unchosen expert's coordinate stays 0. Pairing each expert with
    another slot's gate inverts the ratio."""
    m = _gate_pairing_model(logits)
    x = np.zeros((1, 4))
    x[0, 0] = 1.0
    out, (r, idx, gates) = om.moe_block(m, x)
    assert sorted(idx[0].tolist()) == sorted(chosen)
    y = out[0] - x[0]
    contrib = {e: y[e + 1] / (e + 1.0) for e in range(3)}
    i, j = chosen
    assert contrib[i] / contrib[j] == pytest.approx(math.exp(logits[i] - logits[j]), rel=1e-6)
    unchosen = ({0, 1, 2} - set(chosen)).pop()
    assert y[unchosen + 1] == 0.0
    # the two contributions add up to the common activation a = GELU(1.5) * 1
    assert contrib[i] + contrib[j] == pytest.approx(1.5 * 0.5 * (1.0 + math.erf(1.5 / math.sqrt(2.0))), rel=1e-6)


def test_moe_explicit_choice_uses_the_chosen_experts_gates():
    """Routing a row to another valid pair of experts (as the parity harness
    does where the k-th and (k+1)-th router logits are tied within its
    tolerance) renormalises the softmax over that pair."""
    m = _gate_pairing_model((2.0, 1.0, 0.0))
    x = np.zeros((1, 4))
    x[0, 0] = 1.0
    out, (_, idx, gates) = om.moe_block(m, x, choice=[[0, 2]])
    assert idx[0].tolist() == [0, 2]
    assert gates[0] == pytest.approx([math.exp(2) / (math.exp(2) + 1), 1 / (math.exp(2) + 1)], rel=1e-12)
    y = out[0] - x[0]
    assert y[2] == 0.0 and (y[1] / 1.0) / (y[3] / 3.0) == pytest.approx(math.exp(2.0), rel=1e-6)


def test_planted_swapped_moe_gates_are_caught(monkeypatch):
    real = om.moe_route

    def swapped(model, Hs, choice=None):
        r, idx, gates = real(model, Hs, choice)
        return r, idx, gates[:, ::-1].copy()
    monkeypatch.setattr(om, "moe_route", swapped)
    with pytest.raises(AssertionError):
        test_moe_gate_pairing_with_distinct_experts((2.0, 1.0, 0.0), (0, 1))


def test_gelu_matches_torch_exact():
    x = np.linspace(-6, 6, 101)
    ref = torch.nn.functional.gelu(torch.from_numpy(x), approximate="none").numpy()
    assert np.allclose(om.gelu_exact(x), ref, rtol=0, atol=1e-14)


# ---------------------------------------------------------------- planted mistakes
def test_planted_wrong_gqa_map_is_caught(monkeypatch):
    monkeypatch.setattr(om, "kv_head_of", lambda q, Hq, Hk: q % Hk)
    with pytest.raises(AssertionError):
        test_attention_matches_torch_sdpa(4, 2)


def test_planted_missing_scale_is_caught(monkeypatch):
    orig = om.softmax_rows
    monkeypatch.setattr(om, "softmax_rows", lambda s: orig(s * math.sqrt(8.0)))
    with pytest.raises(AssertionError):
        test_attention_matches_torch_sdpa(4, 2)


def test_planted_wrong_entropy_sign_is_caught(monkeypatch):
    orig = om.entropy_of_logits
    monkeypatch.setattr(om, "entropy_of_logits", lambda l: -orig(l))
    with pytest.raises(AssertionError):
        test_entropy_matches_scipy_with_temperature()


def test_planted_off_by_one_schedule_is_caught(monkeypatch):
    monkeypatch.setattr(om, "freeze_count",
                        lambda U, t, T: U if T - t <= 0 else -(-U // (T - t + 1)))
    with pytest.raises(AssertionError):
        test_freeze_schedule_golden()


def test_planted_renoise_step_is_caught(monkeypatch):
    orig = om.canvas_draw
    monkeypatch.setattr(om, "canvas_draw", lambda s, t, p, b, V: orig(s, t + 1, p, b, V))
    with pytest.raises(AssertionError):
        test_whole_loop_small_vocab(4, 5)


# ---------------------------------------------------------------- FP8 (e4m3) LM head
def test_e4m3_decode_matches_torch_for_every_code():
    codes = np.arange(256, dtype=np.uint8)
    a = on.e4m3_to_f64(codes)
    b = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(np.isnan(a), np.isnan(b)) and np.isnan(a).sum() == 2
    assert np.array_equal(a[~np.isnan(a)], b[~np.isnan(b)])
    assert np.nanmax(a) == 448.0 and a[1] == 2.0 ** -9


def test_e4m3_rounding_matches_torch_cast():
    """Round to nearest, ties to even, against torch's float8_e4m3fn cast:
    random values over the whole range and every midpoint between adjacent
    values (the ties), including the subnormal range and both signs."""
    rng = np.random.default_rng(5)
    vals = on.e4m3_to_f64(np.arange(0x7F, dtype=np.uint8))
    mids = 0.5 * (vals[1:] + vals[:-1])
    x = np.concatenate([rng.uniform(-448, 448, 20000), np.exp2(rng.uniform(-12, 8.8, 20000)) *
                        rng.choice([-1, 1], 20000), mids, -mids, vals, -vals])
    x = np.clip(x, -448, 448)
    got = on.round_to_e4m3(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, ref)


def test_e4m3_scale_exponent_is_the_smallest_that_fits():
    rng = np.random.default_rng(6)
    amax = np.concatenate([np.exp2(rng.uniform(-20, 20, 5000)), 448.0 * np.exp2(np.arange(-10, 10.0)),
                           448.0 * np.exp2(np.arange(-10, 10.0)) * (1 + 2.0 ** -20), [1.0, 3.0, 449.0]])
    e = on.e4m3_scale_exponent(amax)
    assert np.all(448.0 * np.exp2(e.astype(float)) >= amax)
    assert np.all(448.0 * np.exp2(e.astype(float) - 1) < amax)
    assert on.e4m3_scale_exponent(np.array([0.0]))[0] == 0


def test_e4m3_dot_products_are_exact_in_fp64():
    """Every e4m3 value is n 2^-9 with an integer n, so a dot product of two
    code rows is 2^-18 times an integer sum: the fp64 matmul equals it exactly."""
    rng = np.random.default_rng(7)
    a = rng.integers(0, 256, (3, 2816), dtype=np.uint8)
    w = rng.integers(0, 256, (5, 2816), dtype=np.uint8)
    a[(a & 0x7F) == 0x7F] = 0  # no NaN codes
    w[(w & 0x7F) == 0x7F] = 0
    fa, fw = on.e4m3_to_f64(a), on.e4m3_to_f64(w)
    got = fa @ fw.T
    na = [[int(round(v * 512)) for v in row] for row in fa]
    nw = [[int(round(v * 512)) for v in row] for row in fw]
    for i in range(3):
        for j in range(5):
            assert got[i, j] == sum(x * y for x, y in zip(na[i], nw[j])) * 2.0 ** -18


def test_fp8_lm_head_logits_worked_by_hand():
    """Hs row (1, 0.3): largest magnitude 1 -> scale 2^-8 (448 2^-8 = 1.75 >= 1,
    0.875 < 1); 0.3 * 2^8 = 76.8 lies between the e4m3 values 72 and 80 and
    rounds to 80, i.e. 0.3125. With weight rows (1, 1), (2, -4) at scale 2^0
    and (1.5, 1) at 2^-1 the logits are 1.3125, 0.75, 0.90625.
    Hs row (1, 3 2^-17): the small entry scales to 3 2^-9, the e4m3 subnormal
    with mantissa 3, exactly; through the weight row (0, 1) the logit is
    3 2^-17 (a scale twice as large would give 1.5 2^-9, a tie that rounds
    to 2 2^-9, and the logit 4 2^-17)."""
    w = np.array([[1.0, 1.0], [2.0, -4.0], [1.5, 1.0], [0.0, 1.0]])
    m = {"dtype": "bf16", "lm_head_e4m3": on.round_to_e4m3(w), "lm_head_scale": np.array([1.0, 1.0, 0.5, 1.0])}
    got = om.lm_head_logits(m, np.array([[1.0, 0.3], [1.0, 3 * 2.0 ** -17]]))
    assert got[0].tolist() == [1.3125, 2.0 - 4 * 0.3125, 0.5 * (1.5 + 0.3125), 0.3125]
    assert got[0, 2] == 0.90625
    assert got[1, 3] == 3 * 2.0 ** -17


def test_planted_fp8_scale_off_by_one_is_caught(monkeypatch):
    real = on.e4m3_scale_exponent
    monkeypatch.setattr(on, "e4m3_scale_exponent", lambda amax: real(amax) + 1)
    with pytest.raises(AssertionError):
        test_fp8_lm_head_logits_worked_by_hand()
    with pytest.raises(AssertionError):
        test_e4m3_scale_exponent_is_the_smallest_that_fits()


# ---------------------------------------------------------------- layer stack
def _layers_cfg(L, **kw):
    return fx.Config(name="layers", B=2, C=6, S=(5, 0), d=16, Hq=2, Hk=1, h=8, V=32, dtype="f32", max_steps=4,
                     weight_seed=61, canvas_seeds=(1, 2), n_layers=L, **kw)


def test_one_stacked_layer_equals_the_single_layer_model():
    st = None
    outs = []
    for L in (0, 1):
        wl = fx.make_workload(_layers_cfg(L))
        m, pre = oracle_model(wl), oracle_prefix(wl)
        st = om.init_state(wl.seeds, 6, 32) if st is None else st
        outs.append(om.forward(m, pre, st["tok"], None))
    for a, b in zip(outs[0][:3], outs[1][:3]):
        assert np.array_equal(a, b)


def test_second_layer_with_zero_output_projection_is_the_identity():
    """With Wo = 0 in layer 2 its output equals its input, so the two-layer
    model's entropies equal those of layer 1 alone."""
    wl2 = fx.make_workload(_layers_cfg(2))
    m2, pre2 = oracle_model(wl2), oracle_prefix(wl2)
    m2["wo"] = m2["wo"].copy()
    m2["wo"][1] = 0
    m1 = dict(m2, n_layers=1, wq=m2["wq"][:1], wk=m2["wk"][:1], wv=m2["wv"][:1], wo=m2["wo"][:1])
    pre1 = [(k[:1], v[:1]) for k, v in pre2]
    st = om.init_state(wl2.seeds, 6, 32)
    e2, a2, _, x2 = om.forward(m2, pre2, st["tok"], None)
    e1, a1, _, x1 = om.forward(m1, pre1, st["tok"], None)
    assert np.array_equal(x2["layers"][1], x2["layers"][0])
    assert np.array_equal(e1, e2) and np.array_equal(a1, a2)
    # and a non-zero second layer changes them
    e3, *_ = om.forward(oracle_model(wl2), pre2, st["tok"], None)
    assert not np.allclose(e3, e1)


def test_fp8_expert_ffn_worked_by_hand():
    """One expert, d = 2, I = 1, e4m3 weights that are exact at scale 1:
    gate row (1, 0), up row (0, 1), down column (1, -0.5). The token (1.5, 2)
    is exact in e4m3 at its scale 2^-7 (192 and 256), so g = 1.5 and u = 2;
    GELU(1.5) u = 2 * 1.5 * Phi(1.5) = 2.79957... rounds to the bf16 value
    2.796875, whose e4m3 quantization at scale 2^-7 is 358 -> 352, i.e. 2.75;
    the output is 2.75 * (1, -0.5) = (2.75, -1.375)."""
    m = {"dtype": "bf16", "n_experts": 1, "top_k": 1, "moe_inter": 1, "n_shared": 0,
         "w_gate": on.round_to_e4m3(np.array([[[1.0, 0.0]]])), "w_gate_scale": np.ones((1, 1)),
         "w_up": on.round_to_e4m3(np.array([[[0.0, 1.0]]])), "w_up_scale": np.ones((1, 1)),
         "w_down": on.round_to_e4m3(np.array([[[1.0], [-0.5]]])), "w_down_scale": np.ones((1, 2))}
    y = om.expert_ffn(m, 0, np.array([[1.5, 2.0]]))
    assert 2 * 1.5 * 0.5 * (1 + math.erf(1.5 / math.sqrt(2))) == pytest.approx(2.79957, abs=1e-5)
    assert y.tolist() == [[2.75, -1.375]]
    # the storage-dtype expert with the same (dequantized) weights keeps 2.796875
    m16 = {"dtype": "bf16", "w_gate": np.array([[[1.0, 0.0]]]), "w_up": np.array([[[0.0, 1.0]]]),
           "w_down": np.array([[[1.0], [-0.5]]])}
    assert om.expert_ffn(m16, 0, np.array([[1.5, 2.0]])).tolist() == [[2.796875, -1.3984375]]


def test_fp8_rows_matmul_is_the_exact_scaled_integer_sum():
    rng = np.random.default_rng(8)
    x = rng.standard_normal((3, 96))
    w = rng.integers(0, 126, (4, 96)).astype(np.uint8)  # non-negative finite codes
    sw = np.exp2(rng.integers(-6, 3, 4).astype(float))
    got = om.fp8_matmul_rows(x, w, sw)
    qx, ex = on.quantize_rows_e4m3(x)
    for i in range(3):
        for j in range(4):
            n = sum(int(round(a * 512)) * int(round(b * 512))
                    for a, b in zip(on.e4m3_to_f64(qx[i]), on.e4m3_to_f64(w[j])))
            assert got[i, j] == n * 2.0 ** -18 * 2.0 ** ex[i] * sw[j]
