"""The FP8 (e4m3) LM head against the fp64 oracle, through the C ABI (the FP8
deployment of "DiffusionGemma深度拆解：从逐字蹦到整块喷，LLM生成范式的结构性跃迁",
性能数据, and "谷歌DiffusionGemma：并行生成与自纠的新突破", 引入扩散机制).

The row quantization must give the oracle's e4m3 codes and power-of-two
scales bit for bit (both sides divide by a power of two, exactly, and round
to nearest with ties to even). The LM head's entropies must be within 1e-3
nats of the oracle's FP8 logits and the argmax equal outside near-ties; the
full step decodes free-running against the oracle with the same LM head."""
import math

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from oracle import model as om
from oracle import numerics as on
from token_canvas_denoising_b200 import inputs as fx
from tests.oracle_adapter import oracle_model, oracle_prefix, oracle_sched
from tests.parity import run_lockstep

pytestmark = pytest.mark.gpu


def _bf16(bits):
    from token_canvas_denoising_b200.canvas import to_device
    return to_device(bits, "bf16", "cuda")


@pytest.mark.parametrize("M,d,scale", [(300, 256, 1.0), (64, 2816, 1e-3), (7, 128, 40.0)])
def test_row_quantization_is_bit_exact(M, d, scale):
    import ctypes as C
    from token_canvas_denoising_b200 import _lib
    lib = _lib.load()
    bits = fx.normal(71, 1, (M, d), scale, "bf16")
    bits[3 % M, :5] = 0  # some zeros
    x = _bf16(bits)
    codes = torch.empty(M, d, dtype=torch.uint8, device="cuda")
    sc = torch.empty(M, dtype=torch.float32, device="cuda")
    st = lib.dg_quantize_rows_e4m3(C.c_void_p(x.data_ptr()), C.c_void_p(codes.data_ptr()), C.c_void_p(sc.data_ptr()),
                                   M, d, C.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0
    q_o, e_o = on.quantize_rows_e4m3(on.bf16_bits_to_f64(bits))
    assert np.array_equal(sc.cpu().numpy().astype(np.float64), np.exp2(e_o.astype(np.float64)))
    got = codes.cpu().numpy()
    # +0 and -0 are the same value; compare values and the non-zero codes
    assert np.array_equal(on.e4m3_to_f64(got), on.e4m3_to_f64(q_o))
    nz = on.e4m3_to_f64(q_o) != 0
    assert np.array_equal(got[nz], q_o[nz])


@pytest.mark.parametrize("M,d,V,rows", [(300, 256, 8192, None), (256, 2816, 262144, None), (1024, 2816, 262144, 48)])
def test_e4m3_lmhead_matches_oracle(M, d, V, rows):
    from token_canvas_denoising_b200 import ops
    hs_bits = fx.normal(72, 1, (M, d), 1.0, "bf16")
    codes, scales = fx.e4m3_rows(fx.normal(72, 2, (V, d), 1.0 / math.sqrt(d), "f32"))
    invT = np.exp(np.random.default_rng(M).uniform(math.log(0.2), math.log(20), M)).astype(np.float32)
    ent, am = ops.lmhead_entropy_e4m3(_bf16(hs_bits), torch.from_numpy(codes).cuda(),
                                      torch.from_numpy(scales).cuda(), torch.from_numpy(invT).cuda())
    torch.cuda.synchronize()
    sel = np.arange(M) if rows is None else np.random.default_rng(3).choice(M, rows, replace=False)
    m = {"dtype": "bf16", "lm_head_e4m3": codes, "lm_head_scale": scales}
    logits = om.lm_head_logits(m, on.bf16_bits_to_f64(hs_bits[sel]))
    ent_o, am_o, gap_o = om.entropy_argmax(logits, invT[sel].astype(np.float64))
    e = ent.cpu().numpy()[sel]
    a = am.cpu().numpy()[sel]
    assert np.max(np.abs(e - ent_o)) <= 1e-3, np.max(np.abs(e - ent_o))
    sure = gap_o > 1e-3
    assert np.array_equal(a[sure], am_o[sure])
    for r in np.nonzero(~sure)[0]:  # near-ties: the GPU's token is within 1e-3 of the top logit
        assert logits[r, a[r]] >= logits[r, am_o[r]] - 1e-3


@pytest.mark.parametrize("adaptive", [False, True])
def test_fp8_small_full_decode(adaptive):
    from token_canvas_denoising_b200.canvas import from_workload, schedule
    cfg = fx.Config("fp8_small", B=2, C=200, S=(150, 30), d=256, Hq=4, Hk=2, h=128, V=4096, dtype="bf16",
                    max_steps=12, weight_seed=77, canvas_seeds=(6, 7), inv_temp="loguniform", lm_fp8=True)
    wl = fx.make_workload(cfg)
    cv, keep = from_workload(wl)
    try:
        rep, steps = run_lockstep(cfg, cv, oracle_model(wl), oracle_prefix(wl), oracle_sched(cfg, adaptive=adaptive),
                                  schedule(cfg.max_steps, cfg.stop_entropy, adaptive), wl.inv_temp.astype(np.float64))
    finally:
        cv.close()
    print(f"fp8_small adaptive={adaptive}: {steps} steps; {rep.summary()}")
    assert not rep.errors, "\n".join(rep.errors[:20])


@pytest.mark.slow
def test_vocab262k_fp8_full_decode():
    from token_canvas_denoising_b200.canvas import from_workload, schedule
    cfg = fx.CONFIGS["vocab262k_fp8"]
    wl = fx.make_workload(cfg)
    cv, keep = from_workload(wl)
    try:
        rep, steps = run_lockstep(cfg, cv, om.prewiden(oracle_model(wl), ("wq", "wk", "wv", "wo")), oracle_prefix(wl),
                                  oracle_sched(cfg, adaptive=False), schedule(cfg.max_steps, cfg.stop_entropy, False),
                                  wl.inv_temp.astype(np.float64), tensor_steps={0, 1, cfg.max_steps - 1})
        final = cv.get_state()
    finally:
        cv.close()
        del keep
        torch.cuda.empty_cache()
    print(f"vocab262k_fp8: {steps} steps; {rep.summary()}")
    assert not rep.errors, "\n".join(rep.errors[:20])
    assert steps == cfg.max_steps and np.all(final["done"])


@pytest.mark.parametrize("adaptive", [False, True])
def test_fp8_moe_small_full_decode(adaptive):
    """e4m3 expert weights and LM head on a small MoE model (I = 192: a K tail
    of 64 past the last 128-byte block in the down projection), full decode."""
    from token_canvas_denoising_b200.canvas import from_workload, schedule
    cfg = fx.Config("fp8_moe_small", B=1, C=96, S=(150,), d=256, Hq=2, Hk=1, h=128, V=2048, dtype="bf16",
                    max_steps=8, weight_seed=87, canvas_seeds=(5,), n_experts=32, top_k=4, moe_inter=192, n_shared=1,
                    lm_fp8=True, moe_fp8=True)
    wl = fx.make_workload(cfg)
    cv, keep = from_workload(wl)
    try:
        rep, steps = run_lockstep(cfg, cv, oracle_model(wl), oracle_prefix(wl), oracle_sched(cfg, adaptive=adaptive),
                                  schedule(cfg.max_steps, cfg.stop_entropy, adaptive), None)
    finally:
        cv.close()
    print(f"fp8_moe_small adaptive={adaptive}: {steps} steps; {rep.summary()}")
    assert not rep.errors, "\n".join(rep.errors[:20])


@pytest.mark.slow
def test_moe_fp8_full_decode():
    """The moe workload (128 + 1 experts, top-8, I = 704, V = 262,144) with
    e4m3 experts and LM head, 48 free-running steps."""
    from token_canvas_denoising_b200.canvas import from_workload, schedule
    cfg = fx.CONFIGS["moe_fp8"]
    wl = fx.make_workload(cfg)
    cv, keep = from_workload(wl)
    try:
        rep, steps = run_lockstep(cfg, cv, om.prewiden(oracle_model(wl), ("wq", "wk", "wv", "wo")), oracle_prefix(wl),
                                  oracle_sched(cfg, adaptive=False), schedule(cfg.max_steps, cfg.stop_entropy, False),
                                  wl.inv_temp.astype(np.float64), tensor_steps={0, 1, cfg.max_steps - 1})
        final = cv.get_state()
    finally:
        cv.close()
        del keep
        torch.cuda.empty_cache()
    print(f"moe_fp8: {steps} steps; {rep.summary()}")
    assert not rep.errors, "\n".join(rep.errors[:20])
    assert steps == cfg.max_steps and np.all(final["done"])
