"""The planner extras of the library against the oracle: per-GPU footprint,
the "Auto" shard degree ("Tensor Parallelism" docs, section "Auto") and the
per-token time model ("Tensor parallel scaling curves", section "The scaling
math").  Host code only: CPU."""
import ctypes
import itertools

import pytest

import oracle

DIMS = [(8192, 64, 8, 128, 28672, 80), (4096, 32, 32, 128, 11008, 32), (1024, 16, 2, 64, 2816, 4),
        (256, 4, 2, 64, 688, 2), (5120, 40, 40, 128, 13824, 40)]


@pytest.fixture(scope="module")
def tpl():
    from megatron_tensor_transformer_plan_b200 import build
    build.build()
    from megatron_tensor_transformer_plan_b200 import tpl as m
    return m


def _dims(tpl, H, nq, nkv, d, F, L):
    return tpl.make_dims(H, nq, nkv, d, F, L)


@pytest.mark.parametrize("dm", DIMS)
def test_footprint_matches_oracle(tpl, dm):
    H, nq, nkv, d, F, L = dm
    td, od = _dims(tpl, *dm), oracle.Dims(H, nq, nkv, d, F)
    for t, B, S, e in itertools.product((1, 2, 3, 4, 8, 16), (0, 1, 16), (0, 1, 8192), (2, 4)):
        assert tpl.footprint_bytes(td, t, B, S, e) == oracle.footprint_per_gpu(od, L, t, B, S, e), (t, B, S, e)


@pytest.mark.parametrize("dm", DIMS)
def test_auto_t_matches_oracle(tpl, dm):
    H, nq, nkv, d, F, L = dm
    td, od = _dims(tpl, *dm), oracle.Dims(H, nq, nkv, d, F)
    B, S = 16, 8192
    f = [oracle.footprint_per_gpu(od, L, t, B, S, 2) for t in (1, 2, 4, 8)]
    budgets = [0, -1, 1000, 24 * 10**9, 80 * 10**9, 180 * 10**9, 10**13]
    budgets += [x for x in f if x > 0] + [x - 1 for x in f if x > 1]
    for budget, h, max_t in itertools.product(budgets, (0.0, 0.1, 0.5), (1, 2, 3, 4, 8, 16)):
        want = oracle.auto_t(od, L, budget, h, B, S, 2, max_t)
        assert tpl.auto_t(td, budget, h, B, S, 2, max_t) == want, (budget, h, max_t)


def test_auto_t_70b_example_and_status(tpl):
    td = _dims(tpl, 8192, 64, 8, 128, 28672, 80)
    assert tpl.auto_t(td, 80 * 10**9, 0.1, 16, 8192) == 4
    out = ctypes.c_int32(-1)
    assert tpl.tpl_auto_t(ctypes.byref(td), 1000, 0.1, 16, 8192, 2, 8, ctypes.byref(out)) == tpl.TPL_ENOFIT
    assert out.value == 0
    assert tpl.tpl_auto_t(ctypes.byref(td), 10**9, 1.0, 1, 1, 2, 8, ctypes.byref(out)) == tpl.TPL_EINVAL
    assert tpl.tpl_auto_t(ctypes.byref(td), 10**9, 0.1, 1, 1, 2, 0, ctypes.byref(out)) == tpl.TPL_EINVAL
    assert tpl.tpl_auto_t(None, 10**9, 0.1, 1, 1, 2, 8, ctypes.byref(out)) == tpl.TPL_EINVAL
    assert b"budget" in tpl.tpl_status_string(tpl.TPL_ENOFIT)


@pytest.mark.parametrize("n", [1, 2, 4, 8])
def test_tp_estimate_matches_oracle(tpl, n):
    for tc, tm, L, msg, lat, bw in ((0.002, 0.028, 80, 16384, 8e-6, 770e9), (0.0, 0.03, 80, 16384, 8e-6, 100e9),
                                    (1e-3, 5e-3, 32, 1 << 20, 5e-6, 900e9), (0.0, 0.0, 0, 0, 0.0, 1.0)):
        e = tpl.tp_estimate(tc, tm, n, L, msg, lat, bw)
        ar = oracle.allreduce_time(n, msg, lat, bw)
        tot = oracle.tp_time(tc + tm, n, L, ar)
        assert e.t_allreduce == pytest.approx(ar, rel=1e-14, abs=0)
        assert e.t_comm == pytest.approx(2 * L * ar, rel=1e-14, abs=0)
        assert e.t_total == pytest.approx(tot, rel=1e-14, abs=0)
        if tot > 0:
            assert e.speedup == pytest.approx((tc + tm) / tot, rel=1e-14)
            assert e.comm_share == pytest.approx(2 * L * ar / tot, rel=1e-14)


def test_tp_estimate_worked_example(tpl):
    """TP=2 at 30 ms single-GPU with 160 calls of 8 us: 16.28 ms, 1.84x."""
    # t_allreduce of 8 us: latency 8 us and a negligible bandwidth part
    e = tpl.tp_estimate(0.0, 0.030, 2, 80, 0.0, 8e-6, 1e12)
    assert e.t_comm == pytest.approx(1.28e-3, rel=1e-12)
    assert e.t_total == pytest.approx(16.28e-3, rel=1e-12)
    assert round(e.speedup, 2) == 1.84
    out = tpl.tpl_tp_estimate()
    for bad in ((0.0, 0.03, 0, 80, 0.0, 8e-6, 1e12), (0.0, 0.03, 2, 80, 0.0, 8e-6, 0.0),
                (-1.0, 0.03, 2, 80, 0.0, 8e-6, 1e12)):
        assert tpl.tpl_tp_estimate_get(*bad, ctypes.byref(out)) == tpl.TPL_EINVAL


def test_decode_times_from_dims(tpl):
    H, nq, nkv, d, F, L = DIMS[0]
    td, od = _dims(tpl, *DIMS[0]), oracle.Dims(H, nq, nkv, d, F)
    B, S, flops, hbm = 16, 8192, 1.6e15, 6.5e12
    tc, tm = tpl.decode_times(td, B, S, 2, flops, hbm)
    params = L * oracle.layer_params_per_shard(od, 1)
    assert tc == pytest.approx(2 * params * B / flops, rel=1e-14)
    assert tm == pytest.approx(oracle.footprint_per_gpu(od, L, 1, B, S, 2) / hbm, rel=1e-14)
    # the 70B decode step at B = 16 is memory-bound: about 28 ms of HBM time
    # against about 1.4 ms of tensor time at these peaks
    assert tm > 10 * tc


def test_plan_report_reproduces_the_pages_examples(tpl):
    from megatron_tensor_transformer_plan_b200 import plan_report
    rows = plan_report.report("70b", batch=1, seq=8192, gpu_gb=80, headroom=0.1, latency_us=8.0, link_gbs=770.0,
                              t_single_ms=30.0)
    head, est = rows[0], {r["n"]: r for r in rows[1:]}
    assert head["auto_t"] == 2  # one sequence's cache: t = 2 already fits 80 GB cards
    assert head["auto_t_blind_8_gpus"] == 8
    assert est[1]["speedup"] == 1.0 and est[1]["t_comm_ms"] == 0.0
    assert round(est[2]["speedup"], 2) == 1.84  # 16 KB message: about 8 us per call
    assert abs(est[2]["t_total_ms"] - 16.3) < 0.05
    rows = plan_report.report("70b", batch=16, seq=8192, gpu_gb=80, headroom=0.1)
    assert rows[0]["auto_t"] == 4
    assert rows[1]["t_memory_ms"] > rows[1]["t_compute_ms"] > 0


def test_rope_flag_validation(tpl):
    d = tpl.make_dims(1024, 16, 4, 128, 2816, 1, 1e-5, tpl.TPL_NORM | tpl.TPL_ROPE, rope_base=10000.0)
    tpl.Plan(d, 4)
    for bad in (1.0, 0.0, -5.0, float("nan")):
        d = tpl.make_dims(1024, 16, 4, 128, 2816, 1, 1e-5, tpl.TPL_ROPE, rope_base=bad)
        with pytest.raises(tpl.TplError) as e:
            tpl.Plan(d, 4)
        assert e.value.code == tpl.TPL_EINVAL
    # without the flag the base is ignored
    tpl.Plan(tpl.make_dims(1024, 16, 4, 128, 2816, 1, 1e-5, tpl.TPL_NORM, rope_base=0.0), 4)


def test_decode_kernel_count(tpl):
    """Kernels per decode call: five per layer with the mma.sync projections;
    with the tensor-core ones the operand kernel before QKV once per call
    (the fused O and down write the others), 9 per layer in separate mode;
    one more per layer with the rotation."""
    p = tpl.Plan(tpl.make_dims(8192, 64, 8, 128, 28672, 80), 8)
    assert [p.decode_kernel_count(b) for b in (1, 4, 16, 64)] == [6, 6, 6, 6]  # large layer: tcgen05 throughout
    assert p.decode_kernel_count(4, n_layers=80) == 401
    assert p.decode_kernel_count(1, n_layers=80) == 401
    assert p.decode_kernel_count(4, tpl.TPL_REDUCE_SEPARATE) == 9
    assert p.decode_kernel_count(4, tpl.TPL_REDUCE_SEPARATE, n_layers=80) == 720
    p.set_option(tpl.TPL_OPT_GEMV_MODE, 0)
    assert [p.decode_kernel_count(b) for b in (4, 16, 17)] == [5, 5, 6]
    assert p.decode_kernel_count(4, tpl.TPL_REDUCE_SEPARATE) == 7
    small = tpl.Plan(tpl.make_dims(4096, 32, 32, 128, 11008, 32, 1e-5,
                                   tpl.TPL_NORM | tpl.TPL_RESIDUAL | tpl.TPL_ROPE), 4)
    assert [small.decode_kernel_count(b) for b in (1, 2, 6, 7, 8, 16)] == [6, 6, 6, 7, 7, 7]  # tcgen05 from 7 tokens
    assert small.decode_kernel_count(16, n_layers=32) == 5 * 32 + 1 + 32
    with pytest.raises(tpl.TplError):
        p.decode_kernel_count(65)
