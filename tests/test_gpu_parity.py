"""GPU parity: the CUDA path through the C ABI against the CPU oracle on the
five synthetic workloads and on edge cases.

Per step (teacher-forced from identical bytes): codes bit-exact except 1-LSB
flips on at most 1e-5 of the entries, o within 1e-4 relative L2. After the
rollout: the dequantized state within 1e-3 relative Frobenius (checked by a
separate free-running pass whenever a flip occurred).
"""
import numpy as np
import pytest
import torch

import oracle
from quantized_linear_attention_sq_b200 import _abi, synth
from tests import gpu_util as gu
from tests.helpers import oracle_for, random_calib, random_inputs, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from quantized_linear_attention_sq_b200 import build
    build.build()
    torch.cuda.init()


def _report(name, stats, rollout):
    print(f"\n[{name}] steps={stats.steps} entries={stats.entries} flips={stats.flips} "
          f"r_flips={stats.r_flips} max_diff={stats.max_code_diff} worst_o={stats.worst_o:.2e} "
          f"rollout={rollout:.2e} {stats.notes}")


def test_plumbing_config_full():
    w = synth.workload(0)
    stats, rollout = gu.run_parity(w, w.cfg.steps)
    _report("plumbing", stats, rollout)
    stats.check()
    assert rollout <= gu.ROLLOUT_TOL


def test_gdn_layer_config_subset():
    w = synth.workload(1, batch=4)
    stats, rollout = gu.run_parity(w, w.cfg.steps)
    _report("gdn_layer", stats, rollout)
    stats.check()
    assert rollout <= gu.ROLLOUT_TOL


def test_kda_layer_config_subset():
    w = synth.workload(2, batch=4)
    stats, rollout = gu.run_parity(w, w.cfg.steps)
    _report("kda_layer", stats, rollout)
    stats.check()
    assert rollout <= gu.ROLLOUT_TOL


def test_serving_config_all_tiles_two_steps():
    """Batch 512 x 32 value heads in the launch configuration of the
    benchmark, every one of the 16 384 tiles checked against the oracle for
    two steps (from the oracle's FP32 warm-up of all 512 requests)."""
    w = synth.workload(3)
    stats, rollout = gu.run_parity(w, 2)
    _report("serving all tiles", stats, rollout)
    stats.check()
    assert rollout <= gu.ROLLOUT_TOL


def test_serving_config_full_size_sampled_requests():
    """Batch 512 x 32 value heads in the launch configuration of the benchmark;
    the oracle follows 16 sampled requests through all 128 steps."""
    w = synth.workload(3)
    reqs = [0, 37, 64, 101, 150, 200, 222, 255, 290, 318, 360, 401, 444, 470, 499, 511]
    stats, rollout = gu.run_parity(w, w.cfg.steps, check_requests=reqs, use_gpu_warmup=True)
    _report("serving", stats, rollout)
    stats.check()
    assert rollout <= gu.ROLLOUT_TOL
    gap = float(stats.notes[0].split()[-1])
    assert gap <= 1e-4  # GPU FP32 warm-up vs oracle FP32 warm-up


@pytest.mark.parametrize("cid,reqs", [(1, [0, 21, 42, 63]), (2, [0, 50, 101, 127])])
def test_layer_configs_full_batch_sampled(cid, reqs):
    """The GDN layer (batch 64) and KDA layer (batch 128) workloads at full
    batch, one launch per step over all requests; the oracle follows four
    sampled requests for 64 steps."""
    w = synth.workload(cid)
    stats, rollout = gu.run_parity(w, 64, check_requests=reqs, use_gpu_warmup=True)
    _report(f"layer cid={cid} full batch", stats, rollout)
    stats.check()
    assert rollout <= gu.ROLLOUT_TOL


@pytest.mark.parametrize("layer", range(8))
def test_long_rollout_config_full(layer):
    """The 8-layer, batch-256 KDA workload at its full length: every layer
    steps all 256 requests for 2048 steps (inputs drawn on the device); the
    oracle follows two requests per layer (a different pair per layer) with
    the per-step acceptance, and their final dequantized states agree within
    1e-3 relative Frobenius."""
    w = synth.workload(4, layer=layer)
    reqs = [(3 + 37 * layer) % 256, (250 - 29 * layer) % 256]
    stats, final, rollout = gu.run_parity_device_inputs(w, w.cfg.steps, reqs)
    _report(f"long_rollout_l{layer} reqs={reqs}", stats, max(final, rollout))
    stats.check()
    assert final <= gu.ROLLOUT_TOL and rollout <= gu.ROLLOUT_TOL


@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("gate_kind", [0, 1])
def test_edge_shapes_all_widths_and_pivots(d, gate_kind):
    """Every width {2,4,6,8} and pivots mixed, d in {32, 64, 128}, a ragged
    batch of 5 requests scattered over a larger pool in permuted slots."""
    rng = np.random.default_rng(1000 + d + gate_kind)
    B, h_v, h_k = 5, 6, 3
    bits, piv, col, phi = random_calib(rng, h_v, d, gate_kind, widths=(2, 4, 6, 8), pivot_p=0.15,
                                       phi_range=(0.3, 3.0))
    # the generator's own allocation is replaced by the random tables below
    cfg = synth.Config(99, "edge", gate_kind, B, h_v, h_k, d, 12, 64.0, (8,), 8, 0.0, 0.5, 1.0, 0, 0.0)
    w = synth.Workload(cfg, seed=d)
    cal = w.calib()
    cal.unit_bits[...] = bits
    cal.pivot[...] = piv
    cal.col_scale[...] = col
    cal.row_impact[...] = phi
    perm = np.array([7, 2, 9, 0, 4], dtype=np.int32)
    stats, rollout = gu.run_parity(w, 12, slot_perm=perm, n_slots=11)
    _report(f"edge d={d} gate={gate_kind}", stats, rollout)
    stats.check()
    assert rollout <= gu.ROLLOUT_TOL


@pytest.mark.parametrize("gate_kind", [0, 1])
def test_fp32_format_matches_oracle(gate_kind):
    rng = np.random.default_rng(5 + gate_kind)
    B, h_v, h_k, d = 6, 8, 4, 128
    sp = gu.StatePool(B, h_v, h_k, d, gate_kind, _abi.SQ_FMT_FP32)
    bits, piv, col, phi = random_calib(rng, h_v, d, gate_kind)
    o_ = oracle.Oracle(B, h_v, h_k, d, gate_kind, bits, piv, col, phi)
    S = (rng.standard_normal((B, h_v, d, d)) * 0.3).astype(np.float32)
    pool = sp.new_pool()
    sp.quantize_state(pool, torch.from_numpy(S).cuda())
    ref = S.copy()
    o = torch.empty((B, h_v, d), device="cuda")
    for t in range(8):
        q, k, v, beta, g = random_inputs(rng, B, h_v, h_k, d, gate_kind)
        sp.decode_step(pool, *gu.to_dev(q, k, v, beta, g), o)
        o_ref, _ = o_.step_fp32(ref, q, k, v, beta, g, threads=gu.THREADS)
        assert rel_l2(o.cpu().numpy(), o_ref) <= 1e-5
    out = torch.empty_like(pool)
    sp.dequantize_state(pool, out)
    assert rel_l2(out.cpu().numpy(), ref) <= 1e-5
    assert sp.get_status() == 0
    sp.close()


def test_dequantize_matches_oracle_bit_exact():
    w = synth.workload(2, batch=3)
    o_ = oracle_for(oracle, w, n_slots=3)
    sp = gu.gpu_pool_for(w, 3)
    S = gu.oracle_warm_state(w, [0, 1, 2])
    pool_ref = o_.new_pool()
    o_.quantize(pool_ref, S)
    pool = torch.from_numpy(pool_ref.copy()).cuda()
    out = torch.empty((3, w.cfg.h_v, w.cfg.d, w.cfg.d), device="cuda")
    sp.dequantize_state(pool, out)
    ref, _ = o_.dequantize(pool_ref)
    assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))
    sp.close()


def test_empty_batch_is_a_noop():
    w = synth.workload(0)
    sp = gu.gpu_pool_for(w, 1)
    pool = sp.new_pool()
    n0 = sp.launches()
    z = torch.empty(0, device="cuda")
    sp.decode_step(pool, z, z, z, z, z, z)
    sp.quantize_state(pool, torch.empty((0, 4, 64, 64), device="cuda"))
    assert sp.launches() == n0
    assert int(pool.sum()) == 0
    sp.close()


def test_bad_slot_nan_and_saturation_status():
    w = synth.workload(1, batch=3)
    c = w.cfg
    sp = gu.gpu_pool_for(w, 3)
    o_ = oracle_for(oracle, w, n_slots=3)
    S = gu.oracle_warm_state(w, [0, 1, 2])
    pool_ref = o_.new_pool()
    o_.quantize(pool_ref, S)
    pool = torch.from_numpy(pool_ref.copy()).cuda()
    q, k, v, beta, g = w.step_inputs(0)
    slots = np.array([0, 5, 2], np.int32)             # slot 5 does not exist
    v = v.copy()
    v[2, 4, 7] = np.nan                                # NaN in request 2, head 4
    o = torch.full((3, c.h_v, c.d), 7.0, device="cuda")
    sp.decode_step(pool, *gu.to_dev(q, k, v, beta, g), o, torch.from_numpy(slots).cuda())
    o_ref, st_ref = o_.step(pool_ref, q, k, v, beta, g, slots=slots)
    st = sp.get_status()
    assert st == st_ref
    assert st & _abi.SQ_STATUS_BAD_SLOT and st & _abi.SQ_STATUS_NAN
    assert torch.all(o[1] == 0)
    got = pool.cpu().numpy()
    assert np.array_equal(got, pool_ref)               # slot 1 untouched, NaN rows zeroed alike
    on = o.cpu().numpy()
    fin = np.isfinite(o_ref)
    assert rel_l2(on[fin], o_ref[fin]) <= 1e-5
    # saturation: a huge state saturates row scales and pivots at 65504
    S_big = np.full((3, c.h_v, c.d, c.d), 1e9, np.float32)
    pool_ref2 = o_.new_pool()
    st_ref2 = o_.quantize(pool_ref2, S_big)
    pool2 = sp.new_pool()
    sp.quantize_state(pool2, torch.from_numpy(S_big).cuda())
    assert sp.get_status() == st_ref2 and st_ref2 & _abi.SQ_STATUS_SATURATED
    assert np.array_equal(pool2.cpu().numpy(), pool_ref2)
    sp.close()


def test_argument_errors_raise_before_launch():
    w = synth.workload(0)
    sp = gu.gpu_pool_for(w, 1)
    pool = sp.new_pool()
    q, k, v, beta, g = gu.to_dev(*w.step_inputs(0))
    o = torch.empty((1, 4, 64), device="cuda")
    n0 = sp.launches()
    with pytest.raises(ValueError):
        sp.decode_step(pool, q.double(), k, v, beta, g, o)
    with pytest.raises(ValueError):
        sp.decode_step(pool[:-16], q, k, v, beta, g, o)
    with pytest.raises(_abi.SQError):
        _abi.sq_decode_step(sp._h, pool.data_ptr() + 4, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                            beta.data_ptr(), g.data_ptr(), o.data_ptr(), None, 1,
                            torch.cuda.current_stream().cuda_stream)
    assert sp.launches() == n0
    sp.close()
