"""GPU parity of the per-window variant (sq_window_step) against the oracle.

Per-window quantization ("线性注意力每生成一个token都要搬状态，LeapQuant把它压到
8位还不掉点" (wink.run), first technique). Both sides start from the same
quantized bytes and empty window buffers and take the same tokens; after
every token the outputs, the window buffers and the pools are compared:

- o within the step's tolerance (relative L2);
- window records: counts, buffered keys and gates identical; buffered u
  identical except where the fp64 sums of the two sides (different orders)
  straddle an fp32 rounding boundary: at most one fp32 ulp, rarely;
- pools: identical inside a window (the state is frozen) and, after the
  window's requantization, codes identical up to the step's rare 1-LSB flips
  (both sides form the window-end state with the same fp32 operations in
  the same order, so it differs only where the buffered u did).
Where anything differs the GPU continues from the oracle's bytes (teacher
forcing)."""
import numpy as np
import pytest
import torch

import oracle
from quantized_linear_attention_sq_b200 import _abi, synth
from tests.gpu_util import (THREADS, Stats, compare_slots, gpu_pool_for, oracle_warm_state, slot_bytes, to_dev)
from tests.helpers import oracle_for, random_calib, rel_l2

pytestmark = pytest.mark.gpu

U_ULP_RATE = 1e-3  # buffered u values allowed to differ (by one ulp)


def _wrec_view(buf: np.ndarray, n_rec: int, rb: int):
    return buf.reshape(n_rec, rb)


def compare_windows(ref: np.ndarray, got: np.ndarray, rb: int, W: int, d: int, gd: int, counters: dict):
    R, G = _wrec_view(ref, -1, rb), _wrec_view(got, -1, rb)
    assert np.array_equal(R[:, :16], G[:, :16]), "window counts differ"
    k0, k1 = 16, 16 + 4 * W * d
    u1 = k1 + 4 * W * d
    assert np.array_equal(R[:, k0:k1], G[:, k0:k1]), "buffered keys differ"
    assert np.array_equal(R[:, u1:], G[:, u1:]), "buffered gates differ"
    ur = R[:, k1:u1].copy().view(np.float32)
    ug = G[:, k1:u1].copy().view(np.float32)
    assert np.array_equal(np.isnan(ur), np.isnan(ug)), "NaN in one buffer and not the other"
    diff = (ur != ug) & ~np.isnan(ur)
    counters["u_entries"] += ur.size
    if diff.any():
        a, b = ur[diff].astype(np.float64), ug[diff].astype(np.float64)
        ulp = np.spacing(np.maximum(np.abs(a), np.abs(b)).astype(np.float32)).astype(np.float64)
        assert (np.abs(a - b) <= ulp).all(), "a buffered u differs by more than one ulp"
        counters["u_diff"] += int(diff.sum())
    return bool(diff.any())


def run_window_parity(cid, W: int, steps: int, check_requests=None, batch=None, slot_perm=None, n_slots=None):
    """cid: a workload id, or a synth.Workload. slot_perm: [B] GPU pool slot
    of each request (default: request b in slot b) in a pool of n_slots."""
    w = cid if isinstance(cid, synth.Workload) else synth.workload(cid, batch=batch)
    c = w.cfg
    B = w.B
    reqs = list(range(B)) if check_requests is None else list(check_requests)
    sel = np.asarray(reqs)
    o_ = oracle_for(oracle, w, n_slots=len(reqs))
    slots = np.arange(B, dtype=np.int32) if slot_perm is None else np.asarray(slot_perm, np.int32)
    n_slots = n_slots or B
    sp = gpu_pool_for(w, n_slots)
    rb, _ = sp.window_buffer_bytes(W)
    assert rb == o_.window_record_bytes(W)
    gd = c.d if c.gate_kind == _abi.SQ_GATE_KEY_CHANNEL else 1
    # initial state: the checked requests start from the oracle's fp32 state
    S_ref = oracle_warm_state(w, reqs)
    S_all = torch.from_numpy(w.initial_state()).cuda()
    S_all.index_copy_(0, torch.as_tensor(reqs, device="cuda"), torch.from_numpy(S_ref).cuda())
    pool_ref = o_.new_pool()
    o_.quantize(pool_ref, S_ref)
    pool = sp.new_pool()
    slots_t = torch.from_numpy(slots).cuda()
    sp.quantize_state(pool, S_all, slots_t)
    del S_all
    wref = o_.new_window_buffer(W)
    wbuf = sp.new_window_buffer(W)
    gslots = slots[sel]
    assert np.array_equal(slot_bytes(pool, sp, gslots), pool_ref)
    o_dev = torch.empty((B, c.h_v, c.d), device="cuda")
    stats = Stats()
    counters = {"u_entries": 0, "u_diff": 0}
    st_all = 0
    idx = torch.as_tensor(gslots, device="cuda", dtype=torch.long)
    for t in range(steps):
        q, k, v, beta, g = w.step_inputs(t)
        sp.window_step(pool, wbuf, W, *to_dev(q, k, v, beta, g), o_dev, slots_t)
        o_ref, st_ref = o_.window_step(pool_ref, wref, W, q[sel], k[sel], v[sel], beta[sel], g[sel],
                                       threads=THREADS)
        st_all |= st_ref
        o_got = o_dev.cpu().numpy()[sel]
        nan = np.isnan(o_ref)
        assert np.array_equal(nan, np.isnan(o_got)), "NaN outputs differ"
        stats.worst_o = max(stats.worst_o, rel_l2(np.where(nan, 0, o_got), np.where(nan, 0, o_ref)))
        got_w = wbuf.view(n_slots * c.h_v, rb).index_select(0, (idx[:, None] * c.h_v + torch.arange(
            c.h_v, device="cuda")[None]).reshape(-1)).cpu().numpy().reshape(-1)
        u_diff = compare_windows(wref, got_w, rb, W, c.d, gd, counters)
        got = slot_bytes(pool, sp, gslots)
        f0 = stats.flips + stats.r_flips
        compare_slots(o_, pool_ref, got, stats)
        stats.steps += 1
        if u_diff or stats.flips + stats.r_flips != f0:
            pv = pool.view(-1, sp.slot_bytes)
            pv[idx] = torch.from_numpy(pool_ref.reshape(len(reqs), -1)).cuda()
            wv = wbuf.view(n_slots, -1)
            wv[idx] = torch.from_numpy(wref.reshape(len(reqs), -1)).cuda()
    st_gpu = sp.get_status()
    if len(reqs) == B:
        assert st_gpu == st_all, (st_gpu, st_all)
    sp.close()
    return stats, counters


@pytest.mark.parametrize("cid,W,steps", [(0, 4, 11), (0, 16, 35), (0, 1, 5), (0, 64, 70), (0, 16, 200)])
def test_window_plumbing(cid, W, steps):
    stats, cnt = run_window_parity(cid, W, steps)
    print(stats, cnt)
    stats.check()
    assert cnt["u_diff"] <= U_ULP_RATE * cnt["u_entries"], cnt


@pytest.mark.parametrize("cid", [1, 2])
def test_window_layer(cid):
    """GDN and KDA layers (mixed widths, pivots, outlier columns), W = 16,
    over two windows and a bit."""
    stats, cnt = run_window_parity(cid, 16, 35, check_requests=[0, 5, 17, 63])
    print(stats, cnt)
    stats.check()
    assert cnt["u_diff"] <= U_ULP_RATE * cnt["u_entries"], cnt


def test_window_serving_full_size():
    """The GDN serving batch (512 requests x 32 heads) as the bench launches
    it; sampled requests checked against the oracle through one window end."""
    stats, cnt = run_window_parity(3, 16, 18, check_requests=[0, 1, 255, 511])
    print(stats, cnt)
    stats.check()
    assert cnt["u_diff"] <= U_ULP_RATE * cnt["u_entries"], cnt


def test_window_bad_count_and_slot():
    """A window count outside [0, W) skips the tile (o = 0, status bit, the
    pool and the buffer untouched); so does a slot id out of range."""
    w = synth.workload(0)
    c = w.cfg
    sp = gpu_pool_for(w, 2)
    W = 8
    rb, nb = sp.window_buffer_bytes(W)
    pool = sp.new_pool()
    sp.quantize_state(pool, torch.from_numpy(np.repeat(w.initial_state(), 2, 0)).cuda())
    wbuf = sp.new_window_buffer(W)
    wbuf.view(-1, rb)[0, :4] = torch.tensor([W, 0, 0, 0], dtype=torch.uint8)  # slot 0, head 0: count W
    pool0, w0 = pool.clone(), wbuf.clone()
    q, k, v, beta, g = to_dev(*w.step_inputs(0))
    o = torch.full((1, c.h_v, c.d), 7.0, device="cuda")
    sp.get_status()
    sp.window_step(pool, wbuf, W, q, k, v, beta, g, o, torch.tensor([0], dtype=torch.int32, device="cuda"))
    assert sp.get_status() == _abi.SQ_STATUS_WINDOW
    assert (o[0, 0] == 0).all() and (o[0, 1:] != 7.0).all()
    assert torch.equal(wbuf.view(-1, rb)[0], w0.view(-1, rb)[0])
    assert torch.equal(pool, pool0)  # inside a window the pool is only read
    sp.window_step(pool, wbuf, W, q, k, v, beta, g, o, torch.tensor([5], dtype=torch.int32, device="cuda"))
    assert sp.get_status() == _abi.SQ_STATUS_BAD_SLOT
    assert (o == 0).all()
    # an empty batch is a no-op
    pool1, w1 = pool.clone(), wbuf.clone()
    sp.window_step(pool, wbuf, W, q[:0], k[:0], v[:0], beta[:0], g[:0], o[:0])
    assert sp.get_status() == 0
    assert torch.equal(pool, pool1) and torch.equal(wbuf, w1)
    with pytest.raises(_abi.SQError):
        sp.window_step(pool, wbuf, 0, q, k, v, beta, g, o)
    with pytest.raises(_abi.SQError):
        sp.window_step(pool, wbuf, 65, q, k, v, beta, g, o)
    sp.close()


@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("gate_kind", [0, 1])
def test_window_edge_shapes(d, gate_kind):
    """Every width {2,4,6,8} and pivots mixed, d in {32, 64, 128}, a ragged
    batch of 5 requests in permuted slots of a pool of 11; W = 3 over 8
    tokens (two window ends and a partial window)."""
    rng = np.random.default_rng(2000 + d + gate_kind)
    B, h_v, h_k = 5, 6, 3
    bits, piv, col, phi = random_calib(rng, h_v, d, gate_kind, widths=(2, 4, 6, 8), pivot_p=0.15,
                                       phi_range=(0.3, 3.0))
    cfg = synth.Config(98, "window-edge", gate_kind, B, h_v, h_k, d, 8, 64.0, (8,), 8, 0.0, 0.5, 1.0, 0, 0.0)
    w = synth.Workload(cfg, seed=d)
    cal = w.calib()
    cal.unit_bits[...] = bits
    cal.pivot[...] = piv
    cal.col_scale[...] = col
    cal.row_impact[...] = phi
    stats, cnt = run_window_parity(w, 3, 8, slot_perm=np.array([7, 2, 9, 0, 4], np.int32), n_slots=11)
    print(stats, cnt)
    stats.check()
    assert cnt["u_diff"] <= U_ULP_RATE * cnt["u_entries"] + 2, cnt


def test_window_too_long_for_shared_memory_is_rejected():
    """KDA at d = 128 with W = 64: two stages of buffered rows and gates do
    not fit in one CTA's shared memory; the call is refused on the host."""
    w = synth.workload(2, batch=2)
    c = w.cfg
    sp = gpu_pool_for(w, 2)
    pool = sp.new_pool()
    wbuf = sp.new_window_buffer(64)
    q, k, v, beta, g = to_dev(*w.step_inputs(0))
    o = torch.zeros((2, c.h_v, c.d), device="cuda")
    with pytest.raises(_abi.SQError, match="shared memory"):
        sp.window_step(pool, wbuf, 64, q, k, v, beta, g, o)
    sp.close()


class _NaNInput(synth.Workload):
    """The plumbing workload with one NaN in v (request 0, head 1, column 5)
    at token 2."""

    def step_inputs(self, step, requests=None):
        q, k, v, beta, g = super().step_inputs(step, requests)
        if step == 2:
            reqs = list(range(self.B)) if requests is None else list(requests)
            if 0 in reqs:
                v = v.copy()
                v[reqs.index(0), 1, 5] = np.nan
        return q, k, v, beta, g


def test_window_nan_input_matches_oracle():
    """A NaN in v makes that column of u NaN for the rest of the window, o
    NaN, and at the window's end every row of the head holds a NaN: those
    rows get scale 0 and code 0 (status NaN), on both sides alike."""
    w = _NaNInput(synth.CONFIGS[0], seed=0)
    stats, cnt = run_window_parity(w, 4, 9)
    print(stats, cnt)
    stats.check()
