"""Shared machinery of the GPU parity tests: build a CUDA state pool and an
oracle from the same workload, prepare the same initial state for both, run
steps side by side and compare (codes bit-exact up to rare 1-LSB flips, o
to relative L2, state to relative Frobenius)."""
from __future__ import annotations

import os
from dataclasses import dataclass, field

import numpy as np
import torch

import oracle
from quantized_linear_attention_sq_b200 import _abi, synth
from quantized_linear_attention_sq_b200.state import StatePool
from tests.helpers import oracle_for, rel_l2

THREADS = max(1, min(32, oracle.cores_available()))

# Acceptance (per step, teacher-forced from identical input bytes): codes and
# row scales identical except 1-LSB flips (one code step, one fp16 step of a
# row scale or of a pivot value at its row's magnitude) on at most FLIP_RATE
# of the entries; o within O_TOL relative L2. After a free-running rollout:
# dequantized state within ROLLOUT_TOL relative Frobenius.
FLIP_RATE = 1e-5
O_TOL = 1e-4
ROLLOUT_TOL = 1e-3


def gpu_pool_for(w: synth.Workload, n_slots: int, fmt=_abi.SQ_FMT_PACKED) -> StatePool:
    c = w.cfg
    cal = w.calib()
    return StatePool(n_slots, c.h_v, c.h_k, c.d, c.gate_kind, fmt, cal.unit_bits, cal.pivot, cal.col_scale,
                     cal.row_impact)


def to_dev(*xs):
    return [torch.from_numpy(np.ascontiguousarray(x)).cuda() for x in xs]


def oracle_warm_state(w: synth.Workload, requests) -> np.ndarray:
    """FP32 initial state of the given requests: S0, then the workload's
    unquantized warm-up steps (oracle), then the outlier-column gain."""
    c = w.cfg
    S = np.ascontiguousarray(w.initial_state(requests))
    if c.warmup_steps:
        o_ = oracle_for(oracle, w, n_slots=len(requests))
        for t in range(-c.warmup_steps, 0):
            q, k, v, beta, g = w.step_inputs(t, requests)
            o_.step_fp32(S, q, k, v, beta, g, threads=THREADS)
    if c.outlier_frac:
        S *= w.outlier_mask()[None, :, None, :]
    return S


def gpu_warm_state(w: synth.Workload) -> torch.Tensor:
    """FP32 initial state of all B requests computed on the GPU (FP32 kernel)."""
    c = w.cfg
    S = torch.from_numpy(w.initial_state()).cuda()
    if c.warmup_steps:
        fp = gpu_pool_for(w, w.B, _abi.SQ_FMT_FP32)
        o = torch.empty((w.B, c.h_v, c.d), device="cuda")
        for t in range(-c.warmup_steps, 0):
            q, k, v, beta, g = to_dev(*w.step_inputs(t))
            fp.decode_step(S, q, k, v, beta, g, o)
        torch.cuda.synchronize()
        fp.close()
    if c.outlier_frac:
        S *= torch.from_numpy(w.outlier_mask()).cuda()[None, :, None, :]
    return S


@dataclass
class Stats:
    entries: int = 0          # codes / fp16 values compared
    flips: int = 0            # codes or pivot values that differ
    r_flips: int = 0          # row scales that differ (by one fp16 step)
    r_bad: int = 0            # row scales that differ by more than one step
    max_code_diff: int = 0    # in LSB (quantized) or fp16 steps at the row's magnitude (pivots)
    worst_o: float = 0.0
    steps: int = 0
    notes: list = field(default_factory=list)

    def check(self):
        assert self.max_code_diff <= 1, self
        assert self.r_bad == 0, self
        assert self.flips + self.r_flips <= FLIP_RATE * self.entries, self
        assert self.worst_o <= O_TOL, self


def compare_slots(o_: oracle.Oracle, ref: np.ndarray, got: np.ndarray, st: Stats):
    """Compare pools slot by slot (ref/got: uint8 arrays of the same slots)."""
    sb = o_.layout.slot_bytes
    n = ref.size // sb
    d = o_.d
    st.entries += n * o_.h_v * d * d
    if np.array_equal(ref, got):
        return
    for s in range(n):
        a, b = ref[s * sb:(s + 1) * sb], got[s * sb:(s + 1) * sb]
        if np.array_equal(a, b):
            continue
        for h in range(o_.h_v):
            off, nb = o_.layout.head_offset[h], o_.layout.record_bytes[h]
            if np.array_equal(a[off:off + nb], b[off:off + nb]):
                continue
            ca, cb = o_.codes(a, 0, h), o_.codes(b, 0, h)
            ra, rb = o_.row_scales(a, 0, h), o_.row_scales(b, 0, h)
            found = 0
            for i in range(d):
                piv, _ = o_.row_kind(h, i)
                if piv:
                    fa = ca[i].astype(np.uint16).view(np.float16).astype(np.float64)
                    fb = cb[i].astype(np.uint16).view(np.float16).astype(np.float64)
                    diff = np.abs(fa - fb)
                    nflip = int((diff > 0).sum())
                    if nflip:
                        top = np.float16(max(np.abs(fa).max(), np.abs(fb).max()))
                        unit = float(np.spacing(top))
                        st.max_code_diff = max(st.max_code_diff, int(np.ceil(diff.max() / unit)))
                else:
                    dd = np.abs(ca[i] - cb[i])
                    nflip = int((dd > 0).sum())
                    st.max_code_diff = max(st.max_code_diff, int(dd.max()))
                st.flips += nflip
                found += nflip
                if ra[i] != rb[i]:
                    found += 1
                    st.r_flips += 1
                    if abs(int(ra[i]) - int(rb[i])) > 1:
                        st.r_bad += 1
            if len(st.notes) < 6:
                rows = [i for i in range(d) if ra[i] != rb[i] or np.any(ca[i] != cb[i])]
                st.notes.append(f"slot {s} head {h} rows {rows[:4]} kinds {[o_.row_kind(h, i) for i in rows[:2]]}")
            assert found, f"slot {s} head {h}: record differs outside its codes and row scales"


def slot_bytes(pool_t: torch.Tensor, sp: StatePool, slots) -> np.ndarray:
    p = pool_t.view(-1, sp.slot_bytes)
    idx = torch.as_tensor(list(slots), device=p.device, dtype=torch.long)
    return p.index_select(0, idx).cpu().numpy().reshape(-1)


def run_parity(w: synth.Workload, steps: int, check_requests=None, use_gpu_warmup=False, slot_perm=None,
               n_slots=None, layer_inputs=None):
    """Quantize the same FP32 initial state on both sides, then run `steps`
    decode steps. The GPU steps all B requests; the oracle steps the
    requests in `check_requests` (default: all). Returns (Stats, rollout_rel).

    slot_perm: optional [B] int array mapping request -> pool slot on the GPU
    (the oracle keeps its own compact pool)."""
    c = w.cfg
    B = w.B
    reqs = list(range(B)) if check_requests is None else list(check_requests)
    o_ = oracle_for(oracle, w, n_slots=len(reqs))
    n_slots = n_slots or B
    sp = gpu_pool_for(w, n_slots)
    slots = np.arange(B, dtype=np.int32) if slot_perm is None else np.asarray(slot_perm, np.int32)
    slots_t = torch.from_numpy(slots).cuda()
    # ---- initial state
    S_ref = oracle_warm_state(w, reqs)
    if use_gpu_warmup:
        S_gpu = gpu_warm_state(w)
        idx = torch.as_tensor(reqs, device="cuda")
        # the checked requests start from exactly the oracle's fp32 state
        fp_gap = rel_l2(S_gpu.index_select(0, idx).cpu().numpy(), S_ref)
        S_gpu.index_copy_(0, idx, torch.from_numpy(S_ref).cuda())
    else:
        assert len(reqs) == B
        fp_gap = 0.0
        S_gpu = torch.from_numpy(S_ref).cuda()
    pool_ref = o_.new_pool()
    st_q = o_.quantize(pool_ref, S_ref)
    pool = sp.new_pool()
    sp.quantize_state(pool, S_gpu, slots_t)
    torch.cuda.synchronize()
    st_gpu = sp.get_status()
    if len(reqs) == B:
        assert st_gpu == st_q, (st_gpu, st_q)
    del S_gpu
    gslots = slots[reqs]
    stats = Stats()
    got0 = slot_bytes(pool, sp, gslots)
    assert np.array_equal(got0, pool_ref), "quantize_state differs from the oracle"
    init_ref = pool_ref.copy()
    o_dev = torch.empty((B, c.h_v, c.d), device="cuda")
    inputs = layer_inputs or w.step_inputs
    flips_seen = False
    st_all = 0
    for t in range(steps):
        q, k, v, beta, g = inputs(t)
        sp.decode_step(pool, *to_dev(q, k, v, beta, g), o_dev, slots_t)
        sel = np.asarray(reqs)
        o_ref, st_ref = o_.step(pool_ref, q[sel], k[sel], v[sel], beta[sel], g[sel], threads=THREADS)
        st_all |= st_ref
        got = slot_bytes(pool, sp, gslots)
        f0 = stats.flips + stats.r_flips
        compare_slots(o_, pool_ref, got, stats)
        if stats.flips + stats.r_flips != f0:
            flips_seen = True
            # teacher forcing: the GPU continues from the oracle's bytes
            p = pool.view(-1, sp.slot_bytes)
            p[torch.as_tensor(gslots, device="cuda", dtype=torch.long)] = \
                torch.from_numpy(pool_ref.reshape(len(reqs), -1)).cuda()
        o_got = o_dev.cpu().numpy()[sel]
        stats.worst_o = max(stats.worst_o, rel_l2(o_got, o_ref))
        stats.steps += 1
    stats.notes.insert(0, f"fp32 warm-up gap {fp_gap:.3e}")
    st_gpu = sp.get_status()
    if len(reqs) == B:
        assert st_gpu == st_all, (st_gpu, st_all)
    rollout = 0.0
    if flips_seen:
        rollout = free_rollout(w, o_, sp, init_ref, reqs, steps, inputs)
    sp.close()
    return stats, rollout


def free_rollout(w, o_, sp, init_ref, reqs, steps, inputs):
    """Both sides run free from the same bytes; relative Frobenius of the
    dequantized states at the end."""
    c = w.cfg
    n = len(reqs)
    sp2 = gpu_pool_for(w, n)
    pool = torch.from_numpy(init_ref.copy()).cuda()
    ref = init_ref.copy()
    o_dev = torch.empty((n, c.h_v, c.d), device="cuda")
    sel = np.asarray(reqs)
    for t in range(steps):
        q, k, v, beta, g = (x[sel] for x in inputs(t))
        sp2.decode_step(pool, *to_dev(q, k, v, beta, g), o_dev)
        o_.step(ref, q, k, v, beta, g, threads=THREADS)
    S_gpu = torch.empty((n, c.h_v, c.d, c.d), device="cuda")
    sp2.dequantize_state(pool, S_gpu)
    S_ref, _ = o_.dequantize(ref)
    r = rel_l2(S_gpu.cpu().numpy(), S_ref)
    sp2.close()
    return r


def run_parity_device_inputs(w: synth.Workload, steps: int, check_requests, rollout_check=True):
    """run_parity for long rollouts: the GPU steps all B requests with inputs
    drawn on the device (``Workload.step_inputs_device``); the oracle steps
    the requests in `check_requests` on host copies of their rows. Same
    per-step comparison and teacher forcing as run_parity. After the last
    step, returns also the relative Frobenius of the checked requests'
    dequantized states (GPU vs oracle) and, when a flip was seen, of a free
    rollout from the same start."""
    c = w.cfg
    B = w.B
    reqs = list(check_requests)
    sel = np.asarray(reqs)
    sel_t = torch.as_tensor(reqs, device="cuda", dtype=torch.long)
    o_ = oracle_for(oracle, w, n_slots=len(reqs))
    sp = gpu_pool_for(w, B)
    S_ref = oracle_warm_state(w, reqs)
    S_gpu = gpu_warm_state(w)
    S_gpu.index_copy_(0, sel_t, torch.from_numpy(S_ref).cuda())
    pool_ref = o_.new_pool()
    o_.quantize(pool_ref, S_ref)
    pool = sp.new_pool()
    sp.quantize_state(pool, S_gpu)
    torch.cuda.synchronize()
    del S_gpu
    gslots = np.asarray(reqs, np.int32)
    assert np.array_equal(slot_bytes(pool, sp, gslots), pool_ref)
    init_ref = pool_ref.copy()
    o_dev = torch.empty((B, c.h_v, c.d), device="cuda")
    stats = Stats()
    flips_seen = False
    host_inputs = []
    for t in range(steps):
        x = w.step_inputs_device(t)
        sp.decode_step(pool, *x, o_dev)
        xs = [a.index_select(0, sel_t).cpu().numpy() for a in x]
        if rollout_check:
            host_inputs.append(xs)
        o_ref, _ = o_.step(pool_ref, *xs, threads=THREADS)
        got = slot_bytes(pool, sp, gslots)
        f0 = stats.flips + stats.r_flips
        compare_slots(o_, pool_ref, got, stats)
        if stats.flips + stats.r_flips != f0:
            flips_seen = True
            p = pool.view(-1, sp.slot_bytes)
            p[torch.as_tensor(gslots, device="cuda", dtype=torch.long)] = \
                torch.from_numpy(pool_ref.reshape(len(reqs), -1)).cuda()
        stats.worst_o = max(stats.worst_o, rel_l2(o_dev.index_select(0, sel_t).cpu().numpy(), o_ref))
        stats.steps += 1
    # final state of the checked requests: GPU vs oracle (equal unless flips)
    S_g = torch.empty((len(reqs), c.h_v, c.d, c.d), device="cuda")
    sp.dequantize_state(pool, S_g, torch.from_numpy(gslots).cuda())
    S_o, _ = o_.dequantize(pool_ref)
    final = rel_l2(S_g.cpu().numpy(), S_o)
    rollout = 0.0
    if flips_seen and rollout_check:
        n = len(reqs)
        rollout = free_rollout(w, o_, sp, init_ref, list(range(n)), steps, lambda t: host_inputs[t])
    sp.close()
    return stats, final, rollout
