"""GPU: the packed step's S^T k is the exact value rounded once, on columns
built to sit next to fp32 rounding boundaries.

The probe tiles of tests/probe_columns.py make o_j = -P_j exactly, so the
o written by sq_decode_step shows each column's rounded S^T k bit for bit.
Their columns lie 2^-30 .. 2^-44 (relative) from a rounding midpoint, or
exactly on one, with rows of large weight that cancel exactly: an fp64
summation cannot round them with certainty, so these tiles make the kernel
take its exact fixed-point path (counted by sq_get_exact_count), while the
other columns are rounded from the certified fp64 total. Every o must equal
the exact rounding computed here in Python integers and the oracle's o, and
the whole updated state must equal the oracle's byte for byte. Heads of
uniform width (8-bit and 4-bit), all-pivot heads (read and written in place
in the pool), and KDA heads with mixed widths and pivot rows; d = 32, 64,
128; several requests in permuted slots."""
import numpy as np
import pytest
import torch

import oracle
from quantized_linear_attention_sq_b200.state import StatePool
from tests import probe_columns as pc

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from quantized_linear_attention_sq_b200 import build
    build.build()
    torch.cuda.init()


def _run(probes_per_req, gate_kind, slots):
    """probes_per_req[b] = list of probes (one per head) of request b."""
    B = len(probes_per_req)
    h = len(probes_per_req[0])
    d = probes_per_req[0][0].d
    bits, piv, col, phi = pc.calib_for(probes_per_req[0], gate_kind)
    n_slots = max(slots) + 2
    orc = oracle.Oracle(n_slots, h, h, d, gate_kind, bits, piv, col, phi)
    pool = orc.new_pool()
    for b, probes in enumerate(probes_per_req):
        for hh, p in enumerate(probes):
            pc.write_record(orc, pool, slots[b], hh, p)
    ins = [pc.inputs_for(probes, gate_kind) for probes in probes_per_req]
    q, k, v, beta, g = (np.concatenate([x[i] for x in ins]) for i in range(5))
    sp = StatePool(n_slots, h, h, d, gate_kind, 1, bits, piv, col, phi)
    assert sp.pool_bytes == orc.pool_bytes
    dpool = torch.from_numpy(pool.copy()).cuda()
    dq, dk, dv, dbeta, dg = (torch.from_numpy(np.ascontiguousarray(x)).cuda() for x in (q, k, v, beta, g))
    do = torch.full((B, h, d), np.nan, device="cuda")
    sl = np.array(slots, np.int32)
    sp.exact_count(clear=True)
    sp.decode_step(dpool, dq, dk, dv, dbeta, dg, do, torch.from_numpy(sl).cuda())
    torch.cuda.synchronize()
    got_o = do.cpu().numpy()
    n_exact = sp.exact_count()
    st = sp.get_status()
    ref_o, ref_st = orc.step(pool, q, k, v, beta, g, slots=sl)
    got_pool = dpool.cpu().numpy()
    sp.close()
    return got_o, got_pool, ref_o, pool, n_exact, st, ref_st


@pytest.mark.parametrize("d", [32, 64, 128])
def test_gdn_probe_columns_exact(d):
    rng = np.random.default_rng(900 + d)
    reqs = []
    for b in range(3):
        reqs.append([pc.near_probe(rng, d, widths=(8,), cancel=min(4, d // 8)),
                     pc.near_probe(rng, d, widths=(4,)),
                     pc.tie_probe(rng, d, width=8),
                     pc.near_probe(rng, d, all_pivot=True, cancel=2)])
    # one calibration per pool: every request uses the widths of request 0
    for b in range(1, 3):
        reqs[b][1].width[:] = 4
    got_o, got_pool, ref_o, ref_pool, n_exact, st, ref_st = _run(reqs, 0, slots=[4, 0, 2])
    assert st == ref_st == 0
    for b, probes in enumerate(reqs):
        for hh, p in enumerate(probes):
            want = p.expected_o()
            assert np.array_equal(got_o[b, hh], want), (b, hh, np.nonzero(got_o[b, hh] != want))
            assert np.array_equal(ref_o[b, hh], want), (b, hh)
    assert np.array_equal(got_pool, ref_pool)
    assert n_exact > 0  # the boundary columns took the exact path
    print(f"\n[d={d}] exact-path columns: {n_exact} of {3 * 4 * d}")


@pytest.mark.parametrize("d", [64, 128])
def test_kda_probe_columns_exact(d):
    rng = np.random.default_rng(950 + d)
    reqs = []
    for b in range(2):
        reqs.append([pc.near_probe(rng, d, widths=(2, 4, 6, 8), pivot_rows=(1, 5, 9), fine_width=2, cancel=3),
                     pc.tie_probe(rng, d, width=2)])
    # one calibration per pool: request 1 takes request 0's row kinds
    for hh in range(2):
        p0, p1 = reqs[0][hh], reqs[1][hh]
        same = (p0.width == p1.width).all() and (p0.pivot == p1.pivot).all()
        if not same:
            reqs[1][hh] = reqs[0][hh]
    got_o, got_pool, ref_o, ref_pool, n_exact, st, ref_st = _run(reqs, 1, slots=[1, 3])
    assert st == ref_st == 0
    for b, probes in enumerate(reqs):
        for hh, p in enumerate(probes):
            want = p.expected_o()
            assert np.array_equal(got_o[b, hh], want), (b, hh, np.nonzero(got_o[b, hh] != want))
    assert np.array_equal(got_pool, ref_pool)
    assert n_exact > 0
