"""Host-side helpers of bench.py that feed reported numbers: the count of
visible (query, key) pairs behind the prefill-attention FLOP figure, against
brute force over the causal rule (query i of nq positions over a sequence of L
tokens sees tokens 0 .. L - nq + i)."""
import pytest

import bench
from compressed_space_decode_b200.synthetic import Workload


def brute_pairs(lens, nq):
    n = 0
    for L in lens:
        for i in range(nq):
            for t in range(L):
                if t <= L - nq + i:
                    n += 1
    return n


@pytest.mark.parametrize("lens,nq", [([64], 64), ([100], 7), ([5, 40, 0], 12), ([33], 50), ([1], 1)])
def test_causal_pairs_matches_brute_force(lens, nq):
    wl = Workload("t", len(lens), 4, 1, lens, nq=nq, causal=True)
    assert bench.causal_pairs(wl) == brute_pairs(lens, nq)


def test_causal_pairs_full_prefill_is_the_triangle():
    wl = Workload("t", 1, 32, 8, [32768], nq=32768, causal=True)
    assert bench.causal_pairs(wl) == 32768 * 32769 // 2


def test_stage_layout_views_round_trip():
    """The e2e staging row: aligned, non-overlapping slots whose views give
    back each tensor bit for bit after one byte-level copy."""
    import torch
    import bench
    ts = [torch.randn(3, 5, 7).to(torch.bfloat16), torch.arange(17, dtype=torch.int64),
          torch.arange(5, dtype=torch.int32), torch.randn(2, 128)]
    layout, row = bench.stage_layout(ts)
    ends = [o + n for o, n, _, _ in layout]
    assert all(o % 256 == 0 for o, _, _, _ in layout)
    assert all(ends[i] <= layout[i + 1][0] for i in range(len(ts) - 1)) and ends[-1] <= row
    stage = torch.zeros(row, dtype=torch.uint8)
    for (o, n, dt, shp), t in zip(layout, ts):
        stage[o:o + n].view(dt).view(shp).copy_(t)
    copy = stage.clone()
    for (o, n, dt, shp), t in zip(layout, ts):
        assert torch.equal(copy[o:o + n].view(dt).view(shp), t)


@pytest.mark.parametrize("causal,nq", [(False, 1), (True, 5)])
def test_oracle_step_rows_see_their_prefix(causal, nq):
    """The CPU-baseline sample of a step: with a causal chunk of nq appended
    tokens, position i's rows attend over the first L + i + 1 tokens, so each
    row equals the oracle's attention over that prefix alone."""
    import numpy as np
    import oracle
    wl = Workload("t", 2, 4, 2, [70, 45], nq=nq, page_size=64, causal=causal, seed=5)
    o = bench.oracle_sample(wl, 1, 1, device="cpu")
    assert o["adv"] == (nq if causal else 1) and o["q"].shape == (nq * wl.group, 128)
    out = bench.oracle_step(o)
    kc1, kn1, _, _ = oracle.compress(o["s"], o["qt"], o["newk"])
    vc1, vn1, _, _ = oracle.compress(o["s"], o["qt"], o["newv"])
    kc, kn = np.concatenate([o["kc"], kc1]), np.concatenate([o["kn"], kn1])
    vc, vn = np.concatenate([o["vc"], vc1]), np.concatenate([o["vn"], vn1])
    for r in range(out.shape[0]):
        n = 45 + r // wl.group + 1
        ref = oracle.attend(o["s"], o["qt"], o["q"][r:r + 1], kc[:n], kn[:n], vc[:n], vn[:n], [n])
        assert np.allclose(out[r], ref[0], rtol=0, atol=1e-12 * np.abs(ref).max())


def test_oracle_pools_run_their_samples():
    """The all-core CPU-baseline legs: spawned processes that each run the
    oracle's decode step (or its bulk compression) on the same sample, and
    the counts the bench turns into rates."""
    import numpy as np
    from compressed_space_decode_b200 import synthetic
    wl = Workload("t", 1, 4, 1, [100], nq=1, page_size=64, causal=False, seed=6)
    o = bench.oracle_sample(wl, 0, 0, device="cpu")
    pool = bench.OraclePool(o, 2)
    n, dt = pool.run(steps=2)
    pool.close()
    assert n == 4 and dt > 0
    signs, quats = synthetic.rotation_params(7, 1)
    sample = {"s": signs[0].numpy(), "qt": quats[0].numpy(),
              "x": np.random.default_rng(8).standard_normal((16, 128)), "bits": 3}
    pool = bench.OraclePool(sample, 2, worker=bench._compress_worker)
    n, dt = pool.run(steps=3)
    pool.close()
    assert n == 2 * 3 * 16 and dt > 0


def test_clocks_resample_keeps_a_sampled_region():
    """A timed region that nvidia-smi sampled keeps its own clocks (no
    re-run); only an unsampled one is re-sampled over extra steps."""
    c = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": [], "samples": 3}
    calls = []
    assert bench.clocks_or_resample(c, "GPU-x", lambda: calls.append(1), None) is c
    assert not calls
