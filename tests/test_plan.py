"""The launch plan (host logic, no GPU): for every workload shape and every
batch size a fused kernel serves the call with a plan that fits the shared
memory it claims.  With the decode-ahead option, batches of 1..8 whose x
fits take that kernel (two CTAs of 9 warps per SM, each within half the SM,
or one CTA of 17 warps taking more than half of it, so that at most two of
its CTAs share an SM's tensor memory); by default, and otherwise, the
others take the 12-warp kernel, whose single-pass launches use the fixed 3-
or 4-stage code ring (its compile-time waits depend on it), and whose
batches above 8 run as one-pass launches of 8 columns when those fit while
the whole batch would need several passes."""
import pytest

import synth
from lut_dequant_gemv_b200 import binding as B

DEV = B.B200_DEVICE
HALF = DEV["smem_per_sm"] // 2 - 1024


def shapes():
    seen = set()
    for name, ss in synth.workloads().items():
        for s in ss:
            if (s.n_out, s.k_in, s.bits) not in seen:
                seen.add((s.n_out, s.k_in, s.bits))
                yield s


@pytest.mark.parametrize("shape", list(shapes()), ids=lambda s: f"{s.n_out}x{s.k_in}b{s.bits}")
def test_every_batch_gets_a_fitting_fused_plan(shape):
    for batch in range(1, 17):
        p = B.sqz_plan_query(shape.n_out, shape.k_in, shape.bits, batch, **DEV)
        assert p["fused"] == 1, (shape.key, batch)
        assert p["grid"] == min(DEV["sm_count"], (shape.n_out + 15) // 16)
        assert p["launches"] * p["columns_per_launch"] >= batch
        assert (p["launches"] - 1) * p["columns_per_launch"] < batch
        assert p["csr_stage_entries"] >= 0 and p["csr_stage_entries"] % 8 == 0
        assert p["predecode"] == 0  # the default: the 12-warp kernel
        assert p["threads"] == 384
        budget = HALF if p["ctas_per_sm"] == 2 else DEV["smem_optin"]
        assert 0 < p["smem_bytes"] <= budget
        if p["passes"] == 1:
            assert p["ring_stages"] in (3, 4)
        else:
            assert p["ring_stages"] >= 2
        if batch == 1:
            assert p["passes"] == 1 and p["launches"] == 1
            assert p["ctas_per_sm"] == 2, "batch 1 must leave room for the next call's CTA"


@pytest.mark.parametrize("shape", list(shapes()), ids=lambda s: f"{s.n_out}x{s.k_in}b{s.bits}")
def test_decode_ahead_plans_fit(shape):
    for batch in range(1, 17):
        p = B.sqz_plan_query(shape.n_out, shape.k_in, shape.bits, batch, **DEV, predecode=1)
        assert p["fused"] == 1, (shape.key, batch)
        if not p["predecode"]:
            continue
        assert batch <= 8
        assert (p["launches"], p["passes"], p["ring_stages"]) == (1, 1, 4)
        assert p["grid"] == min(DEV["sm_count"], (shape.n_out + 15) // 16)
        if p["threads"] == 9 * 32:  # two CTAs of 8 dense warps per SM, half the SM each
            assert p["ctas_per_sm"] == 2 and 0 < p["smem_bytes"] <= HALF
        else:  # one CTA of 16 dense warps, more than half the SM: no second one fits
            assert p["threads"] == 17 * 32 and p["ctas_per_sm"] == 1
            assert DEV["smem_per_sm"] // 2 < p["smem_bytes"] <= DEV["smem_optin"]


def test_decode_ahead_kernel_serves_small_batches_and_never_above_eight():
    for n, k, bits in ((11008, 4096, 3), (4096, 4096, 4), (5120, 13824, 3), (8192, 22016, 3)):
        for batch in range(1, 17):
            p = B.sqz_plan_query(n, k, bits, batch, **DEV, predecode=1)
            if batch > 8:
                assert p["predecode"] == 0
            elif batch == 1 or (batch == 2 and k <= 13824):
                assert p["predecode"] == 1, (n, k, batch)


def test_batch_one_of_every_workload_shape_shares_the_sm_with_the_next_call():
    for shape in shapes():
        p = B.sqz_plan_query(shape.n_out, shape.k_in, shape.bits, 1, **DEV, predecode=1)
        assert p["predecode"] == 1 and p["ctas_per_sm"] == 2, shape.key


def test_large_batches_split_into_single_pass_launches_of_eight():
    # whole batch of 16 would need passes, 8 columns fit one pass: two launches
    for n, k in ((5120, 5120), (13824, 5120), (4096, 4096)):
        p = B.sqz_plan_query(n, k, 3, 16, **DEV)
        assert (p["launches"], p["columns_per_launch"], p["passes"]) == (2, 8, 1), (n, k, p)
    # 8 columns of K = 13824 do not fit one pass: launches of 4 in one pass each
    # (fewer launches than the passes the whole batch would need)
    for batch, launches in ((16, 4), (8, 2)):
        p = B.sqz_plan_query(5120, 13824, 3, batch, **DEV)
        assert (p["launches"], p["columns_per_launch"], p["passes"]) == (launches, 4, 1), (batch, p)
    # 4 columns carry 4 (not 8) batch columns and fit one pass: launches of 4
    # and 1 instead of 3 passes
    p = B.sqz_plan_query(300, 18432, 3, 5, **DEV)
    assert (p["launches"], p["columns_per_launch"], p["passes"]) == (2, 4, 1), p
    # not even one column fits one pass: x staged in K chunks in one launch
    p = B.sqz_plan_query(40, 98304, 4, 2, **DEV)
    assert (p["launches"], p["columns_per_launch"], p["passes"]) == (1, 2, 7), p
    assert B.sqz_plan_query(40, 98304, 4, 1, **DEV)["fused"] == 0


def test_small_batches_keep_two_ctas_per_sm():
    # batches of 2-4 carry 2 or 4 batch columns through the sparse part and the
    # combine (not 8), so their shared memory fits half an SM where x does
    for n, k, batches in ((5120, 5120, (2, 3, 4)), (11008, 4096, (2, 3, 4)), (4096, 4096, (2, 3, 4)),
                          (13824, 5120, (2, 3))):
        for batch in batches:
            p = B.sqz_plan_query(n, k, 3, batch, **DEV)
            assert (p["launches"], p["passes"], p["ctas_per_sm"]) == (1, 1, 2), (n, k, batch, p)
            assert p["smem_bytes"] <= HALF


def test_plan_query_rejects_bad_arguments():
    for args in ((0, 64, 3, 1), (64, 64, 5, 1), (64, 64, 3, 0), (64, 64, 3, 17)):
        with pytest.raises(B.SqzError) as e:
            B.sqz_plan_query(*args, **DEV)
        assert e.value.status == B.SQZ_ERR_INVALID_ARG
    with pytest.raises(B.SqzError):
        B.sqz_plan_query(64, 64, 3, 1, sm_count=0)


def test_very_long_rows_fall_back_to_the_row_kernel():
    # one batch column of x beyond the shared memory of a CTA
    p = B.sqz_plan_query(64, 1 << 17, 4, 1, **DEV)
    assert p["fused"] == 0 and p["launches"] == 0


@pytest.mark.parametrize("seed", range(12))
def test_random_shapes_get_plans_within_their_shared_memory(seed):
    """Random layer shapes and batches, beyond the workloads: a fused plan,
    when there is one, covers the batch, fits the shared memory it claims
    (half an SM when two CTAs share one) and keeps the ring bounds; only a
    batch-1 call whose single column of x cannot fit falls back to the
    row-per-warp kernel, and then so do no larger batches of a shorter K."""
    import numpy as np

    rng = np.random.default_rng(seed)
    for _ in range(40):
        bits = int(rng.choice([3, 4]))
        step = 32 if bits == 3 else 8
        k_in = step * int(rng.integers(1, 120000 // step))
        n_out = int(rng.integers(1, 30000))
        batch = int(rng.integers(1, 17))
        p = B.sqz_plan_query(n_out, k_in, bits, batch, **DEV)
        if not p["fused"]:
            assert batch == 1 and k_in > 40000, (n_out, k_in, bits, batch)
            continue
        assert p["grid"] == min(DEV["sm_count"], (n_out + 15) // 16)
        assert (p["launches"] - 1) * p["columns_per_launch"] < batch <= p["launches"] * p["columns_per_launch"]
        budget = HALF if p["ctas_per_sm"] == 2 else DEV["smem_optin"]
        assert 0 < p["smem_bytes"] <= budget, (n_out, k_in, bits, batch, p)
        assert p["ring_stages"] in (3, 4) if p["passes"] == 1 else p["ring_stages"] >= 2
        assert p["csr_stage_entries"] >= 0 and p["csr_stage_entries"] % 8 == 0
        if batch == 1:
            assert p["passes"] == 1 and p["launches"] == 1, (n_out, k_in, bits)
            if k_in <= 8192:  # x of 16 KB or less: always room for the next call's CTA
                assert p["ctas_per_sm"] == 2, (n_out, k_in, bits)


def test_x_in_k_chunks_only_when_no_column_launches_are_fewer():
    """The planner stages x in K chunks (several passes) only when no split
    of the batch into single-pass launches of 8, 4, 2 or 1 columns gives
    fewer launches than those passes (and, above 8 columns, when 8 columns
    do not fit one pass)."""
    import numpy as np

    rng = np.random.default_rng(7)
    multi = 0
    for _ in range(300):
        bits = int(rng.choice([3, 4]))
        step = 32 if bits == 3 else 8
        k_in = step * int(rng.integers(60000 // step, 140000 // step))
        n_out = int(rng.integers(1, 20000))
        batch = int(rng.integers(2, 17))
        p = B.sqz_plan_query(n_out, k_in, bits, batch, **DEV)
        if not p["fused"] or p["passes"] == 1:
            continue
        multi += 1
        assert p["launches"] == 1 and p["columns_per_launch"] == batch
        for c in (8, 4, 2, 1):
            if c >= batch:
                continue
            q = B.sqz_plan_query(n_out, k_in, bits, c, **DEV)
            one_pass = q["fused"] and q["launches"] == 1 and q["passes"] == 1
            if one_pass:
                assert not (batch > 8 and c == 8), (n_out, k_in, bits, batch)
                assert -(-batch // c) >= p["passes"], (n_out, k_in, bits, batch, c, p)
    assert multi > 20
