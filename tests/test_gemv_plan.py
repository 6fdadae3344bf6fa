"""The GEMV launch plan (host arithmetic only; runs without a GPU).

The shared-memory ring is only correct when a parity wait can never run more
than one phase ahead of its barrier.  The plan guarantees it by giving every
slot a single consumer warp (or a slot per column group, with no refills).
This checks that invariant, the resource limits and the m-independence of the
k split over a grid of shapes, for both launch modes.
"""
import itertools

import pytest

import verify_weight_streaming_b200 as mr

SMS, OPTIN = 148, 232448          # B200: SMs, opt-in shared memory per block


def cta_groups(plan, n):
    g, cg = plan["grid"], plan["columns_per_group"]
    out = []
    for b in range(g):
        ncols = (b + 1) * n // g - b * n // g
        out.append((ncols + cg - 1) // cg)
    return out


@pytest.mark.parametrize("flags", [0, mr.MR_GEMV_PDL])
def test_plan_invariants(flags):
    ms = range(1, 17)
    ns = [1, 7, 147, 148, 149, 512, 1000, 4864, 6144, 30000]
    ks = [8, 64, 136, 896, 1024, 2048, 2560, 4088, 4096]
    for m, n, k in itertools.product(ms, ns, ks):
        p = mr.mrgemv_bf16_plan(m, n, k, flags, SMS, OPTIN)
        assert 1 <= p["grid"] <= min(SMS, n) or (flags and p["grid"] == 2 * SMS <= n)
        if p["grid"] > SMS:
            # two CTAs per SM: each fits half of the SM's shared memory and
            # registers (at most 128 a thread), and only small row buckets split
            assert p["smem_bytes"] <= 110 * 1024 and p["threads"] <= 256 and p["row_bucket"] <= 4
        # 16 warps at most (every kernel is built for 512 threads of <= 128 registers)
        assert p["threads"] == 32 * p["k_warps"] * p["column_warps"] <= 32 * 16
        assert p["smem_bytes"] <= OPTIN
        assert p["row_bucket"] >= m and p["row_bucket"] in (1, 2, 4, 8, 16)
        S, cwg = p["ring_slots"], p["column_warps"]
        assert S >= 1
        for ng in cta_groups(p, n):
            if ng > S:
                # refills happen: slot s must always be consumed by warp s % cwg
                assert S % cwg == 0, (m, n, k, flags, p)
                for g in range(ng):
                    assert (g % S) % cwg == g % cwg


def test_k_split_depends_on_k_only():
    for k in (8, 512, 896, 1024, 2560, 4096):
        kws = {mr.mrgemv_bf16_plan(m, n, k, f, SMS, OPTIN)["k_warps"]
               for m in range(1, 17) for n in (1, 512, 6144) for f in (0, 1)}
        assert len(kws) == 1, (k, kws)


def test_plan_rejects_like_the_entry_point():
    with pytest.raises(mr.MrError) as e:
        mr.mrgemv_bf16_plan(17, 512, 2560, 0, SMS, OPTIN)
    assert e.value.status == mr.MR_ERR_UNSUPPORTED
    with pytest.raises(mr.MrError) as e:
        mr.mrgemv_bf16_plan(4, 512, 2564, 0, SMS, OPTIN)
    assert e.value.status == mr.MR_ERR_MISALIGNED
    with pytest.raises(mr.MrError) as e:
        mr.mrgemv_bf16_plan(16, 512, 1 << 16, 0, SMS, OPTIN)
    assert e.value.status == mr.MR_ERR_UNSUPPORTED


def test_row_buckets():
    """One row runs in its own kernel; then 2, 4, 8 and 16 rows."""
    want = {1: 1, 2: 2, 3: 4, 4: 4, 5: 8, 8: 8, 9: 16, 16: 16}
    for m, mb in want.items():
        for n, k in ((512, 2560), (4864, 896), (6144, 2560)):
            assert mr.mrgemv_bf16_plan(m, n, k, mr.MR_GEMV_PDL, SMS, OPTIN)["row_bucket"] == mb, (m, n, k)

