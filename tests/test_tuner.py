"""Plan overrides and the tuner's host logic on the CPU: the ABI installs, reports and
removes a shape's plan, rejects inadmissible ones, and the workspace size follows; the
search enumerates only plans the library accepts and finds the minimum of a known
cost; the cache round-trips through its file and installs what it holds."""
import os

import pytest

from rank_linear_lora_b200 import lora_linear as L
from rank_linear_lora_b200 import tuner as T

SHAPE = (4096, 4096, 4096, 8)


@pytest.fixture(autouse=True)
def clean():
    yield
    for shape in (SHAPE, (1024, 512, 3000, 32), (2048, 1024, 1024, 64), (640, 256, 512, 16)):
        L.lora_linear_set_plan(*shape, None)


def test_set_get_clear_and_workspace_follows():
    default = L.lora_linear_get_plan(L.OP_BWD, *SHAPE)
    assert default["side_fwd"] == 1 and default["side_bwd"] == 1 and default["dx_overlap"] == 1
    assert default["da_cluster"] == 2  # pairs, beside the dX GEMM's CTA pairs
    n0 = L.lora_linear_workspace_size(L.OP_BWD, *SHAPE)
    L.lora_linear_set_plan(*SHAPE, dict(side_bwd=2, splitk=[0, 8, 16, 16]))
    p = L.lora_linear_get_plan(L.OP_BWD, *SHAPE)
    assert p["side_bwd"] == 2 and p["splitk"][1:] == [8, 16, 16] and p["g_cluster"] == 0
    assert L.lora_linear_workspace_size(L.OP_BWD, *SHAPE) != n0
    # another shape is untouched
    assert L.lora_linear_get_plan(L.OP_BWD, 4096, 4096, 4096, 16)["side_bwd"] == 1
    L.lora_linear_set_plan(*SHAPE, dict(g_cluster=2, g_group=4))
    p = L.lora_linear_get_plan(L.OP_BWD, *SHAPE)
    assert p["side_bwd"] == 1 and (p["g_cluster"], p["g_group"]) == (2, 4)
    L.lora_linear_set_plan(*SHAPE, None)
    assert L.lora_linear_get_plan(L.OP_BWD, *SHAPE) == default
    assert L.lora_linear_workspace_size(L.OP_BWD, *SHAPE) == n0


@pytest.mark.parametrize("bad,status", [
    (dict(side_fwd=3), 1), (dict(xa_cluster=3), 1), (dict(xa_cluster=8), 1), (dict(g_group=7), 1),
    (dict(g_group=-1), 1), (dict(da_cluster=8), 1), (dict(fwd_tail=4), 1), (dict(splitk=[65, 0, 0, 0]), 1),
    (dict(splitk=[0, -1, 0, 0]), 1)])
def test_rejects_out_of_range_fields(bad, status):
    with pytest.raises(L.LoraError) as e:
        L.lora_linear_set_plan(*SHAPE, bad)
    assert e.value.status == status
    assert L.lora_linear_get_plan(L.OP_BWD, *SHAPE)["side_fwd"] == 1  # nothing installed


def test_rejects_side_kernels_beyond_their_ranks():
    with pytest.raises(L.LoraError) as e:
        L.lora_linear_set_plan(2048, 1024, 1024, 64, dict(side_bwd=1))
    assert e.value.status == 3
    with pytest.raises(L.LoraError) as e:
        L.lora_linear_set_plan(1024, 512, 3000, 32, dict(g_group=3))  # 3 * 32 > 64: partials do not fit
    assert e.value.status == 3
    with pytest.raises(L.LoraError):
        L.lora_linear_set_plan(0, 512, 512, 8, dict())  # invalid shape


@pytest.mark.parametrize("r", [8, 16, 32, 64, 128])
def test_every_candidate_is_accepted(r):
    shape = (2048, 1024, 1024, r)
    start = {k: v for k, v in L.lora_linear_get_plan(L.OP_BWD, *shape).items() if k != "splitk"}
    seen = 0
    for field in T.field_options(r):
        for cand in T.candidates_from(start, field, r):
            L.lora_linear_set_plan(*shape, cand)
            assert L.lora_linear_workspace_size(L.OP_BWD, *shape) > 0
            seen += 1
    L.lora_linear_set_plan(*shape, None)
    assert seen >= 8


def test_coordinate_descent_finds_a_separable_minimum():
    want = dict(side_fwd=1, xa_cluster=2, side_bwd=1, g_cluster=4, g_group=2, da_cluster=1, fwd_tail=2,
                dx_overlap=2)

    def cost(p):
        return sum(abs(p[k] - v) for k, v in want.items())
    start = dict(side_fwd=1, xa_cluster=4, side_bwd=1, g_cluster=1, g_group=1, da_cluster=2, fwd_tail=1,
                 dx_overlap=1)
    best, c, tried = T.coordinate_descent(start, 16, cost)
    assert best == want and c == 0 and len(tried) > 8


def test_cache_round_trip_and_apply(tmp_path):
    path = os.path.join(tmp_path, "plans.json")
    cache = T.PlanCache(path)
    plan = dict(side_fwd=1, xa_cluster=2, side_bwd=1, g_cluster=2, g_group=2, da_cluster=1, fwd_tail=1,
                dx_overlap=2)
    cache.put("devA", 640, 256, 512, 16, "bf16", {"plan": plan, "us": 12.5, "default_us": 13.0})
    cache.put("devB", 640, 256, 512, 16, "bf16", {"plan": dict(side_fwd=2), "us": 9.0})
    cache.save()
    again = T.PlanCache(path)
    assert again.get("devA", 640, 256, 512, 16, "bf16")["plan"] == plan
    assert again.get("devA", 640, 256, 512, 16, "fp8") is None
    assert again.apply("devA") == 1
    got = L.lora_linear_get_plan(L.OP_BWD, 640, 256, 512, 16)
    assert (got["xa_cluster"], got["g_cluster"], got["g_group"], got["dx_overlap"]) == (2, 2, 2, 2)
