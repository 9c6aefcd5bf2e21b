"""Plans on the GPU: every element of the layer's outputs meets the oracle's bounds under
plans the tuner may install (each field away from the library's choice), and a tuning
run installs a plan no slower than the library's own."""
import pytest

from lora_cases import compare_every_element, DeviceLayer
from rank_linear_lora_b200 import inputs
from rank_linear_lora_b200 import lora_linear as L
from rank_linear_lora_b200 import tuner as T

pytestmark = pytest.mark.gpu

SHAPE = (1536, 1024, 2304, 16)
PLANS = [
    dict(side_fwd=2, side_bwd=2),                                  # split-K everywhere
    dict(side_bwd=2, splitk=[3, 5, 7, 9]),                        # odd split counts
    dict(xa_cluster=1, g_cluster=1, g_group=4, da_cluster=1),       # no clusters, 4 token blocks per round
    dict(xa_cluster=2, g_cluster=2, g_group=3, da_cluster=2),
    dict(xa_cluster=4, g_cluster=4, g_group=2),
    dict(fwd_tail=2, dx_overlap=2),                                 # tails whole forward, dA after dX
]


@pytest.fixture(autouse=True)
def clean():
    yield
    L.lora_linear_set_plan(*SHAPE, None)


@pytest.mark.parametrize("plan", PLANS, ids=lambda p: "-".join(f"{k}{v}" for k, v in p.items()))
def test_plan_every_element(plan):
    M, di, do, r = SHAPE
    L.lora_linear_set_plan(*SHAPE, plan)
    spec = inputs.LayerSpec("plan", M, di, do, r, alpha=32.0, seed=0x7A + di)
    inp = inputs.make_inputs(spec)
    dl = DeviceLayer(inp)  # workspaces sized for the plan now in effect
    dl.forward()
    dl.backward()
    dl.check()
    compare_every_element(dl, inp)


def test_tune_installs_a_plan_no_slower_than_the_default():
    res = T.tune(*SHAPE, reps=5, rounds=3)
    assert res["us"] is not None and res["default_us"] is not None
    assert res["us"] <= res["default_us"]
    assert len(res["tried"]) >= 8
    got = L.lora_linear_get_plan(L.OP_BWD, *SHAPE)
    assert all(got[k] == v for k, v in res["plan"].items() if k != "splitk" and T._applies(k, res["plan"]))
    print("tuned:", res["plan"], f"{res['us']:.1f} us vs default {res['default_us']:.1f} us")
