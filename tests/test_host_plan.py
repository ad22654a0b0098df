"""Schedule of the host-buffer step (Fp8AmaxStep.host_plan), on CPU: which
linear goes first and last, in which order each linear's inputs arrive and in
which order its passes run.  Only the shapes matter, so the linears are
stand-ins with the attributes the planner reads."""
from types import SimpleNamespace

from fp8_tensor_scaled_b200.layer import Fp8AmaxLinear as L, Fp8AmaxStep

import workloads


def _plan(shapes, backward=True):
    step = Fp8AmaxStep.__new__(Fp8AmaxStep)
    step.linears = [SimpleNamespace(T=T, inf=i, outf=o, backward=backward) for T, i, o in shapes]
    return step.host_plan()


def test_llama70b_projections():
    cfg = workloads.C3
    plan = _plan([(cfg.tokens, l.in_features, l.out_features) for l in cfg.linears])
    # QKV needs the fewest input bytes for its first pass (dY + X = 151 M
    # elements): it goes first; gate, up and down all leave a 302 M-element
    # tail, and the last of them (down) goes last
    assert [p[0] for p in plan] == [0, 1, 2, 3]
    qkv, gate, up, down = plan
    # QKV: X and W each feed 151 M output elements, dY too; ties -> W last,
    # so wgrad (dY, X) runs first
    assert qkv[1] == (L.DY, L.X, L.W) and qkv[2][0] == L.WGRAD
    # gate: W last (its dependents Y + dX are 302 M; X's would be 470 M)
    assert gate[1][-1] == L.W and gate[2][0] == L.WGRAD
    # down: X last (Y + dW = 302 M; dY's dependents dX + dW would be 470 M)
    assert down[1] == (L.DY, L.W, L.X) and down[2][0] == L.DGRAD


def test_every_linear_once_and_consistent():
    shapes = [(256, 384, 512), (256, 128, 256), (256, 512, 384), (64, 4096, 128)]
    plan = _plan(shapes)
    assert sorted(p[0] for p in plan) == list(range(len(shapes)))
    for _, arrival, passes in plan:
        assert sorted(arrival) == [L.X, L.W, L.DY]
        assert sorted(passes) == [L.FWD, L.DGRAD, L.WGRAD]
        # the first pass needs only the first two inputs to arrive
        assert set(L.PASS_INPUTS[passes[0]]) == set(arrival[:2])


def test_forward_only_linears():
    plan = _plan([(128, 256, 256), (16, 64, 64)], backward=False)
    assert [p[0] for p in plan] == [1, 0]
    for _, arrival, passes in plan:
        assert arrival == (L.W, L.X) and passes == (L.FWD,)
