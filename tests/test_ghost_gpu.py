"""The ghost-norm path (grape_set_norm_method(GRAPE_NORM_GHOST)) through the C ABI (needs a
B200): whole steps against the fp64 oracle, the ghost norms against the direct ones on the
same inputs, and the configurations it refuses."""
import numpy as np
import pytest

import oracle.grape_oracle as O
import workloads as W
from harness import compare, rel_fro, snapshot, to_device

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")

from random_gradient_projection_b200 import GrapeError, GrapeStep, grape  # noqa: E402

SIMT, TC = grape.GRAPE_PATH_SIMT, grape.GRAPE_PATH_TC
GHOST, DIRECT = grape.GRAPE_NORM_GHOST, grape.GRAPE_NORM_DIRECT

CASES = {
    "mlp_2x1024_B4_T128": (W.scaled(W.get("mlp4x1024"), n_layers=2, B=4), 3),
    "vit_shapes_r256_T100": (W.scaled(W.get("vit_b"), layers=((768, 2304), (3072, 768)), B=3, T=100), 2),
    "r512_T64": (W.scaled(W.get("llm7b_slice"), layers=((512, 1024), (1024, 512 * 2)), r=512, B=2, T=64), 2),
    "T1_B3": (W.scaled(W.get("mlp4x1024"), n_layers=2, B=3, T=1), 2),
    # past one 128-token block: the Gram blocks (0,0), (0,1), (1,1), ragged T
    "vit_shapes_r256_T197": (W.scaled(W.get("vit_b"), layers=((768, 2304), (3072, 768)), B=2, T=197), 2),
    # three blocks (six Gram block pairs), the last one 44 tokens long, r = 512
    "r512_T300": (W.scaled(W.get("llm7b_slice"), layers=((512, 1024),), r=512, B=2, T=300), 2),
}


def _run(w, steps, method):
    g = GrapeStep.for_workload(w, path=TC)
    g.set_norm_method(method)
    Ws = [torch.from_numpy(x).cuda() for x in W.make_weights(w)]
    trace = []
    for s in range(steps):
        x = W.make_step_inputs(w, s, threads=8)
        A = [to_device(a, w.dtype) for a in x.A]
        G = [to_device(a, w.dtype) for a in x.Gout]
        g.step(A, G, Ws, s)
        torch.cuda.synchronize()
        trace.append(snapshot(g, w.n_layers))
    out = {"trace": trace, "W": [t.cpu().numpy() for t in Ws]}
    g.close()
    return out


@pytest.mark.parametrize("case", sorted(CASES))
def test_ghost_step_matches_oracle(case):
    w, steps = CASES[case]
    lib = _run(w, steps, GHOST)
    res = O.run(w, steps)
    worst = compare(w, lib, {"trace": res["trace"], "state": res["state"]}, 2e-2, steps)
    print(case, {k: f"{v:.2e}" for k, v in worst.items()})


@pytest.mark.parametrize("case", ["mlp_2x1024_B4_T128", "vit_shapes_r256_T100", "vit_shapes_r256_T197", "r512_T300"])
def test_ghost_norms_equal_direct_norms(case):
    w, _ = CASES[case]
    x = W.make_step_inputs(w, 0, threads=8)
    A = [to_device(a, w.dtype) for a in x.A]
    G = [to_device(a, w.dtype) for a in x.Gout]
    got = {}
    for method in (DIRECT, GHOST):
        g = GrapeStep.for_workload(w, path=TC)
        g.set_norm_method(method)
        got[method] = g.sqnorms(A, G, 0).cpu().numpy().astype(np.float64)
        g.close()
    err = rel_fro(got[GHOST], got[DIRECT])
    # oracle ghost identity on the same fp64 inputs, sample 0, every layer
    h = O.Hyper.of(w)
    ref0 = sum(O.ghost_sqnorm(x.as_f64(x.A[l])[0] @ O.projection_matrix(h.seed, l, 0, w.layers[l][0], w.r),
                              x.as_f64(x.Gout[l])[0]) for l in range(w.n_layers))
    print(case, f"ghost vs direct {err:.2e}; sample 0 vs oracle ghost {abs(got[GHOST][0] / ref0 - 1):.2e}")
    assert err <= 1e-2
    assert abs(got[GHOST][0] / ref0 - 1) <= 2e-2


def test_ghost_refusals():
    long_t = W.scaled(W.get("mlp4x1024"), n_layers=1, B=2, T=129)
    g = GrapeStep.for_workload(long_t, path=TC)
    g.set_norm_method(GHOST)      # any T: the Grams are taken in 128-token blocks
    g.set_norm_method(DIRECT)
    with pytest.raises(GrapeError) as e:
        g.set_norm_method(7)
    assert e.value.code == grape.GRAPE_EINVAL
    g.close()
    g = GrapeStep.for_workload(W.scaled(W.get("mlp4x1024"), n_layers=1, B=2, T=16), path=SIMT)
    with pytest.raises(GrapeError) as e:
        g.set_norm_method(GHOST)
    assert e.value.code == grape.GRAPE_EUNSUPPORTED
    g.close()
