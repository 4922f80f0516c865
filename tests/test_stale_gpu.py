"""GPU parity of PCPP with stale neighbour rows (two K/V sources) against the
float64 oracle: own-strip keys from the current K/V, borrowed rows from the
previous step's (PCPP review, "Core claim")."""
import numpy as np
import pytest

import oracle
from workloads import PRESETS, Workload, f64_to_bf16_bits, make_inputs
from _parity import compare, log_metrics, passes, to_device, to_f64

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from patch_res_diffusion_b200 import build
    build.build()
    import patch_res_diffusion_b200 as npa
    npa.lib()
    yield
    assert npa.npa_device_status() == npa.NPA_OK


def stale_inputs(w: Workload):
    inp = make_inputs(w)
    st = make_inputs(w, seed=w.seed + 100)
    inp["ks"], inp["vs"] = st["k"], st["v"]
    return inp


def run_gpu(w, inp, strips=None):
    import patch_res_diffusion_b200 as npa
    dv = {n: to_device(inp[n]) for n in ("q", "k", "v", "ks", "vs")}
    gk = to_device(inp["gk"]) if w.G else None
    gv = to_device(inp["gv"]) if w.G else None
    o = torch.full_like(dv["q"], float("nan"))
    npa.pcpp_attention_stale(dv["q"], dv["k"], dv["v"], dv["ks"], dv["vs"], w.H, w.W, w.n_strips, w.p,
                             strips=strips, global_k=gk, global_v=gv, out=o)
    return o


def run_oracle(w, inp, queries=None):
    return oracle.pcpp_attention_stale(inp["q"], inp["k"], inp["v"], inp["ks"], inp["vs"], gk=inp.get("gk"),
                                       gv=inp.get("gv"), G=w.G, B=w.B, heads=w.heads, H=w.H, W=w.W, d=w.d,
                                       n_strips=w.n_strips, p=w.p, queries=queries)


CASES = [
    Workload("stale_4x16", "pcpp", B=1, heads=2, H=64, W=64, d=64, n_strips=4, p=0.3),
    Workload("stale_w96_rows4", "pcpp", B=1, heads=2, H=48, W=96, d=64, n_strips=3, p=0.5),
    Workload("stale_r3_kr2", "pcpp", B=2, heads=1, H=40, W=64, d=64, n_strips=4, p=0.25),
    Workload("stale_w200", "pcpp", B=1, heads=1, H=32, W=200, d=64, n_strips=4, p=0.25),
    Workload("stale_d128_global", "pcpp", B=1, heads=2, H=64, W=64, d=128, n_strips=4, p=0.3, G=77),
    Workload("stale_p1_two", "pcpp", B=1, heads=1, H=32, W=64, d=64, n_strips=2, p=1.0),
    Workload("stale_p0", "pcpp", B=1, heads=1, H=32, W=64, d=64, n_strips=4, p=0.0),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_stale_full_parity(w):
    inp = stale_inputs(w)
    m = compare(to_f64(run_gpu(w, inp)), run_oracle(w, inp))
    log_metrics("stale " + w.name, m)
    assert passes(m), m


@pytest.mark.parametrize("begin,count", [(0, 1), (1, 2), (3, 1)])
def test_strip_range(begin, count):
    w = CASES[0]
    inp = stale_inputs(w)
    got = to_f64(run_gpu(w, inp, strips=(begin, count)))
    ref = run_oracle(w, inp)
    s = w.H // w.n_strips * w.W
    sel = slice(begin * s, (begin + count) * s)
    m = compare(got[:, :, sel], ref[:, :, sel])
    assert passes(m), m
    rest = np.ones(w.H * w.W, dtype=bool)
    rest[sel] = False
    assert np.isnan(got[:, :, rest]).all()   # strips outside the range are not written


def test_stale_probe_sources_exact():
    """q = 0, current values one-hot x1, stale values one-hot x3 on 64 probe
    keys: o[t, c] is 0, 1/|S(t)| or 3/|S(t)| by membership and source."""
    w = Workload("stale_probe", "pcpp", B=1, heads=1, H=48, W=40, d=64, n_strips=3, p=0.4)
    N = w.H * w.W
    rng = np.random.default_rng(7)
    keys = sorted(set([0, N - 1] + [r * w.W + c for r in (15, 16, 31, 32, 10, 21, 37, 26) for c in (0, 19, 39)]))
    while len(keys) < 64:
        keys.append(int(rng.integers(N)))
    keys = keys[:64]
    v = np.zeros((1, 1, N, 64))
    vs = np.zeros((1, 1, N, 64))
    for c, j in enumerate(keys):
        v[0, 0, j, c] = 1.0
        vs[0, 0, j, c] = 3.0
    inp = {"q": np.zeros((1, 1, N, 64), dtype=np.uint16),
           "k": f64_to_bf16_bits(rng.standard_normal((1, 1, N, 64))),
           "ks": f64_to_bf16_bits(rng.standard_normal((1, 1, N, 64))),
           "v": f64_to_bf16_bits(v), "vs": f64_to_bf16_bits(vs)}
    o = to_f64(run_gpu(w, inp))[0, 0]
    s = w.H // w.n_strips
    for t in range(N):
        S = set(oracle.pcpp_key_set(w.H, w.W, w.n_strips, w.p, t).tolist())
        for c, j in enumerate(keys):
            if j not in S:
                assert o[t, c] == 0.0, (t, j)
            else:
                scale = 1.0 if (j // w.W) // s == (t // w.W) // s else 3.0
                assert abs(o[t, c] * len(S) / scale - 1.0) < 1e-2, (t, j, o[t, c])


@pytest.mark.parametrize("name", ["pcpp_4x32_p0.3", "pcpp_8x16_p0.8"])
def test_stale_full_workload_every_row(name):
    w = PRESETS[name]
    inp = stale_inputs(w)
    m = compare(to_f64(run_gpu(w, inp)), run_oracle(w, inp))
    log_metrics("stale " + name + " (every row)", m)
    assert passes(m), m


def _random_stale(n, seed=77):
    rng = np.random.default_rng(seed)
    out = []
    for i in range(n):
        H = int(rng.integers(4, 64))
        divisors = [s for s in range(1, H + 1) if H % s == 0 and H // s >= 1]
        n_strips = int(rng.choice(divisors))
        begin = int(rng.integers(0, n_strips))
        count = int(rng.integers(1, n_strips - begin + 1))
        w = Workload(f"rand_stale_{i}", "pcpp", B=int(rng.integers(1, 3)), heads=int(rng.integers(1, 3)), H=H,
                     W=int(rng.integers(3, 100)), d=int(rng.choice([64, 128])), n_strips=n_strips,
                     p=float(rng.choice([0.0, 0.2, 0.5, 1.0])), G=int(rng.choice([0, int(rng.integers(1, 90))])),
                     seed=i)
        out.append((w, (begin, count)))
    return out


@pytest.mark.parametrize("case", _random_stale(12), ids=lambda c: c[0].name)
def test_random_stale_strip_ranges(case):
    """Seeded random two-source geometries and strip ranges: the computed
    strips match the oracle, the others are left untouched."""
    w, (begin, count) = case
    inp = stale_inputs(w)
    got = to_f64(run_gpu(w, inp, strips=(begin, count)))
    ref = run_oracle(w, inp)
    s = w.H // w.n_strips * w.W
    sel = slice(begin * s, (begin + count) * s)
    m = compare(got[:, :, sel], ref[:, :, sel])
    log_metrics("random " + w.name, m)
    assert passes(m), (w, begin, count, m)
    rest = np.ones(w.H * w.W, dtype=bool)
    rest[sel] = False
    assert np.isnan(got[:, :, rest]).all()
