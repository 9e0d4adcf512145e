"""The seeded inputs follow the stated recipes: shapes, fp16 values, the
spread of the regular activations and of the weights, the systematic outlier
dims (count, magnitude range, presence per token), the sparse spikes, and the
outlier-set sizes the oracle finds at each workload's thresholds."""
import numpy as np
import pytest

from int8_mixed_precision_outlier_b200 import synth

# |O| the oracle finds on each workload (seed 0), per threshold
OUTLIER_COUNTS = {"tiny": {6.0: 2}, "7b_decode": {6.0: 4}, "7b_prefill": {6.0: 91},
                  "13b_up": {6.0: 6}, "70b_up": {4.0: 1888, 6.0: 40, float("inf"): 0}}


W_ROWS = 256  # weight statistics use the first rows: the draw is row-major, so they are a prefix


def _parts(name):
    """The recipe's X (all rows) and the first W_ROWS rows of its W, drawn the
    way workload() draws them."""
    cfg = synth.WORKLOADS[name]
    T = max(cfg["T"]) if isinstance(cfg["T"], tuple) else cfg["T"]
    X, dims = synth.make_activations(T, cfg["K"], seed=0, n_dims=cfg["n_dims"], dims=cfg["dims"],
                                     mag=cfg["mag"], presence=cfg["presence"],
                                     spike_rate=cfg["spike_rate"],
                                     spike_mag=cfg.get("spike_mag", (6.5, 20.0)))
    W = synth.make_weight(W_ROWS, cfg["K"], seed=0, sigma=cfg["w_sigma"])
    return dict(X=X, dims=dims, W=W)


@pytest.fixture(scope="module", params=sorted(synth.WORKLOADS))
def wl(request):
    return request.param, synth.WORKLOADS[request.param], _parts(request.param)


@pytest.mark.parametrize("name", ["tiny", "7b_prefill", "7b_decode"])
def test_workload_is_its_recipe(name):
    """workload() returns exactly the recipe's draws, at the full shapes (the
    larger workloads take the same code path)."""
    cfg = synth.WORKLOADS[name]
    w, p = synth.workload(name), _parts(name)
    assert np.array_equal(w["X"], p["X"]) and np.array_equal(w["dims"], p["dims"])
    assert w["W"].shape == (cfg["N"], cfg["K"]) and w["W"].dtype == np.float16
    assert np.array_equal(w["W"][:W_ROWS], p["W"])
    assert w["X"].flags.c_contiguous and w["W"].flags.c_contiguous


def test_shapes_and_types(wl):
    name, cfg, w = wl
    T = max(cfg["T"]) if isinstance(cfg["T"], tuple) else cfg["T"]
    assert w["X"].shape == (T, cfg["K"]) and w["X"].dtype == np.float16
    assert w["W"].dtype == np.float16
    assert np.isfinite(w["X"].astype(np.float32)).all()


def test_value_distributions(wl):
    name, cfg, w = wl
    X = w["X"].astype(np.float64)
    regular = np.delete(X, w["dims"], axis=1)
    if cfg["spike_rate"]:
        regular = regular[np.abs(regular) < 6.0]
    assert abs(regular.mean()) < 0.02 and abs(regular.std() - 1.0) < 0.02
    Wf = w["W"].reshape(-1).astype(np.float64)
    assert abs(Wf.mean()) < 0.1 * cfg["w_sigma"]
    assert abs(Wf.std() / cfg["w_sigma"] - 1.0) < 0.01


def test_systematic_outlier_dims(wl):
    name, cfg, w = wl
    dims = w["dims"]
    assert dims.size == cfg["n_dims"] and np.all(np.diff(dims) > 0)
    if cfg["dims"] is not None:
        assert dims.tolist() == list(cfg["dims"])
    big = np.abs(w["X"][:, dims].astype(np.float32))
    present = big >= np.float32(cfg["mag"][0]) * np.float32(0.999)  # fp16 rounding of the draw
    assert big.max() <= cfg["mag"][1] * 1.001
    frac = present.mean()
    if cfg["presence"] == 1.0:
        assert present.all()
    else:  # present on a token with probability `presence`; absent ones are N(0,1)
        assert abs(frac - cfg["presence"]) < 0.03
    # both signs occur
    vals = w["X"][:, dims].astype(np.float32)[present]
    assert (vals > 0).mean() > 0.4 and (vals < 0).mean() > 0.4


def test_sparse_spikes(wl):
    name, cfg, w = wl
    if not cfg["spike_rate"]:
        pytest.skip("no spikes in this recipe")
    X = np.delete(w["X"], w["dims"], axis=1).astype(np.float32)
    spikes = np.abs(X) >= cfg["spike_mag"][0] * 0.999
    n = X.size
    expect = cfg["spike_rate"] * n
    assert abs(spikes.sum() - expect) < 5 * np.sqrt(expect)
    assert np.abs(X[spikes]).max() <= cfg["spike_mag"][1] * 1.001


def test_outlier_set_sizes(wl, oracle):
    name, cfg, w = wl
    for tau, count in OUTLIER_COUNTS[name].items():
        assert oracle.compact(oracle.detect_outliers(w["X"], tau)).size == count, (name, tau)
    # the systematic dims are always outliers at 6.0
    idx = oracle.compact(oracle.detect_outliers(w["X"], 6.0))
    assert set(w["dims"].tolist()) <= set(idx.tolist())


def test_decode_layers_share_x_rows_and_differ_in_w():
    a = synth.workload("7b_decode", T=4, layer=0)
    b = synth.workload("7b_decode", T=16, layer=1)
    assert np.array_equal(a["X"], b["X"][:4]) and a["dims"].tolist() == b["dims"].tolist()
    assert not np.array_equal(a["W"][:4], b["W"][:4])
