"""Seeded synthetic inputs for the LLM.int8() matmul workloads.

This module only draws random numbers; it holds none of the method's
arithmetic (no thresholds, scales or rounding of the method).  The tests feed
the same bytes to the CPU oracle and to the CUDA path, and the benchmark uses
the same recipes.

The value distributions follow what the pages say about activations of 7B-70B
models: about 99.9% of activations lie in [-1, 1], while a few fixed feature
dimensions (about 0.1% of them, a few dozen at most) carry values 20-100x larger on
almost every token ('LLM quantization, part 2' (hncyxsy.com) §1; '三、模型量化'
(lowentro.cn) Q4 and Q11).  Weights are zero-mean normal.

All draws are numpy PCG64 (`default_rng(seed)`) in float32, then rounded to
float16 (round to nearest even).  Every workload is a plain dict of numpy
arrays so that neither side depends on torch for its inputs.
"""
from __future__ import annotations

import numpy as np

# name -> shapes and outlier structure.  T may be a tuple (decode sweep).
WORKLOADS = {
    "tiny": dict(T=16, K=256, N=256, w_sigma=0.02, n_dims=2, dims=(7, 100),
                 mag=(20.0, 60.0), presence=1.0, spike_rate=0.0, thresholds=(6.0,)),
    "7b_decode": dict(T=(1, 2, 4, 8, 16), K=4096, N=11008, w_sigma=0.02, n_dims=4,
                      dims=None, mag=(20.0, 100.0), presence=1.0, spike_rate=0.0,
                      thresholds=(6.0,)),
    "7b_prefill": dict(T=2048, K=4096, N=4096, w_sigma=0.02, n_dims=4, dims=None,
                       mag=(20.0, 100.0), presence=1.0, spike_rate=1e-5,
                       spike_mag=(6.5, 20.0), thresholds=(6.0,)),
    "13b_up": dict(T=512, K=5120, N=13824, w_sigma=0.015, n_dims=6, dims=None,
                   mag=(20.0, 100.0), presence=0.8, spike_rate=0.0, thresholds=(6.0,)),
    "70b_up": dict(T=4096, K=8192, N=28672, w_sigma=0.01, n_dims=40, dims=None,
                   mag=(20.0, 150.0), presence=1.0, spike_rate=0.0,
                   thresholds=(4.0, 6.0, float("inf"))),
}


def _normal_f32(rng: np.random.Generator, shape, sigma: float = 1.0) -> np.ndarray:
    a = rng.standard_normal(shape, dtype=np.float32)
    if sigma != 1.0:
        a *= np.float32(sigma)
    return a


def make_activations(T: int, K: int, *, seed: int = 0, n_dims: int = 4, dims=None,
                     mag=(20.0, 100.0), presence: float = 1.0, spike_rate: float = 0.0,
                     spike_mag=(6.5, 20.0)) -> tuple[np.ndarray, np.ndarray]:
    """X fp16 [T, K] ~ N(0,1) with `n_dims` systematic large-magnitude feature dims.

    Each chosen dim gets |x| ~ U[mag] with a random sign on each token, present
    on a token with probability `presence`.  Optional sparse spikes: each
    element independently, with probability `spike_rate`, becomes +-U[spike_mag].
    Returns (X fp16, the systematic dims as int64, ascending).
    """
    rng = np.random.default_rng(seed)
    x = _normal_f32(rng, (T, K))
    if dims is None:
        dims = np.sort(rng.choice(K, size=n_dims, replace=False))
    dims = np.asarray(dims, dtype=np.int64)
    if dims.size:
        m = rng.uniform(mag[0], mag[1], size=(T, dims.size)).astype(np.float32)
        sgn = np.where(rng.random((T, dims.size)) < 0.5, -1.0, 1.0).astype(np.float32)
        keep = rng.random((T, dims.size)) < presence
        cur = x[:, dims]
        x[:, dims] = np.where(keep, sgn * m, cur)
    if spike_rate > 0.0:
        hit = rng.random((T, K)) < spike_rate
        cnt = int(hit.sum())
        if cnt:
            sm = rng.uniform(spike_mag[0], spike_mag[1], size=cnt).astype(np.float32)
            ss = np.where(rng.random(cnt) < 0.5, -1.0, 1.0).astype(np.float32)
            x[hit] = sm * ss
    return x.astype(np.float16), dims


def make_weight(N: int, K: int, *, seed: int = 0, sigma: float = 0.02) -> np.ndarray:
    """W fp16 [N, K] (out-features x in-features) ~ N(0, sigma)."""
    rng = np.random.default_rng(np.random.SeedSequence([seed, 0x5745494748]))
    return _normal_f32(rng, (N, K), sigma).astype(np.float16)


def workload(name: str, *, seed: int = 0, T: int | None = None, layer: int = 0) -> dict:
    """Inputs of a named workload: {'X', 'W', 'dims', 'T', 'K', 'N', 'thresholds'}.

    For the decode sweep, X is drawn once with the largest T and the first `T`
    rows are returned, so every T shares the same fixed outlier dims.  `layer`
    selects an independent weight matrix (distinct seed) of the same shape.
    """
    cfg = WORKLOADS[name]
    Ts = cfg["T"] if isinstance(cfg["T"], tuple) else (cfg["T"],)
    Tmax = max(Ts)
    if T is None:
        T = Tmax
    X, dims = make_activations(Tmax, cfg["K"], seed=seed, n_dims=cfg["n_dims"],
                               dims=cfg["dims"], mag=cfg["mag"], presence=cfg["presence"],
                               spike_rate=cfg["spike_rate"],
                               spike_mag=cfg.get("spike_mag", (6.5, 20.0)))
    X = np.ascontiguousarray(X[:T])
    W = make_weight(cfg["N"], cfg["K"], seed=seed + 1000 * layer, sigma=cfg["w_sigma"])
    return dict(X=X, W=W, dims=dims, T=T, K=cfg["K"], N=cfg["N"],
                thresholds=cfg["thresholds"])


def random_case(T: int, K: int, N: int, *, seed: int, n_dims: int = 3,
                mag=(8.0, 40.0), w_sigma: float = 0.05) -> tuple[np.ndarray, np.ndarray]:
    """A small random (X, W) pair for parity sweeps over odd shapes."""
    X, _ = make_activations(T, K, seed=seed, n_dims=min(n_dims, K), mag=mag)
    W = make_weight(N, K, seed=seed, sigma=w_sigma)
    return X, W
