"""Synthetic quality report: TurboQuant against naive uniform rounding.

The claim checked ([TQ-RS] "TurboQuant : compresser le KV-cache…", the paragraph
after "Étape 2 : Quantification Lloyd-Max optimale"): TurboQuant at 3 bits does
better than naive rounding at 4 bits, where naive means rounding every value to
the nearest point of a uniform grid (the page's "en arrondissant chaque valeur
au plus proche dans une grille uniforme").  READING of the naive grid: per
vector, the strongest common form, the min-max grid of 2^b levels; the
symmetric abs-max grid is reported beside it.

Metrics on seeded vectors of the workloads' laws (no dataset):
  mse  mean over vectors of ||x - x_hat||^2 / ||x||^2
  ip   mean over (q, x) of (<q, x> - <q, x_hat>)^2 / mean <q, x>^2, q ~ N(0, I/d)
TurboQuant at b bits here is the MSE quantizer (values; keys in MSE mode); "tq3
prod" is the key mode of the 3-bit setting (2-bit codes + 1-bit QJL), whose
inner products are unbiased but not minimal.  Numbers go to the session's
summary; the test asserts the claim where it holds on these laws and pins the
case where it does not (isotropic Gaussian data, where a per-vector uniform grid
already fits well).
"""
import math

import numpy as np
import pytest

from parity import record

D = 128
N = 3000


def naive_minmax(x, b):
    lo = x.min(1, keepdims=True)
    hi = x.max(1, keepdims=True)
    step = (hi - lo) / ((1 << b) - 1)
    return lo + np.round((x - lo) / step) * step


def naive_absmax(x, b):
    step = np.abs(x).max(1, keepdims=True) / ((1 << (b - 1)) - 1)
    return np.round(x / step) * step


def _metrics(x, xh, q):
    mse = float(np.mean(np.sum((x - xh) ** 2, 1) / np.sum(x ** 2, 1)))
    ip = float(np.mean(np.sum(q * (x - xh), 1) ** 2) / np.mean(np.sum(q * x, 1) ** 2))
    return mse, ip


def _vectors(law, kind):
    from kv_cache_vector_02_b200 import workloads as W
    w = W.WORKLOADS[law].with_(B=1, T=N, layers=1, decode_steps=0)
    x = W.gen_kv(w, kind).numpy().reshape(-1, D)[:N].astype(np.float64)
    q = np.random.default_rng([11, kind]).standard_normal(x.shape) / math.sqrt(D)
    return x, q


def report(orc, law, kind, tq_fn):
    """tq_fn(bits, key_mode_kind, x) -> x_hat for TurboQuant; returns the metric table."""
    x, q = _vectors(law, kind)
    rows = {}
    for b in (3, 4):
        rows["tq%d" % b] = _metrics(x, tq_fn(b, "mse", x), q)
        rows["naive minmax %d" % b] = _metrics(x, naive_minmax(x, b), q)
        rows["naive absmax %d" % b] = _metrics(x, naive_absmax(x, b), q)
    rows["tq3 prod"] = _metrics(x, tq_fn(3, "prod", x), q)
    label = "quality %s %s" % (law, "K" if kind == 0 else "V")
    for name, (mse, ip) in rows.items():
        record("%s %s" % (label, name), {"mse_rel": mse, "ip_rel_err": ip, "vectors": N})
    return rows


def _oracle_tq(orc):
    def f(b, mode, x):
        if mode == "mse":
            o = orc.Oracle(D, b, 0, key_mode=orc.KEY_MSE)
            r = o.compress_vectors(orc.KIND_VALUE, x)
            return o.decompress_vectors(orc.KIND_VALUE, r["codes"], None, r["norm"])
        o = orc.Oracle(D, b, 0, key_mode=orc.KEY_PROD)
        r = o.compress_vectors(orc.KIND_KEY, x)
        return o.decompress_vectors(orc.KIND_KEY, r["codes"], r["signs"], r["norm"], r["gamma"])
    return f


@pytest.mark.parametrize("law", ["tiny", "llama8b", "long70b"])
@pytest.mark.parametrize("kind", [0, 1])
def test_quality_report_oracle(orc, law, kind):
    rows = report(orc, law, kind, _oracle_tq(orc))
    tq3, tq4 = rows["tq3"], rows["tq4"]
    # the MSE quantizer meets the pages' bound (sqrt(3) pi / 2) / 4^b on every law
    assert tq3[0] <= math.sqrt(3) * math.pi / 2 / 4 ** 3 and tq4[0] <= math.sqrt(3) * math.pi / 2 / 4 ** 4
    # 3-bit TurboQuant beats naive 3-bit on both metrics, always
    assert tq3[0] < rows["naive minmax 3"][0] and tq3[1] < rows["naive minmax 3"][1]
    if law == "tiny" and kind == 1:
        # isotropic Gaussian values: per-vector uniform 4-bit rounding is already good
        # here, and the claim does not hold (reported, pinned as such)
        assert rows["naive minmax 4"][0] < tq3[0]
    else:
        # laws with per-channel scales and outlier channels: 3-bit TurboQuant has the
        # smaller inner-product error than naive 4-bit rounding on either grid, and the
        # smaller MSE than the abs-max grid
        assert tq3[1] < rows["naive minmax 4"][1] and tq3[1] < rows["naive absmax 4"][1]
        assert tq3[0] < rows["naive absmax 4"][0]


def _libtq_tq():
    import torch
    from kv_cache_vector_02_b200 import tq
    dev = torch.device("cuda")

    def f(b, mode, x):
        ctx = tq.tq_init(D, b, 0, tq.ROT_HAAR, tq.KEY_PROD)
        kind = tq.KIND_VALUE if mode == "mse" else tq.KIND_KEY
        n = x.shape[0]
        xs = torch.as_tensor(x.astype(np.float16)).reshape(n, 1, D).to(dev)
        nb = (n + 15) // 16
        slots = torch.arange(n, dtype=torch.int32, device=dev)
        cache = torch.zeros((nb, 1, tq.tq_chunk_bytes(ctx, kind)), dtype=torch.uint8, device=dev)
        other = torch.zeros((nb, 1, tq.tq_chunk_bytes(ctx, 1 - kind)), dtype=torch.uint8, device=dev)
        if kind == tq.KIND_VALUE:
            tq.tq_compress(ctx, None, xs, slots, other, cache)
        else:
            tq.tq_compress(ctx, xs, None, slots, cache, other)
        out = torch.empty((n, 1, D), dtype=torch.float32, device=dev)
        tq.tq_decompress(ctx, kind, cache, slots, out)
        torch.cuda.synchronize()
        assert tq.tq_get_device_error(ctx) == 0
        return out.reshape(n, D).cpu().numpy().astype(np.float64)
    return f


@pytest.mark.gpu
@pytest.mark.parametrize("law", ["tiny", "llama8b"])
def test_quality_report_libtq(orc, law):
    """The same report with libtq's own compress and decompress kernels on the fp16
    inputs: the metrics agree with the oracle's to well within their spread."""
    ref = report(orc, law, 0, _oracle_tq(orc))
    got = report(orc, law, 0, _libtq_tq())
    for name in ("tq3", "tq4", "tq3 prod"):
        for a, b in zip(got[name], ref[name]):
            assert abs(a - b) <= 1e-3 * b, (name, a, b)
