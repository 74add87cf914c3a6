"""The attention kernel's exp2 on the FMA pipe (exp2_poly2 in attn_kernel.cu):
its step sequence replayed in numpy float32 must stay within 1.1e-4 relative
of 2^x over the range the softmax feeds it (x <= 8 after the lazy rescale),
and give a tiny non-negative value for masked (-inf) columns."""
import re
from pathlib import Path

import numpy as np

SRC = Path(__file__).resolve().parents[1] / "cluster_routed_sparse_b200" / "csrc" / "attn_kernel.cu"


def _coefficients():
    text = SRC.read_text()
    body = text.split("void exp2_poly2(", 1)[1].split("\n}", 1)[0]
    line = [ln for ln in text.splitlines() if ln.startswith("constexpr float kExp2C3")][0]
    vals = dict(re.findall(r"(kExp2C[123])\s*=\s*([0-9.eE+-]+)f", line))
    magic = re.findall(r"kRoundMagic\s*=\s*([0-9.]+)f", text)
    # Horner order: leading coefficient c3 first, then c2, c1 and the constant 1
    return body, [float(vals["kExp2C3"]), float(vals["kExp2C2"]), float(vals["kExp2C1"]), 1.0], float(magic[0])


def exp2_poly_np(x, c3, c2, c1):
    f32 = np.float32
    x = np.maximum(x.astype(f32), f32(-126.0))
    t = (x + f32(12582912.0)).astype(f32)
    f = (x - (t - f32(12582912.0)).astype(f32)).astype(f32)
    # fmaf == exact product + sum rounded once: evaluate in float64, round to float32
    q = (f.astype(np.float64) * c3 + c2).astype(f32)
    q = (f.astype(np.float64) * q + c1).astype(f32)
    q = (f.astype(np.float64) * q + 1.0).astype(f32)
    bits = q.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_constants_found():
    body, c, magic = _coefficients()
    assert magic == 1.5 * 2 ** 23 and "kRoundMagic" in body and "-126.f" in body
    assert len(c) == 4 and c[3] == 1.0


def test_relative_error_over_softmax_range():
    _, c, _ = _coefficients()
    c3, c2, c1 = np.float32(c[0]), np.float32(c[1]), np.float32(c[2])
    x = np.concatenate([np.linspace(-120.0, 8.0, 2_000_001), np.linspace(-1.0, 1.0, 200_001)]).astype(np.float32)
    y = exp2_poly_np(x, c3, c2, c1).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    assert rel.max() < 1.1e-4, rel.max()


def test_masked_columns_are_negligible():
    _, c, _ = _coefficients()
    y = exp2_poly_np(np.array([-np.inf, -1e30, -200.0, -126.0], np.float32), np.float32(c[0]), np.float32(c[1]),
                     np.float32(c[2]))
    assert np.all(y >= 0) and np.all(np.isfinite(y)) and y.max() <= 2.0 ** -125
