"""Plant mistakes in copies of the oracle and check that the pins catch each.

A pin that lets a plausible mistake through is too weak to trust the oracle
by. Each mutation below edits one line of a temporary copy of the oracle's C
source (dropped term, wrong sign, wrong index, flipped order or tie rule),
builds it into a separate library, and runs every pin against it: at least one
pin must fail. The real oracle is never modified.
"""
import os
import shutil
import tempfile

import pytest

import oracle
from test_oracle_pins import ALL_CHECKS

MUTATIONS = {
    "uncentred_scatter": ("C[a * d + b] += ca * (r[b] - mu[b]);", "C[a * d + b] += r[a] * r[b];"),
    "smallest_eigenvector": ("if (evals[j] > evals[best]) best = j;", "if (evals[j] < evals[best]) best = j;"),
    "jacobi_rotation_sign": ("A[k * n + p] = c * akp - s * akq;", "A[k * n + p] = c * akp + s * akq;"),
    "orientation_flipped": ("double sgn = V[kmax * d + 0] < 0.0 ? -1.0 : 1.0;",
                            "double sgn = V[kmax * d + 0] > 0.0 ? -1.0 : 1.0;"),
    "left_size_floor": ("return ((T + 1) / 2) * g;", "return (T / 2) * g;"),
    "softmax_unnormalised": ("double p = exp(s[t] - ls);", "double p = exp(s[t] - m);"),
    "scale_dropped": ("s[t] = scale * dot_row(qi, k, stride, d, j);", "s[t] = dot_row(qi, k, stride, d, j);"),
    "mass_unnormalised": ("mass[j] += exp(s[j] - ls);", "mass[j] += exp(s[j] - m);"),
    "topk_ascending": ("if (x->m > y->m) return -1;\n  if (x->m < y->m) return 1;",
                       "if (x->m < y->m) return -1;\n  if (x->m > y->m) return 1;"),
    "topk_ties_higher_index": ("return (x->j > y->j) - (x->j < y->j);", "return (x->j < y->j) - (x->j > y->j);"),
    "residual_sign": ("resid[t] = od_[t] - os_[t];", "resid[t] = os_[t] - od_[t];"),
    "reuse_drops_residual": ("o[t] += resid[t];", "o[t] -= resid[t];"),
    "bf16_ties_away": ("double r = nearbyint(m * 256.0);", "double r = round(m * 256.0);"),
    "krylov_start_vector": ("B[e] = 1.0 + (double)(orc_splitmix64((uint64_t)e + 1) >> 11) * 0x1.0p-53;",
                            "B[e] = 1.0 + (double)(orc_splitmix64((uint64_t)e) >> 11) * 0x1.0p-53;"),
    "krylov_no_orthogonalisation": ("for (int e = 0; e < d; ++e) w[e] -= c * B[(size_t)i * d + e];",
                                    "for (int e = 0; e < d; ++e) w[e] -= 0.0 * c * B[(size_t)i * d + e];"),
    "whiten_by_variance": ("wscale[e] = sigma > 0.0 ? 1.0 / sigma : 1.0;",
                           "wscale[e] = sigma > 0.0 ? 1.0 / (sigma * sigma) : 1.0;"),
    "whiten_not_applied": ("for (int e = 0; e < d; ++e) r[e] *= wscale[e];",
                           "for (int e = 0; e < d; ++e) r[e] *= 1.0;"),
}


@pytest.fixture(scope="module")
def workdir():
    d = tempfile.mkdtemp(prefix="orc_mut_")
    yield d
    shutil.rmtree(d, ignore_errors=True)


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(name, workdir):
    old, new = MUTATIONS[name]
    src = open(oracle._SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    path = os.path.join(workdir, f"{name}.c")
    with open(path, "w") as f:
        f.write(src.replace(old, new))
    lib = oracle.load(oracle.build(src=path, out=os.path.join(workdir, f"lib{name}.so")))
    failed = []
    for check in ALL_CHECKS:
        try:
            check(lib)
        except Exception:  # an assertion or a numerical blow-up both count as caught
            failed.append(check.__name__)
    assert failed, f"no pin caught the planted mistake {name!r}"
