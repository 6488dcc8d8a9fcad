"""Each plausible mistake planted in a copy of the oracle source must fail
at least one pin.  The mistakes are edits of the C source on the CPU; the
committed oracle is untouched.  Every mistake keeps all memory accesses in
bounds, so a mutant can only return wrong numbers, never crash."""

import pytest

import oracle
import oracle_pins

# (name, text in cca_oracle.c, replacement, which occurrence: 0 first, -1 all)
MUTANTS = [
    ("window counts self in w", "long lo = t - w;", "long lo = t - w + 1;", 0),
    ("window not group aligned", "return (lo / g) * g;", "return lo;", 0),
    ("pool scored by first query", "last = j * g + g - 1;", "last = j * g;", 0),
    ("pool scale 1/d", "const double scale = 1.0 / sqrt((double)d);\n\n#pragma omp parallel num_threads(cca_oracle_threads())\n    {\n        double *s",
     "const double scale = 1.0 / (double)d;\n\n#pragma omp parallel num_threads(cca_oracle_threads())\n    {\n        double *s", 0),
    ("attention scale 1/d", "const double scale = 1.0 / sqrt((double)d);\n    for (long j = 0; j < nc; ++j) logit[j]",
     "const double scale = 1.0 / (double)d;\n    for (long j = 0; j < nc; ++j) logit[j]", 0),
    ("gqa sum not mean", "a[i] += s[i] / r;", "a[i] += s[i];", -1),
    ("pool K with V", "ks += a[i] * Kh[(size_t)(first + i) * d + c];",
     "ks += a[i] * Vh[(size_t)(first + i) * d + c];", 0),
    ("pool transposed index", "Kh[(size_t)(first + i) * d + c]",
     "Kh[(size_t)(first + c % g) * d + i % d]", 0),
    ("one core token too many", "const long nc = ws / g, nl = t - ws + 1;\n                    const size_t kv",
     "const long nc = ws / g + (ws < T - g ? 1 : 0), nl = t - ws + 1;\n                    const size_t kv", 0),
    ("query misses itself", "const long nc = ws / g, nl = t - ws + 1;\n                    const size_t kv",
     "const long nc = ws / g, nl = t - ws + (t > 0 ? 0 : 1);\n                    const size_t kv", 0),
    ("raw weights misindexed", "out[c] += logit[nc + i] * vraw[i][c];",
     "out[c] += logit[i] * vraw[i][c];", 0),
    ("core values all from group 0", "out[c] += logit[j] * vcore[j][c];",
     "out[c] += logit[j] * vcore[0][c];", 0),
    ("softmax not normalised", "for (long i = 0; i < n; ++i) x[i] /= sum;",
     "for (long i = 0; i < n; ++i) x[i] /= (sum + 1e-3);", 0),
    ("append pools shifted group", "const long j = t / g, first = t - g + 1;",
     "const long j = t / g, first = t - g;", 0),
    ("append writes wrong core slot", "double *kc = c->k_core + (kv * c->core_cap + j) * d;",
     "double *kc = c->k_core + (kv * c->core_cap + (j > 0 ? j - 1 : 0)) * d;", 0),
    ("decode ring index off by one", "kp[nc + i] = c->k_tail + (kv * c->tail_cap +\n                                              p % c->tail_cap) * d;",
     "kp[nc + i] = c->k_tail + (kv * c->tail_cap +\n                                              (p + 1) % c->tail_cap) * d;", 0),
    ("lca scored by last query", "qbar[c] = acc / g;", "qbar[c] = Qg[(size_t)(g - 1) * d + c];", 0),
    ("lca sum of queries", "qbar[c] = acc / g;", "qbar[c] = acc;", 0),
    ("lca scale 1/d", "const double inv_sqrt_d = 1.0 / sqrt((double)d);",
     "const double inv_sqrt_d = 1.0 / (double)d;", 0),
    ("lca heads summed", "wgt[i] += p[i] / (double)r;", "wgt[i] += p[i];", 0),
    ("lca anchor argmin", "if (wgt[i] > wgt[best]) best = i;", "if (wgt[i] < wgt[best]) best = i;", 0),
    ("lca anchor last on ties", "if (wgt[i] > wgt[best]) best = i;", "if (wgt[i] >= wgt[best]) best = i;", 0),
    ("lca positional part pooled", "kc[c] = c < d_content ? kacc : Kg[(size_t)best * d + c];",
     "kc[c] = kacc;", 0),
    ("lca positional part at the front", "kc[c] = c < d_content ? kacc : Kg[(size_t)best * d + c];",
     "kc[c] = c >= d_rope ? kacc : Kg[(size_t)best * d + c];", 0),
    ("lca values from keys", "vacc += wgt[i] * Vg[(size_t)i * d + c];",
     "vacc += wgt[i] * Kg[(size_t)i * d + c];", 0),
    ("lca query rows of head 0 only", "Q + (((size_t)b * Hq + h * r + k) * T + first) * d;",
     "Q + (((size_t)b * Hq + h * r) * T + first) * d;", 0),
    ("lca cache forgets the token's own query", "qbar[e] = (q_sum[qh + e] + q[qh + e]) / g;",
     "qbar[e] = q_sum[qh + e] / g;", 0),
    ("lca cache keeps stale sums", "for (size_t e = 0; e < nq; ++e) q_sum[e] = 0.0;",
     "for (size_t e = 0; e < nq; ++e) q_sum[e] = q_sum[e];", 0),
    ("lca cache anchor ignores the ring position",
     "const size_t best_row = kv * c->tail_cap + (first + best) % c->tail_cap;",
     "const size_t best_row = kv * c->tail_cap + best % c->tail_cap;", 0),
    ("capacity check off by one", "if (t / g >= c->core_cap) return CCA_ORACLE_ECAPACITY;",
     "if (t / g > c->core_cap) return CCA_ORACLE_ECAPACITY;", 0),
]


def _mutate(src, old, new, which):
    assert old in src, f"mutation anchor not found: {old!r}"
    if which == -1:
        return src.replace(old, new)
    return src.replace(old, new, 1)


@pytest.mark.parametrize("name,old,new,which", MUTANTS,
                         ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(tmp_path, name, old, new, which):
    src = _mutate(oracle.source(), old, new, which)
    assert src != oracle.source()
    mutant = oracle.build_variant(src, str(tmp_path / "libmutant.so"))
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(mutant)
        except AssertionError:
            caught.append(pin.__name__)
        except oracle.OracleError:
            caught.append(pin.__name__)
    assert caught, f"no pin caught the planted mistake: {name}"
