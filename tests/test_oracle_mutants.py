"""Plant plausible mistakes in a copy of the oracle and check that a pin fails.

Each mutant is a textual edit of ``oracle/lca_oracle.c`` compiled to a
temporary library on the CPU.  A mutant that every pin accepts would mean the
pins leave that part of the oracle unchecked.
"""
import os

import pytest

import oracle_pins as pins
from oracle import oracle as orc

MUTANTS = {
    # anchor tie-break: highest index instead of lowest
    "tie_break_highest": ("if (w->s[t] > m) { m = w->s[t]; a = t; }",
                          "if (w->s[t] >= m) { m = w->s[t]; a = t; }"),
    # pooling weights from the semantic score only (drops the RoPE part)
    "pool_on_semantic_score": ("return exp(w->s[t] - w->gmax[j]) / w->gden[j];",
                               "return exp(w->sc[t] - w->gmax[j]) / w->gden[j];"),
    # fixed weights (not query-aware; 1/8 is the mean for g = 8)
    "mean_pooling": ("return exp(w->s[t] - w->gmax[j]) / w->gden[j];",
                     "return 0.125;"),
    # pooling weights not normalised inside the group
    "unnormalised_pooling": ("return exp(w->s[t] - w->gmax[j]) / w->gden[j];",
                             "return exp(w->s[t] - w->gmax[j]);"),
    # sign error in the pooling exponent
    "pool_exponent_sign": ("return exp(w->s[t] - w->gmax[j]) / w->gden[j];",
                           "return exp(w->gmax[j] - w->s[t]) / w->gden[j];"),
    # condensed logit without the anchor's positional key
    "no_anchor_key": ("l += dot_row(w->qr, k_r, w->ganc[j], d_r, dtype); /* anchor's K_R */", ""),
    # anchor key taken from the first token of the group
    "anchor_is_first_token": ("l += dot_row(w->qr, k_r, w->ganc[j], d_r, dtype); /* anchor's K_R */",
                              "l += dot_row(w->qr, k_r, j * g, d_r, dtype);"),
    # a +log(g) bias on condensed logits (the page adds no parameter)
    "log_g_bias": ("w->ell[j] = l;", "w->ell[j] = l + log((double)g);"),
    # a trailing partial group instead of leftovers joining the window
    "ceil_group_count": ("return (L - (int64_t)w) / g;", "return (L - (int64_t)w + g - 1) / g;"),
    # pooled latent reads the wrong token rows (index slip)
    "pool_wrong_row": ("cbar[i] += wt * elem(c_kv, t * (int64_t)d_c + i, dtype);",
                       "cbar[i] += wt * elem(c_kv, (t - j * g) * (int64_t)d_c + i, dtype);"),
    # window drops the current (last) token
    "window_drops_current": ("for (int64_t t = win0; t < L; ++t) {\n            double p = exp(",
                             "for (int64_t t = win0; t < L - 1; ++t) {\n            double p = exp("),
    # positional score uses the semantic query (transposed operand)
    "rope_score_wrong_query": ("w->sr[t] = dot_row(w->qr, k_r, t, d_r, dtype);",
                               "w->sr[t] = dot_row(w->qc, k_r, t, d_r, dtype);"),
    # near-tie report: runner-up taken over the whole group, anchor included
    # (every gap would be 0 and no bf16 anchor would ever be compared)
    "tie_gap_second_includes_anchor": ("if (t != a && w->s[t] > second) second = w->s[t];",
                                       "if (w->s[t] > second) second = w->s[t];"),
    # near-tie report: max of s instead of max of |s|
    "max_abs_s_signed": ("if (fabs(w->s[t]) > amax) amax = fabs(w->s[t]);",
                         "if (w->s[t] > amax) amax = w->s[t];"),
    # near-tie report: runner-up excludes the group's first token, not the anchor
    "tie_gap_wrong_token": ("if (t != a && w->s[t] > second) second = w->s[t];",
                            "if (t != t0 && w->s[t] > second) second = w->s[t];"),
    # stored cache: sum over heads instead of the mean (a different temperature)
    "stored_sum_not_mean": ("sbar[u] /= (double)H;", "sbar[u] /= 1.0;"),
    # stored cache: the bias on condensed logits with the wrong sign
    "stored_bias_sign": ("double l = bias;", "double l = -bias;"),
    # stored cache: ties go to the highest index
    "stored_tie_break_highest": ("if (sbar[u] > m) { m = sbar[u]; a = u; }",
                                 "if (sbar[u] >= m) { m = sbar[u]; a = u; }"),
    # stored cache: the pooled latent reads the group's first row only
    "stored_pool_first_row": ("cb[i] += wt * elem(c_kv, (t0 + u) * (int64_t)d_c + i, dtype);",
                              "cb[i] += wt * elem(c_kv, (t0) * (int64_t)d_c + i, dtype);"),
    # stored cache: the anchor key from the group's first token
    "stored_anchor_key_first": ("kanc[jj * (int64_t)d_r + i] = elem(k_r, (t0 + a) * (int64_t)d_r + i, dtype);",
                                "kanc[jj * (int64_t)d_r + i] = elem(k_r, (t0) * (int64_t)d_r + i, dtype);"),
}


@pytest.fixture(scope="module")
def oracle_src():
    with open(orc.SRC) as f:
        return f.read()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, oracle_src, tmp_path):
    old, new = MUTANTS[name]
    assert oracle_src.count(old) >= 1, f"mutant anchor text not found: {name}"
    src = tmp_path / "mutant.c"
    src.write_text(oracle_src.replace(old, new, 1))
    lib_path = str(tmp_path / "libmutant.so")
    orc.build(str(src), lib_path)
    lib = orc.load(lib_path)
    failures = []
    for pin in pins.ALL_PINS:
        try:
            pin(lib)
        except (AssertionError, RuntimeError, IndexError, ValueError):
            # a wrong value, the oracle refusing its own output, or an oracle built on the
            # mutant's segmentation failing on it
            failures.append(pin.__name__)
    assert failures, f"mutant {name} passed every pin"


def test_unmutated_copy_passes(oracle_src, tmp_path):
    src = tmp_path / "copy.c"
    src.write_text(oracle_src)
    lib_path = str(tmp_path / "libcopy.so")
    orc.build(str(src), lib_path)
    lib = orc.load(lib_path)
    for pin in pins.ALL_PINS:
        pin(lib)
    assert os.path.exists(lib_path)


# Plausible mistakes in the GQA oracle (numpy, in oracle.py): each is planted in a
# copy of the function's source, and one of the GQA pins must fail.
GQA_MUTANTS = {
    # query head h read KV head h % H_kv instead of h // (H / H_kv)
    "kv_head_interleaved": ("kv = h // r", "kv = h % H_kv"),
    # pooled key instead of the anchor's key (the positional component mixed)
    "pooled_key_logit": ("logits.append(sg[a])", "logits.append(wt @ sg)"),
    # values not pooled: the anchor's value stands for the group
    "anchor_value": ("values.append(wt @ V[j * g:(j + 1) * g])", "values.append(V[j * g + a])"),
    # uniform pooling weights
    "mean_pooling": ("wt = e / e.sum()", "wt = np.full(len(sg), 1.0 / len(sg))"),
    # tie-break on the highest index
    "tie_break_highest": ("a = int(np.argmax(sg))", "a = len(sg) - 1 - int(np.argmax(sg[::-1]))"),
    # window without its first leftover token
    "window_off_by_one": ("for t in range(win0, L):", "for t in range(win0 + 1, L):"),
}


@pytest.fixture(scope="module")
def gqa_src():
    import inspect
    return inspect.getsource(orc.lca_gqa)


@pytest.mark.parametrize("name", sorted(GQA_MUTANTS))
def test_gqa_mutant_is_caught(name, gqa_src, oracle_lib, monkeypatch):
    old, new = GQA_MUTANTS[name]
    assert gqa_src.count(old) == 1, f"mutant anchor text not found: {name}"
    ns = dict(vars(orc))
    exec(compile(gqa_src.replace(old, new), "<gqa mutant>", "exec"), ns)
    monkeypatch.setattr(orc, "lca_gqa", ns["lca_gqa"])
    failures = []
    for pin in pins.GQA_PINS:
        try:
            pin(oracle_lib)
        except AssertionError:
            failures.append(pin.__name__)
    assert failures, f"GQA mutant {name} passed every pin"
