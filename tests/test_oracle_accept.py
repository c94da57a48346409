"""Pins for the oracle's acceptance walk (no GPU).

Hand-worked cases from the acceptance formula; brute force over every
root->node path for greedy; closed forms when target == draft (sigma = 0);
the inverse CDF against numpy's searchsorted; and distribution preservation:
with drafts sampled from q, the first emitted token is distributed as the
target p (chi-square over 10^6 seeded trials), for a chain and for a star of
iid siblings.  A planted mistake in the residual step must fail that test.
"""
import json
import os

import numpy as np
import pytest
from scipy.stats import chisquare

import oracle
import oracle.accept as oracle_accept
from workloads import get_config, gen_draft_logits, gen_uniforms, make_target_logits


def _load(golden_dir):
    with open(os.path.join(golden_dir, "accept_handworked.json")) as f:
        return json.load(f)


@pytest.mark.parametrize("case", [0, 1, 2])
def test_handworked_stochastic(golden_dir, case):
    fx = _load(golden_dir)
    c = fx["cases"][case]
    target = np.log(np.array(c["target_probs"]))
    draft = np.log(np.array(fx["draft_probs"]))
    u = np.array([c["u_acc"], c["u_res"]])
    r = oracle.accept_stochastic(target, draft, fx["tokens"], fx["parents"], fx["draft_row"], u, 2)
    assert (r["accepted_len"], r["path"], r["bonus"]) == (c["accepted_len"], c["path"], c["bonus"])
    if "greedy" in c:
        g = oracle.accept_greedy(target, fx["tokens"], fx["parents"], 2)
        exp = c["greedy"]
        assert (g["accepted_len"], g["path"], g["bonus"]) == (exp["accepted_len"], exp["path"], exp["bonus"])


def test_inverse_cdf_matches_searchsorted():
    rng = np.random.default_rng(20)
    for _ in range(200):
        w = rng.random(int(rng.integers(1, 40))) * (rng.random() < 0.9)
        w[rng.integers(0, w.shape[0])] += 0.1
        u = float(rng.random())
        i, _ = oracle.inverse_cdf(w, u)
        c = np.cumsum(w)
        assert i == min(int(np.searchsorted(c, u * c[-1], side="right")), w.shape[0] - 1)


def _all_paths(parents):
    n = parents.shape[0]
    paths = [[]]
    for i in range(1, n + 1):
        path, node = [], i
        while node:
            path.append(node)
            node = int(parents[node - 1])
        paths.append(path[::-1])
    return paths


@pytest.mark.parametrize("name,seed", [("tiny", 0), ("7b", 1), ("7b", 2)])
def test_greedy_is_longest_argmax_path(name, seed):
    """Brute force: of all root->node paths, the accepted one is the longest whose
    every token is the argmax of its parent's target row."""
    cfg = get_config(name)
    dl = gen_draft_logits(cfg, seed)
    x = oracle.decode_logits(dl, cfg.logits_dtype)[0]
    t = oracle.build_tree(x, cfg.depth, cfg.k, cfg.m)
    tgt = make_target_logits(cfg, seed, dl, t["draft_row"][None])
    T = oracle.decode_logits(tgt, cfg.logits_dtype)[0]
    best = []
    for path in _all_paths(t["parents"]):
        prev = 0
        ok = True
        for node in path:
            if int(t["tokens"][node - 1]) != int(np.argmax(T[prev])):
                ok = False
                break
            prev = node
        if ok and len(path) > len(best):
            best = path
    r = oracle.accept_greedy(T, t["tokens"], t["parents"], cfg.depth)
    assert r["path"][:r["accepted_len"]] == best
    stop = best[-1] if best else 0
    assert r["bonus"] == int(np.argmax(T[stop]))


def _first_child_chain(parents):
    chain, j = [], 0
    while True:
        kids = [c + 1 for c in range(parents.shape[0]) if parents[c] == j]
        if not kids:
            return chain
        j = kids[0]
        chain.append(j)


@pytest.mark.parametrize("name", ["tiny", "7b"])
def test_sigma0_closed_forms(name):
    """target == draft: greedy follows the rank-0 children; sampling accepts every
    first child and draws the bonus from the leaf's target row."""
    cfg = get_config(name)
    dl = gen_draft_logits(cfg, 4)
    x = oracle.decode_logits(dl, cfg.logits_dtype)[0]
    t = oracle.build_tree(x, cfg.depth, cfg.k, cfg.m)
    tgt = make_target_logits(cfg, 4, dl, t["draft_row"][None], sigma=0.0)
    T = oracle.decode_logits(tgt, cfg.logits_dtype)[0]
    chain = _first_child_chain(t["parents"])
    g = oracle.accept_greedy(T, t["tokens"], t["parents"], cfg.depth)
    assert g["path"][:g["accepted_len"]] == chain
    u = gen_uniforms(cfg, 4)[0].astype(np.float64)
    s = oracle.accept_stochastic(T, x, t["tokens"], t["parents"], t["draft_row"], u, cfg.depth)
    assert s["path"][:s["accepted_len"]] == chain
    leaf = chain[-1]
    p = np.exp(T[leaf] - T[leaf].max())
    c = np.cumsum(p)
    assert s["bonus"] == int(np.searchsorted(c, u[1, leaf] * c[-1], side="right"))


@pytest.mark.parametrize("case", [0, 1])
@pytest.mark.parametrize("rule", ["with_replacement", "without_replacement"])
def test_handworked_without_replacement(golden_dir, case, rule):
    with open(os.path.join(golden_dir, "accept_without_replacement_handworked.json")) as f:
        fx = json.load(f)
    c = fx["cases"][case]
    r = oracle.accept_stochastic(np.log(np.array(fx["target_probs"])), np.log(np.array(fx["draft_probs"])),
                                 fx["tokens"], fx["parents"], fx["draft_row"], np.array([c["u_acc"], c["u_res"]]),
                                 2, without_replacement=rule == "without_replacement")
    assert (r["accepted_len"], r["path"], r["bonus"]) == tuple(c[rule][f] for f in ("accepted_len", "path", "bonus"))


def test_one_child_per_node_rules_coincide():
    """With a single child per node nothing is drawn after a rejection, so both rules agree."""
    cfg = get_config("tiny", k=1, depth=4, m=3, V=50, B=1, logits_dtype="f32")
    draft = oracle.decode_logits(gen_draft_logits(cfg, 4), "f32")[0]
    t = oracle.build_tree(draft, cfg.depth, cfg.k, cfg.m)
    target = make_target_logits(cfg, 4, gen_draft_logits(cfg, 4), t["draft_row"][None])[0].astype(np.float64)
    for s in range(40):
        u = gen_uniforms(cfg, s)[0].astype(np.float64)
        a = oracle.accept_stochastic(target, draft, t["tokens"], t["parents"], t["draft_row"], u, cfg.depth)
        b = oracle.accept_stochastic(target, draft, t["tokens"], t["parents"], t["draft_row"], u, cfg.depth,
                                     without_replacement=True)
        assert (a["accepted_len"], a["path"], a["bonus"]) == (b["accepted_len"], b["path"], b["bonus"])


def _draw_without_replacement(rng, q, count):
    """`count` distinct tokens, each drawn from q restricted to the tokens not drawn yet."""
    w = q.copy()
    out = []
    for _ in range(count):
        c = np.cumsum(w)
        x = min(int(np.searchsorted(c, rng.random() * c[-1], side="right")), q.shape[0] - 1)
        out.append(x)
        w[x] = 0.0
    return np.array(out)


def _chi2_first_token_distinct(trials, seed, rule_without):
    """First emitted token over `trials` walks of a star of 3 distinct siblings
    drawn without replacement from q; the walk uses the rule given."""
    rng = np.random.default_rng(seed)
    V = 8
    p = rng.dirichlet(np.ones(V))
    q = rng.dirichlet(np.ones(V) * 0.5)
    other = np.log(rng.dirichlet(np.ones(V)))
    parents = np.array([0, 0, 0])
    draft_row = np.array([0, -1, -1, -1])
    draft = np.log(q)[None]
    target = np.stack([np.log(p), other, other, other])
    counts = np.zeros(V, dtype=np.int64)
    for _ in range(trials):
        toks = _draw_without_replacement(rng, q, 3)
        u = rng.random((2, 4)).astype(np.float32).astype(np.float64)
        r = oracle.accept_stochastic(target, draft, toks, parents, draft_row, u, 1, without_replacement=rule_without)
        counts[int(toks[r["path"][0] - 1]) if r["accepted_len"] else r["bonus"]] += 1
    return chisquare(counts, trials * p).pvalue


@pytest.mark.slow
def test_sampling_without_replacement_preserves_target_distribution():
    assert _chi2_first_token_distinct(1_000_000, 33, True) > 1e-3


def test_with_replacement_rule_on_distinct_drafts_is_caught():
    """The with-replacement residual chain applied to siblings drawn without
    replacement is biased; the same test must see it."""
    assert _chi2_first_token_distinct(200_000, 34, False) < 1e-6


def _chi2_first_token(trials, shape, seed):
    """First emitted token over `trials` walks with drafts sampled from q."""
    rng = np.random.default_rng(seed)
    V = 8
    p = rng.dirichlet(np.ones(V))
    q = rng.dirichlet(np.ones(V))
    q2 = rng.dirichlet(np.ones(V))
    lp, lq, lq2 = np.log(p), np.log(q), np.log(q2)
    other = np.log(rng.dirichlet(np.ones(V)))
    if shape == "star":
        parents = np.array([0, 0, 0])
        draft_row = np.array([0, -1, -1, -1])
        draft = lq[None]
        target = np.stack([lp, other, other, other])
    else:  # chain of depth 2
        parents = np.array([0, 1])
        draft_row = np.array([0, 1, -1])
        draft = np.stack([lq, lq2])
        target = np.stack([lp, other, other])
    n = parents.shape[0]
    counts = np.zeros(V, dtype=np.int64)
    cq, cq2 = np.cumsum(q), np.cumsum(q2)
    for _ in range(trials):
        if shape == "star":
            toks = np.minimum(np.searchsorted(cq, rng.random(3), side="right"), V - 1)
        else:
            toks = np.array([min(int(np.searchsorted(cq, rng.random(), side="right")), V - 1),
                             min(int(np.searchsorted(cq2, rng.random(), side="right")), V - 1)])
        u = rng.random((2, n + 1)).astype(np.float32).astype(np.float64)
        r = oracle.accept_stochastic(target, draft, toks, parents, draft_row, u, 2)
        first = int(toks[r["path"][0] - 1]) if r["accepted_len"] else r["bonus"]
        counts[first] += 1
    return chisquare(counts, trials * p).pvalue


@pytest.mark.slow
@pytest.mark.parametrize("shape", ["star", "chain"])
def test_sampling_preserves_target_distribution(shape):
    assert _chi2_first_token(1_000_000, shape, seed=30 if shape == "star" else 31) > 1e-3


def test_planted_residual_mistake_is_caught(monkeypatch):
    """Resampling from the unadjusted target after a rejection (a dropped
    subtraction) must fail the same test, even with fewer trials."""
    monkeypatch.setattr(oracle_accept, "_residual", lambda p, q: p)
    assert _chi2_first_token(50_000, "star", seed=32) < 1e-6
