"""Dense "allowed" predicates of the structured mask families, written from
each family's parameters -- independently of the four-vector encoding -- so
that the encoding can be checked by brute force (TEST INFRASTRUCTURE ONLY).

Families named on the FlashMask-3 pages: document, prefix-LM, share-question,
sliding-window and block-sparse ([abstract] acceptodds.com; [explainer]
learnaivisually.com, "four numbers per avenue"), causal masks (baguaai.com,
"Universal Pattern Support").  The 12-mask sweep adds full, bidirectional
document, prefix-LM document, causal blockwise, global + sliding window and
random eviction.  Readings where the pages give no definition:
  causal blockwise(b): floor(j/b) <= floor(i/b)  (bidirectional inside a block)
  global+sliding(G,W): i < G or j < G or |i - j| < W
  random eviction:     j <= i < R_j  (causal, key j evicted from row R_j on)

allowed[i, j] is True where query row i may attend to key j.
"""
from __future__ import annotations

import numpy as np


def _grid(n):
    i = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    return i, j


def _doc_id(n, docs):
    d = np.empty(n, np.int64)
    for t, (a, b) in enumerate(docs):
        d[a:b] = t
    return d


def allowed_full(n):
    return np.ones((n, n), bool)


def allowed_causal(n):
    i, j = _grid(n)
    return j <= i


def allowed_sliding_window(n, w):
    i, j = _grid(n)
    return (j <= i) & (i < j + w)


def allowed_causal_document(n, docs):
    i, j = _grid(n)
    d = _doc_id(n, docs)
    return (d[:, None] == d[None, :]) & (j <= i)


def allowed_bidir_document(n, docs):
    d = _doc_id(n, docs)
    return d[:, None] == d[None, :]


def allowed_prefix_lm(n, prefix):
    i, j = _grid(n)
    return (j < prefix) | (j <= i)


def allowed_prefix_lm_document(n, docs, prefixes):
    i, j = _grid(n)
    d = _doc_id(n, docs)
    start = np.array([docs[t][0] for t in d])
    pre = np.array([prefixes[t] for t in d])
    same = d[:, None] == d[None, :]
    return same & ((j < (start + pre)[None, :]) | (j <= i))


def allowed_share_question(n, groups):
    """A question token is seen causally by every later token of its group; an
    answer token is seen causally only inside its own answer."""
    i, j = _grid(n)
    group = np.full(n, -1, np.int64)
    part = np.full(n, -1, np.int64)  # -1 question, else answer index
    for g, ((qs, qe), answers) in enumerate(groups):
        group[qs:qe] = g
        for a_i, (a, b) in enumerate(answers):
            group[a:b] = g
            part[a:b] = a_i
    same_group = group[:, None] == group[None, :]
    key_is_q = (part == -1)[None, :]
    same_part = part[:, None] == part[None, :]
    return (j <= i) & same_group & (key_is_q | same_part)


def allowed_causal_blockwise(n, block):
    i, j = _grid(n)
    return (j // block) <= (i // block)


def allowed_global_sliding(n, g, w):
    i, j = _grid(n)
    return (i < g) | (j < g) | (np.abs(i - j) < w)


def allowed_random_eviction(n, evict):
    i, j = _grid(n)
    return (j <= i) & (i < np.asarray(evict)[None, :])


def allowed_from_spec(spec) -> np.ndarray:
    """Dispatch on a synth.MaskSpec's family name and parameters."""
    f, n, p = spec.family, spec.n, spec.params
    if f == "full":
        return allowed_full(n)
    if f == "causal":
        return allowed_causal(n)
    if f == "sliding_window":
        return allowed_sliding_window(n, p["w"])
    if f == "causal_document":
        return allowed_causal_document(n, p["docs"])
    if f == "bidir_document":
        return allowed_bidir_document(n, p["docs"])
    if f == "prefix_lm":
        return allowed_prefix_lm(n, p["prefix"])
    if f == "prefix_lm_document":
        return allowed_prefix_lm_document(n, p["docs"], p["prefixes"])
    if f == "share_question":
        return allowed_share_question(n, p["groups"])
    if f == "causal_blockwise":
        return allowed_causal_blockwise(n, p["block"])
    if f == "global_sliding":
        return allowed_global_sliding(n, p["g"], p["w"])
    if f == "random_eviction":
        return allowed_random_eviction(n, p["evict"])
    raise ValueError(f)
