"""The tensor-core forward's barrier protocol as a discrete-event model.

The kernel's roles -- the TMA thread, the MMA thread and the softmax warps of
the two tile slots -- are modelled as sequential programs that arrive on and
wait for phases of mbarriers, following the order of `tc_fwd_kernel` in
`csrc/jfa_tc_fwd.cu`: the two-stage K/V ring released by the last user of a
key tile, per-slot Q buffers, the slots' rows swapped on the CTA's odd items,
and the slot with one key tile fewer issuing its next item's first Q K^T after
its last P.V (waiting for the key tile's load, releasing the stage only as its
sole user).  A copy lands at once and an MMA retires at once, so only the
order of waits and arrivals is checked: the model must finish, and no wait may
be for a phase that the barrier has already passed twice (parity aliasing),
on the item lists of the self-attention bench batch and on random ones.  A
variant with the early Q K^T treated like an in-order one must fail.

Pages: "Meta GEM Training Efficiency: Why LLM-Scale Recommenders Need a
Different Stack", "Bottleneck move 1" (jagged tiles of uneven length).
"""
import numpy as np
import pytest

import oracle
from jagged_attention_recommender_jfa_b200.inputs import draw_lengths


class ProtocolError(Exception):
    pass


def block_items(lens, H, rows=256, tile=128):
    """(n_upper, n_lower, n) key tiles per 256-row item of the causal
    self-attention schedule (upper = first 128 rows of the block)."""
    off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    out = []
    for b, _, t, _ in oracle.schedule(off, off, H, rows, True, False):
        n, row0 = int(lens[b]), int(t) * rows
        nt = []
        for half in range(2):
            lo, hi = row0 + half * tile, min(row0 + (half + 1) * tile, n)
            nt.append(0 if hi <= lo else (hi + tile - 1) // tile)
        out.append((nt[0], nt[1], max(nt)))
    return out


def item_of_turn(r, c, G):
    return r * G + ((G - 1 - c) if (r & 1) else c)


def run_model(items, cta=0, G=1, early_ordered=False):
    """Runs one CTA's roles over its items; raises ProtocolError on a
    deadlock, an aliased wait or a score MMA on a key tile not yet loaded."""
    done = {}

    def arrive(name):
        done[name] = done.get(name, 0) + 1

    mine = []
    r = 0
    while item_of_turn(r, cta, G) < len(items):
        a_, b_, n = items[item_of_turn(r, cta, G)]
        mine.append((b_, a_, n) if r & 1 else (a_, b_, n))   # odd items swap the slots
        r += 1

    def tma():
        g, nq, early = 0, [0, 0], 0

        def load_q(w, t):
            if w[t] == 0:
                return
            if nq[t] > 0:
                yield (("q_free", t), nq[t] - 1)
            arrive(("q_full", t))
            nq[t] += 1

        for w in mine:
            if w[2] == 0:
                continue
            yield from load_q(w, early)
            for j in range(w[2]):
                if j == 1:
                    yield from load_q(w, early ^ 1)
                s = g & 1
                if g >= 2:
                    yield (("k_empty", s), (g >> 1) - 1)
                arrive(("k_full", s))
                if g >= 2:
                    yield (("v_empty", s), (g >> 1) - 1)
                arrive(("v_full", s))
                g += 1
            if w[2] == 1:
                yield from load_q(w, early ^ 1)
            early = 1 if (w[1] == w[2] - 1 and w[0] == w[2]) else 0

    def mma():
        gt, mt, nq = [0, 0], [0, 0], [0, 0]
        first = lambda w, j: 0 if j < w[0] else 1
        last = lambda w, j: 1 if j < w[1] else 0

        issued = {}   # score MMAs issued per key tile of the CTA

        def qk(w, g0, t, j, wait_k, release_k):
            gg, s = g0 + j, (g0 + j) & 1
            if j == 0:
                yield (("q_full", t), nq[t])
                nq[t] += 1
            if wait_k:
                yield (("k_full", s), gg >> 1)
            elif done.get(("k_full", s), 0) < (gg >> 1) + 1:
                raise ProtocolError(f"score MMA on key tile {gg} before its load")
            arrive(("s_full", t))
            issued[gg] = issued.get(gg, 0) + 1
            if release_k:
                # whatever the timing, a stage is released only after every
                # score MMA on its key tile
                if issued[gg] != (j < w[0]) + (j < w[1]):
                    raise ProtocolError(f"key tile {gg} released before all its score MMAs")
                arrive(("k_empty", s))
            if j == w[t] - 1:
                arrive(("q_free", t))

        def ordered(w, g0, t, j):
            return qk(w, g0, t, j, t == first(w, j), t == last(w, j))

        g, early, pv = 0, -1, {}
        for r, w in enumerate(mine):
            if w[2] == 0:
                continue
            g0 = g
            for t in range(2):
                if w[t] > 0 and t != early:
                    if early >= 0 and not early_ordered:
                        yield from qk(w, g0, t, 0, True, True)
                    else:
                        yield from ordered(w, g0, t, 0)
            early = -1
            for j in range(w[2]):
                s = g & 1
                for t in range(2):
                    if j >= w[t]:
                        continue
                    yield (("p_full", t), gt[t])
                    if j == 0 and mt[t] > 0:
                        yield (("o_free", t), mt[t] - 1)
                    if t == first(w, j):
                        yield (("v_full", s), g >> 1)
                    arrive(("pv_done", t))
                    pv[g] = pv.get(g, 0) + 1
                    if t == last(w, j):
                        if pv[g] != (j < w[0]) + (j < w[1]):
                            raise ProtocolError(f"value tile {g} released before all its P.V")
                        arrive(("v_empty", s))
                    gt[t] += 1
                    if j == 0:
                        mt[t] += 1
                    if j + 1 < w[t]:
                        yield from ordered(w, g0, t, j + 1)
                for es in range(2):
                    if j != w[es] - 1 or j + 2 != w[2] or w[es ^ 1] != w[2]:
                        continue
                    nxt = next((w2 for w2 in mine[r + 1:] if w2[2] > 0), None)
                    if nxt is not None and nxt[es] > 0:
                        if early_ordered:
                            yield from ordered(nxt, g0 + w[2], es, 0)
                        else:
                            yield from qk(nxt, g0 + w[2], es, 0, True, nxt[es ^ 1] == 0)
                        early = es
                g += 1

    def softmax(t):
        gt, gkv = 0, 0
        for w in mine:
            n, base = w[t], gkv
            gkv += w[2]
            if n == 0:
                continue
            for j in range(n):
                yield (("s_full", t), gt)
                # the stage's V and bias window (the first user clears V's tail rows)
                yield (("v_full", (base + j) & 1), (base + j) >> 1)
                arrive(("p_full", t))
                gt += 1
            yield (("pv_done", t), gt - 1)
            arrive(("o_free", t))

    roles = {"tma": tma(), "mma": mma(), "slot A": softmax(0), "slot B": softmax(1)}
    pending = {k: None for k in roles}
    finished = set()
    while len(finished) < len(roles):
        progress = False
        for k, gen in roles.items():
            if k in finished:
                continue
            while True:
                req = pending[k]
                if req is not None:
                    name, phase = req
                    have = done.get(name, 0)
                    if have >= phase + 2:
                        raise ProtocolError(f"{k} waits for phase {phase} of {name}, {have} done")
                    if have < phase + 1:
                        break
                try:
                    pending[k] = next(gen)
                    progress = True
                except StopIteration:
                    finished.add(k)
                    progress = True
                    break
        if not progress:
            raise ProtocolError("deadlock: " + ", ".join(f"{k} on {pending[k]}" for k in roles
                                                         if k not in finished))


def test_bench_batch_item_lists():
    lens, _ = draw_lengths("self_bf16", 1)
    items = block_items(lens, 8)
    for cta in range(0, 148, 7):
        run_model(items, cta, 148)


def random_items(rng, count):
    out = []
    for _ in range(count):
        kind = rng.integers(0, 5)
        a_ = int(rng.integers(1, 7))
        if kind == 0:
            b_ = a_ + 1                                  # a causal block
        elif kind == 1:
            b_ = a_                                      # no causal rule, or a partial block
        elif kind == 2:
            b_ = 0                                       # the sequence ends in the upper rows
        elif kind == 3:
            a_, b_ = 0, int(rng.integers(0, 7))          # the upper rows see no key
        else:
            b_ = int(rng.integers(0, 9))                 # any mix
        out.append((a_, b_, max(a_, b_)))
    return out


def test_random_item_lists():
    rng = np.random.default_rng(11)
    for _ in range(3000):
        run_model(random_items(rng, int(rng.integers(1, 12))))


def test_model_rejects_an_early_score_mma_taken_in_order():
    # the early Q K^T of a slot treated as in item order (wait only as first
    # user, release as last user) reads or frees key tiles out of turn
    rng = np.random.default_rng(12)
    failures = 0
    for _ in range(300):
        try:
            run_model(random_items(rng, int(rng.integers(2, 12))), early_ordered=True)
        except ProtocolError:
            failures += 1
    assert failures > 0
