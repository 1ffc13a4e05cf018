"""Pins of the CPU oracle against things other than itself (CPU only).

Each check below ties one part of the oracle to a closed form, a brute-force
enumeration of the definition, a hand-worked fixture, or a library routine
(torch scaled_dot_product_attention / autograd in float64).  The last test
plants mistakes in copies of oracle functions and checks that some pin fails.
"""

import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle import hga_oracle as ho
from hierarchical_routed_sparse_hga_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ----------------------------------------------------------------------------
# helpers
# ----------------------------------------------------------------------------

def tiny_case(seed=0, topk_blocks=2, topk_groups=5, ctx=384, seg=128, first_seg=2,
              hq=4, hkv=2, d=16, batch=2):
    w = synth.custom(batch=batch, n_q_heads=hq, n_kv_heads=hkv, head_dim=d, ctx_len=ctx,
                     seg_len=seg, topk_blocks=topk_blocks, topk_groups=topk_groups,
                     seed=seed, first_seg=first_seg)
    k = synth.widen(synth.keys(w), "f32")
    v = synth.widen(synth.values(w), "f32")
    q_begin = w.segments()[0]
    q = synth.widen(synth.queries(w, q_begin), "f32")
    do = synth.widen(synth.douts(w, q_begin), "f32")
    return w, q, k, v, do, q_begin


def summaries_upto(k, t_end):
    return oracle.build_summaries(k, 0, t_end)


def brute_force_route(q, k, q_begin, topk_blocks, topk_groups, hkv):
    """Literal definition: score = mean over (query, head, key) triples of q.k/sqrt(d)."""
    B, Hq, S, d = q.shape
    G = Hq // hkv
    out_blk, out_grp = {}, {}
    for b in range(B):
        for h in range(hkv):
            for j in range(S // 64):
                own = (q_begin + 64 * j) // 64
                qs = [q[b, hh, 64 * j + t] for hh in range(h * G, (h + 1) * G) for t in range(64)]

                def score(positions):
                    tot = 0.0
                    for qq in qs:
                        for p in positions:
                            tot += float(np.dot(qq, k[b, h, p])) / math.sqrt(d)
                    return tot / (len(qs) * len(positions))

                blk_scores = [(score(range(64 * c, 64 * c + 64)), c) for c in range(own)]
                blk_sorted = sorted(blk_scores, key=lambda sc: (-sc[0], sc[1]))
                chosen = sorted(c for _, c in blk_sorted[:topk_blocks])
                grp_scores = [(score(range(8 * g, 8 * g + 8)), g)
                              for c in chosen for g in range(8 * c, 8 * c + 8)]
                grp_sorted = sorted(grp_scores, key=lambda sc: (-sc[0], sc[1]))
                out_blk[(b, h, j)] = chosen
                out_grp[(b, h, j)] = sorted(g for _, g in grp_sorted[:topk_groups])
    return out_blk, out_grp


def keyset_mask(q_begin, S, T, sel_grp_bh):
    """[S, T] bool: query row t sees key p (routed groups + own block causal)."""
    mask = np.zeros((S, T), bool)
    for t in range(S):
        j = t // 64
        for p in oracle.keyset(q_begin, j, t % 64, sel_grp_bh[j]):
            mask[t, p] = True
    return mask


def sdpa_reference(q, k, v, do, q_begin, masks, hkv):
    """float64 torch SDPA with explicit masks; gradients by autograd with the
    history detached.  masks: [B, Hkv, S, T] bool.  Returns o, lse, dq, dk, dv."""
    B, Hq, S, d = q.shape
    G = Hq // hkv
    T = q_begin + S
    qt = torch.tensor(q, requires_grad=True)
    k_hist = torch.tensor(k[:, :, :q_begin])
    v_hist = torch.tensor(v[:, :, :q_begin])
    k_act = torch.tensor(k[:, :, q_begin:T], requires_grad=True)
    v_act = torch.tensor(v[:, :, q_begin:T], requires_grad=True)
    kf = torch.cat([k_hist, k_act], dim=2).repeat_interleave(G, dim=1)
    vf = torch.cat([v_hist, v_act], dim=2).repeat_interleave(G, dim=1)
    m = torch.tensor(masks).repeat_interleave(G, dim=1)
    o = F.scaled_dot_product_attention(qt, kf, vf, attn_mask=m)
    (o * torch.tensor(do)).sum().backward()
    s = (qt.detach() @ kf.transpose(-1, -2)) / math.sqrt(d)
    lse = torch.logsumexp(s.masked_fill(~m, -math.inf), dim=-1)
    return (o.detach().numpy(), lse.detach().numpy(), qt.grad.numpy(), k_act.grad.numpy(),
            v_act.grad.numpy())


def close(a, b, tol=1e-10):
    return np.max(np.abs(np.asarray(a) - np.asarray(b))) <= tol * max(1.0, np.max(np.abs(b)))


# ----------------------------------------------------------------------------
# pins: summaries
# ----------------------------------------------------------------------------

def check_summaries_closed_form():
    # K[t] = a + b*t per dimension: the mean of an arithmetic run is its midpoint
    d, T = 3, 256
    a, bb = np.array([1.0, -2.0, 0.5]), np.array([0.25, 1.0, -3.0])
    k = (a[None, :] + bb[None, :] * np.arange(T)[:, None])[None, None]
    g, bl = oracle.build_summaries(k, 64, 256)
    for i in range(g.shape[2]):
        first = 64 + 8 * i
        assert close(g[0, 0, i], a + bb * (first + 3.5))
    for i in range(bl.shape[2]):
        first = 64 + 64 * i
        assert close(bl[0, 0, i], a + bb * (first + 31.5))


def test_summaries_closed_form():
    check_summaries_closed_form()


def test_block_summary_is_mean_of_its_groups():
    _, q, k, v, do, q_begin = tiny_case()
    g, bl = oracle.build_summaries(k, 0, k.shape[2])
    B, H, nb, d = bl.shape
    assert close(bl, g.reshape(B, H, nb, 8, d).mean(axis=3))


# ----------------------------------------------------------------------------
# pins: routing
# ----------------------------------------------------------------------------

def golden_inputs(fx, group_x, own_x=None):
    x = np.array(fx[group_x], float)
    if own_x is not None:
        x[32:] = own_x
    T = fx["q_begin"] + fx["seg_len"]
    k = np.zeros((1, 1, T, 2))
    k[0, 0, :, 0] = np.repeat(x, 8)
    k[0, 0, :, 1] = fx["key_y"]
    q = np.zeros((1, 1, fx["seg_len"], 2))
    q[0, 0, :, :] = fx["query"]
    return q, k


def check_route_golden():
    fx = json.load(open(os.path.join(GOLDEN, "route_attn_handworked.json")))
    for case in fx["cases"]:
        q, k = golden_inputs(fx, case["group_x"])
        g, bl = summaries_upto(k, k.shape[2])
        sb, sg, _ = oracle.route(q, bl, g, fx["q_begin"], case["topk_blocks"],
                                 case["topk_groups"], 1)
        assert list(sb[0, 0, 0]) == case["sel_blk"], case["name"]
        if isinstance(case["sel_grp"], str):       # case D: everything selected
            want = list(range(32)) + [-1] * 8
        else:
            want = case["sel_grp"]
        assert list(sg[0, 0, 0]) == want, case["name"]


def test_route_golden():
    check_route_golden()


def check_route_bruteforce(seed=0):
    w, q, k, v, do, q_begin = tiny_case(seed=seed)
    g, bl = summaries_upto(k, k.shape[2])
    sb, sg, tie = oracle.route(q, bl, g, q_begin, w.topk_blocks, w.topk_groups, w.n_kv_heads)
    bb, bg = brute_force_route(q, k, q_begin, w.topk_blocks, w.topk_groups, w.n_kv_heads)
    n = 0
    for key, blocks in bb.items():
        if tie[key]:
            continue
        n += 1
        assert [c for c in sb[key] if c >= 0] == blocks, key
        assert [c for c in sg[key] if c >= 0] == bg[key], key
    assert n >= len(bb) - 1


@pytest.mark.parametrize("seed", [0, 1])
def test_route_bruteforce(seed):
    check_route_bruteforce(seed)


def test_route_exact_ties_take_lower_index():
    # every block identical -> every block ties; lowest indices win at both levels
    d = 4
    rng = np.random.default_rng(5)
    one_block = rng.standard_normal((64, d))
    k = np.tile(one_block, (6, 1))[None, None]
    q = rng.standard_normal((1, 1, 64, d))
    g, bl = summaries_upto(k, k.shape[2])
    sb, sg, tie = oracle.route(q, bl, g, 320, 3, 5, 1)
    assert list(sb[0, 0, 0]) == [0, 1, 2]
    # groups inside a block differ, so level 2 keeps the same within-block
    # ranking in every block; ties across blocks go to the lower block
    order = np.argsort(-(one_block.reshape(8, 8, d).mean(axis=1) @ q[0, 0].mean(axis=0)),
                       kind="stable")
    want = sorted([int(order[0]), int(order[0]) + 8, int(order[0]) + 16,
                   int(order[1]), int(order[1]) + 8])
    assert list(sg[0, 0, 0]) == want
    assert tie[0, 0, 0]


def test_route_first_block_has_no_candidates():
    w, q, k, v, do, _ = tiny_case(first_seg=0)
    g, bl = summaries_upto(k, 128)
    sb, sg, tie = oracle.route(q, bl, g, 0, 2, 5, w.n_kv_heads)
    assert (sb[:, :, 0] == -1).all() and (sg[:, :, 0] == -1).all()
    assert (sb[:, :, 1, 0] == 0).all() and (sb[:, :, 1, 1] == -1).all()


def _tie_case(block_x, group_x=None, topk_blocks=2, topk_groups=5):
    """route() on hand-built summaries (d = 2, one head, one query block whose
    queries are all (1, 0)), so every score is block_x[c]/sqrt(2) at level 1
    and group_x[g]/sqrt(2) at level 2.  Returns (sel_blk, sel_grp, flag)."""
    nb = len(block_x)
    if group_x is None:                  # well separated: no level-2 tie
        group_x = [100.0 - 1.7 * g for g in range(8 * nb)]
    bsum = np.zeros((1, 1, nb + 1, 2))
    bsum[0, 0, :nb, 0] = block_x
    gsum = np.zeros((1, 1, 8 * (nb + 1), 2))
    gsum[0, 0, :8 * nb, 0] = group_x
    q = np.zeros((1, 1, 64, 2))
    q[..., 0] = 1.0
    sb, sg, tie = oracle.route(q, bsum, gsum, 64 * nb, topk_blocks, topk_groups, 1)
    return list(sb[0, 0, 0]), list(sg[0, 0, 0]), bool(tie[0, 0, 0])


def check_near_tie_flags():
    """The near-tie flag, by hand: set iff the k-th and (k+1)-th sorted scores
    of a level differ by at most 1e-3 of the larger magnitude."""
    rel_in, rel_out = 2.0 * (1 - 0.9e-3), 2.0 * (1 - 1.1e-3)
    # level 1, the gap at the k boundary just inside / just outside the window
    sb, _, f = _tie_case([3.0, 2.0, rel_in, 0.5])
    assert f and sb == [0, 1]
    assert not _tie_case([3.0, 2.0, rel_out, 0.5])[2]
    # a close pair next to (not at) the boundary does not flag: (k+1, k+2), (k-1, k)
    assert not _tie_case([3.0, 2.0, 1.0, 0.9995])[2]
    assert not _tie_case([3.0, 2.9995, 1.0, 0.5])[2]
    # the window is relative: large scores 0.5 apart flag, tiny ones 5e-4 apart do not
    assert _tie_case([1000.0, 999.5, 10.0], topk_blocks=1)[2]
    assert not _tie_case([1e-3, 5e-4, 1e-4], topk_blocks=1)[2]
    # no (k+1)-th score when k covers every candidate: exact ties do not flag
    sb, sg, f = _tie_case([1.0, 1.0], group_x=[1.0] * 16, topk_blocks=4, topk_groups=16)
    assert not f and sb == [0, 1, -1, -1] and sg == list(range(16))
    # the first query block has no candidates at all
    assert not _tie_case([], topk_blocks=2)[2]
    # level 2 alone: blocks 0, 1 clear of block 2; groups' 5th/6th scores in or out
    gx = [50.0, 40.0, 30.0, 20.0, 10.0, 10.0 * (1 - 0.9e-3), 1.0, 0.5] + [0.1 * i for i in range(8)]
    _, sg, f = _tie_case([3.0, 2.0, 0.5], group_x=gx + [0.0] * 8)
    assert f and sg == [0, 1, 2, 3, 4]
    gx[5] = 10.0 * (1 - 1.1e-3)
    assert not _tie_case([3.0, 2.0, 0.5], group_x=gx + [0.0] * 8)[2]


def test_near_tie_flags():
    check_near_tie_flags()


def test_planted_target_ranks_first():
    # statistical sanity check on the tiny fp32 workload (not an exactness test)
    w = synth.workloads()["tiny_f32"]
    k = synth.widen(synth.keys(w), w.dtype)
    q_begin = w.segments()[0]
    q = synth.widen(synth.queries(w, q_begin), w.dtype)
    g, bl = summaries_upto(k, k.shape[2])
    hits = 0
    for j in range(w.seg_len // 64):
        s = bl[0, 0, :(q_begin // 64 + j)] @ q[0, 0, 64 * j:64 * j + 64].mean(axis=0)
        hits += int(np.argmax(s) == synth.targets(w, 0, 0, q_begin)[j])
    assert hits == w.seg_len // 64


# ----------------------------------------------------------------------------
# pins: attention forward / backward
# ----------------------------------------------------------------------------

def check_attention_golden():
    fx = json.load(open(os.path.join(GOLDEN, "route_attn_handworked.json")))
    q, k = golden_inputs(fx, "group_x_case_A", own_x=0.0)
    T = k.shape[2]
    v = np.zeros((1, 1, T, 2))
    grp = np.arange(T) // 8
    v[0, 0, :, 0] = np.where(grp < 32, grp, 0)
    v[0, 0, :, 1] = np.where(grp < 32, 0, 1)
    g, bl = summaries_upto(k, T)
    _, sg, _ = oracle.route(q, bl, g, fx["q_begin"], 2, 3, 1)
    o, lse = oracle.attn_fwd(q, k, v, fx["q_begin"], sg, 1)
    env = {"exp": math.exp, "log": math.log, "sqrt": math.sqrt}
    for r in range(64):
        env["r"] = r
        assert abs(lse[0, 0, r] - eval(fx["lse_row_expr"], env)) < 1e-12
        assert abs(o[0, 0, r, 0] - eval(fx["o_row_expr"][0], env)) < 1e-12
        assert abs(o[0, 0, r, 1] - eval(fx["o_row_expr"][1], env)) < 1e-12


def test_attention_golden():
    check_attention_golden()


def check_dense_equivalence(seed=1):
    # top-k covering every candidate block and group -> dense causal attention
    w, q, k, v, do, q_begin = tiny_case(seed=seed, topk_blocks=8, topk_groups=64)
    T = q_begin + w.seg_len
    g, bl = summaries_upto(k, T)
    _, sg, _ = oracle.route(q, bl, g, q_begin, w.topk_blocks, w.topk_groups, w.n_kv_heads)
    o, lse = oracle.attn_fwd(q, k, v, q_begin, sg, w.n_kv_heads)
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, q_begin, sg, w.n_kv_heads)
    pos_q = q_begin + np.arange(w.seg_len)
    causal = np.arange(T)[None, :] <= pos_q[:, None]            # textbook causal mask
    masks = np.broadcast_to(causal, (w.batch, w.n_kv_heads, w.seg_len, T))
    ro, rlse, rdq, rdk, rdv = sdpa_reference(q, k[:, :, :T], v[:, :, :T], do, q_begin,
                                             masks, w.n_kv_heads)
    assert close(o, ro) and close(lse, rlse)
    assert close(dq, rdq) and close(dk, rdk) and close(dv, rdv)


def test_dense_equivalence_fwd_bwd():
    check_dense_equivalence()


def check_masked_sdpa(seed=2):
    # general selection: the oracle equals SDPA with the keyset as its mask
    w, q, k, v, do, q_begin = tiny_case(seed=seed)
    T = q_begin + w.seg_len
    g, bl = summaries_upto(k, T)
    _, sg, _ = oracle.route(q, bl, g, q_begin, w.topk_blocks, w.topk_groups, w.n_kv_heads)
    o, lse = oracle.attn_fwd(q, k, v, q_begin, sg, w.n_kv_heads)
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, q_begin, sg, w.n_kv_heads)
    masks = np.stack([np.stack([keyset_mask(q_begin, w.seg_len, T, sg[b, h])
                                for h in range(w.n_kv_heads)]) for b in range(w.batch)])
    ro, rlse, rdq, rdk, rdv = sdpa_reference(q, k[:, :, :T], v[:, :, :T], do, q_begin,
                                             masks, w.n_kv_heads)
    assert close(o, ro) and close(lse, rlse)
    assert close(dq, rdq) and close(dk, rdk) and close(dv, rdv)


def test_masked_sdpa_general_selection():
    check_masked_sdpa()


def check_finite_differences():
    w, q, k, v, do, q_begin = tiny_case(seed=3, batch=1, hq=2, hkv=1, d=4, ctx=192, seg=128,
                                        first_seg=0, topk_blocks=1, topk_groups=3)
    # first_seg=0: segment [0,128) is active; second segment [128,192) unused
    q_begin = 0
    T = 128
    k = k.copy()
    g, bl = summaries_upto(k, T)
    _, sg, _ = oracle.route(q, bl, g, q_begin, 1, 3, 1)
    dq, dk, dv = oracle.attn_bwd(q, k, v, do, q_begin, sg, 1)

    def loss(qq, kk, vv):
        o, _ = oracle.attn_fwd(qq, kk, vv, q_begin, sg, 1)
        return float((o * do).sum())

    rng = np.random.default_rng(0)
    eps = 1e-6
    for name, arr, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv)):
        for _ in range(6):
            idx = tuple(int(rng.integers(0, n)) for n in grad.shape)
            plus, minus = arr.copy(), arr.copy()
            plus[idx] += eps
            minus[idx] -= eps
            args_p = {"q": (plus, k, v), "k": (q, plus, v), "v": (q, k, plus)}[name]
            args_m = {"q": (minus, k, v), "k": (q, minus, v), "v": (q, k, minus)}[name]
            fd = (loss(*args_p) - loss(*args_m)) / (2 * eps)
            assert abs(fd - grad[idx]) < 1e-6 * max(1.0, abs(fd)), (name, idx)


def test_finite_differences():
    check_finite_differences()


def test_rows_sum_to_one_and_keyset_bound():
    w, q, k, v, do, q_begin = tiny_case(seed=4)
    T = q_begin + w.seg_len
    g, bl = summaries_upto(k, T)
    _, sg, _ = oracle.route(q, bl, g, q_begin, w.topk_blocks, w.topk_groups, w.n_kv_heads)
    o, lse = oracle.attn_fwd(q, k, v, q_begin, sg, w.n_kv_heads)
    G = w.group_heads
    for b in range(w.batch):
        for hq in range(w.n_q_heads):
            h = hq // G
            for t in range(w.seg_len):
                j, r = divmod(t, 64)
                ks = oracle.keyset(q_begin, j, r, sg[b, h, j])
                assert len(ks) <= 8 * w.topk_groups + 64
                assert len(set(ks.tolist())) == len(ks)          # routed groups avoid own block
                s = k[b, h, ks] @ q[b, hq, t] / math.sqrt(w.head_dim)
                assert abs(np.exp(s - lse[b, hq, t]).sum() - 1.0) < 1e-12


def test_history_gets_no_gradient_and_segments_chain():
    # three segments over 384 tokens; dk/dv cover exactly the active slice
    w, q, k, v, do, _ = tiny_case(first_seg=0, topk_blocks=2, topk_groups=6)
    T = w.ctx_len
    gsum = np.zeros((w.batch, w.n_kv_heads, T // 8, w.head_dim))
    bsum = np.zeros((w.batch, w.n_kv_heads, T // 64, w.head_dim))
    for q_begin in w.segments():
        qq = synth.widen(synth.queries(w, q_begin), "f32")
        dd = synth.widen(synth.douts(w, q_begin), "f32")
        out = oracle.segment_step(qq, k, v, dd, q_begin, gsum, bsum, w.topk_blocks,
                                  w.topk_groups, w.n_kv_heads)
        assert out["dk"].shape == (w.batch, w.n_kv_heads, w.seg_len, w.head_dim)
        # every routed group lies strictly before the query block's own block
        for j in range(w.seg_len // 64):
            own = (q_begin + 64 * j) // 64
            sel = out["sel_grp"][:, :, j]
            assert ((sel < 0) | (sel // 8 < own)).all()
    g_all, b_all = oracle.build_summaries(k, 0, T)
    assert close(gsum, g_all) and close(bsum, b_all)


# ----------------------------------------------------------------------------
# planted mistakes: each mutated oracle must fail at least one pin
# ----------------------------------------------------------------------------

def _mut_route_wrong_heads(q, bsum, gsum, q_begin, kb, kg, hkv):
    # mean over the wrong GQA head group (next group)
    B, Hq, S, d = q.shape
    G = Hq // hkv
    q2 = np.roll(q, -G, axis=1)
    return ORIG["route"](q2, bsum, gsum, q_begin, kb, kg, hkv)


def _mut_topk_higher_index(scores, idx, k):
    order = np.lexsort((-idx, -scores))
    return idx[order[:k]], scores[order]


def _mut_block_keys_strict(q_begin, j, sel_row):
    keys, visible = ORIG["_block_keys"](q_begin, j, sel_row)
    n_routed = len(keys) - 64
    visible = visible.copy()
    visible[:, n_routed:] &= ~np.eye(64, dtype=bool)            # diagonal dropped
    return keys, visible


def _mut_summaries_sum(k, t_begin, t_end):
    g, b = ORIG["build_summaries"](k, t_begin, t_end)
    return g * 8, b                                               # group sum, not mean


def _mut_near_tie_next_pair(sorted_scores, k):
    # compares the (k+1)-th and (k+2)-th scores instead of the k-th and (k+1)-th
    if k + 1 >= len(sorted_scores) or k == 0:
        return False
    a, b = sorted_scores[k], sorted_scores[k + 1]
    return abs(a - b) <= ho.TIE_REL * max(abs(a), abs(b))


def _mut_near_tie_absolute(sorted_scores, k):
    # an absolute window instead of a relative one
    if k >= len(sorted_scores) or k == 0:
        return False
    return abs(sorted_scores[k - 1] - sorted_scores[k]) <= ho.TIE_REL


class _MutNearTieLevel1Only:
    """route() asks level 1 first and level 2 only when level 1 did not flag;
    this mutant answers level 2 with False (the level-2 flag dropped)."""

    def __init__(self):
        self.level2_next = False

    def __call__(self, sorted_scores, k):
        if self.level2_next:
            self.level2_next = False
            return False
        flag = ORIG["_near_tie"](sorted_scores, k)
        self.level2_next = not flag
        return flag


ORIG = {"route": ho.route, "_topk_lower_index": ho._topk_lower_index,
        "_block_keys": ho._block_keys, "build_summaries": ho.build_summaries,
        "_near_tie": ho._near_tie}

ALL_PINS = [check_summaries_closed_form, check_route_golden, check_route_bruteforce,
            check_attention_golden, check_dense_equivalence, check_masked_sdpa,
            check_finite_differences, check_near_tie_flags]


@pytest.mark.parametrize("target,mutant", [
    ("route", _mut_route_wrong_heads),
    ("_topk_lower_index", _mut_topk_higher_index),
    ("_block_keys", _mut_block_keys_strict),
    ("build_summaries", _mut_summaries_sum),
    ("_near_tie", _mut_near_tie_next_pair),
    ("_near_tie", _mut_near_tie_absolute),
    ("_near_tie", _MutNearTieLevel1Only()),
])
def test_pins_catch_planted_mistakes(monkeypatch, target, mutant):
    monkeypatch.setattr(ho, target, mutant)
    if hasattr(oracle, target):
        monkeypatch.setattr(oracle, target, mutant)
    failed = 0
    for pin in ALL_PINS:
        try:
            pin()
        except (AssertionError, IndexError):
            failed += 1
    assert failed >= 1, f"no pin caught the planted mistake in {target}"


# ----------------------------------------------------------------------------
# pins: host tier (dedup + remap)
# ----------------------------------------------------------------------------

def test_tier_stage_preserves_attention():
    # staging the distinct selected history groups and remapping the selection
    # must leave every output and gradient unchanged
    w, q, k, v, do, q_begin = tiny_case(seed=6, topk_blocks=3, topk_groups=7)
    S, T = w.seg_len, q_begin + w.seg_len
    g, bl = summaries_upto(k, T)
    _, sg, _ = oracle.route(q, bl, g, q_begin, w.topk_blocks, w.topk_groups, w.n_kv_heads)
    n_qb = S // 64
    stage_cap = ((min(n_qb * w.topk_groups, q_begin // 8) * 8 + 63) // 64) * 64 + S
    uniq, sel_st = oracle.tier_stage(sg, q_begin, S, stage_cap)
    ks = np.full((w.batch, w.n_kv_heads, stage_cap, w.head_dim), np.nan)
    vs = np.full_like(ks, np.nan)
    for b in range(w.batch):
        for h in range(w.n_kv_heads):
            u = uniq[b][h]
            assert (np.diff(u) > 0).all() and (u < q_begin // 8).all()
            rows = (u[:, None] * 8 + np.arange(8)[None, :]).reshape(-1)
            ks[b, h, :len(rows)] = k[b, h, rows]
            vs[b, h, :len(rows)] = v[b, h, rows]
    ks[:, :, stage_cap - S:] = k[:, :, q_begin:T]
    vs[:, :, stage_cap - S:] = v[:, :, q_begin:T]
    o1, l1 = oracle.attn_fwd(q, k, v, q_begin, sg, w.n_kv_heads)
    o2, l2 = oracle.attn_fwd(q, ks, vs, stage_cap - S, sel_st, w.n_kv_heads)
    assert close(o1, o2, 1e-13) and close(l1, l2, 1e-13)
    g1 = oracle.attn_bwd(q, k, v, do, q_begin, sg, w.n_kv_heads)
    g2 = oracle.attn_bwd(q, ks, vs, do, stage_cap - S, sel_st, w.n_kv_heads)
    for a, b_ in zip(g1, g2):
        assert close(a, b_, 1e-13)
    # every history group any query block selected is staged exactly once
    for b in range(w.batch):
        for h in range(w.n_kv_heads):
            sel = sg[b, h]
            want = sorted(set(int(x) for x in sel.ravel() if 0 <= x < q_begin // 8))
            assert list(uniq[b][h]) == want


# ----------------------------------------------------------------------------
# pins: decode (one token per sequence)
# ----------------------------------------------------------------------------

def decode_case(seed=4, ctx=640, hq=4, hkv=2, d=16, batch=3, topk_blocks=3, topk_groups=7):
    w = synth.custom(batch=batch, n_q_heads=hq, n_kv_heads=hkv, head_dim=d, ctx_len=ctx,
                     seg_len=64, topk_blocks=topk_blocks, topk_groups=topk_groups,
                     seed=seed, first_seg=0)
    k = synth.widen(synth.keys(w), "f32")
    v = synth.widen(synth.values(w), "f32")
    rng = np.random.default_rng(seed)
    q_tok = rng.standard_normal((batch, hq, d))
    return w, q_tok, k, v


def check_decode_against_prefill():
    """A query block whose 64 rows all carry the same query routes exactly as
    a decode step of that query at any position of the block, and row r of
    its attention is the decode step at position 64J + r."""
    w, q_tok, k, v = decode_case()
    B, Hq, d = q_tok.shape
    g, bl = summaries_upto(k, w.ctx_len)
    for J in (0, 1, 4, 9):
        q_blk = np.repeat(q_tok[:, :, None, :], 64, axis=2)
        sb, sg, tie = oracle.route(q_blk, bl, g, 64 * J, w.topk_blocks, w.topk_groups, 2)
        o_blk, lse_blk = oracle.attn_fwd(q_blk, k, v, 64 * J, sg, 2)
        for r in (0, 17, 63):
            pos = [64 * J + r] * B
            db, dg, dtie = oracle.decode_route(q_tok, bl, g, pos, w.topk_blocks,
                                               w.topk_groups, 2)
            assert np.array_equal(db, sb[:, :, 0]) and np.array_equal(dg, sg[:, :, 0])
            assert np.array_equal(dtie, tie[:, :, 0])
            o, lse = oracle.decode_attn(q_tok, k, v, pos, dg, 2)
            assert close(o, o_blk[:, :, r]) and close(lse, lse_blk[:, :, r])


def test_decode_against_prefill():
    check_decode_against_prefill()


def check_decode_dense_equivalence():
    """top-k covering every candidate: a decode step is dense causal attention
    of that one query over every earlier token and itself (torch SDPA, f64)."""
    w, q_tok, k, v = decode_case(topk_blocks=64, topk_groups=256)
    g, bl = summaries_upto(k, w.ctx_len)
    pos = [5, 200, 639]
    _, sg, _ = oracle.decode_route(q_tok, bl, g, pos, 64, 256, 2)
    o, lse = oracle.decode_attn(q_tok, k, v, pos, sg, 2)
    G = 2
    for b, p in enumerate(pos):
        for hq in range(4):
            kk = torch.from_numpy(k[b, hq // G, :p + 1])
            vv = torch.from_numpy(v[b, hq // G, :p + 1])
            qq = torch.from_numpy(q_tok[b, hq])[None]
            ref = F.scaled_dot_product_attention(qq[None], kk[None], vv[None])[0, 0].numpy()
            assert close(o[b, hq], ref)
            s = (kk.numpy() @ q_tok[b, hq]) / math.sqrt(q_tok.shape[-1])
            assert abs(lse[b, hq] - (s.max() + math.log(np.exp(s - s.max()).sum()))) < 1e-12


def test_decode_dense_equivalence():
    check_decode_dense_equivalence()


def check_decode_route_bruteforce():
    """Literal definition: block score = mean over the G heads and the
    block's 64 keys of q.k/sqrt(d); exhaustive sort by (-score, index)."""
    w, q_tok, k, v = decode_case(seed=8)
    B, Hq, d = q_tok.shape
    G = Hq // 2
    g, bl = summaries_upto(k, w.ctx_len)
    pos = [64 * 7 + 3, 64 * 9 + 63, 64 * 2]
    sb, sg, tie = oracle.decode_route(q_tok, bl, g, pos, w.topk_blocks, w.topk_groups, 2)
    for b in range(B):
        for h in range(2):
            if tie[b, h]:
                continue
            qs = [q_tok[b, hh] for hh in range(h * G, (h + 1) * G)]

            def score(keys):
                return sum(float(qq @ k[b, h, t]) for qq in qs for t in keys) / (
                    len(qs) * len(keys) * math.sqrt(d))
            J = pos[b] // 64
            blocks = sorted(range(J), key=lambda c: (-score(range(64 * c, 64 * c + 64)), c))
            blocks = sorted(blocks[:w.topk_blocks])
            groups = [8 * c + i for c in blocks for i in range(8)]
            groups = sorted(groups, key=lambda gg: (-score(range(8 * gg, 8 * gg + 8)), gg))
            groups = sorted(groups[:w.topk_groups])
            assert [x for x in sb[b, h] if x >= 0] == blocks
            assert [x for x in sg[b, h] if x >= 0] == groups


def test_decode_route_bruteforce():
    check_decode_route_bruteforce()


def test_decode_first_block_attends_only_itself():
    w, q_tok, k, v = decode_case()
    g, bl = summaries_upto(k, w.ctx_len)
    sb, sg, tie = oracle.decode_route(q_tok, bl, g, [0, 1, 63], 3, 7, 2)
    assert (sb == -1).all() and (sg == -1).all() and not tie.any()
    o, lse = oracle.decode_attn(q_tok, k, v, [0, 1, 63], sg, 2)
    assert close(o[0], np.repeat(v[0, :, 0], 2, axis=0))      # one key: O = its value
    assert close(lse[0], (q_tok[0] * np.repeat(k[0, :, 0], 2, axis=0)).sum(-1) / 4.0)


def _mut_decode_own_block_candidate(q_tok, bsum, gsum, pos, kb, kg, hkv):
    # the incomplete own block scored as a candidate too
    return ORIG_DECODE["decode_route"](q_tok, bsum, gsum, [p + 64 for p in pos], kb, kg, hkv)


def _mut_decode_attn_without_itself(q_tok, k, v, pos, sel_grp, hkv):
    # the token does not attend to its own key
    return ORIG_DECODE["decode_attn"](q_tok, k, v, [p - 1 for p in pos], sel_grp, hkv)


ORIG_DECODE = {"decode_route": ho.decode_route, "decode_attn": ho.decode_attn}
DECODE_PINS = [check_decode_against_prefill, check_decode_dense_equivalence,
               check_decode_route_bruteforce]


@pytest.mark.parametrize("target,mutant", [
    ("decode_route", _mut_decode_own_block_candidate),
    ("decode_attn", _mut_decode_attn_without_itself),
])
def test_decode_pins_catch_planted_mistakes(monkeypatch, target, mutant):
    monkeypatch.setattr(ho, target, mutant)
    monkeypatch.setattr(oracle, target, mutant)
    failed = 0
    for pin in DECODE_PINS:
        try:
            pin()
        except (AssertionError, IndexError, ValueError):
            failed += 1
    assert failed >= 1, f"no pin caught the planted mistake in {target}"


# ----------------------------------------------------------------------------
# pins: strictly causal routing (the query block routed with the mean query
# of the 64 tokens before it)
# ----------------------------------------------------------------------------

def causal_case(seed=21, B=2, hq=4, hkv=2, d=16, n_blocks=8, kb=2, kg=5):
    rng = np.random.default_rng(seed)
    T = 64 * n_blocks
    cent = rng.standard_normal((B, hkv, n_blocks, d))
    k = np.repeat(cent, 64, axis=2) + 0.5 * rng.standard_normal((B, hkv, T, d))
    q_all = rng.standard_normal((B, hq, T, d))
    return k, q_all, kb, kg, hkv


def causal_selection(k, q_all, q_begin, S, kb, kg, hkv):
    g, bl = summaries_upto(k, k.shape[2])
    qs = oracle.query_summaries(q_all, hkv)                 # [B, Hkv, T/64, d]
    J0 = q_begin // 64
    prev = np.zeros((qs.shape[0], hkv, S // 64, qs.shape[-1]))
    for j in range(S // 64):
        if J0 + j >= 1:
            prev[:, :, j] = qs[:, :, J0 + j - 1]
    return oracle.route_causal(prev, bl, g, q_begin, S // 64, kb, kg)


def check_query_summaries():
    k, q_all, kb, kg, hkv = causal_case()
    qs = oracle.query_summaries(q_all, hkv)
    B, Hq, T, d = q_all.shape
    G = Hq // hkv
    for b in range(B):
        for h in range(hkv):
            for J in range(T // 64):
                rows = [q_all[b, hh, t] for hh in range(h * G, (h + 1) * G)
                        for t in range(64 * J, 64 * J + 64)]
                assert close(qs[b, h, J], sum(rows) / len(rows))


def test_query_summaries():
    check_query_summaries()


def check_causal_route_uses_no_later_token():
    """Changing the queries of block J or of any later token leaves the
    selections of blocks <= J as they were; changing block J-1's queries
    changes some selection (the routing does depend on them)."""
    k, q_all, kb, kg, hkv = causal_case()
    q_begin, S = 128, 384
    base = causal_selection(k, q_all, q_begin, S, kb, kg, hkv)
    rng = np.random.default_rng(5)
    for J in (3, 5):
        q2 = q_all.copy()
        q2[:, :, 64 * J:] = rng.standard_normal(q2[:, :, 64 * J:].shape) * 3
        sb, sg, _ = causal_selection(k, q2, q_begin, S, kb, kg, hkv)
        upto = J - q_begin // 64 + 1                        # query blocks J0 .. J
        assert np.array_equal(sb[:, :, :upto], base[0][:, :, :upto])
        assert np.array_equal(sg[:, :, :upto], base[1][:, :, :upto])
    changed = 0
    for J in range(3, 8):
        q2 = q_all.copy()
        q2[:, :, 64 * (J - 1):64 * J] = -q2[:, :, 64 * (J - 1):64 * J]
        sb, sg, _ = causal_selection(k, q2, q_begin, S, kb, kg, hkv)
        changed += int(not np.array_equal(sg, base[1]))
    assert changed >= 3


def test_causal_route_uses_no_later_token():
    check_causal_route_uses_no_later_token()


def check_causal_route_bruteforce():
    """Literal definition: the score of block c for query block J is the mean
    over the previous block's 64 tokens, the G heads and c's 64 keys of
    q.k/sqrt(d); exhaustive sort by (-score, index)."""
    k, q_all, kb, kg, hkv = causal_case(seed=22, d=8, n_blocks=6)
    B, Hq, T, d = q_all.shape
    G = Hq // hkv
    q_begin, S = 64, 320
    sb, sg, tie = causal_selection(k, q_all, q_begin, S, kb, kg, hkv)
    for b in range(B):
        for h in range(hkv):
            for j in range(S // 64):
                J = q_begin // 64 + j
                if tie[b, h, j]:
                    continue
                qs = [q_all[b, hh, t] for hh in range(h * G, (h + 1) * G)
                      for t in range(64 * (J - 1), 64 * J)]

                def score(keys):
                    return sum(float(qq @ k[b, h, t]) for qq in qs for t in keys) / (
                        len(qs) * len(keys) * math.sqrt(d))
                blocks = sorted(range(J), key=lambda c: (-score(range(64 * c, 64 * c + 64)), c))
                blocks = sorted(blocks[:kb])
                groups = [8 * c + i for c in blocks for i in range(8)]
                groups = sorted(groups, key=lambda gg: (-score(range(8 * gg, 8 * gg + 8)), gg))
                groups = sorted(groups[:kg])
                assert [x for x in sb[b, h, j] if x >= 0] == blocks
                assert [x for x in sg[b, h, j] if x >= 0] == groups


def test_causal_route_bruteforce():
    check_causal_route_bruteforce()


def _mut_query_summaries_wrong_group(q, hkv):
    return ORIG_CAUSAL["query_summaries"](np.roll(q, -(q.shape[1] // hkv), axis=1), hkv)


def _mut_route_causal_own_block(q_prev_mean, bsum, gsum, q_begin, n_qb, kb, kg):
    # routes block j with block j's own mean (shifted one block too late):
    # emulated by moving every row one block back, the last from the next
    shifted = np.concatenate([q_prev_mean[:, :, 1:], q_prev_mean[:, :, -1:]], axis=2)
    return ORIG_CAUSAL["route_causal"](shifted, bsum, gsum, q_begin, n_qb, kb, kg)


ORIG_CAUSAL = {"query_summaries": ho.query_summaries, "route_causal": ho.route_causal}
CAUSAL_PINS = [check_query_summaries, check_causal_route_uses_no_later_token,
               check_causal_route_bruteforce]


@pytest.mark.parametrize("target,mutant", [
    ("query_summaries", _mut_query_summaries_wrong_group),
    ("route_causal", _mut_route_causal_own_block),
])
def test_causal_pins_catch_planted_mistakes(monkeypatch, target, mutant):
    monkeypatch.setattr(ho, target, mutant)
    monkeypatch.setattr(oracle, target, mutant)
    failed = 0
    for pin in CAUSAL_PINS:
        try:
            pin()
        except (AssertionError, IndexError, ValueError):
            failed += 1
    assert failed >= 1, f"no pin caught the planted mistake in {target}"


# ----------------------------------------------------------------------------
# pins: the upstream pass (RoPE, storage rounding, layout)
# ----------------------------------------------------------------------------

def check_rope_closed_forms():
    rng = np.random.default_rng(30)
    d, base = 16, 1e6
    x = rng.standard_normal((2, 5, d))
    # complex form: pair (x_i, x_{i+d/2}) as x_i + j x_{i+d/2}, times e^{j p theta_i}
    pos0 = 1000
    y = oracle.rope(x, pos0, base)
    half = d // 2
    theta = np.array([base ** (-2.0 * i / d) for i in range(half)])
    for t in range(5):
        z = (x[:, t, :half] + 1j * x[:, t, half:]) * np.exp(1j * (pos0 + t) * theta)
        assert close(y[:, t, :half], z.real) and close(y[:, t, half:], z.imag)
    # position 0 is the identity; every pair keeps its length
    assert close(oracle.rope(x[:, :1], 0, base), x[:, :1])
    assert close(y[..., :half] ** 2 + y[..., half:] ** 2, x[..., :half] ** 2 + x[..., half:] ** 2)
    # q.k depends only on the distance between the two positions
    q, k = rng.standard_normal((1, d)), rng.standard_normal((1, d))
    a = float(oracle.rope(q, 37, base)[0] @ oracle.rope(k, 5, base)[0])
    b = float(oracle.rope(q, 5037, base)[0] @ oracle.rope(k, 5005, base)[0])
    assert abs(a - b) < 1e-9


def test_rope_closed_forms():
    check_rope_closed_forms()


def check_round_bf16():
    # ties go to even, and torch's float32 -> bfloat16 conversion (round to
    # nearest even) agrees on float32 values
    assert list(oracle.round_bf16(np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8)]))) == \
        [1.0, 1 + 2 ** -6, -1.0]
    rng = np.random.default_rng(31)
    x = (rng.standard_normal(4096) * 10.0 ** rng.integers(-3, 4, 4096)).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(oracle.round_bf16(x.astype(np.float64)), ref)


def test_round_bf16():
    check_round_bf16()


def check_prepare_layout():
    """Token-major projections become head-major tensors; without RoPE and at
    float32 the values pass through unchanged; the summaries and the block
    mean queries are those of the stored tensors."""
    rng = np.random.default_rng(32)
    B, S, Hq, Hkv, d = 2, 128, 4, 2, 8
    qp = rng.standard_normal((B, S, Hq, d)).astype(np.float32).astype(np.float64)
    kp = rng.standard_normal((B, S, Hkv, d)).astype(np.float32).astype(np.float64)
    vp = rng.standard_normal((B, S, Hkv, d)).astype(np.float32).astype(np.float64)
    q, k, v, g, bl, qs = oracle.prepare_segment(qp, kp, vp, 64, None, Hkv, "f32")
    assert np.array_equal(q[1, 3, 70], qp[1, 70, 3]) and np.array_equal(k[0, 1, 5], kp[0, 5, 1])
    assert np.array_equal(v[1, 0, 127], vp[1, 127, 0])
    assert close(g[0, 1, 3], kp[0, 24:32, 1].mean(0)) and close(bl[1, 0, 1], kp[1, 64:, 0].mean(0))
    assert close(qs[0, 1, 0], qp[0, :64, 2:4].mean((0, 1)))
    q2, k2, *_ = oracle.prepare_segment(qp, kp, vp, 64, 1e4, Hkv, "bf16")
    assert np.array_equal(q2, oracle.round_bf16(oracle.rope(q, 64, 1e4)))


def test_prepare_layout():
    check_prepare_layout()


def _mut_rope_sign(x, pos0, base):
    # the rotation turned the other way (sine with the wrong sign)
    d = x.shape[-1]
    y = ORIG_PREP["rope"](x[..., ::1], -pos0, base)
    return y if pos0 else np.concatenate([y[..., :d // 2], -y[..., d // 2:]], axis=-1)


def _mut_rope_freq(x, pos0, base):
    return ORIG_PREP["rope"](x, pos0, base ** 0.5)


def _mut_round_half_up(x):
    m, e = np.frexp(np.asarray(x, np.float64))
    return np.ldexp(np.floor(np.ldexp(m, 8) + 0.5), e - 8)


ORIG_PREP = {"rope": ho.rope, "round_bf16": ho.round_bf16}
PREP_PINS = [check_rope_closed_forms, check_round_bf16, check_prepare_layout]


@pytest.mark.parametrize("target,mutant", [
    ("rope", _mut_rope_sign), ("rope", _mut_rope_freq), ("round_bf16", _mut_round_half_up),
])
def test_prepare_pins_catch_planted_mistakes(monkeypatch, target, mutant):
    monkeypatch.setattr(ho, target, mutant)
    monkeypatch.setattr(oracle, target, mutant)
    failed = 0
    for pin in PREP_PINS:
        try:
            pin()
        except (AssertionError, IndexError, ValueError):
            failed += 1
    assert failed >= 1, f"no pin caught the planted mistake in {target}"
