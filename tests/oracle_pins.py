"""Checks that pin the fp64 oracle to things other than itself.

Each `pin_*` takes an object exposing `attn`, `paged_gather` and
`paged_decode` (the oracle package, or a variant built from a mutated copy
of oracle.c) and raises AssertionError when the oracle disagrees with:

* brute force on tiny inputs (extended precision, no max subtraction);
* closed forms and invariants of softmax attention (rows of P sum to one,
  constant V, a single key, scale 0, causal row 0, identical keys,
  permutation of key/value pairs);
* the online-softmax recurrence for arbitrary tilings and key orders, and the
  split + log-sum-exp merge (FlashAttention optimisation article, 3.2.1-3.2.2);
* an explicit page gather checked against the contiguous rows it was paged from;
* for FP8 inputs: every E4M3 code against torch's float8_e4m3fn conversion and
  the format's closed forms, brute force on the library-decoded values, and the
  bf16 oracle where the descaled values are exactly bfloat16.
"""
from __future__ import annotations

import math

import numpy as np

from online_model import brute_row, online_row, split_combine_row, widen

from tiled_attention_17_b200.inputs import f32_to_bf16_bits

TOL = 1e-12


def _bf16(rng, shape, scale=1.0):
    return f32_to_bf16_bits((rng.standard_normal(shape) * scale).astype(np.float32))


def _visible(i, Nq, Nkv, causal):
    # written out independently of the oracle: count keys j with j <= i + Nkv - Nq
    if not causal:
        return Nkv
    n = 0
    for j in range(Nkv):
        if j <= i + (Nkv - Nq):
            n += 1
    return n


def _close(a, b, tol=TOL, what=""):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    if a.shape != b.shape:
        raise AssertionError(f"{what}: shape {a.shape} vs {b.shape}")
    both_inf = np.isinf(a) & np.isinf(b) & (np.sign(a) == np.sign(b))
    with np.errstate(invalid="ignore"):
        err = np.where(both_inf, 0.0, np.abs(a - b))
    err = np.where(np.isnan(err) & ~both_inf, np.inf, err)
    if not np.all(err <= tol * np.maximum(1.0, np.abs(b))):
        raise AssertionError(f"{what}: max err {np.nanmax(err)} (tol {tol})")


def pin_brute_force(orc):
    rng = np.random.Generator(np.random.PCG64(11))
    shapes = [  # B, Hq, Hkv, Nq, Nkv, d
        (1, 1, 1, 4, 4, 2), (2, 2, 1, 5, 7, 3), (1, 4, 2, 6, 3, 4),
        (1, 2, 2, 8, 8, 4), (1, 3, 1, 1, 6, 2), (1, 1, 1, 7, 5, 3),
    ]
    for (B, Hq, Hkv, Nq, Nkv, d) in shapes:
        for causal in (False, True):
            for scale in (0.7, 1.3):
                q = _bf16(rng, (B, Hq, Nq, d))
                k = _bf16(rng, (B, Hkv, Nkv, d))
                v = _bf16(rng, (B, Hkv, Nkv, d))
                o, lse = orc.attn(q, k, v, causal, scale=scale)
                G = Hq // Hkv
                for b in range(B):
                    for h in range(Hq):
                        kv = h // G
                        for i in range(Nq):
                            ob, lb = brute_row(widen(q[b, h, i]), widen(k[b, kv]), widen(v[b, kv]), scale,
                                               _visible(i, Nq, Nkv, causal))
                            _close(o[b, h, i], ob, what=f"brute o {B,Hq,Hkv,Nq,Nkv,d} c={causal} row {b,h,i}")
                            _close(lse[b, h, i], lb, what=f"brute lse {B,Hq,Hkv,Nq,Nkv,d} c={causal} row {b,h,i}")


def pin_large_scores(orc):
    """Scores of several hundred: a softmax without max subtraction would
    overflow in double; extended-precision brute force does not."""
    rng = np.random.Generator(np.random.PCG64(12))
    q = _bf16(rng, (1, 1, 4, 3), 12.0)
    k = _bf16(rng, (1, 1, 6, 3), 12.0)
    v = _bf16(rng, (1, 1, 6, 3))
    scale = 3.0
    o, lse = orc.attn(q, k, v, False, scale=scale)
    for i in range(4):
        ob, lb = brute_row(widen(q[0, 0, i]), widen(k[0, 0]), widen(v[0, 0]), scale, 6)
        _close(o[0, 0, i], ob, 1e-10, "large-score o")
        _close(lse[0, 0, i], lb, 1e-12, "large-score lse")


def pin_handpicked(orc):
    """q = (1, 0); keys (1,0), (0,1), (-1,0); scale 1: weights e, 1, 1/e."""
    one, zero, neg = 0x3F80, 0x0000, 0xBF80
    q = np.array([[[[one, zero]]]], dtype=np.uint16)
    k = np.array([[[[one, zero], [zero, one], [neg, zero]]]], dtype=np.uint16)
    vals = np.array([[1, 2], [3, 4], [5, 6]], dtype=np.float32)
    v = f32_to_bf16_bits(vals).reshape(1, 1, 3, 2)
    o, lse = orc.attn(q, k, v, False, scale=1.0)
    w = np.array([math.e, 1.0, 1.0 / math.e])
    expect = (w[:, None] * vals).sum(0) / w.sum()
    _close(o[0, 0, 0], expect, what="hand-picked o")
    _close(lse[0, 0, 0], math.log(w.sum()), what="hand-picked lse")
    # causal with Nq = Nkv = 3 would let query 0 see only key 0: O = v_0
    q3 = np.repeat(q, 3, axis=2)
    o3, lse3 = orc.attn(q3, k, v, True, scale=1.0)
    _close(o3[0, 0, 0], vals[0], what="hand-picked causal row 0")
    _close(lse3[0, 0, 0], 1.0, what="hand-picked causal row 0 lse")
    w2 = w[:2]
    _close(o3[0, 0, 1], (w2[:, None] * vals[:2]).sum(0) / w2.sum(), what="hand-picked causal row 1")


def pin_rows_of_p_sum_to_one(orc):
    """With V = identity (d = Nkv) the output row is the probability row."""
    rng = np.random.Generator(np.random.PCG64(13))
    for causal in (False, True):
        Nq, Nkv = 6, 8
        q = _bf16(rng, (1, 1, Nq, 4))
        k = _bf16(rng, (1, 1, Nkv, 4))
        v = f32_to_bf16_bits(np.eye(Nkv, dtype=np.float32)).reshape(1, 1, Nkv, Nkv)
        # identity V needs d == Nkv: pad q/k to d = Nkv with zeros (scores unchanged)
        qp = np.zeros((1, 1, Nq, Nkv), dtype=np.uint16)
        kp = np.zeros((1, 1, Nkv, Nkv), dtype=np.uint16)
        qp[..., :4] = q
        kp[..., :4] = k
        o, _ = orc.attn(qp, kp, v, causal, scale=0.9)
        P = o[0, 0]
        _close(P.sum(axis=1), np.ones(Nq), what=f"row sums causal={causal}")
        if np.any(P < 0):
            raise AssertionError("negative probability")
        if causal:
            for i in range(Nq):
                for j in range(Nkv):
                    if j > i + (Nkv - Nq) and P[i, j] != 0.0:
                        raise AssertionError(f"masked weight P[{i},{j}] = {P[i, j]}")


def pin_constant_v(orc):
    rng = np.random.Generator(np.random.PCG64(14))
    for causal in (False, True):
        c = np.array([1.5, -0.25, 3.0], dtype=np.float32)
        q = _bf16(rng, (1, 2, 5, 3))
        k = _bf16(rng, (1, 1, 5, 3))
        v = np.broadcast_to(f32_to_bf16_bits(c), (1, 1, 5, 3)).copy()
        o, _ = orc.attn(q, k, v, causal, scale=1.1)
        _close(o, np.broadcast_to(c.astype(np.float64), o.shape), what="constant V")


def pin_permutation_invariance(orc):
    rng = np.random.Generator(np.random.PCG64(15))
    q = _bf16(rng, (1, 2, 4, 5))
    k = _bf16(rng, (1, 2, 9, 5))
    v = _bf16(rng, (1, 2, 9, 5))
    o, lse = orc.attn(q, k, v, False, scale=0.8)
    perm = rng.permutation(9)
    o2, lse2 = orc.attn(q, k[:, :, perm], v[:, :, perm], False, scale=0.8)
    _close(o2, o, 1e-13, "permuted o")
    _close(lse2, lse, 1e-13, "permuted lse")


def pin_single_key(orc):
    rng = np.random.Generator(np.random.PCG64(16))
    q = _bf16(rng, (2, 3, 4, 6))
    k = _bf16(rng, (2, 3, 1, 6))
    v = _bf16(rng, (2, 3, 1, 6))
    scale = 0.6
    o, lse = orc.attn(q, k, v, False, scale=scale)
    for b in range(2):
        for h in range(3):
            for i in range(4):
                _close(o[b, h, i], widen(v[b, h, 0]), what="single key o")
                dot = sum(widen(q[b, h, i])[t] * widen(k[b, h, 0])[t] for t in range(6))
                _close(lse[b, h, i], scale * dot, what="single key lse")


def pin_scale_zero(orc):
    rng = np.random.Generator(np.random.PCG64(17))
    for causal in (False, True):
        Nq, Nkv = 5, 7
        q = _bf16(rng, (1, 1, Nq, 3))
        k = _bf16(rng, (1, 1, Nkv, 3))
        v = _bf16(rng, (1, 1, Nkv, 3))
        o, lse = orc.attn(q, k, v, causal, scale=0.0)
        V = widen(v[0, 0])
        for i in range(Nq):
            n = _visible(i, Nq, Nkv, causal)
            _close(o[0, 0, i], V[:n].mean(axis=0), what="scale 0 o")
            _close(lse[0, 0, i], math.log(n), what="scale 0 lse")


def pin_causal_row0(orc):
    rng = np.random.Generator(np.random.PCG64(18))
    q = _bf16(rng, (1, 2, 6, 4))
    k = _bf16(rng, (1, 2, 6, 4))
    v = _bf16(rng, (1, 2, 6, 4))
    o, lse = orc.attn(q, k, v, True, scale=0.5)
    for h in range(2):
        _close(o[0, h, 0], widen(v[0, h, 0]), 0.0, "causal row 0 o")
        dot = float(np.dot(widen(q[0, h, 0]), widen(k[0, h, 0])))
        _close(lse[0, h, 0], 0.5 * dot, what="causal row 0 lse")


def pin_identical_keys(orc):
    rng = np.random.Generator(np.random.PCG64(19))
    q = _bf16(rng, (1, 1, 3, 4))
    k = np.broadcast_to(_bf16(rng, (1, 1, 1, 4)), (1, 1, 6, 4)).copy()
    v = _bf16(rng, (1, 1, 6, 4))
    o, _ = orc.attn(q, k, v, False, scale=1.0)
    _close(o[0, 0], np.broadcast_to(widen(v[0, 0]).mean(axis=0), (3, 4)), what="identical keys")


def pin_online_recurrence(orc):
    rng = np.random.Generator(np.random.PCG64(20))
    Nkv, d = 37, 8
    q = _bf16(rng, (1, 1, 3, d), 2.0)
    k = _bf16(rng, (1, 1, Nkv, d))
    v = _bf16(rng, (1, 1, Nkv, d))
    k[0, 0, ::5] = f32_to_bf16_bits(widen(k[0, 0, ::5]).astype(np.float32) * 4)   # sharp peaks
    scale = 0.9
    o, lse = orc.attn(q, k, v, False, scale=scale)
    K, V = widen(k[0, 0]), widen(v[0, 0])
    for trial in range(20):
        order = rng.permutation(Nkv) if trial % 2 else np.arange(Nkv)
        cuts = np.sort(rng.choice(np.arange(1, Nkv), size=rng.integers(0, 8), replace=False))
        blocks = np.split(order, cuts)
        thr = 0.0 if trial % 3 else 8.0 * math.log(2.0)
        for i in range(3):
            oo, ll = online_row(widen(q[0, 0, i]), K, V, scale, blocks, thr)
            _close(o[0, 0, i], oo, what="online vs oracle o")
            _close(lse[0, 0, i], ll, what="online vs oracle lse")
            os_, ls_ = split_combine_row(widen(q[0, 0, i]), K, V, scale, blocks)
            _close(o[0, 0, i], os_, what="split+combine vs oracle o")
            _close(lse[0, 0, i], ls_, what="split+combine vs oracle lse")


def _page(K, V, page_size, Hkv, rng, extra=3):
    """Page contiguous per-sequence K/V ([S][Hkv, len, d] lists) into a pool."""
    S = len(K)
    d = K[0].shape[-1]
    lens = [x.shape[1] for x in K]
    npages = [(L + page_size - 1) // page_size for L in lens]
    total = sum(npages) + extra
    perm = rng.permutation(total)
    max_pages = max(max(npages), 1) + 1
    table = np.full((S, max_pages), -1, dtype=np.int32)
    kc = _bf16(rng, (total, Hkv, page_size, d))      # unused slots hold junk
    vc = _bf16(rng, (total, Hkv, page_size, d))
    off = 0
    for s in range(S):
        for t in range(npages[s]):
            slot = perm[off + t]
            table[s, t] = slot
            lo, hi = t * page_size, min(lens[s], (t + 1) * page_size)
            kc[slot, :, :hi - lo] = K[s][:, lo:hi]
            vc[slot, :, :hi - lo] = V[s][:, lo:hi]
        off += npages[s]
    return kc, vc, table, np.array(lens, dtype=np.int32)


def pin_paged_gather(orc):
    rng = np.random.Generator(np.random.PCG64(21))
    Hkv, d, ps = 2, 4, 4
    lens = [5, 8, 1, 13, 0]
    K = [_bf16(rng, (Hkv, L, d)) for L in lens]
    V = [_bf16(rng, (Hkv, L, d)) for L in lens]
    kc, vc, table, sl = _page(K, V, ps, Hkv, rng)
    for s in range(len(lens)):
        for h in range(Hkv):
            kg, vg = orc.paged_gather(kc, vc, table, sl, s, h)
            if not (np.array_equal(kg, K[s][h]) and np.array_equal(vg, V[s][h])):
                raise AssertionError(f"gather mismatch seq {s} head {h}")
    bad = table.copy()
    bad[0, 1] = kc.shape[0]
    try:
        orc.paged_gather(kc, vc, bad, sl, 0, 0)
    except RuntimeError:
        pass
    else:
        raise AssertionError("out-of-range block-table entry was not rejected")


def pin_paged_decode(orc):
    """Decode through the pool equals attention on the rows before paging."""
    rng = np.random.Generator(np.random.PCG64(22))
    Hq, Hkv, d, ps = 4, 2, 4, 4
    lens = [5, 8, 1, 13, 3]
    K = [_bf16(rng, (Hkv, L, d)) for L in lens]
    V = [_bf16(rng, (Hkv, L, d)) for L in lens]
    kc, vc, table, sl = _page(K, V, ps, Hkv, rng)
    q = _bf16(rng, (len(lens), Hq, d))
    scale = 0.7
    o, lse = orc.paged_decode(q, kc, vc, table, sl, scale=scale)
    G = Hq // Hkv
    for s in range(len(lens)):
        for h in range(Hq):
            ob, lb = brute_row(widen(q[s, h]), widen(K[s][h // G]), widen(V[s][h // G]), scale, lens[s])
            _close(o[s, h], ob, what=f"decode o seq {s} head {h}")
            _close(lse[s, h], lb, what=f"decode lse seq {s} head {h}")


def _varlen_batch(rng, q_lens, kv_lens, Hq, Hkv, d, page_size):
    """Packed queries, per-sequence contiguous K/V and their paged copy."""
    S = len(q_lens)
    cu = np.zeros(S + 1, dtype=np.int32)
    cu[1:] = np.cumsum(q_lens)
    q = _bf16(rng, (int(cu[-1]), Hq, d))
    K = [_bf16(rng, (Hkv, L, d)) for L in kv_lens]
    V = [_bf16(rng, (Hkv, L, d)) for L in kv_lens]
    kc, vc, table, lens = _page(K, V, page_size, Hkv, rng)
    return q, K, V, kc, vc, table, cu, lens


def pin_paged_prefill_brute_force(orc):
    # every packed query row against its own sequence's keys, by brute force on
    # the contiguous rows (extended precision, explicit visibility count)
    rng = np.random.Generator(np.random.PCG64(31))
    for (q_lens, kv_lens, Hq, Hkv, d, ps) in [([3, 1, 4], [5, 2, 4], 2, 1, 3, 2),
                                               ([2, 5], [7, 5], 4, 2, 2, 3),
                                               ([4, 0, 3], [4, 3, 9], 1, 1, 4, 4)]:
        for causal in (False, True):
            q, K, V, kc, vc, table, cu, lens = _varlen_batch(rng, q_lens, kv_lens, Hq, Hkv, d, ps)
            o, lse = orc.paged_prefill(q, kc, vc, table, cu, lens, causal, scale=0.9)
            G = Hq // Hkv
            for s, (ql, L) in enumerate(zip(q_lens, kv_lens)):
                for h in range(Hq):
                    for i in range(ql):
                        row = cu[s] + i
                        ob, lb = brute_row(widen(q[row, h]), widen(K[s][h // G]), widen(V[s][h // G]), 0.9,
                                           _visible(i, ql, L, causal))
                        _close(o[row, h], ob, what=f"paged prefill o seq {s} row {i} c={causal}")
                        _close(lse[row, h], lb, what=f"paged prefill lse seq {s} row {i} c={causal}")


def pin_paged_prefill_one_query_is_decode(orc):
    # one new token per sequence is the paged decode
    rng = np.random.Generator(np.random.PCG64(32))
    kv_lens = [9, 1, 17, 6]
    q, K, V, kc, vc, table, cu, lens = _varlen_batch(rng, [1] * 4, kv_lens, 4, 2, 3, 4)
    o, lse = orc.paged_prefill(q, kc, vc, table, cu, lens, True, scale=0.7)
    od, ld = orc.paged_decode(q, kc, vc, table, lens, scale=0.7)
    _close(o, od, what="one query vs decode o")
    _close(lse, ld, what="one query vs decode lse")


def pin_paged_prefill_matches_dense(orc):
    # one sequence through the pool equals the contiguous attention of its rows
    rng = np.random.Generator(np.random.PCG64(33))
    for causal in (False, True):
        q, K, V, kc, vc, table, cu, lens = _varlen_batch(rng, [2, 6], [3, 11], 2, 2, 4, 4)
        o, lse = orc.paged_prefill(q, kc, vc, table, cu, lens, causal, scale=0.5)
        qs = np.ascontiguousarray(q[cu[1]:cu[2]].transpose(1, 0, 2))[None]
        od, ld = orc.attn(qs, K[1][None], V[1][None], causal, scale=0.5)
        _close(o[cu[1]:cu[2]], od[0].transpose(1, 0, 2), what="paged prefill vs dense o")
        _close(lse[cu[1]:cu[2]], ld[0].T, what="paged prefill vs dense lse")


# ---------------------------------------------------------------------------
# Backward pass (gradients of attention)
# ---------------------------------------------------------------------------

def _forward_f64(Q, K, V, scale, causal):
    """Attention written out in fp64 on float inputs (not bf16 bits), independent
    of the oracle: explicit mask, softmax with the row max subtracted, O = P V.
    Q [B,Hq,Nq,d], K/V [B,Hkv,Nkv,d]."""
    B, Hq, Nq, d = Q.shape
    Hkv, Nkv = K.shape[1], K.shape[2]
    G = Hq // Hkv
    O = np.zeros_like(Q)
    for b in range(B):
        for h in range(Hq):
            kv = h // G
            S = scale * (Q[b, h] @ K[b, kv].T)
            for i in range(Nq):
                vis = _visible(i, Nq, Nkv, causal)
                if vis == 0:
                    continue
                srow = S[i, :vis]
                e = np.exp(srow - srow.max())
                O[b, h, i] = (e / e.sum()) @ V[b, kv, :vis]
    return O


def pin_bwd_finite_differences(orc):
    # directional derivatives of L = sum(dO * O) by central differences of an
    # independent fp64 forward, against <grad, direction> from the oracle
    rng = np.random.Generator(np.random.PCG64(21))
    for (B, Hq, Hkv, Nq, Nkv, d) in [(1, 2, 1, 5, 6, 3), (1, 1, 1, 4, 4, 2), (2, 4, 2, 3, 7, 2)]:
        for causal in (False, True):
            scale = 0.8
            q, k, v, do = (_bf16(rng, (B, Hq, Nq, d)), _bf16(rng, (B, Hkv, Nkv, d)),
                           _bf16(rng, (B, Hkv, Nkv, d)), _bf16(rng, (B, Hq, Nq, d)))
            dq, dk, dv = orc.attn_bwd(q, k, v, do, causal, scale=scale)
            X = [widen(q), widen(k), widen(v)]
            dO = widen(do)
            grads = [dq, dk, dv]
            eps = 1e-5
            for which in range(3):
                for trial in range(3):
                    E = rng.standard_normal(X[which].shape)
                    Xp = [x.copy() for x in X]
                    Xm = [x.copy() for x in X]
                    Xp[which] += eps * E
                    Xm[which] -= eps * E
                    fd = (np.sum(dO * _forward_f64(*Xp, scale, causal)) -
                          np.sum(dO * _forward_f64(*Xm, scale, causal))) / (2 * eps)
                    an = float(np.sum(grads[which] * E))
                    if abs(fd - an) > 1e-6 * max(1.0, abs(fd)):
                        raise AssertionError(f"bwd finite differences ({'qkv'[which]}) {B,Hq,Hkv,Nq,Nkv,d} "
                                             f"c={causal}: {an} vs {fd}")


def pin_bwd_single_key(orc):
    # one key: P = 1 for every row that sees it, so dQ = dK = 0 and
    # dV_0 = sum of dO over those rows (all query heads of the group)
    rng = np.random.Generator(np.random.PCG64(22))
    for (B, Hq, Hkv, Nq) in [(1, 2, 1, 5), (2, 4, 2, 3)]:
        for causal in (False, True):
            q, k, v, do = (_bf16(rng, (B, Hq, Nq, 4)), _bf16(rng, (B, Hkv, 1, 4)),
                           _bf16(rng, (B, Hkv, 1, 4)), _bf16(rng, (B, Hq, Nq, 4)))
            dq, dk, dv = orc.attn_bwd(q, k, v, do, causal, scale=1.1)
            _close(dq, np.zeros_like(dq), what="single key dq")
            _close(dk, np.zeros_like(dk), what="single key dk")
            G = Hq // Hkv
            want = np.zeros_like(dv)
            for b in range(B):
                for h in range(Hq):
                    for i in range(Nq):
                        if _visible(i, Nq, 1, causal) > 0:
                            want[b, h // G, 0] += widen(do[b, h, i])
            _close(dv, want, what="single key dv")


def pin_bwd_scale_zero(orc):
    # scale 0: uniform weights over the visible keys, no gradient reaches Q or K
    rng = np.random.Generator(np.random.PCG64(23))
    B, Hq, Hkv, Nq, Nkv, d = 1, 2, 1, 6, 4, 3
    for causal in (False, True):
        q, k, v, do = (_bf16(rng, (B, Hq, Nq, d)), _bf16(rng, (B, Hkv, Nkv, d)),
                       _bf16(rng, (B, Hkv, Nkv, d)), _bf16(rng, (B, Hq, Nq, d)))
        dq, dk, dv = orc.attn_bwd(q, k, v, do, causal, scale=0.0)
        _close(dq, np.zeros_like(dq), what="scale 0 dq")
        _close(dk, np.zeros_like(dk), what="scale 0 dk")
        want = np.zeros_like(dv)
        for h in range(Hq):
            for i in range(Nq):
                n = _visible(i, Nq, Nkv, causal)
                for j in range(n):
                    want[0, 0, j] += widen(do[0, h, i]) / n
        _close(dv, want, what="scale 0 dv")


def pin_bwd_key_gradients_sum_to_zero(orc):
    # each row of dS sums to zero (softmax is shift invariant), hence
    # sum_j dK_j = 0 for every KV head
    rng = np.random.Generator(np.random.PCG64(24))
    for (B, Hq, Hkv, Nq, Nkv, d) in [(1, 2, 1, 9, 9, 5), (2, 3, 3, 4, 11, 4)]:
        for causal in (False, True):
            q, k, v, do = (_bf16(rng, (B, Hq, Nq, d)), _bf16(rng, (B, Hkv, Nkv, d)),
                           _bf16(rng, (B, Hkv, Nkv, d)), _bf16(rng, (B, Hq, Nq, d)))
            _, dk, _ = orc.attn_bwd(q, k, v, do, causal, scale=0.9)
            _close(dk.sum(axis=2), np.zeros((B, Hkv, d)), tol=1e-11, what="sum of dK")


def pin_bwd_permutation(orc):
    # non-causal: permuting the (k_j, v_j) pairs permutes dK and dV the same
    # way and leaves dQ unchanged
    rng = np.random.Generator(np.random.PCG64(25))
    B, Hq, Hkv, Nq, Nkv, d = 1, 2, 2, 5, 8, 4
    q, k, v, do = (_bf16(rng, (B, Hq, Nq, d)), _bf16(rng, (B, Hkv, Nkv, d)),
                   _bf16(rng, (B, Hkv, Nkv, d)), _bf16(rng, (B, Hq, Nq, d)))
    perm = rng.permutation(Nkv)
    dq, dk, dv = orc.attn_bwd(q, k, v, do, False, scale=0.6)
    dq2, dk2, dv2 = orc.attn_bwd(q, k[:, :, perm], v[:, :, perm], do, False, scale=0.6)
    _close(dq2, dq, tol=1e-11, what="perm dq")
    _close(dk2, dk[:, :, perm], tol=1e-11, what="perm dk")
    _close(dv2, dv[:, :, perm], tol=1e-11, what="perm dv")


def pin_bwd_grouped_heads(orc):
    # a KV head shared by G query heads gets the sum of the gradients it would
    # get as G separate copies (one per query head)
    rng = np.random.Generator(np.random.PCG64(26))
    B, Hq, Hkv, Nq, Nkv, d = 2, 4, 2, 5, 6, 3
    G = Hq // Hkv
    for causal in (False, True):
        q, k, v, do = (_bf16(rng, (B, Hq, Nq, d)), _bf16(rng, (B, Hkv, Nkv, d)),
                       _bf16(rng, (B, Hkv, Nkv, d)), _bf16(rng, (B, Hq, Nq, d)))
        dq, dk, dv = orc.attn_bwd(q, k, v, do, causal, scale=0.7)
        kr, vr = np.repeat(k, G, axis=1), np.repeat(v, G, axis=1)
        dq1, dk1, dv1 = orc.attn_bwd(q, kr, vr, do, causal, scale=0.7)
        _close(dq1, dq, tol=1e-11, what="gqa dq")
        _close(dk1.reshape(B, Hkv, G, Nkv, d).sum(axis=2), dk, tol=1e-11, what="gqa dk")
        _close(dv1.reshape(B, Hkv, G, Nkv, d).sum(axis=2), dv, tol=1e-11, what="gqa dv")


# --------------------------------------------------------------------------
# FP8 (E4M3) inputs
# --------------------------------------------------------------------------

def _torch_e4m3(codes):
    """E4M3 codes -> float64 through torch's float8_e4m3fn type (a library
    conversion, independent of the oracle's decoder)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def _fp8(rng, shape):
    from tiled_attention_17_b200.inputs import quantize_e4m3
    codes, _ = quantize_e4m3(rng.standard_normal(int(np.prod(shape))).astype(np.float32))
    return codes.reshape(shape)


def pin_e4m3_codes(orc):
    codes = np.arange(256, dtype=np.uint8)
    got = orc.e4m3_decode(codes)
    ref = _torch_e4m3(codes)
    nan = np.isnan(ref)
    if not np.array_equal(np.isnan(got), nan):
        raise AssertionError("e4m3: NaN codes differ from the library's")
    if not np.array_equal(got[~nan], ref[~nan]):
        bad = np.nonzero(got[~nan] != ref[~nan])[0][:4]
        raise AssertionError(f"e4m3: codes {codes[~nan][bad]} decode to {got[~nan][bad]}, library {ref[~nan][bad]}")
    # closed forms of the format: smallest subnormal, smallest normal, one, largest finite, signs
    for code, val in ((0x01, 2.0 ** -9), (0x08, 2.0 ** -6), (0x38, 1.0), (0x7E, 448.0), (0xB8, -1.0),
                      (0xFE, -448.0)):
        if got[code] != val:
            raise AssertionError(f"e4m3 code {code:#x}: {got[code]} != {val}")
    if not (np.isnan(got[0x7F]) and np.isnan(got[0xFF])):
        raise AssertionError("e4m3: S.1111.111 must be NaN")


def pin_fp8_brute_force(orc):
    """FP8 attention on tiny inputs against the textbook definition evaluated
    on the library-decoded, descaled values."""
    rng = np.random.Generator(np.random.PCG64(19))
    for (B, Hq, Hkv, Nq, Nkv, d) in ((1, 2, 1, 5, 7, 4), (2, 2, 2, 6, 6, 3), (1, 1, 1, 3, 9, 8)):
        for causal in (False, True):
            q8, k8, v8 = _fp8(rng, (B, Hq, Nq, d)), _fp8(rng, (B, Hkv, Nkv, d)), _fp8(rng, (B, Hkv, Nkv, d))
            desc = (0.037, 0.0081, 0.0059)
            scale = 0.9
            o, lse = orc.attn_fp8(q8, k8, v8, desc, causal, scale=scale)
            Q, K, V = (_torch_e4m3(x) * s for x, s in zip((q8, k8, v8), desc))
            G = Hq // Hkv
            for b in range(B):
                for h in range(Hq):
                    for i in range(Nq):
                        ob, lb = brute_row(Q[b, h, i], K[b, h // G], V[b, h // G], scale,
                                           _visible(i, Nq, Nkv, causal))
                        _close(o[b, h, i], ob, what=f"fp8 brute o row {b, h, i}")
                        _close(lse[b, h, i], lb, what=f"fp8 brute lse row {b, h, i}")


def pin_fp8_is_bf16_attention(orc):
    """Every E4M3 value times a power of two (within range) is a bfloat16 value,
    so FP8 attention with power-of-two descales must equal the bf16 oracle on
    those values, to rounding."""
    rng = np.random.Generator(np.random.PCG64(23))
    B, Hq, Hkv, Nq, Nkv, d = 1, 4, 2, 40, 56, 16
    q8, k8, v8 = _fp8(rng, (B, Hq, Nq, d)), _fp8(rng, (B, Hkv, Nkv, d)), _fp8(rng, (B, Hkv, Nkv, d))
    for desc in ((1.0, 1.0, 1.0), (2.0 ** -6, 2.0 ** -7, 4.0)):
        bits = [f32_to_bf16_bits((_torch_e4m3(x) * s).astype(np.float32)) for x, s in zip((q8, k8, v8), desc)]
        for causal in (False, True):
            o8, l8 = orc.attn_fp8(q8, k8, v8, desc, causal, scale=0.25)
            ob, lb = orc.attn(*bits, causal, scale=0.25)
            _close(o8, ob, tol=1e-12, what=f"fp8 vs bf16 o desc={desc} causal={causal}")
            _close(l8, lb, tol=1e-12, what=f"fp8 vs bf16 lse desc={desc} causal={causal}")


FP8_PINS = [pin_e4m3_codes, pin_fp8_brute_force, pin_fp8_is_bf16_attention]

BWD_PINS = [pin_bwd_finite_differences, pin_bwd_single_key, pin_bwd_scale_zero,
            pin_bwd_key_gradients_sum_to_zero, pin_bwd_permutation, pin_bwd_grouped_heads]

ALL_PINS = [pin_brute_force, pin_large_scores, pin_handpicked, pin_rows_of_p_sum_to_one,
            pin_constant_v, pin_permutation_invariance, pin_single_key, pin_scale_zero,
            pin_causal_row0, pin_identical_keys, pin_online_recurrence, pin_paged_gather,
            pin_paged_decode, pin_paged_prefill_brute_force, pin_paged_prefill_one_query_is_decode,
            pin_paged_prefill_matches_dense] + BWD_PINS + FP8_PINS
