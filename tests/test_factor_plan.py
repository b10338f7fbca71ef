"""The factorisation's schedule, replayed on the CPU (host logic; no GPU).

``gptq_factor_plan`` lists the launches (leaf factorisations, GEMMs, copies)
and stream events of the blocked Cholesky with its merge tree exactly as
``gptq_quantize_layer`` enqueues them.  Here the plan is

* executed in float64 numpy in random orders that its streams and events
  allow, with each GEMM following the kernel's 128 x 128 tile rules (the flags
  that skip triangular tiles), and compared with the oracle's U -- the upper
  Cholesky factor of H_d^-1 ("LLM 量化技术" blog §2.3 item 3; GPTQ reading card,
  方法适配);
* checked for races: any two launches that no stream order or event orders
  must not write what the other reads or writes.
"""

from __future__ import annotations

import re

import numpy as np
import pytest

import oracle
from synth import make_problem

T = 128   # GEMM tile


def _plan(d, S, side):
    from post_weight_quantization_19_b200 import gptq_factor_plan
    return gptq_factor_plan(d, S, side)


_REF = re.compile(r"^(\w)\+(\d+)$")


def _ref(s):
    m = _REF.match(s)
    assert m, s
    return m.group(1), int(m.group(2))


def parse(text):
    head, ops = None, []
    for ln in text.strip().splitlines():
        kind, rest = ln.split(" ", 1)
        kv = dict(p.split("=", 1) for p in rest.split())
        if kind == "P":
            head = {k: int(v) for k, v in kv.items()}
            continue
        op = {"kind": kind, "s": int(kv["s"])}
        if kind == "L":
            op.update(A=_ref(kv["A"]), ld=int(kv["ld"]), nb=int(kv["nb"]))
        elif kind == "G":
            op.update({k: int(kv[k]) for k in ("M", "N", "K", "lda", "ldb", "ldc", "flags", "tb",
                                               "prio")})
            op.update(alpha=float(kv["alpha"]), beta=float(kv["beta"]), A=_ref(kv["A"]),
                      B=_ref(kv["B"]), C=_ref(kv["C"]))
        elif kind == "C":
            op.update(dst=_ref(kv["dst"]), src=_ref(kv["src"]),
                      **{k: int(kv[k]) for k in ("ldd", "lds", "rows", "cols")})
        else:
            op["e"] = int(kv["e"])
        ops.append(op)
    return head, ops


# ---------------------------------------------------------------- dependencies

def dag(ops):
    """Predecessors of every op: program order per stream plus event edges."""
    last = {}
    rec = {}
    preds = [set() for _ in ops]
    for i, op in enumerate(ops):
        s = op["s"]
        if s in last:
            preds[i].add(last[s])
        if op["kind"] == "E":
            rec[op["e"]] = i
        elif op["kind"] == "W":
            preds[i].add(rec[op["e"]])
        last[s] = i
    return preds


def reach(preds):
    """reach[i]: bitset of ops that must complete before op i."""
    out = []
    for i, ps in enumerate(preds):
        r = 0
        for p in ps:
            r |= out[p] | (1 << p)
        out.append(r)
    return out


# ---------------------------------------------------------------- access sets

def _view(ref, ld, d):
    """(buffer, row0, col0, ld) of a pointer; A views must have row stride d."""
    buf, off = ref
    return buf, off // ld if buf == "A" else 0, off % ld if buf == "A" else off, ld


def _rects(buf, base, ld, rows, cols, d):
    """Rectangles (buf, r0, r1, c0, c1) covered by a rows x cols view.

    A is addressed as a d x d matrix; T views become one conservative 1-D
    interval (row 0, columns = flat offsets)."""
    r0, r1 = rows
    c0, c1 = cols
    if r1 <= r0 or c1 <= c0:
        return []
    if buf == "A":
        assert ld == d
        br, bc = divmod(base, d)
        return [("A", br + r0, br + r1, bc + c0, bc + c1)]
    return [("T", 0, 1, base + r0 * ld + c0, base + (r1 - 1) * ld + c1)]


def _k_range(op, m0, n0):
    klo, khi = 0, op["K"]
    if op["flags"] & 1:
        klo = max(klo, m0)
    if op["flags"] & 2:
        klo = max(klo, n0)
    if op["flags"] & 4:
        khi = min(khi, n0 + T)
    return klo, khi


def _tiles(op):
    M, N = op["M"], op["N"]
    for m0 in range(0, M, T):
        for n0 in range(0, N, T):
            if (op["flags"] & 8) and n0 < m0:
                continue
            yield m0, n0


def access(op, d):
    """(reads, writes) as lists of rectangles."""
    k = op["kind"]
    if k == "L":
        buf, off = op["A"]
        rr = _rects(buf, off, op["ld"], (0, op["nb"]), (0, op["nb"]), d)
        return rr, rr
    if k == "C":
        r = _rects(op["src"][0], op["src"][1], op["lds"], (0, op["rows"]), (0, op["cols"]), d)
        w = _rects(op["dst"][0], op["dst"][1], op["ldd"], (0, op["rows"]), (0, op["cols"]), d)
        return r, w
    if k != "G":
        return [], []
    reads, writes = [], []
    arow, bcol = {}, {}
    for m0, n0 in _tiles(op):
        klo, khi = _k_range(op, m0, n0)
        m1, n1 = min(op["M"], m0 + T), min(op["N"], n0 + T)
        writes += _rects(op["C"][0], op["C"][1], op["ldc"], (m0, m1), (n0, n1), d)
        if op["beta"] != 0.0:
            reads += _rects(op["C"][0], op["C"][1], op["ldc"], (m0, m1), (n0, n1), d)
        if khi > klo:
            a = arow.setdefault(m0, [khi, klo])
            a[0], a[1] = min(a[0], klo), max(a[1], khi)
            b = bcol.setdefault(n0, [khi, klo])
            b[0], b[1] = min(b[0], klo), max(b[1], khi)
    for m0, (klo, khi) in arow.items():
        reads += _rects(op["A"][0], op["A"][1], op["lda"], (m0, min(op["M"], m0 + T)), (klo, khi),
                        d)
    for n0, (klo, khi) in bcol.items():
        n1 = min(op["N"], n0 + T)
        if op["tb"]:
            reads += _rects(op["B"][0], op["B"][1], op["ldb"], (n0, n1), (klo, khi), d)
        else:
            reads += _rects(op["B"][0], op["B"][1], op["ldb"], (klo, khi), (n0, n1), d)
    return reads, writes


def _overlap(a, b):
    return (a[0] == b[0] and a[1] < b[2] and b[1] < a[2] and a[3] < b[4] and b[3] < a[4])


def _any_overlap(xs, ys):
    return any(_overlap(x, y) for x in xs for y in ys)


def _bbox(rs):
    out = {}
    for r in rs:
        b = out.get(r[0])
        out[r[0]] = (r if b is None else
                     (r[0], min(b[1], r[1]), max(b[2], r[2]), min(b[3], r[3]), max(b[4], r[4])))
    return list(out.values())


def races(ops, d):
    preds = dag(ops)
    rch = reach(preds)
    acc = [access(op, d) for op in ops]
    live = [i for i, op in enumerate(ops) if op["kind"] in "LGC"]
    boxes = {i: (_bbox(acc[i][0] + acc[i][1]), _bbox(acc[i][1])) for i in live}
    found = []
    for x, i in enumerate(live):
        for j in live[x + 1:]:
            if (rch[j] >> i) & 1 or (rch[i] >> j) & 1:
                continue
            # unordered: i's writes vs j's accesses, j's writes vs i's accesses
            if not (_any_overlap(boxes[i][1], boxes[j][0]) or _any_overlap(boxes[j][1],
                                                                           boxes[i][0])):
                continue
            ri, wi = acc[i]
            rj, wj = acc[j]
            if _any_overlap(wi, rj + wj) or _any_overlap(wj, ri):
                found.append((i, j))
    return found


def inplace_ok(op, d):
    """A GEMM whose A or B operand overlaps its output may only read it
    tile-privately: one column tile, A the same view as C (each output tile
    then reads only its own rows, all before it writes), B disjoint from C."""
    _, writes = access(op, d)
    ab = access(dict(op, beta=0.0), d)[0]
    bonly = access(dict(op, beta=0.0, A=("Z", 0), lda=op["lda"]), d)[0]
    bonly = [r for r in bonly if r[0] != "Z"]
    if not _any_overlap(writes, ab):
        return True
    a_is_c = op["A"] == op["C"] and op["lda"] == op["ldc"]
    return op["N"] <= T and a_is_c and not _any_overlap(writes, bonly)


# ---------------------------------------------------------------- execution

def _mat(bufs, ref, ld, rows, cols):
    buf, off = ref
    flat = bufs[buf]
    idx = off + np.arange(rows)[:, None] * ld + np.arange(cols)[None, :]
    return flat, idx


def run(ops, bufs, d, rng):
    preds = dag(ops)
    n = len(ops)
    indeg = [len(p) for p in preds]
    succ = [[] for _ in range(n)]
    for i, ps in enumerate(preds):
        for p in ps:
            succ[p].append(i)
    ready = [i for i in range(n) if indeg[i] == 0]
    done = 0
    while ready:
        i = ready.pop(int(rng.integers(len(ready))))
        execute(ops[i], bufs, d)
        done += 1
        for j in succ[i]:
            indeg[j] -= 1
            if indeg[j] == 0:
                ready.append(j)
    assert done == n, "the plan's dependencies have a cycle"


def execute(op, bufs, d):
    k = op["kind"]
    if k == "L":
        flat, idx = _mat(bufs, op["A"], op["ld"], op["nb"], op["nb"])
        X = np.triu(flat[idx])
        X = X + np.triu(X, 1).T
        J = np.arange(op["nb"])[::-1]
        L = np.linalg.cholesky(X[np.ix_(J, J)])
        R = L[np.ix_(J, J)]                      # X = R R^T, R upper
        flat[idx] = np.triu(np.linalg.inv(R))    # U = R^-1, zeros below
    elif k == "C":
        sf, si = _mat(bufs, op["src"], op["lds"], op["rows"], op["cols"])
        df, di = _mat(bufs, op["dst"], op["ldd"], op["rows"], op["cols"])
        df[di] = sf[si]
    elif k == "G":
        M, N, K = op["M"], op["N"], op["K"]
        af, ai = _mat(bufs, op["A"], op["lda"], M, K)
        A = af[ai].copy()
        if op["tb"]:
            bf, bi = _mat(bufs, op["B"], op["ldb"], N, K)
            B = bf[bi].T.copy()
        else:
            bf, bi = _mat(bufs, op["B"], op["ldb"], K, N)
            B = bf[bi].copy()
        cf, ci = _mat(bufs, op["C"], op["ldc"], M, N)
        C = cf[ci].copy()
        out = C.copy()
        for m0, n0 in _tiles(op):
            klo, khi = _k_range(op, m0, n0)
            m1, n1 = min(M, m0 + T), min(N, n0 + T)
            acc = A[m0:m1, klo:khi] @ B[klo:khi, n0:n1] if khi > klo else 0.0
            prev = C[m0:m1, n0:n1] if op["beta"] != 0.0 else 0.0
            out[m0:m1, n0:n1] = op["alpha"] * acc + op["beta"] * prev
        cf[ci] = out


def _check(d, S, side, seeds=(0,), check_races=True):
    head, ops = parse(_plan(d, S, side))
    assert head["d"] == d
    for op in ops:
        if op["kind"] == "G":
            assert op["K"] % 32 == 0 and op["lda"] % 4 == 0 and op["ldb"] % 4 == 0
            assert inplace_ok(op, d), op
    if check_races:
        assert races(ops, d) == []
    X, _ = make_problem(2, d, 3 * d, seed=d)
    Hd, _ = oracle.dampen(oracle.hessian(X), 0.01)
    U_ref = oracle.inverse_upper_cholesky(Hd)
    for seed in seeds:
        bufs = {"A": Hd.astype(np.float64).ravel().copy(),
                "T": np.full(max(head["T"], 1), np.nan)}   # scratch starts as garbage
        run(ops, bufs, d, np.random.default_rng(seed))
        U = np.triu(bufs["A"].reshape(d, d))
        err = np.abs(U - U_ref).max() / np.abs(U_ref).max()
        assert err < 1e-9, (seed, err)
    return head, ops


@pytest.mark.parametrize("d,S", [(512, 0), (608, 0), (1024, 256), (1152, 384), (1184, 512),
                                 (1280, 128)])
def test_plan_with_side_streams_gives_U_in_any_allowed_order(d, S):
    _check(d, S, True, seeds=(0, 1))


@pytest.mark.parametrize("d,S", [(608, 0), (1184, 512)])
def test_plan_on_one_stream_gives_U(d, S):
    head, ops = _check(d, S, False, check_races=False)
    assert {op["s"] for op in ops} == {0}


def test_plan_default_outer_width():
    # wide layers use 1024-column outer blocks; narrower ones one block
    head, _ = parse(_plan(4096, 0, True).split("\n", 1)[0] + "\n")
    assert head["S"] == 4096
    head, _ = parse(_plan(8192, 0, True).split("\n", 1)[0] + "\n")
    assert head["S"] == 1024


def test_plan_trailing_products_have_the_outer_width_as_K():
    # with outer blocks, every update of the matrix above and left of a block
    # (the K = S products) is what carries the flops
    d, S = 1280, 256
    _, ops = parse(_plan(d, S, True))
    big = [op for op in ops if op["kind"] == "G" and op["M"] > S and op["flags"] == 8]
    assert big and all(op["K"] == S for op in big)
