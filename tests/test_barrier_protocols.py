"""Model check of the kernels' mbarrier protocols (host only, no GPU).

Each role of a kernel (the TMA producer thread, the MMA thread, the groups of
worker warps) is written out as the straight-line sequence of barrier
operations its code performs for a given schedule of work, and every
interleaving of the roles and of the asynchronous completions (TMA loads in
any order, tcgen05.commit arrivals in issue order) is explored.  Barriers
follow mbarrier semantics: a phase completes when its arrivals are in (a
group of threads that arrives together counts as one arrival here, as does a
TMA transaction), and a wait on parity P passes while the barrier's current
phase has the other parity.  Two properties are checked in every reachable
state:

* no deadlock: some role or completion can always move until all roles end;
* no phase aliasing: a wait for phase p never meets a barrier that has
  completed p + 2 or more phases (it would wait on a later phase, or pass on
  the wrong one), nor passes before phase p completed.

The abort paths (a wait that runs out) are not modelled.  The planted old
protocol of the TMA-fed readout (one phi-ready barrier for both accumulator
slots) must fail; it is the race that the per-slot barriers fixed.
"""
from collections import namedtuple

import pytest

Op = namedtuple("Op", "kind bar phase")  # kind: wait / arrive / tma / commit


def wait(bar, phase):
    return Op("wait", bar, phase)


def arrive(bar):
    return Op("arrive", bar, None)


def tma(bar):
    return Op("tma", bar, None)


def commit(bar):
    return Op("commit", bar, None)


class ProtocolError(AssertionError):
    pass


def check(roles, max_states=3_000_000):
    """Explore every interleaving of `roles` (name -> list of Op); return the
    number of states visited; raise ProtocolError on a deadlock or a phase
    alias, with the trace that reaches it."""
    names = sorted(roles)
    progs = [roles[n] for n in names]
    bars = sorted({op.bar for p in progs for op in p})
    bid = {b: i for i, b in enumerate(bars)}
    progs = [[(op.kind, bid[op.bar], op.phase) for op in p] for p in progs]

    start = (tuple(0 for _ in progs), tuple(0 for _ in bars), (), ())
    seen = {start}
    stack = [(start, ())]
    while stack:
        (pcs, ph, tmas, commits), trace = stack.pop()
        moves = []
        for r, prog in enumerate(progs):
            if pcs[r] == len(prog):
                continue
            kind, b, p = prog[pcs[r]]
            if kind == "wait":
                k = ph[b]
                if k >= p + 2:
                    raise ProtocolError(f"{names[r]} waits for phase {p} of {bars[b]}, which has completed {k} "
                                        f"phases: {_fmt(trace, names, bars)}")
                if (k & 1) == (p & 1):
                    continue  # blocked
                if k < p + 1:
                    raise ProtocolError(f"{names[r]} passes its wait for phase {p} of {bars[b]} after {k} "
                                        f"phases: {_fmt(trace, names, bars)}")
                moves.append(((r, None), _step(pcs, r), ph, tmas, commits))
            elif kind == "arrive":
                moves.append(((r, None), _step(pcs, r), _bump(ph, b), tmas, commits))
            elif kind == "tma":
                moves.append(((r, None), _step(pcs, r), ph, tuple(sorted(tmas + (b,))), commits))
            else:
                moves.append(((r, None), _step(pcs, r), ph, tmas, commits + (b,)))
        for b in set(tmas):  # a TMA load completes: any of them, in any order
            rest = list(tmas)
            rest.remove(b)
            moves.append(((None, b), pcs, _bump(ph, b), tuple(rest), commits))
        if commits:  # commits complete in issue order
            moves.append(((None, commits[0]), pcs, _bump(ph, commits[0]), tmas, commits[1:]))
        if not moves:
            if any(pcs[r] < len(p) for r, p in enumerate(progs)):
                blocked = [f"{names[r]} at {progs[r][pcs[r]][0]} {bars[progs[r][pcs[r]][1]]} "
                           f"phase {progs[r][pcs[r]][2]}" for r in range(len(progs)) if pcs[r] < len(progs[r])]
                raise ProtocolError(f"deadlock ({'; '.join(blocked)}): {_fmt(trace, names, bars)}")
            continue
        for who, *nxt in moves:
            st = tuple(nxt)
            if st not in seen:
                seen.add(st)
                if len(seen) > max_states:
                    raise RuntimeError("state space too large for this check")
                stack.append((st, trace + (who,)))
    return len(seen)


def _step(pcs, r):
    return pcs[:r] + (pcs[r] + 1,) + pcs[r + 1:]


def _bump(ph, b):
    return ph[:b] + (ph[b] + 1,) + ph[b + 1:]


def _fmt(trace, names, bars):
    out = []
    for r, b in trace[-40:]:
        out.append(names[r] if r is not None else f"done:{bars[b]}")
    return " ".join(out)


# ------------------------------------------------------------------ k4_merge_tma
# Roles as in k4_merge_tma.cu: warp 0 (loads), warp 1 (MMA), the eight worker
# warps (one group).  keys[i] identifies the readout operand (batch, chunk) of
# the CTA's i-th tile.


def k4_tma_roles(keys, per_slot_ready=True):
    n = len(keys)
    ready = (lambda i: f"AReady{i & 1}") if per_slot_ready else (lambda i: "AReady")
    ready_phase = (lambda i: i >> 1) if per_slot_ready else (lambda i: i)

    loads, prev, b_loads = [], None, 0
    for i in range(n + 1):
        if i < n:
            if keys[i] != prev:
                if b_loads > 0:
                    loads.append(wait("BEmpty", b_loads - 1))
                loads.append(tma("BFull"))
                b_loads += 1
                prev = keys[i]
            loads.append(wait("AEmpty", i - 1))  # parity (i & 1) ^ 1
            loads.append(tma("AFull"))
        if i >= 1:
            loads.append(wait("GEmpty", i - 2))  # parity ((i - 1) & 1) ^ 1
            loads.append(tma("GFull"))

    mma, prev, b_loads = [], None, 0
    for i in range(n):
        s = i & 1
        if keys[i] != prev:
            b_loads += 1
            prev = keys[i]
            mma.append(wait("BFull", b_loads - 1))
        mma.append(wait(ready(i), ready_phase(i)))
        mma.append(wait(f"AccEmpty{s}", (i >> 1) - 1))  # parity ((i >> 1) & 1) ^ 1
        mma.append(commit(f"AccFull{s}"))
        if i + 1 >= n or keys[i + 1] != keys[i]:
            mma.append(commit("BEmpty"))
    mma += [commit("Done"), wait("Done", 0)]

    workers = []

    def finish(j):
        workers.extend([wait(f"AccFull{j & 1}", j >> 1), arrive(f"AccEmpty{j & 1}"), wait("GFull", j),
                        arrive("GEmpty")])

    for i in range(n):
        workers += [wait("AFull", i), arrive("AEmpty"), arrive(ready(i))]
        if i > 0:
            finish(i - 1)
    if n > 0:
        finish(n - 1)
    return {"loads": loads, "mma": mma, "workers": workers}


# ------------------------------------------------------------------ k4_readout_merge


def k4_general_roles(keys):
    n = len(keys)
    loads, prev, b_loads = [], None, 0
    for i in range(n):
        s = i & 1
        if keys[i] != prev:
            if b_loads > 0:
                loads.append(wait("BEmpty", b_loads - 1))
            loads.append(tma("BFull"))
            b_loads += 1
            prev = keys[i]
        loads += [wait(f"AEmpty{s}", (i >> 1) - 1), tma(f"AFull{s}")]

    mma, prev, b_loads = [], None, 0
    for i in range(n):
        s = i & 1
        if keys[i] != prev:
            b_loads += 1
            prev = keys[i]
            mma.append(wait("BFull", b_loads - 1))
        mma += [wait(f"AReady{s}", i >> 1), wait(f"AccEmpty{s}", (i >> 1) - 1), commit(f"AccFull{s}"),
                commit(f"AEmpty{s}")]
        if i + 1 >= n or keys[i + 1] != keys[i]:
            mma.append(commit("BEmpty"))
    mma += [commit("Done"), wait("Done", 0)]

    workers = []

    def finish(j):
        workers.extend([wait(f"AccFull{j & 1}", j >> 1), arrive(f"AccEmpty{j & 1}")])

    for i in range(n):
        workers += [wait(f"AFull{i & 1}", i >> 1), arrive(f"AReady{i & 1}")]
        if i > 0:
            finish(i - 1)
    if n > 0:
        finish(n - 1)
    return {"loads": loads, "mma": mma, "workers": workers}


# ------------------------------------------------------------------ k1_state_build


def k1_roles(ntiles, stages=3):
    loads, mma, phi = [], [], []
    for i in range(ntiles):
        st, r = i % stages, i // stages
        loads += [wait(f"Empty{st}", r - 1), tma(f"Full{st}")]
        mma += [wait(f"Phi{st}", r), commit(f"Empty{st}")]
        phi += [wait(f"Full{st}", r), arrive(f"Phi{st}")]
    mma.append(commit("Acc"))
    phi.append(wait("Acc", 0))
    return {"loads": loads, "mma": mma, "phi": phi}


# ------------------------------------------------------------------ k3_sparse_softmax / k3_fp8
# items: (query tiles of the item, KV tiles of its key set) in the CTA's order.
# P is handed to the MMA thread in one part (the kernels' default).  The fp8
# kernel performs the same barrier operations (checked below on the sources).


def k3_roles(items, stages=2):
    loads, kv = [], 0
    for n_item, (_, nkv) in enumerate(items):
        if n_item > 0:
            loads.append(wait("QEmpty", n_item - 1))
        loads.append(tma("QFull"))
        for _ in range(nkv):
            st, r = kv % stages, kv // stages
            loads += [wait(f"KEmpty{st}", r - 1), tma(f"KFull{st}"), wait(f"VEmpty{st}", r - 1),
                      tma(f"VFull{st}")]
            kv += 1

    mma, kv, p_cnt = [], 0, [0, 0]
    for n_item, (nt, nkv) in enumerate(items):
        mma.append(wait("QFull", n_item))
        st = kv % stages
        mma.append(wait(f"KFull{st}", kv // stages))
        mma += [commit(f"SFull{t}") for t in range(nt)]
        mma.append(commit(f"KEmpty{st}"))
        for j in range(nkv):
            st, nst, has_next = kv % stages, (kv + 1) % stages, j + 1 < nkv
            mma.append(wait(f"VFull{st}", kv // stages))
            for t in range(nt):
                mma.append(wait(f"PFull{t}", p_cnt[t]))
                p_cnt[t] += 1
                if not has_next:
                    mma.append(commit(f"OFull{t}"))
                else:
                    if t == 0:
                        mma.append(wait(f"KFull{nst}", (kv + 1) // stages))
                    mma.append(commit(f"SFull{t}"))
            mma.append(commit(f"VEmpty{st}"))
            if has_next:
                mma.append(commit(f"KEmpty{nst}"))
            kv += 1
        mma.append(commit("QEmpty"))
    mma += [commit("Done"), wait("Done", 0)]

    roles = {"loads": loads, "mma": mma}
    for t in range(2):
        sm, s_cnt, o_cnt = [], 0, 0
        for nt, nkv in items:
            if t >= nt:
                continue
            for _ in range(nkv):
                sm += [wait(f"SFull{t}", s_cnt), arrive(f"PFull{t}")]
                s_cnt += 1
            sm.append(wait(f"OFull{t}", o_cnt))
            o_cnt += 1
        roles[f"softmax{t}"] = sm
    return roles


# ------------------------------------------------------------------ tests


def test_checker_finds_a_planted_deadlock_and_alias():
    # a consumer that waits for a phase nobody completes
    with pytest.raises(ProtocolError, match="deadlock"):
        check({"a": [arrive("X")], "b": [wait("X", 0), wait("X", 1)]})
    # a producer that may refill before the consumer waited: the consumer can
    # find two completed phases when it means the first
    with pytest.raises(ProtocolError, match="completed 2 phases"):
        check({"p": [arrive("X"), arrive("X")], "c": [wait("X", 0), wait("X", 1)]})
    # well-formed ping-pong passes
    assert check({"p": [arrive("X"), wait("Y", 0), arrive("X")],
                  "c": [wait("X", 0), arrive("Y"), wait("X", 1)]}) > 0


READOUT_KEYS = [[0, 0, 0, 0], [0, 0, 1, 1], [0, 1, 1, 2], [0, 1, 2, 3], [0, 0, 0, 1, 1]]


@pytest.mark.parametrize("keys", READOUT_KEYS, ids=["".join(map(str, k)) for k in READOUT_KEYS])
def test_tma_readout_protocol(keys):
    assert check(k4_tma_roles(keys)) > 0


def test_tma_readout_single_ready_barrier_fails():
    """The protocol before the fix: the workers can complete two phases of
    the single phi-ready barrier before the MMA thread waits for the first."""
    with pytest.raises(ProtocolError, match="AReady"):
        check(k4_tma_roles([0, 0, 1, 1], per_slot_ready=False))


@pytest.mark.parametrize("keys", READOUT_KEYS, ids=["".join(map(str, k)) for k in READOUT_KEYS])
def test_general_readout_protocol(keys):
    assert check(k4_general_roles(keys)) > 0


@pytest.mark.parametrize("ntiles", [1, 2, 3, 4, 7])
def test_state_build_protocol(ntiles):
    assert check(k1_roles(ntiles)) > 0


K3_SCHEDULES = [[(2, 1)], [(2, 3)], [(1, 2)], [(2, 2), (2, 1)], [(2, 1), (1, 2)], [(1, 1), (2, 2), (1, 1)]]


@pytest.mark.parametrize("items", K3_SCHEDULES, ids=[str(s) for s in K3_SCHEDULES])
def test_sparse_softmax_protocol(items):
    assert check(k3_roles(items)) > 0


def test_fp8_softmax_has_the_bf16_barrier_operations():
    import os
    import re
    csrc = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                        "video_diffusion_hybrid_sparse_b200", "csrc")
    pat = re.compile(r"mbar_wait\(&bars\[[^]]*\][^;]*|mma_commit\(&bars\[[^]]*\]\)|"
                     r"mbar_arrive\(&bars\[[^]]*\]\)|mbar_expect_tx\(&bars\[[^]]*\]")

    def ops(f):
        return pat.findall(open(os.path.join(csrc, f)).read())

    assert ops("k3_sparse_softmax.cu") == ops("k3_fp8.cu") and len(ops("k3_fp8.cu")) > 10
    assert re.search(r"#define VDN_P_PARTS 1\b", open(os.path.join(csrc, "k3_sparse_softmax.cu")).read())
