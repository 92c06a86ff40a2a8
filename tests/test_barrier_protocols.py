"""Model check of the kernels' mbarrier protocols and buffer use (host only).

Each role of a kernel (the TMA producer thread, the MMA thread, the groups of
worker warps) is written out as the straight-line sequence of what its code
does for a given schedule of work: barrier waits and arrivals, TMA loads,
tcgen05.mma issues with the buffers they read and write, tcgen05.commit, and
the intervals in which the warps read or write a shared-memory tile or a
TMEM region.  Every interleaving of the roles and of the asynchronous
completions (TMA loads in any order, commit arrivals in issue order) is
explored.  Barriers follow mbarrier semantics: a phase completes when its
arrivals are in (a group of threads that arrives together counts as one
arrival here, as does a TMA transaction), and a wait on parity P passes
while the barrier's current phase has the other parity.  A TMA load writes
its buffer from issue to completion; an MMA reads and writes its operands
from issue until the first commit issued after it completes (MMAs of one
thread run in issue order, so they never conflict with one another).  In
every reachable state the check asserts:

* no deadlock: some role or completion can always move until all roles end;
* no phase aliasing: a wait for phase p never meets a barrier that has
  completed p + 2 or more phases (it would wait on a later phase, or pass on
  the wrong one), nor passes before phase p completed;
* no buffer hazard: a read finds the version of the data the code means,
  with no write to that buffer in progress, and a write overlaps no other
  role's read or write of it.

The abort paths (a wait that runs out) are not modelled.  The planted old
protocol of the TMA-fed readout (one phi-ready barrier for both accumulator
slots) must fail; it is the race that the per-slot barriers fixed.  Planted
buffer mistakes (a loader that refills before the consumer releases, a
release before the last read) must fail too.
"""
from collections import namedtuple

import pytest

Op = namedtuple("Op", "kind bar phase reads writes")


def wait(bar, phase):
    return Op("wait", bar, phase, (), ())


def arrive(bar):
    return Op("arrive", bar, None, (), ())


def tma(bar, *writes):
    """TMA load(s) completing on `bar`, writing (buffer, version) pairs."""
    return Op("tma", bar, None, (), tuple(writes))


def commit(bar):
    return Op("commit", bar, None, (), ())


def mma(reads=(), writes=()):
    """tcgen05.mma issues reading / writing (buffer, version) pairs (version
    None: not checked)."""
    return Op("mma", None, None, tuple(reads), tuple(writes))


def beg(reads=(), writes=()):
    """This role starts reading / writing the buffers (until `end`)."""
    return Op("beg", None, None, tuple(reads), tuple(writes))


def end(*bufs):
    return Op("end", None, None, tuple(bufs), ())


class ProtocolError(AssertionError):
    pass


def check(roles, max_states=3_000_000):
    """Explore every interleaving of `roles` (name -> list of Op); return the
    number of states visited; raise ProtocolError on a deadlock, a phase
    alias or a buffer hazard, with the trace that reaches it."""
    names = sorted(roles)
    progs = [list(roles[n]) for n in names]
    bars = sorted({op.bar for p in progs for op in p if op.bar is not None})
    bid = {b: i for i, b in enumerate(bars)}
    bufs = sorted({acc[0] for p in progs for op in p for acc in op.reads + op.writes}
                  | {b for p in progs for op in p if op.kind == "end" for b in op.reads})
    uid = {b: i for i, b in enumerate(bufs)}

    def fail(msg, trace):
        raise ProtocolError(f"{msg}: {_fmt(trace, names, bars)}")

    # state: pcs, phases, pending TMAs ((bar, writes), ...), open MMA accesses
    # (since the last commit), commit queue ((bar, accesses), ...), buffer
    # versions, per-role open sync accesses
    start = (tuple(0 for _ in progs), tuple(0 for _ in bars), (), (), (), tuple(None for _ in bufs),
             tuple(() for _ in progs))
    seen = {start}
    stack = [(start, ())]
    while stack:
        state, trace = stack.pop()
        pcs, ph, tmas, mopen, commits, ver, sync = state

        def writers(u, me):
            """Who else is writing buffer u right now (me: role index, 'tma' or 'mma')."""
            out = [w for _, ws in tmas for (w, _) in ws if w == u]
            if me != "mma":
                out += [a for a in mopen if a[0] == "w" and a[1] == u]
                out += [a for _, accs in commits for a in accs if a[0] == "w" and a[1] == u]
            out += [a for r, accs in enumerate(sync) if r != me for a in accs if a[0] == "w" and a[1] == u]
            return out

        def users(u, me):
            out = writers(u, me)
            if me != "mma":
                out += [a for a in mopen if a[1] == u]
                out += [a for _, accs in commits for a in accs if a[1] == u]
            out += [a for r, accs in enumerate(sync) if r != me for a in accs if a[1] == u]
            return out

        def check_access(reads, writes, me, who):
            for b, v in reads:
                u = uid[b]
                if writers(u, me):
                    fail(f"{who} reads {b} while it is being written", trace)
                if v is not None and ver[u] != v:
                    fail(f"{who} reads {b} expecting {v!r}, finds {ver[u]!r}", trace)
            for b, _ in writes:
                if users(uid[b], me):
                    fail(f"{who} writes {b} while another role uses it", trace)

        moves = []
        for r, prog in enumerate(progs):
            if pcs[r] == len(prog):
                continue
            op = prog[pcs[r]]
            npcs = _step(pcs, r)
            if op.kind == "wait":
                b, p = bid[op.bar], op.phase
                k = ph[b]
                if k >= p + 2:
                    fail(f"{names[r]} waits for phase {p} of {op.bar}, which has completed {k} phases", trace)
                if (k & 1) == (p & 1):
                    continue  # blocked
                if k < p + 1:
                    fail(f"{names[r]} passes its wait for phase {p} of {op.bar} after {k} phases", trace)
                moves.append(((r, None), npcs, ph, tmas, mopen, commits, ver, sync))
            elif op.kind == "arrive":
                moves.append(((r, None), npcs, _bump(ph, bid[op.bar]), tmas, mopen, commits, ver, sync))
            elif op.kind == "tma":
                for b, _ in op.writes:
                    if users(uid[b], "tma"):
                        fail(f"{names[r]} starts a TMA load into {b} while it is in use", trace)
                ws = tuple((uid[b], v) for b, v in op.writes)
                moves.append(((r, None), npcs, ph, tuple(sorted(tmas + ((bid[op.bar], ws),))), mopen, commits,
                              ver, sync))
            elif op.kind == "mma":
                check_access(op.reads, op.writes, "mma", names[r])
                accs = tuple(("r", uid[b], v) for b, v in op.reads) + tuple(("w", uid[b], v) for b, v in op.writes)
                moves.append(((r, None), npcs, ph, tmas, mopen + accs, commits, ver, sync))
            elif op.kind == "commit":
                moves.append(((r, None), npcs, ph, tmas, (), commits + ((bid[op.bar], mopen),), ver, sync))
            elif op.kind == "beg":
                check_access(op.reads, op.writes, r, names[r])
                accs = tuple(("r", uid[b], v) for b, v in op.reads) + tuple(("w", uid[b], v) for b, v in op.writes)
                nsync = sync[:r] + (sync[r] + accs,) + sync[r + 1:]
                moves.append(((r, None), npcs, ph, tmas, mopen, commits, ver, nsync))
            else:  # end: close this role's accesses to the buffers; writes take effect
                ended = {uid[b] for b in op.reads}
                nver = list(ver)
                for kind, u, v in sync[r]:
                    if u in ended and kind == "w":
                        nver[u] = v
                keep = tuple(a for a in sync[r] if a[1] not in ended)
                nsync = sync[:r] + (keep,) + sync[r + 1:]
                moves.append(((r, None), npcs, ph, tmas, mopen, commits, tuple(nver), nsync))
        for i, (b, ws) in enumerate(tmas):  # a TMA load completes: any of them, in any order
            if i > 0 and tmas[i - 1] == tmas[i]:
                continue
            nver = list(ver)
            for u, v in ws:
                nver[u] = v
            moves.append(((None, b), pcs, _bump(ph, b), tmas[:i] + tmas[i + 1:], mopen, commits, tuple(nver), sync))
        if commits:  # commits complete in issue order; their MMAs' writes take effect
            b, accs = commits[0]
            nver = list(ver)
            for kind, u, v in accs:
                if kind == "w":
                    nver[u] = v
            moves.append(((None, b), pcs, _bump(ph, b), tmas, mopen, commits[1:], tuple(nver), sync))
        if not moves:
            if any(pcs[r] < len(p) for r, p in enumerate(progs)):
                blocked = [f"{names[r]} at {progs[r][pcs[r]].kind} {progs[r][pcs[r]].bar} "
                           f"phase {progs[r][pcs[r]].phase}" for r in range(len(progs)) if pcs[r] < len(progs[r])]
                fail(f"deadlock ({'; '.join(blocked)})", trace)
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
# the CTA's i-th tile.  Buffers: Q (the q tile), G (o_s, g_s, g_l of a tile),
# B (the operand M_c), Phi0/Phi1 and Acc0/Acc1 (TMEM columns of the two
# accumulator slots).


def k4_tma_roles(keys, per_slot_ready=True, tma_store=True, nq=2):
    """tma_store: the workers merge each tile into the o_s buffer (G) and the
    loader stores it by TMA (reading G until the store's wait_group.read)
    before reloading G.  nq: q tiles in flight (2 when the softmax kernel
    applied the gate and its slot holds a second q tile)."""
    n = len(keys)
    ready = (lambda i: f"AReady{i & 1}") if per_slot_ready else (lambda i: "AReady")
    ready_phase = (lambda i: i >> 1) if per_slot_ready else (lambda i: i)

    loads, prev, b_loads = [], None, 0
    for i in range(n + 1):
        if i < n:
            if keys[i] != prev:
                if b_loads > 0:
                    loads.append(wait("BEmpty", b_loads - 1))
                loads.append(tma("BFull", ("B", keys[i])))
                b_loads += 1
                prev = keys[i]
            loads.append(wait(f"AEmpty{i % nq}", i // nq - 1))  # parity ((i / nq) & 1) ^ 1
            loads.append(tma(f"AFull{i % nq}", (f"Q{i % nq}", i)))
        if i >= 1:
            loads.append(wait("GEmpty", i - 2))  # parity ((i - 1) & 1) ^ 1
            if tma_store and i >= 2:
                loads += [beg(reads=[("G", ("out", i - 2))]), end("G")]
            loads.append(tma("GFull", ("G", i - 1)))
    if tma_store and n > 0:
        loads += [wait("GEmpty", n - 1), beg(reads=[("G", ("out", n - 1))]), end("G")]

    mma_, prev, b_loads = [], None, 0
    for i in range(n):
        s = i & 1
        if keys[i] != prev:
            b_loads += 1
            prev = keys[i]
            mma_.append(wait("BFull", b_loads - 1))
        mma_.append(wait(ready(i), ready_phase(i)))
        mma_.append(wait(f"AccEmpty{s}", (i >> 1) - 1))  # parity ((i >> 1) & 1) ^ 1
        mma_.append(mma(reads=[("B", keys[i]), (f"Phi{s}", i)], writes=[(f"Acc{s}", i)]))
        mma_.append(commit(f"AccFull{s}"))
        if i + 1 >= n or keys[i + 1] != keys[i]:
            mma_.append(commit("BEmpty"))
    mma_ += [commit("Done"), wait("Done", 0)]

    workers = []

    def finish(j):
        s = j & 1
        workers.extend([wait(f"AccFull{s}", j >> 1), beg(reads=[(f"Acc{s}", j)]), end(f"Acc{s}"),
                        arrive(f"AccEmpty{s}"), wait("GFull", j), beg(reads=[("G", j)]), end("G")])
        if tma_store:
            workers.extend([beg(writes=[("G", ("out", j))]), end("G")])
        workers.append(arrive("GEmpty"))

    for i in range(n):
        s = i & 1
        workers += [wait(f"AFull{i % nq}", i // nq), beg(reads=[(f"Q{i % nq}", i)]), end(f"Q{i % nq}"),
                    arrive(f"AEmpty{i % nq}"),
                    beg(writes=[(f"Phi{s}", i)]), end(f"Phi{s}"), arrive(ready(i))]
        if i > 0:
            finish(i - 1)
    if n > 0:
        finish(n - 1)
    return {"loads": loads, "mma": mma_, "workers": workers}


# ------------------------------------------------------------------ k4_readout_merge
# Buffers: A0/A1 (the double-buffered q tile, phi applied in place), B, Acc0/Acc1.


def k4_general_roles(keys):
    n = len(keys)
    loads, prev, b_loads = [], None, 0
    for i in range(n):
        s = i & 1
        if keys[i] != prev:
            if b_loads > 0:
                loads.append(wait("BEmpty", b_loads - 1))
            loads.append(tma("BFull", ("B", keys[i])))
            b_loads += 1
            prev = keys[i]
        loads += [wait(f"AEmpty{s}", (i >> 1) - 1), tma(f"AFull{s}", (f"A{s}", i))]

    mma_, prev, b_loads = [], None, 0
    for i in range(n):
        s = i & 1
        if keys[i] != prev:
            b_loads += 1
            prev = keys[i]
            mma_.append(wait("BFull", b_loads - 1))
        mma_ += [wait(f"AReady{s}", i >> 1), wait(f"AccEmpty{s}", (i >> 1) - 1),
                 mma(reads=[("B", keys[i]), (f"A{s}", ("phi", i))], writes=[(f"Acc{s}", i)]),
                 commit(f"AccFull{s}"), commit(f"AEmpty{s}")]
        if i + 1 >= n or keys[i + 1] != keys[i]:
            mma_.append(commit("BEmpty"))
    mma_ += [commit("Done"), wait("Done", 0)]

    workers = []

    def finish(j):
        s = j & 1
        workers.extend([wait(f"AccFull{s}", j >> 1), beg(reads=[(f"Acc{s}", j)]), end(f"Acc{s}"),
                        arrive(f"AccEmpty{s}")])

    for i in range(n):
        s = i & 1
        workers += [wait(f"AFull{s}", i >> 1), beg(reads=[(f"A{s}", i)], writes=[(f"A{s}", ("phi", i))]),
                    end(f"A{s}"), arrive(f"AReady{s}")]
        if i > 0:
            finish(i - 1)
    if n > 0:
        finish(n - 1)
    return {"loads": loads, "mma": mma_, "workers": workers}


# ------------------------------------------------------------------ k1_state_build
# pieces: tiles of each run of the CTA's range that lies in one state segment.
# Buffers: Stage0..2 (the K and V tiles of a stage; phi is applied to K in
# place), Acc0/Acc1 (the two TMEM accumulators, one per piece in turn).


def k1_roles(pieces, stages=3):
    loads, mma_, phi, epi = [], [], [], []
    i = 0
    for pc, n in enumerate(pieces):
        a = pc & 1
        for k in range(n):
            st, r = i % stages, i // stages
            loads += [wait(f"Empty{st}", r - 1), tma(f"Full{st}", (f"Stage{st}", i))]
            phi += [wait(f"Full{st}", r), beg(reads=[(f"Stage{st}", i)], writes=[(f"Stage{st}", ("phi", i))]),
                    end(f"Stage{st}"), arrive(f"Phi{st}")]
            if k == 0:
                mma_.append(wait(f"AccEmpty{a}", (pc >> 1) - 1))
            mma_ += [wait(f"Phi{st}", r), mma(reads=[(f"Stage{st}", ("phi", i))], writes=[(f"Acc{a}", (pc, k))]),
                     commit(f"Empty{st}")]
            if k == n - 1:
                mma_.append(commit(f"AccFull{a}"))
            i += 1
        epi += [wait(f"AccFull{a}", pc >> 1), beg(reads=[(f"Acc{a}", (pc, n - 1))]), end(f"Acc{a}"),
                arrive(f"AccEmpty{a}")]
    mma_ += [commit("Done"), wait("Done", 0)]
    return {"loads": loads, "mma": mma_, "phi": phi, "epilogue": epi}


# ------------------------------------------------------------------ k3_sparse_softmax / k3_fp8
# items: (query tiles of the item, KV tiles of its key set) in the CTA's order.
# Both softmax kernels (bf16 and fp8, checked below on the sources) hand P
# to the MMA thread in two halves per tile (keys 0-63 on PFull, keys 64-127
# on PFull2).  Buffers: Q (the item's query tiles), K0/K1 and V0/V1 (the
# stages), SPa/SPb per query tile (the two halves of the TMEM columns of S,
# with P written over them), O0/O1 (TMEM output accumulators; the softmax
# warps may rescale them in place before handing over the first half of P,
# modelled at every step).


def k3_roles(items, stages=2, halves=2, fused=False):
    """Roles of k3_sparse_softmax.cu for items [(query tiles, KV tiles), ...].
    Buffers: Q0/Q1 (the two query tiles of the Q slot), K/V stages, SPa/SPb
    (the two halves of a tile's S columns: S, then P over them; under the
    fused readout also num), O0/O1.  fused: the readout operand M_c travels
    as one more K/V stage, the softmax warps write phi(Q_t) over Q_t, the MMA
    thread writes num_t over S_t's columns, the epilogue reads it and
    releases the columns (RDone); the scan (warps 2-3) writes M_c in global
    memory (Mg) and completes its count (ScanDone, a counter in the kernel,
    a barrier of one arrival here), which the producer waits for before it
    copies M_c and the softmax warps before they read z."""
    loads, kv = [], 0
    for n_item, (nt, nkv) in enumerate(items):
        if n_item > 0:
            loads.append(wait("QEmpty", n_item - 1))
        loads.append(tma("QFull", *[(f"Q{t}", ("Q", n_item)) for t in range(nt)]))
        for i in range(nkv + (1 if fused else 0)):
            st, r = kv % stages, kv // stages
            if i == nkv:  # the readout stage: M_c copied from global memory
                loads += [wait("ScanDone", 0), beg(reads=[("Mg", "scanned")]), end("Mg")]
            loads += [wait(f"KEmpty{st}", r - 1), tma(f"KFull{st}", (f"K{st}", kv)), wait(f"VEmpty{st}", r - 1),
                      tma(f"VFull{st}", (f"V{st}", kv))]
            kv += 1

    mma_, kv, p_cnt, s_idx = [], 0, [0, 0], [0, 0]
    phi_cnt, rd_cnt, rd_pend = [0, 0], [0, 0], [False, False]

    parts = ["a", "b"][:halves]
    regions = ["a", "b"]  # the S columns of a tile, whatever the P handoff

    def issue_s(t, n_item, st, kv_):
        mma_.append(mma(reads=[(f"Q{t}", ("Q", n_item)), (f"K{st}", kv_)],
                        writes=[(f"SP{h}{t}", ("S", s_idx[t])) for h in regions]))
        s_idx[t] += 1

    for n_item, (nt, nkv) in enumerate(items):
        mma_.append(wait("QFull", n_item))
        st = kv % stages
        mma_.append(wait(f"KFull{st}", kv // stages))
        for t in range(nt):
            if fused and rd_pend[t]:
                mma_.append(wait(f"RDone{t}", rd_cnt[t]))
                rd_cnt[t] += 1
                rd_pend[t] = False
            issue_s(t, n_item, st, kv)
            mma_.append(commit(f"SFull{t}"))
        mma_.append(commit(f"KEmpty{st}"))
        for j in range(nkv):
            st, nst, has_next = kv % stages, (kv + 1) % stages, j + 1 < nkv
            mma_.append(wait(f"VFull{st}", kv // stages))
            for t in range(nt):
                for h in parts:
                    # one handoff: P.V reads P over both halves of the columns
                    held = [h] if halves == 2 else regions
                    mma_.append(wait(f"PFull{'2' if h == 'b' else ''}{t}", p_cnt[t]))
                    mma_.append(mma(reads=[(f"SP{x}{t}", ("P", p_cnt[t])) for x in held] + [(f"V{st}", kv)],
                                    writes=[(f"O{t}", ("O", n_item, j))]))
                p_cnt[t] += 1
                if not has_next:
                    mma_.append(commit(f"OFull{t}"))
                else:
                    if t == 0:
                        mma_.append(wait(f"KFull{nst}", (kv + 1) // stages))
                    issue_s(t, n_item, nst, kv + 1)
                    mma_.append(commit(f"SFull{t}"))
            mma_.append(commit(f"VEmpty{st}"))
            if has_next:
                mma_.append(commit(f"KEmpty{nst}"))
            kv += 1
        if fused:
            st = kv % stages
            mma_ += [wait(f"KFull{st}", kv // stages), wait(f"VFull{st}", kv // stages)]
            for t in range(nt):
                mma_.append(wait(f"PhiFull{t}", phi_cnt[t]))
                phi_cnt[t] += 1
                mma_.append(mma(reads=[(f"Q{t}", ("phi", n_item)), (f"K{st}", kv), (f"V{st}", kv)],
                                writes=[(f"SP{h}{t}", ("num", n_item)) for h in regions]))
                mma_.append(commit(f"RFull{t}"))
                rd_pend[t] = True
            mma_ += [commit(f"KEmpty{st}"), commit(f"VEmpty{st}")]
            kv += 1
        mma_.append(commit("QEmpty"))
    mma_ += [commit("Done"), wait("Done", 0)]

    roles = {"loads": loads, "mma": mma_}
    if fused:
        roles["scan"] = [beg(writes=[("Mg", "scanned")]), end("Mg"), arrive("ScanDone")]
    for t in range(2):
        sm, s_cnt, o_cnt = [], 0, 0
        for n_item, (nt, nkv) in enumerate(items):
            if t >= nt:
                continue
            for j in range(nkv):
                sm += [wait(f"SFull{t}", s_cnt)]
                sm += [x for h in regions for x in (beg(reads=[(f"SP{h}{t}", ("S", s_cnt))]), end(f"SP{h}{t}"))]
                sm += [beg(writes=[("SPa" + str(t), ("P", s_cnt))]), end(f"SPa{t}")]
                if halves == 1:
                    sm += [beg(writes=[("SPb" + str(t), ("P", s_cnt))]), end(f"SPb{t}")]
                sm += [beg(writes=[(f"O{t}", ("scaled", n_item, j))]), end(f"O{t}"), arrive(f"PFull{t}")]
                if halves == 2:
                    sm += [beg(writes=[(f"SPb{t}", ("P", s_cnt))]), end(f"SPb{t}"), arrive(f"PFull2{t}")]
                s_cnt += 1
            if fused:
                sm += [wait("ScanDone", 0), beg(reads=[("Mg", "scanned")]), end("Mg"),  # z
                       beg(writes=[(f"Q{t}", ("phi", n_item))]), end(f"Q{t}"), arrive(f"PhiFull{t}"),
                       wait(f"OFull{t}", o_cnt), wait(f"RFull{t}", o_cnt),
                       beg(reads=[(f"O{t}", ("O", n_item, nkv - 1))] + [(f"SP{h}{t}", ("num", n_item))
                                                                        for h in regions]),
                       end(f"O{t}", f"SPa{t}", f"SPb{t}"), arrive(f"RDone{t}")]
            else:
                sm += [wait(f"OFull{t}", o_cnt), beg(reads=[(f"O{t}", ("O", n_item, nkv - 1))]), end(f"O{t}")]
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


READOUT_KEYS = [[0, 0, 0, 0], [0, 0, 1, 1], [0, 1, 1, 2], [0, 1, 2, 3], [0, 0, 0, 1, 1], [0, 0, 1, 1, 2, 2]]


@pytest.mark.parametrize("keys", READOUT_KEYS, ids=["".join(map(str, k)) for k in READOUT_KEYS])
@pytest.mark.parametrize("nq", [2, 1], ids=["two_q", "one_q"])
def test_tma_readout_protocol(keys, nq):
    assert check(k4_tma_roles(keys, nq=nq)) > 0


def test_tma_readout_single_ready_barrier_fails():
    """The protocol before the fix: the workers can complete two phases of
    the single phi-ready barrier before the MMA thread waits for the first."""
    with pytest.raises(ProtocolError, match="AReady"):
        check(k4_tma_roles([0, 0, 1, 1], per_slot_ready=False))


@pytest.mark.parametrize("keys", READOUT_KEYS, ids=["".join(map(str, k)) for k in READOUT_KEYS])
def test_general_readout_protocol(keys):
    assert check(k4_general_roles(keys)) > 0


K1_PIECES = [[1], [4], [7], [1, 1], [2, 3], [3, 1, 2], [1, 1, 1, 1], [2, 1, 1, 2]]


@pytest.mark.parametrize("pieces", K1_PIECES, ids=[str(p) for p in K1_PIECES])
def test_state_build_protocol(pieces):
    assert check(k1_roles(pieces)) > 0


@pytest.mark.parametrize("pieces,stages", [([7], 6), ([2, 3, 2], 6), ([4, 5], 8)])
def test_state_build_protocol_deep_pipeline(pieces, stages):
    # the protocol does not depend on the number of stages
    assert check(k1_roles(pieces, stages=stages)) > 0


K3_SCHEDULES = [[(2, 1)], [(2, 3)], [(2, 4)], [(1, 2)], [(2, 2), (2, 1)], [(2, 1), (1, 2)], [(1, 1), (2, 2), (1, 1)],
                [(2, 3), (1, 2), (2, 1)], [(2, 2), (2, 2), (2, 2)]]


@pytest.mark.parametrize("items", K3_SCHEDULES, ids=[str(s) for s in K3_SCHEDULES])
def test_sparse_softmax_protocol(items):
    assert check(k3_roles(items)) > 0


K3_FUSED_SCHEDULES = [[(2, 1)], [(2, 2)], [(1, 2)], [(2, 1), (2, 1)], [(2, 2), (1, 1)], [(1, 1), (2, 2)],
                      [(2, 1), (1, 1), (2, 1)]]


@pytest.mark.parametrize("items", K3_FUSED_SCHEDULES, ids=[str(s) for s in K3_FUSED_SCHEDULES])
def test_fused_readout_protocol(items):
    assert check(k3_roles(items, fused=True)) > 0


def test_fp8_softmax_has_the_bf16_barrier_operations():
    """The e4m3 kernel's barrier operations are the bf16 kernel's without
    the fused readout."""
    assert SOURCE_BARRIER_OPS["k3_fp8.cu"] == K3_OPS


@pytest.mark.parametrize("items", K3_SCHEDULES[:3], ids=[str(s) for s in K3_SCHEDULES[:3]])
def test_single_p_handoff_protocol(items):
    # the one-piece handoff (P for all 128 keys on one barrier) is also sound
    assert check(k3_roles(items, halves=1)) > 0


def _drop(roles, role, pred):
    out = dict(roles)
    out[role] = [op for op in roles[role] if not pred(op)]
    return out


def _drop_last(roles, role, pred):
    ops = list(roles[role])
    i = max(k for k, op in enumerate(ops) if pred(op))
    out = dict(roles)
    out[role] = ops[:i] + ops[i + 1:]
    return out


def _move_before(roles, role, pred_move, pred_anchor):
    """Move every op matching pred_move to just before the preceding op that
    matches pred_anchor."""
    ops = list(roles[role])
    i = 0
    while i < len(ops):
        if pred_move(ops[i]):
            j = i - 1
            while j >= 0 and not pred_anchor(ops[j]):
                j -= 1
            if j >= 0:
                op = ops.pop(i)
                ops.insert(j, op)
        i += 1
    out = dict(roles)
    out[role] = ops
    return out


def _move_o_rescale_before_s_wait(roles):
    ops = list(roles["softmax0"])
    out, pending = [], None
    for i, op in enumerate(ops):
        if op is None:
            continue
        if op.kind == "beg" and op.writes and op.writes[0][1][0] == "scaled":
            # the rescale (this op and its end) goes before the preceding S wait
            ops[i + 1] = None
            out.insert(pending, op)
            out.insert(pending + 1, end(op.writes[0][0]))
            continue
        if op.kind == "wait" and op.bar == "SFull0":
            pending = len(out)
        out.append(op)
    roles = dict(roles)
    roles["softmax0"] = out
    return roles


PLANTED = {
    # the loader refills the q tile without waiting for the workers to release it
    # (with one q slot; with two, the wait for the o_s / gate release orders
    # the refill after the read anyway)
    "readout_loader_skips_q_release": lambda: _drop(k4_tma_roles([0, 0, 1, 1, 1], nq=1), "loads",
                                                    lambda op: op.kind == "wait" and op.bar.startswith("AEmpty")),
    # the workers release the q tile before reading it (one q slot)
    "readout_release_before_read": lambda: _move_before(
        k4_tma_roles([0, 0, 1, 1, 1], nq=1), "workers", lambda op: op.kind == "arrive" and op.bar.startswith("AEmpty"),
        lambda op: op.kind == "beg" and op.reads and op.reads[0][0].startswith("Q")),
    # the loader stores the last output tile without waiting for the merge to finish
    "readout_store_before_merge": lambda: _drop_last(k4_tma_roles([0, 0, 1]), "loads",
                                                     lambda op: op.kind == "wait" and op.bar == "GEmpty"),
    # the loader reloads o_s and the gates without waiting for the merge to finish
    "readout_loader_skips_g_release": lambda: _drop(k4_tma_roles([0, 0, 1, 1]), "loads",
                                                    lambda op: op.kind == "wait" and op.bar == "GEmpty"),
    # the MMA thread reads the readout operand before its load landed
    "readout_mma_skips_operand_load": lambda: _drop(k4_tma_roles([0, 0, 1, 1]), "mma",
                                                    lambda op: op.kind == "wait" and op.bar == "BFull"),
    # the general readout's MMA thread does not wait for phi
    "general_readout_mma_skips_ready": lambda: _drop(k4_general_roles([0, 1, 1]), "mma",
                                                     lambda op: op.kind == "wait" and op.bar.startswith("AReady")),
    # the state build's MMA thread does not wait for phi(K)
    "state_build_mma_skips_phi": lambda: _drop(k1_roles([4]), "mma",
                                               lambda op: op.kind == "wait" and op.bar.startswith("Phi")),
    # the state build's MMA thread starts a piece in an accumulator still being read out
    "state_build_mma_skips_acc_release": lambda: _drop(k1_roles([1, 1, 1]), "mma",
                                                       lambda op: op.kind == "wait" and op.bar.startswith("AccEmpty")),
    # the read-out releases an accumulator before reading it
    "state_build_release_before_read": lambda: _move_before(
        k1_roles([1, 1, 1]), "epilogue", lambda op: op.kind == "arrive" and op.bar.startswith("AccEmpty"),
        lambda op: op.kind == "beg"),
    # the softmax MMA thread does not wait for P
    "softmax_mma_skips_p": lambda: _drop(k3_roles([(2, 2)]), "mma",
                                         lambda op: op.kind == "wait" and op.bar.startswith("PFull")),
    # the MMA thread starts the P.V of the second half of the keys when only
    # the first half of P is stored
    "softmax_mma_skips_second_half": lambda: _drop(k3_roles([(2, 2)]), "mma",
                                                   lambda op: op.kind == "wait" and op.bar.startswith("PFull2")),
    # the softmax warps hand over the first half of P before rescaling O
    "softmax_first_half_before_rescale": lambda: _move_before(
        k3_roles([(1, 3)]), "softmax0", lambda op: op.kind == "arrive" and op.bar == "PFull0",
        lambda op: op.kind == "beg" and op.writes and op.writes[0][0] == "O0"),
    # the loader refills a K stage before the S MMAs that read it completed
    "softmax_loader_skips_k_release": lambda: _drop(k3_roles([(1, 3)]), "loads",
                                                    lambda op: op.kind == "wait" and op.bar.startswith("KEmpty")),
    # the softmax warps rescale O before the commit after S (which also
    # covers the previous P.V into O) landed
    "softmax_rescale_before_s": lambda: _move_o_rescale_before_s_wait(k3_roles([(1, 3)])),
    # fused readout: the next item's first S overwrites num while the epilogue reads it
    "fused_mma_skips_readout_release": lambda: _drop(k3_roles([(2, 1), (2, 1)], fused=True), "mma",
                                                     lambda op: op.kind == "wait" and op.bar.startswith("RDone")),
    # fused readout: the MMA thread reads Q before phi(Q) is written over it
    "fused_mma_skips_phi": lambda: _drop(k3_roles([(2, 1)], fused=True), "mma",
                                         lambda op: op.kind == "wait" and op.bar.startswith("PhiFull")),
    # fused readout: Q released for the next item before the readout MMAs read phi(Q)
    "fused_q_release_before_readout": lambda: _move_before(
        k3_roles([(1, 1), (1, 1)], fused=True), "mma", lambda op: op.kind == "commit" and op.bar == "QEmpty",
        lambda op: op.kind == "wait" and op.bar.startswith("PhiFull")),
    # fused readout: the epilogue reads num before the readout MMAs completed
    "fused_epilogue_skips_num": lambda: _drop(k3_roles([(1, 2)], fused=True), "softmax0",
                                              lambda op: op.kind == "wait" and op.bar == "RFull0"),
    # fused readout: the producer copies M_c before the scan has completed it
    "fused_loader_skips_scan_count": lambda: _drop(k3_roles([(1, 1), (1, 1)], fused=True), "loads",
                                                   lambda op: op.kind == "wait" and op.bar == "ScanDone"),
    # fused readout: the softmax warps read z before the scan has completed it
    "fused_epilogue_skips_scan_count": lambda: _drop(k3_roles([(1, 1)], fused=True), "softmax0",
                                                     lambda op: op.kind == "wait" and op.bar == "ScanDone"),
    # fused readout: the softmax warps write phi over Q before the item's last S landed
    "fused_phi_before_last_s": lambda: _move_before(
        k3_roles([(1, 2)], fused=True), "softmax0", lambda op: op.kind == "beg" and op.writes
        and op.writes[0][0] == "Q0", lambda op: op.kind == "wait" and op.bar == "SFull0"),
}


@pytest.mark.parametrize("name", sorted(PLANTED))
def test_planted_protocol_mistake_is_caught(name):
    with pytest.raises(ProtocolError):
        check(PLANTED[name]())


def test_readout_acc_release_wait_is_implied():
    """In both readouts the MMA thread's wait for a drained accumulator slot
    is implied by the phi-ready wait: the workers arrive on a slot's
    phi-ready barrier for tile i + 2 only after draining tile i.  The model
    finds no hazard without it (the kernels keep it as a safeguard)."""
    for roles in (k4_tma_roles([0, 0, 1, 1, 1]), k4_general_roles([0, 0, 1, 1, 1])):
        assert check(_drop(roles, "mma", lambda op: op.kind == "wait" and op.bar.startswith("AccEmpty"))) > 0


# The barrier operations of each kernel source, in source order, as the role
# programs above model them.  A change to a kernel's barrier use fails here
# until the model (and this list) is brought up to date.
K3_OPS = ("wait:kQEmpty expect_tx:kQFull wait:kKEmpty+st expect_tx:kKFull+st wait:kVEmpty+st "
          "expect_tx:kVFull+st wait:kQFull wait:kKFull+st mma_commit:kSFull+t "
          "mma_commit:kKEmpty+st wait:kVFull+st wait:kPFull+t wait:kPFull2+t "
          "mma_commit:kOFull+t wait:kKFull+nst mma_commit:kSFull+t mma_commit:kVEmpty+st "
          "mma_commit:kKEmpty+nst mma_commit:kQEmpty mma_commit:kDone wait:kSFull+t "
          "arrive:kPFull+t arrive:kPFull2+t wait:kOFull+t")
# the bf16 kernel: the same, with the fused readout's operations in their
# places (the epilogue of a fused tile is a function ahead of the kernel)
K3_FUSED_OPS = ("arrive:kPhiFull+t wait:kOFull+t wait:kRFull+t arrive:kRDone+t " + K3_OPS
                .replace("expect_tx:kVFull+st wait:kQFull",
                         "expect_tx:kVFull+st wait:kKEmpty+st expect_tx:kKFull+st wait:kVEmpty+st "
                         "expect_tx:kVFull+st wait:kQFull")
                .replace("wait:kKFull+st mma_commit:kSFull+t", "wait:kKFull+st wait:kRDone+t mma_commit:kSFull+t")
                .replace("mma_commit:kKEmpty+nst mma_commit:kQEmpty",
                         "mma_commit:kKEmpty+nst wait:kKFull+st wait:kVFull+st wait:kPhiFull+t mma_commit:kRFull+t "
                         "mma_commit:kKEmpty+st mma_commit:kVEmpty+st mma_commit:kQEmpty")
)

SOURCE_BARRIER_OPS = {
    "k1_state_build.cu": "wait:kEmpty+st expect_tx:kFull+st wait:kAccFull wait:kAccEmpty+a wait:kPhi+st "
                         "mma_commit:kEmpty+st mma_commit:kAccFull+a mma_commit:kDone wait:kFull+st arrive:kPhi+st "
                         "wait:kAccFull+buf arrive:kAccEmpty+buf",
    "k3_sparse_softmax.cu": K3_FUSED_OPS,
    "k3_fp8.cu": K3_OPS,
    "k4_merge_tma.cu": "wait:kTBEmpty expect_tx:kTBFull wait:kTAEmpty+qs expect_tx:kTAFull+qs wait:kTGEmpty "
                       "expect_tx:kTGFull wait:kTGEmpty wait:kTBFull wait:kTAReady+s wait:kTAccEmpty+s mma_commit:kTAccFull+s "
                       "mma_commit:kTBEmpty mma_commit:kTDone wait:kTAccFull+s arrive:kTAccEmpty+s wait:kTGFull "
                       "arrive:kTGEmpty wait:kTAFull+i%nq arrive:kTAEmpty+i%nq arrive:kTAReady+(i&1)",
    "k4_readout_merge.cu": "wait:kBEmpty expect_tx:kBFull wait:kAEmpty+s expect_tx:kAFull+s wait:kBFull "
                           "wait:kAReady+s wait:kAccEmpty+s mma_commit:kAccFull+s mma_commit:kAEmpty+s "
                           "mma_commit:kBEmpty mma_commit:kDone4 wait:kAccFull+s arrive:kAccEmpty+s wait:kAFull+s "
                           "arrive:kAReady+s",
}


@pytest.mark.parametrize("src", sorted(SOURCE_BARRIER_OPS))
def test_model_matches_the_kernel_sources(src):
    import os
    import re
    path = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                        "video_diffusion_hybrid_sparse_b200", "csrc", src)
    pat = re.compile(r"(mbar_wait|mma_commit|mbar_arrive|mbar_expect_tx)\(&bars\[([^\]]*)\]")
    ops = " ".join(f"{m.group(1).replace('mbar_', '')}:{m.group(2).replace(' ', '')}"
                   for m in pat.finditer(open(path).read()))
    assert ops == SOURCE_BARRIER_OPS[src]
