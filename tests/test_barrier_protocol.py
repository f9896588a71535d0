"""A discrete model of the mbarrier protocol of the fused per-token kernel
(sparse_lightning_indexer_b200/csrc/slikl_fused_sm100.cu), checked on the CPU.

Every warp role is a generator over the barriers it waits on and arrives at, walking the same
item schedule as the kernel (pass A of the next token alternating with pass B of the current
one). An mbarrier is modelled by its count of completed phases: a wait on parity P passes once
the phase of parity P has completed, i.e. while the completed-phase count has the other parity
(so a fresh barrier passes a wait on parity 1 at once, as in hardware). Asynchronous
completions (cp.async and TMA arrivals, tcgen05.commit) are taken as immediate: they depend on
nothing else, so delaying them cannot create a dependency cycle.

The roles run in random interleavings over random token tile masks. Each run must finish (no
deadlock), and explicit safety checks fail a run in which a buffer is overwritten before its
previous contents were consumed: K stages, S buffers in TMEM and dS tiles. The checks are what
catches parity aliasing, where a waiter that skips phases passes a barrier two phases early.
A negative test keeps the model honest: the producer variant in which each warp waits on a
stage only at the items it owns is caught.

The key-major dK kernel (sparse_lightning_indexer_b200/csrc/slikl_dk_keymajor.cu) is modelled
the same way: its two producers (w-scaled q; records), 16 dS-builder warps, MMA issuer and 4
flush warps over runs of work units, with checks on the reuse of each ring's slots (q, records,
dS tiles) and on the two TMEM dK buffers (a run accumulates only into its own buffer, which
is not reused before its flush).
"""

import itertools
import random

import pytest

N_TILE_BITS = 16


class Bar:
    def __init__(self, count):
        self.count = count
        self.arrivals = 0
        self.phases = 0                      # completed phases

    def ready(self, parity):
        return (self.phases & 1) != parity

    def arrive(self):
        self.arrivals += 1
        assert self.arrivals <= self.count
        if self.arrivals == self.count:
            self.phases += 1
            self.arrivals = 0


class Violation(AssertionError):
    pass


def schedule(masks):
    """The kernel's item order: phase 0 = A(t0); phase k = B(t_{k-1}) and A(t_k) alternated,
    B first, then whichever remains; tiles of a token in index order. Tokens without an
    active tile are skipped."""
    toks = [t for t, m in enumerate(masks) if m]
    items = []
    nxt = 0

    def take_token():
        nonlocal nxt
        if nxt == len(toks):
            return None
        t = toks[nxt]
        tiles = [i for i in range(N_TILE_BITS) if masks[t] >> i & 1]
        tok = dict(t=t, ord=nxt, tiles=tiles)
        nxt += 1
        return tok

    a = take_token()
    b = None
    while a is not None or b is not None:
        ra = list(a["tiles"]) if a else []
        rb = list(b["tiles"]) if b else []
        fa, fb, turn_b = True, True, True
        while ra or rb:
            if rb and (not ra or turn_b):
                tile = rb.pop(0)
                items.append(dict(kind=1, t=b["t"], ord=b["ord"], tile=tile, first=fb, last=not rb))
                fb = False
            else:
                tile = ra.pop(0)
                items.append(dict(kind=0, t=a["t"], ord=a["ord"], tile=tile, first=fa, last=not ra))
                fa = False
            turn_b = not turn_b
        b = a
        a = take_token()
    return items


def build(items, rec, stages=4, owner_producers=False, ns=2, nd=2):
    """Roles of one CTA. rec: record mode (key-major dK; no scatter group, the MMA releases the
    dS tile after the dq product). owner_producers: the known-bad variant. ns / nd: S^T
    buffers in TMEM and dS tiles (with their dK^T buffers); the 128-head instances use one S
    buffer (scatter mode) or two (record mode) and one dS tile, with three K stages."""
    nprod = 7 if rec else 3
    bars = {}

    def bar(name, count):
        bars[name] = Bar(count)

    for s in range(stages):
        bar(f"kv_full{s}", nprod)
        bar(f"kv_empty{s}", 1)
    for b in range(2):
        bar(f"q_full{b}", 1)
        bar(f"q_empty{b}", 1)
        bar(f"s_full{b}", 1)
        bar(f"s_empty{b}", 4)
        bar(f"ds_full{b}", 4)
        bar(f"rows_full{b}", 4)
        bar(f"dk_full{b}", 1)
        bar(f"dk_empty{b}", 1 if rec else 4)
    bar("dq_full", 1)
    bar("dq_empty", 4)
    bar("sm_sync", 4)

    # safety bookkeeping: how many times each buffer was filled, and released by each of the
    # warps that read it (a buffer is free again only when every reader is done with it)
    st = dict(stage_free=[0] * stages, s_fill=[0] * ns, s_free=[[0] * ns for _ in range(4)],
              ds_fill=[[0] * nd for _ in range(4)], ds_free=[[0] * nd for _ in range(4)])

    def freed(key, b):
        return min(w[b] for w in st[key])

    serial = itertools.count()

    def wait(name, parity):
        # each wait carries its own serial number, so a role blocked again on the same
        # barrier (e.g. back-to-back group syncs) does not read as one that never moved
        token = next(serial)
        while not bars[name].ready(parity):
            yield ("wait", name, token)

    def producer(w):
        for g, it in enumerate(items):
            if owner_producers and g % nprod != w:
                continue
            if w == 0 and it["kind"] == 0 and it["first"]:
                qb = it["ord"] & 1
                yield from wait(f"q_empty{qb}", ((it["ord"] >> 1) & 1) ^ 1)
                bars[f"q_full{qb}"].arrive()
            s = g % stages
            yield from wait(f"kv_empty{s}", ((g // stages) & 1) ^ 1)
            # this warp writes its rows of item g into stage s: every earlier item of the stage
            # must have been released by the MMA
            if st["stage_free"][s] < g // stages:
                raise Violation(f"producer {w} overwrote stage {s} (item {g}) still in use")
            if owner_producers:
                for _ in range(nprod):
                    bars[f"kv_full{s}"].arrive()
            else:
                bars[f"kv_full{s}"].arrive()
            yield ("step",)

    def mma():
        gk = gd = nb = 0

        def issue_s(it):
            nonlocal gk
            s, b = gk % stages, gk % ns
            if it["kind"] == 0 and it["first"]:
                yield from wait(f"q_full{it['ord'] & 1}", (it["ord"] >> 1) & 1)
            yield from wait(f"kv_full{s}", (gk // stages) & 1)
            yield from wait(f"s_empty{b}", ((gk // ns) & 1) ^ 1)
            if freed("s_free", b) < gk // ns:
                raise Violation(f"S buffer {b} overwritten (item {gk}) before it was read")
            st["s_fill"][b] += 1
            bars[f"s_full{b}"].arrive()
            if it["kind"] == 0:
                st["stage_free"][s] += 1
                bars[f"kv_empty{s}"].arrive()
            gk += 1
            return s

        if not items:
            return
        i = 0
        stage_cur = yield from issue_s(items[0])
        while i < len(items):
            cur = items[i]
            stage_nxt = None
            if i + 1 < len(items):
                stage_nxt = yield from issue_s(items[i + 1])
            if cur["kind"] == 1:
                b = gd % nd
                if cur["first"]:
                    yield from wait("dq_empty", (nb & 1) ^ 1)
                yield from wait(f"ds_full{b}", (gd // nd) & 1)
                if not rec:
                    yield from wait(f"dk_empty{b}", ((gd // nd) & 1) ^ 1)
                if min(w[b] for w in st["ds_fill"]) != gd // nd + 1:
                    raise Violation(f"dq product read dS buffer {b} not holding item {gd}")
                st["stage_free"][stage_cur] += 1
                bars[f"kv_empty{stage_cur}"].arrive()
                if rec:
                    for w in st["ds_free"]:
                        w[b] += 1
                    bars[f"dk_empty{b}"].arrive()
                else:
                    bars[f"dk_full{b}"].arrive()
                if cur["last"]:
                    bars["dq_full"].arrive()
                    bars[f"q_empty{cur['ord'] & 1}"].arrive()
                    nb += 1
                gd += 1
            stage_cur = stage_nxt
            i += 1
            yield ("step",)

    def scatter(wq):
        gd = 0
        for it in items:
            if it["kind"] != 1:
                continue
            b = gd % nd
            yield from wait(f"rows_full{b}", (gd // nd) & 1)
            yield from wait(f"dk_full{b}", (gd // nd) & 1)
            st["ds_free"][wq][b] += 1
            bars[f"dk_empty{b}"].arrive()
            gd += 1
            yield ("step",)

    phase = [0] * 4

    def group_sync(wq):
        bars["sm_sync"].arrive()
        yield from wait("sm_sync", phase[wq] & 1)
        phase[wq] += 1

    def softmax(wq):
        gk = gd = nb = 0
        for it in items:
            sb = gk % ns
            if it["kind"] == 0:
                if it["first"]:
                    yield from group_sync(wq)
                yield from wait(f"s_full{sb}", (gk // ns) & 1)
                if st["s_fill"][sb] != gk // ns + 1:
                    raise Violation(f"pass A read S buffer {sb} not holding item {gk}")
                st["s_free"][wq][sb] += 1
                bars[f"s_empty{sb}"].arrive()
                if it["last"]:
                    yield from group_sync(wq)
                    yield from group_sync(wq)
            else:
                b = gd % nd
                yield from wait(f"dk_empty{b}", ((gd // nd) & 1) ^ 1)
                if freed("ds_free", b) < gd // nd:
                    raise Violation(f"dS buffer {b} overwritten (item {gd}) before it was read")
                yield from wait(f"s_full{sb}", (gk // ns) & 1)
                if st["s_fill"][sb] != gk // ns + 1:
                    raise Violation(f"pass B read S buffer {sb} not holding item {gk}")
                st["s_free"][wq][sb] += 1
                st["ds_fill"][wq][b] += 1
                bars[f"s_empty{sb}"].arrive()
                bars[f"ds_full{b}"].arrive()
                if not rec:
                    bars[f"rows_full{b}"].arrive()
                gd += 1
                if it["last"]:
                    yield from group_sync(wq)
                    yield from wait("dq_full", nb & 1)
                    bars["dq_empty"].arrive()
                    nb += 1
            gk += 1
            yield ("step",)

    roles = {f"producer{w}": producer(w) for w in range(nprod)}
    roles["mma"] = mma()
    for q in range(4):
        roles[f"softmax{q}"] = softmax(q)
        if not rec:
            roles[f"scatter{q}"] = scatter(q)
    return roles


def run(masks, rec, seed, **kw):
    """Random interleaving until every role ends. Returns None, or the names of the roles
    left waiting (deadlock). Raises Violation on a buffer overwritten too early."""
    rnd = random.Random(seed)
    roles = build(schedule(masks), rec, **kw)
    blocked = {}
    while roles:
        progressed = False
        for name in rnd.sample(list(roles), len(roles)):
            gen = roles[name]
            for _ in range(rnd.randint(1, 6)):
                try:
                    ev = next(gen)
                except StopIteration:
                    del roles[name]
                    blocked.pop(name, None)
                    progressed = True
                    break
                if ev[0] == "wait":
                    if blocked.get(name) != ev:
                        blocked[name] = ev
                        progressed = True
                    break
                blocked.pop(name, None)
                progressed = True
        if not progressed:
            return sorted(roles)
    return None


def random_masks(rnd):
    n = rnd.randint(1, 6)
    out = []
    for _ in range(n):
        kind = rnd.random()
        if kind < 0.15:
            out.append(0)                                   # token without an active tile
        elif kind < 0.4:
            out.append((1 << rnd.randint(1, N_TILE_BITS)) - 1)   # causal-like prefix
        else:
            out.append(rnd.getrandbits(N_TILE_BITS))
    return out


EDGE_MASKS = [[1], [1, 1], [0b11, 1], [1, 0xFFFF], [0xFFFF, 1, 0xFFFF], [0, 0, 1], [0], [],
              [1, 0, 1, 0, 1], [0b1010, 0b0101, 0b1111]]


@pytest.mark.parametrize("rec", [False, True], ids=["scatter", "record"])
def test_protocol_finishes_and_is_safe(rec):
    rnd = random.Random(20261202 + rec)
    cases = EDGE_MASKS + [random_masks(rnd) for _ in range(250)]
    for i, masks in enumerate(cases):
        for seed in range(3):
            stuck = run(masks, rec, seed=1000 * i + seed)
            assert stuck is None, f"deadlock with masks {masks}: {stuck}"


def test_protocol_paired_items_finishes_and_is_safe():
    """The record-mode kernel with items of two slot tiles: two K stages, two S buffers, one
    dS tile (the same barriers and hand-offs over fewer buffers)."""
    rnd = random.Random(20261204)
    cases = EDGE_MASKS + [random_masks(rnd) for _ in range(250)]
    for i, masks in enumerate(cases):
        for seed in range(3):
            stuck = run(masks, True, seed=1000 * i + seed, stages=2, ns=2, nd=1)
            assert stuck is None, f"deadlock with masks {masks}: {stuck}"


@pytest.mark.parametrize("rec", [False, True], ids=["scatter", "record"])
def test_protocol_128_heads_finishes_and_is_safe(rec):
    """The 128-head instances: three K stages, one dS tile (and dK^T buffer), and one S^T
    buffer in scatter mode (two in record mode, which has no dK^T buffers)."""
    rnd = random.Random(20261203 + rec)
    cases = EDGE_MASKS + [random_masks(rnd) for _ in range(250)]
    for i, masks in enumerate(cases):
        for seed in range(3):
            stuck = run(masks, rec, seed=1000 * i + seed, stages=3, ns=2 if rec else 1, nd=1)
            assert stuck is None, f"deadlock with masks {masks}: {stuck}"


def test_schedule_order():
    """Phase k interleaves B(t_{k-1}) and A(t_k), B first; every tile is visited once per
    pass; first / last flags mark each token's pass boundaries."""
    items = schedule([0b11, 0, 0b111])
    got = [(it["kind"], it["t"], it["tile"]) for it in items]
    assert got == [(0, 0, 0), (0, 0, 1),
                   (1, 0, 0), (0, 2, 0), (1, 0, 1), (0, 2, 1), (0, 2, 2),
                   (1, 2, 0), (1, 2, 1), (1, 2, 2)]
    for kind in (0, 1):
        for t in (0, 2):
            mine = [it for it in items if it["kind"] == kind and it["t"] == t]
            assert mine[0]["first"] and mine[-1]["last"]
            assert sum(it["first"] for it in mine) == 1 and sum(it["last"] for it in mine) == 1


def test_owner_only_producers_are_caught():
    """Producers that wait on a stage only at the items they own can pass its empty barrier
    two phases early (a fresh barrier reads as 'previous phase complete'); the model must
    catch that as an overwritten stage or a deadlock."""
    rnd = random.Random(7)
    caught = 0
    for i in range(60):
        masks = random_masks(rnd) + [0xFFFF]
        try:
            if run(masks, rec=True, seed=i, owner_producers=True) is not None:
                caught += 1
        except Violation:
            caught += 1
    assert caught > 0


# ---------------------------------------------------------------------------
# key-major dK kernel (sparse_lightning_indexer_b200/csrc/slikl_dk_keymajor.cu)
# ---------------------------------------------------------------------------

def km_items(runs, group=1):
    """Stages of one CTA. An item is one (query row, work unit); consecutive units on the same
    key block pair form a run (first / last mark its ends). runs = list of run lengths. A stage
    takes up to `group` consecutive items of one run (query rows of fewer than 64 heads share a
    stage), ending at its run's last item, as KmGroup::next forms them."""
    items = []
    for r, n in enumerate(runs):
        for k in range(n):
            items.append(dict(run=r, first=k == 0, last=k == n - 1))
    stages, i = [], 0
    while i < len(items):
        rows = []
        while len(rows) < group and i < len(items):
            rows.append(items[i])
            i += 1
            if rows[-1]["last"]:
                break
        stages.append(dict(run=rows[0]["run"], first=rows[0]["first"], last=rows[-1]["last"],
                           n=len(rows)))
    return stages


def km_build(items, sq=4, sr=5, sd=2, hold=True, builders=16, flushers=4, skip=None):
    """Roles of the key-major kernel over its three rings: w-scaled q (sq slots, loaded by the
    q producer, released by the MMA), records (sr slots, loaded by the record producer,
    released by the builders once read) and dS tiles (sd slots, written by the builders,
    released by the MMA). hold: the builders release the record slot before they wait for the
    dS slot (else, with 128 heads, they wait for the dS slot first). skip names a planted
    mistake: the wait that role leaves out ("qempty": q producer, "rempty": record producer,
    "dsempty": builders)."""
    bars = {}
    for s in range(sq):
        bars[f"qfull{s}"] = Bar(1)
        bars[f"qempty{s}"] = Bar(1)
    for s in range(sr):
        bars[f"rfull{s}"] = Bar(1)
        bars[f"rempty{s}"] = Bar(builders)
    for s in range(sd):
        bars[f"dsr{s}"] = Bar(builders)
        bars[f"dsempty{s}"] = Bar(1)
    for b in range(2):
        bars[f"accf{b}"] = Bar(1)
        bars[f"acce{b}"] = Bar(flushers)
    serial = itertools.count()
    # q_in[s] / rec_in[s] / ds_in[w][s]: the group whose data a slot holds; q_done[s],
    # rec_read[w][s], ds_done[s]: uses of a slot finished by its consumer(s)
    st = dict(q_in=[None] * sq, q_done=[0] * sq, rec_in=[None] * sr,
              rec_read=[[0] * sr for _ in range(builders)],
              ds_in=[[None] * sd for _ in range(builders)], ds_done=[0] * sd,
              acc_run=[None, None], acc_flushed=[[0, 0] for _ in range(flushers)])

    def wait(name, parity):
        token = next(serial)
        while not bars[name].ready(parity):
            yield ("wait", name, token)

    def q_producer():
        for i, _ in enumerate(items):
            s = i % sq
            if skip != "qempty":
                yield from wait(f"qempty{s}", ((i // sq) & 1) ^ 1)
            if st["q_done"][s] < i // sq:
                raise Violation(f"q producer overwrote q slot {s} (group {i}) still in use")
            st["q_in"][s] = i
            bars[f"qfull{s}"].arrive()
            yield ("step",)

    def rec_producer():
        for i, _ in enumerate(items):
            s = i % sr
            if skip != "rempty":
                yield from wait(f"rempty{s}", ((i // sr) & 1) ^ 1)
            if min(w[s] for w in st["rec_read"]) < i // sr:
                raise Violation(f"record producer overwrote records slot {s} (group {i}) "
                                "not yet read")
            st["rec_in"][s] = i
            bars[f"rfull{s}"].arrive()
            yield ("step",)

    def builder(wb):
        for i, _ in enumerate(items):
            r, d = i % sr, i % sd
            yield from wait(f"rfull{r}", (i // sr) & 1)
            if not hold and skip != "dsempty":
                yield from wait(f"dsempty{d}", ((i // sd) & 1) ^ 1)
            if st["rec_in"][r] != i:
                raise Violation(f"builder {wb} read records slot {r} not holding group {i}")
            st["rec_read"][wb][r] += 1
            bars[f"rempty{r}"].arrive()
            yield ("step",)
            if hold and skip != "dsempty":
                yield from wait(f"dsempty{d}", ((i // sd) & 1) ^ 1)
            if st["ds_done"][d] < i // sd:
                raise Violation(f"builder {wb} overwrote dS slot {d} (group {i}) still in use")
            st["ds_in"][wb][d] = i
            bars[f"dsr{d}"].arrive()
            yield ("step",)

    def mma():
        nrun = 0
        for i, it in enumerate(items):
            q, d, ab = i % sq, i % sd, nrun & 1
            yield from wait(f"qfull{q}", (i // sq) & 1)
            yield from wait(f"dsr{d}", (i // sd) & 1)
            if st["q_in"][q] != i:
                raise Violation(f"MMA read q slot {q} not holding group {i}")
            if any(w[d] != i for w in st["ds_in"]):
                raise Violation(f"MMA read dS slot {d} not holding group {i}")
            if it["first"]:
                yield from wait(f"acce{ab}", ((nrun >> 1) & 1) ^ 1)
                if min(w[ab] for w in st["acc_flushed"]) < nrun >> 1:
                    raise Violation(f"dK buffer {ab} reused (run {nrun}) before its flush")
                st["acc_run"][ab] = it["run"]
            elif st["acc_run"][ab] != it["run"]:
                raise Violation(f"run {it['run']} accumulates into buffer {ab} of another run")
            st["q_done"][q] += 1
            st["ds_done"][d] += 1
            bars[f"qempty{q}"].arrive()
            bars[f"dsempty{d}"].arrive()
            if it["last"]:
                bars[f"accf{ab}"].arrive()
                nrun += 1
            yield ("step",)

    def flush(wf):
        nrun = 0
        for it in items:
            if not it["last"]:
                continue
            ab = nrun & 1
            yield from wait(f"accf{ab}", (nrun >> 1) & 1)
            if st["acc_run"][ab] != it["run"]:
                raise Violation(f"flush of run {it['run']} found buffer {ab} holding another run")
            st["acc_flushed"][wf][ab] += 1
            bars[f"acce{ab}"].arrive()
            nrun += 1
            yield ("step",)

    roles = {"q_producer": q_producer(), "rec_producer": rec_producer(), "mma": mma()}
    for w in range(builders):
        roles[f"builder{w}"] = builder(w)
    for w in range(flushers):
        roles[f"flush{w}"] = flush(w)
    return roles


def km_run(runs, seed, group=1, **kw):
    rnd = random.Random(seed)
    roles = km_build(km_items(runs, group), **kw)
    blocked = {}
    while roles:
        progressed = False
        for name in rnd.sample(list(roles), len(roles)):
            gen = roles[name]
            for _ in range(rnd.randint(1, 6)):
                try:
                    ev = next(gen)
                except StopIteration:
                    del roles[name]
                    progressed = True
                    break
                if ev[0] == "wait":
                    if blocked.get(name) != ev:
                        blocked[name] = ev
                        progressed = True
                    break
                blocked.pop(name, None)
                progressed = True
        if not progressed:
            return sorted(roles)
    return None


# (q slots, record slots, dS slots, query rows per stage, chunks held across the dS wait) of
# the kernel's instances
KM_SHAPES = {"16heads": (4, 5, 2, 4, True), "32heads": (4, 8, 2, 2, True),
             "64heads": (4, 8, 2, 1, True), "128heads": (2, 3, 2, 1, False)}


@pytest.mark.parametrize("shape", list(KM_SHAPES))
def test_keymajor_protocol_finishes_and_is_safe(shape):
    sq, sr, sd, group, hold = KM_SHAPES[shape]
    rnd = random.Random(20261203)
    cases = [[1], [1, 1, 1], [32], [1, 32, 1], [5, 5, 5, 5, 5], [3, 4, 5, 6, 7]]
    cases += [[rnd.randint(1, 12) for _ in range(rnd.randint(1, 8))] for _ in range(150)]
    for i, runs in enumerate(cases):
        for seed in range(3):
            assert km_run(runs, seed=1000 * i + seed, group=group, sq=sq, sr=sr, sd=sd,
                          hold=hold) is None, f"deadlock with runs {runs}"


@pytest.mark.parametrize("group", [1, 2, 4])
def test_keymajor_stage_groups(group):
    """Stages keep the item order, hold rows of one run only, at most `group` of them, and
    are full except where a run ends."""
    rnd = random.Random(group)
    for _ in range(200):
        runs = [rnd.randint(1, 13) for _ in range(rnd.randint(1, 9))]
        st = km_items(runs, group)
        assert sum(x["n"] for x in st) == sum(runs)
        for r, n in enumerate(runs):
            mine = [x for x in st if x["run"] == r]
            assert [x["n"] for x in mine] == [group] * (n // group) + ([n % group] if n % group else [])
            assert mine[0]["first"] and mine[-1]["last"]
            assert not any(x["first"] for x in mine[1:]) and not any(x["last"] for x in mine[:-1])


@pytest.mark.parametrize("hold", [True, False])
@pytest.mark.parametrize("skip", ["qempty", "rempty", "dsempty"])
def test_keymajor_planted_mistake_is_caught(skip, hold):
    rnd = random.Random(11)
    caught = 0
    for i in range(40):
        runs = [rnd.randint(1, 12) for _ in range(rnd.randint(2, 8))]
        try:
            if km_run(runs, seed=i, skip=skip, sq=2, sr=2, sd=2, hold=hold) is not None:
                caught += 1
        except Violation:
            caught += 1
    assert caught > 0
