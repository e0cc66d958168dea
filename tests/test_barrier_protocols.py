"""Model check of the kernels' mbarrier protocols (CPU, no GPU).

Each pipeline of the CUDA kernels is restated here as roles (TMA producer,
dequantiser, MMA issuer, elementwise/softmax warps) that wait on and arrive at
barriers with the kernels' own slot and parity formulas. An mbarrier is a
completed-phase counter; a parity wait succeeds when the phase with that
parity has completed, which is only meaningful while the barrier is at most
one phase away from the use the waiter expects. The simulation advances the
roles in random interleavings and completes TMA copies in random order, and
fails on: a deadlock, a slot refilled while its contents are still to be read,
or a wait that sees its barrier two phases away.

Pipelines: the attention forward's K/V ring with the INT8 cache's staged code
slots (a prefix of cache tiles dequantised into the ring, then current tiles
loaded directly), the backward's dQ and dK/dV kernels, and the camera
cross-attention's per-warp ring of staged row tiles.
"""
import random

import pytest


class Bar:
    def __init__(self, count):
        self.count, self.pending, self.completed, self.tx = count, count, 0, 0

    def arrive(self, n=1):
        self.pending -= n
        assert self.pending >= 0, "more arrivals than the barrier's count"
        self._check()

    def expect(self, nbytes):  # arrive.expect_tx
        self.tx += nbytes
        self.arrive()

    def complete_tx(self, nbytes):
        self.tx -= nbytes
        assert self.tx >= 0
        self._check()

    def _check(self):
        if self.pending == 0 and self.tx == 0:
            self.completed += 1
            self.pending = self.count


def wait(name, parity, use):
    """Wait for use `use` (0-based) of barrier `name` to complete."""
    return ("wait", name, parity, use)


def run(roles, bars, seed):
    rng = random.Random(seed)
    waiting = {k: None for k in roles}
    done, copies = set(), []
    while len(done) < len(roles):
        progressed = False
        if copies and rng.random() < 0.5:
            name, nbytes = copies.pop(rng.randrange(len(copies)))
            bars[name].complete_tx(nbytes)
            progressed = True
        order = list(roles)
        rng.shuffle(order)
        for k in order:
            if k in done:
                continue
            w = waiting[k]
            if w is not None:
                _, name, parity, use = w
                b = bars[name]
                if (b.completed & 1) != parity:
                    assert b.completed == use + 1, (k, name, "barrier a phase ahead", b.completed, use)
                    waiting[k] = None
                else:
                    assert b.completed == use, (k, name, "barrier a phase behind", b.completed, use)
                    continue
            try:
                while True:
                    ev = next(roles[k])
                    if ev[0] == "wait":
                        waiting[k] = ev
                        break
                    if ev[0] == "copy":
                        copies.append((ev[1], ev[2]))
                    if ev[0] == "work" and rng.random() < 0.3:
                        break
                progressed = True
            except StopIteration:
                done.add(k)
                progressed = True
        assert progressed or copies, ("deadlock", {k: waiting[k] for k in roles if k not in done})
    assert not copies, "a copy still in flight when the CTA exits"


# ---------------------------------------------------------------------------
# attention forward, INT8 cache: ring of `ring` operand slots, `cslots` code
# slots; iteration it = 2j (K of key tile j) or 2j + 1 (V)
# ---------------------------------------------------------------------------

def forward_int8(staged_tiles, ring, cslots, seed):
    n = len(staged_tiles)
    bars = {}
    for s in range(ring):
        bars[("full", s)] = Bar(128)
        bars[("empty", s)] = Bar(1)
    for s in range(cslots):
        bars[("cfull", s)] = Bar(1)
        bars[("cempty", s)] = Bar(128)
    for t in range(2):
        bars[("S", t)] = Bar(1)
        bars[("P", t)] = Bar(1)
        bars[("O", t)] = Bar(1)
    ring_owner, code_owner = {}, {}
    staged = lambda i: staged_tiles[i >> 1]  # noqa: E731

    def producer():
        for it in range(2 * n):
            if staged(it):
                cs = it % cslots
                yield wait(("cempty", cs), ((it // cslots) & 1) ^ 1, it // cslots - 1)
                assert code_owner.get(cs) is None
                code_owner[cs] = it
                bars[("cfull", cs)].expect(1)
                yield ("copy", ("cfull", cs), 1)
            else:
                if it > 0 and staged(it - 1):  # wait for the whole staged prefix
                    for i2 in range(max(0, it - cslots), it):
                        yield wait(("cempty", i2 % cslots), (i2 // cslots) & 1, i2 // cslots)
                s = it % ring
                yield wait(("empty", s), ((it // ring) & 1) ^ 1, it // ring - 1)
                assert ring_owner.get(s) is None, "ring slot refilled while in use"
                ring_owner[s] = it
                bars[("full", s)].expect(1)
                bars[("full", s)].arrive(127)
                yield ("copy", ("full", s), 1)

    def dequantiser():
        for it in range(2 * n):
            if not staged(it):
                break
            cs, s = it % cslots, it % ring
            yield wait(("cfull", cs), (it // cslots) & 1, it // cslots)
            yield wait(("empty", s), ((it // ring) & 1) ^ 1, it // ring - 1)
            assert code_owner.get(cs) == it and ring_owner.get(s) is None
            ring_owner[s] = it
            yield ("work",)
            bars[("full", s)].arrive(128)
            code_owner[cs] = None
            bars[("cempty", cs)].arrive(128)

    def mma():
        def use(it):
            assert ring_owner.get(it % ring) == it, "operand slot holds another tile"

        def release(it):
            use(it)
            ring_owner[it % ring] = None
            bars[("empty", it % ring)].arrive()

        if n:
            yield wait(("full", 0), 0, 0)
            use(0)
            bars[("S", 0)].arrive()
            bars[("S", 1)].arrive()
            release(0)
        for j in range(n):
            itv, itk = 2 * j + 1, 2 * j + 2
            more = j + 1 < n
            # V of this tile and K of the next one before P of tile 0
            yield wait(("full", itv % ring), (itv // ring) & 1, itv // ring)
            if more:
                yield wait(("full", itk % ring), (itk // ring) & 1, itk // ring)
            yield wait(("P", 0), j & 1, j)
            use(itv)
            if more:
                use(itk)
                bars[("S", 0)].arrive()
            yield wait(("P", 1), j & 1, j)
            release(itv)
            if more:
                bars[("S", 1)].arrive()
                release(itk)
        bars[("O", 0)].arrive()
        bars[("O", 1)].arrive()

    def softmax(t):
        for j in range(n):
            yield wait(("S", t), j & 1, j)
            yield ("work",)
            bars[("P", t)].arrive()
        if n:
            yield wait(("O", t), 0, 0)

    run({"producer": producer(), "dequantiser": dequantiser(), "mma": mma(),
         "softmax0": softmax(0), "softmax1": softmax(1)}, bars, seed)


@pytest.mark.parametrize("ring, cslots", [(3, 4), (4, 2), (3, 3), (2, 5)])
def test_forward_int8_pipeline(ring, cslots):
    """The shipped INT8 depths (3 ring slots, 4 code slots) and others; every
    prefix length of cache tiles, including none (the bf16 case) and all."""
    for n in range(0, 9):
        for n_staged in range(0, n + 1):
            for seed in range(8):
                forward_int8([True] * n_staged + [False] * (n - n_staged), ring, cslots, seed)


# ---------------------------------------------------------------------------
# backward: dQ (query-major) and dK/dV (key-major)
# ---------------------------------------------------------------------------

def backward_dq(n, seed, ks=3, vs=2):
    bars = {("KF", s): Bar(1) for s in range(ks)}
    bars.update({("KE", s): Bar(1) for s in range(ks)})
    bars.update({("VF", s): Bar(1) for s in range(vs)})
    bars.update({("VE", s): Bar(1) for s in range(vs)})
    for name in ("QD", ("S", 0), ("S", 1), "DP", "DONE", ("DS", 0), ("DS", 1), "RD"):
        bars[name] = Bar(1)
    kslot, vslot, sbuf, dp = {}, {}, {}, {}

    def producer():
        bars["QD"].expect(1)
        yield ("copy", "QD", 1)
        for j in range(n):
            yield wait(("KE", j % ks), ((j // ks) & 1) ^ 1, j // ks - 1)
            assert kslot.get(j % ks) is None
            kslot[j % ks] = j
            bars[("KF", j % ks)].expect(1)
            yield ("copy", ("KF", j % ks), 1)
            yield wait(("VE", j % vs), ((j // vs) & 1) ^ 1, j // vs - 1)
            assert vslot.get(j % vs) is None
            vslot[j % vs] = j
            bars[("VF", j % vs)].expect(1)
            yield ("copy", ("VF", j % vs), 1)

    def qk(j, buf):
        assert kslot[j % ks] == j and sbuf.get(buf) in (None, "read")
        sbuf[buf] = ("S", j)

    def mma_s_dq():  # one issuing thread: S = Q Kᵀ and dQ += dS K
        yield wait("QD", 0, 0)
        if n:
            yield wait(("KF", 0), 0, 0)
            qk(0, 0)
            bars[("S", 0)].arrive()
        if n > 1:
            yield wait(("KF", 1), 0, 0)
            qk(1, 1)
            bars[("S", 1)].arrive()
        for j in range(n):
            yield wait(("DS", j & 1), (j >> 1) & 1, j >> 1)
            assert sbuf[j & 1] == ("dS", j) and kslot[j % ks] == j
            sbuf[j & 1] = "read"
            kslot[j % ks] = None
            bars[("KE", j % ks)].arrive()
            if j + 2 < n:
                yield wait(("KF", (j + 2) % ks), ((j + 2) // ks) & 1, (j + 2) // ks)
                qk(j + 2, j & 1)
                bars[("S", j & 1)].arrive()
        bars["DONE"].arrive()

    def issue_dp(j):
        assert vslot[j % vs] == j and (j == 0 or dp.get("read") == j - 1)
        dp["v"] = j
        bars["DP"].arrive()
        vslot[j % vs] = None
        bars[("VE", j % vs)].arrive()

    def mma_dp():  # the other issuing thread: dP = dO Vᵀ
        yield wait("QD", 0, 0)
        if n:
            yield wait(("VF", 0), 0, 0)
            issue_dp(0)
        for j in range(n - 1):
            yield wait("RD", j & 1, j)
            yield wait(("VF", (j + 1) % vs), ((j + 1) // vs) & 1, (j + 1) // vs)
            issue_dp(j + 1)

    def elementwise():
        for j in range(n):
            yield wait(("S", j & 1), (j >> 1) & 1, j >> 1)
            yield wait("DP", j & 1, j)
            assert sbuf[j & 1] == ("S", j) and dp["v"] == j
            dp["read"] = j
            bars["RD"].arrive()
            yield ("work",)
            sbuf[j & 1] = ("dS", j)
            bars[("DS", j & 1)].arrive()
        yield wait("DONE", 0, 0)

    run({"producer": producer(), "mma_s_dq": mma_s_dq(), "mma_dp": mma_dp(),
         "elementwise": elementwise()}, bars, seed)


def backward_dkdv(n, seed, qslots=3, oslots=2):
    """The dK/dV kernel: a Q ring (3) and a ring of dO stages with −D, −L (2),
    each with its own loader; TMEM regions X, Y swap roles per query tile:
    Sᵀ_i into region i % 2, then Pᵀ_i and dSᵀ_i over it; dPᵀ_i into region
    (i + 1) % 2. Region contents are tracked, and every product or store
    checks what it overwrites."""
    bars = {}
    for s in range(qslots):
        bars[("QF", s)], bars[("QE", s)] = Bar(1), Bar(1)
    for s in range(oslots):
        bars[("OF", s)], bars[("OE", s)] = Bar(1), Bar(1)
    for name in ("KV", "ST", "DPT", "DONE"):
        bars[name] = Bar(1)
    for name in ("RD", "PR", "DS"):  # the elementwise warps (one arrival stands for 256)
        bars[name] = Bar(1)
    qring, oring, reg, dp_read = {}, {}, {0: None, 1: None}, set()

    def producer_q():
        bars["KV"].expect(1)
        yield ("copy", "KV", 1)
        for i in range(n):
            s = i % qslots
            yield wait(("QE", s), ((i // qslots) & 1) ^ 1, i // qslots - 1)
            assert qring.get(s) is None, "Q slot refilled while in use"
            qring[s] = i
            bars[("QF", s)].expect(1)
            yield ("copy", ("QF", s), 1)

    def producer_o():
        for i in range(n):
            s = i % oslots
            yield wait(("OE", s), ((i // oslots) & 1) ^ 1, i // oslots - 1)
            assert oring.get(s) is None, "dO slot refilled while in use"
            oring[s] = i
            bars[("OF", s)].expect(1)
            yield ("copy", ("OF", s), 1)

    def issue_s(i):  # Sᵀ_i into region i % 2, over dPᵀ_{i-1} once it has been read out
        assert qring.get(i % qslots) == i
        cur = reg[i % 2]
        assert cur is None or (cur == ("dP", i - 1) and i - 1 in dp_read), ("S over live", cur)
        reg[i % 2] = ("S", i)
        bars["ST"].arrive()

    def issue_dp(i):  # dPᵀ_i into region (i + 1) % 2, after dV and dK of tile i - 1
        assert oring.get(i % oslots) == i
        cur = reg[(i + 1) % 2]
        assert cur is None or cur == ("PdS", i - 1), ("dP over live", cur)
        reg[(i + 1) % 2] = ("dP", i)
        bars["DPT"].arrive()

    def mma():
        # products are modelled at issue (the tensor pipe runs them in order)
        yield wait("KV", 0, 0)
        if n:
            yield wait(("QF", 0), 0, 0)
            yield wait(("OF", 0), 0, 0)
            issue_s(0)
            issue_dp(0)
        for i in range(n):
            more = i + 1 < n
            yield wait("PR", i & 1, i)
            if more:  # the next Sᵀ ahead of dV
                yield wait("RD", i & 1, i)
                yield wait(("QF", (i + 1) % qslots), ((i + 1) // qslots) & 1, (i + 1) // qslots)
                issue_s(i + 1)
            # dV from Pᵀ_i and dO_i
            assert reg[i % 2] in (("P", i), ("PdS", i)) and oring.get(i % oslots) == i
            if more:  # the next dO stage first, so that dK and the next dPᵀ go out together
                yield wait(("OF", (i + 1) % oslots), ((i + 1) // oslots) & 1, (i + 1) // oslots)
            yield wait("DS", i & 1, i)  # dK from dSᵀ_i and Q_i
            assert reg[i % 2] == ("PdS", i) and qring.get(i % qslots) == i
            qring[i % qslots] = None
            bars[("QE", i % qslots)].arrive()
            oring[i % oslots] = None  # dV and the elementwise warps are done with the dO stage
            bars[("OE", i % oslots)].arrive()
            if more:
                issue_dp(i + 1)
        bars["DONE"].arrive()

    def elementwise():
        for i in range(n):
            yield wait("ST", i & 1, i)
            yield wait(("OF", i % oslots), (i // oslots) & 1, i // oslots)
            assert reg[i % 2] == ("S", i) and oring.get(i % oslots) == i  # −L from the stage
            yield ("work",)
            reg[i % 2] = ("P", i)  # Pᵀ over the scores just read
            bars["PR"].arrive()
            yield wait("DPT", i & 1, i)
            assert reg[(i + 1) % 2] == ("dP", i)
            dp_read.add(i)
            bars["RD"].arrive()
            yield ("work",)
            assert reg[i % 2] == ("P", i) and oring.get(i % oslots) == i  # −D from the stage
            reg[i % 2] = ("PdS", i)
            bars["DS"].arrive()
        yield wait("DONE", 0, 0)

    run({"producer_q": producer_q(), "producer_o": producer_o(), "mma": mma(),
         "elementwise": elementwise()}, bars, seed)


def test_backward_dq_pipeline():
    for n in range(0, 12):
        for seed in range(25):
            backward_dq(n, seed)


def test_backward_dkdv_pipeline():
    for n in range(0, 12):
        for seed in range(25):
            backward_dkdv(n, seed)


def test_single_ds_barrier_would_be_caught():
    """The model check is sharp: with one dS barrier instead of two (the
    dQ kernel before the fix), some interleaving lets the elementwise warps
    run two phases ahead of the MMA thread's parity wait."""
    import re
    import inspect
    src = inspect.getsource(backward_dq)
    src = re.sub(r'\("DS", j & 1\), \(j >> 1\) & 1, j >> 1', '("DS", 0), j & 1, j', src)
    src = src.replace('bars[("DS", j & 1)].arrive()', 'bars[("DS", 0)].arrive()')
    scope = dict(globals())
    exec(src, scope)
    with pytest.raises(AssertionError):
        for n in range(2, 8):
            for seed in range(40):
                scope["backward_dq"](n, seed)


def test_missing_prefix_wait_would_be_caught():
    """Likewise for the INT8 producer: without its wait for the staged prefix
    before the first direct load, more code slots than ring slots let a
    parity wait on a ring slot pass a phase early."""
    import inspect
    src = inspect.getsource(forward_int8)
    src = src.replace("if it > 0 and staged(it - 1):", "if False:")
    scope = dict(globals())
    exec(src, scope)
    with pytest.raises(AssertionError):
        for n in range(2, 9):
            for n_staged in range(1, n):
                for seed in range(8):
                    scope["forward_int8"]([True] * n_staged + [False] * (n - n_staged), 2, 5, seed)


@pytest.mark.parametrize("mutation", ["no read-out wait before the next S", "next dP before dS"])
def test_dkdv_region_hazards_would_be_caught(mutation):
    """The dK/dV model is sharp: Sᵀ of the next query tile issued before dPᵀ
    was read out of its region, or dPᵀ of the next tile issued before dK had
    read dSᵀ, is reported in some interleaving."""
    import inspect
    src = inspect.getsource(backward_dkdv)
    if mutation.startswith("no read-out"):
        src = src.replace('                yield wait("RD", i & 1, i)\n', '')
    else:
        src = src.replace(
            '            yield wait("DS", i & 1, i)  # dK from dSᵀ_i and Q_i',
            '            if more:\n'
            '                yield wait(("OF", (i + 1) % oslots), ((i + 1) // oslots) & 1, (i + 1) // oslots)\n'
            '                issue_dp(i + 1)\n'
            '                more = False\n'
            '            yield wait("DS", i & 1, i)  # dK from dSᵀ_i and Q_i')
    assert src != inspect.getsource(backward_dkdv)
    scope = dict(globals())
    exec(src, scope)
    with pytest.raises(AssertionError):
        for n in range(2, 8):
            for seed in range(40):
                scope["backward_dkdv"](n, seed)


# ---------------------------------------------------------------------------
# camera cross-attention: a producer streams each 128-row tile's q (ring of
# qs stages) and, once per run of tiles of one head, that head's camera K/V
# (2 entries); one MMA thread issues S_k into tensor-memory buffer k % 2,
# then P V of the previous tile; the epilogue warpgroup k % 2 takes tile k
# (softmax, then x + O / l over x); a store thread sends each finished tile
# back and then loads the x of tile k + xs into the freed stage (it also arms
# the first xs)
# ---------------------------------------------------------------------------

def camera_pipeline(heads, qs, xper, seed, mutation=None):
    """xper x stages per epilogue warpgroup: tile k, the m-th tile (m = k // 2)
    of warpgroup k % 2, uses x stage (k % 2)·xper + m % xper and the store
    barrier (k % 2, m % 2). Mutation "shared x ring" puts the x stages of
    both warpgroups in one ring of 2·xper + 1 stages (tile k in stage k mod
    that), as an earlier build did."""
    n = len(heads)
    shared = mutation == "shared x ring"
    xs = 2 * xper + 1 if shared else 2 * xper
    stage = (lambda k: k % xs) if shared else (lambda k: (k & 1) * xper + (k >> 1) % xper)
    use = (lambda k: k // xs) if shared else (lambda k: (k >> 1) // xper)
    bars = {("kvfull", e): Bar(1) for e in range(2)}
    bars.update({("kvempty", e): Bar(1) for e in range(2)})
    bars.update({("qfull", s): Bar(1) for s in range(qs)})
    bars.update({("qempty", s): Bar(1) for s in range(qs)})
    bars.update({("xfull", s): Bar(1) for s in range(xs)})
    for j in range(2):
        for name in ("S", "P", "O"):
            bars[(name, j)] = Bar(1)
        for b in range(2):
            bars[("Store", j, b)] = Bar(1)
    kv_owner, q_owner, x_owner = {}, {}, {}
    s_tile, o_tile = {}, {}
    pv_issued, o_read = set(), set()

    def producer():
        run, hprev = -1, None
        for k, h in enumerate(heads):
            if h != hprev:
                if run >= 1 and mutation != "no kv wait":
                    u = (run + 1) // 2 - 1
                    yield wait(("kvempty", (run + 1) & 1), u & 1, u)
                run, hprev = run + 1, h
                e = run & 1
                assert kv_owner.get(e) is None, "K/V entry refilled while in use"
                kv_owner[e] = run
                bars[("kvfull", e)].expect(4)
                for _ in range(4):
                    yield ("copy", ("kvfull", e), 1)
            sq = k % qs
            if k >= qs:
                yield wait(("qempty", sq), (k // qs - 1) & 1, k // qs - 1)
            assert q_owner.get(sq) is None, "q stage refilled while in use"
            q_owner[sq] = k
            bars[("qfull", sq)].expect(2)
            yield ("copy", ("qfull", sq), 1)
            yield ("copy", ("qfull", sq), 1)

    def mma():
        def pv(i, ri, last):
            j = i & 1
            yield wait(("P", j), (i >> 1) & 1, i >> 1)
            assert s_tile.get(j) == i and kv_owner.get(ri & 1) == ri
            assert i < 2 or (i - 2) in o_read, "O buffer overwritten before it was read"
            o_tile[j] = i
            pv_issued.add(i)
            bars[("O", j)].arrive()
            if last:
                kv_owner[ri & 1] = None
                bars[("kvempty", ri & 1)].arrive()

        run, hprev, run_prev = -1, None, 0
        for k, h in enumerate(heads):
            if h != hprev:
                run, hprev = run + 1, h
                yield wait(("kvfull", run & 1), (run >> 1) & 1, run >> 1)
            sq, j = k % qs, k & 1
            yield wait(("qfull", sq), (k // qs) & 1, k // qs)
            assert q_owner.get(sq) == k and kv_owner.get(run & 1) == run
            assert k < 2 or (k - 2) in pv_issued, "S buffer overwritten before its P was used"
            s_tile[j] = k
            q_owner[sq] = None
            bars[("qempty", sq)].arrive()
            bars[("S", j)].arrive()
            if k >= 1:
                yield from pv(k - 1, run_prev, h != heads[k - 1])
            run_prev = run
        if n:
            yield from pv(n - 1, run_prev, True)

    def epilogue(wg):
        for k in range(wg, n, 2):
            m, sx = k >> 1, stage(k)
            yield wait(("S", wg), m & 1, m)
            assert s_tile.get(wg) == k
            yield ("work",)
            bars[("P", wg)].arrive()
            # x first (it has usually landed long before O), then O
            yield wait(("xfull", sx), use(k) & 1, use(k))
            assert x_owner.get(sx) == k, "epilogue reads another tile's x"
            yield wait(("O", wg), m & 1, m)
            assert o_tile.get(wg) == k, "epilogue reads another tile's O"
            yield ("work",)
            o_read.add(k)
            bars[("Store", wg, m & 1)].arrive()

    def store():
        ahead = xs if shared else 2 * xper   # the next tile that uses tile k's stage

        def load_x(t):
            sx = stage(t)
            assert x_owner.get(sx) is None, "x stage refilled while in use"
            x_owner[sx] = t
            bars[("xfull", sx)].expect(2)
            return [("copy", ("xfull", sx), 1), ("copy", ("xfull", sx), 1)]

        loaded = 0
        while loaded < min(n, ahead):
            yield from load_x(loaded)
            loaded += 1
        for k in range(n):
            m = k >> 1
            yield wait(("Store", k & 1, m & 1), (m >> 1) & 1, m >> 1)
            assert x_owner.get(stage(k)) == k and k in o_read
            yield ("work",)
            x_owner[stage(k)] = None
            if k + ahead < n:
                yield from load_x(k + ahead)
                loaded += 1

    run({"producer": producer(), "mma": mma(), "epi0": epilogue(0), "epi1": epilogue(1),
         "store": store()}, bars, seed)


def _camera_heads(rng):
    """Head of every tile of one CTA's range: runs of 1 to 12 tiles."""
    heads, h = [], rng.randint(0, 3)
    for _ in range(rng.randint(1, 4)):
        heads += [h] * rng.randint(1, 12)
        h += 1
    return heads


@pytest.mark.parametrize("qs, xper", [(3, 1), (2, 2), (2, 1), (4, 1), (3, 2)])
def test_camera_pipeline(qs, xper):
    """The shipped depths (3 q stages, 1 x stage per warpgroup) and others;
    ranges of one tile, of one head, and of several heads."""
    for seed in range(300):
        camera_pipeline(_camera_heads(random.Random(seed)), qs, xper, seed)


@pytest.mark.parametrize("mutation", ["no kv wait", "shared x ring"])
def test_camera_hazards_would_be_caught(mutation):
    """(O needs no free barrier: a warpgroup arrives at P of tile i only after
    it has read O of tile i - 2, which the model checks on every P V. A ring
    of x stages shared by the two warpgroups lets one warpgroup wait on a
    stage's next phase before the other has consumed the current one, so the
    parity wait can pass a phase early.)"""
    with pytest.raises(AssertionError):
        for seed in range(300):
            camera_pipeline(_camera_heads(random.Random(seed)), 2, 1, seed, mutation)
