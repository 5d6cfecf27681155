"""Model check of the chain kernel's mbarrier protocol (kla_chunk_tc.cu).

The chain kernel's warp roles talk only through mbarriers.  This test
replays the same wait / arrive / issue / commit sequence of every role, in
many random interleavings (seeded), against a model of an mbarrier (phase
counter + arrival count, parity waits), an in-order tensor pipe (commits
arrive when everything issued before them has finished) and out-of-order TMA
completion.  It fails on:

  * deadlock (no role can move and nothing is in flight),
  * a parity wait that finds its barrier two or more phases ahead -- the
    waiter would then block on a later phase, which on the GPU is a hang,
  * reuse hazards of TMEM accumulators and shared-memory slots: a buffer
    overwritten before its previous reader of the same data has finished.

The sequences below must be kept identical to the kernel's program order,
in both of its modes: the scalar gate and the per-channel gate (KDA).
"""
import random

import pytest


class Bar:
    def __init__(self, count):
        self.count, self.pending, self.phase = count, count, 0

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0
        if self.pending == 0:
            self.phase += 1
            self.pending = self.count


class Hazard(AssertionError):
    pass


def build(N, kda=False):
    bars = {}

    def B(name, count):
        bars[name] = Bar(count)

    for i in range(2):
        B(("full", i), 1); B(("empty", i), 1); B(("u_free", i), 8)
    for i in range(3):
        B(("g_ready", i), 1)
    for name, c in [("bS", 1), ("bW", 1), ("bX", 1), ("bH", 1), ("bHP", 1), ("p_done", 4),
                    ("w_done", 2), ("vpd_ready", 4), ("vp_ready", 4), ("h_done", 8),
                    ("pv_free", 4)]:
        B(name, c)

    W = lambda bar, k: ("wait", bar, k)
    A = lambda bar: ("arrive", bar)
    I = lambda tag, n: ("issue", tag, n)
    Cm = lambda bar: ("commit", bar)
    Do = lambda tag, n: ("do", tag, n)

    roles = {}
    prod = []
    for n in range(N):
        if n >= 2:
            prod.append(W(("empty", n & 1), (n - 2) >> 1))
        prod.append(("tma", n))
    roles["producer"] = prod

    if kda:
        return bars, build_kda_roles(N, W, A, I, Cm, Do, prod)
    m = [W(("full", 0), 0), I("mma2", 0), Cm("bW"), I("mma3", 0),
         W("w_done", 0), I("mma1", 0), Cm("bS")]
    for n in range(N):
        more = n + 1 < N
        m += [W("w_done", n), W("h_done", n), I("mma4", n), Cm("bX")]
        if more:
            m += [W(("full", (n + 1) & 1), (n + 1) >> 1), I("mma2", n + 1), Cm("bW")]
        m += [W("vpd_ready", n), I("mma5", n), Cm("bH"), W("vp_ready", n), W("p_done", n)]
        if n > 0:
            m.append(W("pv_free", n - 1))
        m += [I("mma6", n), Cm("bHP"), Cm(("empty", n & 1))]
        if more:
            if n >= 1:
                m.append(W(("u_free", (n + 1) & 1), (n - 1) >> 1))
            m += [I("mma3", n + 1), W("w_done", n + 1), I("mma1", n + 1), Cm("bS")]
    roles["mma"] = m

    for w in (4, 5):
        seq = []
        for n in range(N):
            seq += [W("bW", n), Do("W", n), A("w_done")]
        roles[f"w{w}"] = seq
    for w in (2, 3, 14, 15):
        seq = []
        for n in range(N):
            if w == 2:
                seq += [Do("G", n), A(("g_ready", n % 3))]
            else:
                seq.append(W(("g_ready", n % 3), n // 3))
            seq += [Do("readG", n), W("bS", n), Do("P", n), A("p_done")]
        roles[f"p{w}"] = seq
    for w in range(6, 14):
        v_rows = (w & 3) < 2
        seq = [A("h_done")]
        for n in range(N):
            seq += [W(("g_ready", n % 3), n // 3), Do("readG", n)]
            if v_rows:
                seq += [W("bX", n), Do("Vpd", n), A("vpd_ready"), A(("u_free", n & 1)),
                        Do("Vp", n), A("vp_ready")]
            seq += [W("bH", n), Do("h", n), A("h_done")]
            if not v_rows:
                seq += [W("bHP", n), Do("o", n), A(("u_free", n & 1)), A("pv_free")]
        roles[f"c{w}"] = seq
    return bars, roles


def build_kda_roles(N, W, A, I, Cm, Do, prod):
    """The per-channel-gate mode: the stage brings W, P, Q o e^G, the decayed
    keys and the per-channel chunk decay, so there are no Q K^T or W
    products and no P or W epilogues; warp 2 copies the decay of chunk n from
    the stage into slot n % 3 of a ring (g_ready); V' is written once (no
    decayed copy) and feeds both MMA 5 and MMA 6; the state update reads the
    decay from the ring."""
    roles = {"producer": prod}
    m = [W(("full", 0), 0), I("mma3", 0)]
    for n in range(N):
        more = n + 1 < N
        m += [W("h_done", n), I("mma4", n), Cm("bX")]
        if more:
            m.append(W(("full", (n + 1) & 1), (n + 1) >> 1))
        m += [W("vpd_ready", n), I("mma5", n), Cm("bH"), W("vp_ready", n)]
        if n > 0:
            m.append(W("pv_free", n - 1))
        m += [I("mma6", n), Cm("bHP"), Cm(("empty", n & 1))]
        if more:
            if n >= 1:
                m.append(W(("u_free", (n + 1) & 1), (n - 1) >> 1))
            m.append(I("mma3", n + 1))
    roles["mma"] = m
    seq = []
    for n in range(N):
        seq += [W(("full", n & 1), n >> 1), Do("D", n), A(("g_ready", n % 3))]
    roles["p2"] = seq
    for w in range(6, 14):
        v_rows = (w & 3) < 2
        seq = [A("h_done")]
        for n in range(N):
            seq.append(W(("g_ready", n % 3), n // 3))
            if v_rows:
                seq += [W("bX", n), Do("Vp", n), A("vpd_ready"), A(("u_free", n & 1)),
                        A("vp_ready")]
            seq += [W("bH", n), Do("h", n), A("h_done")]
            if not v_rows:
                seq += [W("bHP", n), Do("o", n), A(("u_free", n & 1)), A("pv_free")]
        roles[f"c{w}"] = seq
    return roles


def run(N, seed, kda=False, mutate=None):
    rng = random.Random(seed)
    bars, roles = build(N, kda)
    if mutate is not None:
        mutate(roles)
    # per-run speeds: some roles (and the pipe / TMA) run far ahead of others,
    # which is where ordering bugs show up
    speed = {r: rng.choice([0.05, 1.0, 20.0]) for r in list(roles) + ["pipe", "tma"]}
    pc = {r: 0 for r in roles}
    pipe = []            # in-order tensor pipe: ("mma", tag, n) / ("commit", bar)
    tma = []             # in-flight loads (complete in any order)
    done_mma = set()     # (tag, n) finished on the tensor pipe
    issued = set()
    did = {}             # (tag, n) -> number of roles that finished it
    G_written = {}       # slot -> chunk
    G_readers = {}       # chunk -> readers done
    tma_done = {}
    D_written = {}       # per-channel mode: decay ring slot -> chunk
    D_readers = {}       # chunk -> state-update warps that read its decay

    def finished(tag, n, count):
        return did.get((tag, n), 0) >= count

    def check_issue_kda(tag, n):
        if tag in ("mma3", "mma4", "mma5", "mma6") and not tma_done.get(n):
            raise Hazard(f"{tag} of {n} before the stage of chunk {n} landed")
        if tag == "mma3" and n >= 2 and not (finished("Vp", n - 2, 4) and finished("o", n - 2, 4)):
            raise Hazard(f"D_U[{n % 2}] overwritten by chunk {n} while chunk {n - 2} uses it")
        if tag == "mma4" and n >= 1 and not finished("h", n - 1, 8):
            raise Hazard(f"MMA 4 of {n} before h_{n} is written")
        if tag == "mma5":
            if not finished("Vp", n, 4):
                raise Hazard(f"MMA 5 of {n} before V'({n})")
            if n >= 1 and not finished("h", n - 1, 8):
                raise Hazard(f"D_H of {n} overwritten before chunk {n - 1} read it")
        if tag == "mma6":
            if not finished("Vp", n, 4):
                raise Hazard(f"MMA 6 of {n} before V'({n})")
            if n >= 1 and not finished("o", n - 1, 4):
                raise Hazard(f"D_PV of {n} overwritten before chunk {n - 1} read it")

    def check_do_kda(tag, n):
        if tag == "Vp" and n >= 1 and not {("mma5", n - 1), ("mma6", n - 1)} <= done_mma:
            raise Hazard(f"V'({n}) overwrites vp while MMA 5 / 6 of {n - 1} may read it")
        if tag == "h":
            if not {("mma4", n), ("mma5", n)} <= done_mma:
                raise Hazard(f"h_{n + 1} written while MMA 4 / 5 of {n} may read h_{n}")
            if D_written.get(n % 3) != n:
                raise Hazard(f"decay of chunk {n} read from slot {n % 3} before it was written")
            D_readers[n] = D_readers.get(n, 0) + 1
        if tag == "D":
            if not tma_done.get(n):
                raise Hazard(f"decay of chunk {n} copied before its stage landed")
            old = D_written.get(n % 3)
            if old is not None and D_readers.get(old, 0) < 8:
                raise Hazard(f"decay of {n} overwrites slot {n % 3} still read for chunk {old}")
            D_written[n % 3] = n

    def check_issue(tag, n):
        if kda:
            return check_issue_kda(tag, n)
        # TMEM / smem reuse before the previous user is done
        if tag == "mma1":
            if n >= 1 and not finished("P", n - 1, 4):
                raise Hazard(f"D_S overwritten by chunk {n} before P({n - 1}) read it")
            if not finished("W", n, 2):
                raise Hazard(f"MMA 1 of {n} before [W; Q]({n}) is in TMEM")
        if tag == "mma2" and n >= 1 and not finished("W", n - 1, 2):
            raise Hazard(f"D_W overwritten by chunk {n} before W({n - 1}) was read")
        if tag == "mma3" and n >= 2 and not (finished("Vp", n - 2, 4) and finished("o", n - 2, 4)):
            raise Hazard(f"D_U[{n % 2}] overwritten by chunk {n} while chunk {n - 2} uses it")
        if tag == "mma4":
            if not finished("W", n, 2):
                raise Hazard(f"MMA 4 of {n} before [W; Q]({n}) is in TMEM")
            if n >= 1 and not finished("h", n - 1, 8):
                raise Hazard(f"MMA 4 of {n} before h_{n} is written")
        if tag == "mma5":
            if not finished("Vpd", n, 4):
                raise Hazard(f"MMA 5 of {n} before V'({n})")
            if n >= 1 and not finished("h", n - 1, 8):
                raise Hazard(f"D_H of {n} overwritten before chunk {n - 1} read it")
        if tag == "mma6":
            if not (finished("Vp", n, 4) and finished("P", n, 4)):
                raise Hazard(f"MMA 6 of {n} before V'({n}) / P({n})")
            if n >= 1 and not finished("o", n - 1, 4):
                raise Hazard(f"D_PV of {n} overwritten before chunk {n - 1} read it")

    def check_do(tag, n):
        if kda:
            return check_do_kda(tag, n)
        if tag == "Vpd" and n >= 1 and ("mma5", n - 1) not in done_mma:
            raise Hazard(f"V'({n}) overwrites vpd while MMA 5 of {n - 1} may read it")
        if tag == "Vp" and n >= 1 and ("mma6", n - 1) not in done_mma:
            raise Hazard(f"V'({n}) overwrites vp while MMA 6 of {n - 1} may read it")
        if tag == "h" and not {("mma4", n), ("mma5", n)} <= done_mma:
            raise Hazard(f"h_{n + 1} written while MMA 4 of {n} may read h_{n}")
        if tag == "W" and n >= 2 and not {("mma4", n - 2), ("mma1", n - 2)} <= done_mma:
            raise Hazard(f"W({n}) overwrites the W slot while chunk {n - 2} may read it")
        if tag == "P" and n >= 2 and ("mma6", n - 2) not in done_mma:
            raise Hazard(f"P({n}) overwrites the P slot of chunk {n - 2} in use")
        if tag == "P" and ("mma1", n) not in done_mma:
            raise Hazard(f"P({n}) read before Q K^T of {n} finished")
        if tag == "G":
            old = G_written.get(n % 3)
            if old is not None and G_readers.get(old, 0) < 4 + 8:
                raise Hazard(f"G({n}) overwrites slot {n % 3} still read for chunk {old}")
            G_written[n % 3] = n
        if tag == "readG":
            if G_written.get(n % 3) != n:
                raise Hazard(f"G({n}) read before it was written")
            G_readers[n] = G_readers.get(n, 0) + 1

    def enabled():
        out = []
        for r, seq in roles.items():
            if pc[r] >= len(seq):
                continue
            st = seq[pc[r]]
            if st[0] == "wait":
                bar = bars[st[1]]
                k = st[2]
                if bar.phase >= k + 2:
                    raise Hazard(f"{r} waits for phase {k} of {st[1]} but it is at {bar.phase}")
                if bar.phase == k + 1:
                    out.append(("role", r))
            else:
                out.append(("role", r))
        if pipe:
            out.append(("pipe", None))
        if tma:
            out.append(("tma", None))
        return out

    while True:
        opts = enabled()
        if not opts:
            break
        weights = [speed[r if kind == "role" else kind] for kind, r in opts]
        kind, r = rng.choices(opts, weights=weights)[0]
        if kind == "pipe":
            it = pipe.pop(0)
            if it[0] == "mma":
                done_mma.add((it[1], it[2]))
            else:
                bars[it[1]].arrive()
            continue
        if kind == "tma":
            n = tma.pop(rng.randrange(len(tma)))
            tma_done[n] = True
            bars[("full", n & 1)].arrive()
            continue
        st = roles[r][pc[r]]
        pc[r] += 1
        if st[0] == "arrive":
            bars[st[1]].arrive()
        elif st[0] == "issue":
            check_issue(st[1], st[2])
            issued.add((st[1], st[2]))
            pipe.append(("mma", st[1], st[2]))
        elif st[0] == "commit":
            pipe.append(("commit", st[1]))
        elif st[0] == "tma":
            n = st[1]
            if n >= 2 and not {("mma5", n - 2), ("mma6", n - 2)} <= done_mma:
                raise Hazard(f"stage of chunk {n} reloaded while chunk {n - 2} uses it")
            if kda and n >= 2 and not finished("D", n - 2, 1):
                raise Hazard(f"stage of chunk {n} reloaded before the decay of {n - 2} was copied")
            tma_done.pop(n - 2, None)
            tma.append(n)
        elif st[0] == "do":
            check_do(st[1], st[2])
            did[(st[1], st[2])] = did.get((st[1], st[2]), 0) + 1
    stuck = {r: roles[r][pc[r]] for r in roles if pc[r] < len(roles[r])}
    assert not stuck, f"deadlock: {stuck}"
    assert ("mma6", N - 1) in done_mma


@pytest.mark.parametrize("N", [1, 2, 3, 4, 7, 12])
def test_chain_protocol_random_interleavings(N):
    for seed in range(300):
        run(N, seed)


@pytest.mark.parametrize("N", [1, 2, 3, 4, 7, 12])
def test_chain_protocol_per_channel_mode(N):
    """The per-channel-gate mode's own issue order and roles: no deadlock,
    no skipped phase, no stage, decay-ring, V' or accumulator reuse hazard."""
    for seed in range(300):
        run(N, seed, kda=True)


def test_model_catches_a_decay_published_before_it_is_copied():
    """Planted in the model, not the kernel: warp 2 raising the ring's ready
    barrier before copying the chunk's decay must be reported."""
    def swap(roles):
        seq = roles["p2"]
        for i in range(len(seq) - 1):
            if seq[i][0] == "do" and seq[i][1] == "D":
                seq[i], seq[i + 1] = seq[i + 1], seq[i]

    with pytest.raises(AssertionError, match="decay"):
        for seed in range(300):
            run(3, seed, kda=True, mutate=swap)


def test_model_catches_a_skipped_phase():
    """The model must flag the ordering bug it exists to catch: QK^T of the
    next chunk completing twice on one barrier before a P warp waited."""
    bars = {"x": Bar(1)}
    bars["x"].arrive()
    bars["x"].arrive()
    assert bars["x"].phase == 2  # a waiter for phase 0 would now hang
