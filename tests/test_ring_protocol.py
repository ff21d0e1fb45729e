"""Host-side model of the decode kernel's weight ring, run under random
interleavings (CPU only).

The ring is a circle of shared-memory stages. One producer lane copies chunk
i into stage i % n after stage i % n's release barrier ("empty") completed
its phase for chunk i - n; the copy completes the stage's "full" barrier.
Consumer warps wait on "full" with a parity test and arrive on "empty" when
done. An mbarrier parity test only tells a phase from the one before it:
``try_wait.parity(P)`` is true when the barrier's current (incomplete) phase
has the other parity, i.e. when it reads the phase with parity P as the
completed predecessor.

Three consumer protocols are modelled:

* ``owner``: chunk i is consumed by warp i % 11 alone; the other warps skip
  it without waiting (the first persistent decode kernel's GEMV phases), with
  a CTA barrier between phases and K/V chunks consumed by every warp;
* ``owner_fixed``: the same, but a warp first waits until chunk i - n has
  been released before testing chunk i's full barrier. That test has the
  same flaw one level down: a warp 2n chunks ahead reads chunk i - 2n's
  pending release as chunk i - n's, so it only narrows the window;
* ``all_warps``: every warp waits on every chunk in order (a K/V page pair
  two at a time) and arrives on its release barrier, whose arrival count is
  the number of warps (the cooperative kernel's chunks);
* ``owner_all``: every chunk, weight rows and K/V alike, is consumed and
  released by warp i % 11 alone, which first tests that chunk i - n was
  released, then chunk i's full barrier; CTA barriers around each attention
  item (the row-split kernel, which refuses rings of fewer stages than
  consumer warps: a warp's owned chunks are then at most a ring apart).

A violation is a warp reading a stage that does not hold its chunk yet
(stale bytes, or a copy into it still in flight); a deadlock is a state in
which nothing can move.
"""

import random

import pytest

WARPS = 11


class MBarrier:
    def __init__(self, count):
        self.count = count
        self.pending = count
        self.tx = 0
        self.phase = 0

    def _step(self):
        if self.pending == 0 and self.tx == 0:
            self.phase += 1
            self.pending = self.count

    def arrive(self):
        self.pending -= 1
        self._step()

    def arrive_expect_tx(self, nbytes):
        self.tx += nbytes
        self.pending -= 1
        self._step()

    def complete_tx(self, nbytes):
        self.tx -= nbytes
        self._step()

    def try_wait(self, parity):
        return (self.phase & 1) != parity


def chunk_plan(batch, layers=2):
    """Chunk kinds in stream order, with phase breaks: per layer QKV rows,
    K/V page pairs (more with a larger batch), O rows, gate/up, down."""
    plan = []
    for _ in range(layers):
        plan.append(("rows", 4))
        plan.append(("kv", 2 * batch))
        plan.append(("rows", 2))
        plan.append(("rows", 6))
        plan.append(("rows", 4))
    plan.append(("rows", 40))  # LM head
    return plan


def warp_programs(plan, protocol):
    """Per warp, the list of (op, chunk) steps; ('bar', k) is CTA barrier k."""
    progs = [[] for _ in range(WARPS)]
    i = 0
    nbar = 0
    for kind, count in plan:
        for w in range(WARPS):
            progs[w].append(("bar", nbar))
        nbar += 1
        if kind == "rows":
            for c in range(count):
                for w in range(WARPS):
                    if protocol == "all_warps":
                        progs[w] += [("wait", i + c), ("release", i + c)]
                    elif (i + c) % WARPS == w:
                        progs[w] += [("wait", i + c), ("release", i + c)]
                    else:
                        progs[w].append(("skip", i + c))
            i += count
        elif protocol == "owner_all":  # K/V chunks: one owner warp each
            for c in range(count):
                for w in range(WARPS):
                    if (i + c) % WARPS == w:
                        progs[w] += [("wait", i + c), ("release", i + c)]
                    else:
                        progs[w].append(("skip", i + c))
            for w in range(WARPS):
                progs[w].append(("bar", nbar))
            nbar += 1
            i += count
        else:  # K/V pairs: every warp reads both chunks of a pair
            for c in range(0, count, 2):
                for w in range(WARPS):
                    if protocol == "all_warps":
                        progs[w] += [("wait", i + c), ("wait", i + c + 1),
                                     ("release", i + c), ("release", i + c + 1)]
                    else:
                        progs[w] += [("wait", i + c), ("wait", i + c + 1), ("bar", nbar),
                                     ("kvrelease", i + c), ("kvrelease", i + c + 1)]
                nbar += 1
            i += count
    return progs, i, nbar


def simulate(n_stages, batch, protocol, seed):
    """Returns 'ok', 'violation' or 'deadlock' for one random interleaving."""
    rng = random.Random(seed)
    plan = chunk_plan(batch)
    progs, total, nbar = warp_programs(plan, protocol)
    empty_count = WARPS if protocol == "all_warps" else 1
    full = [MBarrier(1) for _ in range(n_stages)]
    empty = [MBarrier(empty_count) for _ in range(n_stages)]
    content = [None] * n_stages   # chunk whose bytes the stage holds
    inflight = [False] * n_stages
    copies = []                   # copies issued, not yet complete: (stage, chunk)
    prod_i = 0
    pc = [0] * WARPS
    at_bar = {}                   # barrier id -> warps arrived

    def warp_step(w, execute):
        if pc[w] >= len(progs[w]):
            return False
        op, x = progs[w][pc[w]]
        if op == "bar":
            arrived = at_bar.setdefault(x, set())
            if w not in arrived:
                if execute:
                    arrived.add(w)
                return True
            if len(arrived) < WARPS:
                return False
            if execute:
                pc[w] += 1
            return True
        if op == "skip":
            if execute:
                pc[w] += 1
            return True
        s = x % n_stages
        par = (x // n_stages) & 1
        if op == "wait":
            ready = full[s].try_wait(par)
            if protocol in ("owner_fixed", "owner_all"):
                ready = ready and empty[s].try_wait(par ^ 1)
            if not ready:
                return False
            if execute:
                if content[s] != x or inflight[s]:
                    raise AssertionError("violation")
                pc[w] += 1
            return True
        if op == "release":
            if execute:
                empty[s].arrive()
                pc[w] += 1
            return True
        if op == "kvrelease":  # one arrival per K/V chunk, by warp 0
            if execute:
                if w == 0:
                    empty[s].arrive()
                pc[w] += 1
            return True
        raise ValueError(op)

    while True:
        moves = []
        if prod_i < total:
            s = prod_i % n_stages
            if empty[s].try_wait(((prod_i // n_stages) & 1) ^ 1):
                moves.append(("prod",))
        for k in range(len(copies)):
            moves.append(("copy", k))
        for w in range(WARPS):
            if warp_step(w, False):
                moves.append(("warp", w))
        if not moves:
            done = prod_i == total and not copies and all(pc[w] == len(progs[w])
                                                          for w in range(WARPS))
            return "ok" if done else "deadlock"
        mv = rng.choice(moves)
        if mv[0] == "prod":
            s = prod_i % n_stages
            full[s].arrive_expect_tx(1)
            inflight[s] = True
            copies.append((s, prod_i))
            prod_i += 1
        elif mv[0] == "copy":
            s, chunk = copies.pop(mv[1])
            content[s] = chunk
            inflight[s] = False
            full[s].complete_tx(1)
        else:
            try:
                warp_step(mv[1], True)
            except AssertionError:
                return "violation"


def outcomes(n_stages, batch, protocol, runs):
    return {simulate(n_stages, batch, protocol, seed) for seed in range(runs)}


def test_mbarrier_model_parity_semantics():
    b = MBarrier(1)
    assert b.try_wait(1) and not b.try_wait(0)   # fresh: the "previous" phase reads complete
    b.arrive_expect_tx(4)
    assert not b.try_wait(0)
    b.complete_tx(4)
    assert b.try_wait(0) and not b.try_wait(1)   # phase 0 done, phase 1 pending


@pytest.mark.parametrize("n_stages", [4, 8])
def test_owner_only_waits_misread_with_fewer_stages_than_warps(n_stages):
    """The cause of the old stalls: a warp that skips chunks it does not own
    reaches chunk i + n while chunk i (same stage) is still pending; the
    pending phase has the other parity and reads as complete."""
    assert "violation" in outcomes(n_stages, 1, "owner", 60)


def test_owner_only_waits_are_safe_with_a_stage_per_warp():
    assert outcomes(11, 1, "owner", 20) == {"ok"}


@pytest.mark.parametrize("n_stages", [2, 3, 4])
def test_waiting_for_the_previous_release_is_not_enough(n_stages):
    assert "violation" in outcomes(n_stages, 2, "owner_fixed", 60)


@pytest.mark.parametrize("batch", [1, 2, 3, 4])
@pytest.mark.parametrize("n_stages", list(range(2, 17)))
def test_all_warps_protocol_never_misreads_or_deadlocks(n_stages, batch):
    assert outcomes(n_stages, batch, "all_warps", 6) == {"ok"}


@pytest.mark.parametrize("batch", [1, 2, 3, 4])
@pytest.mark.parametrize("n_stages", list(range(11, 17)))
def test_row_split_owner_protocol_never_misreads_or_deadlocks(n_stages, batch):
    """The row-split kernel's protocol at the ring sizes it accepts."""
    assert outcomes(n_stages, batch, "owner_all", 6) == {"ok"}


@pytest.mark.parametrize("n_stages", [4, 8])
def test_row_split_owner_protocol_needs_a_stage_per_warp(n_stages):
    """Why the row-split kernel refuses smaller rings: with fewer stages than
    consumer warps a warp can be two rings ahead of a pending chunk, and the
    release test then reads the wrong phase."""
    assert "violation" in outcomes(n_stages, 2, "owner_all", 60)
