"""A host-side model of the fused GLA kernel's cross-CTA protocol, with
threads as CTAs (CPU only; no GPU is faulted or hung).

The protocol the model follows (csrc/gla_fused.cu):
- each CTA draws a ticket from a counter in the workspace header;
  ticket -> (plane, segment);
- every segment but the last of its plane publishes its aggregate and raises
  its flag (one release store);
- every segment but the first waits, bounded, for the flags of all earlier
  segments of its plane, then folds them;
- a ticket past the last segment latches the workspace-state error and does
  no work;
- the last CTA to finish clears the flags and counters.
A limited number of CTAs are resident at once, started in any order.

What the tests check:
- under random residency and timing every run completes with no timeout and
  leaves the header clean, because a segment only waits for tickets drawn
  before it;
- a dirty ticket counter and a dropped flag both end in bounded waits that
  give up, the right error latched and a clean header;
- a control where segments are assigned by launch index instead of ticket
  does starve: a resident CTA waits for a segment whose CTA cannot start.
"""
import random
import threading
import time

import pytest


class Header:
    def __init__(self, n_slots):
        self.lock = threading.Lock()
        self.ctr = [0, 0]
        self.flags = [threading.Event() for _ in range(n_slots)]


class Errors:
    def __init__(self):
        self.lock = threading.Lock()
        self.first = None
        self.all = []

    def latch(self, code):
        with self.lock:
            self.all.append(code)
            if self.first is None:
                self.first = code


def run_launch(BH, P, resident, seed, *, dirty_ticket=0, drop_flag_of=None, by_launch_index=False,
               wait_limit=2.0):
    """One launch of BH * P CTAs, at most `resident` at a time, started in a
    random order.  Returns (errors, header, wall seconds)."""
    rng = random.Random(seed)
    G = BH * P
    hdr = Header(G)
    hdr.ctr[0] = dirty_ticket
    err = Errors()
    sem = threading.Semaphore(resident)
    delays = [(rng.uniform(0, 2e-3), rng.uniform(0, 2e-3)) for _ in range(G)]

    def cta(block):
        with sem:
            if by_launch_index:
                ticket = block
            else:
                with hdr.lock:
                    ticket = hdr.ctr[0]
                    hdr.ctr[0] += 1
            if ticket >= G:
                err.latch("workspace_state")
            else:
                bh, seg = divmod(ticket, P)
                pre, main = delays[block]
                time.sleep(pre)  # the pre-pass
                if seg < P - 1 and ticket != drop_flag_of:
                    hdr.flags[bh * P + seg].set()  # publish the aggregate
                ok = True
                for j in range(seg):  # fold: bounded waits for every earlier segment
                    if not hdr.flags[bh * P + j].wait(timeout=wait_limit):
                        ok = False
                        break
                if not ok:
                    err.latch("timeout")
                time.sleep(main)  # the main pass
            with hdr.lock:
                prev = hdr.ctr[1]
                hdr.ctr[1] += 1
                last = prev == G - 1
            if last:  # leave the header ready for the next call
                for f in hdr.flags:
                    f.clear()
                with hdr.lock:
                    hdr.ctr[0] = 0
                    hdr.ctr[1] = 0

    order = list(range(G))
    rng.shuffle(order)
    threads = [threading.Thread(target=cta, args=(b,)) for b in order]
    t0 = time.time()
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=60)
    assert not any(t.is_alive() for t in threads), "a modelled CTA never finished"
    return err, hdr, time.time() - t0


def clean(hdr):
    return hdr.ctr == [0, 0] and not any(f.is_set() for f in hdr.flags)


@pytest.mark.parametrize("BH,P,resident", [(1, 5, 1), (2, 4, 2), (3, 6, 4), (6, 13, 8), (4, 3, 12)])
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_ticket_order_always_completes(BH, P, resident, seed):
    err, hdr, _ = run_launch(BH, P, resident, seed, wait_limit=5.0)
    assert err.first is None, err.all
    assert clean(hdr)


def test_dirty_ticket_counter_reports_and_leaves_a_clean_header():
    """As in the GPU test of the same case: ticket 0 is never drawn, so
    segment 0 of plane 0 never publishes; the CTA that draws the ticket past
    the end latches the workspace error first, the later segments of plane 0
    time out, the run ends, and the header is clean."""
    err, hdr, wall = run_launch(2, 4, 8, 3, dirty_ticket=1, wait_limit=0.3)
    assert "workspace_state" in err.all
    assert "timeout" in err.all
    assert clean(hdr)
    assert wall < 10.0


def test_dropped_flag_times_out_and_the_run_ends():
    err, hdr, wall = run_launch(2, 5, 10, 4, drop_flag_of=1, wait_limit=0.3)
    assert err.first == "timeout"
    assert clean(hdr)
    assert wall < 10.0


def test_segments_by_launch_index_can_starve():
    """Control: with one resident CTA and segments assigned by launch index,
    a CTA started out of order waits for an earlier segment whose CTA cannot
    start until it leaves; only the bounded wait ends the run."""
    starved = False
    for seed in range(10):
        err, hdr, _ = run_launch(1, 4, 1, seed, by_launch_index=True, wait_limit=0.1)
        starved = starved or ("timeout" in err.all)
    assert starved


# ------------------------------------------------ the transposed boundary scan
#
# One-wave plans run as a cooperative launch (every CTA resident) and
# exchange boundary states in two rounds (csrc/gla_fused.cu):
# - every segment but the last publishes its aggregate A_s and gate totals g_s
#   and raises flag1;
# - each CTA waits (bounded) for all flag1 of its plane, takes the slice
#   [seg * npairs / P, (seg + 1) * npairs / P) of the state's element pairs,
#   runs S_in(s + 1) = diag(e^{g_s}) S_in(s) + A_s over all segments for that
#   slice, writes that slice of every S_in and raises flag2;
# - every segment but the first waits (bounded) for all flag2 of its plane and
#   reads its S_in, which all CTAs of the plane wrote;
# - the arrival count is checked at the end (a dirty header is reported).
# The model carries real numbers (d_k x d_v = 4 x 4, 8 pairs) and checks every
# S_in against the sequential definition, S_in(s) = sum_{t < s}
# diag(e^{g_{t+1} + ... + g_{s-1}}) A_t.

import numpy as np  # noqa: E402


def run_coop_scan(BH, P, seed, *, resident=None, drop_flag2_of=None, dirty_arrivals=0, wait_limit=2.0,
                  dk=4, dv=4):
    rng = np.random.default_rng(seed)
    prng = random.Random(seed)
    G = BH * P
    npairs = dk * dv // 2
    A = rng.standard_normal((BH, P, dk, dv))
    g = -np.abs(rng.standard_normal((BH, P, dk)))  # log-gate totals, <= 0
    sin = np.full((BH, P, dk * dv), np.nan)
    got = np.full((BH, P, dk * dv), np.nan)
    flag1 = [threading.Event() for _ in range(G)]
    flag2 = [threading.Event() for _ in range(G)]
    arrivals = [dirty_arrivals]
    lock = threading.Lock()
    err = Errors()
    sem = threading.Semaphore(resident if resident is not None else G)
    delays = [prng.uniform(0, 2e-3) for _ in range(G)]

    def cta(block):
        with sem:
            with lock:
                arrival = arrivals[0]
                arrivals[0] += 1
            bh, seg = divmod(block, P)  # every CTA resident: the block index names the segment
            time.sleep(delays[block])  # the pre-pass
            if seg < P - 1:
                flag1[bh * P + seg].set()
            ok = all(flag1[bh * P + j].wait(timeout=wait_limit) for j in range(P - 1))
            if not ok:
                err.latch("timeout")
            else:
                u0, u1 = seg * npairs // P, (seg + 1) * npairs // P
                for u in range(u0, u1):
                    e = np.array([2 * u, 2 * u + 1])
                    i = e // dv  # key dim of each element
                    R = np.zeros(2)
                    for s2 in range(P - 1):
                        R = np.exp(g[bh, s2, i]) * R + A[bh, s2].reshape(-1)[e]
                        sin[bh, s2 + 1, e] = R
            if block != drop_flag2_of and ok:
                flag2[bh * P + seg].set()
            if seg > 0:
                if all(flag2[bh * P + j].wait(timeout=wait_limit) for j in range(P)):
                    got[bh, seg] = sin[bh, seg]
                else:
                    err.latch("timeout")
            if arrival >= G:  # checked at the end, off the critical path
                err.latch("workspace_state")

    threads = [threading.Thread(target=cta, args=(b,)) for b in prng.sample(range(G), G)]
    t0 = time.time()
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=60)
    assert not any(t.is_alive() for t in threads), "a modelled CTA never finished"
    # the definition, segment by segment
    ref = np.zeros((BH, P, dk * dv))
    for bh in range(BH):
        for s in range(1, P):
            acc = np.zeros((dk, dv))
            for t in range(s):
                acc += np.exp(g[bh, t + 1:s].sum(axis=0))[:, None] * A[bh, t]
            ref[bh, s] = acc.reshape(-1)
    return err, got, ref, time.time() - t0


@pytest.mark.parametrize("BH,P", [(1, 2), (6, 24), (48, 3), (12, 12), (2, 33)])
@pytest.mark.parametrize("seed", [0, 1])
def test_coop_scan_gives_every_segment_its_incoming_state(BH, P, seed):
    err, got, ref, _ = run_coop_scan(BH, P, seed, wait_limit=5.0)
    assert err.first is None, err.all
    np.testing.assert_allclose(got[:, 1:], ref[:, 1:], rtol=1e-12, atol=1e-12)


def test_coop_scan_dropped_flag2_times_out_and_ends():
    err, _, _, wall = run_coop_scan(2, 6, 5, drop_flag2_of=3, wait_limit=0.3)
    assert err.first == "timeout"
    assert wall < 10.0


def test_coop_scan_reports_a_dirty_arrival_count():
    err, got, ref, _ = run_coop_scan(1, 4, 6, dirty_arrivals=2, wait_limit=2.0)
    assert "workspace_state" in err.all


def test_coop_scan_needs_every_cta_resident():
    """Control: with fewer resident CTAs than segments of a plane, a CTA waits
    for the flag1 of a segment whose CTA cannot start: only the bounded wait
    ends the run.  This is why the scan runs under a cooperative launch."""
    err, _, _, _ = run_coop_scan(1, 6, 7, resident=3, wait_limit=0.2)
    assert "timeout" in err.all
