"""Host-side checks of the factorization's task graph (no GPU).

The factorization kernel behind gptq_prepare_hinv hands out 128 x 128 tile products in the
order gptq_chol_schedule returns, one CTA forming the diagonal blocks (leaves) in the order
j = T-1 .. 0 and, after each leaf j >= 1, the two products the next leaf needs (the panel
tile PANEL(j, j-1) and the diagonal update UPDATE(j, j-1, j-1)).  These tests take that
order from the library and check, on the host:
  * every product appears exactly once;
  * every product's inputs are produced earlier (the leaf of step j before step j's
    products), which makes the dynamic ticket order deadlock-free on any number of CTAs;
  * executing the list with the block formulas in fp64 (small tiles) gives the upper Cholesky
    factor of Hd^-1;
  * an event simulation with many workers and random task times always finishes.
"""
import heapq
import random

import numpy as np
import pytest

from post_weight_quantization_14_b200 import gptq

PANEL, UPDATE, FIN, SUPD, DIAG = 0, 1, 2, 3, 4


def step_of(t):
    typ, a, b, c = t
    return {PANEL: b, UPDATE: c, FIN: a, SUPD: c, DIAG: a}[typ]


def expected_tasks(T):
    """Every product of the factorization except those the leaf CTA forms itself."""
    s = set()
    for j in range(T):
        for i in range(j):
            if i != j - 1:
                s.add((PANEL, i, j, 0))
            for k in range(i, j):
                if not (i == k == j - 1):
                    s.add((UPDATE, i, k, j))
    for i in range(T):
        s.add((DIAG, i, 0, 0))
        for m in range(i + 1, T):
            s.add((FIN, i, m, 0))
            for k in range(i + 1, m + 1):
                s.add((SUPD, i, m, k))
    return s


def global_order(T):
    """The product list with LEAF(j) inserted before the first product of step j."""
    tasks = gptq.gptq_chol_schedule(T)
    seq, cur = [], None
    for t in tasks:
        j = step_of(t)
        if j != cur:
            assert cur is None or j < cur, "steps must run T-1 .. 0"
            for jj in range(T - 1 if cur is None else cur - 1, j - 1, -1):
                seq.append(("LEAF", jj))
            cur = j
        seq.append(t)
    for jj in range((T - 1 if cur is None else cur - 1), -1, -1):
        seq.append(("LEAF", jj))
    return tasks, seq


class Counters:
    """The kernel's dependency counters, advanced as tasks complete."""

    def __init__(self, T):
        self.T = T
        self.a_cnt = np.zeros((T, T), int)
        self.rs_done = np.zeros((T, T), int)
        self.s_cnt = np.zeros((T, T), int)
        self.u_done = np.zeros((T, T), int)
        self.leaf_done = np.zeros(T, int)
        self.diag_done = np.zeros(T, int)

    def ready(self, t):
        T = self.T
        if t[0] == "LEAF":   # the leaf of j, then (j >= 1) the panel tile (j-1, j) and A_{j-1,j-1}'s update
            j = t[1]
            ok = self.a_cnt[j, j] >= T - 1 - j
            if j >= 1:
                ok = ok and self.a_cnt[j - 1, j] >= T - 1 - j and self.a_cnt[j - 1, j - 1] >= T - 1 - j
            return ok
        typ, a, b, c = t
        if typ == PANEL:
            return self.leaf_done[b] >= 1 and self.a_cnt[a, b] >= T - 1 - b
        if typ == UPDATE:
            return self.rs_done[a, c] >= 1 and self.rs_done[b, c] >= 1 and self.a_cnt[a, b] >= T - 1 - c
        if typ == FIN:
            return self.leaf_done[a] >= 1 and self.s_cnt[a, b] >= b - a
        if typ == DIAG:
            return self.leaf_done[a] >= 1
        up = self.diag_done[b] >= 1 if c == b else self.u_done[c, b] >= 1
        return self.rs_done[a, c] >= 1 and up and self.s_cnt[a, b] >= b - c

    def exact(self, t):
        """A read-modify-write task must see exactly the earlier contributions."""
        T = self.T
        if t[0] == "LEAF":
            j = t[1]
            return self.a_cnt[j, j] == T - 1 - j and (j == 0 or self.a_cnt[j - 1, j - 1] == T - 1 - j)
        typ, a, b, c = t
        if typ == UPDATE:
            return self.a_cnt[a, b] == T - 1 - c
        if typ == SUPD:
            return self.s_cnt[a, b] == b - c
        return True

    def done(self, t):
        if t[0] == "LEAF":
            j = t[1]
            self.leaf_done[j] += 1
            if j >= 1:
                self.rs_done[j - 1, j] += 1
                self.a_cnt[j - 1, j - 1] += 1
            return
        typ, a, b, c = t
        if typ == PANEL:
            self.rs_done[a, b] += 1
        elif typ == UPDATE:
            self.a_cnt[a, b] += 1
        elif typ == FIN:
            self.u_done[a, b] += 1
        elif typ == DIAG:
            self.diag_done[a] += 1
        else:
            self.s_cnt[a, b] += 1


@pytest.mark.parametrize("T", [1, 2, 3, 4, 7, 32, 86])
def test_each_product_once(T):
    tasks = gptq.gptq_chol_schedule(T)
    assert len(tasks) == len(set(tasks))
    assert set(tasks) == expected_tasks(T)


@pytest.mark.parametrize("T", [1, 2, 3, 5, 9, 32])
def test_inputs_come_first(T):
    _, seq = global_order(T)
    ctr = Counters(T)
    for t in seq:
        assert ctr.ready(t) and ctr.exact(t), f"{t} runs before its inputs"
        ctr.done(t)
    assert ctr.leaf_done.sum() == T


def test_schedule_rejects_bad_T():
    with pytest.raises(gptq.GPTQError):
        gptq.gptq_chol_schedule(0)


def _reverse_chol_upper(A):
    """R upper with A = R R^T (factor from the bottom-right corner)."""
    J = np.eye(A.shape[0])[::-1]
    L = np.linalg.cholesky(J @ A @ J)
    return J @ L @ J


@pytest.mark.parametrize("T,b", [(1, 4), (2, 3), (5, 4), (8, 2)])
def test_block_formulas_give_hinv_factor(T, b):
    """Run the list in order with the block formulas (tile size b) in fp64."""
    rng = np.random.default_rng(T * 10 + b)
    n = T * b
    X = rng.standard_normal((3 * n, n))
    A0 = X.T @ X + 0.5 * np.eye(n)
    A = A0.copy()
    R = np.zeros((n, n))
    X_inv = {}
    S = np.zeros((n, n))
    U = np.zeros((n, n))
    blk = lambda i: slice(i * b, (i + 1) * b)
    _, seq = global_order(T)
    for t in seq:
        if t[0] == "LEAF":
            j = t[1]
            Rjj = _reverse_chol_upper(A[blk(j), blk(j)])
            R[blk(j), blk(j)] = Rjj
            X_inv[j] = np.linalg.inv(Rjj)
            U[blk(j), blk(j)] = X_inv[j]
            if j >= 1:   # the leaf CTA's two products for the next leaf
                R[blk(j - 1), blk(j)] = A[blk(j - 1), blk(j)] @ X_inv[j].T
                A[blk(j - 1), blk(j - 1)] -= R[blk(j - 1), blk(j)] @ R[blk(j - 1), blk(j)].T
            continue
        typ, a, bb, c = t
        if typ == PANEL:
            i, j = a, bb
            R[blk(i), blk(j)] = A[blk(i), blk(j)] @ X_inv[j].T
        elif typ == UPDATE:
            i, k, j = a, bb, c
            A[blk(i), blk(k)] -= R[blk(i), blk(j)] @ R[blk(k), blk(j)].T
        elif typ == FIN:
            i, m = a, bb
            U[blk(i), blk(m)] = -X_inv[i] @ S[blk(i), blk(m)]
        elif typ == DIAG:
            pass   # a copy of U_jj, already in place
        else:
            i, m, k = a, bb, c
            S[blk(i), blk(m)] += R[blk(i), blk(k)] @ U[blk(k), blk(m)]
    assert np.allclose(np.triu(R) @ np.triu(R).T, A0, rtol=0, atol=1e-9 * np.abs(A0).max())
    U_ref = np.linalg.cholesky(np.linalg.inv(A0)).T   # U^T U = A0^-1, U upper
    assert np.allclose(U, U_ref, rtol=0, atol=1e-9 * np.abs(U_ref).max())


@pytest.mark.parametrize("T,workers,seed", [(6, 3, 0), (12, 40, 1), (20, 147, 2), (9, 1, 3)])
def test_dynamic_tickets_finish(T, workers, seed):
    """Workers take the next ticket when free and wait for its inputs; one worker runs the
    leaves.  With random task times the simulation must always drain."""
    rnd = random.Random(seed)
    tasks = gptq.gptq_chol_schedule(T)
    ctr = Counters(T)
    next_ticket, next_leaf = 0, T - 1
    waiting = []          # (worker, task) holding a ticket whose inputs are not ready
    running = []          # heap of (finish_time, seq, task)
    now, seq_no = 0.0, 0
    free = workers
    leaf_busy = False
    done = 0
    while done < len(tasks) + T:
        progressed = True
        while progressed:
            progressed = False
            if not leaf_busy and next_leaf >= 0 and ctr.ready(("LEAF", next_leaf)):
                heapq.heappush(running, (now + rnd.uniform(5, 40), seq_no, ("LEAF", next_leaf)))
                seq_no += 1
                next_leaf -= 1
                leaf_busy = True
                progressed = True
            while free > 0 and next_ticket < len(tasks):
                waiting.append(tasks[next_ticket])
                next_ticket += 1
                free -= 1
                progressed = True
            for t in list(waiting):
                if ctr.ready(t):
                    assert ctr.exact(t)
                    waiting.remove(t)
                    heapq.heappush(running, (now + rnd.uniform(1, 6), seq_no, t))
                    seq_no += 1
                    progressed = True
        assert running, f"stalled with {len(waiting)} waiting tickets"
        now, _, t = heapq.heappop(running)
        ctr.done(t)
        done += 1
        if t[0] == "LEAF":
            leaf_busy = False
        else:
            free += 1
    assert next_ticket == len(tasks) and next_leaf == -1
