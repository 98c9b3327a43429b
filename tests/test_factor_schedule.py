"""Host-side check of the diagonal-block kernel's phase schedule (no GPU).

The kernel that factors a 128 x 128 diagonal block of the blocked Cholesky (GPTQ deep-dive,
hncyxsy.com/news/243429, §2.4: the Cholesky reformulation; §3.1 step 2) splits it into four
32-column sub-panels and runs, per sub-panel k, three phases: A(k) the factor warp beside the
block products that are ready, B(k) the panel solve and the 32 x 32 inverse, C(k) the next
block column's update and the inverse blocks that become final. The block products of phases
A and C come from a table in csrc/factor.cu (`c_tasks`, `c_task_off`). This test reads that
table from the source and replays the schedule on the block level: every task's inputs must be
final when its phase runs, no block may be written twice in one phase or read by another task
while it is written, every trailing update and every inverse term must be applied exactly once,
and at the end every block of L and of L^-1 must be final.
"""
import os
import re

import pytest

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "post_weight_quantization_24_b200", "csrc", "factor.cu")
NSB = 4


def parse_schedule():
    src = open(SRC).read()
    body = re.search(r"c_tasks\[(\d+)\]\s*=\s*\{(.*?)\};", src, re.S)
    assert body, "task table not found"
    tasks = [(k, int(i), int(j), int(m)) for k, i, j, m in
             re.findall(r"pt::T\(pt::(U|W|F),\s*(\d),\s*(\d),\s*(\d)\)", body.group(2))]
    assert len(tasks) == int(body.group(1))
    off = re.search(r"c_task_off\[(\d+)\]\s*=\s*\{([^}]*)\}", src)
    offsets = [int(x) for x in off.group(2).split(",")]
    assert len(offsets) == int(off.group(1)) == 2 * NSB + 1
    return tasks, offsets


def test_table_parses():
    tasks, off = parse_schedule()
    assert off[0] == 0 and off[-1] == len(tasks)
    assert all(a <= b for a, b in zip(off, off[1:]))


def test_schedule_replay():
    tasks, off = parse_schedule()
    applied = {(i, j): set() for i in range(NSB) for j in range(i + 1)}   # panels applied to S_ij
    l_final = set()                   # blocks (i, m) of L that are final
    x_final = set()                   # blocks (i, j) of L^-1 that are final
    w_terms = {(i, j): set() for i in range(NSB) for j in range(i)}      # terms m in W_ij
    lt_panel = None                   # the sub-panel whose L_rk is in LT

    def phase(p):
        return tasks[off[p]:off[p + 1]]

    def io(t):
        kind, i, j, m = t
        if kind == "U":
            return ("S", i, j), [("S", i, m), ("S", j, m)]
        if kind == "W":
            return ("X", i, j), [("S", i, m), ("X", m, j)]
        return ("X", i, j), [("X", i, i), ("X", i, j)]     # F overwrites what it read

    def check_disjoint(ts, busy=()):
        writes = [io(t)[0] for t in ts]
        assert len(writes) == len(set(writes)), f"a block is written twice in one phase: {ts}"
        for t in ts:
            w, rs = io(t)
            others = set(writes) - {w}
            assert not (set(rs) & others), f"{t} reads a block another task writes: {ts}"
            assert w not in busy and not (set(rs) & set(busy)), f"{t} touches {busy}"

    def run(ts):
        nonlocal lt_panel
        for kind, i, j, m in ts:
            if kind == "U":
                assert i >= j > m and lt_panel == m, (kind, i, j, m, lt_panel)
                assert (i, m) in l_final and (j, m) in l_final
                assert m not in applied[(i, j)]
                applied[(i, j)].add(m)
            elif kind == "W":
                assert i > m >= j and (i, m) in l_final and (m, j) in x_final
                assert m not in w_terms[(i, j)]
                w_terms[(i, j)].add(m)
            else:
                assert i > j and (i, i) in x_final and (i, j) not in x_final
                assert w_terms[(i, j)] == set(range(j, i)), (i, j, w_terms[(i, j)])
                x_final.add((i, j))

    for k in range(NSB):
        # A(k): the factor warp on S_kk beside the table's tasks
        a = phase(2 * k)
        check_disjoint(a, busy=[("S", k, k)])   # the factor warp's block
        assert applied[(k, k)] == set(range(k)), f"S_{k}{k} incomplete at its factorisation"
        run(a)
        l_final.add((k, k))
        # B(k): the panel solve (rows below, needs every earlier panel applied) and I_kk
        for i in range(k + 1, NSB):
            assert applied[(i, k)] == set(range(k)), f"S_{i}{k} incomplete at the solve"
            l_final.add((i, k))
        lt_panel = k
        x_final.add((k, k))
        # C(k): the next block column and the inverse blocks I_kk completes
        c = phase(2 * k + 1)
        assert len(c) <= 3, "phase C runs at most three tasks of four warps"
        check_disjoint(c)
        run(c)
        if k + 1 < NSB:
            assert applied[(k + 1, k + 1)] == set(range(k + 1)), "next diagonal block not ready"

    # everything applied and final
    for (i, j), ms in applied.items():
        assert ms == set(range(j)), f"S_{i}{j}: panels {sorted(ms)} applied"
    assert l_final == {(i, j) for i in range(NSB) for j in range(i + 1)}
    assert x_final == {(i, j) for i in range(NSB) for j in range(i + 1)}
    for (i, j), ms in w_terms.items():
        assert ms == set(range(j, i))


def test_phase_a_has_no_finalisations():
    # phase A's tasks run on single warps with no barrier among them: an F task (which needs
    # its warps to meet before overwriting W_ij) may only appear in phase C
    tasks, off = parse_schedule()
    for k in range(NSB):
        assert all(t[0] != "F" for t in tasks[off[2 * k]:off[2 * k + 1]])


if __name__ == "__main__":
    pytest.main([__file__, "-q"])
