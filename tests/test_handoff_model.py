"""Model check of the single-CTA GEMM kernel's K-block hand-off (CPU only).

Three roles share two barrier rings in ``csrc/bsgemm_kernel.cuh``:
- the TMA producer fills stage s and completes ``full[s]``; before refilling it,
  it waits for ``empty[s]``;
- the MMA warp waits for ``full[s]`` and then for TMEM buffer b (``tmem_empty[b]``).
  It issues the K-block's MMAs and commits ``tmem_full[b]`` after the block's last
  stage and ``empty[s]`` after each stage. At g = 64 a stage holds two K-blocks;
  at g = 256 a K-block spans two stages;
- the promotion warps wait for ``tmem_full[b]``, read the partial and arrive on
  ``tmem_empty[b]``.

Every wait is a parity wait: waiting for phase k passes when the barrier's
completed-phase count c has (c & 1) != (k & 1). That answer is only right when
c == k + 1. A barrier one phase behind (c == k - 1) or two ahead (c == k + 2)
gives the same answer, which is aliasing. The model runs the three roles with
these barriers as counters. The MMA completions are asynchronous, in issue
order, and the TMA completions come in any order. Random schedules are run
over random work lists: whole tiles, split-K pieces and stream-K ranges, with
a partial last K-block. The checks:
- no wait passes at a count other than k + 1, and the roles never deadlock;
- no stage is overwritten while MMAs read it or before they have used it;
- no TMEM buffer is rewritten before the promotion has read it;
- no MMA reads a stage before its copy landed, and no promotion reads an
  unfinished partial.
The stage and buffer counts are those the kernel derives from the tile width
and operand layout. Planted protocol mistakes show the model catches each
kind of fault.
"""
import random

import pytest

BK = 128                       # K bytes per stage
BUDGET = 227 * 1024 - 1024 - 512


def stages(bnq: int, q_mn: bool) -> int:
    q_rows = 128 if (q_mn and bnq < 128) else bnq
    return min(8, BUDGET // (BM_BYTES + q_rows * BK))


BM_BYTES = 128 * BK


def bufs(bnq: int) -> int:
    return 2 if bnq >= 256 else 4 if bnq >= 128 else 8


def work_list(rng, gran, K):
    """K-block ranges [kb0, kb1) of a CTA's work items, as the scheduler hands
    them out: whole tiles, split pieces and stream-K ranges (at g = 64 they start
    on even K-blocks, a unit being one 128-deep stage)."""
    Kb = -(-K // gran)
    items = []
    for _ in range(rng.randint(1, 4)):
        kind = rng.choice(("tile", "piece"))
        if kind == "tile" or Kb == 1:
            items.append((0, Kb))
        else:
            a, b = sorted(rng.sample(range(Kb + 1), 2))
            if gran == 64:
                a -= a & 1
                b = b + (b & 1) if b < Kb else Kb
                b = min(b, Kb)
                if a == b:
                    continue
            items.append((a, b))
    return items or [(0, Kb)]


class Bar:
    __slots__ = ("c",)

    def __init__(self):
        self.c = 0

    def passes(self, k):
        return (self.c & 1) != (k & 1)


def simulate(S, B, gran, K, items, rng, mutation=None):
    full = [Bar() for _ in range(S)]
    empty = [Bar() for _ in range(S)]
    tfull = [Bar() for _ in range(B)]
    tempty = [Bar() for _ in range(B)]
    errors = []

    def check(bar, k, what):
        if bar.c != k + 1:
            errors.append(f"{what}: waited for phase {k}, count was {bar.c}")

    nst = -(-K // BK)

    # producer program: the stage slots it fills, in order
    prod = []
    for kb0, kb1 in items:
        if gran >= BK:
            st0, st1 = kb0 * (gran // BK), kb1 * (gran // BK)
        else:
            st0, st1 = kb0 // 2, (kb1 + 1) // 2
        prod += [None] * (min(st1, nst) - st0)

    # MMA program: a list of steps (wait_full, wait_tmem, commit_tmem_full, commit_empty)
    mma = []
    for kb0, kb1 in items:
        for kb in range(kb0, kb1):
            if gran >= BK:
                for j in range(gran // BK):
                    k0 = kb * gran + j * BK
                    if k0 >= K:
                        break
                    last = j == gran // BK - 1 or k0 + BK >= K
                    mma.append((True, j == 0, last, True))
            else:
                k0 = kb * gran
                t0 = kb & 1
                mma.append((t0 == 0, True, True, t0 == 1 or k0 + gran >= K))
    nblocks = sum(kb1 - kb0 for kb0, kb1 in items)

    p_it = 0                       # producer: stage slots filled
    landing = []                   # TMA copies in flight (stage indices)
    m_i = 0                        # MMA: next step
    m_st = 0                       # MMA: stage slots consumed
    m_blk = 0                      # MMA: K-blocks started
    m_sub = 0                      # MMA: 0 = before its waits, 1 = full passed
    inflight = []                  # MMA commits not yet complete, in issue order
    promo = 0
    reading = [0] * S              # MMA groups in flight that read each stage
    stage_done = 0                 # stage slots whose reads are complete
    blocks_done = 0                # K-blocks whose MMAs are complete
    landed = set()                 # stage slots whose copies landed
    # adversarial pacing: some roles run far slower than the others in this run
    slow = {r for r in ("prod", "land", "mma", "m_done", "promo") if rng.random() < 0.3}
    guard = 0
    while promo < nblocks and not errors:
        guard += 1
        if guard > 200000:
            errors.append("no progress")
            break
        acts = []
        if p_it < len(prod):
            k = p_it // S - (0 if mutation == "producer_phase" else 1)
            if k < 0 or empty[p_it % S].passes(k):
                acts.append("prod")
        if landing:
            acts.append("land")
        if m_i < len(mma):
            wf, wt, _, _ = mma[m_i]
            s = m_st % S
            if m_sub == 0 and wf:
                if full[s].passes(m_st // S):
                    acts.append("m_full")
            else:
                b, k = m_blk % B, m_blk // B - (0 if mutation == "tmem_phase" else 1)
                if not wt or k < 0 or mutation == "skip_tmem_wait" or tempty[b].passes(k):
                    acts.append("m_issue")
        if inflight:
            acts.append("m_done")
        b, k = promo % B, promo // B - (1 if mutation == "promo_phase" else 0)
        if k < 0 or tfull[b].passes(k):
            acts.append("promo")
        if not acts:
            errors.append(f"deadlock: producer {p_it}/{len(prod)}, mma {m_i}/{len(mma)}, promotion {promo}")
            break
        role = {"m_full": "mma", "m_issue": "mma"}
        weights = [0.03 if role.get(x, x) in slow else 1.0 for x in acts]
        a = rng.choices(acts, weights)[0]
        if a == "prod":
            if p_it // S - 1 >= 0 and mutation is None:
                check(empty[p_it % S], p_it // S - 1, f"producer slot {p_it}")
            if reading[p_it % S] or stage_done < p_it - S + 1:
                errors.append(f"producer slot {p_it}: stage {p_it % S} overwritten while in use")
            landing.append(p_it)
            p_it += 1
        elif a == "land":
            slot = landing.pop(rng.randrange(len(landing)))
            landed.add(slot)
            full[slot % S].c += 1
        elif a == "m_full":
            check(full[m_st % S], m_st // S, f"mma step {m_i} (full)")
            m_sub = 1
        elif a == "m_issue":
            wf, wt, ctf, cem = mma[m_i]
            if wt and m_blk // B - 1 >= 0 and mutation is None:
                check(tempty[m_blk % B], m_blk // B - 1, f"mma step {m_i} (tmem_empty)")
            if m_st not in landed:
                errors.append(f"mma step {m_i}: stage slot {m_st} read before its copy landed")
            if wt and promo < m_blk - B + 1:
                errors.append(f"mma step {m_i}: buffer {m_blk % B} rewritten before block "
                              f"{m_blk - B} was promoted")
            reading[m_st % S] += 1
            if mutation == "early_release" and cem:
                empty[m_st % S].c += 1
                stage_done += 1
                cem_late = False
            else:
                cem_late = cem
            inflight.append((m_blk % B if ctf else None, m_st % S if cem_late else None, m_st % S))
            if ctf:
                m_blk += 1
            if cem:
                m_st += 1
            m_i += 1
            m_sub = 0
        elif a == "m_done":
            tb, es, rs = inflight.pop(0)
            reading[rs] -= 1
            if tb is not None:
                tfull[tb].c += 1
                blocks_done += 1
            if es is not None:
                empty[es].c += 1
                stage_done += 1
        else:
            if mutation is None:
                check(tfull[promo % B], promo // B, f"promotion block {promo}")
            if blocks_done < promo + 1:
                errors.append(f"promotion block {promo}: read an unfinished partial")
            tempty[promo % B].c += 1
            promo += 1
    if not errors and (m_i != len(mma) or p_it != len(prod)):
        errors.append("roles finished out of step")
    return errors


CONFIGS = [(bnq, q_mn) for bnq in (16, 32, 64, 128, 256) for q_mn in (False, True)]


@pytest.mark.parametrize("gran", [64, 128, 256])
@pytest.mark.parametrize("bnq,q_mn", CONFIGS)
def test_handoff_never_aliases_or_deadlocks(bnq, q_mn, gran):
    S, B = stages(bnq, q_mn), bufs(bnq)
    rng = random.Random(1000 * bnq + 10 * gran + q_mn)
    for _ in range(60):
        K = rng.choice([BK, 2 * BK, 3 * BK, 5 * BK + 16, 7 * BK, 9 * BK + 64, 17 * BK])
        items = work_list(rng, gran, K)
        errors = simulate(S, B, gran, K, items, rng)
        assert not errors, (S, B, gran, K, items, errors[0])


MUTATIONS = [
    "producer_phase",   # the producer waits for the stage's current phase, not the previous one
    "tmem_phase",       # the MMA waits for the buffer's current phase
    "skip_tmem_wait",   # the MMA does not wait for the promotion to free the buffer
    "early_release",    # the stage is released when the MMAs are issued, not when they finish
    "promo_phase",      # the promotion waits for the previous phase of tmem_full
]


@pytest.mark.parametrize("mutation", MUTATIONS)
def test_model_catches_planted_protocol_mistakes(mutation):
    """Each planted mistake is caught: as a deadlock, a wait passing at the
    wrong phase, or a stage or buffer used out of turn."""
    rng = random.Random(hash(mutation) & 0xFFFF)
    for bnq, q_mn, gran in ((256, False, 128), (128, True, 64), (64, False, 256)):
        S, B = stages(bnq, q_mn), bufs(bnq)
        caught = False
        for _ in range(300):
            K = rng.choice([5 * BK, 9 * BK, 17 * BK])
            items = work_list(rng, gran, K)
            if simulate(S, B, gran, K, items, rng, mutation):
                caught = True
                break
        assert caught, (mutation, bnq, q_mn, gran)
