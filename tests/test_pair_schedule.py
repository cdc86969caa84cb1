"""The NF4 pair GEMM's schedule (host side, from the library) walked with the
kernel's own step and segment arithmetic (CPU, no device): whole rounds of 512 x 256
tiles, then the remaining tiles' K steps in equal ranges over the pairs. Every
(tile, step) is covered exactly once; a tile cut into parts is finished by the pair
holding its first step, which is that pair's last range, while the later parts are
their pairs' first ranges (done before it, so the finishing pair's bounded wait
always ends); no tile has more than four parts; the per-tile counters (two per
tile) and the per-pair partial slots stay inside their regions."""
import ctypes

import pytest

from quantized_lora_fine_b200 import _lib, build

MAX_PAIRS = 80          # partial slots and counter pairs reserved in the workspace
COUNTER_INTS = 2 * MAX_PAIRS


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.load()


def schedule(lib, tiles, steps, pairs, aux=0):
    out = (ctypes.c_int32 * 8)()
    assert lib.qlora_pair_schedule(tiles, aux, steps, pairs, out) == 0
    return list(out)


def tail_range(pr, L, W, A, La):
    """Pair pr's tail steps [b, e) (the kernel's sk_tail_begin / sk_tail_len)."""
    b = pr * La if pr < A else A * La + (pr - A) * L
    ln = La if pr < A else L
    return b, min(b + ln, W)


def pair_of(s, L, A, La):
    """The pair holding tail step s (the kernel's sk_pair_of)."""
    a = A * La
    return s // La if s < a else A + (s - a) // L


def walk(P, R, L, W, base, launch, tiles, steps, A=0, La=0):
    """The kernel's per-pair step sequence and its segments (as the epilogue walks them)."""
    seen = set()
    for pr in range(launch):
        dp = R * steps
        tb, te = tail_range(pr, L, W, A, La)
        n = dp + max(0, te - tb)
        assert n > 0, "a launched pair without work"
        seq = []
        for i in range(n):
            if i < dp:
                r = i // steps
                tile, k = pr + r * P, i - r * steps
            else:
                ti = tb + (i - dp)
                u = ti // steps
                tile, k = base + u, ti - u * steps
            assert 0 <= tile < tiles and 0 <= k < steps
            assert (tile, k) not in seen
            seen.add((tile, k))
            seq.append((tile, k))
        segs, i = [], 0
        while i < n:
            tile, kb = seq[i]
            ln = steps if i < dp else min(steps - kb, n - i)
            segs.append((tile, kb, kb + ln))
            i += ln
        for si, (tile, kb, ke) in enumerate(segs):
            if kb == 0 and ke == steps:
                continue
            u = tile - base
            pf, pl = pair_of(u * steps, L, A, La), pair_of((u + 1) * steps - 1, L, A, La)
            assert pf <= pr <= pl < launch and pl - pf + 1 <= 4
            assert 2 * u + 1 < COUNTER_INTS
            if kb == 0:
                assert pr == pf and si == len(segs) - 1     # finishing part: the pair's last range
            else:
                assert si == R                              # later part: the pair's first range
    assert len(seen) == tiles * steps


@pytest.mark.parametrize("pairs", [1, 2, 3, 5, 7, 16, 37, 64, 72, 73, 74, 80])
def test_schedule_covers_every_step_once(lib, pairs):
    for tiles in list(range(1, 48)) + [64, 97, 256, 512, 688, 1280]:
        for steps in (1, 2, 3, 5, 9, 13, 65, 66, 81, 173, 217):
            P, R, L, W, base, launch, A, La = schedule(lib, tiles, steps, pairs)
            assert P == pairs and A == 0 and launch <= MAX_PAIRS and launch <= 4 * tiles
            walk(P, R, L, W, base, launch, tiles, steps)


def test_q_proj_last_round_is_split(lib):
    """q_proj (8192 x 4096 output: 256 tiles of 64 K steps + 1 LoRA step): 3 whole
    rounds, then 30 or 33 steps per pair on 74 or 73 pairs, instead of a fourth round."""
    assert schedule(lib, 256, 65, 74)[1:4] == [3, 30, 34 * 65]
    assert schedule(lib, 256, 65, 73)[1:4] == [3, 33, 37 * 65]
    assert schedule(lib, 256, 65, 64)[1:3] == [4, 0]


def test_aux_pairs_take_longer_tails(lib):
    """q_proj with its 16 T tiles (272 tiles of 65 steps on 74 pairs): 3 whole rounds,
    then the 16 pairs whose first round was a T tile take 29 more tail steps (9/20 of
    a tile) than the other 58, which take 38: every pair about 233 output-tile steps
    of work."""
    P, R, L, W, base, launch, A, La = schedule(lib, 272, 65, 74, aux=16)
    assert (R, W, base, launch, A, L, La) == (3, 50 * 65, 222, 74, 16, 38, 67)
    assert A * La + (P - A) * L >= W
    walk(P, R, L, W, base, launch, 272, 65, A, La)


@pytest.mark.parametrize("pairs", [1, 2, 3, 5, 7, 16, 37, 73, 74, 80])
def test_schedule_with_aux_tiles(lib, pairs):
    """Aux tiles as the kernel gets them (one per 512-row block ahead of the block's
    output tiles): every step once, at most four parts a tile, parts in order."""
    for blocks in (1, 2, 3, 5, 16, 17, 33, 80):
        for per_block in (1, 2, 3, 16):
            tiles = blocks * (per_block + 1)
            for steps in (1, 2, 5, 9, 65, 66, 217):
                if tiles * steps > 60000:   # the walk is plain Python
                    continue
                P, R, L, W, base, launch, A, La = schedule(lib, tiles, steps, pairs, aux=blocks)
                assert launch <= MAX_PAIRS
                walk(P, R, L, W, base, launch, tiles, steps, A, La)


def test_schedule_refuses_bad_arguments(lib):
    out = (ctypes.c_int32 * 8)()
    assert lib.qlora_pair_schedule(0, 0, 5, 4, out) == 2
    assert lib.qlora_pair_schedule(5, 0, 5, 81, out) == 2
    assert lib.qlora_pair_schedule(5, 6, 5, 4, out) == 2
    assert lib.qlora_pair_schedule(5, -1, 5, 4, out) == 2
    assert lib.qlora_pair_schedule(5, 0, 5, 4, None) == 1


def simulate_flags(P, R, L, W, base, launch, blocks, per_block, steps, ext, aux_last=False, A=0, La=0):
    """Runs the kernel's per-pair step order as a discrete-event model: every pair
    advances one K step per tick unless blocked. An output tile's first LoRA step
    (k = steps - ext) waits until its block's aux tile (tile id = block) is finished,
    i.e. every step of it is done by whichever pairs hold its parts (a split tile's
    finishing pair adds the other parts once they have counted in; it holds its
    pair's last range, so its own wait delays nothing else). Returns the number of
    ticks, or None if the pairs deadlock. aux_last puts the aux tiles after the output
    tiles instead (an order the kernel does not use; the model must catch it)."""
    aux = blocks
    total = aux + blocks * per_block
    seqs = []
    for pr in range(launch):
        dp = R * steps
        tb, te = tail_range(pr, L, W, A, La)
        n = dp + max(0, te - tb)
        seq = []
        for i in range(n):
            if i < dp:
                r = i // steps
                seq.append((pr + r * P, i - r * steps))
            else:
                ti = tb + (i - dp)
                u = ti // steps
                seq.append((base + u, ti - u * steps))
        seqs.append(seq)
    done_steps = [0] * total
    pos = [0] * launch
    ticks = 0
    while any(pos[p] < len(seqs[p]) for p in range(launch)):
        moved = False
        for p in range(launch):
            if pos[p] >= len(seqs[p]):
                continue
            tile, k = seqs[p][pos[p]]
            is_aux = (tile >= total - aux) if aux_last else (tile < aux)
            if not is_aux and k == steps - ext:
                mb = (tile if aux_last else tile - aux) // per_block
                flag_tile = total - aux + mb if aux_last else mb
                if done_steps[flag_tile] < steps:
                    continue                      # the LoRA step waits for the block's T / U
            pos[p] += 1
            done_steps[tile] += 1
            moved = True
        ticks += 1
        if not moved:
            return None
    assert all(d == steps for d in done_steps)
    return ticks


@pytest.mark.parametrize("pairs", [1, 2, 3, 5, 7, 16, 74])
def test_aux_flag_waits_never_deadlock(lib, pairs):
    """The aux tiles (T or U, one per 512-row block) set a per-block flag that the
    output tiles' first LoRA step waits for. Walking the library's schedule with
    those waits and with split tiles finished only after all their parts, every pair
    count and shape finishes: no wait closes a cycle."""
    for blocks in (1, 2, 3, 5, 16, 17):
        for per_block in (1, 2, 3, 16):
            for steps, ext in ((2, 1), (5, 1), (9, 1), (66, 2), (65, 1)):
                tiles = blocks * per_block
                if (tiles + blocks) * steps > 30000:
                    continue
                P, R, L, W, base, launch, A, La = schedule(lib, tiles + blocks, steps, pairs, aux=blocks)
                assert simulate_flags(P, R, L, W, base, launch, blocks, per_block, steps, ext, A=A,
                                      La=La) is not None


def test_aux_flag_model_catches_a_bad_order(lib):
    """The model is not vacuous: with the aux tiles after the output tiles, a single
    pair reaches an output tile's LoRA step before its block's aux tile and waits
    forever."""
    P, R, L, W, base, launch, A, La = schedule(lib, 2 + 2 * 3, 5, 1)
    assert simulate_flags(P, R, L, W, base, launch, 2, 3, 5, 1, aux_last=True) is None
    assert simulate_flags(P, R, L, W, base, launch, 2, 3, 5, 1) is not None
