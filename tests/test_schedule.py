"""The prefill kernel's work schedule, enumerated on the host (no GPU needed).

lightning_attn_fwd_plan runs the same scheduling code the kernel runs (a
host-and-device header) and lists every work item per CTA.  These tests check
the invariants the kernel's correctness rests on, for many batch shapes and
SM counts:

* every output token of every sequence is produced exactly once, and exactly
  one item per sequence ends it (and writes the caller's final state);
* split scan: the local-state items partition the first F blocks of every
  sequence, publish in distinct slots, and each entering state chains exactly
  the local states of the blocks before it, in order;
* balanced hand-over: every entering item has a publishing item for the same
  sequence on the previous CTA, ending where it starts, run first there;
* chunk scan: every chunk is handed out once and waits for its predecessor's
  flag value;
* the static splits are balanced to within a few blocks per CTA.
"""
import collections

import numpy as np
import pytest

from long_context_fwd_b200 import build, ops

BLK = 128
ENTER, PUBLISH, LAST, PHASE1 = 1, 2, 4, 8


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()


def _plan(B, H, N, chunk=0, sms=148):
    info, rec = ops.fwd_plan(B, H, N, chunk, sms)
    return info, [dict(zip(ops.PLAN_FIELDS, map(int, r))) for r in rec]


def _check_outputs(B, H, N, items):
    nseq = B * H
    cover = collections.defaultdict(list)
    lasts = collections.Counter()
    for it in items:
        if it["kind"] != 0:
            continue
        assert it["b"] > 0
        cover[it["seq"]].append((it["a"], it["a"] + it["b"]))
        if it["flags"] & LAST:
            lasts[it["seq"]] += 1
            assert it["a"] + it["b"] == N
    assert sorted(cover) == list(range(nseq))
    for s, iv in cover.items():
        iv.sort()
        assert iv[0][0] == 0 and iv[-1][1] == N, s
        for (a0, a1), (b0, b1) in zip(iv, iv[1:]):
            assert a1 == b0, (s, iv)
        for a0, _ in iv:
            assert a0 % BLK == 0
    assert all(lasts[s] == 1 for s in range(nseq))


SHAPES = [
    # B, H, N
    (1, 64, 8192), (1, 64, 1048576), (4, 64, 32768), (1, 1, 100000), (1, 2, 5000),
    (1, 19, 3000), (1, 37, 1025), (1, 100, 2000), (1, 147, 1200), (1, 148, 1200),
    (1, 149, 1025), (2, 80, 1100), (1, 296, 300), (3, 100, 700), (1, 64, 1152),
    (1, 5, 129), (2, 3, 777), (1, 64, 130), (1, 20, 100000),
]


# 74 and 66: each role of the backward's paired launch is planned for half the
# CTAs of a 148- or 132-SM part
@pytest.mark.parametrize("sms", [148, 132, 160, 74, 66])
@pytest.mark.parametrize("B,H,N", SHAPES)
def test_every_output_once(B, H, N, sms):
    info, items = _plan(B, H, N, sms=sms)
    _check_outputs(B, H, N, items)
    assert info["grid"] <= sms


def _check_chunk_scan(B, H, N, info, items):
    """Chunk scan: ticket w is chunk w // (B*H) of sequence w % (B*H); every
    chunk once; each waits for its predecessor's value in the alternate slot
    and publishes its own."""
    assert info["mode"] == 0
    _check_outputs(B, H, N, items)
    nseq, nch, L = B * H, info["nchunks"], info["L"]
    seen = set()
    for w, it in enumerate(items):
        c = w // nseq
        assert it["cta"] == -1 and it["seq"] == w % nseq and it["a"] == c * L
        seen.add((it["seq"], c))
        assert bool(it["flags"] & PHASE1) == (c + 1 < nch)
        if c > 0:
            assert it["flags"] & ENTER and it["enter_val"] == c
            assert it["enter_slot"] == it["seq"] * 2 + ((c - 1) & 1)
        if c + 1 < nch:
            assert it["pub_slot"] == it["seq"] * 2 + (c & 1) and it["pub_val"] == c + 1
    assert len(seen) == nseq * nch


@pytest.mark.parametrize("B,H,N,chunk", [(1, 4, 3000, 512), (3, 4, 2100, 128), (2, 80, 1100, 256),
                                         (1, 2, 4097, 1024), (1, 64, 8192, 2048)])
def test_explicit_chunks_use_the_chunk_scan(B, H, N, chunk):
    info, items = _plan(B, H, N, chunk)
    assert info["L"] == chunk
    _check_chunk_scan(B, H, N, info, items)


def _per_cta(items):
    by = collections.defaultdict(list)
    for it in items:
        by[it["cta"]].append(it)
    return by


def _check_handover(B, H, N, sms, info, items):
    """Balanced hand-over: equal block shares; a publishing item runs first on
    its CTA, its sequence's entering item last on the next CTA, starting where
    it ends."""
    assert info["mode"] == 1 and info["grid"] == sms
    by = _per_cta(items)
    nblk = -(-N // BLK)
    share = B * H * nblk / sms
    for cta, its in by.items():
        blocks = sum(-(-it["b"] // BLK) for it in its)
        assert abs(blocks - share) <= 1
        for pos, it in enumerate(its):
            if it["flags"] & PUBLISH:
                assert pos == 0 and it["a"] == 0 and it["pub_slot"] == cta
                assert not it["flags"] & LAST
            if it["flags"] & ENTER:
                assert pos == len(its) - 1 and it["enter_slot"] == cta - 1
                prev = by[cta - 1][0]
                assert prev["flags"] & PUBLISH and prev["seq"] == it["seq"]
                assert prev["a"] + prev["b"] == it["a"]
    if B * H % sms == 0:
        assert info["slots"] == 0 and not any(it["flags"] & (ENTER | PUBLISH) for it in items)


@pytest.mark.parametrize("sms", [148, 132, 74])
@pytest.mark.parametrize("B,H,N", [(4, 64, 32768), (1, 149, 1025), (2, 80, 1100), (1, 150, 2500),
                                   (1, 296, 300), (3, 100, 700), (1, 200, 5000)])
def test_balanced_handover(B, H, N, sms):
    info, items = _plan(B, H, N, sms=sms)
    _check_handover(B, H, N, sms, info, items)


@pytest.mark.parametrize("sms", [148, 132, 160, 74, 66])
@pytest.mark.parametrize("B,H,N", [(1, 64, 8192), (1, 64, 1048576), (1, 19, 3000), (1, 37, 1025),
                                   (1, 100, 2000), (1, 147, 1200), (1, 64, 1152),
                                   (1, 20, 100000), (2, 40, 9000)])
def test_split_scan(B, H, N, sms):
    info, items = _plan(B, H, N, sms=sms)
    nseq, nblk = B * H, -(-N // BLK)
    if nseq >= sms:
        return
    if info["mode"] == 0:
        # so few sequences that the chains would be long (chunk scan), or so
        # many that one whole sequence per SM is as fast (whole sequences)
        ok_whole = nblk <= 8 or nseq * nblk / sms > 0.6 * nblk
        assert 8 * nseq < sms or ok_whole, info
        return
    _check_split_scan(B, H, N, sms, info, items)


def _check_split_scan(B, H, N, sms, info, items):
    """Split scan: local-state items partition the first F blocks of every
    sequence in distinct slots; each entering state chains exactly the pieces
    before it, in order; both passes balanced; never slower than one whole
    sequence per SM."""
    nseq, nblk = B * H, -(-N // BLK)
    assert info["mode"] == 2, info
    F, G2, G = info["F"], info["G2"], info["grid"]
    assert G == sms and G2 == sms - nseq and 1 <= F < nblk
    by = _per_cta(items)
    # local-state items partition the first F blocks of every sequence
    local = {}
    cover = collections.defaultdict(list)
    for it in items:
        if it["kind"] == 1:
            assert it["flags"] & PHASE1 and it["flags"] & PUBLISH and it["pub_val"] == 1
            assert not it["flags"] & (ENTER | LAST)
            x = it["seq"] * F + it["a"] // BLK
            y = x + it["b"] // BLK
            assert it["b"] % BLK == 0
            assert it["pub_slot"] not in {v[2] for v in local.values()}
            assert 0 <= it["pub_slot"] < info["slots"]
            local[x] = (y, it["seq"], it["pub_slot"])
            cover[it["seq"]].append((it["a"] // BLK, it["a"] // BLK + it["b"] // BLK))
    for s in range(nseq):
        iv = sorted(cover[s])
        assert iv[0][0] == 0 and iv[-1][1] == F
        assert all(a1 == b0 for (_, a1), (b0, _) in zip(iv, iv[1:]))
    # each entering state chains the local states before it, in order
    for cta, its in by.items():
        for pos, it in enumerate(its):
            if it["kind"] == 0 and it["flags"] & ENTER:
                links = []
                for nxt in its[pos + 1:]:
                    if nxt["kind"] != 2:
                        break
                    links.append(nxt)
                x = it["seq"] * F
                for ln in links:
                    assert ln["a"] == x and x in local
                    assert local[x][0] == ln["b"] and local[x][2] == ln["enter_slot"]
                    x = ln["b"]
                assert x == it["seq"] * F + it["a"] // BLK
                # the kernel notes the chain in a 32-entry shared-memory list
                assert len(links) <= 32
        kinds = [it["kind"] for it in its]
        # local-state items first, then outputs in stream order (so only the
        # first output item can enter a sequence part-way)
        first_out = kinds.index(0) if 0 in kinds else len(kinds)
        assert all(k == 1 for k in kinds[:first_out])
        outs = [it for it in its if it["kind"] == 0]
        assert all(not it["flags"] & ENTER for it in outs[1:])
        assert all((a["seq"], a["a"]) < (b["seq"], b["a"]) for a, b in zip(outs, outs[1:]))
    # both passes are balanced
    P = nseq * F
    for cta, its in by.items():
        lb = sum(it["b"] // BLK for it in its if it["kind"] == 1)
        assert abs(lb - P / G) <= 1
        ob = sum(-(-it["b"] // BLK) for it in its if it["kind"] == 0)
        assert abs(ob - nseq * nblk / G) <= 1.5 + nseq / G2
        assert ob + 0.4 * lb < nblk  # never slower than one whole sequence per SM


def test_split_scan_local_state_fraction():
    # 64 sequences on 148 SMs: the local-state pass covers 1 - 64/148 of the tokens
    info, items = _plan(1, 64, 1048576)
    local = sum(it["b"] for it in items if it["kind"] == 1)
    assert abs(local / (64 * 1048576) - (1 - 64 / 148)) < 1e-3


def test_small_problems_stay_whole_or_ticketed():
    info, _ = _plan(1, 2, 900)  # 8 blocks: whole sequences
    assert info["mode"] == 0 and info["nchunks"] == 1
    info, _ = _plan(1, 4, 1 << 20)  # few long sequences: chunk scan
    assert info["mode"] == 0 and info["nchunks"] > 1


def test_plan_rejects_bad_arguments():
    lib = ops.lib()
    import ctypes
    info = (ctypes.c_int * 8)()
    n = ctypes.c_int(0)
    assert lib.lightning_attn_fwd_plan(1, 1, 0, 0, 148, info, None, 0, ctypes.byref(n)) == 2
    assert lib.lightning_attn_fwd_plan(1, 1, 100, 100, 148, info, None, 0, ctypes.byref(n)) == 2
    assert lib.lightning_attn_fwd_plan(1, 1, 100, 0, 148, None, None, 0, ctypes.byref(n)) == 1
    # too small a record buffer reports the count and LA_ERR_WORKSPACE
    assert lib.lightning_attn_fwd_plan(1, 64, 8192, 0, 148, info, None, 0, ctypes.byref(n)) == 7
    assert n.value > 0


def _random_shapes(n, seed):
    """Seeded shapes over every work split: many sequences (hand-over), the
    split-scan range, few sequences (chunk scan or whole sequences), lengths
    log-uniform from 1 token to 128K, several SM counts."""
    rng = np.random.default_rng(seed)
    for _ in range(n):
        sms = int(rng.choice([148, 132, 160, 114, 80, 8]))
        pick = int(rng.integers(3))
        if pick == 0:
            nseq = int(rng.integers(sms, 6 * sms))
        elif pick == 1:
            nseq = int(rng.integers(max(1, sms // 8), sms))
        else:
            nseq = int(rng.integers(1, max(2, sms // 8)))
        B = int(rng.choice([d for d in range(1, 9) if nseq % d == 0]))
        N = int(rng.integers(1, 1 << int(rng.integers(1, 18))))
        yield B, nseq // B, N, sms


@pytest.mark.parametrize("seed", range(4))
def test_random_shapes_keep_every_invariant(seed):
    modes = collections.Counter()
    for B, H, N, sms in _random_shapes(60, seed):
        info, items = _plan(B, H, N, sms=sms)
        modes[info["mode"]] += 1
        _check_outputs(B, H, N, items)
        assert info["grid"] <= sms
        if info["mode"] == 1:
            _check_handover(B, H, N, sms, info, items)
        elif info["mode"] == 2:
            _check_split_scan(B, H, N, sms, info, items)
        else:
            _check_chunk_scan(B, H, N, info, items)
    assert len(modes) == 3, modes  # the draw reaches every split
