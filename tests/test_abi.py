"""Host-side checks of the C ABI (no GPU needed, no kernel is launched).

Every entry point declared in include/qz.h must be exported by libqz.so, and
every argument error must come back synchronously, before any launch.  The
pointers below are fake addresses that are never dereferenced: each call is
rejected by the host-side checks first.
"""
import ctypes
import os
import re

import pytest

import weight_only_quantization_wise_b200 as qz

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "qz.h")

OK, INVALID, ALIGN, UNSUP, WS = 0, 1, 2, 3, 4
A = ctypes.c_void_p(0x10000)          # fake, 16-byte aligned "device" pointers
B = ctypes.c_void_p(0x20000)
C = ctypes.c_void_p(0x30000)
D = ctypes.c_void_p(0x40000)
Y = ctypes.c_void_p(0x50000)
MIS = ctypes.c_void_p(0x10008)        # 8-byte aligned only


def declared_functions():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"QZ_API\s+[\w\s\*]*?\b(qz_\w+)\s*\(", src)))


def test_header_declarations_are_exported():
    names = declared_functions()
    assert len(names) >= 11
    for n in names:
        assert hasattr(qz.lib, n), n
    assert sorted(qz.EXPORTED_SYMBOLS) == names


def test_status_strings_and_version():
    for s in range(7):
        assert qz.qz_status_string(s)
    assert qz.qz_status_string(99) == "unknown status"
    assert qz.qz_version() >= 100


def test_packed_bytes_formats():
    assert qz.qz_packed_bytes(4096, 4096, 4, False, 128) == (4096 * 2048, 4096 * 32 * 2, 4096 * 32)
    assert qz.qz_packed_bytes(4096, 4096, 8, True, 4096) == (4096 * 4096, 4096 * 2, 0)
    assert qz.qz_packed_bytes(10, 64, 4, True, 0) == (320, 2, 0)
    for bad in [(0, 128, 4, False, 128), (8, 100, 4, False, 128), (8, 128, 4, False, -1)]:
        with pytest.raises(qz.QzError):
            qz.qz_packed_bytes(*bad)
    with pytest.raises(qz.QzError):
        qz.qz_packed_bytes(8, 128, 3, False, 128)


def test_workspace_bytes():
    assert qz.qz_workspace_bytes(qz.QZ_OP_QUANTIZE_PACK, 1, 8, 128, 128) == 0
    assert qz.qz_workspace_bytes(qz.QZ_OP_QUANTIZE_PACK, 1, 8, 128, 0) == 8
    assert qz.qz_workspace_bytes(qz.QZ_OP_DEQUANTIZE, 1, 8, 128, 128) == 0
    big = qz.qz_workspace_bytes(qz.QZ_OP_W4A16_GEMV, 1, 1024, 1024, 128)
    assert big > 0 and big % 4 == 0
    assert qz.qz_workspace_bytes(qz.QZ_OP_W4A16_GEMV, 16, 1024, 1024, 128) >= big
    # the integer decode GEMVs take up to 64 tokens, the FP4A16 GEMV up to 16
    assert qz.qz_workspace_bytes(qz.QZ_OP_W4A16_GEMV, 64, 1024, 1024, 128) > 0
    with pytest.raises(qz.QzError):
        qz.qz_workspace_bytes(qz.QZ_OP_W4A16_GEMV, 65, 1024, 1024, 128)
    with pytest.raises(qz.QzError):
        qz.qz_workspace_bytes(qz.QZ_OP_FP4A16_GEMV, 17, 1024, 1024, 0)
    with pytest.raises(qz.QzError):
        qz.qz_workspace_bytes(99, 1, 8, 128, 128)


def L():
    return qz.lib


@pytest.mark.parametrize("args,expect", [
    ((None, 8, 128, 4, 0, 128, B, C, D, None, 0, None), INVALID),        # null w
    ((A, 8, 128, 4, 0, 128, B, C, None, None, 0, None), INVALID),        # asym without zeros
    ((A, 8, 128, 4, 1, 128, B, C, D, None, 0, None), INVALID),           # sym with zeros
    ((A, 0, 128, 4, 0, 128, B, C, D, None, 0, None), INVALID),           # N = 0
    ((A, 8, 100, 4, 0, 100, B, C, D, None, 0, None), UNSUP),             # K % 8
    ((A, 8, 128, 4, 0, 48, B, C, D, None, 0, None), INVALID),            # K % g
    ((A, 8, 128, 5, 0, 128, B, C, D, None, 0, None), UNSUP),             # bits
    ((MIS, 8, 128, 4, 0, 128, B, C, D, None, 0, None), ALIGN),           # w alignment
    ((A, 8, 128, 4, 0, 0, B, C, D, None, 0, None), WS),                  # per-tensor needs ws
    ((A, 8, 128, 4, 0, 0, B, C, D, Y, 4, None), WS),                     # ws too small
])
def test_quantize_pack_rejects(args, expect):
    assert L().qz_quantize_pack(*args) == expect


@pytest.mark.parametrize("args,expect", [
    ((None, B, C, 8, 128, 4, 0, 128, Y, None), INVALID),
    ((A, B, None, 8, 128, 4, 0, 128, Y, None), INVALID),
    ((A, B, C, 8, 128, 4, 0, 128, MIS, None), ALIGN),
    ((A, B, C, 8, 130, 4, 0, 130, Y, None), UNSUP),
])
def test_dequantize_rejects(args, expect):
    assert L().qz_dequantize(*args) == expect


@pytest.mark.parametrize("args,expect", [
    ((A, B, C, D, 0, 64, 128, 128, Y, None, 0, None), INVALID),          # M = 0
    ((A, B, C, D, 65, 64, 128, 128, Y, None, 0, None), UNSUP),           # M > 64
    ((A, B, C, D, 1, 64, 192, 64, Y, None, 0, None), UNSUP),             # K % 128
    ((A, B, C, D, 1, 64, 256, 48, Y, None, 0, None), INVALID),           # K % g
    ((A, B, C, D, 1, 64, 256, 16, Y, None, 0, None), UNSUP),             # g % 32
    ((A, B, C, None, 1, 64, 256, 128, Y, None, 0, None), INVALID),       # null zeros
    ((MIS, B, C, D, 1, 64, 256, 128, Y, None, 0, None), ALIGN),
    ((A, B, C, D, 1, 4096, 4096, 128, Y, None, 0, None), WS),            # split-K needs ws
])
def test_w4a16_gemv_rejects(args, expect):
    assert L().qz_w4a16_gemv(*args) == expect


@pytest.mark.parametrize("args,expect", [
    ((A, B, C, 0, 64, 128, Y, None, 0, None), INVALID),
    ((A, B, C, 65, 64, 128, Y, None, 0, None), UNSUP),           # M > 64
    ((A, B, None, 1, 64, 128, Y, None, 0, None), INVALID),
    ((A, MIS, C, 1, 64, 128, Y, None, 0, None), ALIGN),
    ((A, B, C, 1, 4096, 4096, Y, None, 0, None), WS),
])
def test_w8a16_gemv_rejects(args, expect):
    assert L().qz_w8a16_gemv(*args) == expect


@pytest.mark.parametrize("args,expect", [
    ((A, B, C, D, 0, 64, 128, 128, Y, None, 0, None), INVALID),
    ((A, B, C, D, 64, 64, 192, 64, Y, None, 0, None), UNSUP),
    ((A, B, C, D, 64, 64, 256, 32, Y, None, 0, None), UNSUP),           # g % 64 for the GEMM
    ((None, B, C, D, 64, 64, 256, 128, Y, None, 0, None), INVALID),
])
def test_w4a16_gemm_rejects(args, expect):
    assert L().qz_w4a16_gemm(*args) == expect


@pytest.mark.parametrize("args,expect", [
    ((A, B, C, 0, 64, 128, Y, None, 0, None), INVALID),                # M = 0
    ((A, B, C, 64, 64, 192, Y, None, 0, None), UNSUP),                 # K % 128
    ((A, B, None, 64, 64, 256, Y, None, 0, None), INVALID),            # null scales
    ((A, B, C, 64, 64, 256, None, None, 0, None), INVALID),            # null y
    ((MIS, B, C, 64, 64, 256, Y, None, 0, None), ALIGN),
    ((A, B, C, 64, 64, 256, MIS, None, 0, None), ALIGN),               # y for the TMA store
    ((A, B, C, 16, 4096, 4096, Y, None, 0, None), WS),                 # M <= 16: GEMV split-K
])
def test_w8a16_gemm_rejects(args, expect):
    assert L().qz_w8a16_gemm(*args) == expect


def gemm_schedule_model(M, N, K, sms):
    """The prefill GEMM's schedule as the header of qz_gemm_sm100.cu states
    it: whole 128 x 256 tiles round robin for the full waves, the K steps of
    the last partial wave (all tiles when they are fewer than the CTAs) laid
    end to end and cut into equal contiguous ranges, one per tail CTA (at
    least 4 steps each, at most 6 CTAs per tail tile on average); no tail
    when the waves are full or sharing would save a CTA fewer than 48 K
    steps ((grid - tail tiles) * KT / grid).
    Returns (act_rows, grid CTAs, tiles, tail tiles, tail CTAs, KT)."""
    act_rows = 256 if M >= 256 else (M + 15) // 16 * 16
    grid = sms * (2 if act_rows <= 64 else 1)
    tiles = -(-N // 128) * -(-M // 256)
    KT = K // 64
    tail = tiles % grid if tiles >= grid else tiles
    if (tiles >= grid and tail == 0) or (grid - tail) * KT < 48 * grid:
        return act_rows, grid, tiles, 0, 0, KT
    ctas = max(1, min(grid, 6 * tail, tail * KT // 4))
    return act_rows, grid, tiles, tail, ctas, KT


def gemm_workspace_model(M, N, K, sms):
    """fp32 slots of act_rows x 128 placed 1 KB further apart than that,
    then one counter per tail tile in blocks of 64."""
    act_rows, _, _, tail, ctas, _ = gemm_schedule_model(M, N, K, sms)
    if ctas == 0:
        return 0
    slots = ctas + tail - 1
    return -(-(slots * (act_rows * 128 + 256) * 4) // 256) * 256 + -(-tail // 64) * 64 * 4


def tail_segments(tail, KT, ctas):
    """(cta, tail tile, kt0, kt1, slot) of every tail segment: CTA c takes
    steps [floor(c S / P), floor((c + 1) S / P)), S = tail * KT, P = ctas."""
    S = tail * KT
    out = []
    for c in range(ctas):
        b0, b1 = c * S // ctas, (c + 1) * S // ctas
        for t in range(b0 // KT, (b1 - 1) // KT + 1):
            out.append((c, t, max(b0, t * KT) - t * KT, min(b1, (t + 1) * KT) - t * KT, c + t))
    return out


@pytest.mark.parametrize("M,N,K,sms", [
    (2048, 8192, 8192, 148), (2048, 4096, 4096, 148), (2048, 11008, 4096, 148),
    (2048, 4096, 11008, 148), (64, 8192, 8192, 148), (32, 1024, 4096, 148),
    (300, 1000, 1024, 148), (17, 128, 128, 148), (2048, 8192, 8192, 97), (257, 130, 640, 5),
])
def test_gemm_tail_schedule_invariants(M, N, K, sms):
    """Every K step of every tail tile is covered once; a tile's segments take
    consecutive slots in K order (so the last arrival adds them in a fixed
    order), no slot is used twice and every slot index is below tail CTAs +
    tail tiles - 1 (the workspace's slot count), and no tail CTA's range is
    shorter than 4 steps."""
    _, _, _, tail, ctas, KT = gemm_schedule_model(M, N, K, sms)
    if ctas == 0:
        return
    segs = tail_segments(tail, KT, ctas)
    assert all(k1 - k0 >= 1 for _, _, k0, k1, _ in segs)
    for t in range(tail):
        mine = sorted((k0, k1, slot) for _, tt, k0, k1, slot in segs if tt == t)
        assert mine[0][0] == 0 and mine[-1][1] == KT
        assert all(a[1] == b[0] for a, b in zip(mine, mine[1:]))
        assert [x[2] for x in mine] == list(range(mine[0][2], mine[0][2] + len(mine)))
    slots = [x[4] for x in segs]
    assert len(set(slots)) == len(slots) and max(slots) < ctas + tail - 1
    S = tail * KT
    assert ctas == 1 or min((c + 1) * S // ctas - c * S // ctas for c in range(ctas)) >= 4


@pytest.mark.parametrize("M,N,K", [
    (2048, 8192, 8192), (2048, 4096, 4096), (2048, 11008, 4096), (2048, 28672, 8192),
    (64, 8192, 8192), (128, 8192, 8192), (48, 1024, 2048), (200, 512, 2048), (33, 128, 128),
    (4096, 4096, 4096), (300, 1000, 1024), (257, 130, 640), (16, 256, 192),
])
def test_gemm_workspace_matches_the_schedule(M, N, K):
    """qz_workspace_bytes_for_sms of both GEMMs is the schedule's workspace
    (fp32 slots of act_rows x 128, then one counter per tail tile) for every
    SM count, and qz_workspace_bytes the largest of them."""
    for op, g in ((qz.QZ_OP_W4A16_GEMM, 128 if K % 128 == 0 else 64), (qz.QZ_OP_W8A16_GEMM, K)):
        want = [gemm_workspace_model(M, N, K, sms) for sms in range(1, 149)]
        got = [qz.qz_workspace_bytes_for_sms(op, M, N, K, g, sms) for sms in range(1, 149)]
        assert got == want
        assert qz.qz_workspace_bytes(op, M, N, K, g) == max(want)


def test_gemm_workspace_follows_the_route():
    # 2048 x 8192 x 8192 on 148 SMs: 512 tiles, 3 whole waves and 68 tail
    # tiles over 148 CTAs: 215 slots of 256 x 128 fp32 (+ 1 KB apart), 68
    # counters (two blocks of 64)
    assert qz.qz_workspace_bytes_for_sms(qz.QZ_OP_W8A16_GEMM, 2048, 8192, 8192, 8192, 148) == \
        215 * (256 * 128 + 256) * 4 + 2 * 64 * 4
    # 4096 tokens x 4096 rows: 512 tiles; on 128 SMs four whole waves, no workspace
    assert qz.qz_workspace_bytes_for_sms(qz.QZ_OP_W4A16_GEMM, 4096, 4096, 4096, 128, 128) == 0
    # 64 tokens: 64 tiles over 296 CTAs (two per SM): 359 slots of 64 x 128
    assert qz.qz_workspace_bytes_for_sms(qz.QZ_OP_W8A16_GEMM, 64, 8192, 8192, 8192, 148) == \
        359 * (64 * 128 + 256) * 4 + 64 * 4
    # 2048 tokens x 4096 x 4096: 256 tiles, the 108-tile last wave would save
    # a CTA only 17 K steps: whole tiles, no workspace
    assert qz.qz_workspace_bytes_for_sms(qz.QZ_OP_W4A16_GEMM, 2048, 4096, 4096, 128, 148) == 0
    assert qz.qz_workspace_bytes(qz.QZ_OP_W4A16_GEMM, 64, 8192, 8192, 128) == \
        qz.qz_workspace_bytes(qz.QZ_OP_W8A16_GEMM, 64, 8192, 8192, 8192)
    for M in (16, 32):      # up to 32 tokens the GEMM entry runs the decode GEMV
        assert (qz.qz_workspace_bytes(qz.QZ_OP_W8A16_GEMM, M, 4096, 4096, 4096) ==
                qz.qz_workspace_bytes(qz.QZ_OP_W8A16_GEMV, M, 4096, 4096, 4096))
        assert (qz.qz_workspace_bytes(qz.QZ_OP_W4A16_GEMM, M, 4096, 4096, 128) ==
                qz.qz_workspace_bytes(qz.QZ_OP_W4A16_GEMV, M, 4096, 4096, 128))
    assert (qz.qz_workspace_bytes(qz.QZ_OP_W8A16_GEMM, 33, 4096, 4096, 4096) !=
            qz.qz_workspace_bytes(qz.QZ_OP_W8A16_GEMV, 33, 4096, 4096, 4096))


@pytest.mark.parametrize("op,M,N,K,g,expect", [
    # Units are 128 rows x 128 k, or 128 rows x 256 k for int4 with M <= 8,
    # K % 256 == 0 and g % 128 == 0 (K/g % 16 == 0); CTAs per SM: the most (up
    # to 3) that give each CTA at least 4 blocks of 128 k.
    # 4096 x 4096, W4 M = 1: 32 tasks x 16 units = 512 units -> 1 CTA per SM,
    # 3 units per CTA, ceil(16/3) + 1 = 7 slots per 32-row subtask, 128
    # subtasks.
    ("W4A16_GEMV", 1, 4096, 4096, 128, 128 * 7 * 1 * 32 * 4 + 2 * 64 * 4),
    # 70B layer: 7168 units -> 3 CTAs per SM (444), 16 units per CTA,
    # ceil(32/16) + 1 = 3 slots, 896 subtasks
    ("W4A16_GEMV", 1, 28672, 8192, 128, 896 * 3 * 1 * 32 * 4 + 14 * 64 * 4),
    # W8: 1024 units of 128 k -> 1 CTA per SM, 6 per CTA, ceil(32/6) + 1 = 7
    ("W8A16_GEMV", 1, 4096, 4096, 4096, 128 * 7 * 1 * 32 * 4 + 2 * 64 * 4),
    # 11008 x 4096, M = 8: 86 tasks x 16 units = 1376 -> 444 CTAs, 3 units
    # each, ceil(16/3) + 1 = 7 slots, 344 subtasks
    ("W4A16_GEMV", 8, 11008, 4096, 128, 344 * 7 * 8 * 32 * 4 + 6 * 64 * 4),
    # M = 16: units of 128 k; 14336 -> 444 CTAs, 32 each, ceil(64/32) + 1 = 3
    ("W4A16_GEMV", 16, 28672, 8192, 128, 896 * 3 * 16 * 32 * 4 + 14 * 64 * 4),
    # one task, K = 8192: 32 units of 256 k -> 32 CTAs, 32 slots (up to 16
    # tokens); with g = 64, M = 17 or K % 256 != 0 units of 128 k -> 64 CTAs
    # and 64 slots
    ("W4A16_GEMV", 1, 128, 8192, 128, 4 * 32 * 1 * 32 * 4 + 64 * 4),
    ("W4A16_GEMV", 16, 128, 8192, 128, 4 * 32 * 16 * 32 * 4 + 64 * 4),
    ("W4A16_GEMV", 1, 128, 8192, 64, 4 * 64 * 1 * 32 * 4 + 64 * 4),
    ("W4A16_GEMV", 17, 128, 8192, 128, 4 * 64 * 17 * 32 * 4 + 64 * 4),
    ("W4A16_GEMV", 1, 128, 8320, 128, 4 * 65 * 1 * 32 * 4 + 64 * 4),
    # 4096 x 11008: 86 groups per row (gathered words, an even count): 32
    # tasks x 43 units = 1376 -> 444 CTAs, 3 units each, ceil(43/3) + 1 = 16
    ("W4A16_GEMV", 1, 4096, 11008, 128, 128 * 16 * 1 * 32 * 4 + 2 * 64 * 4),
])
def test_gemv_plan_workspace(op, M, N, K, g, expect):
    """The stream-K plan (host logic) on a 148-SM device through the
    workspace it asks for: fp32 partial slots [subtask][slot][M][32] plus one
    counter per 32-row subtask; qz_workspace_bytes is at least that."""
    code = getattr(qz, "QZ_OP_" + op)
    assert qz.qz_workspace_bytes_for_sms(code, M, N, K, g, 148) == expect
    assert qz.qz_workspace_bytes(code, M, N, K, g) >= expect


def test_launch_overlap_setter():
    assert qz.lib.qz_set_launch_overlap(2) == INVALID
    assert qz.lib.qz_set_launch_overlap(-1) == INVALID
    for mode in (1, 0):               # ends on the default
        assert qz.lib.qz_set_launch_overlap(mode) == OK


WS_SHAPES = [  # (op, M, N, K, g): decode GEMV shapes, short and long layers, small-M GEMMs
    (qz.QZ_OP_W4A16_GEMV, 1, 4096, 4096, 128), (qz.QZ_OP_W4A16_GEMV, 1, 28672, 8192, 128),
    (qz.QZ_OP_W4A16_GEMV, 16, 8192, 28672, 128), (qz.QZ_OP_W4A16_GEMV, 4, 11008, 4096, 128),
    (qz.QZ_OP_W4A16_GEMV, 3, 17, 128, 32), (qz.QZ_OP_W8A16_GEMV, 1, 28672, 8192, 8192),
    (qz.QZ_OP_W8A16_GEMV, 8, 4096, 11008, 11008), (qz.QZ_OP_W4A16_GEMM, 48, 1024, 2048, 128),
    (qz.QZ_OP_W4A16_GEMM, 32, 8192, 8192, 128), (qz.QZ_OP_W8A16_GEMM, 200, 512, 2048, 2048),
    (qz.QZ_OP_W4A16_GEMM, 2048, 8192, 8192, 128), (qz.QZ_OP_W4A16_GEMM, 12, 4096, 4096, 128),
    (qz.QZ_OP_W4A16_GEMM, 8, 4096, 4096, 128), (qz.QZ_OP_W4A16_GEMV, 8, 300, 2048, 128),
    (qz.QZ_OP_W4A16_GEMV, 1, 4096, 11008, 128), (qz.QZ_OP_W4A16_GEMV, 4, 130, 5632, 256),
]


@pytest.mark.parametrize("op,M,N,K,g", WS_SHAPES)
def test_workspace_bound_serves_every_sm_count(op, M, N, K, g):
    """Grids are sized for the device's own SM count (at most 148), while
    qz_workspace_bytes does not depend on the device: it must be at least the
    workspace of the plan for every count, and equal to the largest.  An int4
    GEMV planned with 256-wide units (M <= 16, K % 256 == 0, scales and zeros
    through the ring: TMA tiles, or gathered words with the two halves' groups
    in the same words) falls back to 128-wide units when its scale or zero
    array is misaligned, so its bound also covers the 128-wide plans, which are the plans
    of the same shape with g = 64 (the plan depends on g only through the
    unit width)."""
    bound = qz.qz_workspace_bytes(op, M, N, K, g)
    per_sms = [qz.qz_workspace_bytes_for_sms(op, M, N, K, g, sms) for sms in range(1, 149)]
    gpr = K // g
    ring = g % 128 == 0 and ((g // 128) & (g // 128 - 1)) == 0
    two_half = (op in (qz.QZ_OP_W4A16_GEMV, qz.QZ_OP_W4A16_GEMM) and M <= 16 and K % 256 == 0
                and ring and (gpr % 16 == 0 or ((N * gpr) % 4 == 0 and (g > 128 or gpr % 2 == 0))))
    if two_half:
        narrow = [qz.qz_workspace_bytes_for_sms(op, M, N, K, 64, sms) for sms in range(1, 149)]
        assert max(max(per_sms), max(narrow)) == bound
    else:
        assert max(per_sms) == bound
    assert per_sms[-1] == qz.qz_workspace_bytes_for_sms(op, M, N, K, g, 148)
    for bad in (0, 149):
        with pytest.raises(qz.QzError):
            qz.qz_workspace_bytes_for_sms(op, M, N, K, g, bad)


def _gptq(w=A, x=B, N=64, K=256, n=128, bits=4, sym=0, g=128, damp=0.01, codes=C, scales=D,
          zeros=Y, ws=None, ws_bytes=0):
    return L().qz_gptq_quantize(w, x, N, K, n, bits, sym, g, damp, codes, scales, zeros, ws,
                                ws_bytes, None)


@pytest.mark.parametrize("kwargs,expect", [
    (dict(), WS),                                    # no workspace
    (dict(bits=3), UNSUP),
    (dict(N=0), INVALID), (dict(n=0), INVALID), (dict(K=0), INVALID),
    (dict(g=100), INVALID),                          # does not divide K
    (dict(g=16, K=256), UNSUP),                      # below 32
    (dict(g=96, K=384), UNSUP),                      # neither nests with the 128-wide blocks
    (dict(K=260, g=4), UNSUP),                       # K % 8 != 0 (and g too small)
    (dict(damp=-1.0), INVALID), (dict(damp=float("nan")), INVALID),
    (dict(zeros=None), INVALID),                     # asymmetric needs zeros
    (dict(sym=1), INVALID),                          # symmetric takes none
    (dict(x=None), INVALID),
    (dict(w=ctypes.c_void_p(0x10001)), ALIGN),
])
def test_gptq_rejects(kwargs, expect):
    assert _gptq(**kwargs) == expect


def test_gptq_workspace_bytes():
    # fp64: two K x K matrices, N x K working weights, N x 128 block errors
    N, K = 4096, 4096
    assert qz.qz_workspace_bytes(qz.QZ_OP_GPTQ, 1, N, K, 128) == \
        2 * K * K * 8 + N * K * 8 + N * 128 * 8
    assert qz.qz_workspace_bytes(qz.QZ_OP_GPTQ, 1, 37, 384, 128) >= 2 * 384 * 384 * 8 + 37 * 384 * 8


@pytest.mark.parametrize("kind,ts,K,expect", [
    (2, None, 256, UNSUP), (0, None, 100, INVALID), (1, None, 256, INVALID),   # NV needs a tensor scale
    (0, C, 256, INVALID), (1, C, 24, INVALID),                                # MX takes none; K % 16
])
def test_fp4_quantize_rejects(kind, ts, K, expect):
    assert L().qz_fp4_quantize(A, 8, K, kind, B, D, ts, None) == expect


def test_fp4_gemv_rejects_and_workspace():
    ts = C
    assert L().qz_fp4a16_gemv(A, B, D, ts, 17, 64, 256, 1, Y, None, 0, None) == UNSUP     # M > 16
    assert L().qz_fp4a16_gemv(A, B, D, ts, 1, 64, 192, 1, Y, None, 0, None) == UNSUP     # K % 128
    assert L().qz_fp4a16_gemv(A, B, D, None, 1, 64, 256, 1, Y, None, 0, None) == INVALID
    assert L().qz_fp4a16_gemv(MIS, B, D, ts, 1, 64, 256, 1, Y, None, 0, None) == ALIGN
    assert L().qz_fp4a16_gemv(A, B, D, ts, 4, 4096, 4096, 1, Y, None, 0, None) == WS
    # the same stream-K plan as the W4A16 GEMV
    assert qz.qz_workspace_bytes(qz.QZ_OP_FP4A16_GEMV, 4, 4096, 4096, 0) == \
        qz.qz_workspace_bytes(qz.QZ_OP_W4A16_GEMV, 4, 4096, 4096, 128)
    assert qz.qz_fp4_packed_bytes(64, 1024, qz.QZ_FP4_MX) == (64 * 512, 64 * 32)
    assert qz.qz_fp4_packed_bytes(64, 1024, qz.QZ_FP4_NV) == (64 * 512, 64 * 64)


def test_fp4a4_gemm_rejects_and_workspace():
    ts = C
    big = ctypes.c_void_p(0x100000)
    assert L().qz_fp4a4_gemm(A, B, D, ts, 64, 64, 192, 1, Y, big, 1 << 20, None) == UNSUP  # K % 256
    assert L().qz_fp4a4_gemm(A, B, D, ts, 64, 64, 256, 2, Y, big, 1 << 20, None) == UNSUP  # kind
    assert L().qz_fp4a4_gemm(A, B, D, None, 64, 64, 256, 1, Y, big, 1 << 20, None) == INVALID
    assert L().qz_fp4a4_gemm(A, B, D, ts, 64, 64, 256, 0, Y, big, 1 << 20, None) == INVALID
    assert L().qz_fp4a4_gemm(A, B, D, ts, 0, 64, 256, 1, Y, big, 1 << 20, None) == INVALID
    assert L().qz_fp4a4_gemm(MIS, B, D, ts, 64, 64, 256, 1, Y, big, 1 << 20, None) == ALIGN
    assert L().qz_fp4a4_gemm(A, B, MIS, ts, 64, 64, 256, 1, Y, big, 1 << 20, None) == ALIGN
    assert L().qz_fp4a4_gemm(A, B, D, ts, 64, 64, 256, 1, Y, None, 0, None) == WS
    assert L().qz_fp4a4_gemm(A, B, D, ts, 64, 64, 256, 1, Y, MIS, 1 << 20, None) == ALIGN
    # activation codes, their scales (NVFP4-sized atoms) and one word for max |a|
    M, K = 2048, 8192
    assert qz.qz_workspace_bytes(qz.QZ_OP_FP4A4_GEMM, M, 8192, K, 0) == \
        M * K // 2 + (M // 128) * (K // 64) * 512 + 256
    assert qz.qz_workspace_bytes(qz.QZ_OP_FP4A4_GEMM, 37, 300, 512, 0) == \
        37 * 256 + 512 * 8 + 256       # 37 x 256 code bytes are already a multiple of 256
    assert qz.qz_fp4_mma_scale_bytes(300, 1024, qz.QZ_FP4_NV) == 3 * (1024 // 64) * 512
    assert qz.qz_fp4_mma_scale_bytes(300, 1024, qz.QZ_FP4_MX) == 3 * (1024 // 128) * 512
    assert L().qz_fp4_scales_to_mma(A, 300, 1000, 1, B, None) == UNSUP
    assert L().qz_fp4_scales_to_mma(None, 300, 1024, 1, B, None) == INVALID
    assert L().qz_fp4_scales_to_mma(A, 300, 1024, 1, MIS, None) == ALIGN
