"""Host checks of two shared-memory / HBM layouts the GEMM epilogues rely on
(their formulas restated from csrc/grouped_parts.cuh and csrc/moe_internal.cuh):

* the warp exchange buffer: 16-byte word j of row i at i * 64 + 16 * (j ^ ((i >> 1) & 3)).
  Shared memory serves a 16-byte-per-thread access in phases of 8 threads, and
  a phase is free of bank conflicts when its 8 words fall in 8 different
  16-byte bank groups ((address / 16) mod 8).  Both access patterns must be:
  row-wise (thread i, word j of row i, j fixed per instruction) and
  column-wise (thread l, word l % 4 of row 8 t + l / 4, t fixed).
* the kept pre-activations: byte offset ((r / 32) * words + j) * 512 + (r % 32) * 16
  of word j of row r.  It must be a bijection onto whole 16-byte words, and one
  word of a warp's 32 consecutive rows (any first row) must cover at most two
  contiguous 512-byte runs.
"""
import itertools


def x_slot(i, j):
    return i * 64 + 16 * (j ^ ((i >> 1) & 3))


def hpre_offset(r, j, words):
    return ((r // 32) * words + j) * 512 + (r % 32) * 16


def _conflict_free(addrs):
    return len({(a // 16) % 8 for a in addrs}) == len(addrs)


def test_exchange_slots_fill_the_buffer_once():
    slots = {x_slot(i, j) for i in range(32) for j in range(4)}
    assert slots == set(range(0, 32 * 64, 16))


def test_exchange_row_wise_access_is_conflict_free():
    for j in range(4):
        for phase in range(4):
            lanes = range(8 * phase, 8 * phase + 8)
            assert _conflict_free([x_slot(i, j) for i in lanes])


def test_exchange_column_wise_access_is_conflict_free():
    for t in range(4):
        for phase in range(4):
            lanes = range(8 * phase, 8 * phase + 8)
            assert _conflict_free([x_slot(8 * t + l // 4, l % 4) for l in lanes])


def test_unswizzled_layout_would_conflict():
    # the same buffer without the XOR: rows 64 bytes apart put two rows' words
    # in one 128-byte line, so a row-wise phase of 8 threads hits 2 bank groups
    assert not _conflict_free([i * 64 + 16 * 0 for i in range(8)])


def test_pre_activation_layout_is_a_bijection():
    for rows, words in [(32, 4), (64, 6), (96, 2)]:
        offs = [hpre_offset(r, j, words) for r in range(rows) for j in range(words)]
        assert sorted(offs) == list(range(0, rows * words * 16, 16))


def test_pre_activation_warp_word_spans_at_most_two_runs():
    words = 8
    for r0, j in itertools.product(range(0, 96), range(words)):
        offs = sorted(hpre_offset(r0 + i, j, words) for i in range(32))
        runs = 1 + sum(1 for a, b in zip(offs, offs[1:]) if b != a + 16)
        assert runs <= 2
        if r0 % 32 == 0:
            assert runs == 1 and offs[0] % 512 == 0
