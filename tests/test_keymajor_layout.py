"""Index arithmetic of the key-major dK kernel's stages, checked on the CPU.

sparse_lightning_indexer_b200/csrc/slikl_dk_keymajor.cu packs G = 64 / N1P query rows of a
run into one stage when N1P < 64, so a stage's contraction is KD = G x N1P wide (64, or 128
with 128 heads): row g's heads are contraction indices g*N1P .. g*N1P + N1P - 1. Two builder
threads per key each write half of the key's K-major dS row in 16-byte chunks of 8
contraction indices, reading the mask bits of their heads from the row's record. The MMA of a
stage with n rows present issues n*N1P/16 steps of 16 contraction indices.

The formulas below restate the kernel's (kPer, kRowsPer, kChRow, the chunk -> row / head /
mask-word mapping, the swizzled store offset and the descriptor offsets). The checks: every
chunk the MMA reads is written exactly once per key, by the thread whose record and mask word
hold those heads; the stores stay inside the dS tile and the descriptors inside their
buffers; q boxes land 1024-byte aligned (the 128-byte swizzle atom), as the MMA descriptors
assume.
"""

import pytest

DS_TILE = 256 * 128                      # one 64-wide column block of the dS tile, bytes


def shape(n1p):
    g = 64 // n1p if n1p < 64 else 1
    kd = g * n1p
    k_per = kd // 16                      # chunks per builder thread
    span = 8 * k_per
    rows_per = span // n1p if span >= n1p else 1
    ch_row = k_per // rows_per
    rec_bytes = 32 if n1p > 64 else 16   # largest record of the instance
    return dict(G=g, KD=kd, kPer=k_per, kRowsPer=rows_per, kChRow=ch_row, RB=rec_bytes)


def builder_chunks(n1p, half, n_rows, rows_per=None):
    """(chunk, row g, first head, mask word, first bit) of one builder thread, rows < n.
    rows_per overrides kRowsPer (a planted mistake)."""
    s = shape(n1p)
    c0 = half * s["kPer"]
    g0, hb = (8 * c0) // n1p, (8 * c0) % n1p
    out = []
    for rr in range(s["kRowsPer"] if rows_per is None else rows_per):
        g = g0 + rr
        if g >= n_rows:
            continue
        for j in range(s["kChRow"]):
            c = c0 + rr * s["kChRow"] + j
            word = hb // 32 + (0 if j < 4 else 1)
            out.append((c, g, hb + 8 * j, word, (j & 3) * 8))
    return out


def check_builders(n1p, **kw):
    s = shape(n1p)
    assert s["kChRow"] <= 8                          # at most two mask words per thread
    for n in range(1, s["G"] + 1):
        for e in (0, 1, 5, 127, 255):                # key of the pair
            written = {}
            for half in (0, 1):
                for c, g, h0, word, bit0 in builder_chunks(n1p, half, n, **kw):
                    for h in range(8):
                        # contraction index 8c + h is head h0 + h of row g
                        assert 8 * c + h == g * n1p + h0 + h
                        head = h0 + h
                        assert head < n1p
                        assert head // 32 == word and head % 32 == bit0 + h
                    # the mask word read lies in the record's mask words, before its dI
                    assert 4 * (word + 1) <= 4 * max(1, n1p // 32)
                    off = (c >> 3) * DS_TILE + e * 128 + ((((c & 7) ^ e) & 7) << 4)
                    assert 0 <= off and off + 16 <= (2 if n1p > 64 else 1) * DS_TILE
                    assert c not in written, "chunk written twice"
                    written[c] = g
            steps = n * (n1p // 16)
            read = {c for ks in range(steps) for c in (2 * ks, 2 * ks + 1)}
            assert read <= set(written), f"unwritten chunks {sorted(read - set(written))}"
            assert all(c < s["KD"] // 8 for c in written)


@pytest.mark.parametrize("n1p", [16, 32, 64, 128])
def test_builder_chunks_cover_the_mma_reads(n1p):
    check_builders(n1p)


def test_planted_mistake_is_caught():
    """Builders that take one query row each at 16 heads leave rows 1 and 3 unwritten."""
    with pytest.raises(AssertionError):
        check_builders(16, rows_per=1)


@pytest.mark.parametrize("n1p", [16, 32, 64, 128])
def test_stage_buffers_and_descriptors(n1p):
    s = shape(n1p)
    kd = s["KD"]
    # q slot: two column blocks of KD rows x 128 B; row g's box at g*N1P*128
    for g in range(s["G"]):
        assert (g * n1p * 128) % 1024 == 0
        assert g * n1p * 128 + n1p * 128 <= kd * 128
    for ks in range(kd // 16):
        assert ks * 2048 + 16 * 128 <= kd * 128                    # A: 16 q rows per step
        b = (ks >> 2) * DS_TILE + (ks & 3) * 32                      # B: 32 bytes of each dS row
        assert b + 32 <= (2 if n1p > 64 else 1) * DS_TILE
    # record slot: G rows of 256 records, each bulk copy 16-byte aligned
    for g in range(s["G"]):
        assert (g * 256 * s["RB"]) % 16 == 0
