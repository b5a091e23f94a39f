"""The index arithmetic of the aligned-copy kernels (copy_in_kernel and copy_out_kernel in
tlg_gemm.cu), restated in Python on a flat byte memory and run on the CPU.

Per warp and piece it follows the kernels' steps: the (row, piece) walk without division, the
aligned 16-byte blocks each lane loads, the neighbour's block taken by shuffle, the byte window
rebuilt from the two, and the whole-block or element stores.  Over random shapes, element
sizes, base offsets and row strides it checks that the copy is exact, that every block loaded
from the caller's matrix holds at least one of its bytes (so stays inside its allocation),
that copy-in writes only the workspace rows (padding included) and that copy-out writes only
the caller's elements."""
import random

import numpy as np
import pytest

U, WARPS = 4, 8  # pieces in flight per warp (kCopyUnroll); warps per block (kCopyWarps)


def bytes_from(lo, hi, s):
    """Bytes [s, s + 16) of the concatenation lo:hi."""
    cat = lo + hi
    return cat[s:s + 16]


def piece_items(rows, pieces, nwarps):
    """Per warp step: the kCopyUnroll (row, piece, live) items, walked as PieceIter does."""
    for w in range(nwarps):
        r, g = divmod(w, pieces)
        dq, dr = divmod(nwarps, pieces)
        while r < rows:
            items = []
            for u in range(U):
                items.append((r, g, r < rows))
                g += dr; r += dq
                if g >= pieces:
                    g -= pieces; r += 1
            yield items


def emu_in(mem, src, src_ld, dst, dst_ld, rows, row_bytes, nblocks, valid_src, allowed_dst):
    pieces = (row_bytes + 511) // 512
    nwarps = nblocks * WARPS
    for items in piece_items(rows, pieces, nwarps):
        lo = []; nx = []
        for (r, g, ok) in items:
            l = [bytes(16)] * 32; n31 = bytes(16)
            if ok:
                sb = src + r * src_ld; se = sb + row_bytes
                for lane in range(32):
                    a = (sb & ~15) + g * 512 + 16 * lane
                    if a < se:
                        assert any(valid_src[a:a + 16]), ("load outside", a)
                        l[lane] = bytes(mem[a:a + 16])
                    if lane == 31 and (sb & 15) and a + 16 < se:
                        assert any(valid_src[a + 16:a + 32])
                        n31 = bytes(mem[a + 16:a + 32])
            lo.append(l); nx.append(n31)
        for u, (r, g, ok) in enumerate(items):
            if not ok:
                break
            sb = src + r * src_ld
            for lane in range(32):
                hi = lo[u][lane + 1] if lane < 31 else nx[u]
                b = g * 32 + lane
                if b * 16 < row_bytes:
                    addr = dst + r * dst_ld + 16 * b
                    assert addr % 16 == 0
                    assert all(allowed_dst[addr:addr + 16]), ("store outside", addr)
                    mem[addr:addr + 16] = bytes_from(lo[u][lane], hi, sb & 15)


def emu_out(mem, src, src_ld, dst, dst_ld, rows, row_bytes, esz, nblocks, valid_src, allowed_dst):
    src_blocks = (row_bytes + 15) // 16
    pieces = ((row_bytes + 29) // 16 + 31) // 32
    nwarps = nblocks * WARPS
    for items in piece_items(rows, pieces, nwarps):
        cur = []; p0 = []
        for (r, g, ok) in items:
            c = [bytes(16)] * 32; q = bytes(16)
            if ok:
                srow = src + r * src_ld
                db = dst + r * dst_ld
                for lane in range(32):
                    b = g * 32 + lane
                    if b < src_blocks:
                        assert all(valid_src[srow + 16 * b: srow + 16 * b + 16]), "load outside"
                        c[lane] = bytes(mem[srow + 16 * b: srow + 16 * b + 16])
                    if lane == 0 and (db & 15) and b >= 1 and b - 1 < src_blocks:
                        q = bytes(mem[srow + 16 * (b - 1): srow + 16 * b])
            cur.append(c); p0.append(q)
        for u, (r, g, ok) in enumerate(items):
            if not ok:
                break
            db = dst + r * dst_ld; de = db + row_bytes; t = db & 15
            for lane in range(32):
                prev = cur[u][lane - 1] if lane > 0 else p0[u]
                out = cur[u][lane] if t == 0 else bytes_from(prev, cur[u][lane], 16 - t)
                b = g * 32 + lane
                a = (db & ~15) + 16 * b
                if a >= db and a + 16 <= de:
                    assert all(allowed_dst[a:a + 16]), "store outside"
                    mem[a:a + 16] = out
                elif a < de and a + 16 > db:
                    for k in range(16 // esz):
                        e = a + k * esz
                        if e < db or e >= de:
                            continue
                        assert all(allowed_dst[e:e + esz]), "elem store outside"
                        mem[e:e + esz] = out[k * esz:(k + 1) * esz]


def round_up(x, a):
    return (x + a - 1) // a * a


def case(rows, cols, esz, src_off, src_pad, nblocks, seed):
    """A caller matrix at an element offset with a padded stride, copied into a workspace
    layout and back out of one."""
    rnd = random.Random(seed)
    row_bytes = cols * esz
    # caller's matrix: element aligned, arbitrary base offset and stride
    c_ld = (cols + src_pad) * esz
    c_base = 4096 + src_off * esz
    c_end = c_base + (rows - 1) * c_ld + row_bytes
    w_ld = round_up(row_bytes, 16)
    w_base = round_up(c_end + 4096, 256)
    w_size = round_up(rows * w_ld, 256)
    size = w_base + w_size + 4096
    mem = bytearray(rnd.getrandbits(8) for _ in range(size))
    valid_c = np.zeros(size, bool)
    for r in range(rows):
        valid_c[c_base + r * c_ld: c_base + r * c_ld + row_bytes] = True
    valid_w = np.zeros(size, bool)
    valid_w[w_base:w_base + w_size] = True
    orig = bytes(mem)
    # copy in: caller -> workspace
    emu_in(mem, c_base, c_ld, w_base, w_ld, rows, row_bytes, nblocks, valid_c, valid_w)
    for r in range(rows):
        assert mem[w_base + r * w_ld: w_base + r * w_ld + row_bytes] == orig[c_base + r * c_ld: c_base + r * c_ld + row_bytes], ("in mismatch", r)
    # caller's bytes untouched
    assert all(mem[i] == orig[i] for i in range(0, w_base))
    # copy out: workspace -> a fresh caller matrix region (same layout as the source)
    mem2 = bytearray(orig)
    ws_vals = bytes(rnd.getrandbits(8) for _ in range(w_size))
    mem2[w_base:w_base + w_size] = ws_vals
    before = bytes(mem2)
    emu_out(mem2, w_base, w_ld, c_base, c_ld, rows, row_bytes, esz, nblocks, valid_w, valid_c)
    for r in range(rows):
        exp = ws_vals[r * w_ld: r * w_ld + row_bytes]
        assert mem2[c_base + r * c_ld: c_base + r * c_ld + row_bytes] == exp, ("out mismatch", r)
    changed = np.frombuffer(bytes(mem2), np.uint8) != np.frombuffer(before, np.uint8)
    assert not (changed & ~valid_c).any(), "out wrote outside the caller's matrix"



@pytest.mark.parametrize("seed", range(0, 400, 50))
def test_copy_kernels_index_arithmetic(seed):
    for s in range(seed, seed + 50):
        rnd = random.Random(s)
        esz = rnd.choice([2, 4])
        rows = rnd.choice([1, 2, 3, 5, 17, 33])
        cols = rnd.choice([1, 2, 3, 7, 8, 9, 63, 64, 65, 255, 256, 257, 300, 520, 1000])
        case(rows, cols, esz, rnd.randrange(0, 8), rnd.randrange(0, 9), rnd.choice([1, 2, 3, 7]), s)
