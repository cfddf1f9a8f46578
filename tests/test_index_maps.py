"""CPU checks of the index arithmetic the kernels rely on, restated from the kernel sources:

* the butterfly sums of the backward kernel (csrc/backward.cuh, butterfly_sum): after the stages
  over the given lane bits, lane l holds the full sums of the values the kernel reads there;
* the thread tiles of the backward kernel (R x 4 per thread) and of the decode kernels (16 x CPL
  per thread, whole head or one of NSL column slices) cover their state slice exactly once;
* the persistent streaming decode (csrc/decode_stream.cuh) visits every head exactly once;
* the four-CTA prefill (csrc/chunk_tc4.cuh): its in-place write-vector conversion reads no
  16-byte group another thread writes, its state-pass thread map covers the CTA's 128 x 32 state
  slice and its output rows once, and its staging entries and slots stay inside their buffers.
"""
import itertools

import numpy as np
import pytest


def butterfly(x, hi, lo):
    """x: [32 lanes, N].  The stages of butterfly_sum over the lane bits hi, hi/2, ..., lo."""
    x = x.copy()
    n = x.shape[1]
    o, m = hi, n
    while o >= lo:
        y = x.copy()
        for lane in range(32):
            up = bool(lane & o)
            partner = lane ^ o
            for k in range(m // 2):
                sent_by_partner = x[partner, k] if (partner & o) else x[partner, k + m // 2]
                keep = x[lane, k + m // 2] if up else x[lane, k]
                y[lane, k] = keep + sent_by_partner
        x = y
        o >>= 1
        m >>= 1
    return x[:, :m]


def lanes_sharing(lane, bits):
    """Lanes that differ from `lane` only in the given bits (the ones a butterfly sums over)."""
    return [l for l in range(32) if (l & ~bits) == (lane & ~bits)]


def test_forward_step_column_sums():
    # 4 partial column sums per lane, summed over lane bits 16 and 8: column c0 + 2 b4 + b3
    rng = np.random.default_rng(0)
    x = rng.standard_normal((32, 4))
    z = butterfly(x, 16, 8)
    for lane in range(32):
        b3, b4 = (lane >> 3) & 1, (lane >> 4) & 1
        assert np.isclose(z[lane, 0], x[lanes_sharing(lane, 24), 2 * b4 + b3].sum())


def test_backward_step_column_sums():
    # 8 values (sum b4: 0 = X^T b, 1 = du) of columns c0 + 2 b3 + k
    rng = np.random.default_rng(1)
    x = rng.standard_normal((32, 8))
    z = butterfly(x, 16, 8)
    for lane in range(32):
        b3, b4 = (lane >> 3) & 1, (lane >> 4) & 1
        for k in range(2):
            assert np.isclose(z[lane, k], x[lanes_sharing(lane, 24), 4 * b4 + 2 * b3 + k].sum())


@pytest.mark.parametrize("nq", [16, 8])
def test_backward_step_row_sums(nq):
    # per-row sums over a row's 8 lanes (bits 4, 2, 1): lane cg holds values (nq/8) cg + k
    rng = np.random.default_rng(nq)
    x = rng.standard_normal((32, nq))
    z = butterfly(x, 4, 1)
    for lane in range(32):
        cg = lane & 7
        for k in range(nq // 8):
            assert np.isclose(z[lane, k], x[lanes_sharing(lane, 7), (nq // 8) * cg + k].sum())


@pytest.mark.parametrize("dk", [64, 128])
def test_backward_tiles_cover_the_slice_once(dk):
    nw, rpw = 8, dk // 8
    r_per = rpw // 4
    seen = np.zeros((dk, 32), dtype=int)
    for warp, lane in itertools.product(range(nw), range(32)):
        cg, rg = lane & 7, lane >> 3
        r0, c0 = rpw * warp + r_per * rg, 4 * cg
        for r, c in itertools.product(range(r_per), range(4)):
            seen[r0 + r, c0 + c] += 1
    assert (seen == 1).all()


@pytest.mark.parametrize("dk,dvf,nsl", [(128, 128, 1), (128, 128, 4), (128, 64, 1), (64, 128, 1), (64, 64, 1)])
def test_decode_tiles_cover_the_head_once(dk, dvf, nsl):
    dv = dvf // nsl
    cpl, rpw = dv // 32, dk // 8
    seen = np.zeros((dk, dvf), dtype=int)
    for block, warp, lane in itertools.product(range(nsl), range(8), range(32)):
        v0 = block * dv
        for rr, c in itertools.product(range(rpw), range(cpl)):
            seen[warp + rr * 8, v0 + lane * cpl + c] += 1
    assert (seen == 1).all()


@pytest.mark.parametrize("nheads,sms", [(8192, 148), (149, 148), (300, 148), (1000, 132)])
def test_streaming_decode_visits_every_head_once(nheads, sms):
    grid = min(nheads, 2 * sms)  # two persistent CTAs per SM
    visits = np.zeros(nheads, dtype=int)
    for cta in range(grid):
        for h in range(cta, nheads, grid):  # heads blockIdx.x, blockIdx.x + gridDim.x, ...
            visits[h] += 1
    assert (visits == 1).all()


def sw128_off16(r, c8, R):
    """Byte offset of the 16-byte group holding columns c8*8 .. c8*8+7 of row r (128-byte swizzle)."""
    blk, ch = c8 >> 3, (c8 & 7) ^ (r & 7)
    return blk * R * 128 + r * 128 + ch * 16


@pytest.mark.parametrize("rank", range(4))
def test_quad_write_vector_conversion_is_race_free(rank):
    """Thread ct (0..255) of the state pass reads 16-byte group vgrp + (ct & 3) of row ct >> 2 of the
    raw v box and writes group ct & 3 of the same row; vgrp = ((32 rank) & 63) / 8."""
    v0 = 32 * rank
    vgrp = (v0 & 63) >> 3
    reads, writes = {}, {}
    for ct in range(256):
        wc, wjb = ct >> 2, ct & 3
        reads[ct] = sw128_off16(wc, vgrp + wjb, 64)
        writes[ct] = sw128_off16(wc, wjb, 64)
    assert len(set(writes.values())) == 256  # every output group written once
    for ct, w in writes.items():
        readers = [t for t, r in reads.items() if r == w]
        assert readers in ([], [ct]), (ct, readers)  # no other thread reads what ct overwrites
    # the raw groups read are this CTA's 32 value columns of the 64-column box
    cols = {(vgrp + (ct & 3)) * 8 + i for ct in range(256) for i in range(8)}
    assert cols == set(range(v0 & 63, (v0 & 63) + 32))


def test_quad_state_pass_thread_map():
    """Chain thread ct: warp cw = ct >> 5, lane; TMEM lane quarter cw & 3 (rows 32 q + lane), column
    half cw >> 2 (16 columns).  E4 covers rows 0..127 x columns 0..31 once; E3 (quarters 0, 1)
    covers rows 0..63; the output store (quarters 2, 3) covers output rows 0..63 once."""
    e4, e3, out = [], [], []
    for ct in range(256):
        cw, lane = ct >> 5, ct & 31
        quarter, half = cw & 3, cw >> 2
        trow, hc = quarter * 32 + lane, half * 16
        e4 += [(trow, hc + i) for i in range(16)]
        if quarter < 2:
            e3 += [(trow, hc + i) for i in range(16)]
        else:
            out += [(trow - 64, hc + i) for i in range(16)]
    assert sorted(e4) == [(r, c) for r in range(128) for c in range(32)]
    assert sorted(e3) == [(r, c) for r in range(64) for c in range(32)]
    assert sorted(out) == [(r, c) for r in range(64) for c in range(32)]


def test_quad_layout_fits():
    """Shared memory: working area and two slots of 65 KiB, S and Wr tiles, gates; the factor block
    (66,048 bytes) fits a slot and a staging entry; bulk copies are 16-byte multiples."""
    blk_stride = 65 * 1024
    fac = 2 * 128 * 128 + 64 * 256 + 128 * 128 + 512
    assert fac == 66048 and fac <= blk_stride
    pieces = [32768, 32768, fac - 65536]
    assert sum(pieces) == fac and all(x % 16 == 0 for x in pieces)
    off_s = blk_stride + 2 * blk_stride
    off_end = off_s + 128 * 128 + 64 * 128 + 128 * 4 + 256 * 4
    assert off_s % 1024 == 0 and (off_s + 128 * 128) % 1024 == 0
    assert off_end + 1024 <= 232448
    # staging: entry r of head (b, h) at ((b H + h) 4 + r) 65 KiB from a 16-byte aligned base
    assert (4 * blk_stride) == 266240 and blk_stride % 16 == 0
