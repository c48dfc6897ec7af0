"""The fused run's lane map (host side, no GPU).

The kernel derives each lane's quad from its warp and lane index in closed
form.  Here that map, read through tdm_fused_lane_map (the same function the
kernel runs), is compared with the plain enumeration of the ordering it
implements: all pairs of overlap quads in (seam, row, column quad) order, 16
per warp with the partner 16 lanes up, the remaining lanes of the last pair
warp filled two at a time with singles, then the singles 32 per warp, every
single in (tile, row, column quad) order.  The projection of ParaChromo §4.3.2
averages entry (s+i, s+j) of tile k with (i, j) of tile k+1, so a pair must
hold exactly those two quads.
"""
import numpy as np
import pytest

tdm = pytest.importorskip("tiled_distance_maps_b200")


def enumerate_plan(T, overlap):
    s = 64 - overlap
    sq, oq = s // 4, overlap // 4

    def desc(k, r, q, paired):
        return q | r << 4 | k << 10 | (0x80000000 if paired else 0)

    pairs, singles = [], []
    for k in range(T):
        for r in range(64):
            for q in range(16):
                if 4 * q + 3 < r:
                    continue
                right = k < T - 1 and r >= s and q >= sq
                left = k > 0 and r < overlap and q < oq
                if right:
                    pairs.append((desc(k, r, q, True), desc(k + 1, r - s, q - sq, True)))
                elif not left:
                    singles.append(desc(k, r, q, False))
    plan, si = [], 0
    for p0 in range(0, len(pairs), 16):
        wl = [0] * 32
        for lane in range(16):
            if p0 + lane < len(pairs):
                wl[lane], wl[lane + 16] = pairs[p0 + lane]
            else:
                wl[lane], wl[lane + 16] = singles[si], singles[si + 1]
                si += 2
        plan += wl
    plan += singles[si:]
    return np.array(plan, dtype=np.uint32).reshape(-1, 32)


@pytest.mark.parametrize("overlap", [4, 8, 12, 16, 20, 24, 28, 32])
@pytest.mark.parametrize("T", [1, 2, 3, 5, 32, 33])
def test_closed_form_equals_the_enumeration(T, overlap):
    got = tdm.fused_lane_map(T, overlap)
    want = enumerate_plan(T, overlap if T > 1 else 0)
    assert got.shape == want.shape == (17 * T, 32)
    np.testing.assert_array_equal(got, want)


@pytest.mark.parametrize("T,overlap", [(1, 12), (4, 12), (7, 32), (100, 4)])
def test_every_quad_once_and_pairs_join_the_overlap(T, overlap):
    m = tdm.fused_lane_map(T, overlap).astype(np.int64)
    q, r, k, paired = m & 15, (m >> 4) & 63, (m >> 10) & 0xFFFF, (m >> 31) & 1
    keys = (k * 64 + r) * 16 + q
    upper = [(kk * 64 + rr) * 16 + qq for kk in range(T) for rr in range(64) for qq in range(16)
             if 4 * qq + 3 >= rr]
    assert np.array_equal(np.sort(keys.ravel()), np.array(upper))
    s = 64 - overlap
    for w in range(m.shape[0]):
        for lane in range(16):
            if paired[w, lane]:
                assert paired[w, lane + 16]
                assert k[w, lane + 16] == k[w, lane] + 1
                assert (r[w, lane] - s, q[w, lane] - s // 4) == (r[w, lane + 16], q[w, lane + 16])
                assert r[w, lane] >= s and 4 * q[w, lane] >= s


def test_bad_arguments_are_rejected():
    for T, o in ((0, 12), (3, 6), (3, 0), (3, 36)):
        with pytest.raises(tdm.TdmError):
            tdm.fused_lane_map(T, o)
