"""Pins of the oracle's INT8 path (PAROAttention, arXiv 2506.16054, review
key_machinery and core_discovery: block-wise INT8 quantisation with groups
aligned to the attention block, for QK^T and for the post-softmax map P).

* exact codes on hand-built blocks (round-half-to-even, clamp at +-127,
  zero blocks, float32 scale arithmetic);
* special case: integer inputs with absmax 127 quantise to themselves with
  scale 1, so with P unrounded the INT8 attention equals the float64
  attention of the same values;
* analytic bound on the effect of rounding P;
* online and row-max modes coincide when a row keeps a single block.

The default P reading, mode "tile" (the exactly normalised P quantised per
(query block, key block) tile with the tile's own absmax / 127), is pinned
by a hand-worked example (tests/golden/int8_tile_n4_b2.txt), a pure-Python
brute force on tiny inputs (loops, Python's half-even round()), a closed
form (equal scores: P = 1/n is exact on the grid, O = the mean of the
dequantised values), independence from the order of the kept list, the
whole-block / sampled-row agreement, and the rounding bound.
"""

import math
import os

import numpy as np

from oracle import paro_ref as ref


def test_codes_half_even_and_clamp():
    # absmax 127 -> inv = 1, scale = 1: codes are the rounded values
    blk = np.array([[127.0, 2.5, 3.5, -2.5], [-0.5, 0.5, 1.5, -127.0]], dtype=np.float32)
    xp = blk.reshape(1, 1, 2, 4)
    q, s = ref.quantize_int8(xp, 2, 2)
    assert q[0, 0].tolist() == [[127, 2, 4, -2], [0, 0, 2, -127]]
    assert s[0, 0, 0] == np.float32(1.0)


def test_scale_arithmetic_is_float32():
    x = np.array([[0.3, -0.1], [0.2, 0.05]], dtype=np.float32).reshape(1, 1, 2, 2)
    q, s = ref.quantize_int8(x, 2, 2)
    amax = np.float32(0.3)
    inv = np.float32(127.0) / amax
    assert s[0, 0, 0] == np.float32(amax / np.float32(127.0))
    want = np.clip(np.rint(x[0, 0] * inv), -127, 127)
    assert (q[0, 0] == want).all()
    # 0.3 * fl32(127/0.3) rounds to 127 exactly
    assert q[0, 0, 0, 0] == 127


def test_zero_block_and_pad_rows():
    x = np.zeros((1, 1, 8, 3), dtype=np.float32)
    x[0, 0, 4:6] = 1.0
    q, s = ref.quantize_int8(x, 6, 4)  # N = 6: block 1 has 2 real rows, 2 pad rows
    assert s[0, 0, 0] == 0 and (q[0, 0, :4] == 0).all()
    assert (q[0, 0, 4:6] == 127).all() and (q[0, 0, 6:] == 0).all()


def integer_inputs(rng, Np, d):
    x = rng.integers(-126, 127, size=(Np, d)).astype(np.float32)
    x[0, 0] = 127.0  # every block of 4 rows gets absmax 127 below
    return x


def test_integer_inputs_reduce_to_float_attention():
    rng = np.random.default_rng(3)
    block, nb, d = 4, 5, 8
    Np = N = block * nb
    xs = []
    for _ in range(3):
        x = rng.integers(-126, 127, size=(Np, d)).astype(np.float32)
        for i in range(nb):
            x[i * block, 0] = 127.0
        xs.append(x)
    # shrink the scores so that the softmax is not one-hot
    q8, sq = ref.quantize_int8(xs[0].reshape(1, 1, Np, d), N, block)
    k8, sk = ref.quantize_int8(xs[1].reshape(1, 1, Np, d), N, block)
    v8, sv = ref.quantize_int8(xs[2].reshape(1, 1, Np, d), N, block)
    assert (sq == 1).all() and (q8[0, 0] == xs[0]).all()
    idx = np.array([[0, 2, 3], [1, 2, 4], [0, 1, 2], [3, 4, 0], [4, 1, 2]], dtype=np.int32)
    idx = np.sort(idx, axis=1)
    # scale inputs by 2^-6 so that S / sqrt(d) stays moderate: use the
    # float path with the same integer values and scales 2^-6
    sq = sq * np.float32(2.0 ** -6)
    sk = sk * np.float32(2.0 ** -6)
    got = ref.attention_int8(q8[0, 0], k8[0, 0], v8[0, 0], sq[0, 0], sk[0, 0], sv[0, 0],
                             N, block, idx, quantize_p=False)
    want = ref.attention_permuted(xs[0].astype(np.float64) * 2.0 ** -6,
                                  xs[1].astype(np.float64) * 2.0 ** -6,
                                  xs[2].astype(np.float64), N, block, idx)
    assert np.abs(got - want).max() < 1e-10
    got_r = ref.attention_int8(q8[0, 0], k8[0, 0], v8[0, 0], sq[0, 0], sk[0, 0], sv[0, 0],
                               N, block, idx, mode="rowmax", quantize_p=False)
    assert np.abs(got_r - want).max() < 1e-10


def test_p_rounding_bound():
    rng = np.random.default_rng(8)
    block, nb, d = 8, 4, 16
    N = Np = block * nb
    x = rng.standard_normal((3, 1, 1, Np, d)).astype(np.float32)
    q8, sq = ref.quantize_int8(x[0] * 0.5, N, block)
    k8, sk = ref.quantize_int8(x[1] * 0.5, N, block)
    v8, sv = ref.quantize_int8(x[2], N, block)
    idx = np.tile(np.arange(nb, dtype=np.int32), (nb, 1))
    for mode in ("tile", "online", "rowmax"):
        exact = ref.attention_int8(q8[0, 0], k8[0, 0], v8[0, 0], sq[0, 0], sk[0, 0], sv[0, 0],
                                   N, block, idx, mode=mode, quantize_p=False)
        quant = ref.attention_int8(q8[0, 0], k8[0, 0], v8[0, 0], sq[0, 0], sk[0, 0], sv[0, 0],
                                   N, block, idx, mode=mode)
        # |dO_r| <= sum_c |dP_rc| |v_c| / l_r with |dP| <= 1/254 and l_r >= 1
        vabs = np.abs(v8[0, 0].astype(np.float64)) * np.repeat(sv[0, 0], block)[:, None]
        bound = vabs.sum(axis=0)[None, :] / 254.0
        assert (np.abs(quant - exact) <= bound + 1e-12).all()
        assert np.abs(quant - exact).max() > 0  # rounding did something


def test_single_block_modes_agree():
    rng = np.random.default_rng(2)
    block, nb, d = 8, 3, 8
    N = Np = block * nb
    x = rng.standard_normal((3, 1, 1, Np, d)).astype(np.float32)
    qs = [ref.quantize_int8(x[t], N, block) for t in range(3)]
    idx = np.arange(nb, dtype=np.int32)[:, None]
    a = ref.attention_int8(qs[0][0][0, 0], qs[1][0][0, 0], qs[2][0][0, 0], qs[0][1][0, 0],
                           qs[1][1][0, 0], qs[2][1][0, 0], N, block, idx, mode="online")
    b = ref.attention_int8(qs[0][0][0, 0], qs[1][0][0, 0], qs[2][0][0, 0], qs[0][1][0, 0],
                           qs[1][1][0, 0], qs[2][1][0, 0], N, block, idx, mode="rowmax")
    assert np.abs(a - b).max() < 1e-12


def test_int32_dot_is_exact_range():
    # the largest |Q8 . K8| over d = 128 fits float32's exact-integer range,
    # so converting the int32 accumulator to float32 loses nothing
    assert 127 * 127 * 128 < 2 ** 24
    assert math.isclose(127 * 127 * 128, 2064512)


def test_row_subset_matches_whole_head():
    """attention_int8_rows evaluates single rows with the same row-wise
    steps: the whole-head function's values (up to float64 summation order,
    which differs between a one-row and a block matrix product), ragged tail
    and a row with an empty kept list included."""
    rng = np.random.default_rng(12)
    block, nb, d = 8, 5, 16
    N = block * nb - 3
    Np = block * nb
    x = rng.standard_normal((3, 1, 1, Np, d)).astype(np.float32)
    x[:, :, :, N:] = 0
    qs = [ref.quantize_int8(x[t], N, block) for t in range(3)]
    idx = np.array([[0, 2, 4], [1, 3, 4], [0, 2, -1], [0, 1, 3], [2, 3, 4]], dtype=np.int32)
    counts = np.array([3, 3, 2, 0, 3], dtype=np.int32)
    args = (qs[0][0][0, 0], qs[1][0][0, 0], qs[2][0][0, 0], qs[0][1][0, 0], qs[1][1][0, 0],
            qs[2][1][0, 0], N, block, idx)
    for mode in ("online", "rowmax"):
        whole = ref.attention_int8(*args, counts=counts, mode=mode)
        pos = [0, 5, 17, 24, 31, 33, N - 1]
        rows = ref.attention_int8_rows(*args, pos, counts=counts, mode=mode)
        assert np.abs(rows - whole[pos]).max() < 1e-12
        assert (rows[3] == 0).all() and (rows[4] == 0).all()  # block 3: empty list


def test_int4_codes_hand_example():
    # absmax 7 -> inv = 1, scale = 1: the codes are the rounded values, |q| <= 7
    blk = np.array([[7.0, 2.5, 3.5, -2.5], [-0.5, 0.5, 1.5, -7.0]], dtype=np.float32)
    q, s = ref.quantize_int8(blk.reshape(1, 1, 2, 4), 2, 2, qmax=7)
    assert q[0, 0].tolist() == [[7, 2, 4, -2], [0, 0, 2, -7]]
    assert s[0, 0, 0] == np.float32(1.0)
    # a general block: float32 arithmetic with Q = 7
    x = np.array([[0.3, -0.1], [0.2, 0.05]], dtype=np.float32).reshape(1, 1, 2, 2)
    q, s = ref.quantize_int8(x, 2, 2, qmax=7)
    inv = np.float32(np.float32(7.0) / np.float32(0.3))
    assert s[0, 0, 0] == np.float32(np.float32(0.3) / np.float32(7.0))
    assert (q[0, 0] == np.clip(np.rint(x[0, 0] * inv), -7, 7)).all() and np.abs(q).max() == 7


def test_int4_pv_exact_when_representable_and_bounded_otherwise():
    rng = np.random.default_rng(17)
    block, nb, d = 4, 3, 8
    N = Np = block * nb
    idx = np.tile(np.arange(nb, dtype=np.int32), (nb, 1))
    # V with values on the 4-bit grid (absmax 7 per block) dequantises exactly;
    # with P rounding off the INT4-PV oracle equals the float attention
    xs = [rng.integers(-6, 7, size=(Np, d)).astype(np.float32) for _ in range(3)]
    for x in xs:
        for i in range(nb):
            x[i * block, 0] = 7.0
    q8, sq = ref.quantize_int8((xs[0] * 0.125).reshape(1, 1, Np, d), N, block)
    k8, sk = ref.quantize_int8((xs[1] * 0.125).reshape(1, 1, Np, d), N, block)
    v4, sv = ref.quantize_int8(xs[2].reshape(1, 1, Np, d), N, block, qmax=7)
    assert (sv == 1).all() and (v4[0, 0] == xs[2]).all() and np.abs(v4).max() == 7
    args = (q8[0, 0], k8[0, 0], v4[0, 0], sq[0, 0], sk[0, 0], sv[0, 0], N, block, idx)
    exact = ref.attention_int8(*args, quantize_p=False, p_levels=7)
    qd = q8[0, 0].astype(np.float64) * np.repeat(sq[0, 0], block)[:, None]
    kd = k8[0, 0].astype(np.float64) * np.repeat(sk[0, 0], block)[:, None]
    want = ref.attention_permuted(qd, kd, xs[2].astype(np.float64), N, block, idx)
    assert np.abs(exact - want).max() < 1e-10
    # 4-bit P: |dO_r| <= sum_c |dP_rc| |v_c| / l_r with |dP| <= 1/14, l_r >= 1
    quant = ref.attention_int8(*args, p_levels=7)
    bound = np.abs(xs[2].astype(np.float64)).sum(axis=0)[None, :] / 14.0
    assert (np.abs(quant - exact) <= bound + 1e-12).all()
    assert np.abs(quant - exact).max() > 0
    # the 4-bit P codes are coarser than the 8-bit ones on the same inputs
    p8 = ref.attention_int8(*args)
    assert np.abs(quant - exact).max() > np.abs(p8 - exact).max()


def _golden_int8(golden_dir):
    vals = {}
    with open(os.path.join(golden_dir, "int8_tile_n4_b2.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                key, *rest = line.split()
                vals[key] = rest
    return vals


def test_tile_mode_golden_hand_worked(golden_dir):
    g = _golden_int8(golden_dir)
    q8, k8, v8 = (np.array([int(x) for x in g[n]], dtype=np.int8)[:, None]
                  for n in ("q8", "k8", "v8"))
    one = np.ones(2, dtype=np.float32)
    idx = np.full((2, 2), -1, dtype=np.int32)
    counts = np.array([len(g["idx0"]), len(g["idx1"])], dtype=np.int32)
    idx[0, :counts[0]] = [int(x) for x in g["idx0"]]
    idx[1, :counts[1]] = [int(x) for x in g["idx1"]]
    want = np.array([float(x) for x in g["out"]])
    got = ref.attention_int8(q8, k8, v8, one, one, one, 4, 2, idx, counts)  # default: tile
    assert np.abs(got[:, 0] - want).max() < 1e-12
    # the online reading keeps a per-row fixed scale: row 1 comes out exact (2.5)
    onl = ref.attention_int8(q8, k8, v8, one, one, one, 4, 2, idx, counts, mode="online")
    assert abs(onl[1, 0] - 2.5) < 1e-12 and abs(got[1, 0] - 2.5) > 2e-3
    # rows evaluated alone still use their whole block's tile scales
    rows = ref.attention_int8_rows(q8, k8, v8, one, one, one, 4, 2, idx, [1, 3], counts)
    assert np.abs(rows[:, 0] - want[[1, 3]]).max() < 1e-12


def _brute_tile(q8, k8, v8, sq, sk, sv, N, block, idx, counts, levels):
    """Pure-Python loops: normalised softmax per row over its kept valid keys,
    then per tile absmax, codes by Python's round() (half to even)."""
    Np, d = len(q8), len(q8[0])
    out = [[0.0] * d for _ in range(Np)]
    for i in range(Np // block):
        rows = [r for r in range(i * block, (i + 1) * block) if r < N]
        kept = [int(j) for j in idx[i][:counts[i]]]
        keys = {j: [c for c in range(j * block, (j + 1) * block) if c < N] for j in kept}
        s = {}
        for r in rows:
            for j in kept:
                for c in keys[j]:
                    dot = sum(int(q8[r][t]) * int(k8[c][t]) for t in range(d))
                    s[r, c] = dot * float(sq[i]) * float(sk[j]) / math.sqrt(d)
        p = {}
        for r in rows:
            cs = [c for j in kept for c in keys[j]]
            if not cs:
                continue
            m = max(s[r, c] for c in cs)
            z = sum(math.exp(s[r, c] - m) for c in cs)
            for c in cs:
                p[r, c] = math.exp(s[r, c] - m) / z
        for j in kept:
            amax = max([p[r, c] for r in rows for c in keys[j]], default=0.0)
            if amax == 0.0:
                continue
            scale = amax / levels
            for r in rows:
                for c in keys[j]:
                    code = round(p[r, c] / scale)
                    for t in range(d):
                        out[r][t] += code * int(v8[c][t]) * scale * float(sv[j])
    return np.array(out)


def test_tile_mode_brute_force_loops():
    rng = np.random.default_rng(31)
    block, N, d = 4, 11, 3  # a ragged last block
    nb = -(-N // block)
    Np = nb * block
    x = rng.standard_normal((3, 1, 1, Np, d)).astype(np.float32)
    x[:, :, :, N:] = 0
    q8, sq = ref.quantize_int8(x[0] * 2, N, block)
    k8, sk = ref.quantize_int8(x[1] * 2, N, block)
    v8, sv = ref.quantize_int8(x[2], N, block)
    idx = np.array([[0, 2, -1], [0, 1, 2], [2, -1, -1]], dtype=np.int32)
    counts = np.array([2, 3, 1], dtype=np.int32)
    for levels in (127, 7):
        want = _brute_tile(q8[0, 0], k8[0, 0], v8[0, 0], sq[0, 0], sk[0, 0], sv[0, 0], N, block,
                           idx, counts, levels)
        got = ref.attention_int8(q8[0, 0], k8[0, 0], v8[0, 0], sq[0, 0], sk[0, 0], sv[0, 0], N,
                                 block, idx, counts, p_levels=levels)
        assert np.abs(got[:N] - want[:N]).max() < 1e-12
        assert (got[N:] == 0).all()


def test_tile_mode_equal_scores_closed_form():
    """All-zero key codes: every score is 0, P = 1/n on the n kept valid keys,
    every tile's codes are 127 and the result is the mean of the dequantised
    values of the kept keys, exactly."""
    rng = np.random.default_rng(4)
    block, N, d = 4, 14, 5
    nb = -(-N // block)
    Np = nb * block
    q8 = rng.integers(-127, 128, size=(Np, d)).astype(np.int8)
    k8 = np.zeros((Np, d), dtype=np.int8)
    v8 = rng.integers(-127, 128, size=(Np, d)).astype(np.int8)
    sq = np.full(nb, 0.5, np.float32)
    sk = np.full(nb, 0.25, np.float32)
    sv = rng.uniform(0.1, 1.0, nb).astype(np.float32)
    idx = np.array([[0, 3], [1, 3], [0, 2], [2, 3]], dtype=np.int32)
    got = ref.attention_int8(q8, k8, v8, sq, sk, sv, N, block, idx)
    vdeq = v8.astype(np.float64) * np.repeat(sv.astype(np.float64), block)[:, None]
    for i in range(nb):
        cols = [c for j in idx[i] for c in range(j * block, (j + 1) * block) if c < N]
        want = vdeq[cols].mean(axis=0)
        assert np.abs(got[i * block:min((i + 1) * block, N)] - want).max() < 1e-12


def test_tile_mode_does_not_depend_on_list_order():
    rng = np.random.default_rng(12)
    block, nb, d = 8, 5, 16
    N = Np = block * nb
    x = rng.standard_normal((3, 1, 1, Np, d)).astype(np.float32)
    q8, sq = ref.quantize_int8(x[0] * 3, N, block)
    k8, sk = ref.quantize_int8(x[1] * 3, N, block)
    v8, sv = ref.quantize_int8(x[2], N, block)
    idx = np.array([[0, 1, 3], [0, 1, 4], [1, 2, 3], [0, 3, 4], [2, 3, 4]], dtype=np.int32)
    a = ref.attention_int8(q8[0, 0], k8[0, 0], v8[0, 0], sq[0, 0], sk[0, 0], sv[0, 0], N, block,
                           idx)
    b = ref.attention_int8(q8[0, 0], k8[0, 0], v8[0, 0], sq[0, 0], sk[0, 0], sv[0, 0], N, block,
                           idx[:, ::-1].copy())
    assert np.abs(a - b).max() < 1e-13
    # the one-pass replay does depend on it once the running max moves
    c = ref.attention_int8(q8[0, 0], k8[0, 0], v8[0, 0], sq[0, 0], sk[0, 0], sv[0, 0], N, block,
                           idx, mode="online")
    d_ = ref.attention_int8(q8[0, 0], k8[0, 0], v8[0, 0], sq[0, 0], sk[0, 0], sv[0, 0], N, block,
                            idx[:, ::-1].copy(), mode="online")
    assert np.abs(c - d_).max() > 1e-6
    # sampled rows equal the whole-head evaluation
    pos = [0, 9, 17, 39]
    rows = ref.attention_int8_rows(q8[0, 0], k8[0, 0], v8[0, 0], sq[0, 0], sk[0, 0], sv[0, 0],
                                   N, block, idx, pos)
    assert np.abs(rows - a[pos]).max() < 1e-13
